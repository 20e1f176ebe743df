"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point declared in include/spec_verify.h, sizes workspaces, names
status codes, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from speculative_decoding_verification_89_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spec_verify.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spec_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    path = build_mod.build()
    return ctypes.CDLL(path)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "spec_verify_chain" in names and "spec_commit_paged" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in spec_verify.h but not exported"


def test_binding_covers_the_header():
    from speculative_decoding_verification_89_b200 import capi
    assert set(_declared()) <= set(capi.EXPORTED)


def test_workspace_bytes(lib):
    f = lib.spec_workspace_bytes
    f.restype = ctypes.c_size_t
    n = f(64, 8, 128256, 1, 0)
    tiles = (128256 + 4095) // 4096
    assert n >= 64 * 17 * tiles * 16 and n % 256 == 0
    assert f(256, 2, 151936, 0, 4) > f(256, 2, 151936, 0, 0)   # S = 7 > 2K+1 = 5
    assert f(1, 300, 1024, 0, 0) == 0          # K above the limit
    assert f(1, 4, 0, 0, 0) == 0               # empty vocabulary
    assert f(1, 4, 10, 7, 0) == 0              # unknown dtype


def test_status_strings(lib):
    f = lib.spec_status_string
    f.restype = ctypes.c_char_p
    for code in range(0, -7, -1):
        assert f(code) and f(code) != b"unknown status"
    assert f(-99) == b"unknown status"


def test_host_argument_errors_launch_nothing(lib):
    P = ctypes.c_void_p
    f = lib.spec_verify_chain
    f.restype = ctypes.c_int
    f.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, P, P, ctypes.c_uint64, P, ctypes.c_uint32,
                  P, P, P, P, P, ctypes.c_size_t, P]
    fake = P(0x10000)          # never dereferenced: checks fail first
    odd = P(0x10008)           # not 16-byte aligned
    base = [fake, 1024, fake, 1024, 0, 4, 3, 1024, fake, fake, 0, fake, 0, fake, fake,
            None, None, fake, 1 << 30, None]
    assert f(*base[:5], 0, *base[6:]) == 0           # B = 0: nothing to do
    bad = list(base); bad[0] = None
    assert f(*bad) == -1                            # null logits
    bad = list(base); bad[0] = odd
    assert f(*bad) == -1                            # misaligned rows
    bad = list(base); bad[1] = 1000
    assert f(*bad) == -1                            # stride below V
    bad = list(base); bad[1] = 1026
    assert f(*bad) == -1                            # row stride not 16-byte multiple
    bad = list(base); bad[4] = 5
    assert f(*bad) == -1                            # dtype
    bad = list(base); bad[6] = 300
    assert f(*bad) == -1                            # K too large
    bad = list(base); bad[17] = None
    assert f(*bad) == -3                            # no workspace
    bad = list(base); bad[18] = 16
    assert f(*bad) == -3                            # workspace too small
    bad = list(base); bad[13] = None
    assert f(*bad) == -1                            # no accept_len output


def test_commit_host_argument_errors(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    f = lib.spec_commit_paged
    f.restype = I
    f.argtypes = [I, I, I, P, P, P, P, I, P, P, I, I, P, P, I, I, I, P, P, P, I, P, P]
    fake = P(0x10000)
    args = [4, 16, 8, fake, fake, None, fake, 1, fake, fake, 64, 9, fake, fake, 32, 8, 128,
            None, None, None, 0, None, None]
    bad = list(args); bad[1] = 0
    assert f(*bad) == -1                  # block size
    bad = list(args); bad[13] = None
    assert f(*bad) == -1                  # stage without pool
    bad = list(args); bad[15] = 1; bad[16] = 3
    assert f(*bad) == -1                  # segment not a multiple of 16 bytes
    bad = list(args); bad[17] = fake; bad[18] = fake; bad[20] = 4096
    assert f(*bad) == -1                  # hidden rows without offsets
    bad = list(args); bad[3] = None
    assert f(*bad) == -1                  # no tables


def test_fused_host_argument_errors(lib):
    """spec_verify_chain_commit and spec_chain_decide_commit refuse bad chain
    or commit arguments before any launch (fake device pointers are never
    dereferenced)."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    fns = [lib.spec_verify_chain_commit, lib.spec_chain_decide_commit]
    for f in fns:
        f.restype = I
        f.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, I, I, I, I, P, P, ctypes.c_uint64,
                      P, ctypes.c_uint32, P, P, P, I, I, P, P, P, P, P, I, P, P, I, I, I, P, P,
                      P, I, P, P, ctypes.c_size_t, P]
    fake = P(0x10000)
    odd = P(0x10008)
    args = [fake, 1024, fake, 1024, 0, 4, 3, 1024, fake, fake, 0, fake, 0, fake, fake, None,
            16, 8, fake, fake, None, fake, fake, 64, fake, fake, 32, 8, 128, None, None, None, 0,
            fake, fake, 1 << 30, None]
    for f in fns:   # B = 0: nothing to do
        assert f(*[0 if i == 5 else a for i, a in enumerate(args)]) == 0
    cases = [
        (5, 4097, -1),          # B above the fused limit
        (6, 300, -1),           # K above the limit
        (16, 0, -1),            # block size
        (25, None, -1),         # K/V stage without a pool
        ((27, 28), (1, 3), -1),  # segment (2 * heads * dim bytes) not a multiple of 16
        (18, None, -1),         # no tables
        (13, None, -1),         # no accept_len (the commit's kept counts)
        (14, None, -1),         # no out_tok
        (4, 7, -1),             # unknown dtype
        (0, odd, -1),           # rows not 16-byte aligned
        (34, odd, -3),          # workspace misaligned
        (35, 64, -3),           # workspace too small
    ]
    for i, v, code in cases:
        bad = list(args)
        for j, x in zip(*((i, v) if isinstance(i, tuple) else ((i,), (v,)))):
            bad[j] = x
        for f in fns:
            assert f(*bad) == code, (i, v)


def test_draft_workspace_and_host_errors(lib):
    P = ctypes.c_void_p
    g = lib.spec_draft_workspace_bytes
    g.restype = ctypes.c_size_t
    n = g(64, 128256, 1)
    assert n % 256 == 0 and n >= 64 * 42 * (16 + 8)
    assert g(1, 0, 1) == 0 and g(1, 10, 9) == 0 and g(-1, 10, 0) == 0
    f = lib.spec_draft_sample
    f.restype = ctypes.c_int
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P,
                  ctypes.c_uint64, P, ctypes.c_uint32, P, P, P, P, P, P, ctypes.c_size_t, P]
    fake, odd = P(0x10000), P(0x10008)
    base = [fake, 1024, 1, 4, 1024, fake, 0, fake, 0, fake, fake, None, None, fake, fake,
            1 << 30, None]
    assert f(*base[:3], 0, *base[4:]) == 0          # B = 0: nothing to do
    for i, v, want in [(0, None, -1), (0, odd, -1), (1, 1000, -1), (2, 4, -1), (5, None, -1),
                       (7, None, -1), (9, None, -1), (10, None, -1), (14, None, -3),
                       (15, 64, -3)]:
        bad = list(base)
        bad[i] = v
        assert f(*bad) == want, (i, v)


def test_outcome_workspace_and_host_errors(lib):
    P = ctypes.c_void_p
    g = lib.spec_outcome_workspace_bytes
    g.restype = ctypes.c_size_t
    assert g(64, 8, 128256, 1, 32) > g(64, 8, 128256, 1, 0) > 0
    assert g(4, 2, 100, 0, 33) == 0 and g(4, 2, 100, 0, -1) == 0
    f = lib.spec_outcome_law
    f.restype = ctypes.c_int
    I, I64 = ctypes.c_int, ctypes.c_int64
    f.argtypes = [P, I64, P, I64, I, I, I, I, P, P, I, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    fake = P(0x10000)
    base = [fake, 1024, fake, 1024, 0, 4, 3, 1024, fake, fake, 8, fake, None, None, fake, fake,
            fake, fake, fake, 1 << 30, None]
    assert f(*base[:5], 0, *base[6:]) == 0          # B = 0
    for i, v, want in [(0, None, -1), (2, None, -1), (8, None, -1), (9, None, -1),
                       (10, 33, -1), (11, None, -1), (14, None, -1), (18, None, -3),
                       (19, 64, -3)]:
        bad = list(base)
        bad[i] = v
        assert f(*bad) == want, (i, v)


def test_saguaro_host_argument_errors(lib):
    """Bad sizes, dtype, list layout or eps are refused before any launch;
    eps = 0, empty lists and B = 0 return at once (the fake pointers are never
    read)."""
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f = lib.spec_saguaro_adjust
    f.restype = I
    f.argtypes = [P, I64, I, I, I, I, P, I, I, ctypes.c_double, P, P]
    fake = P(0x10000)
    base = [fake, 1024, 1, 4, 3, 1000, fake, 8, 0, 0.3, fake, None]
    assert f(*base[:9], 0.0, *base[10:]) == 0        # eps = 0
    assert f(*base[:7], 0, *base[8:]) == 0           # no cached ids
    assert f(*base[:3], 0, *base[4:]) == 0           # B = 0
    for i, v in [(1, 999), (2, 7), (3, -1), (4, -1), (5, 0), (7, 1025), (8, 2), (9, 1.0),
                 (9, -0.5), (9, float("nan")), (0, None), (6, None), (10, None)]:
        bad = list(base)
        bad[i] = v
        assert f(*bad) == -1, (i, v)


def test_vocab_parallel_workspace_and_host_errors(lib):
    """Shard outside the vocabulary, bad rank counts, missing buffers and a
    short workspace are refused on the host; B = 0 returns at once. Every
    call here must be refused before a launch: the pointers are fake."""
    P, I, I64, U32, U64, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                               ctypes.c_uint64, ctypes.c_size_t)
    g = lib.spec_vp_workspace_bytes
    g.restype = SZ
    g.argtypes = [I, I, I, I]
    full = g(64, 8, 16032, 1)
    assert full > g(64, 8, 8000, 1) > 0 and g(64, 300, 1000, 1) == 0 and g(4, 2, 100, 5) == 0
    f = lib.spec_vp_decide
    f.restype = I
    f.argtypes = [P, I64, P, I64, I, I, I, I, I, I, I, I, P, P, P, U64, P, U32, P, P, P, P, SZ, P]
    fake = P(0x10000)
    # tgt, ld, drf, ld, dtype, B, K, Vs, v0, V, R, rank, rows_all, drafts, T, seed, seq_id,
    # round, mass_out, diag, status, ws, ws_bytes, stream
    base = [fake, 1024, fake, 1024, 1, 4, 3, 1000, 1000, 2000, 2, 1, fake, fake, fake, 0, fake,
            0, fake, None, fake, fake, 1 << 30, None]
    assert f(*base[:5], 0, *base[6:]) == 0                 # B = 0
    for i, v, want in [(8, 1001, -1), (8, -1, -1), (9, 1999, -1), (10, 0, -1), (10, 65, -1),
                       (11, 2, -1), (11, -1, -1), (12, None, -1), (13, None, -1),
                       (16, None, -1), (18, None, -1), (0, None, -1), (1, 999, -1),
                       (22, 64, -3), (21, None, -3)]:
        bad = list(base)
        bad[i] = v
        assert f(*bad) == want, (i, v)
    s = lib.spec_vp_shard_stats
    s.restype = I
    s.argtypes = [P, I64, P, I64, I, I, I, I, I, I, P, P, P, P, P, SZ, P]
    sb = [fake, 1024, fake, 1024, 1, 4, 3, 1000, 1000, 2000, fake, fake, fake, fake, fake,
          1 << 30, None]
    for i, v, want in [(10, None, -1), (12, None, -1), (12, P(0x10004), -1), (8, 1001, -1)]:
        bad = list(sb)
        bad[i] = v
        assert s(*bad) == want, (i, v)
