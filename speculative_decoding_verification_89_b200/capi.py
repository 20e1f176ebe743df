"""Thin ctypes binding of libspecverify (include/spec_verify.h).

Argument marshalling only: torch tensors are passed as device pointers and
strides, the current CUDA stream as the stream handle; every step of the
verification runs in the library's CUDA kernels. If the shared library is
missing this module raises on import: there is no other implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspecverify.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m speculative_decoding_verification_89_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

SPEC_OK, SPEC_EINVAL, SPEC_ECUDA, SPEC_EWORKSPACE = 0, -1, -2, -3
SPEC_ENOBLOCKS, SPEC_ETIMEOUT, SPEC_EDEVICE = -4, -5, -6
SPEC_F32, SPEC_BF16 = 0, 1

_p, _i, _i64, _u32, _u64, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                 ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t)

_SIGS = {
    "spec_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "spec_status_string": (ctypes.c_char_p, [_i]),
    "spec_verify_chain": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _u64, _p,
                               _u32, _p, _p, _p, _p, _p, _sz, _p]),
    "spec_chain_row_stats": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _p, _sz,
                                  _p]),
    "spec_chain_decide": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _u64, _p,
                               _u32, _p, _p, _p, _p, _p, _sz, _p]),
    "spec_verify_hier": (_i, [_p, _p, _p, _i64, _i, _i, _i, _i, _i, _p, _p, _u64, _p,
                              _u32, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "spec_commit_paged": (_i, [_i, _i, _i, _p, _p, _p, _p, _i, _p, _p, _i, _i, _p, _p,
                               _i, _i, _i, _p, _p, _p, _i, _p, _p]),
    "spec_verify_chain_commit": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _u64, _p,
                                      _u32, _p, _p, _p, _i, _i, _p, _p, _p, _p, _p, _i, _p,
                                      _p, _i, _i, _i, _p, _p, _p, _i, _p, _p, _sz, _p]),
    "spec_chain_decide_commit": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _u64, _p,
                                      _u32, _p, _p, _p, _i, _i, _p, _p, _p, _p, _p, _i, _p,
                                      _p, _i, _i, _i, _p, _p, _p, _i, _p, _p, _sz, _p]),
    "spec_verify_chain_persistent": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _u64,
                                          _p, _u32, _p, _p, _p, _p, _p, _sz, _p]),
    "spec_verify_chain_commit_persistent": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p,
                                                 _u64, _p, _u32, _p, _p, _p, _i, _i, _p, _p, _p,
                                                 _p, _p, _i, _p, _p, _i, _i, _i, _p, _p, _p, _i,
                                                 _p, _p, _sz, _p]),
    "spec_philox_uniforms": (_i, [_u64, _p, _i, _p, _p]),
    "spec_last_cuda_error": (ctypes.c_char_p, []),
    "spec_verify_chain_noalloc": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _u64, _p,
                                       _u32, _p, _p, _p, _p, _p]),
    "spec_saguaro_adjust": (_i, [_p, _i64, _i, _i, _i, _i, _p, _i, _i, ctypes.c_double, _p, _p]),
    "spec_vp_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "spec_vp_shard_stats": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p,
                                 _sz, _p]),
    "spec_vp_decide": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p,
                            _u64, _p, _u32, _p, _p, _p, _p, _sz, _p]),
    "spec_vp_pick": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p,
                          _p, _p, _p, _p, _sz, _p]),
    "spec_noalloc_test_fail_lookups": (_i, [_i]),
    "spec_test_set_wait_limit_ns": (_i, [_u64]),
    "spec_test_set_copy_wait_limit_ns": (_i, [_u64]),
    "spec_draft_workspace_bytes": (_sz, [_i, _i, _i]),
    "spec_outcome_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "spec_outcome_law": (_i, [_p, _i64, _p, _i64, _i, _i, _i, _i, _p, _p, _i, _p, _p, _p, _p,
                              _p, _p, _p, _p, _sz, _p]),
    "spec_draft_sample": (_i, [_p, _i64, _i, _i, _i, _p, _u64, _p, _u32, _p, _p, _p, _p, _p,
                               _p, _sz, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class SpecError(RuntimeError):
    def __init__(self, fn, code):
        msg = f"{fn}: {spec_status_string(code)} ({code})"
        if code == SPEC_ECUDA:
            msg += f": {_lib.spec_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SPEC_BF16
    if t.dtype == torch.float32:
        return SPEC_F32
    raise TypeError(f"logits must be float32 or bfloat16, got {t.dtype}")


def _rows(t, nrows_per_seq):
    """Row stride (elements) of a [B, n, V] logits tensor with unit element
    stride and evenly spaced rows."""
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("logits must be [B, n, V] with contiguous rows")
    B, n, V = t.shape
    ld = t.stride(1) if n > 1 else t.stride(0)
    if B > 1 and t.stride(0) != n * ld:
        raise ValueError("rows of all sequences must be evenly spaced")
    return ld


def _check(fn, rc):
    if rc != SPEC_OK:
        raise SpecError(fn, rc)


def spec_workspace_bytes(B, K, V, dtype, Ni=0):
    code = dtype if isinstance(dtype, int) else (SPEC_BF16 if dtype == torch.bfloat16 else SPEC_F32)
    return int(_lib.spec_workspace_bytes(B, K, V, code, Ni))


def spec_status_string(code):
    return _lib.spec_status_string(int(code)).decode()


def workspace(B, K, V, dtype, Ni=0, device="cuda"):
    """A zero-filled workspace tensor of the size a call needs (256-byte
    aligned by the allocator)."""
    n = spec_workspace_bytes(B, K, V, dtype, Ni)
    if n == 0:
        raise ValueError("invalid sizes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def spec_verify_chain(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, accept_len,
                      out_tok, dev_status, ws, diag=None, stream=None,
                      _entry="spec_verify_chain"):
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    rc = getattr(_lib, _entry)(
        _ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
        _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, V, _ptr(draft_tok),
        _ptr(temperature), seed, _ptr(seq_id), rnd, _ptr(accept_len), _ptr(out_tok),
        _ptr(diag), _ptr(dev_status), _ptr(ws), ws.numel(), _stream(stream))
    _check(_entry, rc)


def spec_verify_chain_persistent(*args, **kw):
    """spec_verify_chain on the persistent kernel (same arguments)."""
    spec_verify_chain(*args, _entry="spec_verify_chain_persistent", **kw)


def spec_verify_chain_noalloc(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, accept_len,
                              out_tok, dev_status, diag=None, stream=None):
    """spec_verify_chain for callers that cannot allocate: no workspace
    argument; the library's built-in scratch array is used instead (see
    include/spec_verify.h for its size and sharing rules)."""
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    rc = _lib.spec_verify_chain_noalloc(
        _ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
        _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, V, _ptr(draft_tok),
        _ptr(temperature), seed, _ptr(seq_id), rnd, _ptr(accept_len), _ptr(out_tok),
        _ptr(diag), _ptr(dev_status), _stream(stream))
    _check("spec_verify_chain_noalloc", rc)


def spec_chain_row_stats(tgt, drf, temperature, dev_status, ws, stream=None):
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    rc = _lib.spec_chain_row_stats(
        _ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
        _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, V, _ptr(temperature),
        _ptr(dev_status), _ptr(ws), ws.numel(), _stream(stream))
    _check("spec_chain_row_stats", rc)


def spec_chain_decide(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, accept_len,
                      out_tok, dev_status, ws, diag=None, stream=None):
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    rc = _lib.spec_chain_decide(
        _ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
        _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, V, _ptr(draft_tok),
        _ptr(temperature), seed, _ptr(seq_id), rnd, _ptr(accept_len), _ptr(out_tok),
        _ptr(diag), _ptr(dev_status), _ptr(ws), ws.numel(), _stream(stream))
    _check("spec_chain_decide", rc)


VP_ROW_BYTES, VP_MASS_BYTES, VP_MAX_RANKS = 32, 16, 64


def spec_vp_workspace_bytes(B, K, Vs, dtype):
    code = dtype if isinstance(dtype, int) else (SPEC_BF16 if dtype == torch.bfloat16 else SPEC_F32)
    return int(_lib.spec_vp_workspace_bytes(B, K, Vs, code))


def _vp_common(tgt, drf):
    B, Kp1, Vs = tgt.shape
    K = Kp1 - 1
    return (_ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
            _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, Vs)


def spec_vp_shard_stats(tgt, drf, v0, V, draft_tok, temperature, rows_out, dev_status, ws,
                        stream=None):
    """Shard records of the vocabulary-parallel check. tgt [B, K+1, Vs] and
    drf [B, K, Vs]: this rank's columns [v0, v0+Vs) of the rows; rows_out:
    uint8 [B, 2K+1, VP_ROW_BYTES]."""
    rc = _lib.spec_vp_shard_stats(*_vp_common(tgt, drf), v0, V, _ptr(draft_tok),
                                  _ptr(temperature), _ptr(rows_out), _ptr(dev_status), _ptr(ws),
                                  ws.numel(), _stream(stream))
    _check("spec_vp_shard_stats", rc)


def spec_vp_decide(tgt, drf, v0, V, R, rank, rows_all, draft_tok, temperature, seed, seq_id, rnd,
                   mass_out, dev_status, ws, diag=None, stream=None):
    """rows_all: uint8 [R, B, 2K+1, VP_ROW_BYTES] (every rank's records in rank
    order); mass_out: uint8 [B, VP_MASS_BYTES]."""
    rc = _lib.spec_vp_decide(*_vp_common(tgt, drf), v0, V, R, rank, _ptr(rows_all),
                             _ptr(draft_tok), _ptr(temperature), seed, _ptr(seq_id), rnd,
                             _ptr(mass_out), _ptr(diag), _ptr(dev_status), _ptr(ws), ws.numel(),
                             _stream(stream))
    _check("spec_vp_decide", rc)


def spec_vp_pick(tgt, drf, v0, V, R, rank, mass_all, draft_tok, temperature, accept_len, out_tok,
                 dev_status, ws, diag=None, stream=None):
    """mass_all: uint8 [R, B, VP_MASS_BYTES]; out_tok int32 [B, K+1] holds -1 at
    the drawn position unless this rank drew it (max-reduce over ranks)."""
    rc = _lib.spec_vp_pick(*_vp_common(tgt, drf), v0, V, R, rank, _ptr(mass_all),
                           _ptr(draft_tok), _ptr(temperature), _ptr(accept_len), _ptr(out_tok),
                           _ptr(diag), _ptr(dev_status), _ptr(ws), ws.numel(), _stream(stream))
    _check("spec_vp_pick", rc)


def spec_verify_hier(lg_d, lg_i, lg_f, Ni, draft_tok, temperature, seed, seq_id, rnd,
                     win_len, win_tok, win_stat, acc1, acc2, commit_tok, commit_n,
                     dev_status, ws, diag=None, stream=None):
    B, S, V = lg_f.shape
    K = draft_tok.shape[1]
    ld = _rows(lg_f, S)
    if _rows(lg_d, S) != ld or _rows(lg_i, S) != ld:
        raise ValueError("the three exits must share one row stride")
    rc = _lib.spec_verify_hier(
        _ptr(lg_d), _ptr(lg_i), _ptr(lg_f), ld, _dtype_code(lg_f), B, K, V, Ni,
        _ptr(draft_tok), _ptr(temperature), seed, _ptr(seq_id), rnd, _ptr(win_len),
        _ptr(win_tok), _ptr(win_stat), _ptr(acc1), _ptr(acc2), _ptr(commit_tok),
        _ptr(commit_n), _ptr(diag), _ptr(dev_status), _ptr(ws), ws.numel(),
        _stream(stream))
    _check("spec_verify_hier", rc)


def spec_commit_paged(block_tables, seq_lens, base_len, keep, keep_add, free_stack,
                      free_top, Kp1, dev_status, block_size=16, kv_stage=None,
                      kv_pool=None, hid_stage=None, hid_out=None, hid_off=None,
                      stream=None):
    B, max_blocks = block_tables.shape
    num_blocks = free_stack.numel()
    layers, kv_heads, head_dim, hidden = _kv_shapes(kv_stage, kv_pool, hid_stage, num_blocks,
                                                    block_size)
    rc = _lib.spec_commit_paged(
        B, block_size, max_blocks, _ptr(block_tables), _ptr(seq_lens), _ptr(base_len),
        _ptr(keep), keep_add, _ptr(free_stack), _ptr(free_top), num_blocks, Kp1,
        _ptr(kv_stage), _ptr(kv_pool), layers, kv_heads, head_dim, _ptr(hid_stage),
        _ptr(hid_out), _ptr(hid_off), hidden, _ptr(dev_status), _stream(stream))
    _check("spec_commit_paged", rc)


def _kv_shapes(kv_stage, kv_pool, hid_stage, num_blocks, block_size):
    layers = kv_heads = head_dim = hidden = 0
    if kv_stage is not None:
        # kv_stage [B, Kp1, layers, 2, heads, dim]; kv_pool [N, layers, 2, bs, heads, dim]
        layers, _, kv_heads, head_dim = kv_stage.shape[2:]
        if not (kv_stage.is_contiguous() and kv_pool.is_contiguous()):
            raise ValueError("KV buffers must be contiguous")
        if kv_pool.shape[0] != num_blocks or kv_pool.shape[3] != block_size:
            raise ValueError("pool shape does not match the block pool")
    if hid_stage is not None:
        hidden = hid_stage.shape[-1]
    return layers, kv_heads, head_dim, hidden


def spec_verify_chain_commit(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, accept_len,
                             out_tok, block_tables, seq_lens, base_len, free_stack, free_top,
                             dev_status, ws, block_size=16, kv_stage=None, kv_pool=None,
                             hid_stage=None, hid_out=None, hid_off=None, diag=None,
                             stream=None, _entry="spec_verify_chain_commit"):
    """spec_verify_chain, then spec_commit_paged with keep = accept_len,
    keep_add = 1, Kp1 = K + 1, as one call (three launches)."""
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    max_blocks = block_tables.shape[1]
    num_blocks = free_stack.numel()
    layers, kv_heads, head_dim, hidden = _kv_shapes(kv_stage, kv_pool, hid_stage, num_blocks,
                                                    block_size)
    rc = getattr(_lib, _entry)(
        _ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
        _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, V, _ptr(draft_tok),
        _ptr(temperature), seed, _ptr(seq_id), rnd, _ptr(accept_len), _ptr(out_tok),
        _ptr(diag), block_size, max_blocks, _ptr(block_tables), _ptr(seq_lens),
        _ptr(base_len), _ptr(free_stack), _ptr(free_top), num_blocks, _ptr(kv_stage),
        _ptr(kv_pool), layers, kv_heads, head_dim, _ptr(hid_stage), _ptr(hid_out),
        _ptr(hid_off), hidden, _ptr(dev_status), _ptr(ws), ws.numel(), _stream(stream))
    _check(_entry, rc)


def spec_chain_decide_commit(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, accept_len,
                             out_tok, block_tables, seq_lens, base_len, free_stack, free_top,
                             dev_status, ws, **kw):
    """The accept and draw-and-copy launches of spec_verify_chain_commit,
    after spec_chain_row_stats on the same workspace."""
    spec_verify_chain_commit(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, accept_len,
                             out_tok, block_tables, seq_lens, base_len, free_stack, free_top,
                             dev_status, ws, _entry="spec_chain_decide_commit", **kw)


def spec_verify_chain_commit_persistent(*args, **kw):
    """spec_verify_chain_commit on the persistent kernel (same arguments)."""
    spec_verify_chain_commit(*args, _entry="spec_verify_chain_commit_persistent", **kw)


def spec_saguaro_adjust(logits, cached, eps, temperature, stream=None):
    """Saguaro sampling: lower the cached tokens of the draft rows in place.
    logits: [B, n, V] (or [B, V]) float32/bfloat16 with contiguous, evenly
    spaced rows; cached: int32 on the device, [B, n_cached] (one list per
    sequence) or [B, n, n_cached] (one list per row); ids outside [0, V) pad;
    temperature: float [B]."""
    lg = logits if logits.dim() == 3 else logits.unsqueeze(1)
    B, n, V = lg.shape
    ld = lg.stride(1) if n > 1 else lg.stride(0)
    if lg.stride(2) != 1 or (B > 1 and lg.stride(0) != n * ld):
        raise ValueError("logits must be [B, n, V] with evenly spaced contiguous rows")
    per_row = 1 if cached.dim() == 3 else 0
    if cached.dtype != torch.int32 or not cached.is_contiguous() or cached.shape[0] != B or \
            (per_row and cached.shape[1] != n):
        raise ValueError("cached must be contiguous int32 [B, n_cached] or [B, n, n_cached]")
    rc = _lib.spec_saguaro_adjust(_ptr(lg), ld, _dtype_code(lg), B, n, V, _ptr(cached),
                                  cached.shape[-1], per_row, float(eps), _ptr(temperature),
                                  _stream(stream))
    _check("spec_saguaro_adjust", rc)


def spec_philox_uniforms(seed, ctr, out, stream=None):
    """ctr: uint32-valued int32 tensor [n, 4] on the device; out: float [n, 2]."""
    rc = _lib.spec_philox_uniforms(seed, _ptr(ctr), ctr.shape[0], _ptr(out), _stream(stream))
    _check("spec_philox_uniforms", rc)


def spec_draft_workspace_bytes(B, V, dtype):
    code = dtype if isinstance(dtype, int) else (SPEC_BF16 if dtype == torch.bfloat16 else SPEC_F32)
    return int(_lib.spec_draft_workspace_bytes(B, V, code))


def draft_workspace(B, V, dtype, device="cuda"):
    """A workspace tensor of the size a draft step needs."""
    n = spec_draft_workspace_bytes(B, V, dtype)
    if n == 0:
        raise ValueError("invalid sizes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def spec_draft_sample(logits, temperature, seed, seq_id, rnd, pos, out_tok, dev_status, ws,
                      logq=None, entropy=None, stream=None):
    """logits [B, V] (contiguous rows, evenly spaced); out_tok int32 [B];
    optional logq / entropy float64 [B]."""
    if logits.dim() != 2 or logits.stride(1) != 1:
        raise ValueError("logits must be [B, V] with contiguous rows")
    B, V = logits.shape
    rc = _lib.spec_draft_sample(_ptr(logits), logits.stride(0), _dtype_code(logits), B, V,
                                _ptr(temperature), seed, _ptr(seq_id), rnd, _ptr(pos),
                                _ptr(out_tok), _ptr(logq), _ptr(entropy), _ptr(dev_status),
                                _ptr(ws), ws.numel(), _stream(stream))
    _check("spec_draft_sample", rc)


def spec_outcome_workspace_bytes(B, K, V, dtype, n_top):
    code = dtype if isinstance(dtype, int) else (SPEC_BF16 if dtype == torch.bfloat16 else SPEC_F32)
    return int(_lib.spec_outcome_workspace_bytes(B, K, V, code, n_top))


def outcome_workspace(B, K, V, dtype, n_top, device="cuda"):
    n = spec_outcome_workspace_bytes(B, K, V, dtype, n_top)
    if n == 0:
        raise ValueError("invalid sizes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def spec_outcome_law(tgt, drf, draft_tok, temperature, n_top, p_len, dev_status, ws, beta=None,
                     mass=None, top_len=None, top_tok=None, top_prob=None, stream=None):
    """tgt [B, K+1, V], drf [B, K, V] as for spec_verify_chain; p_len float64
    [B, K+1]; top_* [B, n_top]."""
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    rc = _lib.spec_outcome_law(
        _ptr(tgt), _rows(tgt, Kp1), _ptr(drf) if K > 0 else None,
        _rows(drf, K) if K > 0 else 0, _dtype_code(tgt), B, K, V, _ptr(draft_tok),
        _ptr(temperature), n_top, _ptr(p_len), _ptr(beta), _ptr(mass), _ptr(top_len),
        _ptr(top_tok), _ptr(top_prob), _ptr(dev_status), _ptr(ws), ws.numel(), _stream(stream))
    _check("spec_outcome_law", rc)
