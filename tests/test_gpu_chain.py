"""Chain verification on the GPU against the oracle (parity), through the C
ABI. Acceptance rule: accepted counts and tokens bit-exact except at
decisions with fp64 oracle margin < 1e-6 (counted, share < 1e-4);
probabilities within 1e-5 relative."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import run_chain_gpu, run_chain_oracle
from tests.parity import Tally, compare_check, compare_probs

pytestmark = pytest.mark.gpu


def _compare(prob, tag, tally, seqs=None, split=False):
    acc, out, diag, st = run_chain_gpu(prob, split=split)
    assert st == 0, f"{tag}: device status {st}"
    ref = run_chain_oracle(prob, seqs)
    K = prob.draft_tok.shape[1]
    for b, r in ref.items():
        a = int(acc[b])
        toks = [int(x) for x in out[b, :a + 1]]
        assert all(int(x) == -1 for x in out[b, a + 1:]), f"{tag}: padding"
        same = compare_check(f"{tag}/seq{b}", r, a, toks, tally)
        if same:
            compare_probs(f"{tag}/seq{b}", r, diag[b], K, float(prob.temperature[b]))
    return acc


def test_chain_small_hundred_rounds():
    """B=1, K=4, V=1024 fp32, T=1, seed 0, fresh logits each of 100 rounds."""
    tally = Tally()
    for r in range(100):
        _compare(W.chain_small(rnd=r), f"round{r}", tally, split=(r % 2 == 1))
    tally.check_share()


EDGE = [
    # B, K, V, dtype, temperature spec
    (3, 0, 1000, torch.float32, 1.0),          # no drafts: plain draw from p
    (2, 1, 1, torch.float32, 1.0),             # single-token vocabulary
    (2, 2, 7, torch.bfloat16, 0.9),            # row shorter than one vector
    (3, 4, 4096, torch.bfloat16, 0.6),         # the largest one-launch vocabulary
    (3, 4, 4096, torch.float32, 1.7),          # the same in fp32
    (4, 3, 4097, torch.bfloat16, 0.8),         # ragged: one bf16 tile + 1
    (4, 3, 8191, torch.float32, 1.3),          # ragged fp32 tiles, odd tail
    (5, 2, 12345, torch.bfloat16, "mixed"),    # greedy and sampled in a batch
    (2, 40, 3000, torch.bfloat16, 1.0),        # K > 32: two ballot groups
    (3, 5, 777, torch.bfloat16, 0.0),          # all greedy
    (6, 4, 50000, torch.bfloat16, 1e-3),       # near-greedy temperature
    (6, 4, 50000, torch.float32, 50.0),        # flat laws
    (3, 6, 70000, torch.float32, 0.7),         # many tiles, fp32
]


@pytest.mark.parametrize("split", [False, True], ids=["verify", "two_calls"])
@pytest.mark.parametrize("B,K,V,dtype,tspec", EDGE)
def test_chain_edge_cases(B, K, V, dtype, tspec, split):
    """spec_verify_chain (one launch at V <= SPEC_SMALL_V) and the two-call
    form (row statistics, then the check) on the same inputs."""
    if tspec == "mixed":
        T = torch.tensor([0.0, 0.5, 1.0, 0.0, 2.0])[:B]
    else:
        T = float(tspec)
    tally = Tally()
    for r in range(3):
        prob = W.chain_problem(B, K, V, dtype, seed=11 + V, rnd=r, target_std=2.0,
                               draft_noise=1.0, temperature=T, philox_seed=5)
        _compare(prob, f"B{B}K{K}V{V}r{r}", tally, split=split)
    tally.check_share()


@pytest.mark.parametrize("split", [False, True], ids=["verify", "two_calls"])
@pytest.mark.parametrize("V", [2000, 6000])
def test_chain_far_shift(V, split):
    """Temperature 2e-6 on logits of spread 60: the row maxima times 1/(T ln 2)
    lie far above 2^26, where both paths form the exponentials relative to
    the row maximum (V=2000 takes the one-launch path, V=6000 the row
    statistics launch)."""
    tally = Tally()
    for r in range(3):
        prob = W.chain_problem(3, 3, V, torch.float32, seed=21, rnd=r, target_std=60.0,
                               draft_noise=1.0, temperature=2e-6, philox_seed=9)
        assert float(prob.tgt.max()) / (2e-6 * 0.6931471805599453) > 2.0 ** 26
        _compare(prob, f"far/V{V}/r{r}", tally, split=split)
    tally.check_share()


def test_chain_equal_laws_accept_all():
    prob = W.chain_problem(8, 6, 5000, torch.bfloat16, seed=3, temperature=0.9)
    prob.drf = prob.tgt[:, :6].clone()
    acc, out, diag, st = run_chain_gpu(prob)
    assert st == 0 and np.all(acc == 6)
    tally = Tally()
    _compare(prob, "equal", tally)


@pytest.mark.parametrize("split", [False, True], ids=["verify", "two_calls"])
def test_chain_masked_tokens_never_drawn(split):
    prob = W.chain_problem(6, 3, 2048, torch.float32, seed=4, temperature=1.0)
    prob.tgt[:, :, 100:1900] = float("-inf")
    prob.drf[:, :, 100:1000] = float("-inf")
    prob.draft_tok = W.gumbel_drafts(prob.drf, prob.temperature, W.generator(9, "cpu"))
    tally = Tally()
    for r in range(5):
        prob.rnd = r
        acc, out, _, st = run_chain_gpu(prob, split=split)
        assert st == 0
        for b in range(6):
            y = int(out[b, acc[b]])
            assert not (100 <= y < 1900)
        _compare(prob, f"masked{r}", tally, split=split)


def test_chain_greedy_ties_smallest_id():
    B, K, V = 2, 2, 9000
    tgt = torch.zeros((B, K + 1, V))
    tgt[:, :, 4100] = 5.0
    tgt[:, :, 8000] = 5.0
    tgt[:, 2, 77] = 5.0
    prob = W.ChainProblem(tgt, tgt[:, :K].clone(), torch.tensor([[4100, 4100], [4100, 8000]],
                                                               dtype=torch.int32),
                          torch.zeros(B), torch.arange(B, dtype=torch.int32), 0, 0)
    acc, out, _, st = run_chain_gpu(prob)
    assert st == 0
    assert list(out[0]) == [4100, 4100, 77] and acc[0] == 2
    assert list(out[1]) == [4100, 4100, -1] and acc[1] == 1


@pytest.mark.parametrize("split", [False, True], ids=["verify", "two_calls"])
def test_chain_invalid_values_flag_only_their_sequence(split):
    prob = W.chain_problem(4, 3, 1000, torch.float32, seed=6, temperature=1.0)
    prob.draft_tok[1, 2] = 1000          # out of range
    prob.temperature[2] = -1.0           # invalid temperature
    acc, out, _, st = run_chain_gpu(prob, split=split)
    assert st == -6
    assert acc[1] == -1 and acc[2] == -1 and np.all(out[1] == -1) and np.all(out[2] == -1)
    ref = run_chain_oracle(prob, [0, 3])
    tally = Tally()
    for b in (0, 3):
        compare_check(f"seq{b}", ref[b], int(acc[b]), list(out[b, :acc[b] + 1]), tally)


def test_chain_unaligned_rows_rejected_on_host():
    """Rows that do not start on 16-byte boundaries are refused before any
    launch (the row statistics stage them with bulk copies)."""
    from speculative_decoding_verification_89_b200 import capi
    prob = W.chain_problem(2, 2, 1001, torch.bfloat16, seed=1)
    tgt, drf = prob.tgt.cuda(), prob.drf.cuda()   # row stride 2002 bytes
    ws = capi.workspace(2, 2, 1001, torch.bfloat16)
    acc = torch.empty(2, dtype=torch.int32, device="cuda")
    out = torch.empty((2, 3), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(capi.SpecError) as e:
        capi.spec_verify_chain(tgt, drf, prob.draft_tok.cuda(), prob.temperature.cuda(), 0,
                               prob.seq_id.cuda(), 0, acc, out, st, ws)
    assert e.value.code == capi.SPEC_EINVAL


def test_chain_padded_rows():
    B, K, V, ld = 3, 4, 3000, 3008
    base = W.chain_problem(B, K, ld, torch.bfloat16, seed=8, temperature=1.1)
    prob = W.chain_problem(B, K, ld, torch.bfloat16, seed=8, temperature=1.1)
    prob.tgt = base.tgt[:, :, :V]
    prob.drf = base.drf[:, :, :V]
    prob.draft_tok = torch.clamp(base.draft_tok, max=V - 1)
    tally = Tally()
    _compare(prob, "padded", tally)


def test_chain_batch_full_size():
    """B=64, K=8, V=128256 bf16, Zipf-prior targets: every sequence."""
    tally = Tally()
    for r in range(2):
        prob = W.chain_batch(device="cuda", rnd=r)
        _compare(prob, f"full{r}", tally)
    tally.check_share()


def test_acceptance_rate_matches_closed_form():
    """Empirical acceptance over Philox rounds within 5 sigma of the mean of
    1 - TV(p_j, q_j) (drafts drawn from q)."""
    from oracle.verify import softmax
    prob = W.chain_problem(64, 4, 4096, torch.float32, seed=12, temperature=1.0)
    p = [[softmax(prob.tgt[b, j].double().numpy(), 1.0) for j in range(4)] for b in range(64)]
    q = [[softmax(prob.drf[b, j].double().numpy(), 1.0) for j in range(4)] for b in range(64)]
    alpha = np.array([[1 - 0.5 * np.abs(p[b][j] - q[b][j]).sum() for j in range(4)]
                      for b in range(64)])
    gen = W.generator(99, "cpu")
    n, acc0 = 200, 0
    for r in range(n):
        prob.draft_tok = W.gumbel_drafts(prob.drf, prob.temperature, gen)
        prob.rnd = r
        acc, _, _, st = run_chain_gpu(prob, diag=False)
        assert st == 0
        acc0 += int((acc > 0).sum())          # position 0 accepted
    mean = alpha[:, 0].mean()
    N = n * 64
    sd = np.sqrt(np.mean(alpha[:, 0] * (1 - alpha[:, 0])) / N)
    assert abs(acc0 / N - mean) < 5 * sd


def test_device_philox_matches_oracle():
    from oracle.philox import uniforms
    from speculative_decoding_verification_89_b200 import capi
    n = 1 << 20
    g = np.random.default_rng(5)
    ctr = g.integers(0, 2**32, size=(n, 4), dtype=np.uint64)
    ctr[:16] = 0
    ctr[16:32] = 2**32 - 1
    seed = 0x0123456789ABCDEF
    t = torch.from_numpy(ctr.astype(np.uint32).view(np.int32)).cuda()
    out = torch.empty((n, 2), dtype=torch.float32, device="cuda")
    capi.spec_philox_uniforms(seed, t, out)
    u0, u1 = uniforms(seed, ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3])
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got[:, 0], u0) and np.array_equal(got[:, 1], u1)
