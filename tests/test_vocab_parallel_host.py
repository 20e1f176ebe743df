"""Host side of the vocabulary-parallel check, no GPU: the shard partition,
and the exchange between the three launches run by two gloo ranks on CPU.

The launches themselves need a GPU (tests/test_gpu_vocab_parallel.py); here a
stand-in shard object takes their place and writes rank-tagged bytes, so the
test sees whether each rank's decide step receives every rank's records in
rank order, whether the pick step receives every rank's masses, and whether
the max-reduction merges the drawn token into every rank's output."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shards_cover_the_vocabulary_in_whole_tiles():
    from speculative_decoding_verification_89_b200.vocab_parallel import vocab_shards
    for V in (1000, 4097, 32000, 128256, 151936, 262144):
        for R in (1, 2, 3, 4, 8):
            if -(-V // 256) < R:
                continue
            sh = vocab_shards(V, R)
            assert len(sh) == R
            assert sh[0][0] == 0 and sh[-1][0] + sh[-1][1] == V
            for (a, n), (b, _) in zip(sh, sh[1:]):
                assert a + n == b                     # contiguous, no overlap
            assert all(v0 % 256 == 0 and n > 0 for v0, n in sh)
            tiles = [-(-n // 256) for _, n in sh]
            assert max(tiles) - min(tiles) <= 1       # balanced in whole tiles
    assert vocab_shards(128256, 8)[0] == (0, 15872)
    assert vocab_shards(1000, 3) == [(0, 256), (256, 256), (512, 488)]
    with pytest.raises(ValueError):
        vocab_shards(300, 4)                          # 2 tiles cannot feed 4 ranks
    with pytest.raises(ValueError):
        vocab_shards(1000, 0)


class _StandIn:
    """The three launches replaced by byte writes tagged with the rank."""

    def __init__(self, B, K, R, rank):
        self.B, self.K, self.R, self.rank = B, K, R, rank
        per = 2 * K + 1
        self.rows = torch.zeros((B, per, 32), dtype=torch.uint8)
        self.rows_all = torch.zeros((R, B, per, 32), dtype=torch.uint8)
        self.mass = torch.zeros((B, 16), dtype=torch.uint8)
        self.mass_all = torch.zeros((R, B, 16), dtype=torch.uint8)
        self.seen = {}

    def stats(self, tgt, drf, draft_tok, temperature, status, stream=None):
        self.rows.fill_(10 + self.rank)
        self.rows[:, :, 0] = torch.arange(self.B, dtype=torch.uint8)[:, None]

    def decide(self, tgt, drf, draft_tok, temperature, seed, seq_id, rnd, status, diag=None,
               stream=None):
        self.seen["rows_all"] = self.rows_all.clone()
        self.mass.fill_(50 + self.rank)

    def pick(self, tgt, drf, draft_tok, temperature, accept_len, out_tok, status, diag=None,
             stream=None):
        self.seen["mass_all"] = self.mass_all.clone()
        accept_len.fill_(1)
        out_tok.fill_(-1)
        out_tok[:, 0] = draft_tok[:, 0]
        # sequence b's token at position 1 is drawn by rank b % R
        for b in range(self.B):
            if b % self.R == self.rank:
                out_tok[b, 1] = 1000 * (self.rank + 1) + b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from speculative_decoding_verification_89_b200.vocab_parallel import \
        verify_chain_vocab_parallel
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    B, K = 5, 3
    sh = _StandIn(B, K, world, rank)
    drafts = torch.arange(B * K, dtype=torch.int32).reshape(B, K)
    acc = torch.zeros(B, dtype=torch.int32)
    out = torch.zeros((B, K + 1), dtype=torch.int32)
    verify_chain_vocab_parallel(sh, None, None, drafts, None, 0, None, 0, acc, out, None)
    dist.barrier()
    dist.destroy_process_group()
    # numpy copies travel by value (shared tensors would die with this process)
    q.put((rank, sh.seen["rows_all"].numpy(), sh.seen["mass_all"].numpy(), acc.numpy(),
           out.numpy()))


def test_two_gloo_ranks_exchange_in_rank_order():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, K = 5, 3
    for rank, rows_all, mass_all, acc, out in res:
        for r in range(2):
            assert (rows_all[r, :, :, 1:] == 10 + r).all()
            assert list(rows_all[r, :, 0, 0]) == list(range(B))
            assert (mass_all[r] == 50 + r).all()
        assert (acc == 1).all()
        for b in range(B):
            assert out[b, 0] == b * K
            assert out[b, 1] == 1000 * (b % 2 + 1) + b   # the drawing rank's token won
            assert (out[b, 2:] == -1).all()
    assert (res[0][4] == res[1][4]).all()
