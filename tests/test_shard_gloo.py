"""The sharded decode of one long sequence (long_context_compressed_b200/shard.py) on CPU:
two gloo ranks run decode_step with the oracle standing in for the library's kernels, and
both ranks' outputs equal the oracle's attention over the whole (unsharded) sequence.  This
checks the host logic -- shard ranges, the order and layout of the exchanges, the SWA rows
on rank 0 only -- without a GPU; the kernels themselves are checked in test_gpu_shard.py."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleKernels:
    """decode_step's three kernel phases computed by the CPU oracle (float64)."""

    def __init__(self, k, scale):
        self.k, self.scale = k, scale

    def local_topk(self, sh, qI, w):
        import oracle
        s = oracle.index_scores(qI.numpy(), w.numpy(), sh.kI.numpy(), sh.n_valid.numpy())
        loc = oracle.topk(s.astype(np.float32), sh.n_valid.numpy(), self.k)[:, 0]     # [B, k]
        sc = np.where(loc >= 0, np.take_along_axis(s[:, 0], np.maximum(loc, 0), -1), -np.inf).astype(np.float32)
        gi = np.where(loc >= 0, loc + sh.lo, -1).astype(np.int32)
        return torch.from_numpy(np.stack([sc.view(np.int32), gi], -1))             # (score bits, index)

    def attend(self, sh, q, all_pairs):
        import oracle
        G, B, k, _ = all_pairs.shape
        ap = all_pairs.numpy()
        cs = np.ascontiguousarray(ap[..., 0]).view(np.float32).transpose(1, 0, 2).reshape(B, 1, G * k)
        ci = ap[..., 1].transpose(1, 0, 2).reshape(B, 1, G * k)
        pos = oracle.topk(np.ascontiguousarray(cs), np.full((B, 1), G * k, np.int32), k)
        glob = np.where(pos >= 0, np.take_along_axis(ci, np.maximum(pos, 0), -1), -1)
        loc = np.where((glob >= sh.lo) & (glob < sh.hi), glob - sh.lo, -1).astype(np.int32)
        m, l, o = oracle.sparse_attn_partial(q.numpy(), sh.kv.numpy(), sh.swa.numpy(), sh.swa_pos0.numpy(),
                                             sh.q_pos.numpy(), loc, self.scale, with_swa=(sh.rank == 0))
        return torch.from_numpy(np.concatenate([o.reshape(-1), np.stack([m, l], -1).reshape(-1)]))

    def combine(self, sh, gathered, shape):
        import oracle
        B, T, H, D = shape
        n = B * T * H * D
        g = gathered.numpy()
        o = g[:, :n].reshape((-1,) + tuple(shape))
        ml = g[:, n:].reshape(-1, B, T, H, 2)
        return torch.from_numpy(oracle.attn_combine(ml[..., 0], ml[..., 1], o, sh.sink.numpy()))


def _inputs(B=2, N=900, H=8, D=64, W=140, seed=3):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g)
    pos = 4 * N - 1
    return {"q": r(B, 1, H, D), "qI": r(B, 1, 64, 128), "w": torch.rand(B, 1, 64, generator=g),
            "kI": r(B, N, 128), "kv": r(B, N, D), "swa": r(B, W, D), "sink": r(H),
            "swa_pos0": torch.full((B,), pos - W + 1, dtype=torch.int64),
            "q_pos": torch.full((B, 1), pos, dtype=torch.int64),
            "n_valid": torch.tensor([[N], [N - 77]], dtype=torch.int32)}


def _worker(rank, world, port, k, out):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from long_context_compressed_b200 import shard
    x = _inputs()
    N = x["kI"].shape[1]
    lo, hi = shard.shard_range(N, world, rank)
    sh = shard.Shard(rank=rank, world=world, lo=lo, hi=hi, kI=x["kI"][:, lo:hi].contiguous(),
                     kv=x["kv"][:, lo:hi].contiguous(), swa=x["swa"], swa_pos0=x["swa_pos0"], q_pos=x["q_pos"],
                     sink=x["sink"], n_valid=torch.clamp(x["n_valid"] - lo, 0, hi - lo).to(torch.int32))
    y = shard.decode_step(sh, OracleKernels(k, 1 / math.sqrt(x["q"].shape[-1])), shard.TorchDistExchange(),
                          x["q"], x["qI"], x["w"])
    out[rank] = y.numpy()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_equals_whole_sequence(world):
    import oracle
    k = 64
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), k, out), nprocs=world, join=True)
    x = _inputs()
    s = oracle.index_scores(x["qI"].numpy(), x["w"].numpy(), x["kI"].numpy(), x["n_valid"].numpy())
    idx = oracle.topk(s.astype(np.float32), x["n_valid"].numpy(), k)
    ref = oracle.sparse_attn(x["q"].numpy(), x["kv"].numpy(), x["swa"].numpy(), x["swa_pos0"].numpy(),
                             x["q_pos"].numpy(), x["sink"].numpy(), idx, 1 / math.sqrt(x["q"].shape[-1]))
    for r in range(world):
        np.testing.assert_allclose(out[r], ref, rtol=1e-10, atol=1e-12)


def test_shard_ranges_cover_the_entries():
    import sys
    sys.path.insert(0, ROOT)
    from long_context_compressed_b200 import shard
    for N in (1, 7, 262144, 1000003):
        for G in (1, 2, 3, 8):
            rs = [shard.shard_range(N, G, g) for g in range(G)]
            assert rs[0][0] == 0 and rs[-1][1] == N
            assert all(a[1] == b[0] for a, b in zip(rs[:-1], rs[1:]))
            assert max(h - l for l, h in rs) - min(h - l for l, h in rs) <= 1
