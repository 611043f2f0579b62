"""Sharded decode of one long sequence on the GPU.  The new calls against the oracle:
sparse_attn_partial (normalised output within the bf16 tolerance, log-sum-exp m + ln l),
csa_attn_combine (on partials the oracle made), csa_shard_select (bit-exact on gathered
lists the oracle made) and csa_shard_remap.  Then the whole step with G = 1, 2, 4 shards
emulated in one process (the exchanges become stacking on one GPU) against the oracle's
whole-sequence chain: exact scores -> top-k -> attention with the sink."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import shard, synth
from tolerances import bf16_round, check_attn_bf16, check_topk_sets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _np(t):
    return t.float().cpu().numpy()


def _attn_case(B=2, N=3000, H=128, D=512, W=130, k=300, seed=7):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    pos = 4 * N - 1
    return {"q": bf(B, 1, H, D), "kv": bf(B, N, D), "swa": bf(B, W, D), "sink": torch.randn(H, generator=g),
            "swa_pos0": torch.full((B,), pos - W + 1, dtype=torch.int64),
            "q_pos": torch.full((B, 1), pos, dtype=torch.int64),
            "idx": torch.stack([torch.randperm(N, generator=g)[:k].sort().values for _ in range(B)]).to(torch.int32).view(B, 1, k)}


@pytest.mark.parametrize("with_swa,k,H", [(True, 300, 128), (False, 300, 64), (False, 1, 64), (True, 0, 64)])
def test_sparse_attn_partial(csa, with_swa, k, H):
    x = _attn_case(k=max(k, 1), H=H)
    idx = x["idx"] if k > 0 else torch.full((2, 1, 1), -1, dtype=torch.int32)
    scale = 1 / math.sqrt(512)
    o, ml = csa.sparse_attn_partial(x["q"].cuda(), x["kv"].cuda(), x["swa"].cuda(), x["swa_pos0"].cuda(),
                                    x["q_pos"].cuda(), idx.cuda(), scale, with_swa=with_swa)
    m, l, ref = oracle.sparse_attn_partial(_np(x["q"]), _np(x["kv"]), _np(x["swa"]), x["swa_pos0"].numpy(),
                                           x["q_pos"].numpy(), idx.numpy(), scale, with_swa=with_swa)
    check_attn_bf16(_np(o), ref, what=f"partial swa={with_swa} k={k}")
    g = ml.cpu().numpy().astype(np.float64)
    empty = l == 0
    assert np.all(g[..., 1][empty] == 0) and np.all(np.isneginf(g[..., 0][empty]))
    lse_ref = m[~empty] + np.log(l[~empty])
    lse = g[..., 0][~empty] + np.log(g[..., 1][~empty])
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=2e-3)


@pytest.mark.parametrize("G", [1, 2, 5])
def test_attn_combine(csa, G):
    B, T, H, D = 2, 1, 64, 512
    rng = np.random.default_rng(G)
    o = bf16_round(rng.standard_normal((G, B, T, H, D)))
    m = rng.standard_normal((G, B, T, H)) * 3
    l = rng.uniform(0.5, 50, (G, B, T, H))
    l[0, 0, 0, :5] = 0
    m[0, 0, 0, :5] = -np.inf                               # empty pieces
    sink = rng.standard_normal(H).astype(np.float32)
    ref = oracle.attn_combine(m, l, o, sink)
    parts = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16).cuda()
    ml = torch.from_numpy(np.stack([m, l], -1).astype(np.float32)).cuda()
    got = csa.attn_combine(parts, ml, torch.from_numpy(sink).cuda())
    check_attn_bf16(_np(got), ref, what=f"combine G={G}")


@pytest.mark.parametrize("G,k", [(1, 64), (2, 512), (4, 1024), (8, 1024)])
def test_shard_select_and_remap(csa, G, k):
    """Gathered per-shard lists made by the oracle (ascending global indices, -1 padding,
    many exact ties) -> the GPU global top-k equals the oracle's top-k of the whole row."""
    B, N = 2, 20000
    rng = np.random.default_rng(k + G)
    s = (rng.standard_normal((B, 1, N)) * 64).astype(np.float32)
    s[1, 0, ::5] = 7.0
    nv = np.array([[N], [N - 999]], np.int32)
    bounds = [shard.shard_range(N, G, g) for g in range(G)]
    cs, ci = [], []
    for lo, hi in bounds:
        nvl = np.clip(nv - lo, 0, hi - lo).astype(np.int32)
        loc = oracle.topk(np.ascontiguousarray(s[..., lo:hi]), nvl, k)[:, 0]
        cs.append(np.where(loc >= 0, np.take_along_axis(s[:, 0, lo:hi], np.maximum(loc, 0), -1), -np.inf))
        ci.append(np.where(loc >= 0, loc + lo, -1))
    pairs = np.stack([np.stack(cs).astype(np.float32).view(np.int32), np.stack(ci).astype(np.int32)], -1)
    got = csa.shard_select(torch.from_numpy(pairs).cuda(), k).cpu().numpy()
    ref = oracle.topk(s, nv, k)[:, 0]
    for b in range(B):
        assert sorted(x for x in got[b] if x >= 0) == sorted(x for x in ref[b] if x >= 0)
    lo, hi = bounds[-1]
    loc = csa.shard_remap(torch.from_numpy(ref).cuda(), lo, hi, 0).cpu().numpy()
    np.testing.assert_array_equal(loc, np.where((ref >= lo) & (ref < hi), ref - lo, -1))
    back = csa.shard_remap(torch.from_numpy(loc).cuda(), 0, hi - lo, lo).cpu().numpy()
    np.testing.assert_array_equal(back, np.where((ref >= lo) & (ref < hi), ref, -1))
    sc = rng.standard_normal(loc.shape).astype(np.float32)
    pk = csa.shard_pack(torch.from_numpy(sc).cuda(), torch.from_numpy(loc).cuda(), hi - lo, lo).cpu().numpy()
    ok = loc >= 0
    np.testing.assert_array_equal(pk[..., 1], np.where(ok, loc + lo, -1))
    np.testing.assert_array_equal(np.ascontiguousarray(pk[..., 0]).view(np.float32), np.where(ok, sc, -np.inf))


@pytest.mark.parametrize("G", [1, 2, 4])
def test_sharded_decode_emulated(csa, G):
    """The whole sharded step, G shards run one after the other on this GPU, against the
    oracle chain over the unsharded sequence (exact scores -> top-k -> attention + sink)."""
    B, N, H, D, k, W = 2, 12000, 128, 512, 512, 130
    wl = synth.Workload("shard_decode", "bf16", B=B, ctx=4 * N, T=1, q_pos0=4 * N - 1, ratio=4, N=N, H=H, D=D, topk=k)
    ix = synth.draw_indexer(wl)
    at = synth.draw_attention(wl)
    q_pos = torch.full((B, 1), wl.q_pos0, dtype=torch.int64)
    swa_pos0 = torch.full((B,), wl.swa_pos0, dtype=torch.int64)
    nv = torch.from_numpy(oracle.n_visible(q_pos.numpy(), 4, N))
    scale = 1 / math.sqrt(D)
    shards, kern = [], []
    for g in range(G):
        lo, hi = shard.shard_range(N, G, g)
        shards.append(shard.Shard(rank=g, world=G, lo=lo, hi=hi, kI=ix["kI"][:, lo:hi].contiguous().cuda(),
                                  kv=at["kv"][:, lo:hi].contiguous().cuda(), swa=at["swa_kv"].cuda(),
                                  swa_pos0=swa_pos0.cuda(), q_pos=q_pos.cuda(), sink=at["sink"].cuda(),
                                  n_valid=csa.csa_n_valid(q_pos.cuda(), 4, lo, hi)))
        kern.append(shard.GpuKernels(k, scale))
    qI, w, q = ix["qI"].cuda(), ix["w"].cuda(), at["q"].cuda()
    all_pairs = torch.stack([kern[g].local_topk(shards[g], qI, w) for g in range(G)])      # the first all-gather
    gathered = torch.stack([kern[g].attend(shards[g], q, all_pairs).clone() for g in range(G)])  # the second
    out = kern[0].combine(shards[0], gathered, tuple(q.shape))
    glob = kern[0].buf["glob"].cpu().numpy()
    s_ref, smag = oracle.index_scores(_np(ix["qI"]), ix["w"].numpy(), _np(ix["kI"]), nv.numpy(), with_mag=True)
    idx_ref = oracle.topk(s_ref.astype(np.float32), nv.numpy(), k)
    for b in range(B):
        check_topk_sets(glob[b], s_ref[b, 0], k, 1e-5 * smag.max(), what=f"sharded G={G} b={b}")
        # the exact rescoring makes the global selection the oracle's, index for index
        assert np.array_equal(glob[b], idx_ref[b, 0]), f"sharded G={G} b={b}: set differs from the oracle's"
    ref = oracle.sparse_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0.numpy(), q_pos.numpy(),
                             at["sink"].numpy(), idx_ref, scale)
    check_attn_bf16(_np(out), ref, what=f"sharded G={G}")
