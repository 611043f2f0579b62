"""End-to-end chains on the GPU (compress -> index -> top-k -> sparse_attn; compress ->
hca_attn) against the same chain in the oracle.

Index sets: the GPU chain must select exactly the oracle chain's set for every query.
That is stricter than the fp32 rule alone, which only bounds each score's error by
1e-5 * mag (mag: the oracle's sum of |terms|; differences inside that a-priori window
would be allowed by check_topk_sets).  On these seeded inputs the gap between the k-th
and (k+1)-th exact score is at least 0.036 (tiny) and 6e-4 (pro1m), above the fp32
rounding the chains actually carry, so any difference at all is a failure.  Attention
outputs are then compared element by element for every query."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import bf16_round, check_attn_bf16, check_f32, check_topk_sets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def test_tiny_chain_fp32(csa):
    """The tiny fp32 workload chained: the compressor output is the index-key cache and the
    latent cache (c19's chained reading), then scores, top-64 and attention."""
    wl = synth.WORKLOADS["tiny"]
    cz = synth.draw_compressor(wl)
    comp = csa.csa_compress(*(cz[k].cuda() for k in ("C_a", "C_b", "Z_a", "Z_b")), ratio=4)      # [1, 1024, 128]
    comp_ref, cmag = oracle.compress_csa(*(cz[k].numpy() for k in ("C_a", "C_b", "Z_a", "Z_b")), with_mag=True)
    check_f32(comp.cpu().numpy(), comp_ref, cmag, what="tiny compressor", literal=True)
    ix = synth.draw_indexer(wl)
    q_pos = np.array([wl.q_pos], np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    s = csa.csa_index_scores(ix["qI"].cuda(), ix["w"].cuda(), comp, torch.from_numpy(nv).cuda())
    idx = csa.csa_topk(s, torch.from_numpy(nv).cuda(), wl.topk)
    comp_np = comp_ref.astype(np.float32)              # the oracle chain uses its own compressed cache
    s_ref, smag = oracle.index_scores(ix["qI"].numpy(), ix["w"].numpy(), comp_np, nv, with_mag=True)
    idx_np = idx.cpu().numpy()
    idx_ref = oracle.topk(s_ref.astype(np.float32), nv, wl.topk)
    for t in range(wl.T):
        check_topk_sets(idx_np[0, t], s_ref[0, t, :nv[0, t]], wl.topk, 1e-5 * smag[0, t].max(),
                        what=f"tiny chain t={t}")
    assert np.array_equal(idx_np, idx_ref), "tiny chain: index sets differ from the oracle chain's"
    at = synth.draw_attention(wl)
    swa_pos0 = np.array([wl.swa_pos0], np.int64)
    scale = 1 / math.sqrt(wl.D)
    o = csa.sparse_attn(at["q"].cuda(), comp, at["swa_kv"].cuda(), torch.from_numpy(swa_pos0).cuda(),
                        torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), idx, scale).cpu().numpy()
    # attention on the GPU's own (compressed) cache vs the oracle's: both caches agree
    # within 1e-5 of their magnitude, which the fp32 attention tolerance absorbs
    ref, mag = oracle.sparse_attn(at["q"].numpy(), comp_np, at["swa_kv"].numpy(), swa_pos0, q_pos,
                                  at["sink"].numpy(), idx_ref, scale, with_mag=True)
    check_f32(o, ref, np.maximum(mag, np.abs(ref)), what="tiny chain attention")


def test_pro1m_chain_fp8_rerank(csa):
    """Pro 1M decode as the benchmark runs it: e4m3 scores -> top-2048 -> exact rerank ->
    top-1024 -> sparse_attn, against oracle exact scores -> top-1024 -> attention."""
    wl = synth.WORKLOADS["pro1m"]
    ix = synth.draw_indexer(wl)
    q_pos = np.array([wl.q_pos], np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    g_nv = torch.from_numpy(nv).cuda()
    qI, kI, w = ix["qI"].cuda(), ix["kI"].cuda(), ix["w"].cuda()
    k8, ks = csa.csa_quantize_e4m3(kI)
    q8, qs = csa.csa_quantize_e4m3(qI)
    s8 = csa.csa_index_scores(q8, w, k8, g_nv, q_scale=qs, k_scale=ks)
    cand = csa.csa_topk(s8, g_nv, 2 * wl.topk)
    idx = csa.csa_index_rerank(qI, w, kI, cand, wl.topk)
    s_ref, smag = oracle.index_scores(ix["qI"].float().numpy(), ix["w"].numpy(), ix["kI"].float().numpy(), nv,
                                      with_mag=True)
    idx_np = idx.cpu().numpy()
    rec = check_topk_sets(idx_np[0, 0], s_ref[0, 0], wl.topk, 1e-5 * smag.max(), what="pro1m chain")
    idx_ref = oracle.topk(s_ref.astype(np.float32), nv, wl.topk)
    assert np.array_equal(idx_np, idx_ref), f"pro1m chain: the reranked set differs from the oracle's (recall {rec})"
    at = synth.draw_attention(wl)
    swa_pos0 = np.array([wl.swa_pos0], np.int64)
    scale = 1 / math.sqrt(wl.D)
    o = csa.sparse_attn(at["q"].cuda(), at["kv"].cuda(), at["swa_kv"].cuda(), torch.from_numpy(swa_pos0).cuda(),
                        torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), idx, scale).float().cpu().numpy()
    ref = oracle.sparse_attn(at["q"].float().numpy(), at["kv"].float().numpy(), at["swa_kv"].float().numpy(),
                             swa_pos0, q_pos, at["sink"].numpy(), idx_ref, scale)
    check_attn_bf16(o, ref, what="pro1m chain attention")


def test_hca_chain(csa):
    """128:1 compressor output used as the HCA cache tail, then dense attention."""
    wl = synth.Workload("hca_chain", "bf16", B=2, ctx=128 * 40, T=1, q_pos0=128 * 40 - 1, ratio=128, N=40,
                        H=128, D=512, comp_L=128 * 40, comp_c=512)
    cz = synth.draw_compressor(wl, seed=2)
    kv = csa.csa_compress(cz["C"].cuda(), None, cz["Z"].cuda(), None, ratio=128)
    at = synth.draw_attention(wl, seed=2)
    q_pos = np.array([[wl.q_pos0]] * 2, np.int64)
    swa_pos0 = np.array([wl.swa_pos0] * 2, np.int64)
    scale = 1 / math.sqrt(wl.D)
    o = csa.hca_attn(at["q"].cuda(), kv, at["swa_kv"].cuda(), torch.from_numpy(swa_pos0).cuda(),
                     torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), scale).float().cpu().numpy()
    kv_np = bf16_round(oracle.compress_hca(cz["C"].float().numpy(), cz["Z"].float().numpy())).astype(np.float32)
    ref = oracle.hca_attn(at["q"].float().numpy(), kv_np, at["swa_kv"].float().numpy(), swa_pos0, q_pos,
                          at["sink"].numpy(), scale)
    check_attn_bf16(o, ref, what="hca chain")
