"""Indexer parity: fp32 SIMT, bf16 and e4m3 tcgen05 paths vs the CPU oracle; e4m3
quantiser bit-exactness; FP8 top-k recall against the exact (unquantised) ranking."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import check_f32, check_topk_sets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _inputs(wl, seed=0, N=None):
    ix = synth.draw_indexer(wl, seed=seed, N=N)
    q_pos = np.array([wl.q_pos] * wl.B, np.int64)
    nv = oracle.n_visible(q_pos, wl.ratio, ix["kI"].shape[1])
    return ix, q_pos, nv


def _check_scores(gpu, ref, mag, what):
    fin = np.isfinite(ref)
    assert np.all(np.isneginf(gpu[~fin])), f"{what}: invalid tail not -inf"
    check_f32(gpu[fin], ref[fin], mag[fin], what=what)


def test_f32_tiny_full(csa):
    wl = synth.WORKLOADS["tiny"]
    ix, _, nv = _inputs(wl)
    s = csa.csa_index_scores(ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda(), torch.from_numpy(nv).cuda())
    ref, mag = oracle.index_scores(ix["qI"].numpy(), ix["w"].numpy(), ix["kI"].numpy(), nv, with_mag=True)
    _check_scores(s.cpu().numpy().astype(np.float64), ref, mag, "tiny fp32")


@pytest.mark.parametrize("T", [1, 2, 3, 5, 9])
@pytest.mark.parametrize("N", [128, 1000, 3 * 128 + 1])
def test_bf16_ragged(csa, T, N):
    """Several query groups (T not a multiple of the group size), a ragged last key tile,
    and per-query n_valid below N."""
    wl = synth.Workload("idx_ragged", "bf16", B=2, ctx=4 * N, T=T, q_pos0=4 * N - 3 * T - 2, ratio=4, N=N,
                        H=16, D=128, index_dtype="bf16")
    ix, _, nv = _inputs(wl, seed=T * 1000 + N)
    nv[1, 0] = min(N, 5)                                 # a short row
    s = csa.csa_index_scores(ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda(), torch.from_numpy(nv).cuda())
    ref, mag = oracle.index_scores(ix["qI"].float().numpy(), ix["w"].numpy(), ix["kI"].float().numpy(), nv,
                                   with_mag=True)
    _check_scores(s.cpu().numpy().astype(np.float64), ref, mag, f"bf16 T={T} N={N}")


def test_quantizer_bit_exact(csa):
    x = synth.store(synth.normal(0, "quant/x", (3000, 128), std=2.0), "bf16")
    x[7] = 0                                             # all-zero row -> scale 1
    x[8, 5] = 1e-30                                      # tiny values
    codes, scale = csa.csa_quantize_e4m3(x.cuda())
    rc, rs = oracle.quantize_rows_e4m3(x.float().numpy())
    assert np.array_equal(scale.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)
    xf = synth.normal(0, "quant/xf", (257, 128), std=30.0)
    codes, scale = csa.csa_quantize_e4m3(xf.cuda())
    rc, rs = oracle.quantize_rows_e4m3(xf.numpy())
    assert np.array_equal(scale.cpu().numpy(), rs) and np.array_equal(codes.cpu().numpy(), rc)


@pytest.mark.parametrize("T,N", [(1, 1000), (3, 517), (4, 256), (6, 130)])
def test_e4m3_ragged(csa, T, N):
    wl = synth.Workload("idx8", "bf16", B=2, ctx=4 * N, T=T, q_pos0=4 * N - T - 9, ratio=4, N=N, H=16, D=128,
                        index_dtype="e4m3")
    ix, _, nv = _inputs(wl, seed=17 + T)
    q8, qs = oracle.quantize_rows_e4m3(ix["qI"].float().numpy())
    k8, ks = oracle.quantize_rows_e4m3(ix["kI"].float().numpy())
    s = csa.csa_index_scores(torch.from_numpy(q8).cuda(), ix["w"].cuda(), torch.from_numpy(k8).cuda(),
                             torch.from_numpy(nv).cuda(), q_scale=torch.from_numpy(qs).cuda(),
                             k_scale=torch.from_numpy(ks).cuda())
    ref, mag = oracle.index_scores_e4m3(q8, qs, ix["w"].numpy(), k8, ks, nv, with_mag=True)
    _check_scores(s.cpu().numpy().astype(np.float64), ref, mag, f"e4m3 T={T} N={N}")


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_full_decode_workloads(csa, name):
    """Full-size decode indexers: bf16 and the e4m3 variant, every score checked."""
    wl = synth.WORKLOADS[name]
    ix, _, nv = _inputs(wl)
    g_nv = torch.from_numpy(nv).cuda()
    if name == "flash64k":
        s = csa.csa_index_scores(ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda(), g_nv)
        ref, mag = oracle.index_scores(ix["qI"].float().numpy(), ix["w"].numpy(), ix["kI"].float().numpy(), nv,
                                       with_mag=True)
        _check_scores(s.cpu().numpy().astype(np.float64), ref, mag, name + " bf16")
    q8, qs = oracle.quantize_rows_e4m3(ix["qI"].float().numpy())
    k8, ks = oracle.quantize_rows_e4m3(ix["kI"].float().numpy())
    s8 = csa.csa_index_scores(torch.from_numpy(q8).cuda(), ix["w"].cuda(), torch.from_numpy(k8).cuda(), g_nv,
                              q_scale=torch.from_numpy(qs).cuda(), k_scale=torch.from_numpy(ks).cuda())
    ref8, mag8 = oracle.index_scores_e4m3(q8, qs, ix["w"].numpy(), k8, ks, nv, with_mag=True)
    _check_scores(s8.cpu().numpy().astype(np.float64), ref8, mag8, name + " e4m3")


def test_prefill_sampled_rows(csa):
    """Full prefill launch (4096 queries x 32768 keys); the oracle checks sampled query rows."""
    wl = synth.WORKLOADS["flash_prefill"]
    ix, _, nv = _inputs(wl)
    s = csa.csa_index_scores(ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda(), torch.from_numpy(nv).cuda())
    rows = [0, 1, 2, 3, 4, 1023, 2048, 3071, 4092, 4093, 4094, 4095]
    ref, mag = oracle.index_scores(ix["qI"][:, rows].float().numpy(), ix["w"][:, rows].numpy(),
                                   ix["kI"].float().numpy(), nv[:, rows], with_mag=True)
    _check_scores(s[:, rows].cpu().numpy().astype(np.float64), ref, mag, "prefill sampled")
    # every row: the invalid tail is -inf exactly and the valid part is finite
    s_all = s.cpu()
    for t in range(0, wl.T, 97):
        assert torch.isneginf(s_all[0, t, nv[0, t]:]).all() and torch.isfinite(s_all[0, t, :nv[0, t]]).all()


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_e4m3_recall_with_rerank(csa, name):
    """FP8 indexer as the pages run it: e4m3 scores pick 2k candidates, the candidates are
    rescored exactly (bf16 inputs, fp32 accumulation) and the best k kept.  GPU chain
    (quantiser, e4m3 scores, top-2k, rerank) against the exact top-k of the bf16
    inputs (oracle scores + oracle top-k): recall >= 0.99.  Plain e4m3 top-k recall is
    printed for the record."""
    wl = synth.WORKLOADS[name]
    ix, _, nv = _inputs(wl)
    g_nv = torch.from_numpy(nv).cuda()
    qI, kI, w = ix["qI"].cuda(), ix["kI"].cuda(), ix["w"].cuda()
    q8, qs = csa.csa_quantize_e4m3(qI)
    k8, ks = csa.csa_quantize_e4m3(kI)
    s8 = csa.csa_index_scores(q8, w, k8, g_nv, q_scale=qs, k_scale=ks)
    plain = csa.csa_topk(s8, g_nv, wl.topk).cpu().numpy()
    cand = csa.csa_topk(s8, g_nv, 2 * wl.topk)
    idx = csa.csa_index_rerank(qI, w, kI, cand, wl.topk).cpu().numpy()
    ref = oracle.index_scores(ix["qI"].float().numpy(), ix["w"].numpy(), ix["kI"].float().numpy(), nv)
    idx_ref = oracle.topk(ref.astype(np.float32), nv, wl.topk)
    rec_plain, rec = [], []
    for b in range(wl.B):
        rec_plain.append(len(np.intersect1d(plain[b, 0], idx_ref[b, 0])) / wl.topk)
        rec.append(len(np.intersect1d(idx[b, 0], idx_ref[b, 0])) / wl.topk)
    print(f"{name}: e4m3 top-{wl.topk} recall plain {min(rec_plain):.4f}, with 2k rerank {min(rec):.4f}")
    assert min(rec) >= 0.99


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rerank_parity(csa, dtype):
    """csa_index_rerank on seeded candidate lists (-1 padded) against the oracle's plain
    scores of the candidates and the oracle top-k among them (tie window of the fp32
    rescoring error)."""
    B, T, N, kc, k = 2, 3, 5000, 700, 300
    wl = synth.Workload("rerank", dtype, B=B, ctx=4 * N, T=T, q_pos0=4 * N - T, ratio=4, N=N, H=16, D=128,
                        index_dtype=dtype)
    ix = synth.draw_indexer(wl, seed=21)
    cand = synth.random_subset(21, "rerank/cand", torch.full((B, T), N), kc - 40).numpy()
    cand = np.concatenate([cand, np.full((B, T, 40), -1, np.int32)], -1)
    got = csa.csa_index_rerank(ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda(), torch.from_numpy(cand).cuda(),
                               k).cpu().numpy()
    for b in range(B):
        for t in range(T):
            c = cand[b, t][cand[b, t] >= 0]
            s, mag = oracle.index_scores(ix["qI"][b:b + 1, t:t + 1].float().numpy(), ix["w"][b:b + 1, t:t + 1].numpy(),
                                         ix["kI"][b:b + 1, c].float().numpy(), np.array([[len(c)]], np.int32),
                                         with_mag=True)
            pos_rec = check_topk_sets([int(np.searchsorted(c, i)) for i in got[b, t] if i >= 0], s[0, 0], k,
                                      1e-5 * mag.max(), what=f"rerank b={b} t={t}")
            assert pos_rec > 0.99
            assert np.all(np.isin(got[b, t], c))


def test_rerank_short_rows(csa):
    """Fewer valid candidates than k: every valid candidate, ascending, then -1."""
    B, T, N, kc, k = 1, 2, 600, 64, 40
    wl = synth.Workload("rerank_short", "bf16", B=B, ctx=4 * N, T=T, q_pos0=4 * N - T, ratio=4, N=N, H=16, D=128)
    ix = synth.draw_indexer(wl, seed=3)
    cand = np.full((B, T, kc), -1, np.int32)
    cand[0, 0, :25] = np.arange(0, 50, 2)
    cand[0, 1, :kc] = np.arange(kc)
    got = csa.csa_index_rerank(ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda(), torch.from_numpy(cand).cuda(),
                               k).cpu().numpy()
    assert got[0, 0].tolist() == list(range(0, 50, 2)) + [-1] * 15
    assert np.all(np.diff(got[0, 1]) > 0) and got[0, 1].min() >= 0


@pytest.mark.parametrize("mode", ["e4m3", "mxfp4", "bf16"])
@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_keys_ready_prefetch(csa, mode, name):
    """CSA_INDEX_KEYS_READY (first key tiles loaded before the wait for the previous launch)
    gives the same scores and the same select histogram, bit for bit, as the plain call, with
    the query quantiser as the launch just before the indexer (the decode step's order)."""
    wl = synth.WORKLOADS[name]
    ix, _, nv = _inputs(wl)
    g_nv = torch.from_numpy(nv).cuda()
    qI, kI, w = ix["qI"].cuda(), ix["kI"].cuda(), ix["w"].cuda()
    if mode == "e4m3":
        k, ks = csa.csa_quantize_e4m3(kI)
        q, qs = csa.csa_quantize_e4m3(qI)
        quant = lambda: csa.csa_quantize_e4m3(qI, codes=q, scale=qs)
    elif mode == "mxfp4":
        k, ks = csa.csa_quantize_mxfp4_sf128(kI, wl.B)
        q, qs = csa.csa_quantize_mxfp4_sf128(qI, wl.B)
        quant = lambda: csa.csa_quantize_mxfp4_sf128(qI, wl.B, codes=q, sf=qs)
    else:
        k, ks, q, qs = kI, None, qI, None
        quant = lambda: csa.csa_n_valid(torch.zeros_like(g_nv, dtype=torch.int64), 4, 0, 1)
    torch.cuda.synchronize()
    out = {}
    for ready in (False, True, True):
        ws = csa.select_workspace(wl.B, wl.N)
        quant()
        s = csa.csa_index_scores(q, w, k, g_nv, q_scale=qs, k_scale=ks, select_ws=ws, mxfp4=mode == "mxfp4",
                                 keys_ready=ready)
        torch.cuda.synchronize()
        out.setdefault(ready, []).append((s.clone(), ws.clone()))
    base_s, base_ws = out[False][0]
    for s, ws in out[True]:
        assert torch.equal(s, base_s), f"{name} {mode}: scores differ with the key prefetch"
        assert torch.equal(ws, base_ws), f"{name} {mode}: select histogram differs with the key prefetch"
