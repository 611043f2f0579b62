"""Top-k parity: bit-exact indices against the oracle's full sort on the same fp32
score buffers (drawn by the seeded generator, with planted exact ties and +-0.0)."""
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


def _run(csa, scores, nv, k):
    g = csa.csa_topk(scores.cuda(), torch.from_numpy(nv).cuda(), k).cpu().numpy()
    ref = oracle.topk(scores.numpy(), nv, k)
    assert np.array_equal(g, ref), f"mismatch in {np.argwhere((g != ref).any(-1))[:5].tolist()}"
    return g


@pytest.mark.parametrize("B,T,N,k", [
    (1, 8, 1024, 64),          # tiny: row-resident path
    (8, 1, 16384, 512),        # flash decode: chunk path (few rows)
    (1, 1, 262144, 1024),      # pro 1M decode: chunk path (long row)
    (1, 96, 5000, 512),        # many rows, ragged N: row path
    (2, 3, 40000, 700),        # N above the resident limit: chunk path, odd k
    (1, 1, 1 << 20, 2048),     # maximum N and k
])
def test_topk_shapes(csa, B, T, N, k):
    s = synth.draw_scores(0, f"topk/{B}/{T}/{N}", B, T, N, ties=8)
    nv = np.full((B, T), N, np.int32)
    _run(csa, s, nv, k)


@pytest.mark.parametrize("N", [3000, 20000, 100000])
def test_topk_ragged_n_valid(csa, N):
    """Rows with n_valid below N (the tail must be ignored even if it holds large values),
    n_valid < k (all valid then -1), n_valid == k, and n_valid == 0."""
    B, T, k = 1, 6, 512
    s = synth.draw_scores(1, f"topk/ragged/{N}", B, T, N, ties=4)
    nv = np.array([[N, N - 1, N // 2 + 3, k, k - 7, 0]], np.int32)
    s[0, 2, nv[0, 2]:] = 1e30                            # huge values past n_valid must not be chosen
    _run(csa, s, nv, k)


@pytest.mark.parametrize("N", [2048, 50000])
def test_topk_all_equal_and_signed_zero(csa, N):
    """Degenerate rows: every score equal (the k lowest indices win), all +-0.0 mixed,
    and a row where exactly k-1 values exceed a tied block."""
    B, T, k = 1, 3, 256
    s = torch.zeros(B, T, N)
    s[0, 0] = 3.25
    s[0, 1] = torch.where(torch.arange(N) % 3 == 0, torch.tensor(-0.0), torch.tensor(0.0))
    s[0, 2] = 1.0
    pos = synth.uniform(2, "topk/eqpos", (k - 1,)) * N
    s[0, 2, pos.long()] = 2.0
    nv = np.full((B, T), N, np.int32)
    g = _run(csa, s, nv, k)
    assert g[0, 0].tolist() == list(range(k))
    assert g[0, 1].tolist() == list(range(k))


def test_topk_row_sampled_threshold_and_its_fallbacks(csa):
    """Rows of 8,192..32,768 scores try a threshold placed by a strided sample of 1,024
    keys first.  Rows where that cannot work must fall back to the full radix: every score
    equal (the count above the threshold exceeds the candidate space), and a row whose
    sampled positions hold its largest values (too few keys reach the threshold).  Plus a
    plain row and a heavy-tailed one; all bit for bit against the oracle."""
    B, T, N, k = 1, 4, 20000, 512
    s = synth.draw_scores(13, "topk/sampled", B, T, N, ties=4)
    s[0, 0] = 7.5                                            # all equal
    stride = N // 1024
    s[0, 1] = synth.normal(13, "topk/sampled/small", (N,))
    s[0, 1, 0:1024 * stride:stride] = 1000.0 + torch.arange(1024, dtype=torch.float32)
    s[0, 3] = torch.exp(4 * synth.normal(13, "topk/sampled/tail", (N,)))   # heavy tail
    nv = np.array([[N, N, N - 3, N]], np.int32)
    g = _run(csa, s, nv, k)
    assert g[0, 0].tolist() == list(range(k))


def test_topk_workloads_chunk_and_row_paths_agree(csa):
    """The same rows through both paths (as one batch of many rows and as few rows)."""
    N, k = 16384, 512
    s = synth.draw_scores(3, "topk/paths", 1, 80, N, ties=4)
    nv = np.full((1, 80), N, np.int32)
    many = csa.csa_topk(s.cuda(), torch.from_numpy(nv).cuda(), k).cpu()        # row path (80 rows)
    few = torch.cat([csa.csa_topk(s[:, i:i + 8].contiguous().cuda(), torch.from_numpy(nv[:, i:i + 8]).cuda(), k).cpu()
                     for i in range(0, 80, 8)], 1)                            # chunk path (8 rows)
    assert torch.equal(many, few)


def test_topk_workspace_stays_zero(csa):
    """The long-row path leaves its workspace zero-filled, so calls can repeat."""
    N, k = 262144, 1024
    ws = csa.topk_workspace(1, 1, N, k)
    for seed in range(3):
        s = synth.draw_scores(seed, "topk/ws", 1, 1, N)
        nv = np.full((1, 1), N, np.int32)
        g = csa.csa_topk(s.cuda(), torch.from_numpy(nv).cuda(), k, workspace=ws).cpu().numpy()
        assert np.array_equal(g, oracle.topk(s.numpy(), nv, k))
        torch.cuda.synchronize()
        assert int(ws.count_nonzero()) == 0


# ----------------------------------------------------------------------------- fused decode select
def _order_key(x):
    u = np.asarray(x, np.float32).view(np.uint32).copy()
    u[(u << 1) == 0] = 0                                  # -0.0 -> +0.0
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


@pytest.mark.parametrize("B,N,k", [(8, 16384, 512), (1, 262144, 1024), (3, 5000, 700), (1, 1 << 19, 2048)])
def test_select_plain_matches_oracle(csa, B, N, k):
    """csa_score_histogram + csa_topk_select (no rescoring) == full-sort top-k, bit-exact,
    twice in a row on the same workspace (which must come back zeroed)."""
    s = synth.draw_scores(5, f"select/{B}/{N}", B, 1, N, ties=6)
    nv = np.full((B, 1), N, np.int32)
    if B >= 3:
        nv[1, 0] = N // 3
        nv[2, 0] = k - 5                                  # fewer valid than k
    ws = csa.select_workspace(B, N)
    g_s, g_nv = s.cuda(), torch.from_numpy(nv).cuda()
    ref = oracle.topk(s.numpy(), nv, k)
    for _ in range(2):
        csa.csa_score_histogram(g_s, g_nv, ws)
        got = csa.csa_topk_select(g_s, g_nv, k, ws).cpu().numpy()
        assert np.array_equal(got, ref)
    torch.cuda.synchronize()
    hdr = ws.view(torch.int32)
    stride = csa.csa_select_workspace_size(1, N) // 4
    for b in range(B):
        assert int(hdr[b * stride: b * stride + 4096 + 3].count_nonzero()) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_select_rescore_semantics(csa, dtype):
    """Rescoring mode: candidates are the indices whose (low-precision) score falls in the
    bin of the kc-th largest score or above; the result is the exact top-k of the plain
    indexer scores of those candidates (oracle), up to the rescoring error window."""
    B, N, k, kc = 2, 3000, 100, 200
    wl = synth.Workload("sel_rescore", dtype, B=B, ctx=4 * N, T=1, q_pos0=4 * N - 1, ratio=4, N=N, H=16, D=128,
                        index_dtype=dtype)
    ix = synth.draw_indexer(wl, seed=31)
    s = synth.draw_scores(31, "select/rescore", B, 1, N)
    nv = np.array([[N], [N - 777]], np.int32)
    ws = csa.select_workspace(B, N)
    g_s, g_nv = s.cuda(), torch.from_numpy(nv).cuda()
    csa.csa_score_histogram(g_s, g_nv, ws)
    got = csa.csa_topk_select(g_s, g_nv, k, ws, kc=kc, qI=ix["qI"].cuda(), w=ix["w"].cuda(),
                              kI=ix["kI"].cuda()).cpu().numpy()
    for b in range(B):
        v = s[b, 0, :nv[b, 0]].numpy()
        order = np.lexsort((np.arange(v.size), -v.astype(np.float64)))
        bstar = _order_key(v[order[kc - 1]]) >> 20
        cand = np.nonzero((_order_key(v) >> 20) >= bstar)[0]
        ex, mag = oracle.index_scores(ix["qI"][b:b + 1].float().numpy(), ix["w"][b:b + 1].numpy(),
                                      ix["kI"][b:b + 1, cand].float().numpy(), np.array([[len(cand)]], np.int32),
                                      with_mag=True)
        pos = [int(np.searchsorted(cand, i)) for i in got[b, 0] if i >= 0]
        assert np.all(np.isin(got[b, 0], cand))
        check_topk_sets(pos, ex[0, 0], k, 1e-5 * mag.max(), what=f"select rescore b={b}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_select_exported_scores(csa, dtype):
    """idx_scores: beside each selected index the rescored score that ranked it, equal to the
    plain indexer score of that entry (oracle, fp32 rule); -inf beside the -1 pads.  Rows:
    full, ragged, n_valid <= k (every entry taken, rescored too) and n_valid = 0.  The
    selection itself is the one the call makes without idx_scores."""
    B, N, k, kc = 4, 3000, 100, 200
    wl = synth.Workload("sel_scores", dtype, B=B, ctx=4 * N, T=1, q_pos0=4 * N - 1, ratio=4, N=N, H=16, D=128,
                        index_dtype=dtype)
    ix = synth.draw_indexer(wl, seed=37)
    s = synth.draw_scores(37, "select/scores", B, 1, N)
    nv = np.array([[N], [N - 777], [k - 9], [0]], np.int32)
    ws = csa.select_workspace(B, N)
    g_s, g_nv = s.cuda(), torch.from_numpy(nv).cuda()
    qI, w, kI = ix["qI"].cuda(), ix["w"].cuda(), ix["kI"].cuda()
    csa.csa_score_histogram(g_s, g_nv, ws)
    plain = csa.csa_topk_select(g_s, g_nv, k, ws, kc=kc, qI=qI, w=w, kI=kI).cpu().numpy()
    sc = torch.empty((B, 1, k), dtype=torch.float32, device="cuda")
    csa.csa_score_histogram(g_s, g_nv, ws)
    got = csa.csa_topk_select(g_s, g_nv, k, ws, kc=kc, qI=qI, w=w, kI=kI, idx_scores=sc).cpu().numpy()
    sc = sc.cpu().numpy()
    assert np.array_equal(got, plain)
    for b in range(B):
        n = min(int(nv[b, 0]), k)
        sel = got[b, 0, :n]
        if nv[b, 0] <= k:
            assert sel.tolist() == list(range(n))
        assert np.all(got[b, 0, n:] == -1) and np.all(np.isneginf(sc[b, 0, n:]))
        if n == 0:
            continue
        ex, mag = oracle.index_scores(ix["qI"][b:b + 1].float().numpy(), ix["w"][b:b + 1].numpy(),
                                      ix["kI"][b:b + 1, sel].float().numpy(), np.array([[n]], np.int32),
                                      with_mag=True)
        check_f32(sc[b, 0, :n], ex[0, 0], mag[0, 0], what=f"select exported scores {dtype} b={b}")


def test_select_exported_scores_plain(csa):
    """Without rescoring idx_scores holds the input score of each selected index, bit for
    bit (the order key maps back to the float; -0.0 comes back as +0.0), on the shared-memory
    path, on a constant row (the global-memory path) and on a row of n_valid < k; N = 0 gives
    -1 and -inf throughout."""
    B, N, k = 3, 50000, 512
    s = synth.draw_scores(41, "select/scores_plain", B, 1, N, ties=6)
    s[1, 0] = 3.25
    nv = np.array([[N], [N], [k - 3]], np.int32)
    ws = csa.select_workspace(B, N)
    g_s, g_nv = s.cuda(), torch.from_numpy(nv).cuda()
    csa.csa_score_histogram(g_s, g_nv, ws)
    sc = torch.empty((B, 1, k), dtype=torch.float32, device="cuda")
    got = csa.csa_topk_select(g_s, g_nv, k, ws, idx_scores=sc).cpu().numpy()
    sc = sc.cpu().numpy()
    assert np.array_equal(got, oracle.topk(s.numpy(), nv, k))
    for b in range(B):
        ok = got[b, 0] >= 0
        assert np.array_equal(sc[b, 0, ok], s[b, 0].numpy()[got[b, 0, ok]])
        assert np.all(np.isneginf(sc[b, 0, ~ok]))
    e = torch.empty((2, 1, 0), device="cuda")
    nv0 = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    sc0 = torch.zeros((2, 1, 8), dtype=torch.float32, device="cuda")
    i0 = csa.csa_topk_select(e, nv0, 8, csa.select_workspace(2, 0), idx_scores=sc0).cpu().numpy()
    assert np.all(i0 == -1) and np.all(np.isneginf(sc0.cpu().numpy()))


def test_select_fed_by_indexer_histogram(csa):
    """The histogram the indexer epilogue accumulates equals the one the histogram kernel
    builds from the same scores: both selections are identical (e4m3 decode workload)."""
    wl = synth.WORKLOADS["flash64k"]
    ix = synth.draw_indexer(wl)
    q_pos = np.array([wl.q_pos] * wl.B, np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    g_nv = torch.from_numpy(nv).cuda()
    qI, kI, w = ix["qI"].cuda(), ix["kI"].cuda(), ix["w"].cuda()
    q8, qs = csa.csa_quantize_e4m3(qI)
    k8, ks = csa.csa_quantize_e4m3(kI)
    ws1, ws2 = csa.select_workspace(wl.B, wl.N), csa.select_workspace(wl.B, wl.N)
    s_fused = csa.csa_index_scores(q8, w, k8, g_nv, q_scale=qs, k_scale=ks, select_ws=ws1)
    s_plain = csa.csa_index_scores(q8, w, k8, g_nv, q_scale=qs, k_scale=ks)
    assert torch.equal(s_fused, s_plain)
    csa.csa_score_histogram(s_plain, g_nv, ws2)
    a = csa.csa_topk_select(s_fused, g_nv, wl.topk, ws1, kc=2 * wl.topk, qI=qI, w=w, kI=kI)
    b = csa.csa_topk_select(s_plain, g_nv, wl.topk, ws2, kc=2 * wl.topk, qI=qI, w=w, kI=kI)
    assert torch.equal(a, b)
    ref = oracle.index_scores(ix["qI"].float().numpy(), ix["w"].numpy(), ix["kI"].float().numpy(), nv)
    idx_ref = oracle.topk(ref.astype(np.float32), nv, wl.topk)
    got = a.cpu().numpy()
    recall = min(len(np.intersect1d(got[i, 0], idx_ref[i, 0])) / wl.topk for i in range(wl.B))
    print(f"flash64k fused e4m3 select recall {recall:.4f}")
    # the 2k-bin candidates are rescored exactly, so the selection is the oracle's outright
    assert np.array_equal(got, idx_ref), f"flash64k fused select differs from the exact top-k (recall {recall})"


@pytest.mark.parametrize("N", [3000, 50000])
def test_select_degenerate_ties(csa, N):
    """Fused select on rows dominated by ties: a constant row (every candidate ties with
    the k-th score, more ties than the tie list holds), a +-0.0 row, and a row with k-1
    values above a tied block -- the k lowest tied indices must win, as in the full sort."""
    B, k = 3, 512
    s = torch.zeros(B, 1, N)
    s[0, 0] = 3.25
    s[1, 0] = torch.where(torch.arange(N) % 3 == 0, torch.tensor(-0.0), torch.tensor(0.0))
    s[2, 0] = 1.0
    pos = torch.unique((synth.uniform(7, f"select/eqpos/{N}", (4 * k,)) * N).long())[: k - 1]
    s[2, 0, pos] = 2.0
    nv = np.full((B, 1), N, np.int32)
    ws = csa.select_workspace(B, N)
    g_s, g_nv = s.cuda(), torch.from_numpy(nv).cuda()
    csa.csa_score_histogram(g_s, g_nv, ws)
    got = csa.csa_topk_select(g_s, g_nv, k, ws).cpu().numpy()
    assert np.array_equal(got, oracle.topk(s.numpy(), nv, k))
    assert got[0, 0].tolist() == list(range(k))


def test_topk_prefill_rows_full_shape(csa):
    """The chunked-prefill top-k at its own shape, in the launch the prefill step makes:
    4,096 query rows of N = 32,768 scores, n_valid = (pos + 1) / 4 for positions
    126,976..131,071 (31,744..32,768), k = 512.  Rows carry planted exact ties (groups
    of equal values, +-0.0, extra copies of the row's k-th value, so the lower-index rule
    decides at the threshold) and huge values past n_valid.  64 sampled rows (the first
    and the last among them) are compared bit for bit with the oracle's full sort."""
    T, N, k = 4096, 32768, 512
    pos = np.arange(126976, 131072, dtype=np.int64)[None]
    nv = oracle.n_visible(pos, 4, N)
    assert nv.min() == 31744 and nv.max() == 32768
    dev = torch.device("cuda")
    s = synth.normal(11, "topk/prefill", (1, T, N), std=64.0, device=dev)
    # groups of 4 equal values per row
    tp = (synth.uniform(11, "topk/prefill/ties", (T, 32), device=dev) * 31744).long()
    src = s[0].gather(1, tp[:, 0::4])
    for j in range(1, 4):
        s[0].scatter_(1, tp[:, j::4], src)
    s[0, :, 1], s[0, :, 2], s[0, :, 3] = 0.0, -0.0, 0.0
    rows = np.unique(np.concatenate([[0, T - 1], (np.arange(62) * 66 + 5) % T]))[:64]
    g_nv = torch.from_numpy(nv).to(dev)
    for i, r in enumerate(rows.tolist()):
        n = int(nv[0, r])
        kth = torch.topk(s[0, r, :n], k).values[-1]
        extra = (synth.uniform(12, f"topk/prefill/kth/{r}", (3,), device=dev) * n).long()
        s[0, r, extra] = kth                                # three more copies of the k-th value
        if i % 3 == 0 and n < N:
            s[0, r, n:] = 1e30                              # past n_valid: must never be chosen
    got = csa.csa_topk(s, g_nv, k).cpu().numpy()
    host = s[0, torch.from_numpy(rows).to(dev)].cpu().numpy()
    for i, r in enumerate(rows.tolist()):
        ref = oracle.topk(host[i][None, None], nv[:, r:r + 1], k)[0, 0]
        assert np.array_equal(got[0, r], ref), f"row {r}"
