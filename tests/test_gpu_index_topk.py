"""Fused indexer + top-k (csa_index_topk): the indices must equal, bit for bit, the
oracle's full sort of the scores the unfused indexer (csa_index_scores, the same kernel)
writes for the same inputs -- on ragged shapes, on rows that take the fallback, and at
the chunked-prefill shape (4,096 queries x 32,768 keys, top-512)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _operands(ix, dtype):
    """Device operands of both calls: bf16 as drawn, or e4m3 codes and scales (CPU oracle
    quantiser, so the codes do not come from the code under test)."""
    if dtype == "bf16":
        return {"qI": ix["qI"].cuda(), "kI": ix["kI"].cuda(), "q_scale": None, "k_scale": None}
    q8, qs = oracle.quantize_rows_e4m3(ix["qI"].float().numpy())
    k8, ks = oracle.quantize_rows_e4m3(ix["kI"].float().numpy())
    return {"qI": torch.from_numpy(q8).cuda(), "kI": torch.from_numpy(k8).cuda(),
            "q_scale": torch.from_numpy(qs).cuda(), "k_scale": torch.from_numpy(ks).cuda()}


def _run(csa, op, w, nv, k):
    """(fused idx, failed_rows, unfused scores) on the device."""
    g_nv = torch.from_numpy(nv).cuda()
    failed = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    idx = csa.csa_index_topk(op["qI"], w, op["kI"], g_nv, k, q_scale=op["q_scale"], k_scale=op["k_scale"],
                             failed_rows=failed)
    s = csa.csa_index_scores(op["qI"], w, op["kI"], g_nv, q_scale=op["q_scale"], k_scale=op["k_scale"])
    return idx, int(failed.item()), s


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("T,N,k", [(37, 5000, 256), (5, 1000, 64), (8, 32768, 512), (3, 20000, 1024),
                                   (1023, 2048, 64)])
def test_index_topk_matches_unfused(csa, dtype, T, N, k):
    """Ragged query groups and key tiles; rows with n_valid = 0, k - 1, k, k + 1, a short row
    (every key a candidate) and full rows.  The first four shapes spread a row's key tiles
    over many CTAs (one reservation per ballot); the last gives each CTA whole rows (32-slot
    chunks per warp, with zero-filled tails)."""
    B = 2
    wl = synth.Workload("idx_topk", "bf16", B=B, ctx=4 * N, T=T, q_pos0=4 * N - T, ratio=4, N=N, H=16, D=128,
                        index_dtype="bf16")
    ix = synth.draw_indexer(wl, seed=7 * T + N)
    nv = oracle.n_visible(np.array([wl.q_pos] * B, np.int64), 4, N).astype(np.int32)
    nv[1, 0] = 0
    nv[1, 1 % T] = k - 1
    nv[1, 2 % T] = k
    nv[0, 1 % T] = min(N, k + 1)
    nv[0, T - 1] = min(N, 3 * k + 17)
    op = _operands(ix, dtype)
    idx, failed, s = _run(csa, op, ix["w"].cuda(), nv, k)
    ref = oracle.topk(s.cpu().numpy(), nv, k)
    got = idx.cpu().numpy()
    bad = np.argwhere((got != ref).any(-1))
    assert bad.size == 0, f"{dtype} T={T} N={N} k={k}: rows {bad[:5].tolist()} differ (failed rows {failed})"
    assert failed == 0, f"{dtype} T={T} N={N} k={k}: {failed} rows took the fallback on random inputs"


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("case", ["sampled_keys_boosted", "all_keys_equal"])
@pytest.mark.parametrize("T,N,k", [(12, 6000, 256), (1024, 8192, 64)])
def test_index_topk_fallback(csa, dtype, case, T, N, k):
    """Rows the sample misleads.  sampled_keys_boosted: every 16th key (the sampled ones)
    scaled by 6, so for most rows the sampled threshold lies above all but about r = 4k/16
    keys and the candidate list is short (a row whose scores are mostly negative can still
    get enough).  all_keys_equal: every score of a row ties, so the list overflows.  The
    call counts those rows, takes its fallback and still returns the oracle's top-k (the
    lower index wins every tie).  Both reservation modes: one per ballot (12 queries) and
    32-slot chunks (1,024 queries, each CTA walking whole rows)."""
    B = 1
    wl = synth.Workload("idx_topk_fb", "bf16", B=B, ctx=4 * N, T=T, q_pos0=4 * N - T, ratio=4, N=N, H=16, D=128,
                        index_dtype="bf16")
    ix = synth.draw_indexer(wl, seed=99)
    kI = ix["kI"].float()
    if case == "sampled_keys_boosted":
        kI[0, ::16] *= 6.0
    else:
        kI[0] = kI[0, 0]
    ix["kI"] = synth.store(kI, "bf16")
    nv = oracle.n_visible(np.array([wl.q_pos] * B, np.int64), 4, N).astype(np.int32)
    op = _operands(ix, dtype)
    idx, failed, s = _run(csa, op, ix["w"].cuda(), nv, k)
    ref = oracle.topk(s.cpu().numpy(), nv, k)
    assert np.array_equal(idx.cpu().numpy(), ref)
    if case == "all_keys_equal":
        assert failed == T, f"{dtype}: {failed} of {T} tied rows counted as failed"
        assert ref[0, 0].tolist() == list(range(k))
    else:
        assert failed >= T // 2, f"{dtype}: only {failed} of {T} rows took the fallback"


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_index_topk_prefill_shape(csa, dtype):
    """The chunked prefill: 4,096 queries at positions 126,976..131,071 over N = 32,768
    compressed keys (n_valid 31,744..32,768), top-512.  Every row equals csa_topk of the
    unfused scores, and 64 sampled rows (the first and last among them) equal the oracle's
    full sort of those scores; no row takes the fallback."""
    wl = synth.WORKLOADS["flash_prefill"]
    ix = synth.draw_indexer(wl)
    nv = oracle.n_visible(np.array([wl.q_pos] * wl.B, np.int64), wl.ratio, wl.N).astype(np.int32)
    op = _operands(ix, dtype)
    idx, failed, s = _run(csa, op, ix["w"].cuda(), nv, wl.topk)
    plain = csa.csa_topk(s, torch.from_numpy(nv).cuda(), wl.topk)
    assert torch.equal(idx, plain), "fused and unfused top-k differ"
    rows = np.unique(np.concatenate([[0, wl.T - 1], (synth.uniform(3, "index_topk/rows", (62,)) * wl.T).long().numpy()]))
    ref = oracle.topk(s[:, rows].cpu().numpy(), nv[:, rows], wl.topk)
    assert np.array_equal(idx[:, rows].cpu().numpy(), ref)
    assert failed == 0, f"{failed} rows took the fallback"


def test_index_topk_no_keys(csa):
    """N = 0: every row is -1 and failed_rows is set to 0."""
    B, T, k = 2, 5, 16
    qI = torch.zeros((B, T, 64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((B, T, 64), dtype=torch.float32, device="cuda")
    kI = torch.zeros((B, 0, 128), dtype=torch.bfloat16, device="cuda")
    nv = torch.zeros((B, T), dtype=torch.int32, device="cuda")
    failed = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    idx = csa.csa_index_topk(qI, w, kI, nv, k, failed_rows=failed)
    assert (idx.cpu() == -1).all() and int(failed.item()) == 0
