"""Hadamard-rotated e4m3 quantiser (csa_quantize_e4m3_hadamard) against the CPU oracle:
bit-exact codes and scales on ragged row counts, every supported width and both input
types; sampled rows of the full-size decode key caches; the e4m3 indexer on rotated
operands; and the top-k recall on outlier-channel inputs, the case the rotation is for."""
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


def _same(csa, x, what):
    codes, scale = csa.csa_quantize_e4m3(x.cuda(), hadamard=True)
    rc, rs = oracle.quantize_rows_e4m3_hadamard(x.float().numpy())
    got_s = scale.cpu().numpy()
    got_c = codes.cpu().numpy()
    bad = np.argwhere(got_c != rc)
    assert np.array_equal(got_s, rs), f"{what}: scales differ in {np.sum(got_s != rs)} rows"
    assert bad.size == 0, f"{what}: {len(bad)} codes differ, first at {bad[0].tolist()}"


@pytest.mark.parametrize("cols", [32, 64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows", [1, 7, 333, 2049])
def test_bit_exact_ragged(csa, cols, dtype, rows):
    """Row counts that leave the last block of 8 warps partly empty, and one that needs
    a second pass of the grid-stride loop on no GPU (2049 rows stay in one pass)."""
    x = synth.store(synth.normal(rows * 10 + cols, f"had/{dtype}", (rows, cols), std=3.0), dtype)
    _same(csa, x, f"rows={rows} cols={cols} {dtype}")


def test_special_rows(csa):
    """Worked rows (one-hot, e_0 +- e_1), a zero row, a row of negative zeros (+0 codes,
    scale 1), a row of one huge and many tiny values, constant rows and outlier channels."""
    n = 128
    x = torch.zeros(12, n, dtype=torch.float32)
    x[0, 0] = 2.0
    x[1, 0] = x[1, 1] = 1.0
    x[2, 0], x[2, 1] = 1.0, -1.0
    x[3, 5] = -3.0
    x[5] = -0.0
    x[6, 0] = 3.0e4
    x[6, 1:] = 1.0e-3
    x[7] = 1.0
    x[8] = -2.5
    x[9] = synth.normal(1, "had/special", (n,))
    x[9, 3] += 40.0
    x[10, ::2] = 1.0
    x[10, 1::2] = -1.0
    x[11] = torch.arange(n, dtype=torch.float32) - 63.5
    for dtype in ("bf16", "f32"):
        _same(csa, synth.store(x, dtype), f"special {dtype}")
    codes, scale = csa.csa_quantize_e4m3(synth.store(x, "bf16").cuda(), hadamard=True)
    assert scale[5].item() == 1.0 and int(codes[5].abs().sum().item()) == 0


def test_empty_is_a_no_op(csa):
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    codes, scale = csa.csa_quantize_e4m3(x, hadamard=True)
    assert codes.shape == (0, 128) and scale.shape == (0,)


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_full_size_key_cache_sampled(csa, name):
    """The whole index-key cache of the decode workloads in one launch ([B*N, 128] rows);
    the oracle checks 2,048 sampled rows and the first and last rows."""
    wl = synth.WORKLOADS[name]
    kI = synth.draw_indexer(wl)["kI"]
    flat = kI.reshape(-1, 128)
    codes, scale = csa.csa_quantize_e4m3(flat.cuda(), hadamard=True)
    rows = synth.random_subset(7, f"had/{name}/rows", [flat.shape[0]], 2048)[0].numpy()
    rows = np.unique(np.concatenate([rows, [0, flat.shape[0] - 1]]))
    rc, rs = oracle.quantize_rows_e4m3_hadamard(flat[rows].float().numpy())
    assert np.array_equal(scale.cpu().numpy()[rows], rs)
    assert np.array_equal(codes.cpu().numpy()[rows], rc)


def test_indexer_on_rotated_operands(csa):
    """e4m3 scores of rotated queries and keys: the GPU chain (rotated quantiser, e4m3
    indexer) against the oracle's rotated codes and e4m3 score definition."""
    from tolerances import check_f32
    B, T, N = 2, 3, 1000
    x = synth.draw_indexer_outliers(2, B, T, N)
    nv = np.array([[N, 777, 5], [N - 1, 130, N]], np.int32)
    g = {k: v.cuda() for k, v in x.items()}
    q8, qs = csa.csa_quantize_e4m3(g["qI"], hadamard=True)
    k8, ks = csa.csa_quantize_e4m3(g["kI"], hadamard=True)
    s = csa.csa_index_scores(q8, g["w"], k8, torch.from_numpy(nv).cuda(), q_scale=qs, k_scale=ks)
    rq8, rqs = oracle.quantize_rows_e4m3_hadamard(x["qI"].float().numpy())
    rk8, rks = oracle.quantize_rows_e4m3_hadamard(x["kI"].float().numpy())
    ref, mag = oracle.index_scores_e4m3(rq8, rqs, x["w"].numpy(), rk8, rks, nv, with_mag=True)
    got = s.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref)
    assert np.all(np.isneginf(got[~fin]))
    check_f32(got[fin], ref[fin], mag[fin], what="rotated e4m3 scores")


def test_recall_on_outlier_channels(csa):
    """Outlier channels shared by queries and keys (flash64k-sized key cache, k = 512):
    e4m3 top-k recall against the exact ranking is higher with the rotation, and with the
    2k-candidate rerank the rotated chain reaches >= 0.99 (the unrotated one is printed)."""
    B, T, N, k = 2, 1, 16384, 512
    x = synth.draw_indexer_outliers(5, B, T, N)
    nv = np.full((B, T), N, np.int32)
    g_nv = torch.from_numpy(nv).cuda()
    g = {n: v.cuda() for n, v in x.items()}
    ref = oracle.index_scores(x["qI"].float().numpy(), x["w"].numpy(), x["kI"].float().numpy(), nv)
    idx_ref = oracle.topk(ref.astype(np.float32), nv, k)
    rec = {}
    for had in (False, True):
        q8, qs = csa.csa_quantize_e4m3(g["qI"], hadamard=had)
        k8, ks = csa.csa_quantize_e4m3(g["kI"], hadamard=had)
        s8 = csa.csa_index_scores(q8, g["w"], k8, g_nv, q_scale=qs, k_scale=ks)
        plain = csa.csa_topk(s8, g_nv, k).cpu().numpy()
        idx = csa.csa_index_rerank(g["qI"], g["w"], g["kI"], csa.csa_topk(s8, g_nv, 2 * k), k).cpu().numpy()
        rec[had] = (min(len(np.intersect1d(plain[b, 0], idx_ref[b, 0])) / k for b in range(B)),
                    min(len(np.intersect1d(idx[b, 0], idx_ref[b, 0])) / k for b in range(B)))
    print(f"outlier channels: e4m3 top-{k} recall plain / 2k rerank: unrotated {rec[False]}, rotated {rec[True]}")
    assert rec[True][0] > rec[False][0] + 0.05
    assert rec[True][1] >= 0.99
