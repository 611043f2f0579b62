"""The FP4 index QK ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §2 table and §4.2: the
index QK path runs in FP4; format reading c25, OCP MXFP4) on the block-scaled tensor cores:

- csa_quantize_mxfp4_sf128: the codes equal csa_quantize_mxfp4's, and every scale byte,
  moved from the tensor-core layout back to [rows, 4], equals the oracle's;
- csa_index_scores with dtype CSA_MXFP4 against oracle.index_scores on the oracle's own
  dequantised operands (code * 2^(e - 127) per block of 32), fp32 rule 1e-5 * mag, at the
  decode shapes, ragged key counts and several queries per sequence;
- the decode top-k fed by the FP4 scores with the exact bf16 rescoring of the candidates
  of the 4k-th score's bin: recall against the oracle's exact top-k (>= 0.99).  FP4 scores
  are coarser than e4m3 ones, so the candidate list is twice the e4m3 path's."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import check_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _unpack_sf128(sf, batches, rpb):
    """Tensor-core scale layout -> [batches * rpb, 4] (byte 16 m0 + 4 m1 + s of each atom)."""
    tiles = (rpb + 127) // 128
    atoms = sf[: batches * tiles * 512].reshape(batches, tiles, 32, 4, 4)       # [b][tile][m0][m1][s]
    rows = atoms.transpose(0, 1, 3, 2, 4).reshape(batches, tiles * 128, 4)      # row = 32 m1 + m0
    return rows[:, :rpb].reshape(batches * rpb, 4)


def _operands(x, batches, hadamard=True):
    """Oracle codes / scales of rows x [..., 128] and their dequantised values [..., 128]."""
    flat = x.float().numpy().reshape(-1, 128)
    rc, rs = oracle.quantize_rows_mxfp4(flat, hadamard=hadamard)
    deq = oracle.mxfp4_dequantize(rc, rs)
    return rc, rs, deq.reshape(x.shape)


@pytest.mark.parametrize("batches,rpb", [(1, 300), (3, 128), (8, 64), (2, 1000)])
def test_sf128_layout(csa, batches, rpb):
    x = synth.store(synth.normal(rpb, "mx4/sf128", (batches * rpb, 128)), "bf16")
    codes, sf = csa.csa_quantize_mxfp4_sf128(x.cuda(), batches)
    c_ref, s_plain = csa.csa_quantize_mxfp4(x.cuda(), hadamard=True)
    assert torch.equal(codes, c_ref)
    rc, rs, _ = _operands(x, batches)
    assert np.array_equal(_unpack_sf128(sf.cpu().numpy(), batches, rpb), rs)
    assert np.array_equal(s_plain.cpu().numpy(), rs)


@pytest.mark.parametrize("B,T,N", [(8, 1, 16384), (1, 1, 262144), (2, 1, 1000), (1, 3, 130), (2, 2, 777)])
def test_fp4_scores_match_oracle_on_dequantised_operands(csa, B, T, N):
    wl = synth.Workload(f"mx4_{B}_{T}_{N}", "bf16", B=B, ctx=4 * N + T, T=T, q_pos0=4 * N, ratio=4, N=N, H=64,
                        D=512, topk=min(N, 512))
    ix = synth.draw_indexer(wl, seed=N + T)
    q_pos = np.array([wl.q_pos] * B, np.int64)
    nv = oracle.n_visible(q_pos, 4, N)
    if B * T > 1:
        nv.reshape(-1)[-1] = N // 3                       # a ragged row
    q4, qsf = csa.csa_quantize_mxfp4_sf128(ix["qI"].cuda(), B)
    k4, ksf = csa.csa_quantize_mxfp4_sf128(ix["kI"].cuda(), B)
    s = csa.csa_index_scores(q4, ix["w"].cuda(), k4, torch.from_numpy(nv).cuda(), q_scale=qsf, k_scale=ksf,
                             mxfp4=True).cpu().numpy()
    _, _, qd = _operands(ix["qI"], B)
    _, _, kd = _operands(ix["kI"], B)
    ref, mag = oracle.index_scores(qd.astype(np.float32), ix["w"].numpy(), kd.astype(np.float32), nv, with_mag=True)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(s), fin)
    check_f32(s[fin], ref[fin], mag[fin], what=f"mxfp4 B={B} T={T} N={N}")


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_fp4_decode_topk_recall_after_rescoring(csa, name):
    """FP4 scores with the score histogram -> the candidates of the 4k-th score's bin,
    rescored exactly on the bf16 operands -> top-k; recall of the oracle's exact top-k."""
    wl = synth.WORKLOADS[name]
    ix = synth.draw_indexer(wl)
    q_pos = np.array([wl.q_pos] * wl.B, np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    g_nv = torch.from_numpy(nv).cuda()
    qI, kI, w = ix["qI"].cuda(), ix["kI"].cuda(), ix["w"].cuda()
    q4, qsf = csa.csa_quantize_mxfp4_sf128(qI, wl.B)
    k4, ksf = csa.csa_quantize_mxfp4_sf128(kI, wl.B)
    ws = csa.select_workspace(wl.B, wl.N)
    s4 = csa.csa_index_scores(q4, w, k4, g_nv, q_scale=qsf, k_scale=ksf, select_ws=ws, mxfp4=True)
    got = csa.csa_topk_select(s4, g_nv, wl.topk, ws, kc=4 * wl.topk, qI=qI, w=w, kI=kI).cpu().numpy()
    ref = oracle.index_scores(ix["qI"].float().numpy(), ix["w"].numpy(), ix["kI"].float().numpy(), nv)
    idx_ref = oracle.topk(ref.astype(np.float32), nv, wl.topk)
    recall = min(len(np.intersect1d(got[b, 0], idx_ref[b, 0])) / wl.topk for b in range(wl.B))
    print(f"{name} FP4 + 4k rescoring recall {recall:.4f}")
    assert recall >= 0.99
