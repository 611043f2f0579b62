"""csa_compress_index_keys: a step's new index-key entries written straight into the
indexer's caches (bf16 keys for the exact rescoring, e4m3 codes and scales for the
low-precision scan).  Checked three ways:
  - the stored bf16 keys against the oracle compressor (bf16 rounding rule of reading c18);
  - the e4m3 codes and scales against the oracle quantiser (with the Hadamard rotation or
    without) applied to the oracle's own bf16 keys: bit for bit on every row whose stored
    keys reading c18 fixes uniquely; on the other rows (an element within 1e-5 * mag of a
    bf16 rounding boundary, e.g. entries that nearly cancel) every dequantised value must
    lie within one e4m3 step of the oracle's;
  - bit for bit against the unfused library path (csa_compress, then csa_quantize_e4m3),
    and rows outside [pos0, pos0 + L/4) left untouched."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import F32_REL, bf16_round, check_bf16_store

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _np(t):
    return t.float().numpy()


@pytest.mark.parametrize("name,B,L,dtype,carry,hadamard,ncap,pos0", [
    ("decode_flash", 8, 4, "bf16", True, True, 16384, 16383),       # one new entry per sequence
    ("decode_pro", 1, 512, "bf16", True, True, 262144, 262144 - 128),
    ("chunk", 2, 4 * 37 + 3, "bf16", False, False, 100, 5),         # entry 0 without a carry, partial block
    ("fp32_in", 3, 64, "f32", True, True, 40, 20),
    ("prefill", 1, 4096, "bf16", True, True, 32768, 32768 - 1024),
])
def test_compress_index_keys(csa, name, B, L, dtype, carry, hadamard, ncap, pos0):
    wl = synth.Workload(name, dtype, B=B, ctx=L + 4096, T=1, q_pos0=L + 4095, ratio=4, N=ncap, H=64, D=512,
                        comp_L=L, comp_c=128)
    d = synth.draw_compressor(wl, seed=5, tag="index_keys")
    g = {k: v.cuda() for k, v in d.items()}
    pc, pz = (g["prev_Cb"], g["prev_Zb"]) if carry else (None, None)
    n = L // 4
    sentinel = 0x3F80                                        # bf16 1.0 everywhere else
    kI = torch.full((B, ncap, 128), 1.0, dtype=torch.bfloat16, device="cuda")
    k8 = torch.full((B, ncap, 128), 0x55, dtype=torch.uint8, device="cuda")
    ks = torch.full((B, ncap), -3.0, dtype=torch.float32, device="cuda")
    csa.csa_compress_index_keys(g["C_a"], g["C_b"], g["Z_a"], g["Z_b"], pc, pz, kI, pos0=pos0, k8=k8, k_scale=ks,
                                hadamard=hadamard)
    # the unfused path through the library
    ref_kI = csa.csa_compress(g["C_a"], g["C_b"], g["Z_a"], g["Z_b"], pc, pz, ratio=4, out_dtype=torch.bfloat16)
    ref_k8, ref_ks = csa.csa_quantize_e4m3(ref_kI, hadamard=hadamard)
    sl = slice(pos0, pos0 + n)
    assert torch.equal(kI[:, sl], ref_kI) and torch.equal(k8[:, sl], ref_k8) and torch.equal(ks[:, sl], ref_ks)
    for a, b in ((0, pos0), (pos0 + n, ncap)):                # nothing else written
        assert bool((kI[:, a:b].view(torch.int16) == sentinel).all())
        assert bool((k8[:, a:b] == 0x55).all()) and bool((ks[:, a:b] == -3.0).all())
    # against the oracle
    ref, mag = oracle.compress_csa(_np(d["C_a"]), _np(d["C_b"]), _np(d["Z_a"]), _np(d["Z_b"]),
                                   prev_Cb=_np(d["prev_Cb"]) if carry else None,
                                   prev_Zb=_np(d["prev_Zb"]) if carry else None, with_mag=True)
    got = kI[:, sl].float().cpu().numpy()
    check_bf16_store(got, ref, mag, what=f"{name} stored keys")
    lo, hi = bf16_round(ref - F32_REL * mag), bf16_round(ref + F32_REL * mag)
    keys = bf16_round(ref).astype(np.float32)                # the oracle's own stored keys
    quant = oracle.quantize_rows_e4m3_hadamard if hadamard else oracle.quantize_rows_e4m3
    c_ref, s_ref = quant(keys)
    c_gpu, s_gpu = k8[:, sl].cpu().numpy(), ks[:, sl].cpu().numpy()
    amb = lo != hi                                           # elements with two admissible bf16 values
    unique = ~amb.any(-1)
    assert np.array_equal(c_gpu[unique], c_ref[unique]) and np.array_equal(s_gpu[unique], s_ref[unique])
    if (~unique).any():
        # each ambiguous stored key may sit anywhere in its admissible bf16 range; the
        # rotation spreads those ranges over the row (|H| = 1 / sqrt(128) per entry)
        width = (hi - lo)[~unique]
        slack = (width.sum(-1, keepdims=True) / np.sqrt(128.0)) if hadamard else width
        dq_gpu = oracle.e4m3_decode(c_gpu[~unique]) * s_gpu[~unique][:, None]
        dq_ref = oracle.e4m3_decode(c_ref[~unique]) * s_ref[~unique][:, None]
        smax = np.maximum(s_gpu[~unique], s_ref[~unique])[:, None]
        step = 0.125 * (np.maximum(np.abs(dq_ref), np.abs(dq_gpu)) + slack) + 2.0 ** -9 * smax * 1.001
        bad = np.abs(dq_gpu - dq_ref) > step + slack
        assert not bad.any(), (f"{bad.sum()} codes beyond the admissible keys' reach, e.g. gpu "
                               f"{dq_gpu[bad][:4]} ref {dq_ref[bad][:4]}")
        ds = np.abs(s_gpu[~unique] - s_ref[~unique])
        assert np.all(ds <= slack.max(-1) / 448.0 * 1.01 + 1e-6 * s_ref[~unique])


def test_compress_index_keys_bf16_only(csa):
    """Without e4m3 caches only the bf16 keys are written."""
    wl = synth.Workload("bf16_only", "bf16", B=2, ctx=8192, T=1, q_pos0=8191, ratio=4, N=64, H=64, D=512,
                        comp_L=32, comp_c=128)
    d = synth.draw_compressor(wl, seed=9, tag="index_keys")
    g = {k: v.cuda() for k, v in d.items()}
    kI = torch.zeros((2, 64, 128), dtype=torch.bfloat16, device="cuda")
    csa.csa_compress_index_keys(g["C_a"], g["C_b"], g["Z_a"], g["Z_b"], g["prev_Cb"], g["prev_Zb"], kI, pos0=56)
    ref = csa.csa_compress(g["C_a"], g["C_b"], g["Z_a"], g["Z_b"], g["prev_Cb"], g["prev_Zb"], ratio=4)
    assert torch.equal(kI[:, 56:], ref) and int(kI[:, :56].count_nonzero()) == 0
