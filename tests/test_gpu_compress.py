"""Compressor parity (GPU through the C ABI vs the CPU oracle), ragged and full-size cases."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import check_bf16_store, check_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _np(t):
    return t.float().numpy()


def _run_csa(csa, d, out_dtype, carry=True):
    g = {k: v.cuda() for k, v in d.items()}
    pc = g.get("prev_Cb") if carry else None
    pz = g.get("prev_Zb") if carry else None
    out = csa.csa_compress(g["C_a"], g["C_b"], g["Z_a"], g["Z_b"], pc, pz, ratio=4, out_dtype=out_dtype)
    ref, mag = oracle.compress_csa(_np(d["C_a"]), _np(d["C_b"]), _np(d["Z_a"]), _np(d["Z_b"]),
                                   prev_Cb=_np(d["prev_Cb"]) if carry and "prev_Cb" in d else None,
                                   prev_Zb=_np(d["prev_Zb"]) if carry and "prev_Zb" in d else None,
                                   with_mag=True)
    return out.float().cpu().numpy(), ref, mag


@pytest.mark.parametrize("dtype,out_dtype", [("f32", torch.float32), ("bf16", torch.bfloat16),
                                             ("bf16", torch.float32), ("f32", torch.bfloat16)])
@pytest.mark.parametrize("carry", [True, False])
def test_csa_ragged(csa, dtype, out_dtype, carry):
    wl = synth.Workload("ragged", dtype, B=3, ctx=4 * 37 + 3 + 40, T=1, q_pos0=4 * 37 + 3 + 39, ratio=4, N=64,
                        H=16, D=128, comp_L=4 * 37 + 3, comp_c=24)
    d = synth.draw_compressor(wl, seed=7)
    gpu, ref, mag = _run_csa(csa, d, out_dtype, carry)
    assert gpu.shape == (3, 37, 24)
    (check_f32 if out_dtype == torch.float32 else check_bf16_store)(gpu, ref, mag, what="csa ragged")


@pytest.mark.parametrize("name", ["tiny", "flash64k", "pro1m", "flash_prefill"])
def test_csa_workloads(csa, name):
    wl = synth.WORKLOADS[name]
    d = synth.draw_compressor(wl)
    out_dtype = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    gpu, ref, mag = _run_csa(csa, d, out_dtype)
    (check_f32 if wl.dtype == "f32" else check_bf16_store)(gpu, ref, mag, what=name)
    if wl.comp_ci:
        di = synth.draw_compressor(wl, c=wl.comp_ci, tag="index_keys")
        gpu, ref, mag = _run_csa(csa, di, out_dtype)
        check_bf16_store(gpu, ref, mag, what=name + " index keys")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_csa_wide_variant(csa, out_dtype):
    """Enough entries for the 8-channels-per-thread (16-byte load) variant: B = 4 sequences
    of a 4,096-token chunk at c = 512, with the carry."""
    wl = synth.Workload("csa_wide", "bf16", B=4, ctx=4096, T=1, q_pos0=4095, ratio=4, N=1024, H=16, D=128,
                        comp_L=4096, comp_c=512)
    d = synth.draw_compressor(wl, seed=19)
    gpu, ref, mag = _run_csa(csa, d, out_dtype, True)
    (check_f32 if out_dtype == torch.float32 else check_bf16_store)(gpu, ref, mag, what="csa wide")


def test_csa_chunked_equals_whole(csa):
    """Compressing in two chunks with the carry equals one pass, bit-exact on the GPU too."""
    wl = synth.Workload("chunk", "bf16", B=2, ctx=512, T=1, q_pos0=511, ratio=4, N=128, H=16, D=128,
                        comp_L=512, comp_c=64)
    d = {k: v.cuda() for k, v in synth.draw_compressor(wl, seed=3).items() if not k.startswith("prev")}
    whole = csa.csa_compress(d["C_a"], d["C_b"], d["Z_a"], d["Z_b"], ratio=4)
    L1 = 200
    first = csa.csa_compress(*(d[k][:, :L1].contiguous() for k in ("C_a", "C_b", "Z_a", "Z_b")), ratio=4)
    second = csa.csa_compress(*(d[k][:, L1:].contiguous() for k in ("C_a", "C_b", "Z_a", "Z_b")),
                              d["C_b"][:, L1 - 4:L1].contiguous(), d["Z_b"][:, L1 - 4:L1].contiguous(), ratio=4)
    assert torch.equal(torch.cat([first, second], 1), whole)


@pytest.mark.parametrize("dtype,c,L", [("bf16", 512, 128 * 5 + 77), ("f32", 128, 128 * 3), ("bf16", 256, 128 * 2)])
def test_hca_ragged(csa, dtype, c, L):
    wl = synth.Workload("hca_ragged", dtype, B=2, ctx=L, T=1, q_pos0=L - 1, ratio=128, N=8, H=16, D=128,
                        comp_L=L, comp_c=c)
    d = synth.draw_compressor(wl, seed=11)
    out = csa.csa_compress(d["C"].cuda(), None, d["Z"].cuda(), None, ratio=128, out_dtype=torch.float32)
    ref, mag = oracle.compress_hca(_np(d["C"]), _np(d["Z"]), with_mag=True)
    check_f32(out.cpu().numpy(), ref, mag, what="hca ragged")


def test_hca_full(csa):
    wl = synth.WORKLOADS["pro_hca"]
    d = synth.draw_compressor(wl)
    out = csa.csa_compress(d["C"].cuda(), None, d["Z"].cuda(), None, ratio=128)
    assert out.shape == (4, 128, 512) and out.dtype == torch.bfloat16
    ref, mag = oracle.compress_hca(_np(d["C"]), _np(d["Z"]), with_mag=True)
    check_bf16_store(out.float().cpu().numpy(), ref, mag, what="pro_hca compressor")


def test_compress_dominant_logit_selects_row(csa):
    """GPU side of the one-hot pin: a dominant logit returns that raw row exactly."""
    L, c = 64, 16
    Ca = synth.normal(5, "onehot/Ca", (1, L, c))
    Cb = synth.normal(5, "onehot/Cb", (1, L, c))
    Za = torch.zeros(1, L, c)
    Zb = torch.zeros(1, L, c)
    Zb[0, 4 * 5 + 2, :] = 80.0                       # entry 6, b position 2
    out = csa.csa_compress(Ca.cuda(), Cb.cuda(), Za.cuda(), Zb.cuda(), ratio=4).cpu()
    assert torch.allclose(out[0, 6], Cb[0, 22], rtol=0, atol=1e-30)
