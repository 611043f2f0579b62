"""MXFP4 operand quantiser (csa_quantize_mxfp4) against the CPU oracle, bit for bit: the
packed E2M1 codes and the E8M0 block scales, with and without the Hadamard rotation, on
ragged row counts, every supported width, both input types, rows built to land on the
rounding ties, zero and signed-zero rows, extreme magnitudes, and sampled rows of a
full-size decode key cache."""
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


def _pack(codes):
    """Oracle codes (one per byte) -> two per byte, value 2j in the low nibble."""
    c = codes.astype(np.uint8)
    return (c[..., 0::2] & 15) | ((c[..., 1::2] & 15) << 4)


def _same(csa, x, hadamard, what):
    codes, scales = csa.csa_quantize_mxfp4(x.cuda(), hadamard=hadamard)
    rc, rs = oracle.quantize_rows_mxfp4(x.float().numpy(), hadamard=hadamard)
    got_s, got_c = scales.cpu().numpy(), codes.cpu().numpy()
    assert np.array_equal(got_s, rs), f"{what}: {np.sum(got_s != rs)} scales differ"
    bad = np.argwhere(got_c != _pack(rc))
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first at {bad[0].tolist()}"


@pytest.mark.parametrize("cols", [32, 64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hadamard", [False, True])
def test_bit_exact_ragged(csa, cols, dtype, hadamard):
    for rows in (1, 333):
        x = synth.store(synth.normal(rows + cols, f"mx/{dtype}", (rows, cols), std=2.0), dtype)
        _same(csa, x, hadamard, f"rows={rows} cols={cols} {dtype} hadamard={hadamard}")


def test_ties_signs_and_extremes(csa):
    """Rows whose values sit exactly on the E2M1 rounding ties (block max 6 X), zero and
    negative-zero rows, a block with one huge value, subnormal fp32 values and the fp32
    extremes (scale exponent clamped at +-127)."""
    n = 128
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 6.0, 0.5, 1.0, 4.0, 0.1, 5.5, 2.9, 3.1])
    rows = []
    for k in (-10, 0, 3):
        r = np.resize(ties, n) * 2.0 ** k
        r[1::3] *= -1
        rows.append(r)
    rows.append(np.zeros(n))
    rows.append(-np.zeros(n))
    r = np.full(n, 1e-3)
    r[7] = 3e4
    rows.append(r)
    rows.append(np.resize([1e-40, -3e-39, 1e-45, 0.0], n))
    rows.append(np.resize([3.0e38, -1.0e38, 1.0, 2.0e-38], n))
    x = torch.from_numpy(np.array(rows, np.float32))
    _same(csa, x, False, "ties / extremes f32")
    _same(csa, synth.store(x, "bf16"), False, "ties / extremes bf16")
    _same(csa, synth.store(x[:6], "bf16"), True, "ties rotated bf16")


def test_empty_is_a_no_op(csa):
    codes, scales = csa.csa_quantize_mxfp4(torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"))
    assert codes.shape == (0, 64) and scales.shape == (0, 4)


def test_full_size_key_cache_sampled(csa):
    """The flash64k index-key cache ([8 x 16,384, 128] rows) in one launch, rotated; the
    oracle checks 2,048 sampled rows and the first and last rows."""
    wl = synth.WORKLOADS["flash64k"]
    flat = synth.draw_indexer(wl)["kI"].reshape(-1, 128)
    codes, scales = csa.csa_quantize_mxfp4(flat.cuda(), hadamard=True)
    rows = synth.random_subset(11, "mx/flash64k/rows", [flat.shape[0]], 2048)[0].numpy()
    rows = np.unique(np.concatenate([rows, [0, flat.shape[0] - 1]]))
    rc, rs = oracle.quantize_rows_mxfp4(flat[rows].float().numpy(), hadamard=True)
    assert np.array_equal(scales.cpu().numpy()[rows], rs)
    assert np.array_equal(codes.cpu().numpy()[rows], _pack(rc))
