"""Acceptance rules shared by the GPU parity tests.

fp32 stages (1e-5 relative): |gpu - ref| <= 1e-5 * mag, where mag is the
    oracle's forward-error scale of that output (sum of |terms|), so outputs that
    cancel to nearly zero are judged against the size of what was summed.
bf16-stored outputs of fp32 arithmetic (the compressor): the stored value must
    be a bf16 rounding (round-to-nearest-even) of some real within 1e-5 * mag of
    the exact result, i.e. RN(ref - tol) <= gpu <= RN(ref + tol).
bf16 attention: |gpu - ref| <= 2e-2 + 1e-2 * |ref|.
Indices: bit-exact.
"""
import numpy as np

F32_REL = 1e-5
ATTN_ABS, ATTN_REL = 2e-2, 1e-2


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def check_f32(gpu, ref, mag, rel=F32_REL, what=""):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    tol = rel * mag + 1e-30
    bad = ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside 1e-5*mag; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]!r} ref={ref[tuple(i)]!r} mag={mag[tuple(i)]!r}")


def check_bf16_store(gpu, ref, mag, rel=F32_REL, what=""):
    gpu = np.asarray(gpu, np.float64)
    tol = rel * mag
    lo, hi = bf16_round(ref - tol), bf16_round(ref + tol)
    bad = ~((gpu >= lo) & (gpu <= hi))
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} not a bf16 rounding of the exact value; "
                             f"first at {tuple(i)}: gpu={gpu[tuple(i)]!r} ref={ref[tuple(i)]!r}")


def check_attn_bf16(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    bad = ~(err <= ATTN_ABS + ATTN_REL * np.abs(ref))
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside abs 2e-2 + rel 1e-2; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]!r} ref={ref[tuple(i)]!r}; max err {err.max():.3g}")
