"""Acceptance rules shared by the GPU parity tests.

fp32 stages (1e-5 relative): |gpu - ref| <= 1e-5 * mag, where mag is the
    oracle's forward-error scale of that output (sum of |terms|), so outputs that
    cancel to nearly zero are judged against the size of what was summed.
bf16-stored outputs of fp32 arithmetic (the compressor): the stored value must
    be a bf16 rounding (round-to-nearest-even) of some real within 1e-5 * mag of
    the exact result, i.e. RN(ref - tol) <= gpu <= RN(ref + tol).
bf16 attention: |gpu - ref| <= 2e-2 + 1e-2 * |ref|.
Indices: bit-exact.

Every fp32 check also reports the literal figure next to that reading: the largest
|gpu - ref| / |ref| over the outputs with |ref| >= 1e-2 * mag (outputs that are not
mostly cancellation).  check_f32(..., literal=True) asserts it is <= 1e-5 as well; the
reports are printed at the end of the pytest run (tests/conftest.py).
"""
import numpy as np

F32_REL = 1e-5
ATTN_ABS, ATTN_REL = 2e-2, 1e-2
LITERAL_FLOOR = 1e-2
REPORTS = []       # (what, max err/mag, max err/|ref| where |ref| >= 1e-2 mag, entries counted)


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def check_f32(gpu, ref, mag, rel=F32_REL, what="", literal=False):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.asarray(mag, np.float64)
    err = np.abs(gpu - ref)
    tol = rel * mag + 1e-30
    bad = ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside 1e-5*mag; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]!r} ref={ref[tuple(i)]!r} mag={mag[tuple(i)]!r}")
    sel = np.abs(ref) >= LITERAL_FLOOR * mag
    lit = float(np.max(err[sel] / np.abs(ref[sel]))) if sel.any() else 0.0
    c21 = float(np.max(err / (mag + 1e-300)))
    REPORTS.append((what, c21, lit, int(sel.sum())))
    if literal:
        assert lit <= rel, f"{what}: literal relative error {lit:.3g} > {rel} where |ref| >= 1e-2 mag"
    return lit


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


def check_topk_sets(gpu_idx, ref_scores, k, err_bound, what=""):
    """Index sets from scores that carry rounding error: the GPU set may differ from the
    exact top-k only at entries whose exact score is within the error window of the
    k-th largest exact score (|s_i - s_k| <= max(1e-6 |s_k|, 2 E), E = measured max
    score error).  gpu_idx [k] (ascending, -1 padded), ref_scores [n] exact scores."""
    s = np.asarray(ref_scores, np.float64)
    order = np.lexsort((np.arange(s.size), -s))
    ref = np.sort(order[:k])
    sk = s[order[min(k, s.size) - 1]]
    win = max(1e-6 * abs(sk), 2.0 * err_bound)
    g = np.asarray([i for i in gpu_idx if i >= 0])
    assert len(set(g.tolist())) == len(g), f"{what}: duplicate indices"
    assert np.all(np.diff(g) > 0), f"{what}: not ascending"
    diff = np.setxor1d(g, ref)
    bad = [int(i) for i in diff if abs(s[i] - sk) > win]
    assert not bad, f"{what}: {len(bad)} indices differ beyond the tie window (e.g. {bad[:5]}, window {win:.3g})"
    return len(np.intersect1d(g, ref)) / max(1, min(k, s.size))
