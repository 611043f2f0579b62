"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test fixes the oracle to something other than itself: the worked example
and entry counts printed in "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" (§3, §4.1),
closed forms, invariants, library routines for special cases (numpy stable
sort, torch scaled_dot_product_attention in float64, numpy matmul), and brute
force over all subsets on tiny inputs.  Each is chosen so that a plausible slip
in the oracle (a dropped branch, an off-by-one row, a transposed operand, a
wrong sign) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth

RNG = np.random.default_rng(1234)


def rnd(*shape, scale=1.0):
    return (RNG.standard_normal(shape) * scale).astype(np.float32)


# ----------------------------------------------------------------------------- compressor
def test_worked_example_alpha(golden):
    """§4.1: logits log([1,2,1,2,4,2,1,3]) give alpha = [1,2,1,2,4,2,1,3]/16.

    Entry i=1 of a two-block sequence: positions 0..3 are the b-branch rows 0..3
    (block 0), positions 4..7 the a-branch rows 4..7 (block 1).  Channel j holds
    one-hot contents selecting position j, so out[1, j] = alpha_j."""
    g = golden("worked_example_alpha.json")
    w = np.array(g["weights"], np.float64)
    m, L, c = 4, 8, 8
    Zb = np.zeros((L, c), np.float32)
    Za = np.zeros((L, c), np.float32)
    Cb = np.zeros((L, c), np.float32)
    Ca = np.zeros((L, c), np.float32)
    for r in range(m):
        Zb[r, :] = np.log(w[r])
        Za[m + r, :] = np.log(w[m + r])
        Cb[r, r] = 1.0
        Ca[m + r, m + r] = 1.0
    out = oracle.compress_csa(Ca, Cb, Za, Zb, m=m)
    expect = np.array(g["alpha_times_16"], np.float64) / g["denominator"]
    # log() of the weights is rounded to fp32 on input: allow that rounding only.
    np.testing.assert_allclose(out[1], expect, rtol=0, atol=1e-7)
    assert abs(out[1].sum() - 1.0) < 1e-12


def test_compress_row_mapping_one_hot():
    """A dominant logit at one of the 2m rows selects exactly that row's content:
    pins which raw rows (b: (i-1)m..im-1, a: im..(i+1)m-1) feed entry i."""
    m, L, c = 4, 24, 3
    Ca, Cb = rnd(L, c), rnd(L, c)
    for i in range(1, L // m):
        for branch in ("a", "b"):
            for r in range(m):
                Za = np.zeros((L, c), np.float32)
                Zb = np.zeros((L, c), np.float32)
                row = i * m + r if branch == "a" else (i - 1) * m + r
                (Za if branch == "a" else Zb)[row, :] = 80.0
                out = oracle.compress_csa(Ca, Cb, Za, Zb, m=m)
                src = Ca if branch == "a" else Cb
                np.testing.assert_allclose(out[i], src[row], rtol=0, atol=1e-20 + 1e-30)


def test_compress_channels_independent():
    """Each channel has its own softmax: channel j one-hot at a different position."""
    m, L, c = 4, 8, 8
    Ca, Cb = rnd(L, c), rnd(L, c)
    Za = np.zeros((L, c), np.float32)
    Zb = np.zeros((L, c), np.float32)
    for j in range(c):
        if j < m:
            Zb[j, j] = 90.0
        else:
            Za[j, j] = 90.0
    out = oracle.compress_csa(Ca, Cb, Za, Zb, m=m)
    for j in range(c):
        src = Cb if j < m else Ca
        assert out[1, j] == pytest.approx(float(src[j, j]), abs=1e-30)


def test_compress_invariants():
    m, L, c = 4, 64, 16
    Za, Zb = rnd(L, c, scale=3.0), rnd(L, c, scale=3.0)
    # constant content along each channel -> that constant (sum alpha = 1)
    const = rnd(1, c)
    out = oracle.compress_csa(np.repeat(const, L, 0), np.repeat(const, L, 0), Za, Zb, m=m)
    np.testing.assert_allclose(out, np.repeat(const.astype(np.float64), L // m, 0), rtol=1e-6)
    # constant logits -> plain mean of the 2m rows (entry 0: of its m a-rows)
    Ca, Cb = rnd(L, c), rnd(L, c)
    zero = np.zeros((L, c), np.float32)
    out = oracle.compress_csa(Ca, Cb, zero, zero, m=m)
    for i in range(L // m):
        rows = [Ca[i * m:(i + 1) * m]] + ([Cb[(i - 1) * m:i * m]] if i > 0 else [])
        expect = np.concatenate(rows).astype(np.float64).mean(0)
        np.testing.assert_allclose(out[i], expect, rtol=1e-12, atol=1e-12)
    # convexity: output lies within [min, max] of the 2m contributing rows
    out = oracle.compress_csa(Ca, Cb, Za, Zb, m=m)
    for i in range(1, L // m):
        rows = np.concatenate([Cb[(i - 1) * m:i * m], Ca[i * m:(i + 1) * m]])
        assert np.all(out[i] <= rows.max(0) + 1e-12) and np.all(out[i] >= rows.min(0) - 1e-12)


def test_compress_first_entry_is_a_branch_softmax():
    """Entry 0 without a carry reduces to softmax over its m a-rows (torch.softmax in float64)."""
    m, L, c = 4, 16, 8
    Ca, Cb, Za, Zb = rnd(L, c), rnd(L, c), rnd(L, c), rnd(L, c)
    out = oracle.compress_csa(Ca, Cb, Za, Zb, m=m)
    a = torch.softmax(torch.from_numpy(Za[:m].astype(np.float64)), dim=0)
    expect = (a * torch.from_numpy(Ca[:m].astype(np.float64))).sum(0).numpy()
    np.testing.assert_allclose(out[0], expect, rtol=1e-12, atol=1e-14)


def test_compress_carry_chunked_equals_whole():
    """compress(0..L) == compress(0..L1) ++ compress(L1..L, carry = b rows of block L1/m - 1), bit-exact."""
    m, L, c = 4, 64, 8
    Ca, Cb, Za, Zb = rnd(L, c), rnd(L, c), rnd(L, c), rnd(L, c)
    whole = oracle.compress_csa(Ca, Cb, Za, Zb, m=m)
    L1 = 24
    first = oracle.compress_csa(Ca[:L1], Cb[:L1], Za[:L1], Zb[:L1], m=m)
    second = oracle.compress_csa(Ca[L1:], Cb[L1:], Za[L1:], Zb[L1:],
                                 prev_Cb=Cb[L1 - m:L1], prev_Zb=Zb[L1 - m:L1], m=m)
    assert np.array_equal(np.concatenate([first, second]), whole)


def test_compress_partial_block_dropped():
    m, c = 4, 4
    Ca, Cb, Za, Zb = rnd(10, c), rnd(10, c), rnd(10, c), rnd(10, c)
    assert oracle.compress_csa(Ca, Cb, Za, Zb, m=m).shape == (2, c)


def test_hca_compress_pins():
    m, L, c = 128, 384, 8
    C = rnd(L, c)
    zero = np.zeros((L, c), np.float32)
    out = oracle.compress_hca(C, zero, m=m)
    np.testing.assert_allclose(out, C.astype(np.float64).reshape(3, m, c).mean(1), rtol=1e-12, atol=1e-13)
    # a dominant logit selects its row; blocks do not overlap
    Z = rnd(L, c)
    Z[128 + 37, 2] = 200.0
    out = oracle.compress_hca(C, Z, m=m)
    assert out[1, 2] == pytest.approx(float(C[128 + 37, 2]), abs=1e-30)
    Z2 = Z.copy()
    Z2[:128] += rnd(128, c)   # perturb block 0 only
    C2 = C.copy()
    C2[256:] += 1.0           # and block 2's contents
    out2 = oracle.compress_hca(C2, Z2, m=m)
    assert np.array_equal(out2[1], out[1])
    # softmax over a block equals torch.softmax (library routine) weighted sum
    b = torch.softmax(torch.from_numpy(Z[256:384].astype(np.float64)), 0)
    np.testing.assert_allclose(out[2], (b * torch.from_numpy(C[256:384].astype(np.float64))).sum(0).numpy(),
                               rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- counts / causality
def test_entry_counts(golden):
    g = golden("entry_counts.json")
    n = g["n"]
    assert oracle.n_visible([n - 1], 4, 1 << 40)[0] == g["csa_entries"]
    assert oracle.n_visible([n - 1], 128, 1 << 40)[0] == g["hca_entries"]
    assert g["topk"]["flash"] + g["swa_window"] == g["working_set_rows"]["flash_csa"]
    assert g["topk"]["pro"] + g["swa_window"] == g["working_set_rows"]["pro_csa"]
    assert g["hca_entries"] + g["swa_window"] == g["working_set_rows"]["hca"]
    wl = synth.WORKLOADS["pro1m"]
    assert wl.N == g["csa_entries"] and wl.topk == g["topk"]["pro"]
    assert synth.WORKLOADS["pro_hca"].N == g["hca_entries"]


def test_tiny_n_valid(golden):
    g = golden("tiny_n_valid.json")
    assert oracle.n_visible(g["q_pos"], g["ratio"], 1024).tolist() == g["n_valid"]
    # the boundary itself: entry i becomes visible exactly at t = (i+1)m - 1
    for i in range(5):
        t = (i + 1) * 4 - 1
        assert oracle.n_visible([t - 1, t], 4, 100).tolist() == [i, i + 1]


# ----------------------------------------------------------------------------- indexer
def _index_inputs(T=3, N=50, Hi=64, d=128):
    return rnd(1, T, Hi, d), rnd(1, T, Hi), rnd(1, N, d)


def test_index_relu_split_reduces_to_matmul():
    """ReLU(x) - ReLU(-x) = x, so s(q) - s(-q) = sum_h w_h <q_h, k_i> = numpy matmul."""
    qI, w, kI = _index_inputs()
    nv = np.array([[50, 50, 50]], np.int32)
    s_pos = oracle.index_scores(qI, w, kI, nv)
    s_neg = oracle.index_scores(-qI, w, kI, nv)
    lin = np.einsum("th,thd->td", w[0].astype(np.float64), qI[0].astype(np.float64)) @ kI[0].astype(np.float64).T
    np.testing.assert_allclose(s_pos[0] - s_neg[0], lin, rtol=1e-10, atol=1e-9)
    # and s(q) + s(-q) = sum_h w_h |<q_h, k_i>|
    dots = np.einsum("thd,nd->thn", qI[0].astype(np.float64), kI[0].astype(np.float64))
    np.testing.assert_allclose(s_pos[0] + s_neg[0], np.einsum("th,thn->tn", w[0], np.abs(dots)),
                               rtol=1e-10, atol=1e-9)


def test_index_unit_vectors_closed_form():
    """q_{t,h} = e_{a_h}, k_i = e_{b_i}: s_{t,i} = sum_h w_h [a_h == b_i]; also a negative dot contributes 0."""
    Hi, d, N = 64, 128, 20
    a = RNG.integers(0, d, Hi)
    b = RNG.integers(0, d, N)
    q = np.zeros((1, 1, Hi, d), np.float32)
    q[0, 0, np.arange(Hi), a] = 1.0
    k = np.zeros((1, N, d), np.float32)
    k[0, np.arange(N), b] = -1.0
    w = rnd(1, 1, Hi)
    s = oracle.index_scores(q, w, k, np.array([[N]], np.int32))
    assert np.all(s == 0.0)
    s = oracle.index_scores(q, w, -k, np.array([[N]], np.int32))
    expect = np.array([w[0, 0][a == b[i]].astype(np.float64).sum() for i in range(N)])
    np.testing.assert_allclose(s[0, 0], expect, rtol=1e-15, atol=1e-15)


def test_index_rotation_invariance_and_causal_tail():
    """A shared orthogonal rotation of q and k leaves scores unchanged; i >= n_valid is -inf."""
    qI, w, kI = _index_inputs(T=2, N=40)
    Q, _ = np.linalg.qr(RNG.standard_normal((128, 128)))
    nv = np.array([[40, 17]], np.int32)
    s0 = oracle.index_scores(qI.astype(np.float64), w, kI.astype(np.float64), nv)
    s1 = oracle.index_scores((qI.astype(np.float64) @ Q), w, (kI.astype(np.float64) @ Q), nv)
    # rotated inputs are rounded to fp32 on the way in; compare at that precision
    mag = oracle.index_scores(np.abs(qI), np.abs(w), np.abs(kI), np.array([[40, 40]], np.int32))
    assert np.all(np.abs(s0[0, 0] - s1[0, 0]) <= 1e-5 * mag[0, 0] + 1e-6)
    assert np.all(np.isneginf(s0[0, 1, 17:])) and np.all(np.isfinite(s0[0, 1, :17]))


# ----------------------------------------------------------------------------- e4m3
def test_e4m3_codec_points(golden):
    g = golden("e4m3_points.json")
    for code, val in g["decode"]:
        got = oracle.e4m3_decode([code])[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val)
    for x, code in g["encode_ties_to_even"]:
        assert oracle.e4m3_encode([x])[0] == code, x
    for code in g["nan_codes"]:
        assert np.isnan(oracle.e4m3_decode([code])[0])


def test_e4m3_roundtrip_and_monotone():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_decode(codes)
    back = oracle.e4m3_encode(vals.astype(np.float32))
    assert np.array_equal(back, codes)
    pos = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    # nearest: a random value's code is at least as close as both neighbours
    x = (RNG.standard_normal(2000) * 50).astype(np.float32)
    enc = oracle.e4m3_decode(oracle.e4m3_encode(x))
    sorted_vals = np.sort(vals[np.isfinite(vals)])
    for xv, ev in zip(x.astype(np.float64), enc):
        if abs(xv) >= 448:
            assert abs(ev) == 448
            continue
        best = np.min(np.abs(sorted_vals - xv))
        assert abs(ev - xv) == best


def test_quantize_rows():
    x = rnd(6, 128, scale=3.0)
    x[3] = 0.0
    codes, scale = oracle.quantize_rows_e4m3(x)
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    for r in (0, 1, 2, 4, 5):
        amax = np.float32(np.abs(x[r]).max())
        assert scale[r] == np.float32(amax / np.float32(448.0))
        j = int(np.abs(x[r]).argmax())
        assert codes[r, j] & 0x7F == 0x7E
    deq = oracle.e4m3_decode(codes) * scale[:, None]
    # relative error bound of e4m3 rounding (3 mantissa bits): half an ulp, 2^-4 relative for normals
    big = np.abs(x) >= scale[:, None] * 2 ** -6
    assert np.all(np.abs(deq - x)[big] <= 2 ** -4 * np.abs(x)[big] * (1 + 1e-6))


def test_index_e4m3_matches_dequantised_f32():
    """With power-of-two scales the dequantised values are exact in fp32, so the e4m3
    definition must equal the (pinned) fp32 definition on those values."""
    T, N, Hi, d = 2, 30, 64, 128
    q8 = RNG.integers(0, 256, (1, T, Hi, d)).astype(np.uint8)
    k8 = RNG.integers(0, 256, (1, N, d)).astype(np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0
    k8[(k8 & 0x7F) == 0x7F] = 0
    qs = (2.0 ** RNG.integers(-8, -2, (1, T, Hi))).astype(np.float32)
    ks = (2.0 ** RNG.integers(-8, -2, (1, N))).astype(np.float32)
    w = rnd(1, T, Hi)
    nv = np.array([[N, 11]], np.int32)
    s8 = oracle.index_scores_e4m3(q8, qs, w, k8, ks, nv)
    qf = (oracle.e4m3_decode(q8) * qs[..., None]).astype(np.float32)
    kf = (oracle.e4m3_decode(k8) * ks[..., None]).astype(np.float32)
    sf = oracle.index_scores(qf, w, kf, nv)
    np.testing.assert_array_equal(np.isneginf(s8), np.isneginf(sf))
    fin = np.isfinite(sf)
    np.testing.assert_allclose(s8[fin], sf[fin], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- top-k
def _brute_topk(s, nv, k):
    """The unique k-subset S where every member beats every non-member
    (greater score, or equal score and lower index)."""
    cand = range(nv)
    take = min(k, nv)
    for S in itertools.combinations(cand, take):
        Sset = set(S)
        if all((s[i] > s[j]) or (s[i] == s[j] and i < j) for i in Sset for j in cand if j not in Sset):
            return sorted(S) + [-1] * (k - take)
    raise AssertionError("no valid subset")


def test_topk_brute_force_tiny():
    for trial in range(60):
        N = int(RNG.integers(1, 11))
        k = int(RNG.integers(1, 6))
        nv = int(RNG.integers(0, N + 1))
        s = RNG.integers(-3, 4, N).astype(np.float32)       # many exact ties
        if trial % 3 == 0:
            s[s == 0] = -0.0                                  # -0.0 ties +0.0
        got = oracle.topk(s[None, None], [[nv]], k)[0, 0].tolist()
        assert got == _brute_topk(s.astype(np.float64), nv, k), (s, nv, k)


def test_topk_matches_stable_sort_on_tiny_rows():
    """All tiny-workload-sized rows: numpy stable argsort (library routine) of -s, first k, ascending."""
    s = synth.draw_scores(0, "pin/topk", 1, 8, 1024, ties=6).numpy()
    nv = oracle.n_visible(list(range(4088, 4096)), 4, 1024)[None]
    got = oracle.topk(s, nv, 64)
    for t in range(8):
        row = s[0, t, :nv[0, t]].astype(np.float64) + 0.0    # +0.0 folds -0.0
        order = np.argsort(-row, kind="stable")[:64]
        assert got[0, t].tolist() == sorted(order.tolist())


# ----------------------------------------------------------------------------- attention
def _sdpa_with_sink(q, rows, sink, scale):
    """torch scaled_dot_product_attention in float64 over [sink slot; rows]: the sink
    is a key with logit z_s (an additive mask on a zero key) and a zero value."""
    H, D = q.shape
    qt = torch.from_numpy(q.astype(np.float64))[:, None, :]                         # [H, 1, D]
    keys = torch.cat([torch.zeros(1, D, dtype=torch.float64), torch.from_numpy(rows.astype(np.float64))])
    kt = keys[None].expand(H, -1, -1)
    mask = torch.zeros(H, 1, keys.shape[0], dtype=torch.float64)
    mask[:, 0, 0] = torch.from_numpy(sink.astype(np.float64))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=mask, scale=scale)
    return o[:, 0, :].numpy()


def test_sparse_attn_matches_sdpa_with_sink():
    H, D, N, k = 4, 32, 40, 12
    T = 3
    q = rnd(1, T, H, D)
    kv = rnd(1, N, D)
    q_pos = np.array([[300, 301, 302]])
    swa_pos0 = 300 - 127
    swa = rnd(1, 130, D)
    sink = rnd(H)
    idx = np.stack([np.sort(RNG.choice(N, k, replace=False)) for _ in range(T)]).astype(np.int32)[None]
    idx[0, 1, -3:] = -1                                   # padding contributes nothing
    scale = 1 / math.sqrt(D)
    out = oracle.sparse_attn(q, kv, swa, [swa_pos0], q_pos, sink, idx, scale)
    for t in range(T):
        p = q_pos[0, t]
        swa_rows = swa[0, (p - 127 - swa_pos0):(p - swa_pos0 + 1)]
        sel = kv[0, [i for i in idx[0, t] if i >= 0]]
        ref = _sdpa_with_sink(q[0, t], np.concatenate([swa_rows, sel]), sink, scale)
        np.testing.assert_allclose(out[0, t], ref, rtol=1e-12, atol=1e-13)


def test_attention_sink_closed_form():
    """Equal logits z on L rows: p = e^z / (e^{z_s} + L e^z); with all rows v, o = L p v."""
    H, D, N = 3, 16, 20
    v = rnd(D)
    kv = np.repeat(v[None], N, 0)[None]
    swa = np.repeat(v[None], 128, 0)[None]
    q = np.zeros((1, 1, H, D), np.float32)                # z = 0 for every row
    sink = np.array([-1.0, 0.5, 2.0], np.float32)
    k = 7
    idx = np.arange(k, dtype=np.int32)[None, None]
    out = oracle.sparse_attn(q, kv, swa, [1000 - 127], [[1000]], sink, idx, 0.1)
    L = k + 128
    for h in range(H):
        p = 1.0 / (math.exp(float(sink[h])) + L)
        np.testing.assert_allclose(out[0, 0, h], L * p * v.astype(np.float64), rtol=1e-13)


def test_sparse_attn_causal_window_and_poison():
    """SWA rows outside t-127..t and unselected entries are never read: NaN there changes nothing."""
    H, D, N, k = 2, 16, 30, 5
    q = rnd(1, 2, H, D)
    kv = rnd(1, N, D)
    swa = rnd(1, 300, D)
    sink = rnd(H)
    q_pos = np.array([[500, 520]])
    swa_pos0 = 400
    idx = np.array([[[1, 4, 9, 20, 29], [0, 2, 3, -1, -1]]], np.int32)
    ref = oracle.sparse_attn(q, kv, swa, [swa_pos0], q_pos, sink, idx, 0.25)
    kv2, swa2 = kv.copy(), swa.copy()
    used = {1, 4, 9, 20, 29, 0, 2, 3}
    for i in range(N):
        if i not in used:
            kv2[0, i] = np.nan
    for r in range(300):
        p = swa_pos0 + r
        if not (500 - 127 <= p <= 520):
            swa2[0, r] = np.nan
    got = oracle.sparse_attn(q, kv2, swa2, [swa_pos0], q_pos, sink, idx, 0.25)
    assert np.array_equal(got, ref)
    # the window is exactly 128 rows: query 500 must not see position 500-128
    swa3 = swa.copy()
    swa3[0, 500 - 128 - swa_pos0] = np.nan
    assert np.all(np.isfinite(oracle.sparse_attn(q[:, :1], kv, swa3, [swa_pos0], q_pos[:, :1], sink,
                                                 idx[:, :1], 0.25)))


def test_hca_equals_sparse_with_all_entries_and_sdpa():
    H, D, N = 4, 32, 10
    q = rnd(2, 1, H, D)
    kv = rnd(2, N, D)
    swa = rnd(2, 128, D)
    sink = rnd(H)
    t = 128 * 7 + 5                                       # 7 complete blocks
    q_pos = np.array([[t], [t]])
    swa_pos0 = [t - 127, t - 127]
    hca = oracle.hca_attn(q, kv, swa, swa_pos0, q_pos, sink, 0.2, ratio=128)
    idx = np.full((2, 1, N), -1, np.int32)
    idx[:, 0, :7] = np.arange(7)
    sp = oracle.sparse_attn(q, kv, swa, swa_pos0, q_pos, sink, idx, 0.2)
    np.testing.assert_allclose(hca, sp, rtol=1e-14, atol=1e-15)
    kv_poison = kv.copy()
    kv_poison[:, 7:] = np.nan                             # incomplete / future summaries
    assert np.array_equal(oracle.hca_attn(q, kv_poison, swa, swa_pos0, q_pos, sink, 0.2, ratio=128), hca)
    ref = _sdpa_with_sink(q[0, 0], np.concatenate([swa[0], kv[0, :7]]), sink, 0.2)
    np.testing.assert_allclose(hca[0, 0], ref, rtol=1e-12, atol=1e-13)


def test_sink_minus_infinity_is_textbook_softmax():
    H, D = 2, 8
    q = rnd(1, 1, H, D)
    kv = rnd(1, 6, D)
    swa = rnd(1, 128, D)
    sink = np.full(H, -1e30, np.float32)
    idx = np.arange(6, dtype=np.int32)[None, None]
    out = oracle.sparse_attn(q, kv, swa, [0], [[127]], sink, idx, 0.3)
    rows = torch.from_numpy(np.concatenate([swa[0], kv[0]]).astype(np.float64))
    qt = torch.from_numpy(q[0, 0].astype(np.float64))
    ref = torch.softmax(0.3 * qt @ rows.T, dim=-1) @ rows
    np.testing.assert_allclose(out[0, 0], ref.numpy(), rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- generator
def test_generator_splitmix_reference(golden):
    g = golden("splitmix64_seed0.json")
    got = [format(v & ((1 << 64) - 1), "016x") for v in synth.raw_u64(g["state"], 0, 3).tolist()]
    assert got == g["outputs_hex"]
    key = synth.stream_key(0, "abc")
    ints = [synth._mix_int(key + (i + 1) * synth._GOLDEN) for i in range(1000, 1010)]
    assert [v & ((1 << 64) - 1) for v in synth.raw_u64(key, 1000, 10).tolist()] == ints


def test_generator_moments_and_independence():
    x = synth.normal(0, "moments", (200000,)).double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01
    y = synth.normal(0, "moments2", (200000,)).double()
    assert abs(torch.corrcoef(torch.stack([x, y]))[0, 1].item()) < 0.01
    u = synth.uniform(0, "u", (200000,)).double()
    assert 0 <= u.min().item() and u.max().item() < 1 and abs(u.mean().item() - 0.5) < 0.01
    # order-independence: drawing a prefix gives the same values
    assert torch.equal(synth.normal(3, "p", (10,)), synth.normal(3, "p", (1000,))[:10])


# ----------------------------------------------------------------------------- mixed-precision KV storage
def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def test_kv8_worked_block_and_layout():
    """[HA] §4.2 storage precision, on D = 128 (one FP8 block of 64 dims + 64 BF16 RoPE dims).

    Hand-derived expectations:
      - amax = 448 gives the scale 2^0 = 1.  Codes: 448 = 1.75 * 2^8 -> 0 1111 110 = 0x7E;
        -1.0 = 2^0 -> 1 0111 000 = 0xB8; 0.5 = 2^-1 -> 0 0110 000 = 0x30;
        3.0 = 1.5 * 2^1 -> 0 1000 100 = 0x44; 0 -> 0x00.
      - amax = 452 (a BF16 value) needs 2^1: 452 / 2 = 226 lies between 224 (0x76) and
        240 (0x77), so the code is 0x76, which decodes back to 448.
      - amax = 2^-10 (0.0009765625) gives e = ceil(log2(2^-10 / 448)) = -18: 448 * 2^-18 >= 2^-10
        and 448 * 2^-19 < 2^-10.  Then 2^-10 / 2^-18 = 256 = 2^8 -> 0 1111 000 = 0x78.
      - Layout: 64 codes, then 64 BF16 RoPE values, then one fp32 scale, zero padding to 208 bytes.
    """
    assert oracle.kv8_entry_bytes(128) == 208
    assert oracle.kv8_entry_bytes(512) == 608
    rope = _bf16(np.linspace(-3, 3, 64))
    x = np.zeros((3, 128), np.float32)
    x[0, :5] = [448.0, -1.0, 0.5, 3.0, 0.0]
    x[1, 0] = 452.0
    x[2, 7] = 2.0 ** -10
    x[:, 64:] = rope
    e = oracle.kv8_quantize(x)
    assert e.shape == (3, 208)
    assert list(e[0, :5]) == [0x7E, 0xB8, 0x30, 0x44, 0x00]
    assert np.all(e[0, 5:64] == 0)
    assert e[0, 64:192].view(np.uint16).tolist() == (rope.view(np.uint32) >> 16).astype(np.uint16).tolist()
    scales = [float(e[r, 192:196].view(np.float32)[0]) for r in range(3)]
    assert scales == [1.0, 2.0, 2.0 ** -18]
    assert np.all(e[:, 196:] == 0)
    assert e[1, 0] == 0x76 and e[2, 7] == 0x78
    y = oracle.kv8_dequantize(e, 128)
    assert y[0, :5].tolist() == [448.0, -1.0, 0.5, 3.0, 0.0]
    assert y[1, 0] == 448.0 and y[2, 7] == 2.0 ** -10
    np.testing.assert_array_equal(y[:, 64:], x[:, 64:])


def test_kv8_scale_is_the_smallest_power_of_two():
    """s = 2^e with amax <= 448 s < 2 amax (e minimal), per block of 64 dims; zero block -> 1."""
    D = 512
    mags = [1e-6, 3e-3, 0.7, 1.0, 5.0, 448.0, 449.0, 3e4]
    x = np.zeros((len(mags) + 1, D), np.float32)
    for r, mg in enumerate(mags):
        x[r] = _bf16(rnd(D) * mg)
    x[-1, :448] = 0.0                                    # all FP8 blocks zero
    e = oracle.kv8_quantize(x)
    for r in range(x.shape[0]):
        sc = e[r, 448 + 128:448 + 128 + 28].view(np.float32)
        for blk in range(7):
            s = float(sc[blk])
            m, ex = math.frexp(s)
            assert m == 0.5, (r, blk, s)                 # a power of two
            amax = float(np.abs(x[r, blk * 64:(blk + 1) * 64]).max())
            if amax == 0.0:
                assert s == 1.0
            else:
                assert amax <= 448.0 * s and amax > 224.0 * s, (r, blk, amax, s)


def test_kv8_exact_roundtrip_of_every_code():
    """Values code * s for every finite e4m3 code come back with the same code."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes)
    for s in (2.0 ** -12, 1.0, 2.0 ** 5):
        x = np.zeros((len(codes), 128), np.float32)
        x[:, 0] = (vals * s).astype(np.float32)
        x[:, 1] = 448.0 * s                                # pins the block's scale to s
        e = oracle.kv8_quantize(x)
        np.testing.assert_array_equal(e[:, 0], codes)
        assert np.all(e[:, 192:196].view(np.float32) == np.float32(s))
        y = oracle.kv8_dequantize(e, 128)
        np.testing.assert_array_equal(y[:, 0], x[:, 0])


def test_kv8_error_bound_and_block_independence():
    """|x - x'| <= max(|x| 2^-4, s 2^-10) (half an e4m3 step); blocks quantise independently;
    the RoPE dims are bit-exact."""
    D = 512
    x = _bf16(rnd(64, D) * np.exp(rnd(64, 1) * 2))
    e = oracle.kv8_quantize(x)
    y = oracle.kv8_dequantize(e, D)
    sc = e[:, 576:604].view(np.float32)                  # [64, 7]
    s_full = np.repeat(sc, 64, axis=1)
    err = np.abs(x[:, :448].astype(np.float64) - y[:, :448])
    bound = np.maximum(np.abs(x[:, :448]) * 2.0 ** -4, s_full * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-12))
    np.testing.assert_array_equal(y[:, 448:], x[:, 448:])
    x2 = x.copy()
    x2[:, 64:128] *= 16.0                                # change block 1 only
    e2 = oracle.kv8_quantize(x2)
    np.testing.assert_array_equal(e2[:, :64], e[:, :64])
    np.testing.assert_array_equal(e2[:, 128:448], e[:, 128:448])
    assert np.all(e2[:, 580:584].view(np.float32) == e[:, 580:584].view(np.float32) * 16)


# ----------------------------------------------------------------------------- sharded decode pieces
@pytest.mark.parametrize("G", [1, 2, 3, 5])
def test_partial_pieces_recombine_to_full_attention(G):
    """Rows split into G disjoint sets (the SWA rows in set 0, memory rows by a contiguous
    partition of the entries, some sets empty): combining the per-set (m, l, o) with the
    sink added once gives the full attention, checked against the full oracle and against
    torch scaled_dot_product_attention (float64) with the sink as an extra zero row."""
    H, D, N, k, T = 4, 32, 60, 16, 2
    q = rnd(1, T, H, D)
    kv = rnd(1, N, D)
    swa = rnd(1, 130, D)
    sink = rnd(H)
    q_pos, swa_pos0 = np.array([[400, 401]]), 400 - 127
    idx = np.stack([np.sort(RNG.choice(N, k, replace=False)) for _ in range(T)]).astype(np.int32)[None]
    idx[0, 1, -2:] = -1
    scale = 1 / math.sqrt(D)
    bounds = np.linspace(0, N, G + 1).astype(int)
    if G == 3:
        bounds = np.array([0, 0, 30, N])                 # an empty shard
    ms, ls, os_ = [], [], []
    for g in range(G):
        part = np.where((idx >= bounds[g]) & (idx < bounds[g + 1]), idx, -1).astype(np.int32)
        m, l, o = oracle.sparse_attn_partial(q, kv, swa, [swa_pos0], q_pos, part, scale, with_swa=(g == 0))
        ms.append(m); ls.append(l); os_.append(o)
    out = oracle.attn_combine(np.stack(ms), np.stack(ls), np.stack(os_), sink)
    full = oracle.sparse_attn(q, kv, swa, [swa_pos0], q_pos, sink, idx, scale)
    np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-13)
    for t in range(T):
        p = q_pos[0, t]
        rows = np.concatenate([swa[0, (p - 127 - swa_pos0):(p - swa_pos0 + 1)], kv[0, [i for i in idx[0, t] if i >= 0]]])
        np.testing.assert_allclose(out[0, t], _sdpa_with_sink(q[0, t], rows, sink, scale), rtol=1e-12, atol=1e-13)


def test_partial_pieces_empty_set_and_single_set():
    """An empty set gives m = -inf, l = 0, o = 0; a single set reproduces the softmax
    without sink (o = sum softmax(z) row), and adding a sink of -inf changes nothing."""
    H, D, N, T = 2, 16, 10, 1
    q, kv, swa = rnd(1, T, H, D), rnd(1, N, D), rnd(1, 4, D)
    idx = np.full((1, T, 3), -1, np.int32)
    m, l, o = oracle.sparse_attn_partial(q, kv, swa, [1000], np.array([[5]]), idx, 0.3, with_swa=False)
    assert np.all(m == -np.inf) and np.all(l == 0) and np.all(o == 0)
    idx = np.array([[[1, 4, 7]]], np.int32)
    m, l, o = oracle.sparse_attn_partial(q, kv, swa, [1000], np.array([[5]]), idx, 0.3, with_swa=False)
    rows = kv[0, [1, 4, 7]].astype(np.float64)
    z = 0.3 * q[0, 0].astype(np.float64) @ rows.T                       # [H, 3]
    p = np.exp(z - z.max(1, keepdims=True))
    np.testing.assert_allclose(o[0, 0], (p / p.sum(1, keepdims=True)) @ rows, rtol=1e-12)
    np.testing.assert_allclose(m[0, 0], z.max(1), rtol=1e-14)
    np.testing.assert_allclose(l[0, 0], p.sum(1), rtol=1e-14)
    out = oracle.attn_combine(m[None], l[None], o[None], np.full(H, -np.inf, np.float32))
    np.testing.assert_allclose(out, o, rtol=1e-14)


@pytest.mark.parametrize("G", [2, 4])
def test_sharded_topk_equals_full_topk(G):
    """Local top-k of each contiguous shard, then the top-k of the gathered (score, global
    index) lists taken in shard order, equals the top-k of the whole row, ties included
    (the gathered list is ascending in global index, so the lower index still wins)."""
    N, k = 4000, 300
    s = (RNG.standard_normal((1, 2, N)) * 64).astype(np.float32)
    s[0, 1, ::7] = 3.0                                    # many exact ties around the threshold
    s[0, 1, 100:400] = 50.0
    nv = np.array([[N, 3333]], np.int32)
    full = oracle.topk(s, nv, k)
    bounds = np.linspace(0, N, G + 1).astype(int)
    cand_s, cand_i = [], []
    for g in range(G):
        lo, hi = bounds[g], bounds[g + 1]
        nvl = np.clip(nv - lo, 0, hi - lo).astype(np.int32)
        loc = oracle.topk(np.ascontiguousarray(s[..., lo:hi]), nvl, k)
        sc = np.where(loc >= 0, np.take_along_axis(s[..., lo:hi], np.maximum(loc, 0), -1), -np.inf)
        cand_s.append(sc.astype(np.float32)); cand_i.append(np.where(loc >= 0, loc + lo, -1))
    cs, ci = np.concatenate(cand_s, -1), np.concatenate(cand_i, -1)
    pos = oracle.topk(np.ascontiguousarray(cs), np.full((1, 2), cs.shape[-1], np.int32), k)
    got = np.where(pos >= 0, np.take_along_axis(ci, np.maximum(pos, 0), -1), -1)
    got = np.where(np.take_along_axis(cs, np.maximum(pos, 0), -1) == -np.inf, -1, got)
    for t in range(2):
        a = sorted(x for x in got[0, t] if x >= 0)
        b = sorted(x for x in full[0, t] if x >= 0)
        assert a == b


# ----------------------------------------------------------------------------- Hadamard rotation
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024])
def test_hadamard_rows_are_scipy_sylvester(n):
    """Rotating the identity gives H_n / sqrt(n), with H_n the Sylvester matrix of scipy.linalg.hadamard."""
    import scipy.linalg
    y = oracle.hadamard_rotate(np.eye(n))
    assert np.max(np.abs(y * math.sqrt(n) - scipy.linalg.hadamard(n))) < 1e-12


def test_hadamard_textbook_h4():
    """The 4 x 4 Walsh-Hadamard matrix in natural (Sylvester) order, written out."""
    H4 = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], np.float64) / 2.0
    assert np.array_equal(oracle.hadamard_rotate(np.eye(4)), H4)
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    assert np.array_equal(oracle.hadamard_rotate(x), np.array([[5.0, -1.0, -2.0, 0.0]]))


def test_hadamard_is_an_orthogonal_involution():
    """H_n is symmetric with H_n^2 = n I, so R = H_n / sqrt(n) is its own inverse and keeps
    norms and inner products: <Rq, Rk> = <q, k>."""
    q = RNG.standard_normal((6, 128))
    k = RNG.standard_normal((6, 128))
    rq, rk = oracle.hadamard_rotate(q), oracle.hadamard_rotate(k)
    assert np.max(np.abs(oracle.hadamard_rotate(rq) - q)) < 1e-13
    assert np.allclose(np.sum(rq * rk, -1), np.sum(q * k, -1), rtol=1e-13, atol=1e-13)
    assert np.allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-14)


def test_hadamard_spreads_a_spike():
    """A one-hot row c e_j becomes a row of +-c/sqrt(n), the sign of entry i being
    (-1)^popcount(i & j): the energy of one channel spreads evenly over all of them."""
    n = 128
    for j, c in ((0, 3.0), (5, -2.5), (127, 1.0)):
        x = np.zeros((1, n))
        x[0, j] = c
        y = oracle.hadamard_rotate(x)[0]
        sign = np.array([(-1) ** bin(i & j).count("1") for i in range(n)], np.float64)
        assert np.allclose(y, sign * c / math.sqrt(n), rtol=1e-15, atol=0)


def test_hadamard_quantize_worked_rows():
    """Rotated e4m3 quantisation on hand-worked rows of n = 128 (c = 1/sqrt(128)):
    2 e_0 -> 2c everywhere -> every code 448 (0x7E);  e_0 + e_1 -> 2c, 0, 2c, 0, ...;
    e_0 - e_1 -> 0, 2c, ...;  -3 e_5 -> -3c (-1)^popcount(i & 5) -> 0xFE / 0x7E."""
    n = 128
    x = np.zeros((4, n), np.float32)
    x[0, 0] = 2.0
    x[1, 0] = x[1, 1] = 1.0
    x[2, 0], x[2, 1] = 1.0, -1.0
    x[3, 5] = -3.0
    codes, scale = oracle.quantize_rows_e4m3_hadamard(x)
    two_c = np.float32(2.0 / math.sqrt(n))
    assert np.all(codes[0] == 0x7E) and scale[0] == np.float32(two_c / np.float32(448.0))
    assert np.array_equal(codes[1], np.tile([0x7E, 0x00], n // 2))
    assert np.array_equal(codes[2], np.tile([0x00, 0x7E], n // 2))
    assert scale[1] == scale[2] == scale[0]
    neg = np.array([bin(i & 5).count("1") % 2 == 0 for i in range(n)])
    assert np.array_equal(codes[3], np.where(neg, 0xFE, 0x7E))
    assert scale[3] == np.float32(np.float32(3.0 / math.sqrt(n)) / np.float32(448.0))
    z, zs = oracle.quantize_rows_e4m3_hadamard(np.zeros((1, n), np.float32))
    assert np.all(z == 0) and zs[0] == 1.0


def test_hadamard_quantize_is_rotate_then_quantize():
    """The rotated quantiser equals the pinned rotation, rounded to fp32, fed to the pinned
    per-row quantiser; rows are independent."""
    x = torch.randn(5, 64, generator=torch.Generator().manual_seed(7)).bfloat16().float().numpy()
    c, s = oracle.quantize_rows_e4m3_hadamard(x)
    c2, s2 = oracle.quantize_rows_e4m3(oracle.hadamard_rotate(x).astype(np.float32))
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    c3, s3 = oracle.quantize_rows_e4m3_hadamard(x[2:3])
    assert np.array_equal(c3[0], c[2]) and s3[0] == s[2]


def test_hadamard_rejects_bad_width():
    for n in (0, 3, 96, 2048):
        with pytest.raises(ValueError):
            oracle.hadamard_rotate(np.ones((1, n)))
    with pytest.raises(ValueError):
        oracle.quantize_rows_e4m3_hadamard(np.ones((1, 96), np.float32))


def test_hadamard_keeps_index_scores():
    """Rotating queries and keys together leaves the Lightning Indexer scores unchanged."""
    x = synth.draw_indexer_outliers(3, 1, 2, 96, Hi=8, di=128)
    qI, w, kI = (x[k].float().numpy() for k in ("qI", "w", "kI"))
    nv = np.array([[96, 50]], np.int32)
    s0 = oracle.index_scores(qI, w, kI, nv)
    s1 = oracle.index_scores(oracle.hadamard_rotate(qI).astype(np.float32), w,
                             oracle.hadamard_rotate(kI).astype(np.float32), nv)
    fin = np.isfinite(s0)
    assert np.array_equal(fin, np.isfinite(s1))
    assert np.max(np.abs(s1[fin] - s0[fin])) < 1e-4 * np.max(np.abs(s0[fin]))


def test_hadamard_cuts_e4m3_score_error_on_outlier_channels():
    """The point of the rotation: with outlier channels shared by queries and keys, the
    e4m3 scores of the rotated operands are much closer to the exact scores than those of
    the unrotated ones (rms error about 0.3x over seeds); on plain N(0,1) inputs both are
    alike (1.00 +- 0.02)."""
    def rel_err(x, quant):
        qI, w, kI = (x[k].float().numpy() for k in ("qI", "w", "kI"))
        nv = np.full((1, qI.shape[1]), kI.shape[1], np.int32)
        exact = oracle.index_scores(qI, w, kI, nv)
        q8, qs = quant(qI)
        k8, ks = quant(kI)
        d = oracle.index_scores_e4m3(q8, qs, w, k8, ks, nv) - exact
        return float(np.sqrt(np.mean(d * d)) / np.std(exact))
    out = synth.draw_indexer_outliers(11, 1, 8, 512)
    plain, rot = rel_err(out, oracle.quantize_rows_e4m3), rel_err(out, oracle.quantize_rows_e4m3_hadamard)
    assert rot < 0.5 * plain, (plain, rot)
    flat = synth.draw_indexer_outliers(11, 1, 8, 512, channels=(), key_offset=0.0, q_gain=1.0)
    plain, rot = rel_err(flat, oracle.quantize_rows_e4m3), rel_err(flat, oracle.quantize_rows_e4m3_hadamard)
    assert 0.9 < rot / plain < 1.1, (plain, rot)


# ----------------------------------------------------------------------------- FP4 (MXFP4) index operands
def test_e2m1_decode_is_the_bit_field_formula():
    """E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; exponent 0 is
    subnormal (m / 2), otherwise 2^(e-1) (1 + m/2).  All 16 codes from the fields."""
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        v = (m / 2.0) if e == 0 else 2.0 ** (e - 1) * (1 + m / 2.0)
        got = oracle.e2m1_decode([c])[0]
        assert got == (-v if s else v) and (np.signbit(got) == bool(s)), c


def test_e2m1_encode_is_nearest_with_even_ties():
    """Brute force over a dense grid: the code is the nearest of the 8 magnitudes, ties go
    to mantissa bit 0, magnitudes beyond 6 give 6; the sign is kept (also for -0)."""
    mags = oracle.e2m1_decode(np.arange(8))
    xs = np.concatenate([np.arange(-800, 801) / 100.0, [-0.0, 1e-30, 50.0, -1e9]])
    got = oracle.e2m1_encode(xs)
    for x, c in zip(xs, got):
        d = np.abs(mags - abs(x))
        best = [i for i in range(8) if d[i] == d.min()]
        want = best[0] if len(best) == 1 else [i for i in best if i % 2 == 0][0]
        assert c == (want | (8 if np.signbit(x) else 0)), (x, c, want)
    # hand-worked ties
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 7.0: 7, -5.0: 14}
    for x, c in ties.items():
        assert oracle.e2m1_encode([x])[0] == c, x


def test_mxfp4_block_scale_and_layout():
    """Per block of 32: X = 2^(floor(log2 amax) - 2), so amax / X lies in [4, 8); E8M0 code
    = log2 X + 127; blocks are independent; an all-zero block gets X = 1 (code 127)."""
    for amax in (1e-3, 0.3, 1.0, 4.0, 6.0, 7.99, 8.0, 1000.0, 3e30):
        x = np.zeros((1, 64), np.float32)
        x[0, 5] = -amax
        x[0, 40] = 1.0
        c, s = oracle.quantize_rows_mxfp4(x)
        e = math.floor(math.log2(np.float32(amax))) - 2
        assert s[0, 0] == e + 127 and s[0, 1] == 127 - 2       # second block: amax 1 -> X = 1/4
        assert 4.0 <= np.float32(amax) / 2.0 ** e < 8.0
        assert c[0, 40] == 6                                    # 1 / (1/4) = 4
    z, zs = oracle.quantize_rows_mxfp4(np.zeros((2, 32), np.float32))
    assert np.all(z == 0) and np.all(zs == 127)
    x = rnd(3, 128)
    c, s = oracle.quantize_rows_mxfp4(x)
    x2 = x.copy()
    x2[:, 32:64] *= 100.0
    c2, s2 = oracle.quantize_rows_mxfp4(x2)
    keep = np.r_[0:32, 64:128]
    assert np.array_equal(c[:, keep], c2[:, keep]) and np.array_equal(s[:, [0, 2, 3]], s2[:, [0, 2, 3]])


def test_mxfp4_round_trip_and_error_bound():
    """Values code * 2^k with a 4 or 6 in the block round-trip exactly; otherwise each
    element is off by at most half a grid step of its binade (times X), or by the
    saturation to 6 X."""
    rng = np.random.default_rng(5)
    for k in (-20, -3, 0, 7):
        codes = rng.integers(0, 16, (4, 64)).astype(np.uint8)
        codes[:, 0] = 7
        codes[:, 32] = 14
        x = (oracle.e2m1_decode(codes) * 2.0 ** k).astype(np.float32)
        c, s = oracle.quantize_rows_mxfp4(x)
        assert np.array_equal(oracle.mxfp4_dequantize(c, s), x)
    x = rnd(16, 128, scale=3.0)
    c, s = oracle.quantize_rows_mxfp4(x)
    X = 2.0 ** (s.astype(np.float64) - 127).repeat(32, axis=1)
    y = np.abs(x / X)
    err = np.abs(oracle.mxfp4_dequantize(c, s) - x) / X
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    assert np.all(err <= np.maximum(half_step, y - 6.0) + 1e-12)


def test_mxfp4_scores_are_the_definition_on_dequantised_values():
    """The FP4 score is the pinned index score of the dequantised operands; with the
    rotation, rotating q and k first leaves the exact scores unchanged, so the FP4 error
    on outlier-channel inputs drops as it does for e4m3."""
    x = synth.draw_indexer_outliers(4, 1, 4, 256)
    qI, w, kI = (x[k].float().numpy() for k in ("qI", "w", "kI"))
    nv = np.full((1, 4), 256, np.int32)
    exact = oracle.index_scores(qI, w, kI, nv)
    errs = []
    for had in (False, True):
        qc, qs = oracle.quantize_rows_mxfp4(qI, hadamard=had)
        kc, ks = oracle.quantize_rows_mxfp4(kI, hadamard=had)
        s4 = oracle.index_scores(oracle.mxfp4_dequantize(qc, qs), w, oracle.mxfp4_dequantize(kc, ks), nv)
        errs.append(float(np.sqrt(np.mean((s4 - exact) ** 2)) / np.std(exact)))
    assert errs[1] < 0.7 * errs[0], errs


def test_mxfp4_rejects_bad_width():
    for n in (16, 48, 0):
        with pytest.raises(ValueError):
            oracle.quantize_rows_mxfp4(np.ones((1, n), np.float32) if n else np.ones((1, 0), np.float32))
    with pytest.raises(ValueError):
        oracle.mxfp4_dequantize(np.zeros((1, 32), np.uint8), np.full((1, 1), 255, np.uint8))


# ----------------------------------------------------------------------------- partial RoPE
THETA = 160000.0


def test_rope_matches_transformers_rotary_embedding():
    """Library pin: transformers' Llama rotary embedding (its own inverse frequencies, fp32)
    and apply_rotary_pos_emb rotate pairs (i, i + 32) of a 64-dim head; after moving the
    interleaved pairs (2i, 2i+1) of the last 64 dims into that layout the two agree."""
    from transformers import LlamaConfig
    from transformers.models.llama import modeling_llama as ml
    cfg = LlamaConfig(hidden_size=64, num_attention_heads=1, head_dim=64, rope_theta=THETA,
                      max_position_embeddings=1 << 20)
    emb = ml.LlamaRotaryEmbedding(cfg)
    pos = np.array([0, 1, 2, 7, 100, 1000, 4095], np.int64)
    x = RNG.standard_normal((len(pos), 96))
    got = oracle.rope(x, pos, THETA)
    assert np.array_equal(got[:, :32], x[:, :32])
    perm = np.r_[np.arange(0, 64, 2), np.arange(1, 64, 2)]        # interleaved -> half layout
    xh = torch.from_numpy(x[:, 32:][:, perm]).view(1, 1, len(pos), 64)
    cos, sin = emb(xh, torch.from_numpy(pos).view(1, -1))
    ref_h, _ = ml.apply_rotary_pos_emb(xh, xh, cos.double(), sin.double())
    ref = np.empty((len(pos), 64))
    ref[:, perm] = ref_h.view(len(pos), 64).numpy()
    tol = 2e-7 * (pos[:, None] + 1) * np.abs(x[:, 32:]).max()
    assert np.all(np.abs(got[:, 32:] - ref) <= tol)


def test_rope_identity_inverse_norm():
    """Position 0 is the identity; the inverse undoes the rotation; norms are kept; only the
    last 64 dims move."""
    x = RNG.standard_normal((5, 512))
    pos = np.array([0, 3, 4000, 262143, 1 << 20])
    y = oracle.rope(x, pos, THETA)
    assert np.array_equal(y[0], x[0])
    assert np.array_equal(y[:, :448], x[:, :448])
    assert np.max(np.abs(oracle.rope(y, pos, THETA, inverse=True) - x)) < 1e-12
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)


def test_rope_relative_position_and_composition():
    """<R(a) q, R(b) k> depends on a - b only, and R(a) R(b) = R(a + b)."""
    q, k = RNG.standard_normal((2, 4, 128))
    a, b, s = np.array([5, 900, 77, 0]), np.array([2, 1000, 77, 65535]), 12345
    d0 = np.sum(oracle.rope(q, a, THETA) * oracle.rope(k, b, THETA), -1)
    d1 = np.sum(oracle.rope(q, a + s, THETA) * oracle.rope(k, b + s, THETA), -1)
    assert np.allclose(d0, d1, rtol=1e-9, atol=1e-9)
    assert np.allclose(oracle.rope(oracle.rope(q, a, THETA), b, THETA), oracle.rope(q, a + b, THETA), atol=1e-9)


def test_rope_pair_frequencies():
    """RoFormer frequencies: pair 0 turns 1 rad per position, and each next pair turns
    theta^(-1/32) times slower (a geometric ladder ending at theta^(-62/64))."""
    x = np.zeros((32, 64))
    x[np.arange(32), 2 * np.arange(32)] = 1.0
    y = oracle.rope(x, 1, THETA)
    ang = np.arctan2(y[np.arange(32), 2 * np.arange(32) + 1], y[np.arange(32), 2 * np.arange(32)])
    assert abs(ang[0] - 1.0) < 1e-15
    assert np.allclose(ang[1:] / ang[:-1], THETA ** (-1.0 / 32), rtol=1e-12)
    assert np.allclose(oracle.rope(x, 1, 10000.0)[1, 2:4], [math.cos(0.01 ** (1 / 16)), math.sin(0.01 ** (1 / 16))])


def _rope_case(seed=3, B=2, N=40, k=12, H=4, D=128, W=150):
    g = np.random.default_rng(seed)
    t = 4 * N + 3
    return dict(q=g.standard_normal((B, 1, H, D)), kv=g.standard_normal((B, N, D)), swa=g.standard_normal((B, W, D)),
                swa_pos0=np.full(B, t - W + 1), q_pos=np.full((B, 1), t), sink=g.standard_normal(H),
                idx=np.stack([np.sort(g.choice(N, k, replace=False)) for _ in range(B)])[:, None].astype(np.int32))


def test_sparse_attn_rope_is_shift_invariant():
    """Moving every position (query, memory entries, SWA rows) by the same amount leaves the
    RoPE attention output unchanged: scores see position differences only, and the output
    is turned back at the query's position."""
    c = _rope_case()
    N = c["kv"].shape[1]
    kv_pos = np.broadcast_to(oracle.compressed_entry_positions(N, 4), (2, N))
    o0 = oracle.sparse_attn_rope(c["q"], c["kv"], c["swa"], c["swa_pos0"], c["q_pos"], c["sink"], c["idx"], 0.1,
                                 THETA, 4, kv_pos=kv_pos)
    s = 100000
    o1 = oracle.sparse_attn_rope(c["q"], c["kv"], c["swa"], c["swa_pos0"] + s, c["q_pos"] + s, c["sink"], c["idx"],
                                 0.1, THETA, 4, kv_pos=kv_pos + s)
    assert np.max(np.abs(o1 - o0)) < 1e-5 * np.max(np.abs(o0))


def test_sparse_attn_rope_reduces_to_plain_attention_at_one_position():
    """With every attended row at the query's own position the rotations cancel: the RoPE
    attention equals the plain attention of the unrotated inputs (SWA buffer placed outside
    the window so that only the memory rows count)."""
    c = _rope_case(seed=9)
    N = c["kv"].shape[1]
    t = int(c["q_pos"][0, 0])
    swa_pos0 = np.full(2, t - 1000)
    kv_pos = np.full((2, N), t)
    o = oracle.sparse_attn_rope(c["q"], c["kv"], c["swa"], swa_pos0, c["q_pos"], c["sink"], c["idx"], 0.1, THETA, 4,
                                kv_pos=kv_pos)
    plain = oracle.sparse_attn(c["q"], c["kv"], c["swa"], swa_pos0, c["q_pos"], c["sink"], c["idx"], 0.1)
    assert np.max(np.abs(o - plain)) < 1e-5 * np.max(np.abs(plain))
    o_far = oracle.sparse_attn_rope(c["q"], c["kv"], c["swa"], swa_pos0, c["q_pos"], c["sink"], c["idx"], 0.1, THETA, 4)
    assert np.max(np.abs(o_far - plain)) > 1e-3          # real positions do change the result
