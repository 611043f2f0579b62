"""Partial RoPE on the GPU against the oracle ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文"
§6: RoPE on the last 64 dims, the output's same dims turned back after the attention;
reading c26 for pairing, base and positions).

- csa_rope: rows turned at their positions (compressed entries at i * m, SWA rows at their
  token positions), bf16 and fp32, in place and out of place, and the inverse.
- sparse_attn_rope at the flash64k and pro1m shapes, the caches rotated by csa_rope when
  they are built, against oracle.sparse_attn_rope on the unrotated inputs (abs 2e-2 /
  rel 1e-2); the tiny fp32 configuration (D = 128, RoPE on its last 64 dims) with the fp32
  rule; hca_attn_rope at the pro_hca shape against the oracle's pieces composed.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import F32_REL, bf16_round, check_attn_bf16, check_bf16_store, check_f32

pytestmark = pytest.mark.gpu

THETA = 160000.0


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _np(t):
    return t.float().numpy()


def _rope_mag(x, pos):
    """Forward-error scale of the rotated values: |a cos| + |b sin| per output element."""
    D = x.shape[-1]
    mag = np.abs(np.asarray(x, np.float64)).copy()
    a, b = mag[..., D - 64::2], mag[..., D - 63::2]
    i = np.arange(32)
    ang = np.asarray(pos, np.float64)[..., None] * THETA ** (-2.0 * i / 64)
    c, s = np.abs(np.cos(ang)), np.abs(np.sin(ang))
    mag[..., D - 64::2] = a * c + b * s
    mag[..., D - 63::2] = a * s + b * c
    return mag


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("inplace", [False, True])
def test_csa_rope_rows(csa, dtype, inplace):
    B, R, D = 3, 700, 512
    x = synth.store(synth.normal(3, f"rope/rows/{dtype}", (B, R, D)), dtype)
    base = torch.tensor([0, 1 << 20, 126849], dtype=torch.int64)
    for stride, use_base in ((4, False), (1, True), (128, True)):
        pos = (base.numpy()[:, None] if use_base else 0) + np.arange(R)[None] * stride
        g = x.cuda()
        out = g if inplace else None
        got = csa.csa_rope(g, THETA, stride=stride, pos_base=base.cuda() if use_base else None, out=out)
        got = got.float().cpu().numpy()
        ref = oracle.rope(_np(x), np.broadcast_to(pos, (B, R)), THETA)
        mag = _rope_mag(_np(x), np.broadcast_to(pos, (B, R)))
        if dtype == "bf16":
            check_bf16_store(got, ref, mag, what=f"rope rows stride {stride}")
        else:
            check_f32(got, ref, mag, what=f"rope rows stride {stride}")
        assert np.array_equal(got[..., :D - 64], _np(x)[..., :D - 64])      # unrotated dims copied
        back = csa.csa_rope(torch.from_numpy(got).to(x.dtype).cuda(), THETA, stride=stride,
                            pos_base=base.cuda() if use_base else None, inverse=True).float().cpu().numpy()
        tol = 2.0 ** -7 if dtype == "bf16" else 1e-5        # two roundings of the stored rows
        assert np.all(np.abs(back - _np(x)) <= tol * np.abs(_np(x)).max(-1, keepdims=True))


def _rope_chain(csa, wl, seed):
    """GPU: caches rotated by csa_rope, then sparse_attn_rope.  Oracle: sparse_attn_rope on the
    unrotated inputs, over the rows the index lists select (entry i at position 4 i)."""
    at = synth.draw_attention(wl, seed=seed)
    B, N = wl.B, wl.N
    q_pos = np.array([wl.q_pos] * B, np.int64)
    swa_pos0 = np.array([wl.swa_pos0] * B, np.int64)
    nv = oracle.n_visible(q_pos, 4, N)
    idx = synth.random_subset(seed, f"{wl.name}/rope/idx", torch.from_numpy(nv), wl.topk).numpy()
    scale = 1 / math.sqrt(wl.D)
    kv = at["kv"].cuda()
    swa = at["swa_kv"].cuda()
    csa.csa_rope(kv, THETA, stride=4, out=kv)
    csa.csa_rope(swa, THETA, stride=1, pos_base=torch.from_numpy(swa_pos0).cuda(), out=swa)
    out = csa.sparse_attn(at["q"].cuda(), kv, swa, torch.from_numpy(swa_pos0).cuda(), torch.from_numpy(q_pos).cuda(),
                          at["sink"].cuda(), torch.from_numpy(idx).cuda(), scale, rope_theta=THETA)
    refs = []
    for b in range(B):                                     # the oracle on the selected rows only
        sel = idx[b].reshape(-1)
        rows = np.unique(sel[sel >= 0])
        remap = np.full(N, -1, np.int64)
        remap[rows] = np.arange(len(rows))
        idx_b = np.where(idx[b:b + 1] >= 0, remap[np.maximum(idx[b:b + 1], 0)], -1).astype(np.int32)
        kv_b = _np(at["kv"][b:b + 1, torch.from_numpy(rows)])
        refs.append(oracle.sparse_attn_rope(_np(at["q"][b:b + 1]), kv_b, _np(at["swa_kv"][b:b + 1]), swa_pos0[b:b + 1],
                                            q_pos[b:b + 1], at["sink"].numpy(), idx_b, scale, THETA, 4,
                                            kv_pos=(rows * 4)[None]))
    return out, np.concatenate(refs)


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_sparse_attn_rope_decode(csa, name):
    out, ref = _rope_chain(csa, synth.WORKLOADS[name], seed=21)
    check_attn_bf16(out.float().cpu().numpy(), ref, what=f"{name} rope")


def test_sparse_attn_rope_tiny_fp32(csa):
    """The tiny configuration (fp32, D = 128, RoPE on its last 64 dims), with the fp32 rule:
    the oracle's rotated inputs give the magnitude of each output."""
    wl = synth.WORKLOADS["tiny"]
    at = synth.draw_attention(wl, seed=22)
    q_pos = np.array([wl.q_pos], np.int64)
    swa_pos0 = np.array([wl.swa_pos0], np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    idx = synth.random_subset(22, "tiny/rope/idx", torch.from_numpy(nv), wl.topk).numpy()
    scale = 1 / math.sqrt(wl.D)
    kv, swa = at["kv"].cuda(), at["swa_kv"].cuda()
    csa.csa_rope(kv, THETA, stride=4, out=kv)
    csa.csa_rope(swa, THETA, pos_base=torch.from_numpy(swa_pos0).cuda(), out=swa)
    got = csa.sparse_attn(at["q"].cuda(), kv, swa, torch.from_numpy(swa_pos0).cuda(), torch.from_numpy(q_pos).cuda(),
                          at["sink"].cuda(), torch.from_numpy(idx).cuda(), scale, rope_theta=THETA).cpu().numpy()
    ref = oracle.sparse_attn_rope(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(),
                                  idx, scale, THETA, 4)
    qr = oracle.rope(_np(at["q"]), q_pos[:, :, None], THETA)
    kvr = oracle.rope(_np(at["kv"]), oracle.compressed_entry_positions(wl.N, 4)[None], THETA)
    swar = oracle.rope(_np(at["swa_kv"]), swa_pos0[:, None] + np.arange(at["swa_kv"].shape[1])[None], THETA)
    inner, mag = oracle.sparse_attn(qr, kvr, swar, swa_pos0, q_pos, at["sink"].numpy(), idx, scale, with_mag=True)
    mag = np.maximum(mag, np.abs(inner))
    mag[..., 64::2] = mag[..., 64::2] + mag[..., 65::2]     # the inverse turn mixes each pair
    mag[..., 65::2] = mag[..., 64::2]
    # the rotated caches carry fp32 rounding of their own, within 1e-5 of their magnitude
    check_f32(got, ref, 2 * mag, what="tiny fp32 rope")


def test_hca_attn_rope(csa):
    wl = synth.WORKLOADS["pro_hca"]
    at = synth.draw_attention(wl, seed=23)
    q_pos = np.array([wl.q_pos] * wl.B, np.int64)
    swa_pos0 = np.array([wl.swa_pos0] * wl.B, np.int64)
    scale = 1 / math.sqrt(wl.D)
    kv, swa = at["kv"].cuda(), at["swa_kv"].cuda()
    csa.csa_rope(kv, THETA, stride=128, out=kv)
    csa.csa_rope(swa, THETA, pos_base=torch.from_numpy(swa_pos0).cuda(), out=swa)
    got = csa.hca_attn(at["q"].cuda(), kv, swa, torch.from_numpy(swa_pos0).cuda(), torch.from_numpy(q_pos).cuda(),
                       at["sink"].cuda(), scale, rope_theta=THETA).float().cpu().numpy()
    qr = oracle.rope(_np(at["q"]), q_pos[:, :, None], THETA)
    kvr = oracle.rope(_np(at["kv"]), oracle.compressed_entry_positions(wl.N, 128)[None], THETA)
    swar = oracle.rope(_np(at["swa_kv"]), swa_pos0[:, None] + np.arange(at["swa_kv"].shape[1])[None], THETA)
    inner = oracle.hca_attn(qr.astype(np.float32), kvr.astype(np.float32), swar.astype(np.float32), swa_pos0, q_pos,
                            at["sink"].numpy(), scale)
    ref = oracle.rope(inner, q_pos[:, :, None], THETA, inverse=True)
    check_attn_bf16(got, ref, what="pro_hca rope")


def test_rope_attention_shift_invariance(csa):
    """RoPE attention depends on positions only through their differences: moving the
    query, the SWA rows and the entry positions by a common shift (whole blocks) leaves the
    output unchanged within bf16 rounding."""
    wl = synth.Workload("rope_shift", "bf16", B=1, ctx=4 * 2000, T=1, q_pos0=4 * 2000 - 1, ratio=4, N=2000,
                        H=64, D=512, topk=256)
    at = synth.draw_attention(wl, seed=24)
    nv = oracle.n_visible(np.array([wl.q_pos]), 4, wl.N)
    idx = torch.from_numpy(synth.random_subset(24, "rope/shift/idx", torch.from_numpy(nv), wl.topk).numpy()).cuda()
    outs = []
    for shift_blocks in (0, 1 << 16):
        shift = 4 * shift_blocks
        q_pos = torch.tensor([[wl.q_pos0 + shift]], dtype=torch.int64).cuda()
        s0 = torch.tensor([wl.swa_pos0 + shift], dtype=torch.int64).cuda()
        kv, swa = at["kv"].cuda(), at["swa_kv"].cuda()
        # entry i stands at 4 i + shift: base = shift, stride 4
        csa.csa_rope(kv, THETA, stride=4, pos_base=torch.tensor([shift], dtype=torch.int64).cuda(), out=kv)
        csa.csa_rope(swa, THETA, pos_base=s0, out=swa)
        outs.append(csa.sparse_attn(at["q"].cuda(), kv, swa, s0, q_pos, at["sink"].cuda(), idx, 1 / math.sqrt(512),
                                    rope_theta=THETA).float().cpu().numpy())
    check_attn_bf16(outs[1], outs[0].astype(np.float64), what="rope shift")
