"""sparse_attn / hca_attn parity against the CPU oracle (fp32: 1e-5 relative to the
magnitude; bf16: abs 2e-2 + rel 1e-2), on ragged shapes and on the full workloads.
Index lists come from the seeded generator (random ascending subsets of the
visible entries, -1 padded), so attention is tested on its own."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import check_attn_bf16, check_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _np(t):
    return t.float().numpy()


def _case(wl, seed=0, k=None, N=None):
    at = synth.draw_attention(wl, seed=seed, N=N)
    N = at["kv"].shape[1]
    q_pos = np.array([wl.q_pos] * wl.B, np.int64)
    swa_pos0 = np.array([wl.swa_pos0] * wl.B, np.int64)
    nv = oracle.n_visible(q_pos, wl.ratio, N)
    idx = None
    if k is not None:
        idx = synth.random_subset(seed, f"{wl.name}/idx", torch.from_numpy(nv), k).numpy()
    return at, q_pos, swa_pos0, idx


def _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale, rows=None):
    return csa.sparse_attn(at["q"].cuda(), at["kv"].cuda(), at["swa_kv"].cuda(), torch.from_numpy(swa_pos0).cuda(),
                           torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), torch.from_numpy(idx).cuda(),
                           scale).float().cpu().numpy()


def test_f32_tiny_full(csa):
    wl = synth.WORKLOADS["tiny"]
    at, q_pos, swa_pos0, idx = _case(wl, k=wl.topk)
    scale = 1 / math.sqrt(wl.D)
    assert at["swa_kv"].shape[1] == 135                       # positions 3961..4095
    g = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale)
    ref, mag = oracle.sparse_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos,
                                  at["sink"].numpy(), idx, scale, with_mag=True)
    check_f32(g, ref, np.maximum(mag, np.abs(ref)), what="tiny fp32 sparse_attn")


@pytest.mark.parametrize("D,H", [(128, 16), (256, 40), (512, 64), (512, 128)])
@pytest.mark.parametrize("B,T", [(1, 1), (3, 2), (1, 160)])
def test_bf16_ragged(csa, D, H, B, T):
    """Ragged k with -1 padding and out-of-range indices, an SWA buffer that starts
    inside the window, early positions where the window clips at 0, and both the
    split-KV (few queries) and single-pass (many queries) launch shapes."""
    N = 300
    k = 77
    q0 = 150 if T < 100 else 40
    wl = synth.Workload(f"attn_ragged_{D}_{H}", "bf16", B=B, ctx=q0 + T, T=T, q_pos0=q0, ratio=1, N=N, H=H, D=D)
    at, q_pos, swa_pos0, _ = _case(wl, seed=D + H + T)
    # visible entries: N for every query (ratio 1 here); subsets of 60 then padding
    idx = synth.random_subset(D + T, "attn/ragged/idx", torch.full((B, T), N), 60).numpy()
    idx = np.concatenate([idx, np.full((B, T, k - 60), -1, np.int32)], -1)
    idx[..., 61] = N + 5                                  # out of range: contributes nothing
    idx[..., 62] = -7
    swa_pos0 = swa_pos0 + 3                               # first 3 window positions missing from the buffer
    at["swa_kv"] = at["swa_kv"][:, 3:].contiguous()
    scale = 1 / math.sqrt(D)
    g = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale)
    ref = oracle.sparse_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos,
                             at["sink"].numpy(), idx, scale)
    check_attn_bf16(g, ref, what=f"bf16 D={D} H={H} B={B} T={T}")


@pytest.mark.parametrize("D,H,k", [(512, 64, 128), (512, 100, 224), (512, 128, 352), (512, 64, 480),
                                   (512, 128, 1024), (256, 72, 400), (128, 16, 900)])
def test_bf16_split_clusters(csa, D, H, k):
    """Few queries with long row lists: the row list is split over 2..8 CTAs that merge
    their partials inside a thread-block cluster; H not a multiple of 64 leaves the
    last head group partly empty."""
    B, T, N = 2, 1, 4096
    wl = synth.Workload(f"attn_split_{D}_{H}_{k}", "bf16", B=B, ctx=2 * N, T=T, q_pos0=2 * N - 1, ratio=1, N=N,
                        H=H, D=D)
    at, q_pos, swa_pos0, _ = _case(wl, seed=k + H)
    idx = synth.random_subset(k, "attn/split/idx", torch.full((B, T), N), k).numpy()
    scale = 1 / math.sqrt(D)
    g = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale)
    ref = oracle.sparse_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos,
                             at["sink"].numpy(), idx, scale)
    check_attn_bf16(g, ref, what=f"split D={D} H={H} k={k}")


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_bf16_decode_full(csa, name):
    wl = synth.WORKLOADS[name]
    at, q_pos, swa_pos0, idx = _case(wl, k=wl.topk)
    scale = 1 / math.sqrt(wl.D)
    g = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale)
    ref = oracle.sparse_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos,
                             at["sink"].numpy(), idx, scale)
    check_attn_bf16(g, ref, what=name)


def test_bf16_prefill_sampled(csa):
    wl = synth.WORKLOADS["flash_prefill"]
    at, q_pos, swa_pos0, idx = _case(wl, k=wl.topk)
    scale = 1 / math.sqrt(wl.D)
    g = csa.sparse_attn(at["q"].cuda(), at["kv"].cuda(), at["swa_kv"].cuda(), torch.from_numpy(swa_pos0).cuda(),
                        torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), torch.from_numpy(idx).cuda(), scale)
    rows = [0, 1, 127, 128, 2000, 4094, 4095]
    ref = oracle.sparse_attn(_np(at["q"][:, rows]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos[:, rows],
                             at["sink"].numpy(), idx[:, rows], scale)
    check_attn_bf16(g[:, rows].float().cpu().numpy(), ref, what="prefill sampled")
    assert torch.isfinite(g.float()).all()


def test_hca_full(csa):
    wl = synth.WORKLOADS["pro_hca"]
    at, q_pos, swa_pos0, _ = _case(wl)
    scale = 1 / math.sqrt(wl.D)
    g = csa.hca_attn(at["q"].cuda(), at["kv"].cuda(), at["swa_kv"].cuda(), torch.from_numpy(swa_pos0).cuda(),
                     torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), scale).float().cpu().numpy()
    ref = oracle.hca_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(),
                          scale)
    check_attn_bf16(g, ref, what="pro_hca")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_hca_causal_prefix_and_poison(csa, dtype):
    """Only complete summaries are read: NaN in kv rows at or past (pos+1)//128 and in
    SWA rows outside the window leaves the output unchanged."""
    D, H = 128, 32
    wl = synth.Workload("hca_causal", dtype, B=2, ctx=128 * 9 + 50, T=3, q_pos0=128 * 9 + 40, ratio=128, N=20,
                        H=H, D=D)
    at, q_pos, swa_pos0, _ = _case(wl, seed=5)
    scale = 1 / math.sqrt(D)
    args = lambda kv, sw: (at["q"].cuda(), kv.cuda(), sw.cuda(), torch.from_numpy(swa_pos0).cuda(),
                           torch.from_numpy(q_pos).cuda(), at["sink"].cuda(), scale)
    g = csa.hca_attn(*args(at["kv"], at["swa_kv"])).float().cpu().numpy()
    ref = oracle.hca_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(), scale)
    if dtype == "bf16":
        check_attn_bf16(g, ref, what="hca causal")
    else:
        mag = oracle.hca_attn(_np(at["q"]), _np(at["kv"]), _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(),
                              scale, with_mag=True)[1]
        check_f32(g, ref, np.maximum(mag, np.abs(ref)), what="hca causal f32")
    kv2 = at["kv"].clone()
    kv2[:, 9:] = float("nan")                            # 9 complete blocks at positions 1192..1194
    g2 = csa.hca_attn(*args(kv2, at["swa_kv"])).float().cpu().numpy()
    assert np.array_equal(g2, g)


def test_sparse_poison_unselected(csa):
    D, H, N = 512, 64, 2000
    wl = synth.Workload("poison", "bf16", B=1, ctx=4 * N, T=2, q_pos0=4 * N - 2, ratio=4, N=N, H=H, D=D)
    at, q_pos, swa_pos0, idx = _case(wl, k=64, seed=9)
    scale = 1 / math.sqrt(D)
    g = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale)
    keep = np.zeros(N, bool)
    keep[idx[idx >= 0]] = True
    at["kv"][0, torch.from_numpy(~keep)] = float("nan")
    g2 = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, scale)
    assert np.array_equal(g, g2)


def test_sink_closed_form_gpu(csa):
    """q = 0: every logit is 0, so o = sum(rows) / (e^sink + L) -- the sink closed form."""
    D, H, N, k = 512, 128, 64, 16
    wl = synth.Workload("sinkcf", "bf16", B=1, ctx=1000, T=1, q_pos0=999, ratio=1, N=N, H=H, D=D)
    at, q_pos, swa_pos0, _ = _case(wl, seed=4)
    at["q"].zero_()
    v = synth.store(synth.normal(4, "sinkcf/v", (D,)), "bf16")
    at["kv"][:] = v
    at["swa_kv"][:] = v
    idx = np.arange(k, dtype=np.int32)[None, None]
    g = _gpu_sparse(csa, at, q_pos, swa_pos0, idx, 0.05)
    L = k + 128
    for h in range(H):
        p = 1.0 / (math.exp(float(at["sink"][h])) + L)
        check_attn_bf16(g[0, 0, h], L * p * v.double().numpy(), what=f"sink closed form head {h}")
