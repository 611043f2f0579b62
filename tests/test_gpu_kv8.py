"""Mixed-precision KV storage on the GPU ([HA] §4.2 storage precision: RoPE dims BF16,
the rest FP8): csa_quantize_kv8 is bit-exact against the oracle's codec, and
sparse_attn / hca_attn over such entries match the oracle's attention over the
dequantised rows (bf16 tolerance: abs 2e-2 + rel 1e-2).  The entries the attention
tests use are made by the oracle, never by the CUDA path."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth
from tolerances import check_attn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


def _np(t):
    return t.float().numpy()


def _entries(kv_bf16):
    """Oracle entries [B, N, 608] and the dequantised rows [B, N, 512]."""
    e = oracle.kv8_quantize(_np(kv_bf16))
    return e, oracle.kv8_dequantize(e, kv_bf16.shape[-1])


@pytest.mark.parametrize("rows", [1, 37, 1000])
def test_quantize_kv8_bit_exact(csa, rows):
    g = torch.Generator().manual_seed(rows)
    x = torch.randn(rows, 512, generator=g)
    mag = torch.exp(torch.randn(rows, 8, generator=g) * 4).repeat_interleave(64, dim=1)
    x = (x * mag).to(torch.bfloat16)
    if rows > 4:
        x[1, 64:128] = 0                                   # an all-zero block
        x[2, :] = 0
        x[3, 5] = 2.0 ** -130                              # subnormal amax
        x[4, :448] = torch.tensor(448.0).to(torch.bfloat16)
    ref = oracle.kv8_quantize(_np(x))
    got = csa.quantize_kv8(x.cuda()).cpu().numpy()
    np.testing.assert_array_equal(got, ref)


def _case(wl, seed=0):
    at = synth.draw_attention(wl, seed=seed)
    q_pos = np.array([wl.q_pos] * wl.B, np.int64)
    swa_pos0 = np.array([wl.swa_pos0] * wl.B, np.int64)
    return at, q_pos, swa_pos0


def _sparse(csa, at, ent, q_pos, swa_pos0, idx, scale):
    return csa.sparse_attn(at["q"].cuda(), torch.from_numpy(ent).cuda(), at["swa_kv"].cuda(),
                           torch.from_numpy(swa_pos0).cuda(), torch.from_numpy(q_pos).cuda(), at["sink"].cuda(),
                           torch.from_numpy(idx).cuda(), scale).float().cpu().numpy()


@pytest.mark.parametrize("H", [64, 128])
@pytest.mark.parametrize("B,T,q0", [(1, 1, 150), (3, 2, 150), (2, 3, 40), (1, 160, 40)])
def test_kv8_sparse_ragged(csa, H, B, T, q0):
    """Ragged k with -1 padding and out-of-range indices; q0 = 40 clips the window at
    position 0, so the SWA rows are not a multiple of the 32-row tile and padding rows
    sit between them and the memory rows."""
    D, N, k = 512, 300, 77
    wl = synth.Workload(f"kv8_ragged_{H}_{T}", "bf16", B=B, ctx=q0 + T, T=T, q_pos0=q0, ratio=1, N=N, H=H, D=D)
    at, q_pos, swa_pos0 = _case(wl, seed=H + T + q0)
    idx = synth.random_subset(H + T, "kv8/ragged/idx", torch.full((B, T), N), 60).numpy()
    idx = np.concatenate([idx, np.full((B, T, k - 60), -1, np.int32)], -1)
    idx[..., 61] = N + 5
    idx[..., 62] = -7
    ent, kvd = _entries(at["kv"])
    scale = 1 / math.sqrt(D)
    g = _sparse(csa, at, ent, q_pos, swa_pos0, idx, scale)
    ref = oracle.sparse_attn(_np(at["q"]), kvd, _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(), idx, scale)
    check_attn_bf16(g, ref, what=f"kv8 H={H} B={B} T={T} q0={q0}")


@pytest.mark.parametrize("H,k", [(64, 128), (100, 224), (128, 1024), (64, 480)])
def test_kv8_split_clusters(csa, H, k):
    B, T, N, D = 2, 1, 4096, 512
    wl = synth.Workload(f"kv8_split_{H}_{k}", "bf16", B=B, ctx=2 * N, T=T, q_pos0=2 * N - 1, ratio=1, N=N, H=H, D=D)
    at, q_pos, swa_pos0 = _case(wl, seed=k + H)
    idx = synth.random_subset(k, "kv8/split/idx", torch.full((B, T), N), k).numpy()
    ent, kvd = _entries(at["kv"])
    scale = 1 / math.sqrt(D)
    g = _sparse(csa, at, ent, q_pos, swa_pos0, idx, scale)
    ref = oracle.sparse_attn(_np(at["q"]), kvd, _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(), idx, scale)
    check_attn_bf16(g, ref, what=f"kv8 split H={H} k={k}")


@pytest.mark.parametrize("name", ["flash64k", "pro1m"])
def test_kv8_decode_full(csa, name):
    wl = synth.WORKLOADS[name]
    at, q_pos, swa_pos0 = _case(wl)
    nv = oracle.n_visible(q_pos, wl.ratio, at["kv"].shape[1])
    idx = synth.random_subset(0, f"{wl.name}/idx", torch.from_numpy(nv), wl.topk).numpy()
    ent, kvd = _entries(at["kv"])
    scale = 1 / math.sqrt(wl.D)
    g = _sparse(csa, at, ent, q_pos, swa_pos0, idx, scale)
    ref = oracle.sparse_attn(_np(at["q"]), kvd, _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(), idx, scale)
    check_attn_bf16(g, ref, what=f"kv8 {name}")


@pytest.mark.parametrize("q0", [None, 700])
def test_kv8_hca(csa, q0):
    """Dense rows: the full pro_hca shape, and an early position whose visible prefix
    is a few entries (ragged tail tile)."""
    wl = synth.WORKLOADS["pro_hca"]
    if q0 is not None:
        wl = synth.Workload("kv8_hca_early", "bf16", B=2, ctx=q0 + 1, T=1, q_pos0=q0, ratio=128, N=64, H=128, D=512)
    at, q_pos, swa_pos0 = _case(wl)
    ent, kvd = _entries(at["kv"])
    scale = 1 / math.sqrt(wl.D)
    g = csa.hca_attn(at["q"].cuda(), torch.from_numpy(ent).cuda(), at["swa_kv"].cuda(),
                     torch.from_numpy(swa_pos0).cuda(), torch.from_numpy(q_pos).cuda(), at["sink"].cuda(),
                     scale).float().cpu().numpy()
    ref = oracle.hca_attn(_np(at["q"]), kvd, _np(at["swa_kv"]), swa_pos0, q_pos, at["sink"].numpy(), scale)
    check_attn_bf16(g, ref, what=f"kv8 hca q0={q0}")
