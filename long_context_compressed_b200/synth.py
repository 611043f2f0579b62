"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module holds no arithmetic of the method: only a counter-based random
generator, the workload shapes, and recipes that draw each named input tensor.
Both the CUDA path and the CPU oracle consume the same bytes drawn here.

Generator (a published construction): SplitMix64 (Steele, Lea, Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014) used in counter mode --
output i of stream ``key`` is mix(key + (i+1)*0x9E3779B97F4A7C15) -- followed by
53-bit uniforms in [0,1) and the Box-Muller transform for normals.  The stream
key of a tensor is SplitMix64-mixed from (seed, FNV-1a-64 of its name), so every
tensor has an independent, reproducible stream that does not depend on the
order in which tensors are drawn.  Values are drawn in float64, rounded once to
float32, and rounded again (round-to-nearest-even) to bfloat16 where the
workload stores bfloat16.

Workload shapes follow the pages' Flash / Pro configurations ("DeepSeek-V4
混合注意力：从压缩记忆到百万上下文" §2 configuration table and §3 entry counts):
64 index heads of 128 dims, top-k 512 (Flash) / 1024 (Pro), 64 / 128 query
heads, SWA window 128, compression 4:1 and 128:1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_CHUNK = 1 << 24


def _signed(x: int) -> int:
    x &= _MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def _mix_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (reference for the tensor version)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & _MASK64
    return z ^ (z >> 31)


def _fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for byte in name.encode("utf-8"):
        h ^= byte
        h = (h * 0x100000001B3) & _MASK64
    return h


def stream_key(seed: int, name: str) -> int:
    """64-bit key of the named tensor's stream (unsigned Python int)."""
    return _mix_int(_fnv1a64(name) ^ _mix_int(seed * _GOLDEN))


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _signed(_MIX1)
    z = (z ^ _srl(z, 27)) * _signed(_MIX2)
    return z ^ _srl(z, 31)


def raw_u64(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Outputs start..start+count-1 of the counter-mode stream, as int64 bit patterns."""
    ctr = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _mix(ctr * _signed(_GOLDEN) + _signed(key))


def _uniform53(bits: torch.Tensor) -> torch.Tensor:
    return _srl(bits, 11).to(torch.float64) * (2.0 ** -53)


def uniform(seed: int, name: str, shape, lo: float = 0.0, hi: float = 1.0, device="cpu") -> torch.Tensor:
    """U(lo, hi) float32 tensor from the named stream."""
    key = stream_key(seed, name)
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        u = _uniform53(raw_u64(key, s, c, device))
        out[s:s + c] = (lo + (hi - lo) * u).to(torch.float32)
    return out.reshape(shape)


def normal(seed: int, name: str, shape, std: float = 1.0, device="cpu") -> torch.Tensor:
    """N(0, std^2) float32 tensor (Box-Muller on draws 2e and 2e+1 for element e)."""
    key = stream_key(seed, name)
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        bits = raw_u64(key, 2 * s, 2 * c, device).view(c, 2)
        u1 = _uniform53(bits[:, 0])
        u2 = _uniform53(bits[:, 1])
        r = torch.sqrt(-2.0 * torch.log1p(-u1))
        out[s:s + c] = (std * r * torch.cos(2.0 * math.pi * u2)).to(torch.float32)
    return out.reshape(shape)


def store(x: torch.Tensor, dtype: str) -> torch.Tensor:
    """Round a float32 draw to the storage type ('f32' or 'bf16', RN-even)."""
    if dtype == "f32":
        return x.to(torch.float32)
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    raise ValueError(dtype)


def random_subset(seed: int, name: str, n_valid, k: int, device="cpu") -> torch.Tensor:
    """Per row, min(k, n_valid) distinct indices in [0, n_valid), ascending, padded with -1.

    Used as a seeded stand-in for a top-k index list when a stage is tested on
    its own.  n_valid: int tensor [...]; returns int32 [..., k]."""
    nv = torch.as_tensor(n_valid, dtype=torch.int64).reshape(-1)
    rows = []
    for r, v in enumerate(nv.tolist()):
        row = torch.full((k,), -1, dtype=torch.int32)
        if v > 0:
            keys = uniform(seed, f"{name}/{r}", (v,))
            take = min(k, v)
            sel = torch.argsort(keys)[:take].sort().values.to(torch.int32)
            row[:take] = sel
        rows.append(row)
    out = torch.stack(rows).reshape(*torch.as_tensor(n_valid).shape, k)
    return out.to(device)


# --------------------------------------------------------------------------- workloads
@dataclass
class Workload:
    """Shapes of one synthetic workload (all sizes per the pages' configurations)."""
    name: str
    dtype: str                 # storage type of activations: 'f32' or 'bf16'
    B: int                     # sequences
    ctx: int                   # context length n (raw tokens) at the last query
    T: int                     # queries per sequence
    q_pos0: int                # absolute position of the first query (queries are consecutive)
    ratio: int                 # 4 (CSA) or 128 (HCA)
    N: int                     # compressed entries in the cache
    H: int                     # attention query heads
    D: int                     # latent / head dim
    topk: int = 0
    Hi: int = 64               # index heads
    di: int = 128              # index head dim
    window: int = 128          # SWA window
    comp_L: int = 0            # raw tokens compressed per step (0: none)
    comp_c: int = 0            # channels of the KV compressor
    comp_ci: int = 0           # channels of the index-key compressor (0: none)
    index_dtype: str = "bf16"  # 'f32', 'bf16' or 'e4m3'
    w_dist: str = "normal"     # 'uniform' (U(0,1)) or 'normal'
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def q_pos(self):
        return [self.q_pos0 + t for t in range(self.T)]

    @property
    def swa_pos0(self):
        return max(0, self.q_pos0 - self.window + 1)

    @property
    def W(self):
        return self.q_pos0 + self.T - self.swa_pos0


WORKLOADS = {
    # Tiny CSA reference: fp32, n=4096, 1024 entries, c=128, 8 decode queries at 4088..4095.
    "tiny": Workload("tiny", "f32", B=1, ctx=4096, T=8, q_pos0=4088, ratio=4, N=1024, H=16, D=128,
                     topk=64, comp_L=4096, comp_c=128, index_dtype="f32", w_dist="uniform"),
    # Flash-shaped CSA decode at 64K, B=8, one token per sequence.
    "flash64k": Workload("flash64k", "bf16", B=8, ctx=65536, T=1, q_pos0=65535, ratio=4, N=16384,
                         H=64, D=512, topk=512, comp_L=4, comp_c=512, comp_ci=128, index_dtype="e4m3"),
    # Pro-shaped CSA decode at 1M, B=1, FP8 index keys; compressor over the last 512 raw tokens.
    "pro1m": Workload("pro1m", "bf16", B=1, ctx=1 << 20, T=1, q_pos0=(1 << 20) - 1, ratio=4, N=1 << 18,
                      H=128, D=512, topk=1024, comp_L=512, comp_c=512, index_dtype="e4m3"),
    # Flash-shaped chunked prefill: 4096 queries at 126976..131071 of a 131072-token context.
    "flash_prefill": Workload("flash_prefill", "bf16", B=1, ctx=131072, T=4096, q_pos0=126976, ratio=4,
                              N=32768, H=64, D=512, topk=512, comp_L=4096, comp_c=512, comp_ci=128,
                              index_dtype="bf16"),
    # Pro-shaped HCA decode at 1M, B=4; compressor over a 16384-token tail.
    "pro_hca": Workload("pro_hca", "bf16", B=4, ctx=1 << 20, T=1, q_pos0=(1 << 20) - 1, ratio=128,
                        N=8192, H=128, D=512, comp_L=16384, comp_c=512),
}


def draw_compressor(wl: Workload, seed: int = 0, device="cpu", L=None, c=None, tag="kv"):
    """Raw compressor inputs.  CSA: C_a, C_b, Z_a, Z_b and the carry prev_Cb, prev_Zb
    (the b branch of the block before the chunk; absent when the chunk starts at
    position 0).  HCA: C, Z.  All N(0,1), [B, L, c] in the workload's storage type."""
    L = wl.comp_L if L is None else L
    c = wl.comp_c if c is None else c
    sh = (wl.B, L, c)
    g = lambda nm, s: store(normal(seed, f"{wl.name}/{tag}/{nm}", s, device=device), wl.dtype)
    if wl.ratio == 128:
        return {"C": g("C", sh), "Z": g("Z", sh)}
    out = {"C_a": g("C_a", sh), "C_b": g("C_b", sh), "Z_a": g("Z_a", sh), "Z_b": g("Z_b", sh)}
    chunk_start = wl.q_pos0 + wl.T - L
    if chunk_start > 0:
        out["prev_Cb"] = g("prev_Cb", (wl.B, wl.ratio, c))
        out["prev_Zb"] = g("prev_Zb", (wl.B, wl.ratio, c))
    return out


def draw_indexer(wl: Workload, seed: int = 0, device="cpu", N=None):
    """Index queries qI [B,T,Hi,di], head weights w [B,T,Hi] (fp32), index keys kI [B,N,di].
    qI / kI are drawn N(0,1) and stored in f32 (tiny) or bf16; the e4m3 variant is
    quantised from these draws by the code under test, not here."""
    N = wl.N if N is None else N
    sdt = "f32" if wl.index_dtype == "f32" else "bf16"
    qI = store(normal(seed, f"{wl.name}/qI", (wl.B, wl.T, wl.Hi, wl.di), device=device), sdt)
    kI = store(normal(seed, f"{wl.name}/kI", (wl.B, N, wl.di), device=device), sdt)
    if wl.w_dist == "uniform":
        w = uniform(seed, f"{wl.name}/w", (wl.B, wl.T, wl.Hi), device=device)
    else:
        w = normal(seed, f"{wl.name}/w", (wl.B, wl.T, wl.Hi), device=device)
    return {"qI": qI, "w": w, "kI": kI}


def draw_indexer_outliers(seed: int, B: int, T: int, N: int, Hi: int = 64, di: int = 128,
                          channels=(3, 40, 77, 100), key_offset: float = 20.0, q_gain: float = 8.0,
                          device="cpu"):
    """Index inputs with outlier channels, the regime a rotation before low-precision
    scoring is for: N(0,1) draws, then on the given channels every key gets a common
    offset and every query head a larger gain; bf16 storage.  w ~ N(0, 0.1^2) fp32.
    Returns {"qI" [B,T,Hi,di], "w" [B,T,Hi], "kI" [B,N,di]}."""
    tag = f"outliers/{B}x{T}x{N}"
    qI = normal(seed, f"{tag}/qI", (B, T, Hi, di), device=device)
    kI = normal(seed, f"{tag}/kI", (B, N, di), device=device)
    ch = torch.tensor(list(channels), dtype=torch.long, device=device)
    kI[..., ch] += key_offset
    qI[..., ch] *= q_gain
    w = normal(seed, f"{tag}/w", (B, T, Hi), std=0.1, device=device)
    return {"qI": store(qI, "bf16"), "w": w, "kI": store(kI, "bf16")}


def draw_attention(wl: Workload, seed: int = 0, device="cpu", N=None, tag="attn"):
    """Queries q [B,T,H,D], latent cache kv [B,N,D], raw SWA rows swa_kv [B,W,D]
    (absolute positions swa_pos0..swa_pos0+W-1), per-head sink logits [H] (fp32)."""
    N = wl.N if N is None else N
    g = lambda nm, s: store(normal(seed, f"{wl.name}/{tag}/{nm}", s, device=device), wl.dtype)
    return {"q": g("q", (wl.B, wl.T, wl.H, wl.D)), "kv": g("kv", (wl.B, N, wl.D)),
            "swa_kv": g("swa_kv", (wl.B, wl.W, wl.D)),
            "sink": normal(seed, f"{wl.name}/{tag}/sink", (wl.H,), device=device)}


def draw_scores(seed: int, name: str, B: int, T: int, N: int, ties: int = 0, device="cpu"):
    """Synthetic fp32 score rows for testing top-k on its own: N(0, 64^2) values
    (the spread of indexer scores on N(0,1) inputs), with ``ties`` groups of
    planted exact duplicates (including +0.0 / -0.0 pairs)."""
    s = normal(seed, name, (B, T, N), std=64.0, device=device)
    if ties and N > 4:
        pos = (uniform(seed, name + "/tiepos", (B, T, ties, 4)) * N).to(torch.int64).clamp_(0, N - 1)
        for b in range(B):
            for t in range(T):
                for g in range(ties):
                    p = pos[b, t, g].tolist()
                    v = s[b, t, p[0]].item()
                    for j in p[1:]:
                        s[b, t, j] = v
        s[:, :, 1] = 0.0
        s[:, :, 2] = -0.0
        s[:, :, 3] = 0.0
    return s
