// compress.cuh -- token-level Compressor: softmax-gated pooling of raw rows
// into compressed entries, per channel.
//
// "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.1 (CSA, ratio 4, two
// overlapped branches: entry i pools the b-branch rows of block i-1 and the
// a-branch rows of block i over 2m positions) and §5 (HCA, ratio 128, one
// branch, the m rows of block i).  Rows are 0-based; a chunk that does not
// start at position 0 passes the b-branch rows of the preceding block as a
// carry; entry 0 without a carry pools its a rows only; a partial trailing
// block yields no entry.
//
// A streaming reduction: each raw value is read exactly once with 16-byte
// loads (8 bf16 or 4 fp32 channels), the softmax and weighted sum run in fp32
// registers, and the entry is written once.  HBM-bound.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace csa {

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* v) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void load8(const float* p, float* v) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* v) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ void store8(float* p, const float* v) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ void load2(const __nv_bfloat16* p, float* v) {
  const float2 f = __bfloat1622float2(__ldg(reinterpret_cast<const __nv_bfloat162*>(p)));
  v[0] = f.x;
  v[1] = f.y;
}
__device__ __forceinline__ void load2(const float* p, float* v) {
  const float2 f = __ldg(reinterpret_cast<const float2*>(p));
  v[0] = f.x;
  v[1] = f.y;
}
__device__ __forceinline__ void store2(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
}
__device__ __forceinline__ void store2(float* p, const float* v) {
  *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}
template <int CH, typename T>
__device__ __forceinline__ void load_ch(const T* p, float* v) {
  if constexpr (CH == 8) load8(p, v); else load2(p, v);
}
template <int CH, typename T>
__device__ __forceinline__ void store_ch(T* p, const float* v) {
  if constexpr (CH == 8) store8(p, v); else store2(p, v);
}

constexpr float kCompLog2e = 1.4426950408889634f;

// One channel j of one CSA entry: softmax over positions r0 .. 2M-1 of the logits z[r][j]
// (base-2 domain), weighted sum of the contents v[r][j].  Every CSA compressor kernel
// takes its entries from here, so they agree bit for bit.
template <int M, int CH>
__device__ __forceinline__ float pool_channel(float (&z)[2 * M][CH], const float (&v)[2 * M][CH], int j, int r0) {
  float mx = -INFINITY;
#pragma unroll
  for (int r = 0; r < 2 * M; ++r)
    if (r >= r0) {
      z[r][j] *= kCompLog2e;
      mx = fmaxf(mx, z[r][j]);
    }
  float den = 0.f, acc = 0.f;
#pragma unroll
  for (int r = 0; r < 2 * M; ++r) {
    if (r < r0) continue;
    const float e = ex2_approx(z[r][j] - mx);
    den += e;
    acc = fmaf(e, v[r][j], acc);
  }
  return acc / den;
}

// CSA (ratio m = 4): one thread per (sequence, entry, group of CH channels):
// CH = 8 (16-byte loads) when there are enough entries to fill the GPU, CH = 2
// otherwise (a decode step compresses a single block per sequence).  All 2m
// rows are loaded before use; the softmax runs in the base-2 domain.
// Layouts: C_a, C_b, Z_a, Z_b [B, L, c]; prev_Cb, prev_Zb [B, m, c] or null;
// out [B, L/m, c].
template <typename Tin, typename Tout, int M, int CH>
__global__ void __launch_bounds__(256) compress_csa_kernel(const Tin* __restrict__ Ca, const Tin* __restrict__ Cb,
                                                           const Tin* __restrict__ Za, const Tin* __restrict__ Zb,
                                                           const Tin* __restrict__ pCb,
                                                           const Tin* __restrict__ pZb, int B, int64_t L, int c,
                                                           Tout* __restrict__ out) {
  griddep_sync();
  // 32-bit index arithmetic (the host guarantees B * L/M * c/CH < 2^31)
  const uint32_t groups = (uint32_t)c / CH;
  const uint32_t n_entries = (uint32_t)(L / M);
  const uint32_t total = (uint32_t)B * n_entries * groups;
  for (uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x; gid < total; gid += gridDim.x * blockDim.x) {
    const int g = (int)(gid % groups);
    const uint32_t rest = gid / groups;
    const int64_t i = rest % n_entries;
    const int b = (int)(rest / n_entries);
    const int ch = g * CH;
    float z[2 * M][CH], v[2 * M][CH];
    bool has_b = true;
#pragma unroll
    for (int r = 0; r < M; ++r) {
      if (i > 0) {
        const int64_t off = ((int64_t)b * L + (i - 1) * M + r) * c + ch;
        load_ch<CH>(Zb + off, z[r]);
        load_ch<CH>(Cb + off, v[r]);
      } else if (pZb != nullptr) {
        const int64_t off = ((int64_t)b * M + r) * c + ch;
        load_ch<CH>(pZb + off, z[r]);
        load_ch<CH>(pCb + off, v[r]);
      } else {
        has_b = false;
      }
      const int64_t aoff = ((int64_t)b * L + i * M + r) * c + ch;
      load_ch<CH>(Za + aoff, z[M + r]);
      load_ch<CH>(Ca + aoff, v[M + r]);
    }
    const int r0 = has_b ? 0 : M;
    float res[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) res[j] = pool_channel<M, CH>(z, v, j, r0);
    store_ch<CH>(out + ((int64_t)b * n_entries + i) * c + ch, res);
  }
}

// HCA (ratio 128): one CTA per (sequence, entry, block of 64 channels); 256
// threads = 8 groups of 8 channels (16-byte loads, a warp covers 128-byte row
// segments) x 32 row groups of 4 rows.  Every thread loads its 4 rows at once,
// reduces them to a softmax state (max, sum of exponentials, weighted sum) per
// channel, and 64 threads merge the 32 row-group states through shared memory.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) compress_hca_kernel(const Tin* __restrict__ C, const Tin* __restrict__ Z,
                                                           int B, int64_t L, int c, Tout* __restrict__ out) {
  griddep_sync();
  constexpr int M = 128, CH = 8, CG = 8, RG = 32, RPT = M / RG;
  constexpr int PAD = CG * CH + 1;               // conflict-free partial stores and merge reads
  __shared__ float pm[RG][PAD], ps[RG][PAD], pa[RG][PAD];
  const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
  const int64_t n_entries = L / M;
  const int64_t i = blockIdx.y;
  const int b = blockIdx.z;
  const int ch0 = blockIdx.x * CG * CH;
  const int ch = ch0 + cg * CH;
  if (ch < c) {
    const int64_t base = ((int64_t)b * L + i * M) * c + ch;
    float z[RPT][CH], v[RPT][CH];
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      const int64_t off = base + (int64_t)(rg + u * RG) * c;
      load8(Z + off, z[u]);
      load8(C + off, v[u]);
    }
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float m = -INFINITY;
#pragma unroll
      for (int u = 0; u < RPT; ++u) {
        z[u][j] *= kCompLog2e;
        m = fmaxf(m, z[u][j]);
      }
      float sum = 0.f, acc = 0.f;
#pragma unroll
      for (int u = 0; u < RPT; ++u) {
        const float e = ex2_approx(z[u][j] - m);
        sum += e;
        acc = fmaf(e, v[u][j], acc);
      }
      pm[rg][cg * CH + j] = m;
      ps[rg][cg * CH + j] = sum;
      pa[rg][cg * CH + j] = acc;
    }
  }
  __syncthreads();
  const int t = threadIdx.x;
  if (t < CG * CH && ch0 + t < c) {
    float mx = -INFINITY;
#pragma unroll 8
    for (int q = 0; q < RG; ++q) mx = fmaxf(mx, pm[q][t]);
    float sum = 0.f, acc = 0.f;
#pragma unroll 8
    for (int q = 0; q < RG; ++q) {
      const float f = ex2_approx(pm[q][t] - mx);
      sum = fmaf(ps[q][t], f, sum);
      acc = fmaf(pa[q][t], f, acc);
    }
    const float r = acc / sum;
    Tout* o = out + ((int64_t)b * n_entries + i) * c + ch0 + t;
    if constexpr (sizeof(Tout) == 2) *o = __float2bfloat16_rn(r); else *o = r;
  }
}

}  // namespace csa
