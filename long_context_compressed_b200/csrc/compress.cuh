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

// CSA (ratio m = 4): one thread per (sequence, entry, group of 8 channels).
// Layouts: C_a, C_b, Z_a, Z_b [B, L, c]; prev_Cb, prev_Zb [B, m, c] or null;
// out [B, L/m, c].
template <typename Tin, typename Tout, int M>
__global__ void __launch_bounds__(256) compress_csa_kernel(const Tin* __restrict__ Ca, const Tin* __restrict__ Cb,
                                                           const Tin* __restrict__ Za, const Tin* __restrict__ Zb,
                                                           const Tin* __restrict__ pCb,
                                                           const Tin* __restrict__ pZb, int B, int64_t L, int c,
                                                           Tout* __restrict__ out) {
  griddep_sync();
  // 32-bit index arithmetic (the host guarantees B * L/M * c/8 < 2^31)
  const uint32_t groups = (uint32_t)c >> 3;
  const uint32_t n_entries = (uint32_t)(L / M);
  const uint32_t total = (uint32_t)B * n_entries * groups;
  for (uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x; gid < total; gid += gridDim.x * blockDim.x) {
    const int g = (int)(gid % groups);
    const uint32_t rest = gid / groups;
    const int64_t i = rest % n_entries;
    const int b = (int)(rest / n_entries);
    const int ch = g * 8;
    float z[2 * M][8], v[2 * M][8];
    bool has_b = true;
#pragma unroll
    for (int r = 0; r < M; ++r) {
      if (i > 0) {
        const int64_t off = ((int64_t)b * L + (i - 1) * M + r) * c + ch;
        load8(Zb + off, z[r]);
        load8(Cb + off, v[r]);
      } else if (pZb != nullptr) {
        const int64_t off = ((int64_t)b * M + r) * c + ch;
        load8(pZb + off, z[r]);
        load8(pCb + off, v[r]);
      } else {
        has_b = false;
      }
      const int64_t aoff = ((int64_t)b * L + i * M + r) * c + ch;
      load8(Za + aoff, z[M + r]);
      load8(Ca + aoff, v[M + r]);
    }
    const int r0 = has_b ? 0 : M;
    float res[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < 2 * M; ++r)
        if (r >= r0) mx = fmaxf(mx, z[r][j]);
      float den = 0.f, acc = 0.f;
#pragma unroll
      for (int r = 0; r < 2 * M; ++r) {
        if (r < r0) continue;
        const float e = expf(z[r][j] - mx);
        den += e;
        acc = fmaf(e, v[r][j], acc);
      }
      res[j] = acc / den;
    }
    store8(out + ((int64_t)b * n_entries + i) * c + ch, res);
  }
}

// HCA (ratio 128): one CTA per (sequence, entry, block of channels).  Inside
// the CTA, 8-channel groups run along threadIdx.x (coalesced rows) and the 128
// rows are split over row groups; each thread keeps an online softmax state
// (running max, sum of exponentials, weighted sum) over chunks of 8 rows, and
// the row groups merge through shared memory.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) compress_hca_kernel(const Tin* __restrict__ C, const Tin* __restrict__ Z,
                                                           int B, int64_t L, int c, Tout* __restrict__ out) {
  griddep_sync();
  constexpr int M = 128;
  constexpr int CH = 8;
  const int groups = c >> 3;
  const int G = groups < 64 ? groups : 64;       // channel groups per CTA
  const int RG = 256 / G;                        // row groups
  const int tg = threadIdx.x % G;
  const int rg = threadIdx.x / G;
  const int64_t n_entries = L / M;
  const int64_t i = blockIdx.y;
  const int b = blockIdx.z;
  const int ch = (blockIdx.x * G + tg) * CH;
  __shared__ float part[256][3 * CH];

  float m[CH], s[CH], a[CH];
#pragma unroll
  for (int j = 0; j < CH; ++j) { m[j] = -INFINITY; s[j] = 0.f; a[j] = 0.f; }
  const bool active = rg < RG && ch < c;
  if (active) {
    const int rows_per = M / RG;                 // RG divides 128
    const int64_t base = ((int64_t)b * L + i * M) * c + ch;
    for (int r0 = 0; r0 < rows_per; r0 += 8) {
      float z[8][CH], v[8][CH];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int row = rg + (r0 + u) * RG;
        load8(Z + base + (int64_t)row * c, z[u]);
        load8(C + base + (int64_t)row * c, v[u]);
      }
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        float cm = z[0][j];
#pragma unroll
        for (int u = 1; u < 8; ++u) cm = fmaxf(cm, z[u][j]);
        const float nm = fmaxf(m[j], cm);
        const float sc = expf(m[j] - nm);        // 0 on the first chunk (m = -inf)
        float ss = s[j] * sc, aa = a[j] * sc;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float e = expf(z[u][j] - nm);
          ss += e;
          aa = fmaf(e, v[u][j], aa);
        }
        m[j] = nm; s[j] = ss; a[j] = aa;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    part[threadIdx.x][j] = m[j];
    part[threadIdx.x][CH + j] = s[j];
    part[threadIdx.x][2 * CH + j] = a[j];
  }
  __syncthreads();
  if (rg == 0 && ch < c) {
    float res[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float mx = -INFINITY;
      for (int q = 0; q < RG; ++q) mx = fmaxf(mx, part[q * G + tg][j]);
      float ss = 0.f, aa = 0.f;
      for (int q = 0; q < RG; ++q) {
        const float sc = expf(part[q * G + tg][j] - mx);
        ss = fmaf(part[q * G + tg][CH + j], sc, ss);
        aa = fmaf(part[q * G + tg][2 * CH + j], sc, aa);
      }
      res[j] = aa / ss;
    }
    store8(out + ((int64_t)b * n_entries + i) * c + ch, res);
  }
}

}  // namespace csa
