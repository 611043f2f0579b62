// rope.cuh -- partial rotary position embedding of the last 64 dims of a row.
//
// "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §6: only the last 64 dims of each head
// carry RoPE; after the core attention the same dims of the output are turned back
// (inverse RoPE) before the grouped output projection.  The pages give no pairing, base
// or position rule, so (one reading, the same one the oracle states): the RoFormer
// rotation on the pairs (D-64+2i, D-64+2i+1), i < 32, by the angle pos * theta^(-2i/64),
// theta a parameter (the MXFP4 page's compress_rope_theta is 160000); a compressed entry
// i stands at position i * m, an SWA row and a query at their token positions.
//
// The angle is formed and reduced in fp64 (a position near 2^20 times a frequency near 1
// leaves no correct fractional bits in fp32); its cosine and sine and the rotation itself
// run in fp32, rounded once to the output type.
#pragma once
#include <cuda_bf16.h>
#include <cmath>
#include "ptx.cuh"

namespace csa {

constexpr int kRopeDims = 64;

// The 32 pair frequencies theta^(-2i/64), formed once on the host in fp64.
struct RopeFreqs {
  double f[kRopeDims / 2];
};
inline RopeFreqs rope_freqs(double theta) {
  RopeFreqs r;
  for (int i = 0; i < kRopeDims / 2; ++i) r.f[i] = std::pow(theta, -2.0 * (double)i / (double)kRopeDims);
  return r;
}

// cos and sin of the angle pos * freq (inverse: of minus that angle).  The angle is the fp64
// product pos * freq, brought into [-pi, pi] by subtracting the nearest multiple of 2 pi
// with a two-part 2 pi (Cody and Waite's additive reduction: the first fma is exact, so
// the reduced angle carries only the product's own rounding, about 2^-32 rad for angles
// below 2^21), then sincosf of the reduced angle.
__device__ __forceinline__ float2 rope_cs(int64_t pos, double freq, bool inverse) {
  constexpr double kTwoPiHi = 6.283185307179586;            // 2 pi rounded to fp64
  constexpr double kTwoPiLo = 2.4492935982947064e-16;       // 2 pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double a = (double)pos * freq;
  const double n = rint(a * kInvTwoPi);
  const double r = fma(-n, kTwoPiLo, fma(-n, kTwoPiHi, a));
  // sincosf of the fp32-rounded angle, corrected to first order by the rounding residual
  // dr (|dr| <= 2^-23: the neglected dr^2 / 2 term is below 2^-47)
  const float rf = (float)r;
  const float dr = (float)(r - (double)rf);
  float sn, cs;
  sincosf(rf, &sn, &cs);
  const float s1 = fmaf(cs, dr, sn), c1 = fmaf(-sn, dr, cs);
  return make_float2(c1, inverse ? -s1 : s1);
}

// (a, b) turned by the angle whose cosine and sine are cs.
__device__ __forceinline__ float2 rope_turn(float a, float b, float2 cs) {
  return make_float2(fmaf(a, cs.x, -b * cs.y), fmaf(a, cs.y, b * cs.x));
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float v, float* p) { *p = v; }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16* p) { *p = __float2bfloat16_rn(v); }

// Rows x [B, R, D] -> out (may be x): the first D-64 dims copied, the last 64 turned at
// position base[b] + r * stride.  One thread per (row, pair).
template <typename T>
__global__ void __launch_bounds__(256) rope_rows_kernel(const T* __restrict__ x, int64_t B, int64_t R, int D,
                                                       const int64_t* __restrict__ base, int64_t stride,
                                                       const RopeFreqs freqs, int inverse, T* out) {
  griddep_sync();
  const int64_t rows = B * R;
  const int64_t total = rows * (kRopeDims / 2);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(g % (kRopeDims / 2));
    const int64_t row = g / (kRopeDims / 2);
    const int64_t b = row / R, r = row % R;
    const int64_t pos = (base ? base[b] : 0) + r * stride;
    const int64_t o = row * D + (D - kRopeDims) + 2 * i;
    const float2 y = rope_turn(to_f(x[o]), to_f(x[o + 1]), rope_cs(pos, freqs.f[i], inverse != 0));
    from_f(y.x, out + o);
    from_f(y.y, out + o + 1);
  }
  if (x != out) {                                 // the unrotated dims, when not in place
    const int keep = D - kRopeDims;
    const int64_t tk = rows * keep;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < tk; g += (int64_t)gridDim.x * blockDim.x)
      out[(g / keep) * D + g % keep] = x[(g / keep) * D + g % keep];
  }
}

}  // namespace csa
