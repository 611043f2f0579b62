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
// The angle is formed and its cosine and sine taken in fp64 (a position near 2^20 times
// a frequency near 1 leaves no correct fractional bits in fp32); the rotation itself runs
// in fp32 on the stored values and is rounded once to the output type.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace csa {

constexpr int kRopeDims = 64;

// cos and sin of pos * theta^(-2i/64) (inverse: of minus that angle).
__device__ __forceinline__ float2 rope_cs(int64_t pos, int i, double theta, bool inverse) {
  const double freq = pow(theta, -2.0 * (double)i / (double)kRopeDims);
  double s, c;
  sincos((double)pos * freq, &s, &c);
  return make_float2((float)c, inverse ? -(float)s : (float)s);
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
                                                       const int64_t* __restrict__ base, int64_t stride, double theta,
                                                       int inverse, T* out) {
  griddep_sync();
  const int64_t rows = B * R;
  const int64_t total = rows * (kRopeDims / 2);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(g % (kRopeDims / 2));
    const int64_t row = g / (kRopeDims / 2);
    const int64_t b = row / R, r = row % R;
    const int64_t pos = (base ? base[b] : 0) + r * stride;
    const int64_t o = row * D + (D - kRopeDims) + 2 * i;
    const float2 y = rope_turn(to_f(x[o]), to_f(x[o + 1]), rope_cs(pos, i, theta, inverse != 0));
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
