// kv8.cuh -- mixed-precision storage of the compressed KV entries
// ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.2, storage precision: the RoPE
// dims stay BF16, the rest of each compressed entry is FP8): the quantiser and the
// exact conversion the attention loader uses.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace csa {

// Mixed-precision storage of the compressed KV entries ("DeepSeek-V4 混合注意力" §4.2,
// storage precision: the RoPE dims stay BF16, the rest of each entry is FP8).  Entry
// of D = 512 dims, 608 bytes:
//   [0, 448)   e4m3 codes of dims 0..447
//   [448, 576) bf16 RoPE dims 448..511 (bit copy)
//   [576, 604) fp32 scale of each 64-dim FP8 block: s = 2^e, e the smallest integer
//              with amax <= 448 * 2^e (e = 0 for an all-zero block)
//   [604, 608) zero
// code = round-to-nearest-even e4m3 of x * 2^-e (exact scaling, |x * 2^-e| <= 448).
constexpr int kKv8Dims = 512;
constexpr int kKv8Fp8Dims = kKv8Dims - 64;
constexpr int kKv8Bytes = 608;
constexpr int kKv8ScaleOff = kKv8Fp8Dims + 128;

// e of the block scale from the block's amax (a finite, non-negative fp32 value):
// with amax = M * 2^E, M in [1, 2): e = E - 8 if M <= 1.75, else E - 7.
__device__ __forceinline__ int kv8_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  const uint32_t u = __float_as_uint(amax);
  int E;
  uint32_t frac;                                   // M - 1 in units of 2^-23
  if ((u >> 23) != 0) {
    E = (int)(u >> 23) - 127;
    frac = u & 0x7FFFFFu;
  } else {                                         // subnormal: amax = f * 2^-149
    const int k = 31 - __clz(u);
    E = k - 149;
    frac = (u << (23 - k)) & 0x7FFFFFu;
  }
  return frac > 0x600000u ? E - 7 : E - 8;         // 1.75 = 1 + 0x600000 * 2^-23
}

// 2^e as fp32 (0 below the subnormal range, as a rounded conversion gives)
__device__ __forceinline__ float kv8_pow2(int e) {
  if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
  if (e >= -149) return __uint_as_float(1u << (e + 149));
  return 0.f;
}

// One warp per entry: lanes 0..27 quantise 16 FP8 dims each (4 lanes per 64-dim block),
// lanes 28..31 copy 16 RoPE dims each.
__global__ void __launch_bounds__(256) kv8_quantize_kernel(const __nv_bfloat16* __restrict__ kv, int64_t rows,
                                                           uint8_t* __restrict__ entries) {
  griddep_sync();
  const int lane = lane_id();
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint4* src = reinterpret_cast<const uint4*>(kv + r * kKv8Dims) + 2 * lane;   // 16 dims
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    uint8_t* e = entries + r * kKv8Bytes;
    float x[16];
    {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* g = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]), f2 = __bfloat1622float2(g[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
        x[8 + 2 * i] = f2.x;
        x[8 + 2 * i + 1] = f2.y;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));   // the 4 lanes of one block
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (lane < 28) {
      const int ex = kv8_scale_exp(amax);
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float y = ldexpf(x[4 * i + j], -ex);                 // exact
          const uint32_t c = (uint32_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
          word |= c << (8 * j);
        }
        w[i] = word;
      }
      *reinterpret_cast<uint4*>(e + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
      if ((lane & 3) == 0) reinterpret_cast<float*>(e + kKv8ScaleOff)[lane >> 2] = kv8_pow2(ex);
      if (lane == 0) *reinterpret_cast<uint32_t*>(e + kKv8ScaleOff + 28) = 0u;
    } else {
      uint4* dst = reinterpret_cast<uint4*>(e + kKv8Fp8Dims + 32 * (lane - 28));
      dst[0] = a;
      dst[1] = b;
    }
  }
}

// Two e4m3 codes (bits 0..15 of `two`, the lower byte first) times the power-of-two
// scale sc, as a bf16 pair (lower dim in the low half).  Exact: e4m3 -> f16 -> f32 are
// exact widenings, the scaling is by 2^e, and 4 significant bits fit in bf16.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two, float sc) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  __half2 h;
  *reinterpret_cast<__half2_raw*>(&h) = hr;
  const float2 f = __half22float2(h);
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * sc, f.y * sc);
  return *reinterpret_cast<const uint32_t*>(&b);
}

}  // namespace csa
