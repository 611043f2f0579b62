// quantize.cuh -- per-row symmetric e4m3 quantisation for the low-precision
// index QK path ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.2: the index
// QK product runs in low precision; the pages use FP4, this library offers an
// OCP e4m3 variant).  scale = amax / 448 (fp32, IEEE division), code =
// round-to-nearest-even e4m3 of x / scale with saturation to +-448; an
// all-zero row gets scale 1.  One warp per row.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace csa {

__device__ __forceinline__ float load_as_float(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

template <typename Tin>
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const Tin* __restrict__ x, int64_t rows, int cols,
                                                            uint8_t* __restrict__ codes, float* __restrict__ scale) {
  griddep_sync();
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const Tin* xr = x + r * cols;
    float amax = 0.f;
    for (int j = lane_id(); j < cols; j += 32) amax = fmaxf(amax, fabsf(load_as_float(xr, j)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
    for (int j = lane_id(); j < cols; j += 32) {
      const float y = __fdiv_rn(load_as_float(xr, j), s);
      __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
      codes[r * cols + j] = static_cast<uint8_t>(c);
    }
    if (lane_id() == 0) scale[r] = s;
  }
}

}  // namespace csa
