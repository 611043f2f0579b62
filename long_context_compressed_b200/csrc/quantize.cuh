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

// Hadamard-rotated variant for the index vectors ("揭秘DeepSeek-V4-Pro-MXFP4稀疏注意力：
// 哈希索引与DSA如何撑起1M超长上下文？", the Indexer paragraph: the index query is
// Hadamard-rotated before it is scored; the keys take the same rotation, which leaves
// <q, k> unchanged and spreads outlier channels before the e4m3 rounding).
// Row of N values: y = H_N x with H_N the Sylvester-ordered Walsh-Hadamard matrix, by
// the fast transform in fp64.  LPR = N / E lanes share a row, lane g of the row holding
// the E contiguous elements g*E .. g*E+E-1 (16-byte loads and stores): the log2(E)
// butterflies over the low index bits run inside the lane, the log2(LPR) over the high
// bits across lanes (shuffles); butterflies over different bits commute.  Every partial
// sum is an exact fp64 value while the row spans at most 53 - (significand bits) -
// log2(N) binary orders, so the order of the additions does not matter.  Then
// y * (1/sqrt(N)) in fp64, rounded to fp32 (a zero becomes +0), and the per-row
// quantiser above.  x and codes are 16-byte aligned (checked by the caller).  Each pass of
// the grid-stride loop requests the next pass's rows before it transforms its own.
template <int N>
struct HadamardCfg {
  static constexpr int E = N / 4 < 16 ? N / 4 : 16;   // elements per lane (registers)
  static constexpr int LPR = N / E;                    // lanes per row: 4, 8 or 16
  static constexpr int RPW = 32 / LPR;              // rows per warp
};

// 16 raw bytes -> doubles (exact widening)
__device__ __forceinline__ void widen16(const uint4 u, double* v, const __nv_bfloat16*) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = (double)__uint_as_float(w[j] << 16);
    v[2 * j + 1] = (double)__uint_as_float(w[j] & 0xffff0000u);
  }
}
__device__ __forceinline__ void widen16(const uint4 u, double* v, const float*) {
  v[0] = (double)__uint_as_float(u.x);
  v[1] = (double)__uint_as_float(u.y);
  v[2] = (double)__uint_as_float(u.z);
  v[3] = (double)__uint_as_float(u.w);
}

// The butterflies of one row part (E elements per lane, LPR lanes per row, g = lane in the
// row), then y = v * c rounded to fp32 with a zero as +0.
template <int E, int LPR>
__device__ __forceinline__ void hadamard_lane_part(double* v, int g, double c, float* y) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        const double a = v[e], b = v[e + h];
        v[e] = __dadd_rn(a, b);
        v[e + h] = __dsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < LPR; m <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const double o = __shfl_xor_sync(0xffffffffu, v[e], m);
      v[e] = (g & m) ? __dsub_rn(o, v[e]) : __dadd_rn(v[e], o);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) y[e] = __double2float_rn(__dadd_rn(__dmul_rn(v[e], c), 0.0));
}

template <typename Tin, int N>
__global__ void __launch_bounds__(256, 2) hadamard_quantize_e4m3_kernel(const Tin* __restrict__ x, int64_t rows,
                                                                        uint8_t* __restrict__ codes,
                                                                        float* __restrict__ scale) {
  using C = HadamardCfg<N>;
  constexpr int E = C::E, LPR = C::LPR, RPW = C::RPW;
  constexpr int VEC = 16 / (int)sizeof(Tin);   // elements per 16-byte load
  constexpr int NV = E / VEC;                  // 16-byte loads per lane and row
  griddep_sync();
  const double c = __ddiv_rn(1.0, __dsqrt_rn((double)N));
  const int lane = (int)lane_id();
  const int g = lane % LPR;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 5) * RPW;
  // the raw bytes of the next rows are requested before the current rows are transformed
  auto fetch = [&](int64_t rr, uint4* dst) {
#pragma unroll
    for (int k = 0; k < NV; ++k)
      dst[k] = rr < rows ? __ldg(reinterpret_cast<const uint4*>(x + rr * N + g * E + k * VEC)) : make_uint4(0, 0, 0, 0);
  };
  int64_t r0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW;
  uint4 raw[NV];
  fetch(r0 + lane / LPR, raw);
  for (; r0 < rows; r0 += step) {
    const int64_t r = r0 + lane / LPR;
    uint4 nxt[NV];
    fetch(r + step, nxt);
    double v[E];
#pragma unroll
    for (int k = 0; k < NV; ++k) widen16(raw[k], v + k * VEC, x);
    float y[E];
    hadamard_lane_part<E, LPR>(v, g, c, y);
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
    for (int m = 1; m < LPR; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
    if (r < rows) {
      uint32_t packed[E / 4];
#pragma unroll
      for (int q = 0; q < E / 4; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          word |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(y[4 * q + j], s), __NV_SATFINITE, __NV_E4M3) << (8 * j);
        packed[q] = word;
      }
      uint8_t* cr = codes + r * N + g * E;
      if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(cr) = make_uint2(packed[0], packed[1]);
      } else {
#pragma unroll
        for (int q = 0; q < E / 4; q += 4)
          *reinterpret_cast<uint4*>(cr + 4 * q) = make_uint4(packed[q], packed[q + 1], packed[q + 2], packed[q + 3]);
      }
      if (g == 0) scale[r] = s;
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) raw[k] = nxt[k];
  }
}

// MXFP4 operands for the FP4 index QK ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §2
// table and §4.2: the index QK runs in FP4).  OCP MX: E2M1 elements with one E8M0 scale
// per 32 consecutive values, X = 2^(floor(log2 amax) - 2) clamped to 2^-127 .. 2^127 (an
// all-zero block: X = 1); element = nearest E2M1 value of y / X, ties to the even
// mantissa, saturating at 6.  With ROT the rows are first Walsh-Hadamard-rotated exactly
// as in hadamard_quantize_e4m3_kernel.  Layout: codes [rows, N/2] bytes, element 2j in
// the low nibble and 2j+1 in the high nibble; scales [rows, N/32] E8M0 bytes.

// Nearest E2M1 magnitude code of a >= 0: the count of rounding thresholds passed, where a
// tie (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) goes to the code with mantissa bit 0.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  const uint32_t m = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                     (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.0f);
  return (signbit(v) ? 8u : 0u) | m;
}

// Byte offset of E8M0 scale s (block of 32 values) of row i of a sequence's rows in the
// tensor-core scale layout: rows in tiles of 128, each tile one 512-byte atom holding row
// m = m0 + 32 m1 at byte 16 m0 + 4 m1 + s (the layout tcgen05.cp .32x128b.warpx4 moves into
// tensor memory as 4 columns: row m's four scales in column m1 of lane m0).
__device__ __forceinline__ int64_t sf128_offset(int64_t b, int64_t i, int s, int64_t tiles_per_batch) {
  const int m = (int)(i & 127);
  return (b * tiles_per_batch + (i >> 7)) * 512 + 16 * (m & 31) + 4 * (m >> 5) + s;
}

// rpb > 0: the scales go to the tensor-core layout above, rows counted per batch of rpb
// rows (N = 128 only); rpb == 0: scales [rows, N/32].
template <typename Tin, int N, bool ROT>
__global__ void __launch_bounds__(256, 2) quantize_mxfp4_kernel(const Tin* __restrict__ x, int64_t rows,
                                                                uint8_t* __restrict__ codes,
                                                                uint8_t* __restrict__ scales, int64_t rpb) {
  using C = HadamardCfg<N>;
  constexpr int E = C::E, LPR = C::LPR, RPW = C::RPW;
  constexpr int VEC = 16 / (int)sizeof(Tin);
  constexpr int NV = E / VEC;
  constexpr int LPB = 32 / E;                  // lanes per 32-value block
  static_assert(E % 8 == 0 && 32 % E == 0, "a lane holds a whole number of bytes of one block");
  griddep_sync();
  const double c = __ddiv_rn(1.0, __dsqrt_rn((double)N));
  const int lane = (int)lane_id();
  const int g = lane % LPR;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 5) * RPW;
  auto fetch = [&](int64_t rr, uint4* dst) {
#pragma unroll
    for (int k = 0; k < NV; ++k)
      dst[k] = rr < rows ? __ldg(reinterpret_cast<const uint4*>(x + rr * N + g * E + k * VEC)) : make_uint4(0, 0, 0, 0);
  };
  int64_t r0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW;
  uint4 raw[NV];
  fetch(r0 + lane / LPR, raw);
  for (; r0 < rows; r0 += step) {
    const int64_t r = r0 + lane / LPR;
    uint4 nxt[NV];
    fetch(r + step, nxt);
    double v[E];
#pragma unroll
    for (int k = 0; k < NV; ++k) widen16(raw[k], v + k * VEC, x);
    float y[E];
    if constexpr (ROT) {
      hadamard_lane_part<E, LPR>(v, g, c, y);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) y[e] = (float)v[e];      // exact: v holds widened inputs
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
    for (int m = 1; m < LPB; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    int ex = 0;
    if (amax > 0.f) {
      int E2;
      frexpf(amax, &E2);                          // amax = f 2^E2, f in [0.5, 1)
      ex = E2 - 3;
      ex = ex < -127 ? -127 : (ex > 127 ? 127 : ex);
    }
    if (r < rows) {
      uint32_t packed[E / 8];
#pragma unroll
      for (int q = 0; q < E / 8; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) word |= e2m1_code(ldexpf(y[8 * q + j], -ex)) << (4 * j);
        packed[q] = word;
      }
      uint8_t* cr = codes + (r * N + g * E) / 2;
      if constexpr (E == 8) {
        *reinterpret_cast<uint32_t*>(cr) = packed[0];
      } else {
        *reinterpret_cast<uint2*>(cr) = make_uint2(packed[0], packed[1]);
      }
      if (g % LPB == 0) {
        if (rpb > 0)
          scales[sf128_offset(r / rpb, r % rpb, g / LPB, (rpb + 127) >> 7)] = (uint8_t)(ex + 127);
        else
          scales[r * (N / 32) + g / LPB] = (uint8_t)(ex + 127);
      }
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) raw[k] = nxt[k];
  }
}

}  // namespace csa
