// append.cuh -- new index-key entries written straight into the indexer's caches.
//
// One launch does, for each new entry of each sequence:
//   1. the 4:1 overlapped compressor over the c = 128 index-key channels
//      ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.1; the Indexer compresses its
//      own keys, §7 call chain), with the per-channel arithmetic of compress_csa_kernel
//      (pool_channel), so the entry equals csa_compress's bit for bit;
//   2. the entry rounded to bf16: the stored key, read by the exact rescoring;
//   3. that bf16 row, optionally Walsh-Hadamard-rotated ("揭秘DeepSeek-V4-Pro-MXFP4稀疏
//      注意力…", the Indexer paragraph), quantised to e4m3 with its per-row scale (§4.2:
//      the index QK runs in low precision) exactly as csa_quantize_e4m3(_hadamard) does.
// One warp per (sequence, entry); lane l holds channels 4l .. 4l+3, so the rotation's
// butterflies over the low two index bits run inside the lane and the other five across
// lanes (exact fp64 sums: the order of the additions cannot change a bit).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include "compress.cuh"
#include "quantize.cuh"

namespace csa {

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* v) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  v[0] = __uint_as_float(u.x << 16);
  v[1] = __uint_as_float(u.x & 0xffff0000u);
  v[2] = __uint_as_float(u.y << 16);
  v[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* p, float* v) {
  const float4 f = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

// Entry i of sequence b -> row pos0 + i of kI [B, ncap, 128] bf16, and (k8 != null) of
// k8 [B, ncap, 128] e4m3 and ks [B, ncap] fp32.  Raw rows as in compress_csa_kernel:
// C_a, C_b, Z_a, Z_b [B, L, 128]; prev_Cb, prev_Zb [B, 4, 128] or null.
template <typename Tin>
__global__ void __launch_bounds__(256) compress_index_keys_kernel(
    const Tin* __restrict__ Ca, const Tin* __restrict__ Cb, const Tin* __restrict__ Za, const Tin* __restrict__ Zb,
    const Tin* __restrict__ pCb, const Tin* __restrict__ pZb, int B, int64_t L, int hadamard, int64_t ncap,
    int64_t pos0, __nv_bfloat16* __restrict__ kI, uint8_t* __restrict__ k8, float* __restrict__ ks) {
  griddep_sync();
  constexpr int M = 4, C = 128, CH = 4;
  const int64_t n_entries = L / M;
  const int64_t total = (int64_t)B * n_entries;
  const int lane = (int)lane_id();
  const int ch = lane * CH;
  const double hc = __ddiv_rn(1.0, __dsqrt_rn((double)C));
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t wi = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp_id(); wi < total; wi += warps) {
    const int64_t i = wi % n_entries;
    const int b = (int)(wi / n_entries);
    float z[2 * M][CH], v[2 * M][CH];
    bool has_b = true;
#pragma unroll
    for (int r = 0; r < M; ++r) {
      if (i > 0) {
        const int64_t off = ((int64_t)b * L + (i - 1) * M + r) * C + ch;
        load4(Zb + off, z[r]);
        load4(Cb + off, v[r]);
      } else if (pZb != nullptr) {
        const int64_t off = ((int64_t)b * M + r) * C + ch;
        load4(pZb + off, z[r]);
        load4(pCb + off, v[r]);
      } else {
        has_b = false;
      }
      const int64_t aoff = ((int64_t)b * L + i * M + r) * C + ch;
      load4(Za + aoff, z[M + r]);
      load4(Ca + aoff, v[M + r]);
    }
    const int r0 = has_b ? 0 : M;
    float res[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) res[j] = pool_channel<M, CH>(z, v, j, r0);
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(res[0], res[1]);
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(res[2], res[3]);
    const int64_t row = (int64_t)b * ncap + pos0 + i;
    uint2 st;
    st.x = *reinterpret_cast<const uint32_t*>(&h0);
    st.y = *reinterpret_cast<const uint32_t*>(&h1);
    *reinterpret_cast<uint2*>(kI + row * C + ch) = st;
    if (k8 == nullptr) continue;
    // quantise the stored bf16 row
    double dv[CH] = {(double)__low2float(h0), (double)__high2float(h0), (double)__low2float(h1),
                     (double)__high2float(h1)};
    float y[CH];
    if (hadamard) {
      hadamard_lane_part<CH, 32>(dv, lane, hc, y);
    } else {
#pragma unroll
      for (int e = 0; e < CH; ++e) y[e] = (float)dv[e];
    }
    float amax = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < CH; ++e)
      word |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(y[e], s), __NV_SATFINITE, __NV_E4M3) << (8 * e);
    *reinterpret_cast<uint32_t*>(k8 + row * C + ch) = word;
    if (lane == 0) ks[row] = s;
  }
}

}  // namespace csa
