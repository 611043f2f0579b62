// index_topk.cuh -- the pieces of csa_index_topk (indexer scores and their top-k per
// row without writing the score matrix: "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文"
// §4.2, a cheap scan of every key with the expensive work kept to the top-k) other
// than the indexer itself (index_tc_kernel, plain and candidate mode):
//   sample_keys_kernel     every kSampleStride-th key row (and its e4m3 scale) of each
//                          sequence into a dense sample, and each row's sample n_valid
//                          = ceil(n_valid / kSampleStride)
//   cand_threshold_kernel  per row, the r-th largest key among the sampled scores: the
//                          row's candidate threshold (every sampled key at or above it is
//                          also a candidate of the full pass, so a row gets at least r);
//                          it also zeroes the row's candidate count and the call's
//                          failure count
//   cand_select_kernel     per row, the exact top-k of its candidate list (unordered
//                          (key << 32 | ~index) entries, zero = unused slot), written in
//                          ascending index order through a bitmap of the row; a row whose
//                          list is short (fewer than k entries) or overflowed is counted
//                          as failed, and the call then recomputes every row the plain way
#pragma once
#include "topk.cuh"

namespace csa {

constexpr int kSampleStride = 16;     // keys per sampled key
constexpr int kCandCapMax = 8192;     // candidate slots per row (shared memory of the select)
constexpr int kIndexTopkMaxK = 1024;  // sample threshold at rank max(48, 4k/16): ~4k candidates
// Candidate slots per row: min(kCandCapMax, max(4096, 16k)).  Reserved slots = candidates,
// plus (32-slot chunks, when a row spans at most two CTAs) at most 31 unused per
// contributing epilogue warp: at most 16r + 992 for a short row (every key a candidate),
// about 16r + 992 otherwise, r = max(48, 4k/16).

__global__ void __launch_bounds__(256) sample_keys_kernel(const uint8_t* __restrict__ kI,
                                                          const float* __restrict__ ks, int B, int64_t N,
                                                          int64_t Ns, int row_bytes, uint8_t* __restrict__ kI_s,
                                                          float* __restrict__ ks_s,
                                                          const int32_t* __restrict__ n_valid, int64_t rows,
                                                          int32_t* __restrict__ nv_s) {
  griddep_sync();
  const int per_row = row_bytes / 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n16 = (int64_t)B * Ns * per_row;
  for (int64_t j = t0; j < n16; j += stride) {
    const int64_t r = j / per_row;                   // sample row b * Ns + js
    const int c = (int)(j - r * per_row);
    const int64_t b = r / Ns, js = r - b * Ns;
    const uint4* src = reinterpret_cast<const uint4*>(kI + (b * N + js * kSampleStride) * row_bytes);
    reinterpret_cast<uint4*>(kI_s + r * row_bytes)[c] = __ldg(src + c);
  }
  if (ks) {
    for (int64_t j = t0; j < (int64_t)B * Ns; j += stride) {
      const int64_t b = j / Ns, js = j - b * Ns;
      ks_s[j] = __ldg(ks + b * N + js * kSampleStride);
    }
  }
  for (int64_t j = t0; j < rows; j += stride) {
    int nv = n_valid[j];
    nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
    nv_s[j] = (nv + kSampleStride - 1) / kSampleStride;
  }
}

// Radix select over keys in shared memory, 8 bits at a time from the top: after the pass
// at `shift`, prefix/pmask hold the chosen bits of u = key - base and rem the entries
// still to take among those that match them; returns true once every matching entry is
// taken (or the last digit is done).  Keys above base share their bits above the span's
// highest bit, so the first pass starts there and its digits spread over the bins; a
// warp adds to a bin once per distinct bin.  SKIP0: zero keys (unused slots) take no part.
// hist: 256 skewed bins; 256 threads.
template <typename K, bool SKIP0>
__device__ __forceinline__ bool radix_pass(const K* keys, int n, K base, int shift, K& prefix, K& pmask, int& rem,
                                           int* hist, int* scratch, int* res) {
  for (int j = threadIdx.x; j < 256 + 8; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  for (int j0 = 0; j0 < n; j0 += blockDim.x) {
    const int j = j0 + (int)threadIdx.x;
    const K v = j < n ? keys[j] : (K)0;
    const K u = v - base;
    const bool act = j < n && (!SKIP0 || v != (K)0) && (u & pmask) == prefix;
    warp_hist_add(hist, (uint32_t)skew((int)((u >> shift) & 255)), act);
  }
  __syncthreads();
  find_digit_skewed<1>(hist, 256, rem, res, scratch);
  __syncthreads();
  const int d = res[0];
  prefix |= (K)d << shift;
  pmask |= (K)255 << shift;
  rem -= res[1];
  const bool done = hist[skew(d)] == rem || shift == 0;
  __syncthreads();                                   // hist and res are read before the next pass
  return done;
}

// The smallest key of keys[0, n) and the shift of the first 8-bit digit that covers the
// highest bit of (largest - smallest) (0 when all keys are equal).  SKIP0: zero keys are
// left out.
template <typename K, bool SKIP0>
__device__ __forceinline__ int radix_start(const K* keys, int n, K* kmin_out, K* ext) {
  K lo = ~(K)0, hi = (K)0;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const K v = keys[j];
    if (SKIP0 && v == (K)0) continue;
    lo = v < lo ? v : lo;
    hi = v > hi ? v : hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const K a = __shfl_xor_sync(0xffffffffu, lo, o), b = __shfl_xor_sync(0xffffffffu, hi, o);
    lo = a < lo ? a : lo;
    hi = b > hi ? b : hi;
  }
  if (threadIdx.x == 0) {
    ext[0] = ~(K)0;
    ext[1] = (K)0;
  }
  __syncthreads();
  if (lane_id() == 0) {
    atomicMin(&ext[0], lo);
    atomicMax(&ext[1], hi);
  }
  __syncthreads();
  *kmin_out = ext[0];
  const K span = ext[1] - ext[0];
  __syncthreads();
  int top = 0;                                       // highest set bit of span, 0 if none
  for (int b = (int)sizeof(K) * 8 - 1; b > 0; --b)
    if ((span >> b) & (K)1) {
      top = b;
      break;
    }
  return top / 8 * 8;
}

// grid: one CTA of 256 threads per row; dynamic shared memory Ns * 4 bytes.
__global__ void __launch_bounds__(256) cand_threshold_kernel(const float* __restrict__ s_scores, int64_t Ns,
                                                             const int32_t* __restrict__ n_valid, int64_t N, int k,
                                                             int r0, uint32_t* __restrict__ thr,
                                                             int* __restrict__ cand_cnt, int* __restrict__ fail,
                                                             int32_t* __restrict__ failed_rows) {
  extern __shared__ __align__(16) uint32_t skeys[];
  __shared__ int hist[256 + 8];
  __shared__ int scratch[33];
  __shared__ int res[2];
  __shared__ uint32_t ext[2];
  griddep_sync();
  const int64_t row = blockIdx.x;
  if (row == 0 && threadIdx.x == 0) {
    *fail = 0;
    if (failed_rows) *failed_rows = 0;
  }
  if (threadIdx.x == 0) cand_cnt[row] = 0;
  int nv = n_valid[row];
  nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
  if (nv <= k) {                                     // every valid entry is taken: no candidates
    if (threadIdx.x == 0) thr[row] = 0xffffffffu;
    return;
  }
  const int ns = (int)((nv + kSampleStride - 1) / kSampleStride);   // valid samples, 1 .. Ns
  if (ns <= r0) {                                    // a short row: every valid key is a candidate
    if (threadIdx.x == 0) thr[row] = 0u;             // (at most kSampleStride * r0 = 4k of them)
    return;
  }
  const float* srow = s_scores + row * Ns;
  for (int j = threadIdx.x; j < ns; j += blockDim.x) skeys[j] = order_key(srow[j]);
  __syncthreads();
  uint32_t kmin;
  int shift = radix_start<uint32_t, false>(skeys, ns, &kmin, ext);
  uint32_t prefix = 0u, pmask = 0u;
  int rem = r0;
  while (!radix_pass<uint32_t, false>(skeys, ns, kmin, shift, prefix, pmask, rem, hist, scratch, res)) shift -= 8;
  // the r-th largest key: kmin + the prefix, low bits zero where the select stopped early
  // (every key sharing the prefix is at or above it, and the r-th largest is one of them)
  if (threadIdx.x == 0) thr[row] = kmin + prefix;
}

// grid: one CTA of 256 threads per row; dynamic shared memory cap * 8 + ceil(N / 32) * 4.
__global__ void __launch_bounds__(256) cand_select_kernel(const unsigned long long* __restrict__ cand,
                                                          const int* __restrict__ cand_cnt, int cap,
                                                          const int32_t* __restrict__ n_valid, int64_t N, int k,
                                                          int32_t* __restrict__ idx, int* __restrict__ fail,
                                                          int32_t* __restrict__ failed_rows) {
  extern __shared__ __align__(16) unsigned long long cs[];   // [cap] entries, then the row's bitmap
  __shared__ int hist[256 + 8];
  __shared__ int scratch[33];
  __shared__ int res[2];
  __shared__ int nzero;
  __shared__ unsigned long long ext[2];
  griddep_sync();
  const int64_t row = blockIdx.x;
  int nv = n_valid[row];
  nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
  int32_t* out = idx + row * k;
  if (nv <= k) {
    write_all_valid(out, nv, k);
    return;
  }
  const int c = __ldcg(cand_cnt + row);
  auto failed = [&]() {
    if (threadIdx.x == 0) {
      atomicAdd(fail, 1);
      if (failed_rows) atomicAdd(failed_rows, 1);
    }
  };
  if (c < k || c > cap) {                            // short list, or chunks past the capacity
    failed();
    return;
  }
  uint32_t* bm = reinterpret_cast<uint32_t*>(cs + cap);
  const int words = (nv + 31) >> 5;
  if (threadIdx.x == 0) nzero = 0;
  for (int j = threadIdx.x; j < words; j += blockDim.x) bm[j] = 0u;
  __syncthreads();
  const unsigned long long* crow = cand + row * cap;
  int z = 0;
  for (int j = threadIdx.x; j < c; j += blockDim.x) {
    const unsigned long long v = __ldcg(crow + j);
    cs[j] = v;
    z += v == 0ull;
  }
  z = __reduce_add_sync(0xffffffffu, z);
  if (lane_id() == 0 && z) atomicAdd(&nzero, z);
  __syncthreads();
  if (c - nzero < k) {                               // unused slots left fewer than k entries
    failed();
    return;
  }
  // the k-th largest entry (entries are distinct: the low word holds the index)
  unsigned long long kmin;
  int shift = radix_start<unsigned long long, true>(cs, c, &kmin, ext);
  unsigned long long prefix = 0ull, pmask = 0ull;
  int rem = k;
  while (!radix_pass<unsigned long long, true>(cs, c, kmin, shift, prefix, pmask, rem, hist, scratch, res))
    shift -= 8;
  // the k entries whose bits (above the last digit) are at or above the prefix, marked in
  // the row's bitmap
  for (int j = threadIdx.x; j < c; j += blockDim.x) {
    const unsigned long long v = cs[j];
    if (v != 0ull && ((v - kmin) & pmask) >= prefix) {
      const uint32_t i = ~(uint32_t)v;
      if (i < (uint32_t)nv) atomicOr(&bm[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();
  // ascending order: each thread takes a contiguous run of words after one block scan
  const int per = (words + (int)blockDim.x - 1) / (int)blockDim.x;
  const int w0 = (int)threadIdx.x * per;
  const int w1 = w0 + per < words ? w0 + per : words;
  int cntw = 0;
  for (int wd = w0; wd < w1; ++wd) cntw += __popc(bm[wd]);
  int total;
  int pos = block_excl_scan(cntw, scratch, &total);
  for (int wd = w0; wd < w1; ++wd) {
    uint32_t m = bm[wd];
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      if (pos < k) out[pos] = wd * 32 + b;
      ++pos;
    }
  }
  for (int j = total + (int)threadIdx.x; j < k; j += blockDim.x) out[j] = -1;   // (total == k)
}

}  // namespace csa
