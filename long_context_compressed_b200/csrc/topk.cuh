// topk.cuh -- exact top-k selection over fp32 score rows.
//
// For each row (b, t): the k largest s[i] over i < n_valid, ties resolved
// toward the lower index, returned in ascending index order and padded with
// -1 when n_valid < k ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.2 and
// §7: topk(scores, k), k = 512 Flash / 1024 Pro).  -0.0 and +0.0 are the same
// value.  NaN scores are not supported.
//
// Scores become order-preserving uint32 keys; a most-significant-digit radix
// select finds the exact k-th key K* and how many keys equal to K* are taken
// (r); a final pass in index order takes every key > K* and the first r keys
// == K*, with block-wide prefix sums giving each selected index its output
// slot, so the output is ascending without a sort.
//
//  topk_row_kernel    one CTA per row, the row's keys resident in shared memory
//                     (rows up to kRowSmemMax keys); four 8-bit digit passes.
//  topk_hist_kernel + topk_gather_select_kernel
//                     chunk-parallel path for long rows: a 12-bit histogram of
//                     the whole row, every chunk appends the keys at or above
//                     the threshold bin to a candidate list, and the last CTA
//                     to finish selects exactly among the candidates and writes
//                     the row through index bitmaps.  It leaves its workspace
//                     zeroed for the next call (no inter-CTA waiting).
#pragma once
#include "ptx.cuh"

namespace csa {

constexpr int kRowSmemMax = 32768;
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kChunk = 4096;

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0) u = 0;                       // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive warp scan.
__device__ __forceinline__ int warp_incl_scan(int v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if ((int)lane_id() >= o) v += n;
  }
  return v;
}

// Block-wide exclusive scan (blockDim.x a multiple of 32, <= 1024); returns the
// exclusive prefix and writes the block total to *total.  Uses scratch[32].
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int inc = warp_incl_scan(v);
  const int nw = blockDim.x >> 5;
  __syncthreads();
  if (lane_id() == 31) scratch[warp_id()] = inc;
  __syncthreads();
  if (warp_id() == 0) {
    const int x = ((int)lane_id() < nw) ? scratch[lane_id()] : 0;
    const int xi = warp_incl_scan(x);
    scratch[lane_id()] = xi - x;                  // exclusive warp offsets
    if (lane_id() == 31) scratch[32] = xi;
  }
  __syncthreads();
  const int res = scratch[warp_id()] + inc - v;
  *total = scratch[32];
  return res;
}

// Add 1 to hist[bin] with one atomic per distinct bin in the warp.
__device__ __forceinline__ void warp_hist_add(int* hist, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  if ((int)lane_id() == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

// Among bins [0, nbins) of hist, find the digit d whose bin holds the
// `remaining`-th largest element counting from the top: count(bins > d) <
// remaining <= count(bins >= d).  Executed by warp 0; returns d and the count
// strictly above it through shared results res[0], res[1].
__device__ __forceinline__ void find_digit(const int* hist, int nbins, int remaining, int* res) {
  if (warp_id() != 0) return;
  const int per = nbins / 32;
  const int lane = lane_id();
  // lane 0 owns the top `per` bins, lane 31 the bottom ones
  const int hi = nbins - 1 - lane * per;
  int local = 0;
  for (int j = 0; j < per; ++j) local += hist[hi - j];
  const int inc = warp_incl_scan(local);
  const int exc = inc - local;
  const bool here = exc < remaining && remaining <= inc;
  const uint32_t m = __ballot_sync(0xffffffffu, here);
  if (here && lane == __ffs(m) - 1) {
    int above = exc;
    for (int j = 0; j < per; ++j) {
      const int c = hist[hi - j];
      if (above + c >= remaining) {
        res[0] = hi - j;
        res[1] = above;
        break;
      }
      above += c;
    }
  }
}

// Write the selection of a segment in index order.  Every thread owns the
// contiguous index range [lo, hi) and calls get(i) -> key.
template <typename GetKey>
__device__ __forceinline__ void write_selection(int64_t lo, int64_t hi, GetKey get, uint32_t kstar, int r,
                                                int32_t* out, int* scratch) {
  int gt = 0, eq = 0;
  for (int64_t i = lo; i < hi; ++i) {
    const uint32_t key = get(i);
    gt += key > kstar;
    eq += key == kstar;
  }
  int total;
  const int eq_before = block_excl_scan(eq, scratch, &total);
  int take_eq = r - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > eq ? eq : take_eq);
  const int pos0 = block_excl_scan(gt + take_eq, scratch, &total);
  int pos = pos0, taken = 0;
  for (int64_t i = lo; i < hi; ++i) {
    const uint32_t key = get(i);
    if (key > kstar || (key == kstar && taken < take_eq)) {
      out[pos++] = (int32_t)i;
      taken += (key == kstar);
    }
  }
}

__device__ __forceinline__ void write_all_valid(int32_t* out, int nv, int k) {
  for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = j < nv ? j : -1;
}

// ---------------------------------------------------------------- row kernel
// n_valid may be null (every row has N valid entries); map may be null, else the
// output holds map[row, position] instead of the position (used to return the
// original indices of a rescored candidate list; map rows must be ascending so
// that the output stays ascending).
__global__ void __launch_bounds__(1024) topk_row_kernel(const float* __restrict__ scores,
                                                        const int32_t* __restrict__ n_valid, int64_t N, int k,
                                                        int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ map) {
  extern __shared__ __align__(16) uint32_t keys[];  // [min(N, kRowSmemMax)]
  __shared__ int hist[256];
  __shared__ int scratch[33];
  __shared__ int res[2];
  const int64_t row = blockIdx.x;
  int nv = n_valid ? n_valid[row] : (int)N;
  nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
  int32_t* out = idx + row * k;
  const int32_t* mrow = map ? map + row * N : nullptr;
  if (nv <= k) {
    for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = j < nv ? (mrow ? mrow[j] : j) : -1;
    return;
  }
  const float* s = scores + row * N;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) keys[i] = order_key(s[i]);
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int j = threadIdx.x; j < 256; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < nv; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const uint32_t key = i < nv ? keys[i] : 0u;
      const bool act = i < nv && (key & pmask) == prefix;
      warp_hist_add(hist, (key >> shift) & 255u, act);
    }
    __syncthreads();
    find_digit(hist, 256, remaining, res);
    __syncthreads();
    prefix |= (uint32_t)res[0] << shift;
    pmask |= 255u << shift;
    remaining -= res[1];
    __syncthreads();
  }
  const int per = (nv + blockDim.x - 1) / blockDim.x;
  const int64_t lo = (int64_t)threadIdx.x * per;
  const int64_t hi = lo + per < nv ? lo + per : nv;
  write_selection(lo < nv ? lo : nv, hi, [&](int64_t i) { return keys[i]; }, prefix, remaining, out, scratch);
  if (mrow) {
    __syncthreads();
    for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = mrow[out[j]];
  }
}

// ---------------------------------------------------------------- long rows
struct TopkWs {
  // per row: [hist kHistBins][cand_count][done][pad ..] then candidates and bitmaps
  static constexpr int64_t kHeaderInts = kHistBins + 64;
  static __host__ __device__ int64_t row_bytes(int64_t N) {
    const int64_t words = (N + 31) / 32;
    return kHeaderInts * 4 + N * 8 + words * 8;
  }
};

__global__ void __launch_bounds__(512) topk_hist_kernel(const float* __restrict__ scores,
                                                        const int32_t* __restrict__ n_valid, int64_t N, int k,
                                                        uint8_t* __restrict__ ws) {
  __shared__ int hist[kHistBins];
  const int64_t row = blockIdx.y;
  int nv = n_valid[row];
  nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
  const int64_t c0 = (int64_t)blockIdx.x * kChunk;
  if (nv <= k || c0 >= nv) return;
  for (int j = threadIdx.x; j < kHistBins; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  const float* s = scores + row * N;
  const int64_t c1 = c0 + kChunk < nv ? c0 + kChunk : nv;
  for (int64_t i0 = c0; i0 < c1; i0 += blockDim.x) {
    const int64_t i = i0 + threadIdx.x;
    const bool act = i < c1;
    const uint32_t key = act ? order_key(s[i]) : 0u;
    warp_hist_add(hist, key >> (32 - kHistBits), act);
  }
  __syncthreads();
  int* ghist = reinterpret_cast<int*>(ws + row * TopkWs::row_bytes(N));
  for (int j = threadIdx.x; j < kHistBins; j += blockDim.x)
    if (hist[j]) atomicAdd(&ghist[j], hist[j]);
}

__global__ void __launch_bounds__(1024) topk_gather_select_kernel(const float* __restrict__ scores,
                                                                  const int32_t* __restrict__ n_valid, int64_t N,
                                                                  int k, int32_t* __restrict__ idx,
                                                                  uint8_t* __restrict__ ws) {
  __shared__ int hist[256];
  __shared__ int scratch[33];
  __shared__ int res[2];
  __shared__ int is_last;
  __shared__ int hist4k[kHistBins];
  const int64_t row = blockIdx.y;
  int nv = n_valid[row];
  nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
  int32_t* out = idx + row * k;
  const int nchunks = (nv + kChunk - 1) / kChunk;
  if (nv <= k) {
    if (blockIdx.x == 0) write_all_valid(out, nv, k);
    return;
  }
  if ((int)blockIdx.x >= nchunks) return;
  uint8_t* rws = ws + row * TopkWs::row_bytes(N);
  int* ghist = reinterpret_cast<int*>(rws);
  int* cand_count = ghist + kHistBins;
  int* done = cand_count + 1;
  uint32_t* ckey = reinterpret_cast<uint32_t*>(rws + TopkWs::kHeaderInts * 4);
  int32_t* cidx = reinterpret_cast<int32_t*>(ckey + N);
  const int64_t words = (N + 31) / 32;
  uint32_t* bm_gt = reinterpret_cast<uint32_t*>(cidx + N);
  uint32_t* bm_eq = bm_gt + words;

  // threshold bin b*: count(bins > b*) < k <= count(bins >= b*), 128 bins per lane of warp 0
  for (int j = threadIdx.x; j < kHistBins; j += blockDim.x) hist4k[j] = __ldcg(ghist + j);
  __syncthreads();
  find_digit(hist4k, kHistBins, k, res);
  __syncthreads();
  const uint32_t bstar = (uint32_t)res[0];
  // append every key whose top bits are >= b* (warp-aggregated slot reservation)
  const float* s = scores + row * N;
  const int64_t c0 = (int64_t)blockIdx.x * kChunk;
  const int64_t c1 = c0 + kChunk < nv ? c0 + kChunk : nv;
  for (int64_t i0 = c0; i0 < c1; i0 += blockDim.x) {
    const int64_t i = i0 + threadIdx.x;
    uint32_t key = 0;
    bool take = false;
    if (i < c1) {
      key = order_key(s[i]);
      take = (key >> (32 - kHistBits)) >= bstar;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, take);
    if (m) {
      int base = 0;
      if (lane_id() == 0) base = atomicAdd(cand_count, __popc(m));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (take) {
        const int slot = base + __popc(m & ((1u << lane_id()) - 1));
        ckey[slot] = key;
        cidx[slot] = (int32_t)i;
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1) == nchunks - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // ---- last CTA: exact select among the candidates
  const int nc = *((volatile int*)cand_count);
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int j = threadIdx.x; j < 256; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < nc; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const uint32_t key = i < nc ? __ldcg(ckey + i) : 0u;
      const bool act = i < nc && (key & pmask) == prefix;
      warp_hist_add(hist, (key >> shift) & 255u, act);
    }
    __syncthreads();
    find_digit(hist, 256, remaining, res);
    __syncthreads();
    prefix |= (uint32_t)res[0] << shift;
    pmask |= 255u << shift;
    remaining -= res[1];
    __syncthreads();
  }
  // mark candidates > K* and == K* in two index bitmaps
  for (int i = threadIdx.x; i < nc; i += blockDim.x) {
    const uint32_t key = __ldcg(ckey + i);
    const int32_t j = __ldcg(cidx + i);
    if (key > prefix) atomicOr(&bm_gt[j >> 5], 1u << (j & 31));
    else if (key == prefix) atomicOr(&bm_eq[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  // ordered pass over the bitmaps
  const int64_t used_words = ((int64_t)nv + 31) / 32;
  const int64_t per = (used_words + blockDim.x - 1) / blockDim.x;
  const int64_t w_lo = (int64_t)threadIdx.x * per < used_words ? (int64_t)threadIdx.x * per : used_words;
  const int64_t w_hi = w_lo + per < used_words ? w_lo + per : used_words;
  int gt = 0, eq = 0;
  for (int64_t wv = w_lo; wv < w_hi; ++wv) {
    gt += __popc(bm_gt[wv]);
    eq += __popc(bm_eq[wv]);
  }
  int total;
  const int eq_before = block_excl_scan(eq, scratch, &total);
  int take_eq = remaining - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > eq ? eq : take_eq);
  int pos = block_excl_scan(gt + take_eq, scratch, &total);
  int taken = 0;
  for (int64_t wv = w_lo; wv < w_hi; ++wv) {
    uint32_t g = bm_gt[wv], e = bm_eq[wv];
    while (g | e) {
      const int bit = __ffs(g | e) - 1;
      const uint32_t mb = 1u << bit;
      if (g & mb) {
        out[pos++] = (int32_t)(wv * 32 + bit);
      } else if (taken < take_eq) {
        out[pos++] = (int32_t)(wv * 32 + bit);
        ++taken;
      }
      g &= ~mb;
      e &= ~mb;
    }
    bm_gt[wv] = 0;                                  // leave the workspace zeroed
    bm_eq[wv] = 0;
  }
  for (int j = threadIdx.x; j < kHistBins; j += blockDim.x) ghist[j] = 0;
  for (int i = threadIdx.x; i < nc; i += blockDim.x) {
    ckey[i] = 0;
    cidx[i] = 0;
  }
  if (threadIdx.x == 0) {
    *cand_count = 0;
    *done = 0;
  }
}

}  // namespace csa
