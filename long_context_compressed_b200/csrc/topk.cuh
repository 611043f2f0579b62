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
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace csa {

constexpr int kRowSmemMax = 32768;
constexpr int kRowFastMin = 8192;               // rows this long try the sampled threshold first
constexpr int kRowCand = 8192;                  // candidates of that path (shared memory)
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kChunk = 4096;
constexpr int kCandSmem = 8192;                 // candidates the last CTA stages in shared memory

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0) u = 0;                       // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float an order key came from (-0.0 comes back as +0.0).
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
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

// Block-wide version of find_digit for nbins == BPT * blockDim.x: thread i owns
// the BPT bins nbins-BPT*i-1 .. nbins-BPT*(i+1) (top first); a block scan of the
// owned counts locates the bin.  All threads must call it.
template <int BPT = 4>
__device__ __forceinline__ void find_digit_block(const int* hist, int nbins, int remaining, int* res,
                                                 int* scratch) {
  const int hi = nbins - 1 - BPT * (int)threadIdx.x;
  int c[BPT], local = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    c[j] = hist[hi - j];
    local += c[j];
  }
  int total;
  const int exc = block_excl_scan(local, scratch, &total);
  if (exc < remaining && remaining <= exc + local) {
    int above = exc;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (above + c[j] >= remaining) {
        res[0] = hi - j;
        res[1] = above;
        break;
      }
      above += c[j];
    }
  }
}

// Skewed shared-memory histogram index: bin h lives at h + h/32, so threads that
// own consecutive groups of 8 or 16 bins read them without bank conflicts.
__device__ __forceinline__ int skew(int h) { return h + (h >> 5); }

// find_digit_block over a skewed histogram (nbins == BPT * blockDim.x).
template <int BPT>
__device__ __forceinline__ void find_digit_skewed(const int* hist, int nbins, int remaining, int* res,
                                                  int* scratch) {
  const int hi = nbins - 1 - BPT * (int)threadIdx.x;
  int c[BPT], local = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    c[j] = hist[skew(hi - j)];
    local += c[j];
  }
  int total;
  const int exc = block_excl_scan(local, scratch, &total);
  if (exc < remaining && remaining <= exc + local) {
    int above = exc;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (above + c[j] >= remaining) {
        res[0] = hi - j;
        res[1] = above;
        break;
      }
      above += c[j];
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

__global__ void __launch_bounds__(256) fill_f32_kernel(float* __restrict__ p, int64_t n, float v) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) p[i] = v;
}

// ---------------------------------------------------------------- row kernel
// n_valid may be null (every row has N valid entries); map may be null, else the
// output holds map[row, position] instead of the position (used to return the
// original indices of a rescored candidate list; map rows must be ascending so
// that the output stays ascending).  cand_smem: the dynamic shared memory also holds
// kRowCand candidate keys and indices after the row's keys (rows of kRowFastMin or more
// then try the sampled threshold first).  gate: null, or a device int written by an
// earlier launch; 0 -> the launch does nothing.
__global__ void __launch_bounds__(1024) topk_row_kernel(const float* __restrict__ scores,
                                                        const int32_t* __restrict__ n_valid, int64_t N, int k,
                                                        int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ map, int cand_smem,
                                                        const int* __restrict__ gate) {
  griddep_sync();
  if (gate && __ldcg(gate) == 0) return;
  extern __shared__ __align__(16) uint32_t keys[];  // [min(N, kRowSmemMax)], then (long rows) the candidates
  __shared__ __align__(16) int rhist[kHistBins + kHistBins / 32];   // skewed
  __shared__ int scratch[33];
  __shared__ int res[2];
  __shared__ uint32_t ext[2];
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
  // every score of this thread is requested before any is used (one memory round trip)
  {
    constexpr int kPer = kRowSmemMax / 1024;
    float v[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = u * 1024 + (int)threadIdx.x;
      v[u] = i < nv ? __ldg(s + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = u * 1024 + (int)threadIdx.x;
      if (i < nv) keys[i] = order_key(v[u]);
    }
  }
  // ---- long rows: a strided sample of 1024 keys places a threshold t (the lower edge of the
  // sample-histogram bin that holds the sample's 2k*1024/nv-th key, plus a margin) whose count
  // over the row usually lies in [k, kRowCand].  Then only the keys >= t, compacted in index
  // order, enter the radix select, over their own key span (the tail of a row spreads over
  // the histogram instead of piling into the few bins the row's bulk falls in).  Otherwise
  // the full radix below runs.
  if (cand_smem && nv >= kRowFastMin && blockDim.x == 1024) {
    uint32_t* ckey = keys + (N < kRowSmemMax ? N : kRowSmemMax);
    int32_t* cidx = reinterpret_cast<int32_t*>(ckey + kRowCand);
    const int stride = nv / 1024;
    const uint32_t sk = keys[threadIdx.x * stride];
    for (int j = threadIdx.x; j < kHistBins + kHistBins / 32; j += blockDim.x) rhist[j] = 0;
    if (threadIdx.x == 0) {
      ext[0] = 0xffffffffu;
      ext[1] = 0u;
    }
    const uint32_t wmin = __reduce_min_sync(0xffffffffu, sk), wmax = __reduce_max_sync(0xffffffffu, sk);
    __syncthreads();
    if (lane_id() == 0) {
      atomicMin(&ext[0], wmin);
      atomicMax(&ext[1], wmax);
    }
    __syncthreads();
    const uint32_t smin = ext[0];
    const uint32_t sspan = ext[1] - smin;
    const int sbits = sspan ? 32 - __clz(sspan) : 0;
    const int sh = sbits > kHistBits ? sbits - kHistBits : 0;
    atomicAdd(&rhist[skew((int)((sk - smin) >> sh))], 1);
    __syncthreads();
    const int64_t want64 = 2 * (int64_t)k * 1024 / nv + 16;
    const int want = want64 < 1024 ? (int)want64 : 1024;
    find_digit_skewed<kHistBins / 1024>(rhist, kHistBins, want, res, scratch);
    __syncthreads();
    const uint32_t t = smin + ((uint32_t)res[0] << sh);
    // the row's keys >= t, counted and then compacted over contiguous index ranges
    const int per = ((nv + 1023) / 1024) | 1;
    const int lo = min((int)threadIdx.x * per, nv), hi = min(lo + per, nv);
    int c = 0;
    uint32_t cmax = 0u;
    for (int i = lo; i < hi; ++i) {
      const uint32_t key = keys[i];
      c += key >= t;
      cmax = max(cmax, key);
    }
    int C;
    const int off = block_excl_scan(c, scratch, &C);
    if (C >= k && C <= kRowCand) {                       // the whole block takes the same branch
      int o = off;
      for (int i = lo; i < hi; ++i) {
        const uint32_t key = keys[i];
        if (key >= t) {
          ckey[o] = key;
          cidx[o] = i;
          ++o;
        }
      }
      cmax = __reduce_max_sync(0xffffffffu, cmax);
      if (lane_id() == 0) atomicMax(&ext[1], cmax);       // ext[1] already holds the sample max
      __syncthreads();
      const uint32_t cspan = ext[1] - t;
      uint32_t prefix = 0, pmask = 0;
      int remaining = k;
      for (int hb = cspan ? 32 - __clz(cspan) : 0; hb > 0;) {
        const int lb = hb > kHistBits ? hb - kHistBits : 0;
        const uint32_t dmask = (1u << (hb - lb)) - 1;
        for (int j = threadIdx.x; j < kHistBins + kHistBins / 32; j += blockDim.x) rhist[j] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
          const uint32_t u = ckey[i] - t;
          if ((u & pmask) == prefix) atomicAdd(&rhist[skew((int)((u >> lb) & dmask))], 1);
        }
        __syncthreads();
        find_digit_skewed<kHistBins / 1024>(rhist, kHistBins, remaining, res, scratch);
        __syncthreads();
        prefix |= (uint32_t)res[0] << lb;
        pmask |= dmask << lb;
        remaining -= res[1];
        hb = lb;
        __syncthreads();
      }
      const int cper = ((C + 1023) / 1024) | 1;
      const int clo = min((int)threadIdx.x * cper, C), chi = min(clo + cper, C);
      write_selection(clo, chi, [&](int64_t i) { return ckey[i]; }, t + prefix, remaining, out, scratch);
      __syncthreads();
      for (int j = threadIdx.x; j < k; j += blockDim.x) {
        const int32_t ci = cidx[out[j]];
        out[j] = mrow ? mrow[ci] : ci;
      }
      return;
    }
    __syncthreads();
  }
  // radix select with digits of 12, 10 and 10 bits on a skewed histogram
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 0 ? 4095u : 1023u;
    for (int j = threadIdx.x; j < kHistBins + kHistBins / 32; j += blockDim.x) rhist[j] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&rhist[skew((int)((key >> shift) & dmask))], 1);
    }
    __syncthreads();
    if (pass == 0) find_digit_skewed<kHistBins / 1024>(rhist, kHistBins, remaining, res, scratch);
    else find_digit_skewed<1>(rhist, 1024, remaining, res, scratch);
    __syncthreads();
    prefix |= (uint32_t)res[0] << shift;
    pmask |= dmask << shift;
    remaining -= res[1];
    __syncthreads();
  }
  // contiguous index ranges of odd length per thread: conflict-free shared-memory reads
  const int per = ((nv + (int)blockDim.x - 1) / (int)blockDim.x) | 1;
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
                                                        uint8_t* __restrict__ ws, int64_t ws_row_bytes) {
  griddep_sync();
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
  int* ghist = reinterpret_cast<int*>(ws + row * ws_row_bytes);
  for (int j = threadIdx.x; j < kHistBins; j += blockDim.x)
    if (hist[j]) atomicAdd(&ghist[j], hist[j]);
}

__global__ void __launch_bounds__(1024) topk_gather_select_kernel(const float* __restrict__ scores,
                                                                  const int32_t* __restrict__ n_valid, int64_t N,
                                                                  int k, int32_t* __restrict__ idx,
                                                                  uint8_t* __restrict__ ws) {
  griddep_sync();
  __shared__ int hist[256];
  __shared__ int scratch[33];
  __shared__ int res[2];
  __shared__ int is_last;
  __shared__ int hist4k[kHistBins];
  extern __shared__ __align__(16) uint32_t cand_smem[];   // [kCandSmem] keys + [kCandSmem] indices
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
  find_digit_block<4>(hist4k, kHistBins, k, res, scratch);
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

  // ---- last CTA: exact select among the candidates (staged in shared memory when they fit)
  const int nc = *((volatile int*)cand_count);
  uint32_t* skey = cand_smem;
  int32_t* sidx = reinterpret_cast<int32_t*>(cand_smem + kCandSmem);
  const bool in_smem = nc <= kCandSmem;
  if (in_smem) {
    for (int i = threadIdx.x; i < nc; i += blockDim.x) {
      skey[i] = __ldcg(ckey + i);
      sidx[i] = __ldcg(cidx + i);
    }
    __syncthreads();
  }
  auto cand_key = [&](int i) -> uint32_t { return in_smem ? skey[i] : __ldcg(ckey + i); };
  auto cand_idx = [&](int i) -> int32_t { return in_smem ? sidx[i] : __ldcg(cidx + i); };
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int j = threadIdx.x; j < 256; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < nc; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const uint32_t key = i < nc ? cand_key(i) : 0u;
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
    const uint32_t key = cand_key(i);
    const int32_t j = cand_idx(i);
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

// ---------------------------------------------------------------- fused select (decode)
// Per-row workspace of topk_select_kernel: [4096-bin histogram][64-bit counter:
// candidates appended (low word) | CTAs finished (high word)][slot counter][pad]
// [per-chunk (first slot, count) table] then candidate keys [N] and indices [N].  The histogram is
// accumulated by the indexer (csa_index_scores with this workspace); the last CTA
// of each row leaves the row's header zeroed for the next call.
constexpr int kSelMaxChunks = 1024;   // chunks per row (table in the row header)
struct SelectWs {
  static constexpr int64_t kTableInt = kHistBins + 64;            // [chunk] -> (first slot, count)
  static constexpr int64_t kFineInt = kTableInt + 2 * kSelMaxChunks;   // fine histogram of the candidates
  static constexpr int64_t kHeaderInts = kFineInt + kHistBins;
  static __host__ __device__ int64_t row_bytes(int64_t N) {
    return ((kHeaderInts + 2 * N) * 4 + 15) / 16 * 16;
  }
};
// Fine histogram of the candidates' (rescored) keys: 4096 bins of 2^12 keys each, from two
// threshold bins (2 * 2^20 keys) below the kk-th score's bin -- every candidate's score
// lies in that bin or above, and a rescored score near it -- with keys outside the range
// clamped to the end bins.  The last CTA finds the k-th key's fine bin with one scan of
// this histogram and ranks that bin's few keys directly.
__device__ __forceinline__ uint32_t fine_base(uint32_t bstar, bool rescore) {
  const uint32_t below = rescore ? 2u : 0u;
  return (bstar >= below ? bstar - below : 0u) << 20;
}
__device__ __forceinline__ int fine_bin(uint32_t key, uint32_t base) {
  if (key < base) return 0;
  const uint32_t f = (key - base) >> 12;
  return f > (uint32_t)(kHistBins - 1) ? kHistBins - 1 : (int)f;
}
constexpr int kSelThreads = 256;
constexpr int kSelPerThread = 4;     // scores each thread loads per pass of the chunk scan
constexpr int kSelTcRows = 128;      // candidates rescored per tensor-core batch (bf16)
constexpr int kSelKeyBatch = 64;     // candidate key rows per SIMT batch (fp32)
constexpr int kSelCandSmem = 8192;   // candidates the last CTA stages in shared memory
// keys the last CTA ranks directly once a radix digit has narrowed the k-th key to one bin
constexpr int kSelPivot = 256;
constexpr int kSelPrefetch = 2048;   // chunk entries whose scores are fetched with the histogram
constexpr int kSelMaxChunkLen = 16384;  // entries per chunk (shared-memory candidate list)
static_assert(kSelPerThread * (kSelThreads / 32) == 32, "one scan lane per (pass, warp)");
static_assert(kSelMaxChunks % kSelThreads == 0, "chunk table split evenly over the threads");
static_assert(2 * kSelMaxChunks >= CSA_MAX_TOPK, "the last CTA stages k indices in the chunk table's space");
constexpr int64_t kSelMaxN = int64_t(1) << 19;
constexpr int kSelTileBytes = 2 * kSelTcRows * 128;    // candidate key tile, 2 x 128-byte K atoms (bf16)
constexpr int kSelQBytes = 2 * 64 * 128;               // q tile: 64 heads x 128 dims bf16

template <typename T>
__device__ __forceinline__ void unpack_vec(uint4 v, float* f);
template <>
__device__ __forceinline__ void unpack_vec<__nv_bfloat16>(uint4 v, float* f) {   // 8 bf16
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void unpack_vec<float>(uint4 v, float* f) {  // 4 fp32
  f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

// Row r (one query per sequence: T == 1) of scores [rows, N].  Candidates are the
// indices whose score lies in the histogram bin of the kk-th largest score or above
// (kk = kc when RESCORE, else k) -- a superset of the kk largest.  With RESCORE each
// candidate is rescored with the plain indexer definition on full-precision qI / kI
// (fp32 accumulation; bf16 inputs on tcgen05, fp32 inputs on the FMA pipes); the
// exact top-k of the (re)scored candidates, lower index first among equal scores, is
// written in ascending index order by the last CTA of the row (chunks are contiguous
// index ranges: the k indices are bucketed by chunk and ranked inside their bucket).
// sel_scores (may be null) receives, beside each index, the score that ranked it: the
// rescored one with RESCORE, else the input score; -inf beside a -1 pad.  With RESCORE
// and sel_scores, a row of n_valid <= k entries is rescored too (all its entries are
// candidates, and the last CTA takes them all).
template <bool RESCORE, typename Tin>
__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const float* __restrict__ scores,
                                                                  const int32_t* __restrict__ n_valid, int64_t N,
                                                                  int k, int kc, int chunk,
                                                                  const Tin* __restrict__ qI,
                                                                  const float* __restrict__ w,
                                                                  const Tin* __restrict__ kI, int32_t* __restrict__ idx,
                                                                  float* __restrict__ sel_scores,
                                                                  uint8_t* __restrict__ ws) {
  constexpr bool TC = RESCORE && sizeof(Tin) == 2;
  extern __shared__ __align__(1024) uint8_t sel_raw[];
  uint8_t* sel_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sel_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) int histk[kHistBins + kHistBins / 32];   // skewed
  __shared__ int scratch[33];
  __shared__ int res[2];
  __shared__ int lcount, gslot, is_last, pcount;
  __shared__ int wcnt[32], wexc[33];
  __shared__ uint32_t kext[2];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_holder;
  if (TC) {
    if (threadIdx.x == 0) {
      mbar_init(&mma_bar, 1);
      fence_mbar_init();
    }
    if (warp_id() == 0) {
      tmem_alloc(&tmem_holder, 64);
      tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  griddep_sync();
  const int64_t row = blockIdx.y;
  int nv = n_valid[row];
  nv = nv < 0 ? 0 : (nv > (int)N ? (int)N : nv);
  uint8_t* rws = ws + row * SelectWs::row_bytes(N);
  int* ghist = reinterpret_cast<int*>(rws);
  // header: [candidates appended | CTAs finished] as one 64-bit counter, then the slot counter
  unsigned long long* fin = reinterpret_cast<unsigned long long*>(ghist + kHistBins);
  int* slots = ghist + kHistBins + 2;
  int* ctab = reinterpret_cast<int*>(rws) + SelectWs::kTableInt;
  int* gfine = reinterpret_cast<int*>(rws) + SelectWs::kFineInt;
  uint32_t* ckey = reinterpret_cast<uint32_t*>(rws + SelectWs::kHeaderInts * 4);
  int32_t* cidx = reinterpret_cast<int32_t*>(ckey + N);
  int32_t* out = idx + row * k;
  float* oscore = sel_scores ? sel_scores + row * k : nullptr;
  const bool all_valid = nv <= k && !(RESCORE && oscore && nv > 0);
  const bool active = !all_valid && (int64_t)blockIdx.x * chunk < nv;
  if (all_valid && blockIdx.x == 0) {
    write_all_valid(out, nv, k);
    if (oscore)
      for (int j = threadIdx.x; j < k; j += blockDim.x) oscore[j] = j < nv ? scores[row * N + j] : -INFINITY;
    for (int j = threadIdx.x; j < kHistBins; j += blockDim.x) ghist[j] = 0;
  }
  int nloc = 0;
  uint32_t fbase = 0;                                // this row's fine-histogram base key
  // shared-memory map: [key tile 32 KB][q tile 16 KB] (tensor-core rescoring) then
  // lidx / lkey [chunk] and the fp32 rescoring scratch; the last CTA reuses all of it
  uint8_t* tile_s = sel_smem;
  uint8_t* qt_s = tile_s + kSelTileBytes;
  int32_t* lidx = reinterpret_cast<int32_t*>(qt_s + kSelQBytes);
  uint32_t* lkey = reinterpret_cast<uint32_t*>(lidx + chunk);
  float* wsm = reinterpret_cast<float*>(lkey + chunk);               // [64]
  if (active) {
    const int kk = RESCORE ? (kc < nv ? kc : nv) : k;
    const float* srow = scores + row * N;
    const int64_t c0 = (int64_t)blockIdx.x * chunk;
    const int64_t c1 = c0 + chunk < nv ? c0 + chunk : nv;
    // Every load the front half needs is issued here, before any is used: the
    // histogram, this chunk's scores (chunks up to kSelPrefetch entries) and, for the
    // tensor-core rescoring, the query tile and head weights.
    constexpr int kPre = kSelPrefetch / kSelThreads;
    const bool prefetched = c1 - c0 <= kSelPrefetch;
    float pre[kPre];
    if (prefetched) {
#pragma unroll
      for (int u = 0; u < kPre; ++u) {
        const int64_t i = c0 + (int64_t)u * kSelThreads + threadIdx.x;
        pre[u] = i < c1 ? __ldg(srow + i) : 0.f;
      }
    }
    uint4 qv[TC ? 4 : 1];
    float wv = 0.f;
    if (TC) {
      const uint4* q4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(qI) + row * 64 * 128);
#pragma unroll
      for (int u = 0; u < 4; ++u) qv[u] = __ldg(q4 + threadIdx.x + u * kSelThreads);
      if (threadIdx.x < 64) wv = w[row * 64 + threadIdx.x];
    }
    // ---- threshold bin b*: count(bins > b*) < kk <= count(bins >= b*)
    {
      const int4* g4 = reinterpret_cast<const int4*>(ghist);
      int4 v[kHistBins / 4 / kSelThreads];
#pragma unroll
      for (int u = 0; u < kHistBins / 4 / kSelThreads; ++u) v[u] = __ldcg(g4 + threadIdx.x + u * kSelThreads);
#pragma unroll
      for (int u = 0; u < kHistBins / 4 / kSelThreads; ++u) {
        const int h = 4 * (threadIdx.x + u * kSelThreads);
        histk[skew(h)] = v[u].x;
        histk[skew(h + 1)] = v[u].y;
        histk[skew(h + 2)] = v[u].z;
        histk[skew(h + 3)] = v[u].w;
      }
    }
    if (TC) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = threadIdx.x + u * kSelThreads, r = j >> 4, c = j & 15;
        *reinterpret_cast<uint4*>(qt_s + (c >> 3) * 64 * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = qv[u];
      }
      if (threadIdx.x < 64) wsm[threadIdx.x] = wv;
    }
    if (threadIdx.x == 0) lcount = 0;
    __syncthreads();
    find_digit_skewed<kHistBins / kSelThreads>(histk, kHistBins, kk, res, scratch);
    __syncthreads();
    const uint32_t bstar = (uint32_t)res[0];
    fbase = fine_base(bstar, RESCORE);
    // ---- this chunk's candidates, compacted in index order (one warp scans the 32
    // (pass, warp) counts)
    int lbase = 0;
    int pass = 0;
    for (int64_t base0 = c0; base0 < c1; base0 += (int64_t)kSelPerThread * blockDim.x, ++pass) {
      float v[kSelPerThread];
      if (prefetched) {
#pragma unroll
        for (int pp = 0; pp < kPre / kSelPerThread; ++pp)   // static register indices
          if (pp == pass)
#pragma unroll
            for (int u = 0; u < kSelPerThread; ++u) v[u] = pre[pp * kSelPerThread + u];
      } else {
#pragma unroll
        for (int u = 0; u < kSelPerThread; ++u) {
          const int64_t i = base0 + (int64_t)u * blockDim.x + threadIdx.x;
          v[u] = i < c1 ? __ldg(srow + i) : 0.f;
        }
      }
      uint32_t key[kSelPerThread], m[kSelPerThread];
#pragma unroll
      for (int u = 0; u < kSelPerThread; ++u) {
        const int64_t i = base0 + (int64_t)u * blockDim.x + threadIdx.x;
        key[u] = order_key(v[u]);
        m[u] = __ballot_sync(0xffffffffu, i < c1 && (key[u] >> (32 - kHistBits)) >= bstar);
        if (lane_id() == 0) wcnt[u * (kSelThreads / 32) + warp_id()] = __popc(m[u]);
      }
      __syncthreads();
      if (warp_id() == 0) {
        const int x = wcnt[lane_id()];
        const int xi = warp_incl_scan(x);
        wexc[lane_id()] = xi - x;
        if (lane_id() == 31) wexc[32] = xi;
      }
      __syncthreads();
      const uint32_t below = (1u << lane_id()) - 1;
#pragma unroll
      for (int u = 0; u < kSelPerThread; ++u)
        if (m[u] >> lane_id() & 1u) {
          const int slot = lbase + wexc[u * (kSelThreads / 32) + warp_id()] + __popc(m[u] & below);
          lidx[slot] = (int32_t)(base0 + (int64_t)u * blockDim.x + threadIdx.x);
          lkey[slot] = key[u];
        }
      lbase += wexc[32];
    }
    __syncthreads();
    nloc = lbase;
  }
  if (TC && active && nloc > 0) {
    // ---- exact rescoring on tcgen05: candidates (M = 128 per batch) x 64 heads, K = 128
    // (the query tile and head weights were staged with the front-half loads)
    const __nv_bfloat16* kbase = reinterpret_cast<const __nv_bfloat16*>(kI) + row * N * 128;
    const uint32_t idesc = make_idesc(128, 64, 1, 0, 0);
    uint32_t mph = 0;
    for (int cb = 0; cb < nloc; cb += kSelTcRows) {
      const int nb = nloc - cb < kSelTcRows ? nloc - cb : kSelTcRows;
      // gather the batch's key rows (16-byte pieces, all issued before use)
      uint4 v[kSelTcRows * 16 / kSelThreads];
#pragma unroll
      for (int u = 0; u < kSelTcRows * 16 / kSelThreads; ++u) {
        const int j = threadIdx.x + u * kSelThreads, r = j >> 4, c = j & 15;
        v[u] = r < nb ? __ldg(reinterpret_cast<const uint4*>(kbase + (int64_t)lidx[cb + r] * 128) + c)
                      : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kSelTcRows * 16 / kSelThreads; ++u) {
        const int j = threadIdx.x + u * kSelThreads, r = j >> 4, c = j & 15;
        *reinterpret_cast<uint4*>(tile_s + (c >> 3) * kSelTcRows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = v[u];
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (threadIdx.x == 0) {
        const uint32_t ab = smem_u32(tile_s), bb = smem_u32(qt_s);
#pragma unroll
        for (int kq = 0; kq < 8; ++kq) {
          const int atom = kq >> 2, inner = (kq & 3) * 32;
          mma_bf16(tmem_holder, smem_desc(ab + atom * kSelTcRows * 128 + inner, 16, 1024, kLayoutSW128),
                   smem_desc(bb + atom * 64 * 128 + inner, 16, 1024, kLayoutSW128), idesc, kq > 0 ? 1u : 0u);
        }
        mma_commit(&mma_bar);
      }
      mbar_wait(&mma_bar, mph);
      mph ^= 1;
      tc_fence_after();
      if (warp_id() < 4) {
        const int r = warp_id() * 32 + lane_id();           // TMEM lane = candidate row
        const uint32_t ta = tmem_holder + ((uint32_t)(warp_id() * 32) << 16);
        float a0[32], a1[32];
        tmem_ld32(ta, a0);
        tmem_ld32(ta + 32, a1);
        tmem_wait_ld();
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          s0 = fmaf(wsm[h], fmaxf(a0[h], 0.f), s0);
          s1 = fmaf(wsm[32 + h], fmaxf(a1[h], 0.f), s1);
        }
        if (r < nb) lkey[cb + r] = order_key(s0 + s1);
      }
      tc_fence_before();
      __syncthreads();
    }
  } else if (RESCORE && !TC && active && nloc > 0) {
    // ---- exact rescoring on the FMA pipes (fp32 inputs)
    float* qs = wsm + 64;                                            // [64][129]
    float* kb = qs + 64 * 129;                                       // [kSelKeyBatch][128]
    const float* qrow = reinterpret_cast<const float*>(qI) + row * 64 * 128;
    const float* kbase = reinterpret_cast<const float*>(kI) + row * N * 128;
    {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(qrow) + threadIdx.x + u * kSelThreads);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e0 = (threadIdx.x + u * kSelThreads) * 4;
        float f[4];
        unpack_vec<float>(v[u], f);
#pragma unroll
        for (int e = 0; e < 4; ++e) qs[((e0 + e) >> 7) * 129 + ((e0 + e) & 127)] = f[e];
      }
    }
    if (threadIdx.x < 64) wsm[threadIdx.x] = w[row * 64 + threadIdx.x];
    const int l = lane_id();
    for (int cb = 0; cb < nloc; cb += kSelKeyBatch) {
      const int nb = nloc - cb < kSelKeyBatch ? nloc - cb : kSelKeyBatch;
      __syncthreads();
      uint4 v[kSelKeyBatch * 32 / kSelThreads];
#pragma unroll
      for (int u = 0; u < kSelKeyBatch * 32 / kSelThreads; ++u) {
        const int j = threadIdx.x + u * kSelThreads, c = j >> 5, part = j & 31;
        v[u] = c < nb ? __ldg(reinterpret_cast<const uint4*>(kbase + (int64_t)lidx[cb + c] * 128) + part)
                      : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kSelKeyBatch * 32 / kSelThreads; ++u) {
        const int j = threadIdx.x + u * kSelThreads, c = j >> 5, part = j & 31;
        *reinterpret_cast<uint4*>(kb + c * 128 + part * 4) = v[u];
      }
      __syncthreads();
      for (int c = warp_id(); c < nb; c += kSelThreads / 32) {
        const float* kr = kb + c * 128;
        float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll 8
        for (int d = 0; d < 128; d += 2) {
          d0 = fmaf(qs[l * 129 + d], kr[d], d0);
          d1 = fmaf(qs[(l + 32) * 129 + d], kr[d], d1);
          d2 = fmaf(qs[l * 129 + d + 1], kr[d + 1], d2);
          d3 = fmaf(qs[(l + 32) * 129 + d + 1], kr[d + 1], d3);
        }
        float v2 = wsm[l] * fmaxf(d0 + d2, 0.f) + wsm[l + 32] * fmaxf(d1 + d3, 0.f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v2 += __shfl_xor_sync(0xffffffffu, v2, o);
        if (l == 0) lkey[cb + c] = order_key(v2);
      }
    }
    __syncthreads();
  }
  if (TC) {
    __syncthreads();
    if (warp_id() == 0) tmem_dealloc(tmem_holder, 64);
  }
  if (!active) return;
  // ---- append to the row's candidate list, and the candidates' keys to the fine histogram
  if (threadIdx.x == 0) {
    const int g = nloc > 0 ? atomicAdd(slots, nloc) : 0;
    gslot = g;
    reinterpret_cast<int2*>(ctab)[blockIdx.x] = make_int2(g, nloc);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < nloc; c += blockDim.x) {
    const uint32_t key = lkey[c];
    ckey[gslot + c] = key;
    cidx[gslot + c] = lidx[c];
    atomicAdd(&gfine[fine_bin(key, fbase)], 1);
  }
  __syncthreads();
  const int nchunks = (int)((nv + chunk - 1) / chunk);
  if (threadIdx.x == 0) {
    // one counter tells the last CTA both that it is last and how many candidates there are
    const unsigned long long old = atom_add_acq_rel(fin, (1ull << 32) | (unsigned)nloc);
    is_last = (int)(old >> 32) == nchunks - 1;
    lcount = (int)(uint32_t)old + nloc;
  }
  __syncthreads();
  if (!is_last) return;
  // ---- last CTA of the row: exact top-k among the candidates
  const int nc = lcount;
  if (nc <= kSelCandSmem) {
    // Stage the candidates in index order: chunk c's list (index-ordered by the scan)
    // goes to offset pre[c] = the earlier chunks' counts.  Loads of the chunk table
    // and of the first candidates are issued together.
    uint32_t* okey = reinterpret_cast<uint32_t*>(sel_smem);
    int32_t* oidx = reinterpret_cast<int32_t*>(okey + kSelCandSmem);
    int* tslot = oidx + kSelCandSmem;                    // [chunk] first slot of its list
    int* tpre = tslot + kSelMaxChunks;                   // [chunk] offset of its list in index order
    constexpr int CPT = kSelMaxChunks / kSelThreads;
    constexpr int U = 16;                                // candidates per thread per batch
    int2 ct[CPT];                                        // (first slot, count) of this thread's chunks
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
      const int c = threadIdx.x * CPT + u;
      ct[u] = c < nchunks ? __ldcg(reinterpret_cast<const int2*>(ctab) + c) : make_int2(0, 0);
    }
    uint32_t ck[U];
    int32_t ci[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = u * kSelThreads + threadIdx.x;
      ck[u] = i < nc ? __ldcg(ckey + i) : 0u;
      ci[u] = i < nc ? __ldcg(cidx + i) : 0;
    }
    // the fine histogram the chunks accumulated, requested with the first candidates
    int4 gf[kHistBins / 4 / kSelThreads];
#pragma unroll
    for (int u = 0; u < kHistBins / 4 / kSelThreads; ++u)
      gf[u] = __ldcg(reinterpret_cast<const int4*>(gfine) + threadIdx.x + u * kSelThreads);
    if (threadIdx.x == 0) {
      kext[0] = 0xffffffffu;
      kext[1] = 0u;
      pcount = 0;
    }
    {
      int local = 0;
#pragma unroll
      for (int u = 0; u < CPT; ++u) local += ct[u].y;
      int total;
      int off = block_excl_scan(local, scratch, &total);
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        const int c = threadIdx.x * CPT + u;
        if (c < nchunks) {
          tslot[c] = ct[u].x;
          tpre[c] = off;
        }
        off += ct[u].y;
      }
    }
#pragma unroll
    for (int u = 0; u < kHistBins / 4 / kSelThreads; ++u) {
      const int h = 4 * (threadIdx.x + u * kSelThreads);
      histk[skew(h)] = gf[u].x;
      histk[skew(h + 1)] = gf[u].y;
      histk[skew(h + 2)] = gf[u].z;
      histk[skew(h + 3)] = gf[u].w;
    }
    __syncthreads();
    // The k-th key's bin of the fine histogram (bins of 2^12 keys).  If it is an inner bin,
    // the staging pass below also histograms the low 12 bits of that bin's keys, which
    // gives the k-th key itself; an edge bin (keys clamped into it) takes the radix select.
    // No more candidates than k: every one is taken.
    const bool take_all = nc <= k;
    int fstar = 0, fabove = 0;
    if (!take_all) {
      find_digit_skewed<kHistBins / kSelThreads>(histk, kHistBins, k, res, scratch);
      __syncthreads();
      fstar = res[0];
      fabove = res[1];
    }
    const bool pivots = fstar > 0 && fstar < kHistBins - 1;
    for (int j = threadIdx.x; j < kHistBins + kHistBins / 32; j += blockDim.x) histk[j] = 0;
    __syncthreads();
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    const float inv_chunk = 1.f / (float)chunk;
    for (int i0 = 0;;) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kSelThreads + threadIdx.x;
        if (i < nc) {
          int c = (int)((float)ci[u] * inv_chunk);        // ci / chunk, corrected below
          c -= c * chunk > ci[u];
          c += (c + 1) * chunk <= ci[u];
          const int pos = tpre[c] + (i - tslot[c]);
          okey[pos] = ck[u];
          oidx[pos] = ci[u];
          kmin = min(kmin, ck[u]);
          kmax = max(kmax, ck[u]);
        }
        if (pivots && i < nc && fine_bin(ck[u], fbase) == fstar)
          atomicAdd(&histk[skew((int)((ck[u] - fbase) & (kHistBins - 1)))], 1);
      }
      i0 += U * kSelThreads;
      if (i0 >= nc) break;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kSelThreads + threadIdx.x;
        ck[u] = i < nc ? __ldcg(ckey + i) : 0u;
        ci[u] = i < nc ? __ldcg(cidx + i) : 0;
      }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane_id() == 0) {
      atomicMin(&kext[0], kmin);
      atomicMax(&kext[1], kmax);
    }
    __syncthreads();
    kmin = kext[0];
    const uint32_t span = kext[1] - kmin;
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
    bool located = false;
    if (take_all) {                                        // K* = the smallest key, all of them taken
      pmask = 0xffffffffu;
      remaining = nc;
      located = true;
    }
    if (pivots) {
      const int want = k - fabove;                         // keys of the k-th key's bin to take
      find_digit_skewed<kHistBins / kSelThreads>(histk, kHistBins, want, res, scratch);
      __syncthreads();
      prefix = fbase + ((uint32_t)fstar << 12) + (uint32_t)res[0] - kmin;   // K* - kmin
      pmask = 0xffffffffu;
      remaining = want - res[1];
      located = true;
      __syncthreads();
    }
    // otherwise: radix select on u = key - kmin, 12-bit digits from the highest bit of the
    // span down (the candidates share their leading key bits, so the digits spread over the bins)
    for (int hi = (located || !span) ? 0 : 32 - __clz(span); hi > 0;) {
      const int lo = hi > kHistBits ? hi - kHistBits : 0;
      const uint32_t dmask = (1u << (hi - lo)) - 1;
      for (int j = threadIdx.x; j < kHistBins + kHistBins / 32; j += blockDim.x) histk[j] = 0;
      __syncthreads();
      for (int i0 = threadIdx.x; i0 < nc; i0 += 4 * kSelThreads) {   // 4 keys requested at once
        uint32_t uu[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) uu[q] = i0 + q * kSelThreads < nc ? okey[i0 + q * kSelThreads] - kmin : 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (i0 + q * kSelThreads < nc && (uu[q] & pmask) == prefix)
            atomicAdd(&histk[skew((int)((uu[q] >> lo) & dmask))], 1);
      }
      __syncthreads();
      find_digit_skewed<kHistBins / kSelThreads>(histk, kHistBins, remaining, res, scratch);
      __syncthreads();
      prefix |= (uint32_t)res[0] << lo;
      pmask |= dmask << lo;
      remaining -= res[1];
      hi = lo;
      // When the chosen bin holds few keys (the usual case after the first digit), rank
      // them directly: the k-th key K* is the key with fewer than `remaining` keys above
      // it and at least `remaining` at or above it, among the keys of the bin.
      const int nb = histk[skew(res[0])];
      if (hi > 0 && nb <= kSelPivot) {
        uint32_t* piv = reinterpret_cast<uint32_t*>(tpre + kSelMaxChunks);   // [kSelPivot]
        if (threadIdx.x == 0) pcount = 0;
        __syncthreads();
        const uint32_t below = (1u << lane_id()) - 1;
        for (int i0 = 0; i0 < nc; i0 += kSelThreads) {      // one slot claim per warp
          const int i = i0 + threadIdx.x;
          const uint32_t u = i < nc ? okey[i] - kmin : 0u;
          const bool m = i < nc && (u & pmask) == prefix;
          const uint32_t bal = __ballot_sync(0xffffffffu, m);
          int base = 0;
          if (lane_id() == 0 && bal) base = atomicAdd(&pcount, __popc(bal));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (m) piv[base + __popc(bal & below)] = u;
        }
        __syncthreads();
        if ((int)threadIdx.x < nb) {
          const uint32_t v = piv[threadIdx.x];
          int gt = 0, ge = 0;
          int j = 0;
          for (; j + 16 <= nb; j += 16) {                    // 16 keys requested at once
            uint4 x[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) x[q] = *reinterpret_cast<const uint4*>(piv + j + 4 * q);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              gt += (x[q].x > v) + (x[q].y > v) + (x[q].z > v) + (x[q].w > v);
              ge += (x[q].x >= v) + (x[q].y >= v) + (x[q].z >= v) + (x[q].w >= v);
            }
          }
          for (; j < nb; ++j) {
            gt += piv[j] > v;
            ge += piv[j] >= v;
          }
          if (gt < remaining && remaining <= ge) {       // every key equal to K* writes the same
            res[0] = (int)v;
            res[1] = gt;
          }
        }
        __syncthreads();
        prefix = (uint32_t)res[0];
        pmask = 0xffffffffu;
        remaining -= res[1];
        break;
      }
    }
    // ordered emit: every key above K*, and the first `remaining` keys equal to K* (the
    // staged order is index order); each thread walks a contiguous run of odd length
    // (conflict-free banks) after one block scan of its (above, equal) counts
    const int per = ((nc + kSelThreads - 1) / kSelThreads) | 1;
    const int p0 = (int)threadIdx.x * per;
    const int p1 = p0 + per < nc ? p0 + per : nc;
    int cg = 0, ce = 0;
    for (int i0 = p0; i0 < p1; i0 += 4) {                 // 4 keys requested at once
      uint32_t uu[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) uu[q] = i0 + q < p1 ? okey[i0 + q] - kmin : 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        cg += i0 + q < p1 && uu[q] > prefix;
        ce += i0 + q < p1 && uu[q] == prefix;
      }
    }
    int total;
    const int ex = block_excl_scan((cg << 16) | ce, scratch, &total);
    int g = ex >> 16, e = ex & 0xffff;
    // the k indices land in shared memory first (the chunk table's space, free now), then
    // go out as coalesced 16-byte stores
    int32_t* sout = tslot;                                 // [k]; kSelMaxChunks * 2 >= CSA_MAX_TOPK
    for (int i0 = p0; i0 < p1; i0 += 4) {
      uint32_t uu[4];
      int32_t ii[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uu[q] = i0 + q < p1 ? okey[i0 + q] - kmin : 0u;
        ii[q] = i0 + q < p1 ? oidx[i0 + q] : 0;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (i0 + q >= p1) break;
        if (uu[q] > prefix) {
          const int o = g + (e < remaining ? e : remaining);
          if (o < k) {                                     // (bound holds unless the histogram is stale)
            sout[o] = ii[q];
            if (oscore) oscore[o] = key_value(uu[q] + kmin);
          }
          ++g;
        } else if (uu[q] == prefix) {
          if (e < remaining && g + e < k) {
            sout[g + e] = ii[q];
            if (oscore) oscore[g + e] = key_value(uu[q] + kmin);
          }
          ++e;
        }
      }
    }
    for (int j = nc + threadIdx.x; j < k; j += blockDim.x) {   // take_all with nc < k: -1 pads
      sout[j] = -1;
      if (oscore) oscore[j] = -INFINITY;
    }
    __syncthreads();
    if ((k & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0) {
      for (int j = threadIdx.x; j < k / 4; j += blockDim.x)
        reinterpret_cast<int4*>(out)[j] = reinterpret_cast<const int4*>(sout)[j];
    } else {
      for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = sout[j];
    }
    __syncthreads();
  } else {
    // more candidates than shared memory holds (rows dominated by ties): select on the
    // candidate list in global memory
    int32_t* sel = reinterpret_cast<int32_t*>(sel_smem);   // [k] selected indices, then bucketed
    int32_t* bucket = sel + CSA_MAX_TOPK;                  // [k] indices grouped by chunk
    uint32_t* selk = reinterpret_cast<uint32_t*>(bucket + CSA_MAX_TOPK);   // [k] their keys (sel_scores)
    uint32_t* bucketk = selk + CSA_MAX_TOPK;               // [k] keys beside bucket
    int* ccount = reinterpret_cast<int*>(bucketk + CSA_MAX_TOPK);   // [nchunks + 1] per-chunk counts -> offsets
    for (int j = threadIdx.x; j <= nchunks; j += blockDim.x) ccount[j] = 0;
    for (int j = threadIdx.x; j < k; j += blockDim.x) {   // in range even if a slot stays unset
      sel[j] = 0;
      selk[j] = 0u;
    }
    __syncthreads();
    auto cand_key = [&](int i) -> uint32_t { return __ldcg(ckey + i); };
    auto cand_idx = [&](int i) -> int32_t { return __ldcg(cidx + i); };
    // radix select on the 32-bit keys: digits of 11, 11 and 10 bits (skewed 2048-bin histogram)
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const uint32_t dmask = pass == 2 ? 1023u : 2047u;
      for (int j = threadIdx.x; j < 2048 + 64; j += blockDim.x) histk[j] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < nc; i += blockDim.x) {
        const uint32_t key = cand_key(i);
        if ((key & pmask) == prefix) atomicAdd(&histk[skew((int)((key >> shift) & dmask))], 1);
      }
      __syncthreads();
      find_digit_skewed<2048 / kSelThreads>(histk, 2048, remaining, res, scratch);
      __syncthreads();
      prefix |= (uint32_t)res[0] << shift;
      pmask |= dmask << shift;
      remaining -= res[1];
      __syncthreads();
    }
    // selected = keys above K*, plus the `remaining` lowest indices among keys equal to K*.
    // Slots come from warp-aggregated atomics (one per warp, or per distinct chunk within a
    // warp) -- contended shared-memory atomics serialise lane by lane.
    int32_t* eqlist = bucket;                              // keys equal to K* (scratch, before bucketing)
    if (threadIdx.x == 0) {
      lcount = 0;
      gslot = 0;
    }
    __syncthreads();
    for (int i0 = 0; i0 < nc; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const uint32_t key = i < nc ? cand_key(i) : 0u;
      const bool gt = i < nc && key > prefix;
      const bool eq = i < nc && key == prefix;
      const uint32_t mg = __ballot_sync(0xffffffffu, gt), me = __ballot_sync(0xffffffffu, eq);
      int bg = 0, be = 0;
      if (lane_id() == 0) {
        if (mg) bg = atomicAdd(&lcount, __popc(mg));
        if (me) be = atomicAdd(&gslot, __popc(me));
      }
      bg = __shfl_sync(0xffffffffu, bg, 0);
      be = __shfl_sync(0xffffffffu, be, 0);
      const uint32_t below = (1u << lane_id()) - 1;
      if (gt && bg + __popc(mg & below) < k) {
        sel[bg + __popc(mg & below)] = cand_idx(i);
        selk[bg + __popc(mg & below)] = key;
      }
      if (eq && be + __popc(me & below) < CSA_MAX_TOPK) eqlist[be + __popc(me & below)] = cand_idx(i);
    }
    __syncthreads();
    const int ngt = lcount, neq = gslot;
    // the `remaining` lowest indices among the equal keys (rank = equal keys with a lower index)
    if (neq <= CSA_MAX_TOPK) {
      for (int e = threadIdx.x; e < neq; e += blockDim.x) {
        const int32_t j = eqlist[e];
        int rank = 0;
        for (int q = 0; q < neq; ++q) rank += eqlist[q] < j;
        if (rank < remaining && ngt + rank < k) {
          sel[ngt + rank] = j;
          selk[ngt + rank] = prefix;
        }
      }
    } else {
      // more ties than the list holds (degenerate rows, e.g. constant scores): rank against
      // the whole candidate list
      for (int i = threadIdx.x; i < nc; i += blockDim.x) {
        if (cand_key(i) != prefix) continue;
        const int32_t j = cand_idx(i);
        int rank = 0;
        for (int q = 0; q < nc && rank < remaining; ++q) rank += (cand_key(q) == prefix && cand_idx(q) < j);
        if (rank < remaining && ngt + rank < k) {
          sel[ngt + rank] = j;
          selk[ngt + rank] = prefix;
        }
      }
    }
    __syncthreads();
    int nsel = ngt + (remaining < neq ? remaining : neq);   // == k (nv > k)
    nsel = nsel < k ? nsel : k;
    // ascending order: chunks are contiguous index ranges, so order = (chunk, rank in chunk)
    for (int i0 = 0; i0 < nsel; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const bool act = i < nsel;
      const int c = act ? sel[i] / chunk : -1;
      const uint32_t m = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t peers = __match_any_sync(m, c);
        if ((int)lane_id() == __ffs(peers) - 1) atomicAdd(&ccount[c], __popc(peers));
      }
    }
    __syncthreads();
    {
      int total;
      const int per = (nchunks + blockDim.x - 1) / blockDim.x;
      int loc = 0;
      for (int c = threadIdx.x * per; c < (int)(threadIdx.x + 1) * per && c < nchunks; ++c) loc += ccount[c];
      int off = block_excl_scan(loc, scratch, &total);
      __syncthreads();
      for (int c = threadIdx.x * per; c < (int)(threadIdx.x + 1) * per && c < nchunks; ++c) {
        const int n = ccount[c];
        ccount[c] = off;                                   // start of chunk c's bucket
        off += n;
      }
    }
    __syncthreads();
    for (int i0 = 0; i0 < nsel; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const bool act = i < nsel;
      const int32_t j = act ? sel[i] : 0;
      const int c = act ? j / chunk : -1;
      const uint32_t m = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t peers = __match_any_sync(m, c);
        const int leader = __ffs(peers) - 1;
        int base = 0;
        if ((int)lane_id() == leader) base = atomicAdd(&ccount[c], __popc(peers));
        base = __shfl_sync(peers, base, leader);
        bucket[base + __popc(peers & ((1u << lane_id()) - 1))] = j;   // ccount ends at the bucket's end
        bucketk[base + __popc(peers & ((1u << lane_id()) - 1))] = selk[i];
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nsel; i += blockDim.x) {
      const int32_t j = bucket[i];
      const int c = j / chunk;
      const int b_end = ccount[c];                         // end of this chunk's bucket
      const int b_start = c > 0 ? ccount[c - 1] : 0;       // = end of the previous bucket
      int rank = 0;
      for (int q = b_start; q < b_end; ++q) rank += bucket[q] < j;
      out[b_start + rank] = j;
      if (oscore) oscore[b_start + rank] = key_value(bucketk[i]);
    }
    __syncthreads();
  }
  // leave the row's header zeroed for the next call
  for (int j = threadIdx.x; j < kHistBins; j += blockDim.x) {
    ghist[j] = 0;
    gfine[j] = 0;
  }
  if (threadIdx.x == 0) {
    *fin = 0ull;
    *slots = 0;
  }
}

// ---------------------------------------------------------------- sharded decode
// One shard's k best entries as (score, global index) pairs, the unit every GPU
// contributes to the all-gather: local index i in [0, ns) -> (score, i + lo); -1 ->
// (-inf, -1).
struct ShardPair {
  float score;
  int32_t gidx;
};

__global__ void __launch_bounds__(256) shard_pack_kernel(const float* __restrict__ scores,
                                                         const int32_t* __restrict__ loc, int64_t n, int64_t ns,
                                                         int64_t lo, ShardPair* __restrict__ pairs) {
  griddep_sync();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t l = loc[i];
    const bool ok = l >= 0 && l < ns;
    pairs[i] = ok ? ShardPair{scores[i], (int32_t)(l + lo)} : ShardPair{-INFINITY, -1};
  }
}

// The gathered pairs, shard-major [G][B][k], as one row per sequence [B][G * k] of scores
// and global indices: in shard order the valid global indices are ascending, so a top-k
// over positions keeps the lower-index tie rule.
__global__ void __launch_bounds__(256) shard_gather_kernel(const ShardPair* __restrict__ pairs, int G, int B, int k,
                                                           float* __restrict__ row_scores,
                                                           int32_t* __restrict__ row_idx) {
  griddep_sync();
  const int64_t n = (int64_t)G * B * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = i / ((int64_t)B * k), rem = i % ((int64_t)B * k);
    const int64_t b = rem / k, j = rem % k;
    const int64_t o = b * (int64_t)G * k + g * k + j;
    const ShardPair pr = pairs[i];
    row_scores[o] = pr.gidx >= 0 ? pr.score : -INFINITY;   // padding never outranks an entry
    row_idx[o] = pr.gidx;
  }
}

// Index remap between global and shard-local entry numbers: in in [lo, hi) ->
// in - lo + add, else -1 (order kept).  Global -> local: (lo, hi) of the shard, add 0;
// local -> global: (0, shard size), add = the shard's first entry.
__global__ void __launch_bounds__(256) shard_remap_kernel(const int32_t* __restrict__ in, int64_t n, int64_t lo,
                                                          int64_t hi, int64_t add, int32_t* __restrict__ out) {
  griddep_sync();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t g = in[i];
    out[i] = (g >= lo && g < hi) ? (int32_t)(g - lo + add) : -1;
  }
}

}  // namespace csa
