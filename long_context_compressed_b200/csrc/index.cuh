// index.cuh -- Lightning Indexer scores
//   s[b,t,i] = sum_h w[b,t,h] * ReLU(<qI[b,t,h,:], kI[b,i,:]>)   for i < n_valid[b,t]
//   s[b,t,i] = -inf                                                  for n_valid[b,t] <= i < N
// ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.2; 64 index heads of
// 128 dims, keys shared by the heads, no 1/sqrt(d) factor).
//
// index_tc_kernel: a genuine dense contraction on the 5th-generation tensor
// cores.  Keys are the M = 128 operand (one tile = 128 keys x 128 dims), the
// TQ queries x 64 heads of a query group are the N = 64*TQ operand, K = 128.
// Both are staged by TMA (128-byte swizzle, K-major) into shared memory;
// one elected thread issues tcgen05.mma into a double-buffered fp32 TMEM
// accumulator; sixteen epilogue warps (4 sets taking tiles in turn, or 2 sets of
// 8 warps that split the group's queries when only 2 accumulators fit) read
// their 32 TMEM lanes (one key per
// thread), apply ReLU and the head weights, reduce over the 64 heads and store
// one fp32 score per (query, key).  Persistent: one CTA per SM walks a
// contiguous range of (sequence, query group, key tile) work items so that
// the key stream of each SM is sequential.
//   bf16 : kind::f16, fp32 accumulate.
//   e4m3 : kind::f8f6f4 with a per-key scale ks[b,i] and a per-(query, head)
//          scale qs[b,t,h]; both are positive so they commute with ReLU:
//          s = ks * sum_h (w * qs)_h * ReLU(<q8, k8>).
//   mxfp4: kind::mxf4.block_scale (the FP4 index QK of §2 / §4.2): packed E2M1 codes
//          (64 bytes per 128-dim row, 64-byte swizzle) with one E8M0 scale per 32 dims
//          applied inside the MMA.  Scales are stored in the tensor-core layout
//          (csa_quantize_mxfp4_sf128: 512 bytes per 128 rows), copied next to the codes
//          into shared memory by a bulk copy and from there into tensor memory by
//          tcgen05.cp; two MMAs of K = 64 per tile.
//
// index_simt_kernel: fp32 SIMT path (FMA), used for fp32 inputs and for the
// exact rescoring of a candidate list.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace csa {

constexpr int kIdxHeads = 64;
constexpr int kIdxDim = 128;
constexpr int kIdxTileKeys = 128;
constexpr int kMaxAcc = 4;
constexpr int kIdxEpiWarps = 16;
constexpr int kIdxThreads = 64 + 32 * kIdxEpiWarps;   // TMA warp, MMA warp, 16 epilogue warps
constexpr int kKsAhead = 3;                     // key-scale prefetch distance (items of one epilogue set)
constexpr int kKsRing = kKsAhead + 1;
constexpr int kHistBinsIdx = 4096;              // 12-bit histogram of order-preserving score keys

// Order-preserving uint32 key of a score (-0.0 folded to +0.0): key order equals score order.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Its top 12 bits: bin order equals score order.
__device__ __forceinline__ uint32_t score_bin(float x) { return score_key(x) >> 20; }

struct IndexParams {
  const float* w;        // [B, T, 64]
  const float* q_scale;  // [B, T, 64] or null (bf16)
  const float* k_scale;  // [B, N] or null (bf16)
  const int32_t* n_valid;  // [B, T]
  float* scores;         // [B, T, N]
  const uint8_t* q_sf;   // mxfp4: query scales [B][ceil(T*64/128)][512] (tensor-core layout)
  const uint8_t* k_sf;   // mxfp4: key scales [B][ceil(N/128)][512]
  int* hist;             // per-row 4096-bin histogram of the score keys (T == 1), row stride hist_stride, or null
  int64_t hist_stride;   // ints between consecutive rows' histograms
  int B, T;
  int64_t N;
  int TQ;                // queries per group (1, 2 or 4)
  int stages;            // key pipeline depth
  // candidate mode (index_tc_kernel<MODE, true>): no score is written; a valid score whose
  // key is >= thr[row] is appended to row's list cand[row][..] as (key << 32) | ~i.
  // cand_chunk 32: an epilogue warp reserves 32 slots of a row at a time (cand_cnt[row]
  // += 32), fills them in order and zero-fills the unused tail of its last chunk (one
  // atomic per 32 entries; for rows that span few CTAs, so few warps leave a tail).
  // cand_chunk 1: each ballot reserves exactly its entries.  Slots at or past cand_cap
  // are not written (cand_cnt still counts them).
  const uint32_t* thr;          // [B*T]
  int* cand_cnt;                // [B*T]
  unsigned long long* cand;     // [B*T][cand_cap]
  int cand_cap;
  int cand_chunk;               // 32 or 1
  const int* gate;              // null, or a device int written by an earlier launch: 0 -> no work
  // keys_ready: the key operands (codes, scales) are not written by the launch before this
  // one on the stream, so the producer issues the first `stages` key tiles before it waits
  // for that launch (programmatic dependent launch); never together with gate
  int keys_ready;
};

// Operand modes of index_tc_kernel.
enum : int { kIdxBf16 = 0, kIdxE4m3 = 1, kIdxMxfp4 = 2 };

template <int MODE>
struct IndexCfg {
  static constexpr bool FP4 = MODE == kIdxMxfp4;
  static constexpr int kRowBytes = MODE == kIdxBf16 ? 256 : (MODE == kIdxE4m3 ? 128 : 64);   // one 128-dim row
  static constexpr int kCodeBytes = kIdxTileKeys * kRowBytes;               // codes of one key tile
  static constexpr int kSfBytes = FP4 ? 512 : 0;                            // scales of one key tile
  static constexpr int kKeyBytes = kCodeBytes + (FP4 ? 1024 : 0);           // one pipeline stage (1 KiB aligned)
  static constexpr int kQRowBytes = kRowBytes;                              // one (t, h) row
  static constexpr int kAtomBytes = FP4 ? 64 : 128;                         // swizzle width
  static constexpr int kAtoms = kRowBytes / kAtomBytes;                     // K atoms per row
  static constexpr uint32_t kLayout = FP4 ? kLayoutSW64 : kLayoutSW128;
  static constexpr int kKInstr = MODE == kIdxBf16 ? 16 : (MODE == kIdxE4m3 ? 32 : 64);   // K per MMA
  static constexpr int kKSteps = kIdxDim / kKInstr;
  static constexpr int kKBytes = kKInstr * kRowBytes / kIdxDim;             // bytes of K per MMA
};

// Work item w -> (b, query group, key tile), ordered with the key tile fastest.
struct IndexItem {
  int b, qg;
  int64_t kt;
};
__device__ __forceinline__ IndexItem index_item(int64_t w, int QG, int64_t KT) {
  IndexItem it;
  it.kt = w % KT;
  const int64_t r = w / KT;
  it.qg = (int)(r % QG);
  it.b = (int)(r / QG);
  return it;
}
// Advance to the next work item without division (the loops below are latency
// critical: a 64-bit division per item costs several hundred cycles).
__device__ __forceinline__ void index_next(IndexItem& it, int QG, int64_t KT) {
  if (++it.kt == KT) {
    it.kt = 0;
    if (++it.qg == QG) {
      it.qg = 0;
      ++it.b;
    }
  }
}

template <int MODE, bool EMIT = false>
__global__ void __launch_bounds__(kIdxThreads, 1) index_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap qmap,
                                                          const IndexParams p) {
  using Cfg = IndexCfg<MODE>;
  constexpr bool FP8 = MODE == kIdxE4m3;            // per-row scales applied in the epilogue
  constexpr bool FP4 = Cfg::FP4;                    // block scales applied by the MMA
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int TQ = p.TQ;
  const int NQ = TQ * kIdxHeads;                    // MMA N
  const int q_bytes = NQ * Cfg::kQRowBytes;
  uint8_t* q_smem = smem;
  // (mxfp4: the group's 512-byte scale atom after the codes, 1 KiB aligned)
  uint8_t* qsf_smem = smem + ((q_bytes + 1023) & ~1023);
  uint8_t* k_smem = qsf_smem + (FP4 ? 1024 : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(k_smem + (size_t)p.stages * Cfg::kKeyBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + p.stages;
  uint64_t* qfull = bars + 2 * p.stages;
  uint64_t* qempty = qfull + 1;
  uint64_t* tfull = qfull + 2;                      // [kMaxAcc]
  uint64_t* tempty = qfull + 2 + kMaxAcc;           // [kMaxAcc]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qfull + 2 + 2 * kMaxAcc);
  float* w_all = reinterpret_cast<float*>(qfull + 4 + 2 * kMaxAcc);  // [8 epilogue warps][TQ][64]
  float* ks_all = w_all + kIdxEpiWarps * TQ * kIdxHeads;             // [kKsRing][epilogue threads] key-scale ring
  // score histograms of the first two rows this CTA touches (when p.hist is set); in the
  // candidate mode the same place holds each epilogue warp's row thresholds and open
  // 32-slot chunks: [warp][thr 4 | chunk base 4 | slots used 4]
  int* hist_s = reinterpret_cast<int*>(ks_all + kKsRing * 32 * kIdxEpiWarps);   // [2][kHistBinsIdx]

  const int QG = (p.T + TQ - 1) / TQ;
  const int64_t KT = (p.N + kIdxTileKeys - 1) / kIdxTileKeys;
  const int64_t items = (int64_t)p.B * QG * KT;
  const int64_t w0 = items * blockIdx.x / gridDim.x;
  int64_t w1 = items * (blockIdx.x + 1) / gridDim.x;
  // TMEM accumulators in flight (2 or 4); mxfp4 keeps 32 columns for the block scales
  const int acc_fit = (FP4 ? 480 : 512) / NQ;
  const int NACC = acc_fit >= kMaxAcc ? kMaxAcc : (acc_fit >= 2 ? 2 : 1);
  // epilogue sets: one per accumulator; with 2 accumulators each set has 8 warps, two
  // per TMEM lane quarter, splitting the group's queries
  const int nsets = NACC >= 4 ? 4 : 2;
  const int set_warps = kIdxEpiWarps / nsets;
  const uint32_t tmem_cols = FP4 ? 512u : ((uint32_t)(NACC * NQ) < 32 ? 32u : (uint32_t)(NACC * NQ));
  const uint32_t sfa_col0 = (uint32_t)(NACC * NQ);          // mxfp4: [acc] key scales, 4 columns each
  const uint32_t sfb_col0 = sfa_col0 + 4 * kMaxAcc;        // mxfp4: [2] query scales, 4 columns each

  const int warp = warp_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int a = 0; a < kMaxAcc; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], set_warps);             // one arrive per epilogue warp of the set
    }
    fence_mbar_init();
    prefetch_tmap(&kmap);
    prefetch_tmap(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  if (p.hist)
    for (int j = threadIdx.x; j < 2 * kHistBinsIdx; j += blockDim.x) hist_s[j] = 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // key tiles that do not depend on the previous launch stream in while it finishes
  const int npre = p.keys_ready ? (int)(w1 - w0 < p.stages ? w1 - w0 : p.stages) : 0;
  if (npre > 0 && warp == 0 && elect_one()) {
    IndexItem it = index_item(w0, QG, KT);
    for (int j = 0; j < npre; ++j, index_next(it, QG, KT)) {
      mbar_arrive_expect_tx(&full[j], (uint32_t)(Cfg::kCodeBytes + Cfg::kSfBytes));
      uint8_t* dst = k_smem + (size_t)j * Cfg::kKeyBytes;
      for (int a = 0; a < Cfg::kAtoms; ++a)
        tma_load_3d(dst + (size_t)a * kIdxTileKeys * 128, &kmap, &full[j], a * 64, (int)(it.kt * kIdxTileKeys),
                    it.b);
      if (FP4) bulk_load(dst + Cfg::kCodeBytes, p.k_sf + ((int64_t)it.b * KT + it.kt) * 512, 512, &full[j]);
    }
  }
  griddep_sync();
  if (p.gate && __ldcg(p.gate) == 0) w1 = w0;       // gated off: every role walks no items
  const int hist_row0 = index_item(w0, QG, KT).b;   // T == 1 whenever p.hist is set: row = sequence

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      int prev_b = -1, prev_qg = -1;
      uint32_t qe_phase = 0;
      int64_t cnt = 0;
      int st_i = 0;
      uint32_t st_ph = 0;
      IndexItem it = index_item(w0, QG, KT);
      for (int64_t w = w0; w < w1; ++w, ++cnt, index_next(it, QG, KT)) {
        if (it.b != prev_b || it.qg != prev_qg) {
          if (prev_b >= 0) {
            if (!mbar_wait(qempty, qe_phase)) break;
            qe_phase ^= 1;
          }
          mbar_arrive_expect_tx(qfull, (uint32_t)(q_bytes + Cfg::kSfBytes));
          for (int a = 0; a < Cfg::kAtoms; ++a)
            tma_load_3d(q_smem + (size_t)a * NQ * 128, &qmap, qfull, a * 64, it.qg * NQ, it.b);
          if (FP4) {
            const int64_t qtiles = ((int64_t)p.T * kIdxHeads + 127) / 128;
            bulk_load(qsf_smem, p.q_sf + ((int64_t)it.b * qtiles + (int64_t)it.qg * NQ / 128) * 512, 512, qfull);
          }
          prev_b = it.b;
          prev_qg = it.qg;
        }
        const int s = st_i;
        const uint32_t ph = st_ph;
        if (++st_i == p.stages) { st_i = 0; st_ph ^= 1; }
        if (cnt < npre) continue;                   // issued before the grid dependency wait
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(Cfg::kCodeBytes + Cfg::kSfBytes));
        uint8_t* dst = k_smem + (size_t)s * Cfg::kKeyBytes;
        for (int a = 0; a < Cfg::kAtoms; ++a)
          tma_load_3d(dst + (size_t)a * kIdxTileKeys * 128, &kmap, &full[s], a * 64, (int)(it.kt * kIdxTileKeys),
                      it.b);
        if (FP4) bulk_load(dst + Cfg::kCodeBytes, p.k_sf + ((int64_t)it.b * KT + it.kt) * 512, 512, &full[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc = make_idesc(128, NQ, FP8 ? 0u : 1u, 0, 0);
      int prev_b = -1, prev_qg = -1;
      uint32_t qf_phase = 0;
      uint32_t sfb_col = sfb_col0;                   // mxfp4: this group's query-scale columns
      int64_t cnt = 0;
      int st_i = 0, ac_i = 0;
      uint32_t st_ph = 0, ac_ph = 0;
      IndexItem it = index_item(w0, QG, KT);
      for (int64_t w = w0; w < w1; ++w, ++cnt, index_next(it, QG, KT)) {
        if (it.b != prev_b || it.qg != prev_qg) {
          if (prev_b >= 0) mma_commit(qempty);      // old Q free once its MMAs finish
          if (!mbar_wait(qfull, qf_phase)) break;
          qf_phase ^= 1;
          prev_b = it.b;
          prev_qg = it.qg;
          if (FP4) {
            // the group's query scales into tensor memory (alternating column sets, so the
            // previous group's MMAs still read theirs)
            sfb_col = sfb_col0 + (qf_phase ? 0u : 4u);
            tc_fence_after();
            tmem_cp_sf128(tmem_base + sfb_col, smem_desc(smem_u32(qsf_smem), 16, 128, 0));
          }
        }
        const int s = st_i;
        const uint32_t ph = st_ph;
        if (++st_i == p.stages) { st_i = 0; st_ph ^= 1; }
        const int acc = ac_i;
        const uint32_t aph = ac_ph;
        if (++ac_i == NACC) { ac_i = 0; ac_ph ^= 1; }
        if (!mbar_wait(&tempty[acc], aph ^ 1)) break;
        if (!mbar_wait(&full[s], ph)) break;
        tc_fence_after();
        const uint32_t kbase = smem_u32(k_smem + (size_t)s * Cfg::kKeyBytes);
        const uint32_t qbase = smem_u32(q_smem);
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NQ);
        if (FP4) {
          // the tile's key scales into this accumulator's columns (freed with the accumulator)
          tmem_cp_sf128(tmem_base + sfa_col0 + 4u * (uint32_t)acc,
                        smem_desc(kbase + Cfg::kCodeBytes, 16, 128, 0));
        }
#pragma unroll
        for (int kk = 0; kk < Cfg::kKSteps; ++kk) {
          const int byte_k = kk * Cfg::kKBytes;          // byte offset along K
          const int atom = byte_k / Cfg::kAtomBytes;
          const int inner = byte_k % Cfg::kAtomBytes;
          const uint32_t sbo = 8 * Cfg::kAtomBytes;
          const uint64_t adesc =
              smem_desc(kbase + atom * kIdxTileKeys * Cfg::kAtomBytes + inner, 16, sbo, Cfg::kLayout);
          const uint64_t bdesc = smem_desc(qbase + atom * NQ * Cfg::kAtomBytes + inner, 16, sbo, Cfg::kLayout);
          if constexpr (FP4) {
            // scales of dims 64 kk .. 64 kk + 63: bytes 2 kk, 2 kk + 1 of each row's scale word
            const uint32_t sf_byte = 2u * (uint32_t)kk;
            mma_mxf4(d_tmem, adesc, bdesc, make_idesc_mxf4(128, NQ, sf_byte, sf_byte),
                     tmem_base + sfa_col0 + 4u * (uint32_t)acc + (sf_byte << 30), tmem_base + sfb_col + (sf_byte << 30),
                     kk > 0 ? 1u : 0u);
          } else if (FP8) {
            mma_f8(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          } else {
            mma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[acc]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..17)
    // nsets sets take the work items in turn (set s: items w0 + s, w0 + s + nsets, ..);
    // warp w owns TMEM lanes 32*(w%4) .. +31, i.e. one key per thread, and the
    // queries [q_lo, q_hi) of the group.
    const int e = warp - 2;
    const int quarter = warp & 3;                   // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + (int)lane_id();  // key within the tile
    const int es = (e >> 2) % nsets;                // epilogue set
    const int qpart = (e >> 2) / nsets;             // 0, or 0/1 with 2 sets
    const int q_lo = qpart * TQ * nsets / 4, q_hi = (qpart + 1) * TQ * nsets / 4;
    const int acc_shift = NACC == 4 ? 2 : (NACC == 2 ? 1 : 0);
    float* w_s = w_all + e * TQ * kIdxHeads;
    int nv_q[4] = {0, 0, 0, 0};
    // key scales (e4m3) travel by cp.async into a per-thread ring in shared memory,
    // kKsAhead of this set's items ahead along a second iterator: no register waits
    // on a load in flight
    constexpr int kEpiThreads = 32 * kIdxEpiWarps;
    float* ks_ring = ks_all + (threadIdx.x - 64);     // column of this epilogue thread
    IndexItem ahead = index_item(w0, QG, KT);
    int64_t w_ahead = w0;
    for (int j = 0; j < es; ++j) { index_next(ahead, QG, KT); ++w_ahead; }
    int ring_put = 0;
    auto ks_fetch = [&]() {
      if (FP8 && w_ahead < w1) {
        const int64_t ii = ahead.kt * kIdxTileKeys + row;
        if (ii < p.N) cp_async_4(ks_ring + ring_put * kEpiThreads, p.k_scale + (int64_t)ahead.b * p.N + ii);
      }
      cp_async_commit();
      ring_put = ring_put + 1 == kKsRing ? 0 : ring_put + 1;
      w_ahead += nsets;
      for (int j = 0; j < nsets; ++j) index_next(ahead, QG, KT);
    };
    if (FP8)
      for (int j = 0; j < kKsAhead; ++j) ks_fetch();
    int ring_get = 0;
    int prev_b = -1, prev_qg = -1;
    // candidate mode: the group's row thresholds and this warp's open 32-slot chunk per
    // query (base -1: none) live in shared memory (registers are at the cap); every lane
    // reads them, lane 0 writes them
    int* emit_s = hist_s + e * 12;
    int64_t row0 = 0;                               // b * T + qg * TQ of the current group
    auto close_chunks = [&]() {                     // zero-fill the unused tails
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int base = emit_s[4 + q], used = emit_s[8 + q];
        if (base >= 0 && (int)lane_id() >= used && base + 32 <= p.cand_cap)
          p.cand[(row0 + q) * p.cand_cap + base + lane_id()] = 0ull;
      }
      __syncwarp();
      if (lane_id() < 4) {
        emit_s[4 + lane_id()] = -1;
        emit_s[8 + lane_id()] = 0;
      }
      __syncwarp();
    };
    if constexpr (EMIT) {
      if (lane_id() < 4) {
        emit_s[4 + lane_id()] = -1;
        emit_s[8 + lane_id()] = 0;
      }
      __syncwarp();
    }
    IndexItem it = index_item(w0, QG, KT);
    int64_t w = w0;
    int cnt = 0;
    for (int j = 0; j < es; ++j) { index_next(it, QG, KT); ++w; ++cnt; }
    for (; w < w1; w += nsets, cnt += nsets) {
      if (cnt >= nsets)
        for (int j = 0; j < nsets; ++j) index_next(it, QG, KT);
      if (it.b != prev_b || it.qg != prev_qg) {
        if constexpr (EMIT) {
          close_chunks();
          const int tq = it.qg * TQ + (int)lane_id();
          if (lane_id() < 4)
            emit_s[lane_id()] = (int)(((int)lane_id() < TQ && tq < p.T) ? __ldg(p.thr + (int64_t)it.b * p.T + tq)
                                                                        : 0xffffffffu);
          __syncwarp();
          row0 = (int64_t)it.b * p.T + (int64_t)it.qg * TQ;
        }
        // each epilogue warp keeps a private copy of the group's head weights; the
        // weights, query scales and n_valid are all requested before any is used
        // (one memory round trip, overlapping the wait for the first accumulator)
        constexpr int PER = 4 * kIdxHeads / 32;
        const int tq = it.qg * TQ + (int)lane_id();
        const int nv_l = ((int)lane_id() < TQ && tq < p.T) ? __ldg(p.n_valid + (int64_t)it.b * p.T + tq) : 0;
        __syncwarp();
#pragma unroll
        for (int u0 = 0; u0 < PER; u0 += PER / 2) {     // two batches of loads (register budget)
          float wv[PER / 2], sv[PER / 2];
#pragma unroll
          for (int u = 0; u < PER / 2; ++u) {
            const int j = (int)lane_id() + 32 * (u0 + u);
            const int t = it.qg * TQ + j / kIdxHeads;
            const bool in = j < TQ * kIdxHeads && t < p.T;
            const int64_t o = ((int64_t)it.b * p.T + t) * kIdxHeads + (j % kIdxHeads);
            wv[u] = in ? __ldg(p.w + o) : 0.f;
            sv[u] = (FP8 && in) ? __ldg(p.q_scale + o) : 1.f;
          }
#pragma unroll
          for (int u = 0; u < PER / 2; ++u) {
            const int j = (int)lane_id() + 32 * (u0 + u);
            if (j < TQ * kIdxHeads) w_s[j] = FP8 ? wv[u] * sv[u] : wv[u];
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) nv_q[q] = __shfl_sync(0xffffffffu, nv_l, q);
        __syncwarp();
        prev_b = it.b;
        prev_qg = it.qg;
      }
      const int acc = cnt & (NACC - 1);
      const uint32_t aph = (uint32_t)(cnt >> acc_shift) & 1u;
      float ks = 1.f;
      if (FP8) {
        ks_fetch();                                 // item kKsAhead ahead
        cp_async_wait_group<kKsAhead>();            // this item's copy has landed
        ks = ks_ring[ring_get * kEpiThreads];
        ring_get = ring_get + 1 == kKsRing ? 0 : ring_get + 1;
      }
      if (!mbar_wait(&tfull[acc], aph)) break;
      tc_fence_after();
      const int64_t i = it.kt * kIdxTileKeys + row;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q < q_lo) continue;
        if (q >= q_hi) break;
        const int t = it.qg * TQ + q;
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * NQ + q * 64);
        if (t >= p.T) continue;                       // uniform over the warp
        const float* wq = w_s + q * kIdxHeads;
        // four independent chains (heads = 0, 1, 2, 3 mod 4) held as two packed fp32 pairs:
        // one f32x2 FMA per pair of heads, each half rounded as its own fmaf
        unsigned long long a01 = 0ull, a23 = 0ull;
#pragma unroll
        for (int half = 0; half < 2; ++half) {          // 32 heads at a time (register budget)
          float v[32];
          tmem_ld32(taddr + 32 * half, v);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 32; h += 4) {
            const float2 w01 = *reinterpret_cast<const float2*>(wq + 32 * half + h);
            const float2 w23 = *reinterpret_cast<const float2*>(wq + 32 * half + h + 2);
            f32x2_fma(a01, f32x2_pack(w01.x, w01.y), f32x2_pack(fmaxf(v[h], 0.f), fmaxf(v[h + 1], 0.f)));
            f32x2_fma(a23, f32x2_pack(w23.x, w23.y), f32x2_pack(fmaxf(v[h + 2], 0.f), fmaxf(v[h + 3], 0.f)));
          }
        }
        const float2 s01 = f32x2_unpack(a01), s23 = f32x2_unpack(a23);
        const float sc = (s01.x + s01.y) + (s23.x + s23.y);
        if constexpr (EMIT) {
          const uint32_t key = score_key(sc * ks);
          const bool pass = i < p.N && i < nv_q[q] && key >= (uint32_t)emit_s[q];
          const uint32_t m = __ballot_sync(0xffffffffu, pass);
          if (m) {                                    // uniform over the warp
            const int n = __popc(m);
            const int rank = __popc(m & ((1u << lane_id()) - 1u));
            const bool chunked = p.cand_chunk != 1;
            const int base = chunked ? emit_s[4 + q] : -1, used = chunked ? emit_s[8 + q] : 0;
            const int room = base < 0 ? 0 : 32 - used;
            int nb = base;
            if (n > room) {                             // a new chunk (or exactly n slots) for the rest
              int g = 0;
              if (lane_id() == 0) g = atomicAdd(&p.cand_cnt[row0 + q], chunked ? 32 : n);
              nb = __shfl_sync(0xffffffffu, g, 0);
            }
            if (pass) {
              const int slot = rank < room ? base + used + rank : nb + (rank - room);
              if (slot < p.cand_cap)                    // (past it the row fails: never read)
                p.cand[(row0 + q) * p.cand_cap + slot] =
                    ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)i);
            }
            if (chunked) {
              __syncwarp();
              if (lane_id() == 0) {
                emit_s[4 + q] = n > room ? nb : base;
                emit_s[8 + q] = n > room ? n - room : used + n;
              }
              __syncwarp();
            }
          }
        } else if (i < p.N) {
          const bool valid = i < nv_q[q];
          const float val = valid ? sc * ks : -INFINITY;
          p.scores[((int64_t)it.b * p.T + t) * p.N + i] = val;
          if (p.hist && valid) {
            const uint32_t bin = score_bin(val);
            const int slot = it.b - hist_row0;
            if (slot < 2) atomicAdd(&hist_s[slot * kHistBinsIdx + bin], 1);
            else atomicAdd(&p.hist[(int64_t)it.b * p.hist_stride + bin], 1);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&tempty[acc]);
    }
    if constexpr (EMIT) close_chunks();
    if (FP8) cp_async_wait_group<0>();              // no copy may land after the CTA has left
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
  if (p.hist) {
    for (int j = threadIdx.x; j < 2 * kHistBinsIdx; j += blockDim.x) {
      const int c = hist_s[j];
      const int row = hist_row0 + j / kHistBinsIdx;
      if (c != 0 && row < p.B) atomicAdd(&p.hist[(int64_t)row * p.hist_stride + (j % kHistBinsIdx)], c);
    }
  }
}

constexpr int kIdxSimtSmem = (kIdxHeads + 64) * (kIdxDim + 4) * 4;

__device__ __forceinline__ float4 load4f(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4f(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// SIMT path (fp32 FMA): CTA = (tile of 64 keys, query t, sequence b); 256 threads
// as a 16 x 16 grid, each computing 4 keys x 4 heads over the 128 dims from
// shared memory, then ReLU, head weights, and a reduction over the 16 head
// groups.  Inputs fp32 or bf16 (widened exactly to fp32).
//   GATHER = false: keys 0..N-1, scores[b,t,i] (-inf for i >= n_valid[b,t]).
//   GATHER = true : keys cand[b,t,j] for j < kc (the exact rescoring of a
//                   candidate list); out[b,t,j], -inf where cand is outside [0, N).
template <typename Tin, bool GATHER>
__global__ void __launch_bounds__(256) index_simt_kernel(const Tin* __restrict__ qI, const float* __restrict__ w,
                                                         const Tin* __restrict__ kI,
                                                         const int32_t* __restrict__ n_valid,
                                                         const int32_t* __restrict__ cand, int kc, int T, int64_t N,
                                                         float* __restrict__ out) {
  griddep_sync();
  constexpr int KT = 64, PAD = 4;
  extern __shared__ __align__(16) float f32_smem[];
  float(*qs)[kIdxDim + PAD] = reinterpret_cast<float(*)[kIdxDim + PAD]>(f32_smem);
  float(*ks)[kIdxDim + PAD] = reinterpret_cast<float(*)[kIdxDim + PAD]>(f32_smem + kIdxHeads * (kIdxDim + PAD));
  __shared__ float red[16][KT];
  __shared__ float ws[kIdxHeads];
  __shared__ int64_t krow[KT];
  const int b = blockIdx.z, t = blockIdx.y;
  const int64_t bt = (int64_t)b * T + t;
  const int64_t k0 = (int64_t)blockIdx.x * KT;
  const int64_t width = GATHER ? (int64_t)kc : N;     // entries of the output row
  if (threadIdx.x < KT) {
    const int64_t j = k0 + threadIdx.x;
    int64_t r = -1;
    if (j < width) {
      r = GATHER ? (int64_t)cand[bt * kc + j] : j;
      if (r < 0 || r >= N) r = -1;
    }
    krow[threadIdx.x] = r;
  }
  const Tin* qrow = qI + bt * kIdxHeads * kIdxDim;
  for (int j = threadIdx.x; j < kIdxHeads * kIdxDim / 4; j += 256) {
    const int h = j / (kIdxDim / 4), d = (j % (kIdxDim / 4)) * 4;
    *reinterpret_cast<float4*>(&qs[h][d]) = load4f(qrow + h * kIdxDim + d);
  }
  if (threadIdx.x < kIdxHeads) ws[threadIdx.x] = w[bt * kIdxHeads + threadIdx.x];
  __syncthreads();
  for (int j = threadIdx.x; j < KT * kIdxDim / 4; j += 256) {
    const int r = j / (kIdxDim / 4), d = (j % (kIdxDim / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t row = krow[r];
    if (row >= 0) v = load4f(kI + ((int64_t)b * N + row) * kIdxDim + d);
    *reinterpret_cast<float4*>(&ks[r][d]) = v;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
  for (int d = 0; d < kIdxDim; d += 4) {
    float4 kv[4], qv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) kv[u] = *reinterpret_cast<const float4*>(&ks[tx + 16 * u][d]);
#pragma unroll
    for (int v = 0; v < 4; ++v) qv[v] = *reinterpret_cast<const float4*>(&qs[ty + 16 * v][d]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        acc[u][v] = fmaf(kv[u].x, qv[v].x, acc[u][v]);
        acc[u][v] = fmaf(kv[u].y, qv[v].y, acc[u][v]);
        acc[u][v] = fmaf(kv[u].z, qv[v].z, acc[u][v]);
        acc[u][v] = fmaf(kv[u].w, qv[v].w, acc[u][v]);
      }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float s = 0.f;
#pragma unroll
    for (int v = 0; v < 4; ++v) s = fmaf(ws[ty + 16 * v], fmaxf(acc[u][v], 0.f), s);
    red[ty][tx + 16 * u] = s;
  }
  __syncthreads();
  if (threadIdx.x < KT) {
    const int64_t j = k0 + threadIdx.x;
    float s = 0.f;
    for (int g = 0; g < 16; ++g) s += red[g][threadIdx.x];
    if (j < width) {
      bool ok = krow[threadIdx.x] >= 0;
      if (!GATHER) ok = ok && j < n_valid[bt];
      out[bt * width + j] = ok ? s : -INFINITY;
    }
  }
}

}  // namespace csa
