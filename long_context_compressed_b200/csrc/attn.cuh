// attn.cuh -- shared-KV multi-query attention with an attention sink over the
// memory [SWA rows ; compressed rows]:
//   z_j = scale * <q_h, row_j>,  p_j = exp(z_j) / (exp(sink_h) + sum_l exp(z_l)),
//   o_h = sum_j p_j row_j            (the latent row is both key and value)
// "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §4.2 (Shared-KV MQA over the
// selected entries), §6 (128-token SWA branch, sink probability), §7 (memory =
// concat(local_kv, selected_kv), one softmax); "解密DeepSeek-V4-Flash-NVFP4的混合
// 注意力机制…" (sparse_attn(q, kv, attn_sink, topk_idxs, softmax_scale), gather by
// index + online softmax).
//
// Row list of query (b, t) at absolute position pos:
//   SWA rows   : positions max(0, pos-127)..pos that lie inside the SWA buffer
//                (buffer row = position - swa_pos0), in position order;
//   memory rows: sparse_attn -> kv[idx[b,t,e]] for e < k (an index outside
//                [0, N) contributes nothing); hca_attn -> kv[e] for
//                e < min(N, (pos+1)/ratio) (complete blocks only).
//
// attn_tc_kernel (bf16): one CTA per (split, D-slice, query).  The query block
// (H heads padded to the M = 128 operand, all D dims) stays in shared memory;
// KV rows are gathered with 16-byte cp.async into 128-byte-swizzled K-major
// tiles of R rows; S = Q K^T (tcgen05, fp32 in TMEM, double buffered); four
// softmax warps (one head per thread) run the online softmax in the log2
// domain, writing P (bf16) to shared memory; O += P V (tcgen05; the same KV
// tile read as an MN-major operand, restricted to this CTA's D-slice of width
// DH <= 256) accumulates in TMEM.  O is rescaled only when a tile's maximum
// exceeds the running reference by more than 2^8, so exponentials stay <= 256.
// With several splits the CTA writes (O, m, l) partials that attn_combine_kernel
// merges together with the sink.
//
// attn_f32_kernel: fp32 SIMT (one warp per head), exact online softmax.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace csa {

constexpr int kSwaWindow = 128;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnParams {
  const void* q;          // [B, T, H, D]
  const void* kv;         // [B, N, D]
  const void* swa;        // [B, W, D]
  const int64_t* swa_pos0;  // [B]
  const int64_t* q_pos;   // [B, T]
  const float* sink;      // [H]
  const int32_t* idx;     // [B, T, k] (sparse) or null (hca)
  void* out;              // [B, T, H, D]
  float* ws_o;            // [nsplit, B*T, H, D] partial O (nsplit > 1)
  float* ws_ml;           // [nsplit, B*T, H, 2] partial (m, l), log2 domain
  float scale;
  int B, T, H, D, W, k, ratio, nsplit;
  int sparse;             // 1: memory rows from idx (sparse_attn); 0: dense prefix (hca_attn)
  int64_t N;
};

struct RowList {
  int64_t swa_row0;   // first SWA buffer row
  int n_swa;          // SWA rows
  int n_mem;          // memory rows (k for sparse, visible entries for hca)
};

__device__ __forceinline__ RowList make_row_list(const AttnParams& p, int b, int t) {
  RowList rl;
  const int64_t pos = p.q_pos[(int64_t)b * p.T + t];
  const int64_t s0 = p.swa_pos0[b];
  int64_t lo = pos - (kSwaWindow - 1);
  if (lo < 0) lo = 0;
  if (lo < s0) lo = s0;
  int64_t hi = pos;
  if (hi > s0 + p.W - 1) hi = s0 + p.W - 1;
  rl.n_swa = hi >= lo ? (int)(hi - lo + 1) : 0;
  rl.swa_row0 = lo - s0;
  if (p.sparse) {
    rl.n_mem = p.k;
  } else {
    int64_t nv = pos >= 0 ? (pos + 1) / p.ratio : 0;
    if (nv > p.N) nv = p.N;
    rl.n_mem = (int)nv;
  }
  return rl;
}

// Row r of the list -> element offset of its first value, or -1 if it contributes nothing.
__device__ __forceinline__ int64_t row_offset(const AttnParams& p, const RowList& rl, int b, int t, int r,
                                              bool* is_swa) {
  if (r < rl.n_swa) {
    *is_swa = true;
    return ((int64_t)b * p.W + rl.swa_row0 + r) * p.D;
  }
  *is_swa = false;
  const int e = r - rl.n_swa;
  int64_t i;
  if (p.sparse) {
    i = p.idx[((int64_t)b * p.T + t) * p.k + e];
    if (i < 0 || i >= p.N) return -1;
  } else {
    i = e;
  }
  return ((int64_t)b * p.N + i) * p.D;
}

// ------------------------------------------------------------------ fp32 SIMT
// One warp per (b, t, h); lane holds D/32 dims of q and o.  The sink enters as a
// row with logit sink_h and value 0 (initial state m = sink, l = 1, o = 0).
template <int DPL>  // dims per lane
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnParams p) {
  griddep_sync();
  const int h = blockIdx.x * 4 + warp_id();
  const int t = blockIdx.y, b = blockIdx.z;
  if (h >= p.H) return;
  const float* q = static_cast<const float*>(p.q) + (((int64_t)b * p.T + t) * p.H + h) * p.D;
  const float* kv = static_cast<const float*>(p.kv);
  const float* swa = static_cast<const float*>(p.swa);
  float qv[DPL], o[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) {
    qv[j] = q[lane_id() + 32 * j];
    o[j] = 0.f;
  }
  float m = p.sink[h], l = 1.f;
  const RowList rl = make_row_list(p, b, t);
  const int n = rl.n_swa + rl.n_mem;
  for (int r = 0; r < n; ++r) {
    bool sw;
    const int64_t off = row_offset(p, rl, b, t, r, &sw);
    if (off < 0) continue;
    const float* row = (sw ? swa : kv) + off;
    float rv[DPL];
    float dot = 0.f;
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      rv[j] = row[lane_id() + 32 * j];
      dot = fmaf(qv[j], rv[j], dot);
    }
#pragma unroll
    for (int off2 = 16; off2 > 0; off2 >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off2);
    const float z = dot * p.scale;
    const float mn = fmaxf(m, z);
    const float c = expf(m - mn), e = expf(z - mn);
    l = l * c + e;
#pragma unroll
    for (int j = 0; j < DPL; ++j) o[j] = fmaf(o[j], c, e * rv[j]);
    m = mn;
  }
  float* out = static_cast<float*>(p.out) + (((int64_t)b * p.T + t) * p.H + h) * p.D;
  const float inv = 1.f / l;
#pragma unroll
  for (int j = 0; j < DPL; ++j) out[lane_id() + 32 * j] = o[j] * inv;
}

// ------------------------------------------------------------------ tcgen05 bf16
template <int D>
struct AttnCfg {
  static constexpr int R = (D >= 512) ? 32 : 64;           // rows per KV tile
  static constexpr int DH = (D > 256) ? 256 : D;           // D-slice per CTA
  static constexpr int NDH = D / DH;
  static constexpr int kAtoms = D / 64;                    // 128-byte atoms per row
  static constexpr int kKVBytes = R * D * 2;
  static constexpr int kPRowBytes = R * 2;                 // 64 (SW64) or 128 (SW128)
  static constexpr int kPBytes = 128 * kPRowBytes;
  static constexpr uint32_t kPLayout = (kPRowBytes == 128) ? kLayoutSW128 : kLayoutSW64;
  static constexpr int kPSBO = 8 * kPRowBytes;
  static constexpr int kTmemCols = (DH + 2 * R) <= 256 ? 256 : 512;  // O slice + two S buffers
  static constexpr int kSCol0 = DH;                        // S buffers after O
  static constexpr int kThreads = 288;                     // 4 softmax + 4 loader + 1 MMA warps
  static constexpr int kMaxStages = 4;
  static constexpr int kMaxCtaRows = 2048;                 // index values staged per CTA (larger lists stream)
  static constexpr int kBarBytes = 256 + 4 * kMaxCtaRows;
  // heads are taken in groups of kHeadGroup per CTA (more heads: more CTAs), so
  // the Q tile is 64 rows per 64-dim atom and four KV stages always fit
  static constexpr int kHeadGroup = 64;
  static constexpr int kQBytes = kHeadGroup * D * 2;
  static constexpr int kStages = ((232448 - 1024 - kBarBytes - kQBytes - 2 * kPBytes) / kKVBytes) >= kMaxStages
                                     ? kMaxStages
                                     : (232448 - 1024 - kBarBytes - kQBytes - 2 * kPBytes) / kKVBytes;
  static constexpr int kSmem = 1024 + kQBytes + kStages * kKVBytes + 2 * kPBytes + kBarBytes;
  static __host__ __device__ int head_groups(int H) { return (H + kHeadGroup - 1) / kHeadGroup; }
};

// Byte offset of 16-byte chunk c of row r in a K-major tile with 128-byte
// swizzle, whose 64-element atoms are `rows` rows tall.
__device__ __forceinline__ uint32_t sw128_off(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Q [B*T, H, D] is loaded by TMA as D/64 boxes of {64 dims, 64 head rows}
// (head group blockIdx.y / NDH).  The M = 128 MMA operand of atom a also spans the first 64
// rows of atom a+1 (or, for the last atom, the next 8 KB of shared memory):
// finite values whose result rows (>= H) are never used.
template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                           const AttnParams p) {
  using Cfg = AttnCfg<D>;
  constexpr int R = Cfg::R, DH = Cfg::DH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int QR = Cfg::kHeadGroup;
  constexpr int NS = Cfg::kStages;
  uint8_t* q_s = smem;
  uint8_t* kv_s = q_s + Cfg::kQBytes;                       // [NS][kKVBytes]
  uint8_t* p_s = kv_s + NS * Cfg::kKVBytes;                 // [2][kPBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + 2 * Cfg::kPBytes);
  uint64_t* full = bars;        // [4] KV stage loaded (128 cp.async arrivals)
  uint64_t* empty = bars + 4;   // [4] KV stage consumed by PV
  uint64_t* sfull = bars + 8;   // [2] S ready
  uint64_t* sfree = bars + 10;  // [2] S read by softmax
  uint64_t* pfull = bars + 12;  // [2] P written
  uint64_t* pdone = bars + 14;  // [2] PV done (P buffer free, O consistent)
  uint64_t* qfull = bars + 16;
  uint64_t* odone = bars + 17;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 18);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(bars + 20);      // [4 stages][4 loader warps]
  int32_t* idx_s = reinterpret_cast<int32_t*>(bars + 32);         // [kMaxCtaRows] raw index values

  __shared__ float epi_g[Cfg::kHeadGroup];   // per-head output scale (softmax -> epilogue warps)
  __shared__ int epi_have_o;
  const int qi = blockIdx.z;                 // b * T + t
  const int b = qi / p.T, t = qi % p.T;
  const int dh = blockIdx.y % Cfg::NDH;
  const int h0 = (blockIdx.y / Cfg::NDH) * QR;  // first head of this CTA's group
  const int split = blockIdx.x;
  const int warp = warp_id();
  const int32_t* idx_row = p.sparse ? p.idx + ((int64_t)b * p.T + t) * p.k : nullptr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&full[i], 128 + 4);          // cp.async of 128 threads + a mask word per loader warp
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sfree[i], 4);
      mbar_init(&pfull[i], 4);
      mbar_init(&pdone[i], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(odone, 1);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_sync();
  const RowList rl = make_row_list(p, b, t);
  const int n_rows = rl.n_swa + rl.n_mem;
  const int n_tiles_all = (n_rows + R - 1) / R;
  const int tps = (n_tiles_all + p.nsplit - 1) / p.nsplit;
  const int j0 = split * tps;
  const int j1 = min(n_tiles_all, j0 + tps);
  const int nt = j1 > j0 ? j1 - j0 : 0;      // tiles of this CTA
  // the index value behind list row rg (only memory rows of sparse_attn read memory)
  auto fetch_raw = [&](int rg) -> int32_t {
    if (!p.sparse || rg < rl.n_swa || rg >= n_rows) return 0;
    return __ldg(idx_row + (rg - rl.n_swa));
  };
  // element offset of list row rg given its raw index; -1 if it contributes nothing;
  // SWA rows are encoded as -2 - offset
  auto row_src = [&](int rg, int32_t raw) -> int64_t {
    if (rg >= n_rows) return -1;
    if (rg < rl.n_swa) return -2 - ((int64_t)b * p.W + rl.swa_row0 + rg) * D;
    const int64_t i = p.sparse ? (int64_t)raw : (int64_t)(rg - rl.n_swa);
    if (i < 0 || i >= p.N) return -1;
    return ((int64_t)b * p.N + i) * D;
  };


  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ loaders (128 threads)
    const int lt = threadIdx.x - 128;
    if (nt > 0) {
      const __nv_bfloat16* kv = static_cast<const __nv_bfloat16*>(p.kv);
      const __nv_bfloat16* swa = static_cast<const __nv_bfloat16*>(p.swa);
      constexpr int CPR = D / 8;                 // 16-byte chunks per row
      constexpr int TPR = 128 / R;               // loader threads per row
      constexpr int CPT = CPR / TPR;             // chunks per thread and tile
      const int my_r = lt / TPR, my_c = lt % TPR;
      // stage this CTA's index values in shared memory once (coalesced), so no
      // global load sits between the tiles
      const int row0 = j0 * R, nrow = nt * R;
      const bool staged = p.sparse && nrow <= Cfg::kMaxCtaRows;
      if (staged) {
        for (int r = lt; r < nrow; r += 128) {
          const int rg = row0 + r;
          idx_s[r] = (rg >= rl.n_swa && rg < n_rows) ? __ldg(idx_row + (rg - rl.n_swa)) : 0;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      int ks = 0;
      uint32_t kph = 0;
      for (int jj = 0; jj < nt; ++jj) {
        const int rg = (j0 + jj) * R + my_r;
        const int32_t raw = staged ? idx_s[jj * R + my_r] : fetch_raw(rg);
        const int s = ks;
        const uint32_t ph = kph;
        if (++ks == NS) { ks = 0; kph ^= 1; }
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        const int64_t src_off = row_src(rg, raw);
        const __nv_bfloat16* src = src_off >= 0 ? kv + src_off : (src_off <= -2 ? swa + (-2 - src_off) : nullptr);
        uint8_t* tile = kv_s + s * Cfg::kKVBytes;
#pragma unroll 4
        for (int i = 0; i < CPT; ++i) {
          const int ch = my_c + TPR * i;
          uint8_t* dst = tile + sw128_off(my_r, ch, R);
          if (src) cp_async_16(dst, src + ch * 8);
          else st_shared_zero16(dst);                 // finite filler for rows that do not contribute
        }
        fence_proxy_async_smem();
        cp_async_arrive_noinc(&full[s]);
        // validity of this warp's rows (TPR threads per row): one word per loader warp
        const uint32_t bal = __ballot_sync(0xffffffffu, src != nullptr);
        if (lane_id() == 0) {
          uint32_t rows = 0;                          // bit j: row (warp's first row + j)
          for (int j = 0; j < 32 / TPR; ++j) rows |= ((bal >> (j * TPR)) & 1u) << j;
          mask_s[s * 4 + (lt >> 5)] = rows;
          mbar_arrive(&full[s]);
        }
      }
      cp_async_wait_group<0>();                       // none may land after the CTA has left
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ Q by TMA, then the MMA issuer
    if (elect_one() && nt > 0) {
      prefetch_tmap(&qmap);
      mbar_arrive_expect_tx(qfull, (uint32_t)Cfg::kQBytes);
      for (int a = 0; a < Cfg::kAtoms; ++a) tma_load_3d(q_s + a * QR * 128, &qmap, qfull, a * 64, h0, qi);
      const uint32_t idesc_s = make_idesc(128, R, 1, 0, 0);
      const uint32_t idesc_o = make_idesc(128, DH, 1, 0, 1);
      const uint32_t qb = smem_u32(q_s);
      bool ok = mbar_wait(qfull, 0);
      tc_fence_after();
      int ks = 0;
      uint32_t kph = 0;
      auto issue_s = [&](int jj) -> bool {
        const int sb = jj & 1;
        const uint32_t sph = (jj >> 1) & 1;
        const int s = ks;
        const uint32_t ph = kph;
        if (!mbar_wait(&full[s], ph)) return false;
        if (!mbar_wait(&sfree[sb], sph ^ 1)) return false;
        fence_proxy_async_smem();                   // cp.async data -> tensor core reads
        tc_fence_after();
        const uint32_t kb = smem_u32(kv_s + s * Cfg::kKVBytes);
        const uint32_t d = tmem + Cfg::kSCol0 + sb * R;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int atom = kk >> 2, inner = (kk & 3) * 32;
          const uint64_t ad = smem_desc(qb + atom * QR * 128 + inner, 16, 1024, kLayoutSW128);
          const uint64_t bd = smem_desc(kb + atom * R * 128 + inner, 16, 1024, kLayoutSW128);
          mma_bf16(d, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sfull[sb]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int jj = 0; ok && jj < nt; ++jj) {
        const int s = ks;                           // KV stage of tile jj
        if (++ks == NS) { ks = 0; kph ^= 1; }
        if (jj + 1 < nt && !issue_s(jj + 1)) { ok = false; break; }
        const int sb = jj & 1;
        if (!mbar_wait(&pfull[sb], (jj >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pb = smem_u32(p_s + sb * Cfg::kPBytes);
        const uint32_t vb = smem_u32(kv_s + s * Cfg::kKVBytes) + dh * (DH / 64) * R * 128;
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint64_t ad = smem_desc(pb + kk * 32, 16, Cfg::kPSBO, Cfg::kPLayout);
          const uint64_t bd = smem_desc(vb + kk * 2048, R * 128, 1024, kLayoutSW128);
          mma_bf16(tmem, ad, bd, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&pdone[sb]);
        mma_commit(&empty[s]);
      }
      mma_commit(odone);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue (warps 0..3)
    const int h = threadIdx.x;                 // TMEM lane = head row
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool head_ok = h < QR && h0 + h < p.H;    // rows >= QR are the operand's filler
    const float sinkL = head_ok ? p.sink[h0 + h] * kLog2e : 0.f;
    const float zs = p.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // validity of the tile's rows: lane r (and r + 32) checks row r of the tile; the
    // index value is fetched one tile ahead and a warp ballot gives every thread the mask
    int ks = 0;
    uint32_t kph = 0;
    constexpr int RPW = R / 4;                 // tile rows covered by one loader warp
    for (int jj = 0; jj < nt; ++jj) {
      const int sb = jj & 1;
      const uint32_t ph = (jj >> 1) & 1;
      const int s = ks;
      const uint32_t kp = kph;
      if (++ks == NS) { ks = 0; kph ^= 1; }
      // the loaders' row-validity words for this tile (published with full[s])
      if (!mbar_wait(&full[s], kp)) { ok = false; break; }
      uint64_t valid = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) valid |= (uint64_t)(mask_s[s * 4 + w] & ((1ull << RPW) - 1)) << (w * RPW);
      if (!mbar_wait(&sfull[sb], ph)) { ok = false; break; }
      tc_fence_after();
      float z[R];
      tmem_ld32(tmem + lane_base + Cfg::kSCol0 + sb * R, z);
      if constexpr (R == 64) tmem_ld32(tmem + lane_base + Cfg::kSCol0 + sb * R + 32, z + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&sfree[sb]);
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < R; ++c) {
        z[c] = ((valid >> c) & 1) ? z[c] * zs : -INFINITY;
        mt = fmaxf(mt, z[c]);
      }
      // P buffer sb is free once PV of tile jj-2 completed
      if (!mbar_wait(&pdone[sb], ph ^ 1)) { ok = false; break; }
      if (mt > m_used + 8.f) {
        const float m_new = mt;
        if (m_used != -INFINITY && jj > 0) {
          // O must be consistent: PV of tile jj-1 completed
          if (!mbar_wait(&pdone[(jj - 1) & 1], ((jj - 1) >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const float f = ex2_approx(m_used - m_new);
          for (int c0 = 0; c0 < DH; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= f;
            tmem_st32(tmem + lane_base + c0, o);
          }
          tmem_wait_st();
          l *= f;
        }
        m_used = m_new;
      }
      // p = 2^(z - m); rows with no valid column so far keep m = -inf and p = 0
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      float ps0 = 0.f, ps1 = 0.f;
      uint32_t packed[R / 2];
#pragma unroll
      for (int c = 0; c < R; c += 2) {
        const float p0 = ex2_approx(z[c] - mref);        // z = -inf (masked) -> 0
        const float p1 = ex2_approx(z[c + 1] - mref);
        ps0 += p0;
        ps1 += p1;
        __nv_bfloat162 v = __floats2bfloat162_rn(p0, p1);
        packed[c / 2] = *reinterpret_cast<uint32_t*>(&v);
      }
      l += ps0 + ps1;
      uint8_t* prow = p_s + sb * Cfg::kPBytes + h * Cfg::kPRowBytes;
#pragma unroll
      for (int c = 0; c < R / 8; ++c) {
        const int phys = (R == 64) ? (c ^ (h & 7)) : (c ^ ((h >> 1) & 3));
        *reinterpret_cast<uint4*>(prow + phys * 16) =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&pfull[sb]);
    }
    // ---- hand-over to the epilogue: per-head output scale and whether O is valid
    const bool have_o = ok && nt > 0 && mbar_wait(odone, 0);
    float g = 1.f;
    if (p.nsplit == 1) {
      const float M = fmaxf(m_used, sinkL);
      const float fo = (m_used == -INFINITY) ? 0.f : exp2f(m_used - M);
      const float den = l * fo + exp2f(sinkL - M);
      g = fo / den;
    }
    if (h < QR) epi_g[h] = g;
    if (h == 0) epi_have_o = have_o ? 1 : 0;
    if (p.nsplit > 1 && head_ok && dh == 0) {
      float* ml = p.ws_ml + (((int64_t)split * p.B * p.T + qi) * p.H + h0 + h) * 2;
      ml[0] = have_o ? m_used : -INFINITY;
      ml[1] = have_o ? l : 0.f;
    }
  }

  // ------------------------------------------------------------ epilogue
  // TMEM lanes 0..63 hold this CTA's heads; they are readable by warps 0, 1 and
  // (same lane quarters) 4, 5, which split the O columns in two halves.  Each
  // warp moves 32-column chunks out of TMEM and transposes them through shared
  // memory (the KV stages are idle now) so that a store instruction writes four
  // full 128-byte row segments.
  if (warp == 0 || warp == 1 || warp == 4 || warp == 5) {
    asm volatile("bar.sync 2, 128;" ::: "memory");   // epi_g / epi_have_o written by warps 0, 1
    tc_fence_after();
    const bool have_o = epi_have_o != 0;
    const int rw = warp & 3;                           // lane quarter: head rows 32 * rw ..
    const int hw0 = rw * 32;
    const uint32_t lane_q = (uint32_t)(rw * 32) << 16;
    const int c_begin = warp < 4 ? 0 : DH / 2, c_end = warp < 4 ? DH / 2 : DH;
    float* stage = reinterpret_cast<float*>(kv_s) + warp * 32 * 36;
    const float g = epi_g[hw0 + (int)lane_id()];
    const int sub = (int)lane_id() >> 3, q4 = ((int)lane_id() & 7) * 4;   // row within a group of 4, column
    __nv_bfloat16* obase = static_cast<__nv_bfloat16*>(p.out) + ((int64_t)qi * p.H + h0 + hw0) * D + dh * DH;
    float* wbase = p.ws_o + (((int64_t)split * p.B * p.T + qi) * p.H + h0 + hw0) * D + dh * DH;
    for (int c0 = c_begin; c0 < c_end; c0 += 32) {
      float o[32];
      if (have_o) {
        tmem_ld32(tmem + lane_q + c0, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0.f;
      }
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 32; c += 4)
        *reinterpret_cast<float4*>(stage + lane_id() * 36 + c) =
            make_float4(o[c] * g, o[c + 1] * g, o[c + 2] * g, o[c + 3] * g);
      __syncwarp();
#pragma unroll
      for (int r4 = 0; r4 < 32; r4 += 4) {
        const int r = r4 + sub;
        if (h0 + hw0 + r < p.H) {
          const float4 v = *reinterpret_cast<const float4*>(stage + r * 36 + q4);
          if (p.nsplit == 1) {
            __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), bb = __floats2bfloat162_rn(v.z, v.w);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&a);
            u.y = *reinterpret_cast<uint32_t*>(&bb);
            *reinterpret_cast<uint2*>(obase + (int64_t)r * D + c0 + q4) = u;
          } else {
            *reinterpret_cast<float4*>(wbase + (int64_t)r * D + c0 + q4) = v;
          }
        }
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// Merge split partials with the sink: M = max(sink, m_s); den = e^(sink-M) +
// sum_s l_s e^(m_s-M); o = sum_s O_s e^(m_s-M) / den  (log2 domain).  One
// thread per (query, head, 8 dims).
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p) {
  griddep_sync();
  const uint32_t gpr = (uint32_t)(p.D / 8);  // 32-bit index math: B*T*H*D/8 < 2^31 (host-checked)
  const uint32_t groups = (uint32_t)(p.B * p.T * p.H) * gpr;
  const uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= groups) return;
  const int d0 = (int)(g % gpr) * 8;
  const uint32_t qh = g / gpr;               // (b*T + t) * H + h
  const int h = (int)(qh % (uint32_t)p.H);
  const float sinkL = p.sink[h] * kLog2e;
  const int64_t stride_ml = (int64_t)p.B * p.T * p.H * 2;
  const int64_t stride_o = (int64_t)p.B * p.T * p.H * p.D;
  float M = sinkL;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, p.ws_ml[s * stride_ml + qh * 2]);
  float den = exp2f(sinkL - M);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float ms = p.ws_ml[s * stride_ml + qh * 2];
    if (ms == -INFINITY) continue;
    const float f = exp2f(ms - M);
    den = fmaf(p.ws_ml[s * stride_ml + qh * 2 + 1], f, den);
    const float4* src = reinterpret_cast<const float4*>(p.ws_o + s * stride_o + qh * p.D + d0);
    const float4 a = src[0], c = src[1];
    acc[0] = fmaf(a.x, f, acc[0]); acc[1] = fmaf(a.y, f, acc[1]);
    acc[2] = fmaf(a.z, f, acc[2]); acc[3] = fmaf(a.w, f, acc[3]);
    acc[4] = fmaf(c.x, f, acc[4]); acc[5] = fmaf(c.y, f, acc[5]);
    acc[6] = fmaf(c.z, f, acc[6]); acc[7] = fmaf(c.w, f, acc[7]);
  }
  const float inv = 1.f / den;
  uint4 u;
  __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) hv[e] = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + qh * p.D + d0) = u;
}

}  // namespace csa
