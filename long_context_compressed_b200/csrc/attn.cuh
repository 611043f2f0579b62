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
// attn_tc_kernel (bf16): one CTA per (split, D-slice x head group of 64, query).
// The query block (64 heads, padded to the M = 128 operand, all D dims) stays in
// shared memory;
// KV rows are gathered with 16-byte cp.async into 128-byte-swizzled K-major
// tiles of R rows; S = Q K^T (tcgen05, fp32 in TMEM, double buffered); four
// softmax warps (one head per thread) run the online softmax in the log2
// domain, writing P (bf16) back into TMEM over the tile's S columns; O += P V
// (tcgen05 with the A operand read from TMEM; the same KV
// tile read as an MN-major operand, restricted to this CTA's D-slice of width
// DH <= 256) accumulates in TMEM.  O is rescaled only when a tile's maximum
// exceeds the running reference by more than 2^8, so exponentials stay <= 256.
// With several splits (<= 16) the split CTAs of one (query, D-slice, head group)
// are one thread-block cluster: each parks its unnormalised O (bf16) and (m, l) in its
// own shared memory, and after a cluster barrier every CTA merges a slice of the
// heads, sink included, reading the others' shared memory (no partials in HBM,
// no second launch).
//
// attn_f32_kernel: fp32 SIMT (one warp per head), exact online softmax.
#pragma once
#include <cuda_bf16.h>
#include "kv8.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace csa {

constexpr int kSwaWindow = 128;
constexpr int kMaxSplits = 16;   // CTAs of one query's cluster (sizes above 8 are non-portable)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnParams {
  const void* q;          // [B, T, H, D]
  const void* kv;         // [B, N, D]
  const void* swa;        // [B, W, D]
  const int64_t* swa_pos0;  // [B]
  const int64_t* q_pos;   // [B, T]
  const float* sink;      // [H]
  const int32_t* idx;     // [B, T, k] (sparse) or null (hca)
  void* out;              // [B, T, H, D]
  float scale;
  int B, T, H, D, W, k, ratio, nsplit;
  int has_kvmap, has_swamap;   // tensor maps of kv [B, N, D] and swa_kv [B, W, D] were built
  int sparse;             // 1: memory rows from idx (sparse_attn); 0: dense prefix (hca_attn)
  float* ml;              // [B, T, H, 2] or null: partial mode (no sink; write (m, l) per head)
  int64_t N;
  double rope_theta;      // > 0: partial RoPE around the attention (rope.cuh); 0: none
  RopeFreqs rope_freq;    // theta^(-2i/64), i < 32 (when rope_theta > 0)
  void* part_o;           // attn_t_kernel with splits: bf16 [B*T*groups][nsplit][64][D] unnormalised O
  void* part_ml;          // ... and float2 [B*T*groups][nsplit][64] (m (log2), l) of each split
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
  // partial RoPE: dims D-64.. of q turned at the query's position (pairs in adjacent lanes)
  const int64_t qpos = p.q_pos[(int64_t)b * p.T + t];
  const bool rope = p.rope_theta > 0.0;
  float2 rcs[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) {
    const int d = lane_id() + 32 * j;
    rcs[j] = make_float2(1.f, 0.f);
    if (rope && d >= p.D - kRopeDims) {
      rcs[j] = rope_cs(qpos, p.rope_freq.f[(d - (p.D - kRopeDims)) >> 1], false);
      const float other = __shfl_xor_sync(0xffffffffu, qv[j], 1);
      const float2 y = (d & 1) ? rope_turn(other, qv[j], rcs[j]) : rope_turn(qv[j], other, rcs[j]);
      qv[j] = (d & 1) ? y.y : y.x;                    // (d >= D - 64 holds for the whole warp)
    }
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
  for (int j = 0; j < DPL; ++j) {
    float v = o[j] * inv;
    const int d = lane_id() + 32 * j;
    if (rope) {                                        // inverse RoPE of the output at the query's position
      const float other = __shfl_xor_sync(0xffffffffu, v, 1);
      if (d >= p.D - kRopeDims) {
        const float2 cs = make_float2(rcs[j].x, -rcs[j].y);
        const float2 y = (d & 1) ? rope_turn(other, v, cs) : rope_turn(v, other, cs);
        v = (d & 1) ? y.y : y.x;
      }
    }
    out[d] = v;
  }
}

// ------------------------------------------------------------------ tcgen05 bf16
// RT: rows per KV tile.  One S = Q K^T MMA instruction (N = RT rows) costs about the same
// for N = 32 and N = 64 (~46 cycles), so a 32-row tile of D = 512 spends ~0.75 us issuing
// its 32 S instructions; 64-row tiles would halve that per row but leave two stages in
// shared memory at D = 512, which measured slower.
template <int D, int RT = (D >= 512 ? 32 : 64)>
struct AttnCfg {
  static constexpr int R = RT;                             // rows per KV tile
  static constexpr int DH = (D > 256) ? 256 : D;           // D-slice per CTA
  static constexpr int NDH = D / DH;
  static constexpr int kAtoms = D / 64;                    // 128-byte atoms per row
  static constexpr int kKVBytes = R * D * 2;
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
  static constexpr int kStages = ((232448 - 1024 - kBarBytes - kQBytes) / kKVBytes) >= kMaxStages
                                     ? kMaxStages
                                     : (232448 - 1024 - kBarBytes - kQBytes) / kKVBytes;
  static constexpr int kSmem = 1024 + kQBytes + kStages * kKVBytes + kBarBytes;
  static __host__ __device__ int head_groups(int H) { return (H + kHeadGroup - 1) / kHeadGroup; }
};

// KV8 launches 13 warps: warps 9..12 are the converters.
__host__ __device__ constexpr int attn_threads(bool kv8) { return kv8 ? 416 : 288; }

// A zero entry: the source of the staged bytes of KV8 rows that contribute nothing.
__device__ __align__(16) uint8_t g_kv8_zero_entry[kKv8Bytes];

// Byte offset of 16-byte chunk c of row r in a K-major tile with 128-byte
// swizzle, whose 64-element atoms are `rows` rows tall.
__device__ __forceinline__ uint32_t sw128_off(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Q [B*T, H, D] is loaded by TMA as D/64 boxes of {64 dims, 64 head rows}
// (head group blockIdx.y / NDH).  The M = 128 MMA operand of atom a also spans the first 64
// rows of atom a+1 (or, for the last atom, the next 8 KB of shared memory):
// finite values whose result rows (>= H) are never used.
// KV8: memory rows are csa_quantize_kv8 entries (FP8 dims + BF16 RoPE dims, D = 512).
// The loader warps stage each tile's 608-byte entries at the tail of its buffer (one
// bulk copy for a contiguous tile of hca_attn, cp.async per entry otherwise; rows that
// contribute nothing copy a zero entry), counted on the stage's `staged` barrier; four
// converter warps (9..12) then rewrite the tile in place as the bf16 swizzled tile
// (exact: code * 2^e is a bf16 value) and arrive on `full`.  The memory rows start at a
// tile boundary of the row list (the SWA rows are padded with masked rows), so a tile
// is all SWA or all memory.
template <int D, bool KV8, int RT>
__global__ void __launch_bounds__(attn_threads(KV8), 1) attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                           const __grid_constant__ CUtensorMap kvmap,
                                                                           const __grid_constant__ CUtensorMap swamap,
                                                                           const AttnParams p) {
  using Cfg = AttnCfg<D, RT>;
  constexpr int R = Cfg::R, DH = Cfg::DH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int QR = Cfg::kHeadGroup;
  constexpr int NS = Cfg::kStages;
  uint8_t* q_s = smem;
  uint8_t* kv_s = q_s + Cfg::kQBytes;                       // [NS][kKVBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(kv_s + NS * Cfg::kKVBytes);
  uint64_t* full = bars;        // [4] KV stage loaded (128 cp.async arrivals)
  uint64_t* empty = bars + 4;   // [4] KV stage consumed by PV
  uint64_t* sfull = bars + 8;   // [2] S ready
  uint64_t* sfree = bars + 10;  // [2] (unused: S buffer reuse waits for the PV that read its P)
  uint64_t* pfull = bars + 12;  // [2] P written
  uint64_t* pdone = bars + 14;  // [2] PV done (P buffer free, O consistent)
  uint64_t* qfull = bars + 16;
  uint64_t* odone = bars + 17;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 18);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(bars + 20);      // [4 stages][4 loader warps]
  uint64_t* staged = bars + 28;  // [4] KV8: a memory tile's entries are in its buffer's tail
  int32_t* idx_s = reinterpret_cast<int32_t*>(bars + 32);         // [kMaxCtaRows] raw index values

  __shared__ float epi_g[Cfg::kHeadGroup];   // per-head output scale (softmax -> epilogue warps)
  __shared__ int epi_have_o;
  // split partials (nsplit > 1: the CTAs of one query / D-slice / head group form a
  // cluster and merge through distributed shared memory)
  __shared__ float cl_m[Cfg::kHeadGroup], cl_l[Cfg::kHeadGroup];   // running max (log2) and sum
  __shared__ float cl_w[Cfg::kHeadGroup][kMaxSplits];              // merge weights of the splits
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
      if (KV8) mbar_init(&staged[i], 128);   // cp.async arrivals of the 128 loader threads
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
  const int mem0 = KV8 ? (rl.n_swa + R - 1) / R * R : rl.n_swa;   // list row of the first memory row
  const int n_rows = mem0 + rl.n_mem;
  const int n_tiles_all = (n_rows + R - 1) / R;
  // balanced tile ranges: the splits' tile counts differ by at most one
  const int j0 = (int)((int64_t)split * n_tiles_all / p.nsplit);
  const int j1 = (int)((int64_t)(split + 1) * n_tiles_all / p.nsplit);
  const int nt = j1 > j0 ? j1 - j0 : 0;      // tiles of this CTA
  // the index value behind list row rg (only memory rows of sparse_attn read memory)
  auto fetch_raw = [&](int rg) -> int32_t {
    if (!p.sparse || rg < mem0 || rg >= n_rows) return 0;
    return __ldg(idx_row + (rg - mem0));
  };
  // element offset of list row rg given its raw index; -1 if it contributes nothing;
  // SWA rows are encoded as -2 - offset
  // (KV8: offset in entries, i.e. the memory row's entry number)
  auto row_src = [&](int rg, int32_t raw) -> int64_t {
    if (rg >= n_rows) return -1;
    if (rg < rl.n_swa) return -2 - ((int64_t)b * p.W + rl.swa_row0 + rg) * D;
    if (rg < mem0) return -1;                        // padding between the SWA and memory rows
    const int64_t i = p.sparse ? (int64_t)raw : (int64_t)(rg - mem0);
    if (i < 0 || i >= p.N) return -1;
    return KV8 ? (int64_t)b * p.N + i : ((int64_t)b * p.N + i) * D;
  };


  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ loaders (128 threads)
    const int lt = threadIdx.x - 128;
    if (lt == 0) {
      if (p.has_kvmap) prefetch_tmap(&kvmap);
      if (p.has_swamap) prefetch_tmap(&swamap);
    }
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
      const bool staged_idx = p.sparse && nrow <= Cfg::kMaxCtaRows;
      if (staged_idx) {
        for (int r = lt; r < nrow; r += 128) {
          const int rg = row0 + r;
          idx_s[r] = (rg >= mem0 && rg < n_rows) ? __ldg(idx_row + (rg - mem0)) : 0;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      if constexpr (!KV8) {
        int ks = 0;
        uint32_t kph = 0;
        for (int jj = 0; jj < nt; ++jj) {
          const int rg0 = (j0 + jj) * R;
          const int rg = rg0 + my_r;
          const int32_t raw = staged_idx ? idx_s[jj * R + my_r] : fetch_raw(rg);
          const int s = ks;
          const uint32_t ph = kph;
          if (++ks == NS) { ks = 0; kph ^= 1; }
          if (!mbar_wait(&empty[s], ph ^ 1)) break;
          uint8_t* tile = kv_s + s * Cfg::kKVBytes;
          // R consecutive rows of one buffer (SWA rows, or hca_attn's dense memory rows):
          // one TMA box per 64-dim atom, same 128-byte-swizzled layout as the gather
          const bool swa_tile = p.has_swamap && rg0 + R <= rl.n_swa;
          const bool mem_tile = !KV8 && p.has_kvmap && !p.sparse && rg0 >= mem0 && rg0 + R <= n_rows;
          const __nv_bfloat16* src = nullptr;
          if (swa_tile || mem_tile) {
            src = kv;                                   // every row valid
            if (lt == 0) {
              // one box of {64 dims, R rows, all 64-dim atoms}: the atoms land R rows apart,
              // the K-major layout the MMA reads
              mbar_arrive_expect_tx(&full[s], (uint32_t)Cfg::kKVBytes);
              const int y = swa_tile ? (int)rl.swa_row0 + rg0 : rg0 - mem0;
              tma_load_4d(tile, swa_tile ? &swamap : &kvmap, &full[s], 0, y, 0, b);
            } else {
              mbar_arrive(&full[s]);
            }
          } else {
            const int64_t src_off = row_src(rg, raw);
            src = src_off >= 0 ? kv + src_off : (src_off <= -2 ? swa + (-2 - src_off) : nullptr);
#pragma unroll 4
            for (int i = 0; i < CPT; ++i) {
              const int ch = my_c + TPR * i;
              uint8_t* dst = tile + sw128_off(my_r, ch, R);
              if (src) cp_async_16(dst, src + ch * 8);
              else st_shared_zero16(dst);               // finite filler for rows that do not contribute
            }
            fence_proxy_async_smem();
            cp_async_arrive_noinc(&full[s]);
          }
          // validity of this warp's rows (TPR threads per row): one word per loader warp
          const uint32_t bal = __ballot_sync(0xffffffffu, src != nullptr);
          if (lane_id() == 0) {
            uint32_t rows = 0;                          // bit j: row (warp's first row + j)
            for (int j = 0; j < 32 / TPR; ++j) rows |= ((bal >> (j * TPR)) & 1u) << j;
            mask_s[s * 4 + (lt >> 5)] = rows;
            mbar_arrive(&full[s]);
          }
        }
      } else {
        // ---- memory rows as KV8 entries, staged at the tail of the tile's buffer and
        // counted on staged[s]; the converter warps arrive on full[s] for those tiles.
        // SWA rows (by TMA, or copied in place) and the padding rows arrive as before.
        static_assert(D == kKv8Dims && (TPR == 2 || TPR == 4), "KV8 entries: D = 512, 32- or 64-row tiles");
        constexpr int kEC = kKv8Bytes / 16;                 // 16-byte chunks per entry
        constexpr int kStg = Cfg::kKVBytes - R * kKv8Bytes; // staged entries at the buffer's tail
        const uint8_t* kv8 = static_cast<const uint8_t*>(p.kv);
        int ks = 0;
        uint32_t kph = 0;
        for (int jj = 0; jj < nt; ++jj) {
          const int rg0 = (j0 + jj) * R;
          const int rg = rg0 + my_r;
          const int32_t raw = staged_idx ? idx_s[jj * R + my_r] : fetch_raw(rg);
          const int s = ks;
          const uint32_t ph = kph;
          if (++ks == NS) { ks = 0; kph ^= 1; }
          if (!mbar_wait(&empty[s], ph ^ 1)) break;
          uint8_t* tile = kv_s + s * Cfg::kKVBytes;
          const bool swa_tile = p.has_swamap && rg0 + R <= rl.n_swa;
          bool valid = true;
          if (swa_tile) {
            if (lt == 0) {
              mbar_arrive_expect_tx(&full[s], (uint32_t)Cfg::kKVBytes);
              tma_load_4d(tile, &swamap, &full[s], 0, (int)rl.swa_row0 + rg0, 0, b);
            } else {
              mbar_arrive(&full[s]);
            }
          } else if (rg0 < mem0) {
            const int64_t so = row_src(rg, raw);              // SWA row (-2 - offset) or padding (-1)
            const __nv_bfloat16* src = so <= -2 ? swa + (-2 - so) : nullptr;
            valid = src != nullptr;
#pragma unroll 4
            for (int i = 0; i < CPT; ++i) {
              const int ch = my_c + TPR * i;
              uint8_t* dst = tile + sw128_off(my_r, ch, R);
              if (src) cp_async_16(dst, src + ch * 8);
              else st_shared_zero16(dst);
            }
            fence_proxy_async_smem();
            cp_async_arrive_noinc(&full[s]);
          } else if (!p.sparse && rg0 + R <= n_rows) {
            // hca_attn: R consecutive entries, one bulk copy
            if (lt == 0) {
              mbar_arrive_expect_tx(&staged[s], (uint32_t)(R * kKv8Bytes));
              bulk_load(tile + kStg, kv8 + ((int64_t)b * p.N + (rg0 - mem0)) * kKv8Bytes, R * kKv8Bytes, &staged[s]);
            } else {
              mbar_arrive(&staged[s]);
            }
          } else {
            const int64_t so = row_src(rg, raw);              // entry number, or -1
            valid = so >= 0;
            const uint8_t* e = valid ? kv8 + so * kKv8Bytes : g_kv8_zero_entry;
            uint8_t* dst = tile + kStg + my_r * kKv8Bytes;
            for (int c = my_c; c < kEC; c += TPR) cp_async_16(dst + 16 * c, e + 16 * c);
            cp_async_arrive_noinc(&staged[s]);
          }
          const uint32_t bal = __ballot_sync(0xffffffffu, valid);
          if (lane_id() == 0) {
            uint32_t rows = 0;
            for (int j = 0; j < 32 / TPR; ++j) rows |= ((bal >> (j * TPR)) & 1u) << j;
            mask_s[s * 4 + (lt >> 5)] = rows;
            mbar_arrive(&full[s]);
          }
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
        // S buffer sb holds P of tile jj-2 until that tile's PV has run
        if (!mbar_wait(&pdone[sb], sph ^ 1)) return false;
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
        // P (bf16, two per column) sits in TMEM over the S columns of its tile
        const uint32_t pt = tmem + Cfg::kSCol0 + sb * R;
        const uint32_t vb = smem_u32(kv_s + s * Cfg::kKVBytes) + dh * (DH / 64) * R * 128;
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint64_t bd = smem_desc(vb + kk * 2048, R * 128, 1024, kLayoutSW128);
          mma_bf16_ts(tmem, pt + kk * 8, bd, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&pdone[sb]);
        mma_commit(&empty[s]);
      }
      mma_commit(odone);
    }
  } else if (KV8 && warp >= 9) {
    // ------------------------------------------------------------ converters (warps 9..12, KV8)
    // A memory tile's staged entries -> the bf16 swizzled tile, in place: every thread
    // reads its row's share of the entry, the 128 converters meet, then write.
    if constexpr (KV8) {
      constexpr int TPR = 128 / R;
      constexpr int kStg = Cfg::kKVBytes - R * kKv8Bytes;
      const int lc = (int)threadIdx.x - 288;
      const int my_r = lc / TPR, my_c = lc % TPR;
      uint32_t sph = 0;                                     // bit s: parity of staged[s]'s next phase
      int ks = 0;
      for (int jj = 0; jj < nt; ++jj) {
        const int s = ks;
        if (++ks == NS) ks = 0;
        if ((j0 + jj) * R < mem0) continue;                 // SWA / padding tile
        const bool got = mbar_wait(&staged[s], (sph >> s) & 1u);
        sph ^= 1u << s;
        if (!bar_and_128<3>(got)) break;                    // leave together (named barrier below)
        uint8_t* tile = kv_s + s * Cfg::kKVBytes;
        const uint8_t* stg = tile + kStg + my_r * kKv8Bytes;
        // this thread's share of the row: FP8 chunks q = my_c + TPR * i (16 dims each,
        // block q / 4) and RoPE chunks my_c + TPR * i (8 dims each)
        constexpr int NQ = (kKv8Fp8Dims / 16) / TPR, NRP = 8 / TPR;
        uint4 v[NQ], rp[NRP];
        float sc[7];
#pragma unroll
        for (int i = 0; i < NQ; ++i) v[i] = *reinterpret_cast<const uint4*>(stg + 16 * (my_c + TPR * i));
#pragma unroll
        for (int i = 0; i < NRP; ++i)
          rp[i] = *reinterpret_cast<const uint4*>(stg + kKv8Fp8Dims + 16 * (my_c + TPR * i));
#pragma unroll
        for (int i = 0; i < 7; ++i) sc[i] = *reinterpret_cast<const float*>(stg + kKv8ScaleOff + 4 * i);
        asm volatile("bar.sync 3, 128;" ::: "memory");     // staged bytes read: the tile may be written
#pragma unroll
        for (int i = 0; i < NQ; ++i) {                      // 16 FP8 dims -> two bf16 chunks
          const int q = my_c + TPR * i;
          float c;
          if constexpr (TPR == 4) c = sc[i];                // q / 4 == i: a static register index
          else c = sc[q >> 2];
          const uint4 o0 = make_uint4(e4m3x2_to_bf16x2(v[i].x, c), e4m3x2_to_bf16x2(v[i].x >> 16, c),
                                      e4m3x2_to_bf16x2(v[i].y, c), e4m3x2_to_bf16x2(v[i].y >> 16, c));
          const uint4 o1 = make_uint4(e4m3x2_to_bf16x2(v[i].z, c), e4m3x2_to_bf16x2(v[i].z >> 16, c),
                                      e4m3x2_to_bf16x2(v[i].w, c), e4m3x2_to_bf16x2(v[i].w >> 16, c));
          *reinterpret_cast<uint4*>(tile + sw128_off(my_r, 2 * q, R)) = o0;
          *reinterpret_cast<uint4*>(tile + sw128_off(my_r, 2 * q + 1, R)) = o1;
        }
#pragma unroll
        for (int i = 0; i < NRP; ++i)                       // RoPE dims: bf16 as stored
          *reinterpret_cast<uint4*>(tile + sw128_off(my_r, kKv8Fp8Dims / 8 + my_c + TPR * i, R)) = rp[i];
        fence_proxy_async_smem();
        mbar_arrive(&full[s]);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax / epilogue (warps 0..3)
    const int h = threadIdx.x;                 // TMEM lane = head row
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool head_ok = h < QR && h0 + h < p.H;    // rows >= QR are the operand's filler
    // (partial mode: no sink, i.e. a sink logit of -inf)
    const float sinkL = !head_ok ? 0.f : (p.ml ? -INFINITY : p.sink[h0 + h] * kLog2e);
    const float zs = p.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // validity of the tile's rows: lane r (and r + 32) checks row r of the tile; the
    // index value is fetched one tile ahead and a warp ballot gives every thread the mask
    int ks = 0;
    uint32_t kph = 0;
    constexpr int RPW = R / 4;                 // tile rows covered by one loader warp
    // warps 2, 3 own the operand's filler rows (64..127): no softmax for them, only the
    // hand-overs, in the same order as the real rows so every barrier phase stays exact
    // (their P rows stay as they are: O rows 64..127 are never read)
    const int jj_end = warp < 2 ? nt : 0;
    for (int jj = 0; ok && jj < nt && warp >= 2; ++jj) {
      const int sb = jj & 1;
      const uint32_t ph = (jj >> 1) & 1;
      if (!mbar_wait(&sfull[sb], ph)) { ok = false; break; }
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&pfull[sb]);
    }
    for (int jj = 0; jj < jj_end; ++jj) {
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
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < R; ++c) {
        z[c] = ((valid >> c) & 1) ? z[c] * zs : -INFINITY;
        mt = fmaxf(mt, z[c]);
      }
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
      // P over this tile's S columns (the PV operand A is read from TMEM)
      const uint32_t pt = tmem + lane_base + Cfg::kSCol0 + sb * R;
      if constexpr (R == 32) {
        tmem_st16u(pt, packed);
      } else {
        tmem_st16u(pt, packed);
        tmem_st16u(pt + 16, packed + 16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&pfull[sb]);
    }
    // ---- hand-over to the epilogue: per-head output scale and whether O is valid
    const bool have_o = ok && nt > 0 && mbar_wait(odone, 0);
    float g = 1.f;
    if (p.nsplit == 1) {
      if (p.ml) {
        // partial mode: O / l and (m, l) in natural-log units, l = sum_j e^(z_j - m)
        g = (have_o && l > 0.f) ? 1.f / l : 0.f;
        if (head_ok) {
          float2* mlh = reinterpret_cast<float2*>(p.ml) + ((int64_t)qi * p.H + h0 + h);
          *mlh = (have_o && l > 0.f) ? make_float2(m_used * kLn2, l) : make_float2(-INFINITY, 0.f);
        }
      } else {
        const float M = fmaxf(m_used, sinkL);
        const float fo = (m_used == -INFINITY) ? 0.f : exp2f(m_used - M);
        const float den = l * fo + exp2f(sinkL - M);
        g = fo / den;
      }
    }
    if (h < QR) epi_g[h] = g;
    if (h == 0) epi_have_o = have_o ? 1 : 0;
    if (h < QR) {
      cl_m[h] = have_o ? m_used : -INFINITY;
      cl_l[h] = have_o ? l : 0.f;
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
    float* obuf = reinterpret_cast<float*>(kv_s);   // clustered: raw O [64 heads][DH], float4 slots ^ (row & 7)
    for (int c0 = c_begin; c0 < c_end; c0 += 32) {
      float o[32];
      if (have_o) {
        tmem_ld32(tmem + lane_q + c0, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0.f;
      }
      if (p.nsplit > 1) {
        // raw O as bf16, 8 values per 16-byte slot, slots ^ (row & 7) within each 128 bytes
        const int row = hw0 + (int)lane_id();
        uint8_t* orow = reinterpret_cast<uint8_t*>(obuf) + row * DH * 2;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int f = (c0 >> 3) + c;
          const int phys = (f & ~7) | ((f ^ row) & 7);
          uint4 u;
          __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) hv[e] = __floats2bfloat162_rn(o[8 * c + 2 * e], o[8 * c + 2 * e + 1]);
          *reinterpret_cast<uint4*>(orow + phys * 16) = u;
        }
        continue;
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
          __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), bb = __floats2bfloat162_rn(v.z, v.w);
          uint2 u;
          u.x = *reinterpret_cast<uint32_t*>(&a);
          u.y = *reinterpret_cast<uint32_t*>(&bb);
          *reinterpret_cast<uint2*>(obase + (int64_t)r * D + c0 + q4) = u;
        }
      }
      __syncwarp();
    }
  }

  if (p.nsplit > 1) {
    // ------------------------------------------------------------ merge of the splits
    // CTA `rank` of the cluster finishes heads [rank*64/ns, (rank+1)*64/ns): with
    // M = max(sink, m_j), den = 2^(sink - M) + sum_j l_j 2^(m_j - M), the output is
    // sum_j 2^(m_j - M) O_j / den, O_j read from CTA j's shared memory.
    const int ns = p.nsplit;
    const uint32_t rank = cluster_ctarank();
    const int hb = (int)rank * QR / ns, he = ((int)rank + 1) * QR / ns;
    cluster_sync();                                   // every split's O and (m, l) are in place
    for (int hl = threadIdx.x; hl < he - hb; hl += blockDim.x) {
      const int hh = hb + hl;
      float mj[kMaxSplits], lj[kMaxSplits];
      const float sinkL = (h0 + hh >= p.H) ? 0.f : (p.ml ? -INFINITY : p.sink[h0 + hh] * kLog2e);
      float M = sinkL;
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) {
        mj[j] = j < ns ? ld_cluster_f32(cluster_map(smem_u32(&cl_m[hh]), (uint32_t)j)) : -INFINITY;
        lj[j] = j < ns ? ld_cluster_f32(cluster_map(smem_u32(&cl_l[hh]), (uint32_t)j)) : 0.f;
        M = fmaxf(M, mj[j]);
      }
      const bool any = M > -INFINITY;                 // (partial mode: some split has rows)
      float den = any ? ex2_approx(sinkL - M) : 0.f;
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) {
        mj[j] = any ? ex2_approx(mj[j] - M) : 0.f;    // m = -inf (no rows) -> weight 0
        den = fmaf(lj[j], mj[j], den);
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      if (p.ml && h0 + hh < p.H)
        reinterpret_cast<float2*>(p.ml)[(int64_t)qi * p.H + h0 + hh] =
            den > 0.f ? make_float2(M * kLn2, den) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) cl_w[hh][j] = mj[j] * inv;
    }
    __syncthreads();
    constexpr int F = DH / 8;                         // 16-byte slots (8 bf16) per head row
    const uint32_t ob = smem_u32(kv_s);
    uint32_t peer[kMaxSplits];
#pragma unroll
    for (int j = 0; j < kMaxSplits; ++j) peer[j] = cluster_map(ob, (uint32_t)(j < ns ? j : 0));
    for (int it = threadIdx.x; it < (he - hb) * F; it += blockDim.x) {
      const int hh = hb + it / F, f = it % F;
      if (h0 + hh >= p.H) continue;
      const uint32_t off = (uint32_t)(hh * DH * 2 + (((f & ~7) | ((f ^ hh) & 7)) * 16));
      uint4 v[kMaxSplits];
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j)
        if (j < ns) v[j] = ld_cluster_u4(peer[j] + off);
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) {
        if (j < ns) {
          const float wj = cl_w[hh][j];
          const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(hv[e]);
            acc[2 * e] = fmaf(wj, x.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(wj, x.y, acc[2 * e + 1]);
          }
        }
      }
      uint4 u;
      __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) ho[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ((int64_t)qi * p.H + h0 + hh) * D + dh * DH +
                                f * 8) = u;
    }
    cluster_sync();                                   // no CTA leaves while its shared memory is read
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ------------------------------------------------------------------ sharded decode
// G partial results over disjoint row sets (sparse_attn_partial) -> the attention output,
// with the sink added once ([HA] §6 probability over the union of the sets):
// M = max(sink, m_g), den = e^(sink - M) + sum_g l_g e^(m_g - M),
// out = sum_g l_g e^(m_g - M) o_g / den.  One warp per (query, head); 8 dims per 16-byte load.
// Shard g's output rows start at parts + g * part_stride bytes and its (m, l) at
// ml + g * ml_stride bytes (one gathered buffer per shard, or two stacked arrays).
__global__ void __launch_bounds__(256) attn_combine_kernel(const uint8_t* __restrict__ parts_b, int64_t part_stride,
                                                           const uint8_t* __restrict__ ml_b, int64_t ml_stride,
                                                           const float* __restrict__ sink, int G, int64_t rows,
                                                           int H, int D, __nv_bfloat16* __restrict__ out) {
  griddep_sync();
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int h = (int)(r % H);
  const float sinkL = sink[h] * kLog2e;
  float M = sinkL;
  auto mlg = [&](int g) { return reinterpret_cast<const float2*>(ml_b + (int64_t)g * ml_stride)[r]; };
  for (int g = 0; g < G; ++g) {
    const float2 v = mlg(g);
    if (v.y > 0.f) M = fmaxf(M, v.x * kLog2e);
  }
  float den = exp2f(sinkL - M);
  for (int g = 0; g < G; ++g) {
    const float2 v = mlg(g);
    if (v.y > 0.f) den += v.y * exp2f(v.x * kLog2e - M);
  }
  const float inv = 1.f / den;
  for (int c = lane_id(); c < D / 8; c += 32) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int g = 0; g < G; ++g) {
      const float2 v = mlg(g);
      if (!(v.y > 0.f)) continue;
      const float wg = v.y * exp2f(v.x * kLog2e - M) * inv;
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(parts_b + (int64_t)g * part_stride + r * D * 2) + c);
      const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(hv[e]);
        acc[2 * e] = fmaf(wg, x.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(wg, x.y, acc[2 * e + 1]);
      }
    }
    uint4 o;
    __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) ho[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
    reinterpret_cast<uint4*>(out + r * D)[c] = o;
  }
}

}  // namespace csa
