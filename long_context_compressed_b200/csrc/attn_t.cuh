// attn_t.cuh -- shared-KV multi-query attention with an attention sink, rows of the
// memory as the tensor-core M dimension.
//
// What it computes is attn.cuh's definition ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文"
// §4.2 Shared-KV MQA over the selected entries, §6 SWA branch and sink, §7 one softmax
// over concat(SWA rows, selected rows); "解密DeepSeek-V4-Flash-NVFP4的混合注意力机制…"
// sparse_attn(q, kv, attn_sink, topk_idxs, softmax_scale)), for bf16 rows:
//   z_j = scale * <q_h, row_j>,  o_h = sum_j e^{z_j} row_j / (e^{sink_h} + sum_l e^{z_l}).
//
// Decode has few query rows per sequence (one token: 64 or 128 heads) against hundreds of
// memory rows, so the scores are computed transposed, S^T = rows x heads:
//   S^T[r][h] = <row_r, q_h>    tcgen05, M = 128 rows, N = 64 heads, K = D (D/16 MMAs)
//   O^T[d][h] += sum_r row_r[d] P^T[r][h]    M = 128 dims per MMA (D/128 of them),
//                                           N = 64 heads, K = rows (16 per MMA)
// Both MMAs read the same row tile in shared memory (K-major for S^T, MN-major for the
// value side), P^T is written by the softmax threads into shared memory, and O^T lives
// in tensor memory for all D dims of the CTA's 64 heads.  Against the heads x rows form
// this issues 4x fewer MMAs per row (64 heads as N instead of 32 rows) and needs no split
// of D across CTAs.
//
// CTA = (split of the row list, group of 64 heads, query).  Rows arrive in units of 64
// (one shared-memory stage each, two stages; the softmax warps load unit 1 beside the
// loader warps' unit 0): gathered rows by cp.async (16-byte pieces),
// 64 consecutive rows of one buffer (SWA rows, hca_attn's memory rows) by eight TMA boxes
// of 8 rows.  A stage is stored as eight 8-row groups, each group holding its rows' D/64
// 128-byte-swizzled atoms: two adjacent stages are then one 128-row operand, so a CTA with
// two units scores both with one set of MMAs ("pair" mode); otherwise each unit is one
// M = 128 MMA whose upper 64 lanes read the next 64 KB of shared memory and are ignored.
//
// Softmax: TMEM lane = row, so the per-head maximum and sum run across lanes: a butterfly
// over the 32 lanes of a warp (64 values -> 2 per lane), then across the four warps in
// shared memory.  The reference maximum of a head is raised only when a unit's maximum
// exceeds it by more than 2^64 (base 2), so exponentials stay <= 2^64 and O^T is rescaled
// in tensor memory only in that rare case.  With several splits the split CTAs of one
// (query, head group) form a thread-block cluster: each stores its unnormalised O (bf16)
// and per-head (m, l) straight from tensor memory into a workspace, one cluster barrier
// (release / acquire) orders those stores before the reads, and CTA r then merges heads
// [r*64/ns, (r+1)*64/ns) of every split from L2, sink included.  (Measured against this:
// bulk copies of the slices into shared memory, and a push of bf16 slices between the
// CTAs' shared memories; both slower.)
#pragma once
#include <cuda_bf16.h>
#include "attn.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace csa {

template <int D>
struct AttnTCfg {
  static constexpr int HG = 64;                    // heads per CTA (MMA N)
  static constexpr int U = 64;                     // rows per unit / stage
  static constexpr int NS = 2;                     // stages
  static constexpr int kAtoms = D / 64;            // 128-byte atoms per row
  static constexpr int kGroup = kAtoms * 1024;     // bytes of one 8-row group (all atoms)
  static constexpr int kStage = U * D * 2;         // bytes of one stage (8 groups)
  static constexpr int kQ = HG * D * 2;            // q tile: [atom][64 heads][128 B]
  static constexpr int kP = 128 * 128;             // P^T: 128 rows x 64 heads bf16
  static constexpr int kMaxCtaRows = 1024;         // index values staged per CTA
  static constexpr int kOnes = 4096;               // 128 x 16 bf16 ones: the A operand of the row sums
  static constexpr int kMisc = 512 + 4 * kMaxCtaRows + kOnes;
  static constexpr int kSmem = 1024 + NS * kStage + kQ + kP + kMisc;
  static constexpr int kMT = D / 128;              // O^T M-tiles
  static constexpr int kSCol = 256;                // S^T buffers at TMEM columns 256 and 320
  static constexpr int kLCol = 384;                // per-head sums of P (every lane the same) at 384..447
  static constexpr int kThreads = 288;             // 4 softmax + 4 loader + 1 MMA warps
  static constexpr float kRescaleLog2 = 64.f;      // raise a head's reference max beyond this
  static_assert(D == 128 || D == 256 || D == 512, "D");
  static_assert(kStage == kQ, "a stage's upper-half filler reads stay inside shared memory");
};

// Byte offset of 16-byte chunk c of row r inside a stage (8-row groups, atoms of 128 B).
template <int D>
__device__ __forceinline__ uint32_t st_off(int r, int c) {
  return (uint32_t)((r >> 3) * AttnTCfg<D>::kGroup + (c >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Max over the 32 lanes of a warp for 64 values per lane -> lane l holds the results for
// values 2l and 2l+1 (butterfly: at each step a lane keeps the half of its values its lane
// bit selects and combines it with the partner's copy of that half).
template <bool MAX>
__device__ __forceinline__ float2 warp_reduce64(float* v) {
  const int lane = (int)lane_id();
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int half = 32 >> s;                      // 32, 16, 8, 4, 2 values kept
    const int bit = 16 >> s;                       // lane bit of this step
    const bool up = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = up ? v[half + i] : v[i];
      const float send = up ? v[i] : v[half + i];
      const float got = __shfl_xor_sync(0xffffffffu, send, bit);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return make_float2(v[0], v[1]);
}

template <int D>
__global__ void __launch_bounds__(288, 1) attn_t_kernel(const __grid_constant__ CUtensorMap qmap,
                                                        const __grid_constant__ CUtensorMap kvmap,
                                                        const __grid_constant__ CUtensorMap swamap,
                                                        const AttnParams p) {
  using Cfg = AttnTCfg<D>;
  constexpr int HG = Cfg::HG, U = Cfg::U;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kv_s = smem;                                    // [2][kStage]
  uint8_t* q_s = kv_s + Cfg::NS * Cfg::kStage;             // [kQ]
  uint8_t* p_s = q_s + Cfg::kQ;                            // [kP]
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + Cfg::kP);
  uint64_t* full = bars;          // [2] unit loaded (128 cp.async arrivals + 4 mask words)
  uint64_t* empty = bars + 2;     // [2] unit consumed by its PV
  uint64_t* sfull = bars + 4;     // [2] S^T ready
  uint64_t* pfull = bars + 6;     // [2] P^T written (4 softmax warps)
  uint64_t* pdone = bars + 8;     // [2] PV done
  uint64_t* qfull = bars + 10;
  uint64_t* odone = bars + 11;
  uint64_t* qrot = bars + 13;     // RoPE dims of q turned (4 softmax warps)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 12);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(bars + 14);   // [2 stages][4 loader warps], 16 rows each
  int32_t* idx_s = reinterpret_cast<int32_t*>(bars + 64);      // [kMaxCtaRows]
  uint8_t* ones_s = reinterpret_cast<uint8_t*>(idx_s + Cfg::kMaxCtaRows);   // [kOnes] bf16 1.0

  __shared__ float red_max[4][HG];
  __shared__ float m_use[HG], fscale[HG];
  __shared__ float epi_g[HG];
  __shared__ int epi_have_o;
  __shared__ float2 rope_tab[kRopeDims / 2];   // cos, sin of the query position's angles

  const int qi = blockIdx.z;                     // b * T + t
  const int b = qi / p.T, t = qi % p.T;
  const int h0 = blockIdx.y * HG;
  const int split = blockIdx.x;
  const int64_t item = (int64_t)qi * gridDim.y + blockIdx.y;   // (query, head group)
  const int warp = warp_id();
  const int32_t* idx_row = p.sparse ? p.idx + ((int64_t)b * p.T + t) * p.k : nullptr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 128 + 4);
      mbar_init(&empty[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 4);
      mbar_init(&pdone[i], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(odone, 1);
    mbar_init(qrot, 4);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < Cfg::kOnes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(ones_s)[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  fence_proxy_async_smem();                        // generic-proxy writes -> tensor-core reads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_sync();
  const RowList rl = make_row_list(p, b, t);
  const int mem0 = rl.n_swa;                     // list row of the first memory row
  const int n_rows = mem0 + rl.n_mem;
  const int n_units_all = (n_rows + U - 1) / U;
  const int u0 = (int)((int64_t)split * n_units_all / p.nsplit);
  const int u1 = (int)((int64_t)(split + 1) * n_units_all / p.nsplit);
  const int nu = u1 > u0 ? u1 - u0 : 0;          // units of this CTA
  const bool pair = nu == 2;                     // both units scored as one 128-row operand
  const int ntiles = pair ? 1 : nu;
  const int row0 = u0 * U;                       // first list row of this CTA
  const bool rope = p.rope_theta > 0.0;
  // list row rg -> element offset of its row (SWA rows encoded as -2 - offset), or -1
  auto row_src = [&](int rg, int32_t raw) -> int64_t {
    if (rg >= n_rows) return -1;
    if (rg < rl.n_swa) return -2 - ((int64_t)b * p.W + rl.swa_row0 + rg) * D;
    const int64_t i = p.sparse ? (int64_t)raw : (int64_t)(rg - mem0);
    if (i < 0 || i >= p.N) return -1;
    return ((int64_t)b * p.N + i) * D;
  };

  // One unit's rows into its stage by 128 threads (lt = 0..127): warp w of the group fills
  // rows 16w .. 16w+15, four rows per pass: lane l copies 16-byte chunk l % 8 of every
  // 128-byte atom of row 4 * pass + l / 8, so one cp.async of the warp reads four whole
  // 128-byte lines.  A unit of 64 consecutive rows of one buffer goes by eight TMA boxes
  // instead.  Arrives 128 + 4 times on full[s] (the copies of every thread, one validity
  // word per warp).
  const bool staged_idx = p.sparse && nu * U <= Cfg::kMaxCtaRows;
  auto load_unit = [&](int u, int lt, bool use_staged) -> bool {
    const __nv_bfloat16* kv = static_cast<const __nv_bfloat16*>(p.kv);
    const __nv_bfloat16* swa = static_cast<const __nv_bfloat16*>(p.swa);
    const int wl = lt >> 5, lane = (int)lane_id();
    const int sub = lane >> 3, c8 = lane & 7;
    const int s = u & 1;
    const uint32_t ph = (u >> 1) & 1;
    if (!mbar_wait(&empty[s], ph ^ 1)) return false;
    uint8_t* stage = kv_s + s * Cfg::kStage;
    const int rg0 = row0 + u * U;
    const bool swa_tile = p.has_swamap && rg0 + U <= rl.n_swa;
    const bool mem_tile = p.has_kvmap && !p.sparse && rg0 >= mem0 && rg0 + U <= n_rows;
    uint32_t rows = 0xFFFFu;                      // validity of this warp's 16 rows
    if (swa_tile || mem_tile) {
      // eight boxes of {64 dims, 8 rows, all atoms}: each lands as one 8-row group
      if (lt < 32) {
        if (lt == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)Cfg::kStage);
        __syncwarp();
        if (lt < 8) {
          const int y = swa_tile ? (int)rl.swa_row0 + rg0 + 8 * lt : rg0 - mem0 + 8 * lt;
          tma_load_4d(stage + lt * Cfg::kGroup, swa_tile ? &swamap : &kvmap, &full[s], 0, y, 0, b);
        }
        if (lt != 0) mbar_arrive(&full[s]);
      } else {
        mbar_arrive(&full[s]);
      }
    } else {
      const __nv_bfloat16* src[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = 16 * wl + 4 * j + sub;
        const int rg = rg0 + r;
        int32_t raw = 0;
        if (p.sparse && rg >= mem0 && rg < n_rows)
          raw = use_staged ? idx_s[u * U + r] : __ldg(idx_row + (rg - mem0));
        const int64_t so = row_src(rg, raw);
        src[j] = so >= 0 ? kv + so : (so <= -2 ? swa + (-2 - so) : nullptr);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = 16 * wl + 4 * j + sub;
#pragma unroll
        for (int a = 0; a < Cfg::kAtoms; ++a) {
          const int ch = a * 8 + c8;
          uint8_t* dst = stage + st_off<D>(r, ch);
          if (src[j]) cp_async_16(dst, src[j] + ch * 8);
          else st_shared_zero16(dst);             // finite filler for rows that do not contribute
        }
      }
      fence_proxy_async_smem();
      cp_async_arrive_noinc(&full[s]);
      rows = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t bal = __ballot_sync(0xffffffffu, src[j] != nullptr);
#pragma unroll
        for (int q = 0; q < 4; ++q) rows |= ((bal >> (8 * q)) & 1u) << (4 * j + q);
      }
    }
    // row validity, one word per warp of the group (16 rows)
    if (lane == 0) {
      mask_s[s * 4 + wl] = rows;
      mbar_arrive(&full[s]);
    }
    return true;
  };
  // With two or more units the softmax warps, idle until the first S^T lands, fill stage 1
  // (unit 1) while the loader warps fill stage 0: the first two units' copies are issued
  // by 256 threads at once.
  const bool helped = nu >= 2;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ loaders (128 threads)
    const int lt = threadIdx.x - 128;
    if (lt == 0) {
      if (p.has_kvmap) prefetch_tmap(&kvmap);
      if (p.has_swamap) prefetch_tmap(&swamap);
    }
    if (nu > 0) {
      if (staged_idx) {
        for (int r = lt; r < nu * U; r += 128) {
          const int rg = row0 + r;
          idx_s[r] = (rg >= mem0 && rg < n_rows) ? __ldg(idx_row + (rg - mem0)) : 0;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      for (int u = 0; u < nu; ++u) {
        if (u == 1 && helped) continue;           // the softmax warps' unit
        if (!load_unit(u, lt, staged_idx)) break;
      }
      cp_async_wait_group<0>();                   // none may land after the CTA has left
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ q by TMA, then the MMA issuer
    if (elect_one() && nu > 0) {
      prefetch_tmap(&qmap);
      mbar_arrive_expect_tx(qfull, (uint32_t)Cfg::kQ);
      for (int a = 0; a < Cfg::kAtoms; ++a) tma_load_3d(q_s + a * HG * 128, &qmap, qfull, a * 64, h0, qi);
      const uint32_t idesc_s = make_idesc(128, HG, 1, 0, 0);
      const uint32_t idesc_o = make_idesc(128, HG, 1, 1, 1);
      const uint32_t idesc_l = make_idesc(128, HG, 1, 0, 1);
      // all-ones A (128 x 16, no swizzle): ones . P^T = the per-head sum of P in every lane
      const uint64_t ones_desc = smem_desc(smem_u32(ones_s), 128, 256, 0);
      const uint32_t qb = smem_u32(q_s);
      const uint32_t pb = smem_u32(p_s);
      bool ok = rope ? mbar_wait(qrot, 0) : mbar_wait(qfull, 0);
      // S^T of tile j: 128 rows starting at stage (j & 1) (pair: stage 0, both units)
      auto issue_s = [&](int j) -> bool {
        const int sb = j & 1;
        if (pair) {
          if (!mbar_wait(&full[0], 0) || !mbar_wait(&full[1], 0)) return false;
        } else {
          if (!mbar_wait(&full[sb], (j >> 1) & 1)) return false;
        }
        fence_proxy_async_smem();                 // cp.async data -> tensor core reads
        tc_fence_after();
        const uint32_t kb = smem_u32(kv_s + (pair ? 0 : sb) * Cfg::kStage);
        const uint32_t d = tmem + Cfg::kSCol + sb * HG;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int atom = kk >> 2, inner = (kk & 3) * 32;
          const uint64_t ad = smem_desc(kb + atom * 1024 + inner, 16, Cfg::kGroup, kLayoutSW128);
          const uint64_t bd = smem_desc(qb + atom * HG * 128 + inner, 16, 1024, kLayoutSW128);
          mma_bf16(d, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sfull[sb]);
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int sb = j & 1;
        // S^T buffer (j+1)&1 was last read by the softmax of tile j-1, whose pfull was
        // waited before PV(j-1) was issued
        if (j + 1 < ntiles && !issue_s(j + 1)) { ok = false; break; }
        if (!mbar_wait(&pfull[sb], (j >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const int rows_here = pair ? 2 * U : U;
        const int rg_end = n_rows - (row0 + j * U);   // list rows left from this tile's first
        const int nk = (min(rows_here, rg_end) + 15) / 16;
        const uint32_t vb = smem_u32(kv_s + (pair ? 0 : sb) * Cfg::kStage);
        const uint32_t pt = pb + (pair ? 0 : sb * (Cfg::kP / 2));
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t bd = smem_desc(pt + kk * 2048, 8192, 1024, kLayoutSW128);
#pragma unroll
          for (int m = 0; m < Cfg::kMT; ++m) {
            const uint64_t ad = smem_desc(vb + 2 * m * 1024 + kk * 2 * Cfg::kGroup, 1024, Cfg::kGroup, kLayoutSW128);
            mma_bf16(tmem + m * HG, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_bf16(tmem + Cfg::kLCol, ones_desc, bd, idesc_l, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&pdone[sb]);
        if (pair) {
          mma_commit(&empty[0]);
          mma_commit(&empty[1]);
        } else {
          mma_commit(&empty[sb]);
        }
      }
      mma_commit(odone);
    }
    __syncwarp();                                  // the warp is converged again before the cluster barriers
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax (warps 0..3, TMEM lane = row)
    if (helped) load_unit(1, threadIdx.x, false);  // unit 1 into stage 1 (its index values read directly)
    const int r = threadIdx.x;                   // row of the 128-row operand
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool owner = r < HG;                   // owner of head h0 + r's running statistics
    const bool head_ok = owner && h0 + r < p.H;
    const float zs = p.scale * kLog2e;
    float m_run = -INFINITY;                     // owners: running max (log2 domain)
    bool ok = true;
    if (rope) {
      // partial RoPE of q at the query's position: the last 64-dim atom of every head row,
      // turned in shared memory before the first S^T MMA reads it
      const int64_t qpos = p.q_pos[(int64_t)b * p.T + t];
      if (r < kRopeDims / 2) rope_tab[r] = rope_cs(qpos, p.rope_freq.f[r], false);
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (nu > 0) {
        if (!mbar_wait(qfull, 0)) ok = false;
        const int h = r >> 1;                      // head row; this thread takes 4 of its 8 chunks
        uint8_t* line = q_s + (Cfg::kAtoms - 1) * HG * 128 + h * 128;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = (r & 1) * 4 + c4;          // logical 16-byte chunk: dims D-64+8c .. +7
          uint4* ptr = reinterpret_cast<uint4*>(line + ((c ^ (h & 7)) << 4));
          uint4 u = *ptr;
          __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(hv[e]);
            const float2 y = rope_turn(x.x, x.y, rope_tab[4 * c + e]);
            hv[e] = __floats2bfloat162_rn(y.x, y.y);
          }
          *ptr = u;
        }
        fence_proxy_async_smem();                  // generic-proxy writes -> tensor-core reads
        __syncwarp();
        if (lane_id() == 0) mbar_arrive(qrot);
      }
    }
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      // this row's unit, and whether it is a row of this tile at all
      const int unit = pair ? (r >> 6) : j;
      const bool in_tile = pair || r < U;
      const int us = unit & 1;
      if (!mbar_wait(&full[us], (unit >> 1) & 1)) { ok = false; }
      const int rr = r & (U - 1);
      const bool valid = ok && in_tile && ((mask_s[us * 4 + (rr >> 4)] >> (rr & 15)) & 1u);
      if (!mbar_wait(&sfull[sb], (j >> 1) & 1)) ok = false;
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + Cfg::kSCol + sb * HG;
      float z[HG];
      tmem_ld32(s_addr, z);
      tmem_ld32(s_addr + 32, z + 32);
      tmem_wait_ld();
      // per-head maximum over this warp's 32 rows (every lane gets each head's maximum)
      float mine0 = -INFINITY, mine1 = -INFINITY;      // heads lane and lane + 32
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float m = warp_max_f32(valid ? z[h] * zs : -INFINITY);
        if (h == (int)lane_id()) mine0 = m;
        if (h == (int)lane_id() + 32) mine1 = m;
      }
      red_max[warp][lane_id()] = mine0;
      red_max[warp][lane_id() + 32] = mine1;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      bool need = false;
      if (owner) {
        const float tm = fmaxf(fmaxf(red_max[0][r], red_max[1][r]), fmaxf(red_max[2][r], red_max[3][r]));
        float f = 1.f;
        if (tm > m_run + Cfg::kRescaleLog2 || (m_run == -INFINITY && tm > -INFINITY)) {
          if (m_run != -INFINITY) {
            f = ex2_approx(m_run - tm);
            need = true;
          }
          m_run = tm;
        }
        m_use[r] = m_run == -INFINITY ? 0.f : m_run;
        fscale[r] = f;
      }
      // any head raised its reference after O^T holds earlier units: rescale O^T first
      const bool any = !bar_and_128<3>(!need);
      if (any && j > 0) {
        if (!mbar_wait(&pdone[(j - 1) & 1], ((j - 1) >> 1) & 1)) ok = false;
        tc_fence_after();
        // O^T's M-tiles and the sums of P (columns kLCol..) turn by the same per-head factors
        for (int m = 0; m <= Cfg::kMT; ++m) {
          const uint32_t col0 = m < Cfg::kMT ? (uint32_t)(m * HG) : (uint32_t)Cfg::kLCol;
          for (int c0 = 0; c0 < HG; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + col0 + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= fscale[c0 + c];
            tmem_st32(tmem + lane_base + col0 + c0, o);
          }
        }
        tmem_wait_st();
      }
      // p = 2^(z - m_use[h]); rows that do not contribute have z = -inf -> 0
      tmem_ld32(s_addr, z);
      tmem_ld32(s_addr + 32, z + 32);
      tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < HG; ++h) z[h] = valid ? z[h] * zs : -INFINITY;
#pragma unroll
      for (int h = 0; h < HG; h += 4) {
        const float4 mu = *reinterpret_cast<const float4*>(&m_use[h]);
        z[h] = ex2_approx(z[h] - mu.x);
        z[h + 1] = ex2_approx(z[h + 1] - mu.y);
        z[h + 2] = ex2_approx(z[h + 2] - mu.z);
        z[h + 3] = ex2_approx(z[h + 3] - mu.w);
      }
      // P^T buffer sb was last read by PV(j - 2)
      if (j >= 2 && !mbar_wait(&pdone[sb], ((j - 2) >> 1) & 1)) ok = false;
      if (in_tile) {
        uint8_t* prow = p_s + (pair ? 0 : sb * (Cfg::kP / 2)) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int c = 0; c < HG / 8; ++c) {
          uint4 u;
          __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) hv[e] = __floats2bfloat162_rn(z[8 * c + 2 * e], z[8 * c + 2 * e + 1]);
          *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = u;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&pfull[sb]);
    }
    if (helped) cp_async_wait_group<0>();         // (unit 1's copies landed before its S^T was issued)
    const bool have_o = ok && ntiles > 0 && mbar_wait(odone, 0);
    // the per-head sum of P over every unit (the same in every TMEM lane): head r from lane r
    float l_run = 0.f;
    if (warp < 2) {
      tc_fence_after();
      float lv[32];
      tmem_ld32(tmem + lane_base + Cfg::kLCol + (uint32_t)(warp * 32), lv);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c == (int)lane_id()) l_run = lv[c];
      if (!have_o) l_run = 0.f;
    }
    if (owner) {
      float g = 1.f;
      if (p.nsplit == 1) {
        if (p.ml) {
          g = (have_o && l_run > 0.f) ? 1.f / l_run : 0.f;
          if (head_ok) {
            float2* mlh = reinterpret_cast<float2*>(p.ml) + ((int64_t)qi * p.H + h0 + r);
            *mlh = (have_o && l_run > 0.f) ? make_float2(m_run * kLn2, l_run) : make_float2(-INFINITY, 0.f);
          }
        } else {
          const float sinkL = head_ok ? p.sink[h0 + r] * kLog2e : 0.f;
          const float M = fmaxf(m_run, sinkL);
          const float fo = (m_run == -INFINITY || !have_o) ? 0.f : exp2f(m_run - M);
          g = fo / (l_run * fo + exp2f(sinkL - M));
        }
      }
      epi_g[r] = g;
      if (p.nsplit > 1)
        reinterpret_cast<float2*>(p.part_ml)[(item * p.nsplit + split) * HG + r] =
            have_o ? make_float2(m_run, l_run) : make_float2(-INFINITY, 0.f);
    }
    if (r == 0) epi_have_o = have_o ? 1 : 0;
    tc_fence_before();
  }

  // ------------------------------------------------------------ epilogue (warps 0..7)
  // O^T: TMEM lane = dim within an M-tile, column = head.  Warp w reads lane quarter w % 4
  // of M-tiles m = w / 4, w / 4 + 2, ...
  if (warp < 8) {
    asm volatile("bar.sync 4, 256;" ::: "memory");
    tc_fence_after();
    const bool have_o = epi_have_o != 0;
    const int quarter = warp & 3;
    const uint32_t lane_q = (uint32_t)(quarter * 32) << 16;
    const int lane = (int)lane_id();
    // the KV stages are idle: this warp's transpose buffer (64 heads x 32 dims bf16); with
    // splits, this split's partial O [64 heads][D] bf16 in the workspace
    uint8_t* stage = kv_s + warp * (HG * 64);
    __nv_bfloat16* obuf = static_cast<__nv_bfloat16*>(p.part_o) + (item * p.nsplit + split) * HG * D;
    const int nh = min(HG, p.H - h0);
    for (int m = warp >> 2; m < Cfg::kMT; m += 2) {
      const int d = m * 128 + quarter * 32 + lane;
      __syncwarp();
      float oall[HG];
      if (have_o) {
        tmem_ld32(tmem + lane_q + m * HG, oall);
        tmem_ld32(tmem + lane_q + m * HG + 32, oall + 32);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int h = 0; h < HG; ++h) oall[h] = 0.f;
      }
#pragma unroll
      for (int hh = 0; hh < HG; hh += 32) {
        float* o = oall + hh;
        if (p.nsplit > 1) {
          // [head][D] bf16: lanes d, d ^ 1 pair up, the even lane storing even heads and the
          // odd lane odd heads as two adjacent values (one 4-byte store each; per store the
          // warp writes 64 contiguous bytes of two head rows)
          const bool odd = (d & 1) != 0;
#pragma unroll
          for (int h = 0; h < 32; h += 2) {
            const float got = __shfl_xor_sync(0xffffffffu, odd ? o[h] : o[h + 1], 1);
            const __nv_bfloat162 v = odd ? __floats2bfloat162_rn(got, o[h + 1]) : __floats2bfloat162_rn(o[h], got);
            *reinterpret_cast<__nv_bfloat162*>(obuf + (hh + h + (odd ? 1 : 0)) * D + (d & ~1)) = v;
          }
        } else {
#pragma unroll
          for (int h = 0; h < 32; ++h) o[h] *= epi_g[hh + h];
          if (rope && d >= D - kRopeDims) {          // inverse RoPE: pairs (d, d ^ 1) in adjacent lanes
            const float2 cs = rope_tab[(d - (D - kRopeDims)) >> 1];
            const float2 ics = make_float2(cs.x, -cs.y);
#pragma unroll
            for (int h = 0; h < 32; ++h) {
              const float other = __shfl_xor_sync(0xffffffffu, o[h], 1);
              const float2 y = (d & 1) ? rope_turn(other, o[h], ics) : rope_turn(o[h], other, ics);
              o[h] = (d & 1) ? y.y : y.x;
            }
          }
#pragma unroll
          for (int h = 0; h < 32; ++h)
            reinterpret_cast<__nv_bfloat16*>(stage)[(hh + h) * 32 + lane] = __float2bfloat16_rn(o[h]);
        }
      }
      if (p.nsplit > 1) continue;
      __syncwarp();
      __nv_bfloat16* obase = static_cast<__nv_bfloat16*>(p.out) + ((int64_t)qi * p.H + h0) * D + m * 128 + quarter * 32;
#pragma unroll
      for (int it = 0; it < HG / 8; ++it) {
        const int h = it * 8 + (lane >> 2), c = lane & 3;
        if (h < nh)
          *reinterpret_cast<uint4*>(obase + (int64_t)h * D + c * 8) =
              *reinterpret_cast<const uint4*>(stage + h * 64 + c * 16);
      }
      __syncwarp();
    }
  }

  if (p.nsplit > 1) {
    // ------------------------------------------------------------ merge of the splits
    // CTA `rank` finishes heads [rank*64/ns, (rank+1)*64/ns): M = max(sink, m_j),
    // den = 2^(sink - M) + sum_j l_j 2^(m_j - M), out = sum_j 2^(m_j - M) O_j / den.
    // One thread per 8 output dims of a head: it loads the ns (m, l) pairs and the ns
    // 16-byte pieces of O at once (L2 only: they were written by other SMs) and sums.
    const int ns = p.nsplit;
    const int rank = (int)cluster_ctarank();
    const int hb = rank * HG / ns, he = (rank + 1) * HG / ns;
    const __nv_bfloat16* po = static_cast<const __nv_bfloat16*>(p.part_o) + item * ns * HG * D;
    const float2* pml = static_cast<const float2*>(p.part_ml) + item * ns * HG;
    cluster_sync();                                   // release / acquire: every split's O and (m, l) are stored
    constexpr int F = D / 8;                          // 16-byte pieces (8 bf16) per head row
    for (int it = threadIdx.x; it < (he - hb) * F; it += blockDim.x) {
      const int hh = hb + it / F, f = it % F;
      if (h0 + hh >= p.H) continue;
      float2 ml[kMaxSplits];
      uint4 v[kMaxSplits];
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) {
        if (j < ns) {
          ml[j] = __ldcg(pml + j * HG + hh);
          v[j] = __ldcg(reinterpret_cast<const uint4*>(po + ((int64_t)j * HG + hh) * D + f * 8));
        } else {
          ml[j] = make_float2(-INFINITY, 0.f);
          v[j] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      const float sinkL = p.ml ? -INFINITY : p.sink[h0 + hh] * kLog2e;
      float M = sinkL;
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) M = fmaxf(M, ml[j].x);
      const bool any = M > -INFINITY;
      float den = any ? ex2_approx(sinkL - M) : 0.f;
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) {
        ml[j].x = any ? ex2_approx(ml[j].x - M) : 0.f;
        den = fmaf(ml[j].y, ml[j].x, den);
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      if (p.ml && f == 0)
        reinterpret_cast<float2*>(p.ml)[(int64_t)qi * p.H + h0 + hh] =
            den > 0.f ? make_float2(M * kLn2, den) : make_float2(-INFINITY, 0.f);
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxSplits; ++j) {
        const float w = ml[j].x * inv;
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = __bfloat1622float2(hv[e]);
          acc[2 * e] = fmaf(w, x.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(w, x.y, acc[2 * e + 1]);
        }
      }
      if (rope && f * 8 >= D - kRopeDims) {          // inverse RoPE of the merged output
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 cs = rope_tab[(f * 8 - (D - kRopeDims)) / 2 + e];
          const float2 y = rope_turn(acc[2 * e], acc[2 * e + 1], make_float2(cs.x, -cs.y));
          acc[2 * e] = y.x;
          acc[2 * e + 1] = y.y;
        }
      }
      uint4 u;
      __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) ho[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ((int64_t)qi * p.H + h0 + hh) * D + f * 8) = u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, 512);
}

}  // namespace csa
