// csa.cu -- host side of the C ABI declared in include/csa.h: argument
// validation, TMA tensor-map encoding, launch configuration.  All kernels
// live in the *.cuh files of this directory and are compiled into this one
// translation unit (one copy of the device status word).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <tuple>
#include <utility>
#include <mutex>
#include <vector>

#include "../../include/csa.h"
#include "append.cuh"
#include "attn.cuh"
#include "attn_t.cuh"
#include "causal.cuh"
#include "compress.cuh"
#include "index.cuh"
#include "index_topk.cuh"
#include "kv8.cuh"
#include "quantize.cuh"
#include "topk.cuh"

namespace {

using csa::AttnCfg;
using csa::AttnParams;
using csa::IndexParams;

constexpr int kMaxDev = 64;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per CTA on sm_100

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

int sm_count() {
  static int cache[kMaxDev] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

std::atomic<unsigned long long> g_launches{0};

// Status of the kernel launches just enqueued (n of them), counted into the
// library-wide launch counter.
int launch_status(int n = 1) {
  if (cudaGetLastError() != cudaSuccess) return CSA_ERR_CUDA;
  g_launches += (unsigned long long)n;
  return CSA_OK;
}

// Raise a kernel's dynamic shared-memory limit; the attribute is set once per
// (kernel, device) and only raised afterwards, so a call made during stream
// capture after a first eager call issues no runtime call.
template <typename K>
bool set_smem(K kernel, int bytes) {
  struct Grant {
    const void* fn;
    int dev, bytes;
  };
  static std::mutex mu;
  static std::vector<Grant> granted;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lock(mu);
  for (Grant& g : granted)
    if (g.fn == fn && g.dev == dev) {
      if (g.bytes >= bytes) return true;
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
      g.bytes = bytes;
      return true;
    }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  granted.push_back({fn, dev, bytes});
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over [dim2][dim1][inner] with a swizzled box {box0, box1, 1} (128-byte swizzle
// unless another is given).
bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esize, uint64_t inner, uint64_t dim1,
              uint64_t dim2, uint32_t box0, uint32_t box1,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, dim1, dim2};
  cuuint64_t strides[2] = {inner * esize, inner * dim1 * esize};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-tile map of a [dim2, rows, D] bf16 tensor seen as {64 elements, rows, D/64
// atoms, dim2}: one box of {64, box_rows, D/64, 1} holds box_rows full rows with
// each 64-element atom stored box_rows rows apart (128-byte swizzle).
bool make_row_tile_map(CUtensorMap* m, const void* ptr, uint64_t D, uint64_t rows, uint64_t dim2,
                       uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || D % 64 != 0 || D / 64 > 256) return false;
  cuuint64_t dims[4] = {64, rows, D / 64, dim2};
  cuuint64_t strides[3] = {D * 2, 128, rows * D * 2};
  cuuint32_t box[4] = {64, box_rows, (cuuint32_t)(D / 64), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Kernel launch with programmatic stream serialization (PDL): the kernel may begin
// launching while its predecessor in the stream finishes; every kernel of this
// library waits for the predecessor (griddepcontrol.wait) before touching global
// memory.  Set CSA_NO_PDL=1 in the environment to launch without the attribute.
bool use_pdl() {
  static const bool on = [] {
    const char* e = getenv("CSA_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

// Launch with programmatic dependent launch (unless disabled) and, for cluster_x > 1,
// thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
void launch_kc(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (use_pdl()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
void launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  launch_kc(kernel, grid, block, smem, st, 1, std::forward<Args>(args)...);
}

// Clusters of cluster_x CTAs of `kernel` that fit on the device at once (cached);
// 0 if the occupancy query fails.
template <typename... KArgs>
int max_active_clusters(void (*kernel)(KArgs...), int threads, int smem, int cluster_x) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(reinterpret_cast<const void*>(kernel), dev, cluster_x);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  if (!set_smem(kernel, smem)) return 0;
  if (cluster_x > 8 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cluster_x, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = n;
  return n;
}

// ------------------------------------------------------------------ attention split policy
int attn_ndh(int D) { return D > 256 ? D / 256 : 1; }

// CTAs per (query, D-slice, head group) over the row list: one wave of CTAs, at
// least two KV tiles each for sparse_attn (gathered rows: the more SMs issue the
// gathers, the sooner the rows are in) and four for hca_attn (contiguous rows by TMA,
// and it shares the GPU with the chain of the CSA layer).  When that leaves at most four
// tiles per split, the launch takes at most half the SMs, with the fewest splits that
// give the same largest share (the rule of the bf16 kernel below: the step's other
// attention then runs beside it).
int attn_nsplit(int B, int T, int H, int D, int64_t max_rows, bool sparse, int R) {
  const int64_t items = (int64_t)B * T * attn_ndh(D) * ((H + 63) / 64);
  const int sms = sm_count();
  if (items <= 0 || items >= 2 * sms) return 1;
  const int64_t tiles = (max_rows + R - 1) / R;
  const int64_t want = std::max<int64_t>(1, sms / items);
  const int64_t cap = std::max<int64_t>(1, tiles / (sparse ? 2 : 4));
  int64_t ns = std::max<int64_t>(1, std::min<int64_t>(std::min(want, cap), csa::kMaxSplits));   // one cluster
  const int64_t half = std::max<int64_t>(1, sms / 2 / items);
  if (tiles <= 4 * ns && ns > half) {
    ns = half;
    const int64_t share = (tiles + ns - 1) / ns;
    while (ns > 1 && (tiles + ns - 2) / (ns - 1) == share) --ns;
  }
  return (int)ns;
}

// bf16 rows (attn_t_kernel): splits of a query's row list (units of 64 rows) form one
// cluster: as many as the SMs allow for one wave, at most one per unit and at most
// kMaxSplits (the launch may take fewer, while the clusters would not all be resident).
// When that leaves a unit or two per split the launch is latency-bound: it then takes at
// most half the SMs, so an independent launch beside it (another layer's attention, the
// kernels of another chain) runs at the same time, and among the split counts with the
// same largest share of units it takes the fewest.  Measured on the 8-sequence 64K decode
// (10 units per query): alone 12.7 -> 14.9 us, but the CSA + HCA step beside it
// 61.5 -> 51.2 us.
int attn_t_splits(int B, int T, int H, int64_t max_rows) {
  const int64_t items = (int64_t)B * T * ((H + 63) / 64);
  const int64_t units = std::max<int64_t>(1, (max_rows + 63) / 64);
  const int sms = sm_count();
  if (items <= 0 || items >= sms) return 1;
  int64_t ns = std::min<int64_t>(std::min<int64_t>(csa::kMaxSplits, units), std::max<int64_t>(1, sms / items));
  const int64_t half = std::max<int64_t>(1, sms / 2 / items);
  if (units <= 2 * ns && ns > half) {
    ns = half;
    const int64_t share = (units + ns - 1) / ns;
    while (ns > 1 && (units + ns - 2) / (ns - 1) == share) --ns;
  }
  return (int)ns;
}

// Workspace of a split launch: each split's unnormalised O (bf16, 64 heads x D) and its
// per-head (m, l) (two floats), per (query, head group).  The KV8 and fp32 kernels merge
// without one (cluster shared memory; no splits).
size_t attn_t_ws_bytes(int B, int T, int H, int D, int ns) {
  if (ns <= 1) return 0;
  const size_t items = (size_t)B * T * ((H + 63) / 64);
  return items * ns * 64 * ((size_t)D * 2 + 8);
}

size_t attn_ws_bytes(int B, int T, int H, int D, int64_t rows, int dtype) {
  if (dtype != CSA_BF16) return 0;
  return attn_t_ws_bytes(B, T, H, D, attn_t_splits(B, T, H, rows));
}

// bf16 rows: attn_t_kernel (rows as the MMA's M dimension, 64 heads per CTA, all of D).
template <int D>
int launch_attn_t(AttnParams p, int64_t max_rows, void* ws, size_t ws_bytes, cudaStream_t st) {
  using Cfg = csa::AttnTCfg<D>;
  const int groups = (p.H + Cfg::HG - 1) / Cfg::HG;
  const int64_t items = (int64_t)p.B * p.T * groups;
  int ns = attn_t_splits(p.B, p.T, p.H, max_rows);
  auto kernel = csa::attn_t_kernel<D>;
  while (ns > 1) {
    const int fit = max_active_clusters(kernel, Cfg::kThreads, Cfg::kSmem, ns);
    if (fit == 0 && ns > 8) {              // a non-portable size the device does not take
      ns = 8;
      continue;
    }
    if (fit >= items || fit == 0) break;   // 0: the query failed; keep the portable choice
    --ns;
  }
  p.nsplit = ns;
  if (ns > 1) {
    const size_t need = attn_t_ws_bytes(p.B, p.T, p.H, D, ns);
    if (!ws || ws_bytes < need || !aligned16(ws)) return CSA_ERR_INVALID;
    p.part_o = ws;
    p.part_ml = static_cast<uint8_t*>(ws) + items * ns * 64 * (size_t)D * 2;
  }
  CUtensorMap qmap, kvmap, swamap;
  if (!make_map(&qmap, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)D, (uint64_t)p.H, (uint64_t)p.B * p.T,
                64, 64))
    return CSA_ERR_CUDA;
  std::memset(&kvmap, 0, sizeof(kvmap));
  std::memset(&swamap, 0, sizeof(swamap));
  p.has_kvmap = p.N > 0 && make_row_tile_map(&kvmap, p.kv, (uint64_t)D, (uint64_t)p.N, (uint64_t)p.B, 8) ? 1 : 0;
  p.has_swamap = p.W > 0 && make_row_tile_map(&swamap, p.swa, (uint64_t)D, (uint64_t)p.W, (uint64_t)p.B, 8) ? 1 : 0;
  if (!set_smem(kernel, Cfg::kSmem)) return CSA_ERR_CUDA;
  if (ns > 8 && cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return CSA_ERR_CUDA;
  dim3 grid((unsigned)ns, (unsigned)groups, (unsigned)(p.B * p.T));
  launch_kc(kernel, grid, Cfg::kThreads, Cfg::kSmem, st, ns, qmap, kvmap, swamap, p);
  return launch_status();
}

int run_attn_t(const AttnParams& p, int64_t max_rows, void* ws, size_t ws_bytes, cudaStream_t st) {
  switch (p.D) {
    case 128: return launch_attn_t<128>(p, max_rows, ws, ws_bytes, st);
    case 256: return launch_attn_t<256>(p, max_rows, ws, ws_bytes, st);
    case 512: return launch_attn_t<512>(p, max_rows, ws, ws_bytes, st);
    default: return CSA_ERR_UNSUPPORTED;
  }
}

int run_attn(AttnParams p, int dtype, void* ws, size_t ws_bytes, int64_t max_rows, cudaStream_t st) {
  if (p.B == 0 || p.T == 0) return CSA_OK;
  if (dtype == CSA_F32) {
    dim3 grid((p.H + 3) / 4, p.T, p.B);
    switch (p.D) {
      case 32: launch_k(csa::attn_f32_kernel<1>, grid, 128, 0, st, p); break;
      case 64: launch_k(csa::attn_f32_kernel<2>, grid, 128, 0, st, p); break;
      case 128: launch_k(csa::attn_f32_kernel<4>, grid, 128, 0, st, p); break;
      case 256: launch_k(csa::attn_f32_kernel<8>, grid, 128, 0, st, p); break;
      case 512: launch_k(csa::attn_f32_kernel<16>, grid, 128, 0, st, p); break;
      default: return CSA_ERR_UNSUPPORTED;
    }
    return launch_status();
  }
  const bool kv8 = dtype == CSA_BF16_KV8;
  if (!kv8) return run_attn_t(p, max_rows, ws, ws_bytes, st);
  // rows per KV tile: 32 at D = 512 (four stages in shared memory), else 64.  Measured:
  // 64-row tiles at D = 512 (two stages) were slower for gathered, dense and KV8 rows.
  const int R = p.D < 512 ? 64 : 32;
  p.nsplit = attn_nsplit(p.B, p.T, p.H, p.D, max_rows, p.sparse != 0, R);
  (void)ws;
  (void)ws_bytes;
  // grid: (splits of the row list, D-slice x head group of 64, query)
  dim3 grid(p.nsplit, attn_ndh(p.D) * ((p.H + 63) / 64), p.B * p.T);
  // fewer splits while the clusters would not all be resident at once (one CTA per
  // SM, a cluster's CTAs in one GPC)
  const int64_t items = (int64_t)grid.y * grid.z;
  while (p.nsplit > 1) {
    int fit = 0;
    switch (p.D) {
      case 128: fit = max_active_clusters(csa::attn_tc_kernel<128, false, 64>, 288, AttnCfg<128, 64>::kSmem, p.nsplit); break;
      case 256: fit = max_active_clusters(csa::attn_tc_kernel<256, false, 64>, 288, AttnCfg<256, 64>::kSmem, p.nsplit); break;
      case 512:
        fit = kv8 ? max_active_clusters(csa::attn_tc_kernel<512, true, 32>, csa::attn_threads(true),
                                        AttnCfg<512, 32>::kSmem, p.nsplit)
                  : max_active_clusters(csa::attn_tc_kernel<512, false, 32>, 288, AttnCfg<512, 32>::kSmem, p.nsplit);
        break;
      default: break;
    }
    if (fit == 0 && p.nsplit > 8) {        // a non-portable size the device does not take
      p.nsplit = 8;
      continue;
    }
    if (fit >= items || fit == 0) break;   // 0: the query failed; keep the portable choice
    --p.nsplit;
  }
  grid.x = p.nsplit;
  // Q [B*T, H, D] by TMA: boxes of {64 dims, 64 head rows}, rows past H zero-filled
  CUtensorMap qmap, kvmap, swamap;
  if (!make_map(&qmap, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.D, (uint64_t)p.H,
                (uint64_t)p.B * p.T, 64, 64))
    return CSA_ERR_CUDA;
  // kv and swa_kv as boxes of {64 dims, R rows}: contiguous row tiles load by TMA
  const uint32_t rows_per_tile = (uint32_t)R;
  std::memset(&kvmap, 0, sizeof(kvmap));
  std::memset(&swamap, 0, sizeof(swamap));
  // (KV8 entries are not bf16 rows: they are always copied and converted by the loaders)
  p.has_kvmap = !kv8 && p.N > 0 && make_row_tile_map(&kvmap, p.kv, (uint64_t)p.D, (uint64_t)p.N, (uint64_t)p.B,
                                                     rows_per_tile) ? 1 : 0;
  p.has_swamap = p.W > 0 && make_row_tile_map(&swamap, p.swa, (uint64_t)p.D, (uint64_t)p.W, (uint64_t)p.B,
                                              rows_per_tile) ? 1 : 0;
  auto launch = [&](auto kernel, int threads, int smem) -> int {
    if (!set_smem(kernel, smem)) return CSA_ERR_CUDA;
    launch_kc(kernel, grid, threads, smem, st, p.nsplit, qmap, kvmap, swamap, p);
    return CSA_OK;
  };
  int rc = CSA_ERR_UNSUPPORTED;
  if (kv8) {
    if (p.D == 512) rc = launch(csa::attn_tc_kernel<512, true, 32>, csa::attn_threads(true), AttnCfg<512, 32>::kSmem);
  } else if (p.D == 512) {
    rc = launch(csa::attn_tc_kernel<512, false, 32>, 288, AttnCfg<512, 32>::kSmem);
  } else if (p.D == 256) {
    rc = launch(csa::attn_tc_kernel<256, false, 64>, 288, AttnCfg<256, 64>::kSmem);
  } else if (p.D == 128) {
    rc = launch(csa::attn_tc_kernel<128, false, 64>, 288, AttnCfg<128, 64>::kSmem);
  }
  if (rc != CSA_OK) return rc;
  return launch_status();
}

int check_attn_common(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                      const int64_t* q_pos, const float* sink, float scale, int B, int T, int H, int D, int64_t N,
                      int dtype, const void* out) {
  if (B < 0 || T < 0 || H <= 0 || D <= 0 || N < 0 || W < 0) return CSA_ERR_INVALID;
  if ((int64_t)B * T * H * (D / 8) >= (int64_t(1) << 31) || (int64_t)B * T > 65535 * 1024)
    return CSA_ERR_UNSUPPORTED;
  if (dtype != CSA_F32 && dtype != CSA_BF16 && dtype != CSA_BF16_KV8) return CSA_ERR_INVALID;
  if (!(scale == scale)) return CSA_ERR_INVALID;
  if (B == 0 || T == 0) return CSA_OK;
  if (!q || !out || !swa_pos0 || !q_pos || !sink) return CSA_ERR_INVALID;
  if (N > 0 && !kv) return CSA_ERR_INVALID;
  if (W > 0 && !swa_kv) return CSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(out) || (kv && !aligned16(kv)) || (swa_kv && !aligned16(swa_kv)))
    return CSA_ERR_INVALID;
  if (dtype == CSA_BF16) {
    if (D != 128 && D != 256 && D != 512) return CSA_ERR_UNSUPPORTED;
    if (H > 128) return CSA_ERR_UNSUPPORTED;
  } else if (dtype == CSA_BF16_KV8) {
    if (D != csa::kKv8Dims) return CSA_ERR_UNSUPPORTED;
    if (H > 128) return CSA_ERR_UNSUPPORTED;
  } else {
    if (D % 32 != 0 || D > 512) return CSA_ERR_UNSUPPORTED;
  }
  return CSA_OK;
}

}  // namespace

extern "C" {

const char* csa_status_string(int status) {
  switch (status) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID: return "CSA_ERR_INVALID: invalid argument";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED: unsupported shape or dtype";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA: CUDA runtime or launch failure";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT: a kernel abandoned a bounded wait";
    default: return "unknown csa status";
  }
}

int csa_version(void) { return 101; }

int csa_n_valid(const int64_t* q_pos, int64_t count, int ratio, int64_t lo, int64_t hi, int32_t* n_valid,
                void* stream) {
  if (count < 0 || ratio < 1 || lo < 0 || hi < lo || hi - lo > INT32_MAX) return CSA_ERR_INVALID;
  if (count == 0) return CSA_OK;
  if (!q_pos || !n_valid) return CSA_ERR_INVALID;
  const unsigned blocks = (unsigned)std::min<int64_t>((count + 255) / 256, (int64_t)sm_count() * 4);
  launch_k(csa::n_valid_kernel, blocks, 256, 0, as_stream(stream), q_pos, count, ratio, lo, hi, n_valid);
  return launch_status();
}

int csa_test_bounded_wait(int complete, long long limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000LL) return CSA_ERR_INVALID;
  launch_k(csa::bounded_wait_kernel, 1, 32, 0, as_stream(stream), complete ? 1 : 0, (uint64_t)limit_ns);
  return launch_status();
}

int csa_compress(const void* C_a, const void* C_b, const void* Z_a, const void* Z_b, const void* prev_Cb,
                 const void* prev_Zb, int B, int64_t L, int c, int ratio, int in_dtype, int out_dtype, void* out,
                 void* stream) {
  if (B < 0 || L < 0 || c <= 0) return CSA_ERR_INVALID;
  if (ratio != 4 && ratio != 128) return CSA_ERR_INVALID;
  if ((in_dtype != CSA_F32 && in_dtype != CSA_BF16) || (out_dtype != CSA_F32 && out_dtype != CSA_BF16))
    return CSA_ERR_INVALID;
  if ((prev_Cb == nullptr) != (prev_Zb == nullptr)) return CSA_ERR_INVALID;
  if (ratio == 4 && c % 8 != 0) return CSA_ERR_INVALID;
  if (ratio == 128 && (c % 128 != 0 || C_b || Z_b || prev_Cb || prev_Zb)) return CSA_ERR_INVALID;
  const int64_t n_entries = L / ratio;
  if (B == 0 || n_entries == 0) return CSA_OK;
  if (!C_a || !Z_a || !out || (ratio == 4 && (!C_b || !Z_b))) return CSA_ERR_INVALID;
  const void* ptrs[] = {C_a, C_b, Z_a, Z_b, prev_Cb, prev_Zb, out};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CSA_ERR_INVALID;
  cudaStream_t st = as_stream(stream);
  const bool bf_in = in_dtype == CSA_BF16, bf_out = out_dtype == CSA_BF16;
  if (ratio == 4) {
    // 8 channels per thread (16-byte loads) only once that still gives two waves of
    // CTAs: its 2m x 8 live values per thread cap residency at one CTA per SM, which
    // on smaller inputs loses to the 2-channel variant's occupancy
    const int64_t total8 = (int64_t)B * n_entries * (c / 8);
    const bool wide = total8 >= (int64_t)sm_count() * 2 * 256;
    const int64_t total = wide ? total8 : 4 * total8;
    if (total >= (int64_t(1) << 31)) return CSA_ERR_UNSUPPORTED;
    const int64_t blocks64 = (total + 255) / 256;
    const unsigned blocks = (unsigned)std::min<int64_t>(blocks64, (int64_t)sm_count() * 16);
#define CSA_LAUNCH_CSA(TI, TO)                                                                                  \
  do {                                                                                                          \
    if (wide)                                                                                                   \
      launch_k(csa::compress_csa_kernel<TI, TO, 4, 8>, blocks, 256, 0, st, (const TI*)C_a, (const TI*)C_b,      \
               (const TI*)Z_a, (const TI*)Z_b, (const TI*)prev_Cb, (const TI*)prev_Zb, B, L, c, (TO*)out);      \
    else                                                                                                        \
      launch_k(csa::compress_csa_kernel<TI, TO, 4, 2>, blocks, 256, 0, st, (const TI*)C_a, (const TI*)C_b,      \
               (const TI*)Z_a, (const TI*)Z_b, (const TI*)prev_Cb, (const TI*)prev_Zb, B, L, c, (TO*)out);      \
  } while (0)
    if (bf_in && bf_out) CSA_LAUNCH_CSA(__nv_bfloat16, __nv_bfloat16);
    else if (bf_in) CSA_LAUNCH_CSA(__nv_bfloat16, float);
    else if (bf_out) CSA_LAUNCH_CSA(float, __nv_bfloat16);
    else CSA_LAUNCH_CSA(float, float);
#undef CSA_LAUNCH_CSA
  } else {
    if (n_entries > 65535 || B > 65535) return CSA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)((c + 63) / 64), (unsigned)n_entries, (unsigned)B);   // 64 channels per CTA
#define CSA_LAUNCH_HCA(TI, TO) \
  launch_k(csa::compress_hca_kernel<TI, TO>, grid, 256, 0, st, (const TI*)C_a, (const TI*)Z_a, B, L, c, (TO*)out)
    if (bf_in && bf_out) CSA_LAUNCH_HCA(__nv_bfloat16, __nv_bfloat16);
    else if (bf_in) CSA_LAUNCH_HCA(__nv_bfloat16, float);
    else if (bf_out) CSA_LAUNCH_HCA(float, __nv_bfloat16);
    else CSA_LAUNCH_HCA(float, float);
#undef CSA_LAUNCH_HCA
  }
  return launch_status();
}

int csa_compress_index_keys(const void* C_a, const void* C_b, const void* Z_a, const void* Z_b, const void* prev_Cb,
                            const void* prev_Zb, int B, int64_t L, int in_dtype, int hadamard, int64_t n_cap,
                            int64_t pos0, void* kI, uint8_t* k8, float* k_scale, void* stream) {
  if (B < 0 || L < 0 || n_cap < 0 || pos0 < 0) return CSA_ERR_INVALID;
  if (in_dtype != CSA_F32 && in_dtype != CSA_BF16) return CSA_ERR_INVALID;
  if ((prev_Cb == nullptr) != (prev_Zb == nullptr) || (k8 == nullptr) != (k_scale == nullptr)) return CSA_ERR_INVALID;
  const int64_t n_entries = L / 4;
  if (pos0 + n_entries > n_cap) return CSA_ERR_INVALID;
  if (B == 0 || n_entries == 0) return CSA_OK;
  if (!C_a || !C_b || !Z_a || !Z_b || !kI) return CSA_ERR_INVALID;
  const void* ptrs[] = {C_a, C_b, Z_a, Z_b, prev_Cb, prev_Zb, kI, k8};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return CSA_ERR_INVALID;
  const int64_t warps = (int64_t)B * n_entries;
  const unsigned blocks = (unsigned)std::min<int64_t>((warps + 7) / 8, (int64_t)sm_count() * 8);
  cudaStream_t st = as_stream(stream);
  if (in_dtype == CSA_BF16)
    launch_k(csa::compress_index_keys_kernel<__nv_bfloat16>, blocks, 256, 0, st, (const __nv_bfloat16*)C_a,
             (const __nv_bfloat16*)C_b, (const __nv_bfloat16*)Z_a, (const __nv_bfloat16*)Z_b,
             (const __nv_bfloat16*)prev_Cb, (const __nv_bfloat16*)prev_Zb, B, L, hadamard ? 1 : 0, n_cap, pos0,
             (__nv_bfloat16*)kI, k8, k_scale);
  else
    launch_k(csa::compress_index_keys_kernel<float>, blocks, 256, 0, st, (const float*)C_a, (const float*)C_b,
             (const float*)Z_a, (const float*)Z_b, (const float*)prev_Cb, (const float*)prev_Zb, B, L,
             hadamard ? 1 : 0, n_cap, pos0, (__nv_bfloat16*)kI, k8, k_scale);
  return launch_status();
}

int csa_quantize_e4m3(const void* x, int x_dtype, int64_t rows, int cols, uint8_t* codes, float* scale,
                      void* stream) {
  if (rows < 0 || cols <= 0) return CSA_ERR_INVALID;
  if (x_dtype != CSA_F32 && x_dtype != CSA_BF16) return CSA_ERR_INVALID;
  if (rows == 0) return CSA_OK;
  if (!x || !codes || !scale) return CSA_ERR_INVALID;
  const int64_t blocks64 = (rows + 7) / 8;
  const unsigned blocks = (unsigned)std::min<int64_t>(blocks64, (int64_t)sm_count() * 32);
  cudaStream_t st = as_stream(stream);
  if (x_dtype == CSA_BF16)
    launch_k(csa::quantize_e4m3_kernel<__nv_bfloat16>, blocks, 256, 0, st, (const __nv_bfloat16*)x, rows, cols, codes, scale);
  else
    launch_k(csa::quantize_e4m3_kernel<float>, blocks, 256, 0, st, (const float*)x, rows, cols, codes, scale);
  return launch_status();
}

int csa_quantize_e4m3_hadamard(const void* x, int x_dtype, int64_t rows, int cols, uint8_t* codes, float* scale,
                               void* stream) {
  if (rows < 0 || !(cols == 32 || cols == 64 || cols == 128 || cols == 256)) return CSA_ERR_INVALID;
  if (x_dtype != CSA_F32 && x_dtype != CSA_BF16) return CSA_ERR_INVALID;
  if (rows == 0) return CSA_OK;
  if (!x || !codes || !scale) return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(codes)) & 15) return CSA_ERR_INVALID;
  cudaStream_t st = as_stream(stream);
  // 8 warps per block, a warp takes HadamardCfg<N>::RPW rows per pass; two blocks per SM
#define CSA_LAUNCH_HAD(T, N)                                                                              \
  do {                                                                                                    \
    const int64_t rpb = 8 * csa::HadamardCfg<N>::RPW;                                                     \
    const unsigned blocks = (unsigned)std::min<int64_t>((rows + rpb - 1) / rpb, (int64_t)sm_count() * 2); \
    launch_k(csa::hadamard_quantize_e4m3_kernel<T, N>, blocks, 256, 0, st, (const T*)x, rows, codes, scale); \
  } while (0)
#define CSA_LAUNCH_HAD_COLS(T)            \
  switch (cols) {                         \
    case 32: CSA_LAUNCH_HAD(T, 32); break;   \
    case 64: CSA_LAUNCH_HAD(T, 64); break;   \
    case 128: CSA_LAUNCH_HAD(T, 128); break; \
    default: CSA_LAUNCH_HAD(T, 256); break;  \
  }
  if (x_dtype == CSA_BF16) {
    CSA_LAUNCH_HAD_COLS(__nv_bfloat16)
  } else {
    CSA_LAUNCH_HAD_COLS(float)
  }
#undef CSA_LAUNCH_HAD_COLS
#undef CSA_LAUNCH_HAD
  return launch_status();
}

static int quantize_mxfp4_impl(const void* x, int x_dtype, int64_t rows, int cols, int hadamard, uint8_t* codes,
                               uint8_t* scales, int64_t rpb, void* stream);

int csa_quantize_mxfp4(const void* x, int x_dtype, int64_t rows, int cols, int hadamard, uint8_t* codes,
                       uint8_t* scales, void* stream) {
  return quantize_mxfp4_impl(x, x_dtype, rows, cols, hadamard, codes, scales, 0, stream);
}

size_t csa_mxfp4_sf128_bytes(int64_t batches, int64_t rows_per_batch) {
  if (batches <= 0 || rows_per_batch <= 0) return 0;
  return (size_t)batches * (size_t)((rows_per_batch + 127) / 128) * 512;
}

int csa_quantize_mxfp4_sf128(const void* x, int x_dtype, int64_t batches, int64_t rows_per_batch, int hadamard,
                             uint8_t* codes, uint8_t* sf, void* stream) {
  if (batches < 0 || rows_per_batch < 0) return CSA_ERR_INVALID;
  if (batches == 0 || rows_per_batch == 0) return CSA_OK;
  if (!sf || (reinterpret_cast<uintptr_t>(sf) & 15)) return CSA_ERR_INVALID;
  return quantize_mxfp4_impl(x, x_dtype, batches * rows_per_batch, 128, hadamard, codes, sf, rows_per_batch, stream);
}

static int quantize_mxfp4_impl(const void* x, int x_dtype, int64_t rows, int cols, int hadamard, uint8_t* codes,
                               uint8_t* scales, int64_t rpb, void* stream) {
  if (rows < 0 || !(cols == 32 || cols == 64 || cols == 128 || cols == 256)) return CSA_ERR_INVALID;
  if (x_dtype != CSA_F32 && x_dtype != CSA_BF16) return CSA_ERR_INVALID;
  if (rows == 0) return CSA_OK;
  if (!x || !codes || !scales) return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(codes)) & 15) return CSA_ERR_INVALID;
  cudaStream_t st = as_stream(stream);
#define CSA_LAUNCH_MX(T, N, ROT)                                                                              \
  do {                                                                                                        \
    const int64_t rows_pb = 8 * csa::HadamardCfg<N>::RPW;                                                     \
    const unsigned blocks = (unsigned)std::min<int64_t>((rows + rows_pb - 1) / rows_pb, (int64_t)sm_count() * 2); \
    launch_k(csa::quantize_mxfp4_kernel<T, N, ROT>, blocks, 256, 0, st, (const T*)x, rows, codes, scales, rpb); \
  } while (0)
#define CSA_LAUNCH_MX_ROT(T, N)        \
  do {                                 \
    if (hadamard) CSA_LAUNCH_MX(T, N, true); \
    else CSA_LAUNCH_MX(T, N, false);   \
  } while (0)
#define CSA_LAUNCH_MX_COLS(T)                  \
  switch (cols) {                              \
    case 32: CSA_LAUNCH_MX_ROT(T, 32); break;   \
    case 64: CSA_LAUNCH_MX_ROT(T, 64); break;   \
    case 128: CSA_LAUNCH_MX_ROT(T, 128); break; \
    default: CSA_LAUNCH_MX_ROT(T, 256); break;  \
  }
  if (x_dtype == CSA_BF16) {
    CSA_LAUNCH_MX_COLS(__nv_bfloat16)
  } else {
    CSA_LAUNCH_MX_COLS(float)
  }
#undef CSA_LAUNCH_MX_COLS
#undef CSA_LAUNCH_MX_ROT
#undef CSA_LAUNCH_MX
  return launch_status();
}

long long csa_kv8_entry_bytes(int D) { return D == csa::kKv8Dims ? (long long)csa::kKv8Bytes : 0; }

int csa_quantize_kv8(const void* kv, int64_t rows, int D, void* entries, void* stream) {
  if (rows < 0) return CSA_ERR_INVALID;
  if (D != csa::kKv8Dims) return CSA_ERR_UNSUPPORTED;
  if (rows == 0) return CSA_OK;
  if (!kv || !entries || !aligned16(kv) || !aligned16(entries)) return CSA_ERR_INVALID;
  const int64_t blocks64 = (rows + 7) / 8;
  const unsigned blocks = (unsigned)std::min<int64_t>(blocks64, (int64_t)sm_count() * 32);
  launch_k(csa::kv8_quantize_kernel, blocks, 256, 0, as_stream(stream), (const __nv_bfloat16*)kv, rows,
           (uint8_t*)entries);
  return launch_status();
}

// Parameters of index_tc_kernel for one call (scores written, no histogram, no candidates).
static IndexParams index_params(int mode, const float* q_scale, const float* w, const float* k_scale,
                                const int32_t* n_valid, float* scores, int B, int T, int64_t N) {
  const bool fp4 = mode == csa::kIdxMxfp4;
  IndexParams p;
  std::memset(&p, 0, sizeof(p));
  p.w = w;
  p.q_scale = mode == csa::kIdxE4m3 ? q_scale : nullptr;
  p.k_scale = mode == csa::kIdxE4m3 ? k_scale : nullptr;
  p.q_sf = fp4 ? reinterpret_cast<const uint8_t*>(q_scale) : nullptr;
  p.k_sf = fp4 ? reinterpret_cast<const uint8_t*>(k_scale) : nullptr;
  p.n_valid = n_valid;
  p.scores = scores;
  p.B = B;
  p.T = T;
  p.N = N;
  // queries per group: up to 4 (mxfp4: 2, so that a group's query scales are one atom)
  p.TQ = (T >= 4 && !fp4) ? 4 : (T >= 2 ? 2 : 1);
  return p;
}

// One launch of index_tc_kernel (emit: the candidate mode) over p's B x T queries and N keys.
static int launch_index_tc(const void* qI, const void* kI, int mode, IndexParams p, bool emit, cudaStream_t st) {
  const bool fp4 = mode == csa::kIdxMxfp4;
  const int B = p.B, T = p.T;
  const int64_t N = p.N;
  const int key_bytes = mode == csa::kIdxBf16 ? csa::IndexCfg<csa::kIdxBf16>::kKeyBytes
                        : mode == csa::kIdxE4m3 ? csa::IndexCfg<csa::kIdxE4m3>::kKeyBytes
                                                : csa::IndexCfg<csa::kIdxMxfp4>::kKeyBytes;
  const int qrow = mode == csa::kIdxBf16 ? 256 : (mode == csa::kIdxE4m3 ? 128 : 64);
  const int q_bytes = p.TQ * csa::kIdxHeads * qrow;
  const int fixed = 1024 + (q_bytes + 1023) / 1024 * 1024 + (fp4 ? 1024 : 0) +
                    csa::kIdxEpiWarps * p.TQ * csa::kIdxHeads * 4 + 8 * (4 + 2 * csa::kMaxAcc) +
                    csa::kKsRing * 32 * csa::kIdxEpiWarps * 4 + (p.hist ? 2 * csa::kHistBinsIdx * 4 : 0) +
                    (emit ? csa::kIdxEpiWarps * 12 * 4 : 0);
  if (emit && p.hist) return CSA_ERR_INVALID;      // (the two share their shared memory)
  p.stages = std::min(fp4 ? 16 : 12, (kSmemLimit - fixed) / (key_bytes + 16));
  if (p.stages < 2) return CSA_ERR_UNSUPPORTED;
  const int smem = fixed + p.stages * (key_bytes + 16);
  CUtensorMap kmap, qmap;
  const CUtensorMapDataType dt = mode == csa::kIdxBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const int es = mode == csa::kIdxBf16 ? 2 : 1;
  const uint32_t box0 = mode == csa::kIdxBf16 ? 64 : (fp4 ? 64 : 128);        // elements of one swizzle row
  const uint64_t inner = fp4 ? 64 : csa::kIdxDim;                             // elements per row in memory
  const CUtensorMapSwizzle swz = fp4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_map(&kmap, kI, dt, es, inner, (uint64_t)N, (uint64_t)B, box0, csa::kIdxTileKeys, swz) ||
      !make_map(&qmap, qI, dt, es, inner, (uint64_t)T * csa::kIdxHeads, (uint64_t)B, box0,
                (uint32_t)(p.TQ * csa::kIdxHeads), swz))
    return CSA_ERR_CUDA;
  const int QG = (T + p.TQ - 1) / p.TQ;
  const int64_t KT = (N + csa::kIdxTileKeys - 1) / csa::kIdxTileKeys;
  const int64_t items = (int64_t)B * QG * KT;
  const unsigned grid = (unsigned)std::min<int64_t>(items, sm_count());
  // candidate mode: 32-slot chunks when a CTA walks at least one whole row of key tiles
  // (a row then spans at most two CTAs: at most 2 x 16 warps x 31 unused slots); exact
  // reservations otherwise
  if (emit) p.cand_chunk = items / grid >= KT ? 32 : 1;
  auto go = [&](auto kernel) -> int {
    if (!set_smem(kernel, smem)) return CSA_ERR_CUDA;
    launch_k(kernel, grid, csa::kIdxThreads, smem, st, kmap, qmap, p);
    return launch_status();
  };
  if (emit) {
    if (mode == csa::kIdxE4m3) return go(csa::index_tc_kernel<csa::kIdxE4m3, true>);
    if (mode == csa::kIdxBf16) return go(csa::index_tc_kernel<csa::kIdxBf16, true>);
    return CSA_ERR_UNSUPPORTED;
  }
  if (mode == csa::kIdxE4m3) return go(csa::index_tc_kernel<csa::kIdxE4m3>);
  if (mode == csa::kIdxBf16) return go(csa::index_tc_kernel<csa::kIdxBf16>);
  return go(csa::index_tc_kernel<csa::kIdxMxfp4>);
}

int csa_index_scores(const void* qI, const float* q_scale, const float* w, const void* kI, const float* k_scale,
                     int dtype, const int32_t* n_valid, int B, int T, int64_t N, float* scores, void* select_ws,
                     void* stream) {
  return csa_index_scores_ex(qI, q_scale, w, kI, k_scale, dtype, n_valid, B, T, N, scores, select_ws, 0u, stream);
}

int csa_index_scores_ex(const void* qI, const float* q_scale, const float* w, const void* kI, const float* k_scale,
                        int dtype, const int32_t* n_valid, int B, int T, int64_t N, float* scores, void* select_ws,
                        unsigned flags, void* stream) {
  if (flags & ~(unsigned)CSA_INDEX_KEYS_READY) return CSA_ERR_INVALID;
  if (B < 0 || T < 0 || N < 0) return CSA_ERR_INVALID;
  if (dtype != CSA_F32 && dtype != CSA_BF16 && dtype != CSA_E4M3 && dtype != CSA_MXFP4) return CSA_ERR_INVALID;
  if (B == 0 || T == 0 || N == 0) return CSA_OK;
  if (!qI || !w || !kI || !n_valid || !scores) return CSA_ERR_INVALID;
  if ((dtype == CSA_E4M3 || dtype == CSA_MXFP4) && (!q_scale || !k_scale)) return CSA_ERR_INVALID;
  if (!aligned16(qI) || !aligned16(kI)) return CSA_ERR_INVALID;
  if (dtype == CSA_MXFP4 && (!aligned16(q_scale) || !aligned16(k_scale))) return CSA_ERR_INVALID;
  if (N >= (int64_t(1) << 31) || (int64_t)T * csa::kIdxHeads >= (int64_t(1) << 31) || B > 65535)
    return CSA_ERR_UNSUPPORTED;
  cudaStream_t st = as_stream(stream);
  if (dtype == CSA_F32) {
    if (T > 65535) return CSA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)((N + 63) / 64), (unsigned)T, (unsigned)B);
    if (!set_smem(csa::index_simt_kernel<float, false>, csa::kIdxSimtSmem)) return CSA_ERR_CUDA;
    launch_k(csa::index_simt_kernel<float, false>, grid, 256, csa::kIdxSimtSmem, st,
        (const float*)qI, w, (const float*)kI, n_valid, nullptr, 0, T, N, scores);
    return launch_status();
  }
  const int mode = dtype == CSA_BF16 ? csa::kIdxBf16 : (dtype == CSA_E4M3 ? csa::kIdxE4m3 : csa::kIdxMxfp4);
  IndexParams p = index_params(mode, q_scale, w, k_scale, n_valid, scores, B, T, N);
  if (select_ws != nullptr) {
    if (T != 1 || !aligned16(select_ws)) return CSA_ERR_INVALID;
    p.hist = reinterpret_cast<int*>(select_ws);
    p.hist_stride = csa::SelectWs::row_bytes(N) / 4;
  }
  p.keys_ready = (flags & CSA_INDEX_KEYS_READY) ? 1 : 0;
  return launch_index_tc(qI, kI, mode, p, false, st);
}

// ---------------------------------------------------------------- csa_index_topk
// Workspace pieces, each 256-byte aligned: sample keys, sample key scales, sample
// n_valid, sample scores, thresholds, candidate counts, failure count, candidate lists,
// and the score matrix the fallback writes.
struct IndexTopkWs {
  size_t kI_s, ks_s, nv_s, s_scores, thr, cnt, fail, cand, scores, total;
  int64_t Ns;
  int cap, r0;
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

static IndexTopkWs index_topk_layout(int B, int T, int64_t N, int k, int dtype) {
  IndexTopkWs L;
  const int64_t rows = (int64_t)B * T;
  L.Ns = (N + csa::kSampleStride - 1) / csa::kSampleStride;
  // the sampled rank: about 4k candidates expected, and never fewer than 48 samples above
  // the threshold, so that a row comes up short (fewer than k) only some 6 standard
  // deviations from the mean for keys in random order
  L.r0 = std::max(48, (4 * k + csa::kSampleStride - 1) / csa::kSampleStride);
  L.cap = std::min(csa::kCandCapMax, std::max(4096, 16 * k));
  const size_t row_bytes = dtype == CSA_BF16 ? 256 : 128;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  L.kI_s = take((size_t)B * L.Ns * row_bytes);
  L.ks_s = take(dtype == CSA_E4M3 ? (size_t)B * L.Ns * 4 : 0);
  L.nv_s = take((size_t)rows * 4);
  L.s_scores = take((size_t)rows * L.Ns * 4);
  L.thr = take((size_t)rows * 4);
  L.cnt = take((size_t)rows * 4);
  L.fail = take(16);
  L.cand = take((size_t)rows * L.cap * 8);
  L.scores = take((size_t)rows * N * 4);
  L.total = off;
  return L;
}

size_t csa_index_topk_workspace_size(int B, int T, int64_t N, int k, int dtype) {
  if (B <= 0 || T <= 0 || N <= 0 || k < 1) return 0;
  return index_topk_layout(B, T, N, k, dtype).total;
}

int csa_index_topk(const void* qI, const float* q_scale, const float* w, const void* kI, const float* k_scale,
                   int dtype, const int32_t* n_valid, int B, int T, int64_t N, int k, int32_t* idx,
                   int32_t* failed_rows, void* workspace, size_t ws_bytes, void* stream) {
  if (B < 0 || T < 0 || N < 0 || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (dtype != CSA_F32 && dtype != CSA_BF16 && dtype != CSA_E4M3 && dtype != CSA_MXFP4) return CSA_ERR_INVALID;
  if (dtype != CSA_BF16 && dtype != CSA_E4M3) return CSA_ERR_UNSUPPORTED;
  if (k > csa::kIndexTopkMaxK || N > csa::kRowSmemMax || B > 65535 ||
      (int64_t)T * csa::kIdxHeads >= (int64_t(1) << 31) || (int64_t)B * T > INT32_MAX)
    return CSA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return CSA_OK;
  cudaStream_t st = as_stream(stream);
  const int64_t rows = (int64_t)B * T;
  if (N == 0) {                                      // no keys: every row is -1
    if (!n_valid || !idx) return CSA_ERR_INVALID;
    if (failed_rows && cudaMemsetAsync(failed_rows, 0, sizeof(int32_t), st) != cudaSuccess) return CSA_ERR_CUDA;
    launch_k(csa::topk_row_kernel, (unsigned)rows, 1024, 4, st, (const float*)nullptr, n_valid, N, k, idx,
             (const int32_t*)nullptr, 0, (const int*)nullptr);
    return launch_status();
  }
  if (!qI || !w || !kI || !n_valid || !idx) return CSA_ERR_INVALID;
  if (dtype == CSA_E4M3 && (!q_scale || !k_scale)) return CSA_ERR_INVALID;
  if (!aligned16(qI) || !aligned16(kI)) return CSA_ERR_INVALID;
  const IndexTopkWs L = index_topk_layout(B, T, N, k, dtype);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return CSA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* kI_s = ws + L.kI_s;
  float* ks_s = dtype == CSA_E4M3 ? reinterpret_cast<float*>(ws + L.ks_s) : nullptr;
  int32_t* nv_s = reinterpret_cast<int32_t*>(ws + L.nv_s);
  float* s_scores = reinterpret_cast<float*>(ws + L.s_scores);
  uint32_t* thr = reinterpret_cast<uint32_t*>(ws + L.thr);
  int* cnt = reinterpret_cast<int*>(ws + L.cnt);
  int* fail = reinterpret_cast<int*>(ws + L.fail);
  auto* cand = reinterpret_cast<unsigned long long*>(ws + L.cand);
  float* scores = reinterpret_cast<float*>(ws + L.scores);
  const int mode = dtype == CSA_BF16 ? csa::kIdxBf16 : csa::kIdxE4m3;
  const int row_bytes = dtype == CSA_BF16 ? 256 : 128;
  // 1. the key sample and its n_valid
  {
    const int64_t work = std::max<int64_t>((int64_t)B * L.Ns * (row_bytes / 16), rows);
    const unsigned blocks = (unsigned)std::min<int64_t>((work + 255) / 256, (int64_t)sm_count() * 8);
    launch_k(csa::sample_keys_kernel, blocks, 256, 0, st, static_cast<const uint8_t*>(kI), k_scale, B, N, L.Ns,
             row_bytes, kI_s, ks_s, n_valid, rows, nv_s);
    int rc = launch_status();
    if (rc != CSA_OK) return rc;
  }
  // 2. the sample's scores
  int rc = launch_index_tc(qI, kI_s, mode, index_params(mode, q_scale, w, ks_s, nv_s, s_scores, B, T, L.Ns), false,
                           st);
  if (rc != CSA_OK) return rc;
  // 3. per-row thresholds (zeroes the candidate counts and the failure counts)
  {
    const int smem = (int)(L.Ns * 4);
    if (!set_smem(csa::cand_threshold_kernel, std::max(smem, 4))) return CSA_ERR_CUDA;
    launch_k(csa::cand_threshold_kernel, (unsigned)rows, 256, std::max(smem, 4), st, (const float*)s_scores, L.Ns,
             n_valid, N, k, L.r0, thr, cnt, fail, failed_rows);
    rc = launch_status();
    if (rc != CSA_OK) return rc;
  }
  // 4. every key scored; the scores at or above their row's threshold become candidates
  {
    IndexParams p = index_params(mode, q_scale, w, k_scale, n_valid, nullptr, B, T, N);
    p.thr = thr;
    p.cand_cnt = cnt;
    p.cand = cand;
    p.cand_cap = L.cap;
    rc = launch_index_tc(qI, kI, mode, p, true, st);
    if (rc != CSA_OK) return rc;
  }
  // 5. the exact top-k of each row's candidates; rows that cannot be settled are counted
  {
    const int smem = L.cap * 8 + (int)((N + 31) / 32) * 4;
    if (!set_smem(csa::cand_select_kernel, smem)) return CSA_ERR_CUDA;
    launch_k(csa::cand_select_kernel, (unsigned)rows, 256, smem, st, (const unsigned long long*)cand,
             (const int*)cnt, L.cap, n_valid, N, k, idx, fail, failed_rows);
    rc = launch_status();
    if (rc != CSA_OK) return rc;
  }
  // 6. the fallback, gated on the failure count: every row's scores, then the row top-k
  {
    IndexParams p = index_params(mode, q_scale, w, k_scale, n_valid, scores, B, T, N);
    p.gate = fail;
    rc = launch_index_tc(qI, kI, mode, p, false, st);
    if (rc != CSA_OK) return rc;
    const int smem = (int)(N * 4) + (N >= csa::kRowFastMin ? csa::kRowCand * 8 : 0);
    if (!set_smem(csa::topk_row_kernel, smem)) return CSA_ERR_CUDA;
    launch_k(csa::topk_row_kernel, (unsigned)rows, 1024, smem, st, (const float*)scores, n_valid, N, k, idx,
             (const int32_t*)nullptr, N >= csa::kRowFastMin ? 1 : 0, (const int*)fail);
    return launch_status();
  }
}

int csa_index_rerank(const void* qI, const float* w, const void* kI, int dtype, const int32_t* cand, int kc, int B,
                     int T, int64_t N, int k, float* cand_scores, int32_t* idx, void* stream) {
  if (B < 0 || T < 0 || N < 0 || k < 1 || k > CSA_MAX_TOPK || kc < k || kc > csa::kRowSmemMax)
    return CSA_ERR_INVALID;
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_ERR_INVALID;
  if (B == 0 || T == 0) return CSA_OK;
  if (!qI || !w || !kI || !cand || !cand_scores || !idx) return CSA_ERR_INVALID;
  if (!aligned16(qI) || !aligned16(kI)) return CSA_ERR_INVALID;
  if (T > 65535 || B > 65535) return CSA_ERR_UNSUPPORTED;
  cudaStream_t st = as_stream(stream);
  dim3 grid((unsigned)((kc + 63) / 64), (unsigned)T, (unsigned)B);
  if (dtype == CSA_BF16) {
    if (!set_smem(csa::index_simt_kernel<__nv_bfloat16, true>, csa::kIdxSimtSmem)) return CSA_ERR_CUDA;
    launch_k(csa::index_simt_kernel<__nv_bfloat16, true>, grid, 256, csa::kIdxSimtSmem, st, 
        (const __nv_bfloat16*)qI, w, (const __nv_bfloat16*)kI, nullptr, cand, kc, T, N, cand_scores);
  } else {
    if (!set_smem(csa::index_simt_kernel<float, true>, csa::kIdxSimtSmem)) return CSA_ERR_CUDA;
    launch_k(csa::index_simt_kernel<float, true>, grid, 256, csa::kIdxSimtSmem, st, 
        (const float*)qI, w, (const float*)kI, nullptr, cand, kc, T, N, cand_scores);
  }
  int rc = launch_status();
  if (rc != CSA_OK) return rc;
  const int smem = kc * 4;
  if (!set_smem(csa::topk_row_kernel, std::max(smem, 4))) return CSA_ERR_CUDA;
  launch_k(csa::topk_row_kernel, (unsigned)((int64_t)B * T), 1024, smem, st, cand_scores, nullptr, kc, k, idx, cand, 0,
           (const int*)nullptr);
  return launch_status();
}

static bool topk_long_path(int B, int T, int64_t N) {
  const int64_t rows = (int64_t)B * T;
  return N > csa::kRowSmemMax || (rows < 74 && N >= 4 * csa::kChunk);
}

size_t csa_topk_workspace_size(int B, int T, int64_t N, int k) {
  (void)k;
  if (B <= 0 || T <= 0 || N <= 0) return 0;
  if (!topk_long_path(B, T, N)) return 0;
  return (size_t)B * T * (size_t)csa::TopkWs::row_bytes(N);
}

// Checks of csa_topk's arguments other than the workspace: CSA_OK, or the status to
// return before anything is enqueued.
static int topk_check(const float* scores, const int32_t* n_valid, int B, int T, int64_t N, int k,
                      const int32_t* idx) {
  if (B < 0 || T < 0 || N < 0 || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (N > (int64_t(1) << 20)) return CSA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return CSA_OK;
  if (!idx || !n_valid || (N > 0 && !scores)) return CSA_ERR_INVALID;
  const int64_t rows = (int64_t)B * T;
  if (rows > 65535 && topk_long_path(B, T, N)) return CSA_ERR_UNSUPPORTED;
  if (rows > (int64_t(1) << 31) - 1) return CSA_ERR_UNSUPPORTED;
  return CSA_OK;
}

int csa_topk(const float* scores, const int32_t* n_valid, int B, int T, int64_t N, int k, int32_t* idx,
             void* workspace, size_t ws_bytes, void* stream) {
  const int chk = topk_check(scores, n_valid, B, T, N, k, idx);
  if (chk != CSA_OK || B == 0 || T == 0) return chk;
  const int64_t rows = (int64_t)B * T;
  cudaStream_t st = as_stream(stream);
  if (!topk_long_path(B, T, N)) {
    // keys, then (rows of kRowFastMin or more) the sampled path's candidates
    const int smem = (int)std::max<int64_t>(4, std::min<int64_t>(N, csa::kRowSmemMax) * 4) +
                     (N >= csa::kRowFastMin ? csa::kRowCand * 8 : 0);
    if (!set_smem(csa::topk_row_kernel, smem)) return CSA_ERR_CUDA;
    launch_k(csa::topk_row_kernel, (unsigned)rows, 1024, smem, st, scores, n_valid, N, k, idx, nullptr,
             N >= csa::kRowFastMin ? 1 : 0, (const int*)nullptr);
    return launch_status();
  }
  const size_t need = csa_topk_workspace_size(B, T, N, k);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return CSA_ERR_INVALID;
  dim3 grid((unsigned)((N + csa::kChunk - 1) / csa::kChunk), (unsigned)rows);
  launch_k(csa::topk_hist_kernel, grid, 512, 0, st, scores, n_valid, N, k, static_cast<uint8_t*>(workspace),
           (int64_t)csa::TopkWs::row_bytes(N));
  int rc = launch_status();
  if (rc != CSA_OK) return rc;
  const int gsmem = 2 * csa::kCandSmem * 4;
  if (!set_smem(csa::topk_gather_select_kernel, gsmem)) return CSA_ERR_CUDA;
  launch_k(csa::topk_gather_select_kernel, grid, 1024, gsmem, st, scores, n_valid, N, k, idx,
                                                            static_cast<uint8_t*>(workspace));
  return launch_status();
}

size_t csa_select_workspace_size(int B, int64_t N) {
  if (B <= 0 || N <= 0) return 0;
  return (size_t)B * (size_t)csa::SelectWs::row_bytes(N);
}

int csa_score_histogram(const float* scores, const int32_t* n_valid, int B, int64_t N, void* workspace,
                        size_t ws_bytes, void* stream) {
  if (B < 0 || N < 0) return CSA_ERR_INVALID;
  if (N > csa::kSelMaxN || B > 65535) return CSA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return CSA_OK;
  if (!scores || !n_valid || !workspace || ws_bytes < csa_select_workspace_size(B, N) || !aligned16(workspace))
    return CSA_ERR_INVALID;
  dim3 grid((unsigned)((N + csa::kChunk - 1) / csa::kChunk), (unsigned)B);
  // k = 0: every row with a valid entry is histogrammed
  launch_k(csa::topk_hist_kernel, grid, 512, 0, as_stream(stream), scores, n_valid, N, 0,
           static_cast<uint8_t*>(workspace), (int64_t)csa::SelectWs::row_bytes(N));
  return launch_status();
}

int csa_topk_select(const float* scores, const int32_t* n_valid, int B, int64_t N, int k, int kc, const void* qI,
                    const float* w, const void* kI, int dtype, int32_t* idx, float* idx_scores, void* workspace,
                    size_t ws_bytes, void* stream) {
  if (B < 0 || N < 0 || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (N > csa::kSelMaxN || B > 65535) return CSA_ERR_UNSUPPORTED;
  const bool rescore = qI != nullptr;
  if (rescore && (kc < k || !w || !kI || (dtype != CSA_F32 && dtype != CSA_BF16))) return CSA_ERR_INVALID;
  if (rescore && (!aligned16(qI) || !aligned16(kI))) return CSA_ERR_INVALID;
  if (B == 0) return CSA_OK;
  if (!idx || !n_valid || (N > 0 && !scores)) return CSA_ERR_INVALID;
  const size_t need = csa_select_workspace_size(B, N);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return CSA_ERR_INVALID;
  if (N == 0) {
    launch_k(csa::topk_row_kernel, (unsigned)B, 1024, 4, as_stream(stream), scores, n_valid, N, k, idx, nullptr, 0,
             (const int*)nullptr);
    if (idx_scores)
      launch_k(csa::fill_f32_kernel, (unsigned)std::min<int64_t>(((int64_t)B * k + 255) / 256, 1024), 256, 0,
               as_stream(stream), idx_scores, (int64_t)B * k, -INFINITY);
    return launch_status();
  }
  // chunks: one wave (at most one CTA per SM over all rows), at least 512 entries each,
  // at most kSelMaxChunkLen (the chunk's candidate list lives in shared memory)
  const int sms = sm_count();
  int64_t nchunks = std::max<int64_t>(1, std::min<int64_t>((N + 511) / 512, std::max(1, sms / std::max(B, 1))));
  nchunks = std::max<int64_t>(nchunks, (N + csa::kSelMaxChunkLen - 1) / csa::kSelMaxChunkLen);
  nchunks = std::min<int64_t>(nchunks, csa::kSelMaxChunks);
  int chunk = (int)(((N + nchunks - 1) / nchunks + 255) / 256 * 256);
  nchunks = (N + chunk - 1) / chunk;
  const bool tc = rescore && dtype == CSA_BF16;
  const int phase3 = csa::kSelTileBytes + csa::kSelQBytes + chunk * 8 + 64 * 4 +
                     (rescore && !tc ? (64 * 129 + csa::kSelKeyBatch * 128) * 4 : 0);
  // last CTA: staged candidates + chunk table, or (overflow) the bucketed selection
  const int phase4 = (int)std::max<int64_t>(2 * csa::kSelCandSmem * 4 + 2 * csa::kSelMaxChunks * 4 +
                                                csa::kSelPivot * 4,
                                            4 * CSA_MAX_TOPK * 4 + (nchunks + 1) * 4);
  const int smem = 1024 + std::max(phase3, phase4);
  cudaStream_t st = as_stream(stream);
  dim3 grid((unsigned)nchunks, (unsigned)B);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (!rescore) {
    if (!set_smem(csa::topk_select_kernel<false, float>, smem)) return CSA_ERR_CUDA;
    launch_k(csa::topk_select_kernel<false, float>, grid, csa::kSelThreads, smem, st, scores, n_valid, N, k, k,
             chunk, (const float*)nullptr, w, (const float*)nullptr, idx, idx_scores, ws);
  } else if (dtype == CSA_BF16) {
    if (!set_smem(csa::topk_select_kernel<true, __nv_bfloat16>, smem)) return CSA_ERR_CUDA;
    launch_k(csa::topk_select_kernel<true, __nv_bfloat16>, grid, csa::kSelThreads, smem, st, scores, n_valid, N,
             k, kc, chunk, (const __nv_bfloat16*)qI, w, (const __nv_bfloat16*)kI, idx, idx_scores, ws);
  } else {
    if (!set_smem(csa::topk_select_kernel<true, float>, smem)) return CSA_ERR_CUDA;
    launch_k(csa::topk_select_kernel<true, float>, grid, csa::kSelThreads, smem, st, scores, n_valid, N, k, kc,
             chunk, (const float*)qI, w, (const float*)kI, idx, idx_scores, ws);
  }
  return launch_status();
}

size_t csa_attn_workspace_size(int B, int T, int H, int D, int64_t rows_per_query, int dtype) {
  if (B <= 0 || T <= 0 || H <= 0 || D <= 0 || rows_per_query < 0) return 0;
  return attn_ws_bytes(B, T, H, D, rows_per_query, dtype);
}

static int sparse_attn_impl(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                            const int64_t* q_pos, const float* sink, const int32_t* idx, int k, float scale,
                            double theta, int B, int T, int H, int D, int64_t N, int dtype, void* out,
                            void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_attn_common(q, kv, swa_kv, swa_pos0, W, q_pos, sink, scale, B, T, H, D, N, dtype, out);
  if (rc != CSA_OK) return rc;
  if (theta != 0.0 && (!(theta > 1.0) || D < csa::kRopeDims || dtype == CSA_BF16_KV8))
    return !(theta > 1.0) ? CSA_ERR_INVALID : CSA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return rc;
  if (k < 0 || (k > 0 && !idx)) return CSA_ERR_INVALID;
  AttnParams p{};
  p.q = q; p.kv = kv; p.swa = swa_kv; p.swa_pos0 = swa_pos0; p.q_pos = q_pos; p.sink = sink;
  p.idx = idx; p.sparse = 1; p.out = out; p.scale = scale; p.rope_theta = theta;
  if (theta > 0.0) p.rope_freq = csa::rope_freqs(theta);
  p.B = B; p.T = T; p.H = H; p.D = D; p.W = W; p.k = k; p.ratio = 1; p.N = N; p.nsplit = 1;
  // (KV8: the memory rows start at a tile boundary, at most 31 rows after the SWA rows)
  const int64_t max_rows = (int64_t)std::min(W, CSA_SWA_WINDOW) + k + (dtype == CSA_BF16_KV8 ? 31 : 0);
  return run_attn(p, dtype, workspace, ws_bytes, max_rows, as_stream(stream));
}

static int hca_attn_impl(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                         const int64_t* q_pos, const float* sink, int ratio, float scale, double theta, int B, int T,
                         int H, int D, int64_t N, int dtype, void* out, void* workspace, size_t ws_bytes,
                         void* stream) {
  int rc = check_attn_common(q, kv, swa_kv, swa_pos0, W, q_pos, sink, scale, B, T, H, D, N, dtype, out);
  if (rc != CSA_OK) return rc;
  if (theta != 0.0 && (!(theta > 1.0) || D < csa::kRopeDims || dtype == CSA_BF16_KV8))
    return !(theta > 1.0) ? CSA_ERR_INVALID : CSA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return rc;
  if (ratio < 1) return CSA_ERR_INVALID;
  AttnParams p{};
  p.q = q; p.kv = kv; p.swa = swa_kv; p.swa_pos0 = swa_pos0; p.q_pos = q_pos; p.sink = sink;
  p.idx = nullptr; p.sparse = 0; p.out = out; p.scale = scale; p.rope_theta = theta;
  if (theta > 0.0) p.rope_freq = csa::rope_freqs(theta);
  p.B = B; p.T = T; p.H = H; p.D = D; p.W = W; p.k = 0; p.ratio = ratio; p.N = N; p.nsplit = 1;
  const int64_t max_rows = (int64_t)std::min(W, CSA_SWA_WINDOW) + N + (dtype == CSA_BF16_KV8 ? 31 : 0);
  return run_attn(p, dtype, workspace, ws_bytes, max_rows, as_stream(stream));
}

int sparse_attn(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                const int64_t* q_pos, const float* sink, const int32_t* idx, int k, float scale, int B, int T,
                int H, int D, int64_t N, int dtype, void* out, void* workspace, size_t ws_bytes, void* stream) {
  return sparse_attn_impl(q, kv, swa_kv, swa_pos0, W, q_pos, sink, idx, k, scale, 0.0, B, T, H, D, N, dtype, out,
                          workspace, ws_bytes, stream);
}

int sparse_attn_rope(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                     const int64_t* q_pos, const float* sink, const int32_t* idx, int k, float scale,
                     double rope_theta, int B, int T, int H, int D, int64_t N, int dtype, void* out, void* workspace,
                     size_t ws_bytes, void* stream) {
  if (!(rope_theta > 1.0)) return CSA_ERR_INVALID;
  return sparse_attn_impl(q, kv, swa_kv, swa_pos0, W, q_pos, sink, idx, k, scale, rope_theta, B, T, H, D, N, dtype,
                          out, workspace, ws_bytes, stream);
}

int hca_attn(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
             const int64_t* q_pos, const float* sink, int ratio, float scale, int B, int T, int H, int D, int64_t N,
             int dtype, void* out, void* workspace, size_t ws_bytes, void* stream) {
  return hca_attn_impl(q, kv, swa_kv, swa_pos0, W, q_pos, sink, ratio, scale, 0.0, B, T, H, D, N, dtype, out,
                       workspace, ws_bytes, stream);
}

int hca_attn_rope(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                  const int64_t* q_pos, const float* sink, int ratio, float scale, double rope_theta, int B, int T,
                  int H, int D, int64_t N, int dtype, void* out, void* workspace, size_t ws_bytes, void* stream) {
  if (!(rope_theta > 1.0)) return CSA_ERR_INVALID;
  return hca_attn_impl(q, kv, swa_kv, swa_pos0, W, q_pos, sink, ratio, scale, rope_theta, B, T, H, D, N, dtype, out,
                       workspace, ws_bytes, stream);
}

int csa_rope(const void* x, int dtype, int B, int64_t R, int D, const int64_t* pos_base, int64_t stride,
             double theta, int inverse, void* out, void* stream) {
  if (B < 0 || R < 0 || D < csa::kRopeDims || D % 2 != 0 || !(theta > 1.0)) return CSA_ERR_INVALID;
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_ERR_INVALID;
  if (B == 0 || R == 0) return CSA_OK;
  if (!x || !out) return CSA_ERR_INVALID;
  const int64_t total = (int64_t)B * R * (csa::kRopeDims / 2);
  const unsigned blocks = (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
  cudaStream_t st = as_stream(stream);
  if (dtype == CSA_BF16)
    launch_k(csa::rope_rows_kernel<__nv_bfloat16>, blocks, 256, 0, st, (const __nv_bfloat16*)x, (int64_t)B, R, D,
             pos_base, stride, csa::rope_freqs(theta), inverse ? 1 : 0, (__nv_bfloat16*)out);
  else
    launch_k(csa::rope_rows_kernel<float>, blocks, 256, 0, st, (const float*)x, (int64_t)B, R, D, pos_base, stride,
             csa::rope_freqs(theta), inverse ? 1 : 0, (float*)out);
  return launch_status();
}

int sparse_attn_partial(const void* q, const void* kv, const void* swa_kv, const int64_t* swa_pos0, int W,
                        const int64_t* q_pos, const int32_t* idx, int k, float scale, int B, int T, int H, int D,
                        int64_t N, int dtype, void* out, float* ml, void* workspace, size_t ws_bytes, void* stream) {
  if (dtype != CSA_BF16 && dtype != CSA_BF16_KV8) return dtype == CSA_F32 ? CSA_ERR_UNSUPPORTED : CSA_ERR_INVALID;
  // (the sink is not used here: pass a non-null stand-in to the common checks)
  static const float no_sink = 0.f;
  int rc = check_attn_common(q, kv, swa_kv, swa_pos0, W, q_pos, &no_sink, scale, B, T, H, D, N, dtype, out);
  if (rc != CSA_OK || B == 0 || T == 0) return rc;
  if (k < 0 || (k > 0 && !idx) || !ml || (reinterpret_cast<uintptr_t>(ml) & 7)) return CSA_ERR_INVALID;
  AttnParams p{};
  p.q = q; p.kv = kv; p.swa = swa_kv; p.swa_pos0 = swa_pos0; p.q_pos = q_pos; p.sink = nullptr;
  p.idx = idx; p.sparse = 1; p.out = out; p.scale = scale; p.ml = ml;
  p.B = B; p.T = T; p.H = H; p.D = D; p.W = W; p.k = k; p.ratio = 1; p.N = N; p.nsplit = 1;
  const int64_t max_rows = (int64_t)std::min(W, CSA_SWA_WINDOW) + k + (dtype == CSA_BF16_KV8 ? 31 : 0);
  return run_attn(p, dtype, workspace, ws_bytes, max_rows, as_stream(stream));
}

int csa_attn_combine(const void* parts, int64_t part_stride, const float* ml, int64_t ml_stride, const float* sink,
                     int G, int B, int T, int H, int D, void* out, void* stream) {
  if (G < 1 || G > CSA_MAX_SHARDS || B < 0 || T < 0 || H <= 0 || D <= 0 || D % 8 != 0) return CSA_ERR_INVALID;
  const int64_t rows = (int64_t)B * T * H;
  if (rows == 0) return CSA_OK;
  if (!parts || !ml || !sink || !out || !aligned16(parts) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(ml) & 7) || (G > 1 && ((part_stride & 15) || (ml_stride & 7))) ||
      (G > 1 && (part_stride < rows * D * 2 || ml_stride < rows * 8)))
    return CSA_ERR_INVALID;
  const int64_t blocks = (rows + 7) / 8;
  if (blocks > INT32_MAX) return CSA_ERR_UNSUPPORTED;
  launch_k(csa::attn_combine_kernel, (unsigned)blocks, 256, 0, as_stream(stream), (const uint8_t*)parts, part_stride,
           (const uint8_t*)ml, ml_stride, sink, G, rows, H, D, (__nv_bfloat16*)out);
  return launch_status();
}

size_t csa_shard_select_workspace_size(int G, int B, int k) {
  if (G < 1 || B < 1 || k < 1) return 0;
  return (size_t)G * B * k * 8;
}

int csa_shard_pack(const float* scores, const int32_t* loc, int64_t n, int64_t ns, int64_t lo, void* pairs,
                   void* stream) {
  if (n < 0 || ns < 0 || lo < 0 || lo + ns > INT32_MAX) return CSA_ERR_INVALID;
  if (n == 0) return CSA_OK;
  if (!scores || !loc || !pairs || (reinterpret_cast<uintptr_t>(pairs) & 7)) return CSA_ERR_INVALID;
  launch_k(csa::shard_pack_kernel, (unsigned)std::min<int64_t>((n + 255) / 256, (int64_t)sm_count() * 8), 256, 0,
           as_stream(stream), scores, loc, n, ns, lo, (csa::ShardPair*)pairs);
  return launch_status();
}

int csa_shard_select(const void* pairs, int G, int B, int k, int32_t* idx, void* workspace, size_t ws_bytes,
                     void* stream) {
  if (G < 1 || G > CSA_MAX_SHARDS || B < 0 || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (B == 0) return CSA_OK;
  const int64_t n = (int64_t)G * k;
  if (n > csa::kRowSmemMax) return CSA_ERR_UNSUPPORTED;
  if (!pairs || !idx || !workspace || ws_bytes < csa_shard_select_workspace_size(G, B, k) ||
      (reinterpret_cast<uintptr_t>(pairs) & 7))
    return CSA_ERR_INVALID;
  cudaStream_t st = as_stream(stream);
  float* row_scores = static_cast<float*>(workspace);
  int32_t* row_idx = reinterpret_cast<int32_t*>(row_scores + (size_t)B * n);
  const int64_t total = (int64_t)B * n;
  launch_k(csa::shard_gather_kernel, (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8), 256, 0,
           st, (const csa::ShardPair*)pairs, G, B, k, row_scores, row_idx);
  const int smem = (int)std::max<int64_t>(4, n * 4);
  if (!set_smem(csa::topk_row_kernel, smem)) return CSA_ERR_CUDA;
  launch_k(csa::topk_row_kernel, (unsigned)B, 1024, smem, st, (const float*)row_scores, (const int32_t*)nullptr, n, k,
           idx, (const int32_t*)row_idx, 0, (const int*)nullptr);
  return launch_status();
}

int csa_shard_remap(const int32_t* in, int64_t n, int64_t lo, int64_t hi, int64_t add, int32_t* out, void* stream) {
  if (n < 0 || lo < 0 || hi < lo || hi > INT32_MAX || add < 0 || hi - lo + add > INT32_MAX) return CSA_ERR_INVALID;
  if (n == 0) return CSA_OK;
  if (!in || !out) return CSA_ERR_INVALID;
  launch_k(csa::shard_remap_kernel, (unsigned)std::min<int64_t>((n + 255) / 256, (int64_t)sm_count() * 8), 256, 0,
           as_stream(stream), in, n, lo, hi, add, out);
  return launch_status();
}

unsigned long long csa_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ------------------------------------------------------------------ allocation-free top-k
// Scratch for csa_topk_noalloc: a file-scope device array, so callers that cannot
// allocate device memory still get the chunked top-k.  Every GPU that loads this
// library holds it until the process exits.
static __device__ __align__(256) uint8_t g_topk_noalloc_scratch[CSA_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array in the current device's context.  In host code
// the array's name is only a host-side stand-in, so the address is looked up with the
// device current (cudaGetSymbolAddress).  It is looked up on every call, not cached: after
// a cudaDeviceReset the module is loaded again into a new context and the array may
// move.
void* noalloc_scratch_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_topk_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}
}  // namespace

extern "C" {

int csa_topk_noalloc(const float* scores, const int32_t* n_valid, int B, int T, int64_t N, int k, int32_t* idx,
                     void* stream) {
  // every argument is checked before the shared array is touched: a rejected call
  // enqueues nothing
  const int chk = topk_check(scores, n_valid, B, T, N, k, idx);
  if (chk != CSA_OK || B == 0 || T == 0) return chk;
  const size_t need = csa_topk_workspace_size(B, T, N, k);
  if (need == 0) return csa_topk(scores, n_valid, B, T, N, k, idx, nullptr, 0, stream);   // needs no scratch
  if (need > (size_t)CSA_NOALLOC_SCRATCH_BYTES) return CSA_ERR_UNSUPPORTED;                 // beyond the array
  void* scratch = noalloc_scratch_ptr();
  if (scratch == nullptr) return CSA_ERR_CUDA;
  // A completed call leaves the part of the array it used zero-filled, and the
  // chunked top-k needs exactly that at its start; a call cut short, or one that
  // overlapped another on the GPU, would not leave it so.  Clearing the `need`
  // bytes here makes every call independent of what the previous one left behind.
  if (cudaMemsetAsync(scratch, 0, need, as_stream(stream)) != cudaSuccess) return CSA_ERR_CUDA;
  return csa_topk(scores, n_valid, B, T, N, k, idx, scratch, need, stream);
}

int csa_poll_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, csa::g_status, sizeof(int)) != cudaSuccess) return CSA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(csa::g_status, &zero, sizeof(int)) != cudaSuccess) return CSA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
