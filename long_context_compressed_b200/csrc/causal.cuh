// causal.cuh -- visible compressed entries of each query.
//
// "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §6: a query at absolute position t
// attends to compressed entry i only once that entry's block of m raw tokens is
// complete, (i + 1) m <= t + 1, i.e. to entries 0 .. floor((t + 1) / m) - 1.  When
// a GPU holds only the contiguous range [lo, hi) of a sequence's entries (the
// sharded decode), its local entries 0 .. n - 1 are visible with
// n = clamp(floor((t + 1) / m) - lo, 0, hi - lo).
#pragma once
#include "ptx.cuh"

namespace csa {

__global__ void __launch_bounds__(256) n_valid_kernel(const int64_t* __restrict__ q_pos, int64_t count, int ratio,
                                                      int64_t lo, int64_t hi, int32_t* __restrict__ out) {
  griddep_sync();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = q_pos[i];
    int64_t n = t >= 0 ? (t + 1) / ratio - lo : 0;   // complete blocks, as local entries
    n = n < 0 ? 0 : (n > hi - lo ? hi - lo : n);
    out[i] = (int32_t)n;
  }
}

// Failure-detection check of the bounded waits: one thread waits on an mbarrier that
// completes only if `complete` is set, with a limit of limit_ns nanoseconds; a wait
// that runs out records CSA_ERR_TIMEOUT in the status word and the kernel returns.
__global__ void __launch_bounds__(32) bounded_wait_kernel(int complete, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  griddep_sync();
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (complete) mbar_arrive(&bar);
  mbar_wait_for(&bar, 0, limit_ns);
}

}  // namespace csa
