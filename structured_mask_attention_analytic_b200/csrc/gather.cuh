// Device helpers of the index-gather path shared by its preparation kernels
// and the attention kernels.
#pragma once

#include "kernels.h"

namespace sma {

// Gather row of (batch, KV head): the mask's batch row times its head rows.
__device__ __forceinline__ int64_t gather_row(const AttnProblem& p, int b, int hk) {
  const int lb = p.lists.LB > 1 ? b : 0;
  const int lh = p.lists.LH > 1 ? hk : 0;
  return static_cast<int64_t>(lb) * p.lists.LH + lh;
}

// Compacted keys query row q may attend: every selected key, or under the
// bottom-right causal bound k <= q + k_len - Lq only those whose original
// index satisfies it.  The indices ascend, so this is an upper-bound search.
__device__ __forceinline__ int gather_row_limit(const AttnProblem& p, int64_t grow, int q) {
  const int cnt = p.gather.count[grow];
  if (!p.gather.causal) return cnt;
  const int bound = q + p.gather.k_len - p.Lq;
  const int32_t* idx = p.gather.idx + grow * p.gather.cap;
  int lo = 0, hi = cnt;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (idx[mid] <= bound) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

}  // namespace sma
