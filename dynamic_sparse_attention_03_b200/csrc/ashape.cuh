// ashape.cuh -- A-shape (sink + local window) block index (MInference 1.0 page,
// method section "方法介紹": the A-shape pattern keeps the first tokens and a
// local window of recent tokens).  At 64-token block granularity query block
// qb keeps key blocks [0, min(n_sink, qb+1)) and [max(0, qb-n_local+1), qb].
// One warp per (head, query block) writes its ascending list, -1 padded.
#pragma once

#include <cstdint>

namespace dsa {

__global__ void __launch_bounds__(256) a_shape_kernel(int nrows, int nQB, int n_sink, int n_local,
                                                       int32_t* __restrict__ block_idx,
                                                       int32_t* __restrict__ block_cnt, int kcap) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;
  const int qb = row % nQB;
  const int s = min(n_sink, qb + 1);
  const int lo = max(0, qb - n_local + 1);
  const bool joined = lo <= s;
  const int cnt = joined ? qb + 1 : s + (qb - lo + 1);
  int32_t* out = block_idx + (size_t)row * kcap;
  for (int j = lane; j < kcap; j += 32) {
    int v = -1;
    if (j < cnt) v = (joined || j < s) ? j : lo + (j - s);
    out[j] = v;
  }
  if (lane == 0) block_cnt[row] = cnt;
}

}  // namespace dsa
