// index_kernels.cuh -- block-sparse index estimation (MInference 1.0 page,
// method section "方法介紹": mean-pool Q and K over 64-token blocks; because
// pooling commutes with MatMul, Q̄_i·K̄_j is the mean of the block's raw scores;
// keep the best blocks per query block) and the decode centroids (Squeezed
// Attention page, "技术方案": per-cluster centroid keys, here block means).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kBlock = 64;

// ---------------------------------------------------------------- pooling
// One CTA of 256 threads per 64-row block of x [rows][D] (bf16): out = the
// fp32 mean of the 64 rows.  Each thread loads 16-byte vectors; the 64 rows
// are summed as (rows r, r+RP, ...) per thread then over the RP row groups in
// a fixed order, so the result is deterministic.
template <int D>
__global__ void __launch_bounds__(256) pool_blocks_kernel(const __nv_bfloat16* __restrict__ x,
                                                           float* __restrict__ out, int64_t nblocks) {
  constexpr int VPR = D / 8;          // 16-byte vectors per row
  constexpr int RP = 256 / VPR;       // rows per pass
  constexpr int PASSES = kBlock / RP;
  __shared__ float part[RP][D + 1];
  const int64_t blk = blockIdx.x;
  if (blk >= nblocks) return;
  const int vec = threadIdx.x % VPR, rg = threadIdx.x / VPR;
  const uint4* src = reinterpret_cast<const uint4*>(x + blk * kBlock * D);
  uint4 v[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) v[p] = __ldg(src + (size_t)(rg + p * RP) * VPR + vec);
  float acc[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) acc[a] = 0.f;
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float2 f = __bfloat1622float2(h[a]);
      acc[2 * a] += f.x;
      acc[2 * a + 1] += f.y;
    }
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) part[rg][vec * 8 + a] = acc[a];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RP; ++r) s += part[r][c];
    out[blk * D + c] = s * (1.0f / kBlock);
  }
}

// ---------------------------------------------------------------- pooled scores
// S[hl][i][j] = Q̄[h0+hl][i] · K̄[g][j] for the lower-triangular 64x64 tiles
// (tile column <= tile row) of every head of the chunk; fp32 FMA.  256
// threads, each computing a 4x4 sub-tile; operands staged in shared memory
// with the reduction dimension outermost.
template <int D>
__global__ void __launch_bounds__(256) block_scores_kernel(const float* __restrict__ qbar,
                                                            const float* __restrict__ kbar,
                                                            float* __restrict__ S, int nQB, int h0,
                                                            int grp) {
  extern __shared__ __align__(16) float sm_scores[];
  float* As = sm_scores;              // [D][64]
  float* Bs = sm_scores + D * 64;     // [D][64]
  const int hl = blockIdx.y, h = h0 + hl, g = h / grp;
  // triangular tile index -> (rt, ct), ct <= rt
  const int x = blockIdx.x;
  int rt = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((rt + 1) * (rt + 2) / 2 <= x) ++rt;
  while (rt * (rt + 1) / 2 > x) --rt;
  const int ct = x - rt * (rt + 1) / 2;
  const int tid = threadIdx.x;
  const float* qa = qbar + ((size_t)h * nQB + (size_t)rt * 64) * D;
  const float* kb = kbar + ((size_t)g * nQB + (size_t)ct * 64) * D;
  // stage: element (row m, k) -> As[k*64 + m]
  for (int idx = tid; idx < 64 * D / 4; idx += 256) {
    const int m = idx / (D / 4), k4 = (idx % (D / 4)) * 4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (rt * 64 + m < nQB) a = *reinterpret_cast<const float4*>(qa + (size_t)m * D + k4);
    if (ct * 64 + m < nQB) b = *reinterpret_cast<const float4*>(kb + (size_t)m * D + k4);
    As[(k4 + 0) * 64 + m] = a.x; As[(k4 + 1) * 64 + m] = a.y;
    As[(k4 + 2) * 64 + m] = a.z; As[(k4 + 3) * 64 + m] = a.w;
    Bs[(k4 + 0) * 64 + m] = b.x; Bs[(k4 + 1) * 64 + m] = b.y;
    Bs[(k4 + 2) * 64 + m] = b.z; Bs[(k4 + 3) * 64 + m] = b.w;
  }
  __syncthreads();
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const float4 av = *reinterpret_cast<const float4*>(As + k * 64 + ty * 4);
    const float4 bv = *reinterpret_cast<const float4*>(Bs + k * 64 + tx * 4);
    const float ar[4] = {av.x, av.y, av.z, av.w};
    const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(ar[a], br[b], acc[a][b]);
  }
  float* out = S + (size_t)hl * nQB * nQB;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = rt * 64 + ty * 4 + a;
    if (i >= nQB) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = ct * 64 + tx * 4 + b;
      if (j < nQB) out[(size_t)i * nQB + j] = acc[a][b];
    }
  }
}

// Number of non-forced blocks kept for query block i (ratio in parts per
// million, exact integer ceiling).
__host__ __device__ inline int extra_budget(int i, int k_fixed, int64_t ppm) {
  const int forced = (i == 0) ? 1 : 2;
  const int cand = i > 1 ? i - 1 : 0;
  int64_t e;
  if (k_fixed > 0) {
    e = (int64_t)(i + 1 < k_fixed ? i + 1 : k_fixed) - forced;
  } else {
    e = (ppm * (int64_t)(i + 1) + 999999) / 1000000;
  }
  if (e < 0) e = 0;
  if (e > cand) e = cand;
  return (int)e;
}

// ---------------------------------------------------------------- per-row selection
// One CTA per (query block i, head of the chunk): keep blocks {0, i} plus the
// top extra_budget(i) of blocks 1..i-1 by score, ties to the lower block.
template <int NT>
__global__ void __launch_bounds__(NT) block_select_kernel(const float* __restrict__ S, int nQB, int h0,
                                                          int k_fixed, int64_t ppm, int32_t* __restrict__ block_idx,
                                                          int32_t* __restrict__ block_cnt, int kcap) {
  extern __shared__ __align__(16) float row[];
  __shared__ SelectSmem sm;
  const int i = blockIdx.x, hl = blockIdx.y, h = h0 + hl;
  const int L = i > 1 ? i - 1 : 0;
  const int e = extra_budget(i, k_fixed, ppm);
  const float* src = S + ((size_t)hl * nQB + i) * nQB + 1;
  const bool need_scores = (e > 0 && e < L);
  if (need_scores) {
    for (int j = threadIdx.x; j < L; j += NT) row[j] = src[j];
    __syncthreads();
  }
  int32_t* out = block_idx + ((size_t)h * nQB + i) * kcap;
  const int cnt = topk_ascending<NT>(row, L, e, 1, i + 1, out, kcap, sm);
  if (threadIdx.x == 0) block_cnt[(size_t)h * nQB + i] = cnt;
}

}  // namespace dsa
