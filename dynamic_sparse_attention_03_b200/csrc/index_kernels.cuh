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
// Optionally (out_hi/out_lo not null) also writes the mean split for the
// tensor-core scores: hi = the mean rounded to TF32, lo = mean - hi (exact in
// fp32), so hi + lo carries the full fp32 mean.
__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <int D>
__global__ void __launch_bounds__(256) pool_blocks_kernel(const __nv_bfloat16* __restrict__ x,
                                                           float* __restrict__ out, int64_t nblocks,
                                                           float* __restrict__ out_hi = nullptr,
                                                           float* __restrict__ out_lo = nullptr) {
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
    const float mean = s * (1.0f / kBlock);
    if (out) out[blk * D + c] = mean;
    if (out_hi) {
      const float hi = tf32_round(mean);
      out_hi[blk * D + c] = hi;
      out_lo[blk * D + c] = mean - hi;
    }
  }
}

// ---------------------------------------------------------------- TF32 tensor-core helpers
// Instruction descriptor, kind::tf32 with K-major A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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

}  // namespace dsa
