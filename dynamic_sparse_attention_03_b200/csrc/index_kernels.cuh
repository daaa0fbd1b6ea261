// index_kernels.cuh -- block-sparse index estimation (MInference 1.0 page,
// method section "方法介紹": mean-pool Q and K over 64-token blocks; because
// pooling commutes with MatMul, Q̄_i·K̄_j is the mean of the block's raw scores;
// keep the best blocks per query block) and the decode centroids (Squeezed
// Attention page, "技术方案": per-cluster centroid keys, here block means).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kBlock = 64;

// ---------------------------------------------------------------- pooling
// One CTA of 256 threads per 64-row block of x [rows][D] (bf16): the fp32
// mean of the 64 rows.  Each thread loads 16-byte vectors; the 64 rows are
// summed as (rows r, r+RP, ...) per thread then over the RP row groups in a
// fixed order, so the result is deterministic.
//
// Split for the tensor-core scores (FP16 hi/lo): a row of means m, scaled by
// 2^a with a chosen so that max |m| 2^a lies in [2^13, 2^14), becomes
// hi = fp16(m 2^a) and lo = fp16(m 2^a - hi), so hi + lo carries the scaled
// mean to about 22 bits.  A power-of-two scale is exact, and a scale per
// query block (per row of S) or per KV head (all of S's columns) multiplies a
// row of scores by one positive constant, which leaves its order unchanged.
//
//  out     (optional) the fp32 means;
//  amax    (optional) atomic max of the block's max |mean| per group of
//          rows_per_group blocks, the group's first block excluded (float
//          bits: non-negative floats order as unsigned integers);
//  hi, lo  (optional) the split with the block's own scale (query blocks).
// CTAs past the nblocks pooling ones convert conv_rows fp32 rows of conv_src
// (8 per CTA) into conv_hi / conv_lo with the scale of their group's amax
// (the pooled keys, after their pooling launch has finished).
__device__ __forceinline__ float pow2_scale_for(float amax) {
  if (!(amax > 0.f) || !(amax <= 3.0e38f)) return 1.f;
  int e;
  frexpf(amax, &e);                     // amax in [2^(e-1), 2^e)
  const int a = min(max(14 - e, -100), 100);
  return __int_as_float((127 + a) << 23);
}

__device__ __forceinline__ void split_f16(float m, float scale, __half& hi, __half& lo) {
  const float x = m * scale;
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

template <int D>
__global__ void __launch_bounds__(256) pool_blocks_kernel(
    const __nv_bfloat16* __restrict__ x, float* __restrict__ out, int64_t nblocks, unsigned* __restrict__ amax,
    int rows_per_group, __half* __restrict__ hi, __half* __restrict__ lo, const float* __restrict__ conv_src,
    int64_t conv_rows, const unsigned* __restrict__ conv_amax, __half* __restrict__ conv_hi,
    __half* __restrict__ conv_lo) {
  constexpr int VPR = D / 8;          // 16-byte vectors per row
  constexpr int RP = 256 / VPR;       // rows per pass
  constexpr int PASSES = kBlock / RP;
  __shared__ float part[RP][D + 1];
  __shared__ float wmax[8];
  const int64_t blk = blockIdx.x;
  if (blk >= nblocks) {
    // conversion of pooled keys: 8 rows of D per CTA, 256 threads
    constexpr int PER = 8 * D / 256;
    const int64_t r0 = (blk - nblocks) * 8;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = threadIdx.x + 256 * k;
      const int64_t row = r0 + e / D;
      if (row < conv_rows) {
        const float sc = pow2_scale_for(__uint_as_float(conv_amax[row / rows_per_group]));
        __half h, l;
        split_f16(conv_src[row * D + e % D], sc, h, l);
        conv_hi[row * D + e % D] = h;
        conv_lo[row * D + e % D] = l;
      }
    }
    return;
  }
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
  const int c = threadIdx.x;   // D <= 256 columns, one per thread
  float mean = 0.f;
  if (c < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RP; ++r) s += part[r][c];
    mean = s * (1.0f / kBlock);
    if (out) out[blk * D + c] = mean;
  }
  if (!amax && !hi) return;
  float m = fabsf(mean);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  float bm = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) bm = fmaxf(bm, wmax[w]);
  // The first block of each group (the forced sink block of a KV head) stays
  // out of the group's max: sink keys are often far larger than the rest, and
  // a scale set by them would push the other blocks' low halves toward the
  // FP16 subnormal range.  The sink's own split may then overflow to inf; its
  // score column is never ranked (it is always kept).
  if (amax && threadIdx.x == 0 && blk % rows_per_group != 0)
    atomicMax(amax + blk / rows_per_group, __float_as_uint(bm));
  if (hi && c < D) {
    __half h, l;
    split_f16(mean, pow2_scale_for(bm), h, l);
    hi[blk * D + c] = h;
    lo[blk * D + c] = l;
  }
}

// Instruction descriptor, kind::f16 with fp16 A and B (K-major), fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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
