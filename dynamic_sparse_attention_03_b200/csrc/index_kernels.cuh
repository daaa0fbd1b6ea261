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

// ---------------------------------------------------------------- pooled scores on tensor cores
// S = Q̄ K̄^T with fp32-level accuracy from three TF32 products,
// S ~= Qhi Khi + Qhi Klo + Qlo Khi (the dropped Qlo Klo term is ~2^-22
// relative), accumulated in fp32 in TMEM.  One CTA (4 warps) per
// (head, 128 query blocks, 64 key blocks) tile on or below the diagonal: the
// reduction dimension d streams in chunks of 32 floats (one 128-byte swizzle
// atom) through a 2-stage TMA ring; thread 0 issues the MMAs; the 4 warps read
// the accumulators back, one query block per thread, and store the row.
template <int D>
struct ScoreTcLayout {
  static constexpr int kA = 128 * 128;            // 128 rows x 32 fp32
  static constexpr int kB = 64 * 128;             // 64 rows x 32 fp32
  static constexpr int kStage = 2 * kA + 2 * kB;  // hi and lo of both operands
  static constexpr int kBar = 2 * kStage;
  static constexpr int kBytes = kBar + 64;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int NCH = D / 32;
};

__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(128, 2)
    block_scores_tc_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
                           const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                           float* __restrict__ S, int nQB, int h0, int grp, uint32_t* status) {
  using Lay = ScoreTcLayout<D>;
  extern __shared__ uint8_t sc_smem_raw[];
  if (status_timed_out(status)) return;
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sc_smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + Lay::kBar;   // full[2], empty[2], done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kBar + 40);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kBar + 44);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hl = blockIdx.y, h = h0 + hl, g = h / grp;
  // tile x -> (rt, ct): row tile rt (128 query blocks) has column tiles ct = 0 .. 2*rt+1 (64 each)
  const int x = blockIdx.x;
  int rt = (int)((sqrtf(4.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((rt + 1) * (rt + 2) <= x) ++rt;
  while (rt * (rt + 1) > x) --rt;
  const int ct = x - rt * (rt + 1);
  if (ct * 64 >= nQB) return;   // whole tile past the last key block (ragged last row tile)
  if (threadIdx.x == 0) {
    for (int b = 0; b < 5; ++b) mbar_init(bar0 + 8u * b, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, status};
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 16u + 8u * s; };
  const uint32_t done = bar0 + 32u;
  const int arow = h * nQB + rt * 128, brow = g * nQB + ct * 64;
  if (threadIdx.x == 0) {
    auto load = [&](int c) {
      const uint32_t st = sb + (c & 1) * Lay::kStage;
      mbar_arrive_expect_tx(full(c & 1), (uint32_t)Lay::kStage);
      tma_load_2d(st, &tmQh, c * 32, arow, full(c & 1));
      tma_load_2d(st + Lay::kA, &tmQl, c * 32, arow, full(c & 1));
      tma_load_2d(st + 2 * Lay::kA, &tmKh, c * 32, brow, full(c & 1));
      tma_load_2d(st + 2 * Lay::kA + Lay::kB, &tmKl, c * 32, brow, full(c & 1));
    };
    load(0);
    if (Lay::NCH > 1) load(1);
    const uint32_t idesc = umma_idesc_tf32(128, 64);
    bool ok = true;
    for (int c = 0; c < Lay::NCH && ok; ++c) {
      if (!mbar_wait(full(c & 1), (c >> 1) & 1, ab)) { ok = false; break; }
      tc_fence_after();
      const uint32_t st = sb + (c & 1) * Lay::kStage;
      const uint32_t aH = st, aL = st + Lay::kA, bH = st + 2 * Lay::kA, bL = bH + Lay::kB;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t ko = kk * 32;   // 8 fp32 per step
        const uint32_t acc0 = (c > 0 || kk > 0) ? 1u : 0u;
        umma_tf32_ss(tmem, umma_desc_sw128(aH + ko, 16, 1024), umma_desc_sw128(bH + ko, 16, 1024), idesc, acc0);
        umma_tf32_ss(tmem, umma_desc_sw128(aH + ko, 16, 1024), umma_desc_sw128(bL + ko, 16, 1024), idesc, 1u);
        umma_tf32_ss(tmem, umma_desc_sw128(aL + ko, 16, 1024), umma_desc_sw128(bH + ko, 16, 1024), idesc, 1u);
      }
      umma_commit(empty(c & 1));
      if (c + 2 < Lay::NCH) {
        if (!mbar_wait(empty(c & 1), (c >> 1) & 1, ab)) { ok = false; break; }
        load(c + 2);
      }
    }
    umma_commit(done);
  }
  const bool ok = mbar_wait_warp(done, 0, ab);
  if (ok) {
    tc_fence_after();
    const int i = rt * 128 + warp * 32 + lane;
    const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16);
    float* out = S + ((size_t)hl * nQB + i) * nQB + ct * 64;
    const bool vec = (nQB & 3) == 0;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t v[32];
      tmem_ld32(ta + 32 * cc, v);
      tmem_wait_ld();
      reg_fence(v);
      if (i < nQB) {
        const int j0 = ct * 64 + 32 * cc;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = j0 + 4 * q;
          if (vec && j + 3 < nQB) {
            *reinterpret_cast<float4*>(out + 32 * cc + 4 * q) =
                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                            __uint_as_float(v[4 * q + 3]));
          } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
              if (j + b < nQB) out[32 * cc + 4 * q + b] = __uint_as_float(v[4 * q + b]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
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

// Same selection with one warp per row (for rows that fit in shared memory):
// a radix select over the row's keys with a per-warp histogram, then an
// in-order ballot compaction of positions 0..i.  No block-wide barriers.
template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32) block_select_warp_kernel(const float* __restrict__ S, int nQB, int h0,
                                                                       int nrows, int k_fixed, int64_t ppm,
                                                                       int32_t* __restrict__ block_idx,
                                                                       int32_t* __restrict__ block_cnt, int kcap) {
  extern __shared__ __align__(16) float rows_smem[];   // [WARPS][nQB]
  __shared__ uint32_t hist[WARPS][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rix = blockIdx.x * WARPS + w;
  if (rix >= nrows) return;
  const int hl = rix / nQB, i = rix % nQB, h = h0 + hl;
  const int L = i > 1 ? i - 1 : 0;
  const int e = extra_budget(i, k_fixed, ppm);
  int32_t* out = block_idx + ((size_t)h * nQB + i) * kcap;
  float* row = rows_smem + (size_t)w * nQB;
  const bool all = (e >= L), none = (e == 0);
  uint32_t T = 0;
  int need = 0;
  if (!all && !none) {
    const float* src = S + ((size_t)hl * nQB + i) * nQB + 1;
    for (int j = lane; j < L; j += 32) row[j] = src[j];
    __syncwarp();
    uint32_t prefix = 0, mask = 0;
    int rem = e;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int a = 0; a < 8; ++a) hist[w][lane * 8 + a] = 0u;
      __syncwarp();
      for (int j = lane; j < L; j += 32) {
        const uint32_t k = float_key(row[j]);
        if ((k & mask) == prefix) atomicAdd(&hist[w][(k >> shift) & 255u], 1u);
      }
      __syncwarp();
      uint32_t c[8];
      uint32_t s = 0;
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        c[a] = hist[w][255 - 8 * lane - a];
        s += c[a];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
      }
      const uint32_t excl = incl - s;
      const bool owner = excl < (uint32_t)rem && (uint32_t)rem <= incl;
      uint32_t bin = 0, nrem = 0;
      if (owner) {
        uint32_t cum = excl;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          if (cum + c[a] >= (uint32_t)rem) {
            bin = (uint32_t)(255 - 8 * lane - a);
            nrem = (uint32_t)rem - cum;
            break;
          }
          cum += c[a];
        }
      }
      const int src_lane = __ffs(__ballot_sync(0xFFFFFFFFu, owner)) - 1;
      bin = __shfl_sync(0xFFFFFFFFu, bin, src_lane);
      rem = (int)__shfl_sync(0xFFFFFFFFu, nrem, src_lane);
      prefix |= bin << shift;
      mask |= 255u << shift;
      __syncwarp();
    }
    T = prefix;
    need = rem;
  }
  // in-order compaction of positions 0..i (0 and i are forced)
  const unsigned lt = (1u << lane) - 1u;
  int off = 0, eq_before = 0;
  for (int base = 0; base <= i; base += 32) {
    const int p = base + lane;
    const int c = p - 1;
    bool sel = false, is_eq = false;
    if (p <= i) {
      if (c < 0 || c >= L || all) sel = true;
      else if (!none) {
        const uint32_t key = float_key(row[c]);
        sel = key > T;
        is_eq = key == T;
      }
    }
    const unsigned eqm = __ballot_sync(0xFFFFFFFFu, is_eq);
    if (is_eq && eq_before + __popc(eqm & lt) < need) sel = true;
    eq_before += __popc(eqm);
    const unsigned sm = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) {
      const int slot = off + __popc(sm & lt);
      if (slot < kcap) out[slot] = p;
    }
    off += __popc(sm);
  }
  for (int j = off + lane; j < kcap; j += 32) out[j] = -1;
  if (lane == 0) block_cnt[(size_t)h * nQB + i] = off;
}

}  // namespace dsa
