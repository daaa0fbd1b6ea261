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
// S[hl][i][j] = Q̄[h0+hl][i] · K̄[g][j] for the lower-triangular 128x128 tiles
// (tile column <= tile row) of every head of the chunk; fp32 FMA.  256
// threads, each computing an 8x8 sub-tile (rows ty*4+{0..3} and 64+ty*4+{0..3},
// columns likewise with tx), so four 16-byte shared loads feed 64 FMAs.  The
// reduction dimension is staged in chunks of 32, double-buffered through
// registers, transposed so it is outermost in shared memory.
constexpr int kScoreTile = 128;
constexpr int kScoreKC = 32;
constexpr int kScoreLd = 132;   // padded row of the transposed stage
constexpr size_t kScoreSmem = 2 * 2 * kScoreKC * kScoreLd * sizeof(float);

template <int D>
__global__ void __launch_bounds__(256) block_scores_kernel(const float* __restrict__ qbar,
                                                            const float* __restrict__ kbar,
                                                            float* __restrict__ S, int nQB, int h0,
                                                            int grp) {
  extern __shared__ __align__(16) float sm_scores[];
  // [buf][A/B][k][m]
  auto stage = [&](int buf, int ab) { return sm_scores + ((buf * 2 + ab) * kScoreKC) * kScoreLd; };
  const int hl = blockIdx.y, h = h0 + hl, g = h / grp;
  // triangular tile index -> (rt, ct), ct <= rt
  const int x = blockIdx.x;
  int rt = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((rt + 1) * (rt + 2) / 2 <= x) ++rt;
  while (rt * (rt + 1) / 2 > x) --rt;
  const int ct = x - rt * (rt + 1) / 2;
  const int tid = threadIdx.x;
  const float* qa = qbar + ((size_t)h * nQB + (size_t)rt * kScoreTile) * D;
  const float* kb = kbar + ((size_t)g * nQB + (size_t)ct * kScoreTile) * D;
  // loads of one chunk: 128 rows x 32 floats per operand, 4 float4 per thread each
  float4 ra[4], rb[4];
  auto load = [&](int c) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int idx = tid + 256 * q;
      const int m = idx >> 3, k4 = (idx & 7) * 4;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      ra[q] = (rt * kScoreTile + m < nQB) ? *reinterpret_cast<const float4*>(qa + (size_t)m * D + c * kScoreKC + k4) : z;
      rb[q] = (ct * kScoreTile + m < nQB) ? *reinterpret_cast<const float4*>(kb + (size_t)m * D + c * kScoreKC + k4) : z;
    }
  };
  auto store = [&](int buf) {
    float* As = stage(buf, 0);
    float* Bs = stage(buf, 1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int idx = tid + 256 * q;
      const int m = idx >> 3, k4 = (idx & 7) * 4;
      As[(k4 + 0) * kScoreLd + m] = ra[q].x; As[(k4 + 1) * kScoreLd + m] = ra[q].y;
      As[(k4 + 2) * kScoreLd + m] = ra[q].z; As[(k4 + 3) * kScoreLd + m] = ra[q].w;
      Bs[(k4 + 0) * kScoreLd + m] = rb[q].x; Bs[(k4 + 1) * kScoreLd + m] = rb[q].y;
      Bs[(k4 + 2) * kScoreLd + m] = rb[q].z; Bs[(k4 + 3) * kScoreLd + m] = rb[q].w;
    }
  };
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  constexpr int NCH = D / kScoreKC;
  load(0);
  store(0);
  __syncthreads();
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    if (c + 1 < NCH) load(c + 1);
    const float* As = stage(c & 1, 0);
    const float* Bs = stage(c & 1, 1);
#pragma unroll 4
    for (int k = 0; k < kScoreKC; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(As + k * kScoreLd + ty * 4);
      const float4 a1 = *reinterpret_cast<const float4*>(As + k * kScoreLd + 64 + ty * 4);
      const float4 b0 = *reinterpret_cast<const float4*>(Bs + k * kScoreLd + tx * 4);
      const float4 b1 = *reinterpret_cast<const float4*>(Bs + k * kScoreLd + 64 + tx * 4);
      const float ar[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(ar[a], br[b], acc[a][b]);
    }
    if (c + 1 < NCH) store((c + 1) & 1);
    __syncthreads();
  }
  float* out = S + (size_t)hl * nQB * nQB;
  const bool vec = (nQB & 3) == 0;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = rt * kScoreTile + (a < 4 ? ty * 4 + a : 64 + ty * 4 + a - 4);
    if (i >= nQB) continue;
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
      const int j0 = ct * kScoreTile + hb * 64 + tx * 4;
      float* dst = out + (size_t)i * nQB + j0;
      if (vec && j0 + 3 < nQB) {
        *reinterpret_cast<float4*>(dst) =
            make_float4(acc[a][hb * 4], acc[a][hb * 4 + 1], acc[a][hb * 4 + 2], acc[a][hb * 4 + 3]);
      } else {
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (j0 + b < nQB) dst[b] = acc[a][hb * 4 + b];
      }
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
