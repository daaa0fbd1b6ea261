// vs_kernels.cuh -- vertical-slash index (MInference 1.0 page, method section
// "方法介紹": the attention between the last queries and all keys estimates
// the vertical lines and slash lines; Fig. 4: slash lines as 64x64 blocks,
// vertical lines as 1x64 column tiles).
//
// Rows i_r = n - 64 + r.  Pass 1 computes each row's log-sum-exp over its
// causal keys; pass 2 recomputes the scores, forms the probabilities
// P[r][j] = exp(z - lse_r), and sums them per key column (vert) and per
// diagonal offset o = i_r - j (slash).  Both passes tile the keys in blocks of
// 64 per CTA (one q-head); every sum runs in a fixed order, so the scores are
// deterministic run to run.  Then a top-k per head and the per-query-block
// plan (aligned 64x64 blocks for slashes, column entries for verticals).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

struct VSParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* part;        // [Hq][ntiles][64][2]  pass-1 (max, sum) per tile and row (log2 domain)
  float* lse2;        // [Hq][64]
  float* vert;        // [Hq][n]
  float* slash_part;  // [Hq][ntiles][127]
  float* slash;       // [Hq][n]
  int32_t* vsel;      // [Hq][n_vert]
  int32_t* ssel;      // [Hq][n_slash]
  int32_t* block_idx;
  int32_t* block_cnt;
  int32_t* col_idx;
  int32_t* col_cnt;
  int Hq, Hkv, n, nQB, grp, ntiles, n_vert, n_slash, kcap, ccap;
  float scale_log2;
};

// z[r][c] for rows r of the last-64 queries of head h and keys j0+c, c < 64,
// in the log2 domain (scale * log2 e folded in), -inf where j0 + c > i_r.
// Shared memory: Qs [D][64], Ks [D][64] fp32 (reduction dim outermost), Z [64][65].
template <int D>
__device__ __forceinline__ void vs_logits_tile(const VSParams& p, int h, int tile, float* Qs, float* Ks, float* Z) {
  const int g = h / p.grp;
  const int j0 = tile * 64;
  const int i0 = p.n - 64;
  const __nv_bfloat16* qsrc = p.q + ((size_t)h * p.n + i0) * D;
  const __nv_bfloat16* ksrc = p.k + ((size_t)g * p.n + j0) * D;
  for (int idx = threadIdx.x; idx < 64 * D / 8; idx += 256) {
    const int m = idx / (D / 8), k8 = (idx % (D / 8)) * 8;
    const uint4 qa = __ldg(reinterpret_cast<const uint4*>(qsrc + (size_t)m * D + k8));
    const uint4 ka = __ldg(reinterpret_cast<const uint4*>(ksrc + (size_t)m * D + k8));
    const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qa);
    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&ka);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float2 qf = __bfloat1622float2(q2[a]);
      const float2 kf = __bfloat1622float2(k2[a]);
      Qs[(k8 + 2 * a) * 64 + m] = qf.x;
      Qs[(k8 + 2 * a + 1) * 64 + m] = qf.y;
      Ks[(k8 + 2 * a) * 64 + m] = kf.x;
      Ks[(k8 + 2 * a + 1) * 64 + m] = kf.y;
    }
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
  for (int kk = 0; kk < D; ++kk) {
    const float4 av = *reinterpret_cast<const float4*>(Qs + kk * 64 + ty * 4);
    const float4 bv = *reinterpret_cast<const float4*>(Ks + kk * 64 + tx * 4);
    const float ar[4] = {av.x, av.y, av.z, av.w};
    const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(ar[a], br[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = ty * 4 + a;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int c = tx * 4 + b;
      Z[r * 65 + c] = (j0 + c <= i0 + r) ? acc[a][b] * p.scale_log2 : -INFINITY;
    }
  }
  __syncthreads();
}

// Pass 1: per (tile, head): row max and sum of exp2 over the tile's keys.
template <int D>
__global__ void __launch_bounds__(256) vs_pass1_kernel(const VSParams p) {
  extern __shared__ __align__(16) float vsm[];
  float* Qs = vsm;
  float* Ks = Qs + D * 64;
  float* Z = Ks + D * 64;
  const int tile = blockIdx.x, h = blockIdx.y;
  vs_logits_tile<D>(p, h, tile, Qs, Ks, Z);
  // 4 threads per row
  const int r = threadIdx.x >> 2, q = threadIdx.x & 3;
  float mx = -INFINITY;
  for (int c = q; c < 64; c += 4) mx = fmaxf(mx, Z[r * 65 + c]);
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  float s = 0.f;
  if (mx != -INFINITY)
    for (int c = q; c < 64; c += 4) s += exp2f(Z[r * 65 + c] - mx);
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
  if (q == 0) {
    float* o = p.part + (((size_t)h * p.ntiles + tile) * 64 + r) * 2;
    o[0] = mx;
    o[1] = s;
  }
}

// Per (head, row): combine the tile partials in tile order -> lse (log2 domain).
__global__ void __launch_bounds__(64) vs_lse_kernel(const VSParams p) {
  const int h = blockIdx.x, r = threadIdx.x;
  const float* pp = p.part + ((size_t)h * p.ntiles * 64 + r) * 2;
  float M = -INFINITY;
  for (int t = 0; t < p.ntiles; ++t) M = fmaxf(M, pp[(size_t)t * 128]);
  float L = 0.f;
  for (int t = 0; t < p.ntiles; ++t) {
    const float mt = pp[(size_t)t * 128];
    if (mt != -INFINITY) L += pp[(size_t)t * 128 + 1] * exp2f(mt - M);
  }
  p.lse2[h * 64 + r] = M + log2f(L);
}

// Pass 2: probabilities of the tile; column sums (complete) and diagonal
// partial sums of the tile's 127 offsets.
template <int D>
__global__ void __launch_bounds__(256) vs_pass2_kernel(const VSParams p) {
  extern __shared__ __align__(16) float vsm[];
  float* Qs = vsm;
  float* Ks = Qs + D * 64;
  float* Z = Ks + D * 64;
  const int tile = blockIdx.x, h = blockIdx.y;
  vs_logits_tile<D>(p, h, tile, Qs, Ks, Z);
  for (int x = threadIdx.x; x < 64 * 64; x += 256) {
    const int r = x >> 6, c = x & 63;
    const float z = Z[r * 65 + c];
    Z[r * 65 + c] = (z == -INFINITY) ? 0.f : exp2f(z - p.lse2[h * 64 + r]);
  }
  __syncthreads();
  const int t = threadIdx.x;
  if (t < 64) {
    float s = 0.f;
    for (int r = 0; r < 64; ++r) s += Z[r * 65 + t];
    p.vert[(size_t)h * p.n + tile * 64 + t] = s;
  } else if (t < 64 + 127) {
    // offset index od: o = n - 127 - 64*tile + od ; key column c = r + 63 - od
    const int od = t - 64;
    float s = 0.f;
    const int rlo = max(0, od - 63), rhi = min(63, od);
    for (int r = rlo; r <= rhi; ++r) s += Z[r * 65 + (r + 63 - od)];
    p.slash_part[((size_t)h * p.ntiles + tile) * 127 + od] = s;
  }
}

// slash[o] = sum of the (at most two) tile partials covering offset o, in tile order.
__global__ void __launch_bounds__(256) vs_slash_kernel(const VSParams p) {
  const int h = blockIdx.y;
  const int o = blockIdx.x * 256 + threadIdx.x;
  if (o >= p.n) return;
  // tile t covers offsets [n - 127 - 64t, n - 1 - 64t]
  const int tlo = max(0, (p.n - 127 - o + 63) >> 6);   // ceil((n-127-o)/64), clamped
  const int thi = min(p.ntiles - 1, (p.n - 1 - o) >> 6);
  float s = 0.f;
  for (int t = tlo; t <= thi; ++t) {
    const int od = o - (p.n - 127 - 64 * t);
    if (od >= 0 && od < 127) s += p.slash_part[((size_t)h * p.ntiles + t) * 127 + od];
  }
  p.slash[(size_t)h * p.n + o] = s;
}

// Top columns (first 64 forced) and top offsets (offset 0 forced) per head.
template <int NT>
__global__ void __launch_bounds__(NT) vs_topk_kernel(const VSParams p) {
  __shared__ SelectSmem sm;
  const int h = blockIdx.x;
  if (blockIdx.y == 0) {
    const int nf = min(64, p.n);
    topk_ascending<NT>(p.vert + (size_t)h * p.n + nf, p.n - nf, p.n_vert - nf, nf, p.n,
                       p.vsel + (size_t)h * p.n_vert, p.n_vert, sm);
  } else {
    topk_ascending<NT>(p.slash + (size_t)h * p.n + 1, p.n - 1, p.n_slash - 1, 1, p.n,
                       p.ssel + (size_t)h * p.n_slash, p.n_slash, sm);
  }
}

// Plan for (qb, h): blocks touched by the kept offsets, and kept columns whose
// block is not among them.
template <int NT>
__global__ void __launch_bounds__(NT) vs_plan_kernel(const VSParams p) {
  extern __shared__ __align__(16) uint32_t bits[];   // nQB bits
  __shared__ SelectSmem sm;
  const int qb = blockIdx.x, h = blockIdx.y;
  const int nwords = (p.nQB + 31) >> 5;
  for (int w = threadIdx.x; w < nwords; w += NT) bits[w] = 0u;
  __syncthreads();
  const int last = 64 * qb + 63;
  const int32_t* so = p.ssel + (size_t)h * p.n_slash;
  for (int x = threadIdx.x; x < p.n_slash; x += NT) {
    const int o = so[x];
    if (o < 0 || o > last) continue;
    const int near = qb - (o >> 6);
    const int far = qb - ((o + 63) >> 6);
    atomicOr(&bits[near >> 5], 1u << (near & 31));
    if (far >= 0) atomicOr(&bits[far >> 5], 1u << (far & 31));
  }
  __syncthreads();
  // blocks: ordered compaction over positions 0..qb
  {
    const int P = qb + 1;
    const int per = (P + NT - 1) / NT;
    const int p0 = min(P, (int)threadIdx.x * per), p1 = min(P, p0 + per);
    int kept = 0;
    for (int x = p0; x < p1; ++x) kept += (bits[x >> 5] >> (x & 31)) & 1u;
    int total;
    int off = block_excl_scan<NT>(kept, sm, total);
    int32_t* out = p.block_idx + ((size_t)h * p.nQB + qb) * p.kcap;
    for (int x = p0; x < p1; ++x)
      if ((bits[x >> 5] >> (x & 31)) & 1u) {
        if (off < p.kcap) out[off] = x;
        ++off;
      }
    for (int x = total + (int)threadIdx.x; x < p.kcap; x += NT) out[x] = -1;
    if (threadIdx.x == 0) p.block_cnt[(size_t)h * p.nQB + qb] = min(total, p.kcap);
  }
  // columns: kept j <= last with block not selected, in list order
  {
    const int32_t* vi = p.vsel + (size_t)h * p.n_vert;
    const int P = p.n_vert;
    const int per = (P + NT - 1) / NT;
    const int p0 = min(P, (int)threadIdx.x * per), p1 = min(P, p0 + per);
    int kept = 0;
    for (int x = p0; x < p1; ++x) {
      const int j = vi[x];
      kept += (j >= 0 && j <= last && !((bits[j >> 11] >> ((j >> 6) & 31)) & 1u));
    }
    int total;
    int off = block_excl_scan<NT>(kept, sm, total);
    int32_t* out = p.col_idx + ((size_t)h * p.nQB + qb) * p.ccap;
    for (int x = p0; x < p1; ++x) {
      const int j = vi[x];
      if (j >= 0 && j <= last && !((bits[j >> 11] >> ((j >> 6) & 31)) & 1u)) {
        if (off < p.ccap) out[off] = j;
        ++off;
      }
    }
    for (int x = total + (int)threadIdx.x; x < p.ccap; x += NT) out[x] = -1;
    if (threadIdx.x == 0) p.col_cnt[(size_t)h * p.nQB + qb] = min(total, p.ccap);
  }
}

}  // namespace dsa
