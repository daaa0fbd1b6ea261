// vs_kernels.cuh -- vertical-slash index (MInference 1.0 page, method section
// "方法介紹": the attention between the last queries and all keys estimates
// the vertical lines and slash lines; Fig. 4: slash lines as 64x64 blocks,
// vertical lines as 1x64 column tiles).
//
// Rows i_r = n - 64 + r.  The logits z = q_i.k_j * scale (log2 domain) of
// those rows against every key come from one tcgen05 kernel (a dense
// product).  Pass 1 then computes each row's log-sum-exp over its causal keys;
// pass 2 forms the probabilities P[r][j] = 2^(z - lse_r) and sums them per key
// column (vert) and per diagonal offset o = i_r - j (slash).  Both passes tile
// the keys in blocks of 64 per CTA (one q-head) and sum in a fixed order, so
// the scores are deterministic run to run.  Then a top-k per head and the
// per-query-block plan (aligned 64x64 blocks for slashes, column entries for
// verticals).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

struct VSParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* zlog;        // [Hq][64][n] logits of the last 64 queries, log2 domain (scale*log2e folded in)
  uint32_t* status;
  float* part;        // [Hq][ntiles][64][2]  pass-1 (max, sum) per tile and row (log2 domain)
  float* lse2;        // [Hq][64]
  float* vert;        // [Hq][n]
  float* slash_part;  // [Hq][ntiles][127]
  float* slash;       // [Hq][n]
  int32_t* vsel;      // [Hq][n_vert]
  int32_t* ssel;      // [Hq][n_slash]
  uint32_t* dbits;    // [Hq][ceil(nQB/32)] block distances reached by kept offsets
  int32_t* dlist;     // [Hq][nQB] the same distances, ascending
  int32_t* dcount;    // [Hq]
  int32_t* block_idx;
  int32_t* block_cnt;
  int32_t* col_idx;
  int32_t* col_cnt;
  int Hq, Hkv, n, nQB, grp, ntiles, n_vert, n_slash, kcap, ccap;
  float scale_log2;
};

// ---------------------------------------------------------------- logits on tensor cores
// Z[h][r][j] = (q_{n-64+r} . k_j) * scale * log2(e) for the last 64 queries
// of every q-head against all keys of its KV head: a dense product, so it runs
// on tcgen05.  One CTA per (KV head, group of four q-heads, 128 keys): the
// four heads' 64 rows form two M=128 tiles (TMA, 128-byte swizzle), the key
// tile is N=128, fp32 accumulators in TMEM; 8 warps read the accumulators
// back (one row per thread) and store the scaled row segment.  Causal masking
// is left to the passes that read Z.
template <int D>
struct VSLogitLayout {
  static constexpr int NDH = D / 64;
  static constexpr int kHalf = 16384;        // one d-half of 128 rows x 128 B
  static constexpr int kTile = NDH * kHalf;
  static constexpr int kQA = 0, kQB = kTile, kK = 2 * kTile;
  static constexpr int kBar = 3 * kTile;
  static constexpr int kBytes = kBar + 64;
  static constexpr int kSmemAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(256, 2)
    vs_logits_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const VSParams p) {
  using Lay = VSLogitLayout<D>;
  extern __shared__ uint8_t vs_smem_raw[];
  if (status_timed_out(p.status)) return;
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(vs_smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_full = sb + Lay::kBar, bar_mma = bar_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kBar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kBar + 20);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nquads = (p.grp + 3) / 4;
  const int g = blockIdx.y / nquads, quad = blockIdx.y % nquads;
  const int h0 = g * p.grp + 4 * quad;
  const int nh = min(4, p.grp - 4 * quad);
  const int j0 = blockIdx.x * 128;
  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, p.status};
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_full, (uint32_t)(3 * Lay::kTile));
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      const int h = h0 + min(hh, nh - 1);
#pragma unroll
      for (int dh = 0; dh < Lay::NDH; ++dh)
        tma_load_2d(sb + (hh >> 1) * Lay::kTile + dh * Lay::kHalf + (hh & 1) * 8192, &tmQ, dh * 64,
                    h * p.n + p.n - 64, bar_full);
    }
#pragma unroll
    for (int dh = 0; dh < Lay::NDH; ++dh) {
      tma_load_2d(sb + Lay::kK + dh * Lay::kHalf, &tmK, dh * 64, g * p.n + j0, bar_full);
      tma_load_2d(sb + Lay::kK + dh * Lay::kHalf + 8192, &tmK, dh * 64, g * p.n + j0 + 64, bar_full);
    }
    if (mbar_wait(bar_full, 0, ab)) {
      tc_fence_after();
      const uint32_t idesc = umma_idesc_bf16(128, 128, 0);
#pragma unroll
      for (int tile = 0; tile < 2; ++tile) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = umma_desc_sw128(sb + tile * Lay::kTile + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(sb + Lay::kK + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          umma_bf16_ss(tmem + 128u * (uint32_t)tile, a, b, idesc, kk > 0 ? 1u : 0u);
        }
      }
    }
    umma_commit(bar_mma);
  }
  // epilogue: warp w reads TMEM lane quarter w%4 of tile w/4
  const int tile = warp >> 2, q4 = warp & 3;
  const int row = q4 * 32 + lane;
  const int hh = 2 * tile + (row >> 6), r = row & 63;
  const bool ok = mbar_wait_warp(bar_mma, 0, ab);
  if (ok && hh < nh) {
    tc_fence_after();
    float* dst = p.zlog + ((size_t)(h0 + hh) * 64 + r) * p.n + j0;
    const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16) + 128u * (uint32_t)tile;
    const int nchunk = min(128, p.n - j0) / 32;   // the last tile of an n % 128 == 64 sequence has 64 keys
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c >= nchunk) break;
      uint32_t v[32];
      tmem_ld32(ta + 32 * c, v);
      tmem_wait_ld();
      reg_fence(v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 w = make_float4(__uint_as_float(v[4 * q]) * p.scale_log2, __uint_as_float(v[4 * q + 1]) * p.scale_log2,
                                     __uint_as_float(v[4 * q + 2]) * p.scale_log2,
                                     __uint_as_float(v[4 * q + 3]) * p.scale_log2);
        *reinterpret_cast<float4*>(dst + 32 * c + 4 * q) = w;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// z[r][c] (log2 domain) of rows r of the last-64 queries of head h and keys
// j0+c, c < 64, read from the logits above; -inf where j0 + c > i_r.
__device__ __forceinline__ void vs_load_tile(const VSParams& p, int h, int tile, float* Z) {
  const int j0 = tile * 64;
  const int i0 = p.n - 64;
  const float* src = p.zlog + (size_t)h * 64 * p.n + j0;
  for (int x = threadIdx.x; x < 64 * 16; x += 256) {
    const int r = x >> 4, c4 = (x & 15) * 4;
    const float4 v = __ldg(reinterpret_cast<const float4*>(src + (size_t)r * p.n + c4));
    Z[r * 65 + c4 + 0] = (j0 + c4 + 0 <= i0 + r) ? v.x : -INFINITY;
    Z[r * 65 + c4 + 1] = (j0 + c4 + 1 <= i0 + r) ? v.y : -INFINITY;
    Z[r * 65 + c4 + 2] = (j0 + c4 + 2 <= i0 + r) ? v.z : -INFINITY;
    Z[r * 65 + c4 + 3] = (j0 + c4 + 3 <= i0 + r) ? v.w : -INFINITY;
  }
  __syncthreads();
}

// Pass 1: per (tile, head): row max and sum of exp2 over the tile's keys.
__global__ void __launch_bounds__(256) vs_pass1_kernel(const VSParams p) {
  __shared__ __align__(16) float Z[64 * 65];
  const int tile = blockIdx.x, h = blockIdx.y;
  vs_load_tile(p, h, tile, Z);
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
__global__ void __launch_bounds__(256) vs_pass2_kernel(const VSParams p) {
  __shared__ __align__(16) float Z[64 * 65];
  const int tile = blockIdx.x, h = blockIdx.y;
  vs_load_tile(p, h, tile, Z);
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

// Block distances of a head's kept offsets: a kept offset o reaches key
// blocks qb - floor(o/64) and qb - ceil(o/64) of query block qb exactly when
// that distance is <= qb (then o <= 64*qb + 63 holds).  So every query
// block's block list is {qb - delta : delta in D, delta <= qb} for one
// per-head distance set D.  One CTA per head builds D as a bitmap and as an
// ascending list.
template <int NT>
__global__ void __launch_bounds__(NT) vs_dist_kernel(const VSParams p) {
  extern __shared__ __align__(16) uint32_t dbits_s[];   // nQB bits
  __shared__ SelectSmem sm;
  const int h = blockIdx.x;
  const int nwords = (p.nQB + 31) >> 5;
  for (int w = threadIdx.x; w < nwords; w += NT) dbits_s[w] = 0u;
  __syncthreads();
  const int32_t* so = p.ssel + (size_t)h * p.n_slash;
  for (int x = threadIdx.x; x < p.n_slash; x += NT) {
    const int o = so[x];
    if (o < 0) continue;
    const int near = o >> 6, far = (o + 63) >> 6;
    if (near < p.nQB) atomicOr(&dbits_s[near >> 5], 1u << (near & 31));
    if (far < p.nQB) atomicOr(&dbits_s[far >> 5], 1u << (far & 31));
  }
  __syncthreads();
  uint32_t* dbits = p.dbits + (size_t)h * nwords;
  for (int w = threadIdx.x; w < nwords; w += NT) dbits[w] = dbits_s[w];
  const int per = (p.nQB + NT - 1) / NT;
  const int p0 = min(p.nQB, (int)threadIdx.x * per), p1 = min(p.nQB, p0 + per);
  int kept = 0;
  for (int x = p0; x < p1; ++x) kept += (dbits_s[x >> 5] >> (x & 31)) & 1u;
  int total;
  int off = block_excl_scan<NT>(kept, sm, total);
  int32_t* dlist = p.dlist + (size_t)h * p.nQB;
  for (int x = p0; x < p1; ++x)
    if ((dbits_s[x >> 5] >> (x & 31)) & 1u) dlist[off++] = x;
  if (threadIdx.x == 0) p.dcount[h] = total;
}

// Plan for (h, qb), one warp each: blocks qb - delta for the distances
// delta <= qb in ascending block order, then the kept columns j <= 64*qb+63
// whose block's distance qb - j/64 is not in D, in list order.
__global__ void __launch_bounds__(256) vs_plan_kernel(const VSParams p) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.Hq * p.nQB) return;
  const int h = row / p.nQB, qb = row % p.nQB;
  const int32_t* dlist = p.dlist + (size_t)h * p.nQB;
  const int dc = p.dcount[h];
  const uint32_t* dbits = p.dbits + (size_t)h * ((p.nQB + 31) >> 5);
  // number of distances <= qb (dlist ascending): binary search by every lane
  int lo = 0, hi = dc;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (dlist[mid] <= qb) lo = mid + 1;
    else hi = mid;
  }
  const int c = min(lo, p.kcap);
  int32_t* bout = p.block_idx + (size_t)row * p.kcap;
  for (int k = lane; k < p.kcap; k += 32) bout[k] = k < c ? qb - dlist[lo - 1 - k] : -1;
  if (lane == 0) p.block_cnt[row] = c;
  // columns: the kept columns are ascending, so j <= 64*qb+63 is a prefix
  const int32_t* vi = p.vsel + (size_t)h * p.n_vert;
  const int last = 64 * qb + 63;
  lo = 0;
  hi = p.n_vert;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (vi[mid] <= last) lo = mid + 1;
    else hi = mid;
  }
  const int m = lo;
  int32_t* cout = p.col_idx + (size_t)row * p.ccap;
  const unsigned lt = (1u << lane) - 1u;
  int off = 0;
  for (int base = 0; base < m; base += 32) {
    const int x = base + lane;
    bool keep = false;
    int j = 0;
    if (x < m) {
      j = vi[x];
      const int dist = qb - (j >> 6);
      keep = !((dbits[dist >> 5] >> (dist & 31)) & 1u);
    }
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) {
      const int slot = off + __popc(bal & lt);
      if (slot < p.ccap) cout[slot] = j;
    }
    off += __popc(bal);
  }
  for (int k = off + lane; k < p.ccap; k += 32) cout[k] = -1;
  if (lane == 0) p.col_cnt[row] = min(off, p.ccap);
}

}  // namespace dsa
