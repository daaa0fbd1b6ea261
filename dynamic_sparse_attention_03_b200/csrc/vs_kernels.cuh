// vs_kernels.cuh -- vertical-slash index (MInference 1.0 page, method section
// "方法介紹": the attention between the last queries and all keys estimates
// the vertical lines and slash lines; Fig. 4: slash lines as 64x64 blocks,
// vertical lines as 1x64 column tiles).
//
// Rows i_r = n - 64 + r.  The logits z = q_i.k_j * scale (log2 domain) of
// those rows against every key are a dense product and run on tcgen05, tiled
// 128 keys per CTA; they are computed twice and never stored.  The first pass
// keeps each row's maximum and sum of 2^z over the tile's causal keys (a
// partial per tile); the partials give each row's log-sum-exp; the second pass
// forms the probabilities P[r][j] = 2^(z - lse_r) of the tile in shared memory
// and sums them per key column (vert, complete per tile) and per diagonal
// offset o = i_r - j (slash, a partial per tile, combined over the at most two
// tiles an offset spans).  Every sum runs in a fixed order, so the scores are
// deterministic run to run.  Then a top-k per head and the per-query-block
// plan (aligned 64x64 blocks for slashes, column entries for verticals).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kVSTile = 128;              // keys per CTA of the two score passes
constexpr int kVSDiag = kVSTile + 63;     // diagonal offsets one tile touches (191)
constexpr int kVSParts = 8;               // slices of a head's scores ranked apart before the final top-k

struct VSParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  uint32_t* status;
  float* part;        // [Hq][ntiles][64][2]  pass-1 (max, sum) per tile and row (log2 domain)
  float* lse2;        // [Hq][64]
  float* vert;        // [Hq][n]
  float* slash_part;  // [Hq][ntiles][kVSDiag]
  float* slash;       // [Hq][n]
  int32_t* vsel;      // [Hq][n_vert]
  int32_t* ssel;      // [Hq][n_slash]
  int32_t* cand_id;   // [Hq][2][kVSParts][ecap] slice top-k: candidate indices, ascending
  int32_t* cand_cnt;  // [Hq][2][kVSParts]
  float* cand_val;    // [Hq][2][kVSParts * ecap] the candidates gathered in index order
  int32_t* cand_gid;  // [Hq][2][kVSParts * ecap]
  int ecap;
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

// ---------------------------------------------------------------- the score passes
// One CTA per (KV head, group of four q-heads, 128 keys): the four heads' last
// 64 query rows form two M=128 tiles (TMA, 128-byte swizzle), the key tile is
// N=128, the fp32 logits land in TMEM.  8 warps read them back, one row per
// thread (warp w: tile w / 4, TMEM lane quarter w % 4).
//   kPass = 1: each row's maximum and sum of 2^(z - max) over the tile's
//              causal keys -> part;
//   kPass = 2: P = 2^(z - lse) (0 past the causal boundary) of one tile at a
//              time into shared memory (over the operand tiles, which the MMAs
//              no longer need), then per key column the sum over the head's
//              64 rows -> vert, and per diagonal offset the tile's partial sum
//              -> slash_part.
template <int D>
struct VSScoreLayout {
  static constexpr int NDH = D / 64;
  static constexpr int kHalf = 16384;        // one d-half of 128 rows x 128 B
  static constexpr int kTile = NDH * kHalf;
  static constexpr int kQA = 0, kQB = kTile, kK = 2 * kTile;
  static constexpr int kPStride = kVSTile + 1;                 // floats per row of P (padded)
  static constexpr int kPBytes = 128 * kPStride * 4;           // one M=128 tile's P
  static constexpr int kOperands = 3 * kTile;
  static constexpr int kBar = (kOperands > kPBytes ? kOperands : kPBytes);
  static constexpr int kBytes = kBar + 64;
  static constexpr int kSmemAlloc = kBytes + 1024;
};

template <int D, int kPass>
__global__ void __launch_bounds__(256, 2)
    vs_score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const VSParams p) {
  using Lay = VSScoreLayout<D>;
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
  const int tileid = blockIdx.x, j0 = tileid * kVSTile;
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
    umma_commit(bar_mma);   // also once every operand read is done
  }
  const int tile = warp >> 2, q4 = warp & 3;
  const int row = q4 * 32 + lane;
  const int hh = 2 * tile + (row >> 6), r = row & 63;
  const int irow = p.n - 64 + r;               // this row's query position
  const int h = h0 + min(hh, nh - 1);
  const bool ok = mbar_wait_warp(bar_mma, 0, ab);
  const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16) + 128u * (uint32_t)tile;
  if (kPass == 1) {
    if (ok) {
      tc_fence_after();
      float m = -INFINITY, sum = 0.f;
#pragma unroll 1
      for (int c = 0; c < kVSTile / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(ta + 32 * c, v);
        tmem_wait_ld();
        reg_fence(v);
        float z[32];
        float mc = -INFINITY;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          z[x] = (j0 + 32 * c + x <= irow) ? __uint_as_float(v[x]) * p.scale_log2 : -INFINITY;
          mc = fmaxf(mc, z[x]);
        }
        if (mc == -INFINITY) continue;
        const float mn = fmaxf(m, mc);
        float s = 0.f;
#pragma unroll
        for (int x = 0; x < 32; ++x) s += ex2_approx(z[x] - mn);
        sum = (m == -INFINITY ? 0.f : sum * ex2_approx(m - mn)) + s;
        m = mn;
      }
      if (hh < nh) {
        float* o = p.part + (((size_t)h * p.ntiles + tileid) * 64 + r) * 2;
        o[0] = m;
        o[1] = sum;
      }
    }
  } else {
    // P of one M=128 tile at a time in shared memory (the operands are dead:
    // every MMA, and so every operand read, completed before bar_mma)
    float* P = reinterpret_cast<float*>(smem);
    const float lse = p.lse2[(size_t)h * 64 + r];
    fence_proxy_async_smem();   // the operands' async-proxy reads are ordered before these writes
    for (int t2 = 0; t2 < 2; ++t2) {
      if (tile == t2 && ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kVSTile / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(ta + 32 * c, v);
          tmem_wait_ld();
          reg_fence(v);
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const float z = __uint_as_float(v[x]) * p.scale_log2;
            P[row * Lay::kPStride + 32 * c + x] = (j0 + 32 * c + x <= irow) ? ex2_approx(z - lse) : 0.f;
          }
        }
      }
      __syncthreads();
      // the two heads of tile t2: key columns (256 sums) and diagonal partials
      for (int x = threadIdx.x; x < 2 * kVSTile; x += 256) {
        const int hx = x / kVSTile, c = x % kVSTile;
        const int hq = 2 * t2 + hx;
        if (hq < nh && j0 + c < p.n) {
          float s = 0.f;
          for (int rr = 0; rr < 64; ++rr) s += P[(hx * 64 + rr) * Lay::kPStride + c];
          p.vert[(size_t)(h0 + hq) * p.n + j0 + c] = s;
        }
      }
      for (int x = threadIdx.x; x < 2 * kVSDiag; x += 256) {
        const int hx = x / kVSDiag, od = x % kVSDiag;
        const int hq = 2 * t2 + hx;
        if (hq < nh) {
          // offset o = i_r - j = (n - 64 + r) - (j0 + c) = n - 64 - j0 - 127 + od, so c = r + 127 - od
          const int rlo = max(0, od - (kVSTile - 1)), rhi = min(63, od);
          float s = 0.f;
          for (int rr = rlo; rr <= rhi; ++rr) s += P[(hx * 64 + rr) * Lay::kPStride + (rr + kVSTile - 1 - od)];
          p.slash_part[((size_t)(h0 + hq) * p.ntiles + tileid) * kVSDiag + od] = s;
        }
      }
      __syncthreads();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Per (head, row): combine the tile partials -> lse (log2 domain).  One CTA
// per (head, row): each thread folds the tiles t = tid, tid + 128, ... in that
// order, then the threads' (max, sum) pairs are merged by a fixed tree
// (lanes by xor-shuffles, whose two sides compute the same sum, then the four
// warps in order), so the result does not depend on timing.
__device__ __forceinline__ void lse_merge(float& M, float& L, float M2, float L2) {
  if (M2 == -INFINITY) return;
  if (M == -INFINITY) {
    M = M2;
    L = L2;
  } else if (M2 > M) {
    L = L * exp2f(M - M2) + L2;
    M = M2;
  } else {
    L += L2 * exp2f(M2 - M);
  }
}

__global__ void __launch_bounds__(128) vs_lse_kernel(const VSParams p) {
  __shared__ float wm[4], wl[4];
  const int h = blockIdx.x >> 6, r = blockIdx.x & 63;
  const float* pp = p.part + ((size_t)h * p.ntiles * 64 + r) * 2;
  float M = -INFINITY, L = 0.f;
  for (int t = threadIdx.x; t < p.ntiles; t += 128) lse_merge(M, L, pp[(size_t)t * 128], pp[(size_t)t * 128 + 1]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float M2 = __shfl_xor_sync(0xFFFFFFFFu, M, o), L2 = __shfl_xor_sync(0xFFFFFFFFu, L, o);
    lse_merge(M, L, M2, L2);
  }
  if ((threadIdx.x & 31) == 0) {
    wm[threadIdx.x >> 5] = M;
    wl[threadIdx.x >> 5] = L;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    M = wm[0];
    L = wl[0];
    for (int w = 1; w < 4; ++w) lse_merge(M, L, wm[w], wl[w]);
    p.lse2[h * 64 + r] = M + log2f(L);
  }
}

// slash[o] = sum of the (at most two) tile partials covering offset o, in tile order.
__global__ void __launch_bounds__(256) vs_slash_kernel(const VSParams p) {
  const int h = blockIdx.y;
  const int o = blockIdx.x * 256 + threadIdx.x;
  if (o >= p.n) return;
  // tile t covers offsets [n - 64 - kVSTile*t - (kVSTile - 1), n - 1 - kVSTile*t]
  const int base = p.n - 64 - (kVSTile - 1);
  const int tlo = max(0, (base - o + kVSTile - 1) / kVSTile);   // ceil((base - o) / kVSTile), clamped
  const int thi = min(p.ntiles - 1, (p.n - 1 - o) / kVSTile);
  float s = 0.f;
  for (int t = tlo; t <= thi; ++t) {
    const int od = o - (base - kVSTile * t);
    if (od >= 0 && od < kVSDiag) s += p.slash_part[((size_t)h * p.ntiles + t) * kVSDiag + od];
  }
  p.slash[(size_t)h * p.n + o] = s;
}

// Top columns (first 64 forced) and top offsets (offset 0 forced) per head,
// in two launches.  The candidates (columns >= 64, offsets >= 1) of a head are
// cut into kVSParts slices and each slice keeps its own top e (the same order:
// higher score first, equal scores to the lower index); an element of the
// head's top e is beaten by fewer than e others, so it is in its slice's top e
// too.  The final top e is then taken over the slices' survivors gathered in
// index order, which the same order ranks exactly as it ranks the whole row.
template <int NT>
__global__ void __launch_bounds__(NT) vs_topk_part_kernel(const VSParams p) {
  __shared__ SelectSmem sm;
  const int h = blockIdx.x, kind = blockIdx.y, part = blockIdx.z;
  const int nf = kind == 0 ? min(64, p.n) : 1;   // ids always kept
  const float* src = (kind == 0 ? p.vert : p.slash) + (size_t)h * p.n + nf;
  const int L = p.n - nf;
  const int e = (kind == 0 ? p.n_vert : p.n_slash) - nf;
  const int per = (L + kVSParts - 1) / kVSParts;
  const int a = min(L, part * per), b = min(L, a + per);
  const size_t slot = ((size_t)h * 2 + kind) * kVSParts + part;
  int32_t* out = p.cand_id + slot * p.ecap;
  const int cnt = topk_ascending<NT>(src + a, b - a, e, 0, b - a, out, p.ecap, sm);
  __syncthreads();
  for (int j = threadIdx.x; j < cnt; j += NT) out[j] += a;   // slice positions -> candidate indices
  if (threadIdx.x == 0) p.cand_cnt[slot] = cnt;
}

template <int NT>
__global__ void __launch_bounds__(NT) vs_topk_kernel(const VSParams p) {
  __shared__ SelectSmem sm;
  __shared__ int base[kVSParts + 1];
  const int h = blockIdx.x, kind = blockIdx.y;
  const int nf = kind == 0 ? min(64, p.n) : 1;
  const float* src = (kind == 0 ? p.vert : p.slash) + (size_t)h * p.n + nf;
  const int e = (kind == 0 ? p.n_vert : p.n_slash) - nf;
  const size_t hk = (size_t)h * 2 + kind;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int y = 0; y < kVSParts; ++y) {
      base[y] = acc;
      acc += p.cand_cnt[hk * kVSParts + y];
    }
    base[kVSParts] = acc;
  }
  __syncthreads();
  const int Lc = base[kVSParts];
  float* cv = p.cand_val + hk * kVSParts * p.ecap;
  int32_t* ci = p.cand_gid + hk * kVSParts * p.ecap;
  for (int y = 0; y < kVSParts; ++y) {
    const int32_t* ids = p.cand_id + (hk * kVSParts + y) * p.ecap;
    const int c = base[y + 1] - base[y];
    for (int j = threadIdx.x; j < c; j += NT) {
      const int id = ids[j];
      ci[base[y] + j] = id;
      cv[base[y] + j] = src[id];
    }
  }
  __syncthreads();
  int32_t* out = kind == 0 ? p.vsel + (size_t)h * p.n_vert : p.ssel + (size_t)h * p.n_slash;
  const int cap = kind == 0 ? p.n_vert : p.n_slash;
  for (int j = threadIdx.x; j < nf; j += NT) out[j] = j;   // the forced ids come first
  const int cnt = topk_ascending<NT>(cv, Lc, e, 0, Lc, out + nf, cap - nf, sm);
  __syncthreads();
  for (int j = threadIdx.x; j < cnt && j < cap - nf; j += NT) out[nf + j] = ci[out[nf + j]] + nf;
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
