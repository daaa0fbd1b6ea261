// clusters.cuh -- K-means key clusters and cluster-ranked decode (Squeezed
// Attention page, "技术方案": offline, the keys of the fixed context are
// clustered with K-means, every cluster gets a centroid and every key its
// cluster; online, the query is compared with every centroid, the top
// clusters are kept and attention runs only over their keys and values).
//
// Offline build, per (batch, KV head) of the cache, over its first n_ctx keys:
//  kmeans_init_kernel:   centroid c = mean of the contiguous segment
//                        [floor(c n / C), floor((c+1) n / C)) of the keys.
//  kmeans_assign_kernel: every key to its nearest centroid (squared Euclidean
//                        distance, ties to the lower cluster): the key x
//                        centroid product on tcgen05 (256 keys per CTA, the
//                        centroids streamed 128 at a time as bf16 hi + lo
//                        halves, two products) with a running argmin of
//                        |c|^2 - 2 k.c per key.
//  kmeans_csr_kernel:    cluster -> key map: counts, offsets and the keys of
//                        each cluster in ascending token order (a stable
//                        counting sort).
//  kmeans_update_kernel: every non-empty cluster's centroid becomes the mean
//                        of its keys, summed in token order (deterministic);
//                        an empty cluster keeps its centroid.
// Lloyd rounds run (assign, csr, update) `iters` times.
//
// Online decode:
//  cluster_topk_kernel:  per (batch, q-head): the top `keep` non-empty
//                        clusters by q.c (computed for every cluster by
//                        decode_score_kernel, many CTAs), ties to the lower
//                        cluster, as a bitmap;
//  cluster_union_kernel: per (batch, KV head): the union of the group's kept
//                        clusters flattened into one token list with a
//                        per-token head mask, followed by the unclustered
//                        tail [n_ctx, S) that every head attends.
//  cluster_attn_kernel:  kClChunk entries of the union list per CTA: K and V rows
//                        read by position from the cluster-ordered copy
//                        (cluster_pack_kernel) when there is one, else
//                        gathered by token id (16-byte loads, each row read
//                        once for the whole GQA group), an online softmax per
//                        head with the token's head mask, one partial per
//                        chunk; decode_combine_kernel merges the partials.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "decode.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kKmMaxC = 4096;   // clusters per (batch, KV head)

struct KmParams {
  const __nv_bfloat16* k;   // [BG][S][D]
  float* cent;              // [BG][C][D]
  float* cnorm;             // [BG][C] |c|^2
  __nv_bfloat16* chi;       // [BG][C][D] bf16(c)          (the assignment's tensor-core operands)
  __nv_bfloat16* clo;       // [BG][C][D] bf16(c - bf16(c))
  int32_t* assign;          // [BG][n_ctx]
  int32_t* off;             // [BG][C + 1]
  int32_t* tok;             // [BG][n_ctx]
  uint32_t* status;
  int S, n_ctx, C, BG;
};

// The assignment's operands for centroid value c: hi = bf16(c), lo =
// bf16(c - hi).  Keys are bf16 exactly, so k.c = k.hi + k.lo to about 2^-17
// of |k||c| (the two products accumulate in fp32).
__device__ __forceinline__ void km_split(float c, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(c);
  lo = __float2bfloat16_rn(c - __bfloat162float(hi));
}

// ---------------------------------------------------------------- init
// One CTA of D threads per (cluster, batch x KV head): thread = dimension.
template <int D>
__global__ void __launch_bounds__(D) kmeans_init_kernel(const KmParams p) {
  __shared__ float red[D / 32];
  const int c = blockIdx.x, bg = blockIdx.y, t = threadIdx.x;
  const int lo = (int)(((int64_t)c * p.n_ctx) / p.C), hi = (int)(((int64_t)(c + 1) * p.n_ctx) / p.C);
  const __nv_bfloat16* kr = p.k + ((size_t)bg * p.S + lo) * D + t;
  float s = 0.f;
  for (int r = lo; r < hi; ++r, kr += D) s += __bfloat162float(*kr);
  const float mean = s / (float)(hi - lo);
  p.cent[((size_t)bg * p.C + c) * D + t] = mean;
  km_split(mean, p.chi[((size_t)bg * p.C + c) * D + t], p.clo[((size_t)bg * p.C + c) * D + t]);
  float sq = mean * mean;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
  if ((t & 31) == 0) red[t >> 5] = sq;
  __syncthreads();
  if (t == 0) {
    float n2 = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) n2 += red[w];
    p.cnorm[(size_t)bg * p.C + c] = n2;
  }
}

// ---------------------------------------------------------------- assign
// One CTA per (256 keys, batch x KV head).  Warp 0 loads the two 128-key
// tiles once and streams the centroids through a 2-stage ring (TMA, 128-byte
// swizzle: 128 centroids x D as bf16 hi and lo, and their |c|^2); warp 1
// issues S_t = K_t C_hi^T + K_t C_lo^T (M = 128 keys, N = 128 centroids, fp32 in
// TMEM, two buffers per key tile); warps 2-9 each own 32 keys (key tile t =
// (w - 2) / 4, TMEM lane quarter w % 4) and keep a running argmin of
// |c|^2 - 2 k.c over the chunks, which arrive in increasing centroid order (so
// ties go to the lower cluster).  Every wait is bounded.
template <int D>
struct KmAssignLayout {
  static constexpr int NDH = D / 64;
  static constexpr int kHalf = 16384;                // 128 rows x 128 B
  static constexpr int kTile = NDH * kHalf;          // 128 rows x D bf16
  static constexpr int kK = 0;                       // two key tiles
  static constexpr int kRing = 2 * kTile;            // [stage]: hi tile, lo tile
  static constexpr int kStage = 2 * kTile;
  static constexpr int kCn = kRing + 2 * kStage;     // [stage][128] |c|^2
  static constexpr int kBar = kCn + 2 * 128 * 4;
  static constexpr int kBytes = kBar + 128;
  static constexpr int kSmemAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    kmeans_assign_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmH,
                         const __grid_constant__ CUtensorMap tmL, const KmParams p) {
  using Lay = KmAssignLayout<D>;
  extern __shared__ uint8_t km_smem_raw[];
  if (status_timed_out(p.status)) return;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(km_smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + Lay::kBar;
  const uint32_t kbar = bar0;                                    // key tiles landed
  auto full = [&](int s) { return bar0 + 8u * (1 + s); };        // centroid stage landed (+ |c|^2 stored)
  auto empty = [&](int s) { return bar0 + 8u * (3 + s); };       // stage read by the MMAs
  auto sfull = [&](int b) { return bar0 + 8u * (5 + b); };       // S buffer b computed (both key tiles)
  auto sempty = [&](int b) { return bar0 + 8u * (7 + b); };      // S buffer b read by the epilogue
  const uint32_t done = bar0 + 8u * 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kBar + 80);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kBar + 84);
  float* cn_s = reinterpret_cast<float*>(smem + Lay::kCn);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.y, t0 = blockIdx.x * 256;
  const int nchunks = (p.C + 127) / 128;
  if (threadIdx.x == 0) {
    mbar_init(kbar, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(full(s), 2);   // the TMA bytes' arrival + the |c|^2 stores' arrival
      mbar_init(empty(s), 1);
      mbar_init(sfull(s), 1);
      mbar_init(sempty(s), 8);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, p.status};
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      mbar_arrive_expect_tx(kbar, (uint32_t)(2 * Lay::kTile));
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int dh = 0; dh < Lay::NDH; ++dh)
          tma_load_2d(sb + Lay::kK + t * Lay::kTile + dh * Lay::kHalf, &tmK, dh * 64, bg * p.S + t0 + 128 * t, kbar);
    }
    int c = 0;
    for (; c < nchunks; ++c) {
      const int s = c & 1;
      if (c >= 2 && !mbar_wait_warp(empty(s), ((c >> 1) - 1) & 1, ab)) break;
      const int c0 = c * 128;
      if (lane == 0) {
        mbar_arrive_expect_tx(full(s), (uint32_t)(2 * Lay::kTile));
#pragma unroll
        for (int dh = 0; dh < Lay::NDH; ++dh) {
          tma_load_2d(sb + Lay::kRing + s * Lay::kStage + dh * Lay::kHalf, &tmH, dh * 64, bg * p.C + c0, full(s));
          tma_load_2d(sb + Lay::kRing + s * Lay::kStage + Lay::kTile + dh * Lay::kHalf, &tmL, dh * 64,
                      bg * p.C + c0, full(s));
        }
      }
      // |c|^2 of the chunk (+inf past the last centroid: never the argmin),
      // once the epilogue has read this slot's values of chunk c - 2
      if (c >= 2 && !mbar_wait_warp(sempty(s), ((c >> 1) - 1) & 1, ab)) break;
      for (int x = lane; x < 128; x += 32)
        cn_s[s * 128 + x] = (c0 + x < p.C) ? p.cnorm[(size_t)bg * p.C + c0 + x] : __int_as_float(0x7f800000);
      __syncwarp();
      if (lane == 0) mbar_arrive(full(s));
    }
    // this warp's copies in flight land before the CTA exits
    if (lane == 0) {
      mbar_wait_cleanup(kbar, 0, 200000000ull);
      for (int u = max(0, c - 2); u < c; ++u) mbar_wait_cleanup(full(u & 1), (u >> 1) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (warp-uniform walk)
    const bool issuer = elect_one();
    const uint32_t idesc = umma_idesc_bf16(128, 128, 0);
    bool ok = mbar_wait_warp(kbar, 0, ab);
    for (int c = 0; c < nchunks && ok; ++c) {
      const int s = c & 1, b = c & 1;
      if (!(ok = mbar_wait_warp(full(s), (c >> 1) & 1, ab))) break;
      if (c >= 2 && !(ok = mbar_wait_warp(sempty(b), ((c >> 1) - 1) & 1, ab))) break;
      tc_fence_after();
      const uint32_t st = sb + Lay::kRing + s * Lay::kStage;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint32_t dS = tmem + 256u * (uint32_t)t + 128u * (uint32_t)b;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * Lay::kHalf + (kk & 3) * 32);
          const uint64_t a = umma_desc_sw128(sb + Lay::kK + t * Lay::kTile + off, 16, 1024);
          const uint64_t bh = umma_desc_sw128(st + off, 16, 1024);
          const uint64_t bl = umma_desc_sw128(st + Lay::kTile + off, 16, 1024);
          if (issuer) {
            umma_bf16_ss(dS, a, bh, idesc, kk > 0 ? 1u : 0u);
            umma_bf16_ss(dS, a, bl, idesc, 1u);
          }
        }
      }
      if (issuer) {
        umma_commit(empty(s));
        umma_commit(sfull(b));
      }
      __syncwarp();
    }
    if (issuer) {
      umma_commit(done);
      mbar_wait_cleanup(done, 0, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ argmin, one key per thread
    const int t = (warp - 2) >> 2, q4 = warp & 3;
    const int key = t0 + 128 * t + q4 * 32 + lane;
    const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16) + 256u * (uint32_t)t;
    float best = __int_as_float(0x7f800000);
    int bidx = 0;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int b = c & 1;
      if (!(ok = mbar_wait_warp(sfull(b), (c >> 1) & 1, ab))) break;
      // the |c|^2 stores are acquired from the producer's own arrival (the
      // slot cannot move on to chunk c + 2 before this warp releases chunk c)
      if (!(ok = mbar_wait_warp(full(c & 1), (c >> 1) & 1, ab))) break;
      tc_fence_after();
      const float* cn = cn_s + (c & 1) * 128;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t v[32];
        tmem_ld32(ta + 128u * (uint32_t)b + 32u * (uint32_t)q, v);
        tmem_wait_ld();
        reg_fence(v);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float dist = fmaf(-2.f, __uint_as_float(v[x]), cn[32 * q + x]);
          if (dist < best) {   // centroids in increasing order: ties keep the lower one
            best = dist;
            bidx = c * 128 + 32 * q + x;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty(b));
    }
    if (ok && key < p.n_ctx) p.assign[(size_t)bg * p.n_ctx + key] = bidx;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- cluster -> key map
// One CTA of 1024 threads per (batch x KV head): counts with shared atomics,
// a block scan for the offsets, then one warp scatters the tokens in order,
// 32 at a time: lanes with the same cluster (match_any) take consecutive
// places after that cluster's cursor, lower lanes (lower tokens) first.
__global__ void __launch_bounds__(1024) kmeans_csr_kernel(const KmParams p) {
  __shared__ int cnt[kKmMaxC];
  __shared__ int wsum[32];
  const int bg = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* as = p.assign + (size_t)bg * p.n_ctx;
  int32_t* off = p.off + (size_t)bg * (p.C + 1);
  int32_t* tok = p.tok + (size_t)bg * p.n_ctx;
  for (int c = tid; c < p.C; c += 1024) cnt[c] = 0;
  __syncthreads();
  for (int t = tid; t < p.n_ctx; t += 1024) atomicAdd(&cnt[as[t]], 1);
  __syncthreads();
  // exclusive scan of cnt[0..C): each thread a contiguous range
  const int per = (p.C + 1023) / 1024;
  const int c0 = min(p.C, tid * per), c1 = min(p.C, c0 + per);
  int s = 0;
  for (int c = c0; c < c1; ++c) s += cnt[c];
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = wsum[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += v;
    }
    wsum[lane] = wi - w;
  }
  __syncthreads();
  int run = wsum[warp] + incl - s;
  for (int c = c0; c < c1; ++c) {
    const int k = cnt[c];
    off[c] = run;
    cnt[c] = run;   // becomes the cluster's write cursor
    run += k;
  }
  if (tid == 0) off[p.C] = p.n_ctx;
  __syncthreads();
  if (warp == 0) {
    for (int t0 = 0; t0 < p.n_ctx; t0 += 32) {
      const int t = t0 + lane;
      const bool ok = t < p.n_ctx;
      const int c = ok ? as[t] : -1 - lane;   // distinct negative keys for idle lanes
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, c);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      int base = 0;
      if (ok && lane == leader) base = cnt[c];
      base = __shfl_sync(0xFFFFFFFFu, base, leader);
      if (ok) tok[base + rank] = t;
      __syncwarp();
      if (ok && lane == leader) cnt[c] = base + __popc(peers);
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------- update
// One warp per (cluster, batch x KV head), 8 per CTA: lanes own D / 32
// dimensions; the cluster's keys are summed in token order.
template <int D>
__global__ void __launch_bounds__(256) kmeans_update_kernel(const KmParams p) {
  constexpr int PER = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 8 + warp, bg = blockIdx.y;
  if (c >= p.C) return;
  const int32_t* off = p.off + (size_t)bg * (p.C + 1);
  const int a = off[c], b = off[c + 1];
  if (a == b) return;   // empty: keeps its centroid (and |c|^2)
  const int32_t* tok = p.tok + (size_t)bg * p.n_ctx;
  float s[PER];
#pragma unroll
  for (int x = 0; x < PER; ++x) s[x] = 0.f;
  for (int q = a; q < b; ++q) {
    const __nv_bfloat16* kr = p.k + ((size_t)bg * p.S + tok[q]) * D + lane * PER;
    if (PER == 4) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(kr));
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      const float2 v0 = __bfloat1622float2(h2[0]), v1 = __bfloat1622float2(h2[1]);
      s[0] += v0.x;
      s[1 % PER] += v0.y;
      s[2 % PER] += v1.x;
      s[3 % PER] += v1.y;
    } else {
      const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(kr);
      const float2 v0 = __bfloat1622float2(h2);
      s[0] += v0.x;
      s[1 % PER] += v0.y;
    }
  }
  const float inv = 1.f / (float)(b - a);
  float sq = 0.f;
  float* out = p.cent + ((size_t)bg * p.C + c) * D + lane * PER;
  const size_t o2 = ((size_t)bg * p.C + c) * D + lane * PER;
#pragma unroll
  for (int x = 0; x < PER; ++x) {
    const float m = s[x] * inv;
    out[x] = m;
    km_split(m, p.chi[o2 + x], p.clo[o2 + x]);
    sq = fmaf(m, m, sq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
  if (lane == 0) p.cnorm[(size_t)bg * p.C + c] = sq;
}

// ---------------------------------------------------------------- decode: select
struct ClusterParams {
  DecodeParams dp;          // q, kc, vc, o, sel_idx, sel_cnt, uidx (union tokens), umask, ucnt, partials
  const float* cent;        // [BG][C][D]
  const int32_t* off;       // [BG][C + 1]
  const int32_t* tok;       // [BG][n_ctx]
  const float* scores;      // [B * Hq][C] q.c of every cluster (decode_score_kernel)
  int C, n_ctx;
};

// Two launches, so the top-k of every q-head runs in parallel: one CTA per
// (batch, q-head) ranks the (batch, KV head)'s non-empty clusters by that
// head's scores, keeps `keep` of them (ties to the lower cluster) and writes
// them as a bitmap over cluster ids (and the optional selection outputs); one
// CTA per (batch, KV head) ORs the group's bitmaps and flattens the kept
// clusters into one token list with a per-token head mask (clusters in id
// order, each cluster's tokens as the cluster -> key map lists them), then the
// unclustered tail [n_ctx, S) that every head attends.
template <int NT>
__global__ void __launch_bounds__(NT) cluster_topk_kernel(const ClusterParams cp) {
  extern __shared__ __align__(16) uint8_t csm[];
  __shared__ SelectSmem sm;
  const DecodeParams& p = cp.dp;
  const int bh = blockIdx.x;   // b * Hq + h
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.grp;
  const int bg = b * p.Hkv + g;
  const int C = cp.C, nw = (C + 31) >> 5;
  float* sc = reinterpret_cast<float*>(csm);                    // [C] candidates' scores
  int32_t* cand = reinterpret_cast<int32_t*>(sc + C);           // [C] non-empty cluster ids
  int32_t* tmp = cand + C;                                      // [C]
  int32_t* off = tmp + C;                                       // [C + 1]
  uint32_t* bits = reinterpret_cast<uint32_t*>(off + C + 1);    // [nw]
  const int32_t* goff = cp.off + (size_t)bg * (C + 1);
  for (int x = threadIdx.x; x <= C; x += NT) off[x] = goff[x];
  for (int x = threadIdx.x; x < nw; x += NT) bits[x] = 0u;
  __syncthreads();
  // non-empty clusters, ascending (block scan over per-thread ranges)
  const int per = (C + NT - 1) / NT;
  const int c0 = min(C, (int)threadIdx.x * per), c1 = min(C, c0 + per);
  int ne = 0;
  for (int c = c0; c < c1; ++c) ne += off[c + 1] > off[c];
  int ncand;
  int pos = block_excl_scan<NT>(ne, sm, ncand);
  for (int c = c0; c < c1; ++c)
    if (off[c + 1] > off[c]) cand[pos++] = c;
  __syncthreads();
  const float* gsc = cp.scores + (size_t)bh * C;
  for (int y = threadIdx.x; y < ncand; y += NT) sc[y] = gsc[cand[y]];
  __syncthreads();
  const int e = min(p.keep, ncand);
  const int cnt = topk_ascending<NT>(sc, ncand, e, 0, ncand, tmp, C, sm);
  __syncthreads();
  for (int x = threadIdx.x; x < cnt; x += NT) {
    const int c = cand[tmp[x]];
    atomicOr(&bits[c >> 5], 1u << (c & 31));
  }
  if (p.sel_idx) {
    int32_t* out = p.sel_idx + (size_t)bh * p.kcap;
    for (int x = threadIdx.x; x < p.kcap; x += NT) out[x] = x < cnt ? cand[tmp[x]] : -1;
  }
  if (p.sel_cnt && threadIdx.x == 0) p.sel_cnt[bh] = cnt;
  __syncthreads();
  uint32_t* gb = p.kbits + (size_t)bh * nw;
  for (int x = threadIdx.x; x < nw; x += NT) gb[x] = bits[x];
}

template <int GRP, int NT>
__global__ void __launch_bounds__(NT) cluster_union_kernel(const ClusterParams cp) {
  extern __shared__ __align__(16) uint8_t csm[];
  __shared__ SelectSmem sm;
  const DecodeParams& p = cp.dp;
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int C = cp.C, nw = (C + 31) >> 5;
  int32_t* off = reinterpret_cast<int32_t*>(csm);   // [C + 1] the cluster -> key offsets
  int32_t* ubase = off + C + 1;                     // [C] union token offsets
  uint8_t* mask = reinterpret_cast<uint8_t*>(ubase + C);   // [C]
  const int32_t* goff = cp.off + (size_t)bg * (C + 1);
  for (int x = threadIdx.x; x <= C; x += NT) off[x] = goff[x];
  const uint32_t* gb = p.kbits + ((size_t)b * p.Hq + g * GRP) * nw;   // the group's rows are contiguous
  for (int c = threadIdx.x; c < C; c += NT) {
    uint32_t m = 0u;
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) m |= ((gb[(size_t)hh * nw + (c >> 5)] >> (c & 31)) & 1u) << hh;
    mask[c] = (uint8_t)m;
  }
  __syncthreads();
  const int per = (C + NT - 1) / NT;
  const int c0 = min(C, (int)threadIdx.x * per), c1 = min(C, c0 + per);
  int sz = 0;
  for (int c = c0; c < c1; ++c) sz += mask[c] ? off[c + 1] - off[c] : 0;
  int total;
  int ub = block_excl_scan<NT>(sz, sm, total);
  for (int c = c0; c < c1; ++c) {
    ubase[c] = ub;
    if (mask[c]) ub += off[c + 1] - off[c];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* ui = p.uidx + (size_t)bg * p.nb;
  uint8_t* um = p.umask + (size_t)bg * p.nb;
  const int32_t* tk = cp.tok + (size_t)bg * cp.n_ctx;
  const bool packed = p.n_packed > 0;   // positions in the cluster-ordered copy, else token ids
  for (int x = warp; x < C; x += NT / 32) {
    if (!mask[x]) continue;
    const int a = off[x], n = off[x + 1] - a, dst = ubase[x];
    for (int y = lane; y < n; y += 32) {
      ui[dst + y] = packed ? a + y : tk[a + y];
      um[dst + y] = mask[x];
    }
  }
  const int ntail = p.S - cp.n_ctx;
  const uint8_t all = (uint8_t)((1u << GRP) - 1u);
  for (int y = threadIdx.x; y < ntail; y += NT) {
    ui[total + y] = cp.n_ctx + y;
    um[total + y] = all;
  }
  if (threadIdx.x == 0) p.ucnt[bg] = total + ntail;
}

// ---------------------------------------------------------------- decode: attention over the union
// One CTA of 4 warps per (batch x KV head, kClChunk tokens of the union list),
// walking them SUB = 8 TPL at a time: warp w takes tokens 2 TPL w .. of each
// step, the two half warps alternate tokens (TPL tokens per lane: 8, or 4 for
// 8 q-heads per KV head to bound registers), lane % 16 owns D / 16 dims; rows
// are gathered straight from global memory with 16-byte (8-byte at D = 64)
// loads, and an online softmax per (lane, head) runs over the whole chunk.
constexpr int kClChunk = 4096;

template <int D, int GRP>
__global__ void __launch_bounds__(128) cluster_attn_kernel(const DecodeParams p) {
  __shared__ float red[4][kMaxGrp][D + 2];
  const int bg = blockIdx.x, chunk = blockIdx.y;
  const int cnt = p.ucnt[bg];
  const int c0 = chunk * kClChunk;
  if (c0 >= cnt) return;
  const int c1 = min(cnt, c0 + kClChunk);
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int DPL = D / 16;
  const int half = lane >> 4, dl = lane & 15;
  const int32_t* ui = p.uidx + (size_t)bg * p.nb;
  const uint8_t* um = p.umask + (size_t)bg * p.nb;
  const size_t head_base = (size_t)bg * p.S * D;
  float qv[GRP][DPL];
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh)
#pragma unroll
    for (int a = 0; a < DPL; ++a)
      qv[hh][a] = __bfloat162float(p.q[((size_t)b * p.Hq + g * GRP + hh) * D + dl * DPL + a]) * p.scale_log2;
  float m[GRP], l[GRP], acc[GRP][DPL];
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int a = 0; a < DPL; ++a) acc[hh][a] = 0.f;
  }
  constexpr int TPL = GRP >= 8 ? 4 : 8;
  for (int u0 = c0; u0 < c1; u0 += 8 * TPL) {
    // this lane's TPL tokens: union positions u0 + 2 TPL w + 2 it + half
    float kf[TPL][DPL], vf[TPL][DPL];
    uint32_t msk[TPL];
#pragma unroll
    for (int it = 0; it < TPL; ++it) {
      const int u = u0 + 2 * TPL * warp + 2 * it + half;
      msk[it] = 0u;
#pragma unroll
      for (int a = 0; a < DPL; ++a) {
        kf[it][a] = 0.f;
        vf[it][a] = 0.f;
      }
      if (u < c1) {
        msk[it] = um[u];
        // entries below n_packed index the cluster-ordered copy, the rest the cache
        const int idx = ui[u];
        const bool pk = idx < p.n_packed;
        const size_t row = (pk ? ((size_t)bg * p.n_packed + idx) * D : head_base + (size_t)idx * D) + dl * DPL;
        const __nv_bfloat16* kb = pk ? p.kp : p.kc;
        const __nv_bfloat16* vb = pk ? p.vp : p.vc;
        if (DPL == 8) {
          const uint4 kr = __ldg(reinterpret_cast<const uint4*>(kb + row));
          const uint4 vr = __ldg(reinterpret_cast<const uint4*>(vb + row));
          const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
          const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const float2 kk = __bfloat1622float2(k2[a]), vv = __bfloat1622float2(v2[a]);
            kf[it][(2 * a) % DPL] = kk.x;
            kf[it][(2 * a + 1) % DPL] = kk.y;
            vf[it][(2 * a) % DPL] = vv.x;
            vf[it][(2 * a + 1) % DPL] = vv.y;
          }
        } else {
          const uint2 kr = __ldg(reinterpret_cast<const uint2*>(kb + row));
          const uint2 vr = __ldg(reinterpret_cast<const uint2*>(vb + row));
          const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
          const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const float2 kk = __bfloat1622float2(k2[a]), vv = __bfloat1622float2(v2[a]);
            kf[it][(2 * a) % DPL] = kk.x;
            kf[it][(2 * a + 1) % DPL] = kk.y;
            vf[it][(2 * a) % DPL] = vv.x;
            vf[it][(2 * a + 1) % DPL] = vv.y;
          }
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
      float sc[TPL];
#pragma unroll
      for (int it = 0; it < TPL; ++it) {
        float d0 = 0.f;
#pragma unroll
        for (int a = 0; a < DPL; ++a) d0 = fmaf(qv[hh][a], kf[it][a], d0);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) d0 += __shfl_xor_sync(0xFFFFFFFFu, d0, o);
        sc[it] = ((msk[it] >> hh) & 1u) ? d0 : -INFINITY;
      }
      float mb = sc[0];
#pragma unroll
      for (int it = 1; it < TPL; ++it) mb = fmaxf(mb, sc[it]);
      mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 16));
      const float mn = fmaxf(m[hh], mb);
      if (mn == -INFINITY) continue;   // nothing of this head yet (warp-uniform)
      const float alpha = ex2_approx(m[hh] - mn);   // m = -inf -> 0
      float ls = 0.f;
#pragma unroll
      for (int a = 0; a < DPL; ++a) acc[hh][a] *= alpha;
#pragma unroll
      for (int it = 0; it < TPL; ++it) {
        const float pe = ex2_approx(sc[it] - mn);   // -inf -> 0
        ls += pe;
#pragma unroll
        for (int a = 0; a < DPL; ++a) acc[hh][a] = fmaf(pe, vf[it][a], acc[hh][a]);
      }
      l[hh] = l[hh] * alpha + ls;
      m[hh] = mn;
    }
  }
  // merge the half warps (same dims, same running max), then the 4 warps
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) {
    l[hh] += __shfl_xor_sync(0xFFFFFFFFu, l[hh], 16);
#pragma unroll
    for (int a = 0; a < DPL; ++a) acc[hh][a] += __shfl_xor_sync(0xFFFFFFFFu, acc[hh][a], 16);
    if (half == 0) {
#pragma unroll
      for (int a = 0; a < DPL; ++a) red[warp][hh][dl * DPL + a] = acc[hh][a];
    }
    if (lane == 0) {
      red[warp][hh][D] = m[hh];
      red[warp][hh][D + 1] = l[hh];
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < GRP * D; x += 128) {
    const int hh = x / D, c = x % D;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red[w][hh][D]);
    float a = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < 4; ++w) {
        if (red[w][hh][D] == -INFINITY) continue;
        const float wgt = ex2_approx(red[w][hh][D] - M);
        a += wgt * red[w][hh][c];
        L += wgt * red[w][hh][D + 1];
      }
    }
    const size_t ph = (size_t)b * p.Hq + g * GRP + hh;
    p.part_acc[(ph * p.nchmax + chunk) * D + c] = a;
    if (c == 0) {
      p.part_ml[(ph * p.nchmax + chunk) * 2 + 0] = M;
      p.part_ml[(ph * p.nchmax + chunk) * 2 + 1] = L;
    }
  }
}

// ---------------------------------------------------------------- decode: streamed union
// With the cluster-ordered copy, the union list is a few long runs of
// consecutive rows (kept clusters, then the tail), so it streams like the
// block decode: per CTA kClChunk entries in units of 64; the producer warp
// finds the runs of a unit (ballots over consecutive positions) and lane 0
// bulk-copies each run's K and V rows into a ring stage (one copy per run and
// operand, the stage's byte count expected up front); the consumer warps
// score the unit's rows for the group's q-heads with each row's head mask
// and keep an online softmax per (warp, head), as decode_attn_kernel does,
// but eight of them with four rows per lane (fewer registers, two warps per
// scheduler, and a head is skipped for any 8-row slice none of whose rows it
// kept).
constexpr int kClWarps = 8;   // consumer warps: 8 rows of each unit per warp, 4 per lane

template <int D>
struct ClStreamLayout {
  static constexpr int kBlkBytes = 64 * D * 2;                  // 64 K (or V) rows
  static constexpr int kStage = 2 * kBlkBytes;
  static constexpr int kRed = kDecStages * kStage;              // warp partials [warp][head][D + 2]
  static constexpr int kRedBytes = kClWarps * kMaxGrp * (D + 2) * 4;
  static constexpr int kList = kRed + kRedBytes;                // the chunk's list entries (kClChunk ints)
  static constexpr int kMask = kList + kClChunk * 4;            // and their head masks (kClChunk bytes)
  static constexpr int kBar = kMask + kClChunk;
  static constexpr int kBytes = kBar + (2 * kDecStages + 1) * 8 + 16;
};

template <int D, int GRP>
__global__ void __launch_bounds__((kClWarps + 1) * 32, 1) cluster_stream_attn_kernel(const DecodeParams p) {
  using Lay = ClStreamLayout<D>;
  constexpr int NW = kClWarps, TPL = 32 / NW;   // rows per lane per unit
  extern __shared__ __align__(16) uint8_t dsm[];
  const uint32_t sb = smem_u32(dsm);
  const int bg = blockIdx.x, chunk = blockIdx.y;
  const int cnt = p.ucnt[bg];
  const int e0 = chunk * kClChunk;
  if (e0 >= cnt || status_timed_out(p.status)) return;
  const int e1 = min(cnt, e0 + kClChunk);
  const int nu = (e1 - e0 + 63) / 64;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = sb + Lay::kBar;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kDecStages + s); };
  const uint32_t lbar = bar0 + 8u * (2 * kDecStages);   // the chunk's list and masks landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + Lay::kBar + (2 * kDecStages + 1) * 8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), NW);
    }
    mbar_init(lbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const AbortState ab{abort_flag, p.status};
  const int32_t* ui_s = reinterpret_cast<const int32_t*>(dsm + Lay::kList);   // entries e0 .. e1 - 1
  const uint8_t* um_s = dsm + Lay::kMask;
  constexpr uint32_t kRowBytes = D * 2;

  if (warp == NW) {
    // producer warp: the chunk's list entries and head masks come in once
    // (two bulk copies; the list rows are padded to 16 entries, so the rounded
    // sizes stay inside them), then the runs of consecutive positions of each
    // unit are found in shared memory
    if (lane == 0) {
      const uint32_t nl = (uint32_t)((e1 - e0 + 3) & ~3) * 4u, nm = (uint32_t)((e1 - e0 + 15) & ~15);
      mbar_arrive_expect_tx(lbar, nl + nm);
      bulk_load(sb + Lay::kList, p.uidx + (size_t)bg * p.nb + e0, nl, lbar);
      bulk_load(sb + Lay::kMask, p.umask + (size_t)bg * p.nb + e0, nm, lbar);
    }
    bool lok = mbar_wait_warp(lbar, 0, ab);
    int u = 0;
    for (; u < nu && lok; ++u) {
      const int s = u % kDecStages;
      if (u >= kDecStages && !mbar_wait_warp(empty(s), ((u / kDecStages) - 1) & 1, ab)) break;
      const int rb = e0 + 64 * u, rows = min(64, e1 - rb);
      const int pa = lane < rows ? ui_s[64 * u + lane] : -1;
      const int pb = lane + 32 < rows ? ui_s[64 * u + lane + 32] : -1;
      const int up_a = __shfl_up_sync(0xFFFFFFFFu, pa, 1), last_a = __shfl_sync(0xFFFFFFFFu, pa, 31);
      const int up_b = __shfl_up_sync(0xFFFFFFFFu, pb, 1);
      const int prev_b = lane == 0 ? last_a : up_b;
      // a run starts at row 0, after a gap, and where the cache tail begins
      // (positions below n_packed are in the copy, the rest in the cache)
      const bool st_a = lane < rows && (lane == 0 || pa != up_a + 1 || pa == p.n_packed);
      const bool st_b = lane + 32 < rows && (pb != prev_b + 1 || pb == p.n_packed);
      uint64_t starts = (uint64_t)__ballot_sync(0xFFFFFFFFu, st_a) | ((uint64_t)__ballot_sync(0xFFFFFFFFu, st_b) << 32);
      if (lane == 0) mbar_arrive_expect_tx(full(s), (uint32_t)rows * 2u * kRowBytes);
      while (starts) {   // warp-uniform
        const int r = __ffsll((long long)starts) - 1;
        starts &= starts - 1ull;
        const int rn = starts ? __ffsll((long long)starts) - 1 : rows;
        const int pos = __shfl_sync(0xFFFFFFFFu, r < 32 ? pa : pb, r & 31);
        if (lane == 0) {
          const bool pk = pos < p.n_packed;
          const size_t src = (pk ? (size_t)bg * p.n_packed : (size_t)bg * p.S) * D + (size_t)pos * D;
          const uint32_t bytes = (uint32_t)(rn - r) * kRowBytes;
          const uint32_t dst = sb + s * Lay::kStage + (uint32_t)r * kRowBytes;
          bulk_load(dst, (pk ? p.kp : p.kc) + src, bytes, full(s));
          bulk_load(dst + Lay::kBlkBytes, (pk ? p.vp : p.vc) + src, bytes, full(s));
        }
      }
      __syncwarp();
    }
    if (lane == 0) {
      if (!lok) mbar_wait_cleanup(lbar, 0, 200000000ull);
      for (int w = max(0, u - kDecStages); w < u; ++w)
        mbar_wait_cleanup(full(w % kDecStages), (w / kDecStages) & 1, 200000000ull);
    }
    return;
  }
  // consumers: warp w takes rows 2 TPL w .. of every unit; the two half
  // warps take alternate rows, lane%16 owns dims [DPL*(lane%16), +DPL)
  // (dot products and P.V updates as packed f32x2 multiply-adds on pairs of dims)
  constexpr int DPL = D / 16, DP2 = DPL / 2;
  const int half = lane >> 4, dl = lane & 15;
  float2 qv[GRP][DP2];
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh)
#pragma unroll
    for (int j = 0; j < DP2; ++j) {
      const __nv_bfloat16* qr = p.q + ((size_t)b * p.Hq + g * GRP + hh) * D + dl * DPL + 2 * j;
      qv[hh][j] = make_float2(__bfloat162float(qr[0]) * p.scale_log2, __bfloat162float(qr[1]) * p.scale_log2);
    }
  float m[GRP], l[GRP];
  float2 acc[GRP][DP2];
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int j = 0; j < DP2; ++j) acc[hh][j] = make_float2(0.f, 0.f);
  }
  bool ok = mbar_wait_warp(lbar, 0, ab);
  for (int u = 0; u < nu && ok; ++u) {
    const int s = u % kDecStages;
    const int rb = e0 + 64 * u, rows = min(64, e1 - rb);
    if (!mbar_wait_warp(full(s), (u / kDecStages) & 1, ab)) {
      ok = false;
      break;
    }
    const uint8_t* ms = um_s + 64 * u;
    uint32_t msk[TPL];
    uint32_t mor = 0u;
#pragma unroll
    for (int it = 0; it < TPL; ++it) {
      const int key = 2 * TPL * warp + 2 * it + half;
      msk[it] = key < rows ? (uint32_t)ms[key] : 0u;
      mor |= msk[it];
    }
    mor = __reduce_or_sync(0xFFFFFFFFu, mor);
    const uint8_t* kb = dsm + s * Lay::kStage;
    const uint8_t* vb = kb + Lay::kBlkBytes;
    float2 kf[TPL][DP2], vf[TPL][DP2];
#pragma unroll
    for (int it = 0; it < TPL; ++it) {
      const int key = 2 * TPL * warp + 2 * it + half;
      // rows past the unit's end hold stale bytes (the stage has room for 64
      // rows, so the loads stay inside it): their words are zeroed
      const uint32_t keep = key < rows ? 0xFFFFFFFFu : 0u;
      if constexpr (DPL == 8) {
        uint4 kr = *reinterpret_cast<const uint4*>(kb + key * kRowBytes + dl * 16);
        uint4 vr = *reinterpret_cast<const uint4*>(vb + key * kRowBytes + dl * 16);
        kr.x &= keep; kr.y &= keep; kr.z &= keep; kr.w &= keep;
        vr.x &= keep; vr.y &= keep; vr.z &= keep; vr.w &= keep;
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          kf[it][j] = __bfloat1622float2(k2[j]);
          vf[it][j] = __bfloat1622float2(v2[j]);
        }
      } else {
        uint2 kr = *reinterpret_cast<const uint2*>(kb + key * kRowBytes + dl * 8);
        uint2 vr = *reinterpret_cast<const uint2*>(vb + key * kRowBytes + dl * 8);
        kr.x &= keep; kr.y &= keep;
        vr.x &= keep; vr.y &= keep;
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          kf[it][j % DP2] = __bfloat1622float2(k2[j]);
          vf[it][j % DP2] = __bfloat1622float2(v2[j]);
        }
      }
    }
    // release the stage once every warp has its registers
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
      if (!((mor >> hh) & 1u)) continue;   // no row of the unit kept by this head (warp-uniform)
      float sc[TPL];
#pragma unroll
      for (int it = 0; it < TPL; ++it) {
        float2 t = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < DP2; ++j) t = ffma2(qv[hh][j], kf[it][j], t);
        float d0 = t.x + t.y;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) d0 += __shfl_xor_sync(0xFFFFFFFFu, d0, o);
        sc[it] = ((msk[it] >> hh) & 1u) ? d0 : -INFINITY;
      }
      float mb = sc[0];
#pragma unroll
      for (int it = 1; it < TPL; ++it) mb = fmaxf(mb, sc[it]);
      mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 16));
      const float mn = fmaxf(m[hh], mb);
      if (mn == -INFINITY) continue;   // nothing of this head in this warp yet (warp-uniform)
      const float alpha = ex2_approx(m[hh] - mn);   // m = -inf -> 0
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < DP2; ++j) acc[hh][j] = fmul2(acc[hh][j], make_float2(alpha, alpha));
#pragma unroll
      for (int it = 0; it < TPL; ++it) {
        const float pe = ex2_approx(sc[it] - mn);   // -inf -> 0
        ls += pe;
#pragma unroll
        for (int j = 0; j < DP2; ++j) acc[hh][j] = ffma2(make_float2(pe, pe), vf[it][j], acc[hh][j]);
      }
      l[hh] = l[hh] * alpha + ls;
      m[hh] = mn;
    }
  }
  // merge the two half-warps (same dims, same running max), then the NW warps
  float* red = reinterpret_cast<float*>(dsm + Lay::kRed);   // [warp][hh][D + 2]
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) {
    l[hh] += __shfl_xor_sync(0xFFFFFFFFu, l[hh], 16);
#pragma unroll
    for (int j = 0; j < DP2; ++j) {
      acc[hh][j].x += __shfl_xor_sync(0xFFFFFFFFu, acc[hh][j].x, 16);
      acc[hh][j].y += __shfl_xor_sync(0xFFFFFFFFu, acc[hh][j].y, 16);
    }
    float* r = red + ((size_t)warp * kMaxGrp + hh) * (D + 2);
    if (half == 0) {
#pragma unroll
      for (int j = 0; j < DP2; ++j) {
        r[dl * DPL + 2 * j] = acc[hh][j].x;
        r[dl * DPL + 2 * j + 1] = acc[hh][j].y;
      }
    }
    if (lane == 0) {
      r[D] = m[hh];
      r[D + 1] = l[hh];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
  if (!ok) return;
  for (int x = threadIdx.x; x < GRP * D; x += NW * 32) {
    const int hh = x / D, c = x % D;
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[((size_t)w * kMaxGrp + hh) * (D + 2) + D]);
    float a = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < NW; ++w) {
        const float* r = red + ((size_t)w * kMaxGrp + hh) * (D + 2);
        if (r[D] == -INFINITY) continue;
        const float wgt = ex2_approx(r[D] - M);
        a += wgt * r[c];
        L += wgt * r[D + 1];
      }
    }
    const size_t ph = (size_t)b * p.Hq + g * GRP + hh;
    p.part_acc[(ph * p.nchmax + chunk) * D + c] = a;
    if (c == 0) {
      p.part_ml[(ph * p.nchmax + chunk) * 2 + 0] = M;
      p.part_ml[(ph * p.nchmax + chunk) * 2 + 1] = L;
    }
  }
}

// ---------------------------------------------------------------- cluster-ordered copy
// kp[bg][pos] = k[bg][tokens[bg][pos]] (and v) for pos < n_ctx: one warp per
// position, lanes 0-15 copy the K row and lanes 16-31 the V row (16-byte
// vectors at D = 128, 8-byte at D = 64); the reads gather rows, the writes
// stream.  Done once per fixed context, so the decode reads each kept
// cluster as one contiguous range.
template <int D>
__global__ void __launch_bounds__(256) cluster_pack_kernel(const __nv_bfloat16* __restrict__ k,
                                                           const __nv_bfloat16* __restrict__ v,
                                                           const int32_t* __restrict__ tok, int S, int n_ctx,
                                                           __nv_bfloat16* __restrict__ kp,
                                                           __nv_bfloat16* __restrict__ vp) {
  const int bg = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pos = blockIdx.x * 8 + warp;
  if (pos >= n_ctx) return;
  const int t = tok[(size_t)bg * n_ctx + pos];
  const int half = lane >> 4, l16 = lane & 15;
  const __nv_bfloat16* src = (half ? v : k) + ((size_t)bg * S + t) * D;
  __nv_bfloat16* dst = (half ? vp : kp) + ((size_t)bg * n_ctx + pos) * D;
  if constexpr (D == 128) {
    reinterpret_cast<uint4*>(dst)[l16] = __ldg(reinterpret_cast<const uint4*>(src) + l16);
  } else {
    reinterpret_cast<uint2*>(dst)[l16] = __ldg(reinterpret_cast<const uint2*>(src) + l16);
  }
}

}  // namespace dsa
