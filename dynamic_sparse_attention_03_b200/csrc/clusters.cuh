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
//                        distance, ties to the lower cluster): a tiled fp32
//                        key x centroid product (128 keys x 64 centroids per
//                        step) with a running argmin of |c|^2 - 2 k.c.
//  kmeans_csr_kernel:    cluster -> key map: counts, offsets and the keys of
//                        each cluster in ascending token order (a stable
//                        counting sort).
//  kmeans_update_kernel: every non-empty cluster's centroid becomes the mean
//                        of its keys, summed in token order (deterministic);
//                        an empty cluster keeps its centroid.
// Lloyd rounds run (assign, csr, update) `iters` times.
//
// Online decode:
//  cluster_select_kernel: per (batch, KV head): the scores of the non-empty
//                        clusters (q.c for every cluster comes from
//                        decode_score_kernel, many CTAs), the top `keep` per head
//                        (ties to the lower cluster), and the union of the
//                        group's kept clusters flattened into one token list
//                        with a per-token head mask, followed by the
//                        unclustered tail [n_ctx, S) that every head attends.
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
  int32_t* assign;          // [BG][n_ctx]
  int32_t* off;             // [BG][C + 1]
  int32_t* tok;             // [BG][n_ctx]
  int S, n_ctx, C;
};

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
// One CTA of 256 threads per (128 keys, batch x KV head).  Shared memory
// holds the key tile transposed ([D][128] fp32) and a centroid chunk
// transposed ([D][64]); thread (ty, tx) = (tid / 16, tid % 16) owns keys
// 8 ty .. 8 ty + 7 and centroids 4 tx .. 4 tx + 3 of the chunk.
template <int D>
struct KmAssignLayout {
  static constexpr int kKeys = 0;
  static constexpr int kCent = D * 128 * 4;
  static constexpr int kBytes = kCent + D * 64 * 4;
};

template <int D>
__global__ void __launch_bounds__(256) kmeans_assign_kernel(const KmParams p) {
  using Lay = KmAssignLayout<D>;
  extern __shared__ __align__(16) uint8_t kas[];
  float* ks = reinterpret_cast<float*>(kas + Lay::kKeys);   // [D][128]
  float* cs = reinterpret_cast<float*>(kas + Lay::kCent);   // [D][64]
  const int bg = blockIdx.y, t0 = blockIdx.x * 128;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  // key tile, transposed (rows past n_ctx are zero and never written back)
  for (int x = tid; x < 128 * D / 8; x += 256) {
    const int row = x / (D / 8), c8 = x % (D / 8);
    float f[8];
    if (t0 + row < p.n_ctx) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.k + ((size_t)bg * p.S + t0 + row) * D) + c8);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float2 v = __bfloat1622float2(h2[a]);
        f[2 * a] = v.x;
        f[2 * a + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int a = 0; a < 8; ++a) f[a] = 0.f;
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) ks[(c8 * 8 + a) * 128 + row] = f[a];
  }
  float best[8];
  int bidx[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    best[r] = __int_as_float(0x7f800000);
    bidx[r] = 0;
  }
  const float* cent = p.cent + (size_t)bg * p.C * D;
  const float* cn = p.cnorm + (size_t)bg * p.C;
  for (int c0 = 0; c0 < p.C; c0 += 64) {
    __syncthreads();
    for (int x = tid; x < 64 * D / 4; x += 256) {
      const int cc = x / (D / 4), d4 = x % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + cc < p.C) v = __ldg(reinterpret_cast<const float4*>(cent + (size_t)(c0 + cc) * D) + d4);
      cs[(d4 * 4 + 0) * 64 + cc] = v.x;
      cs[(d4 * 4 + 1) * 64 + cc] = v.y;
      cs[(d4 * 4 + 2) * 64 + cc] = v.z;
      cs[(d4 * 4 + 3) * 64 + cc] = v.w;
    }
    __syncthreads();
    float acc[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[r][j] = 0.f;
#pragma unroll 4
    for (int dd = 0; dd < D; ++dd) {
      const float4 ka = *reinterpret_cast<const float4*>(ks + dd * 128 + ty * 8);
      const float4 kb = *reinterpret_cast<const float4*>(ks + dd * 128 + ty * 8 + 4);
      const float4 cv = *reinterpret_cast<const float4*>(cs + dd * 64 + tx * 4);
      const float kv[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
      const float cc4[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][j] = fmaf(kv[r], cc4[j], acc[r][j]);
    }
    // distance up to the key's own |k|^2: |c|^2 - 2 k.c; ties to the lower cluster
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      if (c < p.C) {
        const float n2 = __ldg(cn + c);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float dist = fmaf(-2.f, acc[r][j], n2);
          if (dist < best[r]) {   // clusters arrive in increasing order per thread
            best[r] = dist;
            bidx[r] = c;
          }
        }
      }
    }
  }
  // reduce over the 16 threads that share a key row (lanes tx = 0..15 of a half warp)
#pragma unroll
  for (int r = 0; r < 8; ++r) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xFFFFFFFFu, best[r], o);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bidx[r], o);
      if (ob < best[r] || (ob == best[r] && oi < bidx[r])) {
        best[r] = ob;
        bidx[r] = oi;
      }
    }
    const int t = t0 + ty * 8 + r;
    if (tx == 0 && t < p.n_ctx) p.assign[(size_t)bg * p.n_ctx + t] = bidx[r];
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
#pragma unroll
  for (int x = 0; x < PER; ++x) {
    const float m = s[x] * inv;
    out[x] = m;
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

template <int D, int GRP, int NT>
__global__ void __launch_bounds__(NT) cluster_select_kernel(const ClusterParams cp) {
  extern __shared__ __align__(16) uint8_t csm[];
  __shared__ SelectSmem sm;
  const DecodeParams& p = cp.dp;
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int C = cp.C;
  float* sc = reinterpret_cast<float*>(csm);                        // [GRP][C] (compacted candidates)
  int32_t* cand = reinterpret_cast<int32_t*>(sc + (size_t)GRP * C);  // [C] non-empty cluster ids
  int32_t* tmp = cand + C;                                           // [C]
  int32_t* ubase = tmp + C;                                          // [C] union token offsets
  int32_t* off = ubase + C;                                          // [C + 1] the cluster -> key offsets
  uint8_t* mask = reinterpret_cast<uint8_t*>(off + C + 1);           // [C]
  // the offsets come in once, coalesced: the union loop below reads them per
  // cluster, which from global memory was a chain of dependent loads per warp
  const int32_t* goff = cp.off + (size_t)bg * (C + 1);
  for (int x = threadIdx.x; x <= C; x += NT) off[x] = goff[x];
  __syncthreads();
  // non-empty clusters, ascending (block scan over per-thread ranges)
  const int per = (C + NT - 1) / NT;
  const int c0 = min(C, (int)threadIdx.x * per), c1 = min(C, c0 + per);
  int ne = 0;
  for (int c = c0; c < c1; ++c) {
    mask[c] = 0;
    ne += off[c + 1] > off[c];
  }
  int ncand;
  int pos = block_excl_scan<NT>(ne, sm, ncand);
  for (int c = c0; c < c1; ++c)
    if (off[c + 1] > off[c]) cand[pos++] = c;
  __syncthreads();
  // the candidates' scores, computed for every cluster by decode_score_kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* gsc = cp.scores + ((size_t)b * p.Hq + g * GRP) * C;   // the group's rows are contiguous
  for (int x = threadIdx.x; x < GRP * ncand; x += NT) {
    const int hh = x / ncand, y = x % ncand;
    sc[(size_t)hh * C + y] = gsc[(size_t)hh * C + cand[y]];
  }
  __syncthreads();
  const int e = min(p.keep, ncand);
  for (int hh = 0; hh < GRP; ++hh) {
    const int cnt = topk_ascending<NT>(sc + (size_t)hh * C, ncand, e, 0, ncand, tmp, C, sm);
    __syncthreads();
    const int h = g * GRP + hh;
    for (int x = threadIdx.x; x < cnt; x += NT) mask[cand[tmp[x]]] |= (uint8_t)(1u << hh);
    if (p.sel_idx) {
      int32_t* out = p.sel_idx + ((size_t)b * p.Hq + h) * p.kcap;
      for (int x = threadIdx.x; x < p.kcap; x += NT) out[x] = x < cnt ? cand[tmp[x]] : -1;
    }
    if (p.sel_cnt && threadIdx.x == 0) p.sel_cnt[(size_t)b * p.Hq + h] = cnt;
    __syncthreads();
  }
  // the union's tokens in cluster order, then the tail
  int sz = 0;
  for (int c = c0; c < c1; ++c) sz += mask[c] ? off[c + 1] - off[c] : 0;
  int total;
  int ub = block_excl_scan<NT>(sz, sm, total);
  for (int c = c0; c < c1; ++c) {
    ubase[c] = ub;
    if (mask[c]) ub += off[c + 1] - off[c];
  }
  __syncthreads();
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
  static constexpr int kMask = kRed + kRedBytes;                // 64 head-mask bytes per stage
  static constexpr int kBar = kMask + kDecStages * 64;
  static constexpr int kBytes = kBar + 2 * kDecStages * 8 + 16;
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
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + Lay::kBar + 2 * kDecStages * 8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), NW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const AbortState ab{abort_flag, p.status};
  const int32_t* ui = p.uidx + (size_t)bg * p.nb;
  const uint8_t* um = p.umask + (size_t)bg * p.nb;
  constexpr uint32_t kRowBytes = D * 2;

  if (warp == NW) {
    // producer warp: runs of consecutive positions of each unit
    int u = 0;
    for (; u < nu; ++u) {
      const int s = u % kDecStages;
      if (u >= kDecStages && !mbar_wait_warp(empty(s), ((u / kDecStages) - 1) & 1, ab)) break;
      const int rb = e0 + 64 * u, rows = min(64, e1 - rb);
      const int pa = lane < rows ? ui[rb + lane] : -1;
      const int pb = lane + 32 < rows ? ui[rb + lane + 32] : -1;
      const int up_a = __shfl_up_sync(0xFFFFFFFFu, pa, 1), last_a = __shfl_sync(0xFFFFFFFFu, pa, 31);
      const int up_b = __shfl_up_sync(0xFFFFFFFFu, pb, 1);
      const int prev_b = lane == 0 ? last_a : up_b;
      // a run starts at row 0, after a gap, and where the cache tail begins
      // (positions below n_packed are in the copy, the rest in the cache)
      const bool st_a = lane < rows && (lane == 0 || pa != up_a + 1 || pa == p.n_packed);
      const bool st_b = lane + 32 < rows && (pb != prev_b + 1 || pb == p.n_packed);
      uint64_t starts = (uint64_t)__ballot_sync(0xFFFFFFFFu, st_a) | ((uint64_t)__ballot_sync(0xFFFFFFFFu, st_b) << 32);
      // the unit's head masks ride with its rows (64 bytes, 16-byte aligned)
      const uint32_t mbytes = (uint32_t)((rows + 15) & ~15);
      if (lane == 0) {
        mbar_arrive_expect_tx(full(s), (uint32_t)rows * 2u * kRowBytes + mbytes);
        bulk_load(sb + Lay::kMask + s * 64, um + rb, mbytes, full(s));
      }
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
    if (lane == 0)
      for (int w = max(0, u - kDecStages); w < u; ++w)
        mbar_wait_cleanup(full(w % kDecStages), (w / kDecStages) & 1, 200000000ull);
    return;
  }
  // consumers: warp w takes rows 2 TPL w .. of every unit; the two half
  // warps take alternate rows, lane%16 owns dims [DPL*(lane%16), +DPL)
  constexpr int DPL = D / 16;
  const int half = lane >> 4, dl = lane & 15;
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
  bool ok = true;
  for (int u = 0; u < nu; ++u) {
    const int s = u % kDecStages;
    const int rb = e0 + 64 * u, rows = min(64, e1 - rb);
    if (!mbar_wait_warp(full(s), (u / kDecStages) & 1, ab)) {
      ok = false;
      break;
    }
    const uint8_t* ms = dsm + Lay::kMask + s * 64;
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
    float kf[TPL][DPL], vf[TPL][DPL];
#pragma unroll
    for (int it = 0; it < TPL; ++it) {
      const int key = 2 * TPL * warp + 2 * it + half;
      const bool valid = key < rows;   // rows past the unit's end hold stale bytes: never used
#pragma unroll
      for (int a = 0; a < DPL; ++a) {
        kf[it][a] = 0.f;
        vf[it][a] = 0.f;
      }
      if (valid) {
        if constexpr (DPL == 8) {
          const uint4 kr = *reinterpret_cast<const uint4*>(kb + key * kRowBytes + dl * 16);
          const uint4 vr = *reinterpret_cast<const uint4*>(vb + key * kRowBytes + dl * 16);
          const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
          const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const float2 kk = __bfloat1622float2(k2[a]), vv = __bfloat1622float2(v2[a]);
            kf[it][2 * a] = kk.x;
            kf[it][2 * a + 1] = kk.y;
            vf[it][2 * a] = vv.x;
            vf[it][2 * a + 1] = vv.y;
          }
        } else {
          const uint2 kr = *reinterpret_cast<const uint2*>(kb + key * kRowBytes + dl * 8);
          const uint2 vr = *reinterpret_cast<const uint2*>(vb + key * kRowBytes + dl * 8);
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
    // release the stage once every warp has its registers
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
      if (!((mor >> hh) & 1u)) continue;   // no row of the unit kept by this head (warp-uniform)
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
      if (mn == -INFINITY) continue;   // nothing of this head in this warp yet (warp-uniform)
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
  // merge the two half-warps (same dims, same running max), then the NW warps
  float* red = reinterpret_cast<float*>(dsm + Lay::kRed);   // [warp][hh][D + 2]
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh) {
    l[hh] += __shfl_xor_sync(0xFFFFFFFFu, l[hh], 16);
#pragma unroll
    for (int a = 0; a < DPL; ++a) acc[hh][a] += __shfl_xor_sync(0xFFFFFFFFu, acc[hh][a], 16);
    float* r = red + ((size_t)warp * kMaxGrp + hh) * (D + 2);
    if (half == 0) {
#pragma unroll
      for (int a = 0; a < DPL; ++a) r[dl * DPL + a] = acc[hh][a];
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
