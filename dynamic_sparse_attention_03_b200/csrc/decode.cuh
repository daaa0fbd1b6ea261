// decode.cuh -- centroid-ranked sparse decode (Squeezed Attention page,
// "技术方案", online stage: compare the query with every centroid, keep the top
// clusters, run attention only over the keys and values of those clusters).
// Clusters are the contiguous 64-token blocks of the cache; centroids are the
// block means (built by the pooling kernel).
//
// Kernels:
//  decode_score_kernel: q·c for every (batch, q-head, block), 64 centroid
//    blocks of one (batch, KV head) per CTA, each centroid row read once for
//    the group's q-heads.
//  decode_topk_kernel: one CTA per (batch, q-head): the head's top `keep`
//    blocks (ties to the lower block) plus the last block, as a bitmap.
//  decode_union_kernel: one CTA per (batch, KV head): the union of the group's
//    bitmaps as a block list with a per-block head mask.
//  decode_attn_kernel: one CTA per (batch, KV head, chunk of union blocks).
//    A producer warp streams whole 64-token K and V blocks (contiguous 16 KB
//    each at d = 128) into a 4-stage shared-memory ring with bulk copies;
//    8 consumer warps score the block for every q-head that kept it (packed
//    f32x2 multiply-adds), keep an online softmax per (warp, head), and merge
//    into one partial per chunk.  Each K/V block is read from HBM once for the
//    whole GQA group.
//  decode_combine_kernel: merges the chunk partials of each (batch, q-head).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kDecChunk = 64;      // union blocks per attention CTA
constexpr int kDecStages = 4;
constexpr int kMaxGrp = 8;         // q-heads per KV head supported by the decode path
constexpr int kDecWarps = 8;       // consumer warps of decode_attn_kernel: 8 keys of each block per warp
constexpr int kDecThreads = (kDecWarps + 1) * 32;   // plus the producer warp

struct DecodeParams {
  const __nv_bfloat16* q;      // [B][Hq][D]
  const __nv_bfloat16* kc;     // [B][Hkv][S][D]
  const __nv_bfloat16* vc;
  const float* cent;           // [B][Hkv][nb][D]
  __nv_bfloat16* o;            // [B][Hq][D]
  int32_t* sel_idx;            // optional [B][Hq][kcap]
  int32_t* sel_cnt;            // optional [B][Hq]
  int32_t* uidx;               // ws [B*Hkv][nb]
  uint8_t* umask;              // ws [B*Hkv][nb]
  int32_t* ucnt;               // ws [B*Hkv]
  float* part_ml;              // ws [B*Hq][nchmax][2]
  float* part_acc;             // ws [B*Hq][nchmax][D]
  float* scores;               // ws [B*Hq][nb] q·c
  uint32_t* kbits;             // ws [B*Hq][ceil(nb/32)] kept blocks (or clusters) per q-head
  const __nv_bfloat16* kp;     // optional [B][Hkv][n_packed][D]: K rows in cluster order
  const __nv_bfloat16* vp;     //   (list entries below n_packed are positions in these)
  int n_packed;                // 0 when the list holds cache token ids only
  uint32_t* status;
  int B, Hq, Hkv, S, nb, grp, keep, force_last, kcap, nchmax;
  float scale_log2;
};

// ---------------------------------------------------------------- scores
// Sums C per-lane values over the 32 lanes of a warp and leaves them spread
// over the lanes: each round exchanges half of a lane's values with the lane
// `off` away and adds (the lane keeps the half its bit `off` picks), so the
// 5 rounds take about C shuffles instead of 5 C.  Afterwards lane L holds the
// sums of values L*(C/32) .. L*(C/32) + C/32 - 1 (C >= 32), or of value
// L / (32/C) (C < 32; the 32/C lanes of a group hold the same sum).
template <int C>
__device__ __forceinline__ void warp_sum_spread(float (&v)[C], int lane) {
  int n = C;   // values a lane still holds (a constant once the loop is unrolled)
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool hi = (lane & off) != 0;
      const int h = n / 2;
#pragma unroll
      for (int i = 0; i < C / 2; ++i) {
        if (i < h) {
          const float keep = hi ? v[i + h] : v[i];
          const float send = hi ? v[i] : v[i + h];
          v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
        }
      }
      n = h;
    } else {
      v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], off);
    }
  }
}

// One CTA of 8 warps per (batch x KV head, 64 centroid blocks): each warp
// scores 8 blocks for the group's q-heads, loading its 8 rows together; the
// 8 x GRP dot products are summed over the warp with warp_sum_spread, after
// which the 8 scores of a head sit in 8 lanes and go to 8 consecutive words.
template <int D, int GRP>
__global__ void __launch_bounds__(256) decode_score_kernel(const DecodeParams p) {
  constexpr int PER = D / 32;
  constexpr int C = 8 * GRP;                 // (block, head) dot products per warp
  const int bg = blockIdx.x, t0 = blockIdx.y * 64;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float qreg[GRP][PER];
#pragma unroll
  for (int hh = 0; hh < GRP; ++hh)
#pragma unroll
    for (int a = 0; a < PER; ++a)
      qreg[hh][a] = __bfloat162float(p.q[((size_t)b * p.Hq + g * GRP + hh) * D + lane * PER + a]);
  const float* crow = p.cent + (size_t)bg * p.nb * D;
  float cv[8][PER];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int t = t0 + warp * 8 + r;
    if (t < p.nb) {
      const float* src = crow + (size_t)t * D + lane * PER;
      if constexpr (PER == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
        cv[r][0] = v.x; cv[r][1] = v.y; cv[r][2] = v.z; cv[r][3] = v.w;
      } else if constexpr (PER == 2) {
        const float2 v = __ldg(reinterpret_cast<const float2*>(src));
        cv[r][0] = v.x; cv[r][1] = v.y;
      } else {
#pragma unroll
        for (int a = 0; a < PER; ++a) cv[r][a] = __ldg(src + a);
      }
    } else {
#pragma unroll
      for (int a = 0; a < PER; ++a) cv[r][a] = 0.f;
    }
  }
  // this lane's share of every (block r, head hh) dot product, value r*GRP + hh
  float s[C];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
      float acc = 0.f;
#pragma unroll
      for (int a = 0; a < PER; ++a) acc = fmaf(qreg[hh][a], cv[r][a], acc);
      s[r * GRP + hh] = acc;
    }
  warp_sum_spread<C>(s, lane);
  constexpr int HOLD = C >= 32 ? C / 32 : 1;   // sums this lane holds
  constexpr int REP = C >= 32 ? 1 : 32 / C;    // lanes holding the same sum
  if (lane % REP == 0) {
#pragma unroll
    for (int j = 0; j < HOLD; ++j) {
      const int idx = (C >= 32) ? lane * HOLD + j : lane / REP;
      const int r = idx / GRP, hh = idx % GRP;
      const int t = t0 + warp * 8 + r;
      if (t < p.nb) p.scores[((size_t)b * p.Hq + g * GRP + hh) * p.nb + t] = s[j];
    }
  }
}

// ---------------------------------------------------------------- select
// Two launches, so the top-k of every q-head runs in parallel: one CTA per
// (batch, q-head) selects that head's blocks from its stored scores (the last
// block always kept when force_last) and writes them as a bitmap (and the
// optional selection outputs); one CTA per (batch, KV head) then ORs the
// group's bitmaps into the ascending union list with a head mask per block.
template <int NT>
__global__ void __launch_bounds__(NT) decode_topk_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ SelectSmem sm;
  const int bh = blockIdx.x;   // b * Hq + h
  const int nb = p.nb, nw = (nb + 31) >> 5;
  float* sc = reinterpret_cast<float*>(dsm);                  // [nb]
  int32_t* tmp = reinterpret_cast<int32_t*>(sc + nb);         // [nb]
  uint32_t* bits = reinterpret_cast<uint32_t*>(tmp + nb);     // [nw]
  const float* gsc = p.scores + (size_t)bh * nb;
  for (int x = threadIdx.x; x < nb; x += NT) sc[x] = gsc[x];
  for (int x = threadIdx.x; x < nw; x += NT) bits[x] = 0u;
  __syncthreads();
  const int ncand = p.force_last ? nb - 1 : nb;
  const int cnt = topk_ascending<NT>(sc, ncand, p.keep, 0, nb, tmp, nb, sm);
  __syncthreads();
  for (int x = threadIdx.x; x < cnt; x += NT) atomicOr(&bits[tmp[x] >> 5], 1u << (tmp[x] & 31));
  if (p.sel_idx) {
    int32_t* out = p.sel_idx + (size_t)bh * p.kcap;
    for (int x = threadIdx.x; x < p.kcap; x += NT) out[x] = x < cnt ? tmp[x] : -1;
  }
  if (p.sel_cnt && threadIdx.x == 0) p.sel_cnt[bh] = cnt;
  __syncthreads();
  uint32_t* gb = p.kbits + (size_t)bh * nw;
  for (int x = threadIdx.x; x < nw; x += NT) gb[x] = bits[x];
}

template <int GRP, int NT>
__global__ void __launch_bounds__(NT) decode_union_kernel(const DecodeParams p) {
  __shared__ SelectSmem sm;
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int nb = p.nb, nw = (nb + 31) >> 5;
  const uint32_t* gb = p.kbits + ((size_t)b * p.Hq + g * GRP) * nw;   // the group's rows are contiguous
  auto mask_of = [&](int x) {
    uint32_t m = 0u;
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) m |= ((gb[(size_t)hh * nw + (x >> 5)] >> (x & 31)) & 1u) << hh;
    return m;
  };
  const int per = (nb + NT - 1) / NT;
  const int p0 = min(nb, (int)threadIdx.x * per), p1 = min(nb, p0 + per);
  int kept = 0;
  for (int x = p0; x < p1; ++x) kept += mask_of(x) != 0u;
  int total;
  int off = block_excl_scan<NT>(kept, sm, total);
  int32_t* ui = p.uidx + (size_t)bg * nb;
  uint8_t* um = p.umask + (size_t)bg * nb;
  for (int x = p0; x < p1; ++x) {
    const uint32_t m = mask_of(x);
    if (m) {
      ui[off] = x;
      um[off] = (uint8_t)m;
      ++off;
    }
  }
  if (threadIdx.x == 0) p.ucnt[bg] = total;
}

// ---------------------------------------------------------------- attention over kept blocks
template <int D>
struct DecLayout {
  static constexpr int kBlkBytes = 64 * D * 2;                  // one 64-token K (or V) block
  static constexpr int kStage = 2 * kBlkBytes;
  static constexpr int kRing = kDecStages * kStage;
  static constexpr int kRed = kRing;                            // warp partials
  static constexpr int kRedBytes = kDecWarps * kMaxGrp * (D + 2) * 4;
  static constexpr int kBar = kRed + kRedBytes;
  static constexpr int kBytes = kBar + 2 * kDecStages * 8 + 16;
};

template <int D, int GRP>
__global__ void __launch_bounds__(kDecThreads, 1) decode_attn_kernel(const DecodeParams p) {
  using Lay = DecLayout<D>;
  constexpr int NW = kDecWarps, TPL = 32 / NW;   // keys per lane per block
  extern __shared__ __align__(16) uint8_t dsm[];
  const uint32_t sb = smem_u32(dsm);
  const int bg = blockIdx.x, chunk = blockIdx.y;
  const int cnt = p.ucnt[bg];
  const int u0 = chunk * kDecChunk;
  if (u0 >= cnt || status_timed_out(p.status)) return;
  const int u1 = min(cnt, u0 + kDecChunk);
  const int nu = u1 - u0;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  constexpr int grp = GRP;
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
  const int32_t* ui = p.uidx + (size_t)bg * p.nb + u0;
  const uint8_t* um = p.umask + (size_t)bg * p.nb + u0;
  const size_t head_base = (size_t)bg * p.S * D;

  if (warp == NW) {
    // producer: the chunk's (at most 64) block ids come in once, two per
    // lane, so no unit waits on a list load; lane 0 streams whole K and V
    // blocks
    static_assert(kDecChunk <= 64, "two list entries per producer lane");
    const int ida = lane < nu ? ui[lane] : 0, idb = lane + 32 < nu ? ui[lane + 32] : 0;
    int u = 0;
    for (; u < nu; ++u) {
      const int s = u % kDecStages;
      if (u >= kDecStages && !mbar_wait_warp(empty(s), ((u / kDecStages) - 1) & 1, ab)) break;
      const int blk = __shfl_sync(0xFFFFFFFFu, u < 32 ? ida : idb, u & 31);
      if (lane == 0) {
        const size_t off = head_base + (size_t)blk * 64 * D;
        mbar_arrive_expect_tx(full(s), 2u * Lay::kBlkBytes);
        bulk_load(sb + s * Lay::kStage, p.kc + off, Lay::kBlkBytes, full(s));
        bulk_load(sb + s * Lay::kStage + Lay::kBlkBytes, p.vc + off, Lay::kBlkBytes, full(s));
      }
      __syncwarp();
    }
    if (lane == 0)
      for (int w = max(0, u - kDecStages); w < u; ++w)
        mbar_wait_cleanup(full(w % kDecStages), (w / kDecStages) & 1, 200000000ull);
    return;
  }
  // consumers: warp w takes keys 2 TPL w .. of every block; the two half
  // warps take alternate keys, lane%16 owns dims [DPL*(lane%16), +DPL).
  // (dot products and P.V updates as packed f32x2 multiply-adds on pairs of dims)
  constexpr int DPL = D / 16, DP2 = DPL / 2;   // dims per lane (8 at d=128, 4 at d=64)
  const int half = lane >> 4, dl = lane & 15;
  float2 qv[GRP][DP2];
#pragma unroll
  for (int hh = 0; hh < grp; ++hh)
#pragma unroll
    for (int j = 0; j < DP2; ++j) {
      const __nv_bfloat16* qr = p.q + ((size_t)b * p.Hq + g * grp + hh) * D + dl * DPL + 2 * j;
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
  bool ok = true;
  for (int u = 0; u < nu; ++u) {
    const int s = u % kDecStages;
    if (!mbar_wait_warp(full(s), (u / kDecStages) & 1, ab)) { ok = false; break; }
    const uint8_t msk = um[u];
    const uint8_t* kb = dsm + s * Lay::kStage;
    const uint8_t* vb = kb + Lay::kBlkBytes;
    // TPL keys per lane: key = 2 TPL warp + 2 it + half
    float2 kf[TPL][DP2], vf[TPL][DP2];
#pragma unroll
    for (int it = 0; it < TPL; ++it) {
      const int key = 2 * TPL * warp + 2 * it + half;
      if constexpr (DPL == 8) {
        const uint4 kr = *reinterpret_cast<const uint4*>(kb + key * D * 2 + dl * 16);
        const uint4 vr = *reinterpret_cast<const uint4*>(vb + key * D * 2 + dl * 16);
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          kf[it][j] = __bfloat1622float2(k2[j]);
          vf[it][j] = __bfloat1622float2(v2[j]);
        }
      } else {
        const uint2 kr = *reinterpret_cast<const uint2*>(kb + key * D * 2 + dl * 8);
        const uint2 vr = *reinterpret_cast<const uint2*>(vb + key * D * 2 + dl * 8);
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
    for (int hh = 0; hh < grp; ++hh) {
      if (!((msk >> hh) & 1u)) continue;   // block not kept by this head (warp-uniform)
      float sc[TPL];
#pragma unroll
      for (int it = 0; it < TPL; ++it) {
        float2 t = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < DP2; ++j) t = ffma2(qv[hh][j], kf[it][j], t);
        float d0 = t.x + t.y;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) d0 += __shfl_xor_sync(0xFFFFFFFFu, d0, o);
        sc[it] = d0;
      }
      float mb = sc[0];
#pragma unroll
      for (int it = 1; it < TPL; ++it) mb = fmaxf(mb, sc[it]);
      mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 16));
      const float mn = fmaxf(m[hh], mb);
      const float alpha = ex2_approx(m[hh] - mn);   // m = -inf -> 0
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < DP2; ++j) acc[hh][j] = fmul2(acc[hh][j], make_float2(alpha, alpha));
#pragma unroll
      for (int it = 0; it < TPL; ++it) {
        const float pe = ex2_approx(sc[it] - mn);
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
  for (int hh = 0; hh < grp; ++hh) {
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
  for (int x = threadIdx.x; x < grp * D; x += NW * 32) {
    const int hh = x / D, c = x % D;
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[((size_t)w * kMaxGrp + hh) * (D + 2) + D]);
    float a = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < NW; ++w) {
        const float* r = red + ((size_t)w * kMaxGrp + hh) * (D + 2);
        const float wgt = ex2_approx(r[D] - M);
        a += wgt * r[c];
        L += wgt * r[D + 1];
      }
    }
    const size_t ph = (size_t)b * p.Hq + g * grp + hh;
    p.part_acc[(ph * p.nchmax + chunk) * D + c] = a;
    if (c == 0) {
      p.part_ml[(ph * p.nchmax + chunk) * 2 + 0] = M;
      p.part_ml[(ph * p.nchmax + chunk) * 2 + 1] = L;
    }
  }
}

// ---------------------------------------------------------------- combine
// CHUNK: union entries per attention CTA (blocks here; tokens for the
// cluster-ranked decode).
template <int D, int CHUNK = kDecChunk>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;   // b*Hq + h
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.grp;
  const int nch = (p.ucnt[b * p.Hkv + g] + CHUNK - 1) / CHUNK;
  const float* ml = p.part_ml + (size_t)bh * p.nchmax * 2;
  float M = -INFINITY;
  for (int c = 0; c < nch; ++c) M = fmaxf(M, ml[2 * c]);
  for (int x = threadIdx.x; x < D; x += blockDim.x) {
    float a = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int c = 0; c < nch; ++c) {
        const float wgt = ex2_approx(ml[2 * c] - M);
        a += wgt * p.part_acc[((size_t)bh * p.nchmax + c) * D + x];
        L += wgt * ml[2 * c + 1];
      }
    }
    p.o[(size_t)bh * D + x] = __float2bfloat16_rn(L > 0.f ? a / L : 0.f);
  }
}

}  // namespace dsa
