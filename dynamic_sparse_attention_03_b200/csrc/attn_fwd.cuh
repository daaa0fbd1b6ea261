// attn_fwd.cuh -- causal block-sparse FlashAttention forward on sm_100a.
//
// MInference 1.0 page, method section ("方法介紹"): attention is computed only
// over the key/value blocks the index selected (block-sparse FlashAttention);
// Fig. 4: slash lines as 64x64 blocks, vertical lines as 1x64 column tiles.
//
// Design (one CTA = 7 warps, one work item):
//  * A work item is 128 query rows that share one KV head: the same 64-token
//    query block of two q-heads of a GQA group (rows 0-63 = head A, 64-127 =
//    head B).  Their sorted block lists are merged; each merged entry records
//    which of the two heads chose it.  Column entries (1x64 tiles) of the two
//    heads are merged the same way, 64 columns per slot.
//  * A "tile" is two slots of 64 keys (N = 128 keys).  Warp 0 streams the K
//    tiles and warp 6 the V tiles, each into its own 3-stage shared-memory ring
//    (TMA 2D tile loads with 128-byte swizzle for blocks, 16-byte gathers for
//    columns).  K and V have separate barriers: a K stage is refilled as soon
//    as its QK^T has run, a V stage once its PV has run, so loads run ahead of
//    the softmax.  Warp 0 also publishes per-tile metadata (which rows may see
//    which keys) in a ring with its own barriers.
//  * Warp 1 (one thread) issues tcgen05.mma: S = Q K^T (M=128, N=128, K=d,
//    both operands in shared memory) into a double-buffered TMEM S, and
//    O += P V (M=128, N=d, K=128) with P read from TMEM (double-buffered) and V
//    from shared memory.  Completion is signalled with tcgen05.commit.
//  * Warps 2-5 (thread = row = TMEM lane) run the online softmax: tcgen05.ld
//    of the S row, masks only where a tile needs them, exp2 of
//    (s*scale*log2e - max) in one FMA, a lazy rescale of O in TMEM only when
//    the running max grows by more than 2^8, P (bf16) back into TMEM with
//    tcgen05.st, and the epilogue O / l -> bf16.
//  * TMEM columns: S0 [0,128) S1 [128,256) O [256,256+d) P0 [384,448) P1 [448,512).
//  * Every wait is bounded (1 s); on expiry the CTA records a timeout in the
//    status word, all roles leave their loops, TMEM is freed, the CTA returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dsa {

struct AttnParams {
  const __nv_bfloat16* k;  // for column gathers
  const __nv_bfloat16* v;
  __nv_bfloat16* o;
  float* lse;
  const int32_t* block_idx;
  const int32_t* block_cnt;
  const int32_t* col_idx;
  const int32_t* col_cnt;
  uint32_t* status;
  int kcap, ccap;
  int Hq, Hkv, n, nQB, grp, npairs;
  float scale_log2;
};

// Per-tile metadata for the MMA issuer and the softmax warps.
struct alignas(16) AttnMeta {
  unsigned long long mA[2], mB[2];  // key c of slot s is visible to head A / B rows
  int blk[2];                       // key block of a block slot, -1 otherwise
  int kind[2];                      // 0 empty, 1 block, 2 columns
  int nslots, last;
};

constexpr int kAttnKS = 3;   // K stages
constexpr int kAttnVS = 3;   // V stages
constexpr int kAttnMR = 8;   // metadata ring entries (>= K stages + 2)

template <int D>
struct AttnLayout {
  static constexpr int NDH = D / 64;              // 64-element (128-byte) column halves of d
  static constexpr int kHalf = 16384;             // one d-half of a 128-row tile (128 x 128 B)
  static constexpr int kTile = NDH * kHalf;       // 128 rows x d bf16
  static constexpr int kQ = 0;
  static constexpr int kK0 = kQ + kTile;
  static constexpr int kV0 = kK0 + kAttnKS * kTile;
  static constexpr int kMeta = kV0 + kAttnVS * kTile;
  static constexpr int kCols = kMeta + kAttnMR * (int)sizeof(AttnMeta);   // [producer][slot][64] ints
  static constexpr int kScratchMeta = kCols + 2 * 2 * 64 * 4;             // V producer's own tile record
  static constexpr int kBar = kScratchMeta + (int)sizeof(AttnMeta);
  // barriers: q, kfull[KS], kempty[KS], vfull[VS], vempty[VS], sfull[2], pfull[2], pvdone[2], meta[MR], drain
  static constexpr int kNumBars = 1 + 2 * kAttnKS + 2 * kAttnVS + 6 + kAttnMR + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;   // slack to align the base to 1024
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

enum : int {
  AB_Q = 0,
  AB_KFULL = 1,
  AB_KEMPTY = AB_KFULL + kAttnKS,
  AB_VFULL = AB_KEMPTY + kAttnKS,
  AB_VEMPTY = AB_VFULL + kAttnVS,
  AB_SFULL = AB_VEMPTY + kAttnVS,
  AB_PFULL = AB_SFULL + 2,
  AB_PVDONE = AB_PFULL + 2,
  AB_META = AB_PVDONE + 2,
  AB_DRAIN = AB_META + kAttnMR,
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256, kTmemP = 384;

// D[tmem] (+)= A[tmem] * B[smem]^T, issued by one thread (A from tensor memory).
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Merge cursor over the two heads' sorted lists (blocks first, then columns).
struct AttnLists {
  const int32_t *LA, *LB, *CA, *CB;
  int na, nb, nca, ncb;
};

struct AttnCursor {
  int ia = 0, ib = 0, ja = 0, jb = 0;

  __device__ bool more(const AttnLists& L) const { return ia < L.na || ib < L.nb || ja < L.nca || jb < L.ncb; }

  // Forms the next tile (up to two slots of 64 keys) into M; column slots also
  // record their key columns in cols[slot][0..64) (-1 padded).
  __device__ void next(const AttnLists& L, AttnMeta& M, int (*cols)[64]) {
    for (int sl = 0; sl < 2; ++sl) {
      if (ia < L.na || ib < L.nb) {
        const int a = ia < L.na ? L.LA[ia] : 0x7FFFFFFF;
        const int b = ib < L.nb ? L.LB[ib] : 0x7FFFFFFF;
        const int blk = min(a, b);
        M.kind[sl] = 1;
        M.blk[sl] = blk;
        M.mA[sl] = (a == blk) ? ~0ull : 0ull;
        M.mB[sl] = (b == blk) ? ~0ull : 0ull;
        ia += (a == blk);
        ib += (b == blk);
      } else if (ja < L.nca || jb < L.ncb) {
        unsigned long long mA = 0, mB = 0;
        int c = 0;
        while (c < 64 && (ja < L.nca || jb < L.ncb)) {
          const int a = ja < L.nca ? L.CA[ja] : 0x7FFFFFFF;
          const int b = jb < L.ncb ? L.CB[jb] : 0x7FFFFFFF;
          const int col = min(a, b);
          if (a == col) { mA |= 1ull << c; ++ja; }
          if (b == col) { mB |= 1ull << c; ++jb; }
          cols[sl][c] = col;
          ++c;
        }
        for (; c < 64; ++c) cols[sl][c] = -1;
        M.kind[sl] = 2;
        M.blk[sl] = -1;
        M.mA[sl] = mA;
        M.mB[sl] = mB;
      } else {
        M.kind[sl] = 0;
        M.blk[sl] = -1;
        M.mA[sl] = M.mB[sl] = 0ull;
      }
    }
    M.nslots = (M.kind[0] != 0) + (M.kind[1] != 0);
    M.last = !more(L);
  }
};

// Gathers the 64 rows `cols` of head-row base `src` (row stride D) into a
// 64-key slot of a 128-byte swizzled [d-half][128 keys][128 B] stage.  Warp-wide.
template <int D>
__device__ __forceinline__ void gather_slot(const __nv_bfloat16* src, const int* cols, uint32_t stage, int sl,
                                            int lane) {
  constexpr int VPR = D / 8;
  for (int idx = lane; idx < 64 * VPR; idx += 32) {
    const int c = idx / VPR, v = idx % VPR;
    const int col = cols[c];
    uint4 x = make_uint4(0, 0, 0, 0);
    if (col >= 0) x = __ldg(reinterpret_cast<const uint4*>(src + (size_t)col * D + v * 8));
    const uint32_t o = (uint32_t)((v >> 3) * 16384 + sl * 8192 + c * 128 + (((v & 7) ^ (c & 7)) << 4));
    st_shared_v4(stage + o, x.x, x.y, x.z, x.w);
  }
}

template <int D>
__global__ void __launch_bounds__(224, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using Lay = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  if (status_timed_out(p.status)) return;   // uniform over the CTA: before any barrier or TMEM use
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  AttnMeta* meta = reinterpret_cast<AttnMeta*>(smem + Lay::kMeta);
  int(*colsK)[64] = reinterpret_cast<int(*)[64]>(smem + Lay::kCols);
  int(*colsV)[64] = reinterpret_cast<int(*)[64]>(smem + Lay::kCols + 2 * 64 * 4);
  AttnMeta* vrec = reinterpret_cast<AttnMeta*>(smem + Lay::kScratchMeta);
  const uint32_t bar0 = sb + Lay::kBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_qb = p.Hkv * p.npairs;
  const int qb = p.nQB - 1 - (int)(blockIdx.x / per_qb);   // heaviest query blocks first
  const int rem = (int)(blockIdx.x % per_qb);
  const int g = rem / p.npairs, pr = rem % p.npairs;
  const int hA = g * p.grp + 2 * pr;
  const int hB = (2 * pr + 1 < p.grp) ? hA + 1 : -1;

  if (threadIdx.x == 0) {
    mbar_init(bar(AB_Q), 1);
    for (int s = 0; s < kAttnKS; ++s) {
      mbar_init(bar(AB_KFULL + s), 1);
      mbar_init(bar(AB_KEMPTY + s), 1);
    }
    for (int s = 0; s < kAttnVS; ++s) {
      mbar_init(bar(AB_VFULL + s), 1);
      mbar_init(bar(AB_VEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(AB_SFULL + b), 1);
      mbar_init(bar(AB_PFULL + b), 128);
      mbar_init(bar(AB_PVDONE + b), 1);
    }
    for (int m = 0; m < kAttnMR; ++m) mbar_init(bar(AB_META + m), 1);
    mbar_init(bar(AB_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, p.status};

  const uint32_t sQ = sb + Lay::kQ;
  auto sK = [&](int s) { return sb + Lay::kK0 + (uint32_t)s * Lay::kTile; };
  auto sV = [&](int s) { return sb + Lay::kV0 + (uint32_t)s * Lay::kTile; };

  AttnLists L;
  {
    const size_t rowA = (size_t)hA * p.nQB + qb;
    const size_t rowB = (size_t)(hB >= 0 ? hB : hA) * p.nQB + qb;
    L.LA = p.block_idx + rowA * p.kcap;
    L.LB = p.block_idx + rowB * p.kcap;
    L.CA = p.col_idx ? p.col_idx + rowA * p.ccap : nullptr;
    L.CB = p.col_idx ? p.col_idx + rowB * p.ccap : nullptr;
    L.na = L.nb = L.nca = L.ncb = 0;
    if (warp == 0 || warp == 6) {
      L.na = min(max(p.block_cnt[rowA], 0), p.kcap);
      L.nb = hB >= 0 ? min(max(p.block_cnt[rowB], 0), p.kcap) : 0;
      L.nca = p.col_idx ? min(max(p.col_cnt[rowA], 0), p.ccap) : 0;
      L.ncb = (p.col_idx && hB >= 0) ? min(max(p.col_cnt[rowB], 0), p.ccap) : 0;
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ K producer + metadata
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      mbar_arrive_expect_tx(bar(AB_Q), (uint32_t)Lay::kTile);
#pragma unroll
      for (int dh = 0; dh < Lay::NDH; ++dh) {
        tma_load_2d(sQ + dh * Lay::kHalf, &tmQ, dh * 64, hA * p.n + qb * 64, bar(AB_Q));
        tma_load_2d(sQ + dh * Lay::kHalf + 8192, &tmQ, dh * 64, (hB >= 0 ? hB : hA) * p.n + qb * 64, bar(AB_Q));
      }
    }
    AttnCursor cur;
    int t = 0, issued = 0;
    while (true) {
      const int ks = t % kAttnKS;
      if (t >= kAttnKS && !mbar_wait_warp(bar(AB_KEMPTY + ks), ((t / kAttnKS) - 1) & 1, ab)) break;
      AttnMeta& M = meta[t % kAttnMR];
      if (lane == 0) cur.next(L, M, colsK);
      __syncwarp();
      const int nsl = M.nslots, last = M.last;
      const int k0 = M.kind[0], k1 = M.kind[1];
      const __nv_bfloat16* kbase = p.k + (size_t)g * p.n * D;
      if (k0 == 2) gather_slot<D>(kbase, colsK[0], sK(ks), 0, lane);
      if (k1 == 2) gather_slot<D>(kbase, colsK[1], sK(ks), 1, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(AB_META + (t % kAttnMR)));
        const uint32_t tx = (uint32_t)((k0 == 1) + (k1 == 1)) * 64u * D * 2u;
        mbar_arrive_expect_tx(bar(AB_KFULL + ks), tx);
        for (int sl = 0; sl < 2; ++sl) {
          if (M.kind[sl] != 1) continue;
          const int row = g * p.n + M.blk[sl] * 64;
#pragma unroll
          for (int dh = 0; dh < Lay::NDH; ++dh)
            tma_load_2d(sK(ks) + dh * Lay::kHalf + sl * 8192, &tmK, dh * 64, row, bar(AB_KFULL + ks));
        }
      }
      __syncwarp();
      ++issued;
      if (nsl == 0 || last) break;
      ++t;
    }
    if (lane == 0) {
      for (int u = max(0, issued - kAttnKS); u < issued; ++u)
        mbar_wait_cleanup(bar(AB_KFULL + (u % kAttnKS)), (u / kAttnKS) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) prefetch_tmap(&tmV);
    AttnCursor cur;
    int t = 0, issued = 0;
    while (true) {
      const int vs = t % kAttnVS;
      if (t >= kAttnVS && !mbar_wait_warp(bar(AB_VEMPTY + vs), ((t / kAttnVS) - 1) & 1, ab)) break;
      if (lane == 0) cur.next(L, *vrec, colsV);
      __syncwarp();
      const int nsl = vrec->nslots, last = vrec->last;
      if (nsl == 0) break;
      const int k0 = vrec->kind[0], k1 = vrec->kind[1];
      const int b0 = vrec->blk[0], b1 = vrec->blk[1];
      const __nv_bfloat16* vbase = p.v + (size_t)g * p.n * D;
      if (k0 == 2) gather_slot<D>(vbase, colsV[0], sV(vs), 0, lane);
      if (k1 == 2) gather_slot<D>(vbase, colsV[1], sV(vs), 1, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t tx = (uint32_t)((k0 == 1) + (k1 == 1)) * 64u * D * 2u;
        mbar_arrive_expect_tx(bar(AB_VFULL + vs), tx);
        if (k0 == 1)
#pragma unroll
          for (int dh = 0; dh < Lay::NDH; ++dh)
            tma_load_2d(sV(vs) + dh * Lay::kHalf, &tmV, dh * 64, g * p.n + b0 * 64, bar(AB_VFULL + vs));
        if (k1 == 1)
#pragma unroll
          for (int dh = 0; dh < Lay::NDH; ++dh)
            tma_load_2d(sV(vs) + dh * Lay::kHalf + 8192, &tmV, dh * 64, g * p.n + b1 * 64, bar(AB_VFULL + vs));
      }
      __syncwarp();
      ++issued;
      if (last) break;
      ++t;
    }
    if (lane == 0) {
      for (int u = max(0, issued - kAttnVS); u < issued; ++u)
        mbar_wait_cleanup(bar(AB_VFULL + (u % kAttnVS)), (u / kAttnVS) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_pv = umma_idesc_bf16(128, D, 1);
      bool ok = mbar_wait(bar(AB_Q), 0, ab);
      int t = 0, prev_nsl = 0;
      bool have_prev = false;
      auto issue_pv = [&](int u, int nsl) -> bool {
        if (!mbar_wait(bar(AB_PFULL + (u & 1)), (u >> 1) & 1, ab)) return false;
        if (!mbar_wait(bar(AB_VFULL + (u % kAttnVS)), (u / kAttnVS) & 1, ab)) return false;
        tc_fence_after();
        const uint32_t vst = sV(u % kAttnVS);
        const uint32_t pa = tmem + kTmemP + 64u * (uint32_t)(u & 1);
        for (int kk = 0; kk < nsl * 4; ++kk) {
          const uint64_t b = umma_desc_sw128(vst + kk * 2048, Lay::kHalf, 1024);
          umma_bf16_ts(tmem + kTmemO, pa + 8u * (uint32_t)kk, b, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(AB_VEMPTY + (u % kAttnVS)));
        umma_commit(bar(AB_PVDONE + (u & 1)));
        return true;
      };
      while (ok) {
        const int ks = t % kAttnKS;
        if (!mbar_wait(bar(AB_KFULL + ks), (t / kAttnKS) & 1, ab)) { ok = false; break; }
        const AttnMeta& M = meta[t % kAttnMR];
        const int nsl = M.nslots;
        const int last = M.last;
        if (nsl == 0) break;
        tc_fence_after();
        const uint32_t idesc_qk = umma_idesc_bf16(128, nsl * 64, 0);
        const uint32_t dS = tmem + (uint32_t)(t & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = umma_desc_sw128(sQ + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(sK(ks) + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          umma_bf16_ss(dS, a, b, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(AB_SFULL + (t & 1)));
        umma_commit(bar(AB_KEMPTY + ks));
        if (have_prev && !issue_pv(t - 1, prev_nsl)) { ok = false; break; }
        prev_nsl = nsl;
        have_prev = true;
        if (last) break;
        ++t;
      }
      if (ok && have_prev) issue_pv(t, prev_nsl);
      // Drain: every MMA of this CTA has completed before TMEM is freed.
      umma_commit(bar(AB_DRAIN));
      mbar_wait_cleanup(bar(AB_DRAIN), 0, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue (warps 2-5)
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int grpB = row >> 6;
    const int r = row & 63;
    const uint32_t laddr = tmem + ((uint32_t)(q4 * 32) << 16);
    const unsigned long long causal = (r == 63) ? ~0ull : ((1ull << (r + 1)) - 1ull);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int t = 0;
    bool ok = true, any = false;
    while (true) {
      if (!mbar_wait_warp(bar(AB_META + (t % kAttnMR)), (t / kAttnMR) & 1, ab)) { ok = false; break; }
      const AttnMeta& M = meta[t % kAttnMR];
      const int nsl = M.nslots;
      if (nsl == 0) break;
      const int last = M.last;
      unsigned long long vm0 = grpB ? M.mB[0] : M.mA[0];
      if (M.kind[0] == 1 && M.blk[0] == qb) vm0 &= causal;
      unsigned long long vm1 = 0ull;
      if (nsl > 1) {
        vm1 = grpB ? M.mB[1] : M.mA[1];
        if (M.kind[1] == 1 && M.blk[1] == qb) vm1 &= causal;
      }
      if (!mbar_wait_warp(bar(AB_SFULL + (t & 1)), (t >> 1) & 1, ab)) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      const uint32_t sa = laddr + (uint32_t)(t & 1) * 128u;
      tmem_ld32(sa, r0);
      tmem_ld32(sa + 32, r1);
      tmem_ld32(sa + 64, r2);
      tmem_ld32(sa + 96, r3);
      tmem_wait_ld();
      reg_fence(r0);
      reg_fence(r1);
      reg_fence(r2);
      reg_fence(r3);
      float x[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = __uint_as_float(r0[c]);
        x[32 + c] = __uint_as_float(r1[c]);
        x[64 + c] = __uint_as_float(r2[c]);
        x[96 + c] = __uint_as_float(r3[c]);
      }
      if (__any_sync(0xFFFFFFFFu, (vm0 & vm1) != ~0ull)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          x[c] = ((vm0 >> c) & 1ull) ? x[c] : -INFINITY;
          x[64 + c] = ((vm1 >> c) & 1ull) ? x[64 + c] : -INFINITY;
        }
      }
      // row max of the raw scores (the scale is positive, so it commutes)
      float mt0 = x[0], mt1 = x[1], mt2 = x[2], mt3 = x[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mt0 = fmaxf(mt0, x[c]);
        mt1 = fmaxf(mt1, x[c + 1]);
        mt2 = fmaxf(mt2, x[c + 2]);
        mt3 = fmaxf(mt3, x[c + 3]);
      }
      const float mt = fmaxf(fmaxf(mt0, mt1), fmaxf(mt2, mt3)) * sl2;
      float m_new = m_run;
      bool rescale = false;
      if (m_run == -INFINITY) {
        m_new = mt;
      } else if (mt > m_run + 8.0f) {
        m_new = mt;
        rescale = true;
      }
      const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
      const float nmu = (m_new == -INFINITY) ? 0.f : -m_new;
      // p = 2^(s*scale*log2e - m): two lanes per packed FMA
      float2 s01 = make_float2(0.f, 0.f), s23 = s01;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        const float2 a = ffma2(make_float2(x[c], x[c + 1]), make_float2(sl2, sl2), make_float2(nmu, nmu));
        const float2 b = ffma2(make_float2(x[c + 2], x[c + 3]), make_float2(sl2, sl2), make_float2(nmu, nmu));
        x[c] = ex2_approx(a.x);
        x[c + 1] = ex2_approx(a.y);
        x[c + 2] = ex2_approx(b.x);
        x[c + 3] = ex2_approx(b.y);
        s01 = fadd2(s01, make_float2(x[c], x[c + 1]));
        s23 = fadd2(s23, make_float2(x[c + 2], x[c + 3]));
      }
      l_run = l_run * alpha + ((s01.x + s01.y) + (s23.x + s23.y));
      m_run = m_new;
      // P buffer t&1 was read by PV(t-2); a rescale of O needs PV(t-1) done.
      const bool any_rescale = __any_sync(0xFFFFFFFFu, rescale);
      if (any_rescale && t >= 1) {
        if (!mbar_wait_warp(bar(AB_PVDONE + ((t - 1) & 1)), ((t - 1) >> 1) & 1, ab)) { ok = false; break; }
      } else if (t >= 2) {
        if (!mbar_wait_warp(bar(AB_PVDONE + (t & 1)), ((t - 2) >> 1) & 1, ab)) { ok = false; break; }
      }
      tc_fence_after();
      if (any_rescale && t >= 1) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(laddr + kTmemO + c * 32, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tmem_st32(laddr + kTmemO + c * 32, ov);
        }
      }
      // P (bf16, two keys per 32-bit column) into TMEM buffer t&1: the A operand of PV.
      {
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(x[2 * j], x[2 * j + 1]);
        tmem_st32(laddr + kTmemP + 64u * (uint32_t)(t & 1), pk);
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(x[64 + 2 * j], x[64 + 2 * j + 1]);
        tmem_st32(laddr + kTmemP + 64u * (uint32_t)(t & 1) + 32u, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(AB_PFULL + (t & 1)));
      any = true;
      if (last) break;
      ++t;
    }
    if (ok && any) ok = mbar_wait_warp(bar(AB_PVDONE + (t & 1)), (t >> 1) & 1, ab);
    const int h = grpB ? hB : hA;
    if (ok && h >= 0) {
      tc_fence_after();
      const int i = qb * 64 + r;
      const float inv = (any && l_run > 0.f) ? 1.0f / l_run : 0.f;
      __nv_bfloat16* orow = p.o + ((size_t)h * p.n + i) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (any) {
          tmem_ld32(laddr + kTmemO + c * 32, ov);
          tmem_wait_ld();
          reg_fence(ov);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(ov[q * 8 + 0]) * inv, __uint_as_float(ov[q * 8 + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(ov[q * 8 + 2]) * inv, __uint_as_float(ov[q * 8 + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(ov[q * 8 + 4]) * inv, __uint_as_float(ov[q * 8 + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(ov[q * 8 + 6]) * inv, __uint_as_float(ov[q * 8 + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = w;
        }
      }
      if (p.lse) {
        p.lse[(size_t)h * p.n + i] =
            (any && l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dsa
