// attn_fwd.cuh -- causal block-sparse FlashAttention forward on sm_100a.
//
// MInference 1.0 page, method section ("方法介紹"): attention is computed only
// over the key/value blocks the index selected (block-sparse FlashAttention);
// Fig. 4: slash lines as 64x64 blocks, vertical lines as 1x64 column tiles.
//
// Design (one CTA = 6 warps, one work item):
//  * A work item is 128 query rows that share one KV head: the same 64-token
//    query block of two q-heads of a GQA group (rows 0-63 = head A, 64-127 =
//    head B).  Their sorted block lists are merged; each merged entry records
//    which of the two heads chose it.  Column entries (1x64 tiles) of the two
//    heads are merged the same way, 64 columns per slot.
//  * A "tile" is two slots of 64 keys (N = 128 keys).  Warp 0 loads them: TMA
//    2D tile loads (128-byte swizzle) for blocks, plain 16-byte gathers for
//    columns, into a 2-stage shared-memory ring; per-stage metadata (which
//    rows may see which keys) travels with the stage.
//  * Warp 1 (one elected thread) issues tcgen05.mma: S = Q K^T (M=128, N=128,
//    K=d) into a double-buffered TMEM S, and O += P V (M=128, N=d, K=128) into
//    TMEM O.  Completion is signalled with tcgen05.commit on mbarriers.
//  * Warps 2-5 (128 threads, thread = row = TMEM lane) run the online softmax:
//    tcgen05.ld of the S row, masks, exp2, a lazy rescale of O in TMEM only
//    when the running max grows by more than 2^8, P as bf16 into shared
//    memory (the A operand of the PV MMA), and the epilogue O / l -> bf16.
//  * Every wait is bounded (2 s); on expiry the CTA records a timeout in the
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

struct AttnSlot {
  unsigned long long mA, mB;  // key c of the slot is visible to head A / B rows
  int blk;                    // key block (kind 1)
  int kind;                   // 0 empty, 1 block, 2 columns
};

struct AttnStageMeta {
  AttnSlot sl[2];
  int nslots;
  int last;
  int col[2][64];
};

template <int D>
struct AttnLayout {
  static constexpr int NDH = D / 64;              // 64-element (128-byte) column halves of d
  static constexpr int kHalf = 16384;             // one d-half of a 128-row tile (128 x 128 B)
  static constexpr int kQ = 0;
  static constexpr int kQBytes = NDH * kHalf;
  static constexpr int kKVBytes = NDH * kHalf;    // one K (or V) stage: 128 keys x d
  static constexpr int kK0 = kQ + kQBytes;
  static constexpr int kV0 = kK0 + kKVBytes;
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kP = kK0 + 2 * kStageBytes;  // 128 rows x 128 keys bf16 as two key halves
  static constexpr int kPBytes = 2 * kHalf;
  static constexpr int kMeta = kP + kPBytes;
  static constexpr int kBar = kMeta + 2 * (int)sizeof(AttnStageMeta);
  static constexpr int kNumBars = 12;
  static constexpr int kMisc = kBar + kNumBars * 8;   // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;    // slack to align the base to 1024
};

enum AttnBar { B_QFULL = 0, B_KVFULL0 = 1, B_KVEMPTY0 = 3, B_SFULL0 = 5, B_PFULL0 = 7, B_PVDONE = 9, B_DRAIN = 10 };

constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256, 256+d)

template <int D>
__global__ void __launch_bounds__(192, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using Lay = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  AttnStageMeta* meta = reinterpret_cast<AttnStageMeta*>(smem + Lay::kMeta);
  const uint32_t bar0 = sb + Lay::kBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);

  if (status_timed_out(p.status)) return;   // uniform over the CTA: before any barrier or TMEM use
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_qb = p.Hkv * p.npairs;
  const int qb = p.nQB - 1 - (int)(blockIdx.x / per_qb);   // heaviest query blocks first
  const int rem = (int)(blockIdx.x % per_qb);
  const int g = rem / p.npairs, pr = rem % p.npairs;
  const int hA = g * p.grp + 2 * pr;
  const int hB = (2 * pr + 1 < p.grp) ? hA + 1 : -1;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_KVFULL0), 1);
    mbar_init(bar(B_KVFULL0 + 1), 1);
    mbar_init(bar(B_KVEMPTY0), 1);
    mbar_init(bar(B_KVEMPTY0 + 1), 1);
    mbar_init(bar(B_SFULL0), 1);
    mbar_init(bar(B_SFULL0 + 1), 1);
    mbar_init(bar(B_PFULL0), 128);
    mbar_init(bar(B_PFULL0 + 1), 128);
    mbar_init(bar(B_PVDONE), 1);
    mbar_init(bar(B_DRAIN), 1);
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
  const uint32_t sP = sb + Lay::kP;
  auto sK = [&](int s) { return sb + Lay::kK0 + (uint32_t)s * Lay::kStageBytes; };
  auto sV = [&](int s) { return sb + Lay::kV0 + (uint32_t)s * Lay::kStageBytes; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const size_t rowA = (size_t)hA * p.nQB + qb;
    const size_t rowB = (size_t)(hB >= 0 ? hB : hA) * p.nQB + qb;
    const int32_t* LA = p.block_idx + rowA * p.kcap;
    const int32_t* LB = p.block_idx + rowB * p.kcap;
    const int na = min(max(p.block_cnt[rowA], 0), p.kcap);
    const int nb = hB >= 0 ? min(max(p.block_cnt[rowB], 0), p.kcap) : 0;
    const int32_t* CA = p.col_idx ? p.col_idx + rowA * p.ccap : nullptr;
    const int32_t* CB = p.col_idx ? p.col_idx + rowB * p.ccap : nullptr;
    const int nca = p.col_idx ? min(max(p.col_cnt[rowA], 0), p.ccap) : 0;
    const int ncb = (p.col_idx && hB >= 0) ? min(max(p.col_cnt[rowB], 0), p.ccap) : 0;
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(bar(B_QFULL), (uint32_t)Lay::kQBytes);
#pragma unroll
      for (int dh = 0; dh < Lay::NDH; ++dh) {
        tma_load_2d(sQ + dh * Lay::kHalf, &tmQ, dh * 64, hA * p.n + qb * 64, bar(B_QFULL));
        tma_load_2d(sQ + dh * Lay::kHalf + 8192, &tmQ, dh * 64, (hB >= 0 ? hB : hA) * p.n + qb * 64, bar(B_QFULL));
      }
    }
    int ia = 0, ib = 0, ja = 0, jb = 0;
    int t = 0;
    int issued = 0;
    while (true) {
      const int s = t & 1;
      if (t >= 2) {
        if (!mbar_wait_warp(bar(B_KVEMPTY0 + s), ((t - 2) >> 1) & 1, ab)) break;
      }
      AttnStageMeta& M = meta[s];
      if (lane == 0) {
        for (int sl = 0; sl < 2; ++sl) {
          AttnSlot& S = M.sl[sl];
          if (ia < na || ib < nb) {
            const int a = ia < na ? LA[ia] : 0x7FFFFFFF;
            const int b = ib < nb ? LB[ib] : 0x7FFFFFFF;
            const int blk = min(a, b);
            S.kind = 1;
            S.blk = blk;
            S.mA = (a == blk) ? ~0ull : 0ull;
            S.mB = (b == blk) ? ~0ull : 0ull;
            ia += (a == blk);
            ib += (b == blk);
          } else if (ja < nca || jb < ncb) {
            unsigned long long mA = 0, mB = 0;
            int c = 0;
            while (c < 64 && (ja < nca || jb < ncb)) {
              const int a = ja < nca ? CA[ja] : 0x7FFFFFFF;
              const int b = jb < ncb ? CB[jb] : 0x7FFFFFFF;
              const int col = min(a, b);
              if (a == col) { mA |= 1ull << c; ++ja; }
              if (b == col) { mB |= 1ull << c; ++jb; }
              M.col[sl][c] = col;
              ++c;
            }
            for (; c < 64; ++c) M.col[sl][c] = -1;
            S.kind = 2;
            S.blk = -1;
            S.mA = mA;
            S.mB = mB;
          } else {
            S.kind = 0;
            S.blk = -1;
            S.mA = S.mB = 0ull;
          }
        }
        M.nslots = (M.sl[0].kind != 0) + (M.sl[1].kind != 0);
        M.last = !(ia < na || ib < nb || ja < nca || jb < ncb);
      }
      __syncwarp();
      const int nsl = M.nslots;
      const int last = M.last;
      // columns: 16-byte gathers written in the 128-byte swizzled layout
      for (int sl = 0; sl < nsl; ++sl) {
        if (M.sl[sl].kind != 2) continue;
        constexpr int VPR = D / 8;
        for (int idx = lane; idx < 64 * VPR; idx += 32) {
          const int c = idx / VPR, v = idx % VPR;
          const int col = M.col[sl][c];
          uint4 kv4 = make_uint4(0, 0, 0, 0), vv4 = kv4;
          if (col >= 0) {
            const size_t off = ((size_t)g * p.n + col) * D + v * 8;
            kv4 = __ldg(reinterpret_cast<const uint4*>(p.k + off));
            vv4 = __ldg(reinterpret_cast<const uint4*>(p.v + off));
          }
          const uint32_t o = (uint32_t)((v >> 3) * Lay::kHalf + sl * 8192 + c * 128 + (((v & 7) ^ (c & 7)) << 4));
          st_shared_v4(sK(s) + o, kv4.x, kv4.y, kv4.z, kv4.w);
          st_shared_v4(sV(s) + o, vv4.x, vv4.y, vv4.z, vv4.w);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        uint32_t tx = 0;
        for (int sl = 0; sl < nsl; ++sl)
          if (M.sl[sl].kind == 1) tx += 2u * 64u * D * 2u;
        mbar_arrive_expect_tx(bar(B_KVFULL0 + s), tx);
        for (int sl = 0; sl < nsl; ++sl) {
          if (M.sl[sl].kind != 1) continue;
          const int row = g * p.n + M.sl[sl].blk * 64;
#pragma unroll
          for (int dh = 0; dh < Lay::NDH; ++dh) {
            tma_load_2d(sK(s) + dh * Lay::kHalf + sl * 8192, &tmK, dh * 64, row, bar(B_KVFULL0 + s));
            tma_load_2d(sV(s) + dh * Lay::kHalf + sl * 8192, &tmV, dh * 64, row, bar(B_KVFULL0 + s));
          }
        }
      }
      __syncwarp();
      ++issued;
      if (nsl == 0 || last) break;
      ++t;
    }
    // Clean-up: make sure no copy of ours is still landing in shared memory.
    if (lane == 0) {
      for (int u = max(0, issued - 2); u < issued; ++u)
        mbar_wait_cleanup(bar(B_KVFULL0 + (u & 1)), (u >> 1) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_pv = umma_idesc_bf16(128, D, 1);
      bool ok = mbar_wait(bar(B_QFULL), 0, ab);
      int t = 0, prev_nsl = 0;
      bool have_prev = false;
      auto issue_pv = [&](int u, int nsl) -> bool {
        if (!mbar_wait(bar(B_PFULL0 + (u & 1)), (u >> 1) & 1, ab)) return false;
        tc_fence_after();
        for (int kk = 0; kk < nsl * 4; ++kk) {
          const uint64_t a = umma_desc_sw128(sP + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(sV(u & 1) + kk * 2048, Lay::kHalf, 1024);
          umma_bf16_ss(tmem + 256, a, b, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_KVEMPTY0 + (u & 1)));
        umma_commit(bar(B_PVDONE));
        return true;
      };
      while (ok) {
        const int s = t & 1;
        if (!mbar_wait(bar(B_KVFULL0 + s), (t >> 1) & 1, ab)) { ok = false; break; }
        const int nsl = meta[s].nslots;
        const int last = meta[s].last;
        if (nsl == 0) break;
        tc_fence_after();
        const uint32_t idesc_qk = umma_idesc_bf16(128, nsl * 64, 0);
        const uint32_t dS = tmem + (uint32_t)(t & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = umma_desc_sw128(sQ + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(sK(s) + (kk >> 2) * Lay::kHalf + (kk & 3) * 32, 16, 1024);
          umma_bf16_ss(dS, a, b, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_SFULL0 + (t & 1)));
        if (have_prev && !issue_pv(t - 1, prev_nsl)) { ok = false; break; }
        prev_nsl = nsl;
        have_prev = true;
        if (last) break;
        ++t;
      }
      if (ok && have_prev) issue_pv(t, prev_nsl);
      // Drain: every MMA of this CTA has completed before TMEM is freed.
      umma_commit(bar(B_DRAIN));
      mbar_wait_cleanup(bar(B_DRAIN), 0, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
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
      const int s = t & 1;
      if (!mbar_wait_warp(bar(B_KVFULL0 + s), (t >> 1) & 1, ab)) { ok = false; break; }
      const AttnStageMeta& M = meta[s];
      const int nsl = M.nslots;
      if (nsl == 0) break;
      const int last = M.last;
      unsigned long long vm0 = grpB ? M.sl[0].mB : M.sl[0].mA;
      if (M.sl[0].kind == 1 && M.sl[0].blk == qb) vm0 &= causal;
      unsigned long long vm1 = 0ull;
      if (nsl > 1) {
        vm1 = grpB ? M.sl[1].mB : M.sl[1].mA;
        if (M.sl[1].kind == 1 && M.sl[1].blk == qb) vm1 &= causal;
      }
      if (!mbar_wait_warp(bar(B_SFULL0 + (t & 1)), (t >> 1) & 1, ab)) { ok = false; break; }
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
        x[c] = ((vm0 >> c) & 1ull) ? __uint_as_float(r0[c]) * sl2 : -INFINITY;
        x[32 + c] = ((vm0 >> (32 + c)) & 1ull) ? __uint_as_float(r1[c]) * sl2 : -INFINITY;
        x[64 + c] = ((vm1 >> c) & 1ull) ? __uint_as_float(r2[c]) * sl2 : -INFINITY;
        x[96 + c] = ((vm1 >> (32 + c)) & 1ull) ? __uint_as_float(r3[c]) * sl2 : -INFINITY;
      }
      float mt0 = -INFINITY, mt1 = -INFINITY, mt2 = -INFINITY, mt3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        mt0 = fmaxf(mt0, x[c]);
        mt1 = fmaxf(mt1, x[c + 1]);
        mt2 = fmaxf(mt2, x[c + 2]);
        mt3 = fmaxf(mt3, x[c + 3]);
      }
      const float mt = fmaxf(fmaxf(mt0, mt1), fmaxf(mt2, mt3));
      float m_new = m_run;
      bool rescale = false;
      if (m_run == -INFINITY) {
        m_new = mt;
      } else if (mt > m_run + 8.0f) {
        m_new = mt;
        rescale = true;
      }
      const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
      const float mu = (m_new == -INFINITY) ? 0.f : m_new;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        x[c] = ex2_approx(x[c] - mu);
        x[c + 1] = ex2_approx(x[c + 1] - mu);
        x[c + 2] = ex2_approx(x[c + 2] - mu);
        x[c + 3] = ex2_approx(x[c + 3] - mu);
        s0 += x[c];
        s1 += x[c + 1];
        s2 += x[c + 2];
        s3 += x[c + 3];
      }
      l_run = l_run * alpha + ((s0 + s1) + (s2 + s3));
      m_run = m_new;
      // PV of the previous tile must be done before O is rescaled or P rewritten.
      if (t >= 1) {
        if (!mbar_wait_warp(bar(B_PVDONE), (t - 1) & 1, ab)) { ok = false; break; }
      }
      tc_fence_after();
      if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(laddr + 256 + c * 32, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tmem_st32(laddr + 256 + c * 32, ov);
        }
        tmem_wait_st();
      }
      // P (bf16) -> shared memory, A operand of the PV MMA (K-major, 128-byte swizzle)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int c = half * 64 + ch * 8;
          const uint32_t a = pack_bf16x2(x[c], x[c + 1]);
          const uint32_t b = pack_bf16x2(x[c + 2], x[c + 3]);
          const uint32_t cc = pack_bf16x2(x[c + 4], x[c + 5]);
          const uint32_t d = pack_bf16x2(x[c + 6], x[c + 7]);
          st_shared_v4(sP + half * Lay::kHalf + row * 128 + ((ch ^ (row & 7)) << 4), a, b, cc, d);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL0 + (t & 1)));
      any = true;
      if (last) break;
      ++t;
    }
    if (ok && any) ok = mbar_wait_warp(bar(B_PVDONE), t & 1, ab);
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
          tmem_ld32(laddr + 256 + c * 32, ov);
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
