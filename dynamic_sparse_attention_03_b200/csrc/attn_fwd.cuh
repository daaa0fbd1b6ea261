// attn_fwd.cuh -- causal block-sparse FlashAttention forward on sm_100a.
//
// MInference 1.0 page, method section ("方法介紹"): attention is computed only
// over the key/value blocks the index selected (block-sparse FlashAttention);
// Fig. 4: slash lines as 64x64 blocks, vertical lines as 1x64 column tiles.
//
// Design (one CTA = 12 warps, one work item):
//  * A work item is one 64-token query block of up to four q-heads that share
//    a KV head (a GQA group).  Heads 0,1 form the 128-row query tile A, heads
//    2,3 tile B.  The four sorted block lists are merged; every merged entry
//    records which heads chose it (a 64-bit key mask per head and slot).
//    Column entries (1x64 tiles) of the heads are merged the same way, 64
//    columns per slot.  Each K/V tile therefore crosses shared memory once for
//    both query tiles.
//  * A "tile" is two slots of 64 keys (N = 128 keys).  Warp 0 streams K tiles
//    (and publishes per-tile metadata in a ring with its own barriers), warp 2
//    streams V tiles, each into a 2-stage ring: TMA 2D tile loads (128-byte
//    swizzle, no multicast) for blocks, 16-byte gathers for columns.  A K stage
//    is refilled once both QK^T products have read it, a V stage once both PV
//    products have.
//  * Warp 1 walks the MMA schedule warp-uniformly (one elected lane issues),
//    in the order QK_A(t+1), PV_B(t), QK_B(t+1), PV_A(t+1), ...:
//    S = Q K^T (M=128, shared-memory operands) into TMEM S_A / S_B, and
//    O += P V (M=128, N=d) with P read from TMEM (aliased onto the first 64
//    columns of S) and V from shared memory.  A query tile's products cover
//    only the slots one of its two heads chose: both slots (N=128), one slot
//    (N=64 QK^T, K=64 PV), or none (the tile skips that step; its barriers
//    count processed steps, so the issuer and the softmax warps, which both
//    decide from the step's metadata, stay in phase).  tcgen05.mma operations
//    of a CTA run in issue order, so the PV that reads P(t) finishes before
//    the next QK^T overwrites S.  While one softmax warpgroup works on its
//    tile, the tensor pipe runs the other tile's products.
//  * Warps 4-7 (tile A) and 8-11 (tile B) run the online softmax, one row per
//    thread (= TMEM lane): the row max over the visible keys, then
//    exp2(s*scale*log2e - max) with packed f32x2 FMAs, P (bf16) written back
//    into TMEM with tcgen05.st, a lazy rescale of O in TMEM only when the
//    running max grows by more than 2^8, and the epilogue O / l -> bf16.  A
//    slot that the row's head did not choose costs no exponentials (its P is
//    zero, written only if the other head of the tile chose it).
//  * TMEM columns: S_A [0,128) S_B [128,256) O_A [256,384) O_B [384,512).
//  * Every wait is bounded (1 s, or the caller's limit); on expiry the CTA
//    records a timeout in the status word, all roles leave their loops, TMEM is
//    freed, the CTA returns.
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
  int Hq, Hkv, n, nQB, grp, nquads;
  float scale_log2;
  uint64_t wait_ns;   // bounded-wait limit
  int stall_item;     // test hook: this work item skips its first K load (-1: none)
};

// Per-tile metadata for the MMA issuer and the softmax warpgroups.
struct alignas(16) AttnMeta {
  unsigned long long m[2][4];  // key c of slot s is visible to the rows of head hh of the item
  int blk[2];                  // key block of a block slot, -1 otherwise
  int kind[2];                 // 0 empty, 1 block, 2 columns
  int nslots, last;
};

constexpr int kAttnKS = 2;   // K stages
constexpr int kAttnVS = 2;   // V stages
constexpr int kAttnMR = 8;   // metadata ring entries (>= K stages + 2)

template <int D>
struct AttnLayout {
  static constexpr int NDH = D / 64;              // 64-element (128-byte) column halves of d
  static constexpr int kHalf = 16384;             // one d-half of a 128-row tile (128 x 128 B)
  static constexpr int kTile = NDH * kHalf;       // 128 rows x d bf16
  static constexpr int kQA = 0;
  static constexpr int kQB = kTile;
  static constexpr int kK0 = 2 * kTile;
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
  AB_SFULL = AB_VEMPTY + kAttnVS,   // [tile A, tile B]
  AB_PFULL = AB_SFULL + 2,
  AB_PVDONE = AB_PFULL + 2,
  AB_META = AB_PVDONE + 2,
  AB_DRAIN = AB_META + kAttnMR,
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0, kTmemO = 256;   // + 128 * tile

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

// Writes 32 columns of zeros (32 lanes x 32 columns) at taddr.
__device__ __forceinline__ void tmem_st32_zero(uint32_t taddr) {
  const uint32_t z = 0u;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr), "r"(z)
      : "memory");
}

// Merge cursor over the item's heads' sorted lists (blocks first, then columns).
struct AttnLists {
  const int32_t* L[4];
  const int32_t* C[4];
  int nl[4], nc[4];
  int nh;
};

struct AttnCursor {
  int il[4] = {0, 0, 0, 0}, ic[4] = {0, 0, 0, 0};

  __device__ bool more_blocks(const AttnLists& A) const {
    bool r = false;
#pragma unroll
    for (int h = 0; h < 4; ++h) r |= (h < A.nh && il[h] < A.nl[h]);
    return r;
  }
  __device__ bool more_cols(const AttnLists& A) const {
    bool r = false;
#pragma unroll
    for (int h = 0; h < 4; ++h) r |= (h < A.nh && ic[h] < A.nc[h]);
    return r;
  }

  // Forms the next tile (up to two slots of 64 keys) into M; column slots also
  // record their key columns in cols[slot][0..64) (-1 padded).
  __device__ void next(const AttnLists& A, AttnMeta& M, int (*cols)[64]) {
    for (int sl = 0; sl < 2; ++sl) {
#pragma unroll
      for (int h = 0; h < 4; ++h) M.m[sl][h] = 0ull;
      if (more_blocks(A)) {
        int v[4];
        int blk = 0x7FFFFFFF;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          v[h] = (h < A.nh && il[h] < A.nl[h]) ? A.L[h][il[h]] : 0x7FFFFFFF;
          blk = min(blk, v[h]);
        }
#pragma unroll
        for (int h = 0; h < 4; ++h)
          if (v[h] == blk) {
            M.m[sl][h] = ~0ull;
            ++il[h];
          }
        M.kind[sl] = 1;
        M.blk[sl] = blk;
      } else if (more_cols(A)) {
        int c = 0;
        while (c < 64 && more_cols(A)) {
          int v[4];
          int col = 0x7FFFFFFF;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[h] = (h < A.nh && ic[h] < A.nc[h]) ? A.C[h][ic[h]] : 0x7FFFFFFF;
            col = min(col, v[h]);
          }
#pragma unroll
          for (int h = 0; h < 4; ++h)
            if (v[h] == col) {
              M.m[sl][h] |= 1ull << c;
              ++ic[h];
            }
          cols[sl][c] = col;
          ++c;
        }
        for (; c < 64; ++c) cols[sl][c] = -1;
        M.kind[sl] = 2;
        M.blk[sl] = -1;
      } else {
        M.kind[sl] = 0;
        M.blk[sl] = -1;
      }
    }
    M.nslots = (M.kind[0] != 0) + (M.kind[1] != 0);
    M.last = !(more_blocks(A) || more_cols(A));
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
__global__ void __launch_bounds__(384, 1)
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
  // Work items run KV head by KV head, heaviest query blocks first within a
  // head: the CTAs in flight together read one head's key/value blocks, which
  // stay in L2 for all of them.
  const int per_head = p.nQB * p.nquads;
  const int g = (int)(blockIdx.x / per_head);
  const int rem = (int)(blockIdx.x % per_head);
  const int qb = p.nQB - 1 - rem / p.nquads, quad = rem % p.nquads;
  const int h0 = g * p.grp + 4 * quad;
  const int nh = min(4, p.grp - 4 * quad);
  const bool hasB = nh > 2;

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
      mbar_init(bar(AB_PFULL + b), 4);   // one arrival per softmax warp
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
  const AbortState ab{abort_flag, p.status, p.wait_ns};

  auto sQ = [&](int tile) { return sb + (tile ? Lay::kQB : Lay::kQA); };
  auto sK = [&](int s) { return sb + Lay::kK0 + (uint32_t)s * Lay::kTile; };
  auto sV = [&](int s) { return sb + Lay::kV0 + (uint32_t)s * Lay::kTile; };
  // slot s of a step is computed for query tile X (heads 2X, 2X+1 of the item)
  // when one of those heads chose it
  auto vis = [](const AttnMeta& M, int X, int s) { return (M.m[s][2 * X] | M.m[s][2 * X + 1]) != 0ull; };

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    AttnLists A;
    A.nh = nh;
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      const int h = h0 + min(hh, nh - 1);
      const size_t row = (size_t)h * p.nQB + qb;
      A.L[hh] = p.block_idx + row * p.kcap;
      A.C[hh] = p.col_idx ? p.col_idx + row * p.ccap : nullptr;
      A.nl[hh] = hh < nh ? min(max(p.block_cnt[row], 0), p.kcap) : 0;
      A.nc[hh] = (hh < nh && p.col_idx) ? min(max(p.col_cnt[row], 0), p.ccap) : 0;
    }
    AttnCursor cur;
    const bool isK = (warp == 0);
    const int NS = isK ? kAttnKS : kAttnVS;
    if (isK && lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      // the query tile is read once: its L2 lines go first, ahead of the
      // key/value blocks other query blocks reuse
      const uint64_t once = l2_policy_evict_first();
      mbar_arrive_expect_tx(bar(AB_Q), (uint32_t)(2 * Lay::kTile));
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        const int h = h0 + min(hh, nh - 1);
#pragma unroll
        for (int dh = 0; dh < Lay::NDH; ++dh)
          tma_load_2d_hint(sQ(hh >> 1) + dh * Lay::kHalf + (hh & 1) * 8192, &tmQ, dh * 64, h * p.n + qb * 64,
                           bar(AB_Q), once);
      }
    }
    if (!isK && lane == 0) prefetch_tmap(&tmV);
    const CUtensorMap* tm = isK ? &tmK : &tmV;
    const __nv_bfloat16* base = (isK ? p.k : p.v) + (size_t)g * p.n * D;
    int(*cols)[64] = isK ? colsK : colsV;
    const int full0 = isK ? AB_KFULL : AB_VFULL, empty0 = isK ? AB_KEMPTY : AB_VEMPTY;
    // test hook: the K producer of work item stall_item issues nothing for its
    // first tile, so the MMA warp's wait for it runs out (nothing is in flight)
    const int skipped = (isK && p.stall_item == (int)blockIdx.x) ? 0 : -1;
    int t = 0, issued = 0;
    while (true) {
      const int s = t % NS;
      if (t >= NS && !mbar_wait_warp(bar(empty0 + s), ((t / NS) - 1) & 1, ab)) break;
      AttnMeta& M = isK ? meta[t % kAttnMR] : *vrec;
      if (lane == 0) cur.next(A, M, cols);
      __syncwarp();
      const int nsl = M.nslots, last = M.last;
      if (!isK && nsl == 0) break;
      const int k0 = M.kind[0], k1 = M.kind[1];
      const int b0 = M.blk[0], b1 = M.blk[1];
      const uint32_t stg = isK ? sK(s) : sV(s);
      if (k0 == 2) gather_slot<D>(base, cols[0], stg, 0, lane);
      if (k1 == 2) gather_slot<D>(base, cols[1], stg, 1, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (isK) mbar_arrive(bar(AB_META + (t % kAttnMR)));
        if (t != skipped) {
          const uint32_t tx = (uint32_t)((k0 == 1) + (k1 == 1)) * 64u * D * 2u;
          mbar_arrive_expect_tx(bar(full0 + s), tx);
          if (k0 == 1)
#pragma unroll
            for (int dh = 0; dh < Lay::NDH; ++dh)
              tma_load_2d(stg + dh * Lay::kHalf, tm, dh * 64, g * p.n + b0 * 64, bar(full0 + s));
          if (k1 == 1)
#pragma unroll
            for (int dh = 0; dh < Lay::NDH; ++dh)
              tma_load_2d(stg + dh * Lay::kHalf + 8192, tm, dh * 64, g * p.n + b1 * 64, bar(full0 + s));
        }
      }
      __syncwarp();
      ++issued;
      if (nsl == 0 || last) break;
      ++t;
    }
    // wait for this producer's own copies still in flight (none for a skipped tile)
    if (lane == 0) {
      for (int u = max(0, issued - NS); u < issued; ++u)
        if (u != skipped) mbar_wait_cleanup(bar(full0 + (u % NS)), (u / NS) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule, so every descriptor and TMEM address
    // is warp-uniform and computed once per tile from fixed bases (a
    // descriptor's start field is the shared address >> 4; adding an offset
    // >> 4 moves it, with no carry past the 14-bit field below 256 KB).  One
    // elected lane issues each tcgen05 instruction.
    const bool issuer = elect_one();
    const uint32_t idesc_pv = umma_idesc_bf16(128, D, 1);
    const uint32_t idesc_qk2 = umma_idesc_bf16(128, 128, 0), idesc_qk1 = umma_idesc_bf16(128, 64, 0);
    const uint64_t dQ0 = umma_desc_sw128(sQ(0), 16, 1024), dQ1 = umma_desc_sw128(sQ(1), 16, 1024);
    const uint64_t dK0 = umma_desc_sw128(sK(0), 16, 1024);
    const uint64_t dV0 = umma_desc_sw128(sV(0), Lay::kHalf, 1024);
    // S_X = Q_X K^T over the chosen slots v0 / v1 of K stage ks (key rows
    // 64..127 of a stage start 8192 bytes into each d-half)
    auto qk = [&](int X, int ks, bool v0, bool v1) {
      const uint32_t idesc = (v0 && v1) ? idesc_qk2 : idesc_qk1;
      const uint32_t first = v0 ? 0u : 1u;
      const uint32_t dS = tmem + kTmemS + 128u * (uint32_t)X + 64u * first;
      const uint64_t a0 = X ? dQ1 : dQ0;
      const uint64_t b0 = dK0 + (uint64_t)(((uint32_t)ks * (uint32_t)Lay::kTile + 8192u * first) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * Lay::kHalf + (kk & 3) * 32) >> 4);
        if (issuer) umma_bf16_ss(dS, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
      }
      if (issuer) umma_commit(bar(AB_SFULL + X));
    };
    // O_X += P_X V over the chosen slots of V stage u; the first product of the
    // item into O_X starts the accumulator
    bool acc[2] = {false, false};
    auto pv = [&](int X, int u, bool v0, bool v1) {
      const uint64_t b0 = dV0 + (uint64_t)(((uint32_t)(u % kAttnVS) * (uint32_t)Lay::kTile) >> 4);
      const uint32_t pa = tmem + kTmemS + 128u * (uint32_t)X;   // P aliases the first 64 columns of S
      const uint32_t dO = tmem + kTmemO + 128u * (uint32_t)X;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (kk < 4 ? v0 : v1) {
          if (issuer) umma_bf16_ts(dO, pa + 8u * (uint32_t)kk, b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                                   acc[X] ? 1u : 0u);
          acc[X] = true;
        }
      }
    };
    bool ok = mbar_wait_warp(bar(AB_Q), 0, ab);
    int t = 0, last = 1;
    bool done[2] = {false, false};   // the epilogue's arrival on PVDONE_X was committed
    int nP[2] = {0, 0};   // P phases consumed per query tile
    bool cv[2][2] = {{false, false}, {false, false}};   // chosen slots of step t per tile
    if (ok) ok = mbar_wait_warp(bar(AB_KFULL), 0, ab);
    if (ok) {
      const AttnMeta& M = meta[0];
      last = M.last;
      if (M.nslots > 0) {
        tc_fence_after();
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          cv[X][0] = (X == 0 || hasB) && vis(M, X, 0);
          cv[X][1] = (X == 0 || hasB) && vis(M, X, 1);
          if (cv[X][0] || cv[X][1]) qk(X, 0, cv[X][0], cv[X][1]);
        }
        if (issuer) umma_commit(bar(AB_KEMPTY));
      } else {
        ok = false;
      }
    }
    while (ok) {
      // PV_X(t) ; QK_X(t+1) for X = A, B.  The operand tiles usually land
      // before P does, so their waits come first.
      bool nv[2][2] = {{false, false}, {false, false}};
      int last_next = 1;
      const int ks = (t + 1) % kAttnKS;
      if (!mbar_wait_warp(bar(AB_VFULL + (t % kAttnVS)), (t / kAttnVS) & 1, ab)) break;
      if (!last) {
        if (!mbar_wait_warp(bar(AB_KFULL + ks), ((t + 1) / kAttnKS) & 1, ab)) break;
        const AttnMeta& M = meta[(t + 1) % kAttnMR];
        last_next = M.last;
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          nv[X][0] = (X == 0 || hasB) && vis(M, X, 0);
          nv[X][1] = (X == 0 || hasB) && vis(M, X, 1);
        }
      }
      bool stop = false;
#pragma unroll
      for (int X = 0; X < 2; ++X) {   // unrolled: X is a constant, the per-tile flags stay in registers
        if (!stop && (cv[X][0] || cv[X][1])) {
          if (!mbar_wait_warp(bar(AB_PFULL + X), nP[X] & 1, ab)) {
            stop = true;
          } else {
            ++nP[X];
            tc_fence_after();
            pv(X, t, cv[X][0], cv[X][1]);
            if (last && issuer) umma_commit(bar(AB_PVDONE + X));   // O_X is final once this completes
            done[X] = done[X] || last;
          }
        }
        if (!stop && !last && (nv[X][0] || nv[X][1])) qk(X, ks, nv[X][0], nv[X][1]);
      }
      if (stop) break;
      if (issuer) {
        umma_commit(bar(AB_VEMPTY + (t % kAttnVS)));
        if (!last) umma_commit(bar(AB_KEMPTY + ks));
      }
      if (last) break;
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        cv[X][0] = nv[X][0];
        cv[X][1] = nv[X][1];
      }
      last = last_next;
      ++t;
    }
    // One arrival per query tile on PVDONE (a tile that did not compute the
    // last step, or an aborted run, gets it here), and every MMA of this CTA
    // has completed before TMEM is freed.
    if (issuer) {
      if (!done[0]) umma_commit(bar(AB_PVDONE + 0));
      if (!done[1]) umma_commit(bar(AB_PVDONE + 1));
      umma_commit(bar(AB_DRAIN));
      mbar_wait_cleanup(bar(AB_DRAIN), 0, 200000000ull);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    const int tile = (warp - 4) >> 2;     // 0: warps 4-7, 1: warps 8-11
    const int q4 = warp & 3;              // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;
    const int hh = 2 * tile + (row >> 6);  // head of the item for this row (warp-uniform)
    const int r = row & 63;
    const bool active = (tile == 0) || hasB;
    const uint32_t laddr = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t sS = laddr + kTmemS + 128u * (uint32_t)tile;
    const uint32_t sO = laddr + kTmemO + 128u * (uint32_t)tile;
    const unsigned long long causal = (r == 63) ? ~0ull : ((1ull << (r + 1)) - 1ull);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int t = 0, nS = 0;   // steps seen; S phases consumed (steps this tile computed)
    bool ok = true;
    while (active) {
      if (!mbar_wait_warp(bar(AB_META + (t % kAttnMR)), (t / kAttnMR) & 1, ab)) { ok = false; break; }
      const AttnMeta& M = meta[t % kAttnMR];
      const int nsl = M.nslots;
      if (nsl == 0) break;
      const int last = M.last;
      const bool c0 = vis(M, tile, 0), c1 = nsl > 1 && vis(M, tile, 1);   // slots the tile computed
      if (!c0 && !c1) {   // neither head of this tile chose this step
        if (last) break;
        ++t;
        continue;
      }
      // this row's keys per slot (warp-uniform: a warp's rows share one head)
      unsigned long long vm0 = c0 ? M.m[0][hh] : 0ull;
      if (M.kind[0] == 1 && M.blk[0] == qb) vm0 &= causal;
      unsigned long long vm1 = c1 ? M.m[1][hh] : 0ull;
      if (nsl > 1 && M.kind[1] == 1 && M.blk[1] == qb) vm1 &= causal;
      // a slot is visible, hidden (no exponentials), or partial (the diagonal
      // block, column slots: per-key masks)
      const bool none0 = __all_sync(0xFFFFFFFFu, vm0 == 0ull), none1 = __all_sync(0xFFFFFFFFu, vm1 == 0ull);
      const bool full0 = __all_sync(0xFFFFFFFFu, vm0 == ~0ull), full1 = __all_sync(0xFFFFFFFFu, vm1 == ~0ull);
      if (!mbar_wait_warp(bar(AB_SFULL + tile), nS & 1, ab)) { ok = false; break; }
      ++nS;
      tc_fence_after();
      // the S row of both slots in registers with one TMEM round trip (a slot
      // the tile did not compute, or that this row's head hid, is never read
      // from these registers); hidden keys of partial slots are set to -inf
      uint32_t sv[4][32];
      tmem_ld32(sS, sv[0]);
      tmem_ld32(sS + 32, sv[1]);
      if (nsl > 1) {
        tmem_ld32(sS + 64, sv[2]);
        tmem_ld32(sS + 96, sv[3]);
      }
      tmem_wait_ld();
      reg_fence(sv[0]);
      reg_fence(sv[1]);
      reg_fence(sv[2]);
      reg_fence(sv[3]);
      if (!none0 && !full0) {
        const uint32_t lo = (uint32_t)vm0, hi = (uint32_t)(vm0 >> 32);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sv[0][c] = ((lo >> c) & 1u) ? sv[0][c] : 0xFF800000u;
          sv[1][c] = ((hi >> c) & 1u) ? sv[1][c] : 0xFF800000u;
        }
      }
      if (!none1 && !full1) {
        const uint32_t lo = (uint32_t)vm1, hi = (uint32_t)(vm1 >> 32);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sv[2][c] = ((lo >> c) & 1u) ? sv[2][c] : 0xFF800000u;
          sv[3][c] = ((hi >> c) & 1u) ? sv[3][c] : 0xFF800000u;
        }
      }
      // row max of the raw scores over the visible keys (the scale is positive)
      float x0 = -INFINITY, x1 = -INFINITY, x2 = -INFINITY, x3 = -INFINITY;
      if (!none0) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          x0 = fmax3(x0, __uint_as_float(sv[0][c]), __uint_as_float(sv[0][c + 1]));
          x1 = fmax3(x1, __uint_as_float(sv[0][c + 2]), __uint_as_float(sv[0][c + 3]));
          x2 = fmax3(x2, __uint_as_float(sv[1][c]), __uint_as_float(sv[1][c + 1]));
          x3 = fmax3(x3, __uint_as_float(sv[1][c + 2]), __uint_as_float(sv[1][c + 3]));
        }
      }
      if (!none1) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          x0 = fmax3(x0, __uint_as_float(sv[2][c]), __uint_as_float(sv[2][c + 1]));
          x1 = fmax3(x1, __uint_as_float(sv[2][c + 2]), __uint_as_float(sv[2][c + 3]));
          x2 = fmax3(x2, __uint_as_float(sv[3][c]), __uint_as_float(sv[3][c + 1]));
          x3 = fmax3(x3, __uint_as_float(sv[3][c + 2]), __uint_as_float(sv[3][c + 3]));
        }
      }
      const float mt = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)) * sl2;
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
      // p = 2^(s*scale*log2e - m); P (bf16, two keys per 32-bit column) over
      // the first 64 columns of S, which have all been read above.  A slot
      // the tile computed but this row's head did not choose gets P = 0.
      float2 sum2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        if (!(sl ? c1 : c0)) continue;
        if (sl ? none1 : none0) {
          tmem_st32_zero(sS + 32 * sl);
        } else {
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 ea =
                ffma2(make_float2(__uint_as_float(sv[2 * sl][2 * j]), __uint_as_float(sv[2 * sl][2 * j + 1])),
                      make_float2(sl2, sl2), make_float2(nmu, nmu));
            const float2 eb =
                ffma2(make_float2(__uint_as_float(sv[2 * sl + 1][2 * j]), __uint_as_float(sv[2 * sl + 1][2 * j + 1])),
                      make_float2(sl2, sl2), make_float2(nmu, nmu));
            const float2 pa = make_float2(ex2_approx(ea.x), ex2_approx(ea.y));
            const float2 pb = make_float2(ex2_approx(eb.x), ex2_approx(eb.y));
            sum2 = fadd2(sum2, fadd2(pa, pb));
            pk[j] = pack_bf16x2(pa.x, pa.y);
            pk[16 + j] = pack_bf16x2(pb.x, pb.y);
          }
          tmem_st32(sS + 32 * sl, pk);
        }
      }
      l_run = l_run * alpha + (sum2.x + sum2.y);
      m_run = m_new;
      // O rescale: the PV of the previous step has completed (it was issued
      // before this step's QK^T, and the commit of S waits for every earlier
      // product of the CTA).
      if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(sO + c * 32, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tmem_st32(sO + c * 32, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(AB_PFULL + tile));
      if (last) break;
      ++t;
    }
    const bool any = nS > 0;
    if (active && ok) ok = mbar_wait_warp(bar(AB_PVDONE + tile), 0, ab);
    if (active && ok && hh < nh) {
      tc_fence_after();
      const int h = h0 + hh;
      const int i = qb * 64 + r;
      const float inv = (any && l_run > 0.f) ? 1.0f / l_run : 0.f;
      __nv_bfloat16* orow = p.o + ((size_t)h * p.n + i) * D;
      const uint64_t once = l2_policy_evict_first();   // written once, not read here again
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (any) {
          tmem_ld32(sO + c * 32, ov);
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
          st_global_v4_evict_first(orow + c * 32 + q * 8, w, once);
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
