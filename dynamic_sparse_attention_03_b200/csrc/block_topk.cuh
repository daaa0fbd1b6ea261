// block_topk.cuh -- pooled block scores and the per-query-block top-k in one
// kernel, so the score matrix never leaves the chip (MInference 1.0 page,
// method section "方法介紹": pooled Q̄·K̄ᵀ estimates the block-sparse index;
// the selection keeps the sink and the diagonal block plus the best others,
// ties to the lower block).
//
// A persistent grid walks tiles of (q-head, 128 query blocks), heaviest first.
// A tile's Q̄ (FP16 hi and lo halves of the scaled means, see
// pool_blocks_kernel) sits in tensor memory as the A operand; the KV head's K̄
// (FP16 hi and lo) streams through a TMA ring in chunks of 128 key blocks;
// S = Q̄·K̄ᵀ for a chunk is computed with tcgen05 into one of two TMEM buffers,
// and each query block's row of the chunk is read by two threads (one TMEM
// lane, 64 columns each).  Rather than storing the scores, the kernel
// recomputes them in passes:
//
//   pass 0 (approximate, Q̄hi·K̄hi only): min, max, mean and spread of a
//           sample of the row (the first 32 columns of every 4th chunk), which
//           place a 256-bin value window over the row; rows of at most four
//           chunks are read whole and the window is their range;
//   pass 1 (approximate): a 256-bin histogram of the row in that window gives
//           the bin holding the row's e-th largest score;
//   pass 2 (exact: Q̄hi·K̄hi + Q̄hi·K̄lo + Q̄lo·K̄hi): scores above that bin
//           (widened by a quarter bin on each side) are kept at once, as bits
//           of a per-chunk mask in
//           scratch memory; scores inside it are buffered as (key, id)
//           candidates.  If the kept count and the candidates bracket e, the
//           e-th largest key T and the number of T-valued ids to keep are
//           found among the candidates and the chosen ones join the masks.
//           The approximate passes only choose the window: the result is
//           exact whatever they returned.
//
// A row whose window does not bracket e (or overflows the buffer) falls back
// to exact passes: a 256-bin histogram in the value window, then 8-bit radix
// passes over the order-preserving keys of the boundary set until it is small
// enough to buffer or the key is fully known.  Every exact pass recomputes the
// same scores bit for bit (the same MMA sequence), so the passes agree.
//
// A second kernel writes the lists from the masks, one warp per query block
// (ascending ids; each lane writes the ids of one mask word).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "index_kernels.cuh"
#include "ptx.cuh"

namespace dsa {

template <int D>
struct TopkLayout {
  static constexpr int kStages = 6;                 // ring of stages, each 128 key blocks x 64 fp16
  static constexpr int kTile = 128 * 128;
  static constexpr int kRow = kStages * kTile;      // per-row private words: [128 words][128 rows] u32
  static constexpr int kRowBytes = 128 * 128 * 4;
  static constexpr int kPub = kRow + kRowBytes;     // TopkPub
  static constexpr int kPubBytes = 10 * 128 * 4;
  static constexpr int kBar = kPub + kPubBytes;     // 23 mbarriers
  static constexpr int kCtl = kBar + 256;
  static constexpr int kBytes = kCtl + 64;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int NDC = D / 64;                // d chunks of 64 fp16 (one 128-byte swizzled row)
  static_assert(NDC >= 1 && NDC <= 2, "D is 64 or 128");
  static_assert(kStages % 2 == 0, "stages are claimed in pairs");
};

constexpr int kTopkCap = 32;         // buffered boundary candidates per row thread
constexpr int kTopkMaxPasses = 12;   // 3 + histogram + 4 radix + collect, with margin

struct TopkParams {
  int32_t* block_idx;
  int32_t* block_cnt;
  uint32_t* status;
  uint32_t* masks;     // kept-column bits, see topk_mask_row
  int* next_tile;      // tile counter (zero at launch): CTAs take tiles in order, heaviest first
  int nQB, Hq, grp, kcap, k_fixed, nrt, ntiles;
  int h0, nh;          // q-heads h0 .. h0 + nh - 1 are this launch's (ntiles = nrt * nh)
  int64_t ppm;
  const __half* qhi;   // [Hq * nQB][D] FP16 halves of the scaled query-block means
  const __half* qlo;
};

__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

enum : int {
  kSelDone = 0,
  kSelStats = 1,    // approximate: min / max / mean / spread of a sample
  kSelAHist = 2,    // approximate: histogram in the value window
  kSelWindow = 3,   // exact: keep above the window, buffer inside it
  kSelHist = 4,     // exact fallback: histogram in the value window
  kSelRadix = 5,    // exact fallback: 8-bit key digit inside the boundary set
  kSelCollect = 6,  // exact: keep above the boundary set, buffer inside it
  kSelExact = 7,    // exact: threshold key known, keep in one sweep
};

__device__ __forceinline__ bool topk_hist_mode(int m) { return m == kSelAHist || m == kSelHist || m == kSelRadix; }

struct TopkRow {
  int i, L, e, mode;
  float inv, nlo;              // value bin = round(255 * sat(s * inv + nlo)), see topk_bin
  float wlo, whi;              // window of the exact pass
  float mn, mx, sum, sq, cnt;  // approximate statistics of the sample
  int b0;                      // boundary value bin (fallback)
  uint32_t prefix, mask;       // key digits fixed so far (fallback)
  int shift;
  int rem;                     // ids still to take from the boundary set
  uint32_t T;                  // threshold key (kSelExact)
  int need, eq;                // T-valued ids to keep / seen
  int nd, nc;                  // kept / buffered by this thread in this pass
};

// What the second thread of a row needs of the row's state (published by the
// first thread at each pass end), and what it reports back (its counts).
struct TopkPub {
  int mode[128];
  float inv[128], nlo[128], wlo[128], whi[128];
  int b0[128];
  uint32_t prefix[128], mask[128];
  int shift[128];
  int cnt2[128];   // second thread: nd | nc << 16
};

// Value bin in [0, 255]: y = s * inv + nlo saturated to [0, 1] (a NaN gives
// 0), then b = 255 y rounded to the nearest integer by adding 1.5 * 2^23 in
// the same multiply-add (no float-to-int conversion).  topk_bin_bits returns
// the float's bits, 0x4B400000 + b, whose low 8 bits are b.  Every step is
// monotone in s, so the bin order is the score order; all passes that compare
// bins use this same function.  A window [lo, hi] has inv = 1 / (hi - lo) and
// nlo = -lo * inv; bin b then holds the scores near lo + b (hi - lo) / 255.
__device__ __forceinline__ uint32_t topk_bin_bits(float s, float inv, float nlo) {
  const float y = __saturatef(fmaf(s, inv, nlo));
  return __float_as_uint(fmaf(y, 255.f, 12582912.f));
}
__device__ __forceinline__ int topk_bin(float s, float inv, float nlo) {
  return (int)(topk_bin_bits(s, inv, nlo) - 0x4B400000u);
}

// Private per-row words in shared memory: word w of row r at [w][r] (row r's
// words share one bank, so a warp's 32 rows never conflict).
struct RowWords {
  uint32_t* base;
  uint32_t sbase;   // shared-space address of base
  int r;
  __device__ __forceinline__ uint32_t& operator[](int w) const { return base[w * 128 + r]; }
  __device__ __forceinline__ uint32_t addr(int w) const { return sbase + (uint32_t)(w * 128 + r) * 4u; }
};

__device__ __forceinline__ void hist_clear(const RowWords& W) {
#pragma unroll 8
  for (int w = 0; w < 128; ++w) W[w] = 0u;
}

// 16-bit bin counts, two per word: bins b and b + 128 share word b & 127
// (low and high half).  Adds 1 to bin (b & 255), when `on` for hist_add_if:
// a shared-memory reduction (red, no result), so consecutive adds to one word
// do not wait on each other; both threads of a row add into the same words.
// b may carry bits above the low 8 (topk_bin_bits).  The words are read only
// after a barrier, which orders these adds before the reads.
__device__ __forceinline__ void hist_add(const RowWords& W, uint32_t b) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(W.addr((int)(b & 127u))), "r"((b & 128u) ? 65536u : 1u));
}
__device__ __forceinline__ void hist_add_if(const RowWords& W, uint32_t b, bool on) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "@p red.shared.add.u32 [%0], %1;\n\t}" ::"r"(W.addr((int)(b & 127u))),
      "r"((b & 128u) ? 65536u : 1u), "r"((uint32_t)on));
}

// Upper-tail quantile of the standard normal: z with P(Z > z) = q, from the
// rational approximation of Abramowitz and Stegun (26.2.23, |error| < 4.5e-4).
// Only used to place the approximate histogram's window.
__device__ __forceinline__ float normal_upper_quantile(float q) {
  const bool lower = q > 0.5f;
  const float qq = fminf(fmaxf(lower ? 1.f - q : q, 1e-7f), 0.5f);
  const float t = sqrtf(-2.f * __logf(qq));
  const float z = t - (2.515517f + t * (0.802853f + t * 0.010328f)) /
                          (1.f + t * (1.432788f + t * (0.189269f + t * 0.001308f)));
  return lower ? -z : z;
}

// Bin holding the t-th largest element (1 <= t <= total), scanning 16-bit
// counts from the top: returns the bin, the count strictly above it and its own.
// Two levels, without data-dependent branches until the end: the totals of
// the 32 batches of 8 bins (each word loaded once, both halves summed), then
// the batch holding the t-th element, then its 8 bins.
__device__ __forceinline__ void hist_find(const RowWords& W, int t, int& bin, int& above, int& cnt) {
  int tot[32];   // tot[j]: bins 8j .. 8j+7 (j >= 16: high halves of words 8(j-16) ..)
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    int lo = 0, hi = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t x = W[8 * j + k];
      lo += (int)(x & 0xFFFFu);
      hi += (int)(x >> 16);
    }
    tot[j] = lo;
    tot[16 + j] = hi;
  }
  int acc = 0, jb = 0, ab = 0;
  bool found = false;
#pragma unroll
  for (int j = 31; j >= 0; --j) {
    const bool here = !found && acc + tot[j] >= t;
    jb = here ? j : jb;
    ab = here ? acc : ab;
    found = found || here;
    acc += tot[j];
  }
  above = ab;
  bin = 0;
  cnt = 0;
  if (!found) {   // fewer than t elements in all: bin 0, everything above it
    above = acc;
    return;
  }
  const int sh = jb >= 16 ? 16 : 0, w0 = 8 * (jb & 15);
  int c[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) c[k] = (int)((W[w0 + k] >> sh) & 0xFFFFu);
  bool got = false;
#pragma unroll
  for (int k = 7; k >= 0; --k) {
    const bool here = !got && above + c[k] >= t;
    if (here) {
      bin = 8 * jb + k;
      cnt = c[k];
    }
    if (!got && !here) above += c[k];
    got = got || here;
  }
}

// Candidate buffers: the first thread of a row uses slots [0, kTopkCap), the
// second [kTopkCap, 2 kTopkCap); keys at words [slot], ids at [64 + slot].
// r of the buffered candidates (keys above T, then the lowest-id T-valued
// ones) are chosen and set in the row's masks.
__device__ __forceinline__ void topk_resolve(const RowWords& W, int ncA, int ncB, int r, uint32_t* mrow) {
  const int nc = ncA + ncB;
  auto slot = [&](int x) { return x < ncA ? x : kTopkCap + (x - ncA); };
  if (r <= 0) return;
  uint32_t T = 0;
  int need = 0;
  const bool all = (r >= nc);
  if (!all) {
    for (int x = 0; x < nc; ++x) {
      const uint32_t kx = W[slot(x)];
      int g = 0, eqc = 0;
      for (int y = 0; y < nc; ++y) {
        const uint32_t ky = W[slot(y)];
        g += ky > kx;
        eqc += ky == kx;
      }
      if (g < r && r <= g + eqc) {
        T = kx;
        need = r - g;
        break;
      }
    }
  }
  uint64_t taken = 0ull;   // T-valued candidates chosen (bit per x), lowest ids first
  for (int q = 0; q < need && !all; ++q) {
    int best = -1;
    uint32_t bid = 0xFFFFFFFFu;
    for (int x = 0; x < nc; ++x) {
      const uint32_t id = W[64 + slot(x)];
      if (!((taken >> x) & 1ull) && W[slot(x)] == T && id < bid) {
        bid = id;
        best = x;
      }
    }
    if (best < 0) break;
    taken |= 1ull << best;
  }
  for (int x = 0; x < nc; ++x) {
    if (all || W[slot(x)] > T || ((taken >> x) & 1ull)) {
      const int j = (int)W[64 + slot(x)];
      atomicOr(mrow + (j >> 7) * 4 + ((j & 127) >> 5), 1u << (j & 31));   // no result: a reduction
    }
  }
}

// v[t] for a run-time t: a five-level select tree on the bits of t (an
// indexed register array would live in local memory).
__device__ __forceinline__ uint32_t select32(const uint32_t (&v)[32], int t) {
  uint32_t a[16], b[8], c[4], d[2];
#pragma unroll
  for (int k = 0; k < 16; ++k) a[k] = (t & 1) ? v[2 * k + 1] : v[2 * k];
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = (t & 2) ? a[2 * k + 1] : a[2 * k];
#pragma unroll
  for (int k = 0; k < 4; ++k) c[k] = (t & 4) ? b[2 * k + 1] : b[2 * k];
#pragma unroll
  for (int k = 0; k < 2; ++k) d[k] = (t & 8) ? c[2 * k + 1] : c[2 * k];
  return (t & 16) ? d[1] : d[0];
}

// Buffers the candidates `in` of a group at slots base + nc, ...: key and id
// (candidates are few per group: one select per candidate).  Slots past
// kTopkCap are counted but not stored.
__device__ __forceinline__ void topk_buffer(const uint32_t (&v)[32], uint32_t in, int base, int nc, int jx,
                                            const RowWords& W) {
  while (in) {
    const int t = __ffs(in) - 1;
    in &= in - 1u;
    if (nc < kTopkCap) {
      W[base + nc] = float_key(__uint_as_float(select32(v, t)));
      W[64 + base + nc] = (uint32_t)(jx + t);
    }
    ++nc;
  }
}

// Statistics and histogram work of one thread on 32 consecutive scores of a
// chunk; `valid` has bit t set for the row's candidates.  Branch-free per
// element (selects, zero increments).
__device__ __forceinline__ void topk_accum32(TopkRow& R, const uint32_t (&v)[32], uint32_t valid,
                                             const RowWords& W) {
  const float kInf = __int_as_float(0x7f800000);
  if (R.mode == kSelStats) {
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const bool ok = (valid >> t) & 1u;
      const float s = __uint_as_float(v[t]);
      R.mn = fminf(R.mn, ok ? s : kInf);
      R.mx = fmaxf(R.mx, ok ? s : -kInf);
      const float z = ok ? s : 0.f;
      R.sum += z;
      R.sq = fmaf(z, z, R.sq);
    }
    R.cnt += (float)__popc(valid);
  } else if (R.mode == kSelAHist || R.mode == kSelHist) {
    if (valid == 0xFFFFFFFFu) {
      // whole group: two multiply-adds, the word and the half, one add each
#pragma unroll
      for (int t = 0; t < 32; ++t) hist_add(W, topk_bin_bits(__uint_as_float(v[t]), R.inv, R.nlo));
    } else {
#pragma unroll
      for (int t = 0; t < 32; ++t)
        hist_add_if(W, topk_bin_bits(__uint_as_float(v[t]), R.inv, R.nlo), (valid >> t) & 1u);
    }
  } else if (R.mode == kSelRadix) {
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float s = __uint_as_float(v[t]);
      const uint32_t k = float_key(s);
      const bool member = ((valid >> t) & 1u) && topk_bin(s, R.inv, R.nlo) == R.b0 && (k & R.mask) == R.prefix;
      hist_add_if(W, (k >> R.shift) & 255u, member);
    }
  }
}

// Masks of one group in a pass that keeps ids: `up` = kept at once, `in` =
// buffered candidates (window / collect) or threshold-valued keys (exact).
__device__ __forceinline__ void topk_masks32(const TopkRow& R, const uint32_t (&v)[32], uint32_t valid, uint32_t& up,
                                             uint32_t& in) {
  up = 0u;
  in = 0u;
  if (R.mode == kSelWindow) {
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float s = __uint_as_float(v[t]);
      up |= (uint32_t)(s > R.whi) << t;
      in |= (uint32_t)(s >= R.wlo) << t;
    }
    up &= valid;
    in &= valid & ~up;
  } else if (R.mode == kSelCollect) {
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float s = __uint_as_float(v[t]);
      const int b = topk_bin(s, R.inv, R.nlo);
      const uint32_t km = float_key(s) & R.mask;
      up |= (uint32_t)(b > R.b0 || (b == R.b0 && km > R.prefix)) << t;
      in |= (uint32_t)(b == R.b0 && km == R.prefix) << t;
    }
    up &= valid;
    in &= valid;
  } else if (R.mode == kSelExact) {
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const uint32_t k = float_key(__uint_as_float(v[t]));
      up |= (uint32_t)(k > R.T) << t;
      in |= (uint32_t)(k == R.T) << t;
    }
    up &= valid;
    in &= valid;
  }
}

// The lowest `take` set bits of m.
__device__ __forceinline__ uint32_t low_bits(uint32_t m, int take) {
  uint32_t keep = 0u;
  for (int q = 0; q < take && m; ++q) {
    const uint32_t low = m & (0u - m);
    keep |= low;
    m ^= low;
  }
  return keep;
}

// Bits t of a 32-column group [x0, x0+32) with x0 + t in [xlo, xhi].
__device__ __forceinline__ uint32_t topk_valid_bits(int x0, int xlo, int xhi) {
  const int a = max(xlo - x0, 0), b = min(xhi - x0, 31);
  if (b < a) return 0u;
  const uint32_t hi = (b >= 31) ? 0xFFFFFFFFu : ((2u << b) - 1u);
  return hi & ~((1u << a) - 1u);
}

__device__ __forceinline__ void rows_barrier() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// One warp writes the list of query block i of head h: 0, the kept ids
// ascending (from the row's mask words, `wv` holding word lane + 32 b of
// batch b), i, then -1 up to kcap; and the count.
// Kept-column bit masks: for head h and query block i in row tile rt, the
// row's (rt + 1) chunks x 4 words, tiles of a head packed in order
// (tile rt starts at 512 * rt (rt + 1) / 2 words).
__host__ __device__ __forceinline__ size_t topk_mask_words_per_head(int nrt) {
  return (size_t)512 * nrt * (nrt + 1) / 2;
}
__device__ __forceinline__ uint32_t* topk_mask_row(uint32_t* masks, int nrt, int h, int i) {
  const int rt = i >> 7, r = i & 127;
  return masks + (size_t)h * topk_mask_words_per_head(nrt) + (size_t)512 * rt * (rt + 1) / 2 +
         (size_t)r * (rt + 1) * 4;
}

template <int NB>
__device__ __forceinline__ void topk_emit_row(const TopkParams& p, int h, int i, const uint32_t (&wv)[NB], int nb,
                                              int lane) {
  const int L = i > 1 ? i - 1 : 0;
  const int e = extra_budget(i, p.k_fixed, p.ppm);
  int32_t* out = p.block_idx + ((size_t)h * p.nQB + i) * p.kcap;
  int cnt;
  if (i == 0) {
    if (lane == 0) out[0] = 0;
    cnt = 1;
  } else if (L == 0 || e >= L) {
    for (int j = lane; j <= i; j += 32) out[j] = j;
    cnt = i + 1;
  } else if (e == 0) {
    if (lane == 0) {
      out[0] = 0;
      out[1] = i;
    }
    cnt = 2;
  } else {
    // each lane holds one mask word of a batch of 32; a warp prefix sum of
    // the words' counts places each lane's ids, which it writes in order
    // (no more than e of them: the check below reports a count mismatch)
    int off = 0;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= nb) break;
      uint32_t word = wv[b];
      const int c = __popc(word);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
      }
      int pos = off + incl - c;
      const int w = 32 * b + lane;
      const int jb = (w >> 2) * 128 + (w & 3) * 32;
      int32_t* dst = out + 1;
      while (word) {
        const int t = __ffs(word) - 1;
        word &= word - 1u;
        if (pos < e) dst[pos] = jb + t;
        ++pos;
      }
      off += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) {
      out[0] = 0;
      out[e + 1] = i;
      if (off != e) atomicOr(p.status, kStatusBadList);   // internal consistency check
    }
    cnt = e + 2;
  }
  for (int j = cnt + lane; j < p.kcap; j += 32) out[j] = -1;
  if (lane == 0) p.block_cnt[(size_t)h * p.nQB + i] = cnt;
}

// Warps: 0 = TMA producer (K̄), 1 = MMA issuer, 2..5 =
// first threads of the 128 rows (own the row's selection state; columns 0..63
// of each chunk), 6..9 = second threads (columns 64..127).  The statistics
// pass reads columns 0..31 (all 128 in tiles of at most 4 chunks; first
// threads); the exact fallback that keeps
// threshold-valued ids in column order reads all 128 columns (first threads).
// Warp w reads TMEM lane quarter w % 4.
template <int D>
__global__ void __launch_bounds__(320, 1)
    block_topk_kernel(const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                      const TopkParams p) {
  using Lay = TopkLayout<D>;
  extern __shared__ uint8_t tk_smem_raw[];
  if (status_timed_out(p.status)) return;
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tk_smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + Lay::kBar;
  auto bfull = [&](int s) { return bar0 + 8u * s; };
  auto bempty = [&](int s) { return bar0 + 8u * (8 + s); };
  auto sfull = [&](int b) { return bar0 + 8u * (16 + b); };
  auto sempty = [&](int b) { return bar0 + 8u * (18 + b); };
  const uint32_t qready = bar0 + 168u, done = bar0 + 176u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kCtl);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kCtl + 4);
  volatile int* tile_slot = reinterpret_cast<volatile int*>(smem + Lay::kCtl + 8);
  TopkPub& pub = *reinterpret_cast<TopkPub*>(smem + Lay::kPub);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 16; ++b) mbar_init(bar0 + 8u * b, 1);
    mbar_init(sfull(0), 1);
    mbar_init(sfull(1), 1);
    mbar_init(sempty(0), 8);
    mbar_init(sempty(1), 8);
    mbar_init(qready, 8);
    mbar_init(done, 1);
    *abort_flag = 0;
    *tile_slot = atomicAdd(p.next_tile, 1);
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
  const bool issuer = elect_one();   // the MMA warp's issuing lane (also its committer)
  constexpr uint32_t kColQh = 256, kColQl = 256 + D / 2;   // fp16 pairs per TMEM column
  constexpr int GA = 2;              // stages per group: approximate passes (a chunk's hi, NDC stages used)
  constexpr int GE = 2;              // exact passes (one d chunk's hi and lo)

  // ring bookkeeping (producer: next empty-wait parity and issued-but-unreleased
  // group starts per stage; MMA: next full-wait parity per stage)
  uint32_t eph = 0u, pend = 0u, fph = 0u;
  int spos = 0;                      // next ring stage (producer and MMA walk the same sequence)
  uint32_t chunk_ctr = 0;            // S buffer sequence (MMA and row threads)
  const RowWords W{reinterpret_cast<uint32_t*>(smem + Lay::kRow), sb + (uint32_t)Lay::kRow,
                   (warp & 3) * 32 + lane};

  // producer: make stages [s, s + G) free to overwrite
  auto claim = [&](int s, int G) -> bool {
    for (int t = s; t < s + G; ++t) {
      if ((pend >> t) & 1u) {
        if (!mbar_wait_warp(bempty(t), (eph >> t) & 1u, ab)) return false;
        eph ^= 1u << t;
        pend &= ~(1u << t);
      }
    }
    return true;
  };

  int tcount = 0;
  for (int tile = *tile_slot; tile < p.ntiles && !*abort_flag; tile = *tile_slot, ++tcount) {
    const int rt = p.nrt - 1 - tile / p.nh;
    const int h = p.h0 + tile % p.nh, g = h / p.grp;
    const int nch = rt + 1;   // key chunks of 128 blocks on or before the tile's diagonal

    // -------------------------------------------------------------- row state
    const bool is_row = warp >= 2;
    const bool second = warp >= 6;            // second thread of the row
    const int lq = warp & 3;                  // TMEM lane quarter of this warp
    const int r = lq * 32 + lane;             // row of the tile
    const int i = rt * 128 + r;               // query block
    const bool valid = i < p.nQB;
    uint32_t* mrow = topk_mask_row(p.masks, p.nrt, h, valid ? i : rt * 128);
    TopkRow R;
    R.i = i;
    R.L = i > 1 ? i - 1 : 0;
    R.e = valid ? extra_budget(i, p.k_fixed, p.ppm) : 0;
    R.mode = kSelDone;
    R.nd = 0;
    R.nc = 0;
    R.eq = 0;
    const bool pending0 = valid && !(R.L == 0 || R.e == 0 || R.e >= R.L);
    if (is_row) {
      // this row's Q̄ from global memory into TMEM (fp16 pairs): the first
      // thread moves the hi half, the second the lo half; rows past the last
      // query block get zeros.  The previous tile's MMAs, which read these
      // columns, completed before its last S buffer was handed over.
      {
        const uint4* src = reinterpret_cast<const uint4*>((second ? p.qlo : p.qhi) +
                                                          (size_t)(h * p.nQB + (valid ? i : 0)) * D);
        const uint32_t tl = tmem + ((uint32_t)(lq * 32) << 16) + (second ? kColQl : kColQh);
        uint4 q4[Lay::NDC][8];   // every load in flight before the first store
#pragma unroll
        for (int dc = 0; dc < Lay::NDC; ++dc)
#pragma unroll
          for (int k = 0; k < 8; ++k) q4[dc][k] = valid ? __ldcg(src + dc * 8 + k) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int dc = 0; dc < Lay::NDC; ++dc) {
          uint32_t v[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            v[4 * k] = q4[dc][k].x;
            v[4 * k + 1] = q4[dc][k].y;
            v[4 * k + 2] = q4[dc][k].z;
            v[4 * k + 3] = q4[dc][k].w;
          }
          tmem_st32(tl + dc * 32, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qready);
      if (pending0) {
        R.mode = kSelStats;
        R.mn = __int_as_float(0x7f800000);
        R.mx = -R.mn;
        R.sum = 0.f;
        R.sq = 0.f;
        R.cnt = 0.f;
      }
    }

    // -------------------------------------------------------------- passes
    int pass = 0;
    bool more = __syncthreads_or(is_row && pending0) != 0;
    while (more) {
      const bool approx = pass < 2;
      // the statistics pass reads a sample: every 4th key chunk of long rows
      const int cstep = (pass == 0 && nch > 4) ? 4 : 1;
      if (warp == 0) {
        // ---------------------------------------------------------- K̄ producer
        bool ok = true;
        for (int c = 0; c < nch && ok && !*abort_flag; c += cstep) {
          if (approx) {
            if (!(ok = claim(spos, GA))) break;
            if (lane == 0) {
              mbar_arrive_expect_tx(bfull(spos), (uint32_t)(Lay::NDC * Lay::kTile));
              for (int dc = 0; dc < Lay::NDC; ++dc)
                tma_load_2d(sb + (spos + dc) * Lay::kTile, &tmKh, dc * 64, g * p.nQB + c * 128, bfull(spos));
            }
            pend |= 1u << spos;
            spos = (spos + GA) % Lay::kStages;
          } else {
            for (int dc = 0; dc < Lay::NDC && ok; ++dc) {
              if (!(ok = claim(spos, GE))) break;
              if (lane == 0) {
                mbar_arrive_expect_tx(bfull(spos), (uint32_t)(GE * Lay::kTile));
                tma_load_2d(sb + spos * Lay::kTile, &tmKh, dc * 64, g * p.nQB + c * 128, bfull(spos));
                tma_load_2d(sb + (spos + 1) * Lay::kTile, &tmKl, dc * 64, g * p.nQB + c * 128, bfull(spos));
              }
              pend |= 1u << spos;
              spos = (spos + GE) % Lay::kStages;
            }
          }
          __syncwarp();
        }
      } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // The whole warp walks the issue sequence (warp-uniform operands); the
        // elected lane predicates each instruction.
        const uint32_t idesc = umma_idesc_f16(128, 128);
        bool ok = true;
        if (pass == 0) {
          ok = mbar_wait_warp(qready, (uint32_t)(tcount & 1), ab);
          tc_fence_after();
        }
        for (int c = 0; c < nch && ok; c += cstep) {
          const int sbuf = (int)(chunk_ctr & 1u);
          if (chunk_ctr >= 2u && !(ok = mbar_wait_warp(sempty(sbuf), ((chunk_ctr >> 1) - 1) & 1, ab))) break;
          tc_fence_after();
          const uint32_t dS = tmem + (uint32_t)(sbuf * 128);
          if (approx) {
            if (!(ok = mbar_wait_warp(bfull(spos), (fph >> spos) & 1u, ab))) break;
            fph ^= 1u << spos;
            tc_fence_after();
            const uint64_t d0 = umma_desc_sw128(sb + spos * Lay::kTile, 16, 1024);
#pragma unroll
            for (int dc = 0; dc < Lay::NDC; ++dc) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {   // K = 16 fp16 (32 bytes, 8 TMEM columns) per MMA
                const uint64_t bo = (uint64_t)((dc * Lay::kTile + kk * 32) >> 4);
                if (issuer) umma_f16_ts(dS, tmem + kColQh + dc * 32 + kk * 8, d0 + bo, idesc, (dc | kk) ? 1u : 0u);
              }
            }
            if (issuer) umma_commit(bempty(spos));
            spos = (spos + GA) % Lay::kStages;
          } else {
            for (int dc = 0; dc < Lay::NDC; ++dc) {
              if (!(ok = mbar_wait_warp(bfull(spos), (fph >> spos) & 1u, ab))) break;
              fph ^= 1u << spos;
              tc_fence_after();
              const uint64_t dH = umma_desc_sw128(sb + spos * Lay::kTile, 16, 1024);
              const uint64_t dL = dH + (uint64_t)(Lay::kTile >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t aH = tmem + kColQh + dc * 32 + kk * 8, aL = tmem + kColQl + dc * 32 + kk * 8;
                const uint64_t ko = (uint64_t)((kk * 32) >> 4);
                if (issuer) umma_f16_ts(dS, aH, dH + ko, idesc, (dc | kk) ? 1u : 0u);
                if (issuer) umma_f16_ts(dS, aH, dL + ko, idesc, 1u);
                if (issuer) umma_f16_ts(dS, aL, dH + ko, idesc, 1u);
              }
              if (issuer) umma_commit(bempty(spos));
              spos = (spos + GE) % Lay::kStages;
            }
            if (!ok) break;
          }
          if (issuer) umma_commit(sfull(sbuf));
          __syncwarp();
          ++chunk_ctr;
        }
      } else {
        // ---------------------------------------------------------- row threads
        bool ok = true;
        const int m = R.mode;
        const bool keeps = (m == kSelWindow || m == kSelCollect || m == kSelExact);
        // column groups of 32 this thread reads in this pass
        uint32_t need;
        if (m == kSelStats) need = second ? 0u : (nch <= 4 ? 0xFu : 0x1u);
        else if (m == kSelExact) need = second ? 0u : 0xFu;
        else if (topk_hist_mode(m) || keeps) need = second ? 0xCu : 0x3u;
        else need = 0u;
        const uint32_t wneed = __reduce_or_sync(0xFFFFFFFFu, need);
        const int cbase = second ? kTopkCap : 0;
        for (int c = 0; c < nch; c += cstep) {
          const int sbuf = (int)(chunk_ctr & 1u);
          if (ok) ok = mbar_wait_warp(sfull(sbuf), (chunk_ctr >> 1) & 1, ab);
          tc_fence_after();
          // candidates of row i are key blocks 1 .. i-1
          const int jb = c * 128;
          const int xlo = (c == 0) ? 1 : 0;
          const int xhi = min(R.i - 1 - jb, 127);
          const uint32_t ta = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(sbuf * 128);
          uint32_t* mw = mrow + c * 4;
          if (ok) {
            // one group body, not unrolled: the per-mode 32-wide bodies stay
            // small enough for the instruction cache
#pragma unroll 1
            for (int gq = 0; gq < 4; ++gq) {
              if (!((wneed >> gq) & 1u)) continue;
              uint32_t v[32];
              tmem_ld32(ta + gq * 32, v);
              tmem_wait_ld();
              reg_fence(v);
              if ((need >> gq) & 1u) {
                const uint32_t vb = topk_valid_bits(gq * 32, xlo, xhi);
                if (keeps) {
                  uint32_t up, in;
                  topk_masks32(R, v, vb, up, in);
                  if (m == kSelExact) {
                    // threshold-valued ids are kept lowest id first, in column order
                    const uint32_t keq = low_bits(in, max(R.need - R.eq, 0));
                    R.eq += __popc(in);
                    up |= keq;
                  } else if (in) {
                    topk_buffer(v, in, cbase, R.nc, jb + gq * 32, W);
                    R.nc += __popc(in);
                  }
                  R.nd += __popc(up);
                  mw[gq] = up;
                } else {
                  topk_accum32(R, v, vb, W);
                }
              }
              __syncwarp();
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sempty(sbuf));
          ++chunk_ctr;
        }
        if (!ok) *abort_flag = 1;
        // ---------------------------------------------------------- end of pass
        if (second) pub.cnt2[r] = R.nd | (R.nc << 16);
        __syncwarp();
        rows_barrier();   // both threads' work of this pass is done
        if (!second && R.mode != kSelDone) {
          if (*abort_flag) R.mode = kSelDone;
          const int c2 = pub.cnt2[r];
          const int ndB = c2 & 0xFFFF, ncB = c2 >> 16;
          switch (R.mode) {
            case kSelStats: {
              float lo = R.mn, hi = R.mx;
              // rows of at most 4 chunks were read whole: their window is the
              // row's range (a few scores per bin); longer rows were sampled
              if (nch > 4 && R.cnt > 0.f && R.sum == R.sum && R.mn <= R.mx) {
                // the sample's mean and spread place the window: from one
                // spread below the estimated e-th largest score (a normal
                // model of the row) to six spreads above the mean
                const float mu = R.sum / R.cnt;
                const float sd = sqrtf(fmaxf(R.sq / R.cnt - mu * mu, 0.f));
                const float z = normal_upper_quantile((float)R.e / (float)R.L);
                lo = fmaxf(R.mn, mu + fmaxf(z - 1.f, -3.f) * sd);
                hi = fminf(R.mx, mu + 6.f * sd);
                if (!(hi > lo)) {
                  lo = R.mn;
                  hi = R.mx;
                }
              }
              float inv = (hi > lo) ? 1.f / (hi - lo) : 0.f;
              if (!(inv <= 3.0e38f)) inv = 0.f;
              R.inv = inv;
              R.nlo = (inv > 0.f) ? -lo * inv : 0.f;
              hist_clear(W);
              R.mode = kSelAHist;
            } break;
            case kSelAHist: {
              int bin, above, cnt;
              hist_find(W, R.e, bin, above, cnt);
              const float kInf = __int_as_float(0x7f800000);
              if (R.inv > 0.f) {
                // bin b holds y in [(b - 1/2) / 255, (b + 1/2) / 255): the exact
                // window reaches a quarter bin further on each side
                const float lo = -R.nlo / R.inv, w = 1.f / (255.f * R.inv);
                R.wlo = (bin == 0) ? -kInf : lo + ((float)bin - 0.75f) * w;
                R.whi = (bin == 255) ? kInf : lo + ((float)bin + 0.75f) * w;
              } else {
                R.wlo = -kInf;
                R.whi = kInf;
              }
              R.mode = kSelWindow;
            } break;
            case kSelWindow: {
              const int nd = R.nd + ndB;
              if (nd <= R.e && R.e <= nd + R.nc + ncB && R.nc <= kTopkCap && ncB <= kTopkCap) {
                topk_resolve(W, R.nc, ncB, R.e - nd, mrow);
                R.mode = kSelDone;
              } else {
                hist_clear(W);
                R.mode = kSelHist;
              }
            } break;
            case kSelHist: {
              int bin, above, cnt;
              hist_find(W, R.e, bin, above, cnt);
              R.b0 = bin;
              R.rem = R.e - above;
              R.prefix = 0u;
              R.mask = 0u;
              R.shift = 24;
              if (cnt <= kTopkCap) {   // fits one thread's buffer even if all in its columns
                R.mode = kSelCollect;
              } else {
                hist_clear(W);
                R.mode = kSelRadix;
              }
            } break;
            case kSelRadix: {
              int bin, above, cnt;
              hist_find(W, R.rem, bin, above, cnt);
              R.rem -= above;
              R.prefix |= (uint32_t)bin << R.shift;
              R.mask |= 255u << R.shift;
              R.shift -= 8;
              if (R.mask == 0xFFFFFFFFu) {
                R.T = R.prefix;
                R.need = R.rem;
                R.mode = kSelExact;
              } else if (cnt <= kTopkCap) {
                R.mode = kSelCollect;
              } else {
                hist_clear(W);
              }
            } break;
            case kSelCollect: {
              topk_resolve(W, min(R.nc, kTopkCap), min(ncB, kTopkCap), R.rem, mrow);
              R.mode = kSelDone;
            } break;
            case kSelExact: {
              R.mode = kSelDone;
            } break;
            default:
              break;
          }
          pub.mode[r] = R.mode;
          pub.inv[r] = R.inv;
          pub.nlo[r] = R.nlo;
          pub.wlo[r] = R.wlo;
          pub.whi[r] = R.whi;
          pub.b0[r] = R.b0;
          pub.prefix[r] = R.prefix;
          pub.mask[r] = R.mask;
          pub.shift[r] = R.shift;
        } else if (!second) {
          pub.mode[r] = kSelDone;
        }
        R.nd = 0;
        R.nc = 0;
        R.eq = 0;
        __syncwarp();
        rows_barrier();   // the first threads' transitions (and histogram clears) are done
        if (second) {
          R.mode = pub.mode[r];
          R.inv = pub.inv[r];
          R.nlo = pub.nlo[r];
          R.wlo = pub.wlo[r];
          R.whi = pub.whi[r];
          R.b0 = pub.b0[r];
          R.prefix = pub.prefix[r];
          R.mask = pub.mask[r];
          R.shift = pub.shift[r];
        }
      }
      ++pass;
      // passes 0, 1 and 2 always follow each other (every pending row goes
      // through all three), so the pipeline runs across them without a barrier
      if (pass >= 3) {
        const bool pending = is_row && !second && R.mode != kSelDone && !*abort_flag;
        more = __syncthreads_or(pending) != 0;
      }
      if (more && pass >= kTopkMaxPasses) {
        if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
        *abort_flag = 1;
        more = false;
      }
    }

    // the lists are written from the masks by block_list_kernel
    if (threadIdx.x == 0) *tile_slot = atomicAdd(p.next_tile, 1);
    __syncthreads();   // the per-row region and the ring may take the next tile
  }

  // ---------------------------------------------------------------- clean-up
  if (warp == 0 && lane == 0) {
    for (int t = 0; t < Lay::kStages; ++t)
      if ((pend >> t) & 1u) mbar_wait_cleanup(bempty(t), (eph >> t) & 1u, 200000000ull);
  }
  if (warp == 1) {
    if (issuer) umma_commit(done);
    __syncwarp();
    mbar_wait_cleanup(done, 0, 200000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Writes the block lists from the masks of block_topk_kernel: each warp takes
// (head, query block) rows in a grid-stride loop, loading the next row's mask
// words while it writes the current one.  NB is
// the number of 32-word mask batches a row can have (rows of row tile rt have
// 4 (rt + 1) words), so short rows keep few registers and many warps resident.
template <int NB>
__global__ void __launch_bounds__(256) block_list_kernel(const TopkParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrows = p.Hq * p.nQB;   // below 2^31 (checked by the host)
  const int step = (int)gridDim.x * 8;
  // row = h * nQB + i, advanced by step without a division per row
  const int dh = step / p.nQB, di = step % p.nQB;
  int row = (int)blockIdx.x * 8 + warp;
  if (row >= nrows) return;
  int h = row / p.nQB, i = row % p.nQB;
  auto load = [&](int hh, int ii, uint32_t (&wv)[NB], int& nb) {
    const int nwords = ((ii >> 7) + 1) * 4;
    nb = (nwords + 31) / 32;
    const uint32_t* mr = topk_mask_row(p.masks, p.nrt, hh, ii);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int w = 32 * b + lane;
      wv[b] = (b < nb && w < nwords) ? __ldcg(mr + w) : 0u;
    }
  };
  uint32_t cur[NB], nxt[NB];
  int nbc = 0, nbn = 0;
  load(h, i, cur, nbc);
  for (; row < nrows; row += step) {
    int hn = h + dh, in = i + di;
    if (in >= p.nQB) {
      in -= p.nQB;
      ++hn;
    }
    if (row + step < nrows) load(hn, in, nxt, nbn);
    topk_emit_row<NB>(p, h, i, cur, nbc, lane);
#pragma unroll
    for (int b = 0; b < NB; ++b) cur[b] = nxt[b];
    nbc = nbn;
    h = hn;
    i = in;
  }
}

}  // namespace dsa
