// select.cuh -- block-wide top-k by radix select with ties toward the lower
// index, and ordered compaction of the kept positions.
//
// The problem statement fixes the rule: keep the e highest-scoring candidates,
// equal scores going to the lower index, and return the kept ids in ascending
// order together with the ids that are always kept (sink / diagonal / first
// columns / last block).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace dsa {

struct SelectSmem {
  uint32_t hist[256];
  int warp_sums[32];
  uint32_t bcast[4];
};

// Exclusive prefix sum of one int per thread over the whole block (NT threads,
// a multiple of 32). Also returns the block total.  Contains __syncthreads.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, SelectSmem& sm, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sm.warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < NT / 32) ? sm.warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < NT / 32) sm.warp_sums[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) sm.bcast[3] = (uint32_t)wi;
  }
  __syncthreads();
  int res = sm.warp_sums[warp] + incl - v;
  total = (int)sm.bcast[3];
  __syncthreads();
  return res;
}

// Radix select over keys float_key(src[0..L)): finds the key T of the e-th
// largest element (1 <= e < L) and how many elements equal to T are kept
// (`need`, the lowest-index ones).  Four passes of 8 bits.
template <int NT>
__device__ __forceinline__ void radix_select(const float* src, int L, int e, SelectSmem& sm, uint32_t& T,
                                             int& need) {
  uint32_t prefix = 0, mask = 0;
  int rem = e;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += NT) sm.hist[b] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < L; j += NT) {
      uint32_t k = float_key(src[j]);
      if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8];
      uint32_t s = 0;
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        c[a] = sm.hist[255 - 8 * lane - a];
        s += c[a];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
      }
      const uint32_t excl = incl - s;
      if (excl < (uint32_t)rem && (uint32_t)rem <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          if (cum + c[a] >= (uint32_t)rem) {
            sm.bcast[0] = (uint32_t)(255 - 8 * lane - a);
            sm.bcast[1] = (uint32_t)rem - cum;
            break;
          }
          cum += c[a];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = sm.bcast[0];
    rem = (int)sm.bcast[1];
    prefix |= bin << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  T = prefix;
  need = rem;
}

// Top-e of the candidates src[0..L) placed at positions [c0, c0+L) of an id
// range [0, P); positions outside the candidate range are always kept.  Writes
// the kept ids in ascending order to out[0..cnt) and -1 to out[cnt..cap).
// Returns cnt (the same value in every thread).
template <int NT>
__device__ int topk_ascending(const float* src, int L, int e, int c0, int P, int32_t* out, int cap,
                              SelectSmem& sm) {
  e = e < 0 ? 0 : (e > L ? L : e);
  uint32_t T = 0;
  int need = 0;
  const bool all = (e >= L), none = (e == 0);
  if (!all && !none) radix_select<NT>(src, L, e, sm, T, need);
  // Per-thread contiguous chunk of positions.
  const int per = (P + NT - 1) / NT;
  const int p0 = min(P, (int)threadIdx.x * per), p1 = min(P, p0 + per);
  int eq_before = 0;
  if (!all && !none) {
    int eq = 0;
    for (int p = p0; p < p1; ++p) {
      int c = p - c0;
      if (c >= 0 && c < L && float_key(src[c]) == T) ++eq;
    }
    int tot;
    eq_before = block_excl_scan<NT>(eq, sm, tot);
  }
  // Count kept positions in the chunk.
  int kept = 0;
  {
    int eb = eq_before;
    for (int p = p0; p < p1; ++p) {
      int c = p - c0;
      bool k;
      if (c < 0 || c >= L) k = true;
      else if (all) k = true;
      else if (none) k = false;
      else {
        uint32_t key = float_key(src[c]);
        if (key > T) k = true;
        else if (key == T) k = (eb++ < need);
        else k = false;
      }
      kept += k;
    }
  }
  int total;
  int off = block_excl_scan<NT>(kept, sm, total);
  {
    int eb = eq_before;
    for (int p = p0; p < p1; ++p) {
      int c = p - c0;
      bool k;
      if (c < 0 || c >= L) k = true;
      else if (all) k = true;
      else if (none) k = false;
      else {
        uint32_t key = float_key(src[c]);
        if (key > T) k = true;
        else if (key == T) k = (eb++ < need);
        else k = false;
      }
      if (k) {
        if (off < cap) out[off] = p;
        ++off;
      }
    }
  }
  for (int j = total + (int)threadIdx.x; j < cap; j += NT) out[j] = -1;
  return total;
}

}  // namespace dsa
