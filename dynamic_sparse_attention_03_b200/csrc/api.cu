// api.cu -- host side of the C ABI declared in include/dsa.h: argument checks,
// workspace layout, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "ashape.cuh"
#include "attn_fwd.cuh"
#include "clusters.cuh"
#include "block_topk.cuh"
#include "decode.cuh"
#include "index_kernels.cuh"
#include "vs_kernels.cuh"

using namespace dsa;

namespace {

constexpr size_t kStatusBytes = 256;
constexpr int kMaxN = 1 << 21;
constexpr int kTopkMaxGrid = 1024;   // persistent top-k grid: one CTA per SM, at most this many

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct WsCarve {
  uint8_t* base;
  size_t off = 0;
  explicit WsCarve(void* b) : base(static_cast<uint8_t*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off = align256(off + bytes);
    return p;
  }
};

int cuda_err(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }


int launch_check() { return cuda_err(cudaGetLastError()); }

// Dynamic shared memory above 48 KB needs an opt-in per kernel.
template <typename K>
int set_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return DSA_OK;
  return cuda_err(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2D bf16 view [rows][d] with a 64 x 64 box and 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, int64_t rows, int d) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2D fp16 view [rows][d] with a 64-element (128-byte) x box_rows box and 128-byte swizzle.
bool make_tmap_f16(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2D bf16 view [rows][d] with a 64-element (128-byte) x box_rows box and 128-byte swizzle.
bool make_tmap_rows(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool validate_env() {
  const char* v = std::getenv("DSA_VALIDATE");
  return v && v[0] == '1';
}

// Fault injection for the tests of the bounded waits: with
// DSA_FAULT_INJECT=attn_stall, block_sparse_attn_fwd's first work item issues
// no load for its first K tile and the waits give up after 1 ms, so the call
// ends with DSA_ERR_TIMEOUT in the status word and nothing in flight.
bool stall_injection() {
  const char* v = std::getenv("DSA_FAULT_INJECT");
  return v && std::strcmp(v, "attn_stall") == 0;
}

int max_count(int nQB, int k_fixed, int64_t ppm) {
  int best = 0;
  for (int i = 0; i < nQB; ++i) {
    const int c = (i == 0 ? 1 : 2) + extra_budget(i, k_fixed, ppm);
    best = c > best ? c : best;
  }
  return best;
}

// Device-side list check for block_sparse_attn_fwd in validation mode.
__global__ void validate_lists_kernel(const int32_t* bidx, const int32_t* bcnt, int kcap, const int32_t* cidx,
                                      const int32_t* ccnt, int ccap, int nQB, int Hq, uint32_t* status) {
  const int qb = blockIdx.x, h = blockIdx.y;
  if (threadIdx.x != 0) return;
  const size_t row = (size_t)h * nQB + qb;
  const int nb = bcnt[row];
  bool bad = nb < 0 || nb > kcap;
  const int32_t* b = bidx + row * kcap;
  for (int x = 0; !bad && x < nb; ++x) {
    if (b[x] < 0 || b[x] > qb) bad = true;
    if (x > 0 && b[x] <= b[x - 1]) bad = true;
  }
  if (!bad && cidx) {
    const int nc = ccnt[row];
    if (nc < 0 || nc > ccap) bad = true;
    const int32_t* c = cidx + row * ccap;
    int y = 0;
    for (int x = 0; !bad && x < nc; ++x) {
      const int j = c[x];
      if (j < 0 || j >= 64 * qb) bad = true;
      if (x > 0 && j <= c[x - 1]) bad = true;
      while (y < nb && b[y] < (j >> 6)) ++y;
      if (y < nb && b[y] == (j >> 6)) bad = true;
    }
  }
  if (bad) atomicOr(status, kStatusBadList);
}

template <int D>
int launch_attn(const void* q, const void* k, const void* v, void* o, int Hq, int Hkv, int n, float scale,
                const int32_t* bidx, const int32_t* bcnt, int kcap, const int32_t* cidx, const int32_t* ccnt,
                int ccap, float* lse, uint32_t* status, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, (int64_t)Hq * n, D) || !make_tmap(&tk, k, (int64_t)Hkv * n, D) ||
      !make_tmap(&tv, v, (int64_t)Hkv * n, D))
    return DSA_ERR_CUDA;
  AttnParams p{};
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.block_idx = bidx;
  p.block_cnt = bcnt;
  p.col_idx = cidx;
  p.col_cnt = ccnt;
  p.status = status;
  p.kcap = kcap;
  p.ccap = ccap;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n = n;
  p.nQB = n / 64;
  p.grp = Hq / Hkv;
  p.nquads = (p.grp + 3) / 4;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = kWaitLimitNs;
  p.stall_item = -1;
  if (stall_injection()) {   // test hook: one K load is skipped, its wait runs out after 1 ms
    p.wait_ns = 1000000ull;
    p.stall_item = 0;
  }
  const size_t smem = AttnLayout<D>::kSmemAlloc;
  int rc = set_smem(bsa_fwd_kernel<D>, smem);
  if (rc) return rc;
  const int64_t grid = (int64_t)Hkv * p.nquads * p.nQB;
  bsa_fwd_kernel<D><<<(unsigned)grid, 384, smem, st>>>(tq, tk, tv, p);
  return launch_check();
}

template <int D, int G>
int launch_decode(const DecodeParams& p, int B, int Hkv, int nchmax, size_t sel_smem, cudaStream_t st) {
  int rc;
  decode_score_kernel<D, G><<<dim3(B * Hkv, (p.nb + 63) / 64), 256, 0, st>>>(p);
  if ((rc = launch_check())) return rc;
  if ((rc = set_smem(decode_topk_kernel<256>, sel_smem))) return rc;
  decode_topk_kernel<256><<<B * Hkv * G, 256, sel_smem, st>>>(p);
  if ((rc = launch_check())) return rc;
  decode_union_kernel<G, 256><<<B * Hkv, 256, 0, st>>>(p);
  if ((rc = launch_check())) return rc;
  if ((rc = set_smem(decode_attn_kernel<D, G>, DecLayout<D>::kBytes))) return rc;
  decode_attn_kernel<D, G><<<dim3(B * Hkv, nchmax), kDecThreads, DecLayout<D>::kBytes, st>>>(p);
  return launch_check();
}

template <int D, int G>
int launch_cluster_decode(const ClusterParams& cp, int B, int Hkv, int nchmax, size_t sel_smem, cudaStream_t st) {
  int rc;
  // q.c for every cluster, 64 centroids of one (batch, KV head) per CTA
  DecodeParams sp = cp.dp;
  sp.cent = cp.cent;
  sp.nb = cp.C;
  sp.scores = const_cast<float*>(cp.scores);
  decode_score_kernel<D, G><<<dim3(B * Hkv, (cp.C + 63) / 64), 256, 0, st>>>(sp);
  if ((rc = launch_check())) return rc;
  if ((rc = set_smem(cluster_topk_kernel<256>, sel_smem))) return rc;
  cluster_topk_kernel<256><<<B * Hkv * G, 256, sel_smem, st>>>(cp);
  if ((rc = launch_check())) return rc;
  const size_t uni_smem = (size_t)(cp.C + 1) * 4 + (size_t)cp.C * 5;
  if ((rc = set_smem(cluster_union_kernel<G, 1024>, uni_smem))) return rc;
  cluster_union_kernel<G, 1024><<<B * Hkv, 1024, uni_smem, st>>>(cp);
  if ((rc = launch_check())) return rc;
  if (cp.dp.n_packed > 0) {
    if ((rc = set_smem(cluster_stream_attn_kernel<D, G>, ClStreamLayout<D>::kBytes))) return rc;
    cluster_stream_attn_kernel<D, G>
        <<<dim3(B * Hkv, nchmax), (kClWarps + 1) * 32, ClStreamLayout<D>::kBytes, st>>>(cp.dp);
  } else {
    cluster_attn_kernel<D, G><<<dim3(B * Hkv, nchmax), 128, 0, st>>>(cp.dp);
  }
  return launch_check();
}

}  // namespace

extern "C" {

const char* dsa_version(void) { return "dsa 0.1 sm_100a"; }

int dsa_block_index_capacity(int n, int block, int k_fixed, float keep_ratio) {
  if (n <= 0) return DSA_ERR_INVALID_ARG;
  if (block != 64 || n % 64 != 0 || n > kMaxN) return DSA_ERR_UNSUPPORTED;
  const bool fixed = k_fixed > 0, ratio = keep_ratio > 0.f;
  if (fixed == ratio || !(keep_ratio == keep_ratio) || keep_ratio > 1.0f) return DSA_ERR_INVALID_ARG;
  const int64_t ppm = ratio ? (int64_t)std::floor((double)keep_ratio * 1e6 + 0.5) : 0;
  return max_count(n / 64, fixed ? k_fixed : 0, ppm);
}

int dsa_get_status(const void* ws, dsa_stream_t stream) {
  if (!ws) return DSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof(word), st) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  if (word & kStatusTimeout) return DSA_ERR_TIMEOUT;
  if (word & kStatusBadList) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

int sparse_index_estimate(const void* q, const void* k, int Hq, int Hkv, int n, int d, int block, int k_fixed,
                          float keep_ratio, int32_t* block_idx, int32_t* block_cnt, int kcap, float* pooled_k,
                          void* ws, size_t* ws_bytes, dsa_stream_t stream) {
  if (!k || !ws_bytes || Hkv <= 0 || n <= 0) return DSA_ERR_INVALID_ARG;
  if (block != 64 || (d != 64 && d != 128) || n % 64 != 0 || n > kMaxN) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)Hkv * n >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(k) || (q && !aligned16(q))) return DSA_ERR_INVALID_ARG;
  const int nQB = n / 64;
  const bool pool_only = (q == nullptr);
  int64_t ppm = 0;
  if (pool_only) {
    if (!pooled_k) return DSA_ERR_INVALID_ARG;
  } else {
    if (Hq <= 0 || Hq % Hkv != 0 || !block_idx || !block_cnt || kcap <= 0) return DSA_ERR_INVALID_ARG;
    if ((int64_t)Hq * n >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
    const bool fixed = k_fixed > 0, ratio = keep_ratio > 0.f;
    if (fixed == ratio || !(keep_ratio == keep_ratio) || keep_ratio > 1.0f) return DSA_ERR_INVALID_ARG;
    if (ratio) ppm = (int64_t)std::floor((double)keep_ratio * 1e6 + 0.5);
    if (max_count(nQB, fixed ? k_fixed : 0, ppm) > kcap) return DSA_ERR_CAPACITY;
  }
  WsCarve c(ws);
  uint32_t* status = static_cast<uint32_t*>(c.take(kStatusBytes));
  // FP16 hi/lo halves of the scaled pooled means, the operands of the
  // tensor-core scores (scales: per query block for Q, per KV head for K)
  __half* q_hi = pool_only ? nullptr : static_cast<__half*>(c.take((size_t)Hq * nQB * d * 2));
  __half* q_lo = pool_only ? nullptr : static_cast<__half*>(c.take((size_t)Hq * nQB * d * 2));
  __half* k_hi = pool_only ? nullptr : static_cast<__half*>(c.take((size_t)Hkv * nQB * d * 2));
  __half* k_lo = pool_only ? nullptr : static_cast<__half*>(c.take((size_t)Hkv * nQB * d * 2));
  float* kbar = pooled_k;
  if (!pool_only && !kbar) kbar = static_cast<float*>(c.take((size_t)Hkv * nQB * d * 4));
  // per KV head max |K̄| (float bits) and the top-k tile counter, zeroed together
  unsigned* kmax = pool_only ? nullptr : static_cast<unsigned*>(c.take((size_t)(Hkv + 1) * 4));
  // kept-column bit masks written by the fused score/top-k kernel and read by
  // the list kernel: 16 bytes per (head, query block, key chunk of its tile)
  const int nrt = (nQB + 127) / 128;
  uint32_t* masks = pool_only ? nullptr
                              : static_cast<uint32_t*>(c.take((size_t)Hq * topk_mask_words_per_head(nrt) * 4));
  int* next_tile = pool_only ? nullptr : reinterpret_cast<int*>(kmax + Hkv);
  if (!ws) {
    *ws_bytes = c.off;
    return DSA_OK;
  }
  if (*ws_bytes < c.off) return DSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const int64_t nkb = (int64_t)Hkv * nQB, nqb = (int64_t)Hq * nQB;
  if (!pool_only && cudaMemsetAsync(kmax, 0, (size_t)(Hkv + 1) * 4, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (d == 128)
    pool_blocks_kernel<128><<<(unsigned)nkb, 256, 0, st>>>(kb, kbar, nkb, kmax, nQB, nullptr, nullptr, nullptr, 0,
                                                           nullptr, nullptr, nullptr);
  else
    pool_blocks_kernel<64><<<(unsigned)nkb, 256, 0, st>>>(kb, kbar, nkb, kmax, nQB, nullptr, nullptr, nullptr, 0,
                                                          nullptr, nullptr, nullptr);
  if (int rc = launch_check()) return rc;
  if (pool_only) return DSA_OK;
  const auto* qp = static_cast<const __nv_bfloat16*>(q);
  CUtensorMap tkh, tkl;
  if (!make_tmap_f16(&tkh, k_hi, nkb, d, 128) || !make_tmap_f16(&tkl, k_lo, nkb, d, 128)) return DSA_ERR_CUDA;
  TopkParams tp{};
  tp.block_idx = block_idx;
  tp.block_cnt = block_cnt;
  tp.status = status;
  tp.nQB = nQB;
  tp.Hq = Hq;
  tp.grp = Hq / Hkv;
  tp.kcap = kcap;
  tp.k_fixed = k_fixed > 0 ? k_fixed : 0;
  tp.nrt = nrt;
  tp.masks = masks;
  tp.ppm = ppm;
  tp.qhi = q_hi;
  tp.qlo = q_lo;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return DSA_ERR_CUDA;
  int rc;
  if ((rc = (d == 128) ? set_smem(block_topk_kernel<128>, TopkLayout<128>::kSmemAlloc)
                       : set_smem(block_topk_kernel<64>, TopkLayout<64>::kSmemAlloc)))
    return rc;
  // Q pooling (split with each query block's own scale), then 8 pooled-key
  // rows per extra CTA split with their KV head's scale
  const unsigned qgrid = (unsigned)(nqb + (nkb + 7) / 8);
  if (d == 128)
    pool_blocks_kernel<128><<<qgrid, 256, 0, st>>>(qp, nullptr, nqb, nullptr, nQB, q_hi, q_lo, kbar, nkb, kmax,
                                                   k_hi, k_lo);
  else
    pool_blocks_kernel<64><<<qgrid, 256, 0, st>>>(qp, nullptr, nqb, nullptr, nQB, q_hi, q_lo, kbar, nkb, kmax,
                                                  k_hi, k_lo);
  if ((rc = launch_check())) return rc;
  // pooled scores and the per-row top-k in one kernel (the scores stay on chip)
  tp.h0 = 0;
  tp.nh = Hq;
  tp.ntiles = nrt * Hq;
  tp.next_tile = next_tile;
  const unsigned grid = (unsigned)std::min(std::min(nsm, kTopkMaxGrid), tp.ntiles);
  if (d == 128) block_topk_kernel<128><<<grid, 320, TopkLayout<128>::kSmemAlloc, st>>>(tkh, tkl, tp);
  else block_topk_kernel<64><<<grid, 320, TopkLayout<64>::kSmemAlloc, st>>>(tkh, tkl, tp);
  if ((rc = launch_check())) return rc;
  const int64_t nrows = (int64_t)Hq * nQB;
  // rows of the last row tile have 4 nrt mask words: 32-word batches
  const int nbmax = (4 * nrt + 31) / 32;
  const int64_t list_ctas = std::min<int64_t>((nrows + 7) / 8, (int64_t)nsm * 8);
  if (nbmax <= 2) block_list_kernel<2><<<(unsigned)list_ctas, 256, 0, st>>>(tp);
  else if (nbmax <= 8) block_list_kernel<8><<<(unsigned)list_ctas, 256, 0, st>>>(tp);
  else block_list_kernel<32><<<(unsigned)list_ctas, 256, 0, st>>>(tp);
  if ((rc = launch_check())) return rc;
  return DSA_OK;
}

int vertical_slash_index(const void* q, const void* k, int Hq, int Hkv, int n, int d, int last_q, int n_vert,
                         int n_slash, float scale, int32_t* vert_idx, int32_t* slash_off, int32_t* block_idx,
                         int32_t* block_cnt, int kcap, int32_t* col_idx, int32_t* col_cnt, int ccap, void* ws,
                         size_t* ws_bytes, dsa_stream_t stream) {
  if (!q || !k || !ws_bytes || !block_idx || !block_cnt || !col_idx || !col_cnt) return DSA_ERR_INVALID_ARG;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n < 64) return DSA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || n % 64 != 0 || last_q != 64 || n > kMaxN) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)Hq * n >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (n_vert < 64 || n_vert > n || n_slash < 1 || n_slash > n) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !aligned16(q) || !aligned16(k)) return DSA_ERR_INVALID_ARG;
  const int nQB = n / 64;
  if (kcap < std::min(nQB, 2 * n_slash) || ccap < n_vert) return DSA_ERR_CAPACITY;
  const int ntiles = (n + kVSTile - 1) / kVSTile;
  WsCarve c(ws);
  VSParams p{};
  p.status = static_cast<uint32_t*>(c.take(kStatusBytes));
  p.part = static_cast<float*>(c.take((size_t)Hq * ntiles * 64 * 2 * 4));
  p.lse2 = static_cast<float*>(c.take((size_t)Hq * 64 * 4));
  p.vert = static_cast<float*>(c.take((size_t)Hq * n * 4));
  p.slash_part = static_cast<float*>(c.take((size_t)Hq * ntiles * kVSDiag * 4));
  p.slash = static_cast<float*>(c.take((size_t)Hq * n * 4));
  p.vsel = vert_idx ? vert_idx : static_cast<int32_t*>(c.take((size_t)Hq * n_vert * 4));
  p.ssel = slash_off ? slash_off : static_cast<int32_t*>(c.take((size_t)Hq * n_slash * 4));
  // slice survivors: at most min(e, slice length) per slice and kind
  const int ecap = std::max(1, std::min(std::max(n_vert - 64, n_slash - 1), (n + kVSParts - 1) / kVSParts));
  p.cand_id = static_cast<int32_t*>(c.take((size_t)Hq * 2 * kVSParts * ecap * 4));
  p.cand_cnt = static_cast<int32_t*>(c.take((size_t)Hq * 2 * kVSParts * 4));
  p.cand_val = static_cast<float*>(c.take((size_t)Hq * 2 * kVSParts * ecap * 4));
  p.cand_gid = static_cast<int32_t*>(c.take((size_t)Hq * 2 * kVSParts * ecap * 4));
  p.ecap = ecap;
  p.dbits = static_cast<uint32_t*>(c.take((size_t)Hq * ((nQB + 31) / 32) * 4));
  p.dlist = static_cast<int32_t*>(c.take((size_t)Hq * nQB * 4));
  p.dcount = static_cast<int32_t*>(c.take((size_t)Hq * 4));
  if (!ws) {
    *ws_bytes = c.off;
    return DSA_OK;
  }
  if (*ws_bytes < c.off) return DSA_ERR_INVALID_ARG;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.block_idx = block_idx;
  p.block_cnt = block_cnt;
  p.col_idx = col_idx;
  p.col_cnt = col_cnt;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n = n;
  p.nQB = nQB;
  p.grp = Hq / Hkv;
  p.ntiles = ntiles;
  p.n_vert = n_vert;
  p.n_slash = n_slash;
  p.kcap = kcap;
  p.ccap = ccap;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc;
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, q, (int64_t)Hq * n, d) || !make_tmap(&tk, k, (int64_t)Hkv * n, d)) return DSA_ERR_CUDA;
  const dim3 gl(ntiles, Hkv * ((p.grp + 3) / 4));
  // pass 1 (row maxima and sums per key tile), the rows' log-sum-exp, pass 2
  // (column sums and diagonal partials); the logits are computed in both passes
  if (d == 128) {
    if ((rc = set_smem(vs_score_kernel<128, 1>, VSScoreLayout<128>::kSmemAlloc)) ||
        (rc = set_smem(vs_score_kernel<128, 2>, VSScoreLayout<128>::kSmemAlloc)))
      return rc;
    vs_score_kernel<128, 1><<<gl, 256, VSScoreLayout<128>::kSmemAlloc, st>>>(tq, tk, p);
  } else {
    if ((rc = set_smem(vs_score_kernel<64, 1>, VSScoreLayout<64>::kSmemAlloc)) ||
        (rc = set_smem(vs_score_kernel<64, 2>, VSScoreLayout<64>::kSmemAlloc)))
      return rc;
    vs_score_kernel<64, 1><<<gl, 256, VSScoreLayout<64>::kSmemAlloc, st>>>(tq, tk, p);
  }
  if ((rc = launch_check())) return rc;
  vs_lse_kernel<<<Hq * 64, 128, 0, st>>>(p);
  if ((rc = launch_check())) return rc;
  if (d == 128) vs_score_kernel<128, 2><<<gl, 256, VSScoreLayout<128>::kSmemAlloc, st>>>(tq, tk, p);
  else vs_score_kernel<64, 2><<<gl, 256, VSScoreLayout<64>::kSmemAlloc, st>>>(tq, tk, p);
  if ((rc = launch_check())) return rc;
  vs_slash_kernel<<<dim3((n + 255) / 256, Hq), 256, 0, st>>>(p);
  if ((rc = launch_check())) return rc;
  vs_topk_part_kernel<256><<<dim3(Hq, 2, kVSParts), 256, 0, st>>>(p);
  if ((rc = launch_check())) return rc;
  vs_topk_kernel<1024><<<dim3(Hq, 2), 1024, 0, st>>>(p);
  if ((rc = launch_check())) return rc;
  const size_t dist_smem = (size_t)((nQB + 31) / 32) * 4;
  if ((rc = set_smem(vs_dist_kernel<256>, dist_smem))) return rc;
  vs_dist_kernel<256><<<Hq, 256, dist_smem, st>>>(p);
  if ((rc = launch_check())) return rc;
  vs_plan_kernel<<<(unsigned)(((int64_t)Hq * nQB + 7) / 8), 256, 0, st>>>(p);
  return launch_check();
}

int block_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, int Hq, int Hkv, int n, int d,
                          float scale, const int32_t* block_idx, const int32_t* block_cnt, int kcap,
                          const int32_t* col_idx, const int32_t* col_cnt, int ccap, float* lse, void* ws,
                          size_t* ws_bytes, dsa_stream_t stream) {
  if (!q || !k || !v || !o || !block_idx || !block_cnt || !ws_bytes) return DSA_ERR_INVALID_ARG;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n <= 0 || kcap <= 0) return DSA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || n % 64 != 0 || n > kMaxN) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)Hq * n >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (col_idx && (!col_cnt || ccap <= 0)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!ws) {
    *ws_bytes = kStatusBytes;
    return DSA_OK;
  }
  if (*ws_bytes < kStatusBytes) return DSA_ERR_INVALID_ARG;
  uint32_t* status = static_cast<uint32_t*>(ws);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int nQB = n / 64;
  if (validate_env()) {
    validate_lists_kernel<<<dim3(nQB, Hq), 32, 0, st>>>(block_idx, block_cnt, kcap, col_idx, col_cnt, ccap, nQB,
                                                        Hq, status);
    if (int rc = launch_check()) return rc;
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, status, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (word & kStatusBadList) {
      cudaMemsetAsync(status, 0, 4, st);
      cudaStreamSynchronize(st);
      return DSA_ERR_INVALID_ARG;
    }
  }
  if (d == 128)
    return launch_attn<128>(q, k, v, o, Hq, Hkv, n, scale, block_idx, block_cnt, kcap, col_idx, col_cnt, ccap, lse,
                            status, st);
  return launch_attn<64>(q, k, v, o, Hq, Hkv, n, scale, block_idx, block_cnt, kcap, col_idx, col_cnt, ccap, lse,
                         status, st);
}

int a_shape_index(int Hq, int n, int n_sink, int n_local, int32_t* block_idx, int32_t* block_cnt, int kcap,
                  dsa_stream_t stream) {
  if (!block_idx || !block_cnt || Hq <= 0 || n <= 0 || n_sink < 0 || n_local < 1) return DSA_ERR_INVALID_ARG;
  if (n % 64 != 0 || n > kMaxN) return DSA_ERR_UNSUPPORTED;
  const int nQB = n / 64;
  const int need = std::min(nQB, n_sink + n_local);
  if (kcap < need) return DSA_ERR_CAPACITY;
  const int nrows = Hq * nQB;
  a_shape_kernel<<<(nrows + 7) / 8, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(nrows, nQB, n_sink, n_local,
                                                                                     block_idx, block_cnt, kcap);
  return launch_check();
}

int sparse_decode_attn(const void* q, const void* k_cache, const void* v_cache, const float* centroids, int B,
                       int Hq, int Hkv, int S, int d, int keep, int force_last, float scale, void* o,
                       int32_t* sel_idx, int32_t* sel_cnt, int kcap, void* ws, size_t* ws_bytes,
                       dsa_stream_t stream) {
  if (!q || !k_cache || !v_cache || !centroids || !o || !ws_bytes) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S < 64 || keep < 0) return DSA_ERR_INVALID_ARG;
  if (force_last != 0 && force_last != 1) return DSA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || S % 64 != 0) return DSA_ERR_UNSUPPORTED;
  {
    const int gq = Hq / Hkv;
    if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return DSA_ERR_UNSUPPORTED;
  }
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(centroids)) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  const int nb = S / 64, grp = Hq / Hkv;
  const int ncand = force_last ? nb - 1 : nb;
  const int count = std::min(keep, ncand) + force_last;
  if (sel_idx && kcap < count) return DSA_ERR_CAPACITY;
  const size_t sel_smem = (size_t)nb * 8 + (size_t)((nb + 31) / 32) * 4;   // one q-head's scores, ids, bitmap
  if (sel_smem > 200 * 1024) return DSA_ERR_UNSUPPORTED;
  const int nchmax = (nb + kDecChunk - 1) / kDecChunk;
  WsCarve c(ws);
  DecodeParams p{};
  p.status = static_cast<uint32_t*>(c.take(kStatusBytes));
  p.kbits = static_cast<uint32_t*>(c.take((size_t)B * Hq * ((nb + 31) / 32) * 4));
  p.uidx = static_cast<int32_t*>(c.take((size_t)B * Hkv * nb * 4));
  p.umask = static_cast<uint8_t*>(c.take((size_t)B * Hkv * nb));
  p.ucnt = static_cast<int32_t*>(c.take((size_t)B * Hkv * 4));
  p.part_ml = static_cast<float*>(c.take((size_t)B * Hq * nchmax * 2 * 4));
  p.part_acc = static_cast<float*>(c.take((size_t)B * Hq * nchmax * d * 4));
  p.scores = static_cast<float*>(c.take((size_t)B * Hq * nb * 4));
  if (!ws) {
    *ws_bytes = c.off;
    return DSA_OK;
  }
  if (*ws_bytes < c.off) return DSA_ERR_INVALID_ARG;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(k_cache);
  p.vc = static_cast<const __nv_bfloat16*>(v_cache);
  p.cent = centroids;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.sel_idx = sel_idx;
  p.sel_cnt = sel_cnt;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.nb = nb;
  p.grp = grp;
  p.keep = keep;
  p.force_last = force_last;
  p.kcap = kcap;
  p.nchmax = nchmax;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc;
  switch (grp * 1000 + d) {
#define DSA_DECODE_CASE(G, DD)                                                                  \
  case G * 1000 + DD:                                                                           \
    rc = launch_decode<DD, G>(p, B, Hkv, nchmax, sel_smem, st);                                 \
    break;
    DSA_DECODE_CASE(1, 64) DSA_DECODE_CASE(2, 64) DSA_DECODE_CASE(4, 64) DSA_DECODE_CASE(8, 64)
    DSA_DECODE_CASE(1, 128) DSA_DECODE_CASE(2, 128) DSA_DECODE_CASE(4, 128) DSA_DECODE_CASE(8, 128)
#undef DSA_DECODE_CASE
    default:
      return DSA_ERR_UNSUPPORTED;
  }
  if (rc) return rc;
  if (d == 128) decode_combine_kernel<128><<<B * Hq, 128, 0, st>>>(p);
  else decode_combine_kernel<64><<<B * Hq, 128, 0, st>>>(p);
  return launch_check();
}

int kmeans_clusters(const void* k_cache, int B, int Hkv, int S, int d, int n_ctx, int C, int iters,
                    float* centroids, int32_t* assign, int32_t* offsets, int32_t* tokens, void* ws, size_t* ws_bytes,
                    dsa_stream_t stream) {
  if (!k_cache || !centroids || !assign || !offsets || !tokens || !ws_bytes) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || S <= 0 || n_ctx <= 0 || n_ctx > S || C <= 0 || iters <= 0) return DSA_ERR_INVALID_ARG;
  if (C > n_ctx) return DSA_ERR_INVALID_ARG;   // every starting segment holds a key
  if ((d != 64 && d != 128) || C > kKmMaxC) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv > 65535 || (int64_t)S * d >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv * S >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(k_cache) || !aligned16(centroids)) return DSA_ERR_INVALID_ARG;
  const int BG = B * Hkv;
  WsCarve c(ws);
  uint32_t* status = static_cast<uint32_t*>(c.take(kStatusBytes));
  float* cnorm = static_cast<float*>(c.take((size_t)BG * C * 4));
  // the centroids as bf16 hi / lo halves, the assignment's tensor-core operands
  auto* chi = static_cast<__nv_bfloat16*>(c.take((size_t)BG * C * d * 2));
  auto* clo = static_cast<__nv_bfloat16*>(c.take((size_t)BG * C * d * 2));
  if (!ws) {
    *ws_bytes = c.off;
    return DSA_OK;
  }
  if (*ws_bytes < c.off) return DSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  KmParams p{};
  p.k = static_cast<const __nv_bfloat16*>(k_cache);
  p.cent = centroids;
  p.cnorm = cnorm;
  p.chi = chi;
  p.clo = clo;
  p.assign = assign;
  p.off = offsets;
  p.tok = tokens;
  p.status = status;
  p.S = S;
  p.n_ctx = n_ctx;
  p.C = C;
  p.BG = BG;
  CUtensorMap tk, th, tl;
  if (!make_tmap_rows(&tk, k_cache, (int64_t)BG * S, d, 128) || !make_tmap_rows(&th, chi, (int64_t)BG * C, d, 128) ||
      !make_tmap_rows(&tl, clo, (int64_t)BG * C, d, 128))
    return DSA_ERR_CUDA;
  int rc;
  const dim3 gi(C, BG), ga((n_ctx + 255) / 256, BG), gu((C + 7) / 8, BG);
  if (d == 128) {
    if ((rc = set_smem(kmeans_assign_kernel<128>, KmAssignLayout<128>::kSmemAlloc))) return rc;
    kmeans_init_kernel<128><<<gi, 128, 0, st>>>(p);
  } else {
    if ((rc = set_smem(kmeans_assign_kernel<64>, KmAssignLayout<64>::kSmemAlloc))) return rc;
    kmeans_init_kernel<64><<<gi, 64, 0, st>>>(p);
  }
  if ((rc = launch_check())) return rc;
  for (int it = 0; it < iters; ++it) {
    if (d == 128) kmeans_assign_kernel<128><<<ga, 320, KmAssignLayout<128>::kSmemAlloc, st>>>(tk, th, tl, p);
    else kmeans_assign_kernel<64><<<ga, 320, KmAssignLayout<64>::kSmemAlloc, st>>>(tk, th, tl, p);
    if ((rc = launch_check())) return rc;
    kmeans_csr_kernel<<<BG, 1024, 0, st>>>(p);
    if ((rc = launch_check())) return rc;
    if (d == 128) kmeans_update_kernel<128><<<gu, 256, 0, st>>>(p);
    else kmeans_update_kernel<64><<<gu, 256, 0, st>>>(p);
    if ((rc = launch_check())) return rc;
  }
  return DSA_OK;
}

int cluster_pack_kv(const void* k_cache, const void* v_cache, const int32_t* tokens, int B, int Hkv, int S, int d,
                    int n_ctx, void* k_packed, void* v_packed, dsa_stream_t stream) {
  if (!k_cache || !v_cache || !tokens || !k_packed || !v_packed) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || S <= 0 || n_ctx <= 0 || n_ctx > S) return DSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv > 65535 || (int64_t)S * d >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_packed) || !aligned16(v_packed))
    return DSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid((unsigned)((n_ctx + 7) / 8), (unsigned)(B * Hkv));
  const auto* k = static_cast<const __nv_bfloat16*>(k_cache);
  const auto* v = static_cast<const __nv_bfloat16*>(v_cache);
  auto* kp = static_cast<__nv_bfloat16*>(k_packed);
  auto* vp = static_cast<__nv_bfloat16*>(v_packed);
  if (d == 128) cluster_pack_kernel<128><<<grid, 256, 0, st>>>(k, v, tokens, S, n_ctx, kp, vp);
  else cluster_pack_kernel<64><<<grid, 256, 0, st>>>(k, v, tokens, S, n_ctx, kp, vp);
  return launch_check();
}

int cluster_decode_attn(const void* q, const void* k_cache, const void* v_cache, const float* centroids,
                        const int32_t* offsets, const int32_t* tokens, const void* k_packed, const void* v_packed,
                        int B, int Hq, int Hkv, int S, int d, int n_ctx, int C, int keep, float scale, void* o,
                        int32_t* sel_idx, int32_t* sel_cnt, int kcap, void* ws, size_t* ws_bytes,
                        dsa_stream_t stream) {
  if (!q || !k_cache || !v_cache || !centroids || !offsets || !tokens || !o || !ws_bytes) return DSA_ERR_INVALID_ARG;
  if ((k_packed == nullptr) != (v_packed == nullptr)) return DSA_ERR_INVALID_ARG;
  if (k_packed && (!aligned16(k_packed) || !aligned16(v_packed))) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S <= 0 || n_ctx <= 0 || n_ctx > S || C <= 0 || keep < 0)
    return DSA_ERR_INVALID_ARG;
  if (keep == 0 && n_ctx == S) return DSA_ERR_INVALID_ARG;   // nothing to attend
  if ((d != 64 && d != 128) || C > kKmMaxC) return DSA_ERR_UNSUPPORTED;
  const int grp = Hq / Hkv;
  if (grp != 1 && grp != 2 && grp != 4 && grp != 8) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv > 65535 || (int64_t)S * d >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(centroids)) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (sel_idx && kcap < std::min(keep, C)) return DSA_ERR_CAPACITY;
  // one q-head's candidate scores, ids, top ids, the offsets and a bitmap
  const size_t sel_smem = (size_t)C * 12 + (size_t)(C + 1) * 4 + (size_t)((C + 31) / 32) * 4;
  if (sel_smem > 200 * 1024) return DSA_ERR_UNSUPPORTED;
  const int nchmax = (S + kClChunk - 1) / kClChunk;
  WsCarve c(ws);
  ClusterParams cp{};
  DecodeParams& p = cp.dp;
  p.status = static_cast<uint32_t*>(c.take(kStatusBytes));
  p.kbits = static_cast<uint32_t*>(c.take((size_t)B * Hq * ((C + 31) / 32) * 4));
  // union lists per (batch, KV head), rows padded to 16 entries (the head
  // masks are bulk-copied 16-byte aligned)
  const int lstride = (S + 15) & ~15;
  p.uidx = static_cast<int32_t*>(c.take((size_t)B * Hkv * lstride * 4));
  p.umask = static_cast<uint8_t*>(c.take((size_t)B * Hkv * lstride));
  float* cl_scores = static_cast<float*>(c.take((size_t)B * Hq * C * 4));
  p.ucnt = static_cast<int32_t*>(c.take((size_t)B * Hkv * 4));
  p.part_ml = static_cast<float*>(c.take((size_t)B * Hq * nchmax * 2 * 4));
  p.part_acc = static_cast<float*>(c.take((size_t)B * Hq * nchmax * d * 4));
  if (!ws) {
    *ws_bytes = c.off;
    return DSA_OK;
  }
  if (*ws_bytes < c.off) return DSA_ERR_INVALID_ARG;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(k_cache);
  p.vc = static_cast<const __nv_bfloat16*>(v_cache);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.sel_idx = sel_idx;
  p.sel_cnt = sel_cnt;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.nb = lstride;   // list row stride
  p.grp = grp;
  p.keep = keep;
  p.kcap = kcap;
  p.nchmax = nchmax;
  p.scale_log2 = scale * 1.4426950408889634f;
  cp.cent = centroids;
  cp.off = offsets;
  cp.tok = tokens;
  cp.scores = cl_scores;
  cp.C = C;
  cp.n_ctx = n_ctx;
  p.kp = static_cast<const __nv_bfloat16*>(k_packed);
  p.vp = static_cast<const __nv_bfloat16*>(v_packed);
  p.n_packed = k_packed ? n_ctx : 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc;
  switch (grp * 1000 + d) {
#define DSA_CLUSTER_CASE(G, DD)                                                                 \
  case G * 1000 + DD:                                                                           \
    rc = launch_cluster_decode<DD, G>(cp, B, Hkv, nchmax, sel_smem, st);                        \
    break;
    DSA_CLUSTER_CASE(1, 64) DSA_CLUSTER_CASE(2, 64) DSA_CLUSTER_CASE(4, 64) DSA_CLUSTER_CASE(8, 64)
    DSA_CLUSTER_CASE(1, 128) DSA_CLUSTER_CASE(2, 128) DSA_CLUSTER_CASE(4, 128) DSA_CLUSTER_CASE(8, 128)
#undef DSA_CLUSTER_CASE
    default:
      return DSA_ERR_UNSUPPORTED;
  }
  if (rc) return rc;
  if (d == 128) decode_combine_kernel<128, kClChunk><<<B * Hq, 128, 0, st>>>(p);
  else decode_combine_kernel<64, kClChunk><<<B * Hq, 128, 0, st>>>(p);
  return launch_check();
}

}  // extern "C"
