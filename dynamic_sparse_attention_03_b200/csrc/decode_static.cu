// decode_static.cu -- sparse_decode_attn_static: the centroid-ranked sparse
// decode of sparse_decode_attn, with its scratch memory in a fixed array that
// the library itself holds in device memory, for callers that cannot allocate.
//
// Who needs it: code that is handed device pointers but has no way to obtain
// more device memory -- a plugin inside a host application or serving engine
// whose allocator owns the whole GPU budget and exposes no allocation hook,
// or a latency-critical decode loop that must never call cudaMalloc (it can
// synchronize the device and fail under fragmentation).  Such a caller still
// passes its inputs and outputs, but no workspace.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes
// (32 MiB); every GPU that loads the library keeps it until the process exits.
// Host code must not use the array's name as a device address (on the host it
// names a host-side shadow), so the device address is looked up with
// cudaGetSymbolAddress, with the device current, once per device and context:
// a device reset makes a new primary context, in which the module is loaded
// again and the array may move, so a context change triggers a new lookup.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/dsa.h"
#include "decode.cuh"

using namespace dsa;

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
struct ScratchAddr {
  unsigned long long ctx_id;   // context the address belongs to (0: none yet)
  void* ptr;
};
ScratchAddr g_scratch_addr[kMaxDevices] = {};

// The current context's unique id (driver entry points, found once); 0 if unknown.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess && cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) ==
        cudaSuccess && qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrent>(a);
      get_id = reinterpret_cast<GetId>(b);
    }
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device, looked up on the
// first call per device and again whenever the device's context has changed
// (or its id cannot be read).  nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long id = current_context_id();   // 0 before the context exists
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchAddr& e = g_scratch_addr[dev];
  if (!e.ptr || id == 0 || e.ctx_id != id) {
    void* p = nullptr;
    // (creates the device's primary context if there is none yet)
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
    e.ptr = p;
    e.ctx_id = current_context_id();
  }
  return e.ptr;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

template <int D, int G>
int launch(const DecodeParams& p, int B, int Hkv, int nchmax, size_t sel_smem, cudaStream_t st) {
  if (sel_smem > 48 * 1024 &&
      cudaFuncSetAttribute(decode_topk_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem) !=
          cudaSuccess)
    return DSA_ERR_CUDA;
  decode_score_kernel<D, G><<<dim3(B * Hkv, (p.nb + 63) / 64), 256, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  decode_topk_kernel<256><<<B * Hkv * G, 256, sel_smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  decode_union_kernel<G, 256><<<B * Hkv, 256, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaFuncSetAttribute(decode_attn_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           DecLayout<D>::kBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  decode_attn_kernel<D, G><<<dim3(B * Hkv, nchmax), kDecThreads, DecLayout<D>::kBytes, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  decode_combine_kernel<D><<<B * (Hkv * G), 128, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

extern "C" int sparse_decode_attn_static(const void* q, const void* k_cache, const void* v_cache,
                                         const float* centroids, int B, int Hq, int Hkv, int S, int d, int keep,
                                         int force_last, float scale, void* o, int32_t* sel_idx, int32_t* sel_cnt,
                                         int kcap, dsa_stream_t stream) {
  if (!q || !k_cache || !v_cache || !centroids || !o) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S < 64 || keep < 0) return DSA_ERR_INVALID_ARG;
  if (force_last != 0 && force_last != 1) return DSA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || S % 64 != 0) return DSA_ERR_UNSUPPORTED;
  const int grp = Hq / Hkv;
  if (grp != 1 && grp != 2 && grp != 4 && grp != 8) return DSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache) |
       reinterpret_cast<uintptr_t>(centroids)) & 15u)
    return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  const int nb = S / 64;
  const int ncand = force_last ? nb - 1 : nb;
  const int count = (keep < ncand ? keep : ncand) + force_last;
  if (sel_idx && kcap < count) return DSA_ERR_CAPACITY;
  const size_t sel_smem = (size_t)nb * 8 + (size_t)((nb + 31) / 32) * 4;   // one q-head's scores, ids, bitmap
  if (sel_smem > 200 * 1024) return DSA_ERR_UNSUPPORTED;
  const int nchmax = (nb + kDecChunk - 1) / kDecChunk;
  // Scratch layout (the workspace of sparse_decode_attn): status word, per-head
  // kept bitmaps, union lists and masks, union counts, chunk partials, block scores.
  size_t off = 0;
  const size_t o_status = off; off = up256(off + 256);
  const size_t o_bits = off;   off = up256(off + (size_t)B * Hq * ((nb + 31) / 32) * 4);
  const size_t o_uidx = off;   off = up256(off + (size_t)B * Hkv * nb * 4);
  const size_t o_umask = off;  off = up256(off + (size_t)B * Hkv * nb);
  const size_t o_ucnt = off;   off = up256(off + (size_t)B * Hkv * 4);
  const size_t o_ml = off;     off = up256(off + (size_t)B * Hq * nchmax * 2 * 4);
  const size_t o_acc = off;    off = up256(off + (size_t)B * Hq * nchmax * d * 4);
  const size_t o_sc = off;     off = up256(off + (size_t)B * Hq * nb * 4);
  if (off > kStaticScratchBytes) return DSA_ERR_CAPACITY;
  uint8_t* base = static_cast<uint8_t*>(scratch_on_current_device());
  if (!base) return DSA_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the status word must start at zero.
  if (cudaMemsetAsync(base + o_status, 0, 256, st) != cudaSuccess) return DSA_ERR_CUDA;
  DecodeParams p{};
  p.status = reinterpret_cast<uint32_t*>(base + o_status);
  p.kbits = reinterpret_cast<uint32_t*>(base + o_bits);
  p.uidx = reinterpret_cast<int32_t*>(base + o_uidx);
  p.umask = base + o_umask;
  p.ucnt = reinterpret_cast<int32_t*>(base + o_ucnt);
  p.part_ml = reinterpret_cast<float*>(base + o_ml);
  p.part_acc = reinterpret_cast<float*>(base + o_acc);
  p.scores = reinterpret_cast<float*>(base + o_sc);
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
  switch (grp * 1000 + d) {
    case 1064: return launch<64, 1>(p, B, Hkv, nchmax, sel_smem, st);
    case 2064: return launch<64, 2>(p, B, Hkv, nchmax, sel_smem, st);
    case 4064: return launch<64, 4>(p, B, Hkv, nchmax, sel_smem, st);
    case 8064: return launch<64, 8>(p, B, Hkv, nchmax, sel_smem, st);
    case 1128: return launch<128, 1>(p, B, Hkv, nchmax, sel_smem, st);
    case 2128: return launch<128, 2>(p, B, Hkv, nchmax, sel_smem, st);
    case 4128: return launch<128, 4>(p, B, Hkv, nchmax, sel_smem, st);
    case 8128: return launch<128, 8>(p, B, Hkv, nchmax, sel_smem, st);
    default: return DSA_ERR_UNSUPPORTED;
  }
}
