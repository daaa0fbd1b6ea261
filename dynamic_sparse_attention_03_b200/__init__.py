"""Python binding of libdsa.so: dynamic sparse attention on B200 (sm_100a).

Argument marshalling only: torch tensors are checked for dtype/shape/device,
their device pointers and the current CUDA stream cross the C ABI declared in
include/dsa.h, and every step of the computation runs in the library's CUDA
kernels.  There is no CPU path: if libdsa.so is missing or no GPU is present
the calls raise.

Entry points (same names as the C ABI):
  sparse_index_estimate  block-sparse index (mean-pooled Q/K, top-k with sink+diagonal)
  pool_keys              per-64-token-block mean keys (decode centroids)
  vertical_slash_index   vertical-slash index and its block/column plan
  block_sparse_attn_fwd  causal attention over the chosen blocks and columns
  sparse_decode_attn     centroid-ranked sparse decode
  kmeans_clusters        K-means key clusters of a fixed context (centroids, cluster -> key map)
  cluster_pack_kv        the context's K and V rows copied in cluster order
  cluster_decode_attn    decode ranked by K-means cluster centroids
"""

from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional

import torch

__all__ = [
    "DSAError", "load_library", "SYMBOLS", "sparse_index_estimate", "pool_keys", "vertical_slash_index",
    "block_sparse_attn_fwd", "sparse_decode_attn", "get_status", "block_index_capacity", "Workspace",
    "kmeans_clusters", "cluster_pack_kv", "cluster_decode_attn",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsa.so")

# Every symbol include/dsa.h declares.
SYMBOLS = (
    "sparse_index_estimate",
    "vertical_slash_index",
    "block_sparse_attn_fwd",
    "sparse_decode_attn",
    "sparse_decode_attn_static",
    "a_shape_index",
    "kmeans_clusters",
    "cluster_pack_kv",
    "cluster_decode_attn",
    "dsa_get_status",
    "dsa_block_index_capacity",
    "dsa_version",
)

ERRORS = {
    -1: "DSA_ERR_INVALID_ARG",
    -2: "DSA_ERR_UNSUPPORTED",
    -3: "DSA_ERR_CAPACITY",
    -4: "DSA_ERR_CUDA",
    -5: "DSA_ERR_TIMEOUT",
}


class DSAError(RuntimeError):
    def __init__(self, name: str, rc: int):
        super().__init__(f"{name} failed: {ERRORS.get(rc, rc)} ({rc})")
        self.rc = rc


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.POINTER(ctypes.c_size_t)

_SIGS = {
    "sparse_index_estimate": [_P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _I, _P, _P, _SZ, _P],
    "vertical_slash_index": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _I, _P, _P, _I, _P, _SZ, _P],
    "block_sparse_attn_fwd": [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P, _I, _P, _P, _I, _P, _P, _SZ, _P],
    "sparse_decode_attn": [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _I, _P, _SZ, _P],
    "sparse_decode_attn_static": [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _I, _P],
    "a_shape_index": [_I, _I, _I, _I, _P, _P, _I, _P],
    "kmeans_clusters": [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "cluster_pack_kv": [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P],
    "cluster_decode_attn": [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _I, _P,
                            _SZ, _P],
    "dsa_get_status": [_P, _P],
    "dsa_block_index_capacity": [_I, _I, _I, _F],
    "dsa_version": [],
}


def load_library(path: str = LIB_PATH):
    """Load libdsa.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with `python -m dynamic_sparse_attention_03_b200.build`")
            lib = ctypes.CDLL(path)
            for name, args in _SIGS.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = ctypes.c_char_p if name == "dsa_version" else ctypes.c_int
            _lib = lib
    return _lib


def _check(rc: int, name: str):
    if rc != 0:
        raise DSAError(name, rc)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("dynamic sparse attention runs on CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _need_dtype(t, dt, name):
    if t.dtype != dt:
        raise TypeError(f"{name} must be {dt}, got {t.dtype}")


def _need_shape(t, shape, name):
    # the C entry points trust the sizes they are given: check them here
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


class Workspace:
    """Device scratch for the library calls, grown on demand, one per device.

    The first 256 bytes hold the library's sticky status word; they are zeroed
    when the buffer is (re)allocated and cleared again by get_status()."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf = torch.zeros(256, dtype=torch.uint8, device=self.device)

    def ensure(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            # the old buffer may still be in use by calls queued on any stream:
            # let them finish before its memory can be handed out again (growth
            # happens on the first calls of a size, not in steady state)
            torch.cuda.synchronize(self.device)
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf


_ws_cache: dict = {}


def _workspace(dev: torch.device, ws: Optional[Workspace]) -> Workspace:
    if ws is not None:
        return ws
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    if key not in _ws_cache:
        _ws_cache[key] = Workspace(torch.device("cuda", key[1]))
    return _ws_cache[key]


def _on_device(dev):
    """Context that makes dev the current CUDA device for a library call."""
    return torch.cuda.device(dev)


def _dev_index(dev) -> int:
    dev = torch.device(dev)
    return dev.index if dev.index is not None else torch.cuda.current_device()


def _call_with_ws(name, args_before_ws, dev, ws):
    """Query the workspace size (ws = NULL), then call with the buffer.  The
    tensors' device is made current for the call: the library sizes grids and
    sets kernel attributes for the current device."""
    lib = load_library()
    fn = getattr(lib, name)
    size = ctypes.c_size_t(0)
    with _on_device(dev):
        _check(fn(*args_before_ws, None, ctypes.byref(size), _stream(dev)), name)
        w = _workspace(dev, ws)
        if _dev_index(w.device) != _dev_index(dev):
            raise ValueError(f"workspace is on {w.device}, tensors on {dev}")
        buf = w.ensure(size.value)
        _check(fn(*args_before_ws, _ptr(buf), ctypes.byref(size), _stream(dev)), name)
    return w


def get_status(ws: Optional[Workspace] = None, device=None) -> int:
    """Synchronize the current stream and return (and clear) the device status word."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    w = _workspace(dev, ws)
    with _on_device(w.device):
        return load_library().dsa_get_status(_ptr(w.buf), _stream(w.device))


def block_index_capacity(n: int, k_fixed: int = 0, keep_ratio: float = 0.0) -> int:
    rc = load_library().dsa_block_index_capacity(int(n), 64, int(k_fixed), float(keep_ratio))
    if rc < 0:
        raise DSAError("dsa_block_index_capacity", rc)
    return rc


def sparse_index_estimate(q: torch.Tensor, k: torch.Tensor, k_fixed: int = 0, keep_ratio: float = 0.0,
                          kcap: Optional[int] = None, pooled_k: Optional[torch.Tensor] = None,
                          block_idx: Optional[torch.Tensor] = None, block_cnt: Optional[torch.Tensor] = None,
                          ws: Optional[Workspace] = None):
    """Block-sparse index.  q [Hq][n][d], k [Hkv][n][d] bf16 on one GPU.

    Returns (block_idx [Hq][n/64][kcap] int32, block_cnt [Hq][n/64] int32)."""
    _need_cuda(q, k, pooled_k, block_idx, block_cnt)
    _need_dtype(q, torch.bfloat16, "q")
    _need_dtype(k, torch.bfloat16, "k")
    Hq, n, d = q.shape
    Hkv = k.shape[0]
    if k.shape[1:] != (n, d):
        raise ValueError("k must be [Hkv][n][d] with q's n and d")
    nqb = n // 64
    if kcap is None:
        kcap = block_idx.shape[-1] if block_idx is not None else block_index_capacity(n, k_fixed, keep_ratio)
    if block_idx is None:
        block_idx = torch.empty((Hq, nqb, kcap), dtype=torch.int32, device=q.device)
    if block_cnt is None:
        block_cnt = torch.empty((Hq, nqb), dtype=torch.int32, device=q.device)
    _need_dtype(block_idx, torch.int32, "block_idx")
    _need_dtype(block_cnt, torch.int32, "block_cnt")
    _need_shape(block_idx, (Hq, nqb, kcap), "block_idx")
    _need_shape(block_cnt, (Hq, nqb), "block_cnt")
    if pooled_k is not None:
        _need_dtype(pooled_k, torch.float32, "pooled_k")
        _need_shape(pooled_k, (Hkv, nqb, d), "pooled_k")
    args = [_ptr(q), _ptr(k), Hq, Hkv, n, d, 64, int(k_fixed), float(keep_ratio), _ptr(block_idx),
            _ptr(block_cnt), int(kcap), _ptr(pooled_k)]
    _call_with_ws("sparse_index_estimate", args, q.device, ws)
    return block_idx, block_cnt


def pool_keys(k: torch.Tensor, out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None) -> torch.Tensor:
    """Per-64-token-block mean keys (fp32).  k [..., S, d] bf16 -> [..., S/64, d]."""
    _need_cuda(k, out)
    _need_dtype(k, torch.bfloat16, "k")
    S, d = k.shape[-2], k.shape[-1]
    lead = k.shape[:-2]
    rows = int(math.prod(lead)) if lead else 1
    if out is None:
        out = torch.empty(lead + (S // 64, d), dtype=torch.float32, device=k.device)
    _need_dtype(out, torch.float32, "out")
    _need_shape(out, lead + (S // 64, d), "out")
    args = [None, _ptr(k), 0, rows, S, d, 64, 0, 0.0, None, None, 0, _ptr(out)]
    _call_with_ws("sparse_index_estimate", args, k.device, ws)
    return out


def vertical_slash_index(q: torch.Tensor, k: torch.Tensor, n_vert: int, n_slash: int, scale: Optional[float] = None,
                         last_q: int = 64, kcap: Optional[int] = None, ccap: Optional[int] = None,
                         ws: Optional[Workspace] = None, out: Optional[dict] = None) -> dict:
    """Vertical-slash index and plan.  Returns a dict of int32 tensors:
    vert_idx [Hq][n_vert], slash_off [Hq][n_slash], block_idx [Hq][n/64][kcap],
    block_cnt, col_idx [Hq][n/64][ccap], col_cnt.  Pass a previous result as
    `out` to write into the same tensors."""
    _need_cuda(q, k)
    _need_dtype(q, torch.bfloat16, "q")
    _need_dtype(k, torch.bfloat16, "k")
    Hq, n, d = q.shape
    Hkv = k.shape[0]
    _need_shape(k, (Hkv, n, d), "k")
    nqb = n // 64
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dev = q.device
    if out is not None:
        kcap = out["block_idx"].shape[-1]
        ccap = out["col_idx"].shape[-1]
        _need_cuda(*out.values())
    kcap = min(nqb, 2 * n_slash) if kcap is None else kcap
    ccap = n_vert if ccap is None else ccap
    out = out if out is not None else dict(
        vert_idx=torch.empty((Hq, n_vert), dtype=torch.int32, device=dev),
        slash_off=torch.empty((Hq, n_slash), dtype=torch.int32, device=dev),
        block_idx=torch.empty((Hq, nqb, kcap), dtype=torch.int32, device=dev),
        block_cnt=torch.empty((Hq, nqb), dtype=torch.int32, device=dev),
        col_idx=torch.empty((Hq, nqb, ccap), dtype=torch.int32, device=dev),
        col_cnt=torch.empty((Hq, nqb), dtype=torch.int32, device=dev),
    )
    for nm, shape in (("vert_idx", (Hq, n_vert)), ("slash_off", (Hq, n_slash)), ("block_idx", (Hq, nqb, kcap)),
                      ("block_cnt", (Hq, nqb)), ("col_idx", (Hq, nqb, ccap)), ("col_cnt", (Hq, nqb))):
        _need_dtype(out[nm], torch.int32, nm)
        _need_shape(out[nm], shape, nm)
    args = [_ptr(q), _ptr(k), Hq, Hkv, n, d, int(last_q), int(n_vert), int(n_slash), float(scale),
            _ptr(out["vert_idx"]), _ptr(out["slash_off"]), _ptr(out["block_idx"]), _ptr(out["block_cnt"]), kcap,
            _ptr(out["col_idx"]), _ptr(out["col_cnt"]), ccap]
    _call_with_ws("vertical_slash_index", args, dev, ws)
    return out


def block_sparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_idx: torch.Tensor,
                          block_cnt: torch.Tensor, col_idx: Optional[torch.Tensor] = None,
                          col_cnt: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                          return_lse: bool = False, out: Optional[torch.Tensor] = None,
                          ws: Optional[Workspace] = None):
    """Causal attention over the chosen blocks (and columns).  Returns O [Hq][n][d]
    bf16 (and lse [Hq][n] fp32 when return_lse)."""
    _need_cuda(q, k, v, block_idx, block_cnt, col_idx, col_cnt, out)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _need_dtype(t, torch.bfloat16, nm)
    Hq, n, d = q.shape
    Hkv = k.shape[0]
    nqb = n // 64
    _need_shape(k, (Hkv, n, d), "k")
    _need_shape(v, (Hkv, n, d), "v")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    _need_dtype(o, torch.bfloat16, "out")
    _need_shape(o, (Hq, n, d), "out")
    lse = torch.empty((Hq, n), dtype=torch.float32, device=q.device) if return_lse else None
    kcap = block_idx.shape[-1]
    ccap = col_idx.shape[-1] if col_idx is not None else 0
    _need_dtype(block_idx, torch.int32, "block_idx")
    _need_dtype(block_cnt, torch.int32, "block_cnt")
    _need_shape(block_idx, (Hq, nqb, kcap), "block_idx")
    _need_shape(block_cnt, (Hq, nqb), "block_cnt")
    if (col_idx is None) != (col_cnt is None):
        raise ValueError("col_idx and col_cnt go together")
    if col_idx is not None:
        _need_dtype(col_idx, torch.int32, "col_idx")
        _need_dtype(col_cnt, torch.int32, "col_cnt")
        _need_shape(col_idx, (Hq, nqb, ccap), "col_idx")
        _need_shape(col_cnt, (Hq, nqb), "col_cnt")
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(o), Hq, Hkv, n, d, float(scale), _ptr(block_idx), _ptr(block_cnt), kcap,
            _ptr(col_idx), _ptr(col_cnt), ccap, _ptr(lse)]
    _call_with_ws("block_sparse_attn_fwd", args, q.device, ws)
    return (o, lse) if return_lse else o


def _check_decode_inputs(q, k_cache, v_cache, centroids, out):
    B, Hq, d = q.shape
    Hkv, S = k_cache.shape[1], k_cache.shape[2]
    for t, nm in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_dtype(t, torch.bfloat16, nm)
    _need_shape(k_cache, (B, Hkv, S, d), "k_cache")
    _need_shape(v_cache, (B, Hkv, S, d), "v_cache")
    _need_shape(centroids, (B, Hkv, S // 64, d), "centroids")
    if out is not None:
        _need_dtype(out, torch.bfloat16, "out")
        _need_shape(out, (B, Hq, d), "out")


def sparse_decode_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, centroids: torch.Tensor,
                       keep: int, force_last: int = 1, scale: Optional[float] = None, return_sel: bool = False,
                       out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None):
    """Decode: q [B][Hq][d], caches [B][Hkv][S][d] bf16, centroids [B][Hkv][S/64][d] fp32.
    Returns O [B][Hq][d] bf16 (and sel_idx [B][Hq][kcap], sel_cnt [B][Hq] when return_sel)."""
    _need_cuda(q, k_cache, v_cache, centroids, out)
    _need_dtype(centroids, torch.float32, "centroids")
    B, Hq, d = q.shape
    Hkv, S = k_cache.shape[1], k_cache.shape[2]
    _check_decode_inputs(q, k_cache, v_cache, centroids, out)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    nb = S // 64
    kcap = min(keep, nb - 1 if force_last else nb) + (1 if force_last else 0)
    sel_idx = sel_cnt = None
    if return_sel:
        sel_idx = torch.empty((B, Hq, max(kcap, 1)), dtype=torch.int32, device=q.device)
        sel_cnt = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
    args = [_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(centroids), B, Hq, Hkv, S, d, int(keep), int(force_last),
            float(scale), _ptr(o), _ptr(sel_idx), _ptr(sel_cnt), max(kcap, 1)]
    _call_with_ws("sparse_decode_attn", args, q.device, ws)
    return (o, sel_idx, sel_cnt) if return_sel else o


def sparse_decode_attn_static(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                              centroids: torch.Tensor, keep: int, force_last: int = 1, scale: Optional[float] = None,
                              return_sel: bool = False, out: Optional[torch.Tensor] = None):
    """sparse_decode_attn with no workspace: the library's own fixed 32 MiB
    device array holds the scratch (for callers that cannot allocate device
    memory).  Calls sharing a device must not overlap on the GPU."""
    _need_cuda(q, k_cache, v_cache, centroids, out)
    _need_dtype(centroids, torch.float32, "centroids")
    B, Hq, d = q.shape
    Hkv, S = k_cache.shape[1], k_cache.shape[2]
    _check_decode_inputs(q, k_cache, v_cache, centroids, out)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    nb = S // 64
    kcap = max(min(keep, nb - 1 if force_last else nb) + (1 if force_last else 0), 1)
    sel_idx = sel_cnt = None
    if return_sel:
        sel_idx = torch.empty((B, Hq, kcap), dtype=torch.int32, device=q.device)
        sel_cnt = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
    # the library's scratch array of the current device is used: make q's current
    with _on_device(q.device):
        rc = load_library().sparse_decode_attn_static(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(centroids), B, Hq, Hkv, S, d, int(keep), int(force_last),
            float(scale), _ptr(o), _ptr(sel_idx), _ptr(sel_cnt), kcap, _stream(q.device))
    _check(rc, "sparse_decode_attn_static")
    return (o, sel_idx, sel_cnt) if return_sel else o


def a_shape_index(Hq: int, n: int, n_sink: int, n_local: int, device=None):
    """Static sink + local-window block lists for block_sparse_attn_fwd.
    Returns (block_idx [Hq][n/64][kcap], block_cnt [Hq][n/64])."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    nqb = n // 64
    kcap = max(1, min(nqb, n_sink + n_local))
    bi = torch.empty((Hq, nqb, kcap), dtype=torch.int32, device=dev)
    bc = torch.empty((Hq, nqb), dtype=torch.int32, device=dev)
    with _on_device(dev):
        _check(load_library().a_shape_index(Hq, n, n_sink, n_local, _ptr(bi), _ptr(bc), kcap, _stream(dev)),
               "a_shape_index")
    return bi, bc


def kmeans_clusters(k_cache: torch.Tensor, n_ctx: int, n_clusters: int, iters: int,
                    ws: Optional[Workspace] = None):
    """Lloyd's K-means over the first n_ctx keys of every (batch, KV head) of
    k_cache [B][Hkv][S][d] bf16, started from the means of n_clusters equal
    contiguous segments.  Returns (centroids [B][Hkv][C][d] fp32, assign
    [B][Hkv][n_ctx] int32, offsets [B][Hkv][C+1] int32, tokens [B][Hkv][n_ctx]
    int32): the cluster -> key map lists cluster c's keys, ascending, at
    tokens[offsets[c]:offsets[c+1]]."""
    _need_cuda(k_cache)
    _need_dtype(k_cache, torch.bfloat16, "k_cache")
    B, Hkv, S, d = k_cache.shape
    dev = k_cache.device
    C = int(n_clusters)
    cent = torch.empty((B, Hkv, C, d), dtype=torch.float32, device=dev)
    assign = torch.empty((B, Hkv, n_ctx), dtype=torch.int32, device=dev)
    offsets = torch.empty((B, Hkv, C + 1), dtype=torch.int32, device=dev)
    tokens = torch.empty((B, Hkv, n_ctx), dtype=torch.int32, device=dev)
    args = [_ptr(k_cache), B, Hkv, S, d, int(n_ctx), C, int(iters), _ptr(cent), _ptr(assign), _ptr(offsets),
            _ptr(tokens)]
    _call_with_ws("kmeans_clusters", args, dev, ws)
    return cent, assign, offsets, tokens


def cluster_pack_kv(k_cache: torch.Tensor, v_cache: torch.Tensor, tokens: torch.Tensor, n_ctx: int,
                    out: Optional[tuple] = None):
    """The first n_ctx rows of k_cache / v_cache [B][Hkv][S][d] bf16 copied in
    cluster order (tokens from kmeans_clusters): returns (k_packed, v_packed)
    [B][Hkv][n_ctx][d] with k_packed[b, g, p] = k_cache[b, g, tokens[b, g, p]]."""
    _need_cuda(k_cache, v_cache, tokens)
    _need_dtype(k_cache, torch.bfloat16, "k_cache")
    _need_dtype(v_cache, torch.bfloat16, "v_cache")
    _need_dtype(tokens, torch.int32, "tokens")
    B, Hkv, S, d = k_cache.shape
    _need_shape(v_cache, k_cache.shape, "v_cache")
    _need_shape(tokens, (B, Hkv, int(n_ctx)), "tokens")
    if out is None:
        kp = torch.empty((B, Hkv, int(n_ctx), d), dtype=torch.bfloat16, device=k_cache.device)
        vp = torch.empty_like(kp)
    else:
        kp, vp = out
        _need_cuda(kp, vp)
        for t, nm in ((kp, "k_packed"), (vp, "v_packed")):
            _need_dtype(t, torch.bfloat16, nm)
            _need_shape(t, (B, Hkv, int(n_ctx), d), nm)
    with _on_device(k_cache.device):
        _check(load_library().cluster_pack_kv(_ptr(k_cache), _ptr(v_cache), _ptr(tokens), B, Hkv, S, d,
                                              int(n_ctx), _ptr(kp), _ptr(vp), _stream(k_cache.device)),
               "cluster_pack_kv")
    return kp, vp


def cluster_decode_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, centroids: torch.Tensor,
                        offsets: torch.Tensor, tokens: torch.Tensor, n_ctx: int, keep: int,
                        scale: Optional[float] = None, return_sel: bool = False,
                        out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                        packed: Optional[tuple] = None):
    """Decode over K-means clusters: q [B][Hq][d], caches [B][Hkv][S][d] bf16,
    centroids / offsets / tokens from kmeans_clusters.  Each q-head keeps its
    `keep` best non-empty clusters by q.c (ties to the lower cluster) and attends
    over their keys plus the unclustered tail [n_ctx, S).  `packed` is
    cluster_pack_kv's (k_packed, v_packed), read instead of gathering rows by
    token id (same result).  Returns O [B][Hq][d] bf16 (and sel_idx [B][Hq][keep]
    ascending cluster ids, sel_cnt [B][Hq])."""
    kp, vp = packed if packed is not None else (None, None)
    _need_cuda(q, k_cache, v_cache, centroids, offsets, tokens, out, kp, vp)
    _need_dtype(centroids, torch.float32, "centroids")
    _need_dtype(offsets, torch.int32, "offsets")
    _need_dtype(tokens, torch.int32, "tokens")
    B, Hq, d = q.shape
    Hkv, S = k_cache.shape[1], k_cache.shape[2]
    C = centroids.shape[2]
    _need_shape(k_cache, (B, Hkv, S, d), "k_cache")
    _need_shape(v_cache, (B, Hkv, S, d), "v_cache")
    _need_shape(centroids, (B, Hkv, C, d), "centroids")
    _need_shape(offsets, (B, Hkv, C + 1), "offsets")
    _need_shape(tokens, (B, Hkv, int(n_ctx)), "tokens")
    if kp is not None:
        for t, nm in ((kp, "k_packed"), (vp, "v_packed")):
            _need_dtype(t, torch.bfloat16, nm)
            _need_shape(t, (B, Hkv, int(n_ctx), d), nm)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    kcap = max(min(int(keep), C), 1)
    sel_idx = sel_cnt = None
    if return_sel:
        sel_idx = torch.empty((B, Hq, kcap), dtype=torch.int32, device=q.device)
        sel_cnt = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
    args = [_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(centroids), _ptr(offsets), _ptr(tokens), _ptr(kp), _ptr(vp),
            B, Hq, Hkv, S, d, int(n_ctx), C, int(keep), float(scale), _ptr(o), _ptr(sel_idx), _ptr(sel_cnt), kcap]
    _call_with_ws("cluster_decode_attn", args, q.device, ws)
    return (o, sel_idx, sel_cnt) if return_sel else o
