"""sparse_decode_attn_static -- the decode entry point that allocates nothing.

Some callers cannot allocate device memory (a plugin whose host application's
allocator owns the GPU budget, a decode loop that must not call cudaMalloc);
this entry point keeps its scratch in a fixed array inside the library.  The
test calls it through the C ABI and checks it against sparse_decode_attn (the
workspace version) on two calls in a row with different inputs, so a stale
array from the previous call would show.  This file is collected last."""
import ctypes
import math

import pytest
import torch

import synth
import dynamic_sparse_attention_03_b200 as dsa

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("d,Hq,Hkv", [(128, 32, 8), (64, 16, 8), (128, 8, 1)])
def test_static_scratch_decode_matches_workspace_decode(d, Hq, Hkv):
    """Two calls in a row through the C ABI, each against the workspace decode
    on the same inputs: outputs within the decode's tolerance, selections bit
    for bit (head dims 64 and 128; GQA groups of 4, 2 and 8)."""
    assert torch.cuda.is_available()
    lib = dsa.load_library()
    B, S, keep = 4, 16384, 64
    kcap = keep + 1
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((101 + d + Hq, 202 + d + Hq)):
        w = synth.make_decode("decode-b16-128k", device="cuda", B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=seed)
        cent = dsa.pool_keys(w.k_cache)
        ref_o, ref_si, ref_sc = dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent, keep=keep, return_sel=True)
        o = torch.full_like(w.q, float("nan"))
        si = torch.empty((B, Hq, kcap), dtype=torch.int32, device="cuda")
        sc = torch.empty((B, Hq), dtype=torch.int32, device="cuda")
        rc = lib.sparse_decode_attn_static(_ptr(w.q), _ptr(w.k_cache), _ptr(w.v_cache), _ptr(cent), B, Hq, Hkv, S, d,
                                           keep, 1, ctypes.c_float(1 / math.sqrt(d)), _ptr(o), _ptr(si), _ptr(sc),
                                           kcap, stream)
        assert rc == 0, (call, rc)
        torch.cuda.synchronize()
        err = (o.float() - ref_o.float()).abs()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3, (call, err.max().item())
        assert torch.equal(si, ref_si) and torch.equal(sc, ref_sc), call


def test_static_scratch_decode_without_selection_outputs():
    """The Python wrapper, with no selection outputs requested (sel_idx and
    sel_cnt passed as NULL), twice in a row."""
    B, Hq, Hkv, S, d, keep = 2, 32, 8, 8192, 128, 40
    for seed in (303, 404):
        w = synth.make_decode("decode-b16-128k", device="cuda", B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=seed)
        cent = dsa.pool_keys(w.k_cache)
        ref = dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent, keep=keep)
        got = dsa.sparse_decode_attn_static(w.q, w.k_cache, w.v_cache, cent, keep=keep)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3, seed


def test_static_scratch_rejects_oversized_problems():
    lib = dsa.load_library()
    q = torch.zeros((256, 32, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    cent = torch.zeros((1, 8, 1, 128), dtype=torch.float32, device="cuda")
    # B=256, S=64K: the chunk partials alone need ~67 MB, beyond the 32 MiB
    # array -> DSA_ERR_CAPACITY, checked before anything is launched
    rc = lib.sparse_decode_attn_static(_ptr(q), _ptr(kc), _ptr(kc), _ptr(cent), 256, 32, 8, 1 << 16, 128, 256, 1,
                                       ctypes.c_float(0.088), _ptr(q), None, None, 0,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -3
