"""The Python binding checks dtypes and shapes before it calls the library
(the C entry points trust the sizes they are given).  Host logic only: the
library is replaced by a stub that records the calls, so nothing runs on a
device."""

import contextlib

import pytest
import torch

import dynamic_sparse_attention_03_b200 as dsa

bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


@pytest.fixture
def calls(monkeypatch):
    seen = []

    class StubLib:
        def __getattr__(self, name):
            if name == "dsa_block_index_capacity":
                return lambda *a: 8
            return lambda *a: (seen.append(name), 0)[1]

    monkeypatch.setattr(dsa, "_need_cuda", lambda *a: None)
    monkeypatch.setattr(dsa, "_call_with_ws", lambda name, args, dev, ws: seen.append(name))
    monkeypatch.setattr(dsa, "load_library", lambda *a, **k: StubLib())
    monkeypatch.setattr(dsa, "_stream", lambda dev: None)
    monkeypatch.setattr(dsa, "_on_device", lambda dev: contextlib.nullcontext())
    return seen


def test_prefill_entry_points_accept_consistent_shapes(calls):
    Hq, Hkv, n, d = 4, 2, 1024, 128
    q, k = torch.zeros(Hq, n, d, dtype=bf), torch.zeros(Hkv, n, d, dtype=bf)
    bi, bc = dsa.sparse_index_estimate(q, k, keep_ratio=0.1)
    assert bi.shape == (Hq, n // 64, 8) and bc.shape == (Hq, n // 64)
    dsa.block_sparse_attn_fwd(q, k, k, bi, bc)
    res = dsa.vertical_slash_index(q, k, 100, 64)
    dsa.vertical_slash_index(q, k, 100, 64, out=res)
    dsa.block_sparse_attn_fwd(q, k, k, res["block_idx"], res["block_cnt"], res["col_idx"], res["col_cnt"])
    assert calls == ["sparse_index_estimate", "block_sparse_attn_fwd", "vertical_slash_index",
                     "vertical_slash_index", "block_sparse_attn_fwd"]


def test_prefill_entry_points_reject_inconsistent_shapes(calls):
    Hq, Hkv, n, d = 4, 2, 1024, 128
    q, k = torch.zeros(Hq, n, d, dtype=bf), torch.zeros(Hkv, n, d, dtype=bf)
    with pytest.raises(ValueError):
        dsa.sparse_index_estimate(q, k, keep_ratio=0.1, pooled_k=torch.zeros(1, n // 64, d, dtype=f32))
    with pytest.raises(TypeError):
        dsa.sparse_index_estimate(q, k, keep_ratio=0.1, block_idx=torch.zeros(Hq, 16, 8, dtype=torch.int64))
    bi, bc = torch.zeros(Hq, 16, 8, dtype=i32), torch.zeros(Hq, 16, dtype=i32)
    with pytest.raises(ValueError):
        dsa.block_sparse_attn_fwd(q, k, k[:, :512], bi, bc)                 # v shorter than k
    with pytest.raises(ValueError):
        dsa.block_sparse_attn_fwd(q, k, k, bi[:, :8], bc)                    # lists of another length
    with pytest.raises(ValueError):
        dsa.block_sparse_attn_fwd(q, k, k, bi, bc, torch.zeros(Hq, 16, 4, dtype=i32))   # columns without counts
    assert calls == []


def test_decode_entry_points_check_caches_and_clusters(calls):
    B, Hq, Hkv, S, d = 2, 4, 2, 4096, 128
    q, kc = torch.zeros(B, Hq, d, dtype=bf), torch.zeros(B, Hkv, S, d, dtype=bf)
    cent = dsa.pool_keys(kc)
    assert cent.shape == (B, Hkv, S // 64, d)
    dsa.sparse_decode_attn(q, kc, kc, cent, keep=8, return_sel=True)
    dsa.sparse_decode_attn_static(q, kc, kc, cent, keep=8)
    with pytest.raises(ValueError):
        dsa.sparse_decode_attn(q, kc, kc[:, :, :2048], cent, keep=8)
    C, n_ctx = 16, 4000
    cc = torch.zeros(B, Hkv, C, d, dtype=f32)
    off, tok = torch.zeros(B, Hkv, C + 1, dtype=i32), torch.zeros(B, Hkv, n_ctx, dtype=i32)
    kp, vp = dsa.cluster_pack_kv(kc, kc, tok, n_ctx)
    assert kp.shape == (B, Hkv, n_ctx, d)
    dsa.cluster_decode_attn(q, kc, kc, cc, off, tok, n_ctx, 4, packed=(kp, vp), return_sel=True)
    with pytest.raises(ValueError):
        dsa.cluster_decode_attn(q, kc, kc, cc, off[..., :-1], tok, n_ctx, 4)
    with pytest.raises(TypeError):
        dsa.cluster_pack_kv(kc, kc, tok.long(), n_ctx)
    assert calls == ["sparse_index_estimate", "sparse_decode_attn", "sparse_decode_attn_static", "cluster_pack_kv",
                     "cluster_decode_attn"]
