"""Run-to-run determinism of every entry point (-m gpu).

No kernel here relies on the order in which concurrent threads or CTAs finish:
the persistent top-k kernel takes its tiles from an atomic counter, but every
tile's result is written by that tile alone; sums run in a fixed order.  So two
calls on the same inputs must give bit-identical index lists, outputs, log-sum-
exps and decode selections.  This stands in for a race detector on this pool:
a race on shared or global memory would show up as a difference between runs.
"""

import pytest
import torch

import synth
import dynamic_sparse_attention_03_b200 as dsa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _twice(fn):
    a = fn()
    b = fn()
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    return a, b


def _same(a, b):
    if isinstance(a, dict):
        assert a.keys() == b.keys()
        for key in a:
            assert torch.equal(a[key], b[key]), key
        return
    if isinstance(a, (tuple, list)):
        for x, y in zip(a, b):
            _same(x, y)
        return
    assert torch.equal(a, b)


@pytest.mark.parametrize("n,Hq,Hkv,rho", [(8192, 8, 2, 0.10), (16384, 4, 1, 0.3)])
def test_block_index_and_attention_are_deterministic(n, Hq, Hkv, rho):
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=128, seed=n + Hq)
    idx = _twice(lambda: tuple(t.clone() for t in dsa.sparse_index_estimate(w.q, w.k, keep_ratio=rho)))
    _same(*idx)
    bi, bc = idx[0]
    att = _twice(lambda: dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, return_lse=True))
    _same(*att)


def test_vertical_slash_is_deterministic():
    w = synth.make_prefill("llama3-8b-128k-vs", device=DEV, n=8192, Hq=8, Hkv=2)
    res = _twice(lambda: {k: v.clone() for k, v in dsa.vertical_slash_index(w.q, w.k, 256, 512).items()})
    _same(*res)
    r = res[0]
    att = _twice(lambda: dsa.block_sparse_attn_fwd(w.q, w.k, w.v, r["block_idx"], r["block_cnt"], r["col_idx"],
                                                   r["col_cnt"], return_lse=True))
    _same(*att)


def test_decode_is_deterministic():
    w = synth.make_decode("decode-b16-128k", device=DEV, B=4, S=16384, seed=4)
    cent = _twice(lambda: dsa.pool_keys(w.k_cache))
    _same(*cent)
    out = _twice(lambda: dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent[0], keep=64, return_sel=True))
    _same(*out)


def test_kmeans_and_cluster_decode_are_deterministic():
    w = synth.make_decode("decode-b16-128k", device=DEV, B=1, S=8192, Hq=8, Hkv=2, seed=6)
    n_ctx, C = 8128, 128
    cl = _twice(lambda: dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=2))
    _same(*cl)
    cent, _, off, tok = cl[0]
    packed = dsa.cluster_pack_kv(w.k_cache, w.v_cache, tok, n_ctx)
    for pk in (None, packed):
        out = _twice(lambda: dsa.cluster_decode_attn(w.q, w.k_cache, w.v_cache, cent, off, tok, n_ctx, 48,
                                                     return_sel=True, packed=pk))
        _same(*out)
