"""GPU parity of the K-means cluster build and the cluster-ranked decode
(Squeezed Attention page, "技术方案": offline K-means over the fixed context's
keys; online, the query ranks the centroids, the top clusters are kept and
attention runs over their keys).  -m gpu.

Floating point decides the assignment (an argmin) and the cluster ranking:
the kernels decide in fp32, the oracle in fp64, so a key whose two nearest
centroids are within 1e-4 (relative) of each other may go to either; every
other key must match exactly.  The cluster -> key map is integer work and must
match exactly given the assignment.  Attention outputs are compared with the
oracle fed the CUDA path's clusters and selection (max abs 2e-2, mean abs 2e-3).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
import dynamic_sparse_attention_03_b200 as dsa
from tests.parity import f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIE_REL = 1e-4


def _check_assign(keys, cent, got):
    """got: CUDA assignment; keys, cent fp64.  Exact except near ties; returns
    the number of ambiguous keys."""
    d2 = (keys * keys).sum(1)[:, None] + (cent * cent).sum(1)[None, :] - 2.0 * (keys @ cent.T)
    want = np.argmin(d2, axis=1)
    amb = 0
    for t in np.nonzero(got != want)[0]:
        dg, dw = d2[t, got[t]], d2[t, want[t]]
        assert dg - dw <= TIE_REL * max(abs(dw), 1e-12), (t, got[t], want[t], dg, dw)
        amb += 1
    return amb


@pytest.mark.parametrize("B,Hkv,S,d,n_ctx,C", [(1, 2, 2048, 128, 1984, 32), (2, 1, 1536, 64, 1536, 24),
                                               (1, 1, 4096, 128, 4000, 61)])
def test_kmeans_round_matches_oracle(B, Hkv, S, d, n_ctx, C):
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hkv, Hkv=Hkv, d=d, seed=S + C)
    cent, assign, off, tok = dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=1)
    torch.cuda.synchronize()
    k64 = f64(w.k_cache)
    cent_h, as_h, off_h, tok_h = (x.cpu().numpy() for x in (cent, assign, off, tok))
    amb = 0
    for b in range(B):
        for g in range(Hkv):
            keys = k64[b, g, :n_ctx]
            init = oracle.segment_means(keys, C)
            amb += _check_assign(keys, init, as_h[b, g].astype(np.int64))
            o_ref, t_ref = oracle.cluster_csr(as_h[b, g].astype(np.int64), C)
            assert off_h[b, g].tolist() == o_ref.tolist()
            assert tok_h[b, g].tolist() == t_ref.tolist()
            upd = oracle.kmeans_update(keys, as_h[b, g].astype(np.int64), init)
            np.testing.assert_allclose(cent_h[b, g], upd, rtol=1e-5, atol=1e-6)
    print("ambiguous keys", amb)
    assert amb <= max(2, n_ctx * B * Hkv // 2000)


def test_kmeans_blobs_match_oracle_over_rounds():
    """Well separated blobs: no near ties, so several Lloyd rounds must give the
    oracle's assignment exactly, and centroids within fp32 rounding."""
    r = np.random.default_rng(7)
    C, d, S = 16, 128, 1024
    centers = r.standard_normal((C, d)) * 4.0
    lab = r.integers(0, C, size=S)
    keys = centers[lab] + 0.05 * r.standard_normal((S, d))
    kc = torch.tensor(keys, dtype=torch.float32).to(torch.bfloat16).reshape(1, 1, S, d).contiguous().to(DEV)
    cent, assign, off, tok = dsa.kmeans_clusters(kc, S, C, iters=6)
    torch.cuda.synchronize()
    k64 = f64(kc)[0, 0]
    rc, ra = oracle.kmeans(k64, C, 6)
    assert assign.cpu().numpy()[0, 0].tolist() == ra.tolist()
    np.testing.assert_allclose(cent.cpu().numpy()[0, 0], rc, rtol=1e-5, atol=1e-5)
    o_ref, t_ref = oracle.cluster_csr(ra, C)
    assert off.cpu().numpy()[0, 0].tolist() == o_ref.tolist()
    assert tok.cpu().numpy()[0, 0].tolist() == t_ref.tolist()


def test_kmeans_rounds_are_self_consistent():
    """Several rounds on cache-like data (where near ties may steer the fp32 and
    fp64 runs apart after the first round): the map matches the assignment,
    every non-empty cluster's centroid is the mean of its keys, and the
    objective is no larger than at the segment-mean start (Lloyd's rounds never
    increase it)."""
    B, Hkv, S, d, n_ctx, C = 1, 2, 4096, 128, 4032, 64
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hkv, Hkv=Hkv, d=d, seed=99)
    cent, assign, off, tok = dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=4)
    torch.cuda.synchronize()
    k64 = f64(w.k_cache)
    for g in range(Hkv):
        keys = k64[0, g, :n_ctx]
        a = assign.cpu().numpy()[0, g].astype(np.int64)
        o_ref, t_ref = oracle.cluster_csr(a, C)
        assert off.cpu().numpy()[0, g].tolist() == o_ref.tolist()
        assert tok.cpu().numpy()[0, g].tolist() == t_ref.tolist()
        cg = cent.cpu().numpy()[0, g].astype(np.float64)
        for c in range(C):
            members = keys[a == c]
            if len(members):
                np.testing.assert_allclose(cg[c], members.mean(0), rtol=1e-5, atol=1e-5)
        start = oracle.segment_means(keys, C)
        obj0 = oracle.kmeans_objective(keys, start, oracle.kmeans_assign(keys, start))
        assert oracle.kmeans_objective(keys, cg, a) <= obj0 * (1 + 1e-6)


@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,S,d,n_ctx,C,keep", [(2, 8, 2, 4096, 128, 4032, 64, 16),
                                                      (1, 4, 4, 2048, 64, 2048, 32, 8),
                                                      (1, 8, 1, 3072, 128, 2944, 48, 48),
                                                      (1, 4, 1, 16384, 128, 16320, 256, 192)])
def test_cluster_decode_matches_oracle(B, Hq, Hkv, S, d, n_ctx, C, keep, packed):
    """Both forms of the decode: rows gathered by token id, and rows streamed
    from the cluster-ordered copy.  The last case keeps about 12K rows of one
    (batch, KV head), more than one 4096-row chunk of the kernel, so the
    per-chunk partial softmax states are merged."""
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=C + keep)
    cent, assign, off, tok = dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=2)
    pk = dsa.cluster_pack_kv(w.k_cache, w.v_cache, tok, n_ctx) if packed else None
    o, si, sc = dsa.cluster_decode_attn(w.q, w.k_cache, w.v_cache, cent, off, tok, n_ctx, keep, return_sel=True,
                                        packed=pk)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    q64, k64, v64 = f64(w.q), f64(w.k_cache), f64(w.v_cache)
    cent64, off_h, tok_h = cent.cpu().numpy().astype(np.float64), off.cpu().numpy(), tok.cpu().numpy()
    sel, info = oracle.cluster_select(q64, cent64, off_h.astype(np.int64), keep)
    si_h, sc_h = si.cpu().numpy(), sc.cpu().numpy()
    gsel = {}
    for (b, h), (cand, s, e) in info.items():
        got = si_h[b, h, :sc_h[b, h]]
        assert np.all(si_h[b, h, sc_h[b, h]:] == -1)
        st = oracle.compare_index_sets(got, [], cand, s, e)
        assert not st.startswith("MISMATCH"), (b, h, st)
        gsel[(b, h)] = got.astype(np.int64)
    ref = oracle.cluster_decode_attention(q64, k64, v64, gsel, off_h.astype(np.int64), tok_h.astype(np.int64), n_ctx,
                                          1 / math.sqrt(d))
    oh = f64(o)
    errs = [np.abs(oh[b, h] - O) for (b, h), O in ref.items()]
    mx = max(float(e.max()) for e in errs)
    mean = float(np.mean([e.mean() for e in errs]))
    print("cluster decode", mx, mean)
    assert mx <= 2e-2 and mean <= 2e-3


def test_cluster_decode_keep_all_equals_dense():
    """Keeping every cluster attends every key: dense single-query attention."""
    B, Hq, Hkv, S, d, n_ctx, C = 2, 8, 2, 2048, 128, 1920, 40
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=5)
    cent, _, off, tok = dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=2)
    o = dsa.cluster_decode_attn(w.q, w.k_cache, w.v_cache, cent, off, tok, n_ctx, keep=C)
    kk = w.k_cache.repeat_interleave(Hq // Hkv, 1).float()
    vv = w.v_cache.repeat_interleave(Hq // Hkv, 1).float()
    ref = torch.nn.functional.scaled_dot_product_attention(w.q.float()[:, :, None], kk, vv)[:, :, 0]
    err = (o.float() - ref).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3


def test_cluster_pack_kv_is_the_cluster_order_gather():
    B, Hkv, S, d, n_ctx, C = 2, 2, 2048, 128, 1984, 32
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hkv, Hkv=Hkv, d=d, seed=11)
    _, _, _, tok = dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=2)
    kp, vp = dsa.cluster_pack_kv(w.k_cache, w.v_cache, tok, n_ctx)
    idx = tok.long()[..., None].expand(B, Hkv, n_ctx, d)
    assert torch.equal(kp, torch.gather(w.k_cache, 2, idx))
    assert torch.equal(vp, torch.gather(w.v_cache, 2, idx))


@pytest.mark.parametrize("B,Hq,Hkv,S,d,n_ctx,C,keep", [(2, 8, 2, 4096, 128, 4032, 64, 16),
                                                      (1, 4, 4, 2048, 64, 2048, 32, 8),
                                                      (1, 8, 1, 3072, 128, 2944, 48, 48)])
def test_packed_cluster_decode_equals_gathered(B, Hq, Hkv, S, d, n_ctx, C, keep):
    """The cluster-ordered copy holds the same rows in the same order as the
    token gather: the same clusters are kept, and the outputs differ only by
    the fp32 summation order of the two kernels (each is checked against the
    oracle in test_cluster_decode_matches_oracle)."""
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=C + keep + 1)
    cent, _, off, tok = dsa.kmeans_clusters(w.k_cache, n_ctx, C, iters=2)
    packed = dsa.cluster_pack_kv(w.k_cache, w.v_cache, tok, n_ctx)
    o1, si1, sc1 = dsa.cluster_decode_attn(w.q, w.k_cache, w.v_cache, cent, off, tok, n_ctx, keep, return_sel=True)
    o2, si2, sc2 = dsa.cluster_decode_attn(w.q, w.k_cache, w.v_cache, cent, off, tok, n_ctx, keep, return_sel=True,
                                           packed=packed)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    assert torch.equal(si1, si2) and torch.equal(sc1, sc2)
    err = (o1.float() - o2.float()).abs()
    assert err.max().item() <= 1e-2 and err.mean().item() <= 1e-3


def test_cluster_abi_rejects_bad_arguments():
    kc = torch.zeros((1, 1, 256, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(dsa.DSAError):
        dsa.kmeans_clusters(kc, 256, 300, iters=1)      # more clusters than keys
    with pytest.raises(dsa.DSAError):
        dsa.kmeans_clusters(kc, 300, 8, iters=1)        # context past the cache
    with pytest.raises(dsa.DSAError):
        dsa.kmeans_clusters(kc, 256, 8, iters=0)
    tok = torch.zeros((1, 1, 300), dtype=torch.int32, device=DEV)
    with pytest.raises(dsa.DSAError):
        dsa.cluster_pack_kv(kc, kc, tok, 300)          # context past the cache (the library's check)
    with pytest.raises(ValueError):
        dsa.cluster_pack_kv(kc, kc, tok[..., :200], 256)   # tokens of the wrong length (the binding's check)
