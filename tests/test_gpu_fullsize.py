"""Parity at the workloads' full sizes, in the launch configuration bench.py
times.  Where the fp64 oracle finishes in a minute or so the check is complete:
every row of every head's block index at 32K and 128K, attention on every
query block of every head at 32K, every head's vertical-slash sets and plan at
128K, every batch of the decode.  Where it does not (attention at 128K and 1M,
the 1M index) sampled rows and query blocks are checked one by one.  -m gpu."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
import dynamic_sparse_attention_03_b200 as dsa
from tests.parity import check_attention, check_block_index, f64, lists_from_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sample_rows(nqb, count, rng):
    if count == "all":
        return list(range(nqb))
    rows = {0, 1, 2, nqb - 1, nqb - 2}
    rows |= set(rng.choice(nqb, size=min(count, nqb), replace=False).tolist())
    return sorted(rows)


def _block_sparse_case(name, heads, n_rows, n_att):
    """heads: q-heads to check ("all" for every head); n_rows / n_att: index
    rows / attention query blocks per head, a sample size or "all"."""
    p = synth.CONFIGS[name]
    w = synth.make_prefill(name, device=DEV)
    Hq, n, d = w.q.shape
    grp = Hq // w.k.shape[0]
    nqb = n // 64
    bi, bc = dsa.sparse_index_estimate(w.q, w.k, k_fixed=p["k_fixed"], keep_ratio=p["keep_ratio"])
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    rng = np.random.default_rng(0)
    bi_h, bc_h = bi.cpu().numpy(), bc.cpu().numpy()
    heads = range(Hq) if heads == "all" else heads
    amb = 0
    for h in heads:
        g = h // grp
        q64 = f64(w.q[h:h + 1])
        k64 = f64(w.k[g:g + 1])
        v64 = f64(w.v[g:g + 1])
        rows = _sample_rows(nqb, n_rows, rng)
        _, info, _ = oracle.block_index(q64, k64, k_fixed=p["k_fixed"], keep_ratio=p["keep_ratio"],
                                        rows=None if n_rows == "all" else rows)
        got = {0: {i: bi_h[h, i, :bc_h[h, i]].astype(np.int64) for i in range(nqb)}}
        for i in rows:
            assert np.all(bi_h[h, i, bc_h[h, i]:] == -1)
        st = check_block_index(got, info, f"{name} h={h}")
        amb += st.get("ambiguous", 0)
        att_rows = _sample_rows(nqb, n_att, rng)
        ref = oracle.sparse_attention(q64, k64, v64, got, None, 1 / math.sqrt(d), items=[(0, qb) for qb in att_rows])
        ref = {(h, qb): val for (_, qb), val in ref.items()}
        check_attention(o, ref, f"{name} h={h}")
    print(f"{name}: index rows with an accepted near tie: {amb}")
    return w, bi, bc


def test_llama_32k_block_sparse():
    """Every index row of every head, and attention on every query block."""
    _block_sparse_case("llama3-8b-32k-bs10", heads="all", n_rows="all", n_att="all")


def test_llama_128k_block_sparse():
    """Every index row of every head; attention on sampled query blocks."""
    _block_sparse_case("llama3-8b-128k-bs10", heads="all", n_rows="all", n_att=6)


def test_llama_1m_block_sparse():
    _block_sparse_case("llama3-8b-1m-bs2", heads=[9, 22], n_rows=48, n_att=6)


def test_llama_128k_vertical_slash():
    name = "llama3-8b-128k-vs"
    p = synth.CONFIGS[name]
    w = synth.make_prefill(name, device=DEV)
    Hq, n, d = w.q.shape
    grp = Hq // w.k.shape[0]
    scale = 1 / math.sqrt(d)
    res = dsa.vertical_slash_index(w.q, w.k, p["n_vert"], p["n_slash"])
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, res["block_idx"], res["block_cnt"], res["col_idx"],
                                  res["col_cnt"])
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    vi, so = res["vert_idx"].cpu().numpy(), res["slash_off"].cpu().numpy()
    gb = lists_from_gpu(res["block_idx"], res["block_cnt"])
    gc = lists_from_gpu(res["col_idx"], res["col_cnt"])
    rng = np.random.default_rng(1)
    amb = 0
    for h in range(Hq):
        g = h // grp
        q64, k64, v64 = f64(w.q[h:h + 1]), f64(w.k[g:g + 1]), f64(w.v[g:g + 1])
        ref = oracle.vs_index(q64, k64, 64, p["n_vert"], p["n_slash"], scale)[0]
        assert abs(ref["vert"].sum() - 64) < 1e-8 and abs(ref["slash"].sum() - 64) < 1e-8
        cand, sc, e = ref["vert_info"]
        st = oracle.compare_index_sets(vi[h], np.arange(64), cand, sc, e)
        assert not st.startswith("MISMATCH"), ("vert", h, st)
        amb += st == "ambiguous"
        cand, sc, e = ref["slash_info"]
        st = oracle.compare_index_sets(so[h], [0], cand, sc, e)
        assert not st.startswith("MISMATCH"), ("slash", h, st)
        amb += st == "ambiguous"
        plan = oracle.vs_plan(vi[h], so[h], n)
        for qb in range(n // 64):
            assert gb[h][qb].tolist() == plan[qb][0].tolist(), (h, qb)
            assert gc[h][qb].tolist() == plan[qb][1].tolist(), (h, qb)
        if h not in (2, 29):
            continue
        rows = _sample_rows(n // 64, 4, rng)
        lists = {0: gb[h]}
        cols = {0: gc[h]}
        ra = oracle.sparse_attention(q64, k64, v64, lists, cols, scale, items=[(0, qb) for qb in rows])
        check_attention(o, {(h, qb): val for (_, qb), val in ra.items()}, f"vs h={h}")
    print("vertical-slash sets with an accepted near tie:", amb, "of", 2 * Hq)


def test_decode_b16_128k():
    w = synth.make_decode("decode-b16-128k", device=DEV)
    p = w.params
    B, Hq, d = w.q.shape
    Hkv, S = w.k_cache.shape[1], w.k_cache.shape[2]
    nb = S // 64
    cent = dsa.pool_keys(w.k_cache)
    o, si, sc = dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent, keep=p["keep"], return_sel=True)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    si_h, sc_h = si.cpu().numpy(), sc.cpu().numpy()
    amb = 0
    for b in range(B):
        q64 = f64(w.q[b:b + 1])
        k64 = f64(w.k_cache[b:b + 1])
        v64 = f64(w.v_cache[b:b + 1])
        ref_cent = oracle.decode_centroids(k64)
        np.testing.assert_allclose(cent[b:b + 1].cpu().numpy(), ref_cent, atol=1e-5, rtol=1e-5)
        _, info = oracle.decode_select(q64, ref_cent, p["keep"], 1)
        gsel = {}
        for (_, h), (cand, s, e) in info.items():
            got = si_h[b, h, :sc_h[b, h]]
            st = oracle.compare_index_sets(got, [nb - 1], cand, s, e)
            assert not st.startswith("MISMATCH"), (b, h, st)
            amb += st == "ambiguous"
            gsel[(0, h)] = got.astype(np.int64)
        ref_o = oracle.decode_attention(q64, k64, v64, gsel, 1 / math.sqrt(d))
        oh = f64(o[b:b + 1])
        errs = [np.abs(oh[0, h] - O) for (_, h), O in ref_o.items()]
        assert max(float(e.max()) for e in errs) <= 2e-2
        assert float(np.mean([e.mean() for e in errs])) <= 2e-3
    print("decode (b, h) rows with an accepted near tie:", amb, "of", B * Hq)
