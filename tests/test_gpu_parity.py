"""CUDA path (through the C ABI) against the fp64 oracle on small seeded cases
that still span several tiles and ragged tails.  Run with -m gpu on a B200."""

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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dsa.load_library()
    yield
    torch.cuda.synchronize()
    assert dsa.get_status() == 0


def _ref_attention(q, k, v, lists, cols, scale, items):
    return oracle.sparse_attention(f64(q), f64(k), f64(v), lists, cols, scale, items=items)


# ---------------------------------------------------------------- tiny workload

def test_tiny_index_matches_golden_and_oracle():
    w = synth.make_prefill("tiny-1h-1k-d64", device="cpu")
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    bi, bc = dsa.sparse_index_estimate(q, k, k_fixed=4)
    got = lists_from_gpu(bi, bc)
    lists, info, _ = oracle.block_index(f64(w.q), f64(w.k), k_fixed=4)
    check_block_index(got, info, "tiny")
    from tests.test_golden import read_lists
    want = read_lists("tiny_block_index.txt")
    assert {i: got[0][i].tolist() for i in got[0]} == want


def test_tiny_attention_matches_oracle():
    w = synth.make_prefill("tiny-1h-1k-d64", device="cpu")
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    bi, bc = dsa.sparse_index_estimate(q, k, k_fixed=4)
    o, lse = dsa.block_sparse_attn_fwd(q, k, v, bi, bc, return_lse=True)
    torch.cuda.synchronize()
    got = lists_from_gpu(bi, bc)
    ref = _ref_attention(w.q, w.k, w.v, got, None, 1 / 8.0, None)
    check_attention(o, ref, "tiny")
    lse_h = lse.cpu().numpy()
    for (h, qb), (_, L) in ref.items():
        np.testing.assert_allclose(lse_h[h, qb * 64:(qb + 1) * 64], L, atol=2e-3, rtol=1e-4)


# ---------------------------------------------------------------- block-sparse, GQA

# GQA groups of 4, 1 and 3 q-heads per KV head, and 8 and 5 (two work items
# per KV head and query block: four heads each, or four and one)
@pytest.mark.parametrize("n,d,Hq,Hkv,rho", [(4096, 128, 8, 2, 0.10), (2048, 64, 4, 4, 0.25), (3072, 128, 6, 2, 0.5),
                                            (2048, 128, 16, 2, 0.2), (2048, 64, 10, 2, 0.3),
                                            (9024, 128, 4, 1, 0.15)])   # 141 query blocks: ragged row tile and key chunk
def test_block_index_and_attention(n, d, Hq, Hkv, rho):
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=7 + n)
    bi, bc = dsa.sparse_index_estimate(w.q, w.k, keep_ratio=rho)
    got = lists_from_gpu(bi, bc)
    lists, info, _ = oracle.block_index(f64(w.q), f64(w.k), keep_ratio=rho)
    check_block_index(got, info, f"n={n}")
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc)
    torch.cuda.synchronize()
    nqb = n // 64
    items = [(h, qb) for h in range(Hq) for qb in range(nqb)]
    ref = _ref_attention(w.q, w.k, w.v, got, None, 1 / math.sqrt(d), items)
    check_attention(o, ref, f"n={n} d={d}")


@pytest.mark.parametrize("q_scale,k_scale", [(2.0 ** 12, 2.0 ** -12), (1000.0, 0.001), (0.003, 0.02), (37.0, 1.0)])
def test_block_index_input_scales(q_scale, k_scale):
    """The index operands are FP16 splits of the pooled means after a power-of-
    two scale per query block and per KV head, so the index must not depend on
    the inputs' magnitude: large and small Q and K give the oracle's sets, and
    power-of-two scales give exactly the unscaled lists."""
    n, d, Hq, Hkv, rho = 4096, 128, 8, 2, 0.10
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=77)
    qs = (w.q.float() * q_scale).to(torch.bfloat16)
    ks = (w.k.float() * k_scale).to(torch.bfloat16)
    bi, bc = dsa.sparse_index_estimate(qs, ks, keep_ratio=rho)
    got = lists_from_gpu(bi, bc)
    _, info, _ = oracle.block_index(f64(qs), f64(ks), keep_ratio=rho)
    check_block_index(got, info, f"scales {q_scale}, {k_scale}")
    if math.log2(q_scale).is_integer() and math.log2(k_scale).is_integer():
        bi0, bc0 = dsa.sparse_index_estimate(w.q, w.k, keep_ratio=rho)
        assert torch.equal(bi, bi0) and torch.equal(bc, bc0)


@pytest.mark.parametrize("where,p", [("sink", 8), ("sink", 12), ("sink", 16), ("sink", 20), ("sink", 24),
                                     ("candidate", 8), ("candidate", 12), ("candidate", 16), ("candidate", 20)])
def test_block_index_outlier_key_block(where, p):
    """One key block 2^p times larger than the rest, as attention-sink keys
    often are.  The FP16 split of the pooled keys is scaled once per KV head,
    so an outlier that set that scale would push every other block's low half
    toward the subnormal range; the forced sink block is therefore left out of
    the scale (its own score is never ranked).  The rows keep 30% of their
    candidates, so the boundary falls inside the Gaussian bulk where scores
    are close, and 512 query blocks make long rows."""
    n, d, Hq, Hkv, rho = 32768, 128, 2, 1, 0.3
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=78)
    blk = 0 if where == "sink" else 37
    k = w.k.float()
    k[:, blk * 64:(blk + 1) * 64] *= 2.0 ** p
    k = k.to(torch.bfloat16).contiguous()
    bi, bc = dsa.sparse_index_estimate(w.q, k, keep_ratio=rho)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    got = lists_from_gpu(bi, bc)
    _, info, _ = oracle.block_index(f64(w.q), f64(k), keep_ratio=rho)
    check_block_index(got, info, f"outlier {where} x2^{p}")


def test_block_index_exact_ties_take_the_lower_blocks():
    """Key blocks drawn from four repeated vectors: every row's scores take a
    few values, each shared by many blocks, so the e-th largest sits inside a
    large group of exactly equal scores (equal in fp32 on the GPU and in fp64
    in the oracle).  The selection's window then holds more candidates than
    its buffer and the exact fallback passes run (value histogram, radix
    passes on the keys, threshold sweep); the ties must go to the lower
    blocks, so every row matches the oracle exactly."""
    n, d, Hq, Hkv, rho = 32768, 128, 4, 1, 0.10
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=5)
    nqb = n // 64
    g = torch.Generator(device="cpu").manual_seed(123)
    types = torch.randn((4, d), generator=g).to(torch.bfloat16)
    pick = torch.randint(0, 4, (nqb,), generator=g)
    k = types[pick].repeat_interleave(64, dim=0).reshape(1, n, d).contiguous().to(DEV)
    bi, bc = dsa.sparse_index_estimate(w.q, k, keep_ratio=rho)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    got = lists_from_gpu(bi, bc)
    _, info, _ = oracle.block_index(f64(w.q), f64(k), keep_ratio=rho)
    stats = check_block_index(got, info, "exact ties")
    assert stats.get("ambiguous", 0) == 0, stats


def _random_lists(rng, Hq, nqb, kcap, p_keep, with_cols, ccap=0, empty_rows=()):
    bi = -np.ones((Hq, nqb, kcap), np.int32)
    bc = np.zeros((Hq, nqb), np.int32)
    ci = -np.ones((Hq, nqb, max(ccap, 1)), np.int32)
    cc = np.zeros((Hq, nqb), np.int32)
    for h in range(Hq):
        for qb in range(nqb):
            if (h, qb) in empty_rows:
                continue
            sel = [b for b in range(qb + 1) if rng.random() < p_keep or b == qb]
            sel = sel[-kcap:]
            bi[h, qb, :len(sel)] = sel
            bc[h, qb] = len(sel)
            if with_cols:
                pool = [j for j in range(64 * qb) if (j // 64) not in sel]
                m = min(len(pool), int(rng.integers(0, ccap + 1)))
                cols = sorted(rng.choice(pool, size=m, replace=False).tolist()) if m else []
                ci[h, qb, :m] = cols
                cc[h, qb] = m
    return bi, bc, ci, cc


@pytest.mark.parametrize("with_cols", [False, True])
def test_attention_ragged_lists(with_cols):
    """Random per-head lists (odd and even counts, heads of a pair disagreeing,
    empty rows, column tiles with partial fill) against the oracle."""
    rng = np.random.default_rng(11)
    Hq, Hkv, n, d = 4, 2, 2048, 128
    nqb = n // 64
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=99)
    empty = {(0, 5), (1, 5), (3, 0)}
    bi, bc, ci, cc = _random_lists(rng, Hq, nqb, 12, 0.3, with_cols, ccap=150, empty_rows=empty)
    t = lambda a: torch.from_numpy(a).to(DEV)
    if with_cols:
        o, lse = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, t(bi), t(bc), t(ci), t(cc), return_lse=True)
    else:
        o, lse = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, t(bi), t(bc), return_lse=True)
    torch.cuda.synchronize()
    lists = {h: {qb: bi[h, qb, :bc[h, qb]].astype(np.int64) for qb in range(nqb)} for h in range(Hq)}
    cols = ({h: {qb: ci[h, qb, :cc[h, qb]].astype(np.int64) for qb in range(nqb)} for h in range(Hq)}
            if with_cols else None)
    items = [(h, qb) for h in range(Hq) for qb in range(nqb) if (h, qb) not in empty]
    ref = _ref_attention(w.q, w.k, w.v, lists, cols, 1 / math.sqrt(d), items)
    check_attention(o, ref, f"ragged cols={with_cols}")
    for (h, qb) in empty:
        assert torch.all(o[h, qb * 64:(qb + 1) * 64] == 0)
        assert torch.all(torch.isinf(lse[h, qb * 64:(qb + 1) * 64]))


def test_attention_all_blocks_equals_dense_sdpa():
    """Every causal block selected: equals dense causal attention (torch SDPA on
    the GPU as an independent check besides the oracle)."""
    Hq, Hkv, n, d = 8, 2, 4096, 128
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=5)
    nqb = n // 64
    bi = torch.arange(nqb, device=DEV, dtype=torch.int32)[None, None, :].expand(Hq, nqb, nqb).contiguous()
    bi = torch.where(bi <= torch.arange(nqb, device=DEV)[None, :, None], bi, torch.full_like(bi, -1))
    bc = (torch.arange(nqb, device=DEV, dtype=torch.int32) + 1)[None, :].expand(Hq, nqb).contiguous()
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc)
    kk = w.k.repeat_interleave(Hq // Hkv, 0)
    vv = w.v.repeat_interleave(Hq // Hkv, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(w.q[None].float(), kk[None].float(), vv[None].float(),
                                                           is_causal=True)[0]
    err = (o.float() - ref).abs()
    print("dense vs sdpa", err.max().item(), err.mean().item())
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3


def test_attention_invariants():
    """V = 1 gives O = 1; Q = 0 gives the mean of V over the attended set."""
    Hq, Hkv, n, d = 4, 2, 1024, 128
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=3)
    bi, bc = dsa.sparse_index_estimate(w.q, w.k, keep_ratio=0.3)
    o1 = dsa.block_sparse_attn_fwd(w.q, w.k, torch.ones_like(w.v), bi, bc)
    assert (o1.float() - 1).abs().max().item() == 0.0
    o0 = dsa.block_sparse_attn_fwd(torch.zeros_like(w.q), w.k, w.v, bi, bc)
    torch.cuda.synchronize()
    got = lists_from_gpu(bi, bc)
    v64 = f64(w.v)
    o0h = f64(o0)
    for h in range(Hq):
        for qb in range(n // 64):
            for r in (0, 31, 63):
                i = qb * 64 + r
                keys = [j for b in got[h][qb] for j in range(b * 64, b * 64 + 64) if j <= i]
                mean = v64[h // 2, keys].mean(axis=0)
                assert np.abs(o0h[h, i] - mean).max() < 1e-2


# ---------------------------------------------------------------- vertical-slash

@pytest.mark.parametrize("n,Hq,Hkv", [(2048, 4, 2), (1984, 4, 2), (2048, 16, 2)])
def test_vs_index_plan_and_attention_small(n, Hq, Hkv):
    d = 128
    w = synth.make_prefill("llama3-8b-128k-vs", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=21)
    n_vert, n_slash = 200, 300
    res = dsa.vertical_slash_index(w.q, w.k, n_vert, n_slash)
    torch.cuda.synchronize()
    scale = 1 / math.sqrt(d)
    ref = oracle.vs_index(f64(w.q), f64(w.k), 64, n_vert, n_slash, scale)
    vi = res["vert_idx"].cpu().numpy()
    so = res["slash_off"].cpu().numpy()
    stats = {}
    for h in range(Hq):
        r = ref[h]
        cand, sc, e = r["vert_info"]
        st = oracle.compare_index_sets(vi[h], np.arange(64), cand, sc, e)
        assert not st.startswith("MISMATCH"), (h, "vert", st)
        stats[(h, "v")] = st
        cand, sc, e = r["slash_info"]
        st = oracle.compare_index_sets(so[h], [0], cand, sc, e)
        assert not st.startswith("MISMATCH"), (h, "slash", st)
        stats[(h, "s")] = st
        # the scores themselves
        np.testing.assert_allclose(sum(r["vert"]), 64, atol=1e-9)
    print("vs index", stats)
    # plan: exactly the oracle's plan for the kept sets the GPU chose
    gb = lists_from_gpu(res["block_idx"], res["block_cnt"])
    gc = lists_from_gpu(res["col_idx"], res["col_cnt"])
    for h in range(Hq):
        plan = oracle.vs_plan(vi[h], so[h], n)
        for qb in range(n // 64):
            assert gb[h][qb].tolist() == plan[qb][0].tolist(), (h, qb)
            assert gc[h][qb].tolist() == plan[qb][1].tolist(), (h, qb)
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, res["block_idx"], res["block_cnt"], res["col_idx"], res["col_cnt"])
    torch.cuda.synchronize()
    items = [(h, qb) for h in range(Hq) for qb in range(n // 64)]
    refo = _ref_attention(w.q, w.k, w.v, gb, gc, scale, items)
    check_attention(o, refo, "vs small")


def test_vs_index_exact_ties_take_the_lower_columns():
    """Zero keys make every logit 0, so each of the last 64 rows spreads its
    weight evenly over its causal keys and every column before those rows gets
    the same sum, bit for bit (the same values added in the same order).  The
    kept columns must then be the lowest ones (MInference 1.0 page, method
    section: the top vertical lines; ties to the lower index), also when the
    kept count spans several of the slices the top-k ranks apart first."""
    n, Hq, Hkv, d = 8192, 2, 1, 128
    w = synth.make_prefill("llama3-8b-128k-vs", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=23)
    k0 = torch.zeros_like(w.k)
    for n_vert in (700, 2500):
        res = dsa.vertical_slash_index(w.q, k0, n_vert, 64)
        torch.cuda.synchronize()
        vi = res["vert_idx"].cpu().numpy()
        for h in range(Hq):
            assert vi[h].tolist() == list(range(n_vert)), (n_vert, h)


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("B,Hq,Hkv,S,d,keep", [(2, 8, 2, 8192, 128, 32), (3, 4, 4, 4096, 64, 10), (1, 8, 1, 2048, 128, 100)])
def test_decode_matches_oracle(B, Hq, Hkv, S, d, keep):
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=S + keep)
    cent = dsa.pool_keys(w.k_cache)
    o, si, sc = dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent, keep=keep, return_sel=True)
    torch.cuda.synchronize()
    q64, k64, v64 = f64(w.q), f64(w.k_cache), f64(w.v_cache)
    ref_cent = oracle.decode_centroids(k64)
    np.testing.assert_allclose(cent.cpu().numpy(), ref_cent, atol=1e-5, rtol=1e-5)
    sel, info = oracle.decode_select(q64, ref_cent, keep, 1)
    nb = S // 64
    si_h, sc_h = si.cpu().numpy(), sc.cpu().numpy()
    gsel = {}
    for (b, h), (cand, s, e) in info.items():
        got = si_h[b, h, :sc_h[b, h]]
        assert np.all(si_h[b, h, sc_h[b, h]:] == -1)
        st = oracle.compare_index_sets(got, [nb - 1], cand, s, e)
        assert not st.startswith("MISMATCH"), (b, h, st)
        gsel[(b, h)] = got.astype(np.int64)
    ref_o = oracle.decode_attention(q64, k64, v64, gsel, 1 / math.sqrt(d))
    oh = f64(o)
    errs = [np.abs(oh[b, h] - O) for (b, h), O in ref_o.items()]
    mx = max(float(e.max()) for e in errs)
    mean = float(np.mean([e.mean() for e in errs]))
    print("decode", mx, mean)
    assert mx <= 2e-2 and mean <= 2e-3


def test_decode_keep_all_equals_dense():
    B, Hq, Hkv, S, d = 2, 8, 2, 4096, 128
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=1)
    cent = dsa.pool_keys(w.k_cache)
    o = dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent, keep=S // 64)
    kk = w.k_cache.repeat_interleave(Hq // Hkv, 1).float()
    vv = w.v_cache.repeat_interleave(Hq // Hkv, 1).float()
    ref = torch.nn.functional.scaled_dot_product_attention(w.q.float()[:, :, None], kk, vv)[:, :, 0]
    err = (o.float() - ref).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3


# ---------------------------------------------------------------- errors (host-side checks, no launch)

def test_abi_rejects_bad_arguments():
    q = torch.zeros((2, 1000, 128), dtype=torch.bfloat16, device=DEV)   # n % 64 != 0
    with pytest.raises(dsa.DSAError) as ei:
        dsa.sparse_index_estimate(q, q, keep_ratio=0.1, kcap=8)
    assert ei.value.rc in (-1, -2)
    q = torch.zeros((2, 1024, 96), dtype=torch.bfloat16, device=DEV)    # d = 96
    with pytest.raises(dsa.DSAError) as ei:
        dsa.sparse_index_estimate(q, q, keep_ratio=0.1, kcap=8)
    assert ei.value.rc == -2
    q = torch.zeros((2, 1024, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(dsa.DSAError) as ei:                              # kcap too small
        dsa.sparse_index_estimate(q, q, keep_ratio=0.5, kcap=3)
    assert ei.value.rc == -3
    with pytest.raises(dsa.DSAError):                                     # both budgets
        dsa.sparse_index_estimate(q, q, k_fixed=4, keep_ratio=0.5, kcap=16)


def test_validation_mode_rejects_bad_lists(monkeypatch):
    monkeypatch.setenv("DSA_VALIDATE", "1")
    Hq, n, d = 2, 512, 64
    q = torch.randn((Hq, n, d), device=DEV).to(torch.bfloat16)
    nqb = n // 64
    bi = torch.full((Hq, nqb, 4), -1, dtype=torch.int32, device=DEV)
    bc = torch.ones((Hq, nqb), dtype=torch.int32, device=DEV)
    bi[:, :, 0] = torch.arange(nqb, device=DEV, dtype=torch.int32)
    dsa.block_sparse_attn_fwd(q, q, q, bi, bc)       # valid: diagonal only
    for bad in ("future", "unsorted", "count"):
        b2, c2 = bi.clone(), bc.clone()
        if bad == "future":
            b2[0, 2, 0] = 5
        elif bad == "unsorted":
            b2[1, 3, :2] = torch.tensor([3, 1], dtype=torch.int32)
            c2[1, 3] = 2
        else:
            c2[0, 1] = 9
        with pytest.raises(dsa.DSAError) as ei:
            dsa.block_sparse_attn_fwd(q, q, q, b2, c2)
        assert ei.value.rc == -1


# ---------------------------------------------------------------- A-shape

@pytest.mark.parametrize("n_sink,n_local", [(1, 4), (2, 7), (0, 3)])
def test_a_shape_lists_and_attention(n_sink, n_local):
    Hq, Hkv, n, d = 8, 2, 2048, 128
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=31)
    bi, bc = dsa.a_shape_index(Hq, n, n_sink, n_local)
    got = lists_from_gpu(bi, bc)
    want = oracle.a_shape_lists(n // 64, n_sink, n_local)
    for h in range(Hq):
        for qb in range(n // 64):
            assert got[h][qb].tolist() == want[qb].tolist(), (h, qb)
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc)
    torch.cuda.synchronize()
    items = [(h, qb) for h in range(Hq) for qb in range(n // 64)]
    ref = _ref_attention(w.q, w.k, w.v, got, None, 1 / math.sqrt(d), items)
    check_attention(o, ref, f"a-shape {n_sink}+{n_local}")
