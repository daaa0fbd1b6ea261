"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test ties one oracle function to a closed form, an invariant, a library
routine that computes the same quantity another way, or brute force on tiny
inputs, so that a dropped term, a wrong sign or index, or a transposed operand
anywhere in the oracle fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from oracle import vslash as ovs

BLOCK = 64


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- block index

def test_pooled_score_commutes_with_matmul():
    """MInference 1.0, method section: mean pooling commutes with the matrix
    product, so Q̄_i·K̄_j equals the mean of the 64x64 raw score block."""
    r = rng(1)
    n, d = 256, 16
    q = r.standard_normal((n, d))
    k = r.standard_normal((n, d))
    S = oracle.block_scores(oracle.pool_blocks(q), oracle.pool_blocks(k))
    nb = n // BLOCK
    for i, j in itertools.product(range(nb), range(nb)):
        raw = q[i * BLOCK:(i + 1) * BLOCK] @ k[j * BLOCK:(j + 1) * BLOCK].T
        assert abs(S[i, j] - raw.mean()) < 1e-12 * max(1.0, abs(raw).max())


def test_budget_table():
    """The per-row budget written out by hand from the selection rule:
    fixed k counts the forced sink+diagonal inside k; a ratio counts extra
    blocks beyond them, ceil(rho*(i+1)), capped by the i-1 candidates."""
    fixed4 = {0: 0, 1: 0, 2: 1, 3: 2, 4: 2, 15: 2}
    for i, e in fixed4.items():
        assert oracle.extra_budget(i, 4, 0.0) == e, i
    r10 = {0: 0, 1: 0, 2: 1, 3: 1, 9: 1, 10: 2, 19: 2, 20: 3, 29: 3, 30: 4, 511: 52}
    for i, e in r10.items():
        assert oracle.extra_budget(i, 0, 0.10) == e, i
    r2 = {2: 1, 49: 1, 50: 2, 99: 2, 100: 3, 16383: 328}
    for i, e in r2.items():
        assert oracle.extra_budget(i, 0, 0.02) == e, i
    assert oracle.max_blocks_per_row(16, 4, 0.0) == 4
    assert oracle.max_blocks_per_row(512, 0, 0.10) == 54
    assert oracle.max_blocks_per_row(16384, 0, 0.02) == 330


def test_select_top_matches_python_sort():
    """Brute force: Python's sort on (-score, id) tuples, with many exact ties."""
    r = rng(2)
    for trial in range(200):
        m = int(r.integers(1, 40))
        scores = r.integers(-3, 4, size=m).astype(np.float64)   # heavy ties
        cand = np.sort(r.choice(1000, size=m, replace=False)).astype(np.int64)
        e = int(r.integers(0, m + 1))
        got = oracle.select_top(scores, cand, e)
        ref = sorted(sorted(zip(cand.tolist(), scores.tolist()), key=lambda t: (-t[1], t[0]))[:e])
        assert got.tolist() == [c for c, _ in ref]


def test_block_index_forced_counts_and_bruteforce():
    r = rng(3)
    n, d = 1024, 16
    q = r.standard_normal((2, n, d))
    k = r.standard_normal((1, n, d))
    for kf, rho in ((4, 0.0), (0, 0.10), (0, 0.5)):
        lists, info, _ = oracle.block_index(q, k, k_fixed=kf, keep_ratio=rho)
        for h in range(2):
            for i in range(n // BLOCK):
                sel = lists[h][i].tolist()
                assert sel == sorted(set(sel))
                assert 0 in sel and i in sel
                forced = 1 if i == 0 else 2
                assert len(sel) == forced + oracle.extra_budget(i, kf, rho)
                # brute force over raw 64x64 block means
                means = []
                for j in range(1, i):
                    raw = q[h, i * 64:(i + 1) * 64] @ k[0, j * 64:(j + 1) * 64].T
                    means.append((-raw.mean(), j))
                e = oracle.extra_budget(i, kf, rho)
                want = sorted({0, i} | {j for _, j in sorted(means)[:e]})
                assert sel == want


# ---------------------------------------------------------------- attention

def _sdpa_causal_f64(q, k, v, scale):
    grp = q.shape[0] // k.shape[0]
    qt = torch.from_numpy(q)[None]
    kt = torch.from_numpy(np.repeat(k, grp, axis=0))[None]
    vt = torch.from_numpy(np.repeat(v, grp, axis=0))[None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)[0].numpy()


def test_all_blocks_equals_dense_causal_sdpa():
    """Top-k = all causal blocks must equal dense causal softmax attention
    (torch's scaled_dot_product_attention in float64 as the independent routine)."""
    r = rng(4)
    Hq, Hkv, n, d = 4, 2, 256, 32
    q, k, v = r.standard_normal((Hq, n, d)), r.standard_normal((Hkv, n, d)), r.standard_normal((Hkv, n, d))
    scale = 1 / math.sqrt(d)
    out = oracle.sparse_attention(q, k, v, oracle.dense_lists(Hq, n), None, scale)
    ref = _sdpa_causal_f64(q, k, v, scale)
    for (h, qb), (O, _) in out.items():
        np.testing.assert_allclose(O, ref[h, qb * 64:(qb + 1) * 64], rtol=0, atol=1e-12)


def test_attention_bruteforce_tiny():
    """Element-by-element masked softmax with Python loops on a tiny case."""
    r = rng(5)
    n, d = 192, 4
    q, k, v = r.standard_normal((1, n, d)), r.standard_normal((1, n, d)), r.standard_normal((1, n, d))
    scale = 0.37
    blocks = {0: {0: [0], 1: [1], 2: [0, 2]}}
    cols = {0: {0: [], 1: [5, 17], 2: [70, 100]}}
    out = oracle.sparse_attention(q, k, v, blocks, cols, scale)
    for qb in range(3):
        allowed = set()
        for b in blocks[0][qb]:
            allowed |= set(range(b * 64, b * 64 + 64))
        allowed |= set(cols[0][qb])
        for rr in range(64):
            i = qb * 64 + rr
            keys = [j for j in sorted(allowed) if j <= i]
            z = [sum(q[0, i, t] * k[0, j, t] for t in range(d)) * scale for j in keys]
            mx = max(z)
            w = [math.exp(x - mx) for x in z]
            tot = sum(w)
            o = [sum(w[a] * v[0, keys[a], t] for a in range(len(keys))) / tot for t in range(d)]
            O, lse = out[(0, qb)]
            assert np.allclose(O[rr], o, atol=1e-12)
            assert abs(lse[rr] - (mx + math.log(tot))) < 1e-12


def test_attention_special_values():
    """V = 1 gives O = 1; Q = 0 gives the plain mean of V over the attended
    set and lse = log |A_i|."""
    r = rng(6)
    n, d = 256, 8
    k, v = r.standard_normal((1, n, d)), r.standard_normal((1, n, d))
    blocks = {0: {qb: [0, qb] if qb else [0] for qb in range(4)}}
    cols = {0: {0: [], 1: [], 2: [65, 100], 3: [130]}}
    out1 = oracle.sparse_attention(r.standard_normal((1, n, d)), k, np.ones((1, n, d)), blocks, cols, 0.5)
    for O, _ in out1.values():
        np.testing.assert_allclose(O, 1.0, atol=1e-13)
    out0 = oracle.sparse_attention(np.zeros((1, n, d)), k, v, blocks, cols, 0.5)
    for (h, qb), (O, lse) in out0.items():
        for rr in range(64):
            i = qb * 64 + rr
            keys = [j for b in blocks[0][qb] for j in range(b * 64, b * 64 + 64) if j <= i]
            keys += [j for j in cols[0][qb] if j <= i]
            np.testing.assert_allclose(O[rr], v[0, keys].mean(axis=0), atol=1e-13)
            assert abs(lse[rr] - math.log(len(keys))) < 1e-13


def test_attention_rejects_duplicates():
    r = rng(7)
    x = r.standard_normal((1, 128, 4))
    with pytest.raises(ValueError):
        oracle.sparse_attention(x, x, x, {0: {1: [0, 1]}}, {0: {1: [3]}}, 1.0, items=[(0, 1)])


# ---------------------------------------------------------------- vertical-slash

def test_vs_scores_sum_to_last_q():
    """Every softmax row sums to 1, so the column sums and the diagonal sums
    each total last_q."""
    r = rng(8)
    n, d = 512, 16
    q, k = r.standard_normal((2, n, d)), r.standard_normal((1, n, d))
    vert, slash = oracle.vs_scores(q, k, 64, 1 / math.sqrt(d))
    for h in range(2):
        assert abs(vert[h].sum() - 64) < 1e-10
        assert abs(slash[h].sum() - 64) < 1e-10


def test_vs_scores_closed_form_uniform():
    """Q = 0 makes each row uniform over its i_r+1 causal keys, so
    vert[j] = slash[j] = sum over rows with i_r >= j of 1/(i_r+1)."""
    n, d = 320, 8
    r = rng(9)
    vert, slash = oracle.vs_scores(np.zeros((1, n, d)), r.standard_normal((1, n, d)), 64, 1.0)
    rows = range(n - 64, n)
    for j in range(n):
        want = sum(1.0 / (i + 1) for i in rows if i >= j)
        assert abs(vert[0][j] - want) < 1e-12
        assert abs(slash[0][j] - want) < 1e-12


def test_vs_scores_bruteforce_tiny():
    r = rng(10)
    n, d = 128, 4
    q, k = r.standard_normal((1, n, d)), r.standard_normal((1, n, d))
    vert, slash = oracle.vs_scores(q, k, 64, 0.8)
    bv = [0.0] * n
    bs = [0.0] * n
    for rr in range(64):
        i = n - 64 + rr
        z = [sum(q[0, i, t] * k[0, j, t] for t in range(d)) * 0.8 for j in range(i + 1)]
        mx = max(z)
        w = [math.exp(x - mx) for x in z]
        tot = sum(w)
        for j in range(i + 1):
            bv[j] += w[j] / tot
            bs[i - j] += w[j] / tot
    np.testing.assert_allclose(vert[0], bv, atol=1e-13)
    np.testing.assert_allclose(slash[0], bs, atol=1e-13)


def test_vs_topk_forced_and_sorted():
    r = rng(11)
    n = 1024
    vert, slash = r.random(n), r.random(n)
    vi, so, _, _ = oracle.vs_topk(vert, slash, 100, 30)
    assert vi.size == 100 and so.size == 30
    assert set(range(64)) <= set(vi.tolist()) and 0 in so.tolist()
    want_v = sorted(set(range(64)) | set(sorted(range(64, n), key=lambda j: (-vert[j], j))[:36]))
    want_s = sorted({0} | set(sorted(range(1, n), key=lambda o: (-slash[o], o))[:29]))
    assert vi.tolist() == want_v and so.tolist() == want_s


@pytest.mark.parametrize("seed", [12, 13, 14])
def test_vs_plan_bruteforce_coverage(seed):
    """Brute force over elements: every kept diagonal element (i, i-o) and
    every kept column j <= i is covered by the plan, the block set is exactly
    the set of blocks the kept diagonals touch, and each kept column is listed
    once, either inside a selected block or as a column tile entry."""
    r = rng(seed)
    n = 512
    nb = n // 64
    so = np.union1d([0], r.choice(np.arange(1, n), size=int(r.integers(1, 20)), replace=False))
    vi = np.union1d(np.arange(64), r.choice(np.arange(64, n), size=int(r.integers(0, 30)), replace=False))
    plan = oracle.vs_plan(vi, so, n)
    for qb in range(nb):
        blocks, cols = plan[qb]
        bset = set(blocks.tolist())
        touched = set()
        for i in range(qb * 64, qb * 64 + 64):
            for o in so.tolist():
                if i - o >= 0:
                    touched.add((i - o) // 64)
        assert bset == touched
        for i in range(qb * 64, qb * 64 + 64):
            for j in vi.tolist():
                if j <= i:
                    assert (j // 64 in bset) != (j in cols.tolist())
        assert all(c < qb * 64 for c in cols.tolist())


# ---------------------------------------------------------------- decode

def _sdpa_single_f64(q, k, v, scale):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], scale=scale)[0, 0].numpy()


def test_decode_keep_all_equals_dense():
    r = rng(15)
    B, Hq, Hkv, S, d = 2, 4, 2, 512, 16
    q = r.standard_normal((B, Hq, d))
    kc, vc = r.standard_normal((B, Hkv, S, d)), r.standard_normal((B, Hkv, S, d))
    out, sel, _, _ = oracle.sparse_decode(q, kc, vc, keep=S // 64, force_last=1, scale=0.25)
    for (b, h), O in out.items():
        assert sel[(b, h)].tolist() == list(range(S // 64))
        ref = _sdpa_single_f64(q[b, h], kc[b, h // 2], vc[b, h // 2], 0.25)
        np.testing.assert_allclose(O, ref, atol=1e-12)


def test_decode_zero_query_keeps_lowest_blocks():
    """Q = 0 scores every block 0: the tie-break keeps blocks 0..keep-1 plus
    the last, and the output is the mean of V over those tokens."""
    r = rng(16)
    B, Hq, Hkv, S, d = 1, 2, 1, 1024, 8
    kc, vc = r.standard_normal((B, Hkv, S, d)), r.standard_normal((B, Hkv, S, d))
    out, sel, _, _ = oracle.sparse_decode(np.zeros((B, Hq, d)), kc, vc, keep=5, force_last=1, scale=1.0)
    for (b, h), O in out.items():
        assert sel[(b, h)].tolist() == [0, 1, 2, 3, 4, 15]
        toks = [j for blk in [0, 1, 2, 3, 4, 15] for j in range(blk * 64, blk * 64 + 64)]
        np.testing.assert_allclose(O, vc[0, 0, toks].mean(axis=0), atol=1e-13)


def test_decode_centroid_score_bruteforce():
    """q·c_t equals the mean of q·k over the block's 64 keys; selection equals
    Python's sort on (-score, block)."""
    r = rng(17)
    B, Hq, Hkv, S, d = 1, 2, 1, 640, 8
    q = r.standard_normal((B, Hq, d))
    kc, vc = r.standard_normal((B, Hkv, S, d)), r.standard_normal((B, Hkv, S, d))
    cent = oracle.decode_centroids(kc)
    sel, info = oracle.decode_select(q, cent, keep=3, force_last=1)
    for h in range(Hq):
        means = []
        for t in range(S // 64 - 1):
            dots = [sum(q[0, h, a] * kc[0, 0, j, a] for a in range(d)) for j in range(t * 64, t * 64 + 64)]
            m = sum(dots) / 64
            assert abs(info[(0, h)][1][t] - m) < 1e-12
            means.append((-m, t))
        want = sorted({S // 64 - 1} | {t for _, t in sorted(means)[:3]})
        assert sel[(0, h)].tolist() == want


# ---------------------------------------------------------------- tie rule

def test_tie_rule():
    cand = np.arange(1, 8)
    scores = np.array([5.0, 4.0, 3.0, 3.0000001, 1.0, 0.5, 0.1])
    forced = [0, 8]
    # exact oracle answer
    assert oracle.compare_index_sets([0, 1, 2, 4, 8], forced, cand, scores, 3) == "exact"
    # near tie between ids 3 and 4 at the boundary: either is fine
    assert oracle.compare_index_sets([0, 1, 2, 3, 8], forced, cand, scores, 3) == "ambiguous"
    # dropping a clearly higher candidate is not
    assert oracle.compare_index_sets([0, 2, 3, 4, 8], forced, cand, scores, 3).startswith("MISMATCH")
    # wrong count, missing forced
    assert oracle.compare_index_sets([0, 1, 2, 8], forced, cand, scores, 3).startswith("MISMATCH")
    assert oracle.compare_index_sets([1, 2, 4, 8], forced, cand, scores, 2).startswith("MISMATCH")


def test_tie_rule_every_rejection_branch():
    """Each way a set can break the near-tie rule, in a row that has a near tie
    at the boundary (ids 4 and 3 score 3.0000001 and 3.0, 3 kept), so that only
    the branch under test can reject it:

    * a clearly lower candidate kept: {1, 2, 5} has the right count and both
      clearly higher ids (5.0, 4.0), but id 5 scores 1.0, below the (k+1)-th
      score 3.0 by far more than 1e-4 relative;
    * a candidate just inside the lower bound is accepted (id 3, exactly the
      (k+1)-th score), and one scoring 0.99995 of it is not;
    * ids not strictly ascending, or repeated;
    * an id that is not a candidate (9 > 8, the last forced id)."""
    cand = np.arange(1, 8)
    scores = np.array([5.0, 4.0, 3.0, 3.0000001, 1.0, 0.5, 0.1])
    forced = [0, 8]
    st = oracle.compare_index_sets([0, 1, 2, 5, 8], forced, cand, scores, 3)
    assert st == "MISMATCH: a clearly lower candidate was kept", st
    assert oracle.compare_index_sets([0, 1, 2, 3, 8], forced, cand, scores, 3) == "ambiguous"
    near = scores.copy()
    near[4] = 3.0 * (1 - 0.5e-4)          # id 5 within 1e-4 of the (k+1)-th score: still a near tie
    assert oracle.compare_index_sets([0, 1, 2, 5, 8], forced, cand, near, 3) == "ambiguous"
    far = scores.copy()
    far[4] = 3.0 * (1 - 1.5e-4)           # id 5 just outside the bound
    st = oracle.compare_index_sets([0, 1, 2, 5, 8], forced, cand, far, 3)
    assert st == "MISMATCH: a clearly lower candidate was kept", st
    st = oracle.compare_index_sets([0, 2, 1, 4, 8], forced, cand, scores, 3)
    assert st == "MISMATCH: not strictly ascending", st
    st = oracle.compare_index_sets([0, 1, 1, 4, 8], forced, cand, scores, 3)
    assert st == "MISMATCH: not strictly ascending", st
    st = oracle.compare_index_sets([0, 1, 2, 8, 9], forced, cand, scores, 3)
    assert st == "MISMATCH: an id outside the candidates", st
    # negative scores: "clearly lower" is sign-aware (-3.0 is the (k+1)-th score)
    neg = -scores[::-1].copy()            # ids 1..7 score -0.1, -0.5, -1, -3.0000001, -3, -4, -5
    assert oracle.compare_index_sets([0, 1, 2, 3, 5, 8], forced, cand, neg, 4) == "exact"
    assert oracle.compare_index_sets([0, 1, 2, 3, 4, 8], forced, cand, neg, 4) == "ambiguous"
    st = oracle.compare_index_sets([0, 1, 2, 3, 6, 8], forced, cand, neg, 4)
    assert st == "MISMATCH: a clearly lower candidate was kept", st


# ---------------------------------------------------------------- A-shape

def test_a_shape_closed_form():
    """Counts written out from the definition: min(qb+1, n_sink + n_local) for
    every query block (the two ranges overlap once qb < n_sink + n_local)."""
    lists = oracle.a_shape_lists(40, 2, 5)
    for qb, sel in lists.items():
        assert len(sel) == min(qb + 1, 7)
        assert sel.tolist() == sorted(set(sel.tolist()))
        assert 0 in sel.tolist() and qb in sel.tolist()
    assert lists[10].tolist() == [0, 1, 6, 7, 8, 9, 10]
    assert lists[3].tolist() == [0, 1, 2, 3]
