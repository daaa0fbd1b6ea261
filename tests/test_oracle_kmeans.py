"""Pins of the K-means oracle (CPU only).

Squeezed Attention page, "技术方案": offline K-means over the fixed context's
keys (centroids plus a key -> cluster map), online ranking of the centroids
against the query and attention over the kept clusters' keys.  Each test ties
a function of ``oracle/clusters.py`` to brute force, a closed form, an
invariant of Lloyd's algorithm or a hand-worked example.
"""

import numpy as np
import pytest

import oracle


def rng(seed):
    return np.random.default_rng(seed)


def test_assign_matches_explicit_distance_bruteforce():
    """Nearest centroid from the expanded distance equals the argmin of the
    explicit squared distance sum((k - c)^2), first minimum on ties."""
    r = rng(11)
    for n, C, d in ((40, 7, 5), (64, 16, 3), (33, 1, 8)):
        keys = r.standard_normal((n, d))
        cent = r.standard_normal((C, d))
        got = oracle.kmeans_assign(keys, cent)
        for t in range(n):
            dist = [float(((keys[t] - cent[c]) ** 2).sum()) for c in range(C)]
            assert got[t] == int(np.argmin(dist))


def test_assign_ties_go_to_the_lower_cluster():
    keys = np.array([[0.0, 0.0], [2.0, 0.0]])
    cent = np.array([[1.0, 1.0], [1.0, -1.0], [5.0, 5.0]])   # both keys equidistant to clusters 0 and 1
    assert oracle.kmeans_assign(keys, cent).tolist() == [0, 0]


def test_update_is_the_member_mean_and_keeps_empty_clusters():
    keys = np.array([[1.0, 2.0], [3.0, 4.0], [10.0, 0.0], [20.0, 2.0], [30.0, 4.0]])
    assign = np.array([0, 0, 2, 2, 2])
    old = np.array([[0.0, 0.0], [7.0, 7.0], [0.0, 0.0]])
    new = oracle.kmeans_update(keys, assign, old)
    assert np.allclose(new[0], [2.0, 3.0])
    assert np.allclose(new[1], [7.0, 7.0])          # no keys: unchanged
    assert np.allclose(new[2], [20.0, 2.0])


def test_segment_means_closed_form():
    keys = np.arange(10, dtype=np.float64)[:, None] * np.array([[1.0, -2.0]])
    cm = oracle.segment_means(keys, 3)   # segments [0,3) [3,6) [6,10)
    assert np.allclose(cm[:, 0], [1.0, 4.0, 7.5])
    assert np.allclose(cm[:, 1], [-2.0, -8.0, -15.0])


def test_hand_worked_example():
    """Keys 0, 1, 10, 11 on a line, two clusters started at the segment means
    0.5 and 10.5: the clusters are {0, 1} and {10, 11} from the first round."""
    keys = np.array([[0.0], [1.0], [10.0], [11.0]])
    cent, assign = oracle.kmeans(keys, 2, 3)
    assert assign.tolist() == [0, 0, 1, 1]
    assert np.allclose(cent[:, 0], [0.5, 10.5])
    # started the other way round, the first round still moves every key to its side
    cent, assign = oracle.kmeans(keys, 2, 2, init=np.array([[11.0], [0.0]]))
    assert assign.tolist() == [1, 1, 0, 0]
    assert np.allclose(cent[:, 0], [10.5, 0.5])


def test_one_cluster_is_the_global_mean():
    r = rng(3)
    keys = r.standard_normal((50, 6))
    cent, assign = oracle.kmeans(keys, 1, 4)
    assert np.all(assign == 0)
    assert np.allclose(cent[0], keys.mean(axis=0))


def test_every_key_its_own_cluster():
    """C = n started at the keys themselves: a fixed point, identity map."""
    r = rng(4)
    keys = r.standard_normal((20, 4))
    cent, assign = oracle.kmeans(keys, 20, 3, init=keys)
    assert assign.tolist() == list(range(20))
    assert np.allclose(cent, keys)


def test_objective_never_increases():
    """Lloyd's algorithm: neither the assignment nor the update step can raise
    the sum of squared distances."""
    r = rng(5)
    keys = r.standard_normal((300, 8))
    cent = oracle.segment_means(keys, 12)
    prev = np.inf
    for _ in range(8):
        assign = oracle.kmeans_assign(keys, cent)
        after_assign = oracle.kmeans_objective(keys, cent, assign)
        assert after_assign <= prev + 1e-9
        cent = oracle.kmeans_update(keys, assign, cent)
        after_update = oracle.kmeans_objective(keys, cent, assign)
        assert after_update <= after_assign + 1e-9
        prev = after_update


def test_separated_blobs_are_recovered():
    """Three far-apart blobs with one starting centroid in each: the clusters
    are exactly the blobs and the centroids are the blob means."""
    r = rng(6)
    centers = np.array([[0.0, 0.0, 0.0], [40.0, 0.0, 0.0], [0.0, 40.0, 0.0]])
    lab = r.integers(0, 3, 90)
    keys = centers[lab] + r.standard_normal((90, 3))
    init = np.array([keys[np.nonzero(lab == b)[0][0]] for b in range(3)])
    cent, assign = oracle.kmeans(keys, 3, 5, init=init)
    assert np.array_equal(assign, lab)
    for b in range(3):
        assert np.allclose(cent[b], keys[lab == b].mean(axis=0))


def test_result_centroids_are_member_means():
    r = rng(7)
    keys = r.standard_normal((200, 5))
    cent, assign = oracle.kmeans(keys, 9, 4)
    for c in range(9):
        m = assign == c
        if m.any():
            assert np.allclose(cent[c], keys[m].mean(axis=0))


def test_csr_is_a_stable_partition():
    r = rng(8)
    assign = r.integers(0, 10, 500)
    off, tok = oracle.cluster_csr(assign, 12)
    assert off[0] == 0 and off[-1] == 500 and np.all(np.diff(off) >= 0)
    assert sorted(tok.tolist()) == list(range(500))
    for c in range(12):
        members = tok[off[c]:off[c + 1]]
        assert np.all(assign[members] == c)
        assert np.all(np.diff(members) > 0)
    assert off[11] == off[12] and off[10] == off[11]   # clusters 10, 11 are empty


def _decode_case(seed, B=2, Hq=4, Hkv=2, S=384, n_ctx=320, d=16, C=12):
    r = rng(seed)
    q = r.standard_normal((B, Hq, d))
    k = r.standard_normal((B, Hkv, S, d))
    v = r.standard_normal((B, Hkv, S, d))
    cent = np.zeros((B, Hkv, C, d))
    off = np.zeros((B, Hkv, C + 1), dtype=np.int64)
    tok = np.zeros((B, Hkv, n_ctx), dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            c, a = oracle.kmeans(k[b, g, :n_ctx], C, 3)
            cent[b, g] = c
            off[b, g], tok[b, g] = oracle.cluster_csr(a, C)
    return q, k, v, cent, off, tok, n_ctx


def test_keep_all_clusters_equals_dense_single_query_attention():
    q, k, v, cent, off, tok, n_ctx = _decode_case(9)
    scale = 0.3
    sel, _ = oracle.cluster_select(q, cent, off, keep=10**6)
    out = oracle.cluster_decode_attention(q, k, v, sel, off, tok, n_ctx, scale)
    grp = q.shape[1] // k.shape[1]
    for (b, h), o in out.items():
        g = h // grp
        z = np.array([scale * float(k[b, g, t] @ q[b, h]) for t in range(k.shape[2])])
        w = np.exp(z - z.max())
        ref = (w[:, None] * v[b, g]).sum(axis=0) / w.sum()
        assert np.allclose(o, ref, atol=1e-12)


def test_zero_query_is_the_mean_over_kept_tokens():
    q, k, v, cent, off, tok, n_ctx = _decode_case(10)
    q[:] = 0.0
    sel, info = oracle.cluster_select(q, cent, off, keep=4)
    out = oracle.cluster_decode_attention(q, k, v, sel, off, tok, n_ctx, 1.0)
    grp = q.shape[1] // k.shape[1]
    for (b, h), o in out.items():
        g = h // grp
        cand = info[(b, h)][0]
        assert np.array_equal(sel[(b, h)], cand[:4])   # all scores 0: the lowest ids win
        keys = oracle.cluster_tokens(sel[(b, h)], off[b, g], tok[b, g], n_ctx, k.shape[2])
        assert np.allclose(o, v[b, g, keys].mean(axis=0))


def test_select_bruteforce_and_empty_clusters_excluded():
    q, k, v, cent, off, tok, n_ctx = _decode_case(12, C=40)
    sel, info = oracle.cluster_select(q, cent, off, keep=5)
    grp = q.shape[1] // k.shape[1]
    for (b, h), ids in sel.items():
        g = h // grp
        cnt = np.diff(off[b, g])
        scored = [(-float(cent[b, g, c] @ q[b, h]), c) for c in range(40) if cnt[c] > 0]
        want = sorted(c for _, c in sorted(scored)[:5])
        assert ids.tolist() == want
        assert all(cnt[c] > 0 for c in ids)
