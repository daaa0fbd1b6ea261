"""K-means key clusters and cluster-ranked decode, fp64 (oracle; test infrastructure only).

Squeezed Attention page ("Squeezed Attention：基于语义聚类的长上下文LLM推理加速"),
section "技术方案" (technical approach):

* offline stage: the keys of the fixed context are clustered with K-means, each
  cluster gets a centroid, and every key gets an index to its cluster;
* online stage: the query is compared with every centroid, the top clusters
  are kept, and attention runs only over the keys and values in them.

Readings taken (the page is silent on these):

* K-means is Lloyd's algorithm: assign every key to its nearest centroid in
  Euclidean distance (ties to the lower cluster id), then move every centroid
  to the mean of its keys; a cluster left without keys keeps its centroid.
* The starting centroids are the means of ``C`` equal contiguous segments of
  the context (segment ``c`` = keys ``floor(c n / C) .. floor((c+1) n / C) - 1``),
  unless the caller passes others.
* ``iters`` rounds of (assign, update) are run; the result is the last
  assignment and the centroids computed from it, so every centroid of a
  non-empty cluster is the mean of its keys.
* The cluster -> key map lists each cluster's keys in ascending token order
  (offsets + tokens, a CSR layout).
* Only the first ``n_ctx`` tokens (the fixed context) are clustered; the
  tokens after them (the newest ones, including the current token) are always
  attended.
* Ranking uses the raw dot product q . c over the clusters that have keys,
  ``keep`` of them (ties to the lower id); the softmax scale is the caller's.
"""

from __future__ import annotations

import numpy as np

from .blocksel import select_top


def segment_means(keys: np.ndarray, C: int) -> np.ndarray:
    """Means of C equal contiguous segments of keys [n][d] -> [C][d]."""
    n = keys.shape[0]
    out = np.empty((C, keys.shape[1]), dtype=np.float64)
    for c in range(C):
        lo, hi = (c * n) // C, ((c + 1) * n) // C
        out[c] = keys[lo:hi].mean(axis=0)
    return out


def kmeans_assign(keys: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """Nearest centroid of every key (squared Euclidean distance, ties to the
    lower id).  ||k - c||^2 = ||k||^2 + ||c||^2 - 2 k.c, one matmul."""
    d2 = (keys * keys).sum(axis=1)[:, None] + (cent * cent).sum(axis=1)[None, :] - 2.0 * (keys @ cent.T)
    return np.argmin(d2, axis=1).astype(np.int64)   # argmin returns the first minimum


def kmeans_update(keys: np.ndarray, assign: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """Mean of every cluster's keys; an empty cluster keeps its centroid."""
    C = cent.shape[0]
    sums = np.zeros_like(cent)
    np.add.at(sums, assign, keys)
    cnt = np.bincount(assign, minlength=C).astype(np.float64)
    out = cent.copy()
    nz = cnt > 0
    out[nz] = sums[nz] / cnt[nz][:, None]
    return out


def kmeans(keys: np.ndarray, C: int, iters: int, init: np.ndarray | None = None):
    """Lloyd's K-means: ``iters`` rounds of (assign, update).
    Returns (centroids [C][d], assignment [n])."""
    cent = segment_means(keys, C) if init is None else np.asarray(init, dtype=np.float64).copy()
    assign = np.zeros(keys.shape[0], dtype=np.int64)
    for _ in range(iters):
        assign = kmeans_assign(keys, cent)
        cent = kmeans_update(keys, assign, cent)
    return cent, assign


def kmeans_objective(keys: np.ndarray, cent: np.ndarray, assign: np.ndarray) -> float:
    """Sum of squared distances of the keys to their assigned centroids."""
    diff = keys - cent[assign]
    return float((diff * diff).sum())


def cluster_csr(assign: np.ndarray, C: int):
    """Cluster -> key map: offsets [C+1] and the keys of each cluster in
    ascending token order."""
    order = np.argsort(assign, kind="stable")
    cnt = np.bincount(assign, minlength=C)
    off = np.zeros(C + 1, dtype=np.int64)
    off[1:] = np.cumsum(cnt)
    return off, order.astype(np.int64)


def cluster_select(q: np.ndarray, cent: np.ndarray, off: np.ndarray, keep: int, pairs=None):
    """Kept clusters per (b, h): {(b, h): ascending ids}; plus tie info
    (candidate ids, their scores, the number kept) for the near-tie rule.

    q [B][Hq][d]; cent [B][Hkv][C][d]; off [B][Hkv][C+1]."""
    B, Hq, _ = q.shape
    Hkv = cent.shape[1]
    grp = Hq // Hkv
    pairs = [(b, h) for b in range(B) for h in range(Hq)] if pairs is None else pairs
    sel, info = {}, {}
    for b, h in pairs:
        g = h // grp
        cnt = np.diff(off[b, g])
        cand = np.nonzero(cnt > 0)[0].astype(np.int64)
        s = cent[b, g][cand] @ q[b, h]
        e = min(keep, cand.size)
        sel[(b, h)] = select_top(s, cand, e)
        info[(b, h)] = (cand, s, e)
    return sel, info


def cluster_tokens(clusters: np.ndarray, off: np.ndarray, tok: np.ndarray, n_ctx: int, S: int) -> np.ndarray:
    """Ascending tokens of the given clusters plus the unclustered tail [n_ctx, S)."""
    parts = [tok[off[c]:off[c + 1]] for c in np.asarray(clusters, dtype=np.int64)]
    parts.append(np.arange(n_ctx, S, dtype=np.int64))
    return np.sort(np.concatenate(parts)) if parts else np.zeros(0, dtype=np.int64)


def cluster_decode_attention(q, k_cache, v_cache, sel, off, tok, n_ctx: int, scale: float):
    """Single-query attention over the keys of the kept clusters and the tail:
    {(b, h): O [d]}.  off [B][Hkv][C+1], tok [B][Hkv][n_ctx]."""
    Hq = q.shape[1]
    Hkv, S = k_cache.shape[1], k_cache.shape[2]
    grp = Hq // Hkv
    out = {}
    for (b, h), clusters in sel.items():
        g = h // grp
        keys = cluster_tokens(clusters, off[b, g], tok[b, g], n_ctx, S)
        z = (k_cache[b, g, keys] @ q[b, h]) * scale
        p = np.exp(z - z.max())
        out[(b, h)] = (p @ v_cache[b, g, keys]) / p.sum()
    return out
