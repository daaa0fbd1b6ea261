"""Centroid-ranked sparse decode, fp64 (oracle; test infrastructure only).

Squeezed Attention page ("Squeezed Attention：基于语义聚类的长上下文LLM推理加速"),
section "技术方案" (technical approach): offline, the keys of the fixed context
are grouped and each group gets a centroid; online, the query is compared with
every centroid, the top groups are kept, and attention runs only over the keys
and values of the kept groups.

Readings taken: the groups are the contiguous 64-token blocks of the cache and
a centroid is the block's mean key; ranking uses the raw dot product q . c;
``keep`` blocks are kept among blocks 0..nb-2 (ties toward the lower block)
plus, when ``force_last`` is set, the last block (it holds the newest tokens,
including the current one); the softmax scale is the caller's.
"""

from __future__ import annotations

import numpy as np

from .blocksel import pool_blocks, select_top

BLOCK = 64


def decode_centroids(k_cache: np.ndarray) -> np.ndarray:
    """Per-block mean keys: [B][Hkv][S][d] -> [B][Hkv][S/64][d]."""
    return pool_blocks(k_cache)


def decode_select(q: np.ndarray, cent: np.ndarray, keep: int, force_last: int, pairs=None):
    """Kept blocks per (b, h): {(b, h): ascending int64 array}; plus tie info."""
    B, Hq, d = q.shape
    Hkv, nb = cent.shape[1], cent.shape[2]
    grp = Hq // Hkv
    pairs = [(b, h) for b in range(B) for h in range(Hq)] if pairs is None else pairs
    sel, info = {}, {}
    for b, h in pairs:
        g = h // grp
        s = cent[b, g] @ q[b, h]
        ncand = nb - 1 if force_last else nb
        cand = np.arange(ncand, dtype=np.int64)
        e = min(keep, ncand)
        top = select_top(s[:ncand], cand, e)
        if force_last:
            top = np.union1d(top, np.array([nb - 1], dtype=np.int64))
        sel[(b, h)] = top
        info[(b, h)] = (cand, s[:ncand], e)
    return sel, info


def decode_attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, sel, scale: float):
    """Single-query attention over the tokens of the kept blocks: {(b, h): O [d]}."""
    Hq = q.shape[1]
    Hkv = k_cache.shape[1]
    grp = Hq // Hkv
    out = {}
    for (b, h), blocks in sel.items():
        g = h // grp
        keys = (np.asarray(blocks)[:, None] * BLOCK + np.arange(BLOCK)[None, :]).reshape(-1)
        z = (k_cache[b, g, keys] @ q[b, h]) * scale
        p = np.exp(z - z.max())
        out[(b, h)] = (p @ v_cache[b, g, keys]) / p.sum()
    return out


def sparse_decode(q, k_cache, v_cache, keep, force_last, scale, pairs=None):
    cent = decode_centroids(k_cache)
    sel, info = decode_select(q, cent, keep, force_last, pairs)
    return decode_attention(q, k_cache, v_cache, sel, scale), sel, info, cent
