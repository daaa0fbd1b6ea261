"""Sparse causal softmax attention over chosen key sets, fp64 (oracle; test infrastructure only).

MInference 1.0 page, section "方法介紹" (method): after the index is estimated,
attention is computed only over the chosen parts of the key/value sequence
(block-sparse FlashAttention); Fig. 4: 64x64 blocks and 1x64 column tiles.

For query row i of q-head h (KV head g = h // (Hq/Hkv)) the attended key set is
A_i = (union of the chosen 64-key blocks and chosen single columns of i's query
block) intersected with [0, i] (causal), and

    O_i = sum_{j in A_i} softmax_j(q_i . k_j * scale) v_j,   lse_i = log sum_j exp(q_i . k_j * scale).

The softmax scale is the caller's (1/sqrt(d) in every workload here; the pages
do not state it).  Duplicate keys in a set are an error.
"""

from __future__ import annotations

import numpy as np

BLOCK = 64


def _key_set(blocks, cols) -> np.ndarray:
    blocks = np.asarray(blocks, dtype=np.int64)
    cols = np.asarray(cols if cols is not None else [], dtype=np.int64)
    keys = np.concatenate([(blocks[:, None] * BLOCK + np.arange(BLOCK)[None, :]).reshape(-1), cols])
    if np.unique(keys).size != keys.size:
        raise ValueError("duplicate key in an attended set")
    return keys


def sparse_attention_rows(q_rows: np.ndarray, row_ids: np.ndarray, k: np.ndarray, v: np.ndarray,
                          blocks, cols, scale: float):
    """Attention of the query rows ``row_ids`` (one query block of one head).

    q_rows [m][d]; k, v [n][d] of the head's KV head.  Returns (O [m][d], lse [m])."""
    keys = _key_set(blocks, cols)
    Z = (q_rows @ k[keys].T) * scale                      # [m][|keys|]
    Z[keys[None, :] > row_ids[:, None]] = -np.inf          # causal
    m = Z.max(axis=1, keepdims=True)
    P = np.exp(Z - m)
    l = P.sum(axis=1, keepdims=True)
    O = (P @ v[keys]) / l
    lse = (m + np.log(l))[:, 0]
    return O, lse


def sparse_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, block_lists, col_lists, scale: float,
                     items=None):
    """O and lse for each (h, qb) in ``items`` (default: all).

    block_lists[h][qb] / col_lists[h][qb] (col_lists may be None) give the chosen
    key blocks and columns.  Returns {(h, qb): (O [64][d], lse [64])}."""
    Hq, n, d = q.shape
    Hkv = k.shape[0]
    grp = Hq // Hkv
    nb = n // BLOCK
    if items is None:
        items = [(h, qb) for h in range(Hq) for qb in range(nb)]
    out = {}
    for h, qb in items:
        g = h // grp
        rows = np.arange(qb * BLOCK, qb * BLOCK + BLOCK)
        cols = None if col_lists is None else col_lists[h][qb]
        out[(h, qb)] = sparse_attention_rows(q[h, rows], rows, k[g], v[g], block_lists[h][qb], cols, scale)
    return out


def dense_lists(Hq: int, n: int):
    """Block lists that select every causal block (the dense special case)."""
    nb = n // BLOCK
    return {h: {qb: np.arange(qb + 1, dtype=np.int64) for qb in range(nb)} for h in range(Hq)}
