"""Block-sparse index estimation, fp64 (oracle; test infrastructure only).

MInference 1.0 page, section "方法介紹" (method): for the block-sparse pattern
Q and K are mean-pooled, and because mean pooling commutes with the matrix
product the pooled score estimates the block's attention mass; the top blocks
of each query block become its index.  The selection rule used here -- keep
the first (sink) block and the query block's own (diagonal) block, plus the
top of the remaining causal blocks, ties toward the lower block id -- is the
problem statement's; the pages do not print it.

Readings taken where the pages are silent:
* ranking uses the raw pooled dot product Q̄·K̄ (no 1/sqrt(d), no softmax: both
  are monotone and leave the order unchanged);
* fixed budget ``k_fixed``: the total per query block including the forced
  blocks, i.e. ``e_i = min(i+1, k) - |{0, i}|`` extra blocks;
* ratio budget ``keep_ratio``: extra blocks beyond the forced ones,
  ``e_i = min(i-1, ceil(rho * (i+1)))``, with rho taken in parts per million
  (``round(rho * 1e6)``) so the ceiling is exact integer arithmetic.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 64


def pool_blocks(x: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Mean of each run of ``block`` consecutive rows: [..., n, d] -> [..., n/block, d]."""
    n, d = x.shape[-2], x.shape[-1]
    if n % block:
        raise ValueError("sequence length must be a multiple of the block size")
    xs = np.asarray(x, dtype=np.float64).reshape(x.shape[:-2] + (n // block, block, d))
    return xs.mean(axis=-2)


def ratio_ppm(keep_ratio: float) -> int:
    """The keep ratio as an integer number of parts per million (round half up).

    The ratio is first taken as an fp32 value, as it crosses the C interface."""
    r = float(np.float32(keep_ratio))
    return int(math.floor(r * 1e6 + 0.5))


def extra_budget(i: int, k_fixed: int, keep_ratio: float) -> int:
    """Number of non-forced blocks kept for query block ``i``."""
    forced = 1 if i == 0 else 2
    cand = max(i - 1, 0)           # blocks 1 .. i-1
    if k_fixed > 0:
        e = min(i + 1, k_fixed) - forced
    else:
        ppm = ratio_ppm(keep_ratio)
        e = -((-ppm * (i + 1)) // 1_000_000)      # ceil(ppm*(i+1)/1e6), exact
    return max(0, min(e, cand))


def max_blocks_per_row(n_blocks: int, k_fixed: int, keep_ratio: float) -> int:
    """Largest selected-set size over all query blocks (the needed list capacity)."""
    best = 0
    for i in range(n_blocks):
        forced = 1 if i == 0 else 2
        best = max(best, forced + extra_budget(i, k_fixed, keep_ratio))
    return best


def select_top(scores: np.ndarray, cand: np.ndarray, e: int) -> np.ndarray:
    """The ``e`` candidates with the highest score; equal scores go to the lower id.

    ``np.lexsort`` sorts by its last key first: score descending, then id ascending."""
    if e <= 0 or cand.size == 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((cand, -scores))
    return np.sort(cand[order[:e]])


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Pooled block scores S[i, j] = Q̄_i · K̄_j (full fp64 product)."""
    return qbar @ kbar.T


def block_index(q: np.ndarray, k: np.ndarray, k_fixed: int = 0, keep_ratio: float = 0.0,
                heads=None, rows=None):
    """Block-sparse index for every (q-head, query block).

    q: [Hq][n][d], k: [Hkv][n][d] (fp64 views of the bf16 inputs).
    Returns (lists, scores_info, kbar): ``lists[h][i]`` is the ascending int64
    array of kept key blocks; ``scores_info[h][i]`` is (cand, scores, e) for the
    tie check; ``kbar`` is the pooled K [Hkv][n/64][d].
    ``heads``/``rows`` restrict the work to a sample (all by default).
    """
    Hq, n, d = q.shape
    Hkv = k.shape[0]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    grp = Hq // Hkv
    nb = n // BLOCK
    kbar = pool_blocks(k)
    heads = range(Hq) if heads is None else heads
    lists, info = {}, {}
    for h in heads:
        g = h // grp
        qbar = pool_blocks(q[h])
        S = block_scores(qbar, kbar[g])
        rws = range(nb) if rows is None else rows
        lists[h], info[h] = {}, {}
        for i in rws:
            cand = np.arange(1, i, dtype=np.int64)
            e = extra_budget(i, k_fixed, keep_ratio)
            sc = S[i, 1:i]
            top = select_top(sc, cand, e)
            forced = np.array([0] if i == 0 else [0, i], dtype=np.int64)
            lists[h][i] = np.union1d(forced, top)
            info[h][i] = (cand, sc, e)
    return lists, info, kbar
