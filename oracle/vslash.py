"""Vertical-slash index, fp64 (oracle; test infrastructure only).

MInference 1.0 page, section "方法介紹" (method): for the vertical-slash pattern
the attention between the last queries and all keys estimates which key
columns (vertical lines) and which diagonals (slash lines) matter.  Fig. 4 of
the same page: slash lines are computed as 64x64 blocks, vertical lines as
1x64 column tiles.

Readings taken where the pages are silent:
* the last ``last_q`` (= 64) queries, rows i_r = n - last_q + r, causal softmax
  with scale 1/sqrt(d) (the caller's ``scale``);
* the column score is the sum over those rows of the softmax probabilities,
  vert[j] = sum_r P[r, j]; the diagonal score is slash[o] = sum_r P[r, i_r - o];
* forced items count inside the kept totals: columns 0..63 are always among
  the ``n_vert`` kept columns, offset 0 among the ``n_slash`` kept offsets;
* the execution plan uses aligned 64x64 key blocks: a kept offset o touches
  key blocks qb - floor(o/64) and qb - ceil(o/64) (when >= 0) of query block
  qb whenever o <= 64*qb + 63; a kept column becomes a 1x64 column tile entry
  of query block qb when j <= 64*qb + 63 and its block is not already selected.
"""

from __future__ import annotations

import numpy as np

from .blocksel import select_top

BLOCK = 64


def vs_scores(q: np.ndarray, k: np.ndarray, last_q: int, scale: float, heads=None):
    """Column and diagonal scores of every q-head: (vert [Hq][n], slash [Hq][n])."""
    Hq, n, d = q.shape
    Hkv = k.shape[0]
    grp = Hq // Hkv
    heads = range(Hq) if heads is None else heads
    vert = {}
    slash = {}
    rows = np.arange(n - last_q, n)
    for h in heads:
        g = h // grp
        Z = (q[h, n - last_q:] @ k[g].T) * scale               # [last_q][n]
        Z[np.arange(n)[None, :] > rows[:, None]] = -np.inf   # causal: key j <= query i
        Z -= Z.max(axis=1, keepdims=True)
        P = np.exp(Z)
        P /= P.sum(axis=1, keepdims=True)
        vert[h] = P.sum(axis=0)
        s = np.zeros(n)
        for r, i in enumerate(rows):
            # offsets 0..i pair with keys i..0
            s[: i + 1] += P[r, i::-1]
        slash[h] = s
    return vert, slash


def vs_topk(vert: np.ndarray, slash: np.ndarray, n_vert: int, n_slash: int):
    """Kept columns (first 64 forced) and kept offsets (offset 0 forced), ascending.

    Returns (vert_idx, slash_off, vert_info, slash_info); the *_info tuples are
    (candidates, scores, count) for the near-tie check."""
    n = vert.shape[0]
    nf = min(BLOCK, n)
    cand_v = np.arange(nf, n, dtype=np.int64)
    ev = n_vert - nf
    top_v = select_top(vert[nf:], cand_v, ev)
    vert_idx = np.union1d(np.arange(nf, dtype=np.int64), top_v)
    cand_s = np.arange(1, n, dtype=np.int64)
    es = n_slash - 1
    top_s = select_top(slash[1:], cand_s, es)
    slash_off = np.union1d(np.zeros(1, dtype=np.int64), top_s)
    return vert_idx, slash_off, (cand_v, vert[nf:], ev), (cand_s, slash[1:], es)


def vs_plan(vert_idx: np.ndarray, slash_off: np.ndarray, n: int):
    """Per query block: (blocks ascending, columns ascending)."""
    nb = n // BLOCK
    slash_off = np.asarray(slash_off, dtype=np.int64)
    vert_idx = np.asarray(vert_idx, dtype=np.int64)
    plan = []
    for qb in range(nb):
        last = BLOCK * qb + BLOCK - 1
        o = slash_off[slash_off <= last]
        near = qb - o // BLOCK                    # qb - floor(o/64), always >= 0 here
        far = qb - (-((-o) // BLOCK))             # qb - ceil(o/64), may be -1
        blocks = np.union1d(near, far[far >= 0])
        j = vert_idx[vert_idx <= last]
        cols = j[~np.isin(j // BLOCK, blocks)]
        plan.append((blocks.astype(np.int64), np.sort(cols).astype(np.int64)))
    return plan


def vs_index(q, k, last_q, n_vert, n_slash, scale, heads=None):
    """Full vertical-slash index: {h: dict(vert, slash, vert_idx, slash_off, plan, ...)}."""
    n = q.shape[1]
    vert, slash = vs_scores(q, k, last_q, scale, heads)
    out = {}
    for h in vert:
        vi, so, vinfo, sinfo = vs_topk(vert[h], slash[h], n_vert, n_slash)
        out[h] = dict(vert=vert[h], slash=slash[h], vert_idx=vi, slash_off=so,
                      vert_info=vinfo, slash_info=sinfo, plan=vs_plan(vi, so, n))
    return out
