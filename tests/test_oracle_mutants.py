"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case swaps one oracle function for a plausible wrong variant (a dropped
term, a wrong index, a transposed operand, a wrong tie-break) on the CPU and
checks that at least one pin in test_oracle_pins.py then fails.
"""

import numpy as np
import pytest

import oracle
from oracle import attention as oatt
from oracle import blocksel as obi
from oracle import decode as odec
from oracle import ties as oties
from oracle import vslash as ovs
import tests.test_oracle_pins as pins


def _sum_pool(x, block=64):
    n, d = x.shape[-2], x.shape[-1]
    return np.asarray(x, dtype=np.float64).reshape(x.shape[:-2] + (n // block, block, d)).sum(axis=-2)


def _transposed_scores(qbar, kbar):
    return kbar @ qbar.T


def _no_causal_rows(q_rows, row_ids, k, v, blocks, cols, scale):
    keys = oatt._key_set(blocks, cols)
    Z = (q_rows @ k[keys].T) * scale
    m = Z.max(axis=1, keepdims=True)
    P = np.exp(Z - m)
    l = P.sum(axis=1, keepdims=True)
    return (P @ v[keys]) / l, (m + np.log(l))[:, 0]


def _unscaled_rows(q_rows, row_ids, k, v, blocks, cols, scale):
    return oatt.__dict__["_orig_rows"](q_rows, row_ids, k, v, blocks, cols, 1.0)


def _high_tie_select(scores, cand, e):
    if e <= 0 or cand.size == 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((-cand, -scores))
    return np.sort(cand[order[:e]])


def _slash_plus(q, k, last_q, scale, heads=None):
    vert, slash = ovs.__dict__["_orig_vs"](q, k, last_q, scale, heads)
    return vert, {h: np.roll(s, 1) for h, s in slash.items()}


def _tie_dropping(branch):
    """The near-tie comparison with one rejection branch removed: a set that
    only that branch rejects is accepted instead."""
    real = oties.__dict__["_orig_compare"]

    def cmp(got, forced, cand, scores, e, rel=oties.REL):
        st = real(got, forced, cand, scores, e, rel)
        return "ambiguous" if st == "MISMATCH: " + branch else st
    return cmp


def _tie_lower_bound_variant(sign, use_abs):
    """The near-tie comparison with the lower bound written as
    t_(k+1) + sign * rel * (|t_(k+1)| if use_abs else t_(k+1))."""
    def cmp(got, forced, cand, scores, e, rel=oties.REL):
        got = np.asarray(got, dtype=np.int64)
        forced = np.asarray(forced, dtype=np.int64)
        if got.size and np.any(np.diff(got) <= 0):
            return "MISMATCH: not strictly ascending"
        if not np.all(np.isin(forced, got)):
            return "MISMATCH: a forced element is missing"
        chosen = np.setdiff1d(got, forced)
        if chosen.size != e:
            return "MISMATCH: count"
        if not np.all(np.isin(chosen, cand)):
            return "MISMATCH: an id outside the candidates"
        if e == 0 or e == cand.size:
            return "exact"
        order = np.lexsort((cand, -scores))
        if np.array_equal(np.sort(cand[order[:e]]), chosen):
            return "exact"
        tk, tk1 = scores[order[e - 1]], scores[order[e]]
        if abs(tk - tk1) >= rel * max(abs(tk), abs(tk1)):
            return "MISMATCH: no near tie"
        upper = tk + rel * abs(tk)
        lower = tk1 + sign * rel * (abs(tk1) if use_abs else tk1)
        s_of = dict(zip(cand.tolist(), scores.tolist()))
        if not np.all(np.isin(cand[scores > upper], chosen)):
            return "MISMATCH: a clearly higher candidate was dropped"
        if any(s_of[int(c)] < lower for c in chosen):
            return "MISMATCH: a clearly lower candidate was kept"
        return "ambiguous"
    return cmp


TIE_MUTANTS = {
    "tie_no_lower_bound": lambda: _tie_dropping("a clearly lower candidate was kept"),
    "tie_no_ascending": lambda: _tie_dropping("not strictly ascending"),
    "tie_no_outside": lambda: _tie_dropping("an id outside the candidates"),
    "tie_lower_bound_sign": lambda: _tie_lower_bound_variant(+1.0, True),
    "tie_lower_bound_no_abs": lambda: _tie_lower_bound_variant(-1.0, False),
}


@pytest.mark.parametrize("case", sorted(TIE_MUTANTS))
def test_planted_tie_rule_mistake_is_caught(case, monkeypatch):
    monkeypatch.setitem(oties.__dict__, "_orig_compare", oties.compare_index_sets)
    mutant = TIE_MUTANTS[case]()
    monkeypatch.setattr(oracle, "compare_index_sets", mutant)
    with pytest.raises(AssertionError):
        pins.test_tie_rule_every_rejection_branch()


@pytest.mark.parametrize("case", ["sum_pool", "transposed", "no_causal", "unscaled", "high_tie", "slash_shift"])
def test_planted_mistake_is_caught(case, monkeypatch):
    if case == "sum_pool":
        monkeypatch.setattr(oracle, "pool_blocks", _sum_pool)
        monkeypatch.setattr(obi, "pool_blocks", _sum_pool)
        checks = [pins.test_pooled_score_commutes_with_matmul]
    elif case == "transposed":
        monkeypatch.setattr(oracle, "block_scores", _transposed_scores)
        monkeypatch.setattr(obi, "block_scores", _transposed_scores)
        checks = [pins.test_pooled_score_commutes_with_matmul]
    elif case == "no_causal":
        monkeypatch.setattr(oatt, "sparse_attention_rows", _no_causal_rows)
        checks = [pins.test_all_blocks_equals_dense_causal_sdpa]
    elif case == "unscaled":
        monkeypatch.setitem(oatt.__dict__, "_orig_rows", oatt.sparse_attention_rows)
        monkeypatch.setattr(oatt, "sparse_attention_rows", _unscaled_rows)
        checks = [pins.test_all_blocks_equals_dense_causal_sdpa]
    elif case == "high_tie":
        monkeypatch.setattr(oracle, "select_top", _high_tie_select)
        monkeypatch.setattr(odec, "select_top", _high_tie_select)
        checks = [pins.test_select_top_matches_python_sort, pins.test_decode_zero_query_keeps_lowest_blocks]
    else:
        monkeypatch.setitem(ovs.__dict__, "_orig_vs", ovs.vs_scores)
        monkeypatch.setattr(oracle, "vs_scores", _slash_plus)
        checks = [pins.test_vs_scores_closed_form_uniform]
    for chk in checks:
        with pytest.raises(AssertionError):
            chk()


# ---------------------------------------------------------------- K-means clusters

import tests.test_oracle_kmeans as kpins  # noqa: E402
from oracle import clusters as ocl  # noqa: E402


def _assign_no_cnorm(keys, cent):
    return np.argmin(-2.0 * (keys @ cent.T), axis=1).astype(np.int64)


def _assign_argmax(keys, cent):
    d2 = (keys * keys).sum(axis=1)[:, None] + (cent * cent).sum(axis=1)[None, :] - 2.0 * (keys @ cent.T)
    return np.argmax(d2, axis=1).astype(np.int64)


def _update_sum(keys, assign, cent):
    out = np.zeros_like(cent)
    np.add.at(out, assign, keys)
    return out


def _update_empty_zero(keys, assign, cent):
    C = cent.shape[0]
    sums = np.zeros_like(cent)
    np.add.at(sums, assign, keys)
    cnt = np.maximum(np.bincount(assign, minlength=C), 1).astype(np.float64)
    return sums / cnt[:, None]


def _csr_descending(assign, C):
    off, tok = ocl.__dict__["_orig_csr"](assign, C)
    tok = tok.copy()
    for c in range(C):
        tok[off[c]:off[c + 1]] = tok[off[c]:off[c + 1]][::-1]
    return off, tok


def _tokens_no_tail(clusters, off, tok, n_ctx, S):
    parts = [tok[off[c]:off[c + 1]] for c in np.asarray(clusters, dtype=np.int64)]
    return np.sort(np.concatenate(parts)) if parts else np.zeros(0, dtype=np.int64)


@pytest.mark.parametrize("case", ["no_cnorm", "argmax", "update_sum", "empty_zero", "csr_desc", "high_tie", "no_tail"])
def test_planted_kmeans_mistake_is_caught(case, monkeypatch):
    def patch(name, fn):
        monkeypatch.setattr(ocl, name, fn)
        monkeypatch.setattr(oracle, name, fn)

    if case == "no_cnorm":
        patch("kmeans_assign", _assign_no_cnorm)
        checks = [kpins.test_assign_matches_explicit_distance_bruteforce]
    elif case == "argmax":
        patch("kmeans_assign", _assign_argmax)
        checks = [kpins.test_assign_matches_explicit_distance_bruteforce, kpins.test_hand_worked_example]
    elif case == "update_sum":
        patch("kmeans_update", _update_sum)
        checks = [kpins.test_update_is_the_member_mean_and_keeps_empty_clusters, kpins.test_one_cluster_is_the_global_mean]
    elif case == "empty_zero":
        patch("kmeans_update", _update_empty_zero)
        checks = [kpins.test_update_is_the_member_mean_and_keeps_empty_clusters]
    elif case == "csr_desc":
        monkeypatch.setitem(ocl.__dict__, "_orig_csr", ocl.cluster_csr)
        patch("cluster_csr", _csr_descending)
        checks = [kpins.test_csr_is_a_stable_partition]
    elif case == "high_tie":
        monkeypatch.setattr(ocl, "select_top", _high_tie_select)
        checks = [kpins.test_zero_query_is_the_mean_over_kept_tokens]
    else:
        patch("cluster_tokens", _tokens_no_tail)
        checks = [kpins.test_keep_all_clusters_equals_dense_single_query_attention]
    for chk in checks:
        with pytest.raises(AssertionError):
            chk()
