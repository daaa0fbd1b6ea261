"""Index-set comparison with the near-tie rule (oracle side; test infrastructure only).

The problem statement fixes index parity as bit-exact, except where the
oracle's k-th and (k+1)-th candidate scores differ by less than 1e-4
relative: there several sets are correct.  In such an ambiguous row the set
under test must still hold every forced element, every candidate scoring
clearly above the k-th score, no candidate scoring clearly below the
(k+1)-th, and exactly k non-forced candidates.
"""

from __future__ import annotations

import numpy as np

REL = 1e-4


def compare_index_sets(got, forced, cand, scores, e, rel: float = REL):
    """Return "exact", "ambiguous" (an accepted near-tie row) or a string
    starting with "MISMATCH" that says what is wrong.

    got: ascending ids produced by the code under test (forced included);
    forced: ids that must always be present; cand/scores: the oracle's
    candidates and fp64 scores; e: number of candidates to keep."""
    got = np.asarray(got, dtype=np.int64)
    forced = np.asarray(forced, dtype=np.int64)
    if got.size and np.any(np.diff(got) <= 0):
        return "MISMATCH: not strictly ascending"
    if not np.all(np.isin(forced, got)):
        return "MISMATCH: a forced element is missing"
    chosen = np.setdiff1d(got, forced)
    if chosen.size != e:
        return f"MISMATCH: {chosen.size} non-forced ids, expected {e}"
    if not np.all(np.isin(chosen, cand)):
        return "MISMATCH: an id outside the candidates"
    if e == 0 or e == cand.size:
        return "exact"
    order = np.lexsort((cand, -scores))
    ref = np.sort(cand[order[:e]])
    if np.array_equal(ref, chosen):
        return "exact"
    tk = scores[order[e - 1]]
    tk1 = scores[order[e]]
    if abs(tk - tk1) >= rel * max(abs(tk), abs(tk1)):
        return "MISMATCH: differs from the oracle in a row without a near tie"
    upper = tk + rel * abs(tk)
    lower = tk1 - rel * abs(tk1)
    s_of = dict(zip(cand.tolist(), scores.tolist()))
    must = cand[scores > upper]
    if not np.all(np.isin(must, chosen)):
        return "MISMATCH: a clearly higher candidate was dropped"
    if any(s_of[int(c)] < lower for c in chosen):
        return "MISMATCH: a clearly lower candidate was kept"
    return "ambiguous"
