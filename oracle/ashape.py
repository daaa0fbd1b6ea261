"""A-shape (sink + local window) block index, fp64-free integer oracle (test
infrastructure only).

MInference 1.0 page, method section ("方法介紹"): attention in long contexts
shows three spatial patterns, A-shape, vertical-slash and block-sparse.  The
A-shape keeps the first tokens (attention sink) and a local window of recent
tokens, the same for every input.  Reading taken here: at 64-token block
granularity, query block qb keeps key blocks 0 .. min(n_sink, qb+1)-1 and
max(0, qb-n_local+1) .. qb, as one ascending list without duplicates.
"""

from __future__ import annotations

import numpy as np


def a_shape_lists(n_blocks: int, n_sink: int, n_local: int):
    """{qb: ascending int64 array of kept key blocks}."""
    out = {}
    for qb in range(n_blocks):
        sink = set(range(min(n_sink, qb + 1)))
        local = set(range(max(0, qb - n_local + 1), qb + 1))
        out[qb] = np.array(sorted(sink | local), dtype=np.int64)
    return out
