"""The measurement arithmetic of bench.py, on CPU: the metric's name, the
selected-block FLOP count behind the effective TFLOP/s, and the index's
algorithmic bytes and fractions.  Each is checked against an independent count
from its definition (element by element, block by block), not against a
retyped formula."""
import math
import types

import numpy as np
import pytest
import torch

import bench


def test_metric_name_follows_the_workload():
    assert bench.metric_name("llama3-8b-32k-bs10").endswith("at 32K (selected-block FLOPs)")
    assert bench.metric_name("llama3-8b-128k-bs10").endswith("at 128K (selected-block FLOPs)")
    assert bench.metric_name("llama3-8b-1m-bs2").endswith("at 1M (selected-block FLOPs)")


def _causal_flops_brute(block_cnt, d):
    """4*d FLOP (QK^T and PV, one multiply-add each) per visible (query, key)
    pair, counted pair by pair: an off-diagonal block has 64 x 64 visible
    pairs, the diagonal block those with key <= query."""
    tot = 0
    for cnt in block_cnt.reshape(-1).tolist():
        if cnt <= 0:
            continue
        off = cnt - 1
        diag = sum(1 for r in range(64) for c in range(64) if c <= r)
        tot += (off * 64 * 64 + diag) * 4 * d
    return tot


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_flops_matches_a_pair_count(d):
    rng = np.random.default_rng(5)
    bc = torch.from_numpy(rng.integers(1, 40, size=(3, 17)).astype(np.int32))
    assert bench.prefill_flops(bc, d) == _causal_flops_brute(bc, d)


def test_prefill_flops_of_a_dense_causal_layer():
    """Every block selected: the count is the dense causal attention's
    4*d*n(n+1)/2 (the form the dense comparator uses)."""
    n, d, H = 1024, 128, 2
    nqb = n // 64
    bc = torch.tensor([[qb + 1 for qb in range(nqb)]] * H, dtype=torch.int32)
    assert bench.prefill_flops(bc, d) == 4.0 * d * H * n * (n + 1) / 2


def test_index_roofline_bytes_and_fractions():
    """Q and K read once as bf16 plus the lists written once (kcap ids and a
    count per row), over the measured time, against the given peaks."""
    Hq, Hkv, n, d, kcap = 4, 2, 4096, 128, 30
    w = types.SimpleNamespace(q=torch.empty(Hq, n, d, dtype=torch.bfloat16),
                              k=torch.empty(Hkv, n, d, dtype=torch.bfloat16))
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 500.0}
    r = bench.index_roofline(w, kcap, 0.5, peaks)
    q_bytes = Hq * n * d * 2
    k_bytes = Hkv * n * d * 2
    list_bytes = Hq * (n // 64) * (kcap + 1) * 4
    assert r["bytes"] == q_bytes + k_bytes + list_bytes
    assert math.isclose(r["achieved"], round(r["bytes"] / 0.5e-3 / 1e9, 1))
    assert math.isclose(r["frac"], round(r["bytes"] / 0.5e-3 / 1e9 / 1000.0, 4))
    # the scores: 2*d FLOP per causal (query block, key block) pair
    nqb = n // 64
    pairs = sum(qb + 1 for qb in range(nqb))
    assert r["score_flops"] == 2.0 * d * Hq * pairs
