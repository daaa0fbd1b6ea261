"""Stored expected values under tests/golden/ (written by tests/golden/make_golden.py
from the oracle alone) are reproduced by the oracle, and the planted key
blocks of the tiny workload are among the kept blocks wherever the budget
allows (a recall diagnostic: the pages fix no expected recall)."""
import os

import oracle
import synth

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_lists(name):
    out = {}
    for line in open(os.path.join(HERE, name)):
        if line.startswith("#"):
            continue
        i, rest = line.split(":")
        out[int(i)] = [int(x) for x in rest.split()]
    return out


def test_tiny_block_index_golden():
    want = read_lists("tiny_block_index.txt")
    w = synth.make_prefill("tiny-1h-1k-d64", device="cpu")
    lists, _, _ = oracle.block_index(synth.to_f64(w.q), synth.to_f64(w.k), k_fixed=4)
    assert {i: lists[0][i].tolist() for i in lists[0]} == want
    planted = w.planted[0]
    for i, sel in want.items():
        if i >= 3:
            cand_planted = [b for b in planted if 1 <= b < i]
            assert set(cand_planted[:2]) <= set(sel)
