"""A bounded wait that runs out, and the recovery after it (-m gpu).

Every wait inside the library's kernels gives up after a time limit, records
DSA_ERR_TIMEOUT in the workspace's status word and lets the CTA leave with
nothing in flight, so the context stays usable.  The test makes one wait run
out on purpose through the library's fault-injection switch
(DSA_FAULT_INJECT=attn_stall): the first work item of block_sparse_attn_fwd
issues no load for its first K tile (so nothing is left in flight) and the
waits give up after 1 ms.  Nothing faults, traps or hangs.

The sequence checked: the stalled call returns DSA_OK (it is asynchronous);
dsa_get_status then reports DSA_ERR_TIMEOUT and clears the word; a later call
on the same workspace computes the same output as before the stall.
"""

import math
import time

import pytest
import torch

import oracle
import synth
import dynamic_sparse_attention_03_b200 as dsa
from tests.parity import check_attention, f64, lists_from_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_attention_wait_runs_out_then_recovers(monkeypatch):
    n, d, Hq, Hkv = 4096, 128, 8, 2
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=31)
    ws = dsa.Workspace(DEV)
    bi, bc = dsa.sparse_index_estimate(w.q, w.k, keep_ratio=0.25, ws=ws)
    ref = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, ws=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0

    monkeypatch.setenv("DSA_FAULT_INJECT", "attn_stall")
    out = torch.zeros_like(ref)
    t0 = time.perf_counter()
    dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=out, ws=ws)   # returns DSA_OK: asynchronous
    torch.cuda.synchronize()
    stalled_s = time.perf_counter() - t0
    monkeypatch.delenv("DSA_FAULT_INJECT")
    assert stalled_s < 5.0, stalled_s                      # the 1 ms waits ended the call
    assert dsa.get_status(ws) == -5                        # DSA_ERR_TIMEOUT, now cleared
    assert dsa.get_status(ws) == 0

    again = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, ws=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0
    assert torch.equal(again, ref)
    got = lists_from_gpu(bi, bc)
    items = [(h, qb) for h in (0, Hq - 1) for qb in (0, 17, n // 64 - 1)]
    want = oracle.sparse_attention(f64(w.q), f64(w.k), f64(w.v), got, None, 1 / math.sqrt(d), items=items)
    check_attention(again, want, "after a timeout")


def test_timeout_is_sticky_until_read(monkeypatch):
    """Until dsa_get_status clears it, a recorded timeout makes later launches
    on the same workspace return at once (their CTAs exit at entry): the
    output buffer keeps what it held.  Reading the status clears it."""
    n, d, Hq, Hkv = 2048, 64, 4, 1
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=32)
    ws = dsa.Workspace(DEV)
    bi, bc = dsa.sparse_index_estimate(w.q, w.k, keep_ratio=0.25, ws=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0
    monkeypatch.setenv("DSA_FAULT_INJECT", "attn_stall")
    dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, ws=ws)
    monkeypatch.delenv("DSA_FAULT_INJECT")
    sentinel = torch.full_like(w.q, 7.0)
    dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=sentinel, ws=ws)
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0)                      # skipped: the word still holds the timeout
    assert dsa.get_status(ws) == -5
    fresh = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=sentinel, ws=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0
    assert not torch.any(torch.isnan(fresh.float())) and not torch.all(fresh == 7.0)
