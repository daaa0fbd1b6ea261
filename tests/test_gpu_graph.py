"""The library calls inside a CUDA graph (-m gpu).

Every entry point launches only stream-ordered work on the caller's stream
(kernels and memsets; the workspace size query launches nothing), so after one
eager call has sized the workspace, a layer (index + attention) and a decode
step can be captured once and replayed.  The replays must reproduce the eager
results bit for bit: the kernels are deterministic."""
import pytest
import torch

import synth
import dynamic_sparse_attention_03_b200 as dsa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_prefill_layer_replays_from_a_graph():
    n, d, Hq, Hkv = 4096, 128, 8, 2
    w = synth.make_prefill("llama3-8b-32k-bs10", device=DEV, n=n, Hq=Hq, Hkv=Hkv, d=d, seed=41)
    ws = dsa.Workspace(DEV)
    kcap = dsa.block_index_capacity(n, 0, 0.1)
    bi = torch.empty((Hq, n // 64, kcap), dtype=torch.int32, device=DEV)
    bc = torch.empty((Hq, n // 64), dtype=torch.int32, device=DEV)
    o = torch.empty_like(w.q)

    def layer():
        dsa.sparse_index_estimate(w.q, w.k, keep_ratio=0.1, kcap=kcap, block_idx=bi, block_cnt=bc, ws=ws)
        dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer()                                   # sizes the workspace
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    want_bi, want_bc, want_o = bi.clone(), bc.clone(), o.clone()
    assert dsa.get_status(ws) == 0

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer()
    for _ in range(2):
        bi.fill_(-7)
        bc.fill_(-7)
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(bi, want_bi) and torch.equal(bc, want_bc)
        assert torch.equal(o, want_o)
    assert dsa.get_status(ws) == 0
    del g


def test_decode_step_replays_from_a_graph():
    B, Hq, Hkv, S, d, keep = 4, 32, 8, 16384, 128, 64
    w = synth.make_decode("decode-b16-128k", device=DEV, B=B, S=S, Hq=Hq, Hkv=Hkv, d=d, seed=43)
    ws = dsa.Workspace(DEV)
    cent = dsa.pool_keys(w.k_cache)
    o = torch.empty_like(w.q)

    def step():
        dsa.sparse_decode_attn(w.q, w.k_cache, w.v_cache, cent, keep=keep, out=o, ws=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    want = o.clone()
    assert dsa.get_status(ws) == 0

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, want)
    assert dsa.get_status(ws) == 0
    del g
