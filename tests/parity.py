"""Helpers shared by the GPU parity tests: compare CUDA outputs with the fp64
oracle (index sets under the near-tie rule, attention outputs under the
max/mean absolute error bars)."""

from __future__ import annotations

import collections

import numpy as np
import torch

import oracle

# Output parity bar for bf16 inputs with fp32 accumulation (problem statement).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def lists_from_gpu(idx: torch.Tensor, cnt: torch.Tensor):
    """{h: {qb: ascending np.int64 array}} from [H][nQB][cap] / [H][nQB] tensors."""
    idx_h = idx.cpu().numpy()
    cnt_h = cnt.cpu().numpy()
    out = {}
    for h in range(idx_h.shape[0]):
        out[h] = {}
        for qb in range(idx_h.shape[1]):
            c = int(cnt_h[h, qb])
            row = idx_h[h, qb]
            assert 0 <= c <= row.shape[0]
            assert np.all(row[c:] == -1), "padding after the count must be -1"
            out[h][qb] = row[:c].astype(np.int64)
    return out


def check_block_index(gpu_lists, info, label=""):
    """Near-tie comparison of every (h, i) row the oracle computed."""
    stats = collections.Counter()
    bad = []
    for h in info:
        for i, (cand, sc, e) in info[h].items():
            forced = [0] if i == 0 else [0, i]
            st = oracle.compare_index_sets(gpu_lists[h][i], forced, cand, sc, e)
            stats[st.split(":")[0]] += 1
            if st.startswith("MISMATCH"):
                bad.append((h, i, st))
    print(f"[index parity {label}] {dict(stats)}")
    assert not bad, bad[:5]
    return stats


def check_attention(o_gpu: torch.Tensor, ref: dict, label=""):
    """ref: {(h, qb): (O [64][d], lse)} from the oracle; o_gpu [H][n][d] bf16."""
    errs = []
    mx = 0.0
    for (h, qb), (O, _) in ref.items():
        g = f64(o_gpu[h, qb * 64:(qb + 1) * 64])
        e = np.abs(g - O)
        mx = max(mx, float(e.max()))
        errs.append(e.mean())
    mean = float(np.mean(errs))
    print(f"[attention parity {label}] items={len(ref)} max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    return mx, mean
