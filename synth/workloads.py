"""Seeded synthetic workloads.

Shapes and planted structure follow the workloads of the MInference 1.0 page
("MInference 1.0: Accelerating Pre-filling for Long-Context LLMs via Dynamic
Sparse Attention", sections on the three sparse patterns and Fig. 3/Fig. 4)
and of the Squeezed Attention page (section "技术方案", online stage):

* block-sparse prefill: Q, K, V ~ N(0, sigma^2); a seeded unit vector ``u`` per
  KV head; a fraction of the 64-token key blocks gets ``K += 1.5 u`` and every
  query of that head group gets ``Q += u``, so those key blocks score high;
* vertical-slash prefill: 200 key columns get ``K += 2 u`` (strong verticals)
  and a periodic component makes 50 diagonals strong (slashes);
* decode: a fixed KV cache with the same planted block structure per
  (batch, KV head) and one query token per sequence.

Small structural choices (u, planted block ids, columns, frequencies, offsets)
are drawn on the host with NumPy's PCG64 so they do not depend on the device;
the large Gaussian tensors are drawn with torch's generator on the device the
caller names, in fp32, then rounded to bf16 (round to nearest even).  The bf16
tensors returned are the shared truth for the CUDA path and for the oracle.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

BLOCK = 64

# name -> parameters.  Names say what the workload is.
CONFIGS = {
    # 1 head, 1K tokens, head_dim 64; 4 blocks per query block incl. sink+diag.
    "tiny-1h-1k-d64": dict(kind="block", Hq=1, Hkv=1, n=1024, d=64, sigma=1 / math.sqrt(8.0),
                           plant_frac=0.10, k_fixed=4, keep_ratio=0.0, seed=20260),
    # LLaMA-3-8B-shaped layer at 32K, keep 10% of causal blocks plus sink+diag.
    "llama3-8b-32k-bs10": dict(kind="block", Hq=32, Hkv=8, n=32768, d=128, sigma=1.0,
                               plant_frac=0.10, k_fixed=0, keep_ratio=0.10, seed=20261),
    # Same generator at 128K (the block-sparse 128K prefill point).
    "llama3-8b-128k-bs10": dict(kind="block", Hq=32, Hkv=8, n=131072, d=128, sigma=1.0,
                                plant_frac=0.10, k_fixed=0, keep_ratio=0.10, seed=20265),
    # Vertical-slash at 128K: 1000 columns, 4096 diagonals from the last 64 queries.
    "llama3-8b-128k-vs": dict(kind="vs", Hq=32, Hkv=8, n=131072, d=128, sigma=1.0,
                              n_cols_planted=200, n_diag_planted=50, n_vert=1000, n_slash=4096,
                              last_q=64, seed=20262),
    # 1M tokens, keep 2% of causal blocks plus sink+diag.
    "llama3-8b-1m-bs2": dict(kind="block", Hq=32, Hkv=8, n=1048576, d=128, sigma=1.0,
                             plant_frac=0.02, k_fixed=0, keep_ratio=0.02, seed=20263),
    # Decode over a fixed 128K cache, batch 16, keep 512 blocks + the last one.
    "decode-b16-128k": dict(kind="decode", B=16, Hq=32, Hkv=8, S=131072, d=128, sigma=1.0,
                            plant_frac=0.05, keep=512, force_last=1, seed=20264),
}


def planted_count(n_blocks: int, frac: float) -> int:
    """Number of planted key blocks: the fraction of all key blocks, rounded."""
    return int(round(frac * n_blocks))


@dataclasses.dataclass
class Workload:
    name: str
    q: torch.Tensor          # [Hq][n][d] bf16
    k: torch.Tensor          # [Hkv][n][d] bf16
    v: torch.Tensor          # [Hkv][n][d] bf16
    params: dict
    planted: list            # per KV head: sorted planted block ids (block kind) or columns (vs)


@dataclasses.dataclass
class DecodeWorkload:
    name: str
    q: torch.Tensor          # [B][Hq][d] bf16
    k_cache: torch.Tensor    # [B][Hkv][S][d] bf16
    v_cache: torch.Tensor    # [B][Hkv][S][d] bf16
    params: dict
    planted: list            # [B][Hkv] sorted planted block ids


def _unit(rng: np.random.Generator, d: int) -> np.ndarray:
    u = rng.standard_normal(d)
    return u / np.linalg.norm(u)


def _gauss(shape, sigma: float, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x


def _seed(base: int, tensor_id: int, head: int) -> int:
    return (base * 1_000_003 + tensor_id * 10_007 + head) % (2**62)


def make_prefill(name: str, device="cpu", n: Optional[int] = None, Hq: Optional[int] = None,
                 Hkv: Optional[int] = None, d: Optional[int] = None, seed: Optional[int] = None) -> Workload:
    """Build a prefill workload by name; ``n``/``Hq``/``Hkv``/``d`` override the
    named shape (used for small parity cases with the same recipe)."""
    p = dict(CONFIGS[name])
    if p["kind"] not in ("block", "vs"):
        raise ValueError(f"{name} is not a prefill workload")
    for key, val in (("n", n), ("Hq", Hq), ("Hkv", Hkv), ("d", d), ("seed", seed)):
        if val is not None:
            p[key] = val
    Hq_, Hkv_, n_, d_ = p["Hq"], p["Hkv"], p["n"], p["d"]
    assert n_ % BLOCK == 0 and Hq_ % Hkv_ == 0
    grp = Hq_ // Hkv_
    nb = n_ // BLOCK
    base = p["seed"]
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(base)))
    q = torch.empty((Hq_, n_, d_), dtype=torch.bfloat16, device=device)
    k = torch.empty((Hkv_, n_, d_), dtype=torch.bfloat16, device=device)
    v = torch.empty((Hkv_, n_, d_), dtype=torch.bfloat16, device=device)
    planted = []
    sigma = p["sigma"]
    if p["kind"] == "vs":
        n_freq = d_ // 2
        t = torch.arange(n_, device=device, dtype=torch.float64)
    for g in range(Hkv_):
        u_np = _unit(rng, d_)
        u = torch.tensor(u_np, dtype=torch.float32, device=device)
        kg = _gauss((n_, d_), sigma, _seed(base, 1, g), device)
        if p["kind"] == "block":
            cnt = planted_count(nb, p["plant_frac"])
            blocks = np.sort(rng.choice(nb, size=cnt, replace=False))
            planted.append(blocks.tolist())
            if cnt:
                rows = (torch.tensor(blocks, device=device)[:, None] * BLOCK
                        + torch.arange(BLOCK, device=device)[None, :]).reshape(-1)
                kg[rows] += 1.5 * u
            q_extra = u[None, :]
        else:
            cols = np.sort(rng.choice(n_, size=p["n_cols_planted"], replace=False))
            planted.append(cols.tolist())
            kg[torch.tensor(cols, device=device)] += 2.0 * u
            omega = torch.tensor(rng.uniform(0.0, math.pi, n_freq), dtype=torch.float64, device=device)
            offs = torch.tensor(rng.integers(1, n_, size=p["n_diag_planted"]), dtype=torch.float64,
                                device=device)
            # phi(t) = [cos(w t), sin(w t)] / 8 ; Q_i += 8 phi(i);
            # K_j += (8/sqrt(m)) * sum_m phi(j + o_m), summed with the angle-addition identity.
            wt = t[:, None] * omega[None, :]
            cwt, swt = torch.cos(wt), torch.sin(wt)
            wo = offs[:, None] * omega[None, :]
            C, S = torch.cos(wo).sum(0), torch.sin(wo).sum(0)
            amp = (8.0 / math.sqrt(p["n_diag_planted"])) / 8.0
            k_per = torch.cat([cwt * C - swt * S, swt * C + cwt * S], dim=1) * amp
            kg += k_per.to(torch.float32)
            q_extra = u[None, :] + torch.cat([cwt, swt], dim=1).to(torch.float32)  # 8 * phi(i)
            del wt, cwt, swt, k_per
        k[g] = kg.to(torch.bfloat16)
        del kg
        v[g] = _gauss((n_, d_), sigma, _seed(base, 2, g), device).to(torch.bfloat16)
        for hh in range(grp):
            h = g * grp + hh
            qh = _gauss((n_, d_), sigma, _seed(base, 0, h), device)
            qh += q_extra
            q[h] = qh.to(torch.bfloat16)
            del qh
    return Workload(name=name, q=q, k=k, v=v, params=p, planted=planted)


def make_decode(name: str = "decode-b16-128k", device="cpu", B: Optional[int] = None,
                S: Optional[int] = None, Hq: Optional[int] = None, Hkv: Optional[int] = None,
                d: Optional[int] = None, seed: Optional[int] = None) -> DecodeWorkload:
    p = dict(CONFIGS[name])
    if p["kind"] != "decode":
        raise ValueError(f"{name} is not a decode workload")
    for key, val in (("B", B), ("S", S), ("Hq", Hq), ("Hkv", Hkv), ("d", d), ("seed", seed)):
        if val is not None:
            p[key] = val
    B_, Hq_, Hkv_, S_, d_ = p["B"], p["Hq"], p["Hkv"], p["S"], p["d"]
    assert S_ % BLOCK == 0 and Hq_ % Hkv_ == 0
    grp = Hq_ // Hkv_
    nb = S_ // BLOCK
    base = p["seed"]
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(base)))
    q = torch.empty((B_, Hq_, d_), dtype=torch.bfloat16, device=device)
    kc = torch.empty((B_, Hkv_, S_, d_), dtype=torch.bfloat16, device=device)
    vc = torch.empty((B_, Hkv_, S_, d_), dtype=torch.bfloat16, device=device)
    planted = []
    sigma = p["sigma"]
    cnt = planted_count(nb, p["plant_frac"])
    for b in range(B_):
        row = []
        for g in range(Hkv_):
            u = torch.tensor(_unit(rng, d_), dtype=torch.float32, device=device)
            blocks = np.sort(rng.choice(nb, size=cnt, replace=False))
            row.append(blocks.tolist())
            kg = _gauss((S_, d_), sigma, _seed(base, 1, b * Hkv_ + g), device)
            if cnt:
                rows = (torch.tensor(blocks, device=device)[:, None] * BLOCK
                        + torch.arange(BLOCK, device=device)[None, :]).reshape(-1)
                kg[rows] += 1.5 * u
            kc[b, g] = kg.to(torch.bfloat16)
            del kg
            vc[b, g] = _gauss((S_, d_), sigma, _seed(base, 2, b * Hkv_ + g), device).to(torch.bfloat16)
            qg = _gauss((grp, d_), sigma, _seed(base, 0, b * Hkv_ + g), device) + u[None, :]
            q[b, g * grp:(g + 1) * grp] = qg.to(torch.bfloat16)
        planted.append(row)
    return DecodeWorkload(name=name, q=q, k_cache=kc, v_cache=vc, params=p, planted=planted)


def to_f64(x: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 tensor to a NumPy fp64 array on the host."""
    return x.detach().to("cpu", torch.float32).numpy().astype(np.float64)
