"""Benchmark of the dynamic-sparse-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-decode] [--no-vs] [--no-e2e] [--no-cpu-baseline]
                    [--no-layers] [--sustained-s S]

A step is one prefill layer of the block-sparse path on the named workload
(default: the LLaMA-3-8B-shaped layer at 128K tokens, 32 q-heads / 8 KV
heads, d=128, keep 10% of causal blocks plus sink and diagonal): the block
index (sparse_index_estimate) followed by causal block-sparse attention
(block_sparse_attn_fwd), with inputs resident in HBM.  The metric is the
effective TFLOP/s counting only the FLOPs of the selected blocks (diagonal
blocks at their causal 2080 of 4096 elements); ms_per_step is ms per layer.
The sparse decode GB/s (batch 16, 128K cache, keep 512 + the last block) is
reported beside it under "decode", the vertical-slash layer under
"vertical_slash", and the 32K and 1M block-sparse layers under "layers".
"roofline" holds the attention kernel against the burst tensor peak (a few
launches timed back to back); "roofline_sustained" the same kernel launched
back to back for a few seconds against the sustained peak.

One JSON line is printed by rank 0.  Multi-GPU (torchrun): every rank runs its
own independent layer (weak scaling, no data-path collective); timing is the
max over ranks of the device time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

# DRAM bytes (read + write) of one bsa_fwd_kernel launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of this bench's command, kept
# with the kernel revision they were taken on (profiles/ holds the summary);
# the line reports null for any other revision or workload.
BSA_KERNEL_REVISION = "tile-skip-2"
BSA_TRAFFIC = {("tile-skip-2", "llama3-8b-128k-bs10"): 1.69e9 + 1.02e9}   # {(revision, workload): bytes}
UNIT = "TFLOP/s"
DIAG_ELEMS = 64 * 65 // 2


def metric_name(workload: str) -> str:
    """The headline metric, named for the workload's sequence length."""
    n = synth.CONFIGS[workload]["n"]
    label = f"{n // (1 << 20)}M" if n >= (1 << 20) else f"{n // 1024}K"
    return f"block-sparse prefill effective TFLOP/s at {label} (selected-block FLOPs)"


def prefill_flops(block_cnt: torch.Tensor, d: int) -> float:
    """Selected-block FLOPs: 4*64*64*d per off-diagonal block (QK^T and PV), the
    diagonal block at its 2080 causal elements.  Every block-sparse row holds its
    diagonal block."""
    cnt = block_cnt.to(torch.float64)
    return float(((cnt - 1).clamp(min=0) * 4 * 64 * 64 * d + 4 * DIAG_ELEMS * d).sum().item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.skip = 0

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # nvidia-smi takes a moment to start: the timed region begins once it samples
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0:
                time.sleep(0.02)
            self.skip = len(self.lines)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        mhz, maxmhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[self.skip:] or self.lines[-1:]:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                maxmhz = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": maxmhz, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": maxmhz, "reasons": sorted(reasons),
                "samples": len(mhz)}


def dist_setup(ngpus: int):
    if ngpus <= 1 and "RANK" not in os.environ:
        return 0, 1, 0
    import datetime

    import torch.distributed as dist

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload: str, rank: int) -> int:
    """Each rank runs its own independent layer: the workload's seed offset by rank."""
    return synth.CONFIGS[workload]["seed"] + 1000 * rank


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------ our arm

def workload_config(workload: str, world: int, hq=None, hkv=None) -> dict:
    """The prefill workload's description, the same on both arms."""
    p = synth.CONFIGS[workload]
    kf, rho = p.get("k_fixed", 0), p.get("keep_ratio", 0.0)
    return {"workload": workload, "Hq": hq or p["Hq"], "Hkv": hkv or p["Hkv"], "seq_len": p["n"], "head_dim": p["d"],
            "keep": f"k_fixed={kf}" if kf else f"ratio={rho}+sink+diag", "block": 64,
            "l2": "inputs larger than L2 (Q 1.07 GB, K/V 268 MB each at 128K), no flush",
            "parallelism": f"independent layer per GPU x{world}"}


def run_ours(args, rank, world, local):
    import dynamic_sparse_attention_03_b200 as dsa

    dsa.load_library()
    dev = torch.device("cuda", local)
    p = synth.CONFIGS[args.workload]
    w = synth.make_prefill(args.workload, device=dev, seed=rank_seed(args.workload, rank), Hq=args.hq, Hkv=args.hkv)
    Hq, n, d = w.q.shape
    kf, rho = p.get("k_fixed", 0), p.get("keep_ratio", 0.0)
    kcap = dsa.block_index_capacity(n, kf, rho)
    bi = torch.empty((Hq, n // 64, kcap), dtype=torch.int32, device=dev)
    bc = torch.empty((Hq, n // 64), dtype=torch.int32, device=dev)
    o = torch.empty_like(w.q)
    ws = dsa.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        dsa.sparse_index_estimate(w.q, w.k, k_fixed=kf, keep_ratio=rho, kcap=kcap, block_idx=bi, block_cnt=bc, ws=ws)
        dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flops = prefill_flops(bc, d)
    launches_per_step = 5   # pool K, pool Q, fused block score + top-k, block lists, attention
    # timed region
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    # the index and the attention kernel alone, same stream, for the rooflines:
    # single launches after an idle second, as the burst peaks were measured
    reps = max(3, min(args.steps, 5))
    index_ms, index_best, _ = burst_ms(
        lambda: dsa.sparse_index_estimate(w.q, w.k, k_fixed=kf, keep_ratio=rho, kcap=kcap, block_idx=bi,
                                          block_cnt=bc, ws=ws), reps, stream)
    attn_ms, attn_best, attn_clk = burst_ms(lambda: dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws),
                                            reps, stream)
    # cross-layer index reuse (IndexCache's "full" vs "shared" layers): four
    # layers each estimating their own index, against one estimate shared by
    # all four; the same tensors stand in for every layer (timing only)
    # (the two orders alternate over 3 trials and the medians are kept, so a
    # clock drift during the runs does not favour either)
    nl = 4
    every, once = [], []
    for trial in range(3):
        r0, r1, r2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))

        def every_layer():
            for _ in range(nl):
                step()

        def index_once():
            dsa.sparse_index_estimate(w.q, w.k, k_fixed=kf, keep_ratio=rho, kcap=kcap, block_idx=bi, block_cnt=bc,
                                      ws=ws)
            for _ in range(nl):
                dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws)

        first, second = (every_layer, index_once) if trial % 2 == 0 else (index_once, every_layer)
        r0.record(stream)
        first()
        r1.record(stream)
        second()
        r2.record(stream)
        torch.cuda.synchronize()
        t_first, t_second = r0.elapsed_time(r1), r1.elapsed_time(r2)
        every.append(t_first if trial % 2 == 0 else t_second)
        once.append(t_second if trial % 2 == 0 else t_first)
    e_ms, o_ms = statistics.median(every), statistics.median(once)
    reuse = {"layers": nl, "index_every_layer_ms": round(e_ms, 3), "index_once_ms": round(o_ms, 3),
             "speedup": round(e_ms / o_ms, 4), "trials": 3}
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, world)
    status = dsa.get_status(ws)
    value = flops * world / (ms * 1e-3) / 1e12
    peaks, src = load_peaks()
    achieved = flops / (attn_ms * 1e-3) / 1e12
    # the attention above is timed as single launches of an idle GPU: the burst
    # peak applies.  A seconds-long run of the same kernel, held against the
    # sustained peak, is reported beside it.
    peak = peaks["bf16_tflops"]
    sustained = sustained_attention(dsa, w, bi, bc, o, ws, stream, flops, peaks, seconds=args.sustained_s)
    density = float(bc.to(torch.float64).sum().item()) / (Hq * (n // 64) * (n // 64 + 1) / 2)
    index_roof = index_roofline(w, kcap, index_ms, peaks)
    res = {
        "metric": metric_name(args.workload), "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(args.workload, world, args.hq, args.hkv), selected_block_density=round(density, 5)),
        "breakdown_ms": {"index": round(index_ms, 4), "attention": round(attn_ms, 4)},
        "index_roofline": index_roof,
        "index_reuse": reuse,
        "effective_flops_per_step": flops,
        "roofline": {"bound": "tensor", "kernel": "bsa_fwd_kernel<128>", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": BSA_TRAFFIC.get((BSA_KERNEL_REVISION, args.workload)),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch of this "
                                       f"kernel revision ({BSA_KERNEL_REVISION})",
                     "peak_source": f"{src} bf16_tflops (burst: median of {reps} single launches after 1 s idle)",
                     "timed_launches": reps, "ms": round(attn_ms, 4), "best_ms": round(attn_best, 4),
                     "clocks": attn_clk},
        "roofline_sustained": sustained,
        "clocks": clk.summary(),
        "gpu_launches": (launches_per_step * args.steps) if launches_per_step else None,
        "device_status": status,
    }
    return res, (w, bi, bc, kf, rho, kcap, flops, ws)


def index_roofline(w, kcap, index_ms, peaks):
    """The block index call held against the HBM copy peak (algorithmic bytes:
    Q and K read once as bf16, the lists written once) and, for its scoring,
    against the tensor peak (FP16 products issued: one per approximate pass,
    three per exact pass, 2*d FLOP per causal (query block, key block) pair;
    the statistics pass of long rows reads every 4th key chunk)."""
    Hq, n, d = w.q.shape
    nqb = n // 64
    pairs = Hq * nqb * (nqb + 1) / 2
    idx_bytes = (Hq + w.k.shape[0]) * n * d * 2 + Hq * nqb * (kcap + 1) * 4
    stats_share = 1.0 if nqb <= 512 else 0.25
    tensor_flops = 2.0 * d * pairs * (stats_share + 1 + 3)
    gbs = idx_bytes / (index_ms * 1e-3) / 1e9
    tfs = tensor_flops / (index_ms * 1e-3) / 1e12
    return {"kernels": "pool_blocks (K, Q) + block_topk + block_list", "bound": "hbm", "achieved": round(gbs, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": idx_bytes,
            "score_flops": 2.0 * d * pairs, "score_fp16_split_products": 3,
            "tensor": {"flops_issued": tensor_flops, "achieved_tflops": round(tfs, 1), "peak": peaks["bf16_tflops"],
                       "frac": round(tfs / peaks["bf16_tflops"], 4),
                       "note": "FP16 kind::f16 products, same rate as bf16"}}


def burst_ms(fn, reps, stream, idle_s=1.0):
    """A kernel timed alone, as the burst peak was measured (single launches of
    an idle GPU): the GPU idles for `idle_s`, then `reps` launches run back to
    back, each bracketed by CUDA events on its stream.  Returns the median and
    the best per-launch ms and the clocks sampled meanwhile."""
    torch.cuda.synchronize()
    time.sleep(idle_s)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev[0].record(stream)
        for i in range(reps):
            fn()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]
    return statistics.median(per), min(per), clk.summary()


def sustained_attention(dsa, w, bi, bc, o, ws, stream, flops, peaks, seconds):
    """The attention launched back to back for about `seconds` (a long step: the
    sustained peak applies), timed with CUDA events on its stream."""
    if seconds <= 0:
        return None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = max(2, int(seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3)))
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(launches):
            dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / launches
    tf = flops / (ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    return {"launches": launches, "seconds": round(ms * launches / 1e3, 2), "ms": round(ms, 4),
            "achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s", "frac": round(tf / peak, 4),
            "peak_source": "bf16_tflops_sustained", "clocks": clk.summary()}


def run_layers(args, local, names):
    """The other block-sparse prefill layers (index + attention each), for the
    workloads' own sizes: ms per layer, effective TFLOP/s of the attention
    against the tensor peak, and the index against HBM (and, for its scoring,
    the tensor peak)."""
    import dynamic_sparse_attention_03_b200 as dsa

    dev = torch.device("cuda", local)
    peaks, src = load_peaks()
    out = {}
    for name in names:
        p = synth.CONFIGS[name]
        w = synth.make_prefill(name, device=dev)
        Hq, n, d = w.q.shape
        kf, rho = p.get("k_fixed", 0), p.get("keep_ratio", 0.0)
        kcap = dsa.block_index_capacity(n, kf, rho)
        bi = torch.empty((Hq, n // 64, kcap), dtype=torch.int32, device=dev)
        bc = torch.empty((Hq, n // 64), dtype=torch.int32, device=dev)
        o = torch.empty_like(w.q)
        ws = dsa.Workspace(dev)
        stream = torch.cuda.current_stream(dev)
        reps = 3 if n > 200000 else 5
        for _ in range(2):
            dsa.sparse_index_estimate(w.q, w.k, k_fixed=kf, keep_ratio=rho, kcap=kcap, block_idx=bi, block_cnt=bc,
                                      ws=ws)
            dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws)
        index_ms, _, _ = burst_ms(lambda: dsa.sparse_index_estimate(w.q, w.k, k_fixed=kf, keep_ratio=rho, kcap=kcap,
                                                                     block_idx=bi, block_cnt=bc, ws=ws), reps, stream)
        attn_ms, attn_best, clk = burst_ms(lambda: dsa.block_sparse_attn_fwd(w.q, w.k, w.v, bi, bc, out=o, ws=ws),
                                           reps, stream)
        flops = prefill_flops(bc, d)
        tf = flops / (attn_ms * 1e-3) / 1e12
        density = float(bc.to(torch.float64).sum().item()) / (Hq * (n // 64) * (n // 64 + 1) / 2)
        out[name] = {"index_ms": round(index_ms, 4), "attention_ms": round(attn_ms, 4),
                     "ms_per_layer": round(index_ms + attn_ms, 4), "effective_flops": flops,
                     "effective_tflops_attention": round(tf, 1),
                     "frac_attention": round(tf / peaks["bf16_tflops"], 4),
                     "peak_attention": peaks["bf16_tflops"],
                     "peak_source": f"{src} bf16_tflops (burst: median of {reps} single launches after 1 s idle)",
                     "attention_best_ms": round(attn_best, 4), "clocks": clk,
                     "selected_block_density": round(density, 5), "index_roofline": index_roofline(w, kcap, index_ms,
                                                                                                    peaks),
                     "timed_launches": reps, "status": dsa.get_status(ws)}
        del w, bi, bc, o, ws
        torch.cuda.empty_cache()
    return out


def run_dense(args, ctx, local, attn_flops_ms):
    """Dense causal attention through torch SDPA on the same tensors, for context
    (the pages' "speedup over dense FlashAttention" framing).  Library code, not
    on this package's path; timed like the package's kernels (single launches
    after an idle second) after one warm-up call."""
    import torch.nn.functional as F

    w = ctx[0]
    dev = torch.device("cuda", local)
    Hq, n, d = w.q.shape
    q, k, v = w.q[None], w.k[None], w.v[None]
    stream = torch.cuda.current_stream(dev)
    F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
    torch.cuda.synchronize()
    ms, _, clk = burst_ms(lambda: F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True), 3, stream)
    dense_flops = 4.0 * d * Hq * n * (n + 1) / 2
    return {"impl": "torch SDPA, causal, GQA", "ms": round(ms, 3),
            "tflops": round(dense_flops / (ms * 1e-3) / 1e12, 1),
            "speedup_of_sparse_attention": round(ms / attn_flops_ms, 3), "clocks": clk}


def run_decode(args, local):
    import dynamic_sparse_attention_03_b200 as dsa

    dev = torch.device("cuda", local)
    dw = synth.make_decode("decode-b16-128k", device=dev, B=args.decode_batch)
    p = dw.params
    cent = dsa.pool_keys(dw.k_cache)
    ws = dsa.Workspace(dev)
    o, si, sc = dsa.sparse_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, keep=p["keep"], return_sel=True, ws=ws)
    torch.cuda.synchronize()
    # union of the GQA group's kept blocks: each K/V block read once per (b, KV head)
    B, Hq, dd = dw.q.shape
    Hkv, S = dw.k_cache.shape[1], dw.k_cache.shape[2]
    nb = S // 64
    grp = Hq // Hkv
    mask = torch.zeros((B, Hkv, nb), dtype=torch.bool, device=dev)
    for h in range(Hq):
        idx = si[:, h].long().clamp(min=0)
        valid = torch.arange(si.shape[-1], device=dev)[None, :] < sc[:, h:h + 1]
        m2 = torch.zeros((B, nb), dtype=torch.long, device=dev)
        m2.scatter_add_(1, idx * valid, valid.long())
        m2 = m2 > 0
        mask[:, h // grp] |= m2
    union_blocks = int(mask.sum().item())
    bytes_kv = union_blocks * 2 * 64 * dd * 2
    bytes_cent = B * Hkv * nb * dd * 4
    bytes_io = 2 * B * Hq * dd * 2
    total = bytes_kv + bytes_cent + bytes_io
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        dsa.sparse_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, keep=p["keep"], out=o, ws=ws)
    torch.cuda.synchronize()
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        dsa.sparse_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, keep=p["keep"], out=o, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    # the same step captured once in a CUDA graph and replayed (a serving loop's
    # launch pattern: the five launches of a step without host launch gaps)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
        dsa.sparse_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, keep=p["keep"], out=o, ws=ws)
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_graph = e0.elapsed_time(e1) / reps
    del g
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    dsa.pool_keys(dw.k_cache, out=cent, ws=ws)
    c1.record(stream)
    torch.cuda.synchronize()
    peaks, src = load_peaks()
    gbs = total / (ms * 1e-3) / 1e9
    cent_ms = c0.elapsed_time(c1)
    cent_gbs = (B * Hkv * S * dd * 2 + bytes_cent) / (cent_ms * 1e-3) / 1e9
    del dw
    gbs_graph = total / (ms_graph * 1e-3) / 1e9
    return {"workload": f"decode-b{B}-128k", "ms": round(ms, 4), "GB/s": round(gbs, 1),
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "ms_graph_replay": round(ms_graph, 4),
            "frac_hbm_graph_replay": round(gbs_graph / peaks["hbm_gbs"], 4), "bytes_per_step": total,
            "union_kv_blocks": union_blocks, "centroid_build_ms": round(cent_ms, 4),
            "centroid_build_GB/s": round(cent_gbs, 1), "peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": src}


def run_cluster_decode(args, local):
    """Decode over K-means clusters of the same fixed 128K cache (the Squeezed
    Attention page's offline clustering): 2048 clusters of the first S - 64
    keys (3 Lloyd rounds, timed once as the offline build), then per step every
    q-head keeps its 512 best clusters and attends over them plus the newest
    64 tokens.  GB/s counts the union of a GQA group's kept clusters' K/V rows
    (each row is read once per (batch, KV head)), the centroids and q / o.
    The decode reads the context from a copy in cluster order (made once,
    timed as pack_ms); the token-gather form is timed beside it."""
    import dynamic_sparse_attention_03_b200 as dsa

    dev = torch.device("cuda", local)
    dw = synth.make_decode("decode-b16-128k", device=dev, B=args.decode_batch)
    p = dw.params
    B, Hq, dd = dw.q.shape
    Hkv, S = dw.k_cache.shape[1], dw.k_cache.shape[2]
    C, n_ctx, iters, keep = S // 64, S - 64, 3, p["keep"]
    ws = dsa.Workspace(dev)
    stream = torch.cuda.current_stream(dev)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    cent, _, off, tok = dsa.kmeans_clusters(dw.k_cache, n_ctx, C, iters, ws=ws)
    b1.record(stream)
    torch.cuda.synchronize()
    build_ms = b0.elapsed_time(b1)
    o, si, sc = dsa.cluster_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, off, tok, n_ctx, keep,
                                        return_sel=True, ws=ws)
    torch.cuda.synchronize()
    grp = Hq // Hkv
    size = (off[..., 1:] - off[..., :-1]).long()                      # [B][Hkv][C]
    mask = torch.zeros((B, Hkv, C), dtype=torch.bool, device=dev)
    for h in range(Hq):
        idx = si[:, h].long().clamp(min=0)
        valid = torch.arange(si.shape[-1], device=dev)[None, :] < sc[:, h:h + 1]
        m2 = torch.zeros((B, C), dtype=torch.long, device=dev)
        m2.scatter_add_(1, idx * valid, valid.long())
        mask[:, h // grp] |= m2 > 0
    union_tokens = int((size * mask).sum().item()) + B * Hkv * (S - n_ctx)
    total = union_tokens * 2 * dd * 2 + B * Hkv * C * dd * 4 + 2 * B * Hq * dd * 2
    # the context's K/V copied once in cluster order (also offline): the decode
    # then reads each kept cluster as one contiguous range
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    packed = dsa.cluster_pack_kv(dw.k_cache, dw.v_cache, tok, n_ctx)
    p1.record(stream)
    torch.cuda.synchronize()
    pack_ms = p0.elapsed_time(p1)

    def timed(pk):
        for _ in range(3):
            dsa.cluster_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, off, tok, n_ctx, keep, out=o, ws=ws,
                                    packed=pk)
        torch.cuda.synchronize()
        reps = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            dsa.cluster_decode_attn(dw.q, dw.k_cache, dw.v_cache, cent, off, tok, n_ctx, keep, out=o, ws=ws,
                                    packed=pk)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ms = timed(packed)
    ms_gather = timed(None)
    peaks, src = load_peaks()
    gbs = total / (ms * 1e-3) / 1e9
    del dw, packed
    return {"workload": f"decode-b{B}-128k, {C} K-means clusters of the first S-64 keys, keep {keep} + tail",
            "ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "bytes_per_step": total, "union_tokens": union_tokens, "kv_layout": "cluster-ordered copy",
            "ms_token_gather": round(ms_gather, 4), "kmeans_build_ms": round(build_ms, 2),
            "kmeans_rounds": iters, "pack_ms": round(pack_ms, 3), "peak_hbm_gbs": peaks["hbm_gbs"],
            "peak_source": src}


def run_vs(args, local):
    """Vertical-slash prefill layer at 128K: vertical_slash_index followed by
    block_sparse_attn_fwd over the plan's blocks and column tiles.  Effective
    FLOPs count the selected blocks (the diagonal block at its causal elements)
    plus 4*d FLOP per (row, kept column) pair of every column tile entry."""
    import dynamic_sparse_attention_03_b200 as dsa

    dev = torch.device("cuda", local)
    name = "llama3-8b-128k-vs"
    p = synth.CONFIGS[name]
    w = synth.make_prefill(name, device=dev)
    Hq, n, d = w.q.shape
    ws = dsa.Workspace(dev)
    res = dsa.vertical_slash_index(w.q, w.k, p["n_vert"], p["n_slash"], ws=ws)
    o = dsa.block_sparse_attn_fwd(w.q, w.k, w.v, res["block_idx"], res["block_cnt"], res["col_idx"],
                                  res["col_cnt"], ws=ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    reps = 3
    idx_ms, _, _ = burst_ms(lambda: dsa.vertical_slash_index(w.q, w.k, p["n_vert"], p["n_slash"], ws=ws, out=res),
                            reps, stream)
    att_ms, att_best, clk = burst_ms(lambda: dsa.block_sparse_attn_fwd(w.q, w.k, w.v, res["block_idx"],
                                                                       res["block_cnt"], res["col_idx"],
                                                                       res["col_cnt"], out=o, ws=ws), reps, stream)
    flops = prefill_flops(res["block_cnt"], d) + float(res["col_cnt"].to(torch.float64).sum().item()) * 4 * d * 64
    nqb = n // 64
    density = float(res["block_cnt"].to(torch.float64).sum().item()) / (Hq * nqb * (nqb + 1) / 2)
    peaks, src = load_peaks()
    tf = flops / (att_ms * 1e-3) / 1e12
    # the index: K read once (bf16) and the last 64 query rows, the kept sets
    # and the plan's lists written once; 2 x 2*64*n*d FLOP of logits per q-head
    # (the scores' pass and the sums' pass) on the tensor pipe
    Hkv = w.k.shape[0]
    kcap, ccap = res["block_idx"].shape[-1], res["col_idx"].shape[-1]
    idx_bytes = (Hkv * n * d + Hq * 64 * d) * 2 + Hq * (p["n_vert"] + p["n_slash"]) * 4 + \
        Hq * nqb * (kcap + ccap + 2) * 4
    idx_flops = 2 * 2.0 * 64 * n * d * Hq
    gbs = idx_bytes / (idx_ms * 1e-3) / 1e9
    tfs = idx_flops / (idx_ms * 1e-3) / 1e12
    out = {"workload": name, "index_ms": round(idx_ms, 3), "attention_ms": round(att_ms, 3),
           "ms_per_layer": round(idx_ms + att_ms, 3), "effective_tflops_attention": round(tf, 1),
           "frac_attention": round(tf / peaks["bf16_tflops"], 4), "attention_best_ms": round(att_best, 3),
           "peak_source": f"{src} bf16_tflops (burst: median of {reps} single launches after 1 s idle)",
           "clocks": clk,
           "index_roofline": {"bound": "hbm", "bytes": idx_bytes, "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                              "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                              "tensor_flops": idx_flops, "achieved_tflops": round(tfs, 1),
                              "tensor_frac": round(tfs / peaks["bf16_tflops"], 4)},
           "selected_block_density": round(density, 4), "status": dsa.get_status(ws)}
    del w, res, o
    torch.cuda.empty_cache()
    return out


def run_e2e(args, ctx, local):
    """Same metric through the public API with host buffers: every step copies
    its Q/K/V in from pinned host memory, runs index + attention and copies O
    out.  Steps are pipelined over two device buffer sets on three streams
    (host-to-device, compute, device-to-host), so step i's copies overlap the
    compute of its neighbours; the two copy directions use separate engines."""
    import dynamic_sparse_attention_03_b200 as dsa

    w, bi, bc, kf, rho, kcap, flops, ws = ctx
    dev = torch.device("cuda", local)
    hq, hk, hv = (t.to("cpu").pin_memory() for t in (w.q, w.k, w.v))
    ho = torch.empty_like(hq).pin_memory()
    sets = [(torch.empty_like(w.q), torch.empty_like(w.k), torch.empty_like(w.v), torch.empty_like(w.q))
            for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(i):
        k = i & 1
        dq, dk, dv, do = sets[k]
        with torch.cuda.stream(s_in):
            if used[k]:
                s_in.wait_event(comp_done[k])        # the set's inputs were read by step i-2
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            in_done[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[k])
            if used[k]:
                s_comp.wait_event(out_done[k])       # step i-2's O has left the device
            dsa.sparse_index_estimate(dq, dk, k_fixed=kf, keep_ratio=rho, kcap=kcap, block_idx=bi, block_cnt=bc,
                                      ws=ws)
            dsa.block_sparse_attn_fwd(dq, dk, dv, bi, bc, out=do, ws=ws)
            comp_done[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            ho.copy_(do, non_blocking=True)
            out_done[k].record(s_out)
        used[k] = True

    steps = max(2, min(args.steps, 6))
    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_in.wait_event(out_done[1])                    # the warm-up is over before the clock starts
    for i in range(2, 2 + steps):
        step(i)
    with torch.cuda.stream(s_out):
        e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size()
    del sets
    return {"value": round(flops / (ms * 1e-3) / 1e12, 3), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelining": "2 buffer sets; H2D, compute and D2H streams"}


# ------------------------------------------------------------------ CPU oracle (reference arm and cpu_baseline)

def oracle_sample(workload: str, budget_s: float, w=None, seed_rank: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload: the full block
    index of one q-head plus the attention of sampled query blocks of that head.
    Returns (effective TFLOP/s of the sample, description, seconds, cores)."""
    import oracle

    p = synth.CONFIGS[workload]
    if w is None:
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        w = synth.make_prefill(workload, device=dev, seed=p["seed"] + 1000 * seed_rank)
    Hq, n, d = w.q.shape
    grp = Hq // w.k.shape[0]
    h = 0
    q = synth.to_f64(w.q[h:h + 1])
    k = synth.to_f64(w.k[h // grp:h // grp + 1])
    v = synth.to_f64(w.v[h // grp:h // grp + 1])
    kf, rho = p.get("k_fixed", 0), p.get("keep_ratio", 0.0)
    nqb = n // 64
    t0 = time.perf_counter()
    lists, _, _ = oracle.block_index(q, k, k_fixed=kf, keep_ratio=rho)
    t_index = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    order = [nqb - 1, 0] + rng.permutation(nqb).tolist()
    flops = 0.0
    t_att = 0.0
    items = 0
    for qb in order:
        if t_index + t_att > budget_s and items >= 2:
            break
        t1 = time.perf_counter()
        oracle.sparse_attention(q, k, v, lists, None, 1 / math.sqrt(d), items=[(0, qb)])
        t_att += time.perf_counter() - t1
        cnt = len(lists[0][qb])
        flops += (cnt - 1) * 4 * 64 * 64 * d + 4 * DIAG_ELEMS * d
        items += 1
    # index cost of one head prorated to the sampled query blocks
    t_total = t_att + t_index * items / nqb
    cores = len(os.sched_getaffinity(0))
    desc = (f"oracle fp64 on host: block index of q-head 0 ({nqb} query blocks, {t_index:.2f}s, prorated) + "
            f"attention of {items} sampled query blocks of q-head 0")
    return flops / t_total / 1e12, desc, t_total, cores


def blas_threads():
    """Threads of the BLAS library NumPy's matrix products use (None if unknown)."""
    try:
        import threadpoolctl

        info = [x for x in threadpoolctl.threadpool_info() if x.get("user_api") == "blas"]
        return info[0]["num_threads"] if info else None
    except Exception:
        return None


def run_reference(args, rank, world):
    if rank != 0:
        return None
    vals = []
    desc = ""
    cores = len(os.sched_getaffinity(0))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    p = synth.CONFIGS[args.workload]
    w = synth.make_prefill(args.workload, device=dev, seed=p["seed"])
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        v, desc, secs, cores = oracle_sample(args.workload, budget, w=w)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.mean(vals)
    return {"metric": metric_name(args.workload), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(args.workload, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "blas_threads": blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama3-8b-128k-bs10")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-clusters", action="store_true")
    ap.add_argument("--no-vs", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-layers", action="store_true", help="skip the 32K and 1M layers")
    ap.add_argument("--hq", type=int, default=None,
                    help="query heads (default: the workload's; fewer for a reduced case to profile)")
    ap.add_argument("--hkv", type=int, default=None, help="KV heads (default: the workload's)")
    ap.add_argument("--sustained-s", type=float, default=3.0,
                    help="seconds of back-to-back attention launches for the sustained-peak line (0: skip)")
    ap.add_argument("--decode-batch", type=int, default=16,
                    help="batch of the decode workloads (16 is the reported configuration; smaller for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        world = int(os.environ.get("WORLD_SIZE", args.gpus))
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    res, ctx = run_ours(args, rank, world, local)
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, ctx, local)
    if not args.no_dense:
        res["dense_comparator"] = run_dense(args, ctx, local, res["breakdown_ms"]["attention"])
    if not args.no_layers:
        others = [x for x in ("llama3-8b-32k-bs10", "llama3-8b-1m-bs2") if x != args.workload]
        res["layers"] = run_layers(args, local, others)
    if not args.no_decode:
        res["decode"] = run_decode(args, local)
    if not args.no_clusters:
        res["cluster_decode"] = run_cluster_decode(args, local)
    if not args.no_vs:
        res["vertical_slash"] = run_vs(args, local)
        if "dense_comparator" in res:
            res["vertical_slash"]["speedup_over_dense_attention"] = round(
                res["dense_comparator"]["ms"] / res["vertical_slash"]["attention_ms"], 3)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, secs, cores = oracle_sample(args.workload, 15.0, w=ctx[0])
        res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "blas_threads": blas_threads(),
                               "kind": "oracle", "sample": desc, "seconds": round(secs, 2)}
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
