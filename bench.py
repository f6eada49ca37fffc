#!/usr/bin/env python
"""Benchmark of the DSA forward hot path on B200.

Default workload: DSA prefill, batch 2 x 32768 tokens, causal, H_I=64 / d_I=128
FP8 indexer, top-2048, 128-head MQA over 576-wide bf16 latent rows; plus the
decode workload (64 sequences x 1 token against a 131072-token cache) in the
same run. One step = one ``dsa_forward`` over the whole batch (indexer, top-k,
sparse MLA). Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs the same
per-GPU workload on its own GPU (weak scaling, no data-path collective); the
reported time is the max over ranks. ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from dsa_inputs import CONFIG_ORDER, CONFIGS, gen_inputs  # noqa: E402

METRIC = "DSA prefill tokens/s at 32K ctx; decode tokens/s at 128K ctx (k=2048), %roofline"
CSRC = os.path.join(ROOT, "sparse_attention_long_scores_b200", "csrc")

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum from one ncu
# capture of the small profile case, see --profile-case), with the query rows that
# launch processed and the SHA-256 of the kernel's source file when it was taken. A
# full launch's traffic is scaled from it by the rows it processes (the per-row Q read
# and output write dominate; the once-per-sequence latent rows are under 1 %). When
# the source has changed since the capture the figure no longer describes the kernel,
# and the traffic is reported as null.
TRAFFIC = {
    # --profile-case prefill_chunk: 329.3 MB read + 235.0 MB written, 2048 rows
    ("sparse_mla", "prefill"): {"source": "sparse_mla.cu", "rows": 2048, "bytes": 564293888,
                                "sha256": "a7dee1cf4177f8d389ff2b42f4a20e640f5c073749741b8ea1aa4d00aa048ac4"},
    # --profile-case decode_small: 40.3 MB read + 0.4 MB written, 16 rows
    ("sparse_mla", "decode"): {"source": "sparse_mla.cu", "rows": 16, "bytes": 40730880,
                               "sha256": "a7dee1cf4177f8d389ff2b42f4a20e640f5c073749741b8ea1aa4d00aa048ac4"},
}
DTYPE = "fp8_e4m3+bf16"


# ---------------------------------------------------------------------------
# algorithmic work (what the method must do, not what a kernel happens to do)
# ---------------------------------------------------------------------------


def work(cfg) -> dict:
    """Per-step algorithmic work of each stage.

    indexer  flops = 2 * H_I * d_I per (query row, causal key) of rows that need
             scoring (p + 1 > k); rows with p + 1 <= k select every key unscored.
             bytes = key codes + scales once per sequence, query codes, scales and
             weights, and 4 per score written (the decode roofline: one query row
             per sequence makes it bandwidth-bound).
    topk     bytes = 4 per candidate score read + 4 * k per selected row written.
    fused    indexer + top-k in one kernel: the indexer's flops (prefill); bytes =
             key codes and scales once, queries and weights, 4 * k per row written.
    mla      flops = 2 * H * (Dqk + Dv) per (query row, selected key).
             bytes = 2 * Dqk per selected key + q, idx and out per row (decode).
    decode   bytes = indexer keys + scales + gathered latent rows + q, qI, w, out.
    """
    w_bytes = 4 if cfg.w_dtype == "f32" else 2
    p = cfg.q_pos0 + np.arange(cfg.Lq, dtype=np.int64)
    n = np.minimum(p + 1, cfg.Lk)
    scored = n > cfg.k
    pairs_idx = int(n[scored].sum()) * cfg.B
    sel = int(np.minimum(n, cfg.k).sum()) * cfg.B
    rows_scored = int(scored.sum()) * cfg.B
    tokens = cfg.B * cfg.Lq
    return {
        "indexer_flops": 2.0 * cfg.H_I * cfg.d_I * pairs_idx,
        # indexer bytes: the key codes and scales of every causal key of each
        # sequence, read once, plus the query rows, weights and scores written
        "indexer_bytes": float(cfg.B * min(cfg.Lk, cfg.q_pos0 + cfg.Lq) * (cfg.d_I + 4)
                               + tokens * cfg.H_I * (cfg.d_I + 4 + w_bytes) + 4.0 * pairs_idx),
        "topk_bytes": 4.0 * pairs_idx + 4.0 * cfg.k * rows_scored,
        # fused indexer + top-k: its inputs once and the selected keys out (the scores
        # stay in the L2-resident chunk between scoring and selection)
        "fused_bytes": float(cfg.B * min(cfg.Lk, cfg.q_pos0 + cfg.Lq) * (cfg.d_I + 4)
                             + tokens * cfg.H_I * (cfg.d_I + 4 + w_bytes) + 4.0 * cfg.k * tokens),
        "mla_flops": 2.0 * cfg.H * (cfg.Dqk + cfg.Dv) * sel,
        # attention bytes: each selected latent row once, q and idx in, out written
        "mla_bytes": float(sel * cfg.Dqk * 2 + tokens * (cfg.H * cfg.Dqk * 2 + 4 * cfg.k
                                                         + cfg.H * cfg.Dv * 2)),
        "hbm_bytes": float(cfg.B * cfg.Lk * (cfg.d_I + 4)            # indexer keys + scales
                           + sel * cfg.Dqk * 2                      # gathered latent rows
                           + cfg.B * cfg.Lq * (cfg.H * cfg.Dqk * 2 + cfg.H_I * (cfg.d_I + 4 + w_bytes)
                                               + cfg.H * cfg.Dv * 2)),
    }


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        m = json.load(open(path))
        return {"hbm": float(m["hbm_gbs"]), "bf16": float(m["bf16_tflops"]),
                "bf16_sustained": float(m["bf16_tflops_sustained"]), "source": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------


def dist_max(x: float, world: int) -> float:
    """Max of a per-rank value over all ranks (the step time of a weak-scaling run)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(name: str, rank: int) -> int:
    """Seed of this rank's share of the workload: every rank gets its own sequences."""
    return 1000 + CONFIG_ORDER.index(name) + 97 * rank


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def traffic_per_launch(kernel: str, mode: str, rows_per_launch: float):
    ent = TRAFFIC.get((kernel, mode))
    if not ent:
        return None
    with open(os.path.join(CSRC, ent["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != ent["sha256"]:
            return None
    return ent["bytes"] * rows_per_launch / ent["rows"]


def time_workload(name: str, steps: int, warmup: int, world: int, rank: int, pk: dict,
                  sampler: ClockSampler | None, e2e: bool):
    import sparse_attention_long_scores_b200 as dsa

    cfg = CONFIGS[name]
    inp = gen_inputs(cfg, "cuda", seed=rank_seed(name, rank))
    p = dsa.Problem.from_config(cfg)
    ws = torch.empty(dsa.forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    out = torch.empty((cfg.B, cfg.Lq, cfg.H, cfg.Dv), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        dsa.forward(p, inp, out=out, ws=ws)
    torch.cuda.synchronize()
    dsa.check_status()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    timed_launches = 0
    for i in range(steps):
        dsa.forward(p, inp, out=out, ws=ws)
        timed_launches += dsa.last_launch_count()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    dsa.check_status()
    ms_local = e0.elapsed_time(e1) / steps
    ms = dist_max(ms_local, world)
    # the fused indexer + top-k schedule (dsa_forward_fused), for comparison
    ef0 = torch.cuda.Event(enable_timing=True)
    ef1 = torch.cuda.Event(enable_timing=True)
    dsa.forward(p, inp, out=out, ws=ws, fused=True)
    ef0.record(stream)
    for i in range(steps):
        dsa.forward(p, inp, out=out, ws=ws, fused=True)
    ef1.record(stream)
    torch.cuda.synchronize()
    dsa.check_status()
    fused_ms = dist_max(ef0.elapsed_time(ef1) / steps, world)
    # per-kernel device time: the same steps again through dsa_forward_profiled,
    # which keeps every launch on the caller's stream (no top-k / indexer overlap)
    # so that the events around a launch time that launch alone
    profs = [dsa.LaunchProfiler(4096) for _ in range(steps)]
    for i in range(steps):
        dsa.forward_profiled(p, inp, out, profs[i], ws=ws)
    torch.cuda.synchronize()
    dsa.check_status()
    per_kind, launches = {}, 0
    for pr in profs:
        for kind, d in pr.durations():
            c = per_kind.setdefault(kind, [0.0, 0])
            c[0] += d
            c[1] += 1
        launches += pr.n
    kernels = {k: {"ms_per_step": v[0] / steps, "launches_per_step": v[1] / steps,
                   "avg_launch_ms": v[0] / v[1]} for k, v in per_kind.items()}
    w = work(cfg)
    fp8_peak = 2.0 * pk["bf16_sustained"]   # FP8 dense = 2 x bf16 dense (nominal ratio)
    roof = {}
    decode = cfg.mode == "decode"
    if "indexer_topk" in kernels:
        # fused indexer + top-k: the indexer's FP8 work (prefill), or its algorithmic
        # bytes (decode: key codes and scales once, queries, selected keys written)
        t = kernels["indexer_topk"]["ms_per_step"] * 1e-3
        if decode:
            a = w["fused_bytes"] / t / 1e9
            roof["indexer_topk"] = {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s",
                                    "frac": a / pk["hbm"]}
        else:
            a = w["indexer_flops"] / t / 1e12
            roof["indexer_topk"] = {"bound": "tensor", "achieved": a, "peak": fp8_peak,
                                    "unit": "TFLOP/s", "frac": a / fp8_peak,
                                    "peak_note": "fp8 = 2 x measured bf16 sustained"}
    if "indexer" in kernels:
        t = kernels["indexer"]["ms_per_step"] * 1e-3
        if decode:   # one query row per sequence: every key is read for 16 KFLOP
            a = w["indexer_bytes"] / t / 1e9
            roof["indexer"] = {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s",
                               "frac": a / pk["hbm"]}
        else:
            a = w["indexer_flops"] / t / 1e12
            roof["indexer"] = {"bound": "tensor", "achieved": a, "peak": fp8_peak, "unit": "TFLOP/s",
                               "frac": a / fp8_peak, "peak_note": "fp8 = 2 x measured bf16 sustained"}
    if "topk" in kernels:
        t = kernels["topk"]["ms_per_step"] * 1e-3
        a = w["topk_bytes"] / t / 1e9
        roof["topk"] = {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s",
                        "frac": a / pk["hbm"]}
    if "sparse_mla" in kernels:
        t = kernels["sparse_mla"]["ms_per_step"] * 1e-3
        if decode:   # 64 query rows: each gathered latent row serves one token
            a = w["mla_bytes"] / t / 1e9
            roof["sparse_mla"] = {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s",
                                  "frac": a / pk["hbm"]}
        else:
            a = w["mla_flops"] / t / 1e12
            roof["sparse_mla"] = {"bound": "tensor", "achieved": a, "peak": pk["bf16_sustained"],
                                  "unit": "TFLOP/s", "frac": a / pk["bf16_sustained"],
                                  "peak_note": "measured bf16 sustained"}
    for k, r in roof.items():
        r["traffic"] = traffic_per_launch(k, cfg.mode, cfg.B * cfg.Lq / kernels[k]["launches_per_step"])
    res = {"cfg": cfg, "ms": ms, "tokens_per_s": aggregate_tokens_per_s(cfg.B * cfg.Lq, world, ms),
           "fused": {"entry": "dsa_forward_fused", "ms_per_step": fused_ms,
                     "value": aggregate_tokens_per_s(cfg.B * cfg.Lq, world, fused_ms)},
           "kernels": kernels,
           "roof": roof, "launches": timed_launches, "clocks": clocks, "work": w}
    if cfg.mode == "decode":
        a = w["hbm_bytes"] / (ms * 1e-3) / 1e9
        res["step_roof"] = {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s",
                            "frac": a / pk["hbm"], "traffic": None}
    if e2e:
        res["e2e"] = time_e2e(cfg, p, inp, ws, world)
    del inp, out, ws
    torch.cuda.empty_cache()
    return res


def time_e2e(cfg, p, inp, ws, world, steps: int = 2):
    """Same metric through dsa_forward_host: pinned host inputs -> device -> host out."""
    import sparse_attention_long_scores_b200 as dsa

    host = {k: v.cpu().pin_memory() for k, v in inp.items()}
    host_out = torch.empty((cfg.B, cfg.Lq, cfg.H, cfg.Dv), dtype=torch.bfloat16).pin_memory()
    dev_out = torch.empty((cfg.B, cfg.Lq, cfg.H, cfg.Dv), dtype=torch.bfloat16, device="cuda")
    dsa.forward_host(p, host, inp, host_out, dev_out, ws)     # warm-up
    barrier(world)
    t0 = time.perf_counter()
    for _ in range(steps):
        dsa.forward_host(p, host, inp, host_out, dev_out, ws)
    dt = (time.perf_counter() - t0) / steps
    dt = dist_max(dt, world)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host_out.numel() * host_out.element_size()
    del host, host_out, dev_out
    return {"value": cfg.B * cfg.Lq * world / dt, "unit": "tokens/s", "ms_per_step": dt * 1e3,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


# ---------------------------------------------------------------------------
# oracle (CPU) arm
# ---------------------------------------------------------------------------


def time_indexer_kl(name: str, steps: int, warmup: int, world: int, rank: int, pk: dict):
    """The indexer alignment target (dsa_indexer_kl, forward) on the workload's own
    selected sets: one forward gives idx and the per-head lse, the index scores of the
    selected keys are seeded random stand-ins (the kernel's cost does not depend on
    their values). Timed with CUDA events on the launching stream, p written."""
    import sparse_attention_long_scores_b200 as dsa
    from dsa_inputs import random_scores

    cfg = CONFIGS[name]
    inp = gen_inputs(cfg, "cuda", seed=rank_seed(name, rank))
    p = dsa.Problem.from_config(cfg)
    lse = torch.empty((cfg.B, cfg.Lq, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.int32, device="cuda")
    dsa.forward(p, inp, lse=lse, idx_out=idx)
    q, kv = inp["q"], inp["kv"]
    del inp
    sel = random_scores((cfg.B, cfg.Lq, cfg.k), seed=77 + rank).cuda()
    kl = torch.empty((cfg.B, cfg.Lq), dtype=torch.float32, device="cuda")
    pt = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        dsa.indexer_kl(q, kv, idx, lse, sel, cfg.sm_scale, p_out=pt, kl_out=kl)
    torch.cuda.synchronize()
    dsa.check_status()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        dsa.indexer_kl(q, kv, idx, lse, sel, cfg.sm_scale, p_out=pt, kl_out=kl)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    dsa.check_status()
    ms = dist_max(e0.elapsed_time(e1) / steps, world)
    pairs = work(cfg)["mla_flops"] / (2.0 * cfg.H * (cfg.Dqk + cfg.Dv))
    flops = 2.0 * cfg.H * cfg.Dqk * pairs
    a = flops / (ms * 1e-3) / 1e12
    res = {"workload": cfg.name, "value": aggregate_tokens_per_s(cfg.B * cfg.Lq, world, ms),
           "unit": "tokens/s", "ms_per_step": ms, "launches_per_step": 1,
           "roofline": {"bound": "tensor", "achieved": a, "peak": pk["bf16_sustained"],
                        "unit": "TFLOP/s", "frac": a / pk["bf16_sustained"], "traffic": None,
                        "peak_note": "measured bf16 sustained; work = 2 H Dqk per selected pair"},
           "note": "KL(p || softmax(index scores)) over the forward's top-k sets, p written"}
    del q, kv, idx, lse, sel, kl, pt
    torch.cuda.empty_cache()
    return res


def time_backward(name: str, steps: int, warmup: int, world: int, rank: int, pk: dict):
    """The sparse-stage gradients on the workload's own selected sets, each timed with
    CUDA events on the launching stream: the attention backward (dsa_sparse_mla_bwd,
    dq and dkv from a seeded output gradient) and the indexer backward
    (dsa_indexer_kl_grad on the KL target's p, then dsa_indexer_bwd)."""
    import sparse_attention_long_scores_b200 as dsa
    from dsa_inputs import output_gradient, random_scores

    cfg = CONFIGS[name]
    dev = "cuda"
    inp = gen_inputs(cfg, dev, seed=rank_seed(name, rank))
    p = dsa.Problem.from_config(cfg)
    B, Lq, Lk = cfg.B, cfg.Lq, cfg.Lk
    out = torch.empty((B, Lq, cfg.H, cfg.Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Lq, cfg.H), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Lq, cfg.k), dtype=torch.int32, device=dev)
    dsa.forward(p, inp, out=out, lse=lse, idx_out=idx)
    dout = output_gradient((B, Lq, cfg.H, cfg.Dv), seed=5 + rank, device=dev)
    sel = random_scores((B, Lq, cfg.k), seed=77 + rank).to(dev)
    _, pt = dsa.indexer_kl(inp["q"], inp["kv"], idx, lse, sel, cfg.sm_scale)
    dq = torch.empty((B, Lq, cfg.H, cfg.Dqk), dtype=torch.float32, device=dev)
    dkv = torch.empty((B, Lk, cfg.Dqk), dtype=torch.float32, device=dev)
    ws = torch.empty(dsa.lib().dsa_sparse_mla_bwd_workspace_size(B, Lq, cfg.H, cfg.Dqk, cfg.Dv,
                                                                 cfg.k), dtype=torch.uint8, device=dev)
    dI = torch.empty_like(sel)
    dqI = torch.empty((B, Lq, cfg.H_I, cfg.d_I), dtype=torch.float32, device=dev)
    dkI = torch.empty((B, Lk, cfg.d_I), dtype=torch.float32, device=dev)
    dw = torch.empty((B, Lq, cfg.H_I), dtype=torch.float32, device=dev)
    wsi = torch.empty(dsa.lib().dsa_indexer_bwd_workspace_size(B, Lq, cfg.H_I, cfg.d_I, cfg.k),
                      dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    launches = {}

    def attention():
        dsa.sparse_mla_bwd(inp["q"], inp["kv"], idx, lse, dout, cfg.sm_scale, dq=dq, dkv=dkv,
                           ws=ws)
        launches["attention"] = dsa.last_launch_count()

    def indexer():
        dsa.indexer_kl_grad(sel, pt, idx, Lk, dI=dI)
        n = dsa.last_launch_count()
        dsa.indexer_bwd(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"], idx, dI,
                        dqI=dqI, dkI=dkI, dw=dw, ws=wsi)
        launches["indexer"] = n + dsa.last_launch_count()

    n_steps = max(1, min(steps, 5))

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        dsa.check_status()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        dsa.check_status()
        return dist_max(e0.elapsed_time(e1) / n_steps, world)

    ms_att = timed(attention)
    ms_idx = timed(indexer)
    pairs = work(cfg)["mla_flops"] / (2.0 * cfg.H * (cfg.Dqk + cfg.Dv))
    att_tf = pairs * 2.0 * cfg.H * (3 * cfg.Dqk + 2 * cfg.Dv) / (ms_att * 1e-3) / 1e12
    idx_tf = pairs * 6.0 * cfg.H_I * cfg.d_I / (ms_idx * 1e-3) / 1e12
    res = {"workload": cfg.name,
           "value": aggregate_tokens_per_s(B * Lq, world, ms_att + ms_idx), "unit": "tokens/s",
           "ms_per_step": ms_att + ms_idx, "steps": n_steps,
           "attention": {"ms_per_step": ms_att, "launches_per_step": launches.get("attention"),
                         "roofline": {"bound": "tensor", "achieved": att_tf,
                                      "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                                      "frac": att_tf / pk["bf16_sustained"], "traffic": None,
                                      "peak_note": "measured bf16 sustained; work = "
                                                   "2 H (3 Dqk + 2 Dv) per selected pair"}},
           "indexer": {"ms_per_step": ms_idx, "launches_per_step": launches.get("indexer"),
                       "roofline": {"bound": "tensor", "achieved": idx_tf,
                                    "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                                    "frac": idx_tf / pk["bf16_sustained"], "traffic": None,
                                    "peak_note": "measured bf16 sustained; work = 6 H_I d_I per "
                                                 "selected pair (the three-term bf16 split of the "
                                                 "gradient factors executes 14 H_I d_I)"}},
           "note": "gradients of the sparse training stage: this library's batched tcgen05 bf16 "
                   "GEMMs (fp32 accumulation) over gathered rows, with its gather, "
                   "softmax/ReLU-gradient and scatter-add kernels; the indexer's ReLU mask is "
                   "re-decided exactly in fp64 near zero"}
    del inp, out, lse, idx, dout, sel, pt, dq, dkv, ws, dI, dqI, dkI, dw, wsi
    torch.cuda.empty_cache()
    return res


def oracle_sample(cfg, rows: int, seed: int = 4242):
    """A bounded sample of the workload for the fp64 oracle: one sequence with all
    Lk keys and `rows` query rows at evenly spread positions (decode: the last)."""
    import oracle as ORC

    c1 = cfg.with_(B=1, Lq=rows, q_pos0=0)
    inp = ORC.numpy_inputs(gen_inputs(c1, "cpu", seed=seed))
    if cfg.mode == "decode":
        pos = [cfg.Lk - 1] * rows
    else:
        pos = [min(cfg.Lk - 1, int((i + 0.5) * cfg.Lk / rows)) for i in range(rows)]

    def run(i):
        p = pos[i]
        n = p + 1
        if n > cfg.k:
            sc = ORC.index_scores(inp["qI"][0, i], inp["qI_scale"][0, i], inp["w"][0, i],
                                  inp["kI"][0, :n], inp["kI_scale"][0, :n])
            idx = ORC.topk_select(sc, cfg.k)
        else:
            idx = ORC.topk_select(np.zeros(n), cfg.k)
        ORC.sparse_mla(inp["q"][0, i], inp["kv"][0], idx, cfg.sm_scale, cfg.Dv)

    return run, pos


def cpu_baseline(cfg, budget_s: float = 20.0) -> dict:
    run, pos = oracle_sample(cfg, 1024)
    t0 = time.perf_counter()
    done = 0
    for i in range(len(pos)):
        run(i)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": done / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} query rows of {cfg.name} (one sequence, rows at evenly spread "
                      f"positions, {dt:.1f} s), numpy fp64 with BLAS on {cores} host threads"}


def oracle_backward_sample(cfg, rows: int, seed: int = 4243):
    """A bounded sample of the sparse-stage gradients for the fp64 oracle: `rows`
    query rows at evenly spread positions of one sequence, each with a seeded set of
    min(k, p + 1) causal keys standing in for its top-k set, a seeded output gradient
    and a seeded index-score gradient. One unit is the attention and indexer
    gradients of one row."""
    import oracle as ORC
    from dsa_inputs import output_gradient, random_key_sets, random_scores

    c1 = cfg.with_(B=1, Lq=rows, q_pos0=0)
    inp = ORC.numpy_inputs(gen_inputs(c1, "cpu", seed=seed))
    pos = [min(cfg.Lk - 1, int((i + 0.5) * cfg.Lk / rows)) for i in range(rows)]
    sets = [random_key_sets(1, 1, cfg.k, p, seed=seed + 3 + i)[0, 0].numpy()
            for i, p in enumerate(pos)]
    dout = ORC.numpy_inputs({"d": output_gradient((1, rows, cfg.H, cfg.Dv), seed=seed + 1)})["d"]
    dI = random_scores((1, rows, cfg.k), seed=seed + 2).numpy()

    def run(i):
        ORC.sparse_mla_backward(inp["q"][0, i], inp["kv"][0], sets[i], dout[0, i], cfg.sm_scale,
                                cfg.Dv)
        ORC.indexer_backward(inp["qI"][0, i], inp["qI_scale"][0, i], inp["w"][0, i], inp["kI"][0],
                             inp["kI_scale"][0], sets[i], dI[0, i])

    return run, pos


def cpu_baseline_backward(cfg, budget_s: float = 10.0, rows: int = 64) -> dict:
    run, pos = oracle_backward_sample(cfg, rows)
    t0 = time.perf_counter()
    done = 0
    for i in range(len(pos)):
        run(i)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": done / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"attention and indexer gradients of {done} query rows of {cfg.name} "
                      f"(one sequence, rows at evenly spread positions, seeded key sets of "
                      f"min(k, p + 1) keys, {dt:.1f} s), numpy fp64 with BLAS on {cores} host "
                      f"threads"}


def reference_arm(args):
    cfg = CONFIGS[args.workload]
    rows_per_step = 8
    run, pos = oracle_sample(cfg, rows_per_step * (args.steps + args.warmup))
    i = 0
    for _ in range(args.warmup):
        for _ in range(rows_per_step):
            run(i)
            i += 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(rows_per_step):
            run(i)
            i += 1
    dt = (time.perf_counter() - t0) / args.steps
    v = rows_per_step / dt
    cores = len(os.sched_getaffinity(0))
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": cfg.name, "global_batch": cfg.B, "seq_len": cfg.Lk,
                       "step": f"{rows_per_step} query rows of the workload per step"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows_per_step} query rows per step at evenly spread "
                                       f"positions of {cfg.name}, numpy fp64"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------


PROFILE_CASES = {
    # one 2048-row prefill chunk of the 8K workload (rows 6144..8191, all keys causal)
    "prefill_chunk": ("prefill_8k", dict(Lq=2048, q_pos0=6144)),
    # the same chunk through dsa_forward_fused (top-k inside the indexer kernel)
    "prefill_chunk_fused": ("prefill_8k", dict(Lq=2048, q_pos0=6144)),
    # 16 decode sequences against 131072 cached keys
    "decode_small": ("decode_128k", dict(B=16)),
    # the indexer KL target over the forward's top-k sets of the prefill chunk above
    "kl_chunk": ("prefill_8k", dict(Lq=2048, q_pos0=6144)),
    # the sparse-stage gradients of the last 256 rows of the 8K workload (4 chunks of
    # 64 tokens): attention backward, KL score gradient, indexer backward
    "bwd_chunk": ("prefill_8k", dict(Lq=256, q_pos0=7936)),
}


def profile_case(name: str) -> None:
    """Two untimed passes of a small case, for an ncu capture of its kernels (the
    second pass's launches are the ones to capture)."""
    import sparse_attention_long_scores_b200 as dsa
    from sparse_attention_long_scores_b200.build import build

    build()
    torch.cuda.set_device(0)
    base, kw = PROFILE_CASES[name]
    cfg = CONFIGS[base].with_(**kw)
    inp = gen_inputs(cfg, "cuda")
    p = dsa.Problem.from_config(cfg)
    if name == "kl_chunk":
        from dsa_inputs import random_scores
        lse = torch.empty((cfg.B, cfg.Lq, cfg.H), dtype=torch.float32, device="cuda")
        idx = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.int32, device="cuda")
        dsa.forward(p, inp, lse=lse, idx_out=idx)
        sel = random_scores((cfg.B, cfg.Lq, cfg.k), seed=77).cuda()
        for _ in range(2):
            dsa.indexer_kl(inp["q"], inp["kv"], idx, lse, sel, cfg.sm_scale)
    elif name == "bwd_chunk":
        from dsa_inputs import output_gradient, random_scores
        lse = torch.empty((cfg.B, cfg.Lq, cfg.H), dtype=torch.float32, device="cuda")
        idx = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.int32, device="cuda")
        dsa.forward(p, inp, lse=lse, idx_out=idx)
        dout = output_gradient((cfg.B, cfg.Lq, cfg.H, cfg.Dv), seed=5, device="cuda")
        sel = random_scores((cfg.B, cfg.Lq, cfg.k), seed=77).cuda()
        _, pt = dsa.indexer_kl(inp["q"], inp["kv"], idx, lse, sel, cfg.sm_scale)
        for _ in range(2):
            dsa.sparse_mla_bwd(inp["q"], inp["kv"], idx, lse, dout, cfg.sm_scale)
            dI = dsa.indexer_kl_grad(sel, pt, idx, cfg.Lk)
            dsa.indexer_bwd(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"], idx,
                            dI)
    else:
        for _ in range(2):
            dsa.forward(p, inp, fused=name.endswith("_fused"))
    torch.cuda.synchronize()
    dsa.check_status()
    print(f"profile case {name}: {cfg}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_32k", choices=sorted(CONFIGS))
    ap.add_argument("--decode-workload", default="decode_128k")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-kl", action="store_true", help="skip the indexer KL target line")
    ap.add_argument("--no-backward", action="store_true", help="skip the sparse-stage gradient line")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run a small untimed case for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            reference_arm(args)
        return

    from sparse_attention_long_scores_b200.build import build
    if rank == 0 or not os.path.exists(os.path.join(ROOT, "sparse_attention_long_scores_b200", "libdsa.so")):
        build()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
        dist.barrier()

    pk = peaks()
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local
    sampler = ClockSampler(gpu_index) if rank == 0 else None
    pre = time_workload(args.workload, args.steps, args.warmup, world, rank, pk, sampler,
                        e2e=not args.no_e2e)
    kl = None
    if not args.no_kl:
        kl = time_indexer_kl(args.workload, args.steps, args.warmup, world, rank, pk)
    bwd = None
    if not args.no_backward:
        bwd = time_backward(args.workload, args.steps, args.warmup, world, rank, pk)
    dec = None
    if not args.no_decode:
        dec = time_workload(args.decode_workload, args.steps, args.warmup, world, rank, pk,
                            None, e2e=False)

    if rank == 0:
        cfg = pre["cfg"]
        dom_name = max(pre["kernels"], key=lambda k: pre["kernels"][k]["ms_per_step"])
        dom = dict(pre["roof"].get(dom_name, {}))
        dom.update({"kernel": dom_name, "peak_source": pk["source"]})
        dom.setdefault("traffic", None)
        line = {
            "metric": METRIC, "value": pre["tokens_per_s"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": pre["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
            "config": {"workload": cfg.name, "global_batch": cfg.B * world, "seq_len": cfg.Lk,
                       "per_gpu_batch": cfg.B, "indexer": f"H_I={cfg.H_I} d_I={cfg.d_I} e4m3",
                       "topk": cfg.k, "attention": f"H={cfg.H} Dqk={cfg.Dqk} Dv={cfg.Dv} bf16",
                       "parallelism": f"dp{world} (independent sequences per GPU)",
                       "l2": "inputs larger than L2 (no flush needed)"},
            "roofline": dom,
            "kernels": {k: {**v, **({"roofline": pre["roof"][k]} if k in pre["roof"] else {})}
                        for k, v in pre["kernels"].items()},
            "gpu_launches": pre["launches"],
            "clocks": pre["clocks"],
            "fused_schedule": pre["fused"],
        }
        if "e2e" in pre:
            line["e2e"] = pre["e2e"]
        if dec is not None:
            dc = dec["cfg"]
            line["decode"] = {
                "workload": dc.name, "value": dec["tokens_per_s"], "unit": "tokens/s",
                "ms_per_step": dec["ms"], "roofline": dec.get("step_roof"),
                "kernels": {k: {**v, **({"roofline": dec["roof"][k]} if k in dec["roof"] else {})}
                            for k, v in dec["kernels"].items()},
                "gpu_launches": dec["launches"],
                "fused_schedule": dec["fused"],
                "config": {"batch": dc.B, "cached_tokens": dc.Lk, "topk": dc.k},
            }
        if kl is not None:
            line["indexer_kl"] = kl
        if bwd is not None:
            if world == 1 and not args.no_cpu_baseline:
                bwd["cpu_baseline"] = cpu_baseline_backward(CONFIGS[bwd["workload"]])
            line["backward"] = bwd
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(cfg)
        print(json.dumps(line), flush=True)

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
