#!/usr/bin/env python
"""Sparse-decode benchmark on B200: the fused top-p decode step at a 128K-token KV cache.

One step = one pass of the whole decode path (low-rank index scores over all cached keys
-> histogram top-p selection with sink and window -> exact attention on the gathered K/V
rows -> log-sum-exp combine) for a batch of B=4 sequences x 32 query heads (8 per kv
head), N = 131072 cached tokens, d = 128, r = 16, p = 0.9, sink 4, window 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl spa|reference]

Prints ONE JSON line on rank 0.  ``value`` is the whole-job decode throughput in query
heads per second; the L2 is flushed (256 MiB write) before every step and each step is
timed on the device with CUDA events; the multi-GPU figure divides the units all ranks
processed by the max over ranks of the device time.  ``--impl reference`` times the fp64
CPU oracle on the same workload (rank 0 only).  Extra detail goes to stderr.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import DECODE_CONFIGS, decode_inputs, prefill_inputs  # noqa: E402
from synth.configs import C5  # noqa: E402
from synth.shard import batch_range, global_config  # noqa: E402

METRIC = "sparse-decode queries/s (query heads per second), 128K-token KV cache"
UNIT = "queries/s"
L2_FLUSH_BYTES = 256 << 20
KV_ROW_BYTES = lambda d: 2 * d * 2          # K + V row, bf16


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["spa", "reference"], default="spa")
    ap.add_argument("--config", default="c2_128k", choices=sorted(DECODE_CONFIGS) + ["c5", "c5q", "pbs_32k"],
                    help="decode workload (default); c5: the selection-block-shared prefill; c5q: the per-query "
                         "prefill (b_sel = 1) on the last 1024 queries of the c5 chunk; pbs_32k: the permuted "
                         "block-sparse prefill of a 32K-token sequence")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--local-fraction", type=float, default=0.0,
                    help="head-wise routing: this fraction of every sequence's units is local (sink + window)")
    ap.add_argument("--score", choices=["taylor", "minmax", "mean"], default=None,
                    help="block score of a block-scored workload (c3): second-order Taylor (its own), the min-max "
                         "page score or the mean-pooling score")
    ap.add_argument("--stats", choices=["f32", "bf16"], default=None,
                    help="storage of the block statistics of a block-scored workload (bf16 halves their bytes)")
    ap.add_argument("--rla", action="store_true",
                    help="add the residual linear attention over the rows outside each support (SPLA)")
    ap.add_argument("--path", choices=["separate", "fused"], default="separate",
                    help="decode kernels: separate kernels (default) or the fused persistent kernel where it applies")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = 3000 if a.impl == "spa" else 20
    if a.warmup is None:
        a.warmup = 50 if a.impl == "spa" else 3
    return a


def with_score(cfg, score, stats=None):
    """The workload with another block score or statistics storage (block-scored workloads only)."""
    if (score is None or score == cfg.score) and (stats is None or stats == cfg.stats):
        return cfg
    if cfg.score == "lowrank":
        raise SystemExit(f"--score / --stats apply to block-scored workloads; {cfg.name} uses low-rank index scores")
    return cfg.with_(score=score or cfg.score, stats=stats or cfg.stats)


def workload_desc(cfg):
    return (f"{cfg.name}: {cfg.select} decode, {cfg.score} scores"
            f"{' (bf16 block statistics)' if cfg.stats == 'bf16' else ''}, collapse={cfg.collapse}, B={cfg.B} "
            f"Hq={cfg.Hq} Hkv={cfg.Hkv} d={cfg.d} r={cfg.r} N={cfg.N} p={cfg.topp} k={cfg.topk} sink={cfg.sink} "
            f"window={cfg.window}")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source (profiles/traffic.tsv: kernel, workload, bytes, source sha256 prefix)."""
    path = os.path.join(ROOT, "profiles", "traffic.tsv")
    src = os.path.join(ROOT, "long_context_sparse_spa_b200", "csrc",
                       {"attend": "attend.cu", "scores": "scores.cu", "fused": "fused.cu"}.get(kernel, "select.cu"))
    if not os.path.exists(path) or not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for line in open(path):
        f = line.strip().split("\t")
        if len(f) == 4 and f[0] == kernel and f[1] == workload and f[3] == sha:
            return float(f[2])
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                x = [c.strip() for c in line.split(",")]
                if len(x) >= 9:
                    rows.append(x)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def rla_params(cfg):
    """RMSNorm scale and epsilon of the residual linear attention (a trained parameter in the
    method; fixed seeded values here)."""
    gamma = np.random.default_rng(11).uniform(0.5, 1.5, (cfg.Hq, cfg.d)).astype(np.float32)
    return {"gamma": gamma, "eps": 1e-6}


def cpu_baseline(cfg, x, seconds: float, local=None, rla=None):
    """The fp64 oracle's sparse path (scores -> selection -> attention), as it stands, on the
    host cores: units of the same workload cycled until the time budget is spent."""
    import oracle

    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    units = list(range(cfg.U))
    done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:      # whole rounds over all units
        oracle.decode(cfg, x, units=units, threads=cores, local=local, rla=rla)
        done += len(units)
    dt = time.perf_counter() - t0
    return {"value": done * cfg.heads_per_unit / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} units (one kv head of one sequence each, {cfg.heads_per_unit} query heads) of "
                      f"{cfg.name}, fp64 oracle, {dt:.1f} s"}


def captured_mass_report(cfg, x, idx, counts):
    """Captured mass on the GPU's supports (CPU leg, outside the timed region): for every unit,
    the oracle's dense head-averaged attention distribution over all N cached rows summed over
    the rows of the support the GPU selected ("Oracle-Guided Sparse Prefill" 2.1: the mass P
    a support keeps; "Full Attention Strikes Back" (RTPurbo), key results: attention mass
    beside sparsity)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max(1, cores)) as ex:
        vals = list(ex.map(lambda u: oracle.captured_mass(cfg, x, u, idx[u, :counts[u]]), range(cfg.U)))
    return {"mean": round(float(np.mean(vals)), 5), "min": round(float(np.min(vals)), 5),
            "units": f"all {cfg.U} units", "how": "fp64 oracle, dense head-averaged softmax over all N rows, "
            f"summed over the GPU's support ({time.perf_counter() - t0:.1f} s on {cores} host threads)"}


# ============================================================================ reference arm
def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = with_score(DECODE_CONFIGS[a.config], a.score, a.stats)
    import oracle

    x = decode_inputs(cfg)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    rla = rla_params(cfg) if a.rla else None
    # one step = one unit (a kv head of one sequence: its index scores over all N keys,
    # the top-p cut and exact attention for its query heads), cycling over the units
    for i in range(a.warmup):
        oracle.decode_unit(cfg, x, i % cfg.U, rla=rla)
    t0 = time.perf_counter()
    for i in range(a.steps):
        oracle.decode_unit(cfg, x, i % cfg.U, rla=rla)
    dt = time.perf_counter() - t0
    value = a.steps * cfg.heads_per_unit / dt
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": dt / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_desc(cfg) + (" + SPLA residual linear attention over the rows "
                                                         "outside each support" if rla is not None else ""),
                       "sample": "one unit per step, cycling over the units"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{a.steps} units of {cfg.name}, one per step, single thread "
                                       f"({cores} cores available)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ============================================================================ our arm
def run_spa(a):
    import torch
    import torch.distributed as dist

    import long_context_sparse_spa_b200 as spa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != a.gpus:
        log(f"note: --gpus {a.gpus} but WORLD_SIZE {world}; using WORLD_SIZE")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    base = with_score(DECODE_CONFIGS[a.config], a.score, a.stats)
    # weak scaling: every rank holds its own B sequences (a shard of a global batch of world*B)
    cfg_global = global_config(base, world)
    t = time.perf_counter()
    x = decode_inputs(cfg_global, batch=batch_range(base, rank, world))
    log(f"[rank {rank}] inputs generated in {time.perf_counter() - t:.1f} s")

    def up(arr):
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()

    cfg = base
    lowrank = cfg.score == "lowrank"
    dq, dK, dV = up(x["q"]), up(x["K"]), up(x["V"])
    kinds = {"lowrank": spa.SPA_SCORE_LOWRANK, "taylor": spa.SPA_SCORE_TAYLOR_BLOCK,
             "minmax": spa.SPA_SCORE_MINMAX_BLOCK, "mean": spa.SPA_SCORE_MEAN_BLOCK}
    kw = dict(score_kind=kinds[cfg.score],
              select_kind=spa.SPA_SELECT_TOPP if cfg.select == "topp" else spa.SPA_SELECT_TOPK,
              collapse=spa.SPA_COLLAPSE_GROUP_MEAN if cfg.collapse == "group" else spa.SPA_COLLAPSE_NONE,
              q=dq, K=dK, V=dV, block=cfg.block, score_scale=float(np.float32(cfg.score_scale)),
              sm_scale=float(np.float32(cfg.sm_scale)), topk=cfg.topk, topp=cfg.topp, sink=cfg.sink,
              window=cfg.window, cap=cfg.cap, want_f32=False, want_lse=False, run=False,
              kernel_path=spa.SPA_DECODE_FUSED if a.path == "fused" else spa.SPA_DECODE_SEPARATE)
    if lowrank:
        dqi, dKi = up(x["q_idx"]), up(x["Kidx"])
        kw.update(q_idx=dqi, Kidx=dKi)
    else:
        # block statistics: once per filled block, off the per-step path
        bf16_stats = cfg.stats == "bf16"
        if cfg.score == "minmax":
            bm, bv = spa.block_minmax(dK, cfg.block, bf16=bf16_stats)
        else:
            bm, bv = spa.block_stats(dK, cfg.block, bf16=bf16_stats)
            if cfg.score == "mean":
                bv = None
        kw.update(bmean=bm, bvar=bv)
    # head-wise routing: the first round(f * units per sequence) units of every sequence are local
    units_per_seq = cfg.U // cfg.B
    n_local = int(round(a.local_fraction * units_per_seq))
    local_np = np.array([int(u % units_per_seq < n_local) for u in range(cfg.U)], np.uint8)
    if n_local:
        kw["local_units"] = torch.from_numpy(local_np).cuda()
    # residual linear attention: the state of all N rows is built once, like a prefill would
    # (a decoder then appends one row per token); gamma and eps are fixed seeded values
    rla = rla_params(cfg) if a.rla else None
    if rla is not None:
        S, z = spa.rla_state(dK, dV)
        kw.update(rla_state=S, rla_z=z, rla_gamma=torch.from_numpy(rla["gamma"]).cuda(), rla_eps=rla["eps"])
    plan = spa.decode(**kw)
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    rbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")

    def flush_l2():
        # write a buffer larger than L2, then read another one so that the dirty lines are
        # written back here and not during the next timed step
        wbuf.zero_()
        rbuf.sum()

    for _ in range(a.warmup):
        flush_l2()
        plan.run()
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0, "device status raised during warm-up"
    counts = plan.count.cpu().numpy().astype(np.int64)
    sup_idx = plan.idx.cpu().numpy()
    rows = int(counts.sum()) * cfg.block
    M = cfg.N // cfg.block
    sparsity = 1.0 - counts.sum() / (cfg.U * M)

    # ---- timed region: K steps, L2 flushed before each; a step is bracketed by two events and
    # runs as one uninterrupted sequence of launches (events between its kernels would stop the
    # next kernel from being scheduled while the previous one drains)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(a.steps)]
    for e2 in ev:
        for e in e2:
            e.record()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for i in range(a.steps):
        flush_l2()
        ev[i][0].record()
        plan.run()
        ev[i][1].record()
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = np.array([ev[i][0].elapsed_time(ev[i][1]) for i in range(a.steps)])

    # ---- per-kernel split (for the roofline of the dominant kernel): a separate, untimed pass
    # with events between the kernels
    n_split = min(a.steps, 200)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_split)]
    for e4 in kev:
        for e in e4:
            e.record()
    for i in range(n_split):
        flush_l2()
        plan.run_timed(kev[i])
    torch.cuda.synchronize()
    fused = plan.fused
    k_names = ("fused", "none", "combine") if fused else ("scores", "select", "attend")
    k_ms = {name: np.array([kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(n_split)])
            for j, name in enumerate(k_names)}
    k_ms.pop("none", None)
    dev_s = float(step_ms.sum()) / 1e3
    t_max = dev_s
    if world > 1:
        tt = torch.tensor([dev_s], dtype=torch.float64, device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_max = float(tt.item())
    queries = cfg.B * cfg.Hq * a.steps * world
    value = queries / t_max

    # ---- algorithmic bytes (what the chosen support must move)
    d = cfg.d
    if lowrank:
        score_bytes = cfg.B * cfg.Hkv * cfg.N * cfg.r * 2 + cfg.B * cfg.Hq * cfg.r * 2
        if cfg.collapse == "group":      # a local unit's index keys are not read
            score_bytes -= int(local_np.sum()) * cfg.N * cfg.r * 2
    else:
        n_stats = 1 if cfg.score == "mean" else 2     # (mean) or (mean, var) / (min, max)
        n_stats *= 2 if cfg.stats == "bf16" else 4     # bytes per statistic
        score_bytes = n_stats * cfg.B * cfg.Hkv * M * d + cfg.B * cfg.Hq * d * 2
        if cfg.collapse == "group":      # a local unit's block statistics are not read
            score_bytes -= int(local_np.sum()) * n_stats * M * d
    attend_bytes = rows * KV_ROW_BYTES(d) + 2 * cfg.B * cfg.Hq * d * 2
    if rla is not None:      # the state (S, z) of every kv head and gamma, read once
        attend_bytes += cfg.B * cfg.Hkv * (d * d + d) * 4 + cfg.Hq * d * 4
    step_bytes = score_bytes + attend_bytes
    peak, peak_kind = peaks()
    mean_ms = {k: float(v.mean()) for k, v in k_ms.items()}
    if fused:
        # one kernel moves both streams (index keys and the gathered rows); the combine
        # kernel merges its records
        kbytes = {"fused": step_bytes, "combine": 0}
        dom = "fused"
    else:
        kbytes = {"scores": score_bytes, "attend": attend_bytes, "select": 0}
        dom = max(("scores", "attend"), key=lambda k: mean_ms[k])
    achieved = kbytes[dom] / (mean_ms[dom] * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": peak_kind,
                "traffic": recorded_traffic(dom, cfg.name + ("+rla" if rla is not None else "")),
                "step_achieved": step_bytes / (float(step_ms.mean()) * 1e-3) / 1e9,
                "step_frac": step_bytes / (float(step_ms.mean()) * 1e-3) / 1e9 / peak}
    roofline["algorithmic_bytes_per_launch"] = kbytes[dom]

    # ---- end to end through the public API with host buffers
    n_e2e = min(a.steps, 200)
    hq = x["q"].view(np.int16)
    pin_q = torch.from_numpy(np.ascontiguousarray(hq)).pin_memory()
    h2d = pin_q.numel() * 2
    pin_qi = None
    if lowrank:
        pin_qi = torch.from_numpy(np.ascontiguousarray(x["q_idx"].view(np.int16))).pin_memory()
        h2d += pin_qi.numel() * 2
    out_h = torch.empty(plan.out.shape, dtype=torch.bfloat16).pin_memory()
    cnt_h = torch.empty(plan.count.shape, dtype=torch.int32).pin_memory()
    d2h = out_h.numel() * 2 + cnt_h.numel() * 4
    e2e_ms = []
    for i in range(n_e2e + 3):
        flush_l2()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        dq.view(torch.int16).copy_(pin_q, non_blocking=True)
        if pin_qi is not None:
            dqi.view(torch.int16).copy_(pin_qi, non_blocking=True)
        plan.run()
        out_h.copy_(plan.out, non_blocking=True)
        cnt_h.copy_(plan.count, non_blocking=True)
        s1.record()
        s1.synchronize()
        if i >= 3:
            e2e_ms.append(s0.elapsed_time(s1))
    e2e_local = float(np.sum(e2e_ms)) / 1e3
    if world > 1:
        tt = torch.tensor([e2e_local], dtype=torch.float64, device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_local = float(tt.item())
    e2e_value = cfg.B * cfg.Hq * n_e2e * world / e2e_local

    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": float(step_ms.mean()), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_desc(cfg) + (" + SPLA residual linear attention over the rows outside "
                                                         "each support" if rla is not None else ""),
                       "global_batch": cfg.B * world, "seq_len": cfg.N,
                       "parallelism": f"dp{world} (independent sequence shards, no collective on the data path)",
                       "l2": "flushed before every step (256 MiB device write, then a 256 MiB read)",
                       "support_rows_per_step": rows, "sparsity": round(float(sparsity), 4),
                       "local_units": int(local_np.sum()), "rla": rla is not None,
                       "algorithmic_bytes_per_step": step_bytes},
            "roofline": roofline,
            "kernels_ms": {k: round(v, 5) for k, v in mean_ms.items()},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": float(np.mean(e2e_ms))},
            # per step: the fused persistent kernel and the combine; or scores (with the
            # level-0 histogram fused when one score row serves a kv head), [histogram],
            # selection, attention, log-sum-exp combine
            "gpu_launches": (2 if fused else (4 if (lowrank and cfg.collapse == "group") else 5)) * a.steps,
            "decode_path": "fused persistent kernel + combine" if fused else "separate kernels",
            "clocks": clocks,
            "wall_s_timed_region": w1 - w0,
        }
        if not a.no_cpu_baseline:
            line["config"]["captured_mass"] = captured_mass_report(cfg, x, sup_idx, counts)
        if not a.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(cfg, x, a.cpu_seconds, local=local_np if n_local else None,
                                                rla=rla)
        elif world > 1:
            line["cpu_baseline"] = None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def bf16_dev(x):
    import torch

    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def prefill_flops(cfg, counts):
    """Algorithmic flops of one prefill chunk: query row i of a block attends to the block's
    support and to the block's own rows up to i (QK^T and PV: 4 d flops per (query head, key))."""
    diag = cfg.bq * (cfg.bq + 1) // 2                 # sum over the block's rows of (i + 1)
    keys = cfg.bq * counts.astype(np.int64) + diag    # per unit and query head
    return float(4 * cfg.d * cfg.G * keys.sum())


def prefill_sparsity(cfg, counts):
    """1 - (keys a query reads) / (keys it may read causally), averaged over the chunk's queries:
    query t0 + i of a block reads its support and the block's own rows [t0, t0 + i]."""
    tot, read = 0.0, 0.0
    for u in range(cfg.U):
        j = u // cfg.Hkv
        t0 = cfg.q_start + j * cfg.bq
        for i in range(cfg.bq):
            tot += t0 + i + 1
            read += counts[u] + i + 1
    return 1.0 - read / tot


def prefill_captured_mass(cfg, x, idx, counts):
    """Captured mass of a fixed sample of prefill units (CPU leg, outside the timed region): four
    query blocks (first, one third, two thirds, last) x every kv head, all 64 queries each."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    blocks = sorted({0, cfg.n_blocks // 3, 2 * cfg.n_blocks // 3, cfg.n_blocks - 1})
    units = [(j, g) for j in blocks for g in range(cfg.Hkv)]
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    t0 = time.perf_counter()

    def one(jg):
        j, g = jg
        u = j * cfg.Hkv + g
        return oracle.captured_mass_prefill(cfg, x, j, g, idx[u, :counts[u]])

    with ThreadPoolExecutor(max(1, cores)) as ex:
        vals = list(ex.map(one, units))
    return {"mean": round(float(np.mean(vals)), 5), "min": round(float(np.min(vals)), 5),
            "units": f"{len(units)} units: query blocks {blocks} x {cfg.Hkv} kv heads",
            "how": "fp64 oracle, dense causal head-averaged softmax per query, summed over the support and the "
                   f"block's own rows ({time.perf_counter() - t0:.1f} s on {cores} host threads)"}


def pq_roofline(cfg, counts, ms):
    """Per-query prefill: a gather per (query, kv head), bound by memory.  Algorithmic bytes per
    step: every unit's index keys before its query (32 B each) and its gathered K/V rows
    (support + own position, 512 B each); most re-reads are L2 hits, so the fraction of the HBM
    copy peak can exceed 1."""
    hbm, kind = peaks()
    keys = sum(cfg.q_start + u // cfg.Hkv for u in range(cfg.U))
    rows = int(counts.sum()) + cfg.U
    byts = keys * cfg.r * 2 + rows * KV_ROW_BYTES(cfg.d)
    ach = byts / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "per-query prefill (all kernels of the step)", "achieved": ach, "peak": hbm,
            "unit": "GB/s", "frac": ach / hbm, "peak_source": kind, "traffic": None,
            "algorithmic_bytes_per_step": byts}


def run_prefill(a):
    """--config c5: the selection-block-shared prefill (one chunk of T queries), in TFLOP/s of
    its algorithmic flops; c5q: the per-query prefill (one support per query) on the last 1024
    queries of the same chunk; the L2 is flushed before every step."""
    import oracle

    cfg = C5 if a.config == "c5" else C5.with_(name="c5q", T=1024, q_start=C5.N - 1024, bq=1)
    if a.impl == "reference" and int(os.environ.get("RANK", "0")) != 0:
        return 0
    x = prefill_inputs(cfg)
    if a.impl == "reference":       # the fp64 oracle on host cores, one (query block, kv head) unit per step
        units = [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)]
        flops, t_tot = 0.0, 0.0
        for i in range(a.warmup + a.steps):
            j, g = units[i % len(units)]
            t0 = time.perf_counter()
            sup, _ = oracle.prefill_block(cfg, x, j, g)
            dt = time.perf_counter() - t0
            if i >= a.warmup:
                flops += prefill_flops(cfg.with_(T=cfg.bq), np.array([sup.size]))
                t_tot += dt
        v = flops / t_tot / 1e12
        print(json.dumps({"impl": "reference", "metric": "sparse-prefill TFLOP/s (algorithmic)", "value": v,
                          "unit": "TFLOP/s", "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
                          "ms_per_step": t_tot / a.steps * 1e3, "higher_is_better": True, "dtype": "f64",
                          "data": "synthetic", "config": {"workload": f"{cfg.name} prefill, one unit per step"},
                          "cpu_baseline": {"kind": "oracle", "cores": 1, "value": v,
                                           "sample": f"{a.steps} (query block, kv head) units, fp64 oracle"},
                          "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0
    import torch

    import long_context_sparse_spa_b200 as spa

    plan = spa.prefill(Q=bf16_dev(x["Q"]), q_idx=bf16_dev(x["q_idx"]), K=bf16_dev(x["K"]), V=bf16_dev(x["V"]),
                       Kidx=bf16_dev(x["Kidx"]), q_start=cfg.q_start, score_scale=float(np.float32(cfg.score_scale)),
                       sm_scale=float(np.float32(cfg.sm_scale)), topk=cfg.topk, sink=cfg.sink, bq=cfg.bq,
                       want_f32=False, run=False)
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    rbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
    for _ in range(a.warmup):
        wbuf.zero_(); rbuf.sum(); plan.run()
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0, "device status raised during warm-up"
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(a.steps)]
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    for i in range(a.steps):
        wbuf.zero_(); rbuf.sum()
        ev[i][0].record(); plan.run(); ev[i][1].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    counts = plan.count.cpu().numpy()
    flops = prefill_flops(cfg, counts)
    tflops = flops / (ms * 1e-3) / 1e12
    # the tcgen05 attention kernel alone, in a separate pass (events around it inside the step)
    kern_ms = timed_attention_ms(plan, a.steps, lambda: (wbuf.zero_(), rbuf.sum())) if cfg.bq > 1 else None
    # end to end: the chunk's queries (Q, q_idx) from pinned host memory, output read back
    hq = [torch.from_numpy(np.ascontiguousarray(x[k]).view(np.int16)).pin_memory() for k in ("Q", "q_idx")]
    dq = [plan.keep[0], plan.keep[1]]
    hout = torch.empty(plan.out.shape, dtype=plan.out.dtype).pin_memory()
    n_e2e = min(a.steps, 50)
    e2e = []
    for i in range(n_e2e + 2):
        wbuf.zero_(); rbuf.sum(); torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for h, d in zip(hq, dq):
            d.view(torch.int16).copy_(h, non_blocking=True)
        plan.run()
        hout.copy_(plan.out, non_blocking=True)
        s1.record(); s1.synchronize()
        if i >= 2:
            e2e.append(s0.elapsed_time(s1))
    e2e_ms = float(np.mean(e2e))
    peak = None
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            peak = float(json.load(f)["bf16_tflops"])
    peak_kind = "measured" if peak else "fallback"
    peak = peak or 1590.0
    # the oracle on a bounded sample of units (one host core per unit, all cores)
    cpu = None
    mass = None
    if not a.no_cpu_baseline:
        mass = prefill_captured_mass(cfg, x, plan.idx.cpu().numpy(), counts)
    if not a.no_cpu_baseline:
        units = [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)]
        t0, done, cf = time.perf_counter(), 0, 0.0
        while time.perf_counter() - t0 < a.cpu_seconds and done < len(units):
            j, g = units[done]
            sup, _ = oracle.prefill_block(cfg, x, j, g)
            cf += prefill_flops(cfg.with_(T=cfg.bq), np.array([sup.size]))
            done += 1
        dt = time.perf_counter() - t0
        cpu = {"value": cf / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": f"{done} (query block, kv head) units of {cfg.name}, fp64 oracle, {dt:.1f} s"}
    kind = "selection-block-shared" if cfg.bq > 1 else "per-query (b_sel = 1)"
    out = {"metric": f"sparse-prefill TFLOP/s (algorithmic), {kind}", "value": tflops,
           "unit": "TFLOP/s", "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"{cfg.name}: prefill chunk T={cfg.T} at q_start={cfg.q_start}, N={cfg.N}, "
                                  f"Hq={cfg.Hq} Hkv={cfg.Hkv} d={cfg.d} bq={cfg.bq} top-k={cfg.topk} sink={cfg.sink}",
                      "l2": "flushed before every step (256 MiB device write, then a 256 MiB read)",
                      "support_mean": float(counts.mean()), "algorithmic_gflop_per_step": flops / 1e9,
                      "sparsity": round(float(prefill_sparsity(cfg, counts)), 4), "captured_mass": mass},
           "roofline": (attention_roofline(flops, kern_ms, tflops, peak, peak_kind) if cfg.bq > 1
                        else pq_roofline(cfg, counts, ms)),
           "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": int(sum(h.numel() * 2 for h in hq)),
                   "d2h_bytes_per_step": int(hout.numel() * 2), "ms_per_step": e2e_ms},
           "gpu_launches": (6 if cfg.bq > 1 else 7) * a.steps, "clocks": clocks, "cpu_baseline": cpu}
    print(json.dumps(out))
    return 0


def timed_attention_ms(plan, steps, flush):
    """Mean duration of the prefill's tcgen05 attention kernel: events recorded right before and
    right after it inside real steps (run_timed), the L2 flushed before each step."""
    import torch

    k = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for e in k:
        e.record()
    out = []
    for i in range(min(steps, 20) + 2):
        flush()
        plan.run_timed(k)
        torch.cuda.synchronize()
        if i >= 2:
            out.append(k[0].elapsed_time(k[1]))
    return float(np.mean(out))


def attention_roofline(att_flops, kern_ms, step_tflops, peak, peak_kind):
    """Roofline of the tcgen05 attention kernel at its algorithmic flops (4 d per query head and
    attended key), against the dense bf16 peak; step_frac applies the same to the whole step."""
    achieved = att_flops / (kern_ms * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": "prefill_attend_kernel", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_kind, "kernel_ms": kern_ms,
            "step_frac": step_tflops / peak, "traffic": None}


def pbs_rows(cfg, u, i, counts):
    """Keys attended by query i of unit u of a permuted block-sparse prefill, and its causal keys."""
    j = u // cfg.Hkv
    t0 = j * cfg.b
    seg0 = t0 // cfg.S * cfg.S
    return int(counts[u]) + (t0 - seg0) + i + 1, t0 + i + 1


def pbs_sparsity(cfg, counts):
    """Mean over units of the fraction of causal keys a query does not attend (queries averaged)."""
    out = []
    for u in range(cfg.U):
        att = sum(pbs_rows(cfg, u, i, counts)[0] for i in range(cfg.b))
        cau = sum(pbs_rows(cfg, u, i, counts)[1] for i in range(cfg.b))
        out.append(1.0 - att / cau)
    return float(np.mean(out))


def pbs_captured_mass(cfg, x, idx, counts, n_units=8, queries=(0, 31, 63)):
    """Dense head-averaged causal softmax mass on the attended rows (kept keys, the own segment's
    earlier keys, the causal diagonal), from the oracle, for a spread sample of units."""
    import oracle

    G, b = cfg.G, cfg.b
    units = np.linspace(cfg.Hkv * (cfg.S // b), cfg.U - 1, n_units).astype(int)   # units past the first segment
    vals = []
    for u in units:
        j, g = u // cfg.Hkv, u % cfg.Hkv
        t0 = j * b
        seg0 = t0 // cfg.S * cfg.S
        sup = idx[u, :counts[u]].astype(np.int64)
        for i in queries:
            t = t0 + i
            P = oracle.dense_probs(x["Q"][t, g * G:(g + 1) * G], x["K"][g, :t + 1], float(np.float32(cfg.sm_scale)))
            rows = np.union1d(sup, np.arange(seg0, t + 1))
            vals.append(float(P[rows].sum()))
    return {"mean": round(float(np.mean(vals)), 5), "min": round(float(np.min(vals)), 5),
            "units": f"{len(units)} units (query blocks past the first segment, spread) x queries {list(queries)}",
            "how": "fp64 oracle dense head-averaged causal softmax, summed over the attended rows"}


def pbs_flops(cfg, counts):
    """Algorithmic flops of a permuted block-sparse prefill: the importance pass (2 d per query
    row of the last block and key, b*G rows per kv head) and the attention (4 d per (query head,
    key) over the kept keys, the own segment's earlier keys and the causal diagonal)."""
    imp = 2.0 * cfg.d * cfg.b * cfg.G * cfg.T * cfg.Hkv
    att = 0.0
    diag = cfg.b * (cfg.b + 1) // 2
    for u in range(cfg.U):
        j = u // cfg.Hkv
        t0 = j * cfg.b
        keys = cfg.b * (int(counts[u]) + t0 - t0 // cfg.S * cfg.S) + diag
        att += 4.0 * cfg.d * cfg.G * keys
    return imp + att


def run_pbs(a):
    """--config pbs_32k: the permuted block-sparse prefill (PBS-Attn) of one 32K-token sequence,
    in TFLOP/s of its algorithmic flops; the L2 is flushed before every step."""
    import oracle
    from synth import PBS_32K, pbs_inputs

    cfg = PBS_32K
    if a.impl == "reference" and int(os.environ.get("RANK", "0")) != 0:
        return 0
    x = pbs_inputs(cfg)
    b, G, T, S = cfg.b, cfg.G, cfg.T, cfg.S
    sm = float(np.float32(cfg.sm_scale))

    def oracle_sample(budget_s):
        """The oracle on a bounded sample: kv head 0's importance and permutation, then query
        blocks of that head from the end of the sequence until the budget is spent."""
        t0 = time.perf_counter()
        imp = oracle.pbs_importance(x["Q"][T - b:, 0:G], T - b, x["K"][0], sm)
        perm = oracle.pbs_permutation(imp, S)
        fl = 2.0 * cfg.d * b * G * T
        done = 0
        for j in range(cfg.n_blocks - 1, -1, -1):
            if time.perf_counter() - t0 > budget_s and done:
                break
            sup, _ = oracle.pbs_prefill_unit(x["Q"][j * b:(j + 1) * b, 0:G], j * b, x["K"][0], x["V"][0], perm, S,
                                             cfg.topk, sm)
            t_0 = j * b
            fl += 4.0 * cfg.d * G * (b * (sup.size + t_0 - t_0 // S * S) + b * (b + 1) // 2)
            done += 1
        dt = time.perf_counter() - t0
        return fl / dt / 1e12, dt, done

    if a.impl == "reference":
        v, dt, done = oracle_sample(a.cpu_seconds)
        print(json.dumps({"impl": "reference", "metric": "permuted block-sparse prefill TFLOP/s (algorithmic)",
                          "value": v, "unit": "TFLOP/s", "n_gpus": a.gpus, "steps": 1, "warmup": 0,
                          "ms_per_step": dt * 1e3, "higher_is_better": True, "dtype": "f64", "data": "synthetic",
                          "config": {"workload": f"{cfg.name}: kv head 0 importance + {done} query blocks"},
                          "cpu_baseline": {"kind": "oracle", "cores": 1, "value": v,
                                           "sample": f"kv head 0: importance, permutation, {done} query blocks"},
                          "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0
    import torch

    import long_context_sparse_spa_b200 as spa

    dQ, dK, dV = bf16_dev(x["Q"]), bf16_dev(x["K"]), bf16_dev(x["V"])
    plan = spa.pbs_prefill(Q=dQ, K=dK, V=dV, sm_scale=sm, S=S, topk=cfg.topk, b=b, want_f32=False, run=False)
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    rbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
    for _ in range(a.warmup):
        wbuf.zero_(); rbuf.sum(); plan.run()
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0, "device status raised during warm-up"
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(a.steps)]
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    for i in range(a.steps):
        wbuf.zero_(); rbuf.sum()
        ev[i][0].record(); plan.run(); ev[i][1].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    counts = plan.count.cpu().numpy()
    flops = pbs_flops(cfg, counts)
    tflops = flops / (ms * 1e-3) / 1e12
    att_flops = flops - 2.0 * cfg.d * b * G * T * cfg.Hkv      # without the importance pass
    kern_ms = timed_attention_ms(plan, a.steps, lambda: (wbuf.zero_(), rbuf.sum()))
    hq = torch.from_numpy(np.ascontiguousarray(x["Q"]).view(np.int16)).pin_memory()
    hout = torch.empty(plan.out.shape, dtype=plan.out.dtype).pin_memory()
    e2e = []
    for i in range(min(a.steps, 20) + 2):
        wbuf.zero_(); rbuf.sum(); torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        dQ.view(torch.int16).copy_(hq, non_blocking=True)
        plan.run()
        hout.copy_(plan.out, non_blocking=True)
        s1.record(); s1.synchronize()
        if i >= 2:
            e2e.append(s0.elapsed_time(s1))
    e2e_ms = float(np.mean(e2e))
    peak, peak_kind = None, "fallback"
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            peak = float(json.load(f)["bf16_tflops"])
        peak_kind = "measured"
    peak = peak or 1590.0
    cpu = None
    mass = None
    if not a.no_cpu_baseline:
        mass = pbs_captured_mass(cfg, x, plan.idx.cpu().numpy(), counts)
        v, dt, done = oracle_sample(a.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": f"kv head 0: importance, permutation and {done} query blocks, fp64 oracle, {dt:.1f} s"}
    out = {"metric": "permuted block-sparse prefill TFLOP/s (algorithmic)", "value": tflops, "unit": "TFLOP/s",
           "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"{cfg.name}: causal prefill T={T}, Hq={cfg.Hq} Hkv={cfg.Hkv} d={cfg.d} b={b} "
                                  f"S={S} top-k={cfg.topk} blocks",
                      "l2": "flushed before every step (256 MiB device write, then a 256 MiB read)",
                      "kept_blocks_mean": float(counts.mean() / b), "algorithmic_gflop_per_step": flops / 1e9,
                      "sparsity": round(pbs_sparsity(cfg, counts), 4), "captured_mass": mass},
           "roofline": attention_roofline(att_flops, kern_ms, tflops, peak, peak_kind),
           "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": int(hq.numel() * 2), "d2h_bytes_per_step": int(hout.numel() * 2),
                   "ms_per_step": e2e_ms},
           "gpu_launches": 11 * a.steps, "clocks": clocks, "cpu_baseline": cpu}
    print(json.dumps(out))
    return 0


def main():
    a = parse()
    if a.config == "pbs_32k":
        return run_pbs(a)
    if a.config in ("c5", "c5q"):
        return run_prefill(a)
    if a.impl == "reference":
        return run_reference(a)
    return run_spa(a)


if __name__ == "__main__":
    sys.exit(main())
