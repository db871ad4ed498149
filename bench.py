"""Benchmark of the FASA decode hot path on B200 (prints one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2] [--layers 32]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

A step is one FASA decode (fasa_decode: TIP score -> top-k -> focused
attention) of every layer of a stack of independent layer caches, each
holding the configuration's synthetic KV cache and dominant-FC sketch. The
stack is larger than L2, so every layer's data comes from HBM. Steps are
replayed from one CUDA graph. `value` is achieved HBM GB/s on the algorithmic
(roofline) bytes: sketch of every cached token + K/V rows of the kept tokens +
query and output. Multi-GPU runs are independent replicas (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rope_frequency_chunk_b200 import workloads as W  # noqa: E402

METRIC = "fasa_decode µs/layer-step and achieved HBM GB/s vs peak (32K ctx, k=256)"
L2_BYTES = 126 * 2 ** 20


def roofline_bytes(wl: W.Workload, k: int | None = None, n_dom: int | None = None) -> int:
    """Algorithmic bytes of one decode layer-step (sketch + kept K/V rows + q/out)."""
    k = wl.k if k is None else k
    n_dom = wl.n_dom if n_dom is None else n_dom
    es = wl.elem_bytes
    k_eff = min(k, wl.ctx_len)
    sketch = wl.batch * wl.n_kv_heads * wl.ctx_len * 2 * n_dom * es
    rows = wl.batch * wl.n_kv_heads * k_eff * 2 * W.HEAD_DIM * es
    qo = 2 * wl.batch * wl.n_q_heads * W.HEAD_DIM * es
    return sketch + rows + qo


def sketch_bytes(wl: W.Workload) -> int:
    return wl.batch * wl.n_kv_heads * wl.ctx_len * 2 * wl.n_dom * wl.elem_bytes


def dense_bytes(wl: W.Workload) -> int:
    es = wl.elem_bytes
    return (wl.batch * wl.n_kv_heads * wl.ctx_len * 2 * W.HEAD_DIM * es
            + 2 * wl.batch * wl.n_q_heads * W.HEAD_DIM * es)


def default_layers(wl: W.Workload) -> int:
    per_layer = roofline_bytes(wl)
    n = 32 if wl.name in ("c1", "c2", "c4") else 2
    while n * per_layer < 3 * L2_BYTES and n < 4096:
        n *= 2
    return n


HBM_NOMINAL_GBS = 7700.0  # B200 HBM3e, the HGX figure (context beside the measured peak)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def csrc_sha256(files=None) -> str:
    """Digest of the code of the named library sources (default: all), in
    name order, with comments and runs of white space removed: a figure
    captured from the code holds while that code is unchanged."""
    import hashlib
    import re
    d = os.path.join(ROOT, "rope_frequency_chunk_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(files or os.listdir(d)):
        with open(os.path.join(d, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        text = " ".join(text.split())
        h.update(name.encode() + b"\0" + text.encode() + b"\0")
    return h.hexdigest()


def workload_sig(wl: W.Workload, k: int) -> str:
    """The shape a launch processes: config, batch, heads, context, FCs, budget."""
    return f"{wl.name}-B{wl.batch}-H{wl.n_q_heads}/{wl.n_kv_heads}-L{wl.ctx_len}-n{wl.n_dom}-k{k}-{wl.dtype}"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) of `kernel` on this workload from
    the ncu record in profiles/traffic.json, or None: a figure holds only
    while the library's sources hash to the digest it was captured under."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    e = rec.get(f"{kernel}@{workload}")
    if not e or e.get("csrc_sha256") != csrc_sha256(e.get("sources")):
        return None
    return int(e["bytes_per_launch"])


# ------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.25)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------- oracle leg

def oracle_units(wl: W.Workload, n: int):
    """Prepare n distinct (layer, b, g) units for the oracle (untimed): inputs
    from the generator, cache contents from the oracle's own append."""
    import oracle.fasa_oracle as O
    units = []
    for u in range(n):
        layer, rem = divmod(u, wl.batch * wl.n_kv_heads)
        b, g = divmod(rem, wl.n_kv_heads)
        lp = W.layer_params(wl, layer)
        kk, vv = W.head_kv(wl, lp, layer, b, g)
        qq = W.head_q(wl, lp, layer, b, g)
        k_rot, v_st, sk = O.append_kv(kk, vv, 0, wl.rope_base, lp.dom_idx[g], wl.dtype)
        units.append((qq, k_rot, v_st, sk, lp.dom_idx[g]))
    return units


def oracle_time(wl: W.Workload, units, k: int, budget_s: float = 0.0, calls: int | None = None):
    """Time oracle decodes (one KV head each), cycling over prepared units,
    single-threaded; returns (roofline bytes processed, seconds, calls)."""
    import oracle.fasa_oracle as O
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1)
    except Exception:  # pragma: no cover
        limiter = None
    per_unit = roofline_bytes(wl, k) / (wl.batch * wl.n_kv_heads)
    done, spent = 0, 0.0
    while (calls is None and spent < budget_s) or (calls is not None and done < calls):
        qq, k_rot, v_st, sk, dom = units[done % len(units)]
        t0 = time.perf_counter()
        O.decode_head(qq, wl.q_pos, k_rot, v_st, sk, dom, k, wl.rope_base)
        spent += time.perf_counter() - t0
        done += 1
    if limiter is not None:
        limiter.unregister()
    return per_unit * done, spent, done


# ------------------------------------------------ oracle on every host core

_POOL_UNITS = None


def _pool_init(name, overrides, n_units, k):
    """Worker set-up (untimed): one BLAS thread, the worker's own prepared units."""
    global _POOL_UNITS
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass
    wl = W.CONFIGS[name].replace(**overrides)
    _POOL_UNITS = (wl, oracle_units(wl, n_units), k)


def _pool_run(calls):
    """`calls` oracle decodes on this worker; returns the bytes they cover."""
    wl, units, k = _POOL_UNITS
    b, _, _ = oracle_time(wl, units, k, calls=calls)
    return b


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_all_cores(wl: W.Workload, k: int, budget_s: float, cores: int | None = None):
    """The oracle decode, one (sequence, KV head) per call, on every host core
    at once: a spawned process pool (one single-threaded worker per core, so
    no fork after CUDA), each worker cycling over its own prepared heads.
    Returns (bytes, wall seconds, calls, cores). The pool start and the
    workers' preparation are not timed; timed rounds of doubling size run
    until about budget_s of wall time is spent."""
    import multiprocessing as mp
    cores = cores or host_cores()
    overrides = {f: getattr(wl, f) for f in ("batch", "ctx_len", "k", "n_dom")}
    ctx = mp.get_context("spawn")
    n_units = min(2, wl.batch * wl.n_kv_heads)
    with ctx.Pool(cores, initializer=_pool_init, initargs=(wl.name, overrides, n_units, k)) as pool:
        pool.map(_pool_run, [1] * cores, chunksize=1)  # every worker up and warm (untimed)
        total, wall, done, calls = 0.0, 0.0, 0, 4
        while wall < budget_s:  # rounds of growing size until the budget is spent
            t0 = time.perf_counter()
            total += sum(pool.map(_pool_run, [calls] * cores, chunksize=1))
            wall += time.perf_counter() - t0
            done += calls
            calls *= 2
    return total, wall, done * cores, cores


def run_reference(args, wl):
    """The reference arm: the float64 oracle (the only reference there is),
    on every host core, each step a bounded sample of the workload's
    (sequence, KV head) units."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    k = args.k or wl.k
    steps = max(1, args.steps)
    budget = max(1.0, min(float(args.cpu_seconds), 150.0 / steps))
    total_b, total_t, calls, cores = 0.0, 0.0, 0, host_cores()
    for _ in range(steps):
        b, t, c, cores = oracle_all_cores(wl, k, budget)
        total_b += b
        total_t += t
        calls += c
    gbs = total_b / total_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "ctx_len": wl.ctx_len, "k": k, "n_dom": wl.n_dom,
                   "heads": f"{wl.n_q_heads}/{wl.n_kv_heads}"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{steps} steps of about {budget:.0f} s, {calls} oracle decodes of one "
                                   f"(sequence, KV head) of {wl.name} each, float64 numpy, one single-threaded "
                                   f"process per host core ({cores})"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU leg

def build_stack(wl, n_layers, device, kv_on_host=False):
    import torch
    from rope_frequency_chunk_b200 import fasa as F
    caches, qs = [], []
    for layer in range(n_layers):
        inp = W.layer_inputs(wl, layer=layer)
        c = F.KVCache(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.n_dom, wl.ctx_len, wl.dtype, wl.rope_base,
                      inp.params.dom_idx, device=device, kv_on_host=kv_on_host)
        k = W.to_torch(inp.k, device)
        v = W.to_torch(inp.v, device)
        F.fasa_append_kv(c, k, v, 0)
        del k, v
        caches.append(c)
        qs.append(W.to_torch(inp.q, device))
        del inp
    torch.cuda.synchronize()
    return caches, qs


def time_graph(fn, steps, warmup, stream, dist=None, per_step=None):
    """Capture fn() (one step) in a CUDA graph; replay warmup + steps; return
    device ms for the steps (events on the replay stream), max over ranks.
    With a list `per_step`, also appends each step's device ms (an event
    between consecutive replays)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for i in range(steps):
            g.replay()
            ev[i + 1].record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, "cuda")
    if per_step is not None:
        per_step.extend(ev[i].elapsed_time(ev[i + 1]) for i in range(steps))
    torch.cuda.synchronize()
    del g
    return ms


def max_over_ranks(value: float, dist=None, device: str = "cuda") -> float:
    """The largest of every rank's value (every rank gets it); the value itself
    on one process."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.barrier()
    return float(t.item())


def job_gbs(bytes_per_rank_step: float, ms_per_step: float, world: int) -> float:
    """Whole-job GB/s: every rank moved bytes_per_rank_step per step, and a step
    took ms_per_step (the slowest rank's time)."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


FASA_M_MAX_HOST_BYTES = 16 << 30


def link_copy_gbs(device, nbytes=256 << 20, reps=5):
    """Pinned host -> device copy bandwidth (the host link as the copy engine
    sees it), CUDA events on the copying stream."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    st = torch.cuda.Stream(device=device)
    with torch.cuda.stream(st):
        dst.copy_(src, non_blocking=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(reps):
            dst.copy_(src, non_blocking=True)
        e1.record(st)
    torch.cuda.synchronize()
    return reps * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9


def run_fasa_m(args, wl, k, n_layers, qs, outs, ws, stream, fasa_c_bytes):
    """FASA-M: the same decode on caches whose K and V sit in pinned host
    memory (only the sketch on the device); kept rows cross the host link."""
    import torch
    from rope_frequency_chunk_b200 import fasa as F
    hcaches, _ = build_stack(wl, n_layers, qs[0].device, kv_on_host=True)
    L = wl.ctx_len

    def m_step():
        for c, q, o in zip(hcaches, qs, outs):
            F.fasa_decode(c, L, q, wl.q_pos, k, out=o, workspace=ws)

    msteps = max(3, args.steps // 4)
    per = []
    ms = time_graph(m_step, msteps, args.warmup, stream, None, per_step=per) / msteps
    status = F.fasa_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the FASA-M decode")
    link_bytes = wl.batch * wl.n_kv_heads * min(k, L) * 2 * W.HEAD_DIM * wl.elem_bytes
    copy_gbs = link_copy_gbs(qs[0].device)
    us = 1e3 * ms / n_layers
    res = {"us_per_layer_step": us,
           "us_per_layer_step_percentiles": {f"p{p}": float(np.percentile(per, p)) * 1e3 / n_layers
                                             for p in (10, 50, 90)},
           "gpu_resident_bytes_per_layer": hcaches[0].device_bytes(),
           "fasa_c_resident_bytes_per_layer": fasa_c_bytes,
           "gpu_memory_compression": fasa_c_bytes / hcaches[0].device_bytes(),
           "link_bytes_per_layer_step": link_bytes,
           "link_gbs": link_bytes / (us * 1e-6) / 1e9,
           "link_copy_gbs": copy_gbs,
           "link_frac_of_copy": link_bytes / (us * 1e-6) / 1e9 / copy_gbs,
           "hbm_bytes_per_layer_step": roofline_bytes(wl, k) - link_bytes,
           "note": "K and V in pinned host memory read by the kernels across the host link; the sketch, "
                   "queries and outputs in HBM; link_copy_gbs is a pinned host-to-device copy for scale"}
    del hcaches
    torch.cuda.synchronize()
    return res


def run_multi_query(args, wl, k, n_layers, caches, stream, us_single):
    """Multi-query decode legs: n_q tokens per sequence (one shared kept set
    per KV head, attention on the tensor cores) on the same layer stack."""
    import torch
    from rope_frequency_chunk_b200 import fasa as F
    G = wl.group
    L = wl.ctx_len
    res = {}
    for n_q in args.multi:
        if n_q * G > 64 or n_q > 16:
            continue
        qs = [W.to_torch(W.multi_queries(wl, n_q, layer=i), caches[0].k.device) for i in range(n_layers)]
        outs = [torch.empty_like(q) for q in qs]
        ws = F.fasa_decode_multi_workspace(caches[0], L, n_q, k)

        def step():
            for c, q, o in zip(caches, qs, outs):
                F.fasa_decode_multi(c, L, q, wl.q_pos, k, out=o, workspace=ws)

        msteps = max(3, args.steps // 4)
        per = []
        ms = time_graph(step, msteps, args.warmup, stream, None, per_step=per) / msteps
        status = F.fasa_device_status(clear=True)
        if status != 0:
            raise RuntimeError(f"device status {status} after the multi-query decode")
        us = 1e3 * ms / n_layers
        qbytes = 2 * wl.batch * n_q * wl.n_q_heads * W.HEAD_DIM * wl.elem_bytes
        byts = roofline_bytes(wl, k) - 2 * wl.batch * wl.n_q_heads * W.HEAD_DIM * wl.elem_bytes + qbytes
        res[str(n_q)] = {"us_per_layer_step": us,
                         "us_per_layer_step_p50": float(np.percentile(per, 50)) * 1e3 / n_layers,
                         "query_rows_per_kv_head": n_q * G, "bytes_per_layer_step": byts,
                         "gbs": byts / (us * 1e-6) / 1e9, "us_per_query_token": us / n_q,
                         "speedup_vs_single_query_decodes": n_q * us_single / us}
        del qs, outs, ws
    return res


def run_fasa(args, wl):
    import torch
    from rope_frequency_chunk_b200 import fasa as F

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    device = f"cuda:{local}"
    torch.cuda.set_device(local)
    F.lib()
    F.fasa_set_decode_path({"auto": F.DECODE_AUTO, "fused": F.DECODE_FUSED, "staged": F.DECODE_STAGED}[args.plan])

    k = args.k or wl.k
    n_layers = args.layers or default_layers(wl)
    caches, qs = build_stack(wl, n_layers, device)
    outs = [torch.empty_like(q) for q in qs]
    ws = torch.zeros(max(F.fasa_decode_workspace_bytes(c, wl.ctx_len, k) for c in caches), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.Stream(device=device)
    L = wl.ctx_len

    def decode_step():
        for c, q, o in zip(caches, qs, outs):
            F.fasa_decode(c, L, q, wl.q_pos, k, out=o, workspace=ws)

    scores = torch.empty(wl.batch, wl.n_kv_heads, L, dtype=torch.float32, device=device)

    def score_step():
        for c, q in zip(caches, qs):
            F.fasa_score(c, L, q, wl.q_pos, scores=scores)

    dws = F.fasa_dense_workspace(caches[0], L, device)

    def dense_step():
        for c, q, o in zip(caches, qs, outs):
            F.fasa_dense_decode(c, L, q, wl.q_pos, out=o, workspace=dws)

    plan = F.fasa_decode_path(caches[0], L, k)
    launches = F.fasa_decode_launches(caches[0], L, k)
    hbm_peak, peak_kind = peaks()
    step_ms = []
    with ClockSampler(local) as clk:
        ms = time_graph(decode_step, args.steps, args.warmup, stream, dist, per_step=step_ms)
    clocks = clk.summary()
    status = F.fasa_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed decode")

    per_layer_bytes = roofline_bytes(wl, k)
    step_bytes = per_layer_bytes * n_layers
    ms_step = ms / args.steps
    us_layer = 1e3 * ms_step / n_layers
    gbs = job_gbs(step_bytes, ms_step, world)
    us_dist = {f"p{q}": float(np.percentile(step_ms, q)) * 1e3 / n_layers for q in (10, 50, 90)}

    # the roofline is the whole decode of a layer (all of its launches,
    # back to back in the replayed graph); for the fused plan with one
    # launch per layer that is the fused kernel itself
    fused = plan == F.DECODE_FUSED
    kern = {1: "decode_wide_kernel (score + select + attend, one launch per layer)",
            2: "decode_wide_kernel + attend_mma_kernel (two launches per layer)",
            3: "decode_wide_kernel + attend_mma_kernel + attend_merge_kernel (three launches per layer)",
            4: "score_kernel + filter_kernel + finalize_kernel + attend (four launches per layer)",
            5: "score_kernel + filter_kernel + finalize_kernel + attend + split merge (five launches per layer)"
            }[launches]
    roof = {"bound": "hbm", "kernel": kern, "achieved": gbs / world, "peak": hbm_peak, "unit": "GB/s",
            "frac": gbs / world / hbm_peak,
            "traffic": profiled_traffic("decode_wide_kernel", workload_sig(wl, k)) if launches == 1 else None,
            "bytes_per_launch": per_layer_bytes, "peak_kind": peak_kind, "us_per_launch": us_layer,
            "nominal_peak": HBM_NOMINAL_GBS, "frac_nominal": gbs / world / HBM_NOMINAL_GBS,
            "us_per_layer_percentiles": us_dist}
    if not fused:
        ms_score = time_graph(score_step, args.steps, args.warmup, stream, dist) / args.steps
        score_gbs = sketch_bytes(wl) * n_layers / (ms_score * 1e-3) / 1e9
        roof["score_kernel"] = {"achieved": score_gbs, "frac": score_gbs / hbm_peak,
                                "bytes_per_launch": sketch_bytes(wl), "us_per_launch": 1e3 * ms_score / n_layers}

    extra = {}
    if not args.no_dense:
        dsteps = max(3, args.steps // 8)
        ms_dense = time_graph(dense_step, dsteps, args.warmup, stream, dist) / dsteps
        extra["dense_us_per_layer_step"] = 1e3 * ms_dense / n_layers
        extra["dense_gbs"] = dense_bytes(wl) * n_layers / (ms_dense * 1e-3) / 1e9
        extra["speedup_vs_dense"] = ms_dense / ms_step

    if args.multi and wl.dtype == "bf16" and world == 1:
        extra["multi_query"] = run_multi_query(args, wl, k, n_layers, caches, stream, us_layer)

    kv_host_bytes = 2 * wl.batch * wl.n_kv_heads * L * W.HEAD_DIM * wl.elem_bytes * n_layers
    if not args.no_fasa_m and world == 1 and kv_host_bytes <= FASA_M_MAX_HOST_BYTES:
        extra["fasa_m"] = run_fasa_m(args, wl, k, n_layers, qs, outs, ws, stream, caches[0].device_bytes())
    elif not args.no_fasa_m:
        extra["fasa_m"] = {"skipped": f"host K/V of {kv_host_bytes / 2**30:.1f} GiB for {n_layers} layers "
                                      f"exceeds the {FASA_M_MAX_HOST_BYTES / 2**30:.0f} GiB bound"
                           if world == 1 else "one GPU only"}

    e2e = None
    if not args.no_e2e:
        q_host = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for q in qs]
        for qh, q in zip(q_host, qs):
            qh.copy_(q.cpu())
        o_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]

        def e2e_step():
            for qh, q in zip(q_host, qs):
                q.copy_(qh, non_blocking=True)
            decode_step()
            for oh, o in zip(o_host, outs):
                oh.copy_(o, non_blocking=True)

        esteps = max(3, args.steps // 4)
        ms_e2e = time_graph(e2e_step, esteps, args.warmup, stream, dist) / esteps
        h2d = sum(q.numel() * q.element_size() for q in qs)
        e2e = {"value": job_gbs(step_bytes, ms_e2e, world), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h2d, "ms_per_step": ms_e2e}

    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "heads": f"{wl.n_q_heads}/{wl.n_kv_heads}",
                   "ctx_len": L, "k": k, "n_dom": wl.n_dom, "layers_per_step": n_layers,
                   "parallelism": f"replicas{world}",
                   "l2": f"inputs larger than L2: {n_layers} layer caches "
                         f"({step_bytes / 2**20:.0f} MiB of roofline bytes per step) stepped in order"},
        "us_per_layer_step": us_layer,
        "us_per_layer_step_percentiles": us_dist,
        "tokens_per_s": world * wl.batch / (us_layer * 1e-6),
        "decode_roofline": {"achieved": gbs / world, "peak": hbm_peak, "unit": "GB/s",
                            "frac": gbs / world / hbm_peak, "bytes_per_layer_step": per_layer_bytes,
                            "peak_kind": peak_kind},
        "roofline": roof,
        "decode_plan": "fused" if fused else "staged",
        "clocks": clocks,
        # kernels of this library per layer (fasa_decode_launches): fused 1, or 2 with the split-K
        # attention; staged 4 (score, filter, finalize, attend); +1 when the attention is split
        # over several CTAs per row (the split merge)
        "gpu_launches": launches * n_layers * args.steps,
        "e2e": e2e,
    }
    line.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu:
        units = oracle_units(wl, min(4, wl.batch * wl.n_kv_heads))
        b1, t1, calls1 = oracle_time(wl, units, k, budget_s=args.cpu_seconds)
        ba, ta, callsa, cores = oracle_all_cores(wl, k, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": ba / ta / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{callsa} oracle decodes of one (sequence, KV head) of {wl.name} each in {ta:.1f} s, "
                      f"float64 numpy, one single-threaded process per host core ({cores})",
            "single_thread": {"value": b1 / t1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"{calls1} oracle decodes of one (sequence, KV head) of {wl.name} each, "
                                        f"cycling over {len(units)} prepared heads ({t1:.1f} s), 1 thread"}}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_calibrate(args, wl):
    """Offline FC calibration of one layer: its 65 score planes per calibration
    query, the agreement counts and the dominant sets, each stage timed from
    a CUDA graph with events. Algorithmic bytes: the layer's K cache and the
    calibration queries; the score planes are the implementation's own
    intermediate (written once, read once by the selection)."""
    import torch
    from rope_frequency_chunk_b200 import fasa as F
    torch.cuda.set_device(0)
    k = args.k or wl.k
    n_win = args.cal_win
    inp = W.layer_inputs(wl, layer=0)
    lp = inp.params
    cache = F.KVCache(wl.batch, wl.n_q_heads, wl.n_kv_heads, lp.dom_idx.shape[1], wl.ctx_len, wl.dtype,
                      wl.rope_base, lp.dom_idx)
    F.fasa_append_kv(cache, W.to_torch(inp.k, "cuda"), W.to_torch(inp.v, "cuda"), 0)
    G = wl.group
    sdt = np.float32 if wl.dtype == "f32" else np.uint16
    qw = np.empty((wl.batch, n_win, wl.n_q_heads, W.HEAD_DIM), sdt)
    for b in range(wl.batch):
        for w in range(n_win):
            for g in range(wl.n_kv_heads):
                qw[b, w, g * G:(g + 1) * G] = W.head_q(wl, lp, 0, b, g, step=100 + w)
    q_t = W.to_torch(qw, "cuda")
    L = wl.ctx_len
    rows = wl.batch * wl.n_kv_heads
    planes = torch.empty(wl.batch, wl.n_kv_heads, n_win, F.CAL_PLANES, L, dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.n_kv_heads, 64, dtype=torch.int32, device="cuda")
    dom = torch.empty(wl.n_kv_heads, wl.n_dom, dtype=torch.int32, device="cuda")
    sel_ws = torch.empty(rows * n_win * F.CAL_PLANES * min(k, L) * 4, dtype=torch.uint8, device="cuda")
    ws = torch.empty(F.fasa_calibrate_workspace_bytes(cache, L, n_win, k), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    stages = {
        "scores": lambda: F.fasa_calibrate_scores(cache, L, q_t, L, planes=planes, stream=stream),
        "counts": lambda: F.fasa_calibrate_counts(planes, wl.n_kv_heads, k, counts=counts, workspace=sel_ws,
                                                  stream=stream),
        "dominant": lambda: F.fasa_calibrate_dominant(counts, wl.n_dom, dom_idx=dom, stream=stream),
        "whole": lambda: F.fasa_calibrate(cache, L, q_t, L, k, wl.n_dom, counts=counts, dom_idx=dom,
                                          workspace=ws, stream=stream),
    }
    hbm_peak, peak_kind = peaks()
    with ClockSampler(0) as clk:
        ms = {name: time_graph(fn, args.steps, args.warmup, stream) / args.steps for name, fn in stages.items()}
    status = F.fasa_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed calibration")
    es = wl.elem_bytes
    alg = rows * L * W.HEAD_DIM * es + wl.batch * n_win * wl.n_q_heads * W.HEAD_DIM * es
    plane_bytes = rows * n_win * F.CAL_PLANES * L * 4
    scores_gbs = (rows * L * W.HEAD_DIM * es + plane_bytes) / (ms["scores"] * 1e-3) / 1e9
    line = {
        "metric": "fasa_calibrate ms per layer calibration (calibration queries x budget), algorithmic GB/s",
        "value": alg / (ms["whole"] * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms["whole"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name} calibration", "batch": wl.batch,
                   "heads": f"{wl.n_q_heads}/{wl.n_kv_heads}", "ctx_len": L, "budget": k, "n_win": n_win,
                   "n_dom": wl.n_dom, "parallelism": "single",
                   "l2": f"score planes of {plane_bytes / 2**20:.0f} MiB per step (larger than L2)"},
        "stage_ms": ms,
        "roofline": {"bound": "hbm", "kernel": "calib_score_kernel (65 score planes per query)",
                     "achieved": scores_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": scores_gbs / hbm_peak,
                     "traffic": None, "bytes_per_launch": rows * L * W.HEAD_DIM * es + plane_bytes,
                     "peak_kind": peak_kind, "us_per_launch": 1e3 * ms["scores"]},
        "algorithmic_bytes": alg, "plane_bytes": plane_bytes,
        "clocks": clk.summary(),
        # per whole calibration: the score kernel, the selection launches, overlap, rank
        "gpu_launches": (3 + -(-rows * n_win * F.CAL_PLANES // 65535)) * args.steps,
    }
    print(json.dumps(line))
    return 0


def run_sweep(args, wl):
    """The long-CoT sweep: for each dominant-set size, contexts grow from
    1K to 32K tokens in 1K appends (fasa_append_kv); after each append one
    decode at the new length with the 18.9% budget. Both are timed with
    events per step (median of `--sweep-reps` repetitions, L2 flushed before
    each by writing a buffer larger than L2; re-appending a chunk rewrites the
    same slots with the same values)."""
    import torch
    from rope_frequency_chunk_b200 import fasa as F
    torch.cuda.set_device(0)
    chunk, steps = W.C4_APPEND_CHUNK, W.C4_STEPS
    L_max = chunk * steps
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    reps = max(3, args.sweep_reps)
    result = {}
    hbm_peak, peak_kind = peaks()
    with ClockSampler(0) as clk:
        for n_dom in W.C4_NDOMS:
            w = wl.replace(ctx_len=L_max, n_dom=n_dom)
            inp = W.layer_inputs(w, layer=0, n_dom=n_dom)
            cache = F.KVCache(w.batch, w.n_q_heads, w.n_kv_heads, n_dom, L_max, w.dtype, w.rope_base,
                              inp.params.dom_idx)
            k_all = W.to_torch(inp.k, "cuda")
            v_all = W.to_torch(inp.v, "cuda")
            q = W.to_torch(inp.q, "cuda")
            out = torch.empty_like(q)
            ws = torch.zeros(F.fasa_decode_workspace_bytes(cache, L_max, W.c4_budget(L_max)), dtype=torch.uint8,
                             device="cuda")
            rows = []
            for st in range(steps):
                pos0, L = st * chunk, (st + 1) * chunk
                kn = k_all[:, :, pos0:L].contiguous()
                vn = v_all[:, :, pos0:L].contiguous()
                k = W.c4_budget(L)

                def timed(fn):
                    ts = []
                    for _ in range(reps):
                        flush.fill_(1.0)
                        e0 = torch.cuda.Event(enable_timing=True)
                        e1 = torch.cuda.Event(enable_timing=True)
                        e0.record()
                        fn()
                        e1.record()
                        torch.cuda.synchronize()
                        ts.append(e0.elapsed_time(e1) * 1e3)
                    return float(np.median(ts))

                t_app = timed(lambda: F.fasa_append_kv(cache, kn, vn, pos0))
                for _ in range(args.warmup):
                    F.fasa_decode(cache, L, q, L, k, out=out, workspace=ws)
                t_dec = timed(lambda: F.fasa_decode(cache, L, q, L, k, out=out, workspace=ws))
                alg = roofline_bytes(w.replace(ctx_len=L, k=k), k)
                rows.append({"L": L, "k": k, "append_us": t_app, "decode_us": t_dec,
                             "decode_gbs": alg / (t_dec * 1e-6) / 1e9,
                             "plan": int(F.fasa_decode_path(cache, L, k))})
            status = F.fasa_device_status(clear=True)
            if status != 0:
                raise RuntimeError(f"device status {status} in the sweep")
            result[str(n_dom)] = rows
            del cache, k_all, v_all, ws
    per_step = {nd: float(np.mean([r["append_us"] + r["decode_us"] for r in rows])) for nd, rows in result.items()}
    last = {nd: rows[-1] for nd, rows in result.items()}
    line = {
        "metric": "c4 long-CoT sweep: append + decode us per step (1K..32K in 1K appends), mean over steps",
        "value": per_step["16"], "unit": "us", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
        "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "c4 sweep", "batch": wl.batch, "heads": f"{wl.n_q_heads}/{wl.n_kv_heads}",
                   "n_dom": list(W.C4_NDOMS), "budget": "18.9% of L", "reps": reps,
                   "l2": "flushed before every timed call (a write of twice the L2 size)"},
        "mean_us_per_step": per_step,
        "at_32k": {nd: {"decode_us": r["decode_us"], "decode_gbs": r["decode_gbs"],
                        "frac": r["decode_gbs"] / hbm_peak, "append_us": r["append_us"], "plan": r["plan"]}
                   for nd, r in last.items()},
        "peak": hbm_peak, "peak_kind": peak_kind, "steps_detail": result, "clocks": clk.summary(),
    }
    print(json.dumps(line))
    return 0


def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fasa", choices=["fasa", "reference"])
    ap.add_argument("--config", default="c2", choices=sorted(W.CONFIGS))
    ap.add_argument("--layers", type=int, default=0)
    ap.add_argument("--k", type=int, default=0)
    ap.add_argument("--ctx-len", type=int, default=0)
    ap.add_argument("--n-dom", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--plan", default="auto", choices=["auto", "fused", "staged"],
                    help="launch plan of fasa_decode (default: the library's choice)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-fasa-m", action="store_true", help="skip the FASA-M (host-resident K/V) leg")
    ap.add_argument("--multi", type=lambda s: [int(x) for x in s.split(",") if x], default=[4, 8, 16],
                    help="query tokens per sequence of the multi-query legs (comma list; empty to skip)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--calibrate", action="store_true",
                    help="time the offline FC calibration on one layer of the workload instead of the decode")
    ap.add_argument("--cal-win", type=int, default=8, help="calibration queries per sequence (--calibrate)")
    ap.add_argument("--sweep", action="store_true",
                    help="the c4 long-CoT sweep: append + decode timed per step for every dominant-set size")
    ap.add_argument("--sweep-reps", type=int, default=5)
    return ap


def main(argv=None):
    args = build_parser().parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    wl = W.CONFIGS[args.config]
    if args.ctx_len:
        wl = wl.replace(ctx_len=args.ctx_len, k=W.c4_budget(args.ctx_len) if wl.name == "c4" else wl.k)
    if args.n_dom:
        wl = wl.replace(n_dom=args.n_dom)
    if args.batch:
        wl = wl.replace(batch=args.batch)
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.calibrate:
        return run_calibrate(args, wl)
    if args.sweep:
        return run_sweep(args, W.CONFIGS["c4"])
    return run_fasa(args, wl)


if __name__ == "__main__":
    sys.exit(main())
