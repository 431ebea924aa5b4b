#!/usr/bin/env python
"""Benchmark of one TSP rank step on B200: the rank projects its own K/V and
runs its layer forward (LN1, QKV, causal zigzag attention, O + residual, LN2,
W1 + GELU, W2 + residual) for the 7B dense layer at T = 131072, D = 8.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tsp|reference]

One process per GPU (torchrun for N > 1); every GPU runs TSP rank
(global rank mod D) on its own synthetic inputs: the per-rank work is
independent, so the job scales weakly and needs no collective on the data
path (the barrier and the max-over-ranks timing use NCCL).  Rank 0 prints one
JSON line.  `--impl reference` times the CPU oracle on host cores instead.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TSP layer fwd tokens/s on 1 B200 (7B layer, 128K, D=8); % bf16 tensor peak"
UNIT = "tokens/s"
WORKLOADS = {
    "7b-128k-d8": dict(T=131072, h=4096, H=32, F=16384, D=8, seed=2,
                       desc="7B dense layer (h=4096, 32 heads x 128, FFN 16384, GELU-tanh, pre-LN), "
                            "T=131072, D=8: one TSP rank step = own K/V projection + layer forward "
                            "over 16384 local tokens (2 zigzag chunks of 8192) against 131072 keys"),
    "7b-8k-d8": dict(T=8192, h=4096, H=32, F=16384, D=8, seed=1,
                     desc="7B dense layer, T=8192, D=8, one TSP rank step"),
    "7b-32k-d8": dict(T=32768, h=4096, H=32, F=16384, D=8, seed=4,
                      desc="7B dense layer, T=32768, D=8, one TSP rank step"),
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return m, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def rank_flops(T, h, F, D, rank):
    """Algorithmic FLOPs of one rank step (GEMMs + unmasked causal pairs)."""
    c = T // (2 * D)
    L = 2 * c
    pairs = c * c * (2 * D - 1) + c * (c + 1)          # sum over local tokens of (pos + 1)
    attn = 4 * h * pairs                               # QK^T and PV, all heads
    qkv = 2 * L * h * 3 * h
    o = 2 * L * h * h
    mlp = 2 * 2 * L * h * F
    return {"attention": attn, "qkv": qkv, "o": o, "mlp": mlp, "total": attn + qkv + o + mlp}


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- dist
def dist_setup(n_gpus):
    from folded_tensor_sequence_rank_b200 import dist as tdist
    world, rank, local = tdist.world_info()
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def traffic_record(kernel_file):
    """dram bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    with open(kernel_file, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if rec.get("source_sha") != sha:
        return None
    return rec


# ---------------------------------------------------------------------------- CPU oracle
# The oracle is timed as it stands.  Set-up that does not depend on which rows
# are computed happens once, outside the timed region: drawing the inputs,
# rounding the weights to the layer's fp16 storage (rounding is idempotent, so
# the oracle computes exactly what it would from the raw weights) and holding
# K/V in fp64 (what the oracle converts them to anyway).  What is timed is the
# oracle's per-token work: the tokens' K/V projection and their layer output
# against the full-sequence K/V.
ORACLE_MIN_ROWS = 32  # below this the fixed per-call reads of K/V and the weights dominate


def oracle_state(wl, cache={}):
    import numpy as np
    from folded_tensor_sequence_rank_b200 import inputs
    from oracle import tsp_oracle as O
    T, h, F, D = wl["T"], wl["h"], wl["F"], wl["D"]
    key = (T, h, F, D, wl["seed"])
    if key not in cache:
        cache.clear()
        raw = inputs.rank_inputs(T // D, T, h, F, wl["seed"])
        w = O.stored_weights({n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES})
        st = dict(x=raw["x_local"].double().numpy(), w=w, K=raw["k_full"].double().numpy(),
                  V=raw["v_full"].double().numpy(), pos=O.zigzag_index(T, D, 0))
        del raw
        cache[key] = st
    return cache[key]


def oracle_rows(wl, n_rows, seed=0):
    """Times the oracle on `n_rows` of rank 0's tokens, spread evenly over both
    zigzag chunks (the attention work per row grows with its position, so an
    even spread gives the rank's mean).  Returns (seconds, rows)."""
    import numpy as np
    from oracle import tsp_oracle as O
    st = oracle_state(wl)
    L = wl["T"] // wl["D"]
    c = L // 2
    half = max(1, n_rows // 2)
    offs = (np.arange(half) * c) // half + (seed % max(1, c // half))
    rows = np.concatenate([offs, c + offs])[:max(1, n_rows)]
    t0 = time.perf_counter()
    O.kv_project(st["x"][rows], st["w"])
    O.rank_rows_forward(st["x"][rows], st["pos"][rows], st["K"], st["V"], st["w"], wl["H"])
    return time.perf_counter() - t0, len(rows)


def oracle_full(name):
    """Times the oracle on a whole small configuration: the tiny layer (T=512,
    D=2: every rank, i.e. the unsharded layer over all 512 tokens) or one rank
    of the 7B layer at T=8192, D=8 (its 1024 tokens' K/V projection and layer
    output against stand-in K/V of all 8192 tokens).  Returns (seconds, tokens)."""
    import numpy as np
    from folded_tensor_sequence_rank_b200 import inputs
    from oracle import tsp_oracle as O
    if name == "tiny":
        raw = inputs.layer_inputs(512, 256, 1024, 0)
        x = raw["x"].double().numpy()
        w = O.stored_weights({n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES})
        t0 = time.perf_counter()
        O.layer_forward(x, w, 4)
        return time.perf_counter() - t0, 512
    T, h, F, D, H = 8192, 4096, 16384, 8, 32
    raw = inputs.rank_inputs(T // D, T, h, F, 1)
    x = raw["x_local"].double().numpy()
    w = O.stored_weights({n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES})
    K, V = raw["k_full"].double().numpy(), raw["v_full"].double().numpy()
    pos = O.zigzag_index(T, D, 0)
    t0 = time.perf_counter()
    O.kv_project(x, w)
    O.rank_rows_forward(x, pos, K, V, w, H)
    return time.perf_counter() - t0, T // D


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def one_thread():
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1, user_api="blas")


def sample_rows_for(wl, budget_s):
    """Rows per oracle sample for about `budget_s` seconds of CPU work (at least
    ORACLE_MIN_ROWS, even)."""
    oracle_rows(wl, 2)                                   # untimed: first touch of the inputs
    dt, n = oracle_rows(wl, ORACLE_MIN_ROWS, seed=1)
    rows = max(ORACLE_MIN_ROWS, int(ORACLE_MIN_ROWS * budget_s / max(dt, 1e-3)))
    return rows - rows % 2, dt


def cpu_baseline(wl, budget_s=15.0):
    rows, _ = sample_rows_for(wl, budget_s)
    rows = min(rows, 256)
    dt, n = oracle_rows(wl, rows, seed=2)
    with one_thread():
        dt1, n1 = oracle_rows(wl, ORACLE_MIN_ROWS, seed=3)
    full = {}
    for name, label in (("tiny", "tiny layer h=256, T=512, D=2: every rank (the whole unsharded layer)"),
                        ("7b-8k", "7B layer, T=8192, D=8: rank 0 in full (1024 tokens: K/V projection + layer)")):
        t, tok = oracle_full(name)
        with one_thread():
            t1, _ = oracle_full(name)
        full[name] = {"workload": label, "tokens_per_s": tok / t, "tokens_per_s_1_thread": tok / t1,
                      "seconds": round(t, 3), "seconds_1_thread": round(t1, 3)}
    return {"value": n / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "extrapolated": True,
            "sample": f"{n} of rank 0's {wl['T'] // wl['D']} tokens (half in each zigzag chunk, evenly spaced): "
                      f"their K/V projection and layer output in fp64 numpy against the full {wl['T']}-token K/V, "
                      f"{dt:.1f} s; the rank's tokens/s is extrapolated from this per-token rate",
            "threads_1": {"value": n1 / dt1, "unit": UNIT, "cores": 1,
                          "sample": f"{n1} tokens, the same way, with BLAS limited to one thread"},
            "full_configs": full}


def run_reference(args, wl):
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows, _ = sample_rows_for(wl, budget)
    for i in range(args.warmup):
        oracle_rows(wl, rows, seed=10 + i)
    tot_t, tot_n = 0.0, 0
    for i in range(args.steps):
        dt, n = oracle_rows(wl, rows, seed=100 + i)
        tot_t += dt
        tot_n += n
    value = tot_n / tot_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl["desc"], "T": wl["T"], "D": wl["D"], "rank": 0},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "extrapolated": True,
                             "sample": f"{rows} of rank 0's tokens per step (half per zigzag chunk): K/V projection "
                                       f"and layer output in fp64 numpy; weights rounded and K/V held in fp64 once, "
                                       f"before the timed steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- GPU arm
def run_tsp(args, wl):
    import gc

    import torch
    line, world = measure_tsp(args, wl)
    if line is None:
        return
    if world == 1 and not args.no_extras:
        # the other configurations, measured in the same run on the same GPU
        gc.collect()
        torch.cuda.empty_cache()
        line["other_configs"] = other_configs(args)
    print(json.dumps(line), flush=True)


def other_configs(args):
    """Configurations 3 and 4, the layer's backward and the 32-layer stack,
    each measured by its sweep (see run_sweep_*), kept in compact form."""
    import gc

    import torch
    out = {}
    keep = {"ranks": ("config3_all_8_ranks_128k", ["value", "unit", "layer_spread", "kv_project_ms",
                                                   "layer_forward_ms", "clocks"]),
            "shards": ("config4_shard_sweep_32k", ["by_D"]),
            "layer_bwd": ("layer_backward_128k_rank0", ["value", "unit", "ms_per_step", "tflops", "roofline",
                                                       "part_ms", "clocks"]),
            "stack": ("stack_32_layers_128k", ["value", "unit", "ms_per_step", "ms_per_layer",
                                               "peak_device_bytes_this_run", "per_gpu_bytes_on_8_gpus", "clocks"])}
    fns = {"ranks": run_sweep_ranks, "shards": run_sweep_shards, "layer_bwd": run_sweep_layer_bwd,
           "stack": run_sweep_stack}
    for k, (name, fields) in keep.items():
        sub = argparse.Namespace(**vars(args))
        sub.workload = "7b-128k-d8"
        r = fns[k](sub)
        out[name] = {"metric": r["metric"], **{f: r[f] for f in fields if f in r}}
        gc.collect()
        torch.cuda.empty_cache()
    return out


def measure_tsp(args, wl):
    import torch
    import torch.distributed as dist

    from folded_tensor_sequence_rank_b200 import dist as tdist
    from folded_tensor_sequence_rank_b200 import tsp

    world, grank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    T, h, H, F, D = wl["T"], wl["h"], wl["H"], wl["F"], wl["D"]
    trank = tdist.tsp_rank_for(grank, D)
    L = T // D
    dims = tsp.make_dims(T, h, H, F)
    tsp.lib()

    # synthetic inputs, drawn on the device (parity is the tests' job)
    g = torch.Generator(device="cuda")
    g.manual_seed(wl["seed"] * 1000 + grank)
    def rnd(*shape, std=1.0, dtype=torch.bfloat16):
        return (torch.randn(*shape, generator=g, device="cuda", dtype=torch.float32) * std).to(dtype)
    w_full = {"wq": rnd(h, h, std=0.02), "wk": rnd(h, h, std=0.02), "wv": rnd(h, h, std=0.02),
              "wo": rnd(h, h, std=0.02), "w1": rnd(h, F, std=0.02), "w2": rnd(F, h, std=0.02)}
    sw = tsp.pack_shards(dims, D, w_full)
    del w_full
    kv_std = 0.02 * math.sqrt(h)
    x_local = rnd(L, h)
    K = rnd(T, h, std=kv_std, dtype=torch.float16)
    V = rnd(T, h, std=kv_std, dtype=torch.float16)
    y = torch.empty(L, h, dtype=torch.bfloat16, device="cuda")
    ws = tsp.alloc_workspace(dims, D)
    stream = torch.cuda.current_stream()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(tsp.N_STEP_EVENTS)] for _ in range(args.steps)]

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        tsp.rank_step(dims, sw, trank, x_local, K, V, y, ws)
    torch.cuda.synchronize()
    assert tsp.get_device_status(ws) == tsp.TSP_OK, "device wait timed out during warm-up"

    # --- device-timed steps, inputs resident in HBM
    step_ms = {k: 0.0 for k in ("ln1", "qkv", "attention", "o", "ln2", "w1", "w2")}
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    per_step = []
    for i in range(args.steps):
        tsp.rank_step(dims, sw, trank, x_local, K, V, y, ws, events=evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms = t0.elapsed_time(t1) / args.steps
    names = list(step_ms)
    for ev in evs:
        for j, n in enumerate(names):
            step_ms[n] += ev[j].elapsed_time(ev[j + 1]) / args.steps
    kern_ms = sum(step_ms.values())

    # --- end to end: host (pinned) tokens in, host result out, through the C ABI.
    # Consecutive steps alternate between two streams ("lanes"), each with its
    # own staging buffers, workspace and K/V, so the copy engines move one
    # step's tokens while the SMs compute the other's; every step still does
    # its own host->device and device->host copy.  Each step's kernels wait for
    # the previous step's (the call's compute_after / compute_done events), so
    # the two lanes' kernels never share the SMs.
    lanes = []
    for li in range(2):
        lanes.append(dict(stream=torch.cuda.Stream(), hx=x_local.cpu().pin_memory(),
                          hy=torch.empty(L, h, dtype=torch.bfloat16).pin_memory(),
                          xs=torch.empty_like(x_local), ys=torch.empty_like(y),
                          ws=ws if li == 0 else tsp.alloc_workspace(dims, D),
                          K=K if li == 0 else K.clone(), V=V if li == 0 else V.clone()))
    torch.cuda.synchronize()

    done = [torch.cuda.Event(), torch.cuda.Event()]
    n_host = [0]

    def host_step(ln):
        i = n_host[0]
        n_host[0] += 1
        with torch.cuda.stream(ln["stream"]):
            tsp.rank_step_host(dims, sw, trank, ln["hx"], ln["xs"], ln["K"], ln["V"], ln["ys"], ln["hy"], ln["ws"],
                               stream=ln["stream"], compute_after=done[(i - 1) % 2] if i > 0 else None,
                               compute_done=done[i % 2])
    for i in range(4):
        host_step(lanes[i % 2])
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for ln in lanes:
        ln["stream"].wait_event(e0)
    for i in range(args.steps):
        host_step(lanes[i % 2])
    for ln in lanes:
        stream.wait_stream(ln["stream"])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    for ln in lanes:
        assert tsp.get_device_status(ln["ws"]) == tsp.TSP_OK, "device wait timed out"

    ms, e2e_ms, attn_ms = tdist.max_over_ranks([ms, e2e_ms, step_ms["attention"]], device="cuda")

    if grank == 0:
        pk, src = peaks()
        fl = rank_flops(T, h, F, D, trank)
        peak_tf = pk["bf16_tflops_sustained"]
        attn_tf = fl["attention"] / (attn_ms * 1e-3) / 1e12
        traf = traffic_record(os.path.join(ROOT, "folded_tensor_sequence_rank_b200", "csrc", "attn_sm100.cuh"))
        value = world * L / (ms * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
            "config": {"workload": wl["desc"], "T": T, "D": D, "tsp_rank": trank, "local_tokens": L,
                       "parallelism": f"{world} GPU(s), each an independent TSP rank (rank = gpu mod {D})",
                       "l2": "inputs larger than L2 (K/V 2 x 1 GiB, weights 384 MiB); no flush"},
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_tcgen05<128>", "achieved": attn_tf,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": attn_tf / peak_tf,
                         "peak_source": f"{src} bf16_tflops_sustained (kernel timed inside a long step)",
                         "algorithmic_per_launch": f"{fl['attention']:.4e} FLOP = 4 h x causal pairs",
                         "traffic": (traf["bytes_per_launch"] if traf else None)},
            "step_tflops": fl["total"] / (ms * 1e-3) / 1e12,
            "step_frac_of_peak": fl["total"] / (ms * 1e-3) / 1e12 / peak_tf,
            "kernel_ms": {k: round(v, 4) for k, v in step_ms.items()},
            "kernel_ms_sum": kern_ms,
            "gpu_launches": 7 * args.steps,
            "e2e": {"value": world * L / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": L * h * 2,
                    "d2h_bytes_per_step": L * h * 2},
            "clocks": clk,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(wl)
    else:
        line = None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line, world


STEP_NAMES = ("ln1", "qkv", "attention", "o", "ln2", "w1", "w2")


def _synthetic(T, h, F, seed, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def rnd(*shape, std=1.0, dtype=torch.bfloat16):
        return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)
    w = {"wq": rnd(h, h, std=0.02), "wk": rnd(h, h, std=0.02), "wv": rnd(h, h, std=0.02),
         "wo": rnd(h, h, std=0.02), "w1": rnd(h, F, std=0.02), "w2": rnd(F, h, std=0.02)}
    return rnd, w


def run_sweep_ranks(args):
    """All D = 8 ranks of the 128K layer back to back on one GPU (seed 3): the
    K/V projection of every rank's tokens (what the all-gather assembles), then
    every rank's layer forward.  Reports whole-layer tokens/s = T / (sum of all
    projection and layer times) and the spread of the per-rank layer times,
    (max - min) / mean, which the zigzag partition makes ~0."""
    import torch
    from folded_tensor_sequence_rank_b200 import tsp
    T, h, H, F, D = 131072, 4096, 32, 16384, 8
    L = T // D
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, 3)
    sw = tsp.pack_shards(dims, D, w_full)
    del w_full
    x = rnd(T, h)
    xs = [x.index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    del x
    K = torch.empty(T, h, dtype=torch.float16, device="cuda")
    V = torch.empty_like(K)
    ys = [torch.empty(L, h, dtype=torch.bfloat16, device="cuda") for _ in range(D)]
    ws = tsp.alloc_workspace(dims, D)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def one_layer(record):
        kv_ev = [ev() for _ in range(D + 1)] if record else None
        fw_ev = [ev() for _ in range(D + 1)] if record else None
        s = torch.cuda.current_stream()
        if record:
            kv_ev[0].record(s)
        for r in range(D):
            tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
            if record:
                kv_ev[r + 1].record(s)
        if record:
            fw_ev[0].record(s)
        for r in range(D):
            tsp.layer_forward(dims, sw, r, xs[r], K, V, ys[r], ws)
            if record:
                fw_ev[r + 1].record(s)
        return kv_ev, fw_ev

    for _ in range(args.warmup):
        one_layer(False)
    torch.cuda.synchronize()
    assert tsp.get_device_status(ws) == tsp.TSP_OK, "device wait timed out during warm-up"
    steps = max(1, min(args.steps, 5))
    clocks = ClockSampler(0)
    time.sleep(0.3)
    recs = [one_layer(True) for _ in range(steps)]
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert tsp.get_device_status(ws) == tsp.TSP_OK, "device wait timed out"
    kv_ms = [statistics.median(k[r].elapsed_time(k[r + 1]) for k, _ in recs) for r in range(D)]
    fw_ms = [statistics.median(f[r].elapsed_time(f[r + 1]) for _, f in recs) for r in range(D)]
    total = sum(kv_ms) + sum(fw_ms)
    mean = statistics.mean(fw_ms)
    line = {"metric": "TSP whole-layer fwd tokens/s, all 8 ranks back to back on 1 B200 (7B layer, 128K, D=8)",
            "value": T / (total * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "ms_per_step": total, "higher_is_better": True, "dtype": "fp16", "data": "synthetic",
            "config": {"workload": "7B dense layer, T=131072, D=8, every rank in turn (seed 3)",
                       "l2": "inputs larger than L2; no flush"},
            "kv_project_ms": [round(t, 4) for t in kv_ms], "layer_forward_ms": [round(t, 4) for t in fw_ms],
            "layer_spread": (max(fw_ms) - min(fw_ms)) / mean, "clocks": clk}
    return line


def run_sweep_shards(args):
    """Rank 0 of the 7B layer at T = 32768 for D = 1, 2, 4, 8, 16 (seed 4):
    per-kernel times and rates as the shards shrink (h/D Q columns, F/D FFN
    columns per shard)."""
    import torch
    from folded_tensor_sequence_rank_b200 import tsp
    T, h, H, F = 32768, 4096, 32, 16384
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, 4)
    kv_std = 0.02 * math.sqrt(h)
    K = rnd(T, h, std=kv_std, dtype=torch.float16)
    V = rnd(T, h, std=kv_std, dtype=torch.float16)
    out = {}
    steps = max(1, min(args.steps, 10))
    for D in (1, 2, 4, 8, 16):
        L = T // D
        sw = tsp.pack_shards(dims, D, w_full)
        x = rnd(L, h)
        y = torch.empty(L, h, dtype=torch.bfloat16, device="cuda")
        ws = tsp.alloc_workspace(dims, D)
        for _ in range(args.warmup):
            tsp.rank_step(dims, sw, 0, x, K, V, y, ws)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(tsp.N_STEP_EVENTS)] for _ in range(steps)]
        for i in range(steps):
            tsp.rank_step(dims, sw, 0, x, K, V, y, ws, events=evs[i])
        torch.cuda.synchronize()
        assert tsp.get_device_status(ws) == tsp.TSP_OK, "device wait timed out"
        ms = {n: statistics.median(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(STEP_NAMES)}
        fl = rank_flops(T, h, F, D, 0)
        step = sum(ms.values())
        out[str(D)] = {"tokens_per_s": L / (step * 1e-3), "step_ms": round(step, 4),
                       "kernel_ms": {k: round(v, 4) for k, v in ms.items()},
                       "tflops": {"attention": fl["attention"] / (ms["attention"] * 1e-3) / 1e12,
                                  "qkv": fl["qkv"] / (ms["qkv"] * 1e-3) / 1e12,
                                  "o": fl["o"] / (ms["o"] * 1e-3) / 1e12,
                                  "w1": fl["mlp"] / 2 / (ms["w1"] * 1e-3) / 1e12,
                                  "w2": fl["mlp"] / 2 / (ms["w2"] * 1e-3) / 1e12}}
        del sw, x, y, ws
        torch.cuda.empty_cache()
    line = {"metric": "TSP rank-0 layer fwd tokens/s vs shard count D on 1 B200 (7B layer, 32K)",
            "value": out["8"]["tokens_per_s"], "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "fp16", "data": "synthetic",
            "config": {"workload": "7B dense layer, T=32768, rank 0, D in {1,2,4,8,16} (seed 4); value is D=8"},
            "by_D": out}
    return line


BWD_NAMES = ["ln2_u", "du", "dxn2", "ln2_bwd", "transposes", "dw1", "dw2"]


def run_sweep_mlp_bwd(args):
    """Backward of the MLP half for rank 0 of the 7B layer (T and D from
    --workload; 128K, D = 8 by default: 16384 tokens, seed 5): dY1, dW1, dW2
    from Y1 and dY.  tokens/s =
    L / backward time; the five matmuls (U recomputed, dU, dXn2, dW1, dW2)
    are 2 L h F FLOPs each."""
    import torch
    from folded_tensor_sequence_rank_b200 import tsp
    wl = WORKLOADS[args.workload]
    T, h, H, F, D = wl["T"], wl["h"], wl["H"], wl["F"], wl["D"]
    L = T // D
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, 5)
    sw = tsp.pack_shards(dims, D, w_full)
    y1 = rnd(L, h, dtype=torch.float32)
    dy = rnd(L, h)
    dy1 = torch.empty(L, h, dtype=torch.float32, device="cuda")
    dw1 = torch.empty(h, F, dtype=torch.float32, device="cuda")
    dw2 = torch.empty(F, h, dtype=torch.float32, device="cuda")
    bws = tsp.alloc_mlp_backward_workspace(dims, D)
    for _ in range(args.warmup):
        tsp.mlp_backward(dims, sw, w_full["w1"], w_full["w2"], y1, dy, dy1, dw1, dw2, bws)
    steps = max(1, min(args.steps, 20))
    clocks = ClockSampler(0)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(tsp.N_STEP_EVENTS)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        tsp.mlp_backward(dims, sw, w_full["w1"], w_full["w2"], y1, dy, dy1, dw1, dw2, bws, events=evs[i])
    t1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert tsp.get_device_status(bws) == tsp.TSP_OK, "device wait timed out"
    ms = t0.elapsed_time(t1) / steps
    part = {n: statistics.median(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(BWD_NAMES)}
    gf = 2.0 * L * h * F
    rate = {n: gf / (part[n] * 1e-3) / 1e12 for n in ("du", "dxn2", "dw1", "dw2")}
    line = {"metric": f"TSP MLP-half backward tokens/s on 1 B200 (7B layer, T={T}, D={D}, rank 0)",
            "value": L / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"MLP half of the 7B layer, backward (dY1, dW1, dW2), T={T}, D={D}, rank 0: "
                                   f"{L} tokens, Y1 ~ N(0,1) fp32, dY ~ N(0,1) bf16 (seed 5)",
                       "l2": "inputs larger than L2; no flush"},
            "tflop_per_step": 5 * gf / 1e12, "tflops": 5 * gf / (ms * 1e-3) / 1e12,
            "part_ms": {k: round(v, 4) for k, v in part.items()},
            "gemm_tflops": {k: round(v, 1) for k, v in rate.items()},
            "clocks": clk}
    return line


LBWD_NAMES = ["mlp_half", "d_a", "d_wo", "attention", "prep_dq_ln1", "d_wq", "d_x"]


def run_sweep_layer_bwd(args):
    """The whole layer's backward for rank 0 (T and D from --workload; 128K,
    D = 8 by default): the rank's forward (tsp_rank_step, which stashes Q, A,
    Y1 and the attention's log-sum-exp), then tsp_layer_backward (MLP half,
    dA, dWo, the attention backward, dWq, dX) and tsp_kv_backward (the key
    owner's dWk, dWv and dX terms).  Only the backward is timed.  The
    attention backward's algorithmic work is five products per causal
    (query, key) pair and head dim (S, dP, dV, dK, dQ): 10 h pairs FLOPs."""
    import torch
    from folded_tensor_sequence_rank_b200 import tsp
    wl = WORKLOADS[args.workload]
    T, h, H, F, D = wl["T"], wl["h"], wl["H"], wl["F"], wl["D"]
    L = T // D
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, 6)
    sw = tsp.pack_shards(dims, D, w_full)
    kv_std = 0.02 * math.sqrt(h)
    x = rnd(L, h)
    K = rnd(T, h, std=kv_std, dtype=torch.float16)
    V = rnd(T, h, std=kv_std, dtype=torch.float16)
    y = torch.empty(L, h, dtype=torch.bfloat16, device="cuda")
    ws = tsp.alloc_workspace(dims, D)
    tsp.rank_step(dims, sw, 0, x, K, V, y, ws)
    dy = rnd(L, h)
    dx = torch.empty(L, h, dtype=torch.float32, device="cuda")
    g = {"wq": torch.empty(h, h, device="cuda"), "wo": torch.empty(h, h, device="cuda"),
         "w1": torch.empty(h, F, device="cuda"), "w2": torch.empty(F, h, device="cuda")}
    dwk = torch.empty(h, h, device="cuda")
    dwv = torch.empty(h, h, device="cuda")
    dK = torch.zeros(T, h, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    bws = tsp.alloc_layer_backward_workspace(dims, D)
    kws = tsp.alloc_kv_backward_workspace(dims, D)

    def step(events=None, kv_ev=None):
        tsp.layer_backward(dims, sw, w_full, 0, x, ws, K, V, dy, dx, g, dK, dV, bws, events=events)
        tsp.kv_backward(dims, D, w_full, 0, x, dK, dV, dx, dwk, dwv, kws)
        if kv_ev is not None:
            kv_ev.record()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert tsp.get_device_status(bws) == tsp.TSP_OK, "device wait timed out during warm-up"
    steps = max(1, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(tsp.N_STEP_EVENTS)] for _ in range(steps)]
    kvs = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    clocks = ClockSampler(0)
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        step(evs[i], kvs[i])
    t1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert tsp.get_device_status(bws) == tsp.TSP_OK and tsp.get_device_status(kws) == tsp.TSP_OK
    ms = t0.elapsed_time(t1) / steps
    part = {n: statistics.median(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(LBWD_NAMES)}
    part["kv_backward"] = statistics.median(evs[i][7].elapsed_time(kvs[i]) for i in range(steps))
    fl = rank_flops(T, h, F, D, 0)
    attn_bwd_fl = 2.5 * fl["attention"]
    gemm_fl = 5 * 2.0 * L * h * F + 4 * 2.0 * L * h * h + 4 * 2.0 * L * h * h  # MLP; dA, dWo, dWq, dXn1; kv: dWk, dWv, dXn (2h)
    pk, src = peaks()
    attn_tf = attn_bwd_fl / (part["attention"] * 1e-3) / 1e12
    line = {"metric": f"TSP layer backward tokens/s on 1 B200 (7B layer, T={T}, D={D}, rank 0)",
            "value": L / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "fp16/bf16", "data": "synthetic",
            "config": {"workload": f"backward of one TSP rank of the 7B layer, T={T}, D={D}, rank 0: {L} tokens; "
                                   f"layer backward + key-owner K/V backward (seed 6)",
                       "l2": "inputs larger than L2; no flush"},
            "tflop_per_step": (attn_bwd_fl + gemm_fl) / 1e12,
            "tflops": (attn_bwd_fl + gemm_fl) / (ms * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "attn_bwd_tcgen05<128>", "achieved": attn_tf,
                         "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": attn_tf / pk["bf16_tflops_sustained"],
                         "peak_source": f"{src} bf16_tflops_sustained",
                         "algorithmic_per_launch": f"{attn_bwd_fl:.4e} FLOP = 10 h x causal pairs"},
            "part_ms": {k: round(v, 4) for k, v in part.items()}, "clocks": clk}
    return line


def run_sweep_tp(args):
    """The tensor-parallel baseline beside TSP at the 7B layer, T = 131072,
    D = 8 (seed 7), on one GPU.  Measured: one TP rank's compute (its
    attention and MLP partials over all T tokens with 1/D of the weights), the
    two all-reduces as sums of the D partials in device memory (the whole
    job's reduction arithmetic and HBM traffic, not NVLink), and one TSP rank
    step (the bench's own step) on the same shards.  The all-reduce's
    communication on 8 GPUs is estimated, not measured: a ring all-reduce
    moves 2 (D-1)/D of the [T, h] bf16 tensor per rank, at the 725 GB/s bus
    bandwidth measured on this machine for an 8-rank all-reduce of 1 GiB."""
    import torch
    from folded_tensor_sequence_rank_b200 import stack, tp, tsp
    T, h, H, F, D = 131072, 4096, 32, 16384, 8
    L = T // D
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, 7)
    sw = tsp.pack_shards(dims, D, w_full)
    del w_full
    x = rnd(T, h)
    tws = tsp.alloc_tp_workspace(dims, D)
    parts = [torch.empty(T, h, dtype=torch.float32, device="cuda") for _ in range(D)]
    y1 = torch.empty(T, h, dtype=torch.float32, device="cuda")
    y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    # the TSP rank step on the same shards
    kv_std = 0.02 * math.sqrt(h)
    K = rnd(T, h, std=kv_std, dtype=torch.float16)
    V = rnd(T, h, std=kv_std, dtype=torch.float16)
    xl = rnd(L, h)
    yl = torch.empty(L, h, dtype=torch.bfloat16, device="cuda")
    ws = tsp.alloc_workspace(dims, D)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def tp_rank(k):
        tsp.tp_attention_partial(dims, sw, k, x, parts[k], tws)
        tsp.tp_mlp_partial(dims, sw, k, y1, parts[k], tws)
    for _ in range(args.warmup):
        tp_rank(0)
        tsp.tp_all_reduce(dims, parts, x, y1)
        tsp.tp_all_reduce(dims, parts, y1, y)
        tsp.rank_step(dims, sw, 0, xl, K, V, yl, ws)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    clocks = ClockSampler(0)
    time.sleep(0.3)
    rec = {"tp_rank": [], "all_reduce_x2": [], "tsp_rank": []}
    for _ in range(steps):
        e = [ev() for _ in range(4)]
        e[0].record()
        tp_rank(0)
        e[1].record()
        tsp.tp_all_reduce(dims, parts, x, y1)
        tsp.tp_all_reduce(dims, parts, y1, y)
        e[2].record()
        tsp.rank_step(dims, sw, 0, xl, K, V, yl, ws)
        e[3].record()
        torch.cuda.synchronize()
        rec["tp_rank"].append(e[0].elapsed_time(e[1]))
        rec["all_reduce_x2"].append(e[1].elapsed_time(e[2]))
        rec["tsp_rank"].append(e[2].elapsed_time(e[3]))
    clk = clocks.stop()
    assert tsp.get_device_status(tws) == tsp.TSP_OK and tsp.get_device_status(ws) == tsp.TSP_OK
    ms = {k: statistics.median(v) for k, v in rec.items()}
    comm_ms = 2 * (2 * (D - 1) / D * T * h * 2) / 725e9 * 1e3   # two ring all-reduces of bf16 [T, h]
    tsp_acc = stack.memory_account(dims, D, 1)
    tp_acc = tp.memory_account(dims, D)
    line = {"metric": "TP baseline vs TSP, one layer's forward, per GPU (7B layer, 128K, D=8)",
            "value": ms["tp_rank"] / ms["tsp_rank"], "unit": "TP rank compute time / TSP rank step time",
            "n_gpus": 1, "steps": steps, "warmup": args.warmup, "higher_is_better": False, "dtype": "fp16",
            "data": "synthetic",
            "config": {"workload": "7B dense layer, T=131072, D=8, rank 0 of each scheme, the same shards (seed 7)"},
            "ms": {k: round(v, 4) for k, v in ms.items()},
            "tp_all_reduce_comm_ms_estimated": round(comm_ms, 3),
            "tp_step_ms_with_estimated_comm": round(ms["tp_rank"] + comm_ms, 3),
            "tokens_per_s_whole_layer": {"tsp": T / (ms["tsp_rank"] * 1e-3),
                                         "tp_compute_only": T / (ms["tp_rank"] * 1e-3),
                                         "tp_with_estimated_comm": T / ((ms["tp_rank"] + comm_ms) * 1e-3)},
            "memory_per_gpu_bytes": {"tsp_one_layer": tsp_acc, "tp_one_layer": tp_acc},
            "clocks": clk}
    return line


def _attn_lib_impls(q, a, d_o, K, V, c, kv_len, H, hd, scale, which):
    """Library attention kernels on the rank's two requests (chunk r against
    keys [0, c) and chunk 2D-1-r against keys [0, (2D-r) c), bottom-right
    causal masks), as {name: (forward fn, backward fn or None, info)}.  A
    library that is missing or refuses the shape is reported, not fatal."""
    import torch
    L, h = q.shape
    out = {}

    def bhsd(t, S):  # [S, h] row-major -> [1, H, S, hd]
        return t.view(1, S, H, hd).permute(0, 2, 1, 3)

    def new_bhsd(S):
        return torch.empty(1, S, H, hd, dtype=torch.float16, device="cuda").permute(0, 2, 1, 3)

    if "cudnn" in which:
        try:
            import cudnn
            handle = cudnn.create_handle()
            cudnn.set_stream(handle=handle, stream=torch.cuda.current_stream().cuda_stream)
            DT = cudnn.data_type

            def built(g):
                g.validate()
                g.build_operation_graph()
                g.create_execution_plans([cudnn.heur_mode.A, cudnn.heur_mode.FALLBACK])
                g.check_support()
                g.build_plans()
                return torch.empty(max(g.get_workspace_size(), 1), dtype=torch.uint8, device="cuda")

            def graph():
                return cudnn.pygraph(io_data_type=DT.HALF, intermediate_data_type=DT.FLOAT,
                                     compute_data_type=DT.FLOAT, handle=handle)
            fwd, bwd, outs = [], [], []
            for q0, skv in ((0, kv_len[0]), (c, kv_len[1])):
                qt, kt, vt = bhsd(q[q0:q0 + c], c), bhsd(K[:skv], skv), bhsd(V[:skv], skv)
                ot, st = new_bhsd(c), torch.empty(1, H, c, 1, dtype=torch.float32, device="cuda")
                g = graph()
                tq, tk, tv = g.tensor_like(qt), g.tensor_like(kt), g.tensor_like(vt)
                to, tst = g.sdpa(name="sdpa", q=tq, k=tk, v=tv, generate_stats=True, attn_scale=scale,
                                 use_causal_mask_bottom_right=True)
                to.set_output(True).set_dim(list(ot.shape)).set_stride(list(ot.stride()))
                tst.set_output(True).set_data_type(DT.FLOAT).set_dim(list(st.shape)).set_stride(list(st.stride()))
                fwd.append((g, {tq: qt, tk: kt, tv: vt, to: ot, tst: st}, built(g)))
                outs.append(ot)
                dot = bhsd(d_o[q0:q0 + c], c)
                dqt, dkt, dvt = new_bhsd(c), new_bhsd(skv), new_bhsd(skv)
                g = graph()
                tq, tk, tv, to, tdo, tst = (g.tensor_like(x) for x in (qt, kt, vt, ot, dot, st))
                tdq, tdk, tdv = g.sdpa_backward(name="sdpa_backward", q=tq, k=tk, v=tv, o=to, dO=tdo, stats=tst,
                                                attn_scale=scale, use_causal_mask_bottom_right=True)
                for t, x in ((tdq, dqt), (tdk, dkt), (tdv, dvt)):
                    t.set_output(True).set_dim(list(x.shape)).set_stride(list(x.stride()))
                bwd.append((g, {tq: qt, tk: kt, tv: vt, to: ot, tdo: dot, tst: st, tdq: dqt, tdk: dkt, tdv: dvt},
                            built(g)))

            def run(gs):
                for g, m, w in gs:
                    g.execute(m, w, handle=handle)
            out["cudnn"] = (lambda: run(fwd), lambda: run(bwd),
                            {"version": cudnn.backend_version(),
                             "o": lambda: torch.cat([x.permute(0, 2, 1, 3).reshape(c, h) for x in outs])})
        except Exception as ex:  # noqa: BLE001 - report any library refusal
            out["cudnn"] = (None, None, {"error": repr(ex)[:300]})
    kcat = vcat = None
    if "fa2" in which or "flashinfer" in which:
        kcat = torch.cat([K[:kv_len[0]], K[:kv_len[1]]]).view(-1, H, hd)
        vcat = torch.cat([V[:kv_len[0]], V[:kv_len[1]]]).view(-1, H, hd)
    if "fa2" in which:
        try:
            from flash_attn import flash_attn_varlen_func
            cu_q = torch.tensor([0, c, 2 * c], dtype=torch.int32, device="cuda")
            cu_k = torch.tensor([0, kv_len[0], kv_len[0] + kv_len[1]], dtype=torch.int32, device="cuda")

            def fa(qq, kk, vv):
                return flash_attn_varlen_func(qq, kk, vv, cu_q, cu_k, c, kv_len[1], softmax_scale=scale, causal=True)
            qg, kg, vg = (x.detach().clone().requires_grad_() for x in (q.view(L, H, hd), kcat, vcat))
            o_g = fa(qg, kg, vg)

            def fb():
                qg.grad = kg.grad = vg.grad = None
                o_g.backward(d_o.view(L, H, hd), retain_graph=True)
            out["fa2"] = (lambda: fa(q.view(L, H, hd), kcat, vcat), fb,
                          {"o": lambda: fa(q.view(L, H, hd), kcat, vcat).reshape(L, h)})
        except Exception as ex:  # noqa: BLE001
            out["fa2"] = (None, None, {"error": repr(ex)[:300]})
    if "flashinfer" in which:
        try:
            import flashinfer
            qo = torch.tensor([0, c, 2 * c], dtype=torch.int32, device="cuda")
            kvp = torch.tensor([0, kv_len[0], kv_len[0] + kv_len[1]], dtype=torch.int32, device="cuda")
            wsb = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
            wr = flashinfer.BatchPrefillWithRaggedKVCacheWrapper(wsb, kv_layout="NHD", backend="cute-dsl")
            wr.plan(qo, kvp, H, H, hd, causal=True, sm_scale=scale, q_data_type=torch.float16)
            o_f = wr.run(q.view(L, H, hd), kcat, vcat)
            out["flashinfer_cute_dsl"] = (lambda: wr.run(q.view(L, H, hd), kcat, vcat, out=o_f), None,
                                          {"o": lambda: o_f.view(L, h)})
        except Exception as ex:  # noqa: BLE001
            out["flashinfer_cute_dsl"] = (None, None, {"error": repr(ex)[:300]})
    return out


def run_sweep_attn_lib(args):
    """Context, not part of the product: rank 0's causal attention (forward
    and backward) in this library beside the attention kernels of cuDNN
    (Blackwell SDPA, forward and backward), flash-attn 2 (mma.sync, forward
    and backward) and flashinfer (CuTe DSL Blackwell prefill, forward only),
    all fed the same Q, K, V, dO (Q, O from this library's forward).  The
    rank's work is two requests with bottom-right causal masks: chunk r
    against keys [0, (r+1) c) and chunk 2D-1-r against keys [0, (2D-r) c).
    Every round runs each implementation once, in rotating order, so drift of
    the power-capped clock hits all alike; medians over the rounds."""
    import torch
    from folded_tensor_sequence_rank_b200 import tsp
    wl = WORKLOADS[args.workload]
    T, h, H, F, D, r = wl["T"], wl["h"], wl["H"], wl["F"], wl["D"], 0
    L, hd = T // D, wl["h"] // wl["H"]
    c = L // 2
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, wl["seed"])
    sw = tsp.pack_shards(dims, D, w_full)
    del w_full
    kv_std = 0.02 * math.sqrt(h)
    K = rnd(T, h, std=kv_std, dtype=torch.float16)
    V = rnd(T, h, std=kv_std, dtype=torch.float16)
    x = rnd(L, h)
    y = torch.empty(L, h, dtype=torch.float32, device="cuda")
    ws = tsp.alloc_workspace(dims, D)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    tsp.layer_forward(dims, sw, r, x, K, V, y, ws)
    torch.cuda.synchronize()
    q = tsp.workspace_view(ws, dims, D, "q").clone()
    a = tsp.workspace_view(ws, dims, D, "a").clone()
    lse = tsp.workspace_view(ws, dims, D, "lse").clone()
    d_o = rnd(L, h, std=kv_std, dtype=torch.float16)
    aws = tsp.alloc_attn_backward_workspace(dims, D)
    dq = torch.empty(L, h, dtype=torch.float32, device="cuda")
    dK = torch.zeros(T, h, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    kv_len = [(r + 1) * c, (2 * D - r) * c]
    pairs = sum(float(sum(range(lo + 1, lo + c + 1))) for lo in (r * c, (2 * D - 1 - r) * c))
    fl_f, fl_b = 4.0 * h * pairs, 10.0 * h * pairs

    def ours_fwd():
        tsp.layer_forward(dims, sw, r, x, K, V, y, ws, events=evs)
    impls = {"tsp": (ours_fwd, lambda: tsp.attn_backward(dims, D, r, q, K, V, a, lse, d_o, dq, dK, dV, aws), {})}
    impls.update(_attn_lib_impls(q, a, d_o, K, V, c, kv_len, H, hd, dims.softmax_scale,
                                 ("cudnn", "fa2", "flashinfer")))

    def timed(name, fn):
        if name == "tsp" and fn is ours_fwd:
            fn()
            torch.cuda.synchronize()
            return evs[2].elapsed_time(evs[3])  # the attention launch inside the layer forward
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)
    live = [n for n, (f, _, _) in impls.items() if f is not None]
    for n in live:
        for _ in range(args.warmup):
            impls[n][0]()
            if impls[n][1] is not None:
                impls[n][1]()
    torch.cuda.synchronize()
    rounds = max(3, min(args.steps, 8))
    rec = {n: {"fwd": [], "bwd": []} for n in live}
    clocks = ClockSampler(0)
    time.sleep(0.3)
    for i in range(rounds):
        order = live[i % len(live):] + live[:i % len(live)]
        for n in order:
            rec[n]["fwd"].append(timed(n, impls[n][0]))
        for n in order:
            if impls[n][1] is not None:
                rec[n]["bwd"].append(timed(n, impls[n][1]))
    clk = clocks.stop()
    assert tsp.get_device_status(ws) == tsp.TSP_OK and tsp.get_device_status(aws) == tsp.TSP_OK
    res = {}
    for n, (f, b, info) in impls.items():
        if f is None:
            res[n] = {"error": info.get("error")}
            continue
        d = {"fwd_ms": round(statistics.median(rec[n]["fwd"]), 3)}
        d["fwd_tflops"] = round(fl_f / d["fwd_ms"] / 1e9, 1)
        if rec[n]["bwd"]:
            d["bwd_ms"] = round(statistics.median(rec[n]["bwd"]), 3)
            d["bwd_tflops"] = round(fl_b / d["bwd_ms"] / 1e9, 1)
        if "o" in info:
            d["o_maxabs_vs_tsp"] = float((info["o"]().float() - a.float()).abs().max())
        if "version" in info:
            d["version"] = info["version"]
        res[n] = d
    line = {"metric": "causal attention of one TSP rank beside library kernels on the same work (context)",
            "value": res["tsp"]["fwd_tflops"], "unit": "TFLOP/s (forward, this library)", "n_gpus": 1,
            "steps": rounds, "warmup": args.warmup, "higher_is_better": True, "dtype": "fp16", "data": "synthetic",
            "config": {"workload": f"rank 0 of T={T}, D={D}, {H} heads x {hd}: chunks 0 and {2 * D - 1} "
                                   f"({c} rows each) against keys [0, {kv_len[0]}) and [0, {kv_len[1]})",
                       "flops_fwd": fl_f, "flops_bwd": fl_b},
            "impls": res, "clocks": clk}
    return line


def run_sweep_gemm_lib(args):
    """Context, not part of the product: the rank step's four GEMMs in this
    library (per-kernel CUDA events inside one rank step: the QKV product, O
    with the shard sum and residual, W1 with GELU, W2 with the shard sum and
    residual) beside cuBLAS (torch.matmul, fp16 operands, fp32 accumulation,
    fp16 output, no epilogue) on the same M, K, N.  L2 is flushed before every
    timed launch; each round runs cuBLAS on the four shapes, then one rank
    step; medians over the rounds."""
    import torch
    from folded_tensor_sequence_rank_b200 import tsp
    wl = WORKLOADS[args.workload]
    T, h, H, F, D = wl["T"], wl["h"], wl["H"], wl["F"], wl["D"]
    L = T // D
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    rnd, w_full = _synthetic(T, h, F, wl["seed"])
    sw = tsp.pack_shards(dims, D, w_full)
    del w_full
    kv_std = 0.02 * math.sqrt(h)
    K = rnd(T, h, std=kv_std, dtype=torch.float16)
    V = rnd(T, h, std=kv_std, dtype=torch.float16)
    x = rnd(L, h)
    y = torch.empty(L, h, dtype=torch.bfloat16, device="cuda")
    ws = tsp.alloc_workspace(dims, D)
    shapes = {"qkv": (L, h, 3 * h, 1), "o": (L, h, h, 3), "w1": (L, h, F, 5), "w2": (L, F, h, 6)}
    mats = {n: (rnd(m, k, dtype=torch.float16), rnd(k, nn, std=0.02, dtype=torch.float16))
            for n, (m, k, nn, _) in shapes.items()}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    rec = {n: {"cublas": [], "tsp": []} for n in shapes}
    rounds = max(3, min(args.steps, 10))
    clocks = None
    for i in range(args.warmup + rounds):
        if i == args.warmup:
            clocks = ClockSampler(0)
        for n, (a, b) in mats.items():
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b)
            e1.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                rec[n]["cublas"].append(e0.elapsed_time(e1))
        flush.zero_()
        tsp.rank_step(dims, sw, 0, x, K, V, y, ws, events=evs)
        torch.cuda.synchronize()
        if i >= args.warmup:
            for n, (_, _, _, j) in shapes.items():
                rec[n]["tsp"].append(evs[j].elapsed_time(evs[j + 1]))
    clk = clocks.stop()
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    res = {}
    for n, (m, k, nn, _) in shapes.items():
        fl = 2.0 * m * k * nn
        d = {"m_k_n": [m, k, nn]}
        for impl in ("tsp", "cublas"):
            ms = statistics.median(rec[n][impl])
            d[f"{impl}_ms"] = round(ms, 4)
            d[f"{impl}_tflops"] = round(fl / ms / 1e9, 1)
        res[n] = d
    tot_tsp = sum(r["tsp_ms"] for r in res.values())
    tot_cb = sum(r["cublas_ms"] for r in res.values())
    return {"metric": "the rank step's GEMMs in this library beside cuBLAS on the same shapes (context)",
            "value": round(tot_cb / tot_tsp, 4), "unit": "cuBLAS time / this library's time, four GEMMs",
            "n_gpus": 1, "steps": rounds, "warmup": args.warmup, "higher_is_better": True, "dtype": "fp16",
            "data": "synthetic", "config": {"workload": f"rank 0 of T={T}, D={D}, h={h}, FFN {F}: M = {L} tokens",
                                            "l2": "flushed (256 MiB write) before every timed launch"},
            "gemms": res, "clocks": clk}


def run_sweep_stack(args):
    """A 32-layer stack of the 7B layer at T = 131072 on one GPU, all D = 8
    ranks in turn per layer (K/V projections, then layer forwards), random
    weights per layer.  Reports whole-stack tokens/s = T / forward time, the
    time per layer, the peak device memory of this one-GPU simulation, and
    the per-GPU memory account of the same forward on 8 GPUs."""
    import torch
    from folded_tensor_sequence_rank_b200 import stack, tsp
    T, h, H, F, D, n_layers = 131072, 4096, 32, 16384, 8, 32
    torch.cuda.set_device(0)
    dims = tsp.make_dims(T, h, H, F)
    layers = []
    for i in range(n_layers):
        rnd, w_full = _synthetic(T, h, F, 100 + i)
        layers.append(tsp.pack_shards(dims, D, w_full))
        del w_full
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    x = rnd(T, h)
    xs = [x.index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    del x
    K = torch.empty(T, h, dtype=torch.float16, device="cuda")
    V = torch.empty_like(K)
    ws = tsp.alloc_workspace(dims, D)
    torch.cuda.reset_peak_memory_stats()
    stack.stack_forward(dims, layers[:2], xs, K, V, ws)  # warm-up
    torch.cuda.synchronize()
    assert tsp.get_device_status(ws) == tsp.TSP_OK, "device wait timed out during warm-up"
    steps = max(1, min(args.steps, 2))
    clocks = ClockSampler(0)
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        ys = stack.stack_forward(dims, layers, xs, K, V, ws)
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert tsp.get_device_status(ws) == tsp.TSP_OK, "device wait timed out"
    assert all(torch.isfinite(y.float()).all() for y in ys)
    ms = e0.elapsed_time(e1) / steps
    acc = stack.memory_account(dims, D, n_layers)
    line = {"metric": "TSP 32-layer stack fwd tokens/s, all 8 ranks in turn on 1 B200 (7B layers, 128K, D=8)",
            "value": T / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": 1,
            "ms_per_step": ms, "ms_per_layer": ms / n_layers, "higher_is_better": True, "dtype": "fp16",
            "data": "synthetic",
            "config": {"workload": "32 x 7B dense layer (random weights per layer), T=131072, D=8, every rank in turn"},
            "peak_device_bytes_this_run": torch.cuda.max_memory_allocated(),
            "per_gpu_bytes_on_8_gpus": acc, "clocks": clk}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tsp", choices=["tsp", "reference"])
    ap.add_argument("--workload", default="7b-128k-d8", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations (all 8 ranks, the shard sweep, the backward, the stack) "
                         "that a default 1-GPU run measures after its main line")
    ap.add_argument("--sweep", choices=["ranks", "shards", "stack", "mlp_bwd", "layer_bwd", "tp", "attn_lib", "gemm_lib"],
                    default=None,
                    help="ranks: all 8 ranks of the 128K layer in turn (per-rank spread, whole-layer tokens/s); "
                         "shards: rank 0 at T=32768 for D=1..16; stack: a 32-layer forward at 128K; "
                         "mlp_bwd: the MLP-half backward of rank 0 at 128K; "
                         "layer_bwd: the whole layer's backward of rank 0 at 128K; "
                         "tp: the tensor-parallel baseline layer beside a TSP rank step at 128K; "
                         "attn_lib: the rank's attention beside cuDNN, flash-attn 2 and flashinfer kernels "
                         "on the same work (--workload picks T); "
                         "gemm_lib: the rank step's four GEMMs beside cuBLAS on the same shapes")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = WORKLOADS[args.workload]
    sweeps = {"ranks": run_sweep_ranks, "shards": run_sweep_shards, "mlp_bwd": run_sweep_mlp_bwd,
              "layer_bwd": run_sweep_layer_bwd, "tp": run_sweep_tp, "stack": run_sweep_stack,
              "attn_lib": run_sweep_attn_lib, "gemm_lib": run_sweep_gemm_lib}
    if args.sweep is not None:
        print(json.dumps(sweeps[args.sweep](args)), flush=True)
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_tsp(args, wl)


if __name__ == "__main__":
    main()
