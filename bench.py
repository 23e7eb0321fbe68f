#!/usr/bin/env python
"""Benchmark of the mHC forward hot path on B200: one step = mhc_pre + mhc_post
over T=8192 tokens, n=4 streams, C=4096, bf16 (the LLM-scale sublayer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Under torchrun (N > 1) every rank processes
its own batch of T tokens (weak scaling; the tokens are independent, so no
collective is on the data path) and the step time is the maximum over ranks.

* value      tokens/s of the whole job, inputs resident in HBM, device-timed
             with CUDA events over exactly K steps (barrier + synchronize on
             both sides).  Inputs (X 256 MiB, F_out 64 MiB) exceed the 126 MB
             L2, so no flush is needed between steps.
* e2e        the same metric through the public API with pinned HOST buffers:
             every step copies X and F_out host->device and x_in, the
             coefficients and X_next device->host, pipelined over token
             chunks on three streams (copies in, kernels, copies out).
* roofline   the dominant kernel's algorithmic bytes per launch / its mean
             CUDA-event duration inside the timed region, against the measured
             HBM copy bandwidth.
* cpu_baseline  the fp64 oracle on a bounded sample of tokens (rank 0, N = 1).
* --impl reference  runs the oracle (the reference arm of this method): same
             metric and workload, each step a bounded sample of tokens.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(T=8192, n=4, C=4096, dtype="bf16", seed=1)
METRIC = "mHC fwd tokens/s at n=4,C=4096; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


def algorithmic_bytes(T: int, n: int, C: int, es: int = 2) -> dict:
    """Bytes each kernel must move per launch: mhc_pre reads X once, writes x_in and the
    coefficients, and reads phi once; mhc_post reads X and F_out and the coefficients and
    writes X_next (the (n+1)C read / nC write count of the fused post kernel)."""
    P = n * n + 2 * n
    pre = T * (n * C * es + C * es + (2 * n + n * n) * 4) + n * C * P * es + P * 4
    post = T * (n * C * es + C * es + (n + n * n) * 4 + n * C * es)
    return {"mhc_pre": pre, "mhc_post": post}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s)"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling (200 ms) of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- dist
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own tokens_per_rank per step
    (weak scaling); the time is the maximum over ranks of the timed region."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# -------------------------------------------------------------- oracle leg
def oracle_sample_rate(inp: dict, seconds: float, max_tokens: int):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload's
    tokens; returns (tokens/s, tokens, threads)."""
    import oracle
    oracle.lib()
    T = inp["T"]
    probe = min(8, T)
    t0 = time.perf_counter()
    oracle.mhc_forward(inp["X"][:probe], inp["F"][:probe], inp["phi"], inp["alpha"], inp["b"],
                       inp["t_iters"], inp["eps"])
    per_tok = (time.perf_counter() - t0) / probe
    S = int(max(1, min(max_tokens, T, seconds / max(per_tok, 1e-9))))
    t0 = time.perf_counter()
    oracle.mhc_forward(inp["X"][:S], inp["F"][:S], inp["phi"], inp["alpha"], inp["b"],
                       inp["t_iters"], inp["eps"])
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return S / dt, S, threads


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle, timed on the host cores."""
    if rank != 0:
        return
    import synth
    import oracle
    inp = synth.mhc_inputs(**WORKLOAD)
    oracle.lib()
    T = inp["T"]
    # size each step so the whole run stays within about two minutes
    t0 = time.perf_counter()
    oracle.mhc_forward(inp["X"][:4], inp["F"][:4], inp["phi"], inp["alpha"], inp["b"])
    per_tok = (time.perf_counter() - t0) / 4
    S = int(max(1, min(T, 120.0 / max(per_tok, 1e-9) / max(1, args.steps + args.warmup))))
    for w in range(args.warmup):
        oracle.mhc_forward(inp["X"][:S], inp["F"][:S], inp["phi"], inp["alpha"], inp["b"])
    t0 = time.perf_counter()
    for k in range(args.steps):
        lo = (k * S) % max(1, T - S + 1)
        oracle.mhc_forward(inp["X"][lo:lo + S], inp["F"][lo:lo + S], inp["phi"], inp["alpha"], inp["b"])
    dt = time.perf_counter() - t0
    value = S * args.steps / dt
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    w = WORKLOAD
    sample = f"{S} tokens per step of the T={w['T']}, n={w['n']}, C={w['C']} bf16 workload (inputs widened to fp64)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, synth.mhc_inputs)",
        "config": config_dict(args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(N: int) -> dict:
    w = WORKLOAD
    return {"workload": f"mHC forward sublayer (mhc_pre + mhc_post), T={w['T']} tokens per GPU, "
                        f"n={w['n']}, C={w['C']}, bf16 state, fp32 coefficients, Sinkhorn 20 iterations",
            "T_per_gpu": WORKLOAD["T"], "n": WORKLOAD["n"], "C": WORKLOAD["C"], "t_iters": 20,
            "global_tokens": WORKLOAD["T"] * N, "parallelism": f"dp{N} (independent token batches)",
            "l2": f"no flush: inputs larger than L2 (X {w['T'] * w['n'] * w['C'] * 2 >> 20} MiB, F_out "
                  f"{w['T'] * w['C'] * 2 >> 20} MiB, X_next {w['T'] * w['n'] * w['C'] * 2 >> 20} MiB vs 126 MB L2)"}


# ------------------------------------------------------------------ ours
def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist
    import synth
    import stream_residual_connections_b200 as M

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    inp = synth.mhc_inputs(**WORKLOAD)
    T, n, C = inp["T"], inp["n"], inp["C"]

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) \
            if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(device)

    X, F = to_dev(inp["X"]), to_dev(inp["F"])
    phi = to_dev(np.ascontiguousarray(inp["phi"].T))        # the library's layout: phi^T [P][nC]
    b = torch.from_numpy(inp["b"]).to(device)
    alpha = inp["alpha"]
    x_in = torch.empty((T, C), dtype=torch.bfloat16, device=device)
    Hp = torch.empty((T, n), dtype=torch.float32, device=device)
    Ho = torch.empty((T, n), dtype=torch.float32, device=device)
    Hr = torch.empty((T, n, n), dtype=torch.float32, device=device)
    Xn = torch.empty_like(X)
    stream = torch.cuda.current_stream(device)

    def step():
        M.mhc_pre(X, phi, alpha, b, 20, 1e-6, x_in=x_in, H_pre=Hp, H_post=Ho, H_res=Hr, stream=stream)
        M.mhc_post(X, F, Ho, Hr, X_next=Xn, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier(world, device)

    # --- timed region: K steps, per-kernel events on the launching stream
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(device.index if world == 1 else local)
    if not args.profile:
        clocks.start()
    time.sleep(0.3 if K >= 100 else 0.0)
    torch.cuda.synchronize(device)
    barrier(world, device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(K):
        ev[k][0].record(stream)
        M.mhc_pre(X, phi, alpha, b, 20, 1e-6, x_in=x_in, H_pre=Hp, H_post=Ho, H_res=Hr, stream=stream)
        ev[k][1].record(stream)
        M.mhc_post(X, F, Ho, Hr, X_next=Xn, stream=stream)
        ev[k][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    clk = clocks.stop()
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world, device)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    post_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    ms_per_step = ms / K
    value = job_throughput(world, T, K, ms)

    # the CUDA-core (FMA) projection path on the same inputs, for comparison
    fma_ms = None
    if not args.profile and args.compare_fma:
        M.mhc_set_path(M.MHC_PATH_FMA)
        for _ in range(2):
            M.mhc_pre(X, phi, alpha, b, 20, 1e-6, x_in=x_in, H_pre=Hp, H_post=Ho, H_res=Hr, stream=stream)
        fs, fe = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fs.record(stream)
        for _ in range(5):
            M.mhc_pre(X, phi, alpha, b, 20, 1e-6, x_in=x_in, H_pre=Hp, H_post=Ho, H_res=Hr, stream=stream)
        fe.record(stream)
        torch.cuda.synchronize(device)
        fma_ms = fs.elapsed_time(fe) / 5
        M.mhc_set_path(M.MHC_PATH_AUTO)

    if args.profile:
        if rank == 0:
            print(json.dumps({"profile": True, "T": T, "steps": K, "ms_per_step": ms_per_step,
                              "mhc_pre_ms": pre_ms, "mhc_post_ms": post_ms}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # --- end to end through the public API with host buffers
    Ke = max(1, min(K, args.e2e_steps))
    Xh = torch.from_numpy(np.ascontiguousarray(inp["X"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    Fh = torch.from_numpy(np.ascontiguousarray(inp["F"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (x_in, Hp, Ho, Hr, Xn)]
    h2d = Xh.numel() * 2 + Fh.numel() * 2
    d2h = sum(t.numel() * t.element_size() for t in outs_h)

    # the step pipelined over token chunks on three streams: host->device copies of
    # chunk i+1 and device->host copies of chunk i-1 run while chunk i is mixed
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    bounds = [T * i // args.e2e_chunks for i in range(args.e2e_chunks + 1)]
    devs = (x_in, Hp, Ho, Hr, Xn)

    def e2e_step():
        for c in range(args.e2e_chunks):
            lo, hi = bounds[c], bounds[c + 1]
            with torch.cuda.stream(s_in):
                X[lo:hi].copy_(Xh[lo:hi], non_blocking=True)
                F[lo:hi].copy_(Fh[lo:hi], non_blocking=True)
            stream.wait_stream(s_in)
            M.mhc_pre(X[lo:hi], phi, alpha, b, 20, 1e-6, x_in=x_in[lo:hi], H_pre=Hp[lo:hi], H_post=Ho[lo:hi],
                      H_res=Hr[lo:hi], stream=stream)
            M.mhc_post(X[lo:hi], F[lo:hi], Ho[lo:hi], Hr[lo:hi], X_next=Xn[lo:hi], stream=stream)
            s_out.wait_stream(stream)
            with torch.cuda.stream(s_out):
                for h, d in zip(outs_h, devs):
                    h[lo:hi].copy_(d[lo:hi], non_blocking=True)
        # the next step's first copies overwrite X and F: after this step's reads
        s_in.wait_stream(stream)
        stream.wait_stream(s_out)

    e2e_step()
    torch.cuda.synchronize(device)
    barrier(world, device)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    s_in.wait_stream(stream)
    for _ in range(Ke):
        e2e_step()
    e2.record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    e2e_ms = max_over_ranks(s2.elapsed_time(e2), world, device)
    e2e_value = job_throughput(world, T, Ke, e2e_ms)

    # --- roofline of the dominant kernel
    peak, peak_src = measured_peak()
    ab = algorithmic_bytes(T, n, C)
    kern = {"mhc_pre": pre_ms, "mhc_post": post_ms}
    kern_rows = {}
    for name, kms in kern.items():
        gbs = ab[name] / (kms / 1e3) / 1e9
        kern_rows[name] = {"ms": kms, "algorithmic_bytes": ab[name], "achieved_gbs": gbs,
                           "frac": gbs / peak, "share": kms / (pre_ms + post_ms)}
    dom = max(kern, key=kern.get)
    traffic = TRAFFIC.get(dom)
    roof = {"bound": "hbm", "achieved": kern_rows[dom]["achieved_gbs"], "peak": peak, "unit": "GB/s",
            "frac": kern_rows[dom]["frac"], "traffic": traffic, "kernel": dom,
            "peak_source": peak_src}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, S, threads = oracle_sample_rate(inp, seconds=args.cpu_seconds, max_tokens=T)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"first {S} tokens of the same T={T}, n={n}, C={C} workload, fp64 oracle "
                         f"(mhc_pre + mhc_post), OpenMP over tokens"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded numpy PCG64, synth.mhc_inputs)",
            "config": config_dict(world),
            "gpu_launches": 2 * K,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": Ke, "pipelined_chunks": args.e2e_chunks},
            "roofline": roof,
            "kernels": kern_rows,
            "mhc_pre_fma_path_ms": fma_ms,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------- secondary workloads
def xhc_bytes(T: int, N: int, k: int, m: int, C: int, r: int, kappa_sum: int) -> dict:
    """Bytes each xHC kernel must move per launch.  xhc_route reads X once and
    phi_read, writes x_in, H_pre, the scores, idx and w; xhc_conv_gs reads F_out
    and the conv weights and writes V [T][r+1][C] fp32; xhc_sparse_update reads
    V and the k routed rows of X, writes those rows back, reads phi_act and
    writes the coefficients."""
    R, Kr = 2 * N - m, r + 1
    Pa = k * k + k * Kr
    route = T * N * C * 2 + N * C * R * 2 + T * C * 2 + T * (N + (N - m) + 2 * k) * 4
    conv = T * C * 2 + kappa_sum * C * 4 + T * Kr * C * 4
    update = T * Kr * C * 4 + 2 * T * k * C * 2 + k * C * Pa * 2 + T * (2 * k + Pa) * 4
    return {"xhc_route": route, "xhc_conv_gs": conv, "xhc_sparse_update": update}


def mhc_bwd_bytes(T: int, n: int, C: int) -> int:
    """Bytes the backward must move per call: X, F_out, dX_next and dx_in read once,
    dX and dF_out written once, phi read and dphi written once (fp32)."""
    P = n * n + 2 * n
    return T * (n * C * 2 * 3 + C * 2 * 2) + n * C * P * (2 + 4)


def hc_bytes(T: int, n: int, C: int) -> dict:
    """Bytes per call: hc_pre reads X and theta once and writes x_in and the
    coefficients; mhc_post as in the mHC step."""
    return {"hc_pre": T * n * C * 2 + (n + 2) * C * 2 + T * C * 2 + T * (2 * n + n * n) * 4,
            "mhc_post": T * (2 * (2 * n * C + C) + 4 * (n + n * n))}


def amax_bytes(L: int, T: int, n: int) -> int:
    """Bytes per call: the L x T matrices read once, the per-token gains written once."""
    return L * T * (n * n * 4 + 2 * 4) + L * 2 * 4


def run_secondary(args, local):
    """Timing lines for the other kernels of the method (xHC sublayer, mHC backward,
    HC sublayer, Amax Gain diagnostic) on their own workloads; one JSON line, rank 0
    of a single process."""
    import torch
    import synth
    import stream_residual_connections_b200 as M

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) \
            if a.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(a))
        return t.to(device)

    peak, peak_src = measured_peak()
    K = args.steps
    if args.workload == "xhc":
        wl = dict(synth.WORKLOADS["xhc"])
        if args.tokens:
            wl["T"] = args.tokens
        inp = synth.xhc_inputs(**wl)
        T, N, k, m, C = inp["T"], inp["N"], inp["k"], inp["m"], inp["C"]
        X = to_dev(inp["X"])
        F = to_dev(inp["F"])
        phi_read = to_dev(np.ascontiguousarray(inp["phi_read"].T))
        b_read = to_dev(inp["b_read"])
        kappa = [int(x) for x in inp["kappa"]]
        conv_w = (to_dev(np.concatenate([w.reshape(-1) for w in inp["conv_w"]])), kappa)
        phi_act = to_dev(np.ascontiguousarray(inp["phi_act"].T))
        b_act = to_dev(inp["b_act"])
        r = len(inp["kappa"])
        outs = dict(x_in=torch.empty((T, C), dtype=X.dtype, device=device),
                    H_pre=torch.empty((T, N), device=device), score=torch.empty((T, N - m), device=device),
                    idx=torch.empty((T, k), dtype=torch.int32, device=device),
                    w=torch.empty((T, k), device=device))
        V = torch.empty((T, r + 1, C), dtype=torch.float32, device=device)
        Hr = torch.empty((T, k, k), device=device)
        Hpo = torch.empty((T, k, r + 1), device=device)
        names = ("xhc_route", "xhc_conv_gs", "xhc_sparse_update")

        def launches():
            yield lambda: M.xhc_route(X, phi_read, inp["alpha_read"], b_read, k, m, inp["eps"], stream=stream, **outs)
            yield lambda: M.xhc_conv_gs(F, conv_w, V=V, stream=stream)
            yield lambda: M.xhc_sparse_update(X, V, outs["idx"], outs["w"], phi_act, inp["alpha_act"], b_act,
                                              inp["t_iters"], inp["eps"], H_res=Hr, H_post=Hpo, stream=stream)
        nbytes = xhc_bytes(T, N, k, m, C, r, sum(inp["kappa"]))
        desc = (f"xHC sublayer (xhc_route + xhc_conv_gs + xhc_sparse_update, X updated in place), T={T}, "
                f"N={N}, k={k}, m={m}, C={C}, kappa={list(inp['kappa'])}, bf16 state, Sinkhorn 20 iterations")
    elif args.workload == "hc":
        wl = dict(synth.WORKLOADS["hc_llm"])
        if args.tokens:
            wl["T"] = args.tokens
        inp = synth.hc_inputs(**wl)
        T, n, C = inp["T"], inp["n"], inp["C"]
        X, F = to_dev(inp["X"]), to_dev(inp["F"])
        theta = to_dev(inp["theta"])
        b = to_dev(inp["b"])
        x_in = torch.empty((T, C), dtype=X.dtype, device=device)
        Hp = torch.empty((T, n), device=device)
        Ho = torch.empty((T, n), device=device)
        Hr = torch.empty((T, n, n), device=device)
        Xn = torch.empty_like(X)
        names = ("hc_pre", "mhc_post")

        def launches():
            yield lambda: M.hc_pre(X, theta, inp["alpha"], b, inp["eps"], x_in=x_in, H_pre=Hp, H_post=Ho,
                                   H_res=Hr, stream=stream)
            yield lambda: M.mhc_post(X, F, Ho, Hr, X_next=Xn, stream=stream)
        nbytes = hc_bytes(T, n, C)
        desc = (f"HC sublayer, tanh coefficients (hc_pre + mhc_post), T={T}, n={n}, C={C}, bf16; inputs "
                f"larger than L2 (X {T * n * C * 2 >> 20} MiB), no flush")
    elif args.workload == "mhc_tf32":
        wl = dict(synth.WORKLOADS["mhc_llm"])
        if args.tokens:
            wl["T"] = args.tokens
        inp = synth.mhc_inputs(**wl, phi_dtype="tf32")
        T, n, C = inp["T"], inp["n"], inp["C"]
        X, F = to_dev(inp["X"]), to_dev(inp["F"])
        phiT = to_dev(np.ascontiguousarray(inp["phi"].T))
        pair = M.mhc_phi_tf32_pair(phiT, n, stream=stream)      # once per update of phi
        b = to_dev(inp["b"])
        x_in = torch.empty((T, C), dtype=X.dtype, device=device)
        Hp = torch.empty((T, n), device=device)
        Ho = torch.empty((T, n), device=device)
        Hr = torch.empty((T, n, n), device=device)
        Xn = torch.empty_like(X)
        names = ("mhc_pre", "mhc_post", "mhc_phi_tf32_pair")

        def launches():
            yield lambda: M.mhc_pre(X, pair, inp["alpha"], b, 20, 1e-6, x_in=x_in, H_pre=Hp, H_post=Ho, H_res=Hr,
                                    phi_tf32_pair=True, stream=stream)
            yield lambda: M.mhc_post(X, F, Ho, Hr, X_next=Xn, stream=stream)
            yield lambda: M.mhc_phi_tf32_pair(phiT, n, pair=pair, stream=stream)
        P = n * n + 2 * n
        RH = (P + 15) // 16 * 16
        pre_b = T * (2 * n * C + 2 * C + 4 * (2 * n + n * n)) + 2 * RH * n * C * 2
        nbytes = {"mhc_pre": pre_b, "mhc_post": T * (2 * (2 * n * C + C) + 4 * (n + n * n)),
                  "mhc_phi_tf32_pair": P * n * C * 4 + 2 * RH * n * C * 2}
        desc = (f"mHC forward sublayer with phi in tf32 (the pages' Eq.10 dtype; bf16 pair on tensor cores), "
                f"T={T}, n={n}, C={C}, bf16 state; the pair packing (once per phi update) is timed as a "
                f"third kernel of the loop")
    elif args.workload == "amax":
        Lz, T, n = 64, args.tokens or 65536, 4
        rng = np.random.default_rng(8)
        Hh = (np.eye(n, dtype=np.float32) + rng.standard_normal((Lz, T, n, n), dtype=np.float32) * np.float32(0.1))
        H = torch.from_numpy(Hh).to(device)
        del Hh
        gain = torch.empty((Lz, T, 2), device=device)
        gmax = torch.empty((Lz, 2), device=device)
        names = ("mhc_amax_gain",)
        inp = {"H": None}

        def launches():
            yield lambda: M.mhc_amax_gain(H, gain=gain, gain_max=gmax, stream=stream)
        nbytes = {"mhc_amax_gain": amax_bytes(Lz, T, n)}
        desc = (f"Amax Gain Magnitude of the composite residual map over a stack of L={Lz} layers, T={T} "
                f"tokens, n={n}, fp32 H_res = I + N(0, 0.01) ({Lz * T * n * n * 4 >> 20} MiB, larger than L2, "
                f"no flush); per-token gains and the maxima over tokens written")
    else:
        wl = dict(synth.WORKLOADS["mhc_bwd"])
        if args.tokens:
            wl["T"] = args.tokens
        inp = synth.mhc_grad_inputs(**wl)
        T, n, C = inp["T"], inp["n"], inp["C"]
        X, F = to_dev(inp["X"]), to_dev(inp["F"])
        phi = to_dev(np.ascontiguousarray(inp["phi"].T))
        b = to_dev(inp["b"])
        dXn, dxi = to_dev(inp["dX_next"]), to_dev(inp["dx_in"])
        P = n * n + 2 * n
        bufs = dict(dX=torch.empty_like(X), dF=torch.empty_like(F),
                    dphi=torch.empty((P, n * C), device=device), dalpha=torch.empty(3, device=device),
                    db=torch.empty(P, device=device),
                    workspace=torch.empty(max(M.mhc_backward_workspace_bytes(T, n, C), 256), dtype=torch.uint8,
                                          device=device))
        names = ("mhc_backward",)

        def launches():
            yield lambda: M.mhc_backward(X, F, phi, inp["alpha"], b, dXn, dxi, 20, 1e-6, stream=stream, **bufs)
        nbytes = {"mhc_backward": mhc_bwd_bytes(T, n, C)}
        desc = f"mHC sublayer backward (recompute + unrolled Sinkhorn reverse), T={T}, n={n}, C={C}, bf16"

    for _ in range(args.warmup):
        for f in launches():
            f()
    torch.cuda.synchronize(device)
    # the fp64 oracle on a bounded sample of the same workload's tokens (host cores)
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        oracle.lib()
        if args.workload == "mhc_tf32":
            def oracle_step(S):
                oracle.mhc_forward(inp["X"][:S], inp["F"][:S], inp["phi"], inp["alpha"], inp["b"], 20, 1e-6)
            what = "mhc_pre + mhc_post, tf32 phi"
        elif args.workload == "hc":
            def oracle_step(S):
                co = oracle.hc_pre(inp["X"][:S], inp["theta"], inp["alpha"], inp["b"], inp["eps"])
                oracle.mhc_post(inp["X"][:S], inp["F"][:S], co["H_post"], co["H_res"])
            what = "hc_pre + mhc_post"
        elif args.workload == "amax":
            def oracle_step(S):
                oracle.amax_gain(H[:, :S].cpu().numpy())
            what = "mhc_amax_gain, L=64"
        elif args.workload == "xhc":
            def oracle_step(S):
                rt = oracle.xhc_route(inp["X"][:S], inp["phi_read"], inp["alpha_read"], inp["b_read"], k, m,
                                      inp["eps"])
                V0 = oracle.xhc_conv_gs(inp["F"][:S], inp["conv_w"], seq_len=T)
                oracle.xhc_sparse_update(inp["X"][:S], V0, rt["idx"], rt["w"], inp["phi_act"], inp["alpha_act"],
                                         inp["b_act"], inp["t_iters"], inp["eps"])
            what = "xhc_route + xhc_conv_gs + xhc_sparse_update"
        else:
            def oracle_step(S):
                oracle.mhc_backward(inp["X"][:S], inp["F"][:S], inp["phi"], inp["alpha"], inp["b"],
                                    inp["dX_next"][:S], inp["dx_in"][:S], 20, 1e-6)
            what = "mhc_backward"
        t_a = time.perf_counter()
        oracle_step(4)
        per_tok = (time.perf_counter() - t_a) / 4
        S = int(max(4, min(T, args.cpu_seconds / max(per_tok, 1e-9))))
        t_a = time.perf_counter()
        oracle_step(S)
        dt = time.perf_counter() - t_a
        cpu = {"value": S / dt, "unit": "tokens/s", "cores": int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)),
               "kind": "oracle", "sample": f"first {S} tokens of the same workload, fp64 oracle ({what})"}
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for kk in range(K):
        ev[kk][0].record(stream)
        for j, f in enumerate(launches()):
            f()
            ev[kk][j + 1].record(stream)
    end.record(stream)
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(end) / K
    rows = {}
    for j, name in enumerate(names):
        kms = sum(e[j].elapsed_time(e[j + 1]) for e in ev) / K
        gbs = nbytes[name] / (kms / 1e3) / 1e9
        rows[name] = {"ms": kms, "algorithmic_bytes": nbytes[name], "achieved_gbs": gbs, "frac": gbs / peak}
    print(json.dumps({"workload": args.workload, "config": desc, "steps": K, "warmup": args.warmup,
                      "ms_per_step": ms, "tokens_per_s": T / (ms / 1e3), "kernels": rows, "peak_gbs": peak,
                      "peak_source": peak_src, "cpu_baseline": cpu}), flush=True)


# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of the current
# kernels, from one --set full capture at T=6144 scaled to T=8192 by the token
# count (profiles/mhc_pre_tc_T6144_n4_C4096_full.md, mhc_post_...).  Set to
# None whenever a kernel changes after its capture.
TRAFFIC = {"mhc_pre": 331.7e6, "mhc_post": 542.2e6}


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--e2e-chunks", type=int, default=8,
                   help="token chunks the e2e step is pipelined over (copies overlap the kernels)")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--compare-fma", type=int, default=1,
                   help="also time mhc_pre's CUDA-core projection path (5 launches, not in the step)")
    p.add_argument("--profile", action="store_true",
                   help="only warm-up + timed kernel launches (for ncu); no e2e, clocks or oracle")
    p.add_argument("--tokens", type=int, default=None, help="override T (profiling of small cases)")
    p.add_argument("--n", type=int, default=None, help="override n of the mHC forward (the n sweep)")
    p.add_argument("--C", type=int, default=None, help="override C of the mHC forward")
    p.add_argument("--workload", choices=("mhc_fwd", "xhc", "mhc_bwd", "hc", "amax", "mhc_tf32"), default="mhc_fwd",
                   help="mhc_fwd: the benchmark line; xhc / mhc_bwd: timing lines for the other kernels")
    args = p.parse_args(argv)
    global METRIC
    if args.tokens:
        WORKLOAD["T"] = args.tokens
    if args.n:
        WORKLOAD["n"] = args.n
    if args.C:
        WORKLOAD["C"] = args.C
    METRIC = f"mHC fwd tokens/s at n={WORKLOAD['n']},C={WORKLOAD['C']}; achieved HBM GB/s vs B200 peak"
    world, rank, local = dist_env()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return 0
    if args.workload != "mhc_fwd":
        run_secondary(args, local)
        return 0
    run_ours(args, world, rank, local)
    return 0


if __name__ == "__main__":
    sys.exit(main())
