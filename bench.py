#!/usr/bin/env python3
"""Benchmark of the TACT-KV codec: compress + decompress throughput of a synthetic visual-KV batch.

One step = compress every unit of the batch (DCT along S, DCT along H/W with energy sums,
allocation, DCT along H/W with quantization and packing) and decompress every payload back to
bf16, i.e. the whole hot path once.  Default workload: the 4B-class medical VLM layout
(34 layers x K/V of one sequence = 68 units, 64x16x16 grid, 4 KV heads x 256, 1 bit/element),
inputs resident in HBM before timing; the batch (2.28 GB) is far larger than L2, so no flush is
needed between steps.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank compresses its own batch of
the same size (units are independent, no data-path collective): weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV compress+decompress GB/s (bf16 input) and % of B200 HBM roofline"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="med4b")
    ap.add_argument("--bits", type=int, default=None, help="nominal bits/element (default: the workload's first)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-groups", type=int, default=32, help="unit groups pipelined over streams in the e2e run")
    ap.add_argument("--e2e-streams", type=int, default=4, help="streams (each with a workspace) in the e2e run")
    ap.add_argument("--units", type=int, default=None, help="use only the first U units of the batch (profiling)")
    return ap.parse_args()


# ------------------------------------------------------------------------------------ helpers ---
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", gpu_id], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for name, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id_for_smi(dev_index: int) -> str:
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev_index] if vis else str(dev_index)


def blas_threads() -> int:
    try:
        import numpy as np
        from threadpoolctl import threadpool_info
        np.dot(np.ones((64, 64)), np.ones((64, 64)))
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_round_trip_seconds(x_np, w, bits, n_units=1):
    """Time the CPU oracle (as it stands) compressing and decompressing n_units unit(s)."""
    from oracle import tactkv_oracle as O
    t = time.perf_counter()
    for _ in range(n_units):
        p = O.compress_unit(x_np, w.S, w.H, w.W, x_np.shape[1], x_np.shape[2], bits)
        O.decompress_unit(p)
    return time.perf_counter() - t


# ---------------------------------------------------------------------- multi-rank host logic ---
def rank_workload(w, rank: int):
    """The batch rank `rank` compresses: same shape and size on every rank, independent seeds
    (units are independent, so N ranks process N batches: weak scaling)."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time: every rank must call this (one all-reduce MAX)."""
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world: int, bytes_per_rank: int, ms: float) -> float:
    """Whole-job throughput: the bytes all ranks processed over the slowest rank's time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


# ---------------------------------------------------------------------------- reference arm ---
def run_reference(args, w, bits, rank):
    """The base contract's reference arm for this codec: the CPU oracle on the host cores."""
    if rank != 0:
        return
    import numpy as np
    import torch
    from dct_transform_coding_b200.workloads import make_unit, unit_seed
    sample_heads, D = 1, 32                                    # calibrate on 32 channels
    seed = unit_seed(w, 0, 0, 0)

    def sample(hd):
        x = make_unit(w.S, w.H, w.W, 1, hd, rho=w.rho, nu=w.nu, scale=w.scale, dtype=w.dtype, seed=seed)
        return x.float().numpy().astype(np.float64) if w.dtype == torch.float32 else x.float().numpy()

    t32 = oracle_round_trip_seconds(sample(D), w, bits)
    budget = 120.0 / max(1, args.steps + args.warmup)
    hd = 32
    while hd * 2 <= w.channels and t32 * (hd * 2) / 32 <= budget:
        hd *= 2
    x = sample(hd)
    for _ in range(args.warmup):
        oracle_round_trip_seconds(x, w, bits)
    times = [oracle_round_trip_seconds(x, w, bits) for _ in range(args.steps)]
    step = statistics.mean(times)
    nbytes = w.tokens * hd * 2
    value = nbytes / step / 1e9
    cores = blas_threads()
    desc = (f"1 unit of {w.name} (sequence 0, layer 0, K) restricted to its first {hd} of {w.channels} "
            f"channels ({w.S}x{w.H}x{w.W} grid, {bits} bit/elem), compress + decompress per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, bits),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, bits):
    return {"workload": w.name, "units": w.n_units, "S": w.S, "H": w.H, "W": w.W, "heads": w.heads,
            "head_dim": w.head_dim, "bits_per_element": bits, "input_bytes": w.n_units * w.elements_per_unit * 2,
            "l2": "inputs larger than L2 (no flush)"}


# --------------------------------------------------------------------------------- our arm ---
def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from dct_transform_coding_b200.workloads import WORKLOADS, Workload
    import dataclasses
    w = WORKLOADS[args.workload]
    bits = args.bits or w.bits[0]
    if args.impl == "reference":
        run_reference(args, w, bits, rank)
        return

    import torch
    import torch.distributed as dist
    from dct_transform_coding_b200 import tactkv as T
    from dct_transform_coding_b200.workloads import make_batch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # every rank compresses its own batch (independent seeds per rank): weak scaling
    wr = rank_workload(w, rank)
    x = make_batch(wr, device=dev, units=list(range(args.units)) if args.units else None)
    U, Tk, heads, D = x.shape
    all_units = list(wr.units())
    layers = [u[1] for u in all_units]
    kvs = [u[2] for u in all_units]
    cap = T.payload_capacity(w.S, w.H, w.W, heads, D, bits)
    payload = torch.zeros((U, (cap + 15) // 16 * 16), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x)
    cu = T.make_units(x, w.S, w.H, w.W, bits, heads=heads, head_dim=D, payload=payload, layers=layers, kvs=kvs)
    du = T.make_units(None, w.S, w.H, w.W, bits, heads=heads, head_dim=D, payload=payload, out=out,
                      layers=layers, kvs=kvs, n_units=U)
    ws = T.alloc_workspace(cu, dev)
    stream = torch.cuda.current_stream(dev)
    sp = int(stream.cuda_stream)

    def check(st, what):
        if st != T.TACTKV_OK:
            raise T.TactkvError(st, what)

    def step():
        check(T.tactkv_compress(cu, ws.data_ptr(), ws.numel(), sp), "compress")
        n = T.tactkv_last_launches()
        check(T.tactkv_decompress(du, ws.data_ptr(), ws.numel(), sp), "decompress")
        return n + T.tactkv_last_launches()

    def profiled_step(cu_p, du_p, ev_c, ev_d):
        check(T.tactkv_compress_profiled(cu_p, ws.data_ptr(), ws.numel(), sp, [e.cuda_event for e in ev_c]),
              "compress")
        check(T.tactkv_decompress_profiled(du_p, ws.data_ptr(), ws.numel(), sp, [e.cuda_event for e in ev_d]),
              "decompress")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = T.tactkv_device_status(ws.data_ptr(), ws.numel(), sp)
    check(st, "device status")

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id_for_smi(local)) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    launches = 0
    t0.record(stream)
    for k in range(args.steps):
        launches += step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    elapsed_ms = t0.elapsed_time(t1)
    if world > 1:
        elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    ms_step = elapsed_ms / args.steps

    # per-kernel attribution: separate profiled steps (the profiled entry points record an event at
    # every kernel boundary); not part of the timed region above
    # a call records the stage events again in every wave, so the profiled steps run one wave's
    # worth of units (at most 256) and the times are scaled to the whole batch
    n_sub = min(U, 256)
    cu_p, du_p = cu[:n_sub], du[:n_sub]
    scale = U / n_sub
    n_prof = min(5, args.steps)
    evs_c = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_prof)]
    evs_d = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_prof)]
    for e in [e for es in evs_c + evs_d for e in es]:
        e.record(stream)   # torch creates the CUDA event on its first record
    for k in range(n_prof):
        profiled_step(cu_p, du_p, evs_c[k], evs_d[k])
    torch.cuda.synchronize(dev)
    # stages: the S and H/W passes alternate per group of units, so they are timed together
    names_c = ["fdct_s+fdct_hw", "reduce_var+allocate", "pack"]
    names_d = ["decode_index", "idct_hw+idct_s"]
    kern = {n: scale * statistics.mean(evs_c[k][i].elapsed_time(evs_c[k][i + 1]) for k in range(n_prof))
            for i, n in enumerate(names_c)}
    kern.update({n: scale * statistics.mean(evs_d[k][i].elapsed_time(evs_d[k][i + 1]) for k in range(n_prof))
                 for i, n in enumerate(names_d)})
    ms_c = scale * statistics.mean(evs_c[k][0].elapsed_time(evs_c[k][3]) for k in range(n_prof))
    ms_d = scale * statistics.mean(evs_d[k][0].elapsed_time(evs_d[k][2]) for k in range(n_prof))

    # bytes: payload sizes actually written (header field total_bytes)
    hdr = payload[:, :64].cpu().numpy()
    pay_bytes = int(sum(int.from_bytes(bytes(h[48:56]), "little") for h in hdr))
    in_bytes = U * Tk * heads * D * 2
    alg_c = in_bytes + pay_bytes                     # read bf16 K/V, write payloads
    alg_d = pay_bytes + in_bytes                     # read payloads, write bf16 K/V
    peak, peak_kind = measured_peaks()
    value = job_gbs(world, in_bytes, ms_step)
    if args.units:
        w = dataclasses.replace(w, sequences=1, layers=U, kv=(0,))   # describe what actually ran
    achieved = (alg_c + alg_d) / (ms_step * 1e-3) / 1e9
    dominant = max(kern, key=kern.get)
    kernels = {n: {"ms": round(kern[n], 4), "share": round(kern[n] / (ms_c + ms_d), 4)} for n in kern}

    traffic = None
    tpath = os.path.join(ROOT, "profiles", f"{w.name}_step_dram_bytes.txt")
    if os.path.exists(tpath):
        for line in open(tpath):
            if line.startswith("dram_bytes_per_step:"):
                traffic = int(line.split(":")[1])

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_of(w, bits),
        # compress / decompress alone, from the profiled (one stream, kernel after kernel) steps
        "compress_gbs": round(in_bytes / (ms_c * 1e-3) / 1e9, 2),
        "decompress_gbs": round(in_bytes / (ms_d * 1e-3) / 1e9, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "compress+decompress step",
                     "algorithmic_bytes_per_step": alg_c + alg_d, "peak_kind": peak_kind,
                     "compress_frac": round(alg_c / (ms_c * 1e-3) / 1e9 / peak, 4),
                     "decompress_frac": round(alg_d / (ms_d * 1e-3) / 1e9 / peak, 4),
                     "dominant_kernel": dominant},
        "kernels": kernels,
        "gpu_launches": launches,
        "clocks": clocks,
    }

    if not args.no_e2e:
        result["e2e"] = e2e_run(args, T, x, payload, out, cu, du, ws, stream, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, bits, x)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def e2e_run(args, T, x, payload, out, cu, du, ws, stream, world):
    """The same metric through the C ABI from pinned host memory: each step copies the K/V in,
    compresses, copies the payloads out, decompresses and copies the reconstruction out.  The
    batch goes in groups of units over a few streams (each with its own workspace), so that the
    host-link copies of one group overlap the kernels of the others (32 groups over 4 streams
    measured best among 16/3, 32/3, 24/4 and 32/4 on med4b)."""
    import torch
    import torch.distributed as dist
    dev = x.device
    U = x.shape[0]
    xh = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    xh.copy_(x)
    ph = torch.empty(payload.shape, dtype=payload.dtype, pin_memory=True)
    oh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    G = max(1, min(U, args.e2e_groups))
    bounds = [(U * g // G, U * (g + 1) // G) for g in range(G)]
    bounds = [(a, b) for a, b in bounds if b > a]
    streams = [torch.cuda.Stream(dev) for _ in range(max(1, min(args.e2e_streams, len(bounds))))]
    largest = max(b - a for a, b in bounds)
    wss = [T.alloc_workspace(cu[:largest], dev) for _ in streams]

    def one():
        start = torch.cuda.Event()
        start.record(stream)
        for s in streams:
            s.wait_event(start)
        for g, (a, b) in enumerate(bounds):
            s, wsg = streams[g % len(streams)], wss[g % len(streams)]
            sp = int(s.cuda_stream)
            with torch.cuda.stream(s):
                x[a:b].copy_(xh[a:b], non_blocking=True)
                T.tactkv_compress(cu[a:b], wsg.data_ptr(), wsg.numel(), sp)
                ph[a:b].copy_(payload[a:b], non_blocking=True)
                T.tactkv_decompress(du[a:b], wsg.data_ptr(), wsg.numel(), sp)
                oh[a:b].copy_(out[a:b], non_blocking=True)
        for s in streams:
            done = torch.cuda.Event()
            done.record(s)
            stream.wait_event(done)

    one()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        one()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / args.e2e_steps
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    in_bytes = x.numel() * x.element_size()
    return {"value": round(job_gbs(world, in_bytes, ms), 2), "unit": "GB/s",
            "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": payload.numel() + out.numel() * out.element_size(),
            "ms_per_step": round(ms, 3), "groups": len(bounds), "streams": len(streams)}


def cpu_baseline(w, bits, x):
    """The oracle as it stands on the host cores, on whole units of the same batch (bounded)."""
    import numpy as np
    cores = blas_threads()
    xs = x[0].float().cpu().numpy()
    t = oracle_round_trip_seconds(xs, w, bits)
    n = 1
    if t < 10.0:
        extra = min(2, int(10.0 // max(t, 1e-3)))
        if extra:
            t += sum(oracle_round_trip_seconds(x[1 + i].float().cpu().numpy(), w, bits) for i in range(extra))
            n += extra
    nbytes = n * w.elements_per_unit * 2
    del np
    return {"value": round(nbytes / t / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} whole unit(s) of {w.name} (layers 0.., K/V), compress + decompress, fp64 NumPy",
            "seconds": round(t, 2)}


if __name__ == "__main__":
    main()
