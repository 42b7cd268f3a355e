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
NOMINAL_HBM_GBS = 8000.0     # B200 HBM3e nominal, reported beside the measured copy peak


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="med4b")
    ap.add_argument("--bits", type=int, default=None, help="nominal bits/element (default: the workload's first)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-groups", type=int, default=32, help="unit groups pipelined over streams in the e2e run")
    ap.add_argument("--e2e-streams", type=int, default=4, help="streams (each with a workspace) in the e2e run")
    ap.add_argument("--streams", type=int, default=1,
                    help="streams of the timed step: the batch goes in that many unit groups, one per stream "
                         "(each with its own workspace), joined at the end of every step")
    ap.add_argument("--units", type=int, default=None, help="use only the first U units of the batch (profiling)")
    ap.add_argument("--no-others", action="store_true", help="skip the other workloads' lines")
    ap.add_argument("--no-attention", action="store_true", help="skip the decode-time attention measurement")
    ap.add_argument("--q-per-kv", type=int, default=2, help="query heads per K/V head in the attention step")
    ap.add_argument("--other-units", type=int, default=128, help="units of each other workload measured")
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
                                          "-lms", "50", "-i", gpu_id], stdout=subprocess.PIPE,
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


def oracle_round_trip_seconds(x_np, w, bits, n_units=1):
    """Time the CPU oracle (as it stands) compressing and decompressing n_units unit(s), on one
    host thread: its NumPy calls are held to a single BLAS/OpenMP thread, so the core count the
    baseline reports (1) is the one it used."""
    from threadpoolctl import threadpool_limits
    from oracle import tactkv_oracle as O
    with threadpool_limits(limits=1):
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
    """The base contract's reference arm for this codec: the CPU oracle, as it stands, on the host.
    Each step compresses and decompresses one whole unit of the workload (units taken in turn), or,
    when K + W whole units would not end within about four minutes, the first channels of one."""
    if rank != 0:
        return
    import numpy as np
    import torch
    from dct_transform_coding_b200.workloads import make_workload_unit

    all_units = list(w.units())

    def unit(k, channels=None):
        x = make_workload_unit(w, *all_units[k % len(all_units)])
        if channels is not None:
            x = x.reshape(x.shape[0], -1)[:, :channels].reshape(x.shape[0], 1, channels)
        return x.float().numpy().astype(np.float64) if w.dtype == torch.float32 else x.float().numpy()

    t_unit = oracle_round_trip_seconds(unit(0), w, bits)
    total = args.steps + args.warmup
    channels = None
    if t_unit * total > 240.0:
        channels = 32
        while channels * 2 <= w.channels and t_unit * total * channels * 2 / w.channels <= 240.0:
            channels *= 2
    for k in range(args.warmup):
        oracle_round_trip_seconds(unit(k, channels), w, bits)
    times = [oracle_round_trip_seconds(unit(args.warmup + k, channels), w, bits) for k in range(args.steps)]
    step = statistics.mean(times)
    nbytes = w.tokens * (channels or w.channels) * 2
    value = nbytes / step / 1e9
    what = "one whole unit" if channels is None else f"the first {channels} of the {w.channels} channels of one unit"
    desc = (f"{what} of {w.name} per step (units in turn from (sequence 0, layer 0, K); {w.S}x{w.H}x{w.W} grid, "
            f"{bits} bit/elem), compress + decompress by the fp64 NumPy oracle on one host thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, bits),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc},
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

    n_str = max(1, min(args.streams, U))
    groups = [(U * k // n_str, U * (k + 1) // n_str) for k in range(n_str)]
    side = [torch.cuda.Stream(dev) for _ in range(n_str)] if n_str > 1 else []
    side_ws = [T.alloc_workspace(cu[a:b], dev) for a, b in groups] if n_str > 1 else []

    def step():
        if n_str == 1:
            check(T.tactkv_compress(cu, ws.data_ptr(), ws.numel(), sp), "compress")
            n = T.tactkv_last_launches()
            check(T.tactkv_decompress(du, ws.data_ptr(), ws.numel(), sp), "decompress")
            return n + T.tactkv_last_launches()
        # groups of units on their own streams: one group's forward transforms (bound by data
        # movement) can overlap another's decoding (bound by instructions)
        start = torch.cuda.Event()
        start.record(stream)
        n = 0
        for (a, b), s_, w_ in zip(groups, side, side_ws):
            s_.wait_event(start)
            spg = int(s_.cuda_stream)
            check(T.tactkv_compress(cu[a:b], w_.data_ptr(), w_.numel(), spg), "compress")
            n += T.tactkv_last_launches()
            check(T.tactkv_decompress(du[a:b], w_.data_ptr(), w_.numel(), spg), "decompress")
            n += T.tactkv_last_launches()
        for s_ in side:
            done = torch.cuda.Event()
            done.record(s_)
            stream.wait_event(done)
        return n

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

    prof = profile_stages(T, cu, du, ws, stream, U, min(5, args.steps))

    # bytes: payload sizes actually written (header field total_bytes)
    hdr = payload[:, :64].cpu().numpy()
    pay_bytes = int(sum(int.from_bytes(bytes(h[48:56]), "little") for h in hdr))
    in_bytes = U * Tk * heads * D * 2
    peak, peak_kind = measured_peaks()
    value = job_gbs(world, in_bytes, ms_step)
    if args.units:
        w = dataclasses.replace(w, sequences=1, layers=U, kv=(0,))   # describe what actually ran
    roofline = stage_roofline(prof, in_bytes, pay_bytes, U * w.tokens, ms_step, peak, peak_kind, w.name)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "io_dtype": "bf16", "data": "synthetic",
        "config": config_of(w, bits),
        # compress / decompress alone, from the profiled (one stream, kernel after kernel) steps
        "compress_gbs": round(in_bytes / (prof["compress_ms"] * 1e-3) / 1e9, 2),
        "decompress_gbs": round(in_bytes / (prof["decompress_ms"] * 1e-3) / 1e9, 2),
        "roofline": roofline,
        "kernels": {n: {"ms": round(v, 4), "share": round(v / (prof["compress_ms"] + prof["decompress_ms"]), 4)}
                    for n, v in prof["stages"].items()},
        "gpu_launches": launches,
        "clocks": clocks,
    }

    if rank == 0 and not args.no_attention and len(set(kvs)) == 2:
        result["attention_decode"] = attention_bench(T, w, bits, payload, out, du, ws, stream, layers, kvs, peak,
                                                     peak_kind, q_per_kv=args.q_per_kv)
    if not args.no_e2e:
        result["e2e"] = e2e_run(args, T, x, payload, out, cu, du, ws, stream, world)
    del x, out, payload, ws
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wr, bits, args.units)
    if rank == 0 and world == 1 and not args.no_others and not args.units:
        result["other_workloads"] = other_workloads(T, args, w.name, dev, peak, peak_kind)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def attention_bench(T, w, bits, payload, out, du, ws, stream, layers, kvs, peak, peak_kind, q_per_kv=2, iters=20):
    """One decode step of attention for every layer of the batch, straight from the compressed K/V
    (units with kv 0 / 1 of the same layer), against the same step done by decompressing K and V to
    bf16, straight into the [layers, heads, tokens, head_dim] layout SDPA takes (through the output
    strides), and running torch's scaled_dot_product_attention on them; both warmed up first.  The
    roofline counts the bytes the step must read (the K and V payloads, the queries) and write
    (outputs, m, l)."""
    import torch
    kvs = kvs[:payload.shape[0]]
    ki = [i for i, kv in enumerate(kvs) if kv == 0]
    vi = [i for i, kv in enumerate(kvs) if kv == 1]
    ki, vi = ki[:min(len(ki), len(vi), 128)], vi[:min(len(ki), len(vi), 128)]
    U = len(ki)
    dev = payload.device
    Hq, D = w.heads * q_per_kv, w.head_dim
    q = torch.randn((U, Hq, D), device=dev, generator=torch.Generator(device=dev).manual_seed(17))
    pk, pv = payload[ki].contiguous(), payload[vi].contiguous()
    lay = [layers[i] for i in ki]
    T.attention_decode(q, pk, pv, w.S, w.H, w.W, bits, heads=w.heads, head_dim=D, layers=lay, check=True)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(iters):
        T.attention_decode(q, pk, pv, w.S, w.H, w.W, bits, heads=w.heads, head_dim=D, layers=lay)
    ev[1].record(stream)
    sp = int(stream.cuda_stream)
    qh = q.to(torch.bfloat16)[:, :, None, :]
    Kb = torch.empty((U, w.heads, w.tokens, D), dtype=torch.bfloat16, device=dev)   # [U, heads, T, D]
    Vb = torch.empty_like(Kb)
    dk = T.make_units(None, w.S, w.H, w.W, bits, heads=w.heads, head_dim=D, payload=pk,
                      out=Kb.permute(0, 2, 1, 3), layers=lay, kvs=[0] * U)
    dv = T.make_units(None, w.S, w.H, w.W, bits, heads=w.heads, head_dim=D, payload=pv,
                      out=Vb.permute(0, 2, 1, 3), layers=lay, kvs=[1] * U)

    def baseline():
        for units in (dk, dv):
            st = T.tactkv_decompress(units, ws.data_ptr(), ws.numel(), sp)
            if st != T.TACTKV_OK:
                raise T.TactkvError(st, "attention baseline")
        with torch.cuda.stream(stream):
            torch.nn.functional.scaled_dot_product_attention(qh, Kb, Vb, enable_gqa=True)

    for _ in range(3):
        baseline()
    ev[2].record(stream)
    for _ in range(iters):
        baseline()
    ev[3].record(stream)
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / iters
    ms_ref = ev[2].elapsed_time(ev[3]) / iters
    hdr = torch.cat([pk, pv])[:, :64].cpu().numpy()
    pay_bytes = int(sum(int.from_bytes(bytes(h[48:56]), "little") for h in hdr))
    alg = pay_bytes + q.numel() * 4 + U * Hq * (D + 2) * 4
    kv_bf16 = 2 * U * w.tokens * w.channels * 2
    return {"layers": U, "q_heads": Hq, "ms_per_step": round(ms, 4),
            "ms_decompress_then_sdpa": round(ms_ref, 4), "speedup": round(ms_ref / ms, 2),
            "kv_bf16_bytes_served": kv_bf16, "value": round(kv_bf16 / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "roofline": {"bound": "hbm", "algorithmic_bytes": alg,
                         "achieved": round(alg / (ms * 1e-3) / 1e9, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(alg / (ms * 1e-3) / 1e9 / peak, 4), "peak_kind": peak_kind}}


STAGES_C = ["forward", "allocate", "pack"]          # compress: DCTs with energies, allocation, packing
STAGES_D = ["decode_index", "idct_hw", "idct_s"]    # decompress: payload index, decode + inverse W/H, inverse S


def profile_stages(T, cu, du, ws, stream, U, n_prof):
    """Per-stage device times of one step, from the profiled entry points (an event at every stage
    boundary), outside the timed region.  A call records the stage events again in every wave, so
    the profiled steps run one wave's worth of units (at most 256), scaled to the whole batch."""
    import torch
    n_sub = min(U, 256)
    cu_p, du_p = cu[:n_sub], du[:n_sub]
    scale = U / n_sub
    evs_c = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_prof)]
    evs_d = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_prof)]
    for e in [e for es in evs_c + evs_d for e in es]:
        e.record(stream)   # torch creates the CUDA event on its first record
    sp = int(stream.cuda_stream)
    for k in range(n_prof):
        st = T.tactkv_compress_profiled(cu_p, ws.data_ptr(), ws.numel(), sp, [e.cuda_event for e in evs_c[k]])
        if st != T.TACTKV_OK:
            raise T.TactkvError(st, "compress")
        st = T.tactkv_decompress_profiled(du_p, ws.data_ptr(), ws.numel(), sp, [e.cuda_event for e in evs_d[k]])
        if st != T.TACTKV_OK:
            raise T.TactkvError(st, "decompress")
    torch.cuda.synchronize()
    mean = statistics.mean
    stages = {n: scale * mean(evs_c[k][i].elapsed_time(evs_c[k][i + 1]) for k in range(n_prof))
              for i, n in enumerate(STAGES_C)}
    stages.update({n: scale * mean(evs_d[k][i].elapsed_time(evs_d[k][i + 1]) for k in range(n_prof))
                   for i, n in enumerate(STAGES_D)})
    return {"stages": stages,
            "compress_ms": scale * mean(evs_c[k][0].elapsed_time(evs_c[k][3]) for k in range(n_prof)),
            "decompress_ms": scale * mean(evs_d[k][0].elapsed_time(evs_d[k][3]) for k in range(n_prof))}


def stage_roofline(prof, in_bytes, pay_bytes, bins_x_units, ms_step, peak, peak_kind, name):
    """Roofline of the dominant kernel (each stage below is one kernel, reduce_var + allocate aside):
    its algorithmic bytes (what the method itself must move through HBM in that kernel) over its
    measured time.  forward (the three forward DCTs) reads the bf16 input; allocate writes the gains
    and bit widths (5 B per bin) and the headers; pack writes the codes; decode_index reads gains and
    widths; idct_hw (decoding with the inverse DCTs along W and H) reads the codes; idct_s (the
    inverse DCT along S) writes the bf16 output.  The whole step's fraction (both directions'
    algorithmic bytes over the timed step) is reported beside it."""
    meta = 5 * bins_x_units
    codes = max(0, pay_bytes - meta)
    alg = {"forward": in_bytes, "allocate": meta, "pack": codes, "decode_index": meta, "idct_hw": codes,
           "idct_s": in_bytes}
    stages = prof["stages"]
    dom = max(stages, key=stages.get)
    achieved = alg[dom] / (stages[dom] * 1e-3) / 1e9
    step_achieved = 2 * (in_bytes + pay_bytes) / (ms_step * 1e-3) / 1e9
    traffic = dram_traffic(name, dom)
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "traffic_gbs": round(traffic / (stages[dom] * 1e-3) / 1e9, 1) if traffic else None,
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "kernel": dom, "kernel_ms": round(stages[dom], 4), "algorithmic_bytes": alg[dom],
            "peak_kind": peak_kind,
            "step_achieved": round(step_achieved, 1), "step_frac": round(step_achieved / peak, 4),
            "step_frac_of_nominal_8tbs": round(step_achieved / NOMINAL_HBM_GBS, 4),
            "compress_frac": round((in_bytes + pay_bytes) / (prof["compress_ms"] * 1e-3) / 1e9 / peak, 4),
            "decompress_frac": round((in_bytes + pay_bytes) / (prof["decompress_ms"] * 1e-3) / 1e9 / peak, 4)}


def dram_traffic(name, stage):
    """DRAM bytes (read + write) of one launch of the stage's kernel on this workload, from the ncu
    summary in profiles/ (lines `stage <name>: <bytes>`), or None when none was taken at this build."""
    path = os.path.join(ROOT, "profiles", f"{name}_dram_bytes.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        if line.startswith(f"stage {stage}:"):
            return int(line.split(":")[1])
    return None


def other_workloads(T, args, main_name, dev, peak, peak_kind):
    """The other benchmark workloads in the same run: one wave of up to --other-units units of each
    (the codec's cost is per unit, so a wave stands for the batch), 10 timed steps, no e2e."""
    import torch
    from dct_transform_coding_b200.workloads import WORKLOADS, make_batch
    out = {}
    for name, bits_list in (("tiny", None), ("med4b_b8", (1, 2, 4)), ("med32b", None), ("video", None)):
        if name == main_name:
            continue
        w = WORKLOADS[name]
        U = min(w.n_units, args.other_units)
        x = make_batch(w, device=dev, units=list(range(U)))
        all_units = list(w.units())[:U]
        layers, kvs = [u[1] for u in all_units], [u[2] for u in all_units]
        for bits in (bits_list or w.bits):
            flags = T.TACTKV_FP32_IO if x.dtype == torch.float32 else 0
            cap = T.payload_capacity(w.S, w.H, w.W, w.heads, w.head_dim, bits, flags)
            payload = torch.zeros((U, (cap + 15) // 16 * 16), dtype=torch.uint8, device=dev)
            y = torch.empty_like(x)
            cu = T.make_units(x, w.S, w.H, w.W, bits, heads=w.heads, head_dim=w.head_dim, payload=payload,
                              layers=layers, kvs=kvs, flags=flags)
            du = T.make_units(None, w.S, w.H, w.W, bits, heads=w.heads, head_dim=w.head_dim, payload=payload,
                              out=y, layers=layers, kvs=kvs, n_units=U, flags=flags)
            ws = T.alloc_workspace(cu, dev)
            stream = torch.cuda.current_stream(dev)
            sp = int(stream.cuda_stream)

            def step():
                T.tactkv_compress(cu, ws.data_ptr(), ws.numel(), sp)
                T.tactkv_decompress(du, ws.data_ptr(), ws.numel(), sp)

            for _ in range(3):
                step()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            a.record(stream)
            for _ in range(10):
                step()
            b.record(stream)
            torch.cuda.synchronize(dev)
            st = T.tactkv_device_status(ws.data_ptr(), ws.numel(), sp)
            if st != T.TACTKV_OK:
                raise T.TactkvError(st, f"{name} device status")
            ms = a.elapsed_time(b) / 10
            prof = profile_stages(T, cu, du, ws, stream, U, 3)
            hdr = payload[:, :64].cpu().numpy()
            pay_bytes = int(sum(int.from_bytes(bytes(h[48:56]), "little") for h in hdr))
            in_bytes = x.numel() * 2          # the metric's unit: bf16 bytes of K/V
            rl = stage_roofline(prof, in_bytes, pay_bytes, U * w.tokens, ms, peak, peak_kind, name)
            out[f"{name}@{bits}"] = {"units": U, "ms_per_step": round(ms, 4),
                                     "value": round(in_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                                     "step_frac": rl["step_frac"], "dominant": rl["kernel"],
                                     "dominant_frac": rl["frac"],
                                     "stages_ms": {k: round(v, 4) for k, v in prof["stages"].items()}}
            del payload, y, ws
        del x
        torch.cuda.empty_cache()
    return out


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
                st = T.tactkv_compress(cu[a:b], wsg.data_ptr(), wsg.numel(), sp)
                ph[a:b].copy_(payload[a:b], non_blocking=True)
                st = st or T.tactkv_decompress(du[a:b], wsg.data_ptr(), wsg.numel(), sp)
                oh[a:b].copy_(out[a:b], non_blocking=True)
                if st != T.TACTKV_OK:
                    raise T.TactkvError(st, "e2e step")
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


def cpu_baseline(w, bits, n_units=None):
    """The oracle as it stands, on one host thread, on whole units of the same workload (units
    taken in order from the first, up to about 10 s of work)."""
    import numpy as np
    import torch
    from dct_transform_coding_b200.workloads import make_workload_unit
    all_units = list(w.units())[:n_units or None]

    def unit(k):
        x = make_workload_unit(w, *all_units[k % len(all_units)])
        return x.float().numpy().astype(np.float64) if w.dtype == torch.float32 else x.float().numpy()

    t = oracle_round_trip_seconds(unit(0), w, bits)
    n = 1
    while t < 10.0 and n < 3:
        t += oracle_round_trip_seconds(unit(n), w, bits)
        n += 1
    nbytes = n * w.elements_per_unit * 2
    return {"value": round(nbytes / t / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} whole unit(s) of {w.name} (units 0..{n - 1}), compress + decompress, fp64 NumPy "
                      f"oracle on one host thread", "seconds": round(t, 2)}

if __name__ == "__main__":
    main()
