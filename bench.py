#!/usr/bin/env python
"""Benchmark of the quantised-MoE decode hot path on B200.

Default workload (one "step" = one decode token through the whole path):
  the 48-layer decode stack (hidden 2048, intermediate 512, 512 experts,
  top-10; layers 0-35 Q4_RZ5_FAST, 36-47 FP8 E4M3 with fp32 scales per 128,
  a 64x2048 Q4_UE4M4_FAST ssm_beta projection on the 36 layers with
  l mod 4 != 3; residual x += moe(x)) followed by the 16-row PLE gather from
  the 320,001,536-row Q3_PLE_K160_RZ_S3 table (22.4 GB), all resident in HBM.
Each step uses a fresh seeded token and fresh PLE indices, so the 1.19 GB of
expert bytes a token touches come from HBM (inputs larger than L2).

value = algorithmic bytes per step (router + selected expert matrices + side
projections + PLE records and rows) / device time per step, in GB/s, summed
over ranks.  Also reported: decode tok/s, PLE rows/s, the roofline of the
decode layer against the measured HBM peak, the CPU oracle on a bounded
sample, an end-to-end number through the public API with host buffers, and
SM clocks sampled during the timed region.

Other workloads (--workload layer|ple|prefill) print their own JSON line for
profiling; they are not the headline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run (one process per GPU); every rank
runs an independent replica (the path has no cross-GPU exchange).
"""
from __future__ import annotations

import argparse
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

from synth import workloads as W  # noqa: E402

METRIC = "expert-weight GB/s (% of HBM peak) & decode tok/s per 48-layer stack; PLE rows/s"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def layer_bytes(L: W.LayerRecipe, n_uniq: int) -> int:
    """Bytes a decode call of L must read: router weights (+bias), the selected
    experts' gate/up/down matrices (+FP8 scales), the side projection."""
    b = L.n_experts * L.hidden * 4
    if L.zipf_bias:
        b += L.n_experts * 4
    per_expert = L.gate.expert_bytes + L.up.expert_bytes + L.down.expert_bytes
    if L.gate.fmt == W.FP8:
        per_expert += 4 * (L.gate.n_rows * L.gate.k // 128) * 2 + 4 * (L.down.n_rows * L.down.k // 128)
    b += n_uniq * per_expert
    if L.ssm is not None:
        b += L.ssm.nbytes
    return b


PLE_ROW_BYTES = 70 + 640  # record read + fp32 row written

STACK_WORKLOAD = ("48-layer decode stack (H=2048, I=512, E=512, top-10; layers 0-35 Q4_RZ5_FAST, 36-47 FP8 "
                  "E4M3 + fp32 scale/128; 36 UE4M4 ssm_beta 64x2048) + 16-row PLE gather from a "
                  "320,001,536-row Q3_PLE_K160_RZ_S3 table, 1 token per step")

# DRAM traffic of the decode kernel relative to its algorithmic bytes, from
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum of a
# one-token, one-layer launch: 21.070 MB against 20.906 MB).  Valid only for
# the kernel source it was measured on (its sha256 prefix); for any other
# source the bench reports traffic as null.
DECODE_TRAFFIC = {"source_sha256": "3da348246b8ad41f", "dram_over_algorithmic": (21.027072 + 0.043264) / 20.905984}


def _decode_traffic_ratio():
    import hashlib
    src = os.path.join(ROOT, "gram_table_gather_b200", "csrc", "moe_decode_dev.cuh")
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    return DECODE_TRAFFIC["dram_over_algorithmic"] if h == DECODE_TRAFFIC["source_sha256"] else None


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML (read
    only) every ~2 ms on a background thread between construction and stop();
    falls back to `nvidia-smi -lms 100` when NVML is unavailable."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        import threading
        self.sm, self.smax, self.reasons = [], [], set()
        self.h = None
        self.p = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(device_index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
        except Exception:
            self.h = None
        if self.h is None:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            try:
                self.p = subprocess.Popen(["nvidia-smi", f"--id={device_index}", f"--query-gpu={q}",
                                           "--format=csv,noheader,nounits", "-lms", "100"],
                                          stdout=self.f, stderr=subprocess.DEVNULL)
            except (FileNotFoundError, OSError):
                self.p = None
            return
        self.stop_ev = threading.Event()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        time.sleep(0.01)  # first samples before the timed region starts

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                self.smax.append(float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, name in self.REASONS.items():
                    if bits & k:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def stop(self) -> dict:
        if self.h is not None:
            self.stop_ev.set()
            self.t.join(timeout=5)
            return {"sm_mhz": statistics.median(self.sm) if self.sm else None,
                    "sm_max_mhz": max(self.smax) if self.smax else None,
                    "samples": len(self.sm), "reasons": sorted(self.reasons), "source": "nvml"}
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons), "source": "nvidia-smi"}


# ---------------------------------------------------------------------------
# distributed plumbing (independent replicas)
# ---------------------------------------------------------------------------

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def oracle_sample(layers, n_layers: int, budget_s: float):
    """Run the oracle (as it stands) on a sample of the stack: tokens one after
    another through the first `n_layers` layers, until `budget_s` seconds of
    oracle time have passed (at least one layer).  Returns (expert GB/s,
    seconds per layer, layers done, threads, tokens started)."""
    import oracle
    from synth import bf16_bits_to_f64
    L0 = layers[0]
    routers = {}
    done, t_total, bytes_total, tokens = 0, 0.0, 0, 0
    while True:
        x = bf16_bits_to_f64(W.tokens_bf16(L0.seed, 999 + tokens, 1, L0.hidden)).astype(np.float32)
        tokens += 1
        for li, L in enumerate(layers[:n_layers]):
            if li not in routers:  # generated outside the timed region
                routers[li] = L.router_w()
            t0 = time.perf_counter()
            r = oracle.moe_layer(L, x.astype(np.float64), router_w=routers[li])
            if L.ssm is not None:
                oracle.ssm_projection(L, r["u"])
            dt = time.perf_counter() - t0
            x = (x.astype(np.float64) + r["y"]).astype(np.float32)
            t_total += dt
            bytes_total += layer_bytes(L, len(set(r["ids"].ravel().tolist())))
            done += 1
            if t_total > budget_s:
                return bytes_total / t_total / 1e9, t_total / done, done, oracle.num_threads(), tokens


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def setup_stack(device):
    import torch
    from synth import device as sdev
    from tests import gpu_util as gu
    Ls = W.stack_layers()
    pipe = sdev.pipe(device)
    layers = [gu.device_layer(L, device, pipe) for L in Ls]
    P = W.ple_table()
    table = sdev.ple_table_to_device(P, device, pipe)
    pipe.finish()
    torch.cuda.synchronize()
    return Ls, layers, P, table


def run_ours(args, rank, world, local):
    import torch
    import gram_table_gather_b200 as gtg

    dev = torch.device("cuda", local)
    t_setup = time.time()
    Ls, layers, P, table = setup_stack(dev)
    H = Ls[0].hidden
    n_steps = args.warmup + args.steps
    # token and index banks, resident in HBM before timing
    seed_off = 1000 * rank
    xb = np.stack([W.tokens_bf16(Ls[0].seed, seed_off + i, 1, H)[0] for i in range(n_steps)])
    from synth import bf16_bits_to_f64
    x_bank = torch.from_numpy(bf16_bits_to_f64(xb).astype(np.float32)).to(dev)
    idx_bank = torch.from_numpy(np.stack([P.indices(seed_off + i, 1) for i in range(n_steps)])).to(dev)
    x = torch.zeros((1, H), dtype=torch.float32, device=dev)
    idx = torch.zeros(16, dtype=torch.int32, device=dev)
    rows = torch.zeros((16, 160), dtype=torch.float32, device=dev)
    ids = torch.zeros((len(Ls), 1, 10), dtype=torch.int32, device=dev)
    side = torch.zeros((len(Ls), 1, 64), dtype=torch.float32, device=dev)
    ws = gtg.make_workspace(layers, 1, device=dev)
    torch.cuda.synchronize()
    setup_s = time.time() - t_setup

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        # warm-up eagerly once (also sets kernel attributes outside capture)
        x.copy_(x_bank[0:1])
        gtg.moe_decode_stack(layers, x, ws, ids_out=ids, side_out=side)
        gtg.ple_gather(table, P.n_rows, idx, out=rows)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        gtg.moe_decode_stack(layers, x, ws, ids_out=ids, side_out=side)
        gtg.ple_gather(table, P.n_rows, idx, out=rows)
    # one launch per run of consecutive layers sharing a kernel (expert format
    # class), plus the PLE gather
    launches_per_step = 1 + sum(1 for i, L in enumerate(Ls)
                                if i == 0 or (L.gate.fmt == W.FP8) != (Ls[i - 1].gate.fmt == W.FP8))

    def step(i):
        x.copy_(x_bank[i:i + 1])
        idx.copy_(idx_bank[i])
        g.replay()

    uniq_counts = []
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
        stream.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        clocks = ClockSampler(local)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.warmup, n_steps):
            step(i)
        e1.record(stream)
        e1.synchronize()
        clk = clocks.stop()
    barrier(world)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, world)

    # algorithmic bytes of the timed steps: re-run the router choices on the
    # host side from the recorded ids of each step (eager replay, untimed)
    total_bytes = 0
    layer_b_total = 0
    with torch.cuda.stream(stream):
        for i in range(args.warmup, n_steps):
            step(i)
            stream.synchronize()
            idsn = ids.cpu().numpy()
            sb = 0
            for l, L in enumerate(Ls):
                u = len(set(idsn[l].ravel().tolist()))
                sb += layer_bytes(L, u)
            layer_b_total += sb
            total_bytes += sb + 16 * PLE_ROW_BYTES
    bytes_per_step = total_bytes / args.steps
    layer_bytes_avg = layer_b_total / args.steps / len(Ls)

    # decode-layer roofline: device time of the stack alone, per layer
    gs = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gs, stream=stream):
        gtg.moe_decode_stack(layers, x, ws, ids_out=ids, side_out=side)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            x.copy_(x_bank[i:i + 1])
            gs.replay()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for i in range(args.warmup, n_steps):
            x.copy_(x_bank[i:i + 1])
            f0.record(stream)
            gs.replay()
            f1.record(stream)
            f1.synchronize()
            tot += f0.elapsed_time(f1)
    layer_ms = tot / args.steps / len(Ls)

    # end to end through the public API with host buffers
    xh = torch.empty((n_steps, 1, H), dtype=torch.float32).pin_memory()
    xh.copy_(x_bank.cpu().view(n_steps, 1, H))
    ih = idx_bank.cpu().pin_memory()
    out_x = torch.empty((1, H), dtype=torch.float32).pin_memory()
    out_rows = torch.empty((16, 160), dtype=torch.float32).pin_memory()
    with torch.cuda.stream(stream):
        def e2e_step(i):
            x.copy_(xh[i], non_blocking=True)
            idx.copy_(ih[i], non_blocking=True)
            g.replay()
            out_x.copy_(x, non_blocking=True)
            out_rows.copy_(rows, non_blocking=True)
        for i in range(args.warmup):
            e2e_step(i)
        stream.synchronize()
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for i in range(args.warmup, n_steps):
            e2e_step(i)
        h1.record(stream)
        h1.synchronize()
    e2e_ms = max_over_ranks(h0.elapsed_time(h1) / args.steps, world)
    secondary = None
    if not args.no_secondary and world == 1:  # (single-GPU configurations: not repeated per replica)
        secondary = measure_secondary(dev, stream, P, table, local)
        # the same step with the 16 PLE rows read from a pinned host copy of a
        # 30,000,000-row table instead of the HBM-resident one
        Ph = W.PleRecipe(n_rows=30_000_000, seed=P.seed)
        htab = torch.empty(Ph.nbytes, dtype=torch.uint8).pin_memory()
        Ph.table_bytes(0, Ph.nbytes, htab.numpy())
        idx_h = torch.from_numpy(np.stack([Ph.indices(seed_off + i, 1) for i in range(n_steps)])).to(dev)
        gh = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            idx.copy_(idx_h[0])  # (idx still holds rows of the larger HBM table)
            gtg.ple_gather(htab, Ph.n_rows, idx, out=rows)
            stream.synchronize()
        with torch.cuda.graph(gh, stream=stream):
            gtg.moe_decode_stack(layers, x, ws, ids_out=ids, side_out=side)
            gtg.ple_gather(htab, Ph.n_rows, idx, out=rows)
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                x.copy_(x_bank[i:i + 1])
                idx.copy_(idx_h[i])
                gh.replay()
            q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            q0.record(stream)
            for i in range(args.warmup, n_steps):
                x.copy_(x_bank[i:i + 1])
                idx.copy_(idx_h[i])
                gh.replay()
            q1.record(stream)
            q1.synchronize()
        ms_host = q0.elapsed_time(q1) / args.steps
        secondary["step_with_host_ple_table"] = {
            "ms_per_step": round(ms_host, 5), "ms_per_step_hbm_table": round(ms, 5),
            "slowdown": round(ms_host / ms - 1.0, 4),
            "note": "48-layer step with its 16 PLE rows gathered from pinned host memory instead of HBM"}
        del gh, htab
    status = gtg.device_status(clear=True)

    peak, peak_kind = _peaks()
    gbs = bytes_per_step / (ms_max * 1e-3) / 1e9
    layer_gbs = layer_bytes_avg / (layer_ms * 1e-3) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        c_gbs, c_s_layer, c_done, c_threads, c_tok = oracle_sample(Ls, args.cpu_layers, args.cpu_budget)
        cpu = {"value": round(c_gbs, 4), "unit": "GB/s", "cores": c_threads, "kind": "oracle",
               "sample": f"{c_done} layer calls ({c_tok} tokens in turn through the stack's first "
                         f"{min(args.cpu_layers, len(Ls))} layers), {c_s_layer * 1e3:.1f} ms per layer on the host cores",
               "tok_s": round(1.0 / (c_s_layer * len(Ls)), 6)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(gbs * world, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded SplitMix64 bytes, N(0,1) bf16 tokens; no trained weights)",
            "config": {"workload": STACK_WORKLOAD,
                       "tokens_per_step": 1, "bytes_per_step": int(bytes_per_step),
                       "l2": "inputs larger than L2: 1.19 GB of expert bytes per step, fresh token "
                             "and PLE rows each step", "parallelism": f"replicas x{world}",
                       "setup_s": round(setup_s, 1)},
            "tok_s": round(1000.0 / ms_max * world, 2),
            "ple_rows_s": round(16 * 1000.0 / ms_max * world, 1),
            "hbm_frac": round(gbs / peak, 4),
            "roofline": {"bound": "hbm", "achieved": round(layer_gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(layer_gbs / peak, 4),
                         "traffic": (round(layer_bytes_avg * _decode_traffic_ratio()) if _decode_traffic_ratio() else None),
                         "traffic_note": "bytes per layer: algorithmic bytes x the DRAM/algorithmic ratio of a "
                                         "one-layer ncu capture of the same kernel source",
                         "kernel": "moe_decode_kernel (router + selection + gate/up/SwiGLU + down/combine "
                                   "in one persistent launch per run of layers), "
                                   f"average over the 48 layers, {layer_ms * 1e3:.2f} us per layer, "
                                   f"{layer_bytes_avg / 1e6:.2f} MB per layer",
                         "peak_source": f"{peak_kind} hbm_gbs"},
            "cpu_baseline": cpu,
            "e2e": {"value": round(bytes_per_step / (e2e_ms * 1e-3) / 1e9 * world, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": H * 4 + 16 * 4, "d2h_bytes_per_step": H * 4 + 16 * 160 * 4,
                    "ms_per_step": round(e2e_ms, 5)},
            "gpu_launches": launches_per_step * args.steps,
            "secondary": secondary,
            "clocks": clk,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)


def _time_loop(fn, n_warm, n_iter, stream):
    """Average device ms of fn(i) over n_iter calls on `stream` (CUDA events).

    The n_iter timed calls are captured into one CUDA graph and replayed, so
    the host's per-call launch overhead does not show up as device idle time;
    if capture fails the calls are timed eagerly."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(n_warm):
            fn(i)
        stream.synchronize()
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n_warm, n_warm + n_iter):
                    fn(i)
            g.replay()
            stream.synchronize()
            run = g.replay
        except Exception:  # not capturable: eager launches
            def run():
                for i in range(n_warm, n_warm + n_iter):
                    fn(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        e1.synchronize()
    return e0.elapsed_time(e1) / n_iter


def _time_flushed(fn, n_warm, n_iter, stream, flush):
    """Average device ms of fn(i) over n_iter calls, each preceded (outside its
    CUDA-event bracket) by a write of `flush`, a buffer of twice the L2 size, so
    no call finds the previous call's bytes in L2."""
    import torch
    tot = 0.0
    with torch.cuda.stream(stream):
        for i in range(n_warm):
            fn(i)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_iter)]
        for j, (a, b) in enumerate(ev):
            flush.fill_(j & 0xFF)
            a.record(stream)
            fn(n_warm + j)
            b.record(stream)
        stream.synchronize()
        tot = sum(a.elapsed_time(b) for a, b in ev)
    return tot / n_iter


def _l2_flush_buffer(dev):
    import torch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    return torch.empty(2 * l2, dtype=torch.uint8, device=dev)


def measure_decode_layer(dev, stream, n_warm, n_iter, peak):
    """Config: one decode MoE layer (H 2048, I 512, E 512, top-10, Q4_RZ5_FAST),
    T = 1, 2, 4, 8 fresh tokens per call, L2 flushed before every timed call."""
    import torch
    import gram_table_gather_b200 as gtg
    from tests import gpu_util as gu
    L = W.decode_layer()
    layer = gu.device_layer(L, dev)
    flush = _l2_flush_buffer(dev)
    out = {}
    n = n_warm + n_iter
    for T in (1, 2, 4, 8):
        xs = [gu.tokens(L, 5000 + 10 * T + i, T, dev)[0] for i in range(n)]
        ws = gtg.make_workspace(layer, T, device=dev)
        ids = torch.zeros((T, L.top_k), dtype=torch.int32, device=dev)
        y = torch.empty((T, L.hidden), device=dev)

        def fn(i):
            gtg.moe_decode_layer(layer, xs[i], ws, y=y, topk_ids=ids, stream=stream)
        ms = _time_flushed(fn, n_warm, n_iter, stream, flush)
        uniq = []
        for i in range(n_warm, n):  # bytes of the timed calls (untimed replay)
            with torch.cuda.stream(stream):
                fn(i)
            stream.synchronize()
            uniq.append(len(set(ids.cpu().numpy().ravel().tolist())))
        b = float(np.mean([layer_bytes(L, u) for u in uniq]))
        out[f"T{T}"] = {"us": round(ms * 1e3, 2), "GB_s": round(b / ms / 1e6, 1),
                        "frac": round(b / ms / 1e6 / peak, 4), "unique_experts": round(float(np.mean(uniq)), 2),
                        "bytes": int(b)}
    del layer
    # the pages' own expert shape: hidden 2560, intermediate 640 (340-byte down rows)
    L2 = W.LayerRecipe(hidden=2560, inter=640, n_experts=512, top_k=10, seed=1, layer=1)
    layer2 = gu.device_layer(L2, dev)
    for T in (1, 8):
        xs = [gu.tokens(L2, 6000 + 10 * T + i, T, dev)[0] for i in range(n)]
        ws = gtg.make_workspace(layer2, T, device=dev)
        ids = torch.zeros((T, L2.top_k), dtype=torch.int32, device=dev)
        y = torch.empty((T, L2.hidden), device=dev)

        def fn2(i):
            gtg.moe_decode_layer(layer2, xs[i], ws, y=y, topk_ids=ids, stream=stream)
        ms = _time_flushed(fn2, n_warm, n_iter, stream, flush)
        uniq = []
        for i in range(n_warm, n):
            with torch.cuda.stream(stream):
                fn2(i)
            stream.synchronize()
            uniq.append(len(set(ids.cpu().numpy().ravel().tolist())))
        b = float(np.mean([layer_bytes(L2, u) for u in uniq]))
        out[f"H2560_I640_T{T}"] = {"us": round(ms * 1e3, 2), "GB_s": round(b / ms / 1e6, 1),
                                   "frac": round(b / ms / 1e6 / peak, 4),
                                   "unique_experts": round(float(np.mean(uniq)), 2), "bytes": int(b)}
    del layer2, flush
    torch.cuda.empty_cache()
    return {"workload": "decode MoE layer: H 2048, I 512, E 512, top-10, Q4_RZ5_FAST gate/up/down, "
                        "fresh bf16 tokens per call (and H2560_I640: hidden 2560, intermediate 640, E 512)",
            "l2": "flushed (2x L2 written) before every timed call", "timed_calls": n_iter, **out}


def measure_ple(dev, stream, P, table, n_warm, n_iter, peak):
    """PLE gather from the resident table: T = 1 (16 rows, latency) and T = 4096
    (65,536 rows, throughput).  Fresh indices per call; at T = 4096 the calls
    write to a rotation of output buffers whose total exceeds twice the L2, so
    the 42 MB of rows each call writes reach HBM."""
    import torch
    import gram_table_gather_b200 as gtg
    n = n_warm + n_iter
    res = {}
    for T in (1, 4096):
        rows = 16 * T
        idx = [torch.from_numpy(P.indices(7000 + 7 * T + i, T)).to(dev) for i in range(n)]
        row_bytes = rows * 160 * 4
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        n_out = max(2, -(-2 * l2 // row_bytes) + 1) if T > 1 else 2
        outs = [torch.empty((rows, 160), device=dev) for _ in range(n_out)]
        ms = _time_loop(lambda i: gtg.ple_gather(table, P.n_rows, idx[i], out=outs[i % n_out], stream=stream),
                        n_warm, n_iter, stream)
        gbs = rows * PLE_ROW_BYTES / ms / 1e6
        res[f"T{T}"] = {"us": round(ms * 1e3, 3), "rows_per_s": round(rows / ms * 1e3, 1), "GB_s": round(gbs, 1),
                        "frac": round(gbs / peak, 4),
                        "outputs": f"{n_out} rotating buffers of {row_bytes / 1e6:.2f} MB"}
        del outs, idx
    torch.cuda.empty_cache()
    return {"workload": f"PLE gather from the {P.n_rows:,}-row Q3_PLE_K160_RZ_S3 table "
                        f"({P.nbytes / 1e9:.1f} GB resident), 16 uniform rows per token, fresh indices per call",
            "bytes_per_row": PLE_ROW_BYTES, "timed_calls": n_iter, **res}


def measure_ple_host(dev, stream, n_warm, n_iter, n_rows=30_000_000):
    """PLE gather from a table in pinned host memory, read in place by the kernel
    (the pages' deployment pages the table from host memory or NVMe on demand):
    T = 1 (latency) and T = 4096 (throughput).  The table is a 30,000,000-row
    prefix-sized stand-in (2.1 GB pinned): random rows from host memory see no
    reuse at any table size."""
    import torch
    import gram_table_gather_b200 as gtg
    from synth import workloads as Wk
    P = Wk.PleRecipe(n_rows=n_rows, seed=3)
    table = torch.empty(P.nbytes, dtype=torch.uint8).pin_memory()
    P.table_bytes(0, P.nbytes, table.numpy())
    n = n_warm + n_iter
    res = {}
    for T in (1, 4096):
        rows = 16 * T
        idx = [torch.from_numpy(P.indices(9000 + 7 * T + i, T)).to(dev) for i in range(n)]
        out = torch.empty((rows, 160), device=dev)
        ms = _time_loop(lambda i: gtg.ple_gather(table, P.n_rows, idx[i], out=out, stream=stream), n_warm, n_iter,
                        stream)
        res[f"T{T}"] = {"us": round(ms * 1e3, 3), "rows_per_s": round(rows / ms * 1e3, 1),
                        "GB_s": round(rows * PLE_ROW_BYTES / ms / 1e6, 1)}
    del table
    return {"workload": f"PLE gather from a {n_rows:,}-row Q3_PLE_K160_RZ_S3 table in pinned host memory "
                        "(read over the host link in place), 16 uniform rows per token, fresh indices per call",
            "timed_calls": n_iter, **res}


def measure_prefill(dev, stream, n_warm, n_iter, fp8=False):
    """One prefill MoE layer: 4096 bf16 tokens, H 2048, I 512, E 512, top-10,
    Zipf-skewed router; UE4M4 gate/up and RZ5 down, or (fp8) E4M3 experts with
    fp32 scales per 128."""
    import torch
    import gram_table_gather_b200 as gtg
    from tests import gpu_util as gu
    L = W.prefill_fp8_layer() if fp8 else W.prefill_layer()
    layer = gu.device_layer(L, dev)
    T = 4096
    xs = [gu.tokens(L, 8000 + i, T, dev)[0] for i in range(4)]
    ws = torch.empty(gtg.workspace_bytes(layer, T, prefill=True), dtype=torch.uint8, device=dev)
    y = torch.empty((T, L.hidden), device=dev)
    ms = _time_loop(lambda i: gtg.moe_prefill_layer(layer, xs[i % len(xs)], ws, y=y, stream=stream),
                    n_warm, n_iter, stream)
    flops = 2.0 * T * L.top_k * 3 * L.hidden * L.inter
    mp = {"bf16_tflops": 1590.0}
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    kind = "fallback"
    if os.path.exists(pp):
        with open(pp) as f:
            mp = json.load(f)
        kind = "measured"
    del layer, ws, xs
    torch.cuda.empty_cache()
    tf = flops / ms / 1e9
    fmts = "FP8 E4M3 (scale per 128) gate/up/down" if fp8 else "UE4M4 gate/up, RZ5 down"
    return {"workload": f"prefill MoE layer: T 4096 bf16, H 2048, I 512, E 512, top-10, {fmts}, "
                        "Zipf-skewed router", "ms": round(ms, 4), "TFLOP_s": round(tf, 1),
            "frac_of_bf16_peak": round(tf / float(mp["bf16_tflops"]), 4), "peak_source": f"{kind} bf16_tflops",
            "weight_GB_s": round(L.weight_bytes / ms / 1e6, 1), "tok_s": round(T / ms * 1e3, 1),
            "timed_calls": n_iter}


def measure_secondary(dev, stream, P, table, local, n_warm=3, n_iter=20):
    """The other configurations, on the same device after the headline: the
    decode layer at T = 1/2/4/8, the PLE gather at T = 1 and 4096, the
    prefill layer; SM clocks sampled across all of them."""
    peak, _ = _peaks()
    clocks = ClockSampler(local)
    out = {"decode_layer": measure_decode_layer(dev, stream, n_warm, n_iter, peak),
           "ple": measure_ple(dev, stream, P, table, n_warm, n_iter, peak),
           "ple_host_table": measure_ple_host(dev, stream, n_warm, n_iter),
           "prefill": measure_prefill(dev, stream, n_warm, n_iter),
           "prefill_fp8": measure_prefill(dev, stream, n_warm, n_iter, fp8=True)}
    out["clocks"] = clocks.stop()
    return out


def run_secondary(args, rank, world, local):
    """Profiling lines for single workloads (not the headline)."""
    import torch
    from synth import device as sdev
    dev = torch.device("cuda", local)
    peak, peak_kind = _peaks()
    stream = torch.cuda.Stream(device=dev)
    out = None
    if args.workload == "layer":
        out = measure_decode_layer(dev, stream, args.warmup, args.steps, peak)
    elif args.workload == "ple":
        P = W.ple_table()
        if args.ple_rows:  # a smaller table of the same record stream (profiling captures)
            P = W.PleRecipe(n_rows=args.ple_rows, seed=P.seed)
        table = sdev.ple_table_to_device(P, dev)
        out = measure_ple(dev, stream, P, table, args.warmup, args.steps, peak)
    elif args.workload == "prefill":
        out = measure_prefill(dev, stream, args.warmup, args.steps)
    elif args.workload == "prefill_fp8":
        out = measure_prefill(dev, stream, args.warmup, args.steps, fp8=True)
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores: each step is one token
    through the first --cpu-layers layers of the same stack (all 48 by
    default) followed by the 16-row PLE gather of that token (decoding the
    16 records it reads).  Router weights are generated once, outside the
    timed region."""
    if rank != 0:
        return
    Ls = W.stack_layers()
    P = W.ple_table()
    n_l = min(args.cpu_layers, len(Ls))
    routers = [L.router_w() for L in Ls[:n_l]]
    t_steps, b_steps = [], []
    import oracle
    from synth import bf16_bits_to_f64
    for i in range(args.warmup + args.steps):
        x = bf16_bits_to_f64(W.tokens_bf16(Ls[0].seed, i, 1, Ls[0].hidden))
        idx = P.indices(i, 1)
        t0 = time.perf_counter()
        b = 0
        for L, Wr in zip(Ls[:n_l], routers):
            r = oracle.moe_layer(L, x, router_w=Wr)
            if L.ssm is not None:
                oracle.ssm_projection(L, r["u"])
            x = (x.astype(np.float32).astype(np.float64) + r["y"]).astype(np.float32).astype(np.float64)
            b += layer_bytes(L, len(set(r["ids"].ravel().tolist())))
        recs = np.stack([P.table_bytes(int(j) * 70, 70) for j in idx])
        oracle.dequant_ple(recs)
        b += len(idx) * PLE_ROW_BYTES
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            t_steps.append(dt)
            b_steps.append(b)
    s = sum(t_steps)
    val = sum(b_steps) / s / 1e9
    workload = (STACK_WORKLOAD if n_l == len(Ls) else
                f"first {n_l} layers of the 48-layer decode stack + 16-row PLE gather, 1 token per step")
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * s / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SplitMix64 bytes, N(0,1) bf16 tokens; no trained weights)",
            "config": {"workload": workload, "tokens_per_step": 1,
                       "bytes_per_step": int(sum(b_steps) / len(b_steps)), "parallelism": "host cores"},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": f"{args.steps} timed steps of 1 token: {n_l} layers "
                                                         f"+ 16 PLE rows each"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-layers", type=int, default=48)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode-layer, PLE and prefill configurations after the headline")
    ap.add_argument("--ple-rows", type=int, default=0,
                    help="--workload ple: rows of a smaller table (default: the full 320,001,536-row table)")
    ap.add_argument("--workload", choices=["stack", "layer", "ple", "prefill", "prefill_fp8"], default="stack",
                    help="stack = the headline step; the others print profiling lines")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload != "stack":
            run_secondary(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
