#!/usr/bin/env python
"""Throughput of the hybrid BF16/Int4 partial-sum compression path on B200.

One step is one pass of the online path over one batch of P ranks' bf16 partial sums, resident in
HBM: hq_quantize_pack then hq_dequant_reduce (``--path split``, the default) or
hq_compress_reduce (``--path fused``).  ``value`` is partial-sum bytes (P*T*H*2 per step, all
ranks) per second over the timed steps.  Calibration and selection run once per calibration, not
per batch; they are timed on their own and reported under ``offline``.

Prints one JSON line.  ``--impl reference`` times the CPU oracle instead (the reference arm of
this benchmark: a plain single-threaded C restatement of the method).  Under torchrun each rank
runs an independent replica on its own GPU (the method has no data-path collective on one node
here); the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "partial-sum GB/s compressed+reduced (1 B200), % of HBM peak; compression ratio"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal
L2_BYTES = 126 * 2**20
SECOND_WORKLOAD = {"prefill70b": "prefill7b", "prefill7b": "prefill70b"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["hq", "reference"], default="hq")
    ap.add_argument("--path", choices=["split", "fused"], default="split")
    ap.add_argument("--workload", default="prefill70b")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cold-reps", type=int, default=20, help="launches of each kernel timed alone, L2 flushed")
    ap.add_argument("--second-steps", type=int, default=400,
                    help="timed steps of the second large workload (0: skip it)")
    ap.add_argument("--small-steps", type=int, default=200,
                    help="timed steps of each of the two small workloads, decode and pr1 (0: skip them)")
    ap.add_argument("--no-next", dest="next_paths", action="store_false",
                    help="skip the two-step, partial-sync and per-rank-buffer measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-clocks", action="store_true")
    return ap.parse_args()


def workload(name: str) -> synth.Config:
    if name in synth.CONFIGS:
        return synth.CONFIGS[name]
    for c in synth.sweep_configs():
        if c.name == name:
            return c
    raise SystemExit(f"unknown workload {name}")


def describe(cfg: synth.Config) -> str:
    dist = {"normal": "N(0, std_h)", "student_t3": "Student-t(3) x std_h", "uniform": "U(-1,1)"}[cfg.dist]
    s = f"{cfg.name}: P={cfg.P} ranks, bf16 partial sums [T={cfg.T}, H={cfg.H}], k={cfg.k} kept, {dist}"
    if cfg.dist != "uniform":
        s += f", std_h ~ LogNormal(0,{cfg.sigma}), {cfg.n_out} outlier cols x{cfg.out_mult:g}"
    if cfg.spike_p:
        s += f", spikes p={cfg.spike_p} x{cfg.spike_mult:g}"
    return s + f"; {cfg.calib_batches} calib batches of {cfg.calib_T} rows, EMA {cfg.beta}"


def algo_bytes(cfg: synth.Config) -> dict:
    """Bytes each call must move (reads + writes), parameters included."""
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    Hr = H - k
    params = P * H * (4 + 4 + 1)
    return {
        "calibrate": P * T * H * 2 + 4 * P * H * 4,
        "select": 2 * P * H * 4 + params + H * 4,
        "quantize_pack": P * T * H * 2 + P * T * Hr // 2 + P * T * k * 2 + P * H * 5 + H * 4,
        "dequant_reduce": P * T * Hr // 2 + P * T * k * 2 + T * H * 2 + P * H * 5 + H * 4,
        "compress_reduce": P * T * H * 2 + T * H * 2 + params + H * 4,
    }


def compression_ratio(cfg):
    return (16.0 * cfg.H) / (4.0 * (cfg.H - cfg.k) + 16.0 * cfg.k)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: copy bandwidth)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int, enabled: bool):
        self.proc = None
        self.gpu = gpu_index
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100", "-i", str(gpu_index)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [p.strip() for p in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------------------------
# distributed plumbing (replicas; the max-over-ranks timing is the only collective)
# ---------------------------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if args.impl == "hq" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------------------------
class OracleStep:
    """The online path on the CPU oracle over rows [0, S) of the workload's evaluation batch:
    quantize-pack and dequant-reduce, with parameters calibrated and selected once beforehand."""

    def __init__(self, cfg, x_rows: np.ndarray):
        import oracle

        self.o = oracle.get()
        self.cfg = cfg
        self.x = x_rows
        emin, emax = self.o.calibrate(x_rows, cfg.beta, True)
        self.sel = self.o.select_topk(emin, emax, cfg.k)

    def run(self, S: int) -> float:
        cfg, o, sel = self.cfg, self.o, self.sel
        xs = np.ascontiguousarray(self.x[:, :S])
        t0 = time.perf_counter()
        codes, side = o.quantize_pack(xs, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
        o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
        return time.perf_counter() - t0


def host_rows(cfg, S, device=None):
    """Rows [0, S) of the evaluation batch for all ranks (from the GPU generator when a GPU is
    present -- the same values as the host generator -- else from the host generator)."""
    cs, _ = synth.colscale(cfg)
    if device is not None:
        import torch

        buf = torch.empty((cfg.P, cfg.T, cfg.H), dtype=torch.int16, device=device)
        synth.fill_gpu(cfg, synth.EVAL, 0, buf, torch.from_numpy(cs).to(device))
        out = buf[:, :S].cpu().numpy().view(np.uint16).copy()
        del buf
        return out
    return synth.fill_cpu(cfg, synth.EVAL, 0, rows=(0, S), cs=cs)


def cpu_rows_for(step: OracleStep, seconds: float, cap: int) -> tuple[int, float]:
    """Rows per oracle step so that one step takes about `seconds`."""
    probe = min(cap, 8)
    dt = step.run(probe)
    per_row = max(dt / probe, 1e-7)
    return max(1, min(cap, int(seconds / per_row))), per_row


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return
    budget = 150.0  # seconds for the whole --steps/--warmup run
    cap = min(cfg.T, 4096)
    x = host_rows(cfg, cap)
    step = OracleStep(cfg, x)
    S, per_row = cpu_rows_for(step, budget / max(1, args.steps + args.warmup), cap)
    for _ in range(args.warmup):
        step.run(S)
    t = sum(step.run(S) for _ in range(args.steps))
    part_bytes = cfg.P * S * cfg.H * 2
    value = part_bytes * args.steps / t / 1e9
    sample = (f"rows 0..{S - 1} of the evaluation batch, all {cfg.P} ranks, per step "
              f"(quantize-pack + dequant-reduce), single thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": describe(cfg), "P": cfg.P, "T": cfg.T, "H": cfg.H, "k": cfg.k,
                   "path": "split", "step": "quantize_pack+dequant_reduce", "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "host_cpus": os.cpu_count(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "compression_ratio": compression_ratio(cfg),
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------------------------
# The source files each kernel is compiled from (its own header plus what it includes).
KERNEL_SOURCES = {
    "calibrate": ["k_calibrate.cuh", "hq_common.cuh"],
    "select": ["k_select.cuh", "hq_common.cuh"],
    "quantize_pack": ["k_quantize.cuh", "hq_common.cuh", "hq_tma.cuh"],
    "dequant_reduce": ["k_dequant.cuh", "hq_common.cuh", "hq_tma.cuh"],
    "compress_reduce": ["k_fused.cuh", "k_dequant.cuh", "hq_common.cuh", "hq_tma.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources of one kernel and of the launch code in hq_api.cu."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_tensor_activation_b200", "csrc")
    for f in sorted(KERNEL_SOURCES[kernel]) + ["hq_api.cu"]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM traffic per launch recorded by an ncu capture of the same kernel source, else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(f"{kernel}@{workload}")
        if e and e.get("source_hash") == kernel_source_hash(kernel):
            return e["bytes_per_launch"]
    except Exception:
        pass
    return None


def _kernel_entry(nbytes, t_ms, peak):
    gbs = nbytes / (t_ms * 1e-3) / 1e9
    return {"us": 1e3 * t_ms, "bytes": nbytes, "GB/s": gbs, "frac": gbs / peak, "frac_nominal": gbs / NOMINAL_HBM_GBS}


class Workload:
    """One workload resident on the GPU: calibration state and parameters (offline), the
    evaluation batch x, and the wire and output buffers."""

    def __init__(self, cfg, dev):
        import torch

        import bit_tensor_activation_b200 as hq

        self.hq, self.cfg, self.dev = hq, cfg, dev
        P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
        cs, _ = synth.colscale(cfg)
        cs_dev = torch.from_numpy(cs).to(dev)
        self.B = hq.Buffers(P, T, H, k, device=dev)
        self.cal = torch.empty((P, cfg.calib_T, H), dtype=torch.int16, device=dev)
        for b in range(cfg.calib_batches):
            synth.fill_gpu(cfg, synth.CALIB, b, self.cal, cs_dev, T=cfg.calib_T)
            hq.hq_calibrate(self.cal, self.B.ema_min, self.B.ema_max, cfg.beta, b == 0)
        self.select()
        self.x = torch.empty((P, T, H), dtype=torch.int16, device=dev)
        synth.fill_gpu(cfg, synth.EVAL, 0, self.x, cs_dev)
        self.fused_out = torch.empty_like(self.B.out)
        torch.cuda.synchronize()

    # offline calls (once per calibration)
    def calibrate(self):
        self.hq.hq_calibrate(self.cal, self.B.ema_min, self.B.ema_max, self.cfg.beta, False)

    def select(self):
        B = self.B
        self.hq.hq_select_topk(B.ema_min, B.ema_max, self.cfg.k, B.keep_idx, B.rest_idx, B.scale, B.inv_scale,
                               B.zero)

    # online calls (every batch)
    def quantize_pack(self, xin=None):
        B = self.B
        self.hq.hq_quantize_pack(self.x if xin is None else xin, B.keep_idx, B.rest_idx, B.inv_scale, B.zero,
                                 B.codes, B.side)

    def dequant_reduce(self, res=None):
        B = self.B
        self.hq.hq_dequant_reduce(B.codes, B.side, B.keep_idx, B.rest_idx, B.scale, B.zero,
                                  B.out if res is None else res)

    def compress_reduce(self, xin=None, res=None):
        B = self.B
        self.hq.hq_compress_reduce(self.x if xin is None else xin, B.keep_idx, B.rest_idx, B.scale, B.inv_scale,
                                   B.zero, self.fused_out if res is None else res)

    def step_calls(self, path, xin=None, res=None):
        if path == "split":
            return [("quantize_pack", lambda: self.quantize_pack(xin)), ("dequant_reduce", lambda: self.dequant_reduce(res))]
        return [("compress_reduce", lambda: self.compress_reduce(xin, res))]


def time_steps(W: Workload, path, K, warmup, stream):
    """K steps back to back with an event before every call: (total ms, {kernel: mean ms})."""
    import torch

    calls = W.step_calls(path)
    for _ in range(warmup):
        for _, c in calls:
            c()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in calls] for _ in range(K)]
    ev.append([torch.cuda.Event(enable_timing=True)])
    torch.cuda.synchronize()
    for i in range(K):
        for j, (_, c) in enumerate(calls):
            ev[i][j].record(stream)
            c()
    ev[K][0].record(stream)
    torch.cuda.synchronize()
    per = {}
    for j, (n, _) in enumerate(calls):
        nxt = (lambda i: ev[i][j + 1]) if j + 1 < len(calls) else (lambda i: ev[i + 1][0])
        per[n] = sum(ev[i][j].elapsed_time(nxt(i)) for i in range(K)) / K
    return ev[0][0].elapsed_time(ev[K][0]), per


def time_cold(fns, reps, stream, flush):
    """Each call timed alone, the L2 flushed (a write larger than L2) before every launch: mean ms."""
    import torch

    out = {}
    for n, f in fns:
        f()  # warm the launch path
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            f()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        out[n] = tot / reps
    return out


def measure_workload(W: Workload, K, warmup, cold_reps, stream, flush, peak):
    """Split and fused steps, per-kernel times in the step and cold, offline calls cold."""
    cfg = W.cfg
    ab = algo_bytes(cfg)
    part = cfg.P * cfg.T * cfg.H * 2
    ms_s, per_s = time_steps(W, "split", K, warmup, stream)
    ms_f, per_f = time_steps(W, "fused", max(3, K // 2), warmup, stream)
    cold = time_cold([("quantize_pack", W.quantize_pack), ("dequant_reduce", W.dequant_reduce),
                      ("compress_reduce", W.compress_reduce)], cold_reps, stream, flush)
    off = time_cold([("calibrate", W.calibrate), ("select", W.select)], max(3, cold_reps // 4), stream, flush)
    return {
        "split_ms": ms_s / K, "fused_ms": ms_f / max(3, K // 2),
        "value": part / (ms_s / K * 1e-3) / 1e9,
        "fused_value": part / (ms_f / max(3, K // 2) * 1e-3) / 1e9,
        "kernels": {n: _kernel_entry(ab[n], t, peak) for n, t in per_s.items()},
        "fused_kernel": {n: _kernel_entry(ab[n], t, peak) for n, t in per_f.items()},
        "kernels_cold": {n: _kernel_entry(ab[n], t, peak) for n, t in cold.items()},
        "offline": {n: _kernel_entry(ab[n], t, peak) for n, t in off.items()},
    }


def measure_next(W: Workload, reps, stream, flush, peak):
    """The next stages on the same workload, each timed with the L2 flushed before every call:
    the two-step all-reduce on one GPU (step 1 = the split path, step 2 = the reducers' blocks
    re-quantized and dequantized one by one), partial-channel synchronisation of the first half
    of the features (the _ld calls on the column block), and the reduction over one wire buffer
    per rank against the stacked buffer."""
    import torch

    import bit_tensor_activation_b200 as hq
    from bit_tensor_activation_b200 import exchange as ex

    cfg, B, dev = W.cfg, W.B, W.dev
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    res = {}
    params = ex.HybridParams(B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero)
    part = P * T * H * 2

    # two-step: step-2 grids from two calibration batches through step 1
    k2 = k
    cs_dev = torch.from_numpy(synth.colscale(cfg)[0]).to(dev)
    cal = []
    for b in range(2):
        c = torch.empty((P, T, H), dtype=torch.int16, device=dev)
        synth.fill_gpu(cfg, synth.CALIB, 100 + b, c, cs_dev)
        cal.append(c.view(torch.bfloat16))
    p2 = ex.step_two_params_simulated(cal, params, k2, cfg.beta)
    del cal
    Tb = T // P
    out1 = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    out2 = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    codes2 = torch.empty((P, Tb, (H - k2) // 8), dtype=torch.int32, device=dev)
    side2 = torch.empty((P, k2, Tb), dtype=torch.bfloat16, device=dev)
    x = W.x.view(torch.bfloat16)

    ws = torch.empty(hq.hq_two_step_workspace_bytes(P, T, H, k, k2), dtype=torch.uint8, device=dev)

    def two_step():
        hq.hq_two_step_reduce(x, params.keep_idx, params.rest_idx, params.scale, params.inv_scale, params.zero,
                              p2.keep_idx, p2.rest_idx, p2.scale, p2.inv_scale, p2.zero, ws, out2)

    def step1():  # the library call's first two launches: every rank's wire, reduced to bf16
        hq.hq_quantize_pack(x, params.keep_idx, params.rest_idx, params.inv_scale, params.zero, B.codes, B.side)
        hq.hq_dequant_reduce(B.codes, B.side, params.keep_idx, params.rest_idx, params.scale, params.zero, out1)

    t = time_cold([("two_step", two_step), ("step1", step1)], reps, stream, flush)
    ex.two_step_simulated(x, params, p2, out1, B.out, B.codes, B.side, codes2, side2)
    hq.hq_two_step_reduce(x, params.keep_idx, params.rest_idx, params.scale, params.inv_scale, params.zero,
                          p2.keep_idx, p2.rest_idx, p2.scale, p2.inv_scale, p2.zero, ws, out2)
    torch.cuda.synchronize()
    same = bool(torch.equal(out2.view(torch.int16), B.out.view(torch.int16)))
    del ws
    res["two_step"] = {"call": "hq_two_step_reduce", "equals_python_composition": same,
                       "ms_per_step": t["two_step"], "value": part / (t["two_step"] * 1e-3) / 1e9, "unit": "GB/s",
                       "step2_us": 1e3 * (t["two_step"] - t["step1"]), "launches_per_step": 4,
                       "step2_wire_bytes_per_reducer": Tb * ((H - k2) // 2 + 2 * k2)}

    # partial-channel synchronisation of features [0, H/2)
    Hs = H // 2
    ks = k // 2
    emin = torch.empty((P, Hs), dtype=torch.float32, device=dev)
    emax = torch.empty_like(emin)
    hq.hq_calibrate_ld(W.x[:, :, :Hs], emin, emax, cfg.beta, True)
    Bs = hq.Buffers(P, T, Hs, ks, device=dev)
    hq.hq_select_topk(emin, emax, ks, Bs.keep_idx, Bs.rest_idx, Bs.scale, Bs.inv_scale, Bs.zero)
    outp = torch.empty((T, H), dtype=torch.bfloat16, device=dev)

    def partial():
        hq.hq_quantize_pack_ld(W.x[:, :, :Hs], Bs.keep_idx, Bs.rest_idx, Bs.inv_scale, Bs.zero, Bs.codes, Bs.side)
        hq.hq_dequant_reduce_ld(Bs.codes, Bs.side, Bs.keep_idx, Bs.rest_idx, Bs.scale, Bs.zero, outp[:, :Hs])

    t = time_cold([("partial", partial)], reps, stream, flush)
    sync_bytes = P * T * Hs * 2
    res["partial_sync"] = {"features_synced": Hs, "kept": ks, "ms_per_step": t["partial"],
                           "value": sync_bytes / (t["partial"] * 1e-3) / 1e9, "unit": "GB/s of synchronised partial sums",
                           "wire_bytes_per_rank_row": hq.hq_wire_bytes_per_row(Hs, ks),
                           "full_wire_bytes_per_rank_row": hq.hq_wire_bytes_per_row(H, k)}

    # the reduction over one wire buffer per rank (what a rank reading its peers in place runs)
    W.quantize_pack()
    cl = [B.codes[r].clone() for r in range(P)]
    sl = [B.side[r].clone() for r in range(P)]
    outr = torch.empty_like(B.out)

    def ranks():
        hq.hq_dequant_reduce_ranks(cl, sl, B.keep_idx, B.rest_idx, B.scale, B.zero, outr)

    t = time_cold([("ranks", ranks), ("stacked", W.dequant_reduce)], reps, stream, flush)
    ab = algo_bytes(cfg)["dequant_reduce"]
    torch.cuda.synchronize()
    res["ranks"] = {"per_rank_buffers": _kernel_entry(ab, t["ranks"], peak), "stacked": _kernel_entry(ab, t["stacked"], peak),
                    "equal": bool(torch.equal(outr.view(torch.int16), B.out.view(torch.int16)))}
    return res


def run_hq(args, cfg, world, rank, local):
    import torch

    import bit_tensor_activation_b200 as hq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    peak, peak_src = measured_peak()
    ab = algo_bytes(cfg)
    part_bytes = P * T * H * 2
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    W = Workload(cfg, dev)
    names = [n for n, _ in W.step_calls(args.path)]
    calls = W.step_calls(args.path)
    for _ in range(args.warmup):
        for _, c in calls:
            c()
    torch.cuda.synchronize()
    st = hq.hq_read_device_error()
    if st != hq.HQ_OK:
        raise RuntimeError(f"device error after warm-up: {hq.hq_status_string(st)}")

    # ---- the timed steps: inputs resident in HBM, larger than L2 ------------------------------------
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in calls] for _ in range(K)]
    ev.append([torch.cuda.Event(enable_timing=True)])
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(local, not args.no_clocks)
    time.sleep(0.3 if not args.no_clocks else 0.0)
    wall0 = time.perf_counter()
    for i in range(K):
        for j, (_, c) in enumerate(calls):
            ev[i][j].record(stream)
            c()
    ev[K][0].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    barrier(world)
    ms_local = ev[0][0].elapsed_time(ev[K][0])
    ms = max_over_ranks(ms_local, world, dev)
    per_kernel = {}
    for j, n in enumerate(names):
        nxt = (lambda i: ev[i][j + 1]) if j + 1 < len(names) else (lambda i: ev[i + 1][0])
        per_kernel[n] = sum(ev[i][j].elapsed_time(nxt(i)) for i in range(K)) / K  # ms per launch

    # ---- each kernel alone with a cold L2, the alternate path, the offline calls --------------------
    Ka = max(3, min(K, 400))
    alt_path = "fused" if args.path == "split" else "split"
    ms_alt, per_alt = time_steps(W, alt_path, Ka, 3, stream)
    cold = time_cold([("quantize_pack", W.quantize_pack), ("dequant_reduce", W.dequant_reduce),
                      ("compress_reduce", W.compress_reduce)], args.cold_reps, stream, flush)
    offline = time_cold([("calibrate", W.calibrate), ("select", W.select)], max(3, args.cold_reps // 4), stream,
                        flush)
    W.select()  # the parameters the checks below use
    nxt = measure_next(W, max(3, args.cold_reps // 2), stream, flush, peak) if args.next_paths else None

    # ---- fused output equals split output on this workload -------------------------------------------
    W.quantize_pack()
    W.dequant_reduce()
    W.compress_reduce()
    fused_equal = bool(torch.equal(W.B.out.view(torch.int16), W.fused_out.view(torch.int16)))

    # ---- e2e: public API with pinned host buffers, copies inside the timed region ----------------
    # Every step copies its input from pinned host memory and its result back, inside the timed
    # region. Steps are pipelined the way a serving loop would run them: the next step's input
    # copy (its own stream) overlaps this step's compute and result copy (a third stream), with
    # two device input and result buffers and events ordering every reuse.
    e2e = None
    if args.e2e_steps > 0:
        x = W.x
        xh = x.cpu().pin_memory()
        xd = [torch.empty_like(x) for _ in range(2)]
        res = [torch.empty_like(W.B.out) for _ in range(2)]
        oh = [torch.empty(r.shape, dtype=r.dtype).pin_memory() for r in res]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        copied_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(computed[b])  # step i-2 is done with xd[b]
                    xd[b].copy_(xh, non_blocking=True)
                    in_ready[b].record(s_in)
                stream.wait_event(in_ready[b])
                if i >= 2:
                    stream.wait_event(copied_out[b])  # step i-2's result has left res[b]
                for _, call in W.step_calls(args.path, xd[b], res[b]):
                    call()
                computed[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(computed[b])
                    oh[b].copy_(res[b], non_blocking=True)
                    copied_out[b].record(s_out)

        e2e_steps(2)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        e2e_steps(args.e2e_steps)
        tail = torch.cuda.Event()
        tail.record(s_out)
        stream.wait_event(tail)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
        e2e = {"value": world * part_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": oh[0].numel() * oh[0].element_size(), "ms_per_step": e2e_ms,
               "pipelined": "next step's input copy overlaps this step's compute and result copy"}
        # the last copied-back result against the device-resident reduction of the same input
        torch.cuda.synchronize()
        check = W.B.out if args.path == "split" else W.fused_out
        if not torch.equal(oh[(args.e2e_steps - 1) & 1].view(torch.int16).to(dev), check.view(torch.int16)):
            raise RuntimeError("the end-to-end result differs from the device-resident reduction")
        del xh, xd, res, oh

    st = hq.hq_read_device_error()
    if st != hq.HQ_OK:
        raise RuntimeError(f"device error: {hq.hq_status_string(st)}")

    # ---- the second large workload, same run (per-kernel figures for the bandwidth target) -------
    workloads = {}
    second = SECOND_WORKLOAD.get(cfg.name)
    if second and args.second_steps > 0 and world == 1:
        del W
        torch.cuda.empty_cache()
        cfg2 = workload(second)
        W2 = Workload(cfg2, dev)
        m = measure_workload(W2, args.second_steps, 5, args.cold_reps, stream, flush, peak)
        m["config"] = describe(cfg2)
        m["compression_ratio"] = compression_ratio(cfg2)
        workloads[second] = m
        st = hq.hq_read_device_error()
        if st != hq.HQ_OK:
            raise RuntimeError(f"device error ({second}): {hq.hq_status_string(st)}")
        del W2
    # the two small workloads (launch-bound: reported for coverage of every configuration)
    if args.small_steps > 0 and world == 1:
        for small in ("decode", "pr1"):
            if small == cfg.name:
                continue
            cfg3 = workload(small)
            W3 = Workload(cfg3, dev)
            m = measure_workload(W3, args.small_steps, 5, args.cold_reps, stream, flush, peak)
            m["config"] = describe(cfg3)
            m["compression_ratio"] = compression_ratio(cfg3)
            m["elements_per_s"] = cfg3.P * cfg3.T * cfg3.H / (m["split_ms"] * 1e-3)
            workloads[small] = m
            st = hq.hq_read_device_error()
            if st != hq.HQ_OK:
                raise RuntimeError(f"device error ({small}): {hq.hq_status_string(st)}")
            del W3

    # ---- CPU baseline (rank 0, N = 1) -----------------------------------------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cap = min(T, 2048)
        step = OracleStep(cfg, host_rows(cfg, cap, dev))
        S, _ = cpu_rows_for(step, args.cpu_seconds, cap)
        t = step.run(S)
        reps = max(1, round(args.cpu_seconds / t))
        t += sum(step.run(S) for _ in range(reps - 1))
        cpu = {"value": reps * P * S * H * 2 / t / 1e9, "unit": "GB/s", "cores": 1, "host_cpus": os.cpu_count(),
               "kind": "oracle",
               "sample": f"rows 0..{S - 1} of the evaluation batch, all {P} ranks, {reps} passes of quantize-pack + "
                         f"dequant-reduce (parameters calibrated and selected once), {t:.1f} s single-threaded"}

    if rank != 0:
        return
    kernels = {n: _kernel_entry(ab[n], t_ms, peak) for n, t_ms in per_kernel.items()}
    dominant = max(per_kernel, key=per_kernel.get)
    dom_gbs = kernels[dominant]["GB/s"]
    step_bytes = sum(ab[n] for n in names)
    value = world * part_bytes * K / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": describe(cfg), "P": P, "T": T, "H": H, "k": k, "path": args.path,
                   "step": "+".join(names),
                   "offline": "calibrate + select run once per calibration; timed alone under 'offline'",
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2 ({part_bytes / 2**20:.0f} MiB of partial sums per step), no flush"
                   if part_bytes > L2_BYTES else "inputs smaller than L2 (L2-resident between steps)"},
        "hbm_frac_step": step_bytes * K / (ms_local * 1e-3) / 1e9 / peak,
        "compression_ratio": compression_ratio(cfg),
        "elements_per_s": world * P * T * H * K / (ms * 1e-3),
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": dom_gbs, "peak": peak, "unit": "GB/s",
                     "frac": dom_gbs / peak, "traffic": ncu_traffic(dominant, cfg.name), "peak_source": peak_src,
                     "bytes_per_launch": ab[dominant], "frac_nominal": dom_gbs / NOMINAL_HBM_GBS,
                     "nominal_peak": NOMINAL_HBM_GBS},
        "kernels": kernels,
        "kernels_cold": {n: _kernel_entry(ab[n], t_ms, peak) for n, t_ms in cold.items()},
        "offline": {n: _kernel_entry(ab[n], t_ms, peak) for n, t_ms in offline.items()},
        "alt_paths": {alt_path: {"ms_per_step": ms_alt / Ka, "value": part_bytes / (ms_alt / Ka * 1e-3) / 1e9,
                                 "kernel_ms": per_alt}},
        "workloads": workloads,
        "next": nxt,
        "fused_equals_split": fused_equal,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": len(names) * K,
        "clocks": clk,
        "wall_s_timed": wall,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    cfg = workload(args.workload)
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, cfg, world, rank)
        else:
            run_hq(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
