"""Bandwidth against size over the sweep workloads: uniform U(-1,1) partial sums for
P in {2,4,8}, H in {4096,8192}, T in {1,64,512,4096,16384}, k/H in {0, 1/64, 1/32}.

For every point the inputs are generated on the GPU and calibrated with 8 batches of 256 rows.
Then quantize-pack, dequant-reduce (bf16 output) and compress-reduce are each timed.

- Timing: CUDA events, median of --reps launches after 3 warm-up launches.
- L2: before each timed launch, a buffer larger than L2 is written and then read, so every launch
  starts from a clean, cold L2.
- Output: each kernel's algorithmic bytes (inputs read once, outputs written once, parameters
  included) per second, and that figure over the measured copy bandwidth.

    python sweep.py --out sweep.md [--reps 10] [--json sweep.json]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bit_tensor_activation_b200 as hq  # noqa: E402
import synth  # noqa: E402


def algo_bytes(P: int, T: int, H: int, k: int) -> dict:
    Hr = H - k
    return {
        "quantize_pack": 2 * P * T * H + P * T * Hr // 2 + 2 * P * T * k + 5 * P * H + 4 * H,
        "dequant_reduce": P * T * Hr // 2 + 2 * P * T * k + 2 * T * H + 5 * P * H + 4 * H,
        "compress_reduce": 2 * P * T * H + 2 * T * H + 9 * P * H + 4 * H,
    }


def peak_gbs() -> float:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return 6650.0


def run_point(cfg: synth.Config, reps: int, flush: torch.Tensor) -> dict:
    dev = torch.device("cuda")
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    cs, _ = synth.colscale(cfg)
    cs_dev = torch.from_numpy(cs).to(dev)
    B = hq.Buffers(P, T, H, k, device=dev)
    cal = torch.empty((P, cfg.calib_T, H), dtype=torch.int16, device=dev)
    for b in range(cfg.calib_batches):
        synth.fill_gpu(cfg, synth.CALIB, b, cal, cs_dev, T=cfg.calib_T)
        hq.hq_calibrate(cal, B.ema_min, B.ema_max, cfg.beta, b == 0)
    del cal
    hq.hq_select_topk(B.ema_min, B.ema_max, k, B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero)
    x = torch.empty((P, T, H), dtype=torch.int16, device=dev)
    synth.fill_gpu(cfg, synth.EVAL, 0, x, cs_dev)
    fused = torch.empty_like(B.out)
    calls = {
        "quantize_pack": lambda: hq.hq_quantize_pack(x, B.keep_idx, B.rest_idx, B.inv_scale, B.zero, B.codes, B.side),
        "dequant_reduce": lambda: hq.hq_dequant_reduce(B.codes, B.side, B.keep_idx, B.rest_idx, B.scale, B.zero, B.out),
        "compress_reduce": lambda: hq.hq_compress_reduce(x, B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero, fused),
    }
    ab = algo_bytes(P, T, H, k)
    res = {}
    for name, call in calls.items():
        for _ in range(3):
            call()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            flush.sum()  # leaves L2 holding clean lines of the flush buffer
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        us = statistics.median(ts)
        res[name] = {"us": us, "bytes": ab[name], "GB/s": ab[name] / us / 1e3}
    st = hq.hq_read_device_error()
    if st != hq.HQ_OK:
        raise RuntimeError(f"{cfg.name}: device error {hq.hq_status_string(st)}")
    return res


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default="sweep.md")
    ap.add_argument("--json", default=None)
    ap.add_argument("--reps", type=int, default=10)
    args = ap.parse_args()
    peak = peak_gbs()
    flush = torch.empty(512 * 2**20 // 4, dtype=torch.int32, device="cuda")
    rows, records = [], []
    for cfg in synth.sweep_configs():
        r = run_point(cfg, args.reps, flush)
        records.append({"name": cfg.name, "P": cfg.P, "T": cfg.T, "H": cfg.H, "k": cfg.k, **r})
        cells = [f"{r[n]['us']:.1f} µs, {r[n]['GB/s']:.0f} GB/s ({r[n]['GB/s'] / peak:.2f})"
                 for n in ("quantize_pack", "dequant_reduce", "compress_reduce")]
        mb = r["quantize_pack"]["bytes"] / 1e6
        rows.append(f"| {cfg.P} | {cfg.H} | {cfg.T} | {cfg.k} | {mb:.1f} | " + " | ".join(cells) + " |")
        print(rows[-1], flush=True)
    with open(args.out, "w") as f:
        f.write(f"Fractions are of the measured copy bandwidth, {peak:.1f} GB/s. Every launch starts from a "
                f"clean, cold L2; median of {args.reps} launches.\n\n")
        f.write("| P | H | T | k | quantize bytes (MB) | quantize_pack | dequant_reduce (bf16) | compress_reduce |\n")
        f.write("|---|---|---|---|---|---|---|---|\n")
        f.write("\n".join(rows) + "\n")
    if args.json:
        with open(args.json, "w") as f:
            json.dump({"peak_gbs": peak, "points": records}, f, indent=1)


if __name__ == "__main__":
    main()
