"""Selection ablation: the error each choice of BF16 features leaves in the reduced sum, and the
cost of rounding every rank's dequantized shard to bf16 before the sum.

The page "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication" (section
"Key Observations and Future Directions") reports that choosing the BF16 features by their
aggregated quantization range works much better than choosing them at random.  This tool
measures that on the synthetic workloads, through the CUDA path only:

- calibration and selection run on the GPU (``hq_calibrate``, ``hq_select_topk``);
- each variant then runs quantize-pack and a reduction, with fp32 output, on the same
  evaluation batch;
- the result is compared with the exact sum of the bf16 partial sums, taken in fp64.

Variants:

- ``topk``: the k features with the largest summed ranges, with the default reduction (one FMA
  per rank).
- ``topk_bf16_shards``: the same features, with each rank's dequantized value rounded to bf16
  before it is added (``hq_dequant_reduce_bf16_shards``, the literal reading of the page's
  inference step).
- ``random_k``: k features drawn uniformly with a fixed seed.  The 4-bit grids are the same,
  because they are computed for every feature.
- ``int4_only``: k = 0.
- ``bf16_only``: k = H, the uncompressed bf16 wire; only the fp32 summation remains.
- ``two_step``: the two-step compressed all-reduce of ``bit_tensor_activation_b200.exchange``
  (reduce-scatter, then all-gather), the scheme the "Flash Communication" abstract among the
  source pages names without an algorithm: step 1 is the ``topk`` path with bf16 output, and
  reducer j owns row block j of it; in step 2 each reducer quantizes its block again with its
  own grid (calibrated on its reduced calibration blocks; one kept set selected over the
  reducers' statistics) and every block is dequantized with its reducer's grid. On one GPU the
  P blocks are handled one by one, a P = 1 quantize-pack and dequant-reduce each; the time
  reported is step 2's.

For every variant the tool reports MSE, MSE relative to the mean square of the exact sum, the
largest absolute error and the wire compression ratio.  It also times the variant's reduction:
CUDA events, median of --reps launches, with a buffer larger than L2 written and read before
each launch.

    python ablation.py [--workloads decode,prefill7b,prefill70b] [--out ablation.md] [--json a.json]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bit_tensor_activation_b200 as hq  # noqa: E402
import synth  # noqa: E402

VARIANTS = ("topk", "topk_bf16_shards", "random_k", "int4_only", "bf16_only", "two_step")


def peak_gbs() -> float:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return 6650.0


def reduce_bytes(P: int, T: int, H: int, k: int) -> int:
    """Algorithmic bytes of one reduction with fp32 output: wire read once, output written once,
    parameters included."""
    return P * T * (H - k) // 2 + 2 * P * T * k + 4 * T * H + 5 * P * H + 4 * H


def timed_us(call, reps: int, flush: torch.Tensor) -> float:
    for _ in range(3):
        call()
    ts = []
    for _ in range(reps):
        flush.fill_(1)
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    return statistics.median(ts)


def run_workload(cfg: synth.Config, reps: int, flush: torch.Tensor, seed: int) -> list[dict]:
    dev = torch.device("cuda")
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    cs, _ = synth.colscale(cfg)
    cs_dev = torch.from_numpy(cs).to(dev)
    ema_min = torch.empty((P, H), dtype=torch.float32, device=dev)
    ema_max = torch.empty_like(ema_min)
    cal = torch.empty((P, cfg.calib_T, H), dtype=torch.int16, device=dev)
    for b in range(cfg.calib_batches):
        synth.fill_gpu(cfg, synth.CALIB, b, cal, cs_dev, T=cfg.calib_T)
        hq.hq_calibrate(cal, ema_min, ema_max, cfg.beta, b == 0)
    del cal
    keep = torch.empty(k, dtype=torch.int32, device=dev)
    rest = torch.empty(H - k, dtype=torch.int32, device=dev)
    scale = torch.empty((P, H), dtype=torch.float32, device=dev)
    inv = torch.empty_like(scale)
    zero = torch.empty((P, H), dtype=torch.uint8, device=dev)
    hq.hq_select_topk(ema_min, ema_max, k, keep, rest, scale, inv, zero)
    x = torch.empty((P, T, H), dtype=torch.int16, device=dev)
    synth.fill_gpu(cfg, synth.EVAL, 0, x, cs_dev)

    exact = torch.zeros((T, H), dtype=torch.float64, device=dev)
    for r in range(P):
        exact += x[r].view(torch.bfloat16).double()
    mean_sq = float((exact * exact).mean())

    rng = np.random.default_rng(seed)
    rand_keep = np.sort(rng.choice(H, k, replace=False)).astype(np.int32)
    sets = {
        "topk": (keep, rest),
        "random_k": (torch.from_numpy(rand_keep).to(dev),
                     torch.from_numpy(np.setdiff1d(np.arange(H), rand_keep).astype(np.int32)).to(dev)),
        "int4_only": (torch.empty(0, dtype=torch.int32, device=dev), torch.arange(H, dtype=torch.int32, device=dev)),
        "bf16_only": (torch.arange(H, dtype=torch.int32, device=dev), torch.empty(0, dtype=torch.int32, device=dev)),
    }
    out = torch.empty((T, H), dtype=torch.float32, device=dev)
    rows = []
    for name in VARIANTS:
        if name == "two_step":
            rows.append(two_step(cfg, x, exact, mean_sq, keep, rest, scale, inv, zero, cs_dev, reps, flush))
            continue
        kk, rr = sets["topk" if name == "topk_bf16_shards" else name]
        kn = kk.shape[0]
        codes = torch.empty((P, T, (H - kn) // 8), dtype=torch.int32, device=dev)
        side = torch.empty((P, kn, T), dtype=torch.int16, device=dev)
        hq.hq_quantize_pack(x, kk, rr, inv, zero, codes, side)
        fn = hq.hq_dequant_reduce_bf16_shards if name == "topk_bf16_shards" else hq.hq_dequant_reduce

        def call(fn=fn, codes=codes, side=side, kk=kk, rr=rr):
            fn(codes, side, kk, rr, scale, zero, out)

        us = timed_us(call, reps, flush)
        call()
        err = out.double() - exact
        mse = float((err * err).mean())
        rows.append({
            "workload": cfg.name, "variant": name, "k": kn, "mse": mse, "rel_mse": mse / mean_sq,
            "max_abs_err": float(err.abs().max()), "ratio": 2 * H / ((H - kn) / 2 + 2 * kn),
            "reduce_us": us, "reduce_gbs": reduce_bytes(P, T, H, kn) / us / 1e3,
        })
        del codes, side
    st = hq.hq_read_device_error()
    if st != hq.HQ_OK:
        raise RuntimeError(f"{cfg.name}: device error {hq.hq_status_string(st)}")
    return rows


def two_step(cfg, x, exact, mean_sq, keep, rest, scale, inv, zero, cs_dev, reps, flush) -> dict:
    """The two-step all-reduce of the exchange module on one GPU: step 1 is the hybrid reduction;
    in step 2 every reducer re-quantizes its row block with its own grid (calibrated on its
    reduced calibration blocks) and the blocks are dequantized one by one."""
    from bit_tensor_activation_b200 import exchange as ex

    dev = x.device
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    params = ex.HybridParams(keep, rest, scale, inv, zero)

    def cal_batches():
        cal = torch.empty((P, cfg.calib_T, H), dtype=torch.int16, device=dev)
        for b in range(cfg.calib_batches):
            synth.fill_gpu(cfg, synth.CALIB, b, cal, cs_dev, T=cfg.calib_T)
            yield cal.view(torch.bfloat16)

    p2 = ex.step_two_params_simulated(cal_batches(), params, k, cfg.beta)
    Tb = T // P
    out1 = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, H), dtype=torch.float32, device=dev)
    codes = torch.empty((P, T, (H - k) // 8), dtype=torch.int32, device=dev)
    side = torch.empty((P, k, T), dtype=torch.bfloat16, device=dev)
    codes2 = torch.empty((P, Tb, (H - k) // 8), dtype=torch.int32, device=dev)
    side2 = torch.empty((P, k, Tb), dtype=torch.bfloat16, device=dev)
    xb = x.view(torch.bfloat16)
    ex.two_step_simulated(xb, params, p2, out1, out, codes, side, codes2, side2)

    def step2():
        for j in range(P):
            rows = slice(j * Tb, (j + 1) * Tb)
            hq.hq_quantize_pack(out1[rows].unsqueeze(0), p2.keep_idx, p2.rest_idx, p2.inv_scale[j:j + 1],
                                p2.zero[j:j + 1], codes2[j:j + 1], side2[j:j + 1])
            hq.hq_dequant_reduce(codes2[j:j + 1], side2[j:j + 1], p2.keep_idx, p2.rest_idx, p2.scale[j:j + 1],
                                 p2.zero[j:j + 1], out[rows])

    us = timed_us(step2, reps, flush)
    step2()
    err = out.double() - exact
    mse = float((err * err).mean())
    step2_bytes = (2 * T * H + T * (H - k) // 2 + 2 * T * k) + (T * (H - k) // 2 + 2 * T * k + 4 * T * H)
    return {"workload": cfg.name, "variant": "two_step", "k": k, "mse": mse, "rel_mse": mse / mean_sq,
            "max_abs_err": float(err.abs().max()), "ratio": 2 * H / ((H - k) / 2 + 2 * k),
            "reduce_us": us, "reduce_gbs": step2_bytes / us / 1e3}


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default="decode,prefill7b,prefill70b")
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--seed", type=int, default=5, help="seed of the random-k feature draw")
    ap.add_argument("--out", default=None)
    ap.add_argument("--json", default=None)
    args = ap.parse_args()
    peak = peak_gbs()
    flush = torch.empty(512 * 2**20 // 4, dtype=torch.int32, device="cuda")
    lines = ["| workload | variant | k | compression | MSE | MSE / mean square of the sum | max abs error | "
             "reduce µs (fp32 out) | GB/s (fraction of measured HBM) |",
             "|---|---|---|---|---|---|---|---|---|"]
    records = []
    for name in args.workloads.split(","):
        for r in run_workload(synth.CONFIGS[name], args.reps, flush, args.seed):
            records.append(r)
            lines.append(f"| {r['workload']} | {r['variant']} | {r['k']} | {r['ratio']:.3f} | {r['mse']:.4g} | "
                         f"{r['rel_mse']:.3g} | {r['max_abs_err']:.4g} | {r['reduce_us']:.1f} | "
                         f"{r['reduce_gbs']:.0f} ({r['reduce_gbs'] / peak:.2f}) |")
            print(lines[-1], flush=True)
    if args.out:
        with open(args.out, "w") as f:
            f.write("\n".join(lines) + "\n")
    if args.json:
        with open(args.json, "w") as f:
            json.dump({"peak_gbs": peak, "rows": records}, f, indent=1)


if __name__ == "__main__":
    main()
