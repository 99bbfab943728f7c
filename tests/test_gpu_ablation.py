"""The selection ablation (ablation.py) through the CUDA path, on the decode workload.

The page "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication" (section
"Key Observations and Future Directions") finds that choosing the BF16 features by their
quantization range beats a random choice.  These are properties of the measured errors, not
bit-exact values: top-k must beat random k by a wide margin, random k must be about as bad as
no BF16 features at all, keeping every feature must leave only the fp32 summation error, and
rounding each rank's shard to bf16 must change the error only slightly.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import ablation  # noqa: E402


def test_selection_ablation_decode():
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.int32, device="cuda")
    rows = {r["variant"]: r for r in ablation.run_workload(synth.CONFIGS["decode"], 3, flush, seed=5)}
    assert set(rows) == set(ablation.VARIANTS)
    top, rnd, int4 = rows["topk"]["rel_mse"], rows["random_k"]["rel_mse"], rows["int4_only"]["rel_mse"]
    assert top < rnd / 20, (top, rnd)
    assert 0.5 < rnd / int4 < 2.0, (rnd, int4)
    assert rows["bf16_only"]["rel_mse"] < 1e-12
    shard = rows["topk_bf16_shards"]["rel_mse"]
    assert 0.9 * top <= shard <= 1.5 * top, (shard, top)
    assert rows["topk"]["ratio"] == pytest.approx(2 * 4096 / ((4096 - 64) / 2 + 2 * 64))
    # a second, re-quantized all-gather step adds its own 4-bit error, but stays far from random k
    two = rows["two_step"]["rel_mse"]
    assert top <= two < 4 * top, (two, top)
    assert two < rnd / 20, (two, rnd)


def test_two_step_bit_exact_with_the_oracle():
    """The two-step form (quantized reduce-scatter, then re-quantized all-gather) on the CUDA path
    against the same composition of oracle functions, element by element."""
    import numpy as np

    import oracle
    from gpu_helpers import DEV, assert_same, gpu_calibrate_batches, gpu_dequant, gpu_quantize, gpu_select, \
        to_dev_u16, u16

    o = oracle.get()
    cfg = synth.CONFIGS["decode"].with_(name="two_step", P=3, T=40, H=1024, k=32, n_out=8, calib_batches=2,
                                        calib_T=24)
    cs, _ = synth.colscale(cfg)
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
    x_np = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    H = cfg.H

    def oracle_step1(sel, xx):
        c, sd = o.quantize_pack(xx, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
        return o.dequant_reduce(c, sd, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])

    emin, emax = o.calibrate_batches(cal, cfg.beta)
    sel = o.select_topk(emin, emax, cfg.k)
    e2min, e2max = o.calibrate_batches([oracle_step1(sel, c)[None] for c in cal], cfg.beta)
    sel2 = o.select_topk(e2min, e2max, cfg.k)
    z_ref = oracle_step1(sel2, oracle_step1(sel, x_np)[None])

    gmin, gmax = gpu_calibrate_batches(cal, cfg.beta, cfg.P, H)
    B = gpu_select(gmin, gmax, cfg.k)

    def gpu_step1(prm, xx):
        codes, side = gpu_quantize(xx, prm)
        return gpu_dequant(codes, side, prm, H)

    ys = [gpu_step1(B, to_dev_u16(c))[None].contiguous() for c in cal]
    g2min, g2max = gpu_calibrate_batches(ys, cfg.beta, 1, H)
    B2 = gpu_select(g2min, g2max, cfg.k)
    z = gpu_step1(B2, gpu_step1(B, to_dev_u16(x_np))[None].contiguous())
    assert_same(u16(z), z_ref, "two-step output")
    assert np.array_equal(B2["keep_idx"].cpu().numpy(), sel2["keep_idx"])
