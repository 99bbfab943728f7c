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
