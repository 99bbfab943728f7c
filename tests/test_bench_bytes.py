"""The algorithmic bytes behind the benchmark's roofline figures, checked against totals worked
out independently for the four named workloads.

Per call, with H' = H - k:
- quantize-pack reads 2PTH and writes PTH'/2 + 2PTk;
- dequant-reduce reads PTH'/2 + 2PTk and writes 2TH (bf16 out);
- compress-reduce reads 2PTH and writes 2TH.
The benchmark adds the parameters each call reads (5 bytes per (rank, feature) of scale and
zero, 4 per index; inv_scale too for the fused call), which the totals below leave out.
"""
import pytest

import bench
import synth

# workload: (quantize-pack, dequant-reduce, compress-reduce) bytes without parameters, ratio
TOTALS = {
    "pr1": (20_864, 12_672, 24_576, 3.657),
    "decode": (1_323_008, 536_576, 1_310_720, 3.821),
    "prefill7b": (341_835_776, 106_954_752, 301_989_888, 3.657),
    "prefill70b": (1_367_343_104, 427_819_008, 1_207_959_552, 3.657),
}


@pytest.mark.parametrize("name", list(TOTALS))
def test_algorithmic_bytes(name):
    cfg = synth.CONFIGS[name]
    P, H = cfg.P, cfg.H
    ab = bench.algo_bytes(cfg)
    q, d, f, ratio = TOTALS[name]
    assert ab["quantize_pack"] - (5 * P * H + 4 * H) == q
    assert ab["dequant_reduce"] - (5 * P * H + 4 * H) == d
    assert ab["compress_reduce"] - (9 * P * H + 4 * H) == f
    assert bench.compression_ratio(cfg) == pytest.approx(ratio, abs=5e-4)


def test_compression_ratio_limits():
    cfg = synth.CONFIGS["prefill7b"]
    assert bench.compression_ratio(cfg.with_(k=0)) == 4.0           # all 4-bit
    assert bench.compression_ratio(cfg.with_(k=cfg.H)) == 1.0       # all bf16
