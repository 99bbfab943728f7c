"""Every output of the CUDA path is written inside its bounds.

Each output tensor is a view into a larger buffer filled with a sentinel byte; after the calls the
bytes in front of and behind every output must still hold the sentinel, and the outputs must
still equal the oracle's.  The shapes have ragged tails (T not a multiple of 32, H not a multiple
of 256, odd P) and take both dequant-reduce staging paths.
"""
import numpy as np
import pytest
import torch

import bit_tensor_activation_b200 as hq
import synth
from gpu_helpers import DEV, assert_no_device_error, assert_same, f32bits, oracle_pipeline, to_dev_u16, u16, u32

pytestmark = pytest.mark.gpu

GUARD_BYTES = 256
SENTINEL = 0xA5


def guarded(shape, dtype):
    """A tensor of `shape` inside a buffer with GUARD_BYTES of sentinel on each side."""
    esize = torch.empty((), dtype=dtype).element_size()
    n = int(np.prod(shape))
    g = GUARD_BYTES // esize
    raw = torch.full((n * esize + 2 * GUARD_BYTES,), SENTINEL, dtype=torch.uint8, device=DEV)
    buf = raw.view(dtype)
    return raw, buf[g:g + n].view(*shape)


def assert_guards(raw, what):
    b = raw.cpu().numpy()
    head, tail = b[:GUARD_BYTES], b[-GUARD_BYTES:]
    assert (head == SENTINEL).all(), f"{what}: bytes in front of the output were written"
    assert (tail == SENTINEL).all(), f"{what}: bytes behind the output were written"


CASES = [
    synth.CONFIGS["prefill70b"].with_(name="70b_ragged", T=19, H=8200, k=264, n_out=100, calib_batches=2,
                                      calib_T=23),
    synth.CONFIGS["prefill7b"].with_(name="7b_ragged", P=3, T=37, H=3000, k=96, n_out=40, calib_batches=2,
                                     calib_T=41),
    synth.CONFIGS["pr1"],
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_outputs_stay_in_bounds(cfg):
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, rows=(0, cfg.calib_T), T=cfg.calib_T) for b in range(cfg.calib_batches)]
    x_np = synth.fill_cpu(cfg, synth.EVAL, 0)
    ref = oracle_pipeline(cfg, cal, x_np)
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    raws = {}

    def g(name, shape, dtype):
        raw, t = guarded(shape, dtype)
        raws[name] = raw
        return t

    emin, emax = g("ema_min", (P, H), torch.float32), g("ema_max", (P, H), torch.float32)
    for b, c in enumerate(cal):
        hq.hq_calibrate(to_dev_u16(c), emin, emax, cfg.beta, b == 0)
    keep, rest = g("keep_idx", (k,), torch.int32), g("rest_idx", (H - k,), torch.int32)
    scale, inv = g("scale", (P, H), torch.float32), g("inv_scale", (P, H), torch.float32)
    zero = g("zero", (P, H), torch.uint8)
    hq.hq_select_topk(emin, emax, k, keep, rest, scale, inv, zero)
    x = to_dev_u16(x_np)
    codes = g("codes", (P, T, (H - k) // 8), torch.int32)
    side = g("side", (P, k, T), torch.int16)
    hq.hq_quantize_pack(x, keep, rest, inv, zero, codes, side)
    out_b = g("out_bf16", (T, H), torch.int16)
    out_f = g("out_f32", (T, H), torch.float32)
    hq.hq_dequant_reduce(codes, side, keep, rest, scale, zero, out_b)
    hq.hq_dequant_reduce(codes, side, keep, rest, scale, zero, out_f)
    lit_b = g("bf16_shards_bf16", (T, H), torch.int16)
    hq.hq_dequant_reduce_bf16_shards(codes, side, keep, rest, scale, zero, lit_b)
    fused = g("fused", (T, H), torch.int16)
    wcodes = g("wire_codes", (P, T, (H - k) // 8), torch.int32)
    wside = g("wire_side", (P, k, T), torch.int16)
    hq.hq_compress_reduce(x, keep, rest, scale, inv, zero, fused, wcodes, wside)
    torch.cuda.synchronize()
    assert_no_device_error()
    for name, raw in raws.items():
        assert_guards(raw, name)
    assert_same(f32bits(emin), f32bits(ref["emin"]), "ema_min")
    assert_same(keep.cpu().numpy(), ref["sel"]["keep_idx"], "keep_idx")
    assert_same(u32(codes), ref["codes"], "codes")
    assert_same(u16(side), ref["side"], "side")
    assert_same(u16(out_b), ref["out_b"], "out bf16")
    assert_same(f32bits(out_f), f32bits(ref["out_f"]), "out f32")
    assert_same(u16(lit_b), ref["lit_b"], "bf16-shard reduction")
    assert_same(u16(fused), ref["out_b"], "fused")
    assert_same(u32(wcodes), ref["codes"], "wire codes")
    assert_same(u16(wside), ref["side"], "wire side")
