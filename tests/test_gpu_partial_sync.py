"""Partial-channel synchronisation (reading R20) on the GPU, against the oracle.

The block [c0, c0 + Hs) of every rank's partial sum goes through calibration, selection,
quantize-pack and dequant-reduce (and the fused call) by the ``_ld`` calls, which read and write
column views of wider rows.  Each output buffer starts out as one rank's own partial sum, so after
the call it must equal that rank's row of the oracle's result: the reduced block inside, the
rank's own values, untouched, outside.  The shapes take both dequant staging paths (rows of code
words of a multiple of 16 bytes or not) and both side-buffer paths (T % 8 == 0 or not).
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import bit_tensor_activation_b200 as hq  # noqa: E402
import oracle  # noqa: E402
from gpu_helpers import DEV, assert_no_device_error, assert_same, f32bits, to_dev_u16, u16, u32  # noqa: E402

# (P, T, ld, c0, Hs, k, fp32 out)
CASES = [
    (3, 40, 1040, 264, 512, 32, False),    # TMA code rows, staged side tiles
    (2, 37, 2048, 0, 1000, 16, False),     # cp.async code rows, side read from memory
    (4, 64, 4096, 2048, 2048, 64, True),   # the upper half of a 4096-wide row, fp32 out
    (2, 24, 512, 504, 8, 0, False),        # the last 8 features only, all 4-bit
]


@pytest.mark.parametrize("P,T,ld,c0,Hs,k,f32", CASES, ids=[f"P{c[0]}_T{c[1]}_ld{c[2]}_c{c[3]}_H{c[4]}_k{c[5]}"
                                                           for c in CASES])
def test_partial_sync_block(P, T, ld, c0, Hs, k, f32):
    cfg = synth.CONFIGS["decode"].with_(name="blk", P=P, T=T, H=ld, k=0, n_out=16, calib_batches=2, calib_T=T)
    cs, _ = synth.colscale(cfg)
    o = oracle.get()
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, cs=cs) for b in range(2)]
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    blk = lambda a: np.ascontiguousarray(a[:, :, c0:c0 + Hs])  # noqa: E731
    # oracle on the block (it is the dense [P][T][Hs] tensor as far as the path is concerned)
    emin, emax = o.calibrate_batches([blk(c) for c in cal], cfg.beta)
    sel = o.select_topk(emin, emax, k)
    codes_r, side_r = o.quantize_pack(blk(x), sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    y = o.partial_sync(x, c0, Hs, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"])
    # GPU: the _ld calls on column views of the full-width tensors
    xd = [to_dev_u16(c) for c in cal]
    ema_min = torch.empty((P, Hs), dtype=torch.float32, device=DEV)
    ema_max = torch.empty_like(ema_min)
    for b, c in enumerate(xd):
        hq.hq_calibrate_ld(c[:, :, c0:c0 + Hs], ema_min, ema_max, cfg.beta, b == 0)
    B = hq.Buffers(P, T, Hs, k, device=DEV)
    hq.hq_select_topk(ema_min, ema_max, k, B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero)
    X = to_dev_u16(x)
    hq.hq_quantize_pack_ld(X[:, :, c0:c0 + Hs], B.keep_idx, B.rest_idx, B.inv_scale, B.zero, B.codes, B.side)
    outs = {}
    for r in range(P):  # rank r's buffer holds its own partial sum before the reduction
        out = X[r].clone()
        hq.hq_dequant_reduce_ld(B.codes, B.side, B.keep_idx, B.rest_idx, B.scale, B.zero, out[:, c0:c0 + Hs])
        fused = X[r].clone()
        hq.hq_compress_reduce_ld(X[:, :, c0:c0 + Hs], B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero,
                                 fused[:, c0:c0 + Hs])
        outs[r] = (out, fused)
    f32out = None
    if f32:
        f32out = torch.full((T, ld), -7.0, dtype=torch.float32, device=DEV)
        hq.hq_dequant_reduce_ld(B.codes, B.side, B.keep_idx, B.rest_idx, B.scale, B.zero, f32out[:, c0:c0 + Hs])
    assert_no_device_error()
    assert_same(f32bits(ema_min), f32bits(emin), "ema_min")
    assert_same(f32bits(ema_max), f32bits(emax), "ema_max")
    assert_same(B.keep_idx.cpu().numpy(), sel["keep_idx"], "keep_idx")
    assert_same(B.rest_idx.cpu().numpy(), sel["rest_idx"], "rest_idx")
    assert_same(B.zero.cpu().numpy(), sel["zero"], "zero")
    assert_same(u32(B.codes), codes_r, "codes")
    assert_same(u16(B.side), side_r, "side")
    for r, (out, fused) in outs.items():
        assert_same(u16(out), y[r], f"rank {r}: dequant-reduce")
        assert_same(u16(fused), y[r], f"rank {r}: fused")
    if f32:
        want = o.dequant_reduce(codes_r, side_r, Hs, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                                out_f32=True)
        got = f32out.cpu().numpy()
        assert_same(f32bits(got[:, c0:c0 + Hs]), f32bits(want), "fp32 block")
        outside = np.ones(ld, bool)
        outside[c0:c0 + Hs] = False
        assert np.all(got[:, outside] == -7.0), "fp32 output outside the block was written"


def test_ld_arguments_are_checked():
    P, T, H, k = 1, 8, 64, 8
    B = hq.Buffers(P, T, H, k, device=DEV)
    x = torch.zeros((P, T, 72), dtype=torch.int16, device=DEV)
    with pytest.raises(hq.HQError):  # the block would start 2 bytes past a 16-byte boundary
        hq.hq_quantize_pack_ld(x[:, :, 1:65], B.keep_idx, B.rest_idx, B.inv_scale, B.zero, B.codes, B.side)
    lib = hq.lib()
    st = torch.cuda.current_stream().cuda_stream
    p = x.data_ptr()
    assert lib.hq_calibrate_ld(p, 60, P, T, H, 0.9, 1, B.ema_min.data_ptr(), B.ema_max.data_ptr(), st) == \
        hq.HQ_ERR_INVALID_ARG  # ld < H
    assert lib.hq_calibrate_ld(p, 68, P, T, H, 0.9, 1, B.ema_min.data_ptr(), B.ema_max.data_ptr(), st) == \
        hq.HQ_ERR_INVALID_ARG  # ld % 8 != 0
    assert_no_device_error()
