"""Failure detection in the real TMA pipelines, without faulting or hanging the GPU.

hq_selftest_set_pipeline_stall delays every pipeline producer's first load well past a short bound
on the consumers' waits.  The consumers then give up, the kernel records HQ_ERR_TIMEOUT and raises
its abort flag, and the producer -- which still issues its first ring loads -- waits for them on
its normal (long) bound before the CTA exits.  Each test then restores the normal bounds and checks
that the same call on the same context is bit-exact with the oracle again.  Nothing traps, asserts
or spins without a bound.
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
from gpu_helpers import (DEV, assert_no_device_error, assert_same, f32bits, gpu_dequant, gpu_fused,  # noqa: E402
                         gpu_quantize, params_to_dev, to_dev_u16, u16, u32)

CONSUMER_LIMIT = 20_000          # about 10 us
PRODUCER_DELAY = 100_000_000     # about 50 ms: far beyond the consumers' bound (and the 100 us wait hint)


def _problem():
    """4 ranks x 64 rows x 4096 features, 128 kept: every kernel takes its TMA pipeline."""
    cfg = synth.CONFIGS["prefill7b"].with_(name="stall", P=4, T=64, calib_batches=1, calib_T=64)
    cs, _ = synth.colscale(cfg)
    o = oracle.get()
    emin, emax = o.calibrate(synth.fill_cpu(cfg, synth.CALIB, 0, cs=cs), cfg.beta, True)
    sel = o.select_topk(emin, emax, cfg.k)
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out = o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                           out_f32=True)
    return cfg, sel, x, codes, side, out


def _run(kernel, cfg, prm, xd, codes_d, side_d):
    if kernel == "quantize_pack":
        return gpu_quantize(xd, prm)
    if kernel == "dequant_reduce":
        return gpu_dequant(codes_d, side_d, prm, cfg.H, out_f32=True)
    return gpu_fused(xd, prm, out_f32=True)[0]


@pytest.mark.parametrize("kernel", ["quantize_pack", "dequant_reduce", "compress_reduce"])
def test_consumer_wait_expires_and_producer_drains(kernel):
    cfg, sel, x, codes, side, out = _problem()
    prm = params_to_dev(sel)
    xd = to_dev_u16(x)
    codes_d = torch.from_numpy(codes.view(np.int32)).to(DEV)
    side_d = to_dev_u16(side)
    assert_no_device_error()
    hq.hq_selftest_set_pipeline_stall(CONSUMER_LIMIT, PRODUCER_DELAY)
    try:
        _run(kernel, cfg, prm, xd, codes_d, side_d)
        status = hq.hq_read_device_error()
    finally:
        hq.hq_selftest_set_pipeline_stall(0, 0)
    assert status == hq.HQ_ERR_TIMEOUT, hq.hq_status_string(status)
    assert hq.hq_read_device_error() == hq.HQ_OK, "reading the error word clears it"
    # same context, normal bounds: the call is exact again
    got = _run(kernel, cfg, prm, xd, codes_d, side_d)
    assert_no_device_error()
    if kernel == "quantize_pack":
        assert_same(u32(got[0]), codes, "codes")
        assert_same(u16(got[1]), side, "side")
    else:
        assert_same(f32bits(got), f32bits(out), f"{kernel} output")


def test_stall_setting_is_checked_on_the_host():
    for c, d in ((1, 0), (0, 1), (-1, 5), (5, -1), (5, 1 << 40)):
        with pytest.raises(hq.HQError):
            hq.hq_selftest_set_pipeline_stall(c, d)
    hq.hq_selftest_set_pipeline_stall(0, 0)


def test_error_recorded_on_one_stream_is_read_on_another():
    """The error word is device-wide: a timeout recorded by a kernel on stream A is returned by a
    read ordered on stream B once A's work is done, and the read clears it."""
    a, b = torch.cuda.Stream(DEV), torch.cuda.Stream(DEV)
    assert hq.hq_read_device_error() == hq.HQ_OK
    hq.hq_selftest_bounded_wait(1_000_000, stream=a)
    a.synchronize()
    assert hq.hq_read_device_error(stream=b) == hq.HQ_ERR_TIMEOUT
    assert hq.hq_read_device_error(stream=a) == hq.HQ_OK
