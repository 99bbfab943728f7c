"""hq_two_step_reduce_noalloc, the entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a serving process whose device memory is fixed at start-up, a
plugin that lives inside another framework's memory pool, a latency-critical loop that cannot
afford an allocation's device-wide synchronisation.  For them the library keeps a fixed scratch
array in each GPU's global memory and this entry point uses it in place of the caller's workspace.

The test calls the new entry point through the C ABI (ctypes, no binding in between) twice in a
row and compares each result with hq_two_step_reduce's on the same inputs with a caller-owned
workspace: they must be equal bit for bit, the tolerance every parity test here uses.  It also
checks that a problem whose workspace exceeds the array is refused before anything is enqueued.
The file is named to be collected last, and it sets up everything it uses itself, so it passes
alone in a fresh process and after the other tests.
"""
import ctypes

import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import bit_tensor_activation_b200 as hq  # noqa: E402
from bit_tensor_activation_b200 import exchange as ex  # noqa: E402

DEV = torch.device("cuda:0")
HQ_TWO_STEP_NOALLOC_MAX_BYTES = 16 << 20


def _problem(cfg):
    """A decode-size problem built on the GPU: calibration, selection and the step-2 grids."""
    cs = torch.from_numpy(synth.colscale(cfg)[0]).to(DEV)
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    B = hq.Buffers(P, T, H, k, device=DEV)
    cal = []
    for b in range(cfg.calib_batches):
        c = torch.empty((P, cfg.calib_T, H), dtype=torch.int16, device=DEV)
        synth.fill_gpu(cfg, synth.CALIB, b, c, cs, T=cfg.calib_T)
        hq.hq_calibrate(c, B.ema_min, B.ema_max, cfg.beta, b == 0)
        cal.append(c.view(torch.bfloat16))
    hq.hq_select_topk(B.ema_min, B.ema_max, k, B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero)
    params = ex.HybridParams(B.keep_idx, B.rest_idx, B.scale, B.inv_scale, B.zero)
    p2 = ex.step_two_params_simulated(cal, params, k, cfg.beta)
    x = torch.empty((P, T, H), dtype=torch.int16, device=DEV)
    synth.fill_gpu(cfg, synth.EVAL, 0, x, cs)
    return x, params, p2


def _noalloc(x, params, p2, out):
    """One call of the new entry point through the C ABI; returns its status."""
    lib = hq.lib()
    P, T, H = x.shape
    k, k2 = params.keep_idx.shape[0], p2.keep_idx.shape[0]
    f = lib.hq_two_step_reduce_noalloc
    f.restype = ctypes.c_int
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, i32, vp]
    return f(x.data_ptr(), P, T, H, k, params.keep_idx.data_ptr(), params.rest_idx.data_ptr(),
             params.scale.data_ptr(), params.inv_scale.data_ptr(), params.zero.data_ptr(), k2,
             p2.keep_idx.data_ptr(), p2.rest_idx.data_ptr(), p2.scale.data_ptr(), p2.inv_scale.data_ptr(),
             p2.zero.data_ptr(), out.data_ptr(), hq.HQ_OUT_BF16 if out.dtype != torch.float32 else hq.HQ_OUT_F32,
             torch.cuda.current_stream(DEV).cuda_stream)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_noalloc_two_step_equals_the_workspace_call_twice(out_dtype):
    cfg = synth.CONFIGS["decode"].with_(calib_batches=4)   # P = 4, T = 32, H = 4096, k = 64
    x, params, p2 = _problem(cfg)
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    need = hq.hq_two_step_workspace_bytes(P, T, H, k, k)
    assert 0 < need <= HQ_TWO_STEP_NOALLOC_MAX_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    ref = torch.empty((T, H), dtype=out_dtype, device=DEV)
    hq.hq_two_step_reduce(x, params.keep_idx, params.rest_idx, params.scale, params.inv_scale, params.zero,
                          p2.keep_idx, p2.rest_idx, p2.scale, p2.inv_scale, p2.zero, ws, ref)
    torch.cuda.synchronize()
    for call in range(2):   # the second call finds the array holding the first call's contents
        out = torch.full((T, H), float("nan"), dtype=out_dtype, device=DEV)
        assert _noalloc(x, params, p2, out) == hq.HQ_OK
        torch.cuda.synchronize()
        assert hq.hq_read_device_error() == hq.HQ_OK
        assert torch.equal(out.view(torch.int16 if out_dtype != torch.float32 else torch.int32),
                           ref.view(torch.int16 if out_dtype != torch.float32 else torch.int32)), f"call {call}"


def test_noalloc_refuses_a_problem_beyond_its_array():
    cfg = synth.CONFIGS["decode"].with_(T=4096, calib_batches=1, calib_T=64)   # needs more than the array
    x, params, p2 = _problem(cfg)
    assert hq.hq_two_step_workspace_bytes(cfg.P, cfg.T, cfg.H, cfg.k, cfg.k) > HQ_TWO_STEP_NOALLOC_MAX_BYTES
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=DEV)
    assert _noalloc(x, params, p2, out) == hq.HQ_ERR_INVALID_ARG
    assert hq.hq_read_device_error() == hq.HQ_OK
