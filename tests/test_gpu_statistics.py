"""Error statistics of the CUDA path's own output at the largest sweep sizes.

Page "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section
"Combating Quantization Errors with Tensor Parallelism": quantizing each rank's partial sum
before the reduction adds one rounding error per rank, uniform over a grid step, so on uniform
partial sums the summed error follows the Irwin-Hall law.  Its variance is sum_r scale_r^2 / 12,
its mean is 0, and for two ranks it has the triangular density.  The oracle is checked against the
same law on small inputs (tests/pins.py, pin_irwin_hall).  Here it is checked on the GPU path
itself, at sizes the oracle cannot run in a test: the U(-1, 1) sweep workloads with T = 16384
rows, through calibration, selection, quantize-pack and dequant-reduce (fp32 output), and through
the fused call.  The reference for the error is the exact fp64 sum of the bf16 inputs.  Only
elements inside every rank's grid count; clamped ones carry a larger error by design.
"""
import math

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from gpu_helpers import DEV, assert_no_device_error, gpu_dequant, gpu_fused, gpu_quantize, gpu_select  # noqa: E402

import bit_tensor_activation_b200 as hq  # noqa: E402

SWEEP = {c.name: c for c in synth.sweep_configs()}


def _device_path(cfg):
    """The whole path on the device: returns the inputs, the parameters and both fp32 outputs."""
    cs, _ = synth.colscale(cfg)
    cs_dev = torch.from_numpy(cs).to(DEV)
    buf = torch.empty((cfg.P, cfg.calib_T, cfg.H), dtype=torch.int16, device=DEV)
    emin = torch.empty((cfg.P, cfg.H), dtype=torch.float32, device=DEV)
    emax = torch.empty_like(emin)
    for b in range(cfg.calib_batches):
        synth.fill_gpu(cfg, synth.CALIB, b, buf, cs_dev, T=cfg.calib_T)
        hq.hq_calibrate(buf, emin, emax, cfg.beta, b == 0)
    del buf
    B = gpu_select(emin, emax, cfg.k)
    x = torch.empty((cfg.P, cfg.T, cfg.H), dtype=torch.int16, device=DEV)
    synth.fill_gpu(cfg, synth.EVAL, 0, x, cs_dev)
    codes, side = gpu_quantize(x, B)
    out = gpu_dequant(codes, side, B, cfg.H, out_f32=True)
    del codes, side
    fused, _, _ = gpu_fused(x, B, out_f32=True)
    assert_no_device_error()
    return x, B, out, fused


def _errors(x, B, out, rows=1024):
    """Yield, per block of rows, the summed error of the 4-bit features inside every rank's grid,
    each element's predicted variance sum_r scale_r^2 / 12, and the mean scale."""
    rest = B["rest_idx"].long()
    s = B["scale"][:, rest].double()
    z = B["zero"][:, rest].double()
    pred = (s ** 2).sum(0) / 12.0
    for t0 in range(0, x.shape[1], rows):
        f = x[:, t0:t0 + rows, :].view(torch.bfloat16).index_select(2, rest).double()
        e = out[t0:t0 + rows].index_select(1, rest).double() - f.sum(0)
        a = f / s[:, None, :] + z[:, None, :]
        inr = ((a >= -0.5) & (a <= 15.5)).all(0)
        yield e[inr], pred.expand_as(e)[inr], s.mean().item()


@pytest.mark.parametrize("name", ["sweep_P8_H8192_T16384_k256", "sweep_P4_H4096_T16384_k0"])
def test_summed_error_variance_is_irwin_hall(name):
    cfg = SWEEP[name]
    x, B, out, fused = _device_path(cfg)
    assert torch.equal(out, fused), "fused == split"
    n, se, se2, sp = 0, 0.0, 0.0, 0.0
    for e, p, _ in _errors(x, B, out):
        n += e.numel()
        se += e.sum().item()
        se2 += (e * e).sum().item()
        sp += p.sum().item()
    assert n >= 0.9 * cfg.T * (cfg.H - cfg.k), f"only {n} elements inside every rank's grid"
    mean, pred = se / n, sp / n
    ratio = (se2 / n - mean * mean) / pred
    assert abs(ratio - 1.0) < 0.05, f"Var(error) / Irwin-Hall prediction = {ratio:.4f}"
    assert abs(mean) < 5 * math.sqrt(pred / n), f"summed error is biased: mean {mean:.3e}"


def test_two_rank_error_is_triangular():
    cfg = SWEEP["sweep_P2_H8192_T16384_k0"]
    x, B, out, _ = _device_path(cfg)
    g = torch.Generator(device=DEV).manual_seed(7)
    parts = []
    for e, _, s_mean in _errors(x, B, out):
        keep = torch.rand(e.shape, generator=g, device=DEV) < 0.02   # about 2.6 M of 130 M elements
        parts.append((e[keep] / s_mean).cpu().numpy())
    u = np.sort(np.concatenate(parts))   # in units of the grid step: ~ U(-1/2, 1/2) + U(-1/2, 1/2)
    assert u.size > 1_000_000
    cdf = np.clip(np.where(u < 0, 0.5 * (u + 1) ** 2, 1 - 0.5 * (1 - u) ** 2), 0, 1)
    emp = np.arange(1, u.size + 1) / u.size
    ks = np.max(np.abs(emp - cdf))
    assert ks < 0.02, f"KS distance to the triangular law = {ks:.4f}"
