"""The seeded input generator: determinism, counter-based access, distributions."""
import math

import numpy as np
import pytest

import synth
from pins import bf16_to_f32


def test_series_log_cos_match_libm():
    for x in [2.0 ** -53, 1e-300, 1e-10, 0.1, 0.3, 0.5, 0.70710678, 0.9, 0.999999, 1.0]:
        assert abs(synth.log_series(x) - math.log(x)) <= 4e-16 * max(1.0, abs(math.log(x)))
    for u in np.linspace(0, 1, 1001, endpoint=False):
        assert abs(synth.cos2pi_series(float(u)) - math.cos(2 * math.pi * u)) <= 1e-15


def test_deterministic_and_counter_based():
    cfg = synth.CONFIGS["decode"]
    cs, _ = synth.colscale(cfg)
    a = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    b = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    assert np.array_equal(a, b)
    blk = synth.fill_cpu(cfg, synth.EVAL, 0, ranks=(1, 3), rows=(5, 9), cols=(100, 140), cs=cs)
    assert np.array_equal(blk, a[1:3, 5:9, 100:140])
    rng = np.random.default_rng(0)
    for _ in range(50):
        r, t, h = int(rng.integers(cfg.P)), int(rng.integers(cfg.T)), int(rng.integers(cfg.H))
        assert synth.one(cfg, synth.EVAL, 0, r, t, h, cs) == a[r, t, h]
    c = synth.fill_cpu(cfg, synth.CALIB, 0, T=cfg.calib_T, cs=cs)
    assert not np.array_equal(c, a), "calibration and evaluation batches are different draws"
    assert not np.array_equal(a[0], a[1]), "ranks are different draws"


def test_column_structure_and_distributions():
    cfg = synth.CONFIGS["decode"].with_(T=256)
    cs, outl = synth.colscale(cfg)
    assert len(outl) == cfg.n_out and len(set(outl.tolist())) == cfg.n_out
    base = np.delete(cs, outl)
    assert abs(np.log(base).std() - cfg.sigma) < 0.05 and abs(np.log(base).mean()) < 0.05
    x = bf16_to_f32(synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)).astype(np.float64)
    z = x / cs[None, None, :]
    spikes = np.abs(z) > 8
    assert 0.0005 < spikes.mean() < 0.002, "spike rate ~0.1%"
    zc = np.where(spikes, np.nan, z)
    assert abs(np.nanstd(zc) - 1.0) < 0.02 and abs(np.nanmean(zc)) < 0.01
    std_out = x[:, :, outl].std()
    assert std_out > 30 * np.delete(x, outl, axis=2).std(), "outlier columns dominate the range"

    t3 = synth.CONFIGS["prefill70b"].with_(T=64, H=1024, n_out=8)
    cs3, _ = synth.colscale(t3)
    y = bf16_to_f32(synth.fill_cpu(t3, synth.EVAL, 0, cs=cs3)).astype(np.float64) / cs3
    kurt = np.mean(y ** 4) / np.mean(y ** 2) ** 2
    assert kurt > 6, "Student-t(3) values are heavy-tailed"

    u = synth.sweep_configs()[0].with_(T=64)
    csu, _ = synth.colscale(u)
    v = bf16_to_f32(synth.fill_cpu(u, synth.EVAL, 0, cs=csu))
    assert v.min() >= -1 and v.max() <= 1 and abs(v.mean()) < 0.01 and abs(v.var() - 1 / 3) < 0.01


def test_sweep_table():
    pts = synth.sweep_configs()
    assert len(pts) == 90
    assert {p.P for p in pts} == {2, 4, 8} and {p.H for p in pts} == {4096, 8192}
    assert {p.T for p in pts} == {1, 64, 512, 4096, 16384}
    assert all(p.k % 8 == 0 and p.dist == "uniform" for p in pts)


@pytest.mark.gpu
def test_gpu_generator_matches_host():
    import torch

    for name in ("pr1", "decode"):
        cfg = synth.CONFIGS[name]
        cs, _ = synth.colscale(cfg)
        want = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
        out = torch.empty((cfg.P, cfg.T, cfg.H), dtype=torch.int16, device="cuda")
        synth.fill_gpu(cfg, synth.EVAL, 0, out, torch.from_numpy(cs).cuda())
        got = out.cpu().numpy().view(np.uint16)
        assert np.array_equal(got, want), name
    cfg = synth.CONFIGS["prefill70b"]
    cs, _ = synth.colscale(cfg)
    out = torch.empty((cfg.P, cfg.T, cfg.H), dtype=torch.int16, device="cuda")
    synth.fill_gpu(cfg, synth.CALIB, 7, out, torch.from_numpy(cs).cuda())
    rng = np.random.default_rng(1)
    rows = rng.integers(0, cfg.T, 16)
    host = out.cpu().numpy().view(np.uint16)
    for t in rows:
        want = synth.fill_cpu(cfg, synth.CALIB, 7, rows=(int(t), int(t) + 1), cs=cs)
        assert np.array_equal(host[:, t:t + 1, :], want)
