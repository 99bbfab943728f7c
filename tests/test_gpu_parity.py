"""CUDA path vs the CPU oracle, through the C ABI, on seeded synthetic inputs.

Integer and index results (codes, zero points, keep/rest sets, side buffers) and the fp32 results
(moving averages, scales, reduced outputs) must all be bit-identical: both sides evaluate the same
sequence of correctly rounded fp32 operations, and the reduction order over ranks is fixed.
Small and mid-size problems are compared element by element; so are the whole wire buffers and
outputs of the two full-size workloads (prefill 7B and 70B shapes), whose 32-batch calibration is
compared on sampled columns the oracle computes one by one.
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
from gpu_helpers import (DEV, assert_no_device_error, assert_same, compare_all, f32bits,  # noqa: E402
                         gpu_calibrate_batches, gpu_dequant, gpu_fused, gpu_quantize, gpu_select, params_to_dev,
                         to_dev_u16, u16, u32)


def _batches(cfg, cs, T=None):
    return [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T if T is None else T, cs=cs)
            for b in range(cfg.calib_batches)]


@pytest.mark.parametrize("name", ["pr1", "decode"])
def test_named_small_configs_bit_exact(name):
    cfg = synth.CONFIGS[name]
    cs, outl = synth.colscale(cfg)
    ref = compare_all(cfg, _batches(cfg, cs), synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs))
    assert set(outl.tolist()) <= set(ref["sel"]["keep_idx"].tolist())


# Mid-size shapes: several slices / row blocks with ragged tails, k = 0 and k = H, odd P.
MID = [
    synth.CONFIGS["prefill7b"].with_(name="7b_ragged", T=37, H=3000, k=96, n_out=40, calib_batches=3, calib_T=41),
    synth.CONFIGS["prefill70b"].with_(name="70b_ragged", T=19, H=8200, k=264, n_out=100, calib_batches=2, calib_T=23),
    synth.CONFIGS["decode"].with_(name="p3_k0", P=3, T=50, H=1032, k=0, calib_batches=2, calib_T=7),
    synth.CONFIGS["decode"].with_(name="p5_kH", P=5, T=9, H=520, k=520, n_out=8, calib_batches=2, calib_T=5),
    synth.CONFIGS["pr1"].with_(name="h8", P=4, T=33, H=8, k=8, n_out=1, calib_batches=2, calib_T=3),
    synth.CONFIGS["pr1"].with_(name="h8k0", P=1, T=1, H=8, k=0, n_out=1, calib_batches=1, calib_T=1),
    synth.CONFIGS["decode"].with_(name="p16", P=16, T=21, H=2048, k=32, calib_batches=2, calib_T=9),
    synth.CONFIGS["decode"].with_(name="p64", P=64, T=5, H=264, k=16, n_out=8, calib_batches=1, calib_T=4),
    synth.sweep_configs()[5].with_(name="sweep_mid", T=100, calib_batches=2, calib_T=64),
]


@pytest.mark.parametrize("cfg", MID, ids=[c.name for c in MID])
def test_mid_shapes_bit_exact(cfg):
    cs, _ = synth.colscale(cfg)
    compare_all(cfg, _batches(cfg, cs), synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs))


# (P, T, H, k, runs of kept features): code rows of 182 words (staged with cp.async) and of 384
# words (staged with TMA; slices with more kept features than the staged side tile holds sum
# them from HBM).
CLUSTERED = [
    (3, 40, 2560, 1104, np.r_[0:8, 100:1100, 1500:1580, 2544:2560]),
    (3, 70, 4096, 1024, np.r_[0:40, 256:900, 1024:1031, 2000:2300, 4063:4096]),
]


@pytest.mark.parametrize("P,T,H,k,big", CLUSTERED, ids=["cp_async", "tma"])
def test_clustered_kept_features_bit_exact(P, T, H, k, big):
    """Kept features in long runs (whole groups and slices kept) stress the compact layout."""
    o = oracle.get()
    rng = np.random.default_rng(3)
    assert len(big) <= k
    x = synth.fill_cpu(synth.CONFIGS["decode"].with_(P=P, T=T, H=H, n_out=4), synth.EVAL, 0,
                       cs=np.ones(H))
    emin = -np.ones((P, H), np.float32)
    emax = np.ones((P, H), np.float32)
    emax[:, big] = 50.0
    emin[:, big] = -50.0
    emax += rng.uniform(0, 0.01, (P, H)).astype(np.float32)
    sel = o.select_topk(emin, emax, k)
    assert set(big.tolist()) <= set(sel["keep_idx"].tolist())
    prm = params_to_dev(sel)
    B = gpu_select(torch.from_numpy(emin).to(DEV), torch.from_numpy(emax).to(DEV), k)
    assert np.array_equal(B["keep_idx"].cpu().numpy(), sel["keep_idx"])
    codes_r, side_r = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out_r = o.dequant_reduce(codes_r, side_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    xd = to_dev_u16(x)
    codes, side = gpu_quantize(xd, prm)
    out = gpu_dequant(codes, side, prm, H)
    fused, _, _ = gpu_fused(xd, prm)
    assert_no_device_error()
    assert np.array_equal(u32(codes), codes_r) and np.array_equal(u16(side), side_r)
    assert np.array_equal(u16(out), out_r) and np.array_equal(u16(fused), out_r)


# Kept features per 256-feature slice of H = 4096, planted: every count the kept-sum paths of the
# TMA dequant-reduce distinguish (none, up to 8, 16 and 32 staged kept features, more than fit the
# staged side tile), with row counts that give a CTA one row block or several.
SLICE_KEPT = [0, 1, 3, 4, 5, 7, 8, 9, 15, 16, 17, 24, 31, 32, 33, 19]


@pytest.mark.parametrize("P,T", [(5, 72), (8, 72), (2, 2048), (4, 4096), (16, 64), (64, 8)])
def test_kept_counts_per_slice_bit_exact(P, T):
    o = oracle.get()
    H = 4096
    rng = np.random.default_rng(11)
    big = np.sort(np.concatenate([256 * s + rng.choice(256, n, replace=False) for s, n in enumerate(SLICE_KEPT)]))
    k = len(big)
    assert (H - k) % 32 == 0 and T % 8 == 0  # code rows and side rows both staged by TMA
    x = synth.fill_cpu(synth.CONFIGS["decode"].with_(P=P, T=T, H=H, n_out=4), synth.EVAL, 0, cs=np.ones(H))
    emin = -np.ones((P, H), np.float32) - rng.uniform(0, 0.01, (P, H)).astype(np.float32)
    emax = np.ones((P, H), np.float32)
    emax[:, big] = 40.0
    sel = o.select_topk(emin, emax, k)
    assert np.array_equal(sel["keep_idx"], big)
    prm = params_to_dev(sel)
    codes_r, side_r = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out_r = o.dequant_reduce(codes_r, side_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    out_rf = o.dequant_reduce(codes_r, side_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                              out_f32=True)
    lit_r = o.dequant_reduce(codes_r, side_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                             bf16_shards=True)
    codes, side = gpu_quantize(to_dev_u16(x), prm)
    out = gpu_dequant(codes, side, prm, H)
    out_f = gpu_dequant(codes, side, prm, H, out_f32=True)
    lit = gpu_dequant(codes, side, prm, H, bf16_shards=True)
    assert_no_device_error()
    assert_same(u32(codes), codes_r, "codes")
    assert_same(u16(side), side_r, "side")
    assert_same(u16(out), out_r, "out bf16")
    assert_same(f32bits(out_f), f32bits(out_rf), "out f32")
    assert_same(u16(lit), lit_r, "bf16-shard reduction")


@pytest.mark.parametrize("T", [40, 37])
def test_halo_past_the_preloaded_candidates(T):
    """Slice 0 keeps 7 features, so its last code word needs the next 7 non-kept features (the
    halo); slice 1 starts with 12 kept features, so 3 of those halo features lie beyond the 16
    features after the slice whose parameters quantize-pack preloads (found by walking keep_idx)
    and beyond the 8 columns it stages (read from x directly).  Codes, side and output bit-exact."""
    o = oracle.get()
    P, H = 3, 1024
    big = np.array(sorted([3, 40, 77, 120, 160, 200, 250] + list(range(256, 268)) + [300, 333, 500, 640, 900]))
    k = len(big)
    assert k % 8 == 0
    rng = np.random.default_rng(13)
    x = synth.fill_cpu(synth.CONFIGS["decode"].with_(P=P, T=T, H=H, n_out=4), synth.EVAL, 0, cs=np.ones(H))
    emin = -np.ones((P, H), np.float32) - rng.uniform(0, 0.01, (P, H)).astype(np.float32)
    emax = np.ones((P, H), np.float32)
    emax[:, big] = 40.0
    sel = o.select_topk(emin, emax, k)
    assert np.array_equal(sel["keep_idx"], big)
    Cb = 256 - 7  # compact position of slice 0's first halo feature
    assert (8 - Cb % 8) % 8 == 7 and sel["rest_idx"][Cb + 6] == 274  # the last one is past 256 + 16
    prm = params_to_dev(sel)
    codes_r, side_r = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out_r = o.dequant_reduce(codes_r, side_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    codes, side = gpu_quantize(to_dev_u16(x), prm)
    out = gpu_dequant(codes, side, prm, H)
    fused, fcodes, fside = gpu_fused(to_dev_u16(x), prm, wire=True)
    assert_no_device_error()
    assert_same(u32(codes), codes_r, "codes")
    assert_same(u16(side), side_r, "side")
    assert_same(u16(out), out_r, "out")
    assert_same(u16(fused), out_r, "fused")
    assert_same(u32(fcodes), codes_r, "fused codes")
    assert_same(u16(fside), side_r, "fused side")


def test_select_ties_and_special_values():
    o = oracle.get()
    P, H = 3, 4096
    rng = np.random.default_rng(5)
    emin = (-rng.integers(0, 4, (P, H))).astype(np.float32)   # many exact ties
    emax = rng.integers(0, 4, (P, H)).astype(np.float32)
    emin[0, 10], emax[0, 10] = np.nan, np.nan                  # NaN statistics -> range 0
    emax[1, 20] = np.inf                                       # infinite range -> degenerate scale
    emin[2, 30] = -np.inf
    emin[1, 40], emax[1, 40] = -1e-39, 1e-39                   # subnormal scale -> degenerate
    emin[2, 50], emax[2, 50] = 3e38, 3.3e38                    # huge but finite
    emin[0, 60], emax[0, 60] = -3e38, 3e38                     # range overflows to inf
    for k in (0, 8, 256, 2048, 4088, 4096):
        sel = o.select_topk(emin, emax, k)
        B = gpu_select(torch.from_numpy(emin).to(DEV), torch.from_numpy(emax).to(DEV), k)
        assert_no_device_error()
        assert np.array_equal(B["keep_idx"].cpu().numpy(), sel["keep_idx"]), k
        assert np.array_equal(B["rest_idx"].cpu().numpy(), sel["rest_idx"]), k
        assert np.array_equal(f32bits(B["scale"]), f32bits(sel["scale"]))
        assert np.array_equal(f32bits(B["inv_scale"]), f32bits(sel["inv_scale"]))
        assert np.array_equal(B["zero"].cpu().numpy(), sel["zero"])
    all_equal = np.zeros((P, H), np.float32)
    sel = o.select_topk(all_equal - 1, all_equal + 1, 64)
    B = gpu_select(torch.from_numpy(all_equal - 1).to(DEV), torch.from_numpy(all_equal + 1).to(DEV), 64)
    assert B["keep_idx"].cpu().numpy().tolist() == list(range(64)) == sel["keep_idx"].tolist()


def test_special_input_values_bit_exact():
    """NaN, +-inf, -0, huge and subnormal partial sums in x, and in calibration."""
    o = oracle.get()
    cfg = synth.CONFIGS["decode"].with_(P=4, T=24, H=1024, k=32, calib_batches=2, calib_T=16)
    cs, _ = synth.colscale(cfg)
    cal = _batches(cfg, cs)
    cal[1][2, 3, 7] = 0x7FC0          # NaN in calibration
    cal[0][1, :, 9] = 0x8000          # a column of -0
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    specials = [0x7FC0, 0xFFC1, 0x7F80, 0xFF80, 0x8000, 0x0001, 0x8001, 0x7F7F, 0xFF7F]
    rng = np.random.default_rng(9)
    for v in specials:
        for _ in range(40):
            x[rng.integers(cfg.P), rng.integers(cfg.T), rng.integers(cfg.H)] = v
    compare_all(cfg, cal, x)


def test_tiny_scales_bit_exact():
    """Scales below 2^-109 (partial sums of magnitude ~1e-35): the dequant kernel decodes such
    slices with explicit shifts instead of pre-divided scales, still bit-exact."""
    o = oracle.get()
    P, T, H, k = 3, 20, 1024, 16
    rng = np.random.default_rng(21)
    vals = (rng.standard_normal((P, T, H)) * 1e-35).astype(np.float32)
    vals[:, :, 300:700] *= 1e30          # ordinary magnitudes in some slices
    from pins import f32_to_bf16_torch
    x = f32_to_bf16_torch(vals.ravel()).reshape(P, T, H)
    emin, emax = o.calibrate(x, 0.9, True)
    sel = o.select_topk(emin, emax, k)
    assert (sel["scale"] < 2.0 ** -109).any() and (sel["scale"] > 1e-10).any()
    prm = params_to_dev(sel)
    codes_r, side_r = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out_r = o.dequant_reduce(codes_r, side_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"], out_f32=True)
    xd = to_dev_u16(x)
    codes, side = gpu_quantize(xd, prm)
    out = gpu_dequant(codes, side, prm, H, out_f32=True)
    fused, _, _ = gpu_fused(xd, prm, out_f32=True)
    assert_no_device_error()
    assert np.array_equal(u32(codes), codes_r)
    assert np.array_equal(f32bits(out), f32bits(out_r))
    assert np.array_equal(f32bits(fused), f32bits(out_r))


def test_empty_rows_are_no_ops():
    prm = params_to_dev(oracle.get().select_topk(-np.ones((2, 64), np.float32), np.ones((2, 64), np.float32), 8))
    x = torch.empty((2, 0, 64), dtype=torch.int16, device=DEV)
    codes, side = gpu_quantize(x, prm)
    out = gpu_dequant(codes, side, prm, 64)
    fused, _, _ = gpu_fused(x, prm)
    assert out.numel() == 0 and fused.numel() == 0
    assert_no_device_error()


def test_bounded_wait_times_out_and_context_survives():
    """A pipeline wait that nothing satisfies gives up after its limit, records HQ_ERR_TIMEOUT,
    and the context keeps working (no trap, no hang)."""
    assert hq.hq_read_device_error() == hq.HQ_OK
    hq.hq_selftest_bounded_wait(2_000_000)  # ~1 ms
    assert hq.hq_read_device_error() == hq.HQ_ERR_TIMEOUT
    assert hq.hq_read_device_error() == hq.HQ_OK
    cfg = synth.CONFIGS["pr1"]
    cs, _ = synth.colscale(cfg)
    compare_all(cfg, _batches(cfg, cs), synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs))


@pytest.mark.parametrize("H,k", [(256, 8), (4096, 128)], ids=["fallback_dequant", "tma_dequant"])
@pytest.mark.parametrize("where", ["last", "first"])
def test_bad_index_is_recorded_not_dereferenced(H, k, where):
    """keep_idx holding an index outside [0, H): every kernel that reads it clamps it and reports
    HQ_ERR_BAD_INDEX, and reading the error word clears it."""
    P, T = 2, 40
    prm = params_to_dev(oracle.get().select_topk(-np.ones((P, H), np.float32), np.ones((P, H), np.float32), k))
    bad = prm["keep_idx"].clone()
    if where == "last":
        bad[-1] = H + 1000
    else:
        bad[0] = -5
    prm["keep_idx"] = bad
    x = torch.zeros((P, T, H), dtype=torch.int16, device=DEV)
    codes, side = gpu_quantize(x, prm)
    assert hq.hq_read_device_error() == hq.HQ_ERR_BAD_INDEX, "quantize-pack"
    assert hq.hq_read_device_error() == hq.HQ_OK, "reading clears the word"
    gpu_dequant(codes, side, prm, H)
    assert hq.hq_read_device_error() == hq.HQ_ERR_BAD_INDEX, "dequant-reduce"
    gpu_fused(x, prm)
    assert hq.hq_read_device_error() == hq.HQ_ERR_BAD_INDEX, "compress-reduce"
    assert hq.hq_read_device_error() == hq.HQ_OK


# ---------------------------------------------------------------------------------------------
# Full-size workloads in the launch shapes the benchmark times
# ---------------------------------------------------------------------------------------------
def _gpu_batch(cfg, purpose, batch, cs_dev, T=None):
    T = cfg.T if T is None else T
    out = torch.empty((cfg.P, T, cfg.H), dtype=torch.int16, device=DEV)
    synth.fill_gpu(cfg, purpose, batch, out, cs_dev, T=T)
    return out


@pytest.mark.parametrize("name", ["prefill7b", "prefill70b"])
def test_full_size_calibration_sampled(name):
    cfg = synth.CONFIGS[name]
    cs, outl = synth.colscale(cfg)
    cs_dev = torch.from_numpy(cs).to(DEV)
    buf = torch.empty((cfg.P, cfg.calib_T, cfg.H), dtype=torch.int16, device=DEV)
    emin = torch.empty((cfg.P, cfg.H), dtype=torch.float32, device=DEV)
    emax = torch.empty_like(emin)
    for b in range(cfg.calib_batches):
        synth.fill_gpu(cfg, synth.CALIB, b, buf, cs_dev, T=cfg.calib_T)
        hq.hq_calibrate(buf, emin, emax, cfg.beta, b == 0)
    B = gpu_select(emin, emax, cfg.k)
    assert_no_device_error()
    keep = set(B["keep_idx"].cpu().numpy().tolist())
    assert set(outl.tolist()) <= keep, "planted outlier columns must be selected"
    gmin, gmax = emin.cpu().numpy(), emax.cpu().numpy()
    o = oracle.get()
    rng = np.random.default_rng(17)
    cols = np.concatenate([rng.choice(cfg.H, 10, replace=False), outl[:2]])
    for h in cols:
        r = int(rng.integers(cfg.P))
        cal = [synth.fill_cpu(cfg, synth.CALIB, b, ranks=(r, r + 1), cols=(int(h), int(h) + 1), T=cfg.calib_T, cs=cs)
               for b in range(cfg.calib_batches)]
        em, ex = o.calibrate_batches(cal, cfg.beta)
        assert f32bits(gmin[r, h]) == f32bits(em[0, 0]) and f32bits(gmax[r, h]) == f32bits(ex[0, 0]), (r, h)


@pytest.mark.parametrize("name", ["prefill7b", "prefill70b"])
def test_full_size_select_quantize_reduce_whole_tensors(name):
    """The full-size evaluation batch, in the launch configuration the benchmark times: selection,
    then the whole codes and side buffers and the whole bf16 output of the split path, the fused
    path (with and without its wire outputs) and the bf16-shard reduction, each compared with the
    oracle element by element over all T rows.  The host regenerates the batch with the same
    counter-based generator; the parameters come from the oracle (a shorter calibration: any
    statistics serve as selection input)."""
    cfg = synth.CONFIGS[name]
    o = oracle.get()
    cs, outl = synth.colscale(cfg)
    cal = _batches(cfg.with_(calib_batches=4), cs, T=48)
    emin, emax = o.calibrate_batches(cal, cfg.beta)
    sel = o.select_topk(emin, emax, cfg.k)
    B = gpu_select(torch.from_numpy(emin).to(DEV), torch.from_numpy(emax).to(DEV), cfg.k)
    assert_same(B["keep_idx"].cpu().numpy(), sel["keep_idx"], "keep_idx")
    assert_same(B["rest_idx"].cpu().numpy(), sel["rest_idx"], "rest_idx")
    assert_same(f32bits(B["scale"]), f32bits(sel["scale"]), "scale")
    assert_same(f32bits(B["inv_scale"]), f32bits(sel["inv_scale"]), "inv_scale")
    assert_same(B["zero"].cpu().numpy(), sel["zero"], "zero")
    prm = params_to_dev(sel)
    x = _gpu_batch(cfg, synth.EVAL, 0, torch.from_numpy(cs).to(DEV))
    codes, side = gpu_quantize(x, prm)
    out = gpu_dequant(codes, side, prm, cfg.H)
    lit = gpu_dequant(codes, side, prm, cfg.H, bf16_shards=True)
    fused, _, _ = gpu_fused(x, prm)
    fused_w, wcodes, wside = gpu_fused(x, prm, wire=True)
    assert_no_device_error()
    del x
    xh = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    c_r, s_r = o.quantize_pack(xh, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    del xh
    assert_same(u32(codes), c_r, "codes")
    assert_same(u16(side), s_r, "side")
    assert_same(u32(wcodes), c_r, "fused wire codes")
    assert_same(u16(wside), s_r, "fused wire side")
    o_r = o.dequant_reduce(c_r, s_r, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    assert_same(u16(out), o_r, "out bf16")
    assert_same(u16(fused), o_r, "fused bf16")
    assert_same(u16(fused_w), o_r, "fused bf16 (wire written too)")
    l_r = o.dequant_reduce(c_r, s_r, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                           bf16_shards=True)
    assert_same(u16(lit), l_r, "bf16-shard reduction")


# ---------------------------------------------------------------------------------------------
# The 90 sweep workloads at full size, in the launch shapes the sweep tool times
# ---------------------------------------------------------------------------------------------
SWEEP = synth.sweep_configs()


@pytest.mark.parametrize("cfg", SWEEP, ids=[c.name for c in SWEEP])
def test_sweep_point_sampled(cfg):
    """Calibration on sampled columns, selection in full, and quantize-pack, dequant-reduce and the
    fused call on sampled rows (every feature of each), against the oracle; fused == split over
    the whole output."""
    o = oracle.get()
    P, T, H, k = cfg.P, cfg.T, cfg.H, cfg.k
    cs, _ = synth.colscale(cfg)
    cs_dev = torch.from_numpy(cs).to(DEV)
    buf = torch.empty((P, cfg.calib_T, H), dtype=torch.int16, device=DEV)
    emin = torch.empty((P, H), dtype=torch.float32, device=DEV)
    emax = torch.empty_like(emin)
    for b in range(cfg.calib_batches):
        synth.fill_gpu(cfg, synth.CALIB, b, buf, cs_dev, T=cfg.calib_T)
        hq.hq_calibrate(buf, emin, emax, cfg.beta, b == 0)
    del buf
    gmin, gmax = emin.cpu().numpy(), emax.cpu().numpy()
    rng = np.random.default_rng(cfg.seed)
    for h in rng.choice(H, 3, replace=False):
        r = int(rng.integers(P))
        cal = [synth.fill_cpu(cfg, synth.CALIB, b, ranks=(r, r + 1), cols=(int(h), int(h) + 1), T=cfg.calib_T, cs=cs)
               for b in range(cfg.calib_batches)]
        em, ex = o.calibrate_batches(cal, cfg.beta)
        assert f32bits(gmin[r, h]) == f32bits(em[0, 0]) and f32bits(gmax[r, h]) == f32bits(ex[0, 0]), (r, h)
    sel = o.select_topk(gmin, gmax, k)
    B = gpu_select(emin, emax, k)
    for name in ("keep_idx", "rest_idx", "zero"):
        assert np.array_equal(B[name].cpu().numpy(), sel[name]), name
    for name in ("scale", "inv_scale"):
        assert np.array_equal(f32bits(B[name]), f32bits(sel[name])), name
    x = torch.empty((P, T, H), dtype=torch.int16, device=DEV)
    synth.fill_gpu(cfg, synth.EVAL, 0, x, cs_dev)
    codes, side = gpu_quantize(x, B)
    out = gpu_dequant(codes, side, B, H)
    fused, _, _ = gpu_fused(x, B)
    assert_no_device_error()
    assert torch.equal(out, fused), "fused == split over the whole output"
    rows = sorted({0, T - 1, int(rng.integers(T)), int(rng.integers(T))})
    ridx = torch.tensor(rows, device=DEV)
    codes_h = u32(codes.index_select(1, ridx))
    side_h = u16(side.index_select(2, ridx))
    out_h = u16(out.index_select(0, ridx))
    for i, t in enumerate(rows):
        xr = synth.fill_cpu(cfg, synth.EVAL, 0, rows=(t, t + 1), cs=cs)
        c_r, s_r = o.quantize_pack(xr, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
        o_r = o.dequant_reduce(c_r, s_r, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
        assert_same(codes_h[:, i:i + 1], c_r, f"codes row {t}")
        assert_same(side_h[:, :, i:i + 1], s_r, f"side row {t}")
        assert_same(out_h[i:i + 1], o_r, f"out row {t}")


def test_per_rank_calls_equal_the_batched_call():
    """A real rank calls quantize-pack with P = 1 on its own partial sum and its own parameter
    row; stacking those wire buffers gives the batched (P > 1) call's buffers bit for bit, and
    reducing them gives the batched output."""
    cfg = synth.CONFIGS["prefill7b"].with_(name="per_rank", P=5, T=72, H=2048, k=64, n_out=16, calib_batches=2,
                                           calib_T=40)
    cs, _ = synth.colscale(cfg)
    cal = _batches(cfg, cs)
    x_np = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    emin, emax = gpu_calibrate_batches(cal, cfg.beta, cfg.P, cfg.H)
    B = gpu_select(emin, emax, cfg.k)
    x = to_dev_u16(x_np)
    codes, side = gpu_quantize(x, B)
    out = gpu_dequant(codes, side, B, cfg.H)
    per_codes, per_side = [], []
    for r in range(cfg.P):
        row = {n: (B[n][r:r + 1].contiguous() if n in ("scale", "inv_scale", "zero") else B[n]) for n in B}
        # calibration of one rank alone gives that rank's row of the batched statistics
        e1, e2 = gpu_calibrate_batches([c[r:r + 1] for c in cal], cfg.beta, 1, cfg.H)
        assert torch.equal(e1, emin[r:r + 1]) and torch.equal(e2, emax[r:r + 1])
        c_r, s_r = gpu_quantize(x[r:r + 1].contiguous(), row)
        per_codes.append(c_r)
        per_side.append(s_r)
    assert_no_device_error()
    assert torch.equal(torch.cat(per_codes), codes)
    assert torch.equal(torch.cat(per_side), side)
    out2 = gpu_dequant(torch.cat(per_codes), torch.cat(per_side), B, cfg.H)
    assert torch.equal(out2, out)


@pytest.mark.parametrize("P,T,H,k", [(2, 40, 32768, 1024), (64, 8, 32768, 512)], ids=["h_max", "p_and_h_max"])
def test_maximum_sizes_bit_exact(P, T, H, k):
    """The largest shapes the ABI accepts: H = 32768 (selection keys fill 128 KB of shared memory)
    and P = 64 ranks (the TMA dequant-reduce kernel's constants then take 128 KB of its shared
    memory), through the whole path, element by element against the oracle."""
    cfg = synth.CONFIGS["decode"].with_(name=f"max_{P}_{H}", P=P, T=T, H=H, k=k, n_out=64, calib_batches=2,
                                        calib_T=16)
    cs, _ = synth.colscale(cfg)
    compare_all(cfg, _batches(cfg, cs), synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs))
