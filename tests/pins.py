"""Pins of the CPU oracle against facts fixed by the pages and by the mathematics.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the oracle disagrees
with something that does not come from the oracle itself: values worked by hand
(``tests/golden``), numpy / torch library routines, brute-force searches on tiny inputs,
closed forms, error bounds, and the Irwin-Hall law of summed quantization errors from the page
"Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section
"Combating Quantization Errors with Tensor Parallelism".  ``tests/test_oracle_pins.py`` runs
them against the committed oracle and against deliberately broken copies of it, so each pin is
shown to catch the mistakes it is meant to catch.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------------
# bf16 helpers written with numpy only
# ---------------------------------------------------------------------------------------------
def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    return (np.asarray(u16, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_torch(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 by torch's own conversion (a library routine)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(f, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f32_bits(v) -> int:
    return int(np.array([v], np.float32).view(np.uint32)[0])


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_values(rng, n, scale=1.0):
    """Random bf16 bit patterns of N(0, scale) values."""
    return f32_to_bf16_torch((rng.standard_normal(n) * scale).astype(np.float32))


# ---------------------------------------------------------------------------------------------
# Output rounding (reading R11)
# ---------------------------------------------------------------------------------------------
def pin_bf16_round(o):
    rng = _rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 10,
        # exact ties: low 16 bits = 0x8000, with even and odd kept halves
        (np.arange(200, dtype=np.uint32) * 0x10000 + 0x3F808000).view(np.float32),
        (np.arange(200, dtype=np.uint32) * 0x10000 + 0xBF818000).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38, 1e-40, -1e-40,
                  np.finfo(np.float32).max], np.float32),
    ])
    want = f32_to_bf16_torch(vals)
    got = np.array([o.bf16_round(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want), "bf16 rounding differs from torch's RNE conversion"
    assert o.bf16_round(float("nan")) == 0x7FC0


# ---------------------------------------------------------------------------------------------
# The 4-bit quantizer (reading R6)
# ---------------------------------------------------------------------------------------------
def pin_quantize_golden(o):
    for c in _golden("quantize_cases.json")["cases"]:
        v = float(c["v"])
        got = o.quantize_one(v, float(c["inv"]), int(c["zero"]))
        assert got == c["q"], f"quantize({c['v']}, inv={c['inv']}, zero={c['zero']}) = {got}, want {c['q']} ({c['why']})"


def pin_quantize_nearest_grid(o):
    """q minimises |x - (q - zero) * scale| over 0..15 (brute force in double), except where
    x*inv_scale is within fp32 rounding of a half-integer (where both neighbours are correct)."""
    rng = _rng(2)
    n = 3000
    x = bf16_to_f32(_bf16_values(rng, n, 3.0))
    scale = (rng.uniform(0.05, 1.0, n)).astype(np.float32)
    inv = (np.float32(1.0) / scale).astype(np.float32)
    zero = rng.integers(0, 16, n)
    for i in range(n):
        got = o.quantize_one(float(x[i]), float(inv[i]), int(zero[i]))
        grid = (np.arange(16) - zero[i]) * float(scale[i])
        d = np.abs(float(x[i]) - grid)
        best = int(np.argmin(d))
        if got != best:
            a = float(x[i]) / float(scale[i])
            frac = abs(a - math.floor(a) - 0.5)
            assert frac < 1e-5 and abs(got - best) == 1, (
                f"x={x[i]} scale={scale[i]} zero={zero[i]}: q={got}, nearest grid point {best}")


# ---------------------------------------------------------------------------------------------
# Parameters (reading R3)
# ---------------------------------------------------------------------------------------------
def pin_params_golden(o):
    cases = _golden("params_cases.json")["cases"]
    emin = np.array([[c["ema_min"] for c in cases]], np.float32)
    emax = np.array([[c["ema_max"] for c in cases]], np.float32)
    scale, inv, zero, _ = o.params(emin, emax)
    for j, c in enumerate(cases):
        assert f32_bits(scale[0, j]) == int(c["scale_hex"], 16), f"scale for {c}: {scale[0, j]!r}"
        assert f32_bits(inv[0, j]) == int(c["inv_hex"], 16), f"inv_scale for {c}: {inv[0, j]!r}"
        assert int(zero[0, j]) == c["zero"], f"zero for {c}: {zero[0, j]}"


def pin_params_closed_form(o):
    """Against the closed form evaluated in double: the grid spans [lo, hi] with 15 steps,
    0 lies on the grid, lo quantizes to 0 and hi to 15."""
    rng = _rng(3)
    P, H = 3, 2000
    a = rng.standard_normal((P, H)) * rng.lognormal(0, 2, (P, H))
    b = a + np.abs(rng.standard_normal((P, H))) * rng.lognormal(0, 2, (P, H))
    emin, emax = a.astype(np.float32), b.astype(np.float32)
    scale, inv, zero, rng_ = o.params(emin, emax)
    lo = np.minimum(emin.astype(np.float64), 0.0)
    hi = np.maximum(emax.astype(np.float64), 0.0)
    s_exact = (hi - lo) / 15.0
    assert np.all(np.abs(scale - s_exact) <= 2.0 * np.spacing(scale.astype(np.float32)).astype(np.float64)), "scale != (hi-lo)/15"
    assert np.all(np.abs(inv.astype(np.float64) * scale - 1.0) <= 2.0 ** -22), "inv_scale is not 1/scale"
    z_exact = -lo / scale.astype(np.float64)
    assert np.all(np.abs(zero - z_exact) <= 0.5 + 1e-5), "zero is not round(-lo/scale)"
    assert np.all((zero >= 0) & (zero <= 15))
    assert np.allclose(rng_, hi - lo, rtol=2 ** -23, atol=0), "range != hi - lo"
    for r in range(P):
        for h in range(0, H, 97):
            q_lo = o.quantize_one(float(lo[r, h]), float(inv[r, h]), int(zero[r, h]))
            q_hi = o.quantize_one(float(hi[r, h]), float(inv[r, h]), int(zero[r, h]))
            assert q_lo == 0 and q_hi == 15, f"lo->{q_lo}, hi->{q_hi} at ({r},{h})"
            assert o.quantize_one(0.0, float(inv[r, h]), int(zero[r, h])) == zero[r, h]


# ---------------------------------------------------------------------------------------------
# Calibration (reading R1)
# ---------------------------------------------------------------------------------------------
def pin_calibrate_single_batch(o):
    """One batch: the statistics are numpy's min / max over the rows (NaN ignored, -0 as +0)."""
    rng = _rng(4)
    P, T, H = 3, 37, 61
    x = _bf16_values(rng, P * T * H, 2.0).reshape(P, T, H)
    x[0, 5, 7] = 0x7FC0          # NaN
    x[1, :, 3] = 0x8000          # a column of -0
    x[2, :, 4] = 0xFF80          # a column of -inf
    emin, emax = o.calibrate(x, 0.9, True)
    f = bf16_to_f32(x).astype(np.float64)
    want_min = np.nanmin(f, axis=1) + 0.0
    want_max = np.nanmax(f, axis=1) + 0.0
    assert np.array_equal(emin, want_min.astype(np.float32)), "batch min"
    assert np.array_equal(emax, want_max.astype(np.float32)), "batch max"
    assert not np.signbit(emin[1, 3]) and not np.signbit(emax[1, 3]), "-0 must be stored as +0"


def pin_calibrate_ema(o):
    """Moving average: against the recurrence in double (within a few fp32 ulp), and against the
    closed form beta**n * m0 when every batch after the first has a zero extreme."""
    rng = _rng(5)
    P, T, H = 2, 9, 40
    beta = 0.9
    batches = [_bf16_values(rng, P * T * H, 1.0 + b).reshape(P, T, H) for b in range(12)]
    emin, emax = o.calibrate_batches(batches, beta)
    b32 = np.float32(beta)
    omb = np.float64(np.float32(1.0) - b32)
    mins = [np.nanmin(bf16_to_f32(x).astype(np.float64), axis=1) for x in batches]
    maxs = [np.nanmax(bf16_to_f32(x).astype(np.float64), axis=1) for x in batches]
    dmin, dmax = mins[0].copy(), maxs[0].copy()
    for b in range(1, len(batches)):
        dmin = np.float64(b32) * dmin + omb * mins[b]
        dmax = np.float64(b32) * dmax + omb * maxs[b]
    tol_min = 24 * np.spacing(np.abs(dmin).astype(np.float32)).astype(np.float64)
    tol_max = 24 * np.spacing(np.abs(dmax).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(emin - dmin) <= tol_min), "ema_min vs double recurrence"
    assert np.all(np.abs(emax - dmax) <= tol_max), "ema_max vs double recurrence"
    # closed form: a first batch of constant m0, then all-zero batches -> beta**n * m0 for both
    m0 = 3.0
    first = np.full((1, 4, 8), f32_to_bf16_torch(np.array([m0], np.float32))[0], np.uint16)
    zeros = np.zeros((1, 4, 8), np.uint16)
    emn, emx = o.calibrate(first, beta, True)
    for n in range(1, 9):
        emn, emx = o.calibrate(zeros, beta, False, emn, emx)
        want = (float(b32) ** n) * m0
        tol = (n + 1) * np.spacing(np.float32(want))
        assert np.all(np.abs(emx - want) <= tol) and np.all(np.abs(emn - want) <= tol), f"beta^{n} * m0"


def pin_calibrate_ema_golden(o):
    """One moving-average update worked by hand (tests/golden/ema_cases.json): two products and
    a sum, each rounded to fp32, with 1 - beta an fp32 subtraction.  Each case's value differs
    from the one a single rounding (fused, double-precision or delta-form update) or the literal
    0.1f would give."""
    g = _golden("ema_cases.json")
    for c in g["cases"]:
        a = f32_to_bf16_torch(np.array([c["a"]], np.float32))[0]
        b = f32_to_bf16_torch(np.array([c["b"]], np.float32))[0]
        assert bf16_to_f32(np.array([a]))[0] == c["a"] and bf16_to_f32(np.array([b]))[0] == c["b"]
        emn, emx = o.calibrate(np.full((1, 3, 8), a, np.uint16), g["beta"], True)
        emn, emx = o.calibrate(np.full((1, 3, 8), b, np.uint16), g["beta"], False, emn, emx)
        want = int(c["ema_hex"], 16)
        for name, v in (("ema_min", emn), ("ema_max", emx)):
            got = v.view(np.uint32)
            assert np.all(got == want), f"{name} after (a={c['a']}, b={c['b']}): {got[0, 0]:08X}, want {want:08X}"


# ---------------------------------------------------------------------------------------------
# Selection (readings R4, R5)
# ---------------------------------------------------------------------------------------------
def pin_select_golden(o):
    g = _golden("select_ties.json")
    rng_ = np.array(g["range"], np.float32)
    for c in g["cases"]:
        keep, rest, score = o.select(rng_, c["k"])
        assert score.tolist() == g["expect_score"], "score = sum over ranks"
        assert keep.tolist() == c["keep"] and rest.tolist() == c["rest"], f"k={c['k']}: keep {keep}, rest {rest}"


def pin_select_rank_order_golden(o):
    """The score is summed in fp32 in rank order (tests/golden/order_cases.json, "score"): at
    2^24 the spacing is 2, so ranges 2^24, 1, 1 sum to 2^24, not 2^24 + 2, and that decides
    which feature is kept."""
    g = _golden("order_cases.json")["score"]
    rng_ = np.array(g["range"], np.float32)
    for c in g["cases"]:
        keep, rest, score = o.select(rng_, c["k"])
        assert score.tolist() == g["expect_score"], f"score {score.tolist()}"
        assert keep.tolist() == c["keep"] and rest.tolist() == c["rest"], f"k={c['k']}: keep {keep}, rest {rest}"


def pin_select_brute_force(o):
    """Python's sorted() with key (-score, column) on random and tie-heavy inputs."""
    rng = _rng(6)
    for trial in range(40):
        P = int(rng.integers(1, 5))
        H = int(rng.integers(8, 64)) // 8 * 8
        if trial % 2:
            rg = rng.integers(0, 4, (P, H)).astype(np.float32)     # many ties
        else:
            rg = np.abs(rng.standard_normal((P, H))).astype(np.float32)
        k = int(rng.integers(0, H // 8 + 1)) * 8
        keep, rest, score = o.select(rg, k)
        s = [math.fsum(float(rg[r, h]) for r in range(P)) for h in range(H)]
        assert np.allclose(score, s, rtol=P * 2 ** -23, atol=0), "score"
        order = sorted(range(H), key=lambda h: (-float(score[h]), h))
        assert keep.tolist() == sorted(order[:k]), f"trial {trial}: keep"
        assert rest.tolist() == sorted(order[k:]), f"trial {trial}: rest"


# ---------------------------------------------------------------------------------------------
# Quantize-pack layout (readings R6, R7)
# ---------------------------------------------------------------------------------------------
def pin_pack_golden(o):
    g = _golden("pack_example.json")
    H, k = g["H"], g["k"]
    cal = f32_to_bf16_torch(np.array(g["calib_rows"], np.float32)).reshape(1, 2, H)
    emin, emax = o.calibrate(cal, 0.9, True)
    sel = o.select_topk(emin, emax, k)
    assert np.all(sel["scale"] == g["expect_scale"]) and np.all(sel["inv_scale"] == g["expect_inv_scale"])
    assert np.all(sel["zero"] == g["expect_zero"])
    assert sel["keep_idx"].tolist() == g["expect_keep"] and sel["rest_idx"].tolist() == g["expect_rest"]
    x = f32_to_bf16_torch(np.array(g["x"], np.float32)).reshape(1, 1, H)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    assert ["%08X" % w for w in codes.ravel()] == g["expect_codes_hex"], "packed word"
    assert np.array_equal(side.ravel(), x.ravel()[g["expect_keep"]]), "side buffer"
    out = o.dequant_reduce(codes, side, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"], out_f32=True)
    assert out.ravel().tolist() == g["expect_out"]


def pin_pack_unpack(o):
    """Codes unpacked with numpy bit operations equal the element-wise quantizer, in rest_idx
    order; the side buffer holds the kept columns' bits."""
    rng = _rng(7)
    P, T, H, k = 2, 5, 64, 16
    x = _bf16_values(rng, P * T * H, 2.0).reshape(P, T, H)
    emin = np.full((P, H), -3.0, np.float32) * rng.uniform(0.5, 1.5, (P, H)).astype(np.float32)
    emax = np.full((P, H), 3.0, np.float32) * rng.uniform(0.5, 1.5, (P, H)).astype(np.float32)
    sel = o.select_topk(emin, emax, k)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    nib = (codes[..., None] >> (np.arange(8, dtype=np.uint32) * 4)) & 0xF
    q = nib.reshape(P, T, H - k)
    f = bf16_to_f32(x)
    for r in range(P):
        for t in range(T):
            for c, h in enumerate(sel["rest_idx"]):
                want = o.quantize_one(float(f[r, t, h]), float(sel["inv_scale"][r, h]), int(sel["zero"][r, h]))
                assert q[r, t, c] == want, f"code ({r},{t},col {h})"
    assert np.array_equal(side, x[:, :, sel["keep_idx"]].transpose(0, 2, 1)), "side [P][k][T]"


# ---------------------------------------------------------------------------------------------
# Dequant-reduce (readings R9, R10, R11)
# ---------------------------------------------------------------------------------------------
def _numpy_rank_sum(f):
    acc = np.zeros(f.shape[1:], np.float32)
    for r in range(f.shape[0]):
        acc = (acc + f[r]).astype(np.float32)
    return acc


def pin_reduce_all_kept(o):
    """k = H: the reduction is the plain fp32 sum of the bf16 inputs in rank order."""
    rng = _rng(8)
    P, T, H = 5, 7, 32
    x = _bf16_values(rng, P * T * H, 4.0).reshape(P, T, H)
    emin, emax = o.calibrate(x, 0.9, True)
    sel = o.select_topk(emin, emax, H)
    out = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"], out_f32=True)
    want = _numpy_rank_sum(bf16_to_f32(x))
    assert np.array_equal(out, want), "k=H must be the exact rank-ordered fp32 sum"
    outb = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"])
    assert np.array_equal(outb, f32_to_bf16_torch(want)), "bf16 output = RNE of the fp32 sum"


def pin_nan_outputs(o):
    """Reading R11: a NaN sum is written as the canonical quiet NaN in both output types; a NaN
    in a 4-bit feature quantizes to the zero point and so adds exactly 0 (reading R6)."""
    P, T, H, k = 2, 1, 16, 8
    emin = np.full((P, H), -2.0, np.float32)
    emax = np.full((P, H), 2.0, np.float32)
    emax[:, :k] = 100.0                     # features 0..7 are kept
    sel = o.select_topk(emin, emax, k)
    assert sel["keep_idx"].tolist() == list(range(k))
    vals = np.zeros((P, T, H), np.float32)
    vals[0, 0, 0] = np.nan                  # kept: NaN + 0
    vals[0, 0, 1], vals[1, 0, 1] = np.inf, -np.inf   # kept: inf + -inf
    vals[0, 0, 2] = -np.nan                 # kept: negative NaN payload
    vals[0, 0, 8], vals[1, 0, 8] = np.nan, 1.0       # 4-bit: NaN -> zero point, adds 0
    x = f32_to_bf16_torch(vals.ravel()).reshape(P, T, H)
    x[0, 0, 2] = 0xFFC1
    of = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"], out_f32=True)
    ob = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"])
    bits = of.view(np.uint32)
    assert bits[0, 0] == bits[0, 1] == bits[0, 2] == 0x7FC00000, [hex(b) for b in bits[0, :3]]
    assert ob[0, 0] == ob[0, 1] == ob[0, 2] == 0x7FC0
    assert np.isfinite(of[0, 8]) and abs(float(of[0, 8]) - 1.0) <= float(sel["scale"][1, 8]) / 2 * 1.0001


def pin_reduce_dequant_sum(o):
    """Each reduced element is sum_r (q_r - zero_r) * scale_r of its own codes, within the
    rounding of P fp32 steps; kept ones are the sum of the side values."""
    rng = _rng(9)
    P, T, H, k = 4, 6, 48, 8
    x = _bf16_values(rng, P * T * H, 2.0).reshape(P, T, H)
    emin, emax = o.calibrate(x, 0.9, True)
    sel = o.select_topk(emin, emax, k)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out = o.dequant_reduce(codes, side, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"], out_f32=True)
    q = ((codes[..., None] >> (np.arange(8, dtype=np.uint32) * 4)) & 0xF).reshape(P, T, H - k).astype(np.float64)
    rest, keep = sel["rest_idx"], sel["keep_idx"]
    terms = (q - sel["zero"][:, None, rest]) * sel["scale"][:, None, rest].astype(np.float64)
    want = terms.sum(axis=0)
    bound = P * 2.0 ** -23 * np.abs(terms).sum(axis=0) + 1e-30
    assert np.all(np.abs(out[:, rest] - want) <= bound), "dequantized sum"
    sf = bf16_to_f32(side).transpose(0, 2, 1)  # [P][T][k]
    kept = sf.astype(np.float64).sum(axis=0)
    assert np.all(np.abs(out[:, keep] - kept) <= P * 2.0 ** -23 * np.abs(sf).sum(axis=0)), "kept sum"
    assert np.array_equal(out[:, keep], _numpy_rank_sum(sf)), "kept: exact rank-ordered sum"


def pin_reduce_order_golden(o):
    """Rounding and rank order of the reduction, worked by hand (tests/golden/order_cases.json):
    a 4-bit feature takes one rounding per rank (a fused multiply-add), and both 4-bit and kept
    features are summed in rank order 0..P-1 -- cases whose result changes under a separate
    multiply and add, under reversed rank order, or with an exact accumulator."""
    g = _golden("order_cases.json")
    P = g["P"]
    cases = g["dequant_4bit"]
    words, zero, scale = _one_group([[c["qz"][r] for c in cases] for r in range(P)],
                                    [[c["scale"][r] for c in cases] for r in range(P)])
    side = np.zeros((P, 0, 1), np.uint16)
    out = o.dequant_reduce(words, side, 8, np.zeros(0, np.int32), np.arange(8, dtype=np.int32), scale, zero,
                           out_f32=True)
    for i, c in enumerate(cases):
        got = f32_bits(out[0, i])
        assert got == int(c["out_hex"], 16), f"4-bit case {i}: {got:08X}, want {c['out_hex']}"
    kept = g["kept"]
    k = 8
    side = np.zeros((P, k, 1), np.uint16)
    for j, c in enumerate(kept):
        for r in range(P):
            side[r, j, 0] = int(c["side_hex"][r], 16)
    keep = np.arange(k, dtype=np.int32)
    words = np.zeros((P, 1, 0), np.uint32)
    out = o.dequant_reduce(words, side, k, keep, np.zeros(0, np.int32), np.ones((P, k), np.float32),
                           np.zeros((P, k), np.uint8), out_f32=True)
    for j, c in enumerate(kept):
        got = f32_bits(out[0, j])
        assert got == int(c["out_hex"], 16), f"kept case {j}: {got:08X}, want {c['out_hex']}"


def pin_reduce_error_bound(o):
    """Per-element error against the exact sum of the inputs (double): at most
    sum_r (scale_r / 2 + slop) when every rank is inside its grid (reading R8)."""
    cfg = synth.CONFIGS["decode"].with_(T=16)
    cs, _ = synth.colscale(cfg)
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(4)]
    emin, emax = o.calibrate_batches(cal, cfg.beta)
    sel = o.select_topk(emin, emax, cfg.k)
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    out = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"], out_f32=True)
    f = bf16_to_f32(x).astype(np.float64)
    exact = f.sum(axis=0)
    rest = sel["rest_idx"]
    s = sel["scale"][:, rest].astype(np.float64)[:, None, :]
    z = sel["zero"][:, rest].astype(np.float64)[:, None, :]
    a = f[:, :, rest] / s + z
    inr = np.all((a >= -0.5) & (a <= 15.5), axis=0)
    bound = (s / 2 + 2.0 ** -22 * (np.abs(f[:, :, rest]) + 16 * s)).sum(axis=0) + cfg.P * 2.0 ** -24 * np.abs(f[:, :, rest]).sum(axis=0)
    err = np.abs(out[:, rest] - exact[:, rest])
    assert inr.mean() > 0.5, f"only {inr.mean():.2f} of elements inside every rank's grid"
    assert np.all(err[inr] <= bound[inr]), f"error bound violated: max excess {np.max(err[inr] - bound[inr])}"


def irwin_hall_stats(o, P=4, H=1024, T=256, k=0, seed=1234):
    """Summed quantization error on U(-1,1) partial sums versus the Irwin-Hall prediction."""
    cfg = synth.Config("ih", P=P, T=T, H=H, k=k, seed=seed, dist="uniform", sigma=0.0,
                       calib_batches=8, calib_T=256)
    cs, _ = synth.colscale(cfg)
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
    emin, emax = o.calibrate_batches(cal, cfg.beta)
    sel = o.select_topk(emin, emax, k)
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    out = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"], out_f32=True)
    f = bf16_to_f32(x).astype(np.float64)
    rest = sel["rest_idx"]
    e = out[:, rest].astype(np.float64) - f[:, :, rest].sum(axis=0)
    s = sel["scale"][:, rest].astype(np.float64)
    a = f[:, :, rest] / s[:, None, :] + sel["zero"][:, rest].astype(np.float64)[:, None, :]
    inr = np.all((a >= -0.5) & (a <= 15.5), axis=0)
    pred = np.broadcast_to((s ** 2).sum(axis=0) / 12.0, e.shape)
    return e[inr], pred[inr], s


def pin_irwin_hall(o):
    """Page "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication", section
    "Combating Quantization Errors with Tensor Parallelism": quantizing the partial sums
    before synchronisation gives a summed error distributed as a sum of P independent uniform
    errors (Irwin-Hall).  Its variance must be sum_r scale_r^2 / 12 within 5%, its mean ~0, and
    for P = 2 its shape the triangular Irwin-Hall(2) law."""
    e, pred, _ = irwin_hall_stats(o, P=4)
    assert e.size >= 100_000
    ratio = np.var(e) / np.mean(pred)
    assert abs(ratio - 1.0) < 0.05, f"Var(error) / Irwin-Hall prediction = {ratio:.4f}"
    assert abs(np.mean(e)) < 5 * math.sqrt(np.mean(pred) / e.size), "summed error is biased"
    e2, pred2, s2 = irwin_hall_stats(o, P=2, seed=99)
    u = np.sort(e2 / s2.mean())   # in units of the grid step, ~ U(-1/2,1/2) + U(-1/2,1/2)
    cdf = np.where(u < 0, 0.5 * (u + 1) ** 2, 1 - 0.5 * (1 - u) ** 2)
    cdf = np.clip(cdf, 0, 1)
    emp = np.arange(1, u.size + 1) / u.size
    ks = np.max(np.abs(emp - cdf))
    assert ks < 0.02, f"KS distance to the triangular law = {ks:.4f}"


# ---------------------------------------------------------------------------------------------
# Selection against the page's observations
# ---------------------------------------------------------------------------------------------
def pin_outliers_selected(o):
    """"Leveraging Outliers for Efficient Communication": the few features with enormous ranges
    are consistent, so range-based selection must keep every planted outlier column."""
    for name in ("pr1", "decode"):
        cfg = synth.CONFIGS[name]
        cs, outl = synth.colscale(cfg)
        cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
        emin, emax = o.calibrate_batches(cal, cfg.beta)
        sel = o.select_topk(emin, emax, cfg.k)
        assert set(outl.tolist()) <= set(sel["keep_idx"].tolist()), f"{name}: outlier columns not all kept"
        assert len(sel["keep_idx"]) == cfg.k and len(sel["rest_idx"]) == cfg.H - cfg.k
        assert sorted(sel["keep_idx"].tolist() + sel["rest_idx"].tolist()) == list(range(cfg.H))


def selection_mse(o, cfg=None, trials=3):
    """MSE of the reduced output for range-based top-k, random k columns, and k = 0."""
    cfg = cfg or synth.CONFIGS["decode"]
    cs, _ = synth.colscale(cfg)
    cal = [synth.fill_cpu(cfg, synth.CALIB, b, T=cfg.calib_T, cs=cs) for b in range(cfg.calib_batches)]
    emin, emax = o.calibrate_batches(cal, cfg.beta)
    x = synth.fill_cpu(cfg, synth.EVAL, 0, cs=cs)
    exact = bf16_to_f32(x).astype(np.float64).sum(axis=0)

    def mse(keep):
        keep = np.sort(np.asarray(keep, np.int32))
        rest = np.setdiff1d(np.arange(cfg.H, dtype=np.int32), keep).astype(np.int32)
        sel = o.select_topk(emin, emax, 0)
        out = o.compress_reduce(x, keep, rest, sel["scale"], sel["inv_scale"], sel["zero"], out_f32=True)
        return float(np.mean((out - exact) ** 2))

    top = o.select_topk(emin, emax, cfg.k)["keep_idx"]
    rng = _rng(11)
    rand = np.mean([mse(rng.choice(cfg.H, cfg.k, replace=False)) for _ in range(trials)])
    return mse(top), rand, mse([])


def pin_selection_benefit(o):
    """"Key Observations and Future Directions": random high-precision features help little over
    pure Int4, range-based selection helps a lot."""
    top, rand, none = selection_mse(o)
    assert top < 0.2 * none, f"top-k MSE {top} vs pure Int4 {none}"
    assert rand > 0.7 * none, f"random-k MSE {rand} vs pure Int4 {none}"


# ---------------------------------------------------------------------------------------------
# Dequant-reduce, literal variant: each rank's dequantized value rounded to bf16 (reading R19)
# ---------------------------------------------------------------------------------------------
def _one_group(qz_rows, scale_rows):
    """Codes, zero points and scales for one 8-feature group of P ranks and one row, with
    q - zero = qz_rows[r][i] in -15..15 (zero = max(0, -(q - zero)), so both stay in 0..15)."""
    qz = np.asarray(qz_rows, np.int64)
    P, n = qz.shape
    zero = np.zeros((P, 8), np.uint8)
    q = np.zeros((P, 8), np.int64)
    zero[:, :n] = np.maximum(0, -qz)
    q[:, :n] = qz + zero[:, :n]
    words = np.zeros((P, 1, 1), np.uint32)
    for r in range(P):
        words[r, 0, 0] = sum(int(q[r, i]) << (4 * i) for i in range(8))
    scale = np.ones((P, 8), np.float32)
    scale[:, :n] = np.asarray(scale_rows, np.float32)
    return words, zero, scale


def pin_bf16_shards_golden(o):
    """Values worked by hand (tests/golden/bf16_shards_cases.json): ties go to the even bf16
    neighbour, each shard is rounded before the fp32 rank sum, the sum itself is not."""
    g = _golden("bf16_shards_cases.json")
    cases = g["cases"]
    assert len(cases) == 8
    words, zero, scale = _one_group([[c["qz"][r] for c in cases] for r in range(g["P"])],
                                    [[c["scale"][r] for c in cases] for r in range(g["P"])])
    keep, rest = np.zeros(0, np.int32), np.arange(8, dtype=np.int32)
    side = np.zeros((g["P"], 0, 1), np.uint16)
    lit = o.dequant_reduce(words, side, 8, keep, rest, scale, zero, out_f32=True, bf16_shards=True)
    std = o.dequant_reduce(words, side, 8, keep, rest, scale, zero, out_f32=True)
    for i, c in enumerate(cases):
        assert f32_bits(lit[0, i]) == f32_bits(c["f32"]), f"case {i} ({c['why']}): {lit[0, i]} != {c['f32']}"
        assert f32_bits(std[0, i]) == f32_bits(c["std"]), f"case {i} standard reading: {std[0, i]} != {c['std']}"


def _random_wire(rng, P, T, H, k, scale):
    zero = rng.integers(0, 16, (P, H)).astype(np.uint8)
    codes = rng.integers(0, 2**32, (P, T, (H - k) // 8), dtype=np.uint64).astype(np.uint32)
    side = _bf16_values(rng, P * k * T, 3.0).reshape(P, k, T)
    keep = np.sort(rng.choice(H, k, replace=False)).astype(np.int32)
    rest = np.setdiff1d(np.arange(H), keep).astype(np.int32)
    return codes, side, keep, rest, scale.astype(np.float32), zero


def pin_bf16_shards_exact_products(o):
    """Power-of-two scales make every product (q - zero) * scale a bf16 value (at most 4
    significant bits), so the literal reading must equal the standard one bit for bit, in both
    output types, kept features included."""
    rng = _rng(41)
    P, T, H, k = 4, 6, 64, 16
    scale = np.ldexp(1.0, rng.integers(-12, 6, (P, H)))
    codes, side, keep, rest, scale, zero = _random_wire(rng, P, T, H, k, scale)
    for f32 in (True, False):
        lit = o.dequant_reduce(codes, side, H, keep, rest, scale, zero, out_f32=f32, bf16_shards=True)
        std = o.dequant_reduce(codes, side, H, keep, rest, scale, zero, out_f32=f32)
        assert np.array_equal(lit.view(np.uint32 if f32 else np.uint16), std.view(np.uint32 if f32 else np.uint16))


def pin_bf16_shards_rounding_bound(o):
    """One rank: the output is the shard's value rounded to bf16, so it is a bf16 number within
    half a bf16 spacing of the fp32 product (bf16 has 8 significant bits: at most 2^-8 of the
    value), and differs from the product wherever the product is not a bf16 number."""
    rng = _rng(43)
    P, T, H, k = 1, 40, 64, 8
    scale = rng.uniform(0.01, 3.0, (P, H))
    codes, side, keep, rest, scale, zero = _random_wire(rng, P, T, H, k, scale)
    lit = o.dequant_reduce(codes, side, H, keep, rest, scale, zero, out_f32=True, bf16_shards=True)
    nib = ((codes[..., None] >> (np.arange(8, dtype=np.uint32) * 4)) & 0xF).reshape(P, T, H - k)
    v = ((nib.astype(np.float64) - zero[:, rest].astype(np.float64)[:, None, :])
         * scale[:, rest].astype(np.float64)[:, None, :]).astype(np.float32)[0]   # fp32 products, [T][H-k]
    got = lit[:, rest]
    assert (got.view(np.uint32) & 0xFFFF == 0).all(), "a shard value that is not a bf16 number"
    err = np.abs(got.astype(np.float64) - v.astype(np.float64))
    assert (err <= np.ldexp(np.abs(v.astype(np.float64)), -8)).all(), "rounding error above half a bf16 spacing"
    off_grid = (v.view(np.uint32) & 0xFFFF) != 0
    assert off_grid.sum() > 100 and (err[off_grid] > 0).all(), "shards were not rounded"


# ---------------------------------------------------------------------------------------------
# Partial-channel synchronisation (reading R20)
# ---------------------------------------------------------------------------------------------
def pin_partial_sync_golden(o):
    """A case worked by hand (tests/golden/partial_sync_example.json): the block's grid-point
    values sum exactly, with and without the block kept in bf16; outside the block every rank
    keeps its own input."""
    g = _golden("partial_sync_example.json")
    P, H, c0, Hs = g["P"], g["H"], g["c0"], g["Hs"]
    x = f32_to_bf16_torch(np.array(g["x"], np.float32)).reshape(P, 1, H)
    assert np.array_equal(bf16_to_f32(x).reshape(P, H), np.array(g["x"], np.float32))
    for k in g["k_cases"]:
        keep = np.arange(k, dtype=np.int32)
        rest = np.arange(k, Hs, dtype=np.int32)
        y = o.partial_sync(x, c0, Hs, keep, rest, np.full((P, Hs), g["scale"], np.float32),
                           np.full((P, Hs), g["inv_scale"], np.float32), np.full((P, Hs), g["zero"], np.uint8))
        assert bf16_to_f32(y).reshape(P, H).tolist() == g["expect_y"], f"k={k}: {bf16_to_f32(y).reshape(P, H)}"


def pin_partial_sync_extremes(o):
    """Hs = H is the whole path (every rank gets the reduced tensor); Hs = 0 leaves every rank
    its own partial sum; outside any block each rank's output is its input, bit for bit, and
    values outside the block do not change the block's result."""
    rng = _rng(51)
    P, T, H, k = 3, 5, 64, 8
    x = _bf16_values(rng, P * T * H, 2.0).reshape(P, T, H)
    emin, emax = o.calibrate(x, 0.9, True)
    sel = o.select_topk(emin, emax, k)
    full = o.compress_reduce(x, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"])
    y = o.partial_sync(x, 0, H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["inv_scale"], sel["zero"])
    for r in range(P):
        assert np.array_equal(y[r], full), f"Hs = H, rank {r}"
    y0 = o.partial_sync(x, 8, 0, np.zeros(0, np.int32), np.zeros(0, np.int32), np.zeros((P, 0), np.float32),
                        np.zeros((P, 0), np.float32), np.zeros((P, 0), np.uint8))
    assert np.array_equal(y0, x), "Hs = 0"
    c0, Hs = 16, 32
    xb = np.ascontiguousarray(x[:, :, c0:c0 + Hs])
    eb_min, eb_max = o.calibrate(xb, 0.9, True)
    sb = o.select_topk(eb_min, eb_max, k)
    args = (sb["keep_idx"], sb["rest_idx"], sb["scale"], sb["inv_scale"], sb["zero"])
    yb = o.partial_sync(x, c0, Hs, *args)
    blk = o.compress_reduce(xb, *args[:2], sb["scale"], sb["inv_scale"], sb["zero"])
    outside = np.ones(H, bool)
    outside[c0:c0 + Hs] = False
    assert np.array_equal(yb[:, :, outside], x[:, :, outside]), "outside the block"
    for r in range(P):
        assert np.array_equal(yb[r, :, c0:c0 + Hs], blk), f"block, rank {r}"
    x2 = x.copy()
    x2[:, :, outside] = _bf16_values(rng, int(outside.sum()) * P * T, 5.0).reshape(P, T, -1)
    yb2 = o.partial_sync(x2, c0, Hs, *args)
    assert np.array_equal(yb2[:, :, c0:c0 + Hs], yb[:, :, c0:c0 + Hs]), "the block depends on values outside it"


ALL_PINS = [
    pin_bf16_round, pin_quantize_golden, pin_quantize_nearest_grid, pin_params_golden,
    pin_params_closed_form, pin_calibrate_single_batch, pin_calibrate_ema, pin_calibrate_ema_golden,
    pin_select_golden, pin_select_rank_order_golden, pin_select_brute_force, pin_pack_golden, pin_pack_unpack,
    pin_reduce_all_kept, pin_nan_outputs, pin_reduce_dequant_sum, pin_reduce_order_golden, pin_reduce_error_bound,
    pin_irwin_hall, pin_outliers_selected,
    pin_selection_benefit, pin_bf16_shards_golden, pin_bf16_shards_exact_products, pin_bf16_shards_rounding_bound,
    pin_partial_sync_golden, pin_partial_sync_extremes,
]
