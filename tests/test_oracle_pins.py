"""The oracle against its pins, and planted mistakes against the pins.

The second half copies ``oracle/hq_oracle.c`` to a temporary directory, plants one plausible
mistake (a swapped decay, a dropped rank, a reversed nibble order, a wrong tie-break, ...),
builds it, and checks that at least one pin fails.  Nothing of this touches a GPU.
"""
import os
import shutil

import pytest

import oracle
import pins

ORACLE_SRC = os.path.join(os.path.dirname(oracle.__file__), "hq_oracle.c")


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.get())


# (name, text in hq_oracle.c, replacement)
MUTANTS = [
    ("ema_decay_swapped", "float a = beta * ema_min[i];", "float a = one_minus_beta * ema_min[i];"),
    ("first_batch_ignored", "if (first_batch) {", "if (0) {"),
    ("calib_drops_last_row", "for (int t = 0; t < T; ++t) {\n        float v", "for (int t = 0; t < T - 1; ++t) {\n        float v"),
    ("zero_not_in_range", "float lo = (ema_min[i] < 0.0f) ? ema_min[i] : 0.0f;", "float lo = ema_min[i];"),
    ("scale_over_16", "float s = rg / 15.0f;", "float s = rg / 16.0f;"),
    ("zero_point_floor", "float zf = rintf((-lo) * inv);", "float zf = floorf((-lo) * inv);"),
    ("score_max_not_sum", "acc = acc + range[(size_t)r * H + h];",
     "acc = (range[(size_t)r * H + h] > acc) ? range[(size_t)r * H + h] : acc;"),
    ("ties_to_higher_col", "return (a->col < b->col) ? -1 : (a->col > b->col) ? 1 : 0;",
     "return (a->col < b->col) ? 1 : (a->col > b->col) ? -1 : 0;"),
    ("keep_not_sorted", "qsort(keep_idx, (size_t)k, sizeof(int32_t), ref_ascending);", ""),
    ("rint_after_zero", "float n = rintf(a);", "float n = rintf(a + (float)zero) - (float)zero;"),
    ("nan_to_code_0", "if (isnan(a)) return zero;", "if (isnan(a)) return 0u;"),
    ("nibbles_reversed", "crow[c / 8] |= (uint32_t)q << (4 * (c % 8));", "crow[c / 8] |= (uint32_t)q << (4 * (7 - c % 8));"),
    ("side_from_rest", "* T + t] = row[keep_idx[j]];", "* T + t] = row[rest_idx[j]];"),
    ("side_row_major", "side[((size_t)r * k + j) * T + t] = row", "side[((size_t)r * T + t) * k + j] = row"),
    ("reduce_drops_last_rank", "for (int r = 0; r < P; ++r) {\n        uint32_t word",
     "for (int r = 0; r < P - 1; ++r) {\n        uint32_t word"),
    ("dequant_sign_flipped", "acc = fmaf((float)(q - (int)zero[p])", "acc = fmaf((float)((int)zero[p] - q)"),
    ("kept_sum_rank0_only", "for (int r = 0; r < P; ++r) acc = acc + ref_bf16_value(side",
     "for (int r = 0; r < 1; ++r) acc = acc + ref_bf16_value(side"),
    ("fp32_nan_payload_kept", "if (!isnan(f)) return f;", "return f;"),
    ("bf16_truncates", "if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u))) keep += 1u;", ""),
    ("bf16_shards_not_rounded", "acc = acc + ref_bf16_value(ref_bf16_round(v));", "acc = acc + v;"),
    ("bf16_shards_truncated", "acc = acc + ref_bf16_value(ref_bf16_round(v));",
     "uint32_t u; memcpy(&u, &v, sizeof u); acc = acc + ref_bf16_value((uint16_t)(u >> 16));"),
    ("bf16_shards_rounds_the_sum", "acc = acc + ref_bf16_value(ref_bf16_round(v));",
     "acc = ref_bf16_value(ref_bf16_round(acc + v));"),
    ("bf16_shards_sign_flipped", "float v = (float)(q - (int)zero[p]) * scale[p];",
     "float v = (float)((int)zero[p] - q) * scale[p];"),
    # rounding and order choices of the readings R1, R3, R4, R9, R10
    ("dequant_mul_then_add", "acc = fmaf((float)(q - (int)zero[p]), scale[p], acc);",
     "acc = acc + (float)(q - (int)zero[p]) * scale[p];"),
    ("dequant_exact_accumulator", "acc = fmaf((float)(q - (int)zero[p]), scale[p], acc);",
     "static double dacc; if (r == 0) dacc = 0.0; dacc += (double)(q - (int)zero[p]) * scale[p]; acc = (float)dacc;"),
    ("dequant_ranks_reversed", "for (int r = 0; r < P; ++r) {\n        uint32_t word",
     "for (int r = P - 1; r >= 0; --r) {\n        uint32_t word"),
    ("kept_ranks_reversed", "for (int r = 0; r < P; ++r) acc = acc + ref_bf16_value(side",
     "for (int r = P - 1; r >= 0; --r) acc = acc + ref_bf16_value(side"),
    ("score_ranks_reversed", "for (int r = 0; r < P; ++r) acc = acc + range[(size_t)r * H + h];",
     "for (int r = P - 1; r >= 0; --r) acc = acc + range[(size_t)r * H + h];"),
    ("score_in_double", "float acc = 0.0f;\n    for (int r = 0; r < P; ++r) acc = acc + range[(size_t)r * H + h];",
     "double dacc = 0.0;\n    for (int r = 0; r < P; ++r) dacc = dacc + range[(size_t)r * H + h];\n    float acc = (float)dacc;"),
    ("decay_complement_literal", "const float one_minus_beta = 1.0f - beta;", "const float one_minus_beta = 0.1f;"),
    ("ema_fused_update", "a = beta * ema_max[i];\n        b = one_minus_beta * bmax;\n        ema_max[i] = a + b;",
     "ema_max[i] = fmaf(beta, ema_max[i], one_minus_beta * bmax);"),
    ("ema_delta_form", "a = beta * ema_max[i];\n        b = one_minus_beta * bmax;\n        ema_max[i] = a + b;",
     "ema_max[i] = ema_max[i] + one_minus_beta * (bmax - ema_max[i]);"),
    ("ema_in_double", "a = beta * ema_max[i];\n        b = one_minus_beta * bmax;\n        ema_max[i] = a + b;",
     "ema_max[i] = (float)((double)beta * ema_max[i] + (double)one_minus_beta * bmax);"),
    ("inv_scale_15_over_range", "float inv = 1.0f / s;", "float inv = 15.0f / rg;"),
    ("scale_times_reciprocal", "float s = rg / 15.0f;", "float s = rg * (1.0f / 15.0f);"),
    # partial-channel synchronisation (R20)
    ("partial_sync_block_shifted", "y[((size_t)r * T + t) * H + c0 + h] = red[(size_t)t * Hs + h];",
     "y[((size_t)r * T + t) * H + (c0 + h + 1) % H] = red[(size_t)t * Hs + h];"),
    ("partial_sync_outside_zeroed", "for (size_t i = 0; i < rows * (size_t)H; ++i) y[i] = x[i];",
     "for (size_t i = 0; i < rows * (size_t)H; ++i) y[i] = 0;"),
    ("partial_sync_rank0_outside", "for (size_t i = 0; i < rows * (size_t)H; ++i) y[i] = x[i];",
     "for (size_t i = 0; i < rows * (size_t)H; ++i) y[i] = x[i % ((size_t)T * H)];"),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    d = tmp_path_factory.mktemp("oracle_mutants")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(mutant_dir, name, old, new):
    src = open(ORACLE_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = mutant_dir / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = str(mutant_dir / f"lib_{name}.so")
    import subprocess

    subprocess.run(["gcc", *oracle.CFLAGS, str(path), "-o", so, "-lm"], check=True)
    mutant = oracle.Oracle(so)
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            return
    pytest.fail(f"no pin caught the planted mistake {name}")
