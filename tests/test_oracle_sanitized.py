"""The oracle under the host sanitizers: built with AddressSanitizer and UndefinedBehaviorSanitizer
(no recovery), then run through the pins that call every one of its functions, in a child process
with the sanitizer runtimes preloaded.  An out-of-bounds access, a use after free, a signed
overflow or any other undefined behaviour in the oracle aborts the child and fails the test.
(compute-sanitizer is not used on the GPU side; its role there is played by the guard-band and
bad-index tests.)"""
import os
import shutil
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PINS = ["pin_bf16_round", "pin_quantize_golden", "pin_quantize_nearest_grid", "pin_params_golden",
        "pin_params_closed_form", "pin_calibrate_single_batch", "pin_calibrate_ema_golden", "pin_select_golden",
        "pin_select_rank_order_golden", "pin_select_brute_force", "pin_pack_golden", "pin_pack_unpack",
        "pin_reduce_all_kept", "pin_nan_outputs", "pin_reduce_dequant_sum", "pin_reduce_order_golden",
        "pin_bf16_shards_golden", "pin_bf16_shards_exact_products", "pin_bf16_shards_rounding_bound",
        "pin_partial_sync_golden", "pin_partial_sync_extremes"]

_CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import oracle, pins
o = oracle.Oracle(sys.argv[2])
for name in sys.argv[3:]:
    getattr(pins, name)(o)
print("SANITIZED_OK", len(sys.argv) - 3, flush=True)
"""


def _runtime(name):
    p = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


def _sanitized_run(tmp_path, source_text, pins):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not installed")
    src = tmp_path / "hq_oracle.c"
    src.write_text(source_text)
    so = str(tmp_path / "libhq_oracle_sanitized.so")
    flags = [f for f in oracle.CFLAGS if not f.startswith("-O")]
    subprocess.run(["gcc", "-O1", "-g", *flags, "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
                    "-fno-omit-frame-pointer", str(src), "-o", so, "-lm"], check=True)
    env = dict(os.environ, LD_PRELOAD=f"{asan}:{ubsan}", ASAN_OPTIONS="detect_leaks=0:abort_on_error=1",
               UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1")
    return subprocess.run([sys.executable, "-c", _CHILD, ROOT, so, *pins], capture_output=True, text=True, env=env,
                          timeout=600)


ORACLE_SRC = os.path.join(ROOT, "oracle", "hq_oracle.c")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_oracle_under_asan_and_ubsan(tmp_path):
    r = _sanitized_run(tmp_path, open(ORACLE_SRC).read(), PINS)
    assert r.returncode == 0 and f"SANITIZED_OK {len(PINS)}" in r.stdout, (r.stdout + r.stderr)[-4000:]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_a_planted_overflow_is_reported(tmp_path):
    """The same build with a one-word overrun of a code row planted: the sanitizer must stop it."""
    src = open(ORACLE_SRC).read()
    old = "for (int w = 0; w < W; ++w) crow[w] = 0u;"
    assert src.count(old) == 1
    r = _sanitized_run(tmp_path, src.replace(old, "for (int w = 0; w <= W; ++w) crow[w] = 0u;"), ["pin_pack_unpack"])
    assert r.returncode != 0 and "AddressSanitizer" in r.stderr, (r.stdout + r.stderr)[-2000:]
