"""CPU oracle for the hybrid BF16/Int4 compression of tensor-parallel partial sums.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  It wraps ``libhq_oracle.so``, a plain
single-threaded C restatement (``hq_oracle.c``) of the page "Revolutionizing LLM Inference: The
Power of Efficient Low-Bit Communication", section "The Hybrid Quantization Algorithm".  It
shares no code with the CUDA path and never imports it.

Every function takes and returns numpy arrays:
  x         uint16 [P, T, H]   bf16 bits of the P ranks' partial sums
  ema_*     float32 [P, H]
  keep_idx  int32 [k], rest_idx int32 [H-k] (both ascending)
  scale, inv_scale float32 [P, H]; zero uint8 [P, H]
  codes     uint32 [P, T, (H-k)/8]; side uint16 [P, k, T] (feature-major)
  out       uint16 [T, H] (bf16 bits) or float32 [T, H]
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_DIR, "libhq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(verbose: bool = False, extra_flags=(), out: str | None = None) -> str:
    """Compile hq_oracle.c with gcc; returns the path of the shared library."""
    out = out or _SO
    cmd = ["gcc", *CFLAGS, *extra_flags, os.path.join(_DIR, "hq_oracle.c"), "-o", out, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return out


class Oracle:
    """ctypes view of one build of the oracle library (the default one, or a test variant)."""

    def __init__(self, path: str = _SO):
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run oracle.build()")
        lib = ctypes.CDLL(path)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        lib.hq_ref_calibrate.argtypes = [vp, i32, i32, i32, f32, i32, vp, vp]
        lib.hq_ref_calibrate.restype = None
        lib.hq_ref_params.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp]
        lib.hq_ref_params.restype = None
        lib.hq_ref_select.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        lib.hq_ref_select.restype = i32
        lib.hq_ref_select_topk.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.hq_ref_select_topk.restype = i32
        lib.hq_ref_quantize_pack.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.hq_ref_quantize_pack.restype = None
        lib.hq_ref_dequant_reduce.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32]
        lib.hq_ref_dequant_reduce.restype = None
        lib.hq_ref_dequant_reduce_bf16_shards.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32]
        lib.hq_ref_dequant_reduce_bf16_shards.restype = None
        lib.hq_ref_compress_reduce.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp]
        lib.hq_ref_compress_reduce.restype = i32
        lib.hq_ref_partial_sync.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.hq_ref_partial_sync.restype = i32
        lib.hq_ref_bf16_round.argtypes = [f32]
        lib.hq_ref_bf16_round.restype = ctypes.c_uint16
        lib.hq_ref_quantize_one.argtypes = [f32, f32, ctypes.c_uint]
        lib.hq_ref_quantize_one.restype = ctypes.c_uint
        self.lib = lib

    # -- Calibration ------------------------------------------------------------------------
    def calibrate(self, x, beta, first_batch, ema_min=None, ema_max=None):
        """Fold one batch x [P, T, H] into the moving averages; returns (ema_min, ema_max)."""
        x = _c(x, np.uint16)
        P, T, H = x.shape
        if first_batch:
            ema_min = np.zeros((P, H), np.float32)
            ema_max = np.zeros((P, H), np.float32)
        else:
            ema_min = _c(ema_min, np.float32).copy()
            ema_max = _c(ema_max, np.float32).copy()
        self.lib.hq_ref_calibrate(_p(x), P, T, H, float(beta), int(bool(first_batch)), _p(ema_min), _p(ema_max))
        return ema_min, ema_max

    # -- Selection of High Precision Features ------------------------------------------------
    def params(self, ema_min, ema_max):
        ema_min, ema_max = _c(ema_min, np.float32), _c(ema_max, np.float32)
        P, H = ema_min.shape
        scale = np.empty((P, H), np.float32)
        inv = np.empty((P, H), np.float32)
        zero = np.empty((P, H), np.uint8)
        rng = np.empty((P, H), np.float32)
        self.lib.hq_ref_params(_p(ema_min), _p(ema_max), P, H, _p(scale), _p(inv), _p(zero), _p(rng))
        return scale, inv, zero, rng

    def select(self, rng, k):
        rng = _c(rng, np.float32)
        P, H = rng.shape
        score = np.empty(H, np.float32)
        keep = np.empty(max(k, 1), np.int32)
        rest = np.empty(max(H - k, 1), np.int32)
        if self.lib.hq_ref_select(_p(rng), P, H, k, _p(score), _p(keep), _p(rest)) != 0:
            raise ValueError("hq_ref_select failed")
        return keep[:k].copy(), rest[: H - k].copy(), score

    def select_topk(self, ema_min, ema_max, k):
        """Returns dict(keep_idx, rest_idx, scale, inv_scale, zero, score)."""
        ema_min, ema_max = _c(ema_min, np.float32), _c(ema_max, np.float32)
        P, H = ema_min.shape
        keep = np.empty(max(k, 1), np.int32)
        rest = np.empty(max(H - k, 1), np.int32)
        scale = np.empty((P, H), np.float32)
        inv = np.empty((P, H), np.float32)
        zero = np.empty((P, H), np.uint8)
        score = np.empty(H, np.float32)
        rc = self.lib.hq_ref_select_topk(_p(ema_min), _p(ema_max), P, H, k, _p(keep), _p(rest),
                                         _p(scale), _p(inv), _p(zero), _p(score))
        if rc != 0:
            raise ValueError("hq_ref_select_topk failed")
        return dict(keep_idx=keep[:k].copy(), rest_idx=rest[: H - k].copy(), scale=scale,
                    inv_scale=inv, zero=zero, score=score)

    # -- Inference -----------------------------------------------------------------------------
    def quantize_pack(self, x, keep_idx, rest_idx, inv_scale, zero):
        x = _c(x, np.uint16)
        P, T, H = x.shape
        k = len(keep_idx)
        keep, rest = _c(keep_idx, np.int32), _c(rest_idx, np.int32)
        inv, zero = _c(inv_scale, np.float32), _c(zero, np.uint8)
        codes = np.empty((P, T, (H - k) // 8), np.uint32)
        side = np.empty((P, k, T), np.uint16)
        self.lib.hq_ref_quantize_pack(_p(x), P, T, H, k, _p(keep), _p(rest), _p(inv), _p(zero),
                                      _p(codes), _p(side))
        return codes, side

    def dequant_reduce(self, codes, side, H, keep_idx, rest_idx, scale, zero, out_f32=False, bf16_shards=False):
        """R9/R10/R11; bf16_shards=True: the literal variant R19 (each rank's dequantized value
        rounded to bf16 before the rank-ordered sum)."""
        codes, side = _c(codes, np.uint32), _c(side, np.uint16)
        P, T = codes.shape[0], codes.shape[1]
        k = len(keep_idx)
        keep, rest = _c(keep_idx, np.int32), _c(rest_idx, np.int32)
        scale, zero = _c(scale, np.float32), _c(zero, np.uint8)
        out = np.empty((T, H), np.float32 if out_f32 else np.uint16)
        fn = self.lib.hq_ref_dequant_reduce_bf16_shards if bf16_shards else self.lib.hq_ref_dequant_reduce
        fn(_p(codes), _p(side), P, T, H, k, _p(keep), _p(rest), _p(scale), _p(zero), _p(out), int(bool(out_f32)))
        return out

    def compress_reduce(self, x, keep_idx, rest_idx, scale, inv_scale, zero, out_f32=False):
        x = _c(x, np.uint16)
        P, T, H = x.shape
        k = len(keep_idx)
        keep, rest = _c(keep_idx, np.int32), _c(rest_idx, np.int32)
        scale, inv, zero = _c(scale, np.float32), _c(inv_scale, np.float32), _c(zero, np.uint8)
        out = np.empty((T, H), np.float32 if out_f32 else np.uint16)
        rc = self.lib.hq_ref_compress_reduce(_p(x), P, T, H, k, _p(keep), _p(rest), _p(scale), _p(inv),
                                             _p(zero), _p(out), int(bool(out_f32)), None, None)
        if rc != 0:
            raise MemoryError("hq_ref_compress_reduce failed")
        return out

    def partial_sync(self, x, c0, Hs, keep_idx, rest_idx, scale, inv_scale, zero):
        """R20: every rank's output [P, T, H]: the reduced block [c0, c0 + Hs) (bf16), its own
        partial sum elsewhere.  keep/rest index the block; scale/inv_scale/zero are [P, Hs]."""
        x = _c(x, np.uint16)
        P, T, H = x.shape
        k = len(keep_idx)
        keep, rest = _c(keep_idx, np.int32), _c(rest_idx, np.int32)
        scale, inv, zero = _c(scale, np.float32), _c(inv_scale, np.float32), _c(zero, np.uint8)
        y = np.empty_like(x)
        if self.lib.hq_ref_partial_sync(_p(x), P, T, H, c0, Hs, k, _p(keep), _p(rest), _p(scale), _p(inv),
                                        _p(zero), _p(y)) != 0:
            raise ValueError("hq_ref_partial_sync failed")
        return y

    def bf16_round(self, f: float) -> int:
        return int(self.lib.hq_ref_bf16_round(f))

    def quantize_one(self, v: float, inv_scale: float, zero: int) -> int:
        return int(self.lib.hq_ref_quantize_one(v, inv_scale, zero))

    # -- The whole path on one batch -----------------------------------------------------------
    def calibrate_batches(self, batches, beta):
        ema_min = ema_max = None
        for b, x in enumerate(batches):
            ema_min, ema_max = self.calibrate(x, beta, b == 0, ema_min, ema_max)
        return ema_min, ema_max


def _c(a, dtype):
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def _p(a):
    return a.ctypes.data if a is not None else None


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from the committed source (built on first use if missing)."""
    global _default
    if _default is None:
        if not os.path.exists(_SO):
            build()
        _default = Oracle(_SO)
    return _default
