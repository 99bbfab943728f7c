"""Seeded synthetic tensor-parallel partial sums, the inputs of both the oracle and the CUDA path.

This module holds none of the compression method's arithmetic: it only makes inputs.  The
workloads follow the page "Revolutionizing LLM Inference: The Power of Efficient Low-Bit
Communication": per-rank partial sums of a row-parallel layer ("Combating Quantization Errors
with Tensor Parallelism") whose features have a consistent structure with a few columns of
enormous range ("Leveraging Outliers for Efficient Communication").  The trained models of
"Experimental Validation and Results" are not available, so these seeded synthetic tensors
stand in for their activations.

Each value is a pure function of (seed, purpose, batch, rank, row, column), computed by the
same C code on the host (``libhqsynth.so``) and on the GPU (``libhqsynth_gpu.so``), so a test
can regenerate any element of a full-size GPU batch on the CPU.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_DIR, "libhqsynth.so")
_GPU_SO = os.path.join(_DIR, "libhqsynth_gpu.so")

CALIB = 3
EVAL = 4
DIST = {"normal": 0, "student_t3": 1, "uniform": 2}


@dataclass(frozen=True)
class Config:
    """One synthetic workload: P simulated ranks, each with a bf16 partial sum [T, H]."""

    name: str
    P: int
    T: int
    H: int
    k: int
    seed: int
    dist: str = "normal"
    sigma: float = 0.5          # column std ~ LogNormal(0, sigma)
    n_out: int = 0              # planted outlier columns (shared by all ranks and batches)
    out_mult: float = 1.0       # their std multiplier
    spike_p: float = 0.0        # iid spike probability per element
    spike_mult: float = 1.0
    calib_batches: int = 4
    calib_T: int = 16           # rows per calibration batch
    beta: float = 0.9           # moving-average decay

    @property
    def elements(self) -> int:
        return self.P * self.T * self.H

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS = {
    "pr1": Config("pr1", P=2, T=16, H=256, k=8, seed=0, sigma=0.5, n_out=8, out_mult=50.0,
                  calib_batches=4, calib_T=16),
    "decode": Config("decode", P=4, T=32, H=4096, k=64, seed=1, sigma=0.5, n_out=32, out_mult=100.0,
                     spike_p=0.001, spike_mult=20.0, calib_batches=16, calib_T=32),
    "prefill7b": Config("prefill7b", P=8, T=4096, H=4096, k=128, seed=2, sigma=0.7, n_out=64,
                        out_mult=200.0, calib_batches=32, calib_T=4096),
    "prefill70b": Config("prefill70b", P=8, T=8192, H=8192, k=256, seed=3, dist="student_t3", sigma=0.7,
                         n_out=128, out_mult=300.0, calib_batches=32, calib_T=8192),
}


def sweep_configs() -> list[Config]:
    """The 90-point bandwidth sweep: uniform U(-1,1) partial sums, no outlier structure.

    Calibration: 8 batches of 256 rows each (the sweep's batch shape is not specified
    elsewhere, so this is the reading taken), decay 0.9.
    """
    out = []
    i = 0
    for P in (2, 4, 8):
        for H in (4096, 8192):
            for T in (1, 64, 512, 4096, 16384):
                for frac in (0, 64, 32):
                    k = 0 if frac == 0 else H // frac
                    out.append(Config(f"sweep_P{P}_H{H}_T{T}_k{k}", P=P, T=T, H=H, k=k, seed=4 + i,
                                      dist="uniform", sigma=0.0, calib_batches=8, calib_T=256))
                    i += 1
    return out


def build(verbose: bool = False) -> None:
    """Compile the host generator (gcc) and the device generator (nvcc, sm_100a)."""
    host = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
            "-fopenmp", os.path.join(_DIR, "hq_synth.c"), "-o", _HOST_SO, "-lm"]
    dev = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-fmad=false",
           "-Xcompiler", "-fPIC", "-shared", os.path.join(_DIR, "hq_synth_gpu.cu"), "-o", _GPU_SO]
    for cmd in (host, dev):
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)


_host = None
_gpu = None


def _load_host():
    global _host
    if _host is None:
        if not os.path.exists(_HOST_SO):
            raise RuntimeError(f"{_HOST_SO} is missing: run synth.build()")
        lib = ctypes.CDLL(_HOST_SO)
        u64, i32, dbl = ctypes.c_uint64, ctypes.c_int, ctypes.c_double
        vp = ctypes.c_void_p
        lib.syn_colscale.argtypes = [u64, i32, dbl, i32, dbl, vp, vp]
        lib.syn_colscale.restype = i32
        lib.syn_fill.argtypes = [u64, i32, i32, i32, i32, vp, dbl, dbl, i32, i32, i32, i32, i32, i32, vp]
        lib.syn_fill.restype = None
        lib.syn_one.argtypes = [u64, i32, i32, i32, i32, dbl, dbl, dbl, i32, i32, i32]
        lib.syn_one.restype = ctypes.c_uint16
        lib.syn_log_for_test.argtypes = [dbl]
        lib.syn_log_for_test.restype = dbl
        lib.syn_cos2pi_for_test.argtypes = [dbl]
        lib.syn_cos2pi_for_test.restype = dbl
        _host = lib
    return _host


def _load_gpu():
    global _gpu
    if _gpu is None:
        if not os.path.exists(_GPU_SO):
            raise RuntimeError(f"{_GPU_SO} is missing: run synth.build()")
        lib = ctypes.CDLL(_GPU_SO)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.syn_fill_gpu.argtypes = [u64, i32, i32, i32, i32, i32, i32, vp, dbl, dbl, vp, vp]
        lib.syn_fill_gpu.restype = i32
        _gpu = lib
    return _gpu


def colscale(cfg: Config) -> tuple[np.ndarray, np.ndarray]:
    """Per-column scale (float64 [H]) and the planted outlier columns (int32 [n_out])."""
    cs = np.empty(cfg.H, dtype=np.float64)
    outl = np.empty(max(cfg.n_out, 1), dtype=np.int32)
    rc = _load_host().syn_colscale(cfg.seed, cfg.H, cfg.sigma, cfg.n_out, cfg.out_mult,
                                   cs.ctypes.data, outl.ctypes.data)
    if rc != 0:
        raise ValueError(f"syn_colscale failed ({rc})")
    if cfg.dist == "uniform":
        cs[:] = 1.0
    return cs, outl[: cfg.n_out].copy()


def fill_cpu(cfg: Config, purpose: int, batch: int, ranks=None, rows=None, cols=None,
             T: int | None = None, cs: np.ndarray | None = None) -> np.ndarray:
    """A block of batch (purpose, batch) as uint16 bf16 bits, shape [nr, nt, nh]."""
    T = cfg.T if T is None else T
    r0, r1 = ranks if ranks is not None else (0, cfg.P)
    t0, t1 = rows if rows is not None else (0, T)
    h0, h1 = cols if cols is not None else (0, cfg.H)
    if not (0 <= r0 <= r1 <= cfg.P and 0 <= t0 <= t1 <= T and 0 <= h0 <= h1 <= cfg.H):
        raise ValueError("block outside the tensor")
    if cs is None:
        cs = colscale(cfg)[0]
    out = np.empty((r1 - r0, t1 - t0, h1 - h0), dtype=np.uint16)
    _load_host().syn_fill(cfg.seed, purpose, batch, cfg.H, DIST[cfg.dist], cs.ctypes.data,
                          cfg.spike_p, cfg.spike_mult, r0, r1, t0, t1, h0, h1, out.ctypes.data)
    return out


def one(cfg: Config, purpose: int, batch: int, r: int, t: int, h: int, cs: np.ndarray) -> int:
    return int(_load_host().syn_one(cfg.seed, purpose, batch, cfg.H, DIST[cfg.dist], float(cs[h]),
                                    cfg.spike_p, cfg.spike_mult, r, t, h))


def fill_gpu(cfg: Config, purpose: int, batch: int, out, cs_dev, T: int | None = None, stream=None) -> None:
    """Fill a contiguous device tensor ``out`` (int16/uint16 [P, T, H]) with batch (purpose, batch).

    ``cs_dev`` is the column scale as a float64 device tensor; ``out`` and ``cs_dev`` are torch
    tensors (torch is only plumbing here).
    """
    import torch

    T = cfg.T if T is None else T
    if out.numel() != cfg.P * T * cfg.H or not out.is_contiguous() or out.element_size() != 2:
        raise ValueError("out must be a contiguous 2-byte tensor of P*T*H elements")
    if stream is None:
        stream = torch.cuda.current_stream(out.device).cuda_stream
    rc = _load_gpu().syn_fill_gpu(cfg.seed, purpose, batch, cfg.P, T, cfg.H, DIST[cfg.dist],
                                  cs_dev.data_ptr(), cfg.spike_p, cfg.spike_mult, out.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"syn_fill_gpu failed ({rc})")


def log_series(x: float) -> float:
    return _load_host().syn_log_for_test(x)


def cos2pi_series(u: float) -> float:
    return _load_host().syn_cos2pi_for_test(u)
