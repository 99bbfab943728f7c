"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and compute the
oracle's expectations on the same seeded inputs.  Imported only by tests marked ``gpu``."""
from __future__ import annotations

import numpy as np
import torch

import bit_tensor_activation_b200 as hq
import oracle
import synth

DEV = torch.device("cuda:0")


def to_dev_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def f32bits(t) -> np.ndarray:
    a = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def params_to_dev(sel: dict) -> dict:
    return dict(
        keep_idx=torch.from_numpy(sel["keep_idx"]).to(DEV),
        rest_idx=torch.from_numpy(sel["rest_idx"]).to(DEV),
        scale=torch.from_numpy(sel["scale"]).to(DEV),
        inv_scale=torch.from_numpy(sel["inv_scale"]).to(DEV),
        zero=torch.from_numpy(sel["zero"]).to(DEV),
    )


def gpu_calibrate_batches(batches, beta, P, H):
    emin = torch.empty((P, H), dtype=torch.float32, device=DEV)
    emax = torch.empty((P, H), dtype=torch.float32, device=DEV)
    for b, x in enumerate(batches):
        hq.hq_calibrate(x if isinstance(x, torch.Tensor) else to_dev_u16(x), emin, emax, beta, b == 0)
    return emin, emax


def gpu_select(emin, emax, k):
    P, H = emin.shape
    B = dict(keep_idx=torch.empty(k, dtype=torch.int32, device=DEV),
             rest_idx=torch.empty(H - k, dtype=torch.int32, device=DEV),
             scale=torch.empty((P, H), dtype=torch.float32, device=DEV),
             inv_scale=torch.empty((P, H), dtype=torch.float32, device=DEV),
             zero=torch.empty((P, H), dtype=torch.uint8, device=DEV))
    hq.hq_select_topk(emin, emax, k, B["keep_idx"], B["rest_idx"], B["scale"], B["inv_scale"], B["zero"])
    return B


def gpu_quantize(x, prm):
    P, T, H = x.shape
    k = prm["keep_idx"].shape[0]
    codes = torch.empty((P, T, (H - k) // 8), dtype=torch.int32, device=DEV)
    side = torch.empty((P, k, T), dtype=torch.int16, device=DEV)
    hq.hq_quantize_pack(x, prm["keep_idx"], prm["rest_idx"], prm["inv_scale"], prm["zero"], codes, side)
    return codes, side


def gpu_dequant(codes, side, prm, H, out_f32=False, bf16_shards=False):
    T = codes.shape[1]
    out = torch.empty((T, H), dtype=torch.float32 if out_f32 else torch.int16, device=DEV)
    fn = hq.hq_dequant_reduce_bf16_shards if bf16_shards else hq.hq_dequant_reduce
    fn(codes, side, prm["keep_idx"], prm["rest_idx"], prm["scale"], prm["zero"], out)
    return out


def gpu_fused(x, prm, out_f32=False, wire=False):
    P, T, H = x.shape
    k = prm["keep_idx"].shape[0]
    out = torch.empty((T, H), dtype=torch.float32 if out_f32 else torch.int16, device=DEV)
    codes = side = None
    if wire:
        codes = torch.empty((P, T, (H - k) // 8), dtype=torch.int32, device=DEV)
        side = torch.empty((P, k, T), dtype=torch.int16, device=DEV)
    hq.hq_compress_reduce(x, prm["keep_idx"], prm["rest_idx"], prm["scale"], prm["inv_scale"], prm["zero"],
                          out, codes, side)
    return out, codes, side


def assert_same(got: np.ndarray, want: np.ndarray, what: str):
    """Bit equality with the first differing element reported."""
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} of {got.size} differ; first at {i}: "
                             f"got {got[i]!r} (0x{int(got[i]):X}) want {want[i]!r} (0x{int(want[i]):X})")


def assert_no_device_error():
    st = hq.hq_read_device_error()
    assert st == hq.HQ_OK, hq.hq_status_string(st)


def oracle_pipeline(cfg: synth.Config, cal, x):
    """Oracle results for calibration batches `cal` and evaluation batch `x` (numpy)."""
    o = oracle.get()
    emin, emax = o.calibrate_batches(cal, cfg.beta)
    sel = o.select_topk(emin, emax, cfg.k)
    codes, side = o.quantize_pack(x, sel["keep_idx"], sel["rest_idx"], sel["inv_scale"], sel["zero"])
    out_b = o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"])
    out_f = o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                             out_f32=True)
    lit_b = o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                             bf16_shards=True)
    lit_f = o.dequant_reduce(codes, side, cfg.H, sel["keep_idx"], sel["rest_idx"], sel["scale"], sel["zero"],
                             out_f32=True, bf16_shards=True)
    return dict(emin=emin, emax=emax, sel=sel, codes=codes, side=side, out_b=out_b, out_f=out_f,
                lit_b=lit_b, lit_f=lit_f)


def compare_all(cfg, cal, x_np):
    """Whole path on the GPU vs the oracle, element by element."""
    ref = oracle_pipeline(cfg, cal, x_np)
    emin, emax = gpu_calibrate_batches(cal, cfg.beta, cfg.P, cfg.H)
    B = gpu_select(emin, emax, cfg.k)
    x = to_dev_u16(x_np)
    codes, side = gpu_quantize(x, B)
    out_b = gpu_dequant(codes, side, B, cfg.H)
    out_f = gpu_dequant(codes, side, B, cfg.H, out_f32=True)
    lit_b = gpu_dequant(codes, side, B, cfg.H, bf16_shards=True)
    lit_f = gpu_dequant(codes, side, B, cfg.H, out_f32=True, bf16_shards=True)
    fb, _, _ = gpu_fused(x, B)
    ff, wc, ws = gpu_fused(x, B, out_f32=True, wire=True)
    assert_no_device_error()
    assert_same(f32bits(emin), f32bits(ref["emin"]), "ema_min")
    assert_same(f32bits(emax), f32bits(ref["emax"]), "ema_max")
    assert_same(B["keep_idx"].cpu().numpy(), ref["sel"]["keep_idx"], "keep_idx")
    assert_same(B["rest_idx"].cpu().numpy(), ref["sel"]["rest_idx"], "rest_idx")
    assert_same(f32bits(B["scale"]), f32bits(ref["sel"]["scale"]), "scale")
    assert_same(f32bits(B["inv_scale"]), f32bits(ref["sel"]["inv_scale"]), "inv_scale")
    assert_same(B["zero"].cpu().numpy(), ref["sel"]["zero"], "zero")
    assert_same(u32(codes), ref["codes"], "codes")
    assert_same(u16(side), ref["side"], "side")
    assert_same(u16(out_b), ref["out_b"], "out bf16")
    assert_same(f32bits(out_f), f32bits(ref["out_f"]), "out f32")
    assert_same(u16(lit_b), ref["lit_b"], "bf16-shard reduction, bf16 out")
    assert_same(f32bits(lit_f), f32bits(ref["lit_f"]), "bf16-shard reduction, f32 out")
    assert_same(u16(fb), ref["out_b"], "fused bf16")
    assert_same(f32bits(ff), f32bits(ref["out_f"]), "fused f32")
    assert_same(u32(wc), ref["codes"], "fused wire codes")
    assert_same(u16(ws), ref["side"], "fused wire side")
    return ref
