"""Python binding of libhq.so: hybrid BF16/Int4 compression of tensor-parallel partial sums on B200.

Thin ctypes marshalling over the C ABI in ``include/hq.h``; every step of the path runs in the
library's CUDA kernels.  The functions carry the C names and take torch tensors (torch is only
used for device memory and streams): each tensor is checked for device, dtype, shape and
contiguity, and its data pointer is passed with the current CUDA stream.  A nonzero status
raises ``HQError``.  There is no CPU fallback: importing this package on a machine without the
built ``libhq.so`` raises.

Shapes (P ranks, T rows, H features, k kept features, H' = H - k):
  x [P, T, H] bf16; ema_min/ema_max [P, H] f32; keep_idx [k] i32; rest_idx [H'] i32;
  scale/inv_scale [P, H] f32; zero [P, H] u8; codes [P, T, H'/8] i32 (bit pattern of uint32);
  side [P, k, T] bf16 (feature-major); out [T, H] bf16 or f32.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python bit_tensor_activation_b200/build.py` "
                      "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_lib.hq_calibrate.argtypes = [_vp, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp]
_lib.hq_select_topk.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.hq_quantize_pack.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.hq_dequant_reduce.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
_lib.hq_dequant_reduce_bf16_shards.argtypes = _lib.hq_dequant_reduce.argtypes
_lib.hq_compress_reduce.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                    _vp, _vp, _vp]
for _f in ("hq_calibrate", "hq_select_topk", "hq_quantize_pack", "hq_dequant_reduce",
           "hq_dequant_reduce_bf16_shards", "hq_compress_reduce", "hq_read_device_error"):
    getattr(_lib, _f).restype = _i32
_lib.hq_read_device_error.argtypes = [_vp]
_lib.hq_status_string.argtypes = [_i32]
_lib.hq_status_string.restype = ctypes.c_char_p
_lib.hq_selftest_bounded_wait.argtypes = [ctypes.c_longlong, _vp]
_lib.hq_selftest_bounded_wait.restype = _i32
_lib.hq_dequant_reduce_ranks.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
_lib.hq_dequant_reduce_ranks.restype = _i32
_lib.hq_two_step_reduce.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp,
                                    _vp, _vp, ctypes.c_size_t, _vp, _i32, _vp]
_lib.hq_two_step_reduce.restype = _i32
_lib.hq_two_step_reduce_noalloc.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                            _vp, _vp, _vp, _vp, _i32, _vp]
_lib.hq_two_step_reduce_noalloc.restype = _i32
_lib.hq_two_step_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32]
_lib.hq_two_step_workspace_bytes.restype = ctypes.c_size_t
_lib.hq_calibrate_ld.argtypes = [_vp, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp]
_lib.hq_quantize_pack_ld.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.hq_dequant_reduce_ld.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp]
_lib.hq_compress_reduce_ld.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                       _vp, _vp, _vp]
for _f in ("hq_calibrate_ld", "hq_quantize_pack_ld", "hq_dequant_reduce_ld", "hq_compress_reduce_ld"):
    getattr(_lib, _f).restype = _i32
_lib.hq_selftest_set_pipeline_stall.argtypes = [ctypes.c_longlong, ctypes.c_longlong]
_lib.hq_selftest_set_pipeline_stall.restype = _i32
_lib.hq_wire_bytes_per_row.argtypes = [_i32, _i32]
_lib.hq_wire_bytes_per_row.restype = ctypes.c_int64

HQ_OK, HQ_ERR_INVALID_ARG, HQ_ERR_MISALIGNED, HQ_ERR_CUDA, HQ_ERR_TIMEOUT, HQ_ERR_BAD_INDEX = range(6)
HQ_OUT_BF16, HQ_OUT_F32 = 0, 1

EXPORTS = ["hq_calibrate", "hq_select_topk", "hq_quantize_pack", "hq_dequant_reduce",
           "hq_dequant_reduce_bf16_shards", "hq_compress_reduce", "hq_status_string", "hq_read_device_error", "hq_wire_bytes_per_row",
           "hq_selftest_bounded_wait", "hq_selftest_set_pipeline_stall", "hq_calibrate_ld", "hq_quantize_pack_ld",
           "hq_dequant_reduce_ld", "hq_compress_reduce_ld", "hq_dequant_reduce_ranks", "hq_two_step_reduce",
           "hq_two_step_workspace_bytes", "hq_two_step_reduce_noalloc"]


class HQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {hq_status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded C library (for callers that pass raw pointers)."""
    return _lib


def hq_status_string(status: int) -> str:
    return _lib.hq_status_string(int(status)).decode()


def hq_wire_bytes_per_row(H: int, k: int) -> int:
    return int(_lib.hq_wire_bytes_per_row(H, k))


def _stream(stream, device):
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t, dtypes, shape, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() else None


def _ptr_rows(t, dtypes, shape, name):
    """(pointer, row pitch in elements) of a view whose rows are dense but may be further apart
    than their width, e.g. x[:, :, c0:c0 + Hs] of a contiguous [P, T, ld] tensor."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    st = t.stride()
    ld = st[-2]
    if st[-1] != 1 or (t.dim() == 3 and t.shape[0] > 1 and st[0] != t.shape[1] * ld):
        raise ValueError(f"{name}: rows must be dense, ld apart, and the ranks' rows back to back")
    return (t.data_ptr() if t.numel() else None), ld


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)
_F32 = (torch.float32,)
_I32 = (torch.int32,)
_U8 = (torch.uint8,)
_CODES = (torch.int32, torch.uint32)


def _check(status, where):
    if status != HQ_OK:
        raise HQError(status, where)


def hq_calibrate(x, ema_min, ema_max, beta: float, first_batch: bool, stream=None) -> None:
    P, T, H = x.shape
    args = (_ptr(x, _BF16, (P, T, H), "x"), P, T, H, float(beta), int(bool(first_batch)),
            _ptr(ema_min, _F32, (P, H), "ema_min"), _ptr(ema_max, _F32, (P, H), "ema_max"),
            _stream(stream, x.device))
    _check(_lib.hq_calibrate(*args), "hq_calibrate")


def hq_select_topk(ema_min, ema_max, k: int, keep_idx, rest_idx, scale, inv_scale, zero, stream=None) -> None:
    P, H = ema_min.shape
    args = (_ptr(ema_min, _F32, (P, H), "ema_min"), _ptr(ema_max, _F32, (P, H), "ema_max"), P, H, k,
            _ptr(keep_idx, _I32, (k,), "keep_idx"), _ptr(rest_idx, _I32, (H - k,), "rest_idx"),
            _ptr(scale, _F32, (P, H), "scale"), _ptr(inv_scale, _F32, (P, H), "inv_scale"),
            _ptr(zero, _U8, (P, H), "zero"), _stream(stream, ema_min.device))
    _check(_lib.hq_select_topk(*args), "hq_select_topk")


def hq_quantize_pack(x, keep_idx, rest_idx, inv_scale, zero, codes, side, stream=None) -> None:
    P, T, H = x.shape
    k = keep_idx.shape[0]
    args = (_ptr(x, _BF16, (P, T, H), "x"), P, T, H, k, _ptr(keep_idx, _I32, (k,), "keep_idx"),
            _ptr(rest_idx, _I32, (H - k,), "rest_idx"), _ptr(inv_scale, _F32, (P, H), "inv_scale"),
            _ptr(zero, _U8, (P, H), "zero"), _ptr(codes, _CODES, (P, T, (H - k) // 8), "codes"),
            _ptr(side, _BF16, (P, k, T), "side"), _stream(stream, x.device))
    _check(_lib.hq_quantize_pack(*args), "hq_quantize_pack")


def _dequant_args(codes, side, keep_idx, rest_idx, scale, zero, out, stream):
    P, T, W = codes.shape
    k = keep_idx.shape[0]
    H = out.shape[1]
    if W != (H - k) // 8:
        raise ValueError("codes width does not match H and k")
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    args = (_ptr(codes, _CODES, (P, T, W), "codes"), _ptr(side, _BF16, (P, k, T), "side"), P, T, H, k,
            _ptr(keep_idx, _I32, (k,), "keep_idx"), _ptr(rest_idx, _I32, (H - k,), "rest_idx"),
            _ptr(scale, _F32, (P, H), "scale"), _ptr(zero, _U8, (P, H), "zero"),
            _ptr(out, _BF16 + _F32, (T, H), "out"), odt, _stream(stream, codes.device))
    return args


def hq_dequant_reduce(codes, side, keep_idx, rest_idx, scale, zero, out, stream=None) -> None:
    _check(_lib.hq_dequant_reduce(*_dequant_args(codes, side, keep_idx, rest_idx, scale, zero, out, stream)),
           "hq_dequant_reduce")


def hq_dequant_reduce_bf16_shards(codes, side, keep_idx, rest_idx, scale, zero, out, stream=None) -> None:
    """The literal variant: each rank's dequantized value is rounded to bf16 before it is added."""
    _check(_lib.hq_dequant_reduce_bf16_shards(*_dequant_args(codes, side, keep_idx, rest_idx, scale, zero, out,
                                                             stream)), "hq_dequant_reduce_bf16_shards")


def hq_compress_reduce(x, keep_idx, rest_idx, scale, inv_scale, zero, out, codes=None, side=None,
                       stream=None) -> None:
    P, T, H = x.shape
    k = keep_idx.shape[0]
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    args = (_ptr(x, _BF16, (P, T, H), "x"), P, T, H, k, _ptr(keep_idx, _I32, (k,), "keep_idx"),
            _ptr(rest_idx, _I32, (H - k,), "rest_idx"), _ptr(scale, _F32, (P, H), "scale"),
            _ptr(inv_scale, _F32, (P, H), "inv_scale"), _ptr(zero, _U8, (P, H), "zero"),
            _ptr(out, _BF16 + _F32, (T, H), "out"), odt,
            _ptr(codes, _CODES, (P, T, (H - k) // 8), "codes"), _ptr(side, _BF16, (P, k, T), "side"),
            _stream(stream, x.device))
    _check(_lib.hq_compress_reduce(*args), "hq_compress_reduce")


def hq_dequant_reduce_ranks(codes, side, keep_idx, rest_idx, scale, zero, out, stream=None) -> None:
    """The reduction over P separate wire buffers: codes is a list of P [T, (H-k)/8] int32 tensors,
    side a list of P [k, T] bf16 tensors (each may live on another GPU this process can read)."""
    P = len(codes)
    T, W = codes[0].shape
    k = keep_idx.shape[0]
    H = out.shape[1]
    if W != (H - k) // 8 or len(side) != P:
        raise ValueError("codes width, H, k and the number of side buffers must agree")
    cptr = (ctypes.c_void_p * P)(*[_ptr(c, _CODES, (T, W), f"codes[{r}]") for r, c in enumerate(codes)])
    sptr = (ctypes.c_void_p * P)(*[_ptr(s_, _BF16, (k, T), f"side[{r}]") for r, s_ in enumerate(side)])
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    args = (ctypes.cast(cptr, _vp), ctypes.cast(sptr, _vp) if k else None, P, T, H, k,
            _ptr(keep_idx, _I32, (k,), "keep_idx"), _ptr(rest_idx, _I32, (H - k,), "rest_idx"),
            _ptr(scale, _F32, (P, H), "scale"), _ptr(zero, _U8, (P, H), "zero"),
            _ptr(out, _BF16 + _F32, (T, H), "out"), odt, _stream(stream, out.device))
    _check(_lib.hq_dequant_reduce_ranks(*args), "hq_dequant_reduce_ranks")


def hq_two_step_workspace_bytes(P: int, T: int, H: int, k: int, k2: int) -> int:
    return int(_lib.hq_two_step_workspace_bytes(P, T, H, k, k2))


def hq_two_step_reduce(x, keep_idx, rest_idx, scale, inv_scale, zero, keep2, rest2, scale2, inv_scale2, zero2,
                       workspace, out, stream=None) -> None:
    """The two-step all-reduce of P simulated ranks x [P, T, H] on one GPU; workspace is a uint8
    device tensor of at least hq_two_step_workspace_bytes(...) bytes."""
    P, T, H = x.shape
    k, k2 = keep_idx.shape[0], keep2.shape[0]
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    args = (_ptr(x, _BF16, (P, T, H), "x"), P, T, H, k, _ptr(keep_idx, _I32, (k,), "keep_idx"),
            _ptr(rest_idx, _I32, (H - k,), "rest_idx"), _ptr(scale, _F32, (P, H), "scale"),
            _ptr(inv_scale, _F32, (P, H), "inv_scale"), _ptr(zero, _U8, (P, H), "zero"), k2,
            _ptr(keep2, _I32, (k2,), "keep2"), _ptr(rest2, _I32, (H - k2,), "rest2"),
            _ptr(scale2, _F32, (P, H), "scale2"), _ptr(inv_scale2, _F32, (P, H), "inv_scale2"),
            _ptr(zero2, _U8, (P, H), "zero2"), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
            _ptr(out, _BF16 + _F32, (T, H), "out"), odt, _stream(stream, x.device))
    _check(_lib.hq_two_step_reduce(*args), "hq_two_step_reduce")


def hq_two_step_reduce_noalloc(x, keep_idx, rest_idx, scale, inv_scale, zero, keep2, rest2, scale2, inv_scale2,
                               zero2, out, stream=None) -> None:
    """hq_two_step_reduce with the library's fixed scratch array instead of a workspace, for
    callers that cannot allocate device memory (problems up to HQ_TWO_STEP_NOALLOC_MAX_BYTES of
    workspace; calls that overlap on the GPU race on the array)."""
    P, T, H = x.shape
    k, k2 = keep_idx.shape[0], keep2.shape[0]
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    args = (_ptr(x, _BF16, (P, T, H), "x"), P, T, H, k, _ptr(keep_idx, _I32, (k,), "keep_idx"),
            _ptr(rest_idx, _I32, (H - k,), "rest_idx"), _ptr(scale, _F32, (P, H), "scale"),
            _ptr(inv_scale, _F32, (P, H), "inv_scale"), _ptr(zero, _U8, (P, H), "zero"), k2,
            _ptr(keep2, _I32, (k2,), "keep2"), _ptr(rest2, _I32, (H - k2,), "rest2"),
            _ptr(scale2, _F32, (P, H), "scale2"), _ptr(inv_scale2, _F32, (P, H), "inv_scale2"),
            _ptr(zero2, _U8, (P, H), "zero2"), _ptr(out, _BF16 + _F32, (T, H), "out"), odt,
            _stream(stream, x.device))
    _check(_lib.hq_two_step_reduce_noalloc(*args), "hq_two_step_reduce_noalloc")


# -- partial-channel synchronisation: the same calls on a block of features [c0, c0 + Hs) -------
# Pass column views: x[:, :, c0:c0 + Hs] of a contiguous [P, T, ld] tensor, out[:, c0:c0 + Hs] of a
# contiguous [T, ld] tensor.  Only the block's columns of out are written.
def hq_calibrate_ld(x, ema_min, ema_max, beta: float, first_batch: bool, stream=None) -> None:
    P, T, H = x.shape
    px, ldx = _ptr_rows(x, _BF16, (P, T, H), "x")
    args = (px, ldx, P, T, H, float(beta), int(bool(first_batch)), _ptr(ema_min, _F32, (P, H), "ema_min"),
            _ptr(ema_max, _F32, (P, H), "ema_max"), _stream(stream, x.device))
    _check(_lib.hq_calibrate_ld(*args), "hq_calibrate_ld")


def hq_quantize_pack_ld(x, keep_idx, rest_idx, inv_scale, zero, codes, side, stream=None) -> None:
    P, T, H = x.shape
    k = keep_idx.shape[0]
    px, ldx = _ptr_rows(x, _BF16, (P, T, H), "x")
    args = (px, ldx, P, T, H, k, _ptr(keep_idx, _I32, (k,), "keep_idx"), _ptr(rest_idx, _I32, (H - k,), "rest_idx"),
            _ptr(inv_scale, _F32, (P, H), "inv_scale"), _ptr(zero, _U8, (P, H), "zero"),
            _ptr(codes, _CODES, (P, T, (H - k) // 8), "codes"), _ptr(side, _BF16, (P, k, T), "side"),
            _stream(stream, x.device))
    _check(_lib.hq_quantize_pack_ld(*args), "hq_quantize_pack_ld")


def hq_dequant_reduce_ld(codes, side, keep_idx, rest_idx, scale, zero, out, stream=None) -> None:
    P, T, W = codes.shape
    k = keep_idx.shape[0]
    H = out.shape[1]
    if W != (H - k) // 8:
        raise ValueError("codes width does not match the block width and k")
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    po, ldo = _ptr_rows(out, _BF16 + _F32, (T, H), "out")
    args = (_ptr(codes, _CODES, (P, T, W), "codes"), _ptr(side, _BF16, (P, k, T), "side"), P, T, H, k,
            _ptr(keep_idx, _I32, (k,), "keep_idx"), _ptr(rest_idx, _I32, (H - k,), "rest_idx"),
            _ptr(scale, _F32, (P, H), "scale"), _ptr(zero, _U8, (P, H), "zero"), po, ldo, odt,
            _stream(stream, codes.device))
    _check(_lib.hq_dequant_reduce_ld(*args), "hq_dequant_reduce_ld")


def hq_compress_reduce_ld(x, keep_idx, rest_idx, scale, inv_scale, zero, out, codes=None, side=None,
                          stream=None) -> None:
    P, T, H = x.shape
    k = keep_idx.shape[0]
    odt = HQ_OUT_F32 if out.dtype == torch.float32 else HQ_OUT_BF16
    px, ldx = _ptr_rows(x, _BF16, (P, T, H), "x")
    po, ldo = _ptr_rows(out, _BF16 + _F32, (T, H), "out")
    args = (px, ldx, P, T, H, k, _ptr(keep_idx, _I32, (k,), "keep_idx"), _ptr(rest_idx, _I32, (H - k,), "rest_idx"),
            _ptr(scale, _F32, (P, H), "scale"), _ptr(inv_scale, _F32, (P, H), "inv_scale"),
            _ptr(zero, _U8, (P, H), "zero"), po, ldo, odt,
            _ptr(codes, _CODES, (P, T, (H - k) // 8), "codes"), _ptr(side, _BF16, (P, k, T), "side"),
            _stream(stream, x.device))
    _check(_lib.hq_compress_reduce_ld(*args), "hq_compress_reduce_ld")


def hq_selftest_bounded_wait(limit_cycles: int, stream=None, device=None) -> None:
    """Launches a wait that nothing satisfies; it gives up after limit_cycles and records
    HQ_ERR_TIMEOUT (read it with hq_read_device_error)."""
    _check(_lib.hq_selftest_bounded_wait(int(limit_cycles), _stream(stream, device)), "hq_selftest_bounded_wait")


def hq_selftest_set_pipeline_stall(consumer_limit_cycles: int, producer_delay_cycles: int) -> None:
    """Self-test of the pipelines' abort path: later pipeline launches delay their producers and
    bound their consumers' waits by consumer_limit_cycles; (0, 0) restores the normal bounds."""
    _check(_lib.hq_selftest_set_pipeline_stall(int(consumer_limit_cycles), int(producer_delay_cycles)),
           "hq_selftest_set_pipeline_stall")


def hq_read_device_error(stream=None, device=None) -> int:
    """Takes and clears the device error word atomically, after the work ordered before it on the
    stream (0 = none)."""
    return int(_lib.hq_read_device_error(_stream(stream, device)))


class Buffers:
    """Device buffers for one (P, T, H, k) problem, allocated by torch (plumbing only)."""

    def __init__(self, P: int, T: int, H: int, k: int, device="cuda", out_dtype=torch.bfloat16):
        dev = torch.device(device)
        self.P, self.T, self.H, self.k = P, T, H, k
        self.ema_min = torch.empty((P, H), dtype=torch.float32, device=dev)
        self.ema_max = torch.empty((P, H), dtype=torch.float32, device=dev)
        self.keep_idx = torch.empty((k,), dtype=torch.int32, device=dev)
        self.rest_idx = torch.empty((H - k,), dtype=torch.int32, device=dev)
        self.scale = torch.empty((P, H), dtype=torch.float32, device=dev)
        self.inv_scale = torch.empty((P, H), dtype=torch.float32, device=dev)
        self.zero = torch.empty((P, H), dtype=torch.uint8, device=dev)
        self.codes = torch.empty((P, T, (H - k) // 8), dtype=torch.int32, device=dev)
        self.side = torch.empty((P, k, T), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((T, H), dtype=out_dtype, device=dev)
