"""The C ABI without a GPU: libhq.so loads, exports every function include/hq.h declares, and the
host-side argument checks return their documented status before anything touches the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hq.h")


@pytest.fixture(scope="module")
def hq():
    import bit_tensor_activation_b200 as m

    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("hq_calibrate", "hq_select_topk", "hq_quantize_pack", "hq_dequant_reduce",
              "hq_compress_reduce", "hq_status_string", "hq_read_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(hq):
    lib = hq.lib()
    for n in declared_functions():
        assert hasattr(lib, n), f"libhq.so does not export {n}"
    assert sorted(hq.EXPORTS) == declared_functions()


def test_status_strings(hq):
    assert hq.hq_status_string(0) == "HQ_OK"
    assert hq.hq_status_string(5) == "HQ_ERR_BAD_INDEX"
    assert hq.hq_status_string(99) == "HQ_ERR_UNKNOWN"
    assert hq.hq_wire_bytes_per_row(8192, 256) == (8192 - 256) // 2 + 512
    assert hq.hq_wire_bytes_per_row(8, 16) == -1


# Fake, never-dereferenced device addresses: every call below fails validation first.
A = 0x10000  # 64 KiB aligned
MIS = A + 4  # 4-byte but not 16-byte aligned


def _calls(lib):
    c = ctypes.c_void_p
    return {
        "calibrate": lambda x=A, P=2, T=4, H=64, beta=0.9, emn=A, emx=A: lib.hq_calibrate(
            c(x), P, T, H, ctypes.c_float(beta), 1, c(emn), c(emx), None),
        "select": lambda P=2, H=64, k=8, keep=A, rest=A, sc=A, inv=A, z=A: lib.hq_select_topk(
            c(A), c(A), P, H, k, c(keep), c(rest), c(sc), c(inv), c(z), None),
        "quantize": lambda x=A, P=2, T=4, H=64, k=8, keep=A, rest=A, codes=A, side=A: lib.hq_quantize_pack(
            c(x), P, T, H, k, c(keep), c(rest), c(A), c(A), c(codes), c(side), None),
        "dequant": lambda P=2, T=4, H=64, k=8, out=A, odt=0, side=A: lib.hq_dequant_reduce(
            c(A), c(side), P, T, H, k, c(A), c(A), c(A), c(A), c(out), odt, None),
        "dequant_bf16_shards": lambda P=2, T=4, H=64, k=8, out=A, odt=0, side=A: lib.hq_dequant_reduce_bf16_shards(
            c(A), c(side), P, T, H, k, c(A), c(A), c(A), c(A), c(out), odt, None),
        "fused": lambda P=2, T=4, H=64, k=8, out=A, codes=None, side=None: lib.hq_compress_reduce(
            c(A), P, T, H, k, c(A), c(A), c(A), c(A), c(A), c(out), 0, c(codes) if codes else None,
            c(side) if side else None, None),
    }


@pytest.mark.parametrize("case,kw,status", [
    ("calibrate", dict(P=0), 1), ("calibrate", dict(P=65), 1), ("calibrate", dict(H=12), 1),
    ("calibrate", dict(H=0), 1), ("calibrate", dict(H=32776), 1), ("calibrate", dict(T=0), 1),
    ("calibrate", dict(beta=1.0), 1), ("calibrate", dict(beta=-0.1), 1), ("calibrate", dict(beta=float("nan")), 1),
    ("calibrate", dict(x=0), 1), ("calibrate", dict(emn=0), 1), ("calibrate", dict(x=MIS), 2),
    ("calibrate", dict(emx=MIS), 2),
    ("select", dict(k=4), 1), ("select", dict(k=72), 1), ("select", dict(k=-8), 1), ("select", dict(keep=0), 1),
    ("select", dict(rest=0), 1), ("select", dict(sc=MIS), 2), ("select", dict(z=A + 8), 2),
    ("select", dict(keep=A + 2), 2),
    ("quantize", dict(T=-1), 1), ("quantize", dict(k=12), 1), ("quantize", dict(side=0), 1),
    ("quantize", dict(codes=0), 1), ("quantize", dict(x=A + 8), 2), ("quantize", dict(side=MIS), 2),
    ("quantize", dict(codes=A + 2), 2),
    ("dequant", dict(odt=2), 1), ("dequant", dict(out=0), 1), ("dequant", dict(out=MIS), 2),
    ("dequant", dict(side=0), 1),
    ("dequant_bf16_shards", dict(odt=2), 1), ("dequant_bf16_shards", dict(out=0), 1),
    ("dequant_bf16_shards", dict(out=MIS), 2), ("dequant_bf16_shards", dict(side=0), 1),
    ("dequant_bf16_shards", dict(k=12), 1),
    ("fused", dict(codes=A), 1), ("fused", dict(side=A), 1), ("fused", dict(out=MIS), 2),
    ("fused", dict(P=70), 1),
])
def test_host_validation(hq, case, kw, status):
    assert _calls(hq.lib())[case](**kw) == status


def test_empty_arrays_may_be_null(hq):
    """k == 0: keep_idx and side may be NULL; k == H: rest_idx and codes may be NULL.  T == 0 is
    a no-op that returns HQ_OK without touching the device."""
    lib = hq.lib()
    c = ctypes.c_void_p
    assert lib.hq_quantize_pack(c(A), 2, 0, 64, 0, None, c(A), c(A), c(A), c(A), None, None) == 0
    assert lib.hq_quantize_pack(c(A), 2, 0, 64, 64, c(A), None, c(A), c(A), None, c(A), None) == 0
    assert lib.hq_dequant_reduce(None, c(A), 2, 0, 64, 64, c(A), None, c(A), c(A), c(A), 0, None) == 0
    assert lib.hq_dequant_reduce_bf16_shards(None, c(A), 2, 0, 64, 64, c(A), None, c(A), c(A), c(A), 0, None) == 0
    assert lib.hq_compress_reduce(c(A), 2, 0, 64, 0, None, c(A), c(A), c(A), c(A), c(A), 1, None, None, None) == 0


def test_binding_rejects_wrong_tensors(hq):
    import torch

    x = torch.zeros((2, 4, 64), dtype=torch.bfloat16)  # CPU tensor
    e = torch.zeros((2, 64))
    with pytest.raises(TypeError):
        hq.hq_calibrate(x, e, e, 0.9, True)


def test_oracle_and_cuda_path_share_no_code():
    """The oracle and the CUDA path never include, import or link each other."""
    pkg = os.path.join(ROOT, "bit_tensor_activation_b200")
    orc = os.path.join(ROOT, "oracle")
    for d, forbidden in ((pkg, ("oracle", "hq_ref_", "synth")), (orc, ("bit_tensor_activation_b200", "csrc", "hq_api", "synth"))):
        for dirpath, _, files in os.walk(d):
            for f in files:
                if f.endswith((".py", ".c", ".cu", ".cuh", ".h")):
                    text = open(os.path.join(dirpath, f)).read()
                    for word in forbidden:
                        if d == orc and f == "__init__.py" and word == "synth":
                            continue
                        assert not re.search(rf"(import|include|from)\s+[\"<]?{word}", text), (f, word)
