"""The C-ABI library loads and exports every entry point its header declares;
host-side argument checks return their status codes before any CUDA call
(CPU only: no call here reaches the GPU)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def clib():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "fp8w8a8_build", os.path.join(ROOT, "fp8_w8a8_linear_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return ctypes.CDLL(mod.build())


def _declared():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(fp8_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(clib):
    names = _declared()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(clib, n), n


def test_version_and_status_strings(clib):
    clib.fp8_status_string.restype = ctypes.c_char_p
    assert clib.fp8_version() >= 100
    assert clib.fp8_status_string(0) == b"FP8_OK"
    assert clib.fp8_status_string(3) == b"FP8_ERR_SHAPE"
    assert clib.fp8_status_string(99) == b"FP8_ERR_UNKNOWN"


def _sig(clib):
    P, I = ctypes.c_void_p, ctypes.c_int64
    clib.fp8_quant_act.argtypes = [P, I, I, I, P, P, P]
    clib.fp8_repack_qat.argtypes = [P, P, I, I, P, P, P]
    clib.fp8_rowwise_linear.argtypes = [P, P, P, P, I, I, I, P, P]
    clib.fp8_convert_fnuz.argtypes = [P, P, I, I, P, P, P]
    clib.fp8_cast_e4m3.argtypes = [P, I, P, P]
    clib.fp8_linear_bf16.argtypes = [P, P, P, I, I, I, P, P, P, P]
    I32 = ctypes.c_int32
    clib.fp8_moe_route.argtypes = [P, I, I32, I32, P, P, P, P]
    clib.fp8_moe_combine.argtypes = [P, P, I, I32, I, P, P, P]
    clib.fp8_moe_gather.argtypes = [P, P, P, I, I, I32, P, P, P]


FAKE = 0x10000  # never dereferenced: every case below fails a host check first


def test_host_checks_return_before_any_launch(clib):
    _sig(clib)
    a = FAKE
    # quant: K % 16, ldx < K, null, misaligned
    assert clib.fp8_quant_act(a, 4, 24, 24, a, a, None) == 3
    assert clib.fp8_quant_act(a, 4, 32, 16, a, a, None) == 1
    assert clib.fp8_quant_act(None, 4, 32, 32, a, a, None) == 1
    assert clib.fp8_quant_act(a + 2, 4, 32, 32, a, a, None) == 2
    assert clib.fp8_quant_act(a, -1, 32, 32, a, a, None) == 1
    assert clib.fp8_quant_act(a, 0, 32, 32, a, a, None) == 0     # empty: nothing enqueued
    # repack: K % 32
    assert clib.fp8_repack_qat(a, a, 8, 48, a, a, None) == 3
    assert clib.fp8_repack_qat(a, a, 8, 64, a + 8, a, None) == 2
    assert clib.fp8_repack_qat(a, a, 0, 64, a, a, None) == 0
    # GEMM: K % 16, K limit, null, alignment, empty
    assert clib.fp8_rowwise_linear(a, a, a, a, 4, 8, 40, a, None) == 3
    assert clib.fp8_rowwise_linear(a, a, a, a, 4, 8, 65536 + 16, a, None) == 1
    assert clib.fp8_rowwise_linear(a, None, a, a, 4, 8, 32, a, None) == 1
    assert clib.fp8_rowwise_linear(a, a, a + 1, a, 4, 8, 32, a, None) == 2
    assert clib.fp8_rowwise_linear(a, a, a, a + 2, 4, 8, 32, a, None) == 2
    assert clib.fp8_rowwise_linear(a, a, a, a, 0, 8, 32, a, None) == 0
    assert clib.fp8_linear_bf16(a, a, a, 4, 8, 32, None, a, a, None) == 1
    # FNUZ conversion and cast
    assert clib.fp8_convert_fnuz(a, a, 4, 24, a, a, None) == 3
    assert clib.fp8_cast_e4m3(a, -5, a, None) == 1
    assert clib.fp8_cast_e4m3(a + 4, 5, a, None) == 2
    assert clib.fp8_cast_e4m3(a, 0, a, None) == 0
    # MoE: expert count, top_k limits, alignment, K % 16
    assert clib.fp8_moe_route(a, 16, 2, 0, a, a, a, None) == 1
    assert clib.fp8_moe_route(a, 16, 2, 1025, a, a, a, None) == 1
    assert clib.fp8_moe_route(a + 2, 16, 2, 8, a, a, a, None) == 2
    assert clib.fp8_moe_combine(a, a, 16, 17, 64, None, a, None) == 1
    assert clib.fp8_moe_combine(a, a, 16, 0, 64, None, a, None) == 1
    assert clib.fp8_moe_gather(a, a, a, 32, 24, 2, a, a, None) == 3
