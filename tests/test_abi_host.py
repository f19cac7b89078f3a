"""Host-side checks of the C ABI (no kernel launch; runs without a GPU).

The library must load on a machine without a GPU, export every entry point
include/convrot.h declares, and reject bad arguments with the documented
status before touching the device.
"""

import ctypes
import os
import re

import numpy as np
import pytest

import activation_quantized_linear_b200 as cr
from activation_quantized_linear_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")

lib = cr._lib
vp = ctypes.c_void_p
FAKE = 0x10000          # a 16-byte aligned address that is never dereferenced
MISALIGNED = 0x10008


DEBUG_HEADER = os.path.join(ROOT, "include", "convrot_debug.h")


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(convrot_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 14
    raw = ctypes.CDLL(build.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in convrot.h but not exported"


def test_version_and_error_string():
    assert lib.convrot_version() >= 100
    assert isinstance(lib.convrot_last_error_string(), bytes)


@pytest.mark.parametrize("G", [0, 1, 2, 8, 32, 128, 512, -4])
def test_rotation_rejects_group_size(G):
    R = np.eye(max(G, 1), dtype=np.float32)
    h = vp()
    st = lib.convrot_rotation_create(R.ctypes.data, G, ctypes.byref(h))
    assert st == cr.UNSUPPORTED
    assert h.value is None
    assert b"group size" in lib.convrot_last_error_string()


def test_rotation_rejects_non_orthogonal_and_null():
    h = vp()
    R = np.eye(16, dtype=np.float32)
    R[0, 1] = 0.01
    assert lib.convrot_rotation_create(R.ctypes.data, 16, ctypes.byref(h)) == cr.INVALID_ARG
    assert b"orthogonal" in lib.convrot_last_error_string()
    assert lib.convrot_rotation_create(None, 16, ctypes.byref(h)) == cr.INVALID_ARG
    assert lib.convrot_rotation_create(R.ctypes.data, 16, None) == cr.INVALID_ARG


def test_null_handle_rejected():
    assert lib.convrot_rotation_destroy(None) == cr.INVALID_ARG
    assert lib.convrot_rotate_quant_act(FAKE, 4, 256, None, FAKE, FAKE, None) == cr.INVALID_ARG
    assert lib.convrot_dequant_derotate(FAKE, FAKE, 1, 4, 256, None, FAKE, None) == cr.INVALID_ARG
    assert lib.convrot_quantize_weight(FAKE, 4, 256, None, FAKE, FAKE, None) == cr.INVALID_ARG


def test_gemm_shape_and_pointer_checks():
    g = lib.convrot_int8_gemm
    # N not a multiple of 16, K not a multiple of 16, negative M
    assert g(FAKE, FAKE, FAKE, FAKE, 1, None, 8, 24, 64, FAKE, None) == cr.INVALID_ARG
    assert g(FAKE, FAKE, FAKE, FAKE, 1, None, 8, 32, 40, FAKE, None) == cr.INVALID_ARG
    assert g(FAKE, FAKE, FAKE, FAKE, 1, None, -1, 32, 64, FAKE, None) == cr.INVALID_ARG
    assert g(FAKE, FAKE, FAKE, FAKE, 1, None, 8, 32, 1 << 20, FAKE, None) == cr.UNSUPPORTED
    # M == 0 is a no-op that never touches the pointers
    assert g(None, None, None, None, 1, None, 0, 32, 64, None, None) == cr.OK
    # null / misaligned operands
    assert g(None, FAKE, FAKE, FAKE, 1, None, 8, 32, 64, FAKE, None) == cr.INVALID_ARG
    assert g(MISALIGNED, FAKE, FAKE, FAKE, 1, None, 8, 32, 64, FAKE, None) == cr.ALIGNMENT
    assert g(FAKE, FAKE, MISALIGNED, FAKE, 1, None, 8, 32, 64, FAKE, None) == cr.ALIGNMENT
    assert g(FAKE, FAKE, FAKE, FAKE, 1, None, 8, 32, 64, MISALIGNED, None) == cr.ALIGNMENT
    assert g(FAKE, None, FAKE, FAKE, 1, None, 8, 32, 64, FAKE, None) == cr.INVALID_ARG
    # scale length must be 1 or N
    assert g(FAKE, FAKE, FAKE, FAKE, 3, None, 8, 32, 64, FAKE, None) == cr.INVALID_ARG
    assert g(FAKE, FAKE, FAKE, FAKE, 1, MISALIGNED, 8, 32, 64, FAKE, None) == cr.ALIGNMENT
    s = lib.convrot_int8_gemm_s32
    assert s(FAKE, FAKE, 8, 20, 64, FAKE, None) == cr.INVALID_ARG
    assert s(FAKE, FAKE, 0, 32, 64, None, None) == cr.OK


def test_workspace_size():
    M, N, K = 4608, 11520, 3840
    need = lib.convrot_workspace_bytes(cr.OP_LINEAR_INT8, M, N, K)
    assert need >= M * K + 4 * M and need % 256 == 0
    assert lib.convrot_workspace_bytes(99, M, N, K) == 0
    assert lib.convrot_workspace_bytes(cr.OP_LINEAR_INT8, 0, N, K) == 0
    # slices of at most 2N tokens: all of M here, 2N = 2048 rows for N = 1024
    assert lib.convrot_workspace_bytes(cr.OP_LINEAR_INT8_SLICED, M, N, K) == need
    sliced = lib.convrot_workspace_bytes(cr.OP_LINEAR_INT8_SLICED, M, 1024, K)
    assert sliced == lib.convrot_workspace_bytes(cr.OP_LINEAR_INT8, 2048, 1024, K)


def test_default_path_and_checked_workspace_sizes():
    M, N, K = 4608, 11520, 3840
    dq = lib.convrot_workspace_bytes(cr.OP_LINEAR_DEQUANT, M, N, K)
    assert dq == 2 * N * K  # already a multiple of 256
    chk = lib.convrot_workspace_bytes(cr.OP_LINEAR_CHECKED, M, N, K)
    # the decoded weight + 256 rows of output + the sums, or the int8 codes if larger
    assert chk == max(dq + 2 * 256 * N + 256, lib.convrot_workspace_bytes(cr.OP_LINEAR_INT8, M, N, K))
    # few tokens: only M rows are checked
    assert lib.convrot_workspace_bytes(cr.OP_LINEAR_CHECKED, 3, 1024, 1024) == (
        2 * 1024 * 1024 + 256 * ((2 * 3 * 1024 + 255) // 256) + 256)


def test_check_state_on_the_host():
    cr.check_reset()
    assert cr.check_state(0) == (False, 0)
    assert cr.check_min_cosine() == 0.99
    cr.check_set_min_cosine(1.2)
    assert cr.check_min_cosine() == 1.2
    for bad in (0.0, -1.0, 1.6, float("nan")):
        with pytest.raises(cr.ConvRotError) as e:
            cr.check_set_min_cosine(bad)
        assert e.value.status == cr.INVALID_ARG
    cr.check_set_min_cosine(0.99)
    assert lib.convrot_check_state(-1, None, None) == cr.INVALID_ARG


def test_checked_rejects_before_device():
    f = lib.convrot_linear_checked
    path = ctypes.c_int(7)
    # no rotation handle, then no workspace: errors before any CUDA call, nothing latched
    assert f(FAKE, 8, 256, 32, None, FAKE, FAKE, 1, None, FAKE, FAKE, 1 << 24, ctypes.byref(path),
             None) == cr.INVALID_ARG
    assert path.value == 0
    g = lib.convrot_linear_dequant
    assert g(FAKE, 8, 256, 24, None, FAKE, FAKE, 1, None, FAKE, FAKE, 1 << 24, None) == cr.INVALID_ARG
    assert g(FAKE, 8, 256, 32, None, FAKE, FAKE, 1, None, FAKE, None, 0, None) == cr.WORKSPACE
    assert lib.convrot_dense_linear(FAKE, 8, 64, 24, FAKE, None, FAKE, None) == cr.INVALID_ARG
    assert lib.convrot_dense_linear(MISALIGNED, 8, 64, 32, FAKE, None, FAKE, None) == cr.ALIGNMENT
    assert cr.check_state(0) == (False, 0)


def test_bench_probe_is_its_own_library():
    """The int8 issue-rate probe lives in libconvrot_bench.so, which the
    benchmark loads; the layer's library does not export it.  Its argument
    checks answer before any device work."""
    raw = ctypes.CDLL(build.LIB_PATH)
    assert not hasattr(raw, "convrot_measure_int8_mma_rate")
    assert not hasattr(raw, "convrot_bench_int8_mma_rate")
    probe = ctypes.CDLL(build.BENCH_LIB_PATH)
    f = probe.convrot_bench_int8_mma_rate
    f.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.c_void_p]
    f.restype = ctypes.c_int
    tops = ctypes.c_double(0.0)
    assert f(0, ctypes.byref(tops), None) == cr.INVALID_ARG
    assert f(200001, ctypes.byref(tops), None) == cr.INVALID_ARG
    assert f(100, None, None) == cr.INVALID_ARG


def test_linear_rejects_before_device():
    f = lib.convrot_linear_int8
    assert f(FAKE, 8, 256, 24, None, FAKE, FAKE, 1, None, FAKE, FAKE, 1 << 20, None) == cr.INVALID_ARG
    assert f(FAKE, 8, 256, 32, None, FAKE, FAKE, 1, None, FAKE, FAKE, 1 << 20, None) == cr.INVALID_ARG


def test_binding_validates_tensors_on_cpu():
    import torch
    x = torch.zeros(4, 256, dtype=torch.float32)
    with pytest.raises(TypeError):
        cr.rotate_quant_act(x, None)
    with pytest.raises(ValueError):
        cr.rotate_quant_act(x.to(torch.bfloat16), None)  # not a CUDA tensor


def test_header_compiles_as_c_and_links(tmp_path):
    """include/convrot.h is a C ABI: a C99 program compiled with gcc against the
    header alone links libconvrot.so and gets the documented argument errors."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(cr.library_path())
    exe = str(tmp_path / "abi_smoke")
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-pedantic",
           os.path.join(root, "tests", "c_abi", "abi_smoke.c"),
           "-I", os.path.join(root, "include"), "-L", lib_dir, "-lconvrot",
           "-Wl,-rpath," + lib_dir, "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    assert "c abi ok" in res.stdout


def test_debug_library_exports_both_headers():
    """libconvrot_debug.so (CONVROT_DEBUG=1) exports everything convrot.h
    declares plus the fault hook of convrot_debug.h; the release library
    does not export the hook."""
    dbg = ctypes.CDLL(build.DEBUG_LIB_PATH)
    for n in declared_functions() + declared_functions(DEBUG_HEADER):
        assert hasattr(dbg, n), f"{n} not exported by the debug library"
    assert declared_functions(DEBUG_HEADER) == ["convrot_debug_set_fault"]
    assert not hasattr(ctypes.CDLL(build.LIB_PATH), "convrot_debug_set_fault")


def test_debug_fault_codes_checked_on_the_host():
    dbg = cr.load_library(build.DEBUG_LIB_PATH)
    f = dbg.convrot_debug_set_fault
    f.argtypes = [ctypes.c_int]
    f.restype = ctypes.c_int
    assert f(3) == cr.INVALID_ARG and f(-1) == cr.INVALID_ARG
    assert b"unknown fault" in dbg.convrot_last_error_string()
    assert f(0) == cr.OK
