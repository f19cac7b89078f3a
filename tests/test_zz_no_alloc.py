"""The allocation-free int8-compute entry point, convrot_linear_int8_noalloc.

It exists for callers that may not allocate device memory and have no
workspace to pass: a plugin inside a framework that owns all device memory and
gives its extensions no scratch allocator, or a serving path where an
allocation (which can synchronize the device and can fail with out of memory
mid-request) is not allowed.  It keeps the intermediate int8 codes and
per-token scales in a fixed static device array instead of a caller workspace.

These tests call it through the C ABI and require the same output as the
regular entry point, convrot_linear_int8 with a workspace, on two calls in a
row (the second must not depend on what the first left in the shared scratch),
within the layer tolerance of the other tests (relative L2 <= 2e-3; the two
run the same kernels, so the outputs are in fact identical).  This file is
collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


def _layer(lin, index, M=None):
    import activation_quantized_linear_b200 as cr
    inp = workloads.make_layer_inputs(lin, index, M=M)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    return inp.x.cuda(), Wq, s_w, inp.bias.cuda(), rot


def _call_noalloc(lib, x, Wq, s_w, rot, bias, y):
    M, K = x.shape
    N = Wq.shape[0]
    return lib.convrot_linear_int8_noalloc(
        ctypes.c_void_p(x.data_ptr()), M, K, N, rot.handle, ctypes.c_void_p(Wq.data_ptr()),
        ctypes.c_void_p(s_w.data_ptr()), s_w.numel(), ctypes.c_void_p(bias.data_ptr()),
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _call_with_workspace(cr, x, Wq, s_w, rot, bias):
    ws = torch.empty(cr.workspace_bytes(x.shape[0], Wq.shape[0], x.shape[1]),
                     dtype=torch.uint8, device="cuda")
    return cr.linear_int8(x, Wq, s_w, rot, bias, workspace=ws)


def test_noalloc_matches_workspace_entry_point_two_calls():
    import activation_quantized_linear_b200 as cr
    torch.cuda.set_device(0)
    lib = cr._lib
    assert lib.convrot_noalloc_scratch_bytes() == 32 << 20
    # call 1: the Z-Image QKV shape (17.7 MB of scratch); call 2: a small layer
    cases = [(workloads.WORKLOADS["zimage_dit_block"][0], 3, None),
             (workloads.WORKLOADS["single_1024"][0], 4, None)]
    for lin, index, M in cases:
        x, Wq, s_w, bias, rot = _layer(lin, index, M)
        y = torch.empty((x.shape[0], Wq.shape[0]), dtype=torch.bfloat16, device="cuda")
        y.fill_(float("nan"))
        st = _call_noalloc(lib, x, Wq, s_w, rot, bias, y)
        assert st == cr.OK, lib.convrot_last_error_string()
        y_ref = _call_with_workspace(cr, x, Wq, s_w, rot, bias)
        torch.cuda.synchronize()
        assert oracle.rel_l2(y.cpu(), y_ref.cpu()) <= 2e-3
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    cr.check_status()


def test_noalloc_slices_batches_beyond_its_scratch():
    """4608 tokens of K = 10240 need 47 MB of codes, more than the 32 MiB
    array: the entry point runs them in row slices and still returns the
    workspace entry point's output, bit for bit, on two calls in a row."""
    import activation_quantized_linear_b200 as cr
    torch.cuda.set_device(0)
    lib = cr._lib
    lin = workloads.WORKLOADS["zimage_dit_block"][2]  # 4608 x 10240 -> 3840
    assert lin.M * lin.K > lib.convrot_noalloc_scratch_bytes()
    x, Wq, s_w, bias, rot = _layer(lin, 5)
    y_ref = _call_with_workspace(cr, x, Wq, s_w, rot, bias)
    for _ in range(2):
        y = torch.full((x.shape[0], Wq.shape[0]), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _call_noalloc(lib, x, Wq, s_w, rot, bias, y)
        assert st == cr.OK, lib.convrot_last_error_string()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    cr.check_status()
