"""The debug library (libconvrot_debug.so: the same sources built with
CONVROT_DEBUG=1, include/convrot_debug.h), through its C ABI.

compute-sanitizer is closed on this machine, so the debug build is the memory
checker of the kernels: every kernel checks the indices of its stores and
scale/bias reads, and records an index out of range in the status word
instead of touching memory.  These tests:
  * run the layer through the debug library and require the release
    library's outputs bit for bit, with a clean status word;
  * inject the short-rows fault (the kernels check against one row fewer
    than the output holds): the status must read CONVROT_ERR_BOUNDS, the last
    row must stay untouched and every other row must be the normal output;
  * inject the skipped-stage fault (the int8 GEMMs' producers leave their
    first ring stage empty): the consumer's bounded wait must run out, the
    kernel must return and report CONVROT_ERR_TIMEOUT, and the next call on
    the same context must compute the normal result.
No test traps, faults or hangs the GPU: the checks skip the access they
catch, and every wait in the kernels is bounded.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads
from activation_quantized_linear_b200 import build

pytestmark = pytest.mark.gpu

NONE, SKIP_STAGE, SHORT_ROWS = 0, 1, 2
SENTINEL = 0x5A


@pytest.fixture(scope="module")
def libs():
    import activation_quantized_linear_b200 as cr
    torch.cuda.set_device(0)
    dbg = cr.load_library(build.DEBUG_LIB_PATH)
    dbg.convrot_debug_set_fault.argtypes = [ctypes.c_int]
    dbg.convrot_debug_set_fault.restype = ctypes.c_int
    yield cr, dbg
    dbg.convrot_debug_set_fault(NONE)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


class DebugLayer:
    """One G = 256 layer's tensors, run through the debug library."""

    def __init__(self, cr, dbg, M, N, K, seed):
        self.cr, self.dbg = cr, dbg
        lin = workloads.Linear("debug", M, K, N, G=256)
        inp = workloads.make_layer_inputs(lin, seed)
        self.R = np.ascontiguousarray(workloads.sylvester_rotation(256), np.float32)
        self.rot = cr.Rotation(self.R)                   # release library
        h = ctypes.c_void_p()
        assert dbg.convrot_rotation_create(self.R.ctypes.data, 256, ctypes.byref(h)) == cr.OK
        self.h = h                                       # debug library
        self.x, self.bias = inp.x.cuda(), inp.bias.cuda()
        self.Wq, self.s_w = cr.quantize_weight(inp.W.cuda(), self.rot)
        self.M, self.N, self.K = M, N, K

    def close(self):
        self.dbg.convrot_rotation_destroy(self.h)
        self.rot.close()

    def rotate(self, xq, s_tok):
        return self.dbg.convrot_rotate_quant_act(_p(self.x), self.M, self.K, self.h, _p(xq),
                                                 _p(s_tok), _stream())

    def gemm(self, xq, s_tok, y):
        return self.dbg.convrot_int8_gemm(_p(xq), _p(s_tok), _p(self.Wq), _p(self.s_w), 1,
                                          _p(self.bias), self.M, self.N, self.K, _p(y), _stream())

    def decode(self, out):
        return self.dbg.convrot_dequant_derotate(_p(self.Wq), _p(self.s_w), 1, self.N, self.K,
                                                 self.h, _p(out), _stream())

    def status(self):
        return self.dbg.convrot_check_status(_stream())


def _filled(shape, dtype):
    t = torch.empty(shape, dtype=dtype, device="cuda")
    t.view(torch.uint8).fill_(SENTINEL)
    return t


def _untouched(t):
    return bool((t.reshape(-1).view(torch.uint8) == SENTINEL).all())


@pytest.mark.parametrize("M", [300, 16, 2])
def test_debug_library_matches_release_bit_for_bit(libs, M):
    cr, dbg = libs
    L = DebugLayer(cr, dbg, M, 512, 1024, seed=M)
    xq_r, st_r = cr.rotate_quant_act(L.x, L.rot)
    y_r = cr.int8_gemm(xq_r, st_r, L.Wq, L.s_w, L.bias)
    W_r = cr.dequant_derotate(L.Wq, L.s_w, L.rot)
    xq, st = _filled((M, L.K), torch.int8), _filled((M,), torch.float32)
    y, W = _filled((M, L.N), torch.bfloat16), _filled((L.N, L.K), torch.bfloat16)
    assert L.rotate(xq, st) == cr.OK
    assert L.gemm(xq, st, y) == cr.OK
    assert L.decode(W) == cr.OK
    assert L.status() == cr.OK, dbg.convrot_last_error_string()
    assert torch.equal(xq, xq_r) and torch.equal(st.view(torch.int32), st_r.view(torch.int32))
    assert torch.equal(y.view(torch.int16), y_r.view(torch.int16))
    assert torch.equal(W.view(torch.int16), W_r.view(torch.int16))
    L.close()


@pytest.mark.parametrize("M", [300, 16, 2])
def test_short_rows_fault_is_caught_and_skipped(libs, M):
    """The kernels believe the outputs one row shorter: the last row's stores
    are out of range, caught, skipped and reported; nothing else changes."""
    cr, dbg = libs
    L = DebugLayer(cr, dbg, M, 512, 1024, seed=M + 1)
    xq_r, st_r = cr.rotate_quant_act(L.x, L.rot)
    y_r = cr.int8_gemm(xq_r, st_r, L.Wq, L.s_w, L.bias)
    W_r = cr.dequant_derotate(L.Wq, L.s_w, L.rot)
    xq, st = _filled((M, L.K), torch.int8), _filled((M,), torch.float32)
    y, W = _filled((M, L.N), torch.bfloat16), _filled((L.N, L.K), torch.bfloat16)
    assert dbg.convrot_debug_set_fault(SHORT_ROWS) == cr.OK
    try:
        assert L.rotate(xq, st) == cr.OK
        assert L.status() == cr.BOUNDS
        assert b"out-of-range" in dbg.convrot_last_error_string()
        # the GEMM reads the complete codes of the release library
        assert L.gemm(xq_r, st_r, y) == cr.OK
        assert L.status() == cr.BOUNDS
        assert L.decode(W) == cr.OK
        assert L.status() == cr.BOUNDS
    finally:
        dbg.convrot_debug_set_fault(NONE)
    assert L.status() == cr.OK  # the word was cleared by the reads above
    assert _untouched(xq[-1]) and _untouched(st[-1:])
    assert torch.equal(xq[:-1], xq_r[:-1]) and torch.equal(st[:-1], st_r[:-1])
    assert _untouched(y[-1]) and torch.equal(y[:-1].view(torch.int16), y_r[:-1].view(torch.int16))
    # the decode sees the weight as one flat array: its last 256 elements are skipped
    Wf, Wrf = W.reshape(-1), W_r.reshape(-1)
    assert _untouched(Wf[-256:])
    assert torch.equal(Wf[:-256].view(torch.int16), Wrf[:-256].view(torch.int16))
    L.close()


@pytest.mark.parametrize("M", [300, 16])
def test_skipped_stage_times_out_and_the_context_recovers(libs, M):
    """An int8 GEMM whose producers leave their first ring stage empty: the
    MMA issuer's bounded wait (about a second) runs out, the kernel drains
    and returns, the status reads CONVROT_ERR_TIMEOUT, and the same GEMM
    computes the normal result right after on the same context.  M = 300 runs
    the CTA-pair kernel, M = 16 the few-token kernel (a cluster of 8 CTAs
    splitting K)."""
    cr, dbg = libs
    L = DebugLayer(cr, dbg, M, 512, 1024, seed=M + 2)
    xq_r, st_r = cr.rotate_quant_act(L.x, L.rot)
    y_r = cr.int8_gemm(xq_r, st_r, L.Wq, L.s_w, L.bias)
    y = _filled((M, L.N), torch.bfloat16)
    assert dbg.convrot_debug_set_fault(SKIP_STAGE) == cr.OK
    try:
        assert L.gemm(xq_r, st_r, y) == cr.OK
        assert L.status() == cr.TIMEOUT
        assert b"timeout" in dbg.convrot_last_error_string()
    finally:
        dbg.convrot_debug_set_fault(NONE)
    assert L.gemm(xq_r, st_r, y) == cr.OK
    assert L.status() == cr.OK
    assert torch.equal(y.view(torch.int16), y_r.view(torch.int16))
    L.close()
