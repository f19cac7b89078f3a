"""ConvRot int8_tensorwise linear layer on NVIDIA B200 (sm_100a).

A thin ctypes binding over libconvrot.so (C ABI in include/convrot.h).  Torch
provides device memory and the current stream only; every step of the layer
runs in the library's CUDA kernels.  There is no CPU fallback: if the library
is missing, importing the binding raises.

Entry points (same names as the C ABI, without the `convrot_` prefix; the
16-bit float tensors may be bf16 or fp16, which selects the `_f16` C entry):
    Rotation(R)                               the G x G rotation block, on the current device
    quantize_weight(W, rot)          -> (Wq, s_w)
    dequant_derotate(Wq, s_w, rot)   -> W_hat (bf16, or `dtype` / out's dtype)
    rotate_quant_act(x, rot)         -> (xq, s_tok)
    int8_gemm(xq, s_tok, Wq, s_w, bias)      -> y (out's, `dtype`'s or bias's dtype; bf16 by default)
    int8_gemm_s32(xq, Wq)                    -> acc (int32)
    linear_int8(x, Wq, s_w, rot, bias)       -> y (x's dtype)
    linear_int8_noalloc(x, Wq, s_w, rot, bias) -> y (bf16; the library's static scratch)
    dense_linear(x, W, bias)                 -> y (the default path's 16-bit matmul)
    linear_dequant(x, Wq, s_w, rot, bias)    -> y (the default path: decode, then dense_linear)
    linear_checked(x, Wq, s_w, rot, bias)    -> (y, path) (int8 compute, first call checked)
    check_state(device), check_reset(), check_set_min_cosine(t), check_min_cosine()
    workspace_bytes(M, N, K), check_status(), selftest_wait_timeout(ms)
    ConvRotLinear(W, R, bias, mode)           the layer: forward, decode_weight
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

__all__ = [
    "ConvRotError", "Rotation", "quantize_weight", "dequant_derotate", "rotate_quant_act",
    "int8_gemm", "int8_gemm_s32", "linear_int8", "workspace_bytes", "check_status",
    "device_supported", "library_path", "ConvRotLinear", "linear_int8_noalloc",
    "noalloc_scratch_bytes", "selftest_wait_timeout", "dense_linear", "linear_dequant",
    "linear_checked", "check_state", "check_reset", "check_set_min_cosine", "check_min_cosine",
]

OK, INVALID_ARG, UNSUPPORTED, CUDA, WORKSPACE, TIMEOUT, ALIGNMENT, BOUNDS = range(8)
OP_LINEAR_INT8, OP_LINEAR_INT8_SLICED, OP_LINEAR_DEQUANT, OP_LINEAR_CHECKED = 1, 2, 3, 4
PATH_INT8, PATH_DEQUANT = 1, 2
CHECK_ROWS = 256
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "WORKSPACE",
                5: "TIMEOUT", 6: "ALIGNMENT", 7: "BOUNDS"}


class ConvRotError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"convrot {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return _build.LIB_PATH


def load_library(path: str) -> ctypes.CDLL:
    """libconvrot.so, or a library built from the same sources (the debug
    library, build.DEBUG_LIB_PATH), with the C signatures of include/convrot.h."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python activation_quantized_linear_b200/build.py`"
            " (the layer has no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sigs = {
        "convrot_version": ([], i32),
        "convrot_device_supported": ([i32], i32),
        "convrot_last_error_string": ([], ctypes.c_char_p),
        "convrot_rotation_create": ([vp, i32, ctypes.POINTER(vp)], i32),
        "convrot_rotation_destroy": ([vp], i32),
        "convrot_rotation_info": ([vp, ctypes.POINTER(i32), ctypes.POINTER(i32)], i32),
        "convrot_quantize_weight": ([vp, i64, i64, vp, vp, vp, vp], i32),
        "convrot_dequant_derotate": ([vp, vp, i64, i64, i64, vp, vp, vp], i32),
        "convrot_rotate_quant_act": ([vp, i64, i64, vp, vp, vp, vp], i32),
        "convrot_int8_gemm": ([vp, vp, vp, vp, i64, vp, i64, i64, i64, vp, vp], i32),
        "convrot_int8_gemm_s32": ([vp, vp, i64, i64, i64, vp, vp], i32),
        "convrot_linear_int8": ([vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "convrot_workspace_bytes": ([i32, i64, i64, i64], sz),
        "convrot_linear_int8_noalloc": ([vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp], i32),
        "convrot_noalloc_scratch_bytes": ([], sz),
        "convrot_check_status": ([vp], i32),
        "convrot_selftest_wait_timeout": ([i32, vp], i32),
        "convrot_quantize_weight_f16": ([vp, i64, i64, vp, vp, vp, vp], i32),
        "convrot_dequant_derotate_f16": ([vp, vp, i64, i64, i64, vp, vp, vp], i32),
        "convrot_rotate_quant_act_f16": ([vp, i64, i64, vp, vp, vp, vp], i32),
        "convrot_int8_gemm_f16": ([vp, vp, vp, vp, i64, vp, i64, i64, i64, vp, vp], i32),
        "convrot_linear_int8_f16": ([vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "convrot_check_state": ([i32, ctypes.POINTER(i32), ctypes.POINTER(i32)], i32),
        "convrot_check_reset": ([], None),
        "convrot_check_set_min_cosine": ([ctypes.c_double], i32),
        "convrot_check_min_cosine": ([], ctypes.c_double),
    }
    for f in ("", "_f16"):
        sigs["convrot_dense_linear" + f] = ([vp, i64, i64, i64, vp, vp, vp, vp], i32)
        sigs["convrot_linear_dequant" + f] = (
            [vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp, sz, vp], i32)
        sigs["convrot_linear_checked" + f] = (
            [vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp, sz, ctypes.POINTER(i32), vp], i32)
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = load_library(_build.LIB_PATH)


def _check(status: int) -> None:
    if status != OK:
        raise ConvRotError(status, _lib.convrot_last_error_string().decode())


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


FLOAT16 = (torch.bfloat16, torch.float16)


def _tensor(t, name: str) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")


def _shape(t: torch.Tensor | None, name: str, shape: tuple) -> None:
    """An optional caller-supplied tensor must have exactly `shape`."""
    if t is None:
        return
    _tensor(t, name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _layer_shapes(x, Wq, s_w, bias, out) -> tuple[int, int, int]:
    """The layer's size contract, checked before anything reaches the C ABI
    (which takes raw pointers and cannot see a size): Wq [N, K] for x [M, K],
    one weight scale or N of them (s_w None: no scale), N biases, out [M, N].
    Returns (M, K, N)."""
    for t, name in ((x, "x"), (Wq, "Wq")):
        _tensor(t, name)
    if x.dim() != 2 or Wq.dim() != 2:
        raise ValueError(f"x and Wq must be 2-D, got {tuple(x.shape)} and {tuple(Wq.shape)}")
    M, K = x.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError(f"Wq has {Wq.shape[1]} input features, x has {K}")
    if s_w is not None:
        _tensor(s_w, "s_w")
        if s_w.numel() not in (1, N):
            raise ValueError(f"s_w must hold 1 or N = {N} scales, got {s_w.numel()}")
    if bias is not None:
        _tensor(bias, "bias")
        if bias.numel() != N:
            raise ValueError(f"bias must hold N = {N} values, got {bias.numel()}")
    _shape(out, "out", (M, N))
    return M, K, N


def _on_current_device(**tensors) -> None:
    """Every tensor handed to the library must live on the current CUDA device:
    the library launches there and resolves its per-device state (rotation
    copy, static scratch, status word) there."""
    dev = torch.cuda.current_device()
    for name, t in tensors.items():
        if t is not None and (t.device.type != "cuda" or t.device.index != dev):
            raise ValueError(f"{name} is on {t.device}; the current device is cuda:{dev}")


def _need16(t: torch.Tensor, name: str, ndim: int) -> None:
    """A bf16 or fp16 tensor (the layer's two activation formats)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in FLOAT16:
        raise TypeError(f"{name} must be bfloat16 or float16, got {t.dtype}")
    _need(t, name, t.dtype, ndim)


def _fn(name: str, dtype: torch.dtype):
    """The C entry point for a 16-bit float format: name (bf16) or name_f16."""
    return getattr(_lib, name + ("_f16" if dtype == torch.float16 else ""))


def device_supported(device: int = 0) -> bool:
    return bool(_lib.convrot_device_supported(device))


class Rotation:
    """The orthogonal G x G block R (float32), copied to the current device.

    A normalized Sylvester-Hadamard R (bit for bit) selects the butterfly
    kernels; any other orthogonal R the dense ones."""

    def __init__(self, R):
        if isinstance(R, torch.Tensor):
            R = R.detach().to("cpu").float().numpy()
        R = np.ascontiguousarray(R, dtype=np.float32)
        if R.ndim != 2 or R.shape[0] != R.shape[1]:
            raise ValueError("R must be a square matrix")
        self._R = R
        h = ctypes.c_void_p()
        _check(_lib.convrot_rotation_create(R.ctypes.data, int(R.shape[0]), ctypes.byref(h)))
        self._h = h
        g, syl = ctypes.c_int(), ctypes.c_int()
        _check(_lib.convrot_rotation_info(h, ctypes.byref(g), ctypes.byref(syl)))
        self.G = g.value
        self.is_sylvester = bool(syl.value)
        self.device = torch.cuda.current_device()

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise ValueError("rotation was closed")
        return self._h

    @property
    def matrix(self) -> np.ndarray:
        return self._R

    def close(self) -> None:
        if getattr(self, "_h", None) is not None:
            _lib.convrot_rotation_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quantize_weight(W: torch.Tensor, rot: Rotation, Wq: torch.Tensor | None = None,
                    s_w: torch.Tensor | None = None):
    """W [N, K] bf16 or fp16 -> (Wq [N, K] int8, s_w [1] float32)."""
    _tensor(W, "W")
    if W.dim() == 2:
        _shape(Wq, "Wq", tuple(W.shape))
        _shape(s_w, "s_w", (1,))
    _need16(W, "W", 2)
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq is None else Wq
    s_w = torch.empty(1, dtype=torch.float32, device=W.device) if s_w is None else s_w
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    _on_current_device(W=W, Wq=Wq, s_w=s_w)
    _check(_fn("convrot_quantize_weight", W.dtype)(_ptr(W), N, K, rot.handle, _ptr(Wq), _ptr(s_w),
                                                    _stream()))
    return Wq, s_w


def dequant_derotate(Wq: torch.Tensor, s_w: torch.Tensor, rot: Rotation,
                     out: torch.Tensor | None = None,
                     dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Wq [N, K] int8, s_w [1] or [N] float32 -> W_hat [N, K] in `dtype` (bf16 or
    fp16; the dtype of `out` when given)."""
    _tensor(Wq, "Wq")
    _tensor(s_w, "s_w")
    if Wq.dim() == 2:
        if s_w.numel() not in (1, Wq.shape[0]):
            raise ValueError(f"s_w must hold 1 or N = {Wq.shape[0]} scales, got {s_w.numel()}")
        _shape(out, "out", tuple(Wq.shape))
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    N, K = Wq.shape
    out = torch.empty((N, K), dtype=dtype, device=Wq.device) if out is None else out
    _need16(out, "out", 2)
    _on_current_device(Wq=Wq, s_w=s_w, out=out)
    _check(_fn("convrot_dequant_derotate", out.dtype)(_ptr(Wq), _ptr(s_w), s_w.numel(), N, K,
                                                       rot.handle, _ptr(out), _stream()))
    return out


def rotate_quant_act(x: torch.Tensor, rot: Rotation, xq: torch.Tensor | None = None,
                     s_tok: torch.Tensor | None = None):
    """x [M, K] bf16 or fp16 -> (xq [M, K] int8, s_tok [M] float32)."""
    _tensor(x, "x")
    if x.dim() == 2:
        _shape(xq, "xq", tuple(x.shape))
        _shape(s_tok, "s_tok", (x.shape[0],))
    _need16(x, "x", 2)
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    s_tok = torch.empty(M, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _need(xq, "xq", torch.int8, 2)
    _need(s_tok, "s_tok", torch.float32, 1)
    _on_current_device(x=x, xq=xq, s_tok=s_tok)
    _check(_fn("convrot_rotate_quant_act", x.dtype)(_ptr(x), M, K, rot.handle, _ptr(xq),
                                                     _ptr(s_tok), _stream()))
    return xq, s_tok


def int8_gemm(xq: torch.Tensor, s_tok: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor,
              bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
              dtype: torch.dtype | None = None) -> torch.Tensor:
    """y = xq . Wq^T * s_tok[:, None] * s_w + bias, rounded once to a 16-bit
    float: the dtype of `out` when given, else `dtype`, else the bias's dtype,
    else bf16.  The bias, if any, is in the output's dtype."""
    M, K, N = _layer_shapes(xq, Wq, s_w, bias, out)
    _tensor(s_tok, "s_tok")
    if s_tok.numel() != M:
        raise ValueError(f"s_tok must hold M = {M} scales, got {s_tok.numel()}")
    _need(xq, "xq", torch.int8, 2)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_tok, "s_tok", torch.float32, 1)
    _need(s_w, "s_w", torch.float32, 1)
    if out is None:
        dtype = dtype or (bias.dtype if bias is not None else torch.bfloat16)
        out = torch.empty((M, N), dtype=dtype, device=xq.device)
    _need16(out, "out", 2)
    if bias is not None:
        _need(bias, "bias", out.dtype, 1)
    _on_current_device(xq=xq, s_tok=s_tok, Wq=Wq, s_w=s_w, bias=bias, out=out)
    _check(_fn("convrot_int8_gemm", out.dtype)(_ptr(xq), _ptr(s_tok), _ptr(Wq), _ptr(s_w),
                                                s_w.numel(), _ptr(bias), M, N, K, _ptr(out),
                                                _stream()))
    return out


def int8_gemm_s32(xq: torch.Tensor, Wq: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """acc = xq . Wq^T as int32 (diagnostic form of the GEMM)."""
    _tensor(xq, "xq")
    _tensor(Wq, "Wq")
    if xq.dim() == 2 and Wq.dim() == 2:
        if Wq.shape[1] != xq.shape[1]:
            raise ValueError(f"Wq has {Wq.shape[1]} input features, xq has {xq.shape[1]}")
        _shape(out, "out", (xq.shape[0], Wq.shape[0]))
    _need(xq, "xq", torch.int8, 2)
    _need(Wq, "Wq", torch.int8, 2)
    M, K = xq.shape
    N = Wq.shape[0]
    out = torch.empty((M, N), dtype=torch.int32, device=xq.device) if out is None else out
    _need(out, "out", torch.int32, 2)
    _on_current_device(xq=xq, Wq=Wq, out=out)
    _check(_lib.convrot_int8_gemm_s32(_ptr(xq), _ptr(Wq), M, N, K, _ptr(out), _stream()))
    return out


def workspace_bytes(M: int, N: int, K: int, sliced: bool = False, op: int | None = None) -> int:
    """Workspace of linear_int8 for all M tokens at once, or (sliced=True) for
    slices of at most 2N tokens; any size down to one row works.  `op` names
    another operation (OP_LINEAR_DEQUANT, OP_LINEAR_CHECKED)."""
    if op is None:
        op = OP_LINEAR_INT8_SLICED if sliced else OP_LINEAR_INT8
    return int(_lib.convrot_workspace_bytes(op, M, N, K))


def _workspace(workspace: torch.Tensor | None, need: int, device) -> torch.Tensor:
    if workspace is None:
        return torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8, 1)
    _on_current_device(workspace=workspace)
    return workspace


def linear_int8(x: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor, rot: Rotation,
                bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The int8-compute forward: rotate+quantize x per token, int8 GEMM, rescale.
    x, bias and the output share one 16-bit float format (bf16 or fp16)."""
    M, K, N = _layer_shapes(x, Wq, s_w, bias, out)
    _need16(x, "x", 2)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    if bias is not None:
        _need(bias, "bias", x.dtype, 1)
    need = workspace_bytes(M, N, K)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _need(workspace, "workspace", torch.uint8, 1)
    out = torch.empty((M, N), dtype=x.dtype, device=x.device) if out is None else out
    _need(out, "out", x.dtype, 2)
    _on_current_device(x=x, Wq=Wq, s_w=s_w, bias=bias, out=out, workspace=workspace)
    _check(_fn("convrot_linear_int8", x.dtype)(_ptr(x), M, K, N, rot.handle, _ptr(Wq), _ptr(s_w),
                                                s_w.numel(), _ptr(bias), _ptr(out),
                                                _ptr(workspace), workspace.numel(), _stream()))
    return out


def linear_int8_noalloc(x: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor, rot: Rotation,
                       bias: torch.Tensor | None = None,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """linear_int8 for callers that cannot allocate device memory: the
    intermediate codes and scales live in the library's static scratch
    (noalloc_scratch_bytes() bytes per GPU).  Pass `out` to allocate nothing."""
    M, K, N = _layer_shapes(x, Wq, s_w, bias, out)
    _need(x, "x", torch.bfloat16, 2)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", torch.bfloat16, 2)
    _on_current_device(x=x, Wq=Wq, s_w=s_w, bias=bias, out=out)
    _check(_lib.convrot_linear_int8_noalloc(_ptr(x), M, K, N, rot.handle, _ptr(Wq), _ptr(s_w),
                                            s_w.numel(), _ptr(bias), _ptr(out), _stream()))
    return out


def dense_linear(x: torch.Tensor, W: torch.Tensor, bias: torch.Tensor | None = None,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """The default path's matmul: y = x W^T + bias, x, W, bias and y in one
    16-bit float format, fp32 accumulation on the tensor cores."""
    _tensor(W, "W")
    M, K, N = _layer_shapes(x, W, None, bias, out)
    _need16(x, "x", 2)
    _need(W, "W", x.dtype, 2)
    if bias is not None:
        _need(bias, "bias", x.dtype, 1)
    out = torch.empty((M, N), dtype=x.dtype, device=x.device) if out is None else out
    _need(out, "out", x.dtype, 2)
    _on_current_device(x=x, W=W, bias=bias, out=out)
    _check(_fn("convrot_dense_linear", x.dtype)(_ptr(x), M, K, N, _ptr(W), _ptr(bias), _ptr(out),
                                                 _stream()))
    return out


def _linear_args(x, Wq, s_w, bias, out):
    M, K, N = _layer_shapes(x, Wq, s_w, bias, out)
    _need16(x, "x", 2)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    if bias is not None:
        _need(bias, "bias", x.dtype, 1)
    out = torch.empty((M, N), dtype=x.dtype, device=x.device) if out is None else out
    _need(out, "out", x.dtype, 2)
    _on_current_device(x=x, Wq=Wq, s_w=s_w, bias=bias, out=out)
    return M, K, N, out


def linear_dequant(x: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor, rot: Rotation,
                   bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The default path: decode the weight (into the workspace), then dense_linear."""
    M, K, N, out = _linear_args(x, Wq, s_w, bias, out)
    workspace = _workspace(workspace, workspace_bytes(M, N, K, op=OP_LINEAR_DEQUANT), x.device)
    _check(_fn("convrot_linear_dequant", x.dtype)(
        _ptr(x), M, K, N, rot.handle, _ptr(Wq), _ptr(s_w), s_w.numel(), _ptr(bias), _ptr(out),
        _ptr(workspace), workspace.numel(), _stream()))
    return out


def linear_checked(x: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor, rot: Rotation,
                   bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None) -> tuple[torch.Tensor, int]:
    """The int8-compute forward whose first call per (layer shape, token bucket)
    is checked against the default path; returns (y, PATH_INT8 or PATH_DEQUANT)."""
    M, K, N, out = _linear_args(x, Wq, s_w, bias, out)
    workspace = _workspace(workspace, workspace_bytes(M, N, K, op=OP_LINEAR_CHECKED), x.device)
    path = ctypes.c_int(0)
    _check(_fn("convrot_linear_checked", x.dtype)(
        _ptr(x), M, K, N, rot.handle, _ptr(Wq), _ptr(s_w), s_w.numel(), _ptr(bias), _ptr(out),
        _ptr(workspace), workspace.numel(), ctypes.byref(path), _stream()))
    return out, path.value


def check_state(device: int | None = None) -> tuple[bool, int]:
    """(latched onto the default path, number of checked keys) of a CUDA device."""
    dev = torch.cuda.current_device() if device is None else int(device)
    latched, keys = ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.convrot_check_state(dev, ctypes.byref(latched), ctypes.byref(keys)))
    return bool(latched.value), int(keys.value)


def check_reset() -> None:
    """Forget every checked key and latch (as a process restart would)."""
    _lib.convrot_check_reset()


def check_set_min_cosine(threshold: float) -> None:
    _check(_lib.convrot_check_set_min_cosine(float(threshold)))


def check_min_cosine() -> float:
    return float(_lib.convrot_check_min_cosine())


def noalloc_scratch_bytes() -> int:
    return int(_lib.convrot_noalloc_scratch_bytes())


def check_status(stream: torch.cuda.Stream | None = None) -> None:
    """Synchronize and raise if a kernel gave up a bounded wait since the last check."""
    s = (stream or torch.cuda.current_stream()).cuda_stream
    _check(_lib.convrot_check_status(s))


def selftest_wait_timeout(limit_ms: int = 20) -> None:
    """Enqueue the failure-detection self-test: a kernel whose bounded wait runs
    out after `limit_ms`; the next check_status() raises ConvRotError(TIMEOUT)."""
    _check(_lib.convrot_selftest_wait_timeout(int(limit_ms), _stream()))


class ConvRotLinear:
    """A ConvRot int8_tensorwise linear: int8 weight, per-tensor scale, rotation R.

    `forward` runs in the input's format (bf16 or fp16; the bias, if any, must
    match it) on the path `mode` names: "int8" (int8 compute), "dequant" (the
    default path: decode the weight, then a 16-bit matmul) or "checked" (int8
    compute whose first call per layer shape and token bucket is checked
    against the default path, falling back to it on a mismatch).
    `decode_weight` is the default path's weight decode (dequantize +
    derotate), to W's format unless `dtype` says otherwise."""

    MODES = ("int8", "dequant", "checked")

    def __init__(self, W: torch.Tensor, R, bias: torch.Tensor | None = None, mode: str = "int8"):
        if mode not in self.MODES:
            raise ValueError(f"mode must be one of {self.MODES}, got {mode!r}")
        self.rotation = R if isinstance(R, Rotation) else Rotation(R)
        self.Wq, self.s_w = quantize_weight(W, self.rotation)
        self.dtype = W.dtype
        self.bias = bias
        self.mode = mode
        self.last_path = None
        self._ws = None

    @property
    def out_features(self) -> int:
        return self.Wq.shape[0]

    @property
    def in_features(self) -> int:
        return self.Wq.shape[1]

    def decode_weight(self, out: torch.Tensor | None = None,
                      dtype: torch.dtype | None = None) -> torch.Tensor:
        return dequant_derotate(self.Wq, self.s_w, self.rotation, out=out,
                                dtype=dtype or self.dtype)

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        M = x.shape[0]
        op = {"int8": OP_LINEAR_INT8, "dequant": OP_LINEAR_DEQUANT,
              "checked": OP_LINEAR_CHECKED}[self.mode]
        need = workspace_bytes(M, self.out_features, self.in_features, op=op)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
        args = (x, self.Wq, self.s_w, self.rotation, self.bias)
        if self.mode == "int8":
            self.last_path = PATH_INT8
            return linear_int8(*args, out=out, workspace=self._ws)
        if self.mode == "dequant":
            self.last_path = PATH_DEQUANT
            return linear_dequant(*args, out=out, workspace=self._ws)
        y, self.last_path = linear_checked(*args, out=out, workspace=self._ws)
        return y

    __call__ = forward
