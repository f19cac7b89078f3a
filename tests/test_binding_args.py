"""The Python binding's size checks, run on the CPU.

The C ABI takes raw pointers, so it cannot see that a weight is narrower than
the activations say, or that an output, bias or scale is too short: the
kernels would read or write past the allocation.  The binding therefore checks
every size before the call, and does so before it checks the device, so the
rejections below run with CPU tensors.  A tensor of the right size on the CPU
is then refused for not being on the GPU.
"""

import pytest
import torch

import activation_quantized_linear_b200 as cr

M, K, N = 8, 256, 64


def _t(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def _layer(**over):
    a = dict(x=_t(M, K), Wq=_t(N, K, dtype=torch.int8), s_w=_t(1, dtype=torch.float32),
             bias=_t(N), out=None)
    a.update(over)
    return a


BAD_LAYER = {
    "narrow_weight": (dict(Wq=_t(N, K // 2, dtype=torch.int8)), "input features"),
    "scale_length": (dict(s_w=_t(N - 1, dtype=torch.float32)), "scales"),
    "bias_length": (dict(bias=_t(N + 16)), "bias"),
    "out_rows": (dict(out=_t(M - 1, N)), "out must have shape"),
    "out_cols": (dict(out=_t(M, N // 2)), "out must have shape"),
}

LAYER_CALLS = {
    "linear_int8": lambda a: cr.linear_int8(a["x"], a["Wq"], a["s_w"], None, a["bias"], out=a["out"]),
    "linear_int8_noalloc": lambda a: cr.linear_int8_noalloc(a["x"], a["Wq"], a["s_w"], None,
                                                            a["bias"], out=a["out"]),
    "linear_dequant": lambda a: cr.linear_dequant(a["x"], a["Wq"], a["s_w"], None, a["bias"],
                                                  out=a["out"]),
    "linear_checked": lambda a: cr.linear_checked(a["x"], a["Wq"], a["s_w"], None, a["bias"],
                                                  out=a["out"]),
    "int8_gemm": lambda a: cr.int8_gemm(a["x"].to(torch.int8), _t(M, dtype=torch.float32), a["Wq"],
                                        a["s_w"], a["bias"], out=a["out"]),
}


@pytest.mark.parametrize("call", sorted(LAYER_CALLS))
@pytest.mark.parametrize("bad", sorted(BAD_LAYER))
def test_layer_size_rejected(call, bad):
    over, words = BAD_LAYER[bad]
    with pytest.raises(ValueError, match=words):
        LAYER_CALLS[call](_layer(**over))


@pytest.mark.parametrize("call", sorted(LAYER_CALLS))
def test_right_sizes_on_cpu_refused_for_the_device(call):
    with pytest.raises(ValueError, match="CUDA tensor"):
        LAYER_CALLS[call](_layer())


def test_gemm_token_scales_length():
    with pytest.raises(ValueError, match="s_tok"):
        cr.int8_gemm(_t(M, K, dtype=torch.int8), _t(M + 1, dtype=torch.float32),
                     _t(N, K, dtype=torch.int8), _t(1, dtype=torch.float32))


def test_dense_linear_sizes():
    with pytest.raises(ValueError, match="input features"):
        cr.dense_linear(_t(M, K), _t(N, K + 16))
    with pytest.raises(ValueError, match="bias"):
        cr.dense_linear(_t(M, K), _t(N, K), _t(N - 1))
    with pytest.raises(ValueError, match="out must have shape"):
        cr.dense_linear(_t(M, K), _t(N, K), None, out=_t(N, M))


def test_s32_gemm_sizes():
    with pytest.raises(ValueError, match="input features"):
        cr.int8_gemm_s32(_t(M, K, dtype=torch.int8), _t(N, K - 16, dtype=torch.int8))
    with pytest.raises(ValueError, match="out must have shape"):
        cr.int8_gemm_s32(_t(M, K, dtype=torch.int8), _t(N, K, dtype=torch.int8),
                         out=_t(M, N + 1, dtype=torch.int32))


def test_kernel_output_sizes():
    with pytest.raises(ValueError, match="xq must have shape"):
        cr.rotate_quant_act(_t(M, K), None, xq=_t(M, K - 32, dtype=torch.int8))
    with pytest.raises(ValueError, match="s_tok must have shape"):
        cr.rotate_quant_act(_t(M, K), None, s_tok=_t(M - 1, dtype=torch.float32))
    with pytest.raises(ValueError, match="Wq must have shape"):
        cr.quantize_weight(_t(N, K), None, Wq=_t(N, K // 2, dtype=torch.int8))
    with pytest.raises(ValueError, match="s_w must have shape"):
        cr.quantize_weight(_t(N, K), None, s_w=_t(2, dtype=torch.float32))
    with pytest.raises(ValueError, match="scales"):
        cr.dequant_derotate(_t(N, K, dtype=torch.int8), _t(N + 1, dtype=torch.float32), None)
    with pytest.raises(ValueError, match="out must have shape"):
        cr.dequant_derotate(_t(N, K, dtype=torch.int8), _t(1, dtype=torch.float32), None,
                            out=_t(K, N))
