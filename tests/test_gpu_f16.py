"""Parity of the fp16 forms of every entry point against the CPU oracle (fmt
"f16"), through the C ABI.  The pages' int8 layers take BF16 or FP16
activations (int8 Compute page); the tolerances are those of the bf16 tests:

  * activation / weight codes: at most 1 LSB apart on at most 0.1 % of them;
  * scales: relative 1e-6 (Sylvester) or G * 2^-24 (dense R);
  * decoded fp16 weight: bit-exact for the Sylvester R, within 1 fp16 ulp for
    a dense R;
  * GEMM epilogue: within 1 fp16 ulp of the float64 value rounded once, plus
    the float32 rounding of acc * scale (2^-21 of its magnitude);
  * layer output: relative L2 <= 2e-3 against the oracle and cosine >= 0.999
    against the unquantized float64 layer at G = 256.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu_helpers import Guarded, assert_codes_close

pytestmark = pytest.mark.gpu

F16 = torch.float16
cr = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global cr
    import activation_quantized_linear_b200 as mod
    cr = mod
    torch.cuda.set_device(0)
    assert mod.device_supported(0), "these kernels are built for sm_100a (B200)"
    yield


def _rotation(G, kind):
    return workloads.sylvester_rotation(G) if kind == "sylvester" else workloads.qr_rotation(G, seed=6000 + G)


def _scale_rtol(G, kind):
    return 1e-6 if kind == "sylvester" else G * 2.0 ** -24


def f16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def f16_ulp(v) -> np.ndarray:
    """Spacing of fp16 numbers at |v| (2^-24 in the subnormal range)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.ldexp(1.0, (e - 10).astype(np.int64))


def _codes(rng, shape):
    return rng.integers(-127, 128, size=shape, dtype=np.int64).astype(np.int8)


@pytest.mark.parametrize("G,kind,M,K", [
    (256, "sylvester", 129, 3840), (256, "sylvester", 7, 12288), (64, "sylvester", 33, 1024),
    (16, "sylvester", 5, 256), (4, "sylvester", 65, 512), (64, "qr", 9, 1024), (256, "qr", 3, 2048),
])
def test_rotate_quant_act_f16(G, kind, M, K):
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    x = workloads.make_activation(M, K, seed=G + M + K, dtype=F16)
    x[min(1, M - 1)] = 0
    xq_buf = Guarded((M, K), torch.int8)
    xq, s_tok = cr.rotate_quant_act(x.cuda(), rot, xq=xq_buf.tensor)
    torch.cuda.synchronize()
    xq_buf.check()
    ref_q, ref_s = oracle.rotate_quant_act(x, R)
    np.testing.assert_allclose(s_tok.cpu().numpy(), ref_s, rtol=_scale_rtol(G, kind), atol=0)
    assert_codes_close(xq.cpu().numpy(), ref_q)
    assert float(s_tok[min(1, M - 1)]) == 0.0


@pytest.mark.parametrize("G,kind,N,K", [(256, "sylvester", 136, 1024), (16, "sylvester", 64, 256),
                                        (64, "qr", 48, 512)])
def test_quantize_weight_f16(G, kind, N, K):
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    W = workloads.make_weight(N, K, seed=N + K, dtype=F16)
    Wq, s_w = cr.quantize_weight(W.cuda(), rot)
    ref_q, ref_s = oracle.quantize_weight(W, R)
    np.testing.assert_allclose(s_w.cpu().numpy()[0], ref_s, rtol=_scale_rtol(G, kind))
    assert_codes_close(Wq.cpu().numpy(), ref_q)


@pytest.mark.parametrize("G,kind,N,K", [(256, "sylvester", 1000, 3840), (4, "sylvester", 136, 1024),
                                        (64, "sylvester", 120, 2048), (16, "qr", 64, 512),
                                        (256, "qr", 32, 1024)])
def test_dequant_derotate_f16(G, kind, N, K):
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    W = workloads.make_weight(N, K, seed=N * 3 + K + G)
    Wq, s_w = oracle.quantize_weight(W, R)
    out = Guarded((N, K), F16)
    W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(),
                                torch.tensor([s_w], dtype=torch.float32, device="cuda"), rot,
                                out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    ref = oracle.dequant_derotate(Wq, s_w, R, "f16")
    if kind == "sylvester":
        np.testing.assert_array_equal(f16_bits(W_hat), oracle.f16_bits(ref))
    else:
        got = oracle.as_f64(W_hat.cpu())
        assert np.all(np.abs(got - ref) <= f16_ulp(ref)), "more than 1 fp16 ulp"


@pytest.mark.parametrize("G", [16, 256])
def test_dequant_derotate_f16_scales(G):
    """fp16 has subnormals where weights live (below 2^-14): small, short-mantissa
    and per-channel scales, bit-exact against the oracle."""
    N, K = 160, 1024
    R = workloads.sylvester_rotation(G)
    rot = cr.Rotation(R)
    rng = np.random.default_rng(G + 1)
    Wq = _codes(rng, (N, K))
    for s_w in (2.0 ** -9, 3 * 2.0 ** -20, 1.234567e-6, 7.5e-4):
        W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(),
                                    torch.tensor([s_w], dtype=torch.float32, device="cuda"), rot,
                                    dtype=F16)
        ref = oracle.dequant_derotate(Wq, np.float32(s_w), R, "f16")
        np.testing.assert_array_equal(f16_bits(W_hat), oracle.f16_bits(ref))
    s = (rng.random(N) * 1e-3 + 1e-6).astype(np.float32)
    s[::3] = 2.0 ** -12
    W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(), torch.from_numpy(s).cuda(), rot,
                                dtype=F16)
    ref = oracle.dequant_derotate(Wq, s, R, "f16")
    np.testing.assert_array_equal(f16_bits(W_hat), oracle.f16_bits(ref))


@pytest.mark.parametrize("M,N,K,with_bias,per_channel", [
    (300, 1024, 1024, True, False), (129, 272, 144, False, True), (7, 144, 64, True, False),
    (64, 512, 512, True, True), (2, 528, 2048, True, True),  # two tokens: the dp4a product
])
def test_int8_gemm_f16(M, N, K, with_bias, per_channel):
    rng = np.random.default_rng(M * N + K)
    a = _codes(rng, (M, K))
    b = _codes(rng, (N, K))
    s_tok = (rng.random(M) * 0.05).astype(np.float32)
    s_tok[0] = 0.0
    s_w = (rng.random(N) * 2e-3 + 1e-4).astype(np.float32) if per_channel else np.float32(1.3e-3)
    bias = workloads.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.5, F16) if with_bias else None
    out = Guarded((M, N), F16)
    y = cr.int8_gemm(torch.from_numpy(a).cuda(), torch.from_numpy(s_tok).cuda(),
                     torch.from_numpy(b).cuda(), torch.from_numpy(np.atleast_1d(s_w)).cuda(),
                     bias.cuda() if bias is not None else None, out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    acc = oracle.int8_gemm_acc(a, b)
    sw = np.broadcast_to(np.atleast_1d(s_w).astype(np.float64), (N,))
    ref = oracle.epilogue(acc, s_tok, s_w, bias, "f16")
    got = oracle.as_f64(y.cpu())
    mag = np.abs(acc.astype(np.float64) * s_tok.astype(np.float64)[:, None] * sw[None, :])
    if bias is not None:
        mag = mag + np.abs(oracle.as_f64(bias))[None, :]
    bad = np.abs(got - ref) > f16_ulp(ref) + mag * 2.0 ** -21
    assert not bad.any(), f"{bad.sum()} fp16 outputs off by more than 1 ulp"
    if with_bias:
        np.testing.assert_array_equal(got[0], oracle.as_f64(bias))


@pytest.mark.parametrize("kind", ["sylvester", "qr"])
@pytest.mark.parametrize("M", [64, 1, 200])
def test_linear_int8_f16(kind, M):
    lin = workloads.WORKLOADS["single_1024"][0]
    inp = workloads.make_layer_inputs(lin, 0, rotation=kind, M=M, dtype=F16)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    y = cr.linear_int8(inp.x.cuda(), Wq, s_w, rot, inp.bias.cuda())
    assert y.dtype == F16
    y_ref, *_ = oracle.linear_int8(inp.x, Wq.cpu().numpy(), float(s_w.item()), inp.R, inp.bias, "f16")
    got = oracle.as_f64(y.cpu())
    assert oracle.rel_l2(got, y_ref) <= 2e-3
    y_dense = oracle.linear_dense(inp.x, inp.W, inp.bias)
    assert oracle.cosine(got, y_dense) >= 0.999


def test_layer_module_f16():
    lin = workloads.Linear("f16_module", 96, 2048, 1024, G=256)
    inp = workloads.make_layer_inputs(lin, 2, dtype=F16)
    layer = cr.ConvRotLinear(inp.W.cuda(), inp.R, inp.bias.cuda())
    y = layer(inp.x.cuda())
    W_hat = layer.decode_weight()
    assert y.dtype == F16 and W_hat.dtype == F16
    y_dec = oracle.linear_dense(inp.x, oracle.as_f64(W_hat.cpu()), inp.bias)
    assert oracle.cosine(oracle.as_f64(y.cpu()), y_dec) >= 0.999
    with pytest.raises(TypeError):
        cr.linear_int8(inp.x.cuda(), layer.Wq, layer.s_w, layer.rotation,
                       inp.bias.cuda().to(torch.bfloat16))  # bias must match x's format
