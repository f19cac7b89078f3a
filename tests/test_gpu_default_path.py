"""The default path and the checked int8 forward, through the C ABI.

  * dense_linear: the default path's 16-bit matmul y = f16(x W^T + b).  With
    small-integer operands every product and partial sum is exact in fp32, so
    the result is bit-exact against the oracle.  With random operands the
    bound follows from the arithmetic: one rounding of the exact sum to the
    16-bit format (1 ulp with the fp32 rounding before it), plus fp32
    accumulation on the tensor cores, one rounding per 16-element K step and
    per running sum, each at most 2^-23 of sum_k |x_k W_k|.
  * linear_dequant: the decoded weight in the workspace bit-exact (Sylvester R)
    and the output within the dense_linear bound of the oracle's default path.
  * linear_checked: the first call per key checks against the default path
    and returns the int8 result bit for bit; a mismatch (forced through the
    threshold, on the host) or a kernel timeout (the bounded-wait self-test)
    latches the device onto the default path, with one warning.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu_helpers import Guarded, bf16_bits, bf16_ulp

pytestmark = pytest.mark.gpu

cr = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global cr
    import activation_quantized_linear_b200 as mod
    cr = mod
    torch.cuda.set_device(0)
    assert mod.device_supported(0), "these kernels are built for sm_100a (B200)"
    yield


@pytest.fixture
def fresh_check():
    """Every checked-forward test starts and ends with no checked key, no latch
    and the default threshold."""
    cr.check_reset()
    cr.check_set_min_cosine(0.99)
    yield
    cr.check_reset()
    cr.check_set_min_cosine(0.99)


def f16_ulp(v) -> np.ndarray:
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.ldexp(1.0, (e - 10).astype(np.int64))


def ulp16(v, dtype) -> np.ndarray:
    return f16_ulp(v) if dtype == torch.float16 else bf16_ulp(v)


def fmt_of(dtype) -> str:
    return "f16" if dtype == torch.float16 else "bf16"


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def dense_bound(x64, W64, b64, K) -> np.ndarray:
    """fp32 accumulation bound: (K/16 + 16) roundings of at most 2^-23 of sum |x W|."""
    mag = np.abs(x64) @ np.abs(W64).T
    if b64 is not None:
        mag = mag + np.abs(b64)[None, :]
    return mag * (K / 16 + 16) * 2.0 ** -23


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K", [(300, 272, 144), (7, 144, 64), (513, 1040, 4096), (1, 16, 16)])
def test_dense_linear_exact_on_small_integers(dtype, M, N, K):
    rng = np.random.default_rng(M + N + K)
    x = rng.integers(-3, 4, (M, K)).astype(np.float32)
    W = rng.integers(-3, 4, (N, K)).astype(np.float32)
    b = rng.integers(-50, 51, N).astype(np.float32)
    out = Guarded((M, N), dtype)
    y = cr.dense_linear(torch.from_numpy(x).to(dtype).cuda(), torch.from_numpy(W).to(dtype).cuda(),
                        torch.from_numpy(b).to(dtype).cuda(), out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    ref = oracle.round16(oracle.linear_dense(x, W, b), fmt_of(dtype))
    np.testing.assert_array_equal(oracle.as_f64(y.cpu()), ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K,with_bias", [(300, 1024, 3840, True), (129, 272, 144, False),
                                             (1, 256, 1024, True), (1000, 528, 2048, True)])
def test_dense_linear_random(dtype, M, N, K, with_bias):
    x = workloads.make_activation(M, K, seed=M + K, dtype=dtype)
    W = workloads.make_weight(N, K, seed=N + K, dtype=dtype)
    b = workloads.make_weight(1, N, seed=N, dtype=dtype)[0] if with_bias else None
    out = Guarded((M, N), dtype)
    y = cr.dense_linear(x.cuda(), W.cuda(), b.cuda() if b is not None else None, out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    x64, W64 = oracle.as_f64(x), oracle.as_f64(W)
    b64 = oracle.as_f64(b) if b is not None else None
    ref = oracle.round16(oracle.linear_dense(x64, W64, b64), fmt_of(dtype))
    got = oracle.as_f64(y.cpu())
    tol = ulp16(ref, dtype) + dense_bound(x64, W64, b64, K)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{bad.sum()} outputs outside the fp32-accumulation bound"


def test_dense_linear_errors():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(24, 64, dtype=torch.bfloat16, device="cuda")  # N % 16 != 0
    with pytest.raises(cr.ConvRotError) as e:
        cr.dense_linear(x, W)
    assert e.value.status == cr.INVALID_ARG
    with pytest.raises(TypeError):
        cr.dense_linear(x, W.to(torch.float16))
    y = cr.dense_linear(x[:0], torch.zeros(16, 64, dtype=torch.bfloat16, device="cuda"))
    assert y.shape == (0, 16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("G,kind,M", [(256, "sylvester", 200), (64, "sylvester", 1), (16, "qr", 64)])
def test_linear_dequant(dtype, G, kind, M):
    lin = workloads.Linear("dequant", M, 1024, 1536, G=G)
    inp = workloads.make_layer_inputs(lin, 1, rotation=kind, dtype=dtype)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    N, K = 1536, 1024
    ws = torch.empty(cr.workspace_bytes(M, N, K, op=cr.OP_LINEAR_DEQUANT), dtype=torch.uint8,
                     device="cuda")
    y = cr.linear_dequant(inp.x.cuda(), Wq, s_w, rot, inp.bias.cuda(), workspace=ws)
    torch.cuda.synchronize()
    Wq_h, s_h = Wq.cpu().numpy(), float(s_w.item())
    W_hat = oracle.dequant_derotate(Wq_h, s_h, inp.R, fmt_of(dtype))
    W_ws = oracle.as_f64(ws[:2 * N * K].view(dtype).view(N, K).cpu())
    if kind == "sylvester":
        np.testing.assert_array_equal(W_ws, W_hat)
    else:
        assert np.all(np.abs(W_ws - W_hat) <= ulp16(W_hat, dtype)), "decode off by more than 1 ulp"
    ref = oracle.linear_dequant(inp.x, Wq_h, s_h, inp.R, inp.bias, fmt_of(dtype))
    got = oracle.as_f64(y.cpu())
    x64, b64 = oracle.as_f64(inp.x), oracle.as_f64(inp.bias)
    tol = ulp16(ref, dtype) + dense_bound(x64, W_hat, b64, K)
    if kind != "sylvester":  # a decoded weight 1 ulp apart moves the sum by at most that much
        tol = tol + np.abs(x64) @ ulp16(W_hat, dtype).T
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{bad.sum()} outputs outside the bound"


def test_linear_dequant_per_channel_scale():
    lin = workloads.Linear("dequant", 96, 512, 640, G=64)
    inp = workloads.make_layer_inputs(lin, 2)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    rng = np.random.default_rng(5)
    s = (float(s_w.item()) * (1 + 0.2 * rng.random(640))).astype(np.float32)
    y = cr.linear_dequant(inp.x.cuda(), Wq, torch.from_numpy(s).cuda(), rot, inp.bias.cuda())
    Wq_h = Wq.cpu().numpy()
    W_hat = oracle.dequant_derotate(Wq_h, s, inp.R)
    x64, b64 = oracle.as_f64(inp.x), oracle.as_f64(inp.bias)
    ref = oracle.linear_dequant(x64, Wq_h, s, inp.R, b64)
    got = oracle.as_f64(y.cpu())
    assert np.all(np.abs(got - ref) <= bf16_ulp(ref) + dense_bound(x64, W_hat, b64, 512))


def test_linear_dequant_workspace_errors():
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(64, 256, dtype=torch.int8, device="cuda")
    s_w = torch.ones(1, device="cuda")
    rot = cr.Rotation(workloads.sylvester_rotation(16))
    small = torch.empty(2 * 64 * 256 - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.linear_dequant(x, Wq, s_w, rot, workspace=small)
    assert e.value.status == cr.WORKSPACE


def _layer(M, N=1024, K=1024, G=256, index=0, dtype=torch.bfloat16):
    inp = workloads.make_layer_inputs(workloads.Linear("checked", M, K, N, G=G), index, dtype=dtype)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    return inp.x.cuda(), Wq, s_w, rot, inp.bias.cuda()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_checked_first_call_then_int8(fresh_check, dtype, capfd):
    x, Wq, s_w, rot, b = _layer(300, dtype=dtype)
    y_int8 = cr.linear_int8(x, Wq, s_w, rot, b)
    y, path = cr.linear_checked(x, Wq, s_w, rot, b)
    assert path == cr.PATH_INT8
    np.testing.assert_array_equal(bits16(y), bits16(y_int8))
    assert cr.check_state(0) == (False, 1)
    # same key (M bucket 9 holds 257..512 tokens): no new check
    y2, path2 = cr.linear_checked(x[:260].contiguous(), Wq, s_w, rot, b)
    assert path2 == cr.PATH_INT8 and cr.check_state(0) == (False, 1)
    np.testing.assert_array_equal(bits16(y2), bits16(y_int8[:260]))
    # another bucket and another shape are new keys
    cr.linear_checked(x[:3].contiguous(), Wq, s_w, rot, b)
    x2, Wq2, s2, rot2, b2 = _layer(64, N=512, K=2048, G=64, index=1, dtype=dtype)
    _, path3 = cr.linear_checked(x2, Wq2, s2, rot2, b2)
    assert path3 == cr.PATH_INT8 and cr.check_state(0) == (False, 3)
    assert "int8 compute disabled" not in capfd.readouterr().err


def test_checked_mismatch_latches_default_path(fresh_check, capfd):
    x, Wq, s_w, rot, b = _layer(200)
    y_dq = cr.linear_dequant(x, Wq, s_w, rot, b)
    cr.check_set_min_cosine(1.2)  # no result can match: the fallback runs, no kernel is faulty
    out = Guarded((200, 1024), torch.bfloat16)
    y, path = cr.linear_checked(x, Wq, s_w, rot, b, out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    assert path == cr.PATH_DEQUANT
    np.testing.assert_array_equal(bf16_bits(y), bf16_bits(y_dq))
    assert cr.check_state(0)[0] is True
    err = capfd.readouterr().err
    assert err.count("int8 compute disabled on CUDA device 0") == 1 and "cosine" in err
    # latched: every later call takes the default path, with no second warning
    cr.check_set_min_cosine(0.99)
    x2, Wq2, s2, rot2, b2 = _layer(64, N=512, K=2048, G=64, index=1)
    y2, path2 = cr.linear_checked(x2, Wq2, s2, rot2, b2)
    assert path2 == cr.PATH_DEQUANT
    np.testing.assert_array_equal(bf16_bits(y2), bf16_bits(cr.linear_dequant(x2, Wq2, s2, rot2, b2)))
    assert "int8 compute disabled" not in capfd.readouterr().err
    cr.check_reset()
    _, path3 = cr.linear_checked(x2, Wq2, s2, rot2, b2)
    assert path3 == cr.PATH_INT8


def test_checked_kernel_timeout_latches(fresh_check, capfd):
    """A kernel that gave up a bounded wait (the self-test, which faults
    nothing) counts as a failed int8 kernel on the first call."""
    x, Wq, s_w, rot, b = _layer(128)
    cr.selftest_wait_timeout(5)
    y, path = cr.linear_checked(x, Wq, s_w, rot, b)
    assert path == cr.PATH_DEQUANT
    np.testing.assert_array_equal(bf16_bits(y), bf16_bits(cr.linear_dequant(x, Wq, s_w, rot, b)))
    assert "timeout" in capfd.readouterr().err
    cr.check_status()  # the status word was read and cleared by the check


def test_checked_argument_errors_latch_nothing(fresh_check):
    x, Wq, s_w, rot, b = _layer(32)
    with pytest.raises(cr.ConvRotError) as e:
        cr.linear_checked(x, Wq, s_w, rot, b, workspace=torch.empty(256, dtype=torch.uint8,
                                                                   device="cuda"))
    assert e.value.status == cr.WORKSPACE
    with pytest.raises(cr.ConvRotError) as e:
        cr.linear_checked(x[:, :1000].contiguous(), Wq[:, :1000].contiguous(), s_w, rot, b)
    assert e.value.status == cr.INVALID_ARG  # K % G != 0
    assert cr.check_state(0) == (False, 0)
    y, path = cr.linear_checked(x[:0], Wq, s_w, rot, b)
    assert y.shape == (0, 1024) and path == cr.PATH_INT8


def test_layer_modes(fresh_check):
    lin = workloads.Linear("modes", 96, 2048, 1024, G=256)
    inp = workloads.make_layer_inputs(lin, 3)
    W, b, x = inp.W.cuda(), inp.bias.cuda(), inp.x.cuda()
    ys = {}
    for mode in cr.ConvRotLinear.MODES:
        layer = cr.ConvRotLinear(W, inp.R, b, mode=mode)
        ys[mode] = layer(x)
        assert layer.last_path == (cr.PATH_DEQUANT if mode == "dequant" else cr.PATH_INT8)
    np.testing.assert_array_equal(bf16_bits(ys["checked"]), bf16_bits(ys["int8"]))
    y_dense = oracle.linear_dense(inp.x, inp.W, inp.bias)
    for mode in cr.ConvRotLinear.MODES:
        assert oracle.cosine(oracle.as_f64(ys[mode].cpu()), y_dense) >= 0.999
    with pytest.raises(ValueError):
        cr.ConvRotLinear(W, inp.R, b, mode="fp32")
