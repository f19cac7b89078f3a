"""Per-kernel parity of the CUDA path against the CPU oracle on small and odd
shapes (several tiles plus ragged tails), through the C ABI.

Tolerances (fixed by the acceptance criteria of the layer):
  * int32 accumulators: bit-exact given identical int8 codes;
  * activation / weight codes: at most 1 LSB apart on at most 0.1 % of the
    elements (float32 rotation order and reciprocal-vs-division at .5 ties);
  * scales: relative 1e-6;
  * derotated bf16 weight: bit-exact for the Sylvester R (exact integer sums and
    a single correct rounding), within 1 bf16 ulp for a dense R;
  * layer output: relative L2 <= 2e-3 against the oracle, and cosine >= 0.999
    against the unquantized float64 layer.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu_helpers import (Guarded, assert_codes_close, bf16_bits, bf16_ulp,
                                to_cuda_bf16)

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


def _rotation(G, kind):
    return workloads.sylvester_rotation(G) if kind == "sylvester" else workloads.qr_rotation(G, seed=6000 + G)


def _scale_rtol(G, kind):
    """Relative tolerance of a float32 absmax scale against the float64 oracle.
    The butterfly adds exact-sign terms with a few roundings: 1e-6.  A dense R
    sums G float32 products: the classic bound G * 2^-24 of a float32 dot product."""
    return 1e-6 if kind == "sylvester" else G * 2.0 ** -24


def _codes(rng, shape):
    return rng.integers(-127, 128, size=shape, dtype=np.int64).astype(np.int8)


# ---------------------------------------------------------------------------
# int8 GEMM main loop: bit-exact int32
# ---------------------------------------------------------------------------
GEMM_SHAPES = [
    (1, 16, 16), (7, 144, 64), (128, 256, 128), (129, 272, 144), (257, 512, 1024),
    (300, 1024, 3840), (64, 1024, 1024), (1000, 528, 2048), (33, 4096, 256), (97, 1008, 4096),
    # one or two tokens whose codes fit 64 KB take the dp4a product: one, two
    # and eight 4 KB row blocks, several rows per warp, the largest K it takes
    # and the first past it (swap-AB); and a few more swap-AB token counts
    (2, 21504, 3072), (1, 1040, 8192), (2, 528, 32768), (2, 528, 32784), (1, 4096, 4096),
    (5, 1040, 8192), (8, 528, 8192), (3, 4096, 4096),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_int8_gemm_s32_bit_exact(M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    a = _codes(rng, (M, K))
    b = _codes(rng, (N, K))
    out = Guarded((M, N), torch.int32)
    acc = cr.int8_gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.int8_gemm_acc(a, b))


@pytest.mark.parametrize("M,N,K", [(130, 272, 15360), (130, 144, 131072), (3, 144, 131072),
                                   (2, 144, 16384)])
def test_int8_gemm_s32_extremes(M, N, K):
    """Largest accumulators: |acc| = 127^2 K, at the workloads' K = 15360 and at
    the interface's limit K = 131072 (127^2 * 131072 < 2^31), on the three
    GEMM paths (CTA pairs for M > 128, swap-AB below, the dp4a product for one
    or two tokens with at most 64 KB of codes: M = 2, K = 16384)."""
    a = np.full((M, K), 127, np.int8)
    a[1::2] = -127
    a[min(5, M - 1), ::2] = 0
    b = np.full((N, K), 127, np.int8)
    b[3] = -127
    b[7, :100] = 0
    acc = cr.int8_gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
    ref = oracle.int8_gemm_acc(a, b)
    assert abs(int(ref[0, 0])) == 127 * 127 * K
    np.testing.assert_array_equal(acc.cpu().numpy(), ref)


def test_int8_gemm_deterministic():
    rng = np.random.default_rng(11)
    a = torch.from_numpy(_codes(rng, (777, 3072))).cuda()
    b = torch.from_numpy(_codes(rng, (1280, 3072))).cuda()
    s_tok = torch.rand(777, device="cuda") * 0.01
    s_w = torch.tensor([1e-3], device="cuda")
    bias = torch.randn(1280, device="cuda").to(torch.bfloat16)
    y1 = cr.int8_gemm(a, s_tok, b, s_w, bias)
    y2 = cr.int8_gemm(a, s_tok, b, s_w, bias)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


# ---------------------------------------------------------------------------
# int8 GEMM epilogue: rescale + bias -> bf16
# ---------------------------------------------------------------------------
def _assert_epilogue_close(y_gpu, acc, s_tok, s_w, bias):
    ref = oracle.epilogue(acc, s_tok, s_w, bias)  # s_w: per tensor or per output channel
    got = oracle.as_f64(y_gpu)
    mag = np.abs(acc.astype(np.float64) * s_tok.astype(np.float64)[:, None]
                 * np.abs(np.asarray(s_w, np.float64)).max())
    if bias is not None:
        mag = mag + np.abs(oracle.as_f64(bias))[None, :]
    tol = bf16_ulp(ref) + mag * 2.0 ** -21
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{bad.sum()} epilogue outputs off by more than 1 ulp"


@pytest.mark.parametrize("M,N,K,with_bias,per_channel", [
    (64, 1024, 1024, True, False), (129, 272, 144, False, False), (7, 144, 64, True, True),
    (257, 512, 256, True, True), (100, 1008, 2048, True, True),
    (3, 1040, 4096, True, False), (1, 2048, 3072, False, True), (8, 528, 8192, True, True),
    (2, 1040, 4096, True, True),
])
def test_int8_gemm_epilogue(M, N, K, with_bias, per_channel):
    rng = np.random.default_rng(M + N + K)
    a = _codes(rng, (M, K))
    b = _codes(rng, (N, K))
    s_tok = (rng.random(M) * 0.05).astype(np.float32)
    s_tok[0] = 0.0  # a zero token: output row = bias
    s_w = (rng.random(N) * 2e-3 + 1e-4).astype(np.float32) if per_channel else np.float32(1.3e-3)
    bias = workloads.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.5) if with_bias else None
    out = Guarded((M, N), torch.bfloat16)
    y = cr.int8_gemm(torch.from_numpy(a).cuda(), torch.from_numpy(s_tok).cuda(),
                     torch.from_numpy(b).cuda(), torch.from_numpy(np.atleast_1d(s_w)).cuda(),
                     bias.cuda() if bias is not None else None, out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    acc = oracle.int8_gemm_acc(a, b)
    _assert_epilogue_close(y.cpu(), acc, s_tok, s_w, bias)
    if with_bias:
        np.testing.assert_array_equal(oracle.as_f64(y[0].cpu()), oracle.as_f64(bias))


# ---------------------------------------------------------------------------
# activation rotate + quantize
# ---------------------------------------------------------------------------
RQA_CASES = [
    (G, kind, M, K)
    for G in (4, 16, 64, 256) for kind in ("sylvester", "qr")
    for (M, K) in ((1, 256), (7, 1024), (129, 3840))
] + [(256, "sylvester", 33, 15360), (256, "sylvester", 17, 32768), (64, "sylvester", 20, 12288),
     (256, "qr", 9, 10240), (16, "sylvester", 65, 5120), (256, "sylvester", 300, 2048),
     (256, "sylvester", 3001, 3840)]  # several persistent row-block passes, half-empty last block


@pytest.mark.parametrize("G,kind,M,K", RQA_CASES)
def test_rotate_quant_act_parity(G, kind, M, K):
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    assert rot.is_sylvester == (kind == "sylvester")
    x = workloads.make_activation(M, K, seed=G + M + K, n_outliers=4)
    x[min(2, M - 1)] = 0  # an all-zero token
    xq_buf = Guarded((M, K), torch.int8)
    s_buf = Guarded((M,), torch.float32)
    xq, s_tok = cr.rotate_quant_act(x.cuda(), rot, xq=xq_buf.tensor, s_tok=s_buf.tensor)
    torch.cuda.synchronize()
    xq_buf.check()
    s_buf.check()
    ref_q, ref_s = oracle.rotate_quant_act(x, R)
    np.testing.assert_allclose(s_tok.cpu().numpy(), ref_s, rtol=_scale_rtol(G, kind), atol=0)
    assert_codes_close(xq.cpu().numpy(), ref_q)
    assert float(s_tok[min(2, M - 1)]) == 0.0 and not xq[min(2, M - 1)].any()


@pytest.mark.parametrize("G", [16, 256])
def test_token_scale_is_the_correctly_rounded_quotient(G):
    """s_tok = RN_float32(max|x_rot| / 127), bit for bit.  Token i holds one
    nonzero element v_i, so its rotated row is +-v_i / sqrt(G) in one group
    and the absmax |v_i| / sqrt(G) is exact; the expected scale is the float32
    quotient, which numpy rounds once (float32 division is IEEE).  The v_i span
    normal scales and the tiny ones whose scale is a float32 subnormal."""
    rng = np.random.default_rng(77 + G)
    M, K = 4096, 512
    exps = np.concatenate([rng.uniform(-40.0, 60.0, M - 512), rng.uniform(-124.0, -112.0, 512)])
    v = (rng.uniform(1.0, 2.0, M) * np.exp2(exps) * rng.choice([-1.0, 1.0], M))
    v = torch.from_numpy(v).to(torch.bfloat16)
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    cols = torch.from_numpy(rng.integers(0, K, M))
    x[torch.arange(M), cols] = v
    rot = cr.Rotation(workloads.sylvester_rotation(G))
    _, s_tok = cr.rotate_quant_act(x.cuda(), rot)
    a = (np.abs(v.float().numpy()) * np.float32(1.0 / np.sqrt(G))).astype(np.float32)
    assert np.all(a > 0)
    expect = a / np.float32(127.0)
    assert np.any(expect < np.finfo(np.float32).tiny)  # subnormal scales are covered
    np.testing.assert_array_equal(s_tok.cpu().numpy().view(np.uint32), expect.view(np.uint32))


def test_rotate_quant_act_empty():
    rot = cr.Rotation(workloads.sylvester_rotation(256))
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    xq, s = cr.rotate_quant_act(x, rot)
    assert xq.shape == (0, 256) and s.shape == (0,)


def test_rotate_quant_act_rejects_bad_k():
    rot = cr.Rotation(workloads.sylvester_rotation(256))
    x = torch.zeros((4, 320), dtype=torch.bfloat16, device="cuda")  # 320 % 256 != 0
    with pytest.raises(cr.ConvRotError) as e:
        cr.rotate_quant_act(x, rot)
    assert e.value.status == cr.INVALID_ARG
    x = torch.zeros((4, 65536), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.rotate_quant_act(x, rot)
    assert e.value.status == cr.UNSUPPORTED


# ---------------------------------------------------------------------------
# weight quantization and dequant + derotate
# ---------------------------------------------------------------------------
WQ_CASES = [(G, kind, N, K) for G in (4, 16, 64, 256) for kind in ("sylvester", "qr")
            for (N, K) in ((16, 256), (136, 1024))] + [(256, "sylvester", 1000, 3840)]


@pytest.mark.parametrize("G,kind,N,K", WQ_CASES)
def test_quantize_weight_parity(G, kind, N, K):
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    W = workloads.make_weight(N, K, seed=N + K + G)
    Wq, s_w = cr.quantize_weight(W.cuda(), rot)
    ref_q, ref_s = oracle.quantize_weight(W, R)
    np.testing.assert_allclose(s_w.cpu().numpy()[0], ref_s, rtol=_scale_rtol(G, kind))
    assert_codes_close(Wq.cpu().numpy(), ref_q)


@pytest.mark.parametrize("G,kind,N,K", WQ_CASES + [(256, "sylvester", 12288 // 8, 3072),
                                                   (64, "sylvester", 4999, 3840)])
def test_dequant_derotate_parity(G, kind, N, K):
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    W = workloads.make_weight(N, K, seed=N * 3 + K + G)
    Wq, s_w = oracle.quantize_weight(W, R)
    out = Guarded((N, K), torch.bfloat16)
    W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(),
                                torch.tensor([s_w], dtype=torch.float32, device="cuda"), rot,
                                out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    ref = oracle.dequant_derotate(Wq, s_w, R)
    got = oracle.as_f64(W_hat.cpu())
    if kind == "sylvester":
        np.testing.assert_array_equal(bf16_bits(W_hat), oracle.bf16_bits(ref))
    else:
        assert np.all(np.abs(got - ref) <= bf16_ulp(ref)), "more than 1 bf16 ulp"
    # decode accuracy at the pages' group size; smaller groups spread the outlier
    # columns over fewer entries, so their per-tensor scale is coarser
    assert oracle.cosine(got, W) >= (0.9998 if G == 256 else 0.995)


@pytest.mark.parametrize("kind", ["sylvester", "qr"])
def test_dequant_derotate_per_channel_scale(kind):
    """A scale per output channel multiplies along the OUTPUT axis (PR #194
    fixed a broadcast that scaled the input axis: square weights decoded at corr
    0.82).  Non-square on purpose, so a wrong axis cannot pass silently."""
    N, K, G = 272, 512, 64
    R = _rotation(G, kind)
    rot = cr.Rotation(R)
    rng = np.random.default_rng(5)
    Wq = _codes(rng, (N, K))
    s = (rng.random(N) * 1e-3 + 1e-4).astype(np.float32)
    W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(), torch.from_numpy(s).cuda(), rot)
    ref = oracle.dequant_derotate(Wq, s, R)
    got = oracle.as_f64(W_hat.cpu())
    if kind == "sylvester":
        np.testing.assert_array_equal(got, ref)
    else:
        assert np.all(np.abs(got - ref) <= bf16_ulp(ref))


@pytest.mark.parametrize("G", [16, 256])
def test_dequant_derotate_short_mantissa_scales(G):
    """Scales with few significant bits make many products s_w * 2^-k * sum
    exact, some of them exactly halfway between two bf16 values, where only
    round-half-to-even is right.  The decode must still round each value once
    (bit-exact against the oracle), per tensor and per output channel, with
    long- and short-mantissa channel scales mixed."""
    N, K = 160, 1024
    R = workloads.sylvester_rotation(G)
    rot = cr.Rotation(R)
    rng = np.random.default_rng(G)
    Wq = _codes(rng, (N, K))
    for s_w in (2.0 ** -9, 0.375 * 2.0 ** -6, (65 / 128) * 2.0 ** -8):
        W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(),
                                    torch.tensor([s_w], dtype=torch.float32, device="cuda"), rot)
        ref = oracle.dequant_derotate(Wq, s_w, R)
        np.testing.assert_array_equal(bf16_bits(W_hat), oracle.bf16_bits(ref))
    s = (rng.random(N) * 1e-3 + 1e-4).astype(np.float32)
    s[::3] = 2.0 ** -10
    s[1::7] = 0.75 * 2.0 ** -9
    W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(), torch.from_numpy(s).cuda(), rot)
    ref = oracle.dequant_derotate(Wq, s, R)
    np.testing.assert_array_equal(oracle.as_f64(W_hat.cpu()), ref)


# ---------------------------------------------------------------------------
# the whole int8-compute layer
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["sylvester", "qr"])
@pytest.mark.parametrize("M", [64, 1, 130])
def test_linear_int8_single_1024(kind, M):
    lin = workloads.WORKLOADS["single_1024"][0]
    inp = workloads.make_layer_inputs(lin, 0, rotation=kind, M=M)
    Wq, s_w = oracle.quantize_weight(inp.W, inp.R)
    rot = cr.Rotation(inp.R)
    out = Guarded((M, lin.N), torch.bfloat16)
    y = cr.linear_int8(inp.x.cuda(), torch.from_numpy(Wq).cuda(),
                       torch.tensor([s_w], device="cuda"), rot, inp.bias.cuda(), out=out.tensor)
    torch.cuda.synchronize()
    out.check()
    y_ref, *_ = oracle.linear_int8(inp.x, Wq, s_w, inp.R, inp.bias)
    assert oracle.rel_l2(y.cpu(), y_ref) <= 2e-3
    assert oracle.cosine(y.cpu(), oracle.linear_dense(inp.x, inp.W, inp.bias)) >= 0.999


def test_linear_int8_workspace_errors():
    rot = cr.Rotation(workloads.sylvester_rotation(256))
    x = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((32, 256), dtype=torch.int8, device="cuda")
    s_w = torch.ones(1, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.linear_int8(x, Wq, s_w, rot, workspace=small)
    assert e.value.status == cr.WORKSPACE


def test_layer_module_two_modes_agree():
    """int8-compute against the default path (decode + dense bf16 matmul)."""
    lin = workloads.WORKLOADS["single_1024"][0]
    inp = workloads.make_layer_inputs(lin, 0)
    layer = cr.ConvRotLinear(inp.W.cuda(), inp.R, inp.bias.cuda())
    y_int8 = layer(inp.x.cuda())
    y_dec = torch.nn.functional.linear(inp.x.cuda().float(), layer.decode_weight().float(),
                                       inp.bias.cuda().float())
    assert oracle.cosine(y_int8.cpu(), y_dec.cpu()) >= 0.999


def test_check_status_clean():
    cr.check_status()


# ---------------------------------------------------------------------------
# CUDA graphs: the int8-compute forward captured once and replayed
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M", [64, 300])
def test_linear_int8_cuda_graph_replay(M):
    """convrot_linear_int8 (rotate+quantize, chained GEMM) captured in a CUDA
    graph and replayed on new inputs written into the captured buffers gives the
    eager results bit for bit."""
    lin = workloads.Linear("graph", M, 1024, 2048, G=256)
    inp = workloads.make_layer_inputs(lin, 3)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    bias = inp.bias.cuda()
    x = inp.x.cuda()
    ws = torch.empty(cr.workspace_bytes(M, lin.N, lin.K), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, lin.N), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up off the capture stream, as torch asks
        cr.linear_int8(x, Wq, s_w, rot, bias, out=y, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cr.linear_int8(x, Wq, s_w, rot, bias, out=y, workspace=ws)
    for seed in (11, 12):
        x_new = workloads.make_activation(M, lin.K, seed=seed).cuda()
        x.copy_(x_new)
        graph.replay()
        torch.cuda.synchronize()
        y_eager = cr.linear_int8(x_new, Wq, s_w, rot, bias)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
    cr.check_status()


# ---------------------------------------------------------------------------
# failure detection: a bounded wait that runs out is reported, nothing hangs
# ---------------------------------------------------------------------------
def test_bounded_wait_timeout_is_reported():
    cr.check_status()  # clean to start with
    cr.selftest_wait_timeout(20)
    with pytest.raises(cr.ConvRotError) as e:
        cr.check_status()
    assert e.value.status == cr.TIMEOUT
    cr.check_status()  # reading the status cleared it
    with pytest.raises(cr.ConvRotError) as e:
        cr.selftest_wait_timeout(0)
    assert e.value.status == cr.INVALID_ARG
    # the context still computes: a small GEMM, bit-exact
    rng = np.random.default_rng(99)
    a, b = _codes(rng, (65, 256)), _codes(rng, (144, 256))
    acc = cr.int8_gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.int8_gemm_acc(a, b))
    cr.check_status()


# ---------------------------------------------------------------------------
# workspace slicing: a smaller workspace processes the tokens in row slices
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_linear_int8_sliced_workspace(dtype):
    """Slices of at most 2N tokens (the Int8 Compute page's memory bound), of
    100 tokens, and of a single token give the one-pass result bit for bit."""
    M, K, N = 700, 1024, 256
    lin = workloads.Linear("sliced", M, K, N, G=256)
    inp = workloads.make_layer_inputs(lin, 5, dtype=dtype)
    rot = cr.Rotation(inp.R)
    Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
    x, bias = inp.x.cuda(), inp.bias.cuda()
    full = cr.workspace_bytes(M, N, K)
    y_ref = cr.linear_int8(x, Wq, s_w, rot, bias, workspace=torch.empty(full, dtype=torch.uint8, device="cuda"))
    sliced = cr.workspace_bytes(M, N, K, sliced=True)
    assert sliced < full
    one_row = cr.workspace_bytes(1, N, K)
    for nbytes in (sliced, cr.workspace_bytes(100, N, K), one_row):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        y = cr.linear_int8(x, Wq, s_w, rot, bias, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), nbytes
    with pytest.raises(cr.ConvRotError) as e:
        cr.linear_int8(x, Wq, s_w, rot, bias,
                       workspace=torch.empty(one_row - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == cr.WORKSPACE


def test_int8_mma_issue_rate():
    """The benchmark's probe of the tensor cores' own int8 rate (its own
    library): positive, below the part's clock peak (148 SMs x 8192 MAC/clk x
    2 at 1.965 GHz = 4.77 POPS) and above the bf16 GEMM rate."""
    import bench
    tops = bench.Int8RateProbe().measure_int8_mma_rate(8192)
    assert 1650.0 < tops < 4800.0, tops
