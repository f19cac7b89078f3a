"""Full-size parity on the synthetic workloads, in the launch configuration the
bench times (rotate_quant_act, then int8_gemm, on the whole batch).

The CPU oracle cannot run a whole 4608 x 11520 x 3840 layer in seconds, so:
  * the weight quantizer is checked in full (scale and every code);
  * the activation codes and scales are checked in full (every token);
  * the layer output is checked on seeded sampled token rows (first, last, the
    tail of the last 128-row block, and random rows), every column;
  * the int32 accumulators of the GEMM at the workloads' sizes are checked
    bit-exact on sampled rows, every column, from random full-range codes;
  * properties that hold at any size are checked on every row.

Tolerances are those of test_gpu_kernels.py.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu_helpers import assert_codes_close, bf16_bits, bf16_ulp, sample_rows

pytestmark = pytest.mark.gpu

BIG = [(w, i) for w in ("zimage_dit_block", "flux1_dev_blocks", "wan22_a14b_video_dit")
       for i in range(len(workloads.WORKLOADS[w]))]


@pytest.fixture(scope="module")
def cr():
    import activation_quantized_linear_b200 as mod
    torch.cuda.set_device(0)
    return mod


def _epilogue_tolerance(y_gpu, acc, s_tok, s_w, bias):
    ref = oracle.epilogue(acc, s_tok, s_w, bias)
    got = oracle.as_f64(y_gpu)
    mag = (np.abs(acc.astype(np.float64)) * s_tok.astype(np.float64)[:, None] * np.float64(s_w)
           + np.abs(oracle.as_f64(bias))[None, :])
    return got, ref, bf16_ulp(ref) + mag * 2.0 ** -21


def _check_linear(cr, lin, index, R, name):
    inp = workloads.make_layer_inputs(lin, index)
    rot = cr.Rotation(R)
    # ---- weight: full check
    Wq_g, s_w_g = cr.quantize_weight(inp.W.cuda(), rot)
    Wq_ref, s_w_ref = oracle.quantize_weight(inp.W, R)
    s_w = float(s_w_g.item())
    assert abs(s_w - float(s_w_ref)) <= 1e-6 * float(s_w_ref), name
    Wq = Wq_g.cpu().numpy()
    assert_codes_close(Wq, Wq_ref)
    # ---- the bench's two launches on the whole batch
    x = inp.x.cuda()
    xq_g, s_tok_g = cr.rotate_quant_act(x, rot)
    y_g = cr.int8_gemm(xq_g, s_tok_g, Wq_g, s_w_g, inp.bias.cuda())
    torch.cuda.synchronize()
    cr.check_status()
    xq = xq_g.cpu().numpy()
    s_tok = s_tok_g.cpu().numpy()
    # properties on every token: codes in range, the largest |code| of a token is 127
    assert xq.min() >= -127 and xq.max() <= 127
    amax = np.abs(xq.astype(np.int32)).max(axis=1)
    assert np.all((amax == 127) | (s_tok == 0)), name
    # every token's codes and scale against the oracle (full tensors)
    xq_all, s_all = oracle.rotate_quant_act(inp.x, R)
    np.testing.assert_allclose(s_tok, s_all, rtol=1e-6)
    assert_codes_close(xq, xq_all)
    del xq_all, s_all
    rows = sample_rows(lin.M, 256, seed=index)
    x_s = inp.x[rows]
    # GEMM + epilogue: the oracle's accumulators from the GPU's codes (bit-exact
    # by construction of the int8 product), then the epilogue within 1 ulp
    acc = oracle.int8_gemm_acc(xq[rows], Wq)
    y_rows = y_g[torch.from_numpy(rows).cuda()].cpu()
    got, ref, tol = _epilogue_tolerance(y_rows, acc, s_tok[rows], s_w, inp.bias)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{name}: {bad.sum()} outputs off by more than 1 ulp"
    # the whole int8 layer from the oracle's own codes, and the unquantized layer:
    # cosine >= 0.999 at the pages' group size, G = 256; smaller groups spread
    # the outlier channels less, so there the GPU must match the method's own
    # accuracy (the oracle's cosine, less 1e-4)
    y_ref, *_ = oracle.linear_int8(x_s, Wq_ref, s_w_ref, R, inp.bias)
    assert oracle.rel_l2(y_rows, y_ref) <= 2e-3, name
    y_dense = oracle.linear_dense(x_s, inp.W, inp.bias)
    bar = 0.999 if lin.G == 256 else min(0.999, oracle.cosine(y_ref, y_dense) - 1e-4)
    assert oracle.cosine(y_rows, y_dense) >= bar, name
    return inp, rot, Wq_g, s_w_g, y_g, rows


@pytest.mark.parametrize("workload,idx", BIG, ids=[f"{w}-{workloads.WORKLOADS[w][i].name}" for w, i in BIG])
def test_full_size_linear(cr, workload, idx):
    lin = workloads.WORKLOADS[workload][idx]
    windex = list(workloads.WORKLOADS).index(workload)
    R = workloads.sylvester_rotation(lin.G)
    inp, rot, Wq_g, s_w_g, y_g, rows = _check_linear(cr, lin, windex, R, f"{workload}/{lin.name}")
    if workload == "wan22_a14b_video_dit":
        # the default path on the same weight: decode to bf16 (bit-exact), and
        # the two paths' outputs agree on the sampled tokens
        W_hat = cr.dequant_derotate(Wq_g, s_w_g, rot)
        ref = oracle.dequant_derotate(Wq_g.cpu().numpy(), float(s_w_g.item()), inp.R)
        w_rows = sample_rows(lin.N, 128, seed=idx + 7)
        np.testing.assert_array_equal(bf16_bits(W_hat[torch.from_numpy(w_rows).cuda()]),
                                      oracle.bf16_bits(ref[w_rows]))
        y_dec = oracle.linear_dense(inp.x[rows], oracle.as_f64(W_hat.cpu()), inp.bias)
        y_int = oracle.as_f64(y_g[torch.from_numpy(rows).cuda()].cpu())
        assert oracle.cosine(y_int, y_dec) >= 0.999


SWEEP = [(g, m) for g in workloads.GROUP_SIZES for m in (1, 16, 128, 1024, 8192)]


@pytest.mark.parametrize("G,M", SWEEP, ids=[f"G{g}-M{m}" for g, m in SWEEP])
def test_group_size_and_skinny_sweep(cr, G, M):
    lin = workloads.Linear(f"k4096_m{M}_g{G}", M, 4096, 4096, G=G)
    _check_linear(cr, lin, 4, workloads.sylvester_rotation(G), lin.name)


@pytest.mark.parametrize("G", workloads.GROUP_SIZES)
def test_decode_12288x3072(cr, G):
    N, K = workloads.DEROTATE_SWEEP_SHAPE
    R = workloads.sylvester_rotation(G)
    rot = cr.Rotation(R)
    W = workloads.make_weight(N, K, seed=4000 + G)
    Wq, s_w = oracle.quantize_weight(W, R)
    W_hat = cr.dequant_derotate(torch.from_numpy(Wq).cuda(), torch.tensor([s_w], device="cuda"), rot)
    rows = sample_rows(N, 512, seed=G)
    ref = oracle.dequant_derotate(Wq[rows], s_w, R)
    np.testing.assert_array_equal(bf16_bits(W_hat[torch.from_numpy(rows).cuda()]), oracle.bf16_bits(ref))
    assert oracle.cosine(W_hat.cpu(), W) >= (0.9998 if G == 256 else 0.995)


# int32 accumulators at the workloads' sizes.  Each shape reaches a different
# part of the CTA-pair GEMM's schedule: the Z-Image QKV (36 x 45 tiles, several
# persistent passes per pair, s32 output wider than 1024 columns), the Wan
# down-projection (M*K > 64 MB: the grouped tile raster), K = N = 4096 at
# M = 8192 (512 tiles: many waves of the double-buffered TMEM accumulators),
# K = N = 4096 at M = 1024 (64 tiles on the 74 CTA pairs: one wave).
S32_FULL = [("zimage_qkv", 4608, 11520, 3840), ("wan_down", 7800, 5120, 13824),
            ("k4096_m8192", 8192, 4096, 4096), ("flux_in_proj", 4608, 21504, 3072),
            ("k4096_m1024_one_wave", 1024, 4096, 4096)]


@pytest.mark.parametrize("name,M,N,K", S32_FULL, ids=[c[0] for c in S32_FULL])
def test_full_size_int32_bit_exact(cr, name, M, N, K):
    rng = np.random.default_rng(M + N + K)
    a = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    b = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    acc = cr.int8_gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
    torch.cuda.synchronize()
    cr.check_status()
    rows = sample_rows(M, 256, seed=K)
    got = acc[torch.from_numpy(rows).cuda()].cpu().numpy()
    np.testing.assert_array_equal(got, oracle.int8_gemm_acc(a[rows], b))
