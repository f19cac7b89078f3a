"""CPU oracle of the ConvRot int8_tensorwise linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the tests, the package smoke check and the CPU-baseline leg of the bench
call it.  It shares no code with the CUDA library.

Plain numpy, float64 throughout, written for reading rather than speed.  Each
function states the passage it follows.  The sources are five web pages on the
scheme:

* [PR194]  "feat(quantization): share the int8_convrot scheme and read it for
           Krea-2 and Z-Image" (InvokeAI-7 pull request #194);
* [PR10185] "feat(wan): load ComfyUI int8 convrot checkpoints" (InvokeAI pull
           request #10185);
* [INT8C]  Invoke documentation, "int8 Compute";
* [CTQ]    "Quantizing AI Models with convert_to_quant (Windows + NVIDIA)";
* [SNOVA]  ComfyUI Wiki, "SenseNova-U1.5 ConvRot for ComfyUI".

Notation: x [M, K] activations, W [N, K] weight (out x in), G the group size,
R [G, G] the orthogonal rotation block, B_R = blockdiag(R, ..., R) with K/G
blocks along the input dimension.

Readings where the pages leave a step open (each is a choice, stated once):

* direction: the weight is stored rotated as W_rot = W . B_R and decoded with
  B_R^T; activations are rotated with the same B_R, so x_rot . W_rot^T = x . W^T.
  [PR194] "Summary" only fixes the shape of the decode, a product
  [out, in/G, G] @ [G, G]; with a symmetric (Hadamard) R the direction is moot.
* scale: one float32 scale per tensor for the weight ([CTQ] "How INT8 ConvRot
  Quantization Works", `--scaling_mode tensor`) and one per token for the
  activation ([INT8C], opening section), both absmax / 127, symmetric codes
  in [-127, 127] (never -128).
* per-output-channel weight scale: a weight may instead carry one float32
  scale per output channel, s_w[n] = max_k |W_rot[n, k]| / 127 ([PR194]
  "Summary", Z-Image's fused QKV, whose per-output-channel scale splits with
  its weight; "QA Instructions", int8 carries one scale per output channel).
  It multiplies along the OUTPUT axis: row n of the decoded weight and column
  n of the layer output.  [PR194]'s scale-layout fix names the mistake this
  excludes: a length-N scale left to trailing-axis broadcasting scales the
  input axis (wrong values for square weights, a size error for the rest).
  A scale array of any length other than 1 or N is refused.
* rounding: round half to even, no learned/SVD rounding ([CTQ] `--simple`).
* the code decision round(v / s) is taken in float32, the CUDA kernels'
  precision, since the pages fix none: v and s are first rounded to float32,
  then divided with IEEE float32 division, then rounded half to even.
* a token whose rotated row is all zero gets s_tok = 0 and all-zero codes, so
  its output row is the bias.
* epilogue: y = bf16_rn(acc * s_tok * s_w + bias), evaluated in float64 and
  rounded once to bf16.
* 16-bit formats: the layer runs with BF16 or FP16 activations ([INT8C],
  opening section and the "Running in FP32" row of its table); in fp16 the
  inputs are read exactly and every output (decoded weight, layer output) is
  rounded once to fp16 instead of bf16.
"""

from __future__ import annotations

import numpy as np

INT8_QMAX = 127


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def as_f64(a) -> np.ndarray:
    """Any array-like (numpy, or a CPU torch tensor of any float dtype) -> float64."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").float().numpy()
    return np.asarray(a, dtype=np.float64)


def bf16_round(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as
    float64.  A single rounding, straight from float64: 8 significant bits,
    exponent floor of the bf16 normal range (2^-126) for subnormals.  Values
    beyond the bf16 range are not produced by this layer and are not handled.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)                    # v = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)               # bf16 normal floor: 2^-126 = 0.5 * 2^-125
    ulp = np.ldexp(1.0, e - 8)            # spacing of 8-significant-bit numbers
    return np.rint(v / ulp) * ulp         # np.rint rounds half to even; exact in fp64


def f16_round(v) -> np.ndarray:
    """Round float64 values to the nearest IEEE fp16 (ties to even), returned as
    float64.  A single rounding, straight from float64: 11 significant bits,
    exponent floor of the fp16 normal range (2^-14), so subnormals are
    multiples of 2^-24; magnitudes that round above 65504 become infinite.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)                    # v = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -13)                # fp16 normal floor: 2^-14 = 0.5 * 2^-13
    ulp = np.ldexp(1.0, e - 11)           # spacing of 11-significant-bit numbers
    r = np.rint(v / ulp) * ulp
    return np.where(np.abs(r) > 65504.0, np.copysign(np.inf, v), r)


def round16(v, fmt: str) -> np.ndarray:
    """The 16-bit output rounding of the layer: "bf16" or "f16"."""
    if fmt == "bf16":
        return bf16_round(v)
    if fmt == "f16":
        return f16_round(v)
    raise ValueError(fmt)


def f16_bits(v) -> np.ndarray:
    """fp16-representable float64 values -> their uint16 bit patterns."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits(v) -> np.ndarray:
    """bf16-representable float64 values -> their uint16 bit patterns."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def block_rotate(A, R) -> np.ndarray:
    """A . B_R: every contiguous group of G entries along the last (input)
    dimension is multiplied on the right by R.

    [PR194] "Summary": the rotation is block-diagonal along the input
    dimension; the decode is the product [out, in/G, G] @ [G, G].
    """
    A = as_f64(A)
    R = as_f64(R)
    G = R.shape[0]
    rows, K = A.shape
    if K % G:
        raise ValueError("K must be a multiple of G")
    return (A.reshape(rows, K // G, G) @ R).reshape(rows, K)


def quantize_symmetric(v, scale) -> np.ndarray:
    """Codes clamp(round_half_even(v / scale), -127, 127) as int8, the decision
    taken in float32; a zero scale gives zero codes.

    [CTQ] "How INT8 ConvRot Quantization Works" (`--int8`, `--simple`);
    [INT8C] opening section ("quantizes its input to int8").
    """
    v32 = np.asarray(v, dtype=np.float64).astype(np.float32)
    s32 = np.broadcast_to(np.asarray(scale, dtype=np.float32), v32.shape)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(v32 / s32)
    q = np.where(s32 == 0, 0.0, q)
    return np.clip(q, -INT8_QMAX, INT8_QMAX).astype(np.int8)


# ---------------------------------------------------------------------------
# the layer's operations
# ---------------------------------------------------------------------------

def weight_scale_column(s_w, N) -> np.ndarray:
    """The weight scale laid along the output axis, as float64 [N, 1]: a scalar
    (or a length-1 array) is one scale per tensor, a length-N array one scale
    per output channel (row n of the weight).  Any other length is refused,
    not broadcast.

    [PR194] "Summary" (per-output-channel scales split with their weight) and
    its scale-layout fix (a `[out]` scale must not scale the input axis).
    """
    s = np.asarray(s_w, dtype=np.float32).reshape(-1)
    if s.size == 1:
        return np.full((N, 1), np.float64(s[0]))
    if s.size != N:
        raise ValueError(f"weight scale of length {s.size} for {N} output channels")
    return s.astype(np.float64)[:, None]


def quantize_weight(W, R, per_channel: bool = False):
    """Offline weight quantization: rotate W in G-blocks along its input
    dimension, take the scale absmax / 127 over the whole tensor (or, with
    per_channel, over each output channel's row), round to int8.

    [CTQ] "How INT8 ConvRot Quantization Works": `--int8 --scaling_mode tensor
    --simple --convrot --convrot-group-size G` ("one global scale per tensor");
    [PR194] "Summary" and "QA Instructions" for the per-output-channel form.
    Returns (Wq int8 [N, K], s_w float32 scalar, or float32 [N] per channel).
    """
    W_rot = block_rotate(W, R)
    if per_channel:
        a = np.max(np.abs(W_rot), axis=1) if W_rot.shape[1] else np.zeros(W_rot.shape[0])
        s_w = (a / INT8_QMAX).astype(np.float32)
        return quantize_symmetric(W_rot, s_w[:, None]), s_w
    a = np.max(np.abs(W_rot)) if W_rot.size else 0.0
    s_w = np.float32(a / INT8_QMAX)
    return quantize_symmetric(W_rot, s_w), s_w


def dequant_derotate(Wq, s_w, R, fmt: str = "bf16") -> np.ndarray:
    """Default (weight-decode) path: W_hat[n] = bf16(s_w[n] * Wq[n] . B_R^T)
    (fp16 with fmt="f16"); s_w is one scale per tensor or per output channel.

    [PR194] "Summary": each quantized layer "dequantizes and derotates per
    forward"; the derotation is the product [out, in/G, G] @ [G, G].
    Returns the 16-bit values as float64 [N, K].
    """
    R = as_f64(R)
    Wq = np.asarray(Wq, np.float64)
    return round16(weight_scale_column(s_w, Wq.shape[0]) * block_rotate(Wq, R.T), fmt)


def rotate_quant_act(x, R):
    """int8_compute, step 1: rotate each token by the same R, then quantize it to
    int8 with one scale per token, s_tok = max_k |x_rot[m, k]| / 127.

    [INT8C] opening section: each layer "rotates and quantizes its input to
    int8 per token"; the "Layer / Why" table gives the reason (one outlier
    channel would otherwise set the scale of the whole token).
    Returns (xq int8 [M, K], s_tok float32 [M]).
    """
    x_rot = block_rotate(x, R)
    a = np.max(np.abs(x_rot), axis=1) if x_rot.shape[1] else np.zeros(x_rot.shape[0])
    s_tok = (a / INT8_QMAX).astype(np.float32)
    return quantize_symmetric(x_rot, s_tok[:, None]), s_tok


def int8_gemm_acc(xq, Wq) -> np.ndarray:
    """int8_compute, step 2: acc[m, n] = sum_k xq[m, k] * Wq[n, k] in int32.

    [INT8C] opening section ("multiplies int8 by int8" on the int8 tensor
    cores).  Evaluated as a float64 matrix product: every operand and every
    partial sum is an integer of magnitude <= 127^2 * K < 2^53, so each float64
    addition is exact and the result does not depend on summation order.
    """
    a = np.asarray(xq, dtype=np.int64)
    b = np.asarray(Wq, dtype=np.int64)
    K = a.shape[1]
    if INT8_QMAX * INT8_QMAX * K >= 2 ** 53:
        raise ValueError("K too large for an exact float64 product")
    acc = a.astype(np.float64) @ b.astype(np.float64).T
    if acc.size and np.max(np.abs(acc)) >= 2 ** 31:
        raise OverflowError("accumulator exceeds int32")
    return acc.astype(np.int64).astype(np.int32)


def epilogue(acc, s_tok, s_w, bias=None, fmt: str = "bf16") -> np.ndarray:
    """int8_compute, step 3: y = bf16(acc * s_tok[m] * s_w[n] + bias[n]) (fp16
    with fmt="f16"); s_w is one scale per tensor or per output channel n.

    [INT8C] opening section and "Layer / Why" table (outputs are BF16/FP16);
    the bias is the nn.Linear bias the layer replaces ([PR194] "Summary").
    Returns the 16-bit values as float64 [M, N].
    """
    acc = np.asarray(acc, np.float64)
    y = (acc
         * np.asarray(s_tok, np.float32).astype(np.float64)[:, None]
         * weight_scale_column(s_w, acc.shape[1]).T)
    if bias is not None:
        y = y + as_f64(bias)[None, :]
    return round16(y, fmt)


def linear_int8(x, Wq, s_w, R, bias=None, fmt: str = "bf16"):
    """The whole int8_compute forward: rotate+quantize, int8 GEMM, epilogue.

    [INT8C] opening section.  Returns (y, xq, s_tok, acc).
    """
    xq, s_tok = rotate_quant_act(x, R)
    acc = int8_gemm_acc(xq, Wq)
    return epilogue(acc, s_tok, s_w, bias, fmt), xq, s_tok, acc


def linear_dequant(x, Wq, s_w, R, bias=None, fmt: str = "bf16") -> np.ndarray:
    """The default path of a ConvRot layer: decode the weight to the 16-bit
    format, then y = f16(x . W_hat^T + b), the exact sum rounded once.

    [INT8C] opening section (a layer that does not compute in int8 unpacks its
    weight to BF16 or FP16 and multiplies in that precision) and "When
    something goes wrong" (the default path is what the first int8 result is
    checked against).  The sum is taken in float64; the pages fix no
    summation precision for the matmul.  Returns float64 [M, N].
    """
    W_hat = dequant_derotate(Wq, s_w, R, fmt)
    return round16(linear_dense(x, W_hat, bias), fmt)


def linear_dense(x, W, bias=None) -> np.ndarray:
    """Unquantized reference layer y = x . W^T + b in float64 (no rounding)."""
    y = as_f64(x) @ as_f64(W).T
    if bias is not None:
        y = y + as_f64(bias)[None, :]
    return y


# ---------------------------------------------------------------------------
# metrics used by the acceptance checks
# ---------------------------------------------------------------------------

def cosine(a, b) -> float:
    a = as_f64(a).ravel()
    b = as_f64(b).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def rel_l2(a, ref) -> float:
    a = as_f64(a).ravel()
    ref = as_f64(ref).ravel()
    return float(np.linalg.norm(a - ref) / np.linalg.norm(ref))
