"""CPU oracle of the ConvRot int8 linear layer (test infrastructure only).

Only the tests, the package smoke check and the bench's CPU-baseline leg may
import this package; the CUDA library never does.
"""

from .convrot_oracle import (  # noqa: F401
    INT8_QMAX,
    as_f64,
    bf16_bits,
    bf16_round,
    block_rotate,
    cosine,
    dequant_derotate,
    epilogue,
    f16_bits,
    f16_round,
    int8_gemm_acc,
    linear_dense,
    linear_dequant,
    linear_int8,
    quantize_symmetric,
    quantize_weight,
    rel_l2,
    rotate_quant_act,
    round16,
    weight_scale_column,
)
