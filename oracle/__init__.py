"""CPU oracle for the STQ1_0 matmul -- test infrastructure, never part of the product path.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.
"""

from .stq1 import *  # noqa: F401,F403
from .stq1 import (  # noqa: F401
    BLOCK_BYTES, BLOCK_WEIGHTS, GROUP, GROUPS_PER_BLOCK, FLAG_WEIGHT_UP,
    OracleValueError, codebook, pattern_of_code, code_of, code_parts,
    fp16_bits, fp16_value, bf16_bits_rne, bf16_to_f64,
    pack_blocks, unpack_blocks, packed_size,
    encode_plain, encode_sherry, wls_scale, zero_lane_choice, weighted_error,
    decode, dequant_bf16, gemv, gemv_abs, tolerance, route_pairs, moe_gateup,
    half_from_struct, E4M3_MAX, e4m3_value, e4m3_round, quantize_x_e4m3, moe_gateup_fp8,
    bf16_bits_from_f64, silu, swiglu_bf16, moe_combine, moe_ffn,
    STQ2_BLOCK_BYTES, encode_stq2, decode_stq2, stq2_codes, stq2_wls_scale, stq2_weighted_error,
    hessian_error, diagonal_error, greedy_allocate,
)
