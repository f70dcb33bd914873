"""CPU oracle for the H-BitLinear forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package. It shares no code with
``hadamard_bit_quant_b200`` and never imports it.
"""
from .hbl_oracle import *  # noqa: F401,F403
from .hbl_oracle import (EPS, SQRT7, INT4_RANGE, INT8_RANGE, TERN_RANGE, TIE_WINDOW,  # noqa: F401
                         round_clip, exact_sum_rounded, weight_scale, ternarize, weight_quant,
                         hadamard_matrix, hadamard, quantize_int8, quantize_int4, quantize_act,
                         gemm_int, to_bf16, dequant, forward, forward_rows, RMS_EPS, rmsnorm, forward_ln,
                         rotate_weights, rotated_weight_quant, hadamard_backward, quantize_qkv,
                         dequantize_qkv)
