"""CPU float64 oracle for the rotation + INT4 W4A4 hot path.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference leg may import this package.  The product path (the CUDA library
and its Python binding) never imports it and fails loudly when its extension is missing.

Pinned: every function here is checked in ``tests/test_oracle_pins.py`` against closed
forms, invariants, textbook constructions, published generator vectors and brute force.
Parity unpinned: the particular pair lists that the greedy selection returns (any list that
satisfies the algorithm's stated properties is acceptable; the properties themselves are
pinned, and the CUDA-side host selection must match this one exactly).
"""
from .oracle import *  # noqa: F401,F403
from .oracle import (NONE, Plan, SplitMix64, TQResult, GemmResult, Quantized,  # noqa: F401
                     activation_transform, weight_transform, transform_quant, pack_weights,
                     gemm, group_dots, quantize, pack_nibbles, unpack_nibbles, select_pairs,
                     select_pairs_group, hadamard_matrix, fwht, hadamard_rotate,
                     hadamard_rotate_explicit, givens_rotate, givens_matrix, smooth_scales,
                     apply_smoothing, bf16_to_f64, bf16_round, RRSPrep, rrs_prepare,
                     rrs_transform_quant, rrs_pack_weights, rrs_gemm, LEVELS8, quantize_mixed,
                     transform_quant_mixed, pack_weights_mixed, gemm_mixed)
