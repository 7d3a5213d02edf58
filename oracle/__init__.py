"""CPU oracle for the batched single-token decoder step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls, links or
executes anything in this package: only the tests, the smoke check and the
benchmark's CPU-baseline leg do. It shares no code with the CUDA library.

Precision policy: the decoders on the pages keep every tensor in f32. The
oracle stores f32 at the same points (projection outputs, norm outputs,
attention outputs, residual stream, KV cache, logits) and forms each
reduction in f64, so its only rounding is the rounding to f32 storage.
Where f32 arithmetic decides an integer (the ties-to-even activation
quantiser, the greedy argmax) it works in f32 as the pages do.

Parity status of each function is stated in its docstring; all are pinned by
tests in tests/test_oracle_*.py against closed forms, library routines,
invariants or brute force. No function is "parity unpinned".
"""
from .decoder import (  # noqa: F401
    layer_norm, rms_norm, quantize_rows_i8_te, dequantize_rows_i8, quantize_weight_rows,
    int8_dot_acc, linear_f32, linear_w8a8, linear_w8a32, rope_cos_sin, apply_rope_neox,
    softmax_weights, attention_decode, gelu_tanh, silu, argmax_first, OracleDecoder,
)
