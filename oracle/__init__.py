"""CPU oracle for the RMA attention hot path (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The CUDA library never calls it.
"""
from .rma_oracle import *  # noqa: F401,F403
from .rma_oracle import (Config, State, new_state, state_from_arrays, copy_state, decode_step, admit,
                         prefill_block, bf16_to_f64, f64_to_bf16, f32_to_bf16,
                         attention_kv_bytes_per_sequence, full_attention_kv_bytes_per_token,
                         STATUS_PENDING_OVERFLOW, STATUS_NAN_SCORE, STATUS_PREFILL_PENDING_OVERFLOW, admit_plan)
from .rma_oracle_fp8 import (Fp8State, e4m3_to_f64, f32_to_e4m3, row_exponent, quantize_rows, dequantize_rows,
                             quantize_state, fp8_state_from_arrays, decode_step_fp8, admit_fp8)
