"""Float64 CPU oracle for the MoDA attention path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
and reference arm may import this package. It shares no code with the CUDA
path and imports nothing from it.
"""
from .moda_oracle import (backward, depth_write, depth_write_q8, dequantize_q8, forward,  # noqa: F401
                          forward_rows, quantize_q8, round_to_bf16, to_f64)
