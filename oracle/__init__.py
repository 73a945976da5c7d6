"""Float64 CPU oracle for the MoDA attention path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
and reference arm may import this package. It shares no code with the CUDA
path and imports nothing from it.
"""
from .moda_oracle import backward, depth_write, forward, forward_rows, to_f64  # noqa: F401
