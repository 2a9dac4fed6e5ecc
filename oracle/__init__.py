"""CPU oracle for the quantized attention prefill path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
library under ``quantized_exact_attention_qattn_b200`` and never imports it.
"""
from . import encoders, qattn_oracle  # noqa: F401
