"""Float64 CPU oracle of the KDA recurrence (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it.
"""
from .kda_oracle import expand_heads, kda_backward, kda_decode_step, kda_forward

__all__ = ["expand_heads", "kda_backward", "kda_decode_step", "kda_forward"]
