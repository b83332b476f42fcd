"""Float64 CPU oracle of the KDA recurrence (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it.
"""
from .kda_erase import erase_chunked, erase_forward
from .kda_oracle import expand_heads, kda_backward, kda_decode_step, kda_forward
from .kda_prep import (L2_EPS, conv_update, kda_decode_token, kda_forward_prepared, kda_gate, l2norm_rows,
                       output_gate, short_conv_qkv, short_conv_silu, sigmoid, softplus)

__all__ = ["expand_heads", "kda_backward", "kda_decode_step", "kda_forward", "L2_EPS", "conv_update",
           "kda_decode_token", "kda_forward_prepared", "kda_gate", "l2norm_rows", "output_gate", "short_conv_qkv",
           "short_conv_silu", "sigmoid", "softplus", "erase_forward", "erase_chunked"]
