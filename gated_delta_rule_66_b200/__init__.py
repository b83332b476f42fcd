"""KDA recurrence on B200 (sm_100a): a C-ABI CUDA library and a thin binding.

``fwd``, ``decode_step``, ``bwd`` and ``workspace_bytes`` are loaded lazily
from the compiled library on first use; importing the package alone (for
example to reach :mod:`.inputs`) does not require a GPU.
"""

_EXPORTS = ("fwd", "decode_step", "bwd", "workspace_bytes", "KdaError", "library")


def __getattr__(name):
    if name in _EXPORTS:
        from . import kda
        return getattr(kda, name)
    raise AttributeError(name)
