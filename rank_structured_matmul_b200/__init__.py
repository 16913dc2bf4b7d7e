"""DyRA approximated linear layer for NVIDIA B200 (sm_100a).

The compute runs in libdyra.so (hand-written CUDA: tcgen05/TMA kernels for
bf16, SIMT kernels for fp32) behind the C ABI of include/dyra.h; `dyra` is
its ctypes binding and `prep` the host-side offline preparation.
"""

from . import dyra, prep  # noqa: F401
from .dyra import DyraError, DyraLinear  # noqa: F401
