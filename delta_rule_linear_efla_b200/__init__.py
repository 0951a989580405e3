"""B200-native Exact Flow Linear Attention (EFLA): forward, decode and backward passes.

The computation lives in libefla.so (hand-written CUDA for sm_100a behind the
C ABI in include/efla.h); `efla` is its Python binding and `inputs` the seeded
synthetic workloads.  Importing the package does not load the library; the
first call does, and raises if it is missing.
"""
from . import inputs  # noqa: F401
from .efla import (  # noqa: F401
    ABI_SYMBOLS, EflaError, EflaFunction, alpha, bwd, chunk_fwd, chunk_fwd_path, efla_attention,
    kernel_launches, last_device_error, load_library, recurrent_step, state_affine, status_str,
    workspace_size,
)
