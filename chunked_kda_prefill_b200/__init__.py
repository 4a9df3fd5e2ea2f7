"""B200-native chunked Kimi Delta Attention (KDA) prefill.

Hand-written sm_100a CUDA kernels behind a C ABI (include/kda.h, libkda.so); this package is
the thin Python binding over it.  Build the library with
``python -m chunked_kda_prefill_b200.build``.
"""
from ._lib import EXPORTS, LIB_PATH, KdaError, KdaShape, load  # noqa: F401
from .api import (KdaPlan, LAYOUTS, decode, device_status, flash_kda, flash_kda_noalloc,  # noqa: F401
                  forward_kernel_names, forward_summary, kernels_per_forward, make_plan,
                  noalloc_status, plan, state_chain)
from .context_parallel import flash_kda_context_parallel  # noqa: F401
