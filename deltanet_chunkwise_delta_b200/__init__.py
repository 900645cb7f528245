"""B200-native chunkwise DeltaNet forward pass (with Gated DeltaNet and Gated
Delta Product).

The computation lives in a CUDA library for sm_100a (``csrc/``, C ABI in
``include/deltanet.h``); this package only builds it, marshals arguments and
draws synthetic inputs (``workloads``).
"""
from ._lib import (DeltaNetError, deltanet_fwd, deltanet_fwd_noalloc,  # noqa: F401
                   gated_deltanet_fwd, gated_deltaproduct_fwd, get_error, last_launches,
                   last_schedule, load, release_workspace, set_kernel_events, status_string)

__all__ = ["deltanet_fwd", "gated_deltanet_fwd", "gated_deltaproduct_fwd",
           "deltanet_fwd_noalloc", "get_error", "release_workspace", "last_schedule",
           "last_launches", "set_kernel_events", "status_string", "DeltaNetError", "load"]
