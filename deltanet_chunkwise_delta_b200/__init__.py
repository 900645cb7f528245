"""B200-native chunkwise DeltaNet forward pass.

The computation lives in a CUDA library for sm_100a (``csrc/``, C ABI in
``include/deltanet.h``); this package only builds it, marshals arguments and
draws synthetic inputs (``workloads``).
"""
from ._lib import (DeltaNetError, deltanet_fwd, get_error, last_schedule,  # noqa: F401
                   load, release_workspace, status_string)

__all__ = ["deltanet_fwd", "get_error", "release_workspace", "last_schedule", "status_string",
           "DeltaNetError", "load"]
