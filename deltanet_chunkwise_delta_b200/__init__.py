"""B200-native chunkwise DeltaNet forward pass (with Gated DeltaNet, Gated Delta
Product and Kimi Delta Attention).

The computation lives in a CUDA library for sm_100a (``csrc/``, C ABI in
``include/deltanet.h``); this package only builds it, marshals arguments and
draws synthetic inputs (``workloads``).
"""
from ._lib import (DeltaNetError, chunk_state_rows, deltanet_fwd,  # noqa: F401
                   deltanet_fwd_noalloc, deltanet_fwd_states, gated_deltanet_fwd, gated_deltaproduct_fwd, get_error, last_launches,
                   last_schedule, load, release_workspace, set_kernel_events, status_string,
                   test_set_wait, kda_fwd)

__all__ = ["deltanet_fwd", "gated_deltanet_fwd", "gated_deltaproduct_fwd", "kda_fwd",
           "deltanet_fwd_states", "chunk_state_rows",
           "deltanet_fwd_noalloc", "get_error", "release_workspace", "last_schedule",
           "last_launches", "set_kernel_events", "status_string", "test_set_wait",
           "DeltaNetError", "load"]
