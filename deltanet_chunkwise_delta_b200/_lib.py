"""ctypes binding of the C ABI in include/deltanet.h.

Argument marshalling only: torch tensors are described as ``dn_tensor``
structs (pointer, dtype, shape, strides in elements) and handed to the shared
library.  Every step of the computation runs in the library's CUDA kernels;
there is no other implementation to fall back to.  If the library is missing
or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

from . import build as _build

DN_OK, DN_ERR_INVALID_ARG, DN_ERR_UNSUPPORTED, DN_ERR_ALIAS, DN_ERR_CUDA, \
    DN_ERR_WORKSPACE, DN_ERR_SEQLENS, DN_ERR_TIMEOUT = range(8)
DN_F32, DN_BF16, DN_I32 = 0, 1, 2

EXPORTED = ("deltanet_fwd", "deltanet_fwd_ex", "gated_deltanet_fwd", "gated_deltanet_fwd_ex",
            "gated_deltaproduct_fwd", "gated_deltaproduct_fwd_ex", "deltanet_fwd_states",
            "deltanet_status_string",
            "deltanet_get_error", "deltanet_release_workspace", "deltanet_last_schedule",
            "deltanet_fwd_noalloc", "deltanet_last_launches", "deltanet_set_kernel_events",
            "deltanet_test_set_wait", "kda_fwd", "kda_fwd_ex")


class DnTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class DeltaNetError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _build.LIB


def load(path: Optional[str] = None):
    """Load the shared library (built in-tree by ``build.py``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = path or _build.LIB
        if not os.path.exists(path):
            raise RuntimeError(
                f"DeltaNet CUDA library not found at {path}; run "
                "`python -m deltanet_chunkwise_delta_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(DnTensor)
        lib.deltanet_fwd.restype = ctypes.c_int
        lib.deltanet_fwd.argtypes = [P, P, P, P, P, P, ctypes.c_int, P, P, ctypes.c_void_p]
        lib.deltanet_fwd_ex.restype = ctypes.c_int
        lib.deltanet_fwd_ex.argtypes = [P, P, P, P, P, P, ctypes.c_int, P, P, ctypes.c_void_p,
                                        ctypes.c_int]
        lib.gated_deltanet_fwd.restype = ctypes.c_int
        lib.gated_deltanet_fwd.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, P, P,
                                           ctypes.c_void_p]
        lib.gated_deltanet_fwd_ex.restype = ctypes.c_int
        lib.gated_deltanet_fwd_ex.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, P, P,
                                              ctypes.c_void_p, ctypes.c_int]
        lib.gated_deltaproduct_fwd.restype = ctypes.c_int
        lib.gated_deltaproduct_fwd.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                               P, P, ctypes.c_void_p]
        lib.gated_deltaproduct_fwd_ex.restype = ctypes.c_int
        lib.gated_deltaproduct_fwd_ex.argtypes = [P, P, P, P, P, P, P, ctypes.c_int,
                                                  ctypes.c_int, P, P, ctypes.c_void_p,
                                                  ctypes.c_int]
        lib.kda_fwd.restype = ctypes.c_int
        lib.kda_fwd.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, P, P, ctypes.c_void_p]
        lib.kda_fwd_ex.restype = ctypes.c_int
        lib.kda_fwd_ex.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, P, P, ctypes.c_void_p,
                                   ctypes.c_int]
        lib.deltanet_fwd_states.restype = ctypes.c_int
        lib.deltanet_fwd_states.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, P, P, P,
                                            ctypes.c_void_p, ctypes.c_int]
        lib.deltanet_fwd_noalloc.restype = ctypes.c_int
        lib.deltanet_fwd_noalloc.argtypes = [P, P, P, P, P, ctypes.c_int, P, P, ctypes.c_void_p]
        lib.deltanet_status_string.restype = ctypes.c_char_p
        lib.deltanet_status_string.argtypes = [ctypes.c_int]
        lib.deltanet_get_error.restype = ctypes.c_int
        lib.deltanet_get_error.argtypes = [ctypes.c_void_p]
        lib.deltanet_release_workspace.restype = None
        lib.deltanet_release_workspace.argtypes = []
        lib.deltanet_last_launches.restype = ctypes.c_int
        lib.deltanet_last_launches.argtypes = []
        lib.deltanet_set_kernel_events.restype = None
        lib.deltanet_set_kernel_events.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        lib.deltanet_test_set_wait.restype = None
        lib.deltanet_test_set_wait.argtypes = [ctypes.c_ulonglong, ctypes.c_int]
        lib.deltanet_last_schedule.restype = None
        lib.deltanet_last_schedule.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                               ctypes.POINTER(ctypes.c_int)]
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().deltanet_status_string(int(status)).decode()


_DT = {torch.float32: DN_F32, torch.bfloat16: DN_BF16, torch.int32: DN_I32}


def describe(t: Optional[torch.Tensor]) -> Optional[DnTensor]:
    """dn_tensor view of a tensor (strides in elements); None stays None."""
    if t is None:
        return None
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    d = DnTensor()
    d.data = t.data_ptr() if t.numel() > 0 else None
    d.dtype = _DT[t.dtype]
    d.ndim = t.dim()
    for i in range(4):
        d.shape[i] = t.shape[i] if i < t.dim() else 0
        d.stride[i] = t.stride(i) if i < t.dim() else 0
    return d


def _ref(d: Optional[DnTensor]):
    return None if d is None else ctypes.byref(d)


def call(q, k, v, beta, initial_state, cu_seqlens, chunk_size, out, final_state, stream,
         seg_chunks: int = 0) -> int:
    """Raw call: returns the dn_status code (no exception)."""
    lib = load()
    ds = [describe(t) for t in (q, k, v, beta, initial_state, cu_seqlens, out, final_state)]
    args = [_ref(x) for x in ds[:6]] + [int(chunk_size)] + [_ref(x) for x in ds[6:]]
    if seg_chunks:
        return lib.deltanet_fwd_ex(*args, stream, int(seg_chunks))
    return lib.deltanet_fwd(*args, stream)


def call_gated(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
               stream, seg_chunks: int = 0) -> int:
    """Raw Gated DeltaNet call: returns the dn_status code (no exception)."""
    lib = load()
    ds = [describe(t) for t in (q, k, v, beta, g, initial_state, cu_seqlens, out, final_state)]
    args = [_ref(x) for x in ds[:7]] + [int(chunk_size)] + [_ref(x) for x in ds[7:]]
    if seg_chunks:
        return lib.gated_deltanet_fwd_ex(*args, stream, int(seg_chunks))
    return lib.gated_deltanet_fwd(*args, stream)


def call_kda(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
             stream, seg_chunks: int = 0) -> int:
    """Raw Kimi Delta Attention call: returns the dn_status code (no exception)."""
    lib = load()
    ds = [describe(t) for t in (q, k, v, beta, g, initial_state, cu_seqlens, out, final_state)]
    args = [_ref(x) for x in ds[:7]] + [int(chunk_size)] + [_ref(x) for x in ds[7:]]
    if seg_chunks:
        return lib.kda_fwd_ex(*args, stream, int(seg_chunks))
    return lib.kda_fwd(*args, stream)


def _stream_handle(device, stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def deltanet_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: torch.Tensor,
                 initial_state: Optional[torch.Tensor] = None,
                 cu_seqlens: Optional[torch.Tensor] = None, chunk_size: int = 64,
                 out: Optional[torch.Tensor] = None,
                 final_state: Optional[torch.Tensor] = None,
                 output_final_state: bool = True, stream=None, seg_chunks: int = 0):
    """DeltaNet forward on CUDA tensors through the C ABI.

    Shapes: q, k [B, T, H, d_k]; v [B, T, H, d_v]; beta [B, T, H] fp32;
    initial_state [N, H, d_k, d_v] fp32 or None; cu_seqlens int32 [N+1] or None.
    Allocates ``out`` / ``final_state`` when not given.  Returns
    (out, final_state or None).  Asynchronous on ``stream`` (default: torch's
    current stream).
    """
    if not q.is_cuda:
        raise ValueError("deltanet_fwd runs on CUDA tensors only")
    B, T, H, _ = q.shape
    dk, dv = q.shape[3], v.shape[3]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    st = call(q, k, v, beta, initial_state, cu_seqlens, chunk_size, out, final_state,
              _stream_handle(q.device, stream), seg_chunks)
    if st != DN_OK:
        raise DeltaNetError(st, status_string(st))
    return out, final_state


def gated_deltanet_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: torch.Tensor,
                       g: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                       cu_seqlens: Optional[torch.Tensor] = None, chunk_size: int = 64,
                       out: Optional[torch.Tensor] = None,
                       final_state: Optional[torch.Tensor] = None,
                       output_final_state: bool = True, stream=None, seg_chunks: int = 0):
    """Gated DeltaNet forward on CUDA tensors through the C ABI.

    As ``deltanet_fwd``, plus ``g`` [B, T, H] fp32: the per-token decay as its
    natural log, g = ln a (the state update is S <- a (I - beta k^T k) S + beta k^T v).
    """
    if not q.is_cuda:
        raise ValueError("gated_deltanet_fwd runs on CUDA tensors only")
    B, T, H, _ = q.shape
    dk, dv = q.shape[3], v.shape[3]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    st = call_gated(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    _stream_handle(q.device, stream), seg_chunks)
    if st != DN_OK:
        raise DeltaNetError(st, status_string(st))
    return out, final_state


def kda_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: torch.Tensor,
            g: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
            cu_seqlens: Optional[torch.Tensor] = None, chunk_size: int = 64,
            out: Optional[torch.Tensor] = None, final_state: Optional[torch.Tensor] = None,
            output_final_state: bool = True, stream=None, seg_chunks: int = 0):
    """Kimi Delta Attention forward on CUDA tensors through the C ABI.

    As ``deltanet_fwd``, plus ``g`` [B, T, H, d_k] fp32: the decay of every key channel
    as its natural log (the state update is S <- (I - beta k^T k) Diag(a) S + beta k^T v).
    """
    if not q.is_cuda:
        raise ValueError("kda_fwd runs on CUDA tensors only")
    B, T, H, _ = q.shape
    dk, dv = q.shape[3], v.shape[3]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    st = call_kda(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                  _stream_handle(q.device, stream), seg_chunks)
    if st != DN_OK:
        raise DeltaNetError(st, status_string(st))
    return out, final_state


def chunk_state_rows(B: int, T: int, cu_seqlens: Optional[torch.Tensor] = None,
                     chunk_size: int = 64) -> int:
    """Rows of the chunk-states buffer: B * ceil(T / C) for a dense batch; for packed
    input ceil(T / C) + N, a bound on the sum of ceil(L_n / C)."""
    n_c = (T + chunk_size - 1) // chunk_size
    return B * n_c if cu_seqlens is None else n_c + cu_seqlens.numel() - 1


def deltanet_fwd_states(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: torch.Tensor,
                        g: Optional[torch.Tensor] = None,
                        initial_state: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None, chunk_size: int = 64,
                        out: Optional[torch.Tensor] = None,
                        final_state: Optional[torch.Tensor] = None,
                        chunk_states: Optional[torch.Tensor] = None, stream=None,
                        seg_chunks: int = 0):
    """DeltaNet (g None) or Gated DeltaNet forward that also returns the state
    entering every chunk: chunk_states [rows, H, d_k, d_v] fp32 with row = global
    chunk index (see ``chunk_state_rows``; allocated zeroed when not given).
    Returns (out, final_state, chunk_states)."""
    if not q.is_cuda:
        raise ValueError("deltanet_fwd_states runs on CUDA tensors only")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    if chunk_states is None:
        rows = chunk_state_rows(B, T, cu_seqlens, chunk_size)
        chunk_states = torch.zeros((rows, H, dk, dv), dtype=torch.float32, device=q.device)
    ds = [describe(t) for t in (q, k, v, beta, g, initial_state, cu_seqlens, out, final_state,
                                chunk_states)]
    args = [_ref(x) for x in ds[:7]] + [int(chunk_size)] + [_ref(x) for x in ds[7:]]
    st = load().deltanet_fwd_states(*args, _stream_handle(q.device, stream), int(seg_chunks))
    if st != DN_OK:
        raise DeltaNetError(st, status_string(st))
    return out, final_state, chunk_states


def gated_deltaproduct_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           beta: torch.Tensor, g: torch.Tensor, n_h: int,
                           initial_state: Optional[torch.Tensor] = None,
                           cu_seqlens: Optional[torch.Tensor] = None, chunk_size: int = 64,
                           out: Optional[torch.Tensor] = None,
                           final_state: Optional[torch.Tensor] = None,
                           output_final_state: bool = True, stream=None, seg_chunks: int = 0):
    """Gated Delta Product forward on CUDA tensors through the C ABI.

    q [B, T, H, d_k]; k [B, T * n_h, H, d_k], v [B, T * n_h, H, d_v] and beta
    [B, T * n_h, H] with the n_h writes of each token on consecutive rows; g
    [B, T, H] (ln a, one per token); cu_seqlens counts tokens.  Returns
    (out [B, T, H, d_v], final_state or None).
    """
    if not q.is_cuda:
        raise ValueError("gated_deltaproduct_fwd runs on CUDA tensors only")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    ds = [describe(t) for t in (q, k, v, beta, g, initial_state, cu_seqlens, out, final_state)]
    args = [_ref(x) for x in ds[:7]] + [int(n_h), int(chunk_size)] + [_ref(x) for x in ds[7:]]
    lib = load()
    stream_h = _stream_handle(q.device, stream)
    if seg_chunks:
        st = lib.gated_deltaproduct_fwd_ex(*args, stream_h, int(seg_chunks))
    else:
        st = lib.gated_deltaproduct_fwd(*args, stream_h)
    if st != DN_OK:
        raise DeltaNetError(st, status_string(st))
    return out, final_state


def deltanet_fwd_noalloc(q, k, v, beta, initial_state=None, chunk_size: int = 64, out=None,
                         final_state=None, stream=None):
    """The forward pass through the entry point that allocates no device memory
    (for callers that cannot allocate; see include/deltanet.h).  Dense bf16
    batches with d_k = d_v = 128 only.  ``out`` and ``final_state`` are allocated
    here with torch when not given: the C call itself allocates nothing."""
    B, T, H, _ = q.shape
    if out is None:
        out = torch.empty((B, T, H, v.shape[3]), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((B, H, q.shape[3], v.shape[3]), dtype=torch.float32,
                                  device=q.device)
    ds = [describe(t) for t in (q, k, v, beta, initial_state, out, final_state)]
    st = load().deltanet_fwd_noalloc(*[_ref(x) for x in ds[:5]], int(chunk_size),
                                     *[_ref(x) for x in ds[5:]],
                                     _stream_handle(q.device, stream))
    if st != DN_OK:
        raise DeltaNetError(st, status_string(st))
    return out, final_state


def get_error(stream=None, device=None) -> int:
    """Synchronise the stream and return (and clear) its device-side error flag."""
    return load().deltanet_get_error(_stream_handle(device, stream))


def test_set_wait(wait_ns: int = 0, stall_chunk: int = 0) -> None:
    """Test hook of the bounded device waits for the following calls on this
    thread: their time-out (0: the default 2 s) and, with stall_chunk > 0, a
    wait at chunk stall_chunk - 1 of every run that nothing completes
    (deltanet_test_set_wait in include/deltanet.h).  test_set_wait() restores
    normal calls."""
    load().deltanet_test_set_wait(int(wait_ns), int(stall_chunk))


def release_workspace() -> None:
    load().deltanet_release_workspace()


def last_launches() -> int:
    return load().deltanet_last_launches()


def set_kernel_events(start=None, stop=None) -> None:
    """Bracket the boundary-pass kernel of following calls with two
    torch.cuda.Event objects (enable_timing=True, already recorded once so that
    their handles exist); call with no arguments to stop."""
    load().deltanet_set_kernel_events(start.cuda_event if start is not None else None,
                                      stop.cuda_event if stop is not None else None)


def last_schedule(with_first: bool = False):
    """(segments per chain, chunks per segment) of the last dense call on this
    thread; with ``with_first`` also the chunks of the first segment."""
    g, s, s0 = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    load().deltanet_last_schedule(ctypes.byref(g), ctypes.byref(s), ctypes.byref(s0))
    return (g.value, s.value, s0.value) if with_first else (g.value, s.value)
