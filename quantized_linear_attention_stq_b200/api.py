"""Python binding of the C ABI in include/stq.h (argument marshalling only).

Every computation runs in libstq.so on the GPU. This module checks tensor dtypes, shapes,
devices and contiguity, passes raw pointers and the current CUDA stream through ctypes, and turns
status codes into exceptions. There is no CPU fallback: if the library is missing the first call
raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstq.so")

STQ_OK, STQ_ERR_INVALID_ARG, STQ_ERR_UNSUPPORTED, STQ_ERR_CUDA = 0, 1, 2, 3
STQ_ERR_NONFINITE, STQ_ERR_TIMEOUT, STQ_ERR_BOUNDS = 4, 5, 6
GATE_SCALAR, GATE_CHANNEL, GATE_CHANNEL_DECAY_FIRST = 0, 1, 2
SCALES_ROW_COLUMN, SCALES_UNIFORM = 0, 1  # stq_scale_mode
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}

# Every function the public header declares (checked against include/stq.h by the tests).
EXPORTS = (
    "stq_abi_version", "stq_status_string", "stq_layout_create", "stq_layout_destroy",
    "stq_layout_bytes_per_request", "stq_layout_head_offset", "stq_layout_head_bytes",
    "stq_layout_head_bits", "stq_init_state", "stq_decode_step", "stq_prefill_workspace_bytes",
    "stq_prefill_chunk", "stq_prefill_chunk_noalloc", "stq_dequantize", "stq_allocate_widths", "stq_row_impact",
    "stq_selftest_wait_timeout",
)


class StqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class _Desc(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("head_bits", ctypes.POINTER(ctypes.c_uint8)), ("gate", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("scale_mode", ctypes.c_int32), ("scale_dtype", ctypes.c_int32),
                ("scale_fit_rounds", ctypes.c_int32)]


_lock = threading.Lock()
_lib_handle = None


def lib() -> ctypes.CDLL:
    """Load libstq.so (raises if it has not been built)."""
    global _lib_handle
    with _lock:
        if _lib_handle is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m quantized_linear_attention_stq_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            L.stq_abi_version.restype = i32
            L.stq_status_string.argtypes, L.stq_status_string.restype = [i32], ctypes.c_char_p
            L.stq_layout_create.argtypes = [ctypes.POINTER(_Desc), ctypes.POINTER(P)]
            L.stq_layout_create.restype = i32
            L.stq_layout_destroy.argtypes, L.stq_layout_destroy.restype = [P], None
            L.stq_layout_bytes_per_request.argtypes, L.stq_layout_bytes_per_request.restype = [P], sz
            for n in ("stq_layout_head_offset", "stq_layout_head_bytes"):
                getattr(L, n).argtypes, getattr(L, n).restype = [P, i32], sz
            L.stq_layout_head_bits.argtypes, L.stq_layout_head_bits.restype = [P, i32], i32
            L.stq_init_state.argtypes = [P, P, i32, P, i32, P, P, P, P]
            L.stq_init_state.restype = i32
            L.stq_decode_step.argtypes = [P, P, i32, P, i32, i32, i32, P, P, P, P, P, P, P, P, P]
            L.stq_decode_step.restype = i32
            L.stq_prefill_workspace_bytes.argtypes = [P, i32, i32, i32]
            L.stq_prefill_workspace_bytes.restype = sz
            L.stq_prefill_chunk.argtypes = [P, P, i32, P, i32, i32, i32, P, P, P, P, P, P, P, P, sz, P, P]
            L.stq_prefill_chunk.restype = i32
            L.stq_prefill_chunk_noalloc.argtypes = [P, P, i32, P, i32, i32, i32, P, P, P, P, P, P, P, P, P]
            L.stq_prefill_chunk_noalloc.restype = i32
            L.stq_dequantize.argtypes = [P, P, i32, P, i32, P, P, P]
            L.stq_dequantize.restype = i32
            L.stq_allocate_widths.argtypes = [i32, i32, P, P, i32, ctypes.c_uint64, P]
            L.stq_allocate_widths.restype = i32
            L.stq_row_impact.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P]
            L.stq_row_impact.restype = i32
            L.stq_selftest_wait_timeout.argtypes, L.stq_selftest_wait_timeout.restype = [P, P], i32
            _lib_handle = L
    return _lib_handle


def status_string(status: int) -> str:
    return lib().stq_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != STQ_OK:
        raise StqError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype, shape, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


class Layout:
    """Host-side description of one model's quantized state (see stq_layout_desc)."""

    def __init__(self, head_bits: Sequence[int], d: int, gate: int = GATE_SCALAR,
                 in_dtype: torch.dtype = torch.bfloat16, scale_mode: int = SCALES_ROW_COLUMN,
                 scale_dtype: torch.dtype = torch.float32, fit_rounds: int = 0):
        self.head_bits = [int(b) for b in head_bits]
        self.H, self.d, self.gate, self.in_dtype = len(self.head_bits), int(d), int(gate), in_dtype
        self.scale_mode = int(scale_mode)
        self.scale_dtype = scale_dtype
        self.fit_rounds = int(fit_rounds)
        if in_dtype not in _DTYPES:
            raise TypeError(f"unsupported input dtype {in_dtype}")
        if scale_dtype not in _DTYPES:
            raise TypeError(f"unsupported scale dtype {scale_dtype}")
        arr = (ctypes.c_uint8 * self.H)(*self.head_bits)
        desc = _Desc(self.H, self.d, self.d, ctypes.cast(arr, ctypes.POINTER(ctypes.c_uint8)),
                     self.gate, _DTYPES[in_dtype], self.scale_mode, _DTYPES[scale_dtype], self.fit_rounds)
        handle = ctypes.c_void_p()
        _check(lib().stq_layout_create(ctypes.byref(desc), ctypes.byref(handle)), "stq_layout_create")
        self._h = handle

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib_handle is not None:
            _lib_handle.stq_layout_destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    @property
    def bytes_per_request(self) -> int:
        return lib().stq_layout_bytes_per_request(self._h)

    def head_offset(self, h: int) -> int:
        return lib().stq_layout_head_offset(self._h, h)

    def head_bytes(self, h: int) -> int:
        return lib().stq_layout_head_bytes(self._h, h)

    def head_bits_of(self, h: int) -> int:
        return lib().stq_layout_head_bits(self._h, h)

    def alloc_pool(self, slots: int, device="cuda") -> torch.Tensor:
        """A zeroed pool of `slots` request blocks (uint8)."""
        return torch.zeros(slots * self.bytes_per_request, dtype=torch.uint8, device=device)


def _pool_slots(layout: Layout, pool: torch.Tensor) -> int:
    if pool.dtype != torch.uint8 or pool.dim() != 1 or not pool.is_contiguous():
        raise ValueError("pool must be a contiguous 1-D uint8 tensor")
    return pool.numel() // layout.bytes_per_request


def init_state(layout: Layout, pool, slots, S0, w, status=None, stream=None):
    B = slots.numel()
    dev = pool.device
    _need(slots, "slots", torch.int32, (B,), dev)
    _need(S0, "S0", torch.float32, (B, layout.H, layout.d, layout.d), dev)
    _need(w, "w", torch.float32, (layout.H, layout.d), dev)
    _check(lib().stq_init_state(layout.handle, _ptr(pool), _pool_slots(layout, pool), _ptr(slots), B,
                                _ptr(S0), _ptr(w), _ptr(status), _stream(stream)), "stq_init_state")


def decode_step(layout: Layout, pool, slots, q, k, v, beta, alpha, w, o, head_begin: int = 0,
                status=None, stream=None):
    """One in-place decode step for heads [head_begin, head_begin + q.shape[1])."""
    B, hc, d = q.shape
    dev = pool.device
    _need(slots, "slots", torch.int32, (B,), dev)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, layout.in_dtype, (B, hc, d), dev)
    _need(beta, "beta", torch.float32, (B, hc), dev)
    _need(alpha, "alpha", torch.float32, (B, hc) if layout.gate == GATE_SCALAR else (B, hc, d), dev)
    _need(w, "w", torch.float32, (hc, d), dev)
    _need(o, "o", torch.float32, (B, hc, d), dev)
    _check(lib().stq_decode_step(layout.handle, _ptr(pool), _pool_slots(layout, pool), _ptr(slots), B,
                                 head_begin, hc, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(w),
                                 _ptr(o), _ptr(status), _stream(stream)), "stq_decode_step")


def prefill_workspace_bytes(layout: Layout, B: int, T: int, chunk: int) -> int:
    return lib().stq_prefill_workspace_bytes(layout.handle, B, T, chunk)


def prefill_chunk(layout: Layout, pool, slots, q, k, v, beta, alpha, w, o, chunk: int = 64,
                  workspace=None, status=None, stream=None):
    """Chunked prefill of T tokens (q, k, v: [B, H, T, d]) for all heads, in place."""
    B, H, T, d = q.shape
    dev = pool.device
    _need(slots, "slots", torch.int32, (B,), dev)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, layout.in_dtype, (B, H, T, d), dev)
    _need(beta, "beta", torch.float32, (B, H, T), dev)
    _need(alpha, "alpha", torch.float32, (B, H, T) if layout.gate == GATE_SCALAR else (B, H, T, d), dev)
    _need(w, "w", torch.float32, (H, d), dev)
    _need(o, "o", torch.float32, (B, H, T, d), dev)
    # with a workspace of prefill_workspace_bytes() the tensor-core chunk form runs as three
    # kernels (chunk-parallel inputs and readout around the sequential state kernel); without one
    # it runs as one kernel
    need = prefill_workspace_bytes(layout, B, T, chunk)
    ws_ptr, ws_bytes = None, 0
    if need and workspace is not None:
        ws_bytes = workspace.numel() * workspace.element_size()
        if ws_bytes < need:
            raise ValueError(f"prefill workspace of {ws_bytes} bytes is below the {need} bytes it needs")
        ws_ptr = _ptr(workspace)
    _check(lib().stq_prefill_chunk(layout.handle, _ptr(pool), _pool_slots(layout, pool), _ptr(slots), B, T, chunk,
                                   _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(w), _ptr(o),
                                   ws_ptr, ws_bytes, _ptr(status), _stream(stream)),
           "stq_prefill_chunk")


def prefill_chunk_noalloc(layout: Layout, pool, slots, q, k, v, beta, alpha, w, o, chunk: int = 64, status=None,
                          stream=None):
    """prefill_chunk for callers that cannot allocate device memory: the workspace is a fixed
    32 MiB array inside the library (see stq_prefill_chunk_noalloc in include/stq.h); calls whose
    device work overlaps race on it."""
    B, H, T, d = q.shape
    dev = pool.device
    _need(slots, "slots", torch.int32, (B,), dev)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, layout.in_dtype, (B, H, T, d), dev)
    _need(beta, "beta", torch.float32, (B, H, T), dev)
    _need(alpha, "alpha", torch.float32, (B, H, T) if layout.gate == GATE_SCALAR else (B, H, T, d), dev)
    _need(w, "w", torch.float32, (H, d), dev)
    _need(o, "o", torch.float32, (B, H, T, d), dev)
    _check(lib().stq_prefill_chunk_noalloc(layout.handle, _ptr(pool), _pool_slots(layout, pool), _ptr(slots), B, T,
                                           chunk, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(w), _ptr(o),
                                           _ptr(status), _stream(stream)),
           "stq_prefill_chunk_noalloc")


def dequantize(layout: Layout, pool, slots, S_out, status=None, stream=None):
    B = slots.numel()
    dev = pool.device
    _need(slots, "slots", torch.int32, (B,), dev)
    _need(S_out, "S_out", torch.float32, (B, layout.H, layout.d, layout.d), dev)
    _check(lib().stq_dequantize(layout.handle, _ptr(pool), _pool_slots(layout, pool), _ptr(slots), B, _ptr(S_out),
                                _ptr(status), _stream(stream)), "stq_dequantize")


def selftest_wait_timeout(status, stream=None):
    """Run the bounded-wait self-test: it ORs the timeout bit into `status` (device int32 [1])
    after about two seconds of device time."""
    _need(status, "status", torch.int32, (1,), status.device)
    _check(lib().stq_selftest_wait_timeout(_ptr(status), _stream(stream)), "stq_selftest_wait_timeout")


def status_flags(status: torch.Tensor) -> list:
    """Names of the conditions OR-ed into a device status word (synchronizes)."""
    v = int(status.item())
    return [status_string(c) for c in (STQ_ERR_NONFINITE, STQ_ERR_TIMEOUT, STQ_ERR_BOUNDS) if v & (1 << c)]


def allocate_widths(distortion, mean_log_retention, d: int, num_pivots: int, budget_bytes: int) -> list:
    """Lifetime-aware widths per head (host only): distortion [H][3] at widths 4, 6, 8 and the mean
    log-retention [H] of each head's gate; see stq_allocate_widths in include/stq.h."""
    import numpy as np

    D = np.ascontiguousarray(np.asarray(distortion, dtype=np.float64))
    lr = np.ascontiguousarray(np.asarray(mean_log_retention, dtype=np.float64))
    H = lr.shape[0]
    if D.shape != (H, 3):
        raise ValueError("distortion must be [H][3]")
    out = np.zeros(H, dtype=np.uint8)
    _check(lib().stq_allocate_widths(H, int(d), D.ctypes.data_as(ctypes.c_void_p), lr.ctypes.data_as(ctypes.c_void_p),
                                     int(num_pivots), int(budget_bytes), out.ctypes.data_as(ctypes.c_void_p)),
           "stq_allocate_widths")
    return [int(x) for x in out]


def row_impact(q, k, beta, alpha, gate: int = GATE_SCALAR, stream=None) -> torch.Tensor:
    """Key-row impact scores w [H][d] from calibration tokens q, k [T][H][d], beta [T][H] and
    alpha [T][H] (scalar gate) or [T][H][d]; see stq_row_impact in include/stq.h."""
    T, H, d = q.shape
    dev = q.device
    if q.dtype not in _DTYPES:
        raise TypeError("q must be float32 or bfloat16")
    _need(k, "k", q.dtype, (T, H, d), dev)
    _need(beta, "beta", torch.float32, (T, H), dev)
    _need(alpha, "alpha", torch.float32, (T, H) if gate == GATE_SCALAR else (T, H, d), dev)
    _need(q, "q", q.dtype, (T, H, d), dev)
    w = torch.empty(H, d, dtype=torch.float32, device=dev)
    _check(lib().stq_row_impact(T, H, d, int(gate), _DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(beta), _ptr(alpha),
                                _ptr(w), _stream(stream)), "stq_row_impact")
    return w
