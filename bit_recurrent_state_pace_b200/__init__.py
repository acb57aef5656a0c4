"""Python binding of libpace (PACE periodic low-bit recurrent-state decode).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of ``libpace.so``.  PyTorch supplies device memory and streams.
The functions keep the C names of ``include/pace.h``; ``PacePool`` is a
convenience owner of the three device regions a pool needs.

Importing this package loads ``libpace.so`` from this directory and raises
``ImportError`` if it is missing (build it with
``python -m bit_recurrent_state_pace_b200.build``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "PaceError", "lib", "LIB_PATH",
    "PACE_SCALE_COL", "PACE_SCALE_ROW", "PACE_IO_BF16", "PACE_IO_F32",
    "PACE_OK", "PACE_ERR_INVALID_ARG", "PACE_ERR_UNSUPPORTED", "PACE_ERR_CUDA", "PACE_ERR_DEVICE_FLAGS",
    "PACE_FLAG_NONFINITE", "PACE_FLAG_SCALE_OVERFLOW", "PACE_FLAG_BUFFER_FULL", "PACE_FLAG_TIMEOUT",
    "PACE_FILL_COMMIT",
    "pace_pool_bytes", "pace_init_pool", "pace_destroy_pool", "pace_pool_layout",
    "pace_pool_load", "pace_pool_export", "pace_decode_step", "pace_commit_period",
    "pace_decode_step_range", "pace_commit_period_range", "pace_decay_rates",
    "pace_select_head_bits", "pace_prefill", "pace_prefill_range", "pace_host_staging_bytes",
    "pace_decode_host", "pace_set_commit_threshold", "pace_window_scratch_bytes", "pace_window_step",
    "pace_window_step_static", "PACE_WINDOW_STATIC_SCRATCH_BYTES", "pace_set_commit_engine",
    "PACE_COMMIT_MMA", "PACE_COMMIT_TCGEN05", "pace_debug_wait_fault",
    "pace_quantize", "pace_dequantize", "pace_pool_status", "pace_pool_clear_status",
    "pace_gdn_step_f32", "pace_gdn_step_bf16", "pace_status_string", "pace_version",
    "PacePool",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpace.so")

PACE_SCALE_COL, PACE_SCALE_ROW = 0, 1
PACE_IO_BF16, PACE_IO_F32 = 0, 1
PACE_FLAG_NONFINITE = 0x1
PACE_FLAG_SCALE_OVERFLOW = 0x2
PACE_FLAG_BUFFER_FULL = 0x4
PACE_FLAG_TIMEOUT = 0x8
PACE_FILL_COMMIT = 0x100
PACE_WINDOW_STATIC_SCRATCH_BYTES = 8 << 20
PACE_COMMIT_MMA, PACE_COMMIT_TCGEN05 = 0, 1
PACE_OK, PACE_ERR_INVALID_ARG, PACE_ERR_UNSUPPORTED, PACE_ERR_CUDA, PACE_ERR_DEVICE_FLAGS = 0, 1, 2, 3, 4


class PaceError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {_status_name(status)} ({status})")
        self.status = status


class _Desc(ctypes.Structure):
    _fields_ = [("num_slots", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("period", ctypes.c_int32),
                ("scale_axis", ctypes.c_int32), ("io_dtype", ctypes.c_int32),
                ("head_bits", ctypes.POINTER(ctypes.c_uint8)), ("buffer_e4m3", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libpace.so not found at {LIB_PATH}: build it with "
                          "`python -m bit_recurrent_state_pace_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P, S, I32, I64, U32p, U16p, F32p = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p)
    Sp = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "pace_pool_bytes": [ctypes.POINTER(_Desc), Sp, Sp, Sp],
        "pace_init_pool": [ctypes.POINTER(_Desc), P, P, P, P, ctypes.POINTER(ctypes.c_void_p)],
        "pace_pool_layout": [P, I32, Sp, Sp, Sp],
        "pace_pool_load": [P, F32p, P],
        "pace_pool_export": [P, F32p, P],
        "pace_decode_step": [P, P, P, P, P, P, F32p, P],
        "pace_commit_period": [P, P],
        "pace_decode_step_range": [P, I32, I32, I32, P, P, P, P, P, F32p, P],
        "pace_commit_period_range": [P, I32, I32, I32, P],
        "pace_decay_rates": [P, I64, I32, I32, P, P],
        "pace_prefill": [P, I64, P, P, P, P, P, F32p, P],
        "pace_host_staging_bytes": [P, Sp],
        "pace_set_commit_threshold": [P, ctypes.c_float],
        "pace_set_commit_engine": [P, I32],
        "pace_debug_wait_fault": [P, ctypes.c_uint64, ctypes.c_uint32],
        "pace_window_scratch_bytes": [P, Sp],
        "pace_window_step": [P, P, P, P, P, P, F32p, P, P],
        "pace_window_step_static": [P, P, P, P, P, P, F32p, P],
        "pace_decode_host": [P, I32, P, P, P, P, P, P, P, P, P, P],
        "pace_prefill_range": [P, I32, I32, I64, P, P, P, P, P, F32p, P],
        "pace_select_head_bits": [P, I32, I32, P],
        "pace_quantize": [F32p, I64, I32, I32, I32, I32, P, U16p, U32p, P],
        "pace_dequantize": [P, U16p, I64, I32, I32, I32, I32, F32p, P],
        "pace_pool_status": [P, P, ctypes.POINTER(ctypes.c_uint32)],
        "pace_pool_clear_status": [P, P],
        "pace_gdn_step_f32": [F32p, P, P, P, P, P, I32, F32p, I64, I32, I32, P],
        "pace_gdn_step_bf16": [U16p, P, P, P, P, P, I32, F32p, I64, I32, I32, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.pace_destroy_pool.argtypes = [P]
    L.pace_destroy_pool.restype = None
    L.pace_status_string.argtypes = [ctypes.c_int]
    L.pace_status_string.restype = ctypes.c_char_p
    L.pace_version.argtypes = []
    L.pace_version.restype = ctypes.c_char_p
    return L


lib = _load()


def _status_name(s: int) -> str:
    return lib.pace_status_string(int(s)).decode()


def _check(fn: str, status: int, ok=(PACE_OK,)) -> int:
    if status not in ok:
        raise PaceError(fn, status)
    return status


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libpace takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libpace takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _desc(B, H, d_k, d_v, P, axis, io, head_bits, buffer_e4m3=0) -> Tuple[_Desc, ctypes.Array]:
    vals = [int(b) for b in head_bits]
    bits_arr = (ctypes.c_uint8 * max(len(vals), 1))(*vals)
    d = _Desc(B, H, d_k, d_v, P, axis, io, ctypes.cast(bits_arr, ctypes.POINTER(ctypes.c_uint8)),
              int(buffer_e4m3))
    return d, bits_arr


# ---------------------------------------------------------------- C names

def pace_pool_bytes(B, H, d_k, d_v, P, axis, io, head_bits, buffer_e4m3=0) -> Tuple[int, int, int]:
    d, keep = _desc(B, H, d_k, d_v, P, axis, io, head_bits, buffer_e4m3)
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("pace_pool_bytes", lib.pace_pool_bytes(ctypes.byref(d), ctypes.byref(a), ctypes.byref(b),
                                                   ctypes.byref(c)))
    return a.value, b.value, c.value


def pace_init_pool(B, H, d_k, d_v, P, axis, io, head_bits, state, buffer, aux, stream=None,
                   buffer_e4m3=0) -> int:
    d, keep = _desc(B, H, d_k, d_v, P, axis, io, head_bits, buffer_e4m3)
    out = ctypes.c_void_p()
    _check("pace_init_pool", lib.pace_init_pool(ctypes.byref(d), _ptr(state), _ptr(buffer), _ptr(aux),
                                                 _stream(stream), ctypes.byref(out)))
    return out.value


def pace_destroy_pool(handle: int) -> None:
    lib.pace_destroy_pool(handle)


def pace_pool_layout(handle: int, head: int) -> Tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("pace_pool_layout", lib.pace_pool_layout(handle, head, ctypes.byref(a), ctypes.byref(b),
                                                     ctypes.byref(c)))
    return a.value, b.value, c.value


def pace_pool_load(handle: int, S: torch.Tensor, stream=None) -> None:
    _check("pace_pool_load", lib.pace_pool_load(handle, _ptr(S), _stream(stream)))


def pace_pool_export(handle: int, S: torch.Tensor, stream=None) -> None:
    _check("pace_pool_export", lib.pace_pool_export(handle, _ptr(S), _stream(stream)))


def pace_decode_step(handle: int, q, k, v, alpha, beta, o, stream=None) -> None:
    _check("pace_decode_step", lib.pace_decode_step(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                                     _ptr(beta), _ptr(o), _stream(stream)))


def pace_commit_period(handle: int, stream=None) -> None:
    _check("pace_commit_period", lib.pace_commit_period(handle, _stream(stream)))


def pace_window_scratch_bytes(handle: int) -> int:
    n = ctypes.c_size_t()
    _check("pace_window_scratch_bytes", lib.pace_window_scratch_bytes(handle, ctypes.byref(n)))
    return n.value


def pace_window_step(handle: int, q, k, v, alpha, beta, o, scratch, stream=None) -> None:
    _check("pace_window_step", lib.pace_window_step(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                                    _ptr(beta), _ptr(o), _ptr(scratch), _stream(stream)))


def pace_window_step_static(handle: int, q, k, v, alpha, beta, o, stream=None) -> None:
    """pace_window_step with the library's own device scratch (no allocation)."""
    _check("pace_window_step_static", lib.pace_window_step_static(
        handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o), _stream(stream)))


def pace_set_commit_threshold(handle: int, tau: float) -> None:
    _check("pace_set_commit_threshold", lib.pace_set_commit_threshold(handle, float(tau)))


def pace_set_commit_engine(handle: int, engine: int) -> None:
    _check("pace_set_commit_engine", lib.pace_set_commit_engine(handle, int(engine)))


def pace_debug_wait_fault(handle: int, wait_limit_ns: int, extra_tx_bytes: int) -> None:
    _check("pace_debug_wait_fault", lib.pace_debug_wait_fault(handle, int(wait_limit_ns), int(extra_tx_bytes)))


def pace_host_staging_bytes(handle: int) -> int:
    n = ctypes.c_size_t()
    _check("pace_host_staging_bytes", lib.pace_host_staging_bytes(handle, ctypes.byref(n)))
    return n.value


def _host_ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("pace_decode_host takes contiguous host tensors")
    return t.data_ptr()


def pace_decode_host(handle: int, n_tokens: int, q, k, v, alpha, beta, o, staging, stream,
                     h2d_stream, d2h_stream) -> None:
    _check("pace_decode_host", lib.pace_decode_host(
        handle, n_tokens, _host_ptr(q), _host_ptr(k), _host_ptr(v), _host_ptr(alpha), _host_ptr(beta),
        _host_ptr(o), _ptr(staging), _stream(stream), _stream(h2d_stream), _stream(d2h_stream)))


def pace_prefill(handle: int, T: int, q, k, v, alpha, beta, o=None, stream=None) -> None:
    _check("pace_prefill", lib.pace_prefill(handle, T, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                             _ptr(beta), _ptr(o), _stream(stream)))


def pace_prefill_range(handle: int, slot_begin: int, slot_count: int, T: int, q, k, v, alpha, beta,
                       o=None, stream=None) -> None:
    _check("pace_prefill_range", lib.pace_prefill_range(handle, slot_begin, slot_count, T, _ptr(q),
                                                         _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                                         _ptr(o), _stream(stream)))


def pace_decay_rates(alpha: torch.Tensor, num_heads: int, io: int, rates: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Mean -ln(alpha) per head over the rows of a device gate matrix [rows][num_heads]."""
    if rates is None:
        rates = torch.empty(num_heads, dtype=torch.float64, device=alpha.device)
    rows = alpha.numel() // num_heads
    _check("pace_decay_rates", lib.pace_decay_rates(_ptr(alpha), rows, num_heads, io, _ptr(rates),
                                                     _stream(stream)))
    return rates


def pace_select_head_bits(rates: Sequence[float], num_int8: int) -> list:
    """Host: 8 bits for the num_int8 heads with the slowest decay, 4 for the rest."""
    vals = [float(r) for r in rates]
    arr = (ctypes.c_double * max(len(vals), 1))(*vals)
    out = (ctypes.c_uint8 * max(len(vals), 1))()
    _check("pace_select_head_bits", lib.pace_select_head_bits(
        ctypes.cast(arr, ctypes.c_void_p), len(vals), num_int8, ctypes.cast(out, ctypes.c_void_p)))
    return [int(out[i]) for i in range(len(vals))]


def pace_decode_step_range(handle: int, slot_begin: int, slot_count: int, blocks_per_sm: int,
                           q, k, v, alpha, beta, o, stream=None) -> None:
    _check("pace_decode_step_range",
           lib.pace_decode_step_range(handle, slot_begin, slot_count, blocks_per_sm, _ptr(q), _ptr(k),
                                      _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o), _stream(stream)))


def pace_commit_period_range(handle: int, slot_begin: int, slot_count: int, blocks_per_sm: int,
                             stream=None) -> None:
    _check("pace_commit_period_range",
           lib.pace_commit_period_range(handle, slot_begin, slot_count, blocks_per_sm, _stream(stream)))


def pace_quantize(S, n_mats, d_k, d_v, bits, axis, codes, scales, flags=None, stream=None) -> None:
    _check("pace_quantize", lib.pace_quantize(_ptr(S), n_mats, d_k, d_v, bits, axis, _ptr(codes),
                                               _ptr(scales), _ptr(flags), _stream(stream)))


def pace_dequantize(codes, scales, n_mats, d_k, d_v, bits, axis, S, stream=None) -> None:
    _check("pace_dequantize", lib.pace_dequantize(_ptr(codes), _ptr(scales), n_mats, d_k, d_v, bits,
                                                   axis, _ptr(S), _stream(stream)))


def pace_pool_status(handle: int, stream=None) -> int:
    f = ctypes.c_uint32()
    _check("pace_pool_status", lib.pace_pool_status(handle, _stream(stream), ctypes.byref(f)),
           ok=(PACE_OK, PACE_ERR_DEVICE_FLAGS))
    return f.value


def pace_pool_clear_status(handle: int, stream=None) -> None:
    _check("pace_pool_clear_status", lib.pace_pool_clear_status(handle, _stream(stream)))


def pace_gdn_step_f32(S, q, k, v, alpha, beta, io, o, n, d_k, d_v, stream=None) -> None:
    _check("pace_gdn_step_f32", lib.pace_gdn_step_f32(_ptr(S), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                                       _ptr(beta), io, _ptr(o), n, d_k, d_v,
                                                       _stream(stream)))


def pace_gdn_step_bf16(S, q, k, v, alpha, beta, io, o, n, d_k, d_v, stream=None) -> None:
    _check("pace_gdn_step_bf16", lib.pace_gdn_step_bf16(_ptr(S), _ptr(q), _ptr(k), _ptr(v),
                                                         _ptr(alpha), _ptr(beta), io, _ptr(o), n,
                                                         d_k, d_v, _stream(stream)))


def pace_status_string(status: int) -> str:
    return _status_name(status)


def pace_version() -> str:
    return lib.pace_version().decode()


# ---------------------------------------------------------------- pool owner

class PacePool:
    """Allocates a pool's three device regions with torch and binds them.

    ``state``, ``buffer`` and ``aux`` are uint8 device tensors; their layout is
    the one documented in ``include/pace.h``.
    """

    def __init__(self, B: int, H: int, d_k: int, d_v: int, P: int, head_bits: Sequence[int],
                 axis: str = "col", io: str = "bf16", device="cuda", stream=None,
                 buffer_e4m3: bool = False):
        self.B, self.H, self.d_k, self.d_v, self.P = B, H, d_k, d_v, P
        self.buffer_e4m3 = bool(buffer_e4m3)
        self.head_bits = [int(b) for b in head_bits]
        self.axis = PACE_SCALE_COL if axis == "col" else PACE_SCALE_ROW
        self.io = PACE_IO_BF16 if io == "bf16" else PACE_IO_F32
        self.io_torch = torch.bfloat16 if io == "bf16" else torch.float32
        sb, bb, ab = pace_pool_bytes(B, H, d_k, d_v, P, self.axis, self.io, self.head_bits,
                                     int(self.buffer_e4m3))
        self.state = torch.empty(sb, dtype=torch.uint8, device=device)
        self.buffer = torch.zeros(bb, dtype=torch.uint8, device=device)
        self.aux = torch.empty(ab, dtype=torch.uint8, device=device)
        self.handle = pace_init_pool(B, H, d_k, d_v, P, self.axis, self.io, self.head_bits,
                                     self.state, self.buffer, self.aux, stream, int(self.buffer_e4m3))
        self.slot_stride = pace_pool_layout(self.handle, 0)[2]

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and pace_destroy_pool is not None:   # module globals are gone at interpreter exit
            try:
                pace_destroy_pool(h)
            except Exception:
                pass
            self.handle = None

    # layout helpers -----------------------------------------------------
    def record(self, b: int, h: int) -> torch.Tensor:
        """View of head (b, h)'s record (codes then fp16 scales) in the state region."""
        off, nbytes, stride = pace_pool_layout(self.handle, h)
        start = b * stride + off
        return self.state[start:start + nbytes]

    def fill(self) -> torch.Tensor:
        return self.aux[: 4 * self.B * self.H].view(torch.int32).view(self.B, self.H)

    # calls ----------------------------------------------------------------
    def load(self, S: torch.Tensor, stream=None) -> None:
        pace_pool_load(self.handle, S, stream)

    def export(self, S: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        if S is None:
            S = torch.empty(self.B, self.H, self.d_v, self.d_k, dtype=torch.float32,
                            device=self.state.device)
        pace_pool_export(self.handle, S, stream)
        return S

    def decode_step(self, q, k, v, alpha, beta, o=None, stream=None) -> torch.Tensor:
        if o is None:
            o = torch.empty(self.B, self.H, self.d_v, dtype=torch.float32, device=self.state.device)
        pace_decode_step(self.handle, q, k, v, alpha, beta, o, stream)
        return o

    def commit_period(self, stream=None) -> None:
        pace_commit_period(self.handle, stream)

    def decode_step_range(self, slot_begin, slot_count, q, k, v, alpha, beta, o, blocks_per_sm=0,
                          stream=None) -> torch.Tensor:
        pace_decode_step_range(self.handle, slot_begin, slot_count, blocks_per_sm, q, k, v, alpha,
                               beta, o, stream)
        return o

    def prefill(self, q, k, v, alpha, beta, o=None, stream=None) -> Optional[torch.Tensor]:
        """T tokens [T][B][H][d] through the chunked fp32 prefill; returns o."""
        pace_prefill(self.handle, int(q.shape[0]), q, k, v, alpha, beta, o, stream)
        return o

    def window_step(self, q, k, v, alpha, beta, o=None, stream=None) -> torch.Tensor:
        """One pure-write-window step (window length = P) for every head."""
        if getattr(self, "_wscratch", None) is None:
            self._wscratch = torch.empty(pace_window_scratch_bytes(self.handle), dtype=torch.uint8,
                                         device=self.state.device)
        if o is None:
            o = torch.empty(self.B, self.H, self.d_v, dtype=torch.float32, device=self.state.device)
        pace_window_step(self.handle, q, k, v, alpha, beta, o, self._wscratch, stream)
        return o

    def set_commit_engine(self, engine: int) -> None:
        """PACE_COMMIT_MMA (default) or PACE_COMMIT_TCGEN05 for later commits."""
        pace_set_commit_engine(self.handle, engine)

    def set_commit_threshold(self, tau: float) -> None:
        """Adaptive period: a head is committed early once the Frobenius norm of
        its update since the last rounding reaches tau (inf: fixed period)."""
        pace_set_commit_threshold(self.handle, tau)

    def decode_host(self, q, k, v, alpha, beta, o=None, stream=None) -> None:
        """T decode steps (each followed by the commit of full heads) from host
        tensors [T][B][H][d]; outputs land in the host tensor o (fp32
        [T][B][H][d_v], pinned for full speed) once `stream` completes."""
        if getattr(self, "_staging", None) is None:
            self._staging = torch.empty(pace_host_staging_bytes(self.handle), dtype=torch.uint8,
                                        device=self.state.device)
            self._h2d = torch.cuda.Stream(self.state.device)
            self._d2h = torch.cuda.Stream(self.state.device)
        s = stream if stream is not None else torch.cuda.current_stream(self.state.device)
        pace_decode_host(self.handle, int(q.shape[0]), q, k, v, alpha, beta, o, self._staging, s,
                         self._h2d, self._d2h)

    def commit_period_range(self, slot_begin, slot_count, blocks_per_sm=0, stream=None) -> None:
        pace_commit_period_range(self.handle, slot_begin, slot_count, blocks_per_sm, stream)

    def status(self, stream=None) -> int:
        return pace_pool_status(self.handle, stream)

    def clear_status(self, stream=None) -> None:
        pace_pool_clear_status(self.handle, stream)
