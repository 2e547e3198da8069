"""Python binding of libpa.so, the paged-KV attention library for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA kernels behind the
C ABI declared in include/pa.h; torch tensors supply device memory and streams. The names
mirror the C entry points (pa_plan_create, pa_forward, pa_mla_forward, ...). If libpa.so is
missing the first call raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "PaError", "Plan", "pa_plan_create", "pa_plan_destroy", "pa_plan_get_info", "pa_plan_prepare",
    "pa_forward", "pa_mla_forward", "pa_status_string", "pa_last_error_message", "pa_version",
    "lib_path", "load_library", "PA_PATH_AUTO", "PA_PATH_SIMT", "SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libpa.so")

PA_F32, PA_BF16, PA_F16 = 0, 1, 2
PA_PATH_AUTO, PA_PATH_SIMT = 0, 1
_DTYPES = {torch.float32: PA_F32, torch.bfloat16: PA_BF16, torch.float16: PA_F16}
STATUS = ["PA_OK", "PA_ERR_INVALID_ARGUMENT", "PA_ERR_SHAPE", "PA_ERR_DTYPE", "PA_ERR_BOUNDS",
          "PA_ERR_ALIAS", "PA_ERR_UNSUPPORTED", "PA_ERR_CUDA"]
# every entry point include/pa.h declares
SYMBOLS = ["pa_plan_create", "pa_plan_destroy", "pa_plan_get_info", "pa_plan_prepare", "pa_forward",
           "pa_forward_ex", "pa_forward_static_workspace", "pa_mla_forward", "pa_mla_forward_ex", "pa_append", "pa_backward",
           "pa_mla_backward",
           "pa_plan_device_status", "pa_sparse_select", "pa_sparse_forward", "pa_sparse_forward_ex",
           "pa_status_string", "pa_last_error_message", "pa_version"]
PA_SPARSE_MAX_BLOCKS = 16384
# bits of pa_plan_info.last_kernels
PA_KERNEL_DECODE_TC, PA_KERNEL_PREFILL_TC, PA_KERNEL_MLA_TC, PA_KERNEL_SIMT = 1, 2, 4, 8
PA_KERNEL_MERGE, PA_KERNEL_SPARSE, PA_KERNEL_APPEND, PA_KERNEL_BACKWARD_TC, PA_KERNEL_BACKWARD_SIMT = 16, 32, 64, 128, 256

_P = ctypes.c_void_p
_I = ctypes.c_int32


class PaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.name = STATUS[status] if 0 <= status < len(STATUS) else f"status {status}"
        super().__init__(f"{self.name}: {message}")


class _Options(ctypes.Structure):
    _fields_ = [("kv_chunk", ctypes.c_int32), ("path", ctypes.c_int32), ("trace_events", ctypes.c_void_p)]


class _Info(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_queries", ctypes.c_int32),
                ("table_width", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("device", ctypes.c_int32),
                ("last_launches", ctypes.c_int32), ("workspace_bytes", ctypes.c_int64),
                ("uploaded_bytes", ctypes.c_int64), ("last_kernels", ctypes.c_int32)]


_lib = None


def load_library(path: Optional[str] = None):
    """Load libpa.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or lib_path
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with paged_kv_attention_39_b200/build.py "
                           "(or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(path)
    lib.pa_plan_create.restype = ctypes.c_int
    lib.pa_plan_create.argtypes = [_P, _P, _I, _P, _I, _I, _I, ctypes.c_int, _P, ctypes.POINTER(_P)]
    lib.pa_plan_destroy.restype = ctypes.c_int
    lib.pa_plan_destroy.argtypes = [_P]
    lib.pa_plan_get_info.restype = ctypes.c_int
    lib.pa_plan_get_info.argtypes = [_P, ctypes.POINTER(_Info)]
    lib.pa_plan_prepare.restype = ctypes.c_int
    lib.pa_plan_prepare.argtypes = [_P, ctypes.c_int, ctypes.c_int, _I, _I, _I, _I, ctypes.c_int, _I, _P,
                                    ctypes.POINTER(_Options)]
    fwd = [_P, _P, _P, _P, ctypes.c_int, _I, _I, _I, _I, ctypes.c_float, ctypes.c_int, _I, _P, _P, _P]
    lib.pa_forward.restype = ctypes.c_int
    lib.pa_forward.argtypes = fwd
    lib.pa_forward_ex.restype = ctypes.c_int
    lib.pa_forward_ex.argtypes = fwd + [ctypes.POINTER(_Options)]
    mla = [_P, _P, _P, _P, _P, ctypes.c_int, _I, _I, _I, ctypes.c_float, ctypes.c_int, _I, _P, _P, _P]
    lib.pa_mla_forward.restype = ctypes.c_int
    lib.pa_mla_forward.argtypes = mla
    lib.pa_mla_forward_ex.restype = ctypes.c_int
    lib.pa_mla_forward_ex.argtypes = mla + [ctypes.POINTER(_Options)]
    lib.pa_forward_static_workspace.restype = ctypes.c_int
    lib.pa_forward_static_workspace.argtypes = [_P, _P, _P, _P, ctypes.c_int, _I, _I, _I, _I, ctypes.c_float,
                                                ctypes.c_int, _I, _I, _P, _P, _P]
    lib.pa_append.restype = ctypes.c_int
    lib.pa_append.argtypes = [_P, _P, _P, _P, _P, ctypes.c_int, _I, _I, _I, _P]
    lib.pa_backward.restype = ctypes.c_int
    lib.pa_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _I, _I, _I, _I, ctypes.c_float, ctypes.c_int,
                                _I, _P, _P, _P, _P]
    lib.pa_mla_backward.restype = ctypes.c_int
    lib.pa_mla_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _I, _I, _I, ctypes.c_float,
                                    ctypes.c_int, _I, _P, _P, _P, _P, _P]
    lib.pa_plan_device_status.restype = ctypes.c_int
    lib.pa_plan_device_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int32)]
    lib.pa_sparse_select.restype = ctypes.c_int
    lib.pa_sparse_select.argtypes = [_P, _P, _P, ctypes.c_int, _I, _I, _I, ctypes.c_float, ctypes.c_int, _I, _I, _I,
                                     _P, _I, _P, _I, _P]
    lib.pa_sparse_forward.restype = ctypes.c_int
    lib.pa_sparse_forward.argtypes = [_P, _P, _P, _P, ctypes.c_int, _I, _I, _I, _I, ctypes.c_float, ctypes.c_int, _I,
                                      _I, _P, _I, _P, _P, _P]
    lib.pa_sparse_forward_ex.restype = ctypes.c_int
    lib.pa_sparse_forward_ex.argtypes = lib.pa_sparse_forward.argtypes + [ctypes.POINTER(_Options)]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_status_string.argtypes = [ctypes.c_int]
    lib.pa_last_error_message.restype = ctypes.c_char_p
    lib.pa_last_error_message.argtypes = []
    lib.pa_version.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    if path == lib_path:
        _lib = lib
    return lib


def _check(st: int) -> None:
    if st != 0:
        raise PaError(st, load_library().pa_last_error_message().decode())


def _stream_ptr(stream, device) -> Optional[int]:
    if stream is None:
        if device is None or device < 0 or not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream(device)
    return int(getattr(stream, "cuda_stream", stream)) or None


def _i32(x) -> torch.Tensor:
    return torch.as_tensor(x, dtype=torch.int32).detach().cpu().contiguous()


def pa_status_string(status: int) -> str:
    return load_library().pa_status_string(status).decode()


def pa_last_error_message() -> str:
    return load_library().pa_last_error_message().decode()


def pa_version() -> str:
    return load_library().pa_version().decode()


class Plan:
    """Owner of a pa_plan handle (destroyed with the object)."""

    def __init__(self, handle: int, num_queries: int, device: int, host: tuple):
        self.handle = handle
        self.num_queries = num_queries
        self.device = device
        self._host = host  # keeps the host arrays of the upload alive

    def close(self) -> None:
        if self.handle:
            _check(load_library().pa_plan_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def pa_plan_create(seq_lens, query_offsets, block_tables, page_size: int, num_pages: int,
                   device: Optional[int] = None, stream=None) -> Plan:
    """Validate a schedule and upload it once; device=-1 makes a host-only plan."""
    lib = load_library()
    sl, qo, bt = _i32(seq_lens), _i32(query_offsets), _i32(block_tables)
    if bt.dim() == 1:
        bt = bt.view(max(1, sl.numel()), -1) if bt.numel() else bt.view(sl.numel(), 0)
    if device is None:
        device = torch.cuda.current_device() if torch.cuda.is_available() else -1
    handle = _P()
    st = lib.pa_plan_create(sl.data_ptr() if sl.numel() else None, qo.data_ptr(), sl.numel(),
                            bt.data_ptr() if bt.numel() else None, bt.shape[1] if bt.dim() == 2 else 0,
                            int(page_size), int(num_pages), int(device), _stream_ptr(stream, device),
                            ctypes.byref(handle))
    _check(st)
    return Plan(handle.value, int(qo[-1]), int(device), (sl, qo, bt))


def pa_plan_destroy(plan: Plan) -> None:
    plan.close()


def pa_plan_get_info(plan: Plan) -> dict:
    info = _Info()
    _check(load_library().pa_plan_get_info(plan.handle, ctypes.byref(info)))
    return {k: getattr(info, k) for k, _ in _Info._fields_}


def pa_plan_device_status(plan: Plan) -> int:
    """Diagnostic: the plan's device error word (0 = no kernel reported a failure)."""
    code = ctypes.c_int32(0)
    _check(load_library().pa_plan_device_status(plan.handle, ctypes.byref(code)))
    return int(code.value)


def _opts(kv_chunk: int, path: int, trace=None):
    """Options struct; `trace` is a ctypes array of three cudaEvent_t handles, or None."""
    ev = ctypes.cast(trace, ctypes.c_void_p) if trace is not None else None
    return ctypes.byref(_Options(int(kv_chunk), int(path), ev))


def trace_events(events):
    """Three torch.cuda.Event objects -> the array pa_forward_options.trace_events takes.

    torch creates the CUDA event behind an Event lazily, on its first record: record each one
    once here so that the handles exist.
    """
    for e in events:
        if not e.cuda_event:
            e.record()
    return (ctypes.c_void_p * 3)(*[int(e.cuda_event) for e in events])


def pa_plan_prepare(plan: Plan, dtype: torch.dtype, num_q_heads: int, num_kv_heads: int,
                    head_dim: int, v_head_dim: int, causal: bool = True, window: int = 0,
                    mla: bool = False, stream=None, kv_chunk: int = 0, path: int = PA_PATH_AUTO) -> None:
    _check(load_library().pa_plan_prepare(plan.handle, int(mla), _DTYPES[dtype], num_q_heads,
                                          num_kv_heads, head_dim, v_head_dim, int(bool(causal)),
                                          int(window), _stream_ptr(stream, plan.device),
                                          _opts(kv_chunk, path)))


def _ptr(t: Optional[torch.Tensor]):
    return t.data_ptr() if t is not None else None


def pa_forward(plan: Plan, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
               out: torch.Tensor, lse: torch.Tensor, scale: float, causal: bool = True,
               window: int = 0, stream=None, kv_chunk: int = 0, path: int = PA_PATH_AUTO,
               trace=None) -> None:
    """q [Nq, Hq, D], k_cache [P, ps, Hkv, D], v_cache [P, ps, Hkv, Dv] -> out, lse (in place)."""
    for t in (q, k_cache, v_cache, out, lse):
        if not t.is_contiguous():
            raise ValueError("pa_forward takes contiguous tensors")
    if lse.dtype != torch.float32:
        raise ValueError("lse must be float32")
    _check(load_library().pa_forward_ex(
        plan.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), _DTYPES[q.dtype], q.shape[1],
        k_cache.shape[2], q.shape[2], v_cache.shape[3], float(scale), int(bool(causal)), int(window),
        _ptr(out), _ptr(lse), _stream_ptr(stream, plan.device), _opts(kv_chunk, path, trace)))


def pa_sparse_select(plan: Plan, q: torch.Tensor, k_cache: torch.Tensor, selection: torch.Tensor, scale: float,
                     block_size: int, topk: int, causal: bool = True, window: int = 0,
                     block_scores: Optional[torch.Tensor] = None, num_q_heads: Optional[int] = None,
                     stream=None) -> None:
    """Proxy block scores and top-K selection: selection [Nq, Hkv, width] int32 (in place), and
    block_scores [Nq, Hkv, scores_width] float32 when given."""
    for t in (q, k_cache, selection) + ((block_scores,) if block_scores is not None else ()):
        if not t.is_contiguous():
            raise ValueError("pa_sparse_select takes contiguous tensors")
    if selection.dtype != torch.int32:
        raise ValueError("selection must be int32")
    if block_scores is not None and block_scores.dtype != torch.float32:
        raise ValueError("block_scores must be float32")
    _check(load_library().pa_sparse_select(
        plan.handle, _ptr(q), _ptr(k_cache), _DTYPES[q.dtype], num_q_heads or q.shape[1], k_cache.shape[2],
        q.shape[2], float(scale), int(bool(causal)), int(window), int(block_size), int(topk), _ptr(selection),
        selection.shape[2], _ptr(block_scores), block_scores.shape[2] if block_scores is not None else 0,
        _stream_ptr(stream, plan.device)))


def pa_sparse_forward(plan: Plan, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      selection: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, scale: float, block_size: int,
                      causal: bool = True, window: int = 0, stream=None, kv_chunk: int = 0,
                      path: int = PA_PATH_AUTO, trace=None) -> None:
    """Attention over the blocks in selection [Nq, Hkv, width] int32 -> out, lse (in place)."""
    for t in (q, k_cache, v_cache, selection, out, lse):
        if not t.is_contiguous():
            raise ValueError("pa_sparse_forward takes contiguous tensors")
    if lse.dtype != torch.float32 or selection.dtype != torch.int32:
        raise ValueError("lse must be float32 and selection int32")
    _check(load_library().pa_sparse_forward_ex(
        plan.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), _DTYPES[q.dtype], q.shape[1], k_cache.shape[2],
        q.shape[2], v_cache.shape[3], float(scale), int(bool(causal)), int(window), int(block_size),
        _ptr(selection), selection.shape[2], _ptr(out), _ptr(lse), _stream_ptr(stream, plan.device),
        _opts(kv_chunk, path, trace)))


def pa_append(plan: Plan, new_k: torch.Tensor, new_v: torch.Tensor, k_cache: torch.Tensor,
              v_cache: torch.Tensor, stream=None) -> None:
    """Write new_k [Nq, Hkv, D] / new_v [Nq, Hkv, Dv] into the plan's cache slots (in place)."""
    for t in (new_k, new_v, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("pa_append takes contiguous tensors")
    _check(load_library().pa_append(plan.handle, _ptr(new_k), _ptr(new_v), _ptr(k_cache), _ptr(v_cache),
                                    _DTYPES[new_k.dtype], k_cache.shape[2], k_cache.shape[3], v_cache.shape[3],
                                    _stream_ptr(stream, plan.device)))


def pa_mla_backward(plan: Plan, q_latent: torch.Tensor, q_rope: torch.Tensor, latent_cache: torch.Tensor,
                    rope_cache: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, d_out: torch.Tensor,
                    d_q_latent: torch.Tensor, d_q_rope: torch.Tensor, d_latent_cache: torch.Tensor,
                    d_rope_cache: torch.Tensor, scale: float, causal: bool = True, window: int = 0,
                    stream=None) -> None:
    """Gradients of pa_mla_forward: d_q_latent / d_q_rope written, d_latent_cache / d_rope_cache
    (float32) accumulated."""
    ts = (q_latent, q_rope, latent_cache, rope_cache, out, lse, d_out, d_q_latent, d_q_rope, d_latent_cache,
          d_rope_cache)
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("pa_mla_backward takes contiguous tensors")
    _check(load_library().pa_mla_backward(
        plan.handle, _ptr(q_latent), _ptr(q_rope), _ptr(latent_cache), _ptr(rope_cache), _ptr(out), _ptr(lse),
        _ptr(d_out), _DTYPES[q_latent.dtype], q_latent.shape[1], q_latent.shape[2], q_rope.shape[2], float(scale),
        int(bool(causal)), int(window), _ptr(d_q_latent), _ptr(d_q_rope), _ptr(d_latent_cache), _ptr(d_rope_cache),
        _stream_ptr(stream, plan.device)))


def pa_backward(plan: Plan, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, out: torch.Tensor,
                lse: torch.Tensor, d_out: torch.Tensor, d_q: torch.Tensor, d_k_cache: torch.Tensor,
                d_v_cache: torch.Tensor, scale: float, causal: bool = True, window: int = 0, stream=None) -> None:
    """Gradients of pa_forward: d_q written, d_k_cache / d_v_cache (float32) accumulated."""
    for t in (q, k_cache, v_cache, out, lse, d_out, d_q, d_k_cache, d_v_cache):
        if not t.is_contiguous():
            raise ValueError("pa_backward takes contiguous tensors")
    _check(load_library().pa_backward(
        plan.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), _ptr(d_out), _DTYPES[q.dtype],
        q.shape[1], k_cache.shape[2], q.shape[2], v_cache.shape[3], float(scale), int(bool(causal)), int(window),
        _ptr(d_q), _ptr(d_k_cache), _ptr(d_v_cache), _stream_ptr(stream, plan.device)))


def pa_forward_static_workspace(plan: Plan, q: torch.Tensor, k_cache: torch.Tensor,
                                v_cache: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, scale: float,
                                causal: bool = True, window: int = 0, kv_chunk: int = 0, stream=None) -> None:
    """Split-KV decode that allocates no memory: scratch in the library's fixed device array
    (for callers that cannot allocate while attention runs; see include/pa.h)."""
    for t in (q, k_cache, v_cache, out, lse):
        if not t.is_contiguous():
            raise ValueError("pa_forward_static_workspace takes contiguous tensors")
    _check(load_library().pa_forward_static_workspace(
        plan.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), _DTYPES[q.dtype], q.shape[1], k_cache.shape[2],
        q.shape[2], v_cache.shape[3], float(scale), int(bool(causal)), int(window), int(kv_chunk), _ptr(out),
        _ptr(lse), _stream_ptr(stream, plan.device)))


def pa_mla_forward(plan: Plan, q_latent: torch.Tensor, q_rope: torch.Tensor,
                   latent_cache: torch.Tensor, rope_cache: torch.Tensor, out: torch.Tensor,
                   lse: torch.Tensor, scale: float, causal: bool = True, window: int = 0,
                   stream=None, kv_chunk: int = 0, path: int = PA_PATH_AUTO, trace=None) -> None:
    """MLA: q_latent [Nq, H, R], q_rope [Nq, H, P], latent [pages, ps, 1, R], rope [.., 1, P]."""
    for t in (q_latent, q_rope, latent_cache, rope_cache, out, lse):
        if not t.is_contiguous():
            raise ValueError("pa_mla_forward takes contiguous tensors")
    _check(load_library().pa_mla_forward_ex(
        plan.handle, _ptr(q_latent), _ptr(q_rope), _ptr(latent_cache), _ptr(rope_cache),
        _DTYPES[q_latent.dtype], q_latent.shape[1], q_latent.shape[2], q_rope.shape[2], float(scale),
        int(bool(causal)), int(window), _ptr(out), _ptr(lse), _stream_ptr(stream, plan.device),
        _opts(kv_chunk, path, trace)))


def plan_for(wl, device: Optional[int] = None, stream=None) -> Plan:
    """pa_plan_create from a workload object of the seeded input module."""
    s = wl.sched
    return pa_plan_create(s.seq_lens, s.query_offsets, s.block_tables, s.page_size, s.num_pages,
                          device=device, stream=stream)
