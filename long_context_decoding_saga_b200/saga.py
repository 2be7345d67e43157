"""Python binding of libsaga (the C ABI in include/saga.h).

Argument marshalling only: each function checks tensor dtypes, shapes and
devices, passes raw device pointers and the current CUDA stream to the
library, and turns a negative return code into SagaError.  Every step of the
decode path runs in the library's CUDA kernels; there is no fallback.  If
libsaga.so has not been built this module raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsaga.so")

SAGA_OK = 0
SAGA_ERR_ARG = -1
SAGA_ERR_UNSUPPORTED = -2
SAGA_ERR_WORKSPACE = -3
SAGA_ERR_CUDA = -4
SAGA_OUT_F32 = 0
SAGA_OUT_BF16 = 1
SAGA_STATUS_LEN_CLAMPED = 0x1
SAGA_STATUS_TIMEOUT = 0x2

EXPORTED = ("saga_workspace_bytes", "saga_kv_append", "atopn_refresh_threshold", "atopn_select_workspace_bytes",
            "atopn_select_threshold", "saga_decode_attn", "saga_trace_next_attention", "saga_get_status", "saga_last_error", "saga_abi_version",
            "saga_noalloc_scratch_bytes", "saga_decode_attn_noalloc", "saga_noalloc_get_status",
            "saga_noalloc_last_error", "saga_decode_step", "saga_test_expire_next_wait", "saga_read_probe_sink_words",
            "saga_read_probe", "saga_merge_workspace_bytes", "saga_key_head_merge", "saga_merge_last_error",
            "saga_qkv_project", "saga_qkv_workspace_bytes")


class SagaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libsaga error {code}: {msg}")
        self.code = code


class SagaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("h_q", ctypes.c_int), ("h_k", ctypes.c_int), ("h_v", ctypes.c_int),
                ("d", ctypes.c_int), ("l_cap", ctypes.c_int)]

    @classmethod
    def of(cls, batch, h_q, h_k, h_v, d, l_cap) -> "SagaShape":
        return cls(int(batch), int(h_q), int(h_k), int(h_v), int(d), int(l_cap))

    def astuple(self):
        return (self.batch, self.h_q, self.h_k, self.h_v, self.d, self.l_cap)


class SagaMergeShape(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int), ("hidden", ctypes.c_int), ("d", ctypes.c_int), ("h_q", ctypes.c_int),
                ("h_k", ctypes.c_int)]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def load(path: Optional[str] = None):
    """Load libsaga.so (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with long_context_decoding_saga_b200.build.build()")
    lib = ctypes.CDLL(path)
    sp = ctypes.POINTER(SagaShape)
    lib.saga_workspace_bytes.argtypes = [sp]
    lib.saga_workspace_bytes.restype = ctypes.c_size_t
    lib.saga_kv_append.argtypes = [sp, _P, _P, _P, _P, _I, _P, _P]
    lib.saga_kv_append.restype = _I
    lib.saga_qkv_project.argtypes = [sp, _I, _P, _P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t, _P]
    lib.saga_qkv_project.restype = _I
    lib.saga_qkv_workspace_bytes.argtypes = [sp, _I]
    lib.saga_qkv_workspace_bytes.restype = ctypes.c_size_t
    lib.atopn_refresh_threshold.argtypes = [sp, _P, _P, _I, _P, _I, _P, _P, ctypes.c_size_t, _P]
    lib.atopn_refresh_threshold.restype = _I
    lib.atopn_select_workspace_bytes.argtypes = [_I]
    lib.atopn_select_workspace_bytes.restype = ctypes.c_size_t
    lib.atopn_select_threshold.argtypes = [_P, _I, _I, ctypes.c_longlong, _I, _P, _P, ctypes.c_size_t, _P]
    lib.atopn_select_threshold.restype = _I
    lib.saga_decode_attn.argtypes = [sp, _P, _P, _P, _I, _P, _I, _I, ctypes.c_longlong, _P, _P, _I, _P, _P, _P,
                                     ctypes.c_size_t, _P]
    lib.saga_decode_attn.restype = _I
    lib.saga_decode_step.argtypes = [sp, _P, _P, _P, _P, _P, _I, _P, _I, _I, ctypes.c_longlong, _P, _P, _I, _P, _P,
                                     _P, ctypes.c_size_t, _P]
    lib.saga_decode_step.restype = _I
    lib.saga_trace_next_attention.argtypes = [_P, _P]
    lib.saga_trace_next_attention.restype = _I
    lib.saga_get_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint)]
    lib.saga_get_status.restype = _I
    lib.saga_last_error.argtypes = []
    lib.saga_last_error.restype = ctypes.c_char_p
    lib.saga_abi_version.argtypes = []
    lib.saga_abi_version.restype = _I
    lib.saga_noalloc_scratch_bytes.argtypes = []
    lib.saga_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.saga_decode_attn_noalloc.argtypes = [sp, _P, _P, _P, _I, _P, _I, _I, ctypes.c_longlong, _P, _P, _I, _P, _P,
                                             _P]
    lib.saga_decode_attn_noalloc.restype = _I
    lib.saga_noalloc_get_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint)]
    lib.saga_noalloc_get_status.restype = _I
    lib.saga_test_expire_next_wait.argtypes = [ctypes.c_uint]
    lib.saga_test_expire_next_wait.restype = _I
    mp = ctypes.POINTER(SagaMergeShape)
    lib.saga_merge_workspace_bytes.argtypes = [mp]
    lib.saga_merge_workspace_bytes.restype = ctypes.c_size_t
    lib.saga_key_head_merge.argtypes = [mp, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    lib.saga_key_head_merge.restype = _I
    lib.saga_merge_last_error.argtypes = []
    lib.saga_merge_last_error.restype = ctypes.c_char_p
    lib.saga_read_probe_sink_words.argtypes = []
    lib.saga_read_probe_sink_words.restype = ctypes.c_size_t
    lib.saga_read_probe.argtypes = [_P, ctypes.c_size_t, _P, _P]
    lib.saga_read_probe.restype = _I
    lib.saga_noalloc_last_error.argtypes = []
    lib.saga_noalloc_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(rc: int):
    if rc != SAGA_OK:
        raise SagaError(rc, load().saga_last_error().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _expect(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def abi_version() -> int:
    return load().saga_abi_version()


def saga_workspace_bytes(shape: SagaShape) -> int:
    n = load().saga_workspace_bytes(ctypes.byref(shape))
    if n == 0:
        raise SagaError(SAGA_ERR_ARG, load().saga_last_error().decode(errors="replace"))
    return int(n)


def alloc_workspace(shape: SagaShape, device=None) -> torch.Tensor:
    """Zero-filled workspace of saga_workspace_bytes(shape) bytes on `device`."""
    return torch.zeros(saga_workspace_bytes(shape), dtype=torch.uint8, device=device or "cuda")


def saga_kv_append(shape: SagaShape, k_cache, v_cache, k_new, v_new, pos: int, seq_len_dev=None, stream=None):
    B, hq, hk, hv, d, lc = shape.astuple()
    _expect(k_cache, "k_cache", torch.bfloat16, (B, hk, lc, d))
    _expect(v_cache, "v_cache", torch.bfloat16, (B, hv, lc, d))
    _expect(k_new, "k_new", torch.bfloat16, (B, hk, d))
    _expect(v_new, "v_new", torch.bfloat16, (B, hv, d))
    if seq_len_dev is not None:
        _expect(seq_len_dev, "seq_len_dev", torch.int32)
    _check(load().saga_kv_append(ctypes.byref(shape), _ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new),
                                 int(pos), _ptr(seq_len_dev), _stream(stream)))


def saga_qkv_workspace_bytes(shape: SagaShape, hidden: int) -> int:
    n = load().saga_qkv_workspace_bytes(ctypes.byref(shape), int(hidden))
    if n == 0:
        raise SagaError(SAGA_ERR_ARG, load().saga_last_error().decode(errors="replace"))
    return int(n)


def alloc_qkv_workspace(shape: SagaShape, hidden: int, device=None) -> torch.Tensor:
    """Zero-filled workspace of saga_qkv_workspace_bytes(shape, hidden) bytes on `device`."""
    return torch.zeros(saga_qkv_workspace_bytes(shape, hidden), dtype=torch.uint8, device=device or "cuda")


def saga_qkv_project(shape: SagaShape, x, w_qkv, q_out, k_cache, v_cache, pos: int, workspace=None,
                     seq_len_dev=None, stream=None):
    """Eq. 1 for the new token: q_out = x W_Q, and x W_K, x W_V written into row pos of the caches.
    Returns the workspace (a fresh zero-filled one when none is passed)."""
    B, hq, hk, hv, d, lc = shape.astuple()
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise SagaError(SAGA_ERR_ARG, "x must be a 2-D tensor [batch, hidden]")
    D = int(x.shape[1])
    _expect(x, "x", torch.bfloat16, (B, D))
    _expect(w_qkv, "w_qkv", torch.bfloat16, ((hq + hk + hv) * d, D))
    _expect(q_out, "q_out", torch.bfloat16, (B, hq, d))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, hk, lc, d))
    _expect(v_cache, "v_cache", torch.bfloat16, (B, hv, lc, d))
    if seq_len_dev is not None:
        _expect(seq_len_dev, "seq_len_dev", torch.int32)
    if workspace is None:
        n = load().saga_qkv_workspace_bytes(ctypes.byref(shape), D)
        if n:  # else the call below reports why
            workspace = torch.zeros(n, dtype=torch.uint8, device=x.device)
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8)
    _check(load().saga_qkv_project(ctypes.byref(shape), D, _ptr(x), _ptr(w_qkv), _ptr(q_out), _ptr(k_cache),
                                   _ptr(v_cache), int(pos), _ptr(seq_len_dev), _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(stream)))
    return workspace


def atopn_refresh_threshold(shape: SagaShape, q, k_cache, seq_len: int, n_top: int, tau, workspace,
                            seq_len_dev=None, stream=None):
    B, hq, hk, hv, d, lc = shape.astuple()
    _expect(q, "q", torch.bfloat16, (B, hq, d))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, hk, lc, d))
    _expect(tau, "tau", torch.float32, (B, hq))
    _expect(workspace, "workspace", torch.uint8)
    if seq_len_dev is not None:
        _expect(seq_len_dev, "seq_len_dev", torch.int32)
    _check(load().atopn_refresh_threshold(ctypes.byref(shape), _ptr(q), _ptr(k_cache), int(seq_len),
                                          _ptr(seq_len_dev), int(n_top), _ptr(tau), _ptr(workspace),
                                          workspace.numel(), _stream(stream)))


def atopn_select_threshold(scores, row_len: int, n_top: int, tau, workspace, stream=None):
    """tau[r] = n_top-th largest of scores[r, :row_len] (scores: fp32 [rows, row_stride])."""
    _expect(scores, "scores", torch.float32)
    if scores.dim() != 2:
        raise ValueError("scores must be 2-D [rows, row_stride]")
    rows, stride = scores.shape
    _expect(tau, "tau", torch.float32, (rows,))
    _expect(workspace, "workspace", torch.uint8)
    _check(load().atopn_select_threshold(_ptr(scores), int(rows), int(row_len), int(stride), int(n_top), _ptr(tau),
                                         _ptr(workspace), workspace.numel(), _stream(stream)))


def saga_decode_attn(shape: SagaShape, q, k_cache, v_cache, seq_len: int, n_top: int, refresh_interval: int, step: int,
                     tau, out, workspace, sel_count=None, sel_idx=None, seq_len_dev=None, stream=None):
    B, hq, hk, hv, d, lc = shape.astuple()
    _expect(q, "q", torch.bfloat16, (B, hq, d))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, hk, lc, d))
    _expect(v_cache, "v_cache", torch.bfloat16, (B, hv, lc, d))
    _expect(tau, "tau", torch.float32, (B, hq))
    if out.dtype == torch.float32:
        out_dtype = SAGA_OUT_F32
    elif out.dtype == torch.bfloat16:
        out_dtype = SAGA_OUT_BF16
    else:
        raise TypeError("out must be float32 or bfloat16")
    _expect(out, "out", out.dtype, (B, hq, d))
    _expect(workspace, "workspace", torch.uint8)
    if sel_count is not None:
        _expect(sel_count, "sel_count", torch.int32, (B, hq))
    if sel_idx is not None:
        _expect(sel_idx, "sel_idx", torch.int32, (B, hq, lc))
    if seq_len_dev is not None:
        _expect(seq_len_dev, "seq_len_dev", torch.int32)
    _check(load().saga_decode_attn(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), int(seq_len),
                                   _ptr(seq_len_dev), int(n_top), int(refresh_interval), int(step), _ptr(tau),
                                   _ptr(out), out_dtype, _ptr(sel_count), _ptr(sel_idx), _ptr(workspace),
                                   workspace.numel(), _stream(stream)))


def saga_decode_step(shape: SagaShape, q, k_new, v_new, k_cache, v_cache, seq_len: int, n_top: int,
                     refresh_interval: int, step: int, tau, out, workspace, sel_count=None, sel_idx=None,
                     seq_len_dev=None, stream=None):
    """saga_kv_append at seq_len - 1 and saga_decode_attn, with the append done inside the attention kernels."""
    B, hq, hk, hv, d, lc = shape.astuple()
    _expect(q, "q", torch.bfloat16, (B, hq, d))
    _expect(k_new, "k_new", torch.bfloat16, (B, hk, d))
    _expect(v_new, "v_new", torch.bfloat16, (B, hv, d))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, hk, lc, d))
    _expect(v_cache, "v_cache", torch.bfloat16, (B, hv, lc, d))
    _expect(tau, "tau", torch.float32, (B, hq))
    if out.dtype == torch.float32:
        out_dtype = SAGA_OUT_F32
    elif out.dtype == torch.bfloat16:
        out_dtype = SAGA_OUT_BF16
    else:
        raise TypeError("out must be float32 or bfloat16")
    _expect(out, "out", out.dtype, (B, hq, d))
    _expect(workspace, "workspace", torch.uint8)
    if sel_count is not None:
        _expect(sel_count, "sel_count", torch.int32, (B, hq))
    if sel_idx is not None:
        _expect(sel_idx, "sel_idx", torch.int32, (B, hq, lc))
    if seq_len_dev is not None:
        _expect(seq_len_dev, "seq_len_dev", torch.int32)
    _check(load().saga_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                   _ptr(v_cache), int(seq_len), _ptr(seq_len_dev), int(n_top), int(refresh_interval),
                                   int(step), _ptr(tau), _ptr(out), out_dtype, _ptr(sel_count), _ptr(sel_idx),
                                   _ptr(workspace), workspace.numel(), _stream(stream)))


def saga_trace_next_attention(ev_start: Optional[torch.cuda.Event], ev_end: Optional[torch.cuda.Event]):
    """Bracket the attention kernels of the next saga_decode_attn call on this thread with two CUDA events."""
    if ev_start is None or ev_end is None:
        _check(load().saga_trace_next_attention(None, None))
        return
    for ev in (ev_start, ev_end):
        if ev.cuda_event == 0:  # torch creates the event on first record
            ev.record()
    _check(load().saga_trace_next_attention(ctypes.c_void_p(ev_start.cuda_event), ctypes.c_void_p(ev_end.cuda_event)))


def saga_decode_attn_noalloc(shape: SagaShape, q, k_cache, v_cache, seq_len: int, n_top: int, refresh_interval: int,
                             step: int, tau, out, sel_count=None, sel_idx=None, seq_len_dev=None, stream=None):
    """saga_decode_attn with the library's built-in scratch instead of a caller workspace (allocates nothing)."""
    B, hq, hk, hv, d, lc = shape.astuple()
    _expect(q, "q", torch.bfloat16, (B, hq, d))
    _expect(k_cache, "k_cache", torch.bfloat16, (B, hk, lc, d))
    _expect(v_cache, "v_cache", torch.bfloat16, (B, hv, lc, d))
    _expect(tau, "tau", torch.float32, (B, hq))
    if out.dtype == torch.float32:
        out_dtype = SAGA_OUT_F32
    elif out.dtype == torch.bfloat16:
        out_dtype = SAGA_OUT_BF16
    else:
        raise TypeError("out must be float32 or bfloat16")
    _expect(out, "out", out.dtype, (B, hq, d))
    if sel_count is not None:
        _expect(sel_count, "sel_count", torch.int32, (B, hq))
    if sel_idx is not None:
        _expect(sel_idx, "sel_idx", torch.int32, (B, hq, lc))
    if seq_len_dev is not None:
        _expect(seq_len_dev, "seq_len_dev", torch.int32)
    lib = load()
    rc = lib.saga_decode_attn_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), int(seq_len),
                                      _ptr(seq_len_dev), int(n_top), int(refresh_interval), int(step), _ptr(tau),
                                      _ptr(out), out_dtype, _ptr(sel_count), _ptr(sel_idx), _stream(stream))
    if rc != SAGA_OK:
        raise SagaError(rc, lib.saga_noalloc_last_error().decode(errors="replace"))


def saga_noalloc_get_status(stream=None) -> int:
    """Status word (SAGA_STATUS_* bits) of the last saga_decode_attn_noalloc call on the current device."""
    lib = load()
    v = ctypes.c_uint(0)
    rc = lib.saga_noalloc_get_status(_stream(stream), ctypes.byref(v))
    if rc != SAGA_OK:
        raise SagaError(rc, lib.saga_noalloc_last_error().decode(errors="replace"))
    return int(v.value)


def saga_test_expire_next_wait(limit_ns: int):
    """Test hook: the next decode call's keep kernel (a sparse reuse step) waits on a barrier nothing arrives
    at, for at most limit_ns, then unwinds and flags SAGA_STATUS_TIMEOUT (0 cancels)."""
    _check(load().saga_test_expire_next_wait(int(limit_ns)))


def key_head_merge(x, q, w_k, h_k: int, workspace=None, stream=None):
    """The closed-form GQA-to-SAGA key-head merge (saga_key_head_merge).  x: bf16 [T, D], q: bf16 [T, h_q, d],
    w_k: fp32 [h_k, D, d].  Returns (pair_loss fp32 [h_k, h_k], pairing int32 [h_k], merged fp32
    [h_k / 2, D, d], workspace)."""
    _expect(x, "x", torch.bfloat16)
    _expect(q, "q", torch.bfloat16)
    _expect(w_k, "w_k", torch.float32)
    T, D = x.shape
    h_q, d = q.shape[1], q.shape[2]
    if tuple(q.shape) != (T, h_q, d) or tuple(w_k.shape) != (h_k, D, d):
        raise ValueError("shapes: x [T, D], q [T, h_q, d], w_k [h_k, D, d]")
    shape = SagaMergeShape(int(T), int(D), int(d), int(h_q), int(h_k))
    lib = load()
    need = lib.saga_merge_workspace_bytes(ctypes.byref(shape))
    if need == 0:
        raise SagaError(SAGA_ERR_ARG, lib.saga_merge_last_error().decode(errors="replace"))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    loss = torch.empty((h_k, h_k), dtype=torch.float32, device=x.device)
    pairing = torch.empty(h_k, dtype=torch.int32, device=x.device)
    merged = torch.empty((h_k // 2, D, d), dtype=torch.float32, device=x.device)
    rc = lib.saga_key_head_merge(ctypes.byref(shape), _ptr(x), _ptr(q), _ptr(w_k), _ptr(loss), _ptr(pairing),
                                 _ptr(merged), _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != SAGA_OK:
        raise SagaError(rc, lib.saga_merge_last_error().decode(errors="replace"))
    return loss, pairing, merged, workspace


def read_probe(buf: torch.Tensor, sink: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One streaming read of buf (any CUDA tensor, 16-byte aligned) by the library's pure-read probe kernel;
    returns the sink tensor it writes (pass it back in to reuse it)."""
    if not buf.is_cuda:
        raise ValueError("buf must be a CUDA tensor")
    lib = load()
    if sink is None:
        sink = torch.empty(int(lib.saga_read_probe_sink_words()), dtype=torch.int32, device=buf.device)
    rc = lib.saga_read_probe(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink), _stream(stream))
    if rc != SAGA_OK:
        raise SagaError(rc, "saga_read_probe failed")
    return sink


def saga_get_status(workspace, stream=None) -> int:
    _expect(workspace, "workspace", torch.uint8)
    v = ctypes.c_uint(0)
    _check(load().saga_get_status(_ptr(workspace), _stream(stream), ctypes.byref(v)))
    return int(v.value)
