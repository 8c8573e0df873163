"""ctypes binding of libsinkattn.so (include/sink_attn.h).

Argument marshalling only: shapes and pointers of torch CUDA tensors go in,
the C-ABI entry points do all the work on the current (or given) stream.
There is no CPU fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsinkattn.so")
_lib = None

STATUS = {
    0: "SINK_ATTN_OK",
    1: "SINK_ATTN_ERR_NULL",
    2: "SINK_ATTN_ERR_SHAPE",
    3: "SINK_ATTN_ERR_ALIGN",
    4: "SINK_ATTN_ERR_UNSUPPORTED",
    5: "SINK_ATTN_ERR_CUDA",
    6: "SINK_ATTN_ERR_DEVICE_TIMEOUT",
    7: "SINK_ATTN_ERR_WORKSPACE",
}

EXPORTS = ("sink_attn_fwd", "sink_attn_fwd_pair", "sink_attn_fwd_with", "sink_attn_fwd_kernel_for", "sink_attn_bwd", "sink_attn_bwd_workspace_size", "sink_attn_status_string",
           "sink_attn_last_device_error", "sink_attn_device_error", "sink_attn_fwd_launches", "sink_attn_bwd_launches", "sink_attn_profile_events",
           "sink_attn_decode", "sink_attn_decode_workspace_size", "sink_attn_decode_launches",
           "sink_attn_decode_e4m3", "sink_attn_decode_e4m3_f8pv", "sink_attn_selftest_wait")


class SinkAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("max_seqlen", ctypes.c_int), ("total_tokens", ctypes.c_int),
                ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int)]


class DecodeDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("new_tokens", ctypes.c_int), ("cache_capacity", ctypes.c_int),
                ("max_seqlen", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int)]


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Loads libsinkattn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libsinkattn.so not found at {_LIB_PATH}; build it with "
                               "`python -m sink_sliding_window_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        DP = ctypes.POINTER(Dims)
        L.sink_attn_fwd.argtypes = [DP, P, P, P, P, P, I, ctypes.c_float, P, P, P]
        L.sink_attn_fwd.restype = I
        L.sink_attn_fwd_pair.argtypes = L.sink_attn_fwd.argtypes
        L.sink_attn_fwd_pair.restype = I
        L.sink_attn_fwd_with.argtypes = [DP, P, P, P, P, P, I, ctypes.c_float, P, P, I, P]
        L.sink_attn_fwd_with.restype = I
        L.sink_attn_fwd_kernel_for.argtypes = [DP, I]
        L.sink_attn_fwd_kernel_for.restype = I
        L.sink_attn_bwd.argtypes = [DP, P, P, P, P, P, I, ctypes.c_float, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.sink_attn_bwd.restype = I
        L.sink_attn_bwd_workspace_size.argtypes = [DP]
        L.sink_attn_bwd_workspace_size.restype = ctypes.c_size_t
        L.sink_attn_status_string.argtypes = [I]
        L.sink_attn_status_string.restype = ctypes.c_char_p
        L.sink_attn_last_device_error.argtypes = [P]
        L.sink_attn_last_device_error.restype = I
        L.sink_attn_device_error.argtypes = [P]
        L.sink_attn_device_error.restype = I
        L.sink_attn_fwd_launches.argtypes = [DP]
        L.sink_attn_fwd_launches.restype = I
        L.sink_attn_bwd_launches.argtypes = [DP]
        L.sink_attn_bwd_launches.restype = I
        L.sink_attn_profile_events.argtypes = [I, P, P]
        L.sink_attn_profile_events.restype = I
        DD = ctypes.POINTER(DecodeDims)
        L.sink_attn_decode.argtypes = [DD, P, P, P, P, P, P, P, I, ctypes.c_float, P, P, P, ctypes.c_size_t, P]
        L.sink_attn_decode.restype = I
        L.sink_attn_decode_e4m3.argtypes = [DD, P, P, P, P, P, P, P, P, P, I, ctypes.c_float, P, P, P,
                                            ctypes.c_size_t, P]
        L.sink_attn_decode_e4m3.restype = I
        L.sink_attn_decode_e4m3_f8pv.argtypes = L.sink_attn_decode_e4m3.argtypes
        L.sink_attn_decode_e4m3_f8pv.restype = I
        L.sink_attn_decode_workspace_size.argtypes = [DD, I]
        L.sink_attn_decode_workspace_size.restype = ctypes.c_size_t
        L.sink_attn_decode_launches.argtypes = [DD, I]
        L.sink_attn_decode_launches.restype = I
        L.sink_attn_selftest_wait.argtypes = [ctypes.c_ulonglong, P, P]
        L.sink_attn_selftest_wait.restype = I
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return load().sink_attn_status_string(int(status)).decode()


def make_dims(T, Hq, Hkv, D, batch, max_seqlen) -> Dims:
    return Dims(int(batch), int(max_seqlen), int(T), int(Hq), int(Hkv), int(D))


def _ptr(t):
    """Device address of a CUDA tensor (None for None).  Every pointer of the C
    ABI is a device pointer; a host tensor here is refused, since its address
    would reach the kernels as if it were device memory."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _geometry(q, k, cu_seqlens, batch, max_seqlen):
    if q.dim() == 4:  # [B, S, H, D]
        B, S = q.shape[0], q.shape[1]
        q = q.reshape(B * S, q.shape[2], q.shape[3])
        k = k.reshape(B * S, k.shape[2], k.shape[3])
        batch, max_seqlen = B, S
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    if cu_seqlens is not None:
        batch = cu_seqlens.numel() - 1
        if max_seqlen is None:
            max_seqlen = T
    if batch is None or max_seqlen is None:
        raise ValueError("give cu_seqlens, or batch and max_seqlen, or 4-D [B,S,H,D] tensors")
    return make_dims(T, Hq, Hkv, D, batch, max_seqlen), T, Hq, Hkv, D


# sink_attn_fwd_kernel_id values of the C ABI.
FWD_KERNELS = {"auto": 0, "one_tile": 1, "two_tiles": 2, "pair": 3}


def fwd(q, k, v, sinks, cu_seqlens=None, window=0, scale=None, *, batch=None, max_seqlen=None, out=None, lse=None,
        stream=None, kernel="auto"):
    """sink_attn_fwd (kernel="auto"), or sink_attn_fwd_with one of the
    library's forward kernels ("one_tile", "two_tiles", "pair").  q [T,Hq,D]
    (or [B,S,Hq,D]), k/v [T,Hkv,D] bf16 CUDA; sinks [Hq] fp32; cu_seqlens
    int32 [B+1] CUDA or None.  Returns (out like q, lse [Hq, T] fp32)."""
    if kernel not in FWD_KERNELS:
        raise ValueError(f"unknown forward kernel {kernel!r}; expected one of {sorted(FWD_KERNELS)}")
    dims, T, Hq, Hkv, D = _geometry(q, k, cu_seqlens, batch, max_seqlen)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    args = (ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(cu_seqlens), int(window), float(scale),
            _ptr(out), _ptr(lse))
    if kernel == "auto":
        name, st = "sink_attn_fwd", load().sink_attn_fwd(*args, _stream_handle(stream))
    else:
        name, st = "sink_attn_fwd_with", load().sink_attn_fwd_with(*args, FWD_KERNELS[kernel], _stream_handle(stream))
    if st != 0:
        raise SinkAttnError(st, name)
    return out, lse


def fwd_pair(q, k, v, sinks, cu_seqlens=None, window=0, scale=None, *, batch=None, max_seqlen=None, out=None,
             lse=None, stream=None):
    """sink_attn_fwd_pair: the forward on CTA pairs (tcgen05 M = 256);
    arguments and results as fwd()."""
    dims, T, Hq, Hkv, D = _geometry(q, k, cu_seqlens, batch, max_seqlen)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    st = load().sink_attn_fwd_pair(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(cu_seqlens),
                                   int(window), float(scale), _ptr(out), _ptr(lse), _stream_handle(stream))
    if st != 0:
        raise SinkAttnError(st, "sink_attn_fwd_pair")
    return out, lse


def fwd_kernel_for(T, Hq, Hkv, D, batch, max_seqlen, window) -> str:
    """Name of the forward kernel sink_attn_fwd runs for these sizes."""
    d = make_dims(T, Hq, Hkv, D, batch, max_seqlen)
    k = int(load().sink_attn_fwd_kernel_for(ctypes.byref(d), int(window)))
    return {v: n for n, v in FWD_KERNELS.items()}.get(k, "invalid")


def bwd_workspace_size(T, Hq, Hkv, D, batch, max_seqlen) -> int:
    d = make_dims(T, Hq, Hkv, D, batch, max_seqlen)
    return int(load().sink_attn_bwd_workspace_size(ctypes.byref(d)))


def bwd(q, k, v, sinks, out, lse, dout, cu_seqlens=None, window=0, scale=None, *, batch=None, max_seqlen=None,
        dq=None, dk=None, dv=None, dsinks=None, workspace=None, stream=None):
    """sink_attn_bwd.  Returns (dq, dk, dv, dsinks)."""
    dims, T, Hq, Hkv, D = _geometry(q, k, cu_seqlens, batch, max_seqlen)
    if scale is None:
        scale = D ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dsinks = torch.empty((Hq,), dtype=torch.float32, device=q.device) if dsinks is None else dsinks
    L = load()
    need = int(L.sink_attn_bwd_workspace_size(ctypes.byref(dims)))
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=q.device)
    st = L.sink_attn_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(cu_seqlens), int(window),
                         float(scale), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dsinks),
                         _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream_handle(stream))
    if st != 0:
        raise SinkAttnError(st, "sink_attn_bwd")
    return dq, dk, dv, dsinks


def decode_dims(batch, new_tokens, cache_capacity, max_seqlen, Hq, Hkv, D=64) -> DecodeDims:
    return DecodeDims(int(batch), int(new_tokens), int(cache_capacity), int(max_seqlen), int(Hq), int(Hkv), int(D))


def decode_workspace_size(batch, new_tokens, cache_capacity, max_seqlen, Hq, Hkv, window=0, D=64) -> int:
    d = decode_dims(batch, new_tokens, cache_capacity, max_seqlen, Hq, Hkv, D)
    return int(load().sink_attn_decode_workspace_size(ctypes.byref(d), int(window)))


def decode_launches(batch, new_tokens, cache_capacity, max_seqlen, Hq, Hkv, window=0, D=64) -> int:
    d = decode_dims(batch, new_tokens, cache_capacity, max_seqlen, Hq, Hkv, D)
    return int(load().sink_attn_decode_launches(ctypes.byref(d), int(window)))


def decode(q, k_new, v_new, k_cache, v_cache, cache_seqlens, sinks, window=0, scale=None, *, max_seqlen=None,
           out=None, lse=None, workspace=None, stream=None):
    """sink_attn_decode.  q [B, Lq, Hq, D], k_new / v_new [B, Lq, Hkv, D],
    k_cache / v_cache [B, C, Hkv, D] (bf16, CUDA; the new tokens are written
    into the cache), cache_seqlens int32 [B] CUDA (tokens cached before this
    call; not modified), sinks [Hq] fp32.  max_seqlen bounds
    cache_seqlens + Lq (default: C + Lq).  Returns (out [B, Lq, Hq, D],
    lse [Hq, B * Lq])."""
    B, Lq, Hq, D = q.shape
    C, Hkv = k_cache.shape[1], k_cache.shape[2]
    if max_seqlen is None:
        max_seqlen = C + Lq
    if scale is None:
        scale = D ** -0.5
    dims = decode_dims(B, Lq, C, max_seqlen, Hq, Hkv, D)
    L = load()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, B * Lq), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = int(L.sink_attn_decode_workspace_size(ctypes.byref(dims), int(window)))
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=q.device)
    st = L.sink_attn_decode(ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                            _ptr(cache_seqlens), _ptr(sinks), int(window), float(scale), _ptr(out), _ptr(lse),
                            _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream_handle(stream))
    if st != 0:
        raise SinkAttnError(st, "sink_attn_decode")
    return out, lse


def decode_e4m3(q, k_new, v_new, k_cache, v_cache, cache_seqlens, k_scale, v_scale, sinks, window=0, scale=None, *,
                max_seqlen=None, out=None, lse=None, workspace=None, stream=None, f8pv=False):
    """sink_attn_decode_e4m3: as decode(), with k_cache / v_cache holding e4m3
    codes ([B, C, Hkv, D] uint8 or torch.float8_e4m3fn) and k_scale / v_scale
    fp32 [Hkv] dequantisation scales.  f8pv: sink_attn_decode_e4m3_f8pv (the
    PV product in FP8, P rounded to e4m3)."""
    B, Lq, Hq, D = q.shape
    C, Hkv = k_cache.shape[1], k_cache.shape[2]
    if max_seqlen is None:
        max_seqlen = C + Lq
    if scale is None:
        scale = D ** -0.5
    dims = decode_dims(B, Lq, C, max_seqlen, Hq, Hkv, D)
    L = load()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, B * Lq), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = int(L.sink_attn_decode_workspace_size(ctypes.byref(dims), int(window)))
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=q.device)
    fn, name = ((L.sink_attn_decode_e4m3_f8pv, "sink_attn_decode_e4m3_f8pv") if f8pv
                else (L.sink_attn_decode_e4m3, "sink_attn_decode_e4m3"))
    st = fn(ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens),
            _ptr(k_scale), _ptr(v_scale), _ptr(sinks), int(window), float(scale), _ptr(out), _ptr(lse),
            _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream_handle(stream))
    if st != 0:
        raise SinkAttnError(st, name)
    return out, lse


def decode_e4m3_f8pv(*args, **kw):
    """sink_attn_decode_e4m3_f8pv (see decode_e4m3)."""
    return decode_e4m3(*args, f8pv=True, **kw)


def device_error(stream=None) -> int:
    return int(load().sink_attn_last_device_error(_stream_handle(stream)))


def selftest_wait(limit_ns: int, out=None, stream=None):
    """sink_attn_selftest_wait: one block waits on mbarriers nothing completes
    (see the header).  Returns ({first returned true, its us, second returned
    true, its us}, recorded device error code); synchronises through
    device_error()."""
    import torch
    if out is None:
        out = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    st = load().sink_attn_selftest_wait(int(limit_ns), _ptr(out), _stream_handle(stream))
    if st != 0:
        raise SinkAttnError(st, "sink_attn_selftest_wait")
    code = device_error(stream)
    return [int(v) for v in out.cpu().tolist()], code


def fwd_launches(T, Hq, Hkv, D, batch, max_seqlen) -> int:
    d = make_dims(T, Hq, Hkv, D, batch, max_seqlen)
    return int(load().sink_attn_fwd_launches(ctypes.byref(d)))


def bwd_launches(T, Hq, Hkv, D, batch, max_seqlen) -> int:
    d = make_dims(T, Hq, Hkv, D, batch, max_seqlen)
    return int(load().sink_attn_bwd_launches(ctypes.byref(d)))


PROFILE_FWD = 0
PROFILE_BWD_MAIN = 1


def profile_events(which: int, begin=None, end=None) -> None:
    """Registers torch.cuda.Event objects (created with enable_timing=True)
    that the library records right before and after one kernel launch
    (PROFILE_FWD: the forward kernel; PROFILE_BWD_MAIN: the backward's
    tensor-core kernel).  profile_events(which) clears the slot."""
    if (begin is not None and not begin.cuda_event) or (end is not None and not end.cuda_event):
        raise ValueError("record each event once before registering it (torch creates it on first record)")
    b = None if begin is None else ctypes.c_void_p(begin.cuda_event)
    e = None if end is None else ctypes.c_void_p(end.cuda_event)
    st = load().sink_attn_profile_events(int(which), b, e)
    if st != 0:
        raise SinkAttnError(st, "sink_attn_profile_events")
