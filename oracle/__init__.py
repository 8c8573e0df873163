"""fp64 CPU oracle for sink attention (causal GQA + learned per-head sink +
sliding window + intra-document masking).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package; the
product path (``sink_sliding_window_b200``) never does, and it shares no code
with it.  The arithmetic lives in ``sink_attn_oracle.c`` (plain C, fp64,
OpenMP over independent rows); this module only compiles it and marshals
numpy arrays through ctypes.

Every function here is the plain definition (see the C file's header for the
formula, the readings taken where the pages are silent, and the citations).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "sink_attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_sinkattn.so")
_lock = threading.Lock()


def build(force: bool = False, src: str = SOURCE, out: str = _LIB_PATH) -> str:
    """Compile the C oracle (or another copy of its source) into a shared
    library."""
    with _lock:
        if (not force and os.path.exists(out)
                and os.path.getmtime(out) >= os.path.getmtime(src)):
            return out
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-ffp-contract=off", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
        return out


def _bind(path):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    Dbl = ctypes.c_double
    common = [I, I, I, I, I, P]
    lib.oracle_fwd_f64.argtypes = common + [P, P, P, P, I, Dbl, P, P, I]
    lib.oracle_fwd_bf16.argtypes = common + [P, P, P, P, I, Dbl, P, P, I]
    lib.oracle_fwd_rows_f64.argtypes = common + [P, P, P, P, I, Dbl, P, I64, P, P, I]
    lib.oracle_fwd_rows_bf16.argtypes = common + [P, P, P, P, I, Dbl, P, I64, P, P, I]
    lib.oracle_bwd_f64.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, P, P, P, I]
    lib.oracle_bwd_bf16.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, P, P, P, I]
    lib.oracle_bwd_dq_rows_f64.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, I64, P, I]
    lib.oracle_bwd_dq_rows_bf16.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, I64, P, I]
    lib.oracle_bwd_dkv_rows_f64.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, I64, P, P, I]
    lib.oracle_bwd_dkv_rows_bf16.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, I64, P, P, I]
    lib.oracle_bwd_dsinks_f64.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, I]
    lib.oracle_bwd_dsinks_bf16.argtypes = common + [P, P, P, P, I, Dbl, P, P, P, I]
    lib.oracle_bf16_to_f64.argtypes = [P, P, I64]
    for f in ("oracle_fwd_f64", "oracle_fwd_bf16", "oracle_fwd_rows_f64", "oracle_fwd_rows_bf16",
              "oracle_bwd_f64", "oracle_bwd_bf16", "oracle_bwd_dq_rows_f64", "oracle_bwd_dq_rows_bf16",
              "oracle_bwd_dkv_rows_f64", "oracle_bwd_dkv_rows_bf16", "oracle_bwd_dsinks_f64",
              "oracle_bwd_dsinks_bf16", "oracle_bf16_to_f64", "oracle_max_threads"):
        getattr(lib, f).restype = I
    return lib


class Oracle:
    """A loaded copy of the C oracle (the committed one by default)."""

    def __init__(self, lib_path: str):
        self.lib = _bind(lib_path)

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def fwd(self, q, k, v, sinks, cu_seqlens, window, scale, nthreads=0):
        """Forward definition.

        q: [T,Hq,D], k/v: [T,Hkv,D]; either all uint16 bf16 bit patterns or
        all float64.  sinks: [Hq] (float32 for the bf16 variant, float64
        otherwise).  cu_seqlens: int32 [B+1] on the host.  Returns
        (out [T,Hq,D] f64, lse [Hq,T] f64)."""
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        cu = _cu(cu_seqlens, T)
        B = cu.shape[0] - 1
        out = np.empty((T, Hq, D), np.float64)
        lse = np.empty((Hq, T), np.float64)
        if _is_bf16_bits(q):
            args = [np.ascontiguousarray(x, np.uint16) for x in (q, k, v)]
            s = np.ascontiguousarray(sinks, np.float32)
            fn = self.lib.oracle_fwd_bf16
        else:
            args = [np.ascontiguousarray(x, np.float64) for x in (q, k, v)]
            s = np.ascontiguousarray(sinks, np.float64)
            fn = self.lib.oracle_fwd_f64
        rc = fn(T, Hq, Hkv, D, B, _ptr(cu), *map(_ptr, args), _ptr(s), int(window), float(scale),
                _ptr(out), _ptr(lse), int(nthreads))
        _check(rc, "oracle fwd")
        return out, lse

    def fwd_rows(self, q, k, v, sinks, cu_seqlens, window, scale, rows, nthreads=0):
        """Forward definition for selected query tokens (every head).

        Returns (out [n,Hq,D] f64, lse [Hq,n] f64) for tokens ``rows``."""
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        cu = _cu(cu_seqlens, T)
        B = cu.shape[0] - 1
        r = np.ascontiguousarray(rows, np.int64)
        n = r.shape[0]
        out = np.empty((n, Hq, D), np.float64)
        lse = np.empty((Hq, n), np.float64)
        if _is_bf16_bits(q):
            args = [np.ascontiguousarray(x, np.uint16) for x in (q, k, v)]
            s = np.ascontiguousarray(sinks, np.float32)
            fn = self.lib.oracle_fwd_rows_bf16
        else:
            args = [np.ascontiguousarray(x, np.float64) for x in (q, k, v)]
            s = np.ascontiguousarray(sinks, np.float64)
            fn = self.lib.oracle_fwd_rows_f64
        rc = fn(T, Hq, Hkv, D, B, _ptr(cu), *map(_ptr, args), _ptr(s), int(window), float(scale),
                _ptr(r), n, _ptr(out), _ptr(lse), int(nthreads))
        _check(rc, "oracle fwd_rows")
        return out, lse

    def bwd(self, q, k, v, sinks, cu_seqlens, window, scale, dout, out_for_D=None, nthreads=0):
        """Backward definition.

        ``dout`` has the dtype convention of ``q``.  ``out_for_D`` (optional,
        same convention) is the saved output used for D_i = dout_i . out_i;
        by default the oracle's own fp64 output is used.  Returns
        (dq [T,Hq,D], dk [T,Hkv,D], dv [T,Hkv,D], dsinks [Hq]), float64."""
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        cu = _cu(cu_seqlens, T)
        B = cu.shape[0] - 1
        dq = np.empty((T, Hq, D), np.float64)
        dk = np.empty((T, Hkv, D), np.float64)
        dv = np.empty((T, Hkv, D), np.float64)
        ds = np.empty((Hq,), np.float64)
        if _is_bf16_bits(q):
            conv, sconv, fn = np.uint16, np.float32, self.lib.oracle_bwd_bf16
        else:
            conv, sconv, fn = np.float64, np.float64, self.lib.oracle_bwd_f64
        args = [np.ascontiguousarray(x, conv) for x in (q, k, v)]
        s = np.ascontiguousarray(sinks, sconv)
        o = None if out_for_D is None else np.ascontiguousarray(out_for_D, conv)
        do = np.ascontiguousarray(dout, conv)
        rc = fn(T, Hq, Hkv, D, B, _ptr(cu), *map(_ptr, args), _ptr(s), int(window), float(scale),
                _ptr(o), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds), int(nthreads))
        _check(rc, "oracle bwd")
        return dq, dk, dv, ds

    def _bwd_args(self, q, k, v, sinks, dout, out_for_D):
        if _is_bf16_bits(q):
            conv, sconv, sfx = np.uint16, np.float32, "bf16"
        else:
            conv, sconv, sfx = np.float64, np.float64, "f64"
        args = [np.ascontiguousarray(x, conv) for x in (q, k, v)]
        s = np.ascontiguousarray(sinks, sconv)
        o = None if out_for_D is None else np.ascontiguousarray(out_for_D, conv)
        do = np.ascontiguousarray(dout, conv)
        return args, s, o, do, sfx

    def bwd_dq_rows(self, q, k, v, sinks, cu_seqlens, window, scale, dout, rows, out_for_D=None, nthreads=0):
        """dq of the backward definition for the query tokens ``rows`` (every
        head).  Returns dq_rows [n, Hq, D] float64."""
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        cu = _cu(cu_seqlens, T)
        r = np.ascontiguousarray(rows, np.int64)
        out = np.empty((r.shape[0], Hq, D), np.float64)
        args, s, o, do, sfx = self._bwd_args(q, k, v, sinks, dout, out_for_D)
        fn = getattr(self.lib, f"oracle_bwd_dq_rows_{sfx}")
        rc = fn(T, Hq, Hkv, D, cu.shape[0] - 1, _ptr(cu), *map(_ptr, args), _ptr(s), int(window), float(scale),
                _ptr(o), _ptr(do), _ptr(r), r.shape[0], _ptr(out), int(nthreads))
        _check(rc, "oracle bwd_dq_rows")
        return out

    def bwd_dkv_rows(self, q, k, v, sinks, cu_seqlens, window, scale, dout, keys, out_for_D=None, nthreads=0):
        """dk and dv of the backward definition for the key tokens ``keys``
        (sorted ascending; every key/value head).  Returns (dk_rows, dv_rows),
        each [n, Hkv, D] float64."""
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        cu = _cu(cu_seqlens, T)
        kk = np.ascontiguousarray(keys, np.int64)
        dk = np.empty((kk.shape[0], Hkv, D), np.float64)
        dv = np.empty((kk.shape[0], Hkv, D), np.float64)
        args, s, o, do, sfx = self._bwd_args(q, k, v, sinks, dout, out_for_D)
        fn = getattr(self.lib, f"oracle_bwd_dkv_rows_{sfx}")
        rc = fn(T, Hq, Hkv, D, cu.shape[0] - 1, _ptr(cu), *map(_ptr, args), _ptr(s), int(window), float(scale),
                _ptr(o), _ptr(do), _ptr(kk), kk.shape[0], _ptr(dk), _ptr(dv), int(nthreads))
        _check(rc, "oracle bwd_dkv_rows")
        return dk, dv

    def bwd_dsinks(self, q, k, v, sinks, cu_seqlens, window, scale, dout, out_for_D=None, nthreads=0):
        """dsinks of the backward definition alone (one forward pass of
        work).  Returns dsinks [Hq] float64."""
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        cu = _cu(cu_seqlens, T)
        ds = np.empty((Hq,), np.float64)
        args, s, o, do, sfx = self._bwd_args(q, k, v, sinks, dout, out_for_D)
        fn = getattr(self.lib, f"oracle_bwd_dsinks_{sfx}")
        rc = fn(T, Hq, Hkv, D, cu.shape[0] - 1, _ptr(cu), *map(_ptr, args), _ptr(s), int(window), float(scale),
                _ptr(o), _ptr(do), _ptr(ds), int(nthreads))
        _check(rc, "oracle bwd_dsinks")
        return ds

    def bf16_bits_to_f64(self, a):
        """Exact widening of bf16 bit patterns (uint16) to float64."""
        a = np.ascontiguousarray(a, np.uint16)
        out = np.empty(a.shape, np.float64)
        _check(self.lib.oracle_bf16_to_f64(_ptr(a), _ptr(out), a.size), "bf16 widen")
        return out


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _cu(cu_seqlens, T):
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    if cu.ndim != 1 or cu[0] != 0 or cu[-1] != T:
        raise ValueError("cu_seqlens must be 1-D, start at 0 and end at T")
    return cu


def _is_bf16_bits(a):
    return a.dtype == np.uint16


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed with code {rc}")


_default = None


def default() -> Oracle:
    """The committed oracle, compiled on first use."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def fwd(*a, **kw):
    return default().fwd(*a, **kw)


def fwd_rows(*a, **kw):
    return default().fwd_rows(*a, **kw)


def bwd(*a, **kw):
    return default().bwd(*a, **kw)


def bwd_dq_rows(*a, **kw):
    return default().bwd_dq_rows(*a, **kw)


def bwd_dkv_rows(*a, **kw):
    return default().bwd_dkv_rows(*a, **kw)


def bwd_dsinks(*a, **kw):
    return default().bwd_dsinks(*a, **kw)


def bf16_bits_to_f64(a):
    return default().bf16_bits_to_f64(a)


def max_threads() -> int:
    return default().max_threads()
