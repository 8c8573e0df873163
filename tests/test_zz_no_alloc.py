"""sink_attn_bwd_noalloc: the backward for callers that cannot allocate
device memory (for example code running inside an allocator callback, or a
host that must not grow device memory after start-up).  It uses a fixed
scratch array inside the library instead of a caller workspace.

Checked here, through the C ABI: on two calls in a row its dq, dk, dv and
dsinks match the regular sink_attn_bwd (caller-provided workspace) within
the tolerances of the other parity tests, and sizes beyond the built-in
array are refused before any launch.  The file name sorts last so that a
run stopping at the first failure has run every other test already.
"""
import ctypes

import numpy as np
import pytest

from sink_sliding_window_b200 import synth
from tests.gpu_util import TOL_LSE, TOL_OUT, check, dev, dev_bf16, host_f64, run_bwd, run_fwd

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024


@pytest.fixture(scope="module")
def env():
    import torch
    from sink_sliding_window_b200 import build, ops
    assert torch.cuda.is_available()
    build.build()
    L = ops.load()
    P = ctypes.c_void_p
    L.sink_attn_bwd_noalloc.argtypes = [ctypes.POINTER(ops.Dims), P, P, P, P, P, ctypes.c_int, ctypes.c_float,
                                        P, P, P, P, P, P, P, P]
    L.sink_attn_bwd_noalloc.restype = ctypes.c_int
    return torch, ops, L


def _call_noalloc(torch, ops, L, w, a, out, lse):
    q, k, v = dev_bf16(a["q"]), dev_bf16(a["k"]), dev_bf16(a["v"])
    s, do = dev(a["sinks"]), dev_bf16(a["dout"])
    cu = None if w.uniform_seqlen is not None else dev(w.cu_seqlens)
    dims = ops.make_dims(w.T, w.Hq, w.Hkv, 64, w.batch,
                         w.uniform_seqlen if w.uniform_seqlen is not None else w.max_seqlen)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = torch.empty((w.Hq,), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = L.sink_attn_bwd_noalloc(ctypes.byref(dims), p(q), p(k), p(v), p(s), p(cu), w.window, w.scale, p(out),
                                 p(lse), p(do), p(dq), p(dk), p(dv), p(ds),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, ops.status_string(st)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    return dq, dk, dv, ds


@pytest.mark.parametrize("case", ["uniform", "packed"])
def test_noalloc_matches_workspace_backward_twice(env, case):
    torch, ops, L = env
    if case == "uniform":
        w = synth.Workload("noalloc", 2 * 700, 16, 2, 64, synth.uniform_cu_seqlens(2, 700), 700, 96, 0.125, seed=3)
    else:
        cu = np.array([0, 1, 300, 301, 1200, 1500], np.int32)
        w = synth.Workload("noalloc", 1500, 16, 2, 64, cu, None, 0, 0.125, seed=4)
    assert ops.bwd_workspace_size(w.T, w.Hq, w.Hkv, 64, w.batch, w.max_seqlen) <= SCRATCH_BYTES
    a = w.generate(with_dout=True)
    out, lse = run_fwd(w, a, ops)
    ref = [host_f64(t) for t in run_bwd(w, a, ops, out, lse)]
    for call in range(2):  # the second call finds the first call's leftovers in the array
        got = [host_f64(t) for t in _call_noalloc(torch, ops, L, w, a, out, lse)]
        for name, g, r, tol in zip(("dq", "dk", "dv", "dsinks"), got, ref, (TOL_OUT, TOL_OUT, TOL_OUT, TOL_LSE)):
            check(g, r, tol, f"{case} call {call} {name}")
        assert np.array_equal(got[3], ref[3]), "dsinks is reduced in a fixed order"


def test_noalloc_rejects_oversize(env):
    torch, ops, L = env
    T, Hq = 4096, 64  # needs ~65 MiB of scratch
    dims = ops.make_dims(T, Hq, 8, 64, 1, T)
    assert ops.bwd_workspace_size(T, Hq, 8, 64, 1, T) > SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: refused before any launch
    st = L.sink_attn_bwd_noalloc(ctypes.byref(dims), fake, fake, fake, fake, None, 0, 0.125, fake, fake, fake,
                                 fake, fake, fake, fake, None)
    assert st == 7, ops.status_string(st)  # SINK_ATTN_ERR_WORKSPACE
