"""Helpers shared by the GPU parity tests: moving the seeded bf16 inputs to
the device, reading results back, and the tolerance checks (max-abs error
relative to the oracle tensor's max-abs: 1e-2 for out/dq/dk/dv, 1e-3 for
lse/dsinks)."""
import numpy as np
import torch

TOL_OUT = 1e-2
TOL_LSE = 1e-3


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    denom = float(np.max(np.abs(ref))) if ref.size else 1.0
    return float(np.max(np.abs(got - ref))) / max(denom, 1e-30)


def check(got, ref, tol, what):
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    e = rel_err(got, ref)
    assert e <= tol, f"{what}: relative max-abs error {e:.3e} > {tol:.0e}"
    return e


def run_fwd(w, arrays, ops, stream=None):
    """Calls sink_attn_fwd on the workload's arrays; returns (out, lse) tensors."""
    q, k, v = dev_bf16(arrays["q"]), dev_bf16(arrays["k"]), dev_bf16(arrays["v"])
    s = dev(arrays["sinks"])
    if w.uniform_seqlen is not None:
        out, lse = ops.fwd(q, k, v, s, None, w.window, w.scale, batch=w.batch, max_seqlen=w.uniform_seqlen,
                           stream=stream)
    else:
        cu = dev(w.cu_seqlens)
        out, lse = ops.fwd(q, k, v, s, cu, w.window, w.scale, max_seqlen=w.max_seqlen, stream=stream)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    return out, lse


def run_bwd(w, arrays, ops, out, lse, stream=None):
    """sink_attn_bwd on the workload's arrays with the forward's saved
    out / lse; returns (dq, dk, dv, dsinks) tensors."""
    q, k, v = dev_bf16(arrays["q"]), dev_bf16(arrays["k"]), dev_bf16(arrays["v"])
    s = dev(arrays["sinks"])
    do = dev_bf16(arrays["dout"])
    if w.uniform_seqlen is not None:
        r = ops.bwd(q, k, v, s, out, lse, do, None, w.window, w.scale, batch=w.batch,
                    max_seqlen=w.uniform_seqlen, stream=stream)
    else:
        cu = dev(w.cu_seqlens)
        r = ops.bwd(q, k, v, s, out, lse, do, cu, w.window, w.scale, max_seqlen=w.max_seqlen, stream=stream)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    return r
