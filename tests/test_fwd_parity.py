"""The forward kernels (CUDA, through the C ABI: sink_attn_fwd_with with each
kernel, sink_attn_fwd, sink_attn_fwd_pair) against the fp64 oracle on the
same seeded bf16 inputs: whole tensors on small cases that still span several
tiles and a ragged tail, sampled rows (every head) at the full workload
sizes, and the edge cases of the method (tiny and single-token documents,
window edges, sinks of -inf / -1e4 / 0 / +1e4, every supported GQA ratio)."""
import numpy as np
import pytest

import oracle
from sink_sliding_window_b200 import synth
from tests.gpu_util import TOL_LSE, TOL_OUT, check, dev, dev_bf16, host_f64, run_fwd

pytestmark = pytest.mark.gpu


class _KernelOps:
    """The binding with fwd pinned to one of the library's forward kernels
    (through sink_attn_fwd_with)."""

    def __init__(self, mod, kernel):
        self._mod = mod
        self.kernel = kernel

    def fwd(self, *args, **kw):
        return self._mod.fwd(*args, kernel=self.kernel, **kw)

    def __getattr__(self, name):
        return getattr(self._mod, name)


@pytest.fixture(scope="module", params=["one_tile", "two_tiles", "pair"])
def ops(request):
    """Every case runs through each forward kernel: one query tile per CTA,
    two tiles per CTA, and CTA pairs (M = 256)."""
    import torch
    from sink_sliding_window_b200 import build, ops as _ops
    assert torch.cuda.is_available()
    build.build()
    return _KernelOps(_ops, request.param)


@pytest.mark.parametrize("name", ["tiny:w32", "tiny:full"])
def test_tiny_whole(ops, name):
    w = synth.workload(name)
    a = w.generate()
    out, lse = run_fwd(w, a, ops)
    ro, rl = oracle.fwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale)
    check(host_f64(out), ro, TOL_OUT, f"{name} out")
    check(host_f64(lse), rl, TOL_LSE, f"{name} lse")


def _small(T, Hq, Hkv, cu, window, seed, sinks=None, scale=0.125):
    w = synth.Workload("edge", T, Hq, Hkv, 64, np.asarray(cu, np.int32), None, window, scale, seed=seed)
    a = w.generate()
    if sinks is not None:
        a["sinks"] = np.asarray(sinks, np.float32)
    return w, a


def _whole_check(ops, w, a, what):
    out, lse = run_fwd(w, a, ops)
    ro, rl = oracle.fwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale)
    check(host_f64(out), ro, TOL_OUT, f"{what} out")
    check(host_f64(lse), rl, TOL_LSE, f"{what} lse")


@pytest.mark.parametrize("S", [1, 2, 15, 16, 17, 127, 128, 129, 300])
@pytest.mark.parametrize("window", [0, 1, 2, 127, 128, 129])
def test_lengths_and_windows(ops, S, window):
    B = 2
    w, a = _small(B * S, 8, 1, np.arange(B + 1) * S, window, seed=S * 1000 + window)
    _whole_check(ops, w, a, f"S={S} W={window}")


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32, 64, 128])
def test_gqa_ratios(ops, G):
    Hkv = 2
    w, a = _small(400, G * Hkv, Hkv, [0, 37, 38, 400], 100, seed=G)
    _whole_check(ops, w, a, f"G={G}")


@pytest.mark.parametrize("scale", [1.0, 4.0])
@pytest.mark.parametrize("window", [0, 64])
def test_wide_logits(ops, scale, window):
    """Logits 8-32x wider than at scale 1/8: a row's running reference max is
    raised on many key steps, so the O rescale runs repeatedly."""
    w, a = _small(700, 8, 1, [0, 250, 700], window, seed=11, scale=scale)
    _whole_check(ops, w, a, f"scale={scale} W={window}")


def test_sink_extremes(ops):
    sinks = [-np.inf, -1e4, 0.0, 1e4, 0.5, -0.5, 3.0, -np.inf]
    for window in (0, 64):
        w, a = _small(700, 8, 1, [0, 250, 700], window, seed=5, sinks=sinks)
        _whole_check(ops, w, a, f"sinks W={window}")


def test_packed_tiny_documents(ops):
    # documents of length 1 and 0, and a document cut inside a query tile
    cu = [0, 1, 1, 2, 19, 20, 150, 151, 300]
    for window in (0, 3, 200):
        w, a = _small(300, 16, 2, cu, window, seed=11)
        _whole_check(ops, w, a, f"packed W={window}")


def test_uniform_vs_packed_api(ops):
    """The same uniform batch through cu_seqlens = NULL and through explicit
    cu_seqlens gives identical bits."""
    w = synth.workload("tiny:w32")
    a = w.generate()
    out1, lse1 = run_fwd(w, a, ops)
    w2 = synth.Workload("p", w.T, w.Hq, w.Hkv, 64, w.cu_seqlens, None, w.window, w.scale)
    out2, lse2 = run_fwd(w2, a, ops)
    assert (out1 == out2).all() and (lse1 == lse2).all()


def _sampled(ops, name, n_rows, seed=0):
    w = synth.workload(name, seed=seed)
    a = w.generate()
    out, lse = run_fwd(w, a, ops)
    rows = w.sample_rows(n_rows)
    ro, rl = oracle.fwd_rows(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, rows)
    got_o = host_f64(out[rows])
    got_l = host_f64(lse[:, rows])
    check(got_o, ro, TOL_OUT, f"{name} out (sampled rows)")
    check(got_l, rl, TOL_LSE, f"{name} lse (sampled rows)")
    # properties that hold at any size
    import torch
    assert torch.isfinite(lse).all() and torch.isfinite(out.float()).all()
    return w, out, lse


@pytest.mark.parametrize("name", ["prefill4k:w128", "prefill4k:full"])
def test_prefill4k_sampled(ops, name):
    _sampled(ops, name, 96)


@pytest.mark.parametrize("name", ["varlen64k:w128", "varlen64k:full"])
def test_varlen_sampled(ops, name):
    _sampled(ops, name, 64)


@pytest.mark.parametrize("name", ["long60k:w128", "long60k:full"])
def test_long60k_sampled(ops, name):
    _sampled(ops, name, 24)


def test_prefill4k_window_whole_group(ops):
    """Whole-tensor comparison on one document and one KV group of the
    gpt-oss prefill shapes (window 128): the oracle's cost allows it."""
    w = synth.workload("prefill4k:w128")
    a = w.generate()
    out, lse = run_fwd(w, a, ops)
    S, g, G = 4096, 3, 8
    sl = slice(S, 2 * S)  # document 1
    q = a["q"][sl, g * G:(g + 1) * G]
    k = a["k"][sl, g:g + 1]
    v = a["v"][sl, g:g + 1]
    ro, rl = oracle.fwd(q, k, v, a["sinks"][g * G:(g + 1) * G], np.array([0, S], np.int32), w.window, w.scale)
    check(host_f64(out[sl, g * G:(g + 1) * G]), ro, TOL_OUT, "prefill4k w128 doc1 group3 out")
    check(host_f64(lse[g * G:(g + 1) * G, sl]), rl, TOL_LSE, "prefill4k w128 doc1 group3 lse")


def test_deterministic(ops):
    w = synth.workload("prefill4k:full")
    a = w.generate()
    o1, l1 = run_fwd(w, a, ops)
    o2, l2 = run_fwd(w, a, ops)
    assert (o1 == o2).all() and (l1 == l2).all()


@pytest.fixture(scope="module")
def ops_mod():
    import torch
    from sink_sliding_window_b200 import build, ops as _ops
    assert torch.cuda.is_available()
    build.build()
    return _ops


@pytest.mark.parametrize("name", ["prefill4k:full", "prefill4k:w128"])
def test_kernels_agree(ops_mod, name):
    """sink_attn_fwd, sink_attn_fwd_pair and every kernel of
    sink_attn_fwd_with agree to rounding on the prefill shapes (each is also
    checked against the oracle above), and sink_attn_fwd is bit-identical to
    the kernel it reports through sink_attn_fwd_kernel_for."""
    import torch
    w = synth.workload(name)
    a = w.generate()
    o_auto, l_auto = run_fwd(w, a, ops_mod)
    chosen = ops_mod.fwd_kernel_for(w.T, w.Hq, w.Hkv, w.D, w.batch, w.max_seqlen, w.window)
    assert chosen in ("one_tile", "two_tiles", "pair")
    scale_o = float(o_auto.float().abs().max())
    for kn in ("one_tile", "two_tiles", "pair"):
        o, l = run_fwd(w, a, _KernelOps(ops_mod, kn))
        if kn == chosen:
            assert (o == o_auto).all() and (l == l_auto).all()
        assert float((o.float() - o_auto.float()).abs().max()) <= 1e-2 * scale_o
        assert float((l - l_auto).abs().max()) <= 1e-3 * float(l_auto.abs().max())
        assert torch.isfinite(l).all()
    o_p, l_p = ops_mod.fwd_pair(dev_bf16(a["q"]), dev_bf16(a["k"]), dev_bf16(a["v"]), dev(a["sinks"]), None,
                                w.window, w.scale, batch=w.batch, max_seqlen=w.uniform_seqlen)
    o_w, l_w = run_fwd(w, a, _KernelOps(ops_mod, "pair"))
    torch.cuda.synchronize()
    assert (o_p == o_w).all() and (l_p == l_w).all()
