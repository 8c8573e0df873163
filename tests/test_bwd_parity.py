"""sink_attn_bwd (CUDA, through the C ABI) against the fp64 oracle's
backward.

sink_attn_bwd takes the forward's saved out (bf16) and lse (fp32) as inputs.
For parity both sides get identical inputs: the oracle's own forward output
rounded to those API dtypes is handed to the GPU backward, and the oracle's
backward forms D_i = dout_i . out_i from the same bf16 bits.  Tolerances:
1e-2 (dq, dk, dv) and 1e-3 (dsinks) of the oracle tensor's max-abs.

A second group of tests chains the GPU forward into the GPU backward, as a
training step does, against the oracle in fp64 end to end.  There the sink
gradient also carries the bf16 rounding of the saved output, which the API
cannot avoid; those tests bound it by the rounding error itself."""
import numpy as np
import pytest

import oracle
from sink_sliding_window_b200 import synth
from tests.gpu_util import TOL_LSE, TOL_OUT, check, dev, dev_bf16, host_f64, rel_err, run_bwd, run_fwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    import torch
    from sink_sliding_window_b200 import build, ops as _ops
    assert torch.cuda.is_available()
    build.build()
    return _ops


def _whole(ops, w, a, what):
    ro, rl = oracle.fwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale)
    out_bits = synth.f32_to_bf16_bits(ro.astype(np.float32))
    dq, dk, dv, ds = run_bwd(w, a, ops, dev_bf16(out_bits), dev(rl.astype(np.float32)))
    rq, rk, rv, rs = oracle.bwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, a["dout"],
                                out_for_D=out_bits)
    errs = dict(
        dq=check(host_f64(dq), rq, TOL_OUT, f"{what} dq"),
        dk=check(host_f64(dk), rk, TOL_OUT, f"{what} dk"),
        dv=check(host_f64(dv), rv, TOL_OUT, f"{what} dv"),
        dsinks=check(host_f64(ds), rs, TOL_LSE, f"{what} dsinks"),
    )
    return errs


@pytest.mark.parametrize("name", ["tiny:w32", "tiny:full"])
def test_tiny_whole(ops, name):
    w = synth.workload(name)
    a = w.generate(with_dout=True)
    _whole(ops, w, a, name)


def _small(T, Hq, Hkv, cu, window, seed, sinks=None):
    w = synth.Workload("edge", T, Hq, Hkv, 64, np.asarray(cu, np.int32), None, window, 0.125, seed=seed)
    a = w.generate(with_dout=True)
    if sinks is not None:
        a["sinks"] = np.asarray(sinks, np.float32)
    return w, a


@pytest.mark.parametrize("S", [1, 17, 128, 129, 300])
@pytest.mark.parametrize("window", [0, 1, 127, 129])
def test_lengths_and_windows(ops, S, window):
    B = 2
    w, a = _small(B * S, 8, 1, np.arange(B + 1) * S, window, seed=S * 100 + window)
    _whole(ops, w, a, f"S={S} W={window}")


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32, 64, 128])
def test_gqa_ratios(ops, G):
    w, a = _small(400, G * 2, 2, [0, 37, 38, 400], 100, seed=G + 50)
    _whole(ops, w, a, f"G={G}")


def test_sink_extremes(ops):
    sinks = [-np.inf, -1e4, 0.0, 1e4, 0.5, -0.5, 3.0, -np.inf]
    for window in (0, 64):
        w, a = _small(500, 8, 1, [0, 250, 500], window, seed=7, sinks=sinks)
        _whole(ops, w, a, f"sinks W={window}")


def test_packed_documents(ops):
    cu = [0, 1, 1, 2, 19, 20, 150, 151, 420]
    for window in (0, 3, 200):
        w, a = _small(420, 16, 2, cu, window, seed=13)
        _whole(ops, w, a, f"packed W={window}")


def test_training_4k_window_whole(ops):
    """gpt-oss training shapes, sliding-window layer: whole tensors."""
    w = synth.workload("prefill4k:w128")
    a = w.generate(with_dout=True)
    errs = _whole(ops, w, a, "bwd 4k w128")
    print("bwd 4k w128 relative errors", errs)


@pytest.mark.parametrize("doc,g", [(0, 0), (3, 7)])
def test_training_4k_full_slices(ops, doc, g):
    """gpt-oss training shapes, full-causal layer, in the same launch
    configuration the benchmark times: whole (document, key/value group)
    slices of dq, dk, dv compared with the oracle run on that slice alone (a
    document and a group are independent sub-problems)."""
    w = synth.workload("prefill4k:full")
    a = w.generate(with_dout=True)
    out, lse = run_fwd(w, a, ops)
    dq, dk, dv, ds = run_bwd(w, a, ops, out, lse)
    S, G = 4096, 8
    sl = slice(doc * S, (doc + 1) * S)
    hs = slice(g * G, (g + 1) * G)
    rq, rk, rv, rs = oracle.bwd(a["q"][sl, hs], a["k"][sl, g:g + 1], a["v"][sl, g:g + 1], a["sinks"][hs],
                                np.array([0, S], np.int32), 0, w.scale, a["dout"][sl, hs])
    check(host_f64(dq[sl, hs]), rq, TOL_OUT, "dq slice")
    check(host_f64(dk[sl, g:g + 1]), rk, TOL_OUT, "dk slice")
    check(host_f64(dv[sl, g:g + 1]), rv, TOL_OUT, "dv slice")


def _chain(ops, w, a, what):
    out, lse = run_fwd(w, a, ops)
    dq, dk, dv, ds = run_bwd(w, a, ops, out, lse)
    ro, rl = oracle.fwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale)
    rq, rk, rv, rs = oracle.bwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, a["dout"])
    check(host_f64(dq), rq, TOL_OUT, f"{what} chained dq")
    check(host_f64(dk), rk, TOL_OUT, f"{what} chained dk")
    check(host_f64(dv), rv, TOL_OUT, f"{what} chained dv")
    # Saving out in bf16 moves each element by at most 2^-9 of itself
    # (round to nearest), so D_i moves by at most 2^-9 sum_d |dout_id out_id|
    # and dsinks_h by at most 2^-9 sum_i P_sink,i sum_d |dout_id out_id|.
    # Allow twice that plus the 1e-3 parity budget.
    do = oracle.bf16_bits_to_f64(a["dout"])
    psink = np.exp(a["sinks"].astype(np.float64)[:, None] - rl)
    bound = 2.0 * 2.0 ** -9 * (psink * np.einsum("thd,thd->ht", np.abs(do), np.abs(ro))).sum(1)
    err = np.abs(host_f64(ds) - rs)
    assert np.all(err <= bound + TOL_LSE * np.abs(rs).max()), f"{what} chained dsinks {err} vs bound {bound}"
    return rel_err(host_f64(ds), rs)


@pytest.mark.parametrize("name", ["tiny:w32", "tiny:full", "prefill4k:w128"])
def test_fwd_bwd_chain(ops, name):
    w = synth.workload(name)
    a = w.generate(with_dout=True)
    e = _chain(ops, w, a, name)
    print(f"{name}: chained dsinks relative error {e:.2e}")


def test_dsinks_4k_full_vs_oracle(ops):
    """gpt-oss training shapes, full-causal layer, whole problem: the sink
    gradient against the oracle's.  Both sides get identical saved inputs
    (the oracle's forward output rounded to bf16 and its lse rounded to
    fp32), and the oracle evaluates dsinks_h = -sum_i P_sink,i D_i over every
    row of every document (one fp64 forward pass of work).  Also: dsinks is
    bitwise reproducible run to run, and dk / dv (reduced inside TMEM in a
    fixed order) are too."""
    w = synth.workload("prefill4k:full")
    a = w.generate(with_dout=True)
    ro, rl = oracle.fwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale)
    out_bits = synth.f32_to_bf16_bits(ro.astype(np.float32))
    out, lse = dev_bf16(out_bits), dev(rl.astype(np.float32))
    r1 = run_bwd(w, a, ops, out, lse)
    r2 = run_bwd(w, a, ops, out, lse)
    assert (r1[3] == r2[3]).all(), "dsinks must be bitwise reproducible"
    assert (r1[1] == r2[1]).all() and (r1[2] == r2[2]).all(), "dk/dv are reduced in TMEM in a fixed order"
    rs = oracle.bwd_dsinks(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, a["dout"],
                           out_for_D=out_bits)
    e = check(host_f64(r1[3]), rs, TOL_LSE, "bwd 4k full dsinks vs oracle")
    print(f"bwd 4k full: dsinks relative error {e:.2e} against the oracle")
