"""sink_attn_bwd at the full long-context and packed-document sizes, in the
launch configuration the benchmark uses, against the fp64 oracle.

The oracle's whole backward is quadratic in the sequence length, so at these
sizes it is evaluated only where it is cheap and still decisive:
  * dq for a seeded sample of query tokens (document starts and ends, the
    first and last rows of a tile, random tokens), every head;
  * dk and dv for chosen key tokens, every key/value head: on a window layer
    any token (a key is seen by at most W queries); on a full-causal layer
    keys near the end of a document, whose readers are few, plus the first
    key of the shortest packed document;
  * dsinks through the identity dsinks_h = -sum_i e^{s_h - lse_i} (dout_i .
    out_i) over the saved out / lse, which holds at any size (the value
    itself is checked against the oracle by test_dsinks_window_vs_oracle
    here, on the window layers whose oracle forward is cheap, and by the 4k
    full-causal test in test_bwd_parity.py).
The GPU forward feeds the GPU backward, as in a training step; the oracle
runs in fp64 from the same bf16 inputs.  Tolerance: 1e-2 of the oracle
slice's max-abs for dq, dk, dv (as in the small parity tests)."""
import numpy as np
import pytest

import oracle
from sink_sliding_window_b200 import synth
from tests.gpu_util import TOL_OUT, check, host_f64, run_bwd, run_fwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    import torch
    from sink_sliding_window_b200 import build, ops as _ops
    assert torch.cuda.is_available()
    build.build()
    return _ops


def key_sample(w, n_random=48):
    """Key tokens whose dk/dv the oracle can afford at this workload."""
    cu = w.cu_seqlens.astype(np.int64)
    keys = set()
    if w.window > 0:
        keys.update(int(t) for t in w.sample_rows(n_random))
        return np.array(sorted(keys), np.int64)
    # Full causal: key j is read by every later query of its document, so
    # only keys close to a document's end are cheap.  Take the last 160
    # keys of the last document (two key tiles and a partial one), the last
    # 8 keys of the first few documents, and the whole of the shortest one.
    last_a, last_e = int(cu[-2]), int(cu[-1])
    keys.update(range(max(last_a, last_e - 160), last_e))
    for b in range(min(w.batch, 6)):
        a, e = int(cu[b]), int(cu[b + 1])
        keys.update(range(max(a, e - 8), e))
    lens = np.diff(cu)
    b = int(np.argmin(np.where(lens > 0, lens, np.iinfo(np.int64).max)))
    if lens[b] <= 1024:
        keys.update(range(int(cu[b]), int(cu[b + 1]), 7))
    return np.array(sorted(keys), np.int64)


def _fullsize(ops, name, seed=0):
    import torch
    w = synth.workload(name, seed=seed)
    a = w.generate(with_dout=True)
    out, lse = run_fwd(w, a, ops)
    dq, dk, dv, ds = run_bwd(w, a, ops, out, lse)
    rows = w.sample_rows(24)
    keys = key_sample(w)
    r = torch.from_numpy(rows).cuda()
    kk = torch.from_numpy(keys).cuda()
    got_dq = host_f64(dq.index_select(0, r))
    got_dk = host_f64(dk.index_select(0, kk))
    got_dv = host_f64(dv.index_select(0, kk))

    rq = oracle.bwd_dq_rows(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, a["dout"], rows)
    rk, rv = oracle.bwd_dkv_rows(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, a["dout"],
                                 keys)
    errs = dict(dq=check(got_dq, rq, TOL_OUT, f"{name} dq rows"),
                dk=check(got_dk, rk, TOL_OUT, f"{name} dk keys"),
                dv=check(got_dv, rv, TOL_OUT, f"{name} dv keys"))

    # dsinks over the saved out / lse, summed in fp64 one document block at
    # a time (no fp64 copy of the whole output).
    ps_dv = np.zeros(w.Hq)
    s = a["sinks"].astype(np.float64)
    do_all = torch.from_numpy(a["dout"].view(np.int16)).view(torch.bfloat16)
    lse_h = host_f64(lse)
    step = 8192
    for t0 in range(0, w.T, step):
        o = host_f64(out[t0:t0 + step])
        do = do_all[t0:t0 + step].double().numpy()
        Dv = np.einsum("thd,thd->ht", o, do)
        ps_dv += (np.exp(s[:, None] - lse_h[:, t0:t0 + step]) * Dv).sum(1)
    errs["dsinks"] = check(host_f64(ds), -ps_dv, 1e-4, f"{name} dsinks vs fp64 sum over saved out/lse")
    print(f"{name}: {len(rows)} query rows, {len(keys)} keys, relative errors {errs}")
    return errs


@pytest.mark.parametrize("name", ["long60k:w128", "long60k:full", "varlen64k:w128", "varlen64k:full"])
def test_bwd_fullsize(ops, name):
    _fullsize(ops, name)


@pytest.mark.parametrize("seed", [1, 2])
def test_bwd_varlen_full_other_seeds(ops, seed):
    """The packed-document full-causal backward on two more seeds (other
    document lengths and values): dq is the tensor closest to its tolerance
    on seed 0, so its margin is shown on more than one draw."""
    _fullsize(ops, "varlen64k:full", seed=seed)


@pytest.mark.parametrize("name", ["long60k:w128", "varlen64k:w128"])
def test_dsinks_window_vs_oracle(ops, name):
    """The sink gradient of the long window-128 layers against the oracle's,
    from identical saved inputs (the oracle's output rounded to bf16, its lse
    rounded to fp32): tolerance 1e-3 of the oracle's max-abs."""
    from tests.gpu_util import TOL_LSE, dev, dev_bf16
    w = synth.workload(name)
    a = w.generate(with_dout=True)
    ro, rl = oracle.fwd(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale)
    out_bits = synth.f32_to_bf16_bits(ro.astype(np.float32))
    del ro
    _, _, _, ds = run_bwd(w, a, ops, dev_bf16(out_bits), dev(rl.astype(np.float32)))
    rs = oracle.bwd_dsinks(a["q"], a["k"], a["v"], a["sinks"], w.cu_seqlens, w.window, w.scale, a["dout"],
                           out_for_D=out_bits)
    e = check(host_f64(ds), rs, TOL_LSE, f"{name} dsinks vs oracle")
    print(f"{name}: dsinks relative error {e:.2e} against the oracle")
