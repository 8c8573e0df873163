"""Pins for the fp64 oracle: checks against facts fixed by the mathematics
of sink attention, independent of the oracle's own code.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with the fact.  They are run against the committed oracle
(tests/test_oracle_pins.py) and against deliberately broken copies of its
source (tests/test_oracle_mutations.py), to show that a plausible mistake in
the oracle trips at least one of them.

The definition being pinned (attention sink as an extra softmax logit that
carries no value, named in Megatron-LM issue 1739 "gpt-oss implementation",
section "Attention Sinks", and in the transformers blog "Tricks from OpenAI
gpt-oss", kernels section):
    out_i = sum_j e^{l_ij - m} v_j / (e^{s_h - m} + sum_j e^{l_ij - m}),
    lse_i = log(e^{s_h} + sum_j e^{l_ij}),  l_ij = scale q_i . k_j,
with keys j restricted to the query's own document, j <= i, and, for a
sliding-window layer of width W, i - j < W.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers
def rand_problem(seed, T, Hq, Hkv, D, cu=None, sink_std=1.0, q_std=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, Hq, D)) * q_std
    k = rng.standard_normal((T, Hkv, D))
    v = rng.standard_normal((T, Hkv, D))
    s = rng.standard_normal(Hq) * sink_std
    if cu is None:
        cu = np.array([0, T], np.int32)
    return q, k, v, s, np.asarray(cu, np.int32)


def torch_sink_reference(q, k, v, sinks, cu, window, scale):
    """Library special case: sink attention is ordinary softmax attention
    with one extra key whose logit is s_h and whose value is the zero
    vector.  Built from torch.softmax / torch.logsumexp in float64."""
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((T, Hq, D))
    lse = np.zeros((Hq, T))
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        L = e - a
        if L == 0:
            continue
        i = torch.arange(L)[:, None]
        j = torch.arange(L)[None, :]
        allowed = j <= i
        if window > 0:
            allowed &= (i - j) < window
        for h in range(Hq):
            g = h // G
            Q = torch.from_numpy(q[a:e, h])
            K = torch.from_numpy(k[a:e, g])
            V = torch.from_numpy(v[a:e, g])
            logits = (Q @ K.T) * scale
            logits = logits.masked_fill(~allowed, float("-inf"))
            ext = torch.cat([logits, torch.full((L, 1), float(sinks[h]), dtype=torch.float64)], dim=1)
            P = torch.softmax(ext, dim=1)
            Vext = torch.cat([V, torch.zeros(1, D, dtype=torch.float64)], dim=0)
            out[a:e, h] = (P @ Vext).numpy()
            lse[h, a:e] = torch.logsumexp(ext, dim=1).numpy()
    return out, lse


def brute_force(q, k, v, sinks, cu, window, scale):
    """Hand-written loops over scalars (tiny inputs only)."""
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(T)]
    lse = [[0.0] * T for _ in range(Hq)]
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        for i in range(e - a):
            for h in range(Hq):
                g = h // G
                terms = []  # (weight exponent, value row)
                for jj in range(i + 1):
                    if window > 0 and not (i - jj < window):
                        continue
                    dot = 0.0
                    for d in range(D):
                        dot += float(q[a + i, h, d]) * float(k[a + jj, g, d])
                    terms.append((scale * dot, a + jj))
                z = math.exp(float(sinks[h]))
                num = [0.0] * D
                for l, jt in terms:
                    w = math.exp(l)
                    z += w
                    for d in range(D):
                        num[d] += w * float(v[jt, g, d])
                for d in range(D):
                    out[a + i][h][d] = num[d] / z
                lse[h][a + i] = math.log(z)
    return np.array(out), np.array(lse)


def assert_close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- pins
def pin_library_special_case(O):
    """P1: equals torch softmax over [logits, s_h] times [V; 0]."""
    cases = [
        (dict(T=37, Hq=4, Hkv=2, D=16), None, 0),
        (dict(T=37, Hq=4, Hkv=2, D=16), None, 5),
        (dict(T=40, Hq=6, Hkv=2, D=8), [0, 7, 8, 29, 40], 0),
        (dict(T=40, Hq=6, Hkv=2, D=8), [0, 7, 8, 29, 40], 4),
        (dict(T=33, Hq=8, Hkv=1, D=64), None, 32),
    ]
    for n, (dims, cu, W) in enumerate(cases):
        q, k, v, s, cu = rand_problem(100 + n, cu=cu, **dims)
        out, lse = O.fwd(q, k, v, s, cu, W, 0.125)
        ro, rl = torch_sink_reference(q, k, v, s, cu, W, 0.125)
        assert_close(out, ro, 1e-12, f"P1 out case {n}")
        assert_close(lse, rl, 1e-12, f"P1 lse case {n}")


def pin_no_sink_is_causal_sdpa(O):
    """P2: sink = -inf reproduces plain causal softmax attention
    (torch scaled_dot_product_attention, is_causal=True, float64)."""
    T, Hq, Hkv, D = 45, 4, 2, 16
    q, k, v, _, cu = rand_problem(7, T, Hq, Hkv, D)
    s = np.full(Hq, -np.inf)
    out, lse = O.fwd(q, k, v, s, cu, 0, 0.125)
    G = Hq // Hkv
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]
    K = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)[None]
    V = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=0.125)
    assert_close(out, ref[0].permute(1, 0, 2).numpy(), 1e-12, "P2 out")
    logits = (Q @ K.transpose(-1, -2)) * 0.125
    logits = logits.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    assert_close(lse, torch.logsumexp(logits, -1)[0].numpy(), 1e-12, "P2 lse")


def pin_wide_window_is_full_causal(O):
    """P3: a window at least as long as the document is full causal
    (bitwise: the same keys in the same order)."""
    T = 50
    q, k, v, s, cu = rand_problem(3, T, 4, 1, 8, cu=[0, 20, 50])
    full = O.fwd(q, k, v, s, cu, 0, 0.125)
    for W in (30, 50, 1000):
        win = O.fwd(q, k, v, s, cu, W, 0.125)
        assert np.array_equal(full[0], win[0]) and np.array_equal(full[1], win[1]), f"P3 W={W}"
    win = O.fwd(q, k, v, s, cu, 29, 0.125)
    assert not np.array_equal(full[0], win[0]), "P3: W=29 must differ on a 30-token document"


def pin_huge_sink(O):
    """P4: s_h = +1e4 takes all the probability: out -> 0, lse -> s_h."""
    q, k, v, _, cu = rand_problem(4, 30, 2, 1, 8)
    s = np.full(2, 1e4)
    out, lse = O.fwd(q, k, v, s, cu, 0, 0.125)
    assert float(np.max(np.abs(out))) < 1e-12, "P4 out"
    assert_close(lse, np.full_like(lse, 1e4), 1e-9, "P4 lse")


def pin_probabilities_sum_to_one(O):
    """P5: with v = 1 the output is sum_j P_ij, and P_sink = e^{s_h - lse};
    the two add up to 1 for every row."""
    T, Hq = 60, 4
    q, k, _, s, cu = rand_problem(5, T, Hq, 2, 8, cu=[0, 1, 21, 60], sink_std=3.0)
    v = np.ones((T, 2, 8))
    for W in (0, 1, 7):
        out, lse = O.fwd(q, k, v, s, cu, W, 0.125)
        psink = np.exp(s[None, :] - lse.T)  # [T, Hq]
        assert_close(out[:, :, 0] + psink, np.ones((T, Hq)), 1e-12, f"P5 W={W}")


def pin_zero_query_closed_form(O):
    """P6: q = 0 makes every logit 0, so
    out_i = sum_{j in K(i)} v_j / (e^{s_h} + |K(i)|), lse = ln(e^{s_h} + |K(i)|)."""
    cu = [0, 9, 30]
    T, Hq, Hkv, D = 30, 4, 2, 8
    _, k, v, s, cu = rand_problem(6, T, Hq, Hkv, D, cu=cu)
    q = np.zeros((T, Hq, D))
    for W in (0, 4):
        out, lse = O.fwd(q, k, v, s, cu, W, 0.125)
        for b in range(len(cu) - 1):
            a, e = cu[b], cu[b + 1]
            for i in range(e - a):
                lo = 0 if W <= 0 else max(0, i - W + 1)
                n = i - lo + 1
                for h in range(Hq):
                    g = h // (Hq // Hkv)
                    z = math.exp(s[h]) + n
                    exp_out = v[a + lo:a + i + 1, g].sum(0) / z
                    assert_close(out[a + i, h], exp_out, 1e-13, f"P6 out W={W} t={a+i} h={h}")
                    assert abs(lse[h, a + i] - math.log(z)) < 1e-13, f"P6 lse W={W} t={a+i} h={h}"


def pin_brute_force(O):
    """P7a: independent scalar loops on tiny inputs."""
    for n, (cu, W) in enumerate([([0, 8], 0), ([0, 8], 3), ([0, 3, 4, 8], 0), ([0, 3, 4, 8], 2)]):
        q, k, v, s, cu = rand_problem(20 + n, 8, 2, 1, 4, cu=cu)
        out, lse = O.fwd(q, k, v, s, cu, W, 0.5)
        bo, bl = brute_force(q, k, v, s, cu, W, 0.5)
        assert_close(out, bo, 1e-13, f"P7 out case {n}")
        assert_close(lse, bl, 1e-13, f"P7 lse case {n}")


def pin_hand_example(O):
    """P7b: the worked example in tests/golden/hand_example.json, computed
    by hand from the definition (two tokens, one head, D = 1)."""
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        ex = json.load(f)
    q = np.array(ex["q"], np.float64).reshape(-1, 1, 1)
    k = np.array(ex["k"], np.float64).reshape(-1, 1, 1)
    v = np.array(ex["v"], np.float64).reshape(-1, 1, 1)
    s = np.array(ex["sinks"], np.float64)
    cu = np.array([0, q.shape[0]], np.int32)
    for case in ex["cases"]:
        out, lse = O.fwd(q, k, v, s, cu, case["window"], ex["scale"])
        assert_close(out[:, 0, 0], case["out"], 1e-14, f"hand example out W={case['window']}")
        assert_close(lse[0], case["lse"], 1e-14, f"hand example lse W={case['window']}")
        dout = np.array(ex["dout"], np.float64).reshape(-1, 1, 1)
        dq, dk, dv, ds = O.bwd(q, k, v, s, cu, case["window"], ex["scale"], dout)
        assert_close(ds, [case["dsink"]], 1e-14, f"hand example dsink W={case['window']}")
        assert_close(dv[:, 0, 0], case["dv"], 1e-14, f"hand example dv W={case['window']}")


def _loss(O, q, k, v, s, cu, W, scale, dout):
    out, _ = O.fwd(q, k, v, s, cu, W, scale)
    return float(np.sum(out * dout))


def pin_finite_differences(O):
    """P8: the backward pass is the gradient of L = sum(dout * out):
    central differences (h = 1e-6) on every sink and on random coordinates
    and random directions of q, k, v; with and without window, packed."""
    scale = 0.3
    for n, (cu, W) in enumerate([([0, 16], 0), ([0, 16], 5), ([0, 6, 16], 0), ([0, 6, 16], 3)]):
        q, k, v, s, cu = rand_problem(40 + n, 16, 4, 2, 8, cu=cu)
        dout = np.random.default_rng(90 + n).standard_normal(q.shape)
        dq, dk, dv, ds = O.bwd(q, k, v, s, cu, W, scale, dout)
        h = 1e-6
        rng = np.random.default_rng(60 + n)

        def fd(name, idx=None, direction=None):
            args = {"q": q, "k": k, "v": v, "s": s}
            base = args[name]
            plus, minus = base.copy(), base.copy()
            if direction is None:
                plus[idx] += h
                minus[idx] -= h
            else:
                plus += h * direction
                minus -= h * direction
            ap = dict(args, **{name: plus})
            am = dict(args, **{name: minus})
            lp = _loss(O, ap["q"], ap["k"], ap["v"], ap["s"], cu, W, scale, dout)
            lm = _loss(O, am["q"], am["k"], am["v"], am["s"], cu, W, scale, dout)
            return (lp - lm) / (2 * h)

        for hh in range(4):
            g = fd("s", idx=(hh,))
            assert abs(g - ds[hh]) <= 1e-6 * max(1.0, abs(g)), f"P8 dsink[{hh}] {ds[hh]} vs fd {g}"
        for name, grad in (("q", dq), ("k", dk), ("v", dv)):
            for _ in range(6):
                idx = tuple(int(rng.integers(0, m)) for m in grad.shape)
                g = fd(name, idx=idx)
                assert abs(g - grad[idx]) <= 1e-6 * max(1.0, abs(g)), f"P8 d{name}{idx} {grad[idx]} vs fd {g}"
            u = rng.standard_normal(grad.shape)
            g = fd(name, direction=u)
            an = float(np.sum(grad * u))
            assert abs(g - an) <= 1e-6 * max(1.0, abs(g)), f"P8 d{name} direction {an} vs fd {g}"


def pin_structure(O):
    """P9: GQA equals MHA with K/V repeated; packed documents equal separate
    runs; permuting documents permutes outputs; a window row equals full
    attention over just the last W keys (all bitwise)."""
    cu = [0, 11, 12, 40]
    T, Hq, Hkv, D = 40, 6, 2, 8
    q, k, v, s, cu = rand_problem(9, T, Hq, Hkv, D, cu=cu)
    G = Hq // Hkv
    for W in (0, 5):
        o1, l1 = O.fwd(q, k, v, s, cu, W, 0.125)
        o2, l2 = O.fwd(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), s, cu, W, 0.125)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2), f"P9 GQA vs MHA W={W}"
        for b in range(len(cu) - 1):
            a, e = cu[b], cu[b + 1]
            ob, lb = O.fwd(q[a:e], k[a:e], v[a:e], s, [0, e - a], W, 0.125)
            assert np.array_equal(ob, o1[a:e]) and np.array_equal(lb, l1[:, a:e]), f"P9 doc {b} W={W}"
        # documents in reverse order
        order = [2, 1, 0]
        segs = [(cu[b], cu[b + 1]) for b in order]
        perm = np.concatenate([np.arange(a, e) for a, e in segs])
        cu_p = np.concatenate([[0], np.cumsum([e - a for a, e in segs])]).astype(np.int32)
        op, lp = O.fwd(q[perm], k[perm], v[perm], s, cu_p, W, 0.125)
        assert np.array_equal(op, o1[perm]) and np.array_equal(lp, l1[:, perm]), f"P9 permute W={W}"
    # window row == full attention over the W keys ending at the query
    W = 5
    o1, l1 = O.fwd(q, k, v, s, cu, W, 0.125)
    for t in (20, 25, 39):
        sl = slice(t - W + 1, t + 1)
        ow, lw = O.fwd(q[sl], k[sl], v[sl], s, [0, W], 0, 0.125)
        assert np.array_equal(ow[-1], o1[t]) and np.array_equal(lw[:, -1], l1[:, t]), f"P9 window row t={t}"


def pin_rows_match_full(O):
    """The row-sampled forward returns exactly the rows of the full one."""
    q, k, v, s, cu = rand_problem(11, 50, 4, 2, 8, cu=[0, 17, 50])
    for W in (0, 6):
        o, l = O.fwd(q, k, v, s, cu, W, 0.125)
        rows = np.array([0, 5, 16, 17, 30, 49])
        orow, lrow = O.fwd_rows(q, k, v, s, cu, W, 0.125, rows)
        assert np.array_equal(orow, o[rows]) and np.array_equal(lrow, l[:, rows]), f"rows W={W}"


def pin_bf16_widening(O):
    """bf16 inputs are widened exactly: the bf16 entry point equals the
    fp64 one on the widened values (bitwise)."""
    rng = np.random.default_rng(12)
    bits = lambda shape: (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q, k, v = bits((20, 4, 8)), bits((20, 2, 8)), bits((20, 2, 8))
    s = rng.standard_normal(4).astype(np.float32)
    cu = np.array([0, 20], np.int32)
    widen = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    a = O.fwd(q, k, v, s, cu, 3, 0.125)
    b = O.fwd(widen(q), widen(k), widen(v), s.astype(np.float64), cu, 3, 0.125)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]), "bf16 widening"
    dout = bits((20, 4, 8))
    ga = O.bwd(q, k, v, s, cu, 3, 0.125, dout)
    gb = O.bwd(widen(q), widen(k), widen(v), s.astype(np.float64), cu, 3, 0.125, widen(dout))
    assert all(np.array_equal(x, y) for x, y in zip(ga, gb)), "bf16 widening bwd"


def pin_restricted_backward(O):
    """dq for chosen query tokens and dk/dv for chosen key tokens equal the
    matching rows of the full backward (same sums, same order)."""
    for n, (cu, W) in enumerate([([0, 40], 0), ([0, 40], 6), ([0, 9, 10, 40], 0), ([0, 9, 10, 40], 5)]):
        q, k, v, s, cu = rand_problem(70 + n, 40, 4, 2, 8, cu=cu)
        dout = np.random.default_rng(80 + n).standard_normal(q.shape)
        dq, dk, dv, _ = O.bwd(q, k, v, s, cu, W, 0.25, dout)
        rows = np.array([0, 3, 9, 10, 25, 39])
        assert_close(O.bwd_dq_rows(q, k, v, s, cu, W, 0.25, dout, rows), dq[rows], 1e-12, f"dq rows case {n}")
        keys = np.array([0, 8, 9, 10, 30, 39])
        rk, rv = O.bwd_dkv_rows(q, k, v, s, cu, W, 0.25, dout, keys)
        assert_close(rk, dk[keys], 1e-12, f"dk rows case {n}")
        assert_close(rv, dv[keys], 1e-12, f"dv rows case {n}")
        # the sink gradient alone equals the full backward's
        ds = O.bwd(q, k, v, s, cu, W, 0.25, dout)[3]
        assert_close(O.bwd_dsinks(q, k, v, s, cu, W, 0.25, dout), ds, 1e-12, f"dsinks alone case {n}")


def _probabilities(q, k, s, cu, W, scale):
    """P_ij = e^{l_ij - lse_i} and P_sink,i = e^{s_h - lse_i}, written out in
    numpy from the definition (independent of the oracle): P [Hq, T, T]
    (zero where key j is not allowed for query i) and Psink [Hq, T]."""
    T, Hq, _ = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    P = np.zeros((Hq, T, T))
    Psink = np.zeros((Hq, T))
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        for i in range(a, e):
            lo = a if W <= 0 else max(a, i - W + 1)
            for h in range(Hq):
                lg = scale * (k[lo:i + 1, h // G] @ q[i, h])
                m = max(float(s[h]), float(lg.max()))
                z = math.exp(float(s[h]) - m) + float(np.exp(lg - m).sum())
                P[h, i, lo:i + 1] = np.exp(lg - m) / z
                Psink[h, i] = math.exp(float(s[h]) - m) / z
    return P, Psink


def pin_saved_output_for_D(O):
    """The backward's optional saved output (``out_for_D``, the output the
    caller kept from its forward) enters only through D_i = dout_i . X_i:
      (a) X = the oracle's own forward output gives exactly the results of
          X = None, in the full backward and in both restricted ones;
      (b) for another X, dsinks_h = -sum_i P_sink,i (dout_i . X_i);
      (c) dv does not move, and dq, dk move by the closed-form change of
          dS_ij by -P_ij dout_i . (X_i - out_i):
            dq_i += -scale sum_j P_ij delta_i k_j,
            dk_j += -scale sum_{i, h in group} P_ij delta_i q_i,
          delta_i = dout_i . (X_i - out_i);
      (d) the restricted backwards take X at the right rows;
      (e) the bf16 entry point widens X exactly, like every other input."""
    scale = 0.3
    for n, (cu, W) in enumerate([([0, 16], 0), ([0, 16], 5), ([0, 6, 16], 0), ([0, 5, 7, 16], 3)]):
        q, k, v, s, cu = rand_problem(140 + n, 16, 4, 2, 8, cu=cu)
        T, Hq, D = q.shape
        G = Hq // k.shape[1]
        rng = np.random.default_rng(150 + n)
        dout = rng.standard_normal(q.shape)
        out, lse = O.fwd(q, k, v, s, cu, W, scale)
        base = O.bwd(q, k, v, s, cu, W, scale, dout)
        same = O.bwd(q, k, v, s, cu, W, scale, dout, out_for_D=out)
        assert all(np.array_equal(x, y) for x, y in zip(base, same)), f"saved output = own output, case {n}"
        rows = np.array([0, 5, 6, 11, 15])
        assert np.array_equal(O.bwd_dq_rows(q, k, v, s, cu, W, scale, dout, rows, out_for_D=out),
                              O.bwd_dq_rows(q, k, v, s, cu, W, scale, dout, rows)), f"dq rows own output {n}"
        rk0, rv0 = O.bwd_dkv_rows(q, k, v, s, cu, W, scale, dout, rows)
        rk1, rv1 = O.bwd_dkv_rows(q, k, v, s, cu, W, scale, dout, rows, out_for_D=out)
        assert np.array_equal(rk0, rk1) and np.array_equal(rv0, rv1), f"dk/dv rows own output {n}"

        X = out + 0.5 * rng.standard_normal(out.shape)
        dq0, dk0, dv0, ds0 = base
        dq1, dk1, dv1, ds1 = O.bwd(q, k, v, s, cu, W, scale, dout, out_for_D=X)
        P, Psink = _probabilities(q, k, s, cu, W, scale)
        DX = np.einsum("thd,thd->ht", dout, X)  # [Hq, T]
        assert_close(ds1, -(Psink * DX).sum(axis=1), 1e-12, f"dsinks from saved output, case {n}")
        assert_close(O.bwd_dsinks(q, k, v, s, cu, W, scale, dout, out_for_D=X), -(Psink * DX).sum(axis=1), 1e-12,
                     f"dsinks alone from saved output, case {n}")
        assert np.array_equal(dv0, dv1), f"dv must not depend on the saved output, case {n}"
        delta = np.einsum("thd,thd->ht", dout, X - out)  # [Hq, T]
        kk = np.repeat(k, G, axis=1)  # [T, Hq, D]: key j as seen by head h
        ddq = -scale * np.einsum("hij,jhd->ihd", P * delta[:, :, None], kk)
        assert_close(dq1 - dq0, ddq, 1e-12, f"dq shift from saved output, case {n}")
        ddk_h = -scale * np.einsum("hij,ihd->jhd", P * delta[:, :, None], q)  # [T, Hq, D]
        ddk = ddk_h.reshape(T, Hq // G, G, D).sum(axis=2)
        assert_close(dk1 - dk0, ddk, 1e-12, f"dk shift from saved output, case {n}")
        assert_close(O.bwd_dq_rows(q, k, v, s, cu, W, scale, dout, rows, out_for_D=X), dq1[rows], 1e-12,
                     f"dq rows with saved output, case {n}")
        rk, rv = O.bwd_dkv_rows(q, k, v, s, cu, W, scale, dout, rows, out_for_D=X)
        assert_close(rk, dk1[rows], 1e-12, f"dk rows with saved output, case {n}")
        assert_close(rv, dv1[rows], 1e-12, f"dv rows with saved output, case {n}")

    # (e) bf16 bits of a saved output: the bf16 entry points equal the fp64
    # ones on the widened values, bitwise.
    rng = np.random.default_rng(160)
    bits = lambda shape: (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    widen = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    q, k, v, do, xo = bits((20, 4, 8)), bits((20, 2, 8)), bits((20, 2, 8)), bits((20, 4, 8)), bits((20, 4, 8))
    s = rng.standard_normal(4).astype(np.float32)
    cu = np.array([0, 7, 20], np.int32)
    wq, wk, wv, wdo, wxo, ws = widen(q), widen(k), widen(v), widen(do), widen(xo), s.astype(np.float64)
    ga = O.bwd(q, k, v, s, cu, 3, 0.125, do, out_for_D=xo)
    gb = O.bwd(wq, wk, wv, ws, cu, 3, 0.125, wdo, out_for_D=wxo)
    assert all(np.array_equal(x, y) for x, y in zip(ga, gb)), "bf16 saved output widening (bwd)"
    rows = np.array([0, 6, 7, 19])
    assert np.array_equal(O.bwd_dq_rows(q, k, v, s, cu, 3, 0.125, do, rows, out_for_D=xo),
                          O.bwd_dq_rows(wq, wk, wv, ws, cu, 3, 0.125, wdo, rows, out_for_D=wxo)), \
        "bf16 saved output widening (dq rows)"
    ka = O.bwd_dkv_rows(q, k, v, s, cu, 3, 0.125, do, rows, out_for_D=xo)
    kb = O.bwd_dkv_rows(wq, wk, wv, ws, cu, 3, 0.125, wdo, rows, out_for_D=wxo)
    assert np.array_equal(ka[0], kb[0]) and np.array_equal(ka[1], kb[1]), "bf16 saved output widening (dk/dv rows)"
    assert np.array_equal(O.bwd_dsinks(q, k, v, s, cu, 3, 0.125, do, out_for_D=xo),
                          O.bwd_dsinks(wq, wk, wv, ws, cu, 3, 0.125, wdo, out_for_D=wxo)), \
        "bf16 saved output widening (dsinks alone)"


ALL_PINS = [
    pin_library_special_case,
    pin_no_sink_is_causal_sdpa,
    pin_wide_window_is_full_causal,
    pin_huge_sink,
    pin_probabilities_sum_to_one,
    pin_zero_query_closed_form,
    pin_brute_force,
    pin_hand_example,
    pin_finite_differences,
    pin_structure,
    pin_rows_match_full,
    pin_bf16_widening,
    pin_restricted_backward,
    pin_saved_output_for_D,
]
