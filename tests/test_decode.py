"""sink_attn_decode (CUDA, through the C ABI) against the fp64 oracle.

Decode evaluates the forward definition at the newest positions of each
sequence, so the oracle is the forward itself: every sequence's whole token
history is packed as one document per sequence and oracle.fwd_rows evaluates
the rows of the new tokens.  The GPU sees the same tokens through its cache:
history position p < L0 sits in slot p mod C (later positions overwrite
earlier ones, so a ring keeps the last C), the new tokens are passed
separately and appended by the call.  Slots that hold no token are filled
with NaN: no result may depend on them.  Tolerances: 1e-2 (out) and 1e-3
(lse) of the oracle tensor's max-abs."""
import numpy as np
import pytest

import oracle
from sink_sliding_window_b200 import synth
from tests.gpu_util import TOL_LSE, TOL_OUT, check, dev, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

NAN_BF16 = np.uint16(0x7FC0)
SCALE = 0.125


@pytest.fixture(scope="module")
def ops():
    import torch
    from sink_sliding_window_b200 import build, ops as _ops
    assert torch.cuda.is_available()
    build.build()
    return _ops


def _cache_from_history(hist, cu, cached, C):
    """[B][C][H][D] cache holding positions p < cached[b] at slot p mod C;
    untouched slots are NaN."""
    B = len(cached)
    H, D = hist.shape[1], hist.shape[2]
    cache = np.full((B, C, H, D), NAN_BF16, np.uint16)
    for b in range(B):
        for p in range(int(cached[b])):
            cache[b, p % C] = hist[int(cu[b]) + p]
    return cache


def _oracle_rows(a, cached, Lq, window, seqs=None):
    """Oracle out / lse for the new tokens of the sequences `seqs` (all by
    default), one sequence at a time (each sequence is its own document)."""
    cu = a["cu"]
    seqs = range(len(cached)) if seqs is None else seqs
    Hq, D = a["q_new"].shape[2], a["q_new"].shape[3]
    outs, lses = [], []
    for b in seqs:
        lo, hi = int(cu[b]), int(cu[b + 1])
        L = hi - lo
        q = np.zeros((L, Hq, D), np.uint16)
        q[int(cached[b]):] = a["q_new"][b]
        rows = np.arange(int(cached[b]), L, dtype=np.int64)
        o, l = oracle.fwd_rows(q, a["k"][lo:hi], a["v"][lo:hi], a["sinks"], np.array([0, L], np.int32), window,
                               SCALE, rows)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses, axis=1)


def _run(ops, cached, Lq, Hq, Hkv, C, window, seed, sinks=None, check_all=True, seqs=None):
    import torch
    a = synth.decode_inputs(seed, cached, Lq, Hq, Hkv)
    if sinks is not None:
        a["sinks"] = np.asarray(sinks, np.float32)
    cu = a["cu"]
    B = len(cached)
    kc0 = _cache_from_history(a["k"], cu, cached, C)
    vc0 = _cache_from_history(a["v"], cu, cached, C)
    new_idx = np.concatenate([np.arange(int(cu[b]) + int(cached[b]), int(cu[b + 1])) for b in range(B)])
    k_new = a["k"][new_idx].reshape(B, Lq, Hkv, 64)
    v_new = a["v"][new_idx].reshape(B, Lq, Hkv, 64)
    kc, vc = dev_bf16(kc0), dev_bf16(vc0)
    seqlens = dev(np.asarray(cached, np.int32))
    out, lse = ops.decode(dev_bf16(a["q_new"]), dev_bf16(k_new), dev_bf16(v_new), kc, vc, seqlens,
                          dev(a["sinks"]), window, SCALE, max_seqlen=int(max(cached)) + Lq)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    # The new tokens are in their slots; nothing else changed (bitwise).
    ke, ve = kc0.copy(), vc0.copy()
    for b in range(B):
        for t in range(Lq):
            ke[b, (int(cached[b]) + t) % C] = k_new[b, t]
            ve[b, (int(cached[b]) + t) % C] = v_new[b, t]
    assert np.array_equal(kc.view(torch.int16).cpu().numpy().view(np.uint16), ke), "k cache after append"
    assert np.array_equal(vc.view(torch.int16).cpu().numpy().view(np.uint16), ve), "v cache after append"
    seqs = list(range(B)) if seqs is None else list(seqs)
    ro, rl = _oracle_rows(a, cached, Lq, window, seqs)
    got_o = host_f64(out)[seqs].reshape(-1, Hq, 64)
    got_l = host_f64(lse).reshape(Hq, B, Lq)[:, seqs].reshape(Hq, -1)
    eo = check(got_o, ro, TOL_OUT, "decode out")
    el = check(got_l, rl, TOL_LSE, "decode lse")
    return eo, el


@pytest.mark.parametrize("window", [0, 100])
def test_linear_cache_one_token(ops, window):
    """One new token, a linear cache (C >= every length), lengths across tile
    edges, including an empty cache."""
    _run(ops, [0, 1, 99, 127, 128, 129, 300, 1000], 1, 16, 2, 1152, window, seed=1)


@pytest.mark.parametrize("Lq", [1, 2, 5])
def test_ring_cache_window(ops, Lq):
    """Sliding-window layer on a ring of exactly window + Lq - 1 slots,
    before and after the ring wraps."""
    W = 128
    _run(ops, [0, 5, 126, 127, 128, 129, 200, 1000], Lq, 16, 2, W + Lq - 1, W, seed=2 + Lq)


def test_small_window_ring_several_tokens(ops):
    """Window 16 on an 18-slot ring with 3 new tokens: the causal mask among
    the new tokens and the window edge both matter."""
    _run(ops, [0, 2, 17, 40, 333], 3, 16, 2, 18, 16, seed=7)


@pytest.mark.parametrize("G,Lq", [(1, 1), (4, 2), (8, 4), (16, 4)])
def test_group_sizes_and_rows(ops, G, Lq):
    """G x Lq query rows per head group from 1 to 64 (every register-tile
    variant of the kernel)."""
    _run(ops, [0, 64, 257], Lq, 2 * G, 2, 512, 0, seed=10 + G)


def test_sink_extremes(ops):
    sinks = [-np.inf, -1e4, 0.0, 1e4, 0.5, -0.5, 3.0, -np.inf]
    for window, C in ((0, 640), (64, 64)):
        _run(ops, [0, 1, 63, 64, 600], 1, 8, 1, C, window, seed=20, sinks=sinks)


def test_wide_cache_with_window_skips_old_slots(ops):
    """A linear cache much longer than the window: only the slot tiles the
    window reaches are visited."""
    _run(ops, [50, 1500, 4000], 1, 16, 2, 4200, 100, seed=30)


@pytest.mark.parametrize("window,C", [(0, 8192), (128, 128)])
def test_gpt_oss_decode_full_size(ops, window, C):
    """gpt-oss heads (Hq 64, Hkv 8), 64 sequences at 8191 cached tokens plus
    one new token: full-causal layer on a linear cache and window-128 layer
    on a 128-slot ring; the oracle checks 6 of the 64 sequences, all heads."""
    cached = [8191] * 62 + [0, 4000]
    _run(ops, cached, 1, 64, 8, C, window, seed=40, seqs=[0, 1, 31, 61, 62, 63])


def test_launch_count(ops):
    assert ops.decode_launches(4, 1, 256, 257, 64, 8) == 3
    assert ops.decode_launches(0, 1, 256, 257, 64, 8) == 0
    assert ops.decode_launches(64, 1, 128, 8192, 64, 8, window=128) == 2


# ----------------------------------------------------------------- e4m3 cache
def _f8pv_bounds(qd, kd, vd, sinks, cu, cached, Lq, window, seqs, ro, rl):
    """Per-element bounds for the FP8 PV variant, from the definition and the
    e4m3 format.  The kernel rounds each unnormalised weight p_j = 2^(x_j - m)
    (m its running reference, with 1 <= max(p, sink term) <= 2^8 and so
    Z = sum p + sink term >= 1) to e4m3: |p~ - p| <= 2^-4 p in e4m3's normal
    range (p >= 2^-6) and <= 2^-10 below it.  With the same p~ in the row
    sums, out~ - out = sum_j (p~_j - p_j)(v_j - out) / Z~, hence (pi_j =
    p_j / Z, the normalised weights; 1 / Z <= pi_max):
      |out~ - out| <= 2^-4 sum_j pi_j |v_j - out| + 2^-10 pi_max sum_j |v_j - out|
      |lse~ - lse| <= 2^-4 sum_j pi_j + 2^-10 pi_max N.
    Returns (out bound [rows, Hq, D], lse bound [Hq, rows]) for the rows of
    `seqs` in the order of ro / rl."""
    Hq = qd.shape[2]
    G = Hq // kd.shape[1]
    ob, lb = [], []
    r = 0
    for b in seqs:
        lo = int(cu[b])
        for t in range(Lq):
            pos = int(cached[b]) + t
            j0 = max(0, pos - window + 1) if window > 0 else 0
            K = kd[lo + j0:lo + pos + 1]  # [N, Hkv, D]
            V = vd[lo + j0:lo + pos + 1]
            ob_r = np.zeros((Hq, kd.shape[2]))
            for h in range(Hq):
                g = h // G
                logits = SCALE * (K[:, g] @ qd[b, t, h])
                pi = np.exp(logits - rl[h, r])
                dev_ = np.abs(V[:, g] - ro[r, h][None, :])  # [N, D]
                ob_r[h] = 2.0 ** -4 * (pi[:, None] * dev_).sum(0) + 2.0 ** -10 * pi.max() * dev_.sum(0)
                lb.append((h, r, 2.0 ** -4 * pi.sum() + 2.0 ** -10 * pi.max() * len(pi)))
            ob.append(ob_r)
            r += 1
    lbound = np.zeros((Hq, r))
    for h, rr, v in lb:
        lbound[h, rr] = v
    return np.stack(ob), lbound


def _run_e4m3(ops, cached, Lq, Hq, Hkv, C, window, seed, seqs=None, heavy=False, f8pv=False):
    """The e4m3-cache decode: history tokens enter the cache as host-quantised
    codes (per-head scale = amax / 448), the new tokens are quantised by the
    call.  The oracle gets the dequantised values code * scale exactly (fp64),
    so the comparison measures the kernel, not the quantisation.  heavy: the
    history slots instead hold codes drawn uniformly over every finite e4m3
    code of both signs (scale 1/64): heavy-tailed logits, so the running
    reference max of a row is raised on many tiles, not just the first."""
    import torch
    from tests import e4m3
    a = synth.decode_inputs(seed, cached, Lq, Hq, Hkv)
    cu = a["cu"]
    B = len(cached)
    kf = synth.bf16_bits_to_f32(a["k"])
    vf = synth.bf16_bits_to_f32(a["v"])
    if heavy:
        ks = np.full(Hkv, 1.0 / 64.0, np.float32)
        vs = np.full(Hkv, 1.0 / 64.0, np.float32)
    else:
        ks = (np.abs(kf).max(axis=(0, 2)) / np.float32(448.0)).astype(np.float32)
        vs = (np.abs(vf).max(axis=(0, 2)) / np.float32(448.0)).astype(np.float32)
    ck = e4m3.quantize(kf * (np.float32(1.0) / ks)[None, :, None])
    cv = e4m3.quantize(vf * (np.float32(1.0) / vs)[None, :, None])
    if heavy:
        rng = np.random.default_rng(seed)
        hist = np.concatenate([np.arange(int(cu[b]), int(cu[b]) + int(cached[b])) for b in range(B)]).astype(np.int64)
        for c in (ck, cv):
            shape = (len(hist), Hkv, 64)
            c[hist] = (rng.integers(0, 0x7F, size=shape) | (rng.integers(0, 2, size=shape) << 7)).astype(np.uint8)
    kc0 = np.full((B, C, Hkv, 64), 0x7F, np.uint8)  # unused slots hold the NaN code
    vc0 = np.full((B, C, Hkv, 64), 0x7F, np.uint8)
    for b in range(B):
        for p in range(int(cached[b])):
            kc0[b, p % C] = ck[int(cu[b]) + p]
            vc0[b, p % C] = cv[int(cu[b]) + p]
    new_idx = np.concatenate([np.arange(int(cu[b]) + int(cached[b]), int(cu[b + 1])) for b in range(B)])
    k_new = a["k"][new_idx].reshape(B, Lq, Hkv, 64)
    v_new = a["v"][new_idx].reshape(B, Lq, Hkv, 64)
    kc, vc = torch.from_numpy(kc0).cuda(), torch.from_numpy(vc0).cuda()
    call = ops.decode_e4m3_f8pv if f8pv else ops.decode_e4m3
    out, lse = call(dev_bf16(a["q_new"]), dev_bf16(k_new), dev_bf16(v_new), kc, vc, dev(np.asarray(cached, np.int32)),
                    dev(ks), dev(vs), dev(a["sinks"]), window, SCALE, max_seqlen=int(max(cached)) + Lq)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    ke, ve = kc0.copy(), vc0.copy()
    for b in range(B):
        for t in range(Lq):
            ke[b, (int(cached[b]) + t) % C] = ck[int(cu[b]) + int(cached[b]) + t]
            ve[b, (int(cached[b]) + t) % C] = cv[int(cu[b]) + int(cached[b]) + t]
    assert np.array_equal(kc.cpu().numpy(), ke), "e4m3 k cache after append (quantisation of the new tokens)"
    assert np.array_equal(vc.cpu().numpy(), ve), "e4m3 v cache after append"
    kd = e4m3.decode(ck) * ks[None, :, None].astype(np.float64)
    vd = e4m3.decode(cv) * vs[None, :, None].astype(np.float64)
    qd = synth.bf16_bits_to_f32(a["q_new"]).astype(np.float64)
    seqs = list(range(B)) if seqs is None else list(seqs)
    outs, lses = [], []
    for b in seqs:
        lo, hi = int(cu[b]), int(cu[b + 1])
        L = hi - lo
        q = np.zeros((L, Hq, 64))
        q[int(cached[b]):] = qd[b]
        rows = np.arange(int(cached[b]), L, dtype=np.int64)
        o, l = oracle.fwd_rows(q, kd[lo:hi], vd[lo:hi], a["sinks"].astype(np.float64), np.array([0, L], np.int32),
                               window, SCALE, rows)
        outs.append(o)
        lses.append(l)
    got_o = host_f64(out)[seqs].reshape(-1, Hq, 64)
    got_l = host_f64(lse).reshape(Hq, B, Lq)[:, seqs].reshape(Hq, -1)
    ro, rl = np.concatenate(outs), np.concatenate(lses, axis=1)
    if not f8pv:
        check(got_o, ro, TOL_OUT, "e4m3 decode out")
        check(got_l, rl, TOL_LSE, "e4m3 decode lse")
        return
    # FP8 PV: P is rounded to e4m3 before the MMA; the bound of that rounding
    # (_f8pv_bounds) plus the usual budget for the other roundings.
    qd_new = qd.reshape(B, Lq, Hq, 64)
    ob, lb = _f8pv_bounds(qd_new, kd, vd, a["sinks"], cu, cached, Lq, window, seqs, ro, rl)
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_l)), "FP8 PV decode: non-finite values"
    eo = np.abs(got_o - ro)
    assert np.all(eo <= 1.05 * ob + TOL_OUT * np.abs(ro).max()), \
        f"FP8 PV decode out beyond its bound: worst excess {np.max(eo - 1.05 * ob - TOL_OUT * np.abs(ro).max()):.3e}"
    el = np.abs(got_l - rl)
    assert np.all(el <= 1.05 * lb + TOL_LSE * np.abs(rl).max()), \
        f"FP8 PV decode lse beyond its bound: worst excess {np.max(el - 1.05 * lb - TOL_LSE * np.abs(rl).max()):.3e}"
    print(f"FP8 PV decode: out error {eo.max():.3e} (bound max {ob.max():.3e}), lse error {el.max():.3e}")


@pytest.mark.parametrize("window,C,Lq", [(0, 1152, 1), (100, 1152, 1), (128, 128, 1), (128, 129, 2), (16, 18, 3)])
def test_e4m3_cache(ops, window, C, Lq):
    _run_e4m3(ops, [0, 1, 99, 127, 128, 129, 300, 1000], Lq, 16, 2, C, window, seed=60 + Lq)


@pytest.mark.parametrize("G,Lq", [(8, 4), (16, 4)])
def test_e4m3_cache_row_variants(ops, G, Lq):
    _run_e4m3(ops, [0, 64, 257], Lq, 2 * G, 2, 512, 0, seed=70 + G)


@pytest.mark.parametrize("window", [0, 100])
def test_e4m3_cache_heavy_tailed(ops, window):
    """Many reference-max raises per CTA in the e4m3 variant (each one a CTA
    vote, an exact tile max and a rescale of O)."""
    _run_e4m3(ops, [1000, 2000, 4095, 3], 1, 16, 2, 4096, window, seed=90 + window, heavy=True)


@pytest.mark.parametrize("window,C", [(0, 8192), (128, 128)])
def test_e4m3_cache_gpt_oss_full_size(ops, window, C):
    """gpt-oss heads, 64 sequences: the full-causal layer's 8192-slot cache
    is split over several CTAs and combined; the window-128 layer's 128-slot
    ring fits one CTA per (sequence, key/value head), which then finishes
    the rows itself (no combine launch)."""
    _run_e4m3(ops, [8191] * 62 + [0, 4000], 1, 64, 8, C, window, seed=80, seqs=[0, 31, 62, 63])


# -------------------------------------------- e4m3 cache, FP8 PV product
@pytest.mark.parametrize("window,C,Lq", [(0, 1152, 1), (100, 1152, 1), (128, 128, 1), (128, 129, 2), (16, 18, 3)])
def test_e4m3_f8pv(ops, window, C, Lq):
    """sink_attn_decode_e4m3_f8pv: the PV product on the FP8 tensor-core path
    (P rounded to e4m3), against the oracle within the bound that rounding
    implies; the cache after append is checked bit for bit."""
    _run_e4m3(ops, [0, 1, 99, 127, 128, 129, 300, 1000], Lq, 16, 2, C, window, seed=160 + Lq, f8pv=True)


@pytest.mark.parametrize("G,Lq", [(1, 1), (8, 1), (8, 4), (16, 4)])
def test_e4m3_f8pv_row_variants(ops, G, Lq):
    """Every register-tile variant (8, 16, 32, 64 query rows)."""
    _run_e4m3(ops, [0, 64, 257], Lq, 2 * G, 2, 512, 0, seed=170 + G, f8pv=True)


@pytest.mark.parametrize("window,C", [(0, 8192), (128, 128)])
def test_e4m3_f8pv_gpt_oss_full_size(ops, window, C):
    """gpt-oss heads, 64 sequences at 8191 cached tokens + 1 (split and
    combined on the 8192-slot cache; one CTA per head group on the ring)."""
    _run_e4m3(ops, [8191] * 62 + [0, 4000], 1, 64, 8, C, window, seed=180, seqs=[0, 31, 62, 63], f8pv=True)
