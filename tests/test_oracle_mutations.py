"""Plants plausible mistakes in copies of the oracle's C source (on the
CPU, never in the committed file) and checks that the pins catch each one.
This shows the pins constrain every part of the oracle that a mistake could
hit: the sink term, the window edge, the GQA mapping, the scale, lse, and
each term of the backward pass."""
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

import oracle
from tests import oracle_pins

_SAVED_OUT = "const double* o = out_for_D ? out_for_D + (t * Hq + h) * (int64_t)D : orow;"

# name -> (anchor, replacement[, which occurrence of the anchor, default 0])
MUTATIONS = {
    "sink dropped from the denominator": ("double Z = exp(sink - m);", "double Z = 0.0 * exp(sink - m);"),
    "window one key too wide": ("int64_t lo = t - (int64_t)window + 1;", "int64_t lo = t - (int64_t)window;"),
    "GQA head mapping h % Hkv": ("const int g = h / G;", "const int g = h % Hkv;"),
    "scale not applied": ("double l = scale * dot;", "double l = dot;"),
    "sink scaled like a logit": ("double m = sink;", "sink = sink * scale; double m = sink;"),
    "lse without the log": ("return m + log(Z);", "return m + Z;"),
    "row max ignores the sink": ("double m = sink;", "double m = -INFINITY;"),
    "dS without the D term": ("double dS = P * (dP - Di);", "double dS = P * dP;"),
    "dsink sign": ("dsink_part[task * G + hh] -= exp(sinks[h] - lse) * Di;",
                   "dsink_part[task * G + hh] += exp(sinks[h] - lse) * Di;"),
    "dv uses q": ("dvj[d] += P * doi[d];", "dvj[d] += P * qi[d];"),
    "dk misses scale": ("dkj[d] += scale * dS * qi[d];", "dkj[d] += dS * qi[d];"),
    "dq uses v": ("dqi[d] += scale * dS * kj[d];", "dqi[d] += scale * dS * vj[d];"),
    "documents not respected": ("int64_t a = cu_seqlens[doc_of(cu_seqlens, B, t)];", "int64_t a = 0;"),
    # The saved output used for D_i (out_for_D): the same line sits in the
    # full backward (occurrence 0), the dsinks-only one (1), the dq-rows one
    # (2) and the dk/dv-rows one (3); each is mutated on its own.
    **{f"saved output ignored ({where})": (_SAVED_OUT, "const double* o = orow;", n)
       for n, where in ((0, "bwd"), (1, "dsinks alone"), (2, "dq rows"), (3, "dk/dv rows"))},
    **{f"saved output indexed [Hq][T] ({where})": (
        _SAVED_OUT, "const double* o = out_for_D ? out_for_D + ((int64_t)h * T + t) * (int64_t)D : orow;", n)
       for n, where in ((0, "bwd"), (1, "dsinks alone"), (2, "dq rows"), (3, "dk/dv rows"))},
    "dsinks alone: sink term sign": ("term[(int64_t)h * T + t] = exp(sinks[h] - lse) * Di;",
                                     "term[(int64_t)h * T + t] = -exp(sinks[h] - lse) * Di;"),
    "dsinks alone: lse of the wrong sign": ("term[(int64_t)h * T + t] = exp(sinks[h] - lse) * Di;",
                                            "term[(int64_t)h * T + t] = exp(sinks[h] + lse) * Di;"),
    "saved output widened from dout (bf16 bwd)": (
        "double* od = out_for_D_bf16 ? widen(out_for_D_bf16, (int64_t)T * Hq * D) : NULL;",
        "double* od = out_for_D_bf16 ? widen(dout, (int64_t)T * Hq * D) : NULL;"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


_RUNNER = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import oracle_pins
O = oracle.Oracle({lib!r})
failed = []
for pin in oracle_pins.ALL_PINS:
    try:
        pin(O)
    except (AssertionError, RuntimeError, ValueError) as e:
        failed.append(pin.__name__)
print("FAILED_PINS", failed)
sys.exit(3 if failed else 0)
"""


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(workdir, name):
    old, new, *nth = MUTATIONS[name]
    nth = nth[0] if nth else 0
    src = open(oracle.SOURCE).read()
    assert src.count(old) > nth, f"mutation anchor not found: {old} (occurrence {nth})"
    at = -1
    for _ in range(nth + 1):
        at = src.index(old, at + 1)
    mutated = src[:at] + new + src[at + len(old):]
    tag = "".join(c if c.isalnum() else "_" for c in name)
    path = os.path.join(workdir, f"{tag}.c")
    with open(path, "w") as f:
        f.write(mutated)
    lib = oracle.build(force=True, src=path, out=os.path.join(workdir, f"lib{tag}.so"))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    # A mutated oracle may also crash (e.g. index past its scratch buffer) or
    # hang; run it in a child process: any non-zero exit is a catch.
    env = dict(os.environ, OMP_NUM_THREADS="2")
    try:
        r = subprocess.run([sys.executable, "-c", _RUNNER.format(root=root, lib=lib)],
                           capture_output=True, text=True, timeout=300, env=env)
        caught = r.returncode != 0
        detail = (r.stdout + r.stderr)[-300:]
    except subprocess.TimeoutExpired:
        caught, detail = True, "timed out"
    assert caught, f"no pin caught the mutation '{name}': {detail}"
