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
    old, new = MUTATIONS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    mutated = src.replace(old, new, 1)
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
