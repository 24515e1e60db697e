"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that the pins catch every one of them.  The real oracle source is never
modified: each mutant is a textual edit of a temporary copy, compiled to its
own shared library."""
import os
import subprocess
import tempfile

import pytest

import oracle
from tests.oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

# (name, original text, planted text)
MUTANTS = [
    ("wrong sign of the prediction",
     "u[a] = x.beta * (x.v[a] - acc);", "u[a] = x.beta * (x.v[a] + acc);"),
    ("dropped writing strength",
     "u[a] = x.beta * (x.v[a] - acc);", "u[a] = (x.v[a] - acc);"),
    ("read-out of the pre-update state",
     "oa += row[c] * (scale * x.q[c]);",
     "oa += (row[c] - u[a] * x.k[c]) * (scale * x.q[c]);"),
    ("transposed state in the prediction",
     "for (int c = 0; c < dk; ++c) acc += row[c] * x.k[c];",
     "for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dk + a] * x.k[c];"),
    ("channel decay on the value index",
     "for (int c = 0; c < dk; ++c) row[c] *= exp(x.g[c]);",
     "for (int c = 0; c < dk; ++c) row[c] *= exp(x.g[a]);"),
    ("scale dropped from the read-out",
     "oa += row[c] * (scale * x.q[c]);", "oa += row[c] * x.q[c];"),
    ("backward: dropped Sh^T dp term of dk",
     "dkt[c] += acc;", "dkt[c] += 0.0 * acc;"),
    ("backward: scalar dg without the chain factor a",
     "dg[th] = s * al;", "dg[th] = s;"),
    ("backward: channel dg without the chain factor a",
     "dg[th * dk + c] = da[c] * al;", "dg[th * dk + c] = da[c];"),
    ("backward: dv without beta",
     "dvt[a] = x.beta * du[a];", "dvt[a] = du[a];"),
    ("backward: wrong sign in dbeta",
     "db += du[a] * (x.v[a] - p[a]);", "db += du[a] * (x.v[a] + p[a]);"),
    ("backward: state gradient not decayed",
     "for (size_t e = 0; e < ss; ++e) dS[e] *= al;", "(void)ss;"),
]


def _build_mutant(old, new, tmpdir):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    src = src.replace(old, new, 1)
    c = os.path.join(tmpdir, "m.c")
    so = os.path.join(tmpdir, "m.so")
    open(c, "w").write(src)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                    so, c, "-lm"], check=True)
    return oracle.load_library(so)


def _failed_pins(lib):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a mutant's numbers may overflow
@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new):
    with tempfile.TemporaryDirectory() as d:
        lib = _build_mutant(old, new, d)
        failed = _failed_pins(lib)
    assert failed, f"no pin caught the planted mistake: {name}"
