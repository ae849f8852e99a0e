"""The oracle's pins must catch plausible mistakes.

Each case compiles a copy of ``oracle/attn_oracle.c`` with one deliberate
error (a dropped term, a wrong sign or index, a transposed operand, a changed
constant), points the oracle module at it through ORACLE_LIB, and runs the pin
tests in a subprocess: at least one pin has to fail.  CPU only.
"""
import os
import subprocess
import sys

import pytest

from oracle import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attn_oracle.c")

# (name, text to find, replacement, -k expression selecting the pins that should catch it)
MUTANTS = [
    ("causal mask drops the diagonal", "return causal ? i + 1 : N;", "return causal ? (i > 0 ? i : 1) : N;",
     "closed or brute or worked or torch"),
    ("LSE without the row max", "*lse_i = m + log(l);", "*lse_i = log(l);", "closed or brute or torch"),
    ("naive softmax not normalised", "for (long j = 0; j < n; ++j) w[j] /= l;", "",
     "worked or online or softmax"),
    ("online sum not rescaled", "l = (m == -INFINITY ? 0.0 : l * exp(m - m_new)) + add;",
     "l = (m == -INFINITY ? 0.0 : l) + add;", "worked or online or softmax"),
    ("tiled O not rescaled", "for (long t = 0; t < d; ++t) oi[t] *= alpha;", "", "block or tiled or demo"),
    ("backward drops D", "double ds = prow[j] * (dprow[j] - D);", "double ds = prow[j] * dprow[j];",
     "bwd or backward or grad or finite or autograd"),
    ("dK uses K instead of Q", "dkj[t] += ds * qi[t];", "dkj[t] += ds * kj[t];",
     "bwd or backward or grad or finite or autograd"),
    ("rectangular causal aligned top-left", "const long nk = causal ? Nk - Nq + i + 1 : Nk;",
     "const long nk = causal ? i + 1 : Nk;", "rect"),
    ("block mask causal excludes the diagonal", "(!causal || j <= i)", "(!causal || j < i)", "blockmask"),
    ("Philox multiplier changed", "0xD2E7470EE14C6C93ull", "0xD2E7470EE14C6C95ull", "philox or dropout"),
    ("dropout bytes taken in the wrong order", "(w[b / 8] >> (8 * (b % 8)))", "(w[b % 4] >> (8 * (b / 4 % 8)))",
     "philox or dropout"),
    ("dropout scale 255 / t", "const double s_keep = t > 0 ? 256.0 / t : 0.0;",
     "const double s_keep = t > 0 ? 255.0 / t : 0.0;", "dropout"),
    ("dropout dV from the undropped weights", "const double pz = prow[j] * zrow[j];", "const double pz = prow[j];",
     "dropout"),
    ("head backward: key pass skips the diagonal query", "for (long i = causal ? j : 0; i < N; ++i) {",
     "for (long i = causal ? j + 1 : 0; i < N; ++i) {", "head"),
    ("head backward: weight from the key's row statistics", "- rm[i]) / rl[i];", "- rm[j]) / rl[i];", "head"),
    ("head backward: dV ignores the dropout mask", "const double pz = p * z;", "const double pz = p;", "head"),
]


@pytest.mark.parametrize("name,find,repl,kexpr", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_the_mutant(tmp_path, name, find, repl, kexpr):
    src = open(SRC).read()
    assert src.count(find) >= 1, "mutation site not found: %s" % find
    mutated = tmp_path / "attn_oracle_mutant.c"
    mutated.write_text(src.replace(find, repl, 1))
    lib = str(tmp_path / "liboracle_mutant.so")
    oracle.compile_source(str(mutated), lib)
    env = dict(os.environ, ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"), "-k", kexpr],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    # pytest exits 1 when a test failed; 0 would mean every selected pin passed
    assert r.returncode == 1, "mutant '%s' survived (exit %d):\n%s" % (name, r.returncode, r.stdout[-2000:])


def test_unmutated_source_passes_the_same_selection(tmp_path):
    """Control: the real source, built the same way, passes every selection above."""
    lib = str(tmp_path / "liboracle_copy.so")
    oracle.compile_source(SRC, lib)
    kexpr = " or ".join("(%s)" % m[3] for m in MUTANTS)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"), "-k", kexpr],
                       cwd=ROOT, env=dict(os.environ, ORACLE_LIB=lib), capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
