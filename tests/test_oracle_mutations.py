"""The oracle pins must reject plausible mistakes.

Each case plants one mistake in a private copy of oracle.c (on the CPU, in a
temporary directory), builds it, and runs the pin suite against it in a
subprocess: the suite has to fail. This shows the pins of test_oracle.py are
not vacuous for the kinds of error an implementation of these equations
typically makes.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    # rotation direction of the second component flipped
    "rope_sign": ("y[base + 2 * m + 1] = x0 * s + x1 * c;",
                  "y[base + 2 * m + 1] = x0 * s - x1 * c;"),
    # half-split pairing (m, m + d/2) instead of adjacent pairs
    "rope_pairing": ("double x0 = x[base + 2 * m], x1 = x[base + 2 * m + 1];",
                     "double x0 = x[base + m], x1 = x[base + m + d / 2];"),
    # frequency exponent without the factor 2
    "rope_frequency": ("pow(p->theta, -2.0 * (double)m / (double)d)",
                       "pow(p->theta, -1.0 * (double)m / (double)d)"),
    # the axes of h and w swapped
    "rope_axes": ("pos[1] = (n / p->grid_w) % p->grid_h;", "pos[1] = n % p->grid_w;"),
    # transposed state in the numerator
    "state_transposed": ("num += qr[a] * S[(size_t)a * D + c];",
                         "num += qr[a] * S[(size_t)c * D + a];"),
    # rotated query in the denominator (Eq. 2 keeps it un-rotated)
    "den_rotated": ("for (int a = 0; a < D; ++a) den += qphi[a] * z[a];",
                    "for (int a = 0; a < D; ++a) den += qr[a] * z[a];"),
    # eps dropped
    "no_eps": ("den += p->eps;\n  for (int c = 0; c < D; ++c) {",
               "den += 0.0;\n  for (int c = 0; c < D; ++c) {"),
    # ReLU dropped on the keys
    "no_relu_k": ("kphi[a] = relu((double)k_head[(size_t)j * D + a]);",
                  "kphi[a] = (double)k_head[(size_t)j * D + a];"),
    # block-causal apply state forgets the carried state
    "block_no_carry": ("for (size_t e = 0; e < (size_t)D * D; ++e) Sap[e] = S[e] + Sblk[e];\n      for (int a = 0; a < D; ++a) zap[a] = z[a] + zblk[a];\n      if (oh)",
                       "for (size_t e = 0; e < (size_t)D * D; ++e) Sap[e] = Sblk[e];\n      for (int a = 0; a < D; ++a) zap[a] = z[a] + zblk[a];\n      if (oh)"),
    # gate applied as sigmoid(-g)
    "gate_sign": ("o *= 1.0 / (1.0 + exp(-gl));", "o *= 1.0 / (1.0 + exp(gl));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: " + name
    mut = tmp_path / "oracle_mutant.c"
    mut.write_text(src.replace(old, new, 1))
    env = dict(os.environ, ORACLE_SRC=str(mut), ORACLE_LIB=str(tmp_path / "liborc_mutant.so"))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins accepted the mutant %s:\n%s" % (name, r.stdout[-2000:])
