"""Planted mistakes in the oracle (on the CPU): each mutation of nm_oracle.c
must make at least one pin in test_oracle_pins.py fail.  The mutated copy is
built and tested in a temporary directory; the committed oracle is untouched."""
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    ("run = run + sq;", "run = run + sq + sq;"),                           # doubled term
    ("part = part + run;", "part = run;"),                                 # dropped run
    ("H[j] = total / (double)T;", "H[j] = total / (double)(T + 1);"),     # wrong divisor
    ("(s[p] == s[q] && p < q)", "(s[p] == s[q] && p > q)"),               # tie direction
    ("if (rank < n) idx", "if (rank <= n) idx"),                          # off by one
    ("double h = H[j] + eps;", "double h = H[j];"),                       # dropped eps
    ("uint8_t nib = (uint8_t)(idx[0] | (idx[1] << 2));",
     "uint8_t nib = (uint8_t)(idx[1] | (idx[0] << 2));"),                 # swapped nibble
    ("int a = q[2 * w] - 2 * w, b = q[2 * w + 1] - 2 * w;",
     "int a = q[2 * w] - w, b = q[2 * w + 1] - w;"),                      # window offset
    ("int64_t src = g * m + 2 * w + c;", "int64_t src = g * m + w + c;"),  # lift stride
    ("vals[i * (G * n) + g * n + k] = v[idx[k]];",
     "vals[i * (G * n) + g * n + k] = v[k];"),                            # wrong value index
    ("double p = bf16_to_f64(X[t * ldx + k]) * bf16_to_f64(V[r * ldv + k]);",
     "double p = bf16_to_f64(X[k * ldx + t]) * bf16_to_f64(V[r * ldv + k]);"),  # transposed
    ("s[q] = 0.0f; /* zero-padded tail */", "s[q] = 1e30f;"),              # padding wins
    ("double q = rint(", "double q = round("),                             # ties away
    ("(d == bd && (c & 1) == 0)", "(d == bd && (c & 1) == 1)"),           # e4m3 ties to odd
    ("amax > 0.0f ? amax / 448.0f", "amax > 0.0f ? amax / 447.0f"),       # fp8 scale
]


@pytest.mark.slow
@pytest.mark.parametrize("old,new", MUTATIONS)
def test_planted_mistake_is_caught(old, new):
    src = open(os.path.join(ROOT, "oracle", "nm_oracle.c")).read()
    assert old in src, old
    with tempfile.TemporaryDirectory() as d:
        for sub in ("oracle", "datagen", "tests"):
            shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub),
                            ignore=shutil.ignore_patterns("*.so", "__pycache__"))
        with open(os.path.join(d, "oracle", "nm_oracle.c"), "w") as f:
            f.write(src.replace(old, new))
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            "tests/test_oracle_pins.py"], cwd=d, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode != 0, "mutation not caught: " + new
