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
    ("count[e] += m * m;", "count[e] += m;"),                             # dropped square
    ("H[j] = sum / (double)T;", "H[j] = sum / (double)(T + 1);"),         # wrong divisor
    ("uint64_t m = e ? (uint64_t)(128 + f) : (uint64_t)f;",
     "uint64_t m = (uint64_t)(128 + f);"),                                # subnormal hidden bit
    ("big_add_shifted(n, count[e], 2 * (e ? e : 1));",
     "big_add_shifted(n, count[e], 2 * e);"),                             # subnormal exponent
    ("if (round_bit && (sticky || (sig & 1u))) sig += 1;",
     "if (round_bit) sig += 1;"),                                         # ties away from zero
    ("sticky = (int)BIT(p);", "sticky = 0;"),                             # dropped sticky bits
    ("double s = h * w2;", "float s = (float)h * (float)w2;"),            # fp32 arithmetic in S
    ("double h = H[j] + eps;", "float h = (float)H[j] + (float)eps;"),    # fp32 add in S
    ("mine[e] += e ? (uint64_t)(128 + f) : (uint64_t)f;",
     "mine[e] += e ? (uint64_t)(128 + f) : 0;"),                          # gamma drops subnormals
    ("double gamma = total / ((double)R * (double)K);",
     "double gamma = total / ((double)R * (double)(K + 1));"),             # gamma divisor
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


def _run_mutation(old, new):
    """Build the oracle with one planted mistake in a temporary copy and run
    the pins against it; returns the pins' exit status (non-zero = caught)."""
    src = open(os.path.join(ROOT, "oracle", "nm_oracle.c")).read()
    assert old in src, old
    with tempfile.TemporaryDirectory() as d:
        for sub in ("oracle", "datagen", "tests"):
            shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub),
                            ignore=shutil.ignore_patterns("*.so", "__pycache__"))
        with open(os.path.join(d, "oracle", "nm_oracle.c"), "w") as f:
            f.write(src.replace(old, new))
        env = dict(os.environ, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            "tests/test_oracle_pins.py"], cwd=d, capture_output=True, text=True,
                           timeout=600, env=env)
        return r.returncode


@pytest.fixture(scope="module")
def mutation_results():
    # the mutated builds run side by side (each pins run stops at its first failure)
    from concurrent.futures import ThreadPoolExecutor
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {m: ex.submit(_run_mutation, *m) for m in MUTATIONS}
        return {m: f.result() for m, f in futs.items()}


@pytest.mark.slow
@pytest.mark.parametrize("old,new", MUTATIONS)
def test_planted_mistake_is_caught(old, new, mutation_results):
    assert mutation_results[(old, new)] != 0, "mutation not caught: " + new
