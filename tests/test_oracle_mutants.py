"""Each planted mistake in the oracle is caught by at least one pin.

The oracle source itself holds no planted mistake.  Each test copies
``oracle/lse_merge_oracle.c`` into a temporary directory, changes one
statement of the copy by a text substitution (a plausible slip in writing the
method down: a dropped term, a flipped sign, a swapped index, a skipped
branch), compiles that copy, and runs every pin against it in a child
process, so that a mistake that indexes out of range can only crash the
child.  The substitution must match exactly once, so a later edit of the
oracle that moves a statement makes the test fail loudly instead of testing
nothing.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# name -> (statement as it stands in the oracle, the same statement with the mistake)
MUTANTS = {
    "merged lse without the max term": (
        "*olse = m + log(denom);",
        "*olse = log(denom);"),
    "weight exponent with the sign flipped": (
        "double e = exp(l - m);",
        "double e = exp(m - l);"),
    "batch and head strides swapped": (
        "const int64_t o_row = (int64_t)b * os[1] + (int64_t)h * os[2];\n"
        "            const int64_t l_row = (int64_t)b * ls[1] + (int64_t)h * ls[2];",
        "const int64_t o_row = (int64_t)b * os[2] + (int64_t)h * os[1];\n"
        "            const int64_t l_row = (int64_t)b * ls[2] + (int64_t)h * ls[1];"),
    "empty shards not skipped (0 * NaN leaks)": (
        "if (l == -INFINITY) continue;",
        ";"),
    "plain mean instead of lse weights": (
        "for (int d = 0; d < D; ++d) out[d] /= denom;",
        "for (int d = 0; d < D; ++d) out[d] /= (double)R;"),
    "first shard dropped": (
        "for (int r = 0; r < R; ++r) {\n"
        "                double l = (double)partial_lse[l_row + (int64_t)r * ls[0]];\n"
        "                if (l == -INFINITY) continue;",
        "for (int r = 1; r < R; ++r) {\n"
        "                double l = (double)partial_lse[l_row + (int64_t)r * ls[0]];\n"
        "                if (l == -INFINITY) continue;"),
    "state update with its two weights swapped": (
        "const double ea = (la == -INFINITY) ? 0.0 : exp(la - m);\n"
        "            const double en = (ln == -INFINITY) ? 0.0 : exp(ln - m);",
        "const double en = (la == -INFINITY) ? 0.0 : exp(la - m);\n"
        "            const double ea = (ln == -INFINITY) ? 0.0 : exp(ln - m);"),
    "exchange: owner's head offset dropped": (
        "const int64_t h0 = (int64_t)q * Hq;",
        "const int64_t h0 = 0;"),
}

CHILD = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pins import ALL_PINS
lib = oracle.load({path!r})
caught = []
for pin in ALL_PINS:
    try:
        pin(lib)
    except Exception as exc:
        caught.append(pin.__name__)
print("CAUGHT", ",".join(caught))
"""


def planted_source(tmp_path, name: str) -> str:
    """A copy of the oracle source with the mistake `name` planted in it."""
    good, bad = MUTANTS[name]
    with open(oracle.SRC) as fh:
        src = fh.read()
    assert src.count(good) == 1, f"the statement of mutant {name!r} is not in the oracle exactly once"
    path = tmp_path / "lse_merge_oracle_planted.c"
    path.write_text(src.replace(good, bad))
    return str(path)


def test_the_oracle_source_holds_no_planted_mistake():
    with open(oracle.SRC) as fh:
        src = fh.read()
    for name, (good, bad) in MUTANTS.items():
        assert src.count(good) == 1, name
        assert bad not in src or bad in good, name


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    path = str(tmp_path / "liboracle_planted.so")
    oracle.build(path, src=planted_source(tmp_path, name))
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), path=path)
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=300)
    if proc.returncode != 0:
        # the mutant crashed the child process: that is a detection as well
        return
    line = [l for l in proc.stdout.splitlines() if l.startswith("CAUGHT")][-1]
    caught = [c for c in line[len("CAUGHT "):].split(",") if c]
    assert caught, f"mutant {name!r} passed every pin"
