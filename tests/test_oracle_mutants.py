"""Each planted mistake in the oracle is caught by at least one pin.

The mutants are compiled from the oracle source with -DORACLE_MUTANT=k into a
temporary directory and checked in a child process, so that a mutant that
indexes out of range can only crash the child.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MUTANTS = {
    1: "merged lse without the max term",
    2: "weight exponent with the sign flipped",
    3: "batch and head strides swapped",
    4: "empty shards not skipped (0 * NaN leaks)",
    5: "plain mean instead of lse weights",
    6: "first shard dropped",
    7: "state update with its two weights swapped",
    8: "exchange: owner's head offset dropped",
}

CHILD = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pins import ALL_PINS
lib = oracle.load({path!r})
assert lib.oracle_mutant() == {k}
caught = []
for pin in ALL_PINS:
    try:
        pin(lib)
    except Exception as exc:
        caught.append(pin.__name__)
print("CAUGHT", ",".join(caught))
"""


@pytest.mark.parametrize("k", sorted(MUTANTS), ids=lambda k: MUTANTS[k])
def test_mutant_is_caught(tmp_path, k):
    path = str(tmp_path / f"liboracle_m{k}.so")
    oracle.build(path, mutant=k)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), path=path, k=k)
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=300)
    if proc.returncode != 0:
        # the mutant crashed the child process: that is a detection as well
        return
    line = [l for l in proc.stdout.splitlines() if l.startswith("CAUGHT")][-1]
    caught = [c for c in line[len("CAUGHT "):].split(",") if c]
    assert caught, f"mutant {k} ({MUTANTS[k]}) passed every pin"
