"""The multi-threaded oracle driver (used only to time the CPU baseline on
every host core) gives exactly the single-threaded oracle's result: it only
splits the batch axis and calls the same function on each range."""
import numpy as np
import pytest

import oracle
from lse_weighted_merge_b200 import synth


@pytest.mark.parametrize("name,B,threads", [
    ("r16_b512_h16_d512", 7, 3),            # [B,H,R,D], ranges of unequal length
    ("r8_b256_h64_d128_rankmajor", 5, 0),   # [R,B,H,D], one thread per core (capped at B)
    ("r4_b64_h32_d128_masked", 9, 4),       # empty shards and rows
])
def test_threads_equal_one_thread(name, B, threads):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, B=B)
    args = (inp["o"], inp["lse"], inp["R"], inp["B"], inp["H"], inp["D"], inp["o_strides"],
            inp["lse_strides"], synth.DTYPES[w.in_dtype])
    one = oracle.merge(*args)
    st = {}
    many = oracle.merge(*args, threads=threads, stats=st)
    assert 1 <= st["threads"] <= B
    if threads:
        assert st["threads"] == min(threads, B)
    assert np.array_equal(one[0], many[0])
    assert np.array_equal(one[1], many[1])
