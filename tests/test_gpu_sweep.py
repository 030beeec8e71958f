"""A seeded random sweep of merge shapes around the AUTO planner's boundaries
(R near 16, row slices near 128, partials near 8 MB, ragged and 16-byte D,
both layouts, every dtype pair), each checked against the fp64 oracle.  The
planner's choice is read back through lse_merge_plan_query, and a host-side
test checks that the cases take every kernel path."""
import numpy as np
import pytest
import torch

from gpu_util import TORCH_DT, parity, upload
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import synth

DTS = ("f32", "f16", "bf16")


def _cases(n=48, seed=2024):
    rng = np.random.Generator(np.random.PCG64(seed))
    base = synth.WORKLOADS["r4_b64_h32_d128_masked"]
    out = []
    for i in range(n):
        kind = i % 4
        if i % 8 == 7:     # R > 16 over many rows: the persistent kernel's long form
            R, B, H = int(rng.choice([17, 20, 33])), int(rng.choice([64, 128])), 64
            D = int(rng.choice([128, 200, 256]))
            ind, outd = DTS[int(rng.integers(0, 3))], DTS[int(rng.integers(0, 3))]
            layout = "bhrd" if rng.random() < 0.6 else "rbhd"
            out.append(dict(R=R, B=B, H=H, D=D, in_dtype=ind, out_dtype=outd, layout=layout,
                            seed=3000 + i, base=base))
            continue
        if kind == 0:      # few rows: LATENCY / WIDE boundary
            R, B, H = int(rng.integers(1, 40)), int(rng.integers(1, 4)), int(rng.integers(1, 9))
        elif kind == 1:    # R around 16: STREAM/VECTOR vs WIDE
            R, B, H = int(rng.choice([15, 16, 17, 24, 33])), int(rng.integers(8, 40)), 16
        elif kind == 2:    # row slices around 128
            R, B, H = int(rng.integers(2, 9)), int(rng.integers(1, 10)), int(rng.integers(8, 33))
        else:              # partials around 8 MB
            R, B, H = 8, int(rng.choice([60, 64, 70, 128])), 64
        D = int(rng.choice([8, 24, 64, 100, 128, 200, 512]))
        ind, outd = DTS[int(rng.integers(0, 3))], DTS[int(rng.integers(0, 3))]
        layout = "bhrd" if rng.random() < 0.6 else "rbhd"
        out.append(dict(R=R, B=B, H=H, D=D, in_dtype=ind, out_dtype=outd, layout=layout,
                        seed=3000 + i, base=base))
    return out


CASES = _cases()


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[f"c{i}_R{c['R']}_B{c['B']}_H{c['H']}_D{c['D']}_"
                                             f"{c['in_dtype']}{c['out_dtype']}_{c['layout']}"
                                             for i, c in enumerate(CASES)])
def test_random_shape_matches_oracle(case):
    c = dict(case)
    base, seed = c.pop("base"), c.pop("seed")
    inp = synth.make_inputs(base, seed=seed, poison_empty=True, **c)
    d_o, d_l, _ = upload(inp)
    out = torch.empty((inp["B"], inp["H"], inp["D"]), dtype=TORCH_DT[inp["out_dtype"]], device="cuda")
    out_lse = torch.empty((inp["B"], inp["H"]), dtype=torch.float32, device="cuda")
    rc, plan = nat.plan_query(d_o.data_ptr(), d_l.data_ptr(), inp["R"], inp["B"], inp["H"],
                              inp["D"], (inp["o_strides"], inp["lse_strides"]),
                              synth.DTYPES[inp["in_dtype"]], synth.DTYPES[inp["out_dtype"]],
                              out.data_ptr(), out_lse.data_ptr())
    assert rc == nat.OK
    c.pop("layout")
    parity(inp, what=f"{c} {case['layout']} seed {seed} via {plan['path_name']}")


def test_the_sweep_takes_every_path():
    """Host only: the planner's choice for each case, from pointer values alone
    (plan_query never dereferences them), covers all five kernel paths."""
    seen = set()
    long_form = 0
    for case in CASES:
        c = dict(case)
        base = c.pop("base")
        c.pop("seed")
        w = synth.Workload(**{**base.__dict__, **c})
        o_str, l_str = synth.strides(w.layout, w.R, w.B, w.H, w.D)
        rc, plan = nat.plan_query(0x7F0000000000, 0x7F1000000000, w.R, w.B, w.H, w.D,
                                  (o_str, l_str), synth.DTYPES[w.in_dtype],
                                  synth.DTYPES[w.out_dtype], 0x7F2000000000, 0x7F3000000000)
        assert rc == nat.OK
        seen.add(plan["path_name"])
        long_form += plan["path"] == nat.PATH_STREAM and w.R > plan["rc"]
    assert seen == {"latency", "wide", "vector", "stream", "scalar"}, seen
    assert long_form >= 3, long_form
