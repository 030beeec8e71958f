"""The latency path inside a CUDA graph: captured merges replay to the same
bits as eager calls and match the oracle."""
import numpy as np
import pytest
import torch

from gpu_util import check, run_oracle
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["r2_b1_h2_d64", "r8_b1_h8_d128", "r4_b64_h32_d128_masked"])
def test_graph_replay_matches_eager_and_oracle(name):
    inp = synth.make_inputs(synth.WORKLOADS[name])
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    d_o = torch.from_numpy(inp["o"].view(np.int16)).cuda()
    d_l = torch.from_numpy(inp["lse"]).cuda()
    st = (inp["o_strides"], inp["lse_strides"])
    ind, outd = synth.DTYPES[inp["in_dtype"]], synth.DTYPES[inp["out_dtype"]]
    eager = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    eager_l = torch.empty((B, H), dtype=torch.float32, device="cuda")
    nat.merge_raw(d_o.data_ptr(), d_l.data_ptr(), R, B, H, D, st, ind, outd, eager.data_ptr(),
                  eager_l.data_ptr(), torch.cuda.current_stream().cuda_stream)
    outs = [torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    outl = [torch.zeros((B, H), dtype=torch.float32, device="cuda") for _ in range(4)]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        s = torch.cuda.current_stream().cuda_stream
        for o_t, l_t in zip(outs, outl):
            nat.merge_raw(d_o.data_ptr(), d_l.data_ptr(), R, B, H, D, st, ind, outd,
                          o_t.data_ptr(), l_t.data_ptr(), s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    want, want_lse = run_oracle(inp)
    for o_t, l_t in zip(outs, outl):
        assert torch.equal(o_t.view(torch.int16), eager.view(torch.int16))
        assert torch.equal(l_t, eager_l)
        check(o_t.double().cpu().numpy(), l_t.double().cpu().numpy(), want, want_lse, "bf16", name)
    del g


CAPTURE_FIRST = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from lse_weighted_merge_b200 import _native as nat, synth
w = synth.WORKLOADS["r16_b512_h16_d512"]
inp = synth.make_inputs(w, B=64)
R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
o = torch.from_numpy(inp["o"].view(np.int16)).cuda()
l = torch.from_numpy(inp["lse"]).cuda()
outs = [torch.empty((B, H, D), dtype=torch.float32, device="cuda") for _ in range(2)]
ols = [torch.empty((B, H), dtype=torch.float32, device="cuda") for _ in range(2)]
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):          # the library's first call of the process
    s = torch.cuda.current_stream().cuda_stream
    for path, out, ol in ((nat.PATH_STREAM, outs[0], ols[0]), (nat.PATH_VECTOR, outs[1], ols[1])):
        nat.merge_raw(o.data_ptr(), l.data_ptr(), R, B, H, D, (inp["o_strides"], inp["lse_strides"]),
                      nat.BF16, nat.F32, out.data_ptr(), ol.data_ptr(), s, path)
g.replay()
torch.cuda.synchronize()
assert torch.equal(outs[0], outs[1]) and torch.equal(ols[0], ols[1])
assert torch.isfinite(outs[0]).all()
print("OK")
"""


def test_first_call_inside_a_capture():
    """The persistent path sizes its grid on first use (an occupancy query);
    that must also work when the very first call of a process is captured."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    p = subprocess.run([sys.executable, "-c", CAPTURE_FIRST.format(root=root)],
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0 and "OK" in p.stdout, p.stdout + p.stderr
