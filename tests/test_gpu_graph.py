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
