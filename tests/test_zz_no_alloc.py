"""The exchange-and-merge entry point that allocates nothing.

Callers that cannot reach cudaMalloc at this step -- a serving runtime whose
spare HBM already belongs to its KV-cache pool, or a decode step that must
not let an allocation synchronise the device -- call
lse_merge_cp_exchange_merge_noalloc.  It takes every rank's workspace from
one static array in device memory (16 MiB per GPU) instead of from the
caller.  These tests call it through the C ABI and check, on two calls in a
row with different data, that its outputs match those of the allocating
entry point (lse_merge_cp_exchange_merge with workspaces from the caller)
within the parity tolerance of the other GPU tests; and that a problem too
large for the array, or a launch that does not play every rank, is refused
before anything runs.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from gpu_util import TORCH_DT, check
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import cp, synth

pytestmark = pytest.mark.gpu


def _inputs(world, B, H, D, seed):
    base = synth.CP_WORKLOADS["cp_w8_b64_h32_d128_masked"]
    return synth.make_inputs(base, seed=seed, poison_empty=True, R=world, B=B, H=H, D=D)


def _to_device(inp):
    W, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    t = torch.from_numpy(inp["o"].view(np.int16)).cuda().view(torch.bfloat16).view(W, B, H, D)
    l = torch.from_numpy(inp["lse"]).cuda().view(W, B, H)
    return [t[s].contiguous() for s in range(W)], [l[s].contiguous() for s in range(W)]


def _noalloc(lo, ll, world, B, H, D, rank_count=None):
    Hq = H // world
    n = world if rank_count is None else rank_count
    outs = [(torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda"),
             torch.empty((B, Hq), dtype=torch.float32, device="cuda")) for _ in range(n)]
    args = nat.cp_args(world, 0, [x.data_ptr() for x in lo[:n]], [x.data_ptr() for x in ll[:n]],
                       [o.data_ptr() for o, _ in outs], [l.data_ptr() for _, l in outs], [],
                       B, H, D, nat.BF16, nat.BF16, 2 * 10**9)
    args.rank_count = n
    rc = nat.cp_exchange_merge_noalloc_raw(args, torch.cuda.current_stream().cuda_stream,
                                           check=False)
    return rc, outs


def test_noalloc_matches_the_allocating_entry_point_on_two_calls():
    world, B, H, D = 8, 16, 32, 128
    for call, seed in enumerate((41, 42)):
        inp = _inputs(world, B, H, D, seed)
        lo, ll = _to_device(inp)
        ws = [cp.cp_workspace(world, B, H, D, torch.bfloat16, "cuda") for _ in range(world)]
        ref = cp.cp_exchange_merge(lo, ll, ws)
        rc, outs = _noalloc(lo, ll, world, B, H, D)
        assert rc == nat.OK, nat.strerror(rc)
        torch.cuda.synchronize()
        for q in range(world):
            check(outs[q][0].double().cpu().numpy(), outs[q][1].double().cpu().numpy(),
                  ref[q][0].double().cpu().numpy(), ref[q][1].double().cpu().numpy(),
                  "bf16", f"call {call} rank {q}")


def test_noalloc_refuses_what_it_cannot_run():
    # 8 ranks of B=64, H=64, D=512 bf16 need ~58 MB of workspaces: too large
    world, B, H, D = 8, 64, 64, 512
    need = world * nat.cp_workspace_bytes(world, B, H, D, nat.BF16)
    assert need > 16 << 20
    lo = [torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    ll = [torch.zeros((B, H), dtype=torch.float32, device="cuda") for _ in range(world)]
    rc, _ = _noalloc(lo, ll, world, B, H, D)
    assert rc == nat.ESCRATCH
    # a launch that does not play every rank could never complete its waits
    rc, _ = _noalloc(lo[:2], ll[:2], 2, 4, 4, 128, rank_count=1)
    assert rc == nat.EDIMS
