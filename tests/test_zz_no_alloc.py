"""The exchange-and-merge entry point that allocates nothing.

Callers that cannot reach cudaMalloc at this step -- a serving runtime whose
spare HBM already belongs to its KV-cache pool, or a decode step that must
not let an allocation synchronise the device -- call
lse_merge_cp_exchange_merge_noalloc.  It takes every rank's workspace from
one static array in device memory (16 MiB per GPU) instead of from the
caller.  These tests call it through the C ABI and check:
  * on two calls in a row with different data, that its outputs match those
    of the allocating entry point (lse_merge_cp_exchange_merge with
    workspaces from the caller) and the fp64 oracle of the exchange, within
    the parity tolerance of the other GPU tests, for every input/output
    dtype and two shapes; the outputs are filled with NaN before each call,
    so a skipped merge cannot pass; every rank's status word reads 0; and the
    second call leaves the device's free memory unchanged;
  * that a wait made to run out (a test flag keeps the last rank from
    sending) is reported by lse_merge_cp_noalloc_status, leaves the waiting
    ranks' outputs unwritten, and that the next call is correct again;
  * that a problem too large for the array, or a launch that does not play
    every rank, is refused before anything runs.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TORCH_DT, check
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import cp, synth

pytestmark = pytest.mark.gpu

TIMEOUT_NS = 2 * 10**9


def _inputs(world, B, H, D, seed, in_dtype="bf16", out_dtype="bf16"):
    base = synth.CP_WORKLOADS["cp_w8_b64_h32_d128_masked"]
    return synth.make_inputs(base, seed=seed, poison_empty=True, R=world, B=B, H=H, D=D,
                             in_dtype=in_dtype, out_dtype=out_dtype)


def _to_device(inp):
    W, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    o = inp["o"]
    raw = torch.from_numpy(o.view(np.int16) if o.dtype == np.uint16 else o.view(np.int32)).cuda()
    t = raw.view(TORCH_DT[inp["in_dtype"]]).view(W, B, H, D)
    l = torch.from_numpy(inp["lse"]).cuda().view(W, B, H)
    return [t[s].contiguous() for s in range(W)], [l[s].contiguous() for s in range(W)]


def _args(lo, ll, outs, world, B, H, D, in_dtype, out_dtype, flags=0, timeout_ns=TIMEOUT_NS):
    args = nat.cp_args(world, 0, [x.data_ptr() for x in lo], [x.data_ptr() for x in ll],
                       [o.data_ptr() for o, _ in outs], [l.data_ptr() for _, l in outs], [],
                       B, H, D, synth.DTYPES[in_dtype], synth.DTYPES[out_dtype], timeout_ns, flags)
    args.rank_count = len(lo)
    return args


def _nan_outputs(n, B, Hq, D, out_dtype):
    return [(torch.full((B, Hq, D), float("nan"), dtype=TORCH_DT[out_dtype], device="cuda"),
             torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda"))
            for _ in range(n)]


def _noalloc(lo, ll, world, B, H, D, in_dtype="bf16", out_dtype="bf16", flags=0, timeout_ns=TIMEOUT_NS):
    outs = _nan_outputs(len(lo), B, H // world, D, out_dtype)
    args = _args(lo, ll, outs, world, B, H, D, in_dtype, out_dtype, flags, timeout_ns)
    rc = nat.cp_exchange_merge_noalloc_raw(args, torch.cuda.current_stream().cuda_stream,
                                           check=False)
    return rc, outs, args


def _host(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("world,B,H,D,in_dt,out_dt", [
    (8, 16, 32, 128, "bf16", "bf16"),
    (8, 16, 32, 128, "f16", "f16"),
    (4, 5, 12, 64, "f32", "f32"),
    (2, 3, 2, 512, "bf16", "f32"),
])
def test_noalloc_matches_the_allocating_entry_point_and_the_oracle_on_two_calls(
        world, B, H, D, in_dt, out_dt):
    Hq = H // world
    for call, seed in enumerate((41, 42)):
        inp = _inputs(world, B, H, D, seed + D, in_dt, out_dt)
        lo, ll = _to_device(inp)
        ws = [cp.cp_workspace(world, B, H, D, TORCH_DT[in_dt], "cuda") for _ in range(world)]
        ref = cp.cp_exchange_merge(lo, ll, ws, out_dtype=TORCH_DT[out_dt])
        outs = _nan_outputs(world, B, Hq, D, out_dt)
        args = _args(lo, ll, outs, world, B, H, D, in_dt, out_dt)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        rc = nat.cp_exchange_merge_noalloc_raw(args, torch.cuda.current_stream().cuda_stream,
                                               check=False)
        assert rc == nat.OK, nat.strerror(rc)
        torch.cuda.synchronize()
        if call == 1:   # the first call may load the kernel's module; the second allocates nothing
            assert torch.cuda.mem_get_info()[0] == free_before
        rc, status = nat.cp_noalloc_status(args, check=False)
        assert rc == nat.OK and status == [0] * world, (rc, status)
        want, want_lse = oracle.cp_exchange_merge(inp["o"], inp["lse"], world, B, H, D,
                                                  synth.DTYPES[in_dt])
        for q in range(world):
            got, got_lse = _host(outs[q][0]), _host(outs[q][1])
            check(got, got_lse, want[q], want_lse[q], out_dt, f"call {call} rank {q} vs oracle")
            check(got, got_lse, _host(ref[q][0]), _host(ref[q][1]), out_dt,
                  f"call {call} rank {q} vs allocating entry point")


def test_a_wait_that_runs_out_is_reported_and_the_next_call_recovers():
    world, B, H, D = 4, 2, 4, 128
    inp = _inputs(world, B, H, D, 77)
    lo, ll = _to_device(inp)
    # the last rank sends nothing: ranks 0..2 wait 2 ms for it, then give up
    rc, outs, args = _noalloc(lo, ll, world, B, H, D, flags=nat.CP_FLAG_TEST_SILENT_LAST_RANK,
                              timeout_ns=2_000_000)
    assert rc == nat.OK, nat.strerror(rc)
    rc, status = nat.cp_noalloc_status(args, check=False)
    assert rc == nat.OK
    assert status == [1 << (world - 1)] * (world - 1) + [0], status
    for q in range(world - 1):   # outputs of a rank whose wait ran out are not written
        assert bool(torch.isnan(outs[q][0]).all()) and bool(torch.isnan(outs[q][1]).all())
    want, want_lse = oracle.cp_exchange_merge(inp["o"], inp["lse"], world, B, H, D, oracle.BF16)
    # the silent rank itself received every other rank's rows and merged them
    q = world - 1
    check(_host(outs[q][0]), _host(outs[q][1]), want[q], want_lse[q], "bf16", "silent rank")
    # the next call starts from cleared headers: every rank completes again
    rc, outs, args = _noalloc(lo, ll, world, B, H, D)
    assert rc == nat.OK
    rc, status = nat.cp_noalloc_status(args, check=False)
    assert rc == nat.OK and status == [0] * world, status
    for q in range(world):
        check(_host(outs[q][0]), _host(outs[q][1]), want[q], want_lse[q], "bf16", f"rank {q} after")


def test_noalloc_refuses_what_it_cannot_run():
    # 8 ranks of B=64, H=64, D=512 bf16 need ~58 MB of workspaces: too large
    world, B, H, D = 8, 64, 64, 512
    need = world * nat.cp_workspace_bytes(world, B, H, D, nat.BF16)
    assert need > nat.CP_NOALLOC_SCRATCH_BYTES
    lo = [torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    ll = [torch.zeros((B, H), dtype=torch.float32, device="cuda") for _ in range(world)]
    rc, outs, args = _noalloc(lo, ll, world, B, H, D)
    assert rc == nat.ESCRATCH
    assert all(bool(torch.isnan(o).all()) for o, _ in outs)   # nothing ran
    rc, _ = nat.cp_noalloc_status(args, check=False)
    assert rc == nat.ESCRATCH
    # a launch that does not play every rank could never complete its waits
    rc, _, _ = _noalloc(lo[:1], ll[:1], 2, 4, 4, 128)
    assert rc == nat.EDIMS
