"""Context-parallel exchange + merge on the GPU vs the fp64 oracle, through the
C ABI.  Every rank's data lives on the one GPU and one cooperative launch
plays all ranks, so the ranks' waits on one another complete inside a single
kernel.  Covered: 1 to 8 ranks, every dtype pair, ragged and masked inputs
(empty partials holding NaN, all-empty rows), repeated calls (the receive
slots alternate and the call count lives in the workspace), replays of a
captured CUDA graph, a wait that runs out (a sender that never sends: the
status word is set, the outputs stay untouched, the kernel returns), the
group class on one rank, and the IPC set-up calls across two processes."""
import multiprocessing
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TORCH_DT, check
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import cp, synth

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def inputs(name=None, seed=None, **over):
    base = synth.CP_WORKLOADS[name or "cp_w8_b64_h32_d128_masked"]
    return synth.make_inputs(base, seed=seed, poison_empty=True, **over)


def to_device(inp):
    """Rank s's local partials o [B, H, D] and lse [B, H] as CUDA tensors."""
    W, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    o = inp["o"]
    raw = torch.from_numpy(o.view(np.int16) if o.dtype == np.uint16 else o)
    t = raw.cuda().view(TORCH_DT[inp["in_dtype"]]).view(W, B, H, D)
    l = torch.from_numpy(inp["lse"]).cuda().view(W, B, H)
    return [t[s].contiguous() for s in range(W)], [l[s].contiguous() for s in range(W)]


def want(inp):
    return oracle.cp_exchange_merge(inp["o"], inp["lse"], inp["R"], inp["B"], inp["H"], inp["D"],
                                    synth.DTYPES[inp["in_dtype"]])


def workspaces(inp):
    return [cp.cp_workspace(inp["R"], inp["B"], inp["H"], inp["D"],
                            TORCH_DT[inp["in_dtype"]], "cuda") for _ in range(inp["R"])]


def compare(outs, inp, what):
    w_o, w_l = want(inp)
    for q, (o, l) in enumerate(outs):
        check(o.double().cpu().numpy(), l.double().cpu().numpy(), w_o[q], w_l[q],
              inp["out_dtype"], f"{what} rank {q}")


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("B,Hq,D", [(1, 1, 64), (3, 2, 128), (5, 3, 8), (2, 1, 512)])
def test_exchange_merge_parity(world, B, Hq, D):
    inp = inputs(R=world, B=B, H=world * Hq, D=D, seed=world * 100 + D + B)
    lo, ll = to_device(inp)
    outs = cp.cp_exchange_merge(lo, ll, workspaces(inp))
    torch.cuda.synchronize()
    compare(outs, inp, f"w{world} B{B} Hq{Hq} D{D}")


@pytest.mark.parametrize("in_dt,out_dt,D", [("f32", "f32", 4), ("f32", "bf16", 36), ("f16", "f32", 64),
                                            ("bf16", "f16", 24), ("f16", "f16", 128)])
def test_exchange_merge_dtypes(in_dt, out_dt, D):
    inp = inputs(R=4, B=3, H=8, D=D, in_dtype=in_dt, out_dtype=out_dt, seed=7 + D)
    lo, ll = to_device(inp)
    outs = cp.cp_exchange_merge(lo, ll, workspaces(inp), out_dtype=TORCH_DT[out_dt])
    torch.cuda.synchronize()
    compare(outs, inp, f"{in_dt}->{out_dt} D{D}")


@pytest.mark.parametrize("cross", [False, True], ids=["one-gpu-protocol", "cross-gpu-protocol"])
@pytest.mark.parametrize("name", sorted(synth.CP_WORKLOADS))
def test_exchange_merge_workloads(name, cross):
    inp = inputs(name)
    lo, ll = to_device(inp)
    outs = cp.cp_exchange_merge(lo, ll, workspaces(inp), cross_gpu_protocol=cross)
    torch.cuda.synchronize()
    compare(outs, inp, name)


@pytest.mark.parametrize("cross", [False, True], ids=["one-gpu-protocol", "cross-gpu-protocol"])
def test_exchange_merge_large(cross):
    """8 ranks of B=256 H=64 D=128 (34 MB of partials): many CTAs per rank, so
    every receiver collects counts from many sending CTAs of each sender."""
    inp = inputs(R=8, B=256, H=64, D=128, seed=900)
    lo, ll = to_device(inp)
    outs = cp.cp_exchange_merge(lo, ll, workspaces(inp), cross_gpu_protocol=cross)
    torch.cuda.synchronize()
    compare(outs, inp, "large")


@pytest.mark.parametrize("cross", [False, True], ids=["one-gpu-protocol", "cross-gpu-protocol"])
def test_repeated_calls_alternate_slots_and_count_on_device(cross):
    base = inputs(R=4, B=6, H=8, D=128, seed=1)
    ws = workspaces(base)
    U = base["B"] * (base["H"] // 4) * (base["D"] * 2 // 16)
    for call in range(1, 6):
        inp = inputs(R=4, B=6, H=8, D=128, seed=100 + call)
        lo, ll = to_device(inp)
        outs = cp.cp_exchange_merge(lo, ll, ws, cross_gpu_protocol=cross)
        torch.cuda.synchronize()
        compare(outs, inp, f"call {call}")
        for q in range(4):
            hdr = ws[q][:256].view(torch.int64).cpu()
            landed = [int(hdr[s]) for s in range(4)]
            assert landed == [0 if s == q else call * U for s in range(4)], (q, landed)
            assert int(hdr[16]) == call << 20                 # rank q's arrival count
            assert cp.cp_status(ws[q]) == 0


def test_prepared_call_reused_over_updated_buffers():
    inp = inputs(R=4, B=5, H=8, D=64, seed=60)
    lo, ll = to_device(inp)
    call = cp.CPMergeCall(lo, ll, workspaces(inp))
    for k in range(3):
        nxt = inputs(R=4, B=5, H=8, D=64, seed=61 + k)
        nlo, nll = to_device(nxt)
        for s_ in range(4):
            lo[s_].copy_(nlo[s_])
            ll[s_].copy_(nll[s_])
        outs = call()
        torch.cuda.synchronize()
        compare(outs, nxt, f"prepared call {k}")


@pytest.mark.parametrize("cross", [False, True], ids=["one-gpu-protocol", "cross-gpu-protocol"])
def test_graph_replays_are_new_calls(cross):
    inp = inputs(R=8, B=2, H=16, D=128, seed=3)
    lo, ll = to_device(inp)
    ws = workspaces(inp)
    outs = cp.cp_exchange_merge(lo, ll, ws, cross_gpu_protocol=cross)    # eager call 1
    torch.cuda.synchronize()
    compare(outs, inp, "eager")
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            outs = cp.cp_exchange_merge(lo, ll, ws, cross_gpu_protocol=cross)
    torch.cuda.synchronize()
    for rep in range(3):
        nxt = inputs(R=8, B=2, H=16, D=128, seed=50 + rep)
        nlo, nll = to_device(nxt)
        for s_ in range(8):
            lo[s_].copy_(nlo[s_])
            ll[s_].copy_(nll[s_])
        g.replay()
        torch.cuda.synchronize()
        compare(outs, nxt, f"replay {rep}")
    assert int(ws[0][:256].view(torch.int64)[16].item()) == 4 << 20     # 4 calls arrived


def test_a_sender_that_never_sends_times_out():
    """World 2, but the launch plays rank 0 only: rank 1 never sends, so rank
    0's bounded wait runs out (2 ms), sets bit 1 of its status word and leaves
    its outputs untouched; its own rows did land in rank 1's workspace."""
    inp = inputs(R=2, B=4, H=4, D=128, seed=11)
    lo, ll = to_device(inp)
    ws = workspaces(inp)
    out = torch.full((4, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out_lse = torch.full((4, 2), 7.0, dtype=torch.float32, device="cuda")
    cp.cp_exchange_merge(lo[:1], ll[:1], ws, rank_begin=0, timeout_s=0.002, outs=[(out, out_lse)])
    torch.cuda.synchronize()
    assert cp.cp_status(ws[0]) == 0b10
    assert cp.cp_status(ws[1]) == 0
    assert bool((out == 7.0).all()) and bool((out_lse == 7.0).all())
    U = 4 * 2 * (128 * 2 // 16)
    assert int(ws[1][:8].view(torch.int64).item()) == U    # rank 0's units landed at rank 1
    assert int(ws[0][:256].view(torch.int64)[16].item()) == 1 << 20    # one call arrived
    # restart: zero every workspace, then a full call is correct again
    for w in ws:
        w.zero_()
    outs = cp.cp_exchange_merge(lo, ll, ws)
    torch.cuda.synchronize()
    compare(outs, inp, "after restart")
    assert cp.cp_status(ws[0]) == 0 and cp.cp_status(ws[1]) == 0


@pytest.mark.parametrize("cross", [False, True], ids=["one-gpu-protocol", "cross-gpu-protocol"])
@pytest.mark.parametrize("world,B,Hq,D", [(2, 3, 1, 64), (8, 5, 3, 128), (4, 2, 2, 8)])
def test_writes_stay_inside_outputs_and_workspaces(world, B, Hq, D, cross):
    """Outputs and workspaces are carved out of larger buffers whose guard
    bytes hold a canary pattern; after two calls no guard byte has changed
    (the only writes are inside the documented extents)."""
    G = 4096                                        # guard bytes on each side
    inp = inputs(R=world, B=B, H=world * Hq, D=D, seed=500 + world + D)
    lo, ll = to_device(inp)
    nbytes = nat.cp_workspace_bytes(world, B, world * Hq, D, nat.BF16)
    canary = 0xA5
    ws_buf = [torch.full((G + nbytes + G,), canary, dtype=torch.uint8, device="cuda")
              for _ in range(world)]
    for w in ws_buf:
        w[G:G + nbytes].zero_()
    o_bytes, l_bytes = B * Hq * D * 2, B * Hq * 4
    out_buf = [torch.full((G + o_bytes + G,), canary, dtype=torch.uint8, device="cuda")
               for _ in range(world)]
    lse_buf = [torch.full((G + l_bytes + G,), canary, dtype=torch.uint8, device="cuda")
               for _ in range(world)]
    outs = [(o[G:G + o_bytes].view(torch.bfloat16).view(B, Hq, D),
             l[G:G + l_bytes].view(torch.float32).view(B, Hq)) for o, l in zip(out_buf, lse_buf)]
    for _ in range(2):
        cp.cp_exchange_merge(lo, ll, [w[G:G + nbytes] for w in ws_buf], outs=outs,
                             cross_gpu_protocol=cross)
    torch.cuda.synchronize()
    compare(outs, inp, "guarded")
    for name, bufs, n in (("workspace", ws_buf, nbytes), ("out", out_buf, o_bytes),
                          ("out_lse", lse_buf, l_bytes)):
        for q, buf in enumerate(bufs):
            assert bool((buf[:G] == canary).all()), f"{name} {q}: write before the buffer"
            assert bool((buf[G + n:] == canary).all()), f"{name} {q}: write past the buffer"


def test_rejected_arguments_raise():
    inp = inputs(R=2, B=1, H=2, D=64, seed=0)
    lo, ll = to_device(inp)
    ws = workspaces(inp)
    with pytest.raises(ValueError):
        cp.cp_exchange_merge(lo, ll, ws[:1] * 3)           # H = 2 not a multiple of 3
    with pytest.raises(nat.LseMergeError) as ei:
        cp.cp_exchange_merge(lo, ll, [ws[0], ws[0]])       # one workspace passed twice
    assert ei.value.code == nat.EALIAS
    with pytest.raises(nat.LseMergeError) as ei:
        cp.cp_exchange_merge(lo, ll, ws, timeout_s=0.0)
    assert ei.value.code == nat.EDIMS


def _one_rank_group(q):
    sys.path.insert(0, ROOT)
    try:
        import torch.distributed as dist
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method="tcp://127.0.0.1:" + str(29900 + os.getpid() % 90),
                                rank=0, world_size=1)
        g = cp.CPExchangeMerge(2, 4, 64, torch.bfloat16)
        o = torch.randn(2, 4, 64, device="cuda").to(torch.bfloat16)
        lse = torch.randn(2, 4, device="cuda")
        out, out_lse = g(o, lse)
        torch.cuda.synchronize()
        ok = bool(torch.equal(out, o)) and bool(torch.equal(out_lse, lse)) and g.status() == 0
        g.close()
        dist.destroy_process_group()
        q.put(("ok", ok))
    except Exception as exc:
        q.put(("error", repr(exc)))


def test_group_of_one_rank_on_the_gpu():
    """The group class end to end on one GPU: a workspace from the library,
    one call (with a single rank the exchange is the identity), status, close."""
    ctx = multiprocessing.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_one_rank_group, args=(q,))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=60)
    assert res == ("ok", True), res


def _ipc_owner(q_out, q_in):
    sys.path.insert(0, ROOT)
    from lse_weighted_merge_b200 import _native as n
    torch.cuda.set_device(0)
    ws = n.cp_workspace_create(4096)
    q_out.put(n.cp_ipc_handle(ws))
    q_in.get(timeout=120)                  # the peer has mapped, read, zeroed and unmapped it
    q_out.put(("status", n.cp_status(ws)))
    n.cp_workspace_destroy(ws)


def _ipc_peer(q_in, q_out):
    sys.path.insert(0, ROOT)
    from lse_weighted_merge_b200 import _native as n
    torch.cuda.set_device(0)
    h = q_in.get(timeout=120)
    peer = n.cp_ipc_open(h)
    st = n.cp_status(peer)
    n.cp_workspace_zero(peer, 4096)
    n.cp_ipc_close(peer)
    q_out.put(("peer", st))


def test_ipc_handles_between_two_processes():
    """The IPC set-up calls between two processes on one GPU (no kernel runs):
    one creates a workspace and exports its handle, the other maps it, reads
    its status word, zeroes it and unmaps it."""
    ctx = multiprocessing.get_context("spawn")
    a_to_b, b_to_a, done = ctx.Queue(), ctx.Queue(), ctx.Queue()
    owner = ctx.Process(target=_ipc_owner, args=(a_to_b, b_to_a))
    owner.start()
    h = a_to_b.get(timeout=300)
    assert isinstance(h, bytes) and len(h) == nat.CP_IPC_HANDLE_BYTES
    peer_q = ctx.Queue()
    peer_q.put(h)
    peer = ctx.Process(target=_ipc_peer, args=(peer_q, done))
    peer.start()
    assert done.get(timeout=300) == ("peer", 0)
    peer.join(timeout=60)
    b_to_a.put("go")
    assert a_to_b.get(timeout=120) == ("status", 0)
    owner.join(timeout=60)
    assert peer.exitcode == 0 and owner.exitcode == 0
