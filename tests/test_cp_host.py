"""Context-parallel exchange + merge on the host: the workspace layout, the
argument validation of lse_merge_cp_exchange_merge (through
lse_merge_cp_validate, which launches nothing), and the multi-process group
logic of CPExchangeMerge on CPU ranks (gloo, world size 2) with a fake device
backend: agreement checks, IPC handle exchange, the launch arguments of each
rank, timeout status, restart, host-side liveness check and tear-down."""
import os
import sys

import pytest
import torch.multiprocessing as mp

from lse_weighted_merge_b200 import _native as nat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Fake, aligned addresses far apart (never dereferenced).
LO, LL, OO, OL = 0x7f0000000000, 0x7f1000000000, 0x7f2000000000, 0x7f3000000000
WS = 0x7f4000000000
STEP = 0x10000000


def _up(x, a=256):
    return (x + a - 1) // a * a


@pytest.mark.parametrize("world,B,H,D,dt", [(1, 1, 2, 64, nat.BF16), (2, 1, 2, 64, nat.BF16),
                                            (8, 64, 32, 128, nat.BF16), (4, 3, 12, 4, nat.F32),
                                            (8, 5, 8, 512, nat.F16)])
def test_workspace_layout(world, B, H, D, dt):
    eb = 4 if dt == nat.F32 else 2
    Hq = H // world
    o_bytes = 2 * (world - 1) * B * Hq * D * eb
    l_off = _up(256 + o_bytes)
    want = _up(l_off + 2 * (world - 1) * B * Hq * 4)
    assert nat.cp_workspace_bytes(world, B, H, D, dt) == want


@pytest.mark.parametrize("args,code", [
    ((0, 1, 2, 64, nat.BF16), nat.EDIMS), ((9, 1, 9, 64, nat.BF16), nat.EDIMS),
    ((2, 1, 3, 64, nat.BF16), nat.EDIMS), ((2, 0, 2, 64, nat.BF16), nat.EDIMS),
    ((2, 1, 2, 4, nat.BF16), nat.EALIGN), ((2, 1, 2, 2, nat.F32), nat.EALIGN),
    ((2, 1 << 14, 1 << 10, 1 << 10, nat.BF16), nat.EDIMS),   # 32 GiB: 2^31 units
    ((2, (1 << 14) - 1, 1 << 10, 1 << 10, nat.BF16), None),  # one batch less: accepted
    ((2, 1, 2, 64, 7), nat.EDTYPE)])
def test_workspace_bytes_rejects(args, code):
    if code is None:
        assert nat.cp_workspace_bytes(*args) > 0
        return
    with pytest.raises(nat.LseMergeError) as ei:
        nat.cp_workspace_bytes(*args)
    assert ei.value.code == code


def make(world=2, rank_begin=0, rank_count=None, B=2, H=4, D=64, i=nat.BF16, o=nat.BF16,
         timeout_ns=10**9, lo=None, ll=None, oo=None, ol=None, ws=None, flags=0):
    n = world - rank_begin if rank_count is None else rank_count
    lo = lo if lo is not None else [LO + k * STEP for k in range(n)]
    ll = ll if ll is not None else [LL + k * STEP for k in range(n)]
    oo = oo if oo is not None else [OO + k * STEP for k in range(n)]
    ol = ol if ol is not None else [OL + k * STEP for k in range(n)]
    ws = ws if ws is not None else [WS + q * STEP for q in range(world)]
    a = nat.cp_args(world, rank_begin, lo, ll, oo, ol, ws, B, H, D, i, o, timeout_ns, flags)
    a.rank_count = n
    return a


def test_validate_accepts_good_arguments():
    for world in (1, 2, 4, 8):
        assert nat.cp_validate(make(world=world, H=8)) == nat.OK
    assert nat.cp_validate(make(world=4, rank_begin=3, rank_count=1, H=8)) == nat.OK
    assert nat.cp_validate(make(i=nat.F32, o=nat.F16, D=4)) == nat.OK
    assert nat.cp_validate(make(flags=nat.CP_FLAG_CROSS_GPU_PROTOCOL)) == nat.OK
    assert nat.cp_validate(make(flags=nat.CP_FLAG_TEST_SILENT_LAST_RANK)) == nat.OK
    # inputs are only read: two played ranks may share one input buffer
    assert nat.cp_validate(make(lo=[LO, LO], ll=[LL, LL])) == nat.OK


@pytest.mark.parametrize("kw,code", [
    (dict(i=5), nat.EDTYPE), (dict(o=-1), nat.EDTYPE),
    (dict(world=0, ws=[]), nat.EDIMS), (dict(world=9, H=9, rank_count=1, ws=[WS + q * STEP for q in range(8)]), nat.EDIMS), (dict(H=3), nat.EDIMS),
    (dict(B=0), nat.EDIMS), (dict(D=0), nat.EDIMS),
    (dict(rank_begin=1, rank_count=2), nat.EDIMS), (dict(rank_begin=-1, rank_count=1), nat.EDIMS),
    (dict(rank_count=0), nat.EDIMS),
    (dict(timeout_ns=0), nat.EDIMS), (dict(timeout_ns=61 * 10**9), nat.EDIMS),
    (dict(flags=4), nat.EDIMS),
    (dict(D=4), nat.EALIGN), (dict(i=nat.F32, D=2), nat.EALIGN),
    (dict(ws=[WS, 0]), nat.ENULL), (dict(lo=[LO, 0]), nat.ENULL), (dict(ol=[0, OL]), nat.ENULL),
    (dict(ws=[WS, WS + STEP + 128]), nat.EALIGN), (dict(lo=[LO + 8, LO + STEP]), nat.EALIGN),
    (dict(oo=[OO, OO + STEP + 4]), nat.EALIGN), (dict(ll=[LL + 2, LL + STEP]), nat.EALIGN),
    (dict(ws=[WS, WS + 256]), nat.EALIAS),              # two workspaces overlap
    (dict(oo=[WS + 512, OO + STEP]), nat.EALIAS),       # an output inside a workspace
    (dict(oo=[LO + 64, OO + STEP]), nat.EALIAS),        # an output over an input
    (dict(ol=[OO + 16, OL + STEP]), nat.EALIAS),        # out_lse over out_o
    (dict(oo=[OO, OO + 64]), nat.EALIAS),               # two ranks' outputs overlap
    (dict(lo=[WS + STEP, LO + STEP]), nat.EALIAS),      # an input inside a workspace
])
def test_validate_rejects(kw, code):
    assert nat.cp_validate(make(**kw)) == code


def test_more_than_eight_pointers_is_a_value_error():
    with pytest.raises(ValueError):
        nat.cp_args(9, 0, [LO], [LL], [OO], [OL], [WS + q * STEP for q in range(9)], 1, 9, 64,
                    nat.BF16, nat.BF16, 10**9)


def test_validate_null_args_and_launch_rejects_before_cuda():
    assert nat.lib.lse_merge_cp_validate(None) == nat.ENULL
    # a rejected call returns its code without touching CUDA (no GPU here)
    assert nat.cp_exchange_merge_raw(make(H=3), check=False) == nat.EDIMS


def test_setup_calls_reject_null_pointers():
    assert nat.lib.lse_merge_cp_workspace_create(256, None) == nat.ENULL
    assert nat.lib.lse_merge_cp_workspace_destroy(None) == nat.ENULL
    assert nat.lib.lse_merge_cp_ipc_handle(None, None) == nat.ENULL
    assert nat.lib.lse_merge_cp_ipc_open(None, None) == nat.ENULL
    assert nat.lib.lse_merge_cp_ipc_close(None) == nat.ENULL
    assert nat.lib.lse_merge_cp_status(None, None) == nat.ENULL
    assert nat.lib.lse_merge_cp_workspace_zero(None, 256) == nat.ENULL
    with pytest.raises(ValueError):
        nat.cp_ipc_open(b"short")


# ------------------------------------------------------------ the group, on gloo ranks

class FakeBackend:
    """Host stand-in for the device calls: fake addresses, handles that encode
    them, and a launch that runs the library's own argument validation."""

    def __init__(self, rank):
        self.rank = rank
        self.base = WS + rank * (1 << 36)
        self.log = []
        self.fake_status = 0
        self.fail_create = False
        self.fail_open = False

    def workspace_bytes(self, *a):
        return nat.cp_workspace_bytes(*a)

    def device(self):
        return None     # CPU tensors: no device to match

    def create(self, nbytes):
        if self.fail_create:
            raise MemoryError("no device memory left")
        self.log.append(("create", nbytes))
        return self.base

    def handle(self, ptr):
        return ptr.to_bytes(8, "little") + bytes(nat.CP_IPC_HANDLE_BYTES - 8)

    def open(self, handle):
        if self.fail_open:
            raise OSError("cannot map the peer's memory")
        assert len(handle) == nat.CP_IPC_HANDLE_BYTES
        ptr = int.from_bytes(handle[:8], "little") + (1 << 35)   # mapped at another address
        self.log.append(("open", ptr))
        return ptr

    def close(self, ptr):
        self.log.append(("close", ptr))

    def destroy(self, ptr):
        self.log.append(("destroy", ptr))

    def zero(self, ptr, nbytes):
        self.log.append(("zero", ptr, nbytes))

    def sync(self):
        self.log.append(("sync",))

    def status(self, ptr):
        return self.fake_status

    def launch(self, args, stream):
        rc = nat.cp_validate(args)
        self.log.append(("launch", rc, args.world, args.rank_begin, args.rank_count,
                         [args.ws[q] for q in range(args.world)]))


def _put_and_exit(q, res):
    q.put(res)
    q.close()
    q.join_thread()     # flush the queue before the abrupt exit
    os._exit(0)


def _group_worker(rank, world, port, q, scenario):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from lse_weighted_merge_b200 import cp
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    res = {"rank": rank}
    try:
        be = FakeBackend(rank)
        H = 8 if (scenario == "mismatch" and rank == 1) else 4
        D = 4 if (scenario == "bad_shape" and rank == 0) else 64
        be.fail_create = scenario == "create_fails" and rank == 1
        be.fail_open = scenario == "open_fails" and rank == 0
        try:
            g = cp.CPExchangeMerge(2, H, D, torch.bfloat16, backend=be)
        except (ValueError, RuntimeError) as exc:
            res["error"] = f"{type(exc).__name__}: {exc}"
            res["log"] = list(be.log)
            q.put(res)
            return
        res["peers"] = list(g.peers)
        res["ws"] = g.ws
        if scenario == "lost":
            if rank == 1:
                _put_and_exit(q, res)          # leaves between steps, without a word
            try:
                g.check_peers(timeout_s=3.0)
            except cp.PeerLost as exc:
                res["lost"] = str(exc)
            _put_and_exit(q, res)
        o = torch.zeros((2, 4, 64), dtype=torch.bfloat16)
        lse = torch.zeros((2, 4), dtype=torch.float32)
        out, out_lse = g(o, lse)
        res["out_shape"] = (tuple(out.shape), tuple(out_lse.shape), out.dtype == torch.bfloat16)
        first = g._args
        g(o, lse, out=out, out_lse=out_lse)
        res["args_reused"] = g._args is first    # same buffers: the argument block is kept
        with pytest.raises(ValueError):
            g(o[:, :2], lse)                          # wrong shape: rejected on the host
        res["launch"] = [e for e in be.log if e[0] == "launch"]
        assert len(res["launch"]) == 2
        g.check_peers(timeout_s=20.0)
        be.fake_status = 1 << (1 - rank)
        res["status"] = g.status()
        try:
            g(o, lse)
            res["raised_when_broken"] = False
        except RuntimeError:
            res["raised_when_broken"] = True
        g.reset()
        be.fake_status = 0
        res["zeroed"] = [e for e in be.log if e[0] == "zero"]
        res["synced_before_zero"] = [e[0] for e in be.log].index("sync") < \
            [e[0] for e in be.log].index("zero")
        res["after_reset"] = g.status() == 0 and not g.broken
        g(o, lse)
        g.close()
        res["teardown"] = [e for e in be.log if e[0] in ("close", "destroy")]
        dist.destroy_process_group()
    except Exception as exc:    # report, so that the parent test fails with the reason
        res["exception"] = repr(exc)
    q.put(res)


def _run_group(scenario):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + hash(scenario)) % 900
    procs = [ctx.Process(target=_group_worker, args=(r, 2, port, q, scenario)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r["rank"])
    for p in procs:
        p.join(timeout=60)
    return res, [p.exitcode for p in procs]


def test_group_setup_step_status_reset_close():
    res, codes = _run_group("normal")
    assert codes == [0, 0]
    for r in res:
        assert "exception" not in r, r
        rank, other = r["rank"], 1 - r["rank"]
        ws_other = WS + other * (1 << 36)
        assert r["peers"][rank] == r["ws"] == WS + rank * (1 << 36)
        assert r["peers"][other] == ws_other + (1 << 35)
        assert r["out_shape"] == ((2, 2, 64), (2, 2), True)
        assert r["args_reused"]
        for (_, rc, world, begin, count, ws) in r["launch"]:
            assert (rc, world, begin, count) == (nat.OK, 2, rank, 1)
            assert ws == r["peers"]
        assert r["status"] == 1 << other and r["raised_when_broken"]
        assert r["zeroed"] and r["zeroed"][0][1] == r["ws"] and r["after_reset"]
        assert r["synced_before_zero"]
        assert r["teardown"] == [("close", ws_other + (1 << 35)), ("destroy", r["ws"])]


def test_group_rejects_disagreeing_shapes_on_every_rank():
    res, codes = _run_group("mismatch")
    assert codes == [0, 0]
    assert all("disagree" in r.get("error", "") for r in res), res


@pytest.mark.parametrize("scenario,kind,words", [
    ("bad_shape", "ValueError", "rank 0"),
    ("create_fails", "RuntimeError", "rank 1: workspace"),
    ("open_fails", "RuntimeError", "rank 0: mapping"),
])
def test_a_set_up_failure_on_one_rank_raises_on_every_rank(scenario, kind, words):
    """No rank is left waiting in a collective: every rank raises the same
    error, and a rank that had created its workspace frees it again."""
    res, codes = _run_group(scenario)
    assert codes == [0, 0]
    for r in res:
        assert r.get("error", "").startswith(kind) and words in r["error"], r
        created = [e for e in r["log"] if e[0] == "create"]
        freed = [e for e in r["log"] if e[0] == "destroy"]
        assert len(created) == len(freed), r["log"]
        opened = [e for e in r["log"] if e[0] == "open"]
        closed = [e for e in r["log"] if e[0] == "close"]
        assert len(opened) == len(closed), r["log"]


def test_group_reports_a_lost_peer():
    res, codes = _run_group("lost")
    assert codes == [0, 0]
    assert "ranks [1]" in res[0].get("lost", ""), res[0]
