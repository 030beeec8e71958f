"""Context-parallel exchange + merge: tensors in, one C-ABI launch, tensors out.

Under context-parallel decode every rank holds the partials (o, lse) of its
own KV shard for all H heads; rank q owns heads [q*H/world, (q+1)*H/world)
and needs every rank's partials of those heads, merged (page "[flashinfer]
FlashInfer의 Context-Parallel Decode 최적화: Fused A2A + LSE Reduce", section
"들어가며" for the partials and section "코드 분석 / 1. Fused Kernel 구현"
for writing straight into the owner's buffer and merging there).  One kernel
does both steps: see ``lse_merge_cp_exchange_merge`` in include/lse_merge.h.

Two ways in:
  * ``cp_exchange_merge`` plays any set of ranks in one launch on one GPU
    (all ``world`` ranks at once when every rank's data lives on that GPU);
  * ``CPExchangeMerge`` is the multi-process form: one process per GPU, its
    workspace shared with the peers through CUDA IPC, one launch per rank and
    step.
"""
from __future__ import annotations

import datetime
import itertools

from . import _native
from .api import dtype_code

DEFAULT_TIMEOUT_S = 2.0
_INSTANCES = itertools.count()


def cp_workspace(world: int, B: int, H: int, D: int, dtype, device):
    """A zeroed workspace tensor (uint8) for one rank of ``world``."""
    import torch
    n = _native.cp_workspace_bytes(world, B, H, D, dtype_code(dtype))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def cp_status(ws) -> int:
    """The status word of a workspace tensor: 0, or bit s for each sender s
    whose rows never landed before the wait ran out (synchronises)."""
    import torch
    off = _native.CP_STATUS_OFFSET
    return int(ws[off:off + 4].view(torch.int32).item()) & 0xFFFFFFFF


def _check_local(o, l, B: int, H: int, D: int, dtype) -> None:
    import torch
    if tuple(o.shape) != (B, H, D) or o.dtype != dtype or not o.is_contiguous():
        raise ValueError(f"local_o must be a contiguous [B, H, D] = {(B, H, D)} tensor of {dtype}")
    if tuple(l.shape) != (B, H) or l.dtype != torch.float32 or not l.is_contiguous():
        raise ValueError(f"local_lse must be a contiguous float32 [B, H] = {(B, H)} tensor")


def _ptr(x) -> int:
    return x if isinstance(x, int) else x.data_ptr()


class CPMergeCall:
    """A prepared exchange + merge over fixed buffers.

    Validates the tensors and builds the C argument block once; each call is
    then a single launch on the current (or given) stream, which keeps the
    host cost of an eager step to the launch itself.  Arguments are those of
    ``cp_exchange_merge``; ``outs`` holds the output pairs it writes.
    """

    def __init__(self, local_o, local_lse, workspaces, *, rank_begin: int = 0, out_dtype=None,
                 timeout_s: float = DEFAULT_TIMEOUT_S, outs=None, cross_gpu_protocol: bool = False):
        import torch
        world = len(workspaces)
        n = len(local_o)
        if n < 1 or len(local_lse) != n:
            raise ValueError("local_o and local_lse must list the same ranks (at least one)")
        B, H, D = local_o[0].shape
        if H % world:
            raise ValueError(f"H = {H} is not a multiple of world = {world}")
        Hq = H // world
        dev = local_o[0].device
        in_dtype = local_o[0].dtype
        out_dtype = out_dtype or in_dtype
        for o, l in zip(local_o, local_lse):
            if not (o.is_cuda and l.is_cuda) or o.device != dev or l.device != dev:
                raise ValueError("all tensors must be on one CUDA device (there is no CPU path)")
            _check_local(o, l, B, H, D, in_dtype)
        if outs is None:
            outs = [(torch.empty((B, Hq, D), dtype=out_dtype, device=dev),
                     torch.empty((B, Hq), dtype=torch.float32, device=dev)) for _ in range(n)]
        # keep every buffer alive as long as the argument block points at it
        self._keep = (list(local_o), list(local_lse), list(workspaces))
        self.outs = outs
        self.device = dev
        self.args = _native.cp_args(world, rank_begin, [o.data_ptr() for o in local_o],
                                    [l.data_ptr() for l in local_lse],
                                    [o.data_ptr() for o, _ in outs], [l.data_ptr() for _, l in outs],
                                    [_ptr(w) for w in workspaces], B, H, D, dtype_code(in_dtype),
                                    dtype_code(out_dtype), int(timeout_s * 1e9),
                                    _native.CP_FLAG_CROSS_GPU_PROTOCOL if cross_gpu_protocol else 0)
        rc = _native.cp_validate(self.args)
        if rc != _native.OK:
            _native._raise(rc)

    def __call__(self, stream=None):
        import torch
        if torch.cuda.current_device() == self.device.index:
            s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
            _native.cp_exchange_merge_raw(self.args, s)
        else:   # the library launches on the current device: make it the tensors' one
            with torch.cuda.device(self.device):
                s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
                _native.cp_exchange_merge_raw(self.args, s)
        return self.outs


def cp_exchange_merge(local_o, local_lse, workspaces, *, rank_begin: int = 0, out_dtype=None,
                      timeout_s: float = DEFAULT_TIMEOUT_S, outs=None,
                      cross_gpu_protocol: bool = False):
    """Exchange heads between ranks and merge, in one launch on the current stream.

    local_o:    list of CUDA tensors [B, H, D] (float32 / float16 / bfloat16,
                contiguous), the partials of ranks rank_begin, rank_begin + 1, ...
    local_lse:  list of contiguous float32 CUDA tensors [B, H], same ranks.
    workspaces: the workspace of every rank q < world (``cp_workspace``
                tensors or raw device pointers), zeroed before the first call;
                ``world`` = len(workspaces).
    outs:       optional list of preallocated (out [B, H/world, D], out_lse
                [B, H/world]) pairs.
    Returns one (out, out_lse) pair per played rank.  A rank whose wait runs
    out (timeout_s) leaves its outputs unwritten and sets its workspace's
    status word (``cp_status``).  cross_gpu_protocol=True runs the protocol
    of ranks on different GPUs (system scope, two receive slots) although
    every rank is on this one, to test it.  For repeated calls over the same
    buffers, ``CPMergeCall`` prepares the arguments once.
    """
    return CPMergeCall(local_o, local_lse, workspaces, rank_begin=rank_begin, out_dtype=out_dtype,
                       timeout_s=timeout_s, outs=outs, cross_gpu_protocol=cross_gpu_protocol)()


class PeerLost(RuntimeError):
    """A peer rank did not check in on the host before the deadline."""


class NativeBackend:
    """The device side of CPExchangeMerge: library calls on the current GPU."""
    workspace_bytes = staticmethod(_native.cp_workspace_bytes)
    create = staticmethod(_native.cp_workspace_create)
    destroy = staticmethod(_native.cp_workspace_destroy)
    zero = staticmethod(_native.cp_workspace_zero)
    status = staticmethod(_native.cp_status)
    handle = staticmethod(_native.cp_ipc_handle)
    open = staticmethod(_native.cp_ipc_open)
    close = staticmethod(_native.cp_ipc_close)

    @staticmethod
    def device():
        import torch
        return torch.cuda.current_device()

    @staticmethod
    def sync() -> None:
        import torch
        torch.cuda.synchronize()

    @staticmethod
    def launch(args, stream: int) -> None:
        _native.cp_exchange_merge_raw(args, stream)


class CPExchangeMerge:
    """Exchange + merge across the ranks of a torch.distributed group, one GPU each.

    Construction is collective: every rank allocates its workspace on its
    current CUDA device, the ranks check that they agree on (B, H, D, dtypes)
    and exchange CUDA IPC handles, and each maps its peers' workspaces.  Each
    step of the set-up shares its local outcome with the other ranks, so a
    failure on one rank (a bad shape, an allocation, an IPC mapping) makes
    every rank raise, after releasing what it had set up, instead of leaving
    the others waiting in the next collective.  Each call then launches one
    kernel on the rank's current stream that stores the rows other ranks own
    into their workspaces over NVLink and merges the rows this rank owns.
    The group itself is only used on the host (set-up, ``check_peers``,
    ``reset``, ``close``); no collective runs per step.

    A peer that never sends makes this rank's kernel give up after
    ``timeout_s`` (its outputs stay unwritten); ``status()`` then reads
    non-zero, further calls raise, and every rank must call ``reset()``.
    """

    def __init__(self, B: int, H: int, D: int, dtype, out_dtype=None, *, group=None,
                 timeout_s: float = DEFAULT_TIMEOUT_S, backend=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.B, self.H, self.D = int(B), int(H), int(D)
        self.in_dtype = dtype_code(dtype)
        self.out_dtype = dtype_code(out_dtype or dtype)
        self.timeout_ns = int(timeout_s * 1e9)
        self.backend = backend or NativeBackend()
        self.device = self.backend.device()
        self.broken = False
        self.calls = 0
        self._checks = 0
        self._args_key = None
        self._args = None
        # instances are numbered in construction order, the same on every rank
        self._uid = next(_INSTANCES)
        self.ws = None
        self.peers = []

        # 1. the same problem on every rank, and one this library can run
        err = None
        try:
            if not 1 <= self.world <= _native.CP_MAX_WORLD:
                raise ValueError(f"world size {self.world} outside 1..{_native.CP_MAX_WORLD}")
            if self.H % self.world:
                raise ValueError(f"H = {self.H} is not a multiple of world = {self.world}")
            self.nbytes = self.backend.workspace_bytes(self.world, self.B, self.H, self.D,
                                                       self.in_dtype)
        except Exception as exc:   # shared with the other ranks below, then raised everywhere
            err = f"rank {self.rank}: {exc}"
        me = (self.B, self.H, self.D, self.in_dtype, self.out_dtype, self.timeout_ns)
        every = self._gather((me, err))
        errors = [e for _, e in every if e]
        if errors:
            raise ValueError("; ".join(errors))
        if any(x != me for x, _ in every):
            raise ValueError(f"ranks disagree on (B, H, D, dtypes, timeout): {[x for x, _ in every]}")

        # 2. this rank's workspace and its IPC handle
        handle, err = None, None
        try:
            self.ws = self.backend.create(self.nbytes)
            handle = self.backend.handle(self.ws)
        except Exception as exc:
            err = f"rank {self.rank}: workspace: {exc}"
        every = self._gather((handle, err))
        errors = [e for _, e in every if e]
        if errors:
            self._release()
            raise RuntimeError("; ".join(errors))

        # 3. the peers' workspaces mapped here
        err = None
        try:
            for q in range(self.world):
                self.peers.append(self.ws if q == self.rank else self.backend.open(every[q][0]))
        except Exception as exc:
            err = f"rank {self.rank}: mapping a peer's workspace: {exc}"
        errors = [e for e in self._gather(err) if e]
        if errors:
            self._release()
            raise RuntimeError("; ".join(errors))

    def _gather(self, obj) -> list:
        out = [None] * self.world
        self.dist.all_gather_object(out, obj, group=self.group)
        return out

    def _release(self) -> None:
        """Unmap the peers' workspaces and free this rank's (local, no collective)."""
        for q, p in enumerate(self.peers):
            if q != self.rank:
                self.backend.close(p)
        self.peers = []
        if self.ws is not None:
            self.backend.destroy(self.ws)
            self.ws = None

    def __call__(self, local_o, local_lse, out=None, out_lse=None, stream: int | None = None):
        """Send this rank's partials (local_o [B, H, D], local_lse [B, H]) and
        merge the heads it owns: returns (out [B, H/world, D], out_lse [B, H/world]).
        Passing the same out / out_lse (and inputs) on every step keeps the
        prepared argument block; new buffers rebuild it."""
        import torch
        if self.broken:
            raise RuntimeError("a wait ran out in an earlier call: call reset() on every rank")
        if self.ws is None:
            raise RuntimeError("this exchange has been closed")
        Hq = self.H // self.world
        dev = local_o.device
        _check_local(local_o, local_lse, self.B, self.H, self.D, _torch_dtype(self.in_dtype))
        if self.device is not None and dev.index != self.device:
            raise ValueError(f"local_o is on {dev}, the workspace on cuda:{self.device}")
        if out is None:
            out = torch.empty((self.B, Hq, self.D), dtype=_torch_dtype(self.out_dtype), device=dev)
        if out_lse is None:
            out_lse = torch.empty((self.B, Hq), dtype=torch.float32, device=dev)
        key = (local_o.data_ptr(), local_lse.data_ptr(), out.data_ptr(), out_lse.data_ptr())
        if self._args_key != key:      # the argument block is rebuilt only for new buffers
            self._args = _native.cp_args(self.world, self.rank, [key[0]], [key[1]], [key[2]],
                                         [key[3]], self.peers, self.B, self.H, self.D,
                                         self.in_dtype, self.out_dtype, self.timeout_ns)
            self._args_key = key
        args = self._args
        if dev.type == "cuda":
            with torch.cuda.device(dev):
                self.backend.launch(args, stream if stream is not None
                                    else torch.cuda.current_stream(dev).cuda_stream)
        else:   # only a host-side test backend takes CPU tensors
            self.backend.launch(args, stream or 0)
        self.calls += 1
        return out, out_lse

    def status(self) -> int:
        """0, or bit s for each sender whose rows did not land in time (synchronises)."""
        st = self.backend.status(self.ws)
        if st:
            self.broken = True
        return st

    def check_peers(self, timeout_s: float = 10.0) -> None:
        """Host-side liveness check between steps: every rank posts a key in
        the group's store and waits for all the others'.  Raises PeerLost
        naming the ranks that did not post in time."""
        # the default process group's key-value store: torch offers no public
        # accessor for it, and it works with every backend (NCCL included)
        store = self.dist.distributed_c10d._get_default_store()
        prefix = f"lse_cp/{self._uid}/alive/{self._checks}/"
        self._checks += 1
        store.set(prefix + str(self.rank), b"1")
        keys = [prefix + str(q) for q in range(self.world)]
        try:
            store.wait(keys, datetime.timedelta(seconds=timeout_s))
        except Exception as exc:   # the store reports a timeout as a generic error
            missing = [q for q in range(self.world) if not store.check([prefix + str(q)])]
            raise PeerLost(f"ranks {missing} did not check in within {timeout_s} s") from exc

    def reset(self) -> None:
        """Collective restart after a wait ran out: once no rank's kernel
        runs any more (each synchronises its device, then all pass a
        barrier), every rank zeroes its workspace; a second barrier keeps any
        rank from sending into a workspace not yet zeroed."""
        self.backend.sync()
        self.dist.barrier(group=self.group)
        self.backend.zero(self.ws, self.nbytes)
        self.dist.barrier(group=self.group)
        self.broken = False
        self.calls = 0

    def close(self) -> None:
        """Collective: every rank unmaps its peers' workspaces, then, once all
        have, frees its own."""
        if self.ws is None:
            return
        self.backend.sync()            # none of this rank's kernels still writes to a peer
        for q, p in enumerate(self.peers):
            if q != self.rank:
                self.backend.close(p)
        self.peers = [self.ws]
        self.dist.barrier(group=self.group)
        self.backend.destroy(self.ws)
        self.ws = None
        self.peers = []


def _torch_dtype(code: int):
    import torch
    return {_native.F32: torch.float32, _native.F16: torch.float16, _native.BF16: torch.bfloat16}[code]
