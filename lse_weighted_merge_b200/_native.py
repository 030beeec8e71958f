"""ctypes binding of liblse_merge.so (argument marshalling only).

Every step of the merge runs in the library's CUDA kernels.  There is no
Python or CPU fallback: if the library is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblse_merge.so")

F32, F16, BF16 = 0, 1, 2
PATH_AUTO, PATH_VECTOR, PATH_LATENCY, PATH_SCALAR, PATH_STREAM, PATH_WIDE = 0, 1, 2, 3, 4, 5
PATH_NAMES = {PATH_VECTOR: "vector", PATH_LATENCY: "latency", PATH_SCALAR: "scalar",
              PATH_STREAM: "stream", PATH_WIDE: "wide"}

OK, EDTYPE, EDIMS, ENULL, ESTRIDE, EALIAS, ELAUNCH, EALIGN, EPATH, EUNSUP, ECUDA, ESCRATCH = (
    0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10, -11)
EDEVICE = -12
LAYOUT_BHRD, LAYOUT_RBHD = 0, 1
HOST_MAX_CHUNKS = 64
HOST_PIPELINE = 1
CP_MAX_WORLD = 8
CP_STATUS_OFFSET = 64
CP_IPC_HANDLE_BYTES = 64
CP_FLAG_CROSS_GPU_PROTOCOL = 1
CP_FLAG_TEST_SILENT_LAST_RANK = 2
CP_NOALLOC_SCRATCH_BYTES = 16 << 20

# Every symbol include/lse_merge.h declares.
EXPORTS = ("lse_merge", "lse_merge_with_path", "lse_merge_plan_query", "lse_merge_state_update",
           "lse_merge_decode_partials", "lse_merge_decode_attention", "lse_merge_strerror",
           "lse_merge_last_cuda_error", "lse_merge_version", "lse_merge_cp_workspace_bytes",
           "lse_merge_cp_validate", "lse_merge_cp_exchange_merge", "lse_merge_cp_workspace_create",
           "lse_merge_cp_workspace_destroy", "lse_merge_cp_ipc_handle", "lse_merge_cp_ipc_open",
           "lse_merge_cp_ipc_close", "lse_merge_cp_status", "lse_merge_cp_workspace_zero",
           "lse_merge_cp_exchange_merge_noalloc", "lse_merge_cp_noalloc_status",
           "lse_merge_decode_workspace_bytes", "lse_merge_decode_attention_ws",
           "lse_merge_host_stage_bytes", "lse_merge_host_create", "lse_merge_host_destroy",
           "lse_merge_host")
ABI_VERSION = 4


class Strides(ctypes.Structure):
    _fields_ = [("o_r", ctypes.c_int64), ("o_b", ctypes.c_int64), ("o_h", ctypes.c_int64),
                ("lse_r", ctypes.c_int64), ("lse_b", ctypes.c_int64), ("lse_h", ctypes.c_int64)]


class StateStrides(ctypes.Structure):
    _fields_ = [("o_b", ctypes.c_int64), ("o_h", ctypes.c_int64),
                ("lse_b", ctypes.c_int64), ("lse_h", ctypes.c_int64)]


class AttnStrides(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("q_b", "q_h", "k_b", "k_h", "k_l", "v_b", "v_h", "v_l")]


class Plan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("vec", ctypes.c_int), ("lanes", ctypes.c_int),
                ("rc", ctypes.c_int), ("nv", ctypes.c_int), ("slices_per_row", ctypes.c_int),
                ("block", ctypes.c_int),
                ("grid", ctypes.c_int64), ("groups", ctypes.c_int64)]

    def as_dict(self) -> dict:
        d = {f: getattr(self, f) for f, _ in self._fields_}
        d["path_name"] = PATH_NAMES.get(self.path, "?")
        return d


_P8 = ctypes.c_void_p * CP_MAX_WORLD


class CpArgs(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int), ("rank_begin", ctypes.c_int), ("rank_count", ctypes.c_int),
                ("local_o", _P8), ("local_lse", _P8), ("out_o", _P8), ("out_lse", _P8),
                ("ws", _P8), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("D", ctypes.c_int), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("timeout_ns", ctypes.c_int64), ("flags", ctypes.c_int)]


def cp_args(world: int, rank_begin: int, local_o, local_lse, out_o, out_lse, ws,
            B: int, H: int, D: int, in_dtype: int, out_dtype: int, timeout_ns: int,
            flags: int = 0) -> CpArgs:
    """Fill lse_merge_cp_args from lists of raw pointers (one per played rank / per rank)."""
    def arr(ptrs):
        if len(ptrs) > CP_MAX_WORLD:
            raise ValueError(f"at most {CP_MAX_WORLD} ranks, got {len(ptrs)} pointers")
        a = _P8()
        for i, x in enumerate(ptrs):
            a[i] = int(x) if x else None
        return a
    return CpArgs(int(world), int(rank_begin), len(local_o), arr(local_o), arr(local_lse),
                  arr(out_o), arr(out_lse), arr(ws), int(B), int(H), int(D),
                  int(in_dtype), int(out_dtype), int(timeout_ns), int(flags))


class LseMergeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"lse_merge failed ({code}): {what}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m lse_weighted_merge_b200.build` "
            "(nvcc, sm_100a). The merge has no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    common = [vp, vp, i, i, i, i, ctypes.POINTER(Strides), i, i, vp, vp, vp]
    lib.lse_merge.argtypes = common
    lib.lse_merge.restype = i
    lib.lse_merge_with_path.argtypes = common + [i]
    lib.lse_merge_with_path.restype = i
    lib.lse_merge_plan_query.argtypes = [vp, vp, i, i, i, i, ctypes.POINTER(Strides), i, i, vp, vp,
                                         i, ctypes.POINTER(Plan)]
    lib.lse_merge_plan_query.restype = i
    lib.lse_merge_state_update.argtypes = [vp, vp, vp, vp, i, i, i, ctypes.POINTER(StateStrides),
                                           i, i, vp]
    lib.lse_merge_state_update.restype = i
    attn = [vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, ctypes.POINTER(AttnStrides), i]
    lib.lse_merge_decode_partials.argtypes = attn + [vp, vp, vp]
    lib.lse_merge_decode_partials.restype = i
    lib.lse_merge_decode_attention.argtypes = attn + [i, vp, vp, vp]
    lib.lse_merge_decode_attention.restype = i
    lib.lse_merge_decode_attention_ws.argtypes = attn + [i, vp, ctypes.c_int64, vp, vp, vp]
    lib.lse_merge_decode_attention_ws.restype = i
    lib.lse_merge_decode_workspace_bytes.argtypes = [i, i, i, i, i, ctypes.POINTER(ctypes.c_int64)]
    lib.lse_merge_decode_workspace_bytes.restype = i
    lib.lse_merge_host_stage_bytes.argtypes = [i, i, i, i, i, i, ctypes.POINTER(ctypes.c_int64)]
    lib.lse_merge_host_stage_bytes.restype = i
    lib.lse_merge_host_create.argtypes = [ctypes.c_int64, ctypes.POINTER(vp)]
    lib.lse_merge_host_create.restype = i
    lib.lse_merge_host_destroy.argtypes = [vp]
    lib.lse_merge_host_destroy.restype = i
    lib.lse_merge_host.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, vp, vp, i, i, vp]
    lib.lse_merge_host.restype = i
    lib.lse_merge_strerror.argtypes = [i]
    lib.lse_merge_strerror.restype = ctypes.c_char_p
    lib.lse_merge_last_cuda_error.argtypes = []
    lib.lse_merge_last_cuda_error.restype = i
    lib.lse_merge_version.argtypes = []
    lib.lse_merge_version.restype = i
    lib.lse_merge_cp_workspace_bytes.argtypes = [i, i, i, i, i, ctypes.POINTER(ctypes.c_int64)]
    lib.lse_merge_cp_workspace_bytes.restype = i
    lib.lse_merge_cp_validate.argtypes = [ctypes.POINTER(CpArgs)]
    lib.lse_merge_cp_validate.restype = i
    lib.lse_merge_cp_exchange_merge.argtypes = [ctypes.POINTER(CpArgs), vp]
    lib.lse_merge_cp_exchange_merge.restype = i
    lib.lse_merge_cp_exchange_merge_noalloc.argtypes = [ctypes.POINTER(CpArgs), vp]
    lib.lse_merge_cp_exchange_merge_noalloc.restype = i
    lib.lse_merge_cp_noalloc_status.argtypes = [ctypes.POINTER(CpArgs), ctypes.POINTER(ctypes.c_uint32)]
    lib.lse_merge_cp_noalloc_status.restype = i
    lib.lse_merge_cp_workspace_create.argtypes = [ctypes.c_int64, ctypes.POINTER(vp)]
    lib.lse_merge_cp_workspace_create.restype = i
    lib.lse_merge_cp_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.lse_merge_cp_status.restype = i
    lib.lse_merge_cp_workspace_zero.argtypes = [vp, ctypes.c_int64]
    lib.lse_merge_cp_workspace_zero.restype = i
    lib.lse_merge_cp_workspace_destroy.argtypes = [vp]
    lib.lse_merge_cp_workspace_destroy.restype = i
    lib.lse_merge_cp_ipc_handle.argtypes = [vp, vp]
    lib.lse_merge_cp_ipc_handle.restype = i
    lib.lse_merge_cp_ipc_open.argtypes = [vp, ctypes.POINTER(vp)]
    lib.lse_merge_cp_ipc_open.restype = i
    lib.lse_merge_cp_ipc_close.argtypes = [vp]
    lib.lse_merge_cp_ipc_close.restype = i
    if lib.lse_merge_version() != ABI_VERSION:
        raise ImportError(f"{LIB_PATH}: ABI version {lib.lse_merge_version()} != {ABI_VERSION}")
    return lib


lib = _load()

# Vectorcall forwarding of the per-call entry points (csrc/pyfast.c), built
# next to the library; it calls the same C functions for a fraction of
# ctypes' marshalling cost.  Without it the ctypes calls below are used.
try:
    from . import _fast
except ImportError:
    _fast = None


def strerror(code: int) -> str:
    return lib.lse_merge_strerror(int(code)).decode()


def _strides(s) -> ctypes.POINTER(Strides) | None:
    if s is None:
        return None
    if isinstance(s, Strides):
        return ctypes.pointer(s)
    return ctypes.pointer(Strides(*[int(x) for x in _stride_tuple(s)]))


def _stride_tuple(s):
    """Strides as the flat (o_r, o_b, o_h, lse_r, lse_b, lse_h) tuple, or None."""
    if s is None:
        return None
    if isinstance(s, Strides):
        return (s.o_r, s.o_b, s.o_h, s.lse_r, s.lse_b, s.lse_h)
    if len(s) == 6:
        return tuple(s)
    o, l = s
    return (*[int(x) for x in o], *[int(x) for x in l])


def merge_raw(o_ptr: int, lse_ptr: int, R: int, B: int, H: int, D: int, strides,
              in_dtype: int, out_dtype: int, out_ptr: int, out_lse_ptr: int, stream: int = 0,
              path: int = PATH_AUTO, check: bool = True) -> int:
    """Call lse_merge_with_path on raw device pointers; raises on error if ``check``."""
    if _fast is not None:
        rc = _fast.merge(o_ptr, lse_ptr, R, B, H, D, _stride_tuple(strides), in_dtype, out_dtype,
                         out_ptr, out_lse_ptr, stream or 0, path)
    else:
        rc = lib.lse_merge_with_path(o_ptr, lse_ptr, R, B, H, D, _strides(strides), in_dtype,
                                     out_dtype, out_ptr, out_lse_ptr, stream or None, path)
    if check and rc != OK:
        extra = ""
        if rc == ELAUNCH:
            extra = f" (cudaError {lib.lse_merge_last_cuda_error()})"
        raise LseMergeError(rc, strerror(rc) + extra)
    return rc


def plan_query(o_ptr: int, lse_ptr: int, R: int, B: int, H: int, D: int, strides,
               in_dtype: int, out_dtype: int, out_ptr: int, out_lse_ptr: int,
               path: int = PATH_AUTO) -> tuple[int, dict | None]:
    """Host-only: the launch plan (or the error code) for these arguments."""
    plan = Plan()
    rc = lib.lse_merge_plan_query(o_ptr, lse_ptr, R, B, H, D, _strides(strides), in_dtype,
                                  out_dtype, out_ptr, out_lse_ptr, path, ctypes.byref(plan))
    return rc, (plan.as_dict() if rc == OK else None)


def state_update_raw(acc_ptr: int, lse_acc_ptr: int, new_ptr: int, lse_new_ptr: int, B: int,
                     H: int, D: int, new_strides, acc_dtype: int, new_dtype: int,
                     stream: int = 0, check: bool = True) -> int:
    """Call lse_merge_state_update; ``new_strides`` = (o_b, o_h, lse_b, lse_h) or None."""
    if _fast is not None:
        st = None if new_strides is None else tuple(int(x) for x in new_strides)
        rc = _fast.state_update(acc_ptr, lse_acc_ptr, new_ptr, lse_new_ptr, B, H, D, st,
                                acc_dtype, new_dtype, stream or 0)
    else:
        st = None if new_strides is None else ctypes.pointer(StateStrides(*[int(x) for x in new_strides]))
        rc = lib.lse_merge_state_update(acc_ptr, lse_acc_ptr, new_ptr, lse_new_ptr, B, H, D, st,
                                        acc_dtype, new_dtype, stream or None)
    if check and rc != OK:
        extra = ""
        if rc == ELAUNCH:
            extra = f" (cudaError {lib.lse_merge_last_cuda_error()})"
        raise LseMergeError(rc, strerror(rc) + extra)
    return rc


def _check(rc: int, check: bool) -> int:
    if check and rc != OK:
        extra = ""
        if rc == ELAUNCH:
            extra = f" (cudaError {lib.lse_merge_last_cuda_error()})"
        raise LseMergeError(rc, strerror(rc) + extra)
    return rc


def decode_raw(q_ptr: int, k_ptr: int, v_ptr: int, kv_len_ptr: int, B: int, Hq: int, Hkv: int,
               L: int, D: int, R: int, scale: float, strides, dtype: int, out_ptr: int,
               out_lse_ptr: int, stream: int = 0, fused: bool = True, out_dtype: int = BF16,
               check: bool = True, workspace: int = 0, workspace_bytes: int = 0) -> int:
    """lse_merge_decode_attention_ws (fused with a workspace pointer),
    lse_merge_decode_attention (fused, no workspace: the cluster form) or
    lse_merge_decode_partials (fp32 partials [B,Hq,R,D] / [B,Hq,R] into
    out_ptr / out_lse_ptr).  ``strides`` = (q_b, q_h, k_b, k_h, k_l, v_b, v_h,
    v_l) in elements, or None (dense)."""
    st = None if strides is None else ctypes.pointer(AttnStrides(*[int(x) for x in strides]))
    args = (q_ptr, k_ptr, v_ptr, kv_len_ptr or None, B, Hq, Hkv, L, D, R, float(scale), st, dtype)
    if fused and workspace:
        rc = lib.lse_merge_decode_attention_ws(*args, out_dtype, workspace, int(workspace_bytes),
                                               out_ptr, out_lse_ptr, stream or None)
    elif fused:
        rc = lib.lse_merge_decode_attention(*args, out_dtype, out_ptr, out_lse_ptr, stream or None)
    else:
        rc = lib.lse_merge_decode_partials(*args, out_ptr, out_lse_ptr, stream or None)
    return _check(rc, check)


def host_stage_bytes(R: int, B: int, H: int, D: int, in_dtype: int, out_dtype: int) -> int:
    n = ctypes.c_int64(0)
    rc = lib.lse_merge_host_stage_bytes(R, B, H, D, in_dtype, out_dtype, ctypes.byref(n))
    if rc != OK:
        _raise(rc)
    return n.value


def host_create(stage_bytes: int) -> int:
    """lse_merge_host_create on the current device; returns the context handle."""
    h = ctypes.c_void_p()
    rc = lib.lse_merge_host_create(int(stage_bytes), ctypes.byref(h))
    if rc != OK:
        _raise(rc)
    return h.value


def host_destroy(ctx: int) -> None:
    rc = lib.lse_merge_host_destroy(ctx)
    if rc != OK:
        _raise(rc)


def host_merge_raw(ctx: int, h_o: int, h_lse: int, R: int, B: int, H: int, D: int, layout: int,
                   in_dtype: int, out_dtype: int, h_out: int, h_out_lse: int, chunks: int,
                   flags: int = 0, stream: int = 0, check: bool = True) -> int:
    """lse_merge_host: the pipelined merge of partials in host memory."""
    rc = lib.lse_merge_host(ctx, h_o, h_lse, R, B, H, D, layout, in_dtype, out_dtype, h_out,
                            h_out_lse, chunks, flags, stream or None)
    return _check(rc, check)


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, R: int, D: int) -> int:
    n = ctypes.c_int64(0)
    rc = lib.lse_merge_decode_workspace_bytes(B, Hq, Hkv, R, D, ctypes.byref(n))
    if rc != OK:
        _raise(rc)
    return n.value


def _raise(rc: int):
    extra = ""
    if rc in (ELAUNCH, ECUDA):
        extra = f" (cudaError {lib.lse_merge_last_cuda_error()})"
    raise LseMergeError(rc, strerror(rc) + extra)


def cp_workspace_bytes(world: int, B: int, H: int, D: int, in_dtype: int) -> int:
    n = ctypes.c_int64(0)
    rc = lib.lse_merge_cp_workspace_bytes(world, B, H, D, in_dtype, ctypes.byref(n))
    if rc != OK:
        _raise(rc)
    return n.value


def cp_validate(args: CpArgs) -> int:
    """Host-only: the code lse_merge_cp_exchange_merge would return for ``args``
    before launching (OK when it would launch)."""
    return lib.lse_merge_cp_validate(ctypes.byref(args))


def cp_exchange_merge_raw(args: CpArgs, stream: int = 0, check: bool = True) -> int:
    if _fast is not None:
        rc = _fast.cp_exchange_merge(ctypes.addressof(args), stream or 0)
    else:
        rc = lib.lse_merge_cp_exchange_merge(ctypes.byref(args), stream or None)
    if check and rc != OK:
        _raise(rc)
    return rc


def cp_exchange_merge_noalloc_raw(args: CpArgs, stream: int = 0, check: bool = True) -> int:
    """lse_merge_cp_exchange_merge_noalloc: every rank in one launch, the
    workspaces taken from the library's static device array (args.ws unused)."""
    rc = lib.lse_merge_cp_exchange_merge_noalloc(ctypes.byref(args), stream or None)
    if check and rc != OK:
        _raise(rc)
    return rc


def cp_noalloc_status(args: CpArgs, check: bool = True):
    """lse_merge_cp_noalloc_status: the status word of every rank of the last
    no-alloc call with these sizes (0: all of that rank's waits completed).
    Returns (code, [status of rank 0, ..., rank world-1])."""
    st = (ctypes.c_uint32 * max(1, int(args.world)))()
    rc = lib.lse_merge_cp_noalloc_status(ctypes.byref(args), st)
    if check and rc != OK:
        _raise(rc)
    return rc, [int(st[q]) for q in range(int(args.world))]


def cp_workspace_create(nbytes: int) -> int:
    p = ctypes.c_void_p()
    rc = lib.lse_merge_cp_workspace_create(int(nbytes), ctypes.byref(p))
    if rc != OK:
        _raise(rc)
    return p.value


def cp_status(ptr: int) -> int:
    st = ctypes.c_uint32(0)
    rc = lib.lse_merge_cp_status(ptr, ctypes.byref(st))
    if rc != OK:
        _raise(rc)
    return st.value


def cp_workspace_zero(ptr: int, nbytes: int) -> None:
    rc = lib.lse_merge_cp_workspace_zero(ptr, int(nbytes))
    if rc != OK:
        _raise(rc)


def cp_workspace_destroy(ptr: int) -> None:
    rc = lib.lse_merge_cp_workspace_destroy(ptr)
    if rc != OK:
        _raise(rc)


def cp_ipc_handle(ptr: int) -> bytes:
    buf = ctypes.create_string_buffer(CP_IPC_HANDLE_BYTES)
    rc = lib.lse_merge_cp_ipc_handle(ptr, buf)
    if rc != OK:
        _raise(rc)
    return buf.raw


def cp_ipc_open(handle: bytes) -> int:
    if len(handle) != CP_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {CP_IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    buf = ctypes.create_string_buffer(bytes(handle), CP_IPC_HANDLE_BYTES)
    p = ctypes.c_void_p()
    rc = lib.lse_merge_cp_ipc_open(buf, ctypes.byref(p))
    if rc != OK:
        _raise(rc)
    return p.value


def cp_ipc_close(ptr: int) -> None:
    rc = lib.lse_merge_cp_ipc_close(ptr)
    if rc != OK:
        _raise(rc)
