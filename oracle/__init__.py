"""fp64 CPU oracle of the LSE-weighted merge -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this package.  The product path
(``lse_weighted_merge_b200``) never imports it and shares no code with it.

The arithmetic lives in ``lse_merge_oracle.c`` (plain C, fp64), which states
the merge of the page "[flashinfer] FlashInfer의 Context-Parallel Decode
최적화: Fused A2A + LSE Reduce", sections "들어가며" and "코드 분석 / 1. Fused
Kernel 구현".  This module only compiles that file with gcc and marshals numpy
arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lse_merge_oracle.c")
# Runs the unchanged merge on several host threads (CPU-baseline timing only).
THREADS_SRC = os.path.join(HERE, "oracle_threads.c")
LIB = os.path.join(HERE, "liboracle.so")

# Element types, numbered like the public C-ABI (defined again here on purpose).
F32, F16, BF16 = 0, 1, 2


def build(out_path: str = LIB, src: str = SRC) -> str:
    """Compile the oracle with gcc (``src``: another copy of the source, as the
    tests that plant a mistake in one use)."""
    cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-fno-fast-math", "-pthread",
           src, THREADS_SRC, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    i64p = ctypes.POINTER(ctypes.c_int64)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_widen.restype = ctypes.c_double
    lib.oracle_widen.argtypes = [ctypes.c_uint32, ctypes.c_int]
    lib.oracle_lse_merge.restype = ctypes.c_int
    lib.oracle_lse_merge.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, i64p, i64p, ctypes.c_int, dp, dp]
    lib.oracle_attention_shard.restype = None
    lib.oracle_attention_shard.argtypes = [
        dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
        ctypes.c_int, dp, dp]
    lib.oracle_state_update.restype = ctypes.c_int
    lib.oracle_state_update.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_int64, ctypes.c_int64, dp, dp]
    lib.oracle_lse_merge_threads.restype = ctypes.c_int
    lib.oracle_lse_merge_threads.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, i64p, i64p, ctypes.c_int, dp, dp, ctypes.c_int,
        ctypes.POINTER(ctypes.c_int)]
    lib.oracle_host_threads.restype = ctypes.c_int
    lib.oracle_cp_exchange_merge.restype = ctypes.c_int
    lib.oracle_cp_exchange_merge.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, dp, dp]
    return lib


_cached: dict[str, ctypes.CDLL] = {}


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the oracle library, building it first if it is missing or stale."""
    path = path or LIB
    if path in _cached:
        return _cached[path]
    if path == LIB and (not os.path.exists(LIB)
                        or os.path.getmtime(LIB) < max(os.path.getmtime(SRC),
                                                       os.path.getmtime(THREADS_SRC))):
        build(LIB)
    lib = _bind(ctypes.CDLL(path))
    _cached[path] = lib
    return lib


def widen(bits: int, dtype: int, lib: ctypes.CDLL | None = None) -> float:
    return (lib or load()).oracle_widen(int(bits), int(dtype))


def merge(partial_o: np.ndarray, partial_lse: np.ndarray, R: int, B: int, H: int,
          D: int, o_strides, lse_strides, in_dtype: int,
          lib: ctypes.CDLL | None = None, threads: int = 1, stats: dict | None = None):
    """Run the fp64 merge.

    partial_o: a flat numpy buffer holding the raw elements (uint16 bit
    patterns for F16/BF16, float32 for F32); partial_lse: flat float32.
    Strides are (r, b, h) in elements; the d stride is 1.
    threads: 1 runs oracle_lse_merge on the calling thread; any other value
    splits the batches over that many host threads (0: one per core), each
    running the same function; ``stats["threads"]`` receives the count used.
    Returns (out [B, H, D] float64, out_lse [B, H] float64).
    """
    lib = lib or load()
    po = np.ascontiguousarray(partial_o)
    pl = np.ascontiguousarray(partial_lse, dtype=np.float32)
    want = np.float32 if in_dtype == F32 else np.uint16
    if po.dtype != want:
        raise TypeError(f"partial_o must be {np.dtype(want).name} for dtype {in_dtype}")
    os_ = (ctypes.c_int64 * 3)(*[int(s) for s in o_strides])
    ls_ = (ctypes.c_int64 * 3)(*[int(s) for s in lse_strides])
    out = np.empty((B, H, D), dtype=np.float64)
    out_lse = np.empty((B, H), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    if threads == 1:
        rc = lib.oracle_lse_merge(po.ctypes.data, pl.ctypes.data, R, B, H, D, os_, ls_, in_dtype,
                                  out.ctypes.data_as(dp), out_lse.ctypes.data_as(dp))
        used = 1
    else:
        n = ctypes.c_int(0)
        rc = lib.oracle_lse_merge_threads(po.ctypes.data, pl.ctypes.data, R, B, H, D, os_, ls_,
                                          in_dtype, out.ctypes.data_as(dp),
                                          out_lse.ctypes.data_as(dp), int(threads),
                                          ctypes.byref(n))
        used = n.value
    if stats is not None:
        stats["threads"] = used
    if rc != 0:
        raise ValueError(f"oracle_lse_merge returned {rc}")
    return out, out_lse


def attention_shard(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                    begin: int, end: int, lib: ctypes.CDLL | None = None):
    """Softmax attention of q [D] over keys [begin, end) of k, v [L, D] (fp64)."""
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    L, D = k.shape
    o = np.empty(D, dtype=np.float64)
    lse = np.empty(1, dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_attention_shard(q.ctypes.data_as(dp), k.ctypes.data_as(dp),
                               v.ctypes.data_as(dp), L, D, float(scale), begin, end,
                               o.ctypes.data_as(dp), lse.ctypes.data_as(dp))
    return o, float(lse[0])


def state_update(acc: np.ndarray, lse_acc: np.ndarray, acc_dtype: int, new: np.ndarray,
                 lse_new: np.ndarray, new_dtype: int, B: int, H: int, D: int,
                 new_strides=None, lse_new_strides=None, lib: ctypes.CDLL | None = None):
    """Fold ``new`` into the accumulator ``acc`` (fp64 result, nothing modified).

    acc: flat dense [B, H, D] storage (uint16 bits or float32); lse_acc: [B, H]
    float32; new: flat storage with (b, h) element strides ``new_strides``
    (default dense [B, H, D]); lse_new with ``lse_new_strides`` (default
    dense [B, H]).  Returns (out [B, H, D] float64, out_lse [B, H] float64).
    """
    lib = lib or load()
    nb, nh = new_strides or (H * D, D)
    lb, lh = lse_new_strides or (H, 1)
    a = np.ascontiguousarray(acc)
    n = np.ascontiguousarray(new)
    la = np.ascontiguousarray(lse_acc, dtype=np.float32)
    ln = np.ascontiguousarray(lse_new, dtype=np.float32)
    out = np.empty((B, H, D), dtype=np.float64)
    out_lse = np.empty((B, H), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = lib.oracle_state_update(a.ctypes.data, la.ctypes.data, acc_dtype, n.ctypes.data,
                                 ln.ctypes.data, new_dtype, B, H, D, nb, nh, lb, lh,
                                 out.ctypes.data_as(dp), out_lse.ctypes.data_as(dp))
    if rc != 0:
        raise ValueError(f"oracle_state_update returned {rc}")
    return out, out_lse


def cp_exchange_merge(local_o: np.ndarray, local_lse: np.ndarray, world: int, B: int, H: int,
                      D: int, in_dtype: int, lib: ctypes.CDLL | None = None):
    """Exchange heads between ``world`` ranks, then merge (fp64).

    local_o: flat [world, B, H, D] raw elements (uint16 bits or float32), rank
    s's partials in block s; local_lse: [world, B, H] float32.  Rank q owns
    heads [q*H/world, (q+1)*H/world).  Returns (out [world, B, H/world, D],
    out_lse [world, B, H/world]) float64, block q being rank q's result.
    """
    lib = lib or load()
    po = np.ascontiguousarray(local_o)
    pl = np.ascontiguousarray(local_lse, dtype=np.float32)
    want = np.float32 if in_dtype == F32 else np.uint16
    if po.dtype != want:
        raise TypeError(f"local_o must be {np.dtype(want).name} for dtype {in_dtype}")
    if po.size != world * B * H * D or pl.size != world * B * H:
        raise ValueError("local_o / local_lse sizes do not match world, B, H, D")
    if H % world:
        raise ValueError("H must be a multiple of world")
    Hq = H // world
    out = np.empty((world, B, Hq, D), dtype=np.float64)
    out_lse = np.empty((world, B, Hq), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = lib.oracle_cp_exchange_merge(po.ctypes.data, pl.ctypes.data, world, B, H, D, in_dtype,
                                      out.ctypes.data_as(dp), out_lse.ctypes.data_as(dp))
    if rc != 0:
        raise ValueError(f"oracle_cp_exchange_merge returned {rc}")
    return out, out_lse
