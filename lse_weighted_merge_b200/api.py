"""The torch-facing call: tensors in, one C-ABI launch, tensors out."""
from __future__ import annotations

import threading

from ._native import (BF16, F16, F32, PATH_AUTO, PATH_LATENCY, PATH_SCALAR, PATH_STREAM,
                      PATH_VECTOR,
                      LseMergeError, decode_raw, decode_workspace_bytes, merge_raw, plan_query,
                      state_update_raw,
                      strerror)


def dtype_code(dtype) -> int:
    import torch
    codes = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
    if dtype not in codes:
        raise TypeError(f"unsupported dtype {dtype}; use float32, float16 or bfloat16")
    return codes[dtype]


def _rbh_strides(partial_o, partial_lse, layout: str):
    """(r, b, h) element strides and (R, B, H, D) from tensors in ``layout``."""
    if partial_o.dim() != 4 or partial_lse.dim() != 3:
        raise ValueError("partial_o must be 4-D and partial_lse 3-D")
    if partial_o.stride(-1) != 1:
        raise ValueError("partial_o must be contiguous along D")
    so, sl = partial_o.stride(), partial_lse.stride()
    if layout == "bhrd":
        B, H, R, D = partial_o.shape
        want = (B, H, R)
        o_str, l_str = (so[2], so[0], so[1]), (sl[2], sl[0], sl[1])
    elif layout == "rbhd":
        R, B, H, D = partial_o.shape
        want = (R, B, H)
        o_str, l_str = (so[0], so[1], so[2]), (sl[0], sl[1], sl[2])
    else:
        raise ValueError(f"layout must be 'bhrd' or 'rbhd', not {layout!r}")
    if tuple(partial_lse.shape) != want:
        raise ValueError(f"partial_lse shape {tuple(partial_lse.shape)} != {want}")
    return (R, B, H, D), (o_str, l_str)


def merge(partial_o, partial_lse, *, layout: str = "bhrd", out_dtype=None, out=None,
          out_lse=None, path: int = PATH_AUTO):
    """Merge partials with their lse weights on the GPU.

    partial_o:   CUDA tensor [B, H, R, D] (layout "bhrd", the partial axis at
                 dim -2) or [R, B, H, D] (layout "rbhd"), float32 / float16 /
                 bfloat16, any strides with stride 1 along D.
    partial_lse: CUDA float32 tensor [B, H, R] or [R, B, H] (same layout).
    out_dtype:   output element type (default: partial_o's).
    out, out_lse: optional preallocated dense [B, H, D] and [B, H] outputs.
    Returns (out [B, H, D], out_lse [B, H]).  Enqueued on the current stream.
    """
    import torch
    if not partial_o.is_cuda or not partial_lse.is_cuda:
        raise ValueError("merge runs on CUDA tensors only (there is no CPU path)")
    if partial_lse.dtype != torch.float32:
        raise TypeError("partial_lse must be float32")
    (R, B, H, D), st = _rbh_strides(partial_o, partial_lse, layout)
    out_dtype = out_dtype or partial_o.dtype
    dev = partial_o.device
    if out is None:
        out = torch.empty((B, H, D), dtype=out_dtype, device=dev)
    if out_lse is None:
        out_lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if tuple(out.shape) != (B, H, D) or not out.is_contiguous() or out.dtype != out_dtype:
        raise ValueError("out must be a contiguous [B, H, D] tensor of out_dtype")
    if tuple(out_lse.shape) != (B, H) or not out_lse.is_contiguous() or out_lse.dtype != torch.float32:
        raise ValueError("out_lse must be a contiguous float32 [B, H] tensor")
    if partial_lse.device != dev or out.device != dev or out_lse.device != dev:
        raise ValueError("all tensors must be on the same CUDA device")
    args = (partial_o.data_ptr(), partial_lse.data_ptr(), R, B, H, D, (*st[0], *st[1]),
            dtype_code(partial_o.dtype), dtype_code(out_dtype), out.data_ptr(), out_lse.data_ptr())
    if torch.cuda.current_device() == dev.index:
        merge_raw(*args, torch.cuda.current_stream().cuda_stream, path)
    else:   # the library launches on the current device: make it the tensors' one
        with torch.cuda.device(dev):
            merge_raw(*args, torch.cuda.current_stream().cuda_stream, path)
    return out, out_lse


# Host contexts of merge_host (lse_merge_host_create), one per device, kept
# between calls and grown when a call needs a larger staging area.
# merge_host's contexts are shared by every thread; one call at a time per
# process uses them (the copies and merges it enqueues still overlap).
_HOST_CTX: dict = {}
_HOST_LOCK = threading.Lock()


def release_host_workspace() -> None:
    """Free the host contexts (device staging areas, streams and events) that
    merge_host keeps between calls; each waits for its last call first."""
    from ._native import host_destroy
    with _HOST_LOCK:
        for (dev_index, _), ctx in list(_HOST_CTX.items()):
            import torch
            with torch.cuda.device(dev_index):
                host_destroy(ctx)
        _HOST_CTX.clear()


def _host_context(device, need: int) -> int:
    """The host context of `device`, remade larger when `need` staging bytes
    exceed its area (the old one is destroyed after its last call)."""
    import torch
    from ._native import host_create, host_destroy
    for key in [k for k in _HOST_CTX if k[0] == device.index]:
        if key[1] >= need:
            return _HOST_CTX[key]
        with torch.cuda.device(device):
            host_destroy(_HOST_CTX.pop(key))
    with torch.cuda.device(device):
        ctx = host_create(need)
    _HOST_CTX[(device.index, need)] = ctx
    return ctx


def merge_host(partial_o, partial_lse, *, layout: str = "bhrd", out_dtype=None, chunks: int = 8,
               device=None, out=None, out_lse=None, sync: bool = True, pipeline: bool = False):
    """Merge partials that live in (pinned) host memory; results land in host memory.

    One call of the C ABI's lse_merge_host on a host context this module
    keeps per device: the batch is cut into ``chunks`` slices along B; slice
    i is copied to the GPU on one stream while slice i-1 is merged (one kernel
    launch on a second stream) and slice i-2's result is copied back on a
    third, so the merge and the device-to-host copies hide behind the
    host-to-device copy of the partials, which bounds the whole call.
    Layouts ("bhrd" [B,H,R,D] or "rbhd" [R,B,H,D], dense) and dtypes as in
    merge().  Pass pinned ``out``/``out_lse`` to avoid a host allocation per
    call; pinned inputs for full copy speed.

    Returns the host tensors (out [B, H, D], out_lse [B, H]).  With
    ``sync=False`` the call returns once everything is enqueued; the current
    stream of ``device`` is made to wait for the last copy, so synchronising
    that stream (or the device) makes the results valid.

    ``pipeline=True`` (with ``sync=False``, for a stream of batches) lets this
    call's uploads start as soon as the previous call's uploads end, instead
    of after the previous call's last copy back (LSE_MERGE_HOST_PIPELINE):
    slice i's staging bytes are reused once the previous call has merged
    slice i.  The uploads then no longer wait for the current stream, so the
    host inputs must not be written by device work still pending there
    (inputs filled by the CPU, the usual case, are fine); give consecutive
    pipelined calls distinct host outputs, or read each call's outputs before
    the next call's copies back can overwrite them.
    """
    import torch
    from ._native import (HOST_MAX_CHUNKS, HOST_PIPELINE, LAYOUT_BHRD, LAYOUT_RBHD, host_merge_raw,
                          host_stage_bytes)
    if partial_o.is_cuda or partial_lse.is_cuda:
        raise ValueError("merge_host takes host tensors; use merge() for device tensors")
    if partial_lse.dtype != torch.float32:
        raise TypeError("partial_lse must be float32")
    (R, B, H, D), _ = _rbh_strides(partial_o, partial_lse, layout)
    if not (partial_o.is_contiguous() and partial_lse.is_contiguous()):
        raise ValueError("merge_host wants contiguous host tensors")
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    out_dtype = out_dtype or partial_o.dtype
    if out is None:
        out = torch.empty((B, H, D), dtype=out_dtype).pin_memory()
    if out_lse is None:
        out_lse = torch.empty((B, H), dtype=torch.float32).pin_memory()
    if out.is_cuda or out_lse.is_cuda:
        raise ValueError("merge_host writes host tensors: out and out_lse must be on the CPU")
    if tuple(out.shape) != (B, H, D) or not out.is_contiguous() or out.dtype != out_dtype:
        raise ValueError("out must be a contiguous [B, H, D] tensor of out_dtype")
    if tuple(out_lse.shape) != (B, H) or not out_lse.is_contiguous() or out_lse.dtype != torch.float32:
        raise ValueError("out_lse must be a contiguous float32 [B, H] tensor")
    ind, outd = dtype_code(partial_o.dtype), dtype_code(out_dtype)
    chunks = max(1, min(int(chunks), B, HOST_MAX_CHUNKS))
    with _HOST_LOCK:
        with torch.cuda.device(device):
            ctx = _host_context(device, host_stage_bytes(R, B, H, D, ind, outd))
            s = torch.cuda.current_stream(device)
            host_merge_raw(ctx, partial_o.data_ptr(), partial_lse.data_ptr(), R, B, H, D,
                           LAYOUT_BHRD if layout == "bhrd" else LAYOUT_RBHD, ind, outd,
                           out.data_ptr(), out_lse.data_ptr(), chunks,
                           HOST_PIPELINE if pipeline else 0, s.cuda_stream)
    if sync:
        s.synchronize()
    return out, out_lse


def merge_state_(o_acc, lse_acc, o_new, lse_new):
    """Fold one new partial into an accumulator, in place, on the GPU.

    o_acc [B, H, D] (contiguous; float32 / float16 / bfloat16) and lse_acc
    [B, H] (contiguous float32) are read and overwritten with the merge of
    themselves and (o_new [B, H, D], any strides with stride 1 along D;
    lse_new [B, H] float32).  An accumulator with lse_acc = -inf is empty: the
    values in its o_acc never reach the result.  Returns (o_acc, lse_acc).
    """
    import torch
    for t in (o_acc, lse_acc, o_new, lse_new):
        if not t.is_cuda:
            raise ValueError("merge_state_ runs on CUDA tensors only (there is no CPU path)")
    if lse_acc.dtype != torch.float32 or lse_new.dtype != torch.float32:
        raise TypeError("lse tensors must be float32")
    if o_acc.dim() != 3 or not o_acc.is_contiguous() or not lse_acc.is_contiguous():
        raise ValueError("o_acc must be a contiguous [B, H, D] tensor, lse_acc contiguous [B, H]")
    B, H, D = o_acc.shape
    if tuple(o_new.shape) != (B, H, D) or tuple(lse_acc.shape) != (B, H) or \
            tuple(lse_new.shape) != (B, H) or o_new.stride(-1) != 1:
        raise ValueError("shapes must be o [B, H, D] (stride 1 along D) and lse [B, H]")
    dev = o_acc.device
    if any(t.device != dev for t in (lse_acc, o_new, lse_new)):
        raise ValueError("all tensors must be on the same CUDA device")
    st = (o_new.stride(0), o_new.stride(1), lse_new.stride(0), lse_new.stride(1))
    with torch.cuda.device(dev):
        state_update_raw(o_acc.data_ptr(), lse_acc.data_ptr(), o_new.data_ptr(),
                         lse_new.data_ptr(), B, H, D, st, dtype_code(o_acc.dtype),
                         dtype_code(o_new.dtype), torch.cuda.current_stream(dev).cuda_stream)
    return o_acc, lse_acc


# Workspaces of the fused decode attention, one per (device, stream): zeroed
# once when made, left ready (counters at 0) by every call, so calls on one
# stream can share one; calls on different streams get different ones.
_decode_ws: dict = {}
_decode_ws_lock = threading.Lock()


def _decode_workspace(dev, stream_handle: int, nbytes: int):
    import torch
    key = (dev.index, stream_handle)
    with _decode_ws_lock:
        ws = _decode_ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.zeros(max(nbytes, 1 << 16), dtype=torch.uint8, device=dev)
            _decode_ws[key] = ws
        return ws


def decode_attention(q, k, v, *, splits: int | None = None, scale: float | None = None,
                     kv_len=None, out_dtype=None, fused: bool | str | None = None):
    """Split-KV decode attention on the GPU, its partials merged by LSE weight.

    q [B, Hq, D]; k, v [B, Hkv, L, D] (bf16 or fp16, stride 1 along D, other
    strides free); Hq a multiple of Hkv; D 64 or 128; kv_len an optional int32
    CUDA tensor [B] of valid key counts.  The keys of each sequence are cut
    into ``splits`` shards (default: enough shards for about two CTAs per SM,
    a power of two of at least 64 keys each, at most 64).

    fused=False (the default): the partials kernel, then merge(), two
    launches; on B200 the fastest form (the partials stay in L2 and the
    second launch overlaps the first one's drain).  fused=True: one launch;
    each shard's CTA writes its fp32 partial into a workspace kept for this
    device and stream, and the last shard of each (sequence, KV head) to
    finish merges them (lse_merge_decode_attention_ws), 1-3 % slower than
    the two launches on large batches.  fused="cluster": one launch in which the shards of a
    (sequence, KV head) form a thread-block cluster and merge through
    distributed shared memory, no workspace (splits 1, 2, 4 or 8; cluster
    scheduling leaves SM slots idle, so it is slower on large batches).
    Returns (out [B, Hq, D], lse [B, Hq]) with the natural-log lse of the
    scaled scores.
    """
    import math
    import torch
    B, Hq, D = q.shape
    _, Hkv, L, _ = k.shape
    if tuple(v.shape) != tuple(k.shape) or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k and v must be [B, Hkv, L, D] with q [B, Hq, D]")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("decode_attention runs on CUDA tensors only")
    if q.stride(-1) != 1 or k.stride(-1) != 1 or v.stride(-1) != 1:
        raise ValueError("q, k and v must be contiguous along D")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    if fused is None:
        fused = False
    if fused not in (True, False, "cluster"):
        raise ValueError("fused must be True, False or 'cluster'")
    dev = q.device
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if splits is None:
        want = max(1, -(-2 * sms // (B * Hkv)))
        cap = 8 if fused == "cluster" else 64
        splits = 1
        while splits < want and splits < cap and splits * 64 < L:
            splits *= 2
    scale = (1.0 / math.sqrt(D)) if scale is None else float(scale)
    out_dtype = out_dtype or q.dtype
    st = (q.stride(0), q.stride(1), k.stride(0), k.stride(1), k.stride(2),
          v.stride(0), v.stride(1), v.stride(2))
    klen = 0
    if kv_len is not None:
        if kv_len.dtype != torch.int32 or not kv_len.is_cuda or kv_len.numel() != B:
            raise ValueError("kv_len must be an int32 CUDA tensor of B lengths")
        kv_len = kv_len.contiguous()
        klen = kv_len.data_ptr()
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev).cuda_stream
        if fused:
            out = torch.empty((B, Hq, D), dtype=out_dtype, device=dev)
            lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
            ws_ptr, ws_bytes = 0, 0
            if fused is True:
                ws_bytes = decode_workspace_bytes(B, Hq, Hkv, splits, D)
                ws_ptr = _decode_workspace(dev, s, ws_bytes).data_ptr()
            decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), klen, B, Hq, Hkv, L, D, splits,
                       scale, st, dtype_code(q.dtype), out.data_ptr(), lse.data_ptr(), s,
                       fused=True, out_dtype=dtype_code(out_dtype), workspace=ws_ptr,
                       workspace_bytes=ws_bytes)
            return out, lse
        po = torch.empty((B, Hq, splits, D), dtype=torch.float32, device=dev)
        pl = torch.empty((B, Hq, splits), dtype=torch.float32, device=dev)
        decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), klen, B, Hq, Hkv, L, D, splits,
                   scale, st, dtype_code(q.dtype), po.data_ptr(), pl.data_ptr(), s, fused=False)
        return merge(po, pl, out_dtype=out_dtype)
