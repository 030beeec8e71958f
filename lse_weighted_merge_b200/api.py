"""The torch-facing call: tensors in, one C-ABI launch, tensors out."""
from __future__ import annotations

from ._native import (BF16, F16, F32, PATH_AUTO, PATH_LATENCY, PATH_SCALAR, PATH_STREAM,
                      PATH_VECTOR,
                      LseMergeError, merge_raw, plan_query, strerror)


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
    stream = torch.cuda.current_stream(dev).cuda_stream
    merge_raw(partial_o.data_ptr(), partial_lse.data_ptr(), R, B, H, D, st,
              dtype_code(partial_o.dtype), dtype_code(out_dtype), out.data_ptr(),
              out_lse.data_ptr(), stream, path)
    return out, out_lse
