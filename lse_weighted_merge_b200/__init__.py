"""B200 (sm_100a) LSE-weighted merge of context-parallel decode partials.

    out, out_lse = merge(partial_o, partial_lse)

combines R partial attention outputs o_r (one per KV shard) and their
log-sum-exp values lse_r into the output of attention over the whole KV
sequence (page "[flashinfer] FlashInfer의 Context-Parallel Decode 최적화:
Fused A2A + LSE Reduce", sections "들어가며" and "코드 분석 / 1. Fused Kernel
구현").  PyTorch only supplies device memory and the current stream; the
merge itself is one launch of the library's CUDA kernel through its C ABI.
"""
from __future__ import annotations

# The binding is loaded on first use, so that the input generators (synth)
# and the build script import without the compiled library.  Using any of
# these names without liblse_merge.so raises ImportError: there is no
# fallback.
_CP = ("cp_exchange_merge", "CPMergeCall", "cp_workspace", "cp_status", "CPExchangeMerge", "PeerLost")
_API = ("merge", "merge_state_", "merge_host", "release_host_workspace", "merge_raw",
        "state_update_raw", "decode_attention", "decode_raw", "plan_query", "strerror", "LseMergeError", "dtype_code",
        "F32", "F16", "BF16", "PATH_AUTO", "PATH_VECTOR", "PATH_LATENCY", "PATH_SCALAR",
        "PATH_STREAM")
__all__ = list(_API) + list(_CP)


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    if name in _CP:
        from . import cp
        return getattr(cp, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
