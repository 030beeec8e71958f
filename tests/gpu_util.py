"""Helpers of the GPU parity tests: upload seeded inputs, run the C-ABI merge,
compare with the fp64 oracle under the parity tolerance.

Tolerance (written here once, used by every GPU test):
  * bf16 / fp16 output: |gpu - oracle| <= 4e-3 * (1 + |oracle|); the
    round-to-nearest-even of the output alone contributes up to 2^-9 |x|
    (bf16) or 2^-12 |x| (fp16);
  * fp32 output: |gpu - oracle| <= 1e-5 * (1 + |oracle|); fp32 accumulation
    of R products adds about R * 2^-24 * max|o| at worst;
  * merged lse: |gpu - oracle| <= max(1e-5, 2^-22 |oracle|): 1e-5 absolute
    wherever fp32 can hold it (|lse| < 41.9, which covers every workload);
    beyond that two fp32 ulps, since the fp32 output itself cannot be closer
    than half an ulp (3e-5 at |lse| = 1000);
  * a row whose shards are all empty: out exactly 0 and lse exactly -inf;
  * no NaN anywhere unless an input lse is NaN or +inf.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import synth

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
OUT_TOL = {"bf16": 4e-3, "f16": 4e-3, "f32": 1e-5}
LSE_TOL = 1e-5


def upload(inp: dict, device="cuda", o_offset_elems: int = 0):
    """partial_o and partial_lse on the device (raw storage, optional misalignment)."""
    o = inp["o"]
    raw = torch.from_numpy(o.view(np.int16) if o.dtype == np.uint16 else o.view(np.int32))
    if o_offset_elems:
        pad = torch.zeros(o_offset_elems, dtype=raw.dtype)
        raw = torch.cat([pad, raw])
    d_o = raw.to(device)
    d_l = torch.from_numpy(inp["lse"]).to(device)
    return d_o, d_l, o_offset_elems * d_o.element_size()


def run_gpu(inp: dict, path: int = nat.PATH_AUTO, out_dtype: str | None = None,
            o_offset_elems: int = 0, stream: torch.cuda.Stream | None = None):
    """One C-ABI merge of ``inp``; returns (out float64 [B,H,D], lse float64 [B,H], raw out)."""
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    out_dtype = out_dtype or inp["out_dtype"]
    d_o, d_l, off = upload(inp, o_offset_elems=o_offset_elems)
    out = torch.empty((B, H, D), dtype=TORCH_DT[out_dtype], device="cuda")
    out_lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    s = stream or torch.cuda.current_stream()
    s.wait_stream(torch.cuda.current_stream())   # inputs were uploaded on the current stream
    nat.merge_raw(d_o.data_ptr() + off, d_l.data_ptr(), R, B, H, D,
                  (inp["o_strides"], inp["lse_strides"]), synth.DTYPES[inp["in_dtype"]],
                  synth.DTYPES[out_dtype], out.data_ptr(), out_lse.data_ptr(), s.cuda_stream, path)
    s.synchronize()
    return out.double().cpu().numpy(), out_lse.double().cpu().numpy(), out


def run_oracle(inp: dict):
    return oracle.merge(inp["o"], inp["lse"], inp["R"], inp["B"], inp["H"], inp["D"],
                        inp["o_strides"], inp["lse_strides"], synth.DTYPES[inp["in_dtype"]])


def check(got, got_lse, want, want_lse, out_dtype: str, what: str = "") -> dict:
    """Assert parity; return error statistics."""
    tol = OUT_TOL[out_dtype]
    assert got.shape == want.shape and got_lse.shape == want_lse.shape, what
    assert not np.isnan(got).any(), f"{what}: NaN in out"
    assert not np.isnan(got_lse).any(), f"{what}: NaN in out_lse"
    err = np.abs(got - want) / (1.0 + np.abs(want))
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"{what}: max |gpu-oracle|/(1+|oracle|) = {worst:.3e} > {tol:g}"
    empty = want_lse == -np.inf
    assert np.array_equal(got_lse == -np.inf, empty), f"{what}: -inf rows differ"
    assert np.all(got[empty] == 0.0), f"{what}: an all-empty row is not 0"
    wl = want_lse[~empty]
    lerr = np.abs(got_lse[~empty] - wl) / np.maximum(LSE_TOL, 2.0 ** -22 * np.abs(wl))
    lworst = float(lerr.max()) if lerr.size else 0.0
    assert lworst <= 1.0, f"{what}: lse error {lworst:.3f} x its bound"
    big = np.abs(want) > 1e-2
    rel = float((np.abs(got - want)[big] / np.abs(want[big])).max()) if big.any() else 0.0
    return {"max_scaled_err": worst, "lse_err_over_bound": lworst, "max_rel_err": rel,
            "empty_rows": int(empty.sum())}


def parity(inp: dict, path: int = nat.PATH_AUTO, what: str = "", **kw) -> dict:
    got, got_lse, _ = run_gpu(inp, path, **kw)
    want, want_lse = run_oracle(inp)
    return check(got, got_lse, want, want_lse, kw.get("out_dtype") or inp["out_dtype"], what)
