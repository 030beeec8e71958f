"""Seeded synthetic inputs for the LSE-weighted merge.

This module only draws random numbers and packs them into the storage layout
(fp32 -> bf16/fp16 by round-to-nearest-even).  It holds none of the merge's
arithmetic, so both the CUDA path's tests/bench and the CPU oracle can be fed
from it.

The workloads follow the shapes of context-parallel decode: R partials (one
per KV shard) of B*H rows of head dimension D, with a log-sum-exp per partial
row.  Shapes and value distributions are listed in ``WORKLOADS``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

DTYPES = {"f32": 0, "f16": 1, "bf16": 2}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    R: int
    B: int
    H: int
    D: int
    in_dtype: str
    out_dtype: str
    layout: str          # "bhrd": o [B,H,R,D], lse [B,H,R];  "rbhd": o [R,B,H,D], lse [R,B,H]
    o_sigma: float       # partial_o ~ N(0, o_sigma^2)
    lse_kind: str        # "uniform" (a, b) | "normal" (mean, std)
    lse_args: tuple
    seed: int
    empty_shard_p: float = 0.0   # P(lse_r = -inf) per (b, h, r)
    empty_row_p: float = 0.0     # P(all shards of a row are -inf) per (b, h)
    note: str = field(default="", compare=False)

    @property
    def rows(self) -> int:
        return self.B * self.H

    def bytes_read(self) -> int:
        """Algorithmic bytes read: every partial element and every lse once."""
        return self.R * self.B * self.H * (self.D * ELEM_BYTES[self.in_dtype] + 4)

    def bytes_written(self) -> int:
        """Algorithmic bytes written: every output element and merged lse once."""
        return self.B * self.H * (self.D * ELEM_BYTES[self.out_dtype] + 4)

    def bytes_total(self) -> int:
        return self.bytes_read() + self.bytes_written()


# The five decode-merge workloads.  Names say what they are.
WORKLOADS = {
    w.name: w for w in [
        Workload("r2_b1_h2_d64", 2, 1, 2, 64, "bf16", "bf16", "bhrd", 1.0,
                 "uniform", (-5.0, 5.0), 1000,
                 note="tiny decode merge; also carries the split-attention check"),
        Workload("r8_b1_h8_d128", 8, 1, 8, 128, "bf16", "bf16", "bhrd", 1.0,
                 "uniform", (0.0, 12.0), 1001,
                 note="single-token decode latency shape"),
        Workload("r4_b64_h32_d128_masked", 4, 64, 32, 128, "bf16", "bf16", "bhrd", 1.0,
                 "normal", (6.0, 3.0), 1002, empty_shard_p=0.10, empty_row_p=0.01,
                 note="10% empty shards, 1% fully empty rows"),
        Workload("r8_b256_h64_d128_rankmajor", 8, 256, 64, 128, "f16", "f16", "rbhd", 0.5,
                 "uniform", (-20.0, 20.0), 1003,
                 note="rank-major (strided) partials"),
        Workload("r16_b512_h16_d512", 16, 512, 16, 512, "bf16", "f32", "bhrd", 1.0,
                 "normal", (8.0, 4.0), 1004,
                 note="large bandwidth-bound merge, fp32 output"),
    ]
}

# Context-parallel exchange + merge: R = world ranks, layout "rbhd" = rank s's
# local partials [B, H, D] in block s.  The first two are the shapes of the
# CP-decode page's result table (batch 1, heads 2, dim 64; batch 1, heads 8,
# dim 128; the page states no world size, so 2 and 8 ranks are chosen).
CP_WORKLOADS = {
    w.name: w for w in [
        Workload("cp_w2_b1_h2_d64", 2, 1, 2, 64, "bf16", "bf16", "rbhd", 1.0,
                 "uniform", (-5.0, 5.0), 1100, note="CP decode, 2 ranks, one head each"),
        Workload("cp_w8_b1_h8_d128", 8, 1, 8, 128, "bf16", "bf16", "rbhd", 1.0,
                 "uniform", (0.0, 12.0), 1101, note="CP decode, 8 ranks, one head each"),
        Workload("cp_w8_b64_h32_d128_masked", 8, 64, 32, 128, "bf16", "bf16", "rbhd", 1.0,
                 "normal", (6.0, 3.0), 1102, empty_shard_p=0.10, empty_row_p=0.01,
                 note="CP decode, 8 ranks, batch 64, 10% empty shards, 1% empty rows"),
        Workload("cp_w8_b256_h64_d128", 8, 256, 64, 128, "bf16", "bf16", "rbhd", 1.0,
                 "normal", (6.0, 3.0), 1103,
                 note="CP decode, 8 ranks, batch 256: a bandwidth-bound exchange"),
    ]
}

SMALL = "r2_b1_h2_d64"
LARGE = "r16_b512_h16_d512"


def strides(layout: str, R: int, B: int, H: int, D: int):
    """(r, b, h) element strides of partial_o and partial_lse for a dense layout."""
    if layout == "bhrd":
        return (D, H * R * D, R * D), (1, H * R, R)
    if layout == "rbhd":
        return (B * H * D, H * D, D), (B * H, H, 1)
    raise ValueError(f"unknown layout {layout!r}")


def pack(values_f32: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to the storage dtype (round-to-nearest-even).

    Returns float32 for "f32" and the uint16 bit patterns for "f16"/"bf16".
    """
    values_f32 = np.ascontiguousarray(values_f32, dtype=np.float32)
    if dtype == "f32":
        return values_f32
    if dtype == "f16":
        return values_f32.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch  # torch's fp32 -> bf16 cast rounds to nearest even
        t = torch.from_numpy(values_f32).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16)
    raise ValueError(f"unknown dtype {dtype!r}")


def draw_lse(rng: np.random.Generator, w: Workload, n: int) -> np.ndarray:
    if w.lse_kind == "uniform":
        a, b = w.lse_args
        return rng.uniform(a, b, size=n).astype(np.float32)
    if w.lse_kind == "normal":
        mu, sd = w.lse_args
        return (mu + sd * rng.standard_normal(n, dtype=np.float32)).astype(np.float32)
    raise ValueError(w.lse_kind)


def make_inputs(w: Workload, seed: int | None = None, poison_empty: bool = False,
                **overrides) -> dict:
    """Draw one seeded batch of partials for workload ``w``.

    Returns a dict with the packed partial_o (flat), partial_lse (flat fp32),
    their (r, b, h) strides and the sizes.  With ``poison_empty`` the partial
    rows of empty shards are filled with NaN, to show that they are not read.
    ``overrides`` replace Workload fields (e.g. R=3, D=96) for edge cases.
    """
    if overrides:
        w = Workload(**{**w.__dict__, **overrides})
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    R, B, H, D = w.R, w.B, w.H, w.D
    o_str, l_str = strides(w.layout, R, B, H, D)
    n_o = R * B * H * D
    o = rng.standard_normal(n_o, dtype=np.float32)
    if w.o_sigma != 1.0:
        o *= np.float32(w.o_sigma)
    lse = draw_lse(rng, w, R * B * H)
    if w.empty_shard_p > 0 or w.empty_row_p > 0:
        shard_mask = rng.random(R * B * H) < w.empty_shard_p
        row_mask = rng.random(B * H) < w.empty_row_p
        # lse index of (r, b, h) in this layout
        r_i, b_i, h_i = np.meshgrid(np.arange(R), np.arange(B), np.arange(H), indexing="ij")
        l_idx = (r_i * l_str[0] + b_i * l_str[1] + h_i * l_str[2]).ravel()
        row_of = (b_i * H + h_i).ravel()
        empty = np.zeros(R * B * H, dtype=bool)
        empty[l_idx] = shard_mask | row_mask[row_of]
        lse[empty] = -np.inf
        if poison_empty:
            o_rows = (r_i * o_str[0] + b_i * o_str[1] + h_i * o_str[2]).ravel()
            for start in o_rows[empty[l_idx]]:
                o[start:start + D] = np.nan
    return {
        "workload": w,
        "o": pack(o, w.in_dtype),
        "lse": lse,
        "o_strides": o_str,
        "lse_strides": l_str,
        "R": R, "B": B, "H": H, "D": D,
        "in_dtype": w.in_dtype, "out_dtype": w.out_dtype,
    }


def make_attention_qkv(seed: int, rows: int, L: int, D: int):
    """Q [rows, D], K and V [rows, L, D], fp32 N(0, 1), for the split-attention check."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((rows, D), dtype=np.float32)
    k = rng.standard_normal((rows, L, D), dtype=np.float32)
    v = rng.standard_normal((rows, L, D), dtype=np.float32)
    return q, k, v
