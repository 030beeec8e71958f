"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``pin_*`` function takes a loaded oracle library and raises
AssertionError when the oracle disagrees with something that does not come
from the oracle itself: hand-derived closed forms (tests/golden), library
routines (numpy / scipy softmax and logsumexp, numpy / torch dtype
conversions) and exact invariants of the merge.  They are collected by
tests/test_oracle_pins.py and, against oracle builds with planted mistakes,
by tests/test_oracle_mutants.py.

Definition pinned: page "[flashinfer] FlashInfer의 Context-Parallel Decode
최적화: Fused A2A + LSE Reduce", section "들어가며" (each rank's partial o_r
and lse_r over its KV shard) and section "코드 분석 / 1. Fused Kernel 구현"
(weights from lse, sum over the partial axis, divide by denom).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
from lse_weighted_merge_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "merge_hand_cases.json")
GOLDEN_STATE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                            "state_update_hand_cases.json")
GOLDEN_CP = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                         "cp_exchange_hand_cases.json")


def _num(x):
    if isinstance(x, str):
        return {"nan": math.nan, "-inf": -math.inf, "inf": math.inf}[x]
    return float(x)


def place(o_logical: np.ndarray, lse_logical: np.ndarray, layout: str, dtype: str):
    """Lay logical o [R,B,H,D] and lse [R,B,H] out densely in ``layout``."""
    R, B, H, D = o_logical.shape
    if layout == "bhrd":
        o = np.transpose(o_logical, (1, 2, 0, 3))
        lse = np.transpose(lse_logical, (1, 2, 0))
    else:
        o, lse = o_logical, lse_logical
    os_, ls_ = synth.strides(layout, R, B, H, D)
    o_packed = synth.pack(np.ascontiguousarray(o, dtype=np.float32).ravel(), dtype)
    return o_packed, np.ascontiguousarray(lse, dtype=np.float32).ravel(), os_, ls_


def run(lib, o_logical, lse_logical, layout="bhrd", dtype="f32"):
    R, B, H, D = o_logical.shape
    o, lse, os_, ls_ = place(o_logical, lse_logical, layout, dtype)
    return oracle.merge(o, lse, R, B, H, D, os_, ls_, synth.DTYPES[dtype], lib=lib)


def widened(o_logical, dtype):
    """The exact values the oracle should see after storage rounding (library cast)."""
    o32 = np.asarray(o_logical, dtype=np.float32)
    if dtype == "f16":
        return o32.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        import torch
        return torch.from_numpy(o32).to(torch.bfloat16).double().numpy()
    return o32.astype(np.float64)


# --------------------------------------------------------------------------- pins

def pin_decoders(lib):
    """fp16 / bf16 / fp32 widening equals numpy / torch conversions, bit for bit."""
    import torch
    bits = np.arange(65536, dtype=np.uint16)
    want16 = bits.view(np.float16).astype(np.float64)
    wantbf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got16 = np.array([lib.oracle_widen(int(b), oracle.F16) for b in bits])
    gotbf = np.array([lib.oracle_widen(int(b), oracle.BF16) for b in bits])
    for got, want in ((got16, want16), (gotbf, wantbf)):
        nan = np.isnan(want)
        assert np.array_equal(np.isnan(got), nan)
        assert np.array_equal(got[~nan], want[~nan])
    rng = np.random.Generator(np.random.PCG64(7))
    f = rng.standard_normal(1000, dtype=np.float32) * np.float32(1e3)
    got = np.array([lib.oracle_widen(int(b), oracle.F32) for b in f.view(np.uint32)])
    assert np.array_equal(got, f.astype(np.float64))


def pin_golden(lib):
    """Hand-derived closed forms in tests/golden/merge_hand_cases.json."""
    with open(GOLDEN) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        R, B, H, D = c["R"], c["B"], c["H"], c["D"]
        o = np.array([_num(x) for x in c["o"]], dtype=np.float32)
        lse = np.array([_num(x) for x in c["lse"]], dtype=np.float32)
        os_, ls_ = synth.strides(c["layout"], R, B, H, D)
        out, out_lse = oracle.merge(synth.pack(o, c["in_dtype"]), lse, R, B, H, D, os_, ls_,
                                    synth.DTYPES[c["in_dtype"]], lib=lib)
        want = np.array([_num(x) for x in c["out"]]).reshape(B, H, D)
        want_lse = np.array([_num(x) for x in c["out_lse"]]).reshape(B, H)
        tol = c["tol"]
        assert not np.isnan(out).any(), c["name"]
        assert np.all(np.abs(out - want) <= tol), (c["name"], out, want)
        fin = np.isfinite(want_lse)
        assert np.array_equal(np.isfinite(out_lse), fin), c["name"]
        assert np.array_equal(out_lse[~fin], want_lse[~fin]), c["name"]
        assert np.all(np.abs(out_lse[fin] - want_lse[fin]) <= tol), (c["name"], out_lse, want_lse)


def pin_r1_identity(lib):
    """R = 1: out is the partial itself and lse passes through, exactly."""
    rng = np.random.Generator(np.random.PCG64(11))
    for dtype in ("f32", "f16", "bf16"):
        for layout in ("bhrd", "rbhd"):
            o = rng.standard_normal((1, 3, 5, 7)).astype(np.float32) * 3
            lse = rng.uniform(-30, 30, (1, 3, 5)).astype(np.float32)
            out, out_lse = run(lib, o, lse, layout, dtype)
            assert np.array_equal(out, widened(o[0], dtype)), (dtype, layout)
            assert np.array_equal(out_lse, lse[0].astype(np.float64)), (dtype, layout)


def pin_equal_lse_mean(lib):
    """Equal lse in every shard: out is the arithmetic mean, lse = lse + ln R."""
    rng = np.random.Generator(np.random.PCG64(12))
    for R in (2, 3, 8, 16):
        for dtype in ("f32", "bf16"):
            o = rng.standard_normal((R, 2, 3, 16)).astype(np.float32)
            c = np.float32(rng.uniform(-10, 10))
            lse = np.full((R, 2, 3), c, dtype=np.float32)
            out, out_lse = run(lib, o, lse, "bhrd", dtype)
            want = np.mean(widened(o, dtype), axis=0)
            assert np.allclose(out, want, rtol=1e-14, atol=1e-14), (R, dtype)
            assert np.allclose(out_lse, float(c) + math.log(R), rtol=0, atol=1e-13), (R, dtype)


def pin_empty_shards_drop_out(lib):
    """Empty shards (lse = -inf, o poisoned with NaN) change nothing, and an
    all-empty row gives zeros and -inf."""
    rng = np.random.Generator(np.random.PCG64(13))
    R, B, H, D = 6, 3, 4, 8
    o = rng.standard_normal((R, B, H, D)).astype(np.float32)
    lse = rng.uniform(-4, 4, (R, B, H)).astype(np.float32)
    keep = rng.random((R, B, H)) > 0.4
    keep[0, 0, 0] = keep[1, 0, 1] = True
    keep[:, 2, 3] = False                       # one row fully empty
    o_p = o.copy()
    lse_p = lse.copy()
    for r, b, h in zip(*np.nonzero(~keep)):
        o_p[r, b, h, :] = np.nan
        lse_p[r, b, h] = -np.inf
    out, out_lse = run(lib, o_p, lse_p)
    assert not np.isnan(out).any()
    assert np.all(out[2, 3] == 0.0) and out_lse[2, 3] == -np.inf
    for b in range(B):
        for h in range(H):
            idx = np.nonzero(keep[:, b, h])[0]
            if len(idx) == 0:
                continue
            sub_o = o[idx, b:b + 1, h:h + 1, :]
            sub_l = lse[idx, b:b + 1, h:h + 1]
            want, want_lse = run(lib, sub_o, sub_l)
            assert np.allclose(out[b, h], want[0, 0], rtol=1e-14, atol=1e-14)
            assert abs(out_lse[b, h] - want_lse[0, 0]) <= 1e-13


def pin_shift_invariance(lib):
    """Adding c to every lse leaves out unchanged and shifts the merged lse by c."""
    rng = np.random.Generator(np.random.PCG64(14))
    o = rng.standard_normal((5, 2, 3, 12)).astype(np.float32)
    lse = (rng.integers(-256, 256, (5, 2, 3)) / 64.0).astype(np.float32)   # exact in fp32
    for c in (3.5, -17.25, 40.0):
        out0, lse0 = run(lib, o, lse)
        out1, lse1 = run(lib, o, lse + np.float32(c))
        assert np.allclose(out0, out1, rtol=1e-13, atol=1e-13), c
        assert np.allclose(lse1 - lse0, c, rtol=0, atol=1e-12), c


def pin_permutation_invariance(lib):
    """Reordering the shards leaves the result unchanged."""
    rng = np.random.Generator(np.random.PCG64(15))
    o = rng.standard_normal((7, 2, 2, 9)).astype(np.float32)
    lse = rng.uniform(-8, 8, (7, 2, 2)).astype(np.float32)
    out0, lse0 = run(lib, o, lse)
    for _ in range(3):
        p = rng.permutation(7)
        out1, lse1 = run(lib, o[p], lse[p])
        assert np.allclose(out0, out1, rtol=1e-13, atol=1e-13)
        assert np.allclose(lse0, lse1, rtol=0, atol=1e-13)


def pin_associativity(lib):
    """merge(merge(A), merge(B)) = merge(A u B): the online-softmax combine.
    The two intermediate results are fed back as fp32, so agreement is to fp32
    rounding of the intermediates."""
    rng = np.random.Generator(np.random.PCG64(16))
    R, B, H, D = 9, 2, 3, 10
    o = rng.standard_normal((R, B, H, D)).astype(np.float32)
    lse = rng.uniform(-6, 6, (R, B, H)).astype(np.float32)
    full, full_lse = run(lib, o, lse)
    for split in (1, 4, 8):
        a, a_lse = run(lib, o[:split], lse[:split])
        b, b_lse = run(lib, o[split:], lse[split:])
        o2 = np.stack([a, b]).astype(np.float32)
        l2 = np.stack([a_lse, b_lse]).astype(np.float32)
        two, two_lse = run(lib, o2, l2)
        assert np.allclose(two, full, rtol=0, atol=2e-6), split
        assert np.allclose(two_lse, full_lse, rtol=0, atol=2e-6), split


def _numpy_attention(q, k, v, scale):
    """Full softmax attention and its log-sum-exp from scipy's library routines."""
    from scipy.special import logsumexp, softmax
    s = (k @ q) * scale
    return softmax(s) @ v, float(logsumexp(s))


def pin_attention_shard(lib):
    """The oracle's shard attention equals scipy softmax attention on the same keys."""
    rng = np.random.Generator(np.random.PCG64(17))
    L, D = 16, 8
    q = rng.standard_normal(D)
    k = rng.standard_normal((L, D))
    v = rng.standard_normal((L, D))
    scale = 1 / math.sqrt(D)
    for lo, hi in ((0, 16), (0, 8), (8, 16), (3, 4), (5, 16)):
        o, lse = oracle.attention_shard(q, k, v, scale, lo, hi, lib=lib)
        want, want_lse = _numpy_attention(q, k[lo:hi], v[lo:hi], scale)
        assert np.allclose(o, want, rtol=1e-12, atol=1e-12), (lo, hi)
        assert abs(lse - want_lse) <= 1e-12, (lo, hi)
    o, lse = oracle.attention_shard(q, k, v, scale, 6, 6, lib=lib)
    assert lse == -math.inf and np.all(o == 0.0)


def pin_split_attention_identity(lib):
    """Partials of softmax attention over a KV sequence split into shards merge
    to full attention over the unsplit sequence (the reason the merge exists:
    context-parallel decode, the page's introduction).  Partials come from
    scipy, full attention from scipy; only the merge is the oracle's.  The
    partials pass through fp32 storage, hence the 1e-6 bound."""
    rng = np.random.Generator(np.random.PCG64(18))
    B, H, L, D = 3, 3, 16, 8
    scale = 1 / math.sqrt(D)
    for bounds in ((0, 8, 16), (0, 3, 16), (0, 0, 16), (0, 5, 11, 16), (0, 1, 2, 3, 16)):
        R = len(bounds) - 1
        o_parts = np.zeros((R, B, H, D))
        l_parts = np.full((R, B, H), -np.inf)
        full = np.zeros((B, H, D))
        full_lse = np.zeros((B, H))
        for b in range(B):
            for h in range(H):
                q = rng.standard_normal(D)
                k = rng.standard_normal((L, D))
                v = rng.standard_normal((L, D))
                full[b, h], full_lse[b, h] = _numpy_attention(q, k, v, scale)
                for r in range(R):
                    lo, hi = bounds[r], bounds[r + 1]
                    if hi > lo:
                        o_parts[r, b, h], l_parts[r, b, h] = _numpy_attention(
                            q, k[lo:hi], v[lo:hi], scale)
        for layout in ("bhrd", "rbhd"):
            out, out_lse = run(lib, o_parts.astype(np.float32), l_parts.astype(np.float32), layout)
            assert np.allclose(out, full, rtol=0, atol=1e-6), (bounds, layout)
            assert np.allclose(out_lse, full_lse, rtol=0, atol=1e-6), (bounds, layout)


def pin_layout_and_row_independence(lib):
    """The same logical partials give bit-identical results in every layout
    (dense [B,H,R,D], rank-major [R,B,H,D], padded strides), and each row's
    result depends on that row alone (B != H so a swapped index shows)."""
    rng = np.random.Generator(np.random.PCG64(19))
    R, B, H, D = 4, 2, 5, 6
    o = rng.standard_normal((R, B, H, D)).astype(np.float32)
    lse = rng.uniform(-5, 5, (R, B, H)).astype(np.float32)
    a, a_l = run(lib, o, lse, "bhrd")
    b_, b_l = run(lib, o, lse, "rbhd")
    assert np.array_equal(a, b_) and np.array_equal(a_l, b_l)
    # padded: o [B, H, R, D+3] and lse [H, B, R] (head-major), d stride 1
    pad = np.full((B, H, R, D + 3), np.nan, dtype=np.float32)
    pad[..., :D] = np.transpose(o, (1, 2, 0, 3))
    lhm = np.ascontiguousarray(np.transpose(lse, (2, 1, 0)))
    os_ = ((D + 3), H * R * (D + 3), R * (D + 3))
    ls_ = (1, R, B * R)
    c, c_l = oracle.merge(pad.ravel(), lhm.ravel(), R, B, H, D, os_, ls_, oracle.F32, lib=lib)
    assert np.array_equal(a, c) and np.array_equal(a_l, c_l)
    for bb in range(B):
        for hh in range(H):
            one, one_l = run(lib, o[:, bb:bb + 1, hh:hh + 1], lse[:, bb:bb + 1, hh:hh + 1])
            assert np.array_equal(one[0, 0], a[bb, hh]) and one_l[0, 0] == a_l[bb, hh]


def pin_extreme_spread(lib):
    """lse spread far beyond exp's range: no inf or NaN, result = dominant shard."""
    rng = np.random.Generator(np.random.PCG64(20))
    o = rng.standard_normal((3, 1, 2, 5)).astype(np.float32)
    lse = np.array([[[500.0, -800.0]], [[-900.0, 30.0]], [[-400.0, -900.0]]], dtype=np.float32)
    out, out_lse = run(lib, o, lse)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(out_lse))
    assert np.array_equal(out[0, 0], o[0, 0, 0].astype(np.float64))
    assert np.array_equal(out[0, 1], o[1, 0, 1].astype(np.float64))
    assert out_lse[0, 0] == 500.0 and out_lse[0, 1] == 30.0


def pin_state_golden(lib):
    """Hand-derived folds of one partial into an accumulator."""
    with open(GOLDEN_STATE) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        D = c["D"]
        acc = synth.pack(np.array([_num(x) for x in c["acc"]], np.float32), c["acc_dtype"])
        new = synth.pack(np.array([_num(x) for x in c["new"]], np.float32), c["new_dtype"])
        la = np.array([_num(c["lse_acc"])], np.float32)
        ln = np.array([_num(c["lse_new"])], np.float32)
        out, out_lse = oracle.state_update(acc, la, synth.DTYPES[c["acc_dtype"]], new, ln,
                                           synth.DTYPES[c["new_dtype"]], 1, 1, D, lib=lib)
        want = np.array([_num(x) for x in c["out"]])
        assert not np.isnan(out).any(), c["name"]
        assert np.all(np.abs(out[0, 0] - want) <= c["tol"]), (c["name"], out, want)
        wl = _num(c["out_lse"])
        if wl == -math.inf:
            assert out_lse[0, 0] == -math.inf, c["name"]
        else:
            assert abs(out_lse[0, 0] - wl) <= c["tol"], (c["name"], out_lse, wl)


def pin_state_chain_is_the_merge(lib):
    """Folding R shards one by one into an empty accumulator (fp32 in between)
    gives the R-way merge, by associativity of the combine; and one fold of
    same-dtype partials is the R = 2 merge exactly."""
    rng = np.random.Generator(np.random.PCG64(21))
    R, B, H, D = 6, 2, 3, 10
    o = rng.standard_normal((R, B, H, D)).astype(np.float32)
    lse = rng.uniform(-8, 8, (R, B, H)).astype(np.float32)
    lse[2, 1, 1] = -np.inf
    full, full_lse = run(lib, o, lse)
    acc = np.full((B, H, D), np.nan, np.float32)
    la = np.full((B, H), -np.inf, np.float32)
    for r in range(R):
        out, ol = oracle.state_update(acc.ravel(), la, oracle.F32, o[r].ravel(), lse[r], oracle.F32,
                                      B, H, D, lib=lib)
        acc, la = out.astype(np.float32), ol.astype(np.float32)
    assert np.allclose(acc, full, rtol=0, atol=2e-6)
    assert np.allclose(la, full_lse, rtol=0, atol=2e-6)
    two, two_lse = run(lib, o[:2], lse[:2])
    one, one_lse = oracle.state_update(o[0].ravel(), lse[0], oracle.F32, o[1].ravel(), lse[1],
                                       oracle.F32, B, H, D, lib=lib)
    assert np.array_equal(one, two) and np.array_equal(one_lse, two_lse)
    # strided new operand: the same data laid out with padded rows
    padded = np.zeros((B, H, D + 5), np.float32)
    padded[..., :D] = o[1]
    lhm = np.ascontiguousarray(lse[1].T)     # [H, B]
    alt, alt_lse = oracle.state_update(o[0].ravel(), lse[0], oracle.F32, padded.ravel(), lhm.ravel(),
                                       oracle.F32, B, H, D, new_strides=(H * (D + 5), D + 5),
                                       lse_new_strides=(1, B), lib=lib)
    assert np.array_equal(alt, one) and np.array_equal(alt_lse, one_lse)


def _nums(a):
    return np.vectorize(_num, otypes=[np.float64])(np.array(a, dtype=object))


def pin_cp_golden(lib):
    """Hand-derived exchange + merge results (head ownership by rank)."""
    with open(GOLDEN_CP) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        world, B, H, D = c["world"], c["B"], c["H"], c["D"]
        o = synth.pack(_nums(c["o"]).astype(np.float32).ravel(), c["dtype"])
        lse = _nums(c["lse"]).astype(np.float32).ravel()
        out, out_lse = oracle.cp_exchange_merge(o, lse, world, B, H, D, synth.DTYPES[c["dtype"]],
                                                lib=lib)
        want, want_lse = _nums(c["out"]), _nums(c["out_lse"])
        assert not np.isnan(out).any(), c["name"]
        assert np.all(np.abs(out - want) <= c["tol"]), (c["name"], out, want)
        fin = np.isfinite(want_lse)
        assert np.array_equal(np.isneginf(out_lse), np.isneginf(want_lse)), c["name"]
        assert np.all(np.abs(out_lse[fin] - want_lse[fin]) <= c["tol"]), (c["name"], out_lse)


def pin_cp_partitions_the_merge(lib):
    """The ranks' outputs, laid side by side along the head axis, are the
    world-way merge of all heads (each head merged once, by its owner); with
    one rank the exchange is the identity merge of that rank's partials; and
    reordering the senders changes no output."""
    rng = np.random.Generator(np.random.PCG64(33))
    for world, B, H, D, dt in ((4, 3, 8, 5, "bf16"), (2, 2, 6, 3, "f32"), (8, 1, 8, 4, "f16")):
        o = rng.standard_normal((world, B, H, D)).astype(np.float32)
        lse = rng.uniform(-6, 6, (world, B, H)).astype(np.float32)
        lse[world - 1, 0, H - 1] = -np.inf
        packed = synth.pack(o.ravel(), dt)
        out, out_lse = oracle.cp_exchange_merge(packed, lse, world, B, H, D, synth.DTYPES[dt],
                                                lib=lib)
        Hq = H // world
        full, full_lse = oracle.merge(packed, lse, world, B, H, D, (B * H * D, H * D, D),
                                      (B * H, H, 1), synth.DTYPES[dt], lib=lib)
        side = np.concatenate([out[q] for q in range(world)], axis=1)       # [B, H, D]
        side_lse = np.concatenate([out_lse[q] for q in range(world)], axis=1)
        assert np.array_equal(side, full) and np.array_equal(side_lse, full_lse), (world, dt)
        perm = rng.permutation(world)
        po = synth.pack(o[perm].ravel(), dt)
        pout, pout_lse = oracle.cp_exchange_merge(po, lse[perm], world, B, H, D,
                                                  synth.DTYPES[dt], lib=lib)
        assert np.allclose(pout, out, rtol=0, atol=1e-12) and np.allclose(pout_lse, out_lse,
                                                                          rtol=0, atol=1e-12)
        one, one_lse = oracle.cp_exchange_merge(synth.pack(o[0].ravel(), dt), lse[0], 1, B, H, D,
                                                synth.DTYPES[dt], lib=lib)
        assert np.array_equal(one[0], widened(o[0], dt))
        assert np.array_equal(one_lse[0], lse[0].astype(np.float64))


ALL_PINS = [
    pin_decoders, pin_golden, pin_r1_identity, pin_equal_lse_mean,
    pin_empty_shards_drop_out, pin_shift_invariance, pin_permutation_invariance,
    pin_associativity, pin_attention_shard, pin_split_attention_identity,
    pin_layout_and_row_independence, pin_extreme_spread, pin_state_golden,
    pin_state_chain_is_the_merge, pin_cp_golden, pin_cp_partitions_the_merge,
]
