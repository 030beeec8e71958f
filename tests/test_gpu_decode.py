"""Split-KV decode attention (the producer of the partials) on the GPU vs the
fp64 oracle attention: the fused kernel in both forms (the workspace form,
whose last split merges, and the cluster form), the unfused partials, their
merge, ragged and empty sequences, grouped heads, strided caches, dtypes.

Tolerance of the attention outputs (derived from the arithmetic, not from a
run): the exponentiated scores P enter the P.V tensor-core product rounded
to the input type (relative 2^-9 for bf16, 2^-11 for fp16) while the
normaliser keeps them in fp32, so a row's output can move by at most
2^-9 * max_j |v_j| (bf16) over its keys; the output type's rounding adds
2^-9 |o| (bf16) or 2^-11 |o| (fp16).  The lse comes from fp32-accumulated
scores: bounded here by 2e-4 absolute (D * 2^-24 * sum_d |q_d k_d| * scale
stays below 6e-5 for these N(0,1) inputs, and tensor-core accumulation may
round differently from IEEE order).  Empty sequences and splits: exactly 0
and -inf.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from lse_weighted_merge_b200 import _native as nat

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}
P_ULP = {"bf16": 2.0 ** -9, "f16": 2.0 ** -11}
OUT_ULP = {"bf16": 2.0 ** -9, "f16": 2.0 ** -11, "f32": 2.0 ** -23}
LSE_TOL = 2e-4


def make(B, Hq, Hkv, L, D, dtype="bf16", seed=0, layout="bhld"):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, D), generator=g).to(TDT[dtype])
    if layout == "bhld":
        k = torch.randn((B, Hkv, L, D), generator=g).to(TDT[dtype])
        v = torch.randn((B, Hkv, L, D), generator=g).to(TDT[dtype])
    else:   # [B, L, Hkv, D] storage viewed as [B, Hkv, L, D]
        k = torch.randn((B, L, Hkv, D), generator=g).to(TDT[dtype]).permute(0, 2, 1, 3)
        v = torch.randn((B, L, Hkv, D), generator=g).to(TDT[dtype]).permute(0, 2, 1, 3)
    return q, k, v


def reference(q, k, v, scale, lens, rows=None, bounds=None):
    """fp64 oracle attention per (b, h) row over keys [lo, hi) (default [0, len_b))."""
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    qd = q.double().numpy()
    rows = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hq)]
    out, lse, vmax = {}, {}, {}
    cache = {}
    for b, h in rows:
        hk = h // G
        if (b, hk) not in cache:
            cache[(b, hk)] = (k[b, hk].double().numpy(), v[b, hk].double().numpy())
        kk, vv = cache[(b, hk)]
        lo, hi = bounds(b) if bounds else (0, int(lens[b]))
        o, l = oracle.attention_shard(qd[b, h], kk, vv, scale, lo, hi)
        out[(b, h)], lse[(b, h)] = o, l
        vmax[(b, h)] = float(np.abs(vv[lo:hi]).max()) if hi > lo else 0.0
    return out, lse, vmax


def check_rows(got, got_lse, want, want_lse, vmax, in_dt, out_dt, what):
    worst = 0.0
    for key, o in want.items():
        b, h = key
        g = got[b, h].double().cpu().numpy()
        gl = float(got_lse[b, h])
        assert not np.isnan(g).any() and not math.isnan(gl), (what, key)
        if want_lse[key] == -math.inf:
            assert np.all(g == 0.0) and gl == -math.inf, (what, key, gl)
            continue
        bound = P_ULP[in_dt] * vmax[key] + OUT_ULP[out_dt] * np.abs(o) + 1e-6
        err = np.abs(g - o)
        assert np.all(err <= bound), (what, key, float((err / bound).max()))
        assert abs(gl - want_lse[key]) <= LSE_TOL, (what, key, gl, want_lse[key])
        worst = max(worst, float((err / bound).max()))
    return worst


def workspace(B, Hq, Hkv, R, D):
    """A zeroed workspace of the fused workspace form."""
    return torch.zeros(nat.decode_workspace_bytes(B, Hq, Hkv, R, D), dtype=torch.uint8, device="cuda")


def counters_are_zero(ws, B, Hkv):
    return bool((ws[:B * Hkv * 4].view(torch.int32) == 0).all())


def run(q, k, v, R, scale, kv_len=None, fused=True, out_dt="bf16", mode="ws", ws=None):
    """One call of the C ABI: fused (mode "ws": lse_merge_decode_attention_ws,
    with `ws` or a fresh zeroed workspace; mode "cluster":
    lse_merge_decode_attention) or the partials (fused=False)."""
    B, Hq, D = q.shape
    _, Hkv, L, _ = k.shape
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    st = (qd.stride(0), qd.stride(1), kd.stride(0), kd.stride(1), kd.stride(2),
          vd.stride(0), vd.stride(1), vd.stride(2))
    klen = torch.tensor(kv_len, dtype=torch.int32, device="cuda") if kv_len is not None else None
    dt = nat.BF16 if q.dtype == torch.bfloat16 else nat.F16
    s = torch.cuda.current_stream().cuda_stream
    if fused:
        out = torch.empty((B, Hq, D), dtype=TDT[out_dt], device="cuda")
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        wkw = {}
        if mode == "ws":
            ws = workspace(B, Hq, Hkv, R, D) if ws is None else ws
            wkw = dict(workspace=ws.data_ptr(), workspace_bytes=ws.numel())
        nat.decode_raw(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                       klen.data_ptr() if klen is not None else 0, B, Hq, Hkv, L, D, R, scale,
                       st, dt, out.data_ptr(), lse.data_ptr(), s, fused=True,
                       out_dtype={"bf16": nat.BF16, "f16": nat.F16, "f32": nat.F32}[out_dt], **wkw)
        torch.cuda.synchronize()
        if mode == "ws":   # the call leaves its counters at 0, ready for the next one
            assert counters_are_zero(ws, B, Hkv)
        return out.cpu(), lse.cpu()
    po = torch.empty((B, Hq, R, D), dtype=torch.float32, device="cuda")
    pl = torch.empty((B, Hq, R), dtype=torch.float32, device="cuda")
    nat.decode_raw(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                   klen.data_ptr() if klen is not None else 0, B, Hq, Hkv, L, D, R, scale, st,
                   dt, po.data_ptr(), pl.data_ptr(), s, fused=False)
    torch.cuda.synchronize()
    return po.cpu(), pl.cpu()


SHAPES = [  # B, Hq, Hkv, L, D, R
    (1, 2, 1, 16, 64, 2),       # the tiny decode merge: 16 keys in two shards
    (2, 8, 2, 300, 128, 4),     # ragged last tile, group of 4
    (3, 4, 4, 1000, 64, 8),     # one query head per KV head
    (1, 16, 1, 97, 128, 2),     # a full 16-row group
    (2, 6, 3, 33, 64, 1),       # one split
    (2, 12, 4, 5, 128, 8),      # fewer keys than splits: empty splits
]


@pytest.mark.parametrize("mode", ["ws", "cluster"])
@pytest.mark.parametrize("B,Hq,Hkv,L,D,R", SHAPES)
def test_fused_attention_matches_oracle(B, Hq, Hkv, L, D, R, mode):
    q, k, v = make(B, Hq, Hkv, L, D, seed=L + R)
    scale = 1 / math.sqrt(D)
    out, lse = run(q, k, v, R, scale, mode=mode)
    want, want_lse, vmax = reference(q, k, v, scale, [L] * B)
    check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", f"fused {mode}")


@pytest.mark.parametrize("B,Hq,Hkv,L,D,R", [
    (2, 8, 2, 300, 128, 3),     # a split count the cluster form does not take
    (1, 4, 1, 2000, 64, 16),
    (1, 8, 8, 4096, 128, 64),   # many splits of one sequence
    (2, 4, 2, 10, 128, 32),     # more splits than keys: most splits empty
])
def test_workspace_form_takes_any_split_count(B, Hq, Hkv, L, D, R):
    q, k, v = make(B, Hq, Hkv, L, D, seed=3 * L + R)
    scale = 1 / math.sqrt(D)
    out, lse = run(q, k, v, R, scale, mode="ws")
    want, want_lse, vmax = reference(q, k, v, scale, [L] * B)
    check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", f"ws R={R}")


def test_workspace_reused_by_consecutive_calls():
    """Three calls in a row share one workspace (zeroed once): each call's
    last split resets its counters, so the next call merges its own
    partials and nothing of the previous call leaks in."""
    B, Hq, Hkv, L, D, R = 3, 8, 2, 700, 128, 4
    ws = workspace(B, Hq, Hkv, R, D)
    scale = 1 / math.sqrt(D)
    for call in range(3):
        q, k, v = make(B, Hq, Hkv, L, D, seed=100 + call)
        out, lse = run(q, k, v, R, scale, mode="ws", ws=ws)
        want, want_lse, vmax = reference(q, k, v, scale, [L] * B)
        check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", f"call {call}")


@pytest.mark.parametrize("B,Hq,Hkv,L,D,R", SHAPES)
def test_partials_are_the_split_attentions(B, Hq, Hkv, L, D, R):
    q, k, v = make(B, Hq, Hkv, L, D, seed=2 * L + R)
    scale = 1 / math.sqrt(D)
    po, pl = run(q, k, v, R, scale, fused=False)
    per = (L + R - 1) // R
    for r in range(R):
        lo, hi = min(L, r * per), min(L, r * per + per)
        want, want_lse, vmax = reference(q, k, v, scale, [L] * B, bounds=lambda b: (lo, hi))
        check_rows(po[:, :, r], pl[:, :, r], want, want_lse, vmax, "bf16", "f32", f"split {r}")


def test_partials_merged_equal_fused():
    from lse_weighted_merge_b200 import merge
    B, Hq, Hkv, L, D, R = 2, 8, 2, 777, 128, 4
    q, k, v = make(B, Hq, Hkv, L, D, seed=9)
    scale = 0.1
    po, pl = run(q, k, v, R, scale, fused=False)
    mo, ml = merge(po.cuda(), pl.cuda(), out_dtype=torch.float32)
    for mode in ("ws", "cluster"):
        fo, fl = run(q, k, v, R, scale, fused=True, out_dt="f32", mode=mode)
        torch.cuda.synchronize()
        # all merge the same fp32 partials; only the summation order differs
        assert torch.allclose(mo.cpu(), fo, rtol=0, atol=1e-5), mode
        assert torch.allclose(ml.cpu(), fl, rtol=0, atol=1e-5), mode


def test_ragged_and_empty_sequences():
    B, Hq, Hkv, L, D, R = 5, 8, 2, 200, 64, 4
    lens = [200, 0, 3, 131, 64]
    q, k, v = make(B, Hq, Hkv, L, D, seed=11)
    scale = 1 / math.sqrt(D)
    want, want_lse, vmax = reference(q, k, v, scale, lens)
    for fused in (True, "cluster", False):
        if fused:
            out, lse = run(q, k, v, R, scale, kv_len=lens, mode="cluster" if fused == "cluster" else "ws")
        else:
            from lse_weighted_merge_b200 import merge
            po, pl = run(q, k, v, R, scale, kv_len=lens, fused=False)
            out, lse = merge(po.cuda(), pl.cuda(), out_dtype=torch.bfloat16)
            out, lse = out.cpu(), lse.cpu()
        check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", f"lens fused={fused}")
        assert torch.all(out[1] == 0) and torch.all(lse[1] == -math.inf)


@pytest.mark.parametrize("D", [64, 128])
def test_many_units_ragged_lengths(D):
    """Many (batch, KV head, split) units, several waves of CTAs, with ragged
    lengths (empty, shorter than a tile, shorter than the split count) that
    change the tile counts from unit to unit.  Every row is checked, fused
    and unfused."""
    from lse_weighted_merge_b200 import merge
    B, Hq, Hkv, L, R = 96, 8, 2, 150, 8   # 1536 units
    rng = np.random.Generator(np.random.PCG64(21 + D))
    lens = [int(x) for x in rng.integers(0, L + 1, B)]
    lens[:4] = [0, 1, 7, L]
    q, k, v = make(B, Hq, Hkv, L, D, seed=23 + D)
    scale = 1 / math.sqrt(D)
    want, want_lse, vmax = reference(q, k, v, scale, lens)
    out, lse = run(q, k, v, R, scale, kv_len=lens, mode="ws")
    check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", "many units ws")
    po, pl = run(q, k, v, R, scale, kv_len=lens, fused=False)
    mo, ml = merge(po.cuda(), pl.cuda(), out_dtype=torch.bfloat16)
    check_rows(mo.cpu(), ml.cpu(), want, want_lse, vmax, "bf16", "bf16", "many units partials")


@pytest.mark.parametrize("mode", ["ws", "cluster"])
@pytest.mark.parametrize("out_dt", ["bf16", "f16", "f32"])
def test_fp16_inputs_and_out_dtypes(out_dt, mode):
    B, Hq, Hkv, L, D, R = 2, 8, 4, 257, 128, 2
    q, k, v = make(B, Hq, Hkv, L, D, dtype="f16", seed=13)
    scale = 1 / math.sqrt(D)
    out, lse = run(q, k, v, R, scale, out_dt=out_dt, mode=mode)
    want, want_lse, vmax = reference(q, k, v, scale, [L] * B)
    check_rows(out, lse, want, want_lse, vmax, "f16", out_dt, "f16")


def test_strided_cache_layout():
    B, Hq, Hkv, L, D, R = 2, 8, 2, 150, 128, 4
    q, k, v = make(B, Hq, Hkv, L, D, seed=15, layout="blhd")
    assert not k.is_contiguous()
    scale = 1 / math.sqrt(D)
    out, lse = run(q, k, v, R, scale)
    want, want_lse, vmax = reference(q, k, v, scale, [L] * B)
    check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", "strided")


def test_large_decode_sampled_rows():
    B, Hq, Hkv, L, D, R = 16, 32, 8, 4096, 128, 4
    g = torch.Generator(device="cuda").manual_seed(17)
    q = torch.randn((B, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, Hkv, L, D), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, Hkv, L, D), generator=g, device="cuda").to(torch.bfloat16)
    scale = 1 / math.sqrt(D)
    from lse_weighted_merge_b200 import decode_attention
    out, lse = decode_attention(q, k, v, splits=R, fused=True)
    out2, lse2 = decode_attention(q, k, v, splits=R, fused=False)
    out3, lse3 = decode_attention(q, k, v, splits=R, fused="cluster")
    torch.cuda.synchronize()
    rng = np.random.Generator(np.random.PCG64(5))
    rows = [(int(b), int(h)) for b, h in zip(rng.integers(0, B, 24), rng.integers(0, Hq, 24))]
    want, want_lse, vmax = reference(q.cpu(), k.cpu(), v.cpu(), scale, [L] * B, rows=rows)
    check_rows(out.cpu(), lse.cpu(), want, want_lse, vmax, "bf16", "bf16", "large fused")
    check_rows(out2.cpu(), lse2.cpu(), want, want_lse, vmax, "bf16", "bf16", "large unfused")
    check_rows(out3.cpu(), lse3.cpu(), want, want_lse, vmax, "bf16", "bf16", "large cluster")


@pytest.mark.parametrize("fused", [True, "cluster"], ids=["ws", "cluster"])
def test_graph_capture_of_fused_attention(fused):
    B, Hq, Hkv, L, D, R = 2, 8, 2, 512, 128, 8
    q, k, v = make(B, Hq, Hkv, L, D, seed=19)
    from lse_weighted_merge_b200 import decode_attention
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    eager, eager_lse = decode_attention(qd, kd, vd, splits=R, fused=fused)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # the capture stream's workspace is made before capture
        decode_attention(qd, kd, vd, splits=R, fused=fused)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        o, l = decode_attention(qd, kd, vd, splits=R, fused=fused)
    for _ in range(3):   # replays reuse the workspace: each leaves its counters at 0
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, eager) and torch.equal(l, eager_lse)
    del g


@pytest.mark.parametrize("B,Hq,Hkv,L", [(1, 8, 1, 8192), (1, 32, 8, 4096), (3, 16, 4, 1500)])
def test_automatic_splits_and_fusion(B, Hq, Hkv, L):
    """decode_attention with its default split count and fused/unfused choice."""
    from lse_weighted_merge_b200 import decode_attention
    D = 128
    q, k, v = make(B, Hq, Hkv, L, D, seed=B * L)
    out, lse = decode_attention(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    want, want_lse, vmax = reference(q, k, v, 1 / math.sqrt(D), [L] * B)
    check_rows(out.cpu(), lse.cpu(), want, want_lse, vmax, "bf16", "bf16", "auto")


@pytest.mark.parametrize("B", [2, 80])
@pytest.mark.parametrize("fused", [True, "ws", False], ids=["cluster", "ws", "partials"])
def test_outputs_written_exactly_in_bounds(fused, B):
    """Outputs (and the workspace) carved out of larger buffers with canary
    guard bytes: after a call no guard byte has changed and q, k, v are left
    as they were.  B=80 gives 640 units, more CTAs than the device holds
    at once."""
    Hq, Hkv, L, D, R = 8, 2, 300, 128, 4
    q, k, v = make(B, Hq, Hkv, L, D, seed=77)
    scale = 1 / math.sqrt(D)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    q0, k0, v0 = qd.clone(), kd.clone(), vd.clone()
    G, canary = 4096, 0x3C
    o_bytes = B * Hq * D * 2 if fused else B * Hq * R * D * 4
    l_bytes = B * Hq * 4 if fused else B * Hq * R * 4
    o_buf = torch.full((G + o_bytes + G,), canary, dtype=torch.uint8, device="cuda")
    l_buf = torch.full((G + l_bytes + G,), canary, dtype=torch.uint8, device="cuda")
    w_bytes = nat.decode_workspace_bytes(B, Hq, Hkv, R, D)
    w_buf = torch.full((G + w_bytes + G,), canary, dtype=torch.uint8, device="cuda")
    w_buf[G:G + w_bytes].zero_()
    wkw = dict(workspace=w_buf.data_ptr() + G, workspace_bytes=w_bytes) if fused == "ws" else {}
    st = (qd.stride(0), qd.stride(1), kd.stride(0), kd.stride(1), kd.stride(2),
          vd.stride(0), vd.stride(1), vd.stride(2))
    nat.decode_raw(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), 0, B, Hq, Hkv, L, D, R, scale, st,
                   nat.BF16, o_buf.data_ptr() + G, l_buf.data_ptr() + G,
                   torch.cuda.current_stream().cuda_stream, fused=bool(fused),
                   **({"out_dtype": nat.BF16} if fused else {}), **wkw)
    torch.cuda.synchronize()
    for buf, n in ((o_buf, o_bytes), (l_buf, l_bytes), (w_buf, w_bytes)):
        assert bool((buf[:G] == canary).all()) and bool((buf[G + n:] == canary).all())
    assert torch.equal(qd, q0) and torch.equal(kd, k0) and torch.equal(vd, v0)
    if fused:
        out = o_buf[G:G + o_bytes].view(torch.bfloat16).view(B, Hq, D).cpu()
        lse = l_buf[G:G + l_bytes].view(torch.float32).view(B, Hq).cpu()
        want, want_lse, vmax = reference(q, k, v, scale, [L] * B)
        check_rows(out, lse, want, want_lse, vmax, "bf16", "bf16", "guarded fused")
