"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Covers the five decode-merge workloads at full size in the launch
configuration the benchmark uses (AUTO), every kernel path, every dtype
pair, ragged and tiny shapes, empty shards and rows (with NaN planted in
empty partials), extreme lse spreads, misaligned pointers and strides, the
public torch-facing call in both layouts, determinism, non-default streams,
and 64-bit offsets past 2 GiB on sampled rows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TORCH_DT, check, parity, run_gpu, run_oracle
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import synth

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
ALL_DT = ("f32", "f16", "bf16")


@pytest.mark.parametrize("name", list(W))
def test_workload_full_size(name):
    inp = synth.make_inputs(W[name])
    stats = parity(inp, what=name)
    if name == "r4_b64_h32_d128_masked":
        assert stats["empty_rows"] > 0


@pytest.mark.parametrize("name", list(W))
@pytest.mark.parametrize("path", [nat.PATH_VECTOR, nat.PATH_SCALAR, nat.PATH_LATENCY,
                                  nat.PATH_STREAM, nat.PATH_WIDE])
def test_workload_every_path(name, path):
    w = W[name]
    # a reduced batch keeps the scalar path quick; the latency path is one CTA
    B = 1 if path == nat.PATH_LATENCY else min(w.B, 8)
    H = 1 if path == nat.PATH_LATENCY else w.H
    inp = synth.make_inputs(w, B=B, H=H, seed=w.seed + 17)
    parity(inp, path=path, what=f"{name}/{path}")


def test_empty_shards_poisoned_with_nan():
    w = W["r4_b64_h32_d128_masked"]
    for path in (nat.PATH_AUTO, nat.PATH_SCALAR, nat.PATH_VECTOR, nat.PATH_STREAM, nat.PATH_WIDE):
        inp = synth.make_inputs(w, poison_empty=True)
        o = inp["o"]
        assert (((o & 0x7f80) == 0x7f80) & ((o & 0x7f) != 0)).any()   # bf16 NaNs are planted
        stats = parity(inp, path=path, what=f"poisoned/{path}")
        assert stats["empty_rows"] > 0


@pytest.mark.parametrize("in_dt", ALL_DT)
@pytest.mark.parametrize("out_dt", ALL_DT)
def test_dtype_pairs(in_dt, out_dt):
    base = W["r8_b1_h8_d128"]
    inp = synth.make_inputs(base, in_dtype=in_dt, out_dtype=out_dt, B=3, H=7, R=5, D=96)
    for path in (nat.PATH_AUTO, nat.PATH_VECTOR, nat.PATH_SCALAR, nat.PATH_STREAM, nat.PATH_WIDE):
        parity(inp, path=path, what=f"{in_dt}->{out_dt}/{path}")


@pytest.mark.parametrize("R", [4, 8, 16])
@pytest.mark.parametrize("in_dt,out_dt", [("f16", "f32"), ("f32", "bf16"), ("bf16", "f16"),
                                          ("f32", "f32")])
@pytest.mark.parametrize("poison", [False, True], ids=["no_empty", "empty_nan"])
def test_stream_with_r_equal_to_its_partial_count(R, in_dt, out_dt, poison):
    """R = 4, 8 or 16 on the persistent kernel runs its R == RC instantiation
    (no partial-index checks).  Without empty shards every warp takes the
    fold loop with no per-partial test; with NaN-poisoned empty shards and
    all-empty rows the warps that hold one take the checked loop.  6144
    rows, more slices than the full persistent grid has lane groups, so
    lanes walk several slices; D=200 leaves lanes past the last column (the
    first loads of those read column 0 of their row instead)."""
    w = W["r4_b64_h32_d128_masked"]
    kw = dict(R=R, B=256, H=24, D=200, in_dtype=in_dt, out_dtype=out_dt, seed=R * 31 + len(in_dt))
    if not poison:
        kw.update(empty_shard_p=0.0, empty_row_p=0.0)
    inp = synth.make_inputs(w, poison_empty=poison, **kw)
    rc, plan = nat.plan_query(0x7f0000000000, 0x7f1000000000, R, 256, 24, 200,
                              (inp["o_strides"], inp["lse_strides"]), synth.DTYPES[in_dt],
                              synth.DTYPES[out_dt], 0x7f2000000000, 0x7f3000000000,
                              path=nat.PATH_STREAM)
    assert rc == nat.OK and plan["rc"] == R
    stats = parity(inp, path=nat.PATH_STREAM, what=f"R{R} {in_dt}->{out_dt} poison={poison}")
    if poison:
        assert stats["empty_rows"] > 0


@pytest.mark.parametrize("R", [1, 2, 3, 5, 8, 9, 16, 17, 33, 40, 64, 100, 257])
@pytest.mark.parametrize("D", [4, 8, 24, 64, 100, 128, 256, 264, 512, 1024])
def test_ragged_shapes(R, D):
    base = W["r2_b1_h2_d64"]
    inp = synth.make_inputs(base, R=R, D=D, B=3, H=5, lse_args=(-30.0, 30.0), seed=R * 1000 + D)
    parity(inp, what=f"R{R}/D{D}")
    parity(inp, path=nat.PATH_SCALAR, what=f"R{R}/D{D}/scalar")
    if D % 8 == 0:
        parity(inp, path=nat.PATH_VECTOR, what=f"R{R}/D{D}/vector")
        parity(inp, path=nat.PATH_WIDE, what=f"R{R}/D{D}/wide")
        if R <= 16:
            parity(inp, path=nat.PATH_STREAM, what=f"R{R}/D{D}/stream")


@pytest.mark.parametrize("layout", ["bhrd", "rbhd"])
def test_many_rows_ragged_tail(layout):
    # 3*37*... rows: grid tail not a multiple of the block, several CTAs per SM
    inp = synth.make_inputs(W["r2_b1_h2_d64"], R=6, B=37, H=41, D=192, layout=layout, seed=5)
    parity(inp, what=layout)
    parity(inp, path=nat.PATH_VECTOR, what=layout + "/vector")
    parity(inp, path=nat.PATH_STREAM, what=layout + "/stream")


@pytest.mark.parametrize("B,H", [(5, 1031), (1000, 3), (1, 65536)])
def test_row_index_arithmetic(B, H):
    # prime, small and power-of-two head counts: the row/head split of every group
    inp = synth.make_inputs(W["r2_b1_h2_d64"], R=3, B=B, H=H, D=256, seed=B + H)
    parity(inp, what=f"B{B}/H{H}")
    parity(inp, path=nat.PATH_STREAM, what=f"B{B}/H{H}/stream")


def test_r1_is_identity_on_gpu():
    inp = synth.make_inputs(W["r16_b512_h16_d512"], R=1, B=4, H=8, out_dtype="bf16")
    got, got_lse, _ = run_gpu(inp)
    # bf16 in -> bf16 out with weight exactly 1: the stored values come back unchanged
    src = torch.from_numpy(inp["o"].view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(got.ravel(), src)
    assert np.array_equal(got_lse.ravel(), inp["lse"].astype(np.float64))


def test_all_rows_empty():
    inp = synth.make_inputs(W["r8_b256_h64_d128_rankmajor"], B=2, H=3)
    inp["lse"][:] = -np.inf
    for path in (nat.PATH_AUTO, nat.PATH_VECTOR, nat.PATH_SCALAR, nat.PATH_STREAM, nat.PATH_WIDE):
        got, got_lse, _ = run_gpu(inp, path)
        assert np.all(got == 0.0) and not np.signbit(got).any()
        assert np.all(got_lse == -np.inf)


@pytest.mark.parametrize("spread", [(-20.0, 20.0), (-200.0, 200.0), (-1000.0, 1000.0)])
def test_extreme_lse_spread(spread):
    inp = synth.make_inputs(W["r16_b512_h16_d512"], B=4, H=16, lse_args=spread, lse_kind="uniform")
    parity(inp, what=str(spread))


def test_misaligned_pointer_and_strides():
    w = W["r8_b1_h8_d128"]
    inp = synth.make_inputs(w, B=2, H=8)
    # partial_o starting 2 bytes past a 16-byte boundary: scalar path
    parity(inp, o_offset_elems=1, what="offset")
    rc, plan = nat.plan_query(0x7f0000000002, 0x7f1000000000, 8, 2, 8, 128,
                              (inp["o_strides"], inp["lse_strides"]), nat.BF16, nat.BF16,
                              0x7f2000000000, 0x7f3000000000)
    assert plan["path"] == nat.PATH_SCALAR
    # padded rows of D+1 elements (odd stride)
    R, B, H, D = 4, 3, 5, 33
    rng = np.random.Generator(np.random.PCG64(3))
    vals = rng.standard_normal((B, H, R, D + 1), dtype=np.float32)
    lse = rng.uniform(-3, 3, (B, H, R)).astype(np.float32)
    inp2 = {"o": synth.pack(vals.ravel(), "f16"), "lse": lse.ravel(),
            "o_strides": (D + 1, H * R * (D + 1), R * (D + 1)), "lse_strides": (1, H * R, R),
            "R": R, "B": B, "H": H, "D": D, "in_dtype": "f16", "out_dtype": "f32"}
    parity(inp2, what="odd-stride")


def test_public_merge_both_layouts():
    from lse_weighted_merge_b200 import merge
    inp = synth.make_inputs(W["r8_b256_h64_d128_rankmajor"], B=4, H=8)
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    o_rbhd = torch.from_numpy(inp["o"].view(np.int16)).view(torch.float16).reshape(R, B, H, D).cuda()
    l_rbhd = torch.from_numpy(inp["lse"]).reshape(R, B, H).cuda()
    want, want_lse = run_oracle(inp)
    out, out_lse = merge(o_rbhd, l_rbhd, layout="rbhd")
    check(out.double().cpu().numpy(), out_lse.double().cpu().numpy(), want, want_lse, "f16", "rbhd")
    # the same data as a [B,H,R,D] view (non-contiguous) and as a dense copy
    o_view, l_view = o_rbhd.permute(1, 2, 0, 3), l_rbhd.permute(1, 2, 0)
    for o_t, l_t in ((o_view, l_view), (o_view.contiguous(), l_view.contiguous())):
        out, out_lse = merge(o_t, l_t, layout="bhrd", out_dtype=torch.float32)
        check(out.double().cpu().numpy(), out_lse.double().cpu().numpy(), want, want_lse, "f32", "bhrd")
    with pytest.raises(ValueError):
        merge(o_rbhd.cpu(), l_rbhd.cpu(), layout="rbhd")


@pytest.mark.parametrize("R,D", [(4, 128), (37, 72)], ids=["R4", "R37-long-form"])
def test_outputs_written_exactly_in_bounds(R, D):
    inp = synth.make_inputs(W["r4_b64_h32_d128_masked"], B=3, H=5, R=R, D=D)
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    d_o = torch.from_numpy(inp["o"].view(np.int16)).cuda()
    d_l = torch.from_numpy(inp["lse"]).cuda()
    pad = 4096
    for path in (nat.PATH_AUTO, nat.PATH_VECTOR, nat.PATH_SCALAR, nat.PATH_STREAM, nat.PATH_WIDE):
        canvas = torch.full((pad + B * H * D + pad,), 12345, dtype=torch.int16, device="cuda")
        lcanvas = torch.full((pad + B * H + pad,), 7.0, dtype=torch.float32, device="cuda")
        nat.merge_raw(d_o.data_ptr(), d_l.data_ptr(), R, B, H, D, (inp["o_strides"], inp["lse_strides"]),
                      nat.BF16, nat.BF16, canvas.data_ptr() + pad * 2, lcanvas.data_ptr() + pad * 4,
                      torch.cuda.current_stream().cuda_stream, path)
        torch.cuda.synchronize()
        c = canvas.cpu()
        lc = lcanvas.cpu()
        assert torch.all(c[:pad] == 12345) and torch.all(c[pad + B * H * D:] == 12345)
        assert torch.all(lc[:pad] == 7.0) and torch.all(lc[pad + B * H:] == 7.0)


def test_deterministic_and_stream_ordered():
    inp = synth.make_inputs(W["r16_b512_h16_d512"], B=16)
    a, al, _ = run_gpu(inp)
    s = torch.cuda.Stream()
    b, bl, _ = run_gpu(inp, stream=s)
    assert np.array_equal(a, b) and np.array_equal(al, bl)
    # every vector-family path computes the same sums in the same order
    for path in (nat.PATH_VECTOR, nat.PATH_STREAM):
        c, cl, _ = run_gpu(inp, path)
        assert np.array_equal(a, c) and np.array_equal(al, cl)


def test_split_attention_tiny_check():
    """Partials of real softmax attention over a KV sequence of 16 split into
    shards merge, on the GPU, to attention over the unsplit sequence (fp64
    oracle attention; fp32 partials and fp32 output)."""
    B, H, L, D = 1, 2, 16, 64
    q, k, v = synth.make_attention_qkv(1000, B * H, L, D)
    scale = 1.0 / math.sqrt(D)
    for bounds in ((0, 8, 16), (0, 3, 16), (0, 0, 16), (0, 4, 9, 13, 16)):
        R = len(bounds) - 1
        o = np.zeros((B, H, R, D), np.float32)
        lse = np.zeros((B, H, R), np.float32)
        full = np.zeros((B, H, D))
        full_lse = np.zeros((B, H))
        for row in range(B * H):
            b, h = divmod(row, H)
            full[b, h], full_lse[b, h] = oracle.attention_shard(q[row], k[row], v[row], scale, 0, L)
            for r in range(R):
                po, pl = oracle.attention_shard(q[row], k[row], v[row], scale, bounds[r], bounds[r + 1])
                o[b, h, r], lse[b, h, r] = po, pl
        inp = {"o": o.ravel(), "lse": lse.ravel(), "R": R, "B": B, "H": H, "D": D,
               "o_strides": synth.strides("bhrd", R, B, H, D)[0],
               "lse_strides": synth.strides("bhrd", R, B, H, D)[1], "in_dtype": "f32",
               "out_dtype": "f32"}
        for path in (nat.PATH_AUTO, nat.PATH_SCALAR):
            got, got_lse, _ = run_gpu(inp, path)
            check(got, got_lse, full, full_lse, "f32", f"attention {bounds}")


def test_offsets_beyond_2gib_sampled_rows():
    """A merge whose partial_o spans > 2 GiB (64-bit offsets), checked on
    sampled rows that the oracle computes one by one."""
    R, B, H, D = 16, 1100, 64, 1024          # 2.2 GiB of bf16 partials
    gen = torch.Generator(device="cuda").manual_seed(99)
    o = torch.randn((B, H, R, D), generator=gen, device="cuda").to(torch.bfloat16)
    lse = (torch.rand((B, H, R), generator=gen, device="cuda") * 24 - 12)
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    out_lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    nat.merge_raw(o.data_ptr(), lse.data_ptr(), R, B, H, D, None, nat.BF16, nat.BF16,
                  out.data_ptr(), out_lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    rng = np.random.Generator(np.random.PCG64(1))
    rows = list(rng.integers(0, B * H, 48)) + [0, B * H - 1]
    for row in rows:
        b, h = divmod(int(row), H)
        o_row = o[b, h].contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()
        l_row = lse[b, h].cpu().numpy()
        want, want_lse = oracle.merge(o_row, l_row, R, 1, 1, D, (D, 0, 0), (1, 0, 0), oracle.BF16)
        got = out[b, h].double().cpu().numpy().reshape(1, 1, D)
        got_lse = out_lse[b, h].double().cpu().numpy().reshape(1, 1)
        check(got, got_lse, want, want_lse, "bf16", f"row {row}")
    del o
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["r8_b256_h64_d128_rankmajor", "r4_b64_h32_d128_masked"])
@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_merge_host_pipelined(name, chunks):
    """Host tensors in, host tensors out, copies overlapped with the merge in
    batch slices: the result matches the oracle and the single device call
    within tolerance (a slice may take another kernel path than the whole
    batch, e.g. WIDE for a few rows, and sum in another order)."""
    from lse_weighted_merge_b200 import merge, merge_host
    w = W[name]
    inp = synth.make_inputs(w, B=min(w.B, 24))
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    tdt = TORCH_DT[inp["in_dtype"]]
    shape_o = (B, H, R, D) if w.layout == "bhrd" else (R, B, H, D)
    shape_l = shape_o[:3]
    h_o = torch.from_numpy(inp["o"].view(np.int16)).view(tdt).reshape(shape_o).pin_memory()
    h_l = torch.from_numpy(inp["lse"]).reshape(shape_l).pin_memory()
    out, out_lse = merge_host(h_o, h_l, layout=w.layout, chunks=chunks)
    assert not out.is_cuda and out.shape == (B, H, D)
    dev_out, dev_lse = merge(h_o.cuda(), h_l.cuda(), layout=w.layout)
    torch.cuda.synchronize()
    want, want_lse = run_oracle(inp)
    check(dev_out.double().cpu().numpy(), dev_lse.double().cpu().numpy(), want, want_lse,
          inp["out_dtype"], name + "/device")
    check(out.double().numpy(), out_lse.double().numpy(), want, want_lse, inp["out_dtype"], name)


@pytest.mark.parametrize("layout", ["bhrd", "rbhd"])
def test_merge_host_pipelined_calls_in_a_row(layout):
    """Consecutive pipelined calls (each call's uploads start before the
    previous call's copies back end), a default call and a call with another
    chunk count among them, each with its own inputs and host outputs: after
    one synchronisation every result matches the oracle."""
    from lse_weighted_merge_b200 import merge_host
    w = W["r4_b64_h32_d128_masked"]
    plan = [(8, True), (8, True), (8, False), (8, True), (3, True), (3, True)]
    results = []
    for k, (chunks, pipe) in enumerate(plan):
        inp = synth.make_inputs(w, seed=700 + k, poison_empty=True, layout=layout)
        R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
        shape_o = (B, H, R, D) if layout == "bhrd" else (R, B, H, D)
        h_o = torch.from_numpy(inp["o"].view(np.int16)).view(torch.bfloat16).reshape(shape_o).pin_memory()
        h_l = torch.from_numpy(inp["lse"]).reshape(shape_o[:3]).pin_memory()
        out, out_lse = merge_host(h_o, h_l, layout=layout, chunks=chunks, sync=False, pipeline=pipe)
        results.append((inp, out, out_lse, h_o, h_l))
    torch.cuda.synchronize()
    for k, (inp, out, out_lse, _, _) in enumerate(results):
        want, want_lse = run_oracle(inp)
        check(out.double().numpy(), out_lse.double().numpy(), want, want_lse, inp["out_dtype"],
              f"call {k} {plan[k]}")


@pytest.mark.parametrize("R,B,H,D,want", [(64, 1, 8, 128, nat.PATH_WIDE), (128, 4, 8, 512, nat.PATH_WIDE),
                                          (48, 2, 3, 64, nat.PATH_WIDE), (64, 64, 32, 128, nat.PATH_WIDE),
                                          (24, 128, 32, 128, nat.PATH_STREAM)])
def test_many_partials_auto_path(R, B, H, D, want):
    """Large R (many KV splits) against the oracle, with empty shards holding
    NaN and all-empty rows among the inputs: a few rows take the wide path,
    many rows the persistent kernel's long form."""
    w = W["r4_b64_h32_d128_masked"]
    inp = synth.make_inputs(w, R=R, B=B, H=H, D=D, seed=R + B, poison_empty=True)
    parity(inp, what=f"auto R{R}")
    rc, plan = nat.plan_query(0x7f0000000000, 0x7f1000000000, R, B, H, D,
                              (inp["o_strides"], inp["lse_strides"]), nat.BF16, nat.BF16,
                              0x7f2000000000, 0x7f3000000000)
    assert plan["path"] == want


@pytest.mark.parametrize("R,D,layout,in_dt,out_dt", [
    (17, 128, "bhrd", "bf16", "bf16"),    # one chunk of 16 and a ragged one of 1
    (32, 512, "bhrd", "bf16", "f32"),     # two slices per row, two full chunks
    (33, 64, "rbhd", "f16", "f16"),       # chunks of 8 (8 columns a row), rank-major
    (100, 8, "bhrd", "f32", "bf16"),      # chunks of 4 (two fp32 columns a row: 4 lanes)
    (257, 256, "rbhd", "bf16", "bf16"),   # many chunks
    (24, 1000, "bhrd", "f16", "f32"),     # ragged last slice of a long row
])
def test_long_form_of_the_persistent_kernel(R, D, layout, in_dt, out_dt):
    """R > 16 on the persistent kernel (chunks with a running max): every
    dtype pair and both layouts against the oracle, with empty shards holding
    NaN and all-empty rows; the same inputs forced through the wide path
    agree too."""
    w = W["r4_b64_h32_d128_masked"]
    inp = synth.make_inputs(w, R=R, B=12, H=16, D=D, layout=layout, in_dtype=in_dt,
                            out_dtype=out_dt, seed=R * 7 + D, poison_empty=True)
    parity(inp, nat.PATH_STREAM, what=f"long R{R} D{D} {layout} {in_dt}->{out_dt}")
    parity(inp, nat.PATH_WIDE, what=f"wide R{R} D{D} {layout} {in_dt}->{out_dt}")


def test_host_context_through_the_c_abi():
    """lse_merge_host on a context of its own: a call whose staging needs
    exceed the context's area is refused before anything is enqueued; a
    call that fits merges host partials into host outputs, matching the
    oracle; the context is destroyed after its last call."""
    w = W["r4_b64_h32_d128_masked"]
    inp = synth.make_inputs(w, B=16, seed=31, poison_empty=True)
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    h_o = torch.from_numpy(inp["o"].view(np.int16)).pin_memory()
    h_l = torch.from_numpy(inp["lse"]).pin_memory()
    out = torch.full((B, H, D), float("nan"), dtype=torch.bfloat16).pin_memory()
    out_lse = torch.full((B, H), float("nan"), dtype=torch.float32).pin_memory()
    need = nat.host_stage_bytes(R, B, H, D, nat.BF16, nat.BF16)
    small = nat.host_create(need - 256)
    try:
        rc = nat.host_merge_raw(small, h_o.data_ptr(), h_l.data_ptr(), R, B, H, D, nat.LAYOUT_BHRD,
                                nat.BF16, nat.BF16, out.data_ptr(), out_lse.data_ptr(), 4,
                                check=False)
        assert rc == nat.ESCRATCH
    finally:
        nat.host_destroy(small)
    ctx = nat.host_create(need)
    try:
        s = torch.cuda.current_stream()
        nat.host_merge_raw(ctx, h_o.data_ptr(), h_l.data_ptr(), R, B, H, D, nat.LAYOUT_BHRD,
                           nat.BF16, nat.BF16, out.data_ptr(), out_lse.data_ptr(), 5,
                           stream=s.cuda_stream)
        s.synchronize()
    finally:
        nat.host_destroy(ctx)
    want, want_lse = run_oracle(inp)
    check(out.double().numpy(), out_lse.double().numpy(), want, want_lse, "bf16", "host context")
