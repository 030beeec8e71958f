"""In-place state update (fold one partial into an accumulator) on the GPU vs
the fp64 oracle, through the C ABI: every dtype pair, the 16-byte and the
element paths, empty sides holding NaN, strided inputs, and a chain of folds
that must equal the R-way merge."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import OUT_TOL, TORCH_DT, check
from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import synth

pytestmark = pytest.mark.gpu
ALL_DT = ("f32", "f16", "bf16")


def make(B, H, D, acc_dt, new_dt, seed, la=(-6, 6), ln=(-6, 6)):
    rng = np.random.Generator(np.random.PCG64(seed))
    acc = synth.pack(rng.standard_normal(B * H * D, dtype=np.float32), acc_dt)
    new = synth.pack(rng.standard_normal(B * H * D, dtype=np.float32), new_dt)
    lse_a = rng.uniform(*la, B * H).astype(np.float32)
    lse_n = rng.uniform(*ln, B * H).astype(np.float32)
    return acc, lse_a, new, lse_n


def dev(a, dt=None):
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    return t.cuda()


def run(acc, lse_a, new, lse_n, B, H, D, acc_dt, new_dt, strides=None):
    d_acc, d_la, d_new, d_ln = dev(acc), dev(lse_a), dev(new), dev(lse_n)
    nat.state_update_raw(d_acc.data_ptr(), d_la.data_ptr(), d_new.data_ptr(), d_ln.data_ptr(),
                         B, H, D, strides, synth.DTYPES[acc_dt], synth.DTYPES[new_dt],
                         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    got = d_acc.view(TORCH_DT[acc_dt]).double().cpu().numpy().reshape(B, H, D)
    return got, d_la.double().cpu().numpy().reshape(B, H)


@pytest.mark.parametrize("acc_dt", ALL_DT)
@pytest.mark.parametrize("new_dt", ALL_DT)
@pytest.mark.parametrize("D", [96, 100])        # 16-byte path / element path
def test_state_update_dtype_pairs(acc_dt, new_dt, D):
    B, H = 5, 7
    acc, la, new, ln = make(B, H, D, acc_dt, new_dt, seed=D)
    la[3] = -np.inf                              # an empty accumulator row
    ln[4] = -np.inf                              # an empty new row
    la[5] = ln[5] = -np.inf                      # both empty
    want, want_lse = oracle.state_update(acc, la, synth.DTYPES[acc_dt], new, ln,
                                         synth.DTYPES[new_dt], B, H, D)
    got, got_lse = run(acc, la, new, ln, B, H, D, acc_dt, new_dt)
    check(got, got_lse, want, want_lse, acc_dt, f"{acc_dt}<-{new_dt} D{D}")


@pytest.mark.parametrize("acc_dt,new_dt", [("f32", "bf16"), ("bf16", "f16"), ("f16", "f32")])
@pytest.mark.parametrize("D", [264, 300, 512, 520, 1000])
def test_state_update_long_rows(acc_dt, new_dt, D):
    """Rows of more than 32 chunks of 8, which one group of 32 lanes folds
    in two or more passes (D = 264 ... 1000), the last pass ragged for most;
    300 and 1000 take the element path."""
    B, H = 3, 5
    acc, la, new, ln = make(B, H, D, acc_dt, new_dt, seed=D + 7)
    la[2] = -np.inf
    ln[6] = -np.inf
    want, want_lse = oracle.state_update(acc, la, synth.DTYPES[acc_dt], new, ln,
                                         synth.DTYPES[new_dt], B, H, D)
    got, got_lse = run(acc, la, new, ln, B, H, D, acc_dt, new_dt)
    check(got, got_lse, want, want_lse, acc_dt, f"{acc_dt}<-{new_dt} D{D}")


def test_empty_sides_are_not_read():
    B, H, D = 3, 4, 64
    acc, la, new, ln = make(B, H, D, "bf16", "bf16", seed=1)
    nan_acc = np.full_like(acc, 0x7fc0)          # bf16 NaN everywhere
    la[:] = -np.inf
    got, got_lse = run(nan_acc, la, new, ln, B, H, D, "bf16", "bf16")
    src = torch.from_numpy(new.view(np.int16)).view(torch.bfloat16).double().numpy().reshape(B, H, D)
    assert np.array_equal(got, src) and np.array_equal(got_lse, ln.reshape(B, H).astype(np.float64))
    acc, la, new, ln = make(B, H, D, "f32", "f16", seed=2)
    nan_new = np.full_like(new, 0x7e00)          # f16 NaN everywhere
    ln[:] = -np.inf
    got, got_lse = run(acc, la, nan_new, ln, B, H, D, "f32", "f16")
    assert np.array_equal(got, acc.reshape(B, H, D).astype(np.float64))
    assert np.array_equal(got_lse, la.reshape(B, H).astype(np.float64))


def test_strided_new_operand():
    B, H, D = 4, 6, 128
    rng = np.random.Generator(np.random.PCG64(3))
    acc, la, _, _ = make(B, H, D, "f32", "bf16", seed=4)
    padded = synth.pack(rng.standard_normal(B * H * (D + 8), dtype=np.float32), "bf16")
    lse_hm = rng.uniform(-5, 5, H * B).astype(np.float32)       # [H, B]
    strides = (H * (D + 8), D + 8, 1, B)
    want, want_lse = oracle.state_update(acc, la, oracle.F32, padded, lse_hm, oracle.BF16, B, H, D,
                                         new_strides=strides[:2], lse_new_strides=strides[2:])
    got, got_lse = run(acc, la, padded, lse_hm, B, H, D, "f32", "bf16", strides)
    check(got, got_lse, want, want_lse, "f32", "strided")


def test_chain_of_folds_is_the_merge():
    """Folding 16 partials one by one into an empty fp32 accumulator equals
    the 16-way merge (GPU lse_merge and the oracle), within fp32 rounding."""
    w = synth.WORKLOADS["r16_b512_h16_d512"]
    inp = synth.make_inputs(w, B=8)
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    o = torch.from_numpy(inp["o"].view(np.int16)).view(torch.bfloat16).reshape(B, H, R, D).cuda()
    lse = torch.from_numpy(inp["lse"]).reshape(B, H, R).cuda()
    acc = torch.full((B, H, D), float("nan"), dtype=torch.float32, device="cuda")
    la = torch.full((B, H), float("-inf"), dtype=torch.float32, device="cuda")
    from lse_weighted_merge_b200 import merge, merge_state_
    for r in range(R):
        merge_state_(acc, la, o[:, :, r], lse[:, :, r])
    full, full_lse = merge(o, lse, out_dtype=torch.float32)
    torch.cuda.synchronize()
    want, want_lse = oracle.merge(inp["o"], inp["lse"], R, B, H, D, inp["o_strides"],
                                  inp["lse_strides"], oracle.BF16)
    check(acc.double().cpu().numpy(), la.double().cpu().numpy(), want, want_lse, "f32", "chain")
    assert torch.allclose(acc, full, rtol=0, atol=2e-5 * (1 + full.abs().max().item()))


def test_large_state_update_full_parity():
    B, H, D = 512, 16, 512
    acc, la, new, ln = make(B, H, D, "f32", "bf16", seed=5, la=(0, 16), ln=(0, 16))
    want, want_lse = oracle.state_update(acc, la, oracle.F32, new, ln, oracle.BF16, B, H, D)
    got, got_lse = run(acc, la, new, ln, B, H, D, "f32", "bf16")
    check(got, got_lse, want, want_lse, "f32", "large")


@pytest.mark.parametrize("acc_dt,D", [("f32", 96), ("bf16", 100), ("f16", 8), ("f32", 300),
                                      ("bf16", 512), ("f32", 1000)])
def test_writes_stay_inside_the_accumulator(acc_dt, D):
    """The accumulator and its lse are carved out of larger buffers whose
    guard bytes hold a canary pattern: after a fold no guard byte has
    changed, and the new partial and its lse are left as they were."""
    B, H, G = 5, 3, 4096
    acc, la, new, ln = make(B, H, D, acc_dt, "bf16", seed=D)
    want, want_lse = oracle.state_update(acc, la, synth.DTYPES[acc_dt], new, ln, synth.DTYPES["bf16"],
                                         B, H, D)
    raw = torch.from_numpy(acc.view(np.uint8).copy())
    canary = 0x5A
    a_buf = torch.full((G + raw.numel() + G,), canary, dtype=torch.uint8)
    a_buf[G:G + raw.numel()] = raw
    l_raw = torch.from_numpy(la.view(np.uint8).copy())
    l_buf = torch.full((G + l_raw.numel() + G,), canary, dtype=torch.uint8)
    l_buf[G:G + l_raw.numel()] = l_raw
    a_buf, l_buf = a_buf.cuda(), l_buf.cuda()
    d_new, d_ln = dev(new), dev(ln)
    new0, ln0 = d_new.clone(), d_ln.clone()
    nat.state_update_raw(a_buf.data_ptr() + G, l_buf.data_ptr() + G, d_new.data_ptr(), d_ln.data_ptr(),
                         B, H, D, None, synth.DTYPES[acc_dt], synth.DTYPES["bf16"],
                         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    n = raw.numel()
    assert bool((a_buf[:G] == canary).all()) and bool((a_buf[G + n:] == canary).all())
    assert bool((l_buf[:G] == canary).all()) and bool((l_buf[G + l_raw.numel():] == canary).all())
    assert torch.equal(d_new, new0) and torch.equal(d_ln, ln0)
    got = a_buf[G:G + n].view(TORCH_DT[acc_dt]).double().cpu().numpy().reshape(B, H, D)
    got_lse = l_buf[G:G + l_raw.numel()].view(torch.float32).double().cpu().numpy().reshape(B, H)
    check(got, got_lse, want, want_lse, acc_dt, f"guarded {acc_dt} D{D}")
