"""The C-ABI library on the host: it loads, exports every declared symbol, and
its argument validation and launch planning behave as documented.  Nothing
here launches a kernel; rejected calls return before any CUDA call, and the
planner only inspects pointer values, never dereferences them."""
import ctypes
import os
import re
import subprocess

import pytest

from lse_weighted_merge_b200 import _native as nat
from lse_weighted_merge_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lse_merge.h")

# Fake, suitably aligned device addresses far apart (never dereferenced).
PO, PL, OUT, OUTL = 0x7f0000000000, 0x7f1000000000, 0x7f2000000000, 0x7f3000000000


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(lse_merge\w*)\s*\(", text, re.M)))


def test_header_and_binding_agree():
    assert sorted(nat.EXPORTS) == declared_functions()


def test_every_declared_symbol_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", nat.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(nat.lib, name)


def test_version_and_strerror():
    assert nat.lib.lse_merge_version() == nat.ABI_VERSION == 4
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10, -11):
        assert nat.strerror(code) and "unknown lse_merge error" not in nat.strerror(code)
    assert "unknown lse_merge error" in nat.strerror(-99)


def q(R=2, B=1, H=2, D=64, strides=None, i=nat.BF16, o=nat.BF16, po=PO, pl=PL, out=OUT,
      outl=OUTL, path=nat.PATH_AUTO):
    return nat.plan_query(po, pl, R, B, H, D, strides, i, o, out, outl, path)


@pytest.mark.parametrize("kw,code", [
    (dict(i=3), nat.EDTYPE), (dict(o=-1), nat.EDTYPE),
    (dict(R=0), nat.EDIMS), (dict(B=0), nat.EDIMS), (dict(H=-1), nat.EDIMS), (dict(D=0), nat.EDIMS),
    (dict(po=0), nat.ENULL), (dict(pl=0), nat.ENULL), (dict(out=0), nat.ENULL), (dict(outl=0), nat.ENULL),
    (dict(strides=((-64, 128, 64), (1, 2, 1))), nat.ESTRIDE),
    (dict(strides=((64, 128, 64), (1, -2, 1))), nat.ESTRIDE),
    (dict(po=PO + 1), nat.EALIGN), (dict(pl=PL + 2), nat.EALIGN), (dict(outl=OUTL + 1), nat.EALIGN),
    (dict(i=nat.F32, po=PO + 2), nat.EALIGN), (dict(out=OUT + 1), nat.EALIGN),
    (dict(out=PO + 64), nat.EALIAS), (dict(outl=PL), nat.EALIAS), (dict(outl=OUT + 8), nat.EALIAS),
    (dict(out=PL), nat.EALIAS),
    (dict(path=7), nat.EPATH),
    (dict(D=60, path=nat.PATH_WIDE), nat.EPATH),
    (dict(D=60, path=nat.PATH_STREAM), nat.EPATH),
    (dict(B=64, H=64, path=nat.PATH_LATENCY), nat.EPATH),
    (dict(B=1, H=32, path=nat.PATH_LATENCY), nat.EPATH),     # 128 threads > one 64-thread CTA
    (dict(D=60, path=nat.PATH_VECTOR), nat.EPATH),
    (dict(po=PO + 2, path=nat.PATH_VECTOR), nat.EPATH),
    (dict(R=2 ** 30, B=2 ** 30, H=2 ** 30, D=2 ** 30), nat.EDIMS),
])
def test_validation(kw, code):
    rc, plan = q(**kw)
    assert rc == code, (kw, rc, nat.strerror(rc))
    assert plan is None


def test_rejected_calls_return_before_any_cuda_call():
    # Argument errors come back from lse_merge itself, with nothing enqueued.
    assert nat.merge_raw(0, PL, 2, 1, 2, 64, None, nat.BF16, nat.BF16, OUT, OUTL, check=False) == nat.ENULL
    assert nat.merge_raw(PO, PL, 0, 1, 2, 64, None, nat.BF16, nat.BF16, OUT, OUTL, check=False) == nat.EDIMS
    assert nat.merge_raw(PO, PL, 2, 1, 2, 64, None, 9, nat.BF16, OUT, OUTL, check=False) == nat.EDTYPE
    assert nat.merge_raw(PO, PL, 2, 1, 2, 64, None, nat.BF16, nat.BF16, PO, OUTL, check=False) == nat.EALIAS
    with pytest.raises(nat.LseMergeError) as ei:
        nat.merge_raw(PO, PL, 2, 1, 2, 64, None, nat.BF16, nat.BF16, PO, OUTL)
    assert ei.value.code == nat.EALIAS
    assert nat.lib.lse_merge(None, None, 1, 1, 1, 1, None, 0, 0, None, None, None) == nat.ENULL


def test_plans_of_the_five_workloads():
    blk = 64
    expect = {  # name -> (path, lanes, rc, nv, slices, block, grid); STREAM grids are sized at launch
        "r2_b1_h2_d64": (nat.PATH_LATENCY, 8, 4, 1, 1, 32, 1),
        "r8_b1_h8_d128": (nat.PATH_WIDE, 16, 4, 1, 1, 32, 8),
        "r4_b64_h32_d128_masked": (nat.PATH_VECTOR, 8, 4, 2, 1, blk, 64 * 32 * 8 // blk),
        "r8_b256_h64_d128_rankmajor": (nat.PATH_STREAM, 8, 8, 2, 1, blk, 0),
        "r16_b512_h16_d512": (nat.PATH_STREAM, 32, 16, 1, 2, blk, 0),
    }
    for name, w in synth.WORKLOADS.items():
        st = synth.strides(w.layout, w.R, w.B, w.H, w.D)
        rc, plan = nat.plan_query(PO, PL, w.R, w.B, w.H, w.D, st, synth.DTYPES[w.in_dtype],
                                  synth.DTYPES[w.out_dtype], OUT, OUTL)
        assert rc == 0, name
        got = (plan["path"], plan["lanes"], plan["rc"], plan["nv"], plan["slices_per_row"],
               plan["block"], plan["grid"])
        assert got == expect[name], (name, got)
        assert plan["vec"] == 8 and plan["rc"] * plan["nv"] <= 16
        assert plan["groups"] == w.B * w.H * plan["slices_per_row"]
        if plan["path"] == nat.PATH_WIDE:
            continue
        # every 16-byte column of a row is owned by exactly one lane slot
        dv = w.D // 8
        assert plan["slices_per_row"] * plan["lanes"] * plan["nv"] >= dv
        assert (plan["slices_per_row"] - 1) * plan["lanes"] * plan["nv"] < dv


def test_fallback_to_scalar_and_forced_paths():
    # D not a multiple of 8 bf16 elements -> scalar; misaligned stride -> scalar
    assert q(D=60)[1]["path"] == nat.PATH_SCALAR
    assert q(strides=((65, 130, 65), (1, 2, 1)), D=64)[1]["path"] == nat.PATH_SCALAR
    assert q(po=PO + 2)[1]["path"] == nat.PATH_SCALAR
    # f32 output of a bf16 row needs 16-byte alignment of out (8 elements = 32 B)
    assert q(o=nat.F32, out=OUT + 8)[1]["path"] == nat.PATH_SCALAR
    # f32 input: 4 elements per vector; bf16 out then needs 8-byte alignment
    assert q(i=nat.F32, D=12)[1]["vec"] == 4
    assert q(i=nat.F32, o=nat.BF16, out=OUT + 8)[1]["path"] == nat.PATH_LATENCY
    for path in (nat.PATH_VECTOR, nat.PATH_LATENCY, nat.PATH_SCALAR, nat.PATH_STREAM,
                 nat.PATH_WIDE):
        rc, plan = q(path=path)
        assert rc == 0 and plan["path"] == path
    rc, plan = q(B=64, H=64, R=16, path=nat.PATH_STREAM)
    assert rc == 0 and plan["grid"] == 0 and plan["rc"] == 16
    rc, plan = q(B=64, H=64, path=nat.PATH_SCALAR)
    assert plan["grid"] == 64 * 64 * 32 // plan["block"] and plan["lanes"] == 32


@pytest.mark.parametrize("R,want_rc,want_nv,want_lanes,want_path", [
    (1, 4, 2, 4, nat.PATH_VECTOR), (3, 4, 2, 4, nat.PATH_VECTOR), (5, 8, 1, 8, nat.PATH_VECTOR),
    (9, 16, 1, 16, nat.PATH_VECTOR), (16, 16, 1, 16, nat.PATH_STREAM),   # 16 x 0.5 MB = 8 MB
    (17, 8, 1, 8, nat.PATH_WIDE), (33, 8, 1, 8, nat.PATH_WIDE),            # 4096 rows x 8 lanes:
    (100, 8, 1, 8, nat.PATH_WIDE)])                                        # too few for the long form
def test_rc_nv_and_lanes_follow_R(R, want_rc, want_nv, want_lanes, want_path):
    rc, plan = q(R=R, D=64, B=64, H=64)      # 8 vectors per row, beyond one CTA, < 8 MB
    assert rc == 0 and (plan["rc"], plan["nv"], plan["lanes"], plan["path"]) == \
        (want_rc, want_nv, want_lanes, want_path)


@pytest.mark.parametrize("R,D,lanes,rc,slices,block", [
    (64, 8, 4, 4, 1, 64), (64, 64, 8, 8, 1, 64), (64, 128, 16, 16, 1, 64), (64, 512, 32, 16, 2, 128),
    (64, 1000, 32, 16, 4, 128), (32, 128, 16, 16, 1, 32), (17, 64, 8, 8, 1, 32),
    (257, 512, 32, 16, 2, 128), (40, 128, 16, 16, 1, 64), (20, 128, 16, 16, 1, 32)])
def test_wide_plan(R, D, lanes, rc, slices, block):
    rc_, plan = q(R=R, D=D, B=3, H=5, path=nat.PATH_WIDE)
    assert rc_ == 0
    assert (plan["lanes"], plan["rc"], plan["slices_per_row"], plan["block"]) == (lanes, rc, slices, block)
    assert plan["grid"] == plan["groups"] == 15 * slices


def test_latency_path_keeps_one_column_per_lane():
    rc, plan = q(R=2, D=64, B=1, H=2)
    assert plan["path"] == nat.PATH_LATENCY and plan["nv"] == 1 and plan["lanes"] == 8
    assert plan["block"] == 32 and plan["grid"] == 1


def test_path_choice_by_size():
    # a few rows: each spread over a CTA
    assert q(R=8, B=2, H=8, D=128)[1]["path"] == nat.PATH_WIDE
    # under one wave of work (< 8 MB of partials): one-shot VECTOR
    assert q(R=4, B=64, H=32, D=128)[1]["path"] == nat.PATH_VECTOR
    # 8 MB .. 256 MB: persistent STREAM
    assert q(R=8, B=64, H=64, D=128, o=nat.F32)[1]["path"] == nat.PATH_STREAM


def test_stream_from_its_size_threshold_up():
    # 16 partials of 512 bf16 in 1100 batches x 16 heads = 288 MB of partials: still STREAM
    big = q(R=16, B=1100, H=16, D=512, o=nat.F32, out=0x7fa000000000, outl=0x7fb000000000)[1]
    assert big["path"] == nat.PATH_STREAM and big["grid"] == 0
    small = q(R=16, B=512, H=16, D=512, o=nat.F32)[1]
    assert small["path"] == nat.PATH_STREAM and small["grid"] == 0
    # R > 16 over many rows: the persistent kernel in chunks of partials; over a
    # few rows (<= 128 slices): the partials of a row spread over one CTA (WIDE)
    long = q(R=17, B=64, H=128)[1]                 # 8192 rows x 8 lanes (D=64): the long form
    assert long["path"] == nat.PATH_STREAM and long["rc"] == 8 and long["nv"] == 1
    assert q(R=17, B=64, H=64)[1]["path"] == nat.PATH_WIDE   # 4096 x 8 lanes: WIDE
    assert q(R=24, B=128, H=32, D=128)[1]["path"] == nat.PATH_STREAM
    assert q(R=128, B=16, H=32, D=128)[1]["path"] == nat.PATH_WIDE
    assert q(R=64, B=4, H=8)[1]["path"] == nat.PATH_WIDE
    assert q(R=17, B=64, H=64, path=nat.PATH_VECTOR)[1]["path"] == nat.PATH_VECTOR
    assert q(R=17, B=64, H=64, path=nat.PATH_WIDE)[1]["path"] == nat.PATH_WIDE


@pytest.mark.parametrize("D,lanes,nv,slices", [(8, 4, 1, 1), (24, 4, 1, 1), (128, 8, 2, 1),
                                                (256, 16, 2, 1), (264, 32, 2, 1), (1024, 32, 2, 2),
                                                (4096, 32, 2, 8)])
def test_lanes_and_slices_follow_D(D, lanes, nv, slices):
    rc, plan = q(R=2, D=D, B=8, H=64)
    assert rc == 0 and (plan["lanes"], plan["nv"], plan["slices_per_row"]) == (lanes, nv, slices)



def sq(B=2, H=3, D=64, st=None, a=nat.BF16, n=nat.BF16, acc=OUT, lacc=OUTL, new=PO, lnew=PL):
    return nat.state_update_raw(acc, lacc, new, lnew, B, H, D, st, a, n, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(a=5), nat.EDTYPE), (dict(n=-1), nat.EDTYPE),
    (dict(B=0), nat.EDIMS), (dict(D=0), nat.EDIMS),
    (dict(acc=0), nat.ENULL), (dict(lacc=0), nat.ENULL), (dict(new=0), nat.ENULL), (dict(lnew=0), nat.ENULL),
    (dict(st=(-64, 64, 3, 1)), nat.ESTRIDE), (dict(st=(192, 64, 3, -1)), nat.ESTRIDE),
    (dict(acc=OUT + 1), nat.EALIGN), (dict(lacc=OUTL + 2), nat.EALIGN), (dict(a=nat.F32, acc=OUT + 2), nat.EALIGN),
    (dict(new=OUT + 64), nat.EALIAS), (dict(lacc=OUT + 4), nat.EALIAS), (dict(lnew=OUTL), nat.EALIAS),
    (dict(lnew=OUT), nat.EALIAS),
    (dict(B=2 ** 30, H=2 ** 30, D=2 ** 30), nat.EDIMS),
])
def test_state_update_validation(kw, code):
    # rejected before any CUDA call
    assert sq(**kw) == code, (kw, nat.strerror(code))


WS = 0x7f5000000000


def dq(B=2, Hq=8, Hkv=2, L=100, D=128, R=4, scale=0.1, st=None, dt=nat.BF16, q=PO, k=PL,
       v=0x7f4000000000, out=OUT, outl=OUTL, fused=True, odt=nat.BF16, ws=0, wsb=1 << 30):
    return nat.decode_raw(q, k, v, 0, B, Hq, Hkv, L, D, R, scale, st, dt, out, outl,
                          fused=fused, out_dtype=odt, check=False, workspace=ws,
                          workspace_bytes=wsb)


@pytest.mark.parametrize("kw,code", [
    (dict(dt=nat.F32), nat.EUNSUP), (dict(dt=7), nat.EDTYPE), (dict(odt=9), nat.EDTYPE),
    (dict(D=96), nat.EUNSUP), (dict(D=256), nat.EUNSUP), (dict(Hq=6, Hkv=4), nat.EUNSUP),
    (dict(Hq=34, Hkv=2), nat.EUNSUP), (dict(R=3), nat.EUNSUP), (dict(R=16), nat.EUNSUP),
    (dict(B=0), nat.EDIMS), (dict(L=0), nat.EDIMS), (dict(R=0), nat.EDIMS), (dict(B=70000), nat.EDIMS),
    (dict(scale=float("nan")), nat.EDIMS), (dict(scale=float("inf")), nat.EDIMS),
    (dict(q=0), nat.ENULL), (dict(out=0), nat.ENULL),
    (dict(q=PO + 8), nat.EALIGN), (dict(st=(8 * 128, 130, 2 * 100 * 128, 100 * 128, 128,
                                            2 * 100 * 128, 100 * 128, 128)), nat.EALIGN),
    (dict(st=(-1, 128, 0, 0, 128, 0, 0, 128)), nat.ESTRIDE),
    (dict(out=PL + 64), nat.EALIAS), (dict(outl=PO), nat.EALIAS),
    (dict(fused=False, out=PL), nat.EALIAS),
])
def test_decode_attention_validation(kw, code):
    assert dq(**kw) == code, (kw, nat.strerror(code))


def test_decode_valid_arguments_pass_validation():
    # valid arguments get past validation (here, without a GPU, the launch itself fails)
    for kw in (dict(), dict(R=3, fused=False), dict(R=64, fused=False), dict(D=64, Hq=16, Hkv=1),
               dict(ws=WS), dict(ws=WS, R=3), dict(ws=WS, R=64), dict(ws=WS, R=1000, L=50)):
        assert dq(**kw) in (nat.OK, nat.ELAUNCH), kw


def test_decode_workspace_layout_and_validation():
    # counters [B, Hkv] u32, then lse [B, Hq, R] and o [B, Hq, R, D] fp32, each part 256-aligned
    B, Hq, Hkv, R, D = 2, 8, 2, 4, 128
    need = nat.decode_workspace_bytes(B, Hq, Hkv, R, D)
    assert need == 256 + 256 + B * Hq * R * D * 4
    assert nat.decode_workspace_bytes(3, 4, 4, 5, 64) == 256 + 256 + 3 * 4 * 5 * 64 * 4
    assert dq(ws=WS, wsb=need) in (nat.OK, nat.ELAUNCH)
    assert dq(ws=WS, wsb=need - 1) == nat.EDIMS            # too short
    assert dq(ws=WS + 8, wsb=need) == nat.EALIGN           # not 16-byte aligned
    assert dq(ws=OUT - 64, wsb=need) == nat.EALIAS         # overlaps the output
    assert dq(ws=PL + 128, wsb=need) == nat.EALIAS         # overlaps k
    for bad in (dict(B=0), dict(Hq=6, Hkv=4), dict(R=0)):
        args = {**dict(B=B, Hq=Hq, Hkv=Hkv, R=R, D=D), **bad}
        with pytest.raises(nat.LseMergeError):
            nat.decode_workspace_bytes(args["B"], args["Hq"], args["Hkv"], args["R"], args["D"])


def test_fast_forwarding_extension_is_built_and_checks_its_arguments():
    """The vectorcall extension forwards to the same C entry points: a call
    the library rejects returns the library's code (no CUDA call is made),
    and Python-level mistakes raise before C is reached."""
    from lse_weighted_merge_b200 import _fast
    st = (64, 256, 128, 1, 4, 2)
    assert _fast.merge(PO, PL, 2, 1, 0, 64, st, nat.BF16, nat.BF16, OUT, OUTL, 0, 0) == nat.EDIMS
    assert _fast.merge(PO, PL, 2, 1, 2, 64, None, 7, nat.BF16, OUT, OUTL, 0, 0) == nat.EDTYPE
    assert _fast.merge(0, PL, 2, 1, 2, 64, None, nat.BF16, nat.BF16, OUT, OUTL, 0, 0) == nat.ENULL
    assert _fast.state_update(PO, PL, OUT, OUTL, 0, 2, 64, None, nat.F32, nat.BF16, 0) == nat.EDIMS
    with pytest.raises(TypeError):
        _fast.merge(PO, PL, 2, 1, 2, 64)                       # too few arguments
    with pytest.raises(TypeError):
        _fast.merge(PO, PL, 2, 1, 2, 64, (1, 2), 2, 2, OUT, OUTL, 0, 0)   # strides tuple of 2
    with pytest.raises(OverflowError):
        _fast.merge(PO, PL, 2**40, 1, 2, 64, None, 2, 2, OUT, OUTL, 0, 0)
    with pytest.raises(OverflowError):
        _fast.merge(-5, PL, 2, 1, 2, 64, None, 2, 2, OUT, OUTL, 0, 0)     # a negative pointer
    # merge_raw takes every strides form it documents and routes through the extension
    for s in (st, ((64, 256, 128), (1, 4, 2)), nat.Strides(*st)):
        assert nat.merge_raw(PO, PL, 2, 1, 0, 64, s, nat.BF16, nat.BF16, OUT, OUTL, 0,
                             check=False) == nat.EDIMS


def test_host_pipeline_stage_bytes_and_null_context():
    # staging of one call: partials, lse, outputs, merged lse, each 256-aligned
    R, B, H, D = 16, 512, 16, 512
    up = lambda x: -(-x // 256) * 256
    want = up(R * B * H * D * 2) + up(R * B * H * 4) + up(B * H * D * 4) + up(B * H * 4)
    assert nat.host_stage_bytes(R, B, H, D, nat.BF16, nat.F32) == want
    assert nat.host_stage_bytes(3, 5, 7, 9, nat.F32, nat.F16) == \
        up(3 * 5 * 7 * 9 * 4) + up(3 * 5 * 7 * 4) + up(5 * 7 * 9 * 2) + up(5 * 7 * 4)
    with pytest.raises(nat.LseMergeError):
        nat.host_stage_bytes(0, B, H, D, nat.BF16, nat.F32)
    with pytest.raises(nat.LseMergeError):
        nat.host_stage_bytes(R, B, H, D, 9, nat.F32)
    # no context: refused before any CUDA call
    assert nat.host_merge_raw(0, PO, PL, R, B, H, D, nat.LAYOUT_BHRD, nat.BF16, nat.F32, OUT, OUTL,
                              8, check=False) == nat.ENULL
    assert nat.strerror(nat.EDEVICE) != nat.strerror(999)
