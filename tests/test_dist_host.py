"""The multi-rank host logic of bench.py on CPU ranks (gloo, world size 2):
rank discovery, barrier, max-over-ranks timing, weak-scaling accounting, and
the reference arm printing from rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, l = bench.dist_env()
    dist = bench.dist_init(w, backend="gloo")
    dev = torch.device("cpu")
    bench.barrier(dist, dev)
    got = bench.max_over_ranks(10.0 + rank, dist, dev)
    flag = bench.max_over_ranks(1.0 if rank == 1 else 0.0, dist, dev)
    dist.destroy_process_group()
    q.put((rank, w, r, l, got, flag))


def test_two_gloo_ranks_agree_on_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, r, l, got, flag in res:
        assert (w, r, l) == (2, rank, rank)
        assert got == 11.0 and flag == 1.0


def test_weak_scaling_accounting():
    sys.path.insert(0, ROOT)
    import bench
    from lse_weighted_merge_b200 import synth
    w = synth.WORKLOADS[synth.LARGE]
    cfg = bench.config_block(w, 4, "x")
    assert cfg["global_batch"] == 4 * w.B and cfg["bytes_per_step"] == 151_552_000
    assert w.bytes_read() == 134_742_016 and w.bytes_written() == 16_809_984
    assert bench.n_sets(w.bytes_total(), 126 * 2**20) == 3
    assert bench.n_sets(792, 126 * 2**20) == 256


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0 and p.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_next_rows_get_an_oracle_baseline():
    """bench.py times the fp64 oracle beside the state-update, decode-attention
    and exchange lines (bounded samples, one thread)."""
    sys.path.insert(0, ROOT)
    import bench
    extra = {"state_update": {}, "decode_attention": {"b64_hq32_hkv8_l4096_d128_r4": {}},
             "cp_exchange_merge": {"cp_w2_b1_h2_d64": {}}}
    bench.next_rows_cpu_baselines(extra, budget_s=0.02)
    rows = [extra["state_update"], extra["decode_attention"]["b64_hq32_hkv8_l4096_d128_r4"],
            extra["cp_exchange_merge"]["cp_w2_b1_h2_d64"]]
    for row in rows:
        cb = row["cpu_baseline"]
        assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0 and cb["sample"]
