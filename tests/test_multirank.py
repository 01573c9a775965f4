"""Host side of the multi-GPU bench path, on CPU with two gloo ranks.

Under torchrun every rank runs its own independent batch (weak scaling, no data-path collective):
the only collectives are the barrier around the timed region and the max-over-ranks of the step
time. These tests run that logic with world_size 2 on the gloo backend, plus the reference arm's
rank handling (only rank 0 works and prints).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import bench
    from gated_delta_rule_143_b200.inputs import CHUNK_WORKLOADS, WORKLOAD_SEEDS, make_chunk_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # a per-rank "step time": the job's time is the slowest rank's
        ms = bench.max_over_ranks(1.5 + rank, world)
        w = CHUNK_WORKLOADS[bench.WORKLOAD]
        seed = bench.rank_seed(WORKLOAD_SEEDS[bench.WORKLOAD], rank, 0)
        # each rank's batch differs (small shapes stand in for the workload's)
        x = make_chunk_inputs(1, 64, 2, 32, 32, w.mode, "bf16", seed)
        digest = float(x["k"].float().sum())
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "seed": seed, "digest": digest,
                       "value": bench.job_throughput(w.B * w.T, ms, world)}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_max_step_time(tmp_path):
    world = 2
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert res[0]["ms"] == res[1]["ms"] == 2.5  # max over ranks, seen identically by both
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["digest"] != res[1]["digest"]  # independent batches per rank
    # whole-job rate: both ranks' tokens over the slowest rank's time
    assert res[0]["value"] == pytest.approx(2 * 8 * 4096 / 2.5e-3)


def test_job_throughput_is_weak_scaling_sum():
    import bench
    assert bench.job_throughput(1000, 2.0, 1) == pytest.approx(5e5)
    assert bench.job_throughput(1000, 2.0, 4) == pytest.approx(2e6)


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_kernel_code_digest_ignores_comments_only():
    """Recorded DRAM counters stay valid across comment edits of the kernel source, not code edits."""
    import bench
    a = "int f(int x) {  // doubles\n    return 2 * x;  /* the\n factor */\n}\n"
    b = "// new header\nint f(int x) {\n\n    return 2 * x;\n}\n"
    c = "int f(int x) {\n    return 3 * x;\n}\n"
    assert bench.kernel_code_digest(a) == bench.kernel_code_digest(b)
    assert bench.kernel_code_digest(a) != bench.kernel_code_digest(c)


@pytest.mark.parametrize("plan", ["fused", "prep_fused", "two_pass", "cuda_core", "scan"])
def test_kernel_bytes_split_the_step_bytes(plan):
    """The roofline's per-kernel algorithmic bytes add up to the whole step's, on every plan (the
    segment scan's state kernel writes only intermediates, so it carries none)."""
    import bench
    from gated_delta_rule_143_b200.inputs import CHUNK_WORKLOADS
    for w in CHUNK_WORKLOADS.values():
        nc = -(-w.T // w.chunk)
        c1 = (nc + 1) // 2 if plan == "prep_fused" else 0  # some chunks pre-computed, some not
        parts = bench.kernel_bytes(w, plan, c1)
        assert sum(b for _, b in parts) == bench.chunk_bytes(w)
        assert all(b > 0 for name, b in parts if not (plan == "scan" and name == "chunk_state"))


def _retry_rank_main(rank, world, port, out_dir):
    import datetime

    import bench
    from gated_delta_rule_143_b200._lib import GdrError

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        calls = []

        def record():  # rank 0's device status fails on the first run only
            calls.append(1)
            bench.barrier(world)
            if rank == 0 and len(calls) == 1:
                raise GdrError(-6, "a kernel's bounded wait expired (wait kind 2, block 3, thread 0, detail 0x0)")
            return 7

        out = bench.with_status_retry("rec", record, world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"out": out, "calls": len(calls), "retries": bench.STATUS_RETRIES}, f)
    finally:
        dist.destroy_process_group()


def test_status_retry_is_taken_by_every_rank(tmp_path):
    """A record whose device status fails on one rank runs again on every rank (same collectives),
    and the failure is kept for the bench line."""
    world = 2
    port = _free_port()
    mp.start_processes(_retry_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["out"] for r in res] == [7, 7] and [r["calls"] for r in res] == [2, 2]
    assert res[0]["retries"][0]["record"] == "rec" and "bounded wait" in res[0]["retries"][0]["error"]
    assert res[1]["retries"][0]["error"] == "on another rank"


def test_status_retry_gives_up_after_a_second_failure():
    import bench
    from gated_delta_rule_143_b200._lib import GdrError

    def record():
        raise GdrError(-6, "expired")

    before = len(bench.STATUS_RETRIES)
    with pytest.raises(RuntimeError):
        bench.with_status_retry("rec2", record, 1)
    assert len(bench.STATUS_RETRIES) == before + 2
    assert bench.with_status_retry("rec3", lambda: 5, 1) == 5
