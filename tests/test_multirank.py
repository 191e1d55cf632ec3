"""Host logic of bench.py's multi-GPU path, run as world_size-2 gloo ranks on
the CPU: one replica per rank (weak scaling), time = max over ranks, whole-job
throughput over all ranks, and only rank 0 prints.  No data-path collective
exists to test: the ranks never exchange tensors other than the timing."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        got_ws, got_rank, got_local = bench.dist_env()
        # each rank times a different duration; every rank must see the slowest
        elapsed = 1.0 + rank
        slowest = bench.max_over_ranks(elapsed, ws, "cpu")
        value = bench.whole_job_value(1e9, 10, ws, slowest)
        # the reference arm: rank 0 alone prints, the others return without work
        out = io.StringIO()
        if rank != 0:
            class A:
                gpus, warmup, steps = ws, 3, 1
            with redirect_stdout(out):
                rc = bench.reference_arm(A())
        else:
            rc = 0
        q.put((rank, got_ws, got_rank, got_local, slowest, value, rc, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_rank1_stays_silent():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got_ws, got_rank, got_local, slowest, value, rc, printed in res:
        assert (got_ws, got_rank, got_local) == (ws, rank, rank)
        assert slowest == 2.0                      # max over ranks, identical everywhere
        assert value == pytest.approx(1e9 * 10 * ws / 2.0 / 1e9)
        assert rc == 0
        assert printed == ""                       # only rank 0 prints a line


def test_whole_job_value_is_weak_scaling_aggregate():
    import bench
    one = bench.whole_job_value(4e6, 100, 1, 0.5)
    assert bench.whole_job_value(4e6, 100, 8, 0.5) == pytest.approx(8 * one)
    # a slower slowest rank lowers the aggregate in proportion
    assert bench.whole_job_value(4e6, 100, 8, 1.0) == pytest.approx(4 * one)


def test_reference_arm_prints_one_json_line_on_rank0(monkeypatch):
    """The oracle arm on rank 0 prints one JSON line with impl=reference."""
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(bench, "reference_steps",
                        lambda w, steps, warmup: (1e-3 * steps, "stub sample"))

    class A:
        gpus, warmup, steps = 1, 3, 1
    out = io.StringIO()
    with redirect_stdout(out):
        assert bench.reference_arm(A()) == 0
    lines = [l for l in out.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["higher_is_better"]
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    # a reported step is a measured one: ms_per_step x steps = the timed seconds
    assert rec["ms_per_step"] * rec["steps"] == pytest.approx(1e-3 * A.steps * 1e3)
    assert rec["cpu_baseline"]["host"]["nproc"] >= 1


def test_oracle_bundles_pair_every_retrieval_with_a_streaming_pair():
    """The all-core oracle run splits the pairs into bundles of equal cost."""
    import bench
    import synth
    w = synth.llama3_8b_decode()
    bundles = bench._bundles(w)
    flat = sorted(p for b in bundles for p in b)
    assert flat == list(range(w.B * w.H_kv))
    for b in bundles:
        assert sorted(int(w.head_kind[p % w.H_kv]) for p in b) == [0, 1]
