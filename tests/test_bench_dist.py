"""The multi-rank plumbing of bench.py, on CPU with two gloo ranks.

R-SWA shards by sequence with no exchange, so `bench.py --gpus N` runs one
independent replica per rank: each rank draws its own inputs, the timed
region is bracketed by barriers, the reported time is the maximum over the
ranks and the reported units are their sum.  The reference arm (the oracle
on the host) runs on rank 0 only; the other ranks exit without work.  These
tests run the same functions under a real two-process gloo group.
"""

from __future__ import annotations

import contextlib
import datetime
import io
import json
import multiprocessing as mp
import os
import socket
import sys

import pytest

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, out) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        env = bench.dist_env()
        # rank r took 1.5 + r seconds for 100 * (r + 1) tokens
        el_max, tok_sum = bench.reduce_max_sum(1.5 + rank, 100.0 * (rank + 1))
        seeds = [bench.replica_seed(1000, layer, rank) for layer in range(4)]
        dist.barrier()
        buf = io.StringIO()
        argv = sys.argv
        sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(WORLD), "--steps", "4", "--warmup", "3",
                    "--cpu-budget", "0.05"]
        try:
            with contextlib.redirect_stdout(buf):
                rc = bench.main()
        finally:
            sys.argv = argv
        dist.barrier()
        # the prefill workload's reference arm follows the same rule
        pbuf = io.StringIO()
        sys.argv = ["bench.py", "--impl", "reference", "--workload", "prefill", "--gpus", str(WORLD),
                    "--steps", "4", "--warmup", "3", "--cpu-budget", "0.05"]
        try:
            with contextlib.redirect_stdout(pbuf):
                prc = bench.main()
        finally:
            sys.argv = argv
        dist.barrier()
        out.put({"rank": rank, "env": env, "el_max": el_max, "tok_sum": tok_sum, "seeds": seeds,
                 "rc": rc, "stdout": buf.getvalue(), "prefill_rc": prc, "prefill_stdout": pbuf.getvalue()})
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(WORLD):
            item = out.get(timeout=240)
            res[item["rank"]] = item
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()  # this test's own child, by handle
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return res


def test_env_is_read_per_rank(ranks):
    for r in range(WORLD):
        assert ranks[r]["env"] == (WORLD, r, r)


def test_time_is_max_and_units_are_summed_over_ranks(ranks):
    for r in range(WORLD):
        assert ranks[r]["el_max"] == pytest.approx(2.5)
        assert ranks[r]["tok_sum"] == pytest.approx(300.0)
    import bench
    assert bench.whole_job_rate(ranks[0]["tok_sum"], ranks[0]["el_max"]) == pytest.approx(120.0)


def test_replicas_draw_distinct_inputs(ranks):
    s0, s1 = set(ranks[0]["seeds"]), set(ranks[1]["seeds"])
    assert len(s0) == 4 and len(s1) == 4 and not (s0 & s1)


def test_reference_arm_runs_on_rank0_only(ranks):
    assert ranks[0]["rc"] == 0 and ranks[1]["rc"] == 0
    assert ranks[1]["stdout"].strip() == ""
    lines = [ln for ln in ranks[0]["stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == WORLD
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_single_process_reduction_is_identity():
    import bench
    assert bench.reduce_max_sum(0.25, 7.0) == (0.25, 7.0)


def test_prefill_reference_arm_runs_on_rank0_only(ranks):
    assert ranks[0]["prefill_rc"] == 0 and ranks[1]["prefill_rc"] == 0
    assert ranks[1]["prefill_stdout"].strip() == ""
    lines = [ln for ln in ranks[0]["prefill_stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["ms_per_step"] > 0
