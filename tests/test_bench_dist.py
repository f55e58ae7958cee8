"""The benchmark's multi-rank host logic on CPU (gloo, world size 2).

The decode path does not shard: with N GPUs every rank decodes its own
request, the time is the maximum over ranks and the value counts all ranks'
tokens.  These tests run that logic with two gloo ranks; no GPU is involved."""
import argparse
import json
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, what):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench

    args = argparse.Namespace(impl="reference")
    res = {}
    if what == "max":
        _, r, _, pg = bench.dist_setup(args)
        bench.barrier(pg)
        ms = 10.0 + 5.0 * r   # rank 1 is the slow one
        res["max"] = bench.max_over_ranks(pg, ms)
        res["whole_job"] = bench.whole_job(res["max"], 64, world)
        bench.barrier(pg)
        pg.destroy_process_group()
    elif what == "reference-nonzero-rank":
        if rank == 0:
            _, _, _, pg = bench.dist_setup(args)
            pg.destroy_process_group()
        else:
            bench.run_reference(args)   # returns at once on ranks other than 0
        res["done"] = True
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def _run(tmp_path, what, world=2):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), what)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    return [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]


def test_max_over_ranks_and_whole_job_value(tmp_path):
    res = _run(tmp_path, "max")
    for r in res:
        assert r["max"] == 15.0
        ms_per_token, tok_s = r["whole_job"]
        # 2 ranks x 64 tokens in the slowest rank's 15 ms
        assert ms_per_token == pytest.approx(15.0 / 128)
        assert tok_s == pytest.approx(128 / 15e-3)


def test_reference_arm_runs_on_rank0_only(tmp_path, capfd):
    res = _run(tmp_path, "reference-nonzero-rank")
    assert all(r["done"] for r in res)


def test_whole_job_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job(20.0, 10, 1) == pytest.approx((2.0, 500.0))


def test_requests_option_is_checked_before_any_gpu_work():
    """--requests outside 2..16 is refused while parsing the arguments; inside
    it, the batch workload takes it (default 8)."""
    import bench
    with pytest.raises(SystemExit):
        bench.parse(["--workload", "batch8", "--requests", "17"])
    with pytest.raises(SystemExit):
        bench.parse(["--workload", "batch8", "--requests", "1"])
    a = bench.parse(["--workload", "batch8", "--requests", "16"])
    assert a.requests == 16 and a.steps == bench.BATCH_GENERATED
    assert bench.parse(["--workload", "batch8"]).requests == 0
