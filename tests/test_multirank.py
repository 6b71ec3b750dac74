"""The host side of the multi-process bench on CPU: two gloo ranks, as torchrun
would start them.  The decode path shards by sequence with no data-path
collective, so what crosses ranks is only the timing plumbing: the job time is
the slowest rank's, the job rate counts every rank's rows, every rank draws
its own sequences, and only rank 0 prints."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, what):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    res = {}
    if what == "plumbing":
        r, w = bench.init_ranks("gloo")
        res["rank_world"] = [r, w]
        res["max"] = bench.max_over_ranks(10.0 + 5.0 * r, w, "cpu")
        res["seed_shift"] = bench.rank_seed_shift(r)
        import torch.distributed as dist
        dist.destroy_process_group()
    else:
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3",
                             "--ref-rows", "2"], backend="gloo")
        res["rc"] = rc
        res["stdout"] = buf.getvalue()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def _run(tmp_path, what, world=2):
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), what),
                       nprocs=world, join=True, start_method="spawn")
    return [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]


def test_two_ranks_time_is_the_slowest_rank(tmp_path):
    import bench
    res = _run(tmp_path, "plumbing")
    assert [r["rank_world"] for r in res] == [[0, 2], [1, 2]]
    assert [r["max"] for r in res] == [15.0, 15.0]
    assert len({r["seed_shift"] for r in res}) == 2          # disjoint batches
    # 64 rows per rank, 10 steps, 2 ranks in 2 ms (the slowest rank): 640,000 rows/s
    assert bench.job_rate(64, 10, 2, 2.0) == pytest.approx(640000.0)


@pytest.mark.timeout(600)
def test_reference_arm_prints_on_rank_zero_only(tmp_path):
    res = _run(tmp_path, "reference")
    assert all(r["rc"] == 0 for r in res)
    assert res[1]["stdout"] == ""
    line = json.loads(res[0]["stdout"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
