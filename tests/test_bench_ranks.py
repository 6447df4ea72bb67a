"""Multi-rank logic of bench.py on CPU: two gloo ranks on 127.0.0.1 take the bench's collective
steps (barrier, max over ranks of the per-rank times) and compute the whole-job rate, and the
reference arm runs on rank 0 alone.  No GPU: the replica path has no data-path collective, so
this is all of the N > 1 logic."""
import argparse
import json
import os
import pathlib
import socket
import sys

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        res = {}
        # each rank's own times; the job's time is the slowest rank's
        mine = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        bench.rank_barrier()
        res["max"] = bench.max_over_ranks(mine)
        res["rate"] = bench.whole_job_rate(100.0, world, res["max"][0])
        bench.rank_barrier()
        args = argparse.Namespace(workload="tiny_fp32", steps=2, warmup=1, n_split=None, batch=0, length=0)
        line = bench.run_reference(args, rank, world)
        res["reference"] = line
        bench.rank_barrier()
        (pathlib.Path(out_dir) / f"rank{rank}.json").write_text(json.dumps(res))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    r = [json.loads((tmp_path / f"rank{i}.json").read_text()) for i in range(world)]
    for i in range(world):
        assert r[i]["max"] == [2.0, 5.0, 0.5]                   # element-wise max over both ranks
        assert r[i]["rate"] == pytest.approx(100.0 * 2 / 2e-3)  # both ranks' units over the slowest time
    ref = r[0]["reference"]
    assert r[1]["reference"] is None                            # rank 1 does no work in the reference arm
    assert ref["impl"] == "reference" and ref["n_gpus"] == world and ref["scaling"] == "weak"
    assert ref["value"] > 0 and ref["cpu_baseline"]["kind"] == "oracle"
    assert ref["e2e"]["h2d_bytes_per_step"] == 0 and ref["e2e"]["d2h_bytes_per_step"] == 0


def test_single_process_is_the_identity():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.max_over_ranks([3.0, 1.5]) == [3.0, 1.5]
    bench.rank_barrier()  # no process group: nothing to wait for
    assert bench.whole_job_rate(10.0, 1, 2.0) == pytest.approx(5000.0)
