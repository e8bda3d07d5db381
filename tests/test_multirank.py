"""The replica path of bench.py on two ranks: world_size-2 gloo process
groups on the CPU (one process per rank, as torchrun starts them)."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(world)
    bench.barrier(w)
    res = {"world": w, "rank": r, "local": local, "backend": dist.get_backend(),
           # the bench's aggregation: max of the per-rank times, sum of the per-rank units
           "max": bench.max_over_ranks(10.0 * (r + 1), w, "cpu"),
           "sum": bench.sum_over_ranks(1344.0, w, "cpu")}

    class Args:
        gpus, steps, warmup = world, 1, 3
    if r != 0:  # the reference arm: ranks other than 0 leave at once without work
        res["reference_rc"] = bench.run_reference(Args, None, w, r)
    bench.barrier(w)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)


def test_two_rank_aggregation_on_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, g in enumerate(got):
        assert (g["world"], g["rank"], g["local"], g["backend"]) == (2, r, r, "gloo")
        assert g["max"] == 20.0 and g["sum"] == 2688.0
    assert got[1]["reference_rc"] == 0
