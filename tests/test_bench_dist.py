"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

bench.py runs one independent batch per rank (sequences do not interact, so
the path shards with no exchange); the whole-job number is the units all ranks
processed over the slowest rank's time. These checks run the same helpers
bench.py uses under torchrun, with the gloo backend instead of NCCL.
"""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_setup(backend="gloo")
    res = {
        "world": w, "rank": r,
        "max": bench.max_over_ranks(1.5 + r, w),
        "sum": bench.sum_over_ranks(10.0 * (r + 1), w),
        "seed": bench.rank_seed(7, r),
        # rank r processed 100 * (r + 1) units in (r + 1) seconds
        "job": bench.whole_job_throughput(100.0 * (r + 1), float(r + 1), w),
    }
    bench.barrier(w)
    torch.save(res, os.path.join(out_dir, f"rank{r}.pt"))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r, x in enumerate(res):
        assert x["world"] == 2 and x["rank"] == r
        assert x["max"] == 2.5                       # max over ranks of 1.5 + r
        assert x["sum"] == 30.0                      # 10 + 20
        assert x["job"] == pytest.approx(300.0 / 2.0)  # (100 + 200) units / slowest 2 s
    assert res[0]["seed"] != res[1]["seed"]          # each rank draws its own batch


def test_single_rank_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_setup() == (1, 0, 0)
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.whole_job_throughput(50.0, 2.0, 1) == 25.0


def test_traffic_digest_ignores_comments_only():
    # The DRAM capture of a kernel stays valid through edits to its comments
    # and blank lines, and not through any edit to its code.
    sys.path.insert(0, ROOT)
    import bench
    src = 'int a = 1; // count\n/* block\n comment */ const char* s = "x//y\\"z";\n\n  a++;\n'
    assert bench.strip_comments(src) == 'int a = 1;\n const char* s = "x//y\\"z";\n  a++;'
    assert bench.strip_comments(src.replace("count", "number")) == bench.strip_comments(src)
    assert bench.strip_comments(src.replace("a++", "a--")) != bench.strip_comments(src)

