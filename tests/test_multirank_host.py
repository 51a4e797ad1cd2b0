"""Host side of `bench.py --gpus N`: world-size-2 gloo ranks on the CPU.

With N > 1 every rank runs its own independent GEMM (weak scaling, no data
exchange); the only collectives are the barrier and the max over ranks of
the timed region.  These tests run that logic on two CPU processes.
"""
import importlib.util
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, out_dir):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = load_bench()
        # rank r "took" 1 + r seconds for 10 steps of 2e12 flops each
        elapsed = bench.max_over_ranks(dist, 1.0 + rank, torch.device("cpu"))
        rate = bench.job_rate(2e12, 10, world, elapsed)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"elapsed": elapsed, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_agree_on_max_time(tmp_path):
    world = 2
    mp.start_processes(rank_main, args=(world, free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r in res:
        assert r["elapsed"] == 2.0                      # the slowest rank's time
        assert r["rate"] == 2e12 * 10 * world / 2.0     # all ranks' work / max time


def test_single_rank_needs_no_group():
    bench = load_bench()
    assert bench.max_over_ranks(None, 3.5, None) == 3.5
    assert bench.job_rate(1.0, 4, 1, 2.0) == 2.0


def test_reference_arm_other_ranks_do_no_work():
    """Under torchrun only rank 0 runs and prints the reference arm."""
    bench = load_bench()
    sys_argv = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    try:
        args = bench.parse()
    finally:
        sys.argv = sys_argv
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(args, 2, 1)
    assert rc == 0 and buf.getvalue() == ""
