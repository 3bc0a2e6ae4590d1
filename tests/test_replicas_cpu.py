"""The N > 1 path of bench.py on CPU: two gloo ranks (replicas only, no data-path collective).

Checks the plumbing the GPU run relies on: barriers, the max over ranks of
every timed figure, whole-job throughput over all ranks, and that the
reference arm does its work on rank 0 only."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch
    import bench
    reps = bench.Replicas("gloo", torch.device("cpu"))
    reps.barrier()
    ms = reps.max(10.0 + 5.0 * rank)              # each rank's own step time
    tput = reps.throughput(2048, ms)
    # the reference arm: rank 0 alone runs it; every other rank returns at once, printing nothing
    buf = io.StringIO()
    ran_reference = None
    if rank != 0:
        class Args:
            steps, warmup, ref_rows = 1, 3, 4
        with redirect_stdout(buf):
            ran_reference = bench.run_reference(Args())
    reps.barrier()
    reps.close()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(f"{reps.world} {ms} {tput} {buf.getvalue()!r} {ran_reference!r}\n")


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    lines = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for r, (w, ms, tput, printed, ret) in enumerate(lines):
        assert int(w) == world
        assert float(ms) == 15.0                     # the slowest rank's time, on every rank
        assert abs(float(tput) - world * 2048 / 0.015) < 1e-6 * float(tput)
        if r != 0:
            assert printed == "''" and ret == "None"
