"""The N > 1 path of bench.py on CPU: two gloo ranks (data-parallel replicas).

Checks the plumbing the GPU run relies on: barriers, the max over ranks of
every timed figure, whole-job throughput over all ranks, the one exchange of
data-parallel training (the adapter gradients summed over ranks, in place,
in the stack's flat gradient layout), and that the reference arm does its
work on rank 0 only."""
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
    # adapter gradients of a small stack in the flat layout: rank k holds (k + 1) * (1, 2, 3, ...)
    from layer_streamed_nf4_b200 import synth
    from layer_streamed_nf4_b200.stack import ProjLayout, grad_layout
    cfg = synth.STACKS["0.5b"]
    projs = [ProjLayout(n, K, N, 0, 0) for n, K, N in cfg.projections]
    offs, n = grad_layout(projs, 2, cfg.rank)
    g = torch.arange(1, n + 1, dtype=torch.float64).to(torch.float32) * (rank + 1)
    reps.allreduce_sum(g)
    ok_sum = bool(torch.equal(g, torch.arange(1, n + 1, dtype=torch.float64).to(torch.float32) * 3))
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
        f.write(f"{reps.world} {ms} {tput} {buf.getvalue()!r} {ran_reference!r} {ok_sum}\n")


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    lines = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for r, (w, ms, tput, printed, ret, ok_sum) in enumerate(lines):
        assert int(w) == world
        assert ok_sum == "True"                      # gradients summed over both ranks, on both ranks
        assert float(ms) == 15.0                     # the slowest rank's time, on every rank
        assert abs(float(tput) - world * 2048 / 0.015) < 1e-6 * float(tput)
        if r != 0:
            assert printed == "''" and ret == "None"


def test_grad_layout_is_disjoint_and_aligned():
    """The flat gradient buffer: per (layer, projection) dA [r, K] then dB [N, r], no overlap, every
    tensor on a 16-byte boundary; the 8B stack's adapters are 32 x 1.31 M fp32 values (168 MB)."""
    from layer_streamed_nf4_b200 import synth
    from layer_streamed_nf4_b200.stack import ProjLayout, grad_layout
    for name, cfg in synth.STACKS.items():
        projs = [ProjLayout(n, K, N, 0, 0) for n, K, N in cfg.projections]
        for r in (cfg.rank, 8, 24):
            offs, n = grad_layout(projs, 3, r)
            spans = []
            for (l, pi), o in offs.items():
                p = projs[pi]
                for start, size in ((o, r * p.K), (o + r * p.K, r * p.N)):
                    assert (start * 4) % 16 == 0, (name, r, l, pi)
                    spans.append((start, start + size))
            spans.sort()
            assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
            assert spans[-1][1] <= n
    cfg = synth.STACKS["8b"]
    _, n = grad_layout([ProjLayout(nm, K, N, 0, 0) for nm, K, N in cfg.projections], cfg.layers, cfg.rank)
    assert n == cfg.layers * cfg.rank * sum(K + N for _, K, N in cfg.projections) == 32 * 1310720
