"""Benchmark: layer-streamed NF4 LoRA linears, fwd + bwd, on the Llama-3.1-8B
shaped stack (32 layers x 7 projections, T = 2048 tokens, r = 16, alpha = 32,
NF4 codes streamed from pinned host RAM through a VRAM pool of 20 layer
slots, which at 2048 tokens hides the PCIe copies behind compute; the
two-slot pool is timed beside it as mode streamed_S2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = forward over layers 0..31 then backward over 31..0, every
projection through lora_linear_fwd / lora_linear_bwd of the C ABI, base
weights streamed by the layer pool.  Prints ONE JSON line (rank 0).

--impl reference times the CPU oracle (fp64, host cores) on a bounded sample
of the same workload and prints the same metric.  With N > 1 every rank runs
an independent replica (weak scaling; the method has no exchange step).
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "train tok/s, 8B-shape NF4 LoRA fwd+bwd; % of bf16 tensor-core peak"
UNIT = "tok/s"
WORKLOAD = "8b"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        loaded = [v for v in sms if mx is None or v >= 0.3 * mx] or sms
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sms)}


def _dist():
    n = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return n, rank, local


class Replicas:
    """The N > 1 plumbing: one process per GPU (launched by torchrun), each a data-parallel replica of the
    path on its own tokens.  The one exchange of data-parallel training is the sum of the adapter gradients
    over ranks, once per step (allreduce_sum); the layer stream and the linears do not shard.  Timed regions
    are bracketed by barriers, every timed figure is the max over ranks, and throughput counts the tokens
    of all ranks."""

    def __init__(self, backend: str, device):
        import torch.distributed as dist
        self.world, self.rank, self.local = _dist()
        self.device = device
        self.dist = dist
        if self.world > 1 and not dist.is_initialized():
            from datetime import timedelta
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=300), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if self.world == 1:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def allreduce_sum(self, t):
        """t summed over the ranks in place (enqueued on the current stream); nothing with one rank."""
        if self.world > 1:
            self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM)

    def throughput(self, tokens_per_rank: int, ms: float) -> float:
        return self.world * tokens_per_rank / (ms / 1e3)

    def close(self):
        if self.world > 1 and self.dist.is_initialized():
            self.dist.destroy_process_group()


# ----------------------------------------------------------------- ours ---

# streamed[_S<slots>][_T<tokens>] and no_h2d_T<tokens>
_POOL_MODE = re.compile(r"^(streamed|no_h2d)(?:_S(\d+))?(?:_T(\d+))?$")

def run_ours(args):
    import torch
    from layer_streamed_nf4_b200 import lsnf4, synth
    from layer_streamed_nf4_b200.stack import HostIO, Stack

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    reps = Replicas("nccl", torch.device("cuda", local))
    cfg = synth.STACKS[WORKLOAD]
    T = args.tokens or cfg.tokens
    L = args.layers or cfg.layers
    args.slots = max(1, min(args.slots, L))
    stream = torch.cuda.Stream()
    peaks = _peaks()

    barrier = reps.barrier
    max_over_ranks = reps.max

    def train_step(st, micro=1, **kw):
        """One step of the path (micro > 1: that many micro-batches, the adapter gradients accumulated over
        them), then (N > 1) the adapter gradients summed over the replicas."""
        for i in range(micro):
            st.step(accumulate=i > 0, **kw)
        reps.allreduce_sum(st.grads)

    results = {}
    host_issue = {}
    kernel = None
    pool_stats = None
    clocks = None
    st_main = Stack(cfg, layers=L, tokens=T, mode="streamed", n_slots=args.slots, seed=synth.SEED + rank,
                    stream=stream, lanes=args.lanes, api=args.api,
                    dequant_ahead=bool(args.dequant_ahead))
    wanted = [m for m in args.modes.split(",") if m]
    modes = ["streamed"] + [m for m in wanted
                            if m in ("no_h2d", "resident", "proj", "dpo", "recompute", "shared", "grouped",
                                     "bf16_base")
                            or _POOL_MODE.match(m) or m.startswith("accum")]
    mode_tokens = {m: T for m in modes}
    mode_copies = {}
    # Extra work of the step variants: the reference forward of preference
    # training (base term only) and the recomputed forward of checkpointing.
    base_flop = 2.0 * sum(K * N for _, K, N in cfg.projections) * T * L
    fwd_flop = base_flop + 2.0 * cfg.rank * sum(K + N for _, K, N in cfg.projections) * T * L
    mode_kwargs = {"dpo": {"reference": True}, "recompute": {"recompute": True}}
    for mode in modes:
        kw = mode_kwargs.get(mode, {})
        if mode == "streamed":
            st = st_main
        elif mode == "proj":            # no_h2d through the per-projection calls on two lanes
            st = st_main.with_mode("no_h2d", lanes=2, api="proj")
        elif _POOL_MODE.match(mode) and mode not in ("no_h2d",):
            # streamed_S<n>: the same stream of weights through a pool of n slots; _T<n>: under a batch of
            # n tokens (its own activations); no_h2d_T<n>: the pre-filled pool under that batch
            m = _POOL_MODE.match(mode)
            pool_mode = m.group(1)
            slots = int(m.group(2)) if m.group(2) else args.slots
            if m.group(3):
                mode_tokens[mode] = int(m.group(3))
                st = st_main.with_tokens(mode_tokens[mode], pool_mode, n_slots=slots)
            else:
                st = st_main.with_mode(pool_mode, n_slots=slots)
        elif mode.startswith("accum"):        # n micro-batches of T tokens per step, gradients accumulated
            kw = {"micro": int(mode[len("accum"):])}
            mode_tokens[mode] = kw["micro"] * T
            st = st_main.with_mode("streamed", n_slots=args.slots)
        elif mode in ("dpo", "recompute"):    # step variants over the same streamed pool
            st = st_main.with_mode("streamed", n_slots=args.slots)
        elif mode in ("shared", "grouped"):   # q|k|v and gate|up read one input each (no_h2d pool)
            st = st_main.with_inputs(shared_inputs=True, grouped=(mode == "grouped"))
        elif mode == "bf16_base":             # the same shapes with a bf16 base: no NF4 conversion at all (no_h2d)
            import dataclasses
            st = Stack(dataclasses.replace(cfg, base="bf16"), layers=L, tokens=T, mode="no_h2d",
                       seed=synth.SEED + rank, stream=stream, lanes=args.lanes, api=args.api)
        else:
            st = st_main.with_mode(mode)
        # Clocks of the value's mode: the sampler starts before the warm-up
        # (nvidia-smi needs a moment to start), so the timed steps are covered.
        sampler = ClockSampler(local) if mode == "streamed" else None
        if sampler:
            sampler.__enter__()
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                train_step(st, **kw)
        stream.synchronize()
        barrier()
        torch.cuda.synchronize()
        ps0_mode = st.pool_stats()
        if mode == "streamed":
            ps0 = ps0_mode
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            h0 = time.perf_counter()
            for _ in range(args.steps):
                train_step(st, **kw)
            host_ms = (time.perf_counter() - h0) * 1e3 / args.steps
            t1.record(stream)
        t1.synchronize()
        host_issue[mode] = host_ms
        if sampler:
            sampler.__exit__()
            clocks = sampler.summary()
        torch.cuda.synchronize()
        barrier()
        ms = t0.elapsed_time(t1) / args.steps
        ms = max_over_ranks(ms)
        results[mode] = ms
        ps1_mode = st.pool_stats()
        if ps0_mode and ps1_mode:
            mode_copies[mode] = (ps1_mode["copies"] - ps0_mode["copies"]) / args.steps
        if mode == "streamed":
            ps1 = st.pool_stats()
            pool_stats = {k: ps1[k] - ps0[k] for k in ps1}
            # Second timed region, same steps, every library launch bracketed
            # by CUDA events on its stream: per-kernel device time and work.
            # (The events cost host time, so the step time above is taken
            # without them.)  It runs with one lane, so that no launch waits
            # for SMs held by another lane's kernel inside its events; the
            # dequantisation one layer ahead runs on that lane too, so the
            # layer calls get bf16 bases (and launch the same GEMMs) as in the
            # timed steps.
            st_k = st.with_mode("streamed", n_slots=args.slots, lanes=1)
            st_k.ahead_on_compute_stream()
            lanes_opt = lsnf4.get_option(lsnf4.LSN_OPT_LAYER_LANES)
            lsnf4.set_option(lsnf4.LSN_OPT_LAYER_LANES, 1)
            try:
                with torch.cuda.stream(stream):
                    train_step(st_k)
                stream.synchronize()
                barrier()
                lsnf4.timing_enable(True)
                with torch.cuda.stream(stream):
                    for _ in range(args.steps):
                        train_step(st_k)
                stream.synchronize()
                kernel = lsnf4.timing_read()
                lsnf4.timing_enable(False)
            finally:
                lsnf4.set_option(lsnf4.LSN_OPT_LAYER_LANES, lanes_opt)
            st_k.check_status()
            st_k.close()
            barrier()
        st.check_status()
        if st is not st_main:
            st.close()
            st = None
            torch.cuda.empty_cache()

    # End to end through the public API with host buffers: every step copies
    # its input hidden states (layer-0 projection inputs) from pinned host
    # memory and its result (layer-0 input gradients) back, on a copy stream
    # that overlaps each transfer with the neighbouring step's compute
    # (stack.HostIO); the first step's inputs and the last step's result are
    # inside the timed region too.
    e2e = None
    if not args.no_e2e:
        st = st_main
        h_in, h_out = HostIO.host_buffers(st)
        io = HostIO(st, h_in, h_out, stream=stream)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ps0 = st.pool_stats() or {"bytes_copied": 0}
        with torch.cuda.stream(stream):
            e0.record(stream)
            io.run(args.steps, lambda: train_step(st))
            e1.record(stream)
        e1.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        ps = st.pool_stats() or {"bytes_copied": 0}
        e2e = {"value": reps.throughput(T, ems), "unit": UNIT,
               "h2d_bytes_per_step": int(io.bytes_in() + (ps["bytes_copied"] - ps0["bytes_copied"]) / max(args.steps, 1)),
               "d2h_bytes_per_step": int(io.bytes_out()), "ms_per_step": ems,
               "transfers": "inputs and result of every step over PCIe, overlapped with the neighbouring steps"}

    st_main.check_status()
    reps.close()
    if rank != 0:
        st_main.close()
        return

    ms = results["streamed"]
    flop_step = st_main.flop_per_step()
    value = reps.throughput(T, ms)

    g = {k: kernel[k] for k in ("gemm_fwd", "gemm_bwd")}
    g_ms = sum(v["ms"] for v in g.values())
    g_flop = sum(v["work"] for v in g.values())
    g_launch = sum(v["launches"] for v in g.values())
    achieved = g_flop / (g_ms / 1e3) / 1e12 if g_ms > 0 else 0.0
    peak = peaks["bf16_tflops_sustained"]
    launches = sum(v["kernels"] for v in kernel.values())
    step_kernel_ms = sum(v["ms"] for v in kernel.values()) / args.steps
    dq = kernel["dequant"]
    h2d_gbs = (pool_stats["bytes_copied"] / (pool_stats["copy_ms"] / 1e3) / 1e9
               if pool_stats and pool_stats["copy_ms"] > 0 else None)
    def mode_flop_per_step(m):
        f = flop_step * mode_tokens[m] / T
        if m == "dpo":
            f += base_flop
        elif m == "recompute":
            f += fwd_flop
        return f

    extra_modes = {m: {"ms_per_step": results[m], "host_issue_ms_per_step": host_issue.get(m),
                       "tokens": mode_tokens[m],
                       "tok_s": world * mode_tokens[m] / (results[m] / 1e3),
                       "flop_per_step": mode_flop_per_step(m),
                       "pct_bf16_peak": 100 * mode_flop_per_step(m) / (results[m] / 1e3) / 1e12 / peaks["bf16_tflops"],
                       "layer_copies_per_step": mode_copies.get(m)}
                   for m in results}
    traffic = _traffic_from_profile()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(cfg, T, L, args.slots, world),
                   "api": args.api,
                   "lanes": args.lanes if args.api == "proj" else 1,
                   "nf4_conversion": {0: "nf4_dequant then bf16 GEMM",
                                      1: "inside the GEMM (shared memory), both directions",
                                      2: "forward: inside the GEMM (tensor memory); backward: nf4_dequant then "
                                         "bf16 GEMM"}[args.fused_nf4],
                   "programmatic_dependent_launch": not args.no_pdl,
                   "gemm_schedule": gemm_schedule(args),
                   "dequant_spare_sms": args.dequant_spare_sms,
                   "dequant_ahead": st_main.ahead,
                   "l2": "inputs larger than L2 (per step ~11 GB of activations; every layer's NF4 codes read twice)"},
        "pct_bf16_peak": 100 * flop_step / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        "flop_per_step": flop_step,
        "modes": extra_modes,
        "roofline": {"bound": "tensor", "kernel": "lsn_gemm_kernel (fwd y and bwd dX GEMMs)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel timed inside a long step)",
                     "frac_of_burst": achieved / peaks["bf16_tflops"],
                     "launches": g_launch, "flop_per_launch": g_flop / max(g_launch, 1),
                     "ms_per_launch": g_ms / max(g_launch, 1),
                     "traffic": traffic},
        "kernels": {k: {"launches": v["launches"], "ms_per_step": v["ms"] / args.steps,
                        "share_of_kernel_time": v["ms"] / max(sum(x["ms"] for x in kernel.values()), 1e-9)}
                    for k, v in kernel.items() if v["launches"]},
        "dequant_share_of_step": dq["ms"] / args.steps / ms,
        "pool": {"h2d_gbs": h2d_gbs, "bytes_per_step": pool_stats["bytes_copied"] / args.steps if pool_stats else 0,
                 "copies_per_step": pool_stats["copies"] / args.steps if pool_stats else 0,
                 "exposed_copy_ms": ms - results["no_h2d"] if "no_h2d" in results else None},
        "step_kernel_ms": step_kernel_ms,
        "peak_mem_gb": torch.cuda.max_memory_allocated() / 1e9,
        "gpu_launches": launches,
        "gpu": torch.cuda.get_device_name(local),
        "clocks": clocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        rows = max(args.cpu_rows, os.cpu_count() or 1)
        line["cpu_baseline"] = cpu_baseline(args, sample_rows=rows, budget_s=args.cpu_budget)
    st_main.close()
    print(json.dumps(line))


def _traffic_from_profile():
    """DRAM bytes per GEMM launch from the committed ncu summary, if it records one for this kernel build."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d.get("gemm_dram_bytes_per_launch")
    except Exception:
        return None


# ------------------------------------------------------------ reference ---

_ORACLE_CASES = {}


def _oracle_cases(sample_rows: int):
    """Inputs of the oracle sample: `sample_rows` token rows of the workload's distributions for each of the
    seven projections of one layer, weights NF4 through the oracle's own quantiser (built once, untimed)."""
    import oracle
    from layer_streamed_nf4_b200 import synth
    if sample_rows not in _ORACLE_CASES:
        cfg = synth.STACKS[WORKLOAD]
        cases = []
        for pi, (name, K, N) in enumerate(cfg.projections):
            c = synth.linear_case(sample_rows, K, N, cfg.rank, cfg.alpha, seed=synth.SEED, layer=0, proj=pi)
            q = oracle.nf4_quantize(c.W)
            Wb = oracle.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], c.W.size).reshape(N, K)
            cases.append((c, Wb))
        _ORACLE_CASES[sample_rows] = cases
    return _ORACLE_CASES[sample_rows]


def cpu_baseline(args, sample_rows: int, budget_s: float):
    """The oracle (fp64, plain loops, OpenMP over rows) on a bounded sample: `sample_rows` token rows through
    the seven projections of one 8B-shaped layer, fwd + bwd.  Step time per token is scaled by the layer count
    (derived, arithmetic)."""
    import oracle
    from layer_streamed_nf4_b200 import synth
    cfg = synth.STACKS[WORKLOAD]
    L = cfg.layers
    cores = oracle.threads()                          # the threads its OpenMP loops actually use
    cases = _oracle_cases(sample_rows)
    work_all = sum(c.K * c.N for c, _ in cases)
    work_done = 0
    t0 = time.perf_counter()
    for c, Wb in cases:
        oracle.lora_fwd(c.x, Wb, c.A, c.B, c.scale)
        oracle.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale)
        oracle.lora_bwd_dadb(c.x, c.dY, c.A, c.B, c.scale)
        work_done += c.K * c.N
        if time.perf_counter() - t0 > budget_s:     # out of budget: scale by the share of the layer done
            break
    t_total = time.perf_counter() - t0
    rows_done = sample_rows
    s_per_token_step = t_total / rows_done * L * (work_all / work_done)
    return {"value": 1.0 / s_per_token_step, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{rows_done} token rows through the 7 projections of one {cfg.name} layer (fwd+bwd, "
                      f"fp64 oracle, OpenMP); per-step time = layer time x {L} layers (derived, arithmetic)",
            "seconds": t_total}


def gemm_schedule(args) -> str:
    """The GEMM schedule in force, as the library reports it."""
    from layer_streamed_nf4_b200 import lsnf4
    if lsnf4.get_option(lsnf4.LSN_OPT_STREAM_K):
        text = "stream-K where tiles leave the last round partly empty"
    elif lsnf4.get_option(lsnf4.LSN_OPT_GEMM_TAIL_SPLIT):
        text = "whole tiles round robin, the last partial round cut into 64-column quanta (128 for MN-major W)"
    else:
        text = "whole tiles round robin"
    if lsnf4.get_option(lsnf4.LSN_OPT_GEMM_MIN_UNITS):
        text += ", on the fewest SMs for the same rounds"
    if lsnf4.get_option(lsnf4.LSN_OPT_LAYER_MERGE):
        text = ("layer calls: projection 0's GEMM, then projections 1..n-1 as one launch with a balanced "
                "schedule of whole tiles; single GEMMs: " + text)
    return text


def workload_config(cfg, T: int, L: int, slots: int, world: int) -> dict:
    """The workload both arms report (the reference arm times a bounded sample of it, stated in its
    cpu_baseline)."""
    return {"workload": f"{cfg.name} NF4 LoRA stack: {L} layers x 7 projections (q,k,v,o,gate,up,down), "
                        f"T={T} tokens (batch 1 x seq {T}), r={cfg.rank}, alpha={cfg.alpha:g}, "
                        f"base NF4 blk-64 + double quant streamed from pinned host RAM, "
                        f"{slots}-slot VRAM pool ({L} layers)",
            "tokens": T, "layers": L, "rank": cfg.rank, "pool_slots": slots, "base": cfg.base,
            "parallelism": f"dp{world}" + (" (adapter gradients summed over ranks each step)" if world > 1 else "")}


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return
    from layer_streamed_nf4_b200 import synth
    cfg = synth.STACKS[WORKLOAD]
    vals = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(args, sample_rows=max(args.ref_rows, os.cpu_count() or 1), budget_s=1e9)
        if i >= args.warmup:
            vals.append(cb)
    v = statistics.median(c["value"] for c in vals)
    s_step = sum(c["seconds"] for c in vals) / len(vals)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": s_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(cfg, cfg.tokens, cfg.layers, min(getattr(args, "slots", 20), cfg.layers), world),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def run_case(args):
    """One projection of the 8B-shaped stack, lora_linear_fwd + lora_linear_bwd, NF4 base, repeated: the small,
    self-contained launch sequence used for focused profiles (prints its own JSON line)."""
    import torch
    from layer_streamed_nf4_b200 import lsnf4, synth
    cfg = synth.STACKS[WORKLOAD]
    proj = {name: (pi, K, N) for pi, (name, K, N) in enumerate(cfg.projections)}
    pi, K, N = proj[args.case]
    T, r = args.tokens or cfg.tokens, cfg.rank
    scale = cfg.alpha / r
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    W = synth.device_normal((N, K), 0.02, synth.SEED, 0, pi, synth.T_W, device=dev)
    blob = torch.zeros(lsnf4.nf4_blob_bytes(N, K), dtype=torch.uint8, device=dev)
    w = lsnf4.nf4_weight_in_blob(N, K, blob.data_ptr())
    qws = torch.zeros(lsnf4.nf4_quantize_ws_bytes(N, K), dtype=torch.uint8, device=dev)
    lsnf4.nf4_quantize(W, w, qws, qws.numel())
    del W, qws
    base = lsnf4.base_nf4(w)
    x = synth.device_normal((T, K), 1.0, synth.SEED, 0, pi, synth.T_X, device=dev, dtype=torch.bfloat16)
    dY = synth.device_normal((T, N), 1.0, synth.SEED, 0, pi, synth.T_DY, device=dev, dtype=torch.bfloat16)
    A = synth.device_uniform((r, K), 1.0 / K ** 0.5, synth.SEED, 0, pi, synth.T_A, device=dev, dtype=torch.bfloat16)
    B = synth.device_normal((N, r), 0.01, synth.SEED, 0, pi, synth.T_B, device=dev, dtype=torch.bfloat16)
    y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dA = torch.zeros((r, K), dtype=torch.float32, device=dev)
    dB = torch.zeros((N, r), dtype=torch.float32, device=dev)
    nbytes = lsnf4.lora_ws_bytes(T, K, N, r, lsnf4.LSN_BASE_NF4)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)

    def one():
        lsnf4.lora_linear_fwd(base, x, T, A, B, r, scale, y, ws, nbytes)
        lsnf4.lora_linear_bwd(base, x, dY, T, A, B, r, scale, dX, dA, dB, False, ws, nbytes)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        one()
    e1.record()
    e1.synchronize()
    lsnf4.ws_status(ws)
    ms = e0.elapsed_time(e1) / args.steps
    flop = 2.0 * T * N * (K + r) + 2.0 * T * K * (N + r)
    print(json.dumps({"case": args.case, "T": T, "K": K, "N": N, "r": r, "ms_fwd_bwd": ms,
                      "gemm_tflops_if_all_time_were_gemm": flop / (ms / 1e3) / 1e12}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tokens", type=int, default=0, help="override T (default: the workload's 2048)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (default 32)")
    ap.add_argument("--slots", type=int, default=24,
                    help="VRAM pool slots of the timed stream (default 24 of 32 layers: the smallest measured "
                         "window that hides the copies behind compute at 2048 tokens on one B200)")
    ap.add_argument("--modes", default="no_h2d,resident,proj,streamed_S2,streamed_T8192,streamed_S2_T8192,"
                                       "no_h2d_T8192,accum4,dpo,recompute,shared,grouped,bf16_base",
                    help="extra modes timed after the streamed one (streamed_T<n>: streamed with n tokens; "
                         "streamed_S<n>: streamed through n pool slots; streamed_S<n>_T<m>: both; no_h2d_T<n>: "
                         "the pre-filled pool with n tokens; accum<n>: n micro-batches per step, gradients "
                         "accumulated; bf16_base: the same shapes with an un-quantised base, the bound on what "
                         "any NF4 conversion scheme can save)")
    ap.add_argument("--api", choices=["layer", "proj"], default="layer",
                    help="one library call per layer, or one per projection")
    ap.add_argument("--lanes", type=int, default=2, help="streams the seven projections of a layer are spread over")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=768, help="token rows of the timed oracle sample")
    ap.add_argument("--cpu-budget", type=float, default=60.0)
    ap.add_argument("--ref-rows", type=int, default=64, help="token rows per step of the reference arm")
    ap.add_argument("--fused-nf4", type=int, default=0, choices=[0, 1, 2],
                    help="NF4 conversion: 0 = nf4_dequant then the bf16 GEMM; 1 = inside the GEMM into shared "
                         "memory (both directions); 2 = inside the forward GEMM into tensor memory")
    ap.add_argument("--no-pdl", action="store_true", help="ordinary launches instead of programmatic dependent ones")
    ap.add_argument("--gemm-min-units", type=int, default=0, choices=[0, 1],
                    help="persistent GEMMs on every SM (0, default) or on the fewest SMs that finish in the same "
                         "number of tile rounds (1)")
    ap.add_argument("--dequant-spare-sms", type=int, default=0,
                    help="run the dequantisation-ahead on SMs of its own, sized for this many SMs left free by "
                         "the GEMMs (0: beside the GEMM CTAs, the capped grid of the dequantisation ahead)")
    ap.add_argument("--layer-merge", type=int, default=-1, choices=[-1, 0, 1],
                    help="run projections 1..n-1 of each layer call as one merged GEMM launch (1) or one launch per "
                         "projection (0); -1 (default): the library's default")
    ap.add_argument("--tail-split", type=int, default=-1, choices=[-1, 0, 1],
                    help="GEMM schedule: cut the tiles of a partly filled last round into 64-column quanta shared "
                         "evenly over the SM pairs (1) or not (0); -1 (default): the library's default")
    ap.add_argument("--stream-k", type=int, default=0, choices=[0, 1],
                    help="GEMM schedule: whole tiles round robin (0, default), or stream-K where tiles leave the "
                         "last wave partly empty (1)")
    ap.add_argument("--dequant-ahead", type=int, default=1, choices=[0, 1],
                    help="dequantise each layer on a side stream one layer ahead (1, default) or inside the layer call")
    ap.add_argument("--case", default="", help="profile one 8B projection (q,k,v,o,gate,up,down) instead of the stack")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "ours" and (args.fused_nf4 or args.no_pdl or args.stream_k or args.gemm_min_units
                                or args.dequant_spare_sms or args.tail_split >= 0 or args.layer_merge >= 0):
        from layer_streamed_nf4_b200 import lsnf4
        if args.layer_merge >= 0:
            lsnf4.set_option(lsnf4.LSN_OPT_LAYER_MERGE, args.layer_merge)
        if args.tail_split >= 0:
            lsnf4.set_option(lsnf4.LSN_OPT_GEMM_TAIL_SPLIT, args.tail_split)
        lsnf4.set_option(lsnf4.LSN_OPT_GEMM_MIN_UNITS, args.gemm_min_units)
        lsnf4.set_option(lsnf4.LSN_OPT_DEQUANT_SPARE_SMS, args.dequant_spare_sms)
        if args.fused_nf4:
            lsnf4.set_option(lsnf4.LSN_OPT_FUSED_NF4, args.fused_nf4)
        if args.no_pdl:
            lsnf4.set_option(lsnf4.LSN_OPT_PDL, 0)
        if args.stream_k:
            lsnf4.set_option(lsnf4.LSN_OPT_STREAM_K, 1)
    if args.impl == "reference":
        run_reference(args)
    elif args.case:
        run_case(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
