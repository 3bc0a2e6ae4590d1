"""The bit-exactness gate at the workloads' stated depth.

"Exact Layer Streaming" (abstract) claims a streamed run equal to a resident
run of the same numerics, forward and backward checked separately, and the
Soup benchmarks README (v0.73.0, protocol notes and gate ledger) reports why
depth matters: the pages' aliasing defect left the forward exact while the
gradients were wrong on 62 of 64 and 78 of 80 layers of the big NF4 stacks,
and the repaired gate was re-run over every layer (320/320 at 72B).  Here
each workload is gated over all of its layers: the Qwen2.5-3B shape (36 bf16
layers), the Llama-3.1-8B shape in the exact configuration the benchmark
times (32 NF4 layers, 2048 tokens, whole-layer calls on two lanes,
dequantisation one layer ahead, a 24-slot pool, and 20 slots) and with the pages' two
slots, and the Qwen2.5-72B shape (80 NF4 layers of ~432 MiB through a
2-slot pool, every layer's adapter gradients).  Resident = the same blobs
copied once into one device buffer and driven by the same launches."""
import pytest

from layer_streamed_nf4_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from layer_streamed_nf4_b200 import lsnf4
    return lsnf4


def _snapshot(st):
    """Copies of every output the step leaves: the flat adapter-gradient buffer (every dA and dB of every
    layer) and the y / dX buffers (every layer with keep_outputs, else the last ones written)."""
    return {"grads": st.grads.clone(),
            "y": {k: v.clone() for k, v in st.y.items()},
            "dX": {k: v.clone() for k, v in st.dX.items()}}


def _layers_differing(st, snap):
    """(forward equal?, input gradients equal?, layers whose dA or dB differ)."""
    import torch
    fwd = all(torch.equal(st.y[k], snap["y"][k]) for k in st.y)
    dx = all(torch.equal(st.dX[k], snap["dX"][k]) for k in st.dX)
    bad = []
    for l in range(st.L):
        lo = st.grad_offsets[l, 0]
        hi = st.grad_offsets[l + 1, 0] if l + 1 < st.L else st.grads.numel()
        if not torch.equal(st.grads[lo:hi], snap["grads"][lo:hi]):
            bad.append(l)
    return fwd, dx, bad


def _gate(cfg, tokens, slot_list, keep_outputs=True, distinct=True, steps=2):
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    res = Stack(cfg, tokens=tokens, mode="resident", keep_outputs=keep_outputs, distinct_activations=distinct)
    res.step()
    torch.cuda.synchronize()
    res.check_status()
    snap = _snapshot(res)
    assert float(snap["grads"].abs().sum()) > 0
    for slots in slot_list:
        st = res.with_mode("streamed", n_slots=slots)
        for g in (st.grads, *st.y.values(), *st.dX.values()):
            g.fill_(float("nan"))                        # nothing of the resident run can pass for a result
        c0 = st.pool_stats()["copies"]
        for _ in range(steps):                           # no accumulation: every step's gradients are the same
            st.step()
        torch.cuda.synchronize()
        st.check_status()
        copies = st.pool_stats()["copies"] - c0
        L = cfg.layers
        assert copies == (2 * L - slots) + (steps - 1) * (2 * L - 2 * slots), (slots, copies)
        fwd, dx, bad = _layers_differing(st, snap)
        assert fwd, f"{cfg.name}, {slots} slots: streamed forward differs from resident"
        assert dx and not bad, f"{cfg.name}, {slots} slots: streamed backward differs on layers {bad}"
        st.close()
    res.close()


def test_gate_3b_every_layer(lib):
    """Qwen2.5-3B shape, bf16 base, 36 layers, 1024 tokens: every y, dX, dA, dB of every layer, through the
    pages' two-slot pool and through a 6-slot one."""
    _gate(synth.STACKS["3b"], 1024, (2, 6))


def test_gate_8b_benchmark_configuration(lib):
    """The configuration the benchmark times: Llama-3.1-8B shape, NF4, 32 layers, 2048 tokens, whole-layer
    calls on two lanes, dequantisation one layer ahead, 24 pool slots (and 20); and the same with the pages'
    two slots.  Every y, dX, dA, dB of every layer equals the resident run's."""
    from layer_streamed_nf4_b200.stack import Stack
    cfg = synth.STACKS["8b"]
    assert cfg.layers == 32 and cfg.tokens == 2048
    probe = Stack(cfg, layers=1, tokens=64, mode="streamed")
    assert probe.ahead and probe.api == "layer" and lib.get_option(lib.LSN_OPT_LAYER_LANES) == 2
    probe.close()
    _gate(cfg, 2048, (24, 20, 2))


def test_gate_72b_every_layer(lib):
    """Qwen2.5-72B shape, NF4 (~432 MiB per layer blob), 80 layers, 1024 tokens, through the pages'
    two-slot pool: every layer's dA and dB equal the resident run's (the gradients the pages found wrong on
    78 of 80 layers before their repair), and so do the last layer's y and the first layer's dX (the
    buffers of the other layers are reused; all layers share one set of activations, so ~35 GB of blobs
    stay the only large allocation)."""
    import torch
    cfg = synth.STACKS["72b"]
    assert cfg.layers == 80
    free, _ = torch.cuda.mem_get_info()
    assert free > 60e9, f"needs ~45 GB of device memory, {free / 1e9:.1f} GB free"
    _gate(cfg, 1024, (2,), keep_outputs=False, distinct=False)
