"""The layer pool and the bit-exactness gate.

"Exact Layer Streaming" (abstract) gates streaming on bit-exactness against a
resident run of the same numerics, forward and backward as two separate
claims, and reports an aliasing defect that left the forward exact while the
gradients were wrong on most layers above ~165 MiB per NF4 layer (the Soup
benchmarks README, protocol notes).  Here: streamed == resident with
torch.equal for every y and dX of every projection and every dA/dB of every
layer, on stacks of each workload shape (the 72B-shaped layer is ~432 MiB),
plus a planted aliasing fault that the gate must catch, and host-side fault
injection."""
import pytest

from layer_streamed_nf4_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from layer_streamed_nf4_b200 import lsnf4
    return lsnf4


def _run(cfg, layers, tokens, mode, fault=None, steps=1, lanes=2, api="layer"):
    import torch
    from layer_streamed_nf4_b200 import lsnf4
    from layer_streamed_nf4_b200.stack import Stack
    st = Stack(cfg, layers=layers, tokens=tokens, mode=mode, keep_outputs=True, lanes=lanes, api=api)
    if fault is not None:
        lsnf4.layer_pool_inject_fault(st.pool, fault)
    for _ in range(steps):
        st.step()
    torch.cuda.synchronize()
    st.check_status()
    return st


def _compare(a, b):
    """(forward equal?, backward equal?, list of layers whose dA/dB differ)."""
    import torch
    fwd = all(torch.equal(a.y[k], b.y[k]) for k in a.y)
    bad = sorted({l for (l, pi) in a.dA if not (torch.equal(a.dA[l, pi], b.dA[l, pi]) and
                                                torch.equal(a.dB[l, pi], b.dB[l, pi]))})
    bwd = not bad and all(torch.equal(a.dX[k], b.dX[k]) for k in a.dX)
    return fwd, bwd, bad


@pytest.mark.parametrize("name,layers,tokens,fused", [("0.5b", 24, 512, 0), ("8b", 4, 2048, 0), ("8b", 3, 2048, 1),
                                                     ("8b", 3, 2048, 2), ("72b", 3, 1024, 0)])
def test_streamed_equals_resident(lib, name, layers, tokens, fused):
    """Resident through the per-projection calls on one stream, streamed through the layer calls (whose
    bases arrive dequantised one layer ahead).  With the NF4 conversion inside the GEMM (1: in shared
    memory, both directions; 2: in tensor memory, forward only, the forward sweep then passes the codes
    themselves) the fused GEMMs run whole tiles: the other GEMMs then take whole tiles too."""
    from tests.helpers import lib_option
    with lib_option(lib, lib.LSN_OPT_FUSED_NF4, fused), lib_option(lib, lib.LSN_OPT_STREAM_K, 0 if fused else 1):
        _streamed_equals_resident(lib, name, layers, tokens)


def _streamed_equals_resident(lib, name, layers, tokens):
    cfg = synth.STACKS[name]
    res = _run(cfg, layers, tokens, "resident", lanes=1, api="proj")   # per-projection calls on one stream
    stm = _run(cfg, layers, tokens, "streamed", steps=2)              # whole-layer calls
    fwd, bwd, bad = _compare(stm, res)
    assert fwd, f"{name}: streamed forward differs from resident"
    # two streamed steps without accumulation: gradients are those of one step
    assert bwd, f"{name}: streamed backward differs from resident on layers {bad}"
    s = stm.pool_stats()
    assert s["copies"] == (2 * layers - 2) + (2 * layers - 4), s   # first step 2L-2, steady state 2L-4
    stm.close()


@pytest.mark.parametrize("name,layers,tokens", [("0.5b", 4, 512), ("8b", 2, 1024)])
def test_lane_count_does_not_change_results(lib, name, layers, tokens):
    """The projections of a layer issued on 1, 2 or 3 streams, or as one layer call, give the same bits."""
    cfg = synth.STACKS[name]
    one = _run(cfg, layers, tokens, "no_h2d", lanes=1, api="proj")
    whole = _run(cfg, layers, tokens, "no_h2d", api="layer")
    fwd, bwd, bad = _compare(whole, one)
    assert fwd and bwd, ("layer call", bad)
    whole.close()
    for lanes in (2, 3):
        many = _run(cfg, layers, tokens, "no_h2d", lanes=lanes, api="proj")
        fwd, bwd, bad = _compare(many, one)
        assert fwd and bwd, (lanes, bad)
        many.close()
    one.close()


def _oracle_weight(orc, st, l, pi):
    """The oracle's dequantised bf16 bits of projection pi of layer l: the stack's fp32 weight regenerated
    from its seed, quantised and dequantised by the oracle itself."""
    p = st.proj[pi]
    W = synth.device_normal((p.N, p.K), 0.02, st.seed, l, pi, synth.T_W, device=st.dev).cpu().numpy()
    q = orc.nf4_quantize(W)
    return orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size).reshape(W.shape)


def _bits(t):
    import numpy as np
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_recompute_and_reference_steps(lib, orc):
    """A backward that recomputes each layer's forward, and a step that first runs the adapter-off
    reference forward, give the same y, dX, dA, dB as the plain step, and match the oracle: the
    recomputing step's dA, dB (in full) and dX (sampled token rows), and the reference forward's y
    against the oracle's plain x W^T.  The reference outputs are also the base term bit for bit (equal to
    an adapter-on forward with B = 0)."""
    import numpy as np
    import torch
    from tests.helpers import assert_close, bf16_tensor_to_f64
    cfg = synth.STACKS["8b"]
    plain = _run(cfg, 3, 256, "streamed")
    from layer_streamed_nf4_b200.stack import Stack
    st = Stack(cfg, layers=3, tokens=256, mode="streamed", keep_outputs=True)
    st.step(reference=True, recompute=True)
    torch.cuda.synchronize()
    st.check_status()
    assert st.pool_stats()["copies"] == 2 * 3 - 2        # the reference forward reads no layer of its own
    fwd, bwd, bad = _compare(st, plain)
    assert fwd and bwd, bad
    rows = np.sort(np.random.default_rng(31).choice(256, size=24, replace=False))
    for l in range(3):
        for pi in (0, 2, 6):                                  # q, v, down
            Wb = _oracle_weight(orc, st, l, pi)
            x, dY, A, B = _bits(st.x[l, pi]), _bits(st.dY[l, pi]), _bits(st.A[l, pi]), _bits(st.B[l, pi])
            rA, rB = orc.lora_bwd_dadb(x, dY, A, B, st.scale)
            assert_close(st.dA[l, pi].cpu().numpy(), rA, f"recompute dA {l},{pi}")
            assert_close(st.dB[l, pi].cpu().numpy(), rB, f"recompute dB {l},{pi}")
            assert_close(bf16_tensor_to_f64(st.dX[l, pi])[rows], orc.lora_bwd_dx(dY, Wb, A, B, st.scale, rows=rows),
                         f"recompute dX {l},{pi}")
            base = orc.lora_fwd(x, Wb, A, np.zeros_like(B), st.scale, rows=rows)      # x W^T alone
            assert_close(bf16_tensor_to_f64(st.y_ref[l, pi])[rows], base, f"reference y {l},{pi}")
    for k in st.B:
        st.B[k].zero_()
    st.forward()
    torch.cuda.synchronize()
    assert all(torch.equal(st.y[k], st.y_ref[k]) for k in st.y)
    st.close()
    plain.close()


@pytest.mark.parametrize("mode", ["streamed", "no_h2d"])
def test_dequant_ahead_gives_the_same_bits(lib, mode):
    """Dequantising each layer on a side stream one layer ahead (bf16 bases into the layer calls) and
    dequantising inside the layer calls give the same bits."""
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    cfg = synth.STACKS["8b"]
    inside = Stack(cfg, layers=3, tokens=256, mode=mode, keep_outputs=True, dequant_ahead=False)
    ahead = Stack(cfg, layers=3, tokens=256, mode=mode, keep_outputs=True, dequant_ahead=True)
    assert ahead.ahead and not inside.ahead
    default = Stack(cfg, layers=2, tokens=64, mode=mode)
    assert default.ahead and default.with_mode("resident").ahead
    assert not default.with_mode("no_h2d", api="proj").ahead or default.with_mode("no_h2d", api="proj").api == "proj"
    default.close()
    for st in (inside, ahead):
        st.step()
        st.step(reference=True, recompute=True)
    torch.cuda.synchronize()
    ahead.check_status()
    fwd, bwd, bad = _compare(ahead, inside)
    assert fwd and bwd, bad
    assert all(torch.equal(ahead.y_ref[k], inside.y_ref[k]) for k in ahead.y_ref)
    inside.close()
    ahead.close()


def test_resident_constants_give_the_same_bits(lib):
    """Streaming only the packed codes (constants kept in device memory) and streaming whole NF4 blobs give
    the same bits; the pool then copies the codes alone."""
    cfg = synth.STACKS["8b"]
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    runs = []
    for rc in (False, True):
        st = Stack(cfg, layers=3, tokens=256, mode="streamed", keep_outputs=True, resident_constants=rc)
        st.step()
        torch.cuda.synchronize()
        st.check_status()
        runs.append(st)
    whole, codes = runs
    fwd, bwd, bad = _compare(codes, whole)
    assert fwd and bwd, bad
    assert codes.const_bytes > 0 and whole.const_bytes == 0
    assert codes.layer_bytes + codes.const_bytes == whole.layer_bytes
    assert codes.layer_bytes == sum(p.N * p.K // 2 for p in codes.proj)       # 8B shapes: no padding
    for st in runs:
        s = st.pool_stats()
        assert s["bytes_copied"] == s["copies"] * st.layer_bytes, s
        st.close()


def test_first_layer_reads_token_embeddings(lib):
    """0.5B workload: the layer-0 inputs of q, k and v are the rows of the resident embedding table that
    the token ids pick; the ids cover the vocabulary uniformly."""
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    cfg = synth.STACKS["0.5b"]
    st = Stack(cfg, layers=2, tokens=512, mode="streamed")
    ids = st.token_ids
    assert ids.shape == (512,) and int(ids.min()) >= 0 and int(ids.max()) < cfg.vocab
    assert abs(float(ids.double().mean()) / cfg.vocab - 0.5) < 0.05
    assert st.embedding.shape == (cfg.vocab, cfg.hidden) and st.embedding.dtype == torch.bfloat16
    rows = st.embedding[ids]
    for pi in range(3):                              # q, k, v
        assert torch.equal(st.x[0, pi], rows)
    assert not torch.equal(st.x[1, 0], rows)         # later layers: their own synthetic inputs
    st.step()
    torch.cuda.synchronize()
    st.check_status()
    st.close()


def test_slot_poisoning(lib):
    """With every slot filled with 0xFF bytes before each copy, a correct pool still gives the resident
    bits (no kernel reads a slot outside its acquire..release window), and the planted stale slot, now
    holding the sentinel instead of an older layer, is caught as before."""
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    cfg = synth.STACKS["8b"]
    res = _run(cfg, 4, 256, "resident")
    for fault, equal in ((None, True), (lib.LSN_POOL_FAULT_STALE_SLOT, False)):
        st = Stack(cfg, layers=4, tokens=256, mode="streamed", keep_outputs=True)
        lib.layer_pool_set_debug(st.pool, lib.LSN_POOL_DEBUG_POISON)
        with pytest.raises(lib.LsnError) as e:        # unknown flag bits: refused, the setting stays
            lib.layer_pool_set_debug(st.pool, 4)
        assert e.value.status == lib.LSN_ERR_INVALID_ARG
        if fault is not None:
            lib.layer_pool_inject_fault(st.pool, fault)
        st.step()
        st.step()
        torch.cuda.synchronize()
        fwd, bwd, bad = _compare(st, res)
        assert (fwd and bwd) == equal, (fault, bad)
        st.close()


def test_no_h2d_equals_resident(lib):
    cfg = synth.STACKS["8b"]
    res = _run(cfg, 3, 512, "resident")
    pre = _run(cfg, 3, 512, "no_h2d")
    fwd, bwd, bad = _compare(pre, res)
    assert fwd and bwd, bad


def test_planted_aliasing_is_caught(lib):
    """A pool that hands back a stale slot (the aliasing defect) must fail the gate."""
    cfg = synth.STACKS["8b"]
    res = _run(cfg, 4, 256, "resident")
    bad_run = _run(cfg, 4, 256, "streamed", fault=lib.LSN_POOL_FAULT_STALE_SLOT)
    fwd, bwd, bad = _compare(bad_run, res)
    assert not (fwd and bwd), "the bit-exactness gate missed a planted aliasing fault"


def test_injected_copy_failure_then_reset(lib):
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    cfg = synth.STACKS["8b"]
    st = Stack(cfg, layers=3, tokens=256, mode="streamed", keep_outputs=True)
    lib.layer_pool_inject_fault(st.pool, lib.LSN_POOL_FAULT_COPY_ERROR)
    with pytest.raises(lib.LsnError) as e:
        st.step()
    assert e.value.status == lib.LSN_ERR_CUDA
    torch.cuda.synchronize()
    lib.layer_pool_reset(st.pool)
    st.step()
    torch.cuda.synchronize()
    res = _run(cfg, 3, 256, "resident")
    fwd, bwd, bad = _compare(st, res)
    assert fwd and bwd, bad
    st.close()


def test_pool_rules(lib):
    import torch
    n = 1 << 20
    host = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    host2 = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    host.fill_(1)
    host2.fill_(2)
    pool = lib.layer_pool_create(1, n, 0)
    try:
        with pytest.raises(lib.LsnError) as e:                       # pageable memory is refused
            pageable = torch.empty(n, dtype=torch.uint8)
            lib.layer_pool_register(pool, 0, pageable.data_ptr(), n)
        assert e.value.status == lib.LSN_ERR_INVALID_ARG
        with pytest.raises(lib.LsnError) as e:                       # larger than a slot
            lib.layer_pool_register(pool, 0, host.data_ptr(), n + 1)
        assert e.value.status == lib.LSN_ERR_INVALID_ARG
        lib.layer_pool_register(pool, 0, host.data_ptr(), n)
        lib.layer_pool_register(pool, 1, host2.data_ptr(), n)
        s = torch.cuda.current_stream()
        p0 = lib.layer_pool_acquire(pool, 0, s)
        with pytest.raises(lib.LsnError) as e:                       # the only slot is in use
            lib.layer_pool_prefetch(pool, 1)
        assert e.value.status == lib.LSN_ERR_STATE
        lib.layer_pool_release(pool, 0, s)
        with pytest.raises(lib.LsnError) as e:                       # release of a layer not held
            lib.layer_pool_release(pool, 0, s)
        assert e.value.status == lib.LSN_ERR_STATE
        p1 = lib.layer_pool_acquire(pool, 1, s)
        assert p1 == p0                                              # same slot, reused after release
        lib.layer_pool_release(pool, 1, s)
        lib.layer_pool_wait_idle(pool, 10000)
        st = lib.layer_pool_stats(pool)
        assert st["copies"] == 2 and st["bytes_copied"] == 2 * n and st["misses"] == 2
    finally:
        lib.layer_pool_destroy(pool)


def test_prefetch_keeps_a_resident_layer(lib):
    """Prefetching a layer that is already in a slot protects that slot: the next copy takes another
    slot even where the protected one was released longer ago, and the later acquire copies nothing."""
    import torch
    n = 1 << 20
    hosts = [torch.full((n,), i + 1, dtype=torch.uint8, pin_memory=True) for i in range(3)]
    pool = lib.layer_pool_create(2, n, 0)
    try:
        for i, h in enumerate(hosts):
            lib.layer_pool_register(pool, i, h.data_ptr(), n)
        s = torch.cuda.current_stream()
        p0 = lib.layer_pool_acquire(pool, 0, s)
        lib.layer_pool_release(pool, 0, s)
        p1 = lib.layer_pool_acquire(pool, 1, s)
        lib.layer_pool_release(pool, 1, s)
        assert p0 != p1
        lib.layer_pool_prefetch(pool, 0)              # resident, released first: now protected
        lib.layer_pool_prefetch(pool, 2)              # must take layer 1's slot
        c = lib.layer_pool_stats(pool)["copies"]
        assert lib.layer_pool_acquire(pool, 0, s) == p0
        assert lib.layer_pool_acquire(pool, 2, s) == p1
        assert lib.layer_pool_stats(pool)["copies"] == c == 3
        lib.layer_pool_release(pool, 0, s)
        lib.layer_pool_release(pool, 2, s)
        lib.layer_pool_wait_idle(pool, 10000)
    finally:
        lib.layer_pool_destroy(pool)


@pytest.mark.parametrize("slots,ahead,api", [(3, True, "layer"), (5, True, "layer"), (5, False, "layer"),
                                             (4, False, "proj"), (8, True, "layer")])
def test_slot_window_copies_and_bits(lib, slots, ahead, api):
    """With S slots each sweep keeps S layers in flight; a step copies 2L-2S layers in steady state
    (2L-S in the first), and the results equal the resident run bit for bit."""
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    cfg = synth.STACKS["8b"]
    L = 8
    res = _run(cfg, L, 256, "resident", lanes=1, api="proj")
    st = Stack(cfg, layers=L, tokens=256, mode="streamed", n_slots=slots, keep_outputs=True, api=api,
               dequant_ahead=ahead)
    assert st.ahead == ahead and st.n_slots == slots
    counts = []
    for _ in range(3):
        c0 = st.pool_stats()["copies"]
        st.step()
        counts.append(st.pool_stats()["copies"] - c0)
    torch.cuda.synchronize()
    st.check_status()
    assert counts == [2 * L - slots, 2 * L - 2 * slots, 2 * L - 2 * slots], counts
    fwd, bwd, bad = _compare(st, res)
    assert fwd and bwd, bad
    st.close()


def test_grouped_stack_matches_shared_inputs(lib, orc):
    """A stack whose q|k|v and gate|up run as groups gives the same y, dA and dB as the same stack run
    ungrouped, streamed or resident; the grouped dX (the group's summed input gradient) equals the
    ungrouped sum within bf16 rounding and the oracle's sum of the members' dX on sampled token rows."""
    import numpy as np
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    from tests.helpers import assert_close, bf16_tensor_to_f64
    from tests.helpers import lib_option
    cfg = synth.STACKS["8b"]
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):      # whole tiles: y the same bits grouped or not
        shared = Stack(cfg, layers=2, tokens=512, mode="resident", keep_outputs=True, shared_inputs=True)
        shared.step()
        grouped = shared.with_inputs(shared_inputs=True, grouped=True, mode="streamed")
        grouped.step()
        torch.cuda.synchronize()
    grouped.check_status()
    assert all(torch.equal(shared.y[k], grouped.y[k]) for k in shared.y)
    assert all(torch.equal(shared.dA[k], grouped.dA[k]) and torch.equal(shared.dB[k], grouped.dB[k]) for k in shared.dA)
    rows = np.sort(np.random.default_rng(32).choice(512, size=16, replace=False))
    for l in range(2):
        for members in ((0, 1, 2), (4, 5)):
            ref = sum(shared.dX[l, pi].double() for pi in members)
            got = grouped.dX[l, members[0]].double()
            err = float((got - ref).norm() / ref.norm())
            assert err < 5e-3, (l, members, err)
            want = sum(orc.lora_bwd_dx(_bits(grouped.dY[l, pi]), _oracle_weight(orc, grouped, l, pi),
                                       _bits(grouped.A[l, pi]), _bits(grouped.B[l, pi]), grouped.scale, rows=rows)
                       for pi in members)
            assert_close(bf16_tensor_to_f64(grouped.dX[l, members[0]])[rows], want, f"grouped dX {l},{members}")
    grouped.close()


@pytest.mark.parametrize("name,tokens,pis", [("8b", 2048, (0, 6)), ("8b", 8192, (1, 6)), ("3b", 1024, (1, 4)),
                                               ("72b", 1024, (0, 6))])
def test_full_size_stack_against_oracle(lib, orc, name, tokens, pis):
    """One layer of a workload stack at its stated size in the timed launch configuration (layer calls,
    streamed through the pool, NF4 weights dequantised one layer ahead, projection 0's GEMM then the merged
    launch of the others): y and dX on sampled token rows and dA, dB in full for two projections (the
    8B q and down, the 8B k and down at 8192 tokens (a merged launch of 4864 tiles), the 3B bf16 k and gate,
    the 72B q and down of ~29568 x 8192), against the oracle.  The
    oracle quantises (or rounds to bf16) the fp32 weights itself; inputs are the seeded generator's, read
    back from the device."""
    import numpy as np
    import torch
    from layer_streamed_nf4_b200.stack import Stack
    from tests.helpers import assert_close, bf16_tensor_to_f64
    cfg = synth.STACKS[name]
    st = Stack(cfg, layers=1, tokens=tokens, mode="streamed", keep_outputs=True)
    assert st.ahead == (cfg.base == "nf4")
    st.step()
    torch.cuda.synchronize()
    st.check_status()
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    rows = np.sort(np.random.default_rng(8).choice(tokens, size=32, replace=False))
    for pi in pis:
        p = st.proj[pi]
        W = synth.device_normal((p.N, p.K), 0.02, st.seed, 0, pi, synth.T_W, device=st.dev).cpu().numpy()
        if cfg.base == "nf4":
            q = orc.nf4_quantize(W)
            Wb = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size).reshape(W.shape)
        else:
            Wb = synth.to_bf16_bits(W)
        x, dY, A, B = bits(st.x[0, pi]), bits(st.dY[0, pi]), bits(st.A[0, pi]), bits(st.B[0, pi])
        assert_close(bf16_tensor_to_f64(st.y[0, pi])[rows], orc.lora_fwd(x, Wb, A, B, st.scale, rows=rows), f"{p.name} y")
        assert_close(bf16_tensor_to_f64(st.dX[0, pi])[rows], orc.lora_bwd_dx(dY, Wb, A, B, st.scale, rows=rows),
                     f"{p.name} dX")
        rA, rB = orc.lora_bwd_dadb(x, dY, A, B, st.scale)
        assert_close(st.dA[0, pi].cpu().numpy(), rA, f"{p.name} dA")
        assert_close(st.dB[0, pi].cpu().numpy(), rB, f"{p.name} dB")
    st.close()


def test_two_holders_keep_the_slot_until_both_release(lib):
    """A layer acquired on two streams: the reader with the long queue releases first, the other second,
    then a copy of another layer is started into the (only) slot.  The copy must wait for both releases,
    so the long reader still sees the first layer's codes (poison mode on: a premature copy would show
    the 0xFF sentinel or the second layer)."""
    import torch
    from tests.helpers import DeviceNF4
    rows, cols = 256, 4096
    ws = [DeviceNF4(rows, cols).quantize(synth.normal_f32((rows, cols), 0.02, synth.SEED, 500, i, synth.T_W))
          for i in range(2)]
    torch.cuda.synchronize()
    nbytes = ws[0].blob.numel()
    hosts = [d.blob.cpu().pin_memory() for d in ws]
    ref = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    lib.nf4_dequant(ws[0].w, ref)
    pool = lib.layer_pool_create(1, nbytes, 0)
    try:
        lib.layer_pool_set_debug(pool, lib.LSN_POOL_DEBUG_POISON)
        for i, h in enumerate(hosts):
            lib.layer_pool_register(pool, i, h.data_ptr(), nbytes)
        a, b = torch.cuda.Stream(), torch.cuda.Stream()
        out = torch.zeros((rows, cols), dtype=torch.bfloat16, device="cuda")
        pa = lib.layer_pool_acquire(pool, 0, a)
        pb = lib.layer_pool_acquire(pool, 0, b)
        assert pa == pb                                   # one slot, two holders
        with torch.cuda.stream(a):
            torch.cuda._sleep(200_000_000)                # a long queue ahead of the reader (bounded spin)
        w = lib.nf4_weight_in_blob(rows, cols, pa)
        lib.nf4_dequant(w, out, a)                        # reads the slot after the spin
        lib.layer_pool_release(pool, 0, a)                # the long reader releases first
        lib.layer_pool_release(pool, 0, b)                # the idle holder second
        lib.layer_pool_prefetch(pool, 1)                  # takes the slot: must wait for both
        torch.cuda.synchronize()
        assert torch.equal(out, ref), "the slot was overwritten while a holder still read it"
        p1 = lib.layer_pool_acquire(pool, 1, b)
        w1 = lib.nf4_weight_in_blob(rows, cols, p1)
        lib.nf4_dequant(w1, out, b)
        lib.layer_pool_release(pool, 1, b)
        want = torch.empty_like(ref)
        lib.nf4_dequant(ws[1].w, want)
        torch.cuda.synchronize()
        assert torch.equal(out, want)                     # and the copy did land afterwards
        lib.layer_pool_wait_idle(pool, 10000)
    finally:
        lib.layer_pool_destroy(pool)


@pytest.mark.parametrize("shared,grouped", [(False, False), (True, True)])
def test_host_io_steps(lib, shared, grouped):
    """Steps fed from pinned host memory (stack.HostIO, the bench's end-to-end path): every step takes the
    host's inputs (here different from the stack's own), its result reaches the host, and that result is
    bit for bit a plain step's on the same inputs.  With grouped projections there is one host buffer per
    distinct input and one per group's input gradient."""
    import torch
    from layer_streamed_nf4_b200.stack import HostIO, Stack
    cfg = synth.STACKS["8b"]
    st = Stack(cfg, layers=3, tokens=512, mode="streamed", n_slots=2, keep_outputs=True, shared_inputs=shared)
    if grouped:
        st = st.with_inputs(shared_inputs=True, grouped=True, mode="streamed")
    h_in, h_out = HostIO.host_buffers(st)
    assert len(h_in) == (4 if shared else 7) and len(h_out) == (4 if grouped else 7)
    g = torch.Generator().manual_seed(7)
    for h in h_in:
        h.copy_(torch.randn(h.shape, generator=g).to(h.dtype))
    HostIO(st, h_in, h_out).run(3, st.step)
    torch.cuda.synchronize()
    st.check_status()
    for h, t in zip(h_in, HostIO.inputs_of(st)):
        assert torch.equal(h, t.cpu()), "the step did not take the host's inputs"
    got = [h.clone() for h in h_out]
    st.step()
    torch.cuda.synchronize()
    for h, t in zip(got, HostIO.outputs_of(st)):
        assert torch.equal(h, t.cpu()), "the host result differs from a plain step's"
    st.close()


@pytest.mark.parametrize("name,tokens", [("8b", 2048), ("0.5b", 512)])
def test_merged_gemms_in_the_stack(lib, name, tokens):
    """The stack's layer calls with projections 1..n-1 as one merged GEMM launch (LSN_OPT_LAYER_MERGE; the
    dequantisation ahead hands the calls bf16 bases): streamed with merging is torch.equal to resident
    without it, for every y, dX, dA and dB."""
    from tests.helpers import lib_option
    cfg = synth.STACKS[name]
    with lib_option(lib, lib.LSN_OPT_LAYER_MERGE, 0):
        res = _run(cfg, 3, tokens, "resident")
    with lib_option(lib, lib.LSN_OPT_LAYER_MERGE, 1):
        st = _run(cfg, 3, tokens, "streamed", steps=2)
    fwd, bwd, bad = _compare(st, res)
    assert fwd and bwd, bad
