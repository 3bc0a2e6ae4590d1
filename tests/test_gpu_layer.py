"""The whole-layer calls (lora_layer_fwd / lora_layer_bwd) through the C ABI.

They launch the projections of a decoder layer together (one dequantisation
kernel, one down-projection kernel, one token-reduction kernel for all of
them) and can carry u = x A^T from the forward to the backward.  Each
projection's results must be bit for bit those of the single-linear calls
on the same inputs, and within the oracle tolerances."""
import numpy as np
import pytest

from layer_streamed_nf4_b200 import synth
from tests.helpers import DeviceNF4, assert_close, bf16_tensor_to_f64, bits_to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from layer_streamed_nf4_b200 import lsnf4
    return lsnf4


class Layer:
    """Device tensors of n projections sharing T and r (seeded like the stacks)."""

    def __init__(self, lib, shapes, T, r, kind, seed=5):
        import torch
        self.lib, self.T, self.r, self.kind = lib, T, r, kind
        self.scale = 2.0
        dev = torch.device("cuda")
        self.p = []
        for pi, (K, N) in enumerate(shapes):
            # host inputs from the shared seeded generator; the oracle sees these, never device results
            c = synth.linear_case(T, K, N, r, self.scale * r, seed=seed * 100 + pi)
            d = {"K": K, "N": N, "case": c}
            if kind == "nf4":
                d["nf4"] = DeviceNF4(N, K).quantize(c.W)
                d["base"] = lib.base_nf4(d["nf4"].w)
            else:
                d["Wb"] = bits_to_device_bf16(synth.to_bf16_bits(c.W))
                d["base"] = lib.base_bf16(d["Wb"], N, K)
            for k in ("x", "dY", "A", "B"):
                d[k] = bits_to_device_bf16(getattr(c, k)) if getattr(c, k).size else \
                    torch.empty(getattr(c, k).shape, dtype=torch.bfloat16, device=dev)
            self.p.append(d)

    def outputs(self):
        import torch
        out = []
        for d in self.p:
            out.append({"y": torch.empty((self.T, d["N"]), dtype=torch.bfloat16, device="cuda"),
                        "dX": torch.empty((self.T, d["K"]), dtype=torch.bfloat16, device="cuda"),
                        "dA": torch.zeros((self.r, d["K"]), dtype=torch.float32, device="cuda"),
                        "dB": torch.zeros((d["N"], self.r), dtype=torch.float32, device="cuda"),
                        "u": torch.zeros((self.T, self.r), dtype=torch.float32, device="cuda")})
        return out

    def single(self, accumulate=False, out=None):
        import torch
        lib = self.lib
        out = out or self.outputs()
        k = lib.LSN_BASE_NF4 if self.kind == "nf4" else lib.LSN_BASE_BF16
        for d, o in zip(self.p, out):
            n = lib.lora_ws_bytes(self.T, d["K"], d["N"], self.r, k)
            ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
            lib.lora_linear_fwd(d["base"], d["x"], self.T, d["A"], d["B"], self.r, self.scale, o["y"], ws, n)
            lib.lora_linear_bwd(d["base"], d["x"], d["dY"], self.T, d["A"], d["B"], self.r, self.scale, o["dX"],
                                o["dA"], o["dB"], accumulate, ws, n)
            torch.cuda.synchronize()
            lib.ws_status(ws)
        return out

    def layer(self, keep_u=True, accumulate=False, out=None, off=()):
        """One lora_layer_fwd + lora_layer_bwd over the projections; those in `off` with the adapter off."""
        import torch
        lib = self.lib
        out = out or self.outputs()
        projs = [lib.lora_proj(d["base"], d["x"], d["A"], d["B"], y=o["y"], dY=d["dY"], dX=o["dX"], dA=o["dA"],
                               dB=o["dB"], u=o["u"] if keep_u else None) if i not in off else
                 lib.lora_proj(d["base"], d["x"], None, None, y=o["y"], dY=d["dY"], dX=o["dX"])
                 for i, (d, o) in enumerate(zip(self.p, out))]
        arr = lib.proj_array(projs)
        n = lib.layer_ws_bytes(arr, self.T, self.r)
        ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
        lib.lora_layer_fwd(arr, self.T, self.r, self.scale, ws, n)
        lib.lora_layer_bwd(arr, self.T, self.r, self.scale, accumulate, ws, n)
        torch.cuda.synchronize()
        lib.ws_status(ws)
        return out


SHAPES_8B = [(4096, 4096), (4096, 1024), (4096, 1024), (4096, 4096), (4096, 14336), (4096, 14336), (14336, 4096)]
SMALL = [(256, 256), (256, 64), (256, 128), (256, 256), (256, 512), (256, 512), (512, 256)]


def _equal(a, b, names=("y", "dX", "dA", "dB")):
    import torch
    for i, (u, v) in enumerate(zip(a, b)):
        for k in names:
            assert torch.equal(u[k], v[k]), f"projection {i}: {k} differs"


@pytest.mark.parametrize("shapes,T,kind", [(SMALL, 300, "nf4"), (SMALL, 77, "bf16"), (SHAPES_8B, 2048, "nf4")])
def test_layer_equals_single_calls(lib, shapes, T, kind):
    L = Layer(lib, shapes, T, 16, kind)
    ref = L.single()
    _equal(L.layer(keep_u=True), ref)
    _equal(L.layer(keep_u=False), ref)


def test_kept_u_is_x_times_a_transposed(lib, orc):
    """The u the forward keeps equals the oracle's x A^T (fp32 accumulation of exact bf16 products)."""
    L = Layer(lib, SMALL[:3], 130, 16, "nf4")
    out = L.layer(keep_u=True)
    for d, o in zip(L.p, out):
        c = d["case"]
        x = synth.bf16_bits_to_f32(c.x).astype(np.float64)
        A = synth.bf16_bits_to_f32(c.A).astype(np.float64)
        assert_close(o["u"].cpu().numpy(), x @ A.T, "u")


def test_layer_accumulates_like_single_calls(lib):
    import torch
    L = Layer(lib, SMALL, 200, 8, "nf4")
    a = L.single()
    a = L.single(accumulate=True, out=a)
    b = L.layer()
    b = L.layer(accumulate=True, out=b)
    _equal(a, b, ("dA", "dB"))
    assert all(float(o["dA"].abs().sum()) > 0 for o in b)


def test_layer_against_oracle(lib, orc):
    """One small layer checked directly against the fp64 oracle."""
    L = Layer(lib, SMALL[:2], 96, 16, "nf4", seed=9)
    out = L.layer()
    for d, o in zip(L.p, out):
        c = d["case"]
        q = orc.nf4_quantize(c.W)                  # the oracle quantises the fp32 weight itself
        Wb = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], c.W.size).reshape(c.W.shape)
        x, dY, A, B = c.x, c.dY, c.A, c.B
        assert_close(bf16_tensor_to_f64(o["y"]), orc.lora_fwd(x, Wb, A, B, L.scale), "y")
        assert_close(bf16_tensor_to_f64(o["dX"]), orc.lora_bwd_dx(dY, Wb, A, B, L.scale), "dX")
        rA, rB = orc.lora_bwd_dadb(x, dY, A, B, L.scale)
        assert_close(o["dA"].cpu().numpy(), rA, "dA")
        assert_close(o["dB"].cpu().numpy(), rB, "dB")


def test_layer_with_fused_nf4_equals_unfused(lib):
    from tests.helpers import lib_option
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):          # the fused kernel runs whole tiles
        with lib_option(lib, lib.LSN_OPT_FUSED_NF4, 1):
            L = Layer(lib, [(4096, 9536), (9536, 4096), (4096, 1024)], 512, 16, "nf4")
            a = L.layer()
        _equal(a, L.layer())


def test_layer_with_tmem_fused_forward(lib, orc):
    """Layer calls with the forward GEMMs converting NF4 in tensor memory (LSN_OPT_FUSED_NF4 = 2): the same
    bits as the single-linear calls in that mode, y against the oracle, and the backward unchanged."""
    from tests.helpers import lib_option
    with lib_option(lib, lib.LSN_OPT_FUSED_NF4, 2):
        L = Layer(lib, [(4096, 9536), (4096, 14336), (9536, 4096), (4096, 1024)], 512, 16, "nf4", seed=8)
        a = L.layer()
        _equal(a, L.single())
    b = L.layer()
    _equal(a, b, ("dX", "dA", "dB", "u"))
    rows = np.sort(np.random.default_rng(4).choice(512, size=24, replace=False))
    for d, o in zip(L.p, a):
        c = d["case"]
        q = orc.nf4_quantize(c.W)
        Wb = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], c.W.size).reshape(c.W.shape)
        assert_close(bf16_tensor_to_f64(o["y"])[rows], orc.lora_fwd(c.x, Wb, c.A, c.B, L.scale, rows=rows), "y")


def test_scheduling_options_give_the_same_bits(lib):
    """GEMMs on the fewest SMs for their number of tile rounds (LSN_OPT_GEMM_MIN_UNITS), the last round's
    tiles cut into column quanta (LSN_OPT_GEMM_TAIL_SPLIT, either setting) and a batched dequantisation
    confined to SMs of its own (LSN_OPT_DEQUANT_SPARE_SMS) change where work runs, not what it computes:
    the same bits as the defaults."""
    import torch
    from tests.helpers import lib_option
    L = Layer(lib, SHAPES_8B, 2048, 16, "nf4", seed=9)
    a = L.layer()
    with lib_option(lib, lib.LSN_OPT_GEMM_MIN_UNITS, 1):
        _equal(a, L.layer())
    split = lib.get_option(lib.LSN_OPT_GEMM_TAIL_SPLIT)
    with lib_option(lib, lib.LSN_OPT_GEMM_TAIL_SPLIT, 1 - split):
        _equal(a, L.layer())
    outs = [torch.empty((d["N"], d["K"]), dtype=torch.bfloat16, device="cuda") for d in L.p]
    ref = [torch.empty_like(o) for o in outs]
    for d, r in zip(L.p, ref):
        lib.nf4_dequant(d["nf4"].w, r)
    with lib_option(lib, lib.LSN_OPT_DEQUANT_SPARE_SMS, 12):
        lib.nf4_dequant_batch([d["nf4"].w for d in L.p], outs, blocks_per_sm=2)
    torch.cuda.synchronize()
    assert all(torch.equal(o, r) for o, r in zip(outs, ref))


@pytest.mark.parametrize("shapes,T,off", [(SHAPES_8B, 2048, ()), (SMALL, 300, (2,)),
                                          ([(960, 704), (960, 320), (704, 960), (960, 64)], 77, ())])
def test_merged_layer_gemms(lib, orc, shapes, T, off):
    """LSN_OPT_LAYER_MERGE: with bf16 bases, projections 1..n-1 of a layer call run as one multi-problem GEMM
    launch (a balanced static schedule of whole tiles over the SM pairs), forward and backward.  The same
    bits as one launch per projection, for every y, dX, dA and dB: the 8B layer, a ragged set with one
    projection's adapter off, and a ragged set with partial column tiles at T = 77; oracle checks on
    sampled rows."""
    from tests.helpers import lib_option
    L = Layer(lib, shapes, T, 16, "bf16", seed=13)
    with lib_option(lib, lib.LSN_OPT_LAYER_MERGE, 0):
        a = L.layer(off=off)
    with lib_option(lib, lib.LSN_OPT_LAYER_MERGE, 1):
        b = L.layer(off=off)
        b2 = L.layer(off=off)
    _equal(b, a)
    _equal(b2, a)
    rows = np.sort(np.random.default_rng(4).choice(T, size=min(T, 24), replace=False))
    for pi in sorted({1, len(shapes) - 1, *off}):
        c = L.p[pi]["case"]
        Wb = synth.to_bf16_bits(c.W)
        Bm = np.zeros_like(c.B) if pi in off else c.B
        assert_close(bf16_tensor_to_f64(b[pi]["y"])[rows], orc.lora_fwd(c.x, Wb, c.A, Bm, L.scale, rows=rows),
                     f"merged y {pi}")
        assert_close(bf16_tensor_to_f64(b[pi]["dX"])[rows], orc.lora_bwd_dx(c.dY, Wb, c.A, Bm, L.scale, rows=rows),
                     f"merged dX {pi}")


def test_merged_launch_limits(lib):
    """The merged launch takes at most 8 problems: a call with 9 projections (8 after the first) merges
    them, one with 10 runs one launch per projection; both give the bits of the single-linear calls."""
    from tests.helpers import lib_option
    shapes9 = [(256, 256), (256, 64), (256, 128), (256, 256), (256, 512), (256, 512), (512, 256), (256, 192),
               (320, 256)]
    for shapes in (shapes9, shapes9 + [(256, 320)]):
        L = Layer(lib, shapes, 300, 16, "bf16", seed=17)
        a = L.single()
        with lib_option(lib, lib.LSN_OPT_LAYER_MERGE, 1):
            b = L.layer()
        _equal(b, a)


def test_layer_zero_tokens(lib):
    import torch
    L = Layer(lib, SMALL[:2], 0, 16, "nf4")
    out = L.layer()
    assert all(float(o["dA"].abs().sum()) == 0.0 and float(o["dB"].abs().sum()) == 0.0 for o in out)


def test_layer_lanes_option_gives_the_same_bits(lib):
    L = Layer(lib, SMALL, 257, 16, "nf4", seed=3)
    a = L.layer()                                     # default: two lanes
    lib.set_option(lib.LSN_OPT_LAYER_LANES, 1)
    try:
        b = L.layer()
    finally:
        lib.set_option(lib.LSN_OPT_LAYER_LANES, 2)
    _equal(a, b)
    _equal(a, L.single())


def test_dependent_launch_option_gives_the_same_bits(lib):
    L = Layer(lib, SMALL, 190, 16, "nf4", seed=4)
    a = L.layer()
    lib.set_option(lib.LSN_OPT_PDL, 0)
    try:
        b = L.layer()
        c = L.single()
    finally:
        lib.set_option(lib.LSN_OPT_PDL, 1)
    _equal(a, b)
    _equal(a, c)


def test_adapter_off_is_the_base_term(lib, orc):
    """A projection with A = B = NULL gives exactly the base term: the adapter-on call with B = 0 (whose
    LoRA K-block adds exact zeros) and, within tolerance, the oracle's x W^T."""
    import torch
    L = Layer(lib, SMALL[:4], 150, 16, "nf4", seed=6)
    ref = L.outputs()
    off = L.outputs()
    for d in L.p:
        d["B"].zero_()
    projs_on = [lib.lora_proj(d["base"], d["x"], d["A"], d["B"], y=o["y"], dY=d["dY"], dX=o["dX"], dA=o["dA"],
                              dB=o["dB"]) for d, o in zip(L.p, ref)]
    projs_off = [lib.lora_proj(d["base"], d["x"], None, None, y=o["y"], dY=d["dY"], dX=o["dX"])
                 for d, o in zip(L.p, off)]
    for projs in (projs_on, projs_off):
        arr = lib.proj_array(projs)
        n = lib.layer_ws_bytes(arr, L.T, L.r)
        ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
        lib.lora_layer_fwd(arr, L.T, L.r, L.scale, ws, n)
        lib.lora_layer_bwd(arr, L.T, L.r, L.scale, False, ws, n)
        torch.cuda.synchronize()
        lib.ws_status(ws)
    # dX of the adapter-on call with B = 0 is dY W + s (dY 0) A: the base term again
    _equal(off, ref, ("y", "dX"))
    for d, o in zip(L.p, off):
        c = d["case"]
        q = orc.nf4_quantize(c.W)
        Wb = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], c.W.size).reshape(c.W.shape)
        zeroB = np.zeros_like(c.B)
        assert_close(bf16_tensor_to_f64(o["y"]), orc.lora_fwd(c.x, Wb, c.A, zeroB, L.scale), "y (adapter off)")


# ------------------------------------------------------------------ groups --

GROUPS = (1, 1, 1, 0, 2, 2, 0)       # q|k|v and gate|up read the same input
SMALL_G = [(256, 256), (256, 128), (256, 64), (256, 256), (256, 512), (256, 384), (512, 256)]


def _grouped_setup(lib, shapes, T, kind, seed):
    """One x per group (q, k, v share x_attn; gate, up share x_mlp), bases laid out back to back
    (one buffer per layer, like a pool slot)."""
    import torch
    L = Layer(lib, shapes, T, 16, kind, seed=seed)
    for pi in (1, 2):
        L.p[pi]["x"] = L.p[0]["x"]
        L.p[pi]["case"].x = L.p[0]["case"].x
    L.p[5]["x"] = L.p[4]["x"]
    L.p[5]["case"].x = L.p[4]["case"].x
    if kind == "bf16":
        total = sum(d["N"] * d["K"] for d in L.p)
        L.wbuf = torch.empty(total, dtype=torch.bfloat16, device="cuda")
        off = 0
        for d in L.p:
            n = d["N"] * d["K"]
            L.wbuf[off:off + n].copy_(d["Wb"].reshape(-1))
            d["Wb"] = L.wbuf[off:off + n].view(d["N"], d["K"])
            d["base"] = lib.base_bf16(d["Wb"], d["N"], d["K"])
            off += n
    return L


def _run_layer(lib, L, out, groups):
    import torch
    projs = []
    for pi, (d, o) in enumerate(zip(L.p, out)):
        lead = groups[pi] == 0 or pi == 0 or groups[pi - 1] != groups[pi]
        projs.append(lib.lora_proj(d["base"], d["x"], d["A"], d["B"], y=o["y"], dY=d["dY"],
                                   dX=o["dX"] if lead else None, dA=o["dA"], dB=o["dB"], u=o["u"],
                                   group=groups[pi]))
    arr = lib.proj_array(projs)
    n = lib.layer_ws_bytes(arr, L.T, L.r)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    lib.lora_layer_fwd(arr, L.T, L.r, L.scale, ws, n)
    lib.lora_layer_bwd(arr, L.T, L.r, L.scale, False, ws, n)
    torch.cuda.synchronize()
    lib.ws_status(ws)
    return out


@pytest.mark.parametrize("shapes,T,kind", [(SHAPES_8B, 2048, "nf4"), (SMALL_G, 300, "bf16"), (SMALL_G, 77, "nf4"),
                                          ([(896, 896), (896, 128), (896, 128), (896, 896), (896, 4864),
                                            (896, 4864), (4864, 896)], 512, "bf16")])
def test_grouped_projections(lib, orc, shapes, T, kind):
    """Grouped forward: with whole-tile GEMMs the same bits as ungrouped (with the last round's tiles cut into
    column quanta or not); with the stream-K schedule (whose
    split points depend on the GEMM's shape) within tolerance of the oracle.  Grouped backward: the
    group's dX is the sum of the members' input gradients (checked against the oracle's sum on sampled
    rows); dA, dB the same bits."""
    from tests.helpers import lib_option
    L = _grouped_setup(lib, shapes, T, kind, seed=21)
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):
        plain = _run_layer(lib, L, L.outputs(), (0,) * 7)
        grp = _run_layer(lib, L, L.outputs(), GROUPS)
        _equal(grp, plain, ("y", "dA", "dB", "u"))
        # The other tail-split setting cuts the grouped GEMMs' last rounds differently: the same bits.
        with lib_option(lib, lib.LSN_OPT_GEMM_TAIL_SPLIT, 1 - lib.get_option(lib.LSN_OPT_GEMM_TAIL_SPLIT)):
            grp2 = _run_layer(lib, L, L.outputs(), GROUPS)
        _equal(grp2, grp, ("y", "dA", "dB", "u"))
        leaders = (0, 3, 4, 6)
        _equal([grp2[i] for i in leaders], [grp[i] for i in leaders], ("dX",))
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 1):
        plain = _run_layer(lib, L, L.outputs(), (0,) * 7)
        grp = _run_layer(lib, L, L.outputs(), GROUPS)
    _equal(grp, plain, ("dA", "dB", "u"))
    _equal([grp[3], grp[6]], [plain[3], plain[6]], ("dX",))          # ungrouped projections
    rows = np.sort(np.random.default_rng(3).choice(T, size=min(T, 48), replace=False))
    for pi in (0, 2, 5):
        c = L.p[pi]["case"]
        if kind == "nf4":
            q = orc.nf4_quantize(c.W)
            Wb = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], c.W.size).reshape(c.W.shape)
        else:
            Wb = synth.to_bf16_bits(c.W)
        assert_close(bf16_tensor_to_f64(grp[pi]["y"])[rows], orc.lora_fwd(c.x, Wb, c.A, c.B, L.scale, rows=rows),
                     f"group member {pi} y")
    for members in ((0, 1, 2), (4, 5)):
        ref = 0.0
        for pi in members:
            c = L.p[pi]["case"]
            if kind == "nf4":
                q = orc.nf4_quantize(c.W)
                Wb = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], c.W.size).reshape(c.W.shape)
            else:
                Wb = synth.to_bf16_bits(c.W)
            ref = ref + orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, L.scale, rows=rows)
        assert_close(bf16_tensor_to_f64(grp[members[0]]["dX"])[rows], ref, f"group {members} dX")


def test_group_arguments_are_checked(lib):
    import torch
    L = _grouped_setup(lib, SMALL_G, 64, "nf4", seed=2)
    out = L.outputs()
    projs = [lib.lora_proj(d["base"], d["x"], d["A"], d["B"], y=o["y"], dY=d["dY"], dX=o["dX"], dA=o["dA"],
                           dB=o["dB"], group=GROUPS[pi]) for pi, (d, o) in enumerate(zip(L.p, out))]
    arr = lib.proj_array(projs)
    n = lib.layer_ws_bytes(arr, L.T, L.r)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.LsnError) as e:           # members 1, 2, 5 carry a dX
        lib.lora_layer_bwd(arr, L.T, L.r, L.scale, False, ws, n)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    projs[3].group = 1                               # o has its own x: cannot join q, k, v
    projs[3].dX = None
    with pytest.raises(lib.LsnError) as e:
        lib.lora_layer_fwd(lib.proj_array(projs), L.T, L.r, L.scale, ws, n)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
