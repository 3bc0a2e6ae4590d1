"""GPU parity of the LoRA linear forward and backward through the C ABI
against the fp64 oracle: y, dX, dA, dB within a relative Frobenius error of
5e-3 and a max-abs error of 2e-2 x RMS of the oracle tensor.

The oracle never sees anything the CUDA path produced: it quantises the
fp32 base weight itself and dequantises its own codes."""
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


def _oracle_w_bits(orc, W, kind):
    if kind == "nf4":
        q = orc.nf4_quantize(W)
        return orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size).reshape(W.shape)
    return synth.to_bf16_bits(W)


class Linear:
    """Device-side inputs of one LoRA linear plus its base, set up through the C ABI."""

    def __init__(self, lib, c, kind):
        import torch
        self.lib, self.c, self.kind = lib, c, kind
        self.x = bits_to_device_bf16(c.x)
        self.dY = bits_to_device_bf16(c.dY)
        self.A = bits_to_device_bf16(c.A)
        self.B = bits_to_device_bf16(c.B)
        if kind == "nf4":
            self.nf4 = DeviceNF4(c.N, c.K).quantize(c.W)
            self.base = lib.base_nf4(self.nf4.w)
            k = lib.LSN_BASE_NF4
        else:
            self.Wb = bits_to_device_bf16(synth.to_bf16_bits(c.W))
            self.base = lib.base_bf16(self.Wb, c.N, c.K)
            k = lib.LSN_BASE_BF16
        self.ws_bytes = lib.lora_ws_bytes(c.T, c.K, c.N, c.r, k)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device="cuda")

    def fwd(self):
        import torch
        y = torch.empty((self.c.T, self.c.N), dtype=torch.bfloat16, device="cuda")
        self.lib.lora_linear_fwd(self.base, self.x, self.c.T, self.A, self.B, self.c.r, self.c.scale, y, self.ws,
                                 self.ws_bytes)
        return y

    def bwd(self, accumulate=False, dA=None, dB=None, want_dx=True):
        import torch
        c = self.c
        dX = torch.empty((c.T, c.K), dtype=torch.bfloat16, device="cuda") if want_dx else None
        dA = torch.zeros((c.r, c.K), dtype=torch.float32, device="cuda") if dA is None else dA
        dB = torch.zeros((c.N, c.r), dtype=torch.float32, device="cuda") if dB is None else dB
        self.lib.lora_linear_bwd(self.base, self.x, self.dY, c.T, self.A, self.B, c.r, c.scale, dX, dA, dB,
                                 accumulate, self.ws, self.ws_bytes)
        return dX, dA, dB

    def status(self):
        self.lib.ws_status(self.ws)


def _full_parity(lib, orc, c, kind):
    import torch
    L = Linear(lib, c, kind)
    y = L.fwd()
    dX, dA, dB = L.bwd()
    torch.cuda.synchronize()
    L.status()
    Wb = _oracle_w_bits(orc, c.W, kind)
    assert_close(bf16_tensor_to_f64(y), orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale), "y")
    assert_close(bf16_tensor_to_f64(dX), orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale), "dX")
    rA, rB = orc.lora_bwd_dadb(c.x, c.dY, c.A, c.B, c.scale)
    assert_close(dA.cpu().numpy(), rA, "dA")
    assert_close(dB.cpu().numpy(), rB, "dB")
    return L


@pytest.mark.parametrize("kind", ["nf4", "bf16"])
def test_single_linear_config(lib, orc, kind):
    """256 tokens, 512 -> 512, r = 8, alpha = 16 (the single-linear workload)."""
    s = synth.SINGLE
    c = synth.linear_case(s["T"], s["K"], s["N"], s["r"], s["alpha"], seed=synth.SEED)
    _full_parity(lib, orc, c, kind)


@pytest.mark.parametrize("T,K,N,r", [(1, 64, 64, 8), (77, 128, 192, 16), (200, 896, 128, 16), (131, 192, 896, 24),
                                     (300, 512, 256, 64), (129, 256, 384, 8)])
def test_ragged_and_small_shapes(lib, orc, T, K, N, r):
    c = synth.linear_case(T, K, N, r, 2.0 * r, seed=T * 7 + K)
    _full_parity(lib, orc, c, "nf4")


@pytest.mark.parametrize("T,K,N", [(300, 256, 9472), (300, 9472, 256)])
def test_pair_kernel_with_ragged_rows(lib, orc, T, K, N):
    """Shapes with >= 74 pair tiles run the 2-SM kernel (forward for the first,
    input gradient for the second), here with a ragged last 256-row tile."""
    c = synth.linear_case(T, K, N, 16, 32.0, seed=T + K)
    _full_parity(lib, orc, c, "nf4")


@pytest.mark.parametrize("T,K,N", [(512, 4096, 9536), (300, 9536, 4096)])
def test_fused_nf4_equals_bf16_base_of_its_dequant(lib, T, K, N):
    """The NF4 weight converted inside the GEMM gives exactly the bits of the same
    GEMM run on nf4_dequant's bf16 weight (same values, same MMA order; the
    fused kernel runs whole tiles, so both take the whole-tile schedule).  The
    shapes put one direction on the fused pair kernel, with a partial last
    N tile and, for K % 128 == 64, a half-empty last contraction stage."""
    from tests.helpers import lib_option
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):
        _fused_equals_unfused(lib, T, K, N)


def _fused_equals_unfused(lib, T, K, N):
    import torch
    lib.set_option(lib.LSN_OPT_FUSED_NF4, 1)
    c = synth.linear_case(T, K, N, 16, 32.0, seed=T + N)
    Lq = Linear(lib, c, "nf4")
    Wd = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    lib.nf4_dequant(Lq.nf4.w, Wd)
    Lb = Linear(lib, c, "bf16")
    Lb.Wb = Wd
    Lb.base = lib.base_bf16(Wd, N, K)
    try:
        a = (Lq.fwd(), *Lq.bwd())
    finally:
        lib.set_option(lib.LSN_OPT_FUSED_NF4, 0)
    b = (Lb.fwd(), *Lb.bwd())
    c2 = (Lq.fwd(), *Lq.bwd())                      # default path: dequantise + bf16 GEMM
    torch.cuda.synchronize()
    Lq.status()
    Lb.status()
    for name, u, v in zip(("y", "dX", "dA", "dB"), c2, b):
        assert torch.equal(u, v), "unfused " + name
    for name, u, v in zip(("y", "dX", "dA", "dB"), a, b):
        assert torch.equal(u, v), name


@pytest.mark.parametrize("T,K,N,r", [(2048, 4096, 4096, 16), (300, 4096, 9536, 16), (512, 4096, 14336, 8),
                                     (257, 14336, 4096, 32)])
def test_tmem_fused_forward(lib, orc, T, K, N, r):
    """The forward GEMM that converts the NF4 codes straight into tensor memory (W as the A operand, y^T in
    the accumulator, transposed in the epilogue): y against the oracle on sampled rows (the last one
    included), and against the whole-tile GEMM on nf4_dequant's bf16 weight.  The shapes cover full and
    ragged token tiles, a partial last W tile and ranks 8 to 32."""
    import torch
    from tests.helpers import lib_option
    c = synth.linear_case(T, K, N, r, 2.0 * r, seed=T + K + N + r)
    L = Linear(lib, c, "nf4")
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):
        ref = L.fwd()                                  # nf4_dequant, then the bf16 GEMM
        with lib_option(lib, lib.LSN_OPT_FUSED_NF4, 2):
            y = L.fwd()
            y2 = L.fwd()
    torch.cuda.synchronize()
    L.status()
    assert torch.equal(y, y2), "rerun differs"
    d = (y.float() - ref.float()).abs()
    assert float(d.max()) <= 2.0 ** -7 * float(ref.float().abs().max()), float(d.max())
    rows = np.sort(np.random.default_rng(13).choice(T, size=min(T, 40), replace=False))
    rows[-1] = T - 1
    Wb = _oracle_w_bits(orc, c.W, "nf4")
    assert_close(bf16_tensor_to_f64(y)[rows], orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale, rows=rows), "y (tensor-memory NF4)")
    print("tmem-fused y bit-identical to dequant + GEMM:", bool(torch.equal(y, ref)))


def test_b_zero_gives_the_base_product(lib, orc):
    c = synth.linear_case(160, 256, 320, 16, 32.0, seed=3)
    c.B[:] = 0
    L = Linear(lib, c, "nf4")
    y = L.fwd()
    import torch
    torch.cuda.synchronize()
    Wb = _oracle_w_bits(orc, c.W, "nf4")
    ref = synth.bf16_bits_to_f32(c.x).astype(np.float64) @ synth.bf16_bits_to_f32(Wb).astype(np.float64).T
    assert_close(bf16_tensor_to_f64(y), ref, "y(B=0)")


def test_zero_tokens(lib):
    import torch
    c = synth.linear_case(0, 128, 128, 8, 16.0, seed=1)
    L = Linear(lib, c, "nf4")
    y = L.fwd()
    dX, dA, dB = L.bwd()
    torch.cuda.synchronize()
    assert y.numel() == 0 and float(dA.abs().sum()) == 0.0 and float(dB.abs().sum()) == 0.0


def test_accumulate_adds_into_gradients(lib, orc):
    import torch
    c = synth.linear_case(96, 128, 192, 16, 32.0, seed=9)
    L = Linear(lib, c, "bf16")
    _, dA1, dB1 = L.bwd()
    _, dA2, dB2 = L.bwd(accumulate=True, dA=dA1.clone(), dB=dB1.clone())
    torch.cuda.synchronize()
    rA, rB = orc.lora_bwd_dadb(c.x, c.dY, c.A, c.B, c.scale)
    assert_close(dA2.cpu().numpy(), 2 * rA, "dA accumulated")
    assert_close(dB2.cpu().numpy(), 2 * rB, "dB accumulated")


def test_deterministic_rerun(lib):
    import torch
    c = synth.linear_case(384, 512, 1024, 16, 32.0, seed=12)
    L = Linear(lib, c, "nf4")
    a = (L.fwd(), *L.bwd())
    b = (L.fwd(), *L.bwd())
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


# Full-size decoder projections at the timed launch configuration; y and dX
# on 64 sampled token rows (computed one by one by the oracle), dA and dB in
# full.
SAMPLED = [
    ("8b-q", 2048, 4096, 4096),
    ("8b-kv", 2048, 4096, 1024),
    ("8b-down", 2048, 14336, 4096),
    ("0.5b-up", 512, 896, 4864),
    ("3b-gate", 1024, 2048, 11008),
    ("72b-down", 1024, 29568, 8192),
]


@pytest.mark.parametrize("name,T,K,N", SAMPLED)
def test_full_size_sampled_rows(lib, orc, name, T, K, N):
    import torch
    c = synth.linear_case(T, K, N, 16, 32.0, seed=sum(map(ord, name)))
    kind = "bf16" if name.startswith(("0.5b", "3b")) else "nf4"
    L = Linear(lib, c, kind)
    y = L.fwd()
    dX, dA, dB = L.bwd()
    torch.cuda.synchronize()
    L.status()
    rows = np.sort(np.random.default_rng(5).choice(T, size=64, replace=False))
    rows[-1] = T - 1
    Wb = _oracle_w_bits(orc, c.W, kind)
    assert_close(bf16_tensor_to_f64(y)[rows], orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale, rows=rows), f"{name} y")
    assert_close(bf16_tensor_to_f64(dX)[rows], orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale, rows=rows), f"{name} dX")
    rA, rB = orc.lora_bwd_dadb(c.x, c.dY, c.A, c.B, c.scale)
    assert_close(dA.cpu().numpy(), rA, f"{name} dA")
    assert_close(dB.cpu().numpy(), rB, f"{name} dB")


@pytest.mark.parametrize("T,K,N,rows", [(2048, 4096, 4096, 48), (300, 9536, 9536, 32), (300, 6400, 7680, 32)])
def test_stream_k_schedule(lib, orc, T, K, N, rows):
    """GEMMs whose tiles leave the last wave partly empty take the stream-K schedule, in both directions
    here: the 8B q shape (128 pair tiles for 74 pairs), a ragged 2-SM shape (76 pair tiles, a half-empty
    last contraction stage) and a ragged 1-SM one (180 and 150 tiles for 148 SMs).  Results match the
    oracle, repeat bit for bit, and differ from the whole-tile schedule only by the rounding of the split
    sums."""
    import torch
    from tests.helpers import lib_option
    c = synth.linear_case(T, K, N, 16, 32.0, seed=T + K + N)
    L = Linear(lib, c, "nf4")
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 1):
        a = (L.fwd(), *L.bwd())
        b = (L.fwd(), *L.bwd())
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):
        w = (L.fwd(), *L.bwd())
    torch.cuda.synchronize()
    L.status()
    for u, v in zip(a, b):
        assert torch.equal(u, v), "stream-K rerun differs"
    assert not torch.equal(a[0], w[0]) and not torch.equal(a[1], w[1]), "the stream-K schedule did not run"
    for u, v in zip(a[:2], w[:2]):
        d = (u.float() - v.float()).abs()
        assert float(d.max()) <= 2.0 ** -6 * float(v.float().abs().max()), "beyond the rounding of split sums"
    assert torch.equal(a[2], w[2]) and torch.equal(a[3], w[3])     # dA, dB do not come from the GEMM
    Wb = _oracle_w_bits(orc, c.W, "nf4")
    sel = np.sort(np.random.default_rng(9).choice(T, size=rows, replace=False)) if rows else None
    y_ref = orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale, rows=sel)
    dx_ref = orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale, rows=sel)
    y, dX = bf16_tensor_to_f64(a[0]), bf16_tensor_to_f64(a[1])
    assert_close(y if sel is None else y[sel], y_ref, "y")
    assert_close(dX if sel is None else dX[sel], dx_ref, "dX")


@pytest.mark.parametrize("T,K,N,rows", [(2048, 4096, 4096, 48), (2048, 4096, 14336, 32), (300, 9536, 9536, 0)])
def test_tail_split_schedule(lib, orc, T, K, N, rows):
    """The tail split (LSN_OPT_GEMM_TAIL_SPLIT) cuts the tiles of a partly filled last round into column
    quanta: the 8B q shape (128 pair tiles: 54 tiles in the last round), the 8B gate shape (448 tiles
    forward: 4 in the last round; its backward fills whole rounds of 128-column quanta and stays whole)
    and a ragged shape whose last-round tiles are the partial last column block (76 tiles, N = 37.25
    tiles: three of each tile's four quanta lie past N).  Every output element is still one MMA chain
    over the whole contraction, so the bits equal the whole-tile schedule's; results match the oracle."""
    import torch
    from tests.helpers import lib_option
    c = synth.linear_case(T, K, N, 16, 32.0, seed=T + K + 2 * N)
    L = Linear(lib, c, "nf4")
    with lib_option(lib, lib.LSN_OPT_STREAM_K, 0):
        with lib_option(lib, lib.LSN_OPT_GEMM_TAIL_SPLIT, 1):
            a = (L.fwd(), *L.bwd())
        with lib_option(lib, lib.LSN_OPT_GEMM_TAIL_SPLIT, 0):
            w = (L.fwd(), *L.bwd())
    torch.cuda.synchronize()
    L.status()
    for name, u, v in zip(("y", "dX", "dA", "dB"), a, w):
        assert torch.equal(u, v), f"tail split changed {name}"
    Wb = _oracle_w_bits(orc, c.W, "nf4")
    sel = np.sort(np.random.default_rng(11).choice(T, size=rows, replace=False)) if rows else None
    y, dX = bf16_tensor_to_f64(a[0]), bf16_tensor_to_f64(a[1])
    assert_close(y if sel is None else y[sel], orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale, rows=sel), "y")
    assert_close(dX if sel is None else dX[sel], orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale, rows=sel), "dX")


def test_bounded_wait_gives_up_and_the_context_stays_usable(lib, orc):
    """A wait on an mbarrier that nothing arrives on ends after its limit with a timeout status (no
    hang), and kernels launched afterwards still compute correct results."""
    import time
    t0 = time.perf_counter()
    assert lib.selftest_wait_timeout(2000) == lib.LSN_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 30.0
    test_single_linear_config(lib, orc, "nf4")
