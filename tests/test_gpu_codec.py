"""GPU parity of the NF4 codec: nf4_quantize and nf4_dequant through the C ABI
must be bit-exact with the oracle (packed bytes, second-level codes, s2,
offset, dequantised bf16)."""
import numpy as np
import pytest

from layer_streamed_nf4_b200 import synth
from tests.helpers import DeviceNF4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from layer_streamed_nf4_b200 import lsnf4
    return lsnf4


def _weights(kind, rows, cols, seed):
    W = synth.normal_f32((rows, cols), 0.02, seed, 900, kind)
    if kind == 1:        # planted zero blocks, a lone outlier, tiny and subnormal values
        flat = W.reshape(-1, 64)           # one row per 64-block
        nb = flat.shape[0]
        flat[0] = 0.0
        flat[min(3, nb - 1)] = 0.0
        flat[min(5, nb - 1), 7] = 3.5
        flat[min(7, nb - 1)] *= np.float32(1e-30)
        flat[min(9, nb - 1)] = np.float32(1e-42)
        W = flat.reshape(rows, cols)
    if kind == 2:        # equal absmax everywhere: s2 == 0 in every group
        W = np.clip(W, -0.01, 0.01)
        W[:, ::64] = 0.01
    return W


def _check_codec(lib, orc, W):
    import torch
    rows, cols = W.shape
    d = DeviceNF4(rows, cols).quantize(W)
    packed, qa, s2, off = d.arrays()
    ref = orc.nf4_quantize(W)
    assert np.array_equal(packed, ref["packed"]), "packed codes differ"
    assert np.array_equal(qa, ref["absmax_q"]), "second-level codes differ"
    assert np.array_equal(s2.view(np.uint32), ref["s2"].view(np.uint32)), "s2 differ"
    assert np.array(off).view(np.uint32) == np.array(ref["offset"]).view(np.uint32), "offset differs"
    out = torch.empty(rows * cols, dtype=torch.int16, device="cuda")
    lib.nf4_dequant(d.w, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint16)
    want = orc.nf4_dequant(ref["packed"], ref["absmax_q"], ref["s2"], ref["offset"], rows * cols)
    assert np.array_equal(got, want), f"dequant differs at {np.flatnonzero(got != want)[:5]}"


@pytest.mark.parametrize("shape,kind", [((512, 512), 0), ((64, 192), 0), ((1000, 128), 1), ((256, 4096), 2),
                                        ((1, 64), 0), ((3, 64), 1), ((896, 896), 0), ((128, 896), 0)])
def test_codec_bit_exact(lib, orc, shape, kind):
    _check_codec(lib, orc, _weights(kind, *shape, seed=hash(shape) % 1000))


def test_codec_bit_exact_8b_mlp_projection(lib, orc):
    """Full-size 8B gate/up weight (14336 x 4096), every byte compared."""
    W = synth.normal_f32((14336, 4096), 0.02, synth.SEED, 0, 4, synth.T_W)
    _check_codec(lib, orc, W)


def test_quantize_is_deterministic(lib):
    import torch
    W = _weights(0, 512, 512, 5)
    a = DeviceNF4(512, 512).quantize(W)
    b = DeviceNF4(512, 512).quantize(W)
    torch.cuda.synchronize()
    assert torch.equal(a.blob, b.blob)


def test_dequant_batch_equals_single_calls():
    """nf4_dequant_batch over weights of several shapes (more than one launch's worth) gives the bits of
    one nf4_dequant per weight."""
    import torch
    from layer_streamed_nf4_b200 import lsnf4
    shapes = [(64, 64), (128, 4096), (1024, 4096), (4096, 1024), (192, 320)] * 4
    ws, singles, outs = [], [], []
    for i, (r, c) in enumerate(shapes):
        d = DeviceNF4(r, c).quantize(torch.randn((r, c), generator=torch.Generator().manual_seed(i)).numpy() * 0.02)
        ws.append(d)
        a = torch.empty((r, c), dtype=torch.bfloat16, device="cuda")
        lsnf4.nf4_dequant(d.w, a)
        singles.append(a)
        outs.append(torch.empty((r, c), dtype=torch.bfloat16, device="cuda"))
    for bps in (0, 1, 3):
        for o in outs:
            o.zero_()
        lsnf4.nf4_dequant_batch([d.w for d in ws], outs, blocks_per_sm=bps)
        torch.cuda.synchronize()
        for a, b in zip(singles, outs):
            assert torch.equal(a, b), bps


def test_codec_bit_exact_at_first_level_ties(lib, orc):
    """Blocks whose w / absmax fall exactly on the midpoints between adjacent levels (absmax a power of two)
    and one or two fp32 steps either side, at four scales: the GPU's thresholds decide every one of them
    as the oracle's exact nearest-level rule does (ties to the lower index)."""
    from tests.helpers import first_level_tie_weights
    W = first_level_tie_weights(orc.nf4_codebook())
    assert W.shape[0] % 2 == 0
    _check_codec(lib, orc, W.reshape(-1, 128))          # blocks run along the flattened rows


@pytest.mark.parametrize("off_exp,s2_exp,m_lo,m_hi", [(-12, -5, -1.0 / 128, 1.0), (-5, -5, -1.0, -0.5)])
def test_codec_bit_exact_at_second_level_ties(lib, orc, off_exp, s2_exp, m_lo, m_hi):
    """Weights whose second-level values (absmax - offset) / s2 fall exactly on the midpoints of adjacent
    entries of the k/127 table, and one or two fp32 steps either side (over a hundred exact ties on the
    positive side, sixty on the negative): codes, s2, offset and dequantised bf16 equal the oracle's."""
    from tests.helpers import second_level_tie_weights
    W, _, _ = second_level_tie_weights(orc.dq_table()[:255], off_exp, s2_exp, m_lo, m_hi)
    _check_codec(lib, orc, W.reshape(-1, 256))
