"""Pins for the oracle's LoRA linear forward and backward.

The method ("Can You Fine-Tune a 27B Model on a Laptop?", 1:36-1:58; the
sourcefeed article "An 8B Fine-Tune Now Fits in 4 GB of VRAM", section "The
trick is that frozen weights are just data") trains a thin pair of matrices per
layer over a frozen base: y = x W^T + s (x A^T) B^T, with gradients for x, A
and B only.  Pins: numpy's matmul on the merged weight W + s B A (a different
formula with the same value), the B = 0 special case, and central differences
of L = sum(y * dY), which are exact for a function linear in each argument.
"""
import numpy as np
import pytest

from layer_streamed_nf4_b200 import synth


def _f(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _case(T=4, K=64, N=64, r=2, alpha=4.0, seed=21):
    return synth.linear_case(T, K, N, r, alpha, seed=seed, b_std=0.3)


def _wbits(c):
    return synth.to_bf16_bits(c.W)


def test_b_zero_is_the_plain_matmul(orc):
    c = _case(T=5, K=128, N=64, r=4)
    Wb = _wbits(c)
    Bz = np.zeros_like(c.B)
    y = orc.lora_fwd(c.x, Wb, c.A, Bz, c.scale)
    assert np.allclose(y, _f(c.x) @ _f(Wb).T, rtol=1e-12, atol=1e-12)


def test_forward_equals_merged_weight(orc):
    c = _case(T=6, K=64, N=128, r=3, alpha=6.0)
    Wb = _wbits(c)
    y = orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale)
    W_eff = _f(Wb) + c.scale * _f(c.B) @ _f(c.A)
    assert np.allclose(y, _f(c.x) @ W_eff.T, rtol=1e-12, atol=1e-12)


def test_dx_equals_merged_weight(orc):
    c = _case(T=6, K=64, N=128, r=3, alpha=6.0)
    Wb = _wbits(c)
    dX = orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale)
    W_eff = _f(Wb) + c.scale * _f(c.B) @ _f(c.A)
    assert np.allclose(dX, _f(c.dY) @ W_eff, rtol=1e-12, atol=1e-12)


def test_row_selection_matches_full(orc):
    c = _case(T=9, K=64, N=64, r=2)
    Wb = _wbits(c)
    rows = np.array([8, 0, 3])
    y = orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale)
    dX = orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale)
    assert np.array_equal(orc.lora_fwd(c.x, Wb, c.A, c.B, c.scale, rows=rows), y[rows])
    assert np.array_equal(orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, c.scale, rows=rows), dX[rows])


def _bf16_neighbours(bits):
    """Bit patterns of the bf16 values one ulp above and one ulp below a bf16 value."""
    b = int(bits)
    if b & 0x7fff == 0:
        return np.uint16(0x0001), np.uint16(0x8001)
    if b & 0x8000:                      # negative: a larger pattern is a more negative value
        return np.uint16(b - 1), np.uint16(b + 1)
    return np.uint16(b + 1), np.uint16(b - 1)


def _loss(orc, x, W, A, B, dY, s):
    return float(np.sum(orc.lora_fwd(x, W, A, B, s) * _f(dY)))


@pytest.mark.parametrize("seed", [31, 32])
def test_gradients_by_central_differences(orc, seed):
    """d(sum y*dY)/d(x, A, B) by differencing two neighbouring bf16 inputs; L is linear in each."""
    c = _case(T=4, K=64, N=64, r=2, alpha=4.0, seed=seed)
    Wb = _wbits(c)
    s = c.scale
    dX = orc.lora_bwd_dx(c.dY, Wb, c.A, c.B, s)
    dA, dB = orc.lora_bwd_dadb(c.x, c.dY, c.A, c.B, s)
    rng = np.random.default_rng(seed)
    for name, arr, grad in (("x", c.x, dX), ("A", c.A, dA), ("B", c.B, dB)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, d)) for d in arr.shape)
            hi, lo = _bf16_neighbours(arr[idx])
            ph, pl = arr.copy(), arr.copy()
            ph[idx], pl[idx] = hi, lo
            args = {"x": c.x, "A": c.A, "B": c.B}
            args_h = dict(args, **{name: ph})
            args_l = dict(args, **{name: pl})
            Lh = _loss(orc, args_h["x"], Wb, args_h["A"], args_h["B"], c.dY, s)
            Ll = _loss(orc, args_l["x"], Wb, args_l["A"], args_l["B"], c.dY, s)
            h = float(_f(np.array([hi], np.uint16))[0] - _f(np.array([lo], np.uint16))[0])
            fd = (Lh - Ll) / h
            assert fd == pytest.approx(grad[idx], rel=1e-6, abs=1e-9 * max(1.0, abs(Lh))), (name, idx)


def test_dadb_against_numpy(orc):
    c = _case(T=7, K=128, N=64, r=4, alpha=8.0)
    dA, dB = orc.lora_bwd_dadb(c.x, c.dY, c.A, c.B, c.scale)
    x, dY, A, B = _f(c.x), _f(c.dY), _f(c.A), _f(c.B)
    assert np.allclose(dA, c.scale * (dY @ B).T @ x, rtol=1e-12, atol=1e-12)
    assert np.allclose(dB, c.scale * dY.T @ (x @ A.T), rtol=1e-12, atol=1e-12)
