"""Pins for the oracle's NF4 codec, each against something other than the oracle.

The pages ("Can You Fine-Tune a 27B Model on a Laptop?", 2:19-2:29) name a
4-bit format for bell-curve weights plus a second quantisation of its
constants, but print no levels or values; the oracle takes QLoRA's published
normal-quantile construction (the paper the sourcefeed article "An 8B Fine-Tune
Now Fits in 4 GB of VRAM" links).  The pins below use closed forms, a library
routine (scipy), exact rational arithmetic and special cases whose result is
known exactly.
"""
from fractions import Fraction

import numpy as np
import pytest
from scipy import special

P_MAX = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def test_ppnd16_against_scipy_ndtri(orc):
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 2001), [1e-300, 1e-100, 1e-20, 1e-10, 0.02425, 0.075, 0.5,
                                                         0.925, 0.97575, 1 - 1e-10, 1 - 1e-15]])
    for p in ps:
        ref = special.ndtri(p)
        got = orc.ppnd16(p)
        assert got == pytest.approx(ref, rel=2e-14, abs=1e-15), p


def test_nf4_levels_invariants(orc):
    c = orc.nf4_codebook()
    assert c.dtype == np.float32 and c.shape == (16,)
    assert c[0] == -1.0 and c[15] == 1.0          # end points exact
    assert c[7] == 0.0                              # an exact zero level
    assert np.all(np.diff(c.astype(np.float64)) > 0)
    assert int(np.sum(c < 0)) == 7 and int(np.sum(c > 0)) == 8


def test_nf4_levels_closed_form(orc):
    """Phi(c_i * Phi^-1(p_max)) must equal the i-th equal step of the quantile range."""
    c = orc.nf4_codebook().astype(np.float64)
    zmax = special.ndtri(P_MAX)
    for j in range(1, 9):                           # positives: 8 steps
        assert special.ndtr(c[7 + j] * zmax) == pytest.approx(0.5 + (P_MAX - 0.5) * j / 8, abs=1e-7)
    for j in range(1, 8):                           # negatives: 7 steps
        assert special.ndtr(-c[7 - j] * zmax) == pytest.approx(0.5 + (P_MAX - 0.5) * j / 7, abs=1e-7)


def test_nf4_levels_golden_file(orc):
    """The stored table (written by tests/golden/make_golden.py from the oracle) is unchanged."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nf4_levels.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    want = np.array([int(r[1], 16) for r in rows], dtype=np.uint32).view(np.float32)
    assert np.array_equal(orc.nf4_codebook().view(np.uint32), want.view(np.uint32))


def _fp32_nearest_of(fr: Fraction) -> np.float32:
    """The fp32 value nearest to an exact rational (ties to even), by exhaustive neighbour check."""
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda v: (abs(Fraction(float(v)) - fr), int(np.array(v).view(np.uint32)) & 1))
    return np.float32(best)


def test_dq_table_closed_form(orc):
    t = orc.dq_table()
    for k in range(-127, 128):
        assert t[k + 127] == _fp32_nearest_of(Fraction(k, 127)), k
    assert t[255] == 0.0 and t[127] == 0.0 and t[0] == -1.0 and t[254] == 1.0


def _exact_nearest(v: np.float32, levels) -> int:
    fv = Fraction(float(v))
    dist = [abs(fv - Fraction(float(c))) for c in levels]
    m = min(dist)
    return dist.index(m)                            # first = lower index on a tie


def _straddle_points(levels):
    """fp32 values around each exact midpoint of adjacent levels, plus the levels themselves."""
    pts = []
    for a, b in zip(levels[:-1], levels[1:]):
        mid = (Fraction(float(a)) + Fraction(float(b))) / 2
        f = np.float32(float(mid))
        pts += [f, np.nextafter(f, np.float32(-2)), np.nextafter(f, np.float32(2)),
                np.nextafter(np.nextafter(f, np.float32(2)), np.float32(2)), np.float32(a), np.float32(b)]
    return pts


def test_nearest_nf4_exact(orc):
    c = orc.nf4_codebook()
    rng = np.random.default_rng(7)
    pts = list(rng.uniform(-1, 1, 3000).astype(np.float32)) + _straddle_points(c)
    pts += [np.float32(0.0), np.float32(-0.0), np.float32(1e-30), np.float32(-1e-30)]
    for v in pts:
        assert orc.nearest_nf4(v) == _exact_nearest(v, c), float(v)


def test_nearest_tie_goes_to_lower_index(orc):
    c = orc.nf4_codebook()
    # Find adjacent levels whose exact midpoint is an fp32 value: that value is a tie.
    ties = 0
    for i in range(15):
        mid = (Fraction(float(c[i])) + Fraction(float(c[i + 1]))) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:
            ties += 1
            assert orc.nearest_nf4(f) == i
    t = orc.dq_table()
    for i in range(254):
        mid = (Fraction(float(t[i])) + Fraction(float(t[i + 1]))) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:
            ties += 1
            assert orc.nearest_dq(f) == i
    assert ties > 0


def test_nearest_dq_exact(orc):
    t = orc.dq_table()[:255]
    rng = np.random.default_rng(8)
    pts = list(rng.uniform(-1, 1, 800).astype(np.float32)) + _straddle_points(t)[::3]
    for v in pts:
        assert orc.nearest_dq(v) == _exact_nearest(v, t), float(v)


def _blocks_of_levels(rng, nblk, exps, c):
    """Weights whose every 64-block is level[i] * 2^e, each block holding a +-1 level."""
    idx = rng.integers(0, 16, size=(nblk, 64))
    idx[np.arange(nblk), rng.integers(0, 64, size=nblk)] = rng.choice([0, 15], size=nblk)
    W = c[idx].astype(np.float64) * np.ldexp(1.0, exps)[:, None]
    return idx, W.astype(np.float32)


def test_roundtrip_codebook_points_equal_scale(orc):
    """Every element a level times one power of two: codes come back exactly and so does absmax."""
    c = orc.nf4_codebook()
    rng = np.random.default_rng(3)
    nblk = 600
    idx, W = _blocks_of_levels(rng, nblk, np.full(nblk, -5), c)
    q = orc.nf4_quantize(W, want_absmax=True)
    assert np.all(q["absmax"] == np.float32(2.0 ** -5))
    assert q["offset"] == np.float32(2.0 ** -5)
    assert np.all(q["s2"] == 0) and np.all(q["absmax_q"] == 127)
    codes = np.stack([q["packed"] >> 4, q["packed"] & 15], axis=1).reshape(-1)
    assert np.array_equal(codes, idx.reshape(-1))
    deq = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size)
    # level * 2^-5 is exact in fp32, so dequant is that value rounded once to bf16.
    want = np.array([orc.f32_to_bf16_bits(v) for v in W.reshape(-1)[:4096]], np.uint16)
    assert np.array_equal(deq[:4096], want)


def test_roundtrip_codebook_points_varying_scale(orc):
    """Codes are exact whatever the per-block power-of-two absmax."""
    c = orc.nf4_codebook()
    rng = np.random.default_rng(4)
    nblk = 700
    idx, W = _blocks_of_levels(rng, nblk, rng.integers(-12, 3, size=nblk), c)
    q = orc.nf4_quantize(W)
    codes = np.stack([q["packed"] >> 4, q["packed"] & 15], axis=1).reshape(-1)
    assert np.array_equal(codes, idx.reshape(-1))


def test_equal_absmax_special_case(orc):
    """All blocks share one (non power of two) absmax: second level is exact, absmax_hat = absmax."""
    rng = np.random.default_rng(5)
    a = np.float32(0.0371)
    W = rng.uniform(-1, 1, size=(300, 64)).astype(np.float32) * a
    W[:, 5] = a
    W = np.clip(W, -a, a)
    q = orc.nf4_quantize(W, want_absmax=True)
    assert np.all(q["absmax"] == a) and q["offset"] == a
    assert np.all(q["absmax_q"] == 127)
    for b in (0, 77, 299):
        assert orc.absmax_hat(q["absmax_q"], q["s2"], q["offset"], b) == a


def test_offset_is_the_mean(orc):
    rng = np.random.default_rng(6)
    W = rng.normal(0, 0.02, size=(97 * 64 * 5,)).astype(np.float32)
    q = orc.nf4_quantize(W, want_absmax=True)
    import math
    exact = np.float32(math.fsum(float(v) for v in q["absmax"]) / q["absmax"].size)
    assert abs(int(np.array(q["offset"]).view(np.int32)) - int(np.array(exact).view(np.int32))) <= 1


def test_second_level_error_bound(orc):
    """|absmax_hat - absmax| <= s2 / 254 (half a step of the k/127 code) + fp32 rounding."""
    rng = np.random.default_rng(9)
    W = rng.normal(0, 0.02, size=(1000, 64)).astype(np.float32)
    W[:300] *= 3.0
    q = orc.nf4_quantize(W, want_absmax=True)
    for b in range(0, 1000, 7):
        ah = float(orc.absmax_hat(q["absmax_q"], q["s2"], q["offset"], b))
        s2 = float(q["s2"][b // 256])
        assert abs(ah - float(q["absmax"][b])) <= s2 / 254 * (1 + 1e-5) + 4e-7 * abs(ah)


def test_zero_block_and_ragged_group(orc):
    """A zero block codes to the zero level; 192 blocks give one short second-level group."""
    rng = np.random.default_rng(10)
    W = rng.normal(0, 0.02, size=(64 * 192,)).astype(np.float32)
    W[64 * 3:64 * 4] = 0.0
    q = orc.nf4_quantize(W, want_absmax=True)
    assert q["s2"].size == 1 and q["absmax_q"].size == 192
    assert np.all(q["packed"][32 * 3:32 * 4] == 0x77)
    deq = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size)
    assert np.all((deq[64 * 3:64 * 4] & 0x7fff) == 0)


def test_quantize_rejects_nonfinite(orc):
    W = np.zeros(128, np.float32)
    W[3] = np.nan
    with pytest.raises(ValueError):
        orc.nf4_quantize(W)
    W[3] = np.inf
    with pytest.raises(ValueError):
        orc.nf4_quantize(W)


def test_quantize_brute_force_tiny(orc):
    """Brute force on a tiny input: every step recomputed with numpy fp32 scalars and exact rationals."""
    rng = np.random.default_rng(11)
    W = rng.normal(0, 0.02, size=(300 * 64,)).astype(np.float32)
    q = orc.nf4_quantize(W, want_absmax=True)
    c = orc.nf4_codebook()
    t = orc.dq_table()[:255]
    blocks = W.reshape(-1, 64)
    am = np.abs(blocks).max(axis=1)
    assert np.array_equal(am, q["absmax"])
    for b in range(0, 300, 37):
        for i in range(0, 64, 5):
            v = np.float32(blocks[b, i] / am[b])
            qq = _exact_nearest(v, c)
            byte = q["packed"][(b * 64 + i) // 2]
            got = (byte >> 4) if i % 2 == 0 else (byte & 15)
            assert got == qq
    off = q["offset"]
    for g in range(2):
        cb = (am[g * 256:(g + 1) * 256] - off).astype(np.float32)
        s2 = np.float32(np.abs(cb).max())
        assert q["s2"][g] == s2
        for j in range(0, cb.size, 9):
            v = np.float32(cb[j] / s2)
            assert q["absmax_q"][g * 256 + j] == _exact_nearest(v, t)


def _bf16_rne_torch(x32: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of fp32 values, rounded to nearest even by torch (a library conversion)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_dequant_exact_at_second_level_points(orc):
    """Second level with s2 != 0, closed form: every block is level points times its absmax, the absmax
    values of a group sit at offset - d, offset and offset + d (d differs per group, one group is ragged),
    so the second-level values are exactly -1, 0, +1 (codes 0, 127, 254) and absmax_hat equals the absmax.
    Then dequantisation must give bf16(w) for every element, whatever the group: a wrong s2 index, a
    wrong table entry or a dropped offset changes absmax_hat and breaks the equality."""
    c = orc.nf4_codebook()
    rng = np.random.default_rng(21)
    off = 2.0 ** -5
    ds = [2.0 ** -7, 2.0 ** -6, 3 * 2.0 ** -8, 2.0 ** -8]
    sizes = [256, 256, 256, 100]                         # the last group is ragged
    absmax = []
    for d, n in zip(ds, sizes):
        pattern = np.resize([off - d, off + d, off, off + d, off - d, off], n)
        if pattern.sum() != n * off:                     # keep each group's mean exactly off
            pattern[-1] = off
        absmax += list(pattern)
    absmax = np.array(absmax, np.float32)
    assert float(np.sum(absmax.astype(np.float64))) == off * absmax.size
    nblk = absmax.size
    idx = rng.integers(0, 16, size=(nblk, 64))
    idx[np.arange(nblk), rng.integers(0, 64, size=nblk)] = rng.choice([0, 15], size=nblk)
    W = (c[idx].astype(np.float32) * absmax[:, None]).astype(np.float32)
    q = orc.nf4_quantize(W, want_absmax=True)
    assert q["offset"] == np.float32(off)
    assert np.array_equal(q["s2"], np.array(ds, np.float32))
    assert set(np.unique(q["absmax_q"])) <= {0, 127, 254} and len(set(np.unique(q["absmax_q"]))) == 3
    codes = np.stack([q["packed"] >> 4, q["packed"] & 15], axis=1).reshape(-1)
    assert np.array_equal(codes, idx.reshape(-1))
    deq = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size)
    assert np.array_equal(deq, _bf16_rne_torch(W.reshape(-1)))


def test_dequant_second_level_random_groups(orc):
    """Second level with s2 != 0 on N(0, 0.02) weights whose groups have very different absmax spreads:
    (i) every element equals bf16(level[q] * absmax_hat) with absmax_hat rebuilt in numpy fp32 from the
    stored code, its group's s2 and the offset; (ii) every element lies within the format's error bound of
    the original weight: half the widest gap between adjacent levels times the block absmax, plus the
    level times half a second-level step (s2/254), plus bf16 rounding."""
    c = orc.nf4_codebook()
    tab = orc.dq_table()
    rng = np.random.default_rng(22)
    spreads = [1.0, 6.0, 0.2, 2.5, 1.0]
    W = np.concatenate([rng.normal(0, 0.02, size=(256 * 64,)) * s for s in spreads]).astype(np.float32)
    W = W[:W.size - 64 * 37]                             # a ragged last group
    q = orc.nf4_quantize(W, want_absmax=True)
    assert np.all(q["s2"] > 0) and q["s2"].max() > 3 * q["s2"].min() and len(set(q["s2"].tolist())) == q["s2"].size
    deq = orc.nf4_dequant(q["packed"], q["absmax_q"], q["s2"], q["offset"], W.size)
    nblk = W.size // 64
    blk = np.arange(nblk)
    ah = (tab[q["absmax_q"]] * q["s2"][blk // 256]).astype(np.float32) + np.float32(q["offset"])
    ah = ah.astype(np.float32)
    codes = np.stack([q["packed"] >> 4, q["packed"] & 15], axis=1).reshape(-1)
    want = _bf16_rne_torch((c[codes].reshape(nblk, 64) * ah[:, None]).astype(np.float32).reshape(-1))
    assert np.array_equal(deq, want)
    got = (deq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    half_gap = float(np.max(np.diff(c.astype(np.float64)))) / 2
    a = np.repeat(q["absmax"].astype(np.float64), 64)
    s2 = np.repeat(q["s2"][blk // 256].astype(np.float64), 64)
    bound = half_gap * a + np.abs(c[codes].astype(np.float64)) * s2 / 254 * (1 + 1e-5) + 2.0 ** -8 * np.abs(got) + 1e-9
    assert np.all(np.abs(got - W.astype(np.float64)) <= bound)


def test_first_level_ties_constructed(orc):
    """Weights built on the exact midpoints between adjacent levels (absmax a power of two, so w / absmax is
    the midpoint itself) and one or two fp32 steps either side: the oracle's codes equal the exact nearest
    level with ties to the lower index."""
    from tests.helpers import first_level_tie_weights
    c = orc.nf4_codebook()
    W = first_level_tie_weights(c)
    q = orc.nf4_quantize(W, want_absmax=True)
    codes = np.stack([q["packed"] >> 4, q["packed"] & 15], axis=1).reshape(W.shape)
    ties = 0
    for b in range(W.shape[0]):
        a = q["absmax"][b]
        assert a == np.abs(W[b]).max() and np.log2(a) == int(np.log2(a))
        for i in range(64):
            v = np.float32(W[b, i] / a)
            assert codes[b, i] == _exact_nearest(v, c), (b, i, float(v))
            for k in range(15):
                if Fraction(float(v)) == (Fraction(float(c[k])) + Fraction(float(c[k + 1]))) / 2:
                    ties += 1
                    assert codes[b, i] == k
    assert ties > 0


@pytest.mark.parametrize("off_exp,s2_exp,m_lo,m_hi", [(-12, -5, -1.0 / 128, 1.0), (-5, -5, -1.0, -0.5)])
def test_second_level_ties_constructed(orc, off_exp, s2_exp, m_lo, m_hi):
    """Weights whose second-level values land exactly on the midpoints of adjacent entries of the k/127
    table (and one or two fp32 steps either side): the offset comes out exactly 2^off_exp, every tie group
    has s2 = 2^s2_exp, and each block's code is the exact nearest entry with ties to the lower index."""
    from tests.helpers import second_level_tie_weights
    tab = orc.dq_table()[:255]
    W, n_groups, where = second_level_tie_weights(tab, off_exp, s2_exp, m_lo, m_hi)
    q = orc.nf4_quantize(W, want_absmax=True)
    assert q["offset"] == np.float32(2.0 ** off_exp)
    assert np.all(q["s2"][:n_groups] == np.float32(2.0 ** s2_exp))
    ties = 0
    for b, v in where:
        got_v = np.float32((np.float32(q["absmax"][b]) - q["offset"]) / q["s2"][b // 256])
        assert got_v == v
        assert q["absmax_q"][b] == _exact_nearest(v, tab), (b, float(v))
        k = int(q["absmax_q"][b])
        if k < 254 and Fraction(float(v)) == (Fraction(float(tab[k])) + Fraction(float(tab[k + 1]))) / 2:
            ties += 1
    assert ties >= 3 and len(where) > 100
