"""Test helpers: tolerance metrics and device-side setup through the C ABI."""
from __future__ import annotations

import contextlib

import numpy as np

# Tolerances on floating-point outputs (y, dX, dA, dB) against the fp64
# oracle, per tensor: relative Frobenius error and max-abs error in units of
# the oracle's RMS.
REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2


@contextlib.contextmanager
def lib_option(lib, option: int, value: int):
    """Set one of the library's process-wide options for the duration of a block."""
    old = lib.get_option(option)
    lib.set_option(option, value)
    try:
        yield
    finally:
        lib.set_option(option, old)


def err_metrics(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    fro = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    mx = float(np.max(np.abs(diff)) / max(rms, 1e-300)) if ref.size else 0.0
    return fro, mx


def assert_close(got, ref, name=""):
    fro, mx = err_metrics(got, ref)
    assert fro <= REL_FRO and mx <= MAX_ABS_RMS, f"{name}: rel_fro={fro:.3e} max_abs/rms={mx:.3e}"
    return fro, mx


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def bits_to_device_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class DeviceNF4:
    """An NF4 weight in device memory laid out as one blob (the pool's layer layout)."""

    def __init__(self, rows: int, cols: int, device="cuda"):
        import torch
        from layer_streamed_nf4_b200 import lsnf4
        self.rows, self.cols = rows, cols
        self.blob = torch.zeros(lsnf4.nf4_blob_bytes(rows, cols), dtype=torch.uint8, device=device)
        self.w = lsnf4.nf4_weight_in_blob(rows, cols, self.blob.data_ptr())
        self.layout = lsnf4.nf4_blob_layout(rows, cols)

    def quantize(self, W_f32, stream=None):
        import torch
        from layer_streamed_nf4_b200 import lsnf4
        if isinstance(W_f32, np.ndarray):
            W_f32 = torch.from_numpy(np.ascontiguousarray(W_f32, np.float32)).cuda()
        n = lsnf4.nf4_quantize_ws_bytes(self.rows, self.cols)
        ws = torch.zeros(max(n, 16), dtype=torch.uint8, device=W_f32.device)
        lsnf4.nf4_quantize(W_f32, self.w, ws, n, stream)
        return self

    def arrays(self):
        """packed, absmax_q, s2, offset as host numpy arrays."""
        import torch
        torch.cuda.synchronize()
        b = self.blob.cpu().numpy()
        o = self.layout
        numel = self.rows * self.cols
        nblk = numel // 64
        ngrp = (nblk + 255) // 256
        packed = b[o[0]:o[0] + numel // 2].copy()
        qa = b[o[1]:o[1] + nblk].copy()
        s2 = b[o[2]:o[2] + 4 * ngrp].copy().view(np.float32)
        off = b[o[3]:o[3] + 4].copy().view(np.float32)[0]
        return packed, qa, s2, off


# ------------------------------------------------ inputs built on ties ---
#
# Weights whose quantisation decisions land exactly on the midpoints between
# adjacent levels (and one or two fp32 steps either side), at both levels of
# the format.  Built from the levels and the second-level table with exact
# rational arithmetic; they exercise the "ties go to the lower index" rule
# where a one-ulp disagreement between two implementations would show.

def _f32_neighbours(x, n=2):
    """The fp32 values within n steps of fp32(x) (x a Fraction or float)."""
    f = np.float32(float(x))
    out = [f]
    lo = hi = f
    for _ in range(n):
        lo = np.nextafter(lo, np.float32(-np.inf))
        hi = np.nextafter(hi, np.float32(np.inf))
        out += [lo, hi]
    return out


def first_level_tie_weights(levels, exps=(-6, -1, -20, -100), rows_per_exp=2):
    """Blocks whose absmax is a power of two 2^e (element 0 is +-2^e) and whose other elements are 2^e
    times fp32 values at and around every exact midpoint of adjacent levels, so that w / absmax is that
    value exactly.  Returns fp32 [n_blocks, 64]."""
    from fractions import Fraction
    vals = []
    for a, b in zip(levels[:-1], levels[1:]):
        mid = (Fraction(float(a)) + Fraction(float(b))) / 2
        vals += [v for v in _f32_neighbours(mid) if -1.0 <= float(v) <= 1.0]
    vals = np.array(vals, np.float32)
    blocks = []
    for e in exps:
        scale = np.float32(2.0 ** e)
        for rep in range(rows_per_exp):
            for start in range(0, vals.size, 63):
                chunk = vals[start:start + 63]
                blk = np.zeros(64, np.float32)
                blk[0] = scale if (rep + start) % 2 == 0 else -scale
                blk[1:1 + chunk.size] = chunk * scale
                if chunk.size < 63:                          # pad with the levels themselves
                    pad = np.resize(np.asarray(levels, np.float32), 63 - chunk.size)
                    blk[1 + chunk.size:] = pad * scale
                blocks.append(blk)
    return np.stack(blocks)


def second_level_tie_weights(table, off_exp, s2_exp, m_lo, m_hi, seed=0, ballast_max_exp=-3):
    """A weight whose second-level values v = (absmax - offset) / s2 land exactly on the midpoints of
    adjacent entries of the second-level table within [m_lo, m_hi] (and one or two fp32 steps either
    side).  The offset (mean of all block absmax values) is made exactly 2^off_exp by ballast blocks in
    groups of their own; each tie group holds a block with absmax = offset + 2^s2_exp or offset - 2^s2_exp,
    which makes its s2 exactly 2^s2_exp, so that v = (absmax - offset) * 2^-s2_exp is exact.  Only targets
    whose absmax is an fp32 value and whose subtraction is exact are kept.
    Returns (W fp32 [n_blocks, 64], number of tie groups, list of (block, target v))."""
    from fractions import Fraction
    off = Fraction(2) ** off_exp
    s2 = Fraction(2) ** s2_exp
    targets = []
    for a, b in zip(table[:-1], table[1:]):
        mid = (Fraction(float(a)) + Fraction(float(b))) / 2
        if not (m_lo <= mid <= m_hi):
            continue
        for v in _f32_neighbours(mid):
            am = off + Fraction(float(v)) * s2
            if am < 0 or abs(Fraction(float(v))) > 1:
                continue
            if Fraction(float(np.float32(float(am)))) != am:             # absmax must be an fp32 value
                continue
            targets.append((am, np.float32(v)))
    # anchor of every tie group: |c| = s2 exactly
    anchor = off + s2 if m_hi > 0 else off - s2
    assert anchor >= 0
    per_group = 255
    groups = []
    for i in range(0, len(targets), per_group):
        chunk = targets[i:i + per_group]
        groups.append([anchor] + [t[0] for t in chunk] + [off] * (per_group - len(chunk)))
    n_tie = 256 * len(groups)
    tie_sum = sum(sum(g) for g in groups)
    # ballast: enough blocks for the mean to come out exactly off, absmax values summing to the rest
    cap = Fraction(2) ** ballast_max_exp
    n_total = n_tie + 256
    while n_total * off < tie_sum or (n_total * off - tie_sum) > (n_total - n_tie) * cap:
        n_total += 256
    n_total += 256                                       # room for the pieces that carry the low bits
    rest = n_total * off - tie_sum
    ballast = []
    while rest > 0:
        piece = min(cap, rest)
        f = np.float32(float(piece))
        if Fraction(float(f)) > piece:
            f = np.nextafter(f, np.float32(0))
        ballast.append(Fraction(float(f)))
        rest -= Fraction(float(f))
    ballast += [Fraction(0)] * (n_total - n_tie - len(ballast))
    assert len(ballast) == n_total - n_tie and sum(ballast) + tie_sum == n_total * off
    absmax = [a for g in groups for a in g] + ballast
    rng = np.random.default_rng(seed)
    W = np.zeros((len(absmax), 64), np.float32)
    for bi, am in enumerate(absmax):
        a = np.float32(float(am))
        if a == 0:
            continue
        W[bi] = (rng.uniform(-1, 1, 64) * float(a)).astype(np.float32)
        W[bi] = np.clip(W[bi], -a, a)
        W[bi, rng.integers(0, 64)] = a if bi % 2 else -a
    where = []
    for gi in range(len(groups)):
        for j, t in enumerate(targets[gi * per_group:(gi + 1) * per_group]):
            where.append((gi * 256 + 1 + j, t[1]))
    return W, len(groups), where
