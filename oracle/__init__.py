"""CPU oracle for the layer-streamed NF4 LoRA linear (fp64, plain loops).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.
It shares no code with the CUDA library (``layer_streamed_nf4_b200``).

Every function wraps one routine of ``oracle.cpp`` through ctypes; arrays are
numpy, bf16 tensors travel as their uint16 bit patterns.  The source cites the
passages of the pages each step follows.  Parity status of each part (what pins
it, see ``tests/test_oracle_*.py``):

* ``ppnd16``            pinned against scipy's ndtri (library routine).
* ``nf4_codebook``      pinned by closed form (exact 0 and +-1, monotone,
                        Phi(c_i * Phi^-1(p_max)) equal to its quantile step).
* ``dq_table``          pinned by its closed form k/127.
* ``nearest_*``         pinned by exact rational arithmetic (fractions).
* ``nf4_quantize``      pinned by exact round trips on codebook points, by the
                        equal-absmax special case, by the second-level error
                        bound and by an exact-rational recomputation on small
                        inputs.
* ``nf4_dequant``       pinned by the same round trips.
* ``lora_fwd`` / ``lora_bwd_*``  pinned by numpy matmul (B = 0 and merged
                        weights W + s B A) and by central finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_OUT_DIR = os.path.join(_HERE, "_build")
_SO = os.path.join(_OUT_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``oracle.cpp`` into ``_build/liboracle.so`` (g++, OpenMP)."""
    with _lock:
        if (not force and os.path.exists(_SO)
                and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
            return _SO
        os.makedirs(_OUT_DIR, exist_ok=True)
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC])
        os.replace(tmp, _SO)
        return _SO


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    lib.orc_ppnd16.restype = ctypes.c_double
    lib.orc_ppnd16.argtypes = [ctypes.c_double]
    lib.orc_nf4_codebook.argtypes = [_f32p]
    lib.orc_dq_table.argtypes = [_f32p]
    lib.orc_f32_to_bf16.restype = ctypes.c_uint16
    lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.orc_nearest_nf4.restype = ctypes.c_int
    lib.orc_nearest_nf4.argtypes = [ctypes.c_float]
    lib.orc_nearest_dq.restype = ctypes.c_int
    lib.orc_nearest_dq.argtypes = [ctypes.c_float]
    lib.orc_nf4_quantize.restype = ctypes.c_int
    lib.orc_nf4_quantize.argtypes = [_f32p, ctypes.c_int64, _u8p, _u8p, _f32p, _f32p, _f32p]
    lib.orc_absmax_hat.restype = ctypes.c_float
    lib.orc_absmax_hat.argtypes = [_u8p, _f32p, ctypes.c_float, ctypes.c_int64]
    lib.orc_nf4_dequant.argtypes = [_u8p, _u8p, _f32p, ctypes.c_float, ctypes.c_int64, _u16p]
    common = [_u16p, _u16p, _u16p, _u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
              ctypes.c_int64, ctypes.c_double]
    lib.orc_lora_fwd.argtypes = common + [_i64p, ctypes.c_int64, _f64p]
    lib.orc_lora_bwd_dx.argtypes = common + [_i64p, ctypes.c_int64, _f64p]
    lib.orc_lora_bwd_dadb.argtypes = common + [_f64p, _f64p]
    lib.orc_threads.restype = ctypes.c_int
    lib.orc_threads.argtypes = []
    _lib = lib
    return lib


def _p(a: np.ndarray, typ):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(typ)


# ----------------------------------------------------------------- codec ---

def threads() -> int:
    """Threads the oracle's OpenMP loops run on in this process."""
    return int(_load().orc_threads())


def ppnd16(p: float) -> float:
    return float(_load().orc_ppnd16(float(p)))


def nf4_codebook() -> np.ndarray:
    out = np.zeros(16, np.float32)
    _load().orc_nf4_codebook(_p(out, _f32p))
    return out


def dq_table() -> np.ndarray:
    out = np.zeros(256, np.float32)
    _load().orc_dq_table(_p(out, _f32p))
    return out


def f32_to_bf16_bits(v: float) -> int:
    return int(_load().orc_f32_to_bf16(float(np.float32(v))))


def nearest_nf4(v: float) -> int:
    return int(_load().orc_nearest_nf4(float(np.float32(v))))


def nearest_dq(v: float) -> int:
    return int(_load().orc_nearest_dq(float(np.float32(v))))


def nblocks(numel: int) -> int:
    return numel // 64


def ngroups(numel: int) -> int:
    return (numel // 64 + 255) // 256


def nf4_quantize(W: np.ndarray, want_absmax: bool = False):
    """NF4 + double quantisation of an fp32 weight (numel % 64 == 0).

    Returns a dict: packed uint8 [numel/2], absmax_q uint8 [nblk],
    s2 float32 [ngroups], offset float (fp32 value), and, if asked, the exact
    first-level absmax float32 [nblk].
    """
    W = np.ascontiguousarray(W, dtype=np.float32).reshape(-1)
    n = W.size
    if n % 64:
        raise ValueError("numel must be a multiple of 64")
    packed = np.zeros(n // 2, np.uint8)
    qa = np.zeros(nblocks(n), np.uint8)
    s2 = np.zeros(ngroups(n), np.float32)
    off = np.zeros(1, np.float32)
    am = np.zeros(nblocks(n), np.float32)
    rc = _load().orc_nf4_quantize(_p(W, _f32p), n, _p(packed, _u8p), _p(qa, _u8p), _p(s2, _f32p),
                                  _p(off, _f32p), _p(am, _f32p))
    if rc != 0:
        raise ValueError("oracle nf4_quantize rejected the input (non-finite value)")
    out = {"packed": packed, "absmax_q": qa, "s2": s2, "offset": np.float32(off[0])}
    if want_absmax:
        out["absmax"] = am
    return out


def absmax_hat(absmax_q: np.ndarray, s2: np.ndarray, offset, b: int) -> np.float32:
    qa = np.ascontiguousarray(absmax_q, np.uint8)
    s = np.ascontiguousarray(s2, np.float32)
    return np.float32(_load().orc_absmax_hat(_p(qa, _u8p), _p(s, _f32p), float(offset), int(b)))


def nf4_dequant(packed: np.ndarray, absmax_q: np.ndarray, s2: np.ndarray, offset, numel: int) -> np.ndarray:
    """Dequantise to bf16 bit patterns (uint16 [numel])."""
    packed = np.ascontiguousarray(packed, np.uint8)
    absmax_q = np.ascontiguousarray(absmax_q, np.uint8)
    s2 = np.ascontiguousarray(s2, np.float32)
    out = np.zeros(numel, np.uint16)
    _load().orc_nf4_dequant(_p(packed, _u8p), _p(absmax_q, _u8p), _p(s2, _f32p), float(offset),
                            int(numel), _p(out, _u16p))
    return out


# ----------------------------------------------------------- LoRA linear ---

def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 tensors are passed as uint16 bit patterns"
    return a


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, r.size


def lora_fwd(x, W, A, B, s: float, rows=None) -> np.ndarray:
    """y = x W^T + s (x A^T) B^T in fp64; x [T,K], W [N,K], A [r,K], B [N,r] (bf16 bits)."""
    x, W, A, B = _u16(x), _u16(W), _u16(A), _u16(B)
    T, K = x.shape
    N = W.shape[0]
    r = A.shape[0]
    rr, nr = _rows(rows)
    y = np.zeros((nr if rr is not None else T, N), np.float64)
    _load().orc_lora_fwd(_p(x, _u16p), _p(W, _u16p), _p(A, _u16p), _p(B, _u16p), T, K, N, r, float(s),
                         _p(rr, _i64p) if rr is not None else None, nr, _p(y, _f64p))
    return y


def lora_bwd_dx(dY, W, A, B, s: float, rows=None) -> np.ndarray:
    """dX = dY W + s (dY B) A in fp64."""
    dY, W, A, B = _u16(dY), _u16(W), _u16(A), _u16(B)
    T, N = dY.shape
    K = W.shape[1]
    r = A.shape[0]
    rr, nr = _rows(rows)
    dX = np.zeros((nr if rr is not None else T, K), np.float64)
    _load().orc_lora_bwd_dx(_p(dY, _u16p), _p(W, _u16p), _p(A, _u16p), _p(B, _u16p), T, K, N, r, float(s),
                            _p(rr, _i64p) if rr is not None else None, nr, _p(dX, _f64p))
    return dX


def lora_bwd_dadb(x, dY, A, B, s: float):
    """dA = s (dY B)^T x [r,K] and dB = s dY^T (x A^T) [N,r] in fp64."""
    x, dY, A, B = _u16(x), _u16(dY), _u16(A), _u16(B)
    T, K = x.shape
    N = dY.shape[1]
    r = A.shape[0]
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    _load().orc_lora_bwd_dadb(_p(x, _u16p), _p(dY, _u16p), _p(A, _u16p), _p(B, _u16p), T, K, N, r,
                              float(s), _p(dA, _f64p), _p(dB, _f64p))
    return dA, dB
