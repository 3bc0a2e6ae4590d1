"""ctypes binding of liblsnf4.so (the C ABI in ``include/lsnf4.h``).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Functions keep the C names; tensors may be passed as torch tensors
(their ``data_ptr()`` is used, they must be contiguous CUDA tensors) or as raw
integer device addresses.  ``stream`` defaults to torch's current CUDA stream.
A failing call raises :class:`LsnError` with the library's message.

If the shared library is missing this module raises on import: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("LSNF4_LIB", os.path.join(HERE, "liblsnf4.so"))

if not os.path.exists(LIB_PATH):
    raise ImportError(f"liblsnf4.so not found at {LIB_PATH}; build it with "
                      f"`python -m layer_streamed_nf4_b200.build` (there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

LSN_OK, LSN_ERR_INVALID_ARG, LSN_ERR_CUDA, LSN_ERR_NO_MEMORY, LSN_ERR_TIMEOUT, LSN_ERR_UNSUPPORTED, LSN_ERR_STATE = range(7)
LSN_BASE_NF4, LSN_BASE_BF16 = 0, 1
LSN_POOL_FAULT_NONE, LSN_POOL_FAULT_STALE_SLOT, LSN_POOL_FAULT_COPY_ERROR = 0, 1, 2
LSN_POOL_DEBUG_POISON = 1
LSN_OPT_FUSED_NF4 = 1
LSN_OPT_LAYER_LANES = 2
LSN_OPT_PDL = 3
LSN_OPT_STREAM_K = 4
LSN_OPT_GEMM_MIN_UNITS = 5
LSN_OPT_DEQUANT_SPARE_SMS = 6
LSN_OPT_GEMM_TAIL_SPLIT = 7
LSN_OPT_LAYER_MERGE = 8

STATUS_NAMES = {0: "LSN_OK", 1: "LSN_ERR_INVALID_ARG", 2: "LSN_ERR_CUDA", 3: "LSN_ERR_NO_MEMORY",
                4: "LSN_ERR_TIMEOUT", 5: "LSN_ERR_UNSUPPORTED", 6: "LSN_ERR_STATE"}

# Every symbol the header declares (checked by the CPU test-suite).
EXPORTS = (
    "lsn_last_error", "lsn_version", "lsn_nf4_codebook", "lsn_dq_codebook",
    "lsn_nf4_packed_bytes", "lsn_nf4_absmax_bytes", "lsn_nf4_s2_bytes", "lsn_nf4_blob_bytes",
    "lsn_nf4_blob_layout", "lsn_nf4_quantize_ws_bytes", "nf4_quantize", "nf4_dequant",
    "lsn_lora_ws_bytes", "lora_linear_fwd", "lora_linear_bwd", "lsn_ws_status",
    "layer_pool_create", "layer_pool_register", "layer_pool_prefetch", "layer_pool_acquire",
    "layer_pool_release", "layer_pool_wait_idle", "layer_pool_stats", "layer_pool_reset",
    "layer_pool_inject_fault", "layer_pool_destroy", "lsn_timing_enable", "lsn_timing_read",
    "nf4_quantize_noalloc", "lsn_set_option", "lsn_get_option", "lsn_gemm_merged_schedule",
    "lsn_layer_ws_bytes", "lora_layer_fwd", "lora_layer_bwd", "nf4_dequant_batch",
    "lsn_selftest_wait_timeout", "layer_pool_set_debug",
)


class LsnError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class NF4Weight(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("packed", ctypes.c_void_p),
                ("absmax_q", ctypes.c_void_p), ("absmax_s2", ctypes.c_void_p), ("offset", ctypes.c_void_p)]


class Base(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("nf4", NF4Weight), ("bf16", ctypes.c_void_p)]


class LoraProj(ctypes.Structure):
    """One projection of a layer call (lsn_lora_proj)."""
    _fields_ = [("W", Base), ("x", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("dY", ctypes.c_void_p), ("dX", ctypes.c_void_p), ("dA", ctypes.c_void_p),
                ("dB", ctypes.c_void_p), ("u", ctypes.c_void_p), ("group", ctypes.c_int)]


LSN_LAYER_MAX_PROJ = 16

KERNEL_KINDS = ("gemm_fwd", "gemm_bwd", "dequant", "lora_down", "lora_tgrad", "quantize")


class KernelTiming(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_uint64 * 6), ("kernels", ctypes.c_uint64 * 6), ("ms", ctypes.c_double * 6),
                ("work", ctypes.c_double * 6)]


class PoolStats(ctypes.Structure):
    _fields_ = [("copies", ctypes.c_uint64), ("bytes_copied", ctypes.c_uint64), ("hits", ctypes.c_uint64),
                ("misses", ctypes.c_uint64), ("copy_ms", ctypes.c_double)]


_vp, _i64, _sz, _i = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("lsn_last_error", ctypes.c_char_p, [])
_sig("lsn_version", _i, [])
_sig("lsn_nf4_codebook", None, [ctypes.POINTER(ctypes.c_float)])
_sig("lsn_dq_codebook", None, [ctypes.POINTER(ctypes.c_float)])
for _n in ("lsn_nf4_packed_bytes", "lsn_nf4_absmax_bytes", "lsn_nf4_s2_bytes", "lsn_nf4_blob_bytes",
           "lsn_nf4_quantize_ws_bytes"):
    _sig(_n, _sz, [_i64, _i64])
_sig("lsn_nf4_blob_layout", None, [_i64, _i64, ctypes.POINTER(_sz)])
_sig("nf4_quantize", _i, [_vp, ctypes.POINTER(NF4Weight), _vp, _sz, _vp])
_sig("nf4_dequant", _i, [ctypes.POINTER(NF4Weight), _vp, _vp])
_sig("nf4_dequant_batch", _i, [_i, ctypes.POINTER(NF4Weight), ctypes.POINTER(_vp), _i, _vp])
_sig("nf4_quantize_noalloc", _i, [_vp, ctypes.POINTER(NF4Weight), _vp])
_sig("lsn_lora_ws_bytes", _sz, [_i64, _i64, _i64, _i, _i])
_sig("lora_linear_fwd", _i, [ctypes.POINTER(Base), _vp, _i64, _vp, _vp, _i, ctypes.c_float, _vp, _vp, _sz, _vp])
_sig("lora_linear_bwd", _i, [ctypes.POINTER(Base), _vp, _vp, _i64, _vp, _vp, _i, ctypes.c_float, _vp, _vp, _vp, _i,
                             _vp, _sz, _vp])
_sig("lsn_ws_status", _i, [_vp, _vp])
_sig("lsn_selftest_wait_timeout", _i, [_i, _vp])
_sig("lsn_layer_ws_bytes", _sz, [_i, ctypes.POINTER(LoraProj), _i64, _i])
_sig("lora_layer_fwd", _i, [_i, ctypes.POINTER(LoraProj), _i64, _i, ctypes.c_float, _vp, _sz, _vp])
_sig("lora_layer_bwd", _i, [_i, ctypes.POINTER(LoraProj), _i64, _i, ctypes.c_float, _i, _vp, _sz, _vp])
_sig("lsn_set_option", _i, [_i, _i])
_sig("lsn_get_option", _i, [_i])
_IP = ctypes.POINTER(ctypes.c_int)
_sig("lsn_gemm_merged_schedule", _i, [_i, _i, _IP, _IP, _IP, _IP, _i])
_sig("lsn_timing_enable", _i, [_i])
_sig("lsn_timing_read", _i, [ctypes.POINTER(KernelTiming)])
_sig("layer_pool_create", _i, [_i, _sz, _i, ctypes.POINTER(_vp)])
_sig("layer_pool_register", _i, [_vp, _i, _vp, _sz])
_sig("layer_pool_prefetch", _i, [_vp, _i])
_sig("layer_pool_acquire", _i, [_vp, _i, _vp, ctypes.POINTER(_vp)])
_sig("layer_pool_release", _i, [_vp, _i, _vp])
_sig("layer_pool_wait_idle", _i, [_vp, _i])
_sig("layer_pool_stats", _i, [_vp, ctypes.POINTER(PoolStats)])
_sig("layer_pool_reset", _i, [_vp])
_sig("layer_pool_inject_fault", _i, [_vp, _i])
_sig("layer_pool_set_debug", _i, [_vp, _i])
_sig("layer_pool_destroy", None, [_vp])


def lib_path() -> str:
    return LIB_PATH


def last_error() -> str:
    return _lib.lsn_last_error().decode(errors="replace")


def _check(st: int, where: str):
    if st != LSN_OK:
        raise LsnError(st, where, last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------- codec ---

def version() -> int:
    return _lib.lsn_version()


def nf4_codebook():
    out = (ctypes.c_float * 16)()
    _lib.lsn_nf4_codebook(out)
    return list(out)


def dq_codebook():
    out = (ctypes.c_float * 256)()
    _lib.lsn_dq_codebook(out)
    return list(out)


def nf4_packed_bytes(rows, cols): return _lib.lsn_nf4_packed_bytes(rows, cols)
def nf4_absmax_bytes(rows, cols): return _lib.lsn_nf4_absmax_bytes(rows, cols)
def nf4_s2_bytes(rows, cols): return _lib.lsn_nf4_s2_bytes(rows, cols)
def nf4_blob_bytes(rows, cols): return _lib.lsn_nf4_blob_bytes(rows, cols)
def nf4_quantize_ws_bytes(rows, cols): return _lib.lsn_nf4_quantize_ws_bytes(rows, cols)


def nf4_blob_layout(rows, cols):
    out = (_sz * 4)()
    _lib.lsn_nf4_blob_layout(rows, cols, out)
    return list(out)


def make_nf4_weight(rows, cols, packed, absmax_q, absmax_s2, offset) -> NF4Weight:
    return NF4Weight(rows, cols, _ptr(packed), _ptr(absmax_q), _ptr(absmax_s2), _ptr(offset))


def nf4_weight_in_blob(rows, cols, base_addr: int) -> NF4Weight:
    """View of an NF4 weight stored at ``base_addr`` in the blob layout."""
    o = nf4_blob_layout(rows, cols)
    return NF4Weight(rows, cols, base_addr + o[0], base_addr + o[1], base_addr + o[2], base_addr + o[3])


def nf4_quantize(W, out: NF4Weight, ws, ws_bytes: int, stream=None):
    _check(_lib.nf4_quantize(_ptr(W), ctypes.byref(out), _ptr(ws), ws_bytes, _stream(stream)), "nf4_quantize")


def nf4_quantize_noalloc(W, out: NF4Weight, stream=None):
    """nf4_quantize with the library's fixed scratch array instead of a workspace (see lsnf4.h)."""
    _check(_lib.nf4_quantize_noalloc(_ptr(W), ctypes.byref(out), _stream(stream)), "nf4_quantize_noalloc")


NF4_NOALLOC_MAX_ELEMS = 1 << 26


def nf4_dequant(w: NF4Weight, W_out, stream=None):
    _check(_lib.nf4_dequant(ctypes.byref(w), _ptr(W_out), _stream(stream)), "nf4_dequant")


def dequant_batch_args(weights, outs):
    """(n, weight array, output-pointer array) for nf4_dequant_batch; keep the arrays alive while used."""
    n = len(weights)
    return n, (NF4Weight * n)(*weights), (ctypes.c_void_p * n)(*[_ptr(o) for o in outs])


def nf4_dequant_batch(weights, outs, blocks_per_sm: int = 0, stream=None):
    n, wa, oa = dequant_batch_args(weights, outs)
    _check(_lib.nf4_dequant_batch(n, wa, oa, blocks_per_sm, _stream(stream)), "nf4_dequant_batch")


# --------------------------------------------------------- LoRA linear ---

def base_nf4(w: NF4Weight) -> Base:
    return Base(LSN_BASE_NF4, w.rows, w.cols, w, None)


def base_bf16(W, rows: int, cols: int) -> Base:
    return Base(LSN_BASE_BF16, rows, cols, NF4Weight(), _ptr(W))


def lora_ws_bytes(T, K, N, r, kind) -> int:
    return _lib.lsn_lora_ws_bytes(T, K, N, r, kind)


def lora_linear_fwd(W: Base, x, T: int, A, B, r: int, scale: float, y, ws, ws_bytes: int, stream=None):
    _check(_lib.lora_linear_fwd(ctypes.byref(W), _ptr(x), T, _ptr(A), _ptr(B), r, scale, _ptr(y), _ptr(ws),
                                ws_bytes, _stream(stream)), "lora_linear_fwd")


def lora_linear_bwd(W: Base, x, dY, T: int, A, B, r: int, scale: float, dX, dA, dB, accumulate: bool, ws,
                    ws_bytes: int, stream=None):
    _check(_lib.lora_linear_bwd(ctypes.byref(W), _ptr(x), _ptr(dY), T, _ptr(A), _ptr(B), r, scale, _ptr(dX),
                                _ptr(dA), _ptr(dB), int(bool(accumulate)), _ptr(ws), ws_bytes, _stream(stream)),
           "lora_linear_bwd")


# ------------------------------------------------------------ whole layer ---

def lora_proj(W: Base, x, A, B, y=None, dY=None, dX=None, dA=None, dB=None, u=None, group: int = 0) -> LoraProj:
    return LoraProj(W, _ptr(x), _ptr(A), _ptr(B), _ptr(y), _ptr(dY), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(u), group)


def proj_array(projs) -> ctypes.Array:
    return (LoraProj * len(projs))(*projs)


def layer_ws_bytes(projs, T: int, r: int) -> int:
    arr = projs if isinstance(projs, ctypes.Array) else proj_array(projs)
    return _lib.lsn_layer_ws_bytes(len(arr), arr, T, r)


def lora_layer_fwd(projs, T: int, r: int, scale: float, ws, ws_bytes: int, stream=None):
    arr = projs if isinstance(projs, ctypes.Array) else proj_array(projs)
    _check(_lib.lora_layer_fwd(len(arr), arr, T, r, scale, _ptr(ws), ws_bytes, _stream(stream)), "lora_layer_fwd")


def lora_layer_bwd(projs, T: int, r: int, scale: float, accumulate: bool, ws, ws_bytes: int, stream=None):
    arr = projs if isinstance(projs, ctypes.Array) else proj_array(projs)
    _check(_lib.lora_layer_bwd(len(arr), arr, T, r, scale, int(bool(accumulate)), _ptr(ws), ws_bytes,
                               _stream(stream)), "lora_layer_bwd")


def selftest_wait_timeout(limit_us: int = 1000, stream=None) -> int:
    """Status of the bounded-wait self-test: LSN_ERR_TIMEOUT is the expected outcome."""
    return _lib.lsn_selftest_wait_timeout(limit_us, _stream(stream))


def ws_status(ws, stream=None):
    _check(_lib.lsn_ws_status(_ptr(ws), _stream(stream)), "lsn_ws_status")


# -------------------------------------------------------------- options ---

def set_option(option: int, value: int):
    _check(_lib.lsn_set_option(option, int(value)), "lsn_set_option")


def get_option(option: int) -> int:
    return int(_lib.lsn_get_option(option))


def gemm_merged_schedule(units: int, ntiles, cost):
    """The merged GEMM launch's tile lists: one list of tile numbers per worker (host-only call)."""
    n = len(ntiles)
    total = int(sum(ntiles))
    nt = (ctypes.c_int * n)(*ntiles)
    cs = (ctypes.c_int * n)(*cost)
    start = (ctypes.c_int * (units + 1))()
    tile = (ctypes.c_int * max(total, 1))()
    _check(_lib.lsn_gemm_merged_schedule(units, n, nt, cs, start, tile, total), "lsn_gemm_merged_schedule")
    return [list(tile[start[u]:start[u + 1]]) for u in range(units)]


# -------------------------------------------------------- kernel timing ---

def timing_enable(on: bool = True):
    _check(_lib.lsn_timing_enable(int(bool(on))), "lsn_timing_enable")


def timing_read() -> dict:
    """Per kernel kind: launches, summed device ms, summed algorithmic work (flop or bytes)."""
    t = KernelTiming()
    _check(_lib.lsn_timing_read(ctypes.byref(t)), "lsn_timing_read")
    return {k: {"launches": int(t.launches[i]), "kernels": int(t.kernels[i]), "ms": float(t.ms[i]),
                "work": float(t.work[i])} for i, k in enumerate(KERNEL_KINDS)}


# ---------------------------------------------------------- layer pool ---

def layer_pool_create(n_slots: int, slot_bytes: int, device: int = 0) -> int:
    h = _vp()
    _check(_lib.layer_pool_create(n_slots, slot_bytes, device, ctypes.byref(h)), "layer_pool_create")
    return h.value


def layer_pool_register(pool: int, layer: int, host_pinned, nbytes: int):
    _check(_lib.layer_pool_register(pool, layer, _ptr(host_pinned), nbytes), "layer_pool_register")


def layer_pool_prefetch(pool: int, layer: int):
    _check(_lib.layer_pool_prefetch(pool, layer), "layer_pool_prefetch")


def layer_pool_acquire(pool: int, layer: int, stream=None) -> int:
    p = _vp()
    _check(_lib.layer_pool_acquire(pool, layer, _stream(stream), ctypes.byref(p)), "layer_pool_acquire")
    return p.value


def layer_pool_release(pool: int, layer: int, stream=None):
    _check(_lib.layer_pool_release(pool, layer, _stream(stream)), "layer_pool_release")


def layer_pool_wait_idle(pool: int, timeout_ms: int):
    _check(_lib.layer_pool_wait_idle(pool, timeout_ms), "layer_pool_wait_idle")


def layer_pool_stats(pool: int) -> dict:
    s = PoolStats()
    _check(_lib.layer_pool_stats(pool, ctypes.byref(s)), "layer_pool_stats")
    return {"copies": s.copies, "bytes_copied": s.bytes_copied, "hits": s.hits, "misses": s.misses,
            "copy_ms": s.copy_ms}


def layer_pool_reset(pool: int):
    _check(_lib.layer_pool_reset(pool), "layer_pool_reset")


def layer_pool_inject_fault(pool: int, fault: int):
    _check(_lib.layer_pool_inject_fault(pool, fault), "layer_pool_inject_fault")


def layer_pool_set_debug(pool: int, flags: int):
    _check(_lib.layer_pool_set_debug(pool, flags), "layer_pool_set_debug")


def layer_pool_destroy(pool: int):
    _lib.layer_pool_destroy(pool)
