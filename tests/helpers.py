"""Test helpers: tolerance metrics and device-side setup through the C ABI."""
from __future__ import annotations

import numpy as np

# Tolerances on floating-point outputs (y, dX, dA, dB) against the fp64
# oracle, per tensor: relative Frobenius error and max-abs error in units of
# the oracle's RMS.
REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2


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
