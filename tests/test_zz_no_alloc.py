"""nf4_quantize_noalloc: quantisation for callers that cannot hand the library
device memory (their allocator owns all of it, or an allocation's implicit
synchronisation is not acceptable where they quantise).  It uses a fixed
scratch array inside the library instead of a caller workspace, so its
results must be bit-identical to nf4_quantize's, call after call, and a call
must not change the device's free memory.

This file is collected last on purpose (pytest orders files by name), so a
run that stops at the first failure has already run every other test."""
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


def _pair(lib, W):
    """(blob from nf4_quantize with a workspace, blob from nf4_quantize_noalloc)."""
    import torch
    rows, cols = W.shape
    Wd = W if isinstance(W, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    ref = DeviceNF4(rows, cols).quantize(Wd)
    got = DeviceNF4(rows, cols)
    got.blob.fill_(0xA5)                      # garbage where the result must land
    lib.nf4_quantize_noalloc(Wd, got.w)
    torch.cuda.synchronize()
    return ref, got


def _same(ref, got):
    import torch
    numel = ref.rows * ref.cols
    o = ref.layout
    nblk = numel // 64
    ngrp = (nblk + 255) // 256
    for lo, n in ((o[0], numel // 2), (o[1], nblk), (o[2], 4 * ngrp), (o[3], 4)):
        assert torch.equal(ref.blob[lo:lo + n], got.blob[lo:lo + n])


def test_noalloc_matches_workspace_version_twice_in_a_row(lib):
    W1 = synth.normal_f32((512, 512), 0.02, synth.SEED, 77, 1, synth.T_W)
    W2 = synth.normal_f32((14336, 4096), 0.02, synth.SEED, 77, 2, synth.T_W)   # 58.7M elements, below the limit
    W2[5, :64] = 0.0                                                            # a zero block
    for W in (W1, W2, W1):                   # consecutive calls share the scratch array
        ref, got = _pair(lib, W)
        _same(ref, got)


def test_noalloc_at_exactly_the_limit(lib):
    """A weight of exactly LSN_NF4_NOALLOC_MAX_ELEMS elements (16384 x 4096) fills the scratch array to its
    last absmax and partial sum; the result still equals nf4_quantize's bit for bit."""
    import torch
    rows, cols = 16384, 4096
    assert rows * cols == lib.NF4_NOALLOC_MAX_ELEMS
    W = synth.device_normal((rows, cols), 0.02, synth.SEED, 79, 0, synth.T_W, device=torch.device("cuda", 0))
    W[-1, -64:] *= 40.0                      # the last block and group carry the largest absmax
    ref, got = _pair(lib, W)
    _same(ref, got)


def test_noalloc_leaves_free_memory_unchanged(lib):
    import torch
    W = synth.normal_f32((1024, 1024), 0.02, synth.SEED, 78, 0, synth.T_W)
    Wd = torch.from_numpy(W).cuda()
    d = DeviceNF4(1024, 1024)
    lib.nf4_quantize_noalloc(Wd, d.w)        # first call on this device resolves the scratch address
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        lib.nf4_quantize_noalloc(Wd, d.w)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_weights_above_the_limit(lib):
    rows = lib.NF4_NOALLOC_MAX_ELEMS // 64 + 1
    w = lib.make_nf4_weight(rows, 64, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    with pytest.raises(lib.LsnError) as e:
        lib.nf4_quantize_noalloc(1 << 20, w)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    assert "limit" in str(e.value)
