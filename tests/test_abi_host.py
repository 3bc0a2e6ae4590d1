"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and its host-side logic (tables, sizes, argument checks) is right.
No call here launches GPU work."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from layer_streamed_nf4_b200 import build
    build.build()
    from layer_streamed_nf4_b200 import lsnf4
    return lsnf4


def _header_functions():
    src = open(os.path.join(ROOT, "include", "lsnf4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set()
    for m in re.finditer(r"^\s*(?:const\s+)?[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M):
        name = m.group(1)
        if name not in ("defined",):
            names.add(name)
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _header_functions()
    assert len(declared) >= 25, declared
    so = ctypes.CDLL(lib.lib_path())
    missing = [n for n in sorted(declared) if not hasattr(so, n)]
    assert not missing, missing
    assert set(lib.EXPORTS) == declared


def test_codebook_matches_oracle_bitwise(lib, orc):
    got = np.array(lib.nf4_codebook(), np.float32)
    assert np.array_equal(got.view(np.uint32), orc.nf4_codebook().view(np.uint32))
    dq = np.array(lib.dq_codebook(), np.float32)
    assert np.array_equal(dq.view(np.uint32), orc.dq_table().view(np.uint32))


def test_sizes_and_blob_layout(lib):
    rows, cols = 14336, 4096
    assert lib.nf4_packed_bytes(rows, cols) == rows * cols // 2
    assert lib.nf4_absmax_bytes(rows, cols) == rows * cols // 64
    assert lib.nf4_s2_bytes(rows, cols) == 4 * ((rows * cols // 64 + 255) // 256)
    o = lib.nf4_blob_layout(rows, cols)
    assert all(v % 1024 == 0 for v in o)
    assert o[0] == 0 and o[1] >= rows * cols // 2 and o[2] - o[1] >= rows * cols // 64
    assert lib.nf4_blob_bytes(rows, cols) == o[3] + 1024
    # workspace grows with the problem and covers the dequantised base for NF4
    small = lib.lora_ws_bytes(256, 512, 512, 8, lib.LSN_BASE_BF16)
    big = lib.lora_ws_bytes(256, 512, 512, 8, lib.LSN_BASE_NF4)
    assert big >= small + 512 * 512 * 2


@pytest.mark.parametrize("r", [0, 4, 7, 72])
def test_bad_rank_is_rejected_before_any_launch(lib, r):
    W = lib.base_bf16(1 << 20, 512, 512)
    with pytest.raises(lib.LsnError) as e:
        lib.lora_linear_fwd(W, 1 << 20, 16, 1 << 20, 1 << 20, r, 2.0, 1 << 20, 1 << 20, 1 << 30, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG


def test_bad_shapes_and_pointers_are_rejected(lib):
    W = lib.base_bf16(1 << 20, 500, 512)                       # N not a multiple of 64
    with pytest.raises(lib.LsnError) as e:
        lib.lora_linear_fwd(W, 1 << 20, 16, 1 << 20, 1 << 20, 8, 2.0, 1 << 20, 1 << 20, 1 << 30, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    W = lib.base_bf16(1 << 20, 512, 512)
    with pytest.raises(lib.LsnError) as e:                     # misaligned x
        lib.lora_linear_fwd(W, (1 << 20) + 2, 16, 1 << 20, 1 << 20, 8, 2.0, 1 << 20, 1 << 20, 1 << 30, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    with pytest.raises(lib.LsnError) as e:                     # workspace too small
        lib.lora_linear_fwd(W, 1 << 20, 16, 1 << 20, 1 << 20, 8, 2.0, 1 << 20, 1 << 20, 64, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    w = lib.make_nf4_weight(64, 100, 1 << 20, 1 << 20, 1 << 20, 1 << 20)   # cols % 64 != 0
    with pytest.raises(lib.LsnError) as e:
        lib.nf4_dequant(w, 1 << 20, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    w = lib.make_nf4_weight(64, 128, None, 1 << 20, 1 << 20, 1 << 20)       # NULL packed
    with pytest.raises(lib.LsnError) as e:
        lib.nf4_dequant(w, 1 << 20, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG


def test_empty_weight_is_a_no_op(lib):
    w = lib.make_nf4_weight(0, 64, None, None, None, None)
    lib.nf4_dequant(w, None, stream=0)


def test_pool_rejects_bad_arguments(lib):
    with pytest.raises(lib.LsnError) as e:
        lib.layer_pool_create(0, 1024, 0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    with pytest.raises(lib.LsnError) as e:
        lib.layer_pool_create(2, 0, 0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG


@pytest.mark.parametrize("T", [0, 1, 63, 64, 2048, 100000])
@pytest.mark.parametrize("K,N", [(64, 64), (896, 4864), (4096, 1024), (14336, 4096)])
def test_workspace_sizes_for_edge_shapes(lib, T, K, N):
    for r in (8, 16, 64):
        for kind in (lib.LSN_BASE_NF4, lib.LSN_BASE_BF16):
            n = lib.lora_ws_bytes(T, K, N, r, kind)
            assert n >= 256 + (N * K * 2 if kind == lib.LSN_BASE_NF4 else 0)


def test_last_error_is_never_null(lib):
    assert isinstance(lib.last_error(), str)
    assert lib.version() >= 100


def test_struct_layouts_match_the_header(lib, tmp_path):
    """ctypes' view of the ABI structs equals the C compiler's (sizes and field offsets)."""
    import ctypes
    import subprocess
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "lsnf4.h"\n'
        "int main(void) {\n"
        '  printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(lsn_nf4_weight), sizeof(lsn_base), sizeof(lsn_lora_proj),\n'
        "         offsetof(lsn_base, nf4), offsetof(lsn_lora_proj, x), offsetof(lsn_lora_proj, u),\n"
        "         offsetof(lsn_lora_proj, group));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [ctypes.sizeof(lib.NF4Weight), ctypes.sizeof(lib.Base), ctypes.sizeof(lib.LoraProj),
            lib.Base.nf4.offset, lib.LoraProj.x.offset, lib.LoraProj.u.offset, lib.LoraProj.group.offset]
    assert got == want


def test_a_c_program_links_and_calls_the_library(lib, tmp_path):
    """The ABI from C alone: a program built against the header and linked to the .so calls the host-side
    entry points (version, the NF4 levels, the blob layout, an argument error with its message)."""
    import subprocess
    src = tmp_path / "use.c"
    src.write_text(
        '#include <stdio.h>\n#include <stdlib.h>\n#include "lsnf4.h"\n'
        "int main(void) {\n"
        "  float lv[16]; size_t o[4];\n"
        "  lsn_nf4_codebook(lv);\n"
        "  lsn_nf4_blob_layout(4096, 14336, o);\n"
        "  lsn_nf4_weight w = {64, 100, 0, 0, 0, 0};\n"
        "  lsn_status st = nf4_dequant(&w, 0, 0);\n"
        '  printf("%d %.9g %.9g %.9g %zu %zu %zu %zu %zu %d %s\\n", lsn_version(), lv[0], lv[7], lv[15],\n'
        "         o[0], o[1], o[2], o[3], lsn_nf4_blob_bytes(4096, 14336), (int)st,\n"
        '         lsn_last_error()[0] ? "message" : "empty");\n'
        "  return 0;\n}\n")
    exe = tmp_path / "use"
    libdir = os.path.dirname(lib.lib_path())
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-llsnf4",
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert int(out[0]) == lib.version()
    assert [float(v) for v in out[1:4]] == [-1.0, 0.0, 1.0]
    assert [int(v) for v in out[4:8]] == lib.nf4_blob_layout(4096, 14336)
    assert int(out[8]) == lib.nf4_blob_bytes(4096, 14336)
    assert int(out[9]) == lib.LSN_ERR_INVALID_ARG and out[10] == "message"


def _fake_projs(lib, shapes, kind):
    projs = []
    for K, N in shapes:
        if kind == lib.LSN_BASE_NF4:
            base = lib.base_nf4(lib.make_nf4_weight(N, K, 1 << 20, 1 << 20, 1 << 20, 1 << 20))
        else:
            base = lib.base_bf16(1 << 20, N, K)
        projs.append(lib.lora_proj(base, 1 << 20, 1 << 20, 1 << 20, y=1 << 20, dY=1 << 20, dX=1 << 20, dA=1 << 20,
                                   dB=1 << 20))
    return projs


def test_layer_workspace_sizes(lib):
    shapes = [(4096, 4096), (4096, 1024), (4096, 1024), (4096, 4096), (4096, 14336), (4096, 14336), (14336, 4096)]
    nf4 = lib.layer_ws_bytes(_fake_projs(lib, shapes, lib.LSN_BASE_NF4), 2048, 16)
    bf = lib.layer_ws_bytes(_fake_projs(lib, shapes, lib.LSN_BASE_BF16), 2048, 16)
    assert nf4 - bf == sum(K * N * 2 for K, N in shapes)         # the dequantised copies
    assert bf >= 256 + 7 * 2048 * 16 * (2 + 4 + 4)
    assert lib.layer_ws_bytes(_fake_projs(lib, shapes, lib.LSN_BASE_BF16), 2048, 12) == 0    # bad rank
    assert lib.layer_ws_bytes(_fake_projs(lib, shapes * 3, lib.LSN_BASE_BF16), 2048, 16) == 0  # n > 16


def test_layer_calls_reject_bad_arguments(lib):
    projs = _fake_projs(lib, [(256, 256), (256, 64)], lib.LSN_BASE_BF16)
    need = lib.layer_ws_bytes(projs, 128, 8)
    with pytest.raises(lib.LsnError) as e:                        # workspace too small
        lib.lora_layer_fwd(projs, 128, 8, 2.0, 1 << 20, need - 1, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    bad = _fake_projs(lib, [(256, 256), (256, 100)], lib.LSN_BASE_BF16)   # N % 64 != 0
    with pytest.raises(lib.LsnError) as e:
        lib.lora_layer_bwd(bad, 128, 8, 2.0, False, 1 << 20, 1 << 30, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    mis = _fake_projs(lib, [(256, 256)], lib.LSN_BASE_BF16)
    mis[0].u = (1 << 20) + 4                                       # misaligned u
    with pytest.raises(lib.LsnError) as e:
        lib.lora_layer_fwd(mis, 128, 8, 2.0, 1 << 20, 1 << 30, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    with pytest.raises(lib.LsnError) as e:                        # empty projection list
        lib.lora_layer_fwd(lib.proj_array([]), 128, 8, 2.0, 1 << 20, 1 << 30, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG


def test_options(lib):
    assert lib.get_option(lib.LSN_OPT_LAYER_LANES) == 2
    with pytest.raises(lib.LsnError) as e:
        lib.set_option(lib.LSN_OPT_LAYER_LANES, 3)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    lib.set_option(lib.LSN_OPT_LAYER_LANES, 1)
    assert lib.get_option(lib.LSN_OPT_LAYER_LANES) == 1
    lib.set_option(lib.LSN_OPT_LAYER_LANES, 2)
    assert lib.get_option(lib.LSN_OPT_FUSED_NF4) == 0
    assert lib.get_option(lib.LSN_OPT_PDL) == 1
    lib.set_option(lib.LSN_OPT_PDL, 0)
    assert lib.get_option(lib.LSN_OPT_PDL) == 0
    lib.set_option(lib.LSN_OPT_PDL, 1)
    assert lib.get_option(lib.LSN_OPT_STREAM_K) == 0
    assert lib.get_option(lib.LSN_OPT_GEMM_MIN_UNITS) == 0
    assert lib.get_option(lib.LSN_OPT_GEMM_TAIL_SPLIT) == 0
    assert lib.get_option(lib.LSN_OPT_LAYER_MERGE) == 1
    assert lib.get_option(lib.LSN_OPT_DEQUANT_SPARE_SMS) == 0
    for opt, bad in ((lib.LSN_OPT_FUSED_NF4, 3), (lib.LSN_OPT_DEQUANT_SPARE_SMS, -1)):
        with pytest.raises(lib.LsnError) as e:
            lib.set_option(opt, bad)
        assert e.value.status == lib.LSN_ERR_INVALID_ARG
    lib.set_option(lib.LSN_OPT_DEQUANT_SPARE_SMS, 20)
    assert lib.get_option(lib.LSN_OPT_DEQUANT_SPARE_SMS) == 20
    lib.set_option(lib.LSN_OPT_DEQUANT_SPARE_SMS, 0)
    assert lib.get_option(12345) == -1


def test_pool_debug_rejects_a_null_pool(lib):
    with pytest.raises(lib.LsnError) as e:
        lib.layer_pool_set_debug(None, lib.LSN_POOL_DEBUG_POISON)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG


def test_dequant_batch_rejects_bad_arguments(lib):
    w = lib.make_nf4_weight(64, 128, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    with pytest.raises(lib.LsnError) as e:                       # misaligned output
        lib.nf4_dequant_batch([w], [(1 << 20) + 2], stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    bad = lib.make_nf4_weight(64, 100, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    with pytest.raises(lib.LsnError) as e:                       # cols % 64 != 0
        lib.nf4_dequant_batch([w, bad], [1 << 20, 1 << 21], stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG
    lib.nf4_dequant_batch([], [], stream=0)                      # nothing to do


def test_huge_nf4_shapes_are_rejected_without_overflow(lib):
    """rows * cols is never formed before it is known to fit: shapes whose product overflows int64 (or
    exceeds the library's element limit) are argument errors for the codec calls, the allocation-free one
    included, and nothing is launched."""
    for rows, cols in ((1 << 40, 1 << 40), ((1 << 62) // 64, 128), ((1 << 46) // 64 + 1, 64)):
        w = lib.make_nf4_weight(rows, cols, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
        for call in (lambda: lib.nf4_dequant(w, 1 << 20, stream=0),
                     lambda: lib.nf4_quantize(1 << 20, w, 1 << 20, 1 << 40, stream=0),
                     lambda: lib.nf4_quantize_noalloc(1 << 20, w, stream=0)):
            with pytest.raises(lib.LsnError) as e:
                call()
            assert e.value.status == lib.LSN_ERR_INVALID_ARG
            assert "too large" in str(e.value)


def test_noalloc_checks_its_arguments_like_the_workspace_version(lib):
    """nf4_quantize_noalloc applies the same descriptor checks as nf4_quantize (NULL arrays, 16-byte packed,
    4-byte constants) and its element limit, all before any device work."""
    bad = [lib.make_nf4_weight(64, 128, None, 1 << 20, 1 << 20, 1 << 20),          # NULL packed
           lib.make_nf4_weight(64, 128, (1 << 20) + 8, 1 << 20, 1 << 20, 1 << 20),  # packed not 16-byte aligned
           lib.make_nf4_weight(64, 128, 1 << 20, 1 << 20, (1 << 20) + 2, 1 << 20),  # s2 not 4-byte aligned
           lib.make_nf4_weight(64, 128, 1 << 20, 1 << 20, 1 << 20, (1 << 20) + 1),  # offset not 4-byte aligned
           lib.make_nf4_weight(64, 100, 1 << 20, 1 << 20, 1 << 20, 1 << 20)]        # cols % 64 != 0
    for w in bad:
        for call in (lambda: lib.nf4_quantize(1 << 20, w, 1 << 20, 1 << 30, stream=0),
                     lambda: lib.nf4_quantize_noalloc(1 << 20, w, stream=0)):
            with pytest.raises(lib.LsnError) as e:
                call()
            assert e.value.status == lib.LSN_ERR_INVALID_ARG
    over = lib.make_nf4_weight(lib.NF4_NOALLOC_MAX_ELEMS // 4096 + 1, 4096, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    with pytest.raises(lib.LsnError) as e:
        lib.nf4_quantize_noalloc(1 << 20, over, stream=0)
    assert e.value.status == lib.LSN_ERR_INVALID_ARG and "limit" in str(e.value)


def test_merged_gemm_schedule(lib):
    """The merged launch's host-made schedule (no device touched): every tile of every problem goes to
    exactly one worker; each worker's list runs in decreasing cost; the busiest worker's summed cost is
    within one tile of the ideal share (the greedy bound); for the forward GEMMs of projections 1..6 of
    the 8B layer at 2048 tokens on 74 SM pairs it is 688 contraction blocks (ideal 687.7, 886 - 66 = 820
    for separate launches of those six).  Bad arguments are rejected."""
    ntiles = [32, 32, 128, 448, 448, 128]          # k, v, o, gate, up, down: 256 x 256 pair tiles
    cost = [33, 33, 33, 33, 33, 113]               # 128-wide contraction blocks + the LoRA block
    lists = lib.gemm_merged_schedule(74, ntiles, cost)
    flat = sorted(t for lst in lists for t in lst)
    assert flat == list(range(sum(ntiles)))
    first = [0]
    for n in ntiles:
        first.append(first[-1] + n)
    def c(t):
        i = max(j for j in range(len(ntiles)) if first[j] <= t)
        return cost[i]
    loads = [sum(c(t) for t in lst) for lst in lists]
    ideal = sum(n * k for n, k in zip(ntiles, cost)) / 74
    assert max(loads) <= ideal + max(cost)
    assert max(loads) == 688
    for lst in lists:
        costs = [c(t) for t in lst]
        assert costs == sorted(costs, reverse=True)
    # the backward's six (dX of k, v, o, gate, up, down): contraction 1024, 1024, 4096, 14336, 14336, 4096
    b = lib.gemm_merged_schedule(74, [128, 128, 128, 128, 128, 448], [9, 9, 33, 113, 113, 33])
    assert sorted(t for lst in b for t in lst) == list(range(1088))
    for bad in ((0, [1], [1]), (4, [1], [0]), (4, [-1], [3])):
        with pytest.raises(lib.LsnError):
            lib.gemm_merged_schedule(*bad)
