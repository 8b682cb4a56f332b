"""C ABI checks that need no GPU: the library builds for sm_100a, loads, and
exports every entry point declared in include/nvfp4.h; the pure host helpers
(sizes, status strings) return the documented values; argument errors are
reported before anything touches the device."""
import os
import re

import pytest

import nvfp4_w4a4_quantized_05_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:nvfp4_status_t|size_t|uint64_t|int|const char\s*\*)\s+([a-z][a-z0-9_]*)\s*\(",
                                src, re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    L = nv.lib()
    declared = _declared_symbols()
    assert len(declared) >= 23
    assert {"mxfp4_quantize_act", "mxfp4_gemm", "mxfp4_scale_bytes", "w4a16_gemm"} <= set(declared)
    missing = [n for n in declared if not hasattr(L, n)]
    assert not missing, missing
    assert set(declared) <= set(nv.__all__)


def test_status_strings_and_version():
    assert nv.nvfp4_status_string(0) == "ok"
    for s in range(1, 7):
        assert nv.nvfp4_status_string(s) not in ("", "unknown status")
    assert nv.nvfp4_status_string(99) == "unknown status"
    assert re.fullmatch(r"\d+\.\d+\.\d+", nv.nvfp4_version())


@pytest.mark.parametrize("rows,k", [(1, 16), (16, 256), (130, 320), (8192, 4096), (0, 64)])
def test_size_helpers(rows, k):
    assert nv.nvfp4_codes_bytes(rows, k) == rows * k // 2
    pr = (rows + 127) // 128 * 128
    pc = (k // 16 + 3) // 4 * 4
    assert nv.nvfp4_scale_bytes(rows, k) == pr * pc
    if k % 32 == 0:
        assert nv.mxfp4_scale_bytes(rows, k) == pr * ((k // 32 + 3) // 4 * 4)


def test_grouped_scale_bound_covers_any_split():
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(50):
        E = int(rng.integers(1, 40))
        sizes = rng.integers(0, 300, size=E)
        need = int(sum((s + 127) // 128 * 128 for s in sizes)) * (64 // 16)
        assert nv.nvfp4_grouped_scale_bytes(int(sizes.sum()), E, 64) >= need


def test_workspace_sizes():
    assert nv.nvfp4_workspace_bytes(nv.OP_QUANTIZE_ACT) >= 24
    assert nv.nvfp4_workspace_bytes(nv.OP_QUANTIZE_ACT, 0, 0, 0, 128) >= 16 + 4 * 128 + 4 * 129
    assert nv.nvfp4_workspace_bytes(nv.OP_QUANTIZE_WEIGHT_2D) >= 24
    assert nv.nvfp4_workspace_bytes(nv.OP_GEMM) == 0


def test_argument_errors_are_reported_before_launch():
    # null pointers, bad k, bad groups: returned synchronously, no device touched
    assert nv.nvfp4_quantize_act(0, 16, 256, 256, None, 0, 0, 0, 0, 0, 0) == 1
    assert nv.nvfp4_quantize_act(16, 16, 250, 256, None, 0, 16, 16, 16, 16, 0) == 2
    assert nv.nvfp4_quantize_act(16, 16, 256, 256, None, 3, 16, 16, 16, 16, 0) == 1
    assert nv.nvfp4_quantize_weight_2d(16, 17, 256, 256, 16, 16, None, 16, 16, 0) == 2
    assert nv.nvfp4_gemm(16, 16, 16, 16, 16, 16, 16, 64, 16, 64, 96, None, 0) == 2   # k % 64
    assert nv.nvfp4_gemm(0, 16, 16, 16, 16, 16, 16, 64, 16, 64, 128, None, 0) == 1
    assert nv.nvfp4_gemm(8, 16, 16, 16, 16, 16, 16, 64, 16, 64, 128, None, 0) == 3   # misaligned
    assert nv.nvfp4_grouped_gemm(16, 16, 16, 16, 300, 16, 16, 16, 16, 64, 128, 10, None, 0) == 2
    assert nv.nvfp4_probe_cvt(0, 0, 0, 10, 0) == 1
    # MXFP4 and W4A16 entry points
    assert nv.mxfp4_quantize_act(0, 16, 256, 256, 16, 16, 0) == 1            # null input
    assert nv.mxfp4_quantize_act(16, 16, 48, 48, 16, 16, 0) == 2             # k % 32
    assert nv.mxfp4_quantize_act(16, 16, 256, 256, 8, 16, 0) == 3            # misaligned codes
    assert nv.mxfp4_gemm(16, 16, 16, 16, 16, 64, 16, 64, 96, None, 0) == 2   # k % 64
    assert nv.mxfp4_gemm(0, 16, 16, 16, 16, 64, 16, 64, 128, None, 0) == 1
    assert nv.w4a16_gemm(16, 128, 16, 16, 16, 16, 64, 65, 64, 128, 0) == 2   # m above 64
    assert nv.w4a16_gemm(16, 96, 16, 16, 16, 16, 64, 8, 64, 96, 0) == 2     # k % 64
    assert nv.w4a16_gemm(0, 128, 16, 16, 16, 16, 64, 8, 64, 128, 0) == 1    # null activations
    assert nv.w4a16_gemm(8, 128, 16, 16, 16, 16, 64, 8, 64, 128, 0) == 3    # misaligned activations
