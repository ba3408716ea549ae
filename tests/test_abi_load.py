"""The C-ABI library loads without a GPU and exports every symbol include/stq1.h declares."""

import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "stq1.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(stq1_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    import sub_bit_sparse_b200 as m
    lib = ctypes.CDLL(m.LIB_PATH)
    names = _declared_functions()
    assert len(names) >= 8
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(m.SIGNATURES)
    assert m.LIB.stq1_version() >= 100


def test_error_codes_are_distinct_and_negative():
    src = open(os.path.join(ROOT, "include", "stq1.h")).read()
    codes = dict(re.findall(r"#define (STQ1_ERR_\w+) \((-\d+)\)", src))
    vals = [int(v) for v in codes.values()]
    assert len(vals) == len(set(vals)) and all(v < 0 for v in vals)
    import sub_bit_sparse_b200 as m
    assert {int(v): k for k, v in codes.items()} == m.ERRORS


def test_host_side_argument_checks_need_no_gpu():
    # Shape checks run before anything touches the device.
    import sub_bit_sparse_b200 as m
    L = m.LIB
    assert L.stq1_gemv(None, None, None, 16, 256, 1, None, 0, None) == -2
    assert L.stq1_gemv(1 << 20, 1 << 20, 1 << 20, 16, 300, 1, None, 0, None) == -1
    assert L.stq1_gemv(1 << 20, 1 << 20, 1 << 20, 16, 256, 0, None, 0, None) == -1
    assert L.stq1_gemv((1 << 20) + 8, 1 << 20, 1 << 20, 16, 256, 1, None, 0, None) == -6
    assert L.stq1_dequant(None, None, 1, 256, None) == -2
    assert L.stq1_dequant(1 << 20, 1 << 20, 1, 255, None) == -1
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 4, 8, 4, 64, 256, 0, None, 0, None) == -1
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 4, 2, 4, 63, 256, 0, None, 0, None) == -1
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 4, 2, 4, 64, 256, 1, None, 0, None) == -2
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 4, 2, 4, 64, 256, 8, None, 0, None) == -8
    # the fp8 variant is a supported flag: without a workspace it is the workspace error
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 4, 2, 4, 64, 256, 2, None, 0, None) == -7
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 4, 2, 4, 64, 256, 0, None, 0, None) == -7
    assert L.stq1_gemv_workspace(16, 300, 1) == 0
    assert L.stq1_moe_workspace(16, 8, 256, 4096, 7168, 0) > 0
    # prefill-sized calls: the fp8 variant stages E4M3 rows (1 byte per element
    # instead of 2) plus the per-token copy and the scales
    bf, f8 = L.stq1_moe_workspace(4096, 8, 256, 4096, 7168, 0), L.stq1_moe_workspace(4096, 8, 256, 4096, 7168, 2)
    assert f8 == bf - 32768 * 7168 + 4096 * 7168 + 4096 * 4 + 32768 * 4
    # empty inputs are shape errors, never launches
    assert L.stq1_gemv(1 << 20, 1 << 20, 1 << 20, 0, 256, 1, None, 0, None) == -1
    assert L.stq1_moe_gateup(1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 0, 2, 4, 64, 256, 0, None, 0, None) == -1
    assert L.stq1_swiglu(1 << 20, 1 << 20, 0, 64, None) == -1
    assert L.stq1_swiglu(1 << 20, 1 << 20, 4, 63, None) == -1
    assert L.stq1_moe_combine(1 << 20, None, 1 << 20, 0, 8, 64, None) == -1
    assert L.stq1_moe_ffn(1 << 20, 1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 0, 8, 4, 512, 256, 0, None, 0,
                          None) == -1
    assert L.stq1_quantize(1 << 20, None, 0, 256, 0, 3, 1 << 20, None) == -1
    assert L.stq1_quantize(None, None, 4, 256, 0, 3, 1 << 20, None) == -2
    assert L.stq1_quantize(1 << 20, None, 4, 300, 0, 3, 1 << 20, None) == -1
    assert L.stq1_quantize(1 << 20, None, 4, 256, 7, 3, 1 << 20, None) == -8
    assert L.stq1_quantize(1 << 20, None, 4, 256, 1, -1, 1 << 20, None) == -8
    assert L.stq1_quantize((1 << 20) + 4, None, 4, 256, 0, 3, 1 << 20, None) == -6
    assert L.stq1_quantize(1 << 20, None, 4, 256, 0, 3, (1 << 20) + 1, None) == -6
    assert L.stq1_quantize(1 << 20, (1 << 20) + 4, 4, 256, 1, 3, 1 << 20, None) == -6   # h read as float4
    assert L.stq1_quantize_x_e4m3(None, 4, 256, 1 << 20, 1 << 20, None) == -2
    assert L.stq1_quantize_x_e4m3(1 << 20, 4, 250, 1 << 20, 1 << 20, None) == -1
    assert L.stq1_quantize_x_e4m3(1 << 20, 0, 256, 1 << 20, 1 << 20, None) == -1
    assert L.stq1_quantize_x_e4m3((1 << 20) + 2, 4, 256, 1 << 20, 1 << 20, None) == -6
    assert L.stq1_selftest_wait(2, None) == -8
    assert L.stq1_gemv_prefetch(1 << 20, 1 << 20, 1 << 20, 16, 256, 1, None, 0, 1 << 20, -16, None) == -1
    assert L.stq1_gemv_prefetch(1 << 20, 1 << 20, 1 << 20, 16, 256, 1, None, 0, (1 << 20) + 8, 64, None) == -6
    assert L.stq1_gemv_prefetch(1 << 20, 1 << 20, 1 << 20, 16, 300, 1, None, 0, None, 0, None) == -1
    # mixed-precision allocation entries
    assert L.stq1_quantize_stq2(None, None, 4, 256, 0, 1 << 20, None) == -2
    assert L.stq1_quantize_stq2(1 << 20, None, 0, 256, 0, 1 << 20, None) == -1
    assert L.stq1_quantize_stq2(1 << 20, None, 4, 300, 0, 1 << 20, None) == -1
    assert L.stq1_quantize_stq2(1 << 20, None, 4, 256, -1, 1 << 20, None) == -8
    assert L.stq1_quantize_stq2((1 << 20) + 4, None, 4, 256, 0, 1 << 20, None) == -6
    assert L.stq1_quantize_stq2(1 << 20, (1 << 20) + 2, 4, 256, 3, 1 << 20, None) == -6
    assert L.stq1_quantize_stq2(1 << 20, (1 << 20) + 4, 4, 256, 3, 1 << 20, None) == -6   # h read as float4
    assert L.stq1_hessian_diag(None, 1, 4, 256, 1 << 20, None) == -2
    assert L.stq1_hessian_diag(1 << 20, 0, 4, 256, 1 << 20, None) == -1
    assert L.stq1_hessian_diag(1 << 20, 1, 0, 256, 1 << 20, None) == -1
    assert L.stq1_hessian_diag(1 << 20, 70000, 4, 256, 1 << 20, None) == -1
    P = 1 << 20
    assert L.stq1_hessian_error(0, None, P, P, P, 1, 4, 256, 4, P, None) == -2
    assert L.stq1_hessian_error(2, P, P, P, P, 1, 4, 256, 4, P, None) == -8
    assert L.stq1_hessian_error(0, P, P, P, P, 1, 4, 300, 4, P, None) == -1
    assert L.stq1_hessian_error(0, P, P, P, P, 0, 4, 256, 4, P, None) == -1
    assert L.stq1_hessian_error(0, P, P, P, P, 1, 0, 256, 4, P, None) == -1
    assert L.stq1_hessian_error(0, P, P, P, P, 1, 4, 256, 0, P, None) == -1
    assert L.stq1_hessian_error(1, P + 1, P, P, P, 1, 4, 256, 4, P, None) == -6
    assert L.stq1_hessian_error(1, P, P, P + 8, P, 1, 4, 256, 4, P, None) == -6
    assert L.stq1_hessian_error(1, P, P, P, P, 1, 4, 256, 4, P + 4, None) == -6


def test_debug_build_exports_the_same_symbols():
    from sub_bit_sparse_b200 import build as b
    path = b.build(debug=True)                         # no-op when up to date; nvcc only, no GPU
    lib = ctypes.CDLL(path)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    lib.stq1_build_flags.restype = ctypes.c_int
    assert lib.stq1_build_flags() == 1
    import sub_bit_sparse_b200 as m
    if not m.DEBUG_BUILD:
        assert m.LIB.stq1_build_flags() == 0
