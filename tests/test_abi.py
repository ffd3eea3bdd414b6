"""The C ABI without a GPU: the library loads, exports every symbol that
include/moe_fp8.h declares, and rejects bad arguments on the host before any
CUDA call. No kernel is launched here."""
import ctypes
import os
import re

import pytest

from fine_grained_fp8_sigmoid_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_fp8.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:MOE_API\s+)?(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_declares_the_boundary_calls():
    names = set(_declared())
    for n in ["moe_route", "moe_quant_1x128", "moe_permute", "moe_grouped_gemm_fp8",
              "moe_combine", "moe_bias_update"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert _lib.status_string(0) == "MOE_OK"
    assert _lib.status_string(4) == "MOE_ERR_TIMEOUT"
    assert lib.moe_version() == 200


def test_workspace_sizes(lib):
    assert lib.moe_kgrouped_gemm_fp8_workspace() >= 4
    assert lib.moe_grouped_scaled_gemm_fp8_workspace() >= 4
    assert lib.moe_permute_workspace(8192, 256) == 2 * 32 * 256 * 4
    assert lib.moe_permute_workspace(0, 256) == 0
    rows = 8192 * 8 + 8192
    ws = lib.moe_grouped_gemm_fp8_workspace(8192, 8, 7168, 2048)
    a256 = lambda n: (n + 255) // 256 * 256
    # H codes, H scales, two int32 tile counters, each part 256-byte aligned
    assert ws == a256(a256(rows * 2048) + rows * 16 * 4) + 2 * 4


def test_gemm_launch_count_query(lib):
    # one persistent launch per phase, wide and narrow tiles alike
    assert lib.moe_grouped_gemm_fp8_launches(7168, 2048) == 2
    assert lib.moe_grouped_gemm_fp8_launches(7424, 2048) == 2
    assert lib.moe_grouped_gemm_fp8_launches(0, 2048) == -1


def test_host_side_argument_checks(lib):
    N = None
    s = ctypes.c_void_p(0)
    # cols not a multiple of 128 / negative sizes: rejected before any CUDA call
    assert lib.moe_quant_1x128(N, 4, 100, N, N, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_quant_1x128(N, -1, 128, N, N, s) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_quant_128x128(N, 100, 128, N, N, s) == _lib.MOE_ERR_UNSUPPORTED
    # K_r > N_r, K_r > 16, N_r > 256
    assert lib.moe_route(N, N, N, N, 4, 64, 4, 5, N, N, N, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_route(N, N, N, N, 4, 64, 64, 17, N, N, N, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_route(N, N, N, N, 4, 64, 512, 8, N, N, N, s) == _lib.MOE_ERR_UNSUPPORTED
    # permute: N_r > 1024, missing outputs
    assert lib.moe_permute(N, 4, 2, 2000, N, N, 0, N, N, N, N, N, N, N, 0, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_permute(N, 4, 2, 8, N, N, 0, N, N, N, N, N, N, N, 0, s) == _lib.MOE_ERR_INVALID_ARG
    # GEMM: d not a multiple of 256, I not a multiple of 128
    assert lib.moe_grouped_gemm_fp8(N, N, N, 8, 2, N, N, 4, N, N, N, N, N, N, 384, 128,
                                    N, N, N, 0, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_grouped_gemm_fp8(N, N, N, 8, 2, N, N, 4, N, N, N, N, N, N, 256, 100,
                                    N, N, N, 0, s) == _lib.MOE_ERR_UNSUPPORTED
    # fused router + quantisation: d not a multiple of 128
    assert lib.moe_route_quant(N, N, N, 4, 192, 8, 2, N, N, N, N, N, s) == _lib.MOE_ERR_UNSUPPORTED
    # K-grouped GEMM: M not a multiple of 128, N not a multiple of 256, G = 0
    assert lib.moe_kgrouped_gemm_fp8(N, N, N, N, N, 4, 100, 256, 128, N, N, 0, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_kgrouped_gemm_fp8(N, N, N, N, N, 4, 128, 384, 128, N, N, 0, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_kgrouped_gemm_fp8(N, N, N, N, N, 0, 128, 256, 128, N, N, 0, s) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_kgrouped_gemm_fp8(N, N, N, N, N, 4, 128, 256, 128, N, N, 0, s) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(N, N, N, N, N, 4, 2, 12, N, s) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_bias_update(N, N, 8, 4, 2, ctypes.c_float(0.001), N, s) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_wait_timeout(0, s) == _lib.MOE_ERR_INVALID_ARG
    st = ctypes.c_int()
    assert lib.moe_get_error(None) == _lib.MOE_ERR_INVALID_ARG


def test_empty_inputs_are_no_ops(lib):
    s = ctypes.c_void_p(0)
    assert lib.moe_quant_1x128(None, 0, 256, None, None, s) == 0
    assert lib.moe_route(None, None, None, None, 0, 64, 8, 2, None, None, None, s) == 0
    assert lib.moe_combine(None, None, None, None, None, 0, 2, 256, None, s) == 0
