"""The C-ABI library loads and exports every entry point include/qlin.h
declares; host-side argument validation rejects bad calls before anything
touches a device (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "qlin_build", os.path.join(ROOT, "quantized_w8a8_linear_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import quantized_w8a8_linear_b200 as q
    return q


def test_header_declares_the_named_entry_points(q):
    names = q.exported_symbols()
    for required in ("qlin_quantize_weight", "qlin_int8_outlier_forward", "qlin_fp8_forward",
                     "qlin_workspace_bytes", "qlin_int8_prep", "qlin_int8_gemm_i32", "qlin_fp8_prep",
                     "qlin_get_device_status", "qlin_last_error_string"):
        assert required in names


def test_library_exports_every_declared_symbol(q):
    lib = ctypes.CDLL(q.LIB_PATH)
    missing = [n for n in q.exported_symbols() if not hasattr(lib, n)]
    assert missing == []
    assert lib.qlin_version() == 100


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "qlin.h"\nint main(void){return qlin_version()==100?0:1;}\n')
    import subprocess
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                           "-I", os.path.join(ROOT, "include"), str(src)])


def test_workspace_sizes(q):
    M, N, K = 4352, 12288, 3072
    ws = q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, M, N, K)
    # Xq + X_O + W_O at worst case (every column an outlier) + small arrays
    assert ws >= M * K + 2 * M * K + 2 * N * K
    assert q.qlin_workspace_bytes(q.QLIN_OP_FP8, M, N, K) >= M * K + 4 * M
    assert q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, -1, N, K) == 0
    assert q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, M, N, 0) == 0


def test_workspace_holds_stream_k_slots(q):
    # two 128 x 256 int32 partial slots per stream-K CTA (at most 160 CTAs,
    # at most one per k-block iteration) on top of the other arrays
    M, N, K = 4352, 12288, 3072
    ws = q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, M, N, K)
    assert ws >= M * K + 2 * M * K + 2 * N * K + 2 * 160 * 128 * 256 * 4
    M, N, K = 64, 256, 256   # 1 tile x 2 k-blocks: 2 CTAs at most
    small = q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, M, N, K)
    base = M * K + 2 * M * K + 2 * N * K
    assert base + 2 * 2 * 128 * 256 * 4 <= small < base + 2 * 2 * 128 * 256 * 4 + (1 << 16)


def test_fp8_workspace_holds_its_gemm_scratch(q):
    # FP8 forward: e4m3 codes + s_x + the GEMM scratch; the scratch: arrival
    # counters for the 128 x 256 tiles' 4 column groups + two fp32 128 x 256
    # partial slots per stream-K CTA (at most 160, at most one per k-block)
    M, N, K = 512, 12288, 4096
    scratch = q.qlin_workspace_bytes(q.QLIN_OP_FP8_GEMM, M, N, K)
    tiles = (M // 128) * (N // 256)
    assert 2 * 160 * 128 * 256 * 4 + 4 * 4 * tiles <= scratch < 2 * 160 * 128 * 256 * 4 + 4 * 4 * tiles + 512
    assert q.qlin_workspace_bytes(q.QLIN_OP_FP8, M, N, K) >= M * K + 4 * M + scratch
    M, N, K = 128, 256, 256   # one tile of 2 k-blocks: 2 stream-K CTAs at most
    assert q.qlin_workspace_bytes(q.QLIN_OP_FP8_GEMM, M, N, K) >= 2 * 2 * 128 * 256 * 4


def test_nvfp4_scale_buffer_layout(q):
    # E4M3 block scales [N, K/16], then the fp32 tensor scale at a 16-byte boundary
    for N, K in [(8, 64), (257, 128), (12288, 4096)]:
        off = q.nvfp4_scale_offset(N, K)
        assert off >= N * K // 16 and off % 16 == 0 and off - N * K // 16 < 16


def test_nvfp4_rejects_k_not_multiple_of_64(q):
    st = q.lib.qlin_nvfp4_weight_only_forward(ctypes.c_void_p(4096), q.QLIN_BF16, 8, 96, ctypes.c_void_p(4096),
                                              ctypes.c_void_p(4096), 8, None, ctypes.c_void_p(4096), None)
    assert st == q.QLIN_ERR_ALIGNMENT
    st = q.lib.qlin_nvfp4_weight_only_forward(ctypes.c_void_p(4096), q.QLIN_F16, 8, 128, ctypes.c_void_p(4096),
                                              ctypes.c_void_p(4096), 8, None, ctypes.c_void_p(4096), None)
    assert st == q.QLIN_ERR_UNSUPPORTED   # bf16 activations only


def test_gemm_schedule_modes(q):
    for mode in (0, 1, 2):
        assert q.lib.qlin_set_gemm_schedule(mode) == q.QLIN_OK
    assert q.lib.qlin_set_gemm_schedule(3) == q.QLIN_ERR_INVALID_ARG
    assert b"schedule" in q.lib.qlin_last_error_string()
    assert q.lib.qlin_set_gemm_schedule(0) == q.QLIN_OK


@pytest.mark.parametrize("K,dt,expect", [(15, 1, 3), (0, 1, 3), (32784, 1, 2), (64, 7, 1)])
def test_host_validation_rejects_before_launch(q, K, dt, expect):
    # X pointer is a fake aligned address: validation fails before any use
    st = q.lib.qlin_int8_outlier_forward(ctypes.c_void_p(4096), dt, 8, K, ctypes.c_void_p(4096),
                                         ctypes.c_void_p(4096), 8, 6.0, None, ctypes.c_void_p(4096),
                                         ctypes.c_void_p(4096), 1 << 30, None)
    assert st == expect
    assert len(q.lib.qlin_last_error_string()) > 0


def test_misaligned_pointer_rejected(q):
    st = q.lib.qlin_int8_outlier_forward(ctypes.c_void_p(4100), 1, 8, 64, ctypes.c_void_p(4096),
                                         ctypes.c_void_p(4096), 8, 6.0, None, ctypes.c_void_p(4096),
                                         ctypes.c_void_p(4096), 1 << 30, None)
    assert st == q.QLIN_ERR_ALIGNMENT
    assert b"aligned" in q.lib.qlin_last_error_string()


def test_binding_has_no_cpu_path(q):
    import torch
    x = torch.zeros((4, 16), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        q.qlin_int8_outlier_forward(x, torch.zeros((4, 16), dtype=torch.int8), torch.ones(4))
