"""Python binding of libqlin.so -- a B200 (sm_100a) quantized W8A8 linear layer.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libqlin.so, called through its C ABI (include/qlin.h) with
ctypes. PyTorch supplies device memory and the current CUDA stream. There is
no CPU fallback: if the library is missing, importing it raises.

Functions keep the C names:

    Wq, s_w = qlin_quantize_weight(W, QLIN_W_INT8_ROW)
    Y = qlin_int8_outlier_forward(X, Wq, s_w, threshold=6.0)
    Wq8, s8 = qlin_quantize_weight(W, QLIN_W_FP8_TENSOR)
    xs = qlin_calibrate_input_scale(X_calibration)
    Y = qlin_fp8_forward(X, Wq8, s8, QLIN_W_FP8_TENSOR, x_scale=xs)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlin.so")

QLIN_OK, QLIN_ERR_INVALID_ARG, QLIN_ERR_UNSUPPORTED, QLIN_ERR_ALIGNMENT = 0, 1, 2, 3
QLIN_ERR_WORKSPACE, QLIN_ERR_CUDA, QLIN_ERR_TIMEOUT = 4, 5, 6
QLIN_F16, QLIN_BF16 = 0, 1
QLIN_W_INT8_ROW, QLIN_W_FP8_TENSOR, QLIN_W_FP8_CHANNEL, QLIN_W_INT4_G128, QLIN_W_INT8_BLOCK32 = 0, 1, 2, 3, 4
QLIN_W_NVFP4 = 5
QLIN_OP_INT8_OUTLIER, QLIN_OP_FP8, QLIN_OP_W4A8, QLIN_OP_QUANTIZE_WEIGHT, QLIN_OP_INT8_PREP = 0, 1, 2, 3, 4
QLIN_OP_INT8_BLOCK, QLIN_OP_FP8_GEMM = 5, 6

_STATUS_NAMES = {0: "QLIN_OK", 1: "QLIN_ERR_INVALID_ARG", 2: "QLIN_ERR_UNSUPPORTED", 3: "QLIN_ERR_ALIGNMENT",
                 4: "QLIN_ERR_WORKSPACE", 5: "QLIN_ERR_CUDA", 6: "QLIN_ERR_TIMEOUT"}


class QlinError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python quantized_w8a8_linear_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    st = ctypes.c_int
    sigs = {
        "qlin_workspace_bytes": (sz, [i32, i64, i64, i64]),
        "qlin_quantize_weight": (st, [P, i32, i64, i64, i32, P, P, P, sz, P]),
        "qlin_calibrate_input_scale": (st, [P, i32, i64, i64, P, P, sz, P]),
        "qlin_int8_outlier_forward": (st, [P, i32, i64, i64, P, P, i64, f32, P, P, P, sz, P]),
        "qlin_fp8_forward": (st, [P, i32, i64, i64, P, P, i32, i64, P, P, P, P, sz, P]),
        "qlin_int8_outlier_prepare": (st, [P, i32, i64, i64, P, P, i64, f32, P, sz, P]),
        "qlin_int8_outlier_forward_noalloc": (st, [P, i32, i64, i64, P, P, i64, f32, P, P, P]),
        "qlin_int8_outlier_gemm": (st, [i32, i64, i64, P, P, i64, P, P, P, sz, P]),
        "qlin_int8_outlier_gemm_i32": (st, [i64, i64, P, i64, P, P, sz, P]),
        "qlin_fp8_gemm": (st, [i32, i64, i64, P, P, P, P, i32, i64, P, P, P, P, sz, P]),
        "qlin_w4a8_forward": (st, [P, i32, i64, i64, P, P, i64, P, P, P, sz, P]),
        "qlin_fp_linear_forward": (st, [P, i32, i64, i64, P, i64, P, P, P]),
        "qlin_fp8_weight_only_forward": (st, [P, i32, i64, i64, P, P, i64, P, P, P]),
        "qlin_nvfp4_weight_only_forward": (st, [P, i32, i64, i64, P, P, i64, P, P, P]),
        "qlin_int8_block_forward": (st, [P, i32, i64, i64, P, P, i64, P, P, P, sz, P]),
        "qlin_int8_block_prep": (st, [P, i32, i64, i64, P, P, P]),
        "qlin_w4a8_gemm": (st, [i32, i64, i64, P, P, P, P, i64, P, P, P]),
        "qlin_w4a8_prep": (st, [P, i32, i64, i64, P, P, P]),
        "qlin_w4a8_group_i32": (st, [P, P, i64, i64, i64, i32, P, P]),
        "qlin_int8_prep": (st, [P, i32, i64, i64, f32, P, P, P, P, P, P, i64, P, sz, P]),
        "qlin_outlier_weights": (st, [P, P, i64, i64, P, P, i32, P, i64, P]),
        "qlin_int8_gemm_i32": (st, [P, P, i64, i64, i64, P, P]),
        "qlin_fp8_prep": (st, [P, i32, i64, i64, P, P, P, P]),
        "qlin_e4m3_encode_f32": (st, [P, P, i64, P]),
        "qlin_get_device_status": (st, [P, i32]),
        "qlin_set_wait_timeout_ns": (st, [ctypes.c_uint64]),
        "qlin_set_gemm_schedule": (st, [ctypes.c_int]),
        "qlin_debug_inject_wait_timeout": (st, [ctypes.c_int]),
        "qlin_last_error_string": (ctypes.c_char_p, []),
        "qlin_version": (i32, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def exported_symbols():
    """Names declared in include/qlin.h that this library must export."""
    import re
    hdr = os.path.join(os.path.dirname(_HERE), "include", "qlin.h")
    with open(hdr) as f:
        text = f.read()
    return sorted(set(re.findall(r"^QLIN_API\s+[\w\s\*]+?\b(qlin_\w+)\s*\(", text, flags=re.M)))


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _check(status: int):
    if status != QLIN_OK:
        raise QlinError(status, lib.qlin_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libqlin takes CUDA tensors (device pointers)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return QLIN_BF16
    if t.dtype == torch.float16:
        return QLIN_F16
    raise TypeError(f"activations must be fp16 or bf16, got {t.dtype}")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


_ws_cache = {}


def workspace(op: int, M: int, N: int, K: int, device) -> torch.Tensor:
    """A (cached) device workspace of qlin_workspace_bytes(op, M, N, K) bytes."""
    n = int(lib.qlin_workspace_bytes(op, M, N, K))
    dev = torch.device(device)
    key = (dev.index, op)
    t = _ws_cache.get(key)
    if t is None or t.numel() < n:
        t = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
        _ws_cache[key] = t
    return t


def qlin_workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return int(lib.qlin_workspace_bytes(op, M, N, K))


# ---------------------------------------------------------------------------
# public API
# ---------------------------------------------------------------------------

def qlin_quantize_weight(W: torch.Tensor, mode: int):
    """Offline weight quantisation. Returns (Wq, w_scale) on W's device."""
    N, K = W.shape
    dev = W.device
    if mode == QLIN_W_INT8_ROW:
        Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        s = torch.empty((N,), dtype=torch.float32, device=dev)
    elif mode == QLIN_W_FP8_TENSOR:
        Wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
        s = torch.empty((1,), dtype=torch.float32, device=dev)
    elif mode == QLIN_W_FP8_CHANNEL:
        Wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
        s = torch.empty((N, 1), dtype=torch.bfloat16, device=dev)
    elif mode == QLIN_W_INT4_G128:
        Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((N, K // 128), dtype=torch.float32, device=dev)
    elif mode == QLIN_W_INT8_BLOCK32:
        Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        s = torch.empty((N, K // 32), dtype=torch.float32, device=dev)
    elif mode == QLIN_W_NVFP4:
        Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((nvfp4_scale_offset(N, K) + 4,), dtype=torch.uint8, device=dev)
    else:
        raise ValueError(mode)
    ws = workspace(QLIN_OP_QUANTIZE_WEIGHT, 0, N, K, dev)
    _check(lib.qlin_quantize_weight(_ptr(W), _dt(W), N, K, mode, _ptr(Wq), _ptr(s), _ptr(ws), ws.numel(),
                                    _stream(dev)))
    return Wq, s


def nvfp4_scale_offset(N: int, K: int) -> int:
    """Byte offset of the fp32 tensor scale in a QLIN_W_NVFP4 w_scale buffer
    (after the E4M3 block scales [N, K/16], rounded up to 16 bytes)."""
    return (N * K // 16 + 15) // 16 * 16


def nvfp4_scales(w_scale: torch.Tensor, N: int, K: int):
    """(E4M3 block scales uint8 [N, K/16], fp32 tensor scale [1]) views of a QLIN_W_NVFP4 w_scale buffer."""
    off = nvfp4_scale_offset(N, K)
    return w_scale[: N * K // 16].view(N, K // 16), w_scale[off:off + 4].view(torch.float32)


def qlin_calibrate_input_scale(X: torch.Tensor) -> torch.Tensor:
    """Static FP8 input scale by max calibration: absmax(X) / 448 (device fp32 [1])."""
    M, K = X.shape
    out = torch.empty((1,), dtype=torch.float32, device=X.device)
    ws = workspace(QLIN_OP_QUANTIZE_WEIGHT, M, 0, K, X.device)
    _check(lib.qlin_calibrate_input_scale(_ptr(X), _dt(X), M, K, _ptr(out), _ptr(ws), ws.numel(),
                                          _stream(X.device)))
    return out


def qlin_int8_outlier_forward(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, threshold: float = 6.0,
                              bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                              ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """LLM.int8 linear: Y[M,N] = int8(X \\ O) Wq^T (dequantised) + X[:,O] W_O^T + bias."""
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    if ws is None:
        ws = workspace(QLIN_OP_INT8_OUTLIER, M, N, K, X.device)
    _check(lib.qlin_int8_outlier_forward(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), N, float(threshold),
                                         _ptr(bias), _ptr(Y), _ptr(ws), ws.numel(), _stream(X.device)))
    return Y


def qlin_int8_outlier_forward_noalloc(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                                      threshold: float = 6.0, bias: Optional[torch.Tensor] = None,
                                      Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """LLM.int8 linear with the library's built-in scratch (no workspace argument)."""
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    _check(lib.qlin_int8_outlier_forward_noalloc(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), N,
                                                 float(threshold), _ptr(bias), _ptr(Y), _stream(X.device)))
    return Y


def qlin_int8_outlier_prepare(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, threshold: float,
                              ws: torch.Tensor) -> None:
    """Stage 1 of the LLM.int8 forward: outlier set, codes, scales, X_O, W_O into `ws`."""
    M, K = X.shape
    N = Wq.shape[0]
    _check(lib.qlin_int8_outlier_prepare(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), N, float(threshold),
                                         _ptr(ws), ws.numel(), _stream(X.device)))


def qlin_int8_outlier_gemm(dtype: torch.dtype, M: int, K: int, Wq: torch.Tensor, w_scale: torch.Tensor,
                           Y: torch.Tensor, ws: torch.Tensor, bias: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Stage 2 of the LLM.int8 forward: tcgen05 GEMM + fused epilogue, reading `ws`."""
    N = Wq.shape[0]
    dt = QLIN_BF16 if dtype == torch.bfloat16 else QLIN_F16
    _check(lib.qlin_int8_outlier_gemm(dt, M, K, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), _ptr(Y), _ptr(ws),
                                      ws.numel(), _stream(Wq.device)))
    return Y


def qlin_int8_outlier_gemm_i32(M: int, K: int, Wq: torch.Tensor, ws: torch.Tensor) -> torch.Tensor:
    """int32 accumulator of the LLM.int8 GEMM without the outlier columns, from
    the workspace a prepare call filled (parity export of the same kernel)."""
    N = Wq.shape[0]
    C = torch.empty((M, N), dtype=torch.int32, device=Wq.device)
    _check(lib.qlin_int8_outlier_gemm_i32(M, K, _ptr(Wq), N, _ptr(C), _ptr(ws), ws.numel(), _stream(Wq.device)))
    return C


def qlin_fp8_gemm(Xq: torch.Tensor, s_x: Optional[torch.Tensor], Wq: torch.Tensor, w_scale: torch.Tensor,
                  wmode: int, dtype: torch.dtype, x_scale: Optional[torch.Tensor] = None,
                  bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """GEMM stage of the FP8 forward on codes from qlin_fp8_prep. ws: optional
    scratch of workspace(QLIN_OP_FP8_GEMM, ...) bytes (lets the GEMM split
    tiles along K across CTAs); None: whole tiles only."""
    M, K = Xq.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=dtype, device=Xq.device)
    dt = QLIN_BF16 if dtype == torch.bfloat16 else QLIN_F16
    _check(lib.qlin_fp8_gemm(dt, M, K, _ptr(Xq), _ptr(s_x), _ptr(Wq), _ptr(w_scale), wmode, N, _ptr(x_scale),
                             _ptr(bias), _ptr(Y), _ptr(ws), 0 if ws is None else ws.numel(), _stream(Xq.device)))
    return Y


def qlin_fp8_forward(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor, wmode: int,
                     x_scale: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                     Y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """FP8 E4M3 W8A8 linear (static per-tensor or dynamic per-token / per-channel scales)."""
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    if ws is None:
        ws = workspace(QLIN_OP_FP8, M, N, K, X.device)
    _check(lib.qlin_fp8_forward(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), wmode, N, _ptr(x_scale),
                                _ptr(bias), _ptr(Y), _ptr(ws), ws.numel(), _stream(X.device)))
    return Y


def qlin_w4a8_forward(X: torch.Tensor, Wq4: torch.Tensor, w_scale: torch.Tensor,
                      bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """W4A8 linear: int4 per-group-128 weights, per-token int8 activations."""
    M, K = X.shape
    N = Wq4.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    if ws is None:
        ws = workspace(QLIN_OP_W4A8, M, N, K, X.device)
    _check(lib.qlin_w4a8_forward(_ptr(X), _dt(X), M, K, _ptr(Wq4), _ptr(w_scale), N, _ptr(bias), _ptr(Y),
                                 _ptr(ws), ws.numel(), _stream(X.device)))
    return Y


def qlin_fp_linear_forward(X: torch.Tensor, W: torch.Tensor, bias: Optional[torch.Tensor] = None,
                           Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Unquantised 16-bit linear Y = X W^T + bias (X, W, bias in one dtype), tcgen05 kind::f16."""
    M, K = X.shape
    N = W.shape[0]
    if W.dtype != X.dtype or (bias is not None and bias.dtype != X.dtype):
        raise TypeError("X, W and bias must share one 16-bit dtype")
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    _check(lib.qlin_fp_linear_forward(_ptr(X), _dt(X), M, K, _ptr(W), N, _ptr(bias), _ptr(Y), _stream(X.device)))
    return Y


def qlin_fp8_weight_only_forward(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                                 bias: Optional[torch.Tensor] = None,
                                 Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Weight-only FP8 linear: Y = X (bf16(decode(Wq) * w_scale))^T + bias, bf16 activations."""
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    _check(lib.qlin_fp8_weight_only_forward(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), _ptr(Y),
                                            _stream(X.device)))
    return Y


def qlin_nvfp4_weight_only_forward(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                                   bias: Optional[torch.Tensor] = None,
                                   Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """NVFP4 weight-only linear: Y = s_t * X (e2m1(code) * e4m3(s_b))^T + bias, bf16 activations."""
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    _check(lib.qlin_nvfp4_weight_only_forward(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), N, _ptr(bias),
                                              _ptr(Y), _stream(X.device)))
    return Y


def qlin_int8_block_forward(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                            bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                            ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block-scaled int8 linear: one fp32 weight scale per 32 weights of a row, per-token int8 activations."""
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    if ws is None:
        ws = workspace(QLIN_OP_INT8_BLOCK, M, N, K, X.device)
    _check(lib.qlin_int8_block_forward(_ptr(X), _dt(X), M, K, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), _ptr(Y),
                                       _ptr(ws), ws.numel(), _stream(X.device)))
    return Y


def qlin_int8_block_prep(X: torch.Tensor):
    """Activation stage of the block-scaled int8 forward: int8 codes as fp16 values [M,K] and s_x [M]."""
    M, K = X.shape
    Xq16 = torch.empty((M, K), dtype=torch.float16, device=X.device)
    s_x = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(lib.qlin_int8_block_prep(_ptr(X), _dt(X), M, K, _ptr(Xq16), _ptr(s_x), _stream(X.device)))
    return Xq16, s_x


def qlin_w4a8_prep(X: torch.Tensor, Xq: Optional[torch.Tensor] = None, s_x: Optional[torch.Tensor] = None):
    """Activation stage of the W4A8 forward: per-token int8 codes and fp32 scales."""
    M, K = X.shape
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if s_x is None:
        s_x = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(lib.qlin_w4a8_prep(_ptr(X), _dt(X), M, K, _ptr(Xq), _ptr(s_x), _stream(X.device)))
    return Xq, s_x


def qlin_w4a8_gemm(Xq: torch.Tensor, s_x: torch.Tensor, Wq4: torch.Tensor, w_scale: torch.Tensor,
                   dtype: torch.dtype, bias: Optional[torch.Tensor] = None,
                   Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """GEMM stage of the W4A8 forward on int8 codes and per-token scales."""
    M, K = Xq.shape
    N = Wq4.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=dtype, device=Xq.device)
    dt = QLIN_BF16 if dtype == torch.bfloat16 else QLIN_F16
    _check(lib.qlin_w4a8_gemm(dt, M, K, _ptr(Xq), _ptr(s_x), _ptr(Wq4), _ptr(w_scale), N, _ptr(bias), _ptr(Y),
                              _stream(Xq.device)))
    return Y


def qlin_w4a8_group_i32(Xq: torch.Tensor, Wq4: torch.Tensor, group: int) -> torch.Tensor:
    """int32 partials C_g [M,N] of one group, as the W4A8 GEMM computes them (parity export)."""
    M, K = Xq.shape
    N = Wq4.shape[0]
    C = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _check(lib.qlin_w4a8_group_i32(_ptr(Xq), _ptr(Wq4), M, N, K, int(group), _ptr(C), _stream(Xq.device)))
    return C


def qlin_int8_prep(X: torch.Tensor, threshold: float = 6.0):
    """LLM.int8 activation prep alone (parity export). Returns a dict of device tensors."""
    M, K = X.shape
    dev = X.device
    ostride = (K + 7) // 8 * 8
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    s_x = torch.empty((M,), dtype=torch.float32, device=dev)
    flags = torch.empty(((K + 31) // 32,), dtype=torch.int32, device=dev)
    O = torch.empty((K,), dtype=torch.int32, device=dev)
    count = torch.empty((1,), dtype=torch.int32, device=dev)
    X_O = torch.zeros((M, ostride), dtype=X.dtype, device=dev)
    ws = workspace(QLIN_OP_INT8_PREP, M, 0, K, dev)
    _check(lib.qlin_int8_prep(_ptr(X), _dt(X), M, K, float(threshold), _ptr(Xq), _ptr(s_x), _ptr(flags), _ptr(O),
                              _ptr(count), _ptr(X_O), ostride, _ptr(ws), ws.numel(), _stream(dev)))
    return dict(Xq=Xq, s_x=s_x, flags=flags, O=O, count=count, X_O=X_O, ostride=ostride)


def qlin_outlier_weights(Wq: torch.Tensor, w_scale: torch.Tensor, O: torch.Tensor, count: torch.Tensor,
                         dtype: torch.dtype) -> torch.Tensor:
    """W_O [N, round_up(K,8)] = dtype(fp32(Wq[:,O]) * w_scale) (parity export)."""
    N, K = Wq.shape
    ostride = (K + 7) // 8 * 8
    W_O = torch.zeros((N, ostride), dtype=dtype, device=Wq.device)
    dt = QLIN_BF16 if dtype == torch.bfloat16 else QLIN_F16
    _check(lib.qlin_outlier_weights(_ptr(Wq), _ptr(w_scale), N, K, _ptr(O), _ptr(count), dt, _ptr(W_O), ostride,
                                    _stream(Wq.device)))
    return W_O


def qlin_int8_gemm_i32(Xq: torch.Tensor, Wq: torch.Tensor) -> torch.Tensor:
    """Raw tcgen05 int8 GEMM: C[M,N] int32 = Xq Wq^T (parity export)."""
    M, K = Xq.shape
    N = Wq.shape[0]
    C = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _check(lib.qlin_int8_gemm_i32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(C), _stream(Xq.device)))
    return C


def qlin_fp8_prep(X: torch.Tensor, x_scale: Optional[torch.Tensor] = None):
    """FP8 activation codes (uint8 e4m3 [M,K]) and, in dynamic mode, per-token scales."""
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    s_x = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(lib.qlin_fp8_prep(_ptr(X), _dt(X), M, K, _ptr(x_scale), _ptr(Xq), _ptr(s_x), _stream(X.device)))
    return Xq, s_x


def qlin_e4m3_encode_f32(t: torch.Tensor, codes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """E4M3 codes of fp32 values with the device conversion the FP8 kernels use (parity export)."""
    t = t.reshape(-1)
    if codes is None:
        codes = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
    _check(lib.qlin_e4m3_encode_f32(_ptr(t), _ptr(codes), t.numel(), _stream(t.device)))
    return codes


def qlin_get_device_status(reset: bool = False) -> int:
    v = ctypes.c_int32(0)
    _check(lib.qlin_get_device_status(ctypes.byref(v), 1 if reset else 0))
    return int(v.value)


def qlin_set_wait_timeout_ns(ns: int) -> None:
    _check(lib.qlin_set_wait_timeout_ns(int(ns)))


def qlin_debug_inject_wait_timeout(on: bool) -> None:
    """Test switch: later GEMM launches wait once on a barrier nothing arrives on (bounded)."""
    _check(lib.qlin_debug_inject_wait_timeout(1 if on else 0))


def qlin_set_gemm_schedule(mode: int) -> None:
    """0 automatic, 1 whole tiles only, 2 stream-K wherever possible (int8 GEMMs)."""
    _check(lib.qlin_set_gemm_schedule(int(mode)))


__all__ = [n for n in dir() if n.startswith(("qlin_", "QLIN_"))] + ["QlinError", "workspace", "lib"]
