"""CPU oracle for the quantized W8A8 linear layer -- TEST INFRASTRUCTURE.

Only ``tests/``, the package's ``smoke()`` check and ``bench.py``'s CPU
baseline leg may import this module. The product library never does, and it
shares no code with the CUDA path.

This is a thin ctypes wrapper around ``oracle.c`` (plain C, compiled with
``-O2 -ffp-contract=off``, OpenMP over output rows). Inputs are numpy arrays
or CPU torch tensors; fp16/bf16 tensors cross as their raw 16-bit patterns.
The C file states, function by function, which passage of the model-card
pages each definition follows.

Parity status of every function is pinned by ``tests/test_oracle_*.py``
against facts that do not come from the oracle itself (format definitions,
torch's own float8/bf16 casts, closed forms, brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F16, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2 -ffp-contract=off -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
               "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, f32, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_int
        sig = {
            "orc_f16_to_double": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_bf16_to_double": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_double_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
            "orc_double_to_f16": (ctypes.c_uint16, [ctypes.c_double]),
            "orc_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e4m3_encode": (ctypes.c_uint8, [f32]),
            "orc_e4m3_encode_search": (ctypes.c_uint8, [f32]),
            "orc_e4m3_encode_bits": (ctypes.c_uint8, [f32]),
            "orc_e4m3_compare_encoders": (ctypes.c_int64, [ctypes.c_uint64, ctypes.c_uint64]),
            "orc_e4m3_encode_range": (None, [ctypes.c_uint64, ctypes.c_uint64, P]),
            "orc_q_int8": (i32, [f32, f32]),
            "orc_q_int4": (i32, [f32, f32]),
            "orc_q_e4m3": (ctypes.c_uint8, [f32, f32]),
            "orc_int8_scale": (f32, [f32]),
            "orc_e4m3_scale": (f32, [f32]),
            "orc_recip": (f32, [f32]),
            "orc_absmax_scale": (f32, [P, i32, i64, f32]),
            "orc_quantize_weight_int8": (None, [P, i32, i64, i64, P, P]),
            "orc_quantize_weight_fp8_tensor": (None, [P, i32, i64, i64, P, P]),
            "orc_quantize_weight_fp8_channel": (None, [P, i32, i64, i64, P, P]),
            "orc_quantize_weight_int4": (None, [P, i32, i64, i64, i64, P, P]),
            "orc_int4_unpack": (i32, [P, i64, i64, i64]),
            "orc_int8_outlier_prep": (None, [P, i32, i64, i64, f32, P, P, P, P, P, P, i64]),
            "orc_outlier_weights": (None, [P, P, i64, i64, P, ctypes.c_int32, i32, P, i64]),
            "orc_int8_outlier_forward": (i32, [P, i32, i64, i64, P, P, i64, f32, P, P, i64,
                                               P, P, P]),
            "orc_fp8_static_prep": (None, [P, i32, i64, i64, f32, P]),
            "orc_fp8_dynamic_prep": (None, [P, i32, i64, i64, P, P]),
            "orc_fp8_forward": (None, [P, i32, i64, i64, P, f32, P, i64, f32, P, P, i64,
                                       P, P, P, P, P]),
            "orc_w4a8_forward": (None, [P, i32, i64, i64, P, P, i64, i64, P, P, i64,
                                        P, P, P, P, P]),
            "orc_quantize_weight_int8_block": (None, [P, i32, i64, i64, i64, P, P]),
            "orc_int8_block_forward": (None, [P, i32, i64, i64, P, P, i64, i64, P, P, i64,
                                              P, P, P, P, P]),
            "orc_fp_linear_forward": (None, [P, i32, i64, i64, P, i64, P, P, i64, P, P]),
            "orc_fp8_weight_only_dequant": (None, [P, P, i64, i64, P]),
            "orc_fp8_weight_only_forward": (None, [P, i32, i64, i64, P, P, i64, P, P, i64, P, P]),
            "orc_e2m1_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e2m1_encode": (ctypes.c_uint8, [f32]),
            "orc_quantize_weight_nvfp4": (None, [P, i32, i64, i64, P, P, P]),
            "orc_nvfp4_code": (ctypes.c_uint8, [P, i64, i64, i64]),
            "orc_nvfp4_weight_only_forward": (None, [P, i32, i64, i64, P, P, f32, i64, P, P, i64, P, P]),
            "orc_nvfp4_forward": (None, [P, i32, i64, i64, P, P, f32, i64, P, P, i64, P, P, P, P, P]),
            "orc_num_threads": (i32, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ---------------------------------------------------------------------------
# marshalling helpers (no arithmetic of the method here)
# ---------------------------------------------------------------------------

def _bits16(x) -> tuple:
    """(uint16 numpy array, dtype code) for an fp16/bf16 torch tensor or uint16 array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            dt = {torch.float16: F16, torch.bfloat16: BF16}[x.dtype]
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)), dt
    except ImportError:  # pragma: no cover
        pass
    raise TypeError("expected an fp16/bf16 torch tensor")


def _np(x, dtype) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows: Optional[Sequence[int]]):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size


def bits_to_torch(bits: np.ndarray, dt: int):
    import torch
    t = torch.from_numpy(bits.view(np.int16).copy())
    return t.view(torch.bfloat16 if dt == BF16 else torch.float16)


# ---------------------------------------------------------------------------
# scalar codecs
# ---------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(t: float) -> int:
    return lib().orc_e4m3_encode(float(t))


def e4m3_encode_search(t: float) -> int:
    return lib().orc_e4m3_encode_search(float(t))


def e4m3_encode_bits(t: float) -> int:
    """Third encoder, integer arithmetic on the fp32 bit fields (pins e4m3_encode)."""
    return lib().orc_e4m3_encode_bits(float(t))


def e4m3_compare_encoders(lo: int, count: int) -> int:
    """Mismatches of e4m3_encode vs e4m3_encode_bits over fp32 bit patterns [lo, lo+count)."""
    return int(lib().orc_e4m3_compare_encoders(int(lo), int(count)))


def e4m3_encode_range(lo: int, count: int) -> np.ndarray:
    """e4m3_encode of the floats with bit patterns lo .. lo+count-1."""
    out = np.empty((count,), np.uint8)
    lib().orc_e4m3_encode_range(int(lo), int(count), _p(out))
    return out


def q_int8(v: float, inv: float) -> int:
    return lib().orc_q_int8(float(v), float(inv))


def q_e4m3(v: float, inv: float) -> int:
    return lib().orc_q_e4m3(float(v), float(inv))


def int8_scale(absmax: float) -> float:
    return lib().orc_int8_scale(float(absmax))


def e4m3_scale(absmax: float) -> float:
    return lib().orc_e4m3_scale(float(absmax))


def num_threads() -> int:
    return lib().orc_num_threads()


# ---------------------------------------------------------------------------
# weight quantisation / calibration
# ---------------------------------------------------------------------------

def absmax_scale(X, qmax: float) -> float:
    xb, dt = _bits16(X)
    return lib().orc_absmax_scale(_p(xb), dt, xb.size, float(qmax))


def quantize_weight(W, mode: str, group: int = 128):
    """Offline weight quantisation. mode: int8_row | fp8_tensor | fp8_channel | int4_g128 | int8_block.

    Returns (Wq, w_scale) as numpy arrays: int8 [N,K] + fp32 [N]; uint8 e4m3
    [N,K] + fp32 [1]; uint8 e4m3 [N,K] + uint16 bf16 bits [N]; uint8 packed
    [N,K/2] + fp32 [N,K/group]; int8 [N,K] + fp32 [N,K/group] (block scales).
    """
    wb, dt = _bits16(W)
    N, K = W.shape
    L = lib()
    if mode == "int8_row":
        q = np.zeros((N, K), np.int8)
        s = np.zeros((N,), np.float32)
        L.orc_quantize_weight_int8(_p(wb), dt, N, K, _p(q), _p(s))
    elif mode == "fp8_tensor":
        q = np.zeros((N, K), np.uint8)
        s = np.zeros((1,), np.float32)
        L.orc_quantize_weight_fp8_tensor(_p(wb), dt, N, K, _p(q), _p(s))
    elif mode == "fp8_channel":
        q = np.zeros((N, K), np.uint8)
        s = np.zeros((N,), np.uint16)
        L.orc_quantize_weight_fp8_channel(_p(wb), dt, N, K, _p(q), _p(s))
    elif mode == "int8_block":
        assert K % group == 0
        q = np.zeros((N, K), np.int8)
        s = np.zeros((N, K // group), np.float32)
        L.orc_quantize_weight_int8_block(_p(wb), dt, N, K, group, _p(q), _p(s))
    elif mode == "int4_g128":
        assert K % group == 0
        q = np.zeros((N, K // 2), np.uint8)
        s = np.zeros((N, K // group), np.float32)
        L.orc_quantize_weight_int4(_p(wb), dt, N, K, group, _p(q), _p(s))
    else:
        raise ValueError(mode)
    return q, s


# ---------------------------------------------------------------------------
# LLM.int8
# ---------------------------------------------------------------------------

def int8_outlier_prep(X, threshold: float = 6.0):
    """dict(Xq int8 [M,K], s_x f32 [M], is_outlier u8 [K], O i32 [count], X_O u16 bits [M,count])."""
    xb, dt = _bits16(X)
    M, K = X.shape
    Xq = np.zeros((M, K), np.int8)
    s_x = np.zeros((M,), np.float32)
    flag = np.zeros((K,), np.uint8)
    O = np.zeros((max(K, 1),), np.int32)
    cnt = np.zeros((1,), np.int32)
    ostr = max(K, 1)
    X_O = np.zeros((M, ostr), np.uint16)
    lib().orc_int8_outlier_prep(_p(xb), dt, M, K, float(threshold), _p(Xq), _p(s_x), _p(flag),
                                _p(O), _p(cnt), _p(X_O), ostr)
    n = int(cnt[0])
    return dict(Xq=Xq, s_x=s_x, is_outlier=flag, O=O[:n].copy(), count=n,
                X_O=X_O[:, :n].copy(), dt=dt)


def outlier_weights(Wq: np.ndarray, s_w: np.ndarray, O: np.ndarray, dt: int) -> np.ndarray:
    """W_O bits [N, count] = dtype(fp32(Wq[:,O]) * s_w)."""
    Wq = _np(Wq, np.int8)
    s_w = _np(s_w, np.float32)
    O = _np(O, np.int32)
    N, K = Wq.shape
    n = O.size
    W_O = np.zeros((N, max(n, 1)), np.uint16)
    lib().orc_outlier_weights(_p(Wq), _p(s_w), N, K, _p(O), n, dt, _p(W_O), max(n, 1))
    return W_O[:, :n].copy()


def int8_outlier_forward(X, Wq, s_w, threshold: float = 6.0, bias=None,
                         rows: Optional[Sequence[int]] = None, want_c: bool = True):
    """dict(C int32 [R,N], Y64 f64 [R,N], Y u16 bits [R,N]) for rows R (all if None)."""
    xb, dt = _bits16(X)
    M, K = X.shape
    Wq = _np(Wq, np.int8)
    s_w = _np(s_w, np.float32)
    N = Wq.shape[0]
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    C = np.zeros((R, N), np.int32) if want_c else None
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    rc = lib().orc_int8_outlier_forward(_p(xb), dt, M, K, _p(Wq), _p(s_w), N, float(threshold),
                                        _p(bb), _p(r), nr, _p(C), _p(Y64), _p(Y))
    if rc != 0:
        raise OverflowError("int32 accumulator overflow")
    return dict(C=C, Y64=Y64, Y=Y, dt=dt)


# ---------------------------------------------------------------------------
# FP8
# ---------------------------------------------------------------------------

def fp8_static_prep(X, input_scale: float) -> np.ndarray:
    xb, dt = _bits16(X)
    M, K = X.shape
    Xq = np.zeros((M, K), np.uint8)
    lib().orc_fp8_static_prep(_p(xb), dt, M, K, float(input_scale), _p(Xq))
    return Xq


def fp8_dynamic_prep(X):
    xb, dt = _bits16(X)
    M, K = X.shape
    Xq = np.zeros((M, K), np.uint8)
    s_x = np.zeros((M,), np.float32)
    lib().orc_fp8_dynamic_prep(_p(xb), dt, M, K, _p(Xq), _p(s_x))
    return Xq, s_x


def fp8_forward(X, Wq, w_scale, x_scale: Optional[float] = None, bias=None,
                rows: Optional[Sequence[int]] = None):
    """FP8 linear. w_scale: fp32 scalar (per tensor) or uint16 bf16 bits [N] (per channel).
    x_scale: fp32 static input scale, or None for dynamic per-token scales."""
    xb, dt = _bits16(X)
    M, K = X.shape
    Wq = _np(Wq, np.uint8)
    N = Wq.shape[0]
    w_scale = np.asarray(w_scale)
    if w_scale.dtype == np.uint16:
        wsb, wst = np.ascontiguousarray(w_scale.reshape(-1)), 0.0
    else:
        wsb, wst = None, float(w_scale.reshape(-1)[0])
    xs = -1.0 if x_scale is None else float(x_scale)
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Xq = np.zeros((M, K), np.uint8)
    s_x = np.zeros((M,), np.float32)
    acc = np.zeros((R, N), np.float64)
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_fp8_forward(_p(xb), dt, M, K, _p(Wq), wst, _p(wsb), N, xs, _p(bb), _p(r), nr,
                          _p(Xq), _p(s_x), _p(acc), _p(Y64), _p(Y))
    return dict(Xq=Xq, s_x=s_x, acc=acc, Y64=Y64, Y=Y, dt=dt)


def fp8_weight_only_dequant(Wq, s_w_bits) -> np.ndarray:
    """bf16 bits [N,K] of W_deq = bf16(decode(Wq) * s_w) (weight.to(bf16) * weight_scale)."""
    Wq = _np(Wq, np.uint8)
    N, K = Wq.shape
    sw = np.ascontiguousarray(np.asarray(s_w_bits, dtype=np.uint16).reshape(-1))
    out = np.zeros((N, K), np.uint16)
    lib().orc_fp8_weight_only_dequant(_p(Wq), _p(sw), N, K, _p(out))
    return out


def fp8_weight_only_forward(X, Wq, s_w_bits, bias=None, rows: Optional[Sequence[int]] = None):
    """Weight-only FP8 linear: Y = X W_deq^T + bias, activations unquantised.
    s_w_bits: uint16 bf16 bits [N] (the [out,1] scale)."""
    xb, dt = _bits16(X)
    M, K = X.shape
    Wq = _np(Wq, np.uint8)
    N = Wq.shape[0]
    sw = np.ascontiguousarray(np.asarray(s_w_bits, dtype=np.uint16).reshape(-1))
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_fp8_weight_only_forward(_p(xb), dt, M, K, _p(Wq), _p(sw), N, _p(bb), _p(r), nr, _p(Y64), _p(Y))
    return dict(Y64=Y64, Y=Y, dt=dt)


# ---------------------------------------------------------------------------
# NVFP4 weights (E2M1 codes, E4M3 per-16 scales, fp32 tensor scale)
# ---------------------------------------------------------------------------

def e2m1_decode(c: int) -> float:
    return float(lib().orc_e2m1_decode(int(c)))


def e2m1_encode(t: float) -> int:
    return int(lib().orc_e2m1_encode(float(t)))


def quantize_weight_nvfp4(W):
    """(codes uint8 [N,K/2] packed in blocks of 32, block scales uint8 e4m3 [N,K/16], tensor scale float)."""
    wb, dt = _bits16(W)
    N, K = W.shape
    assert K % 32 == 0
    q = np.zeros((N, K // 2), np.uint8)
    sb = np.zeros((N, K // 16), np.uint8)
    st = np.zeros((1,), np.float32)
    lib().orc_quantize_weight_nvfp4(_p(wb), dt, N, K, _p(q), _p(sb), _p(st))
    return q, sb, float(st[0])


def nvfp4_code(Wq, K: int, j: int, k: int) -> int:
    Wq = _np(Wq, np.uint8)
    return int(lib().orc_nvfp4_code(_p(Wq), K, j, k))


def nvfp4_weight_only_forward(X, Wq, s_b, s_t: float, bias=None, rows: Optional[Sequence[int]] = None):
    """NVFP4 weight-only linear: Y = s_t * X (code * s_b)^T + bias, activations unquantised."""
    xb, dt = _bits16(X)
    M, K = X.shape
    Wq = _np(Wq, np.uint8)
    sb = _np(s_b, np.uint8)
    N = Wq.shape[0]
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_nvfp4_weight_only_forward(_p(xb), dt, M, K, _p(Wq), _p(sb), float(s_t), N, _p(bb), _p(r), nr,
                                        _p(Y64), _p(Y))
    return dict(Y64=Y64, Y=Y, dt=dt)


def nvfp4_forward(X, Wq, s_bw, s_tw: float, bias=None, rows: Optional[Sequence[int]] = None):
    """NVFP4 activations and weights (W4A4): X quantised per call like a weight,
    Y = s_tx * s_tw * (cx * sbx)(cw * sbw)^T + bias. Returns Y64, Y, Xq, s_bx, s_tx."""
    xb, dt = _bits16(X)
    M, K = X.shape
    assert K % 32 == 0
    Wq = _np(Wq, np.uint8)
    sbw = _np(s_bw, np.uint8)
    N = Wq.shape[0]
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Xq = np.zeros((M, K // 2), np.uint8)
    sbx = np.zeros((M, K // 16), np.uint8)
    stx = np.zeros((1,), np.float32)
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_nvfp4_forward(_p(xb), dt, M, K, _p(Wq), _p(sbw), float(s_tw), N, _p(bb), _p(r), nr, _p(Xq), _p(sbx),
                            _p(stx), _p(Y64), _p(Y))
    return dict(Y64=Y64, Y=Y, Xq=Xq, s_bx=sbx, s_tx=float(stx[0]), dt=dt)


# ---------------------------------------------------------------------------
# W4A8
# ---------------------------------------------------------------------------

def w4a8_forward(X, Wq4, s_w, group: int = 128, bias=None, rows: Optional[Sequence[int]] = None,
                 want_cg: bool = False):
    xb, dt = _bits16(X)
    M, K = X.shape
    Wq4 = _np(Wq4, np.uint8)
    s_w = _np(s_w, np.float32)
    N = Wq4.shape[0]
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Xq = np.zeros((M, K), np.int8)
    s_x = np.zeros((M,), np.float32)
    Cg = np.zeros((R, N, K // group), np.int32) if want_cg else None
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_w4a8_forward(_p(xb), dt, M, K, _p(Wq4), _p(s_w), N, group, _p(bb), _p(r), nr,
                           _p(Xq), _p(s_x), _p(Cg), _p(Y64), _p(Y))
    return dict(Xq=Xq, s_x=s_x, Cg=Cg, Y64=Y64, Y=Y, dt=dt)


# ---------------------------------------------------------------------------
# Block-scaled int8 weights (one scale per 32 weights of a row)
# ---------------------------------------------------------------------------

def int8_block_forward(X, Wq, s_w, block: int = 32, bias=None, rows: Optional[Sequence[int]] = None,
                       want_cb: bool = False):
    """Y = s_x[i] * sum_b s_w[j,b] * C_b[i,j] + bias, per-token int8 activations,
    int8 weights with fp32 scales [N, K/block]."""
    xb, dt = _bits16(X)
    M, K = X.shape
    Wq = _np(Wq, np.int8)
    s_w = _np(s_w, np.float32)
    N = Wq.shape[0]
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Xq = np.zeros((M, K), np.int8)
    s_x = np.zeros((M,), np.float32)
    Cb = np.zeros((R, N, K // block), np.int32) if want_cb else None
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_int8_block_forward(_p(xb), dt, M, K, _p(Wq), _p(s_w), N, block, _p(bb), _p(r), nr,
                                 _p(Xq), _p(s_x), _p(Cb), _p(Y64), _p(Y))
    return dict(Xq=Xq, s_x=s_x, Cb=Cb, Y64=Y64, Y=Y, dt=dt)


# ---------------------------------------------------------------------------
# Unquantised 16-bit linear (layers kept in fp16)
# ---------------------------------------------------------------------------

def fp_linear_forward(X, W, bias=None, rows: Optional[Sequence[int]] = None):
    """Y = X W^T + bias with X, W (and bias) in one 16-bit dtype; Y64 exact in
    fp64, Y rounded once to that dtype."""
    xb, dt = _bits16(X)
    wb, wdt = _bits16(W)
    assert wdt == dt, "X and W must share a dtype"
    M, K = X.shape
    N = W.shape[0]
    bb = None if bias is None else _bits16(bias)[0]
    r, nr = _rows(rows)
    R = M if r is None else nr
    Y64 = np.zeros((R, N), np.float64)
    Y = np.zeros((R, N), np.uint16)
    lib().orc_fp_linear_forward(_p(xb), dt, M, K, _p(wb), N, _p(bb), _p(r), nr, _p(Y64), _p(Y))
    return dict(Y64=Y64, Y=Y, dt=dt)
