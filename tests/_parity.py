"""Shared helpers of the GPU parity tests (comparison only, no method arithmetic).

Floating-point outputs are checked two ways, per output row:

1. the bar of the method's statement: the GPU's bf16/fp16 output and the
   oracle's output rounded to the same dtype agree within a normwise relative
   error of 2e-3 (||y_gpu - y_oracle|| / ||y_oracle|| <= 2e-3);
2. a rounding-level bound against the oracle's fp64 value before rounding:
   ||y_gpu - y64|| <= ||round(y64) - y64|| + EXTRA * ||y64||, i.e. the GPU is
   as close to the exact result as correct rounding is, up to the fp32
   arithmetic of the kernels (EXTRA = 5e-4 for the integer path, whose only
   fp32 steps are the dequant and the outlier sum).

The direct bound ||y_gpu - y64|| / ||y64|| <= 2e-3 cannot hold for bf16:
rounding the exact value alone costs up to 2^-8 per element (1.6e-3 normwise
on average, above 2e-3 on some rows).
"""
import numpy as np
import torch

import oracle

ROW_REL_TOL = 2e-3
EXTRA_INT8 = 5e-4


def as_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _rows_err(a: np.ndarray, ref: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(a - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def assert_rows_close(y_gpu: torch.Tensor, ref: dict, rows=None, tol=ROW_REL_TOL, extra=EXTRA_INT8, what=""):
    """ref: an oracle result dict with Y (16-bit bits), Y64 (fp64) and dt."""
    yg = y_gpu.detach().cpu()
    if rows is not None:
        yg = yg[rows]
    yg = yg.double().numpy()
    assert np.all(np.isfinite(yg)), f"{what}: non-finite output"
    y_or = oracle.bits_to_torch(np.ascontiguousarray(ref["Y"]), ref["dt"]).double().numpy()
    y64 = ref["Y64"]
    e1 = _rows_err(yg, y_or)
    worst = int(np.argmax(e1))
    assert e1.max() <= tol, f"{what}: max row rel err vs oracle output {e1.max():.3e} at row {worst} (tol {tol})"
    d_gpu = np.linalg.norm(yg - y64, axis=1)
    d_rnd = np.linalg.norm(y_or - y64, axis=1)
    bound = d_rnd + extra * np.linalg.norm(y64, axis=1) + 1e-30
    bad = np.nonzero(d_gpu > bound)[0]
    assert bad.size == 0, (f"{what}: rows farther from the exact value than rounding explains: {bad[:5]} "
                           f"({d_gpu[bad[0]]:.3e} > {bound[bad[0]]:.3e})")
    return e1


def sample_rows(M, n=24, seed=0, must=()):
    rng = np.random.default_rng(seed)
    base = set(int(r) for r in must if r < M)
    base |= {0, M - 1, min(M - 1, 127), min(M - 1, 128)}
    extra = rng.choice(M, size=min(M, n), replace=False)
    return sorted(base | set(int(r) for r in extra))
