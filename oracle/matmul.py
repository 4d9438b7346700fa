"""Y = X . W in FP64, its error scale, and the acceptance test.

Test infrastructure only (see ``oracle/__init__.py``).

The operation is the problem statement of "Low Bit Metal Kernels" (INT4
dequant + matmul listing): Y[M, N] = X[M, K] . W[K, N] with W dequantised just
before use. The listing accumulates in half precision; the oracle accumulates
in FP64 instead, which is the exact result up to FP64 rounding.

Acceptance (the bound every GPU output is held to):
    |y - y_ref| <= 4e-3 * S + ulp16(|y_ref|),  S = sum_k |x_k * w_kn|,
where ulp16(v) is one FP16 unit in the last place of v: 2^(floor(log2 v) - 10)
for v >= 2^-14 and 2^-24 below.
"""

import numpy as np

REL_TOL = 4e-3


def as_f64(a):
    """Exact widening of an FP16/BF16/FP32 array (or torch tensor) to float64."""
    if hasattr(a, "detach"):  # a torch tensor: widen on the CPU, exactly
        import torch
        return a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def matmul_f64(X, W):
    """Y_ref = X . W with FP64 accumulation. X [M, K], W [K, N] -> float64 [M, N]."""
    X = as_f64(X)
    W = as_f64(W)
    if X.ndim != 2 or W.ndim != 2 or X.shape[1] != W.shape[0]:
        raise ValueError("shapes do not chain")
    return X @ W


def abs_scale(X, W):
    """S = |X| . |W| (FP64): the size of the terms each output sums."""
    return np.abs(as_f64(X)) @ np.abs(as_f64(W))


def ulp16(v):
    """One FP16 ulp of |v| (elementwise): 2^(floor(log2|v|) - 10), 2^-24 below 2^-14."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    out = np.full(a.shape, 2.0 ** -24)
    big = a >= 2.0 ** -14
    out[big] = np.exp2(np.floor(np.log2(a[big])) - 10)
    return out


def error_ratio(Y, Y_ref, S):
    """|y - y_ref| / (4e-3 * S + ulp16(y_ref)) elementwise; <= 1 means accepted."""
    Y = as_f64(Y)
    bound = REL_TOL * np.asarray(S, dtype=np.float64) + ulp16(Y_ref)
    err = np.abs(Y - Y_ref)
    err = np.where(np.isnan(Y), np.inf, err)
    return err / bound


def check(Y, Y_ref, S):
    """(ok, max_ratio): ok when every element meets the acceptance bound."""
    r = error_ratio(Y, Y_ref, S)
    m = float(np.max(r)) if r.size else 0.0
    return m <= 1.0, m
