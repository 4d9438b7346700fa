"""Glue between the seeded inputs, the oracle and the CUDA path for tests.

Everything expected comes from ``oracle/``; everything compared comes from the
CUDA library through its C ABI. Inputs come from ``workloads``.
"""

import numpy as np

from oracle import int4, lut3, matmul


def sample_columns(N, count, seed=0):
    """Sorted distinct columns: both ends plus ``count`` seeded random ones."""
    if count >= N:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    cols = set(rng.choice(N, size=count, replace=False).tolist())
    cols.update({0, N - 1})
    return np.array(sorted(cols))


def oracle_int4(W, group, mode):
    q, s, zp = int4.quantize(W, group, mode)
    return dict(q=q, s=s, zp=zp, packed=int4.pack_nibbles(q), deq=int4.dequant(q, s, group, zp))


def check_outputs(Y_gpu, X, deq, cols=None):
    """Compare GPU outputs (torch [M, N]) with the oracle on the given columns.

    ``deq`` is the oracle's dequantised weight restricted to ``cols`` (or all
    columns). Returns the max error ratio (<= 1 passes) and asserts it."""
    Xd = matmul.as_f64(X)
    Y = matmul.as_f64(Y_gpu)
    if cols is not None:
        Y = Y[:, cols]
    Y_ref = matmul.matmul_f64(Xd, deq)
    S = matmul.abs_scale(Xd, deq)
    ok, worst = matmul.check(Y, Y_ref, S)
    assert ok, f"max error ratio {worst:.3g} > 1"
    return worst


def lut3_oracle(idx, cb, ex):
    return lut3.dequant(idx, cb, ex)
