"""MXFP8 activation quantisation on the GPU against the oracle: codes and
scales bit for bit (the format has exactly one correct encoding under the
block-scale and rounding reading the oracle states)."""

import numpy as np
import pytest

import workloads
from oracle import mxfp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    return torch


@pytest.fixture(scope="module")
def lbq():
    import bit_weight_only_pack_b200 as lbq
    return lbq


def _planted(torch, X):
    """Blocks the scale rule and the rounding have to get right."""
    X[0, 0:32] = 0.0                                    # all-zero block: scale 127
    X[0, 32:64] = -0.0
    X[0, 64] = 1.0                                      # amax exactly a power of two
    X[0, 96] = 0.75                                     # scale 2^-9, element 384
    X[0, 128:160] = 3.0e-3 * torch.arange(32, dtype=torch.float32).to(X.dtype)
    X[0, 160:192] = 0.0
    X[0, 160] = -1.0e-30 if X.dtype == torch.bfloat16 else -6e-8   # a block whose amax is tiny and negative
    X[0, 192] = 1.0
    X[0, 193] = 1.0 / 256 * 1.03125                      # small elements next to a large one
    X[0, 194] = -(1.0 / 256) * 1.0625
    if X.dtype == torch.bfloat16 and X.shape[1] >= 320:
        # scale byte clamped to 0: amax 2^-125 asks for 2^(-125 - 8), below 2^-127
        X[0, 224:256] = 0.0
        X[0, 224] = 2.0 ** -125
        X[0, 225] = -(2.0 ** -127) * 1.5
        X[0, 226] = 2.0 ** -131                          # a BF16 subnormal in the same block
        # the block's largest element is itself a BF16 subnormal
        X[0, 288:320] = 0.0
        X[0, 288] = -(2.0 ** -130) * 1.5
        X[0, 289] = 2.0 ** -133
    return X


@pytest.mark.parametrize("xdt", ["bf16", "f16"])
@pytest.mark.parametrize("M,K", [(1, 4096), (3, 96), (17, 1024)])
def test_quantize_mxfp8_bit_exact(torch, lbq, xdt, M, K):
    X = workloads.activations_host(40 + M + K, M, K, xdt)
    if xdt == "bf16":
        X = X * (torch.arange(M, dtype=torch.float32)[:, None] * 7 - 9).exp2().to(X.dtype)  # rows 2^-9 .. 2^103
    else:
        # FP16 rows 2^-14 .. 2^4 (the small rows are largely FP16 subnormals)
        X = (X.float() * (torch.arange(M, dtype=torch.float32)[:, None] % 4 * 6 - 14).exp2()).to(X.dtype)
    if K >= 256:
        X = _planted(torch, X.clone())
    codes, scales = lbq.quantize_mxfp8(X.cuda())
    torch.cuda.synchronize()
    rc, rs = mxfp8.quantize(X.to(torch.float64).numpy())
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)
    lbq.device_status()


def test_quantize_mxfp8_rejects_bad_shapes(torch, lbq):
    X = torch.zeros((2, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lbq.LbqError):
        lbq.quantize_mxfp8(X)
