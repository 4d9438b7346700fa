"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds input generators and workload shapes only: no quantisation,
packing or matmul arithmetic. Both the oracle-side tests and the CUDA-side
tests/bench draw their inputs from here.

The shapes stand in for Llama-3-8B-class projection layers (decode at batch
1..16, prefill of 512..8192 tokens); no trained weights or datasets are used.

Two backends produce the same *distributions* from the same seed:
* ``"numpy"``: ``numpy.random.default_rng(seed)`` on the host (tests, oracle);
* ``"torch"``: a seeded ``torch.Generator`` on a device (large bench inputs,
  generated in place on the GPU). The two backends do not produce the same
  numbers; anything compared against the oracle uses the values actually fed
  to the GPU.
"""

import numpy as np

# (name, K, N) of the seven per-layer projections of a Llama-3-8B-shaped layer.
LLAMA3_8B_PROJ = (
    ("q", 4096, 4096),
    ("k", 4096, 1024),
    ("v", 4096, 1024),
    ("o", 4096, 4096),
    ("gate", 4096, 14336),
    ("up", 4096, 14336),
    ("down", 14336, 4096),
)
LLAMA3_8B_LAYERS = 32

CONFIGS = {
    "c1": dict(desc="single W4A16 GEMV", M=(1,), K=4096, N=4096, mode="sym", group=32,
               x_dtype="f16", y_dtype="f16", seed=0),
    "c2": dict(desc="Llama-3-8B-shaped decode step, 7 projections x 32 layers", M=(1,),
               mode="asym", group=32, x_dtype="f16", y_dtype="f16", seed=1000),
    "c3": dict(desc="decode batch sweep", M=(1, 2, 4, 8, 16), K=8192, N=28672, mode="sym",
               group=(64, 128), x_dtype="bf16", y_dtype="bf16", seed=3, outlier_frac=1e-3,
               outlier_mult=20.0),
    "c4": dict(desc="prefill GEMM", M=(512, 2048, 8192), K=4096, N=14336, mode="asym", group=128,
               x_dtype="bf16", y_dtype="bf16", seed=4),
    "c5": dict(desc="3-bit LUT weights", M=(1, 2048), K=4096, N=14336, mode="lut3",
               x_dtype="bf16", y_dtype="bf16", seed=5),
}

W_STD = 0.02
X_SEED_OFFSET = 500000


def c2_seed(layer, proj):
    """Seed of projection ``proj`` (0..6) of layer ``layer`` (0..31) in the decode step."""
    return CONFIGS["c2"]["seed"] + 7 * layer + proj


# ----------------------------------------------------------------------------- host (numpy)

def weights_host(seed, K, N, std=W_STD, outlier_frac=0.0, outlier_mult=1.0):
    """W float32 [K, N] ~ N(0, std); optionally exactly round(frac*K*N) entries,
    chosen uniformly without replacement, multiplied by ``outlier_mult``."""
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((K, N), dtype=np.float32) * np.float32(std)
    if outlier_frac > 0:
        count = int(round(outlier_frac * K * N))
        pos = rng.choice(K * N, size=count, replace=False)
        W.reshape(-1)[pos] *= np.float32(outlier_mult)
    return W


def activations_host(seed, M, K, dtype):
    """X [M, K] ~ N(0, 1) rounded to ``dtype`` ('f16' or 'bf16'); returned as a
    torch CPU tensor of that dtype (numpy has no bf16)."""
    import torch
    rng = np.random.default_rng(seed + X_SEED_OFFSET)
    x = torch.from_numpy(rng.standard_normal((M, K), dtype=np.float32))
    return x.to(torch.float16 if dtype == "f16" else torch.bfloat16)


def lut3_host(seed, K, N):
    """(idx uint8 [K, N] uniform 0..7, codebooks uint8 [K/64, N/8, 8] = E4M3 of
    N(0,1) samples, exponents uint8 [K/64, N/8] = 127 + U{-10..-4})."""
    import torch
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, 8, size=(K, N), dtype=np.uint8)
    cb32 = torch.from_numpy(rng.standard_normal((K // 64, N // 8, 8), dtype=np.float32))
    cb = cb32.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ex = (127 + rng.integers(-10, -3, size=(K // 64, N // 8))).astype(np.uint8)
    return idx, cb, ex


def mx_activations_host(seed, M, K, scale_lo=118, scale_hi=134):
    """MXFP8 activations drawn directly in the format: E4M3 codes uint8 [M, K]
    uniform over the non-NaN bytes, UE8M0 scale bytes uint8 [M, K/32] uniform
    over scale_lo..scale_hi."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(M, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] -= 1
    scales = rng.integers(scale_lo, scale_hi + 1, size=(M, K // 32), dtype=np.uint8)
    return codes, scales


# ----------------------------------------------------------------------------- device (torch)

def _gen(seed, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights_device(seed, K, N, device, std=W_STD, outlier_frac=0.0, outlier_mult=1.0):
    """Same distribution as :func:`weights_host`, generated on ``device``."""
    import torch
    g = _gen(seed, device)
    W = torch.randn((K, N), generator=g, device=device, dtype=torch.float32).mul_(std)
    if outlier_frac > 0:
        count = int(round(outlier_frac * K * N))
        pos = torch.randperm(K * N, generator=g, device=device)[:count]
        W.view(-1)[pos] *= outlier_mult
    return W


def activations_device(seed, M, K, dtype, device):
    import torch
    g = _gen(seed + X_SEED_OFFSET, device)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    return x.to(torch.float16 if dtype == "f16" else torch.bfloat16)


def lut3_device(seed, K, N, device):
    import torch
    g = _gen(seed, device)
    idx = torch.randint(0, 8, (K, N), generator=g, device=device, dtype=torch.uint8)
    cb = torch.randn((K // 64, N // 8, 8), generator=g, device=device).to(torch.float8_e4m3fn)
    ex = (127 + torch.randint(-10, -3, (K // 64, N // 8), generator=g, device=device)).to(torch.uint8)
    return idx, cb.view(torch.uint8), ex
