"""Seeded synthetic inputs for the W4A16 linear layer.

This module only draws random numbers: it holds none of the layer's arithmetic (no
quantization, packing, dequantization or products). Both the FP64 oracle's checks and the CUDA
path take their inputs from here. Every generator is seeded (numpy PCG64) and returns uint16
bit patterns of the 16-bit float type, so the two sides see identical bits.

Distributions follow the workloads the layer is measured on:
  * weights ~ N(0, 0.02) in fp16;
  * weights ~ N(0, 0.02) with a fixed fraction of entries (a seeded sample without
    replacement) multiplied by a constant (outliers);
  * weights ~ 0.02 * Student-t(nu=5) in fp16;
  * activations ~ N(0, 1) in fp16 or bf16;
  * calibration inputs for the calibrated encoders: rows with correlated channels (a rank-K/8
    common part plus independent noise) and 1% of the channels (a seeded sample) scaled by 10,
    the outlier channels that activation-aware methods look for.
"""
import numpy as np
import torch

F16 = 0
BF16 = 1


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _to_bits(x32: np.ndarray, dtype: int) -> np.ndarray:
    """Round float32 samples to the 16-bit input type and return the bit patterns."""
    if dtype == F16:
        return np.ascontiguousarray(x32.astype(np.float16)).view(np.uint16)
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def weights_normal(K, N, seed, std=0.02):
    return _to_bits(_rng(seed).standard_normal((K, N), dtype=np.float32) * np.float32(std), F16)


def weights_outliers(K, N, seed, std=0.02, frac=0.001, mult=20.0):
    rng = _rng(seed)
    w = rng.standard_normal((K, N), dtype=np.float32) * np.float32(std)
    n_out = int(round(frac * K * N))
    idx = rng.choice(K * N, size=n_out, replace=False)
    w.reshape(-1)[idx] *= np.float32(mult)
    return _to_bits(w, F16)


def weights_student_t(K, N, seed, nu=5.0, scale=0.02):
    w = _rng(seed).standard_t(nu, size=(K, N)).astype(np.float32) * np.float32(scale)
    return _to_bits(w, F16)


def activations(M, K, seed, dtype=F16, std=1.0):
    return _to_bits(_rng(seed).standard_normal((M, K), dtype=np.float32) * np.float32(std), dtype)


def calibration(S, K, seed, dtype=F16, outlier_frac=0.01, outlier_mult=10.0):
    """S calibration rows of K input channels: Z B / sqrt(r) + 0.5 E with Z [S, r], B [r, K],
    E [S, K] standard normal (r = max(1, K / 8)), then a seeded 1% of the channels times 10."""
    rng = _rng(seed)
    r = max(1, K // 8)
    Z = rng.standard_normal((S, r), dtype=np.float32)
    B = rng.standard_normal((r, K), dtype=np.float32)
    x = (Z @ B) / np.float32(np.sqrt(r)) + np.float32(0.5) * rng.standard_normal((S, K), dtype=np.float32)
    n_out = max(1, int(round(outlier_frac * K)))
    idx = rng.choice(K, size=n_out, replace=False)
    x[:, idx] *= np.float32(outlier_mult)
    return _to_bits(x, dtype)


def column_sample(N, count, seed):
    """A seeded sample of output columns that always holds the first and the last column."""
    rng = _rng(seed)
    cols = set(int(c) for c in rng.choice(N, size=min(count, N), replace=False))
    cols.update({0, N - 1})
    return np.array(sorted(cols), dtype=np.int64)
