"""Pins of the FP8 (E4M3) oracle of the W8A8 comparison path: decoding of all 256 codes and
rounding of fp32-exact values against torch's float8_e4m3fn type, round trips, saturation, the
scale of the largest element, and the E4M3 rounding bound on the layer output."""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from weight_only_int4_07_b200 import synthetic


def test_decode_matches_torch_for_all_codes():
    b = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.e4m3_decode(b)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert np.array_equal(np.signbit(ref[~both_nan]), np.signbit(got[~both_nan]))
    assert fp8.e4m3_decode(np.array([0x7E], dtype=np.uint8))[0] == 448.0
    assert fp8.e4m3_decode(np.array([0x01], dtype=np.uint8))[0] == 2.0 ** -9


def test_encode_matches_torch_on_fp32_values():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.uniform(-448, 448, 20000), rng.standard_normal(20000), rng.standard_normal(20000) * 1e-2,
        rng.standard_normal(5000) * 2.0 ** -8,
    ]).astype(np.float32)
    # every midpoint between adjacent positive codes (exact in fp32) and its negative
    pos = fp8.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp8.e4m3_encode(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_round_trip_and_saturation():
    b = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(fp8.e4m3_encode(fp8.e4m3_decode(b)), b)
    assert fp8.e4m3_encode(np.array([1e6]))[0] == 0x7E
    assert fp8.e4m3_encode(np.array([-1e6]))[0] == 0xFE
    assert fp8.e4m3_encode(np.array([464.0]))[0] == 0x7E


def test_largest_element_maps_to_the_largest_code():
    K, N = 256, 64
    Wb = synthetic.weights_outliers(K, N, 8)
    q, s = fp8.quantize_weights(Wb)
    W = oracle.decode16(Wb)
    n_arg = np.argmax(np.abs(W), axis=0)
    for n in range(N):
        assert (q[n, n_arg[n]] & 0x7F) == 0x7E
    assert q.shape == (N, K) and s.dtype == np.float32
    z, sz = fp8.quantize_weights(np.zeros((K, 8), dtype=np.uint16))
    assert np.all(z == 0) and np.all(sz == 1.0)


@pytest.mark.parametrize("a_dtype", [0, 1])
def test_layer_error_within_the_e4m3_rounding_bound(a_dtype):
    """Each E4M3 rounding in the normal range is within 2^-4 relative (3 mantissa bits), so the
    W8A8 output stays within ((1 + 2^-4)^2 - 1) sum|a w| of the exact product, plus the
    subnormal steps (2^-10 s per value)."""
    M, K, N = 4, 512, 96
    Wb = synthetic.weights_normal(K, N, 9)
    Ab = synthetic.activations(M, K, 10, dtype=a_dtype)
    qw, sw = fp8.quantize_weights(Wb)
    qa, sa = fp8.quantize_acts(Ab, a_dtype)
    y, _ = fp8.linear(qa, sa, qw, sw)
    A, W = oracle.decode16(Ab, a_dtype), oracle.decode16(Wb)
    exact = A @ W
    absum = np.abs(A) @ np.abs(W)
    sub = (2.0 ** -10) * (sa[:, None] * (np.abs(W).sum(axis=0))[None, :] +
                          (np.abs(A).sum(axis=1))[:, None] * sw[None, :])
    bound = ((1 + 2.0 ** -4) ** 2 - 1) * absum + sub + 1e-12
    assert np.all(np.abs(y - exact) <= bound)
