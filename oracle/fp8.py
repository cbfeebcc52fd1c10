"""W8A8 FP8 (E4M3) linear layer in FP64 -- TEST INFRASTRUCTURE ONLY (tests, smoke and the
bench's CPU baseline use it; the library never does).

The comparison path of "INT8 vs INT4 Quantization, in depth", section "Two regimes: waiting for
memory, waiting for math" and its worked example: 8-bit weights and 8-bit activations feed an
8-bit tensor-core GEMM, so the layer reads twice the weight bytes of W4A16 but runs the math at
twice the 16-bit rate. The pages fix neither the 8-bit format nor the scaling; the readings
taken: FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
finite value 448, S.1111.111 = NaN), one FP32 scale per output channel for the weights and per
row for the activations, s = fp32(amax / 448) (1 when amax = 0), codes = E4M3 round-to-nearest-
even of x / s in FP64 with saturation to +-448, and y[m, n] = sum_k (qa s_a[m]) (qw s_w[n]).
"""
import numpy as np

from . import oracle as _o

E4M3_MAX = 448.0


def e4m3_decode(bits):
    """uint8 E4M3 bit patterns -> float64 (NaN for S.1111.111), from the format's definition."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


_POS = e4m3_decode(np.arange(127, dtype=np.uint8))   # 0x00 .. 0x7E, increasing, 0 .. 448


def e4m3_encode(x):
    """float64 -> E4M3 bits: round to nearest, ties to the even code, saturate to +-448 (finite
    inputs only; the sign of a zero result follows the input)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_POS, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    dlo, dhi = a - _POS[lo], _POS[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(_POS[hi] == a, hi, pick)
    return (pick | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def scales_from_amax(amax):
    """s = fp32(amax / 448), and 1 where amax is 0."""
    s = (np.asarray(amax, dtype=np.float64) / E4M3_MAX).astype(np.float32)
    return np.where(s == 0.0, np.float32(1.0), s).astype(np.float32)


def quantize_weights(W_bits):
    """fp16 W [K, N] -> (codes uint8 [N, K] (one row per output channel, K contiguous),
    scales float32 [N])."""
    W = _o.decode16(W_bits, _o.F16)
    s = scales_from_amax(np.max(np.abs(W), axis=0))
    q = e4m3_encode(W / s.astype(np.float64)[None, :])
    return np.ascontiguousarray(q.T), s


def quantize_acts(A_bits, a_dtype):
    """16-bit A [M, K] -> (codes uint8 [M, K], scales float32 [M])."""
    A = _o.decode16(A_bits, a_dtype)
    s = scales_from_amax(np.max(np.abs(A), axis=1))
    return e4m3_encode(A / s.astype(np.float64)[:, None]), s


def linear(qa, sa, qw, sw):
    """y[m, n] = sum_k (qa[m, k] sa[m]) (qw[n, k] sw[n]) and sum_k |...| in FP64."""
    A = e4m3_decode(qa) * np.asarray(sa, dtype=np.float64)[:, None]
    W = e4m3_decode(qw) * np.asarray(sw, dtype=np.float64)[:, None]
    return A @ W.T, np.abs(A) @ np.abs(W).T
