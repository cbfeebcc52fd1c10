"""Pins of the FP64 oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a value printed on a page
(fixtures under tests/golden/, each with its citation), a library routine (numpy / torch
conversions, numpy matmul), a closed form constructed so its answer is known, or a brute-force
search over all 16 codes.
"""
import json
import os

import numpy as np
import pytest
import torch

from weight_only_int4_07_b200 import synthetic

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _round_half_up(x, digits):
    from decimal import ROUND_HALF_UP, Decimal

    return float(Decimal(repr(x)).quantize(Decimal(1).scaleb(-digits), rounding=ROUND_HALF_UP))


# ----------------------------------------------------------------------------- 16-bit formats
def test_fp16_decode_exhaustive_vs_numpy(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle_mod.decode16(bits, oracle_mod.F16)
    ref = bits.view(np.float16).astype(np.float64)
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_fp16_encode_vs_numpy(oracle_mod):
    rng = np.random.default_rng(1)
    # log-uniform magnitudes across the whole fp16 range and beyond, both signs
    x = np.exp(rng.uniform(np.log(1e-9), np.log(1e6), 200_000)) * rng.choice([-1.0, 1.0], 200_000)
    # exact midpoints between neighbouring fp16 values (ties), including subnormals and the top
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mids = (lo + hi) / 2
    specials = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e5, np.inf, -np.inf,
                         2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -26])
    x = np.concatenate([x, mids, -mids, specials])
    ours = oracle_mod.encode16(x, oracle_mod.F16)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    assert oracle_mod.encode16(np.array([np.nan]), oracle_mod.F16)[0] & 0x7C00 == 0x7C00


def test_bf16_decode_exhaustive_vs_torch(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle_mod.decode16(bits, oracle_mod.BF16)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_bf16_encode_vs_torch(oracle_mod):
    # float32-representable inputs: torch rounds float32 -> bfloat16 once, ties to even
    rng = np.random.default_rng(2)
    x32 = (np.exp(rng.uniform(np.log(1e-40), np.log(1e38), 200_000))
           * rng.choice([-1.0, 1.0], 200_000)).astype(np.float32)
    # exact bf16 midpoints (float32 with the low 16 bits = 0x8000)
    base = rng.integers(0, 0x7F7F, 50_000, dtype=np.uint32) << 16
    mids = (base | 0x8000).view(np.float32)
    x32 = np.concatenate([x32, mids, np.array([0.0, -0.0, 3.0e38, 3.4e38], dtype=np.float32)])
    ours = oracle_mod.encode16(x32.astype(np.float64), oracle_mod.BF16)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ----------------------------------------------------------------------------- sizes (pages)
def test_packed_layout_example(oracle_mod, golden_dir):
    g = json.load(open(os.path.join(golden_dir, "packed_layout_example.json")))
    K, N, group = g["K"], g["N"], g["group"]
    cb, sb, zb = oracle_mod.sizes(K, N, group, g["sym"])
    # shapes printed on the page
    assert cb == g["qweight_shape"][0] * g["qweight_shape"][1] * 4
    assert sb == g["scales_shape"][0] * g["scales_shape"][1] * 2
    assert zb == g["qzeros_shape"][0] * g["qzeros_shape"][1] * 4
    # megabytes as printed (decimal MB, to the printed digits)
    assert round(cb / 1e6, 1) == g["printed_MB"]["qweight"]
    assert round(sb / 1e6, 2) == g["printed_MB"]["scales"]
    assert round(zb / 1e6, 2) == g["printed_MB"]["qzeros"]
    assert round((cb + sb + zb) / 1e6, 1) == g["printed_total_MB"]
    fp16 = K * N * 2
    assert round(fp16 / 1e6, 1) == g["printed_fp16_MB"]
    assert round((cb + sb + zb) / fp16, 2) == g["printed_ratio"]


def test_bits_and_bytes_per_weight(oracle_mod, golden_dir):
    facts = {f["name"]: f for f in json.load(open(os.path.join(golden_dir, "format_facts.json")))["facts"]}
    K, N = 8192, 1024
    # g128, FP16 scale, no zero: 0.515625 byte per weight, i.e. 4.125 bits
    cb, sb, zb = oracle_mod.sizes(K, N, 128, True)
    assert zb == 0
    assert (cb + sb) / (K * N) == facts["bytes_per_weight_g128_fp16_scale"]["value"]
    assert 8 * (cb + sb) / (K * N) == facts["bits_per_weight_g128_scale_only"]["value"]
    # with an INT4 zero per group
    for name, g in (("bits_per_weight_g128_scale_and_zero", 128), ("bits_per_weight_g32_scale_and_zero", 32)):
        cb, sb, zb = oracle_mod.sizes(K, N, g, False)
        bits = 8 * (cb + sb + zb) / (K * N)
        assert bits == facts[name]["exact"]
        # the page rounds half up (4.625 -> 4.63)
        assert _round_half_up(bits, facts[name]["printed_digits"]) == facts[name]["printed"]
        assert round(100 * bits / 16) == facts[name]["fp16_percent_printed"]


# ----------------------------------------------------------------------------- packing
def test_two_codes_per_byte_eight_per_word(oracle_mod, golden_dir):
    facts = {f["name"]: f for f in json.load(open(os.path.join(golden_dir, "format_facts.json")))["facts"]}
    rng = np.random.default_rng(3)
    K, N = 64, 16
    codes = rng.integers(-2**31, 2**31, size=(K // 8, N), dtype=np.int64).astype(np.int32)
    q = oracle_mod.unpack_codes(codes, K, sym=False)
    # byte view: little-endian word, byte b of word (j, n) holds k = 8j + 2b (low) and 8j + 2b + 1
    by = codes.view(np.uint8).reshape(K // 8, N, 4)
    per_word = facts["codes_per_word32"]["value"]
    per_byte = facts["codes_per_byte"]["value"]
    assert per_word == 4 * per_byte
    for j in range(K // 8):
        for b in range(4):
            assert np.array_equal(q[8 * j + 2 * b], by[j, :, b] % 16)
            assert np.array_equal(q[8 * j + 2 * b + 1], by[j, :, b] // 16)


def test_nibble_order_and_code_ranges(oracle_mod, golden_dir):
    facts = {f["name"]: f for f in json.load(open(os.path.join(golden_dir, "format_facts.json")))["facts"]}
    rng_f = facts["signed_int4_range"]
    word = np.array([[0x76543210, np.int32(np.uint32(0xFEDCBA98).view(np.int32))]], dtype=np.int32)
    qa = oracle_mod.unpack_codes(word, 8, sym=False)
    assert qa[:, 0].tolist() == list(range(8))
    assert qa[:, 1].tolist() == list(range(8, 16))
    qs = oracle_mod.unpack_codes(word, 8, sym=True)
    assert qs[:, 0].tolist() == list(range(8))
    assert qs[:, 1].tolist() == list(range(-8, 0))
    allq = np.concatenate([qs[:, 0], qs[:, 1]])
    assert allq.min() == rng_f["lo"] and allq.max() == rng_f["hi"]
    assert len(set(allq.tolist())) == rng_f["levels"]


def test_all_16_codes_dequantize(oracle_mod):
    # brute force: every nibble value through unpack -> dequant, scale 1, every zero-point
    K, N, group = 16, 16, 16
    words = np.zeros((K // 8, N), dtype=np.int64)
    for k in range(K):
        words[k // 8, :] |= (k & 0xF) << (4 * (k % 8))
    codes = words.astype(np.uint32).view(np.int32)
    scales = np.full((1, N), 0x3C00, dtype=np.uint16)  # 1.0
    zw = np.zeros((1, N // 8), dtype=np.int64)
    for n in range(N):
        zw[0, n // 8] |= (n & 0xF) << (4 * (n % 8))
    zeros = zw.astype(np.uint32).view(np.int32)
    W = oracle_mod.dequant(codes, scales, zeros, K, N, group, sym=False)
    for k in range(K):
        for n in range(N):
            assert W[k, n] == (k - n)
    Ws = oracle_mod.dequant(codes, scales, None, K, N, group, sym=True)
    assert sorted(Ws[:, 0].tolist()) == list(range(-8, 8))


# ----------------------------------------------------------------------------- quantizer
def _grid_case(sym, group=32, K=64, N=16, seed=4):
    """W built exactly on a known grid: W = (q - z) * s with s a power of two per group and
    every group reaching both ends of its range, so the quantizer's answer is known."""
    rng = np.random.default_rng(seed)
    G = K // group
    s_exp = rng.integers(-10, -3, size=(G, N))
    s = 2.0 ** s_exp
    if sym:
        q = rng.integers(-7, 8, size=(K, N))
        z = np.zeros((G, N), dtype=np.int64)
        for g in range(G):
            q[g * group, :] = 7        # amax reached: s = amax / 7 exactly
    else:
        z = rng.integers(1, 15, size=(G, N))
        q = rng.integers(0, 16, size=(K, N))
        for g in range(G):
            q[g * group, :] = 0        # lo = -z s
            q[g * group + 1, :] = 15   # hi = (15 - z) s
    W = (q - np.repeat(z, group, axis=0)) * np.repeat(s, group, axis=0)
    Wb = W.astype(np.float16)
    assert np.array_equal(Wb.astype(np.float64), W)   # exactly representable
    return Wb.view(np.uint16), q, z, s


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_known_grid(oracle_mod, sym):
    Wb, q, z, s = _grid_case(sym)
    K, N = Wb.shape
    group = 32
    st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
    assert st == oracle_mod.OK
    assert np.array_equal(oracle_mod.decode16(scales), s)
    assert np.array_equal(oracle_mod.unpack_codes(codes, K, sym), q)
    if not sym:
        assert np.array_equal(oracle_mod.unpack_zeros(zeros, K // group, N), z)
    # and the dequantized weights give back W exactly
    assert np.array_equal(oracle_mod.dequant(codes, scales, zeros, K, N, group, sym),
                          Wb.view(np.float16).astype(np.float64))


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("group", [32, 128])
def test_quantize_is_nearest_grid_point(oracle_mod, sym, group):
    """Brute force: each code is the nearest of the 16 grid points (q - z) * s (ties: even q - z)
    for every weight inside the grid's range; weights outside it take the nearest end."""
    K, N = 256, 64
    Wb = synthetic.weights_student_t(K, N, seed=5)
    st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
    assert st == oracle_mod.OK
    W = oracle_mod.decode16(Wb)
    q = oracle_mod.unpack_codes(codes, K, sym)
    s = np.repeat(oracle_mod.decode16(scales), group, axis=0)
    if sym:
        z = np.zeros_like(q)
        cand = np.arange(-8, 8)
    else:
        z = np.repeat(oracle_mod.unpack_zeros(zeros, K // group, N), group, axis=0)
        cand = np.arange(16)
    grid = (cand[None, None, :] - z[:, :, None]) * s[:, :, None]          # [K, N, 16]
    dist = np.abs(W[:, :, None] - grid)
    best = dist.min(axis=2)
    chosen = np.abs(W - (q - z) * s)
    assert np.array_equal(chosen, best)
    # ties go to an even (q - z)
    ntie = (dist == best[:, :, None]).sum(axis=2)
    assert np.all(((q - z)[ntie > 1] % 2) == 0)


def test_quantize_tie_breaks_to_even():
    import oracle as o
    # one group of 8 weights, s = 2^-6 (hi = 15 s, lo = 0): weights at k + 0.5 ticks
    s = 2.0 ** -6
    ticks = np.array([15, 0, 0.5, 1.5, 2.5, 3.5, 4.5, 5.5])
    W = (ticks * s).astype(np.float16).reshape(8, 1).repeat(8, axis=1)
    st, codes, scales, zeros = o.quantize(W.view(np.uint16), 8, False)
    assert st == o.OK
    assert o.decode16(scales)[0, 0] == s
    assert o.unpack_zeros(zeros, 1, 8)[0, 0] == 0
    q = o.unpack_codes(codes, 8, False)[:, 0]
    assert q.tolist() == [15, 0, 0, 2, 2, 4, 4, 6]


def test_quantize_step_count_matches_tick_gap(oracle_mod, golden_dir):
    """The asymmetric grid spans its range in 15 steps (16 levels); an 8-bit grid over the same
    range has 255, so the INT4 tick is 255/15 = 17 times the INT8 tick."""
    facts = {f["name"]: f for f in json.load(open(os.path.join(golden_dir, "format_facts.json")))["facts"]}
    tick = facts["int8_vs_int4_tick_gap"]
    assert tick["int8_steps"] / tick["int4_steps"] == tick["printed"]
    K, N, group = 128, 64, 128
    Wb = synthetic.weights_normal(K, N, seed=6)
    st, codes, scales, zeros = oracle_mod.quantize(Wb, group, False)
    W = oracle_mod.decode16(Wb)
    lo = np.minimum(W.min(axis=0), 0)
    hi = np.maximum(W.max(axis=0), 0)
    s = oracle_mod.decode16(scales)[0]
    steps = (hi - lo) / s
    assert np.all(np.abs(steps - tick["int4_steps"]) <= tick["int4_steps"] * 2.0 ** -10)


def test_quantize_scale_against_numpy_rounding(oracle_mod):
    """The stored fp16 scale is the correctly rounded range / steps (numpy's float16 cast)."""
    K, N, group = 256, 128, 32
    Wb = synthetic.weights_outliers(K, N, seed=7, frac=0.01)
    W = Wb.view(np.float16).astype(np.float64).reshape(K // group, group, N)
    for sym in (False, True):
        st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
        if sym:
            ref = (np.abs(W).max(axis=1) / 7.0).astype(np.float16)
        else:
            ref = ((np.maximum(W.max(axis=1), 0) - np.minimum(W.min(axis=1), 0)) / 15.0).astype(np.float16)
        assert np.array_equal(scales, ref.view(np.uint16))


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_error_within_half_tick(oracle_mod, sym):
    K, N, group = 512, 64, 128
    Wb = synthetic.weights_normal(K, N, seed=8)
    st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
    W = oracle_mod.decode16(Wb)
    What = oracle_mod.dequant(codes, scales, zeros, K, N, group, sym)
    q = oracle_mod.unpack_codes(codes, K, sym)
    s = np.repeat(oracle_mod.decode16(scales), group, axis=0)
    lo_code, hi_code = (-8, 7) if sym else (0, 15)
    inside = (q > lo_code) & (q < hi_code)
    assert np.all(np.abs(W - What)[inside] <= s[inside] / 2)


def test_quantize_invariants(oracle_mod):
    K, N, group = 256, 64, 32
    Wb = synthetic.weights_normal(K, N, seed=9)
    W16 = Wb.view(np.float16)
    for sym in (False, True):
        st, c1, s1, z1 = oracle_mod.quantize(Wb, group, sym)
        # scaling by a power of two scales s and keeps every code and zero
        st, c2, s2, z2 = oracle_mod.quantize((W16 * np.float16(4)).view(np.uint16), group, sym)
        assert np.array_equal(c1, c2)
        assert np.array_equal(oracle_mod.decode16(s2), 4 * oracle_mod.decode16(s1))
        if not sym:
            assert np.array_equal(z1, z2)
    # symmetric: negating W negates the codes (none of them is -8 here) and keeps the scales
    st, c1, s1, _ = oracle_mod.quantize(Wb, group, True)
    st, c3, s3, _ = oracle_mod.quantize((-W16).view(np.uint16), group, True)
    q1 = oracle_mod.unpack_codes(c1, K, True)
    assert q1.min() > -8
    assert np.array_equal(oracle_mod.unpack_codes(c3, K, True), -q1)
    assert np.array_equal(s1, s3)


def test_quantize_degenerate_and_nonfinite(oracle_mod):
    K, N, group = 64, 16, 32
    Wb = synthetic.weights_normal(K, N, seed=10).copy()
    Wb[:32, 3] = 0               # all-zero group -> s = 1, z = 0, codes = z, w = 0
    for sym in (False, True):
        st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
        assert st == oracle_mod.OK
        assert scales[0, 3] == 0x3C00
        What = oracle_mod.dequant(codes, scales, zeros, K, N, group, sym)
        assert np.all(What[:32, 3] == 0)
        if not sym:
            assert oracle_mod.unpack_zeros(zeros, K // group, N)[0, 3] == 0
    Wn = Wb.copy()
    Wn[40, 5] = 0x7C00           # +inf
    st, *_ = oracle_mod.quantize(Wn, group, False)
    assert st == oracle_mod.ENONFINITE
    Wn[40, 5] = 0x7E00           # NaN
    st, *_ = oracle_mod.quantize(Wn, group, True)
    assert st == oracle_mod.ENONFINITE


def test_quantize_group_equals_k_is_per_channel(oracle_mod):
    """group = K gives one scale per output channel: the same codes as quantizing each column
    alone as a K x 8 matrix whose eight columns are copies of it."""
    K, N = 128, 16
    Wb = synthetic.weights_normal(K, N, seed=11)
    st, codes, scales, zeros = oracle_mod.quantize(Wb, K, False)
    assert scales.shape == (1, N)
    q = oracle_mod.unpack_codes(codes, K, False)
    for n in (0, 7, 15):
        col = np.repeat(Wb[:, n:n + 1], 8, axis=1)
        st, c1, s1, z1 = oracle_mod.quantize(col, K, False)
        assert np.array_equal(oracle_mod.unpack_codes(c1, K, False)[:, 0], q[:, n])
        assert s1[0, 0] == scales[0, n]


# ----------------------------------------------------------------------------- the layer
@pytest.mark.parametrize("a_dtype", [0, 1])
def test_linear_matches_numpy_matmul(oracle_mod, a_dtype):
    M, K, N, group = 3, 256, 64, 128
    Wb = synthetic.weights_normal(K, N, seed=12)
    A = synthetic.activations(M, K, seed=13, dtype=a_dtype)
    st, codes, scales, zeros = oracle_mod.quantize(Wb, group, False)
    What = oracle_mod.dequant(codes, scales, zeros, K, N, group, False)
    a = oracle_mod.decode16(A, a_dtype)
    ref = a @ What
    refabs = np.abs(a) @ np.abs(What)
    Y, Yabs = oracle_mod.linear(A, a_dtype, codes, scales, zeros, N, group, False)
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(Yabs, refabs, rtol=1e-12, atol=0)
    cols = np.array([5, 0, 63, 17])
    Yc, _ = oracle_mod.linear(A, a_dtype, codes, scales, zeros, N, group, False, cols=cols)
    assert np.array_equal(Yc, Y[:, cols])
    assert np.allclose(oracle_mod.matmul(A, a_dtype, What), ref, rtol=1e-12, atol=1e-12)


def test_linear_unit_rows_return_dequantized_rows(oracle_mod):
    K, N, group = 64, 32, 32
    Wb = synthetic.weights_normal(K, N, seed=14)
    for sym in (False, True):
        st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
        What = oracle_mod.dequant(codes, scales, zeros, K, N, group, sym)
        rows = [0, 7, 8, 31, 32, 63]
        A = np.zeros((len(rows), K), dtype=np.uint16)
        for i, k in enumerate(rows):
            A[i, k] = 0x3C00
        Y, _ = oracle_mod.linear(A, 0, codes, scales, zeros, N, group, sym)
        assert np.array_equal(Y, What[rows])


def test_quantized_layer_tracks_the_fp16_layer(oracle_mod):
    """End to end: the W4A16 output differs from the FP16 layer by at most the half-tick
    bound sum_k |a_k| * s_k / 2 (weights that were not clipped)."""
    M, K, N, group = 2, 512, 32, 128
    Wb = synthetic.weights_normal(K, N, seed=15)
    A = synthetic.activations(M, K, seed=16)
    st, codes, scales, zeros = oracle_mod.quantize(Wb, group, False)
    Y, _ = oracle_mod.linear(A, 0, codes, scales, zeros, N, group, False)
    a = oracle_mod.decode16(A)
    W = oracle_mod.decode16(Wb)
    s = np.repeat(oracle_mod.decode16(scales), group, axis=0)
    bound = np.abs(a) @ (s / 2) * (1 + 2.0 ** -9)
    assert np.all(np.abs(Y - a @ W) <= bound)


# ----------------------------------------------------------------------------- tiled layout
def _slots(word):
    """The eight nibbles of a word, slot 0 first."""
    return [(int(word) >> (4 * i)) & 0xF for i in range(8)]


def test_tiled_layout_positions_and_bijection(oracle_mod):
    """The tiled buffer is a permutation of the plain words into unit records: each word lands
    once, at the byte the layout's definition gives (closed forms for chosen words: unit record
    t * K/128 + c, block h at 2048 h, channel slot n XOR 2h, word w), with its codes in slot
    order (e0, e2, e4, e6, e1, e3, e5, e7); every record carries its unit's scales and zeros."""
    K, N, group = 256, 384, 64
    G = 128 // group
    rows = K // 8
    rng = np.random.default_rng(17)
    codes = rng.integers(-2**31, 2**31, size=(rows, N), dtype=np.int64).astype(np.int32)
    scales = np.arange((K // group) * N, dtype=np.uint16).reshape(K // group, N)
    zeros = np.arange((K // group) * (N // 8), dtype=np.int32).reshape(K // group, N // 8)
    buf = oracle_mod.repack(codes, scales, zeros, K, N, group, False)
    off = oracle_mod.tiled_offsets(K, N, group, False)
    R = off["record"]
    assert R == 8192 + G * 256 + G * 64 and off["total"] == (N // 128) * (K // 128) * R
    assert off["zeros_bytes"] == G * 64 and oracle_mod.tiled_offsets(K, N, group, True)["zeros_bytes"] == 0
    assert oracle_mod.tiled_offsets(K, N, group, True)["record"] == 8192 + G * 256
    assert len(buf) == off["total"]

    def word_at(byte):
        return int(buf[byte: byte + 4].view(np.uint32)[0])

    def check(byte, j, n):
        e = _slots(np.uint32(codes[j, n]))
        assert _slots(word_at(byte)) == [e[0], e[2], e[4], e[6], e[1], e[3], e[5], e[7]]

    check(0, 0, 0)                      # record 0, block 0, channel 0, word 0
    check(4, 1, 0)                      # four consecutive rows of one channel in 16 bytes
    check(12, 3, 0)
    check(16, 0, 1)                     # then the next channel (slot 1 XOR 0)
    check(2048 + 16 * 2, 4, 0)          # block 1 (rows 4..7): channel 0 sits in slot 0 XOR 2
    check(2048 + 16 * 0, 4, 2)          # ... and channel 2 in slot 2 XOR 2 = 0
    check(3 * 2048 + 16 * (5 ^ 6) + 8, 12 + 2, 5)      # block 3, slot 5 XOR 6, word 2
    check(R, 16, 0)                     # next record along K
    check(2 * R + 16 * 1, 0, 129)                      # t = 1, c = 0: record 1 * K/128 + 0
    check(3 * R + 2048 + 16 * (1 ^ 2) + 4, 21, 129)   # t = 1, c = 1, block 1, word 1
    # a bijection: decode every code word of every record and compare the multisets
    def decode(tw):
        s_ = _slots(np.uint32(tw))
        e = [s_[0], s_[4], s_[1], s_[5], s_[2], s_[6], s_[3], s_[7]]
        return sum(v << (4 * i) for i, v in enumerate(e))
    recs = buf.reshape(-1, R)
    words = recs[:, :8192].copy().view(np.uint32).reshape(-1)
    back = np.array(sorted(decode(tw) for tw in words), dtype=np.int64)
    assert np.array_equal(back, np.sort((codes.astype(np.int64) & 0xFFFFFFFF).reshape(-1)))
    # scales and zeros of unit (t, c): plain group rows c*G .. c*G + G-1, the tile's channels
    for t in range(N // 128):
        for c in range(K // 128):
            rec = recs[t * (K // 128) + c]
            sc = rec[8192: 8192 + G * 256].copy().view(np.uint16).reshape(G, 128)
            zr = rec[8192 + G * 256:].copy().view(np.int32).reshape(G, 16)
            assert np.array_equal(sc, scales[c * G: c * G + G, 128 * t: 128 * t + 128])
            assert np.array_equal(zr, zeros[c * G: c * G + G, 16 * t: 16 * t + 16])


def test_tiled_layout_symmetric_is_offset_binary(oracle_mod):
    """Symmetric codes -8..7 are stored as q + 8 (0..15) in the tiled buffer."""
    K, N, group = 128, 128, 32
    q = np.tile(np.arange(-8, 8), 4 * N // 16 * K // 4)[: K * N].reshape(K, N)
    words = np.zeros((K // 8, N), dtype=np.int64)
    for k in range(K):
        words[k // 8] |= (q[k] & 0xF).astype(np.int64) << (4 * (k % 8))
    codes = words.astype(np.uint32).view(np.int32)
    scales = np.full((K // group, N), 0x3C00, dtype=np.uint16)
    buf = oracle_mod.repack(codes, scales, None, K, N, group, True)
    t = buf[: K * N // 2].view(np.int32)
    # word (j = 0, n = 0) sits at position 0: its slots hold q[0, 0..7 even], q[.. odd] + 8
    e = [q[k, 0] + 8 for k in range(8)]
    assert _slots(np.uint32(t[0])) == [e[0], e[2], e[4], e[6], e[1], e[3], e[5], e[7]]


def test_tiled_layout_zero_point_groups_store_scale_zero(oracle_mod):
    """A (group, channel) whose codes all equal its zero point -- the degenerate group, whose
    dequantized weights are all zero -- stores scale 0 in the tiled buffer; every other scale is
    copied. Dequantizing either buffer gives the same weights."""
    K, N, group = 256, 128, 64
    Wb = np.array(np.random.default_rng(5).standard_normal((K, N)) * 0.02, dtype=np.float16).view(np.uint16).copy()
    Wb[64:128, 7] = 0                  # a group of zeros: scale rounds to 0, stored 1, codes = zero point
    Wb[:64, 9] = 0x0001                # a sub-2^-25 range: the same
    for sym in (0, 1):
        st, codes, scales, zeros = oracle_mod.quantize(Wb, group, sym)
        assert scales[1, 7] == 0x3C00 and scales[0, 9] == 0x3C00
        buf = oracle_mod.repack(codes, scales, zeros, K, N, group, sym)
        off = oracle_mod.tiled_offsets(K, N, group, sym)
        G = 128 // group
        recs = buf.reshape(-1, off["record"])
        sc = np.concatenate([recs[c][8192: 8192 + G * 256].copy().view(np.uint16).reshape(G, 128)
                             for c in range(K // 128)])          # tile 0: [K/g, 128]
        expect = scales[:, :128].copy()
        expect[1, 7] = 0
        expect[0, 9] = 0
        assert np.array_equal(sc, expect)
        zeroed = scales.copy()
        zeroed[1, 7] = zeroed[0, 9] = 0
        assert np.array_equal(oracle_mod.dequant(codes, zeroed, zeros, K, N, group, sym),
                              oracle_mod.dequant(codes, scales, zeros, K, N, group, sym))
