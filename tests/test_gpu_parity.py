"""GPU parity: the CUDA path against the FP64 oracle, element by element, through the C ABI.

Bars: codes, scales, zeros and the repacked buffer bit-exact; every GEMM output within
|y - y_ref| <= 2e-3 * sum_k |a_k * w_k| + 1e-5, y the kernel's 16-bit output widened to FP64.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_07_b200 import native, synthetic

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-5
_cache = {}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from weight_only_int4_07_b200 import build

    build.build()
    native.lib()
    torch.cuda.set_device(0)


def _weights(kind, K, N, seed):
    key = ("W", kind, K, N, seed)
    if key not in _cache:
        gen = {"normal": synthetic.weights_normal, "outliers": synthetic.weights_outliers,
               "student_t": synthetic.weights_student_t}[kind]
        _cache[key] = gen(K, N, seed)
    return _cache[key]


def _quantized(kind, K, N, group, sym, seed):
    """(W bits, oracle codes/scales/zeros, GPU codes/scales/zeros)."""
    key = ("Q", kind, K, N, group, sym, seed)
    if key not in _cache:
        Wb = _weights(kind, K, N, seed)
        st, oc, os_, oz = oracle.quantize(Wb, group, sym)
        assert st == oracle.OK
        W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).cuda()
        gc, gs, gz = native.w4a16_quantize(W, group, sym)
        torch.cuda.synchronize()
        _cache[key] = (Wb, (oc, os_, oz), (gc, gs, gz))
    return _cache[key]


def _to_np16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _acts(M, K, seed, dtype):
    Ab = synthetic.activations(M, K, seed, dtype=dtype)
    tdt = torch.float16 if dtype == synthetic.F16 else torch.bfloat16
    A = torch.from_numpy(Ab.view(np.int16)).view(tdt).cuda()
    return Ab, A


def _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym, cols=None, out_rel=0.0):
    """C within REL * sum|a w| + ABS of the oracle, element by element; out_rel * |y| more where
    a test's rows are dominated by one term (a 16-bit output rounding alone is up to 2^-8 |y|
    in bf16)."""
    Y, Yabs = oracle.linear(Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)
    y = oracle.decode16(_to_np16(C), a_dtype)
    if cols is not None:
        y = y[:, cols]
    err = np.abs(y - Y)
    bound = REL * Yabs + ABS + out_rel * np.abs(Y)
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outputs outside the bound; worst ratio "
                           f"{(err / bound).max():.3f}")
    return float((err / bound).max())


# ----------------------------------------------------------------------------- quantize
QUANT_CASES = [
    # kind, K, N, group, sym, seed
    ("normal", 512, 256, 128, 0, 0),          # the tiny configuration
    ("normal", 384, 264, 32, 1, 1),           # ragged N (not a multiple of the 256-thread block)
    ("student_t", 1024, 520, 64, 0, 2),
    ("outliers", 2048, 1032, 128, 1, 3),
    ("normal", 4096, 6144, 128, 0, 4),        # 8B qkv shape
    ("student_t", 8192, 8192, 32, 1, 5),      # format variant, full size
    ("outliers", 8192, 28672, 128, 0, 6),     # sweep shape, full size
]


@pytest.mark.parametrize("kind,K,N,group,sym,seed", QUANT_CASES)
def test_quantize_bit_exact(kind, K, N, group, sym, seed):
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized(kind, K, N, group, sym, seed)
    assert np.array_equal(gc.cpu().numpy(), oc)
    assert np.array_equal(_to_np16(gs), os_)
    if sym:
        assert gz is None
    else:
        assert np.array_equal(gz.cpu().numpy(), oz)


def test_quantize_degenerate_groups_bit_exact():
    K, N, group = 256, 128, 32
    Wb = synthetic.weights_normal(K, N, seed=7).copy()
    Wb[:32, 5] = 0                     # all-zero group
    Wb[32:64, 9] = 0x0001              # sub-2^-25 range: scale rounds to zero
    for sym in (0, 1):
        st, oc, os_, oz = oracle.quantize(Wb, group, sym)
        W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).cuda()
        gc, gs, gz = native.w4a16_quantize(W, group, sym)
        assert np.array_equal(gc.cpu().numpy(), oc)
        assert np.array_equal(_to_np16(gs), os_)
        if not sym:
            assert np.array_equal(gz.cpu().numpy(), oz)


def test_quantize_reports_nonfinite():
    K, N, group = 256, 128, 128
    Wb = synthetic.weights_normal(K, N, seed=8).copy()
    Wb[77, 3] = 0x7C00                 # +inf
    for sym in (0, 1):
        W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).cuda()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        gc, gs, gz = native.w4a16_quantize(W, group, sym, dev_status=status)
        assert int(status.item()) == native.ENONFINITE
        # the other groups are still exact
        st, oc, os_, oz = oracle.quantize(Wb, group, sym)
        assert st == oracle.ENONFINITE
        ok_cols = np.arange(N) != 3
        assert np.array_equal(gc.cpu().numpy()[:, ok_cols], oc[:, ok_cols])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    W = torch.from_numpy(synthetic.weights_normal(K, N, seed=9).view(np.int16)).view(torch.float16).cuda()
    native.w4a16_quantize(W, group, 0, dev_status=status)
    assert int(status.item()) == 0


# ----------------------------------------------------------------------------- repack
@pytest.mark.parametrize("K,N,group,sym", [(512, 256, 128, 0), (256, 384, 32, 1), (4096, 6144, 128, 0),
                                            (8192, 8192, 32, 1)])
def test_repack_bit_exact(K, N, group, sym):
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("normal" if K < 8192 else "student_t", K, N, group,
                                                 sym, 4 if K == 4096 else (5 if K == 8192 else 11))
    ref = oracle.repack(oc, os_, oz, K, N, group, sym)
    off = oracle.tiled_offsets(K, N, group, sym)
    assert native.w4a16_repack_bytes(K, N, group, sym) == off["total"]
    buf = native.w4a16_repack(gc, gs, gz, K, N, group, sym).cpu().numpy()
    assert buf.size == ref.size
    recs, rrec = buf.reshape(-1, off["record"]), ref.reshape(-1, off["record"])
    for name, a, n in (("codes", 0, off["codes_bytes"]), ("scales", off["scales"], off["scales_bytes"]),
                       ("zeros", off["zeros"], off["zeros_bytes"])):
        assert np.array_equal(recs[:, a:a + n], rrec[:, a:a + n]), name


# ----------------------------------------------------------------------------- GEMM, small
SMALL_GEMM = [
    # M, K, N, group, sym, a_dtype
    (1, 512, 256, 128, 0, 0),     # the tiny configuration
    (1, 384, 264, 32, 1, 1),
    (2, 1024, 520, 64, 0, 0),
    (3, 256, 1032, 128, 1, 1),
    (5, 768, 136, 32, 0, 1),
    (8, 1024, 264, 128, 0, 0),
    (13, 512, 392, 64, 1, 0),
    (16, 2048, 1032, 128, 0, 1),
    (17, 512, 256, 32, 0, 0),
    (33, 1024, 520, 128, 1, 1),
    (64, 512, 384, 64, 0, 0),
]


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", SMALL_GEMM)
@pytest.mark.parametrize("kernel", [native.KERNEL_AUTO, native.KERNEL_GEMV])
def test_gemm_small_full_output(M, K, N, group, sym, a_dtype, kernel):
    kind = "student_t" if sym else "normal"
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized(kind, K, N, group, sym, 20 + K + N)
    Ab, A = _acts(M, K, 100 + M, a_dtype)
    C = native.w4a16_gemm(A, gc, gs, gz, N, group, sym, kernel=kernel)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


@pytest.mark.parametrize("a_dtype", [0, 1])
@pytest.mark.parametrize("sym", [0, 1])
def test_gemm_unit_rows_return_dequantized_rows(a_dtype, sym):
    K, N, group = 512, 256, 64
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("normal", K, N, group, sym, 31)
    rows = [0, 1, 7, 8, 63, 64, 200, 511]
    Ab = np.zeros((len(rows), K), dtype=np.uint16)
    one = 0x3C00 if a_dtype == 0 else 0x3F80
    for i, k in enumerate(rows):
        Ab[i, k] = one
    tdt = torch.float16 if a_dtype == 0 else torch.bfloat16
    A = torch.from_numpy(Ab.view(np.int16)).view(tdt).cuda()
    C = native.w4a16_gemm(A, gc, gs, gz, N, group, sym)
    What = oracle.dequant(oc, os_, oz, K, N, group, sym)
    expect = oracle.decode16(oracle.encode16(What[rows], a_dtype), a_dtype)   # one rounding
    got = oracle.decode16(_to_np16(C), a_dtype)
    assert np.array_equal(got, expect)


def test_gemm_zero_weights_give_zero():
    K, N, group = 256, 128, 32
    Wb = np.zeros((K, N), dtype=np.uint16)
    W = torch.zeros((K, N), dtype=torch.float16, device="cuda")
    for sym in (0, 1):
        gc, gs, gz = native.w4a16_quantize(W, group, sym)
        Ab, A = _acts(4, K, 5, 0)
        C = native.w4a16_gemm(A, gc, gs, gz, N, group, sym)
        assert torch.count_nonzero(C).item() == 0
    assert Wb.sum() == 0


def test_gemm_deterministic():
    M, K, N, group = 4, 2048, 1032, 128
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("normal", K, N, group, 0, 40)
    Ab, A = _acts(M, K, 41, 1)
    C1 = native.w4a16_gemm(A, gc, gs, gz, N, group, 0)
    C2 = native.w4a16_gemm(A, gc, gs, gz, N, group, 0)
    assert torch.equal(C1.view(torch.int16), C2.view(torch.int16))


# ----------------------------------------------------------------------------- full-size, sampled
LLAMA8B = [(4096, 6144), (4096, 4096), (4096, 28672), (14336, 4096)]


@pytest.mark.parametrize("K,N", LLAMA8B)
def test_gemm_llama8b_decode_sampled(K, N):
    group, sym, a_dtype = 128, 0, 0
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("normal", K, N, group, sym, 1000 + N)
    Ab, A = _acts(1, K, 2000 + K, a_dtype)
    cols = synthetic.column_sample(N, 512, seed=K + N)
    C = native.w4a16_gemm(A, gc, gs, gz, N, group, sym)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)


@pytest.mark.parametrize("M", [1, 16, 256])
def test_gemm_sweep_shape_sampled(M):
    K, N, group, sym, a_dtype = 8192, 28672, 128, 0, 1
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("outliers", K, N, group, sym, 6)
    Ab, A = _acts(M, K, 3000 + M, a_dtype)
    cols = synthetic.column_sample(N, 128, seed=M)
    C = native.w4a16_gemm(A, gc, gs, gz, N, group, sym)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)


@pytest.mark.parametrize("sym,group,a_dtype", [(s, g, d) for s in (0, 1) for g in (32, 128) for d in (0, 1)])
def test_gemm_format_variants_sampled(sym, group, a_dtype):
    K = N = 8192
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("student_t", K, N, group, sym, 5)
    for M in (1, 16, 256):
        Ab, A = _acts(M, K, 4000 + M, a_dtype)
        cols = synthetic.column_sample(N, 64, seed=M + group)
        C = native.w4a16_gemm(A, gc, gs, gz, N, group, sym)
        torch.cuda.synchronize()
        _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)


# ----------------------------------------------------------------------------- tiled layout + tcgen05
def _tiled(kind, K, N, group, sym, seed):
    key = ("T", kind, K, N, group, sym, seed)
    if key not in _cache:
        Wb, o, (gc, gs, gz) = _quantized(kind, K, N, group, sym, seed)
        _cache[key] = (Wb, o, native.w4a16_repack(gc, gs, gz, K, N, group, sym))
    return _cache[key]


TILED_GEMM = [
    # M, K, N, group, sym, a_dtype
    (1, 512, 256, 128, 0, 0),
    (16, 512, 256, 32, 1, 1),
    (17, 1024, 384, 64, 0, 0),
    (32, 768, 128, 32, 0, 1),
    (33, 1024, 256, 128, 1, 0),
    (64, 2048, 512, 128, 0, 1),
    (100, 512, 384, 64, 1, 1),
    (128, 1024, 256, 32, 0, 0),
    (200, 512, 128, 128, 0, 1),
    (256, 1024, 384, 64, 0, 0),
    (300, 512, 256, 32, 1, 1),
]


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", TILED_GEMM)
@pytest.mark.parametrize("kernel", [native.KERNEL_TC, native.KERNEL_AUTO])
def test_gemm_tiled_full_output(M, K, N, group, sym, a_dtype, kernel):
    kind = "student_t" if sym else "normal"
    Wb, (oc, os_, oz), tiled = _tiled(kind, K, N, group, sym, 60 + K + N)
    Ab, A = _acts(M, K, 500 + M, a_dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                              kernel=kernel, dev_status=status)
    except native.W4A16Error as e:
        # the AUTO dispatch may pick a kernel that has no tiled variant for this M
        assert kernel == native.KERNEL_AUTO and e.status == native.EUNSUPPORTED
        return
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


@pytest.mark.parametrize("a_dtype", [0, 1])
@pytest.mark.parametrize("sym", [0, 1])
@pytest.mark.parametrize("reps", [5, 25])
def test_gemm_tc_unit_rows_return_dequantized_rows(a_dtype, sym, reps):
    K, N, group = 512, 256, 64
    Wb, (oc, os_, oz), tiled = _tiled("normal", K, N, group, sym, 31)
    # 40 rows (a 64-row tile, two MMA threads) or 200 rows (a 256-row tile, N = 256 MMAs)
    rows = [0, 1, 7, 8, 63, 64, 200, 511] * reps
    Ab = np.zeros((len(rows), K), dtype=np.uint16)
    one = 0x3C00 if a_dtype == 0 else 0x3F80
    for i, k in enumerate(rows):
        Ab[i, k] = one
    tdt = torch.float16 if a_dtype == 0 else torch.bfloat16
    A = torch.from_numpy(Ab.view(np.int16)).view(tdt).cuda()
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                          kernel=native.KERNEL_TC)
    What = oracle.dequant(oc, os_, oz, K, N, group, sym)
    expect = oracle.decode16(oracle.encode16(What[rows], a_dtype), a_dtype)   # one rounding
    got = oracle.decode16(_to_np16(C), a_dtype)
    assert np.array_equal(got, expect)


@pytest.mark.parametrize("M", [1, 8, 16, 17, 32, 64, 128, 256])
def test_gemm_sweep_shape_all_columns(M):
    """The (8192, 28672) sweep layer in the launch configuration the benchmark times (tiled
    layout, AUTO dispatch, one workspace reused as the benchmark does): every output element
    against the oracle."""
    K, N, group, sym, a_dtype = 8192, 28672, 128, 0, 1
    Wb, (oc, os_, oz), tiled = _tiled("outliers", K, N, group, sym, 6)
    Ab, A = _acts(M, K, 6000 + M, a_dtype)
    ws = torch.zeros(native.w4a16_workspace_bytes(M, N, K, group), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED, workspace=ws,
                          dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)
    assert torch.count_nonzero(ws[:65536]).item() == 0


@pytest.mark.parametrize("M", [512, 2048])
def test_gemm_tc_sweep_shape_sampled(M):
    """The sweep layer at the large-M points: 2 and 8 row blocks of 256 per channel tile; a
    sample of columns (the FP64 oracle of all 28672 would take minutes), always including the
    first and last channel tile."""
    K, N, group, sym, a_dtype = 8192, 28672, 128, 0, 1
    Wb, (oc, os_, oz), tiled = _tiled("outliers", K, N, group, sym, 6)
    Ab, A = _acts(M, K, 6000 + M, a_dtype)
    cols = np.unique(np.concatenate([synthetic.column_sample(N, 96, seed=M + 1), np.arange(128),
                                     np.arange(N - 128, N)]))
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)


TC_STREAM = [
    # M, K, N, group, sym, a_dtype     (units = N/128 * ceil(M/BN) * K/128 against one CTA per SM)
    (17, 8192, 256, 128, 0, 1),        # 2 tiles x 64 units < 148: one unit per CTA, tiles cut 64 ways
    (32, 4096, 1280, 64, 1, 0),        # 320 units: tiles cut in two or three
    (64, 2048, 9600, 128, 0, 1),       # 1200 units, about 8 per CTA
    (100, 1024, 2048, 32, 0, 0),
    (128, 3072, 640, 128, 1, 1),       # 5 tiles x 24 units: every tile cut among about 30 CTAs
    (256, 2048, 1024, 64, 0, 1),
    (600, 1024, 512, 128, 0, 1),       # three row blocks of 256 (the last ragged) per channel tile
    (9, 8192, 1024, 128, 0, 0),        # 9 rows forced onto the tensor cores
]


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", TC_STREAM)
def test_gemm_tc_stream_full_output(M, K, N, group, sym, a_dtype):
    """The stream-K tensor-core kernel: full output within the bound, counters left at zero, and
    a second call on the same workspace bit-identical (the cut tiles are summed in CTA order)."""
    kind = "student_t" if sym else "outliers"
    Wb, (oc, os_, oz), tiled = _tiled(kind, K, N, group, sym, 130 + K + N)
    Ab, A = _acts(M, K, 1600 + M, a_dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(native.w4a16_workspace_bytes(M, N, K, group), dtype=torch.uint8, device="cuda")
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                          kernel=native.KERNEL_TC, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)
    assert torch.count_nonzero(ws[:65536]).item() == 0
    C2 = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                           kernel=native.KERNEL_TC, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(C.view(torch.int16), C2.view(torch.int16))


@pytest.mark.parametrize("sym,group,a_dtype", [(s, g, d) for s in (0, 1) for g in (32, 128) for d in (0, 1)])
def test_gemm_tc_format_variants_sampled(sym, group, a_dtype):
    K = N = 8192
    Wb, (oc, os_, oz), tiled = _tiled("student_t", K, N, group, sym, 5)
    for M, kernel in ((16, native.KERNEL_TC), (256, native.KERNEL_TC), (1, native.KERNEL_GEMV),
                      (4, native.KERNEL_GEMV), (16, native.KERNEL_AUTO)):
        Ab, A = _acts(M, K, 7000 + M, a_dtype)
        cols = synthetic.column_sample(N, 64, seed=M + group + 1)
        C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                              kernel=kernel)
        torch.cuda.synchronize()
        _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)


# ----------------------------------------------------------------------------- tiled layout, M <= 16
DECODE_GEMM = [
    # M, K, N, group, sym, a_dtype
    (1, 128, 128, 128, 0, 0),         # one unit: no split
    (1, 512, 256, 128, 0, 0),         # the tiny configuration
    (2, 512, 256, 32, 1, 1),
    (3, 1024, 384, 64, 0, 0),
    (5, 768, 128, 32, 0, 1),
    (8, 2048, 512, 128, 1, 0),
    (13, 1024, 256, 64, 1, 1),
    (16, 1536, 1024, 128, 0, 1),
]


@pytest.mark.parametrize("K,N", LLAMA8B)
def test_gemm_llama8b_decode_tiled_all_columns(K, N):
    """The four Llama-3-8B decode layers at M = 1 in the launch configuration of the benchmark
    (tiled layout, AUTO dispatch): every output column."""
    group, sym, a_dtype = 128, 0, 0
    Wb, (oc, os_, oz), tiled = _tiled("normal", K, N, group, sym, 1000 + N)
    Ab, A = _acts(1, K, 2000 + K, a_dtype)
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", DECODE_GEMM)
def test_gemm_gemv_mma_full_output(M, K, N, group, sym, a_dtype):
    """The decode kernel (persistent stream-K, warp-level MMA) at M = 1..16 on the tiled layout."""
    kind = "student_t" if sym else "normal"
    Wb, (oc, os_, oz), tiled = _tiled(kind, K, N, group, sym, 70 + K + N)
    Ab, A = _acts(M, K, 1300 + M, a_dtype)
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                          kernel=native.KERNEL_GEMV)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


@pytest.mark.parametrize("M", [2, 4])
def test_gemm_gemv_mma_sweep_shape_all_columns(M):
    K, N, group, sym, a_dtype = 8192, 28672, 128, 0, 1
    Wb, (oc, os_, oz), tiled = _tiled("outliers", K, N, group, sym, 6)
    Ab, A = _acts(M, K, 9700 + M, a_dtype)
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                          kernel=native.KERNEL_GEMV)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


# ----------------------------------------------------------------------------- stream-K decode GEMV
STREAM_GEMM = [
    # M, K, N, group, sym, a_dtype      (units = N/128 * K/128 against one CTA per SM)
    (1, 128, 128, 128, 0, 0),           # one unit, one CTA
    (1, 8192, 128, 128, 0, 1),          # one tile cut among 64 CTAs
    (2, 16384, 256, 128, 1, 0),         # two tiles, each cut among about 74 CTAs
    (1, 4096, 1024, 32, 0, 0),          # 256 units: tiles cut in two
    (8, 2048, 1280, 64, 1, 1),
    (9, 1024, 2560, 128, 0, 1),         # two n8 tiles of rows
    (16, 1024, 768, 32, 1, 0),
    (1, 14336, 512, 128, 1, 1),         # long K, symmetric
    (2, 4096, 6144, 128, 0, 0),         # every CTA holds whole tiles and cut ones
]


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", STREAM_GEMM)
def test_gemm_stream_full_output(M, K, N, group, sym, a_dtype):
    kind = "student_t" if sym else "outliers"
    Wb, (oc, os_, oz), tiled = _tiled(kind, K, N, group, sym, 110 + K + N)
    Ab, A = _acts(M, K, 1500 + M, a_dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(native.w4a16_workspace_bytes(M, N, K, group), dtype=torch.uint8, device="cuda")
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                          kernel=native.KERNEL_GEMV, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)
    # the tile counters are back at zero, and a second call on the same workspace is identical
    assert torch.count_nonzero(ws[:65536]).item() == 0
    C2 = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                           kernel=native.KERNEL_GEMV, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(C.view(torch.int16), C2.view(torch.int16))


@pytest.mark.parametrize("a_dtype", [0, 1])
@pytest.mark.parametrize("sym", [0, 1])
@pytest.mark.parametrize("group", [128, 32])
def test_gemm_stream_unit_rows_return_dequantized_rows(a_dtype, sym, group):
    """A = unit rows: each output row is one dequantized weight row rounded once, bit for bit,
    through the post-scaled (group 128) and the pre-scaled (group 32) paths."""
    K, N = 1024, 384
    Wb, (oc, os_, oz), tiled = _tiled("normal", K, N, group, sym, 41)
    rows = [0, 1, 2, 3, 8, 9, 31, 32, 63, 64, 127, 128, 500, 777, 1022, 1023]
    Ab = np.zeros((len(rows), K), dtype=np.uint16)
    one = 0x3C00 if a_dtype == 0 else 0x3F80
    for i, k in enumerate(rows):
        Ab[i, k] = one
    tdt = torch.float16 if a_dtype == 0 else torch.bfloat16
    A = torch.from_numpy(Ab.view(np.int16)).view(tdt).cuda()
    What = oracle.dequant(oc, os_, oz, K, N, group, sym)
    expect = oracle.decode16(oracle.encode16(What[rows], a_dtype), a_dtype)
    for m in (1, 5, 16):
        C = native.w4a16_gemm(A[:m].contiguous(), tiled, None, None, N, group, sym,
                              layout=native.LAYOUT_TILED, kernel=native.KERNEL_GEMV)
        assert np.array_equal(oracle.decode16(_to_np16(C), a_dtype), expect[:m])


@pytest.mark.parametrize("a_dtype", [0, 1])
def test_gemm_stream_zero_weights_give_exact_zero(a_dtype):
    """All-zero weight columns give exactly zero (the bound there is 1e-5 absolute), asymmetric
    (code 0, zero 0) and symmetric (offset-binary code 8, zero 8): u - z is exactly 0."""
    K, N = 2048, 512
    W = torch.zeros((K, N), dtype=torch.float16, device="cuda")
    W[:, 256:] = torch.from_numpy(synthetic.weights_normal(K, 256, seed=3).view(np.int16)).view(
        torch.float16).cuda()
    for sym in (0, 1):
        for group in (128, 64):
            gc, gs, gz = native.w4a16_quantize(W, group, sym)
            tiled = native.w4a16_repack(gc, gs, gz, K, N, group, sym)
            for M in (1, 11):
                Ab, A = _acts(M, K, 7 + M, a_dtype)
                C = native.w4a16_gemm(A, tiled, None, None, N, group, sym,
                                      layout=native.LAYOUT_TILED, kernel=native.KERNEL_GEMV)
                assert torch.count_nonzero(C[:, :256]).item() == 0
                assert torch.count_nonzero(C[:, 256:]).item() > 0


@pytest.mark.parametrize("sym", [0, 1])
def test_gemm_stream_bf16_rows_outside_fp16_range(sym):
    """bf16 activations far outside the fp16 range (rows scaled by 2^40, 2^-60, and a row whose
    largest value is 1e30), full output within the bound: at group 128 the decode kernel scales
    each bf16 row by a power of two before its fp16 arithmetic and scales the sums back, or keeps
    bf16 when a row spans too many binades for an exact conversion."""
    K, N, group = 2048, 512, 128
    Wb, (oc, os_, oz), tiled = _tiled("normal", K, N, group, sym, 61)
    g = torch.Generator().manual_seed(62)
    A32 = torch.randn((4, K), generator=g, dtype=torch.float32)
    A32[0] *= 2.0 ** 40
    A32[1] *= 2.0 ** -60
    A32[2, 77] = 1e30
    A = A32.to(torch.bfloat16)
    # rows 0-1 alone: each row within 31 binades of its maximum, so the fp16 arithmetic on the
    # scaled rows; all four: row 2 spans about 100 binades, so the bf16 arithmetic
    for m in (2, 4):
        Am = A[:m].contiguous()
        Ab = Am.view(torch.int16).numpy().view(np.uint16)
        C = native.w4a16_gemm(Am.cuda(), tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                              kernel=native.KERNEL_GEMV)
        torch.cuda.synchronize()
        assert torch.isfinite(C.float()).all()
        # row 2 is dominated by its 1e30 term (|y| ~ sum|a w|), where the bf16 output rounding
        # alone reaches 2^-8 |y|, above 2e-3 sum|a w|: that rounding is added to the bound
        _check_gemm(C, Ab, 1, oc, os_, oz, N, group, sym, out_rel=2.0 ** -8)


@pytest.mark.parametrize("M", [1, 8, 16])
@pytest.mark.parametrize("K,N", [(8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)])
def test_gemm_llama70b_decode_all_columns(K, N, M):
    """The Llama-3-70B-shaped layers (bf16) at the stack's batch sizes, in the launch
    configuration of the benchmark (tiled layout, AUTO dispatch): every output element."""
    group, sym, a_dtype = 128, 0, 1
    Wb, (oc, os_, oz), tiled = _tiled("normal", K, N, group, sym, 3000 + N)
    Ab, A = _acts(M, K, 4000 + K + M, a_dtype)
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


@pytest.mark.parametrize("M", [6, 9])
def test_gemm_auto_sweep_shape_skinny_all_columns(M):
    """M rows of A too long to sit in the decode kernel's shared memory whole: the AUTO dispatch
    runs the decode kernel over K slices (CTA groups of one launch, FP32 outputs added in slice
    order) or
    the tensor-core kernel, every output within the bound."""
    K, N, group, sym, a_dtype = 8192, 28672, 128, 0, 1
    Wb, (oc, os_, oz), tiled = _tiled("outliers", K, N, group, sym, 6)
    Ab, A = _acts(M, K, 9900 + M, a_dtype)
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED)
    torch.cuda.synchronize()
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", [
    (16, 8192, 9600, 128, 0, 1),    # eight K slices of 1024: 8-unit tiles, 4 or 5 units per CTA
    (8, 8192, 6144, 32, 1, 0),      # two slices (the smaller g32 sym records leave room)
    (12, 16384, 8192, 64, 0, 1),    # eight slices of 2048
])
def test_gemm_stream_k_slices_full_output(M, K, N, group, sym, a_dtype):
    """The decode kernel over K slices, each served by its own CTAs of one launch: full output
    within the bound, stages that run across a tile boundary of the slice (two copies), every
    slice's counters left at zero, and a second call identical."""
    kind = "student_t" if sym else "outliers"
    Wb, (oc, os_, oz), tiled = _tiled(kind, K, N, group, sym, 170 + M)
    Ab, A = _acts(M, K, 1700 + M, a_dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(native.w4a16_workspace_bytes(M, N, K, group), dtype=torch.uint8, device="cuda")
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                          kernel=native.KERNEL_GEMV, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)
    assert torch.count_nonzero(ws[:65536]).item() == 0
    C2 = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED,
                           kernel=native.KERNEL_GEMV, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(C.view(torch.int16), C2.view(torch.int16))


# ----------------------------------------------------------------------------- naive path
@pytest.mark.parametrize("sym,group,a_dtype,K,N", [(0, 128, 0, 1024, 384), (1, 128, 1, 1024, 384),
                                                   (0, 32, 1, 1024, 384), (1, 64, 0, 1024, 384),
                                                   (0, 64, 0, 192, 264), (0, 128, 1, 4096, 6144)])
def test_dequantize_bit_exact(sym, group, a_dtype, K, N):
    """The expanded 16-bit weight equals the oracle's FP64 (q - z) * s rounded once (N = 264: a
    ragged last block of column groups; 4096 x 6144: the 8B qkv shape)."""
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("student_t" if sym else "normal", K, N, group, sym, 77)
    tdt = torch.float16 if a_dtype == 0 else torch.bfloat16
    Wd = native.w4a16_dequantize(gc, gs, gz, K, N, group, sym, dtype=tdt)
    torch.cuda.synchronize()
    expect = oracle.encode16(oracle.dequant(oc, os_, oz, K, N, group, sym), a_dtype)
    assert np.array_equal(_to_np16(Wd), expect)


@pytest.mark.parametrize("M,a_dtype", [(1, 0), (16, 1), (256, 1)])
def test_naive_path_within_bound(M, a_dtype):
    """Dequantize, then the library GEMM (FP32 accumulation): the naive path of the pages, held to
    the same bound as the fused kernels."""
    K, N, group, sym = 2048, 1024, 128, 0
    Wb, (oc, os_, oz), (gc, gs, gz) = _quantized("normal", K, N, group, sym, 78)
    Ab, A = _acts(M, K, 79 + M, a_dtype)
    prev = torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction
    prev_bf = torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
    try:
        Wd = native.w4a16_dequantize(gc, gs, gz, K, N, group, sym, dtype=A.dtype)
        C = torch.matmul(A, Wd)
        torch.cuda.synchronize()
    finally:
        torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = prev
        torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = prev_bf
    _check_gemm(C, Ab, a_dtype, oc, os_, oz, N, group, sym)
