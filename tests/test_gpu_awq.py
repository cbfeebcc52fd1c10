"""AWQ on the GPU (w4a16_awq_quantize) against the FP64 oracle ("4.3 Weight-only INT4",
section 3): codes, scales, zeros and input factors bit for bit on full small layers and on a
2048 x 2048 layer; at that size also a lower layer-output error than RTN and the encoded layer
running through the fused GEMM (inputs divided by the factors) within the bound."""
import numpy as np
import pytest
import torch

import oracle
from oracle import awq as oawq
from weight_only_int4_07_b200 import native, synthetic

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-5


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from weight_only_int4_07_b200 import build

    build.build()
    native.lib()
    torch.cuda.set_device(0)


def _dev16(bits, dtype):
    tdt = torch.float16 if dtype == synthetic.F16 else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).cuda()


def _np(t, dt):
    return t.cpu().numpy().view(dt)


@pytest.mark.parametrize("K,N,S,group,sym,x_dtype", [
    (256, 128, 256, 128, 0, 0),
    (256, 64, 128, 32, 1, 1),
    (192, 96, 100, 64, 0, 1),
])
def test_awq_bit_exact_full(K, N, S, group, sym, x_dtype):
    Wb = synthetic.weights_normal(K, N, 400 + K)
    Xb = synthetic.calibration(S, K, 401 + K, dtype=x_dtype, outlier_frac=0.02, outlier_mult=20.0)
    oc, os_, oz, osb, ai = oawq.awq(Wb, Xb, x_dtype, group, sym)
    gc, gs, gz, gsi = native.w4a16_awq_quantize(_dev16(Wb, synthetic.F16), _dev16(Xb, x_dtype), group, sym)
    torch.cuda.synchronize()
    assert np.array_equal(_np(gsi.view(torch.int16), np.uint16), osb)
    assert np.array_equal(_np(gs.view(torch.int16), np.uint16), os_)
    assert np.array_equal(_np(gc, np.int32), oc)
    if not sym:
        assert np.array_equal(_np(gz, np.int32), oz)


@pytest.mark.parametrize("sym,x_dtype", [(0, 0), (1, 1)])
def test_awq_bit_exact_2048(sym, x_dtype):
    """A 2048 x 2048 layer with 512 calibration rows (the size of the error test below): the
    factors, codes, scales and zeros bit for bit against the oracle, whose alpha and clip
    searches take every candidate over the whole layer."""
    K, N, S, group = 2048, 2048, 512, 128
    Wb = synthetic.weights_normal(K, N, 420 + sym)
    Xb = synthetic.calibration(S, K, 421 + sym, dtype=x_dtype, outlier_frac=0.02, outlier_mult=20.0)
    oc, os_, oz, osb, ai = oawq.awq(Wb, Xb, x_dtype, group, sym)
    gc, gs, gz, gsi = native.w4a16_awq_quantize(_dev16(Wb, synthetic.F16), _dev16(Xb, x_dtype), group, sym)
    torch.cuda.synchronize()
    assert np.array_equal(_np(gsi.view(torch.int16), np.uint16), osb)
    assert np.array_equal(_np(gs.view(torch.int16), np.uint16), os_)
    assert np.array_equal(_np(gc, np.int32), oc)
    if not sym:
        assert np.array_equal(_np(gz, np.int32), oz)


@pytest.mark.parametrize("sym", [0, 1])
def test_awq_layer_beats_rtn_and_runs_through_the_gemm(sym):
    K, N, S, group = 2048, 2048, 512, 128
    Wb = synthetic.weights_normal(K, N, 410)
    Xb = synthetic.calibration(S, K, 411, dtype=synthetic.F16, outlier_frac=0.02, outlier_mult=20.0)
    W, X = _dev16(Wb, synthetic.F16), _dev16(Xb, synthetic.F16)
    codes, scales, zeros, s_in = native.w4a16_awq_quantize(W, X, group, sym)
    rq = native.w4a16_quantize(W, group, sym)
    X64, W64, s64 = X.double(), W.double(), s_in.double()
    Da = native.w4a16_dequantize(codes, scales, zeros, K, N, group, sym, dtype=torch.float16).double()
    Dr = native.w4a16_dequantize(rq[0], rq[1], rq[2], K, N, group, sym, dtype=torch.float16).double()
    e_awq = float(((X64 @ W64 - (X64 / s64) @ Da) ** 2).sum())
    e_rtn = float(((X64 @ (W64 - Dr)) ** 2).sum())
    assert e_awq < 0.9 * e_rtn, (e_awq, e_rtn)
    # inference: the layer's input divided by s (fp16), through the fused kernel, against the
    # FP64 oracle of the same encoded weight and the same input bits
    M = 4
    A = _dev16(synthetic.activations(M, K, 412), synthetic.F16)
    Ap = (A.float() / s_in.float()).to(torch.float16)
    tiled = native.w4a16_repack(codes, scales, zeros, K, N, group, sym)
    C = native.w4a16_gemm(Ap, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED)
    torch.cuda.synchronize()
    Apb = _np(Ap.view(torch.int16), np.uint16)
    oc, os_ = _np(codes, np.int32), _np(scales.view(torch.int16), np.uint16)
    oz = None if sym else _np(zeros, np.int32)
    cols = synthetic.column_sample(N, 128, seed=413)
    Y, Yabs = oracle.linear(Apb, oracle.F16, oc, os_, oz, N, group, sym, cols=cols)
    y = oracle.decode16(_np(C.view(torch.int16), np.uint16), oracle.F16)[:, cols]
    assert np.all(np.abs(y - Y) <= REL * Yabs + ABS)
