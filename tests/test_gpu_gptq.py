"""GPTQ on the GPU (w4a16_gptq_quantize) against the FP64 oracle ("4.3 Weight-only INT4",
section 2): codes, scales and zeros bit for bit on full small layers and on sampled output
channels of a larger one, the property the method exists for (a lower layer-output error than
RTN) at a realistic size, and the status for a curvature that is not positive definite."""
import numpy as np
import pytest
import torch

import oracle
from oracle import gptq as ogptq
from weight_only_int4_07_b200 import native, synthetic

pytestmark = pytest.mark.gpu


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
    (512, 256, 384, 32, 1, 1),
    (320, 96, 200, 64, 0, 1),     # a ragged last block of 64 channels; S not a multiple of 32
    (384, 264, 512, 128, 1, 0),   # N not a multiple of the 32-channel CTA
    (352, 64, 300, 32, 0, 0),     # K not a multiple of 64: a ragged last block of the factorisation
])
def test_gptq_bit_exact_full(K, N, S, group, sym, x_dtype):
    Wb = synthetic.weights_normal(K, N, 300 + K)
    Xb = synthetic.calibration(S, K, 301 + K, dtype=x_dtype)
    oc, os_, oz = ogptq.gptq(Wb, Xb, x_dtype, group, sym)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gc, gs, gz = native.w4a16_gptq_quantize(_dev16(Wb, synthetic.F16), _dev16(Xb, x_dtype), group, sym,
                                            dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(_np(gc, np.int32), oc)
    assert np.array_equal(_np(gs.view(torch.int16), np.uint16), os_)
    if not sym:
        assert np.array_equal(_np(gz, np.int32), oz)


def test_gptq_bit_exact_sampled_columns():
    """K = 2048, N = 4096: the oracle quantizes 16 of the output channels (every channel is
    independent given H), the GPU all of them; the sampled channels agree bit for bit."""
    K, N, S, group, sym = 2048, 4096, 1024, 128, 0
    Wb = synthetic.weights_outliers(K, N, 310)
    Xb = synthetic.calibration(S, K, 311, dtype=synthetic.F16)
    gc, gs, gz = native.w4a16_gptq_quantize(_dev16(Wb, synthetic.F16), _dev16(Xb, synthetic.F16), group, sym)
    torch.cuda.synchronize()
    cols = np.r_[0:8, 2048:2056]   # two whole zeros words
    oc, os_, oz = ogptq.gptq(np.ascontiguousarray(Wb[:, cols]), Xb, synthetic.F16, group, sym)
    assert np.array_equal(_np(gc, np.int32)[:, cols], oc)
    assert np.array_equal(_np(gs.view(torch.int16), np.uint16)[:, cols], os_)
    gzw = _np(gz, np.int32)
    assert np.array_equal(gzw[:, [0, 256]], oz)


def test_gptq_bit_exact_sampled_columns_deep_factorisation():
    """K = 4096 (64 blocks of 64 channels: six levels of the recursive factorisation), symmetric,
    group 64, bf16 calibration rows; 16 sampled output channels, among them the last CTA's, agree
    with the oracle bit for bit."""
    K, N, S, group, sym = 4096, 4096, 1024, 64, 1
    Wb = synthetic.weights_outliers(K, N, 312)
    Xb = synthetic.calibration(S, K, 313, dtype=synthetic.BF16)
    gc, gs, _ = native.w4a16_gptq_quantize(_dev16(Wb, synthetic.F16), _dev16(Xb, synthetic.BF16), group, sym)
    torch.cuda.synchronize()
    cols = np.r_[8:16, 4080:4088]
    oc, os_, _ = ogptq.gptq(np.ascontiguousarray(Wb[:, cols]), Xb, synthetic.BF16, group, sym)
    assert np.array_equal(_np(gc, np.int32)[:, cols], oc)
    assert np.array_equal(_np(gs.view(torch.int16), np.uint16)[:, cols], os_)


@pytest.mark.parametrize("sym", [0, 1])
def test_gptq_lowers_output_error_at_layer_size(sym):
    """The 8B o-proj shape (4096 x 4096) with 512 calibration rows: GPTQ's layer-output error on
    the calibration inputs is well below RTN's (the objective of section 2.1)."""
    K, N, S, group = 4096, 4096, 512, 128
    Wb = synthetic.weights_normal(K, N, 320)
    Xb = synthetic.calibration(S, K, 321, dtype=synthetic.F16)
    W = _dev16(Wb, synthetic.F16)
    X = _dev16(Xb, synthetic.F16)
    gq = native.w4a16_gptq_quantize(W, X, group, sym)
    rq = native.w4a16_quantize(W, group, sym)
    X64, W64 = X.double(), W.double()

    def err(q):
        What = native.w4a16_dequantize(q[0], q[1], q[2], K, N, group, sym, dtype=torch.float16).double()
        return float(((X64 @ (W64 - What)) ** 2).sum())

    e_gptq, e_rtn = err(gq), err(rq)
    assert e_gptq < 0.8 * e_rtn, (e_gptq, e_rtn)


def test_gptq_reports_a_curvature_that_is_not_positive_definite():
    K, N, group = 128, 64, 128
    W = _dev16(synthetic.weights_normal(K, N, 330), synthetic.F16)
    X = torch.zeros((16, K), dtype=torch.float16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.w4a16_gptq_quantize(W, X, group, 0, damp=0.0, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == native.ENONFINITE
