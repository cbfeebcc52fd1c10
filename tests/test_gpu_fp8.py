"""The W8A8 FP8 comparison path on the GPU against the FP64 oracle: E4M3 codes and scales bit for
bit (weights and activations), and the kind::f8f6f4 GEMM within the bound on full small outputs
and sampled columns of the sweep layer."""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as ofp8
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


@pytest.mark.parametrize("K,N,kind", [(256, 128, "normal"), (1024, 384, "outliers"), (4096, 6144, "student_t")])
def test_fp8_weight_codes_bit_exact(K, N, kind):
    gen = {"normal": synthetic.weights_normal, "outliers": synthetic.weights_outliers,
           "student_t": synthetic.weights_student_t}[kind]
    Wb = gen(K, N, 500 + K)
    oq, os_ = ofp8.quantize_weights(Wb)
    gq, gs = native.w4a16_fp8_quantize_weights(_dev16(Wb, synthetic.F16))
    torch.cuda.synchronize()
    assert np.array_equal(gq.cpu().numpy(), oq)
    assert np.array_equal(gs.cpu().numpy(), os_)


@pytest.mark.parametrize("M,K,a_dtype", [(1, 256, 0), (37, 1024, 1), (256, 8192, 1)])
def test_fp8_activation_codes_bit_exact(M, K, a_dtype):
    Ab = synthetic.activations(M, K, 510 + M, dtype=a_dtype)
    oq, os_ = ofp8.quantize_acts(Ab, a_dtype)
    gq, gs = native.w4a16_fp8_quantize_acts(_dev16(Ab, a_dtype))
    torch.cuda.synchronize()
    assert np.array_equal(gq.cpu().numpy(), oq)
    assert np.array_equal(gs.cpu().numpy(), os_)


def _check(C, qa, sa, qw, sw, cols=None, dtype=0):
    Y, Yabs = ofp8.linear(qa, sa, qw if cols is None else qw[cols], sw if cols is None else sw[cols])
    y = oracle.decode16(C.view(torch.int16).cpu().numpy().view(np.uint16), dtype)
    if cols is not None:
        y = y[:, cols]
    bad = np.abs(y - Y) > REL * Yabs + ABS
    assert not bad.any(), f"{bad.sum()} outputs outside the bound"


@pytest.mark.parametrize("M,K,N,a_dtype", [(1, 1024, 384, 0), (17, 1024, 256, 1), (100, 512, 640, 0),
                                          (256, 2048, 384, 1), (300, 1024, 256, 0)])
def test_fp8_gemm_full_output(M, K, N, a_dtype):
    Wb = synthetic.weights_normal(K, N, 520 + N)
    Ab = synthetic.activations(M, K, 521 + M, dtype=a_dtype)
    qw, sw = ofp8.quantize_weights(Wb)
    qa, sa = ofp8.quantize_acts(Ab, a_dtype)
    gq, gs = native.w4a16_fp8_quantize_weights(_dev16(Wb, synthetic.F16))
    aq, asc = native.w4a16_fp8_quantize_acts(_dev16(Ab, a_dtype))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tdt = torch.float16 if a_dtype == 0 else torch.bfloat16
    C = native.w4a16_fp8_gemm(aq, asc, gq, gs, dtype=tdt, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check(C, qa, sa, qw, sw, dtype=a_dtype)


def test_fp8_gemm_sweep_layer_sampled():
    K, N, M = 8192, 28672, 256
    Wb = synthetic.weights_outliers(K, N, 530)
    Ab = synthetic.activations(M, K, 531, dtype=synthetic.BF16)
    gq, gs = native.w4a16_fp8_quantize_weights(_dev16(Wb, synthetic.F16))
    aq, asc = native.w4a16_fp8_quantize_acts(_dev16(Ab, synthetic.BF16))
    C = native.w4a16_fp8_gemm(aq, asc, gq, gs, dtype=torch.bfloat16)
    torch.cuda.synchronize()
    cols = synthetic.column_sample(N, 64, seed=532)
    _check(C, aq.cpu().numpy(), asc.cpu().numpy(), gq.cpu().numpy(), gs.cpu().numpy(), cols=cols, dtype=1)
