"""w4a16_gemm_noalloc, the entry point for callers that cannot allocate device memory.

Some callers of this layer cannot hand w4a16_gemm a workspace: a plugin inside a host
application that owns every device allocation, or a latency-critical loop that must never call
cudaMalloc because it can block and synchronise the device. For them the library keeps the
split-K partial sums in one static device array. This test calls that entry point through the
C ABI twice in a row -- the second call finds the first call's partial sums still in the shared
array -- and checks both outputs against the FP64 oracle's layer output within the acceptance
bound, and against w4a16_gemm's output within the same bound. One case has more than 16 rows,
so the entry point runs its 16-row chunks one after another on the shared array. It also checks
that a call needing more than the static array holds is refused. It lives in a file of its own,
collected last, and passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_07_b200 import native, synthetic

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-5


def _abi():
    from weight_only_int4_07_b200 import build

    build.build()
    L = native.lib()
    P, I = ctypes.c_void_p, ctypes.c_int
    L.w4a16_gemm_noalloc.argtypes = [P, I, I, I, P, P, P, I, I, I, P, P]
    L.w4a16_gemm_noalloc.restype = I
    return L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("M,K,N,group,sym,a_dtype", [(1, 4096, 6144, 128, 0, 0), (5, 2048, 1032, 32, 1, 1),
                                                     (20, 2048, 1032, 128, 0, 1)])
def test_noalloc_matches_gemm_on_two_calls(M, K, N, group, sym, a_dtype):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    L = _abi()
    Wb = synthetic.weights_normal(K, N, seed=900 + K)
    W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).cuda()
    codes, scales, zeros = native.w4a16_quantize(W, group, sym)
    st, oc, os_, oz = oracle.quantize(Wb, group, sym)
    assert np.array_equal(codes.cpu().numpy(), oc)   # the oracle's output below is for these weights
    tdt = torch.float16 if a_dtype == 0 else torch.bfloat16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        Ab = synthetic.activations(M, K, seed=910 + call, dtype=a_dtype)
        A = torch.from_numpy(Ab.view(np.int16)).view(tdt).cuda()
        ref = native.w4a16_gemm(A, codes, scales, zeros, N, group, sym, kernel=native.KERNEL_GEMV)
        C = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
        rc = L.w4a16_gemm_noalloc(_p(A), a_dtype, M, K, _p(codes), _p(scales), _p(zeros), N, group,
                                  sym, _p(C), stream)
        assert rc == native.OK, native.status_str(rc)
        torch.cuda.synchronize()
        Y, Yabs = oracle.linear(Ab, a_dtype, oc, os_, oz, N, group, sym)
        y = C.double().cpu().numpy()
        y_ref = ref.double().cpu().numpy()
        assert np.all(np.abs(y - Y) <= REL * Yabs + ABS), f"call {call}: outside the bound of the oracle"
        assert np.all(np.abs(y - y_ref) <= REL * Yabs + ABS), f"call {call}: differs from w4a16_gemm"


def test_noalloc_refuses_calls_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = _abi()
    # M = 16, N = 65536: the split-K partial sums need far more than the static scratch holds;
    # the call is refused on the host before any launch, so these addresses are never used
    A = ctypes.c_void_p(1 << 20)
    rc = L.w4a16_gemm_noalloc(A, 0, 16, 4096, A, A, A, 65536, 128, 0, A, None)
    assert rc == native.EWORKSPACE
