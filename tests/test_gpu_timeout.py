"""The bounded device waits run out on purpose, and the device stays usable.

Every wait inside the kernels (a pipeline barrier, or a tile counter that another CTA of the
same launch sets) gives up after a time limit, and each suspension of a waiting thread is at most
that limit. Two ways to make the waits run out, neither of which faults or traps anything:
  * w4a16_set_wait_limit_ns(1): the first pipeline wait whose copy has not landed within 1 ns
    gives up, in the middle of the weight stream, with copies and MMAs in flight;
  * tile counters that start far below zero instead of at zero (a flag nothing will set): the
    CTA that sums a cut tile waits for a count it never sees (limit 1 ms).
Either way the kernel records W4A16_ETIMEOUT in dev_status, stops issuing, lets its copies and
MMAs in flight complete, frees its tensor memory and returns. The test then restores the default
limit, zeroes the workspace again (the header asks for that after a timeout) and checks that the
next call on the same device is exact against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
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
    yield
    native.w4a16_set_wait_limit_ns(0)


def _layer(K, N, group, sym, seed):
    Wb = synthetic.weights_normal(K, N, seed)
    st, oc, os_, oz = oracle.quantize(Wb, group, sym)
    W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).cuda()
    gc, gs, gz = native.w4a16_quantize(W, group, sym)
    return (oc, os_, oz), native.w4a16_repack(gc, gs, gz, K, N, group, sym)


# The 1 ns limit runs out for certain only where a wait comes before any copy can have landed:
# the tensor-core kernel's dequant warps wait for their first weight records at once. The decode
# kernel first stages A, by which time its first weight stages may already be there, so it is
# driven to a timeout through its tile counters instead.
@pytest.mark.parametrize("M,kernel,how", [(1, native.KERNEL_GEMV, "counters"), (8, native.KERNEL_GEMV, "counters"),
                                          (64, native.KERNEL_TC, "limit"), (64, native.KERNEL_TC, "counters"),
                                          (256, native.KERNEL_TC, "limit"), (256, native.KERNEL_TC, "counters")])
def test_waits_run_out_then_the_device_recovers(M, kernel, how):
    K, N, group, sym, a_dtype = 8192, 28672, 128, 0, 1
    (oc, os_, oz), tiled = _layer(K, N, group, sym, 21)
    Ab = synthetic.activations(M, K, 22 + M, dtype=a_dtype)
    A = torch.from_numpy(Ab.view(np.int16)).view(torch.bfloat16).cuda()
    ws = torch.zeros(native.w4a16_workspace_bytes(M, N, K, group), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if how == "counters":
        ws[:65536] = 0x80                   # every tile counter reads as -2139062144
    torch.cuda.synchronize()
    prev = native.w4a16_set_wait_limit_ns(1 if how == "limit" else 1_000_000)
    try:
        native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED, kernel=kernel,
                          workspace=ws, dev_status=status)
        torch.cuda.synchronize()            # the launch returned: no wait was left without a limit
    finally:
        native.w4a16_set_wait_limit_ns(prev)
    assert int(status.item()) == native.ETIMEOUT
    # the device still works: the same call with the default limit, on a zeroed workspace
    ws.zero_()
    status.zero_()
    C = native.w4a16_gemm(A, tiled, None, None, N, group, sym, layout=native.LAYOUT_TILED, kernel=kernel,
                          workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    cols = synthetic.column_sample(N, 256, seed=M)
    Y, Yabs = oracle.linear(Ab, a_dtype, oc, os_, oz, N, group, sym, cols=cols)
    y = oracle.decode16(C.view(torch.int16).cpu().numpy().view(np.uint16), a_dtype)[:, cols]
    assert np.all(np.abs(y - Y) <= REL * Yabs + ABS)
    assert torch.count_nonzero(ws[:65536]).item() == 0


