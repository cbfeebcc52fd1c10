"""C-ABI checks that need no GPU: the library loads, exports every symbol the headers declare,
and its host-side logic (argument checks, sizes, dispatch) answers without touching a device.

Every call below either is a pure host function or is rejected by the host-side checks before
any CUDA call is made; no compute call is issued.
"""
import ctypes
import glob
import os
import re

import pytest

from weight_only_int4_07_b200 import native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*W4A16_API\s+[\w\s\*]+?\b(w4a16_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    from weight_only_int4_07_b200 import build

    build.build()
    return native.lib()


def test_headers_declare_the_entry_points():
    names = _declared_symbols()
    for required in ("w4a16_quantize", "w4a16_gemm", "w4a16_repack", "w4a16_repack_bytes",
                     "w4a16_workspace_bytes", "w4a16_select_kernel", "w4a16_status_str",
                     "w4a16_dequantize", "w4a16_gptq_quantize", "w4a16_gptq_workspace_bytes",
                     "w4a16_awq_quantize", "w4a16_awq_workspace_bytes",
                     "w4a16_fp8_quantize_weights", "w4a16_fp8_quantize_acts", "w4a16_fp8_gemm"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared_symbols():
        assert hasattr(L, name), name
        assert getattr(L, name) is not None


def test_library_exports_nothing_else(L):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", native.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert exported == set(_declared_symbols())


def test_status_strings(L):
    assert native.status_str(0) == "W4A16_OK"
    assert native.status_str(-5) == "W4A16_EWORKSPACE"
    assert native.status_str(12345) == "W4A16_UNKNOWN"
    assert native.w4a16_version() >= 100


def test_repack_bytes(L):
    # one record per 128 x 128 unit: 8192 bytes of codes, then G = 128/g groups of 256 bytes of
    # scales and (asymmetric) 64 bytes of zeros
    K, N = 4096, 4096
    units = (K // 128) * (N // 128)
    for g in (32, 64, 128):
        G = 128 // g
        assert native.w4a16_repack_bytes(K, N, g, 0) == units * (8192 + G * 256 + G * 64)
        assert native.w4a16_repack_bytes(K, N, g, 1) == units * (8192 + G * 256)
    assert native.w4a16_repack_bytes(K, 8, 128, 0) == 0          # N not a multiple of 128
    assert native.w4a16_repack_bytes(192, 128, 32, 0) == 0       # K not a multiple of 128
    assert native.w4a16_repack_bytes(4096, 4096, 48, 0) == 0     # group not supported


def test_select_kernel_and_workspace_are_host_only(L):
    for M in (1, 2, 8, 16, 17, 32, 256, 2048):
        k = native.w4a16_select_kernel(M, 4096, 4096, 128)
        assert k in (native.KERNEL_GEMV, native.KERNEL_TC)
        # up to 8 rows the decode GEMV (whole K or K slices); 16 rows at K = 4096 need K slices,
        # where the two-tile decode kernel loses to the tensor-core GEMM; larger M: tensor cores
        assert k == (native.KERNEL_GEMV if M <= 8 else native.KERNEL_TC)
        assert native.w4a16_workspace_bytes(M, 4096, 4096, 128) >= 0
    # 12 rows at K = 1024 fit in shared memory whole: the decode GEMV
    assert native.w4a16_select_kernel(12, 4096, 1024, 128) == native.KERNEL_GEMV
    assert native.w4a16_workspace_bytes(0, 4096, 4096, 128) == 0
    assert native.w4a16_workspace_bytes(1, 4096, 4000, 128) == 0


# Fake device addresses: the checks below reject the call before any CUDA call, so the
# addresses are never dereferenced.
A16 = ctypes.c_void_p(1 << 20)
B16 = ctypes.c_void_p(2 << 20)
C16 = ctypes.c_void_p(3 << 20)
D16 = ctypes.c_void_p(4 << 20)
MIS = ctypes.c_void_p((5 << 20) + 8)


def _gemm(L, A=A16, dt=0, M=1, K=256, wq=B16, layout=0, scales=C16, zeros=D16, N=256, g=128,
          sym=0, C=A16, ws=None, wsb=1 << 30, kernel=0):
    return L.w4a16_gemm(A, dt, M, K, wq, layout, scales, zeros, N, g, sym, C, ws, wsb, kernel, None,
                        None)


def test_gemm_rejects_bad_arguments(L):
    assert _gemm(L, K=100) == native.EINVAL                    # K % 8
    assert _gemm(L, N=100) == native.EINVAL                    # N % 8
    assert _gemm(L, K=264, g=128) == native.EINVAL             # K % group
    assert _gemm(L, g=16) == native.EUNSUPPORTED               # group
    assert _gemm(L, M=0) == native.EINVAL
    assert _gemm(L, dt=2) == native.EINVAL
    assert _gemm(L, layout=3) == native.EINVAL
    assert _gemm(L, sym=2) == native.EINVAL
    assert _gemm(L, kernel=7) == native.EINVAL
    assert _gemm(L, A=None) == native.EINVAL
    assert _gemm(L, wq=None) == native.EINVAL
    assert _gemm(L, C=None) == native.EINVAL
    assert _gemm(L, scales=None) == native.EINVAL
    assert _gemm(L, zeros=None, sym=0) == native.EINVAL        # asymmetric needs zeros
    assert _gemm(L, zeros=D16, sym=1) == native.EINVAL         # symmetric takes none
    assert _gemm(L, A=MIS) == native.EALIGN
    assert _gemm(L, C=MIS) == native.EALIGN
    assert _gemm(L, scales=MIS) == native.EALIGN
    assert _gemm(L, layout=1, N=8) == native.EUNSUPPORTED      # tiled needs N % 128
    need = native.w4a16_workspace_bytes(1, 256, 256, 128)
    if need > 0:
        assert _gemm(L, ws=D16, wsb=need - 1) == native.EWORKSPACE
        assert _gemm(L, ws=None, wsb=need) == native.EWORKSPACE
        assert _gemm(L, ws=MIS, wsb=need) == native.EALIGN


def test_quantize_rejects_bad_arguments(L):
    q = L.w4a16_quantize
    assert q(A16, 256, 256, 128, 0, B16, C16, None, None, None) == native.EINVAL   # asym, no zeros
    assert q(A16, 256, 256, 128, 1, B16, C16, D16, None, None) == native.EINVAL    # sym, zeros
    assert q(A16, 250, 256, 128, 0, B16, C16, D16, None, None) == native.EINVAL
    assert q(A16, 256, 256, 100, 0, B16, C16, D16, None, None) == native.EUNSUPPORTED
    assert q(MIS, 256, 256, 128, 0, B16, C16, D16, None, None) == native.EALIGN
    assert q(None, 256, 256, 128, 0, B16, C16, D16, None, None) == native.EINVAL
    assert q(A16, 256, 256, 128, 3, B16, C16, D16, None, None) == native.EINVAL


def test_repack_rejects_bad_arguments(L):
    r = L.w4a16_repack
    assert r(A16, B16, C16, 256, 8, 128, 0, D16, None) == native.EUNSUPPORTED
    assert r(A16, B16, None, 256, 128, 128, 0, D16, None) == native.EINVAL
    assert r(A16, B16, C16, 256, 128, 128, 1, D16, None) == native.EINVAL
    assert r(A16, B16, C16, 256, 128, 128, 0, MIS, None) == native.EALIGN


def test_dequantize_rejects_bad_arguments_before_any_launch(L):
    P = ctypes.c_void_p
    ok = dict(codes=P(1 << 20), scales=P(2 << 20), zeros=P(3 << 20), K=256, N=128, group=128, sym=0,
              dt=native.F16, W=P(4 << 20))

    def call(**kw):
        a = dict(ok, **kw)
        return L.w4a16_dequantize(a["codes"], a["scales"], a["zeros"], a["K"], a["N"], a["group"],
                                  a["sym"], a["dt"], a["W"], None)
    assert call(group=48) == native.EUNSUPPORTED
    assert call(K=100) == native.EINVAL
    assert call(dt=7) == native.EINVAL
    assert call(W=None) == native.EINVAL
    assert call(sym=1) == native.EINVAL                   # zeros given for a symmetric weight
    assert call(zeros=None) == native.EINVAL              # asymmetric without zeros
    assert call(W=P((4 << 20) + 8)) == native.EALIGN


def test_gptq_rejects_bad_arguments_before_any_launch(L):
    P = ctypes.c_void_p
    K, N = 256, 128
    need = L.w4a16_gptq_workspace_bytes(K, N)
    assert need == 16 * K * K + 8 * K * N + 1024 * N + 256
    assert L.w4a16_gptq_workspace_bytes(0, N) == 0
    ok = dict(W=P(1 << 20), X=P(2 << 20), xdt=native.F16, S=64, K=K, N=N, group=128, sym=0, damp=0.01,
              codes=P(3 << 20), scales=P(4 << 20), zeros=P(5 << 20), ws=P(6 << 20), wsb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return L.w4a16_gptq_quantize(a["W"], a["X"], a["xdt"], a["S"], a["K"], a["N"], a["group"], a["sym"],
                                     ctypes.c_double(a["damp"]), a["codes"], a["scales"], a["zeros"], a["ws"],
                                     a["wsb"], None, None)
    assert call(group=48) == native.EUNSUPPORTED
    assert call(S=0) == native.EINVAL
    assert call(xdt=5) == native.EINVAL
    assert call(damp=-1.0) == native.EINVAL
    assert call(damp=float("nan")) == native.EINVAL
    assert call(zeros=None) == native.EINVAL
    assert call(sym=1) == native.EINVAL
    assert call(ws=None) == native.EINVAL
    assert call(wsb=need - 1) == native.EWORKSPACE
    assert call(X=P((2 << 20) + 2)) == native.EALIGN
    big = 65536   # the factorisations are blocked, so only the workspace grows with K
    assert L.w4a16_gptq_workspace_bytes(big, N) == 16 * big * big + 8 * big * N + 1024 * N + 256


def test_awq_rejects_bad_arguments_before_any_launch(L):
    P = ctypes.c_void_p
    K, N, S = 256, 128, 100
    need = L.w4a16_awq_workspace_bytes(K, N, S)
    parts = 2 * 2   # ceil(100 / 64) * ceil(128 / 64), already even
    assert need == 8 * (K * K + K * N + 2 * K + 64 + parts) + 256
    assert L.w4a16_awq_workspace_bytes(K, N, 0) == 0
    ok = dict(W=P(1 << 20), X=P(2 << 20), xdt=native.F16, S=S, K=K, N=N, group=128, sym=0,
              codes=P(3 << 20), scales=P(4 << 20), zeros=P(5 << 20), s_in=P(6 << 20), ws=P(7 << 20), wsb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return L.w4a16_awq_quantize(a["W"], a["X"], a["xdt"], a["S"], a["K"], a["N"], a["group"], a["sym"],
                                    a["codes"], a["scales"], a["zeros"], a["s_in"], a["ws"], a["wsb"], None, None)
    assert call(group=96) == native.EUNSUPPORTED
    assert call(S=0) == native.EINVAL
    assert call(xdt=3) == native.EINVAL
    assert call(s_in=None) == native.EINVAL
    assert call(zeros=None) == native.EINVAL
    assert call(wsb=need - 8) == native.EWORKSPACE
    assert call(s_in=P((6 << 20) + 4)) == native.EALIGN


def test_fp8_rejects_bad_arguments_before_any_launch(L):
    P = ctypes.c_void_p
    a, b, c = P(1 << 20), P(2 << 20), P(3 << 20)
    assert L.w4a16_fp8_quantize_weights(a, 200, 128, b, c, None) == native.EUNSUPPORTED
    assert L.w4a16_fp8_quantize_weights(a, 256, 128, None, c, None) == native.EINVAL
    assert L.w4a16_fp8_quantize_weights(P((1 << 20) + 2), 256, 128, b, c, None) == native.EALIGN
    assert L.w4a16_fp8_quantize_acts(a, 0, 0, 256, b, c, None) == native.EINVAL
    assert L.w4a16_fp8_quantize_acts(a, 4, 1, 256, b, c, None) == native.EINVAL
    assert L.w4a16_fp8_quantize_acts(a, 0, 1, 100, b, c, None) == native.EUNSUPPORTED
    d = P(4 << 20)
    assert L.w4a16_fp8_gemm(a, b, 1, 256, c, d, 100, P(5 << 20), 0, None, None) == native.EUNSUPPORTED
    assert L.w4a16_fp8_gemm(a, b, 0, 256, c, d, 128, P(5 << 20), 0, None, None) == native.EINVAL
    assert L.w4a16_fp8_gemm(a, b, 1, 256, c, d, 128, P(5 << 20), 2, None, None) == native.EINVAL
    assert L.w4a16_fp8_gemm(a, b, 1, 256, c, P((4 << 20) + 4), 128, P(5 << 20), 0, None, None) == native.EALIGN


def test_workspace_covers_the_k_slices_of_the_decode_kernel():
    """16 rows of A for K = 8192 do not fit in the decode kernel's shared memory whole: the
    workspace then also holds the FP32 outputs of its K slices (at least two of M x N x 4 B)."""
    M, N, K = 16, 28672, 8192
    assert native.w4a16_workspace_bytes(M, N, K, 128) >= 65536 + 2 * M * N * 4
    # one row fits whole: counters plus the cut-tile sums only
    assert native.w4a16_workspace_bytes(1, N, K, 128) < 65536 + M * N * 4
    # 8 rows: two slices of 4096, served by the two CTA groups of one launch
    assert native.w4a16_workspace_bytes(8, N, K, 128) >= 65536 + 2 * 8 * N * 4


@pytest.mark.parametrize("K,N", [(8192, 28672), (8192, 10240), (8192, 57344), (28672, 8192), (4096, 28672)])
def test_dispatch_on_the_benchmarked_layers(K, N):
    """The sweep layer and the 70B and 8B layers (bf16, g128): the decode GEMV up to 8 rows, whole
    K or sliced; from 9 rows the tensor-core GEMM, since 9-16 rows of these K need K slices, where
    the decode kernel's two 8-row MMA tiles make it slower than the tensor-core GEMM."""
    for M in range(1, 9):
        assert native.w4a16_select_kernel(M, N, K, 128) == native.KERNEL_GEMV
    for M in (9, 12, 16, 17, 64, 256):
        assert native.w4a16_select_kernel(M, N, K, 128) == native.KERNEL_TC


def test_wait_limit_setter_is_host_only(L):
    """w4a16_set_wait_limit_ns returns the previous limit; 0 restores the 2 s default."""
    prev = native.w4a16_set_wait_limit_ns(12345)
    assert native.w4a16_set_wait_limit_ns(0) == 12345
    assert native.w4a16_set_wait_limit_ns(prev) == 2_000_000_000


def _in_child(env, code):
    import subprocess
    import sys

    e = dict(os.environ)
    e.update(env)
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=e, capture_output=True, text=True,
                          timeout=300)


def test_force_kernel_environment_overrides_the_dispatch(L):
    """W4A16_FORCE_KERNEL=gemv|tc (read once per process) replaces the M-based choice."""
    code = ("from weight_only_int4_07_b200 import native; "
            "print(native.w4a16_select_kernel(1, 4096, 4096, 128), native.w4a16_select_kernel(512, 4096, 4096, 128))")
    for value, expect in (("tc", "2 2"), ("gemv", "1 1"), ("", "1 2")):
        r = _in_child({"W4A16_FORCE_KERNEL": value}, code)
        assert r.returncode == 0, r.stderr
        assert r.stdout.split() == expect.split(), value


def test_log_environment_prints_the_dispatch(L):
    """W4A16_LOG=1 prints one line per w4a16_gemm call with the shape and the kernel chosen,
    before any launch (here the call then fails on the host without a device: no compute)."""
    code = ("import ctypes; from weight_only_int4_07_b200 import native; L = native.lib(); "
            "p = ctypes.c_void_p(1 << 20); "
            "L.w4a16_gemm(p, 0, 1, 256, p, 1, None, None, 256, 128, 0, p, p, 1 << 30, 0, None, None)")
    r = _in_child({"W4A16_LOG": "1", "CUDA_VISIBLE_DEVICES": ""}, code)
    assert r.returncode == 0, r.stderr
    assert "[w4a16] gemm M=1 N=256 K=256 g=128 sym=0 layout=1 -> gemv" in r.stderr
    r = _in_child({"W4A16_LOG": "0", "CUDA_VISIBLE_DEVICES": ""}, code)
    assert "[w4a16]" not in r.stderr
