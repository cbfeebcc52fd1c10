"""Thin Python binding of the C ABI in include/w4a16.h (ctypes; argument marshalling only).

Each function has the name of the C entry point it calls. Tensors are torch CUDA tensors: the
binding passes their data pointers and the current CUDA stream and checks the returned status.
Every step of the layer runs in the CUDA library; there is no fallback of any kind: if
libw4a16.so is missing the first call raises.
"""
import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libw4a16.so")

OK = 0
EINVAL = -1
EALIGN = -2
EUNSUPPORTED = -3
ENONFINITE = -4
EWORKSPACE = -5
ECUDA = -6
ETIMEOUT = -7

F16 = 0
BF16 = 1
LAYOUT_PLAIN = 0
LAYOUT_TILED = 1
KERNEL_AUTO = 0
KERNEL_GEMV = 1
KERNEL_TC = 2

_DTYPES = {torch.float16: F16, torch.bfloat16: BF16}
_TORCH_DTYPES = {F16: torch.float16, BF16: torch.bfloat16}

_lib = None


class W4A16Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")


def lib():
    """The loaded ctypes library, with the argument types of include/w4a16.h."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"the W4A16 CUDA library is not built ({LIB_PATH} is missing); "
                           "run `python -m weight_only_int4_07_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.w4a16_quantize.argtypes = [P, I, I, I, I, P, P, P, P, P]
    L.w4a16_quantize.restype = I
    L.w4a16_dequantize.argtypes = [P, P, P, I, I, I, I, I, P, P]
    L.w4a16_dequantize.restype = I
    L.w4a16_gptq_workspace_bytes.argtypes = [I, I]
    L.w4a16_gptq_workspace_bytes.restype = S
    L.w4a16_gptq_quantize.argtypes = [P, P, I, I, I, I, I, I, ctypes.c_double, P, P, P, P, S, P, P]
    L.w4a16_gptq_quantize.restype = I
    L.w4a16_awq_workspace_bytes.argtypes = [I, I, I]
    L.w4a16_awq_workspace_bytes.restype = S
    L.w4a16_awq_quantize.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P, P, S, P, P]
    L.w4a16_awq_quantize.restype = I
    L.w4a16_fp8_quantize_weights.argtypes = [P, I, I, P, P, P]
    L.w4a16_fp8_quantize_weights.restype = I
    L.w4a16_fp8_quantize_acts.argtypes = [P, I, I, I, P, P, P]
    L.w4a16_fp8_quantize_acts.restype = I
    L.w4a16_fp8_gemm.argtypes = [P, P, I, I, P, P, I, P, I, P, P]
    L.w4a16_fp8_gemm.restype = I
    L.w4a16_repack_bytes.argtypes = [I, I, I, I]
    L.w4a16_repack_bytes.restype = S
    L.w4a16_repack.argtypes = [P, P, P, I, I, I, I, P, P]
    L.w4a16_repack.restype = I
    L.w4a16_workspace_bytes.argtypes = [I, I, I, I]
    L.w4a16_workspace_bytes.restype = S
    L.w4a16_select_kernel.argtypes = [I, I, I, I]
    L.w4a16_select_kernel.restype = I
    L.w4a16_gemm.argtypes = [P, I, I, I, P, I, P, P, I, I, I, P, P, S, I, P, P]
    L.w4a16_gemm.restype = I
    L.w4a16_status_str.argtypes = [I]
    L.w4a16_status_str.restype = ctypes.c_char_p
    L.w4a16_version.argtypes = []
    L.w4a16_version.restype = I
    L.w4a16_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.w4a16_set_wait_limit_ns.restype = ctypes.c_uint64
    _lib = L
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(fn, status):
    if status != OK:
        raise W4A16Error(fn, status)


def status_str(status: int) -> str:
    return lib().w4a16_status_str(int(status)).decode()


w4a16_status_str = status_str


def w4a16_version() -> int:
    return int(lib().w4a16_version())


def w4a16_set_wait_limit_ns(ns: int) -> int:
    """Limit of every bounded device wait for later launches (0 = the 2 s default); returns the
    previous limit."""
    return int(lib().w4a16_set_wait_limit_ns(int(ns)))


def w4a16_quantize(W, group, sym, codes=None, scales=None, zeros=None, dev_status=None):
    """RTN group quantization of fp16 W [K, N] on the GPU -> (codes, scales, zeros)."""
    K, N = W.shape
    dev = W.device
    if codes is None:
        codes = torch.empty((K // 8, N), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty((K // group, N), dtype=torch.float16, device=dev)
    if zeros is None and not sym:
        zeros = torch.empty((K // group, N // 8), dtype=torch.int32, device=dev)
    st = lib().w4a16_quantize(_ptr(W), K, N, group, int(sym), _ptr(codes), _ptr(scales),
                              _ptr(zeros), _ptr(dev_status), _stream())
    _check("w4a16_quantize", st)
    return codes, scales, (None if sym else zeros)


def w4a16_gptq_workspace_bytes(K, N) -> int:
    return int(lib().w4a16_gptq_workspace_bytes(K, N))


def w4a16_gptq_quantize(W, X, group, sym, damp=0.01, codes=None, scales=None, zeros=None,
                        workspace=None, dev_status=None):
    """GPTQ of fp16 W [K, N] with 16-bit calibration inputs X [S, K] on the GPU -> (codes,
    scales, zeros) in the plain packed format."""
    K, N = W.shape
    S = X.shape[0]
    dev = W.device
    if codes is None:
        codes = torch.empty((K // 8, N), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty((K // group, N), dtype=torch.float16, device=dev)
    if zeros is None and not sym:
        zeros = torch.empty((K // group, N // 8), dtype=torch.int32, device=dev)
    nbytes = w4a16_gptq_workspace_bytes(K, N)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    st = lib().w4a16_gptq_quantize(_ptr(W), _ptr(X), _DTYPES[X.dtype], S, K, N, group, int(sym),
                                   float(damp), _ptr(codes), _ptr(scales), _ptr(zeros),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _ptr(dev_status), _stream())
    _check("w4a16_gptq_quantize", st)
    return codes, scales, (None if sym else zeros)


def w4a16_awq_workspace_bytes(K, N, S) -> int:
    return int(lib().w4a16_awq_workspace_bytes(K, N, S))


def w4a16_awq_quantize(W, X, group, sym, codes=None, scales=None, zeros=None, s_in=None,
                       workspace=None, dev_status=None):
    """AWQ of fp16 W [K, N] with 16-bit calibration inputs X [S, K] on the GPU -> (codes, scales,
    zeros, s_in): the packed S W and the fp16 factors that divide the layer's input."""
    K, N = W.shape
    S = X.shape[0]
    dev = W.device
    if codes is None:
        codes = torch.empty((K // 8, N), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty((K // group, N), dtype=torch.float16, device=dev)
    if zeros is None and not sym:
        zeros = torch.empty((K // group, N // 8), dtype=torch.int32, device=dev)
    if s_in is None:
        s_in = torch.empty(K, dtype=torch.float16, device=dev)
    nbytes = w4a16_awq_workspace_bytes(K, N, S)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    st = lib().w4a16_awq_quantize(_ptr(W), _ptr(X), _DTYPES[X.dtype], S, K, N, group, int(sym),
                                  _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(s_in), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                  _stream())
    _check("w4a16_awq_quantize", st)
    return codes, scales, (None if sym else zeros), s_in


def w4a16_fp8_quantize_weights(W):
    """fp16 W [K, N] -> (Wq uint8 [N, K] E4M3 codes, w_scales float32 [N]) on the GPU."""
    K, N = W.shape
    Wq = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    sw = torch.empty(N, dtype=torch.float32, device=W.device)
    _check("w4a16_fp8_quantize_weights",
           lib().w4a16_fp8_quantize_weights(_ptr(W), K, N, _ptr(Wq), _ptr(sw), _stream()))
    return Wq, sw


def w4a16_fp8_quantize_acts(A, Aq=None, sa=None):
    """16-bit A [M, K] -> (Aq uint8 [M, K] E4M3 codes, a_scales float32 [M]) on the GPU."""
    M, K = A.shape
    if Aq is None:
        Aq = torch.empty((M, K), dtype=torch.uint8, device=A.device)
    if sa is None:
        sa = torch.empty(M, dtype=torch.float32, device=A.device)
    _check("w4a16_fp8_quantize_acts",
           lib().w4a16_fp8_quantize_acts(_ptr(A), _DTYPES[A.dtype], M, K, _ptr(Aq), _ptr(sa), _stream()))
    return Aq, sa


def w4a16_fp8_gemm(Aq, sa, Wq, sw, dtype=None, C=None, dev_status=None):
    """C[M, N] = (Aq . Wq^T) * sa[m] * sw[n], FP32 accumulation, C in `dtype` (fp16 default)."""
    M, K = Aq.shape
    N = Wq.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.float16 if dtype is None else dtype, device=Aq.device)
    _check("w4a16_fp8_gemm", lib().w4a16_fp8_gemm(_ptr(Aq), _ptr(sa), M, K, _ptr(Wq), _ptr(sw), N, _ptr(C),
                                                  _DTYPES[C.dtype], _ptr(dev_status), _stream()))
    return C


def w4a16_dequantize(codes, scales, zeros, K, N, group, sym, dtype=None, out=None):
    """The packed weight as a 16-bit [K, N] matrix, (q - z) * s rounded once (the naive path)."""
    dtype = torch.float16 if dtype is None else dtype
    if out is None:
        out = torch.empty((K, N), dtype=dtype, device=codes.device)
    st = lib().w4a16_dequantize(_ptr(codes), _ptr(scales), _ptr(zeros), K, N, group, int(sym),
                                _DTYPES[out.dtype], _ptr(out), _stream())
    _check("w4a16_dequantize", st)
    return out


def w4a16_repack_bytes(K, N, group, sym) -> int:
    return int(lib().w4a16_repack_bytes(K, N, group, int(sym)))


def w4a16_repack(codes, scales, zeros, K, N, group, sym, out=None):
    """Plain packed weight -> one tiled uint8 buffer (see the header for the layout)."""
    nbytes = w4a16_repack_bytes(K, N, group, sym)
    if nbytes == 0:
        _check("w4a16_repack", EUNSUPPORTED)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=codes.device)
    st = lib().w4a16_repack(_ptr(codes), _ptr(scales), _ptr(zeros), K, N, group, int(sym),
                            _ptr(out), _stream())
    _check("w4a16_repack", st)
    return out


def w4a16_workspace_bytes(M, N, K, group) -> int:
    return int(lib().w4a16_workspace_bytes(M, N, K, group))


def w4a16_select_kernel(M, N, K, group) -> int:
    return int(lib().w4a16_select_kernel(M, N, K, group))


def w4a16_gemm(A, wq, scales, zeros, N, group, sym, layout=LAYOUT_PLAIN, C=None, workspace=None,
               kernel=KERNEL_AUTO, dev_status=None):
    """C[M, N] = A[M, K] . dequant(W) with FP32 accumulation; C in the dtype of A."""
    M, K = A.shape
    a_dtype = _DTYPES[A.dtype]
    if C is None:
        C = torch.empty((M, N), dtype=A.dtype, device=A.device)
    need = w4a16_workspace_bytes(M, N, K, group)
    if workspace is None and need > 0:
        # the tile counters at the front of a workspace must start at zero
        workspace = torch.zeros(need, dtype=torch.uint8, device=A.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().w4a16_gemm(_ptr(A), a_dtype, M, K, _ptr(wq), int(layout), _ptr(scales), _ptr(zeros),
                          N, group, int(sym), _ptr(C), _ptr(workspace), ws_bytes, int(kernel),
                          _ptr(dev_status), _stream())
    _check("w4a16_gemm", st)
    return C


_noalloc_ready = False


def w4a16_gemm_noalloc(A, codes, scales, zeros, N, group, sym, C=None):
    """C[M, N] = A[M, K] . dequant(W) for callers that cannot allocate device memory: the split-K
    partial sums live in the library's static scratch (see include/w4a16.h for its limit and
    for why calls that overlap on the GPU race)."""
    global _noalloc_ready
    L = lib()
    if not _noalloc_ready:
        P, I = ctypes.c_void_p, ctypes.c_int
        L.w4a16_gemm_noalloc.argtypes = [P, I, I, I, P, P, P, I, I, I, P, P]
        L.w4a16_gemm_noalloc.restype = I
        _noalloc_ready = True
    M, K = A.shape
    if C is None:
        C = torch.empty((M, N), dtype=A.dtype, device=A.device)
    st = L.w4a16_gemm_noalloc(_ptr(A), _DTYPES[A.dtype], M, K, _ptr(codes), _ptr(scales), _ptr(zeros),
                              N, group, int(sym), _ptr(C), _stream())
    _check("w4a16_gemm_noalloc", st)
    return C
