"""bit_gemm_group_b200 -- Python binding of libwq (include/wq.h).

Group-wise affine weight quantization and fused-dequantize W4A16 / W8A8 matrix
products for NVIDIA B200 (sm_100a).  This module only marshals arguments:
each function with a ``wq_`` name calls the C entry point of the same name
with the tensors' device pointers and the current CUDA stream; every step runs
in the library's CUDA kernels.  There is no CPU fallback: importing works
without a GPU, but every call needs ``libwq.so`` (built by ``build()``) and an
sm_100 device, and raises ``WQError`` otherwise.

The helpers without the prefix (``quantize_pack``, ``dequant``, ``gemm_w4a16``,
``quant_act_i8``, ``gemm_w8a8``) allocate the outputs with torch and call the
``wq_`` functions.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwq.so")

WQ_OK = 0
WQ_ERR_ARG = -1
WQ_ERR_UNSUPPORTED = -2
WQ_ERR_ALIGN = -3
WQ_ERR_CUDA = -4
WQ_ERR_NONFINITE = -5
WQ_ERR_TIMEOUT = -6
WQ_ERR_WORKSPACE = -8
WQ_ERR_NO_DEVICE = -9

WQ_F32, WQ_BF16, WQ_F16 = 0, 1, 2

# every symbol include/wq.h declares
EXPORTED = (
    "wq_quantize_pack", "wq_dequant", "wq_w4a16_workspace_bytes", "wq_gemm_w4a16",
    "wq_quant_act_i8",
    "wq_w8a8_workspace_bytes", "wq_gemm_w8a8", "wq_get_device_status",
    "wq_status_str", "wq_last_cuda_error", "wq_selftest_wait_timeout",
    "wq_gemm_w4a16_noalloc",
    "wq_channel_absmax", "wq_smooth_scales", "wq_quantize_i8_smooth", "wq_quant_act_i8_smooth",
    "wq_gemm_w8a8_smooth", "wq_quant_kv", "wq_quantize_fp8_rows", "wq_gemm_fp8",
    "wq_gptq_workspace_bytes", "wq_gptq_quantize", "wq_gemm_w8a16",
)


class WQError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        name = _status_name(status)
        detail = ""
        if status == WQ_ERR_CUDA and _lib is not None:
            detail = ": " + _lib.wq_last_cuda_error().decode()
        super().__init__(f"{where} -> {name}{detail}")


_lib = None


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libwq.so in-tree (nvcc, sm_100a)."""
    from . import _compile as _b
    return _b.build(force=force, verbose=verbose)


def lib():
    """Load libwq.so once; raise loudly if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise WQError(WQ_ERR_NO_DEVICE,
                          f"libwq.so missing at {LIB_PATH}; run bit_gemm_group_b200.build()")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _lib = L
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t


def _declare(L):
    L.wq_quantize_pack.argtypes = [_P, _INT, _I64, _I64, _INT, _INT, _INT, _P, _P, _P, _P]
    L.wq_dequant.argtypes = [_P, _P, _P, _I64, _I64, _INT, _INT, _INT, _P, _INT, _P]
    L.wq_w4a16_workspace_bytes.argtypes = [_I64, _I64, _I64]
    L.wq_w4a16_workspace_bytes.restype = _SZ
    L.wq_gemm_w4a16.argtypes = [_P, _I64, _I64, _P, _P, _P, _I64, _INT, _INT, _P, _P, _SZ, _P]
    L.wq_quant_act_i8.argtypes = [_P, _I64, _I64, _P, _P, _P]
    L.wq_w8a8_workspace_bytes.argtypes = [_I64, _I64]
    L.wq_w8a8_workspace_bytes.restype = _SZ
    L.wq_gemm_w8a8.argtypes = [_P, _I64, _I64, _P, _P, _I64, _P, _P, _SZ, _P, _P]
    L.wq_get_device_status.argtypes = [_P, _INT]
    L.wq_status_str.argtypes = [_INT]
    L.wq_status_str.restype = ctypes.c_char_p
    L.wq_gemm_w4a16_noalloc.argtypes = [_P, _I64, _I64, _P, _P, _P, _I64, _INT, _INT, _P, _P]
    L.wq_gemm_w4a16_noalloc.restype = _INT
    L.wq_selftest_wait_timeout.argtypes = [_INT, _P]
    L.wq_selftest_wait_timeout.restype = _INT
    L.wq_last_cuda_error.argtypes = []
    L.wq_last_cuda_error.restype = ctypes.c_char_p
    L.wq_channel_absmax.argtypes = [_P, _INT, _I64, _I64, _P, _P]
    L.wq_smooth_scales.argtypes = [_P, _P, _I64, ctypes.c_float, _P, _P]
    L.wq_quantize_i8_smooth.argtypes = [_P, _INT, _I64, _I64, _P, _P, _P, _P]
    L.wq_quant_act_i8_smooth.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]
    L.wq_gemm_w8a8_smooth.argtypes = [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _SZ, _P, _P]
    L.wq_quant_kv.argtypes = [_P, _P, _INT, _I64, _I64, _I64, _P, _P, _P, _P, _P]
    L.wq_quantize_fp8_rows.argtypes = [_P, _INT, _I64, _I64, _P, _P, _P]
    L.wq_gemm_fp8.argtypes = [_P, _I64, _I64, _P, _P, _I64, _P, _P, _SZ, _P, _P]
    L.wq_gemm_w8a16.argtypes = [_P, _I64, _I64, _P, _INT, _P, _I64, _P, _P]
    L.wq_gptq_workspace_bytes.argtypes = [_I64, _I64]
    L.wq_gptq_workspace_bytes.restype = _SZ
    L.wq_gptq_quantize.argtypes = [_P, _INT, _I64, _I64, _P, _INT, _INT, _P, _P, _P, _P, _SZ, _P]
    for name in ("wq_quantize_pack", "wq_dequant", "wq_gemm_w4a16", "wq_quant_act_i8",
                 "wq_gemm_w8a8", "wq_get_device_status", "wq_channel_absmax",
                 "wq_smooth_scales", "wq_quantize_i8_smooth", "wq_quant_act_i8_smooth",
                 "wq_gemm_w8a8_smooth", "wq_quant_kv", "wq_quantize_fp8_rows", "wq_gemm_fp8",
                 "wq_gptq_quantize"):
        getattr(L, name).restype = _INT


def _status_name(status):
    if _lib is not None:
        return _lib.wq_status_str(status).decode()
    return str(status)


def _check(status, where):
    if status != WQ_OK:
        raise WQError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise WQError(WQ_ERR_ARG, "tensor is not on a CUDA device (no CPU fallback)")
    if not t.is_contiguous():
        raise WQError(WQ_ERR_ARG, "tensor must be contiguous (row-major)")
    return ctypes.c_void_p(t.data_ptr())


def _bf16(t, what):
    """Pointer of a tensor that an entry point takes as bf16 (no dtype tag)."""
    if isinstance(t, torch.Tensor) and t.dtype != torch.bfloat16:
        raise WQError(WQ_ERR_ARG, f"{what} must be bfloat16, got {t.dtype}")
    return _ptr(t)


def _fits(t, nbytes, what):
    """Refuse a buffer smaller than the bytes the call will touch: the C ABI
    receives bare pointers and cannot check their extent."""
    if isinstance(t, torch.Tensor):
        have = t.numel() * t.element_size()
        if have < nbytes:
            raise WQError(WQ_ERR_ARG, f"{what} holds {have} bytes, the call needs {int(nbytes)}")


def _groups(K, group_size):
    return K // group_size if group_size > 0 and K % group_size == 0 else 0


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


_DTYPE_TAG = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16, torch.float16: WQ_F16}


# ---------------------------------------------------------------- C-named calls

def wq_quantize_pack(W, group_size, bits, sym, codes, scales, zeros=None, stream=None):
    N, K = W.shape
    if bits == 4:
        G = _groups(K, group_size)
        _fits(codes, N * K // 2, "codes")
        _fits(scales, 2 * N * G, "scales")
        _fits(zeros, 2 * N * G, "zeros")
    elif bits == 8:
        _fits(codes, N * K, "codes")
        _fits(scales, 4 * N, "scales")
    st = lib().wq_quantize_pack(_ptr(W), _DTYPE_TAG.get(W.dtype, -1), N, K, group_size, bits,
                                int(bool(sym)), _ptr(codes), _ptr(scales), _ptr(zeros),
                                _stream(stream))
    _check(st, "wq_quantize_pack")


def wq_dequant(codes, scales, zeros, N, K, group_size, bits, sym, out, stream=None):
    tag = _DTYPE_TAG.get(out.dtype, -1)
    if bits == 4:
        G = _groups(K, group_size)
        _fits(codes, N * K // 2, "codes")
        _fits(scales, 2 * N * G, "scales")
        _fits(zeros, 2 * N * G, "zeros")
    elif bits == 8:
        _fits(codes, N * K, "codes")
        _fits(scales, 4 * N, "scales")
    _fits(out, N * K * out.element_size(), "out")
    st = lib().wq_dequant(_ptr(codes), _ptr(scales), _ptr(zeros), N, K, group_size, bits,
                          int(bool(sym)), _ptr(out), tag, _stream(stream))
    _check(st, "wq_dequant")


def wq_w4a16_workspace_bytes(M, N, K):
    return int(lib().wq_w4a16_workspace_bytes(M, N, K))


def wq_gemm_w4a16(X, codes, scales, zeros, N, group_size, sym, Y, ws=None, stream=None):
    M, K = X.shape
    G = _groups(K, group_size)
    _fits(codes, N * K // 2, "codes")
    _fits(scales, 2 * N * G, "scales")
    _fits(zeros, 2 * N * G, "zeros")
    _fits(Y, 2 * M * N, "Y")
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().wq_gemm_w4a16(_bf16(X, "X"), M, K, _ptr(codes), _ptr(scales), _ptr(zeros), N,
                             group_size, int(bool(sym)), _bf16(Y, "Y"), _ptr(ws), ws_bytes,
                             _stream(stream))
    _check(st, "wq_gemm_w4a16")


def wq_gemm_w4a16_noalloc(X, codes, scales, zeros, N, group_size, sym, Y, stream=None):
    """Decode product (M <= 16) on library-owned scratch: no workspace, no
    allocation.  Overlapping calls race; the first call per device must not
    be inside a stream capture."""
    M, K = X.shape
    G = _groups(K, group_size)
    _fits(codes, N * K // 2, "codes")
    _fits(scales, 2 * N * G, "scales")
    _fits(zeros, 2 * N * G, "zeros")
    _fits(Y, 2 * M * N, "Y")
    st = lib().wq_gemm_w4a16_noalloc(_bf16(X, "X"), M, K, _ptr(codes), _ptr(scales),
                                     _ptr(zeros), N, group_size, int(bool(sym)), _bf16(Y, "Y"),
                                     _stream(stream))
    _check(st, "wq_gemm_w4a16_noalloc")


def wq_quant_act_i8(X, q, s, stream=None):
    M, K = X.shape
    _fits(q, M * K, "q")
    _fits(s, 4 * M, "s")
    st = lib().wq_quant_act_i8(_bf16(X, "X"), M, K, _ptr(q), _ptr(s), _stream(stream))
    _check(st, "wq_quant_act_i8")


def wq_w8a8_workspace_bytes(M, K):
    return int(lib().wq_w8a8_workspace_bytes(M, K))


def wq_gemm_w8a8(X, Wq, w_scales, Y, ws, acc_out=None, stream=None):
    M, K = X.shape
    N = Wq.shape[0]
    _fits(Wq, N * K, "Wq")
    _fits(w_scales, 4 * N, "w_scales")
    _fits(Y, 2 * M * N, "Y")
    _fits(acc_out, 4 * M * N, "acc_out")
    st = lib().wq_gemm_w8a8(_bf16(X, "X"), M, K, _ptr(Wq), _ptr(w_scales), N, _bf16(Y, "Y"),
                            _ptr(ws), ws.numel() * ws.element_size(), _ptr(acc_out),
                            _stream(stream))
    _check(st, "wq_gemm_w8a8")


def wq_channel_absmax(A, out, stream=None):
    R, K = A.shape
    _fits(out, 4 * K, "out")
    st = lib().wq_channel_absmax(_ptr(A), _DTYPE_TAG.get(A.dtype, -1), R, K, _ptr(out),
                                 _stream(stream))
    _check(st, "wq_channel_absmax")


def wq_smooth_scales(act_absmax, w_absmax, alpha, s, stream=None):
    K = act_absmax.numel()
    _fits(w_absmax, 4 * K, "w_absmax")
    _fits(s, 4 * K, "s")
    st = lib().wq_smooth_scales(_ptr(act_absmax), _ptr(w_absmax), act_absmax.numel(),
                                float(alpha), _ptr(s), _stream(stream))
    _check(st, "wq_smooth_scales")


def wq_quantize_i8_smooth(W, s, q, scales, stream=None):
    N, K = W.shape
    _fits(s, 4 * K, "s")
    _fits(q, N * K, "q")
    _fits(scales, 4 * N, "scales")
    st = lib().wq_quantize_i8_smooth(_ptr(W), _DTYPE_TAG.get(W.dtype, -1), N, K, _ptr(s),
                                     _ptr(q), _ptr(scales), _stream(stream))
    _check(st, "wq_quantize_i8_smooth")


def wq_quant_act_i8_smooth(X, s, q, sx, stream=None):
    M, K = X.shape
    _fits(s, 4 * K, "s")
    _fits(q, M * K, "q")
    _fits(sx, 4 * M, "sx")
    st = lib().wq_quant_act_i8_smooth(_bf16(X, "X"), M, K, _ptr(s), _ptr(q), _ptr(sx),
                                      _stream(stream))
    _check(st, "wq_quant_act_i8_smooth")


def wq_gemm_w8a8_smooth(X, Wq, w_scales, s, Y, ws, acc_out=None, stream=None):
    M, K = X.shape
    N = Wq.shape[0]
    _fits(s, 4 * K, "s")
    _fits(Wq, N * K, "Wq")
    _fits(w_scales, 4 * N, "w_scales")
    _fits(Y, 2 * M * N, "Y")
    _fits(acc_out, 4 * M * N, "acc_out")
    st = lib().wq_gemm_w8a8_smooth(_bf16(X, "X"), M, K, _ptr(Wq), _ptr(w_scales), _ptr(s), N,
                                   _bf16(Y, "Y"), _ptr(ws), ws.numel() * ws.element_size(),
                                   _ptr(acc_out), _stream(stream))
    _check(st, "wq_gemm_w8a8_smooth")


def wq_quant_kv(K, V, qk, sk, qv, sv, stream=None):
    BH, S, D = K.shape
    _fits(V, K.numel() * K.element_size(), "V")
    _fits(qk, BH * S * D, "qk")
    _fits(qv, BH * S * D, "qv")
    _fits(sk, 4 * BH * D, "sk")
    _fits(sv, 4 * BH * S, "sv")
    st = lib().wq_quant_kv(_ptr(K), _ptr(V), _DTYPE_TAG.get(K.dtype, -1), BH, S, D, _ptr(qk),
                           _ptr(sk), _ptr(qv), _ptr(sv), _stream(stream))
    _check(st, "wq_quant_kv")


def wq_quantize_fp8_rows(A, q, scales, stream=None):
    R, K = A.shape
    _fits(q, R * K, "q")
    _fits(scales, 4 * R, "scales")
    st = lib().wq_quantize_fp8_rows(_ptr(A), _DTYPE_TAG.get(A.dtype, -1), R, K, _ptr(q),
                                    _ptr(scales), _stream(stream))
    _check(st, "wq_quantize_fp8_rows")


def wq_gemm_fp8(X, Wq, w_scales, Y, ws, acc_out=None, stream=None):
    M, K = X.shape
    N = Wq.shape[0]
    _fits(Wq, N * K, "Wq")
    _fits(w_scales, 4 * N, "w_scales")
    _fits(Y, 2 * M * N, "Y")
    _fits(acc_out, 4 * M * N, "acc_out")
    st = lib().wq_gemm_fp8(_bf16(X, "X"), M, K, _ptr(Wq), _ptr(w_scales), N, _bf16(Y, "Y"),
                           _ptr(ws), ws.numel() * ws.element_size(), _ptr(acc_out),
                           _stream(stream))
    _check(st, "wq_gemm_fp8")


WQ_W8_INT8, WQ_W8_E4M3 = 0, 1


def wq_gemm_w8a16(X, Wq, w_fmt, w_scales, Y, stream=None):
    M, K = X.shape
    N = Wq.shape[0]
    _fits(Wq, N * K, "Wq")
    _fits(w_scales, 4 * N, "w_scales")
    _fits(Y, 2 * M * N, "Y")
    st = lib().wq_gemm_w8a16(_bf16(X, "X"), M, K, _ptr(Wq), int(w_fmt), _ptr(w_scales), N,
                             _bf16(Y, "Y"), _stream(stream))
    _check(st, "wq_gemm_w8a16")


def wq_gptq_quantize(W, U, group_size, sym, codes, scales, zeros, ws, stream=None):
    N, K = W.shape
    G = _groups(K, group_size)
    _fits(U, 8 * K * K, "U")
    _fits(codes, N * K // 2, "codes")
    _fits(scales, 2 * N * G, "scales")
    _fits(zeros, 2 * N * G, "zeros")
    st = lib().wq_gptq_quantize(_ptr(W), _DTYPE_TAG.get(W.dtype, -1), N, K, _ptr(U), group_size,
                                int(bool(sym)), _ptr(codes), _ptr(scales), _ptr(zeros),
                                _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "wq_gptq_quantize")


def wq_get_device_status(reset=True, stream=None):
    """Synchronize the stream and return the first kernel-detected error code."""
    return int(lib().wq_get_device_status(_stream(stream), int(bool(reset))))


def wq_selftest_wait_timeout(limit_us, stream=None):
    """Launch the bounded-wait self-test kernel (records WQ_ERR_TIMEOUT)."""
    _check(lib().wq_selftest_wait_timeout(int(limit_us), _stream(stream)),
           "wq_selftest_wait_timeout")


def wq_status_str(status):
    return lib().wq_status_str(status).decode()


def wq_last_cuda_error():
    return lib().wq_last_cuda_error().decode()


# ----------------------------------------------------------- allocating helpers

def quantize_pack(W, group_size=128, bits=4, sym=True):
    """Returns (codes, scales, zeros).  bits=4: codes uint8 [N, K/2], fp16
    scales/zeros [N, K/g] (zeros None if sym).  bits=8: int8 [N, K], fp32 [N]."""
    N, K = W.shape
    dev = W.device
    if bits == 4:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // group_size), dtype=torch.float16, device=dev)
        zeros = None if sym else torch.empty_like(scales)
    else:
        codes = torch.empty((N, K), dtype=torch.int8, device=dev)
        scales = torch.empty((N,), dtype=torch.float32, device=dev)
        zeros = None
        group_size = K
    wq_quantize_pack(W, group_size, bits, sym, codes, scales, zeros)
    return codes, scales, zeros


def dequant(codes, scales, zeros, K, group_size=128, bits=4, sym=True,
            out_dtype=torch.float32):
    N = codes.shape[0]
    out = torch.empty((N, K), dtype=out_dtype, device=codes.device)
    wq_dequant(codes, scales, zeros, N, K, K if bits == 8 else group_size, bits, sym, out)
    return out


def w4a16_workspace(M, N, K, device):
    """A zero-filled workspace for wq_gemm_w4a16 (None when M > 16)."""
    n = wq_w4a16_workspace_bytes(M, N, K)
    return torch.zeros((n,), dtype=torch.uint8, device=device) if n else None


def gemm_w4a16(X, codes, scales, zeros, group_size=128, sym=True, ws=None):
    M, K = X.shape
    N = codes.shape[0]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = w4a16_workspace(M, N, K, X.device)
    wq_gemm_w4a16(X, codes, scales, zeros, N, group_size, sym, Y, ws)
    return Y


def quant_act_i8(X):
    M, K = X.shape
    q = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s = torch.empty((M,), dtype=torch.float32, device=X.device)
    wq_quant_act_i8(X, q, s)
    return q, s


def gemm_w8a8(X, Wq, w_scales, want_acc=False):
    M, K = X.shape
    N = Wq.shape[0]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    ws = torch.empty((max(1, wq_w8a8_workspace_bytes(M, K)),), dtype=torch.uint8,
                     device=X.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=X.device) if want_acc else None
    wq_gemm_w8a8(X, Wq, w_scales, Y, ws, acc)
    return (Y, acc) if want_acc else Y


# ------------------------------------------------------ SmoothQuant helpers

def channel_absmax(A):
    out = torch.empty((A.shape[1],), dtype=torch.float32, device=A.device)
    wq_channel_absmax(A, out)
    return out


def smooth_scales(act_absmax, w_absmax, alpha=0.5):
    s = torch.empty_like(act_absmax, dtype=torch.float32)
    wq_smooth_scales(act_absmax, w_absmax, alpha, s)
    return s


def quantize_i8_smooth(W, s):
    N, K = W.shape
    q = torch.empty((N, K), dtype=torch.int8, device=W.device)
    sc = torch.empty((N,), dtype=torch.float32, device=W.device)
    wq_quantize_i8_smooth(W, s, q, sc)
    return q, sc


def quant_act_i8_smooth(X, s):
    M, K = X.shape
    q = torch.empty((M, K), dtype=torch.int8, device=X.device)
    sx = torch.empty((M,), dtype=torch.float32, device=X.device)
    wq_quant_act_i8_smooth(X, s, q, sx)
    return q, sx


def gemm_w8a8_smooth(X, Wq, w_scales, s, want_acc=False):
    M, K = X.shape
    N = Wq.shape[0]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    ws = torch.empty((max(1, wq_w8a8_workspace_bytes(M, K)),), dtype=torch.uint8,
                     device=X.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=X.device) if want_acc else None
    wq_gemm_w8a8_smooth(X, Wq, w_scales, s, Y, ws, acc)
    return (Y, acc) if want_acc else Y


def quant_kv(K, V):
    """KV-cache INT8 of K, V [BH, S, D]: (qk, sk [BH, D], qv, sv [BH, S])."""
    BH, S, D = K.shape
    qk = torch.empty((BH, S, D), dtype=torch.int8, device=K.device)
    qv = torch.empty((BH, S, D), dtype=torch.int8, device=K.device)
    sk = torch.empty((BH, D), dtype=torch.float32, device=K.device)
    sv = torch.empty((BH, S), dtype=torch.float32, device=K.device)
    wq_quant_kv(K, V, qk, sk, qv, sv)
    return qk, sk, qv, sv


# ------------------------------------------------------------------ FP8 helpers

def quantize_fp8_rows(A):
    """Per-row E4M3: (codes uint8 [R, K], scales fp32 [R])."""
    R, K = A.shape
    q = torch.empty((R, K), dtype=torch.uint8, device=A.device)
    s = torch.empty((R,), dtype=torch.float32, device=A.device)
    wq_quantize_fp8_rows(A, q, s)
    return q, s


def gemm_fp8(X, Wq, w_scales, want_acc=False):
    M, K = X.shape
    N = Wq.shape[0]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    ws = torch.empty((max(1, wq_w8a8_workspace_bytes(M, K)),), dtype=torch.uint8,
                     device=X.device)
    acc = torch.empty((M, N), dtype=torch.float32, device=X.device) if want_acc else None
    wq_gemm_fp8(X, Wq, w_scales, Y, ws, acc)
    return (Y, acc) if want_acc else Y


# ------------------------------------------------------------------ GPTQ helper

def gemm_w8a16(X, Wq, w_scales, w_fmt=None):
    """W8A16 product of bf16 X [M, K] with 8-bit per-channel weights: int8
    codes (from quantize_pack(W, K, 8)) or E4M3 codes (from
    quantize_fp8_rows(W)); the format follows Wq's dtype unless given."""
    if w_fmt is None:
        w_fmt = WQ_W8_INT8 if Wq.dtype == torch.int8 else WQ_W8_E4M3
    Y = torch.empty((X.shape[0], Wq.shape[0]), dtype=torch.bfloat16, device=X.device)
    wq_gemm_w8a16(X, Wq, w_fmt, w_scales, Y)
    return Y


def gptq_quantize(W, U, sym=True, group_size=128):
    """GPTQ INT4 of W [N, K] with the fp64 factor U [K, K] (device tensors):
    (codes, scales, zeros) in the wq_quantize_pack format."""
    N, K = W.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // group_size), dtype=torch.float16, device=W.device)
    zeros = None if sym else torch.empty((N, K // group_size), dtype=torch.float16,
                                         device=W.device)
    ws = torch.empty((max(1, int(lib().wq_gptq_workspace_bytes(N, K))),), dtype=torch.uint8,
                     device=W.device)
    wq_gptq_quantize(W, U, group_size, sym, codes, scales, zeros, ws)
    return codes, scales, zeros
