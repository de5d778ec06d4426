"""CPU oracle for group-wise weight quantization (TEST INFRASTRUCTURE ONLY).

Thin numpy/ctypes wrapper around ``liboracle.so`` (plain single-threaded C99,
``wq_oracle.c``).  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product path (the
CUDA library and its binding in ``bit_gemm_group_b200``) never does, and the
two share no code.

Arrays are numpy; 16-bit float data (bf16, fp16) travels as its uint16 bit
pattern.  Every function returns its outputs plus the oracle status code.
"""
import ctypes
import numpy as np

from . import build as _build

OK = 0
ERR_ARG = -1
ERR_NONFINITE = -5
ERR_OVERFLOW = -7

F32, BF16, F16 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


def _declare(L):
    L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
    L.oracle_f32_to_f16.restype = ctypes.c_uint16
    L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.oracle_f16_to_f32.restype = ctypes.c_float
    L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    L.oracle_f32_to_bf16.restype = ctypes.c_uint16
    L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_f32.restype = ctypes.c_float
    L.oracle_round_half_even.argtypes = [ctypes.c_float]
    L.oracle_round_half_even.restype = ctypes.c_float
    for name in ("oracle_f32_to_f16_array", "oracle_f16_to_f32_array",
                 "oracle_f32_to_bf16_array", "oracle_bf16_to_f32_array"):
        getattr(L, name).argtypes = [_P, _P, _I64]
        getattr(L, name).restype = None
    L.oracle_quantize_int4.argtypes = [_P, _INT, _I64, _I64, _INT, _INT, _P, _P, _P]
    L.oracle_quantize_int8_rows.argtypes = [_P, _INT, _I64, _I64, _P, _P]
    L.oracle_quant_act_i8.argtypes = [_P, _INT, _I64, _I64, _P, _P]
    L.oracle_dequant_int4.argtypes = [_P, _P, _P, _I64, _I64, _INT, _INT, _P]
    L.oracle_dequant_int8_rows.argtypes = [_P, _P, _I64, _I64, _P]
    L.oracle_gemm_w4a16.argtypes = [_P, _I64, _I64, _P, _P, _P, _I64, _INT, _INT,
                                    _I64, _I64, _P]
    L.oracle_gemm_w8a8_acc.argtypes = [_P, _P, _I64, _I64, _I64, _I64, _I64, _I64,
                                       _I64, _P]
    L.oracle_w8a8_rescale.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P]
    L.oracle_channel_absmax.argtypes = [_P, _INT, _I64, _I64, _P]
    L.oracle_smooth_scales.argtypes = [_P, _P, _I64, ctypes.c_double, _P]
    L.oracle_quantize_int8_rows_smoothed.argtypes = [_P, _INT, _I64, _I64, _P, _P, _P]
    L.oracle_quant_act_i8_smoothed.argtypes = [_P, _INT, _I64, _I64, _P, _P, _P]
    L.oracle_quant_kv.argtypes = [_P, _P, _INT, _I64, _I64, _I64, _P, _P, _P, _P]
    L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
    L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
    L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_to_f32.restype = ctypes.c_float
    L.oracle_quantize_fp8_rows.argtypes = [_P, _INT, _I64, _I64, _P, _P]
    L.oracle_gemm_fp8.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I64, _I64,
                                  _P, _P]
    L.oracle_gemm_w8a16.argtypes = [_P, _I64, _I64, _P, _INT, _P, _I64, _I64, _I64, _P]
    L.oracle_gptq_hinv_chol.argtypes = [_P, _INT, _I64, _I64, ctypes.c_double, _P]
    L.oracle_gptq_quantize.argtypes = [_P, _INT, _I64, _I64, _P, _INT, _INT, _P, _P, _P]
    for name in ("oracle_quantize_int4", "oracle_quantize_int8_rows",
                 "oracle_quant_act_i8", "oracle_dequant_int4",
                 "oracle_dequant_int8_rows", "oracle_gemm_w4a16",
                 "oracle_gemm_w8a8_acc", "oracle_w8a8_rescale",
                 "oracle_channel_absmax", "oracle_smooth_scales",
                 "oracle_quantize_int8_rows_smoothed", "oracle_quant_act_i8_smoothed",
                 "oracle_quant_kv", "oracle_quantize_fp8_rows", "oracle_gemm_fp8",
                 "oracle_gemm_w8a16", "oracle_gptq_hinv_chol", "oracle_gptq_quantize"):
        getattr(L, name).restype = _INT


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _tag_and_bits(W, dtype_tag):
    """Return (contiguous array, tag).  float32 arrays are tagged F32; uint16
    arrays carry bf16 or fp16 bits and need an explicit tag."""
    if W.dtype == np.float32:
        return _c(W, np.float32), F32
    if W.dtype == np.uint16:
        if dtype_tag not in (BF16, F16):
            raise ValueError("uint16 input needs dtype_tag BF16 or F16")
        return _c(W, np.uint16), dtype_tag
    raise TypeError(f"unsupported input dtype {W.dtype}")


# --- conversions -------------------------------------------------------------

def f32_to_f16(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_f16_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_to_f32(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_f16_to_f32_array(_ptr(h), _ptr(out), h.size)
    return out


def f32_to_bf16(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(b):
    b = _c(b, np.uint16)
    out = np.empty(b.shape, np.float32)
    lib().oracle_bf16_to_f32_array(_ptr(b), _ptr(out), b.size)
    return out


def round_half_even(v: float) -> float:
    return float(lib().oracle_round_half_even(ctypes.c_float(v)))


# --- quantizers ----------------------------------------------------------------

def quantize_int4(W, group_size=128, sym=True, dtype_tag=None):
    """INT4 group-wise quantize + pack.  W: [N, K] float32, or uint16 bits with
    dtype_tag BF16/F16.  Returns (codes u8 [N, K/2], scales u16 (fp16 bits)
    [N, K/g], zeros u16 [N, K/g] or None for sym, status)."""
    W, tag = _tag_and_bits(W, dtype_tag)
    N, K = W.shape
    G = K // group_size if group_size > 0 else 0
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, G), np.uint16)
    zeros = None if sym else np.zeros((N, G), np.uint16)
    st = lib().oracle_quantize_int4(_ptr(W), tag, N, K, group_size, int(bool(sym)),
                                    _ptr(codes), _ptr(scales), _ptr(zeros))
    return codes, scales, zeros, st


def quantize_int8_rows(W, dtype_tag=None):
    """Per-output-channel symmetric INT8.  Returns (q int8 [N, K], scales f32 [N], status)."""
    W, tag = _tag_and_bits(W, dtype_tag)
    N, K = W.shape
    q = np.zeros((N, K), np.int8)
    s = np.zeros((N,), np.float32)
    st = lib().oracle_quantize_int8_rows(_ptr(W), tag, N, K, _ptr(q), _ptr(s))
    return q, s, st


def quant_act_i8(X, dtype_tag=None):
    """Per-token dynamic INT8.  Returns (q int8 [M, K], scales f32 [M], status)."""
    X, tag = _tag_and_bits(X, dtype_tag)
    M, K = X.shape
    q = np.zeros((M, K), np.int8)
    s = np.zeros((M,), np.float32)
    st = lib().oracle_quant_act_i8(_ptr(X), tag, M, K, _ptr(q), _ptr(s))
    return q, s, st


def channel_absmax(A, dtype_tag=None):
    """SmoothQuant statistic: max_r |A[r, k]| per column.  Returns (f32 [K], status)."""
    A, tag = _tag_and_bits(A, dtype_tag)
    R, K = A.shape
    out = np.zeros((K,), np.float32)
    st = lib().oracle_channel_absmax(_ptr(A), tag, R, K, _ptr(out))
    return out, st


def smooth_scales(act_absmax, w_absmax, alpha=0.5):
    """SmoothQuant migration factors s [K] (f32).  Returns (s, status)."""
    a = _c(act_absmax, np.float32)
    w = _c(w_absmax, np.float32)
    s = np.zeros(a.shape, np.float32)
    st = lib().oracle_smooth_scales(_ptr(a), _ptr(w), a.shape[0], float(alpha), _ptr(s))
    return s, st


def quantize_int8_rows_smoothed(W, s, dtype_tag=None):
    """Per-channel INT8 of W diag(s).  Returns (q int8 [N, K], scales f32 [N], status)."""
    W, tag = _tag_and_bits(W, dtype_tag)
    N, K = W.shape
    s = _c(s, np.float32)
    q = np.zeros((N, K), np.int8)
    sc = np.zeros((N,), np.float32)
    st = lib().oracle_quantize_int8_rows_smoothed(_ptr(W), tag, N, K, _ptr(s), _ptr(q), _ptr(sc))
    return q, sc, st


def quant_act_i8_smoothed(X, s, dtype_tag=None):
    """Per-token INT8 of X diag(s)^-1.  Returns (q int8 [M, K], scales f32 [M], status)."""
    X, tag = _tag_and_bits(X, dtype_tag)
    M, K = X.shape
    s = _c(s, np.float32)
    q = np.zeros((M, K), np.int8)
    sc = np.zeros((M,), np.float32)
    st = lib().oracle_quant_act_i8_smoothed(_ptr(X), tag, M, K, _ptr(s), _ptr(q), _ptr(sc))
    return q, sc, st


def quant_kv(Kc, Vc, dtype_tag=None):
    """KV-cache INT8 of K, V [BH, S, D]: K per channel, V per token.
    Returns (qk int8 [BH, S, D], sk f32 [BH, D], qv int8 [BH, S, D], sv f32 [BH, S], status)."""
    Kc, tag = _tag_and_bits(Kc, dtype_tag)
    Vc, tag2 = _tag_and_bits(Vc, dtype_tag)
    assert tag == tag2 and Kc.shape == Vc.shape
    BH, S, D = Kc.shape
    qk = np.zeros((BH, S, D), np.int8)
    qv = np.zeros((BH, S, D), np.int8)
    sk = np.zeros((BH, D), np.float32)
    sv = np.zeros((BH, S), np.float32)
    st = lib().oracle_quant_kv(_ptr(Kc), _ptr(Vc), tag, BH, S, D, _ptr(qk), _ptr(sk), _ptr(qv),
                               _ptr(sv))
    return qk, sk, qv, sv, st


def f32_to_e4m3(x):
    x = np.asarray(x, np.float32).ravel()
    return np.array([lib().oracle_f32_to_e4m3(float(v)) for v in x], np.uint8)


def e4m3_to_f32(c):
    c = np.asarray(c, np.uint8).ravel()
    return np.array([lib().oracle_e4m3_to_f32(int(v)) for v in c], np.float32)


def quantize_fp8_rows(W, dtype_tag=None):
    """Per-row E4M3 (weights per output channel, activations per token).
    Returns (q uint8 e4m3 codes [R, K], scales f32 [R], status)."""
    W, tag = _tag_and_bits(W, dtype_tag)
    R, K = W.shape
    q = np.zeros((R, K), np.uint8)
    s = np.zeros((R,), np.float32)
    st = lib().oracle_quantize_fp8_rows(_ptr(W), tag, R, K, _ptr(q), _ptr(s))
    return q, s, st


def gemm_fp8(qx, sx, qw, sw, m0, m1, n0, n1):
    """FP8 W8A8 product over a window: (Y fp64, exact fp64 sums, status)."""
    qx = _c(qx, np.uint8); qw = _c(qw, np.uint8)
    sx = _c(sx, np.float32); sw = _c(sw, np.float32)
    M, K = qx.shape
    N = qw.shape[0]
    Y = np.zeros((m1 - m0, n1 - n0), np.float64)
    acc = np.zeros((m1 - m0, n1 - n0), np.float64)
    st = lib().oracle_gemm_fp8(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), M, N, K, m0, m1, n0, n1,
                               _ptr(Y), _ptr(acc))
    return Y, acc, st


W_I8, W_E4M3 = 0, 1


def gemm_w8a16(X_bf16_bits, qw, w_fmt, sw, n0=0, n1=None):
    """fp64 Y[:, n0:n1] = X * (diag(sw) value(qw))^T, 8-bit weights (int8
    codes or E4M3 bytes), X as uint16 bf16 bits [M, K]: (Y, status)."""
    X = _c(X_bf16_bits, np.uint16)
    qw = _c(qw.view(np.uint8) if qw.dtype == np.int8 else qw, np.uint8)
    sw = _c(sw, np.float32)
    M, K = X.shape
    N = qw.shape[0]
    n1 = N if n1 is None else n1
    Y = np.zeros((M, n1 - n0), np.float64)
    st = lib().oracle_gemm_w8a16(_ptr(X), M, K, _ptr(qw), int(w_fmt), _ptr(sw), N, n0, n1,
                                 _ptr(Y))
    return Y, st


def gptq_hinv_chol(X, damp=0.01, dtype_tag=None):
    """GPTQ factor U [K, K] (fp64, upper) of H^-1, H = 2 X^T X + damp mean(diag H) I."""
    X, tag = _tag_and_bits(X, dtype_tag)
    T, K = X.shape
    U = np.zeros((K, K), np.float64)
    st = lib().oracle_gptq_hinv_chol(_ptr(X), tag, T, K, float(damp), _ptr(U))
    return U, st


def gptq_quantize(W, U, group_size=128, sym=True, dtype_tag=None):
    """GPTQ INT4: (codes u8 [N, K/2], scales f16 bits [N, G], zeros f16 bits or None, status)."""
    W, tag = _tag_and_bits(W, dtype_tag)
    N, K = W.shape
    U = _c(U, np.float64)
    G = K // group_size
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, G), np.uint16)
    zeros = None if sym else np.zeros((N, G), np.uint16)
    st = lib().oracle_gptq_quantize(_ptr(W), tag, N, K, _ptr(U), group_size, int(bool(sym)),
                                    _ptr(codes), _ptr(scales), _ptr(zeros))
    return codes, scales, zeros, st


def dequant_int4(codes, scales, zeros, K, group_size=128, sym=True):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint16)
    N = codes.shape[0]
    out = np.zeros((N, K), np.float32)
    st = lib().oracle_dequant_int4(_ptr(codes), _ptr(scales), _ptr(zeros), N, K,
                                   group_size, int(bool(sym)), _ptr(out))
    return out, st


def dequant_int8_rows(q, scales):
    q = _c(q, np.int8)
    scales = _c(scales, np.float32)
    N, K = q.shape
    out = np.zeros((N, K), np.float32)
    st = lib().oracle_dequant_int8_rows(_ptr(q), _ptr(scales), N, K, _ptr(out))
    return out, st


# --- products --------------------------------------------------------------------

def gemm_w4a16(X_bf16_bits, codes, scales, zeros, group_size=128, sym=True,
               n0=0, n1=None):
    """fp64 Y[:, n0:n1] = X * dequant(W)^T.  X as uint16 bf16 bits [M, K]."""
    X = _c(X_bf16_bits, np.uint16)
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint16)
    M, K = X.shape
    N = codes.shape[0]
    n1 = N if n1 is None else n1
    Y = np.zeros((M, n1 - n0), np.float64)
    st = lib().oracle_gemm_w4a16(_ptr(X), M, K, _ptr(codes), _ptr(scales),
                                 _ptr(zeros), N, group_size, int(bool(sym)),
                                 n0, n1, _ptr(Y))
    return Y, st


def gemm_w8a8_acc(qx, qw, m0=0, m1=None, n0=0, n1=None):
    qx = _c(qx, np.int8)
    qw = _c(qw, np.int8)
    M, K = qx.shape
    N = qw.shape[0]
    m1 = M if m1 is None else m1
    n1 = N if n1 is None else n1
    acc = np.zeros((m1 - m0, n1 - n0), np.int32)
    st = lib().oracle_gemm_w8a8_acc(_ptr(qx), _ptr(qw), M, N, K, m0, m1, n0, n1,
                                    _ptr(acc))
    return acc, st


def w8a8_rescale(acc, sx, sw, m0=0, n0=0):
    acc = _c(acc, np.int32)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    m1 = m0 + acc.shape[0]
    n1 = n0 + acc.shape[1]
    Y = np.zeros(acc.shape, np.float64)
    st = lib().oracle_w8a8_rescale(_ptr(acc), _ptr(sx), _ptr(sw), m0, m1, n0, n1,
                                   _ptr(Y))
    return Y, st
