"""CPU oracle for the W4A4 rotated linear layer -- TEST INFRASTRUCTURE.

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It wraps the plain C implementation in ``hq_oracle.c``
(built by ``build_oracle.py`` with strict IEEE semantics) with numpy marshalling
and shares nothing with the CUDA library.

Each function names the passage it follows (page title, section):

* rotation, H with an all-ones first row, group-wise application --
  "OffQ: Taming Structured Outliers in LLM Quantization by Offsetting",
  Methodology 2 and 3;
* per-token symmetric 4-bit activations, W4A4 integer matmul, the single
  low-rank error matrix on the salient rows and its 4-bit residual path --
  "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
  Technical summary sections 1, 2.2, 3;
* activation L2 norm per channel as the saliency measure --
  "Adaptacion a cualquier ancho de bits (CMPQ)", Methodology A;
* the layer computes Y = W X -- "WaterSIC", Technical summary section 1.

Array conventions: activations / weights are numpy arrays whose element type
is named by a dtype tag: "f16" (numpy float16), "bf16" (numpy uint16 holding
bfloat16 bit patterns) or "f32" (numpy float32).  Packed int4 tensors are
uint8 [rows, ceil(cols/2)] with element 2j in the low nibble of byte j.  fp16
scales are returned as numpy float16.
"""
import ctypes as _ct

import numpy as _np

from .build_oracle import build as _build

_lib = _ct.CDLL(_build())

_DT = {"f16": 0, "bf16": 1, "f32": 2}
_P = _ct.c_void_p
_I64 = _ct.c_int64
_I32 = _ct.c_int32


def _sig(name, args, res=None):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_sig("hqo_hadamard_dense", [_I32, _P, _P])
_sig("hqo_rotate_rows", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P])
_sig("hqo_rotate_normalised", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P])
_sig("hqo_rotate_dense_f64", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P])
_sig("hqo_pack_s4", [_P, _I64, _I64, _P])
_sig("hqo_unpack_s4", [_P, _I64, _I64, _P])
_sig("hqo_unpack_u4", [_P, _I64, _I64, _P])
_sig("hqo_rotate_quant", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P, _P, _P])
_sig("hqo_rotate_quant8", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P, _P])
_sig("hqo_w4_pack", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P, _P])
_sig("hqo_w4_dequant", [_P, _P, _P, _I64, _I64, _I32, _P])
_sig("hqo_serq_prepare", [_P, _I64, _I64, _P, _P, _P, _I32, _P, _I32, _P, _P, _P])
_sig("hqo_accum", [_P, _I64, _I64, _P, _P, _I64, _I32, _P, _P, _I32, _P, _P], _ct.c_int)
_sig("hqo_accum8", [_P, _I64, _I64, _P, _P, _I64, _I32, _P, _P, _I32, _P, _P], _ct.c_int)
_sig("hqo_epilogue_f64", [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P])
_sig("hqo_rotate_quant_asym", [_P, _ct.c_int, _I64, _I64, _I32, _P, _P, _P, _P])
_sig("hqo_accum_asym", [_P, _P, _I64, _I64, _I32, _P, _P, _I64, _I32, _P, _P, _I32, _P, _P], _ct.c_int)
_sig("hqo_epilogue_asym_f64", [_P, _P, _I64, _I64, _I64, _I32, _I32, _P, _P, _P, _P])
_sig("hqo_linear_rows_f64", [_P, _P, _I64, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _P, _I64, _P])
_sig("hqo_linear_fp64", [_P, _ct.c_int, _I64, _I64, _P, _ct.c_int, _I64, _P])
_sig("hqo_salient_channels", [_P, _ct.c_int, _I64, _I64, _I32, _P, _I32, _P, _P])
_sig("hqo_f32_to_f16_array", [_P, _I64, _P])
_sig("hqo_f16_to_f32_array", [_P, _I64, _P])


def _c(a, dtype):
    return _np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _raw(x, xdtype):
    want = {"f16": _np.float16, "bf16": _np.uint16, "f32": _np.float32}[xdtype]
    return _c(x, want)


def _signs(d, g):
    if d is None:
        return None
    d = _c(d, _np.int8)
    assert d.shape == (g,) and d[0] == 1 and _np.all(_np.abs(d) == 1)
    return d


# ---------------------------------------------------------------- conversions
def f32_to_f16(a):
    """IEEE binary32 -> binary16, round to nearest even (bit patterns as float16)."""
    a = _c(a, _np.float32)
    out = _np.empty(a.shape, _np.uint16)
    _lib.hqo_f32_to_f16_array(_ptr(a), a.size, _ptr(out))
    return out.view(_np.float16)


def f16_to_f32(a):
    a = _c(a, _np.float16).view(_np.uint16)
    out = _np.empty(a.shape, _np.float32)
    _lib.hqo_f16_to_f32_array(_ptr(a), a.size, _ptr(out))
    return out


# ---------------------------------------------------------------- rotation
def hadamard_dense(g, d=None):
    """H[i][j] = d[i] * (-1)^popcount(i&j) as int8 [g, g] (OffQ, Methodology 2)."""
    H = _np.empty((g, g), _np.int8)
    _lib.hqo_hadamard_dense(g, _ptr(_signs(d, g)), _ptr(H))
    return H


def rotate_rows(X, xdtype, g, d=None):
    """u = X * blockdiag(diag(d) H_sylv), unnormalised fp32 butterfly."""
    X = _raw(X, xdtype)
    M, K = X.shape
    u = _np.empty((M, K), _np.float32)
    _lib.hqo_rotate_rows(_ptr(X), _DT[xdtype], M, K, g, _ptr(_signs(d, g)), _ptr(u))
    return u


def rotate_normalised(W, wdtype, g, d=None):
    """W_rot = fl32(u * fl32(1/sqrt(g))): the rotation folded into the weights."""
    W = _raw(W, wdtype)
    N, K = W.shape
    out = _np.empty((N, K), _np.float32)
    _lib.hqo_rotate_normalised(_ptr(W), _DT[wdtype], N, K, g, _ptr(_signs(d, g)), _ptr(out))
    return out


def rotate_dense_f64(X, xdtype, g, d=None):
    """Dense fp64 product X * blockdiag(H) (no butterfly)."""
    X = _raw(X, xdtype)
    M, K = X.shape
    out = _np.empty((M, K), _np.float64)
    _lib.hqo_rotate_dense_f64(_ptr(X), _DT[xdtype], M, K, g, _ptr(_signs(d, g)), _ptr(out))
    return out


# ---------------------------------------------------------------- packing
def pack_s4(q):
    q = _c(q, _np.int8)
    R, C = q.shape
    out = _np.empty((R, (C + 1) // 2), _np.uint8)
    _lib.hqo_pack_s4(_ptr(q), R, C, _ptr(out))
    return out


def unpack_s4(p, cols):
    p = _c(p, _np.uint8)
    q = _np.empty((p.shape[0], cols), _np.int8)
    _lib.hqo_unpack_s4(_ptr(p), p.shape[0], cols, _ptr(q))
    return q


def unpack_u4(p, cols):
    p = _c(p, _np.uint8)
    q = _np.empty((p.shape[0], cols), _np.int8)
    _lib.hqo_unpack_u4(_ptr(p), p.shape[0], cols, _ptr(q))
    return q


# ---------------------------------------------------------------- quantisers
def rotate_quant(X, xdtype, g, d=None, return_u=False):
    """(Xq [M, K/2] uint8, sx [M] fp32): rotate then per-token symmetric int4."""
    X = _raw(X, xdtype)
    M, K = X.shape
    Xq = _np.empty((M, K // 2), _np.uint8)
    sx = _np.empty((M,), _np.float32)
    u = _np.empty((M, K), _np.float32) if return_u else None
    _lib.hqo_rotate_quant(_ptr(X), _DT[xdtype], M, K, g, _ptr(_signs(d, g)), _ptr(Xq), _ptr(sx), _ptr(u))
    return (Xq, sx, u) if return_u else (Xq, sx)


def rotate_quant8(X, xdtype, g, d=None):
    """W4A8 activations (DynamicPTQ, Methodology 2): (Xq8 [M, K] int8, sx [M]
    fp32) -- the same rotation with per-token symmetric 8-bit codes in
    [-127, 127]."""
    X = _raw(X, xdtype)
    M, K = X.shape
    Xq8 = _np.empty((M, K), _np.int8)
    sx = _np.empty((M,), _np.float32)
    _lib.hqo_rotate_quant8(_ptr(X), _DT[xdtype], M, K, g, _ptr(_signs(d, g)), _ptr(Xq8), _ptr(sx))
    return Xq8, sx


def w4_pack(W, wdtype, gw):
    """(Wq, sw, zw): per-channel symmetric (gw = 0; sw [N]) or group asymmetric
    int4 (sw, zw group-major [K/gw, N])."""
    W = _raw(W, wdtype)
    N, K = W.shape
    Wq = _np.empty((N, K // 2), _np.uint8)
    G = K // gw if gw else 1
    sw = _np.empty((G, N) if gw else (N,), _np.uint16)   # group-major [K/gw][N]
    zw = _np.empty((G, N), _np.uint16) if gw else None
    _lib.hqo_w4_pack(_ptr(W), _DT[wdtype], N, K, gw, _ptr(Wq), _ptr(sw), _ptr(zw))
    return Wq, sw.view(_np.float16), (zw.view(_np.float16) if gw else None)


def w4_dequant(Wq, sw, zw, K, gw):
    Wq = _c(Wq, _np.uint8)
    N = Wq.shape[0]
    out = _np.empty((N, K), _np.float32)
    zp = None if zw is None else _c(zw, _np.float16)
    _lib.hqo_w4_dequant(_ptr(Wq), _ptr(_c(sw, _np.float16)), _ptr(zp), N, K, gw, _ptr(out))
    return out


def serq_prepare(Wrot, Wq, sw, zw, gw, sal, return_e=False):
    """(Rq [N, ceil(r/2)] uint8, sr [N] fp16): SERQ's single error matrix R on
    the salient inputs S, quantised per output row to int4."""
    Wrot = _c(Wrot, _np.float32)
    N, K = Wrot.shape
    sal = _c(sal, _np.int32)
    r = sal.shape[0]
    Rq = _np.empty((N, (r + 1) // 2), _np.uint8)
    sr = _np.empty((N,), _np.uint16)
    e = _np.empty((N, r), _np.float32) if return_e else None
    zp = None if zw is None else _c(zw, _np.float16)
    _lib.hqo_serq_prepare(_ptr(Wrot), N, K, _ptr(_c(Wq, _np.uint8)), _ptr(_c(sw, _np.float16)), _ptr(zp),
                          gw, _ptr(sal), r, _ptr(Rq), _ptr(sr), _ptr(e))
    out = (Rq, sr.view(_np.float16))
    return out + (e,) if return_e else out


# ---------------------------------------------------------------- GEMM
def accum(Xq, K, Wq, zw, gw, Rq=None, sal=None):
    """Exact integer accumulators: acc [M, N, G] int64 and acc_c [M, N] int64."""
    Xq = _c(Xq, _np.uint8)
    Wq = _c(Wq, _np.uint8)
    M, N = Xq.shape[0], Wq.shape[0]
    G = K // gw if gw else 1
    r = 0 if sal is None else len(sal)
    acc = _np.empty((M, N, G), _np.int64)
    acc_c = _np.zeros((M, N), _np.int64)
    zp = None if zw is None else _c(zw, _np.float16)
    salp = None if r == 0 else _c(sal, _np.int32)
    Rqp = None if r == 0 else _c(Rq, _np.uint8)
    ovf = _lib.hqo_accum(_ptr(Xq), M, K, _ptr(Wq), _ptr(zp), N, gw, _ptr(Rqp), _ptr(salp), r,
                         _ptr(acc), _ptr(acc_c))
    assert ovf == 0, "accumulator exceeds int32"
    return acc, acc_c


def accum8(Xq8, K, Wq, zw, gw, Rq=None, sal=None):
    """W4A8 integer accumulators from 8-bit activation codes Xq8 [M, K] int8:
    acc [M, N, G] int64 and acc_c [M, N] int64 (same definitions as accum)."""
    Xq8 = _c(Xq8, _np.int8)
    Wq = _c(Wq, _np.uint8)
    M, N = Xq8.shape[0], Wq.shape[0]
    G = K // gw if gw else 1
    r = 0 if sal is None else len(sal)
    acc = _np.empty((M, N, G), _np.int64)
    acc_c = _np.zeros((M, N), _np.int64)
    zp = None if zw is None else _c(zw, _np.float16)
    salp = None if r == 0 else _c(sal, _np.int32)
    Rqp = None if r == 0 else _c(Rq, _np.uint8)
    ovf = _lib.hqo_accum8(_ptr(Xq8), M, K, _ptr(Wq), _ptr(zp), N, gw, _ptr(Rqp), _ptr(salp), r,
                          _ptr(acc), _ptr(acc_c))
    assert ovf == 0, "accumulator exceeds int32"
    return acc, acc_c


def rotate_quant_asym(X, xdtype, g, d=None):
    """OffQ per-group asymmetric activations: (Xq [M, K/2] unsigned nibbles,
    sx [M, K/g] float32, zx [M, K/g] int32)."""
    X = _raw(X, xdtype)
    M, K = X.shape
    Xq = _np.empty((M, K // 2), _np.uint8)
    sx = _np.empty((M, K // g), _np.float32)
    zx = _np.empty((M, K // g), _np.int32)
    _lib.hqo_rotate_quant_asym(_ptr(X), _DT[xdtype], M, K, g, _ptr(_signs(d, g)), _ptr(Xq), _ptr(sx), _ptr(zx))
    return Xq, sx, zx


def accum_asym(Xq, zx, K, g, Wq, zw, gw, Rq=None, sal=None):
    """Integer accumulators per activation group with asymmetric activations:
    acc [M, N, K/g] int64 and acc_c [M, N, K/g] int64."""
    assert gw == 0 or gw % g == 0, "activation groups must nest in the weight groups"
    Xq = _c(Xq, _np.uint8)
    Wq = _c(Wq, _np.uint8)
    M, N = Xq.shape[0], Wq.shape[0]
    G = K // g
    r = 0 if sal is None else len(sal)
    acc = _np.empty((M, N, G), _np.int64)
    acc_c = _np.zeros((M, N, G), _np.int64)
    zp = None if zw is None else _c(zw, _np.float16)
    salp = None if r == 0 else _c(sal, _np.int32)
    Rqp = None if r == 0 else _c(Rq, _np.uint8)
    ovf = _lib.hqo_accum_asym(_ptr(Xq), _ptr(_c(zx, _np.int32)), M, K, g, _ptr(Wq), _ptr(zp), N, gw, _ptr(Rqp),
                              _ptr(salp), r, _ptr(acc), _ptr(acc_c))
    assert ovf == 0, "accumulator exceeds int32"
    return acc, acc_c


def epilogue_asym_f64(acc, acc_c, g, gw, sx, sw, sr=None):
    """y64 = sum_b sx[m, b] (sw[b', n] acc_b + sr[n] acc_c_b) in fp64."""
    acc = _c(acc, _np.int64)
    M, N, G = acc.shape
    y = _np.empty((M, N), _np.float64)
    srp = None if sr is None else _c(sr, _np.float16)
    accc = None if sr is None else _c(acc_c, _np.int64)
    _lib.hqo_epilogue_asym_f64(_ptr(acc), _ptr(accc), M, N, G, g, gw, _ptr(_c(sx, _np.float32)),
                               _ptr(_c(sw, _np.float16)), _ptr(srp), _ptr(y))
    return y


def epilogue_f64(acc, acc_c, sx, sw, sr=None):
    """y64 = sx * (sum_g sw * acc_g + sr * acc_c) in fp64."""
    acc = _c(acc, _np.int64)
    M, N, G = acc.shape
    y = _np.empty((M, N), _np.float64)
    srp = None if sr is None else _c(sr, _np.float16)
    accc = None if sr is None else _c(acc_c, _np.int64)
    _lib.hqo_epilogue_f64(_ptr(acc), _ptr(accc), M, N, G, _ptr(_c(sx, _np.float32)),
                          _ptr(_c(sw, _np.float16)), _ptr(srp), _ptr(y))
    return y


def linear_rows_f64(Xq, sx, K, Wq, sw, zw, gw, Rq, sr, sal, rows):
    """y64 for the listed rows only (large-size sampling)."""
    rows = _c(rows, _np.int64)
    Wq = _c(Wq, _np.uint8)
    N = Wq.shape[0]
    r = 0 if sal is None else len(sal)
    y = _np.empty((len(rows), N), _np.float64)
    zp = None if zw is None else _c(zw, _np.float16)
    _lib.hqo_linear_rows_f64(_ptr(_c(Xq, _np.uint8)), _ptr(_c(sx, _np.float32)), K, _ptr(Wq),
                             _ptr(_c(sw, _np.float16)), _ptr(zp), N, gw,
                             _ptr(None if r == 0 else _c(Rq, _np.uint8)),
                             _ptr(None if r == 0 else _c(sr, _np.float16)),
                             _ptr(None if r == 0 else _c(sal, _np.int32)), r, _ptr(rows), len(rows), _ptr(y))
    return y


def linear_fp64(X, xdtype, W, wdtype):
    """Unquantised Y = X W^T in fp64 (quantisation-error reporting only)."""
    X = _raw(X, xdtype)
    W = _raw(W, wdtype)
    y = _np.empty((X.shape[0], W.shape[0]), _np.float64)
    _lib.hqo_linear_fp64(_ptr(X), _DT[xdtype], X.shape[0], X.shape[1], _ptr(W), _DT[wdtype], W.shape[0], _ptr(y))
    return y


def salient_channels(X, xdtype, g, d, r):
    """(norm2 [K] fp64, sal [r] int32 ascending): top-r rotated-activation L2 norms."""
    X = _raw(X, xdtype)
    M, K = X.shape
    norm2 = _np.empty((K,), _np.float64)
    sal = _np.empty((min(r, K),), _np.int32)
    _lib.hqo_salient_channels(_ptr(X), _DT[xdtype], M, K, g, _ptr(_signs(d, g)), r, _ptr(norm2), _ptr(sal))
    return norm2, sal


def layer(X, xdtype, W, wdtype, g, d, gw, r):
    """The whole layer as a chain of the functions above (small sizes):
    returns a dict with every intermediate and y64."""
    K = X.shape[1]
    Xq, sx = rotate_quant(X, xdtype, g, d)
    Wrot = rotate_normalised(W, wdtype, g, d)
    Wq, sw, zw = w4_pack(Wrot, "f32", gw)
    _, sal = salient_channels(X, xdtype, g, d, r)
    Rq, sr = serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    acc, acc_c = accum(Xq, K, Wq, zw, gw, Rq, sal)
    y = epilogue_f64(acc, acc_c, sx, sw, sr if r else None)
    return dict(Xq=Xq, sx=sx, Wrot=Wrot, Wq=Wq, sw=sw, zw=zw, sal=sal, Rq=Rq, sr=sr,
                acc=acc, acc_c=acc_c, y=y)
