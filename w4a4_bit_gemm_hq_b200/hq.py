"""User-facing calls of the W4A4 rotated linear layer, one per C-ABI entry point
(same names), plus :class:`W4A4Linear`, which holds a prepared layer.

Every function takes and returns PyTorch CUDA tensors, checks nothing beyond
shapes and dtypes needed to size its outputs (the C ABI validates the rest and
its status is raised as :class:`HQError`), and enqueues on the current stream.

Sources (page title, section): the rotation and quantiser follow "OffQ:
Taming Structured Outliers in LLM Quantization by Offsetting", Methodology 2-3,
and "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
technical summary sections 1-3; the salient channels are those with the
largest activation L2 norm ("CMPQ", Methodology A).
"""
import torch

from . import _lib
from ._lib import HQError, check, dtype_code, lib, ptr, stream_handle

__all__ = [
    "HQError", "hq_rotate_quant", "hq_rotate", "hq_channel_sqnorm", "hq_select_salient", "w4_pack",
    "serq_prepare", "w4a4_linear", "hq_linear_workspace_size", "hq_debug_accum", "hq_last_device_status",
    "hq_debug_wait_probe", "hq_packed_weight_bytes", "wq_tile", "wq_untile", "W4A4Linear",
    "hq_rotate_quant8", "w4a8_linear", "hq_debug_accum8", "hq_rotate_quant_asym", "w4a4_linear_asym",
    "hq_debug_accum_asym", "hq_calib_extreme_tokens", "hq_calib_top1_pca", "hq_calib_householder",
    "hq_calib_channel_absmax", "hq_calib_sorted_perm", "hq_calib_flatten_scales", "hq_permute_channels",
    "calibrate_rotation_and_grouping", "hq_quant_mxfp4", "hq_mxfp4_linear",
]


def _signs_arg(H_signs):
    if H_signs is None:
        return None
    assert H_signs.dtype == torch.int8 and H_signs.is_cuda
    return ptr(H_signs)


def hq_rotate_quant(X, group, H_signs=None, Xq=None, sx=None):
    """(Xq uint8 [M, K/2], sx float32 [M]): grouped Hadamard rotation with H[0,:] = 1,
    per-token symmetric int4 codes packed two per byte."""
    M, K = X.shape
    if Xq is None:
        Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    if sx is None:
        sx = torch.empty((M,), dtype=torch.float32, device=X.device)
    check(lib.hq_rotate_quant(ptr(X), dtype_code(X.dtype), M, K, X.stride(0), group, _signs_arg(H_signs),
                              ptr(Xq), ptr(sx), stream_handle()), "hq_rotate_quant")
    return Xq, sx


def hq_rotate_quant_asym(X, group, H_signs=None, Xq=None, sx=None, zx=None):
    """OffQ per-group asymmetric codes: (Xq uint8 [M, K/2] unsigned nibbles,
    sx float32 [M, K/group], zx int32 [M, K/group])."""
    M, K = X.shape
    Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device) if Xq is None else Xq
    sx = torch.empty((M, K // group), dtype=torch.float32, device=X.device) if sx is None else sx
    zx = torch.empty((M, K // group), dtype=torch.int32, device=X.device) if zx is None else zx
    check(lib.hq_rotate_quant_asym(ptr(X), dtype_code(X.dtype), M, K, X.stride(0), group, _signs_arg(H_signs),
                                   ptr(Xq), ptr(sx), ptr(zx), stream_handle()), "hq_rotate_quant_asym")
    return Xq, sx, zx


def hq_rotate_quant8(X, group, H_signs=None, Xq8=None, sx=None):
    """(Xq8 int8 [M, K], sx float32 [M]): the same rotation with per-token
    symmetric 8-bit codes in [-127, 127] (the W4A8 activations)."""
    M, K = X.shape
    if Xq8 is None:
        Xq8 = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if sx is None:
        sx = torch.empty((M,), dtype=torch.float32, device=X.device)
    check(lib.hq_rotate_quant8(ptr(X), dtype_code(X.dtype), M, K, X.stride(0), group, _signs_arg(H_signs),
                               ptr(Xq8), ptr(sx), stream_handle()), "hq_rotate_quant8")
    return Xq8, sx


def hq_rotate(X, group, H_signs=None, out=None):
    """fp32 X * blockdiag(H) / sqrt(group) (the rotation folded into weights)."""
    M, K = X.shape
    X = X.contiguous()
    if out is None:
        out = torch.empty((M, K), dtype=torch.float32, device=X.device)
    check(lib.hq_rotate(ptr(X), dtype_code(X.dtype), M, K, group, _signs_arg(H_signs), ptr(out), stream_handle()),
          "hq_rotate")
    return out


def hq_channel_sqnorm(X, group, H_signs=None, norm2=None):
    """Accumulates the per-channel sum of squares of the rotated rows into norm2 [K]."""
    M, K = X.shape
    X = X.contiguous()
    if norm2 is None:
        norm2 = torch.zeros((K,), dtype=torch.float32, device=X.device)
    check(lib.hq_channel_sqnorm(ptr(X), dtype_code(X.dtype), M, K, group, _signs_arg(H_signs), ptr(norm2),
                                stream_handle()), "hq_channel_sqnorm")
    return norm2


def hq_select_salient(norm2, r):
    """Indices of the r largest entries (ascending), as an int32 CPU tensor."""
    n = norm2.detach().to("cpu", torch.float32).contiguous()
    out = torch.empty((r,), dtype=torch.int32)
    check(lib.hq_select_salient(ptr(n), n.numel(), r, ptr(out)), "hq_select_salient")
    return out


def hq_packed_weight_bytes(N, K):
    return int(lib.hq_packed_weight_bytes(N, K))


def wq_tile(Wq_rows):
    """Row-major packed weights [N, K/2] -> the tile-major layout of the C ABI,
    shaped [ceil(N/128), K/128, 128, 64] (padding rows are zero)."""
    N, Kh = Wq_rows.shape
    T = (N + 127) // 128
    pad = torch.zeros((T * 128, Kh), dtype=torch.uint8, device=Wq_rows.device)
    pad[:N] = Wq_rows
    return pad.view(T, 128, Kh // 64, 64).permute(0, 2, 1, 3).contiguous()


def wq_untile(Wq, N):
    """Tile-major packed weights -> row-major [N, K/2]."""
    T, KB = Wq.shape[0], Wq.shape[1]
    return Wq.permute(0, 2, 1, 3).reshape(T * 128, KB * 64)[:N]


def w4_pack(W, group):
    """(Wq uint8 tile-major [ceil(N/128), K/128, 128, 64], sw fp16 [N] or [K/group, N],
    zw fp16 [K/group, N] or None)."""
    N, K = W.shape
    W = W.contiguous()
    Wq = torch.empty(((N + 127) // 128, K // 128, 128, 64), dtype=torch.uint8, device=W.device)
    if group:
        sw = torch.empty((K // group, N), dtype=torch.float16, device=W.device)
        zw = torch.empty((K // group, N), dtype=torch.float16, device=W.device)
    else:
        sw = torch.empty((N,), dtype=torch.float16, device=W.device)
        zw = None
    check(lib.w4_pack(ptr(W), dtype_code(W.dtype), N, K, group, ptr(Wq), ptr(sw), ptr(zw), stream_handle()),
          "w4_pack")
    return Wq, sw, zw


def serq_prepare(W_rot, Wq, sw, zw, group, sal_idx):
    """(Rq uint8 [N, ceil(r/2)], sr fp16 [N]): SERQ's single error matrix on the salient inputs."""
    N, K = W_rot.shape
    r = int(sal_idx.numel())
    Rq = torch.empty((N, (r + 1) // 2), dtype=torch.uint8, device=W_rot.device)
    sr = torch.empty((N,), dtype=torch.float16, device=W_rot.device)
    check(lib.serq_prepare(ptr(W_rot), N, K, ptr(Wq), ptr(sw), ptr(zw), group, ptr(sal_idx), r, ptr(Rq), ptr(sr),
                           stream_handle()), "serq_prepare")
    return Rq, sr


def hq_linear_workspace_size(M, N, K, group):
    return int(lib.hq_linear_workspace_size(M, N, K, group))


def w4a4_linear(Xq, sx, Wq, sw, zw, group, A, B, sal_idx, out_dtype=torch.bfloat16, Y=None, workspace=None):
    """Y [M, N] = sx * (sum_b sw * acc_b + sr * acc_c), one fused launch.
    N is taken from the scales (sw [N] or [K/group, N])."""
    M = Xq.shape[0]
    K = Xq.shape[1] * 2
    N = sw.shape[-1]
    r = 0 if sal_idx is None else int(sal_idx.numel())
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=Xq.device)
    need = hq_linear_workspace_size(M, N, K, group)
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=Xq.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.w4a4_linear(ptr(Xq), ptr(sx), M, K, ptr(Wq), ptr(sw), ptr(zw), N, group,
                          ptr(A) if r else None, ptr(B) if r else None, ptr(sal_idx) if r else None, r,
                          ptr(Y), dtype_code(Y.dtype), ptr(workspace), ws_bytes, stream_handle()), "w4a4_linear")
    return Y


def w4a8_linear(Xq8, sx, Wq, sw, zw, group, A, B, sal_idx, out_dtype=torch.bfloat16, Y=None, workspace=None):
    """w4a4_linear on 8-bit activation codes Xq8 int8 [M, K]."""
    M, K = Xq8.shape
    N = sw.shape[-1]
    r = 0 if sal_idx is None else int(sal_idx.numel())
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=Xq8.device)
    need = hq_linear_workspace_size(M, N, K, group)
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=Xq8.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.w4a8_linear(ptr(Xq8), ptr(sx), M, K, ptr(Wq), ptr(sw), ptr(zw), N, group,
                          ptr(A) if r else None, ptr(B) if r else None, ptr(sal_idx) if r else None, r,
                          ptr(Y), dtype_code(Y.dtype), ptr(workspace), ws_bytes, stream_handle()), "w4a8_linear")
    return Y


def w4a4_linear_asym(Xq, sx, zx, Wq, sw, zw, group, A, B, sal_idx, out_dtype=torch.bfloat16, Y=None):
    """Y [M, N] from OffQ per-group asymmetric codes (hq_rotate_quant_asym with
    group 128)."""
    M, K = Xq.shape[0], Xq.shape[1] * 2
    N = sw.shape[-1]
    r = 0 if sal_idx is None else sal_idx.numel()
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=Xq.device)
    check(lib.w4a4_linear_asym(ptr(Xq), ptr(sx), ptr(zx), M, K, ptr(Wq), ptr(sw), ptr(zw), N, group, ptr(A), ptr(B),
                               ptr(sal_idx), r, ptr(Y), dtype_code(Y.dtype), stream_handle()), "w4a4_linear_asym")
    return Y


def hq_debug_accum_asym(Xq, zx, Wq, zw, group, N):
    """Integer accumulators [M, N, K/128] of w4a4_linear_asym (test hook)."""
    M, K = Xq.shape[0], Xq.shape[1] * 2
    acc = torch.empty((M, N, K // 128), dtype=torch.int32, device=Xq.device)
    check(lib.hq_debug_accum_asym(ptr(Xq), ptr(zx), M, K, ptr(Wq), ptr(zw), N, group, ptr(acc), stream_handle()),
          "hq_debug_accum_asym")
    return acc


def hq_debug_accum8(Xq8, Wq, zw, group, A, sal_idx, N, decode=False, workspace=None):
    """Exact int32 accumulators of the W4A8 GEMM kernel: (acc [M, N, G], acc_c [M, N])."""
    M, K = Xq8.shape
    r = 0 if sal_idx is None else int(sal_idx.numel())
    G = K // group if group else 1
    acc = torch.zeros((M, N, G), dtype=torch.int32, device=Xq8.device)
    acc_c = torch.zeros((M, N), dtype=torch.int32, device=Xq8.device)
    need = hq_linear_workspace_size(M, N, K, group) if decode else 0
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=Xq8.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.hq_debug_accum8(ptr(Xq8), M, K, ptr(Wq), ptr(zw), N, group, ptr(A) if r else None,
                              ptr(sal_idx) if r else None, r, ptr(acc), ptr(acc_c), 1 if decode else 0,
                              ptr(workspace), ws_bytes, stream_handle()), "hq_debug_accum8")
    return acc, acc_c


def hq_debug_accum(Xq, Wq, zw, group, A, sal_idx, N, decode=False, workspace=None):
    """Exact int32 accumulators of the GEMM kernel: (acc [M, N, G], acc_c [M, N])."""
    M = Xq.shape[0]
    K = Xq.shape[1] * 2
    r = 0 if sal_idx is None else int(sal_idx.numel())
    G = K // group if group else 1
    acc = torch.zeros((M, N, G), dtype=torch.int32, device=Xq.device)
    acc_c = torch.zeros((M, N), dtype=torch.int32, device=Xq.device)
    need = hq_linear_workspace_size(M, N, K, group) if decode else 0
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=Xq.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.hq_debug_accum(ptr(Xq), M, K, ptr(Wq), ptr(zw), N, group, ptr(A) if r else None,
                             ptr(sal_idx) if r else None, r, ptr(acc), ptr(acc_c), 1 if decode else 0,
                             ptr(workspace), ws_bytes, stream_handle()), "hq_debug_accum")
    return acc, acc_c


# ------------------------------------------------------------ offline calibration
# OffQ, Methodology 1 (Top-1 PCA) and 3 (sorted grouping); SERQ sections 1
# (static flattening) and 3 (offline permutation).

def hq_calib_extreme_tokens(X, S, L, tok=None, T=None):
    """(tok int32 [S], T float32 [S, K]): per calibration sequence (L rows of
    X each) the token of largest max |x| and its values."""
    K = X.shape[1]
    assert X.shape[0] == S * L
    tok = torch.empty((S,), dtype=torch.int32, device=X.device) if tok is None else tok
    T = torch.empty((S, K), dtype=torch.float32, device=X.device) if T is None else T
    check(lib.hq_calib_extreme_tokens(ptr(X), dtype_code(X.dtype), S, L, K, X.stride(0), ptr(tok), ptr(T),
                                      stream_handle()), "hq_calib_extreme_tokens")
    return tok, T


def hq_calib_top1_pca(T, iters=100, v=None, lam=None):
    """(v float32 [K] unit, lam float32 [1]): principal eigenvector of T^T T / S."""
    S, K = T.shape
    assert T.dtype == torch.float32 and T.is_contiguous()
    v = torch.empty((K,), dtype=torch.float32, device=T.device) if v is None else v
    lam = torch.empty((1,), dtype=torch.float32, device=T.device) if lam is None else lam
    check(lib.hq_calib_top1_pca(ptr(T), S, K, iters, ptr(v), ptr(lam), stream_handle()), "hq_calib_top1_pca")
    return v, lam


def hq_calib_householder(X, v, Y=None):
    """Y float32 [M, K] = X Q, Q the reflection that sends +-v to e0."""
    M, K = X.shape
    Y = torch.empty((M, K), dtype=torch.float32, device=X.device) if Y is None else Y
    check(lib.hq_calib_householder(ptr(X), dtype_code(X.dtype), M, K, X.stride(0), ptr(v), ptr(Y),
                                   stream_handle()), "hq_calib_householder")
    return Y


def hq_calib_channel_absmax(X, amax=None):
    """amax float32 [K] = max over rows of |X|."""
    M, K = X.shape
    amax = torch.empty((K,), dtype=torch.float32, device=X.device) if amax is None else amax
    check(lib.hq_calib_channel_absmax(ptr(X), dtype_code(X.dtype), M, K, max(X.stride(0), K), ptr(amax),
                                      stream_handle()), "hq_calib_channel_absmax")
    return amax


def hq_calib_sorted_perm(stat, perm=None):
    """perm int32 [K]: channels in decreasing stat (ties to the lower index)."""
    K = stat.shape[0]
    perm = torch.empty((K,), dtype=torch.int32, device=stat.device) if perm is None else perm
    check(lib.hq_calib_sorted_perm(ptr(stat), K, ptr(perm), stream_handle()), "hq_calib_sorted_perm")
    return perm


def hq_calib_flatten_scales(xmax, wmax, alpha=0.5, s=None):
    """s float32 [K] = xmax^alpha / wmax^(1-alpha)."""
    K = xmax.shape[0]
    s = torch.empty((K,), dtype=torch.float32, device=xmax.device) if s is None else s
    check(lib.hq_calib_flatten_scales(ptr(xmax), ptr(wmax), K, float(alpha), ptr(s), stream_handle()),
          "hq_calib_flatten_scales")
    return s


def hq_permute_channels(X, perm=None, s=None, op=0, Y=None):
    """Y float32 [M, K]: Y[:, j] = X[:, perm[j]] (op 1: / s, op 2: * s, taken at perm[j])."""
    M, K = X.shape
    Y = torch.empty((M, K), dtype=torch.float32, device=X.device) if Y is None else Y
    check(lib.hq_permute_channels(ptr(X), dtype_code(X.dtype), M, K, max(X.stride(0), K),
                                  None if perm is None else ptr(perm), None if s is None else ptr(s), op, ptr(Y),
                                  stream_handle()), "hq_permute_channels")
    return Y


def calibrate_rotation_and_grouping(X_calib, S, L, W, iters=100):
    """The offline OffQ calibration of one layer, every step on the GPU:
    extreme tokens -> Top-1 PCA direction v -> Householder rotation of the
    calibration activations and of the weight rows -> per-channel max |x| ->
    sorted-grouping permutation.  Returns (v, perm, W_cal) with W_cal float32
    [N, K] = (W Q)[:, perm]: activations that arrive as (X Q)[:, perm] give
    the same product X W^T."""
    _, T = hq_calib_extreme_tokens(X_calib, S, L)
    v, _ = hq_calib_top1_pca(T, iters)
    Xr = hq_calib_householder(X_calib, v)
    perm = hq_calib_sorted_perm(hq_calib_channel_absmax(Xr))
    W_cal = hq_permute_channels(hq_calib_householder(W, v), perm)
    return v, perm, W_cal


def hq_quant_mxfp4(X, Xq=None, scales=None):
    """(codes uint8 [M, K/2], scale bytes uint8 [M, K/32]): MXFP4 blocks of 32
    values (E2M1 codes, UE8M0 shared exponent) of the rows of X."""
    M, K = X.shape
    Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device) if Xq is None else Xq
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device=X.device) if scales is None else scales
    check(lib.hq_quant_mxfp4(ptr(X), dtype_code(X.dtype), M, K, X.stride(0), ptr(Xq), ptr(scales),
                             stream_handle()), "hq_quant_mxfp4")
    return Xq, scales


def hq_mxfp4_linear(Xq, sx, Wq, sw, Y=None, accumulate=False):
    """Y float32 [M, N] (+)= X^ W^T for MXFP4 codes and scale bytes."""
    M, N, K = Xq.shape[0], Wq.shape[0], 2 * Xq.shape[1]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=Xq.device)
        accumulate = False
    check(lib.hq_mxfp4_linear(ptr(Xq), ptr(sx), M, K, ptr(Wq), ptr(sw), N, ptr(Y), 1 if accumulate else 0,
                              stream_handle()), "hq_mxfp4_linear")
    return Y


def hq_last_device_status():
    return int(lib.hq_last_device_status(stream_handle()))


def hq_debug_wait_probe(limit_ns):
    check(lib.hq_debug_wait_probe(int(limit_ns), stream_handle()), "hq_debug_wait_probe")


class W4A4Linear:
    """A prepared W4A4 layer (W4A8 with act_bits=8; OffQ per-group asymmetric
    4-bit activations with offq=True): rotation signs, packed weights, SERQ
    term, workspace.

    ``prepare`` runs the offline steps on the GPU: fold the rotation into W,
    pack to int4, pick the r salient input channels from calibration
    activations (largest rotated L2 norm), build SERQ's error matrix.
    ``forward`` is the online path: one rotate/quant launch and one GEMM launch.
    """

    def __init__(self, group, gw, H_signs, Wq, sw, zw, Rq, sr, sal_idx, K, N, out_dtype, act_bits=4, offq=False):
        self.group, self.gw, self.H_signs = group, gw, H_signs
        self.Wq, self.sw, self.zw, self.Rq, self.sr, self.sal_idx = Wq, sw, zw, Rq, sr, sal_idx
        self.K, self.N, self.out_dtype = K, N, out_dtype
        if act_bits not in (4, 8):
            raise ValueError("act_bits must be 4 (W4A4) or 8 (W4A8)")
        if offq and (act_bits != 4 or group != 128):
            raise ValueError("OffQ activations are 4-bit with groups of 128 channels")
        self.act_bits = act_bits
        self.offq = offq
        self._ws = {}

    @staticmethod
    def check_inputs(K, group, r, H_signs=None, sal_idx=None):
        """Host-side checks of the caller-supplied Hadamard signs and salient
        channels (ValueError): H_signs is `group` entries in {+1, -1} with
        H_signs[0] = +1 (the first row of H all ones); sal_idx is r strictly
        ascending indices in [0, K)."""
        if H_signs is not None:
            d = H_signs.detach().to("cpu")
            if d.dim() != 1 or d.numel() != group:
                raise ValueError("H_signs must hold one sign per channel of a group (%d)" % group)
            if not bool(((d == 1) | (d == -1)).all()):
                raise ValueError("H_signs entries must be +1 or -1")
            if int(d[0]) != 1:
                raise ValueError("H_signs[0] must be +1 (the first row of H is all ones)")
        if sal_idx is not None:
            s = sal_idx.detach().to("cpu").to(torch.int64).reshape(-1)
            if s.numel() != r:
                raise ValueError("sal_idx holds %d indices, r = %d" % (s.numel(), r))
            if r and (int(s.min()) < 0 or int(s.max()) >= K):
                raise ValueError("sal_idx entries must lie in [0, K)")
            if r > 1 and not bool((s[1:] > s[:-1]).all()):
                raise ValueError("sal_idx must be strictly ascending")

    @classmethod
    def prepare(cls, W, group, gw, r, H_signs=None, X_calib=None, sal_idx=None, out_dtype=torch.bfloat16,
                act_bits=4, offq=False):
        N, K = W.shape
        cls.check_inputs(K, group, r, H_signs, sal_idx)
        W_rot = hq_rotate(W, group, H_signs)
        Wq, sw, zw = w4_pack(W_rot, gw)
        if sal_idx is None and r > 0:
            norm2 = hq_channel_sqnorm(X_calib, group, H_signs)
            sal_idx = hq_select_salient(norm2, r).to(W.device)
        if r > 0:
            sal_idx = sal_idx.to(device=W.device, dtype=torch.int32).contiguous()
            Rq, sr = serq_prepare(W_rot, Wq, sw, zw, gw, sal_idx)
        else:
            sal_idx, Rq, sr = None, None, None
        del W_rot
        return cls(group, gw, H_signs, Wq, sw, zw, Rq, sr, sal_idx, K, N, out_dtype, act_bits, offq)

    def reset_workspaces(self):
        """Zero the cached workspaces (none is allocated while
        hq_linear_workspace_size reports 0, as it does for every shape)."""
        for ws in self._ws.values():
            ws.zero_()

    def workspace(self, M, device):
        need = hq_linear_workspace_size(M, self.N, self.K, self.gw)
        if need == 0:
            return None
        ws = self._ws.get(need)
        if ws is None:
            ws = torch.zeros((need,), dtype=torch.uint8, device=device)
            self._ws[need] = ws
        return ws

    def forward(self, X, Y=None, Xq=None, sx=None):
        if self.offq:
            Xq, sx, zx = hq_rotate_quant_asym(X, self.group, self.H_signs, Xq, sx)
            return w4a4_linear_asym(Xq, sx, zx, self.Wq, self.sw, self.zw, self.gw, self.Rq, self.sr,
                                    self.sal_idx, self.out_dtype, Y)
        if self.act_bits == 8:
            Xq, sx = hq_rotate_quant8(X, self.group, self.H_signs, Xq, sx)
            return w4a8_linear(Xq, sx, self.Wq, self.sw, self.zw, self.gw, self.Rq, self.sr, self.sal_idx,
                               self.out_dtype, Y, self.workspace(X.shape[0], X.device))
        Xq, sx = hq_rotate_quant(X, self.group, self.H_signs, Xq, sx)
        return w4a4_linear(Xq, sx, self.Wq, self.sw, self.zw, self.gw, self.Rq, self.sr, self.sal_idx,
                           self.out_dtype, Y, self.workspace(X.shape[0], X.device))

    __call__ = forward
