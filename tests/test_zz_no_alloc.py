"""The allocation-free GEMM entry point, called through the C ABI.

w4a4_linear_noalloc serves callers that cannot allocate device memory at call
time (runtimes that plan all their buffers up front, or whose pool is full):
it takes no workspace and never needs one.  Its output must match the CPU
oracle within the tolerance of the other GPU tests, and be byte-identical to
w4a4_linear's (same kernel, same plan, partial sums added in a fixed order) on
two calls in a row, also right after a call of a different, larger shape, and
for a row slice long enough to take several passes of the small-M kernel.
This file is collected last, so a run that stops at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes as ct

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu


def _case(M, N, K, gw, r, seed):
    """Oracle-built operands (packed codes, scales, SERQ rows) for one shape."""
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((M, K)) * 2).astype(np.float16)
    X[:, 3] *= 30
    Wrot = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Xq, sx = O.rotate_quant(X, "f16", 128, None)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", gw)
    sal = np.sort(rng.choice(K, r, replace=False)).astype(np.int32)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    return dict(M=M, N=N, K=K, gw=gw, r=r, Xq=Xq, sx=sx, Wq=Wq, sw=sw, zw=zw, sal=sal, Rq=Rq, sr=sr)


def _y64(c):
    acc, acc_c = O.accum(c["Xq"], c["K"], c["Wq"], c["zw"], c["gw"], c["Rq"], c["sal"])
    return O.epilogue_f64(acc, acc_c, c["sx"], c["sw"], c["sr"] if c["r"] else None)


def _dev(c):
    from w4a4_bit_gemm_hq_b200 import hq
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float16)).cuda()
    return dict(Xq=torch.from_numpy(c["Xq"]).cuda(), sx=torch.from_numpy(c["sx"]).cuda(),
                Wq=hq.wq_tile(torch.from_numpy(c["Wq"]).cuda()), sw=f16(c["sw"]),
                zw=None if c["zw"] is None else f16(c["zw"]),
                Rq=torch.from_numpy(c["Rq"]).cuda(), sr=f16(c["sr"]),
                sal=torch.from_numpy(c["sal"]).cuda() if c["r"] else None)


def _noalloc(lib, c, g, Y):
    P = lambda t: None if t is None else ct.c_void_p(t.data_ptr())
    r = c["r"]
    st = ct.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.w4a4_linear_noalloc(P(g["Xq"]), P(g["sx"]), c["M"], c["K"], P(g["Wq"]), P(g["sw"]), P(g["zw"]),
                                   c["N"], c["gw"], P(g["Rq"]) if r else None, P(g["sr"]) if r else None,
                                   P(g["sal"]) if r else None, r, P(Y), 0, st)


def _close(y, y64, tol=1e-2):
    y = y.astype(np.float64)
    floor = 1e-3 * np.abs(y64).max()
    return float((np.abs(y - y64) / np.maximum(np.abs(y64), floor)).max()) <= tol


@pytest.mark.parametrize("M,N,K,gw,r", [(16, 11008, 4096, 128, 16), (4, 1024, 2048, 0, 8), (33, 520, 1024, 128, 8),
                                        (96, 512, 512, 0, 16)])
def test_noalloc_matches_oracle_and_workspace_entry_on_two_calls(M, N, K, gw, r):
    from w4a4_bit_gemm_hq_b200 import _lib, hq
    c = _case(M, N, K, gw, r, seed=M + N)
    g = _dev(c)
    y64 = _y64(c)
    ref = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], torch.float16)
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc(_lib.lib, c, g, Y) == _lib.HQ_OK
        torch.cuda.synchronize()
        assert torch.equal(Y, ref), "call %d differs from w4a4_linear" % call
        assert _close(Y.float().cpu().numpy(), y64), "call %d outside the tolerance of the oracle" % call
    assert hq.hq_last_device_status() == 0


def test_noalloc_right_after_a_larger_shape():
    # a first call with N = 11008 (every CTA's rows split over several warps)
    # followed by a different shape: both identical to w4a4_linear and within
    # the tolerance of the oracle
    from w4a4_bit_gemm_hq_b200 import _lib, hq
    big = _case(16, 11008, 2048, 128, 16, seed=5)
    gb = _dev(big)
    Yb = torch.empty((16, 11008), dtype=torch.float16, device="cuda")
    assert _noalloc(_lib.lib, big, gb, Yb) == _lib.HQ_OK
    small = _case(8, 2048, 4096, 0, 8, seed=6)
    gs = _dev(small)
    ref = hq.w4a4_linear(gs["Xq"], gs["sx"], gs["Wq"], gs["sw"], gs["zw"], 0, gs["Rq"], gs["sr"], gs["sal"],
                         torch.float16)
    for _ in range(2):
        Y = torch.full((8, 2048), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc(_lib.lib, small, gs, Y) == _lib.HQ_OK
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)
        assert _close(Y.float().cpu().numpy(), _y64(small))
    torch.cuda.synchronize()
    assert _close(Yb.float().cpu().numpy(), _y64(big))
    assert hq.hq_last_device_status() == 0


@pytest.mark.parametrize("gw", [0, 128])
def test_noalloc_needs_no_workspace_for_a_multi_pass_slice(gw):
    # N = 65536 gives every CTA about 443 rows: two passes of at most 16 tiles
    # of 16 rows; the workspace the ABI reports is zero for every shape
    from w4a4_bit_gemm_hq_b200 import _lib, hq
    M, N, K = 64, 65536, 256
    for m in (1, 16, 33, 64):
        assert hq.hq_linear_workspace_size(m, N, K, gw) == 0
    c = _case(M, N, K, gw, 8, seed=7)
    g = _dev(c)
    ref = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], torch.float16)
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    assert _noalloc(_lib.lib, c, g, Y) == _lib.HQ_OK
    torch.cuda.synchronize()
    assert torch.equal(Y, ref)
    assert _close(Y.float().cpu().numpy(), _y64(c))
    assert hq.hq_last_device_status() == 0
