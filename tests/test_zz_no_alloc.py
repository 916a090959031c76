"""The allocation-free GEMM entry point, called through the C ABI.

w4a4_linear_noalloc serves callers that cannot allocate device memory at call
time (runtimes that plan all their buffers up front, or whose pool is full):
instead of a caller-provided workspace it uses a fixed scratch array inside the
library.  Its output must agree with w4a4_linear's (given a workspace) within
the tolerance the other GPU tests use, on two calls in a row (the second call
finds the array as the first left it).  This file is collected last, so a run
that stops at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import ctypes as ct

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, gw, r, seed):
    from w4a4_bit_gemm_hq_b200 import hq
    g = torch.Generator(device="cuda").manual_seed(seed)
    dev = "cuda"
    X = torch.randn((M, K), generator=g, device=dev).half()
    W = (torch.randn((N, K), generator=g, device=dev) * 0.02).half()
    layer = hq.W4A4Linear.prepare(W, 128, gw, r, None, X_calib=X, out_dtype=torch.float16)
    Xq, sx = hq.hq_rotate_quant(X, 128, None)
    return layer, Xq, sx


def _noalloc(lib, layer, Xq, sx, Y, M, K, N):
    P = lambda t: None if t is None else ct.c_void_p(t.data_ptr())
    r = 0 if layer.sal_idx is None else int(layer.sal_idx.numel())
    st = ct.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.w4a4_linear_noalloc(P(Xq), P(sx), M, K, P(layer.Wq), P(layer.sw), P(layer.zw), N, layer.gw,
                                   P(layer.Rq) if r else None, P(layer.sr) if r else None,
                                   P(layer.sal_idx) if r else None, r, P(Y), 0, st)


@pytest.mark.parametrize("M,N,K,gw,r", [(16, 11008, 4096, 128, 16), (4, 1024, 2048, 0, 8), (33, 520, 1024, 128, 8),
                                        (96, 512, 512, 0, 16)])
def test_noalloc_matches_workspace_entry_on_two_calls(M, N, K, gw, r):
    from w4a4_bit_gemm_hq_b200 import _lib, hq
    layer, Xq, sx = _inputs(M, N, K, gw, r, seed=M + N)
    ref = hq.w4a4_linear(Xq, sx, layer.Wq, layer.sw, layer.zw, layer.gw, layer.Rq, layer.sr, layer.sal_idx,
                         torch.float16)
    torch.cuda.synchronize()
    ref64 = ref.double().cpu().numpy()
    floor = 1e-3 * np.abs(ref64).max()
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc(_lib.lib, layer, Xq, sx, Y, M, K, N) == _lib.HQ_OK
        torch.cuda.synchronize()
        y = Y.double().cpu().numpy()
        rel = np.abs(y - ref64) / np.maximum(np.abs(ref64), floor)
        assert np.all(np.isfinite(y)) and rel.max() <= 1e-2, (call, rel.max())
    assert hq.hq_last_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from w4a4_bit_gemm_hq_b200 import _lib, hq
    M, N, K = 64, 131072, 128
    assert hq.hq_linear_workspace_size(M, N, K, 0) > 8 * 1024 * 1024
    layer, Xq, sx = _inputs(M, N, K, 0, 8, seed=7)
    Y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    assert _noalloc(_lib.lib, layer, Xq, sx, Y, M, K, N) == _lib.HQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(Y.abs().sum()) == 0          # nothing was enqueued
