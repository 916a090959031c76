"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, rejects invalid arguments with the
documented status before touching the device, and the host-only helper
(salient channel selection) matches numpy."""
import ctypes as ct
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "hq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(\w+)\s*\(", src)) - {"defined"})


@pytest.fixture(scope="module")
def L():
    from w4a4_bit_gemm_hq_b200 import build_lib
    build_lib.build()
    from w4a4_bit_gemm_hq_b200 import _lib
    return _lib


def test_every_declared_symbol_is_exported(L):
    names = _header_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L.lib, n), n
    assert set(names) == set(L.SIGNATURES), set(names) ^ set(L.SIGNATURES)


def test_status_strings(L):
    for s in range(6):
        assert L.lib.hq_status_str(s).startswith(b"HQ_")


P = ct.c_void_p(16)  # a non-null, 16-byte aligned dummy (never dereferenced: checks fail first)


@pytest.mark.parametrize("M,K,ld,g,xt,want", [
    (-1, 256, 256, 128, 0, 1),      # M < 0
    (4, 256, 256, 3, 0, 1),         # group not a power of two
    (4, 256, 256, 8192, 0, 1),      # group too large
    (4, 384, 384, 256, 0, 1),       # K % group
    (4, 240, 240, 16, 0, 1),        # K % 32
    (4, 256, 128, 128, 0, 1),       # ld_x < K
    (4, 256, 256, 128, 2, 3),       # fp32 activations are not quantised online
    (4, 256, 256, 128, 7, 3),       # unknown dtype
    (4, 32768, 32768, 128, 0, 3),   # K beyond one CTA per row
])
def test_rotate_quant_argument_errors(L, M, K, ld, g, xt, want):
    assert L.lib.hq_rotate_quant(P, xt, M, K, ld, g, None, P, P, None) == want


def test_rotate_quant_alignment_and_null(L):
    assert L.lib.hq_rotate_quant(ct.c_void_p(18), 0, 4, 256, 256, 128, None, P, P, None) == L.HQ_ERR_ALIGN
    assert L.lib.hq_rotate_quant(P, 0, 4, 256, 260, 128, None, P, P, None) == L.HQ_ERR_ALIGN
    assert L.lib.hq_rotate_quant(None, 0, 4, 256, 256, 128, None, P, P, None) == L.HQ_ERR_ARG
    assert L.lib.hq_rotate_quant(None, 0, 0, 256, 256, 128, None, None, None, None) == L.HQ_OK  # M == 0


def test_w4_pack_argument_errors(L):
    assert L.lib.w4_pack(P, 0, 4, 255, 0, P, P, None, None) == L.HQ_ERR_ARG          # odd K
    assert L.lib.w4_pack(P, 0, 4, 256, 96, P, P, P, None) == L.HQ_ERR_ARG           # K % group
    assert L.lib.w4_pack(P, 0, 4, 256, 128, P, P, None, None) == L.HQ_ERR_ARG        # zw missing
    assert L.lib.w4_pack(P, 5, 4, 256, 0, P, P, None, None) == L.HQ_ERR_UNSUPPORTED


def test_serq_prepare_argument_errors(L):
    assert L.lib.serq_prepare(P, 4, 256, P, P, None, 0, P, 300, P, P, None) == L.HQ_ERR_ARG  # r > 256
    assert L.lib.serq_prepare(P, 4, 256, P, P, None, 0, None, 8, P, P, None) == L.HQ_ERR_ARG  # no sal


def _lin(L, M=16, K=256, N=128, g=0, r=8, yt=1, Xq=P, sx=P, A=P, B=P, sal=P, Y=P):
    return L.lib.w4a4_linear(Xq, sx, M, K, P, P, P, N, g, A, B, sal, r, Y, yt, None, 0, None)


def test_linear_argument_errors(L):
    assert _lin(L, K=192) == L.HQ_ERR_UNSUPPORTED          # K % 128
    assert _lin(L, N=100) == L.HQ_ERR_UNSUPPORTED          # N % 8
    assert _lin(L, g=64) == L.HQ_ERR_UNSUPPORTED           # group not a multiple of 128
    assert _lin(L, K=4096, g=4096) == L.HQ_ERR_UNSUPPORTED  # group beyond 2048
    assert _lin(L, g=96) == L.HQ_ERR_ARG                   # K % group
    assert _lin(L, r=72) == L.HQ_ERR_UNSUPPORTED           # r > 64
    assert _lin(L, r=12) == L.HQ_ERR_UNSUPPORTED           # r % 8
    assert _lin(L, r=-1) == L.HQ_ERR_ARG
    assert _lin(L, yt=9) == L.HQ_ERR_UNSUPPORTED
    assert _lin(L, A=None) == L.HQ_ERR_ARG                 # r > 0 without R
    assert _lin(L, Xq=ct.c_void_p(8)) == L.HQ_ERR_ALIGN
    assert _lin(L, M=0) == L.HQ_OK                         # empty
    assert L.lib.hq_linear_workspace_size(0, 128, 256, 0) == 0


def test_wait_probe_rejects_bad_limit(L):
    assert L.lib.hq_debug_wait_probe(0, None) == L.HQ_ERR_ARG
    assert L.lib.hq_debug_wait_probe(2 * 10 ** 9, None) == L.HQ_ERR_ARG


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_salient_matches_numpy(L, seed):
    rng = np.random.default_rng(seed)
    K, r = 1000, 24
    n = rng.random(K).astype(np.float32)
    n[rng.choice(K, 5, replace=False)] = 0.5          # ties
    out = np.zeros(r, np.int32)
    assert L.lib.hq_select_salient(n.ctypes.data, K, r, out.ctypes.data) == 0
    ref = np.sort(np.argsort(-n, kind="stable")[:r])
    assert np.array_equal(out, ref)
    assert L.lib.hq_select_salient(n.ctypes.data, K, K + 1, out.ctypes.data) == L.HQ_ERR_ARG


def _lin_na(L, M=16, K=256, N=128, g=0, r=8, yt=1, Xq=P, sx=P, A=P, B=P, sal=P, Y=P):
    return L.lib.w4a4_linear_noalloc(Xq, sx, M, K, P, P, P, N, g, A, B, sal, r, Y, yt, None)


def test_noalloc_rejects_arguments_before_touching_the_device(L):
    # the same checks as w4a4_linear, all on the host: with no GPU in this
    # process, a call that reached its scratch set-up or memset would report
    # HQ_ERR_CUDA instead of these codes
    assert _lin_na(L, K=192) == L.HQ_ERR_UNSUPPORTED
    assert _lin_na(L, N=100) == L.HQ_ERR_UNSUPPORTED
    assert _lin_na(L, r=12) == L.HQ_ERR_UNSUPPORTED
    assert _lin_na(L, g=96) == L.HQ_ERR_ARG
    assert _lin_na(L, A=None) == L.HQ_ERR_ARG
    assert _lin_na(L, sx=None) == L.HQ_ERR_ARG
    assert _lin_na(L, Y=ct.c_void_p(24)) == L.HQ_ERR_ALIGN
    assert _lin_na(L, yt=9) == L.HQ_ERR_UNSUPPORTED
    assert _lin_na(L, M=0) == L.HQ_OK


def test_select_salient_rejects_nan_norms(L):
    n = np.ones(64, np.float32)
    n[7] = np.nan
    out = np.zeros(4, np.int32)
    assert L.lib.hq_select_salient(n.ctypes.data, 64, 4, out.ctypes.data) == L.HQ_ERR_ARG


def test_binding_validates_salient_indices_and_signs():
    # W4A4Linear.prepare checks caller-supplied salient channels and the
    # Hadamard sign vector on the host before any device work (the tensors
    # here are CPU tensors: a check that let them through would fail later
    # with a different error)
    import torch

    from w4a4_bit_gemm_hq_b200 import hq
    W = torch.zeros((16, 256))
    ok_d = torch.ones(128, dtype=torch.int8)
    for bad in ([3, 3, 7, 9], [9, 7, 3, 1], [0, 1, 2, 256], [-1, 0, 1, 2]):
        with pytest.raises(ValueError):
            hq.W4A4Linear.prepare(W, 128, 0, 4, ok_d, sal_idx=torch.tensor(bad, dtype=torch.int32))
    with pytest.raises(ValueError):   # r disagrees with the given indices
        hq.W4A4Linear.prepare(W, 128, 0, 8, ok_d, sal_idx=torch.tensor([0, 1, 2, 3], dtype=torch.int32))
    bad_d = ok_d.clone()
    bad_d[0] = -1                      # first row of H must stay all ones
    with pytest.raises(ValueError):
        hq.W4A4Linear.prepare(W, 128, 0, 0, bad_d)
    with pytest.raises(ValueError):    # entries other than +-1
        hq.W4A4Linear.prepare(W, 128, 0, 0, torch.full((128,), 2, dtype=torch.int8))
    with pytest.raises(ValueError):    # one sign per channel of a group
        hq.W4A4Linear.prepare(W, 128, 0, 0, torch.ones(64, dtype=torch.int8))


def test_w4a8_argument_errors(L):
    # same checks as the W4A4 calls, on the host
    assert L.lib.hq_rotate_quant8(P, 0, 4, 240, 240, 16, None, P, P, None) == L.HQ_ERR_ARG      # K % 32
    assert L.lib.hq_rotate_quant8(P, 2, 4, 256, 256, 128, None, P, P, None) == L.HQ_ERR_UNSUPPORTED
    assert L.lib.hq_rotate_quant8(ct.c_void_p(18), 0, 4, 256, 256, 128, None, P, P, None) == L.HQ_ERR_ALIGN
    assert L.lib.hq_rotate_quant8(None, 0, 0, 256, 256, 128, None, None, None, None) == L.HQ_OK   # M == 0
    lin8 = lambda **kw: L.lib.w4a8_linear(kw.get("Xq", P), P, kw.get("M", 16), kw.get("K", 256), P, P, P,
                                          kw.get("N", 128), kw.get("g", 0), P, P, P, kw.get("r", 8), P, 1,
                                          None, 0, None)
    assert lin8(K=192) == L.HQ_ERR_UNSUPPORTED
    assert lin8(r=12) == L.HQ_ERR_UNSUPPORTED
    assert lin8(g=96) == L.HQ_ERR_ARG
    assert lin8(Xq=ct.c_void_p(8)) == L.HQ_ERR_ALIGN
    assert lin8(M=0) == L.HQ_OK


def test_offq_argument_errors(L):
    # the OffQ quantiser and GEMM check on the host, before any device work
    rq = lambda **kw: L.lib.hq_rotate_quant_asym(kw.get("X", P), kw.get("xt", 0), kw.get("M", 4), 256,
                                                 kw.get("ld", 256), kw.get("g", 128), None, P, P,
                                                 kw.get("zx", P), None)
    assert rq(g=16) == L.HQ_ERR_UNSUPPORTED              # groups of 32 .. 1024
    assert rq(g=3) == L.HQ_ERR_ARG
    assert rq(xt=2) == L.HQ_ERR_UNSUPPORTED              # fp32 input
    assert rq(zx=None) == L.HQ_ERR_ARG
    assert rq(X=ct.c_void_p(18)) == L.HQ_ERR_ALIGN
    assert rq(ld=200) == L.HQ_ERR_ARG
    assert rq(M=0, X=None, zx=None) == L.HQ_OK
    lin = lambda **kw: L.lib.w4a4_linear_asym(kw.get("Xq", P), kw.get("sx", P), kw.get("zx", P), kw.get("M", 16),
                                              kw.get("K", 256), P, P, P, 128, kw.get("g", 0), P, P, P,
                                              kw.get("r", 8), P, 1, None)
    assert lin(g=64) == L.HQ_ERR_UNSUPPORTED             # weight groups of 128 activation groups
    assert lin(K=4096, g=2048 + 128) == L.HQ_ERR_ARG     # K % group
    assert lin(r=12) == L.HQ_ERR_UNSUPPORTED
    assert lin(zx=None) == L.HQ_ERR_ARG
    assert lin(zx=ct.c_void_p(18)) == L.HQ_ERR_ALIGN
    assert lin(M=0) == L.HQ_OK
    acc = lambda **kw: L.lib.hq_debug_accum_asym(P, kw.get("zx", P), kw.get("M", 4), 256, P, P, 128,
                                                 kw.get("g", 0), P, None)
    assert acc(g=64) == L.HQ_ERR_UNSUPPORTED
    assert acc(zx=None) == L.HQ_ERR_ARG
