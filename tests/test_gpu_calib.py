"""GPU parity of the offline calibration kernels against the CPU oracle
(oracle/calib.py), through the C ABI: Top-1 PCA over the extreme token of each
calibration sequence ("OffQ ...", Methodology 1), sorted grouping of the
channels (Methodology 3 and the ablation), static flattening and the offline
channel permutation ("SERQ ...", technical summary sections 1 and 3).

Index and selection work (extreme tokens, channel max |x|, the sorted
permutation, the permuted copies) matches bit for bit; the fp32 arithmetic of
the power iteration, the reflection and the flattening scales is compared with
the float64 oracle within bounds derived from the arithmetic.
"""
import numpy as np
import pytest
import torch

import oracle.calib as OC
from w4a4_bit_gemm_hq_b200 import synth

pytestmark = pytest.mark.gpu

hq = pytest.importorskip("w4a4_bit_gemm_hq_b200.hq") if torch.cuda.is_available() else None

from test_gpu_parity import assert_same, dev, host, no_device_error  # noqa: E402

U = 2.0 ** -24


def _calib(name, S, L, seed=0):
    wl = synth.WORKLOADS[name]
    X, u, pos = synth.calibration_activations(wl, S, L, seed=seed)
    return wl, X, synth.to_float32(X, wl.xdtype), u, pos


@pytest.mark.parametrize("name,S,L", [("down", 32, 64), ("attn", 8, 33), ("tiny", 3, 1), ("decode", 5, 7)])
def test_extreme_tokens_bit_exact(name, S, L):
    wl, X, Xf, _, pos = _calib(name, S, L)
    tok, T = hq.hq_calib_extreme_tokens(dev(X, wl.xdtype), S, L)
    tok_o, T_o = OC.extreme_tokens(Xf, S, L)
    assert_same(host(tok), tok_o, "token indices")
    assert_same(host(T), T_o, "token values")
    no_device_error()


# K = 300: element-wise kernel; K = 304: the two-launch 16-byte path
@pytest.mark.parametrize("K", [300, 304])
def test_extreme_tokens_ties_nan_and_fp32_strided(K):
    S, L = 4, 6
    rng = np.random.default_rng(9)
    Xf = rng.standard_normal((S * L, K + 20)).astype(np.float32)
    Xf[1, 5] = 50.0
    Xf[4, 9] = -50.0            # ties with row 1 in sequence 0: the earlier token wins
    Xf[7, 2] = np.nan           # ignored by the maximum
    Xd = torch.from_numpy(Xf).cuda()[:, :K]
    tok, T = hq.hq_calib_extreme_tokens(Xd, S, L)
    tok_o, T_o = OC.extreme_tokens(np.ascontiguousarray(Xf[:, :K]), S, L)
    assert_same(host(tok), tok_o, "token indices")
    assert_same(host(T), T_o, "token values")
    assert host(tok)[0] == 1


# 32 x 11008, 16 x 4096, 8 x 8192 tokens fit a cluster's shared memory (cluster
# kernel); 64 x 11008 do not (one-CTA kernel reading T from L2)
@pytest.mark.parametrize("name,S,L", [("down", 32, 64), ("attn", 16, 16), ("large", 8, 8), ("down", 64, 8)])
def test_top1_pca_against_svd(name, S, L):
    wl, X, Xf, u, _ = _calib(name, S, L)
    _, T = hq.hq_calib_extreme_tokens(dev(X, wl.xdtype), S, L)
    v, lam = hq.hq_calib_top1_pca(T, iters=100)
    v_o, lam_o = OC.top1_pca(host(T))
    # planted tokens: lambda2 / lambda1 is small, 100 iterations leave only fp32 rounding
    assert np.abs(host(v).astype(np.float64) - v_o).max() <= 1e-4
    assert abs(float(host(lam)[0]) - lam_o) <= 1e-4 * lam_o
    assert abs(np.linalg.norm(host(v).astype(np.float64)) - 1) <= 1e-5
    assert abs(host(v).astype(np.float64) @ u) / np.linalg.norm(u) > 0.99
    no_device_error()


def test_top1_pca_closed_forms():
    t = np.zeros((1, 64), np.float32)
    t[0, 5], t[0, 9] = -3.0, 4.0
    v, lam = hq.hq_calib_top1_pca(torch.from_numpy(t).cuda(), iters=3)
    np.testing.assert_allclose(host(v)[[5, 9]], [-0.6, 0.8], atol=1e-7)
    assert abs(float(host(lam)[0]) - 25.0) <= 1e-5 * 25
    z = torch.zeros((4, 32), dtype=torch.float32, device="cuda")
    v, lam = hq.hq_calib_top1_pca(z, iters=10)
    e0 = np.zeros(32, np.float32)
    e0[0] = 1
    assert_same(host(v), e0, "all-zero tokens give e0")
    assert float(host(lam)[0]) == 0.0


def _hh_bound(Xf, v32):
    """Per-element bound of the fp32 reflection against float64: the dot
    product (K terms), 2 / (w.w) (K terms), and the final multiply-subtract."""
    K = Xf.shape[1]
    w = OC.householder_w(v32.astype(np.float64))
    ww = w @ w
    X = Xf.astype(np.float64)
    c = 2.0 * (X @ w) / ww
    dot_abs = np.abs(X) @ np.abs(w)
    err_c = (2.0 / ww) * K * 2 * U * dot_abs + K * 2 * U * np.abs(c)
    return np.abs(w)[None, :] * err_c[:, None] + 4 * U * (np.abs(X) + np.abs(c)[:, None] * np.abs(w)[None, :])


@pytest.mark.parametrize("name,S,L", [("down", 16, 16), ("attn", 8, 32)])
def test_householder_within_bound(name, S, L):
    wl, X, Xf, _, _ = _calib(name, S, L)
    _, T = hq.hq_calib_extreme_tokens(dev(X, wl.xdtype), S, L)
    v, _ = hq.hq_calib_top1_pca(T, iters=50)
    v32 = host(v)
    Y = host(hq.hq_calib_householder(dev(X, wl.xdtype), v))
    Y_o = OC.householder_apply(Xf, v32.astype(np.float64))
    assert (np.abs(Y - Y_o) <= _hh_bound(Xf, v32)).all()
    # the weight side, fp32 rows with a stride
    W = synth.to_float32(synth.weights(wl, N=96), wl.wdtype)
    Wp = np.concatenate([W, np.zeros((96, 32), np.float32)], axis=1)
    Wd = torch.from_numpy(Wp).cuda()[:, :wl.K]
    YW = host(hq.hq_calib_householder(Wd, v))
    assert (np.abs(YW - OC.householder_apply(W, v32.astype(np.float64))) <= _hh_bound(W, v32)).all()
    # the extreme tokens now hold more of their energy in channel 0 (most of
    # it where every extreme token carries the planted direction; in attn the
    # first sequence's extreme token is the single massive channel instead)
    Th = host(T)
    Tr = host(hq.hq_calib_householder(T, v))
    assert OC.energy_in_first_channel(Tr) > OC.energy_in_first_channel(Th)
    if name == "down":
        assert OC.energy_in_first_channel(Tr) > 0.9
    no_device_error()


@pytest.mark.parametrize("M,K,dt", [(1000, 11008, "bf16"), (3, 4096, "f16"), (517, 300, "f32"), (0, 64, "f32")])
def test_channel_absmax_bit_exact(M, K, dt):
    rng = np.random.default_rng(M + K)
    Xf = (rng.standard_t(3, size=(M, K)) * 5).astype(np.float32)
    if M > 2:
        Xf[1, 7] = np.nan
        Xf[2, 11] = -np.inf
    X = synth.f32_to_bf16_bits(Xf) if dt == "bf16" else (Xf.astype(np.float16) if dt == "f16" else Xf)
    Xw = synth.to_float32(X, dt) if dt != "f16" else X.astype(np.float32)
    Xd = dev(X, dt) if M > 0 else torch.zeros((0, K), dtype=torch.float32, device="cuda")
    a = hq.hq_calib_channel_absmax(Xd)
    assert_same(host(a), OC.channel_absmax(Xw), "channel max |x|")
    no_device_error()


@pytest.mark.parametrize("K", [1, 300, 4096, 11008])
def test_sorted_perm_bit_exact_with_ties_and_nan(K):
    rng = np.random.default_rng(K)
    stat = np.round(np.abs(rng.standard_normal(K)) * 4).astype(np.float32) / 4   # many ties
    if K > 10:
        stat[[3, 8]] = np.nan
        stat[5] = np.inf
    perm = host(hq.hq_calib_sorted_perm(torch.from_numpy(stat).cuda()))
    assert_same(perm, OC.sorted_perm(stat), "sorted grouping permutation")
    assert sorted(perm.tolist()) == list(range(K))


def test_flatten_scales_within_ulps():
    rng = np.random.default_rng(11)
    K = 11008
    xm = np.abs(rng.standard_t(3, K) * 10).astype(np.float32)
    wm = np.abs(rng.standard_normal(K) * 0.05).astype(np.float32)
    xm[:4] = 0
    wm[4:8] = 0
    for alpha in (0.5, 0.8, 0.0, 1.0):
        s = host(hq.hq_calib_flatten_scales(torch.from_numpy(xm).cuda(), torch.from_numpy(wm).cuda(), alpha))
        s_o = OC.flatten_scales(xm, wm, alpha)
        # two powf results (a few ulp each) and one rounded divide
        assert (np.abs(s.astype(np.float64) - s_o) <= 32 * U * s_o).all(), alpha
        assert (s[:8] == 1.0).all()


# K = 1111: element-wise kernel; K = 1112 (a multiple of 8): rows staged in shared memory
@pytest.mark.parametrize("K", [1111, 1112])
@pytest.mark.parametrize("op", [0, 1, 2])
@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
def test_permute_channels_bit_exact(op, dt, K):
    rng = np.random.default_rng(op + 3)
    M = 333
    Xf = rng.standard_normal((M, K)).astype(np.float32) * 3
    X = synth.f32_to_bf16_bits(Xf) if dt == "bf16" else (Xf.astype(np.float16) if dt == "f16" else Xf)
    Xw = synth.to_float32(X, dt) if dt != "f16" else X.astype(np.float32)
    perm = rng.permutation(K).astype(np.int32)
    s = rng.uniform(0.1, 10.0, K).astype(np.float32)
    Y = hq.hq_permute_channels(dev(X, dt), torch.from_numpy(perm).cuda(), torch.from_numpy(s).cuda(), op)
    assert_same(host(Y), OC.permute_channels(Xw, perm, s, op), "permuted channels")
    Y2 = hq.hq_permute_channels(dev(X, dt), None, torch.from_numpy(s).cuda(), op)
    assert_same(host(Y2), OC.permute_channels(Xw, None, s, op), "scaled channels")
    no_device_error()


def test_permute_out_of_range_index_is_reported():
    X = torch.ones((4, 16), dtype=torch.float32, device="cuda")
    perm = torch.arange(16, dtype=torch.int32, device="cuda")
    perm[3] = 16                        # the kernel's own bounds check turns this into an error
    Y = host(hq.hq_permute_channels(X, perm))
    assert (Y[:, 3] == 0).all() and (np.delete(Y, 3, axis=1) == 1).all()
    assert hq.hq_last_device_status() == hq._lib.HQ_ERR_ARG
    no_device_error()


def test_argument_errors_launch_nothing():
    lib, E = hq._lib.lib, hq._lib
    X = torch.zeros((4, 8), dtype=torch.float16, device="cuda")
    out = torch.full((64,), 7.0, dtype=torch.float32, device="cuda")
    tok = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    p = lambda t: t.data_ptr()
    assert lib.hq_calib_extreme_tokens(p(X), 0, 2, 0, 8, 8, p(tok), p(out), None) == E.HQ_ERR_ARG   # L = 0
    assert lib.hq_calib_extreme_tokens(p(X), 0, 2, 2, 8, 4, p(tok), p(out), None) == E.HQ_ERR_ARG   # ld_x < K
    assert lib.hq_calib_extreme_tokens(p(X), 9, 2, 2, 8, 8, p(tok), p(out), None) == E.HQ_ERR_ARG   # dtype
    assert lib.hq_calib_top1_pca(p(out), 2, 8, -1, p(out), p(out), None) == E.HQ_ERR_ARG             # iters < 0
    assert lib.hq_calib_top1_pca(p(out), 2, 100000, 1, p(out), p(out), None) == E.HQ_ERR_UNSUPPORTED
    assert lib.hq_calib_householder(p(X), 0, 4, 0, 8, p(out), p(out), None) == E.HQ_ERR_ARG          # K = 0
    assert lib.hq_calib_householder(p(X), 0, 4, 60000, 60000, p(out), p(out), None) == E.HQ_ERR_UNSUPPORTED
    assert lib.hq_calib_channel_absmax(p(X), 0, 4, 8, 8, None, None) == E.HQ_ERR_ARG                 # NULL out
    assert lib.hq_calib_sorted_perm(None, 8, p(tok), None) == E.HQ_ERR_ARG
    assert lib.hq_calib_flatten_scales(p(out), p(out), 8, 1.5, p(out), None) == E.HQ_ERR_ARG         # alpha
    assert lib.hq_permute_channels(p(X), 0, 4, 8, 8, None, None, 1, p(out), None) == E.HQ_ERR_ARG    # op 1, no s
    assert lib.hq_permute_channels(p(X), 0, 4, 8, 8, None, None, 3, p(out), None) == E.HQ_ERR_ARG    # op
    torch.cuda.synchronize()
    assert (host(out) == 7.0).all() and (host(tok) == 7).all()   # nothing was written
    no_device_error()


def test_calibration_chain_on_the_down_layer():
    wl, X, Xf, u, _ = _calib("down", 16, 32)
    W = synth.weights(wl, N=256)
    v, perm, W_cal = hq.calibrate_rotation_and_grouping(dev(X, wl.xdtype), 16, 32, dev(W, wl.wdtype), iters=100)
    v32, perm_h = host(v), host(perm)
    # each step against the oracle fed the GPU's previous step
    Xr = hq.hq_calib_householder(dev(X, wl.xdtype), v)
    stat = host(hq.hq_calib_channel_absmax(Xr))
    assert_same(perm_h, OC.sorted_perm(stat), "permutation of the GPU's statistic")
    Wf = synth.to_float32(W, wl.wdtype)
    Wc_o = OC.householder_apply(Wf, v32.astype(np.float64))[:, perm_h]
    assert (np.abs(host(W_cal) - Wc_o) <= _hh_bound(Wf, v32)[:, perm_h]).all()
    # the planted direction lands in channel 0, which sorts first
    assert perm_h[0] == 0
    # the product is kept: (X Q)[:, perm] ((W Q)[:, perm])^T = X W^T
    Xc = host(hq.hq_permute_channels(Xr, perm)).astype(np.float64)
    ref = Xf.astype(np.float64) @ Wf.T.astype(np.float64)
    got = Xc @ host(W_cal).astype(np.float64).T
    assert np.abs(got - ref).max() <= 1e-4 * np.abs(ref).max()
    no_device_error()
