"""Pins of the offline-calibration oracle (oracle/calib.py) against what the
pages and the mathematics fix, independent of the oracle's own code:
brute-force loops on tiny inputs, closed forms, the defining equations of an
eigenvector and of an orthogonal reflection, and invariants of the whole
calibration (the layer's product is unchanged, the outlier direction lands in
channel 0, every group starts with its largest channel).

Sources: "OffQ: Taming Structured Outliers in LLM Quantization by
Offsetting", Methodology 1 and 3 and the ablation on sorted grouping; "SERQ:
Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization", technical
summary sections 1 and 3.
"""
import math

import numpy as np
import pytest

import oracle.calib as OC
from w4a4_bit_gemm_hq_b200 import synth


# ---------------------------------------------------------------- extreme tokens
def test_extreme_tokens_brute_force_ties_and_nan():
    rng = np.random.default_rng(1)
    S, L, K = 3, 5, 7
    X = rng.standard_normal((S * L, K)).astype(np.float32)
    X[0 * L + 2, 4] = -9.0        # sequence 0: token 2 by a negative entry
    X[1 * L + 1, 0] = 8.0         # sequence 1: tokens 1 and 3 tie, the first wins
    X[1 * L + 3, 6] = -8.0
    X[2 * L + 4, 3] = 7.5         # sequence 2: token 4; a NaN elsewhere is ignored
    X[2 * L + 0, 2] = np.nan
    tok, T = OC.extreme_tokens(X, S, L)
    for s in range(S):
        best, bi = -1.0, -1
        for t in range(L):
            m = 0.0
            for k in range(K):
                a = abs(float(X[s * L + t, k]))
                if a == a and a > m:
                    m = a
            if m > best:
                best, bi = m, t
        assert tok[s] == bi
        np.testing.assert_array_equal(T[s], X[s * L + bi])
    assert list(tok) == [2, 1, 4]


def test_extreme_tokens_find_the_planted_tokens():
    wl = synth.WORKLOADS["down"]
    X, u, pos = synth.calibration_activations(wl, 6, 32)
    tok, _ = OC.extreme_tokens(synth.to_float32(X, wl.xdtype), 6, 32)
    np.testing.assert_array_equal(tok, pos)


# ---------------------------------------------------------------- Top-1 PCA
def test_pca_single_token_closed_form():
    t = np.array([3.0, -4.0, 0.0, 12.0])
    v, lam = OC.top1_pca(t[None, :])
    np.testing.assert_allclose(v, t / 13.0, atol=1e-15)      # 12 is the largest component: positive
    assert math.isclose(lam, 169.0, rel_tol=1e-14)


def test_pca_is_uncentred():
    # identical tokens: the uncentred second moment is t t^T (centring would give 0)
    t = np.array([0.5, -2.0, 1.0])
    v, lam = OC.top1_pca(np.stack([t] * 4))
    np.testing.assert_allclose(v, -t / np.linalg.norm(t), atol=1e-14)
    assert math.isclose(lam, float(t @ t), rel_tol=1e-14)


def test_pca_eigen_equation_maximality_and_sign():
    rng = np.random.default_rng(2)
    T = rng.standard_normal((20, 9))
    v, lam = OC.top1_pca(T)
    C = T.T @ T / 20
    assert np.linalg.norm(C @ v - lam * v) <= 1e-12 * lam
    assert abs(np.linalg.norm(v) - 1) < 1e-14
    for _ in range(200):
        x = rng.standard_normal(9)
        x /= np.linalg.norm(x)
        assert x @ C @ x <= lam * (1 + 1e-12)
    k = int(np.argmax(np.abs(v)))
    assert v[k] > 0


def test_pca_recovers_the_planted_direction():
    wl = synth.WORKLOADS["down"]
    X, u, _ = synth.calibration_activations(wl, 16, 16)
    _, T = OC.extreme_tokens(synth.to_float32(X, wl.xdtype), 16, 16)
    v, _ = OC.top1_pca(T)
    assert abs(v @ u) / np.linalg.norm(u) > 0.999


# ---------------------------------------------------------------- Householder
@pytest.mark.parametrize("flip", [False, True])
def test_householder_orthogonal_symmetric_sends_v_to_e0(flip):
    rng = np.random.default_rng(3)
    v = rng.standard_normal(12)
    v /= np.linalg.norm(v)
    v = -v if (v[0] > 0) != flip else v          # both signs of v[0]
    Q = OC.householder_dense(v)
    np.testing.assert_allclose(Q @ Q.T, np.eye(12), atol=1e-14)
    np.testing.assert_allclose(Q, Q.T, atol=0)
    vp = -v if v[0] > 0 else v
    e0 = np.zeros(12)
    e0[0] = 1
    np.testing.assert_allclose(vp @ Q, e0, atol=1e-14)
    X = rng.standard_normal((5, 12))
    np.testing.assert_allclose(OC.householder_apply(X, v), X @ Q, atol=1e-13)
    # a token along the outlier direction becomes a single first-channel value
    y = OC.householder_apply((7.0 * v)[None, :], v)[0]
    assert abs(abs(y[0]) - 7.0) < 1e-13 and np.abs(y[1:]).max() < 1e-13


def test_householder_keeps_the_product():
    rng = np.random.default_rng(4)
    v = rng.standard_normal(16)
    v /= np.linalg.norm(v)
    X, W = rng.standard_normal((6, 16)), rng.standard_normal((5, 16))
    Y = OC.householder_apply(X, v) @ OC.householder_apply(W, v).T
    np.testing.assert_allclose(Y, X @ W.T, atol=1e-12)


# ---------------------------------------------------------------- absmax, sorted grouping
def test_channel_absmax_brute_force():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((9, 6)).astype(np.float32)
    X[3, 2] = np.nan
    X[:, 5] = -0.0
    a = OC.channel_absmax(X)
    for k in range(6):
        m = 0.0
        for i in range(9):
            x = abs(float(X[i, k]))
            if x == x and x > m:
                m = x
        assert a[k] == np.float32(m)
    assert OC.channel_absmax(np.zeros((0, 4), np.float32)).tolist() == [0, 0, 0, 0]


def test_sorted_perm_brute_force_ties_nan():
    stat = np.array([1.0, 3.0, np.nan, 3.0, -np.inf, 2.0, 1.0, 0.0], np.float32)
    perm = OC.sorted_perm(stat)
    assert sorted(perm.tolist()) == list(range(8))
    # selection by hand: largest first, equal values in index order, NaN with -inf (index order)
    assert perm.tolist() == [1, 3, 5, 0, 6, 7, 2, 4]


def test_sorted_grouping_puts_each_groups_largest_first():
    rng = np.random.default_rng(6)
    stat = np.abs(rng.standard_normal(512)).astype(np.float32)
    perm = OC.sorted_perm(stat)
    s = stat[perm]
    assert np.all(s[:-1] >= s[1:])
    for b in range(4):
        grp = s[128 * b:128 * (b + 1)]
        assert grp[0] == grp.max()


# ---------------------------------------------------------------- flattening, permutation
def test_flatten_closed_forms_and_balance():
    xm = np.array([4.0, 9.0, 0.0, 1.0, 2.0])
    wm = np.array([1.0, 4.0, 3.0, 0.0, 8.0])
    s = OC.flatten_scales(xm, wm, 0.5)
    np.testing.assert_allclose(s, [2.0, 1.5, 1.0, 1.0, 0.5], rtol=1e-15)
    ok = (xm > 0) & (wm > 0)
    np.testing.assert_allclose((xm / s)[ok], (wm * s)[ok], rtol=1e-15)   # alpha = 0.5 balances the ranges
    np.testing.assert_allclose(OC.flatten_scales(xm, wm, 1.0)[ok], xm[ok], rtol=1e-15)
    np.testing.assert_allclose(OC.flatten_scales(xm, wm, 0.0)[ok], 1.0 / wm[ok], rtol=1e-15)


def test_permute_brute_force_and_product_invariance():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((4, 6)).astype(np.float32)
    W = rng.standard_normal((3, 6)).astype(np.float32)
    perm = rng.permutation(6).astype(np.int32)
    s = rng.uniform(0.5, 2.0, 6).astype(np.float32)
    for op in (0, 1, 2):
        Y = OC.permute_channels(X, perm, s, op)
        for m in range(4):
            for j in range(6):
                x, c = X[m, perm[j]], perm[j]
                want = x if op == 0 else (np.float32(x / s[c]) if op == 1 else np.float32(x * s[c]))
                assert Y[m, j] == want
    inv = np.argsort(perm)
    np.testing.assert_array_equal(OC.permute_channels(OC.permute_channels(X, perm), inv), X)
    Xs = OC.permute_channels(X, perm, s, 1).astype(np.float64)
    Ws = OC.permute_channels(W, perm, s, 2).astype(np.float64)
    np.testing.assert_allclose(Xs @ Ws.T, X.astype(np.float64) @ W.T.astype(np.float64), rtol=1e-5, atol=1e-5)


# ---------------------------------------------------------------- the whole calibration
def test_calibration_keeps_the_product_and_concentrates_the_outlier():
    wl = synth.WORKLOADS["down"]
    S, L = 8, 16
    X, u, _ = synth.calibration_activations(wl, S, L)
    Xf = synth.to_float32(X, wl.xdtype)
    W = synth.to_float32(synth.weights(wl, N=32), wl.wdtype)
    _, T = OC.extreme_tokens(Xf, S, L)
    v, _ = OC.top1_pca(T)
    Xr = OC.householder_apply(Xf, v)
    perm = OC.sorted_perm(np.max(np.abs(Xr), axis=0))
    Xc, Wc = Xr[:, perm], OC.householder_apply(W, v)[:, perm]
    ref = Xf.astype(np.float64) @ W.T.astype(np.float64)
    assert np.abs(Xc @ Wc.T - ref).max() <= 1e-9 * np.abs(ref).max()
    # the planted direction now sits in channel 0 (position 0 after sorting)
    assert perm[0] == 0
    Tr = OC.householder_apply(T, v)
    assert OC.energy_in_first_channel(Tr) > 0.9
    assert OC.energy_in_first_channel(T) < 0.5
