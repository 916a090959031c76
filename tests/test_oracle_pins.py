"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these re-types an oracle formula: each one checks the oracle against
an independent fact -- a closed form, a library routine (numpy / scipy), an
invariant, or brute force on tiny inputs -- chosen so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails at least one.

Passages (page title, section):
  OffQ, Methodology 2-3: Hadamard H with an all-ones first row, applied per
    channel group; a single concentrated outlier becomes a constant offset.
  SERQ, Technical summary 1, 2.2, 3: per-token 4-bit activations, 4-bit
    weights, integer matmul, a single low-rank error matrix on the salient rows.
  CMPQ, Methodology A: activation L2 norm per channel.
  WaterSIC, Technical summary 1: the layer output is Y = W X.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle as O
from w4a4_bit_gemm_hq_b200 import synth


# ----------------------------------------------------------------- formats
def test_f16_to_f32_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ours = O.f16_to_f32(bits.view(np.float16))
    ref = bits.view(np.float16).astype(np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.all(np.isnan(ours[np.isnan(ref)]))


def test_f32_to_f16_matches_numpy_rne():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 6, 200000).astype(np.float32),
        # exact ties between fp16 neighbours (normal and subnormal range)
        (np.arange(1, 4000, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -24),
        (np.arange(1024, 2048, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -10),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -25, 2.0 ** -26, 6.1e-5], np.float32),
    ])
    ours = O.f32_to_f16(vals).view(np.uint16)
    ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


# ----------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("g", [2, 4, 8, 16, 128, 256, 1024])
def test_hadamard_orthogonal_and_first_row_ones(g):
    d = synth.hadamard_signs(g, seed=g)
    H = O.hadamard_dense(g, d).astype(np.int64)
    assert np.array_equal(H @ H.T, g * np.eye(g, dtype=np.int64))      # H H^T = g I
    assert np.all(H[0] == 1)                                            # H[0,:] = 1
    assert np.array_equal(np.abs(H), np.ones_like(H))


@pytest.mark.parametrize("g", [2, 8, 64, 512])
def test_hadamard_is_sylvester_with_row_signs(g):
    d = synth.hadamard_signs(g, seed=7)
    H = O.hadamard_dense(g, d).astype(np.int64)
    ref = scipy.linalg.hadamard(g).astype(np.int64) * d.astype(np.int64)[:, None]
    assert np.array_equal(H, ref)


# ----------------------------------------------------------------- rotation
@pytest.mark.parametrize("g", [4, 32, 128, 4096])
def test_butterfly_equals_dense_product_on_small_integers(g):
    # small integers: every partial sum is exact in fp32, so the butterfly must
    # reproduce the exact product x * diag(d) * H_sylv (scipy's Sylvester H).
    rng = np.random.default_rng(g)
    K = 2 * g
    x = rng.integers(-50, 51, size=(3, K)).astype(np.float16)
    d = synth.hadamard_signs(g, seed=3)
    u = O.rotate_rows(x, "f16", g, d)
    H = scipy.linalg.hadamard(g).astype(np.float64) * d[:, None]
    ref = np.concatenate([x[:, b * g:(b + 1) * g].astype(np.float64) @ H for b in range(K // g)], axis=1)
    assert np.array_equal(u.astype(np.float64), ref)


@pytest.mark.parametrize("g,dtype", [(128, "f16"), (256, "bf16"), (4096, "bf16"), (64, "f32")])
def test_butterfly_within_sum_tree_bound_of_exact_product(g, dtype):
    rng = np.random.default_rng(11)
    K = 2 * g
    x32 = (rng.standard_t(3, size=(4, K)) * 3).astype(np.float32)
    x = {"f16": x32.astype(np.float16), "bf16": synth.f32_to_bf16_bits(x32), "f32": x32}[dtype]
    xw = synth.to_float32(x, dtype).astype(np.float64)
    d = synth.hadamard_signs(g)
    u = O.rotate_rows(x, dtype, g, d).astype(np.float64)
    H = scipy.linalg.hadamard(g).astype(np.float64) * d[:, None]
    for b in range(K // g):
        blk = xw[:, b * g:(b + 1) * g]
        exact = blk @ H
        bound = np.log2(g) * 2.0 ** -24 * np.abs(blk).sum(axis=1, keepdims=True) * 1.0001
        assert np.all(np.abs(u[:, b * g:(b + 1) * g] - exact) <= bound)


def test_dense_f64_rotation_matches_scipy():
    g = 128
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 256)).astype(np.float16)
    d = synth.hadamard_signs(g)
    H = scipy.linalg.hadamard(g).astype(np.float64) * d[:, None]
    ref = np.concatenate([x[:, :g].astype(np.float64) @ H, x[:, g:].astype(np.float64) @ H], axis=1)
    assert np.array_equal(O.rotate_dense_f64(x, "f16", g, d), ref)


def test_parseval_energy():
    g = 256
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, 1024)).astype(np.float32)
    u = O.rotate_rows(x, "f32", g, synth.hadamard_signs(g)).astype(np.float64)
    lhs = (u ** 2).sum(axis=1)
    rhs = g * (x.astype(np.float64) ** 2).sum(axis=1)
    assert np.allclose(lhs, rhs, rtol=1e-5)


@pytest.mark.parametrize("g", [8, 128, 4096])
def test_offset_closed_form_first_channel(g):
    # OffQ Methodology 2: an outlier concentrated in the group's first channel
    # becomes the same constant on every channel of the group.
    K = 2 * g
    v = 37.25
    x = np.zeros((2, K), np.float16)
    x[0, 0] = v                 # first channel of group 0
    x[1, g] = -v                # first channel of group 1
    d = synth.hadamard_signs(g, seed=1)
    u = O.rotate_rows(x, "f16", g, d)
    assert np.all(u[0, :g] == np.float32(v)) and np.all(u[0, g:] == 0)
    assert np.all(u[1, g:] == np.float32(-v)) and np.all(u[1, :g] == 0)
    Xq, sx = O.rotate_quant(x, "f16", g, d)
    q = O.unpack_s4(Xq, K)
    assert np.all(q[0, :g] == 7) and np.all(q[0, g:] == 0)
    assert np.all(q[1, g:] == -7) and np.all(q[1, :g] == 0)
    cg = np.float32(1.0 / np.sqrt(g))
    assert sx[0] == np.float32(np.float32(v) / np.float32(7.0)) * cg


@pytest.mark.parametrize("c", [1, 5, 77])
def test_single_channel_spreads_with_hadamard_signs(c):
    g = 128
    x = np.zeros((1, g), np.float16)
    x[0, c] = 3.0
    d = synth.hadamard_signs(g, seed=2)
    u = O.rotate_rows(x, "f16", g, d)[0]
    assert np.all(np.abs(u) == 3.0)
    assert np.array_equal(np.sign(u), d[c] * scipy.linalg.hadamard(g)[c].astype(np.float32))


def test_rotation_fold_preserves_layer_output():
    # (X H~)(W H~)^T == X W^T for the orthonormal block rotation H~ = H/sqrt(g).
    g = 64
    rng = np.random.default_rng(3)
    X = rng.standard_normal((5, 192)).astype(np.float32)
    W = rng.standard_normal((7, 192)).astype(np.float32)
    d = synth.hadamard_signs(g)
    Xr = O.rotate_dense_f64(X, "f32", g, d) / np.sqrt(g)
    Wr = O.rotate_dense_f64(W, "f32", g, d) / np.sqrt(g)
    assert np.allclose(Xr @ Wr.T, X.astype(np.float64) @ W.astype(np.float64).T, rtol=1e-12, atol=1e-12)
    Wn = O.rotate_normalised(W, "f32", g, d).astype(np.float64)
    assert np.allclose(Wn, Wr, rtol=0, atol=1e-5 * np.abs(Wr).max())


# ----------------------------------------------------------------- packing
def test_pack_unpack_brute_force_all_bytes():
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    qs = O.unpack_s4(b, 512)
    assert np.array_equal(O.pack_s4(qs), b)
    lo, hi = qs[0, 0::2], qs[0, 1::2]
    vals = np.arange(256)
    assert np.array_equal(lo, ((vals & 15) ^ 8) - 8)          # two's complement low nibble
    assert np.array_equal(hi, ((vals >> 4) ^ 8) - 8)
    qu = O.unpack_u4(b, 512)
    assert np.array_equal(qu[0, 0::2], vals & 15) and np.array_equal(qu[0, 1::2], vals >> 4)


def test_pack_element_order():
    q = np.array([[1, 2, -1, 7, -8, 0]], np.int8)
    assert np.array_equal(O.pack_s4(q)[0], np.array([0x21, 0x7F, 0x08], np.uint8))


# ----------------------------------------------------------------- activation quantiser
@pytest.mark.parametrize("name", ["tiny", "attn", "down"])
def test_activation_quant_round_trip(name):
    wl = synth.WORKLOADS[name]
    M = 16 if name == "tiny" else 6
    K = wl.K
    X = synth.activations(wl, M=M)
    d = synth.hadamard_signs(wl.g)
    Xq, sx, u = O.rotate_quant(X, wl.xdtype, wl.g, d, return_u=True)
    q = O.unpack_s4(Xq, K).astype(np.float64)
    u = u.astype(np.float64)
    amax = np.abs(u).max(axis=1)
    s = amax / 7.0
    assert np.all(np.abs(q) <= 7)
    assert np.all(np.abs(u / s[:, None] - q) <= 0.5 + 1e-5)                  # |u - q s| <= s/2
    idx = np.abs(u).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(M), idx]) == 7)                          # amax element -> +-7
    cg = 1.0 / np.sqrt(wl.g)
    assert np.allclose(sx, s * cg, rtol=2 ** -22)


def test_activation_codes_round_the_fp32_product_ties_to_even():
    # reading of the quantiser: q = rint(fl32(u * fl32(7/amax))), two roundings.
    # u = 1.5 on group 0, amax = 3: fl32(1.5 * fl32(7/3)) is exactly 3.5 (the exact
    # product is 3.49999988), so q = 4 (tie to even), not 3.
    X = np.zeros((2, 32), np.float16)
    X[0, 0], X[0, 8] = 1.5, 3.0
    X[1, 0], X[1, 8] = 2.75, 5.5
    Xq, _ = O.rotate_quant(X, "f16", 8, None)
    q = O.unpack_s4(Xq, 32)
    inv = np.float32(7) / np.float32(3)
    assert np.float32(np.float32(1.5) * inv) == np.float32(3.5)
    assert np.all(q[0, :8] == 4) and np.all(q[0, 8:16] == 7) and np.all(q[0, 16:] == 0)
    assert np.all(q[1, :8] == 4) and np.all(q[1, 8:16] == 7)


def test_activation_zero_row():
    X = np.zeros((2, 256), np.float16)
    X[1, 3] = 1.0
    Xq, sx = O.rotate_quant(X, "f16", 128, None)
    assert sx[0] == 0 and np.all(Xq[0] == 0) and sx[1] > 0


def test_bos_token_sets_a_coarse_step():
    # token 0 is x100 in the tiny workload: its step is about 100x the others'.
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    _, sx = O.rotate_quant(X, wl.xdtype, wl.g, synth.hadamard_signs(wl.g))
    assert sx[0] > 50 * np.median(sx[1:])


def test_rotation_lowers_crest_factor():
    wl = synth.WORKLOADS["decode"]
    X = synth.activations(wl, M=8)
    xf = synth.to_float32(X, wl.xdtype).astype(np.float64)
    u = O.rotate_rows(X, wl.xdtype, wl.g, synth.hadamard_signs(wl.g)).astype(np.float64)
    crest = lambda a: np.abs(a).max(axis=1) / np.sqrt((a ** 2).mean(axis=1))
    assert np.all(crest(u) < crest(xf))


# ----------------------------------------------------------------- weight quantiser
def test_w4_pack_symmetric_round_trip():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    Wq, sw, zw = O.w4_pack(W, "f32", 0)
    assert zw is None and sw.shape == (64,)
    amax = np.abs(W).max(axis=1)
    assert np.array_equal(sw, (amax / np.float32(7)).astype(np.float16))      # numpy's own fp16 rounding
    q = O.unpack_s4(Wq, 512).astype(np.float64)
    s = sw.astype(np.float64)[:, None]
    assert np.all(np.abs(q) <= 7)
    assert np.all(np.abs(W - q * s) <= s / 2 * (1 + 2 ** -20))
    assert np.allclose(O.w4_dequant(Wq, sw, None, 512, 0), q * s, rtol=0, atol=0)


def test_w4_pack_group_asymmetric_round_trip():
    rng = np.random.default_rng(5)
    K, gw = 512, 128
    W = (rng.standard_normal((32, K)) * 0.015).astype(np.float32)
    W[3, :gw] = np.abs(W[3, :gw]) + 0.01             # an all-positive group
    W[4, gw:2 * gw] = 0.0                             # an all-zero group
    Wq, sw, zw = O.w4_pack(W, "f32", gw)
    G = K // gw
    assert sw.shape == (G, 32) and zw.shape == (G, 32)
    z = zw.astype(np.float64)
    assert np.all(z == np.round(z)) and np.all((z >= 0) & (z <= 15))
    q = O.unpack_u4(Wq, K).astype(np.float64)
    s = np.repeat(sw.astype(np.float64).T, gw, axis=1)
    zz = np.repeat(z.T, gw, axis=1)
    err = np.abs(W - (q - zz) * s)
    # half a step, plus the fp16 rounding of the step over a 15-step span
    assert np.all(err <= s * (0.5 + 15 * 2 ** -11 / (1 - 2 ** -11)) * (1 + 2 ** -20))
    Wg = W.reshape(32, G, gw)
    lo = np.minimum(Wg.min(axis=2), 0)
    hi = np.maximum(Wg.max(axis=2), 0)
    span = (hi - lo).astype(np.float32) / np.float32(15)
    expect = np.where(span.astype(np.float16) == 0, np.float16(1), span.astype(np.float16))
    assert np.array_equal(sw, expect.T)
    assert np.all(err[4, gw:2 * gw] == 0)


# ----------------------------------------------------------------- SERQ
def _prepared(name, seed=0, M=None, N=None):
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, seed=seed, M=M)
    W = synth.weights(wl, seed=seed, N=N)
    d = synth.hadamard_signs(wl.g, seed=seed)
    Wrot = O.rotate_normalised(W, wl.wdtype, wl.g, d)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", wl.gw)
    _, sal = O.salient_channels(X, wl.xdtype, wl.g, d, wl.r)
    return wl, X, W, d, Wrot, Wq, sw, zw, sal


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_serq_reduces_error_on_salient_slice(name):
    wl, X, W, d, Wrot, Wq, sw, zw, sal = _prepared(name, N=256 if name == "decode" else None, M=8)
    Rq, sr, E = O.serq_prepare(Wrot, Wq, sw, zw, wl.gw, sal, return_e=True)
    What = O.w4_dequant(Wq, sw, zw, wl.K, wl.gw)
    # E_S is the weight error on the salient columns, W_rot - What
    assert np.array_equal(E, (Wrot - What)[:, sal])
    qr = O.unpack_s4(Rq, wl.r).astype(np.float64)
    Rhat = qr * sr.astype(np.float64)[:, None]
    E = E.astype(np.float64)
    before = np.linalg.norm(E)
    after = np.linalg.norm(E - Rhat)
    assert before > 0 and after < before
    s = sr.astype(np.float64)[:, None]
    elem = np.abs(E - Rhat)
    assert np.all(elem <= np.minimum(np.abs(E), s / 2) * (1 + 2 ** -20) + 1e-30)
    assert np.all(np.abs(qr[np.arange(E.shape[0]), np.abs(E).argmax(axis=1)]) == 7)


def test_serq_full_column_rank_equals_requantising_error():
    # with S = every input channel, R covers the whole error matrix
    wl, X, W, d, Wrot, Wq, sw, zw, _ = _prepared("tiny")
    sal = np.arange(wl.K, dtype=np.int32)
    Rq, sr, E = O.serq_prepare(Wrot, Wq, sw, zw, wl.gw, sal, return_e=True)
    assert np.linalg.norm(E - O.unpack_s4(Rq, wl.K) * sr.astype(np.float64)[:, None]) < 0.2 * np.linalg.norm(E)


# ----------------------------------------------------------------- calibration
def test_salient_channels_are_top_r_norms():
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    d = synth.hadamard_signs(wl.g)
    norm2, sal = O.salient_channels(X, wl.xdtype, wl.g, d, wl.r)
    rot = scipy.linalg.hadamard(wl.g).astype(np.float64) * d[:, None]
    xf = X.astype(np.float64)
    R = np.concatenate([xf[:, b * wl.g:(b + 1) * wl.g] @ rot for b in range(wl.K // wl.g)], axis=1)
    ref = (R ** 2).sum(axis=0)
    assert np.allclose(norm2, ref, rtol=1e-12)
    top = np.sort(np.argsort(-ref, kind="stable")[:wl.r])
    assert np.array_equal(sal, top) and np.all(np.diff(sal) > 0)


# ----------------------------------------------------------------- integer GEMM + epilogue
@pytest.mark.parametrize("gw", [0, 64])
def test_accum_brute_force_matches_numpy_matmul(gw):
    rng = np.random.default_rng(6)
    M, N, K = 5, 7, 256
    qx = rng.integers(-7, 8, (M, K)).astype(np.int8)
    Xq = O.pack_s4(qx)
    if gw:
        qw = rng.integers(0, 16, (N, K)).astype(np.int8)
        Wq = O.pack_s4(qw)  # the nibble bits are what matter; read back unsigned
        qw_u = O.unpack_u4(Wq, K).astype(np.int64)
        z = rng.integers(0, 16, (K // gw, N)).astype(np.float16)
        wv = qw_u - np.repeat(z.astype(np.int64).T, gw, axis=1)
    else:
        qw = rng.integers(-8, 8, (N, K)).astype(np.int8)
        Wq = O.pack_s4(qw)
        z = None
        wv = qw.astype(np.int64)
    sal = np.array([3, 17, 100, 255], np.int32)
    qr = rng.integers(-8, 8, (N, 4)).astype(np.int8)
    Rq = O.pack_s4(qr)
    acc, acc_c = O.accum(Xq, K, Wq, z, gw, Rq, sal)
    G = K // gw if gw else 1
    L = K // G
    for b in range(G):
        ref = qx[:, b * L:(b + 1) * L].astype(np.int64) @ wv[:, b * L:(b + 1) * L].T
        assert np.array_equal(acc[:, :, b], ref)
    assert np.array_equal(acc_c, qx[:, sal].astype(np.int64) @ qr.astype(np.int64).T)


@pytest.mark.parametrize("gw", [0, 128])
def test_accum_extreme_codes_closed_form(gw):
    # every product at its extreme: activation codes -7 against weight values
    # -8 (symmetric codes) or 0 - 15 (asymmetric code 0 with zero point 15);
    # the integer accumulators must equal the closed forms K*56 / 128*105 per
    # group exactly (no wrap-around, no lost term) and fit in int32, and the
    # SERQ term with all codes -8 likewise
    K, N, M = 11008 if gw else 8192, 3, 2
    qx = np.full((M, K), -7, np.int8)
    Xq = O.pack_s4(qx)
    if gw:
        Wq = O.pack_s4(np.zeros((N, K), np.int8))            # unsigned code 0
        z = np.full((K // gw, N), 15.0, np.float16)
        want = 7 * 15 * gw                                     # (-7) * (0 - 15) per element
    else:
        Wq = O.pack_s4(np.full((N, K), -8, np.int8))
        z = None
        want = 56 * K
    sal = np.arange(0, 64, dtype=np.int32) * 7
    Rq = O.pack_s4(np.full((N, 64), -8, np.int8))
    acc, acc_c = O.accum(Xq, K, Wq, z, gw, Rq, sal)
    assert np.all(acc == want) and acc.max() < 2 ** 31
    assert np.all(acc_c == 56 * 64)


def test_w4_pack_zero_point_zero_is_positive_zero():
    # a group whose minimum is 0 has zero point 0, stored as +0 (bits 0x0000),
    # never -0 (0x8000); other zero points are exact small integers
    rng = np.random.default_rng(11)
    K = 256
    W = np.abs(rng.standard_normal((4, K))).astype(np.float32)
    W[:, 0] = 0.0                                   # minimum 0 in group 0 of every row
    W[:, 128:] = -W[:, 128:] - 0.1                  # group 1: all negative -> z = 15
    _, sw, zw = O.w4_pack(W, "f32", 128)
    zb = np.ascontiguousarray(zw).view(np.uint16)
    assert np.all(zb[0] == 0x0000)
    assert np.all(zw[1] == 15.0)


def test_epilogue_against_dequantised_float_matmul():
    wl, X, W, d, Wrot, Wq, sw, zw, sal = _prepared("tiny")
    Xq, sx = O.rotate_quant(X, wl.xdtype, wl.g, d)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, wl.gw, sal)
    acc, acc_c = O.accum(Xq, wl.K, Wq, zw, wl.gw, Rq, sal)
    y = O.epilogue_f64(acc, acc_c, sx, sw, sr)
    # independent formulation: dequantise both operands and multiply (numpy)
    Xhat = O.unpack_s4(Xq, wl.K).astype(np.float64) * sx.astype(np.float64)[:, None]
    What = O.w4_dequant(Wq, sw, zw, wl.K, wl.gw).astype(np.float64)
    Rhat = O.unpack_s4(Rq, wl.r).astype(np.float64) * sr.astype(np.float64)[:, None]
    ref = Xhat @ What.T + Xhat[:, sal] @ Rhat.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = np.array([0, 5, 15])
    assert np.allclose(O.linear_rows_f64(Xq, sx, wl.K, Wq, sw, zw, wl.gw, Rq, sr, sal, rows), y[rows],
                       rtol=1e-13, atol=0)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_quantised_layer_approximates_float_layer(name):
    wl = synth.WORKLOADS[name]
    M, N = (16, 128) if name == "tiny" else (4, 192)
    X = synth.activations(wl, M=M)
    W = synth.weights(wl, N=N)
    d = synth.hadamard_signs(wl.g)
    out = O.layer(X, wl.xdtype, W, wl.wdtype, wl.g, d, wl.gw, wl.r)
    yf = O.linear_fp64(X, wl.xdtype, W, wl.wdtype)
    rel = np.linalg.norm(out["y"] - yf) / np.linalg.norm(yf)
    assert rel < 0.35, rel
    # a sign error or a transposed operand anywhere would give rel ~ 1 or more
    out0 = O.layer(X, wl.xdtype, W, wl.wdtype, wl.g, d, wl.gw, 0)
    rel0 = np.linalg.norm(out0["y"] - yf) / np.linalg.norm(yf)
    assert rel0 < 0.35


# ---------------------------------------------------------------- W4A8 (next row)
# DynamicPTQ, Methodology 2: 8-bit activations on the sensitive layers, weights
# in 4 bit; SERQ section 4 evaluates the same layer at W4A8.  Reading: the same
# rotation and per-token symmetric quantiser with codes in [-127, 127], one
# code per byte.

@pytest.mark.parametrize("name", ["tiny", "attn", "down"])
def test_w4a8_activation_quant_round_trip(name):
    wl = synth.WORKLOADS[name]
    M = 16 if name == "tiny" else 6
    X = synth.activations(wl, M=M)
    d = synth.hadamard_signs(wl.g)
    _, _, u = O.rotate_quant(X, wl.xdtype, wl.g, d, return_u=True)   # the pinned rotation
    q8, sx8 = O.rotate_quant8(X, wl.xdtype, wl.g, d)
    q = q8.astype(np.float64)
    u = u.astype(np.float64)
    amax = np.abs(u).max(axis=1)
    s = amax / 127.0
    assert np.all(np.abs(q) <= 127)
    assert np.all(np.abs(u / s[:, None] - q) <= 0.5 + 1e-4)                  # |u - q s| <= s/2
    idx = np.abs(u).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(M), idx]) == 127)                        # amax element -> +-127
    assert np.allclose(sx8, s / np.sqrt(wl.g), rtol=2 ** -22)
    # 8-bit codes resolve the rotated row 127/7 times finer than the 4-bit ones
    q4 = O.unpack_s4(O.rotate_quant(X, wl.xdtype, wl.g, d)[0], wl.K).astype(np.float64)
    err8 = np.abs(u - q * s[:, None]).max()
    err4 = np.abs(u - q4 * (amax / 7.0)[:, None]).max()
    assert err8 < err4 / 10


def test_w4a8_codes_round_ties_to_even():
    # one channel per group of 8 spreads as a constant over the group; group 1
    # holds 127, so amax = 127, inv = fl32(127/127) = 1 and the codes are
    # rint(u): 2.5 -> 2 and 3.5 -> 4 (ties to even)
    X = np.zeros((2, 16), np.float16)
    X[0, 0], X[0, 8] = 2.5, 127.0
    X[1, 0], X[1, 8] = 3.5, 127.0
    q8, sx8 = O.rotate_quant8(X, "f16", 8, None)
    assert np.all(q8[0, :8] == 2) and np.all(q8[0, 8:] == 127)
    assert np.all(q8[1, :8] == 4) and np.all(q8[1, 8:] == 127)
    assert sx8[0] == np.float32(np.float32(127.0) / np.float32(127.0)) * np.float32(1 / np.sqrt(8))


def test_w4a8_zero_row():
    X = np.zeros((2, 256), np.float16)
    X[1, 3] = 1.0
    q8, sx8 = O.rotate_quant8(X, "f16", 128, None)
    assert sx8[0] == 0 and np.all(q8[0] == 0) and sx8[1] > 0


@pytest.mark.parametrize("gw", [0, 64])
def test_accum8_brute_force_matches_numpy_matmul(gw):
    rng = np.random.default_rng(16)
    M, N, K = 5, 7, 256
    qx = rng.integers(-127, 128, (M, K)).astype(np.int8)
    if gw:
        Wq = O.pack_s4(rng.integers(0, 16, (N, K)).astype(np.int8))
        z = rng.integers(0, 16, (K // gw, N)).astype(np.float16)
        wv = O.unpack_u4(Wq, K).astype(np.int64) - np.repeat(z.astype(np.int64).T, gw, axis=1)
    else:
        qw = rng.integers(-8, 8, (N, K)).astype(np.int8)
        Wq = O.pack_s4(qw)
        z = None
        wv = qw.astype(np.int64)
    sal = np.array([0, 31, 128, 255], np.int32)
    qr = rng.integers(-8, 8, (N, 4)).astype(np.int8)
    acc, acc_c = O.accum8(qx, K, Wq, z, gw, O.pack_s4(qr), sal)
    G = K // gw if gw else 1
    L = K // G
    for b in range(G):
        assert np.array_equal(acc[:, :, b], qx[:, b * L:(b + 1) * L].astype(np.int64) @ wv[:, b * L:(b + 1) * L].T)
    assert np.array_equal(acc_c, qx[:, sal].astype(np.int64) @ qr.astype(np.int64).T)


def test_accum8_int32_worst_case_fits():
    # K (at most 65536) * 127 * 15 (an 8-bit code times an asymmetric weight offset) < 2^31
    assert 65536 * 127 * 15 < 2 ** 31


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_w4a8_layer_against_dequantised_matmul_and_closer_to_float(name):
    wl = synth.WORKLOADS[name]
    M, N = (16, 128) if name == "tiny" else (4, 192)
    wl, X, W, d, Wrot, Wq, sw, zw, sal = _prepared(name, M=M, N=N)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, wl.gw, sal)
    q8, sx8 = O.rotate_quant8(X, wl.xdtype, wl.g, d)
    acc, acc_c = O.accum8(q8, wl.K, Wq, zw, wl.gw, Rq, sal)
    y8 = O.epilogue_f64(acc, acc_c, sx8, sw, sr)
    # independent formulation: dequantise both operands and multiply (numpy)
    Xhat = q8.astype(np.float64) * sx8.astype(np.float64)[:, None]
    What = O.w4_dequant(Wq, sw, zw, wl.K, wl.gw).astype(np.float64)
    Rhat = O.unpack_s4(Rq, wl.r).astype(np.float64) * sr.astype(np.float64)[:, None]
    ref = Xhat @ What.T + Xhat[:, sal] @ Rhat.T
    assert np.allclose(y8, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # 8-bit activations lose less than 4-bit ones against the float layer
    yf = O.linear_fp64(X, wl.xdtype, W, wl.wdtype)
    y4 = O.layer(X, wl.xdtype, W, wl.wdtype, wl.g, d, wl.gw, wl.r)["y"]
    rel8 = np.linalg.norm(y8 - yf) / np.linalg.norm(yf)
    rel4 = np.linalg.norm(y4 - yf) / np.linalg.norm(yf)
    assert rel8 < rel4, (rel8, rel4)


# ----------------------------------------------------------------- OffQ per-group asymmetric activations
# OffQ, Methodology 2 (last point) and 3: the constant offset the all-ones row
# of H creates is absorbed by the zero point of an asymmetric quantiser with one
# scale and zero point per group.

def _asym_setup(seed, M=6, K=512, g=128, outlier=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    if outlier:
        x[0, 0] = 1000.0                           # one concentrated outlier in group 0's first channel
        x[2, g + 0] = -400.0                       # a negative one in group 1
    X = x.astype(np.float16)
    d = synth.hadamard_signs(g, seed=seed)
    return X, d


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_asym_activation_round_trip_and_endpoint_codes(seed):
    g = 128
    X, d = _asym_setup(seed)
    Xq, sx, zx = O.rotate_quant_asym(X, "f16", g, d)
    u = O.rotate_rows(X, "f16", g, d).astype(np.float64)
    q = O.unpack_u4(Xq, X.shape[1]).astype(np.int64)
    M, K = X.shape
    for m in range(M):
        for b in range(K // g):
            ug = u[m, b * g:(b + 1) * g]
            qg = q[m, b * g:(b + 1) * g]
            s = (ug.max() - ug.min()) / 15.0      # the group's own range, in fp64
            rec = s * (qg - zx[m, b])
            # every element within half a step (plus the fp32 rounding of the reciprocal)
            assert np.all(np.abs(rec - ug) <= 0.5 * s * (1 + 1e-5) + 1e-6 * np.abs(ug).max())
            # the ends of the range take the extreme codes
            assert qg.min() == 0 and qg.max() == 15
            # the stored scale is that step times 1/sqrt(g)
            assert abs(sx[m, b] - s / np.sqrt(g)) <= 1e-6 * s / np.sqrt(g)


def test_asym_absorbs_the_rotated_offset():
    # the outlier of row 0 becomes a constant offset of ~1000 over group 0; the
    # per-token symmetric quantiser spends its range on it, the per-group
    # asymmetric one moves it into the zero point
    g = 128
    X, d = _asym_setup(0)
    u = O.rotate_rows(X, "f16", g, d).astype(np.float64)
    assert np.all(u[0, :g] > 900)                  # the offset (OffQ, Methodology 2)
    Xq, sx, zx = O.rotate_quant_asym(X, "f16", g, d)
    qa = O.unpack_u4(Xq, X.shape[1]).astype(np.float64)
    s_a = sx.astype(np.float64) * np.sqrt(g)
    rec_a = s_a[0, 0] * (qa[0, :g] - zx[0, 0])
    Xs, sxs = O.rotate_quant(X, "f16", g, d)
    rec_s = O.unpack_s4(Xs, X.shape[1]).astype(np.float64)[0, :g] * sxs[0] * np.sqrt(g)
    err_a = np.abs(rec_a - u[0, :g]).max()
    err_s = np.abs(rec_s - u[0, :g]).max()
    assert zx[0, 0] < -100                         # the offset sits in the zero point
    assert err_a < err_s / 20


def test_asym_constant_and_zero_groups():
    g = 128
    K = 2 * g
    X = np.zeros((2, K), np.float16)
    X[0, 0] = 3.0                                  # rotated group 0 of row 0: constant 3
    X[1, g] = -5.0                                 # rotated group 1 of row 1: constant -5
    d = synth.hadamard_signs(g, seed=4)
    Xq, sx, zx = O.rotate_quant_asym(X, "f16", g, d)
    q = O.unpack_u4(Xq, K).astype(np.int64)
    s = sx.astype(np.float64) * np.sqrt(g)
    rec = lambda m, b: s[m, b] * (q[m, b * g:(b + 1) * g] - zx[m, b])
    assert np.allclose(rec(0, 0), 3.0, rtol=1e-6) and np.allclose(rec(1, 1), -5.0, rtol=1e-6)
    # all-zero groups: code 0, zero point 0, reconstruction 0
    for m, b in ((0, 1), (1, 0)):
        assert zx[m, b] == 0 and np.all(q[m, b * g:(b + 1) * g] == 0) and np.all(rec(m, b) == 0)


@pytest.mark.parametrize("gw", [0, 128, 256])
def test_accum_asym_matches_numpy(gw):
    rng = np.random.default_rng(11)
    M, N, K, g = 4, 6, 512, 128
    qx = rng.integers(0, 16, (M, K)).astype(np.int8)
    Xq = O.pack_s4(qx)                             # nibble bits; read back unsigned
    zx = rng.integers(-300, 16, (M, K // g)).astype(np.int32)
    if gw:
        Wq = O.pack_s4(rng.integers(0, 16, (N, K)).astype(np.int8))
        z = rng.integers(0, 16, (K // gw, N)).astype(np.float16)
        wv = O.unpack_u4(Wq, K).astype(np.int64) - np.repeat(z.astype(np.int64).T, gw, axis=1)
    else:
        qw = rng.integers(-8, 8, (N, K)).astype(np.int8)
        Wq = O.pack_s4(qw)
        z = None
        wv = qw.astype(np.int64)
    sal = np.array([3, 17, 130, 300, 511], np.int32)
    qr = rng.integers(-8, 8, (N, 5)).astype(np.int8)
    acc, acc_c = O.accum_asym(Xq, zx, K, g, Wq, z, gw, O.pack_s4(qr), sal)
    xv = O.unpack_u4(Xq, K).astype(np.int64) - np.repeat(zx.astype(np.int64), g, axis=1)
    for b in range(K // g):
        sl = slice(b * g, (b + 1) * g)
        assert np.array_equal(acc[:, :, b], xv[:, sl] @ wv[:, sl].T)
        inb = sal // g == b
        assert np.array_equal(acc_c[:, :, b], xv[:, sal[inb]] @ qr[:, inb].astype(np.int64).T)


def test_epilogue_asym_against_dequantised_float_matmul():
    g, gw = 128, 128
    X, d = _asym_setup(5, M=8, K=256)
    rng = np.random.default_rng(12)
    Wrot = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", gw)
    sal = np.array([0, 7, 129, 200], np.int32)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    Xq, sx, zx = O.rotate_quant_asym(X, "f16", g, d)
    acc, acc_c = O.accum_asym(Xq, zx, 256, g, Wq, zw, gw, Rq, sal)
    y = O.epilogue_asym_f64(acc, acc_c, g, gw, sx, sw, sr)
    # independent formulation: dequantise both operands and multiply (numpy)
    Xhat = (O.unpack_u4(Xq, 256).astype(np.float64) - np.repeat(zx, g, axis=1)) * np.repeat(
        sx.astype(np.float64), g, axis=1)
    What = O.w4_dequant(Wq, sw, zw, 256, gw).astype(np.float64)
    Rhat = O.unpack_s4(Rq, len(sal)).astype(np.float64) * sr.astype(np.float64)[:, None]
    ref = Xhat @ What.T + Xhat[:, sal] @ Rhat.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
