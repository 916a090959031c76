"""Pins of the MXFP4 block-quantiser oracle (oracle/mxfp4.py) against what the
format fixes, independent of the oracle's own rounding code: the sixteen codes
decode to the E2M1 values, the round-to-nearest decisions and ties on the grid
written out by hand, the error bound of a nearest-value rounding, the largest
element's landing on 4 or 6, invariance of the codes under power-of-two scaling
of a block, zero blocks, and packing.  Source: "SERQ: Saliency-Aware Low-Rank
Error Reconstruction for LLM Quantization", technical summary sections 2-3
(4-bit paths, INT4 or MXFP4)."""
import numpy as np
import pytest

import oracle.mxfp4 as OM


def test_codes_decode_to_the_e2m1_values():
    vals = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}
    for c in range(16):
        packed = np.array([[c | (c << 4)] * 16], np.uint8)
        d = OM.dequant_mxfp4(packed, np.array([[127]], np.uint8), 32)
        want = (-1.0 if c & 8 else 1.0) * vals[c & 7]
        assert d[0, 0] == want and d[0, 1] == want


@pytest.mark.parametrize("t,code", [
    (0.2, 0), (0.25, 0), (0.3, 1), (0.75, 2), (1.25, 2), (1.3, 3), (1.75, 4), (2.5, 4), (2.6, 5),
    (3.5, 6), (4.9, 6), (5.0, 6), (5.1, 7), (6.0, 7), (7.0, 7), (100.0, 7), (-0.75, 10), (-0.2, 0), (-6.5, 15)])
def test_rounding_and_ties_by_hand(t, code):
    # ties go to 0, 1, 2, 4 (mantissa bit 0); beyond 6 saturates
    assert OM.code_of(t) == code


def test_error_bound_and_largest_element():
    rng = np.random.default_rng(0)
    V = (rng.standard_t(3, size=(16, 256)) * rng.uniform(1e-3, 1e3, size=(16, 1))).astype(np.float32)
    q, sb = OM.quant_mxfp4(V)
    D = OM.dequant_mxfp4(q, sb, 256)
    X = np.ldexp(1.0, np.repeat(sb.astype(np.int64), 32, axis=1) - 127)
    t = np.abs(V.astype(np.float64)) / X
    # grid spacing 0.5 below 2, 1 below 4, 2 above; saturation only above 6
    half = np.where(t < 2, 0.25, np.where(t < 4, 0.5, 1.0))
    err = np.abs(D - V) / X
    assert (err[t <= 6] <= half[t <= 6]).all()
    assert (np.abs(D)[t > 6] == 6 * X[t > 6]).all()
    for m in range(16):
        for b in range(8):
            blk = np.abs(V[m, 32 * b:32 * b + 32])
            k = int(np.argmax(blk))
            assert abs(D[m, 32 * b + k]) / X[m, 32 * b] in (4.0, 6.0)
            amax = float(blk.max())
            assert 4.0 <= amax / X[m, 32 * b] < 8.0


def test_power_of_two_scaling_moves_only_the_scale():
    rng = np.random.default_rng(1)
    V = rng.standard_normal((4, 64)).astype(np.float32)
    q, sb = OM.quant_mxfp4(V)
    for k in (-5, 3, 20):
        q2, sb2 = OM.quant_mxfp4((V * np.float32(2.0 ** k)).astype(np.float32))
        np.testing.assert_array_equal(q2, q)
        np.testing.assert_array_equal(sb2.astype(int), sb.astype(int) + k)


def test_zero_block_and_packing():
    V = np.zeros((2, 64), np.float32)
    V[1, 32:] = np.arange(32, dtype=np.float32) - 16.0
    q, sb = OM.quant_mxfp4(V)
    assert (q[0] == 0).all() and (q[1, :16] == 0).all()
    assert sb[0, 0] == 0 and sb[0, 1] == 0 and sb[1, 0] == 0
    # amax 16 -> E = 2, X = 4: element 2j in the low nibble
    assert sb[1, 1] == 129
    codes = [OM.code_of((j - 16.0) / 4.0) for j in range(32)]
    for j in range(16):
        assert q[1, 16 + j] == codes[2 * j] | (codes[2 * j + 1] << 4)


def test_linear_of_representable_values_is_the_exact_product():
    # values already on the MXFP4 grid quantise to themselves: the product of
    # the codes is the plain matrix product of the inputs
    rng = np.random.default_rng(7)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    def on_grid(rows):
        v = grid[rng.integers(0, 8, size=(rows, 64))] * np.where(rng.random((rows, 64)) < 0.5, -1, 1)
        v[:, 0] = 6.0                        # amax 6 -> E = 0 in block 0
        v[:, 32] = -4.0                      # amax 4 -> E = 0 in block 1
        return (v * np.repeat(np.ldexp(1.0, rng.integers(-6, 6, size=(rows, 2))), 32, axis=1)).astype(np.float32)
    X, W = on_grid(5), on_grid(3)
    qx, sx = OM.quant_mxfp4(X)
    qw, sw = OM.quant_mxfp4(W)
    np.testing.assert_array_equal(OM.dequant_mxfp4(qx, sx, 64), X.astype(np.float64))
    np.testing.assert_array_equal(OM.linear_f64(qx, sx, qw, sw, 64), X.astype(np.float64) @ W.T.astype(np.float64))


def test_linear_brute_force():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((3, 64)).astype(np.float32)
    W = rng.standard_normal((2, 64)).astype(np.float32)
    qx, sx = OM.quant_mxfp4(X)
    qw, sw = OM.quant_mxfp4(W)
    Y = OM.linear_f64(qx, sx, qw, sw, 64)
    for m in range(3):
        for n in range(2):
            acc = 0.0
            for k in range(64):
                cx = (qx[m, k // 2] >> (4 * (k % 2))) & 15
                cw = (qw[n, k // 2] >> (4 * (k % 2))) & 15
                vx = (-1 if cx & 8 else 1) * OM.E2M1[cx & 7] * 2.0 ** (int(sx[m, k // 32]) - 127)
                vw = (-1 if cw & 8 else 1) * OM.E2M1[cw & 7] * 2.0 ** (int(sw[n, k // 32]) - 127)
                acc += vx * vw
            assert Y[m, n] == acc
