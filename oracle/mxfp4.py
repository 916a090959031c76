"""CPU oracle of the MXFP4 block quantiser -- TEST INFRASTRUCTURE.

Only the test suite may import this module.  Plain numpy (float64 holds every
value exactly); it shares nothing with the CUDA library.

Source: "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
Quantization", technical summary section 2 (the main and the residual path
both stay in 4 bit, INT4 or MXFP4) and section 3 (MXFP4 runs natively on
Blackwell tensor cores).  The pages do not define MXFP4; the plain reading is
the Open Compute Project microscaling format: blocks of 32 consecutive values
share one power-of-two scale stored as an 8-bit biased exponent (UE8M0), and
each value is a 4-bit E2M1 float (sign, 2 exponent bits, 1 mantissa bit:
magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).

Readings where the format leaves a choice:

* shared exponent E = floor(log2(amax)) - 2 (2 = the exponent of E2M1's
  largest magnitude 6), stored as the byte E + 127 clamped to [0, 254]; an
  all-zero block stores byte 0 and zero codes;
* element codes: t = v / 2^E rounded to the E2M1 grid to nearest, ties to the
  grid value whose mantissa bit is 0 (0, 1, 2, 4 against 0.5, 1.5, 3, 6), and
  magnitudes above 6 saturate to 6;
* the sign bit is set only for t < 0 with a non-zero rounded magnitude (a
  value that rounds to zero is stored as +0);
* codes are packed two per byte, element 2j in the low nibble of byte j.
"""
import math

import numpy as np

# E2M1 magnitude of each 3-bit code
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def block_exponent(amax):
    """floor(log2(amax)) - 2 for amax > 0 (exact, through frexp)."""
    m, e = math.frexp(float(amax))          # amax = m 2^e, m in [0.5, 1)
    return e - 1 - 2


def round_e2m1(t):
    """Magnitude of t rounded to the E2M1 grid (ties to the even mantissa),
    saturating at 6; t is a float64 value."""
    a = abs(t)
    if a < 2.0:
        r = np.rint(2.0 * a) / 2.0           # steps of 0.5; rint ties to even
    elif a < 4.0:
        r = float(np.rint(a))                # steps of 1
    else:
        r = min(2.0 * float(np.rint(a / 2.0)), 6.0)   # steps of 2, saturated
    return float(r)


def code_of(t):
    """4-bit code of t: sign bit 3 (t < 0), magnitude code bits 0-2."""
    r = round_e2m1(t)
    mag = int(np.nonzero(E2M1 == r)[0][0])
    return (8 if t < 0 and r != 0.0 else 0) | mag


def quant_mxfp4(V):
    """V: float32 [M, K] with K % 32 == 0 -> (codes uint8 [M, K/2],
    scale bytes uint8 [M, K/32]).  Plain loops over blocks and elements."""
    V = np.asarray(V, np.float32)
    M, K = V.shape
    assert K % 32 == 0
    q = np.zeros((M, K), np.uint8)
    sb = np.zeros((M, K // 32), np.uint8)
    for m in range(M):
        for b in range(K // 32):
            blk = V[m, 32 * b:32 * b + 32].astype(np.float64)
            amax = float(np.max(np.abs(blk)))
            if amax == 0.0:
                continue                     # byte 0, codes 0
            E = block_exponent(amax)
            byte = min(max(E + 127, 0), 254)
            sb[m, b] = byte
            X = math.ldexp(1.0, byte - 127)
            for i in range(32):
                q[m, 32 * b + i] = code_of(blk[i] / X)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb


def dequant_mxfp4(packed, sb, K):
    """Values the codes stand for: sign * E2M1[mag] * 2^(byte - 127)."""
    packed = np.asarray(packed, np.uint8)
    M = packed.shape[0]
    q = np.zeros((M, K), np.uint8)
    q[:, 0::2] = packed & 0xF
    q[:, 1::2] = packed >> 4
    mag = E2M1[q & 7]
    sign = np.where(q & 8, -1.0, 1.0)
    X = np.ldexp(1.0, np.repeat(np.asarray(sb, np.int64), 32, axis=1) - 127)
    return sign * mag * X


def linear_f64(qx, sbx, qw, sbw, K):
    """Y = X^ W^T in float64 with X^, W^ the values the MXFP4 codes stand for
    (every product and sum is exact in float64 for these magnitudes)."""
    return dequant_mxfp4(qx, sbx, K) @ dequant_mxfp4(qw, sbw, K).T
