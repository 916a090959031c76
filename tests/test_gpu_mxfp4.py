"""GPU parity of the MXFP4 block quantiser (hq_quant_mxfp4) against the CPU
oracle (oracle/mxfp4.py), through the C ABI: codes and scale bytes bit for
bit, on rotated activations of the workloads (hq_rotate output, fp32), on raw
16-bit rows, on fp32 weight rows with a stride, and on blocks built on the
grid's ties, on zero, tiny and large blocks.  Source: "SERQ: Saliency-Aware
Low-Rank Error Reconstruction for LLM Quantization", technical summary
sections 2-3 (4-bit paths, INT4 or MXFP4)."""
import numpy as np
import pytest
import torch

import oracle.mxfp4 as OM
from w4a4_bit_gemm_hq_b200 import synth

pytestmark = pytest.mark.gpu

hq = pytest.importorskip("w4a4_bit_gemm_hq_b200.hq") if torch.cuda.is_available() else None

from test_gpu_parity import assert_same, dev, host, no_device_error  # noqa: E402


@pytest.mark.parametrize("name,M", [("tiny", 16), ("decode", 4), ("attn", 8), ("down", 6)])
def test_rotated_activations_bit_exact(name, M):
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    d = torch.from_numpy(synth.hadamard_signs(wl.g)).cuda()
    V = hq.hq_rotate(dev(X, wl.xdtype), wl.g, d)            # fp32 rows, the rotation normalised
    q, sb = hq.hq_quant_mxfp4(V)
    q_o, sb_o = OM.quant_mxfp4(host(V))
    assert_same(host(sb), sb_o, "scale bytes")
    assert_same(host(q), q_o, "codes")
    no_device_error()


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_raw_16bit_rows(dt):
    rng = np.random.default_rng(5)
    Xf = (rng.standard_t(3, size=(24, 512)) * 3).astype(np.float32)
    X = synth.f32_to_bf16_bits(Xf) if dt == "bf16" else Xf.astype(np.float16)
    q, sb = hq.hq_quant_mxfp4(dev(X, dt))
    Xw = synth.to_float32(X, dt) if dt == "bf16" else X.astype(np.float32)
    q_o, sb_o = OM.quant_mxfp4(Xw)
    assert_same(host(sb), sb_o, "scale bytes")
    assert_same(host(q), q_o, "codes")


def test_weight_rows_with_stride_ties_and_extremes():
    rng = np.random.default_rng(6)
    K = 256
    W = (rng.standard_normal((10, K)) * 0.02).astype(np.float32)
    # row 0: every grid tie and midpoint at scale 2^-3 (amax 0.9 -> E = -3)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 0.3, 1.3, 2.6, 5.1, 6.0, 0.2, -0.75, -5.0],
                    np.float32)
    W[0, :32] = np.concatenate([ties, -ties]) * np.float32(0.125)
    W[0, 7] = np.float32(7.2 * 0.125)       # amax of the block: 0.9 -> E = -3
    W[1, :32] = 0.0                          # zero block
    W[2, :32] = np.float32(1e-40)            # subnormal block: clamped exponent
    W[3, :32] = np.float32(3e38)             # near the top of the range
    W[4, 32:64] = -0.0
    Wp = np.concatenate([W, np.zeros((10, 16), np.float32)], axis=1)
    Wd = torch.from_numpy(Wp).cuda()[:, :K]
    q, sb = hq.hq_quant_mxfp4(Wd)
    q_o, sb_o = OM.quant_mxfp4(W)
    assert_same(host(sb), sb_o, "scale bytes")
    assert_same(host(q), q_o, "codes")
    assert host(sb)[1, 0] == 0 and (host(q)[1, :16] == 0).all()
    no_device_error()


def test_argument_errors():
    lib, E = hq._lib.lib, hq._lib
    X = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    q = torch.zeros((4, 32), dtype=torch.uint8, device="cuda")
    s = torch.zeros((4, 2), dtype=torch.uint8, device="cuda")
    p = lambda t: t.data_ptr()
    assert lib.hq_quant_mxfp4(p(X), 2, 4, 48, 64, p(q), p(s), None) == E.HQ_ERR_ARG       # K % 32
    assert lib.hq_quant_mxfp4(p(X), 2, 4, 64, 32, p(q), p(s), None) == E.HQ_ERR_ARG       # ld_x < K
    assert lib.hq_quant_mxfp4(p(X) + 4, 2, 4, 64, 64, p(q), p(s), None) == E.HQ_ERR_ALIGN
    assert lib.hq_quant_mxfp4(p(X), 2, 4, 64, 66, p(q), p(s), None) == E.HQ_ERR_ALIGN     # stride 264 bytes
    assert lib.hq_quant_mxfp4(p(X), 2, 0, 64, 64, None, None, None) == E.HQ_OK
    no_device_error()


def _bound(qx, sx, qw, sw, K):
    """fp32 accumulation of K/32 exact block sums: |err| <= (K/32) 2^-24 sum |x^ w^|."""
    ax = np.abs(OM.dequant_mxfp4(qx, sx, K))
    aw = np.abs(OM.dequant_mxfp4(qw, sw, K))
    return (K // 32) * 2.0 ** -24 * (ax @ aw.T)


@pytest.mark.parametrize("M,N,K", [(16, 8, 32), (33, 70, 256), (100, 130, 1024), (7, 2048, 4096)])
def test_mxfp4_linear_within_accumulation_bound(M, N, K):
    rng = np.random.default_rng(M + N)
    X = (rng.standard_t(3, size=(M, K)) * 2).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qx, sx = hq.hq_quant_mxfp4(torch.from_numpy(X).cuda())
    qw, sw = hq.hq_quant_mxfp4(torch.from_numpy(W).cuda())
    Y = host(hq.hq_mxfp4_linear(qx, sx, qw, sw)).astype(np.float64)
    hqx, hsx, hqw, hsw = host(qx), host(sx), host(qw), host(sw)
    Y64 = OM.linear_f64(hqx, hsx, hqw, hsw, K)
    assert (np.abs(Y - Y64) <= _bound(hqx, hsx, hqw, hsw, K)).all()
    no_device_error()


def test_mxfp4_layer_with_residual_term_on_the_down_shape():
    # main product over K = 11008 plus SERQ's residual path on 32 salient
    # channels (one MXFP4 block), the second call accumulating into the first
    wl = synth.WORKLOADS["down"]
    M, N, K, r = 64, 512, wl.K, 32
    X = synth.activations(wl, M=M)
    d = torch.from_numpy(synth.hadamard_signs(wl.g)).cuda()
    V = hq.hq_rotate(dev(X, wl.xdtype), wl.g, d)
    W = (np.random.default_rng(3).standard_normal((N, K)) * 0.015).astype(np.float32)
    sal = np.sort(np.random.default_rng(4).choice(K, r, replace=False))
    R = (np.random.default_rng(5).standard_normal((N, r)) * 0.003).astype(np.float32)
    qx, sx = hq.hq_quant_mxfp4(V)
    qw, sw = hq.hq_quant_mxfp4(torch.from_numpy(W).cuda())
    Vs = V[:, torch.from_numpy(sal).cuda()].contiguous()
    qs, ss = hq.hq_quant_mxfp4(Vs)
    qr, sr = hq.hq_quant_mxfp4(torch.from_numpy(R).cuda())
    Y = hq.hq_mxfp4_linear(qx, sx, qw, sw)
    Y = host(hq.hq_mxfp4_linear(qs, ss, qr, sr, Y=Y, accumulate=True)).astype(np.float64)
    h = [host(t) for t in (qx, sx, qw, sw, qs, ss, qr, sr)]
    Y64 = OM.linear_f64(h[0], h[1], h[2], h[3], K) + OM.linear_f64(h[4], h[5], h[6], h[7], r)
    bound = _bound(h[0], h[1], h[2], h[3], K) + _bound(h[4], h[5], h[6], h[7], r) + 2.0 ** -24 * np.abs(Y64)
    assert (np.abs(Y - Y64) <= bound).all()
    # and the codes of the gathered salient block are the oracle's
    q_o, s_o = OM.quant_mxfp4(host(Vs))
    assert_same(h[4], q_o, "salient codes")
    assert_same(h[5], s_o, "salient scale bytes")
    no_device_error()
