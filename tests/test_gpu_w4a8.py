"""GPU parity of the W4A8 path (8-bit activations; "DynamicPTQ", Methodology 2;
"SERQ ...", section 4) against the CPU oracle, through the C ABI.

hq_rotate_quant8's codes and scales and the integer accumulators of
w4a8_linear's two GEMM kernels must match the oracle bit for bit; the float
output must lie within the tolerance of the W4A4 tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_bit_gemm_hq_b200 import synth

pytestmark = pytest.mark.gpu

hq = pytest.importorskip("w4a4_bit_gemm_hq_b200.hq") if torch.cuda.is_available() else None

from test_gpu_parity import (_dev_inputs, assert_same, assert_y_close, dev, host,  # noqa: E402
                             no_device_error, tile_wq, untile_wq, y_host)


# ------------------------------------------------------------------ 8-bit rotate/quant
@pytest.mark.parametrize("name,M", [("tiny", 16), ("decode", 4), ("attn", 48), ("attn", 300), ("down", 24),
                                    ("down", 200), ("large", 130)])
def test_rotate_quant8_bit_exact_workloads(name, M):
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    d = synth.hadamard_signs(wl.g)
    Xq_o, sx_o = O.rotate_quant8(X, wl.xdtype, wl.g, d)
    Xq, sx = hq.hq_rotate_quant8(dev(X, wl.xdtype), wl.g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    no_device_error()


@pytest.mark.parametrize("g", [8, 128, 256, 1024, 4096])
@pytest.mark.parametrize("M", [5, 700])
def test_rotate_quant8_group_sweep(g, M):
    # M = 5 runs the per-row kernel, M = 700 the streaming one; ties of
    # fl32(u * inv) on x.5 are frequent with 127 levels
    rng = np.random.default_rng(g + M)
    K = 8192
    x = (rng.standard_t(4, size=(M, K)) * 2).astype(np.float32)
    x[1 % M, 7] = 500.0
    X = synth.f32_to_bf16_bits(x)
    d = synth.hadamard_signs(g, seed=g)
    Xq_o, sx_o = O.rotate_quant8(X, "bf16", g, d)
    Xq, sx = hq.hq_rotate_quant8(dev(X, "bf16"), g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")


# ------------------------------------------------------------------ W4A8 GEMM
def _inputs8(M, N, K, gw, r, seed):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((M, K)) * 2).astype(np.float16)
    if M:
        X[:, 5] *= 40
    Wrot = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Xq8, sx = O.rotate_quant8(X, "f16", 128, None)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", gw)
    sal = np.sort(rng.choice(K, r, replace=False)).astype(np.int32)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    t = dict(Xq=np.zeros((M, K // 2), np.uint8), sx=sx, Wq=Wq, sw=sw, zw=zw, sal=sal, Rq=Rq, sr=sr)
    g = _dev_inputs(t)
    g["Xq8"] = torch.from_numpy(Xq8).cuda()
    return Xq8, t, g


W4A8_CASES = [
    # M, N, K, gw, r     (M <= 64: small-M kernel; larger: CTA-pair kernel)
    (16, 128, 256, 0, 8),
    (1, 256, 256, 0, 0),
    (4, 1024, 2048, 128, 16),
    (33, 264, 512, 0, 24),
    (64, 1032, 1024, 256, 64),
    (200, 264, 512, 0, 16),
    (130, 136, 1024, 128, 32),
    (300, 512, 2048, 256, 64),
    (256, 512, 1024, 0, 40),
]


@pytest.mark.parametrize("M,N,K,gw,r", W4A8_CASES)
def test_w4a8_accumulators_bit_exact(M, N, K, gw, r):
    Xq8, t, g = _inputs8(M, N, K, gw, r, seed=M + N)
    acc_o, accc_o = O.accum8(Xq8, K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    for decode in ([False, True] if M <= 64 else [False]):
        acc, acc_c = hq.hq_debug_accum8(g["Xq8"], g["Wq"], g["zw"], gw, g["Rq"], g["sal"], N, decode=decode)
        assert_same(host(acc).astype(np.int64), acc_o, "acc")
        if r:
            assert_same(host(acc_c).astype(np.int64), accc_o, "acc_c")
    no_device_error()


@pytest.mark.parametrize("M,N,K,gw,r", W4A8_CASES)
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_w4a8_linear_within_tolerance(M, N, K, gw, r, out):
    Xq8, t, g = _inputs8(M, N, K, gw, r, seed=M + 3 * N)
    acc_o, accc_o = O.accum8(Xq8, K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    y64 = O.epilogue_f64(acc_o, accc_o, t["sx"], t["sw"], t["sr"] if r else None)
    Y = hq.w4a8_linear(g["Xq8"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], out)
    assert_y_close(y_host(Y), y64, 1e-3 if out == torch.float32 else 1e-2)
    Y2 = hq.w4a8_linear(g["Xq8"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], out)
    assert torch.equal(Y, Y2)
    no_device_error()


@pytest.mark.parametrize("name,M,N", [("decode", 16, 512), ("down", 96, 256), ("attn", 80, 256), ("large", 16, 256)])
def test_w4a8_layer_end_to_end_from_raw_inputs(name, M, N):
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    W = synth.weights(wl, N=N)
    d = synth.hadamard_signs(wl.g)
    Wrot = O.rotate_normalised(W, wl.wdtype, wl.g, d)
    Wq_o, sw_o, zw_o = O.w4_pack(Wrot, "f32", wl.gw)
    _, sal = O.salient_channels(X, wl.xdtype, wl.g, d, wl.r)
    Rq_o, sr_o = O.serq_prepare(Wrot, Wq_o, sw_o, zw_o, wl.gw, sal)
    Xq8_o, sx_o = O.rotate_quant8(X, wl.xdtype, wl.g, d)
    acc_o, accc_o = O.accum8(Xq8_o, wl.K, Wq_o, zw_o, wl.gw, Rq_o, sal)
    y64 = O.epilogue_f64(acc_o, accc_o, sx_o, sw_o, sr_o)
    out_dt = torch.float16 if wl.xdtype == "f16" else torch.bfloat16
    layer = hq.W4A4Linear.prepare(dev(W, wl.wdtype), wl.g, wl.gw, wl.r, torch.from_numpy(d).cuda(),
                                  sal_idx=torch.from_numpy(sal), out_dtype=out_dt, act_bits=8)
    Y = layer(dev(X, wl.xdtype))
    assert_y_close(y_host(Y), y64, 1e-2)
    no_device_error()
