"""GPU parity of OffQ's per-group asymmetric activations ("OffQ ...",
Methodology 2, last point, and Methodology 3) against the CPU oracle, through
the C ABI: the quantiser's codes, scales and integer zero points and the small-M
GEMM's integer accumulators per activation group match bit for bit; the float
output lies within the W4A4 tests' tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_bit_gemm_hq_b200 import synth

pytestmark = pytest.mark.gpu

hq = pytest.importorskip("w4a4_bit_gemm_hq_b200.hq") if torch.cuda.is_available() else None

from test_gpu_parity import _dev_inputs, assert_same, assert_y_close, dev, host, no_device_error, y_host  # noqa: E402


def _rows(M, K, g, seed, xdtype):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4, size=(M, K)).astype(np.float32)
    x[0, 0] = 1000.0                         # rotated into an offset over group 0 (z < 0)
    if M > 1:
        x[1, g] = -400.0                     # a negative offset over group 1 (z > 15)
    if M > 2:
        x[2] = 0.0                           # zero groups
        x[2, 0] = 3.0                        # a constant group
    if M > 3:
        x[3, :g] = 0.125                     # a group whose rotation is one spike (|first| = g / 8)
    if M > 4:
        x[4] = 0.0                           # a tiny spread on a large offset: |u / step| >= 2^22
        x[4, 0] = 1000.0
        x[4, 5] = 2.0 ** -10
    return synth.f32_to_bf16_bits(x) if xdtype == "bf16" else x.astype(np.float16)


@pytest.mark.parametrize("g", [32, 128, 1024])
@pytest.mark.parametrize("M", [1, 5, 300])
@pytest.mark.parametrize("xdtype", ["f16", "bf16"])
def test_rotate_quant_asym_bit_exact(g, M, xdtype):
    K = 2048
    X = _rows(M, K, g, seed=g + M, xdtype=xdtype)
    d = synth.hadamard_signs(g, seed=g)
    Xq_o, sx_o, zx_o = O.rotate_quant_asym(X, xdtype, g, d)
    Xq, sx, zx = hq.hq_rotate_quant_asym(dev(X, xdtype), g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    assert_same(host(zx), zx_o, "zero points")
    no_device_error()


@pytest.mark.parametrize("name,M", [("decode", 100), ("down", 200), ("down", 16)])
@pytest.mark.parametrize("signed", [True, False])
def test_rotate_quant_asym_workloads(name, M, signed):
    # more than 64 rows of a group-128 layer run the streaming kernel (teams
    # of one warp at K = 4096, of three at K = 11008); 16 rows the per-row one
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    d = synth.hadamard_signs(wl.g) if signed else None
    Xq_o, sx_o, zx_o = O.rotate_quant_asym(X, wl.xdtype, wl.g, d)
    Xq, sx, zx = hq.hq_rotate_quant_asym(dev(X, wl.xdtype), wl.g, None if d is None else torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    assert_same(host(zx), zx_o, "zero points")
    no_device_error()


def test_rotate_quant_asym_decode_workload_and_strided_rows():
    wl = synth.WORKLOADS["decode"]
    X = synth.activations(wl, M=16)
    d = synth.hadamard_signs(wl.g)
    Xq_o, sx_o, zx_o = O.rotate_quant_asym(X, wl.xdtype, wl.g, d)
    # rows 64 channels apart in memory (ld_x > K)
    Xp = np.zeros((16, wl.K + 64), np.float16)
    Xp[:, :wl.K] = X
    Xd = dev(Xp, wl.xdtype)[:, :wl.K]
    Xq, sx, zx = hq.hq_rotate_quant_asym(Xd, wl.g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    assert_same(host(zx), zx_o, "zero points")
    no_device_error()


# ------------------------------------------------------------------ OffQ GEMM (small M)
def _inputs_asym(M, N, K, gw, r, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    if M:
        x[:, 5] *= 40
        x[0, 128] = 900.0                    # a group whose rotation sits on one side of 0
    X = x.astype(np.float16)
    Xq, sx, zx = O.rotate_quant_asym(X, "f16", 128, None)
    Wrot = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", gw)
    sal = np.sort(rng.choice(K, r, replace=False)).astype(np.int32)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    t = dict(Xq=Xq, sx=sx, zx=zx, Wq=Wq, sw=sw, zw=zw, sal=sal, Rq=Rq, sr=sr)
    g = _dev_inputs(t)
    g["zx"] = torch.from_numpy(zx).cuda()
    return t, g


OFFQ_CASES = [
    # M, N, K, gw, r   (token counts of each small-M tile width, ragged N)
    (1, 256, 256, 0, 0),
    (5, 264, 512, 128, 8),
    (16, 1024, 2048, 128, 16),
    (33, 264, 512, 0, 24),
    (64, 1032, 1024, 256, 64),
    (8, 512, 4096, 2048, 32),
    # more than 64 tokens: 64-row slices, the last one ragged
    (65, 264, 512, 128, 8),
    (200, 520, 1024, 0, 32),
]


@pytest.mark.parametrize("M,N,K,gw,r", OFFQ_CASES)
def test_offq_accumulators_bit_exact(M, N, K, gw, r):
    t, g = _inputs_asym(M, N, K, gw, r, seed=M + N)
    acc_o, _ = O.accum_asym(t["Xq"], t["zx"], K, 128, t["Wq"], t["zw"], gw)
    acc = hq.hq_debug_accum_asym(g["Xq"], g["zx"], g["Wq"], g["zw"], gw, N)
    assert_same(host(acc).astype(np.int64), acc_o, "acc")
    no_device_error()


@pytest.mark.parametrize("M,N,K,gw,r", OFFQ_CASES)
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_offq_linear_within_tolerance(M, N, K, gw, r, out):
    t, g = _inputs_asym(M, N, K, gw, r, seed=M + 3 * N)
    acc_o, accc_o = O.accum_asym(t["Xq"], t["zx"], K, 128, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    y64 = O.epilogue_asym_f64(acc_o, accc_o, 128, gw, t["sx"], t["sw"], t["sr"] if r else None)
    Y = hq.w4a4_linear_asym(g["Xq"], g["sx"], g["zx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"],
                            out)
    assert_y_close(y_host(Y), y64, 1e-3 if out == torch.float32 else 1e-2)
    Y2 = hq.w4a4_linear_asym(g["Xq"], g["sx"], g["zx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"],
                             g["sal"], out)
    assert torch.equal(Y, Y2)
    no_device_error()


@pytest.mark.parametrize("name,M,N", [("decode", 16, 1024), ("down", 130, 256)])
def test_offq_layer_end_to_end_from_raw_inputs(name, M, N):
    # the layer from raw activations and weights (N cut down): OffQ quantiser,
    # then the OffQ GEMM, through the layer class and through the two calls
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    W = synth.weights(wl, N=N)
    d = synth.hadamard_signs(wl.g)
    Wrot = O.rotate_normalised(W, wl.wdtype, wl.g, d)
    Wq_o, sw_o, zw_o = O.w4_pack(Wrot, "f32", wl.gw)
    _, sal = O.salient_channels(X, wl.xdtype, wl.g, d, wl.r)
    Rq_o, sr_o = O.serq_prepare(Wrot, Wq_o, sw_o, zw_o, wl.gw, sal)
    Xq_o, sx_o, zx_o = O.rotate_quant_asym(X, wl.xdtype, wl.g, d)
    acc_o, accc_o = O.accum_asym(Xq_o, zx_o, wl.K, wl.g, Wq_o, zw_o, wl.gw, Rq_o, sal)
    y64 = O.epilogue_asym_f64(acc_o, accc_o, wl.g, wl.gw, sx_o, sw_o, sr_o)
    out_dt = torch.float16 if wl.xdtype == "f16" else torch.bfloat16
    layer = hq.W4A4Linear.prepare(dev(W, wl.wdtype), wl.g, wl.gw, wl.r, torch.from_numpy(d).cuda(),
                                  sal_idx=torch.from_numpy(sal), out_dtype=out_dt, offq=True)
    Y = layer(dev(X, wl.xdtype))
    assert_y_close(y_host(Y), y64, 1e-2)
    Xq, sx, zx = hq.hq_rotate_quant_asym(dev(X, wl.xdtype), wl.g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    gi = _dev_inputs(dict(Xq=Xq_o, sx=sx_o, Wq=Wq_o, sw=sw_o, zw=zw_o, sal=sal, Rq=Rq_o, sr=sr_o))
    Y2 = hq.w4a4_linear_asym(Xq, sx, zx, gi["Wq"], gi["sw"], gi["zw"], wl.gw, gi["Rq"], gi["sr"], gi["sal"], out_dt)
    assert torch.equal(Y, Y2)
    no_device_error()
