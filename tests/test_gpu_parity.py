"""GPU parity: every CUDA stage against the CPU oracle on the same seeded inputs.

Integer / byte results (packed codes, fp16 scale bit patterns, fp32 activation
scales, int32 accumulators) must match bit for bit.  The float output Y must
match the oracle's fp64 ground truth elementwise within
    |y - y64| <= tol * max(|y64|, 1e-3 * max|y64|)
with tol = 1e-2 for fp16 / bf16 outputs and 1e-3 for fp32 outputs (the
tolerance the layer is specified to, with a floor for outputs near zero).
All calls go through the C ABI (libhq.so).
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_bit_gemm_hq_b200 import synth

pytestmark = pytest.mark.gpu

hq = pytest.importorskip("w4a4_bit_gemm_hq_b200.hq") if torch.cuda.is_available() else None


def dev(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    if dtype == "f16":
        return torch.from_numpy(np.ascontiguousarray(x, np.float16)).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def host(t):
    torch.cuda.synchronize()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def f16bits(a):
    return np.ascontiguousarray(a).view(np.uint16)


def assert_same(a, b, what="values"):
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.dtype.itemsize == 4 and a.dtype.kind == "f":
        a, b = a.view(np.uint32), b.view(np.uint32)
    bad = a != b
    assert not bad.any(), "%s: %d of %d differ, first at %s" % (what, bad.sum(), bad.size, np.argwhere(bad)[:4])


def assert_y_close(y, y64, tol):
    y = y.astype(np.float64)
    ref = np.abs(y64)
    floor = 1e-3 * ref.max() if ref.size else 0.0
    err = np.abs(y - y64)
    bad = err > tol * np.maximum(ref, floor)
    assert not bad.any(), "max rel err %.3g at %s" % ((err / np.maximum(ref, floor)).max(), np.argwhere(bad)[:5])


def y_host(Y):
    y = host(Y)
    if Y.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f32(y)
    return y.astype(np.float32)


def tile_wq(Wq_rows):
    """Row-major packed weights -> the C ABI's tile-major layout (marshalling)."""
    N, Kh = Wq_rows.shape
    T = (N + 127) // 128
    pad = np.zeros((T * 128, Kh), np.uint8)
    pad[:N] = Wq_rows
    return np.ascontiguousarray(pad.reshape(T, 128, Kh // 64, 64).transpose(0, 2, 1, 3))


def untile_wq(Wq, N):
    Wq = np.asarray(Wq)
    T, KB = Wq.shape[0], Wq.shape[1]
    return np.ascontiguousarray(Wq.transpose(0, 2, 1, 3).reshape(T * 128, KB * 64)[:N])


def no_device_error():
    assert hq.hq_last_device_status() == 0


# ------------------------------------------------------------------ K1: rotate + quant
ROT_CASES = [
    ("tiny", 16, None),
    ("decode", 1, None),
    ("decode", 4, None),
    ("decode", 16, None),
    ("attn", 48, None),
    ("down", 24, None),
    ("large", 12, None),
    ("attn", 200, None),
    ("down", 130, None),
    ("large", 100, None),
]


@pytest.mark.parametrize("name,M,_", ROT_CASES)
def test_rotate_quant_bit_exact_workloads(name, M, _):
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    d = synth.hadamard_signs(wl.g)
    Xq_o, sx_o = O.rotate_quant(X, wl.xdtype, wl.g, d)
    Xq, sx = hq.hq_rotate_quant(dev(X, wl.xdtype), wl.g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    no_device_error()


@pytest.mark.parametrize("g", [8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_rotate_quant_bit_exact_group_sweep(g, dtype):
    rng = np.random.default_rng(g)
    M, K = 7, 8192
    x = (rng.standard_t(4, size=(M, K)) * 2).astype(np.float32)
    x[2, 5] = 300.0
    X = x.astype(np.float16) if dtype == "f16" else synth.f32_to_bf16_bits(x)
    d = synth.hadamard_signs(g, seed=g)
    Xq_o, sx_o = O.rotate_quant(X, dtype, g, d)
    Xq, sx = hq.hq_rotate_quant(dev(X, dtype), g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    # H = None means d = 1
    Xq_o, sx_o = O.rotate_quant(X, dtype, g, None)
    Xq, sx = hq.hq_rotate_quant(dev(X, dtype), g, None)
    assert np.array_equal(host(Xq), Xq_o) and np.array_equal(host(sx), sx_o)


def test_rotate_quant_rounding_ties_follow_the_definition():
    # fl32(u * inv) lands exactly on x.5 while the exact product does not: a
    # fused multiply-add would round the other way
    X = np.zeros((3, 32), np.float16)
    X[0, 0], X[0, 8] = 1.5, 3.0
    X[1, 0], X[1, 8] = 2.75, 5.5
    X[2, 0], X[2, 8] = 5.5, 11.0
    Xq_o, sx_o = O.rotate_quant(X, "f16", 8, None)
    Xq, sx = hq.hq_rotate_quant(dev(X, "f16"), 8, None)
    assert_same(host(Xq), Xq_o, "codes")
    assert np.all(O.unpack_s4(host(Xq), 32)[:, :8] == 4)


def test_rotate_quant_edge_rows_and_strides():
    g, K = 128, 512
    X = np.zeros((5, K), np.float16)
    X[1, 0] = 37.25                          # offset case: all codes of group 0 are +7
    X[2, :] = np.float16(1e-3)
    X[3, 300] = -2.0
    X[4, :] = np.linspace(-5, 5, K).astype(np.float16)
    d = synth.hadamard_signs(g)
    Xq_o, sx_o = O.rotate_quant(X, "f16", g, d)
    big = torch.zeros((5, K + 64), dtype=torch.float16, device="cuda")
    big[:, :K] = dev(X, "f16")
    Xq, sx = hq.hq_rotate_quant(big[:, :K], g, torch.from_numpy(d).cuda())   # ld_x = K + 64
    assert np.array_equal(host(Xq), Xq_o) and np.array_equal(host(sx), sx_o)
    assert sx_o[0] == 0 and np.all(Xq_o[0] == 0)
    assert np.all(O.unpack_s4(host(Xq), K)[1, :g] == 7)
    Xq0, sx0 = hq.hq_rotate_quant(big[:0, :K], g, None)       # M == 0
    assert Xq0.shape == (0, K // 2)


@pytest.mark.parametrize("K,g,dtype", [(11008, 128, "bf16"), (8192, 256, "bf16"), (4096, 4096, "bf16"),
                                     (4096, 128, "f16"), (16384, 512, "f16"), (1152, 64, "bf16"), (3072, 1024, "f16")])
def test_rotate_quant_many_rows_per_team(K, g, dtype):
    # more rows than row teams on the device: every team of the streaming kernel
    # walks several rows through its two shared-memory slots; K covers teams of
    # 1 to 4 warps (and a partly idle last warp for 11008 = 86 x 128 channels)
    rng = np.random.default_rng(K + g)
    M = 2500
    x = rng.standard_t(3, size=(M, K)).astype(np.float32)
    x[::97, 3] = 400.0
    x[5] = 0.0
    X = x.astype(np.float16) if dtype == "f16" else synth.f32_to_bf16_bits(x)
    d = synth.hadamard_signs(g, seed=K)
    Xq_o, sx_o = O.rotate_quant(X, dtype, g, d)
    Xq, sx = hq.hq_rotate_quant(dev(X, dtype), g, torch.from_numpy(d).cuda())
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    no_device_error()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_rotate_quant_ties_and_strides_on_128_multiples(dtype):
    # rows of 256 channels (the streaming kernel): exact ties of fl32(u * inv)
    # and a row stride larger than the row
    X = np.zeros((6, 256), np.float32)
    X[0, 0], X[0, 8] = 1.5, 3.0
    X[1, 0], X[1, 8] = 2.75, 5.5
    X[2, 0], X[2, 8] = 5.5, 11.0
    X[3, :] = np.linspace(-3, 3, 256)
    X[4, 200] = -9.0
    Xr = X.astype(np.float16) if dtype == "f16" else synth.f32_to_bf16_bits(X)
    Xq_o, sx_o = O.rotate_quant(Xr, dtype, 8, None)
    big = torch.zeros((6, 256 + 128), dtype=torch.float16 if dtype == "f16" else torch.bfloat16, device="cuda")
    big[:, :256] = dev(Xr, dtype)
    Xq, sx = hq.hq_rotate_quant(big[:, :256], 8, None)
    assert_same(host(Xq), Xq_o, "codes")
    assert_same(host(sx), sx_o, "scales")
    assert np.all(O.unpack_s4(Xq_o, 256)[:3, :8] == 4)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("g", [128, 4096])
def test_rotate_normalised_bit_exact(dtype, g):
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((37, 4096)) * 0.02).astype(np.float32)
    W = {"f16": w.astype(np.float16), "bf16": synth.f32_to_bf16_bits(w), "f32": w}[dtype]
    d = synth.hadamard_signs(g, seed=5)
    ref = O.rotate_normalised(W, dtype, g, d)
    out = hq.hq_rotate(dev(W, dtype), g, torch.from_numpy(d).cuda())
    assert_same(host(out), ref, "rotated")


def test_channel_sqnorm_and_salient_selection():
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    d = synth.hadamard_signs(wl.g)
    norm2_o, sal_o = O.salient_channels(X, wl.xdtype, wl.g, d, wl.r)
    norm2 = hq.hq_channel_sqnorm(dev(X, wl.xdtype), wl.g, torch.from_numpy(d).cuda())
    n = host(norm2).astype(np.float64)
    assert np.allclose(n, norm2_o, rtol=1e-5, atol=1e-6 * norm2_o.max())
    sal = hq.hq_select_salient(norm2, wl.r).numpy()
    # the selected set must be a valid top-r of the exact norms (within fp32 error)
    thresh = np.sort(norm2_o)[-wl.r]
    assert np.all(norm2_o[sal] >= thresh * (1 - 1e-5))
    assert np.array_equal(sal, sal_o)


# ------------------------------------------------------------------ K0: w4_pack, SERQ
@pytest.mark.parametrize("gw", [0, 128, 256])
@pytest.mark.parametrize("N", [64, 300])
def test_w4_pack_bit_exact(gw, N):
    rng = np.random.default_rng(gw + N)
    K = 1024
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[1, :] = 0.0
    if gw:
        W[2, :gw] = np.abs(W[2, :gw]) + 1e-3
    Wq_o, sw_o, zw_o = O.w4_pack(W, "f32", gw)
    Wq, sw, zw = hq.w4_pack(dev(W, "f32"), gw)
    assert_same(untile_wq(host(Wq), N), Wq_o, "codes")
    if N % 128:   # padding rows of the last row tile are zero codes
        assert np.all(host(Wq)[-1, :, N % 128:, :] == 0)
    assert np.array_equal(f16bits(host(sw)), f16bits(sw_o))
    if gw:
        assert np.array_equal(f16bits(host(zw)), f16bits(zw_o))


@pytest.mark.parametrize("wdtype", ["f16", "bf16"])
def test_w4_pack_from_16bit_inputs(wdtype):
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((40, 512)) * 0.02).astype(np.float32)
    W = w.astype(np.float16) if wdtype == "f16" else synth.f32_to_bf16_bits(w)
    for gw in (0, 128):
        Wq_o, sw_o, zw_o = O.w4_pack(W, wdtype, gw)
        Wq, sw, zw = hq.w4_pack(dev(W, wdtype), gw)
        assert np.array_equal(untile_wq(host(Wq), 40), Wq_o) and np.array_equal(f16bits(host(sw)), f16bits(sw_o))


@pytest.mark.parametrize("gw,r", [(0, 8), (128, 16), (0, 64), (256, 40), (128, 0)])
def test_serq_prepare_bit_exact(gw, r):
    rng = np.random.default_rng(r + gw)
    N, K = 200, 1024
    Wrot = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", gw)
    sal = np.sort(rng.choice(K, r, replace=False)).astype(np.int32)
    Rq_o, sr_o = O.serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    Rq, sr = hq.serq_prepare(dev(Wrot, "f32"), torch.from_numpy(tile_wq(Wq)).cuda(), dev(sw, "f16"),
                             None if zw is None else dev(zw, "f16"), gw, torch.from_numpy(sal).cuda())
    assert np.array_equal(host(Rq), Rq_o)
    assert np.array_equal(f16bits(host(sr)), f16bits(sr_o))


# ------------------------------------------------------------------ K2: GEMM
def _gemm_inputs(M, N, K, gw, r, seed=0):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((M, K)) * 2).astype(np.float16)
    if M:
        X[:, 5] *= 40
    Wrot = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Xq, sx = O.rotate_quant(X, "f16", 128, None)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", gw)
    sal = np.sort(rng.choice(K, r, replace=False)).astype(np.int32)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, gw, sal)
    return dict(Xq=Xq, sx=sx, Wq=Wq, sw=sw, zw=zw, sal=sal, Rq=Rq, sr=sr)


def _dev_inputs(t):
    return dict(Xq=torch.from_numpy(t["Xq"]).cuda(), sx=torch.from_numpy(t["sx"]).cuda(),
                Wq=torch.from_numpy(tile_wq(t["Wq"])).cuda(), sw=dev(t["sw"], "f16"),
                zw=None if t["zw"] is None else dev(t["zw"], "f16"),
                sal=torch.from_numpy(t["sal"]).cuda() if len(t["sal"]) else None,
                Rq=torch.from_numpy(t["Rq"]).cuda(), sr=dev(t["sr"], "f16"))


GEMM_CASES = [
    # M, N, K, gw, r
    (16, 128, 256, 0, 8),
    (1, 256, 256, 0, 0),
    (200, 264, 512, 0, 16),
    (130, 136, 1024, 128, 32),
    (300, 512, 2048, 256, 64),
    (129, 1032, 384, 0, 24),
    (64, 384, 4096, 128, 16),
    # per-channel weights with r > 32: the epilogue's SERQ term takes two
    # 32-wide mma.sync K steps (the second one ragged for r = 40)
    (256, 512, 1024, 0, 64),
    (300, 264, 512, 0, 40),
    # the largest weight group the large-M kernel takes (its accumulators are
    # read back as floats: exact while |acc| < 2^22)
    (160, 256, 4096, 2048, 8),
]


@pytest.mark.parametrize("M,N,K,gw,r", GEMM_CASES)
def test_gemm_accumulators_bit_exact(M, N, K, gw, r):
    t = _gemm_inputs(M, N, K, gw, r)
    acc_o, accc_o = O.accum(t["Xq"], K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    g = _dev_inputs(t)
    acc, acc_c = hq.hq_debug_accum(g["Xq"], g["Wq"], g["zw"], gw, g["Rq"], g["sal"], N)
    assert_same(host(acc).astype(np.int64), acc_o, "acc")
    if r:
        assert_same(host(acc_c).astype(np.int64), accc_o, "acc_c")
    no_device_error()


SMALL_CASES = [
    # small-M (swap-operand, stream-K) kernel; several cases split a weight tile
    # across CTAs, which exercises the last-arriver fixup and its counter reset
    (1, 256, 256, 0, 8),
    (4, 1024, 2048, 0, 16),
    (16, 1024, 2048, 128, 16),
    (17, 520, 1024, 128, 8),
    (33, 264, 512, 0, 24),
    (64, 1032, 1024, 256, 64),
    (16, 11008, 4096, 128, 16),
]


@pytest.mark.parametrize("M,N,K,gw,r", SMALL_CASES)
def test_small_m_accumulators_bit_exact(M, N, K, gw, r):
    t = _gemm_inputs(M, N, K, gw, r, seed=2)
    acc_o, accc_o = O.accum(t["Xq"], K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    g = _dev_inputs(t)
    for _ in range(2):
        acc, acc_c = hq.hq_debug_accum(g["Xq"], g["Wq"], g["zw"], gw, g["Rq"], g["sal"], N, decode=True)
        assert_same(host(acc).astype(np.int64), acc_o, "acc")
        if r:
            assert_same(host(acc_c).astype(np.int64), accc_o, "acc_c")
    no_device_error()


@pytest.mark.parametrize("M,N,K,gw,r", SMALL_CASES)
@pytest.mark.parametrize("out", [torch.float16, torch.float32])
def test_small_m_linear_within_tolerance(M, N, K, gw, r, out):
    t = _gemm_inputs(M, N, K, gw, r, seed=3)
    acc_o, accc_o = O.accum(t["Xq"], K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    y64 = O.epilogue_f64(acc_o, accc_o, t["sx"], t["sw"], t["sr"] if r else None)
    g = _dev_inputs(t)
    ws = torch.zeros((hq.hq_linear_workspace_size(M, N, K, gw),), dtype=torch.uint8, device="cuda")
    Y = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], out,
                       workspace=ws)
    assert_y_close(y_host(Y), y64, 1e-3 if out == torch.float32 else 1e-2)
    Y2 = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], out,
                        workspace=ws)
    assert torch.equal(Y, Y2)          # same workspace, counters were reset: identical bytes
    assert int(ws.view(torch.int32)[: (N + 127) // 128].abs().sum()) == 0
    no_device_error()


@pytest.mark.parametrize("sign", [1, -1])
def test_group_accumulators_extreme_codes(sign):
    # every product at its extreme in the largest weight group the large-M
    # kernel takes: activation codes -7 (or +7) against weight values 0 - 15;
    # the group accumulator is +-7*15*2048 and the output matches the oracle
    M, N, K, gw = 256, 264, 4096, 2048
    Xq = np.full((M, K // 2), 0x99 if sign > 0 else 0x77, np.uint8)     # codes -7 / +7
    sx = np.full((M,), 0.25, np.float32)
    Wq = np.zeros((N, K // 2), np.uint8)                                 # unsigned code 0
    zw = np.full((K // gw, N), 15.0, np.float16)
    sw = np.full((K // gw, N), 0.5, np.float16)
    acc_o, _ = O.accum(Xq, K, Wq, zw, gw)
    assert np.all(acc_o == sign * 7 * 15 * gw)
    t = dict(Xq=Xq, sx=sx, Wq=Wq, sw=sw, zw=zw, sal=np.zeros((0,), np.int32),
             Rq=np.zeros((N, 0), np.uint8), sr=np.zeros((N,), np.float16))
    g = _dev_inputs(t)
    acc, _ = hq.hq_debug_accum(g["Xq"], g["Wq"], g["zw"], gw, None, None, N)
    assert_same(host(acc).astype(np.int64), acc_o, "acc")
    y64 = O.epilogue_f64(acc_o, None, sx, sw, None)
    Y = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, None, None, None, torch.float32)
    assert_y_close(y_host(Y), y64, 1e-3)
    no_device_error()


@pytest.mark.parametrize("M,N,K,gw", [(2048, 2560, 256, 0), (1280, 2048, 256, 128)])
def test_gemm_accumulators_many_tiles_per_cta(M, N, K, gw):
    # more output tiles than SMs: every CTA walks several tiles and the
    # accumulator double buffer wraps around
    t = _gemm_inputs(M, N, K, gw, 8, seed=4)
    acc_o, accc_o = O.accum(t["Xq"], K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    g = _dev_inputs(t)
    acc, acc_c = hq.hq_debug_accum(g["Xq"], g["Wq"], g["zw"], gw, g["Rq"], g["sal"], N)
    assert np.array_equal(host(acc).astype(np.int64), acc_o)
    assert np.array_equal(host(acc_c).astype(np.int64), accc_o)


@pytest.mark.parametrize("M,N,K,gw,r", GEMM_CASES)
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float16, torch.float32])
def test_linear_output_within_tolerance(M, N, K, gw, r, out):
    t = _gemm_inputs(M, N, K, gw, r, seed=1)
    acc_o, accc_o = O.accum(t["Xq"], K, t["Wq"], t["zw"], gw, t["Rq"], t["sal"])
    y64 = O.epilogue_f64(acc_o, accc_o, t["sx"], t["sw"], t["sr"] if r else None)
    g = _dev_inputs(t)
    Y = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], out)
    assert_y_close(y_host(Y), y64, 1e-3 if out == torch.float32 else 1e-2)
    Y2 = hq.w4a4_linear(g["Xq"], g["sx"], g["Wq"], g["sw"], g["zw"], gw, g["Rq"], g["sr"], g["sal"], out)
    assert torch.equal(Y, Y2)          # deterministic


# ------------------------------------------------------------------ whole layer
@pytest.mark.parametrize("name,M,N", [("tiny", 16, 128), ("decode", 4, 512), ("attn", 64, 256), ("down", 32, 256),
                                      ("large", 16, 256)])
def test_layer_end_to_end_from_raw_inputs(name, M, N):
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    W = synth.weights(wl, N=N)
    d = synth.hadamard_signs(wl.g)
    ref = O.layer(X, wl.xdtype, W, wl.wdtype, wl.g, d, wl.gw, wl.r)
    out_dt = torch.float16 if wl.xdtype == "f16" else torch.bfloat16
    Xd = dev(X, wl.xdtype)
    layer = hq.W4A4Linear.prepare(dev(W, wl.wdtype), wl.g, wl.gw, wl.r, torch.from_numpy(d).cuda(),
                                  sal_idx=torch.from_numpy(ref["sal"]), out_dtype=out_dt)
    assert np.array_equal(untile_wq(host(layer.Wq), N), ref["Wq"])
    assert np.array_equal(f16bits(host(layer.sw)), f16bits(ref["sw"]))
    assert np.array_equal(host(layer.Rq), ref["Rq"])
    assert np.array_equal(f16bits(host(layer.sr)), f16bits(ref["sr"]))
    Xq, sx = hq.hq_rotate_quant(Xd, wl.g, layer.H_signs)
    assert np.array_equal(host(Xq), ref["Xq"])
    Y = layer(Xd)
    assert_y_close(y_host(Y), ref["y"], 1e-2)
    no_device_error()


@pytest.mark.parametrize("name,M", [("decode", 16), ("attn", 2048), ("down", 4096), ("large", 512),
                                    ("large", 8192)])
def test_full_size_sampled_rows(name, M):
    # the full-size layer in the configuration the benchmark times; the oracle
    # computes its own packed weights (full size) and a sample of output rows
    wl = synth.WORKLOADS[name]
    X = synth.activations(wl, M=M)
    W = synth.weights(wl)
    d = synth.hadamard_signs(wl.g)
    Wrot = O.rotate_normalised(W, wl.wdtype, wl.g, d)
    Wq_o, sw_o, zw_o = O.w4_pack(Wrot, "f32", wl.gw)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(0).choice(M, min(M, 6), replace=False)]))
    _, sal = O.salient_channels(X[rows], wl.xdtype, wl.g, d, wl.r)
    Rq_o, sr_o = O.serq_prepare(Wrot, Wq_o, sw_o, zw_o, wl.gw, sal)
    del Wrot
    Xq_rows, sx_rows = O.rotate_quant(X[rows], wl.xdtype, wl.g, d)
    out_dt = torch.float16 if wl.xdtype == "f16" else torch.bfloat16
    layer = hq.W4A4Linear.prepare(dev(W, wl.wdtype), wl.g, wl.gw, wl.r, torch.from_numpy(d).cuda(),
                                  sal_idx=torch.from_numpy(sal), out_dtype=out_dt)
    assert_same(untile_wq(host(layer.Wq), wl.N), Wq_o, "weight codes")
    assert np.array_equal(host(layer.Rq), Rq_o)
    Xd = dev(X, wl.xdtype)
    Xq, sx = hq.hq_rotate_quant(Xd, wl.g, layer.H_signs)
    assert np.array_equal(host(Xq)[rows], Xq_rows)
    Y = layer(Xd)
    y64 = O.linear_rows_f64(Xq_rows, sx_rows, wl.K, Wq_o, sw_o, zw_o, wl.gw, Rq_o, sr_o, sal,
                            np.arange(len(rows)))
    assert_y_close(y_host(Y)[rows], y64, 1e-2)
    no_device_error()


# ------------------------------------------------------------------ failure path
def test_bounded_wait_records_timeout_and_context_survives():
    assert hq.hq_last_device_status() == 0
    hq.hq_debug_wait_probe(2_000_000)            # 2 ms; nothing ever arrives
    assert hq.hq_last_device_status() == 5        # HQ_ERR_TIMEOUT, then cleared
    assert hq.hq_last_device_status() == 0
    t = _gemm_inputs(16, 128, 256, 0, 8)
    g = _dev_inputs(t)
    acc, _ = hq.hq_debug_accum(g["Xq"], g["Wq"], g["zw"], 0, g["Rq"], g["sal"], 128)
    acc_o, _ = O.accum(t["Xq"], 256, t["Wq"], None, 0, t["Rq"], t["sal"])
    assert np.array_equal(host(acc).astype(np.int64), acc_o)
