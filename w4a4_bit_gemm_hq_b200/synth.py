"""Seeded synthetic inputs for the W4A4 rotated linear layer.

This module only draws numbers: activations, weights, the Hadamard sign vector
and outlier positions, with the shapes and value distributions of the
workloads below.  It holds none of the layer's arithmetic.  Both the test
suite's CPU oracle and the CUDA path receive exactly these arrays.

Every tensor is drawn from its own numpy PCG64 stream, keyed by the workload
seed and a fixed tensor id, so a tensor does not change when another one's
shape does.  bfloat16 tensors are returned as uint16 bit patterns (numpy has
no bfloat16), rounded to nearest even from float32.

Workloads (sizes and distributions of the layer shapes in the task brief):

* ``tiny``     16x256x128, X fp16 N(0,1) with 2 outlier channels x50 and token 0
               x100; W fp16 N(0, 0.02); g = 128; per-channel weights; r = 8.
* ``decode``   M in {1, 4, 16}, K 4096, N 11008; X fp16 N(0,1) with 4 outlier
               channels x30; W fp16 N(0, 0.02); g = 128; group-128 weights; r = 16.
* ``attn``     2048x4096x4096; X bf16 Student-t(3) with X[0, c*] = 1000 (c* the
               first channel of a seeded group); W bf16 N(0, 0.02); g = 4096;
               per-channel weights; r = 32.
* ``down``     4096x11008x4096; X bf16 SiLU(N(0,1)) * N(0,1) with 1% of the
               channels x20; W bf16 N(0, 0.015); g = 128; group-128 weights; r = 32.
* ``large``    M in {512, 2048, 8192}, K 8192, N 28672; X bf16 N(0,1) with 8
               outlier channels x50; W bf16 N(0, 0.01); g = 256; per-channel; r = 64.
"""
from dataclasses import dataclass, field

import numpy as np

_T_X, _T_W, _T_D, _T_OUT, _T_ROW = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    g: int           # Hadamard group size
    gw: int          # weight quantisation group (0 = per output channel)
    r: int           # SERQ rank (number of salient input channels)
    xdtype: str      # "f16" or "bf16" (also the output dtype)
    wdtype: str
    x_kind: str      # distribution recipe of X
    w_sigma: float
    n_outlier: int = 0
    outlier_scale: float = 1.0
    extra: dict = field(default_factory=dict)

    def with_m(self, M):
        return Workload(self.name, M, self.K, self.N, self.g, self.gw, self.r, self.xdtype,
                        self.wdtype, self.x_kind, self.w_sigma, self.n_outlier,
                        self.outlier_scale, dict(self.extra))


WORKLOADS = {
    "tiny": Workload("tiny", 16, 256, 128, 128, 0, 8, "f16", "f16", "normal_outlier_bos", 0.02,
                     n_outlier=2, outlier_scale=50.0, extra={"bos_scale": 100.0}),
    "decode": Workload("decode", 16, 4096, 11008, 128, 128, 16, "f16", "f16", "normal_outlier", 0.02,
                       n_outlier=4, outlier_scale=30.0, extra={"m_sweep": (1, 4, 16)}),
    "attn": Workload("attn", 2048, 4096, 4096, 4096, 0, 32, "bf16", "bf16", "student_t_massive", 0.02,
                     extra={"massive": 1000.0}),
    "down": Workload("down", 4096, 11008, 4096, 128, 128, 32, "bf16", "bf16", "swiglu_salient", 0.015,
                     n_outlier=110, outlier_scale=20.0),
    "large": Workload("large", 8192, 8192, 28672, 256, 0, 64, "bf16", "bf16", "normal_outlier", 0.01,
                      n_outlier=8, outlier_scale=50.0, extra={"m_sweep": (512, 2048, 8192)}),
}


def _rng(seed, tensor_id):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id])))


def f32_to_bf16_bits(a):
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    b = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(b):
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _cast(a, dtype):
    if dtype == "f16":
        return a.astype(np.float16)
    if dtype == "bf16":
        return f32_to_bf16_bits(a)
    return a.astype(np.float32)


def outlier_channels(wl: Workload, seed=0):
    """Sorted positions of the scaled input channels (seeded, no replacement)."""
    if wl.n_outlier == 0:
        return np.zeros((0,), np.int64)
    return np.sort(_rng(seed, _T_OUT).choice(wl.K, size=wl.n_outlier, replace=False))


def hadamard_signs(g, seed=0):
    """The random +-1 diagonal d of H = diag(d) * Sylvester(g), with d[0] = +1
    so that the first row of H stays all ones."""
    d = np.where(_rng(seed, _T_D).random(g) < 0.5, -1, 1).astype(np.int8)
    d[0] = 1
    return d


def activations(wl: Workload, seed=0, M=None):
    """X [M, K] in wl.xdtype (float16, or bf16 bits as uint16)."""
    M = wl.M if M is None else M
    rng = _rng(seed, _T_X)
    K = wl.K
    if wl.x_kind in ("normal_outlier", "normal_outlier_bos"):
        x = rng.standard_normal((M, K), dtype=np.float32)
        x[:, outlier_channels(wl, seed)] *= wl.outlier_scale
        if wl.x_kind == "normal_outlier_bos" and M > 0:
            x[0, :] *= wl.extra["bos_scale"]
    elif wl.x_kind == "student_t_massive":
        x = rng.standard_t(3.0, size=(M, K)).astype(np.float32)
        grp = int(_rng(seed, _T_ROW).integers(0, K // wl.g))
        if M > 0:
            x[0, grp * wl.g] = wl.extra["massive"]
    elif wl.x_kind == "swiglu_salient":
        a = rng.standard_normal((M, K), dtype=np.float32)
        b = rng.standard_normal((M, K), dtype=np.float32)
        x = (a / (1.0 + np.exp(-a))) * b
        x[:, outlier_channels(wl, seed)] *= wl.outlier_scale
    else:
        raise ValueError(wl.x_kind)
    return _cast(x, wl.xdtype)


def weights(wl: Workload, seed=0, N=None):
    """W [N, K] ~ N(0, sigma) in wl.wdtype."""
    N = wl.N if N is None else N
    w = _rng(seed, _T_W).standard_normal((N, wl.K), dtype=np.float32) * np.float32(wl.w_sigma)
    return _cast(w, wl.wdtype)


def to_float32(a, dtype):
    """Widen an input array (float16 / bf16 bits / float32) to float32, exactly."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a)
    return np.asarray(a, np.float32)


_T_CAL, _T_DIR = 6, 7


def calibration_activations(wl: Workload, S, L, seed=0, n_dir=4, massive=400.0):
    """Calibration batch for the offline steps: S sequences of L tokens, X
    [S*L, K] in wl.xdtype, drawn as the workload's activations (its own
    distribution recipe, from a separate stream) plus, in every sequence, one
    token at a seeded position that carries a shared outlier direction.

    The direction ``u`` (float32 [K], returned unnormalised) has n_dir seeded
    channels of magnitude 1 with seeded signs and a dense N(0, 0.02) part, so
    it is neither a single channel nor axis-aligned; the token gets
    a_s * u with a_s uniform in [0.5, 1] * massive (seeded, random sign).
    Returns (X, u, pos) with pos [S] the planted token of each sequence."""
    rng = _rng(seed, _T_CAL)
    base = activations(wl, seed=seed + 1000, M=S * L)
    x = to_float32(base, wl.xdtype).copy().reshape(S, L, wl.K)
    dr = _rng(seed, _T_DIR)
    u = (dr.standard_normal(wl.K) * 0.02).astype(np.float32)
    ch = dr.choice(wl.K, size=n_dir, replace=False)
    u[ch] = np.where(dr.random(n_dir) < 0.5, -1.0, 1.0).astype(np.float32)
    pos = rng.integers(0, L, size=S)
    amp = (rng.uniform(0.5, 1.0, size=S) * massive * np.where(rng.random(S) < 0.5, -1.0, 1.0)).astype(np.float32)
    for s in range(S):
        x[s, pos[s], :] += amp[s] * u
    return _cast(x.reshape(S * L, wl.K), wl.xdtype), u, pos
