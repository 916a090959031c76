// mxfp4.cu -- hq_quant_mxfp4: the MXFP4 block quantiser of the 4-bit paths.
//
// Source: "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
// Quantization", technical summary section 2 (main and residual path both in
// 4 bit, INT4 or MXFP4) and section 3 (MXFP4 on Blackwell tensor cores).  The
// format is the microscaling one: blocks of 32 consecutive values share a
// power-of-two scale stored as a biased 8-bit exponent, and each value is a
// 4-bit E2M1 float (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).
//
// Per block: E = floor(log2(amax)) - 2, byte = clamp(E + 127, 0, 254) (0 for
// an all-zero block), t = v * 2^-(byte - 127) (exact: a power-of-two scaling),
// |t| rounded to the E2M1 grid to nearest with ties to the even mantissa
// (0, 1, 2, 4) and saturated at 6, sign bit for t < 0 with a non-zero
// magnitude, element 2j in the low nibble of byte j.
//
// One thread per block: the 32 values arrive as 16-byte loads, the block
// maximum is the thread's own, 16 bytes of codes and one scale byte leave.
// hq_mxfp4_linear multiplies two such code matrices exactly per block on the
// warp-level int8 MMA (twice an E2M1 value is an integer); the block-scaled
// tensor-core form (tcgen05.mma kind::mxf4) is not built.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"

namespace hq {
namespace {

constexpr int MX_THREADS = 256;

__device__ __forceinline__ void mx_load8(const void* X, int xt, int64_t i, float (&f)[8]) {
    if (xt == HQ_F32) {
        const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) + i);
        const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) + i + 4);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        return;
    }
    const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(X) + i);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (xt == HQ_BF16) {
            f[2 * e] = __uint_as_float(u[e] << 16);
            f[2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
        } else {
            const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
            f[2 * e] = h.x;
            f[2 * e + 1] = h.y;
        }
    }
}

// 4-bit code of t
__device__ __forceinline__ uint32_t mx_code(float t) {
    const float a = fabsf(t);
    float r;
    if (a < 2.0f) r = __fmul_rn(rintf(__fmul_rn(a, 2.0f)), 0.5f);
    else if (a < 4.0f) r = rintf(a);
    else r = fminf(__fmul_rn(rintf(__fmul_rn(a, 0.5f)), 2.0f), 6.0f);
    // 0, 0.5, 1, 1.5, 2 -> 0..4 (twice the value); 3 -> 5, 4 -> 6, 6 -> 7
    const uint32_t mag = r <= 2.0f ? static_cast<uint32_t>(__fmul_rn(r, 2.0f)) : (r == 3.0f ? 5u : (r == 4.0f ? 6u : 7u));
    return (t < 0.0f && mag != 0u) ? (mag | 8u) : mag;
}

__global__ void __launch_bounds__(MX_THREADS) k_mxfp4(const void* __restrict__ X, int xt, int M, int K, int64_t ldx,
                                                     uint8_t* __restrict__ Xq, uint8_t* __restrict__ sb) {
    const int nb = K / 32;
    const int64_t total = static_cast<int64_t>(M) * nb;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / nb;
        const int b = static_cast<int>(i - m * nb);
        const int64_t src = m * ldx + 32 * static_cast<int64_t>(b);
        float v[4][8];
#pragma unroll
        for (int c = 0; c < 4; ++c) mx_load8(X, xt, src + 8 * c, v[c]);
        float amax = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
        uint32_t words[4] = {0u, 0u, 0u, 0u};
        int byte = 0;
        if (amax > 0.f) {
            int lg = ilogbf(amax);
            lg = lg > 200 ? 200 : lg;   // an infinite input saturates its block (inputs should be finite)
            const int E = lg - 2;
            byte = E + 127 < 0 ? 0 : (E + 127 > 254 ? 254 : E + 127);
            const int sh = 127 - byte;   // t = v * 2^sh
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t w = 0u;
#pragma unroll
                for (int e = 0; e < 8; ++e) w |= mx_code(ldexpf(v[c][e], sh)) << (4 * e);
                words[c] = w;
            }
        }
        *reinterpret_cast<uint4*>(Xq + m * (K / 2) + 16 * static_cast<int64_t>(b)) =
            make_uint4(words[0], words[1], words[2], words[3]);
        sb[m * nb + b] = static_cast<uint8_t>(byte);
    }
}

// ---------------------------------------------------------------- k_mx_gemm
// Y[m][n] (+)= sum over blocks b of 2^(Ex + Ew) sum_{k in b} x_k w_k with x, w
// the E2M1 values of the codes.  Twice an E2M1 value is an integer in
// [-12, 12], so one block of one row pair is one exact int8 dot product of 32
// terms: one warp-level mma.sync.m16n8k32.s8 per block computes a 16 x 8 tile's
// block sums exactly (|sum| <= 32 * 144); the tile adds them, scaled by the
// power of two 2^(bx + bw - 256) (exact), in fp32 in block order.  A warp owns
// 32 x 32 outputs, so each expanded fragment feeds several MMAs.
__device__ __forceinline__ uint32_t mx_expand4(uint32_t v) {
    // nibble i = code of element i -> byte i = 2 * value, two's complement
    const uint32_t mag = __byte_perm(0x03020100u, 0x0C080604u, v & 0x7777u);   // 0,1,2,3,4,6,8,12
    uint32_t neg = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) neg |= ((v >> (4 * i + 3)) & 1u) * (0xFFu << (8 * i));
    return (mag & ~neg) | (__vsub4(0u, mag) & neg);
}

__device__ __forceinline__ void mx_mma(int32_t (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^(e - 128) for a scale byte e, exactly (subnormal for e < 2)
__device__ __forceinline__ float mx_half_scale(int e) {
    return __int_as_float(e >= 2 ? (e - 1) << 23 : 1 << (21 + e));
}

// an int32 of magnitude below 2^22 as a float, exactly: its bits added to those
// of 1.5 * 2^23 form the float 1.5 * 2^23 + c
__device__ __forceinline__ float mx_i2f(int32_t c) { return __fsub_rn(__int_as_float(c + 0x4B400000), 12582912.0f); }

constexpr int MXG_WARPS = 8;
constexpr int MXG_MT = 2, MXG_NT = 4;   // a warp's tile: 2 x 16 rows by 4 x 8 columns

__global__ void __launch_bounds__(MXG_WARPS * 32, 2) k_mx_gemm(const uint8_t* __restrict__ Xq, const uint8_t* __restrict__ sx,
                                                           const uint8_t* __restrict__ Wq, const uint8_t* __restrict__ sw,
                                                           int M, int N, int K, float* __restrict__ Y, int accumulate) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int tiles_n = (N + 8 * MXG_NT - 1) / (8 * MXG_NT);
    const int64_t tile = static_cast<int64_t>(blockIdx.x) * MXG_WARPS + warp;
    const int64_t tiles = static_cast<int64_t>((M + 16 * MXG_MT - 1) / (16 * MXG_MT)) * tiles_n;
    if (tile >= tiles) return;   // whole warps only
    const int m0 = static_cast<int>(tile / tiles_n) * 16 * MXG_MT, n0 = static_cast<int>(tile % tiles_n) * 8 * MXG_NT;
    const int nb = K / 32;
    const int64_t ldq = K / 2;
    float y[MXG_MT][MXG_NT][4];
#pragma unroll
    for (int mt = 0; mt < MXG_MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < MXG_NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) y[mt][nt][q] = 0.f;
    // the raw codes and scale bytes of block b + 1 are loaded while block b is
    // expanded and multiplied (the loads' latency off the dependent chain)
    uint32_t ra[MXG_MT][4], rb[MXG_NT][2];
    int ex[MXG_MT][2], ew[MXG_NT][2];
    auto load_block = [&](int b) {
        const int64_t o = 16 * static_cast<int64_t>(b) + 2 * t4;
#pragma unroll
        for (int mt = 0; mt < MXG_MT; ++mt) {
            const int r0 = m0 + 16 * mt + g8, r1 = r0 + 8;
            const bool v0 = r0 < M, v1 = r1 < M;
            ra[mt][0] = v0 ? *reinterpret_cast<const uint16_t*>(Xq + r0 * ldq + o) : 0u;
            ra[mt][1] = v1 ? *reinterpret_cast<const uint16_t*>(Xq + r1 * ldq + o) : 0u;
            ra[mt][2] = v0 ? *reinterpret_cast<const uint16_t*>(Xq + r0 * ldq + o + 8) : 0u;
            ra[mt][3] = v1 ? *reinterpret_cast<const uint16_t*>(Xq + r1 * ldq + o + 8) : 0u;
            ex[mt][0] = v0 ? sx[static_cast<int64_t>(r0) * nb + b] : 0;
            ex[mt][1] = v1 ? sx[static_cast<int64_t>(r1) * nb + b] : 0;
        }
#pragma unroll
        for (int nt = 0; nt < MXG_NT; ++nt) {
            const int nB = n0 + 8 * nt + g8, c0 = n0 + 8 * nt + 2 * t4;
            const bool vB = nB < N;
            rb[nt][0] = vB ? *reinterpret_cast<const uint16_t*>(Wq + nB * ldq + o) : 0u;
            rb[nt][1] = vB ? *reinterpret_cast<const uint16_t*>(Wq + nB * ldq + o + 8) : 0u;
            ew[nt][0] = c0 < N ? sw[static_cast<int64_t>(c0) * nb + b] : 0;
            ew[nt][1] = c0 + 1 < N ? sw[static_cast<int64_t>(c0 + 1) * nb + b] : 0;
        }
    };
    load_block(0);
    for (int b = 0; b < nb; ++b) {
        uint32_t a[MXG_MT][4], bf[MXG_NT][2];
        float fx[MXG_MT][2], fw[MXG_NT][2];
#pragma unroll
        for (int mt = 0; mt < MXG_MT; ++mt) {
#pragma unroll
            for (int i = 0; i < 4; ++i) a[mt][i] = mx_expand4(ra[mt][i]);
            fx[mt][0] = mx_half_scale(ex[mt][0]);
            fx[mt][1] = mx_half_scale(ex[mt][1]);
        }
#pragma unroll
        for (int nt = 0; nt < MXG_NT; ++nt) {
            bf[nt][0] = mx_expand4(rb[nt][0]);
            bf[nt][1] = mx_expand4(rb[nt][1]);
            fw[nt][0] = mx_half_scale(ew[nt][0]);
            fw[nt][1] = mx_half_scale(ew[nt][1]);
        }
        if (b + 1 < nb) load_block(b + 1);
#pragma unroll
        for (int nt = 0; nt < MXG_NT; ++nt)
#pragma unroll
            for (int mt = 0; mt < MXG_MT; ++mt) {
                int32_t c[4] = {0, 0, 0, 0};
                mx_mma(c, a[mt], bf[nt][0], bf[nt][1]);
                // (2x)(2w) / 4 * 2^(bx - 127) * 2^(bw - 127) = c 2^(bx - 128) 2^(bw - 128)
                y[mt][nt][0] = __fmaf_rn(mx_i2f(c[0]), __fmul_rn(fx[mt][0], fw[nt][0]), y[mt][nt][0]);
                y[mt][nt][1] = __fmaf_rn(mx_i2f(c[1]), __fmul_rn(fx[mt][0], fw[nt][1]), y[mt][nt][1]);
                y[mt][nt][2] = __fmaf_rn(mx_i2f(c[2]), __fmul_rn(fx[mt][1], fw[nt][0]), y[mt][nt][2]);
                y[mt][nt][3] = __fmaf_rn(mx_i2f(c[3]), __fmul_rn(fx[mt][1], fw[nt][1]), y[mt][nt][3]);
            }
    }
#pragma unroll
    for (int mt = 0; mt < MXG_MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < MXG_NT; ++nt) {
            const int r0 = m0 + 16 * mt + g8, r1 = r0 + 8, c0 = n0 + 8 * nt + 2 * t4;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = q < 2 ? r0 : r1, cc = c0 + (q & 1);
                if (r < M && cc < N) {
                    float* dst = Y + static_cast<int64_t>(r) * N + cc;
                    *dst = accumulate ? __fadd_rn(*dst, y[mt][nt][q]) : y[mt][nt][q];
                }
            }
        }
}

bool mx_al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace hq

using namespace hq;

extern "C" hq_status hq_quant_mxfp4(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x, uint8_t* Xq,
                                    uint8_t* scales, void* stream) {
    if (!(xt == HQ_F16 || xt == HQ_BF16 || xt == HQ_F32) || M < 0 || K <= 0 || K % 32 != 0 || ld_x < K)
        return HQ_ERR_ARG;
    if (M > INT32_MAX || K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    if (M == 0) return HQ_OK;
    if (!X || !Xq || !scales) return HQ_ERR_ARG;
    const int64_t es = xt == HQ_F32 ? 4 : 2;
    if (!mx_al16(X) || !mx_al16(Xq) || (ld_x * es) % 16 != 0) return HQ_ERR_ALIGN;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return HQ_ERR_CUDA;
    const int64_t blocks = (M * (K / 32) + MX_THREADS - 1) / MX_THREADS;
    const int grid = static_cast<int>(blocks < 8 * nsm ? blocks : 8 * nsm);
    k_mxfp4<<<grid, MX_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(X, xt, static_cast<int>(M),
                                                                      static_cast<int>(K), ld_x, Xq, scales);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

extern "C" hq_status hq_mxfp4_linear(const uint8_t* Xq, const uint8_t* sx, int64_t M, int64_t K, const uint8_t* Wq,
                                     const uint8_t* sw, int64_t N, float* Y, int32_t accumulate, void* stream) {
    if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return HQ_ERR_ARG;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return HQ_OK;
    if (!Xq || !sx || !Wq || !sw || !Y) return HQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(Xq) & 1u) || (reinterpret_cast<uintptr_t>(Wq) & 1u) ||
        (reinterpret_cast<uintptr_t>(Y) & 3u))
        return HQ_ERR_ALIGN;
    const int64_t tiles = ((M + 16 * MXG_MT - 1) / (16 * MXG_MT)) * ((N + 8 * MXG_NT - 1) / (8 * MXG_NT));
    const int64_t grid = (tiles + MXG_WARPS - 1) / MXG_WARPS;
    if (grid > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    k_mx_gemm<<<static_cast<unsigned>(grid), MXG_WARPS * 32, 0, static_cast<cudaStream_t>(stream)>>>(
        Xq, sx, Wq, sw, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), Y, accumulate ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}
