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
// The layer's own GEMM on these codes (tcgen05.mma kind::mxf4) is not part of
// this file.
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
