// pack.cu -- offline weight preparation: kernel K0 (w4_pack, the int4 weight
// quantiser) and SERQ's single error matrix R on the salient input channels
// ("SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
// technical summary section 2.2; group-wise scale and zero point from "OffQ:
// Taming Structured Outliers in LLM Quantization by Offsetting", Methodology 3).
// Neither is on the timed path; both produce bit-exact codes and scales.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <vector>

#include "hq_device.cuh"

namespace hq {

template <int WT>
__device__ __forceinline__ float load_w(const void* W, int64_t i) {
    if constexpr (WT == HQ_F16) {
        return __half2float(reinterpret_cast<const __half*>(W)[i]);
    } else if constexpr (WT == HQ_BF16) {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(W)[i]) << 16);
    } else {
        return reinterpret_cast<const float*>(W)[i];
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

__device__ __forceinline__ uint16_t half_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }
__device__ __forceinline__ float bits_half(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Per output channel symmetric: one warp per row (rows N..Npad-1 of the last
// tile are written as zero codes).
template <int WT>
__global__ void k_pack_sym(const void* __restrict__ W, int64_t N, int64_t Npad, int64_t K, uint8_t* __restrict__ Wq,
                           uint16_t* __restrict__ sw) {
    const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    const int64_t KB = K / 128;
    if (n >= Npad) return;
    if (n >= N) {
        for (int64_t j = lane; j < K / 2; j += 32) Wq[wq_offset(n, j, KB)] = 0;
        return;
    }
    float amax = 0.f;
    for (int64_t k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(load_w<WT>(W, n * K + k)));
    amax = warp_max(amax);
    const uint16_t s16 = half_bits(__fdiv_rn(amax, 7.0f));
    const float s = bits_half(s16);
    if (lane == 0) sw[n] = s16;
    for (int64_t j = lane; j < K / 2; j += 32) {
        int q[2] = {0, 0};
        if (s != 0.f) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float w = load_w<WT>(W, n * K + 2 * j + e);
                q[e] = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(w, s)), -8.f), 7.f));
            }
        }
        Wq[wq_offset(n, j, KB)] = static_cast<uint8_t>((q[0] & 0xF) | ((q[1] & 0xF) << 4));
    }
}

// Per (channel, group) asymmetric over [min(lo,0), max(hi,0)]: one warp per
// (row, group); scales and zero points are stored group-major [K/gw][N].
template <int WT>
__global__ void k_pack_asym(const void* __restrict__ W, int64_t N, int64_t Npad, int64_t K, int gw,
                            uint8_t* __restrict__ Wq, uint16_t* __restrict__ sw, uint16_t* __restrict__ zw) {
    const int64_t G = K / gw;
    const int64_t KB = K / 128;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (item >= Npad * G) return;
    const int64_t n = item / G, b = item % G;
    const int64_t k0 = b * gw;
    if (n >= N) {
        for (int j = lane; j < gw / 2; j += 32) Wq[wq_offset(n, k0 / 2 + j, KB)] = 0;
        return;
    }
    float lo = 0.f, hi = 0.f;
    for (int k = lane; k < gw; k += 32) {
        const float w = load_w<WT>(W, n * K + k0 + k);
        lo = fminf(lo, w);
        hi = fmaxf(hi, w);
    }
    lo = warp_min(lo);
    hi = warp_max(hi);
    uint16_t s16 = half_bits(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    if (bits_half(s16) == 0.f) s16 = 0x3C00u;  // 1.0
    const float s = bits_half(s16);
    // an integer in 0..15; the int round trip makes a zero +0 (never -0)
    const float z = static_cast<float>(static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), 15.f)));
    if (lane == 0) {
        sw[b * N + n] = s16;
        zw[b * N + n] = half_bits(z);
    }
    for (int j = lane; j < gw / 2; j += 32) {
        int q[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float w = load_w<WT>(W, n * K + k0 + 2 * j + e);
            q[e] = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(w, s)) + z, 0.f), 15.f));
        }
        Wq[wq_offset(n, k0 / 2 + j, KB)] = static_cast<uint8_t>(q[0] | (q[1] << 4));
    }
}

// SERQ error matrix: one warp per output row n.  Lane l owns the pairs of
// salient positions (2p, 2p+1) with p = l, l+32, ... (r <= 256).
__global__ void k_serq_prepare(const float* __restrict__ Wrot, int64_t N, int64_t K, const uint8_t* __restrict__ Wq,
                               const uint16_t* __restrict__ sw, const uint16_t* __restrict__ zw, int gw,
                               const int32_t* __restrict__ sal, int r, uint8_t* __restrict__ Rq,
                               uint16_t* __restrict__ sr) {
    const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (n >= N) return;
    const int ld = (r + 1) / 2;
    float e[8];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * (lane + 32 * i) + h;
            float ev = 0.f;
            if (j < r && (sal[j] < 0 || sal[j] >= K)) {
                record_status(HQ_ERR_ARG);   // a salient index outside [0, K): its error term is 0
            } else if (j < r) {
                const int64_t k = sal[j];
                const uint8_t byte = Wq[wq_offset(n, k / 2, K / 128)];
                const int nib = (byte >> (4 * (k & 1))) & 0xF;
                float what;
                if (gw == 0) {
                    what = __fmul_rn(static_cast<float>((nib ^ 8) - 8), bits_half(sw[n]));
                } else {
                    const int64_t b = k / gw;
                    const float z = bits_half(zw[b * N + n]);
                    what = __fmul_rn(__fsub_rn(static_cast<float>(nib), z), bits_half(sw[b * N + n]));
                }
                ev = __fsub_rn(Wrot[n * K + k], what);
                amax = fmaxf(amax, fabsf(ev));
            }
            e[2 * i + h] = ev;
        }
    }
    amax = warp_max(amax);
    const uint16_t s16 = half_bits(__fdiv_rn(amax, 7.0f));
    const float s = bits_half(s16);
    if (lane == 0) sr[n] = s16;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int p = lane + 32 * i;
        if (p < ld) {
            int q[2] = {0, 0};
#pragma unroll
            for (int h = 0; h < 2; ++h)
                if (2 * p + h < r && s != 0.f)
                    q[h] = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(e[2 * i + h], s)), -8.f), 7.f));
            Rq[n * ld + p] = static_cast<uint8_t>((q[0] & 0xF) | ((q[1] & 0xF) << 4));
        }
    }
}

}  // namespace hq

using namespace hq;

extern "C" hq_status w4_pack(const void* W, hq_dtype wt, int64_t N, int64_t K, int32_t group, uint8_t* Wq,
                             uint16_t* sw, uint16_t* zw, void* stream) {
    if (N < 0 || K <= 0 || K % 128 != 0 || group < 0 || (group & 1)) return HQ_ERR_ARG;
    if (group > 0 && K % group != 0) return HQ_ERR_ARG;
    if (wt != HQ_F16 && wt != HQ_BF16 && wt != HQ_F32) return HQ_ERR_UNSUPPORTED;
    if (N == 0) return HQ_OK;
    if (!W || !Wq || !sw || (group > 0 && !zw)) return HQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int threads = 256, wpb = threads / 32;
    const int64_t Npad = (N + 127) / 128 * 128;
    if (group == 0) {
        const unsigned blocks = static_cast<unsigned>((Npad + wpb - 1) / wpb);
        if (wt == HQ_F16) k_pack_sym<HQ_F16><<<blocks, threads, 0, st>>>(W, N, Npad, K, Wq, sw);
        else if (wt == HQ_BF16) k_pack_sym<HQ_BF16><<<blocks, threads, 0, st>>>(W, N, Npad, K, Wq, sw);
        else k_pack_sym<HQ_F32><<<blocks, threads, 0, st>>>(W, N, Npad, K, Wq, sw);
    } else {
        const int64_t items = Npad * (K / group);
        const unsigned blocks = static_cast<unsigned>((items + wpb - 1) / wpb);
        if (wt == HQ_F16) k_pack_asym<HQ_F16><<<blocks, threads, 0, st>>>(W, N, Npad, K, group, Wq, sw, zw);
        else if (wt == HQ_BF16) k_pack_asym<HQ_BF16><<<blocks, threads, 0, st>>>(W, N, Npad, K, group, Wq, sw, zw);
        else k_pack_asym<HQ_F32><<<blocks, threads, 0, st>>>(W, N, Npad, K, group, Wq, sw, zw);
    }
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

extern "C" size_t hq_packed_weight_bytes(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0 || K % 128 != 0) return 0;
    return static_cast<size_t>((N + 127) / 128 * 128) * static_cast<size_t>(K / 2);
}

extern "C" hq_status serq_prepare(const float* W_rot, int64_t N, int64_t K, const uint8_t* Wq, const uint16_t* sw,
                                  const uint16_t* zw, int32_t group, const int32_t* sal_idx, int32_t r, uint8_t* Rq,
                                  uint16_t* sr, void* stream) {
    if (N < 0 || K <= 0 || K % 128 != 0 || r < 0 || r > 256 || r > K || group < 0) return HQ_ERR_ARG;
    if (group > 0 && K % group != 0) return HQ_ERR_ARG;
    if (N == 0) return HQ_OK;
    if (!W_rot || !Wq || !sw || !sr || (group > 0 && !zw) || (r > 0 && (!sal_idx || !Rq))) return HQ_ERR_ARG;
    const int threads = 256, wpb = threads / 32;
    k_serq_prepare<<<static_cast<unsigned>((N + wpb - 1) / wpb), threads, 0, static_cast<cudaStream_t>(stream)>>>(
        W_rot, N, K, Wq, sw, zw, group, sal_idx, r, Rq, sr);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

extern "C" hq_status hq_select_salient(const float* norm2, int64_t K, int32_t r, int32_t* sal) {
    if (!norm2 || !sal || K <= 0 || r < 0 || r > K) return HQ_ERR_ARG;
    for (int64_t k = 0; k < K; ++k)
        if (norm2[k] != norm2[k]) return HQ_ERR_ARG;   // a NaN norm has no order
    std::vector<int64_t> idx(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) idx[static_cast<size_t>(k)] = k;
    // largest first; equal values keep the lower index first
    std::stable_sort(idx.begin(), idx.end(), [&](int64_t a, int64_t b) { return norm2[a] > norm2[b]; });
    std::vector<int64_t> top(idx.begin(), idx.begin() + r);
    std::sort(top.begin(), top.end());
    for (int32_t j = 0; j < r; ++j) sal[j] = static_cast<int32_t>(top[static_cast<size_t>(j)]);
    return HQ_OK;
}
