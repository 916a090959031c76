// calib.cu -- offline calibration on the GPU: the steps that decide, once per
// layer, how channels are rotated, ordered and scaled before the online path
// (rotate/quant + W4A4 GEMM) runs.  Nothing here is on the per-token path;
// the results are folded into the weights.
//
// Sources:
//  * "OffQ: Taming Structured Outliers in LLM Quantization by Offsetting",
//    Methodology 1 (Top-1 PCA: keep only the token of largest L-infinity norm
//    of each calibration sequence, take the principal eigenvector of the
//    covariance of those tokens, rotate so the outlier energy lands in the
//    first channel), Methodology 3 and the ablation in the contributions
//    (channels partitioned into groups of 128, sorted grouping);
//  * "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
//    Quantization", technical summary section 1 (static per-channel flattening
//    in the manner of SmoothQuant, folded into the adjacent weights) and
//    section 3 (the channel permutation applied to the weights offline, the
//    activations arriving permuted by the previous layer).
//
// Kernels (all SIMT: none of this is a dense contraction worth the tensor
// cores, and all of it runs once per layer):
//  k_extreme      one CTA per calibration sequence: max |x| of every token
//                 (exact), the arg max (ties to the earlier token), and the
//                 chosen token widened to fp32.
//  k_top1_pca_cl  power iteration on C = T^T T / S without forming C
//                 (y = T v, z = T^T y / S, v = z / |z|) on a cluster of 8 CTAs
//                 holding T in their shared memory; k_top1_pca, one CTA reading
//                 T from L2, when it does not fit.  Every sum in a fixed order
//                 (deterministic).
//  k_householder  one warp per row: Y = X Q with Q = I - 2 w w^T / (w^T w),
//                 w = v' - e0, v' = +-v with v'[0] <= 0, so Q v' = e0.
//  k_col_absmax   column max |x| with integer atomics on the (non-negative)
//                 float bit patterns: exact, order independent.
//  k_rank         sorted grouping: position of every channel in the order of
//                 decreasing statistic (ties to the lower index) by counting,
//                 perm[position] = channel.
//  k_flatten      s[k] = xmax[k]^alpha / wmax[k]^(1 - alpha).
//  k_permute      Y[m][j] = X[m][perm[j]] (divided or multiplied by s[perm[j]]).
// k_token_linf + k_extreme_pick (L <= K), k_extreme_v, k_householder_v,
// k_col_absmax_v and k_permute_rows are the same operations with 16-byte loads, taken when X is 16-byte aligned, its row stride
// a multiple of 16 bytes and K a multiple of 8.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "hq_device.cuh"

namespace hq {

namespace cb {
constexpr int THREADS = 256;
constexpr int PCA_THREADS = 1024;
constexpr int EXT_THREADS = 1024;
constexpr int CL = 8;               // CTAs of the cluster power iteration
constexpr int PCL_THREADS = 512;
constexpr int SMEM_MAX = 227 * 1024;
}  // namespace cb

__device__ __forceinline__ float cb_load(const void* X, int xt, int64_t i) {
    if (xt == HQ_F16) return __half2float(reinterpret_cast<const __half*>(X)[i]);
    if (xt == HQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(X)[i]);
    return reinterpret_cast<const float*>(X)[i];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Sum over the CTA of one value per thread, in a fixed order; every thread
// gets the result.  red: shared, >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();   // red may still be read by a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : 0.f;
    return warp_sum(t);
}

// ---------------------------------------------------------------- k_extreme
__global__ void __launch_bounds__(cb::THREADS) k_extreme(const void* __restrict__ X, int xt, int L, int K,
                                                        int64_t ldx, int32_t* __restrict__ tok,
                                                        float* __restrict__ T) {
    __shared__ float bv[cb::THREADS / 32];
    __shared__ int bi[cb::THREADS / 32];
    const int s = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int64_t row0 = static_cast<int64_t>(s) * L;
    // each warp scans tokens warp, warp + nw, ... in increasing order: a later
    // token replaces the warp's best only when strictly larger
    float best = -1.f;
    int besti = 0;
    for (int t = warp; t < L; t += nw) {
        const int64_t base = (row0 + t) * ldx;
        float m = 0.f;
        for (int k = lane; k < K; k += 32) m = fmaxf(m, fabsf(cb_load(X, xt, base + k)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (m > best) {
            best = m;
            besti = t;
        }
    }
    if (lane == 0) {
        bv[warp] = best;
        bi[warp] = besti;
    }
    __syncthreads();
    float b = bv[0];
    int bidx = bi[0];
    for (int w = 1; w < nw; ++w)
        if (bv[w] > b || (bv[w] == b && bi[w] < bidx)) {
            b = bv[w];
            bidx = bi[w];
        }
    if (threadIdx.x == 0) tok[s] = bidx;
    const int64_t src = (row0 + bidx) * ldx;
    for (int k = threadIdx.x; k < K; k += blockDim.x)
        T[static_cast<int64_t>(s) * K + k] = cb_load(X, xt, src + k);
}

// ---------------------------------------------------------------- 16-byte paths
// Used when X is 16-byte aligned, its row stride a multiple of 16 bytes and K a
// multiple of 8: element i (a multiple of 8) starts an aligned 16-byte (16-bit
// types) or 32-byte (fp32) chunk of 8 values.
__device__ __forceinline__ void cb_load8(const void* X, int xt, int64_t i, float (&f)[8]) {
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

// k_extreme with 1024 threads and four 16-byte chunks per lane in flight.
__global__ void __launch_bounds__(cb::EXT_THREADS) k_extreme_v(const void* __restrict__ X, int xt, int L, int K,
                                                              int64_t ldx, int32_t* __restrict__ tok,
                                                              float* __restrict__ T) {
    __shared__ float bv[cb::EXT_THREADS / 32];
    __shared__ int bi[cb::EXT_THREADS / 32];
    const int s = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int64_t row0 = static_cast<int64_t>(s) * L;
    float best = -1.f;
    int besti = 0;
    for (int t = warp; t < L; t += nw) {
        const int64_t base = (row0 + t) * ldx;
        float m = 0.f;
        for (int k0 = 8 * lane; k0 < K; k0 += 4 * 256) {
            float f[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (k0 + 256 * u < K) cb_load8(X, xt, base + k0 + 256 * u, f[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (k0 + 256 * u < K)
#pragma unroll
                    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[u][e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (m > best) {
            best = m;
            besti = t;
        }
    }
    if (lane == 0) {
        bv[warp] = best;
        bi[warp] = besti;
    }
    __syncthreads();
    float b = bv[0];
    int bidx = bi[0];
    for (int w = 1; w < nw; ++w)
        if (bv[w] > b || (bv[w] == b && bi[w] < bidx)) {
            b = bv[w];
            bidx = bi[w];
        }
    if (threadIdx.x == 0) tok[s] = bidx;
    const int64_t src = (row0 + bidx) * ldx;
    float* dst = T + static_cast<int64_t>(s) * K;
    for (int k0 = 8 * threadIdx.x; k0 < K; k0 += 8 * blockDim.x) {
        float f[8];
        cb_load8(X, xt, src + k0, f);
        *reinterpret_cast<float4*>(dst + k0) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(dst + k0 + 4) = make_float4(f[4], f[5], f[6], f[7]);
    }
}

// The extreme tokens in two launches when L <= K (the usual case): k_token_linf
// gives every token its own warp (max |x| with 16-byte loads) and parks the
// results of sequence s in T's row s; k_extreme_pick (one CTA per sequence)
// reads them, takes the first maximum, and only then overwrites the row with
// the chosen token.
__global__ void __launch_bounds__(cb::THREADS) k_token_linf(const void* __restrict__ X, int xt, int S, int L, int K,
                                                           int64_t ldx, float* __restrict__ T) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= static_cast<int64_t>(S) * L) return;   // whole warps
    const int64_t base = t * ldx;
    float m = 0.f;
    for (int k0 = 8 * lane; k0 < K; k0 += 4 * 256) {
        float f[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (k0 + 256 * u < K) cb_load8(X, xt, base + k0 + 256 * u, f[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (k0 + 256 * u < K)
#pragma unroll
                for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[u][e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int64_t s = t / L, l = t - s * L;
    if (lane == 0) T[s * K + l] = m;
}

__global__ void __launch_bounds__(cb::EXT_THREADS) k_extreme_pick(const void* __restrict__ X, int xt, int L, int K,
                                                                 int64_t ldx, int32_t* __restrict__ tok,
                                                                 float* __restrict__ T) {
    __shared__ float bv[cb::EXT_THREADS / 32];
    __shared__ int bi[cb::EXT_THREADS / 32];
    const int s = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    float* row = T + static_cast<int64_t>(s) * K;
    float best = -1.f;
    int besti = 0;
    for (int l = threadIdx.x; l < L; l += blockDim.x) {   // increasing l per thread: strict > keeps the first
        const float m = row[l];
        if (m > best) {
            best = m;
            besti = l;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, besti, o);
        if (ob > best || (ob == best && oi < besti)) {
            best = ob;
            besti = oi;
        }
    }
    if (lane == 0) {
        bv[warp] = best;
        bi[warp] = besti;
    }
    __syncthreads();   // every read of the row is done before it is overwritten
    float b = bv[0];
    int bidx = bi[0];
    for (int w = 1; w < nw; ++w)
        if (bv[w] > b || (bv[w] == b && bi[w] < bidx)) {
            b = bv[w];
            bidx = bi[w];
        }
    if (threadIdx.x == 0) tok[s] = bidx;
    const int64_t src = (static_cast<int64_t>(s) * L + bidx) * ldx;
    for (int k0 = 8 * threadIdx.x; k0 < K; k0 += 8 * blockDim.x) {
        float f[8];
        cb_load8(X, xt, src + k0, f);
        *reinterpret_cast<float4*>(row + k0) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(row + k0 + 4) = make_float4(f[4], f[5], f[6], f[7]);
    }
}

// ---------------------------------------------------------------- k_top1_pca
// Shared memory: v [K] | y [S] | red [32].
__global__ void __launch_bounds__(cb::PCA_THREADS, 1)
    k_top1_pca(const float* __restrict__ T, int S, int K, int iters, float* __restrict__ vout,
               float* __restrict__ lam) {
    extern __shared__ float sm[];
    float* v = sm;
    float* y = sm + K;
    float* red = y + S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const float invS = __fdiv_rn(1.0f, static_cast<float>(S));

    // start: the calibration token of largest L2 norm (ties to the earlier one)
    for (int s = warp; s < S; s += nw) {
        float a = 0.f;
        for (int k = lane; k < K; k += 32) {
            const float t = T[static_cast<int64_t>(s) * K + k];
            a = __fmaf_rn(t, t, a);
        }
        a = warp_sum(a);
        if (lane == 0) y[s] = a;
    }
    __syncthreads();
    int s0 = 0;
    for (int s = 1; s < S; ++s)
        if (y[s] > y[s0]) s0 = s;
    const float n0 = y[s0];
    __syncthreads();
    float norm = 0.f;   // |C v| of the last iteration (0 before the first)
    bool dead = !(n0 > 0.f);
    if (!dead) {
        const float inv = __fdiv_rn(1.0f, sqrtf(n0));
        for (int k = threadIdx.x; k < K; k += blockDim.x) v[k] = __fmul_rn(T[static_cast<int64_t>(s0) * K + k], inv);
        __syncthreads();
        for (int it = 0; it < iters; ++it) {
            // y = T v
            for (int s = warp; s < S; s += nw) {
                float a = 0.f;
                for (int k = lane; k < K; k += 32) a = __fmaf_rn(T[static_cast<int64_t>(s) * K + k], v[k], a);
                a = warp_sum(a);
                if (lane == 0) y[s] = a;
            }
            __syncthreads();
            // z = T^T y / S (into v: every y has been formed), |z|
            float sq = 0.f;
            for (int k = threadIdx.x; k < K; k += blockDim.x) {
                float z = 0.f;
                for (int s = 0; s < S; ++s) z = __fmaf_rn(T[static_cast<int64_t>(s) * K + k], y[s], z);
                z = __fmul_rn(z, invS);
                v[k] = z;
                sq = __fmaf_rn(z, z, sq);
            }
            norm = sqrtf(block_sum(sq, red));
            if (norm == 0.f) {
                dead = true;
                break;
            }
            const float inv = __fdiv_rn(1.0f, norm);
            for (int k = threadIdx.x; k < K; k += blockDim.x) v[k] = __fmul_rn(v[k], inv);
            __syncthreads();
        }
    }
    if (dead) {
        // no direction (all-zero tokens, or T v = 0): e0
        __syncthreads();
        for (int k = threadIdx.x; k < K; k += blockDim.x) v[k] = k == 0 ? 1.f : 0.f;
        norm = 0.f;
    }
    __syncthreads();
    // sign: the component of largest magnitude is positive (ties to the lower index)
    if (threadIdx.x == 0) {
        int kb = 0;
        for (int k = 1; k < K; ++k)
            if (fabsf(v[k]) > fabsf(v[kb])) kb = k;
        red[0] = v[kb] < 0.f ? -1.f : 1.f;
        *lam = norm;
    }
    __syncthreads();
    const float sg = red[0];
    for (int k = threadIdx.x; k < K; k += blockDim.x) vout[k] = __fmul_rn(v[k], sg);
}

// ---------------------------------------------------------------- k_top1_pca_cl
// The same power iteration on a cluster of cb::CL CTAs when the S tokens fit in
// their shared memory: CTA c holds columns [c Kc, c Kc + Kc) of T and of v, so
// an iteration reads shared memory only.  y = T v is summed over the cluster
// (each CTA reads every CTA's partial through distributed shared memory, in
// rank order, so all CTAs hold the same y), z = T^T y is local, |z|^2 is summed
// over the cluster the same way.  Partials are double-buffered by use count,
// so one hardware cluster barrier per reduction suffices.
// Shared memory: Ts [S][Kc] | v [Kc] | yp [2][S] | y [S] | red [32] | sc [2] | fin [2]
__device__ __forceinline__ float ld_dsmem_f32(uint32_t caddr) {
    float r;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(r) : "r"(caddr) : "memory");
    return r;
}

__global__ void __launch_bounds__(cb::PCL_THREADS, 1)
    k_top1_pca_cl(const float* __restrict__ T, int S, int K, int Kc, int iters, float* __restrict__ vout,
                  float* __restrict__ lam) {
    extern __shared__ float sm[];
    float* Ts = sm;
    float* v = Ts + static_cast<int64_t>(S) * Kc;
    float* yp = v + Kc;
    float* y = yp + 2 * S;
    float* red = y + S;
    float* sc = red + 32;
    float* fin = sc + 2;
    const int rank = static_cast<int>(cluster_ctarank());
    const int k0 = rank * Kc;
    const int kn = K - k0 < Kc ? (K - k0 > 0 ? K - k0 : 0) : Kc;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const float invS = __fdiv_rn(1.0f, static_cast<float>(S));

    for (int i = threadIdx.x; i < S * kn; i += blockDim.x) {
        const int s = i / kn, j = i - s * kn;
        Ts[s * Kc + j] = T[static_cast<int64_t>(s) * K + k0 + j];
    }
    __syncthreads();

    int ny = 0, nsq = 0;   // uses of yp and of sc (buffer = count & 1)
    // y[s] = sum over the cluster of the partials p[s] written by this CTA
    auto cluster_vec = [&](auto partial) {
        float* b = yp + (ny & 1) * S;
        for (int s = warp; s < S; s += nw) {
            const float a = warp_sum(partial(s));
            if (lane == 0) b[s] = a;
        }
        ++ny;
        cluster_sync();
        const uint32_t base = smem_u32(b);
        for (int s = threadIdx.x; s < S; s += blockDim.x) {
            float a = 0.f;
            for (int r = 0; r < cb::CL; ++r) a = __fadd_rn(a, ld_dsmem_f32(mapa_shared(base + 4u * s, r)));
            y[s] = a;
        }
        __syncthreads();
    };
    auto cluster_scalar = [&](float part) {
        const float t = block_sum(part, red);
        float* b = sc + (nsq & 1);
        if (threadIdx.x == 0) *b = t;
        ++nsq;
        cluster_sync();
        float a = 0.f;
        for (int r = 0; r < cb::CL; ++r) a = __fadd_rn(a, ld_dsmem_f32(mapa_shared(smem_u32(b), r)));
        return a;
    };

    // start: the token of largest L2 norm (ties to the earlier one)
    cluster_vec([&](int s) {
        float a = 0.f;
        for (int j = lane; j < kn; j += 32) a = __fmaf_rn(Ts[s * Kc + j], Ts[s * Kc + j], a);
        return a;
    });
    int s0 = 0;
    for (int s = 1; s < S; ++s)
        if (y[s] > y[s0]) s0 = s;
    const float n0 = y[s0];
    float norm = 0.f;
    bool dead = !(n0 > 0.f);
    if (!dead) {
        const float inv = __fdiv_rn(1.0f, sqrtf(n0));
        for (int j = threadIdx.x; j < kn; j += blockDim.x) v[j] = __fmul_rn(Ts[s0 * Kc + j], inv);
        __syncthreads();
        for (int it = 0; it < iters; ++it) {
            cluster_vec([&](int s) {
                float a = 0.f;
                for (int j = lane; j < kn; j += 32) a = __fmaf_rn(Ts[s * Kc + j], v[j], a);
                return a;
            });
            float sq = 0.f;
            for (int j = threadIdx.x; j < kn; j += blockDim.x) {
                float z = 0.f;
                for (int s = 0; s < S; ++s) z = __fmaf_rn(Ts[s * Kc + j], y[s], z);
                z = __fmul_rn(z, invS);
                v[j] = z;
                sq = __fmaf_rn(z, z, sq);
            }
            norm = sqrtf(cluster_scalar(sq));
            if (norm == 0.f) {
                dead = true;
                break;
            }
            const float inv = __fdiv_rn(1.0f, norm);
            for (int j = threadIdx.x; j < kn; j += blockDim.x) v[j] = __fmul_rn(v[j], inv);
            __syncthreads();
        }
    }
    if (dead) {
        __syncthreads();
        for (int j = threadIdx.x; j < kn; j += blockDim.x) v[j] = (k0 + j == 0) ? 1.f : 0.f;
        norm = 0.f;
    }
    __syncthreads();
    // sign: the component of largest magnitude over the whole vector is positive
    if (threadIdx.x == 0) {
        int jb = 0;
        for (int j = 1; j < kn; ++j)
            if (fabsf(v[j]) > fabsf(v[jb])) jb = j;
        fin[0] = kn > 0 ? fabsf(v[jb]) : -1.f;
        fin[1] = kn > 0 ? (v[jb] < 0.f ? -1.f : 1.f) : 1.f;
    }
    cluster_sync();
    if (threadIdx.x == 0) {
        float best = -1.f, sg = 1.f;
        for (int r = 0; r < cb::CL; ++r) {   // ranks in order: the lower index wins ties
            const float a = ld_dsmem_f32(mapa_shared(smem_u32(fin), r));
            if (a > best) {
                best = a;
                sg = ld_dsmem_f32(mapa_shared(smem_u32(fin + 1), r));
            }
        }
        red[0] = sg;
        if (rank == 0) *lam = norm;
    }
    __syncthreads();
    const float sg = red[0];
    for (int j = threadIdx.x; j < kn; j += blockDim.x) vout[k0 + j] = __fmul_rn(v[j], sg);
    // no CTA leaves while another may still read its shared memory
    cluster_sync();
}

// ---------------------------------------------------------------- k_householder
// Shared memory: w [K] | red [32]
__global__ void __launch_bounds__(cb::THREADS) k_householder(const void* __restrict__ X, int xt, int M, int K,
                                                            int64_t ldx, const float* __restrict__ v,
                                                            float* __restrict__ Y) {
    extern __shared__ float sm[];
    float* w = sm;
    float* red = sm + K;
    const float sg = v[0] > 0.f ? -1.f : 1.f;   // v' = sg v has v'[0] <= 0
    float sq = 0.f;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float e = __fmul_rn(sg, v[k]);
        const float wk = k == 0 ? __fsub_rn(e, 1.0f) : e;
        w[k] = wk;
        sq = __fmaf_rn(wk, wk, sq);
    }
    const float ww = block_sum(sq, red);   // >= 1 for a unit v (|w0| >= 1)
    const float two_over = __fdiv_rn(2.0f, ww);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int m = blockIdx.x * nw + warp; m < M; m += gridDim.x * nw) {
        const int64_t base = static_cast<int64_t>(m) * ldx;
        float d = 0.f;
        for (int k = lane; k < K; k += 32) d = __fmaf_rn(cb_load(X, xt, base + k), w[k], d);
        d = warp_sum(d);
        const float c = __fmul_rn(two_over, d);
        float* yr = Y + static_cast<int64_t>(m) * K;
        for (int k = lane; k < K; k += 32) yr[k] = __fsub_rn(cb_load(X, xt, base + k), __fmul_rn(c, w[k]));
    }
}

// k_householder over 8-value chunks, one CTA per row: the dot product
// (thread-strided chunks, then a block sum in a fixed order), then
// y = x - c w chunk by chunk (the row is read again, from L2).  Shared memory:
// w [K] | red [32].
__global__ void __launch_bounds__(cb::THREADS) k_householder_v(const void* __restrict__ X, int xt, int M, int K,
                                                              int64_t ldx, const float* __restrict__ v,
                                                              float* __restrict__ Y) {
    extern __shared__ float sm[];
    float* w = sm;
    float* red = sm + K;
    const float sg = v[0] > 0.f ? -1.f : 1.f;
    float sq = 0.f;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float e = __fmul_rn(sg, v[k]);
        const float wk = k == 0 ? __fsub_rn(e, 1.0f) : e;
        w[k] = wk;
        sq = __fmaf_rn(wk, wk, sq);
    }
    const float ww = block_sum(sq, red);
    const float two_over = __fdiv_rn(2.0f, ww);
    // one CTA per row: the row's chunks are spread over all threads, so each
    // thread walks only K / (8 * blockDim) chunks per pass
    const int step = 8 * blockDim.x;
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const int64_t base = static_cast<int64_t>(m) * ldx;
        float d = 0.f;
        for (int k0 = 8 * threadIdx.x; k0 < K; k0 += step) {
            float f[8];
            cb_load8(X, xt, base + k0, f);
            const float4 wa = *reinterpret_cast<const float4*>(w + k0);
            const float4 wb = *reinterpret_cast<const float4*>(w + k0 + 4);
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) d = __fmaf_rn(f[e], wv[e], d);
        }
        d = block_sum(d, red);
        const float c = __fmul_rn(two_over, d);
        float* yr = Y + static_cast<int64_t>(m) * K;
        for (int k0 = 8 * threadIdx.x; k0 < K; k0 += step) {
            float f[8];
            cb_load8(X, xt, base + k0, f);
            const float4 wa = *reinterpret_cast<const float4*>(w + k0);
            const float4 wb = *reinterpret_cast<const float4*>(w + k0 + 4);
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = __fsub_rn(f[e], __fmul_rn(c, wv[e]));
            *reinterpret_cast<float4*>(yr + k0) = make_float4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<float4*>(yr + k0 + 4) = make_float4(o[4], o[5], o[6], o[7]);
        }
    }
}

// k_col_absmax over 8-column chunks: thread t of the strip owns columns
// [8 t, 8 t + 8).
__global__ void __launch_bounds__(cb::THREADS) k_col_absmax_v(const void* __restrict__ X, int xt, int M, int K,
                                                             int64_t ldx, int rows_per,
                                                             unsigned int* __restrict__ out) {
    const int k0 = 8 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (k0 >= K) return;
    const int m0 = blockIdx.y * rows_per;
    const int m1 = min(M, m0 + rows_per);
    float mx[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int r = m0;
    for (; r + 1 < m1; r += 2) {
        float f[2][8];
        cb_load8(X, xt, static_cast<int64_t>(r) * ldx + k0, f[0]);
        cb_load8(X, xt, static_cast<int64_t>(r + 1) * ldx + k0, f[1]);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fmaxf(fabsf(f[0][e]), fabsf(f[1][e])));
    }
    if (r < m1) {
        float f[8];
        cb_load8(X, xt, static_cast<int64_t>(r) * ldx + k0, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], fabsf(f[e]));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicMax(out + k0 + e, __float_as_uint(mx[e]));
}

// ---------------------------------------------------------------- k_col_absmax
__global__ void __launch_bounds__(cb::THREADS) k_col_absmax(const void* __restrict__ X, int xt, int M, int K,
                                                           int64_t ldx, int rows_per, unsigned int* __restrict__ out) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    const int m0 = blockIdx.y * rows_per;
    const int m1 = min(M, m0 + rows_per);
    float m = 0.f;
    for (int r = m0; r < m1; ++r) m = fmaxf(m, fabsf(cb_load(X, xt, static_cast<int64_t>(r) * ldx + k)));
    // fmaxf skips NaN, so m is a non-negative number: its bit pattern orders as its value
    atomicMax(out + k, __float_as_uint(m));
}

// ---------------------------------------------------------------- k_rank
// NaN ranks as -inf.
__device__ __forceinline__ float cb_key(float x) { return x != x ? -INFINITY : x; }

__global__ void __launch_bounds__(cb::THREADS) k_rank(const float* __restrict__ stat, int K, int32_t* __restrict__ perm) {
    __shared__ float tile[cb::THREADS];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const float si = i < K ? cb_key(stat[i]) : 0.f;
    int rank = 0;
    for (int j0 = 0; j0 < K; j0 += cb::THREADS) {
        __syncthreads();
        const int j = j0 + threadIdx.x;
        tile[threadIdx.x] = j < K ? cb_key(stat[j]) : 0.f;
        __syncthreads();
        const int n = min(cb::THREADS, K - j0);
        for (int t = 0; t < n; ++t) {
            const float sj = tile[t];
            rank += (sj > si || (sj == si && j0 + t < i)) ? 1 : 0;
        }
    }
    if (i < K) perm[rank] = i;
}

// ---------------------------------------------------------------- k_flatten
__global__ void k_flatten(const float* __restrict__ xmax, const float* __restrict__ wmax, int K, float alpha,
                          float* __restrict__ s) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    const float xm = xmax[k], wm = wmax[k];
    // a channel with no activation or no weight range keeps the scale 1
    s[k] = (xm > 0.f && wm > 0.f) ? __fdiv_rn(powf(xm, alpha), powf(wm, 1.0f - alpha)) : 1.0f;
}

// ---------------------------------------------------------------- k_permute
// op: 0 copy, 1 divide by s, 2 multiply by s.  An index outside [0, K) records
// HQ_ERR_ARG in the device status word and writes 0.
__global__ void __launch_bounds__(cb::THREADS) k_permute(const void* __restrict__ X, int xt, int M, int K,
                                                        int64_t ldx, const int32_t* __restrict__ perm,
                                                        const float* __restrict__ s, int op, float* __restrict__ Y) {
    const int64_t total = static_cast<int64_t>(M) * K;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / K;
        const int j = static_cast<int>(i - m * K);
        const int c = perm ? perm[j] : j;
        float y = 0.f;
        if (c < 0 || c >= K) {
            record_status(HQ_ERR_ARG);
        } else {
            y = cb_load(X, xt, m * ldx + c);
            if (op == 1) y = __fdiv_rn(y, s[c]);
            else if (op == 2) y = __fmul_rn(y, s[c]);
        }
        Y[i] = y;
    }
}

// k_permute with the source row staged in shared memory (16-byte loads), then
// gathered from there; four outputs per thread, one 16-byte store.  One CTA per
// row at a time.  Shared memory: row [K] floats.
__global__ void __launch_bounds__(cb::THREADS) k_permute_rows(const void* __restrict__ X, int xt, int M, int K,
                                                             int64_t ldx, const int32_t* __restrict__ perm,
                                                             const float* __restrict__ s, int op,
                                                             float* __restrict__ Y) {
    extern __shared__ float srow[];
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const int64_t base = static_cast<int64_t>(m) * ldx;
        for (int k0 = 8 * threadIdx.x; k0 < K; k0 += 8 * blockDim.x) {
            float f[8];
            cb_load8(X, xt, base + k0, f);
            *reinterpret_cast<float4*>(srow + k0) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(srow + k0 + 4) = make_float4(f[4], f[5], f[6], f[7]);
        }
        __syncthreads();
        float* yr = Y + static_cast<int64_t>(m) * K;
        for (int j0 = 4 * threadIdx.x; j0 < K; j0 += 4 * blockDim.x) {
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = perm ? perm[j0 + e] : j0 + e;
                float y = 0.f;
                if (c < 0 || c >= K) {
                    record_status(HQ_ERR_ARG);
                } else {
                    y = srow[c];
                    if (op == 1) y = __fdiv_rn(y, s[c]);
                    else if (op == 2) y = __fmul_rn(y, s[c]);
                }
                o[e] = y;
            }
            *reinterpret_cast<float4*>(yr + j0) = make_float4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();   // the row is read before the next one is staged
    }
}

static int cb_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

static bool cb_dtype_ok(hq_dtype t) { return t == HQ_F16 || t == HQ_BF16 || t == HQ_F32; }
static hq_status cb_launched() { return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA; }
static bool cb_al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// the 16-byte paths: X aligned, row stride a multiple of 16 bytes, K a multiple of 8
static bool cb_vec(const void* X, hq_dtype xt, int64_t K, int64_t ld_x) {
    const int64_t es = xt == HQ_F32 ? 4 : 2;
    return cb_al16(X) && (ld_x * es) % 16 == 0 && K % 8 == 0;
}

}  // namespace hq

using namespace hq;

extern "C" hq_status hq_calib_extreme_tokens(const void* X, hq_dtype xt, int64_t S, int64_t L, int64_t K,
                                             int64_t ld_x, int32_t* tok, float* T, void* stream) {
    if (!cb_dtype_ok(xt) || S < 0 || L <= 0 || K <= 0 || ld_x < K) return HQ_ERR_ARG;
    if (S > INT32_MAX || L > INT32_MAX || K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    if (S == 0) return HQ_OK;
    if (!X || !tok || !T) return HQ_ERR_ARG;
    if (cb_vec(X, xt, K, ld_x) && cb_al16(T) && L <= K) {
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        const int64_t warps = S * L;
        const int64_t grid = (warps + cb::THREADS / 32 - 1) / (cb::THREADS / 32);
        if (grid > INT32_MAX) return HQ_ERR_UNSUPPORTED;
        k_token_linf<<<static_cast<unsigned>(grid), cb::THREADS, 0, st>>>(X, xt, static_cast<int>(S),
                                                                          static_cast<int>(L), static_cast<int>(K),
                                                                          ld_x, T);
        k_extreme_pick<<<static_cast<unsigned>(S), cb::EXT_THREADS, 0, st>>>(X, xt, static_cast<int>(L),
                                                                             static_cast<int>(K), ld_x, tok, T);
        return cb_launched();
    }
    if (cb_vec(X, xt, K, ld_x) && cb_al16(T))
        k_extreme_v<<<static_cast<unsigned>(S), cb::EXT_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
            X, xt, static_cast<int>(L), static_cast<int>(K), ld_x, tok, T);
    else
        k_extreme<<<static_cast<unsigned>(S), cb::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
            X, xt, static_cast<int>(L), static_cast<int>(K), ld_x, tok, T);
    return cb_launched();
}

extern "C" size_t hq_calib_pca_max_elems(void) { return (cb::SMEM_MAX - 32 * 4) / 4; }

extern "C" hq_status hq_calib_top1_pca(const float* T, int64_t S, int64_t K, int32_t iters, float* v, float* lambda,
                                       void* stream) {
    if (S <= 0 || K <= 0 || iters < 0 || !T || !v || !lambda) return HQ_ERR_ARG;
    if (static_cast<uint64_t>(S) + static_cast<uint64_t>(K) > hq_calib_pca_max_elems()) return HQ_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the tokens fit in the shared memory of a cluster: every iteration runs from shared memory
    const int64_t Kc = ((K + cb::CL - 1) / cb::CL + 3) / 4 * 4;
    const int64_t cl_smem = (S * Kc + Kc + 3 * S + 32 + 4) * 4;
    if (cl_smem <= cb::SMEM_MAX - 1024) {
        const int sm = static_cast<int>(cl_smem);
        if (cudaFuncSetAttribute(k_top1_pca_cl, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess)
            return HQ_ERR_CUDA;
        cudaLaunchConfig_t cfg{};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cb::CL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(cb::CL, 1, 1);
        cfg.blockDim = dim3(cb::PCL_THREADS, 1, 1);
        cfg.dynamicSmemBytes = sm;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, k_top1_pca_cl, T, static_cast<int>(S), static_cast<int>(K),
                               static_cast<int>(Kc), static_cast<int>(iters), v, lambda) != cudaSuccess)
            return HQ_ERR_CUDA;
        return cb_launched();
    }
    const int smem = static_cast<int>((S + K + 32) * 4);
    if (cudaFuncSetAttribute(k_top1_pca, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    k_top1_pca<<<1, cb::PCA_THREADS, smem, st>>>(T, static_cast<int>(S), static_cast<int>(K), iters, v, lambda);
    return cb_launched();
}

extern "C" hq_status hq_calib_householder(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                                          const float* v, float* Y, void* stream) {
    if (!cb_dtype_ok(xt) || M < 0 || K <= 0 || ld_x < K) return HQ_ERR_ARG;
    if (M > INT32_MAX || K + 32 > (cb::SMEM_MAX / 4)) return HQ_ERR_UNSUPPORTED;
    if (M == 0) return HQ_OK;
    if (!X || !v || !Y) return HQ_ERR_ARG;
    const int smem = static_cast<int>((K + 32) * 4);
    const bool vec = cb_vec(X, xt, K, ld_x) && cb_al16(Y);
    auto kern = vec ? k_householder_v : k_householder;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    // warp per row (element-wise kernel) or CTA per row (16-byte kernel)
    const int64_t want = vec ? M : (M + cb::THREADS / 32 - 1) / (cb::THREADS / 32);
    const int64_t cap = (vec ? 8 : 4) * static_cast<int64_t>(cb_sm_count());
    const int grid = static_cast<int>(want < cap ? want : cap);
    kern<<<grid, cb::THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
        X, xt, static_cast<int>(M), static_cast<int>(K), ld_x, v, Y);
    return cb_launched();
}

extern "C" hq_status hq_calib_channel_absmax(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                                             float* amax, void* stream) {
    if (!cb_dtype_ok(xt) || M < 0 || K <= 0 || ld_x < K || !amax) return HQ_ERR_ARG;
    if (M > INT32_MAX || K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    if (M > 0 && !X) return HQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax, 0, static_cast<size_t>(K) * sizeof(float), st) != cudaSuccess) return HQ_ERR_CUDA;
    if (M == 0) return HQ_OK;
    const bool vec = cb_vec(X, xt, K, ld_x);
    const int64_t cols_per = vec ? 8 * cb::THREADS : cb::THREADS;   // columns per CTA strip
    const int gx = static_cast<int>((K + cols_per - 1) / cols_per);
    // about four CTAs per SM in all, each over a contiguous run of rows
    int gy = (4 * cb_sm_count() + gx - 1) / gx;
    if (gy > M) gy = static_cast<int>(M);
    const int rows_per = static_cast<int>((M + gy - 1) / gy);
    gy = static_cast<int>((M + rows_per - 1) / rows_per);
    (vec ? k_col_absmax_v : k_col_absmax)<<<dim3(gx, gy), cb::THREADS, 0, st>>>(
        X, xt, static_cast<int>(M), static_cast<int>(K), ld_x, rows_per, reinterpret_cast<unsigned int*>(amax));
    return cb_launched();
}

extern "C" hq_status hq_calib_sorted_perm(const float* stat, int64_t K, int32_t* perm, void* stream) {
    if (K <= 0 || !stat || !perm) return HQ_ERR_ARG;
    if (K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    k_rank<<<static_cast<unsigned>((K + cb::THREADS - 1) / cb::THREADS), cb::THREADS, 0,
             static_cast<cudaStream_t>(stream)>>>(stat, static_cast<int>(K), perm);
    return cb_launched();
}

extern "C" hq_status hq_calib_flatten_scales(const float* xmax, const float* wmax, int64_t K, float alpha, float* s,
                                             void* stream) {
    if (K <= 0 || !xmax || !wmax || !s || !(alpha >= 0.f && alpha <= 1.f)) return HQ_ERR_ARG;
    if (K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    k_flatten<<<static_cast<unsigned>((K + cb::THREADS - 1) / cb::THREADS), cb::THREADS, 0,
                static_cast<cudaStream_t>(stream)>>>(xmax, wmax, static_cast<int>(K), alpha, s);
    return cb_launched();
}

extern "C" hq_status hq_permute_channels(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                                         const int32_t* perm, const float* s, int32_t op, float* Y, void* stream) {
    if (!cb_dtype_ok(xt) || M < 0 || K <= 0 || ld_x < K || op < 0 || op > 2) return HQ_ERR_ARG;
    if (M > INT32_MAX || K > INT32_MAX) return HQ_ERR_UNSUPPORTED;
    if (M == 0) return HQ_OK;
    if (!X || !Y || (op != 0 && !s)) return HQ_ERR_ARG;
    if (cb_vec(X, xt, K, ld_x) && cb_al16(Y) && K * 4 <= cb::SMEM_MAX - 1024) {
        // the source row staged in shared memory, gathered from there
        const int smem = static_cast<int>(K * 4);
        if (cudaFuncSetAttribute(k_permute_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return HQ_ERR_CUDA;
        const int grid = static_cast<int>(M < 4 * cb_sm_count() ? M : 4 * cb_sm_count());
        k_permute_rows<<<grid, cb::THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
            X, xt, static_cast<int>(M), static_cast<int>(K), ld_x, perm, s, op, Y);
        return cb_launched();
    }
    const int64_t blocks = (M * K + cb::THREADS - 1) / cb::THREADS;
    const int grid = static_cast<int>(blocks < 8 * cb_sm_count() ? blocks : 8 * cb_sm_count());
    k_permute<<<grid, cb::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        X, xt, static_cast<int>(M), static_cast<int>(K), ld_x, perm, s, op, Y);
    return cb_launched();
}
