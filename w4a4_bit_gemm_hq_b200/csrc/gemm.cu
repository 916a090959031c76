// gemm.cu -- kernel K2: the W4A4 GEMM with SERQ's fused rank-r term, on the
// sm_100a tensor cores (tcgen05.mma kind::i8, int32 accumulators in tensor
// memory), for the large-M (prefill) shapes.
//
// Source: "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
// Quantization", technical summary section 2.2 (the linear layer on 4-bit
// operands plus one residual path over the salient rows, X[:,S] R^T, also in
// 4 bit) and section 3 (a single 4-bit matmul: no sequential low-rank factors,
// no intermediate quantisation); "OffQ: Taming Structured Outliers in LLM
// Quantization by Offsetting", Methodology 3 (group-wise scale and zero point).
//
// Design (one CTA per SM, persistent over 128 x BN output tiles):
//  * tcgen05 has no int4 MMA, so 7 producer warps read the packed codes with
//    16-byte loads (prefetched one stage ahead in registers), expand them to
//    int8 in registers (16*q for activations and symmetric weights, u - z for
//    asymmetric weights) and store them into 128-byte-swizzled K-major smem
//    tiles: A = 128 activation rows x 128 K, B = BN weight rows x 128 K.
//  * one thread issues tcgen05.mma (M=128, N=BN, K=32) x 4 per stage into a
//    double-buffered int32 accumulator in tensor memory; tcgen05.commit frees
//    the smem stage and, at the end of a tile (per-channel weights) or of a
//    weight group (group weights), hands the accumulator to the epilogue.
//  * 8 epilogue warps (2 per TMEM lane quarter, splitting the columns) load
//    the accumulator with tcgen05.ld, dequantise with sx[m] * sw[n] (or sum the
//    per-group sw[b][n] * acc_b), add sr[n] * (X[m,S] . Rq[n,:]) computed with
//    dp4a (the SERQ term as an epilogue add: no second launch), round once and
//    store.
//  * every mbarrier wait is bounded; on timeout the status word records
//    HQ_ERR_TIMEOUT and the roles skip to teardown, which waits for in-flight
//    MMAs before freeing tensor memory.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "hq_device.cuh"
#include "hq_gemm.cuh"

namespace hq {

namespace pf {
constexpr int BM = 128;
constexpr int BK = 128;               // int8 K per stage = one 128-byte swizzle row
constexpr int THREADS = 512;
constexpr int MMA_WARP = 4;
constexpr int EPI_WARP0 = 8;
constexpr int NPROD = 7 * 32;         // producer threads: warps 0-3 and 5-7
constexpr int RQ_LD = 64;             // bytes per unpacked Rq row (r <= 64) in the per-warp scratch
}  // namespace pf

// Shared memory: an int8 operand ring read by the tensor core (STAGES deep) and
// a packed-code ring (PD deep) that each producer thread fills with cp.async
// for its own 16-byte chunks (and, for group weights, the zero-point pair of
// its weight row), PD stages ahead of their use.
template <int BN, bool ASYM>
struct PfSmem {
    static constexpr int STAGES = (BN == 256) ? 2 : 3;
    static constexpr int PD = (BN == 256) ? 4 : 5;
    static constexpr int A_BYTES = pf::BM * pf::BK;
    static constexpr int B_BYTES = BN * pf::BK;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NCHUNK = (pf::BM + BN) * 4;                   // 16-byte packed chunks per stage
    static constexpr int NCH = (NCHUNK + pf::NPROD - 1) / pf::NPROD;  // per producer thread
    static constexpr int PK_DATA = NCHUNK * 16;
    static constexpr int PK_Z = ASYM ? BN * 4 * 4 : 0;                 // zero-point pair per weight chunk
    static constexpr int PK_STAGE = ((PK_DATA + PK_Z) + 127) / 128 * 128;
    static constexpr int OFF_PK = STAGES * STAGE;
    static constexpr int OFF_RQ = OFF_PK + PD * PK_STAGE;              // 8 warps x 32 rows x RQ_LD
    static constexpr int OFF_SAL = OFF_RQ + 8 * 32 * pf::RQ_LD;        // int32[128]
    static constexpr int OFF_BAR = OFF_SAL + 128 * 4;
    static constexpr int NBAR = 2 * STAGES + 4 + 1;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16;
    static constexpr int ALLOC = BYTES + 1024;                         // 1024-byte alignment slack
};

__device__ __forceinline__ uint32_t swz_chunk(int row, int chunk) { return static_cast<uint32_t>(chunk ^ (row & 7)); }

// 16-byte (4-byte) async copies that zero-fill when `valid` is false.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)),
                 "r"(valid ? 4 : 0)
                 : "memory");
}

// Producer thread `pi`: issue the async copies of its chunks of one stage
// (tile m0/n0, K-block kb) into packed slot `pk` (smem address).
template <int BN, bool ASYM>
__device__ __forceinline__ void prod_issue(const GemmArgs& p, int m0, int n0, int kb, int pi, uint32_t pk) {
    using L = PfSmem<BN, ASYM>;
    const int64_t kbytes = static_cast<int64_t>(p.K) / 2;
#pragma unroll
    for (int j = 0; j < L::NCH; ++j) {
        const int ci = pi + j * pf::NPROD;
        if (ci >= L::NCHUNK) continue;
        if (ci < pf::BM * 4) {
            const int row = ci >> 2, c = ci & 3;
            const int m = m0 + row;
            const bool ok = m < p.M;
            cp_async16_zfill(pk + ci * 16, ok ? p.Xq + m * kbytes + kb * 64 + c * 16 : p.Xq, ok);
        } else {
            const int cj = ci - pf::BM * 4;
            const int row = cj >> 2, c = cj & 3;
            const int n = n0 + row;
            const bool ok = n < p.N;
            cp_async16_zfill(pk + ci * 16, ok ? p.Wq + wq_offset(n, kb * 64 + c * 16, p.K / 128) : p.Wq, ok);
            if constexpr (ASYM) {
                const int b = (kb * pf::BK) / p.gw;
                cp_async4_zfill(pk + L::PK_DATA + cj * 4, ok ? p.zw + static_cast<int64_t>(b) * p.N + (n & ~1) : p.zw,
                                ok);
            }
        }
    }
}

// Producer thread `pi`: its packed chunks of one stage (slot `pk`, generic
// pointer) -> int8 operand tiles of the stage.
template <int BN, bool ASYM>
__device__ __forceinline__ void prod_unpack(const uint8_t* pk, uint8_t* stage, int pi) {
    using L = PfSmem<BN, ASYM>;
#pragma unroll
    for (int j = 0; j < L::NCH; ++j) {
        const int ci = pi + j * pf::NPROD;
        if (ci >= L::NCHUNK) continue;
        const bool isA = ci < pf::BM * 4;
        const int cl = isA ? ci : ci - pf::BM * 4;
        const int row = cl >> 2, c = cl & 3;
        const uint4 d = *reinterpret_cast<const uint4*>(pk + ci * 16);
        uint8_t* base = stage + (isA ? 0 : L::A_BYTES) + row * 128;
        uint32_t o[8];
        const uint32_t w[4] = {d.x, d.y, d.z, d.w};
        if (!isA && ASYM) {
            // zero point of weight row n = (n0 + row): half (row & 1) of the copied pair
            const uint32_t zp = *reinterpret_cast<const uint32_t*>(pk + L::PK_DATA + cl * 4);
            const uint16_t zh = static_cast<uint16_t>((row & 1) ? (zp >> 16) : (zp & 0xFFFFu));
            const uint32_t z4 = static_cast<uint32_t>(__half2float(__ushort_as_half(zh))) * 0x01010101u;
#pragma unroll
            for (int e = 0; e < 4; ++e) unpack_u4x8_minus_z(w[e], z4, o[2 * e], o[2 * e + 1]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) unpack_s4x8_times16(w[e], o[2 * e], o[2 * e + 1]);
        }
        *reinterpret_cast<uint4*>(base + swz_chunk(row, 2 * c) * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(base + swz_chunk(row, 2 * c + 1) * 16) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Gathered salient activation codes of row m as int8 words in the lo/hi
// permutation of unpack_s4x8_times16 (plain codes, not scaled by 16).
__device__ __forceinline__ void gather_xs(const GemmArgs& p, const int32_t* sal_s, int m, uint32_t (&xs)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) xs[i] = 0;
    if (m >= p.M) return;
    const uint8_t* row = p.Xq + static_cast<int64_t>(m) * (p.K / 2);
    for (int j = 0; j < p.r; ++j) {
        const int k = sal_s[j];
        const int nib = (__ldg(row + (k >> 1)) >> ((k & 1) * 4)) & 0xF;
        const uint32_t code = static_cast<uint32_t>((nib ^ 8) - 8) & 0xFFu;
        // position j = 8*i + 2*e + h  ->  word 2*i + h, byte e
        const int i = j >> 3, e = (j >> 1) & 3, h = j & 1;
        const uint32_t sh = 8u * e;
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (q == 2 * i + h) xs[q] |= code << sh;
    }
}

// Unpacks Rq rows of the warp's 32 columns into the warp's smem scratch:
// lane l -> row l, r/8 words -> r/4 words (16 * code), lo/hi permutation.
__device__ __forceinline__ void stage_rq(const GemmArgs& p, uint8_t* scratch, int n_first, int lane) {
    const int n = n_first + lane;
    uint32_t* dst = reinterpret_cast<uint32_t*>(scratch + lane * pf::RQ_LD);
    const int words = p.r / 8;
    if (n < p.N) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(p.Rq + static_cast<int64_t>(n) * (p.r / 2));
        for (int i = 0; i < words; ++i) {
            uint32_t lo, hi;
            unpack_s4x8_times16(__ldg(src + i), lo, hi);
            dst[2 * i] = lo;
            dst[2 * i + 1] = hi;
        }
    } else {
        for (int i = 0; i < 2 * words; ++i) dst[i] = 0;
    }
}

__device__ __forceinline__ int corr_dot(const uint32_t (&xs)[16], const uint8_t* rq_row, int nwords) {
    int acc = 0;
    const uint4* rv = reinterpret_cast<const uint4*>(rq_row);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (4 * i < nwords) {
            const uint4 q = rv[i];
            acc = __dp4a(static_cast<int>(xs[4 * i + 0]), static_cast<int>(q.x), acc);
            acc = __dp4a(static_cast<int>(xs[4 * i + 1]), static_cast<int>(q.y), acc);
            acc = __dp4a(static_cast<int>(xs[4 * i + 2]), static_cast<int>(q.z), acc);
            acc = __dp4a(static_cast<int>(xs[4 * i + 3]), static_cast<int>(q.w), acc);
        }
    }
    return acc >> 4;  // Rq entries carry a factor 16
}

template <int OUT>
__device__ __forceinline__ void store_out32(void* Y, int64_t off, const float (&y)[32], int nvalid) {
    if constexpr (OUT == HQ_F32) {
        float4* d = reinterpret_cast<float4*>(static_cast<float*>(Y) + off);
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if (8 * (v / 2) < nvalid) d[v] = make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
    } else {
        uint4* d = reinterpret_cast<uint4*>(static_cast<uint16_t*>(Y) + off);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            if (8 * v >= nvalid) break;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = y[8 * v + 2 * e], b = y[8 * v + 2 * e + 1];
                if constexpr (OUT == HQ_BF16) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                    w[e] = *reinterpret_cast<uint32_t*>(&h);
                } else {
                    __half2 h = __floats2half2_rn(a, b);
                    w[e] = *reinterpret_cast<uint32_t*>(&h);
                }
            }
            d[v] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

template <int OUT>
__device__ __forceinline__ void store_out8(void* Y, int64_t off, const float (&y)[8]) {
    if constexpr (OUT == HQ_F32) {
        float4* d = reinterpret_cast<float4*>(static_cast<float*>(Y) + off);
        d[0] = make_float4(y[0], y[1], y[2], y[3]);
        d[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if constexpr (OUT == HQ_BF16) {
                __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * e], y[2 * e + 1]);
                w[e] = *reinterpret_cast<uint32_t*>(&h);
            } else {
                __half2 h = __floats2half2_rn(y[2 * e], y[2 * e + 1]);
                w[e] = *reinterpret_cast<uint32_t*>(&h);
            }
        }
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(Y) + off) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void load_h8(const uint16_t* src, float (&o)[8]) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(src));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
        o[2 * e] = f.x;
        o[2 * e + 1] = f.y;
    }
}

__device__ __forceinline__ void load_h32(const uint16_t* src, float (&o)[32]) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 q = __ldg(s + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
            o[8 * v + 2 * e] = f.x;
            o[8 * v + 2 * e + 1] = f.y;
        }
    }
}

// OUT: HQ_F16 / HQ_BF16 / HQ_F32, or OUT_DEBUG for raw accumulators.
template <int BN, bool ASYM, int OUT>
__global__ void __launch_bounds__(pf::THREADS, 1) k_gemm_pf(const GemmArgs p) {
    using L = PfSmem<BN, ASYM>;
    constexpr int STAGES = L::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
    int32_t* sal_s = reinterpret_cast<int32_t*>(smem + L::OFF_SAL);

    const int MT = (p.M + pf::BM - 1) / pf::BM;
    const int NT = (p.N + BN - 1) / BN;
    const int num_tiles = MT * NT;
    const int KB = p.K / pf::BK;
    const int GPK = ASYM ? p.gw / pf::BK : KB;   // K-blocks per accumulation group
    const int NG = KB / GPK;
    constexpr uint32_t TMEM_COLS = 2 * BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), pf::NPROD);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), 8);
        }
        mbar_init(done_bar, 1);
        fence_mbar_init();
    }
    for (int j = threadIdx.x; j < p.r; j += blockDim.x) sal_s[j] = p.sal[j];
    if (warp == pf::MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < pf::EPI_WARP0 && warp != pf::MMA_WARP) {
        // ======================= producers
        const int pi = (warp < pf::MMA_WARP ? warp : warp - 1) * 32 + lane;
        const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        const int items = my_tiles * KB;
        const uint32_t pk0 = smem_u32(smem + L::OFF_PK);
        auto issue = [&](int item) {
            if (item < items) {
                const int tile = blockIdx.x + (item / KB) * gridDim.x;
                prod_issue<BN, ASYM>(p, (tile % MT) * pf::BM, (tile / MT) * BN, item % KB, pi,
                                     pk0 + (item % L::PD) * L::PK_STAGE);
            }
            cp_async_commit();   // one group per stage (possibly empty)
        };
        for (int d = 0; d < L::PD; ++d) issue(d);
        int stage = 0;
        uint32_t phase = 0;
        for (int item = 0; item < items; ++item) {
            cp_async_wait_group<L::PD - 1>();      // this thread's chunks of `item` have landed
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(empty_bar(stage), phase ^ 1u, p.limit_ns))) break;
            prod_unpack<BN, ASYM>(smem + L::OFF_PK + (item % L::PD) * L::PK_STAGE, smem + stage * L::STAGE, pi);
            issue(item + L::PD);                   // refill the packed slot just read
            fence_proxy_async_smem();
            mbar_arrive(full_bar(stage));
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        cp_async_wait_all();   // nothing in flight when the CTA exits
    } else if (warp == pf::MMA_WARP) {
        // ======================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_i8(pf::BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t aphase = 0;   // bit b: phase parity of accumulator buffer b
            int abuf = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                for (int kb = 0; ok && kb < KB; ++kb) {
                    const bool first = (kb % GPK) == 0;
                    if (first) {
                        if (!mbar_wait(acce_bar(abuf), ((aphase >> abuf) & 1u) ^ 1u, p.limit_ns)) { ok = false; break; }
                        tc_fence_after();
                    }
                    if (!mbar_wait(full_bar(stage), phase, p.limit_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE);
                    const uint64_t adesc = sw128_kmajor_desc(sa);
                    const uint64_t bdesc = sw128_kmajor_desc(sa + L::A_BYTES);
                    const uint32_t dcol = tmem_base + static_cast<uint32_t>(abuf * BN);
#pragma unroll
                    for (int kk = 0; kk < pf::BK / 32; ++kk)
                        mma_i8_ss(dcol, adesc + 2u * kk, bdesc + 2u * kk, IDESC, (first && kk == 0) ? 0u : 1u);
                    tc_commit(empty_bar(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if ((kb % GPK) == GPK - 1) {
                        tc_commit(accf_bar(abuf));
                        aphase ^= 1u << abuf;
                        abuf ^= 1;
                    }
                }
            }
            // all MMAs issued by this thread have completed before teardown
            tc_commit(done_bar);
            mbar_wait(done_bar, 0, p.limit_ns);
        }
        __syncwarp();
    } else {
        // ======================= epilogue
        const int q = warp & 3;                 // TMEM lane quarter
        const int hcol = (warp - pf::EPI_WARP0) >> 2;   // column half
        const int row = 32 * q + lane;
        uint8_t* rq_scr = smem + L::OFF_RQ + (warp - pf::EPI_WARP0) * 32 * pf::RQ_LD;
        const int rwords = p.r / 4;
        uint32_t aphase = 0;   // bit b: phase parity of accumulator buffer b
        int abuf = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            const int m0 = (tile % MT) * pf::BM, n0 = (tile / MT) * BN;
            const int m = m0 + row;
            const bool mvalid = m < p.M;
            float sxm = 0.f;
            if constexpr (OUT != OUT_DEBUG) sxm = mvalid ? p.sx[m] : 0.f;
            uint32_t xs[16];
            if (p.r > 0) gather_xs(p, sal_s, m, xs);
            constexpr int NCHUNK = BN / 2 / 32;
            float ypart[ASYM ? NCHUNK * 32 : 1];
            if constexpr (ASYM) {
                // correction first: ypart = sr[n] * (X[m,S] . R[n,:])
#pragma unroll
                for (int c = 0; c < NCHUNK; ++c) {
                    const int nb = n0 + hcol * (BN / 2) + c * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j) ypart[c * 32 + j] = 0.f;
                    if (p.r > 0 && nb < p.N) {
                        __syncwarp();
                        stage_rq(p, rq_scr, nb, lane);
                        __syncwarp();
                        if constexpr (OUT == OUT_DEBUG) {
                            for (int j = 0; j < 32; ++j) {
                                const int cc = corr_dot(xs, rq_scr + j * pf::RQ_LD, rwords);
                                if (mvalid && nb + j < p.N) p.dbg_acc_c[static_cast<int64_t>(m) * p.N + nb + j] = cc;
                            }
                        } else {
                            float srv[32];
                            load_h32(p.sr + nb, srv);
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int cc = corr_dot(xs, rq_scr + j * pf::RQ_LD, rwords);
                                ypart[c * 32 + j] = __fmul_rn(srv[j], static_cast<float>(cc));
                            }
                        }
                    }
                }
            }
            for (int g = 0; ok && g < NG; ++g) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(accf_bar(abuf), (aphase >> abuf) & 1u, p.limit_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < NCHUNK; ++c) {
                    const int col = hcol * (BN / 2) + c * 32;
                    const int nb = n0 + col;
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                           static_cast<uint32_t>(abuf * BN + col), acc);
                    tmem_wait_ld();
                    if (nb >= p.N) continue;
                    const int nvalid = p.N - nb;
                    if constexpr (OUT == OUT_DEBUG) {
                        if (mvalid) {
                            const int sh = ASYM ? 4 : 8;
                            for (int j = 0; j < 32 && j < nvalid; ++j)
                                p.dbg_acc[(static_cast<int64_t>(m) * p.N + nb + j) * NG + g] =
                                    static_cast<int32_t>(acc[j]) >> sh;
                        }
                        if constexpr (!ASYM) {
                            if (p.r > 0) {
                                __syncwarp();
                                stage_rq(p, rq_scr, nb, lane);
                                __syncwarp();
                                for (int j = 0; j < 32; ++j) {
                                    const int cc = corr_dot(xs, rq_scr + j * pf::RQ_LD, rwords);
                                    if (mvalid && j < nvalid) p.dbg_acc_c[static_cast<int64_t>(m) * p.N + nb + j] = cc;
                                }
                            }
                        }
                    } else if constexpr (ASYM) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float swv[8];
                            load_h8(p.sw + static_cast<int64_t>(g) * p.N + nb + 8 * v, swv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int j = 8 * v + e;
                                ypart[c * 32 + j] = __fmaf_rn(
                                    swv[e], static_cast<float>(static_cast<int32_t>(acc[j]) >> 4), ypart[c * 32 + j]);
                            }
                            if (g == NG - 1 && mvalid && 8 * v < nvalid) {
                                float y[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(sxm, ypart[c * 32 + 8 * v + e]);
                                store_out8<OUT>(p.Y, static_cast<int64_t>(m) * p.N + nb + 8 * v, y);
                            }
                        }
                    } else {
                        if (p.r > 0) {
                            __syncwarp();
                            stage_rq(p, rq_scr, nb, lane);
                            __syncwarp();
                        }
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            if (8 * v >= nvalid) break;
                            float swv[8], srv[8], y[8];
                            load_h8(p.sw + nb + 8 * v, swv);
                            if (p.r > 0) {
                                load_h8(p.sr + nb + 8 * v, srv);
                            } else {
#pragma unroll
                                for (int e = 0; e < 8; ++e) srv[e] = 0.f;
                            }
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int j = 8 * v + e;
                                const int cc = (p.r > 0) ? corr_dot(xs, rq_scr + j * pf::RQ_LD, rwords) : 0;
                                const float a = static_cast<float>(static_cast<int32_t>(acc[j]) >> 8);
                                const float t = __fmaf_rn(srv[e], static_cast<float>(cc), __fmul_rn(swv[e], a));
                                y[e] = __fmul_rn(sxm, t);
                            }
                            if (mvalid) store_out8<OUT>(p.Y, static_cast<int64_t>(m) * p.N + nb + 8 * v, y);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce_bar(abuf));
                aphase ^= 1u << abuf;
                abuf ^= 1;
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == pf::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int BN, bool ASYM, int OUT>
static hq_status launch_pf_t(const GemmArgs& a, cudaStream_t st, int nsm) {
    auto kern = k_gemm_pf<BN, ASYM, OUT>;
    const int smem = PfSmem<BN, ASYM>::ALLOC;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    const int tiles = ((a.M + pf::BM - 1) / pf::BM) * ((a.N + BN - 1) / BN);
    const int grid = tiles < nsm ? tiles : nsm;
    kern<<<grid, pf::THREADS, smem, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status launch_gemm_prefill(const GemmArgs& a, int out, cudaStream_t st, int nsm) {
    if (a.gw == 0) {
        switch (out) {
            case HQ_F16: return launch_pf_t<256, false, HQ_F16>(a, st, nsm);
            case HQ_BF16: return launch_pf_t<256, false, HQ_BF16>(a, st, nsm);
            case HQ_F32: return launch_pf_t<256, false, HQ_F32>(a, st, nsm);
            case OUT_DEBUG: return launch_pf_t<256, false, OUT_DEBUG>(a, st, nsm);
        }
    } else {
        switch (out) {
            case HQ_F16: return launch_pf_t<128, true, HQ_F16>(a, st, nsm);
            case HQ_BF16: return launch_pf_t<128, true, HQ_BF16>(a, st, nsm);
            case HQ_F32: return launch_pf_t<128, true, HQ_F32>(a, st, nsm);
            case OUT_DEBUG: return launch_pf_t<128, true, OUT_DEBUG>(a, st, nsm);
        }
    }
    return HQ_ERR_UNSUPPORTED;
}

}  // namespace hq
