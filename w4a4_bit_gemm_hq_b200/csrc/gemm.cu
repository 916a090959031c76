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
// Design (CTA pairs, one CTA per SM, persistent over 256 x BN output tiles):
//  * the two CTAs of a cluster form a pair; the even CTA issues pair-wide
//    tcgen05.mma (M = 256, N = BN, K = 32): A rows 0-127 come from its own
//    shared memory and rows 128-255 from its partner's, and each CTA holds
//    half of the BN weight rows of B, so each SM stages only its own 128
//    activation rows and BN/2 weight rows.  Each CTA's tensor memory receives
//    its 128 rows x BN of the int32 accumulator.
//  * in each CTA, one thread moves the packed codes of each K-block into a ring
//    of packed slots with the tensor memory accelerator: a 2D tensor-map load
//    of its 128 activation rows (64 bytes each; rows past M read as zero) and a
//    bulk copy of its half of the tile-major weight block (plus the zero points
//    of the block's group for group weights).
//  * tcgen05 has no int4 MMA, so 6 producer warps per CTA expand the packed
//    codes to int8 in registers (16*q for activations and symmetric weights,
//    u - z for asymmetric weights) and store them into 128-byte-swizzled
//    K-major smem tiles; they signal the even CTA's stage barrier, and the
//    pair MMA's commit frees the stage in both CTAs.
//  * the even CTA's MMA thread issues 4 pair MMAs per stage into one of
//    512 / BN int32 accumulator buffers; at the end of a tile (per-channel
//    weights) or of a weight group (group weights) a multicast commit hands the
//    buffer to the epilogues of both CTAs.
//  * 8 epilogue warps per CTA (2 per TMEM lane quarter, splitting the
//    columns) stage the tile's sw, sr, unpacked Rq rows and salient
//    activation codes X[m,S] in smem while the tile's MMAs run, then load the
//    accumulator with tcgen05.ld 16x256b (the mma.sync m16n8 fragment
//    layout), compute the SERQ term X[m,S] . Rq[n,:] with mma.sync m16n8k32
//    on the staged int8 codes in the same layout (an epilogue add: no second
//    launch), dequantise with sx[m] * sw[n] (or sum the per-group
//    sw[b][n] * acc_b), round once and store.
//  * every mbarrier wait is bounded; on timeout the status word records
//    HQ_ERR_TIMEOUT and the roles skip to teardown, which waits for in-flight
//    MMAs before freeing tensor memory.
#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cudaTypedefs.h>
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
constexpr int TMA_WARP = 0;           // lane 0 issues the packed-code copies
constexpr int MMA_WARP = 1;           // lane 0 issues tcgen05.mma; the warp owns TMEM
constexpr int PROD_WARP0 = 2;         // warps 2-7 expand codes to int8
constexpr int NPROD_WARPS = 6;
constexpr int NGROUP_WARPS = 3;       // two producer groups take alternate K-blocks
constexpr int NGROUP = NGROUP_WARPS * 32;
constexpr int EPI_WARP0 = 8;          // warps 8-15: epilogue
constexpr int PK_ROW = 64;            // packed bytes of one row of a K-block
constexpr int RQ_LD = 80;             // bytes per staged int8 row of r <= 64 codes (padded: the
                                      // mma.sync fragment loads of 8 rows x 4 words hit 32 banks)
constexpr int EPI_THREADS = 256;
constexpr uint32_t EPI_BAR = 1;       // named barrier of the epilogue warps
}  // namespace pf

// Shared memory of one CTA of a pair: an int8 operand ring read by the tensor
// core (STAGES deep: 128 activation rows, then BH = BN/2 weight rows, 128 K
// bytes each) and a ring of packed slots (PD deep) filled by the copy engine:
// the 128 activation rows (64 bytes each), the BH weight rows in tile-major
// order and, for group weights, their BH fp16 zero points of the block's group.
template <int BN, bool ASYM, bool A8 = false>
struct PfSmem {
    static constexpr int BH = BN / 2;                                  // weight rows per CTA
    static constexpr int NACC = 512 / BN;                              // accumulator buffers
    static constexpr int STAGES = 4;
    static constexpr int PD = ASYM ? 6 : 4;
    static constexpr int A_BYTES = pf::BM * pf::BK;
    static constexpr int B_BYTES = BH * pf::BK;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    // 16-byte packed chunks per stage the producers expand (8-bit activations
    // arrive in the int8 stage directly from the copy engine)
    static constexpr int NCHUNK = ((A8 ? 0 : pf::BM) + BH) * 4;
    static constexpr int NCH = (NCHUNK + pf::NGROUP - 1) / pf::NGROUP;  // per producer thread and stage
    static constexpr int PK_A = A8 ? 0 : pf::BM * pf::PK_ROW;
    static constexpr int PK_B = BH * pf::PK_ROW;
    static constexpr int PK_Z = ASYM ? BH * 2 : 0;
    static constexpr int PK_STAGE = ((PK_A + PK_B + PK_Z) + 127) / 128 * 128;
    static constexpr int OFF_PK = STAGES * STAGE;
    static constexpr int OFF_RQ = OFF_PK + PD * PK_STAGE;              // tile's Rq rows, BN x RQ_LD int8
    static constexpr int OFF_SW = OFF_RQ + BN * pf::RQ_LD;             // float [2][BN]: sw of the tile (of a group)
    static constexpr int OFF_SR = OFF_SW + 2 * BN * 4;                 // float [BN]
    static constexpr int OFF_XS = OFF_SR + BN * 4;                     // tile's X[m,S] rows, 128 x RQ_LD int8
    static constexpr int OFF_SAL = OFF_XS + pf::BM * pf::RQ_LD;        // int32[128]
    static constexpr int OFF_BAR = OFF_SAL + 128 * 4;
    static constexpr int NBAR = 2 * STAGES + 2 * PD + 2 * NACC + 1;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16;
    static constexpr int ALLOC = BYTES + 1024;                         // 1024-byte alignment slack
    static_assert(ALLOC <= 227 * 1024, "shared memory budget");
    static_assert(BN * NACC == 512, "accumulator buffers fill the tensor memory");
};

__device__ __forceinline__ uint32_t swz_chunk(int row, int chunk) { return static_cast<uint32_t>(chunk ^ (row & 7)); }

// Producer thread `pi`: its packed chunks of one stage (slot `pk`, generic
// pointer) -> int8 operand tiles of the stage.  Chunk ci covers packed bytes
// [16 ci, 16 ci + 16) of the slot: activation row ci / 4 for ci < 512, else
// weight row (ci - 512) / 4, K bytes 16 (ci % 4) onwards.
template <int BN, bool ASYM, bool A8>
__device__ __forceinline__ void prod_unpack(const uint8_t* pk, uint8_t* stage, int pi) {
    using L = PfSmem<BN, ASYM, A8>;
#pragma unroll
    for (int j = 0; j < L::NCH; ++j) {
        const int ci = pi + j * pf::NGROUP;
        if (ci >= L::NCHUNK) continue;
        const bool isA = !A8 && ci < pf::BM * 4;
        const int cl = isA ? ci : ci - (A8 ? 0 : pf::BM * 4);
        const int row = cl >> 2, c = cl & 3;
        const uint4 d = *reinterpret_cast<const uint4*>(pk + ci * 16);
        uint8_t* base = stage + (isA ? 0 : L::A_BYTES) + row * 128;
        uint32_t o[8];
        const uint32_t w[4] = {d.x, d.y, d.z, d.w};
        if (!isA && ASYM) {
            // zero point of weight row n0 + row, an integer in [0, 15] stored as fp16
            const uint16_t zh = *reinterpret_cast<const uint16_t*>(pk + L::PK_A + L::PK_B + row * 2);
            const uint32_t z4 = (static_cast<uint32_t>(__half2float(__ushort_as_half(zh))) & 0xFu) * 0x01010101u;
#pragma unroll
            for (int e = 0; e < 4; ++e) unpack_u4x8_minus_z(w[e], z4, o[2 * e], o[2 * e + 1]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) unpack_s4x8_times16(w[e], o[2 * e], o[2 * e + 1]);
        }
        if constexpr (A8) {
            // 8-bit activations keep their natural K order: interleave each
            // (k0 k2 k4 k6, k1 k3 k5 k7) pair of words back to (k0..k3, k4..k7)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t lo = o[2 * e], hi = o[2 * e + 1];
                o[2 * e] = __byte_perm(lo, hi, 0x5140);
                o[2 * e + 1] = __byte_perm(lo, hi, 0x7362);
            }
        }
        *reinterpret_cast<uint4*>(base + swz_chunk(row, 2 * c) * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(base + swz_chunk(row, 2 * c + 1) * 16) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Column data of output column n for one tile, staged by one epilogue thread:
// sw (per channel, or of group 0) and sr as float, and the SERQ row Rq[n]
// unpacked to r int8 values (16 * code, lo/hi permutation).  Columns past N
// stage zeros.
template <int OUT>
__device__ __forceinline__ void stage_column(const GemmArgs& p, int n, float* sw_d, float* sr_d, uint8_t* rq_d) {
    const bool nv = n < p.N;
    if constexpr (OUT != OUT_DEBUG) {
        *sw_d = nv ? __half2float(__ushort_as_half(__ldg(p.sw + n))) : 0.f;
        *sr_d = (nv && p.r > 0) ? __half2float(__ushort_as_half(__ldg(p.sr + n))) : 0.f;
    }
    if (p.r == 0) return;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.Rq + static_cast<int64_t>(nv ? n : 0) * (p.r / 2));
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = (nv && 8 * i < p.r) ? __ldg(src + i) : 0u;
    uint4* dst = reinterpret_cast<uint4*>(rq_d);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (16 * i >= p.r) break;   // words 2i and 2i+1 hold codes 16i .. 16i+15
        uint32_t a0, a1, b0, b1;
        unpack_s4x8_times16(w[2 * i], a0, a1);
        unpack_s4x8_times16(w[2 * i + 1], b0, b1);
        dst[i] = make_uint4(a0, a1, b0, b1);
    }
}

// Salient activation codes of row m for the staged int8 row `xs_w` (words):
// position j = 8 i + 2 e + h -> word 2 i + h, byte e (the lo/hi permutation of
// unpack_s4x8_times16).  This thread writes the blocks i with i % 2 == half
// (words 2i, 2i+1) of the first `nblk` blocks; blocks past r and rows past M
// are zero.  All loads of the thread are in flight together.
template <bool A8>
__device__ __forceinline__ void gather_xs_smem(const GemmArgs& p, const int32_t* sal_s, int m, uint32_t* xs_w,
                                               int half, int nblk) {
    const bool mv = m < p.M;
    const uint8_t* row = p.Xq + static_cast<int64_t>(mv ? m : 0) * (A8 ? p.K : p.K / 2);
    uint32_t nib[4][8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int i = 2 * b + half;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            nib[b][t] = 0u;
            if (mv && 8 * i < p.r) {
                const int k = sal_s[8 * i + t];
                if (static_cast<unsigned>(k) < static_cast<unsigned>(p.K)) {
                    if constexpr (A8) nib[b][t] = __ldg(row + k);   // the 8-bit code itself
                    else nib[b][t] = (static_cast<uint32_t>(__ldg(row + (k >> 1))) >> ((k & 1) * 4)) & 0xFu;
                } else {
                    record_status(HQ_ERR_ARG);   // a salient index outside [0, K): skipped
                }
            }
        }
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int i = 2 * b + half;
        if (i >= nblk) break;
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t code = (8 * i >= p.r) ? 0u
                                  : A8 ? (nib[b][t] & 0xFFu)
                                       : static_cast<uint32_t>(static_cast<int>(nib[b][t] ^ 8u) - 8) & 0xFFu;
            if (t & 1) hi |= code << (8 * (t >> 1));
            else lo |= code << (8 * (t >> 1));
        }
        xs_w[2 * i] = lo;
        xs_w[2 * i + 1] = hi;
    }
}

template <int OUT>
__device__ __forceinline__ void store_out2(void* Y, int64_t off, float a, float b) {
    if constexpr (OUT == HQ_F32) {
        *reinterpret_cast<float2*>(static_cast<float*>(Y) + off) = make_float2(a, b);
    } else if constexpr (OUT == HQ_BF16) {
        *reinterpret_cast<__nv_bfloat162*>(static_cast<uint16_t*>(Y) + off) = __floats2bfloat162_rn(a, b);
    } else {
        *reinterpret_cast<__half2*>(static_cast<uint16_t*>(Y) + off) = __floats2half2_rn(a, b);
    }
}

// Symmetric-weight epilogue of one 32-column chunk for the warp's 32 rows.
// The accumulator comes from tensor memory in the mma.sync m16n8 fragment
// layout (two 16-lane halves); the SERQ term acc_c = X[m,S] . Rq[n,:] is
// computed on the staged int8 codes with mma.sync m16n8k32 in the same layout;
// then Y = sx[m] * (sr[n] * acc_c + sw[n] * acc), rounded once.
//  tm     tensor-memory address of lane 32q, chunk column 0
//  mq0    first output row of the warp;  n0c  first output column of the chunk
//  scol   column of the chunk within the tile (index into the staged columns)
//  afr    A fragments [row half][K step] of the warp's X[m,S] rows
template <int OUT, int AF>
__device__ __forceinline__ void drain_sym_chunk(const GemmArgs& p, uint32_t tm, int mq0, int n0c, int scol,
                                                const float* sw_s, const float* sr_s, const uint8_t* rq_s,
                                                const uint32_t (&afr)[2][2][4], int ksteps, const float (&sxr)[2][2],
                                                int g, int t) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        uint32_t v[16];
        tmem_ld_16x256b_x4(tm + (static_cast<uint32_t>(16 * mt) << 16), v);
        tmem_wait_ld();
        int32_t cc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) cc[nt][i] = 0;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            if (ks < ksteps) {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const uint32_t* rw =
                        reinterpret_cast<const uint32_t*>(rq_s + (scol + 8 * nt + g) * pf::RQ_LD) + 8 * ks;
                    mma_s8_16x8x32(cc[nt], afr[mt][ks], rw[t], rw[4 + t]);
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            if (n0c + 8 * nt >= p.N) continue;   // N % 8 == 0: whole groups of 8 columns
            const int cl = scol + 8 * nt + 2 * t;
            const int64_t n = n0c + 8 * nt + 2 * t;
            float2 swv = make_float2(0.f, 0.f), srv = make_float2(0.f, 0.f);
            if constexpr (OUT != OUT_DEBUG) {
                swv = *reinterpret_cast<const float2*>(sw_s + cl);
                srv = *reinterpret_cast<const float2*>(sr_s + cl);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int m = mq0 + 16 * mt + g + 8 * h;
                if (m >= p.M) continue;
                // the weight codes carry 16, the activation codes AF
                const int32_t a0 = static_cast<int32_t>(v[4 * nt + 2 * h]) >> (AF == 16 ? 8 : 4);
                const int32_t a1 = static_cast<int32_t>(v[4 * nt + 2 * h + 1]) >> (AF == 16 ? 8 : 4);
                const int32_t c0 = cc[nt][2 * h] >> 4, c1 = cc[nt][2 * h + 1] >> 4;   // Rq codes carry 16
                const int64_t off = static_cast<int64_t>(m) * p.N + n;
                if constexpr (OUT == OUT_DEBUG) {
                    p.dbg_acc[off] = a0;
                    p.dbg_acc[off + 1] = a1;
                    if (p.r > 0) {
                        p.dbg_acc_c[off] = c0;
                        p.dbg_acc_c[off + 1] = c1;
                    }
                } else {
                    const float y0 = __fmul_rn(sxr[mt][h], __fmaf_rn(srv.x, static_cast<float>(c0),
                                                                     __fmul_rn(swv.x, static_cast<float>(a0))));
                    const float y1 = __fmul_rn(sxr[mt][h], __fmaf_rn(srv.y, static_cast<float>(c1),
                                                                     __fmul_rn(swv.y, static_cast<float>(a1))));
                    store_out2<OUT>(p.Y, off, y0, y1);
                }
            }
        }
    }
}

// OUT: HQ_F16 / HQ_BF16 / HQ_F32, or OUT_DEBUG for raw accumulators.
// Launched as clusters of 2 CTAs (an even number of CTAs).
template <int BN, bool ASYM, bool A8, int OUT>
__global__ void __launch_bounds__(pf::THREADS, 1) k_gemm_pf(const GemmArgs p, const __grid_constant__ CUtensorMap tmX) {
    using L = PfSmem<BN, ASYM, A8>;
    // factor of the activation codes in the int8 operand (4-bit codes are
    // expanded as 16 q; 8-bit codes are used as they are)
    constexpr int AF = A8 ? 1 : 16;
    constexpr int STAGES = L::STAGES;
    constexpr int PD = L::PD;
    constexpr int NACC = L::NACC;
    constexpr int BH = L::BH;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived by pointer arithmetic on the __shared__
    // array so that every access through it compiles to a shared-memory
    // instruction (a pointer rebuilt from an integer is generic)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_ctarank();   // 0: issues the pair MMAs
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };                       // even CTA: both CTAs' producers
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };           // each CTA: pair MMA commit
    auto pkfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
    auto pkempty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + PD + s); };
    auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * PD + b); };          // each CTA
    auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * PD + NACC + b); };   // even CTA
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 2 * PD + 2 * NACC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
    int32_t* sal_s = reinterpret_cast<int32_t*>(smem + L::OFF_SAL);

    const int MT = (p.M + 2 * pf::BM - 1) / (2 * pf::BM);
    const int NT = (p.N + BN - 1) / BN;
    const int num_tiles = MT * NT;
    const int KB = p.K / pf::BK;
    const int GPK = ASYM ? p.gw / pf::BK : KB;   // K-blocks per accumulation group
    const int NG = KB / GPK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 2 * pf::NGROUP_WARPS);
            mbar_init(empty_bar(s), 1);
        }
        for (int s = 0; s < PD; ++s) {
            mbar_init(pkfull_bar(s), 1);
            mbar_init(pkempty_bar(s), pf::NGROUP_WARPS);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), 2 * 8);
        }
        mbar_init(done_bar, 1);
        fence_mbar_init();
    }
    for (int j = threadIdx.x; j < p.r; j += blockDim.x) sal_s[j] = p.sal[j];
    if (warp == pf::MMA_WARP) {
        tmem_alloc_pair(smem_u32(tmem_slot), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / npairs + 1 : 0;
    const int items = my_tiles * KB;   // (tile, K-block) pairs of this CTA pair, in order
    const uint32_t pk0 = smem_u32(smem + L::OFF_PK);

    if (warp == pf::TMA_WARP) {
        // ======================= packed-code copies (this CTA's rows)
        if (lane == 0) {
            prefetch_tmap(&tmX);
            const int npad = (p.N + 127) / 128 * 128;   // rows present in the tile-major weight buffer
            int slot = 0;
            uint32_t ph = 0;
            int issued = 0;
            for (int item = 0; item < items; ++item) {
                const int tile = pair + (item / KB) * npairs;
                const int kb = item % KB;
                const int m0 = (tile % MT) * 2 * pf::BM + static_cast<int>(crank) * pf::BM;
                const int nr = (tile / MT) * BN + static_cast<int>(crank) * BH;   // first weight row of this CTA
                if (!mbar_wait(pkempty_bar(slot), ph ^ 1u, p.limit_ns)) break;
                const int stg = item % STAGES;
                if constexpr (A8) {
                    // the 8-bit activation tile goes straight into the stage: wait
                    // until the pair's MMAs have finished reading its previous use
                    if (!mbar_wait_cluster(empty_bar(stg), (static_cast<uint32_t>(item / STAGES) & 1u) ^ 1u, p.limit_ns))
                        break;
                }
                const uint32_t dst = pk0 + slot * L::PK_STAGE;
                const bool has_b = nr < npad;
                const int zrows = ASYM ? ((p.N - nr) < BH ? (p.N - nr) : BH) : 0;
                const int zb = zrows > 0 ? zrows * 2 : 0;
                mbar_arrive_expect_tx(pkfull_bar(slot),
                                      static_cast<uint32_t>((A8 ? L::A_BYTES : L::PK_A) + (has_b ? L::PK_B : 0) + zb));
                if constexpr (A8)   // 128 rows x 128 bytes, 128-byte swizzled: the MMA's K-major layout
                    tma_load_2d(smem_u32(smem + stg * L::STAGE), &tmX, kb * pf::BK, m0, pkfull_bar(slot));
                else
                    tma_load_2d(dst, &tmX, kb * pf::PK_ROW, m0, pkfull_bar(slot));
                if (has_b)
                    bulk_copy_g2s(dst + L::PK_A, p.Wq + wq_offset(nr, kb * 64, KB), L::PK_B, pkfull_bar(slot));
                if constexpr (ASYM) {
                    if (zb > 0)
                        bulk_copy_g2s(dst + L::PK_A + L::PK_B, p.zw + static_cast<int64_t>(kb / GPK) * p.N + nr,
                                      static_cast<uint32_t>(zb), pkfull_bar(slot));
                }
                ++issued;
                if (++slot == PD) { slot = 0; ph ^= 1u; }
            }
            // no copy may still be landing when the CTA exits: wait for the
            // last phase of every slot that was written (immediate unless a
            // consumer gave up)
            for (int i = issued > PD ? issued - PD : 0; i < issued; ++i)
                mbar_wait(pkfull_bar(i % PD), static_cast<uint32_t>(i / PD) & 1u, p.limit_ns);
        }
        __syncwarp();
    } else if (warp >= pf::PROD_WARP0 && warp < pf::PROD_WARP0 + pf::NPROD_WARPS) {
        // ======================= producers: packed codes -> int8 operand tiles
        // Two groups of 3 warps take alternate K-blocks, so one group's
        // barrier waits overlap the other's unpacking (STAGES and PD are even:
        // each group keeps to its own stages and slots).
        static_assert(STAGES % 2 == 0 && PD % 2 == 0, "groups alternate over the rings");
        const int grp = (warp - pf::PROD_WARP0) / pf::NGROUP_WARPS;
        const int pi = ((warp - pf::PROD_WARP0) % pf::NGROUP_WARPS) * 32 + lane;
        const uint32_t full_remote0 = mapa_shared(full_bar(0), 0);
        for (int item = grp; item < items; item += 2) {
            const int stage = item % STAGES, slot = item % PD;
            const uint32_t phase = static_cast<uint32_t>(item / STAGES) & 1u;
            const uint32_t ph = static_cast<uint32_t>(item / PD) & 1u;
            bool ok = mbar_wait(pkfull_bar(slot), ph, p.limit_ns);
            ok = ok && mbar_wait_cluster(empty_bar(stage), phase ^ 1u, p.limit_ns);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
            prod_unpack<BN, ASYM, A8>(smem + L::OFF_PK + slot * L::PK_STAGE, smem + stage * L::STAGE, pi);
            fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(pkempty_bar(slot));
                mbar_arrive_cluster(full_remote0 + 8u * static_cast<uint32_t>(stage));
            }
        }
    } else if (warp == pf::MMA_WARP) {
        // ======================= pair MMA issuer (even CTA)
        if (lane == 0 && crank == 0) {
            constexpr uint32_t IDESC = idesc_i8(2 * pf::BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t aphase = 0;   // bit b: phase parity of accumulator buffer b
            int abuf = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
                for (int kb = 0; ok && kb < KB; ++kb) {
                    const bool first = (kb % GPK) == 0;
                    if (first) {
                        // per-channel weights: the buffer's previous phase (free from the
                        // start); group weights: its epilogues' preload of the next use
                        const uint32_t par = ASYM ? ((aphase >> abuf) & 1u) : (((aphase >> abuf) & 1u) ^ 1u);
                        if (!mbar_wait_cluster(acce_bar(abuf), par, p.limit_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    if (!mbar_wait_cluster(full_bar(stage), phase, p.limit_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE);
                    const uint64_t adesc = sw128_kmajor_desc(sa);
                    const uint64_t bdesc = sw128_kmajor_desc(sa + L::A_BYTES);
                    const uint32_t dcol = tmem_base + static_cast<uint32_t>(abuf * BN);
#pragma unroll
                    for (int kk = 0; kk < pf::BK / 32; ++kk)
                        mma_i8_ss_pair(dcol, adesc + 2u * kk, bdesc + 2u * kk, IDESC,
                                       (!ASYM && first && kk == 0) ? 0u : 1u);   // group weights add onto the preload
                    tc_commit_pair_mc(empty_bar(stage), 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if ((kb % GPK) == GPK - 1) {
                        tc_commit_pair_mc(accf_bar(abuf), 0x3);
                        aphase ^= 1u << abuf;
                        abuf = (abuf + 1 == NACC) ? 0 : abuf + 1;
                    }
                }
            }
            // all MMAs issued by this thread have completed before teardown
            tc_commit_pair(done_bar);
            mbar_wait(done_bar, 0, p.limit_ns);
        }
        __syncwarp();
    } else {
        // ======================= epilogue (this CTA's 128 rows, all BN columns)
        // All 8 warps run every tile and group in lockstep through the named
        // barrier EPI_BAR; a warp whose accumulator wait gave up keeps taking
        // the barriers (skipping the work) so that no warp is left waiting.
        const int et = threadIdx.x - pf::EPI_WARP0 * 32;     // 0 .. 255
        const int q = warp & 3;                              // TMEM lane quarter
        const int hcol = (warp - pf::EPI_WARP0) >> 2;        // column half
        const int row = 32 * q + lane;
        float* sw_s = reinterpret_cast<float*>(smem + L::OFF_SW);
        float* sr_s = reinterpret_cast<float*>(smem + L::OFF_SR);
        uint8_t* rq_s = smem + L::OFF_RQ;
        const uint32_t acce_remote0 = mapa_shared(acce_bar(0), 0);
        uint32_t aphase = 0;   // bit b: phase parity of accumulator buffer b
        int abuf = 0;
        bool ok = true;
        if constexpr (!ASYM) {
            // per-channel weights: one accumulator per tile, drained in the
            // mma.sync fragment layout with the SERQ term on mma.sync
            const uint32_t* xs_w = reinterpret_cast<const uint32_t*>(smem + L::OFF_XS);
            const int g8 = lane >> 2, t4 = lane & 3;
            const int ksteps = (p.r + 31) / 32;
            for (int tile = pair; tile < num_tiles; tile += npairs) {
                const int m0 = (tile % MT) * 2 * pf::BM + static_cast<int>(crank) * pf::BM, n0 = (tile / MT) * BN;
                const int mq0 = m0 + 32 * q;
                // ---- stage the tile's column data and X[m,S] rows while its MMAs run
                named_bar_sync(pf::EPI_BAR, pf::EPI_THREADS);   // previous tile's readers are done
                if (et < BN) stage_column<OUT>(p, n0 + et, sw_s + et, sr_s + et, rq_s + et * pf::RQ_LD);
                if (p.r > 0)
                    gather_xs_smem<A8>(p, sal_s, m0 + row,
                                   reinterpret_cast<uint32_t*>(smem + L::OFF_XS + row * pf::RQ_LD), hcol, 4 * ksteps);
                float sxr[2][2];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int m = mq0 + 16 * mt + g8 + 8 * h;
                        sxr[mt][h] = 0.f;
                        if constexpr (OUT != OUT_DEBUG) sxr[mt][h] = m < p.M ? __ldg(p.sx + m) : 0.f;
                    }
                named_bar_sync(pf::EPI_BAR, pf::EPI_THREADS);
                uint32_t afr[2][2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const uint32_t* r0 = xs_w + (32 * q + 16 * mt + g8) * (pf::RQ_LD / 4) + 8 * ks;
                        const uint32_t* r1 = r0 + 8 * (pf::RQ_LD / 4);
                        const bool on = ks < ksteps;
                        afr[mt][ks][0] = on ? r0[t4] : 0u;
                        afr[mt][ks][1] = on ? r1[t4] : 0u;
                        afr[mt][ks][2] = on ? r0[4 + t4] : 0u;
                        afr[mt][ks][3] = on ? r1[4 + t4] : 0u;
                    }
                if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(accf_bar(abuf), (aphase >> abuf) & 1u, p.limit_ns));
                if (ok) {
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < BN / 2 / 32; ++c) {
                        const int col = hcol * (BN / 2) + c * 32;
                        if (n0 + col >= p.N) break;
                        drain_sym_chunk<OUT, AF>(p,
                                             tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                                 static_cast<uint32_t>(abuf * BN + col),
                                             mq0, n0 + col, col, sw_s, sr_s, rq_s, afr, ksteps, sxr, g8, t4);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acce_remote0 + 8u * static_cast<uint32_t>(abuf));
                }
                aphase ^= 1u << abuf;
                abuf = (abuf + 1 == NACC) ? 0 : abuf + 1;
            }
        } else {
            // group weights: one accumulator per (tile, group), drained into
            // per-thread fp32 partial sums in the mma.sync fragment layout, 64
            // columns x the warp's 32 rows: yp[chunk][row tile][8-col group][row half]
            // holds the column pair (2 t4, 2 t4 + 1).
            //
            // Every buffer is preloaded with the bit pattern of 1.5 * 2^23 before
            // a group's MMAs add onto it, so a drained int32 accumulator reads as
            // the float 1.5 * 2^23 + acc, exactly (|acc| < 2^22): one packed
            // subtract and one packed fma per column pair convert, scale and
            // accumulate, with no integer -> float conversion instruction.
            const uint32_t* xs_w = reinterpret_cast<const uint32_t*>(smem + L::OFF_XS);
            const int g8 = lane >> 2, t4 = lane & 3;
            const int ksteps = (p.r + 31) / 32;
            constexpr int NC = BN / 2 / 32;   // 32-column chunks per warp
            constexpr uint32_t MAGIC = 0x4B400000u;   // bits of 1.5 * 2^23
            const float2 cmag = make_float2(12582912.0f, 12582912.0f);
            auto preload = [&](int b) {
                const uint32_t ta = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                    static_cast<uint32_t>(b * BN + hcol * (BN / 2));
#pragma unroll
                for (int c = 0; c < BN / 2 / 32; ++c) tmem_fill_32x32b_x32(ta + 32u * c, MAGIC);
                tmem_wait_st();
            };
            auto release = [&](int b) {   // the buffer is preloaded: hand it to the MMA
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce_remote0 + 8u * static_cast<uint32_t>(b));
            };
            for (int b = 0; b < NACC; ++b) {
                preload(b);
                release(b);
            }
            for (int tile = pair; tile < num_tiles; tile += npairs) {
                const int m0 = (tile % MT) * 2 * pf::BM + static_cast<int>(crank) * pf::BM, n0 = (tile / MT) * BN;
                const int mq0 = m0 + 32 * q;
                named_bar_sync(pf::EPI_BAR, pf::EPI_THREADS);   // previous tile's readers are done
                if (et < BN) stage_column<OUT>(p, n0 + et, sw_s + et, sr_s + et, rq_s + et * pf::RQ_LD);
                if (p.r > 0)
                    gather_xs_smem<A8>(p, sal_s, m0 + row,
                                   reinterpret_cast<uint32_t*>(smem + L::OFF_XS + row * pf::RQ_LD), hcol, 4 * ksteps);
                float sxr[2][2];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int m = mq0 + 16 * mt + g8 + 8 * h;
                        sxr[mt][h] = 0.f;
                        if constexpr (OUT != OUT_DEBUG) sxr[mt][h] = m < p.M ? __ldg(p.sx + m) : 0.f;
                    }
                named_bar_sync(pf::EPI_BAR, pf::EPI_THREADS);
                // ---- SERQ term first: yp = sr[n] * (X[m,S] . Rq[n,:])
                float2 yp[NC][2][4][2];
                {
                    uint32_t afr[2][2][4];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            const uint32_t* r0 = xs_w + (32 * q + 16 * mt + g8) * (pf::RQ_LD / 4) + 8 * ks;
                            const uint32_t* r1 = r0 + 8 * (pf::RQ_LD / 4);
                            const bool on = ks < ksteps;
                            afr[mt][ks][0] = on ? r0[t4] : 0u;
                            afr[mt][ks][1] = on ? r1[t4] : 0u;
                            afr[mt][ks][2] = on ? r0[4 + t4] : 0u;
                            afr[mt][ks][3] = on ? r1[4 + t4] : 0u;
                        }
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        const int scol = hcol * (BN / 2) + 32 * c;
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            int32_t cc[4][4];
#pragma unroll
                            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                                for (int i = 0; i < 4; ++i) cc[nt][i] = 0;
#pragma unroll
                            for (int ks = 0; ks < 2; ++ks) {
                                if (ks < ksteps) {
#pragma unroll
                                    for (int nt = 0; nt < 4; ++nt) {
                                        const uint32_t* rw = reinterpret_cast<const uint32_t*>(
                                                                 rq_s + (scol + 8 * nt + g8) * pf::RQ_LD) + 8 * ks;
                                        mma_s8_16x8x32(cc[nt], afr[mt][ks], rw[t4], rw[4 + t4]);
                                    }
                                }
                            }
#pragma unroll
                            for (int nt = 0; nt < 4; ++nt) {
                                const int cl = scol + 8 * nt + 2 * t4;
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    // the Rq codes carry a factor 16; yp carries AF (the factor of
                                    // the activation codes) until the end of the tile
                                    const int32_t c0 = AF == 16 ? cc[nt][2 * h] : cc[nt][2 * h] >> 4;
                                    const int32_t c1 = AF == 16 ? cc[nt][2 * h + 1] : cc[nt][2 * h + 1] >> 4;
                                    if constexpr (OUT == OUT_DEBUG) {
                                        const int m = mq0 + 16 * mt + g8 + 8 * h;
                                        const int n = n0 + cl;
                                        if (p.r > 0 && m < p.M && n < p.N) {
                                            p.dbg_acc_c[static_cast<int64_t>(m) * p.N + n] = AF == 16 ? c0 >> 4 : c0;
                                            p.dbg_acc_c[static_cast<int64_t>(m) * p.N + n + 1] = AF == 16 ? c1 >> 4 : c1;
                                        }
                                        yp[c][mt][nt][h] = make_float2(0.f, 0.f);
                                    } else {
                                        yp[c][mt][nt][h] =
                                            (p.r > 0) ? make_float2(__fmul_rn(sr_s[cl], static_cast<float>(c0)),
                                                                    __fmul_rn(sr_s[cl + 1], static_cast<float>(c1)))
                                                      : make_float2(0.f, 0.f);
                                    }
                                }
                            }
                        }
                    }
                }
                // ---- sw of group 0 for this thread's columns (fp16 pairs)
                uint32_t swc[NC][4];
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const int n = n0 + hcol * (BN / 2) + 32 * c + 8 * nt + 2 * t4;
                        swc[c][nt] = 0u;
                        if constexpr (OUT != OUT_DEBUG)
                            if (n < p.N) swc[c][nt] = __ldg(reinterpret_cast<const uint32_t*>(p.sw + n));
                    }
                for (int g = 0; g < NG; ++g) {
                    // next group's sw, in flight while this group's accumulator is awaited
                    uint32_t swn[NC][4];
#pragma unroll
                    for (int c = 0; c < NC; ++c)
#pragma unroll
                        for (int nt = 0; nt < 4; ++nt) {
                            const int n = n0 + hcol * (BN / 2) + 32 * c + 8 * nt + 2 * t4;
                            swn[c][nt] = 0u;
                            if constexpr (OUT != OUT_DEBUG)
                                if (g + 1 < NG && n < p.N)
                                    swn[c][nt] = __ldg(reinterpret_cast<const uint32_t*>(
                                        p.sw + static_cast<int64_t>(g + 1) * p.N + n));
                        }
                    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(accf_bar(abuf), (aphase >> abuf) & 1u, p.limit_ns));
                    if (ok) {
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < NC; ++c) {
                            const int scol = hcol * (BN / 2) + 32 * c;
                            // sw of the chunk's column pairs (yp carries the factor 16 of the
                            // activation codes until the end of the tile)
                            float2 swf[4];
#pragma unroll
                            for (int nt = 0; nt < 4; ++nt)
                                swf[nt] = __half22float2(*reinterpret_cast<const __half2*>(&swc[c][nt]));
#pragma unroll
                            for (int mt = 0; mt < 2; ++mt) {
                                uint32_t v[16];
                                tmem_ld_16x256b_x4(tmem_base + (static_cast<uint32_t>(32 * q + 16 * mt) << 16) +
                                                       static_cast<uint32_t>(abuf * BN + scol),
                                                   v);
                                tmem_wait_ld();
#pragma unroll
                                for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        const float2 f = make_float2(__uint_as_float(v[4 * nt + 2 * h]),
                                                                     __uint_as_float(v[4 * nt + 2 * h + 1]));
                                        if constexpr (OUT == OUT_DEBUG) {
                                            const int m = mq0 + 16 * mt + g8 + 8 * h;
                                            const int n = n0 + scol + 8 * nt + 2 * t4;
                                            if (m < p.M && n < p.N) {
                                                const int64_t o = (static_cast<int64_t>(m) * p.N + n) * NG + g;
                                                p.dbg_acc[o] = static_cast<int32_t>(v[4 * nt + 2 * h] - MAGIC) / AF;
                                                p.dbg_acc[o + NG] = static_cast<int32_t>(v[4 * nt + 2 * h + 1] - MAGIC) / AF;
                                            }
                                        } else {
                                            // f - 1.5 * 2^23 = AF acc exactly; yp += sw (AF acc)
                                            yp[c][mt][nt][h] = __ffma2_rn(swf[nt], __fadd2_rn(f, make_float2(-cmag.x, -cmag.y)),
                                                                          yp[c][mt][nt][h]);
                                        }
                                    }
                                }
                            }
                        }
                        preload(abuf);
                        release(abuf);
                    }
                    aphase ^= 1u << abuf;
                    abuf = (abuf + 1 == NACC) ? 0 : abuf + 1;
#pragma unroll
                    for (int c = 0; c < NC; ++c)
#pragma unroll
                        for (int nt = 0; nt < 4; ++nt) swc[c][nt] = swn[c][nt];
                }
                // ---- Y = sx[m] * yp
                if constexpr (OUT != OUT_DEBUG) {
                    if (ok) {
#pragma unroll
                        for (int c = 0; c < NC; ++c)
#pragma unroll
                            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                                for (int nt = 0; nt < 4; ++nt) {
                                    const int64_t n = n0 + hcol * (BN / 2) + 32 * c + 8 * nt + 2 * t4;
                                    if (n >= p.N) continue;
#pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        const int m = mq0 + 16 * mt + g8 + 8 * h;
                                        if (m >= p.M) continue;
                                        // yp / AF is exact: the same bits as accumulating sw * acc
                                        constexpr float inv_af = 1.0f / AF;
                                        store_out2<OUT>(p.Y, static_cast<int64_t>(m) * p.N + n,
                                                        __fmul_rn(sxr[mt][h], __fmul_rn(yp[c][mt][nt][h].x, inv_af)),
                                                        __fmul_rn(sxr[mt][h], __fmul_rn(yp[c][mt][nt][h].y, inv_af)));
                                    }
                                }
                    }
                }
            }
        }
    }

    // Teardown: neither CTA leaves while its partner may still read its shared
    // memory or arrive on its barriers, or while pair MMAs are in flight (the
    // even CTA's MMA thread waited for them above).
    __syncwarp();
    tc_fence_before();
    cluster_sync();
    if (warp == pf::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

// cuTensorMapEncodeTiled from the driver, found once through the runtime (the
// library links only the CUDA runtime).
static PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 2D tensor map over a row-major array of `outer` rows of `inner` elements,
// `row_bytes` apart; boxes of box_in x box_out elements, out-of-range elements
// read as zero.
hq_status make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle swz) {
    const auto encode = encode_tiled();
    if (!encode) return HQ_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_in, box_out};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? HQ_OK : HQ_ERR_CUDA;
}

// Tensor map of the activation codes: 4-bit codes Xq[M][K/2] in boxes of 64
// packed bytes x 128 rows (into the packed ring); 8-bit codes Xq[M][K] in
// boxes of 128 bytes x 128 rows, 128-byte swizzled, straight into the MMA's
// operand stage.  Rows past M read as zero.
static hq_status xq_tensor_map(const GemmArgs& a, CUtensorMap* map, bool a8) {
    const uint64_t row = static_cast<uint64_t>(a8 ? a.K : a.K / 2);
    return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq, row, static_cast<uint64_t>(a.M), row,
                        a8 ? pf::BK : pf::PK_ROW, pf::BM, a8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int BN, bool ASYM, bool A8, int OUT>
static hq_status launch_pf_t(const GemmArgs& a, cudaStream_t st, int nsm) {
    auto kern = k_gemm_pf<BN, ASYM, A8, OUT>;
    const int smem = PfSmem<BN, ASYM, A8>::ALLOC;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    CUtensorMap tmX;
    const hq_status s = xq_tensor_map(a, &tmX, A8);
    if (s != HQ_OK) return s;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(pf::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // CTA pairs that fit on the device at once (a pair needs two SMs of one
    // cluster-capable group, so this can be below nsm / 2); queried once per
    // device and kernel variant
    // (host threads may launch concurrently: the cache entries are atomic, and
    // a race only repeats the query)
    static std::atomic<int> max_pairs[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HQ_ERR_CUDA;
    int mp = max_pairs[dev].load(std::memory_order_relaxed);
    if (mp == 0) {
        cfg.gridDim = dim3(2 * (nsm / 2), 1, 1);
        if (cudaOccupancyMaxActiveClusters(&mp, kern, &cfg) != cudaSuccess || mp <= 0) return HQ_ERR_CUDA;
        max_pairs[dev].store(mp, std::memory_order_relaxed);
    }
    const int tiles = ((a.M + 2 * pf::BM - 1) / (2 * pf::BM)) * ((a.N + BN - 1) / BN);
    const int pairs = tiles < mp ? tiles : mp;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    if (cudaLaunchKernelEx(&cfg, kern, a, tmX) != cudaSuccess) return HQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}
template <bool A8>
static hq_status launch_pf_a(const GemmArgs& a, int out, cudaStream_t st, int nsm) {
    if (a.gw == 0) {
        switch (out) {
            case HQ_F16: return launch_pf_t<256, false, A8, HQ_F16>(a, st, nsm);
            case HQ_BF16: return launch_pf_t<256, false, A8, HQ_BF16>(a, st, nsm);
            case HQ_F32: return launch_pf_t<256, false, A8, HQ_F32>(a, st, nsm);
            case OUT_DEBUG: return launch_pf_t<256, false, A8, OUT_DEBUG>(a, st, nsm);
        }
    } else {
        switch (out) {
            case HQ_F16: return launch_pf_t<128, true, A8, HQ_F16>(a, st, nsm);
            case HQ_BF16: return launch_pf_t<128, true, A8, HQ_BF16>(a, st, nsm);
            case HQ_F32: return launch_pf_t<128, true, A8, HQ_F32>(a, st, nsm);
            case OUT_DEBUG: return launch_pf_t<128, true, A8, OUT_DEBUG>(a, st, nsm);
        }
    }
    return HQ_ERR_UNSUPPORTED;
}

hq_status launch_gemm_prefill(const GemmArgs& a, int out, cudaStream_t st, int nsm) {
    return a.act_bits == 8 ? launch_pf_a<true>(a, out, st, nsm) : launch_pf_a<false>(a, out, st, nsm);
}

}  // namespace hq
