// gemm_small.cu -- kernel K2 for small M (decode: up to 64 tokens): the same
// W4A4 GEMM with SERQ's fused term as gemm.cu, organised for a layer whose
// cost is streaming the packed weights from HBM once.
//
// Source: "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
// Quantization", technical summary sections 2.2-3 (one 4-bit matmul plus the
// single residual path on the salient rows); group-wise scale and zero point
// from "OffQ: Taming Structured Outliers in LLM Quantization by Offsetting",
// Methodology 3.
//
// With at most 64 tokens the layer does at most 128 MACs per weight byte it
// streams: it is bound by HBM, and the tensor core only has to keep up with
// the weight stream.  What limits a kernel of this size is the latency of
// every serial step (a single thread that issues copies or MMAs, hand-offs
// through barriers), so this one has none: every warp streams, expands and
// multiplies on its own, with warp-level int8 MMAs (m16n8k32) fed from
// registers, and the warps meet once, at the end.
//
// Design (one CTA per SM, no workspace, no cross-CTA traffic):
//  * row slices: CTA c owns the weight rows [c N / grid, (c + 1) N / grid), so
//    every SM streams the same number of weight bytes (within one row) and
//    finishes its own outputs: no split-K partial sums across CTAs.
//  * the slice is cut into 16-row tiles; each warp takes one tile and a
//    contiguous range of its K-blocks (128 inputs), the ranges of a tile
//    splitting K evenly among the warps the tile gets.
//  * weights: each thread owns one 16-byte quarter of two rows (g, g + 8) of
//    every K-block, i.e. 32 codes of each row, and streams them with 16-byte
//    cp.async copies into its own slots of a ring in shared memory, 8 K-blocks
//    ahead (a warp's K-block is one contiguous kilobyte of the tile-major
//    layout).  A thread reads back only what it copied: no barrier.
//  * K order: the MMA's 32-input step pairs input columns 4t..4t+3 and
//    16+4t..16+4t+3 of lane t; the kernel maps them to the low and high nibbles
//    of one packed 32-bit word of 8 codes (inputs k0 k2 k4 k6 / k1 k3 k5 k7),
//    the same for weights and tokens, so expanding a word to the A or B
//    fragment is a mask and a shift, and the dot product is unchanged.
//  * zero points: weights enter the MMA as their unsigned codes u (0..15), and
//    a group's accumulator is acc - z * S with S the token's code sum over the
//    same inputs (per-channel weights: z = 8, the offset of the signed codes).
//    With the tokens staged in shared memory, the CTA sums each token's codes
//    per K-block once; otherwise a second MMA with an all-ones A fragment
//    gives S.
//  * group accumulators start from the bits of 1.5 * 2^23, so at the end of a
//    group the int32 result reads as an exact float offset by that constant:
//    one packed add, then packed fmas for - z * S and the scale sw[b][n].
//  * the group's zero points and scales ride in the same ring: six lanes copy
//    the aligned 16-byte chunks that hold the warp's 16 rows, and the warp
//    reads them after a __syncwarp.
//  * tokens (the activation codes) are staged once per CTA in shared memory
//    by bulk copies after the dependency wait (rows padded by 64 bytes, so
//    the fragment loads hit distinct banks); when they do not fit, each
//    thread loads its fragments through L1, prefetched 8 K-blocks ahead.
//  * the warps of a tile add their partial sums in shared memory in a fixed
//    order; one warp per tile finishes: the SERQ term X[m,S] . Rq[n,:] on
//    mma.sync, sx[m], the store.
//  * OffQ activations (OQ): unsigned codes with a scale and an integer zero
//    point per token and 128-input group, i.e. per K-block.  Per K-block the
//    accumulator is acc = raw - zw Sx - zx (Su - 128 zw), raw the MMA of the
//    unsigned codes, Sx the token's code sum, Su the weight row's code sum
//    (dp4a in the lanes, two shuffles), and it is scaled by sx[m][b] sw[n]
//    there; the SERQ term is an fp32 dot product of the dequantised salient
//    activations with the Rq rows ("OffQ ...", Methodology 2-3).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "hq_device.cuh"
#include "hq_gemm.cuh"

namespace hq {

namespace dk {
constexpr int BK = 128;                  // inputs per K-block
constexpr int TSLOT = 1152;              // one tile's share of a warp's K-block: 2 rows x 32 threads x
                                         // 16 bytes, then 3 + 3 chunks of 8 zero points / scales
constexpr int SMEM_MAX = 232448;         // opt-in dynamic shared memory per block
constexpr int XS_WORDS = 16;             // salient codes per token as int8 words (r <= 64)
constexpr uint32_t MAGIC = 0x4B400000u;  // bits of the float 1.5 * 2^23
constexpr float MAGIC_F = 12582912.0f;
}  // namespace dk

template <int NT>
struct DkCfg {
    static constexpr int W = NT == 64 ? 8 : (NT == 32 ? 12 : 16);   // warps
    static constexpr int TPW = 1;                            // 16-row tiles per warp (2 measured slower)
    static constexpr int THREADS = 32 * W;
    static constexpr int NTT = NT / 8;                       // MMA n-tiles of 8 tokens
    static constexpr int SLOT = TPW * dk::TSLOT;             // bytes of one warp's K-block in its ring
    static constexpr int PART = W * 32 * TPW * NTT * 16;     // partial sums, aliased onto the rings
    static constexpr int MAXROWS = W * TPW * 16;             // rows of one pass
    // after the rings: the token barrier, salient codes, the pass's SERQ rows
    // Rq (r/2 bytes each), sr and sw (fp16 pairs from an even row), and sx
    static constexpr int F_BAR = 0;
    static constexpr int F_XS = 16;
    static constexpr int F_RQ = F_XS + NT * dk::XS_WORDS * 4;
    static constexpr int F_SR = F_RQ + MAXROWS * 32;
    static constexpr int F_SW = F_SR + (MAXROWS + 8) * 2;
    static constexpr int F_SX = F_SW + (MAXROWS + 8) * 2;
    static constexpr int F_AS = (F_SX + NT * 4 + 15) / 16 * 16;       // OffQ: [NT][64] dequantised salient activations
    static constexpr int FIX = F_AS + NT * 64 * 4;
    static constexpr int XITEMS = (NT * dk::XS_WORDS + THREADS - 1) / THREADS;
};

struct DkPlan {
    int grid;      // CTAs; CTA c owns weight rows [c N / grid, (c + 1) N / grid)
    int D;         // K-blocks in flight per warp (8, 4 or 2)
    int ring;      // bytes of the rings (W x D slots)
    int tstride;   // bytes per staged token row (row bytes + 64)
    int tbytes;    // bytes of the staged tokens and their sums (0 when not staged)
};

static int nt_for(int64_t M) { return M <= 8 ? 8 : (M <= 16 ? 16 : (M <= 32 ? 32 : 64)); }

// Launch plan; `staged` tells whether the tokens fit in shared memory.
template <int NT>
static DkPlan dk_plan(int64_t M, int64_t N, int64_t K, bool a8, int nsm, bool& staged, bool oq = false) {
    using C = DkCfg<NT>;
    DkPlan p{};
    const int want = nsm > 0 ? nsm : 148;
    const int64_t tiles = (N + 15) / 16;   // at least one 16-row tile per CTA
    p.grid = static_cast<int>(tiles < want ? tiles : want);
    p.tstride = static_cast<int>(a8 ? K : K / 2) + 64;
    // staged token rows, then their code sums per K-block (int32 [K/128][NT])
    // (OffQ activations: then their zero points and group scales, [K/128][NT] each)
    const int64_t tok = static_cast<int64_t>(NT) * p.tstride + (K / dk::BK) * NT * (oq ? 12 : 4);
    const int depths[3] = {8, 4, 2};
    for (int st = 1; st >= (oq ? 1 : 0); --st) {
        for (int d : depths) {
            if (st && d < 4 && C::TPW == 1) continue;
            const int64_t ring = static_cast<int64_t>(C::W) * d * C::SLOT;
            if (ring >= C::PART && ring + C::FIX + (st ? tok : 0) <= dk::SMEM_MAX) {
                staged = st != 0;
                p.D = d;
                p.ring = static_cast<int>(ring);
                p.tbytes = st ? static_cast<int>(tok) : 0;
                return p;
            }
        }
    }
    staged = false;
    p.D = 0;   // nothing fits (not reached for the supported shapes)
    return p;
}

template <int OUT>
__device__ __forceinline__ void store_one(void* Y, int64_t i, float y) {
    if constexpr (OUT == HQ_F32) {
        static_cast<float*>(Y)[i] = y;
    } else if constexpr (OUT == HQ_BF16) {
        static_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(y);
    } else {
        static_cast<__half*>(Y)[i] = __float2half_rn(y);
    }
}

// d = a * b + c (int8 x int8 -> int32, 16 x 8 x 32); c may alias d.
__device__ __forceinline__ void mma_s8_c(uint32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                         const uint32_t (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %11, %12, %13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]),
          "r"(c[3]));
}

// B fragment words of 8 tokens codes k0..k7 held as two words (k0..k3,
// k4..k7): (k0 k2 k4 k6) and (k1 k3 k5 k7), the order of unpack_s4x8_times16.
__device__ __forceinline__ void tok_words8(uint32_t x0, uint32_t x1, uint32_t& lo, uint32_t& hi) {
    lo = __byte_perm(x0, x1, 0x6420);
    hi = __byte_perm(x0, x1, 0x7531);
}

__device__ __forceinline__ void cp_async_wait_depth(int D) {
    if (D == 8) cp_async_wait_group<7>();
    else if (D == 4) cp_async_wait_group<3>();
    else cp_async_wait_group<1>();
}

// A8: 8-bit activation codes ([M][K] int8, used as they are) instead of packed
// 4-bit codes (expanded as 16 q).  TS: tokens staged in shared memory.
template <int NT, bool ASYM, bool A8, int OUT, bool TS, bool OQ = false>
__global__ void __launch_bounds__(DkCfg<NT>::THREADS, 1) k_gemm_small(const GemmArgs p, const DkPlan plan) {
    static_assert(!OQ || (TS && !A8), "OffQ activations: staged 4-bit tokens");
    using C = DkCfg<NT>;
    constexpr int NTT = C::NTT;
    constexpr int W = C::W;
    constexpr int TPW = C::TPW;
    constexpr int TOKV = A8 ? 2 : 1;                   // uint4 per token fragment and K-block
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* fix = smem + plan.ring;
    const uint32_t tbar = smem_u32(fix + C::F_BAR);
    uint32_t* xs_s = reinterpret_cast<uint32_t*>(fix + C::F_XS);
    const uint8_t* rq_s = fix + C::F_RQ;
    const uint16_t* sr_s = reinterpret_cast<const uint16_t*>(fix + C::F_SR);
    const uint16_t* sw_s = reinterpret_cast<const uint16_t*>(fix + C::F_SW);
    float* sx_s = reinterpret_cast<float*>(fix + C::F_SX);
    uint8_t* tok_s = fix + C::FIX;
    int32_t* tsum_s = reinterpret_cast<int32_t*>(tok_s + NT * plan.tstride);   // [K/128][NT]
    int32_t* zxg_s = tsum_s + (p.K / dk::BK) * NT;                            // OffQ: [K/128][NT] zero points
    float* sxg_s = reinterpret_cast<float*>(zxg_s + (p.K / dk::BK) * NT);     // OffQ: [K/128][NT] group scales
    float* as_s = reinterpret_cast<float*>(fix + C::F_AS);                    // OffQ: [NT][64]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int cta = blockIdx.x;
    const int r0 = static_cast<int>(static_cast<long long>(cta) * p.N / plan.grid);
    const int r1 = static_cast<int>(static_cast<long long>(cta + 1) * p.N / plan.grid);
    const int RG = (r1 - r0 + 16 * TPW - 1) / (16 * TPW);   // groups of TPW 16-row tiles
    const int KB = p.K / dk::BK;
    const int gs = ASYM ? p.gw / dk::BK : KB;         // K-blocks per weight group
    const int G = ASYM ? p.K / p.gw : 1;
    const int64_t xrow = A8 ? p.K : p.K / 2;           // bytes per token row
    const int D = plan.D;
    // the accumulators carry the factor 16 of 4-bit signed activation codes
    constexpr int sh = (A8 || OQ) ? 0 : 4;
    constexpr float inv_act = (A8 || OQ) ? 1.0f : 0.0625f;

    if constexpr (TS) {
        if (tid == 0) {
            mbar_init(tbar, 1);
            fence_mbar_init();
        }
        // token rows past M read as zero
        for (int i = tid; i < (NT - p.M) * (plan.tstride / 16); i += C::THREADS)
            *reinterpret_cast<uint4*>(tok_s + (p.M + i / (plan.tstride / 16)) * plan.tstride + 16 * (i % (plan.tstride / 16))) =
                make_uint4(0, 0, 0, 0);
        __syncthreads();
    }

    // salient activation codes of every token, gathered into xs_s before the
    // finish in the lo/hi word order of unpack_s4x8_times16: the indices now,
    // the codes after the dependency wait, the shared-memory stores at the end
    int salk[C::XITEMS][4];
#pragma unroll
    for (int it = 0; it < C::XITEMS; ++it) {
        const int idx = tid + it * C::THREADS;
        const int m = idx / dk::XS_WORDS, w = idx % dk::XS_WORDS;
        const int i = w >> 1, hh = w & 1;   // word 2i+hh holds positions 8i+2e+hh, byte e
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = 8 * i + 2 * e + hh;
            // (checked when used: a test here would wait for the load)
            salk[it][e] = (idx < NT * dk::XS_WORDS && m < p.M && j < p.r) ? __ldg(p.sal + j) : -1;
        }
    }
    uint32_t xsw[C::XITEMS];
    bool waited = false, gathered = false;
    auto deps = [&]() {
        // the token codes are the preceding kernel's output
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if constexpr (TS) {
            if (warp == 0) {
                if (lane == 0) mbar_arrive_expect_tx(tbar, static_cast<uint32_t>(p.M * xrow));
                __syncwarp();
                for (int m = lane; m < p.M; m += 32)
                    bulk_copy_g2s(smem_u32(tok_s + m * plan.tstride), p.Xq + m * xrow, static_cast<uint32_t>(xrow), tbar);
            }
        }
        waited = true;
    };
    // (issued once the salient indices have arrived, so the loads do not stall)
    auto gather = [&]() {
        if (!waited) deps();
#pragma unroll
        for (int it = 0; it < C::XITEMS; ++it) {
            const int m = (tid + it * C::THREADS) / dk::XS_WORDS;
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = salk[it][e];
                if (k >= p.K) record_status(HQ_ERR_ARG);   // a salient index outside [0, K): skipped
                if (k >= 0 && k < p.K) {
                    const uint8_t* xr = p.Xq + static_cast<int64_t>(m) * xrow;
                    if constexpr (A8) {
                        word |= static_cast<uint32_t>(__ldg(xr + k)) << (8 * e);
                    } else {
                        const int nib = (__ldg(xr + (k >> 1)) >> ((k & 1) * 4)) & 0xF;
                        word |= (static_cast<uint32_t>((nib ^ 8) - 8) & 0xFFu) << (8 * e);
                    }
                }
            }
            xsw[it] = word;
        }
        if constexpr (OQ) {
            // dequantised salient activations sx[m][b] (q - zx[m][b]), b = S_j / 128
            const int KB_ = p.K / dk::BK;
            for (int idx = tid; idx < NT * 64; idx += C::THREADS) {
                const int m = idx >> 6, j = idx & 63;
                float a = 0.f;
                if (m < p.M && j < p.r) {
                    const int k = __ldg(p.sal + j);
                    if (static_cast<unsigned>(k) < static_cast<unsigned>(p.K)) {
                        const int b = k / dk::BK;
                        const int q = (__ldg(p.Xq + static_cast<int64_t>(m) * xrow + (k >> 1)) >> ((k & 1) * 4)) & 0xF;
                        const float sg = OUT == OUT_DEBUG ? 0.f : __ldg(p.sx + static_cast<int64_t>(m) * KB_ + b);
                        a = __fmul_rn(sg, static_cast<float>(q - __ldg(p.zx + static_cast<int64_t>(m) * KB_ + b)));
                    }
                }
                as_s[idx] = a;
            }
        } else if constexpr (OUT != OUT_DEBUG) {   // the debug entry passes no scales
            for (int m = tid; m < NT; m += C::THREADS) sx_s[m] = m < p.M ? p.sx[m] : 0.f;
        }
        gathered = true;
    };

    const uint32_t ring = smem_u32(smem + warp * D * C::SLOT);
    const uint32_t ones[4] = {0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u};
    const uint32_t zero4[4] = {0u, 0u, 0u, 0u};
    const uint32_t mag4[4] = {dk::MAGIC, dk::MAGIC, dk::MAGIC, dk::MAGIC};
    bool tok_ready = !TS;   // (pass 0 of the active warps: tokens landed and summed)

    const int npass = (RG + W - 1) / W;
    for (int pass = 0; pass < npass; ++pass) {
        const int t0 = pass * W;                         // first group of the pass
        const int ntp = (RG - t0) < W ? (RG - t0) : W;   // groups of this pass
        const int S = W / ntp;                           // warps per group
        const int tl = warp % ntp, sp = warp / ntp;
        const bool active = sp < S;
        const int gbase = r0 + 16 * TPW * (t0 + tl);     // the warp's first row
        // rows g and g + 8 of each of the warp's tiles
        int rowA[TPW], rowB[TPW], c0[TPW];
        bool okA[TPW], okB[TPW];
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
            rowA[j] = gbase + 16 * j + gq;
            rowB[j] = rowA[j] + 8;
            okA[j] = rowA[j] < r1;
            okB[j] = rowB[j] < r1;
            c0[j] = (gbase + 16 * j) & ~7;               // first of the tile's 8-row chunks of zero points / scales
        }
        // the finish's operands of this pass's rows [pr0, pr1), in flight during the K loop:
        // Rq rows (r/2 bytes each, a multiple of 4), and the fp16 pairs of sr and
        // (per-channel) sw from the even row pb = pr0 & ~1
        const int pr0 = r0 + 16 * TPW * t0;
        const int pr1 = (r0 + 16 * TPW * (t0 + ntp)) < r1 ? r0 + 16 * TPW * (t0 + ntp) : r1;
        const int pb = pr0 & ~1;
        {
            const int nrq = (pr1 - pr0) * (p.r / 8);
            for (int idx = tid; idx < nrq; idx += C::THREADS)
                cp_async4(smem_u32(rq_s + 4 * idx), p.Rq + static_cast<int64_t>(pr0) * (p.r / 2) + 4 * idx);
            if constexpr (OUT != OUT_DEBUG) {
                const int npair = (pr1 - pb + 1) / 2;
                for (int idx = tid; idx < npair; idx += C::THREADS) {
                    if (p.r > 0) cp_async4(smem_u32(sr_s + 2 * idx), p.sr + pb + 2 * idx);
                    if constexpr (!ASYM) cp_async4(smem_u32(sw_s + 2 * idx), p.sw + pb + 2 * idx);
                }
            }
        }
        const int kb0 = static_cast<int>(static_cast<long long>(sp) * KB / S);
        int kb1 = active ? static_cast<int>(static_cast<long long>(sp + 1) * KB / S) : kb0;
        // partial sums of this warp's K range, in the m16n8 accumulator layout:
        // [j][nt][0,1] = tile j row g, tokens 8 nt + 2 t + {0,1}; [j][nt][2,3] = row g + 8
        float y[TPW][NTT][4];
        int32_t yi[TPW][NTT][4];
#pragma unroll
        for (int j = 0; j < TPW; ++j)
#pragma unroll
            for (int nt = 0; nt < NTT; ++nt)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    y[j][nt][v] = 0.f;
                    yi[j][nt][v] = 0;
                }
        // request cursor: next K-block, its ring slot, its sources (one weight tile
        // after another: consecutive K-blocks of a row are 8 KB apart)
        int ik = kb0, islot = 0, igk = kb0 % gs;
        const uint8_t* srcA[TPW];
        const uint8_t* srcB[TPW];
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
            srcA[j] = p.Wq + (static_cast<int64_t>(rowA[j] >> 7) * KB + kb0) * 8192 + (rowA[j] & 127) * 64 + tq * 16;
            srcB[j] = p.Wq + (static_cast<int64_t>(rowB[j] >> 7) * KB + kb0) * 8192 + (rowB[j] & 127) * 64 + tq * 16;
        }
        // zero points and scales of rows [c0, c0 + 24) of the group, per tile: lane
        // 6 j + 0..2 copies zero-point chunk 0..2 of tile j, 6 j + 3..5 its scale
        // chunks (16-byte chunks of 8 rows; N % 8 == 0)
        const int zt = lane / 6, zl = lane % 6, zj = zl < 3 ? zl : zl - 3;
        const int zc0 = zt < TPW ? c0[zt < TPW ? zt : 0] : 0;
        const bool zlane = ASYM && zt < TPW && zl < (OUT == OUT_DEBUG ? 3 : 6) && zc0 + 8 * zj < p.N;
        const uint16_t* zsrc = nullptr;
        if constexpr (ASYM)
            zsrc = (zl < 3 || OUT == OUT_DEBUG ? p.zw : p.sw) + static_cast<int64_t>(kb0 / gs) * p.N + zc0 + 8 * zj;
        const uint32_t zdst = static_cast<uint32_t>(1024 * TPW + 96 * zt + 48 * (zl / 3) + 16 * zj);
        auto issue = [&]() {
            if (ik < kb1) {
                const uint32_t slot = ring + static_cast<uint32_t>(islot) * C::SLOT;
#pragma unroll
                for (int j = 0; j < TPW; ++j) {
                    if (okA[j]) cp_async16(slot + 1024 * j + lane * 16, srcA[j]);
                    if (okB[j]) cp_async16(slot + 1024 * j + 512 + lane * 16, srcB[j]);
                    srcA[j] += 8192;
                    srcB[j] += 8192;
                }
                if constexpr (ASYM) {
                    if (zlane) cp_async16(slot + zdst, zsrc);
                    if (++igk == gs) {
                        igk = 0;
                        zsrc += p.N;
                    }
                }
                ++ik;
                islot = islot + 1 == D ? 0 : islot + 1;
            }
            cp_async_commit();   // one group per K-block (possibly empty)
        };
        // token codes of K-block kb into L1 ahead of their loads (after the dependency wait only)
        auto tok_prefetch = [&](int kb) {
            if constexpr (!TS) {
                if (kb < kb1) {
#pragma unroll
                    for (int nt = 0; nt < NTT; ++nt) {
                        const int m = 8 * nt + gq;
                        if (m < p.M && tq == 0) prefetch_l1(p.Xq + static_cast<int64_t>(m) * xrow + kb * (A8 ? 128 : 64));
                    }
                }
            }
        };

        if (active) {
            if (warp == 0 && !waited) deps();   // the tokens are on every warp's critical path
            for (int d = 0; d < D; ++d) issue();
            if (!waited) deps();
            for (int d = 0; d < D; ++d) tok_prefetch(kb0 + d);
            if (!tok_ready) {
                if (!mbar_wait(tbar, 0, p.limit_ns)) kb1 = kb0;   // timeout recorded: skip the K loop
                // each token's code sum per K-block (16 sum q for 4-bit codes),
                // shared by the warps of this pass (a prefix of the CTA's warps)
                const int nact = S * ntp * 32;
                for (int idx = tid; idx < KB * NT; idx += nact) {
                    const int kbs = idx / NT, m = idx - kbs * NT;
                    const uint4* src = reinterpret_cast<const uint4*>(tok_s + m * plan.tstride + kbs * (A8 ? 128 : 64));
                    int sum = 0;
#pragma unroll
                    for (int c = 0; c < (A8 ? 8 : 4); ++c) {
                        const uint4 v = src[c];
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            if constexpr (A8) {
                                sum = __dp4a(static_cast<int>(w[e]), 0x01010101, sum);
                            } else {
                                const uint32_t u = OQ ? w[e] : w[e] ^ 0x88888888u;   // q (+ 8 for signed codes) per nibble
                                sum = __dp4a(static_cast<int>((u & 0x0F0F0F0Fu) + ((u >> 4) & 0x0F0F0F0Fu)), 0x01010101, sum);
                            }
                        }
                    }
                    tsum_s[idx] = (A8 || OQ) ? sum : 16 * (sum - 8 * dk::BK);
                    if constexpr (OQ) {
                        const bool mv = m < p.M;
                        zxg_s[idx] = mv ? __ldg(p.zx + static_cast<int64_t>(m) * KB + kbs) : 0;
                        sxg_s[idx] = (mv && OUT != OUT_DEBUG) ? __ldg(p.sx + static_cast<int64_t>(m) * KB + kbs) : 0.f;
                    }
                }
                named_bar_sync(1, nact);
                tok_ready = true;
            }
            uint32_t acc[TPW][NTT][4], ssum[NTT][4];
            int32_t sacc[NTT][2];   // token sums of this warp's share of the current group (staged tokens)
            bool fresh = true;
            int cslot = 0, cgk = kb0 % gs, cg = kb0 / gs;   // consume cursor: ring slot, place in group, group
            for (int kb = kb0; kb < kb1; ++kb) {
                // this thread's copies of K-block kb have landed; the warp's too after the __syncwarp
                cp_async_wait_depth(D);
                if constexpr (ASYM) __syncwarp();
                const uint8_t* slot = smem + (warp * D + cslot) * C::SLOT;
                cslot = cslot + 1 == D ? 0 : cslot + 1;
                uint4 wa[TPW], wb[TPW];
                uint32_t za[TPW], sa[TPW];   // fp16 bits, low half = row g
#pragma unroll
                for (int j = 0; j < TPW; ++j) {
                    wa[j] = *reinterpret_cast<const uint4*>(slot + 1024 * j + lane * 16);
                    wb[j] = *reinterpret_cast<const uint4*>(slot + 1024 * j + 512 + lane * 16);
                    za[j] = sa[j] = 0;
                    if constexpr (ASYM) {
                        const uint16_t* zc = reinterpret_cast<const uint16_t*>(slot + 1024 * TPW + 96 * j);
                        za[j] = zc[rowA[j] - c0[j]] | (static_cast<uint32_t>(zc[rowB[j] - c0[j]]) << 16);
                        if constexpr (OUT != OUT_DEBUG)
                            sa[j] = zc[24 + rowA[j] - c0[j]] | (static_cast<uint32_t>(zc[24 + rowB[j] - c0[j]]) << 16);
                    }
                }
                if constexpr (ASYM) __syncwarp();   // every lane has read the shared chunks before the slot is refilled
                issue();
                tok_prefetch(kb + D);
                // token fragments: per n-tile, the 16 (32 for 8-bit codes) bytes of token
                // 8 nt + g at this lane's quarter of the K-block
                uint4 tn[NTT][TOKV];
#pragma unroll
                for (int nt = 0; nt < NTT; ++nt) {
                    const int m = 8 * nt + gq;
#pragma unroll
                    for (int v = 0; v < TOKV; ++v) {
                        const int64_t off = kb * (A8 ? 128 : 64) + tq * (A8 ? 32 : 16) + 16 * v;
                        if constexpr (TS) {
                            tn[nt][v] = *reinterpret_cast<const uint4*>(tok_s + m * plan.tstride + off);
                        } else {
                            tn[nt][v] = m < p.M ? __ldg(reinterpret_cast<const uint4*>(p.Xq + m * xrow + off))
                                                : make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                int su[TPW][2] = {};   // OffQ: this lane's share of the rows' code sums
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    // A fragments of step s: unsigned codes u (per-channel: signed code + 8)
                    uint32_t af[TPW][4];
#pragma unroll
                    for (int j = 0; j < TPW; ++j) {
                        const uint32_t wA[4] = {wa[j].x, wa[j].y, wa[j].z, wa[j].w};
                        const uint32_t wB[4] = {wb[j].x, wb[j].y, wb[j].z, wb[j].w};
                        const uint32_t fa = ASYM ? wA[s] : wA[s] ^ 0x88888888u;
                        const uint32_t fb = ASYM ? wB[s] : wB[s] ^ 0x88888888u;
                        af[j][0] = fa & 0x0F0F0F0Fu;
                        af[j][1] = fb & 0x0F0F0F0Fu;
                        af[j][2] = (fa >> 4) & 0x0F0F0F0Fu;
                        af[j][3] = (fb >> 4) & 0x0F0F0F0Fu;
                        if constexpr (OQ) {
                            su[j][0] = __dp4a(static_cast<int>(af[j][0] + af[j][2]), 0x01010101, su[j][0]);
                            su[j][1] = __dp4a(static_cast<int>(af[j][1] + af[j][3]), 0x01010101, su[j][1]);
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NTT; ++nt) {
                        uint32_t b0, b1;
                        if constexpr (A8) {
                            const uint4 t0v = tn[nt][0], t1v = tn[nt][TOKV - 1];
                            const uint32_t x[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
                            tok_words8(x[2 * s], x[2 * s + 1], b0, b1);
                        } else if constexpr (OQ) {
                            const uint32_t x[4] = {tn[nt][0].x, tn[nt][0].y, tn[nt][0].z, tn[nt][0].w};
                            b0 = x[s] & 0x0F0F0F0Fu;           // unsigned codes, (k0 k2 k4 k6)
                            b1 = (x[s] >> 4) & 0x0F0F0F0Fu;    // (k1 k3 k5 k7)
                        } else {
                            const uint32_t x[4] = {tn[nt][0].x, tn[nt][0].y, tn[nt][0].z, tn[nt][0].w};
                            unpack_s4x8_times16(x[s], b0, b1);
                        }
                        if (fresh && s == 0) {
#pragma unroll
                            for (int j = 0; j < TPW; ++j) mma_s8_c(acc[j][nt], af[j], b0, b1, (ASYM || OQ) ? mag4 : zero4);
                            if constexpr (!TS) mma_s8_c(ssum[nt], ones, b0, b1, ASYM ? mag4 : zero4);
                        } else {
#pragma unroll
                            for (int j = 0; j < TPW; ++j) mma_s8_c(acc[j][nt], af[j], b0, b1, acc[j][nt]);
                            if constexpr (!TS) mma_s8_c(ssum[nt], ones, b0, b1, ssum[nt]);
                        }
                    }
                }
                if constexpr (TS) {
#pragma unroll
                    for (int nt = 0; nt < NTT; ++nt) {
                        const int2 sv = *reinterpret_cast<const int2*>(tsum_s + kb * NT + 8 * nt + 2 * tq);
                        sacc[nt][0] = (fresh ? 0 : sacc[nt][0]) + sv.x;
                        sacc[nt][1] = (fresh ? 0 : sacc[nt][1]) + sv.y;
                    }
                }
                fresh = false;
                if (!gathered) gather();
                if constexpr (OQ) {
                    // one activation group per K-block: acc = raw - zw Sx - zx (Su - 128 zw),
                    // scaled by sx[m][b] sw[n] (per-channel weights: sw at the end)
#pragma unroll
                    for (int j = 0; j < TPW; ++j) {
                        int sua = su[j][0], sub = su[j][1];
                        sua += __shfl_xor_sync(0xFFFFFFFFu, sua, 1);
                        sua += __shfl_xor_sync(0xFFFFFFFFu, sua, 2);
                        sub += __shfl_xor_sync(0xFFFFFFFFu, sub, 1);
                        sub += __shfl_xor_sync(0xFFFFFFFFu, sub, 2);
                        const int zia = ASYM ? static_cast<int>(__half2float(__ushort_as_half(static_cast<uint16_t>(za[j] & 0xFFFFu)))) : 8;
                        const int zib = ASYM ? static_cast<int>(__half2float(__ushort_as_half(static_cast<uint16_t>(za[j] >> 16)))) : 8;
                        const int sua2 = sua - dk::BK * zia, sub2 = sub - dk::BK * zib;
                        float swa = 1.f, swb = 1.f;
                        if constexpr (ASYM && OUT != OUT_DEBUG) {
                            swa = __half2float(__ushort_as_half(static_cast<uint16_t>(sa[j] & 0xFFFFu)));
                            swb = __half2float(__ushort_as_half(static_cast<uint16_t>(sa[j] >> 16)));
                        }
#pragma unroll
                        for (int nt = 0; nt < NTT; ++nt) {
                            const int ti = kb * NT + 8 * nt + 2 * tq;
                            const int2 sxk = *reinterpret_cast<const int2*>(tsum_s + ti);
                            const int2 zk = *reinterpret_cast<const int2*>(zxg_s + ti);
                            const float2 gk = *reinterpret_cast<const float2*>(sxg_s + ti);
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const int tsx = (v & 1) ? sxk.y : sxk.x, tzx = (v & 1) ? zk.y : zk.x;
                                const int a = static_cast<int>(acc[j][nt][v] - dk::MAGIC) - (v < 2 ? zia : zib) * tsx -
                                              tzx * (v < 2 ? sua2 : sub2);
                                if constexpr (OUT == OUT_DEBUG) {
                                    const int m = 8 * nt + 2 * tq + (v & 1);
                                    const int n = v < 2 ? rowA[j] : rowB[j];
                                    if ((v < 2 ? okA[j] : okB[j]) && m < p.M)
                                        atomicAdd(p.dbg_acc + (static_cast<int64_t>(m) * p.N + n) * KB + kb, a);
                                } else {
                                    const float coef = __fmul_rn((v & 1) ? gk.y : gk.x, v < 2 ? swa : swb);
                                    y[j][nt][v] = __fmaf_rn(coef, static_cast<float>(a), y[j][nt][v]);
                                }
                            }
                        }
                    }
                    fresh = true;
                } else if constexpr (ASYM) {
                    const bool gend = ++cgk == gs;
                    if (gend) cgk = 0;
                    if (gend || kb + 1 == kb1) {
                        // end of a group (or of this warp's share of it): acc - z S, scaled
#pragma unroll
                        for (int j = 0; j < TPW; ++j) {
                            const float zfa = __half2float(__ushort_as_half(static_cast<uint16_t>(za[j] & 0xFFFFu)));
                            const float zfb = __half2float(__ushort_as_half(static_cast<uint16_t>(za[j] >> 16)));
                            if constexpr (OUT == OUT_DEBUG) {
                                const int zia = static_cast<int>(zfa), zib = static_cast<int>(zfb);
#pragma unroll
                                for (int nt = 0; nt < NTT; ++nt) {
#pragma unroll
                                    for (int v = 0; v < 4; ++v) {
                                        const int m = 8 * nt + 2 * tq + (v & 1);
                                        const int n = v < 2 ? rowA[j] : rowB[j];
                                        const int sv = TS ? sacc[nt][v & 1] : static_cast<int>(ssum[nt][v & 1] - dk::MAGIC);
                                        const int a = static_cast<int>(acc[j][nt][v] - dk::MAGIC) - (v < 2 ? zia : zib) * sv;
                                        if ((v < 2 ? okA[j] : okB[j]) && m < p.M)
                                            atomicAdd(p.dbg_acc + (static_cast<int64_t>(m) * p.N + n) * G + cg, a >> sh);
                                    }
                                }
                            } else {
                                const float sfa = __half2float(__ushort_as_half(static_cast<uint16_t>(sa[j] & 0xFFFFu))) * inv_act;
                                const float sfb = __half2float(__ushort_as_half(static_cast<uint16_t>(sa[j] >> 16))) * inv_act;
                                const float2 nmag = make_float2(-dk::MAGIC_F, -dk::MAGIC_F);
                                const float2 nza = make_float2(-zfa, -zfa), nzb = make_float2(-zfb, -zfb);
                                const float2 s2a = make_float2(sfa, sfa), s2b = make_float2(sfb, sfb);
#pragma unroll
                                for (int nt = 0; nt < NTT; ++nt) {
                                    const float2 sf = TS ? make_float2(static_cast<float>(sacc[nt][0]), static_cast<float>(sacc[nt][1]))
                                                         : __fadd2_rn(make_float2(__uint_as_float(ssum[nt][0]), __uint_as_float(ssum[nt][1])), nmag);
                                    const float2 fa = __fadd2_rn(make_float2(__uint_as_float(acc[j][nt][0]), __uint_as_float(acc[j][nt][1])), nmag);
                                    const float2 fb = __fadd2_rn(make_float2(__uint_as_float(acc[j][nt][2]), __uint_as_float(acc[j][nt][3])), nmag);
                                    const float2 ta = __ffma2_rn(nza, sf, fa);   // exact: integers below 2^24
                                    const float2 tb = __ffma2_rn(nzb, sf, fb);
                                    float2 ya = make_float2(y[j][nt][0], y[j][nt][1]), yb = make_float2(y[j][nt][2], y[j][nt][3]);
                                    ya = __ffma2_rn(s2a, ta, ya);
                                    yb = __ffma2_rn(s2b, tb, yb);
                                    y[j][nt][0] = ya.x;
                                    y[j][nt][1] = ya.y;
                                    y[j][nt][2] = yb.x;
                                    y[j][nt][3] = yb.y;
                                }
                            }
                        }
                        fresh = true;
                        if (gend) ++cg;
                    }
                }
            }
            if constexpr (!ASYM && !OQ) {
                // per-channel: signed code = u - 8, exact integer partial sums
                if (kb1 > kb0) {
#pragma unroll
                    for (int j = 0; j < TPW; ++j)
#pragma unroll
                        for (int nt = 0; nt < NTT; ++nt)
#pragma unroll
                            for (int v = 0; v < 4; ++v)
                                yi[j][nt][v] = static_cast<int32_t>(acc[j][nt][v]) -
                                               8 * (TS ? sacc[nt][v & 1] : static_cast<int32_t>(ssum[nt][v & 1]));
                }
            }
        }
        if (!gathered) gather();
        // ---- the warps of a group meet: partial sums through shared memory (over the rings)
        cp_async_wait_all();
        __syncthreads();
        if (active) {
            uint4* part = reinterpret_cast<uint4*>(smem) + (warp * 32 + lane) * (TPW * NTT);
#pragma unroll
            for (int j = 0; j < TPW; ++j)
#pragma unroll
                for (int nt = 0; nt < NTT; ++nt)
                    part[j * NTT + nt] =
                        (ASYM || OQ) ? make_uint4(__float_as_uint(y[j][nt][0]), __float_as_uint(y[j][nt][1]),
                                          __float_as_uint(y[j][nt][2]), __float_as_uint(y[j][nt][3]))
                             : make_uint4(yi[j][nt][0], yi[j][nt][1], yi[j][nt][2], yi[j][nt][3]);
        }
        if (pass == 0) {
#pragma unroll
            for (int it = 0; it < C::XITEMS; ++it) {
                const int idx = tid + it * C::THREADS;
                if (idx < NT * dk::XS_WORDS) xs_s[idx] = xsw[it];
            }
        }
        __syncthreads();
        // ---- finish: warp w < ntp completes group w in its own fragment layout
        if (warp < ntp) {
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
                // partial sums of the group's warps, added in warp order
#pragma unroll
                for (int nt = 0; nt < NTT; ++nt) {
                    float ys[4] = {0.f, 0.f, 0.f, 0.f};
                    int32_t yis[4] = {0, 0, 0, 0};
                    for (int sidx = 0; sidx < S; ++sidx) {
                        const uint4 v = reinterpret_cast<const uint4*>(smem)[((sidx * ntp + warp) * 32 + lane) * (TPW * NTT) + j * NTT + nt];
                        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if constexpr (ASYM || OQ) ys[q] = __fadd_rn(ys[q], __uint_as_float(vv[q]));
                            else yis[q] += static_cast<int32_t>(vv[q]);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        y[j][nt][q] = ys[q];
                        yi[j][nt][q] = yis[q];
                    }
                }
                // SERQ term X[m,S] . Rq[n,:] for rows g, g + 8 and the n-tiles' tokens:
                // one or two 32-input MMA steps; lane t takes packed word 4 s + t of
                // the Rq rows (A, 16 q) and the matching lo/hi words of X[m,S] (B)
                const int rw = p.r / 8;   // packed Rq words per row
                const int nA = r0 + 16 * (TPW * (t0 + warp) + j) + gq, nB = nA + 8;
                uint32_t cc[NTT][4];
#pragma unroll
                for (int nt = 0; nt < NTT; ++nt) cc[nt][0] = cc[nt][1] = cc[nt][2] = cc[nt][3] = 0;
                if constexpr (OQ) {
                    // fp32 SERQ term: sum_j a[m][j] qr[n][j] with the dequantised salient activations
                    if constexpr (OUT != OUT_DEBUG) {
#pragma unroll
                        for (int nt = 0; nt < NTT; ++nt) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int m = 8 * nt + 2 * tq + (q & 1);
                                const int n = q < 2 ? nA : nB;
                                float c = 0.f;
                                if (n < pr1) {
                                    const uint8_t* rq = rq_s + (n - pr0) * (p.r / 2);
                                    for (int jj = 0; jj < p.r; ++jj) {
                                        const int code = ((static_cast<int>(rq[jj >> 1]) >> ((jj & 1) * 4)) & 0xF) ^ 8;
                                        c = __fmaf_rn(as_s[m * 64 + jj], static_cast<float>(code - 8), c);
                                    }
                                }
                                cc[nt][q] = __float_as_uint(c);
                            }
                        }
                    }
                } else if (p.r > 0) {
                    const uint32_t* rqA = reinterpret_cast<const uint32_t*>(rq_s + (nA - pr0) * (p.r / 2));
                    const uint32_t* rqB = reinterpret_cast<const uint32_t*>(rq_s + (nB - pr0) * (p.r / 2));
#pragma unroll
                    for (int st = 0; st < 2; ++st) {
                        const int wi = 4 * st + tq;
                        if (4 * st >= rw) break;
                        const bool has = wi < rw;
                        const uint32_t qa = has && nA < pr1 ? rqA[wi] : 0u;   // (two's complement nibbles)
                        const uint32_t qb = has && nB < pr1 ? rqB[wi] : 0u;
                        uint32_t a[4];
                        unpack_s4x8_times16(qa, a[0], a[2]);
                        unpack_s4x8_times16(qb, a[1], a[3]);
#pragma unroll
                        for (int nt = 0; nt < NTT; ++nt) {
                            const int m = 8 * nt + gq;
                            const uint32_t b0 = has ? xs_s[m * dk::XS_WORDS + 2 * wi] : 0u;
                            const uint32_t b1 = has ? xs_s[m * dk::XS_WORDS + 2 * wi + 1] : 0u;
                            mma_s8_c(cc[nt], a, b0, b1, cc[nt]);
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NTT; ++nt) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int m = 8 * nt + 2 * tq + (q & 1);
                        const int n = q < 2 ? nA : nB;
                        if (n >= pr1 || m >= p.M) continue;
                        const int c = static_cast<int32_t>(cc[nt][q]) >> 4;
                        const int64_t o = static_cast<int64_t>(m) * p.N + n;
                        if constexpr (OQ) {
                            if constexpr (OUT != OUT_DEBUG) {
                                const float srn = p.r > 0 ? __half2float(__ushort_as_half(sr_s[n - pb])) : 0.f;
                                const float base = ASYM ? y[j][nt][q]
                                                        : __fmul_rn(__half2float(__ushort_as_half(sw_s[n - pb])), y[j][nt][q]);
                                store_one<OUT>(p.Y, o, __fmaf_rn(srn, __uint_as_float(cc[nt][q]), base));
                            }
                        } else if constexpr (OUT == OUT_DEBUG) {
                            if constexpr (!ASYM) p.dbg_acc[o] = yi[j][nt][q] >> sh;
                            if (p.r > 0) p.dbg_acc_c[o] = c;
                        } else {
                            const float srn = p.r > 0 ? __half2float(__ushort_as_half(sr_s[n - pb])) : 0.f;
                            const float base = ASYM ? y[j][nt][q]
                                                    : __fmul_rn(__half2float(__ushort_as_half(sw_s[n - pb])),
                                                                static_cast<float>(yi[j][nt][q] >> sh));
                            store_one<OUT>(p.Y, o, __fmul_rn(sx_s[m], __fmaf_rn(srn, static_cast<float>(c), base)));
                        }
                    }
                }
            }
        }
        __syncthreads();   // the ring is reused by the next pass
    }
    if constexpr (TS) {
        // no bulk copy may still be landing when the CTA exits (after a timeout)
        if (tid == 0) mbar_wait(tbar, 0, p.limit_ns);
    }
}

// ------------------------------------------------------------------ host side
bool small_supported(int64_t M, int gw) {
    if (M < 1 || M > 64) return false;
    return gw == 0 || gw % dk::BK == 0;
}

size_t small_workspace_bytes(int64_t, int64_t, int64_t, int, int) { return 0; }

template <int NT, bool ASYM, bool A8, int OUT, bool TS, bool OQ = false>
static hq_status launch_sk_ts(const GemmArgs& a, const DkPlan& plan, cudaStream_t st) {
    auto kern = k_gemm_small<NT, ASYM, A8, OUT, TS, OQ>;
    const int smem = plan.ring + DkCfg<NT>::FIX + plan.tbytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    // Programmatic dependent launch: the kernel may start while the preceding
    // kernel of the stream (normally the activation rotate/quant) is still
    // running; it requests its first weight K-blocks, then waits
    // (griddepcontrol.wait) before it reads activations or writes anything.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(DkCfg<NT>::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, a, plan) != cudaSuccess) return HQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

template <int NT, bool ASYM, bool A8, int OUT>
static hq_status launch_sk_t(const GemmArgs& a, cudaStream_t st, int nsm) {
    const bool oq = a.zx != nullptr;   // OffQ activations
    bool staged = false;
    const DkPlan plan = dk_plan<NT>(a.M, a.N, a.K, A8, nsm, staged, oq);
    if (plan.D == 0) return HQ_ERR_UNSUPPORTED;
    // the debug entry adds the partial group sums of the warps with atomics
    const int64_t G = oq ? a.K / dk::BK : (ASYM ? a.K / a.gw : 0);
    if (OUT == OUT_DEBUG && G > 0 &&
        cudaMemsetAsync(a.dbg_acc, 0, static_cast<size_t>(a.M) * a.N * G * sizeof(int32_t), st) != cudaSuccess)
        return HQ_ERR_CUDA;
    if (oq) {
        if constexpr (A8) return HQ_ERR_UNSUPPORTED;
        else return launch_sk_ts<NT, ASYM, false, OUT, true, true>(a, plan, st);
    }
    return staged ? launch_sk_ts<NT, ASYM, A8, OUT, true>(a, plan, st)
                  : launch_sk_ts<NT, ASYM, A8, OUT, false>(a, plan, st);
}

template <int NT, bool A8>
static hq_status launch_sk_nt(const GemmArgs& a, int out, cudaStream_t st, int nsm) {
    if (a.gw == 0) {
        switch (out) {
            case HQ_F16: return launch_sk_t<NT, false, A8, HQ_F16>(a, st, nsm);
            case HQ_BF16: return launch_sk_t<NT, false, A8, HQ_BF16>(a, st, nsm);
            case HQ_F32: return launch_sk_t<NT, false, A8, HQ_F32>(a, st, nsm);
            case OUT_DEBUG: return launch_sk_t<NT, false, A8, OUT_DEBUG>(a, st, nsm);
        }
    } else {
        switch (out) {
            case HQ_F16: return launch_sk_t<NT, true, A8, HQ_F16>(a, st, nsm);
            case HQ_BF16: return launch_sk_t<NT, true, A8, HQ_BF16>(a, st, nsm);
            case HQ_F32: return launch_sk_t<NT, true, A8, HQ_F32>(a, st, nsm);
            case OUT_DEBUG: return launch_sk_t<NT, true, A8, OUT_DEBUG>(a, st, nsm);
        }
    }
    return HQ_ERR_UNSUPPORTED;
}

hq_status launch_gemm_small(const GemmArgs& a, int out, cudaStream_t st, int nsm) {
    if (!small_supported(a.M, a.gw)) return HQ_ERR_UNSUPPORTED;
    const bool a8 = a.act_bits == 8;
    switch (nt_for(a.M)) {
        case 8: return a8 ? launch_sk_nt<8, true>(a, out, st, nsm) : launch_sk_nt<8, false>(a, out, st, nsm);
        case 16: return a8 ? launch_sk_nt<16, true>(a, out, st, nsm) : launch_sk_nt<16, false>(a, out, st, nsm);
        case 32: return a8 ? launch_sk_nt<32, true>(a, out, st, nsm) : launch_sk_nt<32, false>(a, out, st, nsm);
        default: return a8 ? launch_sk_nt<64, true>(a, out, st, nsm) : launch_sk_nt<64, false>(a, out, st, nsm);
    }
}

}  // namespace hq
