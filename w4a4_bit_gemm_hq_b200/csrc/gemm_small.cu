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
// Design:
//  * operand roles swapped: the MMA's M side (128 TMEM lanes) is 128 weight
//    rows, its N side is the NT (16, 32 or 64) padded tokens, so the tensor
//    core does no wasted work on padding rows of a 128-row activation tile.
//  * stream-K: the (weight-row tile, super-block of 4 K-blocks = 512 inputs)
//    units are split into equal contiguous ranges, one per CTA, so every SM
//    streams the same number of weight bytes whatever N is.  A tile split between CTAs is finished by the
//    last CTA to arrive (an atomic counter per tile in the caller's workspace),
//    which sums the partial results in a fixed order, so the output does not
//    depend on arrival order; it resets the counter for the next call.
//  * two sets of 4 producer warps take alternate K-blocks; each thread owns one
//    weight row of the tile and streams its 64-byte pieces (contiguous 8 KB
//    tile blocks in the tile-major weight layout) into a shared-memory ring with
//    16-byte cp.async copies, 8 K-blocks ahead per set (128 KB in flight per
//    SM: many independent requests, where one bulk-copy issuer per SM could
//    not keep enough bytes in flight).  It expands each row to int8 in
//    registers and writes it straight into tensor memory with tcgen05.st, where
//    the MMA reads its A operand (no shared-memory round trip for the unpacked
//    weights); the tokens are expanded into a 128-byte-swizzled shared tile.
//  * one thread issues tcgen05.mma (A from TMEM) into a double-buffered int32
//    accumulator with one region per weight group of the super-block; 4
//    epilogue warps drain it, scale each group by sw[b][n] (one scalar per
//    lane), and finish with sx[m] and the SERQ term.
//  * every hand-over between roles (an mbarrier round trip, a few hundred
//    cycles) covers a whole super-block, not a single 128-input K-block.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "hq_device.cuh"
#include "hq_gemm.cuh"

namespace hq {

namespace sk {
constexpr int BMW = 128;                 // weight rows per tile = MMA M
constexpr int BK = 128;                  // inputs per K-block
constexpr int PDEPTH = 8;                // K-blocks in flight per producer set
constexpr int PSLOTS = 2 * PDEPTH;       // packed-weight ring slots (128 KB)
constexpr int THREADS = 448;             // warps 0-7 stream + unpack (two sets), 8 TMEM owner, 9 MMA, 10-13 epilogue
constexpr int ALLOC_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int EPI_WARP0 = 10;
constexpr int PBYTES = BMW * 64;         // packed bytes of one weight tile block
constexpr uint32_t TMEM_COLS = 512;
constexpr int XS_WORDS = 16;             // r <= 64
constexpr int UCAP = 16;                 // units whose group scales / zero points are staged in smem
constexpr int MAXG = 4;                  // max weight groups per unit
__host__ __device__ constexpr int sb_for(int nt) { return nt == 64 ? 2 : 4; }   // K-blocks per unit
}  // namespace sk

template <int NT>
struct SkSmem {
    static constexpr int SB = sk::sb_for(NT);
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_TOK = OFF_RING + sk::PSLOTS * sk::PBYTES;        // 2 stages x SB x NT x 128 B
    static constexpr int TOK_BYTES = NT * 128;
    static constexpr int OFF_XS = OFF_TOK + 2 * SB * TOK_BYTES;               // NT x 16 words
    static constexpr int OFF_SAL = OFF_XS + NT * sk::XS_WORDS * 4;            // 64 int32
    static constexpr int OFF_SS = OFF_SAL + 64 * 4;                           // UCAP x MAXG x 128 fp16 scales
    static constexpr int OFF_ZS = OFF_SS + sk::UCAP * sk::MAXG * sk::BMW * 2; // same, zero points
    static constexpr int OFF_BAR = OFF_ZS + sk::UCAP * sk::MAXG * sk::BMW * 2;
    static constexpr int NBAR = 10;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;                       // tmem base, abort, last flag
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
};

struct SkPlan {
    int ntiles;   // weight-row tiles
    int KB;       // K-blocks per row
    int sb;       // K-blocks per unit (super-block)
    int gs;       // K-blocks per weight group (1 for per-channel weights)
    int upt;      // units per tile = ceil(KB / sb)
    int units;    // ntiles * upt
    int grid;     // CTAs
    int maxc;     // max CTAs contributing to one tile
};

__host__ __device__ inline int sk_owner(int u, int units, int grid) {
    return static_cast<int>((static_cast<long long>(u + 1) * grid - 1) / units);
}
__host__ __device__ inline int sk_begin(int c, int units, int grid) {
    return static_cast<int>(static_cast<long long>(c) * units / grid);
}

static int nt_for(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

static SkPlan sk_plan(int64_t M, int64_t N, int64_t K, int gw, int nsm) {
    SkPlan p{};
    p.ntiles = static_cast<int>((N + sk::BMW - 1) / sk::BMW);
    p.KB = static_cast<int>(K / sk::BK);
    p.sb = sk::sb_for(nt_for(M));
    p.gs = gw ? gw / sk::BK : 1;
    p.upt = (p.KB + p.sb - 1) / p.sb;
    p.units = p.ntiles * p.upt;
    const int want = nsm > 0 ? nsm : 148;
    p.grid = p.units < want ? p.units : want;
    p.maxc = 1;
    for (int t = 0; t < p.ntiles; ++t) {
        const int a = sk_owner(t * p.upt, p.units, p.grid);
        const int b = sk_owner((t + 1) * p.upt - 1, p.units, p.grid);
        if (b - a + 1 > p.maxc) p.maxc = b - a + 1;
    }
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

// NT accumulator columns of one lane quarter -> registers (no wait).
template <int NT>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&v)[NT]) {
    if constexpr (NT == 16) {
        tmem_ld_32x32b_x16(taddr, v);
    } else if constexpr (NT == 32) {
        tmem_ld_32x32b_x32(taddr, v);
    } else {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
        tmem_ld_32x32b_x32(taddr, lo);
        tmem_ld_32x32b_x32(taddr + 32, hi);
    }
}

// A8: 8-bit activation codes ([M][K] int8, used as they are) instead of packed
// 4-bit codes (expanded as 16 q).
template <int NT, bool ASYM, bool A8, int OUT>
__global__ void __launch_bounds__(sk::THREADS, 1) k_gemm_small(const GemmArgs p, const SkPlan plan) {
    using L = SkSmem<NT>;
    constexpr int XROW = A8 ? 128 : 64;   // activation bytes per token row and K-block
    constexpr int SB = L::SB;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived by pointer arithmetic on the __shared__
    // array so that every access through it compiles to a shared-memory
    // instruction (a pointer rebuilt from an integer is generic)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(smem + L::OFF_BAR);
    auto fulla = [&](int s) { return bar0 + 8u * s; };          // A stage s written (producer set s)
    auto emptya = [&](int s) { return bar0 + 8u * (2 + s); };   // A stage s consumed (MMA)
    auto accf = [&](int b) { return bar0 + 8u * (4 + b); };
    auto acce = [&](int b) { return bar0 + 8u * (6 + b); };
    const uint32_t done_bar = bar0 + 8u * 8;
    const uint32_t scl_bar = bar0 + 8u * 9;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);   // [0] tmem, [1] abort, [2] last
    volatile uint32_t* abort_flag = misc + 1;
    uint32_t* xs_s = reinterpret_cast<uint32_t*>(smem + L::OFF_XS);
    int32_t* sal_s = reinterpret_cast<int32_t*>(smem + L::OFF_SAL);
    const uint16_t* ss = reinterpret_cast<const uint16_t*>(smem + L::OFF_SS);   // [unit][group][row]
    const uint16_t* zs = reinterpret_cast<const uint16_t*>(smem + L::OFF_ZS);

    const int KB = plan.KB, upt = plan.upt, gs = plan.gs;
    const int u0 = sk_begin(blockIdx.x, plan.units, plan.grid);
    const int u1 = sk_begin(blockIdx.x + 1, plan.units, plan.grid);
    const int nunits = u1 - u0;
    const int nstaged = nunits < sk::UCAP ? nunits : sk::UCAP;
    // unit geometry: tile, first K-block, K-blocks
    auto unit_tile = [&](int u) { return u / upt; };
    auto unit_kb0 = [&](int u) { return (u - (u / upt) * upt) * SB; };
    auto unit_nk = [&](int u) { const int r = KB - unit_kb0(u); return r < SB ? r : SB; };

    if (warp == sk::ALLOC_WARP) {
        if (lane == 0) {
            for (int s = 0; s < 2; ++s) {
                mbar_init(fulla(s), 128);
                mbar_init(emptya(s), 1);
                mbar_init(accf(s), 1);
                mbar_init(acce(s), 4);
            }
            mbar_init(done_bar, 1);
            mbar_init(scl_bar, 128);
            misc[1] = 0;
            fence_mbar_init();
        }
        __syncwarp();
        tmem_alloc(smem_u32(misc), sk::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const uint32_t acc_col0 = 2 * SB * 32;

    auto waitx = [&](uint32_t bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, p.limit_ns)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };

    if (warp < 8) {
        // ======================= producers: two sets of 4 warps take alternate units.
        // Each thread owns one weight row of the tile: it streams the row's
        // 64-byte pieces with cp.async, expands them to int8 and writes them into
        // its lane of the set's tensor-memory A stage; it also expands a share of
        // the unit's tokens into the set's token stage.
        const int pset = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        constexpr int TCH = (NT * (XROW / 16) + 127) / 128;   // token chunks per thread per K-block
        // write cursor (cp.async issue) over this set's K-blocks
        int wli = pset, wkbi = 0, wctr = 0;
        auto issue_next = [&]() {
            if (wli < nunits) {
                const int u = u0 + wli;
                const int64_t blk = static_cast<int64_t>(unit_tile(u)) * KB + unit_kb0(u) + wkbi;
                const int slot = pset * sk::PDEPTH + (wctr % sk::PDEPTH);
                const uint8_t* src = p.Wq + blk * sk::PBYTES + row * 64;
                const uint32_t dst = smem_u32(smem + L::OFF_RING + slot * sk::PBYTES + row * 64);
#pragma unroll
                for (int c = 0; c < 4; ++c) cp_async16(dst + 16 * c, src + 16 * c);
                if (++wkbi == unit_nk(u)) { wkbi = 0; wli += 2; }
            }
            cp_async_commit();   // one group per K-block (possibly empty)
            ++wctr;
        };
        for (int d = 0; d < sk::PDEPTH; ++d) issue_next();
        if (ASYM && nstaged > 0) __all_sync(0xFFFFFFFFu, waitx(scl_bar, 0));   // zero points staged
        asm volatile("griddepcontrol.wait;" ::: "memory");   // tokens are the preceding kernel's output
        // this thread's share of a unit's packed tokens, loaded one unit ahead
        // (an L2 round trip is several hundred ns; it must not sit in the K loop)
        auto load_unit_tokens = [&](int li, uint4 (&tk)[SB][TCH]) {
#pragma unroll
            for (int kbi = 0; kbi < SB; ++kbi)
#pragma unroll
                for (int c = 0; c < TCH; ++c) tk[kbi][c] = make_uint4(0, 0, 0, 0);
            if (li >= nunits) return;
            const int u = u0 + li;
            const int kb0 = unit_kb0(u), nk = unit_nk(u);
#pragma unroll
            for (int kbi = 0; kbi < SB; ++kbi) {
#pragma unroll
                for (int c = 0; c < TCH; ++c) {
                    const int tc = row + 128 * c;
                    const int tr = tc / (XROW / 16), ch = tc % (XROW / 16);
                    if (kbi < nk && tc < NT * (XROW / 16) && tr < p.M)
                        tk[kbi][c] = __ldg(reinterpret_cast<const uint4*>(p.Xq + static_cast<int64_t>(tr) * (A8 ? p.K : p.K / 2) +
                                                                       (kb0 + kbi) * XROW + ch * 16));
                }
            }
        };
        uint4 tk_cur[SB][TCH], tk_nxt[SB][TCH];
        load_unit_tokens(pset, tk_cur);
        int rctr = 0;
        bool ok = true;
        for (int li = pset; ok && li < nunits; li += 2) {
            const int u = u0 + li;
            const int t = unit_tile(u), kb0 = unit_kb0(u), nk = unit_nk(u);
            const int n = t * sk::BMW + row;
            const uint32_t use = static_cast<uint32_t>(li >> 1);     // use count of this set's stage
            load_unit_tokens(li + 2, tk_nxt);
            if (!__all_sync(0xFFFFFFFFu, waitx(emptya(pset), (use & 1u) ^ 1u))) break;
            tc_fence_after();
#pragma unroll
            for (int kbi = 0; kbi < SB; ++kbi) {
                if (kbi >= nk) break;
                const int kb = kb0 + kbi;
                uint32_t z4 = 0;
                if constexpr (ASYM) {
                    const int gi = kbi / gs;
                    uint32_t z = 0;
                    if (n < p.N) {
                        if (li < sk::UCAP) {
                            z = static_cast<uint32_t>(__half2float(__ushort_as_half(zs[(li * sk::MAXG + gi) * sk::BMW + row])));
                        } else {
                            const int g = (kb * sk::BK) / p.gw;
                            z = static_cast<uint32_t>(__half2float(__ushort_as_half(p.zw[static_cast<int64_t>(g) * p.N + n])));
                        }
                    }
                    z4 = z * 0x01010101u;
                }
                cp_async_wait_group<sk::PDEPTH - 1>();   // this thread's piece of the K-block has landed
                const uint8_t* src = smem + L::OFF_RING + (pset * sk::PDEPTH + (rctr % sk::PDEPTH)) * sk::PBYTES + row * 64;
                uint4 c4[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) c4[c] = *reinterpret_cast<const uint4*>(src + (c << 4));
                ++rctr;
                issue_next();                          // refill the slot just read
                uint32_t a[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t w[4] = {c4[c].x, c4[c].y, c4[c].z, c4[c].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if constexpr (ASYM) unpack_u4x8_minus_z(w[e], z4, a[8 * c + 2 * e], a[8 * c + 2 * e + 1]);
                        else unpack_s4x8_times16(w[e], a[8 * c + 2 * e], a[8 * c + 2 * e + 1]);
                        if constexpr (A8) {
                            // 8-bit activations keep their natural K order: interleave the
                            // (k0 k2 k4 k6, k1 k3 k5 k7) words back to (k0..k3, k4..k7)
                            const uint32_t lo = a[8 * c + 2 * e], hi = a[8 * c + 2 * e + 1];
                            a[8 * c + 2 * e] = __byte_perm(lo, hi, 0x5140);
                            a[8 * c + 2 * e + 1] = __byte_perm(lo, hi, 0x7362);
                        }
                    }
                }
                tmem_st_32x32b_x32(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                                       static_cast<uint32_t>((pset * SB + kbi) * 32), a);
                uint8_t* tstage = smem + L::OFF_TOK + (pset * SB + kbi) * L::TOK_BYTES;
#pragma unroll
                for (int c = 0; c < TCH; ++c) {
                    const int tc = row + 128 * c;
                    if (tc < NT * (XROW / 16)) {
                        const int tr = tc / (XROW / 16), ch = tc % (XROW / 16);
                        uint8_t* trow = tstage + tr * 128;
                        if constexpr (A8) {
                            // 16 codes as they are, into 16-byte chunk ch of the swizzled row
                            *reinterpret_cast<uint4*>(trow + ((ch ^ (tr & 7)) << 4)) = tk_cur[kbi][c];
                        } else {
                            uint32_t o[8];
                            const uint32_t w[4] = {tk_cur[kbi][c].x, tk_cur[kbi][c].y, tk_cur[kbi][c].z, tk_cur[kbi][c].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) unpack_s4x8_times16(w[e], o[2 * e], o[2 * e + 1]);
                            *reinterpret_cast<uint4*>(trow + (((2 * ch) ^ (tr & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                            *reinterpret_cast<uint4*>(trow + (((2 * ch + 1) ^ (tr & 7)) << 4)) =
                                make_uint4(o[4], o[5], o[6], o[7]);
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(fulla(pset));
#pragma unroll
            for (int kbi = 0; kbi < SB; ++kbi)
#pragma unroll
                for (int c = 0; c < TCH; ++c) tk_cur[kbi][c] = tk_nxt[kbi][c];
        }
        cp_async_wait_all();   // nothing in flight when the CTA exits
    } else if (warp == sk::MMA_WARP) {
        // ======================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_i8(sk::BMW, NT);
            int abuf = 0;
            uint32_t accph = 0;
            for (int li = 0; li < nunits; ++li) {
                const int u = u0 + li;
                const int t = unit_tile(u), nk = unit_nk(u);
                const bool seg_first = (li == 0) || unit_tile(u - 1) != t;
                const bool seg_last = (li + 1 == nunits) || unit_tile(u + 1) != t;
                const bool grp_first = ASYM || seg_first;
                const bool grp_last = ASYM || seg_last;
                if (grp_first) {
                    if (!waitx(acce(abuf), ((accph >> abuf) & 1u) ^ 1u)) break;
                }
                const int s = li & 1;
                if (!waitx(fulla(s), static_cast<uint32_t>((li >> 1) & 1))) break;
                tc_fence_after();
                const uint32_t acc = tmem_base + acc_col0 + static_cast<uint32_t>(abuf * SB * NT);
                for (int kbi = 0; kbi < nk; ++kbi) {
                    const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + L::OFF_TOK + (s * SB + kbi) * L::TOK_BYTES));
                    const uint32_t dcol = acc + (ASYM ? static_cast<uint32_t>((kbi / gs) * NT) : 0u);
                    const bool fresh = ASYM ? (kbi % gs == 0) : (seg_first && kbi == 0);
#pragma unroll
                    for (int kk = 0; kk < sk::BK / 32; ++kk)
                        mma_i8_ts(dcol, tmem_base + static_cast<uint32_t>((s * SB + kbi) * 32 + kk * 8), bdesc + 2u * kk,
                                  IDESC, (fresh && kk == 0) ? 0u : 1u);
                }
                tc_commit(emptya(s));
                if (grp_last) {
                    tc_commit(accf(abuf));
                    accph ^= 1u << abuf;
                    abuf ^= 1;
                }
            }
            tc_commit(done_bar);
            mbar_wait(done_bar, 0, p.limit_ns);
        }
        __syncwarp();
    } else if (warp >= sk::EPI_WARP0) {
        // ======================= epilogue: drain, finish or hand over
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int ethr = (warp - sk::EPI_WARP0) * 32 + lane;   // 0..127
        if constexpr (ASYM) {
            // weight-side group scales and zero points of the first UCAP units (they
            // do not depend on the preceding kernel): 16-byte async copies of the
            // 128-entry rows, all in flight together, one round trip
            uint8_t* ssw = smem + L::OFF_SS;
            uint8_t* zsw = smem + L::OFF_ZS;
            const int arrays = (OUT == OUT_DEBUG) ? 1 : 2;
            const int items = nstaged * sk::MAXG * arrays * 16;
            const int G = p.K / p.gw;
            for (int idx = ethr; idx < items; idx += 128) {
                const int c = idx % 16, a = (idx / 16) % arrays, gi = (idx / (16 * arrays)) % sk::MAXG;
                const int li = idx / (16 * arrays * sk::MAXG);
                const int u = u0 + li;
                const int g = unit_kb0(u) / gs + gi;
                const int n0 = unit_tile(u) * sk::BMW + c * 8;
                uint8_t* dst = (a == 0 ? zsw : ssw) + ((li * sk::MAXG + gi) * sk::BMW + c * 8) * 2;
                if (n0 < p.N && gi * gs < unit_nk(u) && g < G) {
                    const uint16_t* src = (a == 0 ? p.zw : p.sw) + static_cast<int64_t>(g) * p.N + n0;
                    cp_async16(smem_u32(dst), src);
                } else {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
            cp_async_commit();
            cp_async_wait_all();
            mbar_arrive(scl_bar);
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");   // sx, Xq and the outputs follow the preceding kernel
        // gathered salient activation codes of every token (needed when a tile
        // finishes): int8 words in the lo/hi order of unpack_s4x8_times16
        for (int j = ethr; j < p.r; j += 128) sal_s[j] = p.sal[j];
        named_bar_sync(1, 128);
        for (int idx = ethr; idx < NT * sk::XS_WORDS; idx += 128) {
            const int m = idx / sk::XS_WORDS, w = idx % sk::XS_WORDS;
            uint32_t word = 0;
            if (m < p.M) {
                const uint8_t* xrow = p.Xq + static_cast<int64_t>(m) * (A8 ? p.K : p.K / 2);
                const int i = w >> 1, h = w & 1;   // word 2i+h holds positions 8i+2e+h, byte e
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 8 * i + 2 * e + h;
                    if (j < p.r) {
                        const int k = sal_s[j];
                        if (static_cast<unsigned>(k) < static_cast<unsigned>(p.K)) {
                            if constexpr (A8) {
                                word |= static_cast<uint32_t>(__ldg(xrow + k)) << (8 * e);
                            } else {
                                const int nib = (__ldg(xrow + (k >> 1)) >> ((k & 1) * 4)) & 0xF;
                                word |= (static_cast<uint32_t>((nib ^ 8) - 8) & 0xFFu) << (8 * e);
                            }
                        } else {
                            record_status(HQ_ERR_ARG);   // a salient index outside [0, K): skipped
                        }
                    }
                }
            }
            xs_s[idx] = word;
        }
        named_bar_sync(1, 128);
        if (ASYM && nstaged > 0) waitx(scl_bar, 0);
        int abuf = 0;
        uint32_t accph = 0;
        uint32_t* ws_cnt = static_cast<uint32_t*>(p.ws);
        float* ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(p.ws) + small_counter_bytes(plan.ntiles));
        // the accumulators carry the factor of the activation codes (16 for
        // 4-bit codes, 1 for 8-bit) and 16 for symmetric weight codes
        const int sh = (A8 ? 0 : 4) + (ASYM ? 0 : 4);
        const int G = ASYM ? p.K / p.gw : 1;
        int li = 0;
        while (li < nunits) {
            const int t = unit_tile(u0 + li);
            int le = li + 1;
            while (le < nunits && unit_tile(u0 + le) == t) ++le;
            const int n = t * sk::BMW + row;
            const bool nvalid = n < p.N;
            // operands of the tile's finish, fetched early (their latency hides under the K loop)
            uint32_t rqp[sk::XS_WORDS / 2];
#pragma unroll
            for (int i = 0; i < sk::XS_WORDS / 2; ++i) rqp[i] = 0;
            float swn = 0.f, srn = 0.f;
            if (nvalid) {
                if (p.r > 0) {
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.Rq + static_cast<int64_t>(n) * (p.r / 2));
#pragma unroll
                    for (int i = 0; i < sk::XS_WORDS / 2; ++i)
                        if (i < p.r / 8) rqp[i] = __ldg(src + i);
                }
                if constexpr (OUT != OUT_DEBUG) {
                    if constexpr (!ASYM) swn = __half2float(__ushort_as_half(p.sw[n]));
                    if (p.r > 0) srn = __half2float(__ushort_as_half(p.sr[n]));
                }
            }
            float y[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j) y[j] = 0.f;
            const int drains = ASYM ? le - li : 1;
            for (int di = 0; di < drains; ++di) {
                waitx(accf(abuf), (accph >> abuf) & 1u);
                tc_fence_after();
                const uint32_t acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc_col0 +
                                     static_cast<uint32_t>(abuf * SB * NT);
                if constexpr (ASYM) {
                    const int uli = li + di;
                    const int uu = u0 + uli;
                    const int ng = unit_nk(uu) / gs;
                    for (int gi = 0; gi < ng; ++gi) {
                        uint32_t v[NT];
                        ld_cols<NT>(acc + static_cast<uint32_t>(gi * NT), v);
                        tmem_wait_ld();
                        const int g = unit_kb0(uu) / gs + gi;
                        float s = 0.f;   // the debug entry passes no scales
                        if constexpr (OUT != OUT_DEBUG) {
                            if (uli < sk::UCAP)
                                s = __half2float(__ushort_as_half(ss[(uli * sk::MAXG + gi) * sk::BMW + row]));
                            else if (nvalid)
                                s = __half2float(__ushort_as_half(p.sw[static_cast<int64_t>(g) * p.N + n]));
                        }
#pragma unroll
                        for (int j = 0; j < NT; ++j) {
                            const int a = static_cast<int32_t>(v[j]) >> sh;
                            if constexpr (OUT == OUT_DEBUG) {
                                if (nvalid && j < p.M) p.dbg_acc[(static_cast<int64_t>(j) * p.N + n) * G + g] = a;
                            }
                            y[j] = __fmaf_rn(s, static_cast<float>(a), y[j]);
                        }
                    }
                } else {
                    uint32_t v[NT];
                    ld_cols<NT>(acc, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < NT; ++j) y[j] = static_cast<float>(static_cast<int32_t>(v[j]) >> sh);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce(abuf));
                accph ^= 1u << abuf;
                abuf ^= 1;
            }
            const bool whole = (u0 + li == t * upt) && (u0 + le == (t + 1) * upt);
            bool finish = whole;
            if (!whole) {
                // hand the partial result over: slot = position of this CTA among the tile's contributors
                const int first = sk_owner(t * upt, plan.units, plan.grid);
                const int last = sk_owner((t + 1) * upt - 1, plan.units, plan.grid);
                const int slot = static_cast<int>(blockIdx.x) - first;
                float* part = ws_part + (static_cast<int64_t>(t) * plan.maxc + slot) * NT * sk::BMW;
#pragma unroll
                for (int j = 0; j < NT; ++j) part[j * sk::BMW + row] = y[j];
                // one thread publishes the CTA's partial (the barrier orders every
                // thread's stores before its fence) and counts the arrival; the
                // last arriver's thread fences again before the CTA reads the
                // other contributors' partials
                named_bar_sync(1, 128);
                if (ethr == 0) {
                    __threadfence();
                    const uint32_t old = atomicAdd(ws_cnt + t, 1u);
                    const bool last_one = old == static_cast<uint32_t>(last - first);
                    if (last_one) __threadfence();
                    misc[2] = last_one ? 1u : 0u;
                }
                named_bar_sync(1, 128);
                finish = misc[2] != 0;
                if (finish) {
#pragma unroll
                    for (int j = 0; j < NT; ++j) y[j] = 0.f;
                    // all contributors' partials, CB at a time in flight, summed in slot order
                    constexpr int CB = NT <= 16 ? 4 : (NT <= 32 ? 2 : 1);
                    const int nc = last - first + 1;
                    for (int c0 = 0; c0 < nc; c0 += CB) {
                        float pv[CB][NT];
#pragma unroll
                        for (int cc = 0; cc < CB; ++cc) {
                            const float* pc = ws_part + (static_cast<int64_t>(t) * plan.maxc + c0 + cc) * NT * sk::BMW;
#pragma unroll
                            for (int j = 0; j < NT; ++j) pv[cc][j] = (c0 + cc < nc) ? __ldcg(pc + j * sk::BMW + row) : 0.f;
                        }
#pragma unroll
                        for (int cc = 0; cc < CB; ++cc) {
                            if (c0 + cc < nc) {
#pragma unroll
                                for (int j = 0; j < NT; ++j) y[j] = __fadd_rn(y[j], pv[cc][j]);
                            }
                        }
                    }
                    if (ethr == 0) ws_cnt[t] = 0u;   // ready for the next call
                }
                named_bar_sync(1, 128);           // misc[2] is rewritten by the next tile
            }
            if (finish && nvalid) {
                // SERQ term: (X[m,S] . Rq[n,:]) with Rq[n] of this lane's row
                uint32_t rq[sk::XS_WORDS];
#pragma unroll
                for (int i = 0; i < sk::XS_WORDS / 2; ++i) unpack_s4x8_times16(rqp[i], rq[2 * i], rq[2 * i + 1]);
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j >= p.M) break;
                    int cc = 0;
                    if (p.r > 0) {
#pragma unroll
                        for (int i = 0; i < sk::XS_WORDS; ++i)
                            cc = __dp4a(static_cast<int>(xs_s[j * sk::XS_WORDS + i]), static_cast<int>(rq[i]), cc);
                        cc >>= 4;
                    }
                    if constexpr (OUT == OUT_DEBUG) {
                        if constexpr (!ASYM) p.dbg_acc[static_cast<int64_t>(j) * p.N + n] = static_cast<int32_t>(y[j]);
                        if (p.r > 0) p.dbg_acc_c[static_cast<int64_t>(j) * p.N + n] = cc;
                    } else {
                        const float base = ASYM ? y[j] : __fmul_rn(swn, y[j]);
                        const float v = __fmul_rn(p.sx[j], __fmaf_rn(srn, static_cast<float>(cc), base));
                        store_one<OUT>(p.Y, static_cast<int64_t>(j) * p.N + n, v);
                    }
                }
            }
            li = le;
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == sk::ALLOC_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, sk::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side
bool small_supported(int64_t M, int gw) {
    if (M < 1 || M > 64) return false;
    return gw == 0 || gw / sk::BK <= sk::sb_for(nt_for(M));
}

size_t small_workspace_bytes(int64_t M, int64_t N, int64_t K, int gw, int nsm) {
    if (!small_supported(M, gw) || N <= 0 || K < sk::BK) return 0;
    const SkPlan p = sk_plan(M, N, K, gw, nsm);
    return small_counter_bytes(p.ntiles) + static_cast<size_t>(p.ntiles) * p.maxc * nt_for(M) * sk::BMW * sizeof(float);
}

template <int NT, bool ASYM, bool A8, int OUT>
static hq_status launch_sk_t(const GemmArgs& a, const SkPlan& plan, cudaStream_t st) {
    auto kern = k_gemm_small<NT, ASYM, A8, OUT>;
    const int smem = SkSmem<NT>::ALLOC;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    // Programmatic dependent launch: the kernel may start while the preceding
    // kernel of the stream (normally the activation rotate/quant) is still
    // running; it streams weights, then waits (griddepcontrol.wait) before it
    // reads activations or writes anything.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(sk::THREADS);
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

template <int NT, bool A8>
static hq_status launch_sk_nt(const GemmArgs& a, int out, const SkPlan& plan, cudaStream_t st) {
    if (a.gw == 0) {
        switch (out) {
            case HQ_F16: return launch_sk_t<NT, false, A8, HQ_F16>(a, plan, st);
            case HQ_BF16: return launch_sk_t<NT, false, A8, HQ_BF16>(a, plan, st);
            case HQ_F32: return launch_sk_t<NT, false, A8, HQ_F32>(a, plan, st);
            case OUT_DEBUG: return launch_sk_t<NT, false, A8, OUT_DEBUG>(a, plan, st);
        }
    } else {
        switch (out) {
            case HQ_F16: return launch_sk_t<NT, true, A8, HQ_F16>(a, plan, st);
            case HQ_BF16: return launch_sk_t<NT, true, A8, HQ_BF16>(a, plan, st);
            case HQ_F32: return launch_sk_t<NT, true, A8, HQ_F32>(a, plan, st);
            case OUT_DEBUG: return launch_sk_t<NT, true, A8, OUT_DEBUG>(a, plan, st);
        }
    }
    return HQ_ERR_UNSUPPORTED;
}

hq_status launch_gemm_small(const GemmArgs& a, int out, cudaStream_t st, int nsm) {
    if (!small_supported(a.M, a.gw)) return HQ_ERR_UNSUPPORTED;
    const SkPlan plan = sk_plan(a.M, a.N, a.K, a.gw, nsm);
    const bool a8 = a.act_bits == 8;
    switch (nt_for(a.M)) {
        case 16: return a8 ? launch_sk_nt<16, true>(a, out, plan, st) : launch_sk_nt<16, false>(a, out, plan, st);
        case 32: return a8 ? launch_sk_nt<32, true>(a, out, plan, st) : launch_sk_nt<32, false>(a, out, plan, st);
        default: return a8 ? launch_sk_nt<64, true>(a, out, plan, st) : launch_sk_nt<64, false>(a, out, plan, st);
    }
}

}  // namespace hq
