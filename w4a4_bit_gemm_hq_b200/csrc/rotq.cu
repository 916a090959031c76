// rotq.cu -- kernel K1 on the online path: hq_rotate_quant for 16-bit
// activations whose row length is a multiple of 128.
//
// Source: "OffQ: Taming Structured Outliers in LLM Quantization by
// Offsetting", Methodology 2 (rotation by a Hadamard matrix whose first row is
// all ones turns an outlier concentrated in one channel into a constant offset
// over the group) and Methodology 3 (the rotation applied group-wise); "SERQ:
// Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization", technical
// summary section 1 (4-bit activations, the outliers set the step size).
//
// Per row m and group b of g channels:  u = (x_b .* d) * H_sylv  (fp32
// butterfly, stages h = 1, 2, 4, ... ascending, (a, b) -> (a + b, a - b)),
// amax = max |u| over the row, q = rint(fl32(u * fl32(7 / amax))) packed two
// per byte, sx[m] = fl32(fl32(amax / 7) * fl32(1 / sqrt(g))).
//
// Design (one CTA per SM, 12 warps, persistent over a contiguous block of rows):
//  * thread i of a row owns the 128 consecutive channels [128 i, 128 i + 128)
//    ("unit" i), so every butterfly stage with h < 128 runs in its registers
//    (packed f32x2 adds); groups larger than 128 take their remaining stages
//    across the lanes of one warp (shuffles; an f32x2 fma with a +-1 factor
//    forms a + b in the lower and a - b in the upper lane).
//  * the threads of one row form a "team" (ceil(K / 4096) warps).  Each team
//    owns two row slots in shared memory; its leader thread loads rows into
//    them with the tensor memory accelerator, one 4D tensor-map copy per row,
//    one row ahead of the row being rotated, so several rows per SM are in
//    flight from HBM at all times.
//  * the copy lays a row out as 128-byte lines ordered (half, unit) with the
//    128-byte swizzle: thread i reads line (h * K/128 + i), 16-byte chunk c at
//    chunk c ^ (line & 7), so the 8 threads of each shared-memory phase hit 8
//    different bank groups and each chunk lands in a fixed register.
//  * the sign vector d is expanded once per CTA into a small shared table of
//    per-element sign words that the 16-bit -> fp32 conversion adds in
//    (flipping bit 31 is adding 2^31 modulo 2^32).
//  * the row maximum is a 3-input absolute max per thread, a warp shuffle
//    reduction and, for teams of several warps, one named barrier per row.
//  * codes: fl32(u * inv) is rounded by its own multiply, then the add of
//    1.5 * 2^23 + 8 rounds it to an integer with ties to even and leaves 8 + q
//    in the low nibble of the sum's bits (no borrow for q in [-7, 7]); two such
//    nibbles form a byte with one integer multiply-add, four bytes a word with
//    a byte permute, and xor 0x88 turns offset-8 nibbles into two's complement.
//  * OffQ mode (ASYM, groups of 128): a thread's 128 channels are one group,
//    so its scale and zero point come from its own registers (3-input
//    min / max), and the codes follow the per-group sequence
//    q = clamp(rint(fl32(u * inv)) + z, 0, 15) in fp32, as the per-row kernel.
//  * every wait on a row slot is bounded; on timeout the status word records
//    HQ_ERR_TIMEOUT, the team stops, and the leader waits (bounded) for its
//    copies in flight before the CTA exits.
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "hq_device.cuh"

namespace hq {

namespace rq {
constexpr int UNIT = 128;                 // channels per thread
constexpr int WARPS = 12;
constexpr int THREADS = WARPS * 32;
constexpr int DEPTH = 2;                  // row slots per team
constexpr int MASK_STRIDE = 528;          // bytes per sign pattern (512 + 16: patterns start in different banks)
constexpr int SMEM_BUDGET = 227 * 1024;
constexpr int XT_F16 = 0, XT_BF16 = 1;
}  // namespace rq

__device__ __forceinline__ void tma_load_4d(uint32_t dst_smem, const void* tmap, int c0, int c1, int c2, int c3,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128f(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
    return v;
}

// Packed f32x2 arithmetic (sm_100): each lane is an IEEE round-to-nearest-
// even add (or fma) like __fadd_rn (__fmaf_rn).
__device__ __forceinline__ float2 rq_add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a * b + c with one rounding; with b = +-1 this is exactly c + a or c - a
__device__ __forceinline__ float2 rq_fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
// a - b, as fma(b, -1, a): the product is exact, so this is the one rounding
// of the exact difference (a plain packed add of a negated operand would
// first negate both lanes with separate instructions)
__device__ __forceinline__ float2 rq_sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }

// min(a, b, c), max(a, b, c)
__device__ __forceinline__ float rq_min3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float rq_max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max(|a|, |b|, |c|)
__device__ __forceinline__ float rq_max3abs(float a, float b, float c) {
    float r;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Shared-memory layout of one CTA (offsets from the 1024-byte aligned base).
struct RqLayout {
    uint32_t slot;    // bytes per row slot (K * 2 rounded up to 1024)
    uint32_t ring;    // teams * DEPTH * slot
    uint32_t masks;   // offset of the sign table
    uint32_t red;     // [16 teams][4 warps][2 parities] floats
    uint32_t flags;   // [16] abort flags
    uint32_t bars;    // [teams * DEPTH] mbarriers
    uint32_t bytes;   // total, excluding the alignment slack
};

__host__ __device__ inline RqLayout rq_layout(int K, int teams, int npat) {
    RqLayout L;
    L.slot = (static_cast<uint32_t>(K) * 2u + 1023u) / 1024u * 1024u;
    L.ring = static_cast<uint32_t>(teams) * rq::DEPTH * L.slot;
    L.masks = L.ring;
    L.red = L.masks + (static_cast<uint32_t>(npat) * rq::MASK_STRIDE + 15u) / 16u * 16u;
    L.flags = L.red + 16 * 4 * 2 * 4;
    L.bars = L.flags + 16 * 4;
    L.bytes = L.bars + static_cast<uint32_t>(teams) * rq::DEPTH * 8u;
    return L;
}

// G: Hadamard group; XT: 16-bit input type; SIGNED: d given (else d = 1);
// Q8: 8-bit codes in [-127, 127], one per byte (the W4A8 activations), else
// 4-bit codes in [-7, 7], two per byte; ASYM: OffQ codes in [0, 15] with a
// scale sx [M][K/128] and zero point zx [M][K/128] per group (G = 128).
template <int G, int XT, bool SIGNED, bool Q8, bool ASYM = false>
__global__ void __launch_bounds__(rq::THREADS, 1)
    k_rotq(const __grid_constant__ CUtensorMap tmX, const int8_t* __restrict__ dsign, int M, int K,
           uint8_t* __restrict__ Xq, float* __restrict__ sx, float cg, int team_warps, int teams,
           uint64_t limit_ns, int32_t* __restrict__ zx) {
    static_assert(!ASYM || (G == rq::UNIT && !Q8), "OffQ codes: 4-bit, one group of 128 per thread");
    constexpr int T = G > rq::UNIT ? G / rq::UNIT : 1;   // threads per group
    constexpr int HREG = G < rq::UNIT ? G : rq::UNIT;   // in-register stages: h < HREG
    static_assert(T <= 32, "a group spans at most one warp");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    // a kernel launched after this one with programmatic stream serialization
    // (the small-M GEMM) may start now: it waits for this grid's completion
    // before it reads the activation codes
    asm volatile("griddepcontrol.launch_dependents;");

    const RqLayout L = rq_layout(K, teams, T);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NU = K / rq::UNIT;
    const int team = warp / team_warps;
    const bool in_team = team < teams;
    const int wt = warp - team * team_warps;   // warp within the team
    const int u = wt * 32 + lane;              // unit of this thread
    const bool act = in_team && u < NU;
    const bool leader = in_team && wt == 0 && lane == 0;
    const uint32_t base = smem_u32(smem);
    const uint32_t bar0 = base + L.bars;
    float* red = reinterpret_cast<float*>(smem + L.red);
    volatile uint32_t* flags = reinterpret_cast<volatile uint32_t*>(smem + L.flags);

    if (threadIdx.x == 0) {
        for (int i = 0; i < teams * rq::DEPTH; ++i) mbar_init(bar0 + 8u * i, 1);
        for (int i = 0; i < 16; ++i) flags[i] = 0u;
        fence_mbar_init();
    }
    if constexpr (SIGNED) {
        // d[0] must be +1 (the first row of H all ones); the rotation still
        // uses the given d, and the status word reports the violation
        if (blockIdx.x == 0 && threadIdx.x == 0 && dsign[0] == -1) record_status(HQ_ERR_ARG);
        // sign table: pattern p covers channels 128 p + c (c < 128) of a group
        // (for groups up to 128 channels, d[c mod G]); bf16 entries are two
        // words per element pair (bit 31 = sign of the even element, bit 31 =
        // sign of the odd element), f16 entries one word (bits 15 and 31)
        for (int i = threadIdx.x; i < T * 64; i += blockDim.x) {
            const int p = i / 64, j = i % 64;
            const int c0 = (p * rq::UNIT + 2 * j) % G, c1 = (p * rq::UNIT + 2 * j + 1) % G;
            const uint32_t s0 = dsign[c0] == -1 ? 1u : 0u, s1 = dsign[c1] == -1 ? 1u : 0u;
            uint8_t* tp = smem + L.masks + p * rq::MASK_STRIDE;
            if constexpr (XT == rq::XT_BF16) {
                reinterpret_cast<uint32_t*>(tp)[2 * j] = s0 << 31;
                reinterpret_cast<uint32_t*>(tp)[2 * j + 1] = s1 << 31;
            } else {
                reinterpret_cast<uint32_t*>(tp)[j] = (s0 << 15) | (s1 << 31);
            }
        }
    }
    __syncthreads();

    // this CTA's rows [r0, r1); team t takes rows r0 + t + teams * k
    const int r0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * M / gridDim.x);
    const int r1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * M / gridDim.x);
    const int nrows = (in_team && r0 + team < r1) ? (r1 - r0 - team - 1) / teams + 1 : 0;
    const uint32_t ring = base + static_cast<uint32_t>(team) * rq::DEPTH * L.slot;
    const uint32_t mbase = base + L.masks + static_cast<uint32_t>(T > 1 ? (u % T) : 0) * rq::MASK_STRIDE;
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
    auto issue = [&](int k) {
        const int s = k % rq::DEPTH;
        const uint32_t b = bar0 + 8u * static_cast<uint32_t>(team * rq::DEPTH + s);
        mbar_arrive_expect_tx(b, row_bytes);
        tma_load_4d(ring + s * L.slot, &tmX, 0, 0, 0, r0 + team + teams * k, b);
    };
    int issued = 0;
    if (leader) {
        prefetch_tmap(&tmX);
        for (; issued < rq::DEPTH && issued < nrows; ++issued) issue(issued);
    }
    // 1.5 * 2^23 (+ 8 for 4-bit codes: 8 + q then sits in the low nibble)
    const float2 mg = Q8 ? make_float2(12582912.0f, 12582912.0f) : make_float2(12582920.0f, 12582920.0f);
    constexpr float LEVELS = Q8 ? 127.0f : 7.0f;
    int k = 0;
    for (; k < nrows; ++k) {
        const int m = r0 + team + teams * k;
        const int s = k % rq::DEPTH;
        const uint32_t b = bar0 + 8u * static_cast<uint32_t>(team * rq::DEPTH + s);
        const bool got = mbar_wait(b, static_cast<uint32_t>(k / rq::DEPTH) & 1u, limit_ns);
        if (!got) flags[team] = 1u;

        // ---- load the thread's 128 channels, apply d, widen to fp32
        float2 v[64];
        if (got && act) {
            const uint32_t slot = ring + s * L.slot;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t line = static_cast<uint32_t>(h * NU + u);
                const uint32_t la = slot + line * 128u, sw = line & 7u;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 w = lds128(la + ((static_cast<uint32_t>(c) ^ sw) << 4));
                    const int j0 = 32 * h + 4 * c;   // first element pair of the chunk
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                    if constexpr (XT == rq::XT_BF16) {
                        uint32_t mk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                        if constexpr (SIGNED) {
                            const uint4 ma = lds128(mbase + 8u * j0), mb = lds128(mbase + 8u * j0 + 16u);
                            mk[0] = ma.x; mk[1] = ma.y; mk[2] = ma.z; mk[3] = ma.w;
                            mk[4] = mb.x; mk[5] = mb.y; mk[6] = mb.z; mk[7] = mb.w;
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            v[j0 + e].x = __uint_as_float(wv[e] * 65536u + mk[2 * e]);   // one integer multiply-add
                            v[j0 + e].y = __uint_as_float((wv[e] & 0xFFFF0000u) ^ mk[2 * e + 1]);
                        }
                    } else {
                        uint32_t mk[4] = {0u, 0u, 0u, 0u};
                        if constexpr (SIGNED) {
                            const uint4 ma = lds128(mbase + 4u * j0);
                            mk[0] = ma.x; mk[1] = ma.y; mk[2] = ma.z; mk[3] = ma.w;
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t x = wv[e] ^ mk[e];
                            v[j0 + e] = __half22float2(*reinterpret_cast<const __half2*>(&x));
                        }
                    }
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = make_float2(0.f, 0.f);
        }
        if (T < 32 && team_warps == 1) {
            // the team is this warp: every lane has read the slot, refill it now
            __syncwarp();
            if (leader && issued < nrows && !flags[team]) issue(issued++);
        }

        // ---- butterfly stages h < 128 in registers, ascending
        if constexpr (HREG > 1) {
#pragma unroll
            for (int j = 0; j < 64; ++j) {   // h = 1: inside each pair
                const float a = v[j].x, bb = v[j].y;
                v[j].x = __fadd_rn(a, bb);
                v[j].y = __fsub_rn(a, bb);
            }
        }
#pragma unroll
        for (int h = 2; h < HREG; h <<= 1) {
#pragma unroll
            for (int i = 0; i < rq::UNIT; i += 2) {
                if ((i & h) == 0) {
                    const float2 a = v[i / 2], bb = v[(i + h) / 2];
                    v[i / 2] = rq_add2(a, bb);
                    v[(i + h) / 2] = rq_sub2(a, bb);
                }
            }
        }
        // ---- stages h >= 128
        // groups of 4096 (one warp each): two transposes through this warp's part
        // of the row slot (8 KB, free once read) leave lane l with channels
        // 128 a + 4 l + {0..3} of the group for a = 0..31; the five remaining
        // stages pair a with a ^ (h / 128) in registers.  wq[p][a] holds
        // channels 128 a + 4 l + 2 p + {0, 1}.
        float2 wq[T == 32 ? 2 : 1][T == 32 ? 32 : 1];
        if constexpr (T == 32) {
            const uint32_t slot = ring + s * L.slot;
            const uint32_t p0 = slot + static_cast<uint32_t>(wt * 32) * 128u;          // half-0 lines of the warp's units
            const uint32_t p1 = slot + static_cast<uint32_t>(NU + wt * 32) * 128u;     // half-1 lines
#pragma unroll
            for (int ph = 0; ph < 2; ++ph) {
                // lane l writes row l (256 bytes): channels 4 k + 2 ph + {0, 1}, k = 0..31,
                // 16-byte chunk q stored at q ^ (l & 7)
                const uint32_t rw = lane < 16 ? p0 + 256u * lane : p1 + 256u * (lane - 16);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float2 a = v[4 * q + ph], bb = v[4 * q + 2 + ph];
                    sts128f(rw + ((static_cast<uint32_t>(q) ^ (lane & 7u)) << 4), a.x, a.y, bb.x, bb.y);
                }
                __syncwarp();
#pragma unroll
                for (int a = 0; a < 32; ++a) {
                    const uint32_t ra = a < 16 ? p0 + 256u * a : p1 + 256u * (a - 16);
                    wq[ph][a] = lds64f(ra + (((static_cast<uint32_t>(lane) >> 1) ^ (a & 7u)) << 4) + (lane & 1u) * 8u);
                }
                __syncwarp();
            }
            // the slot has been read and rewritten by this warp's generic stores:
            // order them before the next row's copy into it
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (team_warps == 1 && leader && issued < nrows && !flags[team]) issue(issued++);
#pragma unroll
            for (int sb = 1; sb < 32; sb <<= 1) {
#pragma unroll
                for (int ph = 0; ph < 2; ++ph)
#pragma unroll
                    for (int a = 0; a < 32; ++a)
                        if ((a & sb) == 0) {
                            const float2 x0 = wq[ph][a], x1 = wq[ph][a + sb];
                            wq[ph][a] = rq_add2(x0, x1);
                            wq[ph][a + sb] = rq_sub2(x0, x1);
                        }
            }
        } else {
            // partner lane (unit) u ^ (h / 128) of the same warp
#pragma unroll
            for (int sft = 1; sft < T; sft <<= 1) {
                const float sg = (lane & sft) ? -1.0f : 1.0f;
                const float2 sg2 = make_float2(sg, sg);
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    float2 p;
                    p.x = __shfl_xor_sync(0xFFFFFFFFu, v[j].x, sft);
                    p.y = __shfl_xor_sync(0xFFFFFFFFu, v[j].y, sft);
                    // lower lane: own + partner = a + b; upper lane: partner - own = a - b
                    v[j] = rq_fma2(v[j], sg2, p);
                }
            }
        }

        // ---- row absmax
        float am[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (ASYM) {
            // per-group ranges below; the team still meets once per row
        } else if constexpr (T == 32) {
#pragma unroll
            for (int ph = 0; ph < 2; ++ph)
#pragma unroll
                for (int a = 0; a < 32; ++a) am[a & 3] = rq_max3abs(am[a & 3], wq[ph][a].x, wq[ph][a].y);
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) am[j & 3] = rq_max3abs(am[j & 3], v[j].x, v[j].y);
        }
        float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        bool abort_now;
        if (team_warps > 1) {
            float* rt = red + (team * 4) * 2;
            if (lane == 0) rt[wt * 2 + (k & 1)] = amax;
            named_bar_sync(1u + static_cast<uint32_t>(team), static_cast<uint32_t>(team_warps) * 32u);
            amax = 0.f;
            for (int w = 0; w < team_warps; ++w) amax = fmaxf(amax, rt[w * 2 + (k & 1)]);
            abort_now = flags[team] != 0u;
            // every thread of the team has read the slot: refill it
            if (leader && !abort_now && issued < nrows) issue(issued++);
        } else {
            abort_now = __any_sync(0xFFFFFFFFu, flags[team] != 0u);
        }
        if (abort_now) break;

        // ---- scale, round half to even, pack, store
        const float inv = amax == 0.f ? 0.f : __fdiv_rn(LEVELS, amax);   // amax == 0: every code is 0
        if constexpr (ASYM) {
            if (act) {
                float lo4[4], hi4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) lo4[i] = hi4[i] = v[i].x;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    lo4[j & 3] = rq_min3(lo4[j & 3], v[j].x, v[j].y);
                    hi4[j & 3] = rq_max3(hi4[j & 3], v[j].x, v[j].y);
                }
                const float lo = fminf(fminf(lo4[0], lo4[1]), fminf(lo4[2], lo4[3]));
                const float hi = fmaxf(fmaxf(hi4[0], hi4[1]), fmaxf(hi4[2], hi4[3]));
                float dlt = __fsub_rn(hi, lo);
                if (dlt == 0.f) dlt = lo != 0.f ? fabsf(lo) : 15.f;   // a constant group
                const float ginv = __fdiv_rn(15.f, dlt);
                const float zf = rintf(__fmul_rn(-lo, ginv));        // not clamped
                uint4* dst = reinterpret_cast<uint4*>(Xq + static_cast<int64_t>(m) * (K / 2) + 64 * u);
                // every |fl32(u * ginv)| is at most fl32(max(|lo|, |hi|) * ginv) (rounding is
                // monotone); below 2^22, adding 1.5 * 2^23 rounds it to an integer with ties
                // to even (= rint), adding z is then exact, and the code sits in the low
                // nibble of the sum's bits.  rint(fl32(u ginv)) + z >= rint(fl32(lo ginv)) + z
                // = 0 (rint is odd), so only the upper clamp is needed.  Larger ratios
                // (a tiny spread on a large offset) take the plain sequence.
                if (__fmul_rn(fmaxf(fabsf(lo), fabsf(hi)), ginv) < 4194304.0f) {
                    const float2 zz = make_float2(zf, zf);
                    constexpr float TOP = 12582912.0f + 15.0f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t words[4];
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            uint32_t P[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 x = v[16 * q + 4 * w + e];
                                float2 r = rq_add2(make_float2(__fmul_rn(x.x, ginv), __fmul_rn(x.y, ginv)),
                                                   make_float2(12582912.0f, 12582912.0f));
                                r = rq_add2(r, zz);
                                r.x = fminf(r.x, TOP);
                                r.y = fminf(r.y, TOP);
                                P[e] = (__float_as_uint(r.y) << 4) + __float_as_uint(r.x);   // byte e (low 16 bits)
                            }
                            const uint32_t q01 = (P[1] << 8) + P[0], q23 = (P[3] << 8) + P[2];
                            words[w] = __byte_perm(q01, q23, 0x5410);
                        }
                        dst[q] = make_uint4(words[0], words[1], words[2], words[3]);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t words[4];
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            uint32_t wd = 0;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 x = v[16 * q + 4 * w + e];
                                const float q0 = fminf(fmaxf(__fadd_rn(rintf(__fmul_rn(x.x, ginv)), zf), 0.f), 15.f);
                                const float q1 = fminf(fmaxf(__fadd_rn(rintf(__fmul_rn(x.y, ginv)), zf), 0.f), 15.f);
                                wd |= (static_cast<uint32_t>(q0) | (static_cast<uint32_t>(q1) << 4)) << (8 * e);
                            }
                            words[w] = wd;
                        }
                        dst[q] = make_uint4(words[0], words[1], words[2], words[3]);
                    }
                }
                const int64_t gi = static_cast<int64_t>(m) * (K / rq::UNIT) + u;
                sx[gi] = __fmul_rn(__fdiv_rn(dlt, 15.f), cg);
                zx[gi] = static_cast<int32_t>(zf);
            }
        } else if constexpr (Q8) {
            // the low byte of fl32(fl32(u * inv) + 1.5 * 2^23) is q in two's complement
            auto b4 = [&](float2 x0, float2 x1) {
                const float2 r0 = rq_add2(make_float2(__fmul_rn(x0.x, inv), __fmul_rn(x0.y, inv)), mg);
                const float2 r1 = rq_add2(make_float2(__fmul_rn(x1.x, inv), __fmul_rn(x1.y, inv)), mg);
                return __byte_perm(__byte_perm(__float_as_uint(r0.x), __float_as_uint(r0.y), 0x0040),
                                   __byte_perm(__float_as_uint(r1.x), __float_as_uint(r1.y), 0x0040), 0x5410);
            };
            if (act) {
                if constexpr (T == 32) {
                    // lane l: channels 128 a + 4 l .. + 3 of the warp's group, 4 bytes per a
                    uint32_t* dst = reinterpret_cast<uint32_t*>(Xq + static_cast<int64_t>(m) * K + 4096 * wt) + lane;
#pragma unroll
                    for (int a = 0; a < 32; ++a) dst[32 * a] = b4(wq[0][a], wq[1][a]);
                } else {
                    // 128 bytes per thread, 16 at a time
                    uint4* dst = reinterpret_cast<uint4*>(Xq + static_cast<int64_t>(m) * K + 128 * u);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_uint4(b4(v[8 * q], v[8 * q + 1]), b4(v[8 * q + 2], v[8 * q + 3]),
                                            b4(v[8 * q + 4], v[8 * q + 5]), b4(v[8 * q + 6], v[8 * q + 7]));
                }
            }
        } else if constexpr (T == 32) {
            // lane l: 2 bytes (channels 128 a + 4 l .. + 3) per a, 64 contiguous bytes per warp store
            if (act) {
                uint16_t* dst = reinterpret_cast<uint16_t*>(Xq + static_cast<int64_t>(m) * (K / 2) + 2048 * wt) + lane;
#pragma unroll
                for (int a = 0; a < 32; ++a) {
                    const float2 x0 = wq[0][a], x1 = wq[1][a];
                    const float2 r0 = rq_add2(make_float2(__fmul_rn(x0.x, inv), __fmul_rn(x0.y, inv)), mg);
                    const float2 r1 = rq_add2(make_float2(__fmul_rn(x1.x, inv), __fmul_rn(x1.y, inv)), mg);
                    const uint32_t b0 = (__float_as_uint(r0.y) << 4) + __float_as_uint(r0.x);
                    const uint32_t b1 = (__float_as_uint(r1.y) << 4) + __float_as_uint(r1.x);
                    dst[32 * a] = static_cast<uint16_t>(((b1 << 8) + b0) ^ 0x8888u);
                }
            }
        } else {
            // 64 bytes per thread, 16 at a time
            if (act) {
                uint4* dst = reinterpret_cast<uint4*>(Xq + static_cast<int64_t>(m) * (K / 2) + 64 * u);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t words[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t P[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            // scalar __fmul_rn: the product is rounded before the rounding
                            // add (a packed f32x2 multiply here was contracted with the
                            // add into one fused operation, which rounds exact ties the
                            // other way)
                            const float2 x = v[16 * q + 4 * w + e];
                            const float2 r = rq_add2(make_float2(__fmul_rn(x.x, inv), __fmul_rn(x.y, inv)), mg);
                            P[e] = (__float_as_uint(r.y) << 4) + __float_as_uint(r.x);   // byte e (low 16 bits)
                        }
                        const uint32_t q01 = (P[1] << 8) + P[0], q23 = (P[3] << 8) + P[2];
                        words[w] = __byte_perm(q01, q23, 0x5410) ^ 0x88888888u;
                    }
                    dst[q] = make_uint4(words[0], words[1], words[2], words[3]);
                }
            }
        }
        if (!ASYM && leader) sx[m] = (amax == 0.f) ? 0.f : __fmul_rn(__fdiv_rn(amax, LEVELS), cg);
    }
    // no copy may still be landing when the CTA exits (immediate unless a
    // wait gave up): the rows issued but not consumed
    if (leader) {
        for (int i = k; i < issued; ++i) {
            const uint32_t b = bar0 + 8u * static_cast<uint32_t>(team * rq::DEPTH + i % rq::DEPTH);
            mbar_wait(b, static_cast<uint32_t>(i / rq::DEPTH) & 1u, limit_ns);
        }
    }
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 rq_encode_tiled() {
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

struct RqPlan {
    int team_warps, teams, grid, smem;
};

static bool rq_plan(int64_t M, int64_t K, int group, int nsm, RqPlan* p) {
    if (K % rq::UNIT != 0 || K / rq::UNIT > 128) return false;   // teams of at most 4 warps
    const int NU = static_cast<int>(K / rq::UNIT);
    p->team_warps = (NU + 31) / 32;
    if (p->team_warps > rq::WARPS) return false;
    const int npat = group > rq::UNIT ? group / rq::UNIT : 1;
    int teams = rq::WARPS / p->team_warps;
    while (teams > 0 && static_cast<int>(rq_layout(static_cast<int>(K), teams, npat).bytes) + 1024 > rq::SMEM_BUDGET)
        --teams;
    if (teams == 0) return false;
    p->teams = teams;
    p->smem = static_cast<int>(rq_layout(static_cast<int>(K), teams, npat).bytes) + 1024;
    p->grid = static_cast<int>(M < nsm ? M : nsm);
    return true;
}

// Rows of up to 64 tokens (decode) keep the per-row latency of k_rotate,
// which spreads one row over K/32 threads; the streaming kernel is for
// batches that fill the device.
bool rotq_supported(int64_t M, int64_t K, int group) {
    if (M <= 64) return false;
    RqPlan p;
    return rq_plan(M, K, group, 148, &p);
}

template <int G, int XT, bool SIGNED, bool Q8, bool ASYM = false>
static hq_status launch_rotq_t(const CUtensorMap& tm, const RqPlan& p, const int8_t* d, int M, int K, uint8_t* Xq,
                               float* sx, float cg, uint64_t limit_ns, cudaStream_t st, int32_t* zx = nullptr) {
    auto kern = k_rotq<G, XT, SIGNED, Q8, ASYM>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem) != cudaSuccess)
        return HQ_ERR_CUDA;
    kern<<<p.grid, rq::THREADS, p.smem, st>>>(tm, d, M, K, Xq, sx, cg, p.team_warps, p.teams, limit_ns, zx);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

template <int XT, bool SIGNED, bool Q8>
static hq_status launch_rotq_g(int group, const CUtensorMap& tm, const RqPlan& p, const int8_t* d, int M, int K,
                               uint8_t* Xq, float* sx, float cg, uint64_t limit_ns, cudaStream_t st) {
    switch (group) {
        case 8: return launch_rotq_t<8, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 16: return launch_rotq_t<16, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 32: return launch_rotq_t<32, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 64: return launch_rotq_t<64, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 128: return launch_rotq_t<128, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 256: return launch_rotq_t<256, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 512: return launch_rotq_t<512, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 1024: return launch_rotq_t<1024, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 2048: return launch_rotq_t<2048, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        case 4096: return launch_rotq_t<4096, XT, SIGNED, Q8>(tm, p, d, M, K, Xq, sx, cg, limit_ns, st);
        default: return HQ_ERR_UNSUPPORTED;
    }
}

// Caller has validated the arguments (16-bit type, power-of-two group in
// [8, 4096] dividing K, 16-byte aligned X and Xq, ld_x * 2 a multiple of 16,
// M > 0) and checked rotq_supported().  bits: 4 (packed nibbles, Xq [M][K/2])
// or 8 (one code per byte, Xq [M][K]); zx non-null: OffQ codes (bits 4,
// group 128), sx and zx [M][K/128].
hq_status launch_rotate_quant_stream(int xt, int group, const void* X, int64_t M, int64_t K, int64_t ldx,
                                     const int8_t* d, uint8_t* Xq, float* sx, cudaStream_t st,
                                     uint64_t limit_ns, int bits, int32_t* zx) {
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return HQ_ERR_CUDA;
    RqPlan p;
    if (!rq_plan(M, K, group, nsm, &p)) return HQ_ERR_UNSUPPORTED;
    if (M > (1ll << 31) - 1) return HQ_ERR_UNSUPPORTED;
    const auto encode = rq_encode_tiled();
    if (!encode) return HQ_ERR_CUDA;
    // X viewed as [M][2 halves][K/128 units][64 channels]: one row is one box,
    // laid out in shared memory as 128-byte lines ordered (half, unit)
    CUtensorMap tm;
    const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(K / rq::UNIT), 2, static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[3] = {256, 128, static_cast<cuuint64_t>(ldx) * 2};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(K / rq::UNIT), 2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = encode(&tm, xt == HQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                              4, const_cast<void*>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return HQ_ERR_CUDA;
    const float cg = static_cast<float>(1.0 / __builtin_sqrt(static_cast<double>(group)));
    const int Mi = static_cast<int>(M), Ki = static_cast<int>(K);
    if (zx) {
        if (bits != 4 || group != rq::UNIT) return HQ_ERR_UNSUPPORTED;
        if (xt == HQ_BF16)
            return d ? launch_rotq_t<128, rq::XT_BF16, true, false, true>(tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st, zx)
                     : launch_rotq_t<128, rq::XT_BF16, false, false, true>(tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st, zx);
        return d ? launch_rotq_t<128, rq::XT_F16, true, false, true>(tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st, zx)
                 : launch_rotq_t<128, rq::XT_F16, false, false, true>(tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st, zx);
    }
    if (bits == 8) {
        if (xt == HQ_BF16)
            return d ? launch_rotq_g<rq::XT_BF16, true, true>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st)
                     : launch_rotq_g<rq::XT_BF16, false, true>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st);
        return d ? launch_rotq_g<rq::XT_F16, true, true>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st)
                 : launch_rotq_g<rq::XT_F16, false, true>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st);
    }
    if (xt == HQ_BF16)
        return d ? launch_rotq_g<rq::XT_BF16, true, false>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st)
                 : launch_rotq_g<rq::XT_BF16, false, false>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st);
    return d ? launch_rotq_g<rq::XT_F16, true, false>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st)
             : launch_rotq_g<rq::XT_F16, false, false>(group, tm, p, d, Mi, Ki, Xq, sx, cg, limit_ns, st);
}

}  // namespace hq
