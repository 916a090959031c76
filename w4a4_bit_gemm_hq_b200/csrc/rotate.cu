// rotate.cu -- kernel K1 and its relatives: the grouped Walsh-Hadamard
// rotation of activation rows with an all-ones first row of H, fused with the
// per-token absmax, round-to-nearest-even int4 quantisation and nibble packing
// ("OffQ: Taming Structured Outliers in LLM Quantization by Offsetting",
// Methodology 2-3; "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
// Quantization", technical summary section 1).  The same butterfly also serves
// the offline weight fold (normalised rotation to fp32) and the calibration
// statistic (per-channel sum of squares).
//
// Work mapping: one CTA owns one row at a time and walks rows persistently;
// thread t holds the 32 consecutive channels [32t, 32t+32) of the row in
// registers, loaded with 16-byte vector loads.  Butterfly stages with h < 32
// run in registers (packed f32x2 adds where both operands are pairs), stages
// 32 <= h < 1024 use warp shuffles, and stages h >= 1024 (groups of 2048 and
// 4096) exchange through shared memory.  Every stage is an IEEE fp32 add/sub
// of the pair (u[i], u[i+h]) in ascending h, so the codes are exactly those of
// the plain definition regardless of which thread computes a pair.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "hq_device.cuh"

namespace hq {

constexpr int EPT = 32;  // channels per thread

// QUANT8: one 8-bit code per byte; QUANT_ASYM: OffQ's per-group asymmetric
// 4-bit codes with a scale and an integer zero point per group
enum { MODE_QUANT = 0, MODE_ROTATE = 1, MODE_SQNORM = 2, MODE_QUANT8 = 3, MODE_QUANT_ASYM = 4 };
enum { XT_F16 = 0, XT_BF16 = 1, XT_F32 = 2 };

__device__ __forceinline__ float2 f2sub(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rc, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// Packed IEEE round-to-nearest multiply / add (sm_100 f32x2).
__device__ __forceinline__ float2 f2mul_rn(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rc, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 f2add_rn(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rc, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

template <int G, int XT, int MODE>
__global__ void __launch_bounds__(512) k_rotate(const void* __restrict__ X, int64_t M, int64_t K, int64_t ldx,
                                                 const int8_t* __restrict__ dsign, uint8_t* __restrict__ Xq,
                                                 float* __restrict__ sx, float* __restrict__ out, float cg,
                                                 int32_t* __restrict__ zx) {
    constexpr int TPG = (G > EPT) ? G / EPT : 1;     // threads per group
    constexpr int HREG = (G < EPT) ? G : EPT;        // in-register stages: h < HREG
    constexpr int TSHFL = (TPG < 32) ? TPG : 32;     // shuffle stages: s < TSHFL
    extern __shared__ float xch[];                   // [EPT][blockDim] exchange (G >= 2048)
    __shared__ float red[2][32];   // per-warp maxima, double-buffered by row parity

    // a kernel launched after this one with programmatic stream serialization
    // (the small-M GEMM) may start now: it waits for this grid's completion
    // before it reads the activation codes
    asm volatile("griddepcontrol.launch_dependents;");
    const int t = threadIdx.x;
    const int nthr = blockDim.x;
    const int64_t tpr = K / EPT;
    const bool active = t < tpr;
    const int64_t col0 = static_cast<int64_t>(t) * EPT;

    // Signs of d for this thread's channels: bit i set = flip channel col0 + i.
    uint32_t smask = 0;
    float accsq[MODE == MODE_SQNORM ? EPT : 1];
#pragma unroll
    for (int i = 0; i < (MODE == MODE_SQNORM ? EPT : 1); ++i) accsq[i] = 0.f;
    if (blockIdx.x == 0 && t == 0 && dsign != nullptr && dsign[0] == -1) record_status(HQ_ERR_ARG);   // d[0] must be +1
    if (active && dsign != nullptr) {
        const int p0 = static_cast<int>(col0 % G);
#pragma unroll
        for (int i = 0; i < EPT; ++i) smask |= (dsign[(p0 + i) % G] == -1 ? 1u : 0u) << i;
    }

    // raw 16-byte words of this thread's channels, loaded one row ahead so that
    // the next row's HBM latency hides under this row's butterfly
    constexpr int NRAW = (XT == XT_F32) ? EPT / 4 : EPT / 8;
    uint4 raw[NRAW], raw_next[NRAW];
    auto load_row = [&](int64_t m, uint4 (&r)[NRAW]) {
        if (active && m < M) {
            const uint4* src = (XT == XT_F32)
                                   ? reinterpret_cast<const uint4*>(static_cast<const float*>(X) + m * ldx + col0)
                                   : reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + m * ldx + col0);
#pragma unroll
            for (int j = 0; j < NRAW; ++j) r[j] = __ldg(src + j);
        }
    };
    load_row(blockIdx.x, raw);
    int par = 0;
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x, par ^= 1) {
        load_row(m + gridDim.x, raw_next);
        float2 v[EPT / 2];
        if (active) {
            if constexpr (XT == XT_F32) {
#pragma unroll
                for (int j = 0; j < EPT / 4; ++j) {
                    const uint4 f = raw[j];
                    v[2 * j].x = __uint_as_float(f.x ^ (((smask >> (4 * j)) & 1u) << 31));
                    v[2 * j].y = __uint_as_float(f.y ^ (((smask >> (4 * j + 1)) & 1u) << 31));
                    v[2 * j + 1].x = __uint_as_float(f.z ^ (((smask >> (4 * j + 2)) & 1u) << 31));
                    v[2 * j + 1].y = __uint_as_float(f.w ^ (((smask >> (4 * j + 3)) & 1u) << 31));
                }
            } else {
#pragma unroll
                for (int j = 0; j < EPT / 8; ++j) {
                    const uint4 q = raw[j];
                    uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i0 = 8 * j + 2 * e;   // channel of the pair's low half
                        const uint32_t x = w[e] ^ (((smask >> i0) & 1u) << 15) ^ (((smask >> (i0 + 1)) & 1u) << 31);
                        if constexpr (XT == XT_BF16) {
                            v[4 * j + e].x = __uint_as_float(x << 16);
                            v[4 * j + e].y = __uint_as_float(x & 0xFFFF0000u);
                        } else {
                            __half2 h2 = *reinterpret_cast<const __half2*>(&x);
                            v[4 * j + e] = __half22float2(h2);
                        }
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < EPT / 2; ++i) v[i] = make_float2(0.f, 0.f);
        }

        // ---- in-register stages, ascending h
        if constexpr (HREG > 1) {
#pragma unroll
            for (int i = 0; i < EPT / 2; ++i) {  // h = 1: inside each pair
                const float a = v[i].x, b = v[i].y;
                v[i].x = __fadd_rn(a, b);
                v[i].y = __fsub_rn(a, b);
            }
        }
#pragma unroll
        for (int h = 2; h < HREG; h <<= 1) {
#pragma unroll
            for (int i = 0; i < EPT; i += 2) {
                if ((i & h) == 0) {
                    const float2 a = v[i / 2], b = v[(i + h) / 2];
                    v[i / 2] = f2add_rn(a, b);
                    v[(i + h) / 2] = f2sub(a, b);
                }
            }
        }
        if constexpr (G == 4096) {
            // ---- groups of 4096 (128 threads each): the remaining 7 stages run
            // in registers between two shared-memory transposes.
            // Channel i of the group = 1024 ah + 32 al + b.  So far thread
            // (warp ah, lane al) holds b = 0..31.
            const int tg = t & 127, wg = tg >> 5, ln = t & 31;
            float* ta = xch + (t >> 7) * 4096 + wg * 1024;                          // this warp's 32 x 32 block
            float* tb = xch + static_cast<size_t>(EPT) * nthr + (t >> 7) * 4096;    // the group's 4096 channels
            // T1, within the warp: lane al writes row al (16-byte chunk k of the
            // row at chunk k ^ (al & 7)), then lane b reads column b.
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4*>(ta + ln * 32 + 4 * (k ^ (ln & 7))) =
                    make_float4(v[2 * k].x, v[2 * k].y, v[2 * k + 1].x, v[2 * k + 1].y);
            __syncwarp();
            float2 u[EPT / 2];   // u[j] = channels al = 2j, 2j+1 of column b = lane
#pragma unroll
            for (int j = 0; j < EPT / 2; ++j) {
                u[j].x = ta[(2 * j) * 32 + 4 * ((ln >> 2) ^ ((2 * j) & 7)) + (ln & 3)];
                u[j].y = ta[(2 * j + 1) * 32 + 4 * ((ln >> 2) ^ ((2 * j + 1) & 7)) + (ln & 3)];
            }
            // stages h = 32 .. 512: pairs (al, al + h/32), in registers
#pragma unroll
            for (int j = 0; j < EPT / 2; ++j) {
                const float a0 = u[j].x, b0 = u[j].y;
                u[j].x = __fadd_rn(a0, b0);
                u[j].y = __fsub_rn(a0, b0);
            }
#pragma unroll
            for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
                for (int i = 0; i < EPT; i += 2) {
                    if ((i & h) == 0) {
                        const float2 a0 = u[i / 2], b0 = u[(i + h) / 2];
                        u[i / 2] = f2add_rn(a0, b0);
                        u[(i + h) / 2] = f2sub(a0, b0);
                    }
                }
            }
            // T2, across the group's 4 warps: channel i stored at
            // i ^ (4 (al & 1)); thread (al = tg / 4, c = tg % 4) then reads
            // channels 1024 ah + 32 al + 8 c + e for ah = 0..3, e = 0..7.
#pragma unroll
            for (int j = 0; j < EPT / 2; ++j) {
                tb[wg * 1024 + (2 * j) * 32 + ln] = u[j].x;
                tb[wg * 1024 + (2 * j + 1) * 32 + (ln ^ 4)] = u[j].y;
            }
            __syncthreads();
            const int al = tg >> 2, c4 = tg & 3;
            float w[4][8];
#pragma unroll
            for (int ah = 0; ah < 4; ++ah) {
                const float* src = tb + ah * 1024 + al * 32;
                const float4 p0 = *reinterpret_cast<const float4*>(src + 4 * ((2 * c4) ^ (al & 1)));
                const float4 p1 = *reinterpret_cast<const float4*>(src + 4 * ((2 * c4 + 1) ^ (al & 1)));
                w[ah][0] = p0.x; w[ah][1] = p0.y; w[ah][2] = p0.z; w[ah][3] = p0.w;
                w[ah][4] = p1.x; w[ah][5] = p1.y; w[ah][6] = p1.z; w[ah][7] = p1.w;
            }
            // stages h = 1024 (ah ^ 1), then 2048 (ah ^ 2)
#pragma unroll
            for (int hb = 1; hb <= 2; hb <<= 1) {
#pragma unroll
                for (int ah = 0; ah < 4; ++ah) {
                    if ((ah & hb) == 0) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float a0 = w[ah][e], b0 = w[ah + hb][e];
                            w[ah][e] = __fadd_rn(a0, b0);
                            w[ah + hb][e] = __fsub_rn(a0, b0);
                        }
                    }
                }
            }
            // channel of w[ah][e] within the row: grp0 + 1024 ah + e
            const int64_t grp0 = static_cast<int64_t>(t >> 7) * 4096 + 32 * al + 8 * c4;
            if constexpr (MODE == MODE_ROTATE) {
#pragma unroll
                for (int ah = 0; ah < 4; ++ah) {
                    float4* dst = reinterpret_cast<float4*>(out + m * K + grp0 + 1024 * ah);
                    const float2 c2 = make_float2(cg, cg);
                    const float2 a0 = f2mul_rn(make_float2(w[ah][0], w[ah][1]), c2);
                    const float2 a1 = f2mul_rn(make_float2(w[ah][2], w[ah][3]), c2);
                    const float2 a2 = f2mul_rn(make_float2(w[ah][4], w[ah][5]), c2);
                    const float2 a3 = f2mul_rn(make_float2(w[ah][6], w[ah][7]), c2);
                    dst[0] = make_float4(a0.x, a0.y, a1.x, a1.y);
                    dst[1] = make_float4(a2.x, a2.y, a3.x, a3.y);
                }
            } else if constexpr (MODE == MODE_SQNORM) {
#pragma unroll
                for (int ah = 0; ah < 4; ++ah)
#pragma unroll
                    for (int e = 0; e < 8; ++e) accsq[8 * ah + e] = __fmaf_rn(w[ah][e], w[ah][e], accsq[8 * ah + e]);
            }
            if constexpr (MODE != MODE_QUANT && MODE != MODE_QUANT8) {
                __syncthreads();   // the next row rewrites the cross-warp buffer
            } else {
                constexpr float LEVELS = MODE == MODE_QUANT8 ? 127.0f : 7.0f;
                float amax = 0.f;
#pragma unroll
                for (int ah = 0; ah < 4; ++ah)
#pragma unroll
                    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(w[ah][e]));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                const int nw = nthr >> 5;
                if ((t & 31) == 0) red[par][t >> 5] = amax;
                __syncthreads();
                amax = 0.f;
                for (int wi = 0; wi < nw; ++wi) amax = fmaxf(amax, red[par][wi]);
                uint32_t words[4] = {0u, 0u, 0u, 0u};
                uint32_t bytes[4][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}, {0u, 0u}};
                if (amax != 0.f && MODE == MODE_QUANT8) {
                    const float inv = __fdiv_rn(LEVELS, amax);
                    const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
#pragma unroll
                    for (int ah = 0; ah < 4; ++ah)
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            // the low byte of the sum's bits is the code in two's complement
                            const float2 tq = make_float2(__fmul_rn(w[ah][e], inv), __fmul_rn(w[ah][e + 1], inv));
                            const float2 r = f2add_rn(tq, magic);
                            bytes[ah][e >> 2] |= ((__float_as_uint(r.x) & 0xFFu) | ((__float_as_uint(r.y) & 0xFFu) << 8))
                                                 << (8 * (e & 2));
                        }
                } else if (amax != 0.f) {
                    const float inv = __fdiv_rn(LEVELS, amax);
                    const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
#pragma unroll
                    for (int ah = 0; ah < 4; ++ah) {
                        uint32_t wd = 0;
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            // fl32(u * inv) rounded (never merged into an fma), then the
                            // round-half-even add; the low nibble is the code
                            const float2 tq = make_float2(__fmul_rn(w[ah][e], inv), __fmul_rn(w[ah][e + 1], inv));
                            const float2 r = f2add_rn(tq, magic);
                            wd |= ((__float_as_uint(r.x) & 0xFu) | ((__float_as_uint(r.y) & 0xFu) << 4)) << (4 * e);
                        }
                        words[ah] = wd;
                    }
                }
                if constexpr (MODE == MODE_QUANT8) {
                    uint8_t* qrow = Xq + m * K;
#pragma unroll
                    for (int ah = 0; ah < 4; ++ah)
                        *reinterpret_cast<uint2*>(qrow + grp0 + 1024 * ah) = make_uint2(bytes[ah][0], bytes[ah][1]);
                } else {
                    uint8_t* qrow = Xq + m * (K / 2);
#pragma unroll
                    for (int ah = 0; ah < 4; ++ah)
                        *reinterpret_cast<uint32_t*>(qrow + (grp0 + 1024 * ah) / 2) = words[ah];
                }
                if (t == 0) sx[m] = (amax == 0.f) ? 0.f : __fmul_rn(__fdiv_rn(amax, LEVELS), cg);
            }
        } else {
            // ---- shuffle stages: partner thread t ^ s holds channels +-32s
    #pragma unroll
            for (int s = 1; s < TSHFL; s <<= 1) {
                const bool upper = (t & s) != 0;
    #pragma unroll
                for (int i = 0; i < EPT / 2; ++i) {
                    float2 p;
                    p.x = __shfl_xor_sync(0xFFFFFFFFu, v[i].x, s);
                    p.y = __shfl_xor_sync(0xFFFFFFFFu, v[i].y, s);
                    v[i] = upper ? f2sub(p, v[i]) : f2add_rn(v[i], p);
                }
            }
            // ---- cross-warp stages through shared memory (G >= 2048)
            if constexpr (TPG > 32) {
    #pragma unroll
                for (int s = 32; s < TPG; s <<= 1) {
                    const bool upper = (t & s) != 0;
    #pragma unroll
                    for (int i = 0; i < EPT / 2; ++i) {
                        xch[(2 * i) * nthr + t] = v[i].x;
                        xch[(2 * i + 1) * nthr + t] = v[i].y;
                    }
                    __syncthreads();
    #pragma unroll
                    for (int i = 0; i < EPT / 2; ++i) {
                        float2 p = make_float2(xch[(2 * i) * nthr + (t ^ s)], xch[(2 * i + 1) * nthr + (t ^ s)]);
                        v[i] = upper ? f2sub(p, v[i]) : f2add_rn(v[i], p);
                    }
                    __syncthreads();
                }
            }

            if constexpr (MODE == MODE_QUANT_ASYM) {
                // OffQ per-group asymmetric codes (groups of 32..1024 channels: the
                // TPG threads of a group sit in one warp).  The group's own range
                // [lo, hi] sets the step; the offset the all-ones row of H
                // created goes into the integer zero point (not clamped); a
                // constant group takes the step |lo| / 15 (1 when it is zero).
                float lo = v[0].x, hi = v[0].x;
    #pragma unroll
                for (int i = 0; i < EPT / 2; ++i) {
                    lo = fminf(lo, fminf(v[i].x, v[i].y));
                    hi = fmaxf(hi, fmaxf(v[i].x, v[i].y));
                }
    #pragma unroll
                for (int o = 1; o < TPG; o <<= 1) {
                    lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
                    hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
                }
                float dlt = __fsub_rn(hi, lo);
                if (dlt == 0.f) dlt = lo != 0.f ? fabsf(lo) : 15.f;
                const float inv = __fdiv_rn(15.f, dlt);
                const float zf = rintf(__fmul_rn(-lo, inv));
                uint32_t words[EPT / 8];
    #pragma unroll
                for (int j = 0; j < EPT / 8; ++j) {
                    uint32_t w = 0;
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // q = clamp(rint(fl32(u * inv)) + z, 0, 15); the multiply is
                        // rounded on its own (never merged into an fma)
                        const float q0 = fminf(fmaxf(__fadd_rn(rintf(__fmul_rn(v[4 * j + e].x, inv)), zf), 0.f), 15.f);
                        const float q1 = fminf(fmaxf(__fadd_rn(rintf(__fmul_rn(v[4 * j + e].y, inv)), zf), 0.f), 15.f);
                        w |= (static_cast<uint32_t>(q0) | (static_cast<uint32_t>(q1) << 4)) << (8 * e);
                    }
                    words[j] = w;
                }
                if (active) {
                    *reinterpret_cast<uint4*>(Xq + m * (K / 2) + col0 / 2) = make_uint4(words[0], words[1], words[2], words[3]);
                    if (t % TPG == 0) {
                        const int64_t gi = m * (K / G) + col0 / G;
                        sx[gi] = __fmul_rn(__fdiv_rn(dlt, 15.f), cg);
                        zx[gi] = static_cast<int32_t>(zf);
                    }
                }
            } else if constexpr (MODE == MODE_ROTATE) {
                if (active) {
                    float4* dst = reinterpret_cast<float4*>(out + m * K + col0);
                    const float2 c2 = make_float2(cg, cg);
    #pragma unroll
                    for (int j = 0; j < EPT / 4; ++j) {
                        const float2 a = f2mul_rn(v[2 * j], c2), b = f2mul_rn(v[2 * j + 1], c2);
                        dst[j] = make_float4(a.x, a.y, b.x, b.y);
                    }
                }
            } else if constexpr (MODE == MODE_SQNORM) {
    #pragma unroll
                for (int i = 0; i < EPT / 2; ++i) {
                    accsq[2 * i] = __fmaf_rn(v[i].x, v[i].x, accsq[2 * i]);
                    accsq[2 * i + 1] = __fmaf_rn(v[i].y, v[i].y, accsq[2 * i + 1]);
                }
            } else {
                constexpr float LEVELS = MODE == MODE_QUANT8 ? 127.0f : 7.0f;
                // ---- per-token absmax over the whole row
                float amax = 0.f;
    #pragma unroll
                for (int i = 0; i < EPT / 2; ++i) amax = fmaxf(amax, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
    #pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                const int nw = nthr >> 5;
                if (nw > 1) {
                    // one barrier per row: the other buffer is written by the next
                    // row, and the one after it only once every thread has passed
                    // the next row's barrier (so has finished reading this one)
                    if ((t & 31) == 0) red[par][t >> 5] = amax;
                    __syncthreads();
                    amax = 0.f;
                    for (int w = 0; w < nw; ++w) amax = fmaxf(amax, red[par][w]);
                }
                // ---- scale, round half to even, pack
                uint32_t words[EPT / 8];
                uint32_t bytes[EPT / 4];
    #pragma unroll
                for (int j = 0; j < EPT / 4; ++j) bytes[j] = 0u;
                if (amax == 0.f) {
    #pragma unroll
                    for (int j = 0; j < EPT / 8; ++j) words[j] = 0u;
                } else if (MODE == MODE_QUANT8) {
                    const float inv = __fdiv_rn(LEVELS, amax);
                    const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    #pragma unroll
                    for (int j = 0; j < EPT / 4; ++j) {
                        // channels 4j .. 4j+3: the low byte of each sum's bits is its code
                        const float2 t0 = make_float2(__fmul_rn(v[2 * j].x, inv), __fmul_rn(v[2 * j].y, inv));
                        const float2 t1 = make_float2(__fmul_rn(v[2 * j + 1].x, inv), __fmul_rn(v[2 * j + 1].y, inv));
                        const float2 r0 = f2add_rn(t0, magic), r1 = f2add_rn(t1, magic);
                        bytes[j] = __byte_perm(__byte_perm(__float_as_uint(r0.x), __float_as_uint(r0.y), 0x0040),
                                               __byte_perm(__float_as_uint(r1.x), __float_as_uint(r1.y), 0x0040), 0x5410);
                    }
    #pragma unroll
                    for (int j = 0; j < EPT / 8; ++j) words[j] = 0u;
                } else {
                    const float inv = __fdiv_rn(LEVELS, amax);
                    const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    #pragma unroll
                    for (int j = 0; j < EPT / 8; ++j) {
                        uint32_t w = 0;
    #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            // |u * inv| <= 7 (1 + 2^-23): adding 1.5*2^23 rounds it to an
                            // integer with ties to even; the low nibble of the sum's bits is
                            // that integer in two's complement.
                            // __fmul_rn is never merged into an fma, so fl32(u * inv) is
                            // rounded before the rounding add, as the codes are defined.
                            const float2 t = make_float2(__fmul_rn(v[4 * j + e].x, inv), __fmul_rn(v[4 * j + e].y, inv));
                            const float2 r = f2add_rn(t, magic);
                            const uint32_t b0 = __float_as_uint(r.x) & 0xFu;
                            const uint32_t b1 = __float_as_uint(r.y) & 0xFu;
                            w |= (b0 | (b1 << 4)) << (8 * e);
                        }
                        words[j] = w;
                    }
                }
                if (active) {
                    if constexpr (MODE == MODE_QUANT8) {
                        uint4* dst = reinterpret_cast<uint4*>(Xq + m * K + col0);
                        dst[0] = make_uint4(bytes[0], bytes[1], bytes[2], bytes[3]);
                        dst[1] = make_uint4(bytes[4], bytes[5], bytes[6], bytes[7]);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(Xq + m * (K / 2) + col0 / 2);
                        *dst = make_uint4(words[0], words[1], words[2], words[3]);
                    }
                }
                if (t == 0) sx[m] = (amax == 0.f) ? 0.f : __fmul_rn(__fdiv_rn(amax, LEVELS), cg);
            }
        }
#pragma unroll
        for (int j = 0; j < NRAW; ++j) raw[j] = raw_next[j];
    }

    if constexpr (MODE == MODE_SQNORM) {
        if (active) {
            if constexpr (G == 4096) {
                const int tg = t & 127;
                const int64_t grp0 = static_cast<int64_t>(t >> 7) * 4096 + 32 * (tg >> 2) + 8 * (tg & 3);
#pragma unroll
                for (int ah = 0; ah < 4; ++ah)
#pragma unroll
                    for (int e = 0; e < 8; ++e) atomicAdd(out + grp0 + 1024 * ah + e, accsq[8 * ah + e]);
            } else {
#pragma unroll
                for (int i = 0; i < EPT; ++i) atomicAdd(out + col0 + i, accsq[i]);
            }
        }
    }
}

// ------------------------------------------------------------------ dispatch
template <int XT, int MODE>
static hq_status launch_g(int group, const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* d, uint8_t* Xq,
                          float* sx, float* out, cudaStream_t st, int32_t* zx = nullptr) {
    const int threads = static_cast<int>(((K / EPT) + 31) / 32 * 32);
    const float cg = static_cast<float>(1.0 / __builtin_sqrt(static_cast<double>(group)));
    // G >= 2048: exchange area of EPT floats per thread; G == 4096 uses two
    // (the warp transposes and the cross-warp transpose)
    const size_t shm = (group >= 2048) ? static_cast<size_t>(EPT) * threads * sizeof(float) * (group == 4096 ? 2 : 1) : 0;
    int nsm = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    auto run = [&](auto kern) -> hq_status {
        if (shm > 32 * 1024) {   // with the static smem, anything near 48 KB needs the opt-in
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(shm)) !=
                cudaSuccess)
                return HQ_ERR_CUDA;
        }
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, shm) != cudaSuccess || per_sm < 1)
            return HQ_ERR_CUDA;
        int64_t grid = static_cast<int64_t>(per_sm) * nsm;
        if (grid > M) grid = M;
        kern<<<static_cast<unsigned>(grid), threads, shm, st>>>(X, M, K, ldx, d, Xq, sx, out, cg, zx);
        return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
    };
    if constexpr (MODE == MODE_QUANT_ASYM) {   // groups inside one warp, at least one thread each
        switch (group) {
            case 32: return run(k_rotate<32, XT, MODE>);
            case 64: return run(k_rotate<64, XT, MODE>);
            case 128: return run(k_rotate<128, XT, MODE>);
            case 256: return run(k_rotate<256, XT, MODE>);
            case 512: return run(k_rotate<512, XT, MODE>);
            case 1024: return run(k_rotate<1024, XT, MODE>);
            default: return HQ_ERR_UNSUPPORTED;
        }
    }
    switch (group) {
        case 8: return run(k_rotate<8, XT, MODE>);
        case 16: return run(k_rotate<16, XT, MODE>);
        case 32: return run(k_rotate<32, XT, MODE>);
        case 64: return run(k_rotate<64, XT, MODE>);
        case 128: return run(k_rotate<128, XT, MODE>);
        case 256: return run(k_rotate<256, XT, MODE>);
        case 512: return run(k_rotate<512, XT, MODE>);
        case 1024: return run(k_rotate<1024, XT, MODE>);
        case 2048: return run(k_rotate<2048, XT, MODE>);
        case 4096: return run(k_rotate<4096, XT, MODE>);
        default: return HQ_ERR_UNSUPPORTED;
    }
}

template <int MODE>
static hq_status launch_rotate(int xt, int group, const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* d,
                               uint8_t* Xq, float* sx, float* out, cudaStream_t st, int32_t* zx = nullptr) {
    if (xt == HQ_F16) return launch_g<XT_F16, MODE>(group, X, M, K, ldx, d, Xq, sx, out, st, zx);
    if (xt == HQ_BF16) return launch_g<XT_BF16, MODE>(group, X, M, K, ldx, d, Xq, sx, out, st, zx);
    if constexpr (MODE != MODE_QUANT && MODE != MODE_QUANT8 && MODE != MODE_QUANT_ASYM) {
        if (xt == HQ_F32) return launch_g<XT_F32, MODE>(group, X, M, K, ldx, d, Xq, sx, out, st);
    }
    return HQ_ERR_UNSUPPORTED;
}

// The streaming kernel of rotq.cu: 16-bit rows whose length is a multiple of
// 128 channels (up to 16384); other shapes use k_rotate above.
bool rotq_supported(int64_t M, int64_t K, int group);
hq_status launch_rotate_quant_stream(int xt, int group, const void* X, int64_t M, int64_t K, int64_t ldx,
                                     const int8_t* d, uint8_t* Xq, float* sx, cudaStream_t st, uint64_t limit_ns,
                                     int bits, int32_t* zx = nullptr);

static bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static hq_status check_rotate_args(int xt, int64_t M, int64_t K, int group) {
    if (M < 0 || K <= 0) return HQ_ERR_ARG;
    if (!is_pow2(group) || group < 8 || group > 4096) return HQ_ERR_ARG;
    if (K % group != 0 || K % EPT != 0) return HQ_ERR_ARG;
    if (xt != HQ_F16 && xt != HQ_BF16 && xt != HQ_F32) return HQ_ERR_UNSUPPORTED;
    if (K / EPT > 512) return HQ_ERR_UNSUPPORTED;
    return HQ_OK;
}

}  // namespace hq

using namespace hq;

extern "C" hq_status hq_rotate_quant(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x, int32_t group,
                                     const int8_t* H_signs, uint8_t* Xq, float* sx, void* stream) {
    hq_status s = check_rotate_args(xt, M, K, group);
    if (s != HQ_OK) return s;
    if (xt == HQ_F32) return HQ_ERR_UNSUPPORTED;
    if (ld_x < K) return HQ_ERR_ARG;
    if (M == 0) return HQ_OK;
    if (!X || !Xq || !sx) return HQ_ERR_ARG;
    if (!al16(X) || !al16(Xq) || (ld_x * 2) % 16 != 0) return HQ_ERR_ALIGN;
    if (rotq_supported(M, K, group))
        return launch_rotate_quant_stream(xt, group, X, M, K, ld_x, H_signs, Xq, sx, static_cast<cudaStream_t>(stream),
                                          2000000000ull, 4);
    return launch_rotate<MODE_QUANT>(xt, group, X, M, K, ld_x, H_signs, Xq, sx, nullptr,
                                     static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_rotate_quant8(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x, int32_t group,
                                      const int8_t* H_signs, int8_t* Xq8, float* sx, void* stream) {
    hq_status s = check_rotate_args(xt, M, K, group);
    if (s != HQ_OK) return s;
    if (xt == HQ_F32) return HQ_ERR_UNSUPPORTED;
    if (ld_x < K) return HQ_ERR_ARG;
    if (M == 0) return HQ_OK;
    if (!X || !Xq8 || !sx) return HQ_ERR_ARG;
    if (!al16(X) || !al16(Xq8) || (ld_x * 2) % 16 != 0) return HQ_ERR_ALIGN;
    uint8_t* q = reinterpret_cast<uint8_t*>(Xq8);
    if (rotq_supported(M, K, group))
        return launch_rotate_quant_stream(xt, group, X, M, K, ld_x, H_signs, q, sx, static_cast<cudaStream_t>(stream),
                                          2000000000ull, 8);
    return launch_rotate<MODE_QUANT8>(xt, group, X, M, K, ld_x, H_signs, q, sx, nullptr,
                                      static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_rotate_quant_asym(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                                          int32_t group, const int8_t* H_signs, uint8_t* Xq, float* sx, int32_t* zx,
                                          void* stream) {
    hq_status s = check_rotate_args(xt, M, K, group);
    if (s != HQ_OK) return s;
    if (xt == HQ_F32 || group < 32 || group > 1024) return HQ_ERR_UNSUPPORTED;
    if (ld_x < K) return HQ_ERR_ARG;
    if (M == 0) return HQ_OK;
    if (!X || !Xq || !sx || !zx) return HQ_ERR_ARG;
    if (!al16(X) || !al16(Xq) || (ld_x * 2) % 16 != 0) return HQ_ERR_ALIGN;
    if (group == 128 && rotq_supported(M, K, group))
        return launch_rotate_quant_stream(xt, group, X, M, K, ld_x, H_signs, Xq, sx, static_cast<cudaStream_t>(stream),
                                          2000000000ull, 4, zx);
    return launch_rotate<MODE_QUANT_ASYM>(xt, group, X, M, K, ld_x, H_signs, Xq, sx, nullptr,
                                          static_cast<cudaStream_t>(stream), zx);
}

extern "C" hq_status hq_rotate(const void* X, hq_dtype xt, int64_t M, int64_t K, int32_t group,
                               const int8_t* H_signs, float* out, void* stream) {
    hq_status s = check_rotate_args(xt, M, K, group);
    if (s != HQ_OK) return s;
    if (M == 0) return HQ_OK;
    if (!X || !out) return HQ_ERR_ARG;
    if (!al16(X) || !al16(out)) return HQ_ERR_ALIGN;
    return launch_rotate<MODE_ROTATE>(xt, group, X, M, K, K, H_signs, nullptr, nullptr, out,
                                      static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_channel_sqnorm(const void* X, hq_dtype xt, int64_t M, int64_t K, int32_t group,
                                       const int8_t* H_signs, float* norm2, void* stream) {
    hq_status s = check_rotate_args(xt, M, K, group);
    if (s != HQ_OK) return s;
    if (M == 0) return HQ_OK;
    if (!X || !norm2) return HQ_ERR_ARG;
    if (!al16(X)) return HQ_ERR_ALIGN;
    return launch_rotate<MODE_SQNORM>(xt, group, X, M, K, K, H_signs, nullptr, nullptr, norm2,
                                      static_cast<cudaStream_t>(stream));
}
