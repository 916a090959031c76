// hq_gemm.cuh -- argument block and launchers of the W4A4 GEMM kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"

namespace hq {

constexpr int OUT_DEBUG = 3;  // epilogue variant that stores raw integer accumulators

struct GemmArgs {
    const uint8_t* Xq;      // [M][K/2] packed activation codes ([M][K] int8 when act_bits == 8)
    const float* sx;        // [M]; OffQ activations: [M][K/128], one scale per token and 128-input group
    const int32_t* zx;      // OffQ activations: [M][K/128] integer zero points (else NULL)
    const uint8_t* Wq;      // [N][K/2] packed weight codes
    const uint16_t* sw;     // fp16 bits, [N] or [K/gw][N]
    const uint16_t* zw;     // fp16 bits, [K/gw][N] (gw > 0)
    const uint8_t* Rq;      // [N][r/2] packed SERQ codes
    const uint16_t* sr;     // fp16 bits, [N]
    const int32_t* sal;     // [r]
    void* Y;                // [M][N] output
    int32_t* dbg_acc;       // [M][N][G] (debug epilogue)
    int32_t* dbg_acc_c;     // [M][N]    (debug epilogue)
    void* ws;               // scratch (small-M kernel)
    int M, N, K, gw, r;
    int act_bits;           // 4: Xq packed int4 [M][K/2]; 8: Xq int8 codes [M][K] (W4A8)
    uint64_t limit_ns;      // bounded-wait limit
};

hq_status check_linear(const uint8_t* Xq, const float* sx, int64_t M, int64_t K, const uint8_t* Wq,
                       const uint16_t* sw, const uint16_t* zw, int64_t N, int32_t group, const uint8_t* A,
                       const uint16_t* B, const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt);
hq_status make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle swz);
hq_status launch_gemm_prefill(const GemmArgs& a, int out, cudaStream_t st, int nsm);
hq_status launch_gemm_small(const GemmArgs& a, int out, cudaStream_t st, int nsm);
size_t small_workspace_bytes(int64_t M, int64_t N, int64_t K, int gw, int nsm);
bool small_supported(int64_t M, int gw);

}  // namespace hq
