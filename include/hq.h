/*
 * hq.h -- C ABI of libhq, a B200 (sm_100a) implementation of the W4A4 rotated
 * linear layer: an online grouped Walsh-Hadamard rotation of the activations
 * with per-token symmetric int4 quantisation, packed int4 x int4 GEMM on the
 * tcgen05 tensor cores with int32 accumulation, a per-token x per-channel (or
 * per-group) dequantising epilogue, and SERQ's single rank-r error term on the
 * salient input channels fused into the same launch.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Y[M,N] = X[M,K] * W[N,K]^T (PyTorch Linear layout; the pages write Y = W X,
 *    "WaterSIC", technical summary section 1).
 *  - Pointers named "device" are CUDA device pointers owned by the caller; the
 *    library never frees or keeps them.  Pointers named "host" are host memory.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every device
 *    call only enqueues work on that stream and returns; results are valid
 *    after the stream has been synchronised.  Argument errors are detected on
 *    the host before anything is launched and leave all outputs untouched.
 *  - No call prints, aborts or traps.  Errors are reported by the return code;
 *    a device-side wait that exceeds its time limit records HQ_ERR_TIMEOUT,
 *    read back with hq_last_device_status().
 *  - Packed int4: element 2j is the low nibble of byte j, 2j+1 the high nibble.
 *    Activation codes and symmetric weight codes are two's complement nibbles;
 *    group-asymmetric weight codes are unsigned 0..15 with an integer zero
 *    point.  Packed activation rows (Xq) and SERQ rows (Rq) are row-major,
 *    ceil(cols/2) bytes per row.
 *  - Packed weights (Wq) are TILE-MAJOR: the row-major [N][K/2] byte matrix is
 *    cut into tiles of 128 rows x 64 bytes (128 rows x 128 input channels);
 *    tile (t, kb) is 8192 contiguous bytes at offset (t*(K/128) + kb) * 8192,
 *    row r of the tile at +r*64.  Byte j of row n is therefore at
 *    ((n/128 * (K/128) + j/64) * 128 + n%128) * 64 + j%64.  N is padded to a
 *    multiple of 128 with zero codes: the buffer holds
 *    hq_packed_weight_bytes(N, K) = ceil(N/128)*128 * K/2 bytes.  Every weight
 *    tile a GEMM stage needs is thus one contiguous 8 KB block in HBM.
 *  - fp16 values (scales, zero points) are passed as uint16_t bit patterns.
 *  - Device pointers to packed rows and to X must be 16-byte aligned, and
 *    row strides in bytes must be multiples of 16 (HQ_ERR_ALIGN otherwise).
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HQ_OK = 0,
    HQ_ERR_ARG = 1,          /* a size, a pointer or an index is invalid      */
    HQ_ERR_ALIGN = 2,        /* a pointer or a stride is not 16-byte aligned  */
    HQ_ERR_UNSUPPORTED = 3,  /* valid, but outside what the kernels implement */
    HQ_ERR_CUDA = 4,         /* a CUDA runtime call failed                    */
    HQ_ERR_TIMEOUT = 5       /* a device-side wait gave up (device status)    */
} hq_status;

typedef enum { HQ_F16 = 0, HQ_BF16 = 1, HQ_F32 = 2 } hq_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* hq_status_str(hq_status s);

/* Number of streaming multiprocessors of the current device, or -1. */
int hq_device_sm_count(void);

/* Bytes of a tile-major packed weight buffer for N x K weights (K % 128 == 0). */
size_t hq_packed_weight_bytes(int64_t N, int64_t K);

/*
 * hq_rotate_quant -- online activation transform, kernel K1.
 * Source: "OffQ: Taming Structured Outliers in LLM Quantization by Offsetting",
 * Methodology 2 (Hadamard rotation whose first row is all ones turns an
 * outlier concentrated in one channel into a constant offset over the group)
 * and 3 (group-wise rotation); "SERQ: Saliency-Aware Low-Rank Error
 * Reconstruction for LLM Quantization", technical summary section 1 (4-bit
 * activations, outliers set the step size).
 *
 * For every row m and every group b of `group` consecutive channels:
 *   u = (x_b .* d) * H_sylv            fp32 butterfly, stages h = 1,2,4,...
 *                                      ascending, (a,b) -> (a+b, a-b)
 *   amax = max over the whole row of |u|
 *   q = clamp(rint(fl32(u * fl32(7/amax))), -7, 7)   (all 0 if amax == 0)
 *   sx[m] = fl32(fl32(amax/7) * fl32(1/sqrt(group)))  (0 if amax == 0)
 * so that x*blockdiag(H)/sqrt(group) ~= q * sx[m].  H = diag(d)*Sylvester is a
 * Hadamard matrix with H[0,:] = 1 when d[0] = +1.
 *
 *  X       device, [M][ld_x] elements of type xt (HQ_F16 or HQ_BF16), row-major
 *  ld_x    row stride of X in elements, >= K, ld_x*2 a multiple of 16
 *  group   power of two, 8 <= group <= 4096, K % group == 0, K % 32 == 0
 *  H_signs device, [group] int8 in {+1,-1} with H_signs[0] == +1, or NULL (d = 1).
 *          Entries other than -1 are treated as +1.  H_signs[0] == -1 is
 *          reported as HQ_ERR_ARG in the device status word (read it with
 *          hq_last_device_status()); the outputs are then those of the given d.
 *  Xq      device, [M][K/2] packed int4 codes (output)
 *  sx      device, [M] fp32 scales (output)
 * Errors: HQ_ERR_ARG (M < 0, K <= 0, bad group, K % group, K % 32, NULL
 * pointer with M > 0), HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED (xt not 16-bit),
 * HQ_ERR_CUDA (launch failure).  M == 0 is a no-op.
 */
hq_status hq_rotate_quant(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                          int32_t group, const int8_t* H_signs, uint8_t* Xq, float* sx,
                          void* stream);

/*
 * hq_rotate -- the same rotation without quantisation, normalised:
 *   out[m][k] = fl32(u[m][k] * fl32(1/sqrt(group))).
 * Used offline to fold the rotation into the weights (W_rot = W * H~ keeps
 * X*W^T = (X*H~)*(W*H~)^T for the orthonormal H~ = blockdiag(H)/sqrt(group);
 * implied by OffQ, Methodology 2).
 *  X       device, [M][K] (xt = HQ_F16, HQ_BF16 or HQ_F32), contiguous rows
 *  out     device, [M][K] fp32 (output)
 * Errors as hq_rotate_quant.
 */
hq_status hq_rotate(const void* X, hq_dtype xt, int64_t M, int64_t K, int32_t group,
                    const int8_t* H_signs, float* out, void* stream);

/*
 * hq_channel_sqnorm -- calibration statistic for choosing the salient input
 * channels: norm2[k] += sum_m u[m][k]^2 over the rotated (unnormalised) rows.
 * Source: the per-channel activation L2 norm of "Adaptacion a cualquier
 * ancho de bits: Cuantizacion de precision mixta por canal para LLMs (CMPQ)",
 * Methodology A; SERQ section 2.2 (salient rows are those with the largest
 * accumulated error from activation outliers).
 *  norm2   device, [K] fp32, ACCUMULATED into (zero it before the first call);
 *          the summation order across rows is not fixed (atomics).
 * Errors as hq_rotate_quant.
 */
hq_status hq_channel_sqnorm(const void* X, hq_dtype xt, int64_t M, int64_t K, int32_t group,
                            const int8_t* H_signs, float* norm2, void* stream);

/*
 * hq_select_salient -- host helper: the r largest entries of norm2 (ties to the
 * lower index), written in ascending index order to sal (host, [r] int32).
 *  norm2   host, [K] fp32
 * Errors: HQ_ERR_ARG (NULL, r < 0, r > K, a NaN in norm2).
 */
hq_status hq_select_salient(const float* norm2, int64_t K, int32_t r, int32_t* sal);

/*
 * w4_pack -- offline weight quantiser, kernel K0.  Source: 4-bit weights of
 * SERQ sections 1-3; group-wise scale and zero point of OffQ Methodology 3;
 * uniform grid (OffQ contribution 2).
 *  group == 0: per output channel symmetric:
 *      s16 = fp16(fl32(amax_n/7)); q = clamp(rint(fl32(w/s16)), -8, 7), or 0
 *      when s16 == 0; sw[n] = s16; zw unused (may be NULL).
 *  group  > 0: per (channel, group) asymmetric over [min(lo,0), max(hi,0)]:
 *      s16 = fp16(fl32(fl32(hi-lo)/15)), 1.0 if that is 0;
 *      z = clamp(rint(fl32(-lo/s16)), 0, 15); q = clamp(rint(fl32(w/s16))+z, 0, 15);
 *      sw[b][n] = s16; zw[b][n] = fp16(z) (an integer): group-major layout.
 *  W       device, [N][K] of type wt (HQ_F16, HQ_BF16 or HQ_F32), contiguous
 *  Wq      device, hq_packed_weight_bytes(N, K) bytes, tile-major codes
 *          (output; padding rows are zero)
 *  sw      device, fp16 bits, [N] (group == 0) or [K/group][N] (output)
 *  zw      device, fp16 bits, [K/group][N] (output, group > 0)
 * Errors: HQ_ERR_ARG (sizes, K % 128, K % group, group < 0 or odd, NULLs),
 * HQ_ERR_ALIGN, HQ_ERR_CUDA.
 */
hq_status w4_pack(const void* W, hq_dtype wt, int64_t N, int64_t K, int32_t group,
                  uint8_t* Wq, uint16_t* sw, uint16_t* zw, void* stream);

/*
 * serq_prepare -- SERQ's single low-rank error matrix, offline.
 * Source: "SERQ ...", technical summary section 2.2 (extract the salient rows
 * of the weight error and reconstruct them with one matrix R, so that the
 * residual path is a single 4-bit matmul on those rows) and section 3.
 *   E[n][j] = fl32(W_rot[n][S_j] - What[n][S_j]), What the dequantised w4_pack
 *   output; R = E quantised per output row like a symmetric weight row:
 *   sr[n] = fp16(fl32(amax_j|E[n][j]|/7)), Rq codes in [-8,7].
 *  W_rot   device, [N][K] fp32 (the rotated weights that were packed)
 *  Wq, sw, zw, group   the w4_pack outputs (Wq tile-major) and its group argument
 *  sal_idx device, [r] int32 input channels, strictly ascending, in [0, K)
 *  r       0 <= r <= 256
 *  Rq      device, [N][ceil(r/2)] packed codes (output), the "A" operand
 *  sr      device, [N] fp16 bits (output), the "B" operand
 * Errors: HQ_ERR_ARG, HQ_ERR_CUDA.  An index outside [0, K) is never read
 * through: its error term is taken as 0 and the device status word records
 * HQ_ERR_ARG.
 */
hq_status serq_prepare(const float* W_rot, int64_t N, int64_t K, const uint8_t* Wq,
                       const uint16_t* sw, const uint16_t* zw, int32_t group,
                       const int32_t* sal_idx, int32_t r, uint8_t* Rq, uint16_t* sr,
                       void* stream);

/*
 * w4a4_linear -- the W4A4 GEMM with the fused SERQ term, kernel K2.
 * Source: "SERQ ...", technical summary section 2.2 (Y = X*W^T on 4-bit
 * operands plus one residual path X[:,S]*R^T, all in 4 bit) and section 3
 * (a single 4-bit matmul, no sequential low-rank factors, no intermediate
 * quantisation); OffQ Methodology 3 (group-wise scale and zero point).
 *   acc_b[m][n] = sum_{k in group b} qx[m][k] * (qw[n][k] - z[b][n])  (int32)
 *   acc_c[m][n] = sum_{j<r} qx[m][S_j] * qr[n][j]                      (int32)
 *   Y[m][n]     = sx[m] * (sum_b sw[b][n] * acc_b[m][n] + sr[n] * acc_c[m][n])
 * computed in fp32 and rounded once to yt.  One launch.
 *  Xq, sx   device, hq_rotate_quant outputs, [M][K/2] and [M]
 *  Wq, sw, zw, group   device, w4_pack outputs (Wq tile-major); group is 0 or a
 *           multiple of 128 up to 2048 (HQ_ERR_UNSUPPORTED beyond)
 *  A, B     device, serq_prepare outputs Rq [N][ceil(r/2)] and sr [N] (NULL if r == 0)
 *  sal_idx  device, [r] int32 (NULL if r == 0).  An index outside [0, K) is
 *           never read through: it contributes 0 and the device status word
 *           records HQ_ERR_ARG.
 *  r        0 <= r <= K (HQ_ERR_ARG otherwise); the kernels implement r <= 64
 *           with r % 8 == 0 (HQ_ERR_UNSUPPORTED otherwise)
 *  Y        device, [M][N] of type yt (HQ_F16, HQ_BF16 or HQ_F32) (output)
 *  workspace, ws_bytes   device scratch of at least
 *           hq_linear_workspace_size(M, N, K, group) bytes.  The current
 *           kernels need none: that size is 0 for every shape and workspace
 *           may be NULL.  The parameters stay so that a kernel that needs
 *           scratch can ask for it without a change of the ABI; a caller that
 *           passes scratch must zero it before its first use.
 * Requirements: K % 128 == 0, 0 < K <= 65536, N % 8 == 0; Xq, Wq, sw, zw,
 * B, Y and workspace 16-byte aligned, A 4-byte aligned (HQ_ERR_ALIGN).
 * Errors: HQ_ERR_ARG, HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED, HQ_ERR_CUDA.
 */
size_t hq_linear_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group);

hq_status w4a4_linear(const uint8_t* Xq, const float* sx, int64_t M, int64_t K,
                      const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                      int32_t group, const uint8_t* A, const uint16_t* B,
                      const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * w4a4_linear_noalloc -- w4a4_linear for callers that cannot allocate device
 * memory when they call it.  The pages have no counterpart: this is a service
 * of the library, not a step of the method.
 *
 * Runtimes that plan all their device buffers once at start-up and forbid
 * allocating later, or whose memory pool is exhausted, cannot hand a call
 * scratch memory.  This entry point takes the arguments of w4a4_linear minus
 * the workspace and never uses one: both GEMM kernels finish every output
 * inside the CTA that computes it, so no shape needs scratch.
 *
 *  - Every argument check of w4a4_linear runs first; a rejected call enqueues
 *    nothing.  A shape for which hq_linear_workspace_size would be non-zero
 *    (none with the current kernels) is rejected with HQ_ERR_UNSUPPORTED,
 *    also before anything is enqueued.
 * Arguments, results and the other errors are those of w4a4_linear.
 */
hq_status w4a4_linear_noalloc(const uint8_t* Xq, const float* sx, int64_t M, int64_t K,
                              const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                              int32_t group, const uint8_t* A, const uint16_t* B,
                              const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt, void* stream);

/*
 * W4A8 -- the layer with 8-bit activations for quantisation-sensitive layers.
 * Source: "DynamicPTQ", Methodology 2 (the sensitive layers keep 8-bit
 * activations while the rest of the model runs at 4 bit); "SERQ ...", section
 * 4 (the same reconstruction evaluated at W4A8).  Weights, SERQ term and
 * epilogue are those of the W4A4 calls.
 *
 * hq_rotate_quant8 -- hq_rotate_quant with 8-bit codes:
 *   amax = max over the row of |u|,  q = clamp(rint(fl32(u * fl32(127/amax))), -127, 127)
 *   (all 0 if amax == 0),  sx[m] = fl32(fl32(amax/127) * fl32(1/sqrt(group))).
 *  Xq8     device, [M][K] int8 codes, one per byte, row-major (output)
 * Other arguments, layouts and errors as hq_rotate_quant.
 */
hq_status hq_rotate_quant8(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                           int32_t group, const int8_t* H_signs, int8_t* Xq8, float* sx,
                           void* stream);

/*
 * hq_rotate_quant_asym -- OffQ's per-group asymmetric activation quantiser.
 * Source: "OffQ ...", Methodology 2, last point (the constant offset the
 * all-ones first row of H creates over a group is absorbed by the zero point
 * of an asymmetric quantiser) and Methodology 3 (one scale and zero point per
 * group).  Per row m and Hadamard group b of `group` channels: u = the rotated
 * group as in hq_rotate_quant; lo = min u, hi = max u, dlt = fl32(hi - lo)
 * (|lo| for a constant group, 15 when that is 0); inv = fl32(15 / dlt);
 * z = rint(fl32(-lo * inv)) (an integer, not clamped);
 * q = clamp(rint(fl32(u * inv)) + z, 0, 15);
 * sx[m][b] = fl32(fl32(dlt / 15) * fl32(1/sqrt(group))), zx[m][b] = z.
 *  X, xt, ld_x, group, H_signs   as hq_rotate_quant (16-bit X); group in
 *           [32, 1024] (HQ_ERR_UNSUPPORTED otherwise)
 *  Xq       device, [M][K/2] unsigned codes, element 2j in the low nibble (output)
 *  sx       device, [M][K/group] fp32 (output)
 *  zx       device, [M][K/group] int32 (output)
 * Errors: as hq_rotate_quant.
 */
hq_status hq_rotate_quant_asym(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                               int32_t group, const int8_t* H_signs, uint8_t* Xq, float* sx,
                               int32_t* zx, void* stream);

/*
 * w4a4_linear_asym -- w4a4_linear with OffQ's per-group asymmetric activations
 * (hq_rotate_quant_asym with group 128).  Source: "OffQ ...", Methodology 2
 * and 3; "SERQ ...", section 2.2 for the residual path.
 *   acc_b[m][n] = sum_{k in group b} (qx[m][k] - zx[m][b]) * (qw[n][k] - z[b'][n])
 *   Y[m][n] = sum_b sx[m][b] (sw[b'][n] acc_b[m][n]) + sr[n] sum_j a[m][j] qr[n][j],
 *   a[m][j] = sx[m][b_j] (qx[m][S_j] - zx[m][b_j]), b' = the weight group
 *   holding group b (the per-channel scale sw[n] when group == 0), all in fp32.
 *  Xq       device, [M][K/2] unsigned codes (hq_rotate_quant_asym, group 128)
 *  sx, zx   device, [M][K/128] fp32 scales and int32 zero points
 *  every other argument as w4a4_linear; group 0 or a multiple of 128.
 * Runs the small-M kernel once per slice of up to 64 token rows, in order on
 * the stream (each slice streams the weights; past the first they come from L2
 * when they fit there).  The call needs no workspace.  Errors: as w4a4_linear.
 */
hq_status w4a4_linear_asym(const uint8_t* Xq, const float* sx, const int32_t* zx, int64_t M, int64_t K,
                           const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                           int32_t group, const uint8_t* A, const uint16_t* B, const int32_t* sal_idx,
                           int32_t r, void* Y, hq_dtype yt, void* stream);

/* hq_debug_accum_asym -- the exact integer accumulators acc_b of
 * w4a4_linear_asym, acc [M][N][K/128] int32 (no SERQ term).  Test hook. */
hq_status hq_debug_accum_asym(const uint8_t* Xq, const int32_t* zx, int64_t M, int64_t K,
                              const uint8_t* Wq, const uint16_t* zw, int64_t N, int32_t group,
                              int32_t* acc, void* stream);

/*
 * w4a8_linear -- w4a4_linear with the activation codes of hq_rotate_quant8:
 *   acc_b[m][n] = sum_{k in group b} q8x[m][k] * (qw[n][k] - z[b][n]),
 *   acc_c[m][n] = sum_{j<r} q8x[m][S_j] * qr[n][j],  Y as w4a4_linear.
 *  Xq8     device, [M][K] int8 (16-byte aligned)
 * Every other argument, requirement, workspace rule and error as w4a4_linear.
 */
hq_status w4a8_linear(const int8_t* Xq8, const float* sx, int64_t M, int64_t K,
                      const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                      int32_t group, const uint8_t* A, const uint16_t* B,
                      const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * hq_debug_accum8 -- hq_debug_accum for w4a8_linear's kernels (test hook).
 */
hq_status hq_debug_accum8(const int8_t* Xq8, int64_t M, int64_t K, const uint8_t* Wq,
                          const uint16_t* zw, int64_t N, int32_t group, const uint8_t* A,
                          const int32_t* sal_idx, int32_t r, int32_t* acc, int32_t* acc_c,
                          int32_t decode, void* workspace, size_t ws_bytes, void* stream);

/*
 * hq_debug_accum -- test hook: runs the GEMM kernel of w4a4_linear with the
 * epilogue replaced by a raw store of the exact integer accumulators.
 *  acc     device, int32 [M][N][G] with G = K/group (1 when group == 0)
 *  acc_c   device, int32 [M][N] (may be NULL when r == 0)
 *  decode  0 = the large-M kernel, 1 = the small-M (swap-operand) kernel
 * Same requirements and errors as w4a4_linear.
 */
hq_status hq_debug_accum(const uint8_t* Xq, int64_t M, int64_t K, const uint8_t* Wq,
                         const uint16_t* zw, int64_t N, int32_t group, const uint8_t* A,
                         const int32_t* sal_idx, int32_t r, int32_t* acc, int32_t* acc_c,
                         int32_t decode, void* workspace, size_t ws_bytes, void* stream);

/*
 * hq_last_device_status -- synchronises `stream`, then reads and clears the
 * device status word that kernels set when a bounded wait gives up
 * (HQ_ERR_TIMEOUT) or an internal check fails (HQ_ERR_ARG).  HQ_OK if clean.
 */
hq_status hq_last_device_status(void* stream);

/*
 * hq_debug_wait_probe -- test hook for the failure path: launches one block
 * that waits, with the same bounded wait the GEMM kernels use, on an
 * mbarrier that nothing ever arrives on, with a time limit of `limit_ns`
 * nanoseconds (1 <= limit_ns <= 1e9).  The wait gives up, records
 * HQ_ERR_TIMEOUT in the device status word and the block exits normally, so
 * the context stays usable.  Read the status with hq_last_device_status().
 */
hq_status hq_debug_wait_probe(uint64_t limit_ns, void* stream);

/*
 * ---------------------------------------------------------------------------
 * Offline calibration (once per layer, before the online path; the results
 * are folded into the weights).  Sources: "OffQ: Taming Structured Outliers
 * in LLM Quantization by Offsetting", Methodology 1 (Top-1 PCA over the
 * token of largest L-infinity norm of each calibration sequence), Methodology
 * 3 and the ablation on sorted grouping (groups of 128 channels); "SERQ:
 * Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
 * technical summary section 1 (static per-channel flattening folded into the
 * weights) and section 3 (offline channel permutation of the weights).
 * Element types of X below: HQ_F16, HQ_BF16 or HQ_F32; row stride ld_x in
 * elements (>= K).  No alignment requirement.
 * ---------------------------------------------------------------------------
 */

/*
 * hq_calib_extreme_tokens -- for each calibration sequence s (rows
 * s*L .. s*L+L-1 of X), the token of largest max_k |x[k]| (ties to the earlier
 * token; NaN entries are ignored by the maximum): its index in the sequence,
 * tok[s], and its values widened to fp32, T[s][0..K).
 *  X    device, [S*L][ld_x] calibration activations
 *  tok  device, [S] int32 (output)
 *  T    device, [S][K] fp32 (output), contiguous; while the call runs, row s
 *       may first hold the per-token maxima of sequence s (when L <= K)
 * Errors: HQ_ERR_ARG (S < 0, L <= 0, K <= 0, ld_x < K, bad dtype, NULL with
 * S > 0), HQ_ERR_UNSUPPORTED (a size above INT32_MAX).  S == 0 is a no-op.
 */
hq_status hq_calib_extreme_tokens(const void* X, hq_dtype xt, int64_t S, int64_t L, int64_t K,
                                  int64_t ld_x, int32_t* tok, float* T, void* stream);

/*
 * hq_calib_top1_pca -- the principal eigenvector v of the (uncentred)
 * covariance C = T^T T / S of the S extreme tokens, by `iters` power
 * iterations (v <- C v / |C v|, C never formed) started from the token of
 * largest L2 norm, in fp32 with every sum in a fixed order (the result is
 * deterministic).  v is returned with unit length and its component of
 * largest magnitude positive; lambda[0] = |C v| of the last iteration (the
 * eigenvalue estimate; 0 for iters == 0).  All-zero tokens give v = e0,
 * lambda 0.  Convergence goes as (lambda2 / lambda1)^iters: the caller picks
 * iters.
 *  T       device, [S][K] fp32 (from hq_calib_extreme_tokens)
 *  v       device, [K] fp32 (output);  lambda  device, [1] fp32 (output)
 * Runs as one CTA with v and T v in shared memory: S + K <=
 * hq_calib_pca_max_elems() (HQ_ERR_UNSUPPORTED otherwise).
 * Errors: HQ_ERR_ARG (S <= 0, K <= 0, iters < 0, NULL), HQ_ERR_UNSUPPORTED.
 */
size_t hq_calib_pca_max_elems(void);
hq_status hq_calib_top1_pca(const float* T, int64_t S, int64_t K, int32_t iters, float* v, float* lambda,
                            void* stream);

/*
 * hq_calib_householder -- Y = X Q with the reflection Q = I - 2 w w^T / (w^T w),
 * w = v' - e0, where v' = -v if v[0] > 0 else v: Q is symmetric and
 * orthogonal and maps v' to e0, so the direction of v (the outlier
 * direction) lands in channel 0.  Apply it to the activations and to the
 * weight rows alike (X Q (W Q)^T = X W^T).  fp32 arithmetic: per row
 * c = fl(2 / w^T w) * (x . w), y = x - c w.
 *  v  device, [K] fp32 of unit length;  Y  device, [M][K] fp32 (output)
 * Errors: HQ_ERR_ARG (M < 0, K <= 0, ld_x < K, bad dtype, NULL with M > 0),
 * HQ_ERR_UNSUPPORTED (K > 58080, M above INT32_MAX).  M == 0 is a no-op.
 */
hq_status hq_calib_householder(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                               const float* v, float* Y, void* stream);

/*
 * hq_calib_channel_absmax -- amax[k] = max over rows m of |X[m][k]| (exact;
 * NaN entries are ignored).  amax is overwritten (cleared on the stream
 * first); M == 0 gives zeros.
 *  amax  device, [K] fp32 (output)
 * Errors: HQ_ERR_ARG (M < 0, K <= 0, ld_x < K, bad dtype, NULL),
 * HQ_ERR_UNSUPPORTED (a size above INT32_MAX), HQ_ERR_CUDA.
 */
hq_status hq_calib_channel_absmax(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                                  float* amax, void* stream);

/*
 * hq_calib_sorted_perm -- sorted grouping: perm[j] = the channel at position j
 * in the order of decreasing stat (ties to the lower channel index; NaN sorts
 * as -infinity).  Consecutive runs of `group` positions form the groups, so
 * each group's first channel is its largest, the channel whose outlier the
 * all-ones first row of H turns into the group's offset.
 *  stat  device, [K] fp32;  perm  device, [K] int32 (output), a permutation
 * Errors: HQ_ERR_ARG (K <= 0, NULL), HQ_ERR_UNSUPPORTED (K above INT32_MAX).
 */
hq_status hq_calib_sorted_perm(const float* stat, int64_t K, int32_t* perm, void* stream);

/*
 * hq_calib_flatten_scales -- static flattening: s[k] = xmax[k]^alpha /
 * wmax[k]^(1-alpha) (fp32 powf and an IEEE divide); 1 where xmax[k] or
 * wmax[k] is not positive.  Divide the activation channels by s and multiply
 * the weight columns by s (hq_permute_channels ops 1 and 2).
 *  xmax, wmax  device, [K] fp32 (per-channel max |x|, max |w|);  s  device, [K]
 * Errors: HQ_ERR_ARG (K <= 0, NULL, alpha outside [0, 1]), HQ_ERR_UNSUPPORTED.
 */
hq_status hq_calib_flatten_scales(const float* xmax, const float* wmax, int64_t K, float alpha, float* s,
                                  void* stream);

/*
 * hq_permute_channels -- Y[m][j] = X[m][c] with c = perm[j] (c = j when perm
 * is NULL), op 0: as is, op 1: fl32(x / s[c]), op 2: fl32(x * s[c]); x widened
 * to fp32 first.  The offline permutation (and flattening) of weight columns
 * and, for calibration and tests, of activation rows.  A perm entry outside
 * [0, K) writes 0 and records HQ_ERR_ARG in the device status word
 * (hq_last_device_status).
 *  perm  device, [K] int32 or NULL;  s  device, [K] fp32 (ops 1, 2)
 *  Y     device, [M][K] fp32 (output), contiguous
 * Errors: HQ_ERR_ARG (M < 0, K <= 0, ld_x < K, op outside 0..2, NULL X or Y
 * with M > 0, NULL s with op != 0), HQ_ERR_UNSUPPORTED.  M == 0 is a no-op.
 */
hq_status hq_permute_channels(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x,
                              const int32_t* perm, const float* s, int32_t op, float* Y, void* stream);

/*
 * hq_quant_mxfp4 -- MXFP4 block quantisation of rows of values (the 4-bit
 * format SERQ names beside INT4 for its main and residual paths, "SERQ:
 * Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
 * technical summary sections 2 and 3).  Per block of 32 consecutive values
 * of a row: E = floor(log2(amax)) - 2, scale byte = clamp(E + 127, 0, 254)
 * (UE8M0; 0 for an all-zero block), t = v * 2^-(byte - 127), |t| rounded to
 * the E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6} to nearest with ties to the even
 * mantissa (0, 1, 2, 4) and saturated at 6, sign bit 3 for t < 0 with a
 * non-zero magnitude; element 2j in the low nibble of byte j.  Activations
 * are quantised after hq_rotate (fp32 rows), weights as W_rot.  Inputs must
 * be finite.
 *  X       device, [M][ld_x] (HQ_F16, HQ_BF16 or HQ_F32), 16-byte aligned,
 *          ld_x * element size a multiple of 16
 *  Xq      device, [M][K/2] codes (output), 16-byte aligned
 *  scales  device, [M][K/32] scale bytes (output)
 * Errors: HQ_ERR_ARG (M < 0, K <= 0, K % 32, ld_x < K, bad dtype, NULL with
 * M > 0), HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED (a size above INT32_MAX),
 * HQ_ERR_CUDA.  M == 0 is a no-op.
 */
hq_status hq_quant_mxfp4(const void* X, hq_dtype xt, int64_t M, int64_t K, int64_t ld_x, uint8_t* Xq,
                         uint8_t* scales, void* stream);

/*
 * hq_mxfp4_linear -- Y = X^ W^T for MXFP4 operands (codes and scale bytes as
 * hq_quant_mxfp4 writes them), X^, W^ the values the codes stand for.  Twice
 * an E2M1 value is an integer in [-12, 12], so each 32-value block of a row
 * pair is an exact int8 dot product (warp-level int8 MMA); the block sums are
 * scaled by 2^(Ex + Ew) (exact) and added in fp32 in block order.  The
 * block-scaled tensor-core MMA (tcgen05 kind::mxf4) is not used.  Two calls
 * with accumulate = 1 on the second add SERQ's residual product (salient
 * activation block against the MXFP4 error rows) to the main one.
 *  Xq, sx   device, [M][K/2] codes and [M][K/32] scale bytes (2-byte aligned)
 *  Wq, sw   device, [N][K/2] codes and [N][K/32] scale bytes (row-major)
 *  Y        device, [M][N] fp32 (output; accumulate != 0: added to), 4-byte aligned
 * Errors: HQ_ERR_ARG (M < 0, N < 0, K <= 0, K % 32, NULL with M, N > 0),
 * HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED (a size above INT32_MAX), HQ_ERR_CUDA.
 */
hq_status hq_mxfp4_linear(const uint8_t* Xq, const uint8_t* sx, int64_t M, int64_t K, const uint8_t* Wq,
                          const uint8_t* sw, int64_t N, float* Y, int32_t accumulate, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
