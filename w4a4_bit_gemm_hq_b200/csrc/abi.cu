// abi.cu -- host side of the libhq C ABI: argument checks, kernel selection,
// the device status word and the bounded-wait probe.
#include <cstdint>
#include <cstdlib>
#include <cuda_runtime.h>

#include "hq_device.cuh"
#include "hq_gemm.cuh"

namespace hq {

__device__ unsigned int g_status = 0;

constexpr uint64_t kDefaultLimitNs = 2000000000ull;  // 2 s per bounded wait

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}

__global__ void k_wait_probe(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // nothing ever arrives on this barrier: the wait must give up by itself
    if (threadIdx.x == 0) mbar_wait(b, 0, limit_ns);
    __syncthreads();
}

// Common checks of w4a4_linear / hq_debug_accum.
static hq_status check_gemm(const uint8_t* Xq, int64_t M, int64_t K, const uint8_t* Wq, const uint16_t* zw,
                            int64_t N, int32_t group, const uint8_t* A, const int32_t* sal, int32_t r) {
    if (M < 0 || N < 0 || K <= 0) return HQ_ERR_ARG;
    if (r < 0 || r > K) return HQ_ERR_ARG;
    if (group < 0 || (group > 0 && K % group != 0)) return HQ_ERR_ARG;
    if (K % 128 != 0 || K > 65536 || N % 8 != 0) return HQ_ERR_UNSUPPORTED;
    // group weights: multiples of 128 up to 2048 inputs (the large-M kernel's
    // group accumulators are read back as floats, exact for |acc| < 2^22)
    if (group % 128 != 0 || group > 2048) return HQ_ERR_UNSUPPORTED;
    if (r > 64 || r % 8 != 0) return HQ_ERR_UNSUPPORTED;
    if (M > (1ll << 30) || N > (1ll << 30)) return HQ_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return HQ_OK;
    if (!Xq || !Wq || (group > 0 && !zw)) return HQ_ERR_ARG;
    if (r > 0 && (!A || !sal)) return HQ_ERR_ARG;
    if (!al16(Xq) || !al16(Wq) || (group > 0 && !al16(zw))) return HQ_ERR_ALIGN;
    if (r > 0 && (reinterpret_cast<uintptr_t>(A) & 3u)) return HQ_ERR_ALIGN;
    return HQ_OK;
}

}  // namespace hq

using namespace hq;

extern "C" const char* hq_status_str(hq_status s) {
    switch (s) {
        case HQ_OK: return "HQ_OK";
        case HQ_ERR_ARG: return "HQ_ERR_ARG: invalid argument";
        case HQ_ERR_ALIGN: return "HQ_ERR_ALIGN: pointer or stride not 16-byte aligned";
        case HQ_ERR_UNSUPPORTED: return "HQ_ERR_UNSUPPORTED: outside what the kernels implement";
        case HQ_ERR_CUDA: return "HQ_ERR_CUDA: CUDA runtime error";
        case HQ_ERR_TIMEOUT: return "HQ_ERR_TIMEOUT: a device-side wait gave up";
    }
    return "unknown hq_status";
}

extern "C" int hq_device_sm_count(void) { return sm_count(); }

extern "C" hq_status hq_last_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HQ_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return HQ_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return HQ_ERR_CUDA;
    return static_cast<hq_status>(v);
}

extern "C" hq_status hq_debug_wait_probe(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1 || limit_ns > 1000000000ull) return HQ_ERR_ARG;
    k_wait_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

extern "C" size_t hq_linear_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group) {
    if (M <= 0 || N <= 0 || K <= 0 || !small_supported(M, group)) return 0;
    return small_workspace_bytes(M, N, K, group, sm_count());
}

static hq_status run_gemm(GemmArgs& a, int out, bool small, void* ws, size_t ws_bytes, cudaStream_t st) {
    const int nsm = sm_count();
    if (nsm <= 0) return HQ_ERR_CUDA;
    a.limit_ns = kDefaultLimitNs;
    if (small) {
        const size_t need = small_workspace_bytes(a.M, a.N, a.K, a.gw, nsm);
        if (need > 0 && (!ws || ws_bytes < need)) return HQ_ERR_ARG;
        if (ws && !al16(ws)) return HQ_ERR_ALIGN;
        a.ws = ws;
        return launch_gemm_small(a, out, st, nsm);
    }
    return launch_gemm_prefill(a, out, st, nsm);
}

namespace hq {
// Every check of w4a4_linear except the workspace's (shared with
// w4a4_linear_noalloc, which must not enqueue anything for a rejected call).
hq_status check_linear(const uint8_t* Xq, const float* sx, int64_t M, int64_t K, const uint8_t* Wq,
                       const uint16_t* sw, const uint16_t* zw, int64_t N, int32_t group, const uint8_t* A,
                       const uint16_t* B, const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt) {
    hq_status s = check_gemm(Xq, M, K, Wq, zw, N, group, A, sal_idx, r);
    if (s != HQ_OK) return s;
    if (yt != HQ_F16 && yt != HQ_BF16 && yt != HQ_F32) return HQ_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return HQ_OK;
    if (!sx || !sw || !Y || (r > 0 && !B)) return HQ_ERR_ARG;
    if (!al16(sw) || !al16(Y) || (r > 0 && !al16(B))) return HQ_ERR_ALIGN;
    return HQ_OK;
}
}  // namespace hq

extern "C" hq_status w4a4_linear(const uint8_t* Xq, const float* sx, int64_t M, int64_t K, const uint8_t* Wq,
                                 const uint16_t* sw, const uint16_t* zw, int64_t N, int32_t group, const uint8_t* A,
                                 const uint16_t* B, const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt,
                                 void* workspace, size_t ws_bytes, void* stream) {
    const hq_status s = check_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt);
    if (s != HQ_OK) return s;
    if (M == 0 || N == 0) return HQ_OK;
    GemmArgs a{};
    a.Xq = Xq; a.sx = sx; a.Wq = Wq; a.sw = sw; a.zw = zw; a.Rq = A; a.sr = B; a.sal = sal_idx;
    a.Y = Y;
    a.M = static_cast<int>(M); a.N = static_cast<int>(N); a.K = static_cast<int>(K); a.gw = group; a.r = r;
    a.act_bits = 4;
    return run_gemm(a, yt, small_supported(M, group), workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_debug_accum(const uint8_t* Xq, int64_t M, int64_t K, const uint8_t* Wq, const uint16_t* zw,
                                    int64_t N, int32_t group, const uint8_t* A, const int32_t* sal_idx, int32_t r,
                                    int32_t* acc, int32_t* acc_c, int32_t decode, void* workspace, size_t ws_bytes,
                                    void* stream) {
    hq_status s = check_gemm(Xq, M, K, Wq, zw, N, group, A, sal_idx, r);
    if (s != HQ_OK) return s;
    if (M == 0 || N == 0) return HQ_OK;
    if (!acc || (r > 0 && !acc_c)) return HQ_ERR_ARG;
    if (decode && !small_supported(M, group)) return HQ_ERR_UNSUPPORTED;
    // the debug epilogue stores raw accumulators and reads no scales
    GemmArgs a{};
    a.Xq = Xq; a.Wq = Wq; a.zw = zw; a.Rq = A; a.sal = sal_idx;
    a.dbg_acc = acc; a.dbg_acc_c = acc_c;
    a.M = static_cast<int>(M); a.N = static_cast<int>(N); a.K = static_cast<int>(K); a.gw = group; a.r = r;
    a.act_bits = 4;
    return run_gemm(a, OUT_DEBUG, decode != 0, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ W4A8
// The same GEMM with 8-bit activation codes (hq_rotate_quant8 outputs).
extern "C" hq_status w4a8_linear(const int8_t* Xq8, const float* sx, int64_t M, int64_t K, const uint8_t* Wq,
                                 const uint16_t* sw, const uint16_t* zw, int64_t N, int32_t group, const uint8_t* A,
                                 const uint16_t* B, const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt,
                                 void* workspace, size_t ws_bytes, void* stream) {
    const uint8_t* X8 = reinterpret_cast<const uint8_t*>(Xq8);
    const hq_status s = check_linear(X8, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt);
    if (s != HQ_OK) return s;
    if (M == 0 || N == 0) return HQ_OK;
    GemmArgs a{};
    a.Xq = X8; a.sx = sx; a.Wq = Wq; a.sw = sw; a.zw = zw; a.Rq = A; a.sr = B; a.sal = sal_idx;
    a.Y = Y;
    a.M = static_cast<int>(M); a.N = static_cast<int>(N); a.K = static_cast<int>(K); a.gw = group; a.r = r;
    a.act_bits = 8;
    return run_gemm(a, yt, small_supported(M, group), workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_debug_accum8(const int8_t* Xq8, int64_t M, int64_t K, const uint8_t* Wq, const uint16_t* zw,
                                     int64_t N, int32_t group, const uint8_t* A, const int32_t* sal_idx, int32_t r,
                                     int32_t* acc, int32_t* acc_c, int32_t decode, void* workspace, size_t ws_bytes,
                                     void* stream) {
    const uint8_t* X8 = reinterpret_cast<const uint8_t*>(Xq8);
    hq_status s = check_gemm(X8, M, K, Wq, zw, N, group, A, sal_idx, r);
    if (s != HQ_OK) return s;
    if (M == 0 || N == 0) return HQ_OK;
    if (!acc || (r > 0 && !acc_c)) return HQ_ERR_ARG;
    if (decode && !small_supported(M, group)) return HQ_ERR_UNSUPPORTED;
    GemmArgs a{};
    a.Xq = X8; a.Wq = Wq; a.zw = zw; a.Rq = A; a.sal = sal_idx;
    a.dbg_acc = acc; a.dbg_acc_c = acc_c;
    a.M = static_cast<int>(M); a.N = static_cast<int>(N); a.K = static_cast<int>(K); a.gw = group; a.r = r;
    a.act_bits = 8;
    return run_gemm(a, OUT_DEBUG, decode != 0, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}


// OffQ per-group asymmetric activations (hq_rotate_quant_asym's outputs):
// the small-M kernel, one launch per slice of up to 64 token rows (a slice
// reads the whole weight matrix, which stays in L2 across slices for weights
// up to ~100 MB); activation groups of 128 inputs (one K-block), nested in the
// weight groups.
namespace {
constexpr int64_t kAsymRows = 64;

hq_status check_asym(const float* sx, const int32_t* zx, int64_t M, int32_t group) {
    if (group != 0 && group % 128 != 0) return HQ_ERR_UNSUPPORTED;
    if (M > 0 && (!zx || !sx)) return HQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(zx) & 3u) || (reinterpret_cast<uintptr_t>(sx) & 3u)) return HQ_ERR_ALIGN;
    return HQ_OK;
}

// launches the slices of rows [0, M) in order on one stream
hq_status run_asym_slices(GemmArgs a, int64_t M, int out, size_t y_row_bytes, int64_t acc_row_elems,
                          cudaStream_t st) {
    const int64_t KB = a.K / 128;
    const uint8_t* Xq = a.Xq;
    const float* sx = a.sx;
    const int32_t* zx = a.zx;
    uint8_t* Y = static_cast<uint8_t*>(a.Y);
    int32_t* acc = a.dbg_acc;
    // the kernel stages a slice's codes in shared memory: long rows take
    // thinner slices (an unsupported slice is rejected before any launch)
    int64_t rows = kAsymRows;
    for (int64_t m0 = 0; m0 < M;) {
        a.M = static_cast<int>(M - m0 < rows ? M - m0 : rows);
        a.Xq = Xq + m0 * (a.K / 2);
        a.zx = zx + m0 * KB;
        if (sx) a.sx = sx + m0 * KB;
        if (Y) a.Y = Y + m0 * static_cast<int64_t>(y_row_bytes);
        if (acc) a.dbg_acc = acc + m0 * acc_row_elems;
        const hq_status s = run_gemm(a, out, true, nullptr, 0, st);
        if (s == HQ_ERR_UNSUPPORTED && m0 == 0 && rows > 8) {
            rows /= 2;
            continue;
        }
        if (s != HQ_OK) return s;
        m0 += rows;
    }
    return HQ_OK;
}
}  // namespace

extern "C" hq_status w4a4_linear_asym(const uint8_t* Xq, const float* sx, const int32_t* zx, int64_t M, int64_t K,
                                      const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                                      int32_t group, const uint8_t* A, const uint16_t* B, const int32_t* sal_idx,
                                      int32_t r, void* Y, hq_dtype yt, void* stream) {
    hq_status s = check_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt);
    if (s != HQ_OK) return s;
    s = check_asym(sx, zx, M, group);
    if (s != HQ_OK) return s;
    if (M == 0 || N == 0) return HQ_OK;
    GemmArgs a{};
    a.Xq = Xq; a.sx = sx; a.zx = zx; a.Wq = Wq; a.sw = sw; a.zw = zw; a.Rq = A; a.sr = B; a.sal = sal_idx;
    a.Y = Y;
    a.N = static_cast<int>(N); a.K = static_cast<int>(K); a.gw = group; a.r = r;
    a.act_bits = 4;
    const size_t yrow = static_cast<size_t>(N) * (yt == HQ_F32 ? 4u : 2u);
    return run_asym_slices(a, M, yt, yrow, 0, static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_debug_accum_asym(const uint8_t* Xq, const int32_t* zx, int64_t M, int64_t K,
                                         const uint8_t* Wq, const uint16_t* zw, int64_t N, int32_t group,
                                         int32_t* acc, void* stream) {
    hq_status s = check_gemm(Xq, M, K, Wq, zw, N, group, nullptr, nullptr, 0);
    if (s != HQ_OK) return s;
    if (group != 0 && group % 128 != 0) return HQ_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return HQ_OK;
    if (!acc || !zx) return HQ_ERR_ARG;
    GemmArgs a{};
    a.Xq = Xq; a.zx = zx; a.Wq = Wq; a.zw = zw;
    a.dbg_acc = acc;
    a.N = static_cast<int>(N); a.K = static_cast<int>(K); a.gw = group; a.r = 0;
    a.act_bits = 4;
    return run_asym_slices(a, M, OUT_DEBUG, 0, N * (K / 128), static_cast<cudaStream_t>(stream));
}
