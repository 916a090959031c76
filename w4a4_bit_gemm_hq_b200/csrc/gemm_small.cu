// gemm_small.cu -- small-M (decode) variant of kernel K2; placeholder until
// the swap-operand split-K kernel lands: small M runs the large-M kernel.
#include "hq_gemm.cuh"

namespace hq {

bool small_supported(int64_t) { return false; }
size_t small_workspace_bytes(int64_t, int64_t, int64_t, int, int) { return 0; }
hq_status launch_gemm_small(const GemmArgs&, int, cudaStream_t, int) { return HQ_ERR_UNSUPPORTED; }

}  // namespace hq
