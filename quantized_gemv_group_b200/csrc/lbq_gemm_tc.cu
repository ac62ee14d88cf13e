// lbq_gemm_tc.cu -- batched group GEMM on tcgen05 tensor cores (M >= 64).
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

size_t gemm_group_tc_ws_bytes(int64_t, int64_t, int64_t) { return 0; }
bool gemm_group_tc_supported(int64_t, int64_t, int64_t, int, int) { return false; }
lbq_status launch_gemm_group_tc(const void*, bool, int64_t, const void*, const void*, const void*, int64_t, int64_t,
                                int, int, void*, void*, size_t, cudaStream_t) {
    return LBQ_ERR_UNSUPPORTED;
}

}  // namespace lbq
