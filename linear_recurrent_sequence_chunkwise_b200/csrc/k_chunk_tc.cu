// k_chunk_tc.cu -- tensor-core (tcgen05) chunkwise forward.  Placeholder
// until the kernel lands: it takes no problem.
#include "kernels.h"

namespace ret {

static __device__ int g_err_chunk_tc = 0;

cudaError_t read_clear_error_chunk_tc(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_err_chunk_tc, sizeof(int));
    if (e == cudaSuccess && *flag) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_err_chunk_tc, &zero, sizeof(int));
    }
    return e;
}

bool chunkwise_tc_supported(const RetArgs&) { return false; }

ret_status launch_chunkwise_tc(const RetArgs&, cudaStream_t) {
    return fail(RET_ERR_UNSUPPORTED, "tensor-core chunkwise kernel unavailable");
}

}  // namespace ret
