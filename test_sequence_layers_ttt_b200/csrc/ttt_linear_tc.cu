// Tensor-core TTT-Linear scan (placeholder until the kernel lands).
#include "ttt_internal.h"

namespace ttt {

__device__ unsigned int g_ttt_error_word = 0;

bool linear_tc_supports(const LinearArgs&) { return false; }

cudaError_t launch_linear_tc(const LinearArgs&, cudaStream_t) { return cudaErrorNotSupported; }

cudaError_t read_and_clear_device_error(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_ttt_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_ttt_error_word, &zero, sizeof(unsigned int));
}

}  // namespace ttt
