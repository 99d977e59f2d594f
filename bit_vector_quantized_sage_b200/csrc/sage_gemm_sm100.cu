// tcgen05 / TMEM tensor-core path for M >= 9 (placeholder until the kernel lands).
#include <cuda_runtime.h>

#include "sage_internal.h"

namespace sage {

size_t gemm_workspace_bytes(const sage_matrix* A, int M) {
    return kWsHeader + (size_t)M * A->d_in * 2 + 256;
}

int launch_gemm(const sage_matrix*, const uint16_t*, int, uint16_t*, void*, size_t, sage_stream_t) {
    return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
