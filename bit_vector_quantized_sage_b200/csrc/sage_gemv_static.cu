// sage_gemv_static: the batch 1..8 GEMV of sage_gemv with its scratch memory in
// a fixed device array compiled into this library, for callers that cannot
// hand the library a workspace: code that runs where no allocator may be
// called (an allocator-free plugin or a custom op whose host framework owns
// all device memory), or that cannot grow device memory at the point of the
// call.  The entry point itself allocates nothing: it calls no cudaMalloc or
// cudaFree, no allocating library and no torch, and it runs the same kernel as
// sage_gemv with the array below standing in for the workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "sage_internal.h"

namespace sage {
namespace {

// Scratch of the static-scratch GEMV, laid out like a sage_gemv workspace:
// status word | split-K arrival counters | split-K partial sums.  Being a
// file-scope __device__ array it is zero when the module is loaded; the
// status word and the counters must be zero at the start of every call, and
// every call that completes leaves them zero again (the last CTA to arrive at
// a split block resets that block's counter).  The partial sums need no
// initial value.
constexpr size_t kStaticScratchBytes = size_t(4) << 20;
__device__ __align__(256) uint8_t g_gemv_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchEntry {
    unsigned long long ctx_id;  // context the address belongs to (0: unknown)
    void* ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

// Unique id of the calling thread's current context (cuCtxGetId), or 0 when
// the driver does not provide it.  The driver calls are reached through the
// runtime's entry-point query, so nothing links against libcuda.  Called with
// g_mu held.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool queried = false;
    if (!queried) {
        queried = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(f);
    }
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&c) == CUDA_SUCCESS && c && get_id(c, &id) == CUDA_SUCCESS) return id;
    return 0;
}

// Device address of g_gemv_scratch in the current context, looked up with
// that context current and cached per device together with the context's id:
// a new context on the device (after cudaDeviceReset, say) reloads the
// library's device code, and the address is looked up again.
int scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SAGE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    ScratchEntry& e = g_scratch[dev];
    const unsigned long long id = current_context_id();
    if (!e.ptr || id == 0 || id != e.ctx_id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || !p) return SAGE_ERR_CUDA;
        e.ptr = p;
        e.ctx_id = current_context_id();  // the lookup made the context current if it was not yet
    }
    *out = e.ptr;
    return SAGE_OK;
}

}  // namespace
}  // namespace sage

extern "C" int sage_gemv_static(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y, sage_stream_t stream) {
    using namespace sage;
    int rc = check_matrix(A);
    if (rc) return rc;
    if (!x || !y) return SAGE_ERR_INVALID_ARGUMENT;
    if (M < 1 || M > 8) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(y)) return SAGE_ERR_MISALIGNED;
    if (gemv_workspace_bytes(A, 1, M) > kStaticScratchBytes) return SAGE_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((rc = scratch_for_current_device(&scratch))) return rc;
    GemvJob job{*A, x, y};
    return launch_gemv(&job, 1, M, scratch, kStaticScratchBytes, stream);
}
