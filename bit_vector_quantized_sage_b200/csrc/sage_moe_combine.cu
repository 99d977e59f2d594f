// Router-weighted combine of a mixture-of-experts projection on sm_100a: the
// step after the down projection of a top-k routed MLP (the Qwen3-30B-A3B
// shape that "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World
// Usability" evaluates in Sec. 4.1), where token t's output is the sum over
// its k routed slots of the router weight times that slot's expert output:
//   y[t] = sum_k w[t][k] * y_pair[t * topk + k],   fp32 in slot order, fp16 out.
// One thread per 8 outputs of a token (16-byte loads of the slots' rows).
// Launched with programmatic dependent launch: it starts while the grouped
// GEMV that writes y_pair drains and waits for it before its first load.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
namespace {

__global__ void __launch_bounds__(256) moe_combine_kernel(int T, int topk, int d8, const uint4* __restrict__ y,
                                                          const float* __restrict__ w, uint4* __restrict__ out) {
    dev::pdl_wait();  // the slots' outputs come from the preceding kernel
    const long long total = (long long)T * d8;
    for (long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x; id < total;
         id += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(id / d8), c8 = (int)(id - (long long)t * d8);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int k = 0; k < topk; ++k) {
            const size_t row = (size_t)t * topk + k;
            const float wk = __ldg(w + row);
            const uint4 v = __ldg(y + row * d8 + c8);
            const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(dev::u2h2(h[i]));
                acc[2 * i] = fmaf(wk, f.x, acc[2 * i]);
                acc[2 * i + 1] = fmaf(wk, f.y, acc[2 * i + 1]);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = dev::h22u(__floats2half2_rn(acc[2 * i], acc[2 * i + 1]));
        out[id] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" int sage_moe_combine(int T, int topk, int d_out, const uint16_t* y_pairs, const float* weights,
                                uint16_t* y, sage_stream_t stream) {
    if (!y_pairs || !weights || !y) return SAGE_ERR_INVALID_ARGUMENT;
    if (T < 1 || topk < 1 || d_out < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_out % 8) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(y_pairs) || !aligned16(y) || reinterpret_cast<uintptr_t>(weights) % 4) return SAGE_ERR_MISALIGNED;
    const int d8 = d_out / 8;
    const long long total = (long long)T * d8;
    const int grid = (int)std::max<long long>(1, std::min<long long>((total + 255) / 256, 4LL * current_sm_count()));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(256u);
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe_combine_kernel, T, topk, d8, reinterpret_cast<const uint4*>(y_pairs), weights,
                              reinterpret_cast<uint4*>(y)) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}
