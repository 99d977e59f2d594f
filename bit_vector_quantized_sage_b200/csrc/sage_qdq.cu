// Continuous-parameter decode for blockwise optimisation on sm_100a: the
// forward pass of "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward
// Real-World Usability" Sec. 3.4 / App. A.6 with the discrete assignments
// kept and the codebook (Eqs. 12-13) and radii (softplus) continuous, the
// grid recomputed per row group from the current radii (Eq. 14) and the
// radius codes rounded per Eq. 2.
//
// One persistent grid (a few CTAs per SM).  Each CTA first builds the K unit
// codewords from their angle logits into shared memory (one thread per
// codeword: 7 sigmoids and 7 sin/cos pairs; bank-spread layout, cb_off),
// then walks row groups of 16 subvectors: 16 threads per group, one
// subvector each.  A group's min and
// max radius are two 16-lane shuffle reductions; each thread writes its
// subvector's 8 fp32 weights as two 16-byte stores (a group's 16 threads
// write 512 contiguous bytes).  Per subvector it reads 7 bytes (rho, sign
// byte, index) and writes 32; a 64 MB output stays in L2 during the launch,
// so HBM is not the limit: the L1 pipe is, through the random codeword reads
// from shared memory (hence the bank-spread layout) and the stores.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kQdqThreads = 256;             // 16 row groups of 16 subvectors per round
constexpr float kQdqEps = 1e-4f;             // angles kept eps away from 0 and pi/2 (Eq. 13)
constexpr float kQdqHalfPi = 1.57079632679489662f;

__device__ __forceinline__ float softplus_f(float rho) {
    return rho > 0.f ? rho + log1pf(expf(-rho)) : log1pf(expf(rho));
}

// Codeword k's 8 floats in shared memory, 4 floats of padding after every 4
// codewords: a codeword's two 16-byte halves then fall on bank quads
// (2k + k / 4) mod 8 and the next, so the random codewords of 8 lanes spread
// over all 8 quads instead of 4.
__device__ __forceinline__ uint32_t cb_off(uint32_t k) { return k * 8 + (k >> 2) * 4; }

template <bool V8>
__global__ void __launch_bounds__(kQdqThreads) qdq_forward_kernel(int d_out, int d_in, int log2K,
                                                                  const float* __restrict__ alpha,
                                                                  const float* __restrict__ rho,
                                                                  const uint8_t* __restrict__ signs,
                                                                  const uint16_t* __restrict__ idx,
                                                                  float* __restrict__ W, uint8_t* __restrict__ q,
                                                                  float* __restrict__ codebook_out) {
    __shared__ __align__(16) float cb[256 * 8 + 64 * 4];
    const int K = 1 << log2K, V = 10 - log2K, S = d_in >> 3, G = d_in >> 7;
    const int tid = threadIdx.x;
    if (tid < K) {  // Eq. 12-13: c_1 = cos t_1, c_j = sin t_1 .. sin t_(j-1) cos t_j, c_8 = prod sin
        float s = 1.f;
#pragma unroll
        for (int i = 0; i < 7; ++i) {
            const float a = alpha[tid * 7 + i];
            const float t = kQdqEps + (kQdqHalfPi - 2.f * kQdqEps) / (1.f + expf(-a));
            float st, ct;
            sincosf(t, &st, &ct);
            cb[cb_off(tid) + i] = s * ct;
            s *= st;
        }
        cb[cb_off(tid) + 7] = s;
        if (codebook_out && blockIdx.x == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) codebook_out[tid * 8 + i] = cb[cb_off(tid) + i];
        }
    }
    __syncthreads();
    const int t = tid & 15;                  // subvector within the group
    const float top = (float)((1 << V) - 1);
    const long long groups = (long long)d_out * G;
    for (long long g = (long long)blockIdx.x * (kQdqThreads / 16) + (tid >> 4); g < groups;
         g += (long long)gridDim.x * (kQdqThreads / 16)) {
        const int o = (int)(g / G), gg = (int)(g - (long long)o * G);
        const size_t e = (size_t)o * S + (size_t)gg * 16 + t;  // this subvector's field index
        const float r = softplus_f(__ldg(rho + e));
        float lo = r, hi = r;
#pragma unroll
        for (int m = 8; m; m >>= 1) {  // the group's 16 lanes (an aligned half warp)
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, m, 16));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, m, 16));
        }
        const float delta = (hi - lo) / top;  // Eq. 14
        float qq = 0.f;
        if (delta > 0.f) qq = fminf(fmaxf(floorf((r - lo) / delta + 0.5f), 0.f), top);  // Eq. 2
        const float rh = fmaf(qq, delta, lo);
        if (q) q[e] = (uint8_t)qq;
        const uint32_t sb = __ldg(signs + e);
        const float* c = cb + cb_off(__ldg(idx + e));
        float w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = ((sb >> i) & 1u) ? -(rh * c[i]) : rh * c[i];
        float* dst = W + (size_t)o * d_in + ((size_t)gg * 16 + t) * 8;
        if (V8) {  // one 32-byte store (W 32-byte aligned): half the store instructions
            asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "f"(w[0]), "f"(w[1]),
                         "f"(w[2]), "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]), "f"(w[7])
                         : "memory");
        } else {
            reinterpret_cast<float4*>(dst)[0] = make_float4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<float4*>(dst)[1] = make_float4(w[4], w[5], w[6], w[7]);
        }
    }
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" int sage_qdq_forward(int d_out, int d_in, int log2K, const float* alpha, const float* rho,
                                const uint8_t* signs, const uint16_t* idx, float* W, uint8_t* q, float* codebook,
                                sage_stream_t stream) {
    if (!alpha || !rho || !signs || !idx || !W) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return SAGE_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(W) % 16) return SAGE_ERR_MISALIGNED;
    const long long groups = (long long)d_out * (d_in / 128);
    const long long need = (groups + kQdqThreads / 16 - 1) / (kQdqThreads / 16);
    const int grid = (int)std::max<long long>(1, std::min<long long>(need, 8LL * current_sm_count()));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (reinterpret_cast<uintptr_t>(W) % 32 == 0)
        qdq_forward_kernel<true><<<grid, kQdqThreads, 0, s>>>(d_out, d_in, log2K, alpha, rho, signs, idx, W, q, codebook);
    else
        qdq_forward_kernel<false><<<grid, kQdqThreads, 0, s>>>(d_out, d_in, log2K, alpha, rho, signs, idx, W, q, codebook);
    return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
