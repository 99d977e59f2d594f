// Adaptive bit splitting on sm_100a (Sec. 3.3 of "SAGE: Pushing 2-Bit
// Vector-Quantized LLMs toward Real-World Usability", Eqs. 7-9): the
// energy-weighted relative reconstruction error of an encoded matrix against
// its original weights, in original channel order (Eq. 8), and the choice of
// the split with the smallest error among candidate encodings (Eq. 9).
//
// One persistent grid, one CTA per SM, walks the row octets; within an octet
// a thread takes subvector columns j = tid, tid + blockDim, ...  A thread
// rebuilds its record's 8 rows x 8 weights in fp32 (r^ = mu + q delta times
// the signed fp16 codeword, as the GEMV does), reads the 8 original channels
// perm[8j .. 8j + 7] of each row of W and their energies, and adds
// e (w - w^)^2 and e w^2 in fp64.  The permutation scatters a thread's W
// reads over the octet's 8 rows, but the CTA as a whole reads every element
// of those rows once, so they stay in L1 (8 rows of fp32 W) and each W
// sector comes from HBM once.  Each CTA reduces its sums and stores them; the
// host adds the CTAs' partials in CTA order (the result is deterministic)
// and divides.
#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
using namespace dev;
namespace {

constexpr int kAbsThreads = 512;

int abs_ctas() { return 2 * current_sm_count(); }

template <int V>
__global__ void __launch_bounds__(kAbsThreads) abs_error_kernel(sage_matrix A, const float* __restrict__ W,
                                                                const float* __restrict__ energy,
                                                                double* __restrict__ partials) {
    using F = Fmt<V>;
    const int R8 = (A.d_out + 7) >> 3, S = A.d_in >> 3, G = A.d_in >> 7;
    const uint4* cb = reinterpret_cast<const uint4*>(A.codebook);
    double num = 0.0, den = 0.0;
    for (int b = blockIdx.x; b < R8; b += gridDim.x)
    for (int j = threadIdx.x; j < S; j += blockDim.x) {
        const int blk = b >> 5, ob = b & 31, g = j >> 4, t = j & 15;
        const uint4 rec = __ldg(reinterpret_cast<const uint4*>(A.main + main_word(R8, S, blk, j, ob, 0)));
        const uint32_t wv[4] = {rec.x, rec.y, rec.z, rec.w};
        int ch[8];
        float ev[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            ch[i] = A.perm ? __ldg(A.perm + 8 * j + i) : 8 * j + i;  // original channel of storage column 8j + i
            ev[i] = __ldg(energy + ch[i]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int row = b * 8 + 2 * u + half;
                if (row >= A.d_out) continue;
                const uint2 e = __ldg(reinterpret_cast<const uint2*>(A.meta) + meta_entry(R8, G, blk, g, ob, 2 * u + half));
                const float2 md = __half22float2(u2h2(e.y));
                const float dl = md.y * (float)(1 << V), mp = md.x - dl;
                const uint32_t wa = wv[u];
                const uint32_t wf = half ? rot16(wa) : wa;  // field word (z, q) of this row
                uint4 c = __ldg(cb + ((wf & F::kZMask) >> 7));
                if (!half) {
                    c.x ^= slot_mask<F::slot(0)>(wa);
                    c.y ^= slot_mask<F::slot(1)>(wa);
                    c.z ^= slot_mask<F::slot(2)>(wa);
                } else {
                    c.x ^= slot_mask<F::slot(3)>(wa);
                    c.y ^= slot_mask<F::slot(4)>(wa);
                    c.z ^= slot_mask<F::slot(5)>(wa);
                }
                c.w ^= aux_mask(e.x, t);
                const float r = fmaf(q_unit<V>(wf), dl, mp);  // Eq. 2
                const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
                const float* wr = W + (size_t)row * A.d_in;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 cf = __half22float2(u2h2(cw[k]));
                    const float w0 = __ldg(wr + ch[2 * k]), w1 = __ldg(wr + ch[2 * k + 1]);
                    const float d0 = w0 - r * cf.x, d1 = w1 - r * cf.y;
                    num = fma((double)ev[2 * k] * d0, (double)d0, num);
                    num = fma((double)ev[2 * k + 1] * d1, (double)d1, num);
                    den = fma((double)ev[2 * k] * w0, (double)w0, den);
                    den = fma((double)ev[2 * k + 1] * w1, (double)w1, den);
                }
            }
        }
    }
    // CTA reduction in a fixed order: warps by shuffle, then warp 0 over the warps
    __shared__ double s_num[kAbsThreads / 32], s_den[kAbsThreads / 32];
    for (int o = 16; o; o >>= 1) {
        num += __shfl_xor_sync(0xffffffffu, num, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_num[warp] = num;
        s_den[warp] = den;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, bsum = 0.0;
        for (int w = 0; w < kAbsThreads / 32; ++w) {
            a += s_num[w];
            bsum += s_den[w];
        }
        partials[2 * blockIdx.x] = a;
        partials[2 * blockIdx.x + 1] = bsum;
    }
}

}  // namespace

size_t abs_partials_bytes() { return (size_t)abs_ctas() * 2 * sizeof(double); }
size_t abs_workspace_bytes(int n) { return 256 + (size_t)(n < 1 ? 1 : n) * abs_partials_bytes(); }

namespace {

int abs_launch(const sage_matrix* A, const float* W, const float* energy, double* partials, cudaStream_t s) {
    const int grid = abs_ctas();
    switch (A->log2K) {
        case 4: abs_error_kernel<6><<<grid, kAbsThreads, 0, s>>>(*A, W, energy, partials); break;
        case 5: abs_error_kernel<5><<<grid, kAbsThreads, 0, s>>>(*A, W, energy, partials); break;
        case 6: abs_error_kernel<4><<<grid, kAbsThreads, 0, s>>>(*A, W, energy, partials); break;
        case 7: abs_error_kernel<3><<<grid, kAbsThreads, 0, s>>>(*A, W, energy, partials); break;
        default: abs_error_kernel<2><<<grid, kAbsThreads, 0, s>>>(*A, W, energy, partials); break;
    }
    return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

// Eq. 8 from one candidate's CTA partials, added in CTA order (deterministic).
int abs_finish(const double* h, double* err) {
    double num = 0.0, den = 0.0;
    for (int c = 0; c < abs_ctas(); ++c) {
        num += h[2 * c];
        den += h[2 * c + 1];
    }
    if (!(den > 0.0)) return SAGE_ERR_INVALID_ARGUMENT;
    *err = num / den;
    return SAGE_OK;
}

// Scores candidates [0, n): as many per round as the workspace holds partials
// for, one copy back and one synchronisation per round.
int abs_score(const sage_matrix* cands, int n, const float* W, const float* energy, void* ws, size_t ws_bytes,
              double* errs, sage_stream_t stream) {
    if (!W || !energy || !errs) return SAGE_ERR_INVALID_ARGUMENT;
    if (!ws) return SAGE_ERR_WORKSPACE;
    if (!aligned16(ws) || !aligned16(W)) return SAGE_ERR_MISALIGNED;
    if (ws_bytes < abs_workspace_bytes(1)) return SAGE_ERR_WORKSPACE;
    for (int i = 0; i < n; ++i) {
        const int rc = check_matrix(&cands[i]);
        if (rc) return rc;
    }
    const size_t per = abs_partials_bytes();
    const int batch = (int)std::min<size_t>((size_t)n, (ws_bytes - 256) / per);
    double* partials = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + 256);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::vector<double> h(per / sizeof(double) * (size_t)batch);
    for (int i0 = 0; i0 < n; i0 += batch) {
        const int nb = std::min(batch, n - i0);
        for (int b = 0; b < nb; ++b) {
            const int rc = abs_launch(&cands[i0 + b], W, energy, partials + b * (per / sizeof(double)), s);
            if (rc) return rc;
        }
        if (cudaMemcpyAsync(h.data(), partials, per * nb, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return SAGE_ERR_CUDA;
        for (int b = 0; b < nb; ++b) {
            const int rc = abs_finish(h.data() + b * (per / sizeof(double)), &errs[i0 + b]);
            if (rc) return rc;
        }
    }
    return SAGE_OK;
}

}  // namespace

}  // namespace sage

using namespace sage;

extern "C" int sage_abs_error(const sage_matrix* A, const float* W, const float* energy, void* ws, size_t ws_bytes,
                              double* err, sage_stream_t stream) {
    if (!A) return SAGE_ERR_INVALID_ARGUMENT;
    if (!err) return SAGE_ERR_INVALID_ARGUMENT;
    return abs_score(A, 1, W, energy, ws, ws_bytes, err, stream);
}

extern "C" int sage_abs_select(const sage_matrix* cands, int n, const float* W, const float* energy, void* ws,
                               size_t ws_bytes, int* best, double* errs, sage_stream_t stream) {
    if (!cands || n < 1 || !best) return SAGE_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < n; ++i)
        if (cands[i].d_out != cands[0].d_out || cands[i].d_in != cands[0].d_in) return SAGE_ERR_UNSUPPORTED;
    std::vector<double> e((size_t)n);
    const int rc = abs_score(cands, n, W, energy, ws, ws_bytes, e.data(), stream);
    if (rc) return rc;
    int arg = 0;
    for (int i = 1; i < n; ++i)
        if (e[i] < e[arg]) arg = i;  // Eq. 9; ties keep the earlier candidate
    if (errs)
        for (int i = 0; i < n; ++i) errs[i] = e[i];
    *best = arg;
    return SAGE_OK;
}
