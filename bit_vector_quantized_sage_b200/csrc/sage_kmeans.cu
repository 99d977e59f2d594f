// The encoder's weighted spherical k-means on sm_100a ("SAGE: Pushing 2-Bit
// Vector-Quantized LLMs toward Real-World Usability", Sec. 3.2 "Weighted
// Quantizer Fitting", initialisation details in Sec. 4.1): n sampled
// subvectors (magnitudes p and Eq. 4 weights w), K unit codewords started
// from the unit directions of K chosen samples, then rounds of
//   assignment  z_s = Eq. 6 argmax over the codewords (ties: smallest k),
//   update      c_k = normalise( sum over members s of w_s * p_s / |p_s| ),
// members in sample order; an empty cluster keeps its codeword.
//
// The arithmetic is fp64 with every product, sum, quotient and square root
// rounded on its own (no fused multiply-add) and every sum taken in the CPU
// encoder's order -- a cluster's members in increasing sample order -- so the
// codebook is bit-identical to the CPU encoder's.  Launches per round: one
// assignment kernel (a thread per sample, codebook in shared memory) and one
// update kernel (a CTA per cluster: it scans the assignments in order,
// compacts its members with warp ballots and adds their precomputed terms
// w p / |p| in that order from shared memory).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kKmThreads = 256;   // prep / init / assignment kernels
constexpr int kUpdThreads = 512;  // update kernel: samples scanned per round
constexpr size_t kKmHeader = 256; // workspace header: word 0 = the status word

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

struct KmWs {
    uint32_t* flag;
    int32_t* z;       // [n] cluster of each sample
    uint8_t* live;    // [n] |p| > 0 (zero samples add nothing to any cluster)
    double* v;        // [n][8] w p / |p|
};

KmWs km_carve(void* ws, int n) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    KmWs w;
    w.flag = reinterpret_cast<uint32_t*>(b);
    b += kKmHeader;
    w.z = reinterpret_cast<int32_t*>(b);
    b += round256((size_t)n * 4);
    w.live = b;
    b += round256((size_t)n);
    w.v = reinterpret_cast<double*>(b);
    return w;
}

// |p| of one sample: the squares summed in component order, then the root.
__device__ __forceinline__ double norm8(const double* p) {
    double nn = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) nn = __dadd_rn(nn, __dmul_rn(p[i], p[i]));
    return nn;  // squared; the caller takes the root where it is > 0
}

__global__ void __launch_bounds__(kKmThreads) kmeans_prep_kernel(int n, const double* __restrict__ P,
                                                                 const double* __restrict__ Wt,
                                                                 uint8_t* __restrict__ live, double* __restrict__ v) {
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n; s += gridDim.x * blockDim.x) {
        double p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) p[i] = P[(size_t)s * 8 + i];
        double nn = norm8(p);
        live[s] = nn > 0.0 ? 1 : 0;
        nn = nn > 0.0 ? __dsqrt_rn(nn) : 1.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[(size_t)s * 8 + i] = __ddiv_rn(__dmul_rn(Wt[(size_t)s * 8 + i], p[i]), nn);
    }
}

// Codeword k = unit direction of sample init[k] (all-zero sample: the uniform
// direction 1 / sqrt(8)).  An init entry outside [0, n) is recorded in the
// status word and sample 0 is used in its place.
__global__ void kmeans_init_kernel(int n, int K, const double* __restrict__ P, const int64_t* __restrict__ init,
                                   double* __restrict__ cb, uint32_t* flag) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    long long id = init[k];
    if (id < 0 || id >= n) {
        atomicOr(flag, kDevBadInput);
        id = 0;
    }
    const double* p = P + (size_t)id * 8;
    double nn = norm8(p);
    const bool pos = nn > 0.0;
    nn = pos ? __dsqrt_rn(nn) : 1.0;
    const double u = __ddiv_rn(1.0, __dsqrt_rn(8.0));
#pragma unroll
    for (int i = 0; i < 8; ++i) cb[k * 8 + i] = pos ? __ddiv_rn(p[i], nn) : u;
}

// Eq. 6 for every sample against the current fp64 codebook.
__global__ void __launch_bounds__(kKmThreads) kmeans_assign_kernel(int n, int K, const double* __restrict__ P,
                                                                   const double* __restrict__ Wt,
                                                                   const double* __restrict__ cbg,
                                                                   int32_t* __restrict__ z) {
    __shared__ double cb[256 * 8];
    for (int e = threadIdx.x; e < K * 8; e += blockDim.x) cb[e] = cbg[e];
    __syncthreads();
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n; s += gridDim.x * blockDim.x) {
        double p8[8], w8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            p8[i] = P[(size_t)s * 8 + i];
            w8[i] = Wt[(size_t)s * 8 + i];
        }
        int best = 0;
        double best_score = -1.0;
        for (int k = 0; k < K; ++k) {
            double num = 0.0, den = 0.0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double c = cb[k * 8 + i];
                num = __dadd_rn(num, __dmul_rn(__dmul_rn(w8[i], p8[i]), c));
                den = __dadd_rn(den, __dmul_rn(__dmul_rn(w8[i], c), c));
            }
            if (den <= 0.0) continue;
            const double score = __ddiv_rn(__dmul_rn(num, num), den);
            if (score > best_score) {
                best_score = score;
                best = k;
            }
        }
        z[s] = best_score <= 0.0 ? 0 : best;
    }
}

// Cluster blockIdx.x: the sum of its live members' terms in sample order
// (threads 0..7 hold one component each), then the normalisation.  Samples
// are scanned in chunks of kUpdChunk: the chunk's members are compacted in
// order (warp ballots and one scan of the per-warp counts), their terms
// staged in shared memory by all threads, up to kUpdVals members per round
// trip, and added in order from there; the next chunk's assignments are
// loaded while the current one is summed.
constexpr int kUpdPer = 8;                         // samples per thread and chunk
constexpr int kUpdChunk = kUpdThreads * kUpdPer;   // 4096
constexpr int kUpdVals = 1024;                     // member terms staged per round trip
constexpr int kUpdSmem = kUpdVals * 8 * 8 + kUpdChunk * 4;  // member terms + member list
static_assert((kUpdThreads / 32) * kUpdPer == 128, "the count scan takes 4 counts per lane of one warp");

__global__ void __launch_bounds__(kUpdThreads) kmeans_update_kernel(int n, const int32_t* __restrict__ z,
                                                                    const uint8_t* __restrict__ live,
                                                                    const double* __restrict__ v,
                                                                    double* __restrict__ cb) {
    constexpr int NW = kUpdThreads / 32;
    extern __shared__ __align__(16) uint8_t km_smem[];
    double* vals = reinterpret_cast<double*>(km_smem);                  // [kUpdVals][8]
    int* list = reinterpret_cast<int*>(km_smem + kUpdVals * 8 * 8);    // [kUpdChunk]
    __shared__ int wcount[NW * kUpdPer + 1];  // counts per (r, warp), then their exclusive prefix; [last] = total
    __shared__ double a[8];
    __shared__ double s_nn;
    const int k = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    double acc = 0.0;
    // sample c0 + r * kUpdThreads + tid is this thread's r-th of the chunk: (r, warp, lane) is sample order
    bool nf[kUpdPer];
#pragma unroll
    for (int r = 0; r < kUpdPer; ++r) {
        const int s = r * kUpdThreads + tid;
        nf[r] = s < n ? (live[s] != 0) & (z[s] == k) : false;  // both loads issued together
    }
    for (int c0 = 0; c0 < n; c0 += kUpdChunk) {
        bool f[kUpdPer];
        unsigned bal[kUpdPer];
#pragma unroll
        for (int r = 0; r < kUpdPer; ++r) {
            f[r] = nf[r];
            const int s = c0 + kUpdChunk + r * kUpdThreads + tid;  // the next chunk's
            nf[r] = s < n ? (live[s] != 0) & (z[s] == k) : false;
            bal[r] = __ballot_sync(0xffffffffu, f[r]);
            if (lane == 0) wcount[r * NW + w] = __popc(bal[r]);
        }
        __syncthreads();
        if (w == 0) {  // exclusive scan of the 128 counts in (r, warp) order, 4 per lane
            int c[4], sum = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                c[u] = wcount[lane * 4 + u];
                sum += c[u];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            int ex = incl - sum;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                wcount[lane * 4 + u] = ex;
                ex += c[u];
            }
            if (lane == 31) wcount[NW * kUpdPer] = incl;
        }
        __syncthreads();
        const int total = wcount[NW * kUpdPer];
#pragma unroll
        for (int r = 0; r < kUpdPer; ++r)
            if (f[r]) list[wcount[r * NW + w] + __popc(bal[r] & ((1u << lane) - 1u))] = c0 + r * kUpdThreads + tid;
        __syncthreads();
        for (int m0 = 0; m0 < total; m0 += kUpdVals) {  // uniform: every thread read the same total
            const int cnt = min(kUpdVals, total - m0);
            for (int e0 = tid; e0 < cnt * 8; e0 += 4 * kUpdThreads) {  // up to four terms in flight per thread
                double t[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + u * kUpdThreads;
                    t[u] = e < cnt * 8 ? v[(size_t)list[m0 + (e >> 3)] * 8 + (e & 7)] : 0.0;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + u * kUpdThreads;
                    if (e < cnt * 8) vals[e] = t[u];
                }
            }
            __syncthreads();
            if (tid < 8) {
                int m = 0;
                for (; m + 8 <= cnt; m += 8) {
                    double t[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) t[u] = vals[(m + u) * 8 + tid];
#pragma unroll
                    for (int u = 0; u < 8; ++u) acc = __dadd_rn(acc, t[u]);  // member order
                }
                for (; m < cnt; ++m) acc = __dadd_rn(acc, vals[m * 8 + tid]);
            }
            __syncthreads();  // the terms are rewritten next round
        }
        // the list and the counts are rewritten next chunk only after the barriers above
    }
    if (tid < 8) a[tid] = acc;
    __syncthreads();
    if (tid == 0) {
        double nn = 0.0;
        for (int i = 0; i < 8; ++i) nn = __dadd_rn(nn, __dmul_rn(a[i], a[i]));
        s_nn = nn > 0.0 ? __dsqrt_rn(nn) : 0.0;
    }
    __syncthreads();
    if (tid < 8 && s_nn > 0.0) cb[k * 8 + tid] = __ddiv_rn(a[tid], s_nn);  // empty cluster: unchanged
}

__global__ void kmeans_half_kernel(int n, const double* __restrict__ cb, uint16_t* __restrict__ cb16) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < n) cb16[e] = __half_as_ushort(__double2half(cb[e]));  // nearest even
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" size_t sage_kmeans_workspace_size(int n) {
    if (n < 1 || n > (1 << 30)) return 0;
    return kKmHeader + round256((size_t)n * 4) + round256((size_t)n) + (size_t)n * 64;
}

extern "C" int sage_kmeans(int n, int log2K, const double* P, const double* Wt, const int64_t* init, int iters,
                           double* cb, uint16_t* cb16, void* ws, size_t ws_bytes, sage_stream_t stream) {
    if (!P || !Wt || !init || !cb) return SAGE_ERR_INVALID_ARGUMENT;
    if (n < 1 || n > (1 << 30) || iters < 0 || log2K < 4 || log2K > 8) return SAGE_ERR_UNSUPPORTED;
    if (!ws) return SAGE_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % 16) return SAGE_ERR_MISALIGNED;
    if (ws_bytes < sage_kmeans_workspace_size(n)) return SAGE_ERR_WORKSPACE;
    const int K = 1 << log2K;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const KmWs w = km_carve(ws, n);
    const int sm = current_sm_count();
    const int grid = (int)std::max<long long>(1, std::min<long long>((n + kKmThreads - 1) / kKmThreads, 8LL * sm));
    static bool smem_set[64] = {};  // per device: the update kernel's dynamic shared memory opt-in
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return SAGE_ERR_CUDA;
    if (!smem_set[dev]) {
        if (cudaFuncSetAttribute(kmeans_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUpdSmem) !=
            cudaSuccess)
            return SAGE_ERR_CUDA;
        smem_set[dev] = true;
    }
    kmeans_prep_kernel<<<grid, kKmThreads, 0, s>>>(n, P, Wt, w.live, w.v);
    kmeans_init_kernel<<<(K + 63) / 64, 64, 0, s>>>(n, K, P, init, cb, w.flag);
    for (int it = 0; it < iters; ++it) {
        kmeans_assign_kernel<<<grid, kKmThreads, 0, s>>>(n, K, P, Wt, cb, w.z);
        kmeans_update_kernel<<<K, kUpdThreads, kUpdSmem, s>>>(n, w.z, w.live, w.v, cb);
    }
    if (cb16) kmeans_half_kernel<<<(K * 8 + 255) / 256, 256, 0, s>>>(K * 8, cb, cb16);
    return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
