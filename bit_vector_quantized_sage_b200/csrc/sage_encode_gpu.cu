// The encoder's per-row stage on sm_100a (Sec. 3.1-3.2 of "SAGE: Pushing
// 2-Bit Vector-Quantized LLMs toward Real-World Usability"): for a given
// stored codebook, the signs of every subvector, its Eq. 6 direction (the
// codeword maximising the omega-weighted cosine score) and fitted radius,
// the Eq. 14 grid of every row group of 16 and the Eq. 2 radius codes.
//
// The arithmetic is fp64 with every product, sum and quotient rounded on
// its own (no fused multiply-add), in the order of the CPU encoder, so the
// fields are bit-identical to the CPU encoder's for the same codebook,
// permutation and Eq. 4 weights.  One persistent grid; each CTA holds the
// codebook in fp64 in shared memory and gives 16 threads to a row group
// (one subvector each); the group's radius range is a 16-lane shuffle
// reduction.  sage_pack_device then writes the packed planes from the fields
// on the device, word for word what the host packer writes.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kEncThreads = 256;

__global__ void __launch_bounds__(kEncThreads) encode_rows_kernel(int d_out, int d_in, int log2K,
                                                                  const double* __restrict__ W,
                                                                  const int32_t* __restrict__ perm,
                                                                  const double* __restrict__ omega,
                                                                  const uint16_t* __restrict__ codebook,
                                                                  uint8_t* __restrict__ signs, uint16_t* __restrict__ idx,
                                                                  uint8_t* __restrict__ q, uint16_t* __restrict__ mu,
                                                                  uint16_t* __restrict__ delta) {
    __shared__ double cb[256 * 8];
    const int K = 1 << log2K, V = 10 - log2K, S = d_in >> 3, G = d_in >> 7;
    for (int e = threadIdx.x; e < K * 8; e += blockDim.x)
        cb[e] = (double)__half2float(__ushort_as_half(codebook[e]));  // fp16 -> fp64 is exact
    __syncthreads();
    const int t = threadIdx.x & 15;
    const double top = (double)((1 << V) - 1);
    const long long groups = (long long)d_out * G;
    for (long long gidx = (long long)blockIdx.x * (kEncThreads / 16) + (threadIdx.x >> 4); gidx < groups;
         gidx += (long long)gridDim.x * (kEncThreads / 16)) {
        const int o = (int)(gidx / G), g = (int)(gidx - (long long)o * G);
        const int j = g * 16 + t;
        double p8[8], w8[8];
        uint32_t s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double w = W[(size_t)o * d_in + perm[j * 8 + i]];
            p8[i] = fabs(w);
            if (w < 0.0) s |= 1u << i;
            w8[i] = omega[j * 8 + i];
        }
        // Eq. 6: score_k = (sum w p c)^2 / sum w c^2, ties to the smallest k;
        // an all-zero score gives k = 0, r* = 0
        int best = 0;
        double best_score = -1.0, best_r = 0.0;
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
                best_r = __ddiv_rn(num, den);
            }
        }
        if (best_score <= 0.0) {
            best = 0;
            best_r = 0.0;
        }
        const size_t e = (size_t)o * S + j;
        signs[e] = (uint8_t)s;
        idx[e] = (uint16_t)best;
        // Eq. 14 over the group's 16 fitted radii, stored as fp16 (round to nearest even)
        double lo = best_r, hi = best_r;
#pragma unroll
        for (int m = 8; m; m >>= 1) {  // the group's 16 lanes (an aligned half warp)
            lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, m, 16));
            hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, m, 16));
        }
        const __half mu16 = __double2half(lo);
        const __half dl16 = __double2half(__ddiv_rn(__dsub_rn(hi, lo), top));
        if (t == 0) {
            mu[(size_t)o * G + g] = __half_as_ushort(mu16);
            delta[(size_t)o * G + g] = __half_as_ushort(dl16);
        }
        // Eq. 2 against the stored grid; delta = 0 gives q = 0
        const double mud = (double)__half2float(mu16), dd = (double)__half2float(dl16);
        double qq = 0.0;
        if (dd > 0.0) {
            qq = floor(__dadd_rn(__ddiv_rn(__dsub_rn(best_r, mud), dd), 0.5));
            qq = fmin(fmax(qq, 0.0), top);
        }
        q[e] = (uint8_t)qq;
    }
}

// Packed format v2 on the device (the host packer's layout): blocks of 32
// row octets stored contiguously, subvector-column major inside a block.
__device__ __forceinline__ int pk_octets(int R8, int blk) { return min(32, R8 - blk * 32); }

// One thread per 16-byte main record word (octet b, column j, word u): word u
// holds rows 2u (row A) and 2u + 1 (row B) of the octet.  Row A: z at bits
// 7.., q at bits 23 - V..; row B: z at bits 23.., q at bits 7 - V..; sign
// bits 0-5 of row A / B in the three slot pairs (p, p + 16) of its half.
__global__ void pack_main_kernel(int d_out, int S, int log2K, const uint8_t* __restrict__ signs,
                                 const uint16_t* __restrict__ idx, const uint8_t* __restrict__ q,
                                 uint32_t* __restrict__ main_out) {
    const int V = 10 - log2K, R8 = (d_out + 7) >> 3;
    const uint32_t zm = (1u << log2K) - 1u, qm = (1u << V) - 1u;
    const long long total = (long long)R8 * S * 4;
    for (long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x; id < total;
         id += (long long)gridDim.x * blockDim.x) {
        const int u = (int)(id & 3);
        const long long r = id >> 2;            // record: block-major, then column, then octet
        const int blk = (int)(r / ((long long)S * 32));
        const int nB = pk_octets(R8, blk);
        const long long in_blk = r - (long long)blk * S * 32;
        const int j = (int)(in_blk / nB), ob = (int)(in_blk - (long long)j * nB);
        if (j >= S) continue;  // the last block is shorter: no record there
        uint32_t w = 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int o = (blk * 32 + ob) * 8 + 2 * u + half;
            if (o >= d_out) continue;
            const size_t e = (size_t)o * S + j;
            const uint32_t z = idx[e] & zm, qq = q[e] & qm, sb = signs[e];
            w |= half ? (z << 23) | (qq << (7 - V)) : (z << 7) | (qq << (23 - V));
#pragma unroll
            for (int n = 0; n < 3; ++n) {
                const int k = n + 3 * half;  // sign slots {0 .. 6 - V} then {17 - V .. 15}
                const int pos = k <= 6 - V ? k : (17 - V) + (k - (7 - V));
                w |= ((sb >> (2 * n)) & 1u) << pos;
                w |= ((sb >> (2 * n + 1)) & 1u) << (pos + 16);
            }
        }
        main_out[(size_t)blk * S * 128 + ((size_t)j * nB + ob) * 4 + u] = w;
    }
}

// One thread per 8-byte meta entry (octet b, group g, row t): the group's 16
// sign bits 6 (bits 0-15) and 7 (bits 16-31) of row 8b + t, then mu | delta << 16.
__global__ void pack_meta_kernel(int d_out, int S, int G, const uint8_t* __restrict__ signs,
                                 const uint16_t* __restrict__ mu, const uint16_t* __restrict__ delta,
                                 uint2* __restrict__ meta_out) {
    const int R8 = (d_out + 7) >> 3;
    const long long total = (long long)R8 * G * 8;
    for (long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x; id < total;
         id += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(id & 7);
        const long long r = id >> 3;
        const int blk = (int)(r / ((long long)G * 32));
        const int nB = pk_octets(R8, blk);
        const long long in_blk = r - (long long)blk * G * 32;
        const int g = (int)(in_blk / nB), ob = (int)(in_blk - (long long)g * nB);
        if (g >= G) continue;
        const int o = (blk * 32 + ob) * 8 + t;
        uint2 m = make_uint2(0u, 0u);
        if (o < d_out) {
            const uint8_t* sr = signs + (size_t)o * S + g * 16;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const uint32_t sb = sr[jj];
                m.x |= ((sb >> 6) & 1u) << jj;
                m.x |= ((sb >> 7) & 1u) << (jj + 16);
            }
            m.y = (uint32_t)mu[(size_t)o * G + g] | ((uint32_t)delta[(size_t)o * G + g] << 16);
        }
        meta_out[(size_t)blk * G * 256 + ((size_t)g * nB + ob) * 8 + t] = m;
    }
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" int sage_pack_device(int d_out, int d_in, int log2K, const uint8_t* signs, const uint16_t* idx,
                                const uint8_t* q, const uint16_t* mu, const uint16_t* delta, uint32_t* main_out,
                                uint32_t* meta_out, sage_stream_t stream) {
    if (!signs || !idx || !q || !mu || !delta || !main_out || !meta_out) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return SAGE_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(meta_out) % 8 || reinterpret_cast<uintptr_t>(main_out) % 4)
        return SAGE_ERR_MISALIGNED;
    const int S = d_in / 8, G = d_in / 128;
    const long long R8 = (d_out + 7) / 8;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int cap = 8 * current_sm_count();
    const long long nm = R8 * S * 4, nt = R8 * G * 8;
    pack_main_kernel<<<(int)std::max<long long>(1, std::min<long long>((nm + 255) / 256, cap)), 256, 0, s>>>(
        d_out, S, log2K, signs, idx, q, main_out);
    pack_meta_kernel<<<(int)std::max<long long>(1, std::min<long long>((nt + 255) / 256, cap)), 256, 0, s>>>(
        d_out, S, G, signs, mu, delta, reinterpret_cast<uint2*>(meta_out));
    return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

extern "C" int sage_encode_rows(int d_out, int d_in, int log2K, const double* W, const int32_t* perm,
                                const double* omega, const uint16_t* codebook, uint8_t* signs, uint16_t* idx,
                                uint8_t* q, uint16_t* mu, uint16_t* delta, sage_stream_t stream) {
    if (!W || !perm || !omega || !codebook || !signs || !idx || !q || !mu || !delta) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return SAGE_ERR_UNSUPPORTED;
    const long long groups = (long long)d_out * (d_in / 128);
    const long long need = (groups + kEncThreads / 16 - 1) / (kEncThreads / 16);
    const int grid = (int)std::max<long long>(1, std::min<long long>(need, 4LL * current_sm_count()));
    encode_rows_kernel<<<grid, kEncThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        d_out, d_in, log2K, W, perm, omega, codebook, signs, idx, q, mu, delta);
    return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
