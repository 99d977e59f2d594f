// Test hooks and small helper kernels of libsage (sm_100a):
//  * sage_dequant        -- fp16 reconstruction of W (Eq. 1-2 of the SAGE paper)
//                           with the decode primitives the GEMV/GEMM kernels use;
//  * sage_unpack_device  -- bit-exact extraction of the logical fields;
//  * sage_permute_x      -- the prefill activation reorder x_perm = x[:, perm]
//                           (Sec. 3.5, "reorders activations once per projection");
//  * status word readback.
#include <cuda_runtime.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
using namespace dev;

namespace {

// One thread per (subvector column j, row octet b): decodes the 8 rows of the record.
template <int V>
__global__ void dequant_kernel(sage_matrix A, uint16_t* W) {
    using F = Fmt<V>;
    const int R8 = (A.d_out + 7) >> 3, S = A.d_in >> 3, G = A.d_in >> 7;
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (long long)R8 * S) return;
    const int b = (int)(id % R8), j = (int)(id / R8);
    const int blk = b >> 5, ob = b & 31;
    const uint4 rec = __ldg(reinterpret_cast<const uint4*>(A.main + main_word(R8, S, blk, j, ob, 0)));
    const uint32_t wv[4] = {rec.x, rec.y, rec.z, rec.w};
    const uint4* cb = reinterpret_cast<const uint4*>(A.codebook);
    const int g = j >> 4, t = j & 15;
    for (int u = 0; u < 4; ++u) {
        for (int half = 0; half < 2; ++half) {
            const int row = b * 8 + 2 * u + half;
            if (row >= A.d_out) continue;
            const uint2 e = __ldg(reinterpret_cast<const uint2*>(A.meta) + meta_entry(R8, G, blk, g, ob, 2 * u + half));
            const float2 md = __half22float2(u2h2(e.y));
            const float dl = md.y * (float)(1 << V), mp = md.x - dl;
            const uint32_t wa = wv[u];
            const uint32_t wf = half ? rot16(wa) : wa;  // field word (z, q) of this row
            uint4 c = __ldg(cb + (((wf & F::kZMask) >> 7)));
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
            const float r = fmaf(q_unit<V>(wf), dl, mp);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            uint32_t o[4];
            for (int k = 0; k < 4; ++k) {
                const float2 cf = __half22float2(u2h2(cw[k]));
                o[k] = h22u(__floats2half2_rn(r * cf.x, r * cf.y));
            }
            *reinterpret_cast<uint4*>(W + (size_t)row * A.d_in + (size_t)j * 8) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

template <int V>
__global__ void unpack_kernel(sage_matrix A, uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu,
                              uint16_t* delta) {
    using F = Fmt<V>;
    const int R8 = (A.d_out + 7) >> 3, S = A.d_in >> 3, G = A.d_in >> 7;
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (long long)A.d_out * S) return;
    const int row = (int)(id / S), j = (int)(id % S);
    const int b = row >> 3, t8 = row & 7, u = t8 >> 1, half = t8 & 1;
    const int blk = b >> 5, ob = b & 31;
    const uint32_t wa = __ldg(A.main + main_word(R8, S, blk, j, ob, u));
    const uint2 e = __ldg(reinterpret_cast<const uint2*>(A.meta) + meta_entry(R8, G, blk, j >> 4, ob, t8));
    const uint32_t wf = half ? rot16(wa) : wa;
    const uint32_t z = (wf & F::kZMask) >> 7;
    const uint32_t qq = (wf & F::kQMask) >> (23 - V);
    uint32_t m0, m1, m2;
    if (!half) { m0 = slot_mask<F::slot(0)>(wa); m1 = slot_mask<F::slot(1)>(wa); m2 = slot_mask<F::slot(2)>(wa); }
    else       { m0 = slot_mask<F::slot(3)>(wa); m1 = slot_mask<F::slot(4)>(wa); m2 = slot_mask<F::slot(5)>(wa); }
    const uint32_t m3 = aux_mask(e.x, j & 15);
    // half2 sign masks (bits 15 / 31) back to the sign byte (bit i = component i)
    const uint32_t s = ((m0 >> 15) & 1) | ((m0 >> 30) & 2) | (((m1 >> 15) & 1) << 2) | (((m1 >> 31) & 1) << 3) |
                       (((m2 >> 15) & 1) << 4) | (((m2 >> 31) & 1) << 5) | (((m3 >> 15) & 1) << 6) |
                       (((m3 >> 31) & 1) << 7);
    signs[id] = (uint8_t)s;
    idx[id] = (uint16_t)z;
    q[id] = (uint8_t)qq;
    if ((j & 15) == 0) {
        mu[(size_t)row * G + (j >> 4)] = (uint16_t)(e.y & 0xffff);
        delta[(size_t)row * G + (j >> 4)] = (uint16_t)(e.y >> 16);
    }
}

__global__ void permute_kernel(const uint16_t* x, const int32_t* perm, int M, int d_in, uint16_t* xp) {
    pdl_wait();
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int n8 = d_in >> 3;
    if (id < (long long)M * n8) {
        const int m = (int)(id / n8), c0 = (int)(id % n8) * 8;
        const uint16_t* xr = x + (size_t)m * d_in;
        uint4 o;
        if (perm) {
            const int4 pa = __ldg(reinterpret_cast<const int4*>(perm + c0));
            const int4 pb = __ldg(reinterpret_cast<const int4*>(perm + c0 + 4));
            o.x = (uint32_t)xr[pa.x] | ((uint32_t)xr[pa.y] << 16);
            o.y = (uint32_t)xr[pa.z] | ((uint32_t)xr[pa.w] << 16);
            o.z = (uint32_t)xr[pb.x] | ((uint32_t)xr[pb.y] << 16);
            o.w = (uint32_t)xr[pb.z] | ((uint32_t)xr[pb.w] << 16);
        } else {
            o = *reinterpret_cast<const uint4*>(xr + c0);
        }
        *reinterpret_cast<uint4*>(xp + (size_t)m * d_in + c0) = o;
    }
    pdl_launch_dependents();
}

inline int ok(cudaError_t e) { return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

}  // namespace

int launch_dequant(const sage_matrix* A, uint16_t* W, sage_stream_t stream) {
    const long long n = (long long)((A->d_out + 7) / 8) * (A->d_in / 8);
    const int bs = 256;
    const unsigned grid = (unsigned)((n + bs - 1) / bs);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (A->log2K) {
        case 4: dequant_kernel<6><<<grid, bs, 0, s>>>(*A, W); break;
        case 5: dequant_kernel<5><<<grid, bs, 0, s>>>(*A, W); break;
        case 6: dequant_kernel<4><<<grid, bs, 0, s>>>(*A, W); break;
        case 7: dequant_kernel<3><<<grid, bs, 0, s>>>(*A, W); break;
        default: dequant_kernel<2><<<grid, bs, 0, s>>>(*A, W); break;
    }
    return ok(cudaGetLastError());
}

int launch_unpack(const sage_matrix* A, uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu, uint16_t* delta,
                  sage_stream_t stream) {
    const long long n = (long long)A->d_out * (A->d_in / 8);
    const int bs = 256;
    const unsigned grid = (unsigned)((n + bs - 1) / bs);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (A->log2K) {
        case 4: unpack_kernel<6><<<grid, bs, 0, s>>>(*A, signs, idx, q, mu, delta); break;
        case 5: unpack_kernel<5><<<grid, bs, 0, s>>>(*A, signs, idx, q, mu, delta); break;
        case 6: unpack_kernel<4><<<grid, bs, 0, s>>>(*A, signs, idx, q, mu, delta); break;
        case 7: unpack_kernel<3><<<grid, bs, 0, s>>>(*A, signs, idx, q, mu, delta); break;
        default: unpack_kernel<2><<<grid, bs, 0, s>>>(*A, signs, idx, q, mu, delta); break;
    }
    return ok(cudaGetLastError());
}

int launch_permute(const uint16_t* x, const int32_t* perm, int M, int d_in, uint16_t* xp, sage_stream_t stream) {
    const long long n = (long long)M * (d_in / 8);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return ok(cudaLaunchKernelEx(&cfg, permute_kernel, x, perm, M, d_in, xp));
}

int read_and_clear_status(void* ws, sage_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SAGE_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SAGE_ERR_CUDA;
    if (v == 0) return SAGE_OK;
    if (cudaMemset(ws, 0, sizeof(v)) != cudaSuccess) return SAGE_ERR_CUDA;
    if (v & kDevTimeout) return SAGE_ERR_TIMEOUT;
    if (v & kDevBadInput) return SAGE_ERR_INVALID_ARGUMENT;
    return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
