// Tensor-core path of the packed SAGE layer for batch M >= 9 on sm_100a
// (the prefill GEMM of Sec. 3.5 / App. A.1 of "SAGE: Pushing 2-Bit
// Vector-Quantized LLMs toward Real-World Usability": W_hat tiles are
// reconstructed into shared memory and multiplied there, so the decode is
// amortised over the whole batch).
//
//   y[m][o] = sum_p W_hat[o][p] x_perm[m][p],  M <= 256.
//
// Two kernels per call:
//  * tile_x_kernel writes x_perm (Sec. 3.5: the activations are reordered once
//    per projection) straight into the tcgen05 K-major operand layout, zero
//    padded to N = M rounded up to 16, so every 64-column slab of it is one
//    contiguous bulk copy.
//  * gemm_kernel: one CTA per (256-row block, part of the input columns).  A
//    copy warp bulk-copies the block's packed chunks (16 subvector columns =
//    one radius group) and the x_perm slabs; eight decode warps rebuild each
//    64-column slab of W_hat (Eq. 1-2: r_hat (s (.) c_z), r_hat = mu + q delta,
//    rounded to fp16) into shared memory; one thread issues tcgen05.mma
//    (kind::f16, M = 128, N, K = 16) for the two 128-row halves into two fp32
//    accumulators in tensor memory and commits to an mbarrier that frees the
//    slab's buffers.  The epilogue reads the accumulators with tcgen05.ld.
//    A block split over several CTAs is combined deterministically: every part
//    stores fp32 partial sums and the last part to arrive adds them in order.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
using namespace dev;

namespace {

constexpr int kGW = 16;                       // decode warps: two per (slab column, record half)
constexpr int kGThreads = (kGW + 4) * 32;     // + code copy warp, two MMA warps, x_perm copy warp
constexpr int kGDecodeThreads = kGW * 32;
constexpr int kGOct = 32;                     // row octets per block
constexpr int kGChunkJ = 16;                  // subvector columns per chunk (one radius group)
constexpr int kGSlabJ = 8;                    // subvector columns per MMA slab (64 input channels)
constexpr int kGCodeSlot = kGChunkJ * kGOct * 16 + kGOct * 64;  // records + meta of one chunk
constexpr int kGCodeSlots = 4;
constexpr int kASbo = 1024;                   // bytes between 8-row core-matrix groups of A
constexpr int kAHalf = 16 * kASbo;            // one 128-row half of an A slab
constexpr int kASlab = 2 * kAHalf;            // 256 rows x 64 channels, fp16
constexpr int kBSbo = 1024;                   // B: 8 core matrices of 8 rows x 16 bytes per 8 batch rows

// ------------------------------------------------------------------------
// tcgen05 / TMEM primitives (PTX ISA, sm_100a).
// ------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives (once) on the mbarrier when every MMA this thread issued so far is complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, K-major, no swizzle: core matrices of
// 8 rows x 16 bytes; lbo = bytes between the two K-adjacent core matrices of
// one MMA, sbo = bytes between 8-row groups.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);  // descriptor version 1
}
// Instruction descriptor of kind::f16: fp32 D, fp16 A and B, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void gflag(uint32_t* status, uint32_t bits) { atomicOr(status, bits); }

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory offset in the CTA of the cluster with the given rank.
__device__ __forceinline__ uint32_t map_cluster(uint32_t addr, int rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_cluster_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Set when a bounded wait of the CTA gives up; later waits then return at once.
__shared__ int s_gabort;

__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, uint32_t* status) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_test(bar, parity)) return true;
        if (i > 2048) {
            if (*reinterpret_cast<volatile int*>(&s_gabort)) return false;
            __nanosleep(64);
        }
    }
    *reinterpret_cast<volatile int*>(&s_gabort) = 1;
    gflag(status, kDevTimeout);
    return false;
}

// ------------------------------------------------------------------------
// x_perm in the B-operand layout: slab s (input channels 64s .. 64s+63) is
// [n / 8][kb = 0..7][n % 8] x 16 bytes, 16 bytes = channels 64s + 8kb .. +7
// of batch row n; rows n >= M are zero.
// ------------------------------------------------------------------------
__global__ void tile_x_kernel(const uint16_t* x, const int32_t* perm, int M, int n_pad, int d_in, uint4* xt) {
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long per_slab = (long long)n_pad * 8;
    if (id >= per_slab * (d_in / 64)) return;
    const int s = (int)(id / per_slab);
    const int w = (int)(id - (long long)s * per_slab);
    const int ng = w >> 6, kb = (w >> 3) & 7, r = w & 7;
    const int n = ng * 8 + r, k0 = s * 64 + kb * 8;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (n < M) {
        const uint16_t* xr = x + (size_t)n * d_in;
        if (perm) {
            const int4 pa = __ldg(reinterpret_cast<const int4*>(perm + k0));
            const int4 pb = __ldg(reinterpret_cast<const int4*>(perm + k0 + 4));
            o.x = (uint32_t)xr[pa.x] | ((uint32_t)xr[pa.y] << 16);
            o.y = (uint32_t)xr[pa.z] | ((uint32_t)xr[pa.w] << 16);
            o.z = (uint32_t)xr[pb.x] | ((uint32_t)xr[pb.y] << 16);
            o.w = (uint32_t)xr[pb.z] | ((uint32_t)xr[pb.w] << 16);
        } else {
            o = *reinterpret_cast<const uint4*>(xr + k0);
        }
    }
    xt[id] = o;
}

struct GemmParams {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const uint4* xt;        // x_perm in the B-operand layout (tile_x_kernel)
    uint16_t* y;            // [M][d_out]
    uint32_t* status;
    int d_out, d_in, log2K, M;
    int n_pad;              // M rounded up to 16: the MMA's N
    int n_alloc;            // TMEM columns per accumulator (power of two >= max(32, n_pad))
    int parts;              // CTAs per block (split over the input columns), one cluster
    int red_cols;           // batch columns per round of the cluster reduction
    int b_slots;            // x_perm slabs in flight
    int a_slots;            // decoded W_hat slabs in flight (2 .. kMaxASlots)
};

struct GemmSmem {
    uint32_t cb0, cbraw, code0, a0, b0;
    uint32_t b_bytes;
    uint64_t* bars;
    uint32_t* taddr_slot;
    int* bcast;
    __device__ uint64_t* code_full(int t) const { return bars + (t % kGCodeSlots); }
    __device__ uint64_t* code_empty(int t) const { return bars + kGCodeSlots + (t % kGCodeSlots); }
    __device__ uint64_t* cb_full() const { return bars + 2 * kGCodeSlots; }
    __device__ uint64_t* b_full(int s, int nb) const { return bars + 2 * kGCodeSlots + 1 + (s % nb); }
    __device__ uint64_t* mma_done(int s, int nb) const { return bars + 2 * kGCodeSlots + 1 + 8 + (s % nb); }
    __device__ uint64_t* a_full(int s, int na) const { return bars + 2 * kGCodeSlots + 1 + 16 + (s % na); }
    // the same by ring slot (the loops carry slot and phase instead of dividing)
    __device__ uint64_t* b_full_at(int k) const { return bars + 2 * kGCodeSlots + 1 + k; }
    __device__ uint64_t* mma_done_at(int k) const { return bars + 2 * kGCodeSlots + 1 + 8 + k; }
    __device__ uint64_t* a_full_at(int k) const { return bars + 2 * kGCodeSlots + 1 + 16 + k; }
};

constexpr int kMaxASlots = 4;
__host__ __device__ inline int gemm_smem_bytes(int K, int n_pad, int a_slots, int b_slots) {
    return K * 128 + K * 16 + kGCodeSlots * kGCodeSlot + a_slots * kASlab + b_slots * n_pad * 128 +
           (2 * kGCodeSlots + 1 + 16 + kMaxASlots) * 8 + 64;
}

// Rebuilds one subvector of one row (Eq. 1-2), rounded to fp16: w is the
// record word holding the row, odd selects the row's half of it (rows 2u and
// 2u + 1 share word u), s0..s2 are the row's sign-slot shifts, and the aux
// signs come from the row's group word at bit `col`.  The codeword load may be
// reordered by the compiler (cbsel carries the caller's order token).
__device__ __forceinline__ uint4 decode_sv(const VDec& d, uint32_t w, bool odd, uint32_t s0, uint32_t s1,
                                           uint32_t s2, uint32_t aux, uint32_t sh_aux, float mp, float dl,
                                           uint32_t cbsel) {
    const uint32_t wf = odd ? rot16(w) : w;  // (z, q) field word of this row
    uint4 c = lds128_r(cbsel + (wf & d.zmask));
    c.x ^= (w << s0) & 0x80008000u;
    c.y ^= (w << s1) & 0x80008000u;
    c.z ^= (w << s2) & 0x80008000u;
    c.w ^= (aux << sh_aux) & 0x80008000u;
    const float r = fmaf(__uint_as_float((wf & d.qmask) | 0x3F800000u), dl, mp);
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 cf = __half22float2(u2h2(cw[k]));
        o[k] = h22u(__floats2half2_rn(r * cf.x, r * cf.y));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(kGThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int blk = blockIdx.x / p.parts, part = blockIdx.x - blk * p.parts;
    const int R8 = (p.d_out + 7) >> 3, S = p.d_in >> 3, G = p.d_in >> 7;
    const int n_oct = block_octets(R8, blk);
    const int g0 = part * G / p.parts, g1 = (part + 1) * G / p.parts;
    const int n_chunk = g1 - g0, n_slab = 2 * n_chunk;
    const int K = 1 << p.log2K, NB = p.b_slots, NA = p.a_slots;

    GemmSmem sm;
    {
        uint8_t* q = smem_raw;
        sm.cb0 = smem_u32(q); q += K * 128;
        sm.cbraw = smem_u32(q); q += K * 16;
        sm.code0 = smem_u32(q); q += kGCodeSlots * kGCodeSlot;
        sm.a0 = smem_u32(q); q += NA * kASlab;
        sm.b_bytes = (uint32_t)p.n_pad * 128;
        sm.b0 = smem_u32(q); q += NB * sm.b_bytes;
        sm.bars = reinterpret_cast<uint64_t*>(q); q += (2 * kGCodeSlots + 1 + 16 + kMaxASlots) * 8;
        sm.taddr_slot = reinterpret_cast<uint32_t*>(q); q += 16;
        sm.bcast = reinterpret_cast<int*>(q);
    }
    if (tid == 0) {
        for (int k = 0; k < kGCodeSlots; ++k) {
            mbar_init(sm.code_full(k), 1);
            mbar_init(sm.code_empty(k), kGW);
        }
        mbar_init(sm.cb_full(), 1);
        for (int k = 0; k < 8; ++k) {
            mbar_init(sm.bars + 2 * kGCodeSlots + 1 + k, 1);      // b_full
            mbar_init(sm.bars + 2 * kGCodeSlots + 1 + 8 + k, 2);  // mma_done: a commit from each MMA warp
        }
        for (int k = 0; k < kMaxASlots; ++k) mbar_init(sm.a_full(k, kMaxASlots), kGW);  // one arrival per decode warp
        fence_mbar_init();
        s_gabort = 0;
    }
    const uint32_t tcols = 2u * (uint32_t)p.n_alloc;
    if (warp == 0) {
        tmem_alloc(smem_u32(sm.taddr_slot), tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = *sm.taddr_slot;

    bool wait_last = false;
    if (warp == kGW) {
        // ---------------- copy warp ----------------
        if (lane == 0) {
            mbar_arrive_expect_tx(sm.cb_full(), (uint32_t)K * 16);
            bulk_g2s(sm.cbraw, p.cb, (uint32_t)K * 16, sm.cb_full());
            const uint32_t mb = (uint32_t)(kGChunkJ * n_oct * 16), tb = (uint32_t)(n_oct * 64);
            for (int t = 0; t < n_chunk; ++t) {
                if (t >= kGCodeSlots) gwait(sm.code_empty(t), ((t / kGCodeSlots) - 1) & 1, p.status);
                const int g = g0 + t;
                const uint32_t dst = sm.code0 + (uint32_t)(t % kGCodeSlots) * kGCodeSlot;
                mbar_arrive_expect_tx(sm.code_full(t), mb + tb);
                bulk_g2s(dst, p.main + main_word(R8, S, blk, g * kGChunkJ, 0, 0), mb, sm.code_full(t));
                bulk_g2s(dst + kGChunkJ * kGOct * 16, p.meta + 2 * meta_entry(R8, G, blk, g, 0, 0), tb,
                         sm.code_full(t));
            }
        }
    } else if (warp == kGW + 2) {
        // ---------------- x_perm copy warp ----------------
        // Its own warp, so that a slab's wait for its buffer (the MMAs of slab
        // s - NB) never holds back the code copies, and the reverse.
        if (lane == 0) {
            int bs = 0, bph = 0;  // slab s's buffer slot and the parity of its fill
            for (int s = 0; s < n_slab; ++s) {
                if (s >= NB) gwait(sm.mma_done_at(bs), bph ^ 1, p.status);  // the MMAs of slab s - NB
                mbar_arrive_expect_tx(sm.b_full_at(bs), sm.b_bytes);
                bulk_g2s(sm.b0 + (uint32_t)bs * sm.b_bytes, p.xt + (size_t)(2 * g0 + s) * p.n_pad * 8, sm.b_bytes,
                         sm.b_full_at(bs));
                if (++bs == NB) { bs = 0; bph ^= 1; }
            }
            // no exit while copies are in flight: the MMAs of the last slabs consumed them
            for (int s = max(0, n_slab - NB); s < n_slab; ++s) gwait(sm.b_full(s, NB), (s / NB) & 1, p.status);
        }
    } else if (warp == kGW + 1 || warp == kGW + 3) {
        // ---------------- MMA warps: one thread each issues the tensor-core work ----------------
        // of one 128-row half of the block (its own accumulator); the two warps
        // sit on different schedulers and issue in parallel.
        const int hf = warp == kGW + 1 ? 0 : 1;
        if (lane == 0) {
            // This thread shares its scheduler with four busy decode warps, so
            // its loop is kept short: ring slots and phases are carried, not
            // divided out, and the operand descriptors are the slab base
            // descriptor plus the tile's offset in 16-byte units (the address
            // field cannot carry: shared addresses stay below 2^18).
            const uint32_t idesc = idesc_f16(p.n_pad);
            const uint64_t a_desc0 = smem_desc(sm.a0, 128, kASbo), b_desc0 = smem_desc(sm.b0, 128, kBSbo);
            int as = 0, aph = 0, bs = 0, bph = 0;
            for (int s = 0; s < n_slab; ++s) {
                gwait(sm.a_full_at(as), aph, p.status);
                gwait(sm.b_full_at(bs), bph, p.status);
                tc_fence_after();
                const uint64_t ad = a_desc0 + (uint64_t)((uint32_t)as * (kASlab >> 4));
                const uint64_t bd = b_desc0 + (uint64_t)((uint32_t)bs * (sm.b_bytes >> 4));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(taddr + (uint32_t)(hf * p.n_alloc), ad + (uint64_t)((hf * kAHalf + kk * 256) >> 4),
                            bd + (uint64_t)((kk * 256) >> 4), idesc, (s > 0 || kk > 0) ? 1u : 0u);
                mma_commit(sm.mma_done_at(bs));
                if (++as == NA) { as = 0; aph ^= 1; }
                if (++bs == NB) { bs = 0; bph ^= 1; }
            }
        }
    } else {
        // ---------------- decode warps ----------------
        gwait(sm.cb_full(), 0, p.status);
        for (int e = tid; e < K * 8; e += kGDecodeThreads) sts128(sm.cb0 + e * 16, lds128(sm.cbraw + (e >> 3) * 16));
        named_barrier(1, kGDecodeThreads);
        const VDec d = vdec(p.log2K);
        // Thread <-> one row of the block: rows 32 (warp % 8) + lane; warps 0-7
        // and 8-15 take slab columns 0-3 and 4-7.  The 8 lanes of a quarter warp
        // hold the 8 rows of one octet, so their 16-byte stores land in 8
        // different bank groups and their codeword loads hit 8 different replicas.
        const int r = 32 * (warp & 7) + lane, o = r >> 3, tr = r & 7;
        const int cw = warp >> 3;
        const bool odd = tr & 1;
        const bool active = o < n_oct;
        const int oc = active ? o : 0;  // a row octet that exists: inactive rows decode it and store zeros
        const uint32_t cbsel = sm.cb0 + ((uint32_t)tr << 4);
        const uint32_t s0 = odd ? d.sh3 : d.sh0, s1 = odd ? d.sh4 : d.sh1, s2 = odd ? d.sh5 : d.sh2;
        const uint32_t a_row = (uint32_t)(r >> 7) * kAHalf + (uint32_t)((r & 127) >> 3) * kASbo + (uint32_t)tr * 16;
        int as = 0;                  // slab s's A slot (s mod NA)
        int ms = 0, mph = 0;         // slab s - NA's mma_done slot and parity (over NB)
        for (int t = 0; t < n_chunk; ++t) {
            gwait(sm.code_full(t), (t / kGCodeSlots) & 1, p.status);
            const uint32_t slot = sm.code0 + (uint32_t)(t % kGCodeSlots) * kGCodeSlot;
            uint32_t aux = 0;
            float mp = 0.f, dl = 0.f;
            if (active) {  // this row's group entry: aux signs, mu, delta
                const uint2 e = lds64(slot + kGChunkJ * kGOct * 16 + (uint32_t)(o * 8 + tr) * 8);
                aux = e.x;
                const float2 md = __half22float2(u2h2(e.y));
                dl = md.y * d.vscale;
                mp = md.x - dl;
            }
            for (int h = 0; h < 2; ++h) {
                const int s = 2 * t + h;
                // the A buffer of slab s was last read by the MMAs of slab s - NA
                if (s >= NA) {
                    gwait(sm.mma_done_at(ms), mph, p.status);
                    if (++ms == NB) { ms = 0; mph ^= 1; }
                }
                // The four subvectors' shared loads are independent: non-volatile
                // loads whose addresses carry a token taken after the waits above
                // (chunk resident, slab buffer free) let them overlap; the stores,
                // which consume every result, stay in order before the arrival.
                const uint32_t tok = order_token();
                const uint32_t a_slab = sm.a0 + (uint32_t)as * kASlab + a_row;
                // No branch around each subvector: the four decodes form one
                // straight-line block whose loads and arithmetic interleave.
                uint4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int jl = h * kGSlabJ + 4 * cw + i;  // chunk column
                    const uint32_t w = lds32_r(slot + tok + (uint32_t)(jl * n_oct + oc) * 16 + (uint32_t)(tr >> 1) * 4);
                    v[i] = decode_sv(d, w, odd, s0, s1, s2, aux, (uint32_t)(15 - jl), mp, dl, cbsel + tok);
                    if (!active) v[i] = make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) sts128(a_slab + (uint32_t)(4 * cw + i) * 128, v[i]);
                fence_proxy_async_smem();  // the generic-proxy writes above are read by the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(sm.a_full_at(as));
                if (++as == NA) as = 0;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(sm.code_empty(t));
        }
        // ---------------- epilogue ----------------
        wait_last = true;
    }
    if (warp < 8 && wait_last) {
        gwait(sm.mma_done(n_slab - 1, NB), ((n_slab - 1) / NB) & 1, p.status);
        tc_fence_after();
    }
    const int q4 = warp & 3, hf = (warp >> 2) & 1;
    const int row_local = hf * 128 + q4 * 32 + lane;
    const uint32_t tw = taddr + (uint32_t)(hf * p.n_alloc) + ((uint32_t)(q4 * 32) << 16);
    if (p.parts == 1) {
        const int row = blk * 256 + row_local;
        if (warp < 8) {
            for (int c0 = 0; c0 < p.n_pad; c0 += 16) {
                float v[16];
                tmem_ld16(tw + (uint32_t)c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int n = c0 + i;
                    if (n < p.M && row < p.d_out) p.y[(size_t)n * p.d_out + row] = __half_as_ushort(__float2half_rn(v[i]));
                }
            }
            tc_fence_before();
        }
    } else {
        // The parts of a block form one thread-block cluster.  Round by round over
        // the batch columns, every part stages its fp32 accumulator in its own
        // (now idle) operand buffers; then part r adds the parts' values, in part
        // order, for rows [256 r / parts, 256 (r + 1) / parts) through distributed
        // shared memory and writes those rows of y.
        const uint32_t red0 = sm.code0;
        const int nc = p.red_cols;
        // part r reduces the row quads [64 r / parts, 64 (r + 1) / parts)
        const int qA = part * 64 / p.parts, qB = (part + 1) * 64 / p.parts, nq = qB - qA;
        const bool vec_y = (p.d_out & 3) == 0;
        for (int n0 = 0; n0 < p.M; n0 += nc) {
            const int n1 = min(p.M, n0 + nc);
            if (warp < 8) {
                for (int c0 = n0 & ~15; c0 < n1; c0 += 16) {
                    float v[16];
                    tmem_ld16(tw + (uint32_t)c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int n = c0 + i;
                        if (n >= n0 && n < n1) sts_f32(red0 + (uint32_t)((n - n0) * 256 + row_local) * 4, v[i]);
                    }
                }
                tc_fence_before();
            }
            cluster_sync();
            const int total = nq * (n1 - n0);
            for (int e0 = tid; e0 < total; e0 += 2 * kGThreads) {
                float4 acc[2];
                uint32_t off[2];
                bool ok[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int e = e0 + u * kGThreads;
                    ok[u] = e < total;
                    const int c = ok[u] ? e / nq : 0, q = qA + (ok[u] ? e - c * nq : 0);
                    off[u] = red0 + (uint32_t)(c * 256 + q * 4) * 4;
                    acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                for (int k0 = 0; k0 < p.parts; k0 += 4) {  // parts in order, four at a time in flight
                    float4 t[2][4];
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            t[u][k] = (ok[u] && k0 + k < p.parts) ? ld_cluster_v4(map_cluster(off[u], k0 + k))
                                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            acc[u].x += t[u][k].x;
                            acc[u].y += t[u][k].y;
                            acc[u].z += t[u][k].z;
                            acc[u].w += t[u][k].w;
                        }
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (!ok[u]) continue;
                    const int e = e0 + u * kGThreads, c = e / nq, q = qA + (e - c * nq);
                    const int row = blk * 256 + q * 4;
                    uint16_t* yr = p.y + (size_t)(n0 + c) * p.d_out + row;
                    const uint16_t h0 = __half_as_ushort(__float2half_rn(acc[u].x));
                    const uint16_t h1 = __half_as_ushort(__float2half_rn(acc[u].y));
                    const uint16_t h2 = __half_as_ushort(__float2half_rn(acc[u].z));
                    const uint16_t h3 = __half_as_ushort(__float2half_rn(acc[u].w));
                    if (vec_y && row + 3 < p.d_out) {
                        *reinterpret_cast<uint2*>(yr) = make_uint2((uint32_t)h0 | ((uint32_t)h1 << 16),
                                                                   (uint32_t)h2 | ((uint32_t)h3 << 16));
                    } else {
                        if (row < p.d_out) yr[0] = h0;
                        if (row + 1 < p.d_out) yr[1] = h1;
                        if (row + 2 < p.d_out) yr[2] = h2;
                        if (row + 3 < p.d_out) yr[3] = h3;
                    }
                }
            }
            cluster_sync();  // the remote reads are done before the buffers are reused or the CTA exits
        }
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(taddr, tcols);
    }
}

}  // namespace

namespace {

int gemm_sm_count() { return current_sm_count(); }

size_t round256g(size_t b) { return (b + 255) / 256 * 256; }

// Launch plan and workspace layout of one sage_gemm call:
//   status header | x_perm tiles
struct GemmPlan {
    int n_pad, n_alloc, parts, a_slots, b_slots, n_blocks, smem, red_cols;
    size_t off_xt, total;
};

constexpr int kGemmSmemBudget = 226 * 1024;

GemmPlan gemm_plan(const sage_matrix* A, int M) {
    GemmPlan g;
    g.n_pad = (M + 15) / 16 * 16;
    g.n_alloc = 32;
    while (g.n_alloc < g.n_pad) g.n_alloc *= 2;
    const int R8 = (A->d_out + 7) / 8;
    g.n_blocks = (R8 + kGOct - 1) / kGOct;
    const int G = A->d_in / 128;
    // parts of a block run as one cluster (at most 8: portable cluster size)
    g.parts = std::max(1, std::min(std::min(8, gemm_sm_count() / g.n_blocks), G / 2));
    const int K = 1 << A->log2K;
    // The decoded-slab ring as deep as fits, then the x_perm ring.  The x_perm
    // ring is at least as deep: a slab's mma_done barrier is then never two
    // phases ahead of a decode warp that waits on it.
    g.a_slots = kMaxASlots;
    while (g.a_slots > 2 && gemm_smem_bytes(K, g.n_pad, g.a_slots, g.a_slots) > kGemmSmemBudget) --g.a_slots;
    g.b_slots = g.a_slots;
    while (g.b_slots < 8 && gemm_smem_bytes(K, g.n_pad, g.a_slots, g.b_slots + 1) <= kGemmSmemBudget) ++g.b_slots;
    g.smem = gemm_smem_bytes(K, g.n_pad, g.a_slots, g.b_slots);
    // the cluster reduction stages 256 fp32 per batch column in the code ring and operand buffers
    const int staging = kGCodeSlots * kGCodeSlot + g.a_slots * kASlab + g.b_slots * g.n_pad * 128;
    g.red_cols = std::min(g.n_pad, staging / 1024 / 16 * 16);
    size_t o = kWsHeader;
    g.off_xt = o;
    o += round256g((size_t)(A->d_in / 64) * g.n_pad * 128);
    g.total = o;
    return g;
}

}  // namespace

size_t gemm_workspace_bytes(const sage_matrix* A, int M) { return gemm_plan(A, M).total; }

int launch_gemm(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y, void* ws, size_t ws_bytes,
                sage_stream_t stream) {
    if (M < 9 || M > 256) return SAGE_ERR_UNSUPPORTED;
    const GemmPlan g = gemm_plan(A, M);
    if (ws_bytes < g.total) return SAGE_ERR_WORKSPACE;
    if (g.smem > kGemmSmemBudget) return SAGE_ERR_UNSUPPORTED;
    static SmemLimit limit;
    if (!limit.ensure(gemm_kernel, g.smem)) return SAGE_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint4* xt = reinterpret_cast<uint4*>(w + g.off_xt);
    const long long n_xt = (long long)(A->d_in / 64) * g.n_pad * 8;
    tile_x_kernel<<<(unsigned)((n_xt + 255) / 256), 256, 0, s>>>(x, A->perm, M, g.n_pad, A->d_in, xt);
    if (cudaGetLastError() != cudaSuccess) return SAGE_ERR_CUDA;
    GemmParams p;
    p.main = A->main;
    p.meta = A->meta;
    p.cb = A->codebook;
    p.xt = xt;
    p.y = y;
    p.status = reinterpret_cast<uint32_t*>(w);
    p.d_out = A->d_out;
    p.d_in = A->d_in;
    p.log2K = A->log2K;
    p.M = M;
    p.n_pad = g.n_pad;
    p.n_alloc = g.n_alloc;
    p.parts = g.parts;
    p.red_cols = g.red_cols;
    p.a_slots = g.a_slots;
    p.b_slots = g.b_slots;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = (size_t)g.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // The largest cluster (parts per block) for which every block's cluster is
    // resident at once: a second wave would double the time.
    int parts = g.parts;
    for (; parts > 1; --parts) {
        attr[0].val.clusterDim.x = (unsigned)parts;
        cfg.gridDim = dim3((unsigned)(g.n_blocks * parts));
        int active = 0;
        if (cudaOccupancyMaxActiveClusters(&active, (const void*)gemm_kernel, &cfg) == cudaSuccess && active >= g.n_blocks)
            break;
    }
    (void)cudaGetLastError();
    p.parts = parts;
    attr[0].val.clusterDim.x = (unsigned)parts;
    cfg.gridDim = dim3((unsigned)(g.n_blocks * parts));
    return cudaLaunchKernelEx(&cfg, gemm_kernel, p) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace sage
