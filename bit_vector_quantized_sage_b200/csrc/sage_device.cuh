// Device-side building blocks shared by the libsage kernels (sm_100a):
// PTX wrappers for mbarriers, bulk (TMA) copies, PDL, acquire/release
// accesses, and the decode constants of the packed format v2 (include/sage.h).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace sage {
namespace dev {

// ------------------------------------------------------------------------
// Shared-memory addressing and loads
// ------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Shared-memory loads the compiler may reorder among themselves (no
// `volatile`, no memory clobber).  They must only be used with addresses that
// derive from an order_token() taken after the wait that makes the data
// valid, so that no load can be hoisted above that wait, and their results
// must be consumed (see keep()) before the buffer is released.
__device__ __forceinline__ uint4 lds128_r(uint32_t addr) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32_r(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
// A zero the compiler cannot see through, produced in program order after the
// preceding waits (it is a volatile statement with a memory clobber).
__device__ __forceinline__ uint32_t order_token() {
    uint32_t t;
    asm volatile("mov.u32 %0, 0;" : "=r"(t)::"memory");
    return t;
}
// Forces v to be computed before the next volatile statement (e.g. a buffer release).
__device__ __forceinline__ void keep(float v) { asm volatile("" ::"f"(v)); }

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------------------
// mbarrier (CTA scope)
// ------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Arrival that also raises the expected transaction byte count of the phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Gives up after roughly
// `limit` polls (with nanosleep back-off after the first few thousand) and
// returns false; callers then record a timeout in the status word and carry
// on, so no wait can hang the GPU.
constexpr uint32_t kWaitLimit = 1u << 22;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = kWaitLimit) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_test(bar, parity)) return true;
        if (i > 2048) __nanosleep(64);
    }
    return false;
}

// ------------------------------------------------------------------------
// Bulk asynchronous copy global -> shared (1-D TMA), completes on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.
// ------------------------------------------------------------------------
// Orders this thread's earlier generic-proxy shared-memory accesses before
// its later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read exactly once (the packed planes): evicted first, so
// that the streamed planes do not push out what is reused (kernel code,
// parameters, activations, split-K partials).
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void bulk_g2s_stream(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// ------------------------------------------------------------------------
// Programmatic dependent launch
// ------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------------
// Device-scope atomics and ordered accesses
// ------------------------------------------------------------------------
// Atomic add with acquire-release semantics (returns the old value).
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Release increment: every write of this thread that precedes it (and, after
// a CTA barrier, of the threads that reached the barrier first) becomes
// visible to an acquire load that sees the new value.
__device__ __forceinline__ void red_add_release_gpu(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_gpu(unsigned* p, unsigned v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------------------------
// Packed format v2 decode constants (per radius width V = 10 - log2K).
// ------------------------------------------------------------------------
template <int V>
struct Fmt {
    static constexpr int kLog2K = 10 - V;
    // z occupies bits [7, 7 + log2K) of the (rotated) word -> byte offset z*128
    static constexpr uint32_t kZMask = ((1u << kLog2K) - 1u) << 7;
    // q occupies the top V mantissa bits [23 - V, 23): OR-ing 1.0f gives 1 + q/2^V
    static constexpr uint32_t kQMask = ((1u << V) - 1u) << (23 - V);
    // sign slots {0 .. 6-V} U {17-V .. 15}
    __host__ __device__ static constexpr int slot(int k) { return k <= 6 - V ? k : (17 - V) + (k - (7 - V)); }
};

// XOR mask with the slot's two sign bits moved to bits 15 and 31 (the fp16
// sign bits of a half2).
template <int P>
__device__ __forceinline__ uint32_t slot_mask(uint32_t w) {
    return (w << (15 - P)) & 0x80008000u;
}

__device__ __forceinline__ uint32_t aux_mask(uint32_t aux, int t) {
    return (aux << (15 - t)) & 0x80008000u;
}

__device__ __forceinline__ uint32_t rot16(uint32_t w) { return __funnelshift_l(w, w, 16); }

// 1 + q / 2^V as fp32 bits, from a word whose bits [23-V, 23) hold q.
template <int V>
__device__ __forceinline__ float q_unit(uint32_t w) {
    return __uint_as_float((w & Fmt<V>::kQMask) | 0x3F800000u);
}

// Plane offsets (format v2): blocks of 32 row octets stored contiguously.
__device__ __forceinline__ int block_octets(int R8, int blk) { return min(32, R8 - blk * 32); }
// uint32 word index of word u of the record (column j, local octet o) of block blk.
__device__ __forceinline__ size_t main_word(int R8, int S, int blk, int j, int o, int u) {
    return (size_t)blk * S * 128 + ((size_t)j * block_octets(R8, blk) + o) * 4 + u;
}
// 8-byte entry index of (group g, local octet o, row t) of block blk.
__device__ __forceinline__ size_t meta_entry(int R8, int G, int blk, int g, int o, int t) {
    return (size_t)blk * G * 256 + ((size_t)g * block_octets(R8, blk) + o) * 8 + t;
}

__device__ __forceinline__ __half2 u2h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t h22u(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Per-split decode constants of format v2 (radius width V = 10 - log2K),
// chosen at run time so one kernel serves every split of a launch.
struct VDec {
    uint32_t zmask, qmask;
    uint32_t sh0, sh1, sh2, sh3, sh4, sh5;   // 15 - (sign slot position); slot 5 sits at bit 15 (sh5 = 0)
    uint32_t m0, m1, m2, m3, m4;             // 2^sh0 .. 2^sh4: the same shifts as multiplies
    uint32_t m16;                            // 2^16
    float vscale;                            // 2^V
};

__device__ __forceinline__ uint32_t opaque(uint32_t v) {
    uint32_t r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}

__device__ __forceinline__ VDec vdec(int log2K) {
    const int V = 10 - log2K;
    VDec d;
    d.zmask = ((1u << log2K) - 1u) << 7;
    d.qmask = ((1u << V) - 1u) << (23 - V);
    // slot k sits at bit k for k <= 6 - V, else at bit 10 + k
    auto sh = [&](int k) { return (uint32_t)(k <= 6 - V ? 15 - k : 5 - k); };
    d.sh0 = sh(0); d.sh1 = sh(1); d.sh2 = sh(2); d.sh3 = sh(3); d.sh4 = sh(4); d.sh5 = sh(5);
    // The multipliers are passed through an opaque move, so that the compiler
    // keeps the multiplies (FMA pipe) instead of turning them back into shifts.
    d.m0 = opaque(1u << d.sh0); d.m1 = opaque(1u << d.sh1); d.m2 = opaque(1u << d.sh2);
    d.m3 = opaque(1u << d.sh3); d.m4 = opaque(1u << d.sh4);
    d.m16 = opaque(1u << 16);
    d.vscale = (float)(1 << V);
    return d;
}

}  // namespace dev
}  // namespace sage
