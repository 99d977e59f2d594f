// Packed SAGE GEMV engine for batch 1..8 on sm_100a: the decode path of
// "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World Usability"
// (Sec. 3.5 and App. A.1, Fig. 6a), run as one persistent launch over a list
// of dependent stages (a stage is one GEMV or several GEMVs sharing a launch,
// e.g. the q|k|v projections), and the grouped-expert MoE GEMV on the same
// body.
//
// Work decomposition (B200-first, not the paper's RTX 4090 tiling):
//  * A "unit" is one subvector column j of one 256-row block (32 row octets)
//    of one matrix: a 512-byte slab of the main plane.  The units of a stage
//    are flattened (matrix, block, j) and cut into one contiguous range per
//    CTA of a persistent grid (one CTA per SM); every stage is spread over
//    every CTA.
//  * The copy warp bulk-copies (1-D TMA) codebooks and, chunk by chunk (32
//    columns = two radius groups), the code records and grid/aux meta into a
//    ring of shared-memory slots.  It runs ahead across segments and stages:
//    the packed planes never depend on earlier work, so the next stage's codes
//    stream in while the current stage finishes.
//  * The gather warp builds the ESG-permuted activations x_perm[p] = x[perm[p]]
//    window by window (Sec. 3.5 fuses this gather into the decode GEMV; the
//    fused prologues -- RMSNorm, residual + RMSNorm, SiLU(gate) * up, and the
//    single-position attention read of v -- are applied to the gathered values).
//    The first window of each stage is gathered by the gather and decode warps
//    together, after the stage's inputs are ready.
//  * 8 decode warps: warp w holds row pairs 32 (w % 4) .. 32 (w % 4) + 31 of the
//    256-row block (one 32-bit record word = two rows per thread) and columns
//    8 (w / 4) .. 8 (w / 4) + 7 of each chunk.  Per subvector: the codeword
//    address is one logic op on the word (format v2), the codeword one
//    conflict-free 128-bit load from the replica of the thread's lane position
//    (8 bank-rotated replicas of the codebook), the signs are XORed into the
//    fp16 sign bits, eight fp16 x fp16 products summed in fp32 (mixed-precision
//    FMA; Fig. 6a sums them in fp16) form (s (.) c) . x, and r = mu + q delta
//    (Eq. 2) scales it once, in fp32, into the row's fp32 accumulator.
//  * Rows whose columns are split between CTAs are combined deterministically:
//    partial sums go to the workspace and the last CTA to finish a block adds
//    them in CTA order.  A block whose final outputs are written bumps its
//    stage's completion count; a stage that reads an earlier stage's outputs
//    waits for that count (acquire), so dependent stages need no relaunch.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "sage_device.cuh"
#include "sage_internal.h"
#include "sage_engine.h"

namespace sage {
using namespace dev;

namespace {

constexpr int kOct = 32;               // row octets per block
constexpr int kBlockRows = kOct * 8;   // 256
constexpr int kChunkJ = 32;            // a chunk is two radius groups (aligned)
constexpr int kMainSlot = kChunkJ * kOct * 16;  // 16 KB of code records
constexpr int kMetaSlot = 2 * kOct * 64;        // 4 KB: two groups of 256 rows
constexpr int kSlot = kMainSlot + kMetaSlot;    // one ring slot = one chunk
constexpr int kMaxSlots = 16;
constexpr int kDW = 8;                          // decode warps: 4 row quarters x 2 column parts
constexpr int kParts = kDW / 4;                 // column parts of a chunk (one radius group each)
constexpr int kDT = kDW * 32;                   // decode threads
constexpr int kGT = kDT + 32;                   // threads of a cooperative gather
constexpr int kEpiWarps = 2;                    // epilogue warps (segments dealt out alternately)
constexpr int kThreads = kDT + 32 * (2 + kEpiWarps);  // + copy, gather and epilogue warps
constexpr int kCopyWarp = kDW, kGatherWarp = kDW + 1, kEpiWarp = kDW + 2;
constexpr int kStashSlots = 4;                  // segments between the decode and epilogue warps (at most)
constexpr int kBarDecode = 1, kBarGather = 2;   // named barriers (0 is __syncthreads)
constexpr int kXBufBytes = 8192;                // one activation window buffer
constexpr int kMaxXW = 512;                     // window columns at batch 1
constexpr int kPermBuf = kMaxXW * 32;           // the window's permutation entries
constexpr int kMoeCache = 32;                   // virtual experts staged per CTA
constexpr int kMaxMoeCtas = 256;                // CTAs of a MoE launch (one per SM)
constexpr int kMaxPairsPerVirtual = 8;

// Codebook replicas: codeword z of replica r at byte z*128 + r*16.  Static
// shared memory has a link-time address, so a codeword's address is one logic
// op on the record word plus the load's immediate offset.
__shared__ __align__(1024) uint4 g_rep[256 * 8];

// Codeword at byte offset `off` of the replicas (z * 128 + r * 16): an
// explicit shared-memory load (short scoreboard) whose base is the array's
// link-time shared address, which the assembler can fold into the load.
__device__ __forceinline__ uint4 cw_load(uint32_t base, uint32_t off) { return lds128_r(base + off); }

template <int M>
struct Cfg {
    static constexpr int kXW = kXBufBytes / (16 * M);    // window columns
    static constexpr int kSlots = M <= 2 ? kStashSlots : 2;  // stash ring depth
    static constexpr int kStash = kSlots * kParts * M * kBlockRows * 4;  // [slot][column part][m][row]
};

// ------------------------------------------------------------------------
// Problem sources: where a stage's jobs (one matrix with its input and output
// binding each) come from.  Dense launches carry them in the kernel
// parameters; the MoE launch reads virtual experts from the routing result.
// ------------------------------------------------------------------------
struct JobView {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const int32_t* perm;
    const uint16_t* x;    // plain-prologue input rows, stride d_in
    uint16_t* y;          // output rows, stride d_out
    const int* xrows;     // batch slot -> input row (null: slot m reads row m); shared memory
    const int* yrows;     // batch slot -> output row (null: slot m writes row m); shared memory
    int unit0, d_out, d_in, log2K, S, R8, blk0, Mk, id;
};

// Balanced split of `units` over n_cta CTAs: the first units % n_cta CTAs
// take one unit more.  32-bit arithmetic only.
__device__ __forceinline__ int cta_begin(int units, int n_cta, int c) {
    const int q = units / n_cta, r = units - q * n_cta;
    return q * c + min(c, r);
}
// The CTA whose range [cta_begin(c), cta_begin(c + 1)) holds unit u.
__device__ __forceinline__ int cta_of(int units, int n_cta, int u) {
    const int q = units / n_cta, r = units - q * n_cta;
    const int big = (q + 1) * r;  // units held by the CTAs that take q + 1
    return u < big ? u / (q + 1) : r + (u - big) / q;
}

// The same over a 64-bit total (the MoE cost space).
__device__ __forceinline__ long long cta_begin64(long long total, int n_cta, int c) {
    const long long q = total / n_cta, r = total - q * n_cta;
    return q * c + min((long long)c, r);
}

struct DenseSrc {
    static constexpr bool kVarBatch = false;
    const EngineParams& p;
    __device__ int n_stages() const { return p.n_stages; }
    __device__ const EngineStage& stage(int s) const { return p.st[s]; }
    __device__ int units(int s) const { return p.st[s].units; }
    // first unit of CTA c (c = n_cta: the end) and the CTA holding unit u
    __device__ int cta_u0(int s, int n_cta, int c) const { return cta_begin(p.st[s].units, n_cta, c); }
    __device__ int owner(int s, int n_cta, int u) const { return cta_of(p.st[s].units, n_cta, u); }
    // every CTA of a dense launch holds units (at least 4 per CTA)
    __device__ bool cta_nonempty(int, int, int) const { return true; }
    __device__ int contributors(int, int, int c_first, int c_last) const { return c_last - c_first + 1; }
    __device__ JobView job_at(int s, int u) const {
        const EngineStage& st = p.st[s];
        int k = st.job0;
        while (k + 1 < st.job0 + st.n_jobs && p.jobs[k + 1].unit0 <= u) ++k;
        return job(k);
    }
    __device__ JobView job(int k) const {
        const EngineJob& d = p.jobs[k];
        JobView v;
        v.main = d.main; v.meta = d.meta; v.cb = d.cb; v.perm = d.perm; v.x = d.x; v.y = d.y;
        v.xrows = nullptr; v.yrows = nullptr;
        v.unit0 = d.unit0; v.d_out = d.d_out; v.d_in = d.d_in; v.log2K = d.log2K;
        v.S = d.d_in >> 3; v.R8 = (d.d_out + 7) >> 3; v.blk0 = d.blk0; v.Mk = p.M; v.id = k;
        return v;
    }
};

// Decode batch width of a virtual expert with n pairs (1, 2, 4 or 8): the
// cost weight of its units in the MoE split.
__host__ __device__ constexpr int moe_weight(int n) { return n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : 8; }

// The MoE routing this CTA needs (virtual-expert ids, pair counts and row
// lists of the virtual experts its range touches), built in shared memory by
// the CTA at the start of the MoE kernel.
struct MoeStage {
    int n_virtual, units, vi0, nvi, overflow, n_e, upv;
    long long cost_total;
    int cnt[kMaxExperts];             // pairs per expert
    int first[kMaxExperts + 1];       // first virtual expert of each expert; [n_e]: their number
    long long cost[kMaxExperts + 1];  // first cost unit of each expert (exclusive prefix)
    int bound[kMaxMoeCtas + 1];       // first unit of each CTA (cost-balanced); [n_cta]: the end
    int v_expert[kMoeCache];
    int v_count[kMoeCache];
    int v_xrows[kMoeCache][kMaxPairsPerVirtual];
    int v_yrows[kMoeCache][kMaxPairsPerVirtual];
};

struct MoeSrc {
    static constexpr bool kVarBatch = true;
    const MoeParams& p;
    const MoeStage& ms;
    __device__ int n_stages() const { return 1; }
    __device__ const EngineStage& stage(int) const { return p.st; }
    __device__ int units(int) const { return ms.units; }
    __device__ int upv() const { return ms.upv; }
    // CTA ranges are balanced over decode cost, not units: a unit of a virtual
    // expert with n pairs costs moe_weight(n), the batch width its segments
    // decode with (the decode time per column grows about linearly with it).
    __device__ int cta_u0(int, int, int c) const { return ms.bound[c]; }
    // The unit where CTA c's share of the cost starts (64-bit divisions: built
    // once per launch into ms.bound, one CTA index per thread).
    __device__ int cost_bound(int n_cta, int c) const {
        const long long cp = cta_begin64(ms.cost_total, n_cta, c);
        if (cp >= ms.cost_total) return ms.units;
        int lo = 0, hi = ms.n_e - 1;  // the expert whose cost range holds cp
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ms.cost[mid] <= cp) lo = mid; else hi = mid - 1;
        }
        const int e = lo, c_e = ms.cnt[e], full = c_e / kMaxPairsPerVirtual;
        long long r = cp - ms.cost[e];
        const long long full_cost = (long long)ms.upv * kMaxPairsPerVirtual;
        int k, w;
        if (r < full * full_cost) {
            k = (int)(r / full_cost);
            r -= k * full_cost;
            w = kMaxPairsPerVirtual;
        } else {
            k = full;
            r -= full * full_cost;
            w = moe_weight(c_e - full * kMaxPairsPerVirtual);
        }
        // the first unit whose cost starts at or after cp
        return (ms.first[e] + k) * ms.upv + (int)((r + w - 1) / w);
    }
    // A cost-balanced split can leave a CTA without units (a unit of an
    // 8-pair virtual expert outweighs a CTA's share when there is little
    // work); such CTAs take no part in any block.
    __device__ bool cta_nonempty(int, int, int c) const { return ms.bound[c] < ms.bound[c + 1]; }
    __device__ int contributors(int s, int n_cta, int c_first, int c_last) const {
        int n = 0;
        for (int c = c_first; c <= c_last; ++c) n += cta_nonempty(s, n_cta, c) ? 1 : 0;
        return n;
    }
    __device__ int owner(int, int n_cta, int u) const {  // the last CTA whose range starts at or before u
        int lo = 0, hi = n_cta - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ms.bound[mid] <= u) lo = mid; else hi = mid - 1;
        }
        return lo;
    }
    __device__ JobView job_at(int, int u) const { return job(u / upv()); }
    __device__ JobView job(int vi) const {
        const int k = vi - ms.vi0;  // always staged: a CTA only touches its own range
        const int e = ms.v_expert[k];
        const EngineExpert& d = p.experts[e];
        JobView v;
        v.main = d.main; v.meta = d.meta; v.cb = d.cb; v.perm = d.perm; v.x = p.x; v.y = p.y;
        v.xrows = ms.v_xrows[k]; v.yrows = ms.v_yrows[k];
        v.d_out = p.d_out; v.d_in = p.d_in; v.log2K = d.log2K;
        v.S = p.d_in >> 3; v.R8 = (p.d_out + 7) >> 3;
        v.unit0 = vi * upv();
        v.blk0 = vi * ((v.R8 + kOct - 1) / kOct);
        v.Mk = ms.v_count[k];
        v.id = vi;
        return v;
    }
};

// A segment: one job, one 256-row block, columns [ja, jb) of a CTA's range.
struct Seg {
    JobView v;
    int blk, ja, jb, n_oct;
    bool full;
};

template <class Src>
__device__ __forceinline__ Seg make_seg(const Src& src, int s, int u, int u1) {
    Seg g;
    g.v = src.job_at(s, u);
    const int local = u - g.v.unit0;
    g.blk = local / g.v.S;
    g.ja = local - g.blk * g.v.S;
    g.jb = min(g.v.S, g.ja + (u1 - u));
    g.n_oct = min(kOct, g.v.R8 - g.blk * kOct);
    g.full = (g.ja == 0 && g.jb == g.v.S);
    return g;
}

// Columns [x, y) of chunk c (chunks are cut at 32-column boundaries, i.e.
// every other radius-group boundary).
__device__ __forceinline__ int2 chunk_cols(const Seg& g, int c) {
    const int k = (g.ja >> 5) + c;
    return make_int2(max(g.ja, k << 5), min(g.jb, (k + 1) << 5));
}
__device__ __forceinline__ int n_chunks(const Seg& g) { return ((g.jb - 1) >> 5) - (g.ja >> 5) + 1; }

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bits) { atomicOr(status, bits); }

// A segment decoded but not yet written out (its sums wait in the stash).
struct Pending {
    Seg g;
    int stage;
    int first;   // the CTA's first segment of the stage (split-K slot 0)
};
static_assert(sizeof(Pending) <= 192, "pending-segment table entry outgrew its shared memory");
static_assert(sizeof(JobView) <= 112, "job cache entry outgrew its shared memory");
static_assert(sizeof(EngineStage) <= 128, "stage copy outgrew its shared memory");

// ------------------------------------------------------------------------
// Shared memory
// ------------------------------------------------------------------------
struct Smem {
    uint32_t cb0;       // codebook replicas (g_rep)
    uint32_t ring0;     // chunk ring
    uint32_t cbraw0;    // two raw codebooks
    int cbraw_bytes;
    uint32_t xbuf0;     // two activation windows
    uint32_t perm0;     // the window's permutation entries (8 int32 per column)
    int slots;
    uint32_t* posinfo;  // per window position: job slot << 20 | column j
    const int32_t** posperm;  // per window position: its 8 permutation entries (null: identity)
    float* stash;       // [slot][column part][M][256] decode sums awaiting the epilogue
    float* red;         // [kGT / 32][8] cooperative reductions
    uint64_t* bars;
    int* misc;          // [2] abort flag, [8] window length, [9] batch rows per window, [10] stages whose first window is gathered,
                        // [16..24) flush flags
    float* inv_rms;     // [8] per batch row
    struct Pending* pend;  // segments awaiting their flush (written by decode thread 0)
    EngineStage* stc;   // the stage being gathered (copied from the parameters by the gather warp)
    JobView* jc;        // jobs of the stage's windows, by window job slot (see posinfo)
    __device__ uint32_t slot_addr(int k) const { return ring0 + (uint32_t)k * kSlot; }
    __device__ uint64_t* full(int k) const { return bars + k; }
    __device__ uint64_t* empty(int k) const { return bars + kMaxSlots + k; }
    __device__ uint64_t* cb_full(int h) const { return bars + 2 * kMaxSlots + h; }
    __device__ uint64_t* cb_empty(int h) const { return bars + 2 * kMaxSlots + 2 + h; }
    __device__ uint64_t* x_full(int h) const { return bars + 2 * kMaxSlots + 4 + h; }
    __device__ uint64_t* x_empty(int h) const { return bars + 2 * kMaxSlots + 6 + h; }
    __device__ uint64_t* perm_full() const { return bars + 2 * kMaxSlots + 8; }
    __device__ uint64_t* st_full(int k) const { return bars + 2 * kMaxSlots + 9 + k; }
    __device__ uint64_t* st_empty(int k) const { return bars + 2 * kMaxSlots + 9 + kStashSlots + k; }
    __device__ uint32_t xwin(int w) const { return xbuf0 + (uint32_t)(w & 1) * kXBufBytes; }
    __device__ volatile int* abort_flag() const { return misc + 2; }
};
constexpr int kBars = 2 * kMaxSlots + 9 + 2 * kStashSlots;

constexpr int kPendBytes = kStashSlots * 192;  // pending-segment table (sizeof(Pending) <= 192)
constexpr int kJobCache = 64;                    // job slots of a stage (jobs of one CTA range)
constexpr int kJcBytes = kJobCache * 112 + 128;  // job cache (sizeof(JobView) <= 112) + stage copy

template <int M>
constexpr int fixed_smem() {
    return 2 * kXBufBytes + kPermBuf + kMaxXW * 4 + kMaxXW * 8 + Cfg<M>::kStash + (kGT / 32) * 8 * 4 + kBars * 8 +
           64 * 4 + 8 * 4 + kPendBytes + kJcBytes;
}
// Dynamic shared memory of a launch: raw codebooks + ring + fixed buffers.
template <int M>
int smem_bytes(int slots, int kmax) {
    return 2 * kmax * 16 + slots * kSlot + fixed_smem<M>();
}

template <int M>
__device__ Smem carve(uint8_t* base, int slots, int kmax) {
    Smem s;
    s.slots = slots;
    s.cb0 = smem_u32(g_rep);
    uint8_t* p = base;
    s.ring0 = smem_u32(p); p += slots * kSlot;
    s.cbraw_bytes = kmax * 16;
    s.cbraw0 = smem_u32(p); p += 2 * kmax * 16;
    s.xbuf0 = smem_u32(p); p += 2 * kXBufBytes;
    s.perm0 = smem_u32(p); p += kPermBuf;
    s.posinfo = reinterpret_cast<uint32_t*>(p); p += kMaxXW * 4;
    s.posperm = reinterpret_cast<const int32_t**>(p); p += kMaxXW * 8;
    s.stash = reinterpret_cast<float*>(p); p += Cfg<M>::kStash;
    s.red = reinterpret_cast<float*>(p); p += (kGT / 32) * 8 * 4;
    s.bars = reinterpret_cast<uint64_t*>(p); p += kBars * 8;
    s.misc = reinterpret_cast<int*>(p); p += 64 * 4;
    s.inv_rms = reinterpret_cast<float*>(p); p += 8 * 4;
    s.pend = reinterpret_cast<Pending*>(p); p += kPendBytes;
    s.stc = reinterpret_cast<EngineStage*>(p); p += 128;
    s.jc = reinterpret_cast<JobView*>(p);  // kJobCache entries of 112 bytes
    return s;
}

__device__ __forceinline__ bool wait_bar(const Smem& sm, uint64_t* bar, uint32_t parity, uint32_t* status) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_test(bar, parity)) return true;
        if (i > 2048) {
            if (*sm.abort_flag()) return false;
            __nanosleep(64);
        }
    }
    *sm.abort_flag() = 1;
    flag(status, kDevTimeout);
    return false;
}

// Bounded wait until *cnt >= target (acquire).  One thread polls.
__device__ __forceinline__ bool wait_count(const Smem& sm, const unsigned* cnt, unsigned target, uint32_t* status) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (ld_acquire_gpu(cnt) >= target) return true;
        if (*sm.abort_flag()) return false;
        __nanosleep(i < 64 ? 32 : 128);
    }
    *sm.abort_flag() = 1;
    flag(status, kDevTimeout);
    return false;
}

__device__ __forceinline__ void ring_next(int& slot, int& ph, int slots) {
    if (++slot == slots) {
        slot = 0;
        ph ^= 1;
    }
}

// Activation windows: the chunks of a CTA's stage range are laid end to end;
// a window holds up to `xw` of their columns (a chunk never straddles two
// windows) and every stage starts a new window.  The gather warp and the
// decode warps apply these rules identically.
struct WinPos {
    int win;   // global window index (buffer win & 1)
    int wpos;  // columns placed in the window so far
};
__device__ __forceinline__ int win_place(WinPos& w, int nj, int xw) {
    if (w.wpos + nj > xw) { ++w.win; w.wpos = 0; }
    const int p = w.wpos;
    w.wpos += nj;
    return p;
}
__device__ __forceinline__ void win_break(WinPos& w) {
    if (w.wpos > 0) { ++w.win; w.wpos = 0; }
}

// ------------------------------------------------------------------------
// Copy warp
// ------------------------------------------------------------------------
// Chunks of a stage requested before the stage's first activation window is
// gathered: the gather's small, latency-critical loads (permutation entries,
// inputs, norm weights, the kernel parameters) must not queue in the memory
// system behind the CTA's whole share of the packed planes.  After the
// gather, HBM delivers chunks faster than the decode consumes them.
constexpr int kStartChunks = 2;

template <class Src>
__device__ void copy_role(const Src& src, const Smem& sm, uint32_t* status, int n_cta) {
    const int lane = threadIdx.x & 31;
    int t = 0, slot = 0, ph = 0, ncb = 0;
    const uint16_t* cur_cb = nullptr;
    const uint64_t pol = l2_evict_first();
    for (int s = 0; s < src.n_stages(); ++s) {
        const int U = src.units(s);
        if (U <= 0) continue;
        const int u1 = src.cta_u0(s, n_cta, blockIdx.x + 1);
        int ts = 0;  // chunks of this stage issued so far
        for (int u = src.cta_u0(s, n_cta, blockIdx.x); u < u1;) {
            const Seg g = make_seg(src, s, u, u1);
            u += g.jb - g.ja;
            if (g.v.cb != cur_cb) {
                const int h = ncb & 1;
                if (ncb >= 2) wait_bar(sm, sm.cb_empty(h), ((ncb >> 1) - 1) & 1, status);
                if (lane == 0) {
                    const uint32_t bytes = 16u << g.v.log2K;
                    mbar_arrive_expect_tx(sm.cb_full(h), bytes);
                    bulk_g2s(sm.cbraw0 + h * sm.cbraw_bytes, g.v.cb, bytes, sm.cb_full(h));
                }
                cur_cb = g.v.cb;
                ++ncb;
            }
            const int nc = n_chunks(g), G = g.v.d_in >> 7;
            for (int c = 0; c < nc; ++c, ++t, ++ts, ring_next(slot, ph, sm.slots)) {
                if (ts == kStartChunks) {  // until the stage's first window is gathered
                    for (uint32_t i = 0; i < kWaitLimit && *reinterpret_cast<volatile int*>(sm.misc + 10) <= s; ++i) {
                        if (*sm.abort_flag()) break;
                        __nanosleep(64);
                    }
                }
                if (t >= sm.slots) wait_bar(sm, sm.empty(slot), ph ^ 1, status);
                if (lane == 0) {
                    const int2 cc = chunk_cols(g, c);
                    const int ng = ((cc.y - 1) >> 4) - (cc.x >> 4) + 1;  // radius groups the chunk touches
                    const uint32_t mb = (uint32_t)((cc.y - cc.x) * g.n_oct * 16), tb = (uint32_t)(ng * g.n_oct * 64);
                    mbar_arrive_expect_tx(sm.full(slot), mb + tb);
                    bulk_g2s_stream(sm.slot_addr(slot), g.v.main + main_word(g.v.R8, g.v.S, g.blk, cc.x, 0, 0), mb,
                                    sm.full(slot), pol);
                    bulk_g2s_stream(sm.slot_addr(slot) + kMainSlot,
                                    g.v.meta + 2 * meta_entry(g.v.R8, G, g.blk, cc.x >> 4, 0, 0), tb, sm.full(slot), pol);
                }
            }
        }
    }
    // the CTA may not exit while bulk copies are in flight
    for (int k = max(0, t - sm.slots); k < t; ++k) wait_bar(sm, sm.full(k % sm.slots), (k / sm.slots) & 1, status);
}

// ------------------------------------------------------------------------
// Activation gather (with the fused prologues)
// ------------------------------------------------------------------------
__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t f2h(float f) { return __half_as_ushort(__float2half_rn(f)); }

// Activation loads of the gather, cached in L1.  Every CTA reads the same few
// KB of sources (an activation row, a norm weight vector, an earlier stage's
// outputs) as scattered 2-byte loads; through L2 alone each one is its own
// L2 request, and all CTAs' requests fall on the same few dozen lines, which
// serialises them at the L2 slices (microseconds per window).  Through L1 a
// CTA asks L2 for each line once.  Staleness: no CTA reads a source before
// it is final -- earlier kernels' outputs after the wait on them
// (griddepcontrol.wait), earlier stages' outputs after the acquire of the
// stage's completion count, which the other gathering warps follow through
// a CTA barrier -- and an acquire at GPU scope invalidates the SM's L1.
__device__ __forceinline__ uint16_t ld16(const uint16_t* p, bool) {
    return __ldca(reinterpret_cast<const unsigned short*>(p));
}

// The stage's prologue applied to the 8 input channels cs[] of batch row xr
// (fp16 bits out).  All operand loads are issued before any is used, so one
// item costs one round trip to L2.
template <int PRO>
__device__ __forceinline__ uint4 prologue8(const EngineStage& st, const JobView& v, int xr, const int (&cs)[8],
                                           float inv, bool coh) {
    uint32_t h[8];
    if (PRO == kProPlain || PRO == kProGqa) {
        const uint16_t* base = PRO == kProPlain ? v.x + (size_t)xr * v.d_in : st.pa + (size_t)xr * st.pro_dim;
        uint16_t a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = PRO == kProPlain ? cs[i] : (cs[i] / (st.gqa_hd * st.gqa_grp)) * st.gqa_hd + cs[i] % st.gqa_hd;
            a[i] = ld16(base + c, coh);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = a[i];
    } else if (PRO == kProRmsNorm || PRO == kProResidRmsNorm) {
        const uint16_t* ra = st.pa + (size_t)xr * st.pro_dim;
        const uint16_t* rb = st.pb + (size_t)xr * st.pro_dim;
        uint16_t a[8], b[8], g[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[i] = ld16(ra + cs[i], coh);
            if (PRO == kProResidRmsNorm) b[i] = ld16(rb + cs[i], coh);
            g[i] = ld16(st.pg + cs[i], false);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float x = h2f(a[i]);
            if (PRO == kProResidRmsNorm) x = h2f(f2h(x + h2f(b[i])));  // the residual stream is fp16
            h[i] = f2h(x * h2f(g[i]) * inv);
        }
    } else {  // kProSiluMul
        const uint16_t* ra = st.pa + (size_t)xr * st.pro_dim;
        const uint16_t* rb = st.pb + (size_t)xr * st.pro_dim;
        uint16_t a[8], b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[i] = ld16(ra + cs[i], coh);
            b[i] = ld16(rb + cs[i], coh);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float gt = h2f(a[i]);
            h[i] = f2h(gt / (1.0f + expf(-gt)) * h2f(b[i]));
        }
    }
    return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
}

// 1 / sqrt(mean(v^2) + eps) of each batch row of the prologue's source vector
// (RMSNorm), computed by the `nt` threads of a cooperative gather in a fixed
// order (deterministic).  Only the first window of a stage needs it.
template <int M>
__device__ void rms_rows(const Smem& sm, const EngineStage& st, int tid, int nt, bool coh) {
    float part[M];
#pragma unroll
    for (int m = 0; m < M; ++m) part[m] = 0.f;
    constexpr int B = 8;  // loads in flight per thread and row
    for (int c0 = tid; c0 < st.pro_dim; c0 += B * nt) {
#pragma unroll
        for (int m = 0; m < M; ++m) {
            uint16_t a[B], b[B];
#pragma unroll
            for (int r = 0; r < B; ++r) {
                const int c = c0 + r * nt;
                a[r] = c < st.pro_dim ? ld16(st.pa + (size_t)m * st.pro_dim + c, coh) : (uint16_t)0;
                b[r] = (st.pro == kProResidRmsNorm && c < st.pro_dim) ? ld16(st.pb + (size_t)m * st.pro_dim + c, coh)
                                                                      : (uint16_t)0;
            }
#pragma unroll
            for (int r = 0; r < B; ++r) {
                float x = h2f(a[r]);
                if (st.pro == kProResidRmsNorm) x = h2f(f2h(x + h2f(b[r])));
                part[m] = fmaf(x, x, part[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < M; ++m)
        for (int o = 16; o; o >>= 1) part[m] += __shfl_xor_sync(0xffffffffu, part[m], o);
    const int wid = tid >> 5;
    if ((tid & 31) == 0)
#pragma unroll
        for (int m = 0; m < M; ++m) sm.red[wid * 8 + m] = part[m];
    named_barrier(kBarGather, kGT);
    if (tid < M) {
        float t = 0.f;
        for (int w = 0; w < nt / 32; ++w) t += sm.red[w * 8 + tid];
        sm.inv_rms[tid] = rsqrtf(t / (float)st.pro_dim + st.eps);
    }
}

// Gathers the window's x_perm for items e = tid, tid + nt, ... of (batch row,
// position) and stores them (fp16) into the window buffer.
//
// Plain inputs: a thread takes kGatherBatch items per round and issues all
// their loads before it uses any, so a round costs one memory round trip,
// not one per item (a window of 8 batch rows has 16 items per lane of a lone
// gather warp).  The fused prologues gather a stage's first window with all
// 288 gathering threads (one item each, typically) and keep one item per
// round: their wider operand sets would not fit the registers left.
constexpr int kGatherBatch = 2;

template <int M, class Src>
__device__ void gather_plain(const Src& src, const Smem& sm, int wlen, int xw, uint32_t xb, int tid, int nt) {
    constexpr int U = kGatherBatch;
    const int total = sm.misc[9] * wlen;  // batch rows a window holds (<= M) x positions
    for (int e0 = tid; e0 < total; e0 += U * nt) {
        uint32_t r[U][8];  // direct rows: r[u][0..3]; permuted: eight fp16 values
        uint32_t dst[U];
        bool zero[U], direct[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * nt;
            const bool live = e < total;
            const int ee = live ? e : e0;  // an item that exists: its loads are harmless
            const int m = ee / wlen, p = ee - m * wlen;
            const uint32_t info = sm.posinfo[p];
            const JobView& v = sm.jc[info >> 20];
            const int j = (int)(info & 0xfffffu);
            dst[u] = live ? xb + (uint32_t)(m * xw + p) * 16 : 0xffffffffu;
            zero[u] = m >= v.Mk;  // rows past a virtual expert's pairs
            const int xr = zero[u] ? 0 : (v.xrows ? v.xrows[m] : m);
            const uint16_t* row = v.x + (size_t)xr * v.d_in;
            direct[u] = !v.perm;
            if (direct[u]) {
                const uint4 q = __ldca(reinterpret_cast<const uint4*>(row + j * 8));
                r[u][0] = q.x; r[u][1] = q.y; r[u][2] = q.z; r[u][3] = q.w;
            } else {
                const uint4 pa = lds128(sm.perm0 + p * 32), pb = lds128(sm.perm0 + p * 32 + 16);
                r[u][0] = ld16(row + (int)pa.x, true); r[u][1] = ld16(row + (int)pa.y, true);
                r[u][2] = ld16(row + (int)pa.z, true); r[u][3] = ld16(row + (int)pa.w, true);
                r[u][4] = ld16(row + (int)pb.x, true); r[u][5] = ld16(row + (int)pb.y, true);
                r[u][6] = ld16(row + (int)pb.z, true); r[u][7] = ld16(row + (int)pb.w, true);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (dst[u] == 0xffffffffu) continue;
            uint4 val = direct[u] ? make_uint4(r[u][0], r[u][1], r[u][2], r[u][3])
                                  : make_uint4(r[u][0] | (r[u][1] << 16), r[u][2] | (r[u][3] << 16),
                                               r[u][4] | (r[u][5] << 16), r[u][6] | (r[u][7] << 16));
            if (zero[u]) val = make_uint4(0, 0, 0, 0);
            sts128(dst[u], val);
        }
    }
}

template <int M, int PRO, class Src>
__device__ void gather_items_k(const Src& src, const Smem& sm, int s, int wlen, int xw, uint32_t xb, int tid,
                               int nt, bool coh) {
    if (PRO == kProPlain) {
        gather_plain<M>(src, sm, wlen, xw, xb, tid, nt);
        return;
    }
    const EngineStage& st = *sm.stc;
    const int mrows = sm.misc[9];  // batch rows a window holds (<= M)
    for (int e = tid; e < mrows * wlen; e += nt) {
        const int m = e / wlen, p = e - m * wlen;
        const uint32_t info = sm.posinfo[p];
        const JobView& v = sm.jc[info >> 20];
        const int j = (int)(info & 0xfffffu);
        uint4 val = make_uint4(0, 0, 0, 0);
        if (m < v.Mk) {
            const int xr = v.xrows ? v.xrows[m] : m;
            if (PRO == kProPlain && !v.perm) {
                const uint16_t* row = v.x + (size_t)xr * v.d_in + j * 8;
                val = __ldca(reinterpret_cast<const uint4*>(row));
            } else {
                int cs[8];
                if (v.perm) {
                    const uint4 pa = lds128(sm.perm0 + p * 32), pb = lds128(sm.perm0 + p * 32 + 16);
                    cs[0] = (int)pa.x; cs[1] = (int)pa.y; cs[2] = (int)pa.z; cs[3] = (int)pa.w;
                    cs[4] = (int)pb.x; cs[5] = (int)pb.y; cs[6] = (int)pb.z; cs[7] = (int)pb.w;
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) cs[i] = j * 8 + i;
                }
                val = prologue8<PRO>(st, v, xr, cs, sm.inv_rms[m < 8 ? m : 0], coh);
            }
        }
        sts128(xb + (uint32_t)(m * xw + p) * 16, val);
    }
}

template <int M, class Src>
__device__ void gather_items(const Src& src, const Smem& sm, int s, int wlen, int xw, uint32_t xb, int tid, int nt,
                             bool coh) {
    switch (sm.stc->pro) {  // uniform: one specialised loop per prologue
        case kProRmsNorm: gather_items_k<M, kProRmsNorm>(src, sm, s, wlen, xw, xb, tid, nt, coh); return;
        case kProResidRmsNorm: gather_items_k<M, kProResidRmsNorm>(src, sm, s, wlen, xw, xb, tid, nt, coh); return;
        case kProSiluMul: gather_items_k<M, kProSiluMul>(src, sm, s, wlen, xw, xb, tid, nt, coh); return;
        case kProGqa: gather_items_k<M, kProGqa>(src, sm, s, wlen, xw, xb, tid, nt, coh); return;
        default: gather_items_k<M, kProPlain>(src, sm, s, wlen, xw, xb, tid, nt, coh); return;
    }
}

// The cooperative part of a stage's first window, run by the gather warp and
// the decode warps together (tid in [0, kGT)).
template <int M, class Src>
__device__ void coop_window(const Src& src, const Smem& sm, int s, int w, int xw, bool coh, int tid) {
    const EngineStage& st = *sm.stc;
    named_barrier(kBarGather, kGT);  // inputs ready, permutation entries landed, buffer free
    if (st.pro == kProRmsNorm || st.pro == kProResidRmsNorm) {
        rms_rows<M>(sm, st, tid, kGT, coh);
        named_barrier(kBarGather, kGT);
    }
    const int wlen = sm.misc[8];
    gather_items<M>(src, sm, s, wlen, xw, sm.xwin(w), tid, kGT, coh);
    named_barrier(kBarGather, kGT);
}

// Loads the permutation entries of the window's positions into the shared
// buffer with plain loads (a bulk copy would queue behind the code chunks
// already in the CTA's copy queue).  posperm holds each position's source.
__device__ void load_perm(const Smem& sm, int wlen, int lane) {
    __syncwarp();  // every lane's position entries are written
    for (int q0 = 0; q0 < 2 * wlen; q0 += 32 * 8) {
        uint4 v[8];
        int dst[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int q = q0 + r * 32 + lane;
            dst[r] = -1;
            if (q < 2 * wlen) {
                const int32_t* pm = sm.posperm[q >> 1];
                if (pm) {
                    v[r] = __ldg(reinterpret_cast<const uint4*>(pm + (q & 1) * 4));
                    dst[r] = q;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
            if (dst[r] >= 0) sts128(sm.perm0 + (uint32_t)dst[r] * 16, v[r]);
    }
    __syncwarp();
}

// Fills window `win` (wlen positions, recorded in posinfo) of stage s.
template <int M, class Src>
__device__ __forceinline__ void fill_window(const Src& src, const Smem& sm, uint32_t* status, unsigned* sync, int s,
                                         int win, int wlen, int xw, bool first, bool need_pdl) {
    const int lane = threadIdx.x & 31;
    const EngineStage& st = src.stage(s);
    load_perm(sm, wlen, lane);  // static data: before any wait on earlier work
    if (need_pdl) pdl_wait();        // inputs may come from the preceding kernel
    if (first && st.wait) {
        if (lane == 0) wait_count(sm, sync + kSyncStageDone + (s - 1), src.stage(s - 1).blocks, status);
        __syncwarp();
    }
    if (win >= 2) wait_bar(sm, sm.x_empty(win & 1), ((win >> 1) - 1) & 1, status);
    const bool coh = st.wait != 0;
    if (lane == 0) sm.misc[8] = wlen;
    __syncwarp();
    if (first) {
        coop_window<M>(src, sm, s, win, xw, coh, kDT + lane);
        if (lane == 0) *reinterpret_cast<volatile int*>(sm.misc + 10) = s + 1;  // release the copy warp
    } else {
        gather_items<M>(src, sm, s, wlen, xw, sm.xwin(win), lane, 32, coh);
    }
    mbar_arrive(sm.x_full(win & 1));  // all 32 lanes, each after its own stores
}

template <int M, class Src>
__device__ void gather_role(const Src& src, const Smem& sm, uint32_t* status, unsigned* sync, int n_cta, int xw,
                            bool waited) {
    const int lane = threadIdx.x & 31;
    WinPos wp{0, 0};
    for (int s = 0; s < src.n_stages(); ++s) {
        const int U = src.units(s);
        if (U <= 0) continue;
        const int u0 = src.cta_u0(s, n_cta, blockIdx.x), u1 = src.cta_u0(s, n_cta, blockIdx.x + 1);
        win_break(wp);
        if (u0 < u1) {  // the stage's descriptor, for this warp and the cooperative gather
            __syncwarp();
            if (lane == 0) *sm.stc = src.stage(s);
            __syncwarp();
        }
        // walk the stage's chunks; a window is filled when the next chunk opens a new one (or at the end)
        int wlen = 0, cur = -1, base = -1, last_id = -1;
        bool first = true;
        for (int u = u0; u < u1;) {
            const Seg g = make_seg(src, s, u, u1);
            u += g.jb - g.ja;
            if (base < 0) base = g.v.id;
            if (g.v.id != last_id) {  // cache the job's view: the gather reads it from shared memory
                if (lane == 0) sm.jc[g.v.id - base] = g.v;
                last_id = g.v.id;
            }
            const int nc = n_chunks(g);
            for (int c = 0; c < nc; ++c) {
                const int2 cc = chunk_cols(g, c);
                const int nj = cc.y - cc.x;
                const int pos = win_place(wp, nj, xw);
                if (wp.win != cur) {
                    if (cur >= 0) {
                        fill_window<M>(src, sm, status, sync, s, cur, wlen, xw, first, !waited);
                        waited = true;
                        first = false;
                    }
                    cur = wp.win;
                    wlen = 0;
                    __syncwarp();  // the filled window's positions are no longer read
                }
                if (lane < nj) {
                    sm.posinfo[pos + lane] = ((uint32_t)(g.v.id - base) << 20) | (uint32_t)(cc.x + lane);
                    sm.posperm[pos + lane] = g.v.perm ? g.v.perm + (size_t)(cc.x + lane) * 8 : nullptr;
                }
                wlen = pos + nj;
            }
        }
        if (cur >= 0) {
            fill_window<M>(src, sm, status, sync, s, cur, wlen, xw, first, !waited);
            waited = true;
        }
    }
    if (!waited) pdl_wait();
}

// ------------------------------------------------------------------------
// Decode warps
// ------------------------------------------------------------------------
// (s (.) c) . x for one subvector: the eight fp16 x fp16 products, exact in
// fp32, summed in fp32 by mixed-precision FMAs (fp16 operands, fp32
// accumulator).  The paper's kernel (Fig. 6a) sums them in fp16 instead; an
// fp16 partial sum rounds at 2^-11 of its own size, which a subvector that
// dominates its output row turns into more than 1e-3 of sum |w||x|.
__device__ __forceinline__ float sdot(uint4 c, uint4 x) {
    float d;
    asm("{\n\t"
        ".reg .f16 c0, c1, c2, c3, c4, c5, c6, c7, x0, x1, x2, x3, x4, x5, x6, x7;\n\t"
        "mov.b32 {c0, c1}, %1;\n\t"
        "mov.b32 {c2, c3}, %2;\n\t"
        "mov.b32 {c4, c5}, %3;\n\t"
        "mov.b32 {c6, c7}, %4;\n\t"
        "mov.b32 {x0, x1}, %5;\n\t"
        "mov.b32 {x2, x3}, %6;\n\t"
        "mov.b32 {x4, x5}, %7;\n\t"
        "mov.b32 {x6, x7}, %8;\n\t"
        "fma.rn.f32.f16 %0, c0, x0, 0f00000000;\n\t"
        "fma.rn.f32.f16 %0, c1, x1, %0;\n\t"
        "fma.rn.f32.f16 %0, c2, x2, %0;\n\t"
        "fma.rn.f32.f16 %0, c3, x3, %0;\n\t"
        "fma.rn.f32.f16 %0, c4, x4, %0;\n\t"
        "fma.rn.f32.f16 %0, c5, x5, %0;\n\t"
        "fma.rn.f32.f16 %0, c6, x6, %0;\n\t"
        "fma.rn.f32.f16 %0, c7, x7, %0;\n\t"
        "}"
        : "=&f"(d)
        : "r"(c.x), "r"(c.y), "r"(c.z), "r"(c.w), "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w));
    return d;
}

struct RowPair {
    float mpA, dlA, mpB, dlB;   // r = mp + dl * (1 + q / 2^V)  (Eq. 2)
    uint32_t auxA, auxB;        // component 6/7 signs of the group's 16 subvectors
};

// Decodes column t (position within the radius group) of both rows of a
// record word w against the batch rows' x_perm values.  The shifts that line
// sign bits up with the fp16 sign positions are integer multiplies by powers
// of two held in registers (d.m*): they issue on the FMA pipe, which the
// fp16 dot products leave room on, instead of the integer ALU pipe that the
// masks and field extraction already load.
template <int MK>
__device__ __forceinline__ void decode_word(const VDec& d, uint32_t rep, uint32_t lane_off, uint32_t w, int t,
                                            const RowPair& rp,
                                            const uint4 (&xv)[MK], float (&accA)[MK], float (&accB)[MK]) {
    {   // row A: z at [7, 7 + log2K), q at [23 - V, 23); signs in slots 0..2 and aux
        uint4 c = cw_load(rep, (w & d.zmask) | lane_off);
        c.x ^= (w * d.m0) & 0x80008000u;
        c.y ^= (w * d.m1) & 0x80008000u;
        c.z ^= (w * d.m2) & 0x80008000u;
        c.w ^= (rp.auxA << (15 - t)) & 0x80008000u;
        const float r = fmaf(__uint_as_float((w & d.qmask) | 0x3F800000u), rp.dlA, rp.mpA);
#pragma unroll
        for (int m = 0; m < MK; ++m) accA[m] = fmaf(r, sdot(c, xv[m]), accA[m]);
    }
    {   // row B: its fields sit 16 bits higher (z, from w >> 16) and lower (q, from w << 16);
        // signs in slots 3..5 (slot 5 at bit 15) and aux
        const uint32_t whi = __umulhi(w, d.m16), wlo = w * d.m16;
        uint4 c = cw_load(rep, (whi & d.zmask) | lane_off);
        c.x ^= (w * d.m3) & 0x80008000u;
        c.y ^= (w * d.m4) & 0x80008000u;
        c.z ^= w & 0x80008000u;
        c.w ^= (rp.auxB << (15 - t)) & 0x80008000u;
        const float r = fmaf(__uint_as_float((wlo & d.qmask) | 0x3F800000u), rp.dlB, rp.mpB);
#pragma unroll
        for (int m = 0; m < MK; ++m) accB[m] = fmaf(r, sdot(c, xv[m]), accB[m]);
    }
}

// Decodes this thread's columns of one chunk (ring slot k) into accA/accB:
// the thread's two rows, in radius group `ch` of the chunk.  xw0: shared
// address of the chunk's first column in its window (batch row stride
// xstride bytes).
template <int MK>
__device__ __forceinline__ void decode_chunk(const Smem& sm, const Seg& g, const VDec& d, int k, int2 cc,
                                             uint32_t xw0, uint32_t xstride, int warp, int lane,
                                             float (&accA)[MK], float (&accB)[MK]) {
    const int u = 32 * (warp & 3) + lane, o = u >> 2, wi = u & 3, part = warp >> 2;
    const int gfirst = cc.x >> 4;
    const int grp = ((cc.x >> 5) << 1) + part;           // this thread's radius group
    const int lo = max(cc.x, grp << 4), hi = min(cc.y, (grp + 1) << 4);
    if (o >= g.n_oct || lo >= hi) return;
    // every load below derives its address from a token taken after the
    // caller's waits on this chunk and its activation window
    const uint32_t tok = order_token();
    const uint32_t base = sm.slot_addr(k) + tok;
    const uint32_t rep = static_cast<uint32_t>(__cvta_generic_to_shared(g_rep)) + tok;
    RowPair rp;
    {
        const uint4 mt = lds128_r(base + kMainSlot + (uint32_t)(((grp - gfirst) * g.n_oct + o) * 64 + wi * 16));
        const float2 a = __half22float2(u2h2(mt.y)), b = __half22float2(u2h2(mt.w));
        rp.dlA = a.y * d.vscale;
        rp.mpA = a.x - rp.dlA;
        rp.dlB = b.y * d.vscale;
        rp.mpB = b.x - rp.dlB;
        rp.auxA = mt.x;
        rp.auxB = mt.z;
    }
    const uint32_t lane_off = (uint32_t)(lane & 7) << 4;  // this lane's replica
    const uint32_t rstride = (uint32_t)g.n_oct * 16;
    const uint32_t wbase = base + (uint32_t)(o * 16 + wi * 4) + (uint32_t)(lo - cc.x) * rstride;
    const uint32_t xbase = xw0 + tok + (uint32_t)(lo - cc.x) * 16;
    if (hi - lo == 16) {  // a whole radius group: fixed trip count, constant shifts
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const uint32_t w = lds32_r(wbase + (uint32_t)t * rstride);
            uint4 xv[MK];
#pragma unroll
            for (int m = 0; m < MK; ++m) xv[m] = lds128_r(xbase + (uint32_t)m * xstride + (uint32_t)t * 16);
            decode_word<MK>(d, rep, lane_off, w, t, rp, xv, accA, accB);
        }
    } else {
#pragma unroll 2
        for (int j = lo; j < hi; ++j) {
            const uint32_t r = (uint32_t)(j - lo);
            const uint32_t w = lds32_r(wbase + r * rstride);
            uint4 xv[MK];
#pragma unroll
            for (int m = 0; m < MK; ++m) xv[m] = lds128_r(xbase + (uint32_t)m * xstride + r * 16);
            decode_word<MK>(d, rep, lane_off, w, j & 15, rp, xv, accA, accB);
        }
    }
    // the chunk's sums exist before the caller releases the ring slot
#pragma unroll
    for (int m = 0; m < MK; ++m) {
        keep(accA[m]);
        keep(accB[m]);
    }
}

__device__ __forceinline__ void write_out(const EngineStage& st, const JobView& v, int m, int row, float tot) {
    const int yr = v.yrows ? v.yrows[m] : m;
    const uint16_t yb = f2h(tot);
    v.y[(size_t)yr * v.d_out + row] = yb;
    if (st.epi == kEpiResidual) {  // layer output: fp16(fp16(ea + eb) + y)
        const size_t i = (size_t)yr * v.d_out + row;
        const uint16_t r = f2h(h2f(__ldcg(reinterpret_cast<const unsigned short*>(st.ea + i))) +
                               h2f(__ldcg(reinterpret_cast<const unsigned short*>(st.eb + i))));
        st.eo[i] = f2h(h2f(r) + h2f(yb));
    }
}
// The same with fp16(ea + eb) loaded ahead (rsum: its fp16 bits).
__device__ __forceinline__ void write_out_pre(const EngineStage& st, const JobView& v, int m, int row, float tot,
                                              uint16_t rsum) {
    const int yr = v.yrows ? v.yrows[m] : m;
    const uint16_t yb = f2h(tot);
    const size_t i = (size_t)yr * v.d_out + row;
    v.y[i] = yb;
    st.eo[i] = f2h(h2f(rsum) + h2f(yb));
}

// The split-K combine of one block by its last contributor: every
// contributor's fp32 partials added in CTA order (8 rows per lane, MKC batch
// rows, 8 / MKC contributors' loads in flight at once), then the outputs.
template <int MKC, int M, class Src>
__device__ __forceinline__ void combine_block(const Src& src, const EngineParams& P, int s, const Seg& g, int c_first,
                                              int c_last, int first_slot, int mk, int lane, bool pre,
                                              const uint16_t (&rsum)[8][M <= 2 ? M : 1]) {
    constexpr int NF = 8 / MKC;
    constexpr int RM = M <= 2 ? M : 1;
    float tot[8][MKC];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int m = 0; m < MKC; ++m) tot[i][m] = 0.f;
    for (int c0 = c_first; c0 <= c_last; c0 += NF) {
        float v[NF][8][MKC];
#pragma unroll
        for (int kk = 0; kk < NF; ++kk) {
            const int c = c0 + kk;
            const int sp = (c == c_first) ? first_slot : 0;
            const bool has = c <= c_last && src.cta_nonempty(s, P.n_cta, c);
            const float* src_p = P.partials + ((size_t)((s * P.n_cta + c) * 2 + sp) * 8) * kBlockRows + lane;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int m = 0; m < MKC; ++m)
                    v[kk][i][m] = (has && m < mk) ? __ldcg(src_p + m * kBlockRows + 32 * i) : 0.f;
        }
#pragma unroll
        for (int kk = 0; kk < NF; ++kk)
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int m = 0; m < MKC; ++m) tot[i][m] += v[kk][i][m];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int row = g.blk * kBlockRows + lane + 32 * i;
        if (row < g.v.d_out)
#pragma unroll
            for (int m = 0; m < MKC; ++m)
                if (m < mk) {
                    if (pre) write_out_pre(src.stage(s), g.v, m, row, tot[i][m], rsum[i][m < RM ? m : 0]);
                    else write_out(src.stage(s), g.v, m, row, tot[i][m]);
                }
    }
}

// Epilogue warps: write (or combine) the outputs of the segments the decode
// warps hand over through the stash ring, so that the decode warps never wait
// on global-memory round trips; two warps take alternate segments, so one
// segment's round trips overlap the next one's.  Whole blocks are written directly.  Split
// blocks: every contributor stores its partial sums and publishes them with
// one acquire-release increment of the block's count; the contributor that
// completes the count adds all partials in CTA order.  Blocks whose outputs
// are final are added to the stage's completion count when a later stage of
// the launch reads them.
template <int M, class Src>
__device__ void epi_role(const Src& src, const Smem& sm, const EngineParams& P, int e) {
    const int lane = threadIdx.x & 31;
    constexpr int NS = Cfg<M>::kSlots;
    // segment n goes to epilogue warp n % NE, so that a warp owns stash slots
    // k = e, e + NE, ... and waits on their phases in order
    constexpr int NE = NS % kEpiWarps == 0 ? kEpiWarps : 1;
    if (e >= NE) return;
    int n = 0;  // segment counter (stash slot n % NS)
    for (int s = 0; s < src.n_stages(); ++s) {
        const int U = src.units(s);
        if (U <= 0) continue;
        const int u0 = src.cta_u0(s, P.n_cta, blockIdx.x), u1 = src.cta_u0(s, P.n_cta, blockIdx.x + 1);
        const bool signal = s + 1 < src.n_stages() && src.stage(s + 1).wait;
        unsigned done = 0;
        for (int uu = u0; uu < u1; ++n) {
            if (n % NE != e) {  // another epilogue warp's segment
                const Seg g = make_seg(src, s, uu, u1);
                uu += g.jb - g.ja;
                continue;
            }
            const int k = n % NS;
            wait_bar(sm, sm.st_full(k), (n / NS) & 1, P.status);
            const Pending& q = sm.pend[k];
            const Seg& g = q.g;
            uu += g.jb - g.ja;
            const float* stk = sm.stash + (size_t)k * kParts * M * kBlockRows;
            // the column parts of a row, added in part order
            auto part_sum = [&](int m, int r) {
                float t = 0.f;
#pragma unroll
                for (int pp = 0; pp < kParts; ++pp) t += stk[(pp * M + m) * kBlockRows + r];
                return t;
            };
            const int mk = g.v.Mk;
            // residual epilogue at batch <= 2: fp16(ea + eb) of this lane's rows is
            // loaded before the split-K round trips, off the critical path
            constexpr int RM = M <= 2 ? M : 1;
            const bool pre = M <= 2 && src.stage(s).epi == kEpiResidual;
            uint16_t rsum[8][RM];
            if (pre) {
                const EngineStage& es = src.stage(s);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int m = 0; m < RM; ++m) {
                        const int row = g.blk * kBlockRows + lane + 32 * i;
                        rsum[i][m] = 0;
                        if (row < g.v.d_out && m < mk) {
                            const int yr = g.v.yrows ? g.v.yrows[m] : m;
                            const size_t e = (size_t)yr * g.v.d_out + row;
                            rsum[i][m] = f2h(h2f(__ldcg(reinterpret_cast<const unsigned short*>(es.ea + e))) +
                                             h2f(__ldcg(reinterpret_cast<const unsigned short*>(es.eb + e))));
                        }
                    }
            }
            if (g.full) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = lane + 32 * i, row = g.blk * kBlockRows + r;
                    if (row < g.v.d_out)
#pragma unroll
                        for (int m = 0; m < M; ++m)
                            if (m < mk) {
                                if (pre) write_out_pre(src.stage(s), g.v, m, row, part_sum(m, r), rsum[i][m < RM ? m : 0]);
                                else write_out(src.stage(s), g.v, m, row, part_sum(m, r));
                            }
                }
                ++done;
            } else {
                float* part = P.partials + ((size_t)((s * P.n_cta + blockIdx.x) * 2 + (q.first ? 0 : 1)) * 8) * kBlockRows;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = lane + 32 * i;
#pragma unroll
                    for (int m = 0; m < M; ++m)
                        if (m < mk) part[m * kBlockRows + r] = part_sum(m, r);
                }
                const int b0 = g.v.unit0 + g.blk * g.v.S;
                const int c_first = src.owner(s, P.n_cta, b0), c_last = src.owner(s, P.n_cta, b0 + g.v.S - 1);
                unsigned* cnt = P.counters + src.stage(s).blk0 + g.v.blk0 + g.blk;
                __syncwarp();  // the warp's partial stores precede the release below
                int last = 0;
                if (lane == 0) {
                    const unsigned old = atom_add_acq_rel_gpu(cnt, 1u);
                    last = old == (unsigned)(src.contributors(s, P.n_cta, c_first, c_last) - 1);
                    if (last) st_relaxed_gpu(cnt, 0u);  // restore for the next call
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {  // add the contributors' partials in CTA order, 8 rows per lane
                    const int first_slot = (src.cta_u0(s, P.n_cta, c_first) >= b0) ? 0 : 1;
                    // batch width of the combine: the segment's own row count (MoE virtual
                    // experts carry 1..8 pairs), so that narrow segments keep more
                    // contributors' loads in flight
                    if (mk <= 1)
                        combine_block<1, M>(src, P, s, g, c_first, c_last, first_slot, mk, lane, pre, rsum);
                    else if (mk <= 2)
                        combine_block<(M < 2 ? M : 2), M>(src, P, s, g, c_first, c_last, first_slot, mk, lane, pre, rsum);
                    else if (mk <= 4)
                        combine_block<(M < 4 ? M : 4), M>(src, P, s, g, c_first, c_last, first_slot, mk, lane, pre, rsum);
                    else
                        combine_block<M, M>(src, P, s, g, c_first, c_last, first_slot, mk, lane, pre, rsum);
                    ++done;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(sm.st_empty(k));
        }
        if (signal && done) {
            __syncwarp();  // the warp's output stores precede the release
            if (lane == 0) red_add_release_gpu(P.sync + kSyncStageDone + s, done);
        }
    }
}

// Decode state carried across segments and stages.
struct DecState {
    int t, slot, ph;      // chunk counter, its ring slot and phase parity
    WinPos wp;
    int cur_win;          // window the decode warps hold (-1: none)
};

// Decodes one segment with compile-time batch MK (<= M, the window's batch
// stride) into this thread's stash slot `si`.
template <int MK, int M, class Src>
__device__ __forceinline__ void seg_body(const Src& src, const Smem& sm, const EngineParams& P, int s, const Seg& g,
                                         DecState& ds, int xw, int nseg, bool first_seg) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u = 32 * (warp & 3) + lane, part = warp >> 2;
    const VDec d = vdec(g.v.log2K);
    float accA[MK], accB[MK];
#pragma unroll
    for (int m = 0; m < MK; ++m) accA[m] = accB[m] = 0.f;
    int t = ds.t, slot = ds.slot, ph = ds.ph, cur_win = ds.cur_win;
    WinPos wp = ds.wp;
    const int nc = n_chunks(g);
    for (int c = 0; c < nc; ++c, ++t, ring_next(slot, ph, sm.slots)) {
        const int2 cc = chunk_cols(g, c);
        const int pos = win_place(wp, cc.y - cc.x, xw);
        if (wp.win != cur_win) {  // release the previous window, wait for this one
            if (cur_win >= 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(sm.x_empty(cur_win & 1));
            }
            wait_bar(sm, sm.x_full(wp.win & 1), (wp.win >> 1) & 1, P.status);
            cur_win = wp.win;
        }
        wait_bar(sm, sm.full(slot), ph, P.status);
        decode_chunk<MK>(sm, g, d, slot, cc, sm.xwin(wp.win) + (uint32_t)pos * 16, (uint32_t)xw * 16, warp, lane,
                         accA, accB);
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.empty(slot));
    }
    ds.t = t;
    ds.slot = slot;
    ds.ph = ph;
    ds.cur_win = cur_win;
    ds.wp = wp;
    // hand this thread's two rows (this column half) to the epilogue warp
    constexpr int NS = Cfg<M>::kSlots;
    const int k = nseg % NS;
    if (nseg >= NS) wait_bar(sm, sm.st_empty(k), ((nseg / NS) - 1) & 1, P.status);
    float* st0 = sm.stash + ((size_t)(k * kParts + part) * M) * kBlockRows;
#pragma unroll
    for (int m = 0; m < MK; ++m) {
        st0[m * kBlockRows + 2 * u] = accA[m];
        st0[m * kBlockRows + 2 * u + 1] = accB[m];
    }
    if (tid == 0) {
        sm.pend[k].g = g;
        sm.pend[k].stage = s;
        sm.pend[k].first = first_seg ? 1 : 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.st_full(k));
}

template <int M, class Src>
__device__ void decode_role(const Src& src, const Smem& sm, const EngineParams& P, int xw) {
    const int tid = threadIdx.x;
    int ncb = 0, nseg = 0;
    const uint16_t* cur_cb = nullptr;
    DecState ds{0, 0, 0, {0, 0}, -1};
    for (int s = 0; s < src.n_stages(); ++s) {
        const int U = src.units(s);
        if (U <= 0) continue;
        const int u0 = src.cta_u0(s, P.n_cta, blockIdx.x), u1 = src.cta_u0(s, P.n_cta, blockIdx.x + 1);
        win_break(ds.wp);
        if (u0 < u1) {
            // the stage's first window, gathered together with the gather warp
            // here, where no decode state is live
            if (ds.cur_win >= 0) {
                __syncwarp();
                if ((tid & 31) == 0) mbar_arrive(sm.x_empty(ds.cur_win & 1));
                ds.cur_win = -1;
            }
            coop_window<M>(src, sm, s, ds.wp.win, xw, src.stage(s).wait != 0, tid);
        }
        bool first_seg = true;
        for (int uu = u0; uu < u1; ++nseg) {
            const Seg g = make_seg(src, s, uu, u1);
            uu += g.jb - g.ja;
            if (g.v.cb != cur_cb) {  // rebuild the 8 bank-rotated replicas from the raw copy
                const int h = ncb & 1;
                if (cur_cb) named_barrier(kBarDecode, kDT);
                wait_bar(sm, sm.cb_full(h), (ncb >> 1) & 1, P.status);
                const int K = 1 << g.v.log2K;
                const uint32_t raw = sm.cbraw0 + h * sm.cbraw_bytes;
                for (int e = tid; e < K * 8; e += kDT) sts128(sm.cb0 + e * 16, lds128(raw + (e >> 3) * 16));
                named_barrier(kBarDecode, kDT);
                if (tid == 0) mbar_arrive(sm.cb_empty(h));
                cur_cb = g.v.cb;
                ++ncb;
            }
            if (Src::kVarBatch) {  // virtual experts carry 1..8 pairs
                const int mk = g.v.Mk;
                if (mk <= 1) seg_body<1, M>(src, sm, P, s, g, ds, xw, nseg, first_seg);
                else if (mk <= 2) seg_body<(M < 2 ? M : 2), M>(src, sm, P, s, g, ds, xw, nseg, first_seg);
                else if (mk <= 4) seg_body<(M < 4 ? M : 4), M>(src, sm, P, s, g, ds, xw, nseg, first_seg);
                else seg_body<M, M>(src, sm, P, s, g, ds, xw, nseg, first_seg);
            } else {
                seg_body<M, M>(src, sm, P, s, g, ds, xw, nseg, first_seg);
            }
            first_seg = false;
        }
    }
    if (ds.cur_win >= 0) {
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(sm.x_empty(ds.cur_win & 1));
    }
}

template <int M, class Src>
__device__ void run(const Src& src, const EngineParams& P, uint8_t* smem_raw, int xw, int mrows, bool waited) {
    const Smem sm = carve<M>(smem_raw, P.slots, P.kmax);
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int k = 0; k < kMaxSlots; ++k) {
            mbar_init(sm.full(k), 1);
            mbar_init(sm.empty(k), kDW);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(sm.cb_full(h), 1);
            mbar_init(sm.cb_empty(h), 1);
            mbar_init(sm.x_full(h), 32);
            mbar_init(sm.x_empty(h), kDW);
        }
        mbar_init(sm.perm_full(), 1);
        for (int k = 0; k < kStashSlots; ++k) {
            mbar_init(sm.st_full(k), kDW);
            mbar_init(sm.st_empty(k), 1);
        }
        fence_mbar_init();
        for (int i = 0; i < 64; ++i) sm.misc[i] = 0;
        sm.misc[9] = mrows;
        for (int i = 0; i < 8; ++i) sm.inv_rms[i] = 1.f;
    }
    __syncthreads();
    if (warp == kCopyWarp) {
        copy_role(src, sm, P.status, P.n_cta);
    } else if (warp == kGatherWarp) {
        gather_role<M>(src, sm, P.status, P.sync, P.n_cta, xw, waited);
    } else if (warp >= kEpiWarp) {
        epi_role<M>(src, sm, P, warp - kEpiWarp);
    } else {
        decode_role<M>(src, sm, P, xw);
    }
    __syncthreads();
    // the last CTA out restores the stage completion counts for the next call
    if (tid == 0 && P.uses_sync) {
        const unsigned old = atom_add_acq_rel_gpu(P.sync + kSyncExit, 1u);
        if (old == (unsigned)(P.n_cta - 1)) {
            for (int s = 0; s < kMaxStages; ++s) st_relaxed_gpu(P.sync + kSyncStageDone + s, 0u);
            st_relaxed_gpu(P.sync + kSyncExit, 0u);
        }
    }
}

template <int M>
__global__ void __launch_bounds__(kThreads, 1) engine_kernel(const __grid_constant__ EngineParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    pdl_launch_dependents();
    const DenseSrc src{p};
    run<M>(src, p, smem_raw, Cfg<M>::kXW, M, false);
}

// Virtual experts carry 1..8 pairs each; the kernel's batch stride is 8.
// Grouped-expert GEMV.  Every CTA groups the (token, slot) pairs by expert
// itself -- in expert order and, within an expert, in pair order, into virtual
// experts of at most 8 pairs -- and keeps the virtual experts that its unit
// range covers; all CTAs derive the same grouping from the same pairs
// (deterministic), and no routing kernel or routing round trip precedes the
// decode.
__global__ void __launch_bounds__(kThreads, 1) moe_kernel(const __grid_constant__ MoeParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ MoeStage ms;
    __shared__ int s_m2;
    int* const s_cnt = ms.cnt;
    int* const s_first = ms.first;
    constexpr int MV = kMaxPairsPerVirtual;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, n_e = p.n_experts;
    pdl_launch_dependents();
    pdl_wait();  // the pairs and x come from the preceding kernel
    for (int e = tid; e < n_e; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    for (int q = tid; q < p.n_pairs; q += blockDim.x) {
        const int e = __ldca(p.pair_expert + q);
        if (e >= 0 && e < n_e) atomicAdd(&s_cnt[e], 1);
        else if (blockIdx.x == 0) flag(p.e.status, kDevUnsupported);  // that pair's output is not written
    }
    __syncthreads();
    const int upv = ((((p.d_out + 7) >> 3) + kOct - 1) / kOct) * (p.d_in >> 3);
    if (warp == 0) {  // exclusive scans of the virtual-expert counts and costs, 32 experts at a time
        int carry = 0;
        long long ccarry = 0;
        for (int e0 = 0; e0 < n_e; e0 += 32) {
            const int e = e0 + lane;
            const int c = e < n_e ? s_cnt[e] : 0, full = c / MV, tail = c - full * MV;
            const int v = full + (tail > 0 ? 1 : 0);
            const long long w = (long long)upv * (full * MV + (tail > 0 ? moe_weight(tail) : 0));
            int incl = v;
            long long wincl = w;
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                const long long tw = __shfl_up_sync(0xffffffffu, wincl, o);
                if (lane >= o) {
                    incl += t;
                    wincl += tw;
                }
            }
            if (e < n_e) {
                s_first[e] = carry + incl - v;
                ms.cost[e] = ccarry + wincl - w;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
            ccarry += __shfl_sync(0xffffffffu, wincl, 31);
        }
        if (lane == 0) {
            s_first[n_e] = carry;
            ms.cost[n_e] = ccarry;
            ms.cost_total = ccarry;
            ms.n_e = n_e;
            ms.upv = upv;
            ms.n_virtual = carry;
            ms.units = carry * upv;
        }
    }
    __syncthreads();
    const MoeSrc src{p, ms};
    for (int c = tid; c <= p.e.n_cta; c += blockDim.x) ms.bound[c] = src.cost_bound(p.e.n_cta, c);
    __syncthreads();
    if (tid == 0) {
        const int u0 = src.cta_u0(0, p.e.n_cta, blockIdx.x), u1 = src.cta_u0(0, p.e.n_cta, blockIdx.x + 1);
        ms.vi0 = u0 / upv;
        const int need = u1 > u0 ? (u1 - 1) / upv - ms.vi0 + 1 : 0;
        ms.nvi = min(kMoeCache, need);
        ms.overflow = need > kMoeCache;
        if (ms.overflow) flag(p.e.status, kDevUnsupported);
    }
    __syncthreads();
    // the pairs of the CTA's virtual experts: one warp per expert whose virtual
    // experts meet [vi0, vi0 + nvi), ranking its pairs by a ballot over the pair list
    const int v0 = ms.vi0, v1 = ms.vi0 + ms.nvi;
    for (int e = warp; e < n_e; e += kThreads / 32) {
        const int f0 = s_first[e], f1 = s_first[e + 1];
        if (f1 <= v0 || f0 >= v1) continue;
        int k = 0;  // pairs of expert e before this round
        for (int q0 = 0; q0 < p.n_pairs; q0 += 32) {
            const int q = q0 + lane;
            const bool hit = q < p.n_pairs && __ldca(p.pair_expert + q) == e;
            const unsigned b = __ballot_sync(0xffffffffu, hit);
            if (hit) {
                const int kk = k + __popc(b & ((1u << lane) - 1u));
                const int vi = f0 + kk / MV;
                if (vi >= v0 && vi < v1) {
                    ms.v_xrows[vi - v0][kk % MV] = __ldca(p.pair_xrow + q);
                    ms.v_yrows[vi - v0][kk % MV] = q;
                }
            }
            k += __popc(b);
        }
        for (int vi = max(f0, v0) + lane; vi < min(f1, v1); vi += 32) {
            ms.v_expert[vi - v0] = e;
            ms.v_count[vi - v0] = min(MV, s_cnt[e] - (vi - f0) * MV);
        }
    }
    __syncthreads();
    // the window holds the largest pair count of this CTA's virtual experts
    if (tid == 0) {
        int mmax = 1;
        for (int k = 0; k < ms.nvi; ++k) mmax = max(mmax, ms.v_count[k]);
        int m2 = 1;
        while (m2 < mmax) m2 <<= 1;
        s_m2 = m2;
    }
    __syncthreads();
    if (ms.overflow) return;  // more virtual experts than the staging holds (flagged above)
    run<kMaxPairsPerVirtual>(src, p.e, smem_raw, kXBufBytes / (16 * s_m2), s_m2, true);
}

// ------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------
long long units_of(const sage_matrix& A) {
    const long long R8 = ((long long)A.d_out + 7) / 8;
    return (R8 + kOct - 1) / kOct * (long long)(A.d_in / 8);
}
long long blocks_of(const sage_matrix& A) { return (((long long)A.d_out + 7) / 8 + kOct - 1) / kOct; }
size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Dynamic shared memory per CTA: 227 KB less the static replicas (32 KB) and a
// little static headroom.
constexpr int kSmemBudget = 227 * 1024 - (int)sizeof(g_rep) - 1024;

template <int M>
int slots_for(long long max_units_per_cta, int kmax, int budget) {
    const long long chunks = (max_units_per_cta + kChunkJ - 1) / kChunkJ + 2;
    int n = (int)std::min<long long>(kMaxSlots, std::max<long long>(2, chunks));
    while (n > 2 && smem_bytes<M>(n, kmax) > budget) --n;
    return n;
}

template <class K, class Params>
int launch_pdl(K kernel, const Params& p, int grid, int smem, sage_stream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

// Grid size of an engine launch: one CTA per SM, fewer when there is little work.
int engine_ctas(long long max_stage_units) {
    return (int)std::max<long long>(1, std::min<long long>(current_sm_count(), std::max<long long>(1, max_stage_units / 4)));
}

}  // namespace

size_t engine_workspace_bytes(const EngineStageSpec* stages, int n_stages) {
    long long blocks = 0, umax = 0;
    for (int s = 0; s < n_stages; ++s) {
        long long u = 0;
        for (int i = 0; i < stages[s].n_jobs; ++i) {
            blocks += blocks_of(stages[s].jobs[i].A);
            u += units_of(stages[s].jobs[i].A);
        }
        umax = std::max(umax, u);
    }
    const int n_cta = engine_ctas(umax);
    return kWsHeader + round256((size_t)blocks * 4) + (size_t)n_stages * n_cta * 2 * 8 * kBlockRows * sizeof(float);
}

template <int M>
static int launch_engine_m(const EngineStageSpec* stages, int n_stages, void* ws, sage_stream_t stream) {
    static EngineParams p;  // large: keep off the stack
    static std::mutex mu;
    static SmemLimit limit;
    std::lock_guard<std::mutex> lock(mu);
    p = EngineParams{};
    int nj = 0, kmax = 16;
    long long blk_total = 0, umax = 0;
    bool uses_sync = false;
    for (int s = 0; s < n_stages; ++s) {
        const EngineStageSpec& ss = stages[s];
        EngineStage& st = p.st[s];
        st = ss.stage;
        st.job0 = nj;
        st.n_jobs = ss.n_jobs;
        st.blk0 = (int)blk_total;
        long long unit = 0, blk = 0;
        for (int i = 0; i < ss.n_jobs; ++i) {
            const sage_matrix& A = ss.jobs[i].A;
            EngineJob& d = p.jobs[nj++];
            d.main = A.main; d.meta = A.meta; d.cb = A.codebook; d.perm = A.perm;
            d.x = ss.jobs[i].x; d.y = ss.jobs[i].y;
            d.d_out = A.d_out; d.d_in = A.d_in; d.log2K = A.log2K;
            d.unit0 = (int)unit;
            d.blk0 = (int)blk;
            kmax = std::max(kmax, 1 << A.log2K);
            unit += units_of(A);
            blk += blocks_of(A);
        }
        if (unit >= (1ll << 31) / 2) return SAGE_ERR_UNSUPPORTED;
        st.units = (int)unit;
        st.blocks = (int)blk;
        blk_total += blk;
        umax = std::max(umax, unit);
        if (s > 0 && st.wait) uses_sync = true;
    }
    const int n_cta = engine_ctas(umax);
    long long widest = 0;
    for (int s = 0; s < n_stages; ++s) widest += (p.st[s].units + n_cta - 1) / n_cta;
    p.n_stages = n_stages;
    p.n_cta = n_cta;
    p.M = M;
    p.kmax = kmax;
    p.slots = slots_for<M>(widest, kmax, kSmemBudget);
    p.uses_sync = uses_sync ? 1 : 0;
    const int smem = smem_bytes<M>(p.slots, kmax);
    if (smem > kSmemBudget) return SAGE_ERR_UNSUPPORTED;
    if (!limit.ensure(engine_kernel<M>, smem)) return SAGE_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.status = reinterpret_cast<uint32_t*>(w);
    p.sync = reinterpret_cast<unsigned*>(w);
    p.counters = reinterpret_cast<unsigned*>(w + kWsHeader);
    p.partials = reinterpret_cast<float*>(w + kWsHeader + round256((size_t)blk_total * 4));
    return launch_pdl(engine_kernel<M>, p, n_cta, smem, stream);
}

int launch_engine(const EngineStageSpec* stages, int n_stages, int M, void* ws, size_t ws_bytes, sage_stream_t stream) {
    if (n_stages < 1 || n_stages > kMaxStages) return SAGE_ERR_UNSUPPORTED;
    int nj = 0;
    for (int s = 0; s < n_stages; ++s) nj += stages[s].n_jobs;
    if (nj > kMaxJobs) return SAGE_ERR_UNSUPPORTED;
    if (ws_bytes < engine_workspace_bytes(stages, n_stages)) return SAGE_ERR_WORKSPACE;
    switch (M) {
        case 1: return launch_engine_m<1>(stages, n_stages, ws, stream);
        case 2: return launch_engine_m<2>(stages, n_stages, ws, stream);
        case 3: return launch_engine_m<3>(stages, n_stages, ws, stream);
        case 4: return launch_engine_m<4>(stages, n_stages, ws, stream);
        case 5: return launch_engine_m<5>(stages, n_stages, ws, stream);
        case 6: return launch_engine_m<6>(stages, n_stages, ws, stream);
        case 7: return launch_engine_m<7>(stages, n_stages, ws, stream);
        case 8: return launch_engine_m<8>(stages, n_stages, ws, stream);
        default: return SAGE_ERR_UNSUPPORTED;
    }
}

// One stage of plain GEMVs (sage_gemv, sage_gemv_grouped).
size_t gemv_workspace_bytes(const sage_matrix* mats, int n, int M) {
    (void)M;
    std::vector<EngineJobSpec> jobs((size_t)n);
    for (int i = 0; i < n; ++i) jobs[i].A = mats[i];
    EngineStageSpec st{};
    st.jobs = jobs.data();
    st.n_jobs = n;
    return engine_workspace_bytes(&st, 1);
}

int launch_gemv(const GemvJob* jobs, int n, int M, void* ws, size_t ws_bytes, sage_stream_t stream) {
    std::vector<EngineJobSpec> js((size_t)n);
    for (int i = 0; i < n; ++i) {
        js[i].A = jobs[i].A;
        js[i].x = jobs[i].x;
        js[i].y = jobs[i].y;
    }
    EngineStageSpec st{};
    st.jobs = js.data();
    st.n_jobs = n;
    st.stage.pro = kProPlain;
    st.stage.epi = kEpiPlain;
    return launch_engine(&st, 1, M, ws, ws_bytes, stream);
}

// MoE workspace: header | split-K counters | partials
namespace {
struct MoeWs {
    size_t counters, partials, total;
};
MoeWs moe_ws_layout(int n_pairs, int d_out, int n_cta) {
    MoeWs L;
    size_t o = kWsHeader;
    const int nblk = ((d_out + 7) / 8 + kOct - 1) / kOct;
    L.counters = o; o += round256((size_t)n_pairs * nblk * 4);
    L.partials = o; o += (size_t)n_cta * 2 * 8 * kBlockRows * sizeof(float);
    L.total = o;
    return L;
}
}  // namespace

size_t moe_workspace_bytes(const sage_matrix* experts, int n_experts, int n_pairs) {
    (void)n_experts;
    return moe_ws_layout(std::max(1, n_pairs), experts[0].d_out, current_sm_count()).total;
}

int launch_moe(const sage_matrix* experts, int n_experts, const int32_t* pair_expert, const int32_t* pair_xrow,
               int n_pairs, const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes, sage_stream_t stream) {
    constexpr int MV = kMaxPairsPerVirtual;
    constexpr int kMoeStatic = (int)(sizeof(MoeStage) + 16);
    if (n_experts > kMaxExperts) return SAGE_ERR_UNSUPPORTED;
    const int n_cta = std::min(current_sm_count(), kMaxMoeCtas);
    const MoeWs L = moe_ws_layout(n_pairs, experts[0].d_out, n_cta);
    if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    static MoeParams p;
    static std::mutex mu;
    static SmemLimit limit;
    std::lock_guard<std::mutex> lock(mu);
    p = MoeParams{};
    int kmax = 16;
    for (int e = 0; e < n_experts; ++e) kmax = std::max(kmax, 1 << experts[e].log2K);
    p.e.n_stages = 1;
    p.e.n_cta = n_cta;
    p.e.M = MV;
    p.e.kmax = kmax;
    p.e.slots = slots_for<MV>(1 << 30, kmax, kSmemBudget - kMoeStatic);
    p.e.uses_sync = 0;
    const int smem = smem_bytes<MV>(p.e.slots, kmax);
    if (smem > kSmemBudget - kMoeStatic) return SAGE_ERR_UNSUPPORTED;
    if (!limit.ensure(moe_kernel, smem)) return SAGE_ERR_CUDA;
    p.e.status = reinterpret_cast<uint32_t*>(w);
    p.e.sync = reinterpret_cast<unsigned*>(w);
    p.e.counters = reinterpret_cast<unsigned*>(w + L.counters);
    p.e.partials = reinterpret_cast<float*>(w + L.partials);
    p.st.pro = kProPlain;
    p.st.epi = kEpiPlain;
    p.st.blk0 = 0;
    p.n_experts = n_experts;
    p.d_out = experts[0].d_out;
    p.d_in = experts[0].d_in;
    p.n_pairs = n_pairs;
    p.x = x;
    p.y = y;
    p.pair_expert = pair_expert;
    p.pair_xrow = pair_xrow;
    for (int e = 0; e < n_experts; ++e) {
        p.experts[e].main = experts[e].main;
        p.experts[e].meta = experts[e].meta;
        p.experts[e].cb = experts[e].codebook;
        p.experts[e].perm = experts[e].perm;
        p.experts[e].log2K = experts[e].log2K;
    }
    return launch_pdl(moe_kernel, p, n_cta, smem, stream);
}

}  // namespace sage
