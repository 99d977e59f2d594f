// Packed SAGE GEMV for batch 1..8 on sm_100a (decode path, Sec. 3.5 and App. A.1
// of "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World Usability"),
// its grouped multi-matrix form, and the grouped-expert MoE GEMV.
//
// Work decomposition (B200-first, not the paper's RTX 4090 tiling):
//  * A "unit" is one subvector column j of one 256-row block (32 row octets) of
//    one matrix: a 512-byte slab of the main plane.  The units of all matrices
//    of a launch are flattened (matrix, block, j) and cut into one contiguous
//    range per CTA of a persistent grid (one CTA per SM).  Dense launches are
//    planned on the host (each matrix gets its own CTAs when that costs little
//    balance); MoE launches are planned on the device from the routing.
//  * Two producer warps per CTA.  The copy warp bulk-copies (1-D TMA) the
//    codebooks and, chunk by chunk (16 columns = one radius group), the code
//    records and grid/aux meta into a ring of shared-memory slots, without
//    waiting on the preceding kernel (programmatic dependent launch): none of
//    it is written there.  The activation warp gathers the ESG-permuted
//    x_perm[p] = x[perm[p]] window by window (Sec. 3.5 fuses this gather into
//    the decode GEMV); the permutation entries are copied before the wait on
//    the preceding kernel, only x after it.
//  * Decode warps (dense launches): one thread per row of the 256-row block
//    for the whole segment; it reads its row's half of a record word per
//    column and accumulates the row's outputs itself.  The MoE kernel keeps
//    an octet-per-lane body: lane l decodes the 16-byte record of row octet l
//    (8 rows) per column, and the warps' partial sums are reduced in shared
//    memory.
//  * Per subvector: the codeword address and the radius code each come out of
//    one logic op (format v2), the codeword is one conflict-free 128-bit shared
//    load (8 bank-rotated replicas of the codebook), the signs are XORed into
//    the fp16 sign bits, four half2 FMAs form (s (.) c) . x with fp16 local
//    accumulation (Fig. 6a), and r = mu + q delta (Eq. 2) is applied once, fp32.
//  * Rows whose columns are split between CTAs are combined deterministically:
//    partial sums go to the workspace and the last CTA to finish a block adds
//    them in CTA order (the paper's FP32 split-K combine for small grids).
//    A CTA defers its outputs to the end so that no segment waits for another
//    segment's global round trips.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
using namespace dev;

namespace {

constexpr int kMaxMats = 64;
constexpr int kMaxExperts = 256;
constexpr int kMaxPairsPerVirtual = 8;
constexpr int kOct = 32;               // row octets per block (one per lane)
constexpr int kBlockRows = kOct * 8;
constexpr int kChunkJ = 16;            // a chunk lies inside one radius group
constexpr int kMaxSegs = 4;            // segments stashed before outputs are flushed
constexpr int kMainSlot = kChunkJ * kOct * 16;  // 8 KB of code records
constexpr int kMetaSlot = kOct * 64;            // 2 KB: one group of 256 rows
constexpr int kSlot = kMainSlot + kMetaSlot;    // one ring slot = one chunk
constexpr int kMaxSlots = 16;                   // ring depth limit
constexpr int kSegTab = 32;                     // segment-table capacity per round
constexpr int kSegBytes = 160;                  // shared memory per table entry
// Named barriers besides the decode warps' own (id 1): the activation and
// copy warps (id 3) and the activation and decode warps (id 2).
constexpr int kBarPermIssued = 3;
constexpr int kBarFirstWindow = 2;

template <int M>
struct Cfg {
    static constexpr int kW = 8;                       // decode warps
    static constexpr int kThreads = (kW + 2) * 32;     // + copy warp + activation warp
    static constexpr int kDecodeThreads = kW * 32;
    // Columns per activation window: x_perm for a window is gathered in one go.
    static constexpr int kXW = (M == 1) ? 256 : (M == 2) ? 128 : (M <= 4) ? 64 : 32;
    static constexpr int kXBuf = kXW * M * 16;         // one window of x_perm, [m][column]
    static constexpr int kPermBuf = kXW * 32;          // the window's permutation entries
    static constexpr int kPosInfo = kXW * 4;           // (segment, column) of each window position
    // cross-warp reduction buffer: only the MoE kernel's segment body (batch 8) uses one
    static constexpr int kRed = (M == kMaxPairsPerVirtual) ? kW * 8 * M * 32 * 4 : 0;
    static constexpr int kStash = kMaxSegs * M * kBlockRows * 4;
    static constexpr int kBars = (2 * kMaxSlots + 9) * 8;
    static constexpr int kFixed = 2 * kXBuf + kPermBuf + kPosInfo + kRed + kStash + kSegTab * kSegBytes + kBars + 64;
    // codebook replicas (K_max * 8 * 16) + 2 raw codebooks + ring + fixed
    static int smem(int slots, int kmax) { return kmax * 128 + 2 * kmax * 16 + slots * kSlot + kFixed; }
};

// One matrix as the kernel sees it while working on one of its segments.
struct MatView {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const int32_t* perm;
    const uint16_t* x;      // activations, row stride d_in
    uint16_t* y;            // outputs, row stride d_out
    const int32_t* xrows;   // [Mk] activation row of batch slot m (null: m); shared or global memory
    const int32_t* yrows;   // [Mk] output row of batch slot m (null: m); shared or global memory
    long long unit0;
    int d_out, d_in, log2K, R8, S, blk0, Mk;
};

struct DenseMat {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const int32_t* perm;
    const uint16_t* x;
    uint16_t* y;
    long long unit0, units;
    int d_out, d_in, log2K, blk0;
    int cta0, ncta;        // CTAs [cta0, cta0 + ncta) own this matrix (per-matrix plans)
};

struct ExpertMat {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const int32_t* perm;
    int log2K, pad;
};

struct Common {
    int n_cta;
    int M;                 // dense: batch; MoE: 0 (per virtual expert)
    int slots;             // ring depth (chunks in flight)
    int n_wg;              // decode warp groups (1, 2 or 4); chunk t goes to group t % n_wg
    int kmax;              // largest codebook of the launch (replica area size)
    uint32_t* status;
    unsigned* counters;
    float* partials;       // [n_cta][2][8][kBlockRows]
};

// CTA c covers units [first(c), first(c + 1)).  Stream-K plans split the
// flattened units evenly; per-matrix plans give matrix k its own CTAs and
// split its units evenly among them.  Both are plain arithmetic, so no
// dependent parameter-space loads sit on any critical path.
constexpr int kMaxCta = 256;

struct DenseParams {
    Common c;
    long long total_units;
    int n_mats;
    int per_matrix;
    int cta_start[kMaxCta + 1];   // first unit of each CTA; cta_start[n_cta] = total_units
    DenseMat mats[kMaxMats];
};

struct MoeRoute {
    int n_virtual;
    int pad[3];
};
struct MoeParams {
    Common c;
    int n_experts, d_out, d_in, n_pairs;
    const uint16_t* x;
    uint16_t* y;
    const MoeRoute* route;         // ws
    const int32_t* v_expert;       // ws [n_pairs]
    const int32_t* v_xrows;        // ws [n_pairs][8]
    const int32_t* v_yrows;        // ws [n_pairs][8]
    const int32_t* v_count;        // ws [n_pairs]
    ExpertMat experts[kMaxExperts];
};

// The CTA start table and the matrix descriptors are read from shared-memory
// copies: dependent loads from the parameter space miss the constant cache.
struct DenseProblem {
    const DenseParams& p;
    const int* cs;        // shared copy of p.cta_start
    const DenseMat* ms;   // shared copy of p.mats
    __device__ long long total() const { return p.total_units; }
    __device__ long long cta_begin(int c) const { return cs[min(c, p.c.n_cta)]; }
    __device__ int cta_of(long long u) const {  // the CTA whose range holds unit u
        int lo = 0, hi = p.c.n_cta - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cs[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    }
    __device__ MatView view(long long u) const {
        int k = 0;
        while (k + 1 < p.n_mats && ms[k + 1].unit0 <= u) ++k;
        const DenseMat& d = ms[k];
        MatView v;
        v.main = d.main; v.meta = d.meta; v.cb = d.cb; v.perm = d.perm; v.x = d.x; v.y = d.y;
        v.xrows = nullptr; v.yrows = nullptr; v.unit0 = d.unit0;
        v.d_out = d.d_out; v.d_in = d.d_in; v.log2K = d.log2K;
        v.R8 = (d.d_out + 7) >> 3; v.S = d.d_in >> 3;
        v.blk0 = d.blk0; v.Mk = p.c.M;
        return v;
    }
};

// The routing results this CTA needs (virtual-expert count, and the expert
// and pair count of the virtual experts its range touches, with their
// descriptors) are staged in shared memory once, after the routing kernel.
constexpr int kMoeCache = 32;
struct MoeStage {
    long long total;
    int vi0, nvi;
    int v_expert[kMoeCache];
    int v_count[kMoeCache];
    int v_xrows[kMoeCache][kMaxPairsPerVirtual];  // activation / output rows of the cached virtual experts
    int v_yrows[kMoeCache][kMaxPairsPerVirtual];
    ExpertMat emat[kMoeCache];
};

struct MoeProblem {
    const MoeParams& p;
    const MoeStage& st;
    __device__ int R8() const { return (p.d_out + 7) >> 3; }
    __device__ long long upv() const { return (long long)((R8() + kOct - 1) / kOct) * (p.d_in >> 3); }
    __device__ long long total() const { return st.total; }
    __device__ long long cta_begin(int c) const { return (long long)c * st.total / p.c.n_cta; }
    __device__ int cta_of(long long u) const {
        const long long t = st.total;
        return (int)(((u + 1) * p.c.n_cta + t - 1) / t) - 1;
    }
    __device__ MatView view(long long u) const {
        const long long per = upv();
        const int vi = (int)(u / per);
        const int k = vi - st.vi0;
        const bool cached = k >= 0 && k < st.nvi;
        const int e = cached ? st.v_expert[k] : __ldcg(p.v_expert + vi);
        const ExpertMat& d = cached ? st.emat[k] : p.experts[e];
        MatView v;
        v.main = d.main; v.meta = d.meta; v.cb = d.cb; v.perm = d.perm; v.x = p.x; v.y = p.y;
        v.xrows = cached ? st.v_xrows[k] : p.v_xrows + (size_t)vi * kMaxPairsPerVirtual;
        v.yrows = cached ? st.v_yrows[k] : p.v_yrows + (size_t)vi * kMaxPairsPerVirtual;
        v.unit0 = (long long)vi * per;
        v.d_out = p.d_out; v.d_in = p.d_in; v.log2K = d.log2K;
        v.R8 = R8(); v.S = p.d_in >> 3;
        v.blk0 = vi * ((v.R8 + kOct - 1) / kOct);
        v.Mk = cached ? st.v_count[k] : __ldcg(p.v_count + vi);
        return v;
    }
};

// Batch-slot row of a virtual expert: from the CTA's staged copy in shared
// memory, or (experts outside the staged range) from the workspace in L2.
__device__ __forceinline__ int row_at(const int32_t* rows, int m) {
    return __isShared(rows) ? rows[m] : __ldcg(rows + m);
}

// A segment: one matrix, one 256-row block, columns [ja, jb), plus what the
// split-K combine needs.  Each CTA builds its segment table once, in shared
// memory, so no role ever walks the parameter tables again.
struct Seg {
    MatView v;
    unsigned* counter;      // split blocks: arrival counter
    int blk, ja, jb, n_oct, n_chunks;
    int full;               // the segment covers all columns of its block
    int c_first, c_last;    // CTAs contributing to the block (split blocks)
    int first_slot;         // partial-sum slot of c_first for this block
    int my_slot;            // this CTA's partial-sum slot for this block
};
static_assert(sizeof(Seg) <= kSegBytes, "segment table entry outgrew its shared-memory budget");

template <class Problem>
__device__ Seg make_seg(const Problem& P, long long u, long long u_end, long long cta_u0) {
    Seg s;
    s.v = P.view(u);
    const int local = (int)(u - s.v.unit0);  // unit counts fit in 32 bits (checked on the host)
    s.blk = local / s.v.S;
    s.ja = local - s.blk * s.v.S;
    const long long jb = (long long)s.ja + (u_end - u);
    s.jb = (int)(jb < (long long)s.v.S ? jb : (long long)s.v.S);
    s.n_oct = min(kOct, s.v.R8 - s.blk * kOct);
    s.n_chunks = ((s.jb - 1) >> 4) - (s.ja >> 4) + 1;
    s.full = (s.ja == 0 && s.jb == s.v.S);
    s.counter = nullptr;
    s.c_first = s.c_last = s.first_slot = s.my_slot = 0;
    (void)cta_u0;
    return s;
}

// Split-K bookkeeping of a segment whose block is shared with other CTAs:
// the contributing CTAs, the partial-sum slots and the arrival counter.  Run
// by one lane per segment, in parallel, after the segments are laid out.
template <class Problem>
__device__ void seg_split_info(const Problem& P, const Common& C, Seg& s, long long cta_u0) {
    if (s.full) return;
    const long long b0 = s.v.unit0 + (long long)s.blk * s.v.S;
    s.c_first = P.cta_of(b0);
    s.c_last = P.cta_of(b0 + s.v.S - 1);
    s.first_slot = (P.cta_begin(s.c_first) >= b0) ? 0 : 1;
    s.my_slot = (cta_u0 >= b0) ? 0 : 1;
    s.counter = C.counters + s.v.blk0 + s.blk;
}

// Fills tab[0..n) with the segments of [u, u_end) (at most kSegTab); returns n
// and the first unit not covered.
template <class Problem>
__device__ int build_segs(const Problem& P, const Common& C, long long u, long long u_end, long long cta_u0,
                          Seg* tab, long long* u_next) {
    int n = 0;
    while (u < u_end && n < kSegTab) {
        tab[n++] = make_seg(P, u, u_end, cta_u0);
        const Seg& s = tab[n - 1];
        u += s.jb - s.ja;
    }
    *u_next = u;
    return n;
}

// Column range of chunk c of a segment (chunks are cut at group boundaries).
__device__ __forceinline__ int2 chunk_cols(const Seg& s, int c) {
    const int g = (s.ja >> 4) + c;
    return make_int2(max(s.ja, g << 4), min(s.jb, (g + 1) << 4));
}

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bits) { atomicOr(status, bits); }

// Set when any bounded wait of the CTA gives up; later waits then return at
// once, so a CTA whose pipeline is stuck ends after one wait limit.
__shared__ int s_abort;

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Common& C) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_test(bar, parity)) return true;
        if (i > 2048) {
            if (*reinterpret_cast<volatile int*>(&s_abort)) return false;
            __nanosleep(64);
        }
    }
    *reinterpret_cast<volatile int*>(&s_abort) = 1;
    flag(C.status, kDevTimeout);
    return false;
}

template <int M>
struct Smem {
    uint32_t cb0;     // codebook replicas: entry z*8 + r holds codeword z (16 bytes)
    uint32_t ring0;   // shared address of the chunk ring
    int slots;        // ring depth
    int cbraw_bytes;
    uint32_t cbraw0;  // two raw codebooks (double buffer across segments)
    uint32_t xbuf0;   // two activation windows, each [m][kXW] x 16 bytes
    uint32_t perm0;   // permutation entries of the window being gathered, [kXW] x 32 bytes
    uint32_t* posinfo;  // per window position: segment index << 24 | column j
    float* red;
    float* stash;
    uint64_t* bars;
    int* bcast;
    int* wlen0;       // length of the first activation window
    Seg* segs;
    __device__ uint32_t slot_addr(int k) const { return ring0 + (uint32_t)k * kSlot; }
    __device__ uint64_t* full(int k) const { return bars + k; }
    __device__ uint64_t* empty(int k) const { return bars + kMaxSlots + k; }
    __device__ uint64_t* cb_full(int h) const { return bars + 2 * kMaxSlots + h; }
    __device__ uint64_t* cb_empty(int h) const { return bars + 2 * kMaxSlots + 2 + h; }
    __device__ uint64_t* x_full(int h) const { return bars + 2 * kMaxSlots + 4 + h; }
    __device__ uint64_t* x_empty(int h) const { return bars + 2 * kMaxSlots + 6 + h; }
    __device__ uint64_t* perm_full() const { return bars + 2 * kMaxSlots + 8; }
    __device__ uint32_t xwin(int w) const { return xbuf0 + (uint32_t)(w & 1) * Cfg<M>::kXBuf; }
};

template <int M>
__device__ __forceinline__ Smem<M> carve(uint8_t* base, int slots, int kmax) {
    Smem<M> s;
    s.slots = slots;
    uint8_t* p = base;
    s.cb0 = smem_u32(p); p += kmax * 128;
    s.ring0 = smem_u32(p); p += slots * kSlot;
    s.cbraw_bytes = kmax * 16;
    s.cbraw0 = smem_u32(p); p += 2 * kmax * 16;
    s.xbuf0 = smem_u32(p); p += 2 * Cfg<M>::kXBuf;
    s.perm0 = smem_u32(p); p += Cfg<M>::kPermBuf;
    s.posinfo = reinterpret_cast<uint32_t*>(p); p += Cfg<M>::kPosInfo;
    s.red = reinterpret_cast<float*>(p); p += Cfg<M>::kRed;
    s.stash = reinterpret_cast<float*>(p); p += Cfg<M>::kStash;
    s.segs = reinterpret_cast<Seg*>(p); p += kSegTab * kSegBytes;
    s.bars = reinterpret_cast<uint64_t*>(p); p += (2 * kMaxSlots + 9) * 8;
    s.bcast = reinterpret_cast<int*>(p);
    s.wlen0 = s.bcast + 8;
    return s;
}

// Activation windows.  The chunks of a CTA are laid end to end; a window holds
// up to kXW of their columns (a chunk never straddles two windows) and every
// segment-table round starts a new window.  The activation warp and the
// decode warps apply these same two rules, so they agree on where each
// chunk's x_perm sits without talking to each other.
struct WinPos {
    int win;    // window index (its buffer is win & 1)
    int wpos;   // columns already placed in the window
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

__device__ __forceinline__ void ring_next(int& slot, int& ph, int slots) {
    if (++slot == slots) {
        slot = 0;
        ph ^= 1;
    }
}

// Per-role progress that persists across segment-table rounds.
struct RoleState {
    int t;      // chunk counter
    int slot;   // ring slot of chunk t (t % slots, kept incrementally)
    int ph;     // phase parity of that slot for chunk t ((t / slots) & 1)
    int s;      // segment counter (codebook phases)
    WinPos w;   // activation window placement
    int cur_win;  // decode warps: the x window they hold (-1: none)
};

// ------------------------------------------------------------------------
// Copy warp: bulk copies of codebooks and code chunks into the ring, issued
// as far ahead as the ring allows (before and independent of the wait on the
// preceding kernel: nothing it reads is written by that kernel).
// ------------------------------------------------------------------------
template <int M>
__device__ __forceinline__ void copy_warp(const Common& C, const Smem<M>& sm, int n_seg, RoleState& st,
                                          bool first_round) {
    const int lane = threadIdx.x & 31;
    for (int si = 0; si < n_seg; ++si, ++st.s) {
        const Seg& g = sm.segs[si];
        const int s = st.s;
        if (s >= 2) wait_bar(sm.cb_empty(s & 1), ((s >> 1) - 1) & 1, C);
        const uint32_t cbb = (uint32_t)(16u << g.v.log2K);
        if (lane == 0) {
            mbar_arrive_expect_tx(sm.cb_full(s & 1), cbb);
            bulk_g2s(sm.cbraw0 + (s & 1) * sm.cbraw_bytes, g.v.cb, cbb, sm.cb_full(s & 1));
        }
        // the first codebook goes first; then the first window's permutation
        // entries (activation warp) ahead of the code chunks
        if (first_round && si == 0) named_barrier(kBarPermIssued, 64);
        const int n_oct = g.n_oct, R8 = g.v.R8, S = g.v.S, G = g.v.d_in >> 7, blk = g.blk;
        for (int c = 0; c < g.n_chunks; ++c, ++st.t, ring_next(st.slot, st.ph, sm.slots)) {
            const int k = st.slot;
            if (st.t >= sm.slots) wait_bar(sm.empty(k), st.ph ^ 1, C);
            if (lane == 0) {
                const int2 cc = chunk_cols(g, c);
                const int nj = cc.y - cc.x;
                const uint32_t mb = (uint32_t)(nj * n_oct * 16), tb = (uint32_t)(n_oct * 64);
                mbar_arrive_expect_tx(sm.full(k), mb + tb);
                // the chunk's records: one contiguous range of the block; its group's meta entries
                const uint64_t pol = l2_evict_first();
                bulk_g2s_stream(sm.slot_addr(k), g.v.main + main_word(R8, S, blk, cc.x, 0, 0), mb, sm.full(k), pol);
                bulk_g2s_stream(sm.slot_addr(k) + kMainSlot, g.v.meta + 2 * meta_entry(R8, G, blk, cc.x >> 4, 0, 0),
                                tb, sm.full(k), pol);
            }
        }
    }
}

// The CTA may not exit while bulk copies are in flight.
template <int M>
__device__ void copy_drain(const Common& C, const Smem<M>& sm, const RoleState& st) {
    for (int t = max(0, st.t - sm.slots); t < st.t; ++t) wait_bar(sm.full(t % sm.slots), (t / sm.slots) & 1, C);
}

// ------------------------------------------------------------------------
// Activation warp: x_perm[m][p] = x[m][perm[p]] for one window of columns
// (Sec. 3.5 fuses this gather into the decode GEMV).  The permutation entries
// are bulk-copied first -- for the first window before the wait on the
// preceding kernel, since only x comes from that kernel -- so after the wait
// the gather costs one round trip per window.
// ------------------------------------------------------------------------
// Gathers x_perm for window positions e = gi, gi + gn, ... of the (batch row,
// position) pairs of a window of wlen positions into the window buffer xb.
// All loads of a round are issued before any store.
template <int M, int B>
__device__ __forceinline__ void gather_x(const Smem<M>& sm, int wlen, uint32_t xb, int gi, int gn) {
    constexpr int XW = Cfg<M>::kXW;
    const int total = M * wlen;
    for (int e0 = 0; e0 < total; e0 += B * gn) {
        uint4 val[B];
        uint32_t dst[B];
#pragma unroll
        for (int r = 0; r < B; ++r) {
            const int e = e0 + r * gn + gi;
            dst[r] = 0xffffffffu;
            if (e < total) {
                const int m = e / wlen, p = e - m * wlen;
                const uint32_t info = sm.posinfo[p];
                const Seg& g = sm.segs[info >> 24];
                const int j = (int)(info & 0xffffffu);
                if (m < g.v.Mk) {
                    const int xr_idx = g.v.xrows ? row_at(g.v.xrows, m) : m;
                    const unsigned short* xr =
                        reinterpret_cast<const unsigned short*>(g.v.x) + (size_t)xr_idx * g.v.d_in;
                    // x is read-only while this kernel runs and is first read here,
                    // after the wait on the kernel that wrote it: the scattered
                    // 2-byte reads go through L1, which holds the whole row.
                    if (g.v.perm) {
                        const uint32_t sp = sm.perm0 + p * 32;
                        const uint4 pa = lds128(sp), pb = lds128(sp + 16);
                        val[r].x = (uint32_t)__ldg(xr + pa.x) | ((uint32_t)__ldg(xr + pa.y) << 16);
                        val[r].y = (uint32_t)__ldg(xr + pa.z) | ((uint32_t)__ldg(xr + pa.w) << 16);
                        val[r].z = (uint32_t)__ldg(xr + pb.x) | ((uint32_t)__ldg(xr + pb.y) << 16);
                        val[r].w = (uint32_t)__ldg(xr + pb.z) | ((uint32_t)__ldg(xr + pb.w) << 16);
                    } else {
                        val[r] = __ldg(reinterpret_cast<const uint4*>(xr + j * 8));
                    }
                    dst[r] = xb + (m * XW + p) * 16;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < B; ++r)
            if (dst[r] != 0xffffffffu) sts128(dst[r], val[r]);
    }
}


template <int M>
__device__ __forceinline__ void fill_window(const Common& C, const Smem<M>& sm, int w, int si0, int c0, int nch, bool& waited) {
    const int lane = threadIdx.x & 31;
    fence_proxy_async_smem();  // earlier reads of the permutation buffer precede the copies below
    int si = si0, c = c0, wlen = 0;
    for (int k = 0; k < nch; ++k) {
        const Seg& g = sm.segs[si];
        const int2 cc = chunk_cols(g, c);
        const int nj = cc.y - cc.x;
        if (g.v.perm && lane == 0) {
            mbar_expect_tx(sm.perm_full(), (uint32_t)(nj * 32));
            bulk_g2s(sm.perm0 + wlen * 32, g.v.perm + cc.x * 8, (uint32_t)(nj * 32), sm.perm_full());
        }
        if (lane < nj) sm.posinfo[wlen + lane] = ((uint32_t)si << 24) | (uint32_t)(cc.x + lane);
        wlen += nj;
        if (++c == g.n_chunks) { c = 0; ++si; }
    }
    if (lane == 0) mbar_arrive(sm.perm_full());
    // The first window's permutation entries go ahead of the code chunks in the
    // copy queue: the copy warp starts once they are issued.
    if (w == 0) named_barrier(kBarPermIssued, 64);
    if (!waited) {
        pdl_wait();  // x may be written by the preceding kernel
        waited = true;
    }
    wait_bar(sm.perm_full(), w & 1, C);
    if (w >= 2) wait_bar(sm.x_empty(w & 1), ((w >> 1) - 1) & 1, C);
    __syncwarp();
    if (w == 0) {  // the decode warps, idle until now, help with the first window
        if (lane == 0) *sm.wlen0 = wlen;
        named_barrier(kBarFirstWindow, 32 + Cfg<M>::kDecodeThreads);
        gather_x<M, 2>(sm, wlen, sm.xwin(0), Cfg<M>::kDecodeThreads + lane, 32 + Cfg<M>::kDecodeThreads);
        named_barrier(kBarFirstWindow, 32 + Cfg<M>::kDecodeThreads);
    } else {
        gather_x<M, 8>(sm, wlen, sm.xwin(w), lane, 32);
    }
    mbar_arrive(sm.x_full(w & 1));  // all 32 lanes, each after its own stores
}

template <int M>
__device__ __forceinline__ void act_warp(const Common& C, const Smem<M>& sm, int n_seg, RoleState& st, bool& waited) {
    win_break(st.w);
    int pend = -1, si0 = 0, c0 = 0, nch = 0;
    for (int si = 0; si < n_seg; ++si) {
        const Seg& g = sm.segs[si];
        for (int c = 0; c < g.n_chunks; ++c) {
            const int2 cc = chunk_cols(g, c);
            win_place(st.w, cc.y - cc.x, Cfg<M>::kXW);
            if (st.w.win != pend) {
                if (nch) fill_window<M>(C, sm, pend, si0, c0, nch, waited);
                pend = st.w.win;
                si0 = si;
                c0 = c;
                nch = 0;
            }
            ++nch;
        }
    }
    if (nch) fill_window<M>(C, sm, pend, si0, c0, nch, waited);
}

// ------------------------------------------------------------------------
// Decode warps.
// ------------------------------------------------------------------------
template <int M>
__device__ __forceinline__ void decode_record(const VDec& d, uint4 rec, const uint32_t (&aux)[8], uint32_t sh_aux,
                                              const float (&mup)[8], const float (&dlp)[8], uint32_t cbsel,
                                              const uint4 (&xv)[M], float (&acc)[8][M]) {
    const uint32_t wv[4] = {rec.x, rec.y, rec.z, rec.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t wa = wv[u];
        const uint32_t wb = rot16(wa);
        {   // row A = 2u: z at [7, 7 + log2K), q at [23 - V, 23) of wa; signs in slots 0..2
            uint4 c = lds128(cbsel + (wa & d.zmask));
            c.x ^= (wa << d.sh0) & 0x80008000u;
            c.y ^= (wa << d.sh1) & 0x80008000u;
            c.z ^= (wa << d.sh2) & 0x80008000u;
            c.w ^= (aux[2 * u] << sh_aux) & 0x80008000u;
            const float r = fmaf(__uint_as_float((wa & d.qmask) | 0x3F800000u), dlp[2 * u], mup[2 * u]);
#pragma unroll
            for (int m = 0; m < M; ++m) acc[2 * u][m] = fmaf(r, signed_dot(c, xv[m]), acc[2 * u][m]);
        }
        {   // row B = 2u + 1: the same fields after a 16-bit rotation; signs in slots 3..5
            uint4 c = lds128(cbsel + (wb & d.zmask));
            c.x ^= (wa << d.sh3) & 0x80008000u;
            c.y ^= (wa << d.sh4) & 0x80008000u;
            c.z ^= wa & 0x80008000u;  // slot 5 sits at bit 15 for every split
            c.w ^= (aux[2 * u + 1] << sh_aux) & 0x80008000u;
            const float r = fmaf(__uint_as_float((wb & d.qmask) | 0x3F800000u), dlp[2 * u + 1], mup[2 * u + 1]);
#pragma unroll
            for (int m = 0; m < M; ++m)
                acc[2 * u + 1][m] = fmaf(r, signed_dot(c, xv[m]), acc[2 * u + 1][m]);
        }
    }
}

// Decodes this warp's columns of one ring chunk (chunk c of segment g, in
// ring slot k with phase parity ph): columns lw, lw + wpg, ... of the chunk,
// against the x_perm window at xw, where the chunk's first column sits at
// window position pos.
template <int M, int MS>
__device__ __forceinline__ void decode_chunk(const Smem<MS>& sm, const Common& C, const Seg& g, const VDec& d, int k,
                                             int ph, int c, uint32_t xw, int pos, int lw, int wpg, int lane,
                                             float (&acc)[8][M]) {
    constexpr int XW = Cfg<MS>::kXW;
    const int2 cc = chunk_cols(g, c);
    const int nj = cc.y - cc.x;
    wait_bar(sm.full(k), ph, C);
    const int n_oct = g.n_oct;
    if (lw < nj && lane < n_oct) {
        const uint32_t base = sm.slot_addr(k);
        const uint32_t cbsel = sm.cb0 + ((uint32_t)(lane & 7) << 4);
        uint32_t aux[8];
        float mup[8], dlp[8];
        {   // the group's grid and aux signs for this lane's 8 rows
            uint4 q[4];
            load_meta(base + kMainSlot + lane * 64, lane, q);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                aux[2 * e] = q[e].x;
                aux[2 * e + 1] = q[e].z;
                const float2 m0 = __half22float2(u2h2(q[e].y));
                const float2 m1 = __half22float2(u2h2(q[e].w));
                dlp[2 * e] = m0.y * d.vscale;
                mup[2 * e] = m0.x - dlp[2 * e];
                dlp[2 * e + 1] = m1.y * d.vscale;
                mup[2 * e + 1] = m1.x - dlp[2 * e + 1];
            }
        }
        auto column = [&](int i) {
            const int j = cc.x + i;
            const uint4 rec = lds128(base + (i * n_oct + lane) * 16);
            uint4 xv[M];
#pragma unroll
            for (int m = 0; m < M; ++m) xv[m] = lds128(xw + (m * XW + pos + i) * 16);
            decode_record<M>(d, rec, aux, (uint32_t)(15 - (j & 15)), mup, dlp, cbsel, xv, acc);
        };
        if constexpr (M <= 4) {  // two columns in flight where registers allow
#pragma unroll 2
            for (int i = lw; i < nj; i += wpg) column(i);
        } else {
#pragma unroll 1
            for (int i = lw; i < nj; i += wpg) column(i);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(k));
}

// Decodes one ring chunk (chunk c of segment g, ring slot k, phase parity ph)
// with one thread per row of the 256-row block: row 32 warp + lane, i.e. the
// 8 lanes of a quarter warp hold the 8 rows of one octet.  Per row the grid
// and aux signs are one 8-byte entry; per (row, column) the fields are the
// row's half of one record word, and the codeword comes from the replica of
// the row's position in its octet (no bank conflicts).  acc[m] accumulates the
// row's output for batch row m.
template <int M, int MS>
__device__ __forceinline__ void decode_rows(const Smem<MS>& sm, const Common& C, const Seg& g, const VDec& d, int k,
                                            int ph, int c, uint32_t xw, int pos, int warp, int lane, float (&acc)[M]) {
    constexpr int XW = Cfg<MS>::kXW;
    const int2 cc = chunk_cols(g, c);
    const int nj = cc.y - cc.x;
    wait_bar(sm.full(k), ph, C);
    const int n_oct = g.n_oct;
    const int o = (warp << 2) + (lane >> 3), tr = lane & 7;
    if (o < n_oct) {
        const uint32_t base = sm.slot_addr(k);
        const uint2 e = lds64(base + kMainSlot + (uint32_t)(o * 8 + tr) * 8);
        const float2 md = __half22float2(u2h2(e.y));
        const float dl = md.y * d.vscale, mp = md.x - dl;
        const uint32_t aux = e.x;
        const bool odd = tr & 1;
        const uint32_t s0 = odd ? d.sh3 : d.sh0, s1 = odd ? d.sh4 : d.sh1, s2 = odd ? d.sh5 : d.sh2;
        const uint32_t cbsel = sm.cb0 + ((uint32_t)tr << 4);
        const uint32_t wbase = base + (uint32_t)o * 16 + (uint32_t)(tr >> 1) * 4;
        const uint32_t rstride = (uint32_t)n_oct * 16;
        const uint32_t xbase = xw + (uint32_t)pos * 16;
        // column i of the chunk; its sign bit 7 is aux bit (cc.x + i) % 16
        auto column = [&](int i, uint32_t aux_shift) {
            const uint32_t w = lds32(wbase + (uint32_t)i * rstride);
            const uint32_t wf = odd ? rot16(w) : w;  // (z, q) field word of this row
            uint4 cw = lds128(cbsel + (wf & d.zmask));
            cw.x ^= (w << s0) & 0x80008000u;
            cw.y ^= (w << s1) & 0x80008000u;
            cw.z ^= (w << s2) & 0x80008000u;
            cw.w ^= (aux << aux_shift) & 0x80008000u;
            const float r = fmaf(__uint_as_float((wf & d.qmask) | 0x3F800000u), dl, mp);
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const uint4 xv = lds128(xbase + (uint32_t)(m * XW + i) * 16);
                acc[m] = fmaf(r, signed_dot(cw, xv), acc[m]);
            }
        };
        if (nj == kChunkJ) {  // a whole radius group (cc.x % 16 == 0): fixed trip count, constant shifts
            if constexpr (M == 1) {  // the whole chunk in one schedule (no spills at batch 1)
#pragma unroll
                for (int i = 0; i < kChunkJ; ++i) column(i, (uint32_t)(15 - i));
            } else {
#pragma unroll 8
                for (int i = 0; i < kChunkJ; ++i) column(i, (uint32_t)(15 - i));
            }
        } else {
#pragma unroll 4
            for (int i = 0; i < nj; ++i) column(i, (uint32_t)(15 - ((cc.x + i) & 15)));
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(k));
}

// Writes (or combines) the outputs of the pending segments tab[i0 .. i0 + n).
// Split blocks: every contributor stores its partial sums, the CTA's writes are
// published with one release atomic per block, and the contributor that sees
// the count complete (acquire) adds all partials in CTA order.
template <int M>
__device__ void flush(const Common& C, const Smem<M>& sm, int i0, int n) {
    constexpr int DT = Cfg<M>::kDecodeThreads;
    const int tid = threadIdx.x;
    const int cta = blockIdx.x;
    const int l = tid & 31, r = tid >> 5;
    const int row_local = l * 8 + r;
    bool any_partial = false;
    for (int i = 0; i < n; ++i) {
        const Seg& g = sm.segs[i0 + i];
        const int row = g.blk * kBlockRows + row_local;
        const float* st = sm.stash + (size_t)i * M * kBlockRows;
        if (g.full) {
            if (tid < kBlockRows && row < g.v.d_out) {
#pragma unroll
                for (int m = 0; m < M; ++m)
                    if (m < g.v.Mk) {
                        const int yr = g.v.yrows ? row_at(g.v.yrows, m) : m;
                        g.v.y[(size_t)yr * g.v.d_out + row] = __half_as_ushort(__float2half_rn(st[m * kBlockRows + row_local]));
                    }
            }
        } else {
            any_partial = true;
            float* part = C.partials + ((size_t)(cta * 2 + g.my_slot) * 8) * kBlockRows;
            if (tid < kBlockRows)
#pragma unroll
                for (int m = 0; m < M; ++m)
                    if (m < g.v.Mk) part[m * kBlockRows + row_local] = st[m * kBlockRows + row_local];
        }
    }
    if (!any_partial) return;  // uniform across the decode threads
    named_barrier(1, DT);      // every partial store of the CTA precedes the release below
    if (tid < n) {
        const Seg& g = sm.segs[i0 + tid];
        int last = 0;
        if (!g.full) {
            const unsigned old = atom_add_acq_rel_gpu(g.counter, 1u);
            last = (old == (unsigned)(g.c_last - g.c_first));
            if (last) *reinterpret_cast<volatile unsigned*>(g.counter) = 0u;  // restore for the next call
        }
        sm.bcast[tid] = last;
    }
    named_barrier(1, DT);
    for (int i = 0; i < n; ++i) {
        const Seg& g = sm.segs[i0 + i];
        if (!sm.bcast[i]) continue;
        const int row = g.blk * kBlockRows + row_local;
        if (tid < kBlockRows && row < g.v.d_out) {
            const int c_first = g.c_first, c_last = g.c_last, first_slot = g.first_slot, mk = g.v.Mk;
            float tot[M];
#pragma unroll
            for (int m = 0; m < M; ++m) tot[m] = 0.f;
            constexpr int NF = (M <= 2) ? 16 : 8;  // contributors' loads in flight at once
            for (int c0 = c_first; c0 <= c_last; c0 += NF) {
                float v[NF][M];
#pragma unroll
                for (int k = 0; k < NF; ++k) {
                    const int c = c0 + k;
                    const int sp = (c == c_first) ? first_slot : 0;
                    const float* src = C.partials + ((size_t)(c * 2 + sp) * 8) * kBlockRows + row_local;
#pragma unroll
                    for (int m = 0; m < M; ++m) v[k][m] = (c <= c_last && m < mk) ? __ldcg(src + m * kBlockRows) : 0.f;
                }
#pragma unroll
                for (int k = 0; k < NF; ++k)
#pragma unroll
                    for (int m = 0; m < M; ++m) tot[m] += v[k][m];
            }
#pragma unroll
            for (int m = 0; m < M; ++m)
                if (m < g.v.Mk) {
                    const int yr = g.v.yrows ? row_at(g.v.yrows, m) : m;
                    g.v.y[(size_t)yr * g.v.d_out + row] = __half_as_ushort(__float2half_rn(tot[m]));
                }
        }
    }
    named_barrier(1, DT);  // bcast reuse
}

// Decodes one segment with compile-time batch MK (<= MS, the launch's stash
// stride) and leaves its 256 x MS results in stash slot `slot`.
template <int MK, int MS>
__device__ __forceinline__ void segment_body_impl(const Smem<MS>& sm, const Common& C, const Seg& g, RoleState& st,
                                                  int slot) {
    constexpr int DT = Cfg<MS>::kDecodeThreads;
    static_assert(Cfg<MS>::kW * 32 == kBlockRows, "one decode thread per block row");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const VDec d = vdec(g.v.log2K);
    float acc[MK];
#pragma unroll
    for (int m = 0; m < MK; ++m) acc[m] = 0.f;
    int t = st.t, k = st.slot, ph = st.ph, cur = st.cur_win;
    WinPos w = st.w;
    for (int c = 0; c < g.n_chunks; ++c, ++t, ring_next(k, ph, sm.slots)) {
        const int2 cc = chunk_cols(g, c);
        const int pos = win_place(w, cc.y - cc.x, Cfg<MS>::kXW);
        if (w.win != cur) {  // release the previous x window, wait for this one
            if (cur >= 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(sm.x_empty(cur & 1));
            }
            if (w.win == 0) {  // the first window is gathered together with the activation warp
                pdl_wait();
                named_barrier(kBarFirstWindow, 32 + DT);
                gather_x<MS, 2>(sm, *sm.wlen0, sm.xwin(0), tid, 32 + DT);
                named_barrier(kBarFirstWindow, 32 + DT);
            } else {
                wait_bar(sm.x_full(w.win & 1), (w.win >> 1) & 1, C);
            }
            cur = w.win;
        }
        decode_rows<MK, MS>(sm, C, g, d, k, ph, c, sm.xwin(w.win), pos, warp, lane, acc);
    }
    st.t = t;
    st.slot = k;
    st.ph = ph;
    st.cur_win = cur;
    st.w = w;
    // each thread owns one row: its sums go straight to the stash
    const int row = 32 * warp + lane;
#pragma unroll
    for (int m = 0; m < MS; ++m) {
        float v = 0.f;
#pragma unroll
        for (int mm = 0; mm < MK; ++mm)
            if (mm == m) v = acc[mm];
        sm.stash[((size_t)slot * MS + m) * kBlockRows + row] = v;
    }
    named_barrier(1, DT);
}

// The MoE kernel's segment body: lane <-> row octet, warps split each chunk's
// columns within warp groups, and the warps' partial sums are reduced through
// shared memory.  (Dense launches use segment_body_impl: one thread per row.)
template <int MK, int MS>
__device__ __forceinline__ void segment_body_octets(const Smem<MS>& sm, const Common& C, const Seg& g, RoleState& st,
                                                  int slot) {
    constexpr int W = Cfg<MS>::kW, DT = Cfg<MS>::kDecodeThreads;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const VDec d = vdec(g.v.log2K);
    float acc[8][MK];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int m = 0; m < MK; ++m) acc[r][m] = 0.f;
    int t = st.t, k = st.slot, ph = st.ph, cur = st.cur_win;
    WinPos w = st.w;
    const int wpg = W / C.n_wg, grp = warp / wpg, lw = warp - grp * wpg;
    for (int c = 0; c < g.n_chunks; ++c, ++t, ring_next(k, ph, sm.slots)) {
        const int2 cc = chunk_cols(g, c);
        const int pos = win_place(w, cc.y - cc.x, Cfg<MS>::kXW);
        if (w.win != cur) {  // release the previous x window, wait for this one
            if (cur >= 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(sm.x_empty(cur & 1));
            }
            if (w.win == 0) {  // the first window is gathered together with the activation warp
                pdl_wait();
                named_barrier(kBarFirstWindow, 32 + DT);
                gather_x<MS, 2>(sm, *sm.wlen0, sm.xwin(0), tid, 32 + DT);
                named_barrier(kBarFirstWindow, 32 + DT);
            } else {
                wait_bar(sm.x_full(w.win & 1), (w.win >> 1) & 1, C);
            }
            cur = w.win;
        }
        if ((t & (C.n_wg - 1)) == grp) decode_chunk<MK, MS>(sm, C, g, d, k, ph, c, sm.xwin(w.win), pos, lw, wpg, lane, acc);
    }
    st.t = t;
    st.slot = k;
    st.ph = ph;
    st.cur_win = cur;
    st.w = w;
    // reduce the warps' partial sums in a fixed order into the stash
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int m = 0; m < MK; ++m) sm.red[((warp * 8 + r) * MK + m) * 32 + lane] = acc[r][m];
    named_barrier(1, DT);
    if (tid < kBlockRows) {
        const int l = tid & 31, r = tid >> 5;
        for (int m = 0; m < MS; ++m) {
            float sum = 0.f;
            if (m < MK) {
#pragma unroll
                for (int w2 = 0; w2 < W; ++w2) sum += sm.red[((w2 * 8 + r) * MK + m) * 32 + l];
            }
            sm.stash[((size_t)slot * MS + m) * kBlockRows + l * 8 + r] = sum;
        }
    }
    named_barrier(1, DT);
}

// Out-of-line instance for launches whose segments have different batch
// sizes (the MoE kernel dispatches on each segment's).
template <int MK, int MS>
__device__ __noinline__ void segment_body(const Smem<MS>& sm, const Common& C, const Seg& g, RoleState& st, int slot) {
    segment_body_octets<MK, MS>(sm, C, g, st, slot);
}

template <int MLO, int M>
__device__ __forceinline__ void decode_warps(const Common& C, const Smem<M>& sm, int n_seg, RoleState& st) {
    constexpr int DT = Cfg<M>::kDecodeThreads;
    const int tid = threadIdx.x;
    int npend = 0, i_pend = 0;
    const uint16_t* cur_cb = nullptr;
    win_break(st.w);
    for (int si = 0; si < n_seg; ++si, ++st.s) {
        const Seg& g = sm.segs[si];
        const int s = st.s;
        wait_bar(sm.cb_full(s & 1), (s >> 1) & 1, C);
        if (g.v.cb != cur_cb) {  // build the 8 bank-rotated replicas from the raw copy
            if (cur_cb) named_barrier(1, DT);
            const int K = 1 << g.v.log2K;
            const uint32_t raw = sm.cbraw0 + (s & 1) * sm.cbraw_bytes;
            for (int e = tid; e < K * 8; e += DT) sts128(sm.cb0 + e * 16, lds128(raw + (e >> 3) * 16));
            named_barrier(1, DT);
            cur_cb = g.v.cb;
        }
        if (tid == 0) mbar_arrive(sm.cb_empty(s & 1));
        if constexpr (MLO == M) {
            segment_body_impl<M, M>(sm, C, g, st, npend);
        } else {
            switch (g.v.Mk) {
                case 1: segment_body<1, M>(sm, C, g, st, npend); break;
                case 2: segment_body<2, M>(sm, C, g, st, npend); break;
                case 3: segment_body<3, M>(sm, C, g, st, npend); break;
                case 4: segment_body<4, M>(sm, C, g, st, npend); break;
                case 5: segment_body<5, M>(sm, C, g, st, npend); break;
                case 6: segment_body<6, M>(sm, C, g, st, npend); break;
                case 7: segment_body<7, M>(sm, C, g, st, npend); break;
                default: segment_body<8, M>(sm, C, g, st, npend); break;
            }
        }
        ++npend;
        if (npend == kMaxSegs || si + 1 == n_seg) {
            flush<M>(C, sm, i_pend, npend);
            npend = 0;
            i_pend = si + 1;
        }
    }
}

template <int MLO, int M, class Problem>
__device__ __forceinline__ void run(const Problem& P, const Common& C, uint8_t* smem_raw, bool plan_needs_wait) {
    const Smem<M> sm = carve<M>(smem_raw, C.slots, C.kmax);
    const int tid = threadIdx.x, warp = tid >> 5;
    constexpr int W = Cfg<M>::kW;
    if (tid == 0) {
        for (int k = 0; k < kMaxSlots; ++k) {
            mbar_init(sm.bars + k, 1);              // full: copy warp arrival + bytes
            mbar_init(sm.bars + kMaxSlots + k, W / C.n_wg);  // empty: one arrival per warp of the chunk's group
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(sm.cb_full(h), 1);
            mbar_init(sm.cb_empty(h), 1);
            mbar_init(sm.x_full(h), 32);
            mbar_init(sm.x_empty(h), W);
        }
        mbar_init(sm.perm_full(), 1);
        fence_mbar_init();
        s_abort = 0;
    }
    pdl_launch_dependents();
    if (plan_needs_wait) pdl_wait();  // the plan itself depends on preceding work
    __shared__ long long s_next;
    __shared__ int s_nseg;
    const long long total = P.total();
    const long long u0 = total > 0 ? P.cta_begin(blockIdx.x) : 0;
    const long long u1 = total > 0 ? P.cta_begin(blockIdx.x + 1) : 0;
    RoleState st{0, 0, 0, 0, {0, 0}, -1};
    bool waited = plan_needs_wait;
    for (long long u = u0; u < u1;) {
        if (warp == 0) {  // lane 0 lays the segments out, then one lane per segment adds the split-K data
            if ((tid & 31) == 0) s_nseg = build_segs(P, C, u, u1, u0, sm.segs, &s_next);
            __syncwarp();
            for (int i = tid & 31; i < s_nseg; i += 32) seg_split_info(P, C, sm.segs[i], u0);
        }
        __syncthreads();
        const int n_seg = s_nseg;
        if (warp == W) {
            copy_warp<M>(C, sm, n_seg, st, u == u0);
        } else if (warp == W + 1) {
            act_warp<M>(C, sm, n_seg, st, waited);
        } else {
            decode_warps<MLO, M>(C, sm, n_seg, st);
        }
        u = s_next;
        __syncthreads();  // the segment table is rebuilt for the next round
    }
    if (warp == W) copy_drain<M>(C, sm, st);
    if (warp == W + 1 && !waited) pdl_wait();
}

template <int M>
__global__ void __launch_bounds__(Cfg<M>::kThreads, 1) gemv_kernel(const __grid_constant__ DenseParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ int s_cs[kMaxCta + 1];
    __shared__ DenseMat s_ms[kMaxMats];
    for (int i = threadIdx.x; i <= p.c.n_cta; i += blockDim.x) s_cs[i] = p.cta_start[i];
    for (int i = threadIdx.x; i < p.n_mats; i += blockDim.x) s_ms[i] = p.mats[i];
    __syncthreads();
    const DenseProblem P{p, s_cs, s_ms};
    run<M, M>(P, p.c, smem_raw, false);
}

// Virtual experts carry 1..8 pairs; each segment dispatches on its own count.
__global__ void __launch_bounds__(Cfg<kMaxPairsPerVirtual>::kThreads, 1) moe_kernel(const __grid_constant__ MoeParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ MoeStage st;
    pdl_wait();  // the routing comes from the preceding kernel
    if (threadIdx.x == 0) {
        const long long per = (long long)(((p.d_out + 7) / 8 + kOct - 1) / kOct) * (p.d_in >> 3);
        st.total = (long long)__ldcg(&p.route->n_virtual) * per;
        const long long u0 = (long long)blockIdx.x * st.total / p.c.n_cta;
        const long long u1 = (long long)(blockIdx.x + 1) * st.total / p.c.n_cta;
        st.vi0 = (int)(u0 / per);
        st.nvi = u1 > u0 ? (int)min((long long)kMoeCache, (u1 - 1) / per - st.vi0 + 1) : 0;
    }
    __syncthreads();
    if ((int)threadIdx.x < st.nvi) {
        const int vi = st.vi0 + threadIdx.x;
        const int e = __ldcg(p.v_expert + vi);
        st.v_expert[threadIdx.x] = e;
        st.v_count[threadIdx.x] = __ldcg(p.v_count + vi);
        st.emat[threadIdx.x] = p.experts[e];
    }
    for (int i = threadIdx.x; i < st.nvi * kMaxPairsPerVirtual; i += blockDim.x) {
        const size_t src = (size_t)st.vi0 * kMaxPairsPerVirtual + i;
        st.v_xrows[i / kMaxPairsPerVirtual][i % kMaxPairsPerVirtual] = __ldcg(p.v_xrows + src);
        st.v_yrows[i / kMaxPairsPerVirtual][i % kMaxPairsPerVirtual] = __ldcg(p.v_yrows + src);
    }
    __syncthreads();
    const MoeProblem P{p, st};
    run<1, kMaxPairsPerVirtual>(P, p.c, smem_raw, true);
}

// Groups the (pair -> expert) routing into virtual experts of at most 8 pairs,
// in expert order and, within an expert, pair order (deterministic).
__global__ void moe_route_kernel(const int32_t* pair_expert, const int32_t* pair_xrow, int n_pairs, int n_experts,
                                 MoeRoute* route, int32_t* v_expert, int32_t* v_xrows, int32_t* v_yrows,
                                 int32_t* v_count, uint32_t* status) {
    pdl_wait();
    extern __shared__ int s_cnt[];  // [n_experts]
    for (int e = threadIdx.x; e < n_experts; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    for (int q = threadIdx.x; q < n_pairs; q += blockDim.x) {
        const int e = pair_expert[q];
        if (e >= 0 && e < n_experts) atomicAdd(&s_cnt[e], 1);
        else atomicOr(status, kDevUnsupported);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int nv = 0;
        for (int e = 0; e < n_experts; ++e) {
            const int c = s_cnt[e];
            s_cnt[e] = nv;  // first virtual index of expert e
            nv += (c + kMaxPairsPerVirtual - 1) / kMaxPairsPerVirtual;
        }
        route->n_virtual = nv;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n_experts; e += blockDim.x) {
        int vi = s_cnt[e], k = 0;
        for (int q = 0; q < n_pairs; ++q) {
            if (pair_expert[q] != e) continue;
            if (k == kMaxPairsPerVirtual) { ++vi; k = 0; }
            v_expert[vi] = e;
            v_xrows[(size_t)vi * kMaxPairsPerVirtual + k] = pair_xrow[q];
            v_yrows[(size_t)vi * kMaxPairsPerVirtual + k] = q;
            v_count[vi] = ++k;
        }
    }
    pdl_launch_dependents();
}

int g_sm_count = 0;
std::once_flag g_once;

int sm_count() {
    std::call_once(g_once, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (g_sm_count <= 0) g_sm_count = 148;
    });
    return g_sm_count;
}

long long units_of(const sage_matrix& A) {
    const int R8 = (A.d_out + 7) / 8;
    return (long long)((R8 + kOct - 1) / kOct) * (A.d_in / 8);
}
int blocks_of(const sage_matrix& A) { return ((A.d_out + 7) / 8 + kOct - 1) / kOct; }
size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// CTA counts per matrix for a dense launch.  If giving every matrix its own
// CTAs keeps the largest CTA within 6% of an even split of all units, each
// matrix gets its own CTAs (one codebook per CTA, fewer segments); otherwise
// the plan is plain stream-K over the flattened units (returns empty).
std::vector<int> per_matrix_shares(const std::vector<long long>& units, int n_cta) {
    long long total = 0;
    for (long long u : units) total += u;
    const int n_mat = (int)units.size();
    if (n_mat == 1 || n_mat > n_cta) return {};
    std::vector<int> share((size_t)n_mat);
    int given = 0;
    for (int k = 0; k < n_mat; ++k) {
        share[k] = std::max(1, (int)((double)units[k] * n_cta / total));
        given += share[k];
    }
    while (given < n_cta) {  // hand out the rest to the most loaded matrix
        int best = 0;
        for (int k = 1; k < n_mat; ++k)
            if ((double)units[k] / share[k] > (double)units[best] / share[best]) best = k;
        ++share[best];
        ++given;
    }
    if (given > n_cta) return {};
    double worst = 0;
    for (int k = 0; k < n_mat; ++k) {
        if (share[k] > units[k]) return {};
        worst = std::max(worst, (double)units[k] / share[k]);
    }
    if (worst > 1.06 * (double)total / n_cta) return {};
    return share;
}

// Ring depth: as many chunk slots as fit next to the fixed shared memory (one
// CTA per SM), at most one more than the widest CTA's chunk count.
constexpr int kSmemBudget = 226 * 1024;  // 227 KB per CTA less static shared memory
constexpr int kDenseStatic = (kMaxCta + 1) * 4 + kMaxMats * (int)sizeof(DenseMat);  // gemv_kernel's staged tables
template <int M>
int slots_for(long long max_units_per_cta, int kmax, int budget) {
    const long long chunks = (max_units_per_cta + kChunkJ - 1) / kChunkJ + 2;
    int n = (int)std::min<long long>(kMaxSlots, std::max<long long>(2, chunks));
    while (n > 2 && Cfg<M>::smem(n, kmax) > budget) --n;
    return n;
}

// Decode warp groups: a chunk is decoded by one group, so that a warp handles
// several columns per ring slot; each group needs two slots in flight.
int wg_for(int slots) { return slots >= 8 ? 4 : slots >= 4 ? 2 : 1; }

// Raises the kernel's dynamic shared memory limit when a launch needs more
// than any earlier one (callers hold the launch mutex).
template <class K>
bool ensure_smem(K kernel, int bytes, int& configured) {
    if (bytes <= configured) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    configured = bytes;
    return true;
}

template <class K, class Params>
int launch_pdl(K kernel, const Params& p, int grid, int threads, int smem, sage_stream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}


template <int M>
int launch_m(const GemvJob* jobs, int n, void* ws, sage_stream_t stream) {
    static DenseParams p;  // large: keep off the stack
    static std::mutex mu;
    static int configured = 0;
    std::lock_guard<std::mutex> lock(mu);
    std::vector<long long> units((size_t)n);
    long long unit = 0;
    int blk = 0, kmax = 16;
    for (int i = 0; i < n; ++i) {
        const sage_matrix& A = jobs[i].A;
        kmax = std::max(kmax, 1 << A.log2K);
        DenseMat& d = p.mats[i];
        d.main = A.main; d.meta = A.meta; d.cb = A.codebook; d.perm = A.perm;
        d.x = jobs[i].x; d.y = jobs[i].y;
        d.d_out = A.d_out; d.d_in = A.d_in; d.log2K = A.log2K;
        d.unit0 = unit; d.blk0 = blk;
        units[i] = units_of(A);
        unit += units[i];
        blk += blocks_of(A);
    }
    if (unit >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
    const int n_cta = (int)std::max<long long>(1, std::min<long long>(std::min(sm_count(), kMaxCta), unit / 4));
    const std::vector<int> share = per_matrix_shares(units, n_cta);
    long long widest = 0;
    p.per_matrix = share.empty() ? 0 : 1;
    int cta = 0;
    for (int i = 0; i < n; ++i) {
        p.mats[i].units = units[i];
        p.mats[i].cta0 = cta;
        p.mats[i].ncta = share.empty() ? 0 : share[i];
        cta += p.mats[i].ncta;
        if (!share.empty()) widest = std::max(widest, (units[i] + share[i] - 1) / share[i]);
    }
    if (share.empty()) widest = (unit + n_cta - 1) / n_cta;
    p.n_mats = n;
    p.total_units = unit;
    p.c.n_cta = n_cta;
    for (int c = 0; c <= n_cta; ++c) {
        long long b;
        if (c == n_cta) {
            b = unit;
        } else if (share.empty()) {
            b = (long long)c * unit / n_cta;
        } else {
            int k = 0;
            while (k + 1 < n && p.mats[k + 1].cta0 <= c) ++k;
            b = p.mats[k].unit0 + (long long)(c - p.mats[k].cta0) * p.mats[k].units / p.mats[k].ncta;
        }
        p.cta_start[c] = (int)b;
    }
    p.c.M = M;
    p.c.slots = slots_for<M>(widest, kmax, kSmemBudget - kDenseStatic);
    p.c.n_wg = 1;  // dense launches: every decode warp works on every chunk (one thread per block row)
    p.c.kmax = kmax;
    if (!ensure_smem(gemv_kernel<M>, Cfg<M>::smem(p.c.slots, kmax), configured)) return SAGE_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.c.status = reinterpret_cast<uint32_t*>(w);
    p.c.counters = reinterpret_cast<unsigned*>(w + kWsHeader);
    p.c.partials = reinterpret_cast<float*>(w + kWsHeader + round256((size_t)blk * 4));
    return launch_pdl(gemv_kernel<M>, p, n_cta, Cfg<M>::kThreads, Cfg<M>::smem(p.c.slots, kmax), stream);
}

}  // namespace

size_t gemv_workspace_bytes(const sage_matrix* mats, int n, int M) {
    (void)M;
    long long units = 0;
    int blk = 0;
    for (int i = 0; i < n; ++i) { units += units_of(mats[i]); blk += blocks_of(mats[i]); }
    const int n_cta = (int)std::max<long long>(1, std::min<long long>(sm_count(), units / 4));
    return kWsHeader + round256((size_t)blk * 4) + (size_t)n_cta * 2 * 8 * kBlockRows * sizeof(float);
}

int launch_gemv(const GemvJob* jobs, int n, int M, void* ws, size_t ws_bytes, sage_stream_t stream) {
    if (n > kMaxMats) return SAGE_ERR_UNSUPPORTED;
    std::vector<sage_matrix> mats((size_t)n);
    for (int i = 0; i < n; ++i) mats[i] = jobs[i].A;
    if (ws_bytes < gemv_workspace_bytes(mats.data(), n, M)) return SAGE_ERR_WORKSPACE;
    switch (M) {
        case 1: return launch_m<1>(jobs, n, ws, stream);
        case 2: return launch_m<2>(jobs, n, ws, stream);
        case 3: return launch_m<3>(jobs, n, ws, stream);
        case 4: return launch_m<4>(jobs, n, ws, stream);
        case 5: return launch_m<5>(jobs, n, ws, stream);
        case 6: return launch_m<6>(jobs, n, ws, stream);
        case 7: return launch_m<7>(jobs, n, ws, stream);
        case 8: return launch_m<8>(jobs, n, ws, stream);
        default: return SAGE_ERR_UNSUPPORTED;
    }
}

// MoE workspace: header | route | v_expert | v_xrows | v_yrows | v_count | counters | partials
namespace {
struct MoeWs {
    size_t route, v_expert, v_xrows, v_yrows, v_count, counters, partials, total;
};
MoeWs moe_ws_layout(int n_pairs, int d_out, int n_cta) {
    MoeWs L;
    size_t o = kWsHeader;
    L.route = o; o += 256;
    L.v_expert = o; o += round256((size_t)n_pairs * 4);
    L.v_xrows = o; o += round256((size_t)n_pairs * kMaxPairsPerVirtual * 4);
    L.v_yrows = o; o += round256((size_t)n_pairs * kMaxPairsPerVirtual * 4);
    L.v_count = o; o += round256((size_t)n_pairs * 4);
    const int nblk = ((d_out + 7) / 8 + kOct - 1) / kOct;
    L.counters = o; o += round256((size_t)n_pairs * nblk * 4);
    L.partials = o; o += (size_t)n_cta * 2 * 8 * kBlockRows * sizeof(float);
    L.total = o;
    return L;
}
}  // namespace

size_t moe_workspace_bytes(const sage_matrix* experts, int n_experts, int n_pairs) {
    (void)n_experts;
    return moe_ws_layout(std::max(1, n_pairs), experts[0].d_out, sm_count()).total;
}

int launch_moe(const sage_matrix* experts, int n_experts, const int32_t* pair_expert, const int32_t* pair_xrow,
               int n_pairs, const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes, sage_stream_t stream) {
    constexpr int MV = kMaxPairsPerVirtual;
    if (n_experts > kMaxExperts) return SAGE_ERR_UNSUPPORTED;
    const int n_cta = sm_count();
    const MoeWs L = moe_ws_layout(n_pairs, experts[0].d_out, n_cta);
    if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    static MoeParams p;
    static std::mutex mu;
    static int configured = 0;
    std::lock_guard<std::mutex> lock(mu);
    p.c.n_cta = n_cta;
    p.c.M = 0;
    int kmax = 16;
    for (int e = 0; e < n_experts; ++e) kmax = std::max(kmax, 1 << experts[e].log2K);
    p.c.kmax = kmax;
    p.c.slots = slots_for<MV>(1 << 30, kmax, kSmemBudget - (int)sizeof(MoeStage));
    p.c.n_wg = wg_for(p.c.slots);
    if (!ensure_smem(moe_kernel, Cfg<MV>::smem(p.c.slots, kmax), configured)) return SAGE_ERR_CUDA;
    p.c.status = reinterpret_cast<uint32_t*>(w);
    p.c.counters = reinterpret_cast<unsigned*>(w + L.counters);
    p.c.partials = reinterpret_cast<float*>(w + L.partials);
    p.n_experts = n_experts;
    p.d_out = experts[0].d_out;
    p.d_in = experts[0].d_in;
    p.n_pairs = n_pairs;
    p.x = x;
    p.y = y;
    p.route = reinterpret_cast<const MoeRoute*>(w + L.route);
    p.v_expert = reinterpret_cast<const int32_t*>(w + L.v_expert);
    p.v_xrows = reinterpret_cast<const int32_t*>(w + L.v_xrows);
    p.v_yrows = reinterpret_cast<const int32_t*>(w + L.v_yrows);
    p.v_count = reinterpret_cast<const int32_t*>(w + L.v_count);
    for (int e = 0; e < n_experts; ++e) {
        p.experts[e].main = experts[e].main;
        p.experts[e].meta = experts[e].meta;
        p.experts[e].cb = experts[e].codebook;
        p.experts[e].perm = experts[e].perm;
        p.experts[e].log2K = experts[e].log2K;
    }
    {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = (size_t)n_experts * sizeof(int);
        cfg.stream = reinterpret_cast<cudaStream_t>(stream);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, moe_route_kernel, pair_expert, pair_xrow, n_pairs, n_experts,
                               reinterpret_cast<MoeRoute*>(w + L.route), reinterpret_cast<int32_t*>(w + L.v_expert),
                               reinterpret_cast<int32_t*>(w + L.v_xrows), reinterpret_cast<int32_t*>(w + L.v_yrows),
                               reinterpret_cast<int32_t*>(w + L.v_count), p.c.status) != cudaSuccess)
            return SAGE_ERR_CUDA;
    }
    return launch_pdl(moe_kernel, p, n_cta, Cfg<MV>::kThreads, Cfg<MV>::smem(p.c.slots, kmax), stream);
}

}  // namespace sage
