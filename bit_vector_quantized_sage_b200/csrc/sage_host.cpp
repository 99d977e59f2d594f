// Host half of libsage: status strings, packed-format packer/unpacker, ESG
// permutation, the CPU encoder and argument validation / dispatch of the
// compute entry points.
//
// Method references are to "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward
// Real-World Usability" (section / equation).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <numeric>
#include <thread>
#include <vector>

#include "sage_internal.h"

namespace sage {

// Bit positions of the six sign slots of a main word for radius width V:
// {0 .. 6-V} U {17-V .. 15}, ascending.  Slots 0..2 belong to row A, 3..5 to
// row B; slot k covers bits p_k (component 2n) and p_k + 16 (component 2n+1).
static void sign_slots(int V, int out[6]) {
    int n = 0;
    for (int p = 0; p <= 6 - V; ++p) out[n++] = p;
    for (int p = 17 - V; p <= 15; ++p) out[n++] = p;
}

// Word offsets of octet b's records in the planes (format v2: each block of
// 32 octets is stored contiguously, subvector column major inside the block).
struct PlaneIndex {
    size_t main0, meta0;
    int nB, ob;
    PlaneIndex(int R8, int S, int G, int b) {
        const int blk = b / kBlockOct;
        ob = b % kBlockOct;
        nB = std::min(kBlockOct, R8 - blk * kBlockOct);
        main0 = (size_t)blk * S * kBlockOct * 4;
        meta0 = (size_t)blk * G * kBlockOct * 16;
    }
    size_t main_word(int j, int u) const { return main0 + ((size_t)j * nB + ob) * 4 + u; }
    size_t meta_word(int g, int t) const { return meta0 + (((size_t)g * nB + ob) * 8 + t) * 2; }
};

int current_device() {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

int current_sm_count() {
    static std::mutex mu;
    static int count[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (count[dev] <= 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        count[dev] = n;
    }
    return count[dev];
}

int check_matrix(const sage_matrix* A) {
    if (!A) return SAGE_ERR_INVALID_ARGUMENT;
    if (A->d_out < 1 || A->d_in < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (A->d_in % 128 || A->log2K < 4 || A->log2K > 8) return SAGE_ERR_UNSUPPORTED;
    if (!A->main || !A->meta || !A->codebook) return SAGE_ERR_INVALID_ARGUMENT;
    if (!aligned16(A->main) || !aligned16(A->meta) || !aligned16(A->codebook) ||
        (A->perm && !aligned16(A->perm)))
        return SAGE_ERR_MISALIGNED;
    return SAGE_OK;
}

}  // namespace sage

using namespace sage;

extern "C" {

const char* sage_status_string(int s) {
    switch (s) {
        case SAGE_OK: return "SAGE_OK";
        case SAGE_ERR_INVALID_ARGUMENT: return "SAGE_ERR_INVALID_ARGUMENT";
        case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
        case SAGE_ERR_MISALIGNED: return "SAGE_ERR_MISALIGNED";
        case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
        case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
        case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
        default: return "SAGE_ERR_UNKNOWN";
    }
}

const char* sage_version(void) { return "libsage sm_100a, packed format v2"; }

int sage_packed_sizes(int d_out, int d_in, int log2K, size_t* main_bytes, size_t* meta_bytes) {
    if (!main_bytes || !meta_bytes || d_out < 1 || d_in < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_in % 128 || log2K < 4 || log2K > 8) return SAGE_ERR_UNSUPPORTED;
    const size_t R8 = ((size_t)d_out + 7) / 8;
    *main_bytes = (size_t)(d_in / kSV) * R8 * 16;
    *meta_bytes = (size_t)(d_in / 128) * R8 * 8 * 8;
    return SAGE_OK;
}

int sage_pack(int d_out, int d_in, int log2K, const uint8_t* signs, const uint16_t* idx, const uint8_t* q,
              const uint16_t* mu, const uint16_t* delta, uint32_t* main_out, uint32_t* meta_out) {
    size_t mb, tb;
    int rc = sage_packed_sizes(d_out, d_in, log2K, &mb, &tb);
    if (rc) return rc;
    if (!signs || !idx || !q || !mu || !delta || !main_out || !meta_out) return SAGE_ERR_INVALID_ARGUMENT;
    const int V = 10 - log2K, S = d_in / kSV, G = d_in / 128, R8 = (d_out + 7) / 8;
    const uint32_t zmax = 1u << log2K, qmax = 1u << V;
    for (size_t k = 0; k < (size_t)d_out * S; ++k)
        if (idx[k] >= zmax || q[k] >= qmax) return SAGE_ERR_INVALID_ARGUMENT;
    int slot[6];
    sign_slots(V, slot);
    std::memset(main_out, 0, mb);
    std::memset(meta_out, 0, tb);
    for (int o = 0; o < d_out; ++o) {
        const int b = o >> 3, t = o & 7, u = t >> 1, rowB = t & 1;
        const PlaneIndex ix(R8, S, G, b);
        const uint8_t* srow = signs + (size_t)o * S;
        for (int j = 0; j < S; ++j) {
            uint32_t w = 0;
            const uint32_t z = idx[(size_t)o * S + j], qq = q[(size_t)o * S + j], s = srow[j];
            if (!rowB) w |= (z << 7) | (qq << (23 - V));
            else       w |= (z << 23) | (qq << (7 - V));
            for (int n = 0; n < 3; ++n) {
                const int p = slot[n + 3 * rowB];
                w |= ((s >> (2 * n)) & 1u) << p;
                w |= ((s >> (2 * n + 1)) & 1u) << (p + 16);
            }
            main_out[ix.main_word(j, u)] |= w;
            uint32_t* aux = meta_out + ix.meta_word(j / kGroupSV, t);
            *aux |= ((s >> 6) & 1u) << (j % kGroupSV);
            *aux |= ((s >> 7) & 1u) << (j % kGroupSV + 16);
        }
        for (int g = 0; g < G; ++g)
            meta_out[ix.meta_word(g, t) + 1] =
                (uint32_t)mu[(size_t)o * G + g] | ((uint32_t)delta[(size_t)o * G + g] << 16);
    }
    return SAGE_OK;
}

int sage_unpack(int d_out, int d_in, int log2K, const uint32_t* main_plane, const uint32_t* meta_plane,
                uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu, uint16_t* delta) {
    size_t mb, tb;
    int rc = sage_packed_sizes(d_out, d_in, log2K, &mb, &tb);
    if (rc) return rc;
    if (!signs || !idx || !q || !mu || !delta || !main_plane || !meta_plane) return SAGE_ERR_INVALID_ARGUMENT;
    const int V = 10 - log2K, S = d_in / kSV, G = d_in / 128, R8 = (d_out + 7) / 8;
    const uint32_t zmask = (1u << log2K) - 1, qmask = (1u << V) - 1;
    int slot[6];
    sign_slots(V, slot);
    for (int o = 0; o < d_out; ++o) {
        const int b = o >> 3, t = o & 7, u = t >> 1, rowB = t & 1;
        const PlaneIndex ix(R8, S, G, b);
        for (int j = 0; j < S; ++j) {
            const uint32_t w = main_plane[ix.main_word(j, u)];
            const uint32_t aux = meta_plane[ix.meta_word(j / kGroupSV, t)];
            uint32_t z, qq, s = 0;
            if (!rowB) { z = (w >> 7) & zmask;  qq = (w >> (23 - V)) & qmask; }
            else       { z = (w >> 23) & zmask; qq = (w >> (7 - V)) & qmask; }
            for (int n = 0; n < 3; ++n) {
                const int p = slot[n + 3 * rowB];
                s |= ((w >> p) & 1u) << (2 * n);
                s |= ((w >> (p + 16)) & 1u) << (2 * n + 1);
            }
            s |= ((aux >> (j % kGroupSV)) & 1u) << 6;
            s |= ((aux >> (j % kGroupSV + 16)) & 1u) << 7;
            signs[(size_t)o * S + j] = (uint8_t)s;
            idx[(size_t)o * S + j] = (uint16_t)z;
            q[(size_t)o * S + j] = (uint8_t)qq;
        }
        for (int g = 0; g < G; ++g) {
            const uint32_t md = meta_plane[ix.meta_word(g, t) + 1];
            mu[(size_t)o * G + g] = (uint16_t)(md & 0xffffu);
            delta[(size_t)o * G + g] = (uint16_t)(md >> 16);
        }
    }
    return SAGE_OK;
}

int sage_esg_permutation(int d_in, const double* energy, int32_t* perm_out) {
    if (!energy || !perm_out || d_in < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_in % kSV) return SAGE_ERR_UNSUPPORTED;
    std::vector<int32_t> order(d_in);
    std::iota(order.begin(), order.end(), 0);
    // Eq. 5: sigma sorts by decreasing energy; equal energies keep channel order.
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return energy[a] > energy[b]; });
    const int m = d_in / kSV;  // channels per tier
    for (int tier = 0; tier < kSV; ++tier)
        for (int j = 0; j < m; ++j) perm_out[j * kSV + tier] = order[(size_t)tier * m + j];
    return SAGE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// CPU encoder (Sec. 3.2 weighted fitting, Eq. 4-6; App. A.6 Eq. 14; Eq. 2).
// ---------------------------------------------------------------------------
namespace {

uint16_t to_half_rne(double x) {
    // IEEE binary16, round to nearest even.
    uint16_t sign = std::signbit(x) ? 0x8000 : 0;
    double a = std::fabs(x);
    if (std::isnan(x)) return 0x7e00;
    if (a == 0.0) return sign;
    if (a < std::ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)std::nearbyint(std::ldexp(a, 24)));
    int e;
    std::frexp(a, &e);
    e -= 1;
    double m = std::nearbyint(std::ldexp(a, 10 - e));
    if (m >= 2048.0) { m = 1024.0; ++e; }
    if (e > 15) return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | ((e + 15) << 10) | ((int)m - 1024));
}

double from_half(uint16_t h) {
    const int e = (h >> 10) & 31, f = h & 1023;
    double v = (e == 0) ? std::ldexp((double)f, -24)
             : (e == 31) ? (f ? NAN : INFINITY) : std::ldexp((double)(f | 1024), e - 25);
    return (h & 0x8000) ? -v : v;
}

// Eq. 6 for one subvector: returns z and writes the weighted optimal radius.
inline int best_codeword(const double* p, const double* w, const double* cb, int K, double* r_out) {
    int z = 0;
    double best = -1.0, rz = 0.0;
    for (int k = 0; k < K; ++k) {
        const double* c = cb + k * kSV;
        double num = 0.0, den = 0.0;
        for (int i = 0; i < kSV; ++i) num += w[i] * p[i] * c[i];
        for (int i = 0; i < kSV; ++i) den += w[i] * c[i] * c[i];
        if (den <= 0.0) continue;
        const double sc = num * num / den;
        if (sc > best) { best = sc; z = k; rz = num / den; }
    }
    if (best <= 0.0) { z = 0; rz = 0.0; }
    if (r_out) *r_out = rz;
    return z;
}

template <class F>
void parallel_for(int n, int n_threads, F&& f) {
    if (n_threads <= 1 || n < 64) { for (int i = 0; i < n; ++i) f(i); return; }
    std::vector<std::thread> th;
    const int chunk = (n + n_threads - 1) / n_threads;
    for (int t = 0; t < n_threads; ++t) {
        const int a = t * chunk, b = std::min(n, a + chunk);
        if (a >= b) break;
        th.emplace_back([=, &f] { for (int i = a; i < b; ++i) f(i); });
    }
    for (auto& x : th) x.join();
}

}  // namespace

namespace {
// Eq. 4: omega of storage column 8j + i = e^gamma / mean over the subvector's
// 8 channels of e^gamma, e the energies in storage order.
void omega_columns(int d_in, const double* energy, const int32_t* perm, double gamma, double* omega) {
    for (int j = 0; j < d_in / kSV; ++j) {
        double eg[kSV], mean = 0.0;
        for (int i = 0; i < kSV; ++i) { eg[i] = std::pow(energy[perm[j * kSV + i]], gamma); mean += eg[i]; }
        mean /= kSV;
        for (int i = 0; i < kSV; ++i) omega[(size_t)j * kSV + i] = eg[i] / mean;
    }
}
}  // namespace

extern "C" int sage_encode_inputs(int d_out, int d_in, const double* W, const double* energy, double gamma,
                                  int n_samples, const int64_t* sample, int32_t* perm_out, double* omega_out,
                                  double* P_out, double* Wt_out) {
    if (!W || !energy || !sample || !perm_out || !omega_out || !P_out || !Wt_out) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_out < 1 || d_in < 1 || n_samples < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_in % 128) return SAGE_ERR_UNSUPPORTED;
    const int S = d_in / kSV;
    const int64_t n_sv = (int64_t)d_out * S;
    for (int s = 0; s < n_samples; ++s)
        if (sample[s] < 0 || sample[s] >= n_sv) return SAGE_ERR_INVALID_ARGUMENT;
    const int rc = sage_esg_permutation(d_in, energy, perm_out);
    if (rc) return rc;
    omega_columns(d_in, energy, perm_out, gamma, omega_out);
    for (int s = 0; s < n_samples; ++s) {
        const int64_t o = sample[s] / S, j = sample[s] % S;
        for (int i = 0; i < kSV; ++i) {
            P_out[(size_t)s * kSV + i] = std::fabs(W[o * d_in + perm_out[j * kSV + i]]);
            Wt_out[(size_t)s * kSV + i] = omega_out[(size_t)j * kSV + i];
        }
    }
    return SAGE_OK;
}

extern "C" int sage_encode(int d_out, int d_in, int log2K, const double* W, const double* energy, double gamma,
                           int n_samples, const int64_t* sample, const int64_t* init, int iters, int n_threads,
                           int32_t* perm_out, uint16_t* codebook_out, uint8_t* signs, uint16_t* idx, uint8_t* q,
                           uint16_t* mu, uint16_t* delta) {
    if (!W || !energy || !sample || !init || !perm_out || !codebook_out || !signs || !idx || !q || !mu || !delta)
        return SAGE_ERR_INVALID_ARGUMENT;
    if (d_out < 1 || d_in < 1 || n_samples < 1 || iters < 0) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_in % 128 || log2K < 4 || log2K > 8) return SAGE_ERR_UNSUPPORTED;
    const int K = 1 << log2K, V = 10 - log2K, S = d_in / kSV, G = d_in / 128;
    const int64_t n_sv = (int64_t)d_out * S;
    for (int s = 0; s < n_samples; ++s)
        if (sample[s] < 0 || sample[s] >= n_sv) return SAGE_ERR_INVALID_ARGUMENT;
    for (int k = 0; k < K; ++k)
        if (init[k] < 0 || init[k] >= n_samples) return SAGE_ERR_INVALID_ARGUMENT;
    if (n_threads <= 0) n_threads = (int)std::max(1u, std::thread::hardware_concurrency());

    int rc = sage_esg_permutation(d_in, energy, perm_out);
    if (rc) return rc;

    // Eq. 4 weights per storage column (same for every row), e in permuted order.
    std::vector<double> omega((size_t)d_in);
    omega_columns(d_in, energy, perm_out, gamma, omega.data());
    auto magnitudes = [&](int64_t sv, double* p) {
        const int64_t o = sv / S, j = sv % S;
        for (int i = 0; i < kSV; ++i) p[i] = std::fabs(W[o * d_in + perm_out[j * kSV + i]]);
    };

    // Weighted spherical k-means on the samples.
    std::vector<double> P((size_t)n_samples * kSV), cb((size_t)K * kSV), acc((size_t)K * kSV);
    for (int s = 0; s < n_samples; ++s) magnitudes(sample[s], &P[(size_t)s * kSV]);
    for (int k = 0; k < K; ++k) {
        const double* p = &P[(size_t)init[k] * kSV];
        double nn = 0.0;
        for (int i = 0; i < kSV; ++i) nn += p[i] * p[i];
        nn = std::sqrt(nn);
        for (int i = 0; i < kSV; ++i) cb[k * kSV + i] = nn > 0.0 ? p[i] / nn : 1.0 / std::sqrt((double)kSV);
    }
    std::vector<int> z((size_t)n_samples);
    for (int it = 0; it < iters; ++it) {
        parallel_for(n_samples, n_threads, [&](int s) {
            const int64_t j = sample[s] % S;
            z[s] = best_codeword(&P[(size_t)s * kSV], &omega[(size_t)j * kSV], cb.data(), K, nullptr);
        });
        std::fill(acc.begin(), acc.end(), 0.0);
        for (int s = 0; s < n_samples; ++s) {  // fixed order: deterministic sums
            const double* p = &P[(size_t)s * kSV];
            const double* w = &omega[(size_t)(sample[s] % S) * kSV];
            double nn = 0.0;
            for (int i = 0; i < kSV; ++i) nn += p[i] * p[i];
            if (nn <= 0.0) continue;
            nn = std::sqrt(nn);
            for (int i = 0; i < kSV; ++i) acc[z[s] * kSV + i] += w[i] * p[i] / nn;
        }
        for (int k = 0; k < K; ++k) {
            double nn = 0.0;
            for (int i = 0; i < kSV; ++i) nn += acc[k * kSV + i] * acc[k * kSV + i];
            if (nn <= 0.0) continue;  // empty cluster keeps its codeword
            nn = std::sqrt(nn);
            for (int i = 0; i < kSV; ++i) cb[k * kSV + i] = acc[k * kSV + i] / nn;
        }
    }
    // Stored fp16 codebook; final assignment uses the stored values.
    for (int k = 0; k < K * kSV; ++k) {
        codebook_out[k] = to_half_rne(cb[k]);
        cb[k] = from_half(codebook_out[k]);
    }
    parallel_for(d_out, n_threads, [&](int o) {
        double r[kGroupSV];
        for (int g = 0; g < G; ++g) {
            for (int t = 0; t < kGroupSV; ++t) {
                const int j = g * kGroupSV + t;
                double p[kSV];
                uint8_t s = 0;
                for (int i = 0; i < kSV; ++i) {
                    const double wv = W[(size_t)o * d_in + perm_out[j * kSV + i]];
                    p[i] = std::fabs(wv);
                    if (wv < 0.0) s |= (uint8_t)(1u << i);
                }
                signs[(size_t)o * S + j] = s;
                idx[(size_t)o * S + j] = (uint16_t)best_codeword(p, &omega[(size_t)j * kSV], cb.data(), K, &r[t]);
            }
            double lo = r[0], hi = r[0];
            for (int t = 1; t < kGroupSV; ++t) { lo = std::min(lo, r[t]); hi = std::max(hi, r[t]); }
            const uint16_t m16 = to_half_rne(lo), d16 = to_half_rne((hi - lo) / (double)((1 << V) - 1));
            mu[(size_t)o * G + g] = m16;
            delta[(size_t)o * G + g] = d16;
            const double mv = from_half(m16), dv = from_half(d16);
            for (int t = 0; t < kGroupSV; ++t) {
                double qq = 0.0;
                if (dv > 0.0) {
                    qq = std::floor((r[t] - mv) / dv + 0.5);
                    qq = std::min(std::max(qq, 0.0), (double)((1 << V) - 1));
                }
                q[(size_t)o * S + g * kGroupSV + t] = (uint8_t)qq;
            }
        }
    });
    return SAGE_OK;
}

// ---------------------------------------------------------------------------
// Compute entry points: validation, then the launchers.
// ---------------------------------------------------------------------------
extern "C" {

int sage_workspace_size(int op, const sage_matrix* mats, int n, int M, size_t* bytes) {
    if (!bytes || !mats || n < 1) return SAGE_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < n; ++i)
        if (mats[i].d_out < 1 || mats[i].d_in < 1) return SAGE_ERR_INVALID_ARGUMENT;
    switch (op) {
        case SAGE_OP_GEMV:
        case SAGE_OP_GROUPED: *bytes = gemv_workspace_bytes(mats, n, M); return SAGE_OK;
        case SAGE_OP_GEMM: {
            size_t b = 0;
            for (int i = 0; i < n; ++i) b = std::max(b, std::max(gemm_workspace_bytes(&mats[i], M),
                                                                 gemv_workspace_bytes(&mats[i], 1, M)));
            *bytes = b;
            return SAGE_OK;
        }
        case SAGE_OP_MOE: *bytes = moe_workspace_bytes(mats, n, M); return SAGE_OK;
        case SAGE_OP_ABS: *bytes = abs_workspace_bytes(n); return SAGE_OK;
        default: return SAGE_ERR_INVALID_ARGUMENT;
    }
}

static int check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (!ws) return SAGE_ERR_WORKSPACE;
    if (!aligned16(ws)) return SAGE_ERR_MISALIGNED;
    if (ws_bytes < need) return SAGE_ERR_WORKSPACE;
    return SAGE_OK;
}

int sage_gemv(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y, void* ws, size_t ws_bytes,
              sage_stream_t stream) {
    int rc = check_matrix(A);
    if (rc) return rc;
    if (!x || !y) return SAGE_ERR_INVALID_ARGUMENT;
    if (M < 1 || M > 8) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(y)) return SAGE_ERR_MISALIGNED;
    if ((rc = check_ws(ws, ws_bytes, gemv_workspace_bytes(A, 1, M)))) return rc;
    GemvJob job{*A, x, y};
    return launch_gemv(&job, 1, M, ws, ws_bytes, stream);
}

int sage_gemv_grouped(const sage_matrix* mats, int n, const uint16_t* const* xs, uint16_t* const* ys, int M,
                      void* ws, size_t ws_bytes, sage_stream_t stream) {
    if (!mats || !xs || !ys || n < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (n > 64) return SAGE_ERR_UNSUPPORTED;
    if (M < 1 || M > 8) return SAGE_ERR_UNSUPPORTED;
    std::vector<GemvJob> jobs((size_t)n);
    for (int i = 0; i < n; ++i) {
        int rc = check_matrix(&mats[i]);
        if (rc) return rc;
        if (!xs[i] || !ys[i]) return SAGE_ERR_INVALID_ARGUMENT;
        if (!aligned16(xs[i]) || !aligned16(ys[i])) return SAGE_ERR_MISALIGNED;
        jobs[i] = GemvJob{mats[i], xs[i], ys[i]};
    }
    int rc = check_ws(ws, ws_bytes, gemv_workspace_bytes(mats, n, M));
    if (rc) return rc;
    return launch_gemv(jobs.data(), n, M, ws, ws_bytes, stream);
}

int sage_gemm(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y, void* ws, size_t ws_bytes,
              sage_stream_t stream) {
    int rc = check_matrix(A);
    if (rc) return rc;
    if (!x || !y) return SAGE_ERR_INVALID_ARGUMENT;
    if (M < 1 || M > 256) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(y)) return SAGE_ERR_MISALIGNED;
    if (M <= 8) return sage_gemv(A, x, M, y, ws, ws_bytes, stream);
    if ((rc = check_ws(ws, ws_bytes, gemm_workspace_bytes(A, M)))) return rc;
    return launch_gemm(A, x, M, y, ws, ws_bytes, stream);
}

int sage_moe_gemv(const sage_matrix* experts, int n_experts, const int32_t* pair_expert, const int32_t* pair_xrow,
                  int n_pairs, const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes, sage_stream_t stream) {
    if (!experts || n_experts < 1 || !pair_expert || !pair_xrow || n_pairs < 1 || !x || !y)
        return SAGE_ERR_INVALID_ARGUMENT;
    if (n_experts > 256 || n_pairs > 4096) return SAGE_ERR_UNSUPPORTED;
    for (int e = 0; e < n_experts; ++e) {
        int rc = check_matrix(&experts[e]);
        if (rc) return rc;
        if (experts[e].d_out != experts[0].d_out || experts[e].d_in != experts[0].d_in) return SAGE_ERR_UNSUPPORTED;
    }
    if (!aligned16(x) || !aligned16(y) || !aligned16(pair_expert) || !aligned16(pair_xrow)) return SAGE_ERR_MISALIGNED;
    int rc = check_ws(ws, ws_bytes, moe_workspace_bytes(experts, n_experts, n_pairs));
    if (rc) return rc;
    return launch_moe(experts, n_experts, pair_expert, pair_xrow, n_pairs, x, y, ws, ws_bytes, stream);
}

int sage_dequant(const sage_matrix* A, uint16_t* W, sage_stream_t stream) {
    int rc = check_matrix(A);
    if (rc) return rc;
    if (!W) return SAGE_ERR_INVALID_ARGUMENT;
    if (!aligned16(W)) return SAGE_ERR_MISALIGNED;
    return launch_dequant(A, W, stream);
}

int sage_unpack_device(const sage_matrix* A, uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu,
                       uint16_t* delta, sage_stream_t stream) {
    int rc = check_matrix(A);
    if (rc) return rc;
    if (!signs || !idx || !q || !mu || !delta) return SAGE_ERR_INVALID_ARGUMENT;
    return launch_unpack(A, signs, idx, q, mu, delta, stream);
}

int sage_permute_x(const uint16_t* x, const int32_t* perm, int M, int d_in, uint16_t* x_perm, sage_stream_t stream) {
    if (!x || !x_perm || M < 1 || d_in < 1) return SAGE_ERR_INVALID_ARGUMENT;
    if (d_in % kSV) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(x_perm) || (perm && !aligned16(perm))) return SAGE_ERR_MISALIGNED;
    return launch_permute(x, perm, M, d_in, x_perm, stream);
}

int sage_query_status(void* ws, sage_stream_t stream) {
    if (!ws) return SAGE_ERR_WORKSPACE;
    return read_and_clear_status(ws, stream);
}

}  // extern "C"
