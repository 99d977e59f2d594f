/*
 * SAGE CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct fp64 restatement of what the SAGE packed
 * linear layer computes.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library.  It shares no code, header,
 * table or constant with the CUDA library (bit_vector_quantized_sage_b200).
 *
 * Source: "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World
 * Usability" (Yan et al.), cited by section / equation:
 *   Sec. 3.1 Eq. 1   reconstruction w_hat = r_hat * (s (.) c_z)
 *   Sec. 3.1 Eq. 2   radius grid r_hat = mu_g + q delta_g, q = clip(round((r~ - mu)/delta), 0, 2^V - 1)
 *   Sec. 3.1 Eq. 3   budget B = v + log2 K + V
 *   Sec. 3.2 Eq. 4   activation weights omega_i = e^gamma / mean(e^gamma)
 *   Sec. 3.2 Eq. 5   ESG permutation pi((j-1)v + t) = sigma((t-1)m + j)
 *   Sec. 3.2 Eq. 6   weighted radius and direction assignment
 *   Sec. 3.5         16-bit main word + 2 auxiliary bits per subvector
 *   App. A.6 Eq. 14  mu_g = min r~, delta_g = (max r~ - mu_g) / (2^V - 1), groups of 16 subvectors
 *   App. A.6 Eq. 15  BPW = B/v + 2 b_g / G + K v b_c / N
 *
 * The packed layout decoded by oracle_unpack is the CUDA library's own format
 * (version 2; the paper fixes only the field widths); it is restated here from
 * its written specification, independently of the library's packer.
 *
 * Parity status: every function below is pinned by tests/test_oracle_*.py
 * except oracle_kmeans / oracle_encode beyond determinism and the invariants
 * listed there ("parity unpinned" for the k-means codebook itself: the paper
 * names the algorithm but not its update rule, initialisation or empty-cluster
 * handling).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SV 8            /* subvector dimension v */
#define GROUP_SV 16     /* subvectors per radius group (G / v = 128 / 8) */

/* ------------------------------------------------------------------ */
/* IEEE binary16 <-> binary64, written from the format definition.    */
/* ------------------------------------------------------------------ */

double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp(1024.0 + (double)m, e - 25);     /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round to nearest, ties to even. */
uint16_t oracle_double_to_half(double x) {
    uint16_t sign = (signbit(x) ? 0x8000 : 0);
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {                     /* subnormal range */
        double r = nearbyint(ldexp(a, 24));        /* units of 2^-24 */
        return (uint16_t)(sign | (uint16_t)r);     /* r == 1024 is the smallest normal */
    }
    int E;
    frexp(a, &E);                                   /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;                                  /* a in [2^e, 2^(e+1)) */
    double s = nearbyint(ldexp(a, 10 - e));         /* significand in [1024, 2048] */
    if (s >= 2048.0) { s = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7c00);   /* overflow to infinity */
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(s - 1024.0));
}

/* ------------------------------------------------------------------ */
/* Packed format v2 (the library's layout), restated from its spec.    */
/*                                                                     */
/* R8 = ceil(d_out / 8) row octets (octet b = rows 8b..8b+7); blocks   */
/* of 32 octets (256 rows), block B holding n_B = min(32, R8 - 32B)    */
/* octets.  S = d_in / 8 subvector columns, G = d_in / 128 groups.     */
/* main: uint32 words.  Record (j, octet o of block B) is the 4 words  */
/*   at B * S * 128 + (j * n_B + o) * 4.  Word u holds row A =         */
/*   8(32B + o) + 2u and row B = row A + 1:                            */
/*     z_A at bits [7, 7 + log2K)      q_A at bits [23 - V, 23)        */
/*     z_B at bits [23, 23 + log2K)    q_B at bits [7 - V, 7)          */
/*   six sign slots at the ascending positions p_0 < ... < p_5 of      */
/*   {0 .. 6 - V} U {17 - V .. 15}; slot k owns bits p_k and p_k + 16. */
/*   Slots 0..2 carry row A's component pairs 0..2, slots 3..5 row B's; */
/*   pair n = components (2n, 2n+1): bit p_k is the sign of 2n, bit    */
/*   p_k + 16 the sign of 2n + 1.                                       */
/* meta: 8-byte entries; entry (g, octet o of block B, row t) is at    */
/*   entry index B * G * 256 + (g * n_B + o) * 8 + t:                  */
/*   uint32 aux, uint16 mu, uint16 delta (little endian).              */
/*   aux bit t' = sign of component 6 of subvector 16g + t',           */
/*   aux bit t' + 16 = sign of component 7 of that subvector.          */
/* Rows past d_out in the last octet are zero.                          */
/* ------------------------------------------------------------------ */

static int slot_pos(int V, int k) {
    int n = 0;
    for (int p = 0; p < 16; ++p) {
        int in_low = (p <= 6 - V);
        int in_high = (p >= 17 - V);
        if (in_low || in_high) {
            if (n == k) return p;
            ++n;
        }
    }
    return -1;
}

static uint32_t getbits(uint32_t w, int lo, int n) {
    return (w >> lo) & ((1u << n) - 1u);
}

int oracle_unpack(int d_out, int d_in, int log2K,
                     const uint32_t* main_plane, const uint32_t* meta_plane,
                     uint8_t* signs, uint16_t* idx, uint8_t* q,
                     uint16_t* mu, uint16_t* delta) {
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return 1;
    const int V = 10 - log2K;
    const int S = d_in / SV, G = d_in / 128, R8 = (d_out + 7) / 8;
    for (int o = 0; o < d_out; ++o) {
        const int b = o / 8, t = o % 8, u = t / 2, isB = t & 1;
        const int blk = b / 32, ob = b % 32;
        const int nB = (R8 - 32 * blk < 32) ? R8 - 32 * blk : 32;
        const size_t main0 = (size_t)blk * S * 128, meta0 = (size_t)blk * G * 256;
        for (int j = 0; j < S; ++j) {
            const uint32_t w = main_plane[main0 + ((size_t)j * nB + ob) * 4 + u];
            const uint32_t aux = meta_plane[(meta0 + ((size_t)(j / GROUP_SV) * nB + ob) * 8 + t) * 2];
            uint32_t z, qq;
            if (!isB) { z = getbits(w, 7, log2K);  qq = getbits(w, 23 - V, V); }
            else      { z = getbits(w, 23, log2K); qq = getbits(w, 7 - V, V); }
            uint32_t s = 0;
            for (int n = 0; n < 3; ++n) {
                const int p = slot_pos(V, n + (isB ? 3 : 0));
                s |= getbits(w, p, 1) << (2 * n);
                s |= getbits(w, p + 16, 1) << (2 * n + 1);
            }
            const int tj = j % GROUP_SV;
            s |= getbits(aux, tj, 1) << 6;
            s |= getbits(aux, tj + 16, 1) << 7;
            signs[(size_t)o * S + j] = (uint8_t)s;
            idx[(size_t)o * S + j] = (uint16_t)z;
            q[(size_t)o * S + j] = (uint8_t)qq;
        }
        for (int g = 0; g < G; ++g) {
            const uint32_t md = meta_plane[(meta0 + ((size_t)g * nB + ob) * 8 + t) * 2 + 1];
            mu[(size_t)o * G + g] = (uint16_t)(md & 0xffff);
            delta[(size_t)o * G + g] = (uint16_t)(md >> 16);
        }
    }
    return 0;
}

/* The inverse of oracle_unpack over the same layout: writes every bit
 * of the planes (main_words = ceil(d_out/256) blocks of S * 128 words at
 * most, meta_words likewise G * 512), zero where no field lands.  Fields
 * wider than their slots are rejected (return 2).  Test and benchmark
 * infrastructure only: it lets the CPU baseline start from packed planes
 * without the library's packer. */
int oracle_pack(int d_out, int d_in, int log2K,
                const uint8_t* signs, const uint16_t* idx, const uint8_t* q,
                const uint16_t* mu, const uint16_t* delta,
                uint32_t* main_plane, size_t main_words, uint32_t* meta_plane, size_t meta_words) {
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return 1;
    const int V = 10 - log2K;
    const int S = d_in / SV, G = d_in / 128, R8 = (d_out + 7) / 8;
    memset(main_plane, 0, main_words * 4);
    memset(meta_plane, 0, meta_words * 4);
    for (int o = 0; o < d_out; ++o) {
        const int b = o / 8, t = o % 8, u = t / 2, isB = t & 1;
        const int blk = b / 32, ob = b % 32;
        const int nB = (R8 - 32 * blk < 32) ? R8 - 32 * blk : 32;
        const size_t main0 = (size_t)blk * S * 128, meta0 = (size_t)blk * G * 256;
        for (int j = 0; j < S; ++j) {
            const uint32_t z = idx[(size_t)o * S + j], qq = q[(size_t)o * S + j], s = signs[(size_t)o * S + j];
            if (z >> log2K || qq >> V) return 2;
            const size_t wi = main0 + ((size_t)j * nB + ob) * 4 + u;
            if (wi >= main_words) return 3;
            uint32_t w = 0;
            if (!isB) w |= (z << 7) | (qq << (23 - V));
            else      w |= (z << 23) | (qq << (7 - V));
            for (int n = 0; n < 3; ++n) {
                const int p = slot_pos(V, n + (isB ? 3 : 0));
                w |= ((s >> (2 * n)) & 1u) << p;
                w |= ((s >> (2 * n + 1)) & 1u) << (p + 16);
            }
            main_plane[wi] |= w;
            const size_t ai = (meta0 + ((size_t)(j / GROUP_SV) * nB + ob) * 8 + t) * 2;
            if (ai + 1 >= meta_words) return 3;
            const int tj = j % GROUP_SV;
            meta_plane[ai] |= (((s >> 6) & 1u) << tj) | (((s >> 7) & 1u) << (tj + 16));
        }
        for (int g = 0; g < G; ++g) {
            const size_t mi = (meta0 + ((size_t)g * nB + ob) * 8 + t) * 2 + 1;
            if (mi >= meta_words) return 3;
            meta_plane[mi] = (uint32_t)mu[(size_t)o * G + g] | ((uint32_t)delta[(size_t)o * G + g] << 16);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Reconstruction (Eq. 1 with Eq. 2's grid).                           */
/* W[o][8j + i] = (mu + q delta) * s_i * c_z[i], storage column order. */
/* ------------------------------------------------------------------ */

void oracle_dequant(int d_out, int d_in, int log2K,
                    const uint8_t* signs, const uint16_t* idx, const uint8_t* q,
                    const uint16_t* mu, const uint16_t* delta, const uint16_t* codebook,
                    double* W) {
    const int S = d_in / SV, G = d_in / 128;
    (void)log2K;
    for (int o = 0; o < d_out; ++o) {
        for (int j = 0; j < S; ++j) {
            const int g = j / GROUP_SV;
            const double m = oracle_half_to_double(mu[(size_t)o * G + g]);
            const double d = oracle_half_to_double(delta[(size_t)o * G + g]);
            const double r_hat = m + (double)q[(size_t)o * S + j] * d;
            const uint16_t* c = codebook + (size_t)idx[(size_t)o * S + j] * SV;
            const uint8_t s = signs[(size_t)o * S + j];
            for (int i = 0; i < SV; ++i) {
                const double sgn = ((s >> i) & 1) ? -1.0 : 1.0;
                W[(size_t)o * d_in + (size_t)j * SV + i] = r_hat * sgn * oracle_half_to_double(c[i]);
            }
        }
    }
}

/* fp16 (round to nearest even) copy of a reconstructed matrix. */
void oracle_round_half(size_t n, const double* W, uint16_t* out) {
    for (size_t k = 0; k < n; ++k) out[k] = oracle_double_to_half(W[k]);
}

/* ------------------------------------------------------------------ */
/* y = W_hat x_perm.  W_hat is rounded to fp32, products and sums in   */
/* fp64.  x is fp16 [M][d_in] in original channel order; x_perm[p] =   */
/* x[perm[p]] (perm == NULL: identity).  bound = sum |W32| |x_perm|.   */
/* ------------------------------------------------------------------ */

void oracle_gemv(int d_out, int d_in, int M, const double* W,
                 const uint16_t* x, const int32_t* perm, double* y, double* bound) {
    double* xp = (double*)malloc(sizeof(double) * (size_t)d_in);
    for (int m = 0; m < M; ++m) {
        for (int p = 0; p < d_in; ++p) {
            const int c = perm ? perm[p] : p;
            xp[p] = oracle_half_to_double(x[(size_t)m * d_in + c]);
        }
        for (int o = 0; o < d_out; ++o) {
            double acc = 0.0, b = 0.0;
            const double* row = W + (size_t)o * d_in;
            for (int p = 0; p < d_in; ++p) {
                const double w32 = (double)(float)row[p];
                acc += w32 * xp[p];
                b += fabs(w32) * fabs(xp[p]);
            }
            y[(size_t)m * d_out + o] = acc;
            if (bound) bound[(size_t)m * d_out + o] = b;
        }
    }
    free(xp);
}

/* Fields -> y directly (dequant then gemv), rows [row0, row1) only. */
void oracle_gemv_fields_rows(int d_out, int d_in, int log2K, int row0, int row1,
                             const uint8_t* signs, const uint16_t* idx, const uint8_t* q,
                             const uint16_t* mu, const uint16_t* delta, const uint16_t* codebook,
                             int M, const uint16_t* x, const int32_t* perm,
                             double* y, double* bound) {
    const int S = d_in / SV, G = d_in / 128;
    double* W = (double*)malloc(sizeof(double) * (size_t)d_in);
    double* xp = (double*)malloc(sizeof(double) * (size_t)d_in * M);
    (void)log2K;
    for (int m = 0; m < M; ++m)
        for (int p = 0; p < d_in; ++p)
            xp[(size_t)m * d_in + p] = oracle_half_to_double(x[(size_t)m * d_in + (perm ? perm[p] : p)]);
    for (int o = row0; o < row1 && o < d_out; ++o) {
        oracle_dequant(1, d_in, log2K, signs + (size_t)o * S, idx + (size_t)o * S, q + (size_t)o * S,
                       mu + (size_t)o * G, delta + (size_t)o * G, codebook, W);
        for (int m = 0; m < M; ++m) {
            double acc = 0.0, b = 0.0;
            for (int p = 0; p < d_in; ++p) {
                const double w32 = (double)(float)W[p];
                acc += w32 * xp[(size_t)m * d_in + p];
                b += fabs(w32) * fabs(xp[(size_t)m * d_in + p]);
            }
            y[(size_t)m * d_out + o] = acc;
            if (bound) bound[(size_t)m * d_out + o] = b;
        }
    }
    free(W);
    free(xp);
}

/* ------------------------------------------------------------------ */
/* Encoder steps (Sec. 3.2-3.3, App. A.6).                             */
/* ------------------------------------------------------------------ */

static const double* g_sort_key;
static int cmp_energy_desc(const void* a, const void* b) {
    const int ia = *(const int*)a, ib = *(const int*)b;
    const double ea = g_sort_key[ia], eb = g_sort_key[ib];
    if (ea > eb) return -1;
    if (ea < eb) return 1;
    return (ia < ib) ? -1 : (ia > ib);   /* stable: lower index first */
}

/* Eq. 5: sigma sorts channels by decreasing energy; 8 tiers of m = n/8;
 * storage position j*8 + t holds sigma[t*m + j] (0-based j, t). */
int oracle_esg_perm(int n, const double* energy, int32_t* perm) {
    if (n % SV) return 1;
    int* sigma = (int*)malloc(sizeof(int) * (size_t)n);
    for (int c = 0; c < n; ++c) sigma[c] = c;
    g_sort_key = energy;
    qsort(sigma, (size_t)n, sizeof(int), cmp_energy_desc);
    const int m = n / SV;
    for (int j = 0; j < m; ++j)
        for (int t = 0; t < SV; ++t)
            perm[j * SV + t] = sigma[t * m + j];
    free(sigma);
    return 0;
}

/* Eq. 4: omega_i = e_i^gamma / ((1/v) sum_j e_j^gamma). */
void oracle_omega(const double* e8, double gamma, double* w8) {
    double mean = 0.0;
    for (int i = 0; i < SV; ++i) mean += pow(e8[i], gamma);
    mean /= SV;
    for (int i = 0; i < SV; ++i) w8[i] = pow(e8[i], gamma) / mean;
}

/* Eq. 6: r*_k = sum w p c / sum w c^2, z = argmax_k (sum w p c)^2 / sum w c^2.
 * Ties keep the smallest k; an all-zero score (p == 0) gives z = 0, r* = 0. */
int oracle_assign(const double* p8, const double* w8, const double* cb, int K, double* rstar) {
    int best = 0;
    double best_score = -1.0, best_r = 0.0;
    for (int k = 0; k < K; ++k) {
        double num = 0.0, den = 0.0;
        for (int i = 0; i < SV; ++i) {
            num += w8[i] * p8[i] * cb[k * SV + i];
            den += w8[i] * cb[k * SV + i] * cb[k * SV + i];
        }
        if (den <= 0.0) continue;
        const double score = num * num / den;
        if (score > best_score) { best_score = score; best = k; best_r = num / den; }
    }
    if (best_score <= 0.0) { best = 0; best_r = 0.0; }
    if (rstar) *rstar = best_r;
    return best;
}

/* Eq. 14 over one group of 16 fitted radii; results stored as fp16. */
void oracle_grid(const double* r16, int V, uint16_t* mu16, uint16_t* delta16) {
    double lo = r16[0], hi = r16[0];
    for (int t = 1; t < GROUP_SV; ++t) {
        if (r16[t] < lo) lo = r16[t];
        if (r16[t] > hi) hi = r16[t];
    }
    *mu16 = oracle_double_to_half(lo);
    *delta16 = oracle_double_to_half((hi - lo) / (double)((1 << V) - 1));
}

/* Eq. 2 with the stored fp16 grid; delta == 0 gives q = 0. */
int oracle_quantize(double r, uint16_t mu16, uint16_t delta16, int V) {
    const double mu = oracle_half_to_double(mu16), d = oracle_half_to_double(delta16);
    if (!(d > 0.0)) return 0;
    double qq = floor((r - mu) / d + 0.5);
    if (qq < 0.0) qq = 0.0;
    if (qq > (double)((1 << V) - 1)) qq = (double)((1 << V) - 1);
    return (int)qq;
}

/* Weighted spherical k-means (Sec. 3.2, "Weighted Quantizer Fitting"; Sec. 4.1
 * implementation details: initialised with activation-weighted spherical
 * k-means on 65,536 sampled subvectors, 20 iterations in the paper).  Each iteration assigns
 * every sample by Eq. 6 and moves each codeword to the normalised
 * omega-weighted sum of its members' unit directions; an empty cluster keeps
 * its codeword.  Initial codewords are the unit directions of the samples
 * listed in init[0..K).  P and Wt are n x 8 (magnitudes and weights). */
void oracle_kmeans(int n, const double* P, const double* Wt, int K, const int64_t* init,
                   int iters, double* cb) {
    int* z = (int*)malloc(sizeof(int) * (size_t)n);
    double* acc = (double*)malloc(sizeof(double) * (size_t)K * SV);
    for (int k = 0; k < K; ++k) {
        const double* p = P + (size_t)init[k] * SV;
        double nn = 0.0;
        for (int i = 0; i < SV; ++i) nn += p[i] * p[i];
        nn = sqrt(nn);
        for (int i = 0; i < SV; ++i) cb[k * SV + i] = (nn > 0.0) ? p[i] / nn : 1.0 / sqrt((double)SV);
    }
    for (int it = 0; it < iters; ++it) {
        for (int s = 0; s < n; ++s) z[s] = oracle_assign(P + (size_t)s * SV, Wt + (size_t)s * SV, cb, K, NULL);
        memset(acc, 0, sizeof(double) * (size_t)K * SV);
        for (int s = 0; s < n; ++s) {
            const double* p = P + (size_t)s * SV;
            double nn = 0.0;
            for (int i = 0; i < SV; ++i) nn += p[i] * p[i];
            if (nn <= 0.0) continue;
            nn = sqrt(nn);
            for (int i = 0; i < SV; ++i) acc[z[s] * SV + i] += Wt[(size_t)s * SV + i] * p[i] / nn;
        }
        for (int k = 0; k < K; ++k) {
            double nn = 0.0;
            for (int i = 0; i < SV; ++i) nn += acc[k * SV + i] * acc[k * SV + i];
            if (nn <= 0.0) continue;
            nn = sqrt(nn);
            for (int i = 0; i < SV; ++i) cb[k * SV + i] = acc[k * SV + i] / nn;
        }
    }
    free(z);
    free(acc);
}

/* Per-matrix initialisation of Algorithm 1 (App. A.7) for one (K, V):
 * ESG permutation, omega weights, weighted k-means on the sampled subvectors,
 * fp16 codebook, Eq. 6 assignment of every subvector against the stored
 * codebook, Eq. 14 grid per group (fp16) and Eq. 2 radius codes.
 * W is d_out x d_in in original channel order; sample holds subvector ids
 * o * (d_in/8) + j; init holds positions into sample. */
/* The per-row part of the encoder for a given stored codebook: signs, the
 * Eq. 6 assignment of every subvector (storage column order through perm,
 * omega per storage column), the Eq. 14 grid of every group of 16 and the
 * Eq. 2 radius codes.  codebook: fp16 [K][8] as stored. */
void oracle_encode_rows(int d_out, int d_in, int log2K, const double* W, const int32_t* perm,
                        const double* omega, const uint16_t* codebook,
                        uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu, uint16_t* delta) {
    const int K = 1 << log2K, V = 10 - log2K, S = d_in / SV, G = d_in / 128;
    double* cb = (double*)malloc(sizeof(double) * (size_t)K * SV);
    for (int k = 0; k < K * SV; ++k) cb[k] = oracle_half_to_double(codebook[k]);
    double rs[GROUP_SV];
    for (int o = 0; o < d_out; ++o) {
        for (int g = 0; g < G; ++g) {
            for (int t = 0; t < GROUP_SV; ++t) {
                const int j = g * GROUP_SV + t;
                double p8[SV];
                uint8_t s = 0;
                for (int i = 0; i < SV; ++i) {
                    const double w = W[(size_t)o * d_in + perm[j * SV + i]];
                    p8[i] = fabs(w);
                    if (w < 0.0) s |= (uint8_t)(1u << i);
                }
                signs[(size_t)o * S + j] = s;
                idx[(size_t)o * S + j] = (uint16_t)oracle_assign(p8, omega + (size_t)j * SV, cb, K, &rs[t]);
            }
            oracle_grid(rs, V, &mu[(size_t)o * G + g], &delta[(size_t)o * G + g]);
            for (int t = 0; t < GROUP_SV; ++t)
                q[(size_t)o * S + g * GROUP_SV + t] =
                    (uint8_t)oracle_quantize(rs[t], mu[(size_t)o * G + g], delta[(size_t)o * G + g], V);
        }
    }
    free(cb);
}

int oracle_encode(int d_out, int d_in, int log2K, const double* W, const double* energy,
                  double gamma, int n_samples, const int64_t* sample, const int64_t* init, int iters,
                  int32_t* perm, uint16_t* codebook,
                  uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu, uint16_t* delta) {
    if (d_in % 128 || log2K < 4 || log2K > 8) return 1;
    const int K = 1 << log2K, V = 10 - log2K, S = d_in / SV, G = d_in / 128;
    if (oracle_esg_perm(d_in, energy, perm)) return 1;
    double* omega = (double*)malloc(sizeof(double) * (size_t)d_in);
    for (int j = 0; j < S; ++j) {
        double e8[SV];
        for (int i = 0; i < SV; ++i) e8[i] = energy[perm[j * SV + i]];
        oracle_omega(e8, gamma, omega + (size_t)j * SV);
    }
    double* P = (double*)malloc(sizeof(double) * (size_t)n_samples * SV);
    double* Wt = (double*)malloc(sizeof(double) * (size_t)n_samples * SV);
    for (int s = 0; s < n_samples; ++s) {
        const int64_t id = sample[s];
        const int o = (int)(id / S), j = (int)(id % S);
        for (int i = 0; i < SV; ++i) {
            P[(size_t)s * SV + i] = fabs(W[(size_t)o * d_in + perm[j * SV + i]]);
            Wt[(size_t)s * SV + i] = omega[(size_t)j * SV + i];
        }
    }
    double* cb = (double*)malloc(sizeof(double) * (size_t)K * SV);
    oracle_kmeans(n_samples, P, Wt, K, init, iters, cb);
    for (int k = 0; k < K * SV; ++k) {
        codebook[k] = oracle_double_to_half(cb[k]);
        cb[k] = oracle_half_to_double(codebook[k]);
    }
    oracle_encode_rows(d_out, d_in, log2K, W, perm, omega, codebook, signs, idx, q, mu, delta);
    free(omega); free(P); free(Wt); free(cb);
    return 0;
}

/* Eq. 15: bits per weight of one matrix with N weights. */
double oracle_bpw(int v, int B, int G, int bg, int K, int bc, double N) {
    return (double)B / v + 2.0 * bg / G + (double)K * v * bc / N;
}

/* ------------------------------------------------------------------ */
/* The operations either side of the packed GEMVs in a decoder layer  */
/* (Sec. 3.5: the ESG permutation is fused with the preceding          */
/* normalisation or activation).  fp16 in, fp64 arithmetic, fp16 out   */
/* (the activations a layer stores between its projections).           */
/* ------------------------------------------------------------------ */

/* RMSNorm of each of the M rows of x [M][d] with weight g [d]:
 *   out = fp16( x * g / sqrt(mean(x^2) + eps) ). */
void oracle_rmsnorm(int M, int d, const uint16_t* x, const uint16_t* g, double eps, uint16_t* out) {
    for (int m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int c = 0; c < d; ++c) {
            const double v = oracle_half_to_double(x[(size_t)m * d + c]);
            ss += v * v;
        }
        const double inv = 1.0 / sqrt(ss / (double)d + eps);
        for (int c = 0; c < d; ++c) {
            const double v = oracle_half_to_double(x[(size_t)m * d + c]);
            out[(size_t)m * d + c] = oracle_double_to_half(v * oracle_half_to_double(g[c]) * inv);
        }
    }
}

/* Elementwise fp16 sum (the residual stream): out = fp16(a + b). */
void oracle_add(size_t n, const uint16_t* a, const uint16_t* b, uint16_t* out) {
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_double_to_half(oracle_half_to_double(a[i]) + oracle_half_to_double(b[i]));
}

/* SwiGLU activation: out = fp16( silu(gate) * up ), silu(t) = t / (1 + e^-t). */
void oracle_silu_mul(size_t n, const uint16_t* gate, const uint16_t* up, uint16_t* out) {
    for (size_t i = 0; i < n; ++i) {
        const double t = oracle_half_to_double(gate[i]);
        out[i] = oracle_double_to_half(t / (1.0 + exp(-t)) * oracle_half_to_double(up[i]));
    }
}

/* Router-weighted combine of a mixture-of-experts projection: token t's
 * output is the sum over its top-k slots of the router weight times the
 * slot's expert output, out[t] = fp16( sum_k w[t][k] * y[t*topk + k] ),
 * summed in slot order in fp64.  y: [T*topk][d]; w: [T][topk]; out: [T][d]. */
void oracle_moe_combine(int T, int topk, int d, const uint16_t* y, const double* w, uint16_t* out) {
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int k = 0; k < topk; ++k)
                acc += w[(size_t)t * topk + k] * oracle_half_to_double(y[((size_t)t * topk + k) * d + c]);
            out[(size_t)t * d + c] = oracle_double_to_half(acc);
        }
}

/* Attention over a single cached position (the first token of a sequence):
 * the softmax over one key is 1, so query head h returns the value vector of
 * its key/value head h / (n_heads / n_kv) (grouped-query attention).
 * v: [M][n_kv * hd]; out: [M][n_heads * hd]. */
void oracle_attend_one_position(int M, int n_heads, int n_kv, int hd, const uint16_t* v, uint16_t* out) {
    const int grp = n_heads / n_kv;
    for (int m = 0; m < M; ++m)
        for (int h = 0; h < n_heads; ++h)
            for (int e = 0; e < hd; ++e)
                out[((size_t)m * n_heads + h) * hd + e] = v[((size_t)m * n_kv + h / grp) * hd + e];
}

/* ------------------------------------------------------------------ */
/* Continuous-parameter decode for blockwise optimisation (Sec. 3.4,   */
/* App. A.6; Eqs. 12-14 and Eq. 2): the forward pass that blockwise    */
/* training evaluates, with the discrete assignments (signs, codeword  */
/* indices) kept and the codebook and radii continuous.                */
/* ------------------------------------------------------------------ */

#define QDQ_EPS 1e-4
#define QDQ_HALF_PI 1.57079632679489661923  /* pi / 2 */

/* Eq. 13: theta = eps + (pi/2 - 2 eps) * sigmoid(alpha). */
double oracle_qdq_angle(double alpha) {
    return QDQ_EPS + (QDQ_HALF_PI - 2.0 * QDQ_EPS) / (1.0 + exp(-alpha));
}

/* Eq. 12: the unit codeword of v - 1 = 7 hyperspherical angles,
 *   c_1 = cos t_1,  c_j = sin t_1 ... sin t_{j-1} cos t_j (j = 2..7),
 *   c_8 = sin t_1 ... sin t_7;
 * every angle lies in (0, pi/2), so every component is positive.
 * alpha: [K][7] logits; cb: [K][8]. */
void oracle_codebook_from_angles(int K, const float* alpha, double* cb) {
    for (int k = 0; k < K; ++k) {
        double s = 1.0;
        for (int i = 0; i < SV - 1; ++i) {
            const double t = oracle_qdq_angle((double)alpha[(size_t)k * (SV - 1) + i]);
            cb[(size_t)k * SV + i] = s * cos(t);
            s *= sin(t);
        }
        cb[(size_t)k * SV + SV - 1] = s;
    }
}

/* r~ = softplus(rho) = log(1 + e^rho). */
double oracle_softplus(double rho) {
    return rho > 0.0 ? rho + log1p(exp(-rho)) : log1p(exp(rho));
}

/* The forward pass: per row group of 16 subvectors the grid spans the
 * continuous radii (Eq. 14: mu = min r~, delta = (max r~ - min r~) /
 * (2^V - 1), in full precision: the grid is recomputed from the current
 * radii each step); q = clamp(floor((r~ - mu) / delta + 0.5), 0, 2^V - 1)
 * (Eq. 2; delta = 0 gives q = 0, so a group of equal radii reconstructs
 * their common value); r^ = mu + q delta; W[o][8j + i] = r^ s_i c_{z,i}
 * (Eq. 1), storage column order.  t_out (optional): (r~ - mu) / delta of
 * every subvector (0 where delta = 0), for checking rounding ties.
 * Returns 1 for an unsupported shape. */
int oracle_qdq_forward(int d_out, int d_in, int log2K, const float* alpha, const float* rho,
                       const uint8_t* signs, const uint16_t* idx, double* W, uint8_t* q, double* t_out) {
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return 1;
    const int K = 1 << log2K, V = 10 - log2K, S = d_in / SV, G = d_in / 128;
    double* cb = (double*)malloc(sizeof(double) * (size_t)K * SV);
    if (!cb) return 2;
    oracle_codebook_from_angles(K, alpha, cb);
    for (int o = 0; o < d_out; ++o) {
        for (int g = 0; g < G; ++g) {
            double r[GROUP_SV], lo = 0.0, hi = 0.0;
            for (int t = 0; t < GROUP_SV; ++t) {
                r[t] = oracle_softplus((double)rho[(size_t)o * S + g * GROUP_SV + t]);
                if (t == 0 || r[t] < lo) lo = r[t];
                if (t == 0 || r[t] > hi) hi = r[t];
            }
            const double delta = (hi - lo) / (double)((1 << V) - 1);
            for (int t = 0; t < GROUP_SV; ++t) {
                const int j = g * GROUP_SV + t;
                double tt = 0.0, qq = 0.0;
                if (delta > 0.0) {
                    tt = (r[t] - lo) / delta;
                    qq = floor(tt + 0.5);
                    if (qq < 0.0) qq = 0.0;
                    if (qq > (double)((1 << V) - 1)) qq = (double)((1 << V) - 1);
                }
                if (q) q[(size_t)o * S + j] = (uint8_t)qq;
                if (t_out) t_out[(size_t)o * S + j] = tt;
                const double rh = lo + qq * delta;
                const uint8_t s = signs[(size_t)o * S + j];
                const double* c = cb + (size_t)idx[(size_t)o * S + j] * SV;
                for (int i = 0; i < SV; ++i)
                    W[(size_t)o * d_in + (size_t)j * SV + i] = (((s >> i) & 1) ? -rh : rh) * c[i];
            }
        }
    }
    free(cb);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Adaptive bit splitting (Sec. 3.3, Eqs. 7-9).                        */
/* ------------------------------------------------------------------ */

/* Eq. 8: the energy-weighted relative reconstruction error of one encoded
 * matrix in ORIGINAL channel order,
 *   E = sum_c e_c ||W_:,c - W^_:,c||^2 / sum_c e_c ||W_:,c||^2,
 * with W^ rebuilt from the fields (oracle_dequant, storage column order:
 * storage column p holds original channel perm[p]; perm null = identity).
 * W: [d_out][d_in] fp64, original column order; energy: [d_in].  Returns -1
 * for an unsupported shape or a zero denominator. */
double oracle_abs_error(int d_out, int d_in, int log2K, const uint8_t* signs, const uint16_t* idx,
                        const uint8_t* q, const uint16_t* mu, const uint16_t* delta, const uint16_t* codebook,
                        const int32_t* perm, const double* W, const double* energy) {
    if (d_out < 1 || d_in < 128 || d_in % 128 || log2K < 4 || log2K > 8) return -1.0;
    double* Wh = (double*)malloc(sizeof(double) * (size_t)d_out * d_in);
    if (!Wh) return -1.0;
    oracle_dequant(d_out, d_in, log2K, signs, idx, q, mu, delta, codebook, Wh);
    double num = 0.0, den = 0.0;
    for (int o = 0; o < d_out; ++o)
        for (int p = 0; p < d_in; ++p) {
            const int c = perm ? perm[p] : p;
            const double w = W[(size_t)o * d_in + c], d = w - Wh[(size_t)o * d_in + p];
            num += energy[c] * d * d;
            den += energy[c] * w * w;
        }
    free(Wh);
    return den > 0.0 ? num / den : -1.0;
}
