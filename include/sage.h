/*
 * sage.h -- C ABI of libsage, a B200 (sm_100a) implementation of the SAGE
 * packed linear layer y = W_hat x computed straight from 2.25-bit codes.
 *
 * Method: "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World
 * Usability" (Yan et al.).  Each row of W is cut into subvectors of v = 8
 * input channels (in ESG-permuted order); a subvector is rebuilt as
 *     w_hat = r_hat * (s (.) c_z),   r_hat = mu_g + q * delta_g      (Sec. 3.1, Eq. 1-2)
 * with s the 8 stored signs, c_z one of K nonnegative unit fp16 codewords of a
 * per-matrix codebook, and (mu_g, delta_g) an fp16 radius grid shared by the
 * 16 consecutive subvectors (G = 128 weights) of a row group (App. A.6,
 * Eq. 14).  A subvector costs v + log2 K + V = 18 bits (Eq. 3) for every
 * split (K, V) with log2 K + V = 10 (Sec. 3.3); the layout below keeps the
 * paper's "16-bit main word plus two auxiliary bits" per subvector (Sec. 3.5).
 *
 * Conventions
 *  - Every function returns a sage_status (int).  Argument errors are detected
 *    on the host before anything is enqueued; no compute call enqueues work
 *    after returning an error.
 *  - Device pointers are allocated and owned by the caller.  The library never
 *    allocates device memory and never synchronises the host with the device in
 *    compute calls; work is enqueued on the caller's stream.
 *  - fp16 values cross the ABI as uint16_t bit patterns (IEEE binary16).
 *  - Compute calls take a caller-allocated device workspace of at least
 *    sage_workspace_size() bytes, zero-filled once before first use (cudaMemset).
 *    Its first 256 bytes hold a device status word; the library restores every
 *    other byte it uses to its initial state, so the workspace may be reused
 *    across calls on one stream.  Calls that share a workspace must not overlap
 *    on the device.
 *  - Device pointers must be 16-byte aligned (SAGE_ERR_MISALIGNED otherwise).
 *
 * ------------------------------------------------------------------------
 * Packed format v2 (this library's layout; the paper gives only the widths)
 * ------------------------------------------------------------------------
 *  d_in % 128 == 0, 4 <= log2K <= 8, V = 10 - log2K, K = 2^log2K.
 *  Subvector column j = 0 .. S-1 (S = d_in/8) covers storage columns
 *  8j .. 8j+7; group g = j / 16 (G = d_in/128 groups).  R8 = ceil(d_out/8)
 *  row octets; octet b holds rows 8b .. 8b+7 (rows >= d_out are padding and
 *  must be zero).  Octets form blocks of 32 (256 rows); block B holds
 *  n_B = min(32, R8 - 32B) octets and is stored contiguously, so one block's
 *  columns [ja, jb) are one contiguous range of both planes.
 *
 *  main plane (uint32 words): the 16-byte record of (column j, local octet o
 *    of block B) is words B*S*128 + (j*n_B + o)*4 .. +3.  Word u holds row
 *    A = 8(32B + o) + 2u and row B = row A + 1:
 *      z_A  bits [7, 7 + log2K)        q_A  bits [23 - V, 23)
 *      z_B  bits [23, 23 + log2K)      q_B  bits [7 - V, 7)
 *      six sign slots at the ascending bit positions p_0 < ... < p_5 of
 *      {0 .. 6 - V} U {17 - V .. 15}; slot k owns bits p_k and p_k + 16.
 *      Slots 0..2 hold row A's component pairs 0..2, slots 3..5 row B's;
 *      pair n is components (2n, 2n + 1): bit p_k = sign of component 2n,
 *      bit p_k + 16 = sign of component 2n + 1 (1 = negative).
 *  meta plane: 8-byte entries; entry (group g, local octet o of block B,
 *    row t of the octet) is entry B*G*256 + (g*n_B + o)*8 + t =
 *    { uint32_t aux; uint16_t mu; uint16_t delta; } (little endian):
 *      aux bit t' = sign of component 6 of subvector 16g + t',
 *      aux bit t' + 16 = sign of component 7 of that subvector (t' = 0..15);
 *      mu, delta = fp16 grid of (row, group).
 *  Per 128 weights: 32 B main + 8 B meta = 2.50 bits per weight (Eq. 15).
 *  codebook: fp16 codebook[K][8] (16 bytes per codeword).
 *  perm: int32_t perm[d_in], storage column p holds original input channel
 *    perm[p]; the layer computes y = W_hat * x_perm with x_perm[p] = x[perm[p]]
 *    (Sec. 3.2 Eq. 5 and Sec. 3.5).  NULL means the identity.  The entries
 *    must be a permutation of 0 .. d_in - 1; device arrays are not read on
 *    the host, so this is not checked (an entry out of range reads outside
 *    the row of x).
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SAGE_FORMAT_VERSION 2

typedef struct CUstream_st* sage_stream_t; /* same type as cudaStream_t */

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad enum */
    SAGE_ERR_UNSUPPORTED = 2,      /* shape / split / batch outside what is implemented */
    SAGE_ERR_MISALIGNED = 3,       /* a device pointer is not 16-byte aligned */
    SAGE_ERR_WORKSPACE = 4,        /* workspace missing or smaller than sage_workspace_size() */
    SAGE_ERR_CUDA = 5,             /* a CUDA runtime call failed (launch or query) */
    SAGE_ERR_TIMEOUT = 6           /* a device-side bounded wait gave up (see sage_query_status) */
} sage_status;

/* One packed matrix (all pointers are device pointers; perm may be NULL). */
typedef struct {
    int32_t d_out, d_in, log2K;
    const uint32_t* main;      /* main plane, sage_packed_sizes() bytes */
    const uint32_t* meta;      /* meta plane */
    const uint16_t* codebook;  /* fp16 [K][8] */
    const int32_t* perm;       /* [d_in] or NULL */
} sage_matrix;

/* Operation selector for sage_workspace_size(). */
enum { SAGE_OP_GEMV = 0, SAGE_OP_GEMM = 1, SAGE_OP_MOE = 2, SAGE_OP_GROUPED = 3, SAGE_OP_ABS = 4 };

/* Human-readable name of a status code (static storage). */
const char* sage_status_string(int status);

/* Library build string and format version. */
const char* sage_version(void);

/* Bytes of the main and meta planes of a d_out x d_in matrix (format v2).
 * Errors: INVALID_ARGUMENT (null outputs, d_out < 1), UNSUPPORTED (d_in % 128,
 * log2K outside 4..8). */
int sage_packed_sizes(int d_out, int d_in, int log2K, size_t* main_bytes, size_t* meta_bytes);

/* HOST.  Packs logical fields into the v2 planes (host buffers).
 * signs/idx/q: [d_out][d_in/8] row-major, storage column order (Sec. 3.1:
 *   bit i of signs = 1 when component i is negative; idx < K; q < 2^V);
 * mu/delta: fp16 bits [d_out][d_in/128].  main_out/meta_out: sage_packed_sizes
 * bytes, fully written (padding rows zero).  Errors: INVALID_ARGUMENT (null,
 * idx or q out of range), UNSUPPORTED (shape/split). */
int sage_pack(int d_out, int d_in, int log2K,
              const uint8_t* signs, const uint16_t* idx, const uint8_t* q,
              const uint16_t* mu, const uint16_t* delta,
              uint32_t* main_out, uint32_t* meta_out);

/* HOST.  Inverse of sage_pack (same shapes). */
int sage_unpack(int d_out, int d_in, int log2K,
                const uint32_t* main_plane, const uint32_t* meta_plane,
                uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu, uint16_t* delta);

/* HOST.  ESG permutation (Sec. 3.2, Eq. 5): channels sorted by decreasing
 * energy (ties: lower channel first) into 8 tiers of d_in/8; storage position
 * 8j + t takes the j-th channel of tier t.  perm_out: [d_in].
 * Errors: INVALID_ARGUMENT (null), UNSUPPORTED (d_in % 8). */
int sage_esg_permutation(int d_in, const double* energy, int32_t* perm_out);

/* HOST.  Per-matrix SAGE initialisation (Algorithm 1's per-matrix half, App.
 * A.7, for one fixed (K, V)): ESG permutation (Eq. 5), activation weights
 * (Eq. 4, exponent gamma), weighted spherical k-means over the listed sample
 * subvectors (Sec. 3.2; `iters` iterations, codewords initialised to the
 * directions of sample[init[k]]), fp16 codebook, Eq. 6 assignment of every
 * subvector, fp16 grid per group (Eq. 14) and radius codes (Eq. 2).
 * W: fp64 [d_out][d_in] original channel order; energy: [d_in];
 * sample: subvector ids o*(d_in/8)+j (n_samples); init: K positions into
 * sample.  Outputs as in sage_pack plus perm_out [d_in] and codebook_out
 * (fp16 [K][8]).  n_threads <= 0 uses all hardware threads.
 * Errors: INVALID_ARGUMENT, UNSUPPORTED. */
int sage_encode(int d_out, int d_in, int log2K, const double* W, const double* energy, double gamma,
                int n_samples, const int64_t* sample, const int64_t* init, int iters, int n_threads,
                int32_t* perm_out, uint16_t* codebook_out,
                uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu, uint16_t* delta);

/* HOST.  The inputs of the GPU encoder (sage_kmeans, sage_encode_rows) for
 * one matrix, as sage_encode computes them before its k-means: the ESG
 * permutation (as sage_esg_permutation), the Eq. 4 weight of every storage
 * column (omega_out [d_in], exponent gamma; the weights of subvector column j
 * are omega_out[8j .. 8j + 7]) and, for the listed sample subvectors
 * (ids o*(d_in/8)+j), their magnitudes |W| in storage column order and their
 * weights (P_out, Wt_out: fp64 [n_samples][8]).
 * Errors: INVALID_ARGUMENT (null, sizes, sample ids), UNSUPPORTED (d_in % 128). */
int sage_encode_inputs(int d_out, int d_in, const double* W, const double* energy, double gamma,
                       int n_samples, const int64_t* sample, int32_t* perm_out, double* omega_out,
                       double* P_out, double* Wt_out);

/* Device workspace bytes for one call of `op` over the n matrices `mats`
 * (host array: the single matrix of sage_gemv / sage_gemm, all matrices of a
 * sage_gemv_grouped call, or all experts of a sage_moe_gemv call) at batch M
 * (for SAGE_OP_MOE: the pair count).  Always >= 256.
 * Errors: INVALID_ARGUMENT. */
int sage_workspace_size(int op, const sage_matrix* mats, int n, int M, size_t* bytes);

/* y[M][d_out] = W_hat x_perm for M in 1..8 (Sec. 3.5 decode GEMV; App. A.1):
 * x: fp16 [M][d_in] original channel order (device); y: fp16 [M][d_out].
 * fp32 accumulation; deterministic (identical bits on every run).
 * Errors: INVALID_ARGUMENT, UNSUPPORTED (M outside 1..8), MISALIGNED,
 * WORKSPACE, CUDA. */
int sage_gemv(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y,
              void* ws, size_t ws_bytes, sage_stream_t stream);

/* sage_gemv without a workspace argument.  The SAGE paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory or
 * hand the library a workspace at the point of the call (allocator-free
 * plugins, custom ops whose framework owns all device memory).  It allocates
 * nothing: its scratch is a 4 MiB array compiled into libsage (one per device,
 * resident while the library's device code is loaded), and it runs the same
 * kernel with the same numerics as sage_gemv (identical y bits).
 *   - Limit: the scratch of the call, as sage_workspace_size(SAGE_OP_GEMV, ...)
 *     would report it, must fit in 4 MiB.  About 2.4 MiB go to split-K partial
 *     sums on a 148-SM GPU; the rest holds one 4-byte counter per 256 output
 *     rows, so any d_out up to about 400,000 rows fits.  Larger shapes return
 *     SAGE_ERR_WORKSPACE before anything is launched.
 *   - The first call in each CUDA context (per device, and again after the
 *     context is replaced, e.g. by cudaDeviceReset) looks up the array's
 *     device address in that context; make that first call outside any CUDA
 *     stream capture.
 *   - Calls on one device share the scratch: they must not overlap.  Two calls
 *     in flight at once (different streams, or different host threads without
 *     ordering) race on it and give wrong results.
 *   - The status word and counters in the scratch start at zero and every
 *     completed call leaves them at zero.  A bounded device wait that gives up
 *     (SAGE_ERR_TIMEOUT under sage_gemv; only a GPU stalled for seconds causes
 *     one) is not reported by this entry point, and it may leave split-K
 *     counters non-zero, after which later calls in the same context compute
 *     wrong sums until the context is replaced.  Use sage_gemv with a
 *     workspace where that report, or recovery by zeroing the workspace,
 *     is needed.
 * Errors: as sage_gemv, with WORKSPACE meaning "shape beyond the 4 MiB
 * scratch". */
int sage_gemv_static(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y, sage_stream_t stream);

/* One launch over n matrices (host array `mats`), each with its own input
 * xs[i] ([M][d_in_i]) and output ys[i] ([M][d_out_i]), M in 1..8 -- e.g. the
 * q|k|v or gate|up projections of a decoder layer.  Same numerics as
 * sage_gemv.  n <= 64.  Errors: as sage_gemv. */
int sage_gemv_grouped(const sage_matrix* mats, int n, const uint16_t* const* xs, uint16_t* const* ys,
                      int M, void* ws, size_t ws_bytes, sage_stream_t stream);

/* y = W_hat x_perm for any M >= 1 (Sec. 3.5 prefill GEMM; App. A.1):
 * M <= 8 runs the GEMV kernel; M >= 9 permutes x once and runs the
 * tcgen05/TMEM tensor-core kernel (fp16 operands, fp32 accumulation).
 * Errors: as sage_gemv (UNSUPPORTED for M > 256). */
int sage_gemm(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y,
              void* ws, size_t ws_bytes, sage_stream_t stream);

/* Grouped-expert GEMV for a mixture-of-experts layer: for every pair p,
 * y[p] = W_hat_{pair_expert[p]} x_perm[pair_xrow[p]].  experts: host array of
 * n_experts matrices sharing d_out and d_in (each with its own split,
 * codebook and perm); pair_expert / pair_xrow: device int32 [n_pairs];
 * x: fp16 [rows][d_in]; y: fp16 [n_pairs][d_out].  The pairs of one expert
 * are grouped (on the device, in pair order) into virtual matrices of at most
 * 8 pairs, and each virtual matrix reads the expert's planes once: an expert
 * with up to 8 pairs is read once per call.  pair_xrow entries must be rows
 * of x (not checked on the host).  Errors: as sage_gemv, plus UNSUPPORTED
 * for n_experts > 256 or n_pairs > 4096 and for experts that differ in d_out
 * or d_in; a pair_expert entry outside [0, n_experts) sets
 * SAGE_ERR_UNSUPPORTED in the status word and that pair's output is not
 * written. */
int sage_moe_gemv(const sage_matrix* experts, int n_experts,
                  const int32_t* pair_expert, const int32_t* pair_xrow, int n_pairs,
                  const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes, sage_stream_t stream);

/* Router-weighted combine of a mixture-of-experts projection (the step after
 * the down projection of a top-k routed MLP): for every token t,
 *   y[t][c] = fp16( sum_k weights[t][k] * y_pairs[t * topk + k][c] ),
 * summed in fp32 in slot order (k = 0, 1, ...).  y_pairs: device fp16
 * [T * topk][d_out] (pair p = t * topk + k, the layout sage_moe_gemv writes for
 * pairs listed token by token); weights: device fp32 [T][topk]; y: device fp16
 * [T][d_out] (output).  Launched with programmatic dependent launch: it may
 * start while the preceding kernel on `stream` drains and waits for it before
 * reading.  Errors: INVALID_ARGUMENT (null, T/topk/d_out < 1), UNSUPPORTED
 * (d_out % 8), MISALIGNED (y_pairs or y not 16-byte aligned, weights not
 * 4-byte aligned), CUDA. */
int sage_moe_combine(int T, int topk, int d_out, const uint16_t* y_pairs, const float* weights, uint16_t* y,
                     sage_stream_t stream);

/* ------------------------------------------------------------------------
 * Fused decoder layer.  The packed projections of one transformer decoder
 * layer run as ONE launch of four dependent stages, with the operations
 * between them fused into the activation gather of the next stage (Sec. 3.5:
 * the ESG permutation is fused with the preceding normalisation or
 * activation) and into the output writes:
 *   x1  = fp16(h * attn_norm / sqrt(mean(h^2) + eps))             RMSNorm
 *   q, k, v = W_q x1, W_k x1, W_v x1                             stage 1
 *   a   = attention over the single cached position: query head i reads the
 *         value row of key/value head i / (n_heads / n_kv_heads)
 *   o   = W_o a                                                   stage 2
 *   r   = fp16(h + o);  x3 = fp16(r * mlp_norm / sqrt(mean(r^2) + eps))
 *   gate, up = W_gate x3, W_up x3                                stage 3
 *   m   = fp16(silu(gate) * up),  silu(t) = t / (1 + e^-t)
 *   down = W_down m;   h_out = fp16(r + down)                    stage 4
 * A stage starts decoding as soon as the stage it reads is complete on the
 * whole device (a completion count in the workspace), not at a kernel
 * boundary; the packed planes of later stages stream in meanwhile.  Every
 * projection has the numerics of sage_gemv.  The attention is the first
 * position of a sequence, which needs no key/value cache and no rotary
 * embedding; the rest of a longer sequence's attention is outside libsage.
 * ------------------------------------------------------------------------ */
typedef struct {
    sage_matrix q, k, v, o, gate, up, down;   /* packed projections */
    const uint16_t* attn_norm;   /* fp16 [hidden] RMSNorm weight before q|k|v (device) */
    const uint16_t* mlp_norm;    /* fp16 [hidden] RMSNorm weight before gate|up (device) */
    int32_t n_heads, n_kv_heads, head_dim;
    float eps;
} sage_decoder_layer;

typedef struct {   /* device outputs, fp16 [M][...] (all written) */
    uint16_t *q, *k, *v, *o, *gate, *up, *down, *h_out;
} sage_decoder_outputs;

/* Workspace bytes of sage_decoder_layer_forward (zero-filled once before first
 * use, as for the other compute calls).  Errors: INVALID_ARGUMENT, UNSUPPORTED
 * (shapes that do not form a decoder layer, see sage_decoder_layer_forward). */
int sage_decoder_layer_workspace_size(const sage_decoder_layer* L, int M, size_t* bytes);

/* One decoder layer at batch M (1..8) on input rows h (fp16 [M][hidden], device).
 * Shapes: hidden = d_in of q, k, v, gate, up = d_out of o and down;
 * q.d_out = o.d_in = n_heads * head_dim; k.d_out = v.d_out = n_kv_heads *
 * head_dim (n_heads a multiple of n_kv_heads); gate.d_out = up.d_out =
 * down.d_in.  Errors: INVALID_ARGUMENT (null pointer, eps < 0), UNSUPPORTED
 * (shapes, M), MISALIGNED, WORKSPACE, CUDA; device-side timeouts as for
 * sage_gemv (sage_query_status). */
int sage_decoder_layer_forward(const sage_decoder_layer* L, const uint16_t* h, int M,
                               const sage_decoder_outputs* out, void* ws, size_t ws_bytes, sage_stream_t stream);

/* ------------------------------------------------------------------------
 * The encoder's per-row stage on the GPU (Sec. 3.1-3.2): for a given stored
 * codebook, every subvector's signs, its Eq. 6 direction
 *   z = argmax_k (sum_i w_i p_i c_ki)^2 / sum_i w_i c_ki^2,  p = |W subvector|,
 * (ties to the smallest k; an all-zero score gives z = 0, r* = 0) with fitted
 * radius r* = sum w p c / sum w c^2, the Eq. 14 grid of every row group of 16
 * (mu = min r*, delta = (max r* - min r*) / (2^V - 1), both rounded to fp16,
 * nearest even) and the Eq. 2 codes q = clamp(floor((r* - mu) / delta + 0.5),
 * 0, 2^V - 1) against the stored grid (delta = 0: q = 0).  fp64 with every
 * product, sum and quotient rounded separately, in the CPU encoder's order:
 * the fields equal sage_encode's bit for bit for the same codebook,
 * permutation and weights.
 *   W: device fp64 [d_out][d_in], original column order;
 *   perm: device int32 [d_in] (storage column p holds original channel
 *     perm[p], e.g. sage_esg_permutation's);
 *   omega: device fp64 [d_in], the Eq. 4 weight of each storage column
 *     (omega of subvector group j over storage columns 8j .. 8j + 7);
 *   codebook: device fp16 [K][8], K = 2^log2K (the stored codebook);
 *   signs, idx, q: device u8 / u16 / u8 [d_out][d_in/8]; mu, delta: device
 *     fp16 [d_out][d_in/128] (outputs).
 * The codebook itself comes from sage_kmeans (GPU) or sage_encode (CPU).
 * Errors: INVALID_ARGUMENT (null), UNSUPPORTED (d_in % 128, log2K outside
 * 4..8), CUDA. */
int sage_encode_rows(int d_out, int d_in, int log2K, const double* W, const int32_t* perm, const double* omega,
                     const uint16_t* codebook, uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu,
                     uint16_t* delta, sage_stream_t stream);

/* ------------------------------------------------------------------------
 * The packer on the device: the same planes as sage_pack (format v2), word
 * for word, from device fields, so that an encoding made on the GPU is
 * packed without a round trip through the host.  Shapes and field layouts as
 * sage_pack; main_out / meta_out: device buffers of sage_packed_sizes()
 * bytes, every word written.  Unlike sage_pack, which rejects them, field
 * values wider than their bits (idx >= K, q >= 2^V) are masked to their
 * widths.  Asynchronous on `stream`.  Errors: INVALID_ARGUMENT (null),
 * UNSUPPORTED (d_in % 128, log2K outside 4..8), MISALIGNED (main_out not
 * 4-byte or meta_out not 8-byte aligned), CUDA. */
int sage_pack_device(int d_out, int d_in, int log2K, const uint8_t* signs, const uint16_t* idx, const uint8_t* q,
                     const uint16_t* mu, const uint16_t* delta, uint32_t* main_out, uint32_t* meta_out,
                     sage_stream_t stream);

/* ------------------------------------------------------------------------
 * The encoder's weighted spherical k-means on the GPU (Sec. 3.2 "Weighted
 * Quantizer Fitting"; Sec. 4.1 sets 65,536 sampled subvectors): K = 2^log2K
 * unit codewords start as the unit directions of the samples init[0..K)
 * (an all-zero sample gives the direction 1/sqrt(8) in every component);
 * each of `iters` rounds assigns every sample by Eq. 6 (as sage_encode_rows,
 * against the fp64 codewords) and moves each codeword to the normalised sum
 * of its members' w * p / |p| (members in sample order; all-zero samples add
 * nothing; an empty cluster keeps its codeword).  fp64 with every operation
 * rounded separately, in the CPU encoder's order: the codebook equals
 * sage_encode's k-means bit for bit on the same samples.
 *   P, Wt: device fp64 [n][8]: the sampled subvectors' magnitudes |W| in
 *     storage column order and their Eq. 4 weights;
 *   init: device int64 [K], positions into the n samples;
 *   cb: device fp64 [K][8] (output); cb16: device fp16 [K][8], the codebook
 *     rounded to nearest even (output; may be null);
 *   ws: device memory of sage_kmeans_workspace_size(n) bytes, 16-byte aligned,
 *     zero-filled once before first use (word 0 is its status word), owned by
 *     the caller, not shared with a concurrent call.
 * Asynchronous on `stream`.  Errors: INVALID_ARGUMENT (null pointer),
 * UNSUPPORTED (n outside 1..2^30, iters < 0, log2K outside 4..8), MISALIGNED, WORKSPACE,
 * CUDA; an init entry outside [0, n) is found on the device (sample 0 is read
 * in its place, the codebook is then meaningless) and sage_query_status(ws)
 * returns INVALID_ARGUMENT for it. */
size_t sage_kmeans_workspace_size(int n);  /* 0 for n outside 1..2^30 */
int sage_kmeans(int n, int log2K, const double* P, const double* Wt, const int64_t* init, int iters, double* cb,
                uint16_t* cb16, void* ws, size_t ws_bytes, sage_stream_t stream);

/* ------------------------------------------------------------------------
 * Adaptive bit splitting (Sec. 3.3, Eqs. 7-9).  Each matrix chooses its
 * (K, V) split among the 18-bit candidates by the energy-weighted relative
 * reconstruction error in ORIGINAL channel order (Eq. 8),
 *   E = sum_c e_c ||W_:,c - W^_:,c||^2 / sum_c e_c ||W_:,c||^2,
 * where W^ is rebuilt from the packed codes (storage column p holds original
 * channel perm[p]; no perm = identity) with r^ = mu + q delta in fp32 and the
 * signed fp16 codeword, and sums are in fp64.
 *   sage_abs_error: E of packed matrix A against W (device fp32
 *     [d_out][d_in], original column order, 16-byte aligned) with channel
 *     energies `energy` (device fp32 [d_in]); *err is a HOST double.
 *     Synchronous: it waits for the stream and adds the CTAs' partial sums on
 *     the host in a fixed order (deterministic).  ws: device workspace of
 *     sage_workspace_size(SAGE_OP_ABS, mats, n, ...) bytes: partial sums for
 *     n candidates (n = 1 suffices for every call; sized for all of a
 *     sage_abs_select's candidates, that call scores them all before one
 *     synchronisation, otherwise as many per synchronisation as fit).
 *   sage_abs_select: Eq. 9, the index of the candidate encoding with the
 *     smallest E (ties: the earlier candidate); cands: host array of n packed
 *     encodings of the same W (one per split); errs: host double [n] or null.
 * The encodings come from sage_encode (CPU) or, on the GPU, from
 * sage_kmeans + sage_encode_rows + sage_pack_device, one per split.
 * Errors: INVALID_ARGUMENT (null pointers, zero-energy W), UNSUPPORTED
 * (candidates of different shapes), MISALIGNED, WORKSPACE, CUDA. */
int sage_abs_error(const sage_matrix* A, const float* W, const float* energy, void* ws, size_t ws_bytes,
                   double* err, sage_stream_t stream);
int sage_abs_select(const sage_matrix* cands, int n, const float* W, const float* energy, void* ws,
                    size_t ws_bytes, int* best, double* errs, sage_stream_t stream);

/* ------------------------------------------------------------------------
 * Continuous-parameter decode for blockwise optimisation: the forward pass
 * of Sec. 3.4 and App. A.6.  Blockwise training keeps the discrete
 * assignments (signs, codeword indices) and trains the codebook and the
 * radii as continuous parameters:
 *   - codeword k from 7 hyperspherical angles (Eq. 12):
 *       c_1 = cos t_1, c_j = sin t_1 ... sin t_(j-1) cos t_j (j = 2..7),
 *       c_8 = sin t_1 ... sin t_7, with t_i = eps + (pi/2 - 2 eps) *
 *       sigmoid(alpha_ki), eps = 1e-4 (Eq. 13): unit and positive;
 *   - radius r~ = softplus(rho);
 *   - per row group of 16 subvectors the grid is recomputed from the current
 *     radii, mu = min r~, delta = (max r~ - min r~) / (2^V - 1) (Eq. 14),
 *     q = clamp(floor((r~ - mu) / delta + 0.5), 0, 2^V - 1) (Eq. 2; delta = 0
 *     gives q = 0: a group of equal radii reconstructs their common value);
 *   - W[o][8j + i] = (mu + q delta) s_i c_{z,i} (Eq. 1), storage column order.
 * The straight-through estimator of the backward pass is the caller's: this is
 * the forward only.  fp32 arithmetic throughout (the pages fix no precision
 * for training).
 *   alpha: device fp32 [K][7], K = 2^log2K (V = 10 - log2K);
 *   rho: device fp32 [d_out][d_in/8]; signs: device u8 [d_out][d_in/8] (bit
 *   i: component i negative); idx: device u16 [d_out][d_in/8];
 *   W: device fp32 [d_out][d_in], 16-byte aligned (output);
 *   q: device u8 [d_out][d_in/8] radius codes, or null;
 *   codebook: device fp32 [K][8] unit codewords, or null.
 * Errors: INVALID_ARGUMENT (null alpha, rho, signs, idx or W), UNSUPPORTED
 * (d_in % 128, log2K outside 4..8), MISALIGNED (W), CUDA. */
int sage_qdq_forward(int d_out, int d_in, int log2K, const float* alpha, const float* rho,
                     const uint8_t* signs, const uint16_t* idx, float* W, uint8_t* q, float* codebook,
                     sage_stream_t stream);

/* Test hook: fp16 reconstruction W[d_out][d_in] (storage column order),
 * computed by the same device decode as the kernels (Eq. 1-2). */
int sage_dequant(const sage_matrix* A, uint16_t* W, sage_stream_t stream);

/* Test hook: device unpack of the logical fields (shapes as sage_pack). */
int sage_unpack_device(const sage_matrix* A, uint8_t* signs, uint16_t* idx, uint8_t* q,
                       uint16_t* mu, uint16_t* delta, sage_stream_t stream);

/* x_perm[m][p] = x[m][perm[p]] (fp16, device), the prefill reorder of Sec. 3.5. */
int sage_permute_x(const uint16_t* x, const int32_t* perm, int M, int d_in, uint16_t* x_perm,
                   sage_stream_t stream);

/* Synchronises `stream`, reads and clears the workspace status word.
 * Returns SAGE_OK, SAGE_ERR_TIMEOUT (a bounded device wait gave up),
 * SAGE_ERR_INVALID_ARGUMENT (an input value found invalid on the device, e.g.
 * a sage_kmeans init entry), SAGE_ERR_UNSUPPORTED (a device-side limit was
 * exceeded) or SAGE_ERR_CUDA. */
int sage_query_status(void* ws, sage_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_H_ */
