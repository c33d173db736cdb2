/*
 * jolt.h -- C ABI of the B200 JoLT KV-cache compressor.
 *
 * JoLT ("A JoLT for the KV Cache: Near-Lossless KV Cache Compression via
 * Joint Rank-bit Allocation", Krishnan & Schulz) compresses the prefill KV
 * cache of every layer group, for keys and values separately (a "cell" is one
 * (sequence, group, K|V) tensor X of shape [L_g, H, T, D]), with
 *   1. a partial Tucker decomposition that truncates only the token and the
 *      feature modes (Section 3, "Partial Tucker backbone"),
 *   2. a randomly rotated low-bit residual (Section 3, "Rotated low-bit
 *      residual"),
 *   3. per-cell ranks and bit-widths chosen jointly for all cells by one
 *      Lagrange multiplier under a single byte budget (Section 3, Eqs. 1-4),
 *   4. optionally a randomized token-mode SVD (Section 3.1, "FlashJoLT",
 *      Eq. 5 for the rank cap).
 * It also provides the data-driven layer grouping that precedes compression
 * (Section 3; jolt_layer_groups) and, as an option, the page's own
 * QR-Gaussian residual rotation (jolt_options.rotation).
 *
 * Conventions for every entry point:
 *   * Device pointers are CUDA device (or managed) memory of the current
 *     device; host pointers are ordinary host memory. Each argument says which.
 *   * Every call returns a jolt_status; none aborts or exits. On failure
 *     jolt_last_error() gives a thread-local message.
 *   * Work is enqueued on the given stream and is asynchronous unless the
 *     entry point says it synchronises.
 *   * The library never writes its input caches.
 *   * Device memory the library needs (handles, workspace) comes from the
 *     allocator set by jolt_set_allocator (default: cudaMallocAsync /
 *     cudaFreeAsync on the call's stream).
 */
#ifndef JOLT_H
#define JOLT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JOLT_API __attribute__((visibility("default")))
#else
#define JOLT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* jolt_stream_t;   /* == cudaStream_t */

typedef enum {
  JOLT_OK = 0,
  JOLT_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, bad grid value  */
  JOLT_ERR_UNSUPPORTED_SHAPE = 2,  /* D not 64/128, stride not aligned, ...    */
  JOLT_ERR_BUDGET_INFEASIBLE = 3,  /* budget below the cheapest allocation     */
  JOLT_ERR_OOM = 4,                /* the allocator returned NULL              */
  JOLT_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed        */
  JOLT_ERR_TIMEOUT = 6,            /* a bounded device wait expired            */
  JOLT_ERR_NONFINITE = 7           /* a cell's squared norm is not finite      */
} jolt_status;

enum { JOLT_BF16 = 0, JOLT_F32 = 1 };             /* jolt_layout.dtype        */
enum { JOLT_EXACT = 0, JOLT_RANDOMIZED = 1 };      /* jolt_options.mode        */
enum { JOLT_ROT_HADAMARD = 0, JOLT_ROT_QR_GAUSS = 1 }; /* jolt_options.rotation */
enum { JOLT_MIN_ENUMERATE = 0, JOLT_MIN_GREEDY = 1 }; /* jolt_options.minimizer */

/*
 * Where the cache lives. Element (b, l, h, t, d) of K (and of V, same layout)
 * is at base + b*stride_b + l*stride_l + h*stride_h + t*stride_t + d, strides
 * in ELEMENTS, d contiguous. Layers [group_start[g], group_start[g+1]) form
 * group g (contiguous groups, Section 3: "partition the L layers into G
 * contiguous groups"). rope_theta_k > 0 means the keys were stored after a
 * rotate-half rotary embedding with that base over positions 0..T-1: keys are
 * compressed before RoPE and RoPE is re-applied on decompression (Section 3,
 * "Keys are decomposed before the rotary position embedding").
 */
typedef struct {
  int32_t batch, n_layers, n_heads, seq_len, head_dim;   /* head_dim in {64,128} */
  int32_t n_groups;
  const int32_t* group_start;    /* HOST, n_groups+1 entries, 0 .. n_layers    */
  int32_t dtype;                 /* JOLT_BF16 | JOLT_F32                       */
  int64_t stride_b, stride_l, stride_h, stride_t;
  float rope_theta_k;            /* 0: no RoPE handling                        */
} jolt_layout;

/*
 * Knobs. jolt_default_options() fills the paper's defaults:
 *   mode JOLT_EXACT; bits {0,2,4,8} (Section 3, "Rotated low-bit residual");
 *   rank grids = every integer from 1 (Section 3, "Solving the allocation");
 *   rt_max 0 (exact: min(T, N); randomized: q_cap of Eq. 5);
 *   oversample_p 8, power_iters 2 (randomized range finder);
 *   scale_group 0 (= D: one fp32 scale per row, Eq. 1's 32/d_h term);
 *   budget_tol 0.005 and max_iters 50 (Section 3: "stopping within 0.5% of
 *   the target budget or after 50 iterations");
 *   minimizer JOLT_MIN_ENUMERATE: the per-cell argmin of e + lambda s over
 *   every option. JOLT_MIN_GREEDY is the page's per-cell search ("Solving the
 *   allocation"): for each b, start at the smallest ranks and take whichever
 *   single grid step of r_T or r_d lowers the error most per added byte, while
 *   it lowers e + lambda s; keep the best b.
 *   rotation JOLT_ROT_HADAMARD: R = D^-1/2 H_D diag(s), s seeded per
 *   sequence (the fast path: the tensor-core stream kernels). JOLT_ROT_QR_GAUSS
 *   is the page's own rotation ("Rotated low-bit residual"): R = the Q of the
 *   QR factorization of a seeded D x D standard Gaussian (Philox4x32-10 +
 *   Box-Muller, one matrix per sequence, R's triangular factor with a
 *   positive diagonal), r = R e and e = R^T r summed in fp64 and rounded once
 *   to fp32. It runs on the row-per-thread kernels (a dense D x D product per
 *   row) and is much slower; the handle keeps the matrices (batch*D*D*8 bytes).
 * Grids are HOST arrays of strictly increasing values >= 1, copied at plan
 * time; NULL/0 means "every integer 1..max".
 */
typedef struct {
  int32_t mode;
  int32_t n_bits;
  int32_t bits[8];               /* each in {0,2,3,4,8}, strictly increasing   */
  int32_t n_rt;
  const int32_t* rt_grid;
  int32_t n_rd;
  const int32_t* rd_grid;
  int32_t rt_max;
  int32_t oversample_p, power_iters;
  int32_t scale_group;           /* 0 (= D), 32, 64 or 128; must divide D      */
  int32_t rotation;              /* JOLT_ROT_HADAMARD | JOLT_ROT_QR_GAUSS      */
  double budget_tol;
  int32_t max_iters;
  int32_t minimizer;             /* JOLT_MIN_ENUMERATE | JOLT_MIN_GREEDY       */
  /* Where this plan's cache sits in a larger one that several processes
   * compress under one budget (jolt_compress_begin): its sequence b and
   * group g are sequence seq_base + b and group group_base + g of the whole
   * cache. They only enter the random draws (the rotation of sequence s uses
   * seed + s; the sketch of group g uses group g's counter words) and the
   * identities in jolt_cell_info, so a shard draws exactly what a single
   * process would for the same cells. Default 0. */
  int32_t seq_base, group_base;
  /* The compression ratio C of Eq. (5) (q_cap = 32 or 64 by C <= 4, Section
   * 3.1). 0: this plan's dense bf16 bytes / byte_budget. A shard of a
   * shared-budget compression passes the whole cache's ratio. */
  double cap_ratio;
} jolt_options;

typedef struct jolt_plan_s jolt_plan_t;
typedef struct jolt_handle_s jolt_handle_t;

/* Per-cell result of an allocation (one entry per cell, cell order =
 * sequence, then group, then K before V). */
typedef struct {
  int32_t seq, group, kind;      /* kind 0 = K, 1 = V                          */
  int32_t r_t, r_d, bits;
  int64_t bytes;                 /* Eq. (1) for this cell                      */
  double err_model;              /* Eq. (2) surrogate at the chosen point      */
  double norm_sq;                /* ||X||_F^2 of the cell                      */
} jolt_cell_info;

/* Device views of one compressed cell (for tests and for consumers that
 * decode without this library). All pointers are DEVICE pointers owned by
 * the handle. */
typedef struct {
  int32_t r_t, r_d, bits, scale_group;
  int32_t L, H, T, D, t_pitch;
  const uint16_t* ut;   /* bf16 U_T^ transposed: [r_t][t_pitch], first T used */
  const uint16_t* ud;   /* bf16 U_d^: [D][r_d]                                */
  const uint16_t* core; /* bf16 G^: [L][H][r_t][r_d]                          */
  const uint8_t* codes; /* [L][H][T][bits*D/8], NULL when bits == 0           */
  const float* scales;  /* [L][H][T][D/scale_group], NULL when bits == 0      */
} jolt_cell_view;

JOLT_API void jolt_default_options(jolt_options* opt);

/* Checks layout, budget and options, derives the cells, the rank grids and
 * the Eq. (5) cap, and sizes the workspace. byte_budget B is the target of
 * Eq. (3) for ALL cells together. Synchronises the legacy default stream once
 * (ε² calibration, Section 3 text under Eq. 2). Returns
 * JOLT_ERR_BUDGET_INFEASIBLE when B is below the sum of every cell's cheapest
 * option, JOLT_ERR_UNSUPPORTED_SHAPE for D not in {64,128}, strides not
 * multiples of 8 elements or a mode/shape pair the kernels do not cover. */
JOLT_API jolt_status jolt_plan(const jolt_layout* layout, int64_t byte_budget,
                      const jolt_options* opt, jolt_plan_t** out);
JOLT_API void jolt_free_plan(jolt_plan_t* plan);

/* Compress K and V (DEVICE pointers, layout of the plan) under byte_budget
 * (<= 0: the plan's budget). seed selects the residual rotation and, in
 * randomized mode, the Gaussian sketch (sequence b uses seed + b). The handle
 * owns every compressed buffer. Asynchronous; the handle is usable by later
 * work on the same stream. */
JOLT_API jolt_status jolt_compress(jolt_plan_t* plan, const void* k, const void* v,
                          int64_t byte_budget, uint64_t seed,
                          jolt_stream_t stream, jolt_handle_t** out);

/* One byte budget shared by several processes (one per GPU), each holding
 * part of the cells (Section 3, "Solving the allocation": the allocation
 * separates across cells once the multiplier is fixed, so only per-cell
 * rate-distortion summaries need to travel). Protocol:
 *   1. every rank: jolt_compress_begin on its plan (its own sequences or
 *      layer groups, with seq_base / group_base set), which computes the
 *      spectra and the rate-distortion table of its cells (the steps before
 *      the allocation) and writes one summary record per cell into
 *      summary_dev (DEVICE, n_cells * jolt_summary_bytes(plan) bytes, 16-byte
 *      aligned, owned by the caller);
 *   2. the caller all-gathers the records of every rank into one DEVICE
 *      buffer (NCCL or any transport; the records are plain bytes);
 *   3. every rank: jolt_compress_end with the gathered buffer, which runs the
 *      same multiplier bisection over all n_total cells (deterministic, so
 *      every rank reaches the same allocation bit for bit) and then fits and
 *      encodes its own cells, records [first_cell, first_cell + n_cells).
 * Every rank must pass the same byte_budget and options (grids, bits, scale
 * group, tolerances); records carry a fingerprint of those settings and a
 * mismatch, or a local slice that holds other cells, is reported as
 * JOLT_ERR_INVALID_ARG by the next synchronising call on the handle.
 * Between begin and end the plan holds the cells' spectral state: run no
 * other jolt_compress / jolt_rd_table on that plan in between. The handle
 * from begin is the compressed cache once end has run; before that only
 * jolt_free_handle may be called on it. Both calls are asynchronous. */
JOLT_API int64_t jolt_summary_bytes(const jolt_plan_t* plan);
JOLT_API jolt_status jolt_compress_begin(jolt_plan_t* plan, const void* k, const void* v, int64_t byte_budget,
                                         uint64_t seed, void* summary_dev, jolt_stream_t stream,
                                         jolt_handle_t** out);
JOLT_API jolt_status jolt_compress_end(jolt_handle_t* h, const void* all_summaries_dev, int32_t n_total,
                                       int32_t first_cell, jolt_stream_t stream);

/* Decompress into k_out / v_out (DEVICE, bf16, layout out_layout; NULL means
 * the plan's layout with dtype bf16). Section 3: "Decoding inverts the
 * rotation and adds the dequantized residual to the low-rank reconstruction";
 * keys get RoPE re-applied. Asynchronous. */
JOLT_API jolt_status jolt_decompress(const jolt_handle_t* h, void* k_out, void* v_out,
                            const jolt_layout* out_layout, jolt_stream_t stream);

/* Fused decode attention over the compressed cache (Section 3.1, the decode
 * kernel that evaluates attention directly over the stored factors and the
 * packed residual): one decode step of layer `layer` for every sequence of
 * the handle. For sequence b and query head j (KV head j / G, G = n_q_heads /
 * n_heads <= 8):
 *   out[b][j] = sum_t softmax_t(q[b][j] . k_t / sqrt(D)) v_t,
 * over the T compressed tokens, whose keys and values are the fp32
 * reconstruction decompression would round to bf16 (keys with RoPE
 * re-applied), followed by n_tail dense tokens (tail_k / tail_v), with one
 * softmax over both. Keys are rebuilt tile by tile on chip; values stay in
 * rank space and the rotated residual domain until one final product per
 * query head.
 *   q: DEVICE fp32 [batch][n_q_heads][D], 16-byte aligned, already rotated
 *     for the decode position (RoPE) as the model's queries are.
 *   tail_k, tail_v: DEVICE bf16 [batch][n_heads][n_tail][D] (keys already
 *     rotated), NULL when n_tail == 0; n_tail <= 1024.
 *   out: DEVICE fp32 [batch][n_q_heads][D].
 * The handle must use the Hadamard rotation (JOLT_ERR_UNSUPPORTED_SHAPE for
 * JOLT_ROT_QR_GAUSS), and the value cells of the layer's group a token rank
 * r_T <= 512 (always so in randomized mode, where r_T <= q_cap <= 512;
 * JOLT_ERR_UNSUPPORTED_SHAPE otherwise). The first call on a handle reads the cells' layout to
 * the host (synchronises the handle's stream once); later calls are
 * asynchronous. Workspace comes from the library allocator. */
JOLT_API jolt_status jolt_decode_attention(const jolt_handle_t* h, int32_t layer, const float* q,
                                           int32_t n_q_heads, const uint16_t* tail_k, const uint16_t* tail_v,
                                           int32_t n_tail, float* out, jolt_stream_t stream);

/* Sum over cells of Eq. (1) at the chosen (r_T, r_d, b): the compressed size
 * in bytes. Synchronises the handle's stream. */
JOLT_API jolt_status jolt_bytes(const jolt_handle_t* h, int64_t* payload_bytes);

/* Per-cell allocation (n >= number of cells) and the multiplier lambda of
 * Eq. (4). HOST outputs. Synchronises the handle's stream. */
JOLT_API jolt_status jolt_handle_info(const jolt_handle_t* h, jolt_cell_info* cells,
                             int32_t n, double* lambda, int32_t* iterations);
JOLT_API jolt_status jolt_handle_cell(const jolt_handle_t* h, int32_t cell,
                             jolt_cell_view* view);
JOLT_API int32_t jolt_num_cells(const jolt_plan_t* plan);
JOLT_API void jolt_free_handle(jolt_handle_t* h);

/* Rate-distortion inputs of every cell (Section 3, Eq. 2: the unprojected
 * mode spectra and ||X||^2), computed on the device by the plan's mode.
 * HOST outputs: norm_sq[n_cells]; sig_t[n_cells * n_t] (descending squared
 * token singular values; in randomized mode the q_cap computed values
 * followed by the synthetic tail entry of Section 3.1); sig_d[n_cells * D].
 * n_t is written to *n_t (<= max_t). Synchronises the stream. */
JOLT_API jolt_status jolt_rd_table(jolt_plan_t* plan, const void* k, const void* v,
                          double* norm_sq, double* sig_t, int32_t max_t,
                          int32_t* n_t, double* sig_d, jolt_stream_t stream);

/* The allocator of Eqs. (3)-(4) alone, on the device, from HOST rate-distortion
 * inputs: for cell c, t_t[c*ld_t + r] (r = 0..n_t) and t_d[c*ld_d + r]
 * (r = 0..D) are the tail fractions (discarded energy / ||X||^2 at rank r),
 * eps2[n_bits] the calibration of Eq. (2). Uses the plan's grids, shapes and
 * bit list. HOST outputs: choice[3*c] = (r_t, r_d, bits), bytes[c], and
 * lambda. Synchronises the stream. */
JOLT_API jolt_status jolt_allocate(jolt_plan_t* plan, const double* t_t, int32_t ld_t,
                          const double* t_d, int32_t ld_d, const double* eps2,
                          int64_t byte_budget, int32_t* choice, int64_t* bytes,
                          double* lambda, int32_t* iterations,
                          jolt_stream_t stream);

/* ε²(b) calibration of Section 3 (text under Eq. 2): the fraction of a
 * Gaussian's energy the b-bit quantizer with groups of `group` values fails
 * to recover, over 2^20 Philox4x32-10 / Box-Muller samples rounded to fp32.
 * HOST output eps2[n]. Synchronises the stream. */
JOLT_API jolt_status jolt_eps2(const int32_t* bits, int32_t n, int32_t group,
                      double* eps2, jolt_stream_t stream);

/* jolt_eps2 without any device allocation, for callers that cannot allocate
 * GPU memory while they run (an engine that reserved HBM for its KV pool up
 * front and gives libraries no allocator, or a loop where an allocation is not
 * allowed). The paper has no counterpart to this entry point; it computes the
 * same values as jolt_eps2 with the same kernels.
 *   bits: HOST, n entries (1 <= n <= 8) from {0,2,3,4,8}; group: 32, 64 or 128.
 *   eps2_dev: DEVICE output of n doubles, owned by the caller.
 * Asynchronous on `stream`; the caller synchronises before reading eps2_dev.
 * Partial sums live in a static 9 KB device array that every GPU loading the
 * library holds until exit (limit: 128 partial blocks x 9 slots, i.e. up to 8
 * bit widths and any supported group). The first call in each CUDA context
 * (the primary context of each device, or any other context made current)
 * looks up that array's address there (cudaGetSymbolAddress, with that device
 * current) and caches it; make this first call before any stream capture. A
 * device reset unloads the array: after cudaDeviceReset, do not call this
 * entry point again in the same process. All calls share the array and it
 * keeps the last call's contents: calls whose work overlaps on the GPU race,
 * so issue them on one stream or order them. Arguments beyond the limits
 * return JOLT_ERR_INVALID_ARG with a message naming the limit. */
JOLT_API jolt_status jolt_eps2_noalloc(const int32_t* bits, int32_t n, int32_t group,
                                       double* eps2_dev, jolt_stream_t stream);

/* The residual stage alone (Section 3, "Rotated low-bit residual"), for
 * rows of D fp32 values: r = D^-1/2 H_D diag(s) e with s from `seed`, then
 * absmax quantization to `bits` with one fp32 scale per `group` values and
 * LSB-first packing. DEVICE in/out: e[rows][D]; codes[rows][bits*D/8];
 * scales[rows][D/group]. */
JOLT_API jolt_status jolt_residual_encode(const float* e, int64_t rows, int32_t D,
                                 int32_t bits, int32_t group, uint64_t seed,
                                 uint8_t* codes, float* scales,
                                 jolt_stream_t stream);
/* Inverse: e_hat = diag(s) D^-1/2 H_D dequant(codes). DEVICE in/out. */
JOLT_API jolt_status jolt_residual_decode(const uint8_t* codes, const float* scales,
                                 int64_t rows, int32_t D, int32_t bits,
                                 int32_t group, uint64_t seed, float* e_hat,
                                 jolt_stream_t stream);

/* The residual stage exactly as jolt_compress runs it (the tensor-core
 * stream kernel of Section 3, "Rotated low-bit residual": E = X - U_T^ M^_lh
 * per (layer, head), keys un-RoPE'd first, the seeded Hadamard rotation,
 * absmax quantization, LSB-first packing), on caller-given factors instead of
 * fitted ones, so that its codes and scales can be checked bit for bit.
 *   x: DEVICE bf16 [LH][T][D], 16-byte aligned (LH = layer-head pairs).
 *   ut_t: DEVICE bf16 [r][T], U_T^ transposed (1 <= r <= 512).
 *   m: DEVICE bf16 [LH][r][D], the per-(layer, head) products M^.
 *   rope_theta > 0: x holds keys after a rotate-half RoPE of that base over
 *     positions 0..T-1, undone in fp32 before the residual (as jolt_compress
 *     does for keys).
 *   codes: DEVICE [LH][T][bits*D/8]; scales: DEVICE fp32 [LH][T][D/group]
 *     (both 16-byte aligned). bits in {2,3,4,8}; group 32, 64 or D.
 * Allocates scratch through the library allocator and synchronises the
 * stream; a device status (timeout) is returned as for jolt_compress. */
JOLT_API jolt_status jolt_residual_stream_encode(const void* x, int32_t LH, int32_t T, int32_t D,
                                                 const uint16_t* ut_t, int32_t r, const uint16_t* m,
                                                 int32_t bits, int32_t group, uint64_t seed, float rope_theta,
                                                 uint8_t* codes, float* scales, jolt_stream_t stream);

/* The Gaussian sketch Omega of Section 3.1 (the randomized range finder's
 * test matrix) that jolt_compress and jolt_rd_table draw for every cell of a
 * JOLT_RANDOMIZED plan with this seed: column j of cell c's Omega is row j of
 * omega_t[c] (DEVICE, bf16 bit patterns, [n_cells][k][ld]); entries n >= N_c
 * (N_c = L_g*H*D of the cell) are zero. k (the sketch width, q_cap + p
 * rounded up to 16) and ld (the largest N_c) are written to *k_out / *ld_out
 * (HOST, either may be NULL). omega_t NULL returns only k and ld.
 * JOLT_ERR_INVALID_ARG for an exact-mode plan. Asynchronous. */
JOLT_API jolt_status jolt_sketch(jolt_plan_t* plan, uint64_t seed, uint16_t* omega_t, int32_t* k_out,
                                 int32_t* ld_out, jolt_stream_t stream);

/* Data-driven layer grouping (Section 3, the paragraph that partitions the L
 * layers into G contiguous groups, and its footnote on size bounds): for each
 * sequence b and layer l, an 8-dimensional basis U of the top token-mode
 * singular vectors of the keys K[b, l] unfolded as [T, H*D] (the keys before
 * RoPE when rope_theta_k > 0, undone as for jolt_compress); the score of
 * layers (l, l+1) is the mean squared cosine of the principal angles between
 * the two bases, ||U_l^T U_(l+1)||_F^2 / 8, averaged over the sequences of
 * the batch. A new group starts at layer l when score(l-1, l) is strictly
 * below the median of the n_layers-1 scores (the mean of the two middle ones
 * for an even count), but only once the current group holds 2 layers; a
 * group that holds 8 layers is closed whatever the score; a trailing group of
 * one layer joins its predecessor (so the last group can hold 9).
 * The basis comes from a randomized subspace iteration of width 16 (8
 * vectors + 8 oversampling) with `power_iters` power iterations and a
 * Rayleigh-Ritz step; the sketch is seeded by `seed` (Philox4x32-10). The
 * subspace error falls like (sigma_17 / sigma_8)^(2 power_iters + 1); 4 is a
 * good default. A layer whose keys are all zero has the zero basis (score 0).
 *   layout: as for jolt_plan; n_groups and group_start are not read.
 *     seq_len >= 16, n_layers <= 1024, batch * n_layers <= 65535; strides
 *     even and `k` 8-byte aligned.
 *   k: DEVICE keys in that layout.
 *   power_iters: 0..32.
 *   scores: HOST output of n_layers-1 doubles, or NULL.
 *   group_start: HOST output, room for n_layers+1 entries: 0, the starts,
 *     n_layers. n_groups: HOST output.
 * Allocates its workspace through the library allocator (64 bytes per
 * (sequence, layer, token) plus 4 bytes per key element rounded up to
 * 2048-token chunks, i.e. about twice the bf16 keys over 16) and
 * synchronises `stream`. A non-finite Gram or score (Inf/NaN
 * keys) returns JOLT_ERR_NONFINITE. */
JOLT_API jolt_status jolt_layer_groups(const jolt_layout* layout, const void* k,
                                       int32_t power_iters, uint64_t seed,
                                       double* scores, int32_t* group_start,
                                       int32_t* n_groups, jolt_stream_t stream);

/* Device allocator used for handles and workspace. alloc returns NULL on
 * failure (-> JOLT_ERR_OOM). Passing NULLs restores the default. */
typedef void* (*jolt_alloc_fn)(size_t bytes, jolt_stream_t stream, void* ctx);
typedef void (*jolt_free_fn)(void* ptr, jolt_stream_t stream, void* ctx);
JOLT_API jolt_status jolt_set_allocator(jolt_alloc_fn alloc, jolt_free_fn free_fn,
                               void* ctx);

/* Thread-local description of the last failure on this thread. */
JOLT_API const char* jolt_last_error(void);

/* Number of kernels this library has launched in this process (for
 * launch-count reporting). */
JOLT_API uint64_t jolt_launch_count(void);

/* Stage timing. While enabled, every stage of compress/decompress records a
 * CUDA event before and after itself on the call's stream (no extra host
 * synchronisation); jolt_profile_read waits for the recorded events and
 * returns, per stage, the summed device time and the kernel launches.
 * Enabling (or disabling) clears the counters. Not thread-safe. */
enum {
  JOLT_STAGE_COPY = 0,        /* bf16 working copies (un-RoPE keys)          */
  JOLT_STAGE_FGRAM = 1,       /* feature Gram X_(d) X_(d)^T and ||X||^2      */
  JOLT_STAGE_TOKEN_GRAM = 2,  /* exact mode: token Gram                      */
  JOLT_STAGE_GEMM_XW = 3,     /* randomized: X * W (sketch, power steps)     */
  JOLT_STAGE_GEMM_XTY = 4,    /* randomized: X^T * Y                         */
  JOLT_STAGE_ORTH = 5,        /* randomized: fp64 CholeskyQR of Z            */
  JOLT_STAGE_GEMM_GRAM = 6,   /* randomized: W^T W                           */
  JOLT_STAGE_EIG = 7,         /* eigensolvers (+ the small k x k solves)     */
  JOLT_STAGE_ALLOC = 8,       /* rate-distortion tables + lambda bisection   */
  JOLT_STAGE_FIT = 9,         /* factors, projection, core                   */
  JOLT_STAGE_RESIDUAL = 10,   /* residual, rotation, quantization, packing   */
  JOLT_STAGE_DECOMPRESS = 11, /* decoder                                     */
  JOLT_NUM_STAGES = 12
};
typedef struct {
  double ms;
  int64_t calls;
  int64_t launches;
} jolt_stage_stats;
JOLT_API void jolt_profile_enable(int32_t on);
JOLT_API jolt_status jolt_profile_read(jolt_stage_stats* out, int32_t n);

#ifdef __cplusplus
}
#endif
#endif /* JOLT_H */
