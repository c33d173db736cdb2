// Kernel-side structures and host launchers shared across translation units.
#pragma once
#include <cuda.h>
#include "jolt_internal.cuh"

namespace jolt {

// ------------------------------------------------------------ eigensolver --
struct EighJob {
  int n;
  int want_vec;
  double* A;      // n*n, destroyed
  double* w;      // n, descending
  double* Vt;     // n*n, row j = eigenvector j (if want_vec)
  double* Z;      // n*n scratch (if want_vec)
  double* work;   // 3n scratch: d, e, beta of the tridiagonal reduction
  double* F;      // 5n doubles per requested eigenvector (inverse iteration)
};

jolt_status launch_tridiag(const EighJob* jobs, int njobs, int nmax, cudaStream_t s);
// Multi-block reduction of jobs[0..njobs) (all of size <= nmax); scratch holds
// njobs * (2 nmax + 128) doubles, counters 2 njobs + 1 words.
jolt_status launch_tridiag_multi(const EighJob* jobs, int njobs, int nmax, double* scratch, unsigned int* counters,
                                 int* status, cudaStream_t s);
jolt_status launch_bisect(const EighJob* jobs, int njobs, int nmax, cudaStream_t s);
// Eigenvectors of the leading nvec[job] eigenvalues of jobs of size <= nmax
// (nmax sizes the back-transformation blocks).
jolt_status launch_eigvecs_n(const EighJob* jobs, int njobs, int nvec_max, int nmax, const int* nvec, cudaStream_t s);
jolt_status launch_fgram_x(const CellDesc* cells, int ncells, int D, const float2* cs, int nchunk,
                           double* partial, cudaStream_t s);
jolt_status launch_fgram_rows(const double* const* Y, const int* nrow_used, const int* rmax_of,
                              const int* nlh_of, int ncells, int D, int nchunk, double* partial,
                              cudaStream_t s);
jolt_status launch_sum_chunks(const double* partial, int nchunk, int len, int ncells,
                              double* const* out, double* const* out_last, cudaStream_t s);
jolt_status launch_token_gram(const CellDesc* cells, int ncells, int nmax, const float2* cs,
                              double* const* G, cudaStream_t s);

// ------------------------------------------------------------- allocation --
// Per-cell data the allocator reads (device).
struct CellRD {
  int Lg, H, T, D;
  int n_rt;             // grid entries usable by this cell
  int nt;               // t_T has nt+1 entries
  const double* tT;     // [nt+1]
  const double* tD;     // [D+1]
};

struct AllocState {
  double lo, hi, lam;   // bracket and the multiplier being evaluated
  double tol;
  int64_t budget;
  int max_iters;
  int phase;            // 0: lambda_lo, 1: lambda_hi, 2: bisection, 3: done
  int iter;
  int result_from_hi;   // 1 when the final answer is the kept feasible side
  double lam_final;
  int iters_final;
  int64_t S;
  unsigned arrive;      // blocks of the current evaluation round that have finished
};

// The chosen option of a cell (device).
struct Choice {
  int rT, rd, b, pad;
  int64_t bytes;
  double err;
};

struct AllocArgs {
  const CellRD* cells;
  int ncells;
  const int* rt_grid;       // shared grid values
  const int* rd_grid;
  int n_rd;
  const int* bits;
  const double* eps2;
  const int64_t* rowbytes;  // residual bytes per row for each bit entry
  int n_bits;
  int nchunk;               // option chunks per cell
  double* pv;               // [ncells][nchunk] partial min values
  int* pi;                  // [ncells][nchunk] partial argmins
  int* cur;                 // [ncells] current argmin
  int* keep;                // [ncells] feasible-side argmin
  AllocState* st;
  Choice* out;              // [ncells]
  int* status;
  int greedy;               // 1: the page's greedy per-cell search instead of enumeration
  int n_rt_max;             // the most r_T grid entries of any cell (sizes the search)
};

jolt_status launch_alloc(const AllocArgs& a, const AllocState& init, cudaStream_t s);

// One cell's rate-distortion summary as exchanged between processes that
// share one byte budget: this 64-byte header, then t_T[ntp] and t_D[D + 1]
// (doubles), the record padded to rec_bytes. The header carries the cell's
// shape and grid length, its global (sequence, group, kind), and a
// fingerprint of the allocation settings (grids, bits, scale group,
// tolerance), which every record of one allocation must share.
struct RDRecordHdr {
  uint32_t magic;
  int32_t Lg, H, T, D, n_rt, nt, ntp;
  uint64_t fingerprint;
  double norm_sq;
  int32_t seq, group, kind, rec_bytes;
};
static_assert(sizeof(RDRecordHdr) == 64, "record header is 64 bytes");
constexpr uint32_t RD_MAGIC = 0x3144524Au;
jolt_status launch_write_records(const CellRD* cells, int ncells, const double* const* normsq, const int4* ids,
                                 uint64_t fingerprint, int ntp, int rec_bytes, uint8_t* out, cudaStream_t s);
// CellRD views of n_total gathered records (pointers into the record
// buffer, laid out by this plan's ntp and D, never by a record's own header);
// a record whose header disagrees with this plan (magic, fingerprint, sizes,
// a grid longer than this plan's, or, for the local slice, another cell's
// identity) raises DEV_ERR_MISMATCH and is read as a one-option cell.
jolt_status launch_records_to_rd(const uint8_t* recs, int n_total, int rec_bytes, int ntp, int D, uint64_t fingerprint,
                                 int n_rt_max, int first, int nlocal, const int4* ids, CellRD* out, int* status,
                                 cudaStream_t s);
jolt_status launch_rd_tables(const CellRD* cells, int ncells, const double* const* wT,
                             const double* const* wD, const double* normsq,
                             double* const* tT, double* const* tD, const int* nt_used,
                             const double* const* normsq_in, int* status, cudaStream_t s);
jolt_status launch_eps2(const int* bits_host, int nb, int G, double* eps2_dev, double* scratch,
                        cudaStream_t s);

// ------------------------------------------------------------------ fit ----
// Where one compressed cell lives in the handle's payload (device).
struct CellOut {
  uint16_t* ut;      // [rT][t_pitch] bf16 U_T^ transposed
  uint16_t* ud;      // [D][rd] bf16
  uint16_t* core;    // [Lg][H][rT][rd] bf16
  uint8_t* codes;    // [Lg][H][T][b*D/8]
  float* scales;     // [Lg][H][T][D/G]
  int rT, rd, b, t_pitch;
  int64_t bytes;
};

jolt_status launch_payload_layout(const CellDesc* cells, const Choice* ch, int ncells, int G,
                                  uint8_t* base, int64_t capacity, CellOut* out, int* status,
                                  cudaStream_t s);

struct FitArgs {
  const CellDesc* cells;
  const float2* cs;
  const CellOut* out;
  int ncells;
  int D;
  // exact-mode token factor
  const double* const* VtT;     // eigenvectors of the token Gram (rows)
  const double* const* wT;      // eigenvalues
  double* const* Uf;            // [rmax][T] fp64 scratch (T > N case)
  // projection / feature factor / core
  double* const* Y;             // [Lg*H][rmax][D] fp64
  const int* rmax_of;
  const double* const* VtY;     // eigenvectors of the projected feature Gram
  uint16_t* const* M;           // [Lg*H][rmax][D] bf16 (decoder product M^)
};

jolt_status launch_ut_exact(const FitArgs& a, int Tmax, int rmax_all, cudaStream_t s);
jolt_status launch_project_y(const FitArgs& a, int Tmax, int rmax_all, int lh_max, cudaStream_t s);
jolt_status launch_core(const FitArgs& a, int rmax_all, int lh_max, cudaStream_t s);
jolt_status launch_copy_rt(const CellOut* out, int* rt, int ncells, cudaStream_t s);
jolt_status launch_core_m(const CellOut* out, const CellDesc* cells, uint16_t* const* M, const int* rmax_of,
                          int ncells, int D, int rmax_all, int lh_max, cudaStream_t s);

// ----------------------------------------------------------- residual ------
struct ResidArgs {
  const CellDesc* cells;
  const float2* cs;
  const CellOut* out;
  uint16_t* const* M;           // [Lg*H][rmax][D] bf16 per cell
  const int* rmax_of;
  int G;
  uint64_t seed;
  const double* qrot;           // [batch][D][D] QR-Gaussian rotation; NULL: Hadamard
  // decompress outputs (bf16)
  uint16_t* out_k;              // decompress outputs (bf16), NULL when encoding
  uint16_t* out_v;
  int64_t osb, osl, osh, ost;   // output strides (elements)
};

jolt_status launch_residual_simt(const ResidArgs& a, int ncells, int D, int Tmax, int lh_max,
                                 cudaStream_t s);
jolt_status launch_decompress_simt(const ResidArgs& a, int ncells, int D, int Tmax, int lh_max,
                                   cudaStream_t s);
jolt_status launch_encode_rows(const float* e, int64_t rows, int D, int b, int G, uint64_t seed,
                               uint8_t* codes, float* scales, cudaStream_t s);
jolt_status launch_decode_rows(const uint8_t* codes, const float* scales, int64_t rows, int D,
                               int b, int G, uint64_t seed, float* e, cudaStream_t s);
jolt_status launch_rope_table(int T, int D, double theta, float2* cs, cudaStream_t s);
// The QR-Gaussian rotation of each sequence b (seed + b): q[b][D][D], fp64;
// work holds batch * D * D doubles of scratch.
jolt_status launch_qr_rotation(int D, int batch, uint64_t seed, double* work, double* q, cudaStream_t s);
jolt_status launch_copy_out(const CellOut* out, int* rt, uint16_t** ut, int ncells, cudaStream_t s);

// ------------------------------------------------------- randomized mode ---
jolt_status map_x5(CUtensorMap* m, const void* base, int B, int L, int H, int T, int D, int64_t sb, int64_t sl,
                   int64_t sh, int64_t st);
jolt_status map_3d(CUtensorMap* m, const void* base, int cells, int rows, int cols, int64_t pitch, int box_rows);
jolt_status launch_make_xb(const void* src, int f32, int rope, const float2* cs, int B, int L, int H, int T,
                           int D, int64_t sb, int64_t sl, int64_t sh, int64_t st, uint16_t* dst, cudaStream_t s);
jolt_status launch_omega(uint16_t* wt, int ncells, int k, int ld, const int* Nc, const int* seq, const int* cis,
                         uint64_t seed, cudaStream_t s);
constexpr int GRAM_SPLIT = 4;   // K slices of the fp64 Gram (partials in a scratch buffer)
jolt_status launch_gram_cols(const float* A, int64_t a_cell, const int* rows_of, int k, double* C, int64_t c_cell,
                             int ncells, double* part, cudaStream_t s);
jolt_status launch_rand_spectrum(const double* w_eig, int64_t cs, int q, const double* const* normsq,
                                 double* const* wT, int ncells, cudaStream_t s);
jolt_status launch_yproj(const float* Z, int64_t z_cell, const double* P64, int64_t p_cell, int k, int rmax,
                         const CellOut* outs, const int* nlh, double* const* Y, int lh_max, int D, int ncells,
                         cudaStream_t s);
jolt_status launch_fgram_reduce(const float* part, int nchunk, int D, double* const* C, double* const* normsq,
                                int ncells, cudaStream_t s);

}  // namespace jolt

namespace jolt {
// ------------------------------------------- tensor-core residual streams --
struct StreamMaps {
  CUtensorMap ut;   // U_T^ workspace [cells][rows][tp], box {64 t, 64 r}
  CUtensorMap mt;   // M^T workspace [cells*lhmax][D][rpad_m], box {64 r, D}
  CUtensorMap xk;   // key input, box {64 d, 128 t, 1, 1, 1}
  CUtensorMap xv;   // value input
};
struct StreamArgs {
  int ncells, T, H, lhmax, rpad_m, G;
  const CellDesc* cells;
  const CellOut* outs;
  const float2* cs;
  const float4* csq;     // the RoPE table tiled for the stream kernel (launch_rope_tiled), or null
  uint64_t seed;
  uint16_t* out_k;
  uint16_t* out_v;
  int64_t osb, osl, osh, ost;
  int* status;
};
jolt_status launch_stream(bool compress, int D, const StreamMaps& m, const StreamArgs& a, cudaStream_t s);
// The RoPE table rearranged so that the stream kernel's warps read it with
// coalesced 16-byte loads: for token tile tau (128 tokens), column quarter j
// and pair unit u (pairs 2u, 2u + 1 of the quarter's D/8 pairs), the 128 rows'
// float4 (cos, sin, cos, sin) are contiguous: csq[((tau*4 + j)*(D/16) + u)*128 + row].
// Rows past T hold zeros. ceil(T/128)*128*D/2 float2 entries.
jolt_status launch_rope_tiled(const float2* cs, int T, int D, float4* csq, cudaStream_t s);

// ------------------------------------------------- fused decode attention --
constexpr int DEC_BMAX = 16;      // sequences per launch
struct DecodeCall {
  int B, H, D, T, G, gq, li;      // G query heads per KV head, li = layer within its group
  const CellOut* kout;            // key cell of sequence 0 (device); sequence b at b * cstride
  const CellOut* vout;            // value cells, same stride
  int cstride;
  const float2* cs;               // RoPE table of the keys, or null
  uint64_t seed;                  // rotation seed of sequence 0
  const float* q;                 // [B][H*G][D]
  float* out;                     // [B][H*G][D]
  const uint16_t* tail_k;         // [B][H][ntail][D] bf16, or null
  const uint16_t* tail_v;
  int ntail;
  uint16_t* mtk; int rpk;         // workspace: M^_K^T [B*H][D][rpk]
  float* mv; int rpv;             // workspace: M^_V [B*H][rpv][D]
  float* part; int64_t part_len;  // workspace: split states
  const uint16_t* ut[DEC_BMAX];   // U_T^ of each sequence's key cell and its shape
  int rt_k[DEC_BMAX], tpitch[DEC_BMAX];
  const uint16_t* uv[DEC_BMAX];   // U_T^ of each sequence's value cell and its shape
  int rt_v[DEC_BMAX], tpitch_v[DEC_BMAX];
  int* status;
};
jolt_status launch_decode_attention(const DecodeCall& c, cudaStream_t s);
jolt_status launch_ut_to_ws(const CellOut* outs, uint16_t* ws, int rows, int tp, int ncells, cudaStream_t s);
jolt_status launch_m_transpose(const CellOut* outs, const CellDesc* cells, uint16_t* const* M, const int* rmax_of,
                               uint16_t* Mt, int lhmax, int D, int rpad, int ncells, cudaStream_t s);
jolt_status map_x5_box(CUtensorMap* m, const void* base, int B, int L, int H, int T, int D, int64_t sb,
                       int64_t sl, int64_t sh, int64_t st, int box_t);
jolt_status map_3d_box(CUtensorMap* m, const void* base, int cells, int rows, int cols, int64_t pitch,
                       int box_cols, int box_rows);
}  // namespace jolt

namespace jolt {
// ------------------------------------------ batched dense fp64 (k x k) -----
struct TrsmArgs {
  const double* Rinv;   // R^{-1} (k x k, row-major, upper), read by the forward product
  const double* RinvT;  // R^{-T} (k x k, row-major, lower), read by the backward product
  int64_t r_cell;
  int k;
  int backward;         // 0: X R = B, 1: X R^T = B
  const void* B;        // element (r, j) at B[cell*b_cell + r*ldb_r + j*ldb_c]
  int b64;              // 1: fp64, 0: fp32
  int64_t b_cell, ldb_r, ldb_c;
  const int* rows_of;   // rows per cell (null: rows_fixed)
  int rows_fixed;
  double* X64;          // optional fp64 output at X64[cell*x64_cell + r*ld64_r + j*ld64_c]
  int64_t x64_cell, ld64_r, ld64_c;
  uint16_t* X16;        // optional bf16 output at X16[cell*x16_cell + r*ld16_r + j*ld16_c]
  int64_t x16_cell, ld16_r, ld16_c;
};
jolt_status launch_chol_blocked(double* G, double* RT, int64_t cs, const float* src32, int k, int ncells, int* status,
                                cudaStream_t s);
jolt_status launch_tri_inverse(const double* R, double* Ri, double* RiT, int64_t cs, int k, int ncells,
                               cudaStream_t s);
jolt_status launch_tri_apply(const TrsmArgs& a, int rows_max, int ncells, cudaStream_t s);
jolt_status launch_symmetrize(double* M, int64_t cs, int k, int ncells, cudaStream_t s);
}  // namespace jolt
