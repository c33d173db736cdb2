// Batched small dense fp64 linear algebra for the randomized range finder
// (CholeskyQR and B B^T = R^{-T} (Z^T Z) R^{-1}, "A JoLT for the KV Cache",
// Section 3.1): every kernel runs all cells at once and spreads each matrix
// over many thread blocks.
//
//   chol:  G = R^T R (upper R) by 32-column blocks: factor the diagonal block,
//          solve the block row, subtract the block row's outer product from the
//          trailing matrix; also writes R^T.
//   trsm:  X R = B (forward, reading rows of R^T) or X R^T = B (backward,
//          reading rows of R) for many independent rows: a warp owns four rows,
//          eight lanes per row share the inner products, R stays in L2.
#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {

constexpr int NB = 32;

// fp32 -> fp64 copy (optional), diagonal shift 1e-13 trace/k (1.0 for an
// all-zero matrix), lower triangle of R and R^T cleared.
__global__ void k_chol_prep(double* __restrict__ G, int64_t cs, const float* __restrict__ src32, int k,
                            double* __restrict__ RT) {
  const int cell = blockIdx.x;
  double* g = G + (int64_t)cell * cs;
  double* rt = RT + (int64_t)cell * cs;
  __shared__ double red[32];
  if (src32) {
    const float* s = src32 + (int64_t)cell * cs;
    for (int64_t e = threadIdx.x; e < (int64_t)k * k; e += blockDim.x) g[e] = (double)s[e];
    __syncthreads();
  }
  double tr = 0.0;
  for (int i = threadIdx.x; i < k; i += blockDim.x) tr += g[(int64_t)i * k + i];
  for (int o = 16; o > 0; o >>= 1) tr += __shfl_xor_sync(0xffffffffu, tr, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = tr;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    red[0] = t;
  }
  __syncthreads();
  const double shift = (red[0] > 0.0) ? 1e-13 * red[0] / k : 1.0;
  __syncthreads();
  for (int i = threadIdx.x; i < k; i += blockDim.x) g[(int64_t)i * k + i] += shift;
  for (int64_t e = threadIdx.x; e < (int64_t)k * k; e += blockDim.x) {
    const int i = (int)(e / k), j = (int)(e % k);
    if (i > j) g[e] = 0.0;
    rt[e] = 0.0;
  }
}

// Factor the NB x NB diagonal block J in place (upper), one block per cell.
__global__ void __launch_bounds__(NB * NB) k_chol_diag(double* __restrict__ G, double* __restrict__ RT, int64_t cs,
                                                      int k, int J, int* status) {
  const int cell = blockIdx.x;
  double* g = G + (int64_t)cell * cs;
  double* rt = RT + (int64_t)cell * cs;
  const int j0 = J * NB;
  const int nb = min(NB, k - j0);
  __shared__ double a[NB][NB + 1];
  const int r = threadIdx.x / NB, c = threadIdx.x % NB;
  a[r][c] = (r < nb && c < nb) ? g[(int64_t)(j0 + r) * k + j0 + c] : 0.0;
  __syncthreads();
  for (int j = 0; j < nb; ++j) {
    if (threadIdx.x == 0) {
      double piv = a[j][j];
      if (!(piv > 0.0)) { atomicOr(status, DEV_ERR_CHOL); piv = 1e-300; }
      a[j][j] = sqrt(piv);
    }
    __syncthreads();
    if (r == j && c > j && c < nb) a[j][c] /= a[j][j];
    __syncthreads();
    if (r > j && c >= r && c < nb) a[r][c] -= a[j][r] * a[j][c];
    __syncthreads();
  }
  if (r < nb && c < nb) {
    const double v = (c >= r) ? a[r][c] : 0.0;
    g[(int64_t)(j0 + r) * k + j0 + c] = v;
    rt[(int64_t)(j0 + c) * k + j0 + r] = v;
  }
}

// Block row J: R[J, c] = R_JJ^{-T} G[J, c] for the columns c right of the
// block (forward substitution with the lower R_JJ^T), one column per thread.
__global__ void k_chol_row(double* __restrict__ G, double* __restrict__ RT, int64_t cs, int k, int J) {
  const int cell = blockIdx.y;
  double* g = G + (int64_t)cell * cs;
  double* rt = RT + (int64_t)cell * cs;
  const int j0 = J * NB, nb = min(NB, k - j0);
  const int c = j0 + nb + blockIdx.x * blockDim.x + threadIdx.x;
  __shared__ double d[NB][NB + 1];
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, q = e % NB;
    d[r][q] = (r < nb && q < nb) ? g[(int64_t)(j0 + r) * k + j0 + q] : 0.0;
  }
  __syncthreads();
  if (c >= k) return;
  double x[NB];
#pragma unroll
  for (int i = 0; i < NB; ++i) x[i] = (i < nb) ? g[(int64_t)(j0 + i) * k + c] : 0.0;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    if (i < nb) {
      double acc = x[i];
#pragma unroll
      for (int t = 0; t < i; ++t) acc -= d[t][i] * x[t];
      x[i] = acc / d[i][i];
    }
  }
#pragma unroll
  for (int i = 0; i < NB; ++i)
    if (i < nb) {
      g[(int64_t)(j0 + i) * k + c] = x[i];
      rt[(int64_t)c * k + j0 + i] = x[i];
    }
}

// Trailing update: G[i][j] -= sum_t R[J*NB+t][i] R[J*NB+t][j] for
// J*NB+nb <= i <= j (upper triangle), 64 x 64 tiles.
__global__ void __launch_bounds__(256) k_chol_update(double* __restrict__ G, int64_t cs, int k, int J) {
  const int cell = blockIdx.y;
  double* g = G + (int64_t)cell * cs;
  const int j0 = J * NB, nb = min(NB, k - j0);
  const int base = j0 + nb;
  const int m = k - base;
  if (m <= 0) return;
  const int nt = (m + 63) / 64;
  int b = blockIdx.x, ti = 0;
  while (ti < nt && b >= nt - ti) { b -= nt - ti; ++ti; }
  if (ti >= nt) return;
  const int tj = ti + b;
  __shared__ double P[NB][64];
  __shared__ double Q[NB][64];
  for (int e = threadIdx.x; e < NB * 64; e += blockDim.x) {
    const int t = e / 64, q = e % 64;
    const int ci = base + ti * 64 + q, cj = base + tj * 64 + q;
    P[t][q] = (t < nb && ci < k) ? g[(int64_t)(j0 + t) * k + ci] : 0.0;
    Q[t][q] = (t < nb && cj < k) ? g[(int64_t)(j0 + t) * k + cj] : 0.0;
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
#pragma unroll 8
  for (int t = 0; t < NB; ++t) {
    double a[4], c[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) { a[q] = P[t][ty * 4 + q]; c[q] = Q[t][tx * 4 + q]; }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[p][q] = fma(a[p], c[q], acc[p][q]);
  }
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = base + ti * 64 + ty * 4 + p, j = base + tj * 64 + tx * 4 + q;
      if (i < k && j < k && j >= i) g[(int64_t)i * k + j] -= acc[p][q];
    }
}

jolt_status launch_chol_blocked(double* G, double* RT, int64_t cs, const float* src32, int k, int ncells, int* status,
                                cudaStream_t s) {
  k_chol_prep<<<ncells, 512, 0, s>>>(G, cs, src32, k, RT);
  JOLT_LAUNCHED();
  const int nbk = (k + NB - 1) / NB;
  for (int J = 0; J < nbk; ++J) {
    k_chol_diag<<<ncells, NB * NB, 0, s>>>(G, RT, cs, k, J, status);
    JOLT_LAUNCHED();
    const int rest = k - std::min(k, (J + 1) * NB);
    if (rest <= 0) break;
    dim3 g1((rest + 127) / 128, ncells);
    k_chol_row<<<g1, 128, 0, s>>>(G, RT, cs, k, J);
    JOLT_LAUNCHED();
    const int nt = (rest + 63) / 64;
    dim3 g2(nt * (nt + 1) / 2, ncells);
    k_chol_update<<<g2, 256, 0, s>>>(G, cs, k, J);
    JOLT_LAUNCHED();
  }
  return JOLT_OK;
}

// --------------------------------------------------------- row solves ------
// Rows x of X (one cell per blockIdx.y, 32 rows per block):
//   forward  (upper R, X R = B):   x_j = (b_j - sum_{i<j} x_i R[i][j]) / R[j][j]
//                                  with R[i][j] read as RT[j][i];
//   backward (X R^T = B):          x_j = (b_j - sum_{i>j} x_i R[j][i]) / R[j][j].
// B: element (r, j) at b[r*ldb_r + j*ldb_c] in fp32 or fp64 (b64 != 0).
// Outputs (any may be null): X64[r*ld64_r + j*ld64_c] fp64 and
// X16[r*ld16_r + j*ld16_c] bf16. rows_of[cell] rows exist.

constexpr int TR_ROWS = 32;

__global__ void __launch_bounds__(256) k_trsm_rows2(TrsmArgs a) {
  extern __shared__ double xs[];      // TR_ROWS x k
  const int cell = blockIdx.y;
  const int rows = a.rows_of ? a.rows_of[cell] : a.rows_fixed;
  const int r0 = blockIdx.x * TR_ROWS;
  if (r0 >= rows) return;
  const int k = a.k;
  // load the block's rows of B (coalesced along whichever index is contiguous)
  for (int e = threadIdx.x; e < TR_ROWS * k; e += blockDim.x) {
    int rr, j;
    if (a.ldb_c == 1) { rr = e / k; j = e % k; }
    else { j = e / TR_ROWS; rr = e % TR_ROWS; }
    const int r = r0 + rr;
    double v = 0.0;
    if (r < rows) {
      const int64_t off = (int64_t)cell * a.b_cell + (int64_t)r * a.ldb_r + (int64_t)j * a.ldb_c;
      v = a.b64 ? reinterpret_cast<const double*>(a.B)[off] : (double)reinterpret_cast<const float*>(a.B)[off];
    }
    xs[rr * k + j] = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = warp * 4 + (lane >> 3);      // row of this 8-lane group
  const int sub = lane & 7;
  double* x = xs + rr * k;
  const double* Rm = a.R + (int64_t)cell * a.r_cell;
  const double* RTm = a.RT + (int64_t)cell * a.r_cell;
  if (!a.backward) {
    for (int j = 0; j < k; ++j) {
      const double* col = RTm + (int64_t)j * k;     // R[i][j] = RT[j][i]
      double acc = 0.0;
      for (int i = sub; i < j; i += 8) acc += x[i] * col[i];
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (sub == 0) x[j] = (x[j] - acc) / col[j];
      __syncwarp();
    }
  } else {
    for (int j = k - 1; j >= 0; --j) {
      const double* row = Rm + (int64_t)j * k;      // R[j][i], i > j
      double acc = 0.0;
      for (int i = j + 1 + sub; i < k; i += 8) acc += x[i] * row[i];
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (sub == 0) x[j] = (x[j] - acc) / row[j];
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < TR_ROWS * k; e += blockDim.x) {
    // coalesce along rows for the transposed outputs, along j otherwise
    int q, j;
    if ((a.X16 && a.ld16_r == 1) || (a.X64 && a.ld64_r == 1)) { j = e / TR_ROWS; q = e % TR_ROWS; }
    else { q = e / k; j = e % k; }
    const int r = r0 + q;
    if (r >= rows) continue;
    const double v = xs[q * k + j];
    if (a.X64) a.X64[(int64_t)cell * a.x64_cell + (int64_t)r * a.ld64_r + (int64_t)j * a.ld64_c] = v;
    if (a.X16) a.X16[(int64_t)cell * a.x16_cell + (int64_t)r * a.ld16_r + (int64_t)j * a.ld16_c] = bf16_bits_from_f64(v);
  }
}

jolt_status launch_trsm_rows2(const TrsmArgs& a, int rows_max, int ncells, cudaStream_t s) {
  const size_t smem = (size_t)TR_ROWS * a.k * sizeof(double);
  if (smem > 200 * 1024) { set_error("row solve needs k <= 800 (k=%d)", a.k); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  static size_t set = 0;
  if (smem > set) {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_trsm_rows2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    set = smem;
  }
  dim3 g((rows_max + TR_ROWS - 1) / TR_ROWS, ncells);
  k_trsm_rows2<<<g, 256, smem, s>>>(a);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
