// Batched small dense fp64 linear algebra for the randomized range finder
// (CholeskyQR and B B^T = R^{-T} (Z^T Z) R^{-1}, "A JoLT for the KV Cache",
// Section 3.1): every kernel runs all cells at once and spreads each matrix
// over many thread blocks.
//
//   chol:  G = R^T R (upper R) by 32-column blocks: factor the diagonal block,
//          solve the block row, subtract the block row's outer product from the
//          trailing matrix; also writes R^T.
//   trinv: R^{-1} and R^{-T} by 32 x 32 block back-substitution.
//   apply: X R = B or X R^T = B for many independent rows as a tiled product
//          with R^{-1} or R^{-T}.
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

// ------------------------------------------------- triangular inverse ------
// R^{-1} of an upper triangular R (k x k, row-major, lower part zero) by
// 32 x 32 blocks: the diagonal blocks are inverted first, then the block
// column J of Y = R^{-1} follows by block back-substitution
//   Y[I][J] = -inv(R[I][I]) * sum_{I < K <= J} R[I][K] Y[K][J],   I < J,
// one thread block per (J, cell) holding Y's block column in shared memory.
// Both R^{-1} and its transpose are written in full (zeros included), so the
// products below may read whole tiles.

__global__ void __launch_bounds__(NB) k_trinv_diag(const double* __restrict__ R, double* __restrict__ Ri,
                                                   double* __restrict__ RiT, int64_t cs, int k) {
  const int cell = blockIdx.y, I = blockIdx.x;
  const int i0 = I * NB, nb = min(NB, k - i0);
  const double* r = R + (int64_t)cell * cs;
  __shared__ double Rd[NB][NB + 1];
  __shared__ double Y[NB][NB + 1];
  const int c = threadIdx.x;
  for (int i = 0; i < NB; ++i) Rd[i][c] = (i < nb && c < nb) ? r[(int64_t)(i0 + i) * k + i0 + c] : 0.0;
  __syncthreads();
  // column c of inv(Rd): back substitution, entries below the diagonal are 0
  for (int i = NB - 1; i >= 0; --i) {
    double acc = (i == c) ? 1.0 : 0.0;
    if (i < nb && c < nb && i <= c) {
      for (int m = i + 1; m <= c; ++m) acc -= Rd[i][m] * Y[m][c];
      acc /= Rd[i][i];
    } else {
      acc = 0.0;
    }
    Y[i][c] = acc;
  }
  __syncthreads();
  double* ri = Ri + (int64_t)cell * cs;
  double* rit = RiT + (int64_t)cell * cs;
  for (int i = 0; i < nb; ++i)
    if (c < nb) {
      ri[(int64_t)(i0 + i) * k + i0 + c] = Y[i][c];
      rit[(int64_t)(i0 + c) * k + i0 + i] = Y[i][c];
    }
}

__global__ void __launch_bounds__(256) k_trinv(const double* __restrict__ R, double* __restrict__ Ri,
                                               double* __restrict__ RiT, int64_t cs, int k) {
  extern __shared__ double Ys[];            // rows [0, (J+1)*NB) of block column J, NB wide
  __shared__ double Rp[NB][NB + 1];
  __shared__ double Ts[NB][NB + 1];
  const int cell = blockIdx.y, J = blockIdx.x;
  const int j0 = J * NB, nbj = min(NB, k - j0);
  const int rows = j0 + NB;                 // Y rows held (block rows 0..J)
  const double* r = R + (int64_t)cell * cs;
  double* ri = Ri + (int64_t)cell * cs;
  double* rit = RiT + (int64_t)cell * cs;
  const int t = threadIdx.x;
  // diagonal block J (already inverted), zero-padded past k
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, c = e % NB;
    Ys[(j0 + i) * NB + c] = (i < nbj && c < nbj) ? ri[(int64_t)(j0 + i) * k + j0 + c] : 0.0;
  }
  const int tr = t / 8, tc = t % 8;         // T[tr][tc + 8q]
  for (int I = J - 1; I >= 0; --I) {
    const int i0 = I * NB;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int K = I + 1; K <= J; ++K) {
      const int m0 = K * NB;
      __syncthreads();
      for (int e = t; e < NB * NB; e += blockDim.x) {
        const int i = e / NB, m = e % NB;
        Rp[i][m] = (m0 + m < k) ? r[(int64_t)(i0 + i) * k + m0 + m] : 0.0;
      }
      __syncthreads();
#pragma unroll 8
      for (int m = 0; m < NB; ++m) {
        const double a = Rp[tr][m];
        const double* y = Ys + (m0 + m) * NB;
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = fma(a, y[tc + 8 * q], acc[q]);
      }
    }
    // Y[I][J] = -inv(R[I][I]) T, inv(R[I][I]) staged in Rp
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) Ts[tr][tc + 8 * q] = acc[q];
    for (int e = t; e < NB * NB; e += blockDim.x) {
      const int i = e / NB, m = e % NB;
      Rp[i][m] = ri[(int64_t)(i0 + i) * k + i0 + m];   // full block: i0 + NB <= j0 <= k
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = tc + 8 * q;
      double v = 0.0;
      for (int m = tr; m < NB; ++m) v = fma(Rp[tr][m], Ts[m][c], v);
      Ys[(i0 + tr) * NB + c] = -v;
    }
  }
  __syncthreads();
  // block column J of R^{-1} (rows below block J are zero) and rows of R^{-T}
  for (int e = t; e < k * NB; e += blockDim.x) {
    const int m = e / NB, c = e % NB;
    if (c >= nbj || (m >= j0 && m < rows)) continue;     // the diagonal block is in place
    ri[(int64_t)m * k + j0 + c] = (m < rows) ? Ys[m * NB + c] : 0.0;
  }
  for (int e = t; e < NB * k; e += blockDim.x) {
    const int c = e / k, m = e % k;
    if (c >= nbj) continue;
    rit[(int64_t)(j0 + c) * k + m] = (m < rows) ? Ys[m * NB + c] : 0.0;
  }
}

jolt_status launch_tri_inverse(const double* R, double* Ri, double* RiT, int64_t cs, int k, int ncells,
                               cudaStream_t s) {
  const int nbk = (k + NB - 1) / NB;
  const size_t smem = (size_t)nbk * NB * NB * sizeof(double);
  if (smem > 200 * 1024) { set_error("triangular inverse needs k <= 800 (k=%d)", k); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  static size_t set = 0;
  if (smem > set) {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_trinv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    set = smem;
  }
  k_trinv_diag<<<dim3(nbk, ncells), NB, 0, s>>>(R, Ri, RiT, cs, k);
  JOLT_LAUNCHED();
  k_trinv<<<dim3(nbk, ncells), 256, smem, s>>>(R, Ri, RiT, cs, k);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------- triangular products ------
// Rows x of X (one cell per blockIdx.z) as products with the inverse:
//   forward  (X R = B):    x_j = sum_{i <= j} b_i R^{-1}[i][j]
//   backward (X R^T = B):  x_j = sum_{i >= j} b_i R^{-T}[i][j]
// B: element (r, i) at B[r*ldb_r + i*ldb_c], fp32 or fp64 (b64 != 0).
// Outputs (either may be null): X64[r*ld64_r + j*ld64_c] fp64 and
// X16[r*ld16_r + j*ld16_c] bf16. 64 x 64 output tiles, 4 x 4 per thread on a
// stride-16 lattice; the tile is staged through shared memory so the stores
// run along whichever index is contiguous.

constexpr int AP_T = 64, AP_K = 16;

__global__ void __launch_bounds__(256) k_tri_apply(TrsmArgs a) {
  __shared__ double sm[AP_T * (AP_T + 1)];
  double* Bs = sm;                          // [AP_K][AP_T]   (i, r)
  double* Qs = sm + AP_K * AP_T;            // [AP_K][AP_T]   (i, j)
  const int cell = blockIdx.z;
  const int rows = a.rows_of ? a.rows_of[cell] : a.rows_fixed;
  const int r0 = blockIdx.x * AP_T, j0 = blockIdx.y * AP_T;
  if (r0 >= rows) return;
  const int k = a.k;
  if (j0 >= k) return;
  const double* Q = (a.backward ? a.RinvT : a.Rinv) + (int64_t)cell * a.r_cell;
  const int i_lo = a.backward ? (j0 / AP_K) * AP_K : 0;
  const int i_hi = a.backward ? k : min(k, j0 + AP_T);
  const int t = threadIdx.x, ty = t / 16, tx = t % 16;
  const bool b_rowmajor = a.ldb_c == 1;
  const int64_t boff = (int64_t)cell * a.b_cell;
  double acc[4][4] = {};
  for (int ib = i_lo; ib < i_hi; ib += AP_K) {
    __syncthreads();
#pragma unroll
    for (int u = 0; u < (AP_K * AP_T) / 256; ++u) {
      const int e = t + 256 * u;
      int ii, rr;
      if (b_rowmajor) { rr = e / AP_K; ii = e % AP_K; }
      else { ii = e / AP_T; rr = e % AP_T; }
      const int i = ib + ii, r = r0 + rr;
      double v = 0.0;
      if (i < k && r < rows) {
        const int64_t off = boff + (int64_t)r * a.ldb_r + (int64_t)i * a.ldb_c;
        v = a.b64 ? reinterpret_cast<const double*>(a.B)[off] : (double)reinterpret_cast<const float*>(a.B)[off];
      }
      Bs[ii * AP_T + rr] = v;
      const int qi = e / AP_T, qj = e % AP_T;
      const int iq = ib + qi, jq = j0 + qj;
      Qs[qi * AP_T + qj] = (iq < k && jq < k) ? Q[(int64_t)iq * k + jq] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int ii = 0; ii < AP_K; ++ii) {
      double x[4], y[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) { x[p] = Bs[ii * AP_T + ty + 16 * p]; y[p] = Qs[ii * AP_T + tx + 16 * p]; }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fma(x[p], y[q], acc[p][q]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) sm[(ty + 16 * p) * (AP_T + 1) + tx + 16 * q] = acc[p][q];
  __syncthreads();
  const bool trans = (a.X16 && a.ld16_r == 1) || (a.X64 && a.ld64_r == 1);
  for (int e = t; e < AP_T * AP_T; e += 256) {
    int rr, jj;
    if (trans) { jj = e / AP_T; rr = e % AP_T; }
    else { rr = e / AP_T; jj = e % AP_T; }
    const int r = r0 + rr, j = j0 + jj;
    if (r >= rows || j >= k) continue;
    const double v = sm[rr * (AP_T + 1) + jj];
    if (a.X64) a.X64[(int64_t)cell * a.x64_cell + (int64_t)r * a.ld64_r + (int64_t)j * a.ld64_c] = v;
    if (a.X16) a.X16[(int64_t)cell * a.x16_cell + (int64_t)r * a.ld16_r + (int64_t)j * a.ld16_c] = bf16_bits_from_f64(v);
  }
}

jolt_status launch_tri_apply(const TrsmArgs& a, int rows_max, int ncells, cudaStream_t s) {
  if (rows_max <= 0 || a.k <= 0) return JOLT_OK;
  dim3 g((rows_max + AP_T - 1) / AP_T, (a.k + AP_T - 1) / AP_T, ncells);
  k_tri_apply<<<g, 256, 0, s>>>(a);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
