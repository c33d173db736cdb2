#include <algorithm>
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

// ------------------------------------------------ fp64 tensor-core GEMM ----
// C[m][n] = sum_k A[m][k] B[k][n] per cell (blockIdx.z) on the fp64 tensor
// cores (mma.sync m8n8k4, fp64 in and out). Operands are strided views
// (fp32 or fp64): A[m][k] = a[cell*a_cell + m*a_lm + k*a_lk], likewise B.
// 64 x 64 output tiles, 4 warps of 32 x 32 (4 x 4 fragments), K in steps of
// 16 through two shared-memory stages (row pitch 68 doubles: the fragment
// loads of a warp hit distinct banks), the next stage fetched into registers
// while the current one is multiplied. K range per tile: all of K (kmode 0),
// k < n0 + 64 (kmode 1: C = B R^{-1} with R^{-1} upper), k >= n0 (kmode 2:
// C = B R^{-T}). sym: only tiles with n0 >= m0, each written to (m, n) and
// (n, m). The tile is staged through shared memory so the stores run along
// whichever output index is contiguous.
struct DgemmArgs {
  const void* A; int a64; int64_t a_cell, a_lm, a_lk;
  const void* B; int b64; int64_t b_cell, b_lk, b_ln;
  const int* M_of; int M_fixed;
  const int* K_of; int K_fixed;
  int N, kmode, sym;
  double* C64; int64_t c_cell, c_lm, c_ln;
  uint16_t* C16; int64_t h_cell, h_lm, h_ln;
  int ksplit, ncells;   // ksplit > 1: blockIdx.z = cell + ncells * slice, C64 holds one partial per slice
  int64_t part_stride;  // elements between slices' partials
};

constexpr int DG_T = 64, DG_K = 16, DG_P = 68;

__device__ __forceinline__ void dmma(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

__device__ __forceinline__ double ld_op(const void* p, int is64, int64_t off) {
  return is64 ? reinterpret_cast<const double*>(p)[off] : (double)reinterpret_cast<const float*>(p)[off];
}

__global__ void __launch_bounds__(128) k_dgemm(DgemmArgs g) {
  __shared__ __align__(16) double sm[2 * 2 * DG_K * DG_P];   // [stage][A|B][k][m|n]; reused for the tile
  const int cell = (int)(blockIdx.z % g.ncells), slice = (int)(blockIdx.z / g.ncells);
  int m0, n0;
  if (g.sym) {
    int b = blockIdx.x, ti = 0;
    const int nt = (g.N + DG_T - 1) / DG_T;
    while (ti < nt && b >= nt - ti) { b -= nt - ti; ++ti; }
    if (ti >= nt) return;
    m0 = ti * DG_T;
    n0 = (ti + b) * DG_T;
  } else {
    m0 = blockIdx.x * DG_T;
    n0 = blockIdx.y * DG_T;
  }
  const int M = g.M_of ? g.M_of[cell] : g.M_fixed;
  const int K = g.K_of ? g.K_of[cell] : g.K_fixed;
  if (m0 >= M || n0 >= g.N) return;
  int k_lo = 0, k_hi = K;
  if (g.kmode == 1) k_hi = min(K, n0 + DG_T);
  if (g.kmode == 2) k_lo = (n0 / DG_K) * DG_K;
  if (g.ksplit > 1) {        // this block's slice of K, in whole steps of DG_K
    const int steps = (k_hi - k_lo + DG_K - 1) / DG_K;
    const int per = (steps + g.ksplit - 1) / g.ksplit;
    const int s0 = k_lo + slice * per * DG_K;
    k_hi = min(k_hi, s0 + per * DG_K);
    k_lo = s0;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
  const int gq = lane >> 2, tq = lane & 3;          // fragment row / column group
  const void* A = g.A;
  const void* B = g.B;
  const int64_t aoff = (int64_t)cell * g.a_cell, boff = (int64_t)cell * g.b_cell;
  const bool a_m_fast = g.a_lm == 1, b_n_fast = g.b_ln == 1;
  double ra[8], rb[8];
  auto fetch = [&](int kb) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = tid + 128 * u;
      int mm, kk;
      if (a_m_fast) { mm = e % DG_T; kk = e / DG_T; } else { kk = e % DG_K; mm = e / DG_K; }
      const int gm = m0 + mm, gk = kb + kk;
      ra[u] = (gm < M && gk < k_hi) ? ld_op(A, g.a64, aoff + (int64_t)gm * g.a_lm + (int64_t)gk * g.a_lk) : 0.0;
      int nn, k2;
      if (b_n_fast) { nn = e % DG_T; k2 = e / DG_T; } else { k2 = e % DG_K; nn = e / DG_K; }
      const int gn = n0 + nn, gk2 = kb + k2;
      rb[u] = (gn < g.N && gk2 < k_hi) ? ld_op(B, g.b64, boff + (int64_t)gk2 * g.b_lk + (int64_t)gn * g.b_ln) : 0.0;
    }
  };
  auto stash = [&](int st) {
    double* As = sm + st * 2 * DG_K * DG_P;
    double* Bs = As + DG_K * DG_P;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = tid + 128 * u;
      int mm, kk;
      if (a_m_fast) { mm = e % DG_T; kk = e / DG_T; } else { kk = e % DG_K; mm = e / DG_K; }
      As[kk * DG_P + mm] = ra[u];
      int nn, k2;
      if (b_n_fast) { nn = e % DG_T; k2 = e / DG_T; } else { k2 = e % DG_K; nn = e / DG_K; }
      Bs[k2 * DG_P + nn] = rb[u];
    }
  };
  double c[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) c[i][j][0] = c[i][j][1] = 0.0;
  int st = 0;
  if (k_lo < k_hi) {
    fetch(k_lo);
    stash(0);
  }
  __syncthreads();
  for (int kb = k_lo; kb < k_hi; kb += DG_K) {
    const bool more = kb + DG_K < k_hi;
    if (more) fetch(kb + DG_K);
    const double* As = sm + st * 2 * DG_K * DG_P;
    const double* Bs = As + DG_K * DG_P;
#pragma unroll
    for (int ks = 0; ks < DG_K / 4; ++ks) {
      double a[4], b[4];
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        a[f] = As[(ks * 4 + tq) * DG_P + wm + f * 8 + gq];
        b[f] = Bs[(ks * 4 + tq) * DG_P + wn + f * 8 + gq];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma(c[i][j][0], c[i][j][1], a[i], b[j]);
    }
    if (more) stash(st ^ 1);
    __syncthreads();
    st ^= 1;
  }
  // tile -> shared memory [m][n] (pitch 65), then strided stores
  double* Ts = sm;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int v = 0; v < 2; ++v) Ts[(wm + i * 8 + gq) * (DG_T + 1) + wn + j * 8 + 2 * tq + v] = c[i][j][v];
  __syncthreads();
  double* c64 = g.C64 ? g.C64 + (int64_t)slice * g.part_stride : nullptr;
  auto store = [&](int r, int q, double v) {
    if (c64) c64[(int64_t)cell * g.c_cell + (int64_t)r * g.c_lm + (int64_t)q * g.c_ln] = v;
    if (g.C16) g.C16[(int64_t)cell * g.h_cell + (int64_t)r * g.h_lm + (int64_t)q * g.h_ln] = bf16_bits_from_f64(v);
  };
  const bool m_fast = (g.C64 ? g.c_lm : g.h_lm) == 1;
  for (int e = tid; e < DG_T * DG_T; e += 128) {
    int mm, nn;
    if (m_fast) { nn = e / DG_T; mm = e % DG_T; } else { mm = e / DG_T; nn = e % DG_T; }
    const int r = m0 + mm, q = n0 + nn;
    if (r >= M || q >= g.N) continue;
    const double v = Ts[mm * (DG_T + 1) + nn];
    store(r, q, v);
    if (g.sym && r != q) store(q, r, v);
  }
}

// ---------------------------------------------------------------------------
// The same product with a deeper operand pipeline: 16-byte cp.async copies
// (no register staging) into PS stages of shared memory that keep each
// operand in its own type (fp32 or fp64; fp32 values are widened when the
// fragments are read, which is exact), so several K steps of loads are in
// flight while the fp64 tensor cores work. Used when every 16-byte chunk of
// the operands' contiguous dimension is aligned (A contiguous along m or
// along k, B along n); the register-staged kernel above covers the rest.
// Tile, warps, fragment order and the K order of the sums are those of
// k_dgemm, so both give the same result bit for bit.
constexpr int PS = 4;            // pipeline stages
template <class AT, class BT, bool AMF>
struct DgPipe {
  // A stage: AMF ? [DG_K][DG_T + pad] : [DG_T][DG_K + pad]; B stage: [DG_K][DG_T + pad].
  // Row pitches of 72 (along m or n) or 20 (along k) elements put the
  // fragment reads of a (half-)warp on distinct banks, and keep every row a
  // whole number of 16-byte chunks.
  static constexpr int APAD = AMF ? 8 : 4;
  static constexpr int A_ELEMS = AMF ? DG_K * (DG_T + APAD) : DG_T * (DG_K + APAD);
  static constexpr int BPAD = 8;
  static constexpr int B_ELEMS = DG_K * (DG_T + BPAD);
  static constexpr int A_BYTES = (A_ELEMS * (int)sizeof(AT) + 15) / 16 * 16;
  static constexpr int B_BYTES = (B_ELEMS * (int)sizeof(BT) + 15) / 16 * 16;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SMEM = PS * STAGE;
};

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <class AT, class BT, bool AMF>
__global__ void __launch_bounds__(128) k_dgemm_pipe(DgemmArgs g) {
  using P = DgPipe<AT, BT, AMF>;
  extern __shared__ __align__(16) uint8_t dsm[];
  const int cell = (int)(blockIdx.z % g.ncells), slice = (int)(blockIdx.z / g.ncells);
  int m0, n0;
  if (g.sym) {
    int b = blockIdx.x, ti = 0;
    const int nt = (g.N + DG_T - 1) / DG_T;
    while (ti < nt && b >= nt - ti) { b -= nt - ti; ++ti; }
    if (ti >= nt) return;
    m0 = ti * DG_T;
    n0 = (ti + b) * DG_T;
  } else {
    m0 = blockIdx.x * DG_T;
    n0 = blockIdx.y * DG_T;
  }
  const int M = g.M_of ? g.M_of[cell] : g.M_fixed;
  const int K = g.K_of ? g.K_of[cell] : g.K_fixed;
  if (m0 >= M || n0 >= g.N) return;
  int k_lo = 0, k_hi = K;
  if (g.kmode == 1) k_hi = min(K, n0 + DG_T);
  if (g.kmode == 2) k_lo = (n0 / DG_K) * DG_K;
  if (g.ksplit > 1) {
    const int steps = (k_hi - k_lo + DG_K - 1) / DG_K;
    const int per = (steps + g.ksplit - 1) / g.ksplit;
    const int s0 = k_lo + slice * per * DG_K;
    k_hi = min(k_hi, s0 + per * DG_K);
    k_lo = s0;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
  const int gq = lane >> 2, tq = lane & 3;
  const AT* A = reinterpret_cast<const AT*>(g.A) + (int64_t)cell * g.a_cell;
  const BT* B = reinterpret_cast<const BT*>(g.B) + (int64_t)cell * g.b_cell;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(dsm);
  constexpr int AV = 16 / (int)sizeof(AT), BV = 16 / (int)sizeof(BT);   // elements per 16-byte chunk
  auto load_stage = [&](int st, int kb) {
    const uint32_t sa = sbase + st * P::STAGE, sb = sa + P::A_BYTES;
    if (AMF) {        // A(m, k) contiguous along m: chunks of AV m-values per k row
      constexpr int CH = DG_T / AV;
      for (int c = tid; c < DG_K * CH; c += 128) {
        const int kk = c / CH, mm = (c % CH) * AV;
        const int gm = m0 + mm, gk = kb + kk;
        int valid = (gk < k_hi) ? min(AV, M - gm) : 0;
        if (valid < 0) valid = 0;
        const AT* src = A + (valid ? (int64_t)gk * g.a_lk + gm : 0);
        cp16(sa + (kk * (DG_T + P::APAD) + mm) * (int)sizeof(AT), src, valid * (int)sizeof(AT));
      }
    } else {          // A(m, k) contiguous along k: chunks of AV k-values per m row
      constexpr int CH = DG_K / AV;
      for (int c = tid; c < DG_T * CH; c += 128) {
        const int mm = c / CH, kk = (c % CH) * AV;
        const int gm = m0 + mm, gk = kb + kk;
        int valid = (gm < M) ? min(AV, k_hi - gk) : 0;
        if (valid < 0) valid = 0;
        const AT* src = A + (valid ? (int64_t)gm * g.a_lm + gk : 0);
        cp16(sa + (mm * (DG_K + P::APAD) + kk) * (int)sizeof(AT), src, valid * (int)sizeof(AT));
      }
    }
    {                 // B(k, n) contiguous along n
      constexpr int CH = DG_T / BV;
      for (int c = tid; c < DG_K * CH; c += 128) {
        const int kk = c / CH, nn = (c % CH) * BV;
        const int gn = n0 + nn, gk = kb + kk;
        int valid = (gk < k_hi) ? min(BV, g.N - gn) : 0;
        if (valid < 0) valid = 0;
        const BT* src = B + (valid ? (int64_t)gk * g.b_lk + gn : 0);
        cp16(sb + (kk * (DG_T + P::BPAD) + nn) * (int)sizeof(BT), src, valid * (int)sizeof(BT));
      }
    }
  };
  double c[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) c[i][j][0] = c[i][j][1] = 0.0;
  const int nsteps = (k_hi > k_lo) ? (k_hi - k_lo + DG_K - 1) / DG_K : 0;
#pragma unroll
  for (int st = 0; st < PS - 1; ++st) {
    if (st < nsteps) load_stage(st, k_lo + st * DG_K);
    cp_commit();
  }
  for (int it = 0; it < nsteps; ++it) {
    cp_wait<PS - 2>();
    __syncthreads();
    // refill the stage consumed PS - 1 steps ago (every thread is past it)
    const int nxt = it + PS - 1;
    if (nxt < nsteps) load_stage(nxt % PS, k_lo + nxt * DG_K);
    cp_commit();
    const uint8_t* stg = dsm + (it % PS) * P::STAGE;
    const AT* As = reinterpret_cast<const AT*>(stg);
    const BT* Bs = reinterpret_cast<const BT*>(stg + P::A_BYTES);
#pragma unroll
    for (int ks = 0; ks < DG_K / 4; ++ks) {
      double av[4], bv[4];
      const int kk = ks * 4 + tq;
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        const int mm = wm + f * 8 + gq, nn = wn + f * 8 + gq;
        av[f] = AMF ? (double)As[kk * (DG_T + P::APAD) + mm] : (double)As[mm * (DG_K + P::APAD) + kk];
        bv[f] = (double)Bs[kk * (DG_T + P::BPAD) + nn];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma(c[i][j][0], c[i][j][1], av[i], bv[j]);
    }
  }
  cp_wait<0>();
  __syncthreads();
  double* Ts = reinterpret_cast<double*>(dsm);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int v = 0; v < 2; ++v) Ts[(wm + i * 8 + gq) * (DG_T + 1) + wn + j * 8 + 2 * tq + v] = c[i][j][v];
  __syncthreads();
  double* c64 = g.C64 ? g.C64 + (int64_t)slice * g.part_stride : nullptr;
  auto store = [&](int r, int q, double v) {
    if (c64) c64[(int64_t)cell * g.c_cell + (int64_t)r * g.c_lm + (int64_t)q * g.c_ln] = v;
    if (g.C16) g.C16[(int64_t)cell * g.h_cell + (int64_t)r * g.h_lm + (int64_t)q * g.h_ln] = bf16_bits_from_f64(v);
  };
  const bool m_fast = (g.C64 ? g.c_lm : g.h_lm) == 1;
  for (int e = tid; e < DG_T * DG_T; e += 128) {
    int mm, nn;
    if (m_fast) { nn = e / DG_T; mm = e % DG_T; } else { mm = e / DG_T; nn = e % DG_T; }
    const int r = m0 + mm, q = n0 + nn;
    if (r >= M || q >= g.N) continue;
    const double v = Ts[mm * (DG_T + 1) + nn];
    store(r, q, v);
    if (g.sym && r != q) store(q, r, v);
  }
}

template <class AT, class BT, bool AMF>
static jolt_status launch_pipe(const DgemmArgs& g, dim3 grid, cudaStream_t s) {
  using P = DgPipe<AT, BT, AMF>;
  const int smem = std::max(P::SMEM, DG_T * (DG_T + 1) * 8);
  static bool attr = false;
  if (!attr) {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_dgemm_pipe<AT, BT, AMF>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    attr = true;
  }
  k_dgemm_pipe<AT, BT, AMF><<<grid, 128, smem, s>>>(g);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

static jolt_status launch_dgemm(DgemmArgs g, int M_max, int ncells, cudaStream_t s) {
  if (M_max <= 0 || g.N <= 0 || ncells <= 0) return JOLT_OK;
  if (g.ksplit < 1) g.ksplit = 1;
  {
    // the pipelined kernel needs 16-byte chunks along A's and B's contiguous
    // dimensions: unit strides there, and bases and other strides that are
    // whole 16-byte multiples
    const int ea = g.a64 ? 8 : 4, eb = g.b64 ? 8 : 4;
    const bool amf = g.a_lm == 1, akf = g.a_lk == 1;
    const int64_t a_other = amf ? g.a_lk : g.a_lm;
    const bool a_ok = (amf || akf) && ((a_other * ea) % 16 == 0) && ((g.a_cell * ea) % 16 == 0) &&
                      (reinterpret_cast<uintptr_t>(g.A) % 16 == 0);
    const bool b_ok = g.b_ln == 1 && ((g.b_lk * eb) % 16 == 0) && ((g.b_cell * eb) % 16 == 0) &&
                      (reinterpret_cast<uintptr_t>(g.B) % 16 == 0);
    if (a_ok && b_ok) {
      g.ncells = ncells;
      const int mt = (M_max + DG_T - 1) / DG_T, nt = (g.N + DG_T - 1) / DG_T;
      dim3 grid = g.sym ? dim3(nt * (nt + 1) / 2, 1, ncells * g.ksplit) : dim3(mt, nt, ncells * g.ksplit);
      if (!g.a64 && !g.b64) return amf ? launch_pipe<float, float, true>(g, grid, s) : launch_pipe<float, float, false>(g, grid, s);
      if (!g.a64 && g.b64) return amf ? launch_pipe<float, double, true>(g, grid, s) : launch_pipe<float, double, false>(g, grid, s);
      if (g.a64 && g.b64) return amf ? launch_pipe<double, double, true>(g, grid, s) : launch_pipe<double, double, false>(g, grid, s);
    }
  }
  g.ncells = ncells;
  const int mt = (M_max + DG_T - 1) / DG_T, nt = (g.N + DG_T - 1) / DG_T;
  dim3 grid = g.sym ? dim3(nt * (nt + 1) / 2, 1, ncells * g.ksplit) : dim3(mt, nt, ncells * g.ksplit);
  k_dgemm<<<grid, 128, 0, s>>>(g);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// C[e] = sum over slices of part[slice][e], slices in order (deterministic).
__global__ void k_sum_slices(const double* __restrict__ part, int64_t stride, int nslices, int64_t n,
                             double* __restrict__ C) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    double acc = part[e];
    for (int sl = 1; sl < nslices; ++sl) acc += part[(int64_t)sl * stride + e];
    C[e] = acc;
  }
}

// Rows x of X (one cell per blockIdx.z) as products with the inverse:
//   forward  (X R = B):    x_j = sum_{i <= j} b_i R^{-1}[i][j]
//   backward (X R^T = B):  x_j = sum_{i >= j} b_i R^{-T}[i][j]
// B: element (r, i) at B[r*ldb_r + i*ldb_c], fp32 or fp64 (b64 != 0).
// Outputs (either may be null): X64[r*ld64_r + j*ld64_c] fp64 and
// X16[r*ld16_r + j*ld16_c] bf16.
jolt_status launch_tri_apply(const TrsmArgs& a, int rows_max, int ncells, cudaStream_t s) {
  DgemmArgs g{};
  g.A = a.B; g.a64 = a.b64; g.a_cell = a.b_cell; g.a_lm = a.ldb_r; g.a_lk = a.ldb_c;
  g.B = a.backward ? a.RinvT : a.Rinv; g.b64 = 1; g.b_cell = a.r_cell; g.b_lk = a.k; g.b_ln = 1;
  g.M_of = a.rows_of; g.M_fixed = a.rows_fixed;
  g.K_of = nullptr; g.K_fixed = a.k;
  g.N = a.k; g.kmode = a.backward ? 2 : 1; g.sym = 0;
  g.C64 = a.X64; g.c_cell = a.x64_cell; g.c_lm = a.ld64_r; g.c_ln = a.ld64_c;
  g.C16 = a.X16; g.h_cell = a.x16_cell; g.h_lm = a.ld16_r; g.h_ln = a.ld16_c;
  return launch_dgemm(g, rows_max, ncells, s);
}

// C = A^T A for A = [rows_of[cell]] x k fp32 (row-major, cell stride a_cell),
// C k x k fp64 (cell stride c_cell), exactly symmetric. The long K (rows) is
// split into GRAM_SPLIT slices whose partial Grams go to `part`
// (GRAM_SPLIT * ncells * c_cell doubles) and are then added in order.
jolt_status launch_gram_cols(const float* A, int64_t a_cell, const int* rows_of, int k, double* C, int64_t c_cell,
                             int ncells, double* part, cudaStream_t s) {
  DgemmArgs g{};
  g.A = A; g.a64 = 0; g.a_cell = a_cell; g.a_lm = 1; g.a_lk = k;
  g.B = A; g.b64 = 0; g.b_cell = a_cell; g.b_lk = k; g.b_ln = 1;
  g.M_of = nullptr; g.M_fixed = k;
  g.K_of = rows_of; g.K_fixed = 0;
  g.N = k; g.kmode = 0; g.sym = 1;
  g.c_cell = c_cell; g.c_lm = k; g.c_ln = 1;
  g.C16 = nullptr;
  if (!part) {
    g.C64 = C;
    return launch_dgemm(g, k, ncells, s);
  }
  g.C64 = part; g.ksplit = GRAM_SPLIT; g.part_stride = (int64_t)ncells * c_cell;
  JOLT_TRY(launch_dgemm(g, k, ncells, s));
  const int64_t n = (int64_t)ncells * c_cell;
  k_sum_slices<<<(int)std::min<int64_t>((n + 255) / 256, 148 * 8), 256, 0, s>>>(part, g.part_stride, GRAM_SPLIT, n, C);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
