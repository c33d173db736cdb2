// fp64 Gram matrices and the batched symmetric eigensolver.
//
// Section 3 of "A JoLT for the KV Cache" ("Partial Tucker backbone") needs the
// mode-k singular values and vectors of the token unfolding X_(T) (T x N,
// N = L_g H D) and of the feature unfolding X_(d) (D x L_g H T). They are
// the eigenpairs of the Gram matrices X_(T) X_(T)^T (or X_(T)^T X_(T) when
// T > N) and X_(d) X_(d)^T, formed here in fp64 from the fp32 cell values.
#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {

// ------------------------------------------------------------ reductions ---
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the block; every thread gets the result. `red` >= 32 doubles.
__device__ double block_sum(double v, double* red) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  for (int i = 0; i < nw; ++i) s += red[i];   // fixed order
  return s;
}

// ---------------------------------------------------- feature Gram (fp64) --
// partial[(cell*nchunk + chunk)*(D*D+1) + i*D + j] = sum over the chunk's rows
// of x_i x_j; entry D*D holds the chunk's sum of squares. Rows are (l, h, t).
template <int D>
__global__ void __launch_bounds__(256) k_fgram_x(const CellDesc* __restrict__ cells,
                                                 const float2* __restrict__ cs, int nchunk,
                                                 double* __restrict__ partial) {
  constexpr int RB = 32;               // rows per smem tile
  constexpr int P = D / 16;            // outputs per thread per dim
  __shared__ double xs[RB][D];
  __shared__ double red[32];
  const CellDesc c = cells[blockIdx.y];
  const int64_t rows = (int64_t)c.Lg * c.H * c.T;
  const int64_t per = (rows + nchunk - 1) / nchunk;
  const int64_t r0 = blockIdx.x * per;
  const int64_t r1 = min(rows, r0 + per);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[P][P];
#pragma unroll
  for (int i = 0; i < P; ++i)
#pragma unroll
    for (int j = 0; j < P; ++j) acc[i][j] = 0.0;
  double sq = 0.0;
  for (int64_t rb = r0; rb < r1; rb += RB) {
    for (int e = threadIdx.x; e < RB * D; e += blockDim.x) {
      int rr = e / D, d = e % D;
      int64_t r = rb + rr;
      double val = 0.0;
      if (r < r1) {
        int t = (int)(r % c.T);
        int lh = (int)(r / c.T);
        val = (double)x_elem(c, cs, lh / c.H, lh % c.H, t, d);
      }
      xs[rr][d] = val;
      sq += val * val;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < RB; ++k) {
      double a[P], b[P];
#pragma unroll
      for (int i = 0; i < P; ++i) a[i] = xs[k][ty * P + i];
#pragma unroll
      for (int j = 0; j < P; ++j) b[j] = xs[k][tx * P + j];
#pragma unroll
      for (int i = 0; i < P; ++i)
#pragma unroll
        for (int j = 0; j < P; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double* out = partial + ((int64_t)blockIdx.y * nchunk + blockIdx.x) * (D * D + 1);
#pragma unroll
  for (int i = 0; i < P; ++i)
#pragma unroll
    for (int j = 0; j < P; ++j) out[(ty * P + i) * D + tx * P + j] = acc[i][j];
  double s = block_sum(sq, red);
  if (threadIdx.x == 0) out[D * D] = s;
}

// Same for rows of an fp64 matrix set: rows of Y[cell] = [L_g H][rmax][D],
// only r < r_t(cell) counted.
template <int D>
__global__ void __launch_bounds__(256) k_fgram_rows(const double* const* __restrict__ Y,
                                                    const int* __restrict__ nrow_used,
                                                    const int* __restrict__ rmax_of, const int* __restrict__ nlh_of,
                                                    int nchunk, double* __restrict__ partial) {
  constexpr int RB = 32;
  constexpr int P = D / 16;
  __shared__ double xs[RB][D];
  const int cell = blockIdx.y;
  const double* src = Y[cell];
  const int rmax = rmax_of[cell], ru = nrow_used[cell], nlh = nlh_of[cell];
  const int64_t rows = (int64_t)nlh * rmax;
  const int64_t per = (rows + nchunk - 1) / nchunk;
  const int64_t r0 = blockIdx.x * per;
  const int64_t r1 = min(rows, r0 + per);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[P][P];
#pragma unroll
  for (int i = 0; i < P; ++i)
#pragma unroll
    for (int j = 0; j < P; ++j) acc[i][j] = 0.0;
  for (int64_t rb = r0; rb < r1; rb += RB) {
    for (int e = threadIdx.x; e < RB * D; e += blockDim.x) {
      int rr = e / D, d = e % D;
      int64_t r = rb + rr;
      double val = 0.0;
      if (r < r1 && (int)(r % rmax) < ru) val = src[r * D + d];
      xs[rr][d] = val;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < RB; ++k) {
      double a[P], b[P];
#pragma unroll
      for (int i = 0; i < P; ++i) a[i] = xs[k][ty * P + i];
#pragma unroll
      for (int j = 0; j < P; ++j) b[j] = xs[k][tx * P + j];
#pragma unroll
      for (int i = 0; i < P; ++i)
#pragma unroll
        for (int j = 0; j < P; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double* out = partial + ((int64_t)cell * nchunk + blockIdx.x) * (D * D + 1);
#pragma unroll
  for (int i = 0; i < P; ++i)
#pragma unroll
    for (int j = 0; j < P; ++j) out[(ty * P + i) * D + tx * P + j] = acc[i][j];
  if (threadIdx.x == 0) out[D * D] = 0.0;
}

// out[cell][k] = sum over chunks (in chunk order) of partial[cell][chunk][k]
__global__ void k_sum_chunks(const double* __restrict__ partial, int nchunk, int len,
                             double* const* __restrict__ out, double* const* __restrict__ out_last) {
  const int cell = blockIdx.y;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < len; k += gridDim.x * blockDim.x) {
    double s = 0.0;
    for (int ch = 0; ch < nchunk; ++ch) s += partial[((int64_t)cell * nchunk + ch) * len + k];
    if (k < len - 1) out[cell][k] = s;
    else if (out_last) *out_last[cell] = s;
  }
}

// ------------------------------------------------------ token Gram (fp64) --
// Small side Gram of X_(T): if T <= N, G[t1][t2] = sum_n x(t1,n) x(t2,n);
// else G[n1][n2] = sum_t x(t,n1) x(t,n2). n = (l*H + h)*D + d.
__global__ void __launch_bounds__(256) k_token_gram(const CellDesc* __restrict__ cells,
                                                    const float2* __restrict__ cs,
                                                    double* const* __restrict__ G) {
  constexpr int TB = 64, KB = 16;
  __shared__ double As[KB][TB + 1];
  __shared__ double Bs[KB][TB + 1];
  const CellDesc c = cells[blockIdx.y];
  const int N = c.Lg * c.H * c.D;
  const bool tside = c.T <= N;
  const int n = tside ? c.T : N;
  const int K = tside ? N : c.T;
  const int nt = (n + TB - 1) / TB;
  // upper-triangular tile (ti <= tj) from the linear block index
  int b = blockIdx.x, ti = 0;
  while (ti < nt && b >= nt - ti) { b -= nt - ti; ++ti; }
  if (ti >= nt) return;
  const int tj = ti + b;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int k0 = 0; k0 < K; k0 += KB) {
    for (int e = threadIdx.x; e < KB * TB; e += blockDim.x) {
      int kk = e / TB, ii = e % TB;
      int k = k0 + kk;
      int ia = ti * TB + ii, ib = tj * TB + ii;
      double va = 0.0, vb = 0.0;
      if (k < K) {
        if (tside) {
          int lh = k / c.D, d = k % c.D;
          if (ia < n) va = x_elem(c, cs, lh / c.H, lh % c.H, ia, d);
          if (ib < n) vb = x_elem(c, cs, lh / c.H, lh % c.H, ib, d);
        } else {
          if (ia < n) { int lh = ia / c.D; va = x_elem(c, cs, lh / c.H, lh % c.H, k, ia % c.D); }
          if (ib < n) { int lh = ib / c.D; vb = x_elem(c, cs, lh / c.H, lh % c.H, k, ib % c.D); }
        }
      }
      As[kk][ii] = va;
      Bs[kk][ii] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KB; ++kk) {
      double a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
  double* g = G[blockIdx.y];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int r = ti * TB + ty * 4 + i, q = tj * TB + tx * 4 + j;
      if (r < n && q < n) {
        g[(int64_t)r * n + q] = acc[i][j];
        g[(int64_t)q * n + r] = acc[i][j];
      }
    }
}

// ------------------------------------------------------------ eigensolver --
// One thread block per symmetric matrix A (n x n, row-major, destroyed):
//  1. Householder reduction to tridiagonal form, A = Q T Q^T,
//     Q = H_0 H_1 ... H_{n-3}, H_k = I - beta_k v_k v_k^T on rows k+1..n-1;
//  2. implicit QL iterations with Wilkinson-type shifts on T; one thread
//     computes each sweep's plane rotations and the whole block applies them
//     to the eigenvector matrix, each thread owning rows;
//  3. back-transformation z <- H_k z for k = n-3 .. 0;
//  4. eigenvalues sorted descending, each eigenvector's largest-magnitude
//     entry made positive (first on ties).
// Outputs: w[n]; Vt[j*n + i] = component i of eigenvector j (if want_vec).
constexpr int EIG_THREADS = 512;

// ------------------------------------------- split eigensolver (big n) -----
// For the token-mode matrices only the spectrum is needed before the
// allocation and only the leading r_T eigenvectors after it, so the solver is
// split: (1) Householder tridiagonalization, leaving reflector k in row k of
// A (entries k+1 .. n-1) and d, e, beta in work[0..3n); (2) every eigenvalue
// by bisection on Sturm counts, one thread per eigenvalue; (3) after the
// allocation, eigenvectors of the leading r eigenvalues by inverse iteration
// on the tridiagonal matrix (one thread per vector), then the
// back-transformation by the reflectors (a block per group of vectors).

__global__ void __launch_bounds__(EIG_THREADS) k_tridiag(const EighJob* __restrict__ jobs) {
  const EighJob J = jobs[blockIdx.x];
  const int n = J.n;
  if (n <= 0) return;
  extern __shared__ double sh[];
  double* v = sh;            // n
  double* p = v + n;         // n
  double* red = p + n;       // 32
  double* A = J.A;
  double* dd = J.work;
  double* ee = dd + n;
  double* tau = ee + n;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarp = nt >> 5;
  for (int k = 0; k + 2 < n; ++k) {
    const int m = n - k - 1;
    for (int i = tid; i < m; i += nt) v[i] = A[(int64_t)k * n + (k + 1 + i)];   // row k = column k
    __syncthreads();
    double s = 0.0;
    for (int i = 1 + tid; i < m; i += nt) s += v[i] * v[i];
    s = block_sum(s, red);
    const double x0 = v[0];
    if (s == 0.0) {
      if (tid == 0) { dd[k] = A[(int64_t)k * n + k]; ee[k] = x0; tau[k] = 0.0; }
      __syncthreads();
      continue;
    }
    const double nrm = sqrt(x0 * x0 + s);
    const double alpha = (x0 <= 0.0) ? nrm : -nrm;
    const double v0 = x0 - alpha;
    const double beta = 2.0 / (s + v0 * v0);
    __syncthreads();
    if (tid == 0) v[0] = v0;
    __syncthreads();
    for (int i = warp; i < m; i += nwarp) {
      const double* row = A + (int64_t)(k + 1 + i) * n + (k + 1);
      double acc = 0.0;
      for (int j = lane; j < m; j += 32) acc += row[j] * v[j];
      acc = warp_sum(acc);
      if (lane == 0) p[i] = beta * acc;
    }
    __syncthreads();
    double pv = 0.0;
    for (int i = tid; i < m; i += nt) pv += p[i] * v[i];
    const double Kc = 0.5 * beta * block_sum(pv, red);
    for (int i = tid; i < m; i += nt) p[i] -= Kc * v[i];
    __syncthreads();
    for (int i = warp; i < m; i += nwarp) {
      double* row = A + (int64_t)(k + 1 + i) * n + (k + 1);
      const double vi = v[i], wi = p[i];
      for (int j = lane; j < m; j += 32) row[j] = __dsub_rn(row[j], __dadd_rn(__dmul_rn(vi, p[j]), __dmul_rn(wi, v[j])));   // exactly symmetric
    }
    if (tid == 0) { dd[k] = A[(int64_t)k * n + k]; ee[k] = alpha; tau[k] = beta; }
    for (int i = tid; i < m; i += nt) A[(int64_t)k * n + (k + 1 + i)] = v[i];   // reflector k in row k
    __syncthreads();
  }
  if (tid == 0) {
    if (n >= 2) {
      dd[n - 2] = A[(int64_t)(n - 2) * n + (n - 2)];
      ee[n - 2] = A[(int64_t)(n - 1) * n + (n - 2)];
      tau[n - 2] = 0.0;
    }
    dd[n - 1] = A[(int64_t)(n - 1) * n + (n - 1)];
    ee[n - 1] = 0.0;
    tau[n - 1] = 0.0;
  }
}

// The same reduction with G thread blocks per matrix (one cooperative launch
// over all jobs). Row r of the trailing matrix belongs to warp r mod (G x
// warps per block) for the whole reduction. At column k every block computes
// the reflector itself from row k (A is kept exactly symmetric, so row k
// equals column k), forms p = beta A v for its own rows and publishes them;
// after a job-wide barrier each block rebuilds w = p - (beta/2)(p.v) v from
// all shares (partial sums added in block order, so every block gets the
// same bits) and applies the rank-2 update to its own rows. The owner of row
// k+1 updates it first and publishes it with a per-job flag; the next column
// waits for that flag only, not for every block (its other reads are the
// block's own rows). p and the partial sums alternate between two buffers by
// column parity. A is read through L2 only. Barriers and flags are bounded
// waits: on expiry the block raises the job's abort flag and the timeout
// status and returns, and the others follow at their next wait.
__device__ __forceinline__ unsigned long long gtimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ bool job_barrier(unsigned int* cnt, unsigned int target, volatile int* abort_flag, int* status) {
  __shared__ int ok_s;
  __syncthreads();          // the block's writes of A, p and the partial sums ...
  if (threadIdx.x == 0) {
    __threadfence();        // ... are ordered before the arrival by this fence (cumulative)
    atomicAdd(cnt, 1u);
    int ok = 1;
    const unsigned long long t0 = gtimer_ns();
    while (true) {
      unsigned int c;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(cnt) : "memory");
      if (c >= target) break;
      if (*abort_flag) { ok = 0; break; }
      if (gtimer_ns() - t0 > 2000000000ull) {
        *abort_flag = 1;
        atomicOr(status, DEV_ERR_TIMEOUT);
        ok = 0;
        break;
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// Bounded wait until the job's published-row flag reaches `target`.
__device__ bool wait_flag(volatile unsigned int* flag, unsigned int target, volatile int* abort_flag, int* status) {
  __shared__ int ok_f;
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned long long t0 = gtimer_ns();
    while (true) {
      unsigned int f;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(f) : "l"(flag) : "memory");
      if (f >= target) break;
      if (*abort_flag) { ok = 0; break; }
      if (gtimer_ns() - t0 > 2000000000ull) {
        *abort_flag = 1;
        atomicOr(status, DEV_ERR_TIMEOUT);
        ok = 0;
        break;
      }
    }
    ok_f = ok;
  }
  __syncthreads();
  return ok_f != 0;
}

__device__ __forceinline__ void publish_flag(unsigned int* flag, unsigned int value) {
  __threadfence();
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(value) : "memory");
}

__global__ void __launch_bounds__(EIG_THREADS) k_tridiag_multi(const EighJob* __restrict__ jobs, int G, int nmax,
                                                               double* __restrict__ scratch,
                                                               unsigned int* __restrict__ counters, int* status) {
  const int njobs = gridDim.x / G;
  const int job = blockIdx.x / G, c = blockIdx.x % G;
  const EighJob J = jobs[job];
  const int n = J.n;
  if (n <= 0) return;
  extern __shared__ double sh[];
  double* v = sh;            // n
  double* w = v + n;         // n
  double* red = w + n;       // 32
  double* A = J.A;
  double* dd = J.work;
  double* ee = dd + n;
  double* tau = ee + n;
  double* Pb = scratch + (size_t)job * (2 * nmax + 128);   // p[2][nmax], then partial sums [2][64]
  unsigned int* cnt = counters + job;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(counters + njobs);
  unsigned int* flag = counters + njobs + 1 + job;          // rows published: row k is final when flag >= k
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarp = nt >> 5;
  const int gw = c * nwarp + warp, GW = G * nwarp;
  unsigned int nbar = 0;
  for (int k = 0; k + 2 < n; ++k) {
    const int m = n - k - 1, buf = k & 1;
    double* P = Pb + buf * nmax;
    double* part = Pb + 2 * nmax + buf * 64;
    if (k > 0 && !wait_flag(flag, (unsigned)k, abort_flag, status)) return;
    const double* rowk = A + (int64_t)k * n + (k + 1);
    for (int i = tid; i < m; i += nt) v[i] = __ldcg(rowk + i);
    __syncthreads();
    double s = 0.0;
    for (int i = 1 + tid; i < m; i += nt) s += v[i] * v[i];
    s = block_sum(s, red);
    const double x0 = v[0];
    // this warp's first row past k (rows r with r mod GW == gw)
    const int r0 = k + 1 + (((gw - (k + 1)) % GW) + GW) % GW;
    if (s == 0.0) {
      if (c == 0 && tid == 0) { dd[k] = __ldcg(A + (int64_t)k * n + k); ee[k] = x0; tau[k] = 0.0; }
      if (r0 == k + 1 && lane == 0) publish_flag(flag, (unsigned)(k + 1));   // row k+1 is unchanged
      // one barrier per column in every case, so the two p buffers are never
      // rewritten while a slower block still reads them
      if (!job_barrier(cnt, (++nbar) * (unsigned)G, abort_flag, status)) return;
      continue;
    }
    const double nrm = sqrt(x0 * x0 + s);
    const double alpha = (x0 <= 0.0) ? nrm : -nrm;
    const double v0 = x0 - alpha;
    const double beta = 2.0 / (s + v0 * v0);
    __syncthreads();
    if (tid == 0) v[0] = v0;
    __syncthreads();
    double pv = 0.0;
    for (int r = r0; r < n; r += GW) {
      const int i = r - k - 1;
      const double* row = A + (int64_t)r * n + (k + 1);
      double acc = 0.0;
      for (int j = lane; j < m; j += 32) acc += __ldcg(row + j) * v[j];
      acc = warp_sum(acc);
      if (lane == 0) {
        const double pi = beta * acc;
        P[i] = pi;
        pv += pi * v[i];
      }
    }
    pv = block_sum(pv, red);
    if (tid == 0) part[c] = pv;
    if (!job_barrier(cnt, (++nbar) * (unsigned)G, abort_flag, status)) return;
    double tot = 0.0;
    for (int b = 0; b < G; ++b) tot += __ldcg(part + b);
    const double Kc = 0.5 * beta * tot;
    for (int i = tid; i < m; i += nt) w[i] = __ldcg(P + i) - Kc * v[i];
    __syncthreads();
    for (int r = r0; r < n; r += GW) {
      const int i = r - k - 1;
      double* row = A + (int64_t)r * n + (k + 1);
      const double vi = v[i], wi = w[i];
      // no contraction: entry (i, j) and (j, i) get the same two products
      for (int j = lane; j < m; j += 32)
        row[j] = __dsub_rn(__ldcg(row + j), __dadd_rn(__dmul_rn(vi, w[j]), __dmul_rn(wi, v[j])));
      __syncwarp();
      if (lane == 0) {
        A[(int64_t)k * n + r] = v[i];                       // reflector k in row k
        if (r == k + 1) publish_flag(flag, (unsigned)(k + 1));
      }
    }
    if (c == 0 && tid == 0) { dd[k] = __ldcg(A + (int64_t)k * n + k); ee[k] = alpha; tau[k] = beta; }
  }
  // every row's last update is in before the last diagonal entries are read
  if (!job_barrier(cnt, (++nbar) * (unsigned)G, abort_flag, status)) return;
  if (c == 0 && tid == 0) {
    if (n >= 2) {
      dd[n - 2] = __ldcg(A + (int64_t)(n - 2) * n + (n - 2));
      ee[n - 2] = __ldcg(A + (int64_t)(n - 1) * n + (n - 2));
      tau[n - 2] = 0.0;
    }
    dd[n - 1] = __ldcg(A + (int64_t)(n - 1) * n + (n - 1));
    ee[n - 1] = 0.0;
    tau[n - 1] = 0.0;
  }
}

// ------------------------------------------ cluster tridiagonalization --
// The same Householder reduction with the matrix held in the shared memory of
// a cluster of CS CTAs (distributed shared memory) instead of L2: row r of the
// lower triangle (entries 0..r) lives in CTA r mod CS, so each column costs
// two cluster barriers and three rounds of remote shared-memory reads, and the
// symmetric matrix-vector product and the rank-2 update read and write shared
// memory only. Per column k (trailing indices k+1..n-1):
//   every CTA forms v, beta from the gathered column x (redundantly, bit-
//   identically); A: y1 = the row part of A v for its rows (entries j <= i),
//   y2 = its rows' contribution to the column part (entries i > j) for every
//   j, and a copy of its rows' column k+1; barrier; B: the owner of j sums
//   p_j = beta (y1_j + sum over CTAs of y2_j), every CTA gathers column k+1;
//   barrier; C: every CTA gathers p, forms w = p - (beta p.v / 2) v, updates
//   its rows and, from the gathered column, the next x (the same operations
//   as the owner's update of those entries).
// A warp works on up to four of its rows at once (one pass over j for all
// four), so the shared-memory loads of a pass are independent.
// Outputs as k_tridiag: d, e, beta in work, reflector k in row k of A.
constexpr int TC_THREADS = 512;
constexpr size_t TC_SMEM_MAX = 227 * 1024;

// packed offset of owned row lr (global row rank + CS lr, rank + 1 + CS lr entries)
template <int CS>
__host__ __device__ inline int tc_off(int lr, int rank) { return lr * (rank + 1) + CS * (lr * (lr - 1) / 2); }
template <int CS>
__host__ __device__ inline size_t tc_lsize(int n) {
  const size_t nmx = (n + CS - 1) / CS;
  return nmx * CS + CS * nmx * (nmx - 1) / 2;
}
template <int CS>
__host__ __device__ inline size_t tc_smem_bytes(int n) {
  return (tc_lsize<CS>(n) + 8 * (size_t)n + 2 * (size_t)((n + CS - 1) / CS) + 32) * sizeof(double);
}

template <int CS>
__global__ void __launch_bounds__(TC_THREADS, 1) k_tridiag_cl(const EighJob* __restrict__ jobs, int nmax) {
  const int job = blockIdx.x / CS;
  const int rank = (int)tc_rank();
  const EighJob J = jobs[job];
  const int n = J.n;              // the same for the whole cluster: every CTA returns, or none
  if (n <= 0) return;
  extern __shared__ double sh[];
  // the layout depends on nmax only, so it is the same in every CTA
  const int nmx = (nmax + CS - 1) / CS;
  double* L = sh;                           // owned rows, packed
  double* vv = L + tc_lsize<CS>(nmax);      // v (absolute indices)
  double* ww = vv + nmax;                   // gathered p, then w
  double* xx = ww + nmax;                   // x = current column below the diagonal; xx[k+1] diagonal
  double* yp = xx + nmax;                   // this CTA's y2 (read remotely)
  double* xs = yp + nmax;                   // this CTA's rows' column k+1 (read remotely)
  double* pb = xs + nmax;                   // p_j of this CTA's j (read remotely)
  double* y1 = pb + nmax;                   // row part of A v, owned rows
  int* roff = reinterpret_cast<int*>(y1 + nmx);   // packed offset of each owned row
  double* red = y1 + 2 * nmx;
  double* se = red + 32;                    // e and beta of every column, written out at the end
  double* st = se + nmax;
  double* A = J.A;
  double* dd = J.work;
  double* ee = dd + n;
  double* tau = ee + n;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarp = nt >> 5;
  const int nown = rank < n ? (n - rank + CS - 1) / CS : 0;
  for (int lr = tid; lr < nown; lr += nt) roff[lr] = tc_off<CS>(lr, rank);
  // load the owned rows (lower part) and the first column (row 0 by symmetry)
  for (int lr = warp; lr < nown; lr += nwarp) {
    const int r = rank + CS * lr;
    double* dst = L + tc_off<CS>(lr, rank);
    for (int j = lane; j <= r; j += 32) dst[j] = __ldcg(A + (int64_t)r * n + j);
  }
  double sq = 0.0;
  for (int r = tid; r < n; r += nt) {
    const double x = __ldcg(A + r);         // xx[0] = A[0][0]
    xx[r] = x;
    if (r >= 2) sq += x * x;
  }
  tc_cluster_sync();
  for (int k = 0; k + 2 < n; ++k) {
    // ---- Householder vector of x = xx[k+1 .. n-1]
    const double s = block_sum(sq, red);
    const double x0 = xx[k + 1];
    double beta = 0.0, alpha = x0;
    if (s != 0.0) {
      const double nrm = sqrt(x0 * x0 + s);
      alpha = (x0 <= 0.0) ? nrm : -nrm;
      const double v0 = x0 - alpha;
      beta = 2.0 / (s + v0 * v0);
      for (int r = k + 1 + tid; r < n; r += nt) vv[r] = (r == k + 1) ? v0 : xx[r];
    } else {
      // no reflection: v = 0 makes p, w and the update vanish exactly
      for (int r = k + 1 + tid; r < n; r += nt) vv[r] = 0.0;
    }
    if (tid == 0) { se[k] = alpha; st[k] = beta; }
    __syncthreads();
    // ---- A: y1 (owned rows), y2 partials (all j), copy of column k+1
    const int lr_lo = (k + 1 <= rank) ? 0 : (k + 1 - rank + CS - 1) / CS;   // first owned row >= k+1
    for (int base = lr_lo + warp; base < nown; base += 4 * nwarp) {
      int ro[4], rr[4];
      int rmax = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int lr = base + i * nwarp;
        rr[i] = lr < nown ? rank + CS * lr : -1;     // -1: no row (the j loop skips it)
        ro[i] = lr < nown ? roff[lr] : 0;
        rmax = max(rmax, rr[i]);
      }
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
      for (int j = k + 1 + lane; j <= rmax; j += 32) {
        const double vj = vv[j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (j <= rr[i]) acc[i] += L[ro[i] + j] * vj;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = warp_sum(acc[i]);
      if (lane < 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i == lane && rr[i] >= 0) { y1[base + i * nwarp] = acc[i]; xs[rr[i]] = L[ro[i] + k + 1]; }
      }
    }
    // column k of the owned rows is no longer read: it keeps reflector k
    for (int lr = lr_lo + tid; lr < nown; lr += nt) L[roff[lr] + k] = vv[rank + CS * lr];
    for (int j = k + 1 + tid; j < n; j += nt) {
      int lr = (j < rank) ? 0 : (j - rank) / CS + 1;   // owned rows > j
      // four partial sums (rows lr mod 4), added in a fixed order
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      for (; lr + 3 < nown; lr += 4) {
        const int r = rank + CS * lr;
        a0 += L[roff[lr] + j] * vv[r];
        a1 += L[roff[lr + 1] + j] * vv[r + CS];
        a2 += L[roff[lr + 2] + j] * vv[r + 2 * CS];
        a3 += L[roff[lr + 3] + j] * vv[r + 3 * CS];
      }
      for (; lr < nown; ++lr) a0 += L[roff[lr] + j] * vv[rank + CS * lr];
      yp[j] = (a0 + a1) + (a2 + a3);
    }
    tc_cluster_sync();
    // ---- B: p_j for owned j; gather column k+1
    for (int lr = lr_lo + tid; lr < nown; lr += nt) {
      const int j = rank + CS * lr;
      double part[CS];
#pragma unroll
      for (int c = 0; c < CS; ++c) part[c] = *tc_peer(yp + j, (uint32_t)c);
      double acc = y1[lr];
#pragma unroll
      for (int c = 0; c < CS; ++c) acc += part[c];
      pb[j] = beta * acc;
    }
    for (int r = k + 1 + tid; r < n; r += nt) xx[r] = *tc_peer(xs + r, (uint32_t)(r % CS));
    tc_cluster_sync();
    // ---- C: gather p, w = p - Kc v, update owned rows and the next column
    double pv = 0.0;
    for (int j = k + 1 + tid; j < n; j += nt) {
      const double pj = *tc_peer(pb + j, (uint32_t)(j % CS));
      ww[j] = pj;
      pv += pj * vv[j];
    }
    const double Kc = 0.5 * beta * block_sum(pv, red);
    for (int j = k + 1 + tid; j < n; j += nt) ww[j] -= Kc * vv[j];
    __syncthreads();
    for (int base = lr_lo + warp; base < nown; base += 4 * nwarp) {
      int ro[4], rr[4];
      double vi[4], wi[4];
      int rmax = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int lr = base + i * nwarp;
        rr[i] = lr < nown ? rank + CS * lr : -1;
        ro[i] = lr < nown ? roff[lr] : 0;
        vi[i] = lr < nown ? vv[rr[i]] : 0.0;
        wi[i] = lr < nown ? ww[rr[i]] : 0.0;
        rmax = max(rmax, rr[i]);
      }
      for (int j = k + 1 + lane; j <= rmax; j += 32) {
        const double wj = ww[j], vj = vv[j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (j <= rr[i]) {
            double* e = L + ro[i] + j;
            *e = __dsub_rn(*e, __dadd_rn(__dmul_rn(vi[i], wj), __dmul_rn(wi[i], vj)));
          }
      }
    }
    const double vk = vv[k + 1], wk = ww[k + 1];
    sq = 0.0;
    for (int r = k + 1 + tid; r < n; r += nt) {
      const double x = __dsub_rn(xx[r], __dadd_rn(__dmul_rn(vv[r], wk), __dmul_rn(ww[r], vk)));
      xx[r] = x;
      if (r >= k + 3) sq += x * x;       // the next column's sum of squares
    }
  }
  __syncthreads();
  // d from the owned diagonals; reflector k (column k of rows k+1..n-1) into
  // row k of A; e and beta from CTA 0; the last two columns have no reflector
  for (int lr = warp; lr < nown; lr += nwarp) {
    const int r = rank + CS * lr;
    const double* row = L + roff[lr];
    const int kmax = min(r, n - 2);
    for (int k = lane; k < kmax; k += 32) A[(int64_t)k * n + r] = row[k];
    if (lane == 0) dd[r] = row[r];
    if (lane == 0 && r == n - 1 && n >= 2) ee[n - 2] = row[n - 2];
  }
  if (rank == 0) {
    for (int k = tid; k + 2 < n; k += nt) { ee[k] = se[k]; tau[k] = st[k]; }
    if (tid == 0) {
      if (n >= 2) tau[n - 2] = 0.0;
      ee[n - 1] = 0.0;
      tau[n - 1] = 0.0;
    }
  }
  tc_cluster_sync();          // no CTA leaves while another may still read its shared memory
}

template <int CS>
static jolt_status launch_tridiag_cl(const EighJob* jobs, int njobs, int nmax, cudaStream_t s) {
  const size_t smem = tc_smem_bytes<CS>(nmax);
  { static size_t set = 0; if (smem > set) { JOLT_CUDA_TRY(cudaFuncSetAttribute(k_tridiag_cl<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); set = smem; } }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(njobs * CS);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int nm = nmax;
  JOLT_CUDA_TRY(cudaLaunchKernelEx(&cfg, k_tridiag_cl<CS>, jobs, nm));
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Number of eigenvalues of the tridiagonal (d, e) smaller than x; e2[i] is
// the rounded square of e[i].
__device__ __forceinline__ int sturm_count(const double* d, const double* e2, int n, double x, double pivmin) {
  int c = 0;
  double q = d[0] - x;
  if (fabs(q) < pivmin) q = -pivmin;
  c += q < 0.0;
  for (int i = 1; i < n; ++i) {
    q = (d[i] - x) - e2[i - 1] / q;
    if (fabs(q) < pivmin) q = -pivmin;
    c += q < 0.0;
  }
  return c;
}

// w[j] = j-th largest eigenvalue by multisection on Sturm counts: BIS_L
// lanes per eigenvalue count at BIS_L interior points of the current
// interval, and the interval shrinks to the sub-interval where the count
// passes the eigenvalue's rank (the count is monotone in x), (BIS_L + 1)x per
// round until no interior point is left.
constexpr int BIS_L = 8;

__global__ void __launch_bounds__(256) k_bisect(const EighJob* __restrict__ jobs) {
  const EighJob J = jobs[blockIdx.y];
  const int n = J.n;
  if (n <= 0) return;
  extern __shared__ double sh[];
  double* d = sh;
  double* e = sh + n;
  double* e2 = sh + 2 * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    d[i] = J.work[i];
    const double ei = J.work[n + i];
    e[i] = ei;
    e2[i] = ei * ei;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, sub = lane & (BIS_L - 1), base = lane & ~(BIS_L - 1);
  const int j = blockIdx.x * (blockDim.x / BIS_L) + threadIdx.x / BIS_L;
  const bool act = j < n;
  // Gershgorin bounds (every lane of the warp takes part)
  double lo = 1e300, hi = -1e300, emax = 0.0;
  for (int i = lane; i < n; i += 32) {
    const double r = (i > 0 ? fabs(e[i - 1]) : 0.0) + (i + 1 < n ? fabs(e[i]) : 0.0);
    lo = fmin(lo, d[i] - r);
    hi = fmax(hi, d[i] + r);
    emax = fmax(emax, fabs(e[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    emax = fmax(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  const double nrm = fmax(fabs(lo), fabs(hi));
  const double pivmin = fmax(1e-300, 2.2250738585072014e-308 * fmax(1.0, emax * emax));
  lo -= 4.0 * 2.220446049250313e-16 * nrm + pivmin;
  hi += 4.0 * 2.220446049250313e-16 * nrm + pivmin;
  const int m = n - 1 - (act ? j : 0);    // rank among the ascending eigenvalues
  bool done = !act;
  for (int round = 0; round < 96; ++round) {
    const double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) done = true;
    if (__all_sync(0xffffffffu, done)) break;
    const double x = lo + (hi - lo) * ((double)(sub + 1) / (double)(BIS_L + 1));
    const bool above = (!done && x > lo && x < hi) ? (sturm_count(d, e2, n, x, pivmin) > m) : (x >= hi);
    const unsigned bal = (__ballot_sync(0xffffffffu, above) >> base) & ((1u << BIS_L) - 1u);
    const int f = bal ? (__ffs(bal) - 1) : BIS_L;   // first point past the eigenvalue
    const double xl = __shfl_sync(0xffffffffu, x, base + (f > 0 ? f - 1 : 0));
    const double xh = __shfl_sync(0xffffffffu, x, base + (f < BIS_L ? f : BIS_L - 1));
    if (!done) {
      const double nlo = (f > 0) ? fmax(lo, xl) : lo;
      const double nhi = (f < BIS_L) ? fmin(hi, xh) : hi;
      if (nlo == lo && nhi == hi) done = true;     // no interior point moved the interval
      lo = nlo;
      hi = nhi;
    }
  }
  if (act && sub == 0) J.w[j] = 0.5 * (lo + hi);
}

// Eigenvectors of the leading nvec[job] eigenvalues, step 1: inverse
// iteration on the tridiagonal matrix. T - lam I is factored once by Gaussian
// elimination with partial pivoting (U with two superdiagonals, multipliers
// and swap flags), then three solves from a fixed start vector, each followed
// by normalization. One thread per vector, INV_W vectors per block; a block's
// factors and iterate are interleaved by vector ([array][i][vector] in J.F,
// [i][vector] in J.Z from the block's first vector on), so a warp's accesses
// are contiguous. The recurrences carry their running values in registers;
// the back substitution multiplies by the stored reciprocal pivots.
constexpr int INV_W = 64;

__global__ void __launch_bounds__(INV_W) k_invit(const EighJob* __restrict__ jobs, const int* __restrict__ nvec) {
  const EighJob J = jobs[blockIdx.y];
  const int n = J.n;
  if (n <= 0) return;
  const int nv = min(nvec[blockIdx.y], n);
  const int j0 = blockIdx.x * INV_W;
  if (j0 >= nv) return;
  const int W = min(INV_W, nv - j0), lane = threadIdx.x;
  if (lane >= W) return;
  const int j = j0 + lane;
  const double* d = J.work;
  const double* e = d + n;
  double* F = J.F + (int64_t)j0 * 5 * n;
  double* rdg = F;                          // 1 / pivot of U
  double* u1 = F + (int64_t)n * W;          // first superdiagonal of U
  double* u2 = F + (int64_t)2 * n * W;      // second superdiagonal of U
  double* ml = F + (int64_t)3 * n * W;      // multipliers
  double* sw = F + (int64_t)4 * n * W;      // 1.0 where rows i, i+1 were swapped
  double* z = J.Z + (int64_t)j0 * n;
  auto at = [&](int i) { return (int64_t)i * W + lane; };
  double nrm = 0.0;
  for (int i = 0; i < n; ++i) nrm = fmax(nrm, fabs(__ldg(d + i)) + fabs(__ldg(e + i)) + (i ? fabs(__ldg(e + i - 1)) : 0.0));
  const double lam = J.w[j];
  const double tiny = fmax(nrm, 1e-300) * 2.220446049250313e-16;
  auto guard = [&](double g) { return (fabs(g) < tiny) ? ((g < 0.0) ? -tiny : tiny) : g; };
  // factorization: row i is final after step i
  double dg = __ldg(d) - lam, ui = (n > 1) ? __ldg(e) : 0.0;
  double dn = (n > 1) ? __ldg(d + 1) - lam : 0.0, un = (n > 2) ? __ldg(e + 1) : 0.0;
  for (int i = 0; i + 1 < n; ++i) {
    const double sub = __ldg(e + i);      // row i+1, column i
    double f, u2i = 0.0, swi;
    if (fabs(dg) >= fabs(sub)) {
      f = (dg != 0.0) ? sub / dg : 0.0;
      swi = 0.0;
      dn -= f * ui;
    } else {
      f = dg / sub;
      swi = 1.0;
      const double t = ui;
      ui = dn;
      dn = t - f * dn;
      dg = sub;
      if (i + 2 < n) {
        u2i = un;
        un = -f * un;
      }
    }
    rdg[at(i)] = 1.0 / guard(dg);
    u1[at(i)] = ui;
    u2[at(i)] = u2i;
    ml[at(i)] = f;
    sw[at(i)] = swi;
    dg = dn;
    ui = un;
    dn = (i + 2 < n) ? __ldg(d + i + 2) - lam : 0.0;
    un = (i + 3 < n) ? __ldg(e + i + 2) : 0.0;
  }
  rdg[at(n - 1)] = 1.0 / guard(dg);
  u1[at(n - 1)] = 0.0;
  u2[at(n - 1)] = 0.0;
  double scale = 1.0;
  for (int i = 0; i < n; ++i) z[at(i)] = 1.0 + 0.5 * sin(0.7 * (double)i + 0.3 * (double)j);
  for (int iter = 0; iter < 3; ++iter) {
    // forward: apply the row swaps and multipliers (and the last normalization)
    double zc = scale * z[at(0)];
    for (int i = 0; i + 1 < n; ++i) {
      double zn = scale * z[at(i + 1)];
      if (sw[at(i)] != 0.0) { const double t = zc; zc = zn; zn = t; }
      zn -= ml[at(i)] * zc;
      z[at(i)] = zc;
      zc = zn;
    }
    // back substitution with U
    double z1 = zc * rdg[at(n - 1)], z2 = 0.0;
    z[at(n - 1)] = z1;
    double ss = z1 * z1;
    for (int i = n - 2; i >= 0; --i) {
      const double zi = (z[at(i)] - u1[at(i)] * z1 - u2[at(i)] * z2) * rdg[at(i)];
      z[at(i)] = zi;
      ss += zi * zi;
      z2 = z1;
      z1 = zi;
    }
    scale = 1.0 / sqrt(ss);
  }
  for (int i = 0; i < n; ++i) z[at(i)] *= scale;
}

// Step 2: z <- H_0 H_1 ... H_{n-3} z for a block of up to vb vectors held in
// shared memory; reflector k (row k of A) is read once per block, the next
// one is fetched while the current one is applied. Then the sign convention
// (largest |entry| positive, first on ties) and the rows of Vt.
constexpr int BT_PRE = 8;     // reflector entries a thread prefetches (n <= 256 * 8)

__global__ void __launch_bounds__(256) k_backtr(const EighJob* __restrict__ jobs, const int* __restrict__ nvec,
                                              int vb) {
  const EighJob J = jobs[blockIdx.y];
  const int n = J.n;
  if (n <= 0) return;
  const int nv = min(nvec[blockIdx.y], n);
  const int v0 = blockIdx.x * vb;
  if (v0 >= nv) return;
  const int nb = min(vb, nv - v0);
  extern __shared__ double sh[];
  double* Zs = sh;                        // nb x n
  double* vbuf = sh + (int64_t)vb * n;    // 2 x n
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double* tau = J.work + 2 * n;
  // gather the block's vectors from the interleaved layout of k_invit
  for (int vv = 0; vv < nb; ++vv) {
    const int jj = v0 + vv, b0 = (jj / INV_W) * INV_W, W = min(INV_W, nv - b0), ln = jj - b0;
    const double* z = J.Z + (int64_t)b0 * n;
    for (int i = tid; i < n; i += 256) Zs[(int64_t)vv * n + i] = z[(int64_t)i * W + ln];
  }
  auto load_v = [&](int k, double* r) {
#pragma unroll
    for (int u = 0; u < BT_PRE; ++u) {
      const int i = tid + 256 * u;
      r[u] = (k >= 0 && i < n - k - 1) ? __ldg(J.A + (int64_t)k * n + k + 1 + i) : 0.0;
    }
  };
  auto store_v = [&](int k, const double* r) {
    double* dst = vbuf + (k & 1) * n;
#pragma unroll
    for (int u = 0; u < BT_PRE; ++u) {
      const int i = tid + 256 * u;
      if (k >= 0 && i < n - k - 1) dst[i] = r[u];
    }
  };
  double pre[BT_PRE];
  if (n >= 3) {
    load_v(n - 3, pre);
    store_v(n - 3, pre);
  }
  __syncthreads();
  for (int k = n - 3; k >= 0; --k) {
    load_v(k - 1, pre);                   // next reflector, in flight during this one
    const double beta = __ldg(tau + k);
    const int m = n - k - 1;
    if (beta != 0.0) {
      const double* v = vbuf + (k & 1) * n;
      for (int vv = warp; vv < nb; vv += 8) {
        double* z = Zs + (int64_t)vv * n + (k + 1);
        double acc0 = 0.0, acc1 = 0.0;         // two chains, added in a fixed order
        int i = lane;
        for (; i + 32 < m; i += 64) {
          acc0 += v[i] * z[i];
          acc1 += v[i + 32] * z[i + 32];
        }
        if (i < m) acc0 += v[i] * z[i];
        const double acc = beta * warp_sum(acc0 + acc1);
        for (int i = lane; i < m; i += 32) z[i] -= acc * v[i];
      }
    }
    store_v(k - 1, pre);
    __syncthreads();
  }
  for (int vv = warp; vv < nb; vv += 8) {
    const double* z = Zs + (int64_t)vv * n;
    double best = -1.0;
    int bi = 0x7fffffff;
    for (int i = lane; i < n; i += 32) {
      const double a = fabs(z[i]);
      if (a > best) { best = a; bi = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    const double sg = (z[bi] < 0.0) ? -1.0 : 1.0;
    double* dst = J.Vt + (int64_t)(v0 + vv) * n;
    for (int i = lane; i < n; i += 32) dst[i] = sg * z[i];
  }
}

jolt_status launch_tridiag(const EighJob* jobs, int njobs, int nmax, cudaStream_t s) {
  if (njobs <= 0) return JOLT_OK;
  // matrices that fit a cluster's shared memory: the cluster reduction
  if (nmax >= 48 && tc_smem_bytes<6>(nmax) <= TC_SMEM_MAX) return launch_tridiag_cl<6>(jobs, njobs, nmax, s);
  const size_t smem = (size_t)(2 * nmax + 32) * sizeof(double);
  { static size_t set = 0; if (smem > set) { JOLT_CUDA_TRY(cudaFuncSetAttribute(k_tridiag, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); set = smem; } }
  k_tridiag<<<njobs, EIG_THREADS, smem, s>>>(jobs);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Blocks per job for the multi-block reduction: as many as fit on the device
// at once (cooperative launch), at least two matrix rows per warp.
static int tridiag_blocks_per_job(int njobs, int nmax, size_t smem) {
  static int sms = 0, per_sm = -1;
  static size_t smem_at = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  if (per_sm < 0 || smem_at != smem) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_tridiag_multi, EIG_THREADS, smem) != cudaSuccess)
      per_sm = 0;
    cudaGetLastError();
    smem_at = smem;
  }
  const int cap = sms * per_sm;
  int G = njobs > 0 ? cap / njobs : 0;
  G = std::min(G, std::max(1, nmax / (2 * (EIG_THREADS / 32))));
  return std::min(G, 64);
}

jolt_status launch_tridiag_multi(const EighJob* jobs, int njobs, int nmax, double* scratch, unsigned int* counters,
                                 int* status, cudaStream_t s) {
  if (njobs <= 0) return JOLT_OK;
  // the matrix fits the shared memory of a cluster: k_tridiag_cl, on the
  // smallest cluster whose CTAs hold their rows (more clusters resident)
  if (nmax >= 48 && tc_smem_bytes<6>(nmax) <= TC_SMEM_MAX) return launch_tridiag_cl<6>(jobs, njobs, nmax, s);
  if (nmax >= 48 && tc_smem_bytes<8>(nmax) <= TC_SMEM_MAX) return launch_tridiag_cl<8>(jobs, njobs, nmax, s);
  const size_t smem = (size_t)(2 * nmax + 32) * sizeof(double);
  { static size_t set = 0; if (smem > set) { JOLT_CUDA_TRY(cudaFuncSetAttribute(k_tridiag_multi, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); set = smem; } }
  const int G = tridiag_blocks_per_job(njobs, nmax, smem);
  if (G < 2) return launch_tridiag(jobs, njobs, nmax, s);
  JOLT_CUDA_TRY(cudaMemsetAsync(counters, 0, (size_t)(2 * njobs + 1) * sizeof(unsigned int), s));
  int Gv = G, nm = nmax;
  void* args[] = {(void*)&jobs, (void*)&Gv, (void*)&nm, (void*)&scratch, (void*)&counters, (void*)&status};
  JOLT_CUDA_TRY(cudaLaunchCooperativeKernel((const void*)k_tridiag_multi, dim3(njobs * G), dim3(EIG_THREADS), args,
                                            smem, s));
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_bisect(const EighJob* jobs, int njobs, int nmax, cudaStream_t s) {
  const size_t smem = (size_t)(3 * nmax) * sizeof(double);
  { static size_t set = 0; if (smem > set) { JOLT_CUDA_TRY(cudaFuncSetAttribute(k_bisect, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); set = smem; } }
  dim3 g((nmax + 256 / BIS_L - 1) / (256 / BIS_L), njobs);   // BIS_L lanes per eigenvalue
  k_bisect<<<g, 256, smem, s>>>(jobs);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_eigvecs_n(const EighJob* jobs, int njobs, int nvec_max, int nmax, const int* nvec, cudaStream_t s) {
  if (nvec_max <= 0 || njobs <= 0) return JOLT_OK;
  if (nmax > 256 * BT_PRE) { set_error("eigenvectors need n <= %d (n=%d)", 256 * BT_PRE, nmax); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  k_invit<<<dim3((nvec_max + INV_W - 1) / INV_W, njobs), INV_W, 0, s>>>(jobs, nvec);
  JOLT_LAUNCHED();
  // vectors per block: 16 (two per warp), so that several blocks share an
  // SM and hide each other's shared-memory latency; fewer when n is large
  const int vb = std::max(1, std::min(16, (int)((200 * 1024) / ((size_t)nmax * sizeof(double))) - 2));
  const size_t smem = (size_t)(vb + 2) * nmax * sizeof(double);
  { static size_t set = 0; if (smem > set) { JOLT_CUDA_TRY(cudaFuncSetAttribute(k_backtr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); set = smem; } }
  k_backtr<<<dim3((nvec_max + vb - 1) / vb, njobs), 256, smem, s>>>(jobs, nvec, vb);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_fgram_x(const CellDesc* cells, int ncells, int D, const float2* cs, int nchunk,
                           double* partial, cudaStream_t s) {
  dim3 grid(nchunk, ncells);
  if (D == 128) k_fgram_x<128><<<grid, 256, 0, s>>>(cells, cs, nchunk, partial);
  else k_fgram_x<64><<<grid, 256, 0, s>>>(cells, cs, nchunk, partial);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_fgram_rows(const double* const* Y, const int* nrow_used, const int* rmax_of,
                              const int* nlh_of, int ncells, int D, int nchunk, double* partial,
                              cudaStream_t s) {
  dim3 grid(nchunk, ncells);
  if (D == 128) k_fgram_rows<128><<<grid, 256, 0, s>>>(Y, nrow_used, rmax_of, nlh_of, nchunk, partial);
  else k_fgram_rows<64><<<grid, 256, 0, s>>>(Y, nrow_used, rmax_of, nlh_of, nchunk, partial);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_sum_chunks(const double* partial, int nchunk, int len, int ncells,
                              double* const* out, double* const* out_last, cudaStream_t s) {
  dim3 grid((len + 255) / 256, ncells);
  k_sum_chunks<<<grid, 256, 0, s>>>(partial, nchunk, len, out, out_last);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_token_gram(const CellDesc* cells, int ncells, int nmax, const float2* cs,
                              double* const* G, cudaStream_t s) {
  int nt = (nmax + 63) / 64;
  dim3 grid(nt * (nt + 1) / 2, ncells);
  k_token_gram<<<grid, 256, 0, s>>>(cells, cs, G);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
