// Data-driven layer grouping ("A JoLT for the KV Cache", Section 3: the L
// layers are split into contiguous groups of layers whose top-8 token-mode
// singular vectors line up; a group breaks where the score of two
// consecutive layers falls below the median score, within the size bounds of
// that paragraph's footnote).
//
// Per job (sequence b, layer l) the keys X (T x F, F = H*D, before RoPE)
// go through a randomized subspace iteration of width S = 16 (8 vectors and
// 8 of oversampling):
//   W = X Omega; Q = orth(W);  q times { Z = X^T Q; W = X Z; Q = orth(W) };
//   Z = X^T Q; C = Z^T Z; V8 = top-8 eigenvectors of C (cyclic Jacobi);
//   U = Q V8.
// orth(W) is Cholesky QR done twice, each pass on the Gram plus a small
// shift of its trace (Fukaya, Nakatsukasa, Yanagisawa, Yamamoto, "Shifted
// Cholesky QR for computing the QR factorization of ill-conditioned
// matrices", SIAM J. Sci. Comput. 2020), so that the factorization exists
// for any W. The score of (l, l+1) is the mean squared cosine of the
// principal angles between the two 8-dimensional subspaces,
// ||U_l^T U_(l+1)||_F^2 / 8 = ||V8_l^T (Q_l^T Q_(l+1)) V8_(l+1)||_F^2 / 8,
// averaged over the batch's sequences. One thread then takes the median and
// applies the rule.
//
// Precision: the T-sized passes (X Z, X^T Q) multiply in fp32. X Z sums a
// whole row in fp32; X^T Q sums one 128-row tile in fp32 and the tiles in
// fp64. Grams, Cholesky factors, the Jacobi solve and the scores are fp64;
// Q is kept in fp32.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {
namespace grp {

constexpr int S = 16;             // sketch width
constexpr int NV = 8;             // vectors per layer
constexpr int TM = 128;           // rows per tile in X Z and X^T Q
constexpr int XTQ_TILES = 16;     // tiles per X^T Q block (2048 rows)
constexpr int GRAM_ROWS = 4096;   // rows per Gram partial
constexpr int MAX_LAYERS = 1024;

// Where one job's keys are: for job = b * L + l, element (t, h, d) at
// k + b*sb + l*sl + h*sh + t*st + d (strides in elements).
struct KeySrc {
  const void* k;
  int f32;
  int64_t sb, sl, sh, st;
  int L, H, T, D;
  const float2* cs;   // RoPE cos/sin table [T][D/2], or null
};

__device__ __forceinline__ int64_t job_base(const KeySrc& s, int job) {
  const int b = job / s.L, l = job % s.L;
  return (int64_t)b * s.sb + (int64_t)l * s.sl;
}

// Stage rows [t0, t0 + TM) of head h into xs[row * pitch + d] as fp32, the
// RoPE rotation undone when a table is given (x_i = y_i c + y_j s,
// x_j = y_j c - y_i s, j = i + D/2, no fused multiply-add). Rows past T are
// zero. Each of the NT threads moves TM * D / 4 / NT "quads": elements
// (2q, 2q+1) and their partners (D/2 + 2q, D/2 + 2q + 1), in batches of
// STAGE_BATCH whose loads are all issued before any is used.
constexpr int STAGE_BATCH = 4;
template <int D, int NT>
__device__ __forceinline__ void stage_x(const KeySrc& s, int job, int h, int t0, float* xs, int pitch) {
  constexpr int half = D / 2, QPR = D / 4, NQ = TM * QPR / NT;
  static_assert(NQ % STAGE_BATCH == 0, "quads per thread must be a multiple of the batch");
  const int64_t base = job_base(s, job) + (int64_t)h * s.sh;
#pragma unroll 1
  for (int u0 = 0; u0 < NQ; u0 += STAGE_BATCH) {
    float a0[STAGE_BATCH], a1[STAGE_BATCH], b0[STAGE_BATCH], b1[STAGE_BATCH];
    float4 c[STAGE_BATCH];
#pragma unroll
    for (int u = 0; u < STAGE_BATCH; ++u) {
      const int qi = threadIdx.x + NT * (u0 + u);
      const int r = qi / QPR, q = qi % QPR, t = t0 + r;
      a0[u] = a1[u] = b0[u] = b1[u] = 0.f;
      c[u] = make_float4(1.f, 0.f, 1.f, 0.f);
      if (t < s.T) {
        const int64_t off = base + (int64_t)t * s.st + 2 * q;
        if (s.f32) {
          const float* p = reinterpret_cast<const float*>(s.k);
          const float2 va = *reinterpret_cast<const float2*>(p + off);
          const float2 vb = *reinterpret_cast<const float2*>(p + off + half);
          a0[u] = va.x; a1[u] = va.y; b0[u] = vb.x; b1[u] = vb.y;
        } else {
          const uint16_t* p = reinterpret_cast<const uint16_t*>(s.k);
          const uint32_t wa = *reinterpret_cast<const uint32_t*>(p + off);
          const uint32_t wb = *reinterpret_cast<const uint32_t*>(p + off + half);
          a0[u] = __uint_as_float(wa << 16); a1[u] = __uint_as_float(wa & 0xFFFF0000u);
          b0[u] = __uint_as_float(wb << 16); b1[u] = __uint_as_float(wb & 0xFFFF0000u);
        }
        if (s.cs) c[u] = *reinterpret_cast<const float4*>(s.cs + (int64_t)t * half + 2 * q);
      }
    }
#pragma unroll
    for (int u = 0; u < STAGE_BATCH; ++u) {
      const int qi = threadIdx.x + NT * (u0 + u);
      const int r = qi / QPR, q = qi % QPR;
      float x0 = a0[u], x1 = a1[u], y0 = b0[u], y1 = b1[u];
      if (s.cs) {
        x0 = __fadd_rn(__fmul_rn(a0[u], c[u].x), __fmul_rn(b0[u], c[u].y));
        y0 = __fsub_rn(__fmul_rn(b0[u], c[u].x), __fmul_rn(a0[u], c[u].y));
        x1 = __fadd_rn(__fmul_rn(a1[u], c[u].z), __fmul_rn(b1[u], c[u].w));
        y1 = __fsub_rn(__fmul_rn(b1[u], c[u].z), __fmul_rn(a1[u], c[u].w));
      }
      float* row = xs + r * pitch;
      row[2 * q] = x0;
      row[2 * q + 1] = x1;
      row[half + 2 * q] = y0;
      row[half + 2 * q + 1] = y1;
    }
  }
}

// Omega[f][c], F x S standard normals: Philox4x32-10 words turned into
// normals by Box-Muller, four per counter.
__global__ void k_grp_omega(double* __restrict__ om, int F, uint64_t seed) {
  const int n4 = F * S / 4;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x) {
    const u4 r = philox_at(seed, STREAM_GROUPING, (uint32_t)i);
    const double u0 = ((double)r.x + 0.5) * 0x1p-32, u1 = ((double)r.y + 0.5) * 0x1p-32;
    const double u2 = ((double)r.z + 0.5) * 0x1p-32, u3 = ((double)r.w + 0.5) * 0x1p-32;
    const double r0 = sqrt(-2.0 * log(u0)), r1 = sqrt(-2.0 * log(u2));
    const double t0 = 6.283185307179586 * u1, t1 = 6.283185307179586 * u3;
    om[4 * i + 0] = r0 * cos(t0);
    om[4 * i + 1] = r0 * sin(t0);
    om[4 * i + 2] = r1 * cos(t1);
    om[4 * i + 3] = r1 * sin(t1);
  }
}

// W[job][t][c] = sum_f X[t][f] Z[job][f][c] for one tile of TM rows; the
// Z block of a job starts at Z + job * zstride (zstride 0: one Omega for
// all jobs). 256 threads, each 2 rows x 4 columns; heads staged one at a
// time (X tile [TM][D+1] and Z rows [D][S], both fp32). Three blocks fit an
// SM (shared memory), 24 warps, enough to cover the staging loads' latency.
constexpr int XZ_THREADS = 256;
template <int D>
__global__ void __launch_bounds__(XZ_THREADS, 3) k_grp_xz(KeySrc s, const double* __restrict__ Z, int64_t zstride,
                                                       float* __restrict__ W) {
  extern __shared__ __align__(16) float sm[];
  constexpr int XP = D + 1;
  static_assert((TM * XP) % 4 == 0, "zs must start on a 16-byte boundary");
  float* xs = sm;
  float* zs = sm + TM * XP;       // TM * XP is a multiple of 4: zs stays 16-byte aligned
  const int job = blockIdx.y, t0 = blockIdx.x * TM;
  const int tid = threadIdx.x, cg = tid & 3, rg = tid >> 2;   // rows 2rg, 2rg+1; columns 4cg..4cg+3
  const double* z = Z + (int64_t)job * zstride;
  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
  for (int h = 0; h < s.H; ++h) {
    __syncthreads();
    stage_x<D, XZ_THREADS>(s, job, h, t0, xs, XP);
    {
      constexpr int NZ = D * S / XZ_THREADS;    // 8 (D = 128) or 4 (D = 64) values per thread
      double zv[NZ];
#pragma unroll
      for (int u = 0; u < NZ; ++u) zv[u] = z[(int64_t)h * D * S + tid + XZ_THREADS * u];
#pragma unroll
      for (int u = 0; u < NZ; ++u) zs[tid + XZ_THREADS * u] = (float)zv[u];
    }
    __syncthreads();
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float4 zv = *reinterpret_cast<const float4*>(zs + d * S + 4 * cg);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float x = xs[(2 * rg + j) * XP + d];
        acc[j][0] = fmaf(x, zv.x, acc[j][0]);
        acc[j][1] = fmaf(x, zv.y, acc[j][1]);
        acc[j][2] = fmaf(x, zv.z, acc[j][2]);
        acc[j][3] = fmaf(x, zv.w, acc[j][3]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int t = t0 + 2 * rg + j;
    if (t < s.T)
      *reinterpret_cast<float4*>(W + ((int64_t)job * s.T + t) * S + 4 * cg) =
          make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
  }
}

// P[chunk][job][f][c] = sum over the chunk's rows t of X[t][f] Q[job][t][c],
// f in head blockIdx.y. 2D threads, each 2 features x 4 columns; fp32 sums
// over one tile of TM rows, fp64 across the chunk's tiles.
template <int D>
__global__ void __launch_bounds__(2 * D, 3) k_grp_xtq(KeySrc s, const float* __restrict__ Q, double* __restrict__ P,
                                                   int njobs) {
  extern __shared__ __align__(16) float sm[];
  constexpr int NT = 2 * D;
  constexpr int XP = D + 4;
  static_assert(XP % 4 == 0 && (TM * XP) % 4 == 0, "float2 rows of xs, float4 rows of qs");
  float* xs = sm;                  // [TM][XP]
  float* qs = sm + TM * XP;        // [TM][S]
  const int chunk = blockIdx.x, h = blockIdx.y, job = blockIdx.z;
  const int tid = threadIdx.x, cg = tid & 3, fg = tid >> 2;   // features 2fg, 2fg+1; columns 4cg..4cg+3
  const int F = s.H * D;
  double acc64[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc64[i][c] = 0.0;
  const float* q = Q + (int64_t)job * s.T * S;
  for (int tile = 0; tile < XTQ_TILES; ++tile) {
    const int t0 = (chunk * XTQ_TILES + tile) * TM;
    if (t0 >= s.T) break;
    __syncthreads();
    {
      constexpr int NV4 = TM * S / 4 / NT;   // float4 of Q per thread: 2
      float4 v[NV4];
#pragma unroll
      for (int u = 0; u < NV4; ++u) {
        const int e = tid + NT * u, r = e / (S / 4), c4 = e % (S / 4), t = t0 + r;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < s.T) v[u] = *reinterpret_cast<const float4*>(q + (int64_t)t * S + 4 * c4);
      }
      stage_x<D, NT>(s, job, h, t0, xs, XP);
#pragma unroll
      for (int u = 0; u < NV4; ++u) {
        const int e = tid + NT * u, r = e / (S / 4), c4 = e % (S / 4);
        *reinterpret_cast<float4*>(qs + r * S + 4 * c4) = v[u];
      }
    }
    __syncthreads();
    float acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
#pragma unroll 8
    for (int r = 0; r < TM; ++r) {
      const float2 xv = *reinterpret_cast<const float2*>(xs + r * XP + 2 * fg);
      const float4 qv = *reinterpret_cast<const float4*>(qs + r * S + 4 * cg);
      const float xa[2] = {xv.x, xv.y};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        acc[i][0] = fmaf(xa[i], qv.x, acc[i][0]);
        acc[i][1] = fmaf(xa[i], qv.y, acc[i][1]);
        acc[i][2] = fmaf(xa[i], qv.z, acc[i][2]);
        acc[i][3] = fmaf(xa[i], qv.w, acc[i][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc64[i][c] += (double)acc[i][c];
  }
  double* p = P + (((int64_t)chunk * njobs + job) * F + (int64_t)h * D + 2 * fg) * S + 4 * cg;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) p[(int64_t)i * S + c] = acc64[i][c];
}

// Z[e] = sum over chunks of P[chunk][e], chunks in order.
__global__ void k_grp_zsum(const double* __restrict__ P, int nchunk, int64_t n, double* __restrict__ Z) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    double a = 0.0;
    for (int c = 0; c < nchunk; ++c) a += P[(int64_t)c * n + e];
    Z[e] = a;
  }
}

// Gram partials over GRAM_ROWS-row chunks: G[chunk][g][a][c] =
// sum_t A[t][a] B[t][c] in fp64. Self mode (pairs == 0): g = job, A = B =
// Q[job]. Cross mode: g = b * (L - 1) + l, A = Q[(b, l)], B = Q[(b, l + 1)].
// 256 threads, one entry each; 128-row tiles of both operands in shared
// memory.
__global__ void __launch_bounds__(256) k_grp_gram(const float* __restrict__ Q, int T, int L, int cross,
                                                  int ngram, double* __restrict__ G) {
  __shared__ __align__(16) double as[TM * S];
  __shared__ __align__(16) double bs[TM * S];
  const int chunk = blockIdx.x, g = blockIdx.y;
  int ja = g, jb = g;
  if (cross) {
    const int b = g / (L - 1), l = g % (L - 1);
    ja = b * L + l;
    jb = ja + 1;
  }
  const float* qa = Q + (int64_t)ja * T * S;
  const float* qb = Q + (int64_t)jb * T * S;
  const int tid = threadIdx.x, a = tid >> 4, c = tid & 15;
  double acc = 0.0;
  const int r_end = min(T, (chunk + 1) * GRAM_ROWS);
  for (int t0 = chunk * GRAM_ROWS; t0 < r_end; t0 += TM) {
    __syncthreads();
    for (int e = tid; e < TM * S / 4; e += 256) {
      const int r = e / (S / 4), c4 = e % (S / 4), t = t0 + r;
      float4 va = make_float4(0.f, 0.f, 0.f, 0.f), vb = va;
      if (t < r_end) {
        va = *reinterpret_cast<const float4*>(qa + (int64_t)t * S + 4 * c4);
        vb = *reinterpret_cast<const float4*>(qb + (int64_t)t * S + 4 * c4);
      }
      double* pa = as + r * S + 4 * c4;
      double* pb = bs + r * S + 4 * c4;
      pa[0] = va.x; pa[1] = va.y; pa[2] = va.z; pa[3] = va.w;
      pb[0] = vb.x; pb[1] = vb.y; pb[2] = vb.z; pb[3] = vb.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int r = 0; r < TM; ++r) acc = fma(as[r * S + a], bs[r * S + c], acc);
  }
  G[((int64_t)chunk * ngram + g) * (S * S) + tid] = acc;
}

// One job per block: the Gram of Q[job] from its chunk partials (chunks in
// order), a Cholesky factor R of G + sigma I with sigma = 11 (T S + S (S + 1))
// u tr(G), u = 2^-53 (the shift of shifted Cholesky QR), and R^{-1} (upper)
// into rinv[job]. A zero Gram (all-zero keys) gives R^{-1} = 0, so the basis
// of that job is zero. A non-finite trace sets *status.
__global__ void __launch_bounds__(256) k_grp_chol(const double* __restrict__ G, int nchunk, int njobs, int T,
                                                  double* __restrict__ rinv, int* __restrict__ status) {
  __shared__ double g[S][S + 1];
  __shared__ double R[S][S + 1];
  const int job = blockIdx.x, tid = threadIdx.x;
  {
    double a = 0.0;
    for (int c = 0; c < nchunk; ++c) a += G[((int64_t)c * njobs + job) * (S * S) + tid];
    g[tid >> 4][tid & 15] = a;
  }
  __syncthreads();
  double* out = rinv + (int64_t)job * S * S;
  if (tid == 0) {
    double tr = 0.0;
    for (int i = 0; i < S; ++i) tr += g[i][i];
    if (!isfinite(tr)) {
      atomicExch(status, 1);
      tr = 0.0;
    }
    if (tr <= 0.0) {
      for (int e = 0; e < S * S; ++e) out[e] = 0.0;
    } else {
      const double sigma = 11.0 * ((double)T * S + S * (S + 1)) * 0x1p-53 * tr;
      for (int k = 0; k < S; ++k) {
        double d = g[k][k] + sigma;
        for (int i = 0; i < k; ++i) d -= R[i][k] * R[i][k];
        d = fmax(d, sigma);          // only reached through rounding
        const double rkk = sqrt(d);
        R[k][k] = rkk;
        for (int j = k + 1; j < S; ++j) {
          double v = g[k][j];
          for (int i = 0; i < k; ++i) v -= R[i][k] * R[i][j];
          R[k][j] = v / rkk;
        }
        for (int j = 0; j < k; ++j) R[k][j] = 0.0;
      }
      // R^{-1}, column by column by back substitution
      for (int j = 0; j < S; ++j) {
        double x[S];
        for (int i = 0; i < S; ++i) x[i] = 0.0;
        x[j] = 1.0 / R[j][j];
        for (int i = j - 1; i >= 0; --i) {
          double v = 0.0;
          for (int k = i + 1; k <= j; ++k) v += R[i][k] * x[k];
          x[i] = -v / R[i][i];
        }
        for (int i = 0; i < S; ++i) out[i * S + j] = x[i];
      }
    }
  }
}

// Q[job][t][:] <- Q[job][t][:] R^{-1}[job] (fp64 products, fp32 result), one
// row per thread.
__global__ void __launch_bounds__(256) k_grp_apply(float* __restrict__ Q, int T, const double* __restrict__ rinv) {
  __shared__ double ri[S * S];
  const int job = blockIdx.y;
  ri[threadIdx.x] = rinv[(int64_t)job * S * S + threadIdx.x];
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float* q = Q + ((int64_t)job * T + t) * S;
  double w[S];
#pragma unroll
  for (int c4 = 0; c4 < S / 4; ++c4) {
    const float4 v = *reinterpret_cast<const float4*>(q + 4 * c4);
    w[4 * c4 + 0] = v.x; w[4 * c4 + 1] = v.y; w[4 * c4 + 2] = v.z; w[4 * c4 + 3] = v.w;
  }
  float o[S];
#pragma unroll
  for (int c = 0; c < S; ++c) {
    double a = 0.0;
#pragma unroll
    for (int i = 0; i <= c; ++i) a = fma(w[i], ri[i * S + c], a);
    o[c] = (float)a;
  }
#pragma unroll
  for (int c4 = 0; c4 < S / 4; ++c4)
    *reinterpret_cast<float4*>(q + 4 * c4) = make_float4(o[4 * c4], o[4 * c4 + 1], o[4 * c4 + 2], o[4 * c4 + 3]);
}

// Rayleigh-Ritz, one job per block: C = Z^T Z (S x S, fp64, Z = X^T Q of the
// job), its eigenvectors by the cyclic Jacobi method (Golub & Van Loan,
// "Matrix Computations", Section 8.5: rotation angle from
// tau = (c_qq - c_pp) / (2 c_pq), t = sign(tau) / (|tau| + sqrt(1 + tau^2)),
// c = 1 / sqrt(1 + t^2), s = t c), run by one warp (lanes 0..S-1 update one
// row or column each), at most JACOBI_SWEEPS sweeps, rotations skipped below
// 1e-17 ||C||_F. The NV eigenvectors of the largest eigenvalues (lower
// index first on ties) go to Y[job] (S x NV, row-major).
constexpr int JACOBI_SWEEPS = 30;
__global__ void __launch_bounds__(256) k_grp_rr(const double* __restrict__ Z, int F, double* __restrict__ Y) {
  __shared__ double A[S][S + 1];
  __shared__ double V[S][S + 1];
  const int job = blockIdx.x, tid = threadIdx.x;
  {
    const int a = tid >> 4, c = tid & 15;
    const double* z = Z + (int64_t)job * F * S;
    double acc = 0.0;
    for (int f = 0; f < F; ++f) acc = fma(z[(int64_t)f * S + a], z[(int64_t)f * S + c], acc);
    A[a][c] = acc;
    V[a][c] = (a == c) ? 1.0 : 0.0;
  }
  __syncthreads();
  if (tid < 32) {
    const int lane = tid;
    double nrm = 0.0;
    for (int e = 0; e < S * S; ++e) nrm += A[e / S][e % S] * A[e / S][e % S];
    const double thresh = 1e-17 * sqrt(nrm);
    for (int sweep = 0; sweep < JACOBI_SWEEPS; ++sweep) {
      bool rotated = false;
      for (int p = 0; p < S - 1; ++p) {
        for (int q = p + 1; q < S; ++q) {
          __syncwarp();
          const double apq = A[p][q];
          if (!(fabs(apq) > thresh)) continue;
          const double app = A[p][p], aqq = A[q][q];
          const double tau = (aqq - app) / (2.0 * apq);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          const double c = 1.0 / sqrt(1.0 + t * t), s = t * c;
          __syncwarp();
          if (lane < S) {               // columns p, q of A and V
            const double akp = A[lane][p], akq = A[lane][q];
            A[lane][p] = c * akp - s * akq;
            A[lane][q] = s * akp + c * akq;
            const double vkp = V[lane][p], vkq = V[lane][q];
            V[lane][p] = c * vkp - s * vkq;
            V[lane][q] = s * vkp + c * vkq;
          }
          __syncwarp();
          if (lane < S) {               // rows p, q of A
            const double apk = A[p][lane], aqk = A[q][lane];
            A[p][lane] = c * apk - s * aqk;
            A[q][lane] = s * apk + c * aqk;
          }
          rotated = true;
        }
      }
      __syncwarp();
      if (!rotated) break;
    }
    __syncwarp();
    if (lane == 0) {
      bool used[S];
      for (int i = 0; i < S; ++i) used[i] = false;
      double* y = Y + (int64_t)job * S * NV;
      for (int k = 0; k < NV; ++k) {
        int best = -1;
        for (int i = 0; i < S; ++i)
          if (!used[i] && (best < 0 || A[i][i] > A[best][best])) best = i;
        used[best] = true;
        for (int i = 0; i < S; ++i) y[i * NV + k] = V[i][best];
      }
    }
  }
}

// Scores and groups, one block. Per (sequence b, layer l < L-1):
// M = Y_(b,l)^T (Q_(b,l)^T Q_(b,l+1)) Y_(b,l+1) from the cross-Gram partials,
// pscore = ||M||_F^2 / NV. score[l] = mean over b (b in order). Then the
// median of the L-1 scores (the middle one, or the mean of the two middle
// ones for an even count), and the rule: layer l opens a group when the
// current group holds GROUP_MAX layers, or holds at least GROUP_MIN layers
// and score[l-1] is strictly below the median; a trailing one-layer group
// joins its predecessor. out: scores[L-1] (double), then starts[L+1] and
// n_groups (int32).
constexpr int GROUP_MIN = 2, GROUP_MAX = 8;
__global__ void __launch_bounds__(256) k_grp_score(const double* __restrict__ Gx, int nchunk, int B, int L,
                                                   const double* __restrict__ Y, double* __restrict__ pscore,
                                                   double* __restrict__ scores, int* __restrict__ starts,
                                                   int* __restrict__ n_groups, int* __restrict__ status) {
  __shared__ double sc[MAX_LAYERS];
  __shared__ double srt[MAX_LAYERS];
  const int np = B * (L - 1), n = L - 1;
  for (int pj = threadIdx.x; pj < np; pj += blockDim.x) {
    const int b = pj / (L - 1), l = pj % (L - 1);
    const double* ya = Y + (int64_t)(b * L + l) * S * NV;
    const double* yb = Y + (int64_t)(b * L + l + 1) * S * NV;
    double M[NV][NV];
    for (int k = 0; k < NV; ++k)
      for (int m = 0; m < NV; ++m) M[k][m] = 0.0;
    for (int i = 0; i < S; ++i) {
      double gi[S];
      for (int j = 0; j < S; ++j) {
        double a = 0.0;
        for (int c = 0; c < nchunk; ++c) a += Gx[((int64_t)c * np + pj) * (S * S) + i * S + j];
        gi[j] = a;
      }
      for (int m = 0; m < NV; ++m) {
        double t = 0.0;
        for (int j = 0; j < S; ++j) t = fma(gi[j], yb[j * NV + m], t);
        for (int k = 0; k < NV; ++k) M[k][m] = fma(ya[i * NV + k], t, M[k][m]);
      }
    }
    double f2 = 0.0;
    for (int k = 0; k < NV; ++k)
      for (int m = 0; m < NV; ++m) f2 = fma(M[k][m], M[k][m], f2);
    pscore[pj] = f2 / NV;
  }
  __syncthreads();
  for (int l = threadIdx.x; l < n; l += blockDim.x) {
    double a = 0.0;
    for (int b = 0; b < B; ++b) a += pscore[b * (L - 1) + l];
    a /= B;
    if (!isfinite(a)) atomicExch(status, 1);
    sc[l] = a;
    scores[l] = a;
  }
  __syncthreads();
  // sorted copy by rank (equal values ranked by index)
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const double v = sc[i];
    int r = 0;
    for (int j = 0; j < n; ++j) r += (sc[j] < v) || (sc[j] == v && j < i);
    srt[r] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const double med = (n & 1) ? srt[n / 2] : (srt[n / 2 - 1] + srt[n / 2]) / 2.0;
    int ng = 0, size = 1;
    starts[ng++] = 0;
    for (int l = 1; l < L; ++l) {
      if (size >= GROUP_MAX || (size >= GROUP_MIN && sc[l - 1] < med)) {
        starts[ng++] = l;
        size = 1;
      } else {
        ++size;
      }
    }
    if (ng > 1 && L - starts[ng - 1] == 1) --ng;
    starts[ng] = L;
    *n_groups = ng;
  }
}

// ------------------------------------------------------------------ host ---
static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

struct Work {
  double *om, *Z, *P, *Gp, *rinv, *Y, *pscore, *scores;
  float* W;
  int *starts, *n_groups, *status;
  float2* cs;
};

template <int D>
static jolt_status launch_xz(const KeySrc& ks, const double* Z, int64_t zstride, float* W, int J, cudaStream_t st) {
  constexpr size_t smem = (size_t)(TM * (D + 1) + D * S) * sizeof(float);
  JOLT_CUDA_TRY(cudaFuncSetAttribute(k_grp_xz<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  k_grp_xz<D><<<dim3((ks.T + TM - 1) / TM, J), XZ_THREADS, smem, st>>>(ks, Z, zstride, W);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

template <int D>
static jolt_status launch_xtq(const KeySrc& ks, const float* Q, double* P, double* Z, int J, int nchunk,
                              cudaStream_t st) {
  constexpr size_t smem = (size_t)(TM * (D + 4) + TM * S) * sizeof(float);
  JOLT_CUDA_TRY(cudaFuncSetAttribute(k_grp_xtq<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  k_grp_xtq<D><<<dim3(nchunk, ks.H, J), 2 * D, smem, st>>>(ks, Q, P, J);
  JOLT_LAUNCHED();
  const int64_t n = (int64_t)J * ks.H * D * S;
  k_grp_zsum<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(P, nchunk, n, Z);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Q <- orth(Q): two passes of shifted Cholesky QR.
static jolt_status orth(const Work& w, int T, int L, int J, int ngc, cudaStream_t st) {
  for (int pass = 0; pass < 2; ++pass) {
    k_grp_gram<<<dim3(ngc, J), 256, 0, st>>>(w.W, T, L, 0, J, w.Gp);
    JOLT_LAUNCHED();
    k_grp_chol<<<J, 256, 0, st>>>(w.Gp, ngc, J, T, w.rinv, w.status);
    JOLT_LAUNCHED();
    k_grp_apply<<<dim3((T + 255) / 256, J), 256, 0, st>>>(w.W, T, w.rinv);
    JOLT_LAUNCHED();
  }
  return JOLT_OK;
}

template <int D>
static jolt_status run_groups(const KeySrc& ks, int B, int power_iters, uint64_t seed, const Work& w,
                              cudaStream_t st) {
  const int L = ks.L, T = ks.T, J = B * L, F = ks.H * D;
  const int nchunk = (T + TM * XTQ_TILES - 1) / (TM * XTQ_TILES);
  const int ngc = (T + GRAM_ROWS - 1) / GRAM_ROWS;
  k_grp_omega<<<(F * S / 4 + 255) / 256, 256, 0, st>>>(w.om, F, seed);
  JOLT_LAUNCHED();
  JOLT_TRY(launch_xz<D>(ks, w.om, 0, w.W, J, st));
  JOLT_TRY(orth(w, T, L, J, ngc, st));
  for (int it = 0; it < power_iters; ++it) {
    JOLT_TRY(launch_xtq<D>(ks, w.W, w.P, w.Z, J, nchunk, st));
    JOLT_TRY(launch_xz<D>(ks, w.Z, (int64_t)F * S, w.W, J, st));
    JOLT_TRY(orth(w, T, L, J, ngc, st));
  }
  JOLT_TRY(launch_xtq<D>(ks, w.W, w.P, w.Z, J, nchunk, st));
  k_grp_rr<<<J, 256, 0, st>>>(w.Z, F, w.Y);
  JOLT_LAUNCHED();
  const int np = B * (L - 1);
  k_grp_gram<<<dim3(ngc, np), 256, 0, st>>>(w.W, T, L, 1, np, w.Gp);
  JOLT_LAUNCHED();
  k_grp_score<<<1, 256, 0, st>>>(w.Gp, ngc, B, L, w.Y, w.pscore, w.scores, w.starts, w.n_groups, w.status);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace grp
}  // namespace jolt

using namespace jolt;

extern "C" jolt_status jolt_layer_groups(const jolt_layout* lay, const void* k, int32_t power_iters, uint64_t seed,
                                         double* scores, int32_t* group_start, int32_t* n_groups,
                                         jolt_stream_t stream_) {
  using namespace jolt::grp;
  if (!lay || !k || !group_start || !n_groups) { set_error("null layout/keys/group_start/n_groups"); return JOLT_ERR_INVALID_ARG; }
  const int B = lay->batch, L = lay->n_layers, H = lay->n_heads, T = lay->seq_len, D = lay->head_dim;
  if (B < 1 || L < 1 || H < 1 || T < 1) { set_error("non-positive layout dimension"); return JOLT_ERR_INVALID_ARG; }
  if (D != 64 && D != 128) { set_error("head_dim must be 64 or 128 (got %d)", D); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if (lay->dtype != JOLT_BF16 && lay->dtype != JOLT_F32) { set_error("dtype must be JOLT_BF16 or JOLT_F32"); return JOLT_ERR_INVALID_ARG; }
  if (lay->stride_t < D || lay->stride_h < 1 || lay->stride_l < 1 || lay->stride_b < 1) { set_error("bad strides"); return JOLT_ERR_INVALID_ARG; }
  if ((lay->stride_t | lay->stride_h | lay->stride_l | lay->stride_b) & 1) { set_error("layer grouping needs even strides"); return JOLT_ERR_INVALID_ARG; }
  if (((uintptr_t)k) & 7) { set_error("layer grouping needs 8-byte aligned keys"); return JOLT_ERR_INVALID_ARG; }
  if (lay->rope_theta_k < 0.0f) { set_error("rope_theta_k must be >= 0"); return JOLT_ERR_INVALID_ARG; }
  if (power_iters < 0 || power_iters > 32) { set_error("power_iters must be 0..32"); return JOLT_ERR_INVALID_ARG; }
  if (T < S) { set_error("layer grouping needs seq_len >= %d (got %d)", S, T); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if (L > MAX_LAYERS) { set_error("layer grouping supports up to %d layers (got %d)", MAX_LAYERS, L); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if ((int64_t)B * L > 65535) { set_error("layer grouping supports batch * n_layers <= 65535"); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if (L == 1) {
    group_start[0] = 0;
    group_start[1] = 1;
    *n_groups = 1;
    return JOLT_OK;
  }
  cudaStream_t st = (cudaStream_t)stream_;
  const int J = B * L, F = H * D, np = B * (L - 1);
  const int nchunk = (T + TM * XTQ_TILES - 1) / (TM * XTQ_TILES);
  const int ngc = (T + GRAM_ROWS - 1) / GRAM_ROWS;
  const bool rope = lay->rope_theta_k > 0.0f;
  const size_t b_om = round256((size_t)F * S * 8), b_W = round256((size_t)J * T * S * 4);
  const size_t b_Z = round256((size_t)J * F * S * 8), b_P = round256((size_t)nchunk * J * F * S * 8);
  const size_t b_G = round256((size_t)ngc * std::max(J, np) * S * S * 8), b_R = round256((size_t)J * S * S * 8);
  const size_t b_Y = round256((size_t)J * S * NV * 8), b_ps = round256((size_t)np * 8);
  const size_t b_out = round256((size_t)(L - 1) * 8 + (size_t)(L + 1 + 2) * 4);
  const size_t b_cs = rope ? round256((size_t)T * (D / 2) * 8) : 0;
  const size_t total = b_om + b_W + b_Z + b_P + b_G + b_R + b_Y + b_ps + b_out + b_cs;
  char* base = (char*)dev_alloc(total, st);
  if (!base) { set_error("device allocation of %zu bytes failed", total); return JOLT_ERR_OOM; }
  Work w{};
  char* p = base;
  w.om = (double*)p; p += b_om;
  w.W = (float*)p; p += b_W;
  w.Z = (double*)p; p += b_Z;
  w.P = (double*)p; p += b_P;
  w.Gp = (double*)p; p += b_G;
  w.rinv = (double*)p; p += b_R;
  w.Y = (double*)p; p += b_Y;
  w.pscore = (double*)p; p += b_ps;
  w.scores = (double*)p;
  w.starts = (int*)(p + (size_t)(L - 1) * 8);
  w.n_groups = w.starts + (L + 1);
  w.status = w.n_groups + 1;
  p += b_out;
  w.cs = rope ? (float2*)p : nullptr;
  KeySrc ks{k, lay->dtype == JOLT_F32 ? 1 : 0, lay->stride_b, lay->stride_l, lay->stride_h, lay->stride_t,
            L, H, T, D, w.cs};
  jolt_status rc = JOLT_OK;
  cudaError_t ce = cudaMemsetAsync(w.status, 0, sizeof(int), st);
  if (ce != cudaSuccess) { set_error("cudaMemsetAsync: %s", cudaGetErrorString(ce)); rc = JOLT_ERR_CUDA; }
  if (rc == JOLT_OK && rope) rc = launch_rope_table(T, D, (double)lay->rope_theta_k, w.cs, st);
  if (rc == JOLT_OK) rc = (D == 128) ? run_groups<128>(ks, B, power_iters, seed, w, st)
                                     : run_groups<64>(ks, B, power_iters, seed, w, st);
  std::vector<double> h_sc(L - 1);
  std::vector<int> h_out(L + 3);
  if (rc == JOLT_OK) {
    ce = cudaMemcpyAsync(h_sc.data(), w.scores, (size_t)(L - 1) * 8, cudaMemcpyDeviceToHost, st);
    if (ce == cudaSuccess)
      ce = cudaMemcpyAsync(h_out.data(), w.starts, (size_t)(L + 3) * 4, cudaMemcpyDeviceToHost, st);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
    if (ce != cudaSuccess) { set_error("layer grouping: %s", cudaGetErrorString(ce)); rc = JOLT_ERR_CUDA; }
  }
  dev_free(base, st);
  if (rc != JOLT_OK) return rc;
  const int ng = h_out[L + 1], stat = h_out[L + 2];
  if (stat) { set_error("layer grouping: non-finite Gram or score (keys hold Inf/NaN?)"); return JOLT_ERR_NONFINITE; }
  if (ng < 1 || ng > L) { set_error("layer grouping: bad group count %d", ng); return JOLT_ERR_CUDA; }
  for (int g = 0; g <= ng; ++g) group_start[g] = h_out[g];
  *n_groups = ng;
  if (scores)
    for (int l = 0; l < L - 1; ++l) scores[l] = h_sc[l];
  return JOLT_OK;
}
