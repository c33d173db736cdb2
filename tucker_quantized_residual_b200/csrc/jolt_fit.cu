// The ST-HOSVD fit of one cell after the allocation has fixed (r_T, r_d, b):
// "A JoLT for the KV Cache", Section 3, "Partial Tucker backbone": the token
// mode is truncated first, then the feature factor is computed on the
// projected tensor. Stored factors are bf16 (c = 2 in Eq. 1):
//   U_T^ = bf16(U_T[:, :r_T]),  Y = X x_T U_T^T,
//   U_d  = leading eigenvectors of the feature Gram of Y, U_d^ = bf16(U_d),
//   G^   = bf16(Y x_d U_d^T),   M^_lh = bf16(G^_lh U_d^^T)  (decoder product).
// Every sum here is fp64 over exact products of bf16/fp32 values.
#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {

__device__ __forceinline__ double bf16d(uint16_t b) { return (double)bf16_bits_to_f32(b); }

// Place each cell's sections in the payload: U_T^ (transposed), U_d^, G^,
// codes, scales, each 256-byte aligned. One thread.
__global__ void k_payload_layout(const CellDesc* __restrict__ cells, const Choice* __restrict__ ch,
                                 int ncells, int G, uint8_t* base, int64_t capacity,
                                 CellOut* __restrict__ out, int* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    int64_t o = off;
    off += (bytes + 255) & ~(int64_t)255;
    return o;
  };
  for (int c = 0; c < ncells; ++c) {
    const CellDesc cd = cells[c];
    const Choice k = ch[c];
    CellOut o;
    const int64_t LH = (int64_t)cd.Lg * cd.H;
    o.rT = k.rT; o.rd = k.rd; o.b = k.b;
    o.t_pitch = (cd.T + 7) & ~7;
    o.bytes = k.bytes;
    o.ut = reinterpret_cast<uint16_t*>(base + take((int64_t)k.rT * o.t_pitch * 2));
    o.ud = reinterpret_cast<uint16_t*>(base + take((int64_t)cd.D * k.rd * 2));
    o.core = reinterpret_cast<uint16_t*>(base + take(LH * k.rT * k.rd * 2));
    if (k.b > 0) {
      o.codes = base + take(LH * cd.T * (k.b * cd.D / 8));
      o.scales = reinterpret_cast<float*>(base + take(LH * cd.T * (cd.D / G) * 4));
    } else {
      o.codes = nullptr;
      o.scales = nullptr;
    }
    out[c] = o;
  }
  if (off > capacity) {
    // never reached when the allocation met the budget; if it did not, every
    // cell gets empty sections so that no later kernel writes past the payload
    atomicOr(status, DEV_ERR_INFEASIBLE);
    for (int c = 0; c < ncells; ++c) {
      CellOut o{};
      o.t_pitch = (cells[c].T + 7) & ~7;
      out[c] = o;
    }
  }
}

jolt_status launch_payload_layout(const CellDesc* cells, const Choice* ch, int ncells, int G,
                                  uint8_t* base, int64_t capacity, CellOut* out, int* status,
                                  cudaStream_t s) {
  k_payload_layout<<<1, 32, 0, s>>>(cells, ch, ncells, G, base, capacity, out, status);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ---------------------------------------------------------- token factor ---
// T <= N: U_T = leading eigenvectors of X_(T) X_(T)^T (already sign-fixed).
__global__ void k_ut_from_eig(FitArgs a) {
  const int cell = blockIdx.z, r = blockIdx.y;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  if (r >= o.rT || c.T > c.Lg * c.H * c.D) return;
  const double* v = a.VtT[cell] + (int64_t)r * c.T;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < o.t_pitch; t += gridDim.x * blockDim.x)
    o.ut[(int64_t)r * o.t_pitch + t] = (t < c.T) ? bf16_bits_from_f64(v[t]) : (uint16_t)0;
}

// T > N: U_T[:, r] = X_(T) v_r / sigma_r (fp64) into Uf[r][t].
__global__ void k_ut_from_right(FitArgs a) {
  const int cell = blockIdx.z, r = blockIdx.y;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  const int N = c.Lg * c.H * c.D;
  if (r >= o.rT || c.T <= N) return;
  const double* v = a.VtT[cell] + (int64_t)r * N;
  const double w = a.wT[cell][r];
  const double inv = (w > 0.0) ? 1.0 / sqrt(w) : 0.0;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= c.T) return;
  double acc = 0.0;
  for (int n = 0; n < N; ++n) {
    int lh = n / c.D;
    acc += (double)x_elem(c, a.cs, lh / c.H, lh % c.H, t, n % c.D) * v[n];
  }
  a.Uf[cell][(int64_t)r * c.T + t] = acc * inv;
}

// Sign-fix (largest |.| positive, first on ties) and store bf16, T > N case.
__global__ void __launch_bounds__(256) k_ut_signfix(FitArgs a) {
  const int cell = blockIdx.y, r = blockIdx.x;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  if (r >= o.rT || c.T <= c.Lg * c.H * c.D) return;
  const double* u = a.Uf[cell] + (int64_t)r * c.T;
  double best = -1.0;
  int bi = 0x7fffffff;
  for (int t = threadIdx.x; t < c.T; t += blockDim.x) {
    double x = fabs(u[t]);
    if (x > best) { best = x; bi = t; }
  }
  __shared__ double sb[256];
  __shared__ int si[256];
  sb[threadIdx.x] = best;
  si[threadIdx.x] = bi;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {
    if (threadIdx.x < off) {
      double ob = sb[threadIdx.x + off];
      int oi = si[threadIdx.x + off];
      if (ob > sb[threadIdx.x] || (ob == sb[threadIdx.x] && oi < si[threadIdx.x])) {
        sb[threadIdx.x] = ob;
        si[threadIdx.x] = oi;
      }
    }
    __syncthreads();
  }
  const double sg = (u[si[0]] < 0.0) ? -1.0 : 1.0;
  for (int t = threadIdx.x; t < o.t_pitch; t += blockDim.x)
    o.ut[(int64_t)r * o.t_pitch + t] = (t < c.T) ? bf16_bits_from_f64(sg * u[t]) : (uint16_t)0;
}

jolt_status launch_ut_exact(const FitArgs& a, int Tmax, int rmax_all, cudaStream_t s) {
  dim3 g1((Tmax + 255) / 256, rmax_all, a.ncells);
  k_ut_from_eig<<<g1, 256, 0, s>>>(a);
  JOLT_LAUNCHED();
  k_ut_from_right<<<g1, 256, 0, s>>>(a);
  JOLT_LAUNCHED();
  dim3 g2(rmax_all, a.ncells);
  k_ut_signfix<<<g2, 256, 0, s>>>(a);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------------------ projection ---
// Y[lh][r][d] = sum_t U_T^[t][r] x[lh][t][d]   (fp64)
template <int D>
__global__ void __launch_bounds__(256) k_project_y(FitArgs a) {
  constexpr int RB = 16, TB = 32, PD = D / 16;
  __shared__ double us[RB][TB + 1];
  __shared__ double xs[TB][D + 1];
  const int cell = blockIdx.z, lh = blockIdx.x, r0 = blockIdx.y * RB;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  if (lh >= c.Lg * c.H || r0 >= o.rT) return;
  const int l = lh / c.H, h = lh % c.H;
  const int ri = threadIdx.x / 16, dj = threadIdx.x % 16;
  double acc[PD];
#pragma unroll
  for (int k = 0; k < PD; ++k) acc[k] = 0.0;
  for (int t0 = 0; t0 < c.T; t0 += TB) {
    for (int e = threadIdx.x; e < RB * TB; e += blockDim.x) {
      int rr = e / TB, tt = e % TB;
      int r = r0 + rr, t = t0 + tt;
      us[rr][tt] = (r < o.rT && t < c.T) ? bf16d(o.ut[(int64_t)r * o.t_pitch + t]) : 0.0;
    }
    for (int e = threadIdx.x; e < TB * D; e += blockDim.x) {
      int tt = e / D, d = e % D;
      int t = t0 + tt;
      xs[tt][d] = (t < c.T) ? (double)x_elem(c, a.cs, l, h, t, d) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < TB; ++tt) {
      const double u = us[ri][tt];
#pragma unroll
      for (int k = 0; k < PD; ++k) acc[k] = fma(u, xs[tt][dj * PD + k], acc[k]);
    }
    __syncthreads();
  }
  const int r = r0 + ri;
  if (r < o.rT) {
    double* y = a.Y[cell] + ((int64_t)lh * a.rmax_of[cell] + r) * D;
#pragma unroll
    for (int k = 0; k < PD; ++k) y[dj * PD + k] = acc[k];
  }
}

jolt_status launch_project_y(const FitArgs& a, int /*Tmax*/, int rmax_all, int lh_max, cudaStream_t s) {
  dim3 g(lh_max, (rmax_all + 15) / 16, a.ncells);
  if (a.D == 128) k_project_y<128><<<g, 256, 0, s>>>(a);
  else k_project_y<64><<<g, 256, 0, s>>>(a);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ----------------------------------------------------- feature factor/core --
// U_d^[d][j] = bf16(eigenvector j of the projected feature Gram)[d], j < r_d
__global__ void k_ud_store(FitArgs a) {
  const int cell = blockIdx.x;
  const CellOut o = a.out[cell];
  const int D = a.D;
  const double* v = a.VtY[cell];
  for (int e = threadIdx.x; e < D * o.rd; e += blockDim.x) {
    int d = e / o.rd, j = e % o.rd;
    o.ud[e] = bf16_bits_from_f64(v[(int64_t)j * D + d]);
  }
}

// One block per (CORE_R rows r, lh): G^ rows and M^ rows. The core reads
// U_d^[d][j] across the threads j (consecutive), M^ reads U_d^ staged
// transposed in shared memory ([j][d], consecutive across the threads d);
// each value is the same fp64 sum in the same order (d, then j ascending) as
// a block per row. Shared memory: 48 KB at D = 128.
constexpr int CORE_R = 8;
template <int D>
__global__ void __launch_bounds__(D) k_core(FitArgs a) {
  const int cell = blockIdx.z, lh = blockIdx.y, r0 = blockIdx.x * CORE_R;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  if (lh >= c.Lg * c.H || r0 >= o.rT) return;
  __shared__ double y[CORE_R][D];
  __shared__ double g[CORE_R][D];
  __shared__ uint16_t udt[D * D];    // [j][d], j < rd
  const int rd = o.rd, nr = min(CORE_R, o.rT - r0);
  const int rmax = a.rmax_of[cell];
  for (int e = threadIdx.x; e < D * rd; e += D) udt[(e % rd) * D + e / rd] = o.ud[e];
  for (int i = 0; i < nr; ++i) y[i][threadIdx.x] = a.Y[cell][((int64_t)lh * rmax + r0 + i) * D + threadIdx.x];
  __syncthreads();
  const int j = threadIdx.x;
  if (j < rd) {
    for (int i = 0; i < nr; ++i) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += y[i][d] * bf16d(o.ud[d * rd + j]);
      const uint16_t gb = bf16_bits_from_f64(acc);
      o.core[((int64_t)lh * o.rT + r0 + i) * rd + j] = gb;
      g[i][j] = bf16d(gb);
    }
  }
  __syncthreads();
  const int d = threadIdx.x;
  for (int i = 0; i < nr; ++i) {
    double m = 0.0;
    for (int jj = 0; jj < rd; ++jj) m += g[i][jj] * bf16d(udt[jj * D + d]);
    a.M[cell][((int64_t)lh * rmax + r0 + i) * D + d] = bf16_bits_from_f64(m);
  }
}

jolt_status launch_core(const FitArgs& a, int rmax_all, int lh_max, cudaStream_t s) {
  k_ud_store<<<a.ncells, 256, 0, s>>>(a);
  JOLT_LAUNCHED();
  dim3 g((rmax_all + CORE_R - 1) / CORE_R, lh_max, a.ncells);
  if (a.D == 128) k_core<128><<<g, 128, 0, s>>>(a);
  else k_core<64><<<g, 64, 0, s>>>(a);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt

namespace jolt {

__global__ void k_copy_rt(const CellOut* out, int* rt, int ncells) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < ncells) rt[c] = out[c].rT;
}

__global__ void k_copy_out(const CellOut* out, int* rt, uint16_t** ut, int ncells) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < ncells) { rt[c] = out[c].rT; ut[c] = out[c].ut; }
}

jolt_status launch_copy_out(const CellOut* out, int* rt, uint16_t** ut, int ncells, cudaStream_t s) {
  k_copy_out<<<(ncells + 127) / 128, 128, 0, s>>>(out, rt, ut, ncells);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_copy_rt(const CellOut* out, int* rt, int ncells, cudaStream_t s) {
  k_copy_rt<<<(ncells + 127) / 128, 128, 0, s>>>(out, rt, ncells);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Decoder product from the stored payload: M^[lh][r][d] = bf16(sum_j G^[lh][r][j] U_d^[d][j]),
// the same fp64 sum order as at compression, so the values match bit for bit.
// CORE_R rows per block, U_d^ staged transposed in shared memory.
template <int D>
__global__ void __launch_bounds__(D) k_core_m(const CellOut* __restrict__ outs, const CellDesc* __restrict__ cells,
                                              uint16_t* const* __restrict__ M, const int* __restrict__ rmax_of) {
  const int cell = blockIdx.z, lh = blockIdx.y, r0 = blockIdx.x * CORE_R;
  const CellDesc c = cells[cell];
  const CellOut o = outs[cell];
  if (lh >= c.Lg * c.H || r0 >= o.rT) return;
  __shared__ double g[CORE_R][D];
  __shared__ uint16_t udt[D * D];    // [j][d]
  const int rd = o.rd, nr = min(CORE_R, o.rT - r0);
  for (int e = threadIdx.x; e < D * rd; e += D) udt[(e % rd) * D + e / rd] = o.ud[e];
  for (int i = 0; i < nr; ++i)
    if ((int)threadIdx.x < rd) g[i][threadIdx.x] = bf16d(o.core[((int64_t)lh * o.rT + r0 + i) * rd + threadIdx.x]);
  __syncthreads();
  const int d = threadIdx.x;
  for (int i = 0; i < nr; ++i) {
    double m = 0.0;
    for (int j = 0; j < rd; ++j) m += g[i][j] * bf16d(udt[j * D + d]);
    M[cell][((int64_t)lh * rmax_of[cell] + r0 + i) * D + d] = bf16_bits_from_f64(m);
  }
}

jolt_status launch_core_m(const CellOut* out, const CellDesc* cells, uint16_t* const* M, const int* rmax_of,
                          int ncells, int D, int rmax_all, int lh_max, cudaStream_t s) {
  dim3 g((rmax_all + CORE_R - 1) / CORE_R, lh_max, ncells);
  if (D == 128) k_core_m<128><<<g, 128, 0, s>>>(out, cells, M, rmax_of);
  else k_core_m<64><<<g, 64, 0, s>>>(out, cells, M, rmax_of);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
