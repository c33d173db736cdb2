// Rotated low-bit residual and decompression ("A JoLT for the KV Cache",
// Section 3, "Rotated low-bit residual"): E = X - X~, r = R E along the
// feature axis with R = D^-1/2 H_D diag(s) (seeded randomized Hadamard), per
// group absmax quantization to b bits with one fp32 scale, LSB-first
// packing; decoding dequantizes, applies R^T and adds the backbone
// X~ = U_T^ M^_lh. Keys get RoPE re-applied after decoding.
//
// This file holds the row-per-thread (SIMT) forms: the backbone product is
// summed in fp64 registers (so the residual is the one of the fp64
// reconstruction), the transform runs inside the thread. It
// also holds the page's own rotation, R = the Q of a seeded Gaussian's QR
// factorization, as an option: r = Q e and e = Q^T r are dense row products
// summed in fp64 and rounded once to fp32.
#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {

// fl32(1/sqrt(D)): the quotient and the root are correctly rounded in fp64, then
// rounded once to fp32.
__device__ __forceinline__ float rot_scale_f(int D) { return (float)(1.0 / sqrt((double)D)); }

template <int D>
__device__ __forceinline__ void rotate_row(float* e, const float* sgn) {
#pragma unroll
  for (int d = 0; d < D; ++d) e[d] = __fmul_rn(e[d], sgn[d]);
  fwht_row<D>(e);
  const float rs = rot_scale_f(D);
#pragma unroll
  for (int d = 0; d < D; ++d) e[d] = __fmul_rn(e[d], rs);
}

template <int D>
__device__ __forceinline__ void unrotate_row(float* v, const float* sgn) {
  fwht_row<D>(v);
  const float rs = rot_scale_f(D);
#pragma unroll
  for (int d = 0; d < D; ++d) v[d] = __fmul_rn(__fmul_rn(v[d], rs), sgn[d]);
}

// r_i = fl32(sum_j Q[i][j] e_j), j ascending, fp64 fused multiply-adds. buf is
// this thread's D floats of shared memory.
template <int D>
__device__ __forceinline__ void qr_rotate_row(float* v, const double* __restrict__ Q, float* buf) {
#pragma unroll
  for (int j = 0; j < D; ++j) buf[j] = v[j];
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const double* q = Q + i * D;
    double s = 0.0;
#pragma unroll 8
    for (int j = 0; j < D; ++j) s = fma(q[j], (double)buf[j], s);
    v[i] = (float)s;
  }
}

// e_j = fl32(sum_i Q[i][j] r_i), i ascending, fp64 fused multiply-adds.
template <int D>
__device__ __forceinline__ void qr_unrotate_row(float* v, const double* __restrict__ Q, float* buf) {
#pragma unroll
  for (int j = 0; j < D; ++j) buf[j] = v[j];
#pragma unroll
  for (int j = 0; j < D; ++j) {
    double s = 0.0;
#pragma unroll 8
    for (int i = 0; i < D; ++i) s = fma(Q[i * D + j], (double)buf[i], s);
    v[j] = (float)s;
  }
}

template <int D>
struct PackOp {
  float* e;
  uint8_t* codes;   // row base
  float* scales;    // row base
  template <int G, int B>
  __device__ __forceinline__ void run() { quantize_pack_row<D, G, B>(e, codes, scales); }
};

template <int D>
struct UnpackOp {
  float* v;
  const uint8_t* codes;
  const float* scales;
  template <int G, int B>
  __device__ __forceinline__ void run() { unpack_dequant_row<D, G, B>(codes, scales, v); }
};

// Columns [c0, c0 + W) of X~ row t of (cell, lh), summed in fp64:
// acc[j] = sum_r U_T^[t][r] M^[r][c0 + j]. Each product of two bf16 values is
// exact in fp64 and the sums keep 53 bits, so the result is the fp64 sum the
// reading of the residual (X - U_T^ M^ formed before any rounding to fp32)
// calls for. The U_T^ and M^ tiles are staged in shared memory 32 ranks at a
// time; every thread of the block takes part in the staging.
template <int D, int W>
__device__ __forceinline__ void backbone_cols(const ResidArgs& a, int cell, const CellOut& o, int lh, int t0,
                                              int c0, double* acc, float (*ms)[D], float (*us)[128]) {
  const int rmax = a.rmax_of[cell];
  const uint16_t* M = a.M[cell] + (int64_t)lh * rmax * D;
#pragma unroll
  for (int j = 0; j < W; ++j) acc[j] = 0.0;
  for (int r0 = 0; r0 < o.rT; r0 += 32) {
    for (int e = threadIdx.x; e < 32 * W; e += blockDim.x) {
      int rr = e / W, d = c0 + e % W;
      ms[rr][d] = (r0 + rr < o.rT) ? bf16_bits_to_f32(M[(int64_t)(r0 + rr) * D + d]) : 0.0f;
    }
    for (int e = threadIdx.x; e < 32 * 128; e += blockDim.x) {
      int rr = e / 128, tt = e % 128;
      int t = t0 + tt;
      us[rr][tt] = (r0 + rr < o.rT && t < o.t_pitch) ? bf16_bits_to_f32(o.ut[(int64_t)(r0 + rr) * o.t_pitch + t]) : 0.0f;
    }
    __syncthreads();
    for (int rr = 0; rr < 32; ++rr) {
      const double u = (double)us[rr][threadIdx.x];
#pragma unroll
      for (int j = 0; j < W; ++j) acc[j] = fma(u, (double)ms[rr][c0 + j], acc[j]);
    }
    __syncthreads();
  }
}

// Row t's backbone, four column quarters in turn (32 fp64 partial sums live
// at a time). Encoding (ENC): out = fl32(x - X~) from the fp64 sum, one
// rounding; decoding: out = fl32(X~).
template <int D, bool ENC>
__device__ __forceinline__ void backbone_row(const ResidArgs& a, const CellDesc& c, int cell, const CellOut& o,
                                             int lh, int t0, float* out, float (*ms)[D], float (*us)[128]) {
  constexpr int W = D / 4;
  const int t = t0 + threadIdx.x;
  const int l = lh / c.H, h = lh % c.H;
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    double acc[W];
    backbone_cols<D, W>(a, cell, o, lh, t0, qq * W, acc, ms, us);
    if (t < c.T) {
#pragma unroll
      for (int j = 0; j < W; ++j) {
        if constexpr (ENC) out[qq * W + j] = (float)((double)x_elem(c, a.cs, l, h, t, qq * W + j) - acc[j]);
        else out[qq * W + j] = (float)acc[j];
      }
    }
  }
}

template <int D, bool QR>
__global__ void __launch_bounds__(128) k_residual_simt(ResidArgs a) {
  extern __shared__ float rowbuf[];   // QR: [128][D + 1], one row per thread
  const int cell = blockIdx.z, lh = blockIdx.y, t0 = blockIdx.x * 128;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  if (o.b == 0 || lh >= c.Lg * c.H || t0 >= c.T) return;
  __shared__ float ms[32][D];
  __shared__ float us[32][128];
  __shared__ float sg[D];
  for (int d = threadIdx.x; d < D; d += blockDim.x) sg[d] = hadamard_sign(a.seed + c.seq, d);
  __syncthreads();
  float acc[D];
  backbone_row<D, true>(a, c, cell, o, lh, t0, acc, ms, us);   // E = X - X~
  const int t = t0 + threadIdx.x;
  if (t >= c.T) return;
  if constexpr (QR) qr_rotate_row<D>(acc, a.qrot + (int64_t)c.seq * D * D, rowbuf + threadIdx.x * (D + 1));
  else rotate_row<D>(acc, sg);
  const int64_t row = (int64_t)lh * c.T + t;
  PackOp<D> op{acc, o.codes + row * (o.b * D / 8), o.scales + row * (D / a.G)};
  dispatch_gb<D>(a.G, o.b, op);
}

template <int D, bool QR>
__global__ void __launch_bounds__(128) k_decompress_simt(ResidArgs a) {
  extern __shared__ float rowbuf[];   // QR: [128][D + 1], one row per thread
  const int cell = blockIdx.z, lh = blockIdx.y, t0 = blockIdx.x * 128;
  const CellDesc c = a.cells[cell];
  const CellOut o = a.out[cell];
  if (lh >= c.Lg * c.H || t0 >= c.T) return;
  __shared__ float ms[32][D];
  __shared__ float us[32][128];
  __shared__ float sg[D];
  for (int d = threadIdx.x; d < D; d += blockDim.x) sg[d] = hadamard_sign(a.seed + c.seq, d);
  __syncthreads();
  float acc[D];
  backbone_row<D, false>(a, c, cell, o, lh, t0, acc, ms, us);
  const int t = t0 + threadIdx.x;
  if (t >= c.T) return;
  const int l = lh / c.H, h = lh % c.H;
  if (o.b > 0) {
    float v[D];
    const int64_t row = (int64_t)lh * c.T + t;
    UnpackOp<D> op{v, o.codes + row * (o.b * D / 8), o.scales + row * (D / a.G)};
    dispatch_gb<D>(a.G, o.b, op);
    if constexpr (QR) qr_unrotate_row<D>(v, a.qrot + (int64_t)c.seq * D * D, rowbuf + threadIdx.x * (D + 1));
    else unrotate_row<D>(v, sg);
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = __fadd_rn(acc[d], v[d]);
  }
  if (c.rope) {
    constexpr int half = D / 2;
    const float2* cs = a.cs + (int64_t)t * half;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float2 q = cs[i];
      const float x0 = acc[i], x1 = acc[i + half];
      acc[i] = __fsub_rn(__fmul_rn(x0, q.x), __fmul_rn(x1, q.y));
      acc[i + half] = __fadd_rn(__fmul_rn(x1, q.x), __fmul_rn(x0, q.y));
    }
  }
  uint16_t* dst = (c.kind == 0 ? a.out_k : a.out_v) + (int64_t)c.seq * a.osb + (int64_t)(c.l0 + l) * a.osl +
                  (int64_t)h * a.osh + (int64_t)t * a.ost;
#pragma unroll
  for (int d = 0; d < D; d += 2) {
    uint32_t lo = bf16_bits_from_f32(acc[d]), hi = bf16_bits_from_f32(acc[d + 1]);
    *reinterpret_cast<uint32_t*>(dst + d) = lo | (hi << 16);
  }
}

template <class K>
static jolt_status launch_rows(K kern, dim3 g, size_t smem, const ResidArgs& a, cudaStream_t s) {
  if (smem) JOLT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  kern<<<g, 128, smem, s>>>(a);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_residual_simt(const ResidArgs& a, int ncells, int D, int Tmax, int lh_max,
                                 cudaStream_t s) {
  dim3 g((Tmax + 127) / 128, lh_max, ncells);
  const size_t qs = (size_t)128 * (D + 1) * sizeof(float);
  if (a.qrot) return D == 128 ? launch_rows(k_residual_simt<128, true>, g, qs, a, s)
                              : launch_rows(k_residual_simt<64, true>, g, qs, a, s);
  return D == 128 ? launch_rows(k_residual_simt<128, false>, g, 0, a, s)
                  : launch_rows(k_residual_simt<64, false>, g, 0, a, s);
}

jolt_status launch_decompress_simt(const ResidArgs& a, int ncells, int D, int Tmax, int lh_max,
                                   cudaStream_t s) {
  dim3 g((Tmax + 127) / 128, lh_max, ncells);
  const size_t qs = (size_t)128 * (D + 1) * sizeof(float);
  if (a.qrot) return D == 128 ? launch_rows(k_decompress_simt<128, true>, g, qs, a, s)
                              : launch_rows(k_decompress_simt<64, true>, g, qs, a, s);
  return D == 128 ? launch_rows(k_decompress_simt<128, false>, g, 0, a, s)
                  : launch_rows(k_decompress_simt<64, false>, g, 0, a, s);
}

// ---------------------------------------------------- QR-Gaussian rotation --
// Q of G = Q R for G a D x D matrix of standard normals (Philox4x32-10 words
// of counter (i, 0, STREAM_QRGAUSS, 0) with key seed + b, u = (w + 0.5) 2^-32,
// Box-Muller on (u0, u1) and (u2, u3); G[i][j] = z[i * D + j]). Householder
// reflections H_k = I - beta_k v_k v_k^T with v_k = x - alpha e_1,
// alpha = -sign(x_0) ||x|| (Golub & Van Loan, "Matrix Computations",
// Section 5.1-5.2), Q = H_0 ... H_(D-1) accumulated backwards from I, then
// column k negated where R_kk = alpha_k < 0 so that R's diagonal is positive.
// One block per sequence; A (overwritten by the reflectors) and Q live in
// global memory; reductions in a fixed order.
__global__ void __launch_bounds__(256) k_qr_rotation(int D, uint64_t seed, double* __restrict__ work,
                                                     double* __restrict__ qout) {
  __shared__ double red[256];
  __shared__ double alpha_s[128], beta_s[128];
  const int b = blockIdx.x, tid = threadIdx.x;
  double* A = work + (int64_t)b * D * D;
  double* Q = qout + (int64_t)b * D * D;
  for (int i4 = tid; i4 < D * D / 4; i4 += blockDim.x) {
    const u4 r = philox_at(seed + (uint64_t)b, STREAM_QRGAUSS, (uint32_t)i4);
    const double u0 = ((double)r.x + 0.5) * 0x1p-32, u1 = ((double)r.y + 0.5) * 0x1p-32;
    const double u2 = ((double)r.z + 0.5) * 0x1p-32, u3 = ((double)r.w + 0.5) * 0x1p-32;
    const double r0 = sqrt(-2.0 * log(u0)), r1 = sqrt(-2.0 * log(u2));
    const double t0 = 6.283185307179586 * u1, t1 = 6.283185307179586 * u3;
    A[4 * i4 + 0] = r0 * cos(t0);
    A[4 * i4 + 1] = r0 * sin(t0);
    A[4 * i4 + 2] = r1 * cos(t1);
    A[4 * i4 + 3] = r1 * sin(t1);
  }
  __syncthreads();
  for (int k = 0; k < D; ++k) {
    double part = 0.0;
    for (int i = k + 1 + tid; i < D; i += blockDim.x) part += A[i * D + k] * A[i * D + k];
    red[tid] = part;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
      if (tid < w) red[tid] += red[tid + w];
      __syncthreads();
    }
    const double tail = red[0];           // sum of squares below the diagonal
    const double x0 = A[k * D + k];
    const double nrm = sqrt(tail + x0 * x0);
    const double alpha = (x0 >= 0.0) ? -nrm : nrm;
    const double vk = x0 - alpha;
    const double vtv = vk * vk + tail;
    const double beta = vtv > 0.0 ? 2.0 / vtv : 0.0;
    __syncthreads();                      // every thread has read red[0] and A[k][k]
    if (tid == 0) {
      A[k * D + k] = vk;
      alpha_s[k] = alpha;
      beta_s[k] = beta;
    }
    __syncthreads();
    for (int j = k + 1 + tid; j < D; j += blockDim.x) {
      double w = 0.0;
      for (int i = k; i < D; ++i) w = fma(A[i * D + k], A[i * D + j], w);
      w *= beta;
      for (int i = k; i < D; ++i) A[i * D + j] = fma(-w, A[i * D + k], A[i * D + j]);
    }
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += blockDim.x) Q[e] = (e / D == e % D) ? 1.0 : 0.0;
  __syncthreads();
  for (int k = D - 1; k >= 0; --k) {
    const double beta = beta_s[k];
    for (int j = tid; j < D; j += blockDim.x) {
      double w = 0.0;
      for (int i = k; i < D; ++i) w = fma(A[i * D + k], Q[i * D + j], w);
      w *= beta;
      for (int i = k; i < D; ++i) Q[i * D + j] = fma(-w, A[i * D + k], Q[i * D + j]);
    }
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += blockDim.x)
    if (alpha_s[e % D] < 0.0) Q[e] = -Q[e];
}

jolt_status launch_qr_rotation(int D, int batch, uint64_t seed, double* work, double* q, cudaStream_t s) {
  if (D > 128 || D % 4) { set_error("QR rotation supports D <= 128, D % 4 == 0"); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  k_qr_rotation<<<batch, 256, 0, s>>>(D, seed, work, q);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------ residual stage alone -----
template <int D>
__global__ void __launch_bounds__(128) k_encode_rows(const float* __restrict__ e, int64_t rows, int b,
                                                     int G, uint64_t seed, uint8_t* codes, float* scales) {
  __shared__ float sg[D];
  for (int d = threadIdx.x; d < D; d += blockDim.x) sg[d] = hadamard_sign(seed, d);
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  float v[D];
#pragma unroll
  for (int d = 0; d < D; d += 4) {
    float4 q = *reinterpret_cast<const float4*>(e + row * D + d);
    v[d] = q.x; v[d + 1] = q.y; v[d + 2] = q.z; v[d + 3] = q.w;
  }
  rotate_row<D>(v, sg);
  PackOp<D> op{v, codes + row * (b * D / 8), scales + row * (D / G)};
  dispatch_gb<D>(G, b, op);
}

template <int D>
__global__ void __launch_bounds__(128) k_decode_rows(const uint8_t* __restrict__ codes,
                                                     const float* __restrict__ scales, int64_t rows,
                                                     int b, int G, uint64_t seed, float* e) {
  __shared__ float sg[D];
  for (int d = threadIdx.x; d < D; d += blockDim.x) sg[d] = hadamard_sign(seed, d);
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  float v[D];
  UnpackOp<D> op{v, codes + row * (b * D / 8), scales + row * (D / G)};
  dispatch_gb<D>(G, b, op);
  unrotate_row<D>(v, sg);
#pragma unroll
  for (int d = 0; d < D; d += 4)
    *reinterpret_cast<float4*>(e + row * D + d) = make_float4(v[d], v[d + 1], v[d + 2], v[d + 3]);
}

jolt_status launch_encode_rows(const float* e, int64_t rows, int D, int b, int G, uint64_t seed,
                               uint8_t* codes, float* scales, cudaStream_t s) {
  if (rows <= 0) return JOLT_OK;
  int64_t nb = (rows + 127) / 128;
  if (D == 128) k_encode_rows<128><<<(unsigned)nb, 128, 0, s>>>(e, rows, b, G, seed, codes, scales);
  else k_encode_rows<64><<<(unsigned)nb, 128, 0, s>>>(e, rows, b, G, seed, codes, scales);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_decode_rows(const uint8_t* codes, const float* scales, int64_t rows, int D,
                               int b, int G, uint64_t seed, float* e, cudaStream_t s) {
  if (rows <= 0) return JOLT_OK;
  int64_t nb = (rows + 127) / 128;
  if (D == 128) k_decode_rows<128><<<(unsigned)nb, 128, 0, s>>>(codes, scales, rows, b, G, seed, e);
  else k_decode_rows<64><<<(unsigned)nb, 128, 0, s>>>(codes, scales, rows, b, G, seed, e);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------------------ RoPE table ---
__global__ void k_rope_table(int T, int D, double theta, float2* cs) {
  const int half = D / 2;
  const int64_t n = (int64_t)T * half;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
    int t = (int)(k / half), i = (int)(k % half);
    double inv = pow(theta, -2.0 * (double)i / (double)D);
    double ang = (double)t * inv;
    cs[k] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

jolt_status launch_rope_table(int T, int D, double theta, float2* cs, cudaStream_t s) {
  int64_t n = (int64_t)T * (D / 2);
  int nb = (int)std::min<int64_t>((n + 255) / 256, 4096);
  k_rope_table<<<nb, 256, 0, s>>>(T, D, theta, cs);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
