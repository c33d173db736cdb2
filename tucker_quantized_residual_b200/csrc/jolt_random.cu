// Randomized token-mode range finder ("A JoLT for the KV Cache", Section 3.1,
// "FlashJoLT"): a Gaussian sketch plus power iterations give the leading q_cap
// token-mode singular values and vectors; the energy they miss is appended as
// one synthetic tail entry (||X||^2 minus the computed energy).
//
// The subspace iteration is carried on the feature side, where matrices are
// N x k (N = L_g H D, small) instead of T x k:
//   W_0 = X Omega;  for i: Z_i = X^T W_{i-1}, V_i = Z_i R_i^{-1} (CholeskyQR
//   in fp64), W_i = X V_i;  Z = X^T W_q.
// range(W_q) = range((X X^T)^q X Omega), the subspace of the usual
// power-iterated sketch. With G_W = W_q^T W_q = R^T R, Q = W_q R^{-1} is
// orthonormal, B = Q^T X = R^{-T} Z^T and B B^T = R^{-T} (Z^T Z) R^{-1}; its
// eigenpairs (sigma~^2, U_B) give U_T = Q U_B = W_q (R^{-1} U_B). The
// projection Y = U_T^T X used by the fit is (Z R^{-1} U_B)^T, no extra pass
// over X.
#include <cudaTypedefs.h>

#include <mutex>

#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"
#define JOLT_UMMA_IMPL
#include "jolt_umma.cuh"

namespace jolt {

// ------------------------------------------------------------- tensor maps --
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static jolt_status make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) { set_error("cuTensorMapEncodeTiled unavailable"); return JOLT_ERR_CUDA; }
  uint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { set_error("cuTensorMapEncodeTiled failed (%d)", (int)r); return JOLT_ERR_CUDA; }
  return JOLT_OK;
}

jolt_status map_x5(CUtensorMap* m, const void* base, int B, int L, int H, int T, int D, int64_t sb, int64_t sl,
                   int64_t sh, int64_t st) {
  uint64_t dims[5] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)L, (uint64_t)B};
  uint64_t str[4] = {(uint64_t)st * 2, (uint64_t)sh * 2, (uint64_t)sl * 2, (uint64_t)sb * 2};
  uint32_t box[5] = {64, 64, 1, 1, 1};
  return make_map(m, base, 5, dims, str, box);
}

jolt_status map_x5_box(CUtensorMap* m, const void* base, int B, int L, int H, int T, int D, int64_t sb,
                       int64_t sl, int64_t sh, int64_t st, int box_t) {
  uint64_t dims[5] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)L, (uint64_t)B};
  uint64_t str[4] = {(uint64_t)st * 2, (uint64_t)sh * 2, (uint64_t)sl * 2, (uint64_t)sb * 2};
  uint32_t box[5] = {64, (uint32_t)box_t, 1, 1, 1};
  return make_map(m, base, 5, dims, str, box);
}

jolt_status map_3d_box(CUtensorMap* m, const void* base, int cells, int rows, int cols, int64_t pitch,
                       int box_cols, int box_rows) {
  uint64_t dims[3] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)cells};
  uint64_t str[2] = {(uint64_t)pitch * 2, (uint64_t)pitch * 2 * rows};
  uint32_t box[3] = {(uint32_t)box_cols, (uint32_t)box_rows, 1};
  return make_map(m, base, 3, dims, str, box);
}

// [cells][rows][cols] bf16 with row pitch `pitch` elements; box {64, box_rows}
jolt_status map_3d(CUtensorMap* m, const void* base, int cells, int rows, int cols, int64_t pitch,
                   int box_rows) {
  uint64_t dims[3] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)cells};
  uint64_t str[2] = {(uint64_t)pitch * 2, (uint64_t)pitch * 2 * rows};
  uint32_t box[3] = {64, (uint32_t)box_rows, 1};
  return make_map(m, base, 3, dims, str, box);
}

static int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

jolt_status launch_umma(const umma::Maps& maps, const umma::Problem& p, cudaStream_t s) {
  const int ntiles = p.ncells * p.mt * p.nt;
  if (ntiles == 0) return JOLT_OK;
  const int bn_max = (p.pair && p.wide) ? 2 * umma::BN_MAX : umma::BN_MAX;
  if (p.BN % 16 || p.BN < 16 || p.BN > bn_max) { set_error("bad GEMM tile width %d", p.BN); return JOLT_ERR_INVALID_ARG; }
  if (p.wide) {
    // wide tiles: CTA pairs only, at most 4 N tiles, each two MMAs 16..256
    // wide (multiples of 16) that together fit the widest tile
    bool ok = p.pair && p.nt >= 1 && p.nt <= 4;
    for (int j = 0; ok && j < p.nt; ++j)
      ok = p.ta[j] % 16 == 0 && p.tb[j] % 16 == 0 && p.ta[j] >= 16 && p.tb[j] >= 16 && p.ta[j] <= umma::BN_MAX &&
           p.tb[j] <= umma::BN_MAX && p.ta[j] + p.tb[j] <= p.BN && p.tn0[j] + p.ta[j] + p.tb[j] <= p.N;
    if (!ok) { set_error("bad wide GEMM tiling"); return JOLT_ERR_INVALID_ARG; }
  }
  static bool attr = false;
  if (!attr) {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(umma::k_umma_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       umma::SMEM_DATA_MAX + 1024 + 256));
    attr = true;
  }
  if (p.pair) {
    if ((p.mode != umma::XW && p.mode != umma::XTY) || (p.BN / 2) % 8) {
      set_error("CTA-pair GEMM: X W / X^T Y only, BN/2 a multiple of 8 (BN=%d)", p.BN);
      return JOLT_ERR_INVALID_ARG;
    }
    static bool attr2 = false;
    if (!attr2) {
      JOLT_CUDA_TRY(cudaFuncSetAttribute(umma::k_umma_gemm_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         umma::SMEM_DATA_MAX + 1024 + 256));
      attr2 = true;
    }
    const int mt2 = (p.M + 2 * umma::BM - 1) / (2 * umma::BM);
    const int tiles2 = p.ncells * mt2 * p.nt;
    const int pairs = std::max(1, std::min(tiles2, num_sms() / 2));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(umma::THREADS);
    cfg.dynamicSmemBytes = umma::pair_smem_bytes(p.BN);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    JOLT_CUDA_TRY(cudaLaunchKernelEx(&cfg, umma::k_umma_gemm_pair, maps, p));
    JOLT_LAUNCHED();
    return JOLT_OK;
  }
  const int grid = std::min(ntiles, num_sms());
  umma::k_umma_gemm<<<grid, umma::THREADS, umma::smem_bytes(p.BN), s>>>(maps, p);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// --------------------------------------------------- bf16 working copies ---
// dst (contiguous [B][L][H][T][D] bf16) = bf16_rne(x), x the compression
// target: un-RoPE'd keys in fp32 (rope != 0) or the stored values.
// One thread per (token, 8 rotation pairs) of one (b, l, h) row block
// (blockIdx.y); vec != 0: bf16 input with 16-byte aligned rows, read as
// 8-element vectors, and the cos/sin pairs as float4.
__global__ void __launch_bounds__(256) k_make_xb(const void* __restrict__ src, int f32, int rope, int vec,
                                                 const float2* __restrict__ cs, int L, int H, int T, int D,
                                                 int64_t sb, int64_t sl, int64_t sh, int64_t st,
                                                 uint16_t* __restrict__ dst) {
  const int half = D / 2;
  const int per_row = half / 8;              // 8-pair blocks per row
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= T * per_row) return;
  const int t = e / per_row, i0 = (e - t * per_row) * 8;
  const int blh = blockIdx.y;
  const int h = blh % H, l = (blh / H) % L, b = blh / (H * L);
  const int64_t off = (int64_t)b * sb + (int64_t)l * sl + (int64_t)h * sh + (int64_t)t * st;
  float y0[8], y1[8];
  if (vec) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(src) + off;
    const uint4 w0 = *reinterpret_cast<const uint4*>(p + i0);
    const uint4 w1 = *reinterpret_cast<const uint4*>(p + half + i0);
    const uint32_t a0[4] = {w0.x, w0.y, w0.z, w0.w}, a1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      y0[2 * j] = __uint_as_float(a0[j] << 16);
      y0[2 * j + 1] = __uint_as_float(a0[j] & 0xFFFF0000u);
      y1[2 * j] = __uint_as_float(a1[j] << 16);
      y1[2 * j + 1] = __uint_as_float(a1[j] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (f32) {
        y0[j] = reinterpret_cast<const float*>(src)[off + i0 + j];
        y1[j] = reinterpret_cast<const float*>(src)[off + half + i0 + j];
      } else {
        y0[j] = bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(src)[off + i0 + j]);
        y1[j] = bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(src)[off + half + i0 + j]);
      }
    }
  }
  uint32_t o0[4], o1[4];
  const float4* cs4 = rope ? reinterpret_cast<const float4*>(cs + (int64_t)t * half + i0) : nullptr;
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    float a[2] = {y0[j], y0[j + 1]}, c[2] = {y1[j], y1[j + 1]};
    if (rope) {
      const float4 q = cs4[j / 2];
      const float cc[2] = {q.x, q.z}, ss[2] = {q.y, q.w};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        a[u] = __fadd_rn(__fmul_rn(y0[j + u], cc[u]), __fmul_rn(y1[j + u], ss[u]));
        c[u] = __fsub_rn(__fmul_rn(y1[j + u], cc[u]), __fmul_rn(y0[j + u], ss[u]));
      }
    }
    o0[j / 2] = (uint32_t)bf16_bits_from_f32(a[0]) | ((uint32_t)bf16_bits_from_f32(a[1]) << 16);
    o1[j / 2] = (uint32_t)bf16_bits_from_f32(c[0]) | ((uint32_t)bf16_bits_from_f32(c[1]) << 16);
  }
  uint16_t* d = dst + ((int64_t)blh * T + t) * D;
  *reinterpret_cast<uint4*>(d + i0) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
  *reinterpret_cast<uint4*>(d + half + i0) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
}

jolt_status launch_make_xb(const void* src, int f32, int rope, const float2* cs, int B, int L, int H, int T,
                           int D, int64_t sb, int64_t sl, int64_t sh, int64_t st, uint16_t* dst,
                           cudaStream_t s) {
  if ((int64_t)B * L * H > 65535) { set_error("too many (b, l, h) rows for the copy kernel"); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  const int vec = !f32 && ((sb | sl | sh | st) % 8 == 0) && (reinterpret_cast<uintptr_t>(src) % 16 == 0);
  dim3 g((T * (D / 16) + 255) / 256, B * L * H);
  k_make_xb<<<g, 256, 0, s>>>(src, f32, rope, vec, cs, L, H, T, D, sb, sl, sh, st, dst);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------------- Gaussian sketch ---
// W^T[cell][j][n] = bf16(N(0,1)) for n < N_c(cell), 0 beyond. Four normals per
// Philox4x32-10 call (Box-Muller on (w0, w1) and (w2, w3), fp64), counter
// (e/4, cell_in_sequence, STREAM_SKETCH, 0) with e = j * ld + n, key = seed + b.
__global__ void k_omega(uint16_t* __restrict__ wt, int ncells, int k, int ld, const int* __restrict__ Nc,
                        const int* __restrict__ seq, const int* __restrict__ cis, uint64_t seed) {
  const int cell = blockIdx.y;
  const int64_t n4 = (int64_t)k * ld / 4;
  uint16_t* w = wt + (int64_t)cell * k * ld;
  const int nc = Nc[cell];
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const u4 r = philox_at(seed + (uint64_t)seq[cell], STREAM_SKETCH, (uint32_t)i, (uint32_t)cis[cell]);
    const double u0 = ((double)r.x + 0.5) * 0x1p-32, u1 = ((double)r.y + 0.5) * 0x1p-32;
    const double u2 = ((double)r.z + 0.5) * 0x1p-32, u3 = ((double)r.w + 0.5) * 0x1p-32;
    const double r0 = sqrt(-2.0 * log(u0)), r1 = sqrt(-2.0 * log(u2));
    const double t0 = 6.283185307179586 * u1, t1 = 6.283185307179586 * u3;
    const double z[4] = {r0 * cos(t0), r0 * sin(t0), r1 * cos(t1), r1 * sin(t1)};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t e = 4 * i + c;
      const int n = (int)(e % ld);
      w[e] = (n < nc) ? bf16_bits_from_f64(z[c]) : (uint16_t)0;
    }
  }
}

jolt_status launch_omega(uint16_t* wt, int ncells, int k, int ld, const int* Nc, const int* seq, const int* cis,
                         uint64_t seed, cudaStream_t s) {
  const int64_t n4 = (int64_t)k * ld / 4;
  dim3 g((unsigned)std::min<int64_t>((n4 + 255) / 256, 1024), ncells);
  k_omega<<<g, 256, 0, s>>>(wt, ncells, k, ld, Nc, seq, cis, seed);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

__global__ void k_symmetrize(double* __restrict__ M, int64_t cs, int k) {
  const int cell = blockIdx.y;
  double* m = M + (int64_t)cell * cs;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < (int64_t)k * k; e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / k), j = (int)(e % k);
    if (i < j) {
      const double a = 0.5 * (m[(int64_t)i * k + j] + m[(int64_t)j * k + i]);
      m[(int64_t)i * k + j] = a;
      m[(int64_t)j * k + i] = a;
    }
  }
}

jolt_status launch_symmetrize(double* M, int64_t cs, int k, int ncells, cudaStream_t s) {
  dim3 g2(64, ncells);
  k_symmetrize<<<g2, 256, 0, s>>>(M, cs, k);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Token spectrum for the allocator: the q leading eigenvalues of B B^T and the
// synthetic tail max(0, ||X||^2 - sum of them) (Section 3.1).
__global__ void k_rand_spectrum(const double* __restrict__ w_eig, int64_t cs, int q, const double* const* __restrict__ normsq,
                                double* const* __restrict__ wT) {
  const int cell = blockIdx.x;
  if (threadIdx.x != 0) return;
  const double* w = w_eig + (int64_t)cell * cs;
  double s = 0.0;
  double* o = wT[cell];
  for (int i = 0; i < q; ++i) {
    const double x = fmax(w[i], 0.0);
    o[i] = x;
    s += x;
  }
  o[q] = fmax(*normsq[cell] - s, 0.0);
}

jolt_status launch_rand_spectrum(const double* w_eig, int64_t cs, int q, const double* const* normsq,
                                 double* const* wT, int ncells, cudaStream_t s) {
  k_rand_spectrum<<<ncells, 32, 0, s>>>(w_eig, cs, q, normsq, wT);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Y[lh][r][d] = sum_j Z[(lh*D + d)][j] P[j][r]   (fp64)
template <int D>
__global__ void __launch_bounds__(256) k_yproj(const float* __restrict__ Z, int64_t z_cell, const double* __restrict__ P64,
                                               int64_t p_cell, int k, int rmax, const CellOut* __restrict__ outs,
                                               const int* __restrict__ nlh, double* const* __restrict__ Y) {
  constexpr int RB = 16, JB = 32, PD = D / 16;
  __shared__ double zs[JB][D + 1];
  __shared__ double ps[JB][RB];
  const int cell = blockIdx.z, lh = blockIdx.x, r0 = blockIdx.y * RB;
  const int rT = outs[cell].rT;
  if (lh >= nlh[cell] || r0 >= rT) return;
  const float* z = Z + (int64_t)cell * z_cell + (int64_t)lh * D * k;
  const double* p = P64 + (int64_t)cell * p_cell;
  const int ri = threadIdx.x / 16, dj = threadIdx.x % 16;
  double acc[PD] = {};
  for (int j0 = 0; j0 < k; j0 += JB) {
    for (int e = threadIdx.x; e < JB * D; e += blockDim.x) {
      const int jj = e % JB, d = e / JB;
      zs[jj][d] = (j0 + jj < k) ? (double)z[(int64_t)d * k + j0 + jj] : 0.0;
    }
    for (int e = threadIdx.x; e < JB * RB; e += blockDim.x) {
      const int jj = e / RB, rr = e % RB;
      ps[jj][rr] = (j0 + jj < k && r0 + rr < rT) ? p[(int64_t)(j0 + jj) * rmax + r0 + rr] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < JB; ++jj) {
      const double pv = ps[jj][ri];
#pragma unroll
      for (int q = 0; q < PD; ++q) acc[q] = fma(zs[jj][dj * PD + q], pv, acc[q]);
    }
    __syncthreads();
  }
  const int r = r0 + ri;
  if (r < rT) {
    double* y = Y[cell] + ((int64_t)lh * rmax + r) * D;
#pragma unroll
    for (int q = 0; q < PD; ++q) y[dj * PD + q] = acc[q];
  }
}

jolt_status launch_yproj(const float* Z, int64_t z_cell, const double* P64, int64_t p_cell, int k, int rmax,
                         const CellOut* outs, const int* nlh, double* const* Y, int lh_max, int D, int ncells,
                         cudaStream_t s) {
  dim3 g(lh_max, (rmax + 15) / 16, ncells);
  if (D == 128) k_yproj<128><<<g, 256, 0, s>>>(Z, z_cell, P64, p_cell, k, rmax, outs, nlh, Y);
  else k_yproj<64><<<g, 256, 0, s>>>(Z, z_cell, P64, p_cell, k, rmax, outs, nlh, Y);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// Feature Gram from the fp32 tensor-core partials: C[cell][i][j] =
// sum over chunks (fixed order) of the D x D diagonal blocks of the 128 x 128
// partial tiles; ||X||^2 = trace(C).
__global__ void k_fgram_reduce(const float* __restrict__ part, int nchunk, int D, double* const* __restrict__ C,
                               double* const* __restrict__ normsq) {
  const int cell = blockIdx.y;
  const int nblk = 128 / D;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < D * D; e += gridDim.x * blockDim.x) {
    const int i = e / D, j = e % D;
    double s = 0.0;
    for (int c = 0; c < nchunk; ++c) {
      const float* t = part + ((int64_t)cell * nchunk + c) * 128 * 128;
      for (int b = 0; b < nblk; ++b) s += (double)t[(b * D + i) * 128 + b * D + j];
    }
    C[cell][e] = s;
  }
}

__global__ void k_trace(double* const* __restrict__ C, int D, double* const* __restrict__ normsq) {
  const int cell = blockIdx.x;
  if (threadIdx.x != 0) return;
  double s = 0.0;
  for (int i = 0; i < D; ++i) s += C[cell][i * D + i];
  *normsq[cell] = s;
}

jolt_status launch_fgram_reduce(const float* part, int nchunk, int D, double* const* C, double* const* normsq,
                                int ncells, cudaStream_t s) {
  dim3 g((D * D + 255) / 256, ncells);
  k_fgram_reduce<<<g, 256, 0, s>>>(part, nchunk, D, C, normsq);
  JOLT_LAUNCHED();
  k_trace<<<ncells, 32, 0, s>>>(C, D, normsq);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
