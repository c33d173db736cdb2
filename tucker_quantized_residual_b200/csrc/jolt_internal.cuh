// Internal declarations shared by the CUDA translation units of libjolt.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <math.h>
#include <string>
#include <vector>

#include "../../include/jolt.h"

namespace jolt {

// ---------------------------------------------------------------- errors ---
void set_error(const char* fmt, ...);
uint64_t& launch_counter();

#define JOLT_CUDA_TRY(expr)                                                     \
  do {                                                                          \
    cudaError_t _e = (expr);                                                    \
    if (_e != cudaSuccess) {                                                    \
      ::jolt::set_error("%s failed: %s (%s:%d)", #expr, cudaGetErrorString(_e), \
                        __FILE__, __LINE__);                                    \
      return JOLT_ERR_CUDA;                                                     \
    }                                                                           \
  } while (0)

#define JOLT_LAUNCHED()                                                         \
  do {                                                                          \
    ++::jolt::launch_counter();                                                 \
    cudaError_t _e = cudaGetLastError();                                        \
    if (_e != cudaSuccess) {                                                    \
      ::jolt::set_error("kernel launch failed: %s (%s:%d)",                     \
                        cudaGetErrorString(_e), __FILE__, __LINE__);            \
      return JOLT_ERR_CUDA;                                                     \
    }                                                                           \
  } while (0)

#define JOLT_TRY(expr)                 \
  do {                                 \
    jolt_status _s = (expr);           \
    if (_s != JOLT_OK) return _s;      \
  } while (0)

// device status word bits (kernels OR these in; the host reads them at sync
// points and turns them into a jolt_status)
enum : int {
  DEV_ERR_EIG_NOCONV = 1,
  DEV_ERR_CHOL = 2,
  DEV_ERR_TIMEOUT = 4,
  DEV_ERR_NONFINITE = 8,
  DEV_ERR_INFEASIBLE = 16,
  DEV_ERR_MISMATCH = 32,   // gathered rate-distortion records do not fit this plan
};

// ------------------------------------------------------------- profiling ---
// Records a CUDA event pair around a stage when profiling is enabled.
struct ProfScope {
  ProfScope(int stage, cudaStream_t s);
  ~ProfScope();
  void end();
  int stage;
  cudaStream_t stream;
  uint64_t launches0;
  int slot;
};

// ------------------------------------------------------------- allocator ---
void* dev_alloc(size_t bytes, cudaStream_t s);
void dev_free(void* p, cudaStream_t s);

// ------------------------------------------------------------ rng / math ---
// Philox4x32-10 (Salmon et al., SC'11) from its published definition.
struct u4 { uint32_t x, y, z, w; };

__host__ __device__ inline u4 philox4x32_10(u4 c, uint32_t k0, uint32_t k1) {
  for (int i = 0; i < 10; ++i) {
    uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    c = u4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// stream tags in the third counter word
enum : uint32_t {
  STREAM_HADAMARD = 1,    // residual rotation signs
  STREAM_CALIB = 2,       // eps^2 calibration samples
  STREAM_SKETCH = 3,      // range-finder sketch Omega
  STREAM_QRGAUSS = 4,     // QR-Gaussian rotation matrix
  STREAM_GROUPING = 5     // layer-grouping sketch
};

__host__ __device__ inline u4 philox_at(uint64_t seed, uint32_t stream, uint32_t i, uint32_t hi = 0) {
  return philox4x32_10(u4{i, hi, stream, 0u}, (uint32_t)seed, (uint32_t)(seed >> 32));
}

// Hadamard sign s_i in {+1,-1}: bit 0 of word 0 of Philox((i,0,STREAM_HADAMARD,0)).
__host__ __device__ inline float hadamard_sign(uint64_t seed, int i) {
  return (philox_at(seed, STREAM_HADAMARD, (uint32_t)i).x & 1u) ? -1.0f : 1.0f;
}

// Round a double to the nearest bf16 (ties to even) in one step, returned as
// the raw 16-bit pattern. Finite inputs of bf16 range only.
__host__ __device__ inline uint16_t bf16_bits_from_f64(double x) {
  uint64_t u;
  memcpy(&u, &x, 8);
  uint64_t sign = u & 0x8000000000000000ull;
  uint64_t mag = u & 0x7FFFFFFFFFFFFFFFull;
  int e = (int)(mag >> 52);                      // biased exponent
  if (mag == 0) return (uint16_t)(sign >> 48);
  // bf16 normal range: unbiased >= -126 -> biased >= 897
  if (e >= 897) {
    // keep 7 explicit mantissa bits of 52: drop 45 bits with ties-to-even
    uint64_t lsb = (mag >> 45) & 1ull;
    uint64_t r = mag + 0x0FFFFFFFFFFFull + lsb;   // 2^44 - 1 + lsb
    r &= ~((1ull << 45) - 1);
    double y;
    uint64_t yb = sign | r;
    memcpy(&y, &yb, 8);
    float f = (float)y;                           // exact: y has 8 significant bits
    uint32_t fb;
    memcpy(&fb, &f, 4);
    return (uint16_t)(fb >> 16);
  }
  // below the bf16 normal range: fixed spacing 2^-133
  double q = rint(fabs(x) * 0x1p133);
  double y = q * 0x1p-133;
  float f = (float)(sign ? -y : y);
  uint32_t fb;
  memcpy(&fb, &f, 4);
  return (uint16_t)(fb >> 16);
}

__host__ __device__ inline float bf16_bits_to_f32(uint16_t b) {
  uint32_t fb = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &fb, 4);
  return f;
}

__device__ inline uint16_t bf16_bits_from_f32(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

// --------------------------------------------------------------- cells ----
// One cell = (sequence b, group g, kind K|V): X[l][h][t][d], l < Lg.
struct CellDesc {
  const void* src;        // &cache[b][l0][0][0][0] of K or V
  int64_t sl, sh, st;     // strides in elements
  int Lg, H, T, D;
  int kind;               // 0 = K, 1 = V
  int rope;               // 1: un-RoPE keys on load
  int f32;                // 1: fp32 input, else bf16
  int seq;                // sequence index (seed offset)
  int l0;                 // first layer of the group
  int nt;                 // length of the token spectrum fed to the allocator
  int rtmax;              // largest token rank on the grid
};

// cos/sin table for RoPE: cs[t*(D/2)+i] = (cos, sin)(t * theta^(-2i/D)), fp32
__device__ __forceinline__ float load_elem(const CellDesc& c, int l, int h, int t, int d) {
  int64_t off = (int64_t)l * c.sl + (int64_t)h * c.sh + (int64_t)t * c.st + d;
  if (c.f32) return reinterpret_cast<const float*>(c.src)[off];
  return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(c.src)[off]);
}

// Element of the compression target: un-RoPE'd keys in fp32 with no fused
// multiply-add (x_i = y_i c + y_j s; x_j = y_j c - y_i s), values as stored.
__device__ __forceinline__ float x_elem(const CellDesc& c, const float2* __restrict__ cs,
                                        int l, int h, int t, int d) {
  if (!c.rope) return load_elem(c, l, h, t, d);
  int half = c.D >> 1;
  if (d < half) {
    float yi = load_elem(c, l, h, t, d), yj = load_elem(c, l, h, t, d + half);
    float2 q = cs[(int64_t)t * half + d];
    return __fadd_rn(__fmul_rn(yi, q.x), __fmul_rn(yj, q.y));
  } else {
    int i = d - half;
    float yi = load_elem(c, l, h, t, i), yj = load_elem(c, l, h, t, d);
    float2 q = cs[(int64_t)t * half + i];
    return __fsub_rn(__fmul_rn(yj, q.x), __fmul_rn(yi, q.y));
  }
}

// ----------------------------------------------------- residual rows -------
// Unnormalised natural-order Walsh-Hadamard transform of one row held by one
// thread, fp32, stages h = 1, 2, ..., D/2 with (a, b) -> (a + b, a - b).
template <int D>
__device__ __forceinline__ void fwht_row(float* v) {
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < D; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        float a = v[j], b = v[j + h];
        v[j] = __fadd_rn(a, b);
        v[j + h] = __fsub_rn(a, b);
      }
    }
  }
}

__host__ __device__ inline int qmax_of(int b) { return (1 << (b - 1)) - 1; }

// fl32(a / b) without a divide instruction, by residual corrections
// (P. Markstein, "IA-64 and Elementary Functions", 2000). With rb = RN(1/b),
// q0 = RN(a * rb) is within 1.5 ulp of a / b; one correction
// q1 = RN(q0 + (a - q0 b) rb), the residual exact in one fused multiply-add,
// brings it within one ulp, and by Markstein's theorem a second correction
// from such an estimate returns the correctly rounded quotient. Valid while b
// and 1/b are normal numbers (quot_ok); callers bring b into that range by an
// exact power-of-two scaling of both operands otherwise.
__device__ __forceinline__ bool quot_ok(float b) { return b >= 1e-30f && b <= 1e30f; }
__device__ __forceinline__ float quot_rn(float a, float b, float rb) {
  const float q0 = __fmul_rn(a, rb);
  const float q1 = __fmaf_rn(__fmaf_rn(-q0, b, a), rb, q0);
  return __fmaf_rn(__fmaf_rn(-q1, b, a), rb, q1);
}

// Quantize + pack one rotated row r[D] (fp32) with groups of G values and B
// bits: scale = fl32(absmax / q_max), code = clamp(rint(fl32(r / scale))),
// u = code + 2^(B-1) stored LSB first. codes: B*D/8 bytes (8-byte aligned);
// scales: D/G floats.
template <int D, int G, int B>
__device__ __forceinline__ void quantize_pack_row(const float* r, uint8_t* __restrict__ codes,
                                                  float* __restrict__ scales) {
  constexpr int NW = (B * D) / 64;
  const float qm = (float)qmax_of(B);
  uint64_t words[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) words[w] = 0ull;
#pragma unroll
  for (int g0 = 0; g0 < D; g0 += G) {
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < G; ++j) a = fmaxf(a, fabsf(r[g0 + j]));
    const float sc = __fdiv_rn(a, qm);
    scales[g0 / G] = sc;
    // quotients by quot_rn; a scale outside its range is first brought into
    // it by an exact power-of-two factor applied to both operands
    const float m = quot_ok(sc) ? 1.0f : (sc < 1.0f ? 18446744073709551616.0f : 5.421010862427522e-20f);
    const float sm = __fmul_rn(sc, m), rsm = (sc > 0.0f) ? __frcp_rn(sm) : 0.0f;
#pragma unroll
    for (int j = 0; j < G; ++j) {
      int q = 0;
      if (sc > 0.0f) {
        const float y = quot_rn(__fmul_rn(r[g0 + j], m), sm, rsm);
        q = (int)fminf(fmaxf(rintf(y), -qm), qm);
      }
      const uint64_t u = (uint64_t)(uint32_t)(q + (1 << (B - 1)));
      const int bit = (g0 + j) * B;
      const int wi = bit >> 6, sh = bit & 63;
      words[wi] |= u << sh;
      if (sh + B > 64) words[wi + 1] |= u >> (64 - sh);
    }
  }
  uint64_t* dst = reinterpret_cast<uint64_t*>(codes);
#pragma unroll
  for (int w = 0; w < NW; ++w) dst[w] = words[w];
}

// Unpack + dequantize one row into v[D] (fp32): v_i = fl32((u_i - 2^(B-1)) * scale).
template <int D, int G, int B>
__device__ __forceinline__ void unpack_dequant_row(const uint8_t* __restrict__ codes,
                                                   const float* __restrict__ scales, float* v) {
  constexpr int NW = (B * D) / 64;
  uint64_t words[NW + 1];
  const uint64_t* src = reinterpret_cast<const uint64_t*>(codes);
#pragma unroll
  for (int w = 0; w < NW; ++w) words[w] = src[w];
  words[NW] = 0ull;
  constexpr uint64_t mask = (1ull << B) - 1ull;
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const int bit = i * B;
    const int wi = bit >> 6, sh = bit & 63;
    uint64_t u = words[wi] >> sh;
    if (sh + B > 64) u |= words[wi + 1] << (64 - sh);
    const int q = (int)(u & mask) - (1 << (B - 1));
    v[i] = __fmul_rn((float)q, scales[i / G]);
  }
}

// Calls f.template operator()<G, B>() for the runtime (G, B) pair; returns
// false for an unsupported pair.
template <int D, class F>
__device__ __forceinline__ bool dispatch_gb(int G, int B, F& f) {
#define JOLT_GB(g, b) if (G == g && B == b) { f.template run<g, b>(); return true; }
  JOLT_GB(D, 2) JOLT_GB(D, 3) JOLT_GB(D, 4) JOLT_GB(D, 8)
  JOLT_GB(64, 2) JOLT_GB(64, 3) JOLT_GB(64, 4) JOLT_GB(64, 8)
  JOLT_GB(32, 2) JOLT_GB(32, 3) JOLT_GB(32, 4) JOLT_GB(32, 8)
#undef JOLT_GB
  return false;
}

// ------------------------------------------------ thread-block clusters ----
// Rank of this CTA in its cluster.
__device__ __forceinline__ uint32_t tc_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Generic address of the same shared-memory location in CTA `rank` of the
// cluster (plain loads through it read that CTA's shared memory).
__device__ __forceinline__ const double* tc_peer(const double* local, uint32_t rank) {
  uint64_t a;
  asm("mapa.u64 %0, %1, %2;" : "=l"(a) : "l"(reinterpret_cast<uint64_t>(local)), "r"(rank));
  return reinterpret_cast<const double*>(a);
}
// Every thread of every CTA of the cluster; writes before it are visible to
// the cluster's reads after it.
__device__ __forceinline__ void tc_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace jolt
