// Device helpers of the tensor-core row kernels (the residual / decompress
// stream of jolt_stream.cu and the fused decode attention of
// jolt_decode.cu): TMEM loads and stores, the two-thread-per-row
// Walsh-Hadamard transform, the b-bit quantizer and its packing, and the
// warp-role barriers. Included by those translation units only.
#pragma once
#define JOLT_PTX_HELPERS
#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"
#include "jolt_umma.cuh"

namespace jolt {
namespace strm {

using namespace umma;

constexpr int SBM = 128;
constexpr int SSTAGES = 3;
constexpr int S_A = 128 * 64 * 2;          // U_T^ slice: 128 tokens x 64 ranks
constexpr int S_B = 128 * 64 * 2;          // M^T slice: D rows x 64 ranks (D <= 128)
constexpr int S_X = 128 * 128 * 2;         // input tile: 128 tokens x D
constexpr int S_CODE = 128 * 128;          // packed codes of a tile (<= 8 bits x 128 per row)
constexpr int S_SCALE = 128 * 4 * 4;       // scales of a tile (<= 4 groups per row)
constexpr int S_R1 = (2 * S_X > 2 * (S_CODE + S_SCALE)) ? 2 * S_X : 2 * (S_CODE + S_SCALE);
constexpr int SMEM_STREAM = SSTAGES * (S_A + S_B) + S_R1 + 128 * 16 + 128 * 4 + 1024 + 512;
// the four-threads-per-row stream kernel: code rows staged with a 16-byte pad
constexpr int S_CODEP = 128 * (128 + 16);
constexpr int S_R1Q = (2 * S_X > 2 * (S_CODEP + S_SCALE)) ? 2 * S_X : 2 * (S_CODEP + S_SCALE);
static_assert(S_R1Q <= S_R1 + 8192, "stream staging");
constexpr int SMEM_STREAM4 = SSTAGES * (S_A + S_B) + S_R1Q + 128 * 8 * 4 + 128 * 4 + 1024 + 512;
constexpr int EPI_WARPS = 8;
constexpr int STHREADS = 64 + 32 * EPI_WARPS;

struct Args {
  int ncells, T, H, lhmax, rpad_m, G, ntile_t;
  const CellDesc* cells;
  const CellOut* outs;
  const float2* cs;
  const float4* csq;
  uint64_t seed;
  uint16_t* out_k;
  uint16_t* out_v;
  int64_t osb, osl, osh, ost;
  int* status;
};

struct SMaps {
  CUtensorMap ut;   // [cells][rows][tp] bf16, box {64 t, 64 r}
  CUtensorMap mt;   // [cells*lhmax][D][rpad_m] bf16, box {64 r, D}
  CUtensorMap xk;   // inputs, box {64 d, 128 t, 1, 1, 1}
  CUtensorMap xv;
};

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float* v);
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, float* v) { tmem_ld16(taddr, v); }
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two fp32 values rounded to bf16 (nearest, ties to even), lo in the low half.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * EPI_WARPS) : "memory"); }
// Barrier of the two warps that share a TMEM lane quarter (64 threads).
__device__ __forceinline__ void pair_sync(int q) { asm volatile("bar.sync %0, 64;" ::"r"(2 + q) : "memory"); }
// AND of `ok` over the epilogue threads: every one of them takes the same
// branch after a bounded wait, so none is left at a named barrier alone.
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(32 * EPI_WARPS)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool tile_of(const Args& a, int tile, int& cell, int& t0, int& lh, CellDesc& c,
                                        CellOut& o, bool compress) {
  const int per_cell = a.ntile_t * a.lhmax;
  cell = tile / per_cell;
  const int r = tile - cell * per_cell;
  t0 = (r / a.lhmax) * SBM;
  lh = r % a.lhmax;
  c = a.cells[cell];
  o = a.outs[cell];
  if (lh >= c.Lg * c.H || t0 >= c.T) return false;
  if (compress && o.b == 0) return false;
  return o.rT > 0;
}

// Byte extents of a decoded tile's codes and scales, and whether each can be
// fetched by one bulk copy (16-byte aligned start and length).
struct CodeTile {
  const uint8_t* codes;
  const float* scales;
  uint32_t cbytes, sbytes;
  bool cbulk, sbulk;
};
__device__ __forceinline__ CodeTile code_tile(const CellOut& o, int64_t row0, int nrows, int D, int G) {
  CodeTile ct;
  const int rowbytes = o.b * D / 8, ng = D / G;
  ct.codes = o.codes + row0 * rowbytes;
  ct.scales = o.scales + row0 * ng;
  ct.cbytes = (uint32_t)(nrows * rowbytes);
  ct.sbytes = (uint32_t)(nrows * ng * 4);
  ct.cbulk = ((reinterpret_cast<uintptr_t>(ct.codes) | ct.cbytes) & 15u) == 0;
  ct.sbulk = ((reinterpret_cast<uintptr_t>(ct.scales) | ct.sbytes) & 15u) == 0;
  return ct;
}

// 8 bf16 of row r starting at column col (multiple of 8) of the
// 128-byte-swizzled input tile (64-column boxes of 128 rows).
__device__ __forceinline__ void ld_x8(const uint8_t* xs, int r, int col, float* o) {
  const int box = col >> 6, ch = (col & 63) >> 3;
  const uint4 w = *reinterpret_cast<const uint4*>(xs + box * 16384 + r * 128 + ((ch ^ (r & 7)) << 4));
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o[2 * j] = __uint_as_float(u[j] << 16);
    o[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
  }
}

// Walsh-Hadamard stages of span 1 .. C/2 on one chunk of C values.
template <int C>
__device__ __forceinline__ void fwht_chunk(float* v) {
#pragma unroll
  for (int h = 1; h < C; h <<= 1) {
#pragma unroll
    for (int i = 0; i < C; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = v[j], b = v[j + h];
        v[j] = __fadd_rn(a, b);
        v[j + h] = __fsub_rn(a, b);
      }
    }
  }
}

template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const float* v);
template <>
__device__ __forceinline__ void tmem_st<16>(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<32>(uint32_t taddr, const float* v) {
  tmem_st<16>(taddr, v);
  tmem_st<16>(taddr + 16, v + 16);
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Full transform of the thread's 2C values: in-chunk stages, the span-C stage
// with the partner half, then the span-D/2 stage between the two chunks.
// The partner's values come through tensor memory: each thread stores its
// 2C values in its own TMEM lane at columns xcol + hf * 2C (xcol alternates
// between two regions from tile to tile, so a region is rewritten only after
// the partner has passed the next pair barrier), and reads the partner's
// columns after the barrier.
template <int C>
__device__ __forceinline__ void fwht_pair(float* e, uint32_t lane_base, uint32_t xcol, int hf, int q) {
  fwht_chunk<C>(e);
  fwht_chunk<C>(e + C);
  const uint32_t mine = lane_base + xcol + (uint32_t)(hf * 2 * C);
  const uint32_t theirs = lane_base + xcol + (uint32_t)((hf ^ 1) * 2 * C);
  tmem_st<C>(mine, e);
  tmem_st<C>(mine + C, e + C);
  tmem_wait_st();
  fence_before();
  pair_sync(q);
  fence_after();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float p[C];
    tmem_ld<C>(theirs + k * C, p);
    float* v = e + k * C;
#pragma unroll
    for (int j = 0; j < C; ++j)   // half 0 holds the lower index of each pair (a + b), half 1 the upper (a - b)
      v[j] = hf == 0 ? __fadd_rn(v[j], p[j]) : __fsub_rn(p[j], v[j]);
  }
#pragma unroll
  for (int j = 0; j < C; ++j) {
    const float a = e[j], b = e[j + C];
    e[j] = __fadd_rn(a, b);
    e[j + C] = __fsub_rn(a, b);
  }
}

// b-bit codes of one chunk of C values with one scale: code =
// clamp(rint(fl32(r / sc))). The quotient is taken as r * fl32(1/sc) and
// replaced by the correctly rounded one wherever the product lies within
// 1e-4 of a rounding boundary (it differs from the quotient by at most
// 128 * 2^-23 < 2e-5 there), so the codes equal the divided ones. Rounding
// to the nearest integer (ties to even) is the fp32 addition of
// 1.5 * 2^23 + 2^(b-1), whose low b mantissa bits then hold u = code + 2^(b-1),
// packed LSB first.
// Bit-field insert: the low `len` bits of a into b at bit `pos` (constant
// pos and len after unrolling).
__device__ __forceinline__ uint32_t bfi(uint32_t a, uint32_t b, int pos, int len) {
  uint32_t d;
  asm("bfi.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(pos), "r"(len));
  return d;
}

template <int C, int B>
__device__ __forceinline__ void quant_chunk(const float* r, float sc, uint32_t* w) {
  constexpr int NW = (C * B + 31) / 32;
  constexpr uint32_t mask = (1u << B) - 1u;
  // 1.5 * 2^23 + 2^(b-1): the sum's low b bits are u = rint(y) + 2^(b-1)
  constexpr float magic = 12582912.0f + (float)(1 << (B - 1));
  const float qm = (float)((1 << (B - 1)) - 1);
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0u;
  if (sc > 0.0f) {
    const float inv = __frcp_rn(sc);
    uint32_t need = 0u;
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const float y = fminf(fmaxf(__fmul_rn(r[i], inv), -qm), qm);
      const float t = __fadd_rn(y, magic);
      if (!(0.5f - fabsf(__fsub_rn(y, __fsub_rn(t, magic))) >= 1e-4f)) need |= 1u << i;
      const uint32_t u = __float_as_uint(t);
      const int bit = i * B, wi = bit >> 5, sh = bit & 31;
      // insert the low bits of u (one bit-field insert masks them)
      if (sh + B <= 32) {
        w[wi] = bfi(u, w[wi], sh, B);
      } else {
        w[wi] |= (u & mask) << sh;
        w[wi + 1] |= (u & mask) >> (32 - sh);
      }
    }
    if (need) {
#pragma unroll
      for (int i = 0; i < C; ++i) {
        if (!((need >> i) & 1u)) continue;
        const float qf = fminf(fmaxf(rintf(__fdiv_rn(r[i], sc)), -qm), qm);
        const uint32_t u = (uint32_t)((int)qf + (1 << (B - 1)));
        const int bit = i * B, wi = bit >> 5, sh = bit & 31;
        w[wi] = (w[wi] & ~(mask << sh)) | (u << sh);
        if (sh + B > 32) w[wi + 1] = (w[wi + 1] & ~(mask >> (32 - sh))) | (u >> (32 - sh));
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const uint32_t u = 1u << (B - 1);
      const int bit = i * B, wi = bit >> 5, sh = bit & 31;
      w[wi] |= u << sh;
      if (sh + B > 32) w[wi + 1] |= u >> (32 - sh);
    }
  }
}

template <int C, int B>
__device__ __forceinline__ void dequant_chunk(const uint32_t* w, float sc, float* v) {
  // u in the low mantissa bits of 2^23 gives 2^23 + u exactly; subtracting
  // 2^23 + 2^(b-1) leaves the code as a float
  constexpr uint32_t mask = (1u << B) - 1u;
  constexpr float off = 8388608.0f + (float)(1 << (B - 1));
#pragma unroll
  for (int i = 0; i < C; ++i) {
    const int bit = i * B, wi = bit >> 5, sh = bit & 31;
    uint32_t u;
    if (sh + B <= 32) u = (w[wi] >> sh) & mask;
    else u = __funnelshift_r(w[wi], w[wi + 1], sh) & mask;
    const float q = __fsub_rn(__uint_as_float(0x4B000000u | u), off);
    v[i] = __fmul_rn(q, sc);
  }
}

// Chunk bits (C * B of them, a multiple of 16) to / from memory: 32-bit
// units when C = 32 (4-byte aligned offsets), 16-bit units otherwise.
template <int C, int B>
__device__ __forceinline__ void store_bits(uint8_t* p, const uint32_t* w) {
  if constexpr (C == 32 && B == 2) {
    *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
  } else if constexpr (C == 32 && (B == 4 || B == 8)) {
#pragma unroll
    for (int i = 0; i < B; i += 4) *reinterpret_cast<uint4*>(p + 4 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
  } else if constexpr (C == 32) {
    uint32_t* d = reinterpret_cast<uint32_t*>(p);
#pragma unroll
    for (int i = 0; i < B; ++i) d[i] = w[i];
  } else {
    uint16_t* d = reinterpret_cast<uint16_t*>(p);
#pragma unroll
    for (int i = 0; i < C * B / 16; ++i) d[i] = (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
  }
}
template <int C, int B>
__device__ __forceinline__ void load_bits(const uint8_t* p, uint32_t* w) {
  if constexpr (C == 32 && B == 2) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    w[0] = x.x; w[1] = x.y;
  } else if constexpr (C == 32 && (B == 4 || B == 8)) {
#pragma unroll
    for (int i = 0; i < B; i += 4) {
      const uint4 x = *reinterpret_cast<const uint4*>(p + 4 * i);
      w[i] = x.x; w[i + 1] = x.y; w[i + 2] = x.z; w[i + 3] = x.w;
    }
  } else if constexpr (C == 32) {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = s[i];
  } else {
    const uint16_t* s = reinterpret_cast<const uint16_t*>(p);
#pragma unroll
    for (int i = 0; i < (C * B + 31) / 32; ++i) w[i] = 0u;
#pragma unroll
    for (int i = 0; i < C * B / 16; ++i) w[i >> 1] |= (uint32_t)s[i] << (16 * (i & 1));
  }
}

// Chunk maxima of both halves -> scale of each of this thread's chunks;
// the thread whose chunk opens a group stores the group's scale.
template <int D>
__device__ __forceinline__ void chunk_scales(const float* am, float* pm, int r, int hf, int q, int G, float qm,
                                             float* sc, float* srow) {
  constexpr int C = D / 4;
  pm[(r * 2 + hf) * 2 + 0] = am[0];
  pm[(r * 2 + hf) * 2 + 1] = am[1];
  pair_sync(q);
  float part[2];
  part[0] = pm[(r * 2 + (hf ^ 1)) * 2 + 0];
  part[1] = pm[(r * 2 + (hf ^ 1)) * 2 + 1];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int s0 = k * (D / 2) + hf * C, g = s0 / G;
    float a = 0.0f;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int s1 = kk * (D / 2) + hh * C;
        if (s1 / G == g) a = fmaxf(a, hh == hf ? am[kk] : part[kk]);
      }
    sc[k] = __fdiv_rn(a, qm);
    if (s0 % G == 0) srow[g] = sc[k];
  }
}

}  // namespace strm
}  // namespace jolt
