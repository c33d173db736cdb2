// Residual and decompression passes on tensor cores ("A JoLT for the KV
// Cache", Section 3, "Rotated low-bit residual"):
//   compress:   E = X - U_T^ M^_lh,  r = D^-1/2 H_D diag(s) E (per row),
//               absmax b-bit codes + fp32 scales, packed LSB first;
//   decompress: X^ = bf16([RoPE](U_T^ M^_lh + diag(s) D^-1/2 H_D dequant(codes))).
//
// One persistent CTA per SM walks tiles (cell, 128 tokens, layer-head) with
// the layer-head index fastest, so consecutive tiles share U_T^ rows and the
// RoPE table rows in L2. Warp 0 loads U_T^ / M^ slices and, when compressing,
// the 128 x D input tile with TMA, or, when decoding, the tile's packed codes
// and scales with bulk copies; warp 1 issues tcgen05.mma (backbone tile
// 128 x D in TMEM, K = r_T rounded up to 64, fp32 accumulate).
//
// Warps 2..9 form the epilogue: two threads per row, from two warps on the
// same TMEM lane quarter. Thread half h of a row owns the columns
// [hC, hC + C) and [D/2 + hC, D/2 + hC + C), C = D/4, so each RoPE pair
// (i, i + D/2) stays in one thread. The Walsh-Hadamard stages of span < C and
// the stage of span D/2 run in registers; the stage of span C pairs the two
// halves and goes through a swizzled shared-memory exchange. Every stage
// performs the same fp32 additions as the one-row transform, so the result
// is identical to it. Codes, scales and decoded rows are stored straight
// from registers.
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
constexpr int EPI_WARPS = 8;
constexpr int STHREADS = 64 + 32 * EPI_WARPS;

struct Args {
  int ncells, T, H, lhmax, rpad_m, G, ntile_t;
  const CellDesc* cells;
  const CellOut* outs;
  const float2* cs;
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
      const uint32_t u = __float_as_uint(t) & mask;
      const int bit = i * B, wi = bit >> 5, sh = bit & 31;
      w[wi] |= u << sh;
      if (sh + B > 32) w[wi + 1] |= u >> (32 - sh);
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

template <int D, bool COMPRESS>
__global__ void __launch_bounds__(STHREADS, 1) k_stream(const __grid_constant__ SMaps maps, Args a) {
  constexpr int C = D / 4;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;                                   // SSTAGES x S_A
  uint8_t* sB = sA + SSTAGES * S_A;                     // SSTAGES x S_B
  uint8_t* sR1 = sB + SSTAGES * S_B;                    // 2 x S_X (compress) | 2 x (codes + scales)
  float* sPm = reinterpret_cast<float*>(sR1 + S_R1);   // 128 rows x 2 halves x 2 chunk maxima
  float* sSign = sPm + 128 * 4;                         // D (<= 128)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSign + 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SSTAGES + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sign_seq = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (SSTAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 2 + b); };
  // second input buffer: the X tile (compress) or the codes + scales (decode)
  auto xfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 4 + b); };
  auto xempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 6 + b); };
  auto in_buf = [&](int b) { return sR1 + b * (COMPRESS ? S_X : S_CODE + S_SCALE); };
  // two accumulators (2D columns) and two exchange regions of 2 x D/2 columns
  constexpr int NCOLS = (4 * D <= 256) ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SSTAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), EPI_WARPS);
      mbar_init(xfull_bar(b), 1);
      mbar_init(xempty_bar(b), EPI_WARPS);
    }
    *abort_flag = 0;
    *sign_seq = -1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(NCOLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = a.ncells * a.ntile_t * a.lhmax;
  // Work is dealt out by token tile: a CTA takes every layer-head tile of one
  // 128-token tile in a row (so U_T^ slices and RoPE rows are reused from the
  // caches), and token tiles go round-robin over the CTAs (so cells without a
  // residual, skipped when compressing, do not unbalance the CTAs).
  const int ngroups = a.ncells * a.ntile_t;
  (void)ntiles;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, xb = 0;
      uint32_t ph = 0, xph[2] = {0, 0};
      uint32_t issued_phase[SSTAGES];
      bool issued[SSTAGES];
      uint32_t xissued_phase[2];
      bool xissued[2] = {false, false};
      for (int s = 0; s < SSTAGES; ++s) issued[s] = false;
      bool ok = true;
      for (int tile = blockIdx.x * a.lhmax; tile < ngroups * a.lhmax && ok;
           tile += (tile % a.lhmax == a.lhmax - 1) ? 1 + (gridDim.x - 1) * a.lhmax : 1) {
        int cell, t0, lh;
        CellDesc c;
        CellOut o;
        if (!tile_of(a, tile, cell, t0, lh, c, o, COMPRESS)) continue;
        // the tile's second input (X, or codes + scales) first: it then loads
        // while the tensor cores work on the backbone
        if (COMPRESS || o.b > 0) {
          if (!mbar_wait(xempty_bar(xb), xph[xb] ^ 1, abort_flag, a.status)) break;
          const uint32_t sx = smem_u32(in_buf(xb));
          if (COMPRESS) {
            mbar_expect_tx(xfull_bar(xb), D * 128 * 2);
            const CUtensorMap* xm = (c.kind == 0) ? &maps.xk : &maps.xv;
            const int l = c.l0 + lh / c.H, h = lh % c.H;
            for (int hh = 0; hh < D / 64; ++hh)
              tma_load_5d(sx + hh * 16384, xm, xfull_bar(xb), hh * 64, t0, h, l, c.seq);
          } else {
            const CodeTile ct = code_tile(o, (int64_t)lh * c.T + t0, min(SBM, c.T - t0), D, a.G);
            mbar_expect_tx(xfull_bar(xb), (ct.cbulk ? ct.cbytes : 0u) + (ct.sbulk ? ct.sbytes : 0u));
            if (ct.cbulk) bulk_load(sx, ct.codes, ct.cbytes, xfull_bar(xb));
            if (ct.sbulk) bulk_load(sx + S_CODE, ct.scales, ct.sbytes, xfull_bar(xb));
          }
          xissued[xb] = true;
          xissued_phase[xb] = xph[xb];
          xph[xb] ^= 1;
          xb ^= 1;
        }
        const int nk = (o.rT + 63) / 64;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, a.status)) { ok = false; break; }
          const uint32_t sa = smem_u32(sA + stage * S_A), sb = smem_u32(sB + stage * S_B);
          mbar_expect_tx(full_bar(stage), S_A + D * 128);
          tma_load_3d(sa, &maps.ut, full_bar(stage), t0, kb * 64, cell);
          tma_load_3d(sa + 8192, &maps.ut, full_bar(stage), t0 + 64, kb * 64, cell);
          tma_load_3d(sb, &maps.mt, full_bar(stage), kb * 64, 0, cell * a.lhmax + lh);
          issued[stage] = true;
          issued_phase[stage] = ph;
          if (++stage == SSTAGES) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
      for (int s = 0; s < SSTAGES; ++s)
        if (issued[s]) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try(full_bar(s), issued_phase[s]) && now_ns() - t0 < WAIT_NS) {}
        }
      for (int b = 0; b < 2; ++b)
        if (xissued[b]) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try(xfull_bar(b), xissued_phase[b]) && now_ns() - t0 < WAIT_NS) {}
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph[2] = {0, 0};
      const uint32_t idesc = idesc_bf16(D, 1, 0);
      bool ok = true;
      for (int tile = blockIdx.x * a.lhmax; tile < ngroups * a.lhmax && ok;
           tile += (tile % a.lhmax == a.lhmax - 1) ? 1 + (gridDim.x - 1) * a.lhmax : 1) {
        int cell, t0, lh;
        CellDesc c;
        CellOut o;
        if (!tile_of(a, tile, cell, t0, lh, c, o, COMPRESS)) continue;
        const int nk = (o.rT + 63) / 64;
        if (!mbar_wait(tempty_bar(acc), aph[acc] ^ 1, abort_flag, a.status)) break;
        fence_after();
        const uint32_t dcol = tmem + (uint32_t)(acc * D);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full_bar(stage), ph, abort_flag, a.status)) { ok = false; break; }
          fence_after();
          const uint32_t sa = smem_u32(sA + stage * S_A), sb = smem_u32(sB + stage * S_B);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(dcol, sdesc(sa + kk * 2048, 8192, 1024), sdesc(sb + kk * 32, 16, 1024), idesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(empty_bar(stage));
          if (++stage == SSTAGES) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit(tfull_bar(acc));
        aph[acc] ^= 1;
        acc ^= 1;
      }
    }
  } else {
    // --------------------------------------------------------- epilogue rows
    const int q = warp & 3;                   // TMEM lane quarter
    const int hf = (warp - 2) >> 2;           // column half of the row
    const int rl = q * 32 + lane;             // row within the tile (TMEM lane)
    const int et = threadIdx.x - 64;          // 0..255 among the epilogue threads
    const float rs = (float)(1.0 / sqrt((double)D));
    int acc = 0, xb = 0, xpar = 0;
    uint32_t aph[2] = {0, 0}, xph[2] = {0, 0};
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    for (int tile = blockIdx.x * a.lhmax; tile < ngroups * a.lhmax;
         tile += (tile % a.lhmax == a.lhmax - 1) ? 1 + (gridDim.x - 1) * a.lhmax : 1) {
      int cell, t0, lh;
      CellDesc c;
      CellOut o;
      if (!tile_of(a, tile, cell, t0, lh, c, o, COMPRESS)) continue;
      // Hadamard signs of this tile's sequence
      if (*sign_seq != c.seq) {
        epi_sync();
        if (et < D) sSign[et] = hadamard_sign(a.seed + c.seq, et);
        epi_sync();
        if (et == 0) *sign_seq = c.seq;
        epi_sync();
      }
      const int t = t0 + rl;
      const bool valid = t < c.T;
      const int nrows = min(SBM, c.T - t0);
      const int l = lh / c.H, h = lh % c.H;
      const int b = o.b;
      const int rowbytes = b * D / 8;
      const int ng = D / a.G;
      const int64_t row0 = (int64_t)lh * c.T + t0;   // first residual row of the tile
      const int64_t row = row0 + rl;
      float e[2 * C];
      if (COMPRESS) {
        // the first half of this row's RoPE table entries, fetched before the waits
        const float4* cs4 = reinterpret_cast<const float4*>(a.cs + (int64_t)(valid ? t : 0) * (D / 2) + hf * C);
        float4 csr[C / 4];
        if (c.rope) {
#pragma unroll
          for (int p = 0; p < C / 4; ++p) csr[p] = cs4[p];
        }
        // backbone
        if (!epi_all(mbar_wait(tfull_bar(acc), aph[acc], abort_flag, a.status))) break;
        fence_after();
        const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * D);
        tmem_ld<C>(tb + hf * C, e);
        tmem_ld<C>(tb + D / 2 + hf * C, e + C);
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        aph[acc] ^= 1;
        acc ^= 1;
        // E = [un-RoPE](X) - backbone
        if (!epi_all(mbar_wait(xfull_bar(xb), xph[xb], abort_flag, a.status))) break;
        const uint8_t* xs = in_buf(xb);
#pragma unroll
        for (int u = 0; u < C / 8; ++u) {
          float x0[8], x1[8];
          ld_x8(xs, rl, hf * C + 8 * u, x0);
          ld_x8(xs, rl, D / 2 + hf * C + 8 * u, x1);
          if (c.rope) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const float4 q2 = (4 * u + p < C / 4) ? csr[4 * u + p] : cs4[4 * u + p];
              const float cc[2] = {q2.x, q2.z}, ss[2] = {q2.y, q2.w};
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const float yi = x0[2 * p + j], yj = x1[2 * p + j];
                x0[2 * p + j] = __fadd_rn(__fmul_rn(yi, cc[j]), __fmul_rn(yj, ss[j]));
                x1[2 * p + j] = __fsub_rn(__fmul_rn(yj, cc[j]), __fmul_rn(yi, ss[j]));
              }
            }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            e[8 * u + j] = __fsub_rn(x0[j], e[8 * u + j]);
            e[C + 8 * u + j] = __fsub_rn(x1[j], e[C + 8 * u + j]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(xempty_bar(xb));
        xph[xb] ^= 1;
        xb ^= 1;
        // rotation
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int u = 0; u < C / 4; ++u) {
            const float4 s4 = reinterpret_cast<const float4*>(sSign + k * (D / 2) + hf * C)[u];
            e[k * C + 4 * u + 0] = __fmul_rn(e[k * C + 4 * u + 0], s4.x);
            e[k * C + 4 * u + 1] = __fmul_rn(e[k * C + 4 * u + 1], s4.y);
            e[k * C + 4 * u + 2] = __fmul_rn(e[k * C + 4 * u + 2], s4.z);
            e[k * C + 4 * u + 3] = __fmul_rn(e[k * C + 4 * u + 3], s4.w);
          }
        fwht_pair<C>(e, lane_base, (uint32_t)(2 * D + xpar * D), hf, q);
        xpar ^= 1;
        float am[2] = {0.0f, 0.0f};
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int j = 0; j < C; ++j) {
            e[k * C + j] = __fmul_rn(e[k * C + j], rs);
            am[k] = fmaxf(am[k], fabsf(e[k * C + j]));
          }
        float sc[2];
        float* srow = o.scales + row * ng;
        float dummy[4];
        chunk_scales<D>(am, sPm, rl, hf, q, a.G, (float)qmax_of(b), sc, valid ? srow : dummy);
        if (valid) {
          uint8_t* crow = o.codes + row * rowbytes;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint8_t* dst = crow + (k * (D / 2) + hf * C) * b / 8;
            uint32_t w[C * 8 / 32];
            switch (b) {
              case 2: quant_chunk<C, 2>(e + k * C, sc[k], w); store_bits<C, 2>(dst, w); break;
              case 3: quant_chunk<C, 3>(e + k * C, sc[k], w); store_bits<C, 3>(dst, w); break;
              case 4: quant_chunk<C, 4>(e + k * C, sc[k], w); store_bits<C, 4>(dst, w); break;
              default: quant_chunk<C, 8>(e + k * C, sc[k], w); store_bits<C, 8>(dst, w); break;
            }
          }
        }
      } else {
        if (b > 0) {
          if (!epi_all(mbar_wait(xfull_bar(xb), xph[xb], abort_flag, a.status))) break;
          const CodeTile ct = code_tile(o, row0, nrows, D, a.G);
          const uint8_t* stage_in = in_buf(xb);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int s0 = k * (D / 2) + hf * C;
            if (!valid) {
#pragma unroll
              for (int j = 0; j < C; ++j) e[k * C + j] = 0.0f;
              continue;
            }
            // staged copies are read as shared memory, the fallback from global memory
            const float sc = ct.sbulk ? reinterpret_cast<const float*>(stage_in + S_CODE)[rl * ng + s0 / a.G]
                                      : ct.scales[rl * ng + s0 / a.G];
            const int64_t off = (int64_t)rl * rowbytes + s0 * b / 8;
            uint32_t w[C * 8 / 32];
            switch (b) {
              case 2: if (ct.cbulk) load_bits<C, 2>(stage_in + off, w); else load_bits<C, 2>(ct.codes + off, w);
                      dequant_chunk<C, 2>(w, sc, e + k * C); break;
              case 3: if (ct.cbulk) load_bits<C, 3>(stage_in + off, w); else load_bits<C, 3>(ct.codes + off, w);
                      dequant_chunk<C, 3>(w, sc, e + k * C); break;
              case 4: if (ct.cbulk) load_bits<C, 4>(stage_in + off, w); else load_bits<C, 4>(ct.codes + off, w);
                      dequant_chunk<C, 4>(w, sc, e + k * C); break;
              default: if (ct.cbulk) load_bits<C, 8>(stage_in + off, w); else load_bits<C, 8>(ct.codes + off, w);
                       dequant_chunk<C, 8>(w, sc, e + k * C); break;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(xempty_bar(xb));
          xph[xb] ^= 1;
          xb ^= 1;
          fwht_pair<C>(e, lane_base, (uint32_t)(2 * D + xpar * D), hf, q);
        xpar ^= 1;
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int u = 0; u < C / 4; ++u) {
              const float4 s4 = reinterpret_cast<const float4*>(sSign + k * (D / 2) + hf * C)[u];
              const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) e[k * C + 4 * u + j] = __fmul_rn(__fmul_rn(e[k * C + 4 * u + j], rs), sv[j]);
            }
        } else {
#pragma unroll
          for (int j = 0; j < 2 * C; ++j) e[j] = 0.0f;
        }
        // + backbone
        if (!epi_all(mbar_wait(tfull_bar(acc), aph[acc], abort_flag, a.status))) break;
        fence_after();
        {
          const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * D);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            float v[C];
            tmem_ld<C>(tb + k * (D / 2) + hf * C, v);
#pragma unroll
            for (int j = 0; j < C; ++j) e[k * C + j] = __fadd_rn(v[j], e[k * C + j]);
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        aph[acc] ^= 1;
        acc ^= 1;
        if (valid) {
          if (c.rope) {
            const float4* cs4 = reinterpret_cast<const float4*>(a.cs + (int64_t)t * (D / 2) + hf * C);
#pragma unroll
            for (int p = 0; p < C / 2; ++p) {
              const float4 q2 = cs4[p];
              const float cc[2] = {q2.x, q2.z}, ss[2] = {q2.y, q2.w};
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const float x0 = e[2 * p + j], x1 = e[C + 2 * p + j];
                e[2 * p + j] = __fsub_rn(__fmul_rn(x0, cc[j]), __fmul_rn(x1, ss[j]));
                e[C + 2 * p + j] = __fadd_rn(__fmul_rn(x1, cc[j]), __fmul_rn(x0, ss[j]));
              }
            }
          }
          uint16_t* base = (c.kind == 0 ? a.out_k : a.out_v) + (int64_t)c.seq * a.osb + (int64_t)(c.l0 + l) * a.osl +
                           (int64_t)h * a.osh + (int64_t)t * a.ost;
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int u = 0; u < C / 8; ++u) {
              const float* s = e + k * C + 8 * u;
              uint4 w;
              w.x = bf16x2_bits(s[0], s[1]);
              w.y = bf16x2_bits(s[2], s[3]);
              w.z = bf16x2_bits(s[4], s[5]);
              w.w = bf16x2_bits(s[6], s[7]);
              *reinterpret_cast<uint4*>(base + k * (D / 2) + hf * C + 8 * u) = w;
            }
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS));
  }
}

}  // namespace strm

// ----------------------------------------------------------- launchers ----
// U_T^ from the payload into the workspace [cells][rows][tp], rows r_T ..
// ceil64(r_T)-1 zeroed (they meet zero columns of M^T in the K loop).
__global__ void k_ut_to_ws(const CellOut* __restrict__ outs, uint16_t* __restrict__ ws, int rows, int tp) {
  const int cell = blockIdx.y;
  const CellOut o = outs[cell];
  const int r_end = min(rows, (o.rT + 63) / 64 * 64);
  const int64_t n = (int64_t)r_end * tp;
  uint16_t* dst = ws + (int64_t)cell * rows * tp;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(e / tp), t = (int)(e % tp);
    dst[e] = (r < o.rT && t < o.t_pitch) ? o.ut[(int64_t)r * o.t_pitch + t] : (uint16_t)0;
  }
}

// M^ rows [lh][r][d] -> M^T [cell*lhmax + lh][d][r] (pitch rpad), columns
// r_T .. ceil64(r_T)-1 zeroed.
__global__ void k_m_transpose(const CellOut* __restrict__ outs, const CellDesc* __restrict__ cells,
                              uint16_t* const* __restrict__ M, const int* __restrict__ rmax_of,
                              uint16_t* __restrict__ Mt, int lhmax, int D, int rpad) {
  const int cell = blockIdx.z, lh = blockIdx.y;
  const CellOut o = outs[cell];
  const CellDesc c = cells[cell];
  if (lh >= c.Lg * c.H) return;
  const int r_end = min(rpad, (o.rT + 63) / 64 * 64);
  const uint16_t* src = M[cell] + (int64_t)lh * rmax_of[cell] * D;
  uint16_t* dst = Mt + ((int64_t)cell * lhmax + lh) * D * rpad;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < D * r_end; e += gridDim.x * blockDim.x) {
    const int d = e / r_end, r = e % r_end;
    dst[(int64_t)d * rpad + r] = (r < o.rT) ? src[(int64_t)r * D + d] : (uint16_t)0;
  }
}

jolt_status launch_m_transpose(const CellOut* outs, const CellDesc* cells, uint16_t* const* M, const int* rmax_of,
                               uint16_t* Mt, int lhmax, int D, int rpad, int ncells, cudaStream_t s) {
  dim3 g(16, lhmax, ncells);
  k_m_transpose<<<g, 256, 0, s>>>(outs, cells, M, rmax_of, Mt, lhmax, D, rpad);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

jolt_status launch_ut_to_ws(const CellOut* outs, uint16_t* ws, int rows, int tp, int ncells, cudaStream_t s) {
  dim3 g(256, ncells);
  k_ut_to_ws<<<g, 256, 0, s>>>(outs, ws, rows, tp);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

static int stream_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

jolt_status launch_stream(bool compress, int D, const StreamMaps& m, const StreamArgs& sa, cudaStream_t s) {
  strm::SMaps maps;
  maps.ut = m.ut; maps.mt = m.mt; maps.xk = m.xk; maps.xv = m.xv;
  strm::Args a;
  a.ncells = sa.ncells; a.T = sa.T; a.H = sa.H; a.lhmax = sa.lhmax; a.rpad_m = sa.rpad_m; a.G = sa.G;
  a.ntile_t = (sa.T + 127) / 128;
  a.cells = sa.cells; a.outs = sa.outs; a.cs = sa.cs; a.seed = sa.seed;
  a.out_k = sa.out_k; a.out_v = sa.out_v; a.osb = sa.osb; a.osl = sa.osl; a.osh = sa.osh; a.ost = sa.ost;
  a.status = sa.status;
  const int ntiles = a.ncells * a.ntile_t * a.lhmax;
  if (ntiles == 0) return JOLT_OK;
  const int grid = std::min(ntiles, stream_sms());
  const int smem = strm::SMEM_STREAM;
#define JOLT_STREAM_LAUNCH(DD, CC)                                                                          \
  do {                                                                                                      \
    static bool attr = false;                                                                               \
    if (!attr) {                                                                                            \
      JOLT_CUDA_TRY(cudaFuncSetAttribute(strm::k_stream<DD, CC>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         smem));                                                            \
      attr = true;                                                                                          \
    }                                                                                                       \
    strm::k_stream<DD, CC><<<grid, strm::STHREADS, smem, s>>>(maps, a);                                      \
  } while (0)
  if (D == 128) {
    if (compress) JOLT_STREAM_LAUNCH(128, true);
    else JOLT_STREAM_LAUNCH(128, false);
  } else {
    if (compress) JOLT_STREAM_LAUNCH(64, true);
    else JOLT_STREAM_LAUNCH(64, false);
  }
#undef JOLT_STREAM_LAUNCH
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
