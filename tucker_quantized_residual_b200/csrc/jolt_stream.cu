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
// Warps 2..17 form the epilogue: four threads per row, from four warps on the
// same TMEM lane quarter (details below). Every Walsh-Hadamard stage performs
// the same fp32 additions as the one-row transform, so the result is
// identical to it. Codes, scales and decoded rows are stored straight from
// registers.
#include "jolt_stream.cuh"

namespace jolt {
namespace strm {

using namespace umma;

// ----------------------------------------------------------------------
// Four threads per row: 16 epilogue warps (four per TMEM lane quarter), so
// each SM sub-partition has four epilogue warps to interleave. Thread j of a
// row owns the columns [jC, jC + C) and [D/2 + jC, D/2 + jC + C), C = D/8:
// every RoPE pair (i, i + D/2) stays in one thread, the Walsh-Hadamard
// stages of span < C and the stage of span D/2 run in registers, and the
// stages of span C and 2C pair thread j with threads j^1 and j^2 through two
// exchange regions in tensor memory.
constexpr int QEPI = 16;                       // epilogue warps
constexpr int QTHREADS = 64 + 32 * QEPI;

__device__ __forceinline__ void qepi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * QEPI) : "memory"); }
// the four warps of one TMEM lane quarter (the four threads of each row)
__device__ __forceinline__ void quad_sync(int q) { asm volatile("bar.sync %0, 128;" ::"r"(2 + q) : "memory"); }
__device__ __forceinline__ bool qepi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(32 * QEPI)
      : "memory");
  return r != 0;
}

template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float* v) {
  if constexpr (N == 16) {
    tmem_ld16(taddr, v);
  } else {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
  }
}
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const float* v) {
  if constexpr (N == 16) {
    tmem_st<16>(taddr, v);
  } else {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
  }
}

// One cross-thread butterfly stage: the thread's 2C values go to its own TMEM
// lane at columns xcol + j*2C, the four threads of the row meet at the
// quarter barrier, and each combines with partner j^m: the thread holding the
// lower index of each pair keeps a + b, the other a - b.
template <int C>
__device__ __forceinline__ void xstage(float* e, uint32_t lane_base, uint32_t xcol, int j, int m, int q) {
  tmem_st_n<C>(lane_base + xcol + (uint32_t)(j * 2 * C), e);
  tmem_st_n<C>(lane_base + xcol + (uint32_t)(j * 2 * C + C), e + C);
  tmem_wait_st();
  fence_before();
  quad_sync(q);
  fence_after();
  const int pj = j ^ m;
  // lower: RN(e + p) = fma(e, 1, p); upper: RN(p - e) = fma(e, -1, p), one rounding each
  const float sg = ((j & m) == 0) ? 1.0f : -1.0f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float p[C];
    tmem_ld_n<C>(lane_base + xcol + (uint32_t)(pj * 2 * C + k * C), p);
#pragma unroll
    for (int u = 0; u < C; ++u) e[k * C + u] = __fmaf_rn(e[k * C + u], sg, p[u]);
  }
}

// Natural-order Walsh-Hadamard transform of the row, stages 1, 2, ..., D/2,
// on this thread's two chunks: the same fp32 operations in the same order as
// the one-row transform.
template <int C>
__device__ __forceinline__ void fwht_quad(float* e, uint32_t lane_base, uint32_t x1, uint32_t x2, int j, int q) {
  fwht_chunk<C>(e);
  fwht_chunk<C>(e + C);
  xstage<C>(e, lane_base, x1, j, 1, q);
  xstage<C>(e, lane_base, x2, j, 2, q);
#pragma unroll
  for (int u = 0; u < C; ++u) {
    const float x = e[u], y = e[C + u];
    e[u] = __fadd_rn(x, y);
    e[C + u] = __fsub_rn(x, y);
  }
}

// Bytes of a chunk of C b-bit codes and the widest store unit that divides
// both the chunk and the byte offset of the second chunk of thread 0.
template <int C, int B, int D>
struct ChunkIO {
  static constexpr int W = C * B / 8;
  static constexpr int OFFB = D * B / 16;
  static constexpr int U = ((W % 16 == 0) && (OFFB % 16 == 0)) ? 16
                         : ((W % 8 == 0) && (OFFB % 8 == 0)) ? 8
                         : ((W % 4 == 0) && (OFFB % 4 == 0)) ? 4
                         : ((W % 2 == 0) && (OFFB % 2 == 0)) ? 2 : 1;
};

template <int C, int B, int D>
__device__ __forceinline__ void store_chunk(uint8_t* p, const uint32_t* w) {
  constexpr int U = ChunkIO<C, B, D>::U, W = ChunkIO<C, B, D>::W;
  if constexpr (U == 16) {
#pragma unroll
    for (int i = 0; i < W / 16; ++i)
      *reinterpret_cast<uint4*>(p + 16 * i) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else if constexpr (U == 8) {
#pragma unroll
    for (int i = 0; i < W / 8; ++i) *reinterpret_cast<uint2*>(p + 8 * i) = make_uint2(w[2 * i], w[2 * i + 1]);
  } else if constexpr (U == 4) {
#pragma unroll
    for (int i = 0; i < W / 4; ++i) reinterpret_cast<uint32_t*>(p)[i] = w[i];
  } else if constexpr (U == 2) {
#pragma unroll
    for (int i = 0; i < W / 2; ++i) reinterpret_cast<uint16_t*>(p)[i] = (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) p[i] = (uint8_t)(w[i >> 2] >> (8 * (i & 3)));
  }
}

template <int C, int B, int D>
__device__ __forceinline__ void load_chunk(const uint8_t* p, uint32_t* w) {
  constexpr int U = ChunkIO<C, B, D>::U, W = ChunkIO<C, B, D>::W;
  constexpr int NW = (C * B + 31) / 32;
#pragma unroll
  for (int i = 0; i < NW + 1; ++i) w[i] = 0u;
  if constexpr (U == 16) {
#pragma unroll
    for (int i = 0; i < W / 16; ++i) {
      const uint4 x = *reinterpret_cast<const uint4*>(p + 16 * i);
      w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
    }
  } else if constexpr (U == 8) {
#pragma unroll
    for (int i = 0; i < W / 8; ++i) {
      const uint2 x = *reinterpret_cast<const uint2*>(p + 8 * i);
      w[2 * i] = x.x; w[2 * i + 1] = x.y;
    }
  } else if constexpr (U == 4) {
#pragma unroll
    for (int i = 0; i < W / 4; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  } else if constexpr (U == 2) {
#pragma unroll
    for (int i = 0; i < W / 2; ++i) w[i >> 1] |= (uint32_t)reinterpret_cast<const uint16_t*>(p)[i] << (16 * (i & 1));
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) w[i >> 2] |= (uint32_t)p[i] << (8 * (i & 3));
  }
}

template <int D, bool COMPRESS>
__global__ void __launch_bounds__(QTHREADS, 1) k_stream(const __grid_constant__ SMaps maps, Args a) {
  constexpr int C = D / 8;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;                                   // SSTAGES x S_A
  uint8_t* sB = sA + SSTAGES * S_A;                     // SSTAGES x S_B
  uint8_t* sR1 = sB + SSTAGES * S_B;                    // 2 x S_X (compress) | 2 x (padded codes + scales)
  float* sPm = reinterpret_cast<float*>(sR1 + S_R1Q);  // 128 rows x 4 threads x 2 chunk maxima
  float* sSign = sPm + 128 * 8;                         // D (<= 128)
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
  auto in_buf = [&](int b) { return sR1 + b * (COMPRESS ? S_X : S_CODEP + S_SCALE); };
  // two accumulators (2D columns) and two exchange regions of D columns
  constexpr int NCOLS = (4 * D <= 256) ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SSTAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), QEPI);
      mbar_init(xfull_bar(b), 1);
      mbar_init(xempty_bar(b), QEPI);
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
  // Work is dealt out by token tile: a CTA takes every layer-head tile of one
  // 128-token tile in a row (so U_T^ slices and RoPE rows are reused from the
  // caches), and token tiles go round-robin over the CTAs (so cells without a
  // residual, skipped when compressing, do not unbalance the CTAs).
  const int ngroups = a.ncells * a.ntile_t;

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
            const int nrows = min(SBM, c.T - t0);
            const CodeTile ct = code_tile(o, (int64_t)lh * c.T + t0, nrows, D, a.G);
            mbar_expect_tx(xfull_bar(xb), (ct.cbulk ? ct.cbytes : 0u) + (ct.sbulk ? ct.sbytes : 0u));
            if (ct.cbulk) bulk_load(sx, ct.codes, ct.cbytes, xfull_bar(xb));
            if (ct.sbulk) bulk_load(sx + S_CODEP, ct.scales, ct.sbytes, xfull_bar(xb));
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
    const int j = (warp - 2) >> 2;            // column quarter of the row (0..3)
    const int rl = q * 32 + lane;             // row within the tile (TMEM lane)
    const int et = threadIdx.x - 64;          // 0..511 among the epilogue threads
    const int cA = j * C, cB = D / 2 + j * C; // first columns of this thread's chunks
    const float rs = (float)(1.0 / sqrt((double)D));
    int acc = 0, xb = 0;
    uint32_t aph[2] = {0, 0}, xph[2] = {0, 0};
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t x1 = 2 * D, x2 = 3 * D;    // exchange regions (D columns each)
    for (int tile = blockIdx.x * a.lhmax; tile < ngroups * a.lhmax;
         tile += (tile % a.lhmax == a.lhmax - 1) ? 1 + (gridDim.x - 1) * a.lhmax : 1) {
      int cell, t0, lh;
      CellDesc c;
      CellOut o;
      if (!tile_of(a, tile, cell, t0, lh, c, o, COMPRESS)) continue;
      // Hadamard signs of this tile's sequence
      if (*sign_seq != c.seq) {
        qepi_sync();
        if (et < D) sSign[et] = hadamard_sign(a.seed + c.seq, et);
        qepi_sync();
        if (et == 0) *sign_seq = c.seq;
        qepi_sync();
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
        // this row's RoPE table entries of the two chunks, fetched before the waits
        float2 csr[C];
        if (c.rope) {
          const float4* cq = a.csq + ((int64_t)(t0 / SBM) * 4 + j) * (C / 2) * SBM + rl;
#pragma unroll
          for (int p = 0; p < C / 2; ++p) {
            const float4 v = cq[p * SBM];
            csr[2 * p] = make_float2(v.x, v.y);
            csr[2 * p + 1] = make_float2(v.z, v.w);
          }
        }
        // backbone
        if (!qepi_all(mbar_wait(tfull_bar(acc), aph[acc], abort_flag, a.status))) break;
        fence_after();
        const uint32_t tb = lane_base + (uint32_t)(acc * D);
        tmem_ld_n<C>(tb + cA, e);
        tmem_ld_n<C>(tb + cB, e + C);
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        aph[acc] ^= 1;
        acc ^= 1;
        // E = [un-RoPE](X) - backbone
        if (!qepi_all(mbar_wait(xfull_bar(xb), xph[xb], abort_flag, a.status))) break;
        const uint8_t* xs = in_buf(xb);
#pragma unroll
        for (int u = 0; u < C / 8; ++u) {
          float x0[8], x1v[8];
          ld_x8(xs, rl, cA + 8 * u, x0);
          ld_x8(xs, rl, cB + 8 * u, x1v);
          if (c.rope) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 q2 = csr[8 * u + i];
              const float yi = x0[i], yj = x1v[i];
              x0[i] = __fadd_rn(__fmul_rn(yi, q2.x), __fmul_rn(yj, q2.y));
              x1v[i] = __fsub_rn(__fmul_rn(yj, q2.x), __fmul_rn(yi, q2.y));
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            e[8 * u + i] = __fsub_rn(x0[i], e[8 * u + i]);
            e[C + 8 * u + i] = __fsub_rn(x1v[i], e[C + 8 * u + i]);
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
            const float4 s4 = reinterpret_cast<const float4*>(sSign + (k ? cB : cA))[u];
            e[k * C + 4 * u + 0] = __fmul_rn(e[k * C + 4 * u + 0], s4.x);
            e[k * C + 4 * u + 1] = __fmul_rn(e[k * C + 4 * u + 1], s4.y);
            e[k * C + 4 * u + 2] = __fmul_rn(e[k * C + 4 * u + 2], s4.z);
            e[k * C + 4 * u + 3] = __fmul_rn(e[k * C + 4 * u + 3], s4.w);
          }
        fwht_quad<C>(e, lane_base, x1, x2, j, q);
        float am[2] = {0.0f, 0.0f};
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int u = 0; u < C; ++u) {
            e[k * C + u] = __fmul_rn(e[k * C + u], rs);
            am[k] = fmaxf(am[k], fabsf(e[k * C + u]));
          }
        // scales: the chunk maxima of the row's four threads meet in shared memory
        sPm[(rl * 4 + j) * 2 + 0] = am[0];
        sPm[(rl * 4 + j) * 2 + 1] = am[1];
        quad_sync(q);
        const float qm = (float)qmax_of(b);
        float sc[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int s0 = k ? cB : cA, g = s0 / a.G;
          float mx = 0.0f;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int s1 = kk * (D / 2) + jj * C;
              if (s1 / a.G == g) mx = fmaxf(mx, sPm[(rl * 4 + jj) * 2 + kk]);
            }
          sc[k] = __fdiv_rn(mx, qm);
          if (valid && s0 % a.G == 0) o.scales[row * ng + g] = sc[k];
        }
        if (valid) {
          uint8_t* crow = o.codes + row * rowbytes;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint8_t* dst = crow + (k ? cB : cA) * b / 8;
            uint32_t w[C * 8 / 32 + 1];
            switch (b) {
              case 2: quant_chunk<C, 2>(e + k * C, sc[k], w); store_chunk<C, 2, D>(dst, w); break;
              case 3: quant_chunk<C, 3>(e + k * C, sc[k], w); store_chunk<C, 3, D>(dst, w); break;
              case 4: quant_chunk<C, 4>(e + k * C, sc[k], w); store_chunk<C, 4, D>(dst, w); break;
              default: quant_chunk<C, 8>(e + k * C, sc[k], w); store_chunk<C, 8, D>(dst, w); break;
            }
          }
        }
      } else {
        float4 csr[C / 2];
        if (b > 0) {
          if (!qepi_all(mbar_wait(xfull_bar(xb), xph[xb], abort_flag, a.status))) break;
          const CodeTile ct = code_tile(o, row0, nrows, D, a.G);
          const uint8_t* stage_in = in_buf(xb);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int s0 = k ? cB : cA;
            if (!valid) {
#pragma unroll
              for (int u = 0; u < C; ++u) e[k * C + u] = 0.0f;
              continue;
            }
            // staged copies are read as shared memory, the fallback from global memory
            const float sc = ct.sbulk ? reinterpret_cast<const float*>(stage_in + S_CODEP)[rl * ng + s0 / a.G]
                                      : ct.scales[rl * ng + s0 / a.G];
            const uint8_t* src = ct.cbulk ? stage_in + rl * rowbytes + s0 * b / 8
                                          : ct.codes + (int64_t)rl * rowbytes + s0 * b / 8;
            uint32_t w[C * 8 / 32 + 1];
            switch (b) {
              case 2: load_chunk<C, 2, D>(src, w); dequant_chunk<C, 2>(w, sc, e + k * C); break;
              case 3: load_chunk<C, 3, D>(src, w); dequant_chunk<C, 3>(w, sc, e + k * C); break;
              case 4: load_chunk<C, 4, D>(src, w); dequant_chunk<C, 4>(w, sc, e + k * C); break;
              default: load_chunk<C, 8, D>(src, w); dequant_chunk<C, 8>(w, sc, e + k * C); break;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(xempty_bar(xb));
          xph[xb] ^= 1;
          xb ^= 1;
          fwht_quad<C>(e, lane_base, x1, x2, j, q);
          // times D^-1/2, then the sign: one product by +-D^-1/2 (the sign is
          // exact, so this is the same rounded value)
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int u = 0; u < C / 4; ++u) {
              const float4 s4 = reinterpret_cast<const float4*>(sSign + (k ? cB : cA))[u];
              const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) e[k * C + 4 * u + i] = __fmul_rn(e[k * C + 4 * u + i], __fmul_rn(rs, sv[i]));
            }
        } else {
#pragma unroll
          for (int u = 0; u < 2 * C; ++u) e[u] = 0.0f;
        }
        // this row's RoPE table entries: in flight while the backbone is awaited
        if (c.rope) {
          const float4* cq = a.csq + ((int64_t)(t0 / SBM) * 4 + j) * (C / 2) * SBM + rl;
#pragma unroll
          for (int p = 0; p < C / 2; ++p) csr[p] = cq[p * SBM];
        }
        // + backbone
        if (!qepi_all(mbar_wait(tfull_bar(acc), aph[acc], abort_flag, a.status))) break;
        fence_after();
        {
          const uint32_t tb = lane_base + (uint32_t)(acc * D);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            float v[C];
            tmem_ld_n<C>(tb + (k ? cB : cA), v);
#pragma unroll
            for (int u = 0; u < C; ++u) e[k * C + u] = __fadd_rn(v[u], e[k * C + u]);
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        aph[acc] ^= 1;
        acc ^= 1;
        if (valid) {
          if (c.rope) {
#pragma unroll
            for (int p = 0; p < C / 2; ++p) {
              const float4 q2 = csr[p];
              const float cc[2] = {q2.x, q2.z}, ss[2] = {q2.y, q2.w};
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const float x0 = e[2 * p + i], x1v = e[C + 2 * p + i];
                e[2 * p + i] = __fsub_rn(__fmul_rn(x0, cc[i]), __fmul_rn(x1v, ss[i]));
                e[C + 2 * p + i] = __fadd_rn(__fmul_rn(x1v, cc[i]), __fmul_rn(x0, ss[i]));
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
              *reinterpret_cast<uint4*>(base + (k ? cB : cA) + 8 * u) = w;
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

__global__ void k_rope_tiled(const float2* __restrict__ cs, int T, int D, float4* __restrict__ csq) {
  const int C = D / 8, U = C / 2;             // pairs per column quarter, float4 units
  const int ntile = (T + 127) / 128;
  const int64_t n = (int64_t)ntile * 4 * U * 128;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int row = (int)(e % 128);
    const int64_t r = e / 128;
    const int u = (int)(r % U);
    const int64_t r2 = r / U;
    const int j = (int)(r2 % 4);
    const int tau = (int)(r2 / 4);
    const int t = tau * 128 + row;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < T) {
      const float2 a0 = cs[(int64_t)t * (D / 2) + j * C + 2 * u];
      const float2 a1 = cs[(int64_t)t * (D / 2) + j * C + 2 * u + 1];
      v = make_float4(a0.x, a0.y, a1.x, a1.y);
    }
    csq[e] = v;
  }
}

jolt_status launch_rope_tiled(const float2* cs, int T, int D, float4* csq, cudaStream_t s) {
  const int64_t n = (int64_t)((T + 127) / 128) * 128 * (D / 4);
  k_rope_tiled<<<(int)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, s>>>(cs, T, D, csq);
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
  a.cells = sa.cells; a.outs = sa.outs; a.cs = sa.cs; a.csq = sa.csq; a.seed = sa.seed;
  a.out_k = sa.out_k; a.out_v = sa.out_v; a.osb = sa.osb; a.osl = sa.osl; a.osh = sa.osh; a.ost = sa.ost;
  a.status = sa.status;
  const int ntiles = a.ncells * a.ntile_t * a.lhmax;
  if (ntiles == 0) return JOLT_OK;
  const int grid = std::min(ntiles, stream_sms());
  const int smem = strm::SMEM_STREAM4;
#define JOLT_STREAM_LAUNCH(DD, CC)                                                                          \
  do {                                                                                                      \
    static bool attr = false;                                                                               \
    if (!attr) {                                                                                            \
      JOLT_CUDA_TRY(cudaFuncSetAttribute(strm::k_stream<DD, CC>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         smem));                                                            \
      attr = true;                                                                                          \
    }                                                                                                       \
    strm::k_stream<DD, CC><<<grid, strm::QTHREADS, smem, s>>>(maps, a);                                      \
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
