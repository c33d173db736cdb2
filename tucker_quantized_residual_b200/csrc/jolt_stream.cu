// Residual and decompression passes on tensor cores ("A JoLT for the KV
// Cache", Section 3, "Rotated low-bit residual"):
//   compress:   E = X - U_T^ M^_lh,  r = D^-1/2 H_D diag(s) E (per row),
//               absmax b-bit codes + fp32 scales, packed LSB first;
//   decompress: X^ = bf16([RoPE](U_T^ M^_lh + diag(s) D^-1/2 H_D dequant(codes))).
//
// One persistent CTA per SM walks tiles (cell, 128 tokens, layer-head) with
// the layer-head index fastest, so consecutive tiles share U_T^ rows and the
// RoPE table rows in L2. Warp 0 loads U_T^ / M^ slices (and, when
// compressing, the 128 x D input tile) with TMA; warp 1 issues tcgen05.mma
// (backbone tile 128 x D in TMEM, K = r_T rounded up to 64, fp32 accumulate);
// warps 2..5 each own 32 rows: they read the backbone row from TMEM, the input
// row from the 128-byte-swizzled tile, and run the rotation and the quantizer
// in registers. Packed codes, scales and decoded rows go through padded
// shared staging so that global loads and stores are coalesced.
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
constexpr int ROWPITCH_OUT = 128 * 2 + 16; // decoded bf16 row + pad
constexpr int CODE_PITCH_MAX = 128 + 8;    // packed row (<= 8 bits x 128 / 8) + pad
constexpr int SMEM_STREAM = SSTAGES * (S_A + S_B) + 2 * S_X + 128 * ROWPITCH_OUT + 128 * CODE_PITCH_MAX +
                            128 * 4 * 4 + 1024 + 512;
constexpr int STHREADS = 192;

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

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
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

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// AND of `ok` over the 128 epilogue threads: every one of them takes the same
// branch after a bounded wait, so none is left at a named barrier alone.
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
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

template <int D>
struct RowPack {
  float* e;
  uint8_t* dst;
  float* sc;
  template <int G, int B>
  __device__ __forceinline__ void run() { quantize_pack_row<D, G, B>(e, dst, sc); }
};
template <int D>
struct RowUnpack {
  float* v;
  const uint8_t* src;
  const float* sc;
  template <int G, int B>
  __device__ __forceinline__ void run() { unpack_dequant_row<D, G, B>(src, sc, v); }
};

template <int D, bool COMPRESS>
__global__ void __launch_bounds__(STHREADS, 1) k_stream(const __grid_constant__ SMaps maps, Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;                                   // SSTAGES x S_A
  uint8_t* sB = sA + SSTAGES * S_A;                     // SSTAGES x S_B
  uint8_t* sX = sB + SSTAGES * S_B;                     // 2 x S_X
  uint8_t* sOut = sX + 2 * S_X;                         // 128 x ROWPITCH_OUT
  uint8_t* sCode = sOut + 128 * ROWPITCH_OUT;           // 128 x CODE_PITCH_MAX
  float* sScale = reinterpret_cast<float*>(sCode + 128 * CODE_PITCH_MAX);   // 128 x 4
  float* sSign = sScale + 128 * 4;                      // D
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
  auto xfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 4 + b); };
  auto xempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 6 + b); };
  constexpr int NCOLS = (2 * D <= 128) ? 128 : 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SSTAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);
      mbar_init(xfull_bar(b), 1);
      mbar_init(xempty_bar(b), 4);
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
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        int cell, t0, lh;
        CellDesc c;
        CellOut o;
        if (!tile_of(a, tile, cell, t0, lh, c, o, COMPRESS)) continue;
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
        if (COMPRESS) {
          if (!mbar_wait(xempty_bar(xb), xph[xb] ^ 1, abort_flag, a.status)) break;
          const uint32_t sx = smem_u32(sX + xb * S_X);
          mbar_expect_tx(xfull_bar(xb), D * 128 * 2);
          const CUtensorMap* xm = (c.kind == 0) ? &maps.xk : &maps.xv;
          const int l = c.l0 + lh / c.H, h = lh % c.H;
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(sx + hh * 16384, xm, xfull_bar(xb), hh * 64, t0, h, l, c.seq);
          xissued[xb] = true;
          xissued_phase[xb] = xph[xb];
          xph[xb] ^= 1;
          xb ^= 1;
        }
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
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
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
    const int q = warp & 3;
    const int rl = q * 32 + lane;            // row within the tile (TMEM lane)
    const int et = threadIdx.x - 64;         // 0..127 among the epilogue threads
    int acc = 0, xb = 0;
    uint32_t aph[2] = {0, 0}, xph[2] = {0, 0};
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
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
      const int cpitch = rowbytes + 8;
      const int ng = D / a.G;
      if (!epi_all(mbar_wait(tfull_bar(acc), aph[acc], abort_flag, a.status))) break;
      fence_after();
      float v[D];
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * D);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) tmem_ld32(tb + c0, v + c0);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      aph[acc] ^= 1;
      acc ^= 1;
      const int64_t row0 = (int64_t)lh * c.T + t0;   // first residual row of the tile
      if (COMPRESS) {
        if (!epi_all(mbar_wait(xfull_bar(xb), xph[xb], abort_flag, a.status))) break;
        float x[D];
        const uint8_t* xs = sX + xb * S_X;
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 w = *reinterpret_cast<const uint4*>(xs + hh * 16384 + rl * 128 + ((ch ^ (rl & 7)) << 4));
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              x[hh * 64 + ch * 8 + 2 * j] = __uint_as_float(u[j] << 16);
              x[hh * 64 + ch * 8 + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
            }
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(xempty_bar(xb));
        xph[xb] ^= 1;
        xb ^= 1;
        if (c.rope && valid) {
          const float4* cs4 = reinterpret_cast<const float4*>(a.cs + (int64_t)t * (D / 2));
#pragma unroll
          for (int i = 0; i < D / 2; i += 2) {
            const float4 q2 = cs4[i / 2];
            const float cc[2] = {q2.x, q2.z}, ss[2] = {q2.y, q2.w};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float yi = x[i + j], yj = x[i + j + D / 2];
              x[i + j] = __fadd_rn(__fmul_rn(yi, cc[j]), __fmul_rn(yj, ss[j]));
              x[i + j + D / 2] = __fsub_rn(__fmul_rn(yj, cc[j]), __fmul_rn(yi, ss[j]));
            }
          }
        }
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = __fsub_rn(x[d], v[d]);
        // rotation
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = __fmul_rn(x[d], sSign[d]);
        fwht_row<D>(x);
        const float rs = (float)(1.0 / sqrt((double)D));
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = __fmul_rn(x[d], rs);
        RowPack<D> op{x, sCode + rl * cpitch, sScale + rl * 4};
        dispatch_gb<D>(a.G, b, op);
        epi_sync();
        // coalesced copy of the tile's packed rows and scales to global
        {
          const int wpr = rowbytes / 8;
          uint64_t* gdst = reinterpret_cast<uint64_t*>(o.codes + row0 * rowbytes);
          for (int u = et; u < nrows * wpr; u += 128) {
            const int rr = u / wpr, w = u - rr * wpr;
            gdst[u] = *reinterpret_cast<const uint64_t*>(sCode + rr * cpitch + w * 8);
          }
          float* sdst = o.scales + row0 * ng;
          for (int u = et; u < nrows * ng; u += 128) sdst[u] = sScale[(u / ng) * 4 + (u % ng)];
        }
        epi_sync();
      } else {
        if (b > 0) {
          // coalesced load of the tile's codes and scales into staging
          const int wpr = rowbytes / 8;
          const uint64_t* gsrc = reinterpret_cast<const uint64_t*>(o.codes + row0 * rowbytes);
          for (int u = et; u < nrows * wpr; u += 128) {
            const int rr = u / wpr, w = u - rr * wpr;
            *reinterpret_cast<uint64_t*>(sCode + rr * cpitch + w * 8) = gsrc[u];
          }
          const float* ssrc = o.scales + row0 * ng;
          for (int u = et; u < nrows * ng; u += 128) sScale[(u / ng) * 4 + (u % ng)] = ssrc[u];
          epi_sync();
          if (valid) {
            float e[D];
            RowUnpack<D> op{e, sCode + rl * cpitch, sScale + rl * 4};
            dispatch_gb<D>(a.G, b, op);
            fwht_row<D>(e);
            const float rs = (float)(1.0 / sqrt((double)D));
#pragma unroll
            for (int d = 0; d < D; ++d) v[d] = __fadd_rn(v[d], __fmul_rn(__fmul_rn(e[d], rs), sSign[d]));
          }
        }
        if (c.rope && valid) {
          const float4* cs4 = reinterpret_cast<const float4*>(a.cs + (int64_t)t * (D / 2));
#pragma unroll
          for (int i = 0; i < D / 2; i += 2) {
            const float4 q2 = cs4[i / 2];
            const float cc[2] = {q2.x, q2.z}, ss[2] = {q2.y, q2.w};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float x0 = v[i + j], x1 = v[i + j + D / 2];
              v[i + j] = __fsub_rn(__fmul_rn(x0, cc[j]), __fmul_rn(x1, ss[j]));
              v[i + j + D / 2] = __fadd_rn(__fmul_rn(x1, cc[j]), __fmul_rn(x0, ss[j]));
            }
          }
        }
        // decoded row -> staging (bf16), then coalesced 16-byte stores
        uint8_t* srow = sOut + rl * ROWPITCH_OUT;
#pragma unroll
        for (int d = 0; d < D; d += 8) {
          uint4 w;
          w.x = (uint32_t)bf16_bits_from_f32(v[d]) | ((uint32_t)bf16_bits_from_f32(v[d + 1]) << 16);
          w.y = (uint32_t)bf16_bits_from_f32(v[d + 2]) | ((uint32_t)bf16_bits_from_f32(v[d + 3]) << 16);
          w.z = (uint32_t)bf16_bits_from_f32(v[d + 4]) | ((uint32_t)bf16_bits_from_f32(v[d + 5]) << 16);
          w.w = (uint32_t)bf16_bits_from_f32(v[d + 6]) | ((uint32_t)bf16_bits_from_f32(v[d + 7]) << 16);
          *reinterpret_cast<uint4*>(srow + d * 2) = w;
        }
        epi_sync();
        {
          uint16_t* base = (c.kind == 0 ? a.out_k : a.out_v) + (int64_t)c.seq * a.osb + (int64_t)(c.l0 + l) * a.osl +
                           (int64_t)h * a.osh;
          constexpr int UPR = D * 2 / 16;    // 16-byte units per row
          for (int u = et; u < nrows * UPR; u += 128) {
            const int rr = u / UPR, w = u - rr * UPR;
            *reinterpret_cast<uint4*>(base + (int64_t)(t0 + rr) * a.ost + w * 8) =
                *reinterpret_cast<const uint4*>(sOut + rr * ROWPITCH_OUT + w * 16);
          }
        }
        epi_sync();
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
