// tcgen05 (5th-generation tensor core) GEMM for the randomized token-mode
// range finder of "A JoLT for the KV Cache", Section 3.1 ("FlashJoLT":
// a randomized approximation of the leading token-mode singular vectors).
//
// One persistent CTA per SM: warp 0 issues TMA loads (no multicast), warp 1
// owns the TMEM accumulators and one elected thread issues tcgen05.mma
// (kind::f16, bf16 x bf16 -> fp32), warps 2..5 drain the accumulators with
// tcgen05.ld and store. Two accumulators in TMEM let the epilogue of one tile
// overlap the main loop of the next (one, when the CTA-pair kernel's N tiles
// are wider than 256 columns). Every mbarrier wait is bounded by a
// wall-clock deadline; on expiry the kernel records a timeout in the status
// word, stops issuing, waits (bounded) for its own loads in flight, frees its
// TMEM and returns.
//
// Shapes (per cell c; all operands bf16, 128-byte swizzled 64-wide K slices):
//   XW : Y^T[c] (k x T, bf16, transposed store) = (X_(T) W)^T, K = N_c,
//        A = X tile (K-major), B = W^T [k][N_c] (K-major)
//   XTY: Z[c]   (N_c x k, fp32)               = X_(T)^T Y,    K = T,
//        A = X tile read along t (MN-major), B = Y^T [k][T] (K-major)
//   GRAM: G[c]  (k x k, fp32)                 = Y^T Y,        K = T,
//        A = B = Y^T [k][T] (K-major)
//   WP : U^T[c] (r x T, bf16, transposed)     = (Y P)^T,      K = k,
//        A = Y^T read along t (MN-major), B = P^T [r][k] (K-major)
//   FG : partial feature Gram over a chunk of rows (l, h, t): A = B = the
//        same X tile read along t (MN-major), 128 feature rows (one head of
//        D = 128 or two heads of D = 64), fp32 [cells][chunks][128][128]
#pragma once
#include <cuda.h>
#include "jolt_internal.cuh"

namespace jolt {
namespace umma {

enum Mode : int { XW = 0, XTY = 1, GRAM = 2, WP = 3, FG = 4 };
// FG: k-steps (64 rows each) the tensor cores accumulate before the epilogue
// adds the partial into its fp32 sums
constexpr int FG_PROMOTE = 4;

constexpr int BM = 128;          // rows of an output tile (TMEM lanes)
constexpr int BK = 64;           // K per pipeline stage (128 bytes of bf16)
constexpr int BN_MAX = 256;
constexpr int MAX_STAGES = 8;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int SMEM_DATA_MAX = 224 * 1024;     // pipeline stages (plus 1 KB alignment and barriers)
// Bytes of one pipeline stage for an output tile BN wide (A tile + B tile,
// each a whole number of 1 KB swizzle atoms), and the stages that fit.
__host__ __device__ inline int stage_bytes(int BN) { return A_BYTES + (BN * BK * 2 + 1023) / 1024 * 1024; }
__host__ __device__ inline int num_stages(int BN) {
  const int n = SMEM_DATA_MAX / stage_bytes(BN);
  return n < MAX_STAGES ? n : MAX_STAGES;
}
__host__ __device__ inline int smem_bytes(int BN) { return num_stages(BN) * stage_bytes(BN) + 1024 + 256; }
constexpr int THREADS = 192;
constexpr unsigned long long WAIT_NS = 2000000000ull;   // 2 s per wait

struct Problem {
  int mode;
  int ncells;
  int M, N, Kdim;        // per-cell extents (max over cells for XTY's M)
  int BN;                // output tile width (multiple of 16, <= 256)
  int mt, nt;            // tiles per cell along M and N
  int H, D;              // heads and head dim (X addressing)
  int T, t_pitch;        // tokens, row pitch of the transposed bf16 outputs
  int nbatch;            // batch extent of the X tensor maps (FG: out-of-range fill)
  int fg_chunks, fg_spc; // FG: row chunks per cell, 64-token steps per chunk
  const int* cell_l0;    // [cells] first layer of the cell's group
  const int* cell_b;     // [cells] sequence
  const int* cell_Lg;    // [cells] layers in the group
  const int* cell_kind;  // [cells] 0 = K, 1 = V (selects the X tensor map)
  // outputs
  uint16_t* out_bf16;    // XW: [cells][N][t_pitch]
  float* out_f32;        // XTY: [cells][Mmax][N]; GRAM: [cells][N][N]
  int64_t out_cell_stride;
  const int* wp_rows;    // WP: r_T per cell (columns >= r_T not stored)
  uint16_t* const* wp_dst;   // WP: per-cell U^T base, row pitch t_pitch
  int* status;
  int pair;              // 1: CTA pairs (tcgen05 cta_group::2), M = 256 per pair; XW and XTY only
  // pair mode, N tiles wider than 256: one TMEM accumulator of up to 512
  // columns and two MMAs per 16-wide K step. N tile j covers the columns
  // [tn0[j], tn0[j] + ta[j] + tb[j]); its MMAs are ta[j] and tb[j] wide, and
  // each CTA loads half of each one's B rows with maps.bt (tmap 0) or
  // maps.bt2 (tmap 1), whose boxes are that many rows high. BN is the widest
  // tile (it sizes the pipeline stages).
  int wide;
  int tn0[4], ta[4], tb[4], tmap_a[4], tmap_b[4];
};

struct Maps {
  CUtensorMap xk;     // X of keys (5D: d, t, h, l, b), box {64, 64, 1, 1, 1}
  CUtensorMap xv;     // X of values
  CUtensorMap bt;     // XW: W^T [cells][k][N_c]; XTY/GRAM: Y^T [cells][k][T]; WP: P^T [cells][r][k]; box {64, BN}
  CUtensorMap at;     // GRAM: Y^T, box {64, 128}; WP: Y^T read along t, box {64, 64}
  CUtensorMap bt2;    // wide pair tiles: the second B box height (same tensor as bt)
  // pair mode: bt's box is {64, BN/2}, each CTA of a pair loads its half of the N columns
};

}  // namespace umma

jolt_status launch_umma(const umma::Maps& maps, const umma::Problem& p, cudaStream_t s);

}  // namespace jolt

#if defined(JOLT_UMMA_IMPL) || defined(JOLT_PTX_HELPERS)
#ifndef JOLT_PTX_HELPERS_DONE
#define JOLT_PTX_HELPERS_DONE
namespace jolt {
namespace umma {

// ------------------------------------------------------------ PTX helpers --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: true when the phase completed, false on abort or timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort_flag) return false;
    if (now_ns() - t0 > WAIT_NS) {
      *abort_flag = 1;
      atomicOr(status, DEV_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, tcgen05 version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;                 // version
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::f16, A/B bf16, D fp32, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

}  // namespace umma
}  // namespace jolt
#endif  // JOLT_PTX_HELPERS_DONE
#endif  // helpers

#ifdef JOLT_UMMA_IMPL
namespace jolt {
namespace umma {

// Tile -> (cell, m0, n0)
__device__ __forceinline__ void tile_coords(const Problem& p, int tile, int& cell, int& m0, int& n0) {
  const int per_cell = p.mt * p.nt;
  cell = tile / per_cell;
  const int r = tile - cell * per_cell;
  m0 = (r / p.nt) * BM;
  n0 = (r % p.nt) * p.BN;
}

__device__ __forceinline__ int cell_K(const Problem& p, int cell) {
  if (p.mode == XW) return p.cell_Lg[cell] * p.H * p.D;
  return p.Kdim;
}
__device__ __forceinline__ int cell_M(const Problem& p, int cell) {
  if (p.mode == XTY) return p.cell_Lg[cell] * p.H * p.D;
  if (p.mode == FG) return p.fg_chunks * BM;
  return p.M;
}
// FG: 64-token steps of a cell = (groups of 128 feature rows) x ceil(T/64)
__device__ __forceinline__ int fg_total_steps(const Problem& p, int cell) {
  const int rows = p.cell_Lg[cell] * p.H * p.D;
  return ((rows + 127) / 128) * ((p.T + 63) / 64);
}
// K steps [kb0, kb1) of the tile with row offset m0 in cell `cell`
__device__ __forceinline__ void k_range(const Problem& p, int cell, int m0, int& kb0, int& kb1) {
  if (p.mode == FG) {
    const int c = m0 / BM;
    kb0 = c * p.fg_spc;
    kb1 = min(kb0 + p.fg_spc, fg_total_steps(p, cell));
    return;
  }
  kb0 = 0;
  kb1 = (cell_K(p, cell) + BK - 1) / BK;
}

__global__ void __launch_bounds__(THREADS, 1) k_umma_gemm(const __grid_constant__ Maps maps, Problem p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int STAGES = num_stages(p.BN), STAGE_BYTES = stage_bytes(p.BN);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const int ncols = (2 * p.BN <= 64) ? 64 : (2 * p.BN <= 128) ? 128 : (2 * p.BN <= 256) ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull_bar(b), 1); mbar_init(tempty_bar(b), 4); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = p.ncells * p.mt * p.nt;
  const int a_mn = (p.mode == XTY || p.mode == WP || p.mode == FG) ? 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued_phase[MAX_STAGES];
      bool issued[MAX_STAGES];
      for (int s = 0; s < MAX_STAGES; ++s) issued[s] = false;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        int cell, m0, n0;
        tile_coords(p, tile, cell, m0, n0);
        if (m0 >= cell_M(p, cell)) continue;
        if (p.mode == WP && n0 >= p.wp_rows[cell]) continue;
        int kb0, kb1;
        k_range(p, cell, m0, kb0, kb1);
        if (kb0 >= kb1) continue;
        const CUtensorMap* xm = (p.cell_kind[cell] == 0) ? &maps.xk : &maps.xv;
        const int l0 = p.cell_l0[cell], b = p.cell_b[cell];
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t sa = sbase + stage * STAGE_BYTES, sb = sa + A_BYTES;
          const uint32_t fb = full_bar(stage);
          const uint32_t bbytes = (p.mode == FG) ? 0u : (uint32_t)p.BN * BK * 2;
          mbar_expect_tx(fb, A_BYTES + bbytes);
          const int k0 = kb * BK;
          if (p.mode == FG) {
            const int tsteps = (p.T + 63) / 64;
            const int grp = kb / tsteps, t0 = (kb % tsteps) * 64;
            const int nlh = p.cell_Lg[cell] * p.H;
            for (int half = 0; half < 2; ++half) {
              const int m = grp * 128 + 64 * half;
              const int lh = m / p.D, d0 = m % p.D;
              // a head past the cell reads an out-of-range batch index: zero fill
              const int bb = (lh < nlh) ? b : p.nbatch;
              const int lhc = (lh < nlh) ? lh : 0;
              tma_load_5d(sa + 8192 * half, xm, fb, d0, t0, lhc % p.H, l0 + lhc / p.H, bb);
            }
          } else if (p.mode == XW) {
            // K index n = (l*H + h)*D + d: one (l, h) block per 64-wide slice when D = 64,
            // half of one when D = 128. Rows t = m0 .. m0+127 as two 64-row boxes.
            const int lh = k0 / p.D, d0 = k0 % p.D;
            const int l = l0 + lh / p.H, h = lh % p.H;
            tma_load_5d(sa, xm, fb, d0, m0, h, l, b);
            tma_load_5d(sa + 8192, xm, fb, d0, m0 + 64, h, l, b);
            tma_load_3d(sb, &maps.bt, fb, k0, n0, cell);
          } else if (p.mode == XTY) {
            // rows m = (l*H + h)*D + d: two 64-row halves, each one 64-wide d slice
            for (int half = 0; half < 2; ++half) {
              const int m = m0 + 64 * half;
              const int lh = m / p.D, d0 = m % p.D;
              tma_load_5d(sa + 8192 * half, xm, fb, d0, k0, lh % p.H, l0 + lh / p.H, b);
            }
            tma_load_3d(sb, &maps.bt, fb, k0, n0, cell);
          } else if (p.mode == GRAM) {
            tma_load_3d(sa, &maps.at, fb, k0, m0, cell);
            tma_load_3d(sb, &maps.bt, fb, k0, n0, cell);
          } else {   // WP
            tma_load_3d(sa, &maps.at, fb, m0, k0, cell);
            tma_load_3d(sa + 8192, &maps.at, fb, m0 + 64, k0, cell);
            tma_load_3d(sb, &maps.bt, fb, k0, n0, cell);
          }
          issued[stage] = true;
          issued_phase[stage] = ph;
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
        }
      }
      // drain: every load this thread issued has landed before the CTA exits
      for (int s = 0; s < STAGES; ++s)
        if (issued[s]) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try(full_bar(s), issued_phase[s]) && now_ns() - t0 < WAIT_NS) {}
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph[2] = {0, 0};
      const uint32_t idesc = idesc_bf16(p.BN, a_mn, p.mode == FG ? 1 : 0);
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        int cell, m0, n0;
        tile_coords(p, tile, cell, m0, n0);
        if (m0 >= cell_M(p, cell)) continue;
        if (p.mode == WP && n0 >= p.wp_rows[cell]) continue;
        int kb0, kb1;
        k_range(p, cell, m0, kb0, kb1);
        if (kb0 >= kb1) continue;
        // FG sums squares: its tile is cut into sub-tiles of FG_PROMOTE
        // k-steps, each accumulated afresh and added up by the epilogue in
        // fp32 with round-to-nearest (see the epilogue)
        const int sub = (p.mode == FG) ? FG_PROMOTE : (kb1 - kb0);
        uint32_t dcol = 0;
        for (int kb = kb0; kb < kb1; ++kb) {
          const int ks = (kb - kb0) % sub;
          if (ks == 0) {
            if (!mbar_wait(tempty_bar(acc), aph[acc] ^ 1, abort_flag, p.status)) { ok = false; break; }
            fence_after();
            dcol = tmem + (uint32_t)(acc * p.BN);
          }
          if (!mbar_wait(full_bar(stage), ph, abort_flag, p.status)) { ok = false; break; }
          fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: +32 bytes per 16 K; MN-major: +2 groups of 8 K-rows (2048 bytes)
            const uint64_t da = a_mn ? sdesc(sa + kk * 2048, 8192, 1024) : sdesc(sa + kk * 32, 16, 1024);
            const uint64_t db = (p.mode == FG) ? da : sdesc(sb + kk * 32, 16, 1024);
            mma_bf16(dcol, da, db, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
          if (ks == sub - 1 || kb == kb1 - 1) {
            mma_commit(tfull_bar(acc));
            aph[acc] ^= 1;
            acc ^= 1;
          }
        }
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    int acc = 0;
    uint32_t aph[2] = {0, 0};
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      int cell, m0, n0;
      tile_coords(p, tile, cell, m0, n0);
      const int Mc = cell_M(p, cell);
      if (m0 >= Mc) continue;
      if (p.mode == WP && n0 >= p.wp_rows[cell]) continue;
      int kb0, kb1;
      k_range(p, cell, m0, kb0, kb1);
      if (kb0 >= kb1) continue;
      if (p.mode == FG) {
        // the tile's sub-tiles (FG_PROMOTE k-steps each, accumulated by the
        // tensor cores) summed here in fp32, round-to-nearest: the tensor
        // cores' own fp32 accumulation loses a fraction of an ulp per step
        // toward zero, a bias that grows with the number of steps over a sum
        // of squares, so it is kept to FG_PROMOTE steps at a time
        const int nsub = (kb1 - kb0 + FG_PROMOTE - 1) / FG_PROMOTE;
        float sum[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) sum[i] = 0.0f;
        bool ok = true;
        for (int sidx = 0; sidx < nsub; ++sidx) {
          if (!mbar_wait(tfull_bar(acc), aph[acc], abort_flag, p.status)) { ok = false; break; }
          fence_after();
          const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.BN);
#pragma unroll
          for (int c0 = 0; c0 < 128; c0 += 16) {
            float v[16];
            tmem_ld16(tb + c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) sum[c0 + i] = __fadd_rn(sum[c0 + i], v[i]);
          }
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
          aph[acc] ^= 1;
          acc ^= 1;
        }
        if (!ok) break;
        float* dst = p.out_f32 + ((int64_t)cell * p.fg_chunks + m0 / BM) * (BM * 128) + (int64_t)(q * 32 + lane) * 128;
#pragma unroll
        for (int i = 0; i < 128; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(sum[i], sum[i + 1], sum[i + 2], sum[i + 3]);
        continue;
      }
      if (!mbar_wait(tfull_bar(acc), aph[acc], abort_flag, p.status)) break;
      fence_after();
      const int row = m0 + q * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.BN);
      for (int c0 = 0; c0 < p.BN; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + c0, v);
        const int n = n0 + c0;
        if (p.mode == XW) {
          if (row < p.T) {
            uint16_t* dst = p.out_bf16 + (int64_t)cell * p.out_cell_stride + row;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < p.N) dst[(int64_t)(n + i) * p.t_pitch] = bf16_bits_from_f32(v[i]);
          }
        } else if (p.mode == XTY || p.mode == GRAM) {
          if (row < Mc) {
            float* dst = p.out_f32 + (int64_t)cell * p.out_cell_stride + (int64_t)row * p.N;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < p.N) dst[n + i] = v[i];
          }
        } else {   // WP
          const int rr = p.wp_rows[cell];
          if (row < p.t_pitch) {
            uint16_t* dst = p.wp_dst[cell] + row;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < rr) dst[(int64_t)(n + i) * p.t_pitch] = bf16_bits_from_f32(row < p.T ? v[i] : 0.0f);
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      aph[acc] ^= 1;
      acc ^= 1;
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
  }
}

// ------------------------------------------------------------------------
// CTA-pair variant of the X W and X^T Y passes (tcgen05 cta_group::2): a
// cluster of two CTAs computes a 256 x BN tile. Each CTA loads its own 128
// rows of A and half of the BN columns of B into the same shared-memory
// offsets; the leader CTA (rank 0) issues the 256-row MMA, which reads both
// CTAs' operands and leaves each CTA's 128 rows of the result in that CTA's
// TMEM. Per CTA a stage is 16 KB of A and BN/2 x 128 bytes of B, half the B
// traffic of the single-CTA tile. Barriers: the leader's full[s] counts the
// bytes of both CTAs' loads (the leader's producer arms it); the leader's
// commit arrives on empty[s] and tfull[b] of both CTAs; both CTAs' epilogue
// warps arrive on the leader's tempty[b]. No load is multicast.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void tma2_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma2_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                             int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
__device__ __forceinline__ void mma2_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma2_commit_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__host__ __device__ inline int pair_stage_bytes(int BN) { return A_BYTES + ((BN / 2) * BK * 2 + 1023) / 1024 * 1024; }
__host__ __device__ inline int pair_num_stages(int BN) {
  const int n = SMEM_DATA_MAX / pair_stage_bytes(BN);
  return n < MAX_STAGES ? n : MAX_STAGES;
}
__host__ __device__ inline int pair_smem_bytes(int BN) { return pair_num_stages(BN) * pair_stage_bytes(BN) + 1024 + 256; }

__global__ void __launch_bounds__(THREADS, 1) k_umma_gemm_pair(const __grid_constant__ Maps maps, Problem p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int STAGES = pair_num_stages(p.BN), STAGE_BYTES = pair_stage_bytes(p.BN);
  const int BNH = p.BN / 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES] (leader), empty[STAGES], tfull[2], tempty[2] (leader)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  // two accumulators (the epilogue of one tile overlaps the next tile's main
  // loop) while they fit in TMEM's 512 columns; wide tiles have one
  const int nacc = p.wide ? 1 : 2;
  const int ncols = p.wide ? 512 : (2 * p.BN <= 64) ? 64 : (2 * p.BN <= 128) ? 128 : (2 * p.BN <= 256) ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull_bar(b), 1); mbar_init(tempty_bar(b), 8); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  cluster_sync_all();          // both CTAs' barriers exist before any remote arrival
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const int mt2 = (p.M + 2 * BM - 1) / (2 * BM);
  const int ntiles = p.ncells * mt2 * p.nt;
  const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued_phase[MAX_STAGES];
      bool issued[MAX_STAGES];
      for (int s = 0; s < MAX_STAGES; ++s) issued[s] = false;
      bool ok = true;
      for (int tile = pair_id; tile < ntiles && ok; tile += npairs) {
        const int cell = tile / (mt2 * p.nt);
        const int r = tile - cell * (mt2 * p.nt);
        const int m0 = (r / p.nt) * (2 * BM) + (int)rank * BM;
        const int j = r % p.nt;
        // B rows of this CTA: one box of BN/2 rows, or (wide) one box per MMA
        const int n0 = p.wide ? p.tn0[j] + (int)rank * (p.ta[j] / 2) : j * p.BN + (int)rank * BNH;
        const int n1 = p.wide ? p.tn0[j] + p.ta[j] + (int)rank * (p.tb[j] / 2) : 0;
        const CUtensorMap* bma = (p.wide && p.tmap_a[j]) ? &maps.bt2 : &maps.bt;
        const CUtensorMap* bmb = (p.wide && p.tmap_b[j]) ? &maps.bt2 : &maps.bt;
        const uint32_t sb1 = p.wide ? (uint32_t)(p.ta[j] / 2) * (BK * 2) : 0u;
        const uint32_t stage_tx =
            2u * (uint32_t)(A_BYTES + (p.wide ? (p.ta[j] + p.tb[j]) / 2 : BNH) * BK * 2);
        const int Kc = (p.mode == XW) ? p.cell_Lg[cell] * p.H * p.D : p.Kdim;
        const int nkb = (Kc + BK - 1) / BK;
        const CUtensorMap* xm = (p.cell_kind[cell] == 0) ? &maps.xk : &maps.xv;
        const int l0 = p.cell_l0[cell], b = p.cell_b[cell];
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t sa = sbase + stage * STAGE_BYTES, sb = sa + A_BYTES;
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (rank == 0) mbar_expect_tx(full_bar(stage), stage_tx);
          const int k0 = kb * BK;
          if (p.mode == XW) {
            const int lh = k0 / p.D, d0 = k0 % p.D;
            const int l = l0 + lh / p.H, h = lh % p.H;
            tma2_load_5d(sa, xm, fb, d0, m0, h, l, b);
            tma2_load_5d(sa + 8192, xm, fb, d0, m0 + 64, h, l, b);
          } else {
            for (int half = 0; half < 2; ++half) {
              const int m = m0 + 64 * half;
              const int lh = m / p.D, d0 = m % p.D;
              tma2_load_5d(sa + 8192 * half, xm, fb, d0, k0, lh % p.H, l0 + lh / p.H, b);
            }
          }
          tma2_load_3d(sb, bma, fb, k0, n0, cell);
          if (p.wide) tma2_load_3d(sb + sb1, bmb, fb, k0, n1, cell);
          issued[stage] = true;
          issued_phase[stage] = ph;
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
        }
      }
      // drain: the leader's full barriers count both CTAs' loads, so the
      // leader waits (bounded) for every stage it armed before the final sync
      if (rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) {
            const unsigned long long t0 = now_ns();
            while (!mbar_try(full_bar(s), issued_phase[s]) && now_ns() - t0 < WAIT_NS) {}
          }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph[2] = {0, 0};
      const int a_mn = (p.mode == XTY) ? 1 : 0;
      auto idesc_n = [&](int n) {
        return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)(n >> 3) << 17) |
               ((uint32_t)((2 * BM) >> 4) << 24);
      };
      bool ok = true;
      for (int tile = pair_id; tile < ntiles && ok; tile += npairs) {
        const int cell = tile / (mt2 * p.nt);
        const int j = (tile - cell * (mt2 * p.nt)) % p.nt;
        const int Kc = (p.mode == XW) ? p.cell_Lg[cell] * p.H * p.D : p.Kdim;
        const int nkb = (Kc + BK - 1) / BK;
        // one MMA BN wide, or (wide) two: ta[j] columns, then tb[j] columns
        // whose B rows follow the first MMA's in shared memory
        const int na = p.wide ? p.ta[j] : p.BN;
        const uint32_t idesc = idesc_n(na);
        const uint32_t idesc1 = p.wide ? idesc_n(p.tb[j]) : 0u;
        const uint32_t sb1 = p.wide ? (uint32_t)(p.ta[j] / 2) * (BK * 2) : 0u;
        if (!mbar_wait(tempty_bar(acc), aph[acc] ^ 1, abort_flag, p.status)) break;
        fence_after();
        const uint32_t dcol = tmem + (uint32_t)(acc * p.BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(full_bar(stage), ph, abort_flag, p.status)) { ok = false; break; }
          fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t da = a_mn ? sdesc(sa + kk * 2048, 8192, 1024) : sdesc(sa + kk * 32, 16, 1024);
            const uint64_t db = sdesc(sb + kk * 32, 16, 1024);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            mma2_bf16(dcol, da, db, idesc, accum);
            if (p.wide) mma2_bf16(dcol + (uint32_t)na, da, sdesc(sb + sb1 + kk * 32, 16, 1024), idesc1, accum);
          }
          mma2_commit_both(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma2_commit_both(tfull_bar(acc));
        aph[acc] ^= 1;
        if (nacc == 2) acc ^= 1;
      }
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    int acc = 0;
    uint32_t aph[2] = {0, 0};
    for (int tile = pair_id; tile < ntiles; tile += npairs) {
      const int cell = tile / (mt2 * p.nt);
      const int r = tile - cell * (mt2 * p.nt);
      const int m0 = (r / p.nt) * (2 * BM) + (int)rank * BM;
      const int j = r % p.nt;
      const int n0 = p.wide ? p.tn0[j] : j * p.BN;
      const int wn = p.wide ? p.ta[j] + p.tb[j] : p.BN;
      const int Mc = (p.mode == XTY) ? p.cell_Lg[cell] * p.H * p.D : p.M;
      if (!mbar_wait(tfull_bar(acc), aph[acc], abort_flag, p.status)) break;
      fence_after();
      const int row = m0 + q * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.BN);
      for (int c0 = 0; c0 < wn; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + c0, v);
        const int n = n0 + c0;
        if (p.mode == XW) {
          if (row < p.T) {
            uint16_t* dst = p.out_bf16 + (int64_t)cell * p.out_cell_stride + row;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < p.N) dst[(int64_t)(n + i) * p.t_pitch] = bf16_bits_from_f32(v[i]);
          }
        } else {
          if (row < Mc) {
            float* dst = p.out_f32 + (int64_t)cell * p.out_cell_stride + (int64_t)row * p.N;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < p.N) dst[n + i] = v[i];
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(tempty_bar(acc), 0));
      aph[acc] ^= 1;
      if (nacc == 2) acc ^= 1;
    }
  }
  fence_before();
  __syncthreads();
  cluster_sync_all();          // no remote arrival or MMA is outstanding on either CTA
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
  }
}

}  // namespace umma
}  // namespace jolt

#endif  // JOLT_UMMA_IMPL
