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
#include "jolt_stream.cuh"

namespace jolt {
namespace strm {

using namespace umma;

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
