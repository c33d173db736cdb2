// Fused decode attention over the compressed cache ("A JoLT for the KV
// Cache", Section 3.1: the decode kernel attends directly over the stored
// factors and the packed residual, without materialising the dense cache).
//
// One decode step of layer l: for query head j (already rotated for its
// position), out_j = sum_t softmax_t(q_j . k_t / sqrt(D)) v_t over the T
// compressed tokens and a dense tail of new tokens, with one softmax over
// both. Query head j reads KV head j / G (G query heads per KV head).
//
// Keys are rebuilt tile by tile on chip, as decompression does: the backbone
// U_T^[tile] M^_K (128 tokens x D) on tcgen05 into TMEM, plus the unpacked,
// de-rotated residual (two threads per row, the same transform as the
// decompress kernel), then RoPE. Values never leave rank space: the kernel
// accumulates p^T U_T^V (r_T values per query head) and p^T dequant(codes_V)
// in the rotated domain (D values); the merge kernel applies M^_V and the
// inverse rotation once per query head, which is exact by linearity. The token
// range of each (sequence, KV head) is split over CTAs (flash-decoding); the
// merge kernel combines the splits' softmax states and the dense tail.
//
// Warp roles as in the stream kernel: warp 0 issues TMA loads of U_T^ / M^
// slices and bulk copies of the key codes, warp 1 issues the MMAs, warps
// 2..9 are the epilogue (scores, online softmax, value accumulation).
#include <algorithm>
#include <vector>

#include "jolt_stream.cuh"

namespace jolt {
namespace dec {

using namespace umma;
using namespace strm;

constexpr int GMAX = 8;          // query heads per KV head
constexpr int RVMAX = 512;       // value token rank (rank-space accumulators)
constexpr int BMAX = DEC_BMAX;   // sequences per launch (one U_T^ tensor map each)

// shared-memory layout (bytes, from the 1 KB-aligned base)
constexpr int OFF_RING = 0;
constexpr int OFF_KCODE = SSTAGES * (S_A + S_B);                    // 2 x (codes + scales) of keys
constexpr int TSUB = 32;         // tokens per staged U_T^V slice
constexpr int UP = TSUB + 2;     // its row pitch in bf16 (17 words: rank rows on distinct banks)
constexpr int OFF_U = OFF_KCODE + 2 * (S_CODE + S_SCALE);            // [RVMAX r][UP] bf16
constexpr int OFF_VCODE = OFF_U + RVMAX * UP * 2;                    // [128][<= 128 bytes]
constexpr int OFF_VSCALE = OFF_VCODE + S_CODE;                       // [128][<= 4] fp32
constexpr int OFF_Q = OFF_VSCALE + S_SCALE;                          // [GMAX][128] fp32
constexpr int OFF_P = OFF_Q + GMAX * 128 * 4;                        // [128 t][GMAX] fp32
constexpr int OFF_PART = OFF_P + GMAX * 128 * 4;                     // [GMAX][128][2] fp32
constexpr int OFF_RED = OFF_PART + GMAX * 128 * 2 * 4;               // [2][GMAX][4] fp32
constexpr int OFF_SIGN = OFF_RED + 2 * GMAX * 4 * 4;                 // [128] fp32
constexpr int OFF_ERED = OFF_SIGN + 128 * 4;                         // [4][GMAX][128] fp32 (item end)
constexpr int OFF_BAR = OFF_ERED + 4 * GMAX * 128 * 4;
constexpr int SMEM_DEC = OFF_BAR + 256 + 1024;
static_assert(SMEM_DEC <= 227 * 1024, "decode attention shared memory");

struct Maps {
  CUtensorMap mt;          // M^_K^T workspace [B*H][D][rpk] bf16, box {64 r, D}
  CUtensorMap ut[BMAX];    // U_T^ of each sequence's key cell [rT][t_pitch], box {64 t, 64 r}
};

struct Args {
  int B, H, T, G, gq, li, nsplit, per;     // per: tokens per split (multiple of 128)
  const CellOut* kout;     // key cell of this layer's group for sequence 0; sequence b at b * cstride
  const CellOut* vout;     // value cells, same stride
  int cstride;
  const float2* cs;        // RoPE table (keys), or null
  uint64_t seed;           // rotation seed of sequence 0 (sequence b: seed + b)
  const float* q;          // [B][H*G][D]
  float* part;             // [B][H][nsplit][G][2 + rpv + D]
  int rpv;                 // rank pitch of the value state (multiple of 64)
  int* status;
};

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Work item -> (sequence, KV head, split); consecutive items are the KV heads
// of one (sequence, split), which share U_T^ rows in L2.
__device__ __forceinline__ void item_of(const Args& a, int it, int& b, int& h, int& s) {
  h = it % a.H;
  const int r = it / a.H;
  s = r % a.nsplit;
  b = r / a.nsplit;
}

template <int D>
__global__ void __launch_bounds__(STHREADS, 1) k_dec_attn(const __grid_constant__ Maps maps, Args a) {
  constexpr int C = D / 4;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem + OFF_RING;
  uint8_t* sB = sA + SSTAGES * S_A;
  uint8_t* sK = smem + OFF_KCODE;
  uint16_t* sU = reinterpret_cast<uint16_t*>(smem + OFF_U);
  uint8_t* sVC = smem + OFF_VCODE;
  float* sVS = reinterpret_cast<float*>(smem + OFF_VSCALE);
  float* sQ = reinterpret_cast<float*>(smem + OFF_Q);
  float* sP = reinterpret_cast<float*>(smem + OFF_P);
  float* sPart = reinterpret_cast<float*>(smem + OFF_PART);
  float* sRed = reinterpret_cast<float*>(smem + OFF_RED);
  float* sSign = reinterpret_cast<float*>(smem + OFF_SIGN);
  float* sEred = reinterpret_cast<float*>(smem + OFF_ERED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SSTAGES + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (SSTAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 2 + b); };
  auto xfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 4 + b); };
  auto xempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 6 + b); };
  auto kbuf = [&](int b) { return sK + b * (S_CODE + S_SCALE); };
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
  const int nitems = a.B * a.H * a.nsplit;
  const int G = a.G;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, xb = 0;
      uint32_t ph = 0, xph[2] = {0, 0};
      uint32_t issued_phase[SSTAGES], xissued_phase[2];
      bool issued[SSTAGES], xissued[2] = {false, false};
      for (int s = 0; s < SSTAGES; ++s) issued[s] = false;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        int b, h, s;
        item_of(a, it, b, h, s);
        const CellOut ok_ = a.kout[b * a.cstride];
        const int tb = s * a.per, te = min(a.T, tb + a.per);
        const int nk = (ok_.rT + 63) / 64;
        for (int t0 = tb; t0 < te && ok; t0 += SBM) {
          if (ok_.b > 0) {
            if (!mbar_wait(xempty_bar(xb), xph[xb] ^ 1, abort_flag, a.status)) { ok = false; break; }
            const uint32_t sx = smem_u32(kbuf(xb));
            const CodeTile ct = code_tile(ok_, (int64_t)(a.li * a.H + h) * a.T + t0, min(SBM, te - t0), D, a.gq);
            mbar_expect_tx(xfull_bar(xb), (ct.cbulk ? ct.cbytes : 0u) + (ct.sbulk ? ct.sbytes : 0u));
            if (ct.cbulk) bulk_load(sx, ct.codes, ct.cbytes, xfull_bar(xb));
            if (ct.sbulk) bulk_load(sx + S_CODE, ct.scales, ct.sbytes, xfull_bar(xb));
            xissued[xb] = true;
            xissued_phase[xb] = xph[xb];
            xph[xb] ^= 1;
            xb ^= 1;
          }
          for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, a.status)) { ok = false; break; }
            const uint32_t sa = smem_u32(sA + stage * S_A), sb = smem_u32(sB + stage * S_B);
            mbar_expect_tx(full_bar(stage), S_A + D * 128);
            tma_load_3d(sa, &maps.ut[b], full_bar(stage), t0, kb * 64, 0);
            tma_load_3d(sa + 8192, &maps.ut[b], full_bar(stage), t0 + 64, kb * 64, 0);
            tma_load_3d(sb, &maps.mt, full_bar(stage), kb * 64, 0, b * a.H + h);
            issued[stage] = true;
            issued_phase[stage] = ph;
            if (++stage == SSTAGES) { stage = 0; ph ^= 1; }
          }
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
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph[2] = {0, 0};
      const uint32_t idesc = idesc_bf16(D, 1, 0);
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        int b, h, s;
        item_of(a, it, b, h, s);
        const int rT = a.kout[b * a.cstride].rT;
        const int tb = s * a.per, te = min(a.T, tb + a.per);
        const int nk = (rT + 63) / 64;
        for (int t0 = tb; t0 < te && ok; t0 += SBM) {
          if (!mbar_wait(tempty_bar(acc), aph[acc] ^ 1, abort_flag, a.status)) { ok = false; break; }
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
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int rl = q * 32 + lane;
    const int et = threadIdx.x - 64;
    const float rs = (float)(1.0 / sqrt((double)D));
    const float qk_scale = (float)(1.0 / sqrt((double)D));
    int acc = 0, xb = 0, xpar = 0;
    uint32_t aph[2] = {0, 0}, xph[2] = {0, 0};
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      int b, h, s;
      item_of(a, it, b, h, s);
      const CellOut ko = a.kout[b * a.cstride], vo = a.vout[b * a.cstride];
      const int tb = s * a.per, te = min(a.T, tb + a.per);
      // queries of this KV head and the sequence's rotation signs
      epi_sync();
      for (int e = et; e < G * D; e += 32 * EPI_WARPS)
        sQ[(e / D) * 128 + e % D] = a.q[((int64_t)b * a.H * G + (int64_t)h * G) * D + e];
      if (et < D) sSign[et] = hadamard_sign(a.seed + (uint64_t)b, et);
      epi_sync();
      float m_run[GMAX], l_run[GMAX];
#pragma unroll
      for (int g = 0; g < GMAX; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.0f; }
      // rank-space state: ranks r = et and et + 256, every query head
      float ar[2][GMAX];
      // rotated residual state: column d = et % D, the token part et / D, every query head
      float ae[GMAX];
#pragma unroll
      for (int g = 0; g < GMAX; ++g) { ar[0][g] = 0.0f; ar[1][g] = 0.0f; ae[g] = 0.0f; }
      constexpr int TPARTS = 256 / D;          // token parts of the residual accumulation
      const int dcol = et % D, tpart = et / D;

      for (int t0 = tb; t0 < te; t0 += SBM) {
        const int t = t0 + rl;
        const bool valid = t < te;
        const int nrows = min(SBM, te - t0);
        const int64_t row0 = (int64_t)(a.li * a.H + h) * a.T + t0;
        // ---- key row: residual (rotated domain -> de-rotated), backbone, RoPE
        float e[2 * C];
        if (ko.b > 0) {
          if (!epi_all(mbar_wait(xfull_bar(xb), xph[xb], abort_flag, a.status))) { ok = false; break; }
          const CodeTile ct = code_tile(ko, row0, nrows, D, a.gq);
          const uint8_t* stage_in = kbuf(xb);
          const int rowbytes = ko.b * D / 8, ng = D / a.gq;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int s0 = k * (D / 2) + hf * C;
            if (!valid) {
#pragma unroll
              for (int j = 0; j < C; ++j) e[k * C + j] = 0.0f;
              continue;
            }
            const float sc = ct.sbulk ? reinterpret_cast<const float*>(stage_in + S_CODE)[rl * ng + s0 / a.gq]
                                      : ct.scales[rl * ng + s0 / a.gq];
            const int64_t off = (int64_t)rl * rowbytes + s0 * ko.b / 8;
            uint32_t w[C * 8 / 32];
            switch (ko.b) {
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
        if (!epi_all(mbar_wait(tfull_bar(acc), aph[acc], abort_flag, a.status))) { ok = false; break; }
        fence_after();
        {
          const uint32_t tb2 = lane_base + (uint32_t)(acc * D);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            float v[C];
            tmem_ld<C>(tb2 + k * (D / 2) + hf * C, v);
#pragma unroll
            for (int j = 0; j < C; ++j) e[k * C + j] = __fadd_rn(v[j], e[k * C + j]);
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        aph[acc] ^= 1;
        acc ^= 1;
        if (a.cs && valid) {
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
        // ---- scores of the G query heads: this thread's half of the dot product
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          if (g >= G) break;
          float part = 0.0f;
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int j = 0; j < C; ++j) part = fmaf(sQ[g * 128 + k * (D / 2) + hf * C + j], e[k * C + j], part);
          sPart[(g * 128 + rl) * 2 + hf] = part;
        }
        pair_sync(q);
        float sc[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          sc[g] = -INFINITY;
          if (g < G && valid) sc[g] = __fmul_rn(__fadd_rn(sPart[(g * 128 + rl) * 2], sPart[(g * 128 + rl) * 2 + 1]), qk_scale);
        }
        // ---- online softmax over the tile (max, then sum), every thread keeps the state
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          float m = sc[g];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (hf == 0 && lane == 0) sRed[g * 4 + q] = m;
        }
        epi_sync();
        float mnew[GMAX], alpha[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          const float mt = fmaxf(fmaxf(sRed[g * 4 + 0], sRed[g * 4 + 1]), fmaxf(sRed[g * 4 + 2], sRed[g * 4 + 3]));
          mnew[g] = fmaxf(m_run[g], mt);
          alpha[g] = (g < G) ? expf(m_run[g] - mnew[g]) : 0.0f;
          const float p = (g < G && valid) ? expf(sc[g] - mnew[g]) : 0.0f;
          if (hf == 0) sP[rl * GMAX + g] = p;
          float ssum = p;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
          if (hf == 0 && lane == 0) sRed[GMAX * 4 + g * 4 + q] = ssum;
        }
        // ---- stage the value codes of the tile (zeros past the split)
        if (vo.b > 0) {
          const int vrow = vo.b * D / 8;          // a multiple of 8 bytes
          const uint8_t* src = vo.codes + row0 * vrow;
          for (int w8 = et; w8 < 128 * vrow / 8; w8 += 32 * EPI_WARPS) {
            const int r = (w8 * 8) / vrow;
            reinterpret_cast<uint2*>(sVC)[w8] = (r < nrows) ? reinterpret_cast<const uint2*>(src)[w8] : make_uint2(0u, 0u);
          }
          const int ng = D / a.gq;
          for (int i = et; i < 128 * ng; i += 32 * EPI_WARPS)
            sVS[i] = (i / ng < nrows) ? vo.scales[row0 * ng + i] : 0.0f;
        }
        epi_sync();
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          const float tsum = __fadd_rn(__fadd_rn(sRed[GMAX * 4 + g * 4 + 0], sRed[GMAX * 4 + g * 4 + 1]),
                                       __fadd_rn(sRed[GMAX * 4 + g * 4 + 2], sRed[GMAX * 4 + g * 4 + 3]));
          l_run[g] = fmaf(l_run[g], alpha[g], tsum);
          m_run[g] = mnew[g];
        }
        // every value state takes the tile's rescale
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          ar[0][g] = __fmul_rn(ar[0][g], alpha[g]);
          ar[1][g] = __fmul_rn(ar[1][g], alpha[g]);
          ae[g] = __fmul_rn(ae[g], alpha[g]);
        }
        // ---- rotated value residual: this thread's column over its token part
        if (vo.b > 0) {
          const int ng = D / a.gq;
          const int bit = dcol * vo.b, wi = bit >> 5, sh = bit & 31;
          const uint32_t mask = (1u << vo.b) - 1u;
          const int vrow4 = vo.b * D / 32;      // 32-bit words per row
          const float off = (float)(1 << (vo.b - 1));
          const int t_lo = tpart * (128 / TPARTS), t_hi = min(nrows, t_lo + 128 / TPARTS);
          for (int tt = t_lo; tt < t_hi; ++tt) {
            const uint32_t* wr = reinterpret_cast<const uint32_t*>(sVC) + tt * vrow4;
            uint32_t u = wr[wi] >> sh;
            if (sh + vo.b > 32) u |= wr[wi + 1] << (32 - sh);
            const float dq = __fmul_rn(__fsub_rn((float)(u & mask), off), sVS[tt * ng + dcol / a.gq]);
            const float4 p0 = reinterpret_cast<const float4*>(sP + tt * GMAX)[0];
            const float4 p1 = reinterpret_cast<const float4*>(sP + tt * GMAX)[1];
            const float pv[GMAX] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int g = 0; g < GMAX; ++g) ae[g] = fmaf(pv[g], dq, ae[g]);
          }
        }
        // ---- rank-space values: all ranks, the whole tile at once when they
        // fit the staging buffer, else TSUB tokens at a time
        const int tsub = (vo.rT * (SBM + 2) <= RVMAX * UP) ? SBM : TSUB;
        const int up = tsub + 2;     // odd word pitch: rank rows on distinct banks
        for (int ts = 0; ts < nrows; ts += tsub) {
          epi_sync();   // the previous slice's readers are done with sU
          const int nt = min(tsub, nrows - ts);
          for (int w = et; w < vo.rT * (tsub / 8); w += 32 * EPI_WARPS) {
            const int r = w / (tsub / 8), tq = (w % (tsub / 8)) * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (tq < nt) {
              const uint16_t* src = vo.ut + (int64_t)r * vo.t_pitch + t0 + ts + tq;
              if (tq + 8 <= nt && ((reinterpret_cast<uintptr_t>(src) & 15u) == 0)) {
                v = *reinterpret_cast<const uint4*>(src);
              } else {
                uint16_t tmp[8];
#pragma unroll
                for (int j2 = 0; j2 < 8; ++j2) tmp[j2] = (tq + j2 < nt) ? src[j2] : (uint16_t)0;
                v = make_uint4(tmp[0] | (uint32_t)tmp[1] << 16, tmp[2] | (uint32_t)tmp[3] << 16,
                               tmp[4] | (uint32_t)tmp[5] << 16, tmp[6] | (uint32_t)tmp[7] << 16);
              }
            }
            uint32_t* dst = reinterpret_cast<uint32_t*>(sU + r * up + tq);
            dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
          }
          epi_sync();
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int r = et + 256 * i;
            if (r >= vo.rT) continue;
            for (int tt = 0; tt < nt; ++tt) {
              const float u = bf16f(sU[r * up + tt]);
              const float4 p0 = reinterpret_cast<const float4*>(sP + (ts + tt) * GMAX)[0];
              const float4 p1 = reinterpret_cast<const float4*>(sP + (ts + tt) * GMAX)[1];
              const float pv[GMAX] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
              for (int g = 0; g < GMAX; ++g) ar[i][g] = fmaf(pv[g], u, ar[i][g]);
            }
          }
        }
        epi_sync();   // sP, sRed and the staged values are rewritten by the next tile
      }
      if (!ok) break;
      // ---- this split's softmax state
      float* base = a.part + (((int64_t)b * a.H + h) * a.nsplit + s) * G * (2 + a.rpv + D);
      const int stride = 2 + a.rpv + D;
      if (et < G) {
        base[et * stride + 0] = m_run[et];
        base[et * stride + 1] = l_run[et];
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = et + 256 * i;
        if (r < a.rpv)
#pragma unroll
          for (int g = 0; g < GMAX; ++g)
            if (g < G) base[g * stride + 2 + r] = (r < vo.rT) ? ar[i][g] : 0.0f;
      }
      // the residual state's token parts, added in a fixed order
      epi_sync();
#pragma unroll
      for (int g = 0; g < GMAX; ++g) sEred[(tpart * GMAX + g) * 128 + dcol] = ae[g];
      epi_sync();
      for (int e2 = et; e2 < G * D; e2 += 32 * EPI_WARPS) {
        const int g = e2 / D, d = e2 % D;
        float v = sEred[g * 128 + d];
        for (int tp = 1; tp < TPARTS; ++tp) v = __fadd_rn(v, sEred[(tp * GMAX + g) * 128 + d]);
        base[g * stride + 2 + a.rpv + d] = v;
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

// M^ = bf16(G^_lh U_d^T) of layer li for the key and value cells of every
// sequence: keys transposed and zero-padded for the MMA ([B*H][D][rpk] bf16),
// values row-major for the merge ([B*H][rpv][D] fp32). Products of bf16 values
// summed in fp64 and rounded once, as decompression forms M^.
template <int D>
__global__ void __launch_bounds__(D) k_dec_m(const CellOut* __restrict__ kout, const CellOut* __restrict__ vout,
                                             int cstride, int H, int li, uint16_t* __restrict__ mtk, int rpk,
                                             float* __restrict__ mv, int rpv) {
  const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z >> 1, kind = blockIdx.z & 1;
  const CellOut o = kind == 0 ? kout[b * cstride] : vout[b * cstride];
  const int rp = kind == 0 ? rpk : rpv;
  if (r >= rp) return;
  const int d = threadIdx.x;
  __shared__ double gs[D];
  const bool live = r < o.rT;
  if (live && d < o.rd) gs[d] = (double)bf16f(o.core[((int64_t)(li * H + h) * o.rT + r) * o.rd + d]);
  __syncthreads();
  double m = 0.0;
  if (live)
    for (int j = 0; j < o.rd; ++j) m += gs[j] * (double)bf16f(o.ud[d * o.rd + j]);
  const uint16_t mb = live ? bf16_bits_from_f64(m) : (uint16_t)0;
  if (kind == 0) mtk[((int64_t)(b * H + h) * D + d) * rpk + r] = mb;
  else mv[((int64_t)(b * H + h) * rpv + r) * D + d] = bf16f(mb);
}

// Splits + dense tail -> output: one block per (KV head, sequence), one query
// head at a time. out = (a_rank M^_V + R^T a_res + a_tail) / L.
template <int D>
__global__ void __launch_bounds__(128) k_dec_merge(Args a, const CellOut* __restrict__ vout,
                                                   const float* __restrict__ mv, const uint16_t* __restrict__ tk,
                                                   const uint16_t* __restrict__ tv, int ntail, float* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const CellOut vo = vout[b * a.cstride];
  const int stride = 2 + a.rpv + D, G = a.G;
  __shared__ float sq[D], sres[D], srank[RVMAX], sw[64], stl[1024];
  __shared__ float sred[4];
  __shared__ float sM, sL;
  const float rs = (float)(1.0 / sqrt((double)D));
  const float qk_scale = rs;
  for (int g = 0; g < G; ++g) {
    const float* base = a.part + ((int64_t)b * a.H + h) * a.nsplit * G * stride;
    const float* qv = a.q + ((int64_t)b * a.H * G + (int64_t)h * G + g) * D;
    for (int d = tid; d < D; d += 128) sq[d] = qv[d];
    __syncthreads();
    // tail scores (fp32, fixed order)
    for (int j = tid; j < ntail; j += 128) {
      const uint16_t* kr = tk + (((int64_t)b * a.H + h) * ntail + j) * D;
      float s = 0.0f;
      for (int d = 0; d < D; ++d) s = fmaf(sq[d], bf16f(kr[d]), s);
      stl[j] = __fmul_rn(s, qk_scale);
    }
    __syncthreads();
    if (tid == 0) {
      float M = -INFINITY;
      for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, base[(s * G + g) * stride]);
      for (int j = 0; j < ntail; ++j) M = fmaxf(M, stl[j]);
      float L = 0.0f;
      for (int s = 0; s < a.nsplit; ++s) {
        const float w = expf(base[(s * G + g) * stride] - M);
        sw[s] = w;
        L = fmaf(base[(s * G + g) * stride + 1], w, L);
      }
      for (int j = 0; j < ntail; ++j) {
        stl[j] = expf(stl[j] - M);
        L = __fadd_rn(L, stl[j]);
      }
      sM = M;
      sL = L;
    }
    __syncthreads();
    for (int r = tid; r < a.rpv; r += 128) {
      float v = 0.0f;
      for (int s = 0; s < a.nsplit; ++s) v = fmaf(sw[s], base[(s * G + g) * stride + 2 + r], v);
      srank[r] = (r < vo.rT) ? v : 0.0f;
    }
    for (int d = tid; d < D; d += 128) {
      float v = 0.0f;
      for (int s = 0; s < a.nsplit; ++s) v = fmaf(sw[s], base[(s * G + g) * stride + 2 + a.rpv + d], v);
      sres[d] = v;
    }
    __syncthreads();
    // inverse rotation of the accumulated residual: natural-order FWHT
    // (stages 1, 2, ..., D/2), then * fl32(1/sqrt(D)) and the signs
    for (int hh = 1; hh < D; hh <<= 1) {
      float x0 = 0.0f, x1 = 0.0f;
      int i0 = -1;
      if (tid < D / 2) {
        const int blk = tid / hh, off = tid % hh;
        i0 = blk * 2 * hh + off;
        x0 = sres[i0];
        x1 = sres[i0 + hh];
      }
      __syncthreads();
      if (i0 >= 0) {
        sres[i0] = __fadd_rn(x0, x1);
        sres[i0 + hh] = __fsub_rn(x0, x1);
      }
      __syncthreads();
    }
    for (int d = tid; d < D; d += 128) {
      const float e = __fmul_rn(__fmul_rn(sres[d], rs), hadamard_sign(a.seed + (uint64_t)b, d));
      float v = 0.0f;
      if (vo.b > 0) v = e;
      float bb = 0.0f;
      const float* mrow = mv + (int64_t)(b * a.H + h) * a.rpv * D + d;
      for (int r = 0; r < vo.rT; ++r) bb = fmaf(srank[r], mrow[(int64_t)r * D], bb);
      float tl = 0.0f;
      for (int j = 0; j < ntail; ++j) tl = fmaf(stl[j], bf16f(tv[(((int64_t)b * a.H + h) * ntail + j) * D + d]), tl);
      out[((int64_t)b * a.H * G + (int64_t)h * G + g) * D + d] = __fdiv_rn(__fadd_rn(__fadd_rn(bb, v), tl), sL);
    }
    __syncthreads();
  }
}

}  // namespace dec

static int dec_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

jolt_status launch_decode_attention(const DecodeCall& c, cudaStream_t s) {
  using namespace dec;
  const int B = c.B, H = c.H, D = c.D, T = c.T, G = c.G;
  // split the token range so that about two work items land on each SM
  const int ntile = (T + SBM - 1) / SBM;
  int nsplit = std::max(1, std::min(ntile, (2 * dec_sms() + B * H - 1) / (B * H)));
  const int per = ((ntile + nsplit - 1) / nsplit) * SBM;
  nsplit = (T + per - 1) / per;
  if (nsplit > 64) { set_error("decode attention: %d splits exceed 64", nsplit); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  dec::Args a{};
  a.B = B; a.H = H; a.T = T; a.G = G; a.gq = c.gq; a.li = c.li; a.nsplit = nsplit; a.per = per;
  a.kout = c.kout; a.vout = c.vout; a.cstride = c.cstride; a.cs = c.cs; a.seed = c.seed; a.q = c.q; a.part = c.part; a.rpv = c.rpv;
  a.status = c.status;
  if ((int64_t)B * H * nsplit * G * (2 + c.rpv + D) > c.part_len) { set_error("decode attention: state buffer too small"); return JOLT_ERR_CUDA; }
  dim3 gm(std::max(c.rpk, c.rpv), H, 2 * B);
  if (D == 128) k_dec_m<128><<<gm, 128, 0, s>>>(c.kout, c.vout, c.cstride, H, c.li, c.mtk, c.rpk, c.mv, c.rpv);
  else k_dec_m<64><<<gm, 64, 0, s>>>(c.kout, c.vout, c.cstride, H, c.li, c.mtk, c.rpk, c.mv, c.rpv);
  JOLT_LAUNCHED();
  dec::Maps m;
  JOLT_TRY(map_3d_box(&m.mt, c.mtk, B * H, D, c.rpk, c.rpk, 64, D));
  for (int b = 0; b < B; ++b)
    JOLT_TRY(map_3d_box(&m.ut[b], c.ut[b], 1, std::max(1, c.rt_k[b]), c.tpitch[b], c.tpitch[b], 64, 64));
  for (int b = B; b < BMAX; ++b) m.ut[b] = m.ut[0];
  const int items = B * H * nsplit;
  const int grid = std::min(items, dec_sms());
#define JOLT_DEC_LAUNCH(DD)                                                                                   \
  do {                                                                                                        \
    static bool attr = false;                                                                                 \
    if (!attr) {                                                                                              \
      JOLT_CUDA_TRY(cudaFuncSetAttribute(k_dec_attn<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DEC)); \
      attr = true;                                                                                            \
    }                                                                                                         \
    k_dec_attn<DD><<<grid, STHREADS, SMEM_DEC, s>>>(m, a);                                                     \
  } while (0)
  if (D == 128) JOLT_DEC_LAUNCH(128);
  else JOLT_DEC_LAUNCH(64);
#undef JOLT_DEC_LAUNCH
  JOLT_LAUNCHED();
  dim3 gg(H, B);
  if (D == 128) k_dec_merge<128><<<gg, 128, 0, s>>>(a, c.vout, c.mv, c.tail_k, c.tail_v, c.ntail, c.out);
  else k_dec_merge<64><<<gg, 128, 0, s>>>(a, c.vout, c.mv, c.tail_k, c.tail_v, c.ntail, c.out);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
