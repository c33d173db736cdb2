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
// The rank-space product runs on tcgen05 too: per tile, U_T^V^T (128 ranks x
// 128 tokens per block, TMA) times P (128 tokens x 16: the bf16 high and low
// parts of p for up to 8 query heads, so p keeps about 16 bits) into TMEM;
// the epilogue adds each tile's result into its fp32 state with the online-
// softmax rescale one tile later.
//
// Warp roles as in the stream kernel: warp 0 issues TMA loads of U_T^ / M^
// slices, U_T^V blocks and bulk copies of the key codes, warp 1 issues the
// MMAs (key tile i, then the values of tile i-1), warps 2..9 are the
// epilogue (scores, online softmax, value accumulation).
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
constexpr int OFF_PB = OFF_KCODE + 2 * (S_CODE + S_SCALE);           // 2 x P^T [16][128] bf16, swizzled (1 KB aligned)
constexpr int PB_BYTES = 16 * 128 * 2;
constexpr int OFF_VBUF = OFF_PB + 2 * PB_BYTES;                      // 2 x (codes + scales) of values
constexpr int OFF_Q = OFF_VBUF + 2 * (S_CODE + S_SCALE);             // [GMAX][128] fp32
constexpr int OFF_P = OFF_Q + GMAX * 128 * 4;                        // [128 t][GMAX] fp32
constexpr int OFF_PART = OFF_P + GMAX * 128 * 4;                     // [GMAX][128][2] fp32
constexpr int OFF_RED = OFF_PART + GMAX * 128 * 2 * 4;               // [2][GMAX][4] fp32
constexpr int OFF_SIGN = OFF_RED + 2 * GMAX * 4 * 4;                 // [128] fp32
constexpr int OFF_ERED = OFF_SIGN + 128 * 4;                         // [4][GMAX][128] fp32 (item end)
constexpr int OFF_BAR = OFF_ERED + 4 * GMAX * 128 * 4;
constexpr int SMEM_DEC = OFF_BAR + 256 + 1024;
static_assert(SMEM_DEC <= 227 * 1024, "decode attention shared memory");
static_assert(OFF_PB % 1024 == 0, "P^T operand alignment");
static_assert(S_A == 16384 && S_B == 16384, "a value block fills the A and B slots of a stage");

struct Maps {
  CUtensorMap mt;          // M^_K^T workspace [B*H][D][rpk] bf16, box {64 r, D}
  CUtensorMap ut[BMAX];    // U_T^ of each sequence's key cell [rT][t_pitch], box {64 t, 64 r}
  CUtensorMap uv[BMAX];    // U_T^ of each sequence's value cell [rT][T], box {64 t, 128 r}
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

// GT: query heads per KV head the kernel is compiled for (G <= GT; heads
// g >= G carry zero probability)
template <int D, int GT>
__global__ void __launch_bounds__(STHREADS, 1) k_dec_attn(const __grid_constant__ Maps maps, Args a) {
  constexpr int C = D / 4;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem + OFF_RING;
  uint8_t* sB = sA + SSTAGES * S_A;
  uint8_t* sK = smem + OFF_KCODE;
  uint8_t* sPB = smem + OFF_PB;
  float* sQ = reinterpret_cast<float*>(smem + OFF_Q);
  float* sP = reinterpret_cast<float*>(smem + OFF_P);
  float* sPart = reinterpret_cast<float*>(smem + OFF_PART);
  float* sRed = reinterpret_cast<float*>(smem + OFF_RED);
  float* sSign = reinterpret_cast<float*>(smem + OFF_SIGN);
  float* sEred = reinterpret_cast<float*>(smem + OFF_ERED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SSTAGES + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (SSTAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 2 + b); };
  auto xfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 4 + b); };
  auto xempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 6 + b); };
  auto pfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 8 + b); };    // P^T of a tile written
  auto vfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 10 + b); };   // its value product done
  auto vcfull_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 12 + b); };  // value codes staged
  auto vcempty_bar = [&](int b) { return bar0 + 8u * (2 * SSTAGES + 14 + b); };
  auto kbuf = [&](int b) { return sK + b * (S_CODE + S_SCALE); };
  auto vbuf = [&](int b) { return smem + OFF_VBUF + b * (S_CODE + S_SCALE); };
  // TMEM: two key accumulators (D columns each), then two regions of D
  // columns, by tile parity: the residual exchange of the tile's keys, then
  // the tile's value product (16 columns per block of 128 ranks)
  constexpr int NCOLS = (4 * D <= 256) ? 256 : 512;
  auto xreg = [&](int par) { return (uint32_t)(2 * D + par * D); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SSTAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), EPI_WARPS);
      mbar_init(xfull_bar(b), 1);
      mbar_init(xempty_bar(b), EPI_WARPS);
      mbar_init(pfull_bar(b), EPI_WARPS);
      mbar_init(vfull_bar(b), 1);
      mbar_init(vcfull_bar(b), 1);
      mbar_init(vcempty_bar(b), EPI_WARPS);
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
    // per tile i of an item: its key codes, its key stages, then the value
    // blocks of tile i-1 (and after the last tile, that tile's)
    if (lane == 0) {
      int stage = 0, xb = 0, vb = 0;
      uint32_t ph = 0, xph[2] = {0, 0}, vcph[2] = {0, 0};
      uint32_t issued_phase[SSTAGES], xissued_phase[2], vissued_phase[2];
      bool issued[SSTAGES], xissued[2] = {false, false}, vissued[2] = {false, false};
      for (int s = 0; s < SSTAGES; ++s) issued[s] = false;
      bool ok = true;
      auto next_stage = [&]() -> bool {
        if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, a.status)) return false;
        return true;
      };
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        int b, h, s;
        item_of(a, it, b, h, s);
        const CellOut ok_ = a.kout[b * a.cstride];
        const CellOut vo_ = a.vout[b * a.cstride];
        const int rv = vo_.rT;
        const int tb = s * a.per, te = min(a.T, tb + a.per);
        const int ntile = (te - tb + SBM - 1) / SBM;
        const int nk = (ok_.rT + 63) / 64, nv = (rv + 127) / 128;
        for (int i = 0; i <= ntile && ok; ++i) {
          if (i < ntile) {
            const int t0 = tb + i * SBM;
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
            if (vo_.b > 0) {
              // the tile's value codes and scales (read by the epilogue's residual sum)
              if (!mbar_wait(vcempty_bar(vb), vcph[vb] ^ 1, abort_flag, a.status)) { ok = false; break; }
              const uint32_t sv = smem_u32(vbuf(vb));
              const CodeTile ct = code_tile(vo_, (int64_t)(a.li * a.H + h) * a.T + t0, min(SBM, te - t0), D, a.gq);
              mbar_expect_tx(vcfull_bar(vb), (ct.cbulk ? ct.cbytes : 0u) + (ct.sbulk ? ct.sbytes : 0u));
              if (ct.cbulk) bulk_load(sv, ct.codes, ct.cbytes, vcfull_bar(vb));
              if (ct.sbulk) bulk_load(sv + S_CODE, ct.scales, ct.sbytes, vcfull_bar(vb));
              vissued[vb] = true;
              vissued_phase[vb] = vcph[vb];
              vcph[vb] ^= 1;
              vb ^= 1;
            }
            for (int kb = 0; kb < nk; ++kb) {
              if (!next_stage()) { ok = false; break; }
              const uint32_t sa = smem_u32(sA + stage * S_A), sb = smem_u32(sB + stage * S_B);
              mbar_expect_tx(full_bar(stage), S_A + D * 128);
              tma_load_3d(sa, &maps.ut[b], full_bar(stage), t0, kb * 64, 0);
              tma_load_3d(sa + 8192, &maps.ut[b], full_bar(stage), t0 + 64, kb * 64, 0);
              tma_load_3d(sb, &maps.mt, full_bar(stage), kb * 64, 0, b * a.H + h);
              issued[stage] = true;
              issued_phase[stage] = ph;
              if (++stage == SSTAGES) { stage = 0; ph ^= 1; }
            }
            if (!ok) break;
          }
          if (i >= 1) {
            // U_T^V^T block j of tile i-1: ranks 128j .., two boxes of 64 tokens
            // (16 KB each: into the stage's A and B slots)
            const int t0 = tb + (i - 1) * SBM;
            for (int j = 0; j < nv; ++j) {
              if (!next_stage()) { ok = false; break; }
              const uint32_t sa = smem_u32(sA + stage * S_A), sb = smem_u32(sB + stage * S_B);
              mbar_expect_tx(full_bar(stage), 2 * 16384);
              tma_load_3d(sa, &maps.uv[b], full_bar(stage), t0, 128 * j, 0);
              tma_load_3d(sb, &maps.uv[b], full_bar(stage), t0 + 64, 128 * j, 0);
              issued[stage] = true;
              issued_phase[stage] = ph;
              if (++stage == SSTAGES) { stage = 0; ph ^= 1; }
            }
          }
        }
      }
      for (int s = 0; s < SSTAGES; ++s)
        if (issued[s]) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try(full_bar(s), issued_phase[s]) && now_ns() - t0 < WAIT_NS) {}
        }
      for (int b = 0; b < 2; ++b) {
        if (xissued[b]) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try(xfull_bar(b), xissued_phase[b]) && now_ns() - t0 < WAIT_NS) {}
        }
        if (vissued[b]) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try(vcfull_bar(b), vissued_phase[b]) && now_ns() - t0 < WAIT_NS) {}
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph[2] = {0, 0}, pph[2] = {0, 0};
      const uint32_t idesc = idesc_bf16(D, 1, 0);
      const uint32_t idesc_v = idesc_bf16(16, 0, 0);
      bool ok = true;
      int tc = 0;                 // tiles of this CTA so far (the parity of P^T and the TMEM regions)
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        int b, h, s;
        item_of(a, it, b, h, s);
        const int rT = a.kout[b * a.cstride].rT;
        const int rv = a.vout[b * a.cstride].rT;
        const int tb = s * a.per, te = min(a.T, tb + a.per);
        const int ntile = (te - tb + SBM - 1) / SBM;
        const int nk = (rT + 63) / 64, nv = (rv + 127) / 128;
        for (int i = 0; i <= ntile && ok; ++i) {
          if (i < ntile) {
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
          if (i >= 1) {
            const int par = (tc + i - 1) & 1;
            if (!mbar_wait(pfull_bar(par), pph[par], abort_flag, a.status)) { ok = false; break; }
            pph[par] ^= 1;
            fence_after();
            const uint32_t pb = smem_u32(sPB + par * PB_BYTES);
            for (int j = 0; j < nv; ++j) {
              if (!mbar_wait(full_bar(stage), ph, abort_flag, a.status)) { ok = false; break; }
              fence_after();
              const uint32_t sa = smem_u32(sA + stage * S_A), sb = smem_u32(sB + stage * S_B);
              const uint32_t dv = tmem + xreg(par) + (uint32_t)(16 * j);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_bf16(dv, sdesc((kk < 4 ? sa : sb) + (kk & 3) * 32, 16, 1024),
                         sdesc(pb + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024), idesc_v, kk > 0 ? 1u : 0u);
              mma_commit(empty_bar(stage));
              if (++stage == SSTAGES) { stage = 0; ph ^= 1; }
            }
            if (!ok) break;
            mma_commit(vfull_bar(par));
          }
        }
        tc += ntile;
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
    int acc = 0, xb = 0, vb = 0, tc = 0;
    uint32_t aph[2] = {0, 0}, xph[2] = {0, 0}, vph[2] = {0, 0}, vcph[2] = {0, 0};
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    bool ok = true;
    // P^T rows of heads the kernel does not hold (g >= GT) stay zero
    for (int i2 = et; i2 < 2 * PB_BYTES / 4; i2 += 32 * EPI_WARPS) reinterpret_cast<uint32_t*>(sPB)[i2] = 0u;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      int b, h, s;
      item_of(a, it, b, h, s);
      const CellOut ko = a.kout[b * a.cstride], vo = a.vout[b * a.cstride];
      const int tb = s * a.per, te = min(a.T, tb + a.per);
      const int ntile = (te - tb + SBM - 1) / SBM;
      const int nv = (vo.rT + 127) / 128;
      // queries of this KV head and the sequence's rotation signs
      epi_sync();
      for (int e = et; e < G * D; e += 32 * EPI_WARPS)
        sQ[(e / D) * 128 + e % D] = a.q[((int64_t)b * a.H * G + (int64_t)h * G) * D + e];
      if (et < D) sSign[et] = hadamard_sign(a.seed + (uint64_t)b, et);
      epi_sync();
      float m_run[GT], l_run[GT], alpha_prev[GT];
#pragma unroll
      for (int g = 0; g < GT; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.0f; alpha_prev[g] = 0.0f; }
      // rank-space state: ranks 128 j + rl of the blocks j = hf and hf + 2, every query head
      float ar[2][GT];
      // rotated residual state: column d = et % D, the token part et / D, every query head
      float ae[GT];
#pragma unroll
      for (int g = 0; g < GT; ++g) { ar[0][g] = 0.0f; ar[1][g] = 0.0f; ae[g] = 0.0f; }
      constexpr int TPARTS = 256 / D;          // token parts of the residual accumulation
      const int dcol = et % D, tpart = et / D;
      // the value product of tile (parity par) into the rank state, with the
      // rescale of that tile (alpha_prev)
      auto take_values = [&](int par) -> bool {
        if (!epi_all(mbar_wait(vfull_bar(par), vph[par], abort_flag, a.status))) return false;
        vph[par] ^= 1;
        fence_after();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j = hf + 2 * i;
          if (j >= nv) continue;             // uniform over the warp
          float v[16];
          tmem_ld16(lane_base + xreg(par) + (uint32_t)(16 * j), v);
#pragma unroll
          for (int g = 0; g < GT; ++g)
            ar[i][g] = __fadd_rn(__fmul_rn(ar[i][g], alpha_prev[g]), __fadd_rn(v[g], v[GMAX + g]));
        }
        fence_before();
        return true;
      };

      for (int i = 0; i < ntile; ++i) {
        const int t0 = tb + i * SBM;
        const int par = (tc + i) & 1;
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
          fwht_pair<C>(e, lane_base, xreg(par), hf, q);
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
        // ---- scores of the G query heads: this thread's half of the dot
        // product, the heads' sums side by side
        {
          float part[GT];
#pragma unroll
          for (int g = 0; g < GT; ++g) part[g] = 0.0f;
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int j = 0; j < C; ++j)
#pragma unroll
              for (int g = 0; g < GT; ++g) part[g] = fmaf(sQ[g * 128 + k * (D / 2) + hf * C + j], e[k * C + j], part[g]);
#pragma unroll
          for (int g = 0; g < GT; ++g)
            if (g < G) sPart[(g * 128 + rl) * 2 + hf] = part[g];
        }
        pair_sync(q);
        float sc[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          sc[g] = -INFINITY;
          if (g < G && valid) sc[g] = __fmul_rn(__fadd_rn(sPart[(g * 128 + rl) * 2], sPart[(g * 128 + rl) * 2 + 1]), qk_scale);
        }
        // ---- online softmax over the tile (max, then sum), every thread keeps the state
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          float m = sc[g];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (hf == 0 && lane == 0) sRed[g * 4 + q] = m;
        }
        epi_sync();
        float mnew[GT], alpha[GT];
        uint16_t* pt = reinterpret_cast<uint16_t*>(sPB + par * PB_BYTES);
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float mt = fmaxf(fmaxf(sRed[g * 4 + 0], sRed[g * 4 + 1]), fmaxf(sRed[g * 4 + 2], sRed[g * 4 + 3]));
          mnew[g] = fmaxf(m_run[g], mt);
          alpha[g] = (g < G) ? expf(m_run[g] - mnew[g]) : 0.0f;
          const float p = (g < G && valid) ? expf(sc[g] - mnew[g]) : 0.0f;
          if (hf == 0) sP[rl * GT + g] = p;
          // P^T for the value product: row n = g holds bf16(p), row 8 + g the
          // bf16 of the remainder; 128-byte swizzled K-major rows of 64 tokens
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(p, __bfloat162float(hi)));
          const int n = hf ? GMAX + g : g;
          const int byte = (rl >> 6) * 2048 + n * 128 + ((((rl & 63) >> 3) ^ (n & 7)) << 4) + (rl & 7) * 2;
          pt[byte >> 1] = hf ? __bfloat16_as_ushort(lo) : __bfloat16_as_ushort(hi);
          float ssum = p;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
          if (hf == 0 && lane == 0) sRed[GMAX * 4 + g * 4 + q] = ssum;
        }
        // the tile's P^T is complete in this warp: publish it to the tensor cores
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull_bar(par));
        epi_sync();
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float tsum = __fadd_rn(__fadd_rn(sRed[GMAX * 4 + g * 4 + 0], sRed[GMAX * 4 + g * 4 + 1]),
                                       __fadd_rn(sRed[GMAX * 4 + g * 4 + 2], sRed[GMAX * 4 + g * 4 + 3]));
          l_run[g] = fmaf(l_run[g], alpha[g], tsum);
          m_run[g] = mnew[g];
        }
#pragma unroll
        for (int g = 0; g < GT; ++g) ae[g] = __fmul_rn(ae[g], alpha[g]);
        // ---- rotated value residual: this thread's column over its token part,
        // from the staged codes (or, not staged, from global memory)
        if (vo.b > 0) {
          if (!epi_all(mbar_wait(vcfull_bar(vb), vcph[vb], abort_flag, a.status))) { ok = false; break; }
          const CodeTile vct = code_tile(vo, row0, nrows, D, a.gq);
          const uint8_t* sVC = vct.cbulk ? vbuf(vb) : vct.codes;
          const float* sVS = vct.sbulk ? reinterpret_cast<const float*>(vbuf(vb) + S_CODE) : vct.scales;
          const int ng = D / a.gq;
          const int bit = dcol * vo.b, wi = bit >> 5, sh = bit & 31;
          const uint32_t mask = (1u << vo.b) - 1u;
          const int vrow4 = vo.b * D / 32;      // 32-bit words per row
          const float off = (float)(1 << (vo.b - 1));
          const int t_lo = tpart * (128 / TPARTS), t_hi = min(nrows, t_lo + 128 / TPARTS);
#pragma unroll 4
          for (int tt = t_lo; tt < t_hi; ++tt) {
            const uint32_t* wr = reinterpret_cast<const uint32_t*>(sVC) + tt * vrow4;
            uint32_t u = wr[wi] >> sh;
            if (sh + vo.b > 32) u |= wr[wi + 1] << (32 - sh);
            const float dq = __fmul_rn(__fsub_rn((float)(u & mask), off), sVS[tt * ng + dcol / a.gq]);
            float pv[GT];
            if constexpr (GT == 8) {
              const float4 p0 = reinterpret_cast<const float4*>(sP + tt * GT)[0];
              const float4 p1 = reinterpret_cast<const float4*>(sP + tt * GT)[1];
              pv[0] = p0.x; pv[1] = p0.y; pv[2] = p0.z; pv[3] = p0.w; pv[4] = p1.x; pv[5] = p1.y; pv[6] = p1.z; pv[7] = p1.w;
            } else if constexpr (GT == 4) {
              const float4 p0 = reinterpret_cast<const float4*>(sP + tt * GT)[0];
              pv[0] = p0.x; pv[1] = p0.y; pv[2] = p0.z; pv[3] = p0.w;
            } else {
#pragma unroll
              for (int g = 0; g < GT; ++g) pv[g] = sP[tt * GT + g];
            }
#pragma unroll
            for (int g = 0; g < GT; ++g) ae[g] = fmaf(pv[g], dq, ae[g]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(vcempty_bar(vb));
          vcph[vb] ^= 1;
          vb ^= 1;
        }
        // ---- the previous tile's value product (its region is rewritten two tiles on)
        if (i >= 1 && !take_values((tc + i - 1) & 1)) { ok = false; break; }
#pragma unroll
        for (int g = 0; g < GT; ++g) alpha_prev[g] = alpha[g];
        epi_sync();   // sP, sRed and the staged values are rewritten by the next tile
      }
      if (!ok) break;
      if (ntile > 0 && !take_values((tc + ntile - 1) & 1)) { ok = false; break; }
      tc += ntile;
      // ---- this split's softmax state
      float* base = a.part + (((int64_t)b * a.H + h) * a.nsplit + s) * G * (2 + a.rpv + D);
      const int stride = 2 + a.rpv + D;
      if (et < G) {
        base[et * stride + 0] = m_run[et];
        base[et * stride + 1] = l_run[et];
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = 128 * (hf + 2 * i) + rl;
        if (r < a.rpv)
#pragma unroll
          for (int g = 0; g < GT; ++g)
            if (g < G) base[g * stride + 2 + r] = (r < vo.rT) ? ar[i][g] : 0.0f;
      }
      // the residual state's token parts, added in a fixed order
      epi_sync();
#pragma unroll
      for (int g = 0; g < GT; ++g) sEred[(tpart * GMAX + g) * 128 + dcol] = ae[g];
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
  // value factors: T columns (tokens past T read as zeros), rT rows (ranks
  // past rT read as zeros), boxes of 64 tokens x 128 ranks
  for (int b = 0; b < B; ++b)
    JOLT_TRY(map_3d_box(&m.uv[b], c.uv[b], 1, std::max(1, c.rt_v[b]), T, c.tpitch_v[b], 64, 128));
  for (int b = B; b < BMAX; ++b) { m.ut[b] = m.ut[0]; m.uv[b] = m.uv[0]; }
  const int items = B * H * nsplit;
  const int grid = std::min(items, dec_sms());
#define JOLT_DEC_LAUNCH(DD, GG)                                                                                   \
  do {                                                                                                            \
    static bool attr = false;                                                                                     \
    if (!attr) {                                                                                                  \
      JOLT_CUDA_TRY(cudaFuncSetAttribute(k_dec_attn<DD, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DEC)); \
      attr = true;                                                                                                \
    }                                                                                                             \
    k_dec_attn<DD, GG><<<grid, STHREADS, SMEM_DEC, s>>>(m, a);                                                     \
  } while (0)
  const int gt = (G <= 1) ? 1 : (G <= 2) ? 2 : (G <= 4) ? 4 : 8;
  if (D == 128) {
    if (gt == 1) JOLT_DEC_LAUNCH(128, 1);
    else if (gt == 2) JOLT_DEC_LAUNCH(128, 2);
    else if (gt == 4) JOLT_DEC_LAUNCH(128, 4);
    else JOLT_DEC_LAUNCH(128, 8);
  } else {
    if (gt == 1) JOLT_DEC_LAUNCH(64, 1);
    else if (gt == 2) JOLT_DEC_LAUNCH(64, 2);
    else if (gt == 4) JOLT_DEC_LAUNCH(64, 4);
    else JOLT_DEC_LAUNCH(64, 8);
  }
#undef JOLT_DEC_LAUNCH
  JOLT_LAUNCHED();
  dim3 gg(H, B);
  if (D == 128) k_dec_merge<128><<<gg, 128, 0, s>>>(a, c.vout, c.mv, c.tail_k, c.tail_v, c.ntail, c.out);
  else k_dec_merge<64><<<gg, 128, 0, s>>>(a, c.vout, c.mv, c.tail_k, c.tail_v, c.ntail, c.out);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
