// Rate-distortion tables and the Lagrangian allocator on the device.
//
// "A JoLT for the KV Cache", Section 3:
//  * Eq. (1): s(r_T, r_d, b) = (|g| n_h r_T r_d + T r_T + d_h r_d) c
//             + [b>0] (b + 32/g_q)/8 |g| n_h T d_h, c = 2 (bf16);
//  * Eq. (2): e(r_T, r_d, b) = eps^2(b) tau(r_T, r_d), tau = discarded
//             token-mode + feature-mode mass of the unprojected spectra,
//             divided by ||X||^2;
//  * Eqs. (3)-(4): min sum e s.t. sum s <= B through L(lambda) = sum(e + lambda s),
//             every cell minimised independently (here by exhaustive, segmented
//             argmin over the grid), lambda found by geometric bisection that
//             stops within the tolerance of B or after max_iters.
//  * eps^2(b): the fraction of a Gaussian's energy the b-bit rotated quantizer
//             fails to recover, calibrated once on a Gaussian round trip.
#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {

// ------------------------------------------------------- eps^2 calibration --
constexpr int CALIB_SAMPLES = 1 << 20;

template <int G>
__global__ void __launch_bounds__(256) k_eps2(int nb, int4 bits_lo, int4 bits_hi, double* partial) {
  const int grp = blockIdx.x * blockDim.x + threadIdx.x;     // one group of G samples
  const int ngrp = CALIB_SAMPLES / G;
  int bl[8] = {bits_lo.x, bits_lo.y, bits_lo.z, bits_lo.w, bits_hi.x, bits_hi.y, bits_hi.z, bits_hi.w};
  double err[8], en = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) err[i] = 0.0;
  if (grp < ngrp) {
    float x[G];
#pragma unroll 1
    for (int m = 0; m < G / 4; ++m) {
      u4 w = philox_at(0ull, STREAM_CALIB, (uint32_t)(grp * (G / 4) + m));
      double u0 = ((double)w.x + 0.5) * 0x1p-32, u1 = ((double)w.y + 0.5) * 0x1p-32;
      double u2 = ((double)w.z + 0.5) * 0x1p-32, u3 = ((double)w.w + 0.5) * 0x1p-32;
      double r0 = sqrt(-2.0 * log(u0)), r1 = sqrt(-2.0 * log(u2));
      double t0 = (2.0 * 3.141592653589793) * u1, t1 = (2.0 * 3.141592653589793) * u3;
      x[4 * m + 0] = (float)(r0 * cos(t0));
      x[4 * m + 1] = (float)(r0 * sin(t0));
      x[4 * m + 2] = (float)(r1 * cos(t1));
      x[4 * m + 3] = (float)(r1 * sin(t1));
    }
    float a = 0.0f;
    for (int j = 0; j < G; ++j) {
      a = fmaxf(a, fabsf(x[j]));
      en += (double)x[j] * (double)x[j];
    }
    for (int bi = 0; bi < nb; ++bi) {
      int b = bl[bi];
      if (b == 0) continue;
      float qm = (float)qmax_of(b);
      float sc = __fdiv_rn(a, qm);
      double acc = 0.0;
      for (int j = 0; j < G; ++j) {
        float q = 0.0f;
        if (sc > 0.0f) q = fminf(fmaxf(rintf(__fdiv_rn(x[j], sc)), -qm), qm);
        float xh = __fmul_rn(q, sc);
        double d = (double)x[j] - (double)xh;
        acc += d * d;
      }
      err[bi] = acc;
    }
  }
  // block reduction in a fixed order
  __shared__ double red[9][256];
  for (int i = 0; i < 8; ++i) red[i][threadIdx.x] = err[i];
  red[8][threadIdx.x] = en;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o)
      for (int i = 0; i < 9; ++i) red[i][threadIdx.x] += red[i][threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x < 9) partial[blockIdx.x * 9 + threadIdx.x] = red[threadIdx.x][0];
}

__global__ void k_eps2_final(const double* partial, int nblk, int nb, int4 bits_lo, int4 bits_hi,
                             double* eps2) {
  int bl[8] = {bits_lo.x, bits_lo.y, bits_lo.z, bits_lo.w, bits_hi.x, bits_hi.y, bits_hi.z, bits_hi.w};
  if (threadIdx.x != 0) return;
  double en = 0.0;
  for (int k = 0; k < nblk; ++k) en += partial[k * 9 + 8];
  for (int bi = 0; bi < nb; ++bi) {
    double e = 0.0;
    for (int k = 0; k < nblk; ++k) e += partial[k * 9 + bi];
    eps2[bi] = (bl[bi] == 0) ? 1.0 : e / en;
  }
}

jolt_status launch_eps2(const int* bits_host, int nb, int G, double* eps2_dev, double* scratch,
                        cudaStream_t s) {
  int b[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int i = 0; i < nb && i < 8; ++i) b[i] = bits_host[i];
  int4 lo = make_int4(b[0], b[1], b[2], b[3]), hi = make_int4(b[4], b[5], b[6], b[7]);
  int ngrp = CALIB_SAMPLES / G;
  int nblk = (ngrp + 255) / 256;
  switch (G) {
    case 32: k_eps2<32><<<nblk, 256, 0, s>>>(nb, lo, hi, scratch); break;
    case 64: k_eps2<64><<<nblk, 256, 0, s>>>(nb, lo, hi, scratch); break;
    case 128: k_eps2<128><<<nblk, 256, 0, s>>>(nb, lo, hi, scratch); break;
    default: set_error("unsupported scale group %d", G); return JOLT_ERR_INVALID_ARG;
  }
  JOLT_LAUNCHED();
  k_eps2_final<<<1, 32, 0, s>>>(scratch, nblk, nb, lo, hi, eps2_dev);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------------ tail fractions -----
// t[r] = sum_{i >= r} w_i / ||X||^2 (r = 0..n), summed smallest first, with
// negative rounding noise in w clamped to 0. One thread per cell and table.
__global__ void k_rd_tables(const CellRD* __restrict__ cells, int ncells,
                            const double* const* __restrict__ wT, const double* const* __restrict__ wD,
                            const double* const* __restrict__ normsq_in,
                            double* const* __restrict__ tT, double* const* __restrict__ tD,
                            const int* __restrict__ nt_used, int* status) {
  int job = blockIdx.x * blockDim.x + threadIdx.x;
  if (job >= 2 * ncells) return;
  int c = job >> 1;
  double ns = *normsq_in[c];
  if (!isfinite(ns) || ns <= 0.0) {
    if (!isfinite(ns)) atomicOr(status, DEV_ERR_NONFINITE);
    ns = 1.0;
  }
  const double* w;
  double* t;
  int n;
  if (job & 1) { w = wD[c]; t = tD[c]; n = cells[c].D; }
  else { w = wT[c]; t = tT[c]; n = nt_used[c]; }
  double acc = 0.0;
  t[n] = 0.0;
  bool finite = true;
  for (int i = n - 1; i >= 0; --i) {
    // a non-finite spectrum entry (from Inf/NaN in the cache) is reported and
    // counted as zero, so the table, and every option the allocator decodes
    // from it, stays finite
    double wi = w[i];
    if (!isfinite(wi)) { finite = false; wi = 0.0; }
    acc += fmax(wi, 0.0);
    t[i] = acc / ns;
  }
  t[n] = 0.0;
  if (!finite) atomicOr(status, DEV_ERR_NONFINITE);
}

jolt_status launch_rd_tables(const CellRD* cells, int ncells, const double* const* wT,
                             const double* const* wD, const double* /*unused*/,
                             double* const* tT, double* const* tD, const int* nt_used,
                             const double* const* normsq_in, int* status, cudaStream_t s) {
  int n = 2 * ncells;
  k_rd_tables<<<(n + 127) / 128, 128, 0, s>>>(cells, ncells, wT, wD, normsq_in, tT, tD, nt_used, status);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

// ------------------------------------------------------------ allocation ----
__device__ __forceinline__ void decode_opt(const AllocArgs& a, const CellRD& c, int idx, int& bi,
                                           int& rt, int& rd) {
  int per_b = c.n_rt * a.n_rd;
  bi = idx / per_b;
  int rem = idx - bi * per_b;
  int ti = rem / a.n_rd;
  int di = rem - ti * a.n_rd;
  rt = a.rt_grid[ti];
  rd = a.rd_grid[di];
}

__device__ __forceinline__ int64_t opt_bytes(const AllocArgs& a, const CellRD& c, int bi, int rt, int rd) {
  const int64_t LH = (int64_t)c.Lg * c.H;
  return 2 * (LH * rt * rd + (int64_t)c.T * rt + (int64_t)c.D * rd) + a.rowbytes[bi] * LH * c.T;
}

// Eq. (2). An option whose feature rank exceeds |g| n_h r_T is excluded
// (+inf): the token-projected tensor has feature rank at most |g| n_h r_T, so
// extra feature columns would be an arbitrary null-space basis.
__device__ __forceinline__ double opt_err(const AllocArgs& a, const CellRD& c, int bi, int rt, int rd) {
  if (rd > c.Lg * c.H * rt) return INFINITY;
  return __dmul_rn(a.eps2[bi], __dadd_rn(c.tT[rt], c.tD[rd]));
}

// The greedy search for bit width index bi: its e + lambda s and option index.
__device__ void greedy_lane(const AllocArgs& a, const CellRD& c, double lam, int bi, double& best, int& bidx) {
  int ti = 0, di = 0;
  auto eval = [&](int t, int d, double& e, int64_t& s) {
    const int rt = a.rt_grid[t], rd = a.rd_grid[d];
    e = opt_err(a, c, bi, rt, rd);
    s = opt_bytes(a, c, bi, rt, rd);
    return __dadd_rn(e, __dmul_rn(lam, (double)s));
  };
  for (int guard = 0; guard < c.n_rt + a.n_rd; ++guard) {
    double e0, e1, e2;
    int64_t s0, s1, s2;
    const double v0 = eval(ti, di, e0, s0);
    bool c1 = false, c2 = false;
    double r1 = 0.0, r2 = 0.0;
    if (ti + 1 < c.n_rt) {
      const double v1 = eval(ti + 1, di, e1, s1);
      if (v1 < v0) { c1 = true; r1 = __ddiv_rn(__dsub_rn(e0, e1), (double)(s1 - s0)); }
    }
    if (di + 1 < a.n_rd) {
      const double v2 = eval(ti, di + 1, e2, s2);
      if (v2 < v0) { c2 = true; r2 = __ddiv_rn(__dsub_rn(e0, e2), (double)(s2 - s0)); }
    }
    if (!c1 && !c2) break;
    if (c1 && (!c2 || r1 >= r2)) ++ti;
    else ++di;
  }
  double e;
  int64_t sb;
  best = eval(ti, di, e, sb);
  bidx = (bi * c.n_rt + ti) * a.n_rd + di;
}

// The page's greedy per-cell search ("Solving the allocation"): for each b
// (one lane per bit width) start at the first grid entries and repeatedly
// take whichever single grid step of r_T or r_d lowers the error most per
// added byte, while that step lowers e + lambda s (ties: the r_T step); then
// the best b, first on ties. The result goes to chunk 0 of the partial
// argmins in enumeration-index form, the other chunks get +inf.
__global__ void __launch_bounds__(32) k_alloc_greedy(AllocArgs a) {
  if (a.st->phase == 3) return;
  const int cell = blockIdx.x, lane = threadIdx.x;
  const CellRD c = a.cells[cell];
  const double lam = a.st->lam;
  double best = INFINITY;
  int bidx = 0x7fffffff;
  if (lane < a.n_bits) greedy_lane(a, c, lam, lane, best, bidx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (ob < best || (ob == best && oi < bidx)) { best = ob; bidx = oi; }
  }
  for (int k = lane; k < a.nchunk; k += 32) {
    a.pv[cell * a.nchunk + k] = (k == 0) ? best : INFINITY;
    a.pi[cell * a.nchunk + k] = (k == 0) ? bidx : 0x7fffffff;
  }
}

// One step of the multiplier search on the total bytes S of the current
// argmins; returns what to do with them: 0 nothing, 1 keep <- cur, 2 finish
// with cur, 3 finish with keep, 4 keep <- cur then finish with keep.
__device__ int alloc_step(AllocState* st, long long S, int* status) {
  st->S = S;
  const long long B = st->budget;
  int act = 0;
  if (st->phase == 0) {
    if (S <= B) { act = 2; st->lam_final = st->lam; st->iters_final = 0; st->phase = 3; }
    else { st->phase = 1; st->lam = st->hi; }
  } else if (st->phase == 1) {
    if (S > B) { atomicOr(status, DEV_ERR_INFEASIBLE); act = 2; st->lam_final = st->lam; st->iters_final = 0; st->phase = 3; }
    else { act = 1; st->iter = 1; st->phase = 2; st->lam = sqrt(st->lo * st->hi); }
  } else {
    const double lo_ok = (1.0 - st->tol) * (double)B;
    if ((double)S >= lo_ok && S <= B) {
      act = 2; st->lam_final = st->lam; st->iters_final = st->iter; st->phase = 3;
    } else {
      if (S > B) st->lo = st->lam;
      else { st->hi = st->lam; act = 1; }
      if (st->iter >= st->max_iters) {
        act = (act == 1) ? 4 : 3;
        st->lam_final = st->hi; st->iters_final = st->max_iters; st->phase = 3;
      } else {
        st->iter += 1;
        st->lam = sqrt(st->lo * st->hi);
      }
    }
  }
  return act;
}

// Applies a step's action to cell c: the kept argmin, or the final choice.
__device__ void alloc_apply(const AllocArgs& a, int act, int c) {
  if (act == 1 || act == 4) a.keep[c] = a.cur[c];
  if (act >= 2) {
    const int idx = (act == 2) ? a.cur[c] : a.keep[c];
    const CellRD cc = a.cells[c];
    int bi, rt, rd;
    decode_opt(a, cc, idx, bi, rt, rd);
    Choice ch;
    ch.rT = rt; ch.rd = rd; ch.b = a.bits[bi]; ch.pad = 0;
    ch.bytes = opt_bytes(a, cc, bi, rt, rd);
    ch.err = opt_err(a, cc, bi, rt, rd);
    a.out[c] = ch;
  }
}

// One block: per-cell argmin over chunks, total bytes, one bisection step.
__global__ void __launch_bounds__(512) k_alloc_decide(AllocArgs a) {
  AllocState* st = a.st;
  if (st->phase == 3) return;
  __shared__ long long sbytes[512];
  __shared__ int action;     // 0 none, 1 keep<-cur, 2 finish with cur, 3 finish with keep
  long long mine = 0;
  for (int c = threadIdx.x; c < a.ncells; c += blockDim.x) {
    double best = INFINITY;
    int bidx = 0x7fffffff;
    for (int k = 0; k < a.nchunk; ++k) {
      double v = a.pv[c * a.nchunk + k];
      int i = a.pi[c * a.nchunk + k];
      if (v < best || (v == best && i < bidx)) { best = v; bidx = i; }
    }
    // no finite e + lambda s in any chunk (non-finite inputs): fall back to the
    // first option, whose grid indices are valid, and report the cell
    if (bidx < 0 || bidx >= a.n_bits * a.cells[c].n_rt * a.n_rd) {
      bidx = 0;
      atomicOr(a.status, DEV_ERR_NONFINITE);
    }
    a.cur[c] = bidx;
    int bi, rt, rd;
    decode_opt(a, a.cells[c], bidx, bi, rt, rd);
    mine += opt_bytes(a, a.cells[c], bi, rt, rd);
  }
  sbytes[threadIdx.x] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long S = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) S += sbytes[i];
    const int act = alloc_step(st, S, a.status);
    action = act;
  }
  __syncthreads();
  const int act = action;
  for (int c = threadIdx.x; c < a.ncells; c += blockDim.x) alloc_apply(a, act, c);
}


// The whole search in one block (small problems): per round, a warp per cell
// takes the cell's argmin of e + lambda s over its options (lanes over the
// options, first index on ties, as the chunked evaluation), the block sums
// the bytes and thread 0 takes the bisection step. Same rounds and results
// as the evaluate + decide launches, without a launch per round.
__global__ void __launch_bounds__(1024) k_alloc_single(AllocArgs a, AllocState init) {
  __shared__ AllocState st;
  __shared__ long long sb[32];
  __shared__ int act_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) { st = init; st.arrive = 0u; }
  __syncthreads();
  for (int it = 0; it < init.max_iters + 2; ++it) {
    const double lam = st.lam;
    long long mine = 0;
    for (int c = warp; c < a.ncells; c += nw) {
      const CellRD cd = a.cells[c];
      double best = INFINITY;
      int bidx = 0x7fffffff;
      if (a.greedy) {
        if (lane < a.n_bits) greedy_lane(a, cd, lam, lane, best, bidx);
      } else {
        const int nopt = a.n_bits * cd.n_rt * a.n_rd;
        for (int idx = lane; idx < nopt; idx += 32) {
          int bi, rt, rd;
          decode_opt(a, cd, idx, bi, rt, rd);
          const double v = __dadd_rn(opt_err(a, cd, bi, rt, rd), __dmul_rn(lam, (double)opt_bytes(a, cd, bi, rt, rd)));
          if (v < best) { best = v; bidx = idx; }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
        if (ob < best || (ob == best && oi < bidx)) { best = ob; bidx = oi; }
      }
      if (lane == 0) {
        if (bidx < 0 || bidx >= a.n_bits * cd.n_rt * a.n_rd) {
          bidx = 0;
          atomicOr(a.status, DEV_ERR_NONFINITE);
        }
        a.cur[c] = bidx;
        int bi, rt, rd;
        decode_opt(a, cd, bidx, bi, rt, rd);
        mine += opt_bytes(a, cd, bi, rt, rd);
      }
    }
    if (lane == 0) sb[warp] = mine;
    __syncthreads();
    if (threadIdx.x == 0) {
      long long S = 0;
      for (int w = 0; w < nw; ++w) S += sb[w];
      act_s = alloc_step(&st, S, a.status);
    }
    __syncthreads();
    const int act = act_s;
    for (int c = threadIdx.x; c < a.ncells; c += blockDim.x) alloc_apply(a, act, c);
    if (st.phase == 3) break;
    __syncthreads();
  }
  if (threadIdx.x == 0) *a.st = st;
}


// One evaluation round of the enumeration, by rows: a row is a (bit width,
// r_T grid entry) pair and its options are the r_d grid entries, so the
// option index (bi*n_rt + ti)*n_rd + di needs no division and the byte count
// is s0 + (bytes per unit of r_d) r_d in exact integers; e and e + lambda s
// are rounded exactly as opt_err / opt_bytes give them. Blocks (chunk, cell)
// write their partial argmin; the last block to finish takes the per-cell
// argmins, the total bytes and the bisection step (alloc_step), so a round is
// one launch.
__global__ void __launch_bounds__(256) k_alloc_rows(AllocArgs a) {
  AllocState* st = a.st;
  if (st->phase == 3) return;
  const int cell = blockIdx.y;
  const CellRD c = a.cells[cell];
  const double lam = st->lam;
  const int nrows = a.n_bits * c.n_rt;
  const int per = (nrows + a.nchunk - 1) / a.nchunk;
  const int r0 = blockIdx.x * per, r1 = min(nrows, r0 + per);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int64_t LH = (int64_t)c.Lg * c.H;
  double best = INFINITY;
  int bidx = 0x7fffffff;
  for (int r = r0 + warp; r < r1; r += nw) {
    const int bi = r / c.n_rt, ti = r - bi * c.n_rt;
    const int rt = a.rt_grid[ti];
    const double eb = a.eps2[bi], tt = c.tT[rt];
    const int64_t s0 = 2 * ((int64_t)c.T * rt) + a.rowbytes[bi] * LH * c.T;
    const int64_t srd = 2 * (LH * rt + c.D);
    const int rd_ok = c.Lg * c.H * rt;      // larger feature ranks are excluded (infinite error)
    for (int di = lane; di < a.n_rd; di += 32) {
      const int rd = a.rd_grid[di];
      if (rd > rd_ok) continue;
      const double e = __dmul_rn(eb, __dadd_rn(tt, c.tD[rd]));
      const double v = __dadd_rn(e, __dmul_rn(lam, (double)(s0 + srd * rd)));
      const int idx = r * a.n_rd + di;
      if (v < best || (v == best && idx < bidx)) { best = v; bidx = idx; }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (ob < best || (ob == best && oi < bidx)) { best = ob; bidx = oi; }
  }
  __shared__ double sv[8];
  __shared__ int si[8];
  __shared__ int last_s;
  if (lane == 0) { sv[warp] = best; si[warp] = bidx; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < nw; ++w)
      if (sv[w] < best || (sv[w] == best && si[w] < bidx)) { best = sv[w]; bidx = si[w]; }
    a.pv[cell * a.nchunk + blockIdx.x] = best;
    a.pi[cell * a.nchunk + blockIdx.x] = bidx;
    __threadfence();
    const unsigned n = atomicAdd(&st->arrive, 1u);
    last_s = (n == gridDim.x * gridDim.y - 1);
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  // ---- the last block: per-cell argmins, total bytes, one bisection step
  __shared__ long long sbytes[256];
  __shared__ int action;
  long long mine = 0;
  for (int cc = threadIdx.x; cc < a.ncells; cc += blockDim.x) {
    double b2 = INFINITY;
    int i2 = 0x7fffffff;
    for (int k = 0; k < a.nchunk; ++k) {
      const double v = __ldcg(a.pv + cc * a.nchunk + k);
      const int i = __ldcg(a.pi + cc * a.nchunk + k);
      if (v < b2 || (v == b2 && i < i2)) { b2 = v; i2 = i; }
    }
    if (i2 < 0 || i2 >= a.n_bits * a.cells[cc].n_rt * a.n_rd) {
      i2 = 0;
      atomicOr(a.status, DEV_ERR_NONFINITE);
    }
    a.cur[cc] = i2;
    int bi, rt, rd;
    decode_opt(a, a.cells[cc], i2, bi, rt, rd);
    mine += opt_bytes(a, a.cells[cc], bi, rt, rd);
  }
  sbytes[threadIdx.x] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long S = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) S += sbytes[i];
    action = alloc_step(st, S, a.status);
    st->arrive = 0u;
  }
  __syncthreads();
  const int act = action;
  for (int cc = threadIdx.x; cc < a.ncells; cc += blockDim.x) alloc_apply(a, act, cc);
}

__global__ void k_alloc_init(AllocState* st, AllocState init) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *st = init;
}

// Writes the initial state (phase 0, lambda = lo), then max_iters + 2 rounds,
// each trying one multiplier: one k_alloc_rows launch (evaluation and, in its
// last block, the decision), or k_alloc_greedy + k_alloc_decide for the
// greedy minimizer; rounds after the final decision return at once. Small
// searches run every round inside one k_alloc_single block.
jolt_status launch_alloc(const AllocArgs& a, const AllocState& init, cudaStream_t s) {
  // small searches (all options of all cells within a few per thread): one block
  if ((int64_t)a.ncells * a.n_bits * std::max(a.n_rt_max, 1) * a.n_rd <= (int64_t)16 * 1024) {
    k_alloc_single<<<1, 1024, 0, s>>>(a, init);
    JOLT_LAUNCHED();
    return JOLT_OK;
  }
  AllocState i0 = init;
  i0.arrive = 0u;
  k_alloc_init<<<1, 32, 0, s>>>(a.st, i0);
  JOLT_LAUNCHED();
  dim3 grid(a.nchunk, a.ncells);
  for (int it = 0; it < init.max_iters + 2; ++it) {
    if (a.greedy) {
      k_alloc_greedy<<<a.ncells, 32, 0, s>>>(a);
      JOLT_LAUNCHED();
      k_alloc_decide<<<1, 512, 0, s>>>(a);
    } else {
      k_alloc_rows<<<grid, 256, 0, s>>>(a);
    }
    JOLT_LAUNCHED();
  }
  return JOLT_OK;
}

}  // namespace jolt

namespace jolt {

// ---------------------------------------------- sharded allocation records --
__global__ void k_write_records(const CellRD* __restrict__ cells, const double* const* __restrict__ normsq,
                                const int4* __restrict__ ids, uint64_t fp, int ntp, int rec_bytes,
                                uint8_t* __restrict__ out) {
  const int c = blockIdx.x;
  const CellRD cd = cells[c];
  uint8_t* rec = out + (int64_t)c * rec_bytes;
  double* tT = reinterpret_cast<double*>(rec + sizeof(RDRecordHdr));
  double* tD = tT + ntp;
  for (int i = threadIdx.x; i < ntp; i += blockDim.x) tT[i] = (i <= cd.nt) ? cd.tT[i] : 0.0;
  for (int i = threadIdx.x; i <= cd.D; i += blockDim.x) tD[i] = cd.tD[i];
  if (threadIdx.x == 0) {
    RDRecordHdr h;
    h.magic = RD_MAGIC;
    h.Lg = cd.Lg; h.H = cd.H; h.T = cd.T; h.D = cd.D; h.n_rt = cd.n_rt; h.nt = cd.nt; h.ntp = ntp;
    h.fingerprint = fp;
    h.norm_sq = *normsq[c];
    const int4 id = ids[c];
    h.seq = id.x; h.group = id.y; h.kind = id.z; h.rec_bytes = rec_bytes;
    *reinterpret_cast<RDRecordHdr*>(rec) = h;
  }
}

jolt_status launch_write_records(const CellRD* cells, int ncells, const double* const* normsq, const int4* ids,
                                 uint64_t fingerprint, int ntp, int rec_bytes, uint8_t* out, cudaStream_t s) {
  if (ncells <= 0) return JOLT_OK;
  k_write_records<<<ncells, 128, 0, s>>>(cells, normsq, ids, fingerprint, ntp, rec_bytes, out);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

__global__ void k_records_to_rd(const uint8_t* __restrict__ recs, int n_total, int rec_bytes, int ntp, int D,
                                uint64_t fp, int n_rt_max, int first, int nlocal, const int4* __restrict__ ids,
                                CellRD* __restrict__ out, int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_total) return;
  const uint8_t* rec = recs + (int64_t)i * rec_bytes;
  const RDRecordHdr h = *reinterpret_cast<const RDRecordHdr*>(rec);
  const double* tT = reinterpret_cast<const double*>(rec + sizeof(RDRecordHdr));
  bool ok = h.magic == RD_MAGIC && h.fingerprint == fp && h.rec_bytes == rec_bytes && h.ntp == ntp && h.D == D &&
            h.n_rt >= 1 && h.n_rt <= n_rt_max && h.nt >= 1 && h.nt < ntp && h.Lg >= 1 && h.H >= 1 && h.T >= 1;
  if (i >= first && i < first + nlocal) {
    const int4 id = ids[i - first];
    ok = ok && h.seq == id.x && h.group == id.y && h.kind == id.z;
  }
  CellRD c;
  c.Lg = ok ? h.Lg : 1; c.H = ok ? h.H : 1; c.T = ok ? h.T : 1; c.D = D;
  c.n_rt = ok ? h.n_rt : 1;
  c.nt = ok ? h.nt : 1;
  c.tT = tT;
  c.tD = tT + ntp;
  out[i] = c;
  if (!ok) atomicOr(status, DEV_ERR_MISMATCH);
}

jolt_status launch_records_to_rd(const uint8_t* recs, int n_total, int rec_bytes, int ntp, int D, uint64_t fingerprint,
                                 int n_rt_max, int first, int nlocal, const int4* ids, CellRD* out, int* status,
                                 cudaStream_t s) {
  if (n_total <= 0) return JOLT_OK;
  k_records_to_rd<<<(n_total + 127) / 128, 128, 0, s>>>(recs, n_total, rec_bytes, ntp, D, fingerprint, n_rt_max, first,
                                                        nlocal, ids, out, status);
  JOLT_LAUNCHED();
  return JOLT_OK;
}

}  // namespace jolt
