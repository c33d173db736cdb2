// The C ABI of include/jolt.h: plans, handles and the order of the stages of
// "A JoLT for the KV Cache" (Section 3): spectra of every cell -> rate-distortion
// tables -> one shared-multiplier allocation over all cells -> ST-HOSVD fit
// -> rotated low-bit residual; decompression rebuilds dense bf16.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"
#include "jolt_umma.cuh"

namespace jolt {

// ---------------------------------------------------------------- errors ---
static thread_local char g_err[512] = "";
void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}
static uint64_t g_launches = 0;
uint64_t& launch_counter() { return g_launches; }

// ------------------------------------------------------------- allocator ---
static jolt_alloc_fn g_alloc = nullptr;
static jolt_free_fn g_free = nullptr;
static void* g_ctx = nullptr;

void* dev_alloc(size_t bytes, cudaStream_t s) {
  if (bytes == 0) bytes = 256;
  if (g_alloc) return g_alloc(bytes, s, g_ctx);
  void* p = nullptr;
  if (cudaMallocAsync(&p, bytes, s) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return p;
}
void dev_free(void* p, cudaStream_t s) {
  if (!p) return;
  if (g_free) { g_free(p, s, g_ctx); return; }
  cudaFreeAsync(p, s);
}

// ------------------------------------------------------------- profiling ---
struct ProfRec {
  int stage;
  cudaEvent_t a, b;
  int64_t launches;
};
static bool g_prof_on = false;
static std::vector<ProfRec> g_prof;
static std::vector<cudaEvent_t> g_prof_pool;

static cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

static void prof_clear() {
  for (auto& r : g_prof) {
    if (r.a) g_prof_pool.push_back(r.a);
    if (r.b) g_prof_pool.push_back(r.b);
  }
  g_prof.clear();
}

ProfScope::ProfScope(int st, cudaStream_t s) : stage(st), stream(s), launches0(g_launches), slot(-1) {
  if (!g_prof_on) return;
  ProfRec r{st, prof_event(), prof_event(), 0};
  cudaEventRecord(r.a, s);
  slot = (int)g_prof.size();
  g_prof.push_back(r);
}

void ProfScope::end() {
  if (slot < 0) return;
  cudaEventRecord(g_prof[slot].b, stream);
  g_prof[slot].launches = (int64_t)(g_launches - launches0);
  slot = -1;
}

ProfScope::~ProfScope() { end(); }

// A bump region carved out of one device allocation.
struct Arena {
  uint8_t* base = nullptr;
  size_t size = 0, used = 0;
  template <class T>
  T* take(size_t n) {
    size_t off = (used + 255) & ~(size_t)255;
    used = off + n * sizeof(T);
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
};

}  // namespace jolt

using namespace jolt;

// ------------------------------------------------------------------ plan ---
struct HostCell {
  int seq, group, kind, l0, Lg;
  int N, nmin;     // N = Lg*H*D, nmin = min(T, N)
  int nt;          // token spectrum length fed to the allocator
  int n_rt, rmax;  // usable rank-grid entries and the largest of them
  int64_t min_bytes, max_bytes;   // cheapest and dearest admissible option (Eq. 1)
};

struct jolt_plan_s {
  jolt_layout lay;
  std::vector<int32_t> gstart;
  jolt_options opt;
  std::vector<int32_t> rt_grid, rd_grid, bits;
  std::vector<int64_t> rowbytes;
  int64_t budget = 0;
  int G = 0, D = 0, T = 0, H = 0;
  double C = 0.0;
  int qcap = 0;
  int ncells = 0, nmin_max = 0, rmax_all = 0, lh_max = 0, nt_max = 0;
  std::vector<HostCell> hc;
  std::vector<CellDesc> cdesc;
  CellDesc* cdesc_pinned = nullptr;
  bool cdesc_valid = false;
  const void* cdesc_k = nullptr;
  const void* cdesc_v = nullptr;
  // device
  cudaStream_t init_stream = 0;
  Arena ws;
  int* d_status = nullptr;
  double* d_eps2 = nullptr;
  int64_t* d_rowbytes = nullptr;
  int* d_bits = nullptr;
  int* d_rt = nullptr;
  int* d_rd = nullptr;
  float2* d_cs = nullptr;
  float4* d_csq = nullptr;       // the RoPE table tiled for the stream kernels
  CellDesc* d_cells = nullptr;
  CellRD* d_rd_cells = nullptr;
  int* d_nt = nullptr;
  int* d_rmax = nullptr;
  int* d_nlh = nullptr;
  int* d_rT_used = nullptr;      // r_T per cell (device copy for Y gram)
  int* d_Dn = nullptr;           // D per cell (eigenvector count of the D x D solves)
  // per-cell arrays of pointers (device)
  double** d_GT = nullptr;  double** d_ZT = nullptr;  double** d_VtT = nullptr;
  double** d_wT = nullptr;  double** d_Cd = nullptr;  double** d_wD = nullptr;
  double** d_nsq = nullptr; double** d_tT = nullptr;  double** d_tD = nullptr;
  double** d_Y = nullptr;   double** d_CY = nullptr;  double** d_VtY = nullptr;
  double** d_wY = nullptr;  double** d_ZY = nullptr;  double** d_Uf = nullptr;
  uint16_t** d_M = nullptr; uint16_t** d_dst = nullptr;
  EighJob* d_jobs_spec = nullptr;
  EighJob* d_jobs_fit = nullptr;
  double* d_fpart = nullptr;
  int fchunk = 0;
  double* d_apv = nullptr;
  int* d_api = nullptr;
  int* d_cur = nullptr;
  int* d_keep = nullptr;
  int achunk = 0;
  // host mirrors of pointer arrays
  std::vector<double*> h_tT, h_tD, h_wT, h_wD, h_nsq;
  std::vector<uint16_t*> h_M;
  void* ws_alloc = nullptr;
  // randomized mode (Section 3.1): sketch width k = q + p rounded up to 16,
  // GEMM tile width BN, padded extents, working buffers
  int k = 0, BN = 0, nt_k = 0, kpad = 0, rpad = 0, tp = 0, Ncmax = 0, fg_chunks = 0, fg_spc = 0, q_used = 0;
  int gemm_pair = 0;        // X W / X^T Y on CTA pairs (tcgen05 cta_group::2)
  // k > 256 on CTA pairs: N tiles up to 512 wide (one TMEM accumulator, two
  // MMAs per K step), so X is streamed ceil(k/512) times per pass instead of
  // ceil(k/256); B boxes of two heights hb[0], hb[1]
  int wide = 0, wide_nt = 0, wide_w0 = 0;
  int wtn0[4] = {}, wta[4] = {}, wtb[4] = {}, wmap_a[4] = {}, wmap_b[4] = {}, whb[2] = {};
  // tensor-core residual/decode streams: U_T^ rows and M^T, padded to 64 ranks
  bool tc_in = false;
  int rows_u = 0, rpad_m = 0;
  uint16_t* Ut_ws = nullptr;
  uint16_t* Mt_ws = nullptr;
  bool copy_k = false, copy_v = false;
  uint16_t* Xk = nullptr;  uint16_t* Xv = nullptr;
  uint16_t* Wt = nullptr;  uint16_t* Yt = nullptr;  uint16_t* Pt = nullptr;
  float* Z = nullptr;      float* GW32 = nullptr;   float* fgpart = nullptr;
  double* Gz = nullptr;    double* Rm = nullptr;    double* P0 = nullptr;   double* X1 = nullptr;
  double* MB = nullptr;    double* eZ = nullptr;    double* eVt = nullptr;  double* ew = nullptr;
  double* ework = nullptr; double* trs = nullptr;   double* P64 = nullptr;
  double* eF = nullptr;    double* Rinv = nullptr;  double* RTk = nullptr;
  std::vector<double*> h_FT;     // exact mode: inverse-iteration scratch per cell
  int* d_cl0 = nullptr; int* d_cb = nullptr; int* d_cLg = nullptr; int* d_ckind = nullptr;
  int* d_Nc = nullptr; int* d_cis = nullptr;
  uint16_t** d_utp = nullptr;
  EighJob* d_jobs_rand = nullptr;
  double* eig_scr = nullptr;   unsigned int* eig_cnt = nullptr;   int eig_nmax = 0;
  double* gram_part = nullptr;  // GRAM_SPLIT partial Grams (randomized)
  // shared-budget protocol: summary record layout and the settings' fingerprint
  int ntp = 0, rec_bytes = 0;
  uint64_t fingerprint = 0;
  int4* d_ids = nullptr;        // (global sequence, global group, kind) per cell
};

struct jolt_handle_s {
  jolt_plan_t* plan = nullptr;
  cudaStream_t stream = 0;
  uint64_t seed = 0;
  uint8_t* payload = nullptr;
  int64_t capacity = 0;
  CellOut* d_out = nullptr;
  Choice* d_choice = nullptr;
  AllocState* d_state = nullptr;
  int* d_status = nullptr;
  void* block = nullptr;
  void* qblock = nullptr;        // QR-Gaussian rotation: scratch + Q per sequence
  double* d_qrot = nullptr;      // [batch][D][D], NULL for the Hadamard rotation
  int64_t budget = 0;
  int phase = 0;                 // 1: spectra done (begin), 2: compressed (end)
  const void* k_in = nullptr;    // inputs of a begun two-phase compression
  const void* v_in = nullptr;
  std::vector<CellOut> h_out;    // host copy of the cells' layout (decode attention)
};

static jolt_status status_from_dev(int st) {
  if (st == 0) return JOLT_OK;
  if (st & DEV_ERR_INFEASIBLE) { set_error("byte budget infeasible for the rank/bit grids"); return JOLT_ERR_BUDGET_INFEASIBLE; }
  if (st & DEV_ERR_NONFINITE) { set_error("a cell's squared Frobenius norm is not finite"); return JOLT_ERR_NONFINITE; }
  if (st & DEV_ERR_TIMEOUT) { set_error("a bounded device wait expired"); return JOLT_ERR_TIMEOUT; }
  if (st & DEV_ERR_EIG_NOCONV) { set_error("eigensolver did not converge"); return JOLT_ERR_CUDA; }
  if (st & DEV_ERR_CHOL) { set_error("Cholesky factorization failed (rank-deficient sketch)"); return JOLT_ERR_CUDA; }
  if (st & DEV_ERR_MISMATCH) {
    set_error("gathered rate-distortion records do not match this plan (other settings, sizes, or another cell "
              "in this plan's slice)");
    return JOLT_ERR_INVALID_ARG;
  }
  set_error("device status 0x%x", st);
  return JOLT_ERR_CUDA;
}

static int64_t residual_row_bytes(int b, int D, int G) {
  if (b == 0) return 0;
  return ((int64_t)b * D + 32 * (D / G)) / 8;
}

static jolt_status plan_build_workspace(jolt_plan_s* p);

extern "C" {

void jolt_default_options(jolt_options* o) {
  if (!o) return;
  memset(o, 0, sizeof(*o));
  o->mode = JOLT_EXACT;
  o->n_bits = 4;
  o->bits[0] = 0; o->bits[1] = 2; o->bits[2] = 4; o->bits[3] = 8;
  o->oversample_p = 8;
  o->power_iters = 2;
  o->scale_group = 0;
  o->rotation = JOLT_ROT_HADAMARD;
  o->budget_tol = 0.005;
  o->minimizer = JOLT_MIN_ENUMERATE;
  o->max_iters = 50;
}

const char* jolt_last_error(void) { return g_err; }
uint64_t jolt_launch_count(void) { return g_launches; }

void jolt_profile_enable(int32_t on) {
  prof_clear();
  g_prof_on = on != 0;
}

jolt_status jolt_profile_read(jolt_stage_stats* out, int32_t n) {
  if (!out || n < 1) { set_error("null output"); return JOLT_ERR_INVALID_ARG; }
  for (int i = 0; i < n; ++i) out[i] = jolt_stage_stats{0.0, 0, 0};
  for (auto& r : g_prof) {
    if (r.stage < 0 || r.stage >= n) continue;
    JOLT_CUDA_TRY(cudaEventSynchronize(r.b));
    float ms = 0.0f;
    JOLT_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    out[r.stage].ms += ms;
    out[r.stage].calls += 1;
    out[r.stage].launches += r.launches;
  }
  return JOLT_OK;
}

jolt_status jolt_set_allocator(jolt_alloc_fn a, jolt_free_fn f, void* ctx) {
  if ((a == nullptr) != (f == nullptr)) { set_error("alloc and free must both be set or both NULL"); return JOLT_ERR_INVALID_ARG; }
  g_alloc = a; g_free = f; g_ctx = ctx;
  return JOLT_OK;
}

int32_t jolt_num_cells(const jolt_plan_t* p) { return p ? p->ncells : 0; }

static jolt_status validate(const jolt_layout* L, const jolt_options* o) {
  if (!L || !o || !L->group_start) { set_error("null layout/options/group_start"); return JOLT_ERR_INVALID_ARG; }
  if (L->batch < 1 || L->n_layers < 1 || L->n_heads < 1 || L->seq_len < 1 || L->n_groups < 1) {
    set_error("non-positive layout dimension"); return JOLT_ERR_INVALID_ARG;
  }
  if (L->head_dim != 64 && L->head_dim != 128) { set_error("head_dim must be 64 or 128 (got %d)", L->head_dim); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if (L->dtype != JOLT_BF16 && L->dtype != JOLT_F32) { set_error("dtype must be JOLT_BF16 or JOLT_F32"); return JOLT_ERR_INVALID_ARG; }
  if (L->group_start[0] != 0 || L->group_start[L->n_groups] != L->n_layers) { set_error("groups must cover layers 0..n_layers"); return JOLT_ERR_INVALID_ARG; }
  for (int g = 0; g < L->n_groups; ++g)
    if (L->group_start[g + 1] <= L->group_start[g]) { set_error("group_start must increase"); return JOLT_ERR_INVALID_ARG; }
  if (L->stride_t < L->head_dim || L->stride_h < 1 || L->stride_l < 1 || L->stride_b < 1) { set_error("bad strides"); return JOLT_ERR_INVALID_ARG; }
  if (L->rope_theta_k < 0.0f) { set_error("rope_theta_k must be >= 0"); return JOLT_ERR_INVALID_ARG; }
  if (o->mode != JOLT_EXACT && o->mode != JOLT_RANDOMIZED) { set_error("bad mode"); return JOLT_ERR_INVALID_ARG; }
  if (o->rotation != JOLT_ROT_HADAMARD && o->rotation != JOLT_ROT_QR_GAUSS) { set_error("rotation must be JOLT_ROT_HADAMARD or JOLT_ROT_QR_GAUSS"); return JOLT_ERR_INVALID_ARG; }
  if (o->n_bits < 1 || o->n_bits > 8) { set_error("n_bits must be 1..8"); return JOLT_ERR_INVALID_ARG; }
  for (int i = 0; i < o->n_bits; ++i) {
    int b = o->bits[i];
    if (!(b == 0 || b == 2 || b == 3 || b == 4 || b == 8)) { set_error("bit width %d not in {0,2,3,4,8}", b); return JOLT_ERR_INVALID_ARG; }
    if (i && b <= o->bits[i - 1]) { set_error("bits must increase"); return JOLT_ERR_INVALID_ARG; }
  }
  int G = o->scale_group ? o->scale_group : L->head_dim;
  if (!(G == 32 || G == 64 || G == 128) || L->head_dim % G) { set_error("scale_group must be 32/64/128 and divide D"); return JOLT_ERR_INVALID_ARG; }
  if (o->budget_tol < 0 || o->budget_tol >= 1 || o->max_iters < 1) { set_error("bad tolerance/max_iters"); return JOLT_ERR_INVALID_ARG; }
  if (o->seq_base < 0 || o->group_base < 0) { set_error("seq_base and group_base must be >= 0"); return JOLT_ERR_INVALID_ARG; }
  if (!(o->cap_ratio >= 0.0)) { set_error("cap_ratio must be >= 0"); return JOLT_ERR_INVALID_ARG; }
  if (o->minimizer != JOLT_MIN_ENUMERATE && o->minimizer != JOLT_MIN_GREEDY) { set_error("minimizer must be JOLT_MIN_ENUMERATE or JOLT_MIN_GREEDY"); return JOLT_ERR_INVALID_ARG; }
  auto chk = [](int n, const int32_t* g) {
    if (n < 0 || (n > 0 && !g)) return false;
    for (int i = 0; i < n; ++i) if (g[i] < 1 || (i && g[i] <= g[i - 1])) return false;
    return true;
  };
  if (!chk(o->n_rt, o->rt_grid) || !chk(o->n_rd, o->rd_grid)) { set_error("rank grids must be increasing positive integers"); return JOLT_ERR_INVALID_ARG; }
  return JOLT_OK;
}

static int qcap_eq5(int T, double C) {
  int qmin = (C <= 4.0) ? 32 : 64;
  int q = std::max(qmin, (T + 31) / 32);
  return std::min(q, 512);
}

jolt_status jolt_plan(const jolt_layout* L, int64_t byte_budget, const jolt_options* opt,
                      jolt_plan_t** out) {
  if (!out) { set_error("null out"); return JOLT_ERR_INVALID_ARG; }
  *out = nullptr;
  JOLT_TRY(validate(L, opt));
  if (byte_budget <= 0) { set_error("byte budget must be positive"); return JOLT_ERR_INVALID_ARG; }
  auto* p = new jolt_plan_s();
  p->lay = *L;
  p->gstart.assign(L->group_start, L->group_start + L->n_groups + 1);
  p->lay.group_start = p->gstart.data();
  p->opt = *opt;
  p->rt_grid.assign(opt->rt_grid, opt->rt_grid + (opt->rt_grid ? opt->n_rt : 0));
  p->rd_grid.assign(opt->rd_grid, opt->rd_grid + (opt->rd_grid ? opt->n_rd : 0));
  p->opt.rt_grid = nullptr;
  p->opt.rd_grid = nullptr;
  p->bits.assign(opt->bits, opt->bits + opt->n_bits);
  p->budget = byte_budget;
  p->D = L->head_dim; p->T = L->seq_len; p->H = L->n_heads;
  p->G = opt->scale_group ? opt->scale_group : p->D;
  for (int b : p->bits) p->rowbytes.push_back(residual_row_bytes(b, p->D, p->G));
  const double dense = 2.0 * 2.0 * (double)L->batch * L->n_layers * L->n_heads * (double)L->seq_len * p->D;
  p->C = opt->cap_ratio > 0.0 ? opt->cap_ratio : dense / (double)byte_budget;
  p->qcap = qcap_eq5(p->T, p->C);
  const bool rnd = opt->mode == JOLT_RANDOMIZED;
  // rd grid: default every integer 1..D
  if (p->rd_grid.empty()) for (int r = 1; r <= p->D; ++r) p->rd_grid.push_back(r);
  while (!p->rd_grid.empty() && p->rd_grid.back() > p->D) p->rd_grid.pop_back();
  if (p->rd_grid.empty()) { delete p; set_error("rd grid has no value <= D"); return JOLT_ERR_INVALID_ARG; }
  // cells
  int maxN = 0;
  for (int b = 0; b < L->batch; ++b)
    for (int g = 0; g < L->n_groups; ++g)
      for (int kind = 0; kind < 2; ++kind) {
        HostCell c{};
        c.seq = b; c.group = g; c.kind = kind; c.l0 = p->gstart[g];
        c.Lg = p->gstart[g + 1] - p->gstart[g];
        c.N = c.Lg * p->H * p->D;
        c.nmin = std::min(p->T, c.N);
        maxN = std::max(maxN, c.N);
        p->hc.push_back(c);
      }
  p->ncells = (int)p->hc.size();
  // token-rank bound per cell and the shared rt grid
  int rcap_all = 0;
  for (auto& c : p->hc) {
    int cap = rnd ? std::min(p->qcap, c.nmin) : c.nmin;
    if (opt->rt_max > 0) cap = std::min(cap, opt->rt_max);
    c.nt = rnd ? (std::min(p->qcap, c.nmin) + 1) : c.nmin;
    c.rmax = cap;
    rcap_all = std::max(rcap_all, cap);
  }
  if (p->rt_grid.empty()) for (int r = 1; r <= rcap_all; ++r) p->rt_grid.push_back(r);
  for (auto& c : p->hc) {
    c.n_rt = 0;
    for (int r : p->rt_grid) if (r <= c.rmax) ++c.n_rt;
    if (c.n_rt == 0) { delete p; set_error("rt grid has no value within the token-rank bound"); return JOLT_ERR_INVALID_ARG; }
    c.rmax = p->rt_grid[c.n_rt - 1];
    // cheapest admissible option (r_d <= L_g*H*r_T)
    int64_t best = INT64_MAX;
    const int64_t LH = (int64_t)c.Lg * p->H;
    for (size_t bi = 0; bi < p->bits.size(); ++bi)
      for (int ti = 0; ti < c.n_rt; ++ti) {
        const int rt = p->rt_grid[ti];
        const int rd = p->rd_grid[0];
        if (rd > LH * rt) continue;
        int64_t s = 2 * (LH * rt * rd + (int64_t)p->T * rt + (int64_t)p->D * rd) + p->rowbytes[bi] * LH * p->T;
        best = std::min(best, s);
      }
    if (best == INT64_MAX) {
      delete p;
      set_error("no admissible (r_t, r_d) pair: every r_d exceeds L_g*H*r_t");
      return JOLT_ERR_INVALID_ARG;
    }
    c.min_bytes = best;
    {
      // Eq. (1) grows with each of r_T, r_d and b: the dearest admissible
      // option takes the largest of each (r_d capped at L_g*H*r_T)
      const int rt = c.rmax;
      int rd = 0;
      for (int x : p->rd_grid) if (x <= LH * rt) rd = x;
      c.max_bytes = 2 * (LH * rt * rd + (int64_t)p->T * rt + (int64_t)p->D * rd) + p->rowbytes.back() * LH * p->T;
    }
    p->nmin_max = std::max(p->nmin_max, c.nmin);
    p->rmax_all = std::max(p->rmax_all, c.rmax);
    p->lh_max = std::max(p->lh_max, c.Lg * p->H);
    p->nt_max = std::max(p->nt_max, c.nt);
  }
  if (!rnd && p->nmin_max > 2048) {
    delete p;
    set_error("exact mode needs min(T, L_g*H*D) <= 2048 (got %d); use JOLT_RANDOMIZED", p->nmin_max);
    return JOLT_ERR_UNSUPPORTED_SHAPE;
  }
  if (rnd) {
    int q = 0, nmin_all = INT32_MAX;
    for (auto& c : p->hc) { q = std::max(q, c.nt - 1); nmin_all = std::min(nmin_all, c.nmin); p->Ncmax = std::max(p->Ncmax, c.N); }
    p->q_used = q;
    p->k = ((q + std::max(opt->oversample_p, 0) + 15) / 16) * 16;
    if (p->k > nmin_all) {
      delete p;
      set_error("sketch width k=%d exceeds min(T, L_g*H*D)=%d; use JOLT_EXACT", q + opt->oversample_p, nmin_all);
      return JOLT_ERR_UNSUPPORTED_SHAPE;
    }
    if (opt->power_iters < 0 || opt->power_iters > 8) { delete p; set_error("power_iters must be 0..8"); return JOLT_ERR_INVALID_ARG; }
    const int ntile = (p->k + 255) / 256;
    p->BN = (((p->k + ntile - 1) / ntile) + 15) / 16 * 16;
    p->nt_k = (p->k + p->BN - 1) / p->BN;
    p->kpad = (p->k + 63) / 64 * 64;
    p->gemm_pair = (p->BN / 2) % 8 == 0;   // BN is a multiple of 16, so always
    if (p->gemm_pair && p->k > 256 && p->k <= 2048) {
      const int nt = (p->k + 511) / 512;
      const int w0 = ((p->k + nt - 1) / nt + 15) / 16 * 16;
      int nh = 0;
      bool ok = true;
      for (int j = 0; j < nt && ok; ++j) {
        const int n0 = j * w0, w = std::min(w0, p->k - n0);
        const int a = ((w + 1) / 2 + 15) / 16 * 16, b = w - a;
        if (a < 16 || b < 16 || a > 256 || b > 256) { ok = false; break; }
        p->wtn0[j] = n0; p->wta[j] = a; p->wtb[j] = b;
        int* sel[2] = {&p->wmap_a[j], &p->wmap_b[j]};
        const int hh[2] = {a / 2, b / 2};
        for (int t = 0; t < 2 && ok; ++t) {
          int f = -1;
          for (int u = 0; u < nh; ++u) if (p->whb[u] == hh[t]) f = u;
          if (f < 0) { if (nh == 2) { ok = false; break; } p->whb[nh] = hh[t]; f = nh++; }
          *sel[t] = f;
        }
      }
      if (ok) {
        if (nh == 1) p->whb[1] = p->whb[0];
        p->wide = 1; p->wide_nt = nt; p->wide_w0 = w0;
      }
    }
    p->rpad = (p->rmax_all + 127) / 128 * 128;
    p->tp = (p->T + 7) / 8 * 8;
    const int steps = ((p->Ncmax + 127) / 128) * ((p->T + 63) / 64);
    p->fg_spc = std::max(64, (steps + 31) / 32);
    p->fg_chunks = (steps + p->fg_spc - 1) / p->fg_spc;
    auto aligned = [&](int64_t st) { return st % 8 == 0; };
    const bool tma_ok = L->dtype == JOLT_BF16 && aligned(L->stride_t) && aligned(L->stride_h) &&
                        aligned(L->stride_l) && aligned(L->stride_b);
    p->copy_k = !tma_ok || L->rope_theta_k > 0;
    p->copy_v = !tma_ok;
  }
  int64_t minsum = 0;
  for (auto& c : p->hc) minsum += c.min_bytes;
  if (byte_budget < minsum) {
    delete p;
    set_error("budget %lld below the cheapest allocation %lld", (long long)byte_budget, (long long)minsum);
    return JOLT_ERR_BUDGET_INFEASIBLE;
  }
  p->tp = (p->T + 7) / 8 * 8;
  p->rows_u = (p->rmax_all + 63) / 64 * 64;
  p->rpad_m = p->rows_u;
  // bf16 input whose strides TMA can address (16-byte multiples) takes the
  // tensor-core residual stream; fp32 input uses the per-row kernel
  p->tc_in = L->dtype == JOLT_BF16 && L->stride_t % 8 == 0 && L->stride_h % 8 == 0 && L->stride_l % 8 == 0 &&
             L->stride_b % 8 == 0;
  if (!g_alloc) {
    // With the default allocator, keep freed blocks in the device's default
    // pool instead of returning them at every synchronisation: a handle's
    // payload (gigabytes for long contexts) is then reused by the next call
    // rather than mapped again.
    int dev = 0;
    cudaMemPool_t pool;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
      uint64_t thr = UINT64_MAX;
      cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
    }
    cudaGetLastError();
  }
  // settings every process of a shared-budget allocation must agree on
  {
    uint64_t h = 1469598103934665603ull;
    auto mix = [&](uint64_t x) { for (int i = 0; i < 8; ++i) { h ^= (x >> (8 * i)) & 0xFF; h *= 1099511628211ull; } };
    mix((uint64_t)p->D); mix((uint64_t)p->G); mix((uint64_t)opt->mode); mix((uint64_t)opt->minimizer);
    mix((uint64_t)opt->max_iters);
    uint64_t tb;
    memcpy(&tb, &opt->budget_tol, 8);
    mix(tb);
    mix(p->bits.size());
    for (int b : p->bits) mix((uint64_t)b);
    mix(p->rd_grid.size());
    for (int r : p->rd_grid) mix((uint64_t)r);
    // an explicit token-rank grid must match; the default one is the
    // integers from 1 and agrees on every prefix
    mix(opt->rt_grid ? (uint64_t)opt->n_rt : 0xFFFFFFFFull);
    if (opt->rt_grid) for (int i = 0; i < opt->n_rt; ++i) mix((uint64_t)opt->rt_grid[i]);
    p->fingerprint = h;
  }
  p->ntp = p->nt_max + 1;
  p->rec_bytes = (int)((sizeof(RDRecordHdr) + 8 * (size_t)p->ntp + 8 * (size_t)(p->D + 1) + 255) / 256 * 256);
  jolt_status st = plan_build_workspace(p);
  if (st != JOLT_OK) { jolt_free_plan(p); return st; }
  *out = p;
  return JOLT_OK;
}

}  // extern "C"

// ------------------------------------------------------------- workspace ---
template <class T>
static T* upload(Arena& A, const std::vector<T>& v) {
  return A.take<T>(v.size());
}

static jolt_status plan_build_workspace(jolt_plan_s* p) {
  const int nc = p->ncells, D = p->D, T = p->T;
  p->fchunk = 64;
  p->achunk = 32;
  // two passes: size, then carve
  for (int pass = 0; pass < 2; ++pass) {
    Arena& A = p->ws;
    A.used = 0;
    p->d_status = A.take<int>(4);
    p->d_eps2 = A.take<double>(8);
    p->d_rowbytes = A.take<int64_t>(8);
    p->d_bits = A.take<int>(8);
    p->d_rt = A.take<int>(p->rt_grid.size());
    p->d_rd = A.take<int>(p->rd_grid.size());
    p->d_cs = p->lay.rope_theta_k > 0 ? A.take<float2>((size_t)T * (D / 2)) : nullptr;
    p->d_csq = p->lay.rope_theta_k > 0 ? A.take<float4>((size_t)((T + 127) / 128) * 128 * (D / 4)) : nullptr;
    p->d_cells = A.take<CellDesc>(nc);
    p->d_rd_cells = A.take<CellRD>(nc);
    p->d_nt = A.take<int>(nc);
    p->d_rmax = A.take<int>(nc);
    p->d_nlh = A.take<int>(nc);
    p->d_rT_used = A.take<int>(nc);
    p->d_Dn = A.take<int>(nc);
    p->d_GT = A.take<double*>(nc); p->d_ZT = A.take<double*>(nc); p->d_VtT = A.take<double*>(nc);
    p->d_wT = A.take<double*>(nc); p->d_Cd = A.take<double*>(nc); p->d_wD = A.take<double*>(nc);
    p->d_nsq = A.take<double*>(nc); p->d_tT = A.take<double*>(nc); p->d_tD = A.take<double*>(nc);
    p->d_Y = A.take<double*>(nc); p->d_CY = A.take<double*>(nc); p->d_VtY = A.take<double*>(nc);
    p->d_wY = A.take<double*>(nc); p->d_ZY = A.take<double*>(nc); p->d_Uf = A.take<double*>(nc);
    p->d_M = A.take<uint16_t*>(nc); p->d_dst = A.take<uint16_t*>(nc);
    p->d_jobs_spec = A.take<EighJob>(2 * nc);
    p->d_jobs_fit = A.take<EighJob>(nc);
    p->d_fpart = A.take<double>((size_t)nc * p->fchunk * (D * D + 1));
    p->d_apv = A.take<double>((size_t)nc * p->achunk);
    p->d_api = A.take<int>((size_t)nc * p->achunk);
    p->d_cur = A.take<int>(nc);
    p->d_keep = A.take<int>(nc);
    p->d_ids = A.take<int4>(nc);
    p->Ut_ws = A.take<uint16_t>((size_t)nc * p->rows_u * p->tp);
    p->Mt_ws = A.take<uint16_t>((size_t)nc * p->lh_max * D * p->rpad_m);
    p->eig_nmax = std::max(p->opt.mode == JOLT_RANDOMIZED ? p->k : p->nmin_max, D);
    p->eig_scr = A.take<double>((size_t)nc * (2 * p->eig_nmax + 128));
    p->eig_cnt = A.take<unsigned int>(2 * nc + 1);
    if (p->opt.mode == JOLT_RANDOMIZED) {
      const int k = p->k;
      const size_t kk = (size_t)k * k;
      const jolt_layout& L = p->lay;
      const size_t full = (size_t)L.batch * L.n_layers * p->H * T * D;
      p->Xk = p->copy_k ? A.take<uint16_t>(full) : nullptr;
      p->Xv = p->copy_v ? A.take<uint16_t>(full) : nullptr;
      p->Wt = A.take<uint16_t>((size_t)nc * k * p->Ncmax);
      p->Yt = A.take<uint16_t>((size_t)nc * k * p->tp);
      p->Pt = A.take<uint16_t>((size_t)nc * p->rpad * p->kpad);
      p->Z = A.take<float>((size_t)nc * p->Ncmax * k);
      p->GW32 = A.take<float>((size_t)nc * kk);
      p->fgpart = A.take<float>((size_t)nc * p->fg_chunks * 128 * 128);
      p->Gz = A.take<double>(nc * kk); p->Rm = A.take<double>(nc * kk); p->P0 = A.take<double>(nc * kk);
      p->X1 = A.take<double>(nc * kk); p->MB = A.take<double>(nc * kk); p->eZ = A.take<double>(nc * kk);
      p->eVt = A.take<double>(nc * kk); p->ew = A.take<double>((size_t)nc * k);
      p->ework = A.take<double>((size_t)nc * 3 * k);
      p->eF = A.take<double>((size_t)nc * p->rmax_all * 5 * k);
      p->Rinv = A.take<double>((size_t)nc * kk);
      p->gram_part = A.take<double>((size_t)GRAM_SPLIT * nc * kk);
      p->RTk = A.take<double>((size_t)nc * kk);
      p->trs = nullptr;
      p->P64 = A.take<double>((size_t)nc * k * p->rmax_all);
      p->d_cl0 = A.take<int>(nc); p->d_cb = A.take<int>(nc); p->d_cLg = A.take<int>(nc);
      p->d_ckind = A.take<int>(nc); p->d_Nc = A.take<int>(nc); p->d_cis = A.take<int>(nc);
      p->d_utp = A.take<uint16_t*>(nc);
      p->d_jobs_rand = A.take<EighJob>(2 * nc);
    }
    // per-cell buffers
    std::vector<double*> GT(nc), ZT(nc), VtT(nc), wT(nc), Cd(nc), wD(nc), nsq(nc), tT(nc), tD(nc),
        Y(nc), CY(nc), VtY(nc), wY(nc), ZY(nc), Uf(nc), workT(nc), workD(nc), workY(nc), FT(nc), FY(nc);
    std::vector<uint16_t*> M(nc);
    const bool rnd = p->opt.mode == JOLT_RANDOMIZED;
    for (int i = 0; i < nc; ++i) {
      const HostCell& c = p->hc[i];
      const int n = c.nmin;
      const int64_t LH = (int64_t)c.Lg * p->H;
      if (!rnd) {
        GT[i] = A.take<double>((size_t)n * n);
        ZT[i] = A.take<double>((size_t)n * n);
        VtT[i] = A.take<double>((size_t)n * n);
        wT[i] = A.take<double>(n);
        workT[i] = A.take<double>(3 * n);
        FT[i] = A.take<double>((size_t)c.rmax * 5 * n);
        Uf[i] = (T > c.N) ? A.take<double>((size_t)c.rmax * T) : nullptr;
      } else {
        GT[i] = ZT[i] = VtT[i] = Uf[i] = workT[i] = FT[i] = nullptr;
        wT[i] = A.take<double>(c.nt);
      }
      Cd[i] = A.take<double>((size_t)D * D);
      wD[i] = A.take<double>(D);
      workD[i] = A.take<double>(3 * D);
      nsq[i] = A.take<double>(1);
      tT[i] = A.take<double>(c.nt + 1);
      tD[i] = A.take<double>(D + 1);
      Y[i] = A.take<double>((size_t)LH * c.rmax * D);
      CY[i] = A.take<double>((size_t)D * D);
      VtY[i] = A.take<double>((size_t)D * D);
      wY[i] = A.take<double>(D);
      ZY[i] = A.take<double>((size_t)D * D);
      workY[i] = A.take<double>(3 * D);
      FY[i] = A.take<double>((size_t)5 * D * D);
      M[i] = A.take<uint16_t>((size_t)LH * c.rmax * D);
    }
    if (pass == 0) {
      A.size = A.used + 4096;
      p->ws_alloc = dev_alloc(A.size, p->init_stream);
      if (!p->ws_alloc) { set_error("workspace allocation of %zu bytes failed", A.size); return JOLT_ERR_OOM; }
      A.base = reinterpret_cast<uint8_t*>(p->ws_alloc);
      continue;
    }
    // ---- fill device tables
    cudaStream_t s = p->init_stream;
    JOLT_CUDA_TRY(cudaMemsetAsync(p->d_status, 0, 4 * sizeof(int), s));
    std::vector<int> bits(8, 0);
    for (size_t i = 0; i < p->bits.size(); ++i) bits[i] = p->bits[i];
    std::vector<int64_t> rb(8, 0);
    for (size_t i = 0; i < p->rowbytes.size(); ++i) rb[i] = p->rowbytes[i];
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_bits, bits.data(), 8 * sizeof(int), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_rowbytes, rb.data(), 8 * sizeof(int64_t), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_rt, p->rt_grid.data(), p->rt_grid.size() * sizeof(int), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_rd, p->rd_grid.data(), p->rd_grid.size() * sizeof(int), cudaMemcpyHostToDevice, s));
    std::vector<CellRD> rdc(nc);
    std::vector<int> ntv(nc), rmaxv(nc), nlhv(nc);
    std::vector<EighJob> js(2 * nc), jf(nc);
    for (int i = 0; i < nc; ++i) {
      const HostCell& c = p->hc[i];
      rdc[i] = CellRD{c.Lg, p->H, T, D, c.n_rt, c.nt - 0, tT[i], tD[i]};
      ntv[i] = c.nt;
      rmaxv[i] = c.rmax;
      nlhv[i] = c.Lg * p->H;
      js[i] = EighJob{rnd ? 0 : c.nmin, 1, GT[i], wT[i], VtT[i], ZT[i], workT[i], FT[i]};
      js[nc + i] = EighJob{D, 0, Cd[i], wD[i], nullptr, nullptr, workD[i], nullptr};
      jf[i] = EighJob{D, 1, CY[i], wY[i], VtY[i], ZY[i], workY[i], FY[i]};
    }
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_rd_cells, rdc.data(), nc * sizeof(CellRD), cudaMemcpyHostToDevice, s));
    {
      std::vector<int4> ids(nc);
      for (int i = 0; i < nc; ++i)
        ids[i] = make_int4(p->hc[i].seq + p->opt.seq_base, p->hc[i].group + p->opt.group_base, p->hc[i].kind, 0);
      JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_ids, ids.data(), nc * sizeof(int4), cudaMemcpyHostToDevice, s));
      JOLT_CUDA_TRY(cudaStreamSynchronize(s));
    }
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_nt, ntv.data(), nc * sizeof(int), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_rmax, rmaxv.data(), nc * sizeof(int), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_nlh, nlhv.data(), nc * sizeof(int), cudaMemcpyHostToDevice, s));
    {
      std::vector<int> dv(nc, D);
      JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_Dn, dv.data(), nc * sizeof(int), cudaMemcpyHostToDevice, s));
      JOLT_CUDA_TRY(cudaStreamSynchronize(s));
    }
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_jobs_spec, js.data(), js.size() * sizeof(EighJob), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_jobs_fit, jf.data(), jf.size() * sizeof(EighJob), cudaMemcpyHostToDevice, s));
#define UP(dst, v) JOLT_CUDA_TRY(cudaMemcpyAsync(dst, v.data(), nc * sizeof(v[0]), cudaMemcpyHostToDevice, s))
#define UPI(dst, v) JOLT_CUDA_TRY(cudaMemcpyAsync(dst, v.data(), v.size() * sizeof(int), cudaMemcpyHostToDevice, s))
    UP(p->d_GT, GT); UP(p->d_ZT, ZT); UP(p->d_VtT, VtT); UP(p->d_wT, wT); UP(p->d_Cd, Cd);
    UP(p->d_wD, wD); UP(p->d_nsq, nsq); UP(p->d_tT, tT); UP(p->d_tD, tD); UP(p->d_Y, Y);
    UP(p->d_CY, CY); UP(p->d_VtY, VtY); UP(p->d_wY, wY); UP(p->d_ZY, ZY); UP(p->d_Uf, Uf);
    UP(p->d_M, M);
#undef UP
    p->h_tT = tT; p->h_tD = tD; p->h_wT = wT; p->h_wD = wD; p->h_nsq = nsq; p->h_M = M;
    if (rnd) {
      const int k = p->k;
      const size_t kk = (size_t)k * k;
      std::vector<int> l0v(nc), bv(nc), lgv(nc), kindv(nc), ncv(nc), cisv(nc);
      std::vector<EighJob> jr(2 * nc);
      for (int i = 0; i < nc; ++i) {
        const HostCell& c = p->hc[i];
        l0v[i] = c.l0; bv[i] = c.seq; lgv[i] = c.Lg; kindv[i] = c.kind; ncv[i] = c.N;
        cisv[i] = 2 * (c.group + p->opt.group_base) + c.kind;
        jr[i] = EighJob{k, 1, p->MB + i * kk, p->ew + (size_t)i * k, p->eVt + i * kk, p->eZ + i * kk,
                        p->ework + (size_t)i * 3 * k, p->eF + (size_t)i * p->rmax_all * 5 * k};
        jr[nc + i] = EighJob{D, 0, Cd[i], wD[i], nullptr, nullptr, workD[i], nullptr};
      }
      UPI(p->d_cl0, l0v); UPI(p->d_cb, bv); UPI(p->d_cLg, lgv); UPI(p->d_ckind, kindv);
      UPI(p->d_Nc, ncv); UPI(p->d_cis, cisv);
      JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_jobs_rand, jr.data(), jr.size() * sizeof(EighJob), cudaMemcpyHostToDevice, s));
      // bf16 operand buffers start at zero: padding rows/columns are read by the
      // tensor cores and must not hold NaN bit patterns
      JOLT_CUDA_TRY(cudaMemsetAsync(p->Wt, 0, (size_t)nc * k * p->Ncmax * 2, s));
      JOLT_CUDA_TRY(cudaMemsetAsync(p->Yt, 0, (size_t)nc * k * p->tp * 2, s));
      JOLT_CUDA_TRY(cudaMemsetAsync(p->Pt, 0, (size_t)nc * p->rpad * p->kpad * 2, s));
    }
    if (p->d_cs) {
      JOLT_TRY(launch_rope_table(T, D, (double)p->lay.rope_theta_k, p->d_cs, s));
      JOLT_TRY(launch_rope_tiled(p->d_cs, T, D, p->d_csq, s));
    }
    JOLT_TRY(launch_eps2(p->bits.data(), (int)p->bits.size(), p->G, p->d_eps2, p->d_fpart, s));
    JOLT_CUDA_TRY(cudaStreamSynchronize(s));
  }
  return JOLT_OK;
}

// Device descriptors of the cells for given K/V base pointers.
static jolt_status upload_cells(jolt_plan_s* p, const void* k, const void* v, cudaStream_t s) {
  const jolt_layout& L = p->lay;
  // descriptors depend only on the two base pointers: skip the copy when they
  // are those of the previous call (the copy comes from pinned memory, so it
  // never blocks the host on the stream)
  if (p->cdesc_valid && p->cdesc_k == k && p->cdesc_v == v) return JOLT_OK;
  if (!p->cdesc_pinned) {
    JOLT_CUDA_TRY(cudaMallocHost(&p->cdesc_pinned, p->ncells * sizeof(CellDesc)));
  } else {
    // the previous upload may still be in flight
    JOLT_CUDA_TRY(cudaStreamSynchronize(s));
  }
  p->cdesc.resize(p->ncells);
  const size_t esz = L.dtype == JOLT_F32 ? 4 : 2;
  for (int i = 0; i < p->ncells; ++i) {
    const HostCell& c = p->hc[i];
    CellDesc d{};
    const uint8_t* base = reinterpret_cast<const uint8_t*>(c.kind == 0 ? k : v);
    d.src = base ? base + ((int64_t)c.seq * L.stride_b + (int64_t)c.l0 * L.stride_l) * esz : nullptr;
    d.sl = L.stride_l; d.sh = L.stride_h; d.st = L.stride_t;
    d.Lg = c.Lg; d.H = p->H; d.T = p->T; d.D = p->D;
    d.kind = c.kind;
    d.rope = (c.kind == 0 && L.rope_theta_k > 0) ? 1 : 0;
    d.f32 = L.dtype == JOLT_F32;
    d.seq = c.seq;
    d.l0 = c.l0;
    d.nt = c.nt;
    d.rtmax = c.rmax;
    p->cdesc[i] = d;
  }
  memcpy(p->cdesc_pinned, p->cdesc.data(), p->ncells * sizeof(CellDesc));
  JOLT_CUDA_TRY(cudaMemcpyAsync(p->d_cells, p->cdesc_pinned, p->ncells * sizeof(CellDesc), cudaMemcpyHostToDevice, s));
  p->cdesc_valid = true;
  p->cdesc_k = k;
  p->cdesc_v = v;
  return JOLT_OK;
}

// Spectra of every cell: ||X||^2, feature Gram eigenvalues, token spectrum.
// Tensor maps of the bf16 compression targets (working copies or inputs).
static jolt_status x_maps(jolt_plan_s* p, const void* k_in, const void* v_in, umma::Maps& m) {
  const jolt_layout& L = p->lay;
  const int B = L.batch, Ln = L.n_layers, H = p->H, T = p->T, D = p->D;
  const int64_t ch = (int64_t)T * D, cl = ch * H, cb = cl * Ln;
  if (p->copy_k) JOLT_TRY(map_x5(&m.xk, p->Xk, B, Ln, H, T, D, cb, cl, ch, D));
  else JOLT_TRY(map_x5(&m.xk, k_in, B, Ln, H, T, D, L.stride_b, L.stride_l, L.stride_h, L.stride_t));
  if (p->copy_v) JOLT_TRY(map_x5(&m.xv, p->Xv, B, Ln, H, T, D, cb, cl, ch, D));
  else JOLT_TRY(map_x5(&m.xv, v_in, B, Ln, H, T, D, L.stride_b, L.stride_l, L.stride_h, L.stride_t));
  return JOLT_OK;
}

static umma::Problem gemm_problem(jolt_plan_s* p, int mode, int* status) {
  umma::Problem q{};
  q.mode = mode;
  q.ncells = p->ncells;
  q.H = p->H; q.D = p->D; q.T = p->T; q.t_pitch = p->tp; q.nbatch = p->lay.batch;
  q.cell_l0 = p->d_cl0; q.cell_b = p->d_cb; q.cell_Lg = p->d_cLg; q.cell_kind = p->d_ckind;
  q.status = status;
  return q;
}

// Section 3.1: sketch + power iterations on the feature side, then the
// spectrum of B B^T with the synthetic tail entry; also the feature Gram.
static jolt_status run_range_finder(jolt_plan_s* p, const void* k_in, const void* v_in, uint64_t seed,
                                    int* status, cudaStream_t s) {
  const jolt_layout& L = p->lay;
  const int nc = p->ncells, D = p->D, T = p->T, k = p->k;
  const int64_t kk = (int64_t)k * k;
  ProfScope ps_copy(JOLT_STAGE_COPY, s);
  if (p->copy_k)
    JOLT_TRY(launch_make_xb(k_in, L.dtype == JOLT_F32, L.rope_theta_k > 0, p->d_cs, L.batch, L.n_layers, p->H, T, D,
                            L.stride_b, L.stride_l, L.stride_h, L.stride_t, p->Xk, s));
  if (p->copy_v)
    JOLT_TRY(launch_make_xb(v_in, L.dtype == JOLT_F32, 0, p->d_cs, L.batch, L.n_layers, p->H, T, D,
                            L.stride_b, L.stride_l, L.stride_h, L.stride_t, p->Xv, s));
  ps_copy.end();
  umma::Maps m{};
  JOLT_TRY(x_maps(p, k_in, v_in, m));
  m.at = m.xk;
  m.bt = m.xk;
  // feature Gram (tensor cores, fp32 partials per row chunk, fp64 reduction)
  {
    ProfScope ps(JOLT_STAGE_FGRAM, s);
    umma::Problem q = gemm_problem(p, umma::FG, status);
    q.BN = 128; q.N = 128; q.mt = p->fg_chunks; q.nt = 1;
    q.fg_chunks = p->fg_chunks; q.fg_spc = p->fg_spc;
    q.out_f32 = p->fgpart;
    JOLT_TRY(launch_umma(m, q, s));
    JOLT_TRY(launch_fgram_reduce(p->fgpart, p->fg_chunks, D, p->d_Cd, p->d_nsq, nc, s));
  }
  // W_0^T = Omega^T
  JOLT_TRY(launch_omega(p->Wt, nc, k, p->Ncmax, p->d_Nc, p->d_cb, p->d_cis, seed, s));
  // B operand maps and N tiling of the pair passes (wide tiles when planned)
  auto pair_tiles = [&](umma::Maps& mm, umma::Problem& q, const void* bt, int cols, int64_t pitch,
                        bool wide) -> jolt_status {
    q.pair = p->gemm_pair;
    if (!wide) {
      q.BN = p->BN; q.nt = p->nt_k;
      return map_3d(&mm.bt, bt, nc, k, cols, pitch, p->gemm_pair ? p->BN / 2 : p->BN);
    }
    q.wide = 1; q.BN = p->wide_w0; q.nt = p->wide_nt;
    for (int j = 0; j < p->wide_nt; ++j) {
      q.tn0[j] = p->wtn0[j]; q.ta[j] = p->wta[j]; q.tb[j] = p->wtb[j];
      q.tmap_a[j] = p->wmap_a[j]; q.tmap_b[j] = p->wmap_b[j];
    }
    JOLT_TRY(map_3d(&mm.bt, bt, nc, k, cols, pitch, p->whb[0]));
    return map_3d(&mm.bt2, bt, nc, k, cols, pitch, p->whb[1]);
  };
  auto xw = [&]() -> jolt_status {
    ProfScope ps(JOLT_STAGE_GEMM_XW, s);
    umma::Maps mm = m;
    umma::Problem q = gemm_problem(p, umma::XW, status);
    JOLT_TRY(pair_tiles(mm, q, p->Wt, p->Ncmax, p->Ncmax, p->wide != 0));
    q.M = T; q.N = k; q.mt = (T + 127) / 128;
    q.out_bf16 = p->Yt; q.out_cell_stride = (int64_t)k * p->tp;
    return launch_umma(mm, q, s);
  };
  auto xty = [&]() -> jolt_status {
    ProfScope ps(JOLT_STAGE_GEMM_XTY, s);
    umma::Maps mm = m;
    umma::Problem q = gemm_problem(p, umma::XTY, status);
    JOLT_TRY(pair_tiles(mm, q, p->Yt, T, p->tp, p->wide != 0));
    q.M = p->Ncmax; q.N = k; q.Kdim = T; q.mt = (p->Ncmax + 127) / 128;
    q.out_f32 = p->Z; q.out_cell_stride = (int64_t)p->Ncmax * k;
    return launch_umma(mm, q, s);
  };
  JOLT_TRY(xw());
  for (int it = 0; it < p->opt.power_iters; ++it) {
    JOLT_TRY(xty());
    // V = Z R^{-1} with Z^T Z = R^T R (fp64), stored as the next W^T
    ProfScope ps(JOLT_STAGE_ORTH, s);
    JOLT_TRY(launch_gram_cols(p->Z, (int64_t)p->Ncmax * k, p->d_Nc, k, p->Gz, kk, nc, p->gram_part, s));
    JOLT_TRY(launch_chol_blocked(p->Gz, p->RTk, kk, nullptr, k, nc, status, s));
    JOLT_TRY(launch_tri_inverse(p->Gz, p->Rinv, p->RTk, kk, k, nc, s));
    TrsmArgs ta{};
    ta.Rinv = p->Rinv; ta.RinvT = p->RTk; ta.r_cell = kk; ta.k = k; ta.backward = 0;
    ta.B = p->Z; ta.b64 = 0; ta.b_cell = (int64_t)p->Ncmax * k; ta.ldb_r = k; ta.ldb_c = 1;
    ta.rows_of = p->d_Nc;
    ta.X16 = p->Wt; ta.x16_cell = (int64_t)k * p->Ncmax; ta.ld16_r = 1; ta.ld16_c = p->Ncmax;
    JOLT_TRY(launch_tri_apply(ta, p->Ncmax, nc, s));
    ps.end();
    JOLT_TRY(xw());
  }
  JOLT_TRY(xty());
  // G_W = W^T W (tensor cores) = R^T R
  {
    umma::Maps mm = m;
    JOLT_TRY(map_3d(&mm.at, p->Yt, nc, k, T, p->tp, 128));
    JOLT_TRY(map_3d(&mm.bt, p->Yt, nc, k, T, p->tp, p->BN));
    ProfScope ps(JOLT_STAGE_GEMM_GRAM, s);
    umma::Problem q = gemm_problem(p, umma::GRAM, status);
    q.M = k; q.N = k; q.Kdim = T; q.BN = p->BN; q.mt = (k + 127) / 128; q.nt = p->nt_k;
    q.out_f32 = p->GW32; q.out_cell_stride = kk;
    JOLT_TRY(launch_umma(mm, q, s));
  }
  ProfScope ps_eig(JOLT_STAGE_EIG, s);
  JOLT_TRY(launch_chol_blocked(p->Rm, p->RTk, kk, p->GW32, k, nc, status, s));
  JOLT_TRY(launch_tri_inverse(p->Rm, p->Rinv, p->RTk, kk, k, nc, s));
  // B B^T = R^{-T} (Z^T Z) R^{-1}: Y1 = P0 R^{-1}, then (Y1^T) R^{-1}
  JOLT_TRY(launch_gram_cols(p->Z, (int64_t)p->Ncmax * k, p->d_Nc, k, p->P0, kk, nc, p->gram_part, s));
  {
    TrsmArgs ta{};
    ta.Rinv = p->Rinv; ta.RinvT = p->RTk; ta.r_cell = kk; ta.k = k; ta.backward = 0;
    ta.B = p->P0; ta.b64 = 1; ta.b_cell = kk; ta.ldb_r = k; ta.ldb_c = 1; ta.rows_fixed = k;
    ta.X64 = p->X1; ta.x64_cell = kk; ta.ld64_r = k; ta.ld64_c = 1;
    JOLT_TRY(launch_tri_apply(ta, k, nc, s));
    ta.B = p->X1; ta.ldb_r = 1; ta.ldb_c = k;
    ta.X64 = p->MB;
    JOLT_TRY(launch_tri_apply(ta, k, nc, s));
    JOLT_TRY(launch_symmetrize(p->MB, kk, k, nc, s));
  }
  // spectra only here: eigenvectors follow the allocation (top r_T only)
  JOLT_TRY(launch_tridiag_multi(p->d_jobs_rand, nc, k, p->eig_scr, p->eig_cnt, status, s));
  JOLT_TRY(launch_tridiag(p->d_jobs_rand + nc, nc, D, s));
  JOLT_TRY(launch_bisect(p->d_jobs_rand, 2 * nc, std::max(k, D), s));
  JOLT_TRY(launch_rand_spectrum(p->ew, k, p->q_used, p->d_nsq, p->d_wT, nc, s));
  return JOLT_OK;
}

// U_T^ = bf16(W_q R^{-1} U_B[:, :r_T]) into the payload (tensor cores), and
// Y = (Z R^{-1} U_B[:, :r_T])^T for the feature factor.
static jolt_status run_random_fit(jolt_plan_s* p, const void* k_in, const void* v_in, CellOut* d_out, int* status,
                                  cudaStream_t s) {
  const int nc = p->ncells, T = p->T, k = p->k;
  const int64_t kk = (int64_t)k * k;
  ProfScope ps(JOLT_STAGE_FIT, s);
  JOLT_TRY(launch_copy_out(d_out, p->d_rT_used, p->d_utp, nc, s));
  {
    ProfScope pe(JOLT_STAGE_EIG, s);
    JOLT_TRY(launch_eigvecs_n(p->d_jobs_rand, nc, p->rmax_all, k, p->d_rT_used, s));
  }
  {
    // P = R^{-1} U_B[:, :r_T]: rows of P^T solve x R^T = u (backward)
    TrsmArgs ta{};
    ta.Rinv = p->Rinv; ta.RinvT = p->RTk; ta.r_cell = kk; ta.k = k; ta.backward = 1;
    ta.B = p->eVt; ta.b64 = 1; ta.b_cell = kk; ta.ldb_r = k; ta.ldb_c = 1;
    ta.rows_of = p->d_rT_used;
    ta.X64 = p->P64; ta.x64_cell = (int64_t)k * p->rmax_all; ta.ld64_r = 1; ta.ld64_c = p->rmax_all;
    ta.X16 = p->Pt; ta.x16_cell = (int64_t)p->rpad * p->kpad; ta.ld16_r = p->kpad; ta.ld16_c = 1;
    JOLT_TRY(launch_tri_apply(ta, p->rmax_all, nc, s));
  }
  umma::Maps m{};
  JOLT_TRY(x_maps(p, k_in, v_in, m));
  JOLT_TRY(map_3d(&m.at, p->Yt, nc, k, T, p->tp, 64));
  JOLT_TRY(map_3d(&m.bt, p->Pt, nc, p->rpad, p->kpad, p->kpad, 128));
  umma::Problem q = gemm_problem(p, umma::WP, status);
  q.M = T; q.N = p->rpad; q.Kdim = k; q.BN = 128; q.mt = (T + 127) / 128; q.nt = p->rpad / 128;
  q.wp_rows = p->d_rT_used; q.wp_dst = p->d_utp;
  JOLT_TRY(launch_umma(m, q, s));
  JOLT_TRY(launch_yproj(p->Z, (int64_t)p->Ncmax * k, p->P64, (int64_t)k * p->rmax_all, k, p->rmax_all, d_out,
                        p->d_nlh, p->d_Y, p->lh_max, p->D, nc, s));
  return JOLT_OK;
}

// Residual (k_in != NULL) or decoding pass on tensor cores: the backbone
// U_T^ M^_lh comes from the payload through two small re-layout kernels.
static jolt_status run_stream(jolt_plan_s* p, const jolt_handle_s* h, const void* k_in, const void* v_in,
                              void* k_out, void* v_out, const jolt_layout* ol, cudaStream_t s) {
  const bool compress = k_in != nullptr;
  const int nc = p->ncells, D = p->D;
  const jolt_layout& L = p->lay;
  JOLT_TRY(launch_m_transpose(h->d_out, p->d_cells, p->d_M, p->d_rmax, p->Mt_ws, p->lh_max, D, p->rpad_m, nc, s));
  JOLT_TRY(launch_ut_to_ws(h->d_out, p->Ut_ws, p->rows_u, p->tp, nc, s));
  StreamMaps m{};
  JOLT_TRY(map_3d_box(&m.ut, p->Ut_ws, nc, p->rows_u, p->tp, p->tp, 64, 64));
  JOLT_TRY(map_3d_box(&m.mt, p->Mt_ws, nc * p->lh_max, D, p->rpad_m, p->rpad_m, 64, D));
  if (compress) {
    JOLT_TRY(map_x5_box(&m.xk, k_in, L.batch, L.n_layers, p->H, p->T, D, L.stride_b, L.stride_l, L.stride_h,
                        L.stride_t, 128));
    JOLT_TRY(map_x5_box(&m.xv, v_in, L.batch, L.n_layers, p->H, p->T, D, L.stride_b, L.stride_l, L.stride_h,
                        L.stride_t, 128));
  } else {
    m.xk = m.ut;
    m.xv = m.ut;
  }
  StreamArgs a{};
  a.ncells = nc; a.T = p->T; a.H = p->H; a.lhmax = p->lh_max; a.rpad_m = p->rpad_m; a.G = p->G;
  a.cells = p->d_cells; a.outs = h->d_out; a.cs = p->d_cs; a.csq = p->d_csq; a.seed = h->seed;
  if (!compress) {
    a.out_k = reinterpret_cast<uint16_t*>(k_out);
    a.out_v = reinterpret_cast<uint16_t*>(v_out);
    a.osb = ol->stride_b; a.osl = ol->stride_l; a.osh = ol->stride_h; a.ost = ol->stride_t;
  }
  a.status = h->d_status;
  return launch_stream(compress, D, m, a, s);
}

static jolt_status run_spectra(jolt_plan_s* p, const void* k_in, const void* v_in, uint64_t seed, int* status,
                               cudaStream_t s) {
  const int nc = p->ncells, D = p->D;
  if (p->opt.mode == JOLT_EXACT) {
    ProfScope ps(JOLT_STAGE_FGRAM, s);
    JOLT_TRY(launch_fgram_x(p->d_cells, nc, D, p->d_cs, p->fchunk, p->d_fpart, s));
    JOLT_TRY(launch_sum_chunks(p->d_fpart, p->fchunk, D * D + 1, nc, p->d_Cd, p->d_nsq, s));
  }
  if (p->opt.mode == JOLT_EXACT) {
    {
      ProfScope ps(JOLT_STAGE_TOKEN_GRAM, s);
      JOLT_TRY(launch_token_gram(p->d_cells, nc, p->nmin_max, p->d_cs, p->d_GT, s));
    }
    // spectra only: the token eigenvectors follow the allocation (top r_T)
    ProfScope ps(JOLT_STAGE_EIG, s);
    JOLT_TRY(launch_tridiag_multi(p->d_jobs_spec, nc, p->nmin_max, p->eig_scr, p->eig_cnt, status, s));
    JOLT_TRY(launch_tridiag(p->d_jobs_spec + nc, nc, D, s));
    JOLT_TRY(launch_bisect(p->d_jobs_spec, 2 * nc, std::max(p->nmin_max, D), s));
  } else {
    JOLT_TRY(run_range_finder(p, k_in, v_in, seed, status, s));
  }
  ProfScope ps_rd(JOLT_STAGE_ALLOC, s);
  JOLT_TRY(launch_rd_tables(p->d_rd_cells, nc, p->d_wT, p->d_wD, nullptr, p->d_tT, p->d_tD, p->d_nt,
                            p->d_nsq, status, s));
  return JOLT_OK;
}

static jolt_status run_allocation(jolt_plan_s* p, int64_t budget, const double* eps2, AllocState* st_dev,
                                  Choice* out, int* status, cudaStream_t s) {
  AllocState st{};
  st.lo = 1e-30; st.hi = 1.0; st.lam = st.lo;
  st.tol = p->opt.budget_tol;
  st.budget = budget;
  st.max_iters = p->opt.max_iters;
  st.phase = 0;
  AllocArgs a{};
  a.greedy = p->opt.minimizer == JOLT_MIN_GREEDY;
  a.cells = p->d_rd_cells; a.ncells = p->ncells;
  a.rt_grid = p->d_rt; a.rd_grid = p->d_rd; a.n_rd = (int)p->rd_grid.size(); a.n_rt_max = (int)p->rt_grid.size();
  a.bits = p->d_bits; a.eps2 = eps2; a.rowbytes = p->d_rowbytes; a.n_bits = (int)p->bits.size();
  a.nchunk = p->achunk; a.pv = p->d_apv; a.pi = p->d_api; a.cur = p->d_cur; a.keep = p->d_keep;
  a.st = st_dev; a.out = out; a.status = status;
  return launch_alloc(a, st, s);
}

// Randomized mode reads K and V through TMA unless the plan makes working
// copies; a TMA tensor map needs a 16-byte-aligned base address.
static jolt_status check_tma_inputs(const jolt_plan_s* p, const void* k, const void* v) {
  if (p->opt.mode != JOLT_RANDOMIZED) return JOLT_OK;
  const bool bad_k = !p->copy_k && reinterpret_cast<uintptr_t>(k) % 16;
  const bool bad_v = !p->copy_v && reinterpret_cast<uintptr_t>(v) % 16;
  if (bad_k || bad_v) {
    set_error("randomized mode reads %s through TMA: its base pointer must be 16-byte aligned",
              bad_k ? "K" : "V");
    return JOLT_ERR_UNSUPPORTED_SHAPE;
  }
  return JOLT_OK;
}

extern "C" {

void jolt_free_plan(jolt_plan_t* p) {
  if (!p) return;
  if (p->cdesc_pinned) cudaFreeHost(p->cdesc_pinned);
  if (p->ws_alloc) dev_free(p->ws_alloc, p->init_stream);
  delete p;
}

// Phase 1 of a compression: a handle for this plan's cells, then the spectra
// and rate-distortion tables (the steps before the allocation).
static jolt_status compress_begin(jolt_plan_s* p, const void* k, const void* v, int64_t B, uint64_t seed,
                                  cudaStream_t s, jolt_handle_s** out) {
  int64_t minsum = 0, maxsum = 0, extra = 0;
  for (auto& c : p->hc) {
    minsum += c.min_bytes;
    maxsum += c.max_bytes;
    extra += 5 * 256 + (int64_t)c.rmax * 16;
  }
  if (B < minsum) { set_error("budget %lld below the cheapest allocation %lld", (long long)B, (long long)minsum); return JOLT_ERR_BUDGET_INFEASIBLE; }
  const int nc = p->ncells;
  auto* h = new jolt_handle_s();
  h->plan = p;
  h->stream = s;
  // sequence b of this plan is sequence seq_base + b of the whole cache: its
  // rotation (and sketch) are drawn from seed + seq_base + b
  h->seed = seed + (uint64_t)p->opt.seq_base;
  h->budget = B;
  // the cells' bytes never exceed the budget, nor their dearest options
  h->capacity = std::min(B, maxsum) + extra + 4096;
  Arena A;
  for (int pass = 0; pass < 2; ++pass) {
    A.used = 0;
    h->d_out = A.take<CellOut>(nc);
    h->d_choice = A.take<Choice>(nc);
    h->d_state = A.take<AllocState>(1);
    h->d_status = A.take<int>(4);
    h->payload = A.take<uint8_t>((size_t)h->capacity);
    if (pass == 0) {
      h->block = dev_alloc(A.used + 256, s);
      if (!h->block) { delete h; set_error("handle allocation failed"); return JOLT_ERR_OOM; }
      A.base = reinterpret_cast<uint8_t*>(h->block);
    }
  }
  auto fail = [&](jolt_status st) { jolt_free_handle(h); return st; };
  if (cudaMemsetAsync(h->d_status, 0, 4 * sizeof(int), s) != cudaSuccess) return fail(JOLT_ERR_CUDA);
  jolt_status st;
  if (p->opt.rotation == JOLT_ROT_QR_GAUSS) {
    const size_t qn = (size_t)p->lay.batch * p->D * p->D;
    h->qblock = dev_alloc(2 * qn * sizeof(double), s);
    if (!h->qblock) { set_error("rotation allocation failed"); return fail(JOLT_ERR_OOM); }
    h->d_qrot = reinterpret_cast<double*>(h->qblock) + qn;
    if ((st = launch_qr_rotation(p->D, p->lay.batch, h->seed, reinterpret_cast<double*>(h->qblock), h->d_qrot, s)) !=
        JOLT_OK)
      return fail(st);
  }
  if ((st = upload_cells(p, k, v, s)) != JOLT_OK) return fail(st);
  if ((st = run_spectra(p, k, v, h->seed, h->d_status, s)) != JOLT_OK) return fail(st);
  h->phase = 1;
  *out = h;
  return JOLT_OK;
}

// Phase 2: the allocation (over this plan's cells, or over gathered records
// of every process sharing the budget), then fit and residual of this plan's
// cells.
static jolt_status compress_end(jolt_handle_s* h, const void* k, const void* v, const uint8_t* recs, int n_total,
                                int first, cudaStream_t s) {
  jolt_plan_s* p = h->plan;
  const int nc = p->ncells;
  const uint64_t seed = h->seed;
  jolt_status st;
  {
    ProfScope ps(JOLT_STAGE_ALLOC, s);
    if (!recs) {
      JOLT_TRY(run_allocation(p, h->budget, p->d_eps2, h->d_state, h->d_choice, h->d_status, s));
    } else {
      // every cell's record: CellRD views, then the same bisection as above
      Arena A;
      CellRD* rd = nullptr; double* pv = nullptr; int* pi = nullptr; int* cur = nullptr; int* keep = nullptr;
      Choice* ch = nullptr; AllocState* ast = nullptr;
      void* blk = nullptr;
      for (int pass = 0; pass < 2; ++pass) {
        A.used = 0;
        rd = A.take<CellRD>(n_total);
        pv = A.take<double>((size_t)n_total * p->achunk);
        pi = A.take<int>((size_t)n_total * p->achunk);
        cur = A.take<int>(n_total);
        keep = A.take<int>(n_total);
        ch = A.take<Choice>(n_total);
        ast = A.take<AllocState>(1);
        if (pass == 0) {
          blk = dev_alloc(A.used + 256, s);
          if (!blk) { set_error("allocation scratch for %d cells failed", n_total); return JOLT_ERR_OOM; }
          A.base = reinterpret_cast<uint8_t*>(blk);
        }
      }
      auto run = [&]() -> jolt_status {
        JOLT_TRY(launch_records_to_rd(recs, n_total, p->rec_bytes, p->ntp, p->D, p->fingerprint,
                                      (int)p->rt_grid.size(), first, nc, p->d_ids, rd, h->d_status, s));
        AllocState st0{};
        st0.lo = 1e-30; st0.hi = 1.0; st0.lam = st0.lo;
        st0.tol = p->opt.budget_tol;
        st0.budget = h->budget;
        st0.max_iters = p->opt.max_iters;
        st0.phase = 0;
        AllocArgs a{};
        a.greedy = p->opt.minimizer == JOLT_MIN_GREEDY;
        a.cells = rd; a.ncells = n_total;
        a.rt_grid = p->d_rt; a.rd_grid = p->d_rd; a.n_rd = (int)p->rd_grid.size(); a.n_rt_max = (int)p->rt_grid.size();
        a.bits = p->d_bits; a.eps2 = p->d_eps2; a.rowbytes = p->d_rowbytes; a.n_bits = (int)p->bits.size();
        a.nchunk = p->achunk; a.pv = pv; a.pi = pi; a.cur = cur; a.keep = keep;
        a.st = ast; a.out = ch; a.status = h->d_status;
        JOLT_TRY(launch_alloc(a, st0, s));
        JOLT_CUDA_TRY(cudaMemcpyAsync(h->d_choice, ch + first, nc * sizeof(Choice), cudaMemcpyDeviceToDevice, s));
        JOLT_CUDA_TRY(cudaMemcpyAsync(h->d_state, ast, sizeof(AllocState), cudaMemcpyDeviceToDevice, s));
        return JOLT_OK;
      };
      st = run();
      dev_free(blk, s);
      if (st != JOLT_OK) return st;
    }
  }
  ProfScope ps_fit(JOLT_STAGE_FIT, s);
  JOLT_TRY(launch_payload_layout(p->d_cells, h->d_choice, nc, p->G, h->payload, h->capacity, h->d_out, h->d_status, s));
  FitArgs fa{};
  fa.cells = p->d_cells; fa.cs = p->d_cs; fa.out = h->d_out; fa.ncells = nc; fa.D = p->D;
  fa.VtT = p->d_VtT; fa.wT = p->d_wT; fa.Uf = p->d_Uf; fa.Y = p->d_Y; fa.rmax_of = p->d_rmax;
  fa.VtY = p->d_VtY; fa.M = p->d_M;
  if (p->opt.mode == JOLT_EXACT) {
    JOLT_TRY(launch_copy_rt(h->d_out, p->d_rT_used, nc, s));
    {
      ProfScope pe(JOLT_STAGE_EIG, s);
      JOLT_TRY(launch_eigvecs_n(p->d_jobs_spec, nc, p->rmax_all, p->nmin_max, p->d_rT_used, s));
    }
    JOLT_TRY(launch_ut_exact(fa, p->T, p->rmax_all, s));
    JOLT_TRY(launch_project_y(fa, p->T, p->rmax_all, p->lh_max, s));
  } else {
    JOLT_TRY(run_random_fit(p, k, v, h->d_out, h->d_status, s));
  }
  // feature Gram of Y (rows r < r_T), then its eigenvectors
  JOLT_TRY(launch_copy_rt(h->d_out, p->d_rT_used, nc, s));
  JOLT_TRY(launch_fgram_rows(p->d_Y, p->d_rT_used, p->d_rmax, p->d_nlh, nc, p->D, p->fchunk, p->d_fpart, s));
  JOLT_TRY(launch_sum_chunks(p->d_fpart, p->fchunk, p->D * p->D + 1, nc, p->d_CY, nullptr, s));
  JOLT_TRY(launch_tridiag(p->d_jobs_fit, nc, p->D, s));
  JOLT_TRY(launch_bisect(p->d_jobs_fit, nc, p->D, s));
  JOLT_TRY(launch_eigvecs_n(p->d_jobs_fit, nc, p->D, p->D, p->d_Dn, s));
  JOLT_TRY(launch_core(fa, p->rmax_all, p->lh_max, s));
  ResidArgs ra{};
  ra.cells = p->d_cells; ra.cs = p->d_cs; ra.out = h->d_out; ra.M = p->d_M; ra.rmax_of = p->d_rmax;
  ra.G = p->G; ra.seed = seed; ra.qrot = h->d_qrot;
  ps_fit.end();
  ProfScope ps_res(JOLT_STAGE_RESIDUAL, s);
  // the tensor-core stream kernel implements the Hadamard rotation only
  if (p->tc_in && !h->d_qrot && reinterpret_cast<uintptr_t>(k) % 16 == 0 && reinterpret_cast<uintptr_t>(v) % 16 == 0) {
    JOLT_TRY(run_stream(p, h, k, v, nullptr, nullptr, nullptr, s));
  } else {
    JOLT_TRY(launch_residual_simt(ra, nc, p->D, p->T, p->lh_max, s));
  }
  h->phase = 2;
  return JOLT_OK;
}

jolt_status jolt_compress(jolt_plan_t* p, const void* k, const void* v, int64_t byte_budget,
                          uint64_t seed, jolt_stream_t stream_, jolt_handle_t** out) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!p || !k || !v || !out) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  *out = nullptr;
  JOLT_TRY(check_tma_inputs(p, k, v));
  jolt_handle_s* h = nullptr;
  JOLT_TRY(compress_begin(p, k, v, byte_budget > 0 ? byte_budget : p->budget, seed, s, &h));
  jolt_status st = compress_end(h, k, v, nullptr, p->ncells, 0, s);
  if (st != JOLT_OK) { jolt_free_handle(h); return st; }
  *out = h;
  return JOLT_OK;
}

int64_t jolt_summary_bytes(const jolt_plan_t* p) { return p ? (int64_t)p->rec_bytes : 0; }

jolt_status jolt_compress_begin(jolt_plan_t* p, const void* k, const void* v, int64_t byte_budget, uint64_t seed,
                                void* summary_dev, jolt_stream_t stream_, jolt_handle_t** out) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!p || !k || !v || !out || !summary_dev) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  *out = nullptr;
  if (reinterpret_cast<uintptr_t>(summary_dev) % 16) { set_error("summary_dev must be 16-byte aligned"); return JOLT_ERR_INVALID_ARG; }
  JOLT_TRY(check_tma_inputs(p, k, v));
  jolt_handle_s* h = nullptr;
  JOLT_TRY(compress_begin(p, k, v, byte_budget > 0 ? byte_budget : p->budget, seed, s, &h));
  h->k_in = k;
  h->v_in = v;
  jolt_status st = launch_write_records(p->d_rd_cells, p->ncells, p->d_nsq, p->d_ids, p->fingerprint, p->ntp,
                                        p->rec_bytes, reinterpret_cast<uint8_t*>(summary_dev), s);
  if (st != JOLT_OK) { jolt_free_handle(h); return st; }
  *out = h;
  return JOLT_OK;
}

jolt_status jolt_compress_end(jolt_handle_t* h, const void* all_dev, int32_t n_total, int32_t first_cell,
                              jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!h || !all_dev) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  if (h->phase != 1) { set_error("jolt_compress_end needs a handle from jolt_compress_begin that has not ended"); return JOLT_ERR_INVALID_ARG; }
  const int nc = h->plan->ncells;
  if (n_total < nc || first_cell < 0 || first_cell > n_total - nc) {
    set_error("this plan's %d cells must lie inside the %d gathered records (first_cell %d)", nc, n_total, first_cell);
    return JOLT_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(all_dev) % 16) { set_error("all_summaries_dev must be 16-byte aligned"); return JOLT_ERR_INVALID_ARG; }
  h->stream = s;
  return compress_end(h, h->k_in, h->v_in, reinterpret_cast<const uint8_t*>(all_dev), n_total, first_cell, s);
}

jolt_status jolt_decompress(const jolt_handle_t* h, void* k_out, void* v_out, const jolt_layout* ol,
                            jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!h || !k_out || !v_out) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  if (h->phase != 2) { set_error("the handle's compression has not ended (jolt_compress_end)"); return JOLT_ERR_INVALID_ARG; }
  jolt_plan_s* p = h->plan;
  const jolt_layout& L = ol ? *ol : p->lay;
  if (L.batch != p->lay.batch || L.n_layers != p->lay.n_layers || L.n_heads != p->H || L.seq_len != p->T ||
      L.head_dim != p->D) { set_error("output layout shape differs from the plan"); return JOLT_ERR_INVALID_ARG; }
  if (L.stride_t < p->D || (L.stride_t % 2) || (L.stride_h % 2) || (L.stride_l % 2) || (L.stride_b % 2)) {
    set_error("output strides must be even and stride_t >= head_dim"); return JOLT_ERR_UNSUPPORTED_SHAPE;
  }
  const int nc = p->ncells;
  ProfScope ps(JOLT_STAGE_DECOMPRESS, s);
  JOLT_TRY(launch_core_m(h->d_out, p->d_cells, p->d_M, p->d_rmax, nc, p->D, p->rmax_all, p->lh_max, s));
  ResidArgs ra{};
  ra.cells = p->d_cells; ra.cs = p->d_cs; ra.out = h->d_out; ra.M = p->d_M; ra.rmax_of = p->d_rmax;
  ra.G = p->G; ra.seed = h->seed; ra.qrot = h->d_qrot;
  ra.out_k = reinterpret_cast<uint16_t*>(k_out); ra.out_v = reinterpret_cast<uint16_t*>(v_out);
  ra.osb = L.stride_b; ra.osl = L.stride_l; ra.osh = L.stride_h; ra.ost = L.stride_t;
  const bool tc_out = L.stride_t % 8 == 0 && L.stride_h % 8 == 0 && L.stride_l % 8 == 0 && L.stride_b % 8 == 0 &&
                      (reinterpret_cast<uintptr_t>(k_out) % 16) == 0 && (reinterpret_cast<uintptr_t>(v_out) % 16) == 0;
  if (tc_out && !h->d_qrot) JOLT_TRY(run_stream(p, h, nullptr, nullptr, k_out, v_out, &L, s));
  else JOLT_TRY(launch_decompress_simt(ra, nc, p->D, p->T, p->lh_max, s));
  return JOLT_OK;
}

static jolt_status handle_sync(const jolt_handle_t* h) {
  if (h->phase != 2) { set_error("the handle's compression has not ended (jolt_compress_end)"); return JOLT_ERR_INVALID_ARG; }
  JOLT_CUDA_TRY(cudaStreamSynchronize(h->stream));
  int st = 0;
  JOLT_CUDA_TRY(cudaMemcpy(&st, h->d_status, sizeof(int), cudaMemcpyDeviceToHost));
  return status_from_dev(st);
}

jolt_status jolt_bytes(const jolt_handle_t* h, int64_t* nbytes) {
  if (!h || !nbytes) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  JOLT_TRY(handle_sync(h));
  std::vector<Choice> ch(h->plan->ncells);
  JOLT_CUDA_TRY(cudaMemcpy(ch.data(), h->d_choice, ch.size() * sizeof(Choice), cudaMemcpyDeviceToHost));
  int64_t s = 0;
  for (auto& c : ch) s += c.bytes;
  *nbytes = s;
  return JOLT_OK;
}

jolt_status jolt_handle_info(const jolt_handle_t* h, jolt_cell_info* cells, int32_t n, double* lambda,
                             int32_t* iterations) {
  if (!h) { set_error("null handle"); return JOLT_ERR_INVALID_ARG; }
  jolt_plan_s* p = h->plan;
  if (cells && n < p->ncells) { set_error("need room for %d cells", p->ncells); return JOLT_ERR_INVALID_ARG; }
  JOLT_TRY(handle_sync(h));
  std::vector<Choice> ch(p->ncells);
  JOLT_CUDA_TRY(cudaMemcpy(ch.data(), h->d_choice, ch.size() * sizeof(Choice), cudaMemcpyDeviceToHost));
  AllocState st;
  JOLT_CUDA_TRY(cudaMemcpy(&st, h->d_state, sizeof(st), cudaMemcpyDeviceToHost));
  if (cells) {
    for (int i = 0; i < p->ncells; ++i) {
      const HostCell& c = p->hc[i];
      double nsq = 0.0;
      JOLT_CUDA_TRY(cudaMemcpy(&nsq, p->h_nsq[i], sizeof(double), cudaMemcpyDeviceToHost));
      cells[i] = jolt_cell_info{c.seq + p->opt.seq_base, c.group + p->opt.group_base, c.kind, ch[i].rT, ch[i].rd,
                                ch[i].b, ch[i].bytes, ch[i].err, nsq};
    }
  }
  if (lambda) *lambda = st.lam_final;
  if (iterations) *iterations = st.iters_final;
  return JOLT_OK;
}

jolt_status jolt_handle_cell(const jolt_handle_t* h, int32_t cell, jolt_cell_view* v) {
  if (!h || !v) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  jolt_plan_s* p = h->plan;
  if (cell < 0 || cell >= p->ncells) { set_error("cell %d out of range", cell); return JOLT_ERR_INVALID_ARG; }
  JOLT_TRY(handle_sync(h));
  CellOut o;
  JOLT_CUDA_TRY(cudaMemcpy(&o, h->d_out + cell, sizeof(o), cudaMemcpyDeviceToHost));
  const HostCell& c = p->hc[cell];
  *v = jolt_cell_view{o.rT, o.rd, o.b, p->G, c.Lg, p->H, p->T, p->D, o.t_pitch,
                      o.ut, o.ud, o.core, o.codes, o.scales};
  return JOLT_OK;
}

void jolt_free_handle(jolt_handle_t* h) {
  if (!h) return;
  if (h->block) dev_free(h->block, h->stream);
  if (h->qblock) dev_free(h->qblock, h->stream);
  delete h;
}

jolt_status jolt_rd_table(jolt_plan_t* p, const void* k, const void* v, double* norm_sq, double* sig_t,
                          int32_t max_t, int32_t* n_t, double* sig_d, jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!p || !k || !v || !norm_sq || !sig_t || !n_t || !sig_d) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  if (max_t < p->nt_max) { set_error("max_t must be >= %d", p->nt_max); return JOLT_ERR_INVALID_ARG; }
  JOLT_TRY(check_tma_inputs(p, k, v));
  JOLT_CUDA_TRY(cudaMemsetAsync(p->d_status, 0, sizeof(int), s));
  JOLT_TRY(upload_cells(p, k, v, s));
  JOLT_TRY(run_spectra(p, k, v, (uint64_t)p->opt.seq_base, p->d_status, s));
  JOLT_CUDA_TRY(cudaStreamSynchronize(s));
  int st = 0;
  JOLT_CUDA_TRY(cudaMemcpy(&st, p->d_status, sizeof(int), cudaMemcpyDeviceToHost));
  JOLT_TRY(status_from_dev(st));
  for (int i = 0; i < p->ncells; ++i) {
    const HostCell& c = p->hc[i];
    JOLT_CUDA_TRY(cudaMemcpy(norm_sq + i, p->h_nsq[i], sizeof(double), cudaMemcpyDeviceToHost));
    std::fill(sig_t + (size_t)i * max_t, sig_t + (size_t)(i + 1) * max_t, 0.0);
    JOLT_CUDA_TRY(cudaMemcpy(sig_t + (size_t)i * max_t, p->h_wT[i], c.nt * sizeof(double), cudaMemcpyDeviceToHost));
    JOLT_CUDA_TRY(cudaMemcpy(sig_d + (size_t)i * p->D, p->h_wD[i], p->D * sizeof(double), cudaMemcpyDeviceToHost));
  }
  *n_t = p->nt_max;
  return JOLT_OK;
}

jolt_status jolt_allocate(jolt_plan_t* p, const double* t_t, int32_t ld_t, const double* t_d, int32_t ld_d,
                          const double* eps2, int64_t byte_budget, int32_t* choice, int64_t* bytes,
                          double* lambda, int32_t* iterations, jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!p || !t_t || !t_d || !eps2 || !choice || !bytes) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  if (ld_t < p->nt_max + 1 || ld_d < p->D + 1) { set_error("ld_t >= %d and ld_d >= %d required", p->nt_max + 1, p->D + 1); return JOLT_ERR_INVALID_ARG; }
  const int nc = p->ncells;
  for (int i = 0; i < nc; ++i) {
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->h_tT[i], t_t + (size_t)i * ld_t, (p->hc[i].nt + 1) * sizeof(double), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(p->h_tD[i], t_d + (size_t)i * ld_d, (p->D + 1) * sizeof(double), cudaMemcpyHostToDevice, s));
  }
  double* d_e = p->d_fpart;     // scratch for the given eps^2
  JOLT_CUDA_TRY(cudaMemcpyAsync(d_e, eps2, p->bits.size() * sizeof(double), cudaMemcpyHostToDevice, s));
  AllocState* d_st = reinterpret_cast<AllocState*>(p->d_fpart + 16);
  Choice* d_out = reinterpret_cast<Choice*>(p->d_fpart + 64);
  JOLT_CUDA_TRY(cudaMemsetAsync(p->d_status, 0, sizeof(int), s));
  JOLT_TRY(run_allocation(p, byte_budget, d_e, d_st, d_out, p->d_status, s));
  JOLT_CUDA_TRY(cudaStreamSynchronize(s));
  int st = 0;
  JOLT_CUDA_TRY(cudaMemcpy(&st, p->d_status, sizeof(int), cudaMemcpyDeviceToHost));
  std::vector<Choice> ch(nc);
  JOLT_CUDA_TRY(cudaMemcpy(ch.data(), d_out, nc * sizeof(Choice), cudaMemcpyDeviceToHost));
  AllocState hs;
  JOLT_CUDA_TRY(cudaMemcpy(&hs, d_st, sizeof(hs), cudaMemcpyDeviceToHost));
  for (int i = 0; i < nc; ++i) {
    choice[3 * i] = ch[i].rT; choice[3 * i + 1] = ch[i].rd; choice[3 * i + 2] = ch[i].b;
    bytes[i] = ch[i].bytes;
  }
  if (lambda) *lambda = hs.lam_final;
  if (iterations) *iterations = hs.iters_final;
  return status_from_dev(st);
}

jolt_status jolt_eps2(const int32_t* bits, int32_t n, int32_t group, double* eps2, jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!bits || !eps2 || n < 1 || n > 8) { set_error("bad arguments"); return JOLT_ERR_INVALID_ARG; }
  for (int i = 0; i < n; ++i)
    if (!(bits[i] == 0 || bits[i] == 2 || bits[i] == 3 || bits[i] == 4 || bits[i] == 8)) { set_error("bad bit width"); return JOLT_ERR_INVALID_ARG; }
  if (!(group == 32 || group == 64 || group == 128)) { set_error("group must be 32, 64 or 128"); return JOLT_ERR_INVALID_ARG; }
  size_t nblk = ((1 << 20) / group + 255) / 256;
  double* buf = reinterpret_cast<double*>(dev_alloc((nblk * 9 + 16) * sizeof(double), s));
  if (!buf) { set_error("allocation failed"); return JOLT_ERR_OOM; }
  jolt_status st = launch_eps2(bits, n, group, buf, buf + 16, s);
  if (st == JOLT_OK) {
    if (cudaMemcpyAsync(eps2, buf, n * sizeof(double), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) { set_error("copy failed"); st = JOLT_ERR_CUDA; }
  }
  dev_free(buf, s);
  return st;
}

static jolt_status check_rows(int32_t D, int32_t bits, int32_t group) {
  if (D != 64 && D != 128) { set_error("D must be 64 or 128"); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) { set_error("bits must be 2, 3, 4 or 8"); return JOLT_ERR_INVALID_ARG; }
  if (!(group == 32 || group == 64 || group == D) || D % group) { set_error("bad group"); return JOLT_ERR_INVALID_ARG; }
  return JOLT_OK;
}

jolt_status jolt_residual_encode(const float* e, int64_t rows, int32_t D, int32_t bits, int32_t group,
                                 uint64_t seed, uint8_t* codes, float* scales, jolt_stream_t stream_) {
  JOLT_TRY(check_rows(D, bits, group));
  if (rows < 0 || (rows > 0 && (!e || !codes || !scales))) { set_error("bad arguments"); return JOLT_ERR_INVALID_ARG; }
  return launch_encode_rows(e, rows, D, bits, group, seed, codes, scales, (cudaStream_t)stream_);
}

jolt_status jolt_residual_decode(const uint8_t* codes, const float* scales, int64_t rows, int32_t D,
                                 int32_t bits, int32_t group, uint64_t seed, float* e_hat,
                                 jolt_stream_t stream_) {
  JOLT_TRY(check_rows(D, bits, group));
  if (rows < 0 || (rows > 0 && (!e_hat || !codes || !scales))) { set_error("bad arguments"); return JOLT_ERR_INVALID_ARG; }
  return launch_decode_rows(codes, scales, rows, D, bits, group, seed, e_hat, (cudaStream_t)stream_);
}

}  // extern "C"

// ------------------------------------------------------ single-stage hooks --
extern "C" {

jolt_status jolt_sketch(jolt_plan_t* p, uint64_t seed, uint16_t* omega_t, int32_t* k_out, int32_t* ld_out,
                        jolt_stream_t stream_) {
  if (!p) { set_error("null plan"); return JOLT_ERR_INVALID_ARG; }
  if (p->opt.mode != JOLT_RANDOMIZED) { set_error("the plan is not in JOLT_RANDOMIZED mode: it draws no sketch"); return JOLT_ERR_INVALID_ARG; }
  if (k_out) *k_out = p->k;
  if (ld_out) *ld_out = p->Ncmax;
  if (!omega_t) return JOLT_OK;
  if (reinterpret_cast<uintptr_t>(omega_t) % 8) { set_error("omega_t must be 8-byte aligned"); return JOLT_ERR_INVALID_ARG; }
  return launch_omega(omega_t, p->ncells, p->k, p->Ncmax, p->d_Nc, p->d_cb, p->d_cis, seed + (uint64_t)p->opt.seq_base,
                      (cudaStream_t)stream_);
}

jolt_status jolt_residual_stream_encode(const void* x, int32_t LH, int32_t T, int32_t D, const uint16_t* ut_t,
                                        int32_t r, const uint16_t* m, int32_t bits, int32_t group, uint64_t seed,
                                        float rope_theta, uint8_t* codes, float* scales, jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  JOLT_TRY(check_rows(D, bits, group));
  if (!x || !ut_t || !m || !codes || !scales) { set_error("null pointer"); return JOLT_ERR_INVALID_ARG; }
  if (LH < 1 || T < 1 || r < 1 || r > 512 || !(rope_theta >= 0.0f)) {
    set_error("need LH >= 1, T >= 1, 1 <= r <= 512 and rope_theta >= 0"); return JOLT_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(codes) % 16 ||
      reinterpret_cast<uintptr_t>(scales) % 16) {
    set_error("x, codes and scales must be 16-byte aligned"); return JOLT_ERR_UNSUPPORTED_SHAPE;
  }
  const int tp = (T + 7) / 8 * 8, rows = (r + 63) / 64 * 64;
  Arena A;
  CellDesc* d_cell = nullptr; CellOut* d_out = nullptr; uint16_t** d_M = nullptr; int* d_rmax = nullptr;
  int* d_status = nullptr; uint16_t* ut_ws = nullptr; uint16_t* mt_ws = nullptr; float2* cs = nullptr;
  float4* csq = nullptr;
  void* block = nullptr;
  for (int pass = 0; pass < 2; ++pass) {
    A.used = 0;
    d_cell = A.take<CellDesc>(1);
    d_out = A.take<CellOut>(1);
    d_M = A.take<uint16_t*>(1);
    d_rmax = A.take<int>(1);
    d_status = A.take<int>(4);
    ut_ws = A.take<uint16_t>((size_t)rows * tp);
    mt_ws = A.take<uint16_t>((size_t)LH * D * rows);
    cs = rope_theta > 0.0f ? A.take<float2>((size_t)T * (D / 2)) : nullptr;
    csq = rope_theta > 0.0f ? A.take<float4>((size_t)((T + 127) / 128) * 128 * (D / 4)) : nullptr;
    if (pass == 0) {
      block = dev_alloc(A.used + 256, s);
      if (!block) { set_error("scratch allocation failed"); return JOLT_ERR_OOM; }
      A.base = reinterpret_cast<uint8_t*>(block);
    }
  }
  jolt_status st = JOLT_OK;
  auto run = [&]() -> jolt_status {
    CellDesc c{};
    c.src = x; c.sl = (int64_t)LH * T * D; c.sh = (int64_t)T * D; c.st = D;
    c.Lg = 1; c.H = LH; c.T = T; c.D = D; c.kind = 0; c.rope = rope_theta > 0.0f; c.f32 = 0;
    c.seq = 0; c.l0 = 0; c.nt = 0; c.rtmax = r;
    CellOut o{};
    o.ut = const_cast<uint16_t*>(ut_t); o.codes = codes; o.scales = scales;
    o.rT = r; o.rd = D; o.b = bits; o.t_pitch = T;
    uint16_t* mp = const_cast<uint16_t*>(m);
    JOLT_CUDA_TRY(cudaMemcpyAsync(d_cell, &c, sizeof(c), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(d_out, &o, sizeof(o), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(d_M, &mp, sizeof(mp), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemcpyAsync(d_rmax, &r, sizeof(int), cudaMemcpyHostToDevice, s));
    JOLT_CUDA_TRY(cudaMemsetAsync(d_status, 0, 4 * sizeof(int), s));
    if (cs) {
      JOLT_TRY(launch_rope_table(T, D, (double)rope_theta, cs, s));
      JOLT_TRY(launch_rope_tiled(cs, T, D, csq, s));
    }
    JOLT_TRY(launch_m_transpose(d_out, d_cell, d_M, d_rmax, mt_ws, LH, D, rows, 1, s));
    JOLT_TRY(launch_ut_to_ws(d_out, ut_ws, rows, tp, 1, s));
    StreamMaps mp4{};
    JOLT_TRY(map_3d_box(&mp4.ut, ut_ws, 1, rows, tp, tp, 64, 64));
    JOLT_TRY(map_3d_box(&mp4.mt, mt_ws, LH, D, rows, rows, 64, D));
    JOLT_TRY(map_x5_box(&mp4.xk, x, 1, 1, LH, T, D, c.sl, c.sl, c.sh, c.st, 128));
    mp4.xv = mp4.xk;
    StreamArgs a{};
    a.ncells = 1; a.T = T; a.H = LH; a.lhmax = LH; a.rpad_m = rows; a.G = group;
    a.cells = d_cell; a.outs = d_out; a.cs = cs; a.csq = csq; a.seed = seed; a.status = d_status;
    JOLT_TRY(launch_stream(true, D, mp4, a, s));
    // the host structures above are read by copies still in flight: wait
    JOLT_CUDA_TRY(cudaStreamSynchronize(s));
    int dst = 0;
    JOLT_CUDA_TRY(cudaMemcpy(&dst, d_status, sizeof(int), cudaMemcpyDeviceToHost));
    return status_from_dev(dst);
  };
  st = run();
  cudaStreamSynchronize(s);
  dev_free(block, s);
  return st;
}

}  // extern "C"

// ----------------------------------------------------- decode attention ----
extern "C" jolt_status jolt_decode_attention(const jolt_handle_t* hc, int32_t layer, const float* q,
                                             int32_t n_q_heads, const uint16_t* tail_k, const uint16_t* tail_v,
                                             int32_t n_tail, float* out, jolt_stream_t stream_) {
  cudaStream_t s = (cudaStream_t)stream_;
  if (!hc || !q || !out) { set_error("null argument"); return JOLT_ERR_INVALID_ARG; }
  jolt_handle_s* h = const_cast<jolt_handle_s*>(hc);
  if (h->phase != 2) { set_error("the handle's compression has not ended (jolt_compress_end)"); return JOLT_ERR_INVALID_ARG; }
  jolt_plan_s* p = h->plan;
  const jolt_layout& L = p->lay;
  if (layer < 0 || layer >= L.n_layers) { set_error("layer %d out of range", layer); return JOLT_ERR_INVALID_ARG; }
  if (n_q_heads < p->H || n_q_heads % p->H || n_q_heads / p->H > 8) {
    set_error("n_q_heads must be 1..8 times the %d KV heads", p->H); return JOLT_ERR_INVALID_ARG;
  }
  if (n_tail < 0 || n_tail > 1024 || (n_tail > 0 && (!tail_k || !tail_v))) {
    set_error("n_tail must be 0..1024, with both tail tensors when positive"); return JOLT_ERR_INVALID_ARG;
  }
  if (h->d_qrot) { set_error("fused decode attention implements the Hadamard rotation only"); return JOLT_ERR_UNSUPPORTED_SHAPE; }
  if (reinterpret_cast<uintptr_t>(q) % 16) { set_error("q must be 16-byte aligned"); return JOLT_ERR_INVALID_ARG; }
  // the cells' layout on the host, read once per handle
  if (h->h_out.empty()) {
    JOLT_CUDA_TRY(cudaStreamSynchronize(h->stream));
    h->h_out.resize(p->ncells);
    JOLT_CUDA_TRY(cudaMemcpy(h->h_out.data(), h->d_out, p->ncells * sizeof(CellOut), cudaMemcpyDeviceToHost));
  }
  int g = 0;
  while (g + 1 < L.n_groups && p->gstart[g + 1] <= layer) ++g;
  const int li = layer - p->gstart[g];
  const int H = p->H, D = p->D, G = n_q_heads / H;
  for (int b0 = 0; b0 < L.batch; b0 += DEC_BMAX) {
    const int Bc = std::min(DEC_BMAX, L.batch - b0);
    std::vector<CellOut> ko(Bc), vo(Bc);
    int rk = 1, rv = 1;
    DecodeCall c{};
    for (int b = 0; b < Bc; ++b) {
      ko[b] = h->h_out[((b0 + b) * L.n_groups + g) * 2 + 0];
      vo[b] = h->h_out[((b0 + b) * L.n_groups + g) * 2 + 1];
      rk = std::max(rk, ko[b].rT);
      rv = std::max(rv, vo[b].rT);
      c.ut[b] = ko[b].ut;
      c.rt_k[b] = ko[b].rT;
      c.tpitch[b] = ko[b].t_pitch;
      c.uv[b] = vo[b].ut;
      c.rt_v[b] = vo[b].rT;
      c.tpitch_v[b] = vo[b].t_pitch;
    }
    if (rv > 512) {
      // the rank-space value state holds at most four blocks of 128 ranks
      set_error("fused decode attention needs the value cells' r_T <= 512 (layer %d has %d)", layer, rv);
      return JOLT_ERR_UNSUPPORTED_SHAPE;
    }
    const int rpk = (rk + 63) / 64 * 64, rpv = (rv + 63) / 64 * 64;
    const int64_t part_len = (int64_t)Bc * H * 64 * G * (2 + rpv + D);
    Arena A;
    uint16_t* mtk = nullptr; float* mv = nullptr; float* part = nullptr;
    void* blk = nullptr;
    for (int pass = 0; pass < 2; ++pass) {
      A.used = 0;
      mtk = A.take<uint16_t>((size_t)Bc * H * D * rpk);
      mv = A.take<float>((size_t)Bc * H * rpv * D);
      part = A.take<float>((size_t)part_len);
      if (pass == 0) {
        blk = dev_alloc(A.used + 256, s);
        if (!blk) { set_error("decode attention workspace allocation failed"); return JOLT_ERR_OOM; }
        A.base = reinterpret_cast<uint8_t*>(blk);
      }
    }
    auto run = [&]() -> jolt_status {
      // the handle's own cell records, read in place: sequence b's cells of
      // group g are 2 * n_groups records apart
      c.B = Bc; c.H = H; c.D = D; c.T = p->T; c.G = G; c.gq = p->G; c.li = li;
      c.kout = h->d_out + ((int64_t)b0 * L.n_groups + g) * 2;
      c.vout = c.kout + 1;
      c.cstride = 2 * L.n_groups;
      c.cs = (L.rope_theta_k > 0) ? p->d_cs : nullptr;
      c.seed = h->seed + (uint64_t)b0;
      c.q = q + (int64_t)b0 * n_q_heads * D;
      c.out = out + (int64_t)b0 * n_q_heads * D;
      c.tail_k = n_tail ? tail_k + (int64_t)b0 * H * n_tail * D : nullptr;
      c.tail_v = n_tail ? tail_v + (int64_t)b0 * H * n_tail * D : nullptr;
      c.ntail = n_tail;
      c.mtk = mtk; c.rpk = rpk; c.mv = mv; c.rpv = rpv; c.part = part; c.part_len = part_len;
      c.status = h->d_status;
      return launch_decode_attention(c, s);
    };
    jolt_status st = run();
    dev_free(blk, s);
    if (st != JOLT_OK) return st;
  }
  return JOLT_OK;
}
