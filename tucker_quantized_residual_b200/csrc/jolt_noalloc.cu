// eps^2 calibration for callers that cannot allocate device memory.
//
// Some callers of this library must not allocate GPU memory once they are
// running: a serving engine that has reserved nearly all of HBM for its KV
// pool up front and hands libraries no allocator, or a latency-bound loop
// where an allocation (and the synchronisation or fragmentation it can bring)
// is not allowed. jolt_eps2 gets its partial sums from cudaMallocAsync; this
// variant keeps them in a fixed device array of this file instead, so it
// allocates nothing. The caller passes the bit widths (host) and a device
// buffer for the result.
#include <mutex>
#include <vector>

#include "jolt_internal.cuh"
#include "jolt_kernels.cuh"

namespace jolt {

// Largest partial-sum table the calibration kernels write: one block per 256
// groups of the 2^20 samples (128 blocks for 32-value groups) times 9 slots
// (up to 8 bit widths + the sample energy).
constexpr int NOALLOC_MAX_BLOCKS = 128;
constexpr int NOALLOC_SLOTS = 9;

// The static scratch. Every GPU that loads the library holds these 9 KB until
// the process exits. In host code the name is only a host-side stand-in, so
// host code passes the address from cudaGetSymbolAddress instead.
static __device__ __align__(256) double g_eps2_scratch[NOALLOC_MAX_BLOCKS * NOALLOC_SLOTS];

static std::mutex g_noalloc_mu;

// One cached address per CUDA context that has called in: the array lives in
// the library's module, and every context (the primary context of each
// device, or any other context a caller makes current) loads its own copy.
struct ScratchEntry {
  void* ctx;
  int dev;
  double* ptr;
};
static std::vector<ScratchEntry> g_noalloc_cache;

// The driver's cuCtxGetCurrent, reached through the runtime (the library
// does not link the driver API directly).
typedef int (*CtxGetCurrentFn)(void**);
static CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
    cudaGetLastError();
  }
  return fn;
}

// Device address of the scratch in the current context, looked up once per
// (device, context) with that device current, and cached.
static void* current_ctx() {
  void* ctx = nullptr;
  if (CtxGetCurrentFn f = ctx_get_current())
    if (f(&ctx) != 0) ctx = nullptr;
  return ctx;
}

static jolt_status scratch_address(double** out) {
  int dev = 0;
  JOLT_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  const void* ctx = current_ctx();
  for (const ScratchEntry& e : g_noalloc_cache)
    if (e.dev == dev && e.ctx == ctx) { *out = e.ptr; return JOLT_OK; }
  void* p = nullptr;
  JOLT_CUDA_TRY(cudaGetSymbolAddress(&p, g_eps2_scratch));
  // the lookup makes the device's context current if none was: key the entry
  // on the context that holds the array
  g_noalloc_cache.push_back(ScratchEntry{current_ctx(), dev, reinterpret_cast<double*>(p)});
  *out = reinterpret_cast<double*>(p);
  return JOLT_OK;
}

}  // namespace jolt

using namespace jolt;

extern "C" jolt_status jolt_eps2_noalloc(const int32_t* bits, int32_t n, int32_t group, double* eps2_dev,
                                         jolt_stream_t stream) {
  if (!bits || !eps2_dev) { set_error("null bits or output"); return JOLT_ERR_INVALID_ARG; }
  if (n < 1 || n > NOALLOC_SLOTS - 1) {
    set_error("jolt_eps2_noalloc takes 1..%d bit widths (got %d): its static scratch holds %d slots per block",
              NOALLOC_SLOTS - 1, n, NOALLOC_SLOTS);
    return JOLT_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n; ++i)
    if (!(bits[i] == 0 || bits[i] == 2 || bits[i] == 3 || bits[i] == 4 || bits[i] == 8)) {
      set_error("bad bit width %d", bits[i]);
      return JOLT_ERR_INVALID_ARG;
    }
  if (!(group == 32 || group == 64 || group == 128)) { set_error("group must be 32, 64 or 128"); return JOLT_ERR_INVALID_ARG; }
  const int nblk = ((1 << 20) / group + 255) / 256;
  if (nblk > NOALLOC_MAX_BLOCKS) {
    set_error("calibration with groups of %d needs %d partial blocks, more than the static maximum %d", group, nblk,
              NOALLOC_MAX_BLOCKS);
    return JOLT_ERR_INVALID_ARG;
  }
  double* scratch = nullptr;
  JOLT_TRY(scratch_address(&scratch));
  // every block writes all of its slots before the final kernel reads them, so
  // nothing in the scratch has to start at zero
  return launch_eps2(bits, n, group, eps2_dev, scratch, (cudaStream_t)stream);
}
