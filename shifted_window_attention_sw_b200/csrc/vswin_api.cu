// C ABI of the library: argument validation, error reporting, scratch
// management and dispatch to the fp32 and bf16 paths. See include/vswin.h.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/vswin.h"
#include "internal.h"

namespace vswin {

__device__ int g_error_word;

namespace {

thread_local std::string t_last_error;
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_wait_limit_ns{1000000000ULL};
std::atomic<int> g_force_exact{0};
// Host-side fault injection (vswin_test_inject_failure): failures still to inject.
std::atomic<int> g_inject_cuda{0}, g_inject_alloc{0};
// VSWIN_DEBUG_BOUNDS test hook (vswin_debug_plant_row).
std::atomic<long long> g_plant_slot{-1};
std::atomic<int> g_plant_token{0};

// Takes one pending injected failure of a kind, if any.
bool take_injected(std::atomic<int>& pending) {
  int n = pending.load();
  while (n > 0)
    if (pending.compare_exchange_weak(n, n - 1)) return true;
  return false;
}

// Names every entry call on the NVTX timeline (a no-op unless a tool listens).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
const char* const kKindNames[kKinds] = {"vswin.qkv_gemm", "vswin.attention", "vswin.proj_gemm",
                                        "vswin.other",    "vswin.mlp",       "vswin.attention_bwd"};
std::mutex g_mu;
constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return status;
}

int fail_cuda(cudaError_t e, const char* what) {
  return fail(VSWIN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// Device address of the error word for the current device (looked up once per
// device, with that device current).
int error_word(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VSWIN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_error_word);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(error word)");
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_err_ptr[dev];
  return VSWIN_OK;
}

int make_ctx(KernelCtx* ctx) {
  if (take_injected(g_inject_cuda)) return fail(VSWIN_ERR_CUDA, "injected CUDA failure (test hook)");
  int* err = nullptr;
  const int st = error_word(&err);
  if (st != VSWIN_OK) return st;
  ctx->err = err;
  ctx->wait_limit = g_wait_limit_ns.load();
  ctx->force_exact = g_force_exact.load();
  return VSWIN_OK;
}

// Stream-ordered scratch comes from one library-owned memory pool per device
// whose release threshold keeps freed blocks for the next call: without it
// every synchronisation hands the scratch back to the driver and the next call
// maps it again (hundreds of MB per layer).
cudaMemPool_t g_pool[kMaxDevices] = {nullptr};

int scratch_pool(cudaMemPool_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VSWIN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemPoolCreate");
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemPoolSetAttribute");
    g_pool[dev] = pool;
  }
  *out = g_pool[dev];
  return VSWIN_OK;
}

int scratch_alloc(void** p, size_t bytes, cudaStream_t st) {
  if (take_injected(g_inject_cuda)) return fail(VSWIN_ERR_CUDA, "injected CUDA failure (test hook)");
  if (take_injected(g_inject_alloc))
    return fail(VSWIN_ERR_NO_MEMORY, "scratch allocation of %zu bytes: injected failure (test hook)", bytes);
  cudaMemPool_t pool = nullptr;
  const int status = scratch_pool(&pool);
  if (status != VSWIN_OK) return status;
  cudaError_t e = cudaMallocFromPoolAsync(p, bytes, pool, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(VSWIN_ERR_NO_MEMORY, "scratch allocation of %zu bytes: %s", bytes, cudaGetErrorString(e));
  }
  return VSWIN_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

int build_geom(int B, int T, int H, int W, int C, int heads, const int* window, const int* shift, Geom* g) {
  if (!window || !shift) return fail(VSWIN_ERR_INVALID_ARG, "window and shift must be non-NULL host arrays of 3");
  if (B <= 0 || T <= 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0)
    return fail(VSWIN_ERR_INVALID_ARG, "sizes must be positive (B=%d T=%d H=%d W=%d C=%d heads=%d)", B, T, H, W,
                C, heads);
  if (C % heads != 0) return fail(VSWIN_ERR_INVALID_ARG, "C=%d is not a multiple of heads=%d", C, heads);
  std::memset(g, 0, sizeof(*g));
  g->B = B;
  g->T = T;
  g->H = H;
  g->W = W;
  g->C = C;
  g->heads = heads;
  g->d = C / heads;
  g->L[0] = T;
  g->L[1] = H;
  g->L[2] = W;
  long long nW = 1, N = 1;
  for (int a = 0; a < 3; ++a) {
    if (window[a] < 1) return fail(VSWIN_ERR_INVALID_ARG, "window[%d]=%d must be >= 1", a, window[a]);
    if (shift[a] < 0 || shift[a] >= window[a])
      return fail(VSWIN_ERR_INVALID_ARG, "shift[%d]=%d must lie in [0, window[%d]=%d)", a, shift[a], a, window[a]);
    g->win[a] = window[a];
    g->sh[a] = shift[a];
    const long long Lp = ((long long)g->L[a] + window[a] - 1) / window[a] * window[a];
    if (Lp > (1 << 30)) return fail(VSWIN_ERR_INVALID_ARG, "extent too large");
    g->Lp[a] = (int)Lp;
    g->nw[a] = (int)(Lp / window[a]);
    nW *= g->nw[a];
    N *= window[a];
  }
  if (N > (1 << 20) || nW > (1LL << 30)) return fail(VSWIN_ERR_UNSUPPORTED, "window or grid too large");
  g->nW = (int)nW;
  g->N = (int)N;
  g->Npad = ceil_to(g->N, 16);
  g->table_rows = (2 * window[0] - 1) * (2 * window[1] - 1) * (2 * window[2] - 1);
  g->windows = (long long)B * nW;
  g->tokens = (long long)B * T * H * W;
  if (g->windows * g->N > (1LL << 31) - 1) return fail(VSWIN_ERR_UNSUPPORTED, "B * windows * N exceeds 2^31");
  return VSWIN_OK;
}

int check_layer_ptrs(const void* x, const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                     const void* table, const void* out, const Geom& g, size_t elem, size_t align,
                     bool allow_in_place = false) {
  const void* ptrs[] = {x, Wqkv, bqkv, Wproj, bproj, table, out};
  const char* names[] = {"x", "Wqkv", "bqkv", "Wproj", "bproj", "bias_table", "out"};
  for (int k = 0; k < 7; ++k)
    if (!ptrs[k]) return fail(VSWIN_ERR_INVALID_ARG, "%s is NULL", names[k]);
  const void* big[] = {x, Wqkv, Wproj, out};
  const char* bign[] = {"x", "Wqkv", "Wproj", "out"};
  for (int k = 0; k < 4; ++k)
    if (!aligned(big[k], align)) return fail(VSWIN_ERR_INVALID_ARG, "%s is not %zu-byte aligned", bign[k], align);
  const void* small[] = {bqkv, bproj, table};
  const char* smalln[] = {"bqkv", "bproj", "bias_table"};
  for (int k = 0; k < 3; ++k)
    if (!aligned(small[k], elem)) return fail(VSWIN_ERR_INVALID_ARG, "%s is not %zu-byte aligned", smalln[k], elem);
  const size_t act = (size_t)g.tokens * g.C * elem;
  if (!(allow_in_place && x == out) && overlap(x, act, out, act))
    return fail(VSWIN_ERR_INVALID_ARG, allow_in_place ? "x and out overlap without being equal" : "x and out overlap");
  return VSWIN_OK;
}

// Windows per launch chunk. One chunk per layer is fastest on B200 (more
// (window, head) items per persistent CTA, less wave quantisation) even though
// the scratch then spills from L2 to HBM; the budget (default 1 GiB,
// VSWIN_CHUNK_MB overrides) only bounds memory for very large layers.
long long chunk_windows(const Geom& g) {
  static long long budget = [] {
    const char* s = std::getenv("VSWIN_CHUNK_MB");
    long long mb = s ? std::atoll(s) : 1024;
    if (mb < 1) mb = 1;
    return mb << 20;
  }();
  const long long per = (long long)bf16_scratch_bytes(g, 1);
  long long cap = budget / per;
  if (cap < 1) cap = 1;
  if (cap >= g.windows) return g.windows;
  const long long nchunks = (g.windows + cap - 1) / cap;
  return (g.windows + nchunks - 1) / nchunks;
}

// Copy streams of the host-buffer entry, created once per device (non-blocking,
// so that they do not serialise with the legacy default stream).
constexpr int kHostChunks = 4;
cudaStream_t g_h2d[kMaxDevices] = {nullptr}, g_d2h[kMaxDevices] = {nullptr};
int copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VSWIN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_h2d[dev]) {
    e = cudaStreamCreateWithFlags(&g_h2d[dev], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&g_d2h[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) return fail_cuda(e, "cudaStreamCreateWithFlags");
  }
  *h2d = g_h2d[dev];
  *d2h = g_d2h[dev];
  return VSWIN_OK;
}

// Arguments of the MLP half (see vswin_mlp_forward); M = tokens on success.
int check_mlp_args(const void* x, int B, int T, int H, int W, int C, int hidden, const void* ln_gamma,
                   const void* ln_beta, float ln_eps, const void* W1, const void* b1, const void* W2, const void* b2,
                   const void* out, long long* M_out) {
  if (B <= 0 || T <= 0 || H <= 0 || W <= 0 || C <= 0 || hidden <= 0)
    return fail(VSWIN_ERR_INVALID_ARG, "sizes must be positive (B=%d T=%d H=%d W=%d C=%d hidden=%d)", B, T, H, W,
                C, hidden);
  const void* ptrs[] = {x, ln_gamma, ln_beta, W1, b1, W2, b2, out};
  const char* names[] = {"x", "ln_gamma", "ln_beta", "W1", "b1", "W2", "b2", "out"};
  for (int k = 0; k < 8; ++k)
    if (!ptrs[k]) return fail(VSWIN_ERR_INVALID_ARG, "%s is NULL", names[k]);
  const void* big[] = {x, W1, W2, out};
  const char* bign[] = {"x", "W1", "W2", "out"};
  for (int k = 0; k < 4; ++k)
    if (!aligned(big[k], 16)) return fail(VSWIN_ERR_INVALID_ARG, "%s is not 16-byte aligned", bign[k]);
  const void* vec[] = {ln_gamma, ln_beta, b1, b2};
  const char* vecn[] = {"ln_gamma", "ln_beta", "b1", "b2"};
  for (int k = 0; k < 4; ++k)
    if (!aligned(vec[k], 2)) return fail(VSWIN_ERR_INVALID_ARG, "%s is not 2-byte aligned", vecn[k]);
  if (!(ln_eps >= 0.f) || !std::isfinite(ln_eps))
    return fail(VSWIN_ERR_INVALID_ARG, "ln_eps must be finite and >= 0 (got %g)", (double)ln_eps);
  const long long M = (long long)B * T * H * W;
  if (M > (1LL << 31) - 1) return fail(VSWIN_ERR_UNSUPPORTED, "B * T * H * W exceeds 2^31");
  const size_t act = (size_t)M * C * 2;
  if (x != out && overlap(x, act, out, act))
    return fail(VSWIN_ERR_INVALID_ARG, "x and out overlap without being equal");
  if (!mlp_supported(C, hidden))
    return fail(VSWIN_ERR_UNSUPPORTED,
                "the fused MLP needs C a multiple of 32 up to 128 and hidden a multiple of 64 that splits "
                "into at most 8 chunks whose weights fit in shared memory (C=%d hidden=%d)",
                C, hidden);
  *M_out = M;
  return VSWIN_OK;
}

int forward_bf16_device(const void* x, const Geom& g, const void* Wqkv, const void* bqkv, const void* Wproj,
                        const void* bproj, const void* table, void* out, cudaStream_t st) {
  if (g.d != 32) return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path needs head width 32 (C/heads = %d)", g.d);
  if (!bf16_window_supported(g))
    return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path has no kernel for window (%d,%d,%d)", g.win[0], g.win[1],
                g.win[2]);
  KernelCtx ctx;
  int status = make_ctx(&ctx);
  if (status != VSWIN_OK) return status;
  const long long per_chunk = chunk_windows(g);
  const size_t bytes = bf16_scratch_bytes(g, per_chunk);
  void* scratch = nullptr;
  status = scratch_alloc(&scratch, bytes, st);
  if (status != VSWIN_OK) return status;
  cudaError_t e = cudaSuccess;
  for (long long w0 = 0; w0 < g.windows; w0 += per_chunk) {
    const long long n = (g.windows - w0) < per_chunk ? (g.windows - w0) : per_chunk;
    e = launch_bf16_chunk(g, ctx, x, Wqkv, bqkv, Wproj, bproj, table, out, scratch, w0, n, st);
    if (e != cudaSuccess) {
      cudaFreeAsync(scratch, st);
      return fail_cuda(e, "bf16 kernel launch");
    }
  }
  e = cudaFreeAsync(scratch, st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaFreeAsync");
  return VSWIN_OK;
}

// The block's attention half: the norm folded once into scratch weights, then
// the chunks with the fused statistics / epilogues.
int forward_block_device(const void* x, const Geom& g, const void* gamma, const void* beta, float eps,
                         const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj, const void* table,
                         void* out, cudaStream_t st) {
  if (g.d != 32) return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path needs head width 32 (C/heads = %d)", g.d);
  if (!bf16_window_supported(g))
    return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path has no kernel for window (%d,%d,%d)", g.win[0], g.win[1],
                g.win[2]);
  KernelCtx ctx;
  int status = make_ctx(&ctx);
  if (status != VSWIN_OK) return status;
  const long long per_chunk = chunk_windows(g);
  const size_t chunk_bytes = (bf16_block_scratch_bytes(g, per_chunk) + 255) / 256 * 256;
  // folded weights: C rows, plus 16 rows of column sums for the fused GEMM's extra K step
  const size_t wt_bytes = ((size_t)(g.C + 16) * 3 * g.C * 2 + 255) / 256 * 256;
  const size_t vec_bytes = ((size_t)3 * g.C * 4 + 255) / 256 * 256;
  void* scratch = nullptr;
  status = scratch_alloc(&scratch, chunk_bytes + wt_bytes + 2 * vec_bytes, st);
  if (status != VSWIN_OK) return status;
  uint8_t* fold = static_cast<uint8_t*>(scratch) + chunk_bytes;
  BlockFuse f;
  f.wt = fold;
  f.colsum = reinterpret_cast<float*>(fold + wt_bytes);
  f.bias_ln = reinterpret_cast<float*>(fold + wt_bytes + vec_bytes);
  f.eps = eps;
  cudaError_t e = launch_ln_fold(g, gamma, beta, Wqkv, bqkv, f, st);
  for (long long w0 = 0; e == cudaSuccess && w0 < g.windows; w0 += per_chunk) {
    const long long n = (g.windows - w0) < per_chunk ? (g.windows - w0) : per_chunk;
    e = launch_bf16_chunk(g, ctx, x, Wqkv, bqkv, Wproj, bproj, table, out, scratch, w0, n, st, &f);
  }
  if (e != cudaSuccess) {
    cudaFreeAsync(scratch, st);
    return fail_cuda(e, "bf16 block kernel launch");
  }
  e = cudaFreeAsync(scratch, st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaFreeAsync");
  return VSWIN_OK;
}

}  // namespace

void count_launch(int n) { g_launches.fetch_add((unsigned long long)n); }

namespace {
struct ProfRecord {
  int kind;
  cudaEvent_t start, end;
};
std::atomic<int> g_prof_on{0};
std::mutex g_prof_mu;
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_prof_pool;
cudaEvent_t g_prof_open[kKinds] = {};

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

void debug_plant(long long* slot, int* token) {
  *slot = g_plant_slot.load();
  *token = g_plant_token.load();
}

void prof_begin(int kind, cudaStream_t st) {
  nvtxRangePushA(kKindNames[kind]);
  if (!g_prof_on.load()) return;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  cudaEvent_t e = prof_event();
  if (!e) return;
  cudaEventRecord(e, st);
  g_prof_open[kind] = e;
}

void prof_end(int kind, cudaStream_t st) {
  nvtxRangePop();
  if (!g_prof_on.load()) return;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  cudaEvent_t s = g_prof_open[kind];
  if (!s) return;
  cudaEvent_t e = prof_event();
  if (!e) return;
  cudaEventRecord(e, st);
  g_prof_records.push_back({kind, s, e});
  g_prof_open[kind] = nullptr;
}

}  // namespace vswin

// ---------------------------------------------------------------------------
// Fixed scratch for vswin_wmsa_forward_noalloc.
//
// Some callers cannot allocate device memory on the call path: a plugin or
// real-time host that must stay within memory it reserved up front, code that
// may not synchronise the device (cudaMalloc can), or a process whose
// allocator is owned by another framework. For them the bf16 layer can run
// out of this statically sized array instead of stream-ordered scratch.
// Every GPU that loads this library holds the array until the process exits.
static constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace vswin {
namespace {
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name only stands in for the symbol; its address on a device comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current (the first call on each device does this).
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VSWIN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(no-allocation scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return VSWIN_OK;
}
}  // namespace
}  // namespace vswin

using namespace vswin;

extern "C" {

int vswin_version(void) { return 100; }

const char* vswin_last_error(void) { return t_last_error.c_str(); }

unsigned long long vswin_launch_count(void) { return g_launches.load(); }

void vswin_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns.store(ns ? ns : 1); }

void vswin_set_exact_softmax(int on) { g_force_exact.store(on ? 1 : 0); }

int vswin_test_inject_failure(int kind, int count) {
  if (count < 0) return fail(VSWIN_ERR_INVALID_ARG, "count=%d must be >= 0", count);
  if (kind == VSWIN_INJECT_CUDA)
    g_inject_cuda.store(count);
  else if (kind == VSWIN_INJECT_ALLOC)
    g_inject_alloc.store(count);
  else
    return fail(VSWIN_ERR_INVALID_ARG, "unknown injection kind %d", kind);
  return VSWIN_OK;
}

int vswin_debug_bounds_enabled(void) {
#ifdef VSWIN_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

int vswin_debug_plant_row(long long slot, int token) {
  if (!vswin_debug_bounds_enabled())
    return fail(VSWIN_ERR_UNSUPPORTED, "vswin_debug_plant_row needs a build with VSWIN_DEBUG_BOUNDS");
  g_plant_token.store(token);
  g_plant_slot.store(slot < 0 ? -1 : slot);
  return VSWIN_OK;
}

int vswin_clamp_window(int T, int H, int W, const int* window_in, const int* shift_in, int* window_out,
                       int* shift_out) {
  if (!window_in || !shift_in || !window_out || !shift_out)
    return fail(VSWIN_ERR_INVALID_ARG, "NULL argument to vswin_clamp_window");
  const int L[3] = {T, H, W};
  for (int a = 0; a < 3; ++a) {
    if (L[a] <= 0 || window_in[a] < 1 || shift_in[a] < 0)
      return fail(VSWIN_ERR_INVALID_ARG, "invalid extent, window or shift on axis %d", a);
    if (L[a] <= window_in[a]) {
      window_out[a] = L[a];
      shift_out[a] = 0;
    } else {
      window_out[a] = window_in[a];
      shift_out[a] = shift_in[a];
    }
  }
  return VSWIN_OK;
}

int vswin_wmsa_forward(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                       const int* shift, const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                       const void* bias_table, void* out, void* stream) {
  NvtxRange nvtx_range("vswin_wmsa_forward");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  st = check_layer_ptrs(x, Wqkv, bqkv, Wproj, bproj, bias_table, out, g, 2, 16);
  if (st != VSWIN_OK) return st;
  return forward_bf16_device(x, g, Wqkv, bqkv, Wproj, bproj, bias_table, out, static_cast<cudaStream_t>(stream));
}

int vswin_block_msa_forward(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                            const int* shift, const void* ln_gamma, const void* ln_beta, float ln_eps,
                            const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                            const void* bias_table, void* out, void* stream) {
  NvtxRange nvtx_range("vswin_block_msa_forward");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  st = check_layer_ptrs(x, Wqkv, bqkv, Wproj, bproj, bias_table, out, g, 2, 16, true);
  if (st != VSWIN_OK) return st;
  if (!ln_gamma || !ln_beta) return fail(VSWIN_ERR_INVALID_ARG, "ln_gamma and ln_beta must be non-NULL");
  if (!aligned(ln_gamma, 2) || !aligned(ln_beta, 2))
    return fail(VSWIN_ERR_INVALID_ARG, "ln_gamma and ln_beta must be 2-byte aligned");
  if (!(ln_eps >= 0.f) || !std::isfinite(ln_eps))
    return fail(VSWIN_ERR_INVALID_ARG, "ln_eps must be finite and >= 0 (got %g)", (double)ln_eps);
  return forward_block_device(x, g, ln_gamma, ln_beta, ln_eps, Wqkv, bqkv, Wproj, bproj, bias_table, out,
                              static_cast<cudaStream_t>(stream));
}

int vswin_mlp_forward(const void* x, int B, int T, int H, int W, int C, int hidden, const void* ln_gamma,
                      const void* ln_beta, float ln_eps, const void* W1, const void* b1, const void* W2,
                      const void* b2, void* out, void* stream) {
  NvtxRange nvtx_range("vswin_mlp_forward");
  long long M = 0;
  int st = check_mlp_args(x, B, T, H, W, C, hidden, ln_gamma, ln_beta, ln_eps, W1, b1, W2, b2, out, &M);
  if (st != VSWIN_OK) return st;
  KernelCtx ctx;
  st = make_ctx(&ctx);
  if (st != VSWIN_OK) return st;
  cudaError_t e = launch_mlp(ctx, M, C, hidden, x, ln_gamma, ln_beta, ln_eps, W1, b1, W2, b2, out,
                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "MLP kernel launch");
  return VSWIN_OK;
}

int vswin_block_forward(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                        const int* shift, const void* ln1_gamma, const void* ln1_beta, const void* Wqkv,
                        const void* bqkv, const void* Wproj, const void* bproj, const void* bias_table,
                        const void* ln2_gamma, const void* ln2_beta, int hidden, const void* W1, const void* b1,
                        const void* W2, const void* b2, float ln_eps, void* out, void* stream) {
  NvtxRange nvtx_range("vswin_block_forward");
  // every argument of both halves is checked before anything is launched
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  st = check_layer_ptrs(x, Wqkv, bqkv, Wproj, bproj, bias_table, out, g, 2, 16, true);
  if (st != VSWIN_OK) return st;
  if (!ln1_gamma || !ln1_beta) return fail(VSWIN_ERR_INVALID_ARG, "ln1_gamma and ln1_beta must be non-NULL");
  if (!aligned(ln1_gamma, 2) || !aligned(ln1_beta, 2))
    return fail(VSWIN_ERR_INVALID_ARG, "ln1_gamma and ln1_beta must be 2-byte aligned");
  long long M = 0;
  st = check_mlp_args(out, B, T, H, W, C, hidden, ln2_gamma, ln2_beta, ln_eps, W1, b1, W2, b2, out, &M);
  if (st != VSWIN_OK) return st;
  if (g.d != 32) return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path needs head width 32 (C/heads = %d)", g.d);
  if (!bf16_window_supported(g))
    return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path has no kernel for window (%d,%d,%d)", g.win[0], g.win[1],
                g.win[2]);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = forward_block_device(x, g, ln1_gamma, ln1_beta, ln_eps, Wqkv, bqkv, Wproj, bproj, bias_table, out, s);
  if (st != VSWIN_OK) return st;
  KernelCtx ctx;
  st = make_ctx(&ctx);
  if (st != VSWIN_OK) return st;
  cudaError_t e = launch_mlp(ctx, M, C, hidden, out, ln2_gamma, ln2_beta, ln_eps, W1, b1, W2, b2, out, s);
  if (e != cudaSuccess) return fail_cuda(e, "MLP kernel launch");
  return VSWIN_OK;
}

int vswin_patch_merge_forward(const void* x, int B, int T, int H, int W, int C, const void* ln_gamma,
                              const void* ln_beta, float ln_eps, const void* Wr, const void* br, void* out,
                              void* stream) {
  NvtxRange nvtx_range("vswin_patch_merge_forward");
  if (B <= 0 || T <= 0 || H <= 0 || W <= 0 || C <= 0)
    return fail(VSWIN_ERR_INVALID_ARG, "sizes must be positive (B=%d T=%d H=%d W=%d C=%d)", B, T, H, W, C);
  const void* ptrs[] = {x, ln_gamma, ln_beta, Wr, out};
  const char* names[] = {"x", "ln_gamma", "ln_beta", "Wr", "out"};
  for (int k = 0; k < 5; ++k)
    if (!ptrs[k]) return fail(VSWIN_ERR_INVALID_ARG, "%s is NULL", names[k]);
  const void* big[] = {x, Wr, out};
  const char* bign[] = {"x", "Wr", "out"};
  for (int k = 0; k < 3; ++k)
    if (!aligned(big[k], 16)) return fail(VSWIN_ERR_INVALID_ARG, "%s is not 16-byte aligned", bign[k]);
  if (!aligned(ln_gamma, 2) || !aligned(ln_beta, 2) || (br && !aligned(br, 2)))
    return fail(VSWIN_ERR_INVALID_ARG, "ln_gamma, ln_beta and br must be 2-byte aligned");
  if (!(ln_eps >= 0.f) || !std::isfinite(ln_eps))
    return fail(VSWIN_ERR_INVALID_ARG, "ln_eps must be finite and >= 0 (got %g)", (double)ln_eps);
  const long long tokens = (long long)B * T * H * W;
  const long long merged = (long long)B * T * ((H + 1) / 2) * ((W + 1) / 2);
  if (tokens > (1LL << 40) || merged / 128 > (1LL << 30))
    return fail(VSWIN_ERR_UNSUPPORTED, "input too large (%lld tokens)", tokens);
  if (overlap(x, (size_t)tokens * C * 2, out, (size_t)merged * 2 * C * 2))
    return fail(VSWIN_ERR_INVALID_ARG, "x and out overlap");
  if (!patch_merge_supported(C))
    return fail(VSWIN_ERR_UNSUPPORTED, "patch merging needs C a multiple of 32 (C=%d)", C);
  KernelCtx ctx;
  int st = make_ctx(&ctx);
  if (st != VSWIN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  st = scratch_alloc(&scratch, patch_merge_scratch_bytes(C), s);
  if (st != VSWIN_OK) return st;
  cudaError_t e = launch_patch_merge(ctx, B, T, H, W, C, x, ln_gamma, ln_beta, ln_eps, Wr, br, out, scratch, s);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) return fail_cuda(e, "patch merging launch");
  if (e2 != cudaSuccess) return fail_cuda(e2, "cudaFreeAsync");
  return VSWIN_OK;
}

int vswin_wmsa_forward_f32(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                           const int* shift, const void* Wqkv, const void* bqkv, const void* Wproj,
                           const void* bproj, const void* bias_table, void* out, void* stream) {
  NvtxRange nvtx_range("vswin_wmsa_forward_f32");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  st = check_layer_ptrs(x, Wqkv, bqkv, Wproj, bproj, bias_table, out, g, 4, 4);
  if (st != VSWIN_OK) return st;
  if (g.N > 4096) return fail(VSWIN_ERR_UNSUPPORTED, "fp32 path supports N <= 4096 (N = %d)", g.N);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  size_t nq = 0, no = 0;
  f32_scratch_floats(g, &nq, &no);
  void* scratch = nullptr;
  st = scratch_alloc(&scratch, (nq + no) * sizeof(float), s);
  if (st != VSWIN_OK) return st;
  float* sq = static_cast<float*>(scratch);
  cudaError_t e = launch_f32_forward(g, static_cast<const float*>(x), static_cast<const float*>(Wqkv),
                         static_cast<const float*>(bqkv), static_cast<const float*>(Wproj),
                         static_cast<const float*>(bproj), static_cast<const float*>(bias_table),
                         static_cast<float*>(out), sq, sq + nq, s);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) return fail_cuda(e, "fp32 kernel launch");
  if (e2 != cudaSuccess) return fail_cuda(e2, "cudaFreeAsync");
  return VSWIN_OK;
}

int vswin_wmsa_backward_f32(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                            const int* shift, const void* Wqkv, const void* bqkv, const void* Wproj,
                            const void* bproj, const void* bias_table, const void* dy, void* dx, void* dWqkv,
                            void* dbqkv, void* dWproj, void* dbproj, void* dtable, void* stream) {
  NvtxRange nvtx_range("vswin_wmsa_backward_f32");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  const void* ptrs[] = {x, Wqkv, bqkv, Wproj, bproj, bias_table, dy, dx, dWqkv, dbqkv, dWproj, dbproj, dtable};
  const char* names[] = {"x", "Wqkv", "bqkv", "Wproj", "bproj", "bias_table", "dy",
                         "dx", "dWqkv", "dbqkv", "dWproj", "dbproj", "dtable"};
  for (int k = 0; k < 13; ++k) {
    if (!ptrs[k]) return fail(VSWIN_ERR_INVALID_ARG, "%s is NULL", names[k]);
    if (!aligned(ptrs[k], 4)) return fail(VSWIN_ERR_INVALID_ARG, "%s is not 4-byte aligned", names[k]);
  }
  const size_t act = (size_t)g.tokens * g.C * 4;
  const size_t wq = (size_t)g.C * 3 * g.C * 4, wp = (size_t)g.C * g.C * 4;
  const size_t tb = (size_t)g.table_rows * g.heads * 4;
  // every output against every input it could alias
  const void* outs[] = {dx, dWqkv, dbqkv, dWproj, dbproj, dtable};
  const size_t out_n[] = {act, wq, (size_t)3 * g.C * 4, wp, (size_t)g.C * 4, tb};
  const void* ins[] = {x, dy, Wqkv, bqkv, Wproj, bproj, bias_table};
  const size_t in_n[] = {act, act, wq, (size_t)3 * g.C * 4, wp, (size_t)g.C * 4, tb};
  for (int a = 0; a < 6; ++a) {
    for (int b = 0; b < 7; ++b)
      if (overlap(outs[a], out_n[a], ins[b], in_n[b]))
        return fail(VSWIN_ERR_INVALID_ARG, "gradient buffer %s overlaps an input", names[7 + a]);
    for (int b = a + 1; b < 6; ++b)
      if (overlap(outs[a], out_n[a], outs[b], out_n[b]))
        return fail(VSWIN_ERR_INVALID_ARG, "gradient buffers %s and %s overlap", names[7 + a], names[7 + b]);
  }
  if (g.N > 4096) return fail(VSWIN_ERR_UNSUPPORTED, "fp32 backward supports N <= 4096 (N = %d)", g.N);
  if ((2 * (size_t)g.N + 2 * g.d) * 4 > 48 * 1024 || (size_t)3 * g.C * 4 > 48 * 1024)
    return fail(VSWIN_ERR_UNSUPPORTED, "fp32 backward: window or width too large for its shared-memory rows");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  st = scratch_alloc(&scratch, f32_backward_scratch_bytes(g), s);
  if (st != VSWIN_OK) return st;
  cudaError_t e = launch_f32_backward(
      g, static_cast<const float*>(x), static_cast<const float*>(Wqkv), static_cast<const float*>(bqkv),
      static_cast<const float*>(Wproj), static_cast<const float*>(bproj), static_cast<const float*>(bias_table),
      static_cast<const float*>(dy), static_cast<float*>(dx), static_cast<float*>(dWqkv),
      static_cast<float*>(dbqkv), static_cast<float*>(dWproj), static_cast<float*>(dbproj),
      static_cast<float*>(dtable), scratch, s);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) return fail_cuda(e, "fp32 backward launch");
  if (e2 != cudaSuccess) return fail_cuda(e2, "cudaFreeAsync");
  return VSWIN_OK;
}

int vswin_wmsa_backward(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                        const int* shift, const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                        const void* bias_table, const void* dy, void* dx, void* dWqkv, void* dbqkv, void* dWproj,
                        void* dbproj, void* dtable, void* stream) {
  NvtxRange nvtx_range("vswin_wmsa_backward");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  const void* ptrs[] = {x, Wqkv, bqkv, Wproj, bproj, bias_table, dy, dx, dWqkv, dbqkv, dWproj, dbproj, dtable};
  const char* names[] = {"x", "Wqkv", "bqkv", "Wproj", "bproj", "bias_table", "dy",
                         "dx", "dWqkv", "dbqkv", "dWproj", "dbproj", "dtable"};
  // bf16 activations and x rows are read 16 bytes at a time; bf16 vectors and
  // the table element-wise; the fp32 gradients element-wise
  const size_t align[] = {16, 2, 2, 2, 2, 2, 16, 16, 4, 4, 4, 4, 4};
  for (int k = 0; k < 13; ++k) {
    if (!ptrs[k]) return fail(VSWIN_ERR_INVALID_ARG, "%s is NULL", names[k]);
    if (!aligned(ptrs[k], align[k]))
      return fail(VSWIN_ERR_INVALID_ARG, "%s is not %zu-byte aligned", names[k], align[k]);
  }
  const size_t act = (size_t)g.tokens * g.C * 2;
  const size_t wq = (size_t)g.C * 3 * g.C, wp = (size_t)g.C * g.C;
  const size_t tb = (size_t)g.table_rows * g.heads;
  const void* outs[] = {dx, dWqkv, dbqkv, dWproj, dbproj, dtable};
  const size_t out_n[] = {act, wq * 4, (size_t)3 * g.C * 4, wp * 4, (size_t)g.C * 4, tb * 4};
  const void* ins[] = {x, dy, Wqkv, bqkv, Wproj, bproj, bias_table};
  const size_t in_n[] = {act, act, wq * 2, (size_t)3 * g.C * 2, wp * 2, (size_t)g.C * 2, tb * 2};
  for (int a = 0; a < 6; ++a) {
    for (int b = 0; b < 7; ++b)
      if (overlap(outs[a], out_n[a], ins[b], in_n[b]))
        return fail(VSWIN_ERR_INVALID_ARG, "gradient buffer %s overlaps an input", names[7 + a]);
    for (int b = a + 1; b < 6; ++b)
      if (overlap(outs[a], out_n[a], outs[b], out_n[b]))
        return fail(VSWIN_ERR_INVALID_ARG, "gradient buffers %s and %s overlap", names[7 + a], names[7 + b]);
  }
  if (!bf16_backward_supported(g))
    return fail(VSWIN_ERR_UNSUPPORTED,
                "bf16 backward needs head width 32, C %% 32 == 0 and a (P,7,7) window with P in {1,2,4,8} "
                "(d = %d, C = %d, window (%d,%d,%d)); the fp32 backward covers the rest",
                g.d, g.C, g.win[0], g.win[1], g.win[2]);
  KernelCtx ctx;
  st = make_ctx(&ctx);
  if (st != VSWIN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long chunk = chunk_windows(g);
  void* scratch = nullptr;
  st = scratch_alloc(&scratch, bf16_backward_scratch_bytes(g, chunk), s);
  if (st != VSWIN_OK) return st;
  cudaError_t e = launch_bf16_backward(g, ctx, x, Wqkv, bqkv, Wproj, bias_table, dy, dx,
                                       static_cast<float*>(dWqkv), static_cast<float*>(dbqkv),
                                       static_cast<float*>(dWproj), static_cast<float*>(dbproj),
                                       static_cast<float*>(dtable), scratch, chunk, s);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) return fail_cuda(e, "bf16 backward launch");
  if (e2 != cudaSuccess) return fail_cuda(e2, "cudaFreeAsync");
  return VSWIN_OK;
}

int vswin_wmsa_forward_host(const void* x_host, int B, int T, int H, int W, int C, int heads, const int* window,
                            const int* shift, const void* Wqkv, const void* bqkv, const void* Wproj,
                            const void* bproj, const void* bias_table, void* out_host, void* stream) {
  NvtxRange nvtx_range("vswin_wmsa_forward_host");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  if (!x_host || !out_host) return fail(VSWIN_ERR_INVALID_ARG, "x_host and out_host must be non-NULL");
  const size_t act = (size_t)g.tokens * g.C * 2;
  if (overlap(x_host, act, out_host, act)) return fail(VSWIN_ERR_INVALID_ARG, "x_host and out_host overlap");
  {
    const void* w[] = {Wqkv, bqkv, Wproj, bproj, bias_table};
    const char* wn[] = {"Wqkv", "bqkv", "Wproj", "bproj", "bias_table"};
    for (int k = 0; k < 5; ++k) {
      if (!w[k]) return fail(VSWIN_ERR_INVALID_ARG, "%s is NULL", wn[k]);
      if (!aligned(w[k], k == 0 || k == 2 ? 16 : 2))
        return fail(VSWIN_ERR_INVALID_ARG, "%s is not %d-byte aligned", wn[k], k == 0 || k == 2 ? 16 : 2);
    }
  }
  if (g.d != 32) return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path needs head width 32 (C/heads = %d)", g.d);
  if (!bf16_window_supported(g))
    return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path has no kernel for window (%d,%d,%d)", g.win[0], g.win[1],
                g.win[2]);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t h2d = nullptr, d2h = nullptr;
  st = copy_streams(&h2d, &d2h);
  if (st != VSWIN_OK) return st;
  void* buf = nullptr;
  const size_t act_pad = (act + 255) / 256 * 256;
  st = scratch_alloc(&buf, 2 * act_pad, s);
  if (st != VSWIN_OK) return st;
  uint8_t* xd = static_cast<uint8_t*>(buf);
  uint8_t* od = xd + act_pad;
  // Clips are independent (the roll and the windows stay inside a clip), so the
  // batch goes through in groups of clips: the copy in of group k + 1, the layer
  // on group k and the copy out of group k - 1 overlap on three streams.
  const int nchunk = B < kHostChunks ? B : kHostChunks;
  const int per = (B + nchunk - 1) / nchunk;
  const size_t clip = (size_t)T * H * W * C * 2;
  cudaEvent_t ev[1 + 3 * kHostChunks] = {};
  int nev = 0;
  cudaError_t e = cudaSuccess;
  for (int k = 0; k < 1 + 3 * nchunk && e == cudaSuccess; ++k, ++nev)
    e = cudaEventCreateWithFlags(&ev[k], cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(ev[0], s);  // the device buffers exist on s from here
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h2d, ev[0], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(d2h, ev[0], 0);
  int last_out = -1;
  for (int k = 0; k < nchunk && e == cudaSuccess && st == VSWIN_OK; ++k) {
    const int b0 = k * per, nb = (B - b0) < per ? (B - b0) : per;
    if (nb <= 0) break;
    const size_t off = (size_t)b0 * clip, bytes = (size_t)nb * clip;
    cudaEvent_t ev_in = ev[1 + 3 * k], ev_comp = ev[2 + 3 * k], ev_out = ev[3 + 3 * k];
    e = cudaMemcpyAsync(xd + off, static_cast<const uint8_t*>(x_host) + off, bytes, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in, h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_in, 0);
    if (e != cudaSuccess) break;
    Geom gk;
    st = build_geom(nb, T, H, W, C, heads, window, shift, &gk);
    if (st == VSWIN_OK) st = forward_bf16_device(xd + off, gk, Wqkv, bqkv, Wproj, bproj, bias_table, od + off, s);
    if (st != VSWIN_OK) break;
    e = cudaEventRecord(ev_comp, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(d2h, ev_comp, 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + off, od + off, bytes, cudaMemcpyDeviceToHost, d2h);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out, d2h);
    if (e == cudaSuccess) last_out = 3 + 3 * k;
  }
  if (e != cudaSuccess && st == VSWIN_OK) st = fail_cuda(e, "host-entry copy or event");
  // the buffers are released on s only after every copy out has read them
  if (last_out >= 0) cudaStreamWaitEvent(s, ev[last_out], 0);
  if (st != VSWIN_OK) {  // something was refused part-way: let whatever was queued finish first
    cudaStreamSynchronize(h2d);
    cudaStreamSynchronize(d2h);
  }
  cudaFreeAsync(buf, s);
  e = cudaStreamSynchronize(s);
  if (st == VSWIN_OK && e != cudaSuccess) st = fail_cuda(e, "cudaStreamSynchronize");
  for (int k = 0; k < nev; ++k)
    if (ev[k]) cudaEventDestroy(ev[k]);
  return st;
}

int vswin_wmsa_index_maps(int B, int T, int H, int W, const int* window, const int* shift, int* win_src,
                          int* region, int* bias_idx, void* stream) {
  Geom g;
  int st = build_geom(B, T, H, W, 1, 1, window, shift, &g);
  if (st != VSWIN_OK) return st;
  if (!win_src && !region && !bias_idx) return VSWIN_OK;
  if ((long long)g.N * g.N > (1LL << 31) - 1) return fail(VSWIN_ERR_UNSUPPORTED, "N*N exceeds 2^31");
  cudaError_t e = launch_index_maps(g, win_src, region, bias_idx, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "index map kernel launch");
  return VSWIN_OK;
}

int vswin_poll_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "cudaStreamSynchronize");
  int* err = nullptr;
  int st = error_word(&err);
  if (st != VSWIN_OK) return st;
  int word = 0;
  e = cudaMemcpy(&word, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e, "reading the error word");
  if (word == 0) return VSWIN_OK;
  const int zero = 0;
  e = cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail_cuda(e, "clearing the error word");
  if (word == kErrBounds) return fail(VSWIN_ERR_BOUNDS, "an index check failed; the access was skipped (code 0x%x)", word);
  return fail(VSWIN_ERR_TIMEOUT, "a kernel wait gave up (code 0x%x)", word);
}

int vswin_profile_enable(int on) {
  g_prof_on.store(on ? 1 : 0);
  return VSWIN_OK;
}

int vswin_profile_collect(double* ms, unsigned long long* launches, int nkinds) {
  if (!ms || !launches || nkinds < 0) return fail(VSWIN_ERR_INVALID_ARG, "NULL argument to vswin_profile_collect");
  for (int k = 0; k < nkinds; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  std::lock_guard<std::mutex> lock(g_prof_mu);
  int status = VSWIN_OK;
  for (const ProfRecord& r : g_prof_records) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.end);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.start, r.end);
    if (e != cudaSuccess && status == VSWIN_OK) status = fail_cuda(e, "profile events");
    if (r.kind < nkinds) {
      ms[r.kind] += t;
      launches[r.kind] += 1;
    }
    g_prof_pool.push_back(r.start);
    g_prof_pool.push_back(r.end);
  }
  g_prof_records.clear();
  return status;
}

int vswin_selftest_timeout(void* stream) {
  KernelCtx ctx;
  int st = make_ctx(&ctx);
  if (st != VSWIN_OK) return st;
  cudaError_t e = launch_selftest_timeout(ctx, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "self-test launch");
  return VSWIN_OK;
}

int vswin_wmsa_forward_noalloc(const void* x, int B, int T, int H, int W, int C, int heads, const int* window,
                               const int* shift, const void* Wqkv, const void* bqkv, const void* Wproj,
                               const void* bproj, const void* bias_table, void* out, void* stream) {
  NvtxRange nvtx_range("vswin_wmsa_forward_noalloc");
  Geom g;
  int st = build_geom(B, T, H, W, C, heads, window, shift, &g);
  if (st != VSWIN_OK) return st;
  st = check_layer_ptrs(x, Wqkv, bqkv, Wproj, bproj, bias_table, out, g, 2, 16);
  if (st != VSWIN_OK) return st;
  if (g.d != 32) return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path needs head width 32 (C/heads = %d)", g.d);
  if (!bf16_window_supported(g))
    return fail(VSWIN_ERR_UNSUPPORTED, "bf16 path has no kernel for window (%d,%d,%d)", g.win[0], g.win[1],
                g.win[2]);
  const size_t per_window = bf16_scratch_bytes(g, 1);
  if (per_window > kNoAllocScratchBytes)
    return fail(VSWIN_ERR_UNSUPPORTED,
                "one window of this layer needs %zu bytes of scratch; the no-allocation entry point has %zu bytes "
                "(%zu MiB)",
                per_window, kNoAllocScratchBytes, kNoAllocScratchBytes >> 20);
  KernelCtx ctx;
  st = make_ctx(&ctx);
  if (st != VSWIN_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != VSWIN_OK) return st;
  // Windows go through the fixed array in equal chunks. Nothing in it needs to
  // start at zero: every byte a kernel uses is first written by this call.
  long long cap = (long long)(kNoAllocScratchBytes / per_window);
  if (cap > g.windows) cap = g.windows;
  const long long nchunks = (g.windows + cap - 1) / cap;
  const long long per_chunk = (g.windows + nchunks - 1) / nchunks;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (long long w0 = 0; w0 < g.windows; w0 += per_chunk) {
    const long long n = (g.windows - w0) < per_chunk ? (g.windows - w0) : per_chunk;
    cudaError_t e = launch_bf16_chunk(g, ctx, x, Wqkv, bqkv, Wproj, bproj, bias_table, out, scratch, w0, n, s);
    if (e != cudaSuccess) return fail_cuda(e, "bf16 kernel launch (no-allocation entry)");
  }
  return VSWIN_OK;
}

}  // extern "C"
