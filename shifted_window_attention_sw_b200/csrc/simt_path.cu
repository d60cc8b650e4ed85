// fp32 path: the layer in plain FP32 FMA arithmetic (no tensor cores), plus the
// index-map export and the timeout self-test kernel.
//
// Three launches: gather + QKV projection, per-(window, head, query) masked
// softmax attention, output projection + scatter. Intermediates (qkv, o) live
// in fp32 scratch, [window][slot][channel].
#include <cmath>

#include "internal.h"
#include "sm100.cuh"

namespace vswin {

namespace {

constexpr int kThreads = 128;

// qkv[w][n][j] = sum_c X[w][n][c] Wqkv[c][j] + bqkv[j], X[w][n] = x[source] or 0.
__global__ void __launch_bounds__(kThreads) f32_qkv_kernel(Geom g, const float* __restrict__ x,
                                                           const float* __restrict__ Wqkv,
                                                           const float* __restrict__ bqkv,
                                                           float* __restrict__ qkv) {
  extern __shared__ float xrow[];  // C floats
  const long long row = blockIdx.x;  // window * N + slot
  const long long src = slot_source(g, row / g.N, (int)(row % g.N));
  for (int c = threadIdx.x; c < g.C; c += blockDim.x) xrow[c] = src >= 0 ? x[src * g.C + c] : 0.f;
  __syncthreads();
  const int C3 = 3 * g.C;
  const int j = blockIdx.y * blockDim.x + threadIdx.x;
  if (j >= C3) return;
  float acc = bqkv[j];
  for (int c = 0; c < g.C; ++c) acc = fmaf(xrow[c], Wqkv[(size_t)c * C3 + j], acc);
  qkv[row * C3 + j] = acc;
}

// One block per (query slot, window, head): scores over all keys of the window
// that share the query's region, softmax, then o = P V for that head.
__global__ void __launch_bounds__(kThreads) f32_attention_kernel(Geom g, const float* __restrict__ qkv,
                                                                 const float* __restrict__ table,
                                                                 float* __restrict__ o) {
  extern __shared__ float sm[];
  float* score = sm;          // N
  float* q = sm + g.N;        // d
  __shared__ float red[kThreads / 32];
  __shared__ float bcast;
  const long long win = blockIdx.x;
  const int i = blockIdx.y;
  const int h = blockIdx.z;
  const int C3 = 3 * g.C, d = g.d;
  const int w_in_clip = (int)(win % g.nW);
  const bool shifted = (g.sh[0] | g.sh[1] | g.sh[2]) != 0;
  const float* base = qkv + win * g.N * (long long)C3;
  for (int c = threadIdx.x; c < d; c += blockDim.x) q[c] = base[(size_t)i * C3 + h * d + c];
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)d);
  const int reg_i = shifted ? slot_region(g, w_in_clip, i) : 0;
  float m = -INFINITY;
  for (int j = threadIdx.x; j < g.N; j += blockDim.x) {
    float s = -INFINITY;
    if (!shifted || slot_region(g, w_in_clip, j) == reg_i) {
      const float* k = base + (size_t)j * C3 + g.C + h * d;
      float dot = 0.f;
      for (int c = 0; c < d; ++c) dot = fmaf(q[c], k[c], dot);
      s = dot * scale + table[(size_t)bias_row(g, i, j) * g.heads + h];
    }
    score[j] = s;
    m = fmaxf(m, s);
  }
  // block max
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = red[0];
    for (int k = 1; k < kThreads / 32; ++k) mm = fmaxf(mm, red[k]);
    bcast = mm;
  }
  __syncthreads();
  m = bcast;
  float sum = 0.f;
  for (int j = threadIdx.x; j < g.N; j += blockDim.x) {
    const float p = score[j] == -INFINITY ? 0.f : expf(score[j] - m);
    score[j] = p;
    sum += p;
  }
  __syncthreads();
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float ss = 0.f;
    for (int k = 0; k < kThreads / 32; ++k) ss += red[k];
    bcast = 1.0f / ss;
  }
  __syncthreads();
  const float inv = bcast;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < g.N; ++j) acc = fmaf(score[j], base[(size_t)j * C3 + 2 * g.C + h * d + c], acc);
    o[(win * g.N + i) * (long long)g.C + h * d + c] = acc * inv;
  }
}

// out[source] = o[w][n] Wproj + bproj for every slot that is not padding.
__global__ void __launch_bounds__(kThreads) f32_proj_kernel(Geom g, const float* __restrict__ o,
                                                            const float* __restrict__ Wproj,
                                                            const float* __restrict__ bproj,
                                                            float* __restrict__ out) {
  extern __shared__ float orow[];
  const long long row = blockIdx.x;
  const long long dst = slot_source(g, row / g.N, (int)(row % g.N));
  if (dst < 0) return;  // uniform over the block
  for (int c = threadIdx.x; c < g.C; c += blockDim.x) orow[c] = o[row * g.C + c];
  __syncthreads();
  const int j = blockIdx.y * blockDim.x + threadIdx.x;
  if (j >= g.C) return;
  float acc = bproj[j];
  for (int c = 0; c < g.C; ++c) acc = fmaf(orow[c], Wproj[(size_t)c * g.C + j], acc);
  out[dst * g.C + j] = acc;
}

__global__ void index_maps_kernel(Geom g, int* __restrict__ win_src, int* __restrict__ region,
                                  int* __restrict__ bias_idx) {
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  if (win_src)
    for (long long k = tid; k < g.windows * g.N; k += stride)
      win_src[k] = (int)slot_source(g, k / g.N, (int)(k % g.N));
  if (region)
    for (long long k = tid; k < (long long)g.nW * g.N; k += stride)
      region[k] = slot_region(g, (int)(k / g.N), (int)(k % g.N));
  if (bias_idx)
    for (long long k = tid; k < (long long)g.N * g.N; k += stride)
      bias_idx[k] = bias_row(g, (int)(k / g.N), (int)(k % g.N));
}

// Waits, with the configured limit, on an mbarrier that nothing completes.
__global__ void selftest_timeout_kernel(KernelCtx ctx) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, ctx.err, kErrWaitSelftest, ctx.wait_limit);
  __syncthreads();
}

}  // namespace

size_t f32_scratch_floats(const Geom& g, size_t* qkv_floats, size_t* o_floats) {
  *qkv_floats = (size_t)g.windows * g.N * 3 * g.C;
  *o_floats = (size_t)g.windows * g.N * g.C;
  return *qkv_floats + *o_floats;
}

cudaError_t launch_f32_forward(const Geom& g, const float* x, const float* Wqkv, const float* bqkv,
                               const float* Wproj, const float* bproj, const float* table, float* out,
                               float* scratch_qkv, float* scratch_o, cudaStream_t st) {
  const long long rows = g.windows * g.N;
  if (rows > 2147483647LL) return cudaErrorInvalidConfiguration;
  dim3 g1((unsigned)rows, (3 * g.C + kThreads - 1) / kThreads);
  prof_begin(kKindOther, st);
  f32_qkv_kernel<<<g1, kThreads, g.C * sizeof(float), st>>>(g, x, Wqkv, bqkv, scratch_qkv);
  prof_end(kKindOther, st);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((unsigned)g.windows, g.N, g.heads);
  prof_begin(kKindOther, st);
  f32_attention_kernel<<<g2, kThreads, (g.N + g.d) * sizeof(float), st>>>(g, scratch_qkv, table, scratch_o);
  prof_end(kKindOther, st);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g3((unsigned)rows, (g.C + kThreads - 1) / kThreads);
  prof_begin(kKindOther, st);
  f32_proj_kernel<<<g3, kThreads, g.C * sizeof(float), st>>>(g, scratch_o, Wproj, bproj, out);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_index_maps(const Geom& g, int* win_src, int* region, int* bias_idx, cudaStream_t st) {
  long long work = g.windows * g.N;
  if ((long long)g.N * g.N > work) work = (long long)g.N * g.N;
  long long blocks = (work + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  prof_begin(kKindOther, st);
  index_maps_kernel<<<(unsigned)blocks, 256, 0, st>>>(g, win_src, region, bias_idx);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(const KernelCtx& ctx, cudaStream_t st) {
  prof_begin(kKindOther, st);
  selftest_timeout_kernel<<<1, 32, 0, st>>>(ctx);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace vswin
