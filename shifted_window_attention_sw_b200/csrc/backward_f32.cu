// fp32 backward of the layer (plain FP32 FMA arithmetic, no tensor cores): for
// an output gradient dy, the gradients of x, Wqkv, bqkv, Wproj, bproj and the
// bias table. Chain rule back through the forward's steps ("Video Swin
// Transformer" summary page, Method steps 4-6 and eq. 2): per window and head
// P = softmax(q k^T / sqrt(d) + B) over the query's region, O = P v,
// y = O Wproj + bproj, so
//   dO = dY Wproj^T,   dP = dO v^T,   dS = P * (dP - rowsum(dP * P)),
//   dq = dS k / sqrt(d),   dk = dS^T q / sqrt(d),   dv = P^T dO,
//   dtable[row(i, j)][h] += dS[i][j],   dX = dqkv Wqkv^T,
//   dWqkv = X^T dqkv,  dbqkv = sum of dqkv rows (padding rows included: their
//   q, k, v are the biases), dWproj = O^T dY, dbproj = sum of dY rows.
// The forward is recomputed first (the fp32 path's three kernels), then:
// dO per slot row; a pass per (window, query, head) that rebuilds the query's
// probability row and writes dq, the row's softmax statistics and the table
// gradient (atomics); a pass per (window, key, head) that rebuilds the key's
// column of P and dS from those statistics and writes dk and dv (no atomics);
// dX scattered to the tokens; the weight and bias gradients as row-chunked
// sums (atomics into the caller's zeroed buffers).
#include <cmath>

#include "internal.h"

namespace vswin {

namespace {

constexpr int kT = 128;
constexpr int kGramChunk = 256;  // rows per block of the weight-gradient sums

__device__ float block_sum(float v, float* red) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  __syncthreads();  // red may still be read from a previous call
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  for (int k = 0; k < kT / 32; ++k) s += red[k];
  return s;
}

__device__ float block_max(float v, float* red) {
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
  for (int k = 1; k < kT / 32; ++k) m = fmaxf(m, red[k]);
  return m;
}

// dO[row][c] = sum_j dY[row][j] Wproj[c][j], dY[row] = dy[source(row)] (0 for padding).
__global__ void __launch_bounds__(kT) bwd_dout_kernel(Geom g, const int* __restrict__ src_of,
                                                      const float* __restrict__ dy, const float* __restrict__ Wproj,
                                                      float* __restrict__ dO) {
  extern __shared__ float dyrow[];  // C
  const long long row = blockIdx.x;
  const long long src = src_of[row];
  for (int c = threadIdx.x; c < g.C; c += blockDim.x) dyrow[c] = src >= 0 ? dy[src * g.C + c] : 0.f;
  __syncthreads();
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= g.C) return;
  const float* w = Wproj + (size_t)c * g.C;
  float acc = 0.f;
  for (int j = 0; j < g.C; ++j) acc = fmaf(dyrow[j], w[j], acc);
  dO[row * g.C + c] = acc;
}

// One block per (window, query slot i, head): P[i][:] rebuilt as in the forward,
// dP[i][j] = dO_i . v_j, D_i = sum_j P dP, dS = P (dP - D_i); writes dq_i, the
// statistics (max, 1 / sum, D_i) and adds dS to the table gradient.
__global__ void __launch_bounds__(kT) bwd_attn_rows_kernel(Geom g, const float* __restrict__ qkv,
                                                           const float* __restrict__ table,
                                                           const float* __restrict__ dO, float* __restrict__ dqkv,
                                                           float* __restrict__ dtable, float* __restrict__ stat) {
  extern __shared__ float sm[];
  float* p = sm;             // N: scores, then P, then dS
  float* dp = sm + g.N;      // N
  float* q = dp + g.N;       // d
  float* go = q + g.d;       // d: dO_i
  __shared__ float red[kT / 32];
  const long long win = blockIdx.x;
  const int i = blockIdx.y, h = blockIdx.z;
  const int C3 = 3 * g.C, d = g.d;
  const int w_in_clip = (int)(win % g.nW);
  const bool shifted = (g.sh[0] | g.sh[1] | g.sh[2]) != 0;
  const float* base = qkv + win * g.N * (long long)C3;
  const long long row = win * g.N + i;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    q[c] = base[(size_t)i * C3 + h * d + c];
    go[c] = dO[row * g.C + h * d + c];
  }
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
    p[j] = s;
    m = fmaxf(m, s);
  }
  m = block_max(m, red);
  float sum = 0.f;
  for (int j = threadIdx.x; j < g.N; j += blockDim.x) {
    const float e = p[j] == -INFINITY ? 0.f : expf(p[j] - m);
    p[j] = e;
    sum += e;
  }
  sum = block_sum(sum, red);
  const float inv = 1.0f / sum;
  float dsum = 0.f;
  for (int j = threadIdx.x; j < g.N; j += blockDim.x) {
    const float pj = p[j] * inv;
    float dpj = 0.f;
    if (pj != 0.f) {
      const float* v = base + (size_t)j * C3 + 2 * g.C + h * d;
      for (int c = 0; c < d; ++c) dpj = fmaf(go[c], v[c], dpj);
    }
    p[j] = pj;
    dp[j] = dpj;
    dsum = fmaf(pj, dpj, dsum);
  }
  const float D = block_sum(dsum, red);
  for (int j = threadIdx.x; j < g.N; j += blockDim.x) {
    const float ds = p[j] * (dp[j] - D);
    p[j] = ds;
    if (ds != 0.f) atomicAdd(&dtable[(size_t)bias_row(g, i, j) * g.heads + h], ds);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < g.N; ++j) acc = fmaf(p[j], base[(size_t)j * C3 + g.C + h * d + c], acc);
    dqkv[row * C3 + h * d + c] = acc * scale;
  }
  if (threadIdx.x == 0) {
    float* st = stat + (row * g.heads + h) * 3;
    st[0] = m;
    st[1] = inv;
    st[2] = D;
  }
}

// One block per (window, key slot j, head): column j of P and dS rebuilt from
// the rows' statistics; dk_j = sum_i dS[i][j] q_i / sqrt(d), dv_j = sum_i P[i][j] dO_i.
__global__ void __launch_bounds__(kT) bwd_attn_cols_kernel(Geom g, const float* __restrict__ qkv,
                                                           const float* __restrict__ table,
                                                           const float* __restrict__ dO,
                                                           const float* __restrict__ stat, float* __restrict__ dqkv) {
  extern __shared__ float sm[];
  float* pc = sm;            // N: P[i][j]
  float* dsc = sm + g.N;     // N: dS[i][j]
  float* kj = dsc + g.N;     // d
  float* vj = kj + g.d;      // d
  const long long win = blockIdx.x;
  const int j = blockIdx.y, h = blockIdx.z;
  const int C3 = 3 * g.C, d = g.d;
  const int w_in_clip = (int)(win % g.nW);
  const bool shifted = (g.sh[0] | g.sh[1] | g.sh[2]) != 0;
  const float* base = qkv + win * g.N * (long long)C3;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    kj[c] = base[(size_t)j * C3 + g.C + h * d + c];
    vj[c] = base[(size_t)j * C3 + 2 * g.C + h * d + c];
  }
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)d);
  const int reg_j = shifted ? slot_region(g, w_in_clip, j) : 0;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    float pij = 0.f, dsij = 0.f;
    if (!shifted || slot_region(g, w_in_clip, i) == reg_j) {
      const long long row = win * g.N + i;
      const float* qi = base + (size_t)i * C3 + h * d;
      const float* goi = dO + row * g.C + h * d;
      float dot = 0.f, dpij = 0.f;
      for (int c = 0; c < d; ++c) {
        dot = fmaf(qi[c], kj[c], dot);
        dpij = fmaf(goi[c], vj[c], dpij);
      }
      const float* st = stat + (row * g.heads + h) * 3;
      const float s = dot * scale + table[(size_t)bias_row(g, i, j) * g.heads + h];
      pij = expf(s - st[0]) * st[1];
      dsij = pij * (dpij - st[2]);
    }
    pc[i] = pij;
    dsc[i] = dsij;
  }
  __syncthreads();
  const long long rowj = win * g.N + j;
  for (int c = threadIdx.x; c < 2 * d; c += blockDim.x) {
    float acc = 0.f;
    if (c < d) {
      for (int i = 0; i < g.N; ++i) acc = fmaf(dsc[i], base[(size_t)i * C3 + h * d + c], acc);
      dqkv[rowj * C3 + g.C + h * d + c] = acc * scale;
    } else {
      const int cc = c - d;
      for (int i = 0; i < g.N; ++i) acc = fmaf(pc[i], dO[(win * g.N + i) * g.C + h * d + cc], acc);
      dqkv[rowj * C3 + 2 * g.C + h * d + cc] = acc;
    }
  }
}

// dx[source(row)] = dqkv[row] Wqkv^T for every slot that is not padding.
__global__ void __launch_bounds__(kT) bwd_dx_kernel(Geom g, const int* __restrict__ src_of,
                                                    const float* __restrict__ dqkv, const float* __restrict__ Wqkv,
                                                    float* __restrict__ dx) {
  extern __shared__ float grow[];  // 3C
  const long long row = blockIdx.x;
  const long long dst = src_of[row];
  if (dst < 0) return;  // uniform over the block
  const int C3 = 3 * g.C;
  for (int c = threadIdx.x; c < C3; c += blockDim.x) grow[c] = dqkv[row * C3 + c];
  __syncthreads();
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= g.C) return;
  const float* w = Wqkv + (size_t)c * C3;
  float acc = 0.f;
  for (int j = 0; j < C3; ++j) acc = fmaf(grow[j], w[j], acc);
  dx[dst * g.C + c] = acc;
}

// out[c][j] += sum over this block's rows r of a(r, c) b(r, j), and for c == K1
// bias_out[j] += sum of b(r, j) over rows whose a-row exists or, with
// bias_all_rows, over every row. a(r, c) = A[a_row(r) * K1 + c], a_row(r) =
// a_src ? a_src[r] : r (0 when a_row < 0); b likewise with b_src.
__global__ void __launch_bounds__(kT) bwd_gram_kernel(long long rows, int K1, int K2, const float* __restrict__ A,
                                                      const int* __restrict__ a_src, const float* __restrict__ Bm,
                                                      const int* __restrict__ b_src, int bias_all_rows,
                                                      float* __restrict__ out, float* __restrict__ bias_out,
                                                      int chunk) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = blockIdx.y;  // 0..K1 (K1 = the bias row)
  const long long r0 = (long long)blockIdx.z * chunk;
  long long r1 = r0 + chunk;
  if (r1 > rows) r1 = rows;
  if (j >= K2) return;
  float acc = 0.f;
  for (long long r = r0; r < r1; ++r) {
    const long long ar = a_src ? a_src[r] : r;
    const long long br = b_src ? b_src[r] : r;
    if (br < 0) continue;
    float av;
    if (c == K1) av = (bias_all_rows || ar >= 0) ? 1.f : 0.f;
    else av = ar >= 0 ? A[ar * K1 + c] : 0.f;
    acc = fmaf(av, Bm[br * K2 + j], acc);
  }
  atomicAdd(c == K1 ? &bias_out[j] : &out[(size_t)c * K2 + j], acc);
}

cudaError_t launch_gram(long long rows, int K1, int K2, const float* A, const int* a_src, const float* Bm,
                        const int* b_src, int bias_all_rows, float* out, float* bias_out, cudaStream_t st) {
  long long chunk = kGramChunk;
  if ((rows + chunk - 1) / chunk > 65535) chunk = (rows + 65534) / 65535;
  const dim3 grid((unsigned)((K2 + kT - 1) / kT), (unsigned)(K1 + 1), (unsigned)((rows + chunk - 1) / chunk));
  prof_begin(kKindOther, st);
  bwd_gram_kernel<<<grid, kT, 0, st>>>(rows, K1, K2, A, a_src, Bm, b_src, bias_all_rows, out, bias_out, (int)chunk);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

size_t f32_backward_scratch_bytes(const Geom& g) {
  const size_t rows = (size_t)g.windows * g.N;
  size_t nq = 0, no = 0;
  f32_scratch_floats(g, &nq, &no);
  const size_t floats = nq + no                 // forward qkv, o
                        + (size_t)g.tokens * g.C  // forward output (not returned)
                        + rows * g.C              // dO
                        + rows * 3 * g.C          // dqkv
                        + rows * g.heads * 3;     // per-row statistics
  return floats * sizeof(float) + rows * sizeof(int) + 256;
}

cudaError_t launch_f32_backward(const Geom& g, const float* x, const float* Wqkv, const float* bqkv,
                                const float* Wproj, const float* bproj, const float* table, const float* dy,
                                float* dx, float* dWqkv, float* dbqkv, float* dWproj, float* dbproj, float* dtable,
                                void* scratch, cudaStream_t st) {
  const long long rows = g.windows * g.N;
  if (rows > 2147483647LL || g.N > 65535) return cudaErrorInvalidConfiguration;
  size_t nq = 0, no = 0;
  f32_scratch_floats(g, &nq, &no);
  float* qkv = static_cast<float*>(scratch);
  float* o = qkv + nq;
  float* fwd_out = o + no;
  float* dO = fwd_out + (size_t)g.tokens * g.C;
  float* dqkv = dO + (size_t)rows * g.C;
  float* stat = dqkv + (size_t)rows * 3 * g.C;
  int* src_of = reinterpret_cast<int*>(stat + (size_t)rows * g.heads * 3);

  cudaError_t e = launch_f32_forward(g, x, Wqkv, bqkv, Wproj, bproj, table, fwd_out, qkv, o, st);
  if (e != cudaSuccess) return e;
  e = launch_index_maps(g, src_of, nullptr, nullptr, st);
  if (e != cudaSuccess) return e;
  const int C = g.C, C3 = 3 * g.C;
  e = cudaMemsetAsync(dWqkv, 0, (size_t)C * C3 * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dbqkv, 0, (size_t)C3 * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dWproj, 0, (size_t)C * C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dbproj, 0, (size_t)C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dtable, 0, (size_t)g.table_rows * g.heads * sizeof(float), st);
  if (e != cudaSuccess) return e;

  prof_begin(kKindOther, st);
  bwd_dout_kernel<<<dim3((unsigned)rows, (C + kT - 1) / kT), kT, C * sizeof(float), st>>>(g, src_of, dy, Wproj, dO);
  prof_end(kKindOther, st);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const dim3 ga((unsigned)g.windows, g.N, g.heads);
  const size_t sm_a = (2 * (size_t)g.N + 2 * g.d) * sizeof(float);
  prof_begin(kKindOther, st);
  bwd_attn_rows_kernel<<<ga, kT, sm_a, st>>>(g, qkv, table, dO, dqkv, dtable, stat);
  prof_end(kKindOther, st);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prof_begin(kKindOther, st);
  bwd_attn_cols_kernel<<<ga, kT, sm_a, st>>>(g, qkv, table, dO, stat, dqkv);
  prof_end(kKindOther, st);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  prof_begin(kKindOther, st);
  bwd_dx_kernel<<<dim3((unsigned)rows, (C + kT - 1) / kT), kT, C3 * sizeof(float), st>>>(g, src_of, dqkv, Wqkv, dx);
  prof_end(kKindOther, st);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // dWqkv = X^T dqkv (X gathered from x), dbqkv over every row (padding included)
  e = launch_gram(rows, C, C3, x, src_of, dqkv, nullptr, 1, dWqkv, dbqkv, st);
  if (e != cudaSuccess) return e;
  // dWproj = O^T dY (dY gathered from dy, zero for padding), dbproj over real rows
  return launch_gram(rows, C, C, o, nullptr, dy, src_of, 0, dWproj, dbproj, st);
}

}  // namespace vswin
