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
// Main path (d <= 32 and the item fits in shared memory):
//   * qkv recomputed by a register-tiled FP32 GEMM over the gathered x rows;
//   * dO = dY Wproj^T by the same GEMM (dY gathered, zero on padding slots);
//   * one block per (window, head) with q, k, v and dO of the item, the head's
//     bias-table column and its gradient resident in shared memory: per query
//     row the softmax statistics, O (written for dWproj), D = dO . O, dS and
//     dq, the table gradient summed in shared memory (one global add per table
//     row per block); per key row dk and dv from P and dS rebuilt from the rows'
//     statistics;
//   * dX = dqkv Wqkv^T scattered to the tokens, and dWqkv = X^T dqkv,
//     dWproj = O^T dY with their bias rows as split-K sums of the GEMM (atomics
//     into the caller's zeroed buffers).
// Otherwise the forward is recomputed by the fp32 forward's kernels and the
// attention gradients come from a pass per (window, query, head) and a pass per
// (window, key, head) over global memory.
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"

namespace vswin {

namespace {

constexpr int kT = 128;

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

// ---------------------------------------------------------------------------
// Shared-memory-resident attention gradient of one (window, head) item.
// Rows are stored with stride DM (d rounded up to 16, zero-padded), so every
// product runs over DM channels with no guards. e[n] = (pt (2Mh-1) + ph)
// (2Mw-1) + pw per slot, so the bias row of (i, j) is e[i] - e[j] + e0 with
// e0 the row of a zero offset.
constexpr int kItemMaxThreads = 416;  // 13 warps (at most 128 registers a thread)

__host__ inline size_t item_smem_bytes(int N, int DM, int table_rows) {
  return (size_t)4 * N * DM * sizeof(float) + (size_t)2 * table_rows * sizeof(float) +
         (size_t)N * (3 * sizeof(float) + 2 * sizeof(int));
}

constexpr float kLog2e = 1.4426950408889634f;

// Hardware base-2 exponential (MUFU ex2, relative error about 2^-22); 2^-inf = 0.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int DM>
__device__ __forceinline__ void load_row(const float* __restrict__ src, float (&r)[DM]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int c = 0; c < DM / 4; ++c) {
    const float4 t = s4[c];
    r[4 * c] = t.x;
    r[4 * c + 1] = t.y;
    r[4 * c + 2] = t.z;
    r[4 * c + 3] = t.w;
  }
}

// Dot product of a register row with a shared-memory row (two partial sums).
template <int DM>
__device__ __forceinline__ float dot_row(const float (&a)[DM], const float* __restrict__ b) {
  const float4* b4 = reinterpret_cast<const float4*>(b);
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int c = 0; c < DM / 4; ++c) {
    const float4 t = b4[c];
    s0 = fmaf(a[4 * c], t.x, s0);
    s1 = fmaf(a[4 * c + 1], t.y, s1);
    s0 = fmaf(a[4 * c + 2], t.z, s0);
    s1 = fmaf(a[4 * c + 3], t.w, s1);
  }
  return s0 + s1;
}

template <int DM>
__device__ __forceinline__ void axpy_row(float (&acc)[DM], float w, const float* __restrict__ b) {
  const float4* b4 = reinterpret_cast<const float4*>(b);
#pragma unroll
  for (int c = 0; c < DM / 4; ++c) {
    const float4 t = b4[c];
    acc[4 * c] = fmaf(w, t.x, acc[4 * c]);
    acc[4 * c + 1] = fmaf(w, t.y, acc[4 * c + 1]);
    acc[4 * c + 2] = fmaf(w, t.z, acc[4 * c + 2]);
    acc[4 * c + 3] = fmaf(w, t.w, acc[4 * c + 3]);
  }
}

template <int DM>
__global__ void __launch_bounds__(kItemMaxThreads) bwd_item_kernel(Geom g, const float* __restrict__ qkv,
                                                                    const float* __restrict__ table,
                                                                    const float* __restrict__ dO,
                                                                    float* __restrict__ o, float* __restrict__ dqkv,
                                                                    float* __restrict__ dtable) {
  extern __shared__ float4 smem4[];
  float* sq = reinterpret_cast<float*>(smem4);
  const int N = g.N, d = g.d, TR = g.table_rows, C = g.C, C3 = 3 * g.C;
  float* sk = sq + N * DM;
  float* sv = sk + N * DM;
  float* sdo = sv + N * DM;
  float* stab = sdo + N * DM;  // the head's column of the table
  float* sgrad = stab + TR;    // its gradient
  float* s_m = sgrad + TR;     // per query row: maximum, 1 / sum, D
  float* s_inv = s_m + N;
  float* s_D = s_inv + N;
  int* se = reinterpret_cast<int*>(s_D + N);
  int* sreg = se + N;
  const long long win = blockIdx.x;
  const int h = blockIdx.y;
  const int w_in_clip = (int)(win % g.nW);
  const bool shifted = (g.sh[0] | g.sh[1] | g.sh[2]) != 0;
  const float* base = qkv + win * (long long)N * C3 + h * d;
  const float* dob = dO + win * (long long)N * C + h * d;
  for (int idx = threadIdx.x; idx < N * DM; idx += blockDim.x) {
    const int n = idx / DM, c = idx - n * DM;
    const bool in = c < d;
    sq[idx] = in ? base[(size_t)n * C3 + c] : 0.f;
    sk[idx] = in ? base[(size_t)n * C3 + C + c] : 0.f;
    sv[idx] = in ? base[(size_t)n * C3 + 2 * C + c] : 0.f;
    sdo[idx] = in ? dob[(size_t)n * C + c] : 0.f;
  }
  for (int r = threadIdx.x; r < TR; r += blockDim.x) {
    stab[r] = table[(size_t)r * g.heads + h] * kLog2e;
    sgrad[r] = 0.f;
  }
  const int nh = 2 * g.win[1] - 1, nww = 2 * g.win[2] - 1;
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    int p[3];
    slot_position(g, n, p);
    se[n] = (p[0] * nh + p[1]) * nww + p[2];
    sreg[n] = shifted ? slot_region(g, w_in_clip, n) : 0;
  }
  __syncthreads();
  const int e0 = ((g.win[0] - 1) * nh + (g.win[1] - 1)) * nww + (g.win[2] - 1);
  const float scale = 1.0f / sqrtf((float)d);
  // Scores are kept in base 2: s2 = (q.k / sqrt(d) + B) log2(e), P = 2^(s2 - max).
  const float scale2 = scale * kLog2e;

  // Every pass runs two adjacent lanes per row, each holding half of the
  // channels; the partial products are exchanged so both lanes form the same
  // scores, P and dS. All lanes of a warp walk the same keys (rows past N are
  // carried along masked), so a key that no row of the warp may see is skipped
  // by the whole warp and the exchanges need no divergence handling.
  constexpr int DH = DM / 2;
  const int half = threadIdx.x & 1;
  const int per_pass = blockDim.x >> 1;

  // ---- query rows: maximum, then sum and O, D; then dS, dq and the table gradient
  for (int i0 = 0; i0 < N; i0 += per_pass) {
    const int i = i0 + (threadIdx.x >> 1);
    const bool valid = i < N;
    const int ic = valid ? i : N - 1;
    const int ei = se[ic] + e0, ri = valid ? sreg[ic] : -1;
    float q[DH];
    load_row<DH>(sq + ic * DM + half * DH, q);
    float m = -INFINITY;
#pragma unroll 2
    for (int j = 0; j < N; ++j) {
      const bool ok = sreg[j] == ri;
      if (!__any_sync(0xffffffffu, ok)) continue;
      float dot = dot_row<DH>(q, sk + j * DM + half * DH);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      const float s2 = fmaf(dot, scale2, stab[ei - se[j]]);
      if (ok) m = fmaxf(m, s2);
    }
    float acc[DH];
#pragma unroll
    for (int c = 0; c < DH; ++c) acc[c] = 0.f;
    float l = 0.f;
#pragma unroll 2
    for (int j = 0; j < N; ++j) {
      const bool ok = sreg[j] == ri;
      if (!__any_sync(0xffffffffu, ok)) continue;
      float dot = dot_row<DH>(q, sk + j * DM + half * DH);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      const float pe = ok ? ex2_approx(fmaf(dot, scale2, stab[ei - se[j]]) - m) : 0.f;
      l += pe;
      axpy_row<DH>(acc, pe, sv + j * DM + half * DH);
    }
    const float inv = 1.0f / l;
    float go[DH];
    load_row<DH>(sdo + ic * DM + half * DH, go);
    float D = 0.f;
    float* orow = o + (win * (long long)N + ic) * C + h * d + half * DH;
#pragma unroll
    for (int c = 0; c < DH; ++c) {
      const float oc = acc[c] * inv;
      D = fmaf(go[c], oc, D);
      if (valid && half * DH + c < d) orow[c] = oc;
    }
    D += __shfl_xor_sync(0xffffffffu, D, 1);
    float dq[DH];
#pragma unroll
    for (int c = 0; c < DH; ++c) dq[c] = 0.f;
#pragma unroll 2
    for (int j = 0; j < N; ++j) {
      const bool ok = sreg[j] == ri;
      if (!__any_sync(0xffffffffu, ok)) continue;
      const int r = ei - se[j];
      const float* kj = sk + j * DM + half * DH;
      float dot = dot_row<DH>(q, kj), dp = dot_row<DH>(go, sv + j * DM + half * DH);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      const float pr = ok ? ex2_approx(fmaf(dot, scale2, stab[r]) - m) * inv : 0.f;
      const float ds = pr * (dp - D);
      axpy_row<DH>(dq, ds, kj);
      if (ok && half == 0) atomicAdd(&sgrad[r], ds);
    }
    if (valid) {
      float* dst = dqkv + (win * (long long)N + i) * C3 + h * d + half * DH;
#pragma unroll
      for (int c = 0; c < DH; ++c)
        if (half * DH + c < d) dst[c] = dq[c] * scale;
      if (half == 0) {
        s_m[i] = m;
        s_inv[i] = inv;
        s_D[i] = D;
      }
    }
  }
  __syncthreads();

  // ---- key rows: dk = sum_i dS q_i / sqrt(d), dv = sum_i P dO_i
  for (int j0 = 0; j0 < N; j0 += per_pass) {
    const int j = j0 + (threadIdx.x >> 1);
    const bool valid = j < N;
    const int jc = valid ? j : N - 1;
    const int ej = se[jc] - e0, rj = valid ? sreg[jc] : -1;
    float k[DH], v[DH], dk[DH], dv[DH];
    load_row<DH>(sk + jc * DM + half * DH, k);
    load_row<DH>(sv + jc * DM + half * DH, v);
#pragma unroll
    for (int c = 0; c < DH; ++c) {
      dk[c] = 0.f;
      dv[c] = 0.f;
    }
#pragma unroll 2
    for (int i = 0; i < N; ++i) {
      const bool ok = sreg[i] == rj;
      if (!__any_sync(0xffffffffu, ok)) continue;
      const float* qi = sq + i * DM + half * DH;
      const float* goi = sdo + i * DM + half * DH;
      float dot = dot_row<DH>(k, qi), dp = dot_row<DH>(v, goi);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      const float pr = ok ? ex2_approx(fmaf(dot, scale2, stab[se[i] - ej]) - s_m[i]) * s_inv[i] : 0.f;
      const float ds = pr * (dp - s_D[i]);
      axpy_row<DH>(dk, ds, qi);
      axpy_row<DH>(dv, pr, goi);
    }
    if (valid) {
      float* dst = dqkv + (win * (long long)N + j) * C3 + h * d + half * DH;
#pragma unroll
      for (int c = 0; c < DH; ++c)
        if (half * DH + c < d) {
          dst[C + c] = dk[c] * scale;
          dst[2 * C + c] = dv[c];
        }
    }
  }
  __syncthreads();
  for (int r = threadIdx.x; r < TR; r += blockDim.x)
    if (sgrad[r] != 0.f) atomicAdd(&dtable[(size_t)r * g.heads + h], sgrad[r]);
}

template <int DM>
cudaError_t launch_item(const Geom& g, const float* qkv, const float* table, const float* dO, float* o,
                        float* dqkv, float* dtable, size_t smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_item_kernel<DM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int threads = (2 * g.N + 31) / 32 * 32;  // two lanes per row
  if (threads > kItemMaxThreads) threads = kItemMaxThreads;
  prof_begin(kKindOther, st);
  bwd_item_kernel<DM><<<dim3((unsigned)g.windows, g.heads), threads, smem, st>>>(g, qkv, table, dO, o, dqkv, dtable);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Register-tiled FP32 GEMM, out = A B, in three operand forms:
//   kRowsNT: A(m, k) = A[row(m) lda + k], B(k, n) = Bm[n ldb + k] (a weight
//            used transposed); out[orow(m) ldo + n] = acc (+ bias[n]), rows
//            with orow(m) < 0 skipped;
//   kRowsNN: as kRowsNT with B(k, n) = Bm[k ldb + n];
//   kGram:   A(m, k) = A[row(k) lda + m] for m < Ma, 1 for m == Ma (the bias
//            row), B(k, n) = Bm[brow(k) ldb + n]; the K range is split over
//            blockIdx.z and each block adds its sums to out[m ldo + n]
//            (bias_out[n] for m == Ma).
// row(i) = a_src ? a_src[i] : i, and a negative row reads zeros (likewise brow
// with b_src). 256 threads, a 128 x 96 tile of 8 x 6 per thread, K in steps of
// 16 through two shared-memory buffers with the next step held in registers.
enum { kRowsNT = 0, kRowsNN = 1, kGram = 2 };
constexpr int kGT = 256, kBK = 16, kTM = 8, kTN = 6, kBM = 16 * kTM, kBN = 16 * kTN;
constexpr int kAS = kBM + 4, kBS = kBN + 4;  // padded shared-memory row strides
constexpr int kAL = kBM * kBK / kGT, kBL = kBN * kBK / kGT;

struct GemmArgs {
  long long M, N, K;  // kGram: M = Ma + 1
  const void* A;      // float or bf16 (the kernel's TA)
  long long lda;
  const int* a_src;
  const void* Bm;     // float or bf16 (the kernel's TB)
  long long ldb;
  const int* b_src;
  const float* bias;
  float* out;
  long long ldo;
  const int* out_src;
  float* bias_out;
  long long kchunk;  // kGram: K rows per block
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <int MODE, class TA>
__device__ __forceinline__ float gemm_a(const GemmArgs& a, long long m, long long k, long long k1) {
  const TA* A = static_cast<const TA*>(a.A);
  if (MODE == kGram) {
    if (k >= k1) return 0.f;
    if (m == a.M - 1) return 1.f;
    if (m >= a.M) return 0.f;
    const long long r = a.a_src ? (long long)a.a_src[k] : k;
    return r >= 0 ? to_f32(A[r * a.lda + m]) : 0.f;
  }
  if (m >= a.M || k >= a.K) return 0.f;
  const long long r = a.a_src ? (long long)a.a_src[m] : m;
  return r >= 0 ? to_f32(A[r * a.lda + k]) : 0.f;
}

template <int MODE, class TB>
__device__ __forceinline__ float gemm_b(const GemmArgs& a, long long k, long long n, long long k1) {
  const TB* Bm = static_cast<const TB*>(a.Bm);
  if (n >= a.N) return 0.f;
  if (MODE == kRowsNT) return k < a.K ? to_f32(Bm[n * a.ldb + k]) : 0.f;
  if (MODE == kRowsNN) return k < a.K ? to_f32(Bm[k * a.ldb + n]) : 0.f;
  if (k >= k1) return 0.f;
  const long long r = a.b_src ? (long long)a.b_src[k] : k;
  return r >= 0 ? to_f32(Bm[r * a.ldb + n]) : 0.f;
}

// Element e of this thread's share of a tile: (kk, mm) with kk fastest when the
// operand is contiguous along K in memory, mm fastest otherwise.
template <bool KFAST, int W>
__device__ __forceinline__ void tile_pos(int e, int& kk, int& mm) {
  const int idx = threadIdx.x + kGT * e;
  if (KFAST) {
    kk = idx % kBK;
    mm = idx / kBK;
  } else {
    mm = idx % W;
    kk = idx / W;
  }
}

template <int MODE, class TA, class TB>
__global__ void __launch_bounds__(kGT) f32_gemm_kernel(GemmArgs a) {
  __shared__ __align__(16) float As[2][kBK][kAS];
  __shared__ __align__(16) float Bs[2][kBK][kBS];
  constexpr bool AK = MODE != kGram;   // A contiguous along K
  constexpr bool BK_ = MODE == kRowsNT;  // B contiguous along K
  const long long m0 = (long long)blockIdx.x * kBM, n0 = (long long)blockIdx.y * kBN;
  long long k0 = 0, k1 = a.K;
  if (MODE == kGram) {
    k0 = (long long)blockIdx.z * a.kchunk;
    k1 = k0 + a.kchunk < a.K ? k0 + a.kchunk : a.K;
  }
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float ra[kAL], rb[kBL];
  auto fetch = [&](long long kb) {
#pragma unroll
    for (int e = 0; e < kAL; ++e) {
      int kk, mm;
      tile_pos<AK, kBM>(e, kk, mm);
      ra[e] = gemm_a<MODE, TA>(a, m0 + mm, kb + kk, k1);
    }
#pragma unroll
    for (int e = 0; e < kBL; ++e) {
      int kk, nn;
      tile_pos<BK_, kBN>(e, kk, nn);
      rb[e] = gemm_b<MODE, TB>(a, kb + kk, n0 + nn, k1);
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int e = 0; e < kAL; ++e) {
      int kk, mm;
      tile_pos<AK, kBM>(e, kk, mm);
      As[buf][kk][mm] = ra[e];
    }
#pragma unroll
    for (int e = 0; e < kBL; ++e) {
      int kk, nn;
      tile_pos<BK_, kBN>(e, kk, nn);
      Bs[buf][kk][nn] = rb[e];
    }
  };
  float acc[kTM][kTN];
#pragma unroll
  for (int i = 0; i < kTM; ++i)
#pragma unroll
    for (int j = 0; j < kTN; ++j) acc[i][j] = 0.f;
  int buf = 0;
  if (k0 < k1) {
    fetch(k0);
    stash(0);
  }
  __syncthreads();
  for (long long kb = k0; kb < k1; kb += kBK) {
    const bool more = kb + kBK < k1;
    if (more) fetch(kb + kBK);
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * kTM]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * kTM + 4]);
      const float2 b0 = *reinterpret_cast<const float2*>(&Bs[buf][kk][tx * kTN]);
      const float2 b1 = *reinterpret_cast<const float2*>(&Bs[buf][kk][tx * kTN + 2]);
      const float2 b2 = *reinterpret_cast<const float2*>(&Bs[buf][kk][tx * kTN + 4]);
      const float av[kTM] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[kTN] = {b0.x, b0.y, b1.x, b1.y, b2.x, b2.y};
#pragma unroll
      for (int i = 0; i < kTM; ++i)
#pragma unroll
        for (int j = 0; j < kTN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) {
      stash(buf ^ 1);
      buf ^= 1;
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kTM; ++i) {
    const long long m = m0 + ty * kTM + i;
    if (m >= a.M) continue;
    if (MODE == kGram) {
      float* dst = m == a.M - 1 ? a.bias_out : a.out + m * a.ldo;
#pragma unroll
      for (int j = 0; j < kTN; ++j) {
        const long long n = n0 + tx * kTN + j;
        if (n < a.N) atomicAdd(&dst[n], acc[i][j]);
      }
    } else {
      const long long r = a.out_src ? (long long)a.out_src[m] : m;
      if (r < 0) continue;
      float* dst = a.out + r * a.ldo;
#pragma unroll
      for (int j = 0; j < kTN; ++j) {
        const long long n = n0 + tx * kTN + j;
        if (n < a.N) dst[n] = acc[i][j] + (a.bias ? a.bias[n] : 0.f);
      }
    }
  }
}

template <int MODE, class TA = float, class TB = float>
cudaError_t launch_gemm(GemmArgs a, cudaStream_t st) {
  const long long gx = (a.M + kBM - 1) / kBM, gy = (a.N + kBN - 1) / kBN;
  long long gz = 1;
  if (MODE == kGram) {
    // about two blocks per SM in all, each over a multiple of 16 rows of K
    long long want = (296 + gx * gy - 1) / (gx * gy);
    long long chunk = (a.K + want - 1) / want;
    chunk = (chunk + kBK - 1) / kBK * kBK;
    if (chunk < kBK) chunk = kBK;
    a.kchunk = chunk;
    gz = (a.K + chunk - 1) / chunk;
    if (gz < 1) gz = 1;
  }
  if (gx > 2147483647LL || gy > 65535 || gz > 65535) return cudaErrorInvalidConfiguration;
  prof_begin(kKindOther, st);
  f32_gemm_kernel<MODE, TA, TB><<<dim3((unsigned)gx, (unsigned)gy, (unsigned)gz), kGT, 0, st>>>(a);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gram_bf16(long long rows, int M, int N, const void* A, long long lda, const int* a_src,
                             const void* B, long long ldb, const int* b_src, float* out, float* bias_out,
                             cudaStream_t st) {
  GemmArgs ga{};
  ga.M = M + 1, ga.N = N, ga.K = rows, ga.A = A, ga.lda = lda, ga.a_src = a_src, ga.Bm = B, ga.ldb = ldb;
  ga.b_src = b_src, ga.out = out, ga.ldo = N, ga.bias_out = bias_out;
  return launch_gemm<kGram, __nv_bfloat16, __nv_bfloat16>(ga, st);
}

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

  cudaError_t e = launch_index_maps(g, src_of, nullptr, nullptr, st);
  if (e != cudaSuccess) return e;
  const int C = g.C, C3 = 3 * g.C;
  e = cudaMemsetAsync(dWqkv, 0, (size_t)C * C3 * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dbqkv, 0, (size_t)C3 * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dWproj, 0, (size_t)C * C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dbproj, 0, (size_t)C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dtable, 0, (size_t)g.table_rows * g.heads * sizeof(float), st);
  if (e != cudaSuccess) return e;

  // the resident (window, head) kernel when its rows fit in one block's shared memory
  const int DM = g.d <= 16 ? 16 : (g.d <= 32 ? 32 : 0);
  int dev = 0, optin = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const size_t item_smem = DM ? item_smem_bytes(g.N, DM, g.table_rows) : 0;
  const bool resident = DM != 0 && item_smem <= (size_t)optin && g.heads <= 65535;

  if (resident) {
    // qkv = X Wqkv + bqkv over the gathered slots (a padding slot's row is the bias)
    GemmArgs q{};
    q.M = rows, q.N = C3, q.K = C, q.A = x, q.lda = C, q.a_src = src_of, q.Bm = Wqkv, q.ldb = C3, q.bias = bqkv;
    q.out = qkv, q.ldo = C3;
    if ((e = launch_gemm<kRowsNN>(q, st)) != cudaSuccess) return e;
  } else {
    e = launch_f32_forward(g, x, Wqkv, bqkv, Wproj, bproj, table, fwd_out, qkv, o, st);
    if (e != cudaSuccess) return e;
  }
  // dO = dY Wproj^T, dY gathered from dy (zero on padding slots)
  GemmArgs go{};
  go.M = rows, go.N = C, go.K = C, go.A = dy, go.lda = C, go.a_src = src_of, go.Bm = Wproj, go.ldb = C;
  go.out = dO, go.ldo = C;
  if ((e = launch_gemm<kRowsNT>(go, st)) != cudaSuccess) return e;

  if (resident) {
    e = DM == 16 ? launch_item<16>(g, qkv, table, dO, o, dqkv, dtable, item_smem, st)
                 : launch_item<32>(g, qkv, table, dO, o, dqkv, dtable, item_smem, st);
    if (e != cudaSuccess) return e;
  } else {
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
  }

  // dX[source(row)] = dqkv[row] Wqkv^T for every slot that is not padding
  GemmArgs gx{};
  gx.M = rows, gx.N = C, gx.K = C3, gx.A = dqkv, gx.lda = C3, gx.Bm = Wqkv, gx.ldb = C3;
  gx.out = dx, gx.ldo = C, gx.out_src = src_of;
  if ((e = launch_gemm<kRowsNT>(gx, st)) != cudaSuccess) return e;
  // dWqkv = X^T dqkv (X gathered from x), dbqkv over every slot (padding included)
  GemmArgs gw{};
  gw.M = C + 1, gw.N = C3, gw.K = rows, gw.A = x, gw.lda = C, gw.a_src = src_of, gw.Bm = dqkv, gw.ldb = C3;
  gw.out = dWqkv, gw.ldo = C3, gw.bias_out = dbqkv;
  if ((e = launch_gemm<kGram>(gw, st)) != cudaSuccess) return e;
  // dWproj = O^T dY, dbproj over the slots that are not padding (dY is zero there)
  GemmArgs gp{};
  gp.M = C + 1, gp.N = C, gp.K = rows, gp.A = o, gp.lda = C, gp.Bm = dy, gp.ldb = C, gp.b_src = src_of;
  gp.out = dWproj, gp.ldo = C, gp.bias_out = dbproj;
  return launch_gemm<kGram>(gp, st);
}

}  // namespace vswin
