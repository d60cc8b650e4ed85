// Patch merging between stages on sm_100a tensor cores ("Video Swin
// Transformer" summary page, Method step 2: each 2x2 group of spatial
// neighbours, 4C values, projected to 2C by a linear layer, no temporal
// merging; the code walk-through page, section 1.2: PatchMerging is
// nn.LayerNorm over the 4C values, then nn.Linear(4C, 2C)):
//
//   out[b, t, i, j] = LN(cat(x[2i, 2j], x[2i+1, 2j], x[2i, 2j+1], x[2i+1, 2j+1])) Wr (+ br)
//
// with x[h, w] = 0 beyond an odd H or W. The norm is folded into the weights
// (the same algebra as the block's pre-norm: LN(a) Wr = rstd (a Wt - mean
// colsum(Wt)) + beta Wr with Wt = diag(gamma) Wr), so the GEMM reads the raw
// gathered tokens and each row's mean and rstd are computed from the very
// values the tensor core consumes, as they pass through shared memory.
//
// One CTA = 128 merged tokens x BN output columns, 128 threads. Each thread
// owns one merged token: it gathers that row's 16-byte chunks with cp.async
// (zero-fill for padding), later reads them back from shared memory for the
// row statistics (Welford per 32-value block, merged with Chan's formula),
// and in the epilogue holds that row's TMEM lane. Thread 0 issues the MMAs.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vswin {
namespace {

constexpr int kPmBM = 128, kPmBK = 32, kPmStages = 4, kPmThreads = 128;
constexpr int kPmMaxBN = 256;
constexpr int kPmAStage = kPmBM * kPmBK * 2;      // 8 KB
constexpr int kPmBStage = kPmBK * kPmMaxBN * 2;   // 16 KB

__host__ __device__ constexpr int pm_smem_bytes() { return kPmStages * (kPmAStage + kPmBStage) + 4 * kPmBM * 8 + 256; }

__device__ __forceinline__ uint32_t pm_pack(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct PmArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* wt;  // [4C][2C] diag(gamma) Wr, bf16
  const float* colsum;      // [2C] column sums of wt
  const float* bias;        // [2C] beta Wr + br
  __nv_bfloat16* out;       // [rows][2C]
  long long rows;           // B * T * Hh * Wh
  int T, H, W, C, Hh, Wh, BN;
  float eps;
  KernelCtx ctx;
};

__global__ void __launch_bounds__(kPmThreads) pm_kernel(PmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPmStages * kPmAStage;
  long long* s_src = reinterpret_cast<long long*>(sB + kPmStages * kPmBStage);  // [4][128] element offsets
  uint64_t* bar_free = reinterpret_cast<uint64_t*>(s_src + 4 * kPmBM);            // [stages]
  uint64_t* bar_done = bar_free + kPmStages;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_done + 1);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long m0 = (long long)blockIdx.x * kPmBM;
  const int n0 = blockIdx.y * a.BN;
  const int BN = a.BN, C = a.C, N2 = 2 * C, K = 4 * C;
  const uint32_t tcols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;

  // the four source tokens of this thread's merged row, in the order
  // (dh, dw) = (0,0), (1,0), (0,1), (1,1): element offset or -1 (zero)
  {
    const long long r = m0 + tid;
    long long src[4] = {-1, -1, -1, -1};
    if (r < a.rows) {
      const long long j = r % a.Wh, i = (r / a.Wh) % a.Hh, bt = r / ((long long)a.Wh * a.Hh);
      for (int q = 0; q < 4; ++q) {
        const long long h = 2 * i + (q & 1), w = 2 * j + (q >> 1);
        if (h < a.H && w < a.W) src[q] = ((bt * a.H + h) * a.W + w) * (long long)C;
        // extent: the B * T clips' H * W tokens of C channels
        if (!index_ok(src[q], -1, a.rows / ((long long)a.Hh * a.Wh) * a.H * a.W * C, a.ctx.err)) src[q] = -1;
      }
    }
    for (int q = 0; q < 4; ++q) s_src[q * kPmBM + tid] = src[q];
  }
  if (tid == 0) {
    for (int s = 0; s < kPmStages; ++s) mbar_init(&bar_free[s], 1);
    mbar_init(bar_done, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  const int KB = K / kPmBK;
  const uint32_t lboB = (uint32_t)(BN / 8) * 128u;
  const int bchunks = kPmBK * (BN / 8);
  // A stage: row r's chunk kc (8 channels) at (r / 8) * 512 + kc * 128 + (r % 8) * 16
  auto a_chunk = [&](int s, int row, int kc) { return sA + s * kPmAStage + (row >> 3) * 512 + kc * 128 + (row & 7) * 16; };
  auto load_stage = [&](int kb, int s) {
    const int k0 = kb * kPmBK;
    const int q = k0 / C, c0 = k0 - q * C;  // a K block lies inside one neighbour (C % 32 == 0)
    const long long src = s_src[q * kPmBM + tid];
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      const __nv_bfloat16* p = a.x + (src < 0 ? 0 : src + c0 + kc * 8);
      cp_async_16(a_chunk(s, tid, kc), p, src < 0 ? 0u : 16u);
    }
    uint8_t* dB = sB + s * kPmBStage;
    for (int c = tid; c < bchunks; c += kPmThreads) {
      const int kk = c / (BN / 8), nc = c % (BN / 8);
      cp_async_16(dB + (kk >> 3) * lboB + nc * 128 + (kk & 7) * 16, a.wt + (size_t)(k0 + kk) * N2 + n0 + nc * 8, 16u);
    }
  };

  // running statistics of this thread's row (Welford blocks merged by Chan's rule)
  float mean = 0.f, m2 = 0.f, cnt = 0.f;
  const uint32_t idesc = idesc_bf16(kPmBM, BN, 0, 1);
#pragma unroll 1
  for (int p = 0; p < kPmStages - 1; ++p) {
    if (p < KB) load_stage(p, p);
    cp_async_commit();
  }
#pragma unroll 1
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kPmStages;
    cp_async_wait<kPmStages - 2>();
    // this thread's own 32 values of stage s (it issued their copies)
    {
      float v[32];
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        const uint4 w = *reinterpret_cast<const uint4*>(a_chunk(s, tid, kc));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          v[kc * 8 + 2 * e] = f.x;
          v[kc * 8 + 2 * e + 1] = f.y;
        }
      }
      float bs = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) bs += v[e];
      const float bm = bs * (1.0f / 32.0f);
      float bq = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) bq = fmaf(v[e] - bm, v[e] - bm, bq);
      const float n = cnt + 32.f;
      const float d = bm - mean;
      mean += d * (32.f / n);
      m2 += bq + d * d * (cnt * 32.f / n);
      cnt = n;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && !s_abort) {
      tc_fence_after();
      const uint32_t aaddr = smem_u32(sA + s * kPmAStage);
      const uint32_t baddr = smem_u32(sB + s * kPmBStage);
#pragma unroll
      for (int ks = 0; ks < kPmBK / 16; ++ks)
        umma_ss(tmem, smem_desc(aaddr + ks * 256, 128, 512), smem_desc(baddr + ks * 2 * lboB, lboB, 128), idesc,
                (kb | ks) != 0);
      umma_commit(&bar_free[s]);
    }
    const int nk = kb + kPmStages - 1;
    if (nk < KB) {
      const int ns = nk % kPmStages;
      if (kb >= 1 && !s_abort &&
          !mbar_wait(&bar_free[ns], ((kb - 1) / kPmStages) & 1, a.ctx.err, kErrWaitMma, a.ctx.wait_limit))
        s_abort = 1;
      load_stage(nk, ns);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (tid == 0 && !s_abort) umma_commit(bar_done);
  __syncthreads();
  if (!s_abort && !mbar_wait(bar_done, 0, a.ctx.err, kErrWaitMma, a.ctx.wait_limit)) s_abort = 1;
  __syncthreads();
  tc_fence_after();

  // epilogue: rstd * acc + (-mean * rstd) * colsum + bias for this thread's row
  const long long r = m0 + tid;
  if (!s_abort && m0 + warp * 32 < a.rows) {
    const float rstd = 1.0f / sqrtf(m2 / (float)K + a.eps);
    const float ns = -mean * rstd;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c = 0; c < BN / 16; ++c) {
      uint32_t u[16];
      tmem_ld16(trow + c * 16, u);
      tmem_wait_ld();
      if (r < a.rows) {
        const int col = n0 + c * 16;
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float v0 = fmaf(rstd, __uint_as_float(u[2 * k]), fmaf(ns, a.colsum[col + 2 * k], a.bias[col + 2 * k]));
          const float v1 =
              fmaf(rstd, __uint_as_float(u[2 * k + 1]), fmaf(ns, a.colsum[col + 2 * k + 1], a.bias[col + 2 * k + 1]));
          w[k] = pm_pack(v0, v1);
        }
        uint4* o = reinterpret_cast<uint4*>(a.out + r * N2 + col);
        o[0] = make_uint4(w[0], w[1], w[2], w[3]);
        o[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tcols);
}

// Wt = bf16(diag(gamma) Wr), colsum of the rounded Wt, bias = beta Wr + br
// (br may be null). Block (32 x 32): 32 output columns, the K rows split over
// 32 thread rows (independent loads), partial sums reduced in shared memory.
constexpr int kPmFoldCols = 32, kPmFoldRows = 32;
__global__ void __launch_bounds__(kPmFoldCols * kPmFoldRows)
    pm_fold_kernel(int K, int N2, const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                   const __nv_bfloat16* __restrict__ Wr, const __nv_bfloat16* __restrict__ br,
                   __nv_bfloat16* __restrict__ wt, float* __restrict__ colsum, float* __restrict__ bias) {
  __shared__ float s_cs[kPmFoldRows][kPmFoldCols + 1], s_bb[kPmFoldRows][kPmFoldCols + 1];
  const int tx = threadIdx.x % kPmFoldCols, ty = threadIdx.x / kPmFoldCols;
  const int j = blockIdx.x * kPmFoldCols + tx;
  float cs = 0.f, bb = 0.f;
  if (j < N2) {
    for (int k = ty; k < K; k += kPmFoldRows) {
      const float w = __bfloat162float(Wr[(size_t)k * N2 + j]);
      const __nv_bfloat16 wg = __float2bfloat16_rn(__bfloat162float(gamma[k]) * w);
      wt[(size_t)k * N2 + j] = wg;
      cs += __bfloat162float(wg);
      bb = fmaf(__bfloat162float(beta[k]), w, bb);
    }
  }
  s_cs[ty][tx] = cs;
  s_bb[ty][tx] = bb;
  __syncthreads();
  if (ty == 0 && j < N2) {
    for (int k = 1; k < kPmFoldRows; ++k) {
      cs += s_cs[k][tx];
      bb += s_bb[k][tx];
    }
    colsum[j] = cs;
    bias[j] = bb + (br ? __bfloat162float(br[j]) : 0.f);
  }
}

}  // namespace

bool patch_merge_supported(int C) { return C >= 32 && C % 32 == 0 && 2 * C <= 4096; }

size_t patch_merge_scratch_bytes(int C) {
  const size_t wt = ((size_t)4 * C * 2 * C * 2 + 255) / 256 * 256;
  const size_t vec = ((size_t)2 * C * 4 + 255) / 256 * 256;
  return wt + 2 * vec;
}

cudaError_t launch_patch_merge(const KernelCtx& ctx, int B, int T, int H, int W, int C, const void* x,
                               const void* gamma, const void* beta, float eps, const void* Wr, const void* br,
                               void* out, void* scratch, cudaStream_t st) {
  const int N2 = 2 * C, K = 4 * C;
  const size_t wt_bytes = ((size_t)K * N2 * 2 + 255) / 256 * 256;
  const size_t vec = ((size_t)N2 * 4 + 255) / 256 * 256;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  PmArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.wt = reinterpret_cast<const __nv_bfloat16*>(base);
  a.colsum = reinterpret_cast<const float*>(base + wt_bytes);
  a.bias = reinterpret_cast<const float*>(base + wt_bytes + vec);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.T = T;
  a.H = H;
  a.W = W;
  a.C = C;
  a.Hh = (H + 1) / 2;
  a.Wh = (W + 1) / 2;
  a.rows = (long long)B * T * a.Hh * a.Wh;
  a.BN = N2 <= kPmMaxBN ? N2 : kPmMaxBN;
  while (N2 % a.BN) a.BN -= 16;
  a.eps = eps;
  a.ctx = ctx;
  prof_begin(kKindOther, st);
  pm_fold_kernel<<<(N2 + kPmFoldCols - 1) / kPmFoldCols, kPmFoldCols * kPmFoldRows, 0, st>>>(
      K, N2, static_cast<const __nv_bfloat16*>(gamma), static_cast<const __nv_bfloat16*>(beta),
      static_cast<const __nv_bfloat16*>(Wr), static_cast<const __nv_bfloat16*>(br),
      reinterpret_cast<__nv_bfloat16*>(base), reinterpret_cast<float*>(base + wt_bytes),
      reinterpret_cast<float*>(base + wt_bytes + vec));
  prof_end(kKindOther, st);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(pm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pm_smem_bytes());
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((a.rows + kPmBM - 1) / kPmBM), (unsigned)(N2 / a.BN));
  prof_begin(kKindMlp, st);
  pm_kernel<<<grid, kPmThreads, pm_smem_bytes(), st>>>(a);
  prof_end(kKindMlp, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace vswin
