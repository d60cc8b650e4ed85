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
// Two kernels compute it. pm_ws_kernel (persistent, warp-specialised, the
// weights' column slice resident in shared memory; described above it) runs
// whenever that slice fits; pm_kernel, the tiled form, takes the widest
// channel counts. pm_kernel: one CTA = 128 merged tokens x BN output columns,
// 128 threads. Each thread owns one merged token: it gathers that row's 16-byte
// chunks with cp.async (zero-fill for padding), later reads them back from
// shared memory for the row statistics (Welford per 32-value block, merged with
// Chan's formula), and in the epilogue holds that row's TMEM lane. Thread 0
// issues the MMAs. pm_kernel and the cp.async form of pm_ws_kernel take the
// same steps in the same order (32-channel K blocks, MMAs, statistics,
// epilogue), so they give the same bits; the TMA form takes the K blocks in
// the order (dh, dw, c), 64 channels at a time, so its sums round differently.
#include <cuda.h>
#include <cstring>
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

  const int tid = threadIdx.x, warp = tid >> 5;
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

// ---------------------------------------------------------------------------
// Persistent form (used whenever a BN-column slice of the folded weights fits in
// shared memory next to four A stages): one CTA per SM keeps its K x BN weight
// slice resident and walks row tiles, with the roles in warps of their own:
//
//   warps 0-3   gather: the K blocks (32 or 64 channels, below) of a tile's
//               merged rows into a ring of A stages
//   warp 4      MMA issue (one thread): two or four K = 16 steps a K block
//               into one of two TMEM accumulators
//   warps 5-8   row statistics (thread = row): each K block's values read
//               back from the stage, 32 at a time (Welford block, Chan's
//               merge -- the tiled kernel's arithmetic)
//   warps 9-16  epilogue: rstd * acc + (-mean * rstd) * colsum + bias, bf16,
//               16-byte stores of the merged rows (two warps a lane quarter)
//
// A stage is refilled once the MMA (commit) and the four statistics warps have
// released it; an accumulator once its eight epilogue warps have read it.
//
// Two gathers. With even H and W (every Video Swin stage that merges) the 2x2
// neighbours are a plain view of x: x[bt, 2i + dh, 2j + dw, c] is the element
// (dw * C + c, j, dh, bt * H/2 + i) of a 4-D tensor with byte strides (2, 4C,
// 2WC, 4WC) -- the 2C channels of the token pair (2j, 2j + 1) are contiguous.
// One TMA box (64 channels, Wh columns j, one dh, Lt lines) brings a K block
// of a tile of Lt whole lines of merged tokens (Lt * Wh <= 128 rows) into the
// stage, 128-byte swizzled (rows of 128 bytes, 16-byte chunk index XORed with
// the row's low three bits) -- one instruction a K block, issued by one thread;
// the K order is then (dh, dw, c) and the weight fold permutes Wr's rows to
// match. Otherwise the four gather warps move 128-row tiles with cp.async (4
// lanes a row, 64 contiguous bytes a row and instruction, zero-fill for
// padding) in the pages' K order into the no-swizzle core-matrix layout.
// K block: 32 channels (cp.async gather) or 64 (TMA gather); A stage 8 or 16 KB
__host__ __device__ constexpr int pw_bk(bool tma) { return tma ? 64 : 32; }
__host__ __device__ constexpr int pw_stage_bytes(bool tma) { return kPmBM * pw_bk(tma) * 2; }
constexpr int kPwProdWarps = 4, kPwMmaWarp = 4, kPwStat0 = 5, kPwEpi0 = 9, kPwEpiWarps = 8;
constexpr int kPwThreads = 32 * (kPwEpi0 + kPwEpiWarps);  // 544
constexpr int kPwMaxStages = 8, kPwMinStages = 4;
constexpr int kPwSmemMax = 227 * 1024 - 2048;  // dynamic bytes (the static area takes 1 KB more)

__host__ __device__ constexpr int pw_b_bytes(int K, int BN) { return (K * BN * 2 + 1023) / 1024 * 1024; }
// everything after the A ring: colsum and bias (2 x BN floats), the statistics
// ring (2 x 128 float2), the barriers and the TMEM address
__host__ __device__ constexpr int pw_tail_bytes(int BN) { return 2 * BN * 4 + 2 * kPmBM * 8 + 64 * 8 + 16; }
__host__ __device__ constexpr int pw_smem_bytes(int K, int BN, int NS, bool tma) {
  return pw_b_bytes(K, BN) + NS * pw_stage_bytes(tma) + pw_tail_bytes(BN);
}

struct PwArgs {
  PmArgs p;
  int NS;            // A stages
  int NT;            // column tiles (2C / BN); the grid is a multiple of NT
  int TR;            // merged rows a tile (128; TMA gather: Lt * Wh)
  int Lt;            // TMA gather: lines of merged tokens a tile
  long long mtiles;  // row tiles
};

// K-major, 128-byte swizzle tcgen05 descriptor: LBO 16 B (unused inside one
// swizzle atom), SBO 1024 B (8 rows x 128 B), layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t pw_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void pw_tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                               uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait for the roles that wait long (gather, statistics, epilogue):
// try_wait with a suspend-time hint, so that a waiting warp sleeps until the
// phase completes (or the hint runs out) instead of spinning in the issue
// slots the MMA thread of its sub-partition needs. Gives up after limit_ns
// like mbar_wait.
__device__ __forceinline__ bool pw_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool pw_wait(uint64_t* bar, uint32_t parity, int* err, int code, uint64_t limit_ns) {
  if (pw_try_wait_sleep(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!pw_try_wait_sleep(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) {
      atomicCAS(err, 0, code);
      return false;
    }
  }
  return true;
}

// Position in the ring of A stages: stage s, parity of its use count, and
// whether every stage has been used once (kept incrementally: a division of
// the 64-bit K-block count on every step cost hundreds of cycles).
struct RingPos {
  int s = 0;
  uint32_t par = 0;
  bool wrapped = false;
  __device__ __forceinline__ void next(int ns) {
    if (++s == ns) {
      s = 0;
      par ^= 1u;
      wrapped = true;
    }
  }
};

template <bool kTma>
__global__ void __launch_bounds__(kPwThreads, 1) pm_ws_kernel(const __grid_constant__ CUtensorMap tm_x, PwArgs w) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const PmArgs& a = w.p;
  const int NS = w.NS, NT = w.NT, TR = w.TR;
  constexpr int kBK = pw_bk(kTma), kStage = pw_stage_bytes(kTma);
  const int BN = a.BN, C = a.C, N2 = 2 * C, K = 4 * C, KB = K / kBK;
  uint8_t* sB = smem;                                      // K x BN, MN-major operand layout
  uint8_t* sA = smem + pw_b_bytes(K, BN);                  // NS x (128 x kBK), K-major
  float* sCs = reinterpret_cast<float*>(sA + NS * kStage);     // [BN] colsum
  float* sBias = sCs + BN;                                     // [BN] bias
  float2* sStats = reinterpret_cast<float2*>(sBias + BN);      // [2][128] (-mean * rstd, rstd)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStats + 2 * kPmBM);
  uint64_t* b_full = bars;                   // resident weights landed (128 gathering threads)
  uint64_t* a_full = bars + 1;               // [NS] stage landed (TMA bytes, or 128 gathering threads)
  uint64_t* a_free = a_full + NS;            // [NS] stage read: MMA commit + 4 statistics warps
  uint64_t* acc_full = a_free + NS;          // [2] MMA commit
  uint64_t* acc_free = acc_full + 2;         // [2] 8 epilogue warps
  uint64_t* st_full = acc_free + 2;          // [2] 128 statistics threads
  uint64_t* st_free = st_full + 2;           // [2] 256 epilogue threads
  uint64_t* mma_done = st_free + 2;          // every MMA of this CTA completed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(mma_done + 1);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = blockIdx.x % NT, n0 = nt * BN;
  const long long mtiles = w.mtiles;
  const long long m_first = blockIdx.x / NT, m_step = gridDim.x / NT;
  const uint64_t lim = a.ctx.wait_limit;
  const uint32_t lboB = (uint32_t)(BN / 8) * 128u;  // B: K-group stride
  const uint32_t tcols = 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  // byte offset of 16-byte chunk kc (channels 8kc .. 8kc+7 of the K block) of
  // tile row p inside a stage: 128-byte rows with the chunk index XORed with
  // the row's low three bits (TMA, SWIZZLE_128B), or 8 x 16-byte core matrices
  auto a_off = [&](int p, int kc) -> int {
    return kTma ? p * 128 + ((kc ^ (p & 7)) << 4) : (p >> 3) * 512 + kc * 128 + (p & 7) * 16;
  };

  if (tid == 0) {
    mbar_init(b_full, kPwProdWarps * 32);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&a_full[s], kTma ? 1 : kPwProdWarps * 32);
      mbar_init(&a_free[s], 1 + 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_free[b], kPwEpiWarps);
      mbar_init(&st_full[b], 4 * 32);
      mbar_init(&st_free[b], kPwEpiWarps * 32);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  for (int c = tid; c < BN; c += kPwThreads) {
    sCs[c] = a.colsum[n0 + c];
    sBias[c] = a.bias[n0 + c];
  }
  if (warp == kPwMmaWarp) {
    tmem_alloc(s_tmem, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const long long x_extent = a.rows / ((long long)a.Hh * a.Wh) * a.H * a.W * C;

  if (warp < kPwProdWarps) {
    // ---------------------------------------------------------------- gather
    for (int c = tid; c < K * (BN / 8); c += kPwProdWarps * 32) {
      const int kk = c / (BN / 8), nc = c % (BN / 8);
      cp_async_16(sB + (kk >> 3) * lboB + nc * 128 + (kk & 7) * 16, a.wt + (size_t)kk * N2 + n0 + nc * 8, 16u);
    }
    cp_async_mbar_arrive_noinc(b_full);
    if (kTma) {
      if (tid == 0) {
        const uint32_t box_bytes = (uint32_t)TR * 128u;
        RingPos rp;
        for (long long m = m_first; m < mtiles; m += m_step) {
          // K order (dh, dw, c): a block of 64 of the 2C contiguous channels of
          // the (2j, 2j+1) token pair in row 2i + dh
          int dh = 0, c0 = 0;
          for (int kb = 0; kb < KB; ++kb, rp.next(NS)) {
            if (rp.wrapped && !s_abort &&
                !pw_wait(&a_free[rp.s], rp.par ^ 1u, a.ctx.err, kErrWaitMma, lim))
              s_abort = 1;
            if (!s_abort) {
              mbar_arrive_expect_tx(&a_full[rp.s], box_bytes);
              pw_tma_load_4d(sA + rp.s * kStage, &tm_x, c0, 0, dh, (int)(m * w.Lt), &a_full[rp.s]);
            }
            c0 += kBK;
            if (c0 == N2) {
              c0 = 0;
              ++dh;
            }
          }
        }
      }
    } else {
      const int sub = lane >> 2, cq = lane & 3;
      RingPos rp;
      for (long long m = m_first; m < mtiles; m += m_step) {
        // this lane's four rows: element offset of the (0, 0) neighbour (-1 past the
        // end) and whether the +1 row (bit 0) and +1 column (bit 1) neighbours exist
        long long base[4];
        int has[4];
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
          const long long r = m * kPmBM + warp * 32 + grp * 8 + sub;
          base[grp] = -1;
          has[grp] = 0;
          if (r < a.rows) {
            const long long j = r % a.Wh, i = (r / a.Wh) % a.Hh, bt = r / ((long long)a.Wh * a.Hh);
            base[grp] = ((bt * a.H + 2 * i) * a.W + 2 * j) * (long long)C;
            has[grp] = (2 * i + 1 < a.H ? 1 : 0) | (2 * j + 1 < a.W ? 2 : 0);
          }
        }
        for (int kb = 0; kb < KB; ++kb, rp.next(NS)) {
          const int s = rp.s;
          if (rp.wrapped && !s_abort && !pw_wait(&a_free[s], rp.par ^ 1u, a.ctx.err, kErrWaitMma, lim))
            s_abort = 1;
          const int k0 = kb * kBK;
          const int q = k0 / C, c0 = k0 - q * C;  // a K block lies inside one neighbour (C % 32 == 0)
          uint8_t* dA = sA + s * kStage;
#pragma unroll
          for (int grp = 0; grp < 4; ++grp) {
            const int row = warp * 32 + grp * 8 + sub;
            long long src = -1;
            if (base[grp] >= 0 && ((q & 1) == 0 || (has[grp] & 1)) && ((q >> 1) == 0 || (has[grp] & 2)))
              src = base[grp] + ((q & 1) * (long long)a.W + (q >> 1)) * C;
            if (!index_ok(src, -1, x_extent, a.ctx.err)) src = -1;
            cp_async_16(dA + a_off(row, cq), a.x + (src < 0 ? 0 : src + c0 + cq * 8), src < 0 ? 0u : 16u);
          }
          cp_async_mbar_arrive_noinc(&a_full[s]);
        }
      }
    }
    cp_async_wait_all();  // nothing in flight when the CTA ends
  } else if (warp == kPwMmaWarp) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      if (!mbar_wait(b_full, 0, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
      const uint32_t idesc = idesc_bf16(kPmBM, BN, 0, 1);
      const uint32_t baddr = smem_u32(sB);
      RingPos rp;
      long long t = 0;
      for (long long m = m_first; m < mtiles; m += m_step, ++t) {
        const int buf = (int)(t & 1);
        if (t >= 2 && !s_abort &&
            !mbar_wait(&acc_free[buf], (uint32_t)((t >> 1) - 1) & 1, a.ctx.err, kErrWaitMma, lim))
          s_abort = 1;
        for (int kb = 0; kb < KB; ++kb, rp.next(NS)) {
          const int s = rp.s;
          if (!s_abort && !mbar_wait(&a_full[s], rp.par, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
          // bytes written by cp.async (generic proxy) are read by the tensor core;
          // TMA writes need no fence
          if (!kTma) fence_proxy_async_smem();
          tc_fence_after();
          if (!s_abort) {
            const uint32_t aaddr = smem_u32(sA + s * kStage);
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks)
              umma_ss(tmem + buf * BN, kTma ? pw_desc_sw128(aaddr + ks * 32) : smem_desc(aaddr + ks * 256, 128, 512),
                      smem_desc(baddr + (kb * (kBK / 16) + ks) * 2 * lboB, lboB, 128), idesc, (kb | ks) != 0);
            umma_commit(&a_free[s]);
          }
        }
        if (!s_abort) umma_commit(&acc_full[buf]);
      }
      // every MMA complete before the accumulators are released
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.ctx.err, kErrWaitMma, lim);
    }
    __syncwarp();
  } else if (warp < kPwEpi0) {
    // ---------------------------------------------------------------- row statistics
    const int p = tid - kPwStat0 * 32;  // this thread's row of the tile
    RingPos rp;
    long long t = 0;
    for (long long m = m_first; m < mtiles; m += m_step, ++t) {
      float mean = 0.f, m2 = 0.f, cnt = 0.f;
      for (int kb = 0; kb < KB; ++kb, rp.next(NS)) {
        const int s = rp.s;
        if (!s_abort && !pw_wait(&a_full[s], rp.par, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
        const uint8_t* stage = sA + s * kStage;
        float v[kBK];
#pragma unroll
        for (int kc = 0; kc < kBK / 8; ++kc) {
          const uint4 u = *reinterpret_cast<const uint4*>(stage + a_off(p, kc));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            v[kc * 8 + 2 * e] = f.x;
            v[kc * 8 + 2 * e + 1] = f.y;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_free[s]);
#pragma unroll
        for (int hb = 0; hb < kBK / 32; ++hb) {
          float bs = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) bs += v[hb * 32 + e];
          const float bm = bs * (1.0f / 32.0f);
          float bq = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) bq = fmaf(v[hb * 32 + e] - bm, v[hb * 32 + e] - bm, bq);
          const float n = cnt + 32.f;
          const float d = bm - mean;
          mean += d * (32.f / n);
          m2 += bq + d * d * (cnt * 32.f / n);
          cnt = n;
        }
      }
      const int buf = (int)(t & 1);
      if (t >= 2 && !s_abort &&
          !pw_wait(&st_free[buf], (uint32_t)((t >> 1) - 1) & 1, a.ctx.err, kErrWaitMma, lim))
        s_abort = 1;
      const float rstd = 1.0f / sqrtf(m2 / (float)K + a.eps);
      sStats[buf * kPmBM + p] = make_float2(-mean * rstd, rstd);
      mbar_arrive(&st_full[buf]);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // TMEM lanes 32 * (warp % 4) .. +31; two warps a quarter, each half of the
    // columns (whole 8-column groups)
    const int q = warp & 3, hf = (warp - kPwEpi0) >> 2;
    const int c_lo = (hf * (BN / 8)) / 2 * 8, c_hi = ((hf + 1) * (BN / 8)) / 2 * 8;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    constexpr int kCh = 48;
    long long t = 0;
    for (long long m = m_first; m < mtiles; m += m_step, ++t) {
      const int buf = (int)(t & 1);
      const int lr = q * 32 + lane;  // tile row (TMEM lane)
      const long long r = m * TR + lr;
      const bool row_ok = lr < TR && r < a.rows;
      if (!s_abort && !pw_wait(&acc_full[buf], (uint32_t)(t >> 1) & 1, a.ctx.err, kErrWaitMma, lim)) s_abort = 1;
      if (!s_abort && !pw_wait(&st_full[buf], (uint32_t)(t >> 1) & 1, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
      const float2 st = sStats[buf * kPmBM + lr];
      mbar_arrive(&st_free[buf]);
      tc_fence_after();
      // tcgen05.ld is warp-collective: one decision for the whole warp
      const int go = __shfl_sync(0xffffffffu, (!s_abort && q * 32 < TR && m * TR + q * 32 < a.rows) ? 1 : 0, 0);
      if (go) {
        for (int c0 = c_lo; c0 < c_hi; c0 += kCh) {
          const int n = c_hi - c0 < kCh ? c_hi - c0 : kCh;  // a multiple of 8
          uint32_t u[kCh];
          const uint32_t ta = tmem + lane_base + buf * BN + c0;
#pragma unroll
          for (int j = 0; j < kCh / 8; ++j)
            if (j * 8 < n)
              asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                           : "=r"(u[8 * j + 0]), "=r"(u[8 * j + 1]), "=r"(u[8 * j + 2]), "=r"(u[8 * j + 3]),
                             "=r"(u[8 * j + 4]), "=r"(u[8 * j + 5]), "=r"(u[8 * j + 6]), "=r"(u[8 * j + 7])
                           : "r"(ta + 8 * j));
          tmem_wait_ld_keep(u);
          if (row_ok) {
#pragma unroll
            for (int g8 = 0; g8 < kCh / 8; ++g8) {
              if (g8 * 8 >= n) break;
              const int cc = c0 + g8 * 8;
              const float4 cs0 = *reinterpret_cast<const float4*>(sCs + cc);
              const float4 cs1 = *reinterpret_cast<const float4*>(sCs + cc + 4);
              const float4 bb0 = *reinterpret_cast<const float4*>(sBias + cc);
              const float4 bb1 = *reinterpret_cast<const float4*>(sBias + cc + 4);
              const float cs[8] = {cs0.x, cs0.y, cs0.z, cs0.w, cs1.x, cs1.y, cs1.z, cs1.w};
              const float bb[8] = {bb0.x, bb0.y, bb0.z, bb0.w, bb1.x, bb1.y, bb1.z, bb1.w};
              uint32_t o[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float v0 = fmaf(st.y, __uint_as_float(u[g8 * 8 + 2 * k]), fmaf(st.x, cs[2 * k], bb[2 * k]));
                const float v1 =
                    fmaf(st.y, __uint_as_float(u[g8 * 8 + 2 * k + 1]), fmaf(st.x, cs[2 * k + 1], bb[2 * k + 1]));
                o[k] = pm_pack(v0, v1);
              }
              *reinterpret_cast<uint4*>(a.out + r * N2 + n0 + cc) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPwMmaWarp) tmem_dealloc(tmem, tcols);
}

// Wt = bf16(diag(gamma) Wr), colsum of the rounded Wt, bias = beta Wr + br
// (br may be null). With `dh_major`, row k of Wt is the row of K order
// (dh, dw, c) -- the order the TMA gather brings the neighbours in -- and takes
// row (dh + 2 dw) C + c of Wr, gamma and beta (whose order is the pages'
// (0,0), (1,0), (0,1), (1,1)). Block (8 x 128): 8 output columns, the K rows split over
// 128 thread rows (independent loads, a few rows each), partial sums reduced
// in shared memory by a fixed tree (the same order every call).
constexpr int kPmFoldCols = 8, kPmFoldRows = 128;
__global__ void __launch_bounds__(kPmFoldCols * kPmFoldRows)
    pm_fold_kernel(int K, int N2, const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                   const __nv_bfloat16* __restrict__ Wr, const __nv_bfloat16* __restrict__ br,
                   __nv_bfloat16* __restrict__ wt, float* __restrict__ colsum, float* __restrict__ bias,
                   int C, int dh_major) {
  __shared__ float s_cs[kPmFoldRows][kPmFoldCols + 1], s_bb[kPmFoldRows][kPmFoldCols + 1];
  const int tx = threadIdx.x % kPmFoldCols, ty = threadIdx.x / kPmFoldCols;
  const int j = blockIdx.x * kPmFoldCols + tx;
  float cs = 0.f, bb = 0.f;
  if (j < N2) {
    for (int k = ty; k < K; k += kPmFoldRows) {
      int ks = k;  // source row
      if (dh_major) {
        const int q = k / C, c = k - q * C;  // q = 2 dh + dw
        ks = ((q >> 1) + 2 * (q & 1)) * C + c;
      }
      const float w = __bfloat162float(Wr[(size_t)ks * N2 + j]);
      const __nv_bfloat16 wg = __float2bfloat16_rn(__bfloat162float(gamma[ks]) * w);
      wt[(size_t)k * N2 + j] = wg;
      cs += __bfloat162float(wg);
      bb = fmaf(__bfloat162float(beta[ks]), w, bb);
    }
  }
  s_cs[ty][tx] = cs;
  s_bb[ty][tx] = bb;
  __syncthreads();
  for (int h = kPmFoldRows / 2; h > 0; h >>= 1) {
    if (ty < h) {
      s_cs[ty][tx] += s_cs[ty + h][tx];
      s_bb[ty][tx] += s_bb[ty + h][tx];
    }
    __syncthreads();
  }
  if (ty == 0 && j < N2) {
    colsum[j] = s_cs[0][tx];
    bias[j] = s_bb[0][tx] + (br ? __bfloat162float(br[j]) : 0.f);
  }
}

// bf16 x as a 4-D tensor map (dims[0] innermost), 128-byte swizzle, zero fill
// out of bounds; false when the driver refuses it (the caller then gathers
// with cp.async).
using PwEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
bool encode_x_map(CUtensorMap* m, const void* base, const cuuint64_t* dims, const cuuint64_t* strides,
                  const cuuint32_t* box) {
  static PwEncodeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PwEncodeFn) nullptr;
    return reinterpret_cast<PwEncodeFn>(p);
  }();
  if (!fn) return false;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

  // Which kernel: the persistent one with the widest column slice (a multiple
  // of 16 dividing 2C, at most 256) whose resident weights leave room for four
  // A stages -- the TMA gather when H and W are even and a line of merged
  // tokens fits a tile, else the cp.async gather -- or else the tiled one.
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long lines = (long long)B * T * a.Hh;
  auto slice = [&](bool tma) {
    for (int bn = N2 < kPmMaxBN ? N2 : kPmMaxBN; bn >= 16; bn -= 16)
      if (N2 % bn == 0 && pw_smem_bytes(K, bn, kPwMinStages, tma) <= kPwSmemMax && N2 / bn <= sms) return bn;
    return 0;
  };
  PwArgs w;
  w.p = a;
  CUtensorMap tm;
  memset(&tm, 0, sizeof(tm));
  bool tma = H % 2 == 0 && W % 2 == 0 && a.Wh <= kPmBM && lines <= 0x7fffffffLL && slice(true) > 0;
  if (tma) {
    w.p.BN = slice(true);
    w.Lt = kPmBM / a.Wh;
    if (w.Lt > lines) w.Lt = (int)lines;
    w.TR = w.Lt * a.Wh;
    w.mtiles = (lines + w.Lt - 1) / w.Lt;
    // x[bt, 2i + dh, 2j + dw, c] as (dw * C + c, j, dh, bt * H/2 + i): the 2C
    // channels of a token pair are contiguous
    const cuuint64_t dims[4] = {(cuuint64_t)N2, (cuuint64_t)a.Wh, 2, (cuuint64_t)lines};
    const cuuint64_t strides[3] = {(cuuint64_t)C * 4, (cuuint64_t)W * C * 2, (cuuint64_t)W * C * 4};
    const cuuint32_t box[4] = {(cuuint32_t)pw_bk(true), (cuuint32_t)a.Wh, 1, (cuuint32_t)w.Lt};
    tma = encode_x_map(&tm, x, dims, strides, box);
  }
  const bool persistent = tma || slice(false) > 0;
  if (persistent && !tma) {
    w.p.BN = slice(false);
    w.Lt = 0;
    w.TR = kPmBM;
    w.mtiles = (a.rows + kPmBM - 1) / kPmBM;
  }

  prof_begin(kKindOther, st);
  pm_fold_kernel<<<(N2 + kPmFoldCols - 1) / kPmFoldCols, kPmFoldCols * kPmFoldRows, 0, st>>>(
      K, N2, static_cast<const __nv_bfloat16*>(gamma), static_cast<const __nv_bfloat16*>(beta),
      static_cast<const __nv_bfloat16*>(Wr), static_cast<const __nv_bfloat16*>(br),
      reinterpret_cast<__nv_bfloat16*>(base), reinterpret_cast<float*>(base + wt_bytes),
      reinterpret_cast<float*>(base + wt_bytes + vec), C, tma ? 1 : 0);
  prof_end(kKindOther, st);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  if (persistent) {
    const int pbn = w.p.BN;
    w.NT = N2 / pbn;
    w.NS = (kPwSmemMax - pw_b_bytes(K, pbn) - pw_tail_bytes(pbn)) / pw_stage_bytes(tma);
    if (w.NS > kPwMaxStages) w.NS = kPwMaxStages;
    const int smem = pw_smem_bytes(K, pbn, w.NS, tma);
    e = tma ? cudaFuncSetAttribute(pm_ws_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
            : cudaFuncSetAttribute(pm_ws_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    long long lanes = sms / w.NT;  // CTAs per column slice
    if (lanes > w.mtiles) lanes = w.mtiles;
    const unsigned grid = (unsigned)(lanes * w.NT);
    prof_begin(kKindMlp, st);
    if (tma)
      pm_ws_kernel<true><<<grid, kPwThreads, smem, st>>>(tm, w);
    else
      pm_ws_kernel<false><<<grid, kPwThreads, smem, st>>>(tm, w);
    prof_end(kKindMlp, st);
    count_launch();
    return cudaGetLastError();
  }
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
