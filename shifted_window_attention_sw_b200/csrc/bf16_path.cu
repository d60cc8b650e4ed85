// bf16 path of the layer on sm_100a tensor cores (tcgen05 / TMEM).
//
// Per chunk of windows, four launches:
//   1. row_source_kernel: the source token of every window slot of the chunk
//      (roll + pad + partition as index arithmetic; -1 for padding). The block
//      entry first folds gamma and beta into the QKV weights (ln_fold_kernel,
//      once per call); when the tiled GEMM runs, row_stats_kernel writes the
//      row table and each row's layer-norm statistics instead.
//   2. gemm_ws_kernel<kQKV>: persistent warp-specialised tcgen05 GEMM (gather
//      warps cp.async the rows named by the row table, zero-filling padding;
//      two MMA-issuing warps on different sub-partitions, even and odd tiles;
//      epilogue warps; for the block entry four of them are statistics warps
//      that compute each landed row's layer-norm mean and rstd from the
//      stage and write its -mean as one extra K step). The epilogue adds bqkv,
//      scales q by log2(e)/sqrt(d) and writes per-(window, head) q / k / v
//      slabs in the tensor-core operand layout. gemm_kernel<kQKV> is the tiled
//      fallback used when the persistent kernel's resident weight slice does
//      not fit.
//   3. attention7_kernel: persistent warp-specialised attention for (P,7,7)
//      windows: S = q k^T on tcgen05 into TMEM with the shifted-window mask
//      and a per-row reference folded into one extra MMA step, relative-
//      position bias and exp2 in registers, P as bf16 over S in TMEM,
//      O = P v on tcgen05 with P read from TMEM. attention_kernel handles the
//      other window shapes, one (window, head) per CTA.
//   4. gemm_ws_kernel<kPROJ> (or gemm_kernel<kPROJ>): the attention output
//      times Wproj, epilogue adds bproj (and, for the block entry, the
//      residual, which the producer warps copy into shared memory) and scatters
//      rows back through the row table (reverse partition, roll by +shift,
//      drop padding).
//
// Shared-memory operand layout everywhere: the no-swizzle canonical layout of
// 8-row x 16-byte core matrices (128 contiguous bytes).
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vswin {

// Optional event trace of the attention kernel, compiled in only with
// -DVSWIN_TRACE: CTA 0 records (tag, clock64) pairs per role (preparation
// thread, lane 0 of each softmax warp; for the GEMMs the producer, MMA and
// first epilogue lanes, QKV then projection), read back by
// vswin_trace_read.
#ifdef VSWIN_TRACE
constexpr int kTraceRoles = 23, kTraceCap = 1024;
__device__ long long g_trace[kTraceRoles][kTraceCap][2];
__device__ __forceinline__ void trace_event(int role, int& n, int tag) {
  if (blockIdx.x == 0 && n < kTraceCap) {
    g_trace[role][n][0] = tag;
    g_trace[role][n][1] = clock64();
  }
  ++n;
}
#define VSWIN_TRACE_EVENT(role, n, tag) trace_event(role, n, tag)
#else
#define VSWIN_TRACE_EVENT(role, n, tag) ((void)0)
#endif

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Tokens of the layer: the extent of every row-table entry (-1 = padding).
__host__ __device__ inline long long layer_tokens(const Geom& g) {
  return (long long)g.B * g.T * g.H * g.W;
}

// ============================================================================ GEMM
constexpr int kBM = 128;
constexpr int kBK = 32;
constexpr int kStages = 4;
constexpr int kGemmThreads = 128;
constexpr int kMaxBN = 256;
constexpr int kAStageBytes = kBM * kBK * 2;      // 8 KB
constexpr int kBStageMaxBytes = kBK * kMaxBN * 2;  // 16 KB

enum { kQKV = 0, kPROJ = 1 };

// Where q, k and v of one (window, head) live in the chunk scratch: a q slab of
// `qrows` rows (slot order) then k and v slabs of `kvrows` rows, each row 32
// bf16 in the no-swizzle operand layout ((row/8)*512 + (col/8)*128 +
// (row%8)*16 bytes). For (P,7,7) windows the keys are stored as P*7 rows of 8:
// slot n goes to row (n/7)*8 + n%7, the eighth row of each group is padding,
// so that the softmax walks keys in 8-column groups of one (pt, ph) line.
struct SlabLayout {
  int qrows, kvrows, kv8;
  __host__ __device__ int kv_row(int n) const { return kv8 ? (n / 7) * 8 + n % 7 : n; }
  __host__ __device__ size_t head_elems() const { return (size_t)(qrows + 2 * kvrows) * 32; }
};

__host__ __device__ inline bool window_is_p77(const Geom& g) {
  const int P = g.win[0];
  return g.win[1] == 7 && g.win[2] == 7 && (P == 1 || P == 2 || P == 4 || P == 8 || P == 16);
}

__host__ __device__ inline SlabLayout slab_layout(const Geom& g) {
  SlabLayout L;
  L.qrows = g.Npad;
  L.kv8 = window_is_p77(g) ? 1 : 0;
  // 8-wide key lines, rounded up to a multiple of 32 columns (4 lines)
  L.kvrows = L.kv8 ? ((g.win[0] * 7 * 8 + 31) / 32) * 32 : g.Npad;
  return L;
}

struct GemmArgs {
  Geom g;
  KernelCtx ctx;
  const __nv_bfloat16* A;     // kQKV: x (gathered rows); kPROJ: attention output [rows][C]
  const __nv_bfloat16* Wt;    // [K][Ntot] row-major (used as the MN-major B operand)
  const __nv_bfloat16* bias;  // [Ntot]
  __nv_bfloat16* dst;         // kQKV: q/k/v slabs; kPROJ: out (B,T,H,W,C)
  long long win0;             // first window of the chunk
  long long rows;             // nwin * N
  int K, Ntot, BN;
  float qscale;
  SlabLayout slab;
  const int* rowsrc;          // [rows] source token of each chunk row (-1 = padding), or null
  // Block fusion (all null for the plain layer). QKV: the pre-norm folded into
  // the epilogue -- Wt is diag(gamma) Wqkv, ln_stats[r] = (-mean * rstd, rstd)
  // of chunk row r's token ((0, 0) for padding), ln_colsum the column sums of
  // Wt, ln_bias = bqkv + beta Wqkv. PROJ: resid (x) added to every output row.
  const float2* ln_stats;
  const float* ln_colsum;
  const float* ln_bias;
  const __nv_bfloat16* resid;
  long long lda;  // A row stride in elements (0: C)
  float ln_eps;   // fused pre-norm in the persistent QKV GEMM: statistics computed in the kernel
};

__host__ __device__ constexpr int gemm_smem_bytes() {
  return kStages * (kAStageBytes + kBStageMaxBytes) + kBM * 8 + 256;
}

// Hardware base-2 exponential (MUFU), flush-to-zero; ex2(-inf) = +0.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier over `nthreads` threads (whole warps).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int MODE, bool FUSE>
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_kernel(GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kAStageBytes;
  long long* s_src = reinterpret_cast<long long*>(sB + kStages * kBStageMaxBytes);
  uint64_t* bar_free = reinterpret_cast<uint64_t*>(s_src + kBM);  // kStages
  uint64_t* bar_done = bar_free + kStages;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_done + 1);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geom& g = a.g;
  const long long m0 = (long long)blockIdx.x * kBM;  // first row of the tile (chunk-relative)
  const int n0 = blockIdx.y * a.BN;
  const int BN = a.BN;
  const uint32_t tcols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;

  // Row sources: element offset of the row's first channel, or -1 (zero fill).
  {
    const long long r = m0 + tid;
    long long src = -1;
    if (r < a.rows) {
      if (MODE == kQKV) {
        const long long gr = a.win0 * g.N + r;
        long long tok = slot_source(g, gr / g.N, (int)(gr % g.N));
        if (!index_ok(tok, -1, layer_tokens(g), a.ctx.err)) tok = -1;
        src = tok < 0 ? -1 : tok * g.C;
      } else {
        src = r * (long long)(a.lda ? a.lda : g.C);
      }
    }
    s_src[tid] = src;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bar_free[s], 1);
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

  const int KB = a.K / kBK;
  const uint32_t lboB = (uint32_t)(BN / 8) * 128u;
  const int bchunks = kBK * (BN / 8);

  auto load_stage = [&](int kb, int s) {
    const int k0 = kb * kBK;
    uint8_t* dA = sA + s * kAStageBytes;
    // A: 128 rows x 4 chunks of 8 channels; thread = row.
    const long long src = s_src[tid];
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      uint8_t* d = dA + (tid >> 3) * 512 + kc * 128 + (tid & 7) * 16;
      const __nv_bfloat16* p = a.A + (src < 0 ? 0 : src + k0 + kc * 8);
      cp_async_16(d, p, src < 0 ? 0u : 16u);
    }
    uint8_t* dB = sB + s * kBStageMaxBytes;
    for (int c = tid; c < bchunks; c += kGemmThreads) {
      const int kk = c / (BN / 8), nc = c % (BN / 8);
      uint8_t* d = dB + (kk >> 3) * lboB + nc * 128 + (kk & 7) * 16;
      cp_async_16(d, a.Wt + (size_t)(k0 + kk) * a.Ntot + n0 + nc * 8, 16u);
    }
  };

  const uint32_t idesc = idesc_bf16(kBM, BN, 0, 1);
#pragma unroll 1
  for (int p = 0; p < kStages - 1; ++p) {
    if (p < KB) load_stage(p, p);
    cp_async_commit();
  }
#pragma unroll 1
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kStages;
    cp_async_wait<kStages - 2>();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && !s_abort) {
      tc_fence_after();
      const uint32_t aaddr = smem_u32(sA + s * kAStageBytes);
      const uint32_t baddr = smem_u32(sB + s * kBStageMaxBytes);
#pragma unroll
      for (int ks = 0; ks < kBK / 16; ++ks) {
        const uint64_t ad = smem_desc(aaddr + ks * 256, 128, 512);
        const uint64_t bd = smem_desc(baddr + ks * 2 * lboB, lboB, 128);
        umma_ss(tmem, ad, bd, idesc, (kb | ks) != 0);
      }
      umma_commit(&bar_free[s]);
    }
    const int nk = kb + kStages - 1;
    if (nk < KB) {
      const int ns = nk % kStages;
      if (kb >= 1) {
        // stage ns was last read by the MMAs of k-block kb-1 (its use number (kb-1)/kStages)
        if (!mbar_wait(&bar_free[ns], ((kb - 1) / kStages) & 1, a.ctx.err, kErrWaitMma, a.ctx.wait_limit))
          s_abort = 1;
      }
      load_stage(nk, ns);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (tid == 0) {
    if (!s_abort) umma_commit(bar_done);
  }
  __syncthreads();
  if (!s_abort && !mbar_wait(bar_done, 0, a.ctx.err, kErrWaitMma, a.ctx.wait_limit)) s_abort = 1;
  __syncthreads();
  tc_fence_after();

  // ---------------- epilogue: TMEM -> registers -> bf16 -> global
  // TMEM loads are warp-collective: every lane of a warp whose tile rows start
  // inside the problem executes them; only the stores depend on the lane's row.
  const long long r = m0 + warp * 32 + lane;
  const bool row_ok = r < a.rows;
  if (!s_abort && m0 + warp * 32 < a.rows) {
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    long long dst_row = -1;     // kPROJ: token
    long long slab_win = 0;     // kQKV: chunk-relative window
    int slot = 0;
    float2 st = make_float2(0.f, 0.f);  // kQKV + FUSE: (-mean * rstd, rstd) of the row's token
    if (MODE == kQKV) {
      slab_win = r / g.N;
      slot = (int)(r % g.N);
      if (FUSE && row_ok) st = a.ln_stats[r];
    } else if (row_ok) {
      const long long gr = a.win0 * g.N + r;
      dst_row = slot_source(g, gr / g.N, (int)(gr % g.N));
      if (!index_ok(dst_row, -1, layer_tokens(g), a.ctx.err)) dst_row = -1;
    }
    for (int c = 0; c < BN / 16; ++c) {
      uint32_t u[16];
      tmem_ld16(trow + c * 16, u);
      tmem_wait_ld();
      const int col = n0 + c * 16;
      float v[16];
      if (FUSE && MODE == kQKV && st.y != 0.f) {
        // LN(x) Wqkv + bqkv = rstd * (x Wt - mean * colsum) + ln_bias
#pragma unroll
        for (int k = 0; k < 16; ++k)
          v[k] = fmaf(st.y, __uint_as_float(u[k]), fmaf(st.x, a.ln_colsum[col + k], a.ln_bias[col + k]));
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(u[k]) + __bfloat162float(a.bias[col + k]);
      }
      if (FUSE && MODE == kPROJ && dst_row >= 0) {
        const __nv_bfloat16* xr = a.resid + dst_row * g.C + col;
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] += __bfloat162float(xr[k]);
      }
      uint4 w0, w1;
      if (MODE == kQKV && row_ok) {
        const int which = col / g.C;
        const int hh = (col % g.C) >> 5;
        const int jj = col & 31;  // 0 or 16
        const float sc = which == 0 ? a.qscale : 1.0f;
        w0 = make_uint4(pack_bf16x2(v[0] * sc, v[1] * sc), pack_bf16x2(v[2] * sc, v[3] * sc),
                        pack_bf16x2(v[4] * sc, v[5] * sc), pack_bf16x2(v[6] * sc, v[7] * sc));
        w1 = make_uint4(pack_bf16x2(v[8] * sc, v[9] * sc), pack_bf16x2(v[10] * sc, v[11] * sc),
                        pack_bf16x2(v[12] * sc, v[13] * sc), pack_bf16x2(v[14] * sc, v[15] * sc));
        const SlabLayout& L = a.slab;
        __nv_bfloat16* slab = a.dst + ((size_t)slab_win * g.heads + hh) * L.head_elems() +
                              (which == 0 ? 0 : ((size_t)L.qrows + (size_t)(which - 1) * L.kvrows) * 32);
        const int row = which == 0 ? slot : L.kv_row(slot);
        __nv_bfloat16* e = slab + (row >> 3) * 256 + (jj >> 3) * 64 + (row & 7) * 8;
        *reinterpret_cast<uint4*>(e) = w0;
        *reinterpret_cast<uint4*>(e + 64) = w1;
      } else if (dst_row >= 0) {
        w0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                        pack_bf16x2(v[6], v[7]));
        w1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                        pack_bf16x2(v[14], v[15]));
        __nv_bfloat16* e = a.dst + dst_row * g.C + col;
        *reinterpret_cast<uint4*>(e) = w0;
        *reinterpret_cast<uint4*>(e + 8) = w1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tcols);
}

// ============================================================================ persistent GEMM
//
// Warp-specialised persistent version of the two GEMMs for layers whose
// per-CTA weight slice (K x BN bf16) fits in shared memory: warps 0-3 gather
// 128-row A tiles with cp.async into a ring of STAGES buffers (each thread's
// copies arrive on the stage's mbarrier when they land, so the gatherers only
// wait for a free stage), warps 4 and 17 issue tcgen05.mma (the even and the
// odd tiles) into two TMEM accumulators (BN columns each), warps 5..16 drain an
// accumulator (three warps per TMEM lane quarter, a third of the columns each)
// while the next tile is multiplied. CTA c keeps N-tile c % NT and walks the M-tiles
// c / NT, c / NT + G / NT, ... (G = grid size, a multiple of NT).
constexpr int kWsProdWarps = 4;
constexpr int kWsEpiWarps = 12;
constexpr int kWsMmaWarp = kWsProdWarps;
constexpr int kWsEpi0 = kWsProdWarps + 1;
// A second MMA warp, after the epilogue warps (another SM sub-partition):
// warp kWsMmaWarp issues the even tiles, this one the odd tiles -- each tile
// has its own accumulator (t & 1) and A stage, and a thread's MMA issue slows
// when its sub-partition's other warps keep the issue slots busy.
constexpr int kWsMma2Warp = kWsProdWarps + 1 + kWsEpiWarps;
constexpr int kWsThreads = 32 * (kWsMma2Warp + 1);
constexpr int kWsMaxBBytes = 96 * 1024;

__host__ __device__ inline int ws_a_bytes(int K) { return kBM * K * 2; }
// The fused pre-norm's extra K step (16 columns of A: the row's -mean in two
// bf16 halves; 16 rows of the folded weights: the column sums in two halves).
constexpr int kLnExtraK = 16;
constexpr int kWsStatSlots = 8;  // fused pre-norm: tiles of row statistics in flight
constexpr int kWsResSlots = 3;   // fused residual: tiles of residual rows in flight
__host__ __device__ inline int ws_res_row_bytes(int BN) { return BN * 2 + 16; }  // padded row of a residual tile
// B slice, A stages, bias (BN floats), column-group table (BN / 8 x 16 B), with
// the fused pre-norm the column sums and folded bias (2 x BN floats), barriers,
// with the fused pre-norm a ring of per-row statistics (8 tiles x 128 rows), with
// the fused residual a ring of residual tiles (3 x 128 rows of the BN columns)
// The projection's epilogue stages each tile's rows in shared memory (two
// buffers of 128 padded rows and their output-row indices) and copies them out
// row by row.
__host__ __device__ inline int ws_stage_out_bytes(int BN) { return 2 * kBM * ws_res_row_bytes(BN) + 2 * kBM * 4; }
__host__ __device__ inline int ws_smem_bytes(int K0, int BN, int stages, bool ln = false, bool resid = false,
                                             bool stage_out = false) {
  const int K = ln ? K0 + kLnExtraK : K0;
  return K * BN * 2 + stages * ws_a_bytes(K) + BN * 6 + (ln ? BN * 8 + kWsStatSlots * kBM * 8 : 0) +
         (resid ? kWsResSlots * kBM * ws_res_row_bytes(BN) : 0) + (stage_out ? ws_stage_out_bytes(BN) : 0) + 256;
}

// Destination facts of one group of 8 output columns of the QKV GEMM: element
// offset of the group inside its window's q / k / v block, whether it is a q
// column (row layout of the q slab, scaled by log2(e)/sqrt(d)) and its scale.
struct ColGroup {
  int off, is_q;
  float scale;
  int pad;
};

// Row sources of one chunk: token index (x row) of each window slot, -1 for
// padding. Consumed by the QKV gather and the projection scatter.
__global__ void row_source_kernel(Geom g, long long win0, long long rows, int* __restrict__ out, int* err) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < rows; r += stride) {
    const long long gr = win0 * g.N + r;
    long long tok = slot_source(g, gr / g.N, (int)(gr % g.N));
    if (!index_ok(tok, -1, layer_tokens(g), err)) tok = -1;
    out[r] = (int)tok;
  }
}

#ifdef VSWIN_DEBUG_BOUNDS
// Test hook: overwrite one row-table entry.
__global__ void plant_row_kernel(int* rowsrc, long long r, int token) { rowsrc[r] = token; }
#endif

// Pre-norm folded into the QKV weights ("Video Swin Transformer" summary page,
// eq. 1: the layer reads LN(x)). Since LN(x) = rstd * (x - mean) * gamma + beta,
//   LN(x) Wqkv + bqkv = rstd * (x Wt - mean * colsum(Wt)) + (bqkv + beta Wqkv)
// with Wt = diag(gamma) Wqkv. Wt is rounded to bf16 (gamma * w is exact in
// fp32, so this is the only rounding) and colsum is taken from the rounded Wt
// so that the mean term cancels what x Wt accumulates. Block (32 x 32): 32
// output columns, the C rows split over 32 thread rows (independent loads),
// partial sums reduced in shared memory.
constexpr int kFoldCols = 32, kFoldRows = 32;
__global__ void __launch_bounds__(kFoldCols * kFoldRows) ln_fold_kernel(
    int C, int N3, const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
    const __nv_bfloat16* __restrict__ Wqkv, const __nv_bfloat16* __restrict__ bqkv, __nv_bfloat16* __restrict__ wt,
    float* __restrict__ colsum, float* __restrict__ bias_ln) {
  __shared__ float s_cs[kFoldRows][kFoldCols + 1], s_bb[kFoldRows][kFoldCols + 1];
  const int tx = threadIdx.x % kFoldCols, ty = threadIdx.x / kFoldCols;
  const int j = blockIdx.x * kFoldCols + tx;
  float cs = 0.f, bb = 0.f;
  if (j < N3) {
#pragma unroll 4
    for (int c = ty; c < C; c += kFoldRows) {
      const float w = __bfloat162float(Wqkv[(size_t)c * N3 + j]);
      const __nv_bfloat16 wg = __float2bfloat16_rn(__bfloat162float(gamma[c]) * w);
      wt[(size_t)c * N3 + j] = wg;
      cs += __bfloat162float(wg);
      bb = fmaf(__bfloat162float(beta[c]), w, bb);
    }
  }
  s_cs[ty][tx] = cs;
  s_bb[ty][tx] = bb;
  __syncthreads();
  if (ty == 0 && j < N3) {
    for (int k = 1; k < kFoldRows; ++k) {
      cs += s_cs[k][tx];
      bb += s_bb[k][tx];
    }
    colsum[j] = cs;
    bias_ln[j] = __bfloat162float(bqkv[j]) + bb;
    // rows C .. C + 15 of wt: the column sum as two bf16 halves (hi, lo, hi, lo),
    // then zeros -- the persistent GEMM's extra K step multiplies them with the
    // row's -mean (also two halves), so that the MMA itself subtracts mean x colsum
    const __nv_bfloat16 hi = __float2bfloat16_rn(cs);
    const __nv_bfloat16 lo = __float2bfloat16_rn(cs - __bfloat162float(hi));
    for (int k = 0; k < kLnExtraK; ++k)
      wt[(size_t)(C + k) * N3 + j] = k < 4 ? ((k & 1) ? lo : hi) : __float2bfloat16_rn(0.f);
  }
}

// Row table plus the norm's statistics of each chunk row's token: rowsrc[r] as
// row_source_kernel writes it and stats[r] = (-mean * rstd, rstd) with the
// biased variance and rstd = 1 / sqrt(var + eps) (torch.nn.LayerNorm's
// definition), (0, 0) for a padding row. A warp takes 32 consecutive rows: each
// lane does one row's index math (32-bit: window slots < 2^31, checked by the
// caller), then four lanes per row (rows shuffled to them eight at a time) sum
// C/32 chunks of 8 channels each. NCH = C/32 in 1..4 keeps all four row groups'
// chunks in registers (mean, then squared deviations, from the same values);
// NCH = 0 takes any C, reading each row twice (the second time from L1).
template <int NCH>
__global__ void __launch_bounds__(256) row_stats_kernel(Geom g, long long win0, long long rows,
                                                        const __nv_bfloat16* __restrict__ x, float eps,
                                                        int* __restrict__ rowsrc, float2* __restrict__ stats,
                                                        int* err) {
  const int lane = threadIdx.x & 31, cq = lane & 3, sub = lane >> 2;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  const long long warp0 = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nch = g.C / 32;
  const float inv_c = 1.0f / (float)g.C;
  auto chunk_sum = [](const uint4& v, float acc) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      acc += f.x + f.y;
    }
    return acc;
  };
  auto chunk_sq = [](const uint4& v, float mean, float acc) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      const float d0 = f.x - mean, d1 = f.y - mean;
      acc = fmaf(d0, d0, fmaf(d1, d1, acc));
    }
    return acc;
  };
  auto finish = [&](long long r, int tok, float sum, float ss) {
    // sum and ss are the row's totals (after the four-lane reduction)
    if (cq == 0 && r < rows) {
      const float mean = sum * inv_c;
      const float rstd = 1.0f / sqrtf(ss * inv_c + eps);
      stats[r] = tok < 0 ? make_float2(0.f, 0.f) : make_float2(-mean * rstd, rstd);
    }
  };
  // whole warps iterate together (same trip count), so the shuffles see all lanes
  for (long long R = warp0 * 32; R < rows; R += nwarps * 32) {
    int my_tok = -1;
    if (R + lane < rows) {
      const int gr = (int)(win0 * g.N + R + lane);
      const int gw = gr / g.N;
      my_tok = slot_source32(g, gw, gr - gw * g.N);
      if (!index_ok(my_tok, -1, layer_tokens(g), err)) my_tok = -1;
      rowsrc[R + lane] = my_tok;
    }
    if (NCH > 0) {
      uint4 v[4][NCH > 0 ? NCH : 1];
      int tk[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        tk[s] = __shfl_sync(0xffffffffu, my_tok, s * 8 + sub);
        const __nv_bfloat16* row = x + (size_t)(tk[s] < 0 ? 0 : tk[s]) * g.C;
#pragma unroll
        for (int i = 0; i < NCH; ++i)
          v[s][i] = tk[s] >= 0 ? *reinterpret_cast<const uint4*>(row + (cq + 4 * i) * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < NCH; ++i) sum = chunk_sum(v[s][i], sum);
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        const float mean = sum * inv_c;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < NCH; ++i) ss = chunk_sq(v[s][i], mean, ss);
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        finish(R + s * 8 + sub, tk[s], sum, ss);
      }
    } else {
      for (int s = 0; s < 4; ++s) {
        const int tok = __shfl_sync(0xffffffffu, my_tok, s * 8 + sub);
        const __nv_bfloat16* row = x + (size_t)(tok < 0 ? 0 : tok) * g.C;
        float sum = 0.f;
        if (tok >= 0)
          for (int i = 0; i < nch; ++i) sum = chunk_sum(*reinterpret_cast<const uint4*>(row + (cq + 4 * i) * 8), sum);
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        const float mean = sum * inv_c;
        float ss = 0.f;
        if (tok >= 0)
          for (int i = 0; i < nch; ++i)
            ss = chunk_sq(*reinterpret_cast<const uint4*>(row + (cq + 4 * i) * 8), mean, ss);
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        finish(R + s * 8 + sub, tok, sum, ss);
      }
    }
  }
}

template <int MODE, int STAGES, bool FUSE>
__global__ void __launch_bounds__(kWsThreads, 1) gemm_ws_kernel(GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr bool kLn = FUSE && MODE == kQKV;      // pre-norm folded into the QKV epilogue
  constexpr bool kResid = FUSE && MODE == kPROJ;  // residual added in the projection epilogue
  // K: the MMA's depth -- the x columns, plus for the fused pre-norm one extra
  // step of 16 (the row's -mean against the weights' column sums)
  const int Kx = a.K, K = kLn ? a.K + kLnExtraK : a.K, BN = a.BN;
  uint8_t* sB = smem;                                     // K x BN, MN-major operand layout
  uint8_t* sA = sB + K * BN * 2;                          // STAGES x (128 x K), K-major
  float* sBias = reinterpret_cast<float*>(sA + STAGES * ws_a_bytes(K));  // bias x column scale
  ColGroup* sGrp = reinterpret_cast<ColGroup*>(sBias + BN);                // [BN / 8]
  float* sCs = reinterpret_cast<float*>(sGrp + BN / 8);  // kLn: column sums of Wt
  float* sBb = sCs + BN;                                 // kLn: folded bias x column scale
  uint64_t* bars = reinterpret_cast<uint64_t*>(kLn ? sBb + BN : sCs);
  uint64_t* b_full = bars;                 // B resident
  uint64_t* a_full = bars + 1;             // [STAGES]
  uint64_t* a_free = a_full + STAGES;      // [STAGES]
  uint64_t* acc_full = a_free + STAGES;    // [2]
  uint64_t* acc_free = acc_full + 2;       // [2]
  uint64_t* stats_full = acc_free + 2;     // kLn: [kWsStatSlots] a tile's row statistics written
  uint64_t* a_ext = stats_full + (kLn ? kWsStatSlots : 0);  // kLn: [STAGES] the stage's -mean columns written
  uint64_t* res_full = a_ext + (kLn ? STAGES : 0);          // kResid: [kWsResSlots] residual tile landed
  uint64_t* res_free = res_full + (kResid ? kWsResSlots : 0);  // kResid: [kWsResSlots] residual tile read
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(res_free + (kResid ? kWsResSlots : 0));
  // kLn: (-mean * rstd, rstd) per row of a tile, (0, 0) for padding rows, slot t % 8
  float2* sStats = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(bars) + 256);
  // kResid: the residual rows of a tile (BN columns, padded rows), slot t % 3
  uint8_t* sRes = reinterpret_cast<uint8_t*>(bars) + 256;
  const int res_slot_bytes = kBM * ws_res_row_bytes(BN);
  // projection: staged output tiles [2][128 padded rows], then their output rows [2][128]
  uint8_t* sOut = sRes + (kResid ? kWsResSlots * res_slot_bytes : 0);
  int* sDst = reinterpret_cast<int*>(sOut + 2 * res_slot_bytes);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geom& g = a.g;
  const int NT = a.Ntot / BN;
  const int nt = blockIdx.x % NT;
  const int n0 = nt * BN;
  const long long mtiles = (a.rows + kBM - 1) / kBM;
  const long long m_first = blockIdx.x / NT, m_step = gridDim.x / NT;
  const uint64_t lim = a.ctx.wait_limit;
  const long long lda = a.lda ? a.lda : g.C;  // A row stride (elements)
  const uint32_t lboB = (uint32_t)(BN / 8) * 128u;  // B: K-group stride
  const uint32_t sboA = (uint32_t)(K / 8) * 128u;   // A: 8-row group stride
  const uint32_t tcols = BN <= 64 ? 128 : BN <= 128 ? 256 : 512;
  constexpr int kProdThreads = kWsProdWarps * 32;
  // the fused pre-norm runs eight epilogue warps and four statistics warps,
  // the others twelve epilogue warps (same block size)
  constexpr int kEpiWarps = kLn ? 8 : kWsEpiWarps;
  constexpr int kStatWarps = kLn ? kWsEpiWarps - 8 : 0;
  constexpr int kStat0 = kWsEpi0 + kEpiWarps;
  constexpr int kTraceG = MODE == kQKV ? 17 : 20;  // trace roles of this GEMM
  int trace_n = 0;
  (void)trace_n;
  (void)kTraceG;

  if (tid == 0) {
    mbar_init(b_full, kProdThreads);
    for (int k = 0; k < STAGES; ++k) {
      mbar_init(&a_full[k], kProdThreads);  // one asynchronous arrival per gathering thread
      mbar_init(&a_free[k], 1);  // MMA commit
      if (kLn) mbar_init(&a_ext[k], kStatWarps * 32);  // every statistics thread, after its row's extra columns
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&acc_full[k], 1);
      mbar_init(&acc_free[k], kEpiWarps);
    }
    if (kLn)
      for (int k = 0; k < kWsStatSlots; ++k) mbar_init(&stats_full[k], kProdThreads);
    if (kResid)
      for (int k = 0; k < kWsResSlots; ++k) {
        mbar_init(&res_full[k], kProdThreads);
        mbar_init(&res_free[k], kEpiWarps);
      }
    fence_mbar_init();
    s_abort = 0;
  }
  // per 8-column group: destination facts (the QKV slabs: C is a multiple of
  // 32, so a group lies in one (which, head) slab) and the scale folded into
  // the bias
  for (int c8 = tid; c8 < BN / 8; c8 += kWsThreads) {
    ColGroup cg{0, 0, 1.0f, 0};
    if (MODE == kQKV) {
      const int col = n0 + 8 * c8;
      const int sidx = col >> 5;
      const int which = sidx / g.heads;
      const int hh = sidx - which * g.heads;
      const SlabLayout& L = a.slab;
      cg.off = (int)((size_t)hh * L.head_elems() +
                     (which == 0 ? 0 : ((size_t)L.qrows + (size_t)(which - 1) * L.kvrows) * 32)) +
               ((col & 31) >> 3) * 64;
      cg.is_q = which == 0;
      cg.scale = which == 0 ? a.qscale : 1.0f;
    }
    sGrp[c8] = cg;
  }
  for (int c = tid; c < BN; c += kWsThreads) {
    const float sc = (MODE == kQKV && (((n0 + c) >> 5) / g.heads) == 0) ? a.qscale : 1.0f;
    sBias[c] = __bfloat162float(a.bias[n0 + c]) * sc;
    if (kLn) {
      sCs[c] = a.ln_colsum[n0 + c];
      sBb[c] = a.ln_bias[n0 + c] * sc;
    }
  }
  if (warp == kWsMmaWarp) {
    tmem_alloc(s_tmem, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp < kWsProdWarps) {
    // ---------------------------------------------------------------- producers
    // resident B slice
    for (int c = tid; c < K * (BN / 8); c += kProdThreads) {
      const int kk = c / (BN / 8), nc = c % (BN / 8);
      cp_async_16(sB + (kk >> 3) * lboB + nc * 128 + (kk & 7) * 16, a.Wt + (size_t)kk * a.Ntot + n0 + nc * 8, 16u);
    }
    cp_async_mbar_arrive_noinc(b_full);
    // A gather: warp w fills rows [32w, 32w + 32) in groups of 8 rows; 4 lanes per
    // row, lane l moving chunks l%4, l%4 + 4, ... (64 contiguous bytes per row and
    // instruction).
    const int sub = lane >> 2, cq = lane & 3;
    // Row index of each of this lane's 4 rows in the source matrix (-1:
    // padding): QKV looks it up in the row table.
    auto row_tok = [&](long long m, int grp) -> int {
      const long long r = m * kBM + warp * 32 + grp * 8 + sub;
      if (m >= mtiles || r >= a.rows) return -1;
      return (MODE == kQKV || kResid) ? a.rowsrc[r] : (int)r;
    };
    // the row table's tokens (or, unfused projection, chunk rows) against their extent
    const long long tok_extent = (MODE == kQKV || kResid) ? layer_tokens(g) : a.rows;
    // Three register sets in rotation: the set of tile t is refilled with tile
    // t + 3's rows right after its copies are issued, so no instruction reads a
    // table value before about two tiles have passed (a register copy of a
    // pending load would stall the warp until the load lands).
    int tokA[4], tokB[4], tokC[4];
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {
      tokA[grp] = row_tok(m_first, grp);
      tokB[grp] = row_tok(m_first + m_step, grp);
      tokC[grp] = row_tok(m_first + 2 * m_step, grp);
    }
    auto tile = [&](long long m, long long t, int (&tok)[4]) {
      const int s = (int)(t % STAGES);
      if (tid == 0) VSWIN_TRACE_EVENT(kTraceG + 0, trace_n, 50);
      if (t >= STAGES && !s_abort &&
          !mbar_wait(&a_free[s], (uint32_t)((t / STAGES) - 1) & 1, a.ctx.err, kErrWaitMma, lim))
        s_abort = 1;
      uint8_t* dA = sA + s * ws_a_bytes(K);
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        const int row = warp * 32 + grp * 8 + sub;
        uint8_t* drow = dA + (row >> 3) * sboA + (row & 7) * 16;
        // QKV: the row's source token; the fused projection's table holds the
        // residual's token, its A row is the chunk row itself
        long long src = tok[grp];
        if (!index_ok(src, -1, tok_extent, a.ctx.err)) src = -1;
        if (kResid) {
          const long long rA = m * kBM + row;
          src = (m < mtiles && rA < a.rows) ? rA : -1;
        }
        const long long sg = src < 0 ? 0 : src * lda;
        for (int kc = cq; kc < Kx / 8; kc += 4)
          cp_async_16(drow + kc * 128, a.A + sg + kc * 8, src < 0 ? 0u : 16u);
      }
      cp_async_mbar_arrive_noinc(&a_full[s]);  // arrives once this thread's copies have landed
      if (kResid) {
        // the tile's residual rows (x at the output tokens, this CTA's columns)
        const int rs = (int)(t % kWsResSlots);
        if (t >= kWsResSlots && !s_abort &&
            !mbar_wait(&res_free[rs], (uint32_t)((t / kWsResSlots) - 1) & 1, a.ctx.err, kErrWaitMma, lim))
          s_abort = 1;
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
          const int row = warp * 32 + grp * 8 + sub;
          const int tk = index_ok(tok[grp], -1, tok_extent, a.ctx.err) ? tok[grp] : -1;
          uint8_t* drow = sRes + rs * res_slot_bytes + row * ws_res_row_bytes(BN);
          const __nv_bfloat16* srow = a.resid + (tk < 0 ? 0 : (long long)tk * g.C) + n0;
          for (int kc = cq; kc < BN / 8; kc += 4) cp_async_16(drow + kc * 16, srow + kc * 8, tk < 0 ? 0u : 16u);
        }
        cp_async_mbar_arrive_noinc(&res_full[rs]);
      }
      if (tid == 0) VSWIN_TRACE_EVENT(kTraceG + 0, trace_n, 51);
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) tok[grp] = row_tok(m + 3 * m_step, grp);
    };
    long long t = 0;
    for (long long m = m_first; m < mtiles; m += 3 * m_step, t += 3) {
      tile(m, t, tokA);
      if (m + m_step >= mtiles) break;
      tile(m + m_step, t + 1, tokB);
      if (m + 2 * m_step >= mtiles) break;
      tile(m + 2 * m_step, t + 2, tokC);
    }
    cp_async_wait_all();  // nothing in flight when the CTA ends
  } else if (warp == kWsMmaWarp || warp == kWsMma2Warp) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const int parity = warp == kWsMmaWarp ? 0 : 1;  // the tiles (and accumulator) of this thread
      if (!mbar_wait(b_full, 0, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
      fence_proxy_async_smem();  // the gathered bytes, written by cp.async, are read by the tensor core
      const uint32_t idesc = idesc_bf16(kBM, BN, 0, 1);
      const uint32_t baddr = smem_u32(sB);
      long long t = parity;
      for (long long m = m_first + parity * m_step; m < mtiles; m += 2 * m_step, t += 2) {
        const int s = (int)(t % STAGES), buf = (int)(t & 1);
        if (parity == 0) VSWIN_TRACE_EVENT(kTraceG + 1, trace_n, 60);
        if (!s_abort && !mbar_wait(&a_full[s], (uint32_t)(t / STAGES) & 1, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
        if (kLn && !s_abort && !mbar_wait(&a_ext[s], (uint32_t)(t / STAGES) & 1, a.ctx.err, kErrWaitLoad, lim))
          s_abort = 1;
        fence_proxy_async_smem();
        if (parity == 0) VSWIN_TRACE_EVENT(kTraceG + 1, trace_n, 61);
        if (t >= 2 && !s_abort &&
            !mbar_wait(&acc_free[buf], (uint32_t)((t >> 1) - 1) & 1, a.ctx.err, kErrWaitMma, lim))
          s_abort = 1;
        tc_fence_after();
        if (!s_abort) {
          const uint32_t aaddr = smem_u32(sA + s * ws_a_bytes(K));
          for (int ks = 0; ks < K / 16; ++ks)
            umma_ss(tmem + buf * BN, smem_desc(aaddr + ks * 256, 128, sboA),
                    smem_desc(baddr + ks * 2 * lboB, lboB, 128), idesc, ks > 0);
          umma_commit(&a_free[s]);
          umma_commit(&acc_full[buf]);
          if (parity == 0) VSWIN_TRACE_EVENT(kTraceG + 1, trace_n, 62);
        }
      }
    }
    __syncwarp();
  } else if (kLn && warp >= kStat0) {
    // ---------------------------------------------------------------- statistics (kLn)
    // kLn: the layer norm's statistics of tile t's rows (statistics thread p:
    // row p), from the gathered bf16 values once they have landed -- one pass of
    // sums and sums of squares (fp32, two channels per instruction), the biased
    // variance E[x^2] - mean^2 and rstd = 1 / sqrt(var + eps) (torch.nn.LayerNorm's
    // definition). The row's -mean goes into the stage's extra K step as two bf16
    // halves (-mean_hi, -mean_hi, -mean_lo, -mean_lo, 0 ...), against the folded
    // weights' rows (colsum_hi, colsum_lo, colsum_hi, colsum_lo, 0 ...): the MMA
    // then accumulates x Wt - mean colsum. Padding rows and rows past the end get
    // zeros there and rstd 0; the epilogue reads (0, rstd) from the ring.
    auto tile_stats = [&](long long m, long long t) {
      const int s = (int)(t % STAGES);
      const int p = tid - kStat0 * 32;
      const long long r = m * kBM + p;
      const int tk = (m < mtiles && r < a.rows) ? a.rowsrc[r] : -1;
      if (!s_abort && !mbar_wait(&a_full[s], (uint32_t)(t / STAGES) & 1, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
      uint8_t* row = sA + s * ws_a_bytes(K) + (p >> 3) * sboA + (p & 7) * 16;
      float mean = 0.f, rstd = 0.f;
      if (tk >= 0 && !s_abort) {
        float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
        for (int kc = 0; kc < Kx / 8; ++kc) {
          const uint4 v = *reinterpret_cast<const uint4*>(row + kc * 128);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(h2[k]);
            s1 = __fadd2_rn(s1, f);
            s2 = __ffma2_rn(f, f, s2);
          }
        }
        mean = (s1.x + s1.y) / (float)Kx;
        const float var = fmaxf((s2.x + s2.y) / (float)Kx - mean * mean, 0.f);
        rstd = 1.0f / sqrtf(var + a.ln_eps);
      }
      const __nv_bfloat16 mh = __float2bfloat16_rn(-mean);
      const __nv_bfloat16 ml = __float2bfloat16_rn(-mean - __bfloat162float(mh));
      const uint32_t mhb = __bfloat16_as_ushort(mh), mlb = __bfloat16_as_ushort(ml);
      const uint32_t hh = mhb | (mhb << 16), ll = mlb | (mlb << 16);
      *reinterpret_cast<uint4*>(row + (Kx / 8) * 128) = make_uint4(hh, ll, 0u, 0u);
      *reinterpret_cast<uint4*>(row + (Kx / 8 + 1) * 128) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();  // the extra columns are a tensor-core operand
      mbar_arrive(&a_ext[s]);
      sStats[(t % kWsStatSlots) * kBM + p] = make_float2(0.f, rstd);
      mbar_arrive(&stats_full[t % kWsStatSlots]);
    };
    long long t = 0;
    for (long long m = m_first; m < mtiles; m += m_step, ++t) tile_stats(m, t);
  } else {
    // ---------------------------------------------------------------- epilogue
    // A warp may only touch TMEM lanes 32 * (warp % 4) .. +31: three (two with
    // the fused pre-norm) warps per lane quarter, each taking a share of the
    // columns (whole 8-column groups).
    const int q = warp & 3, hf = (warp - kWsEpi0) >> 2;
    constexpr int kPerQ = kEpiWarps / 4;
    const int c_lo = (hf * (BN / 8)) / kPerQ * 8, c_hi = ((hf + 1) * (BN / 8)) / kPerQ * 8;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const size_t win_elems = (size_t)g.heads * a.slab.head_elems();  // one window's q / k / v block
    // projection: this row's output row, loaded one tile ahead (the loaded
    // value is first used a tile later)
    auto out_row = [&](long long m) -> int {
      const long long r = m * kBM + q * 32 + lane;
      const int dr = (MODE == kPROJ && m < mtiles && r < a.rows) ? a.rowsrc[r] : -1;
      return index_ok(dr, -1, layer_tokens(g), a.ctx.err) ? dr : -1;
    };
    int dr_next = out_row(m_first);
    // columns handled per TMEM wait (the residual's registers and the norm's
    // extra terms need room)
    constexpr int kCh = kResid ? 32 : 48;
    // kResid: the residual of this warp's column chunk, from the tile's slot
    // in shared memory (gathered by the producer warps)
    uint4 xr[kResid ? kCh / 8 : 1];
    long long t = 0;
    for (long long m = m_first; m < mtiles; m += m_step, ++t) {
      const int buf = (int)(t & 1);
      const long long r = m * kBM + q * 32 + lane;
      const bool row_ok = r < a.rows;
      const int dr_cur = dr_next;
      dr_next = out_row(m + m_step);
      // this row's destination: QKV, the window's block and the row term of the
      // q slab and of the k / v slabs; projection, the output row
      __nv_bfloat16* rbase = nullptr;
      int q_term = 0, kv_term = 0;
      // the last key of a 7-key line also zero-fills the line's eighth (padding)
      // row, so that every 32-byte sector of the k / v slabs is written whole
      // (a partly written sector costs a DRAM read to merge when it leaves L2)
      bool kv_pad = false;
      // kLn: (-mean * rstd, rstd) of this row's token, (0, 0) for a padding row
      float2 st = make_float2(0.f, 0.f);
      if (row_ok) {
        if (MODE == kQKV) {
          const int ri = (int)r;  // rows < 2^31 (checked by the caller)
          const int slab_win = ri / g.N;
          const int slot = ri - slab_win * g.N;
          const int kvr = a.slab.kv_row(slot);
          kv_pad = a.slab.kv8 && (kvr & 7) == 6;
          q_term = (slot >> 3) * 256 + (slot & 7) * 8;
          kv_term = (kvr >> 3) * 256 + (kvr & 7) * 8;
          rbase = a.dst + (size_t)slab_win * win_elems;
        } else {
          const long long dr = dr_cur;
          if (dr >= 0) {
            rbase = a.dst + dr * g.C + n0;
          }
        }
      }
      if (warp == kWsEpi0 && lane == 0) VSWIN_TRACE_EVENT(kTraceG + 2, trace_n, 70);
      if (!s_abort && !mbar_wait(&acc_full[buf], (uint32_t)(t >> 1) & 1, a.ctx.err, kErrWaitMma, lim)) s_abort = 1;
      if (kResid && !s_abort &&
          !mbar_wait(&res_full[t % kWsResSlots], (uint32_t)(t / kWsResSlots) & 1, a.ctx.err, kErrWaitLoad, lim))
        s_abort = 1;
      if (kLn) {  // this tile's row statistics, written by the gathering threads
        if (!s_abort &&
            !mbar_wait(&stats_full[t % kWsStatSlots], (uint32_t)(t / kWsStatSlots) & 1, a.ctx.err, kErrWaitLoad, lim))
          s_abort = 1;
        st = sStats[(t % kWsStatSlots) * kBM + q * 32 + lane];
      }
      if (warp == kWsEpi0 && lane == 0) VSWIN_TRACE_EVENT(kTraceG + 2, trace_n, 71);
      tc_fence_after();
      if (!s_abort && m * kBM + q * 32 < a.rows) {
        // all of this warp's columns (up to kCh at a time) loaded before one wait
        for (int c0 = c_lo; c0 < c_hi; c0 += kCh) {
          const int n = c_hi - c0 < kCh ? c_hi - c0 : kCh;  // a multiple of 8
          uint32_t u[kCh];
          if (kResid) {
            const uint8_t* xrow =
                sRes + (t % kWsResSlots) * res_slot_bytes + (q * 32 + lane) * ws_res_row_bytes(BN) + c0 * 2;
#pragma unroll
            for (int j = 0; j < kCh / 8; ++j)
              if (j * 8 < n) xr[j] = *reinterpret_cast<const uint4*>(xrow + 16 * j);
          }
          const uint32_t ta = tmem + lane_base + buf * BN + c0;
#pragma unroll
          for (int j = 0; j < kCh / 8; ++j)
            if (j * 8 < n)
              asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                           : "=r"(u[8 * j + 0]), "=r"(u[8 * j + 1]), "=r"(u[8 * j + 2]), "=r"(u[8 * j + 3]),
                             "=r"(u[8 * j + 4]), "=r"(u[8 * j + 5]), "=r"(u[8 * j + 6]), "=r"(u[8 * j + 7])
                           : "r"(ta + 8 * j));
          tmem_wait_ld_keep(u);
#pragma unroll
          for (int g8 = 0; g8 < kCh / 8; ++g8) {
            if (g8 * 8 >= n) break;
            const int cc = c0 + g8 * 8;
            const ColGroup cg = sGrp[cc >> 3];
            // plain: v = acc * scale + bias * scale. kLn (a token row): the
            // accumulator already holds x Wt - mean colsum
            // (the extra K step), so v = rstd * scale * acc + folded bias * scale; a
            // padding row (rstd = 0) keeps the plain bias
            const float* bsrc = (kLn && st.y != 0.f) ? sBb : sBias;
            const float4 b0 = *reinterpret_cast<const float4*>(bsrc + cc);
            const float4 b1 = *reinterpret_cast<const float4*>(bsrc + cc + 4);
            float2 sc = make_float2(cg.scale, cg.scale);
            if (kLn && st.y != 0.f) sc = make_float2(st.y * cg.scale, st.y * cg.scale);
            // two columns per instruction
            float2 v01 = __ffma2_rn(make_float2(__uint_as_float(u[g8 * 8 + 0]), __uint_as_float(u[g8 * 8 + 1])),
                                    sc, make_float2(b0.x, b0.y));
            float2 v23 = __ffma2_rn(make_float2(__uint_as_float(u[g8 * 8 + 2]), __uint_as_float(u[g8 * 8 + 3])),
                                    sc, make_float2(b0.z, b0.w));
            float2 v45 = __ffma2_rn(make_float2(__uint_as_float(u[g8 * 8 + 4]), __uint_as_float(u[g8 * 8 + 5])),
                                    sc, make_float2(b1.x, b1.y));
            float2 v67 = __ffma2_rn(make_float2(__uint_as_float(u[g8 * 8 + 6]), __uint_as_float(u[g8 * 8 + 7])),
                                    sc, make_float2(b1.z, b1.w));
            if (kResid) {
              const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xr[g8]);
              v01 = __fadd2_rn(v01, __bfloat1622float2(xp[0]));
              v23 = __fadd2_rn(v23, __bfloat1622float2(xp[1]));
              v45 = __fadd2_rn(v45, __bfloat1622float2(xp[2]));
              v67 = __fadd2_rn(v67, __bfloat1622float2(xp[3]));
            }
            const uint4 w = make_uint4(pack_bf16x2(v01.x, v01.y), pack_bf16x2(v23.x, v23.y),
                                       pack_bf16x2(v45.x, v45.y), pack_bf16x2(v67.x, v67.y));
            if (MODE == kPROJ) {  // staged; copied out row by row below
              *reinterpret_cast<uint4*>(sOut + (t & 1) * res_slot_bytes + (q * 32 + lane) * ws_res_row_bytes(BN) +
                                        cc * 2) = w;
            } else if (rbase) {
              __nv_bfloat16* dst = rbase + cg.off + (cg.is_q ? q_term : kv_term);
              *reinterpret_cast<uint4*>(dst) = w;
              if (kv_pad && !cg.is_q) *reinterpret_cast<uint4*>(dst + 8) = make_uint4(0, 0, 0, 0);
            }
          }
        }
      }
      if (MODE == kPROJ && hf == 0) sDst[(t & 1) * kBM + q * 32 + lane] = rbase ? dr_cur : -1;
      tc_fence_before();
      __syncwarp();
      if (warp == kWsEpi0 && lane == 0) VSWIN_TRACE_EVENT(kTraceG + 2, trace_n, 72);
      if (lane == 0) {
        mbar_arrive(&acc_free[buf]);
        if (kResid) mbar_arrive(&res_free[t % kWsResSlots]);
      }
      if (MODE == kPROJ) {
        // the staged tile to its output rows: consecutive threads take consecutive
        // 16-byte chunks of a row (whole rows per warp instruction, not one
        // scattered chunk per thread); the buffer is rewritten two tiles later,
        // after every epilogue warp has passed the next tile's barrier
        named_bar_sync(1, kEpiWarps * 32);
        const int cpr = BN / 8;  // chunks per row
        const uint8_t* sb = sOut + (t & 1) * res_slot_bytes;
        const int* db = sDst + (t & 1) * kBM;
        for (int k = tid - kWsEpi0 * 32; k < kBM * cpr; k += kEpiWarps * 32) {
          const int row = k / cpr, c8 = k - row * cpr;
          const int dr = db[row];
          if (dr >= 0 && !s_abort)
            *reinterpret_cast<uint4*>(a.dst + (long long)dr * g.C + n0 + c8 * 8) =
                *reinterpret_cast<const uint4*>(sb + row * ws_res_row_bytes(BN) + c8 * 16);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWsMmaWarp) tmem_dealloc(tmem, tcols);
}

// ============================================================================ attention
constexpr int kAttnThreads = 128;
constexpr int kD = 32;                 // head width of this path
constexpr int kSlabRowBytes = kD * 2;  // 64
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kOCol = 160;        // O accumulators at columns 160, 192, 224

template <int P_, int MH_, int MW_>
struct Win {
  static constexpr int P = P_, MH = MH_, MW = MW_;
  static constexpr int N = P * MH * MW;
  static constexpr int NPAD = (N + 15) / 16 * 16;
  static constexpr int NB0 = NPAD < 144 ? NPAD : 144;
  static constexpr int NB1 = (NPAD - NB0) < 128 ? (NPAD - NB0) : 128;
  static constexpr int NB2 = NPAD - NB0 - NB1;
  static constexpr int NBLK = NB2 > 0 ? 3 : (NB1 > 0 ? 2 : 1);
  static constexpr int WS = 2 * MW - 1;   // table stride of dh
  static constexpr int TS = (2 * MH - 1) * WS;  // table stride of dt
  static constexpr int TABLE = (2 * P - 1) * TS;
  static constexpr int QTILES = (N + 127) / 128;
  static constexpr int QROWS = QTILES * 128 > NPAD ? QTILES * 128 : NPAD;
  // shared memory map (bytes)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QROWS * kSlabRowBytes;
  static constexpr int OFF_V = OFF_K + NPAD * kSlabRowBytes;
  static constexpr int OFF_T = OFF_V + NPAD * kSlabRowBytes;
  static constexpr int OFF_BAR = OFF_T + (TABLE * 4 + 15) / 16 * 16;
  // At least 80 KB so that no more than two CTAs (2 x 256 TMEM columns) share an SM.
  static constexpr int SMEM = (OFF_BAR + 64) < 81920 ? 81920 : (OFF_BAR + 64);
  static_assert(NB2 <= 128, "window too large for this path");
  static_assert(NPAD <= 400, "window too large for this path");
};

struct AttnArgs {
  Geom g;
  KernelCtx ctx;
  SlabLayout slab;
  float exact_below;           // rows whose softmax sum is below this are recomputed exactly
  const __nv_bfloat16* qkv;    // per (window, head): q | k | v slabs
  const __nv_bfloat16* table;  // [rows][heads]
  __nv_bfloat16* o;            // [nwin][N][C]
  long long win0, nwin;
  // optional (null: not written): per (window slot, head) the reference and the
  // row sum the probabilities were normalised with, in the exp2 domain --
  // P = 2^(s + b - m) / l with s the scaled score and b the table entry
  // (log2 e units); for an exactly recomputed row its true maximum and sum
  float2* stats;
};

// Per-thread row context for one query tile.
template <class Wn>
struct RowCtx {
  const float* tb;  // table row base: tb_smem + c(i); key j reads tb[-e(j)]
  bool okt[Wn::P], okh[Wn::MH], okw[Wn::MW];
};

// Softmax of one key block for the thread's query row: S (TMEM, log2 units,
// already scaled) + bias (log2 units) [+ mask] -> P (bf16, TMEM), row max m
// and row sum l of the block.
template <class Wn, int KB0, int NB, bool MASKED>
__device__ __forceinline__ void softmax_block(uint32_t trow, const RowCtx<Wn>& rc, float& m_out,
                                              float& l_out) {
  float t[NB];
#pragma unroll
  for (int c = 0; c < NB / 16; ++c) {
    uint32_t u[16];
    tmem_ld16(trow + c * 16, u);
#pragma unroll
    for (int k = 0; k < 16; ++k) t[c * 16 + k] = __uint_as_float(u[k]);
  }
  tmem_wait_ld();
  float m = -INFINITY;
#pragma unroll
  for (int jj = 0; jj < NB; ++jj) {
    const int j = KB0 + jj;
    if (j < Wn::N) {
      const int pt = j / (Wn::MH * Wn::MW), ph = (j / Wn::MW) % Wn::MH, pw = j % Wn::MW;
      float v = t[jj] + rc.tb[-(pt * Wn::TS + ph * Wn::WS + pw)];
      if (MASKED) v = (rc.okt[pt] && rc.okh[ph] && rc.okw[pw]) ? v : -INFINITY;
      t[jj] = v;
      m = fmaxf(m, v);
    } else {
      t[jj] = -INFINITY;
    }
  }
  const float mm = (m == -INFINITY) ? 0.f : m;
  float l0 = 0.f, l1 = 0.f;
  uint32_t pk[NB / 2];
#pragma unroll
  for (int jj = 0; jj < NB; jj += 2) {
    const float p0 = ex2_approx(t[jj] - mm);
    const float p1 = ex2_approx(t[jj + 1] - mm);
    l0 += p0;
    l1 += p1;
    pk[jj / 2] = pack_bf16x2(p0, p1);
  }
#pragma unroll
  for (int c = 0; c < NB / 16; ++c) tmem_st8(trow + c * 8, &pk[c * 8]);
  m_out = m;
  l_out = l0 + l1;
}

template <class Wn, bool MASKED>
__device__ __forceinline__ void softmax_all_blocks(int b, uint32_t trow, const RowCtx<Wn>& rc, float* m,
                                                   float* l) {
  if (b == 0) softmax_block<Wn, 0, Wn::NB0, MASKED>(trow, rc, m[0], l[0]);
  if constexpr (Wn::NBLK > 1)
    if (b == 1) softmax_block<Wn, Wn::NB0, Wn::NB1, MASKED>(trow, rc, m[1], l[1]);
  if constexpr (Wn::NBLK > 2)
    if (b == 2) softmax_block<Wn, Wn::NB0 + Wn::NB1, Wn::NB2, MASKED>(trow, rc, m[2], l[2]);
}

template <class Wn>
__device__ __forceinline__ int block_start(int b) {
  return b == 0 ? 0 : (b == 1 ? Wn::NB0 : Wn::NB0 + Wn::NB1);
}
template <class Wn>
__device__ __forceinline__ int block_width(int b) {
  return b == 0 ? Wn::NB0 : (b == 1 ? Wn::NB1 : Wn::NB2);
}

template <class Wn>
__global__ void __launch_bounds__(kAttnThreads, 2) attention_kernel(AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem + Wn::OFF_Q;
  uint8_t* sK = smem + Wn::OFF_K;
  uint8_t* sV = smem + Wn::OFF_V;
  float* sT = reinterpret_cast<float*>(smem + Wn::OFF_T);
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + Wn::OFF_BAR);
  uint64_t* bar_s = bar_ld + 1;
  uint64_t* bar_o = bar_ld + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_ld + 3);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geom& g = a.g;
  const long long nitems = a.nwin * g.heads;
  const uint32_t slab_bytes = Wn::NPAD * kSlabRowBytes;

  if (tid == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  // Rows of the last query tile past the slab are never loaded: keep them zero.
  for (int k = Wn::NPAD * kSlabRowBytes / 16 + tid; k < Wn::QROWS * kSlabRowBytes / 16; k += kAttnThreads)
    reinterpret_cast<uint4*>(sQ)[k] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);

  uint32_t ph_ld = 0, ph_s = 0, ph_o = 0;
  int cur_head = -1;
  const uint32_t qaddr = smem_u32(sQ), kaddr = smem_u32(sK), vaddr = smem_u32(sV);

#pragma unroll 1
  for (long long item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int h = (int)(item / a.nwin);
    const long long wl = item % a.nwin;
    const long long win = a.win0 + wl;
    if (tid == 0) {
      const __nv_bfloat16* base = a.qkv + ((size_t)wl * g.heads + h) * a.slab.head_elems();
      mbar_arrive_expect_tx(bar_ld, 3 * slab_bytes);
      bulk_g2s(sQ, base, slab_bytes, bar_ld);
      bulk_g2s(sK, base + (size_t)Wn::NPAD * kD, slab_bytes, bar_ld);
      bulk_g2s(sV, base + 2 * (size_t)Wn::NPAD * kD, slab_bytes, bar_ld);
    }
    if (h != cur_head) {
      for (int k = tid; k < Wn::TABLE; k += kAttnThreads)
        sT[k] = __bfloat162float(a.table[(size_t)k * g.heads + h]) * kLog2e;
      cur_head = h;
    }
    if (!mbar_wait(bar_ld, ph_ld, a.ctx.err, kErrWaitLoad, a.ctx.wait_limit)) s_abort = 1;
    ph_ld ^= 1;
    // Key slots past N are padding of the operand tile: zero them. A slab row
    // n is spread over four 16-byte pieces at (n/8)*512 + chunk*128 + (n%8)*16.
    for (int k = tid; k < (Wn::NPAD - Wn::N) * 4; k += kAttnThreads) {
      const int n = Wn::N + (k >> 2), chunk = k & 3;
      const int off = (n >> 3) * 512 + chunk * 128 + (n & 7) * 16;
      *reinterpret_cast<uint4*>(sK + off) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sV + off) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (s_abort) break;

    const int split = window_split_bits(g, (int)(win % g.nW));
    const bool masked = split != 0;

#pragma unroll 1
    for (int qt = 0; qt < Wn::QTILES; ++qt) {
      // per-row context
      const int i = qt * 128 + warp * 32 + lane;
      const bool warp_active = qt * 128 + warp * 32 < Wn::N;
      const int ie = i < Wn::N ? i : Wn::N - 1;
      const int pt_i = ie / (Wn::MH * Wn::MW), ph_i = (ie / Wn::MW) % Wn::MH, pw_i = ie % Wn::MW;
      RowCtx<Wn> rc;
      rc.tb = sT + (pt_i + Wn::P - 1) * Wn::TS + (ph_i + Wn::MH - 1) * Wn::WS + (pw_i + Wn::MW - 1);
      {
        const int cut_t = Wn::P - g.sh[0], cut_h = Wn::MH - g.sh[1], cut_w = Wn::MW - g.sh[2];
        const bool rt = pt_i >= cut_t, rh = ph_i >= cut_h, rw = pw_i >= cut_w;
#pragma unroll
        for (int k = 0; k < Wn::P; ++k) rc.okt[k] = !(split & 1) || ((k >= cut_t) == rt);
#pragma unroll
        for (int k = 0; k < Wn::MH; ++k) rc.okh[k] = !(split & 2) || ((k >= cut_h) == rh);
#pragma unroll
        for (int k = 0; k < Wn::MW; ++k) rc.okw[k] = !(split & 4) || ((k >= cut_w) == rw);
      }
      float mrow[3] = {-INFINITY, -INFINITY, -INFINITY}, lrow[3] = {0.f, 0.f, 0.f};

      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          umma_ss(tmem, smem_desc(qaddr + qt * 8192 + ks * 256, 128, 512),
                  smem_desc(kaddr + ks * 256, 128, 512), idesc_bf16(128, Wn::NB0, 0, 0), ks);
        umma_commit(bar_s);
      }
#pragma unroll 1
      for (int b = 0; b < Wn::NBLK; ++b) {
        if (!mbar_wait(bar_s, ph_s, a.ctx.err, kErrWaitMma, a.ctx.wait_limit)) s_abort = 1;
        ph_s ^= 1;
        __syncthreads();
        tc_fence_after();
        if (warp_active && !s_abort) {
          if (masked)
            softmax_all_blocks<Wn, true>(b, trow, rc, mrow, lrow);
          else
            softmax_all_blocks<Wn, false>(b, trow, rc, mrow, lrow);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && !s_abort) {
          tc_fence_after();
          const int kb0 = block_start<Wn>(b), nb = block_width<Wn>(b);
          for (int ks = 0; ks < nb / 16; ++ks)
            umma_ts(tmem + kOCol + 32 * b, tmem + 8 * ks,
                    smem_desc(vaddr + ((kb0 + 16 * ks) >> 3) * 512, 512, 128), idesc_bf16(128, kD, 0, 1),
                    ks > 0);
          if (b + 1 < Wn::NBLK) {
            const int nk0 = block_start<Wn>(b + 1), nnb = block_width<Wn>(b + 1);
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
              umma_ss(tmem, smem_desc(qaddr + qt * 8192 + ks * 256, 128, 512),
                      smem_desc(kaddr + (nk0 >> 3) * 512 + ks * 256, 128, 512), idesc_bf16(128, nnb, 0, 0),
                      ks);
            umma_commit(bar_s);
          } else {
            umma_commit(bar_o);
          }
        }
        if (s_abort) break;
      }
      if (s_abort) break;
      if (!mbar_wait(bar_o, ph_o, a.ctx.err, kErrWaitMma, a.ctx.wait_limit)) s_abort = 1;
      ph_o ^= 1;
      __syncthreads();
      tc_fence_after();
      if (warp_active && !s_abort) {
        float M = mrow[0];
#pragma unroll
        for (int b = 1; b < Wn::NBLK; ++b) M = fmaxf(M, mrow[b]);
        float alpha[3], L = 0.f;
#pragma unroll
        for (int b = 0; b < Wn::NBLK; ++b) {
          alpha[b] = mrow[b] == -INFINITY ? 0.f : ex2_approx(mrow[b] - M);
          L += alpha[b] * lrow[b];
        }
        const float inv = 1.0f / L;
        float o[kD];
#pragma unroll
        for (int k = 0; k < kD; ++k) o[k] = 0.f;
#pragma unroll
        for (int b = 0; b < Wn::NBLK; ++b) {
          uint32_t u0[16], u1[16];
          tmem_ld16(trow + kOCol + 32 * b, u0);
          tmem_ld16(trow + kOCol + 32 * b + 16, u1);
          tmem_wait_ld();
          const float f = alpha[b] * inv;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            o[k] = fmaf(__uint_as_float(u0[k]), f, o[k]);
            o[16 + k] = fmaf(__uint_as_float(u1[k]), f, o[16 + k]);
          }
        }
        if (i < Wn::N) {
          __nv_bfloat16* dst = a.o + ((size_t)wl * Wn::N + i) * g.C + h * kD;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            reinterpret_cast<uint4*>(dst)[q] =
                make_uint4(pack_bf16x2(o[8 * q + 0], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                           pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
        }
      }
      tc_fence_before();
      __syncthreads();
      if (s_abort) break;
    }
    if (s_abort) break;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

template <class Wn>
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e = cudaFuncSetAttribute(attention_kernel<Wn>, cudaFuncAttributeMaxDynamicSharedMemorySize, Wn::SMEM);
  if (e != cudaSuccess) return e;
  const long long items = a.nwin * a.g.heads;
  long long grid = 2LL * sms;
  if (grid > items) grid = items;
  prof_begin(kKindAttn, st);
  attention_kernel<Wn><<<(unsigned)grid, kAttnThreads, Wn::SMEM, st>>>(a);
  prof_end(kKindAttn, st);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================ attention, (P,7,7) windows
//
// Persistent, warp-specialised kernel, one CTA per SM, 512 threads:
//   warps 0-3    preparation of (window, head) items, two in flight: bulk loads
//                of the q / k / v slabs, the head's bias table in log2 units,
//                key norms, the extension rows of the score MMA (below), zeroed
//                v padding;
//   warps 4-15   three softmax groups of four warps (one per TMEM lane
//                quarter); group g owns this CTA's query tiles g, g + 3, ...
//                (128-row tiles, items in order).
// Keys are taken in blocks of up to 14 lines of 8 columns (the 7 keys of one
// (pt, ph) line and a padding column). Per block: S = q k^T into the group's
// 112 TMEM columns (q from TMEM, where the group copies its tile's q rows and
// their extension rows, so that only keys are read from shared memory), the
// group turns S into bf16 P in place (4 columns per line,
// summing p as it goes), then O += P v on the tensor core. Each group issues
// its own MMAs: after a block (a named barrier over its 128 threads) one
// elected lane of the block's issuer warp (the warps take turns) issues the
// block's P v and the next block's scores into the same columns (the tensor
// core runs them in order). The softmax is bound by the latency of its
// instruction chains, so three groups (three softmax warps per SM
// sub-partition) keep the exponential units busy while a group waits for its
// next scores. With three or more tiles per item, a tile's epilogue (O / l to
// memory) runs inside the group's next tile's first block, when its P v has
// long completed.
//
// Softmax reference. Every query row i uses one reference for all its keys,
//   m_i = |q_i| * max_j |k_j| + max(bias) + 1   (log2 units, q pre-scaled),
// an upper bound of every score + bias of the row (Cauchy-Schwarz): no
// exponential overflows, blocks need no rescaling, and O and l accumulate
// straight across blocks. Should the bound's slack make the row sum underflow
// (below 2^-100: logits spanning more than ~69 natural-log units), the row is
// recomputed exactly by a two-pass softmax on the CUDA cores (w7_exact_row).
//
// The reference and the shifted-window mask enter the score MMA as one extra
// K = 16 step whose two 8-column halves read the same 16-byte rows (descriptor
// K stride 0):
//   query row i:  (-m_i/2, 1/2, r_t(i)/2, r_h(i)/2, r_w(i)/2, 0, 0, 0)
//   key j:        (1, -256 (r_t(j) + r_h(j) + r_w(j)), y_t(j), y_h(j), y_w(j), 0, 0, 0)
// where r_a is the region bit of a slot on split axis a (0 on other axes) and
// y_a = -256 (1 - 2 r_a) on split axes. Over both halves the step adds
// -m_i - 256 * #{axes whose regions differ}: every allowed key of row i gets
// the same -m_i (identical step inputs), masked keys end at least 257 below
// the reference and exponentiate to exactly 0. -m_i/2 is rounded towards
// -inf, so the effective reference is never below m_i.
constexpr int kA7PrepWarps = 4;
constexpr int kA7Groups = 3;
constexpr int kA7Soft0 = kA7PrepWarps;                               // first softmax warp
constexpr int kA7Threads = (kA7PrepWarps + 4 * kA7Groups) * 32;  // 512
// Registers per thread: launched at 128 (the most 512 threads get), then the
// preparation warpgroup gives some to the three softmax warpgroups.
constexpr int kA7RegsLaunch = 128, kA7RegsPrep = 48, kA7RegsSoft = 152;
static_assert(128 * kA7RegsPrep + 384 * kA7RegsSoft <= kA7Threads * kA7RegsLaunch, "register budgets");
constexpr uint32_t kA7TmemCols = 512;
// TMEM columns: group g has S / P at [144 g, 144 g + 112) and O at
// [144 g + 112, 144 g + 144); the q rows of its tile at [432 + 16 g, + 16) and
// their extension rows (twice) at [480 + 8 g, + 8). Column offsets stay
// aligned to the widths that access them.
constexpr uint32_t kA7GroupCols = 144;
constexpr uint32_t kA7OCol = 112;
constexpr uint32_t kA7QBase = 432;
constexpr uint32_t kA7QXBase = 480;

template <int P_>
struct W7 {
  static constexpr int P = P_;
  static constexpr int N = P * 49;
  static constexpr int QSLAB = (N + 15) / 16 * 16;           // q slab rows
  static constexpr int KLINES = P * 7;                       // key lines of 7 real keys
  static constexpr int KCOLS = (KLINES * 8 + 31) / 32 * 32;  // k / v slab rows (padded key columns)
  static constexpr int LINES = KCOLS / 8;
  static constexpr int NBLK = (LINES + 13) / 14;
  static constexpr int BL = ((LINES + NBLK - 1) / NBLK + 1) / 2 * 2;  // lines per block but the last
  static constexpr int LAST = LINES - (NBLK - 1) * BL;
  static constexpr int TABLE = (2 * P - 1) * 169;
  static constexpr int QTILES = (N + 127) / 128;
  static constexpr int TAIL = N - (QTILES - 1) * 128;  // rows of the last tile
  // A last tile of at most 32 rows is placed in lane quarter (item & 3), so that
  // its work rotates over the four SM sub-partitions.
  static constexpr bool ROTATE = QTILES > 1 && TAIL <= 32;
  static constexpr int QXROWS = QTILES * 128;
  // shared memory per item buffer
  static constexpr int QB = QSLAB * kSlabRowBytes;
  static constexpr int KB = KCOLS * kSlabRowBytes;
  static constexpr int QXB = QXROWS * 16;
  static constexpr int KXB = KCOLS * 16;
  static constexpr int TB = (TABLE * 4 + 127) / 128 * 128;
  static constexpr int ITEM_BYTES = QB + 2 * KB + QXB + KXB + TB;
  // two item buffers (the next item is prepared while this one is computed)
  // when they fit, else one (temporal windows of 16: 210 KB per item)
  static constexpr int NBUF = 2 * ITEM_BYTES + 256 <= 227 * 1024 ? 2 : 1;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NBUF * QB;
  static constexpr int OFF_V = OFF_K + NBUF * KB;
  static constexpr int OFF_QX = OFF_V + NBUF * KB;
  static constexpr int OFF_KX = OFF_QX + NBUF * QXB;
  static constexpr int OFF_T = OFF_KX + NBUF * KXB;
  static constexpr int OFF_BAR = OFF_T + NBUF * TB;
  static constexpr int SMEM = OFF_BAR + 256;
  static_assert(BL <= 14 && LAST > 0 && LAST % 2 == 0, "key blocks of line pairs must fit 112 TMEM columns");
  // a tile's operand rows beyond the q slab read the following buffers (their
  // results land in TMEM lanes that are never used)
  static_assert(OFF_Q + (NBUF - 1) * QB + QXROWS * kSlabRowBytes <= SMEM, "tile rows must stay inside shared memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Item buffer of this CTA's j-th item, and how many earlier items used it.
template <class Wn>
__device__ __forceinline__ int w7_buf(long long j) {
  return Wn::NBUF == 2 ? (int)(j & 1) : 0;
}
template <class Wn>
__device__ __forceinline__ long long w7_use(long long j) {
  return Wn::NBUF == 2 ? (j >> 1) : j;
}

template <class Wn>
__device__ __forceinline__ int w7_tile_row0(int qt, long long jj) {
  if (Wn::ROTATE && qt == Wn::QTILES - 1) return qt * 128 - 32 * (int)(jj & 3);
  return qt * 128;
}

// Region bit of slot coordinate c on an axis cut at `cut`, when the axis is split.
__device__ __forceinline__ int w7_region(int split_bit, int c, int cut) { return (split_bit && c >= cut) ? 1 : 0; }

// TMEM helpers for the softmax loop without a memory clobber (TMEM is not
// generic memory; their order relative to each other and to the fences is
// kept because all of them are volatile), so that shared-memory loads of the
// bias may be scheduled across them.
template <int N>
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[N]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;");
#pragma unroll
  for (int k = 0; k < N; ++k) asm volatile("" : "+r"(r[k]));
}

// Lines l and l + 1 of a block (16 TMEM columns in u): p = 2^(s + bias) for
// the 7 keys of each real line, 0 for padding columns and padding lines;
// packed into 8 bf16x2 words; the p are added to `sum`.
template <class Wn>
__device__ __forceinline__ void w7_line_pair(int l, const uint32_t (&u)[16], const float* tb_row, uint32_t (&pk)[8],
                                             float& sum) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int line = l + c;
    float p[8];
    if (line < Wn::KLINES) {
      const float* tbr = tb_row - ((line / 7) * 169 + (line % 7) * 13);
#pragma unroll
      for (int pw = 0; pw < 7; ++pw) p[pw] = ex2_approx(__uint_as_float(u[c * 8 + pw]) + tbr[-pw]);
    } else {
#pragma unroll
      for (int pw = 0; pw < 7; ++pw) p[pw] = 0.f;
    }
    p[7] = 0.f;
    sum += ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + p[6]);
#pragma unroll
    for (int k = 0; k < 4; ++k) pk[c * 4 + k] = pack_bf16x2(p[2 * k], p[2 * k + 1]);
  }
}

__device__ __forceinline__ void tmem_st8_reg(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}

// One key block of NL lines (even) starting at line L0 for this thread's query
// row: S (TMEM columns from tS) -> bf16 P in place, 2 lines at a time (P of
// lines 2k, 2k + 1 lands on columns 8k .. 8k + 7, whose scores were read
// before), the next 2 lines' load in flight while the current ones are
// processed. Returns the block's sum of p.
template <class Wn, int NL>
__device__ __forceinline__ float w7_block(uint32_t tS, int L0, const float* tb_row) {
  float sum = 0.f;
  uint32_t ua[16], ub[16];
  tmem_ld16(tS, ua);
  tmem_wait_ld_regs(ua);
#pragma unroll
  for (int k = 0; k < NL / 2; ++k) {
    uint32_t pk[8];
    if ((k & 1) == 0) {
      if (k + 1 < NL / 2) tmem_ld16(tS + 16 * (k + 1), ub);
      w7_line_pair<Wn>(L0 + 2 * k, ua, tb_row, pk, sum);
      tmem_st8_reg(tS + 8 * k, pk);
      if (k + 1 < NL / 2) tmem_wait_ld_regs(ub);
    } else {
      if (k + 1 < NL / 2) tmem_ld16(tS + 16 * (k + 1), ua);
      w7_line_pair<Wn>(L0 + 2 * k, ub, tb_row, pk, sum);
      tmem_st8_reg(tS + 8 * k, pk);
      if (k + 1 < NL / 2) tmem_wait_ld_regs(ua);
    }
  }
  return sum;
}

// Exact recomputation of one query row (rare path, see the reference rule
// above): two-pass softmax over the allowed keys on the CUDA cores, operands
// read from shared memory; writes the row's 32 normalised outputs.
template <class Wn>
__device__ __noinline__ float2 w7_exact_row(const uint8_t* sQ, const uint8_t* sK, const uint8_t* sV,
                                            const float* tb_row, int i, uint32_t okt, uint32_t okh, uint32_t okw,
                                            float* o) {
  float q[32];
  for (int c = 0; c < 4; ++c) {
    const uint4 w = *reinterpret_cast<const uint4*>(sQ + (i >> 3) * 512 + c * 128 + (i & 7) * 16);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h2[k]);
      q[c * 8 + 2 * k] = f.x;
      q[c * 8 + 2 * k + 1] = f.y;
    }
  }
  auto score = [&](int n) {  // q . k of slab row n
    float acc = 0.f;
    for (int c = 0; c < 4; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(sK + (n >> 3) * 512 + c * 128 + (n & 7) * 16);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h2[k]);
        acc = fmaf(q[c * 8 + 2 * k], f.x, acc);
        acc = fmaf(q[c * 8 + 2 * k + 1], f.y, acc);
      }
    }
    return acc;
  };
  float m = -INFINITY;
  for (int line = 0; line < Wn::KLINES; ++line) {
    const int pt = line / 7, ph = line - 7 * pt;
    const uint32_t lm = ((okt >> pt) & (okh >> ph) & 1u) ? okw : 0u;
    for (int pw = 0; pw < 7; ++pw)
      if ((lm >> pw) & 1u) m = fmaxf(m, score(line * 8 + pw) + tb_row[-(pt * 169 + ph * 13 + pw)]);
  }
  float l = 0.f;
  for (int d = 0; d < 32; ++d) o[d] = 0.f;
  for (int line = 0; line < Wn::KLINES; ++line) {
    const int pt = line / 7, ph = line - 7 * pt;
    const uint32_t lm = ((okt >> pt) & (okh >> ph) & 1u) ? okw : 0u;
    for (int pw = 0; pw < 7; ++pw) {
      if (!((lm >> pw) & 1u)) continue;
      const int n = line * 8 + pw;
      const float pr = exp2f(score(n) + tb_row[-(pt * 169 + ph * 13 + pw)] - m);
      l += pr;
      for (int ch = 0; ch < 4; ++ch) {
        const uint4 w = *reinterpret_cast<const uint4*>(sV + (n >> 3) * 512 + ch * 128 + (n & 7) * 16);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h2[k]);
          o[ch * 8 + 2 * k] = fmaf(pr, f.x, o[ch * 8 + 2 * k]);
          o[ch * 8 + 2 * k + 1] = fmaf(pr, f.y, o[ch * 8 + 2 * k + 1]);
        }
      }
    }
  }
  const float inv = 1.0f / l;
  for (int d = 0; d < 32; ++d) o[d] *= inv;
  return make_float2(m, l);
}

// One elected lane of a converged warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Score MMA of one key block of NL lines, q rows from TMEM (tq: 16 columns of
// q, tqx: 8 columns of the extension row): the extension step first (it
// overwrites the accumulator), then the two q . k steps. Key descriptors point
// at the block's first key; one K step of 16 columns is 256 bytes (16 in
// descriptor units).
template <int NL>
__device__ __forceinline__ void w7_issue_s(uint32_t dS, uint32_t tq, uint32_t tqx, uint64_t kxd, uint64_t kd) {
  constexpr uint32_t id = idesc_bf16(128, NL * 8, 0, 0);
  umma_ts(dS, tqx, kxd, id, 0u);
  umma_ts(dS, tq, kd, id, 1u);
  umma_ts(dS, tq + 8, kd + 16, id, 1u);
}

// O (+)= P v for one key block of NL lines: 16 keys (8 P columns, 1 KB of v)
// per MMA.
template <int NL>
__device__ __forceinline__ void w7_issue_pv(uint32_t dO, uint32_t dP, uint64_t vd, bool first) {
  constexpr uint32_t id = idesc_bf16(128, kD, 0, 1);
#pragma unroll
  for (int ks = 0; ks < NL / 2; ++ks)
    umma_ts(dO, dP + 8 * ks, vd + (uint64_t)(64 * ks), id, (first && ks == 0) ? 0u : 1u);
}

// The exact path for query row i of a tile of item buffer X: mask bits of the
// row, w7_exact_row, and the row's 32 outputs to dst.
template <class Wn>
__device__ __noinline__ float2 w7_exact_store(const AttnArgs& a, const uint8_t* smem, int X, long long wl, int i,
                                              __nv_bfloat16* dst) {
  const Geom& g = a.g;
  const int pt_i = i / 49, ph_i = (i / 7) % 7, pw_i = i % 7;
  const int cut_t = Wn::P - g.sh[0], cut_h = 7 - g.sh[1], cut_w = 7 - g.sh[2];
  const int split = window_split_bits(g, (int)((a.win0 + wl) % g.nW));
  uint32_t okt = 0xFFFFFFFFu, okh = 0xFFFFFFFFu, okw = 0x7Fu;
  if (split & 1) {
    okt = 0;
    for (int k = 0; k < Wn::P; ++k) okt |= (uint32_t)((k >= cut_t) == (pt_i >= cut_t)) << k;
  }
  if (split & 2) {
    okh = 0;
    for (int k = 0; k < 7; ++k) okh |= (uint32_t)((k >= cut_h) == (ph_i >= cut_h)) << k;
  }
  if (split & 4) {
    okw = 0;
    for (int k = 0; k < 7; ++k) okw |= (uint32_t)((k >= cut_w) == (pw_i >= cut_w)) << k;
  }
  const float* sT = reinterpret_cast<const float*>(smem + Wn::OFF_T + X * Wn::TB);
  const float* tb_row = sT + (pt_i + Wn::P - 1) * 169 + (ph_i + 6) * 13 + (pw_i + 6);
  float oe[32];
  const float2 ml = w7_exact_row<Wn>(smem + Wn::OFF_Q + X * Wn::QB, smem + Wn::OFF_K + X * Wn::KB,
                                     smem + Wn::OFF_V + X * Wn::KB, tb_row, i, okt, okh, okw, oe);
  for (int k = 0; k < 4; ++k)
    reinterpret_cast<uint4*>(dst)[k] =
        make_uint4(pack_bf16x2(oe[8 * k + 0], oe[8 * k + 1]), pack_bf16x2(oe[8 * k + 2], oe[8 * k + 3]),
                   pack_bf16x2(oe[8 * k + 4], oe[8 * k + 5]), pack_bf16x2(oe[8 * k + 6], oe[8 * k + 7]));
  return ml;
}

__device__ __forceinline__ uint32_t bf16_bits(__nv_bfloat16 v) { return (uint32_t)__bfloat16_as_ushort(v); }

template <class Wn>
__global__ void __launch_bounds__(kA7Threads, 1) attention7_kernel(AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Wn::OFF_BAR);
  uint64_t* ld_full = bars;        // [buffer] q / k / v bytes landed
  uint64_t* prep_done = bars + 2;  // [buffer] item prepared (one arrival per preparation thread)
  uint64_t* buf_free = bars + 4;   // [buffer] item finished (MMA commit + 4 warps per tile)
  uint64_t* s_full = bars + 6;     // [group] scores of the group's next block in TMEM
  uint64_t* o_full = bars + 10;    // [group] O of the group's tile complete
  uint64_t* prep_sync = bars + 14; // preparation warps' own barrier
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 15);
  float* s_red = reinterpret_cast<float*>(smem + Wn::OFF_BAR + 192);  // [buffer][8]
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geom& g = a.g;
  const long long nitems = a.nwin * g.heads;
  const long long nmine =
      nitems > (long long)blockIdx.x ? (nitems - (long long)blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const long long ntiles = nmine * Wn::QTILES;
  const uint64_t lim = a.ctx.wait_limit;
  const int cut_t = Wn::P - g.sh[0], cut_h = 7 - g.sh[1], cut_w = 7 - g.sh[2];

  if (tid == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(&ld_full[k], 1);
      mbar_init(&prep_done[k], kA7PrepWarps * 32);
      mbar_init(&buf_free[k], 5 * Wn::QTILES);
    }
    for (int k = 0; k < kA7Groups; ++k) {
      mbar_init(&s_full[k], 1);
      mbar_init(&o_full[k], 1);
    }
    mbar_init(prep_sync, kA7PrepWarps * 32);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, kA7TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp < kA7PrepWarps) {
    // ------------------------------------------------------------ preparation
    setmaxnreg_dec<kA7RegsPrep>();
    const int pt_ = tid;
    int tab_head0 = -1, tab_head1 = -1;
    float tab_max0 = 0.f, tab_max1 = 0.f;
    uint32_t ph_sync = 0;
    int trace_n = 0;
    (void)trace_n;
    long long j = 0;
    for (long long item = blockIdx.x; item < nitems; item += gridDim.x, ++j) {
      const int X = w7_buf<Wn>(j);
      const uint32_t use = (uint32_t)w7_use<Wn>(j);  // earlier items in buffer X
      if (j >= Wn::NBUF && !mbar_wait(&buf_free[X], (use - 1) & 1, a.ctx.err, kErrWaitMma, lim)) s_abort = 1;
      if (s_abort) break;
      if (pt_ == 0) VSWIN_TRACE_EVENT(0, trace_n, 1);
      const int h = (int)(item / a.nwin);
      const long long wl = item % a.nwin;
      uint8_t* sQ = smem + Wn::OFF_Q + X * Wn::QB;
      uint8_t* sK = smem + Wn::OFF_K + X * Wn::KB;
      uint8_t* sV = smem + Wn::OFF_V + X * Wn::KB;
      uint8_t* sQX = smem + Wn::OFF_QX + X * Wn::QXB;
      uint8_t* sKX = smem + Wn::OFF_KX + X * Wn::KXB;
      float* sT = reinterpret_cast<float*>(smem + Wn::OFF_T + X * Wn::TB);
      float* red = s_red + X * 8;
      if (pt_ == 0) {
        const __nv_bfloat16* base = a.qkv + ((size_t)wl * g.heads + h) * a.slab.head_elems();
        mbar_arrive_expect_tx(&ld_full[X], (uint32_t)(Wn::QB + 2 * Wn::KB));
        bulk_g2s(sQ, base, Wn::QB, &ld_full[X]);
        bulk_g2s(sK, base + (size_t)Wn::QSLAB * kD, Wn::KB, &ld_full[X]);
        bulk_g2s(sV, base + (size_t)(Wn::QSLAB + Wn::KCOLS) * kD, Wn::KB, &ld_full[X]);
      }
      const bool new_table = h != (X ? tab_head1 : tab_head0);
      if (new_table) {
        float mx = -INFINITY;
        for (int k = pt_; k < Wn::TABLE; k += kA7PrepWarps * 32) {
          const float v = __bfloat162float(a.table[(size_t)k * g.heads + h]) * kLog2e;
          sT[k] = v;
          mx = fmaxf(mx, v);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[warp] = mx;  // red[0 .. kA7PrepWarps)
      }
      const int split = window_split_bits(g, (int)((a.win0 + wl) % g.nW));
      // key extension rows (independent of the loaded data)
      for (int n = pt_; n < Wn::KCOLS; n += kA7PrepWarps * 32) {
        const int l = n >> 3, pw = n & 7;
        int rt = 0, rh = 0, rw = 0;
        if (l < Wn::KLINES && pw < 7) {
          rt = w7_region(split & 1, l / 7, cut_t);
          rh = w7_region(split & 2, l % 7, cut_h);
          rw = w7_region(split & 4, pw, cut_w);
        }
        const float yt = (split & 1) ? -256.f * (float)(1 - 2 * rt) : 0.f;
        const float yh = (split & 2) ? -256.f * (float)(1 - 2 * rh) : 0.f;
        const float yw = (split & 4) ? -256.f * (float)(1 - 2 * rw) : 0.f;
        const float z = -256.f * (float)(rt + rh + rw);
        *reinterpret_cast<uint4*>(sKX + (n >> 3) * 128 + (n & 7) * 16) =
            make_uint4(pack_bf16x2(1.f, z), pack_bf16x2(yt, yh), pack_bf16x2(yw, 0.f), 0u);
      }
      if (!mbar_wait(&ld_full[X], use & 1, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
      if (s_abort) break;
      if (pt_ == 0) VSWIN_TRACE_EVENT(0, trace_n, 2);
      // key norms
      {
        float kx = 0.f;
        for (int n = pt_; n < Wn::KLINES * 8; n += kA7PrepWarps * 32) {
          if ((n & 7) == 7) continue;
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(sK + (n >> 3) * 512 + c * 128 + (n & 7) * 16);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = __bfloat1622float2(h2[k]);
              acc = fmaf(f.x, f.x, fmaf(f.y, f.y, acc));
            }
          }
          kx = fmaxf(kx, acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kx = fmaxf(kx, __shfl_xor_sync(0xffffffffu, kx, off));
        if (lane == 0) red[4 + warp] = kx;  // red[4 .. 4 + kA7PrepWarps)
      }
      mbar_arrive(prep_sync);
      if (!mbar_wait(prep_sync, ph_sync, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
      ph_sync ^= 1;
      if (s_abort) break;
      if (new_table) {
        float mx = red[0];
#pragma unroll
        for (int k = 1; k < kA7PrepWarps; ++k) mx = fmaxf(mx, red[k]);
        if (X) {
          tab_max1 = mx;
          tab_head1 = h;
        } else {
          tab_max0 = mx;
          tab_head0 = h;
        }
      }
      float kx2 = red[4];
#pragma unroll
      for (int k = 1; k < kA7PrepWarps; ++k) kx2 = fmaxf(kx2, red[4 + k]);
      const float kmax = sqrtf(kx2);
      const float bmax = X ? tab_max1 : tab_max0;
      // query extension rows
      for (int i = pt_; i < Wn::QXROWS; i += kA7PrepWarps * 32) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (i < Wn::N) {
          float qq = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 qv = *reinterpret_cast<const uint4*>(sQ + (i >> 3) * 512 + c * 128 + (i & 7) * 16);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&qv);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = __bfloat1622float2(h2[k]);
              qq = fmaf(f.x, f.x, fmaf(f.y, f.y, qq));
            }
          }
          float m = sqrtf(qq) * kmax + bmax + 1.0f;
          if (!(m < 3.0e38f)) m = 0.f;  // the row sum then fails the range test: exact path
          const int pt = i / 49, ph = (i / 7) % 7, pw = i % 7;
          const float rt = 0.5f * (float)w7_region(split & 1, pt, cut_t);
          const float rh = 0.5f * (float)w7_region(split & 2, ph, cut_h);
          const float rw = 0.5f * (float)w7_region(split & 4, pw, cut_w);
          w.x = bf16_bits(__float2bfloat16_rd(-0.5f * m)) | (bf16_bits(__float2bfloat16(0.5f)) << 16);
          w.y = pack_bf16x2(rt, rh);
          w.z = pack_bf16x2(rw, 0.f);
        }
        *reinterpret_cast<uint4*>(sQX + (i >> 3) * 128 + (i & 7) * 16) = w;
      }
      // Padding rows of the v slab (8th key of each line, whole padding lines)
      // must be finite for O = P V: zero them (four 16-byte pieces per row).
      {
        constexpr int ndummy = Wn::KLINES + (Wn::LINES - Wn::KLINES) * 8;
        for (int k = pt_; k < ndummy * 4; k += kA7PrepWarps * 32) {
          const int d = k >> 2, chunk = k & 3;
          const int n = d < Wn::KLINES ? d * 8 + 7 : Wn::KLINES * 8 + (d - Wn::KLINES);
          *reinterpret_cast<uint4*>(sV + (n >> 3) * 512 + chunk * 128 + (n & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      if (pt_ == 0) VSWIN_TRACE_EVENT(0, trace_n, 3);
      mbar_arrive(&prep_done[X]);
    }
  } else {
    // ------------------------------------------------------------ softmax groups
    setmaxnreg_inc<kA7RegsSoft>();
    const int grp = (warp - kA7Soft0) >> 2;
    const int qd = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t tG = tmem + (uint32_t)grp * kA7GroupCols;  // the group's columns, lane 0
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;       // this warp's TMEM lanes
    const uint32_t tS = tG + lane_off;
    const uint32_t tQ = tmem + kA7QBase + 16u * (uint32_t)grp;    // the group's q columns, lane 0
    const uint32_t tQX = tmem + kA7QXBase + 8u * (uint32_t)grp;
    const uint32_t s_base = smem_u32(smem);
    uint32_t ph_s = 0, ph_o = 0;
    int turn = 0;  // block counter: the block's issuer warp is the one with qd == turn & 3
    int trace_n = 0;
    (void)trace_n;
    const int trace_role = 1 + warp - kA7Soft0;
    (void)trace_role;
    // Scores of block b of tile t (elected lane). Item buffer X adds
    // X * (buffer bytes) / 16 to a descriptor; q row r is 16 B of extension
    // (r units) and 64 B of q (4 r units); key line l is 128 B / 512 B.
    auto issue_s = [&](long long t, int b) {
      const uint32_t X = (uint32_t)w7_buf<Wn>(t / Wn::QTILES);
      const uint32_t l0 = (uint32_t)(b * Wn::BL);
      const uint64_t bx = smem_desc(s_base + Wn::OFF_KX + X * Wn::KXB + l0 * 128, 0, 128);
      const uint64_t bk = smem_desc(s_base + Wn::OFF_K + X * Wn::KB + l0 * 512, 128, 512);
      if (b == Wn::NBLK - 1)
        w7_issue_s<Wn::LAST>(tG, tQ, tQX, bx, bk);
      else
        w7_issue_s<Wn::BL>(tG, tQ, tQX, bx, bk);
      umma_commit(&s_full[grp]);
    };
    // q rows and extension rows of tile t (this thread's TMEM lane) into the
    // group's q columns, once its item is prepared; the extension row fills
    // both halves of its K step. Every thread of the group stages its lane.
    auto stage_q = [&](long long t) {
      const long long jj = t / Wn::QTILES;
      const int X = w7_buf<Wn>(jj);
      if (!s_abort && !mbar_wait(&prep_done[X], (uint32_t)w7_use<Wn>(jj) & 1, a.ctx.err, kErrWaitLoad, lim))
        s_abort = 1;
      const int r = w7_tile_row0<Wn>((int)(t % Wn::QTILES), jj) + qd * 32 + lane;  // < QXROWS
      const uint8_t* sQ = smem + Wn::OFF_Q + X * Wn::QB;  // rows past the slab read the next buffer
      const uint8_t* sQX = smem + Wn::OFF_QX + X * Wn::QXB;
      uint32_t qv[16], xv[8];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(sQ + (r >> 3) * 512 + c * 128 + (r & 7) * 16);
        qv[4 * c + 0] = w.x;
        qv[4 * c + 1] = w.y;
        qv[4 * c + 2] = w.z;
        qv[4 * c + 3] = w.w;
      }
      const uint4 x = *reinterpret_cast<const uint4*>(sQX + (r >> 3) * 128 + (r & 7) * 16);
      xv[0] = xv[4] = x.x;
      xv[1] = xv[5] = x.y;
      xv[2] = xv[6] = x.z;
      xv[3] = xv[7] = x.w;
      tmem_st16(tQ + lane_off, qv);
      tmem_st8(tQX + lane_off, xv);
    };
    // stage tile t's q with the whole group, then one warp issues its first scores
    auto start_tile = [&](long long t) {
      stage_q(t);
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(1 + grp, 128);
      if (qd == 0) {
        tc_fence_after();
        if (!s_abort && elect_one()) issue_s(t, 0);
        __syncwarp();
      }
    };
    // Per-row context of tile t for this thread.
    struct TileRow {
      long long wl;
      int h, X, i, pt_i, ph_i, pw_i;
      bool active, warp_active;
      const float* tb_row;
    };
    auto tile_row = [&](long long t) {
      TileRow c;
      const long long jj = t / Wn::QTILES;
      const int qt = (int)(t % Wn::QTILES);
      c.X = w7_buf<Wn>(jj);
      const long long item = (long long)blockIdx.x + jj * gridDim.x;
      c.h = (int)(item / a.nwin);
      c.wl = item % a.nwin;
      const int wrow = w7_tile_row0<Wn>(qt, jj) + qd * 32;
      c.i = wrow + lane;
      c.active = c.i >= qt * 128 && c.i < Wn::N;
      c.warp_active = wrow + 31 >= qt * 128 && wrow < Wn::N;
      const int ie = c.i < qt * 128 ? qt * 128 : (c.i < Wn::N ? c.i : Wn::N - 1);
      c.pt_i = ie / 49;
      c.ph_i = (ie / 7) % 7;
      c.pw_i = ie % 7;
      const float* sT = reinterpret_cast<const float*>(smem + Wn::OFF_T + c.X * Wn::TB);
      c.tb_row = sT + (c.pt_i + Wn::P - 1) * 169 + (c.ph_i + 6) * 13 + (c.pw_i + 6);
      return c;
    };
    // O / l of finished tile t (row sum L) to memory (or the exact
    // recomputation of a row), then this warp's share of the item's release.
    auto epilogue = [&](long long t, float L) {
      const TileRow c = tile_row(t);
      if (!s_abort && !mbar_wait(&o_full[grp], ph_o, a.ctx.err, kErrWaitMma, lim)) s_abort = 1;
      ph_o ^= 1;
      tc_fence_after();
      if (c.warp_active && !s_abort) {
        __nv_bfloat16* dst = a.o + ((size_t)c.wl * Wn::N + c.i) * g.C + c.h * kD;
        const bool common = L >= a.exact_below && L <= 3.0e38f;
        const float inv = 1.0f / L;
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {  // two halves of 16 columns
          uint32_t o[16];
          tmem_ld16(tS + kA7OCol + 16 * hv, o);
          tmem_wait_ld_keep(o);
          if (c.active && common) {
#pragma unroll
            for (int k = 0; k < 2; ++k)
              reinterpret_cast<uint4*>(dst)[2 * hv + k] = make_uint4(
                  pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv));
          }
        }
        // the reference was too loose for this row (or overflowed): recompute it exactly
        float2 ml = make_float2(0.f, L);
        if (c.active && !common) ml = w7_exact_store<Wn>(a, smem, c.X, c.wl, c.i, dst);
        if (c.active && a.stats) {
          if (common) {  // the reference the score MMA subtracted: -2 x the extension row's first value
            const uint8_t* sQX = smem + Wn::OFF_QX + c.X * Wn::QXB;
            const uint32_t xw = *reinterpret_cast<const uint32_t*>(sQX + (c.i >> 3) * 128 + (c.i & 7) * 16);
            ml.x = -2.0f * __uint_as_float(xw << 16);
          }
          a.stats[((size_t)c.wl * Wn::N + c.i) * g.heads + c.h] = ml;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        VSWIN_TRACE_EVENT(trace_role, trace_n, 44);
        mbar_arrive(&buf_free[c.X]);
      }
    };
    // A group's next tile is three tiles on. With three or more tiles per item it
    // lies at most one item ahead; with two item buffers that item's
    // preparation never waits for this tile, so the epilogue can wait for the
    // next tile's first block and that tile's first scores can be issued from
    // the last block of this one. Otherwise the next item's preparation may
    // wait for this tile's epilogue, so the epilogue comes first and then the
    // next tile starts.
    constexpr bool kDefer = Wn::NBUF == 2 && Wn::QTILES >= kA7Groups;
    long long t_prev = -1;  // tile whose epilogue is pending
    float L_prev = 0.f;
    if (grp < ntiles) start_tile(grp);
    for (long long t = grp; t < ntiles; t += kA7Groups) {
      const bool next = t + kA7Groups < ntiles;
      const long long jj = t / Wn::QTILES;
      const int X = w7_buf<Wn>(jj);
      if (!s_abort && !mbar_wait(&prep_done[X], (uint32_t)w7_use<Wn>(jj) & 1, a.ctx.err, kErrWaitLoad, lim))
        s_abort = 1;
      const float* tb_row;
      bool warp_active;
      {
        const TileRow c = tile_row(t);
        tb_row = c.tb_row;
        warp_active = c.warp_active;
      }
      const uint32_t v_base = s_base + Wn::OFF_V + X * Wn::KB;
      float L = 0.f;
#pragma unroll
      for (int b = 0; b < Wn::NBLK; ++b, ++turn) {
        const bool last = b == Wn::NBLK - 1;
        if (!s_abort && !mbar_wait(&s_full[grp], ph_s, a.ctx.err, kErrWaitMma, lim)) s_abort = 1;
        ph_s ^= 1;
        if (lane == 0) VSWIN_TRACE_EVENT(trace_role, trace_n, 40);
        tc_fence_after();
        // this tile's last scores are in, so its q columns are free: stage the
        // next tile's (issued below, after the block's P v)
        if (kDefer && last && next) stage_q(t + kA7Groups);
        if (warp_active && !s_abort) {
          if (b < Wn::NBLK - 1)
            L += w7_block<Wn, Wn::BL>(tS, b * Wn::BL, tb_row);
          else
            L += w7_block<Wn, Wn::LAST>(tS, b * Wn::BL, tb_row);
        }
        // the previous tile's O was complete long ago; it must be read before
        // this block's P v (issued after the barrier below) starts a new O
        if (kDefer && b == 0 && t_prev >= 0) {
          epilogue(t_prev, L_prev);
          t_prev = -1;
        }
        tmem_wait_st();
        tc_fence_before();
        if (lane == 0) VSWIN_TRACE_EVENT(trace_role, trace_n, 42);
        named_bar_sync(1 + grp, 128);
        if (qd == (turn & 3)) {  // this warp issues the block's MMAs
          tc_fence_after();
          if (!s_abort && elect_one()) {
            const uint64_t bv = smem_desc(v_base + (uint32_t)(b * Wn::BL) * 512, 512, 128);
            if (last)
              w7_issue_pv<Wn::LAST>(tG + kA7OCol, tG, bv, b == 0);
            else
              w7_issue_pv<Wn::BL>(tG + kA7OCol, tG, bv, b == 0);
            if (last) {
              umma_commit(&o_full[grp]);
              umma_commit(&buf_free[X]);
              if (kDefer && next) issue_s(t + kA7Groups, 0);  // its q was staged above
            } else {
              issue_s(t, b + 1);  // runs after P v, which reads these columns
            }
          }
          __syncwarp();
        }
      }
      if (kDefer) {
        t_prev = t;
        L_prev = L;
      } else {
        epilogue(t, L);
        if (next) start_tile(t + kA7Groups);
      }
    }
    if (t_prev >= 0) epilogue(t_prev, L_prev);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kA7TmemCols);
}

template <class Wn>
cudaError_t launch_attention7(const AttnArgs& a, cudaStream_t st) {
  if (a.slab.qrows != Wn::QSLAB || a.slab.kvrows != Wn::KCOLS || !a.slab.kv8) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e =
      cudaFuncSetAttribute(attention7_kernel<Wn>, cudaFuncAttributeMaxDynamicSharedMemorySize, Wn::SMEM);
  if (e != cudaSuccess) return e;
  // the warpgroups' register budgets draw on the pool the block is launched
  // with: refuse a build whose register count would leave the softmax
  // warpgroups waiting for registers
  cudaFuncAttributes fa{};
  e = cudaFuncGetAttributes(&fa, attention7_kernel<Wn>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < kA7RegsLaunch) return cudaErrorInvalidConfiguration;
  const long long items = a.nwin * a.g.heads;
  long long grid = sms;
  if (grid > items) grid = items;
  prof_begin(kKindAttn, st);
  attention7_kernel<Wn><<<(unsigned)grid, kA7Threads, Wn::SMEM, st>>>(a);
  prof_end(kKindAttn, st);
  count_launch();
  return cudaGetLastError();
}

int pick_bn(int n) {
  if (n <= kMaxBN && n % 16 == 0) return n;
  for (int bn = kMaxBN; bn >= 16; bn -= 16)
    if (n % bn == 0) return bn;
  return 0;
}

// The persistent GEMM runs when its weight slice and two A stages fit in shared
// memory (227 KB per CTA, 1 KB of it static); otherwise the tiled version (e.g.
// C = 544: BN = 32 for the projection, two 139 KB A stages).
bool ws_fits(const GemmArgs& a, bool ln, bool resid = false, bool stage_out = false) {
  return a.rowsrc && a.K * a.BN * 2 <= kWsMaxBBytes && a.K % 32 == 0 && (a.BN / 2) % 8 == 0 &&
         ws_smem_bytes(a.K, a.BN, 2, ln, resid, stage_out) <= 226 * 1024;
}

template <int MODE, bool FUSE>
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t st) {
  const bool resid = FUSE && MODE == kPROJ;
  const bool stage_out = MODE == kPROJ;
  if (ws_fits(a, FUSE && MODE == kQKV, resid, stage_out)) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int NT = a.Ntot / a.BN;
    const long long mtiles = (a.rows + kBM - 1) / kBM;
    long long per_nt = sms / NT;
    if (per_nt < 1) per_nt = 1;
    if (per_nt > mtiles) per_nt = mtiles;
    // four A stages when they fit, else two; at least 116 KB so that one CTA
    // (up to 512 TMEM columns) owns each SM
    const bool ln = FUSE && MODE == kQKV;
    const bool four = ws_smem_bytes(a.K, a.BN, 4, ln, resid, stage_out) <= 220 * 1024;
    int smem_ws = ws_smem_bytes(a.K, a.BN, four ? 4 : 2, ln, resid, stage_out);
    if (smem_ws < 116 * 1024) smem_ws = 116 * 1024;
    auto kern = four ? gemm_ws_kernel<MODE, 4, FUSE> : gemm_ws_kernel<MODE, 2, FUSE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_ws);
    if (e != cudaSuccess) return e;
    prof_begin(MODE == kQKV ? kKindQkv : kKindProj, st);
    kern<<<(unsigned)(per_nt * NT), kWsThreads, smem_ws, st>>>(a);
    prof_end(MODE == kQKV ? kKindQkv : kKindProj, st);
    count_launch();
    return cudaGetLastError();
  }
  cudaError_t e =
      cudaFuncSetAttribute(gemm_kernel<MODE, FUSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes());
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.rows + kBM - 1) / kBM), (unsigned)(a.Ntot / a.BN));
  prof_begin(MODE == kQKV ? kKindQkv : kKindProj, st);
  gemm_kernel<MODE, FUSE><<<grid, kGemmThreads, gemm_smem_bytes(), st>>>(a);
  prof_end(MODE == kQKV ? kKindQkv : kKindProj, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool bf16_window_supported(const Geom& g) {
  const int P = g.win[0], MH = g.win[1], MW = g.win[2];
  return (P == 16 && MH == 7 && MW == 7) || (P == 8 && MH == 7 && MW == 7) || (P == 4 && MH == 7 && MW == 7) ||
         (P == 2 && MH == 7 && MW == 7) ||
         (P == 1 && MH == 7 && MW == 7) || (P == 4 && MH == 4 && MW == 4) || (P == 2 && MH == 2 && MW == 2) ||
         (P == 1 && MH == 1 && MW == 1);
}

size_t bf16_scratch_bytes(const Geom& g, long long nwin) {
  const size_t qkv = (size_t)nwin * g.heads * slab_layout(g).head_elems() * 2;
  const size_t o = (size_t)nwin * g.N * g.C * 2;
  const size_t rows = ((size_t)nwin * g.N * 4 + 255) / 256 * 256;
  return qkv + o + rows;
}

size_t bf16_block_scratch_bytes(const Geom& g, long long nwin) {
  return bf16_scratch_bytes(g, nwin) + ((size_t)nwin * g.N * 8 + 255) / 256 * 256;
}

cudaError_t launch_ln_fold(const Geom& g, const void* gamma, const void* beta, const void* Wqkv, const void* bqkv,
                           const BlockFuse& f, cudaStream_t st) {
  const int n3 = 3 * g.C;
  prof_begin(kKindOther, st);
  ln_fold_kernel<<<(unsigned)((n3 + kFoldCols - 1) / kFoldCols), kFoldCols * kFoldRows, 0, st>>>(
      g.C, n3, static_cast<const __nv_bfloat16*>(gamma), static_cast<const __nv_bfloat16*>(beta),
      static_cast<const __nv_bfloat16*>(Wqkv), static_cast<const __nv_bfloat16*>(bqkv),
      static_cast<__nv_bfloat16*>(f.wt), f.colsum, f.bias_ln);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_bf16_chunk(const Geom& g, const KernelCtx& ctx, const void* x, const void* Wqkv,
                              const void* bqkv, const void* Wproj, const void* bproj, const void* table,
                              void* out, void* scratch, long long win0, long long nwin, cudaStream_t st,
                              const BlockFuse* fuse, float2* attn_stats) {
  __nv_bfloat16* qkv = static_cast<__nv_bfloat16*>(scratch);
  const SlabLayout L = slab_layout(g);
  __nv_bfloat16* o = qkv + (size_t)nwin * g.heads * L.head_elems();
  int* rowsrc = reinterpret_cast<int*>(o + (size_t)nwin * g.N * g.C);
  // fused block: per-row norm statistics after the row table
  float2* stats = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(rowsrc) +
                                            ((size_t)nwin * g.N * 4 + 255) / 256 * 256);

  // fused block: the persistent QKV GEMM computes the norm statistics from the
  // rows it gathers; the tiled one reads them from row_stats_kernel
  bool stats_in_gemm = false;
  if (fuse) {
    GemmArgs probe{};
    probe.rowsrc = rowsrc;
    probe.K = g.C;
    probe.BN = pick_bn(3 * g.C);
    stats_in_gemm = probe.BN != 0 && ws_fits(probe, true);
  }
  {
    const long long rows = nwin * g.N;
    prof_begin(kKindOther, st);
    if (fuse && !stats_in_gemm) {
      // one warp per 32 rows, eight warps per block
      long long blocks = (rows + 255) / 256;
      if (blocks > 4096) blocks = 4096;
      const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
      switch (g.C / 32) {
        case 1: row_stats_kernel<1><<<(unsigned)blocks, 256, 0, st>>>(g, win0, rows, xb, fuse->eps, rowsrc, stats, ctx.err); break;
        case 2: row_stats_kernel<2><<<(unsigned)blocks, 256, 0, st>>>(g, win0, rows, xb, fuse->eps, rowsrc, stats, ctx.err); break;
        case 3: row_stats_kernel<3><<<(unsigned)blocks, 256, 0, st>>>(g, win0, rows, xb, fuse->eps, rowsrc, stats, ctx.err); break;
        case 4: row_stats_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(g, win0, rows, xb, fuse->eps, rowsrc, stats, ctx.err); break;
        default: row_stats_kernel<0><<<(unsigned)blocks, 256, 0, st>>>(g, win0, rows, xb, fuse->eps, rowsrc, stats, ctx.err);
      }
    } else {
      long long blocks = (rows + 255) / 256;
      if (blocks > 2048) blocks = 2048;
      row_source_kernel<<<(unsigned)blocks, 256, 0, st>>>(g, win0, rows, rowsrc, ctx.err);
    }
    prof_end(kKindOther, st);
    count_launch();
#ifdef VSWIN_DEBUG_BOUNDS
    long long plant_slot = -1;
    int plant_token = 0;
    debug_plant(&plant_slot, &plant_token);
    if (plant_slot >= win0 * g.N && plant_slot < win0 * g.N + rows) {
      plant_row_kernel<<<1, 1, 0, st>>>(rowsrc, plant_slot - win0 * g.N, plant_token);
      count_launch();
    }
#endif
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
  }

  GemmArgs ga{};
  ga.g = g;
  ga.ctx = ctx;
  ga.A = static_cast<const __nv_bfloat16*>(x);
  ga.Wt = static_cast<const __nv_bfloat16*>(Wqkv);
  ga.bias = static_cast<const __nv_bfloat16*>(bqkv);
  ga.dst = qkv;
  ga.win0 = win0;
  ga.rows = nwin * g.N;
  ga.K = g.C;
  ga.Ntot = 3 * g.C;
  ga.BN = pick_bn(3 * g.C);
  ga.qscale = kLog2e / sqrtf((float)kD);
  ga.slab = L;
  ga.rowsrc = rowsrc;
  if (fuse) {
    ga.Wt = static_cast<const __nv_bfloat16*>(fuse->wt);
    ga.ln_stats = stats;
    ga.ln_eps = fuse->eps;
    ga.ln_colsum = fuse->colsum;
    ga.ln_bias = fuse->bias_ln;
  }
  cudaError_t e = fuse ? launch_gemm<kQKV, true>(ga, st) : launch_gemm<kQKV, false>(ga, st);
  if (e != cudaSuccess) return e;

  AttnArgs aa{};
  aa.g = g;
  aa.ctx = ctx;
  aa.qkv = qkv;
  aa.table = static_cast<const __nv_bfloat16*>(table);
  aa.o = o;
  aa.win0 = win0;
  aa.nwin = nwin;
  aa.slab = L;
  aa.exact_below = ctx.force_exact ? INFINITY : 7.8886e-31f;  // 2^-100
  aa.stats = attn_stats;
  const int P = g.win[0], MH = g.win[1], MW = g.win[2];
  if (attn_stats && !window_is_p77(g)) return cudaErrorInvalidValue;  // only the (P,7,7) kernel writes them
  if (P == 16 && MH == 7 && MW == 7) e = launch_attention7<W7<16>>(aa, st);
  else if (P == 8 && MH == 7 && MW == 7) e = launch_attention7<W7<8>>(aa, st);
  else if (P == 4 && MH == 7 && MW == 7) e = launch_attention7<W7<4>>(aa, st);
  else if (P == 2 && MH == 7 && MW == 7) e = launch_attention7<W7<2>>(aa, st);
  else if (P == 1 && MH == 7 && MW == 7) e = launch_attention7<W7<1>>(aa, st);
  else if (P == 4 && MH == 4 && MW == 4) e = launch_attention<Win<4, 4, 4>>(aa, st);
  else if (P == 2 && MH == 2 && MW == 2) e = launch_attention<Win<2, 2, 2>>(aa, st);
  else if (P == 1 && MH == 1 && MW == 1) e = launch_attention<Win<1, 1, 1>>(aa, st);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  if (!Wproj) return cudaSuccess;  // the first three steps only (the backward's recomputation)

  GemmArgs gp = ga;
  gp.A = o;
  gp.Wt = static_cast<const __nv_bfloat16*>(Wproj);
  gp.bias = static_cast<const __nv_bfloat16*>(bproj);
  gp.dst = static_cast<__nv_bfloat16*>(out);
  gp.Ntot = g.C;
  gp.BN = pick_bn(g.C);
  gp.qscale = 1.0f;
  if (fuse) {
    gp.resid = static_cast<const __nv_bfloat16*>(x);
    return launch_gemm<kPROJ, true>(gp, st);
  }
  return launch_gemm<kPROJ, false>(gp, st);
}

void bf16_slab_rows(const Geom& g, int* qrows, int* kvrows, int* kv8) {
  const SlabLayout L = slab_layout(g);
  *qrows = L.qrows;
  *kvrows = L.kvrows;
  *kv8 = L.kv8;
}

size_t bf16_chunk_o_offset(const Geom& g, long long nwin) {
  return (size_t)nwin * g.heads * slab_layout(g).head_elems() * 2;
}

size_t bf16_chunk_rows_offset(const Geom& g, long long nwin) {
  return bf16_chunk_o_offset(g, nwin) + (size_t)nwin * g.N * g.C * 2;
}

cudaError_t launch_bf16_dout_slabs(const Geom& g, const KernelCtx& ctx, const void* dy, const void* WprojT,
                                   const void* zero_bias, void* dO, const int* rowsrc, long long win0,
                                   long long nwin, cudaStream_t st) {
  GemmArgs ga{};
  ga.g = g;
  ga.ctx = ctx;
  ga.A = static_cast<const __nv_bfloat16*>(dy);
  ga.Wt = static_cast<const __nv_bfloat16*>(WprojT);
  ga.bias = static_cast<const __nv_bfloat16*>(zero_bias);
  ga.dst = static_cast<__nv_bfloat16*>(dO);
  ga.win0 = win0;
  ga.rows = nwin * g.N;
  ga.K = g.C;
  ga.Ntot = g.C;
  ga.BN = pick_bn(g.C);
  ga.qscale = 1.0f;
  ga.slab.qrows = g.Npad;  // one q-layout slab per (window, head)
  ga.slab.kvrows = 0;
  ga.slab.kv8 = 0;
  ga.rowsrc = rowsrc;
  if (ga.BN == 0) return cudaErrorInvalidValue;
  return launch_gemm<kQKV, false>(ga, st);
}

cudaError_t launch_bf16_dx(const Geom& g, const KernelCtx& ctx, const void* dqkv, const void* WqkvT,
                           const void* zero_bias, void* dx, const int* rowsrc, long long win0, long long nwin,
                           cudaStream_t st) {
  GemmArgs gp{};
  gp.g = g;
  gp.ctx = ctx;
  gp.A = static_cast<const __nv_bfloat16*>(dqkv);
  gp.lda = 3LL * g.C;
  gp.Wt = static_cast<const __nv_bfloat16*>(WqkvT);
  gp.bias = static_cast<const __nv_bfloat16*>(zero_bias);
  gp.dst = static_cast<__nv_bfloat16*>(dx);
  gp.win0 = win0;
  gp.rows = nwin * g.N;
  gp.K = 3 * g.C;
  gp.Ntot = g.C;
  gp.BN = pick_bn(g.C);
  gp.qscale = 1.0f;
  gp.slab = slab_layout(g);
  gp.rowsrc = rowsrc;
  if (gp.BN == 0) return cudaErrorInvalidValue;
  return launch_gemm<kPROJ, false>(gp, st);
}

}  // namespace vswin

#ifdef VSWIN_TRACE
// Copies the trace (roles x capacity x (tag, clock)) to `host` and clears it.
extern "C" int vswin_trace_read(long long* host) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(host, vswin::g_trace, sizeof(vswin::g_trace)) != cudaSuccess) return -1;
  static long long zero[vswin::kTraceRoles][vswin::kTraceCap][2];
  return cudaMemcpyToSymbol(vswin::g_trace, zero, sizeof(zero)) == cudaSuccess ? 0 : -1;
}
#endif
