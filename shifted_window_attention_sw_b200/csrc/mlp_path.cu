// The MLP half of a Video Swin block on sm_100a tensor cores, fused into one
// persistent kernel ("Video Swin Transformer" summary page, Method step 3 and
// eq. 1: layer norm, a two-layer MLP with GELU, residual add):
//
//   out = x + GELU(LN(x) W1 + b1) W2 + b2        per token (row of x)
//
// One CTA per SM walks 128-token tiles. Per tile the tokens are read from HBM
// once (TMA) and the result is written once (TMA store); the hidden
// activations (128 x hidden) never leave the SM:
//   * warp 0 loads x tiles (three in flight) and the weight chunks (W1
//     columns and W2 rows of one hidden chunk of HC = 128 or 64 columns) with
//     TMA -- when every chunk fits in shared memory at once they are loaded
//     once per CTA -- and stores each finished output tile with TMA;
//   * warp 1 issues, per hidden chunk, fc1 = LN(x) W1[:, chunk] into one of
//     two TMEM accumulators, and the last warp fc2 += h_chunk W2[chunk, :]
//     with h read from TMEM (the A operand of a TS MMA) into one of two output
//     accumulators -- two issuing threads on different SM sub-partitions;
//   * warps 2-5 normalise each tile in place as soon as it lands (fp32
//     statistics, bf16 result in the MMA operand layout) and write each
//     tile's output: output accumulator + b2 + x (re-read from global memory,
//     L1-prefetched before the wait), bf16, staged over the tile's buffer;
//   * the GELU warps (four per TMEM lane quarter) turn each fc1 accumulator
//     into h = GELU(acc + b1) (bf16, written over the accumulator's own
//     columns).
//
// GELU: the erf form x * Phi(x) (torch.nn.GELU's default) evaluated as
// 0.5 x (1 + tanh(x (g1 + g3 x^2 + g5 x^4))) with x^2 clamped at 64, whose
// coefficients are a least-squares fit of Phi(x) = (1 + erf(x / sqrt(2))) / 2
// over [-8, 8] (max abs error of the formula 3.3e-5); tanh is the hardware
// tanh.approx.f32 (max relative error about 2^-11), so the GELU value carries
// an absolute error below 1e-3 * |x|, under the bf16 rounding of h.
//
// Operand layouts in shared memory. A tile of x (128 rows x C) is K-major
// with the 64-byte swizzle: blocks of 32 channels, 64-byte rows, the 16-byte
// chunk index XORed with bits 1-2 of the row (one 3D TMA box of (32
// channels, 128 rows, C/32 blocks) with CU_TENSOR_MAP_SWIZZLE_64B writes it;
// the MMA descriptor uses layout type SWIZZLE_64B, SBO = 512 B). Weight
// chunks are MN-major in the no-swizzle canonical layout (8 x 16-byte core
// matrices): element (k, n) at (k/8)*LBO + (n/8)*128 + (k%8)*16 + (n%8)*2,
// one 4D TMA box each.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vswin {
namespace {

constexpr int kMlpMaxHC = 128;       // hidden columns per chunk: 128, or 64 when two 128-column stages do not fit
#ifndef VSWIN_MLP_GELU_PER_QUARTER
#define VSWIN_MLP_GELU_PER_QUARTER 4
#endif
constexpr int kMlpGeluPerQ = VSWIN_MLP_GELU_PER_QUARTER;  // GELU warps per TMEM lane quarter
constexpr int kMlpGeluWarps = 4 * kMlpGeluPerQ;  // each takes 1 / kMlpGeluPerQ of a chunk's columns
constexpr int kMlpFc2Warp = 6 + kMlpGeluWarps;  // issues fc2 (warp 1 issues fc1)
// producer, fc1 issue, 4 norm / output warps, GELU warps, fc2 issue
constexpr int kMlpThreads = (kMlpFc2Warp + 1) * 32;
constexpr int kMlpNorm0 = 2;          // first norm / output warp
constexpr int kMlpGelu0 = 6;          // first GELU warp
constexpr int kMlpXBufs = 3;          // x tiles in flight
constexpr int kMlpMaxC = 128;

// GELU via tanh: coefficients of x (g1 + g3 x^2 + g5 x^4), least-squares fit
// of Phi on [-8, 8] (see the file comment).
constexpr float kG1 = 0.797458471f, kG3 = 0.0370503451f, kG5 = -0.000358732362f;

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU of two values (packed fp32 arithmetic where the ISA has it).
__device__ __forceinline__ float2 gelu2(float2 v) {
  const float2 x2 = __fmul2_rn(v, v);
  const float2 s = make_float2(fminf(x2.x, 64.f), fminf(x2.y, 64.f));
  float2 p = __ffma2_rn(s, make_float2(kG5, kG5), make_float2(kG3, kG3));
  p = __ffma2_rn(s, p, make_float2(kG1, kG1));
  const float2 arg = __fmul2_rn(v, p);
  const float2 t = make_float2(tanh_approx(arg.x), tanh_approx(arg.y));
  const float2 hx = __fmul2_rn(v, make_float2(0.5f, 0.5f));
  return __ffma2_rn(hx, t, hx);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

struct MlpArgs {
  long long M;  // tokens (rows)
  int C, hidden, hc, nch, stages;
  bool resident;  // every weight chunk has its own stage (loaded once per CTA)
  float eps;
  const __nv_bfloat16* x;  // the residual is read back from here
  const __nv_bfloat16* gamma;
  const __nv_bfloat16* beta;
  const __nv_bfloat16* b1;
  const __nv_bfloat16* b2;
  KernelCtx ctx;
};

// Shared-memory plan (bytes from the dynamically allocated base).
struct MlpSmem {
  int x, w, wstage, w2off, gam, bet, b1, b2, bars, total;
};
__host__ __device__ inline MlpSmem mlp_smem(int C, int hidden, int hc, int stages) {
  MlpSmem s;
  const int xb = 128 * C * 2;
  s.x = 0;  // kMlpXBufs tiles
  s.w = kMlpXBufs * xb;
  s.w2off = C * hc * 2;  // W2 chunk after the W1 chunk inside a stage
  s.wstage = 2 * C * hc * 2;
  s.gam = s.w + stages * s.wstage;
  s.bet = s.gam + C * 4;
  s.b1 = s.bet + C * 4;
  s.b2 = s.b1 + hidden * 4;
  s.bars = (s.b2 + C * 4 + 15) / 16 * 16;
  s.total = s.bars + 48 * 8 + 16;
  return s;
}

// Byte offset of 16-byte chunk `k` (channels 8k .. 8k+7) of row r in a tile
// stored K-major with the 64-byte swizzle: blocks of 32 channels (8 KB each:
// 128 rows x 64 B), and inside a row the chunk index XORed with bits 1-2 of
// the row -- what a TMA box with CU_TENSOR_MAP_SWIZZLE_64B writes and what a
// tcgen05 descriptor of layout type SWIZZLE_64B (SBO = 512 B) reads.
__device__ __forceinline__ int sw64_chunk(int r, int k) {
  return (k >> 2) * 8192 + r * 64 + (((k & 3) ^ ((r >> 1) & 3)) << 4);
}

// K-major, 64-byte swizzle descriptor: LBO 16 B (unused inside one swizzle
// atom), SBO 512 B (8 rows x 64 B), layout type 4.
__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(512 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)4 << 61;
  return d;
}

__global__ void __launch_bounds__(kMlpThreads, 1)
    mlp_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_out,
               const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_w2, MlpArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int C = a.C, NCH = a.nch, S = a.stages, HC = a.hc;
  const MlpSmem L = mlp_smem(C, a.hidden, HC, S);
  const int xbytes_tile = 128 * C * 2;
  auto sX = [&](int b) { return smem + L.x + b * xbytes_tile; };
  float* sGam = reinterpret_cast<float*>(smem + L.gam);
  float* sBet = reinterpret_cast<float*>(smem + L.bet);
  float* sB1 = reinterpret_cast<float*>(smem + L.b1);
  float* sB2 = reinterpret_cast<float*>(smem + L.b2);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* x_full = bars;          // [3] x tile landed
  uint64_t* xn_full = bars + 3;     // [3] tile normalised in place (4 norm warps)
  uint64_t* xn_free = bars + 6;     // [3] the tile's fc1 MMAs have read it
  uint64_t* out_full = bars + 9;    // [3] output staged over the tile (4 output warps)
  uint64_t* acc1_full = bars + 12;  // [2]
  uint64_t* h_full = bars + 14;     // [2] h written over the fc1 accumulator (every GELU warp)
  uint64_t* acc2_full = bars + 16;  // [2]
  uint64_t* acc2_free = bars + 18;  // [2] (4 output warps)
  uint64_t* w_full = bars + 20;     // [S <= 8]
  uint64_t* w_free = bars + 28;     // [S <= 8]
  uint64_t* fc2_done = bars + 36;   // [2] fc2 of the chunk in fc1 accumulator k has read h
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 38);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long mtiles = (a.M + 127) / 128;
  const long long ntiles = mtiles > blockIdx.x ? (mtiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const uint64_t lim = a.ctx.wait_limit;
  const uint32_t xbytes = 128u * (uint32_t)C * 2u;
  const uint32_t wbytes = (uint32_t)(2 * C * HC * 2);

  if (tid == 0) {
    for (int k = 0; k < kMlpXBufs; ++k) {
      mbar_init(&x_full[k], 1);
      mbar_init(&xn_full[k], 4);
      mbar_init(&xn_free[k], 1);
      mbar_init(&out_full[k], 4);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&acc1_full[k], 1);
      mbar_init(&h_full[k], kMlpGeluWarps);
      mbar_init(&acc2_full[k], 1);
      mbar_init(&acc2_free[k], 4);
      mbar_init(&fc2_done[k], 1);
    }
    for (int k = 0; k < S; ++k) {
      mbar_init(&w_full[k], 1);
      mbar_init(&w_free[k], 1);
    }
    fence_mbar_init();
    s_abort = 0;
  }
  for (int c = tid; c < C; c += kMlpThreads) {
    sGam[c] = __bfloat162float(a.gamma[c]);
    sBet[c] = __bfloat162float(a.beta[c]);
    sB2[c] = __bfloat162float(a.b2[c]);
  }
  for (int c = tid; c < a.hidden; c += kMlpThreads) sB1[c] = __bfloat162float(a.b1[c]);
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // TMEM columns: fc1 accumulators [0, HC) and [HC, 2 HC) (2 HC <= 256); output
  // accumulators [256, 256 + C) and [256 + C, 256 + 2C).
  const uint32_t tAcc1 = tmem, tAcc2 = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Per tile t: store the output of tile t - 3 from buffer t % 3 (once it
    // has been staged there), then load x of tile t into that buffer and the
    // weight chunks tile t needs.
    if (lane == 0) {
      long long g = 0;  // global chunk counter
      for (long long t = 0; t < ntiles + kMlpXBufs && !s_abort; ++t) {
        const int xb = (int)(t % kMlpXBufs);
        if (t >= kMlpXBufs) {
          const long long ts = t - kMlpXBufs;
          if (!mbar_wait(&out_full[xb], (uint32_t)(ts / kMlpXBufs) & 1, a.ctx.err, kErrWaitMma, lim)) {
            s_abort = 1;
            break;
          }
          tma_store_3d(&tm_out, sX(xb), 0, (int)((blockIdx.x + ts * gridDim.x) * 128), 0);
          bulk_commit();
          bulk_wait_read0();  // the buffer may be overwritten once the store has read it
        }
        if (t >= ntiles) continue;
        mbar_arrive_expect_tx(&x_full[xb], xbytes);
        tma_load_3d(sX(xb), &tm_x, 0, (int)((blockIdx.x + t * gridDim.x) * 128), 0, &x_full[xb]);
        for (int c = 0; c < NCH; ++c, ++g) {
          if (a.resident && t > 0) continue;
          const int s = (int)(g % S);
          if (g >= S && !mbar_wait(&w_free[s], (uint32_t)((g / S) - 1) & 1, a.ctx.err, kErrWaitMma, lim)) {
            s_abort = 1;
            break;
          }
          uint8_t* dst = smem + L.w + s * L.wstage;
          mbar_arrive_expect_tx(&w_full[s], wbytes);
          tma_load_4d(dst, &tm_w1, 0, 0, c * (HC / 8), 0, &w_full[s]);
          tma_load_4d(dst + L.w2off, &tm_w2, 0, 0, 0, c * (HC / 8), &w_full[s]);
        }
      }
      bulk_wait0();  // every store has completed before the CTA ends
    }
    __syncwarp();
  } else if (warp == 1 || warp == kMlpFc2Warp) {
    // ------------------------------------------------------------ MMA issue
    // Two issuing threads on different SM sub-partitions, so that each chunk's
    // 6 + 8 MMAs are issued side by side (a thread's issue slows sharply when
    // its sub-partition's other warps keep the issue slots busy): warp 1
    // issues fc1 = LN(x) W1[:, chunk] into an fc1 accumulator, the fc2 warp
    // fc2 += h W2[chunk, :] once the GELU warps have written h. fc1 of chunk
    // g + 2 reuses the accumulator of chunk g only after chunk g's fc2 has
    // completed (fc2_done).
    if (lane == 0) {
      const uint32_t id1 = idesc_bf16(128, HC, 0, 1);  // A K-major (x), B MN-major (W1)
      const uint32_t id2 = idesc_bf16(128, C, 0, 1);   // A from TMEM (h), B MN-major (W2)
      const uint32_t lbo1 = (uint32_t)(HC / 8) * 128u; // W1 chunk: K-group stride
      const uint32_t lbo2 = (uint32_t)(C / 8) * 128u;  // W2 chunk: K-group stride
      const long long total = ntiles * NCH;
      // chunk g = t * NCH + c; its weight stage and the parity of that stage's
      // use count, all kept incrementally (a 64-bit division by a runtime
      // count costs hundreds of cycles of this thread's issue time): resident
      // weights, stage c and phase 0; streamed, a ring of S stages
      long long t = 0;
      int c = 0, ws = 0;
      uint32_t wph = 0;
      auto advance = [&]() {
        if (++c == NCH) {
          c = 0;
          ++t;
        }
        if (!a.resident && ++ws == S) {
          ws = 0;
          wph ^= 1u;
        }
      };
      if (warp == 1) {
        for (long long g = 0; g < total && !s_abort; ++g, advance()) {
          const int xb = (int)(t % kMlpXBufs);
          // the accumulator's previous chunk (g - 2) has been read by its fc2
          if (g >= 2 && !mbar_wait(&fc2_done[g & 1], (uint32_t)((g - 2) >> 1) & 1, a.ctx.err, kErrWaitMma, lim))
            s_abort = 1;
          // the tile's normalised x (first chunk of a tile) and the weight stage
          if (c == 0 && !s_abort &&
              !mbar_wait(&xn_full[xb], (uint32_t)(t / kMlpXBufs) & 1, a.ctx.err, kErrWaitLoad, lim))
            s_abort = 1;
          const int s = a.resident ? c : ws;
          if (!s_abort && !mbar_wait(&w_full[s], a.resident ? 0u : wph, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
          tc_fence_after();
          if (s_abort) break;
          const uint32_t xa = smem_u32(sX(xb));
          const uint32_t wa = smem_u32(smem + L.w + s * L.wstage);
          const uint32_t d = tAcc1 + (uint32_t)(g & 1) * (uint32_t)HC;
          // K step ks covers channels [16 ks, 16 ks + 16): block ks / 2, 32 B in
          for (int ks = 0; ks < C / 16; ++ks)
            umma_ss(d, smem_desc_sw64(xa + (ks >> 1) * 8192 + (ks & 1) * 32),
                    smem_desc(wa + ks * 2 * lbo1, lbo1, 128), id1, ks > 0);
          umma_commit(&acc1_full[g & 1]);
          if (c == NCH - 1) umma_commit(&xn_free[xb]);
        }
      } else {
        for (long long g = 0; g < total && !s_abort; ++g, advance()) {
          const int ob = (int)(t & 1);
          // h of chunk g is in TMEM (and its fc1 accumulator was read)
          if (!mbar_wait(&h_full[g & 1], (uint32_t)(g >> 1) & 1, a.ctx.err, kErrWaitMma, lim)) s_abort = 1;
          // the output accumulator of this tile was drained two tiles ago
          if (c == 0 && t >= 2 && !s_abort &&
              !mbar_wait(&acc2_free[ob], (uint32_t)((t >> 1) - 1) & 1, a.ctx.err, kErrWaitMma, lim))
            s_abort = 1;
          const int s = a.resident ? c : ws;
          if (!s_abort && !mbar_wait(&w_full[s], a.resident ? 0u : wph, a.ctx.err, kErrWaitLoad, lim)) s_abort = 1;
          tc_fence_after();
          if (s_abort) break;
          const uint32_t wa2 = smem_u32(smem + L.w + s * L.wstage + L.w2off);
          const uint32_t hb = tAcc1 + (uint32_t)(g & 1) * (uint32_t)HC;
          const uint32_t d2 = tAcc2 + (uint32_t)ob * (uint32_t)C;
          // h element k of the chunk sits at column hq * CW + (k - hq * CW) / 2,
          // hq = k / CW, CW = HC / kMlpGeluPerQ (each GELU warp packs its own
          // columns in place)
          const int CW = HC / kMlpGeluPerQ;
          for (int j = 0; j < HC / 16; ++j) {
            const int hq = (16 * j) / CW;
            const uint32_t hcol = (uint32_t)(hq * CW + (16 * j - hq * CW) / 2);
            umma_ts(d2, hb + hcol, smem_desc(wa2 + j * 2 * lbo2, lbo2, 128), id2, (c > 0 || j > 0) ? 1u : 0u);
          }
          if (!a.resident) umma_commit(&w_free[s]);
          if (c == NCH - 1) umma_commit(&acc2_full[ob]);
          umma_commit(&fc2_done[g & 1]);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ norm / output and GELU warps
    const int q = warp & 3;  // TMEM lane quarter
    const int r = q * 32 + lane;  // this thread's row of the tile
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    if (warp < kMlpGelu0) {
      // Warps 2-5: normalise each tile in place (row r of its buffer) as soon as
      // it lands, and write each tile's output: acc2 + b2 + x (x re-read from
      // global memory, loaded before the wait for the accumulator) -> bf16 over
      // the tile's buffer, which the producer then stores with TMA.
      auto normalise = [&](long long t) {
        const int xb = (int)(t % kMlpXBufs);
        if (!s_abort && !mbar_wait(&x_full[xb], (uint32_t)(t / kMlpXBufs) & 1, a.ctx.err, kErrWaitLoad, lim))
          s_abort = 1;
        if (!s_abort) {
          // three passes over the row in shared memory (sum, squared deviations,
          // normalised write-back) keep no copy of it in registers
          uint8_t* row = sX(xb);
          auto chunk = [&](int k) { return *reinterpret_cast<const uint4*>(row + sw64_chunk(r, k)); };
          float sum = 0.f;
          for (int k = 0; k < C / 8; ++k) {
            const uint4 v = chunk(k);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              sum += f.x + f.y;
            }
          }
          const float mean = sum / (float)C;
          float ss = 0.f;
          for (int k = 0; k < C / 8; ++k) {
            const uint4 v = chunk(k);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              const float d0 = f.x - mean, d1 = f.y - mean;
              ss = fmaf(d0, d0, fmaf(d1, d1, ss));
            }
          }
          const float rstd = 1.0f / sqrtf(ss / (float)C + a.eps);
          for (int k = 0; k < C / 8; ++k) {
            const uint4 v = chunk(k);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              const int ch = k * 8 + 2 * e;
              w[e] = pack2(fmaf((f.x - mean) * rstd, sGam[ch], sBet[ch]),
                           fmaf((f.y - mean) * rstd, sGam[ch + 1], sBet[ch + 1]));
            }
            *reinterpret_cast<uint4*>(row + sw64_chunk(r, k)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();  // generic writes -> tensor-core operand reads
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(&xn_full[xb]);
      };
      auto finish_tile = [&](long long t) {
        const int xb = (int)(t % kMlpXBufs), ob = (int)(t & 1);
        const long long grow = (blockIdx.x + t * gridDim.x) * 128 + r;
        const bool real = grow < a.M;
        const __nv_bfloat16* xrow = a.x + (real ? grow : 0) * C;
        // the residual row is brought into L1 while this warp waits for the accumulator
        for (int k = 0; k < C / 8; k += 4)
          asm volatile("prefetch.global.L1 [%0];" ::"l"(xrow + 8 * k));
        if (!s_abort && !mbar_wait(&acc2_full[ob], (uint32_t)(t >> 1) & 1, a.ctx.err, kErrWaitMma, lim))
          s_abort = 1;
        if (!s_abort &&
            !mbar_wait(&xn_free[xb], (uint32_t)(t / kMlpXBufs) & 1, a.ctx.err, kErrWaitMma, lim))
          s_abort = 1;
        tc_fence_after();
        if (!s_abort) {
          const uint32_t ta = tAcc2 + lane_base + (uint32_t)ob * (uint32_t)C;
          uint8_t* buf = sX(xb);
#pragma unroll
          for (int c0 = 0; c0 < kMlpMaxC; c0 += 16) {
            if (c0 >= C) break;
            uint32_t u[16];
            tmem_ld16(ta + c0, u);
            tmem_wait_ld_keep(u);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int ch = c0 + 8 * k;  // first channel of this 8-channel group
              const uint4 xv = real ? *reinterpret_cast<const uint4*>(xrow + ch) : make_uint4(0, 0, 0, 0);
              const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 xf = __bfloat1622float2(x2[e]);
                const float2 bb = *reinterpret_cast<const float2*>(sB2 + ch + 2 * e);
                float2 v = __fadd2_rn(
                    make_float2(__uint_as_float(u[8 * k + 2 * e]), __uint_as_float(u[8 * k + 2 * e + 1])), bb);
                v = __fadd2_rn(v, xf);
                w[e] = pack2(v.x, v.y);
              }
              *reinterpret_cast<uint4*>(buf + sw64_chunk(r, ch >> 3)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        tc_fence_before();
        fence_proxy_async_smem();  // staged rows -> the producer's TMA store
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cta(&acc2_free[ob]);
          mbar_arrive_cta(&out_full[xb]);
        }
      };
      // tiles are normalised one ahead of the output they wait for
      if (ntiles > 0) normalise(0);
      for (long long t = 0; t < ntiles; ++t) {
        if (t + 1 < ntiles) normalise(t + 1);
        finish_tile(t);
      }
    } else {
      // GELU warps: GELU of each hidden chunk, this warp's CW fc1 columns
      // (part hq of the chunk) -> CW/2 columns of bf16 pairs over the first
      // half of the same columns.
      const int hq = (warp - kMlpGelu0) >> 2;
      const int CW = HC / kMlpGeluPerQ;  // this warp's columns of a chunk: 16, 32 or 64
      const long long total = ntiles * NCH;
      int c = 0;  // chunk of the tile (g mod NCH, kept incrementally)
      for (long long g = 0; g < total; ++g, c = c + 1 == NCH ? 0 : c + 1) {
        if (!s_abort && !mbar_wait(&acc1_full[g & 1], (uint32_t)(g >> 1) & 1, a.ctx.err, kErrWaitMma, lim))
          s_abort = 1;
        tc_fence_after();
        if (!s_abort) {
          const uint32_t ta = tAcc1 + lane_base + (uint32_t)(g & 1) * (uint32_t)HC + (uint32_t)(hq * CW);
          const float* b1 = sB1 + c * HC + hq * CW;
          for (int p0 = 0; p0 < CW; p0 += 32) {  // up to 32 columns at a time
            const int n = CW - p0 < 32 ? CW - p0 : 32;
            uint32_t u[32], w[16];
            if (n == 32)
              tmem_ld32(ta + p0, u);
            else
              tmem_ld16(ta + p0, u);
            tmem_wait_ld_keep(u);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (2 * e >= n) break;
              const float2 bb = *reinterpret_cast<const float2*>(b1 + p0 + 2 * e);
              const float2 v =
                  __fadd2_rn(make_float2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), bb);
              const float2 gv = gelu2(v);
              w[e] = pack2(gv.x, gv.y);
            }
            // packed pairs over the first half of this warp's columns
            if (n == 32)
              tmem_st16(ta + p0 / 2, w);
            else
              tmem_st8(ta + p0 / 2, w);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(&h_full[g & 1]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// bf16 tensor map of `rank` dims (dims[0] innermost), strides in bytes for
// dims 1.., box sizes per dim; no swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              const cuuint32_t* box, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Hidden chunk width and weight stages that fit next to the x buffers: one
// stage per chunk (resident) when they all fit, else 2 (streamed), with
// 128-column chunks when possible, else 64; {0, 0} when nothing fits.
struct MlpPlan {
  int hc, stages;
};
MlpPlan mlp_plan(int C, int hidden) {
  for (int hc = kMlpMaxHC; hc >= 64; hc /= 2) {
    if (hidden % hc) continue;
    const int nch = hidden / hc;
    if (nch > 8) continue;
    const int base = mlp_smem(C, hidden, hc, 0).total;
    const int room = (227 * 1024 - 1024 - base) / (2 * C * hc * 2);  // 1 KB left for static shared memory
    if (room >= nch) return {hc, nch};
    if (room >= 2) return {hc, 2};
  }
  return {0, 0};
}

}  // namespace

bool mlp_supported(int C, int hidden) {
  return C >= 32 && C <= kMlpMaxC && C % 32 == 0 && hidden >= 64 && mlp_plan(C, hidden).stages > 0;
}

cudaError_t launch_mlp(const KernelCtx& ctx, long long M, int C, int hidden, const void* x, const void* gamma,
                       const void* beta, float eps, const void* W1, const void* b1, const void* W2, const void* b2,
                       void* out, cudaStream_t st) {
  if (!mlp_supported(C, hidden) || M <= 0 || M > (1LL << 31) - 1) return cudaErrorInvalidValue;
  const MlpPlan plan = mlp_plan(C, hidden);
  const int S = plan.stages, HC = plan.hc;
  CUtensorMap mx, mo, m1, m2;
  // x / out as (32 channels, M rows, C/32 blocks) with the 64-byte swizzle: one
  // box is a 128-row tile in the K-major SWIZZLE_64B operand layout
  const cuuint64_t xd[3] = {32, (cuuint64_t)M, (cuuint64_t)(C / 32)};
  const cuuint64_t xs[2] = {(cuuint64_t)C * 2, 64};
  const cuuint32_t xbox[3] = {32, 128, (cuuint32_t)(C / 32)};
  // W1 [C][hidden] as (8 n, 8 k, hidden/8 n-groups, C/8 k-groups); box = one
  // hidden chunk, all of K
  const cuuint64_t w1d[4] = {8, 8, (cuuint64_t)(hidden / 8), (cuuint64_t)(C / 8)};
  const cuuint64_t w1s[3] = {(cuuint64_t)hidden * 2, 16, (cuuint64_t)hidden * 16};
  const cuuint32_t w1box[4] = {8, 8, (cuuint32_t)(HC / 8), (cuuint32_t)(C / 8)};
  // W2 [hidden][C] as (8 n, 8 k, C/8 n-groups, hidden/8 k-groups); box = the
  // rows of one hidden chunk, all of N
  const cuuint64_t w2d[4] = {8, 8, (cuuint64_t)(C / 8), (cuuint64_t)(hidden / 8)};
  const cuuint64_t w2s[3] = {(cuuint64_t)C * 2, 16, (cuuint64_t)C * 16};
  const cuuint32_t w2box[4] = {8, 8, (cuuint32_t)(C / 8), (cuuint32_t)(HC / 8)};
  if (!make_map(&mx, x, 3, xd, xs, xbox, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&mo, out, 3, xd, xs, xbox, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&m1, W1, 4, w1d, w1s, w1box) || !make_map(&m2, W2, 4, w2d, w2s, w2box))
    return cudaErrorInvalidValue;
  MlpArgs a;
  a.M = M;
  a.C = C;
  a.hidden = hidden;
  a.hc = HC;
  a.nch = hidden / HC;
  a.stages = S;
  a.resident = S == a.nch;
  a.eps = eps;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.gamma = static_cast<const __nv_bfloat16*>(gamma);
  a.beta = static_cast<const __nv_bfloat16*>(beta);
  a.b1 = static_cast<const __nv_bfloat16*>(b1);
  a.b2 = static_cast<const __nv_bfloat16*>(b2);
  a.ctx = ctx;
  const int smem = mlp_smem(C, hidden, HC, S).total;
  cudaError_t e = cudaFuncSetAttribute(mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (M + 127) / 128;
  const int grid = (int)(tiles < sms ? tiles : sms);
  prof_begin(kKindMlp, st);
  mlp_kernel<<<grid, kMlpThreads, smem, st>>>(mx, mo, m1, m2, a);
  prof_end(kKindMlp, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace vswin
