// bf16 backward of the layer on sm_100a tensor cores, for (P,7,7) windows with
// P <= 8 and head width 32 ("Video Swin Transformer" summary page, Method
// steps 4-6 and eq. 2, differentiated): per window and head, with the scaled
// scores S = q k^T / sqrt(d) + B and P = softmax(S) over the query's region,
//   dP = dO v^T,  D_i = dO_i . O_i,  dS = P * (dP - D),
//   dq = dS k / sqrt(d),  dk = dS^T q / sqrt(d),  dv = P^T dO,
//   dtable[row(i, j)][h] += dS[i][j].
//
// Per chunk of windows:
//   1. the forward's first three steps (row table, q / k / v slabs with q
//      scaled by log2(e)/sqrt(d), attention output O) with each query row's
//      softmax reference and sum (exp2 domain) saved;
//   2. dO = dY Wproj^T into per-(window, head) slabs of the q layout (the
//      QKV GEMM with Wproj transposed, no bias);
//   3. bwd_attn_kernel: one CTA per (window, head), q / k / v / dO slabs in
//      shared memory. Keys in blocks of 128 (the MMA's M), queries in tiles
//      of up to 128 (its N); per (key block, query tile):
//        S^T = K Q^T and dP^T = V dO^T on tcgen05 into TMEM (fp32);
//        sixteen warps (TMEM lane = key) rebuild P^T = 2^(S^T + B - m) / l from
//        the saved statistics and form dS^T = P^T (dP^T - D), both written
//        back to TMEM as bf16 over their own scores, dS^T also to shared
//        memory (the MN-major A operand of dq), and the table gradient summed
//        in shared memory;
//        dV += P^T dO and dK += dS^T Q (A from TMEM), dQ_tile += dS K (A
//        from shared memory) on tcgen05, dQ of every query tile resident in
//        TMEM across the key blocks;
//      then dK and dV of the block, and at the end dQ, written as bf16 rows of
//      dqkv [slot][3C], and the table gradient added once per table row;
//   4. dX = dqkv Wqkv^T scattered to the tokens (the projection GEMM with
//      Wqkv transposed), dWqkv = X^T dqkv, dWproj = O^T dY and the bias sums
//      as fp32 split-K sums.
//
// TMEM columns of the attention CTA: S^T / P^T [0, 128), dP^T / dS^T
// [128, 256), dK [256, 288), dV [288, 320), dQ of query tile t [320 + 32 t,
// + 32). P^T of queries [32 c, 32 c + 32) is packed at columns [32 c, 32 c +
// 16) (each quarter written by its own warps over scores they have read),
// likewise dS^T; the TS MMA's 16-query step k reads columns 32 (k / 2) +
// 8 (k % 2).
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vswin {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBwThreads = 512;  // warp w: TMEM lane quarter w % 4, query-column quarter w / 4
constexpr uint32_t kBwTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDK = 256, kColDV = 288, kColDQ = 320;
constexpr int kRowBytes = 64;  // one slab row: 32 bf16

enum : int { kErrBwLoad = 0x111, kErrBwMma = 0x112 };

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Shared-memory add without a returned value.
__device__ __forceinline__ void red_add_shared(float* p, float v) {
  asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(smem_u32(p)), "f"(v) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}

// Window of (P,7,7): slot n = (pt * 7 + ph) * 7 + pw; keys stored as 8-row lines
// of 7 (row (n / 7) * 8 + n % 7, eighth row padding).
template <int P_>
struct BwWin {
  static constexpr int P = P_;
  static constexpr int N = P * 49;
  static constexpr int QSLAB = (N + 15) / 16 * 16;
  static constexpr int KLINES = P * 7;
  static constexpr int KCOLS = (KLINES * 8 + 31) / 32 * 32;
  static constexpr int QT = (QSLAB + 127) / 128;  // query tiles
  static constexpr int NKB = (KCOLS + 127) / 128;  // key blocks
  static constexpr int KROWS = NKB * 128;
  static constexpr int TABLE = (2 * P - 1) * 169;
  static constexpr int E0 = (P - 1) * 169 + 6 * 13 + 6;  // table row of a zero offset
  // shared memory (bytes)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + QSLAB * kRowBytes;
  static constexpr int OFF_K = OFF_DO + QSLAB * kRowBytes;
  static constexpr int OFF_V = OFF_K + KROWS * kRowBytes;
  static constexpr int OFF_DS = OFF_V + KROWS * kRowBytes;  // 128 keys x 128 queries bf16, MN-major A
  static constexpr int OFF_QI = OFF_DS + 128 * 128 * 2;      // per query: (m, 1/l, D, e * 64 + region + 1)
  static constexpr int OFF_KI = OFF_QI + QT * 128 * 16;      // per key row: (e, region or -2)
  static constexpr int OFF_T = OFF_KI + KROWS * 8;           // the head's table column (log2 e units)
  static constexpr int OFF_G = OFF_T + (TABLE * 4 + 15) / 16 * 16;  // its gradient
  static constexpr int OFF_BAR = OFF_G + (TABLE * 4 + 15) / 16 * 16;
  // at least 64 KB from the dS operand on (its MMA reads stay inside the CTA's
  // shared memory whatever the descriptor strides) and at least 116 KB, so that
  // one CTA (512 TMEM columns) owns its SM
  static constexpr int SMEM0 = OFF_BAR + 64 > OFF_DS + 65536 ? OFF_BAR + 64 : OFF_DS + 65536;
  static constexpr int SMEM = SMEM0 > 116 * 1024 ? SMEM0 : 116 * 1024;
  static_assert(kColDQ + 32 * QT <= kBwTmemCols, "dQ of every query tile must fit in TMEM");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct BwdArgs {
  Geom g;
  KernelCtx ctx;
  const __nv_bfloat16* qkv;    // slabs of the chunk: per (window, head) q | k | v
  const __nv_bfloat16* dOs;    // dO slabs: per (window, head) QSLAB rows
  const __nv_bfloat16* o;      // [nwin * N][C] attention output of the forward
  const float2* stats;         // [nwin * N][heads] (m, l)
  const __nv_bfloat16* table;  // [TABLE][heads]
  __nv_bfloat16* dqkv;         // [nwin * N][3C]
  float* dtable;               // [TABLE][heads], accumulated
  long long win0, nwin;  // first window of the chunk (for the window's position), windows in it
  long long head_elems;        // elements of one (window, head) q | k | v block
  int qrows;                   // q slab rows (k slab follows)
  int kvrows;                  // k / v slab rows
};

template <class Wn>
__global__ void __launch_bounds__(kBwThreads, 1) bwd_attn_kernel(BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem + Wn::OFF_Q;
  uint8_t* sDO = smem + Wn::OFF_DO;
  uint8_t* sK = smem + Wn::OFF_K;
  uint8_t* sV = smem + Wn::OFF_V;
  uint8_t* sDS = smem + Wn::OFF_DS;
  float4* sQI = reinterpret_cast<float4*>(smem + Wn::OFF_QI);
  int2* sKI = reinterpret_cast<int2*>(smem + Wn::OFF_KI);
  float* sT = reinterpret_cast<float*>(smem + Wn::OFF_T);
  float* sG = reinterpret_cast<float*>(smem + Wn::OFF_G);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Wn::OFF_BAR);
  uint64_t* ld_full = bars;      // the four slabs landed
  uint64_t* mma_done = bars + 1;  // the MMAs issued so far completed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cq = warp >> 2;
  const Geom& g = a.g;
  const int C = g.C, C3 = 3 * g.C;
  const long long item = blockIdx.x;
  const int h = (int)(item / a.nwin);
  const long long wl = item % a.nwin;
  const uint64_t lim = a.ctx.wait_limit;
  const int w_in_clip = (int)((a.win0 + wl) % g.nW);
  const bool shifted = (g.sh[0] | g.sh[1] | g.sh[2]) != 0;

  if (tid == 0) {
    mbar_init(ld_full, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, kBwTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // ---- loads and per-row facts
  if (tid == 0) {
    const __nv_bfloat16* base = a.qkv + ((size_t)wl * g.heads + h) * a.head_elems;
    const __nv_bfloat16* dob = a.dOs + ((size_t)wl * g.heads + h) * (size_t)Wn::QSLAB * 32;
    mbar_arrive_expect_tx(ld_full, (uint32_t)(2 * Wn::QSLAB + 2 * Wn::KCOLS) * kRowBytes);
    bulk_g2s(sQ, base, Wn::QSLAB * kRowBytes, ld_full);
    bulk_g2s(sK, base + (size_t)a.qrows * 32, Wn::KCOLS * kRowBytes, ld_full);
    bulk_g2s(sV, base + (size_t)(a.qrows + a.kvrows) * 32, Wn::KCOLS * kRowBytes, ld_full);
    bulk_g2s(sDO, dob, Wn::QSLAB * kRowBytes, ld_full);
  }
  for (int r = tid; r < Wn::TABLE; r += kBwThreads) {
    sT[r] = __bfloat162float(a.table[(size_t)r * g.heads + h]) * kLog2e;
    sG[r] = 0.f;
  }
  // key rows past the k / v slabs (the last block's MMA rows) read zeros
  for (int k = tid; k < (Wn::KROWS - Wn::KCOLS) * 4; k += kBwThreads) {
    const int n = Wn::KCOLS + (k >> 2), c = k & 3;
    *reinterpret_cast<uint4*>(sK + (n >> 3) * 512 + c * 128 + (n & 7) * 16) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(sV + (n >> 3) * 512 + c * 128 + (n & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
  for (int n = tid; n < Wn::KROWS; n += kBwThreads) {
    const int line = n >> 3, pw = n & 7;
    int2 ki = make_int2(0, -2);
    if (pw < 7 && line < Wn::KLINES) {
      const int slot = line * 7 + pw;
      ki.x = ((line / 7) * 13 + line % 7) * 13 + pw;
      ki.y = shifted ? slot_region(g, w_in_clip, slot) : 0;
    }
    sKI[n] = ki;
  }
  if (!mbar_wait(ld_full, 0, a.ctx.err, kErrBwLoad, lim)) s_abort = 1;
  __syncthreads();
  // padding key rows (the eighth of each line, whole padding lines) are zero, so
  // that their masked scores and dP stay finite and the dq product (which
  // multiplies zeros of dS with these rows) cannot turn into NaN
  for (int k = tid; k < (Wn::KLINES + (Wn::KCOLS / 8 - Wn::KLINES) * 8) * 4; k += kBwThreads) {
    const int d = k >> 2, c = k & 3;
    const int n = d < Wn::KLINES ? d * 8 + 7 : Wn::KLINES * 8 + (d - Wn::KLINES);
    *reinterpret_cast<uint4*>(sK + (n >> 3) * 512 + c * 128 + (n & 7) * 16) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(sV + (n >> 3) * 512 + c * 128 + (n & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
  // q and dO rows past the window (never written by the GEMMs) are zero
  for (int k = tid; k < (Wn::QSLAB - Wn::N) * 4; k += kBwThreads) {
    const int i = Wn::N + (k >> 2), c = k & 3;
    *reinterpret_cast<uint4*>(sQ + (i >> 3) * 512 + c * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(sDO + (i >> 3) * 512 + c * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
  for (int i = tid; i < Wn::QT * 128; i += kBwThreads) {
    float4 qi = make_float4(0.f, 0.f, 0.f, __int_as_float(0));  // padding query: P = 0, region -1
    if (i < Wn::N) {
      const long long row = wl * Wn::N + i;
      const float2 st = a.stats[row * g.heads + h];
      const __nv_bfloat16* orow = a.o + row * C + h * 32;
      float D = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 ov = *reinterpret_cast<const uint4*>(orow + 8 * c);
        const uint4 dv = *reinterpret_cast<const uint4*>(sDO + (i >> 3) * 512 + c * 128 + (i & 7) * 16);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
        const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 of = __bfloat1622float2(o2[k]), df = __bfloat1622float2(d2[k]);
          D = fmaf(of.x, df.x, fmaf(of.y, df.y, D));
        }
      }
      const int pt = i / 49, ph = (i / 7) % 7, pw = i % 7;
      const int e = (pt * 13 + ph) * 13 + pw;
      const int reg = shifted ? slot_region(g, w_in_clip, i) : 0;
      qi = make_float4(st.x, 1.0f / st.y, D, __int_as_float(e * 64 + reg + 1));
    }
    sQI[i] = qi;
  }
  fence_proxy_async_smem();  // zeroed rows are tensor-core operands
  __syncthreads();

  // ---- MMAs (one elected thread of warp 0)
  const uint32_t sq = smem_u32(sQ), sdo = smem_u32(sDO), sk = smem_u32(sK), sv = smem_u32(sV), sds = smem_u32(sDS);
  auto nq_of = [](int qt) { return Wn::QSLAB - qt * 128 < 128 ? Wn::QSLAB - qt * 128 : 128; };
  // S^T = K_kb Q_qt^T and dP^T = V_kb dO_qt^T (K-major operands: 128-byte steps
  // along the channels, 512-byte steps along the rows)
  auto issue_scores = [&](int s) {
    const int kb = s / Wn::QT, qt = s % Wn::QT, nq = nq_of(qt);
    const uint32_t id = idesc_bf16(128, nq, 0, 0);
    const uint64_t ak = smem_desc(sk + kb * 8192, 128, 512), av = smem_desc(sv + kb * 8192, 128, 512);
    const uint64_t bq = smem_desc(sq + qt * 8192, 128, 512), bo = smem_desc(sdo + qt * 8192, 128, 512);
    umma_ss(tmem + kColS, ak, bq, id, 0u);
    umma_ss(tmem + kColS, ak + 16, bq + 16, id, 1u);
    umma_ss(tmem + kColDP, av, bo, id, 0u);
    umma_ss(tmem + kColDP, av + 16, bo + 16, id, 1u);
  };
  // dV += P^T dO, dK += dS^T Q (A from TMEM, 16 queries per step; B MN-major:
  // 1 KB per 16 rows), dQ_qt += dS K_kb (A = dS from shared memory, MN-major:
  // 2 KB per 8 keys, 128 B per 8 queries)
  auto issue_grads = [&](int s) {
    const int kb = s / Wn::QT, qt = s % Wn::QT, nq = nq_of(qt);
    const uint32_t id = idesc_bf16(128, 32, 0, 1);
    for (int ks = 0; ks < nq / 16; ++ks) {
      const uint32_t acol = 32u * (uint32_t)(ks >> 1) + 8u * (uint32_t)(ks & 1);
      const uint32_t acc = (qt > 0 || ks > 0) ? 1u : 0u;
      umma_ts(tmem + kColDV, tmem + kColS + acol, smem_desc(sdo + qt * 8192 + ks * 1024, 512, 128), id, acc);
      umma_ts(tmem + kColDK, tmem + kColDP + acol, smem_desc(sq + qt * 8192 + ks * 1024, 512, 128), id, acc);
    }
    const uint32_t idq = idesc_bf16(128, 32, 1, 1);
    for (int ks = 0; ks < 8; ++ks)
      umma_ss(tmem + kColDQ + 32u * (uint32_t)qt, smem_desc(sds + ks * 4096, 2048, 128),
              smem_desc(sk + kb * 8192 + ks * 1024, 512, 128), idq, (kb > 0 || ks > 0) ? 1u : 0u);
  };

  const int S = Wn::NKB * Wn::QT;
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  if (warp == 0) {
    if (!s_abort && elect_one()) {
      issue_scores(0);
      umma_commit(mma_done);
    }
    __syncwarp();
  }
  // dK / dV of key block kb to dqkv: column quarter cq of the warp takes dK
  // (cq 0, 1) or dV (cq 2, 3), 16 channels each
  auto write_kv = [&](int kb) {
    const int n = kb * 128 + qd * 32 + lane;
    const bool is_v = cq >= 2;
    const int c16 = (cq & 1) * 16;
    uint32_t u[16];
    tmem_ld8(tmem + lane_base + (is_v ? kColDV : kColDK) + c16, *reinterpret_cast<uint32_t(*)[8]>(&u[0]));
    tmem_ld8(tmem + lane_base + (is_v ? kColDV : kColDK) + c16 + 8, *reinterpret_cast<uint32_t(*)[8]>(&u[8]));
    tmem_wait_ld();
    const int line = n >> 3, pw = n & 7;
    if (!s_abort && pw < 7 && line < Wn::KLINES) {
      const int slot = line * 7 + pw;
      const float sc = is_v ? 1.0f : 1.0f / kLog2e;  // dk: the slab's q carries log2(e) / sqrt(d)
      __nv_bfloat16* dst = a.dqkv + (wl * Wn::N + slot) * C3 + (is_v ? 2 * C : C) + h * 32 + c16;
#pragma unroll
      for (int c = 0; c < 2; ++c)
        reinterpret_cast<uint4*>(dst)[c] = make_uint4(
            pack_bf16x2(__uint_as_float(u[8 * c + 0]) * sc, __uint_as_float(u[8 * c + 1]) * sc),
            pack_bf16x2(__uint_as_float(u[8 * c + 2]) * sc, __uint_as_float(u[8 * c + 3]) * sc),
            pack_bf16x2(__uint_as_float(u[8 * c + 4]) * sc, __uint_as_float(u[8 * c + 5]) * sc),
            pack_bf16x2(__uint_as_float(u[8 * c + 6]) * sc, __uint_as_float(u[8 * c + 7]) * sc));
    }
  };

  uint32_t phase = 0;
  for (int s = 0; s < S; ++s) {
    const int kb = s / Wn::QT, qt = s % Wn::QT, nq = nq_of(qt);
    if (!s_abort && !mbar_wait(mma_done, phase, a.ctx.err, kErrBwMma, lim)) s_abort = 1;
    phase ^= 1;
    tc_fence_after();
    if (qt == 0 && kb > 0) write_kv(kb - 1);  // the previous block's MMAs are complete
    // this warp's query columns of the tile: its quarter, cut at nq
    const int c_begin = cq * 32;
    const int c_end = c_begin + 32 < nq ? c_begin + 32 : nq;
    const int j = qd * 32 + lane;
    const int2 kinfo = sKI[kb * 128 + j];
    const int ebase = Wn::E0 - kinfo.x;
    if (!s_abort && c_begin < c_end) {
      // all of this warp's scores and dP first (one wait), then 8 columns at a time
      uint32_t us_all[32], ud_all[32];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (c_begin + 8 * k < c_end) {
          tmem_ld8(tmem + lane_base + kColS + c_begin + 8 * k, *reinterpret_cast<uint32_t(*)[8]>(&us_all[8 * k]));
          tmem_ld8(tmem + lane_base + kColDP + c_begin + 8 * k, *reinterpret_cast<uint32_t(*)[8]>(&ud_all[8 * k]));
        }
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c0 = c_begin + 8 * k;
        if (c0 >= c_end) break;
        const uint32_t* us = &us_all[8 * k];
        const uint32_t* ud = &ud_all[8 * k];
        float p[8], ds[8];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const float4 qi = sQI[qt * 128 + c0 + cc];
          const int bits = __float_as_int(qi.w);
          const bool ok = (bits & 63) - 1 == kinfo.y;
          const int r = ok ? (bits >> 6) + ebase : 0;
          const float pr = ok ? ex2_approx(__uint_as_float(us[cc]) + sT[r] - qi.x) * qi.y : 0.f;
          const float d = pr * (__uint_as_float(ud[cc]) - qi.z);
          p[cc] = pr;
          ds[cc] = d;
          if (ok) red_add_shared(&sG[r], d);
        }
        const uint32_t pp[4] = {pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                                pack_bf16x2(p[6], p[7])};
        const uint32_t pd[4] = {pack_bf16x2(ds[0], ds[1]), pack_bf16x2(ds[2], ds[3]), pack_bf16x2(ds[4], ds[5]),
                                pack_bf16x2(ds[6], ds[7])};
        const uint32_t pcol = (uint32_t)(c_begin + (c0 - c_begin) / 2);  // packed column (see the file comment)
        tmem_st4(tmem + lane_base + kColS + pcol, pp);
        tmem_st4(tmem + lane_base + kColDP + pcol, pd);
        *reinterpret_cast<uint4*>(sDS + (j >> 3) * 2048 + (c0 >> 3) * 128 + (j & 7) * 16) =
            make_uint4(pd[0], pd[1], pd[2], pd[3]);
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      if (!s_abort && elect_one()) {
        issue_grads(s);
        if (s + 1 < S) issue_scores(s + 1);
        umma_commit(mma_done);
      }
      __syncwarp();
    }
  }
  if (!s_abort && !mbar_wait(mma_done, phase, a.ctx.err, kErrBwMma, lim)) s_abort = 1;
  tc_fence_after();
  write_kv(Wn::NKB - 1);
  // dQ of the query tiles (this warp: tile cq)
  for (int qt = cq; qt < cq + 1 && qt < Wn::QT; ++qt) {
    uint32_t u[32];
    const uint32_t col = kColDQ + 32u * (uint32_t)qt;
    tmem_ld8(tmem + lane_base + col, *reinterpret_cast<uint32_t(*)[8]>(&u[0]));
    tmem_ld8(tmem + lane_base + col + 8, *reinterpret_cast<uint32_t(*)[8]>(&u[8]));
    tmem_ld8(tmem + lane_base + col + 16, *reinterpret_cast<uint32_t(*)[8]>(&u[16]));
    tmem_ld8(tmem + lane_base + col + 24, *reinterpret_cast<uint32_t(*)[8]>(&u[24]));
    tmem_wait_ld();
    const int i = qt * 128 + qd * 32 + lane;
    if (!s_abort && i < Wn::N) {
      const float sc = rsqrtf(32.0f);
      __nv_bfloat16* dst = a.dqkv + (wl * Wn::N + i) * C3 + h * 32;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        reinterpret_cast<uint4*>(dst)[c] = make_uint4(
            pack_bf16x2(__uint_as_float(u[8 * c + 0]) * sc, __uint_as_float(u[8 * c + 1]) * sc),
            pack_bf16x2(__uint_as_float(u[8 * c + 2]) * sc, __uint_as_float(u[8 * c + 3]) * sc),
            pack_bf16x2(__uint_as_float(u[8 * c + 4]) * sc, __uint_as_float(u[8 * c + 5]) * sc),
            pack_bf16x2(__uint_as_float(u[8 * c + 6]) * sc, __uint_as_float(u[8 * c + 7]) * sc));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!s_abort)
    for (int r = tid; r < Wn::TABLE; r += kBwThreads)
      if (sG[r] != 0.f) atomicAdd(&a.dtable[(size_t)r * g.heads + h], sG[r]);
  if (warp == 0) tmem_dealloc(tmem, kBwTmemCols);
}

template <class Wn>
cudaError_t launch_bwd_attn(const BwdArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_attn_kernel<Wn>, cudaFuncAttributeMaxDynamicSharedMemorySize, Wn::SMEM);
  if (e != cudaSuccess) return e;
  const long long items = a.nwin * a.g.heads;
  if (items > 2147483647LL) return cudaErrorInvalidConfiguration;
  prof_begin(kKindAttnBwd, st);
  bwd_attn_kernel<Wn><<<(unsigned)items, kBwThreads, Wn::SMEM, st>>>(a);
  prof_end(kKindAttnBwd, st);
  count_launch();
  return cudaGetLastError();
}

// Weight-gradient sums on tcgen05: out[m][n] += sum_r A(r, m) B(r, n) for m < M
// and bias_out[n] += sum_r B(r, n), over the rows r of the grid's split, with
// A(r, m) = A[arow(r) lda + m], B(r, n) = B[brow(r) ldb + n] (bf16; a negative
// row reads zeros; arow(r) = a_src ? a_src[r] : r, likewise brow). The MMA is
// D[128 x BN] += A^T B: M = the M columns of A plus a column of ones (the bias
// row) and zeros up to 128, N = BN output columns, K = rows, 16 at a time.
// Both operands are MN-major in shared memory (8 rows x 16 bytes per core
// matrix; A: 128 B between column groups, 2 KB between row groups; B: 128 B,
// BN x 16 B). 128 threads gather 64-row tiles with cp.async into four stages
// (each thread's copies arrive on the stage's barrier), thread 0 issues the
// MMAs; at the end each thread adds its accumulator row to out with atomics.
constexpr int kGrThreads = 128;
constexpr int kGrRows = 64;    // rows per tile
constexpr int kGrStages = 4;
constexpr int kGrABytes = kGrRows * 128 * 2;  // 16 KB

__host__ __device__ inline int gram_b_bytes(int BN) { return kGrRows * BN * 2; }
__host__ inline int gram_smem_bytes(int BN) { return kGrStages * (kGrABytes + gram_b_bytes(BN)) + 128; }

struct GramArgs {
  KernelCtx ctx;
  long long rows, rows_per_split;  // rows of the sum, rows per CTA (multiple of 64)
  int M, N, BN;
  const __nv_bfloat16* A;
  long long lda;
  const int* a_src;
  const __nv_bfloat16* B;
  long long ldb;
  const int* b_src;
  float* out;
  float* bias_out;
};

__global__ void __launch_bounds__(kGrThreads, 1) gram_tc_kernel(GramArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int BN = a.BN;
  uint8_t* sA = smem;                                    // [stages][16 KB]
  uint8_t* sB = smem + kGrStages * kGrABytes;            // [stages][64 x BN x 2]
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGrStages * gram_b_bytes(BN));
  uint64_t* empty = full + kGrStages;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(empty + kGrStages);
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN;
  const long long r_begin = (long long)blockIdx.y * a.rows_per_split;
  long long r_end = r_begin + a.rows_per_split;
  if (r_end > a.rows) r_end = a.rows;
  const long long ntiles = r_end > r_begin ? (r_end - r_begin + kGrRows - 1) / kGrRows : 0;
  const uint64_t lim = a.ctx.wait_limit;
  const uint32_t tcols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;

  if (tid == 0) {
    for (int k = 0; k < kGrStages; ++k) {
      mbar_init(&full[k], kGrThreads);
      mbar_init(&empty[k], 1);
    }
    fence_mbar_init();
    s_abort = 0;
  }
  // the constant columns of A in every stage: ones at column M, zeros after
  for (int k = tid; k < kGrStages * kGrRows * (16 - a.M / 8); k += kGrThreads) {
    const int st = k / (kGrRows * (16 - a.M / 8)), rem = k % (kGrRows * (16 - a.M / 8));
    const int r = rem / (16 - a.M / 8), mg = a.M / 8 + rem % (16 - a.M / 8);
    const uint4 v = make_uint4(mg * 8 == a.M ? 0x3F80u : 0u, 0u, 0u, 0u);  // bf16 1.0 in the low half
    *reinterpret_cast<uint4*>(sA + st * kGrABytes + (r >> 3) * 2048 + mg * 128 + (r & 7) * 16) = v;
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(s_tmem, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  auto load_tile = [&](long long t) {
    const int st = (int)(t % kGrStages);
    const long long rt = r_begin + t * kGrRows;
    uint8_t* dA = sA + st * kGrABytes;
    uint8_t* dB = sB + st * gram_b_bytes(BN);
    const int ag = a.M / 8, bg = BN / 8;
    for (int k = tid; k < kGrRows * ag; k += kGrThreads) {
      const int r = k / ag, mg = k % ag;
      const long long row = rt + r;
      long long src = -1;
      if (row < r_end) src = a.a_src ? (long long)a.a_src[row] : row;
      cp_async_16(dA + (r >> 3) * 2048 + mg * 128 + (r & 7) * 16, a.A + (src < 0 ? 0 : src * a.lda) + mg * 8,
                  src < 0 ? 0u : 16u);
    }
    for (int k = tid; k < kGrRows * bg; k += kGrThreads) {
      const int r = k / bg, ng = k % bg;
      const long long row = rt + r;
      long long src = -1;
      if (row < r_end) src = a.b_src ? (long long)a.b_src[row] : row;
      cp_async_16(dB + (r >> 3) * (BN * 16) + ng * 128 + (r & 7) * 16,
                  a.B + (src < 0 ? 0 : src * a.ldb) + n0 + ng * 8, src < 0 ? 0u : 16u);
    }
    cp_async_mbar_arrive_noinc(&full[st]);
  };

  const uint32_t id = idesc_bf16(128, BN, 1, 1);
  for (long long t = 0; t < kGrStages - 1 && t < ntiles; ++t) load_tile(t);
  for (long long t = 0; t < ntiles; ++t) {
    const long long tn = t + kGrStages - 1;  // tile to load now, into the stage tile t - 1 used
    if (tn < ntiles) {
      if (t >= 1 && !s_abort &&
          !mbar_wait(&empty[tn % kGrStages], (uint32_t)((tn / kGrStages) - 1) & 1, a.ctx.err, kErrBwMma, lim))
        s_abort = 1;
      if (!s_abort) load_tile(tn);
    }
    if (tid == 0) {
      const int st = (int)(t % kGrStages);
      if (!s_abort && !mbar_wait(&full[st], (uint32_t)(t / kGrStages) & 1, a.ctx.err, kErrBwLoad, lim)) s_abort = 1;
      fence_proxy_async_smem();
      tc_fence_after();
      if (!s_abort) {
        const uint32_t aa = smem_u32(sA + st * kGrABytes), bb = smem_u32(sB + st * gram_b_bytes(BN));
        for (int ks = 0; ks < kGrRows / 16; ++ks)
          umma_ss(tmem, smem_desc(aa + ks * 4096, 2048, 128), smem_desc(bb + ks * 2 * BN * 16, BN * 16, 128), id,
                  (t > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(&empty[st]);
    }
  }
  cp_async_wait_all();
  // wait for the last tile's MMAs (its stage's empty barrier)
  if (ntiles > 0) {
    const long long tl = ntiles - 1;
    if (!s_abort && !mbar_wait(&empty[tl % kGrStages], (uint32_t)(tl / kGrStages) & 1, a.ctx.err, kErrBwMma, lim))
      s_abort = 1;
  }
  tc_fence_after();
  // thread = accumulator row m (TMEM lane), BN columns
  const int m = warp * 32 + lane;
  if (ntiles > 0 && !s_abort) {
    for (int c0 = 0; c0 < BN; c0 += 8) {
      uint32_t u[8];
      tmem_ld8(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, u);
      tmem_wait_ld();
      float* dst = m < a.M ? a.out + (size_t)m * a.N + n0 + c0 : (m == a.M ? a.bias_out + n0 + c0 : nullptr);
      if (dst)
#pragma unroll
        for (int k = 0; k < 8; ++k) atomicAdd(dst + k, __uint_as_float(u[k]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tcols);
}

// Chooses the split so that every SM gets a CTA or two.
cudaError_t launch_gram_tc(const KernelCtx& ctx, long long rows, int M, int N, const void* A, long long lda,
                           const int* a_src, const void* B, long long ldb, const int* b_src, float* out,
                           float* bias_out, cudaStream_t st) {
  int BN = N;
  if (BN > 256 || BN % 16 != 0) {
    BN = 0;
    for (int bn = 256; bn >= 16; bn -= 16)
      if (N % bn == 0) {
        BN = bn;
        break;
      }
  }
  if (BN == 0 || M % 8 != 0 || M + 1 > 128) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntile = N / BN;
  long long splits = (sms + ntile - 1) / ntile;
  long long per = (rows + splits - 1) / splits;
  per = (per + kGrRows - 1) / kGrRows * kGrRows;
  splits = (rows + per - 1) / per;
  if (splits < 1) splits = 1;
  if (splits > 65535) return cudaErrorInvalidConfiguration;
  GramArgs ga{};
  ga.ctx = ctx;
  ga.rows = rows;
  ga.rows_per_split = per;
  ga.M = M, ga.N = N, ga.BN = BN;
  ga.A = static_cast<const __nv_bfloat16*>(A), ga.lda = lda, ga.a_src = a_src;
  ga.B = static_cast<const __nv_bfloat16*>(B), ga.ldb = ldb, ga.b_src = b_src;
  ga.out = out, ga.bias_out = bias_out;
  const int smem = gram_smem_bytes(BN);
  cudaError_t e = cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  prof_begin(kKindOther, st);
  gram_tc_kernel<<<dim3((unsigned)ntile, (unsigned)splits), kGrThreads, smem, st>>>(ga);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

// out[c][r] = in[r][c] for an R x Cc bf16 matrix (weights used transposed).
__global__ void transpose_bf16_kernel(const __nv_bfloat16* __restrict__ in, __nv_bfloat16* __restrict__ out, int R,
                                      int Cc) {
  __shared__ __nv_bfloat16 t[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int r = r0 + k, c = c0 + threadIdx.x;
    if (r < R && c < Cc) t[k][threadIdx.x] = in[(size_t)r * Cc + c];
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int c = c0 + k, r = r0 + threadIdx.x;
    if (r < R && c < Cc) out[(size_t)c * R + r] = t[threadIdx.x][k];
  }
}

cudaError_t launch_transpose(const void* in, void* out, int R, int Cc, cudaStream_t st) {
  const dim3 grid((unsigned)((Cc + 31) / 32), (unsigned)((R + 31) / 32));
  prof_begin(kKindOther, st);
  transpose_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(static_cast<const __nv_bfloat16*>(in),
                                                      static_cast<__nv_bfloat16*>(out), R, Cc);
  prof_end(kKindOther, st);
  count_launch();
  return cudaGetLastError();
}

// Scratch of one chunk of `nwin` windows, after the forward chunk's own.
struct BwdChunk {
  size_t fwd, stats, dos, dqkv, total;
};

BwdChunk bwd_chunk_layout(const Geom& g, long long nwin) {
  BwdChunk c;
  auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
  c.fwd = up(bf16_scratch_bytes(g, nwin));
  c.stats = up((size_t)nwin * g.N * g.heads * sizeof(float2));
  c.dos = up((size_t)nwin * g.heads * g.Npad * 32 * 2);
  c.dqkv = up((size_t)nwin * g.N * 3 * g.C * 2);
  c.total = c.fwd + c.stats + c.dos + c.dqkv;
  return c;
}

}  // namespace

bool bf16_backward_supported(const Geom& g) {
  return g.d == 32 && g.win[1] == 7 && g.win[2] == 7 &&
         (g.win[0] == 1 || g.win[0] == 2 || g.win[0] == 4 || g.win[0] == 8) && g.C % 32 == 0;
}

size_t bf16_backward_scratch_bytes(const Geom& g, long long nwin) {
  // transposed weights and a zero bias, then the chunk
  const size_t fixed = ((size_t)4 * g.C * g.C * 2 + (size_t)3 * g.C * 2 + 1023) / 1024 * 1024;
  return fixed + bwd_chunk_layout(g, nwin).total;
}

cudaError_t launch_bf16_backward(const Geom& g, const KernelCtx& ctx, const void* x, const void* Wqkv,
                                 const void* bqkv, const void* Wproj, const void* table, const void* dy, void* dx,
                                 float* dWqkv, float* dbqkv, float* dWproj, float* dbproj, float* dtable,
                                 void* scratch, long long chunk, cudaStream_t st) {
  const int C = g.C;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  __nv_bfloat16* wprojT = reinterpret_cast<__nv_bfloat16*>(base);
  __nv_bfloat16* wqkvT = wprojT + (size_t)C * C;
  __nv_bfloat16* zero_bias = wqkvT + (size_t)3 * C * C;
  uint8_t* cbase = base + ((size_t)4 * C * C * 2 + (size_t)3 * C * 2 + 1023) / 1024 * 1024;
  const BwdChunk L = bwd_chunk_layout(g, chunk);
  float2* stats = reinterpret_cast<float2*>(cbase + L.fwd);
  __nv_bfloat16* dos = reinterpret_cast<__nv_bfloat16*>(cbase + L.fwd + L.stats);
  __nv_bfloat16* dqkv = reinterpret_cast<__nv_bfloat16*>(cbase + L.fwd + L.stats + L.dos);

  cudaError_t e = cudaMemsetAsync(zero_bias, 0, (size_t)3 * C * 2, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dWqkv, 0, (size_t)C * 3 * C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dbqkv, 0, (size_t)3 * C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dWproj, 0, (size_t)C * C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dbproj, 0, (size_t)C * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dtable, 0, (size_t)g.table_rows * g.heads * sizeof(float), st);
  if (e == cudaSuccess) e = launch_transpose(Wproj, wprojT, C, C, st);
  if (e == cudaSuccess) e = launch_transpose(Wqkv, wqkvT, C, 3 * C, st);
  if (e != cudaSuccess) return e;

  int qrows = 0, kvrows = 0, kv8 = 0;
  bf16_slab_rows(g, &qrows, &kvrows, &kv8);
  if (!kv8 || qrows != g.Npad) return cudaErrorInvalidValue;
  for (long long w0 = 0; w0 < g.windows; w0 += chunk) {
    const long long nwin = g.windows - w0 < chunk ? g.windows - w0 : chunk;
    // 1. q / k / v slabs, O and the softmax statistics
    e = launch_bf16_chunk(g, ctx, x, Wqkv, bqkv, nullptr, nullptr, table, nullptr, cbase, w0, nwin, st, nullptr,
                          stats);
    if (e != cudaSuccess) return e;
    const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(cbase + bf16_chunk_o_offset(g, nwin));
    const int* rowsrc = reinterpret_cast<const int*>(cbase + bf16_chunk_rows_offset(g, nwin));
    // 2. dO slabs
    e = launch_bf16_dout_slabs(g, ctx, dy, wprojT, zero_bias, dos, rowsrc, w0, nwin, st);
    if (e != cudaSuccess) return e;
    // 3. attention gradients
    BwdArgs ba{};
    ba.g = g;
    ba.ctx = ctx;
    ba.qkv = reinterpret_cast<const __nv_bfloat16*>(cbase);
    ba.dOs = dos;
    ba.o = o;
    ba.stats = stats;
    ba.table = static_cast<const __nv_bfloat16*>(table);
    ba.dqkv = dqkv;
    ba.dtable = dtable;
    ba.win0 = w0;
    ba.nwin = nwin;
    ba.qrows = qrows;
    ba.kvrows = kvrows;
    ba.head_elems = (long long)(qrows + 2 * kvrows) * 32;
    switch (g.win[0]) {
      case 8: e = launch_bwd_attn<BwWin<8>>(ba, st); break;
      case 4: e = launch_bwd_attn<BwWin<4>>(ba, st); break;
      case 2: e = launch_bwd_attn<BwWin<2>>(ba, st); break;
      case 1: e = launch_bwd_attn<BwWin<1>>(ba, st); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    // 4. dX and the parameter gradients
    e = launch_bf16_dx(g, ctx, dqkv, wqkvT, zero_bias, dx, rowsrc, w0, nwin, st);
    if (e != cudaSuccess) return e;
    const long long rows = nwin * g.N;
    // dWqkv = X^T dqkv (X gathered), dbqkv over every slot (padding included);
    // dWproj = O^T dY (dY gathered, zero on padding), dbproj over real slots. On
    // tcgen05 when the C columns and the bias row fit one 128-row tile, else the
    // FP32 sums.
    const bool tc = C + 1 <= 128;
    e = tc ? launch_gram_tc(ctx, rows, C, 3 * C, x, C, rowsrc, dqkv, 3 * C, nullptr, dWqkv, dbqkv, st)
           : launch_gram_bf16(rows, C, 3 * C, x, C, rowsrc, dqkv, 3 * C, nullptr, dWqkv, dbqkv, st);
    if (e != cudaSuccess) return e;
    e = tc ? launch_gram_tc(ctx, rows, C, C, o, C, nullptr, dy, C, rowsrc, dWproj, dbproj, st)
           : launch_gram_bf16(rows, C, C, o, C, nullptr, dy, C, rowsrc, dWproj, dbproj, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace vswin
