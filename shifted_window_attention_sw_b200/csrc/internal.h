// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "geometry.cuh"

namespace vswin {

// Per-launch context: the device error word and the wait limit.
struct KernelCtx {
  int* err;                       // device error word (0 = fine)
  unsigned long long wait_limit;  // ns
  int force_exact;                // test hook: every row through the exact softmax path
};

// Device-side error codes written to the error word.
enum : int {
  kErrWaitLoad = 0x101,
  kErrWaitMma = 0x102,
  kErrWaitSelftest = 0x1FF,
  kErrBounds = 0x201,  // VSWIN_DEBUG_BOUNDS: an index outside its extent (access skipped)
};

// Index check of the gathers and scatters: with VSWIN_DEBUG_BOUNDS, an index
// outside [lo, n) records kErrBounds in the error word and the caller skips
// the access; otherwise every index is taken as valid and nothing is checked.
#ifdef VSWIN_DEBUG_BOUNDS
__device__ __forceinline__ bool index_ok(long long i, long long lo, long long n, int* err) {
  if (i >= lo && i < n) return true;
  atomicCAS(err, 0, kErrBounds);
  return false;
}
#else
__device__ __forceinline__ bool index_ok(long long, long long, long long, int*) { return true; }
#endif

// VSWIN_DEBUG_BOUNDS test hook (vswin_debug_plant_row): the layer slot whose
// row-table entry is overwritten, and the value; slot < 0 when off.
void debug_plant(long long* slot, int* token);

void count_launch(int n = 1);

// Optional per-kernel CUDA-event timing (vswin_profile_enable).
void prof_begin(int kind, cudaStream_t st);
void prof_end(int kind, cudaStream_t st);
enum { kKindQkv = 0, kKindAttn = 1, kKindProj = 2, kKindOther = 3, kKindMlp = 4, kKindAttnBwd = 5, kKinds = 6 };

// fp32 path (simt_path.cu)
cudaError_t launch_f32_forward(const Geom& g, const float* x, const float* Wqkv, const float* bqkv,
                               const float* Wproj, const float* bproj, const float* table, float* out,
                               float* scratch_qkv, float* scratch_o, cudaStream_t st);
size_t f32_scratch_floats(const Geom& g, size_t* qkv_floats, size_t* o_floats);

// fp32 backward (backward_f32.cu): gradients of x, Wqkv, bqkv, Wproj, bproj and
// the table for output gradient dy; scratch of f32_backward_scratch_bytes.
size_t f32_backward_scratch_bytes(const Geom& g);
cudaError_t launch_f32_backward(const Geom& g, const float* x, const float* Wqkv, const float* bqkv,
                                const float* Wproj, const float* bproj, const float* table, const float* dy,
                                float* dx, float* dWqkv, float* dbqkv, float* dWproj, float* dbproj, float* dtable,
                                void* scratch, cudaStream_t st);

cudaError_t launch_index_maps(const Geom& g, int* win_src, int* region, int* bias_idx, cudaStream_t st);

cudaError_t launch_selftest_timeout(const KernelCtx& ctx, cudaStream_t st);

// bf16 path (bf16_path.cu)
bool bf16_window_supported(const Geom& g);
// Scratch for `nwin` windows: QKV slabs then the attention output.
size_t bf16_scratch_bytes(const Geom& g, long long nwin);
// The block's pre-norm and residual fused into the layer: the norm folded into
// the QKV weights (launch_ln_fold fills these buffers once per call) and
// applied per row in the QKV epilogue; x added in the projection epilogue.
struct BlockFuse {
  void* wt;        // [C + 16][3C] bf16: diag(gamma) Wqkv, then the column sums (hi, lo, hi, lo) and zeros
  float* colsum;   // [3C] column sums of wt
  float* bias_ln;  // [3C] bqkv + beta Wqkv
  float eps;
};
cudaError_t launch_ln_fold(const Geom& g, const void* gamma, const void* beta, const void* Wqkv, const void* bqkv,
                           const BlockFuse& f, cudaStream_t st);
// Chunk scratch of the fused block: the layer's plus the per-row norm statistics.
size_t bf16_block_scratch_bytes(const Geom& g, long long nwin);
// One chunk of windows; `fuse` null for the plain layer, else the fused block
// (x is then also the residual, and out may be x itself).
// With Wproj null only the first three steps run (row table, q / k / v slabs,
// attention output o); attn_stats (only for (P,7,7) windows), when given,
// receives each (slot, head) row's softmax reference and sum (exp2 domain).
cudaError_t launch_bf16_chunk(const Geom& g, const KernelCtx& ctx, const void* x, const void* Wqkv,
                              const void* bqkv, const void* Wproj, const void* bproj, const void* table,
                              void* out, void* scratch, long long win0, long long nwin, cudaStream_t st,
                              const BlockFuse* fuse = nullptr, float2* attn_stats = nullptr);
// Chunk scratch of launch_bf16_chunk: q / k / v slabs at 0, the attention
// output o ([nwin * N][C] bf16) and the row table (int per slot) at these offsets.
size_t bf16_chunk_o_offset(const Geom& g, long long nwin);
size_t bf16_chunk_rows_offset(const Geom& g, long long nwin);
// Slab rows of the bf16 path: q rows, k / v rows, and whether keys are stored
// as 8-row lines of 7 keys (slot n at row (n / 7) * 8 + n % 7).
void bf16_slab_rows(const Geom& g, int* qrows, int* kvrows, int* kv8);
// dO slabs for the backward: dy rows gathered through the row table times
// WprojT ([C][C], Wproj transposed), one q-layout slab (Npad rows x 32) per
// (window, head), no bias (zero_bias: C zeros) and no scale.
cudaError_t launch_bf16_dout_slabs(const Geom& g, const KernelCtx& ctx, const void* dy, const void* WprojT,
                                   const void* zero_bias, void* dO, const int* rowsrc, long long win0,
                                   long long nwin, cudaStream_t st);
// dx for the backward: dqkv rows ([nwin * N][3C] bf16) times WqkvT ([3C][C]),
// scattered to the tokens through the row table (padding slots dropped).
cudaError_t launch_bf16_dx(const Geom& g, const KernelCtx& ctx, const void* dqkv, const void* WqkvT,
                           const void* zero_bias, void* dx, const int* rowsrc, long long win0, long long nwin,
                           cudaStream_t st);

// bf16 backward (backward_bf16.cu): gradients of x (bf16) and of Wqkv, bqkv,
// Wproj, bproj and the table (fp32, overwritten) for output gradient dy (bf16),
// windows processed `chunk` at a time in scratch of
// bf16_backward_scratch_bytes(g, chunk).
bool bf16_backward_supported(const Geom& g);
size_t bf16_backward_scratch_bytes(const Geom& g, long long chunk);
cudaError_t launch_bf16_backward(const Geom& g, const KernelCtx& ctx, const void* x, const void* Wqkv,
                                 const void* bqkv, const void* Wproj, const void* table, const void* dy, void* dx,
                                 float* dWqkv, float* dbqkv, float* dWproj, float* dbproj, float* dtable,
                                 void* scratch, long long chunk, cudaStream_t st);
// fp32 sums over rows of bf16 inputs (backward_f32.cu): out[m][n] += sum_r
// A[arow(r)][m] B[brow(r)][n] for m < M, and bias_out[n] += sum_r B[brow(r)][n]
// (rows whose brow < 0 read zeros; arow < 0 reads zeros but still counts for
// the bias). arow(r) = a_src ? a_src[r] : r, likewise brow.
cudaError_t launch_gram_bf16(long long rows, int M, int N, const void* A, long long lda, const int* a_src,
                             const void* B, long long ldb, const int* b_src, float* out, float* bias_out,
                             cudaStream_t st);

// MLP half of a block (mlp_path.cu): out = x + GELU(LN(x) W1 + b1) W2 + b2 for
// M tokens of C channels, one fused persistent kernel. out may be x.
bool mlp_supported(int C, int hidden);
cudaError_t launch_mlp(const KernelCtx& ctx, long long M, int C, int hidden, const void* x, const void* gamma,
                       const void* beta, float eps, const void* W1, const void* b1, const void* W2, const void* b2,
                       void* out, cudaStream_t st);

// Patch merging (merge_path.cu): LN over each 2x2 spatial neighbourhood's 4C
// values, then Wr [4C][2C] (+ br); scratch of patch_merge_scratch_bytes(C)
// holds the folded weights.
bool patch_merge_supported(int C);
size_t patch_merge_scratch_bytes(int C);
cudaError_t launch_patch_merge(const KernelCtx& ctx, int B, int T, int H, int W, int C, const void* x,
                               const void* gamma, const void* beta, float eps, const void* Wr, const void* br,
                               void* out, void* scratch, cudaStream_t st);

}  // namespace vswin
