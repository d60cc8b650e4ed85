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
};

void count_launch(int n = 1);

// Optional per-kernel CUDA-event timing (vswin_profile_enable).
void prof_begin(int kind, cudaStream_t st);
void prof_end(int kind, cudaStream_t st);
enum { kKindQkv = 0, kKindAttn = 1, kKindProj = 2, kKindOther = 3, kKindMlp = 4, kKinds = 5 };

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
  void* wt;        // [C][3C] bf16: diag(gamma) Wqkv
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
cudaError_t launch_bf16_chunk(const Geom& g, const KernelCtx& ctx, const void* x, const void* Wqkv,
                              const void* bqkv, const void* Wproj, const void* bproj, const void* table,
                              void* out, void* scratch, long long win0, long long nwin, cudaStream_t st,
                              const BlockFuse* fuse = nullptr);

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
