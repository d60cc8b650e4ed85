/*
 * vswin -- 3D (shifted-)window multi-head self-attention (Video Swin W-MSA /
 * SW-MSA) for NVIDIA B200 (sm_100a). C ABI.
 *
 * The layer ("Video Swin Transformer" summary page, Method steps 4-6, the
 * window_msa pseudocode and eq. 2; the Video Swin code walk-through page,
 * section 1.2, for the op order of WindowAttention3D):
 *
 *   1. zero-pad the token grid (T, H, W) at the high end of each axis to
 *      multiples of the window (P, Mh, Mw);
 *   2. roll the padded grid by -shift on each axis (content moves toward
 *      index 0), so that rolled coordinate r holds original o = (r+s) mod Lp;
 *   3. partition into windows of N = P*Mh*Mw slots, windows (b, wt, wh, ww)
 *      and slots (pt, ph, pw) both row-major;
 *   4. qkv = X Wqkv + bqkv; head h uses columns [h*d, (h+1)*d) of the q, k and
 *      v blocks (d = C / heads);
 *   5. per window and head: softmax(q k^T / sqrt(d) + B) v over the keys that
 *      share the query's region (only when some shift is nonzero); B[i][j] =
 *      bias_table[(dt+P-1)(2Mh-1)(2Mw-1) + (dh+Mh-1)(2Mw-1) + (dw+Mw-1)][h]
 *      with (dt,dh,dw) = slot position of i minus that of j;
 *   6. y = concat_h(o_h) Wproj + bproj;
 *   7. reverse the partition, roll by +shift, drop the padding.
 *
 * Regions: on a shifted axis, rolled coordinate r is in region 0 when
 * r < Lp - w, 1 when r < Lp - s, else 2 (the slices of the last window that
 * were not neighbours before the roll; summary page, Method step 5). Masked
 * pairs are excluded from the softmax. Padded slots are ordinary keys with
 * zero input (k = bk, v = bv).
 *
 * Layouts (all row-major, contiguous, no strides):
 *   x, out       (B, T, H, W, C)           channels last
 *   Wqkv         [C][3C]                   used as x * Wqkv
 *   bqkv         [3C]
 *   Wproj        [C][C]                    used as o * Wproj
 *   bproj        [C]
 *   bias_table   [(2P-1)(2Mh-1)(2Mw-1)][heads]
 *
 * Conventions for every entry point:
 *   * tensor pointers are DEVICE pointers unless the name ends in _host;
 *     the caller owns every buffer; nothing is retained after the call;
 *   * `stream` is a cudaStream_t (NULL = legacy default stream); work is
 *     enqueued on it and the call returns without synchronising (except
 *     vswin_wmsa_forward_host, which synchronises);
 *   * window and shift are host arrays of 3 ints, taken literally (no
 *     clamping; see vswin_clamp_window);
 *   * the return value is a vswin_status; on failure nothing has been
 *     launched and vswin_last_error() describes the cause. Errors raised by
 *     kernels (a bounded wait that gave up) are reported by vswin_poll_error.
 *   * nothing throws across the ABI; the library is thread-safe (the last
 *     error message is thread-local).
 */
#ifndef VSWIN_H_
#define VSWIN_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VSWIN_OK = 0,
  VSWIN_ERR_INVALID_ARG = 1,  /* bad sizes, window/shift, NULL or misaligned or overlapping pointers */
  VSWIN_ERR_UNSUPPORTED = 2,  /* valid layer that this path does not implement (see each entry) */
  VSWIN_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  VSWIN_ERR_TIMEOUT = 4,      /* a kernel's bounded wait gave up (reported by vswin_poll_error) */
  VSWIN_ERR_NO_MEMORY = 5,    /* scratch allocation failed */
  VSWIN_ERR_BOUNDS = 6        /* a build with VSWIN_DEBUG_BOUNDS caught an index out of its extent */
} vswin_status;

/*
 * bf16 layer forward: x, weights, biases, table and out are bf16; products
 * accumulate in fp32 on the tensor cores (tcgen05). Requires d = C/heads = 32,
 * C a multiple of 32, window (P, Mh, Mw) one of the compiled shapes
 * (16,7,7), (8,7,7), (4,7,7), (2,7,7), (1,7,7), (4,4,4), (2,2,2), (1,1,1)
 * (N = P*Mh*Mw up to 784); otherwise VSWIN_ERR_UNSUPPORTED. Pointers must be 16-byte aligned
 * and x must not overlap out.
 * Scratch: stream-ordered allocation on `stream` from a memory pool the
 * library creates per device and keeps (freed scratch is reused by the next
 * call; the pool grows to the largest call's need and is held until exit):
 * about 324 KB per window of 392 slots at C = 96, in chunks of at most 1 GiB
 * (one chunk for the layers here).
 */
int vswin_wmsa_forward(const void* x, int B, int T, int H, int W, int C, int heads,
                       const int* window, const int* shift,
                       const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                       const void* bias_table, void* out, void* stream);

/*
 * bf16 forward of a block's attention half: out = x + layer(LN(x)), the
 * pre-norm and the residual fused into the layer ("Video Swin Transformer"
 * summary page, Method step 3 and eq. 1; code walk-through page, section 1.2:
 * LayerNorm comes before F.pad, so padded slots are zero tokens for the layer,
 * and the shortcut is added after the window reverse).
 *   LN(x) = (x - mean) / sqrt(var + ln_eps) * ln_gamma + ln_beta per token over
 *   its C channels, var the biased variance (torch.nn.LayerNorm; its default
 *   eps is 1e-5).
 * ln_gamma, ln_beta: bf16 [C], device, 2-byte aligned; ln_eps finite, >= 0.
 * Every other argument, layout and requirement is that of vswin_wmsa_forward,
 * except that out may be x itself (in place); partial overlap is refused.
 * Arithmetic: the norm is folded into the weights once per call
 * (Wt = bf16(diag(gamma) Wqkv), its fp32 column sums, bqkv + beta Wqkv) and
 * applied per row in the QKV epilogue as rstd * (x Wt - mean * colsum(Wt)) +
 * (bqkv + beta Wqkv), with per-token mean and rstd in fp32; the residual is
 * added to the fp32 projection before the one rounding to bf16. Tokens whose
 * variance overflows fp32 (|x| above ~1e19) are out of range. Scratch: the
 * layer's plus 8 bytes per window slot and C*3C*2 + 24*C bytes for the folded
 * weights, from the same pool.
 */
int vswin_block_msa_forward(const void* x, int B, int T, int H, int W, int C, int heads,
                            const int* window, const int* shift,
                            const void* ln_gamma, const void* ln_beta, float ln_eps,
                            const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                            const void* bias_table, void* out, void* stream);

/*
 * bf16 forward of a block's MLP half ("Video Swin Transformer" summary page,
 * Method step 3 and eq. 1: layer norm, a two-layer MLP with GELU, residual
 * add; the code walk-through page, section 1.2, names nn.LayerNorm):
 *   out = x + GELU(LN(x) W1 + b1) W2 + b2       for every token of x
 * x, out       (B, T, H, W, C) bf16, channels last; out may be x (in place),
 *              partial overlap is refused
 * ln_gamma, ln_beta, ln_eps   as for vswin_block_msa_forward
 * W1 [C][hidden], b1 [hidden], W2 [hidden][C], b2 [C]   bf16, row-major
 * GELU is the erf form x * Phi(x) (torch.nn.GELU's default); the kernel
 * evaluates it through a fitted tanh form on the hardware tanh, within 1e-3
 * |x| of the erf form. Products accumulate in fp32 on the tensor cores; the
 * normalised tokens and the hidden activations are rounded to bf16 as MMA
 * operands and never leave the SM; the output is rounded once.
 * Requires C a multiple of 32 up to 128 and hidden a multiple of 64 that
 * splits into at most 8 hidden chunks of 128 (or 64) columns whose weights fit
 * in shared memory -- hidden 4C for C = 32 .. 128 does -- else
 * VSWIN_ERR_UNSUPPORTED; x, out, W1, W2 16-byte aligned, the vectors 2-byte
 * aligned; B*T*H*W < 2^31. No scratch memory.
 */
int vswin_mlp_forward(const void* x, int B, int T, int H, int W, int C, int hidden,
                      const void* ln_gamma, const void* ln_beta, float ln_eps,
                      const void* W1, const void* b1, const void* W2, const void* b2,
                      void* out, void* stream);

/*
 * bf16 forward of one whole Video Swin block ("Video Swin Transformer"
 * summary page, Method step 3 and eq. 1):
 *   z   = x + layer(LN1(x))               vswin_block_msa_forward
 *   out = z + GELU(LN2(z) W1 + b1) W2 + b2 vswin_mlp_forward, in place on out
 * The arguments are those of the two entry points (one ln_eps for both
 * norms); every one of them is checked before anything is launched, and the
 * requirements of both apply. out may be x. Scratch: that of
 * vswin_block_msa_forward.
 */
int vswin_block_forward(const void* x, int B, int T, int H, int W, int C, int heads,
                        const int* window, const int* shift,
                        const void* ln1_gamma, const void* ln1_beta,
                        const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                        const void* bias_table,
                        const void* ln2_gamma, const void* ln2_beta, int hidden,
                        const void* W1, const void* b1, const void* W2, const void* b2,
                        float ln_eps, void* out, void* stream);

/*
 * bf16 patch merging between stages ("Video Swin Transformer" summary page,
 * Method step 2: each 2x2 group of spatial neighbours, 4C values, projected
 * to 2C by a linear layer, no temporal merging; code walk-through page,
 * section 1.2: PatchMerging is a LayerNorm over the 4C values, then
 * Linear(4C, 2C)):
 *   out[b,t,i,j] = LN(cat(x[b,t,2i,2j], x[b,t,2i+1,2j], x[b,t,2i,2j+1],
 *                         x[b,t,2i+1,2j+1])) Wr + br
 * The pages fix neither the order of the four neighbours in the 4C vector
 * nor odd extents: the order is the one written above (channels
 * [(2 dw + dh) C, (2 dw + dh + 1) C) hold neighbour (dh, dw)), and an odd H
 * or W is zero-padded at the high end.
 * x        (B, T, H, W, C) bf16, channels last, 16-byte aligned
 * ln_gamma, ln_beta  [4C] bf16; ln_eps finite, >= 0
 * Wr       [4C][2C] bf16 row-major, 16-byte aligned; br [2C] bf16 or NULL
 * out      (B, T, ceil(H/2), ceil(W/2), 2C) bf16, 16-byte aligned, must not
 *          overlap x
 * Requires C a multiple of 32 (else VSWIN_ERR_UNSUPPORTED). The norm is
 * folded into the weights (bf16(diag(gamma) Wr), its fp32 column sums,
 * beta Wr + br) and applied per row in the epilogue with fp32 statistics of
 * the gathered bf16 values. Scratch: 16 C^2 + 16 C bytes (the folded
 * weights), from the library's pool.
 */
int vswin_patch_merge_forward(const void* x, int B, int T, int H, int W, int C,
                              const void* ln_gamma, const void* ln_beta, float ln_eps,
                              const void* Wr, const void* br, void* out, void* stream);

/*
 * fp32 layer forward (plain FP32 FMA arithmetic, no tensor cores): every
 * tensor is float. The same layer as vswin_wmsa_forward, steps 1-7 above
 * ("Video Swin Transformer" summary page, Method steps 4-6 and eq. 2), with
 * every product and sum in fp32 and the softmax as max, exp, sum, divide.
 * Any d; N <= 4096. Pointers 4-byte aligned; x must not overlap out.
 * Scratch: stream-ordered, from the library's pool (see above).
 */
int vswin_wmsa_forward_f32(const void* x, int B, int T, int H, int W, int C, int heads,
                           const int* window, const int* shift,
                           const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                           const void* bias_table, void* out, void* stream);

/*
 * fp32 backward of the layer (plain FP32 FMA arithmetic, no tensor cores):
 * for the output gradient dy (same layout as out), writes dx (layout of x),
 * dWqkv [C][3C], dbqkv [3C], dWproj [C][C], dbproj [C] and dtable (layout of
 * bias_table) -- the chain rule back through the layer's steps above
 * ("Video Swin Transformer" summary page, Method steps 4-6 and eq. 2; the
 * softmax gradient dS = P * (dP - rowsum(dP * P)), zero on masked pairs;
 * padded slots are keys with zero input, so they reach dbqkv but not dx; the
 * table gradient of head h sums dS over every pair that reads that row).
 * Every tensor is float, 4-byte aligned, on the device; the six gradient
 * buffers are overwritten (not accumulated) and may overlap neither one
 * another nor any input. The forward is recomputed inside the call. Any head
 * width; N <= 4096 and (2N + 2d) * 4 bytes and 12C bytes within 48 KB,
 * otherwise VSWIN_ERR_UNSUPPORTED. Results are not bitwise deterministic
 * (the table and weight gradients are summed with atomics). Scratch: from
 * the library's pool, about (13C + 3 heads) * 4 bytes per window slot plus
 * the forward's output.
 */
int vswin_wmsa_backward_f32(const void* x, int B, int T, int H, int W, int C, int heads,
                            const int* window, const int* shift,
                            const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                            const void* bias_table, const void* dy, void* dx, void* dWqkv, void* dbqkv,
                            void* dWproj, void* dbproj, void* dtable, void* stream);

/*
 * bf16 backward of the layer on the tensor cores ("Video Swin Transformer"
 * summary page, Method steps 4-6 and eq. 2, differentiated as for
 * vswin_wmsa_backward_f32): x, dy, dx (layout of x), Wqkv, bqkv, Wproj,
 * bproj and bias_table are bf16 as in vswin_wmsa_forward; dWqkv [C][3C],
 * dbqkv [3C], dWproj [C][C], dbproj [C] and dtable (layout of bias_table) are
 * float, overwritten (not accumulated). The forward's first three steps are
 * recomputed (q, k, v, the attention output and each row's softmax
 * reference and sum), then dO = dy Wproj^T, the attention gradients per
 * (window, head) on tcgen05 (S and dP, P and dS rebuilt in registers, dq,
 * dk, dv as tensor-core products, the table gradient summed per CTA), dx =
 * dqkv Wqkv^T scattered to the tokens, and the weight and bias gradients as
 * fp32 sums. Products take bf16 operands with fp32 accumulation; P, dS and
 * dqkv are rounded to bf16 on the way (gradient error about 1e-2 relative).
 * Requires head width 32, C % 32 == 0 and a (P,7,7) window with P in
 * {1, 2, 4, 8}, else VSWIN_ERR_UNSUPPORTED (vswin_wmsa_backward_f32 covers
 * every shape). x, dy and dx 16-byte aligned; bf16 vectors, weights and
 * table 2-byte aligned; float outputs 4-byte aligned; outputs may overlap
 * neither one another nor any input. Not bitwise deterministic (atomics in
 * the table and weight gradients). Scratch: from the library's pool, about
 * (5 C + 16 heads) * 2 bytes per window slot plus the forward's chunk scratch.
 */
int vswin_wmsa_backward(const void* x, int B, int T, int H, int W, int C, int heads,
                        const int* window, const int* shift,
                        const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                        const void* bias_table, const void* dy, void* dx, void* dWqkv, void* dbqkv,
                        void* dWproj, void* dbproj, void* dtable, void* stream);

/*
 * bf16 layer forward with the activations in HOST memory: copies x_host to
 * the device, runs the layer, copies the result to out_host and synchronises
 * `stream`. Weights, biases and table are device pointers (they stay resident
 * between calls). The batch goes through in up to four groups of clips (the
 * windows of a clip read only that clip), so that the copy in of one group,
 * the layer on the previous one and the copy out of the one before overlap:
 * the copies run on two streams of the library's (created once per device,
 * non-blocking), ordered against `stream` with events. Page-locked host
 * buffers give asynchronous copies; pageable ones work but are slower. Device
 * buffers for x and out come from the library's stream-ordered pool (see
 * vswin_wmsa_forward). Results are bitwise those of vswin_wmsa_forward.
 */
int vswin_wmsa_forward_host(const void* x_host, int B, int T, int H, int W, int C, int heads,
                            const int* window, const int* shift,
                            const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                            const void* bias_table, void* out_host, void* stream);

/*
 * bf16 layer forward that allocates nothing. No passage of the method's pages
 * corresponds to this: it is an interface for callers that cannot allocate
 * device memory while they run the layer -- hosts that must stay inside
 * memory they reserved beforehand, code that must not risk the device-wide
 * synchronisation an allocation can cause, or processes whose device memory
 * belongs to another allocator. Arguments, layouts, requirements and results
 * are those of vswin_wmsa_forward; only the scratch differs.
 *   * Scratch is one statically sized 32 MiB device array inside this library
 *     (every GPU that loads the library holds it until the process exits).
 *     Windows pass through it in equal chunks, so any batch size works; a
 *     layer whose single window needs more than 32 MiB of scratch is refused
 *     with VSWIN_ERR_UNSUPPORTED and a message giving both sizes (the layers
 *     in this repository need 0.3 MB to 3.3 MB per window).
 *   * No cudaMalloc / cudaMallocAsync / cudaFree or other allocating call is
 *     made. The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   * All calls share the one array and it keeps the last call's contents.
 *     Calls whose kernels overlap on the GPU (different streams, or different
 *     host threads without ordering) race on it and give wrong results: order
 *     them on one stream or synchronise between them. Nothing in the array
 *     needs to start at zero.
 */
int vswin_wmsa_forward_noalloc(const void* x, int B, int T, int H, int W, int C, int heads,
                               const int* window, const int* shift,
                               const void* Wqkv, const void* bqkv, const void* Wproj, const void* bproj,
                               const void* bias_table, void* out, void* stream);

/*
 * Index maps of the layer, written to caller-allocated device int32 buffers
 * (any of them may be NULL to skip it). They spell out steps 1-3 and 5 above:
 * the padding and cyclic shift of the token grid and the window partition
 * ("Video Swin Transformer" summary page, Method steps 4-5 and the window_msa
 * pseudocode), the regions of the shifted-window mask (Method step 5) and the
 * relative-position index of the bias table (Method step 8):
 *   win_src [B*nW*N]  flat source token b*T*H*W + (t*H + h)*W + w of each
 *                     window slot, or -1 for a padding slot;
 *   region  [nW*N]    9*rt + 3*rh + rw of each slot (0 when unshifted);
 *   bias_idx[N*N]     table row used by query slot i and key slot j.
 * nW = prod(ceil(L/w)), N = P*Mh*Mw.
 */
int vswin_wmsa_index_maps(int B, int T, int H, int W, const int* window, const int* shift,
                          int* win_src, int* region, int* bias_idx, void* stream);

/*
 * Host helper: the official code's clamp ("Video Swin Transformer" summary
 * page, "Paper vs code": a window dimension is set to the input size, with
 * shift 0, when the input is not larger than the window). Writes the clamped
 * window and shift (3 ints each).
 */
int vswin_clamp_window(int T, int H, int W, const int* window_in, const int* shift_in,
                       int* window_out, int* shift_out);

/* Thread-local description of the last non-OK status returned on this thread. */
const char* vswin_last_error(void);

/*
 * Synchronises `stream`, then returns and clears the device error word:
 * VSWIN_OK, or VSWIN_ERR_TIMEOUT if a kernel's bounded wait gave up since the
 * last poll, VSWIN_ERR_BOUNDS if a build with VSWIN_DEBUG_BOUNDS caught an
 * index out of its extent (the access was skipped), or VSWIN_ERR_CUDA if
 * synchronisation failed.
 */
int vswin_poll_error(void* stream);

/* Number of kernels this library has launched in this process (all devices). */
unsigned long long vswin_launch_count(void);

/* Limit, in nanoseconds, of every bounded wait in the kernels (default 1e9). */
void vswin_set_wait_limit_ns(unsigned long long ns);

/*
 * Test hook for the bf16 (P,7,7) attention kernel. Its softmax normally uses
 * one reference per query row, |q_i| * max_j |k_j| + max(bias) + 1 (an upper
 * bound of the row's scores), and recomputes a row exactly -- two-pass softmax
 * on the CUDA cores -- only when the row's sum underflows below 2^-100 (logits
 * spanning more than ~69 natural-log units). on != 0 sends every row through
 * that exact path, so that tests can check it; 0 restores the normal rule.
 */
void vswin_set_exact_softmax(int on);

/*
 * Test hook: host-side fault injection. kind VSWIN_INJECT_CUDA makes the next
 * `count` entry calls fail as if a CUDA runtime call had failed (status
 * VSWIN_ERR_CUDA, message naming the injection) before they touch the device;
 * VSWIN_INJECT_ALLOC makes the next `count` scratch allocations fail (status
 * VSWIN_ERR_NO_MEMORY) before anything is launched. count 0 clears the kind.
 * No kernel runs and nothing is allocated for an injected failure. Returns
 * VSWIN_OK, or VSWIN_ERR_INVALID_ARG for an unknown kind or count < 0.
 */
enum { VSWIN_INJECT_CUDA = 1, VSWIN_INJECT_ALLOC = 2 };
int vswin_test_inject_failure(int kind, int count);

/*
 * Test hook of builds with VSWIN_DEBUG_BOUNDS (index checks in the gathers and
 * scatters: an index outside its extent sets the error word and the access is
 * skipped). Every following bf16 layer forward overwrites its row table entry
 * for window slot `slot` (counted over the whole layer) with `token`, after the
 * table is computed; slot < 0 turns this off. In other builds it returns
 * VSWIN_ERR_UNSUPPORTED and changes nothing.
 */
int vswin_debug_plant_row(long long slot, int token);

/* 1 in a build with VSWIN_DEBUG_BOUNDS, else 0. */
int vswin_debug_bounds_enabled(void);

/*
 * Self-test of the timeout path: launches one kernel that waits, with the
 * current limit, on a barrier that nothing completes. It must give up and set
 * the error word, so a following vswin_poll_error returns VSWIN_ERR_TIMEOUT.
 */
int vswin_selftest_timeout(void* stream);

/*
 * Per-kernel timing for benchmarks. While enabled, every kernel launch of the
 * library is bracketed by two CUDA events recorded on its launch stream.
 * vswin_profile_collect waits for the recorded events, adds their elapsed
 * times per kernel kind into ms[kind] and launch counts into launches[kind]
 * (arrays of nkinds entries, kinds VSWIN_KERNEL_*), then forgets them.
 */
enum {
  VSWIN_KERNEL_QKV_GEMM = 0,   /* gather + QKV projection (bf16) */
  VSWIN_KERNEL_ATTENTION = 1,  /* window attention (bf16) */
  VSWIN_KERNEL_PROJ_GEMM = 2,  /* output projection + scatter (bf16) */
  VSWIN_KERNEL_OTHER = 3,      /* fp32 path, index maps, self-test */
  VSWIN_KERNEL_MLP = 4,        /* fused MLP half of a block (bf16) */
  VSWIN_KERNEL_ATTN_BWD = 5,   /* attention gradients of the bf16 backward */
  VSWIN_KERNEL_KINDS = 6
};
int vswin_profile_enable(int on);
int vswin_profile_collect(double* ms, unsigned long long* launches, int nkinds);

/* Library version, major*10000 + minor*100 + patch. */
int vswin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSWIN_H_ */
