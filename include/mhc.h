/*
 * mhc.h -- C ABI of the B200 (sm_100a) mHC layer library, libmhc.so.
 *
 * mHC (manifold-constrained hyper-connections) keeps, for every token, an
 * n-stream residual buffer x in R^{n x C} and per layer computes
 *
 *     h_in   = H_pre x                          (layer input, R^C)
 *     x_next = H_res x + H_post^T F(h_in)       (residual update, R^{n x C})
 *
 * with per-token mappings built from the token's own stream buffer:
 *
 *     r      = sqrt(mean_k x_k^2 + eps)             over all n*C entries
 *     z      = alpha * (x / r) . phi + b             phi in R^{nC x (n^2+2n)}
 *     H_pre  = sigmoid(z[0:n])                       non-negative input map
 *     H_post = 2 sigmoid(z[n:2n])                    non-negative output map
 *     H_res  = SinkhornKnopp_t(exp(z[2n:]))          ~ doubly stochastic
 *
 * Sources, by page and section:
 *   "DeepSeek-Forscher ..." (chatgpz.de feed), section "Von
 *   Residualverbindungen zu Hyperverbindungen": the n-stream buffer, the
 *   three mappings and the update equation;  section "Vielfaeltig
 *   eingeschraenkte Hyperverbindungen": H_res projected onto the doubly
 *   stochastic (Birkhoff) matrices with Sinkhorn-Knopp, 20 iterations, and
 *   non-negative input/output maps;  section "Systemarbeit und
 *   Schulungsaufwand": fused RMSNorm/projection/gating kernels and
 *   recompute in the backward pass.
 *   reportify.cn mHC summary, paragraphs [10], [12], [15]-[21]: the same
 *   constraint, t_max = 20, the reordered RMSNorm, the unified operator, the
 *   Sinkhorn iterations and their custom backward in one operator, the
 *   mapping application fused with the residual merge, and recompute.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers that the caller allocates, owns
 *     and keeps alive until the work on `stream` has finished.  The library
 *     allocates nothing; kernels that need scratch take a caller-provided
 *     workspace whose size is returned by the matching *_workspace_size().
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Calls keep no global state, never synchronise and
 *     never throw.  Host-side argument errors are returned before anything
 *     is launched.
 *   - Layouts are row-major, channel (C) fastest:
 *       x, grad_x_next, grad_x          [T][n][C]   (I/O dtype)
 *       h_in, f_out, grad_h_in, grad_f_out [T][C]   (I/O dtype)
 *       phi, grad_phi                   [n*C][n*n+2n]  float32
 *       b, grad_b                       [n*n+2n]       float32
 *       alpha, grad_alpha               [1]            float32 (device scalar)
 *       H_pre, H_post                   [T][n]         float32
 *       H_res                           [T][n][n]      float32
 *     Token t's stream buffer is flattened as k = i*C + c.  Logit column m of
 *     phi/b is ordered [pre 0..n-1 | post n..2n-1 | res 2n + i*n + j], and
 *     H_res[i][j] weights stream j into output stream i.
 *   - Pointer alignment: every array pointer must be 16-byte aligned
 *     (MHC_ERR_INVALID_ARG otherwise).
 *   - dev_status (optional, may be NULL): a device int the kernels set to a
 *     non-zero mhc_status when they detect a condition at run time
 *     (MHC_ERR_NONFINITE when an RMS value or a logit is not finite;
 *     MHC_ERR_TIMEOUT when a bounded device-side wait ran out, see
 *     mhc_params.wait_ns).  The library only ever writes error codes into it,
 *     never clears it; the caller zeroes it and reads it after synchronising.
 */
#ifndef MHC_H_
#define MHC_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MHC_API __attribute__((visibility("default")))
#else
#define MHC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle; binary-compatible with cudaStream_t. */
typedef struct CUstream_st *mhc_stream_t;

typedef enum mhc_status {
  MHC_OK = 0,
  MHC_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, t_max < 0 */
  MHC_ERR_UNSUPPORTED = 2,  /* n or dtype not built into this library          */
  MHC_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed            */
  MHC_ERR_NONFINITE = 4,    /* (device status) non-finite RMS or logit seen    */
  MHC_ERR_TIMEOUT = 5,      /* (device status) a bounded wait gave up          */
  MHC_ERR_WORKSPACE = 6     /* workspace missing or smaller than required      */
} mhc_status;

typedef enum mhc_dtype {
  MHC_DTYPE_F32 = 0,   /* float32 I/O tensors, float32 arithmetic              */
  MHC_DTYPE_BF16 = 1   /* bfloat16 I/O tensors, float32 accumulation; the phi
                          projection runs on the tensor cores (bf16 operands)  */
} mhc_dtype;

/* Problem description shared by mhc_pre / mhc_post / mhc_backward. */
typedef struct mhc_params {
  int32_t n;      /* streams; the library supports n in {1, 2, 4, 8, 16}; bf16
                     with n = 4, 8 or 16 runs tensor-core kernels (n = 16 with
                     its own CUDA-core epilogues, 288 logits per token), fp32
                     and n <= 2 the CUDA-core kernels; mhc_backward_noalloc
                     takes n <= 8 and runs the CUDA-core kernels             */
  int32_t t_max;  /* Sinkhorn-Knopp iterations (row then column pass), >= 0   */
  int64_t T;      /* tokens, 1 <= T <= 2^31 - 257 (32-bit tile coordinates;
                     bf16 with n >= 8: T * n <= 2^31 - 257)                  */
  int64_t C;      /* channels per stream, >= 8 and a multiple of 8            */
  float eps;      /* RMS epsilon added to the mean square, >= 0               */
  int32_t dtype;  /* mhc_dtype of x, f_out, h_in, x_next and the activation
                     gradients                                                */
  int32_t alpha_groups; /* 0 or 1: one alpha scales all n^2+2n logits;
                           3: alpha = (alpha_pre, alpha_post, alpha_res), one
                           scale per logit group, and grad_alpha has 3 entries */
  int64_t wait_ns;  /* limit, in ns, of every device-side wait of the
                       tensor-core kernels on another warp's or the copy
                       engine's progress; 0 = the default of 2 s.  When a wait
                       runs out the kernel writes MHC_ERR_TIMEOUT to dev_status,
                       finishes the copies and MMAs it already issued, frees
                       its tensor memory and returns; the outputs of that call
                       are undefined, and later calls are unaffected.  A small
                       positive value makes the waits give up on purpose (how
                       the timeout path is tested).  Kernels without such waits
                       ignore it.  Must be >= 0.                               */
} mhc_params;

/* Library version, (major << 16) | minor. */
MHC_API int mhc_version(void);

/* Human-readable text for every mhc_status value (never NULL). */
MHC_API const char *mhc_status_string(int status);

/* Bytes of workspace mhc_pre needs for these params (0 = none). */
MHC_API size_t mhc_pre_workspace_size(const mhc_params *p);

/*
 * mhc_pre -- the "pre" half of an mHC layer for T tokens (sources: the
 * update equation and the mapping definitions above; the fused
 * RMS/projection/gating operator of the "Systemarbeit" section and
 * reportify.cn [17]-[18]; Sinkhorn-Knopp with t_max iterations, [16]).
 *
 *   in : x [T][n][C] (dtype), phi [nC][n^2+2n], b [n^2+2n], alpha [1 or 3]
 *   out: h_in [T][C] (dtype) = sum_i H_pre[i] x[i][:]
 *        H_pre [T][n], H_post [T][n], H_res [T][n][n]   (float32)
 *   workspace: mhc_pre_workspace_size(p) bytes (may be NULL when that is 0).
 * Errors: MHC_ERR_INVALID_ARG, MHC_ERR_UNSUPPORTED, MHC_ERR_WORKSPACE,
 * MHC_ERR_CUDA.  Outputs are undefined when an error is returned.
 */
MHC_API mhc_status mhc_pre(const mhc_params *p, const void *x, const float *phi, const float *b,
                   const float *alpha, void *h_in, float *H_pre, float *H_post, float *H_res,
                   void *workspace, size_t workspace_bytes, int *dev_status,
                   mhc_stream_t stream);

/*
 * mhc_post -- the residual merge (source: the update equation
 * X_{l+1} = H_res X_l + H_post^T F(.), and reportify.cn [20]: application
 * of the output map fused with the residual merge).
 *
 *   in : x [T][n][C], f_out [T][C] (dtype), H_post [T][n], H_res [T][n][n]
 *   out: x_next [T][n][C] (dtype),
 *        x_next[i][c] = sum_j H_res[i][j] x[j][c] + H_post[i] f_out[c]
 * x_next must not alias x or f_out.
 */
MHC_API mhc_status mhc_post(const mhc_params *p, const void *x, const void *f_out,
                            const float *H_post, const float *H_res, void *x_next,
                            int *dev_status, mhc_stream_t stream);

/* Bytes of workspace mhc_backward needs for these params. */
MHC_API size_t mhc_backward_workspace_size(const mhc_params *p);

/*
 * mhc_backward -- gradients of pre+post for T tokens, with the mapping
 * recomputed from (x, phi, b, alpha) rather than stored (sources: the
 * recompute bullet of the "Systemarbeit" section; reportify.cn [19] custom
 * Sinkhorn backward, [21] recompute).  The differentiated scalar is
 *   L = sum grad_x_next . x_next + sum grad_h_in . h_in
 * i.e. grad_x_next = dL/dx_next and grad_h_in = dL/dh_in are the upstream
 * gradients of the two outputs, and f_out is the value F produced.
 *
 *   in : x [T][n][C], phi, b, alpha, f_out [T][C], grad_x_next [T][n][C],
 *        grad_h_in [T][C]
 *   out: grad_x [T][n][C] (dtype), grad_f_out [T][C] (dtype),
 *        grad_phi [nC][n^2+2n], grad_b [n^2+2n], grad_alpha [1 or 3]   (float32)
 * grad_phi / grad_b / grad_alpha are OVERWRITTEN (not accumulated) with sums
 * over the T tokens taken in a fixed order: repeated calls give identical
 * bits.  workspace: at least mhc_backward_workspace_size(p) bytes, 256-byte
 * aligned; its contents on entry do not matter.
 */
MHC_API mhc_status mhc_backward(const mhc_params *p, const void *x, const float *phi,
                                const float *b, const float *alpha, const void *f_out,
                                const void *grad_x_next, const void *grad_h_in, void *grad_x,
                                float *grad_phi, float *grad_b, float *grad_alpha,
                                void *grad_f_out, void *workspace, size_t workspace_bytes,
                                int *dev_status, mhc_stream_t stream);

/*
 * mhc_backward_map / mhc_backward_apply -- the two phases mhc_backward runs,
 * for callers that schedule them separately (both on the same workspace,
 * map first; nothing else may touch the workspace in between).
 *
 * mhc_backward_map: recomputes the mapping and reduces the per-token
 *   C-contractions <grad_h_in, x_i>, <grad_x_next_i, f_out>,
 *   <grad_x_next_i, x_j>; runs the Sinkhorn adjoint and the gate derivatives
 *   (reportify.cn [19]); writes per-token coefficient records and one
 *   partial-sum record of dz and dz . y per mapping CTA into the workspace.
 * mhc_backward_apply: from those records writes grad_x, grad_f_out and
 *   grad_phi (every row of grad_phi summed over all T tokens) and finishes
 *   grad_b and grad_alpha; all sums in a fixed order.  It reads the records
 *   and also uses the rest of the workspace as its own scratch (the const
 *   qualifier states that the records are only read).
 * Arguments, layouts and errors are those of mhc_backward.
 */
MHC_API mhc_status mhc_backward_map(const mhc_params *p, const void *x, const float *phi,
                                    const float *b, const float *alpha, const void *f_out,
                                    const void *grad_x_next, const void *grad_h_in,
                                    void *workspace, size_t workspace_bytes, int *dev_status,
                                    mhc_stream_t stream);
MHC_API mhc_status mhc_backward_apply(const mhc_params *p, const void *x, const float *phi,
                                      const void *grad_x_next, const void *grad_h_in,
                                      void *grad_x, float *grad_phi, float *grad_b,
                                      float *grad_alpha, void *grad_f_out, const void *workspace,
                                      size_t workspace_bytes, int *dev_status,
                                      mhc_stream_t stream);

/*
 * Cross-layer fusion of the forward (sources: reportify.cn [18], the unified
 * operator, and [20], the output map applied together with the residual
 * merge).  In a stack, layer l's post merge writes x_{l+1}, which layer l+1's
 * mapping reads back at once; mhc_post_fused does both in one pass over the
 * stream buffer, so the forward of a layer costs one read of x for h_in and
 * one pass for the merge:
 *
 *   mhc_post_fused(x_l, f_out_l, H_post_l, H_res_l, phi_{l+1}, b_{l+1}, alpha_{l+1})
 *       -> x_{l+1}, H_pre_{l+1}, H_post_{l+1}, H_res_{l+1}
 *   mhc_layer_input(x_{l+1}, H_pre_{l+1}) -> h_in_{l+1}
 *
 * mhc_post_fused -- x_next exactly as mhc_post writes it, and layer l+1's maps
 *   exactly as mhc_pre would compute them from that x_next (the mapping reads
 *   the stored, dtype-rounded x_next).  p->t_max and p->eps are layer l+1's.
 *   phi_next [nC][n^2+2n], b_next, alpha_next as in mhc_pre.  workspace:
 *   mhc_post_fused_workspace_size(p) bytes (may be NULL when that is 0).
 *   x_next must not alias x or f_out.
 * mhc_layer_input -- h_in [T][C] = sum_i H_pre[i] x[i][:] alone (the second
 *   half of mhc_pre).
 * Errors: as mhc_pre.
 */
MHC_API size_t mhc_post_fused_workspace_size(const mhc_params *p);
MHC_API mhc_status mhc_post_fused(const mhc_params *p, const void *x, const void *f_out,
                                  const float *H_post, const float *H_res, const float *phi_next,
                                  const float *b_next, const float *alpha_next, void *x_next,
                                  float *H_pre_next, float *H_post_next, float *H_res_next,
                                  void *workspace, size_t workspace_bytes, int *dev_status,
                                  mhc_stream_t stream);
MHC_API mhc_status mhc_layer_input(const mhc_params *p, const void *x, const float *H_pre,
                                   void *h_in, int *dev_status, mhc_stream_t stream);

/*
 * The layer backward in training order, split around F's backward (sources:
 * the recompute bullet of the "Systemarbeit" section; reportify.cn [20]-[21]).
 * In training, grad_h_in is only known after F's backward, which needs
 * grad_f_out first:
 *
 *   mhc_post_backward(x, f_out, H_post, grad_x_next) -> grad_f_out, red
 *   F's backward (caller)                            -> grad_h_in
 *   mhc_pre_backward(x, phi, b, alpha, grad_x_next, grad_h_in, red)
 *                                                    -> grad_x, grad_phi, grad_b, grad_alpha
 *
 * Together they give exactly what mhc_backward gives for the same
 * (grad_x_next, grad_h_in).
 *
 * mhc_post_backward -- the reverse of the post merge alone, with the
 *   forward's H_post [T][n] (float32, as mhc_pre wrote it):
 *     grad_f_out[c] = sum_i H_post[i] grad_x_next[i][c]        [T][C] (dtype)
 *     red = [ <grad_x_next_i, x_j> (row-major i, j) | <grad_x_next_i, f_out> ]
 *                                                    [T][n*n + n] float32
 *   red carries the derivatives of L with respect to H_res and H_post; the
 *   per-token sums are taken in a fixed order.  grad_f_out must not alias an
 *   input.  No workspace.
 * mhc_pre_backward -- recomputes the mapping from (x, phi, b, alpha), takes
 *   <grad_h_in, x_i> itself and the rest of the mapping's upstream gradient
 *   from red, and writes grad_x [T][n][C] (dtype) and OVERWRITES grad_phi,
 *   grad_b, grad_alpha (float32, fixed-order sums over the T tokens).
 *   workspace: at least mhc_pre_backward_workspace_size(p) bytes, 256-byte
 *   aligned; its contents on entry do not matter.
 * Errors: as mhc_backward (red must be 16-byte aligned like every pointer).
 */
MHC_API mhc_status mhc_post_backward(const mhc_params *p, const void *x, const void *f_out,
                                     const float *H_post, const void *grad_x_next,
                                     void *grad_f_out, float *red, int *dev_status,
                                     mhc_stream_t stream);
MHC_API size_t mhc_pre_backward_workspace_size(const mhc_params *p);
MHC_API mhc_status mhc_pre_backward(const mhc_params *p, const void *x, const float *phi,
                                    const float *b, const float *alpha, const void *grad_x_next,
                                    const void *grad_h_in, const float *red, void *grad_x,
                                    float *grad_phi, float *grad_b, float *grad_alpha,
                                    void *workspace, size_t workspace_bytes, int *dev_status,
                                    mhc_stream_t stream);

/*
 * mhc_backward_noalloc -- mhc_backward for callers that cannot allocate
 * device memory where they run the backward: runtimes that plan every device
 * buffer at start-up and forbid allocation afterwards, plugins that a host
 * framework hands only their input and output buffers, or processes whose
 * framework allocator already holds the whole device (cudaMalloc can also
 * synchronise the device and has no latency bound).  The pages have no
 * counterpart: this is a deployment variant of mhc_backward, not part of the
 * method.
 *
 * Arguments, layouts, results and errors are those of mhc_backward, minus
 * the workspace, and n = 16 is not taken (MHC_ERR_UNSUPPORTED).  The scratch
 * is a library-owned device array of MHC_NOALLOC_SCRATCH_BYTES that every
 * GPU loading this library holds until the process exits.  The call runs the
 * CUDA-core kernels, whose scratch is a per-token record (n = 4: 208 bytes)
 * and a partial sum per 64 tokens; a problem whose scratch exceeds
 * MHC_NOALLOC_SCRATCH_BYTES is rejected with MHC_ERR_WORKSPACE before any
 * launch (n = 4: up to about 20,000 tokens per call).  Every call looks up
 * the array's device address (cudaGetSymbolAddress) on the current device;
 * nothing is cached, so calls made after a device reset use the array of the
 * new context.  The first call on a device may load the module: make it
 * before any stream capture.  All calls share the one array and it keeps the
 * last call's contents (nothing in it needs to start at zero): calls whose
 * work can overlap on the GPU (on different streams, or from several threads
 * without ordering) race on it and must be serialised by the caller.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define MHC_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)
MHC_API mhc_status mhc_backward_noalloc(const mhc_params *p, const void *x, const float *phi,
                                        const float *b, const float *alpha, const void *f_out,
                                        const void *grad_x_next, const void *grad_h_in,
                                        void *grad_x, float *grad_phi, float *grad_b,
                                        float *grad_alpha, void *grad_f_out, int *dev_status,
                                        mhc_stream_t stream);

/*
 * mhc_sinkhorn_knopp -- standalone batched Sinkhorn-Knopp (source: section
 * "Vielfaeltig eingeschraenkte Hyperverbindungen": alternate row and column
 * normalisation, the classical 1967 algorithm; reportify.cn [16]).
 *
 *   in : logits [B][n][n] float32;  out: H [B][n][n] float32
 *   H = exp(logits), then `iters` times {divide every row by its sum, then
 *   every column by its sum}.  With iters >= 1 each row's maximum logit is
 *   subtracted before exp (the first row pass cancels any per-row factor, so
 *   the result is unchanged); with iters == 0 the output is exp(logits).
 *   n in {1, 2, 4, 8, 16}; B >= 1; iters >= 0.
 */
MHC_API mhc_status mhc_sinkhorn_knopp(int n, int iters, int64_t B, const float *logits, float *out,
                              int *dev_status, mhc_stream_t stream);

/*
 * mhc_depth_amax -- composite residual map over depth and its Amax gain
 * (source: section "Warum Hyperverbindungen instabil werden": the gain of
 * the product of the residual mixers over layers, from its maximum row and
 * column sums; "Vielfaeltig eingeschraenkte Hyperverbindungen": bounded
 * for doubly stochastic mixers).
 *
 *   in : H [T][L][n][n] float32 (per token, layer 0 applied first)
 *   out: gain_fwd [T] = max_i sum_j |P_ij|,  gain_bwd [T] = max_j sum_i |P_ij|
 *        where P = H[L-1] ... H[1] H[0]   (float32)
 *   n in {1, 2, 4, 8, 16}; T >= 1; L >= 0 (L = 0 gives P = I, gains 1).
 */
MHC_API mhc_status mhc_depth_amax(int n, int64_t T, int L, const float *H, float *gain_fwd,
                          float *gain_bwd, int *dev_status, mhc_stream_t stream);

/*
 * mhc_recompute_plan -- block size for recomputing the depth stack (source:
 * reportify.cn [21]: the mHC intermediates are dropped after the forward and
 * rebuilt in the backward; [22]: the recompute block is chosen to make the
 * total memory smallest.  The pages state the aim but not the cost; the cost
 * below is this library's reading of it).
 *
 * The L layers are cut into consecutive blocks of at most `block` layers;
 * the first block takes the remainder, so the last block is full.  The
 * forward keeps only each block's input stream x [n][C] per token.  The
 * backward handles the blocks last to first: it recomputes a block's forward
 * and holds, for each of its layers, x_l [n][C], h_in_l [C] and f_out_l [C]
 * while the block's backward runs, then drops that block's input.  At the
 * peak (the last block) the resident activations per token are
 *     R(B) = C * ( n * (ceil(L / B) - 1)  +  (n + 2) * B )   elements,
 * the inputs of the other blocks plus one full block.  (Buffers that every
 * B needs alike, the gradient being passed down and the layer being computed
 * in the forward, are not counted.)  Over real B the minimum is at
 * B = sqrt(n L / (n + 2)).
 *
 *   in : n >= 1 streams, L >= 1 layers
 *   out: *block = the integer B in [1, L] with the smallest R(B) (the smallest
 *        such B on a tie); *resident = R(block) / C (may be NULL).
 *   MHC_ERR_INVALID_ARG for n < 1, L < 1 or block == NULL.  Host only: no
 *   GPU work, no allocation.
 */
MHC_API mhc_status mhc_recompute_plan(int32_t n, int32_t L, int32_t *block, int64_t *resident);

#ifdef __cplusplus
}
#endif

#endif /* MHC_H_ */
