// mhc_dispatch.h -- the host-side launchers behind the C ABI (internal to
// libmhc.so).  Each kernel file defines its launchers; mhc_api.cu and
// mhc_noalloc.cu call them.  All pointers are device pointers; every launcher
// is asynchronous on stream `s` and returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mhc {

// Mapping kernels: the forward; the backward's recompute with every
// C-reduction; or the pre half of the backward in training order, which takes
// <G_i, x_j> and <G_i, f_out> from the post half (`red`, [T][n*n + n]).
// MAP_POSTFWD: layer l's post merge fused with layer l+1's forward mapping.
// MAP_BWD_DOTS (n = 8): the backward's recompute with every C-reduction read
// from `red` ([T][n*n + 2n]: <G_i, x_j>, <G_i, f_out>, <g, x_j>).
enum MapMode { MAP_FWD = 0, MAP_BWD = 1, MAP_BWD_SPLIT = 2, MAP_POSTFWD = 3, MAP_BWD_DOTS = 4 };

// k_sinkhorn.cu
cudaError_t sinkhorn_dispatch(int n, int iters, int64_t B, const float* logits, float* out,
                              int* st, cudaStream_t s);
cudaError_t depth_amax_dispatch(int n, int64_t T, int L, const float* H, float* gf, float* gb,
                                cudaStream_t s);
// k_post.cu
cudaError_t post_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const void* f,
                          const float* Hpost, const float* Hres, void* xn, cudaStream_t s);
cudaError_t hin_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const float* Hpre,
                         void* h_in, cudaStream_t s);
cudaError_t post_bwd_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const void* f,
                              const float* Hpost, const void* G, void* gf, float* red,
                              cudaStream_t s);
// k_map.cu (CUDA cores; red == nullptr selects MAP_BWD, else MAP_BWD_SPLIT)
// ag: 3 = alpha holds the pre, post and res scales (and grad_alpha their three
// gradients); otherwise one shared alpha.
cudaError_t map_fwd_dispatch(int n, int dtype, int64_t T, int64_t C, int iters, float eps,
                             const void* x, const float* phi, const float* b, const float* alpha,
                             int ag, float* Hpre, float* Hpost, float* Hres, int* st,
                             cudaStream_t s);
cudaError_t map_bwd_dispatch(int n, int dtype, int64_t T, int64_t C, int iters, float eps,
                             const void* x, const float* phi, const float* b, const float* alpha,
                             int ag, const void* G, const void* g, const void* f, const float* red,
                             float* coef, float* part, int* st, cudaStream_t s);
// k_map_tc.cu (bf16, n = 4: projection on the tensor cores); mode is a MapMode.
// wait_ns: limit of each wait on another warp's or the copy engine's progress
// (0: the default 2 s); the tensor-core kernels take it, the CUDA-core ones
// have no such waits.
cudaError_t map_tc_dispatch(int mode, int64_t T, int64_t C, int iters, float eps, const void* x,
                            const float* phi, void* phi_split, const float* b, const float* alpha,
                            int ag, float* Hpre, float* Hpost, float* Hres, const void* G,
                            const void* g,
                            const void* f, const float* red, void* urec, float* hrec, float* part,
                            void* kscratch, int* st, int64_t wait_ns, cudaStream_t s);
size_t map_tc_phi_bytes(int64_t C);
// scratch of the channel-split mapping (part records, counters); kscratch
// must hold this many bytes, 256-byte aligned (may be null when it is 0)
size_t map_tc_scratch_bytes(int64_t T, int64_t C);

// phi [K][24] fp32 -> the bf16 split copy of phi^T [48][K] the mapping MMAs read
cudaError_t phi_split_dispatch(int64_t K, const float* phi, void* phi_split, cudaStream_t s);
// k_map8_tc.cu (bf16, n = 8: projection on the tensor cores); mode is MAP_FWD,
// MAP_BWD_SPLIT or MAP_BWD_DOTS (G and f are not read).  Splits phi into
// phi_split (map8_tc_phi_bytes(C) bytes); the backward modes write the per-token records (coef
// [T][Coef<8>::SIZE]), the U rows (urec [T][TcRec8::U_ELEMS] bf16) and one
// partial-sum record per 128 tokens (part); the backward modes keep Sinkhorn
// checkpoints in ck (map8_ck_bytes(T, iters) bytes; unused forward).
cudaError_t map8_tc_dispatch(int mode, int64_t T, int64_t C, int iters, float eps, const void* x,
                             const float* phi, void* phi_split, const float* b,
                             const float* alpha, int ag, float* Hpre, float* Hpost, float* Hres,
                             const void* G, const void* g, const void* f, const float* red,
                             float* coef, void* urec, float* part, float* ck, int* st,
                             int64_t wait_ns, cudaStream_t s);
// Sinkhorn checkpoints of the n = 8 backward mapping (ck, global scratch):
// iters + 1 iterates of 64 floats per token
size_t map8_ck_bytes(int64_t T, int iters);
// k_apply8_tc.cu (bf16, n = 8): grad_x / grad_f_out with phi u on the tensor
// cores (the accumulators stay on chip), grad_phi as a tensor-core contraction
// over the tokens, and grad_b / grad_alpha from the partial sums; phi_split is
// the mapping's bf16 split copy of phi^T; gpart is scratch of
// apply8_tc_scratch_bytes() bytes (grad_phi parts of blocks that CTAs share).
// gf == nullptr skips grad_f_out.
cudaError_t apply8_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_split,
                               const void* G, const void* g, const float* coef, const void* urec,
                               const float* part, int nparts, void* gx, void* gf, float* gphi,
                               float* gb, float* ga, int ag, float* gpart, int* st,
                               int64_t wait_ns, cudaStream_t s);
size_t apply8_tc_scratch_bytes();
size_t map8_tc_phi_bytes(int64_t C);

// k_proj16_tc.cu (bf16, n = 16): splits phi into the tiled bf16 copy phi_t
// (proj16_phi_bytes(C) bytes) and writes each token's 288 projections y and
// its sum of squares into rows [T][ostride] (y at [0, 288), ss at [576]).
cudaError_t proj16_dispatch(int64_t T, int64_t C, const void* x, const float* phi, void* phi_t,
                            float* rows, int64_t ostride, int* st, int64_t wait_ns,
                            cudaStream_t s);
size_t proj16_phi_bytes(int64_t C);
// k_dots_tc.cu (bf16): the backward's C-reductions per token.  n = 16: into
// rows [T][Coef<16>::SIZE] at [288 + d]; full = all 288 (<G_i, x_j> on the
// tensor cores, <g, x_i>, <G_i, f>), otherwise <g, x_i> only (split backward).
// n = 8: <G_i, x_j> (tensor cores), <G_i, f> and <g, x_j> into red [T][80],
// the layout the n = 8 mapping's MAP_BWD_DOTS mode reads.
cudaError_t dots16_dispatch(bool full, int64_t T, int64_t C, const void* x, const void* G,
                            const void* g, const void* f, float* rows, int* st, int64_t wait_ns,
                            cudaStream_t s);
cudaError_t dots8_red_dispatch(int64_t T, int64_t C, const void* x, const void* G, const void* g,
                               const void* f, float* red, int* st, int64_t wait_ns,
                               cudaStream_t s);
// k_wide.cu, bf16 with n = 16: the mapping with the projection on the tensor
// cores (proj16_dispatch) and the rest of the k_wide kernels: MAP_FWD writes
// the maps (rows: [T][Coef<16>::SIZE] scratch); MAP_BWD / MAP_BWD_SPLIT write
// the coefficient records into rows (= coef) and the partial sums, keeping the
// Sinkhorn checkpoints in ck (wide_ck_bytes(T, iters) bytes; unused forward).
cudaError_t wide_map_tc_dispatch(int mode, int64_t T, int64_t C, int iters, float eps,
                                 const void* x, const float* phi, void* phi_t, const float* b,
                                 const float* alpha, int ag, float* Hpre, float* Hpost,
                                 float* Hres, const void* G, const void* g, const void* f,
                                 const float* red, float* rows, float* part, float* ck, int* st,
                                 int64_t wait_ns, cudaStream_t s);
size_t wide_ck_bytes(int64_t T, int iters);

// k_apply16_tc.cu (bf16, n = 16): the apply with phi u and grad_phi on the
// tensor cores.  coef / part: the n = 16 mapping's records and partial sums;
// phi_t: the tiled phi^T copy of proj16_dispatch; urec (apply16_urec_bytes(T))
// and phiu (fp32 [T][16][C]) are scratch.  gf == nullptr skips grad_f_out.
cudaError_t apply16_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_t,
                                const void* G, const void* g, const float* coef,
                                const float* part, int nparts, void* urec, float* phiu, void* gx,
                                void* gf, float* gphi, float* gb, float* ga, int ag, int* st,
                                int64_t wait_ns, cudaStream_t s);
size_t apply16_urec_bytes(int64_t T);
// the phi u scratch also holds grad_phi's partial slots: at least this many bytes
size_t apply16_gphi_part_bytes();
// grad_b and grad_alpha of the n = 16 paths from the mapping's partial sums
cudaError_t wide_bias_dispatch(const float* part, int nparts, float* gb, float* ga, int ag,
                               cudaStream_t s);

// k_wide.cu (n = 16, CUDA cores); the mapping's mode is a MapMode
int wide_map_tokens_per_cta();
cudaError_t wide_map_dispatch(int mode, int dtype, int64_t T, int64_t C, int iters, float eps,
                              const void* x, const float* phi, const float* b, const float* alpha,
                              int ag, float* Hpre, float* Hpost, float* Hres, const void* G,
                              const void* g, const void* f, const float* red, float* coef,
                              float* part, int* st, cudaStream_t s);
cudaError_t wide_post_dispatch(int dtype, int64_t T, int64_t C, const void* x, const void* f,
                               const float* Hpost, const float* Hres, void* xn, cudaStream_t s);
cudaError_t wide_post_bwd_dispatch(int dtype, int64_t T, int64_t C, const void* x, const void* f,
                                   const float* Hpost, const void* G, void* gf, float* red,
                                   cudaStream_t s);
cudaError_t wide_apply_dispatch(int dtype, int64_t T, int64_t C, const void* x, const float* phi,
                                const void* G, const void* g, const float* coef, const float* part,
                                int nparts, void* gx, void* gf, float* gphi, float* gb, float* ga,
                                int ag, cudaStream_t s);
cudaError_t post_map_tc_dispatch(int64_t T, int64_t C, int iters, float eps, const void* x,
                                 const void* f, const float* Hpost_in, const float* Hres_in,
                                 const float* phi_next, void* phi_split, const float* b_next,
                                 const float* alpha_next, int ag, void* x_next, float* Hpre,
                                 float* Hpost, float* Hres, void* kscratch, int* st,
                                 int64_t wait_ns, cudaStream_t s);
// k_apply_tc.cu (bf16, n = 4: phi u and grad_phi on the tensor cores);
// gf == nullptr skips grad_f_out
cudaError_t apply_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_split,
                              const void* G, const void* g, const void* urec, const float* hrec,
                              const float* part, int nparts, void* gx, void* gf, float* gphi,
                              float* gb, float* ga, int ag, void* scratch, int* st,
                              int64_t wait_ns, cudaStream_t s);
size_t apply_tc_scratch_bytes(int64_t T, int64_t C);
// k_bwd.cu (CUDA cores); gf == nullptr skips grad_f_out
cudaError_t apply_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const float* phi,
                           const void* G, const void* g, const float* coef, const float* part,
                           int nparts, void* gx, void* gf, float* gphi, float* gb, float* ga,
                           int ag, cudaStream_t s);

}  // namespace mhc
