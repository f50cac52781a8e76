// mhc_api.cu -- the extern "C" boundary of libmhc.so: argument validation,
// workspace carving and kernel launches.  No entry point allocates,
// synchronises or keeps state between calls.
#include <math.h>

#include <algorithm>

#include "mhc_common.cuh"
#include "mhc_dispatch.h"

namespace {

constexpr int kVersionMajor = 0;
constexpr int kVersionMinor = 2;

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

mhc_status check_params(const mhc_params* p) {
  if (!p) return MHC_ERR_INVALID_ARG;
  if (p->T < 1 || p->C < 8 || (p->C % 8) != 0 || p->t_max < 0) return MHC_ERR_INVALID_ARG;
  if (!(p->eps >= 0.0f) || !isfinite(p->eps)) return MHC_ERR_INVALID_ARG;
  if (p->n != 1 && p->n != 2 && p->n != 4 && p->n != 8 && p->n != 16) return MHC_ERR_UNSUPPORTED;
  if (p->dtype != MHC_DTYPE_F32 && p->dtype != MHC_DTYPE_BF16) return MHC_ERR_UNSUPPORTED;
  if (p->alpha_groups != 0 && p->alpha_groups != 1 && p->alpha_groups != 3)
    return MHC_ERR_INVALID_ARG;
  if (p->wait_ns < 0) return MHC_ERR_INVALID_ARG;
  // tile coordinates of the TMA copies are 32-bit signed: keep T (and a tile
  // past it) inside that range; the bf16 n = 8 and n = 16 backward reductions
  // address x and grad_x_next as T*n rows
  if (p->T > (int64_t)0x7fffffffLL - 256) return MHC_ERR_INVALID_ARG;
  if (p->dtype == MHC_DTYPE_BF16 && p->n >= 8 && p->T * p->n > (int64_t)0x7fffffffLL - 256)
    return MHC_ERR_INVALID_ARG;
  return MHC_OK;
}

mhc_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MHC_OK : MHC_ERR_CUDA; }

// 3: alpha = (alpha_pre, alpha_post, alpha_res); 0 or 1: one shared alpha
int alpha_groups(const mhc_params* p) { return p->alpha_groups == 3 ? 3 : 1; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int coef_size(int n) {
  switch (n) {
    case 1: return mhc::Coef<1>::SIZE;
    case 2: return mhc::Coef<2>::SIZE;
    case 8: return mhc::Coef<8>::SIZE;
    case 16: return mhc::Coef<16>::SIZE;
    default: return mhc::Coef<4>::SIZE;
  }
}
int dz_size(int n) {
  switch (n) {
    case 1: return mhc::Coef<1>::DZ_SIZE;
    case 2: return mhc::Coef<2>::DZ_SIZE;
    case 8: return mhc::Coef<8>::DZ_SIZE;
    case 16: return mhc::Coef<16>::DZ_SIZE;
    default: return mhc::Coef<4>::DZ_SIZE;
  }
}

// bf16 activations with n = 4 or n = 8 take the tensor-core mapping and apply
// kernels (128 tokens per mapping CTA); bf16 with n = 16 the tensor-core
// projection and apply around the k_wide reductions, Sinkhorn and adjoint (32
// tokens per epilogue CTA); every other case the CUDA-core kernels (64 tokens
// per mapping CTA; n = 16 its own).
bool use_tc(const mhc_params* p) { return p->dtype == MHC_DTYPE_BF16 && p->n == 4; }
bool use_tc8(const mhc_params* p) { return p->dtype == MHC_DTYPE_BF16 && p->n == 8; }
// bf16 with n = 16: the projection on the tensor cores, the rest on k_wide
bool use_tc16(const mhc_params* p) { return p->dtype == MHC_DTYPE_BF16 && p->n == 16; }
size_t rows16_bytes(int64_t T) { return (size_t)T * mhc::Coef<16>::SIZE * 4; }

// Backward workspace.  CUDA-core path: per-token coefficient records, then one
// partial-sum record (dz, dz . y) per 64-token mapping CTA.  Tensor-core path
// (n = 4): per-token U rows (bf16) and H records, the partial sums per
// 128-token CTA, the bf16 split copy of phi^T that the mapping MMA reads, and
// the apply kernel's grad_phi partials and slice counters.  Tensor-core path
// (n = 8): the coefficient records, the U rows, the C-reductions of the
// backward mapping, the partial sums, the phi split copy, the grad_phi parts
// of the blocks that the apply's CTAs share, and the mapping's Sinkhorn
// checkpoints.
struct BwdWorkspace {
  size_t coef_off, urec_off, hrec_off, part_off, phi_off, apply_off, kmap_off, red_off, total;
  int nparts;
};

BwdWorkspace bwd_layout(const mhc_params* p) {
  BwdWorkspace w{};
  const bool tc = use_tc(p), tc8 = use_tc8(p);
  const int tokens_per_cta =
      (tc || tc8) ? 128 : (p->n == 16 ? mhc::wide_map_tokens_per_cta() : 64);
  w.nparts = (int)((p->T + tokens_per_cta - 1) / tokens_per_cta);
  size_t off = 0;
  if (tc) {
    w.urec_off = off;
    off = round_up(off + (size_t)p->T * mhc::TcRec::U_BYTES, 256);
    w.hrec_off = off;
    off = round_up(off + (size_t)p->T * mhc::TcRec::H_BYTES, 256);
  } else {
    w.coef_off = off;
    off = round_up(off + (size_t)p->T * coef_size(p->n) * 4, 256);
    if (tc8) {
      w.urec_off = off;
      off = round_up(off + (size_t)p->T * mhc::TcRec8::U_BYTES, 256);
      // the whole backward's C-reductions from the tensor-core kernel, read
      // by the mapping in its MAP_BWD_DOTS mode
      w.red_off = off;
      off = round_up(off + (size_t)p->T * (8 * 8 + 2 * 8) * 4, 256);
    }
    if (use_tc16(p)) {
      w.urec_off = off;
      off = round_up(off + mhc::apply16_urec_bytes(p->T), 256);
    }
  }
  w.part_off = off;
  off = round_up(off + (size_t)w.nparts * dz_size(p->n) * 4, 256);
  w.phi_off = off;
  off = round_up(off + (tc    ? mhc::map_tc_phi_bytes(p->C)
                        : tc8 ? mhc::map8_tc_phi_bytes(p->C)
                              : (use_tc16(p) ? mhc::proj16_phi_bytes(p->C) : 0)),
                 256);
  w.apply_off = off;
  // n = 16: the apply's phi u scratch, which the mapping first uses for its
  // Sinkhorn checkpoints
  size_t apply_bytes = 0;
  if (tc) apply_bytes = mhc::apply_tc_scratch_bytes(p->T, p->C);
  if (tc8) apply_bytes = mhc::apply8_tc_scratch_bytes();
  if (use_tc16(p))
    apply_bytes = std::max({(size_t)p->T * 16 * p->C * 4, mhc::wide_ck_bytes(p->T, p->t_max),
                            mhc::apply16_gphi_part_bytes()});
  off = round_up(off + apply_bytes, 256);
  // the mapping's scratch: n = 4, its channel-split records; n = 8, its Sinkhorn
  // checkpoints
  w.kmap_off = off;
  off = round_up(off + (tc    ? mhc::map_tc_scratch_bytes(p->T, p->C)
                        : tc8 ? mhc::map8_ck_bytes(p->T, p->t_max)
                              : 0),
                 256);
  w.total = off;
  return w;
}

mhc_status check_workspace(const BwdWorkspace& w, void* workspace, size_t bytes) {
  if (workspace == nullptr || bytes < w.total || ((uintptr_t)workspace & 255u) != 0)
    return MHC_ERR_WORKSPACE;
  return MHC_OK;
}

}  // namespace

extern "C" {

int mhc_version(void) { return (kVersionMajor << 16) | kVersionMinor; }

const char* mhc_status_string(int status) {
  switch (status) {
    case MHC_OK: return "MHC_OK: success";
    case MHC_ERR_INVALID_ARG:
      return "MHC_ERR_INVALID_ARG: null or misaligned pointer, or a size/iteration/eps out of range";
    case MHC_ERR_UNSUPPORTED: return "MHC_ERR_UNSUPPORTED: stream count n or dtype not built";
    case MHC_ERR_CUDA: return "MHC_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case MHC_ERR_NONFINITE: return "MHC_ERR_NONFINITE: a kernel saw a non-finite RMS or logit";
    case MHC_ERR_TIMEOUT: return "MHC_ERR_TIMEOUT: a bounded device-side wait gave up";
    case MHC_ERR_WORKSPACE: return "MHC_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown mhc_status";
  }
}

size_t mhc_pre_workspace_size(const mhc_params* p) {
  if (check_params(p) != MHC_OK) return 0;
  // the bf16 split copy of phi, then the channel-split mapping's scratch
  if (use_tc(p))
    return round_up(mhc::map_tc_phi_bytes(p->C), 256) +
           round_up(mhc::map_tc_scratch_bytes(p->T, p->C), 256);
  if (use_tc16(p))  // the tiled phi copy, then the rows of projections
    return round_up(mhc::proj16_phi_bytes(p->C), 256) + round_up(rows16_bytes(p->T), 256);
  return use_tc8(p) ? round_up(mhc::map8_tc_phi_bytes(p->C), 256) : 0;
}

mhc_status mhc_pre(const mhc_params* p, const void* x, const float* phi, const float* b,
                   const float* alpha, void* h_in, float* H_pre, float* H_post, float* H_res,
                   void* workspace, size_t workspace_bytes, int* dev_status, mhc_stream_t stream) {
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(b) || !aligned16(alpha) || !aligned16(h_in) ||
      !aligned16(H_pre) || !aligned16(H_post) || !aligned16(H_res))
    return MHC_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (use_tc(p)) {
    const size_t need = mhc_pre_workspace_size(p);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return MHC_ERR_WORKSPACE;
    char* ws = (char*)workspace;
    st = from_cuda(mhc::map_tc_dispatch(mhc::MAP_FWD, p->T, p->C, p->t_max, p->eps, x, phi, ws, b,
                                        alpha, alpha_groups(p), H_pre, H_post, H_res, nullptr,
                                        nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                        ws + round_up(mhc::map_tc_phi_bytes(p->C), 256),
                                        dev_status, p->wait_ns, s));
  } else if (use_tc8(p)) {
    const size_t need = mhc_pre_workspace_size(p);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return MHC_ERR_WORKSPACE;
    st = from_cuda(mhc::map8_tc_dispatch(mhc::MAP_FWD, p->T, p->C, p->t_max, p->eps, x, phi,
                                         workspace, b, alpha, alpha_groups(p), H_pre, H_post,
                                         H_res, nullptr, nullptr, nullptr, nullptr, nullptr,
                                         nullptr, nullptr, nullptr, dev_status, p->wait_ns, s));
  } else if (use_tc16(p)) {
    const size_t need = mhc_pre_workspace_size(p);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return MHC_ERR_WORKSPACE;
    char* ws = (char*)workspace;
    st = from_cuda(mhc::wide_map_tc_dispatch(
        mhc::MAP_FWD, p->T, p->C, p->t_max, p->eps, x, phi, ws, b, alpha, alpha_groups(p), H_pre,
        H_post, H_res, nullptr, nullptr, nullptr, nullptr,
        (float*)(ws + round_up(mhc::proj16_phi_bytes(p->C), 256)), nullptr, nullptr, dev_status,
        p->wait_ns,
        s));
  } else {
    st = from_cuda(mhc::map_fwd_dispatch(p->n, p->dtype, p->T, p->C, p->t_max, p->eps, x, phi, b,
                                         alpha, alpha_groups(p), H_pre, H_post, H_res, dev_status, s));
  }
  if (st != MHC_OK) return st;
  return from_cuda(mhc::hin_dispatch(p->n, p->dtype, p->T, p->C, x, H_pre, h_in, s));
}

mhc_status mhc_post(const mhc_params* p, const void* x, const void* f_out, const float* H_post,
                    const float* H_res, void* x_next, int* dev_status, mhc_stream_t stream) {
  (void)dev_status;
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(f_out) || !aligned16(H_post) || !aligned16(H_res) ||
      !aligned16(x_next))
    return MHC_ERR_INVALID_ARG;
  if (x_next == x || x_next == f_out) return MHC_ERR_INVALID_ARG;
  return from_cuda(mhc::post_dispatch(p->n, p->dtype, p->T, p->C, x, f_out, H_post, H_res, x_next,
                                      (cudaStream_t)stream));
}

size_t mhc_backward_workspace_size(const mhc_params* p) {
  if (check_params(p) != MHC_OK) return 0;
  return bwd_layout(p).total;
}

mhc_status mhc_backward_map(const mhc_params* p, const void* x, const float* phi, const float* b,
                            const float* alpha, const void* f_out, const void* grad_x_next,
                            const void* grad_h_in, void* workspace, size_t workspace_bytes,
                            int* dev_status, mhc_stream_t stream) {
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(b) || !aligned16(alpha) ||
      !aligned16(f_out) || !aligned16(grad_x_next) || !aligned16(grad_h_in))
    return MHC_ERR_INVALID_ARG;
  const BwdWorkspace w = bwd_layout(p);
  st = check_workspace(w, workspace, workspace_bytes);
  if (st != MHC_OK) return st;
  char* ws = (char*)workspace;
  if (use_tc(p))
    return from_cuda(mhc::map_tc_dispatch(mhc::MAP_BWD, p->T, p->C, p->t_max, p->eps, x, phi,
                                          ws + w.phi_off, b, alpha, alpha_groups(p), nullptr,
                                          nullptr, nullptr, grad_x_next, grad_h_in, f_out, nullptr,
                                          ws + w.urec_off, (float*)(ws + w.hrec_off),
                                          (float*)(ws + w.part_off), ws + w.kmap_off, dev_status,
                                          p->wait_ns, (cudaStream_t)stream));
  if (use_tc8(p)) {
    // the C-reductions (<G_i, x_j> on the tensor cores), then the mapping with
    // only x staged (the projection, the gates, the adjoint)
    st = from_cuda(mhc::dots8_red_dispatch(p->T, p->C, x, grad_x_next, grad_h_in, f_out,
                                           (float*)(ws + w.red_off), dev_status, p->wait_ns,
                                           (cudaStream_t)stream));
    if (st != MHC_OK) return st;
    return from_cuda(mhc::map8_tc_dispatch(mhc::MAP_BWD_DOTS, p->T, p->C, p->t_max, p->eps, x,
                                           phi, ws + w.phi_off, b, alpha, alpha_groups(p), nullptr,
                                           nullptr, nullptr, nullptr, nullptr, nullptr,
                                           (const float*)(ws + w.red_off),
                                           (float*)(ws + w.coef_off), ws + w.urec_off,
                                           (float*)(ws + w.part_off), (float*)(ws + w.kmap_off),
                                           dev_status, p->wait_ns, (cudaStream_t)stream));
  }
  if (use_tc16(p))
    return from_cuda(mhc::wide_map_tc_dispatch(
        mhc::MAP_BWD, p->T, p->C, p->t_max, p->eps, x, phi, ws + w.phi_off, b, alpha,
        alpha_groups(p), nullptr, nullptr, nullptr, grad_x_next, grad_h_in, f_out, nullptr,
        (float*)(ws + w.coef_off), (float*)(ws + w.part_off), (float*)(ws + w.apply_off),
        dev_status, p->wait_ns, (cudaStream_t)stream));
  return from_cuda(mhc::map_bwd_dispatch(p->n, p->dtype, p->T, p->C, p->t_max, p->eps, x, phi, b,
                                         alpha, alpha_groups(p), grad_x_next, grad_h_in, f_out, nullptr,
                                         (float*)(ws + w.coef_off), (float*)(ws + w.part_off),
                                         dev_status, (cudaStream_t)stream));
}

mhc_status mhc_backward_apply(const mhc_params* p, const void* x, const float* phi,
                              const void* grad_x_next, const void* grad_h_in, void* grad_x,
                              float* grad_phi, float* grad_b, float* grad_alpha, void* grad_f_out,
                              const void* workspace, size_t workspace_bytes, int* dev_status,
                              mhc_stream_t stream) {
  (void)dev_status;
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(grad_x_next) || !aligned16(grad_h_in) ||
      !aligned16(grad_x) || !aligned16(grad_phi) || !aligned16(grad_b) ||
      !aligned16(grad_alpha) || !aligned16(grad_f_out))
    return MHC_ERR_INVALID_ARG;
  const BwdWorkspace w = bwd_layout(p);
  st = check_workspace(w, (void*)workspace, workspace_bytes);
  if (st != MHC_OK) return st;
  const char* ws = (const char*)workspace;
  if (use_tc(p))
    return from_cuda(mhc::apply_tc_dispatch(p->T, p->C, x, ws + w.phi_off, grad_x_next, grad_h_in,
                                            ws + w.urec_off, (const float*)(ws + w.hrec_off),
                                            (const float*)(ws + w.part_off), w.nparts, grad_x,
                                            grad_f_out, grad_phi, grad_b, grad_alpha,
                                            alpha_groups(p), (void*)(ws + w.apply_off), dev_status,
                                            p->wait_ns, (cudaStream_t)stream));
  if (use_tc8(p))
    return from_cuda(mhc::apply8_tc_dispatch(
        p->T, p->C, x, ws + w.phi_off, grad_x_next, grad_h_in, (const float*)(ws + w.coef_off),
        ws + w.urec_off, (const float*)(ws + w.part_off), w.nparts, grad_x, grad_f_out,
        grad_phi, grad_b, grad_alpha, alpha_groups(p), (float*)(ws + w.apply_off), dev_status,
        p->wait_ns, (cudaStream_t)stream));
  if (use_tc16(p))
    return from_cuda(mhc::apply16_tc_dispatch(
        p->T, p->C, x, ws + w.phi_off, grad_x_next, grad_h_in, (const float*)(ws + w.coef_off),
        (const float*)(ws + w.part_off), w.nparts, (void*)(ws + w.urec_off),
        (float*)(ws + w.apply_off), grad_x, grad_f_out, grad_phi, grad_b, grad_alpha,
        alpha_groups(p), dev_status, p->wait_ns, (cudaStream_t)stream));
  return from_cuda(mhc::apply_dispatch(p->n, p->dtype, p->T, p->C, x, phi, grad_x_next, grad_h_in,
                                       (const float*)(ws + w.coef_off),
                                       (const float*)(ws + w.part_off), w.nparts, grad_x,
                                       grad_f_out, grad_phi, grad_b, grad_alpha,
                                       alpha_groups(p), (cudaStream_t)stream));
}

mhc_status mhc_backward(const mhc_params* p, const void* x, const float* phi, const float* b,
                        const float* alpha, const void* f_out, const void* grad_x_next,
                        const void* grad_h_in, void* grad_x, float* grad_phi, float* grad_b,
                        float* grad_alpha, void* grad_f_out, void* workspace,
                        size_t workspace_bytes, int* dev_status, mhc_stream_t stream) {
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(grad_x) || !aligned16(grad_phi) || !aligned16(grad_b) ||
      !aligned16(grad_alpha) || !aligned16(grad_f_out))
    return MHC_ERR_INVALID_ARG;
  st = mhc_backward_map(p, x, phi, b, alpha, f_out, grad_x_next, grad_h_in, workspace,
                        workspace_bytes, dev_status, stream);
  if (st != MHC_OK) return st;
  return mhc_backward_apply(p, x, phi, grad_x_next, grad_h_in, grad_x, grad_phi, grad_b,
                            grad_alpha, grad_f_out, workspace, workspace_bytes, dev_status, stream);
}

size_t mhc_post_fused_workspace_size(const mhc_params* p) { return mhc_pre_workspace_size(p); }

mhc_status mhc_post_fused(const mhc_params* p, const void* x, const void* f_out,
                          const float* H_post, const float* H_res, const float* phi_next,
                          const float* b_next, const float* alpha_next, void* x_next,
                          float* H_pre_next, float* H_post_next, float* H_res_next,
                          void* workspace, size_t workspace_bytes, int* dev_status,
                          mhc_stream_t stream) {
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(f_out) || !aligned16(H_post) || !aligned16(H_res) ||
      !aligned16(phi_next) || !aligned16(b_next) || !aligned16(alpha_next) || !aligned16(x_next) ||
      !aligned16(H_pre_next) || !aligned16(H_post_next) || !aligned16(H_res_next))
    return MHC_ERR_INVALID_ARG;
  if (x_next == x || x_next == f_out) return MHC_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (use_tc(p)) {
    const size_t need = mhc_post_fused_workspace_size(p);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return MHC_ERR_WORKSPACE;
    char* ws = (char*)workspace;
    return from_cuda(mhc::post_map_tc_dispatch(
        p->T, p->C, p->t_max, p->eps, x, f_out, H_post, H_res, phi_next, ws, b_next, alpha_next,
        alpha_groups(p), x_next, H_pre_next, H_post_next, H_res_next,
        ws + round_up(mhc::map_tc_phi_bytes(p->C), 256), dev_status, p->wait_ns, s));
  }
  // fp32 or n != 4: the post merge, then the mapping of x_next (both on the GPU),
  // with the same mapping kernel mhc_pre runs
  st = from_cuda(mhc::post_dispatch(p->n, p->dtype, p->T, p->C, x, f_out, H_post, H_res, x_next, s));
  if (st != MHC_OK) return st;
  if (use_tc8(p)) {
    const size_t need = mhc_post_fused_workspace_size(p);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return MHC_ERR_WORKSPACE;
    return from_cuda(mhc::map8_tc_dispatch(mhc::MAP_FWD, p->T, p->C, p->t_max, p->eps, x_next,
                                           phi_next, workspace, b_next, alpha_next,
                                           alpha_groups(p), H_pre_next, H_post_next, H_res_next,
                                           nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                           nullptr, nullptr, dev_status, p->wait_ns, s));
  }
  if (use_tc16(p)) {
    const size_t need = mhc_post_fused_workspace_size(p);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return MHC_ERR_WORKSPACE;
    char* ws = (char*)workspace;
    return from_cuda(mhc::wide_map_tc_dispatch(
        mhc::MAP_FWD, p->T, p->C, p->t_max, p->eps, x_next, phi_next, ws, b_next, alpha_next,
        alpha_groups(p), H_pre_next, H_post_next, H_res_next, nullptr, nullptr, nullptr, nullptr,
        (float*)(ws + round_up(mhc::proj16_phi_bytes(p->C), 256)), nullptr, nullptr, dev_status,
        p->wait_ns,
        s));
  }
  return from_cuda(mhc::map_fwd_dispatch(p->n, p->dtype, p->T, p->C, p->t_max, p->eps, x_next,
                                         phi_next, b_next, alpha_next, alpha_groups(p), H_pre_next,
                                         H_post_next,
                                         H_res_next, dev_status, s));
}

mhc_status mhc_layer_input(const mhc_params* p, const void* x, const float* H_pre, void* h_in,
                           int* dev_status, mhc_stream_t stream) {
  (void)dev_status;
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(H_pre) || !aligned16(h_in)) return MHC_ERR_INVALID_ARG;
  return from_cuda(mhc::hin_dispatch(p->n, p->dtype, p->T, p->C, x, H_pre, h_in,
                                     (cudaStream_t)stream));
}

mhc_status mhc_post_backward(const mhc_params* p, const void* x, const void* f_out,
                             const float* H_post, const void* grad_x_next, void* grad_f_out,
                             float* red, int* dev_status, mhc_stream_t stream) {
  (void)dev_status;
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(f_out) || !aligned16(H_post) || !aligned16(grad_x_next) ||
      !aligned16(grad_f_out) || !aligned16(red))
    return MHC_ERR_INVALID_ARG;
  if (grad_f_out == x || grad_f_out == f_out || grad_f_out == grad_x_next)
    return MHC_ERR_INVALID_ARG;
  return from_cuda(mhc::post_bwd_dispatch(p->n, p->dtype, p->T, p->C, x, f_out, H_post,
                                          grad_x_next, grad_f_out, red, (cudaStream_t)stream));
}

size_t mhc_pre_backward_workspace_size(const mhc_params* p) {
  if (check_params(p) != MHC_OK) return 0;
  return bwd_layout(p).total;
}

mhc_status mhc_pre_backward(const mhc_params* p, const void* x, const float* phi, const float* b,
                            const float* alpha, const void* grad_x_next, const void* grad_h_in,
                            const float* red, void* grad_x, float* grad_phi, float* grad_b,
                            float* grad_alpha, void* workspace, size_t workspace_bytes,
                            int* dev_status, mhc_stream_t stream) {
  mhc_status st = check_params(p);
  if (st != MHC_OK) return st;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(b) || !aligned16(alpha) ||
      !aligned16(grad_x_next) || !aligned16(grad_h_in) || !aligned16(red) || !aligned16(grad_x) ||
      !aligned16(grad_phi) || !aligned16(grad_b) || !aligned16(grad_alpha))
    return MHC_ERR_INVALID_ARG;
  const BwdWorkspace w = bwd_layout(p);
  st = check_workspace(w, workspace, workspace_bytes);
  if (st != MHC_OK) return st;
  char* ws = (char*)workspace;
  cudaStream_t s = (cudaStream_t)stream;
  if (use_tc(p)) {
    st = from_cuda(mhc::map_tc_dispatch(mhc::MAP_BWD_SPLIT, p->T, p->C, p->t_max, p->eps, x,
                                        phi, ws + w.phi_off, b, alpha, alpha_groups(p), nullptr,
                                        nullptr, nullptr, nullptr, grad_h_in, nullptr, red,
                                        ws + w.urec_off, (float*)(ws + w.hrec_off),
                                        (float*)(ws + w.part_off), ws + w.kmap_off, dev_status,
                                        p->wait_ns, s));
    if (st != MHC_OK) return st;
    return from_cuda(mhc::apply_tc_dispatch(p->T, p->C, x, ws + w.phi_off, grad_x_next, grad_h_in,
                                            ws + w.urec_off, (const float*)(ws + w.hrec_off),
                                            (const float*)(ws + w.part_off), w.nparts, grad_x,
                                            nullptr, grad_phi, grad_b, grad_alpha, alpha_groups(p),
                                            (void*)(ws + w.apply_off), dev_status, p->wait_ns, s));
  }
  if (use_tc8(p)) {
    st = from_cuda(mhc::map8_tc_dispatch(mhc::MAP_BWD_SPLIT, p->T, p->C, p->t_max, p->eps, x,
                                         phi, ws + w.phi_off, b, alpha, alpha_groups(p), nullptr,
                                         nullptr, nullptr, nullptr, grad_h_in, nullptr, red,
                                         (float*)(ws + w.coef_off), ws + w.urec_off,
                                         (float*)(ws + w.part_off), (float*)(ws + w.kmap_off),
                                         dev_status, p->wait_ns, s));
    if (st != MHC_OK) return st;
    return from_cuda(mhc::apply8_tc_dispatch(
        p->T, p->C, x, ws + w.phi_off, grad_x_next, grad_h_in, (const float*)(ws + w.coef_off),
        ws + w.urec_off, (const float*)(ws + w.part_off), w.nparts, grad_x, nullptr, grad_phi,
        grad_b, grad_alpha, alpha_groups(p), (float*)(ws + w.apply_off), dev_status, p->wait_ns,
        s));
  }
  if (use_tc16(p)) {
    st = from_cuda(mhc::wide_map_tc_dispatch(
        mhc::MAP_BWD_SPLIT, p->T, p->C, p->t_max, p->eps, x, phi, ws + w.phi_off, b, alpha,
        alpha_groups(p), nullptr, nullptr, nullptr, nullptr, grad_h_in, nullptr, red,
        (float*)(ws + w.coef_off), (float*)(ws + w.part_off), (float*)(ws + w.apply_off),
        dev_status, p->wait_ns, s));
    if (st != MHC_OK) return st;
    return from_cuda(mhc::apply16_tc_dispatch(
        p->T, p->C, x, ws + w.phi_off, grad_x_next, grad_h_in, (const float*)(ws + w.coef_off),
        (const float*)(ws + w.part_off), w.nparts, ws + w.urec_off, (float*)(ws + w.apply_off),
        grad_x, nullptr, grad_phi, grad_b, grad_alpha, alpha_groups(p), dev_status, p->wait_ns,
        s));
  }
  st = from_cuda(mhc::map_bwd_dispatch(p->n, p->dtype, p->T, p->C, p->t_max, p->eps, x, phi, b,
                                       alpha, alpha_groups(p), nullptr, grad_h_in, nullptr, red,
                                       (float*)(ws + w.coef_off), (float*)(ws + w.part_off),
                                       dev_status, s));
  if (st != MHC_OK) return st;
  return from_cuda(mhc::apply_dispatch(p->n, p->dtype, p->T, p->C, x, phi, grad_x_next, grad_h_in,
                                       (const float*)(ws + w.coef_off),
                                       (const float*)(ws + w.part_off), w.nparts, grad_x, nullptr,
                                       grad_phi, grad_b, grad_alpha, alpha_groups(p), s));
}

mhc_status mhc_sinkhorn_knopp(int n, int iters, int64_t B, const float* logits, float* out,
                              int* dev_status, mhc_stream_t stream) {
  if (n != 1 && n != 2 && n != 4 && n != 8 && n != 16) return MHC_ERR_UNSUPPORTED;
  if (B < 1 || iters < 0 || !aligned16(logits) || !aligned16(out)) return MHC_ERR_INVALID_ARG;
  if (B > (int64_t)0x7fffffffLL * 64) return MHC_ERR_INVALID_ARG;
  return from_cuda(mhc::sinkhorn_dispatch(n, iters, B, logits, out, dev_status,
                                          (cudaStream_t)stream));
}

mhc_status mhc_depth_amax(int n, int64_t T, int L, const float* H, float* gain_fwd,
                          float* gain_bwd, int* dev_status, mhc_stream_t stream) {
  (void)dev_status;
  if (n != 1 && n != 2 && n != 4 && n != 8 && n != 16) return MHC_ERR_UNSUPPORTED;
  if (T < 1 || L < 0 || !aligned16(gain_fwd) || !aligned16(gain_bwd)) return MHC_ERR_INVALID_ARG;
  if (L > 0 && !aligned16(H)) return MHC_ERR_INVALID_ARG;
  if (T > (int64_t)0x7fffffffLL * 16) return MHC_ERR_INVALID_ARG;
  return from_cuda(
      mhc::depth_amax_dispatch(n, T, L, H, gain_fwd, gain_bwd, (cudaStream_t)stream));
}

mhc_status mhc_recompute_plan(int32_t n, int32_t L, int32_t* block, int64_t* resident) {
  if (n < 1 || L < 1 || block == nullptr) return MHC_ERR_INVALID_ARG;
  int32_t best = 1;
  int64_t best_r = -1;
  for (int32_t B = 1; B <= L; ++B) {
    const int64_t blocks = ((int64_t)L + B - 1) / B;
    const int64_t r = (int64_t)n * (blocks - 1) + (int64_t)(n + 2) * B;
    if (best_r < 0 || r < best_r) { best_r = r; best = B; }
  }
  *block = best;
  if (resident) *resident = best_r;
  return MHC_OK;
}

}  // extern "C"
