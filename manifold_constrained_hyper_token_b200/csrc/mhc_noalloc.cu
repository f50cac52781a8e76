// mhc_noalloc.cu -- mhc_backward_noalloc: the backward pass with its scratch
// in a fixed, library-owned device array instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where
// they run the backward -- a runtime that plans every device buffer at start-up
// and forbids allocation afterwards, a plugin that a host framework hands only
// its input and output buffers, or a process whose framework caching allocator
// already holds the whole device.  cudaMalloc can also synchronise the device
// and has no latency bound, which latency-critical callers avoid.  Such callers
// pass the same inputs and outputs as to mhc_backward and nothing else.
//
// The scratch is one file-scope __device__ array of MHC_NOALLOC_SCRATCH_BYTES
// (4 MiB).  Every GPU that loads this library holds it until the process
// exits.  Host code cannot use the array's name as a device address (in host
// code it names a host-side shadow), so every call looks the device address up
// with cudaGetSymbolAddress on the current device.  Nothing is cached: after a
// device reset, or once the module is loaded again, the next call gets the
// array's new address.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"


namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MHC_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" mhc_status mhc_backward_noalloc(const mhc_params* p, const void* x, const float* phi,
                                           const float* b, const float* alpha, const void* f_out,
                                           const void* grad_x_next, const void* grad_h_in,
                                           void* grad_x, float* grad_phi, float* grad_b,
                                           float* grad_alpha, void* grad_f_out, int* dev_status,
                                           mhc_stream_t stream) {
  if (p == nullptr) return MHC_ERR_INVALID_ARG;
  if (p->n != 1 && p->n != 2 && p->n != 4 && p->n != 8) return MHC_ERR_UNSUPPORTED;
  if (p->dtype != MHC_DTYPE_F32 && p->dtype != MHC_DTYPE_BF16) return MHC_ERR_UNSUPPORTED;
  if (mhc_backward_workspace_size(p) == 0) return MHC_ERR_INVALID_ARG;  // T, C, t_max or eps
  // this entry point runs the CUDA-core kernels: per-token records, then the
  // per-64-token partial sums
  const int coef_floats = p->n == 1   ? mhc::Coef<1>::SIZE
                          : p->n == 2 ? mhc::Coef<2>::SIZE
                          : p->n == 8 ? mhc::Coef<8>::SIZE
                                      : mhc::Coef<4>::SIZE;
  const int dz_floats = p->n == 1   ? mhc::Coef<1>::DZ_SIZE
                        : p->n == 2 ? mhc::Coef<2>::DZ_SIZE
                        : p->n == 8 ? mhc::Coef<8>::DZ_SIZE
                                    : mhc::Coef<4>::DZ_SIZE;
  const int nparts = (int)((p->T + 63) / 64);
  const size_t coef_bytes = round_up((size_t)p->T * coef_floats * 4, 256);
  const size_t need = coef_bytes + (size_t)nparts * dz_floats * 4;
  if (need > (size_t)MHC_NOALLOC_SCRATCH_BYTES) return MHC_ERR_WORKSPACE;
  auto ok16 = [](const void* q) { return q != nullptr && ((uintptr_t)q & 15u) == 0; };
  if (!ok16(x) || !ok16(phi) || !ok16(b) || !ok16(alpha) || !ok16(f_out) || !ok16(grad_x_next) ||
      !ok16(grad_h_in) || !ok16(grad_x) || !ok16(grad_phi) || !ok16(grad_b) ||
      !ok16(grad_alpha) || !ok16(grad_f_out))
    return MHC_ERR_INVALID_ARG;

  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MHC_ERR_CUDA;

  // Both parts are written in full by the first kernel before the second
  // reads them, so no part of the scratch needs clearing.
  char* ws = (char*)scratch;
  float* coef = (float*)ws;
  float* part = (float*)(ws + coef_bytes);

  cudaStream_t s = (cudaStream_t)stream;
  const int ag = p->alpha_groups == 3 ? 3 : 1;
  cudaError_t e = mhc::map_bwd_dispatch(p->n, p->dtype, p->T, p->C, p->t_max, p->eps, x, phi, b,
                                        alpha, ag, grad_x_next, grad_h_in, f_out, nullptr, coef,
                                        part, dev_status, s);
  if (e != cudaSuccess) return MHC_ERR_CUDA;
  e = mhc::apply_dispatch(p->n, p->dtype, p->T, p->C, x, phi, grad_x_next, grad_h_in, coef, part,
                          nparts, grad_x, grad_f_out, grad_phi, grad_b, grad_alpha, ag, s);
  return e == cudaSuccess ? MHC_OK : MHC_ERR_CUDA;
}
