// k_post.cu -- the two per-token stream mixes that are pure HBM traffic:
//
//   post merge   x_next[i][c] = sum_j H_res[i][j] x[j][c] + H_post[i] f_out[c]
//                (update equation of the chatgpz.de explainer, section "Von
//                Residualverbindungen zu Hyperverbindungen"; reportify.cn [20]:
//                the output map applied in the same pass as the residual merge)
//   layer input  h_in[c] = sum_i H_pre[i] x[i][c]
//
// One CTA walks tokens with a grid stride; its threads cover the token's C
// channels in 16-byte vectors (8 bf16 or 4 fp32 channels), so every warp
// request is a fully used, coalesced 512-byte line set.  The per-token
// coefficients are broadcast loads served by L1.  Activations use streaming
// (evict-first) loads and stores: nothing here is re-read.
#include "mhc_common.cuh"

namespace mhc {

template <typename TIO, int N>
__global__ void __launch_bounds__(256) k_post(int64_t T, int64_t C, const TIO* __restrict__ x,
                                              const TIO* __restrict__ f,
                                              const float* __restrict__ Hpost,
                                              const float* __restrict__ Hres,
                                              TIO* __restrict__ xn) {
  using V = Vec<TIO>;
  constexpr int W = V::N;
  const int64_t nv = C / W;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    float hr[N * N], hp[N];
#pragma unroll
    for (int e = 0; e < N * N; ++e) hr[e] = __ldg(Hres + t * N * N + e);
#pragma unroll
    for (int i = 0; i < N; ++i) hp[i] = __ldg(Hpost + t * N + i);
    const TIO* xt = x + t * N * C;
    TIO* ot = xn + t * N * C;
    for (int64_t v = threadIdx.x; v < nv; v += blockDim.x) {
      float xv[N][W], fv[W];
#pragma unroll
      for (int j = 0; j < N; ++j) V::load_stream(xt + j * C + v * W, xv[j]);
      V::load_stream(f + t * C + v * W, fv);
#pragma unroll
      for (int i = 0; i < N; ++i) {
        float o[W];
#pragma unroll
        for (int e = 0; e < W; ++e) {
          float acc = hp[i] * fv[e];
#pragma unroll
          for (int j = 0; j < N; ++j) acc = fmaf(hr[i * N + j], xv[j][e], acc);
          o[e] = acc;
        }
        V::store_stream(ot + i * C + v * W, o);
      }
    }
  }
}

template <typename TIO, int N>
__global__ void __launch_bounds__(256) k_hin(int64_t T, int64_t C, const TIO* __restrict__ x,
                                             const float* __restrict__ Hpre,
                                             TIO* __restrict__ h_in) {
  using V = Vec<TIO>;
  constexpr int W = V::N;
  const int64_t nv = C / W;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    float hp[N];
#pragma unroll
    for (int i = 0; i < N; ++i) hp[i] = __ldg(Hpre + t * N + i);
    const TIO* xt = x + t * N * C;
    for (int64_t v = threadIdx.x; v < nv; v += blockDim.x) {
      float xv[N][W];
#pragma unroll
      for (int j = 0; j < N; ++j) V::load_stream(xt + j * C + v * W, xv[j]);
      float o[W];
#pragma unroll
      for (int e = 0; e < W; ++e) {
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < N; ++j) acc = fmaf(hp[j], xv[j][e], acc);
        o[e] = acc;
      }
      V::store_stream(h_in + t * C + v * W, o);
    }
  }
}

static int mix_grid(int64_t T, int64_t nv, int block) {
  // enough CTAs to keep every SM's load queue full, one token per CTA visit
  int64_t per_token_blocks = 1;
  (void)nv;
  (void)block;
  int64_t g = T * per_token_blocks;
  const int64_t cap = 148 * 16;
  return (int)(g < cap ? g : cap);
}

template <typename TIO, int N>
static cudaError_t launch_post_t(int64_t T, int64_t C, const void* x, const void* f,
                                 const float* Hpost, const float* Hres, void* xn, cudaStream_t s) {
  const int block = 128;
  const int grid = mix_grid(T, C / Vec<TIO>::N, block);
  k_post<TIO, N><<<grid, block, 0, s>>>(T, C, (const TIO*)x, (const TIO*)f, Hpost, Hres, (TIO*)xn);
  return cudaGetLastError();
}

template <typename TIO, int N>
static cudaError_t launch_hin_t(int64_t T, int64_t C, const void* x, const float* Hpre,
                                void* h_in, cudaStream_t s) {
  const int block = 128;
  const int grid = mix_grid(T, C / Vec<TIO>::N, block);
  k_hin<TIO, N><<<grid, block, 0, s>>>(T, C, (const TIO*)x, Hpre, (TIO*)h_in);
  return cudaGetLastError();
}

cudaError_t post_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const void* f,
                          const float* Hpost, const float* Hres, void* xn, cudaStream_t s) {
#define MHC_POST_CASE(NN)                                                                   \
  case NN:                                                                                  \
    return dtype == MHC_DTYPE_BF16                                                          \
               ? launch_post_t<__nv_bfloat16, NN>(T, C, x, f, Hpost, Hres, xn, s)           \
               : launch_post_t<float, NN>(T, C, x, f, Hpost, Hres, xn, s);
  switch (n) {
    MHC_POST_CASE(1)
    MHC_POST_CASE(2)
    MHC_POST_CASE(4)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_POST_CASE
}

cudaError_t hin_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const float* Hpre,
                         void* h_in, cudaStream_t s) {
#define MHC_HIN_CASE(NN)                                                                    \
  case NN:                                                                                  \
    return dtype == MHC_DTYPE_BF16 ? launch_hin_t<__nv_bfloat16, NN>(T, C, x, Hpre, h_in, s) \
                                   : launch_hin_t<float, NN>(T, C, x, Hpre, h_in, s);
  switch (n) {
    MHC_HIN_CASE(1)
    MHC_HIN_CASE(2)
    MHC_HIN_CASE(4)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_HIN_CASE
}

}  // namespace mhc
