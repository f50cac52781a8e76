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
#include "mhc_dispatch.h"

namespace mhc {

template <typename TIO, int N>
__global__ void __launch_bounds__(256) k_post(int64_t T, int64_t C, const TIO* __restrict__ x,
                                              const TIO* __restrict__ f,
                                              const float* __restrict__ Hpost,
                                              const float* __restrict__ Hres,
                                              TIO* __restrict__ xn) {
  using V = Vec<TIO>;
  constexpr int W = V::N;
  // n >= 8: the token's coefficients sit in shared memory (broadcast reads), so
  // that the registers hold only the streams' values and two CTAs fit an SM
  constexpr bool SH = N >= 8;
  __shared__ float hs[SH ? N * N + N : 1];
  const int64_t nv = C / W;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    float hr[SH ? 1 : N * N], hp[SH ? 1 : N];
    if constexpr (SH) {
      __syncthreads();
      for (int e = threadIdx.x; e < N * N + N; e += blockDim.x)
        hs[e] = e < N * N ? __ldg(Hres + t * N * N + e) : __ldg(Hpost + t * N + (e - N * N));
      __syncthreads();
    } else {
#pragma unroll
      for (int e = 0; e < N * N; ++e) hr[e] = __ldg(Hres + t * N * N + e);
#pragma unroll
      for (int i = 0; i < N; ++i) hp[i] = __ldg(Hpost + t * N + i);
    }
    auto HR = [&](int e) { return SH ? hs[e] : hr[e]; };
    auto HP = [&](int i) { return SH ? hs[N * N + i] : hp[i]; };
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
          float acc = HP(i) * fv[e];
#pragma unroll
          for (int j = 0; j < N; ++j) acc = fmaf(HR(i * N + j), xv[j][e], acc);
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
  // Two vectors per thread per pass: all 2N loads are issued before the first
  // is used, so twice as many bytes are in flight per thread.
  using V = Vec<TIO>;
  constexpr int W = V::N;
  const int64_t nv = C / W;
  const int64_t step = 2 * (int64_t)blockDim.x;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    float hp[N];
#pragma unroll
    for (int i = 0; i < N; ++i) hp[i] = __ldg(Hpre + t * N + i);
    const TIO* xt = x + t * N * C;
    for (int64_t v0 = threadIdx.x; v0 < nv; v0 += step) {
      const int64_t v1 = v0 + blockDim.x;
      const bool two = v1 < nv;
      float xa[N][W], xb[N][W];
#pragma unroll
      for (int j = 0; j < N; ++j) V::load_stream(xt + j * C + v0 * W, xa[j]);
      if (two) {
#pragma unroll
        for (int j = 0; j < N; ++j) V::load_stream(xt + j * C + v1 * W, xb[j]);
      }
      float o[W];
#pragma unroll
      for (int e = 0; e < W; ++e) {
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < N; ++j) acc = fmaf(hp[j], xa[j][e], acc);
        o[e] = acc;
      }
      V::store_stream(h_in + t * C + v0 * W, o);
      if (two) {
#pragma unroll
        for (int e = 0; e < W; ++e) {
          float acc = 0.0f;
#pragma unroll
          for (int j = 0; j < N; ++j) acc = fmaf(hp[j], xb[j][e], acc);
          o[e] = acc;
        }
        V::store_stream(h_in + t * C + v1 * W, o);
      }
    }
  }
}

// Reverse of the post merge alone (first half of the layer backward in
// training order), with the forward's H_post:
//   grad_f_out[c] = sum_i H_post[i] G_i[c]
//   red = [ <G_i, x_j> (row-major i, j) | <G_i, f_out> ]      per token
// One CTA per token visit, threads over 16-byte channel vectors as above;
// each thread keeps the n*n + n partial dot products of its vectors, then the
// CTA adds them in a fixed order (xor tree inside a warp, warps in index
// order), so repeated calls give identical bits.
template <typename TIO, int N>
__global__ void __launch_bounds__(128) k_post_bwd(int64_t T, int64_t C, const TIO* __restrict__ x,
                                                  const TIO* __restrict__ f,
                                                  const float* __restrict__ Hpost,
                                                  const TIO* __restrict__ G,
                                                  TIO* __restrict__ gf, float* __restrict__ red) {
  using V = Vec<TIO>;
  constexpr int W = V::N;
  constexpr int R = N * N + N;
  __shared__ float wsum[4][R];
  const int64_t nv = C / W;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    float hp[N];
#pragma unroll
    for (int i = 0; i < N; ++i) hp[i] = __ldg(Hpost + t * N + i);
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.0f;
    const TIO* xt = x + t * N * C;
    const TIO* Gt = G + t * N * C;
    for (int64_t v = threadIdx.x; v < nv; v += blockDim.x) {
      float xv[N][W], Gv[N][W], fv[W];
#pragma unroll
      for (int j = 0; j < N; ++j) V::load_stream(xt + j * C + v * W, xv[j]);
#pragma unroll
      for (int i = 0; i < N; ++i) V::load_stream(Gt + i * C + v * W, Gv[i]);
      V::load_stream(f + t * C + v * W, fv);
      float o[W];
#pragma unroll
      for (int e = 0; e < W; ++e) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) a = fmaf(hp[i], Gv[i][e], a);
        o[e] = a;
      }
      V::store_stream(gf + t * C + v * W, o);
#pragma unroll
      for (int i = 0; i < N; ++i) {
#pragma unroll
        for (int e = 0; e < W; ++e) {
#pragma unroll
          for (int j = 0; j < N; ++j) acc[i * N + j] = fmaf(Gv[i][e], xv[j][e], acc[i * N + j]);
          acc[N * N + i] = fmaf(Gv[i][e], fv[e], acc[N * N + i]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float v = acc[r];
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
      acc[r] = v;
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) wsum[warp][r] = acc[r];
    }
    __syncthreads();
    if (threadIdx.x < R) {
      const int r = threadIdx.x;
      red[t * R + r] = ((wsum[0][r] + wsum[1][r]) + wsum[2][r]) + wsum[3][r];
    }
    __syncthreads();
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
  if (n == 16) return wide_post_dispatch(dtype, T, C, x, f, Hpost, Hres, xn, s);
#define MHC_POST_CASE(NN)                                                                   \
  case NN:                                                                                  \
    return dtype == MHC_DTYPE_BF16                                                          \
               ? launch_post_t<__nv_bfloat16, NN>(T, C, x, f, Hpost, Hres, xn, s)           \
               : launch_post_t<float, NN>(T, C, x, f, Hpost, Hres, xn, s);
  switch (n) {
    MHC_POST_CASE(1)
    MHC_POST_CASE(2)
    MHC_POST_CASE(4)
    MHC_POST_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_POST_CASE
}

template <typename TIO, int N>
static cudaError_t launch_post_bwd_t(int64_t T, int64_t C, const void* x, const void* f,
                                     const float* Hpost, const void* G, void* gf, float* red,
                                     cudaStream_t s) {
  const int block = 128;  // the fixed reduction order above assumes exactly 4 warps
  const int grid = mix_grid(T, C / Vec<TIO>::N, block);
  k_post_bwd<TIO, N><<<grid, block, 0, s>>>(T, C, (const TIO*)x, (const TIO*)f, Hpost,
                                            (const TIO*)G, (TIO*)gf, red);
  return cudaGetLastError();
}

cudaError_t post_bwd_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const void* f,
                              const float* Hpost, const void* G, void* gf, float* red,
                              cudaStream_t s) {
  if (n == 16) return wide_post_bwd_dispatch(dtype, T, C, x, f, Hpost, G, gf, red, s);
#define MHC_PBWD_CASE(NN)                                                                      \
  case NN:                                                                                     \
    return dtype == MHC_DTYPE_BF16                                                             \
               ? launch_post_bwd_t<__nv_bfloat16, NN>(T, C, x, f, Hpost, G, gf, red, s)         \
               : launch_post_bwd_t<float, NN>(T, C, x, f, Hpost, G, gf, red, s);
  switch (n) {
    MHC_PBWD_CASE(1)
    MHC_PBWD_CASE(2)
    MHC_PBWD_CASE(4)
    MHC_PBWD_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_PBWD_CASE
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
    MHC_HIN_CASE(8)
    MHC_HIN_CASE(16)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_HIN_CASE
}

}  // namespace mhc
