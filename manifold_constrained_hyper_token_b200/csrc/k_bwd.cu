// k_bwd.cu -- the second half of the mHC backward pass (CUDA-core path).
//
// Given the per-token coefficients that k_map<.., BWD=true> recomputed
// (H_res, H_pre, H_post, u = alpha dz / r, kappa), this pass writes
//
//   grad_x[j][c]  = sum_i H_res[i][j] G[i][c] + H_pre[j] g[c]
//                   + sum_m phi[jC+c][m] u[m] - kappa x[j][c]
//   grad_f_out[c] = sum_i H_post[i] G[i][c]     (skipped when grad_f is null:
//                                                 the split backward's pre half)
//   grad_phi[k][m] = sum_t x_t[k] u_t[m]
//
// and finishes grad_b = sum_t dz_t, grad_alpha = sum_t dz_t . y_t from the
// mapping kernel's per-CTA partial sums.
// (reverse mode of the update equation of the chatgpz.de explainer and of
// the RMS-normalised projection; reportify.cn [19]-[21].)
//
// Layout: a CTA owns a slice of CW channels of all n streams, i.e. n*CW rows
// of phi and grad_phi, and walks every token.  The phi rows and the grad_phi
// accumulators stay in registers for the whole kernel, so grad_phi needs no
// cross-CTA reduction: each row is written once, by its owner, after an
// in-CTA sum over warps taken in a fixed order.  Lanes of a warp cover
// (stream, channel) pairs of one token; the other streams' G values arrive by
// warp shuffle.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"

namespace mhc {

namespace bwdk {
constexpr int NT = 256;      // 8 warps
constexpr int NW = NT / 32;
constexpr int TB = 64;       // tokens per staged coefficient batch
}  // namespace bwdk

template <typename TIO, int N> struct ApplyShape {
  static constexpr int LPS = 32 / N;                                    // lanes per stream
  static constexpr int CPL = (sizeof(TIO) == 2 && N == 4) ? 2 : 1;      // channels per lane
  static constexpr int CW = LPS * CPL;                                  // channels per CTA
  static constexpr int M = N * N + 2 * N;
};

template <typename TIO, int N>
__global__ void __launch_bounds__(bwdk::NT) k_bwd_apply(
    int64_t T, int64_t C, const TIO* __restrict__ x, const float* __restrict__ phi,
    const TIO* __restrict__ G, const TIO* __restrict__ g, const float* __restrict__ coef,
    const float* __restrict__ part, int nparts, TIO* __restrict__ grad_x, TIO* __restrict__ grad_f,
    float* __restrict__ grad_phi, float* __restrict__ grad_b, float* __restrict__ grad_alpha,
    int ag) {
  using S = ApplyShape<TIO, N>;
  using CF = Coef<N>;
  using namespace bwdk;
  constexpr int LPS = S::LPS, CPL = S::CPL, M = S::M;
  extern __shared__ __align__(16) float sm[];
  float* cs = sm;  // [TB][CF::SIZE]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int j = lane / LPS, ls = lane % LPS;
  const int64_t c0 = (int64_t)blockIdx.x * S::CW + ls * CPL;
  bool cvalid[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) cvalid[e] = (c0 + e) < C;

  if (blockIdx.x == 0) {
    // grad_b and grad_alpha: add the mapping kernel's per-CTA partial sums.
    // Warp w takes partials w, w + NW, ... in order; the NW results are then
    // added in warp order -- a fixed order, so repeated calls agree bitwise.
    // Columns: M dz sums, then dz . y over the pre, post and res logits (M + 3
    // can exceed a warp's 32 lanes: n = 8 has 83).
    constexpr int NC = M + 3;
    float* wsum = sm;  // [NW][NC]
    for (int col = lane; col < NC; col += 32) {
      float s = 0.0f;
      for (int q = warp; q < nparts; q += NW) s += __ldg(part + (int64_t)q * CF::DZ_SIZE + col);
      wsum[warp * NC + col] = s;
    }
    __syncthreads();
    for (int col = threadIdx.x; col < NC; col += NT) {
      float a = 0.0f;
      for (int w = 0; w < NW; ++w) a += wsum[w * NC + col];
      wsum[NW * NC + col] = a;
      if (col < M) grad_b[col] = a;
      else if (ag == 3) grad_alpha[col - M] = a;
    }
    __syncthreads();
    // one shared alpha: its gradient is the sum of the three group sums
    if (ag != 3 && threadIdx.x == 0)
      *grad_alpha = (wsum[NW * NC + M] + wsum[NW * NC + M + 1]) + wsum[NW * NC + M + 2];
  }

  float ph[CPL][M], gp[CPL][M];
#pragma unroll
  for (int e = 0; e < CPL; ++e)
#pragma unroll
    for (int m = 0; m < M; ++m) {
      ph[e][m] = cvalid[e] ? __ldg(phi + ((int64_t)j * C + c0 + e) * M + m) : 0.0f;
      gp[e][m] = 0.0f;
    }

  for (int64_t tb = 0; tb < T; tb += TB) {
    const int nt = (int)((T - tb) < TB ? (T - tb) : TB);
    __syncthreads();
    {
      const float4* src = reinterpret_cast<const float4*>(coef + tb * CF::SIZE);
      float4* dst = reinterpret_cast<float4*>(cs);
      const int nv = nt * CF::SIZE / 4;
      for (int v = threadIdx.x; v < nv; v += NT) dst[v] = __ldg(src + v);
    }
    __syncthreads();
    for (int q = warp; q < nt; q += NW) {
      const int64_t t = tb + q;
      const float* ct = cs + q * CF::SIZE;
      float xv[CPL], Gv[CPL], gv[CPL];
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        xv[e] = cvalid[e] ? to_f32(x[(t * N + j) * C + c0 + e]) : 0.0f;
        Gv[e] = cvalid[e] ? to_f32(G[(t * N + j) * C + c0 + e]) : 0.0f;
        gv[e] = cvalid[e] ? to_f32(g[t * C + c0 + e]) : 0.0f;
      }
      float u[M];
#pragma unroll
      for (int m = 0; m < M; ++m) u[m] = ct[CF::U + m];
      const float kappa = ct[CF::KAPPA];
      float Gall[N][CPL];
#pragma unroll
      for (int i = 0; i < N; ++i)
#pragma unroll
        for (int e = 0; e < CPL; ++e) Gall[i][e] = __shfl_sync(0xffffffffu, Gv[e], i * LPS + ls);
      float gx[CPL], gf[CPL];
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        float pu = 0.0f;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          pu = fmaf(ph[e][m], u[m], pu);
          gp[e][m] = fmaf(xv[e], u[m], gp[e][m]);
        }
        float a = fmaf(ct[CF::PRE + j], gv[e], pu);
        float b = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) {
          a = fmaf(ct[CF::RES + i * N + j], Gall[i][e], a);
          b = fmaf(ct[CF::POST + i], Gall[i][e], b);
        }
        gx[e] = fmaf(-kappa, xv[e], a);
        gf[e] = b;
      }
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        if (cvalid[e]) {
          if constexpr (sizeof(TIO) == 2) {
            grad_x[(t * N + j) * C + c0 + e] = __float2bfloat16_rn(gx[e]);
            if (j == 0 && grad_f != nullptr) grad_f[t * C + c0 + e] = __float2bfloat16_rn(gf[e]);
          } else {
            grad_x[(t * N + j) * C + c0 + e] = gx[e];
            if (j == 0 && grad_f != nullptr) grad_f[t * C + c0 + e] = gf[e];
          }
        }
      }
    }
  }

  // grad_phi: add the warps' partial sums in warp order, then write.
  __syncthreads();
  float* red = sm;  // [NW][32][CPL*M]
#pragma unroll
  for (int e = 0; e < CPL; ++e)
#pragma unroll
    for (int m = 0; m < M; ++m) red[(warp * 32 + lane) * CPL * M + e * M + m] = gp[e][m];
  __syncthreads();
  constexpr int PER = 32 * CPL * M;
  for (int idx = threadIdx.x; idx < PER; idx += NT) {
    float s = 0.0f;
    for (int w = 0; w < NW; ++w) s += red[w * PER + idx];
    const int ln = idx / (CPL * M), rem = idx % (CPL * M);
    const int e = rem / M, m = rem % M;
    const int jj = ln / LPS, lss = ln % LPS;
    const int64_t c = (int64_t)blockIdx.x * S::CW + lss * CPL + e;
    if (c < C) grad_phi[((int64_t)jj * C + c) * M + m] = s;
  }
}

template <typename TIO, int N>
static cudaError_t launch_apply_t(int64_t T, int64_t C, const void* x, const float* phi,
                                  const void* G, const void* g, const float* coef,
                                  const float* part, int nparts, void* gx, void* gf, float* gphi,
                                  float* gb, float* ga, int ag, cudaStream_t s) {
  using S = ApplyShape<TIO, N>;
  using CF = Coef<N>;
  const size_t smem_c = (size_t)bwdk::TB * CF::SIZE * 4;
  const size_t smem_r = (size_t)bwdk::NW * 32 * S::CPL * S::M * 4;
  const size_t smem = smem_c > smem_r ? smem_c : smem_r;
  auto kern = k_bwd_apply<TIO, N>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (C + S::CW - 1) / S::CW;
  kern<<<(unsigned)grid, bwdk::NT, smem, s>>>(T, C, (const TIO*)x, phi, (const TIO*)G,
                                             (const TIO*)g, coef, part, nparts, (TIO*)gx,
                                             (TIO*)gf, gphi, gb, ga, ag);
  return cudaGetLastError();
}

cudaError_t apply_dispatch(int n, int dtype, int64_t T, int64_t C, const void* x, const float* phi,
                           const void* G, const void* g, const float* coef, const float* part,
                           int nparts, void* gx, void* gf, float* gphi, float* gb, float* ga,
                           int ag, cudaStream_t s) {
  if (n == 16)
    return wide_apply_dispatch(dtype, T, C, x, phi, G, g, coef, part, nparts, gx, gf, gphi, gb, ga,
                               ag, s);
#define MHC_APPLY(NN)                                                                        \
  case NN:                                                                                   \
    return dtype == MHC_DTYPE_BF16                                                           \
               ? launch_apply_t<__nv_bfloat16, NN>(T, C, x, phi, G, g, coef, part, nparts, gx, gf, \
                                                   gphi, gb, ga, ag, s)                              \
               : launch_apply_t<float, NN>(T, C, x, phi, G, g, coef, part, nparts, gx, gf, gphi,  \
                                           gb, ga, ag, s);
  switch (n) {
    MHC_APPLY(1)
    MHC_APPLY(2)
    MHC_APPLY(4)
    MHC_APPLY(8)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_APPLY
}

}  // namespace mhc
