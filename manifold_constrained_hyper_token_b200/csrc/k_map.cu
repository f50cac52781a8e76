// k_map.cu -- per-token mapping kernels on the CUDA cores (fp32 FMA):
//
//   forward   r = sqrt(mean x^2 + eps), y = (x . phi) / r, z = alpha_g y + b
//             (alpha_g: the scale of the logit's group, pre / post / res),
//             H_pre = sigmoid, H_post = 2 sigmoid, H_res = Sinkhorn(exp(z_res))
//   backward  the same recompute, plus the C-reductions
//               dH_pre[i] = <g, x_i>, dH_post[i] = <G_i, f>, dH_res[i][j] = <G_i, x_j>
//             the Sinkhorn adjoint and the gate derivatives, giving
//             dz, u = alpha_g dz / r and kappa = sum_m alpha_g dz_m y_m / (K r^2).
//
// Sources: the RMSNorm/projection/gating operator of the chatgpz.de explainer
// (section "Systemarbeit und Schulungsaufwand") and reportify.cn [17]-[19]:
// the RMS is applied after the projection (one pass over x), Sinkhorn and its
// custom backward run in the same operator, and the backward recomputes the
// mapping instead of storing it ([21]).
//
// Tiling: a CTA owns TM = 64 tokens and walks the token's n*C inputs in
// chunks of CC channels x n streams.  Each chunk is staged in shared memory
// transposed (token fastest) together with the matching phi rows; 256
// threads each accumulate a 4-token x (MP/4)-column block over a quarter of
// the chunk's rows, and the four quarters are added at the end in a fixed
// order.  Every sum in this file is taken in a fixed order: results are
// bitwise reproducible.  This is the fp32-I/O path; bf16 I/O projects on the
// tensor cores instead (k_map_tc.cu).
#include "mhc_common.cuh"
#include "mhc_dispatch.h"

namespace mhc {

namespace mapk {
constexpr int TM = 64;       // tokens per CTA
constexpr int CC = 16;       // channels per chunk (per stream)
constexpr int TMP = TM + 4;  // padded token stride of the staged x tile
constexpr int NT = 256;      // threads
}  // namespace mapk

// Four consecutive activations widened to fp32 (8-byte bf16 or 16-byte fp32
// load; the address is a multiple of 4 elements).
__device__ __forceinline__ void ld4(const float* p, float (&v)[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void ld4(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(q.x << 16);
  v[1] = __uint_as_float(q.x & 0xffff0000u);
  v[2] = __uint_as_float(q.y << 16);
  v[3] = __uint_as_float(q.y & 0xffff0000u);
}

template <int N> struct MapShape {
  static constexpr int M = N * N + 2 * N;
  static constexpr int MP = (M + 3) / 4 * 4;   // padded logit count
  static constexpr int CPG = MP / 4;           // logit columns per thread
  static constexpr int ROWS = N * mapk::CC;    // k-rows per chunk
  static constexpr int RQ = ROWS / 4;          // rows per k-quarter
  static constexpr int STAGE_FLOATS = ROWS * mapk::TMP + ROWS * MP;
};

template <typename TIO, int N>
static size_t map_smem_bytes() {
  using S = MapShape<N>;
  constexpr int VPS = mapk::CC / Vec<TIO>::N;
  size_t stage = (size_t)S::STAGE_FLOATS * 4;
  size_t red = ((size_t)4 * mapk::TM * S::MP + (size_t)mapk::TM * (S::M + 1) +
                (size_t)mapk::TM * N * VPS + (size_t)mapk::TM * (S::M + 3)) * 4;
  size_t two = 2 * stage;
  return two > red ? two : red;
}

// MAP_FWD      : write H_pre / H_post / H_res.
// MAP_BWD      : write coef [T][Coef<N>::SIZE] and, per CTA, the sums over its
//                tokens of dz and dz . y: part [gridDim.x][Coef<N>::DZ_SIZE].
// MAP_BWD_SPLIT: as MAP_BWD, but <G_i, x_j> and <G_i, f_out> come from the
//                post half's reductions `red` [T][n*n + n] (G and f unused).
template <typename TIO, int N, int MODE>
__global__ void __launch_bounds__(mapk::NT) k_map(
    int64_t T, int64_t C, int iters, float eps, const TIO* __restrict__ x,
    const float* __restrict__ phi, const float* __restrict__ bias, const float* __restrict__ alpha_p,
    int ag,
    // forward outputs
    float* __restrict__ Hpre_o, float* __restrict__ Hpost_o, float* __restrict__ Hres_o,
    // backward inputs / outputs
    const TIO* __restrict__ G, const TIO* __restrict__ g, const TIO* __restrict__ f,
    const float* __restrict__ red_in, float* __restrict__ coef_o, float* __restrict__ part_o,
    int* status) {
  constexpr bool BWD = MODE != MAP_FWD;
  constexpr bool SPLIT = MODE == MAP_BWD_SPLIT;
  using S = MapShape<N>;
  using V = Vec<TIO>;
  using namespace mapk;
  constexpr int W = V::N;
  constexpr int M = S::M, MP = S::MP, CPG = S::CPG, ROWS = S::ROWS, RQ = S::RQ;
  constexpr int VPS = CC / W;               // vectors per (token, stream) per chunk
  constexpr int NVEC = TM * N * VPS;        // vectors per chunk
  constexpr int NR = (NVEC + NT - 1) / NT;  // vectors per thread per chunk
  constexpr int NPHI = ROWS * MP;
  constexpr int PR = (NPHI + NT - 1) / NT;

  extern __shared__ __align__(16) float smem[];
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * TM;
  const int64_t K = (int64_t)N * C;
  const int64_t nchunks = (C + CC - 1) / CC;

  // compute role
  const int tg = tid % 16, cg = (tid / 16) % 4, kq = tid / 64;
  float acc[4][CPG];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < CPG; ++c) acc[a][c] = 0.0f;

  // staging role: thread owns vector slots v = tid + NT*r (fixed over chunks)
  float ssq[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) ssq[r] = 0.0f;

  // backward dot role: thread owns token dtok = tid / 4, channels sub*CC/4 ..
  const int dtok = tid / 4, dsub = tid % 4;
  constexpr int DCH = CC / 4;
  float dots[BWD ? M : 1];
#pragma unroll
  for (int m = 0; m < (BWD ? M : 1); ++m) dots[m] = 0.0f;

  float xr[NR][W];
  float pr[PR];

  auto load_chunk = [&](int64_t ch) {
    const int64_t cbase = ch * CC;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int v = tid + NT * r;
      const int tok = v / (N * VPS), rest = v % (N * VPS);
      const int i = rest / VPS, q = rest % VPS;
      const int64_t c = cbase + q * W;
      const int64_t t = t0 + tok;
      if (v < NVEC && t < T && c < C) {
        V::load_stream(x + (t * N + i) * C + c, xr[r]);
      } else {
#pragma unroll
        for (int e = 0; e < W; ++e) xr[r][e] = 0.0f;
      }
    }
#pragma unroll
    for (int r = 0; r < PR; ++r) {
      const int e = tid + NT * r;
      const int row = e / MP, m = e % MP;
      const int i = row / CC, cl = row % CC;
      const int64_t c = cbase + cl;
      pr[r] = (e < NPHI && m < M && c < C) ? __ldg(phi + (i * C + c) * M + m) : 0.0f;
    }
  };
  auto store_chunk = [&](float* stage) {
    float* xs = stage;
    float* ps = stage + ROWS * TMP;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int v = tid + NT * r;
      if (v < NVEC) {
        const int tok = v / (N * VPS), rest = v % (N * VPS);
        const int i = rest / VPS, q = rest % VPS;
#pragma unroll
        for (int e = 0; e < W; ++e) {
          xs[(i * CC + q * W + e) * TMP + tok] = xr[r][e];
          ssq[r] = fmaf(xr[r][e], xr[r][e], ssq[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < PR; ++r) {
      const int e = tid + NT * r;
      if (e < NPHI) ps[e] = pr[r];
    }
  };

  load_chunk(0);
  store_chunk(smem);
  __syncthreads();
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    float* cur = smem + (ch & 1) * S::STAGE_FLOATS;
    float* nxt = smem + ((ch + 1) & 1) * S::STAGE_FLOATS;
    if (ch + 1 < nchunks) load_chunk(ch + 1);
    const float* xs = cur;
    const float* ps = cur + ROWS * TMP;
    // projection partials
#pragma unroll 4
    for (int rr = 0; rr < RQ; ++rr) {
      const int row = kq * RQ + rr;
      const float4 xv = *reinterpret_cast<const float4*>(xs + row * TMP + 4 * tg);
      float pv[CPG];
#pragma unroll
      for (int c = 0; c < CPG; ++c) pv[c] = ps[row * MP + cg * CPG + c];
#pragma unroll
      for (int c = 0; c < CPG; ++c) {
        acc[0][c] = fmaf(xv.x, pv[c], acc[0][c]);
        acc[1][c] = fmaf(xv.y, pv[c], acc[1][c]);
        acc[2][c] = fmaf(xv.z, pv[c], acc[2][c]);
        acc[3][c] = fmaf(xv.w, pv[c], acc[3][c]);
      }
    }
    if constexpr (BWD) {
      const int64_t t = t0 + dtok;
      const int64_t cb = ch * CC + dsub * DCH;
      // C is a multiple of 8 and cb of 4: the DCH = 4 channels are all in range
      // or all out, and each row's 4 values are one aligned vector load
      static_assert(DCH == 4, "four channels per reduction thread");
      if (t < T && cb < C) {
        float Gq[N][DCH], gq[DCH], fq[DCH];
#pragma unroll
        for (int i = 0; i < N; ++i) {
          if constexpr (SPLIT) {
#pragma unroll
            for (int e = 0; e < DCH; ++e) Gq[i][e] = 0.0f;
          } else {
            ld4(G + (t * N + i) * C + cb, Gq[i]);
          }
        }
        ld4(g + t * C + cb, gq);
        if constexpr (SPLIT) {
#pragma unroll
          for (int e = 0; e < DCH; ++e) fq[e] = 0.0f;
        } else {
          ld4(f + t * C + cb, fq);
        }
#pragma unroll
        for (int e = 0; e < DCH; ++e) {
          {
            float xv[N], Gv[N];
#pragma unroll
            for (int i = 0; i < N; ++i) {
              xv[i] = xs[(i * CC + dsub * DCH + e) * TMP + dtok];
              Gv[i] = Gq[i][e];
            }
            const float gv = gq[e];
            const float fv = fq[e];
            if constexpr (SPLIT) {
#pragma unroll
              for (int i = 0; i < N; ++i) dots[N * N + i] = fmaf(gv, xv[i], dots[N * N + i]);
            } else {
#pragma unroll
            for (int i = 0; i < N; ++i) {
#pragma unroll
              for (int j = 0; j < N; ++j) dots[i * N + j] = fmaf(Gv[i], xv[j], dots[i * N + j]);
              dots[N * N + i] = fmaf(gv, xv[i], dots[N * N + i]);
              dots[N * N + N + i] = fmaf(Gv[i], fv, dots[N * N + N + i]);
            }
            }
          }
        }
      }
    }
    if (ch + 1 < nchunks) store_chunk(nxt);
    __syncthreads();
  }

  // ---- reduce partials in a fixed order
  float* red = smem;                     // [4][TM][MP]
  float* ssr = smem + 4 * TM * MP;       // [TM] sum of squares, then [TM][M] dots
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < CPG; ++c) red[(kq * TM + 4 * tg + a) * MP + cg * CPG + c] = acc[a][c];
  // sum of squares: slots of one token are spread over threads; gather them
  // into a [TM][N*VPS] table and add in slot order.
  float* sst = ssr + TM * (BWD ? M + 1 : 1);  // [TM][N*VPS]
  float* dzs = sst + TM * N * VPS;            // [TM][M+3] (backward)
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int v = tid + NT * r;
    if (v < NVEC) sst[v] = ssq[r];
  }
  if constexpr (BWD) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float d = dots[m];
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      dots[m] = d;
    }
    if (dsub == 0) {
#pragma unroll
      for (int m = 0; m < M; ++m) ssr[TM + dtok * M + m] = dots[m];
    }
  }
  __syncthreads();

  if (tid < TM) {
    const int64_t t = t0 + tid;
    if (t < T) {
      float ss = 0.0f;
      for (int s = 0; s < N * VPS; ++s) ss += sst[tid * N * VPS + s];
      const float r = sqrtf(ss / (float)K + eps);
      Alpha3 al;
      al.load(alpha_p, ag);
      float y[M], z[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float yr = red[(0 * TM + tid) * MP + m] + red[(1 * TM + tid) * MP + m] +
                         red[(2 * TM + tid) * MP + m] + red[(3 * TM + tid) * MP + m];
        y[m] = yr / r;
        z[m] = fmaf(al.at<N>(m), y[m], __ldg(bias + m));
      }
      bool bad = !isfinite(r);
#pragma unroll
      for (int m = 0; m < M; ++m) bad |= !isfinite(z[m]);
      if (bad) flag_status(status, MHC_ERR_NONFINITE);
      float spre[N], spost[N];
#pragma unroll
      for (int i = 0; i < N; ++i) {
        spre[i] = sigmoidf_(z[i]);
        spost[i] = sigmoidf_(z[N + i]);
      }
      float zres[N * N], H[N * N];
#pragma unroll
      for (int e = 0; e < N * N; ++e) zres[e] = H[e] = z[2 * N + e];
      sk_forward<N>(H, iters);
      if constexpr (!BWD) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
          Hpre_o[t * N + i] = spre[i];
          Hpost_o[t * N + i] = 2.0f * spost[i];
        }
#pragma unroll
        for (int e = 0; e < N * N; ++e) Hres_o[t * N * N + e] = H[e];
      } else {
        const float* dt = ssr + TM + tid * M;
        const float* rt = red_in + (SPLIT ? t * (N * N + N) : 0);
        float dA[N * N], dz[M];
#pragma unroll
        for (int e = 0; e < N * N; ++e) dA[e] = SPLIT ? __ldg(rt + e) : dt[e];
        float dzres[N * N];
        sk_adjoint<N>(zres, dA, dzres, iters);
#pragma unroll
        for (int i = 0; i < N; ++i) {
          dz[i] = dt[N * N + i] * spre[i] * (1.0f - spre[i]);
          dz[N + i] = (SPLIT ? __ldg(rt + N * N + i) : dt[N * N + N + i]) * 2.0f * spost[i] *
                      (1.0f - spost[i]);
        }
#pragma unroll
        for (int e = 0; e < N * N; ++e) dz[2 * N + e] = dzres[e];
        float dzy[3] = {0.0f, 0.0f, 0.0f};  // dz . y over the pre, post, res logits
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const int grp = m < N ? 0 : (m < 2 * N ? 1 : 2);
          dzy[grp] = fmaf(dz[m], y[m], dzy[grp]);
        }
        using CF = Coef<N>;
        float* co = coef_o + t * CF::SIZE;
#pragma unroll
        for (int e = 0; e < N * N; ++e) co[CF::RES + e] = H[e];
#pragma unroll
        for (int i = 0; i < N; ++i) {
          co[CF::PRE + i] = spre[i];
          co[CF::POST + i] = 2.0f * spost[i];
        }
        float ar[3];
#pragma unroll
        for (int g = 0; g < 3; ++g) ar[g] = al.a[g] / r;
#pragma unroll
        for (int m = 0; m < M; ++m) co[CF::U + m] = ar[m < N ? 0 : (m < 2 * N ? 1 : 2)] * dz[m];
        const float wdzy = fmaf(al.a[2], dzy[2], fmaf(al.a[1], dzy[1], al.a[0] * dzy[0]));
        co[CF::KAPPA] = wdzy / ((float)K * r * r);
#pragma unroll
        for (int m = 0; m < M; ++m) dzs[tid * (M + 3) + m] = dz[m];
#pragma unroll
        for (int g = 0; g < 3; ++g) dzs[tid * (M + 3) + M + g] = dzy[g];
      }
    } else if constexpr (BWD) {
#pragma unroll
      for (int m = 0; m < M + 3; ++m) dzs[tid * (M + 3) + m] = 0.0f;
    }
  }
  if constexpr (BWD) {
    // this CTA's share of grad_b and the three grad_alpha sums, in token order
    __syncthreads();
    if (tid < M + 3) {
      float s = 0.0f;
      for (int q = 0; q < TM; ++q) s += dzs[q * (M + 3) + tid];
      part_o[(int64_t)blockIdx.x * Coef<N>::DZ_SIZE + tid] = s;
    }
  }
}

template <typename TIO, int N, int MODE>
static cudaError_t launch_map_t(int64_t T, int64_t C, int iters, float eps, const void* x,
                                const float* phi, const float* b, const float* alpha, int ag,
                                float* Hpre, float* Hpost, float* Hres, const void* G,
                                const void* g, const void* f, const float* red, float* coef,
                                float* part, int* st, cudaStream_t s) {
  const size_t smem = map_smem_bytes<TIO, N>();
  auto kern = k_map<TIO, N, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (T + mapk::TM - 1) / mapk::TM;
  kern<<<(unsigned)grid, mapk::NT, smem, s>>>(T, C, iters, eps, (const TIO*)x, phi, b, alpha, ag, Hpre,
                                             Hpost, Hres, (const TIO*)G, (const TIO*)g,
                                             (const TIO*)f, red, coef, part, st);
  return cudaGetLastError();
}

cudaError_t map_fwd_dispatch(int n, int dtype, int64_t T, int64_t C, int iters, float eps,
                             const void* x, const float* phi, const float* b, const float* alpha,
                             int ag,
                             float* Hpre, float* Hpost, float* Hres, int* st, cudaStream_t s) {
  if (n == 16)
    return wide_map_dispatch(MAP_FWD, dtype, T, C, iters, eps, x, phi, b, alpha, ag, Hpre, Hpost,
                             Hres, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, st, s);
#define MHC_MAPF(NN)                                                                             \
  case NN:                                                                                       \
    return dtype == MHC_DTYPE_BF16                                                               \
               ? launch_map_t<__nv_bfloat16, NN, MAP_FWD>(T, C, iters, eps, x, phi, b, alpha, ag,    \
                                                          Hpre, Hpost, Hres, nullptr, nullptr,   \
                                                          nullptr, nullptr, nullptr, nullptr,    \
                                                          st, s)                                 \
               : launch_map_t<float, NN, MAP_FWD>(T, C, iters, eps, x, phi, b, alpha, ag, Hpre,      \
                                                  Hpost, Hres, nullptr, nullptr, nullptr,        \
                                                  nullptr, nullptr, nullptr, st, s);
  switch (n) {
    MHC_MAPF(1)
    MHC_MAPF(2)
    MHC_MAPF(4)
    MHC_MAPF(8)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_MAPF
}

template <typename TIO, int N>
static cudaError_t map_bwd_n(int64_t T, int64_t C, int iters, float eps, const void* x,
                             const float* phi, const float* b, const float* alpha, int ag,
                             const void* G,
                             const void* g, const void* f, const float* red, float* coef,
                             float* part, int* st, cudaStream_t s) {
  return red == nullptr
             ? launch_map_t<TIO, N, MAP_BWD>(T, C, iters, eps, x, phi, b, alpha, ag, nullptr, nullptr,
                                             nullptr, G, g, f, nullptr, coef, part, st, s)
             : launch_map_t<TIO, N, MAP_BWD_SPLIT>(T, C, iters, eps, x, phi, b, alpha, ag, nullptr,
                                                   nullptr, nullptr, nullptr, g, nullptr, red,
                                                   coef, part, st, s);
}

cudaError_t map_bwd_dispatch(int n, int dtype, int64_t T, int64_t C, int iters, float eps,
                             const void* x, const float* phi, const float* b, const float* alpha,
                             int ag,
                             const void* G, const void* g, const void* f, const float* red,
                             float* coef, float* part, int* st, cudaStream_t s) {
  if (n == 16)
    return wide_map_dispatch(red == nullptr ? MAP_BWD : MAP_BWD_SPLIT, dtype, T, C, iters, eps, x,
                             phi, b, alpha, ag, nullptr, nullptr, nullptr, G, g, f, red, coef,
                             part, st, s);
#define MHC_MAPB(NN)                                                                          \
  case NN:                                                                                    \
    return dtype == MHC_DTYPE_BF16                                                            \
               ? map_bwd_n<__nv_bfloat16, NN>(T, C, iters, eps, x, phi, b, alpha, ag, G, g, f, red, \
                                              coef, part, st, s)                              \
               : map_bwd_n<float, NN>(T, C, iters, eps, x, phi, b, alpha, ag, G, g, f, red, coef,   \
                                      part, st, s);
  switch (n) {
    MHC_MAPB(1)
    MHC_MAPB(2)
    MHC_MAPB(4)
    MHC_MAPB(8)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_MAPB
}

}  // namespace mhc
