// k_wide.cu -- the mHC layer for a wide stream buffer (n = 16) on the CUDA cores.
//
// The same operators as k_map / k_post / k_bwd (the RMS-normalised
// projection, the gates, Sinkhorn-Knopp and its adjoint, the post merge and
// the backward apply; chatgpz.de explainer, sections "Von
// Residualverbindungen zu Hyperverbindungen" and "Systemarbeit und
// Schulungsaufwand"; reportify.cn [16]-[21]).  At n = 16 a token has M = 288
// logits and a 16 x 16 residual mixer, so the per-thread register tiling of
// those kernels does not fit.  Here:
//
//   k_wide_map        32 tokens per CTA: the projection y = x . phi as a
//                     CUDA-core GEMM over the flattened k = i*C + c (with the
//                     sum of squares); the forward then runs the gates and
//                     Sinkhorn one thread per token; the backward adds the
//                     288 C-reductions per token and stages y, the dot
//                     products and the sum of squares in each token's
//                     coefficient row
//   k_wide_bwd_epi_thread  the backward's per-token epilogue, one thread per
//                     token in a one-warp CTA of 32 tokens: gates, Sinkhorn
//                     and its adjoint, the coefficient record written over the
//                     staged row, and the tile's grad_b / grad_alpha partial
//                     sums
//   k_wide_post       x_next = H_res x + H_post^T f_out, coefficients in
//                     shared memory
//   k_wide_post_bwd   the post half of the backward in training order:
//                     grad_f_out and <G_i, x_j>, <G_i, f_out>
//   k_wide_apply_x    grad_x = phi u + H_res^T G + H_pre g - kappa x and
//                     grad_f_out for 32 tokens x 4 channels of all streams,
//                     the phi u term a GEMM over the logits
//   k_wide_apply_phi  grad_phi = sum_t x_t u_t^T, a GEMM over the tokens
//   k_wide_bias       grad_b and grad_alpha from the mapping CTAs' partials
//
// With bf16 activations the projection, the backward's C-reductions and the
// apply run on the tensor cores instead (k_proj16_tc.cu writes y and the sum of
// squares into the rows, k_dots_tc.cu the C-reductions; here k_wide_fwd_epi
// and k_wide_bwd_epi run the epilogues from those rows with 16 lanes per
// token, one row of the 16 x 16 Sinkhorn matrix per lane, the adjoint from
// every second iterate kept in a global scratch; k_apply16_tc.cu is the apply,
// with k_wide_bias for its grad_b and grad_alpha).
//
// Every sum is taken in a fixed order, so repeated calls give identical bits.
// On the fp32 path the per-token Sinkhorn arrays (16 x 16) live in local
// memory, one token per thread.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"

namespace mhc {

namespace widek {
constexpr int N = 16;
constexpr int M = N * N + 2 * N;   // 288 logits
constexpr int TB = 32;             // tokens per mapping CTA
constexpr int NT = 256;
constexpr int KC = 32;             // projection: k rows per chunk
constexpr int CPT = M / 32;        // logit columns (or dot products) per thread: 9
static_assert(KC * M % NT == 0, "phi chunk split over the threads");
constexpr int CQ = 8;              // reductions: channels per chunk
constexpr int CQP = CQ + 1;        // padded stride of a (token, stream) row
// shared memory of k_wide_map, in floats
constexpr int STG = KC * TB + KC * M;             // 10240: staging (projection)
constexpr int RED_STG = 2 * TB * N * CQP + 2 * TB * CQ;  // 9728: staging (reductions)
constexpr int DZS = TB * (M + 3);                 // 9312: the epilogue's dz rows
static_assert(RED_STG <= STG && DZS <= STG, "staging area");
constexpr int YS_OFF = STG;                       // [TB][M] projections
constexpr int DT_OFF = YS_OFF + TB * M;           // [TB][M] C-reductions
constexpr int SS_OFF = DT_OFF + TB * M;           // [TB] sums of squares
constexpr int SMEM_FLOATS = SS_OFF + TB;
}  // namespace widek

enum WideDots { WD_FULL = 0, WD_PRE = 1, WD_POST = 2 };

// Sinkhorn checkpoints of the backward epilogue on the tensor-core path: every
// second normalisation, iters + 1 iterates of N*N floats per token, laid out
// per token as [iterate][row][column].
constexpr int kWideCkPeriod = 2;

namespace widek {
constexpr int EPI_NT = TB * N;     // the tensor-core path's epilogues: 16 lanes per token
constexpr int TBS = N * N + N;     // floats per token of their transpose buffers (272)
}  // namespace widek

// ------------------------------------------------- 16 lanes per 16 x 16 matrix
// Sinkhorn-Knopp and its adjoint for one token's 16 x 16 matrix spread over
// 16 lanes of a warp: lane i of the half-warp holds row i in registers.  A row
// pass is local to the lane; a column pass goes through the half-warp's
// transpose buffer tb (256 floats; row r stored rotated by r, so that both the
// row writes and the column reads hit 16 different banks) and the 16 floats
// vb that follow it (a token's area is TBS = 272 floats).  Both
// half-warps of a warp run the same steps (the __syncwarp calls are
// warp-wide).  Every sum runs in a fixed order (a row's columns, a column's
// rows, in index order).
__device__ __forceinline__ void sk16_init(float (&a)[widek::N], int iters) {
  constexpr int N = widek::N;
  float mx = 0.0f;
  if (iters > 0) {
    mx = a[0];
#pragma unroll
    for (int j = 1; j < N; ++j) mx = fmaxf(mx, a[j]);
  }
#pragma unroll
  for (int j = 0; j < N; ++j) a[j] = expf(a[j] - mx);
}

// Normalisation q (odd: rows, even: columns); returns the sum this lane's row
// (odd q) or column i (even q) was divided by.
__device__ __forceinline__ float sk16_step(float (&a)[widek::N], int q, int i, float* tb,
                                           float* vb) {
  constexpr int N = widek::N;
  if (q & 1) {
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < N; ++j) acc += a[j];
    const float inv = 1.0f / acc;
#pragma unroll
    for (int j = 0; j < N; ++j) a[j] *= inv;
    return acc;
  }
#pragma unroll
  for (int j = 0; j < N; ++j) tb[i * N + ((j + i) & (N - 1))] = a[j];
  __syncwarp();
  float acc = 0.0f;
#pragma unroll
  for (int r = 0; r < N; ++r) acc += tb[r * N + ((i + r) & (N - 1))];
  vb[i] = 1.0f / acc;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < N; ++j) a[j] *= vb[j];
  __syncwarp();  // tb and vb are rewritten by the next column pass
  return acc;
}

// One step of the adjoint: a is the iterate after normalisation q, s the sum
// this lane's row (odd q) or column i (even q) was divided by, g the gradient
// with respect to that iterate (this lane's row), turned into the gradient
// with respect to the iterate before the step:
//   rows:    g_ij <- (g_ij - sum_k g_ik a_ik) / s_i
//   columns: g_ij <- (g_ij - sum_k g_kj a_kj) / s_j
__device__ __forceinline__ void sk16_adjoint_step(const float (&a)[widek::N], float s,
                                                  float (&g)[widek::N], int q, int i, float* tb,
                                                  float* vb) {
  constexpr int N = widek::N;
  if (q & 1) {
    float d = 0.0f;
#pragma unroll
    for (int j = 0; j < N; ++j) d = fmaf(g[j], a[j], d);
    const float inv = 1.0f / s;
#pragma unroll
    for (int j = 0; j < N; ++j) g[j] = (g[j] - d) * inv;
    return;
  }
#pragma unroll
  for (int j = 0; j < N; ++j) tb[i * N + ((j + i) & (N - 1))] = g[j] * a[j];
  __syncwarp();
  float d = 0.0f;
#pragma unroll
  for (int r = 0; r < N; ++r) d += tb[r * N + ((i + r) & (N - 1))];
  __syncwarp();  // every column is read: tb's first row takes the reciprocals
  vb[i] = d;
  tb[i] = 1.0f / s;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < N; ++j) g[j] = (g[j] - vb[j]) * tb[j];
  __syncwarp();
}

// sum over the 16 lanes of a half-warp, the same bits in every lane
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The C-reductions of one CTA's TB tokens, as dacc[token 4*ty + i][dot tx + 32q]:
//   dot d < 256         <G_i, x_j>   (i = d / 16, j = d % 16)        WD_FULL, WD_POST
//   256 <= d < 272      <g, x_i>     (i = d - 256)                    WD_FULL, WD_PRE
//   272 <= d < 288      <G_i, f>     (i = d - 272)                    WD_FULL, WD_POST
// Channels are taken in chunks of CQ, in order.  With WD_POST the chunk loop
// also writes grad_f_out = sum_i H_post[i] G_i (hp: [TB][N] in shared memory).
template <typename TIO, int WHICH>
__device__ __forceinline__ void wide_dots(int64_t T, int64_t C, int64_t t0, const TIO* x,
                                          const TIO* G, const TIO* g, const TIO* f,
                                          const float* hp, TIO* gf, float* stg,
                                          float (&dacc)[4][widek::CPT]) {
  using namespace widek;
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  float* xq = stg;                        // [TB][N][CQP]
  float* Gq = xq + TB * N * CQP;          // [TB][N][CQP]
  float* gq = Gq + TB * N * CQP;          // [TB][CQ]
  float* fq = gq + TB * CQ;               // [TB][CQ]
  constexpr bool USE_G = WHICH != WD_PRE;
  constexpr bool USE_g = WHICH != WD_POST;
  constexpr bool USE_f = WHICH != WD_PRE;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < CPT; ++q) dacc[i][q] = 0.0f;
  for (int64_t c0 = 0; c0 < C; c0 += CQ) {
    // (token, stream, channel) elements: TB * N * CQ = 4096, 16 per thread; all
    // loads are issued before the first store, so their latencies overlap
    constexpr int RX = TB * N * CQ / NT;
    float xl[RX], Gl[RX];
#pragma unroll
    for (int r = 0; r < RX; ++r) {
      const int e = tid + NT * r;
      const int cc = e & (CQ - 1), j = (e >> 3) & (N - 1), tok = e >> 7;
      const int64_t t = t0 + tok, c = c0 + cc;
      const bool ok = t < T && c < C;
      const int64_t gi = (t * N + j) * C + c;
      xl[r] = ok ? to_f32(x[gi]) : 0.0f;
      if constexpr (USE_G) Gl[r] = ok ? to_f32(G[gi]) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < RX; ++r) {
      const int e = tid + NT * r;
      const int cc = e & (CQ - 1), j = (e >> 3) & (N - 1), tok = e >> 7;
      xq[(tok * N + j) * CQP + cc] = xl[r];
      if constexpr (USE_G) Gq[(tok * N + j) * CQP + cc] = Gl[r];
    }
    {
      // (token, channel) elements: TB * CQ = 256, one per thread
      const int cc = tid & (CQ - 1), tok = tid >> 3;
      const int64_t t = t0 + tok, c = c0 + cc;
      const bool ok = t < T && c < C;
      if constexpr (USE_g) gq[tid] = ok ? to_f32(g[t * C + c]) : 0.0f;
      if constexpr (USE_f) fq[tid] = ok ? to_f32(f[t * C + c]) : 0.0f;
    }
    __syncthreads();
    if constexpr (WHICH == WD_POST) {
      // grad_f_out for (token tid / CQ, channel tid % CQ)
      const int cc = tid & (CQ - 1), tok = tid >> 3;
      const int64_t t = t0 + tok, c = c0 + cc;
      if (t < T && c < C) {
        float b = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) b = fmaf(hp[tok * N + i], Gq[(tok * N + i) * CQP + cc], b);
        if constexpr (sizeof(TIO) == 2) gf[t * C + c] = __float2bfloat16_rn(b);
        else gf[t * C + c] = b;
      }
    }
#pragma unroll
    for (int cc = 0; cc < CQ; ++cc) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = 4 * ty + i;
        const float* xr = xq + tok * N * CQP + cc;
        const float* Gr = Gq + tok * N * CQP + cc;
        if constexpr (WHICH != WD_PRE) {
          // dots tx + 32 q < 256: <G_i, x_j>, j = tx % 16, i = tx / 16 + 2 q
          const float xj = xr[(tx & (N - 1)) * CQP];
#pragma unroll
          for (int q = 0; q < CPT - 1; ++q)
            dacc[i][q] = fmaf(Gr[((tx >> 4) + 2 * q) * CQP], xj, dacc[i][q]);
        }
        // dot 256 + tx: tx < 16 <g, x_tx>; tx >= 16 <G_(tx-16), f>
        if (tx < N) {
          if constexpr (USE_g)
            dacc[i][CPT - 1] = fmaf(gq[tok * CQ + cc], xr[tx * CQP], dacc[i][CPT - 1]);
        } else {
          if constexpr (USE_f)
            dacc[i][CPT - 1] = fmaf(Gr[(tx - N) * CQP], fq[tok * CQ + cc], dacc[i][CPT - 1]);
        }
      }
    }
    __syncthreads();
  }
}

// The per-token epilogue for token t0 + tid: gates, Sinkhorn and, in the
// backward, its adjoint, the coefficient record and the token's dz row.  Its
// 16 x 16 arrays live in local memory: the forward runs it inside k_wide_map,
// the backward in k_wide_bwd_epi, apart from the GEMM loops' registers.
// yr: the token's M projections, dt: its M dot products (backward), ss: its
// sum of squares.  In the backward yr and dt are the token's own coefficient
// row, which is read in full before the record is written over it; the caller
// runs the backward epilogue only for tokens t < T.
template <int MODE>
__device__ __forceinline__ void wide_epilogue(int tid, int64_t t, int64_t T, int64_t K, int iters,
                                           float eps, const float* yr, const float* dt, float ss,
                                           const float* bias, const float* alpha_p, int ag,
                                           float* Hpre_o, float* Hpost_o, float* Hres_o,
                                           const float* red_in, float* coef_o, float* dzs,
                                           int* status, float* ck = nullptr) {
  using namespace widek;
  constexpr bool BWD = MODE != MAP_FWD;
  constexpr bool SPLIT = MODE == MAP_BWD_SPLIT;
  using CF = Coef<N>;
  const bool mine = t < T;
  const float r = sqrtf(ss / (float)K + eps);
  Alpha3 al;
  al.load(alpha_p, ag);
  float spre[N], spost[N], zres[N * N];
  bool bad = !isfinite(r);
  for (int m = 0; m < M; ++m) {
    const float y = yr[m] / r;
    const float z = fmaf(al.at<N>(m), y, __ldg(bias + m));
    bad |= !isfinite(z);
    if (m < N) spre[m] = sigmoidf_(z);
    else if (m < 2 * N) spost[m - N] = sigmoidf_(z);
    else zres[m - 2 * N] = z;
  }
  if (mine && bad) flag_status(status, MHC_ERR_NONFINITE);
  float H[N * N];
  for (int e = 0; e < N * N; ++e) H[e] = zres[e];
  // with a checkpoint area (backward, tensor-core path) the forward keeps every
  // second iterate there and the adjoint rebuilds each one from the nearest
  // (the same iterates and results, a fraction of the recomputation)
  if (BWD && ck != nullptr)
    sk_forward_ckpt<N>(H, iters, ck, TB, kWideCkPeriod);
  else
    sk_forward<N>(H, iters);
  if constexpr (!BWD) {
    if (mine) {
      for (int i = 0; i < N; ++i) {
        Hpre_o[t * N + i] = spre[i];
        Hpost_o[t * N + i] = 2.0f * spost[i];
      }
      for (int e = 0; e < N * N; ++e) Hres_o[t * N * N + e] = H[e];
    }
  } else {
    const float* rt = red_in + (SPLIT && mine ? t * (N * N + N) : 0);
    float dA[N * N], dz[M];
    for (int e = 0; e < N * N; ++e) dA[e] = !mine ? 0.0f : (SPLIT ? __ldg(rt + e) : dt[e]);
    float dzres[N * N];
    if (ck != nullptr)
      sk_adjoint_ckpt<N>(dA, dzres, iters, ck, TB, kWideCkPeriod);
    else
      sk_adjoint<N>(zres, dA, dzres, iters);
    for (int i = 0; i < N; ++i) {
      dz[i] = dt[N * N + i] * spre[i] * (1.0f - spre[i]);
      const float dpost = !mine ? 0.0f : (SPLIT ? __ldg(rt + N * N + i) : dt[N * N + N + i]);
      dz[N + i] = dpost * 2.0f * spost[i] * (1.0f - spost[i]);
    }
    for (int e = 0; e < N * N; ++e) dz[2 * N + e] = dzres[e];
    float dzy[3] = {0.0f, 0.0f, 0.0f};  // dz . y over the pre, post, res logits
    for (int m = 0; m < M; ++m) {
      const int grp = m < N ? 0 : (m < 2 * N ? 1 : 2);
      dzy[grp] = fmaf(dz[m], yr[m] / r, dzy[grp]);
    }
    if (mine) {
      float* co = coef_o + t * CF::SIZE;
      for (int e = 0; e < N * N; ++e) co[CF::RES + e] = H[e];
      for (int i = 0; i < N; ++i) {
        co[CF::PRE + i] = spre[i];
        co[CF::POST + i] = 2.0f * spost[i];
      }
      float ar[3];
      for (int gr = 0; gr < 3; ++gr) ar[gr] = al.a[gr] / r;
      for (int m = 0; m < M; ++m) co[CF::U + m] = ar[m < N ? 0 : (m < 2 * N ? 1 : 2)] * dz[m];
      const float wdzy = fmaf(al.a[2], dzy[2], fmaf(al.a[1], dzy[1], al.a[0] * dzy[0]));
      co[CF::KAPPA] = wdzy / ((float)K * r * r);
      for (int e = CF::KAPPA + 1; e < CF::SIZE; ++e) co[e] = 0.0f;
    }
    for (int m = 0; m < M; ++m) dzs[tid * (M + 3) + m] = mine ? dz[m] : 0.0f;
    for (int gr = 0; gr < 3; ++gr) dzs[tid * (M + 3) + M + gr] = mine ? dzy[gr] : 0.0f;
  }
  }

// MAP_FWD: H_pre / H_post / H_res.  MAP_BWD: coef [T][Coef<16>::SIZE] and per
// CTA the sums over its tokens of dz and dz . y (part [grid][DZ_SIZE]).
// MAP_BWD_SPLIT: as MAP_BWD with <G_i, x_j> and <G_i, f_out> from `red`.
template <typename TIO, int MODE>
__global__ void __launch_bounds__(widek::NT) k_wide_map(
    int64_t T, int64_t C, int iters, float eps, const TIO* __restrict__ x,
    const float* __restrict__ phi, const float* __restrict__ bias,
    const float* __restrict__ alpha_p, int ag, float* __restrict__ Hpre_o,
    float* __restrict__ Hpost_o, float* __restrict__ Hres_o, const TIO* __restrict__ G,
    const TIO* __restrict__ g, const TIO* __restrict__ f, const float* __restrict__ red_in,
    float* __restrict__ coef_o, float* __restrict__ part_o, int* status) {
  using namespace widek;
  constexpr bool BWD = MODE != MAP_FWD;
  constexpr bool SPLIT = MODE == MAP_BWD_SPLIT;
  using CF = Coef<N>;
  extern __shared__ __align__(16) float smem[];
  float* stg = smem;
  float* ys = smem + YS_OFF;
  float* sss = smem + SS_OFF;
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * TB;
  const int64_t K = (int64_t)N * C;

  // ---- projection y[t][m] = sum_k x[t][k] phi[k][m], and the sums of squares
  {
    float* xs = stg;            // [KC][TB]
    float* ps = stg + KC * TB;  // [KC][M]
    float acc[4][CPT], ssp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ssp[i] = 0.0f;
#pragma unroll
      for (int q = 0; q < CPT; ++q) acc[i][q] = 0.0f;
    }
    for (int64_t k0 = 0; k0 < K; k0 += KC) {
      // all loads are issued before the first store, so their latencies overlap
      // (K is a multiple of 128: every phi chunk is whole)
      constexpr int RP = KC * M / NT;  // 36
      float xv[TB * KC / NT], pv[RP];
#pragma unroll
      for (int r = 0; r < TB * KC / NT; ++r) {
        const int64_t t = t0 + ty + 8 * r, k = k0 + tx;
        xv[r] = (t < T && k < K) ? to_f32(x[t * K + k]) : 0.0f;
      }
      const float* pc = phi + k0 * M;
#pragma unroll
      for (int r = 0; r < RP; ++r) pv[r] = __ldg(pc + tid + NT * r);
#pragma unroll
      for (int r = 0; r < TB * KC / NT; ++r) {
        xs[tx * TB + ty + 8 * r] = xv[r];
        ssp[r] = fmaf(xv[r], xv[r], ssp[r]);
      }
#pragma unroll
      for (int r = 0; r < RP; ++r) ps[tid + NT * r] = pv[r];
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < KC; ++kk) {
        const float4 a = *reinterpret_cast<const float4*>(xs + kk * TB + 4 * ty);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          const float bq = ps[kk * M + tx + 32 * q];
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i][q] = fmaf(av[i], bq, acc[i][q]);
        }
      }
      __syncthreads();
    }
    // the backward stages y, the dot products and the sum of squares in the
    // token's coefficient row: [0, M) y, [M, 2M) dots, [2M] sum of squares
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t t = t0 + 4 * ty + i;
#pragma unroll
      for (int q = 0; q < CPT; ++q) {
        if constexpr (BWD) {
          if (t < T) coef_o[t * CF::SIZE + tx + 32 * q] = acc[i][q];
        } else {
          ys[(4 * ty + i) * M + tx + 32 * q] = acc[i][q];
        }
      }
    }
    // token ty + 8r: its 32 k-slots sit in the 32 lanes; xor tree, fixed order
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float v = ssp[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (tx == 0) {
        const int64_t t = t0 + ty + 8 * r;
        if constexpr (BWD) {
          if (t < T) coef_o[t * CF::SIZE + 2 * M] = v;
        } else {
          sss[ty + 8 * r] = v;
        }
      }
    }
  }

  // ---- the C-reductions of the backward
  if constexpr (BWD) {
    float dacc[4][CPT];
    if constexpr (SPLIT)
      wide_dots<TIO, WD_PRE>(T, C, t0, x, nullptr, g, nullptr, nullptr, nullptr, stg, dacc);
    else
      wide_dots<TIO, WD_FULL>(T, C, t0, x, G, g, f, nullptr, nullptr, stg, dacc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t t = t0 + 4 * ty + i;
      if (t >= T) continue;
#pragma unroll
      for (int q = 0; q < CPT; ++q) coef_o[t * CF::SIZE + M + tx + 32 * q] = dacc[i][q];
    }
    return;  // k_wide_bwd_epi finishes these tokens
  }
  __syncthreads();

  // ---- the forward's per-token epilogue, one thread per token
  if constexpr (!BWD) {
    if (tid < TB)
      wide_epilogue<MODE>(tid, t0 + tid, T, K, iters, eps, ys + tid * M, nullptr, sss[tid], bias,
                          alpha_p, ag, Hpre_o, Hpost_o, Hres_o, red_in, coef_o, nullptr, status);
  }
}

// The CUDA-core path's backward epilogue (no checkpoint scratch): one thread
// per token reads the token's staged row (y, dot products, sum of squares)
// from coef, writes the coefficient record over it, and adds the CTA's dz and
// dz . y rows in token order into part [grid][DZ_SIZE].
template <int MODE>
__global__ void __launch_bounds__(32) k_wide_bwd_epi_thread(int64_t T, int64_t C, int iters,
                                                            float eps,
                                                     const float* __restrict__ bias,
                                                     const float* __restrict__ alpha_p, int ag,
                                                     const float* __restrict__ red_in,
                                                     float* __restrict__ coef,
                                                     float* __restrict__ part_o, int* status) {
  using namespace widek;
  using CF = Coef<N>;
  __shared__ float dzs[TB * (M + 3)];
  const int tid = threadIdx.x;
  const int64_t t = (int64_t)blockIdx.x * TB + tid;
  if (t < T) {
    const float* row = coef + t * CF::SIZE;
    wide_epilogue<MODE>(tid, t, T, (int64_t)N * C, iters, eps, row, row + M, row[2 * M], bias,
                        alpha_p, ag, nullptr, nullptr, nullptr, red_in, coef, dzs, status);
  } else {
    for (int m = 0; m < M + 3; ++m) dzs[tid * (M + 3) + m] = 0.0f;
  }
  __syncwarp();
  for (int col = tid; col < M + 3; col += 32) {
    float s = 0.0f;
    for (int q = 0; q < TB; ++q) s += dzs[q * (M + 3) + col];
    part_o[(int64_t)blockIdx.x * CF::DZ_SIZE + col] = s;
  }
}

// The per-token epilogues of the tensor-core path, 16 lanes per token (lane i
// of a half-warp: row i of H_res, pre and post logit i), TB tokens per CTA.
// From the token's row (y at [0, M), the backward's dot products at [M, 2M),
// the sum of squares at [2M]) they compute the gates and Sinkhorn (forward), or
// the record of the apply and the token's dz (backward: the record is written
// over the row once every lane has read it).
template <int MODE>
__global__ void __launch_bounds__(widek::EPI_NT) k_wide_bwd_epi(
    int64_t T, int64_t C, int iters, float eps, const float* __restrict__ bias,
    const float* __restrict__ alpha_p, int ag, const float* __restrict__ red_in,
    float* __restrict__ coef, float* __restrict__ part_o, int* status, float* __restrict__ ck) {
  using namespace widek;
  using CF = Coef<N>;
  constexpr bool SPLIT = MODE == MAP_BWD_SPLIT;
  // the transpose buffers during Sinkhorn, then the CTA's dz rows
  static_assert(TB * TBS <= TB * (M + 3), "overlay");
  __shared__ __align__(16) float sbuf[TB * (M + 3)];
  float* tbs = sbuf;
  float* dzs = sbuf;
  const int lt = threadIdx.x >> 4, i = threadIdx.x & 15;  // token of the CTA, row
  const int64_t t = (int64_t)blockIdx.x * TB + lt;
  const bool live = t < T;
  float* tb = tbs + lt * TBS;
  float* vb = tb + N * N;
  const float* row = coef + (live ? t : 0) * CF::SIZE;
  const int64_t K = (int64_t)N * C;
  // ---- the row's inputs (every lane reads before any lane writes the record)
  const float r = sqrtf((live ? row[2 * M] : 1.0f) / (float)K + eps);
  Alpha3 al;
  al.load(alpha_p, ag);
  float yres[N], a[N], g[N];
  float ypre = 0.0f, ypost = 0.0f, zpre = 0.0f, zpost = 0.0f;
  bool bad = !isfinite(r);
  {
    const float y0 = live ? row[i] / r : 0.0f, y1 = live ? row[N + i] / r : 0.0f;
    ypre = y0;
    ypost = y1;
    zpre = fmaf(al.at<N>(i), y0, __ldg(bias + i));
    zpost = fmaf(al.at<N>(N + i), y1, __ldg(bias + N + i));
    bad |= !isfinite(zpre) || !isfinite(zpost);
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int m = 2 * N + i * N + j;
      yres[j] = live ? row[m] / r : 0.0f;
      a[j] = fmaf(al.a[2], yres[j], __ldg(bias + m));
      bad |= !isfinite(a[j]);
    }
  }
  const float* rt = red_in + (SPLIT && live ? t * (N * N + N) : 0);
#pragma unroll
  for (int j = 0; j < N; ++j)
    g[j] = !live ? 0.0f : (SPLIT ? __ldg(rt + i * N + j) : row[M + i * N + j]);
  const float dpre_in = live ? row[M + N * N + i] : 0.0f;
  const float dpost_in = !live ? 0.0f : (SPLIT ? __ldg(rt + N * N + i) : row[M + N * N + N + i]);
  if (__any_sync(0xffffffffu, live && bad) && live && bad) flag_status(status, MHC_ERR_NONFINITE);
  __syncwarp();
  // ---- Sinkhorn with checkpoints, then its adjoint from them
  float* ckt = ck + (live ? t : 0) * ((int64_t)iters + 1) * N * N + i * N;
  auto ck_store = [&](int c, const float (&v)[N]) {
    if (live) {
      float4* d = reinterpret_cast<float4*>(ckt + (int64_t)c * N * N);
#pragma unroll
      for (int j4 = 0; j4 < N / 4; ++j4)
        d[j4] = make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
    }
  };
  auto ck_load = [&](int c, float (&v)[N]) {
    if (live) {
      const float4* src = reinterpret_cast<const float4*>(ckt + (int64_t)c * N * N);
#pragma unroll
      for (int j4 = 0; j4 < N / 4; ++j4) {
        const float4 q = src[j4];
        v[4 * j4] = q.x;
        v[4 * j4 + 1] = q.y;
        v[4 * j4 + 2] = q.z;
        v[4 * j4 + 3] = q.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) v[j] = 1.0f;
    }
  };
  constexpr int P = kWideCkPeriod;
  sk16_init(a, iters);
  ck_store(0, a);
  for (int q = 1; q <= 2 * iters; ++q) {
    sk16_step(a, q, i, tb, vb);
    if (q % P == 0) ck_store(q / P, a);
  }
  float H[N];  // this lane's row of H_res
#pragma unroll
  for (int j = 0; j < N; ++j) H[j] = a[j];
  for (int step = 2 * iters; step >= 1; --step) {
    const int c = (step - 1) / P;
    ck_load(c, a);
    for (int q = c * P + 1; q < step; ++q) sk16_step(a, q, i, tb, vb);
    const float sq = sk16_step(a, step, i, tb, vb);
    sk16_adjoint_step(a, sq, g, step, i, tb, vb);
  }
  ck_load(0, a);  // the exponentiated logits
  float dzres[N];
#pragma unroll
  for (int j = 0; j < N; ++j) dzres[j] = g[j] * a[j];
  // ---- gates, dz, the record
  const float spre = sigmoidf_(zpre), spost = sigmoidf_(zpost);
  const float dzpre = dpre_in * spre * (1.0f - spre);
  const float dzpost = dpost_in * 2.0f * spost * (1.0f - spost);
  float pres = 0.0f;
#pragma unroll
  for (int j = 0; j < N; ++j) pres = fmaf(dzres[j], yres[j], pres);
  const float dzy0 = half_sum(dzpre * ypre), dzy1 = half_sum(dzpost * ypost);
  const float dzy2 = half_sum(pres);
  if (live) {
    float* co = coef + t * CF::SIZE;
    float4* hr = reinterpret_cast<float4*>(co + CF::RES + i * N);
#pragma unroll
    for (int j4 = 0; j4 < N / 4; ++j4)
      hr[j4] = make_float4(H[4 * j4], H[4 * j4 + 1], H[4 * j4 + 2], H[4 * j4 + 3]);
    co[CF::PRE + i] = spre;
    co[CF::POST + i] = 2.0f * spost;
    const float ar0 = al.a[0] / r, ar1 = al.a[1] / r, ar2 = al.a[2] / r;
    co[CF::U + i] = ar0 * dzpre;
    co[CF::U + N + i] = ar1 * dzpost;
    float4* ur = reinterpret_cast<float4*>(co + CF::U + 2 * N + i * N);
#pragma unroll
    for (int j4 = 0; j4 < N / 4; ++j4)
      ur[j4] = make_float4(ar2 * dzres[4 * j4], ar2 * dzres[4 * j4 + 1], ar2 * dzres[4 * j4 + 2],
                           ar2 * dzres[4 * j4 + 3]);
    if (i == 0) {
      const float wdzy = fmaf(al.a[2], dzy2, fmaf(al.a[1], dzy1, al.a[0] * dzy0));
      co[CF::KAPPA] = wdzy / ((float)K * r * r);
      for (int e = CF::KAPPA + 1; e < CF::SIZE; ++e) co[e] = 0.0f;
    }
  }
  __syncthreads();  // every token's Sinkhorn is done with the transpose buffers
  float* dz = dzs + lt * (M + 3);
  dz[i] = live ? dzpre : 0.0f;
  dz[N + i] = live ? dzpost : 0.0f;
#pragma unroll
  for (int j = 0; j < N; ++j) dz[2 * N + i * N + j] = live ? dzres[j] : 0.0f;
  if (i == 0) {
    dz[M] = live ? dzy0 : 0.0f;
    dz[M + 1] = live ? dzy1 : 0.0f;
    dz[M + 2] = live ? dzy2 : 0.0f;
  }
  __syncthreads();
  // this CTA's sums of dz and dz . y, in token order
  for (int col = threadIdx.x; col < M + 3; col += EPI_NT) {
    float sum = 0.0f;
    for (int q = 0; q < TB; ++q) sum += dzs[q * (M + 3) + col];
    part_o[(int64_t)blockIdx.x * CF::DZ_SIZE + col] = sum;
  }
}

__global__ void __launch_bounds__(widek::EPI_NT) k_wide_fwd_epi(
    int64_t T, int64_t C, int iters, float eps, const float* __restrict__ bias,
    const float* __restrict__ alpha_p, int ag, const float* __restrict__ rows,
    float* __restrict__ Hpre_o, float* __restrict__ Hpost_o, float* __restrict__ Hres_o,
    int* status) {
  using namespace widek;
  using CF = Coef<N>;
  __shared__ __align__(16) float tbs[TB * TBS];
  const int lt = threadIdx.x >> 4, i = threadIdx.x & 15;
  const int64_t t = (int64_t)blockIdx.x * TB + lt;
  const bool live = t < T;
  float* tb = tbs + lt * TBS;
  float* vb = tb + N * N;
  const float* row = rows + (live ? t : 0) * CF::SIZE;
  const float r = sqrtf((live ? row[2 * M] : 1.0f) / (float)(N * C) + eps);
  Alpha3 al;
  al.load(alpha_p, ag);
  const float zpre = fmaf(al.at<N>(i), live ? row[i] / r : 0.0f, __ldg(bias + i));
  const float zpost = fmaf(al.at<N>(N + i), live ? row[N + i] / r : 0.0f, __ldg(bias + N + i));
  bool bad = !isfinite(r) || !isfinite(zpre) || !isfinite(zpost);
  float a[N];
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const int m = 2 * N + i * N + j;
    a[j] = fmaf(al.a[2], live ? row[m] / r : 0.0f, __ldg(bias + m));
    bad |= !isfinite(a[j]);
  }
  if (__any_sync(0xffffffffu, live && bad) && live && bad) flag_status(status, MHC_ERR_NONFINITE);
  sk16_init(a, iters);
  for (int q = 1; q <= 2 * iters; ++q) sk16_step(a, q, i, tb, vb);
  if (live) {
    Hpre_o[t * N + i] = sigmoidf_(zpre);
    Hpost_o[t * N + i] = 2.0f * sigmoidf_(zpost);
    float4* hr = reinterpret_cast<float4*>(Hres_o + t * N * N + i * N);
#pragma unroll
    for (int j4 = 0; j4 < N / 4; ++j4)
      hr[j4] = make_float4(a[4 * j4], a[4 * j4 + 1], a[4 * j4 + 2], a[4 * j4 + 3]);
  }
}

// x_next[i][c] = sum_j H_res[i][j] x[j][c] + H_post[i] f_out[c] (the k_post order)
template <typename TIO>
__global__ void __launch_bounds__(128) k_wide_post(int64_t T, int64_t C, const TIO* __restrict__ x,
                                                   const TIO* __restrict__ f,
                                                   const float* __restrict__ Hpost,
                                                   const float* __restrict__ Hres,
                                                   TIO* __restrict__ xn) {
  using namespace widek;
  using V = Vec<TIO>;
  constexpr int W = V::N, P = W / 2;  // channels per vector, fp32 pairs per vector
  __shared__ __align__(16) float hr[N * N];
  __shared__ float hp[N];
  const int64_t nv = C / W;
  // -0 as the addend makes fma(h, f, -0) the plain product h f, sign of zero included
  const uint64_t nz = f2pack(-0.0f, -0.0f);
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    for (int e = threadIdx.x; e < N * N; e += blockDim.x) hr[e] = __ldg(Hres + t * N * N + e);
    if (threadIdx.x < N) hp[threadIdx.x] = __ldg(Hpost + t * N + threadIdx.x);
    __syncthreads();
    const TIO* xt = x + t * N * C;
    TIO* ot = xn + t * N * C;
    for (int64_t v = threadIdx.x; v < nv; v += blockDim.x) {
      // the vector's channels of every stream as fp32 pairs
      uint64_t xv[N][P], fv[P];
      {
        float tmp[W];
#pragma unroll
        for (int j = 0; j < N; ++j) {
          V::load_stream(xt + j * C + v * W, tmp);
#pragma unroll
          for (int p = 0; p < P; ++p) xv[j][p] = f2pack(tmp[2 * p], tmp[2 * p + 1]);
        }
        V::load_stream(f + t * C + v * W, tmp);
#pragma unroll
        for (int p = 0; p < P; ++p) fv[p] = f2pack(tmp[2 * p], tmp[2 * p + 1]);
      }
      // x_next[i] = H_post[i] f + sum_j H_res[i][j] x[j], the terms added in j order
#pragma unroll 1
      for (int i = 0; i < N; ++i) {
        uint64_t acc[P];
        const uint64_t h0 = f2pack(hp[i], hp[i]);
#pragma unroll
        for (int p = 0; p < P; ++p) acc[p] = f2fma(h0, fv[p], nz);
#pragma unroll
        for (int j4 = 0; j4 < N / 4; ++j4) {
          const float4 h = *reinterpret_cast<const float4*>(hr + i * N + 4 * j4);
          const float hv[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t hh = f2pack(hv[k], hv[k]);
#pragma unroll
            for (int p = 0; p < P; ++p) acc[p] = f2fma(hh, xv[4 * j4 + k][p], acc[p]);
          }
        }
        float o[W];
#pragma unroll
        for (int p = 0; p < P; ++p) {
          float a, b;
          asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(acc[p]));
          o[2 * p] = a;
          o[2 * p + 1] = b;
        }
        V::store_stream(ot + i * C + v * W, o);
      }
    }
  }
}

// The post half of the backward in training order: grad_f_out and
// red [T][N*N + N] = (<G_i, x_j> row-major, then <G_i, f_out>).
template <typename TIO>
__global__ void __launch_bounds__(widek::NT) k_wide_post_bwd(int64_t T, int64_t C,
                                                             const TIO* __restrict__ x,
                                                             const TIO* __restrict__ f,
                                                             const float* __restrict__ Hpost,
                                                             const TIO* __restrict__ G,
                                                             TIO* __restrict__ gf,
                                                             float* __restrict__ red) {
  using namespace widek;
  extern __shared__ __align__(16) float smem[];
  float* hp = smem;        // [TB][N]
  float* stg = smem + TB * N;
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * TB;
  for (int e = tid; e < TB * N; e += NT) {
    const int64_t t = t0 + e / N;
    hp[e] = t < T ? __ldg(Hpost + t * N + e % N) : 0.0f;
  }
  __syncthreads();
  float dacc[4][CPT];
  wide_dots<TIO, WD_POST>(T, C, t0, x, G, nullptr, f, hp, gf, stg, dacc);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + 4 * ty + i;
    if (t >= T) continue;
    float* rt = red + t * (N * N + N);
#pragma unroll
    for (int q = 0; q < CPT - 1; ++q) rt[tx + 32 * q] = dacc[i][q];
    if (tx >= N) rt[N * N + tx - N] = dacc[i][CPT - 1];
  }
}

// grad_x[t][k] (k = j*C + c) = sum_m phi[k][m] u[t][m] + H_pre[j] g[c]
//                              + sum_i H_res[i][j] G[i][c] - kappa x[t][k]  (the k_bwd order)
// grad_f_out[t][c] = sum_i H_post[i] G[i][c]   (when grad_f is not null)
// A CTA owns 32 tokens x 4 channels of all 16 streams (64 k, kk = 4 j + cc), so
// the G values, grad_h_in and the tokens' coefficients are staged once and
// shared by the 16 output streams; the phi u term is a GEMM over the logits.
namespace widek {
constexpr int AX_CC = 4;                       // channels per apply CTA
constexpr int AX_K = N * AX_CC;                // 64 k per CTA
constexpr int AX_H = N * N + 2 * N + 1;        // per token: H_res, H_pre, H_post, kappa
constexpr int AX_US = 32 * 32;                 // [m][token]
constexpr int AX_PS = 32 * AX_K;               // [m][kk]
constexpr int AX_HS = 32 * AX_H;               // [token][AX_H]
constexpr int AX_GS = 32 * N * AX_CC;          // [token][i][cc]
constexpr int AX_GG = 32 * AX_CC;              // [token][cc]
constexpr int AX_SMEM_FLOATS = AX_US + AX_PS + AX_HS + AX_GS + AX_GG;
static_assert(AX_GS % NT == 0, "G tile split over the threads");
}  // namespace widek

template <typename TIO>
__global__ void __launch_bounds__(widek::NT) k_wide_apply_x(
    int64_t T, int64_t C, const TIO* __restrict__ x, const float* __restrict__ phi,
    const TIO* __restrict__ G, const TIO* __restrict__ g, const float* __restrict__ coef,
    TIO* __restrict__ grad_x, TIO* __restrict__ grad_f) {
  using namespace widek;
  using CF = Coef<N>;
  extern __shared__ __align__(16) float sm[];
  float* Us = sm;
  float* ps = Us + AX_US;
  float* hs = ps + AX_PS;
  float* Gs = hs + AX_HS;
  float* gs = Gs + AX_GS;
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int64_t c0 = (int64_t)blockIdx.y * AX_CC;   // C is a multiple of 8: whole groups
  const int64_t K = (int64_t)N * C;
  // this CTA's coefficients, G and grad_h_in; loads are issued before stores
  {
    constexpr int RH = (AX_HS + NT - 1) / NT, RG = AX_GS / NT;
    float hl[RH], gl[RG];
#pragma unroll
    for (int r = 0; r < RH; ++r) {
      const int e = tid + NT * r;
      const int tok = e / AX_H, q = e - tok * AX_H;
      const int64_t t = t0 + tok;
      hl[r] = (e < AX_HS && t < T) ? __ldg(coef + t * CF::SIZE + (q < AX_H - 1 ? q : CF::KAPPA))
                                   : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      const int e = tid + NT * r;
      const int cc = e & (AX_CC - 1), i = (e >> 2) & (N - 1), tok = e >> 6;
      const int64_t t = t0 + tok;
      gl[r] = t < T ? to_f32(G[(t * N + i) * C + c0 + cc]) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < RH; ++r)
      if (tid + NT * r < AX_HS) hs[tid + NT * r] = hl[r];
#pragma unroll
    for (int r = 0; r < RG; ++r) Gs[tid + NT * r] = gl[r];
  }
  if (tid < AX_GG) {
    const int cc = tid & (AX_CC - 1), tok = tid >> 2;
    const int64_t t = t0 + tok;
    gs[tid] = t < T ? to_f32(g[t * C + c0 + cc]) : 0.0f;
  }
  float acc[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.0f;
  for (int m0 = 0; m0 < M; m0 += 32) {
    float ul[4], pl[8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + NT * r, tok = e >> 5, mm = e & 31;
      const int64_t t = t0 + tok;
      ul[r] = t < T ? __ldg(coef + t * CF::SIZE + CF::U + m0 + mm) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = tid + NT * r, kk = e >> 5, mm = e & 31;
      const int64_t k = (int64_t)(kk >> 2) * C + c0 + (kk & 3);
      pl[r] = __ldg(phi + k * M + m0 + mm);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + NT * r;
      Us[(e & 31) * 32 + (e >> 5)] = ul[r];
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = tid + NT * r;
      ps[(e & 31) * AX_K + (e >> 5)] = pl[r];
    }
    __syncthreads();
#pragma unroll 8
    for (int mm = 0; mm < 32; ++mm) {
      const float4 a = *reinterpret_cast<const float4*>(Us + mm * 32 + 4 * ty);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float b0 = ps[mm * AX_K + tx], b1 = ps[mm * AX_K + tx + 32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[i][0] = fmaf(b0, av[i], acc[i][0]);
        acc[i][1] = fmaf(b1, av[i], acc[i][1]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tok = 4 * ty + i;
    const int64_t t = t0 + tok;
    if (t >= T) continue;
    const float* h = hs + tok * AX_H;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int kk = tx + 32 * hh, j = kk >> 2, cc = kk & 3;
      const int64_t c = c0 + cc;
      const float* Gt = Gs + tok * N * AX_CC + cc;
      float a = fmaf(h[CF::PRE + j], gs[tok * AX_CC + cc], acc[i][hh]);
#pragma unroll
      for (int i2 = 0; i2 < N; ++i2) a = fmaf(h[CF::RES + i2 * N + j], Gt[i2 * AX_CC], a);
      const int64_t k = (int64_t)j * C + c;
      const float gx = fmaf(-h[AX_H - 1], to_f32(x[t * K + k]), a);
      if constexpr (sizeof(TIO) == 2) grad_x[t * K + k] = __float2bfloat16_rn(gx);
      else grad_x[t * K + k] = gx;
      if (j == 0 && grad_f != nullptr) {
        float b = 0.0f;
#pragma unroll
        for (int i2 = 0; i2 < N; ++i2) b = fmaf(h[CF::POST + i2], Gt[i2 * AX_CC], b);
        if constexpr (sizeof(TIO) == 2) grad_f[t * C + c] = __float2bfloat16_rn(b);
        else grad_f[t * C + c] = b;
      }
    }
  }
}

// grad_phi[k][m] = sum_t x[t][k] u[t][m]: a CTA owns 32 rows k x 96 logits and
// walks every token in order.
template <typename TIO>
__global__ void __launch_bounds__(widek::NT) k_wide_apply_phi(int64_t T, int64_t C,
                                                              const TIO* __restrict__ x,
                                                              const float* __restrict__ coef,
                                                              float* __restrict__ grad_phi) {
  using namespace widek;
  using CF = Coef<N>;
  __shared__ __align__(16) float xs[32 * 32];   // [token][k]
  __shared__ __align__(16) float us[32 * 96];   // [token][m]
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  const int64_t k0 = (int64_t)blockIdx.x * 32;
  const int m0 = blockIdx.y * 96;
  const int64_t K = (int64_t)N * C;
  float acc[4][3];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = 0.0f;
  for (int64_t t0 = 0; t0 < T; t0 += 32) {
    float xl[4], ul[12];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + NT * r, tok = e >> 5, kk = e & 31;
      const int64_t t = t0 + tok, k = k0 + kk;
      xl[r] = (t < T && k < K) ? to_f32(x[t * K + k]) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 12; ++r) {
      const int e = tid + NT * r, tok = e / 96, mm = e - tok * 96;
      const int64_t t = t0 + tok;
      ul[r] = (t < T && m0 + mm < M) ? __ldg(coef + t * CF::SIZE + CF::U + m0 + mm) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) xs[tid + NT * r] = xl[r];
#pragma unroll
    for (int r = 0; r < 12; ++r) us[tid + NT * r] = ul[r];
    __syncthreads();
#pragma unroll 8
    for (int tok = 0; tok < 32; ++tok) {
      const float4 a = *reinterpret_cast<const float4*>(xs + tok * 32 + 4 * ty);
      const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const float b = us[tok * 96 + tx + 32 * q];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i][q] = fmaf(av[i], b, acc[i][q]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k = k0 + 4 * ty + i;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int m = m0 + tx + 32 * q;
      if (k < K && m < M) grad_phi[k * M + m] = acc[i][q];
    }
  }
}

// grad_b and grad_alpha: the mapping CTAs' partial sums added in a fixed
// order (warp w takes partials w, w + 8, ...; the warps' results in order).
__global__ void __launch_bounds__(widek::NT) k_wide_bias(const float* __restrict__ part,
                                                         int nparts, float* __restrict__ grad_b,
                                                         float* __restrict__ grad_alpha, int ag) {
  using namespace widek;
  constexpr int NC = M + 3, NW = NT / 32;
  __shared__ float wsum[(NW + 1) * NC];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int col = lane; col < NC; col += 32) {
    float s = 0.0f;
    for (int q = warp; q < nparts; q += NW) s += __ldg(part + (int64_t)q * Coef<N>::DZ_SIZE + col);
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

// ------------------------------------------------------------------ host
template <typename TIO, int MODE>
static cudaError_t launch_wide_map(int64_t T, int64_t C, int iters, float eps, const void* x,
                                   const float* phi, const float* b, const float* alpha, int ag,
                                   float* Hpre, float* Hpost, float* Hres, const void* G,
                                   const void* g, const void* f, const float* red, float* coef,
                                   float* part, int* st, cudaStream_t s) {
  const size_t smem = (size_t)widek::SMEM_FLOATS * 4;
  auto kern = k_wide_map<TIO, MODE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (T + widek::TB - 1) / widek::TB;
  kern<<<(unsigned)grid, widek::NT, smem, s>>>(T, C, iters, eps, (const TIO*)x, phi, b, alpha, ag,
                                              Hpre, Hpost, Hres, (const TIO*)G, (const TIO*)g,
                                              (const TIO*)f, red, coef, part, st);
  e = cudaGetLastError();
  if constexpr (MODE != MAP_FWD) {
    if (e != cudaSuccess) return e;
    k_wide_bwd_epi_thread<MODE><<<(unsigned)grid, 32, 0, s>>>(T, C, iters, eps, b, alpha, ag, red,
                                                              coef, part, st);
    e = cudaGetLastError();
  }
  return e;
}

int wide_map_tokens_per_cta() { return widek::TB; }

size_t wide_ck_bytes(int64_t T, int iters) {
  const int64_t ncta = (T + widek::TB - 1) / widek::TB;
  return (size_t)ncta * ((size_t)iters + 1) * widek::N * widek::N * widek::TB * 4;
}

cudaError_t wide_map_tc_dispatch(int mode, int64_t T, int64_t C, int iters, float eps,
                                 const void* x, const float* phi, void* phi_t, const float* b,
                                 const float* alpha, int ag, float* Hpre, float* Hpost,
                                 float* Hres, const void* G, const void* g, const void* f,
                                 const float* red, float* rows, float* part, float* ck, int* st,
                                 int64_t wait_ns, cudaStream_t s) {
  using CF = Coef<widek::N>;
  cudaError_t e = proj16_dispatch(T, C, x, phi, phi_t, rows, CF::SIZE, st, wait_ns, s);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((T + widek::TB - 1) / widek::TB);
  if (mode == MAP_FWD) {
    k_wide_fwd_epi<<<grid, widek::EPI_NT, 0, s>>>(T, C, iters, eps, b, alpha, ag, rows, Hpre,
                                                  Hpost, Hres, st);
    return cudaGetLastError();
  }
  if (mode != MAP_BWD && mode != MAP_BWD_SPLIT) return cudaErrorInvalidValue;
  // the C-reductions on the tensor cores (k_dots_tc.cu), then the epilogue
  e = dots16_dispatch(mode == MAP_BWD, T, C, x, G, g, f, rows, st, wait_ns, s);
  if (e != cudaSuccess) return e;
  if (mode == MAP_BWD)
    k_wide_bwd_epi<MAP_BWD><<<grid, widek::EPI_NT, 0, s>>>(T, C, iters, eps, b, alpha, ag, red,
                                                           rows, part, st, ck);
  else
    k_wide_bwd_epi<MAP_BWD_SPLIT><<<grid, widek::EPI_NT, 0, s>>>(T, C, iters, eps, b, alpha, ag,
                                                                 red, rows, part, st, ck);
  return cudaGetLastError();
}

cudaError_t wide_map_dispatch(int mode, int dtype, int64_t T, int64_t C, int iters, float eps,
                              const void* x, const float* phi, const float* b, const float* alpha,
                              int ag, float* Hpre, float* Hpost, float* Hres, const void* G,
                              const void* g, const void* f, const float* red, float* coef,
                              float* part, int* st, cudaStream_t s) {
  const bool bf = dtype == MHC_DTYPE_BF16;
#define MHC_WMAP(MODE_)                                                                          \
  return bf ? launch_wide_map<__nv_bfloat16, MODE_>(T, C, iters, eps, x, phi, b, alpha, ag, Hpre, \
                                                    Hpost, Hres, G, g, f, red, coef, part, st, s) \
            : launch_wide_map<float, MODE_>(T, C, iters, eps, x, phi, b, alpha, ag, Hpre, Hpost,  \
                                            Hres, G, g, f, red, coef, part, st, s);
  switch (mode) {
    case MAP_FWD: MHC_WMAP(MAP_FWD)
    case MAP_BWD: MHC_WMAP(MAP_BWD)
    case MAP_BWD_SPLIT: MHC_WMAP(MAP_BWD_SPLIT)
    default: return cudaErrorInvalidValue;
  }
#undef MHC_WMAP
}

cudaError_t wide_post_dispatch(int dtype, int64_t T, int64_t C, const void* x, const void* f,
                               const float* Hpost, const float* Hres, void* xn, cudaStream_t s) {
  const int64_t cap = 148 * 16;
  const unsigned grid = (unsigned)(T < cap ? T : cap);
  if (dtype == MHC_DTYPE_BF16)
    k_wide_post<__nv_bfloat16><<<grid, 128, 0, s>>>(T, C, (const __nv_bfloat16*)x,
                                                    (const __nv_bfloat16*)f, Hpost, Hres,
                                                    (__nv_bfloat16*)xn);
  else
    k_wide_post<float><<<grid, 128, 0, s>>>(T, C, (const float*)x, (const float*)f, Hpost, Hres,
                                            (float*)xn);
  return cudaGetLastError();
}

cudaError_t wide_post_bwd_dispatch(int dtype, int64_t T, int64_t C, const void* x, const void* f,
                                   const float* Hpost, const void* G, void* gf, float* red,
                                   cudaStream_t s) {
  using namespace widek;
  const size_t smem = (size_t)(TB * N + RED_STG) * 4;
  const unsigned grid = (unsigned)((T + TB - 1) / TB);
  cudaError_t e;
  if (dtype == MHC_DTYPE_BF16) {
    e = cudaFuncSetAttribute(k_wide_post_bwd<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_wide_post_bwd<__nv_bfloat16><<<grid, NT, smem, s>>>(
        T, C, (const __nv_bfloat16*)x, (const __nv_bfloat16*)f, Hpost, (const __nv_bfloat16*)G,
        (__nv_bfloat16*)gf, red);
  } else {
    e = cudaFuncSetAttribute(k_wide_post_bwd<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    k_wide_post_bwd<float><<<grid, NT, smem, s>>>(T, C, (const float*)x, (const float*)f, Hpost,
                                                  (const float*)G, (float*)gf, red);
  }
  return cudaGetLastError();
}

template <typename TIO>
static cudaError_t launch_wide_apply(int64_t T, int64_t C, const void* x, const float* phi,
                                     const void* G, const void* g, const float* coef,
                                     const float* part, int nparts, void* gx, void* gf,
                                     float* gphi, float* gb, float* ga, int ag, cudaStream_t s) {
  using namespace widek;
  const int64_t K = (int64_t)N * C;
  const size_t smx = (size_t)AX_SMEM_FLOATS * 4;
  cudaError_t e = cudaFuncSetAttribute(k_wide_apply_x<TIO>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smx);
  if (e != cudaSuccess) return e;
  const dim3 gridx((unsigned)((T + 31) / 32), (unsigned)(C / AX_CC));
  k_wide_apply_x<TIO><<<gridx, NT, smx, s>>>(T, C, (const TIO*)x, phi, (const TIO*)G,
                                             (const TIO*)g, coef, (TIO*)gx, (TIO*)gf);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 gridp((unsigned)((K + 31) / 32), (unsigned)((M + 95) / 96));
  k_wide_apply_phi<TIO><<<gridp, NT, 0, s>>>(T, C, (const TIO*)x, coef, gphi);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_wide_bias<<<1, NT, 0, s>>>(part, nparts, gb, ga, ag);
  return cudaGetLastError();
}

cudaError_t wide_bias_dispatch(const float* part, int nparts, float* gb, float* ga, int ag,
                               cudaStream_t s) {
  k_wide_bias<<<1, widek::NT, 0, s>>>(part, nparts, gb, ga, ag);
  return cudaGetLastError();
}

cudaError_t wide_apply_dispatch(int dtype, int64_t T, int64_t C, const void* x, const float* phi,
                                const void* G, const void* g, const float* coef, const float* part,
                                int nparts, void* gx, void* gf, float* gphi, float* gb, float* ga,
                                int ag, cudaStream_t s) {
  return dtype == MHC_DTYPE_BF16
             ? launch_wide_apply<__nv_bfloat16>(T, C, x, phi, G, g, coef, part, nparts, gx, gf,
                                                gphi, gb, ga, ag, s)
             : launch_wide_apply<float>(T, C, x, phi, G, g, coef, part, nparts, gx, gf, gphi, gb,
                                        ga, ag, s);
}

}  // namespace mhc
