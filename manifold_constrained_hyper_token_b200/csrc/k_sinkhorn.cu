// k_sinkhorn.cu -- standalone batched Sinkhorn-Knopp and the depth-product
// Amax gain.
//
// Sinkhorn-Knopp (section "Vielfaeltig eingeschraenkte Hyperverbindungen" of
// the chatgpz.de mHC explainer; reportify.cn [16]): M = exp(logits), then
// `iters` times divide every row by its sum and then every column by its sum.
//
// Layout on the device: each matrix is split into BR x BR blocks, one block
// per thread, so a matrix is owned by G = (N/BR)^2 consecutive lanes of one
// warp (n <= 8: one thread per matrix; n = 16: four threads, each an 8 x 8
// block).  Row and column sums are reduced with warp shuffles inside the
// group; the matrix never leaves registers between the load and the store.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"

namespace mhc {

// Reciprocal of a row or column sum by the approximate reciprocal instruction
// (about one float32 ulp of error; subnormal inputs are not flushed).  The
// correctly rounded division it replaces costs about as many instructions as
// the rest of a normalisation; the standalone estimate is checked against the
// fp64 oracle at 1e-5.  (The layer kernels keep the rounded division: their
// forward and adjoint recompute the same iterates.)
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

template <int N, int BR>
__global__ void __launch_bounds__(256) k_sinkhorn(int iters, int64_t B, const float* __restrict__ logits,
                                                  float* __restrict__ out, int* status) {
  constexpr int NB = N / BR;       // blocks per row
  constexpr int G = NB * NB;       // threads per matrix
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t m = gtid / G;
  const int sub = (int)(gtid % G);
  const int br = sub / NB, bc = sub % NB;
  const bool valid = m < B;

  float A[BR][BR];
#pragma unroll
  for (int i = 0; i < BR; ++i) {
#pragma unroll
    for (int j = 0; j < BR; ++j) A[i][j] = 0.0f;
  }
  if (valid) {
    const float* src = logits + m * N * N + (br * BR) * N + bc * BR;
#pragma unroll
    for (int i = 0; i < BR; ++i) {
      if constexpr (BR % 4 == 0) {
#pragma unroll
        for (int j = 0; j < BR; j += 4) {
          const float4 q = __ldcs(reinterpret_cast<const float4*>(src + i * N + j));
          A[i][j] = q.x; A[i][j + 1] = q.y; A[i][j + 2] = q.z; A[i][j + 3] = q.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < BR; ++j) A[i][j] = src[i * N + j];
      }
    }
  }

  // Row maximum (only when a row pass follows; it cancels exactly).
#pragma unroll
  for (int i = 0; i < BR; ++i) {
    float mx = 0.0f;
    if (iters > 0) {
      mx = A[i][0];
#pragma unroll
      for (int j = 1; j < BR; ++j) mx = fmaxf(mx, A[i][j]);
#pragma unroll
      for (int d = 1; d < NB; d <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
    }
#pragma unroll
    for (int j = 0; j < BR; ++j) A[i][j] = expf(A[i][j] - mx);
  }

  for (int it = 0; it < iters; ++it) {
    // rows: partners differ in bc (lane bits 0 .. log2(NB)-1)
#pragma unroll
    for (int i = 0; i < BR; ++i) {
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < BR; ++j) s += A[i][j];
#pragma unroll
      for (int d = 1; d < NB; d <<= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
      const float inv = rcp_approx(s);
#pragma unroll
      for (int j = 0; j < BR; ++j) A[i][j] *= inv;
    }
    // columns: partners differ in br (lane stride NB)
#pragma unroll
    for (int j = 0; j < BR; ++j) {
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < BR; ++i) s += A[i][j];
#pragma unroll
      for (int d = NB; d < G; d <<= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
      const float inv = rcp_approx(s);
#pragma unroll
      for (int i = 0; i < BR; ++i) A[i][j] *= inv;
    }
  }

  if (valid) {
    float* dst = out + m * N * N + (br * BR) * N + bc * BR;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < BR; ++i) {
#pragma unroll
      for (int j = 0; j < BR; ++j) bad |= !isfinite(A[i][j]);
      if constexpr (BR % 4 == 0) {
#pragma unroll
        for (int j = 0; j < BR; j += 4)
          __stcs(reinterpret_cast<float4*>(dst + i * N + j),
                 make_float4(A[i][j], A[i][j + 1], A[i][j + 2], A[i][j + 3]));
      } else {
#pragma unroll
        for (int j = 0; j < BR; ++j) dst[i * N + j] = A[i][j];
      }
    }
    if (bad) flag_status(status, MHC_ERR_NONFINITE);
  }
}

// Depth product P = H[L-1] ... H[0] per token and its Amax gains.  One thread
// per (token, column j) holds column j of P: (H P)[:, j] = H P[:, j] needs no
// other column.  The n threads of a token are consecutive lanes and read the
// same H entries (one broadcast transaction per load).
template <int N>
__global__ void __launch_bounds__(256) k_depth_amax(int64_t T, int L, const float* __restrict__ H,
                                                    float* __restrict__ gain_fwd,
                                                    float* __restrict__ gain_bwd) {
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t t = gtid / N;
  const int j = (int)(gtid % N);
  const bool valid = t < T;
  float p[N];
#pragma unroll
  for (int i = 0; i < N; ++i) p[i] = (i == j) ? 1.0f : 0.0f;
  if (valid) {
    const float* Ht = H + t * (int64_t)L * N * N;
    for (int l = 0; l < L; ++l) {
      const float* Hl = Ht + (int64_t)l * N * N;
      float q[N];
#pragma unroll
      for (int i = 0; i < N; ++i) {
        float acc = 0.0f;
        if constexpr (N % 4 == 0) {
#pragma unroll
          for (int k = 0; k < N; k += 4) {
            const float4 h = __ldg(reinterpret_cast<const float4*>(Hl + i * N + k));
            acc = fmaf(h.x, p[k], acc);
            acc = fmaf(h.y, p[k + 1], acc);
            acc = fmaf(h.z, p[k + 2], acc);
            acc = fmaf(h.w, p[k + 3], acc);
          }
        } else {
#pragma unroll
          for (int k = 0; k < N; ++k) acc = fmaf(__ldg(Hl + i * N + k), p[k], acc);
        }
        q[i] = acc;
      }
#pragma unroll
      for (int i = 0; i < N; ++i) p[i] = q[i];
    }
  }
  // column sum of |P| (this thread's column) and row sums across the group
  float col = 0.0f;
#pragma unroll
  for (int i = 0; i < N; ++i) col += fabsf(p[i]);
  float gb = col;
#pragma unroll
  for (int d = 1; d < N; d <<= 1) gb = fmaxf(gb, __shfl_xor_sync(0xffffffffu, gb, d));
  float gf = 0.0f;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    float r = fabsf(p[i]);
#pragma unroll
    for (int d = 1; d < N; d <<= 1) r += __shfl_xor_sync(0xffffffffu, r, d);
    gf = fmaxf(gf, r);
  }
  if (valid && j == 0) {
    gain_fwd[t] = gf;
    gain_bwd[t] = gb;
  }
}

template <int N, int BR>
static cudaError_t launch_sk(int iters, int64_t B, const float* logits, float* out, int* st,
                             cudaStream_t s) {
  constexpr int G = (N / BR) * (N / BR);
  const int64_t threads = B * G;
  const int bs = 256;
  const int64_t grid = (threads + bs - 1) / bs;
  k_sinkhorn<N, BR><<<(unsigned)grid, bs, 0, s>>>(iters, B, logits, out, st);
  return cudaGetLastError();
}

cudaError_t sinkhorn_dispatch(int n, int iters, int64_t B, const float* logits, float* out,
                              int* st, cudaStream_t s) {
  switch (n) {
    case 1: return launch_sk<1, 1>(iters, B, logits, out, st, s);
    case 2: return launch_sk<2, 2>(iters, B, logits, out, st, s);
    case 4: return launch_sk<4, 4>(iters, B, logits, out, st, s);
    case 8: return launch_sk<8, 8>(iters, B, logits, out, st, s);
    case 16: return launch_sk<16, 8>(iters, B, logits, out, st, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int N>
static cudaError_t launch_depth(int64_t T, int L, const float* H, float* gf, float* gb,
                                cudaStream_t s) {
  const int64_t threads = T * N;
  const int bs = 256;
  const int64_t grid = (threads + bs - 1) / bs;
  k_depth_amax<N><<<(unsigned)grid, bs, 0, s>>>(T, L, H, gf, gb);
  return cudaGetLastError();
}

cudaError_t depth_amax_dispatch(int n, int64_t T, int L, const float* H, float* gf, float* gb,
                                cudaStream_t s) {
  switch (n) {
    case 1: return launch_depth<1>(T, L, H, gf, gb, s);
    case 2: return launch_depth<2>(T, L, H, gf, gb, s);
    case 4: return launch_depth<4>(T, L, H, gf, gb, s);
    case 8: return launch_depth<8>(T, L, H, gf, gb, s);
    case 16: return launch_depth<16>(T, L, H, gf, gb, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mhc
