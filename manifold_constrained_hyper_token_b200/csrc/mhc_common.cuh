// mhc_common.cuh -- device helpers shared by the mHC kernels: 16-byte vector
// I/O for the two activation dtypes, status reporting, and the per-token
// mapping arithmetic (gates and Sinkhorn-Knopp with its adjoint) that the
// forward and backward kernels both run in registers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mhc.h"

namespace mhc {

// ---------------------------------------------------------------- vector I/O
// One 16-byte vector of the activation dtype, widened to fp32.
template <typename T> struct Vec;

template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float (&v)[4]) {
    float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  __device__ __forceinline__ static void load_stream(const float* p, float (&v)[4]) {
    float4 q = __ldcs(reinterpret_cast<const float4*>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  __device__ __forceinline__ static void store_stream(float* p, const float (&v)[4]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  }
};

template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4 q, float (&v)[8]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static uint4 pack(const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), v);
  }
  __device__ __forceinline__ static void load_stream(const __nv_bfloat16* p, float (&v)[8]) {
    unpack(__ldcs(reinterpret_cast<const uint4*>(p)), v);
  }
  __device__ __forceinline__ static void store_stream(__nv_bfloat16* p, const float (&v)[8]) {
    __stcs(reinterpret_cast<uint4*>(p), pack(v));
  }
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// ------------------------------------------------------------------- status
// Record the first run-time error code in the caller's status word.
__device__ __forceinline__ void flag_status(int* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

// -------------------------------------------------------- per-token mapping
__device__ __forceinline__ float sigmoidf_(float v) { return 1.0f / (1.0f + expf(-v)); }

// Sinkhorn-Knopp for one N x N matrix held by one thread.  On entry A holds
// the logits; on exit the estimate after `iters` iterations of (row pass,
// column pass).  With iters >= 1 the row maximum is subtracted before exp;
// the first row pass cancels that factor exactly in real arithmetic.
template <int N>
__device__ __forceinline__ void sk_init(float (&A)[N * N], int iters) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    float mx = 0.0f;
    if (iters > 0) {
      mx = A[i * N];
#pragma unroll
      for (int j = 1; j < N; ++j) mx = fmaxf(mx, A[i * N + j]);
    }
#pragma unroll
    for (int j = 0; j < N; ++j) A[i * N + j] = expf(A[i * N + j] - mx);
  }
}

// Normalisation number q (1-based): odd q = row pass, even q = column pass.
// `s` receives the sums that were divided out.
template <int N>
__device__ __forceinline__ void sk_step(float (&A)[N * N], int q, float (&s)[N]) {
  if (q & 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      float acc = 0.0f;
#pragma unroll
      for (int j = 0; j < N; ++j) acc += A[i * N + j];
      s[i] = acc;
      const float inv = 1.0f / acc;
#pragma unroll
      for (int j = 0; j < N; ++j) A[i * N + j] *= inv;
    }
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < N; ++i) acc += A[i * N + j];
      s[j] = acc;
      const float inv = 1.0f / acc;
#pragma unroll
      for (int i = 0; i < N; ++i) A[i * N + j] *= inv;
    }
  }
}

template <int N>
__device__ __forceinline__ void sk_forward(float (&A)[N * N], int iters) {
  sk_init<N>(A, iters);
  float s[N];
  for (int q = 1; q <= 2 * iters; ++q) sk_step<N>(A, q, s);
}

// Adjoint of sk_forward.  z holds the logits, dA the gradient with respect
// to the output; on exit dz holds the gradient with respect to the logits.
// Every intermediate iterate is recomputed from the start with the same
// instructions as the forward pass, so the backward sees the forward's exact
// fp32 iterates (O(iters^2) work on 16 registers, no stored iterates).
template <int N>
__device__ __forceinline__ void sk_adjoint(const float (&z)[N * N], float (&dA)[N * N],
                                           float (&dz)[N * N], int iters) {
  float M0[N * N];
#pragma unroll
  for (int e = 0; e < N * N; ++e) M0[e] = z[e];
  sk_init<N>(M0, iters);
  for (int step = 2 * iters; step >= 1; --step) {
    float A[N * N];
#pragma unroll
    for (int e = 0; e < N * N; ++e) A[e] = M0[e];
    float s[N];
    for (int q = 1; q < step; ++q) sk_step<N>(A, q, s);
    sk_step<N>(A, step, s);  // A is now the output of this step, s its sums
    if (step & 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        float d = 0.0f;
#pragma unroll
        for (int j = 0; j < N; ++j) d += dA[i * N + j] * A[i * N + j];
        const float inv = 1.0f / s[i];
#pragma unroll
        for (int j = 0; j < N; ++j) dA[i * N + j] = (dA[i * N + j] - d) * inv;
      }
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) {
        float d = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) d += dA[i * N + j] * A[i * N + j];
        const float inv = 1.0f / s[j];
#pragma unroll
        for (int i = 0; i < N; ++i) dA[i * N + j] = (dA[i * N + j] - d) * inv;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < N * N; ++e) dz[e] = dA[e] * M0[e];
}

// Checkpointed variants for the tensor-core kernels: the forward stores the
// iterate after every P-th normalisation (and the start) in shared memory,
// ck[(j * N * N + e) * stride]; the adjoint rebuilds each iterate from the
// nearest checkpoint with the forward's own instructions (bitwise the same
// iterates), at O(iters * P) instead of O(iters^2) work.
template <int N>
__device__ __forceinline__ void sk_forward_ckpt(float (&A)[N * N], int iters, float* ck, int stride,
                                                int P) {
  sk_init<N>(A, iters);
#pragma unroll
  for (int e = 0; e < N * N; ++e) ck[e * stride] = A[e];
  float s[N];
  for (int q = 1; q <= 2 * iters; ++q) {
    sk_step<N>(A, q, s);
    if (q % P == 0) {
      float* c = ck + (q / P) * N * N * stride;
#pragma unroll
      for (int e = 0; e < N * N; ++e) c[e * stride] = A[e];
    }
  }
}

template <int N>
__device__ __forceinline__ void sk_adjoint_ckpt(float (&dA)[N * N], float (&dz)[N * N], int iters,
                                                const float* ck, int stride, int P) {
  for (int step = 2 * iters; step >= 1; --step) {
    const int c = (step - 1) / P;
    float A[N * N];
    const float* cp = ck + c * N * N * stride;
#pragma unroll
    for (int e = 0; e < N * N; ++e) A[e] = cp[e * stride];
    float s[N];
    for (int q = c * P + 1; q < step; ++q) sk_step<N>(A, q, s);
    sk_step<N>(A, step, s);
    if (step & 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        float d = 0.0f;
#pragma unroll
        for (int j = 0; j < N; ++j) d += dA[i * N + j] * A[i * N + j];
        const float inv = 1.0f / s[i];
#pragma unroll
        for (int j = 0; j < N; ++j) dA[i * N + j] = (dA[i * N + j] - d) * inv;
      }
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) {
        float d = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) d += dA[i * N + j] * A[i * N + j];
        const float inv = 1.0f / s[j];
#pragma unroll
        for (int i = 0; i < N; ++i) dA[i * N + j] = (dA[i * N + j] - d) * inv;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < N * N; ++e) dz[e] = dA[e] * ck[e * stride];
}

// Per-token coefficient record written by the backward mapping kernel and
// read by the backward apply kernel (floats):
//   [0, N*N)            H_res
//   [N*N, N*N+N)        H_pre
//   [.., +N)            H_post
//   [.., +M)            u = alpha * dz / r     (M = N*N + 2N)
//   [.., +1)            kappa = alpha * (dz . y) / (K r^2)
// padded to a multiple of 4 floats.
template <int N> struct Coef {
  static constexpr int M = N * N + 2 * N;
  static constexpr int RES = 0;
  static constexpr int PRE = N * N;
  static constexpr int POST = N * N + N;
  static constexpr int U = N * N + 2 * N;
  static constexpr int KAPPA = U + M;
  static constexpr int SIZE = ((KAPPA + 1) + 3) / 4 * 4;
  // dz record for the bias / alpha sums: [0, M) dz, then dz . y over the
  // pre, post and res logits ([M], [M + 1], [M + 2]), padded.
  static constexpr int DZ_SIZE = ((M + 3) + 3) / 4 * 4;
};

// The logit scales: alpha_pre for the n pre logits, alpha_post for the n post
// logits, alpha_res for the n*n residual logits; one shared alpha (ag != 3)
// is three equal scales.
struct Alpha3 {
  float a[3];
  __device__ __forceinline__ void load(const float* p, int ag) {
    a[0] = __ldg(p);
    a[1] = ag == 3 ? __ldg(p + 1) : a[0];
    a[2] = ag == 3 ? __ldg(p + 2) : a[0];
  }
  // scale of logit m of a layer with N streams (m known at compile time in
  // the unrolled loops, so this is a register choice)
  template <int N>
  __device__ __forceinline__ float at(int m) const {
    return m < N ? a[0] : (m < 2 * N ? a[1] : a[2]);
  }
};

// Per-token records of the tensor-core backward (n = 4), written by the
// mapping kernel and streamed by the apply kernel's TMA:
//   U row  [64] bf16: u_hi (24) | 0 (8) | u_lo (24) | 0 (8), u = alpha dz / r,
//          u_lo = bf16(u - u_hi) -- the MMA operand row, 128 bytes
//   H rec  [28] fp32: H_res (16) | H_pre (4) | H_post (4) | kappa | 0 0 0
struct TcRec {
  static constexpr int U_ELEMS = 64;
  static constexpr int U_BYTES = U_ELEMS * 2;
  static constexpr int H_FLOATS = 28;
  static constexpr int H_BYTES = H_FLOATS * 4;
  static constexpr int H_RES = 0, H_PRE = 16, H_POST = 20, H_KAPPA = 24;
};

// The U row of the n = 8 tensor-core backward (written by the n = 8 mapping,
// read by the phi u and grad_phi MMAs): [192] bf16 = u_hi (80) | 0 (16) |
// u_lo (80) | 0 (16), three 64-element swizzle atoms, 384 bytes.
struct TcRec8 {
  static constexpr int U_ELEMS = 192;
  static constexpr int U_BYTES = U_ELEMS * 2;
  static constexpr int LO = 96;  // first column of u_lo
};

// ------------------------------------------------- paired fp32 arithmetic
// One fma.rn.f32x2 is two IEEE fp32 FMAs on a pair of values held in one
// 64-bit register (element 0 in the low half).
__device__ __forceinline__ uint64_t f2pack(float x, float y) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// two bf16 (one 32-bit word, element 0 in the low half) widened to an fp32
// pair, and an fp32 pair rounded back to two bf16
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
  return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(uint64_t v) {
  float x, y;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(v));
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------- N lanes per N x N Sinkhorn matrix
// Sinkhorn-Knopp and its adjoint for one token's N x N matrix on an aligned
// group of N lanes (N = 4 or 8), lane i holding row i.  Column sums are
// butterflies over the group (xor N/2, .., 1), so every lane of the group gets
// every column's sum, with the same bits.  All groups of a warp run the same
// steps (the shuffles are warp-wide).
template <int N>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = N / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int N>
__device__ __forceinline__ void skl_init(float (&a)[N], int iters) {
  float mx = 0.0f;
  if (iters > 0) {
    mx = a[0];
#pragma unroll
    for (int j = 1; j < N; ++j) mx = fmaxf(mx, a[j]);
  }
#pragma unroll
  for (int j = 0; j < N; ++j) a[j] = expf(a[j] - mx);
}

// Normalisation q (odd: rows, even: columns); s receives the sums divided out
// (odd q: s[0] = this lane's row sum; even q: s[j] = column j's sum).
template <int N>
__device__ __forceinline__ void skl_step(float (&a)[N], int q, float (&s)[N]) {
  if (q & 1) {
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < N; ++j) acc += a[j];
    const float inv = 1.0f / acc;
#pragma unroll
    for (int j = 0; j < N; ++j) a[j] *= inv;
    s[0] = acc;
    return;
  }
#pragma unroll
  for (int j = 0; j < N; ++j) s[j] = group_sum<N>(a[j]);
#pragma unroll
  for (int j = 0; j < N; ++j) a[j] *= 1.0f / s[j];
}

// One adjoint step: a is the iterate after normalisation q, s its sums, g the
// gradient with respect to it (this lane's row), turned into the gradient with
// respect to the iterate before the step:
//   rows:    g_ij <- (g_ij - sum_k g_ik a_ik) / s_i
//   columns: g_ij <- (g_ij - sum_k g_kj a_kj) / s_j
template <int N>
__device__ __forceinline__ void skl_adjoint_step(const float (&a)[N], const float (&s)[N],
                                                 float (&g)[N], int q) {
  if (q & 1) {
    float d = 0.0f;
#pragma unroll
    for (int j = 0; j < N; ++j) d = fmaf(g[j], a[j], d);
    const float inv = 1.0f / s[0];
#pragma unroll
    for (int j = 0; j < N; ++j) g[j] = (g[j] - d) * inv;
    return;
  }
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float d = group_sum<N>(g[j] * a[j]);
    g[j] = (g[j] - d) * (1.0f / s[j]);
  }
}

}  // namespace mhc
