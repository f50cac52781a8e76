// k_apply8_tc.cu -- second phase of the mHC backward for n = 8 streams with
// bf16 activations.  From the per-token records of the n = 8 mapping kernel
// (H_res, H_pre, H_post, kappa, and the U rows u_hi | u_lo of
// u = alpha dz / r) it writes
//
//   grad_x[j][c]   = (phi u)[jC+c] + sum_i H_res[i][j] G[i][c] + H_pre[j] g[c] - kappa x[j][c]
//   grad_f_out[c]  = sum_i H_post[i] G[i][c]
//   grad_phi[k][m] = sum_t x_t[k] u_t[m]
//
// (reverse mode of the update equation of the chatgpz.de explainer and of the
// RMS-normalised projection; reportify.cn [19]-[21]).  At n = 8 an item of the fused
// n = 4 design (x, grad_x_next and grad_h_in of 16 channels x 8 streams x 128
// tokens, the tile's U rows and H records, the slice's phi rows) needs about
// 170 KB of shared memory, and the grad_phi accumulators of three slices do
// not fit beside the phi u accumulators in TMEM, so the two contractions run
// as their own tensor-core kernels:
//
//   k_phiu8   phi u for a (128-token tile, 256 channels of one stream) item:
//             D[128 x 256] = U[128 x 192] . PHI[192 x 256] (tcgen05, bf16
//             operands, fp32 in TMEM), written to an fp32 scratch [T][8][C];
//   k_gx8     grad_x and grad_f_out from that scratch, x, grad_x_next and
//             grad_h_in with coalesced 16-byte loads and stores (CUDA cores),
//             and grad_b / grad_alpha from the mapping's partial sums;
//   k_gphi8   grad_phi for 128 rows of phi: D[128 x 192] += X^T[128 x 128] .
//             U[128 x 192] over every token tile (tcgen05), then
//             grad_phi = D[:, m] + D[:, 96 + m].
//
// U is [u_hi (80) | 0 (16) | u_lo (80) | 0 (16)]: phi u = (u_hi + u_lo) . phi_hi
// and x . u carries u to ~16 bits (x is exact).  All sums are in a fixed order:
// repeated calls give identical bits.  Waits are bounded; a wait that gives up
// records MHC_ERR_TIMEOUT, and the kernel drains what it issued, frees TMEM
// and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

namespace ap8 {
constexpr int N = 8;
constexpr int M = N * N + 2 * N;        // 80 logits
constexpr int TT = 128;                 // tokens per tile
constexpr int NU = TcRec8::U_ELEMS;     // 192
constexpr int ATOM = 128 * 128;         // [128 rows][64 bf16] with the 128-byte swizzle: 16 KB
// k_phiu8
constexpr int KB = 256;                 // channels of one stream per item (MMA N)
constexpr int CH = 16;                  // channels per block of the tiled phi^T copy
constexpr int NL = 2 * M;               // rows per block (80 high, 80 low)
constexpr int PHB = M * CH * 2;         // the 80 high rows of one block: 2.5 KB
constexpr int A_U_OFF = 0;              // U tile: three atoms (48 KB)
constexpr int A_P_OFF = 3 * ATOM;       // phi tile: KB / CH blocks of high rows (40 KB)
constexpr int A_DATA = A_P_OFF + (KB / CH) * PHB;
constexpr int XT = 36;                  // row stride (floats) of the epilogue's transpose buffer
constexpr int A_SMEM = A_DATA + 1024 + 64;
constexpr int A_NT = 128;
constexpr uint32_t A_TMEM = 256;
// k_gphi8
constexpr int CB = 128;                 // phi rows (channels of one stream) per CTA (MMA M)
constexpr int C_X_OFF = 0;              // x tile [128 tokens][128 channels]: two atoms
constexpr int C_U_OFF = 2 * ATOM;       // U tile: three atoms
constexpr int C_STAGE = 5 * ATOM;       // 80 KB
constexpr int C_NS = 2;
constexpr int C_DATA = C_NS * C_STAGE;
constexpr int C_SMEM = C_DATA + 1024 + 64;
constexpr int C_NT = 128;
constexpr uint32_t C_TMEM = 256;
// k_gx8
constexpr int B_NT = 128;
static_assert(A_SMEM <= 232448 && C_SMEM <= 232448, "shared memory");
}  // namespace ap8

namespace {
__device__ __forceinline__ void unpack8b(uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ uint4 pack8b(const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
}  // namespace

// ------------------------------------------------------------------ phi u
__global__ void __launch_bounds__(ap8::A_NT) k_phiu8(const __grid_constant__ CUtensorMap tm_u,
                                                     const __nv_bfloat16* __restrict__ phi_t,
                                                     int64_t T, int64_t C, int ncb,
                                                     float* __restrict__ phiu, int* status,
                                                     uint64_t wait_ns) {
  using namespace ap8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + A_DATA);  // full, mma, fin
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  const uint32_t full = tc::smem_u32(bars), mma_bar = tc::smem_u32(bars + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int item = blockIdx.x;
  const int tile = item / (N * ncb), rem = item % (N * ncb);
  const int j = rem / ncb, cb = rem % ncb;
  const int64_t t0 = (int64_t)tile * TT;
  const int c0 = cb * KB;

  if (threadIdx.x == 0) {
    tc::mbar_init(full, 1);
    tc::mbar_init(mma_bar, 1);
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), A_TMEM);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0) {
    const uint64_t pol = tc::policy_evict_last();  // U and phi are read by many CTAs
    // phi: the high rows of the KB / CH channel blocks of stream j (blocks past
    // the last channel are not loaded; the columns they feed are not stored)
    const int64_t nblk = (C + CH - 1) / CH;
    const int64_t q0 = (int64_t)c0 / CH;
    const int nb = (int)(nblk - q0 < KB / CH ? nblk - q0 : KB / CH);
    tc::mbar_arrive_expect_tx(full, (uint32_t)(3 * ATOM + nb * PHB));
    for (int a = 0; a < 3; ++a)
      tc::tma_load_2d(tc::smem_u32(smem + A_U_OFF + a * ATOM), &tm_u, full, 64 * a, (int)t0, pol);
    for (int q = 0; q < nb; ++q)
      tc::bulk_load(tc::smem_u32(smem + A_P_OFF + q * PHB), phi_t + ((q0 + q) * N + j) * (NL * CH),
                    PHB, full, pol);
  }
  bool ok = true;
  if (warp == 1 && lane == 0) {
    ok = tc::mbar_wait(full, 0, nullptr, wait_ns);
    if (ok) {
      tc::tc_fence_after();
      // D[tok][k] = sum over m' of U[tok][m'] PHI[m'][k]: K-steps 0..4 take u_hi
      // against phi rows 0..79, steps 6..10 u_lo against the same rows; steps 5
      // and 11 would only multiply U's zero padding.  PHI is MN-major with the
      // 32-byte swizzle: 16-channel atoms PHB bytes apart, 8-row groups 256 apart.
      constexpr uint32_t idesc = tc::idesc_bf16(TT, KB, false, true);
      const uint32_t ub = tc::smem_u32(smem + A_U_OFF), pb = tc::smem_u32(smem + A_P_OFF);
      int issued = 0;
#pragma unroll
      for (int s = 0; s < NU / 16; ++s) {
        if (s == 5 || s == 11) continue;
        const int r = s < 5 ? s : s - 6;  // 16-row block of phi^T
        const uint64_t da = tc::smem_desc(ub + (s / 4) * ATOM + (s % 4) * 32, 16, 1024, tc::SWZ_128B);
        const uint64_t db = tc::smem_desc(pb + r * 16 * 32, PHB, 256, tc::SWZ_32B);
        tc::mma_bf16(tmem, da, db, idesc, issued > 0 ? 1u : 0u);
        ++issued;
      }
      tc::mma_commit(mma_bar);
    } else {
      flag_status(status, MHC_ERR_TIMEOUT);
      // the copies already issued land before the CTA exits
      tc::mbar_wait(full, 0, nullptr, tc::kDrainWaitNs);
    }
  }
  // the epilogue: warp w reads TMEM lanes 32w..32w+31 (tokens), 256 columns
  const bool okall = __syncthreads_or(!ok) == 0;
  bool done = okall && tc::mbar_wait(mma_bar, 0, nullptr, wait_ns);
  if (okall && !done) flag_status(status, MHC_ERR_TIMEOUT);
  done = __all_sync(0xffffffffu, done);
  if (done) {
    // each warp turns its 32 token rows x 32 columns around in shared memory (the
    // U tile, free once the MMAs are done), so that 8 lanes store one token's
    // 128 contiguous bytes
    tc::tc_fence_after();
    float* xt = reinterpret_cast<float*>(smem + A_U_OFF) + warp * 32 * XT;
    const uint32_t lb = tmem + ((uint32_t)(32 * warp) << 16);
    const int rr = lane >> 3, cq = lane & 7;
#pragma unroll 1
    for (int q = 0; q < KB / 32; ++q) {
      float v0[16], v1[16];
      tc::tmem_ld16(lb + 32 * q, v0);
      tc::tmem_ld16(lb + 32 * q + 16, v1);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        *reinterpret_cast<float4*>(xt + lane * XT + 4 * e) =
            make_float4(v0[4 * e], v0[4 * e + 1], v0[4 * e + 2], v0[4 * e + 3]);
        *reinterpret_cast<float4*>(xt + lane * XT + 16 + 4 * e) =
            make_float4(v1[4 * e], v1[4 * e + 1], v1[4 * e + 2], v1[4 * e + 3]);
      }
      __syncwarp();
      const int64_t c = (int64_t)c0 + 32 * q + 4 * cq;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + rr;
        const int64_t t = t0 + 32 * warp + r;
        const float4 val = *reinterpret_cast<const float4*>(xt + r * XT + 4 * cq);
        if (t < T && c < C) __stcg(reinterpret_cast<float4*>(phiu + (t * N + j) * C + c), val);
      }
      __syncwarp();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // an MMA still running after a failed wait finishes before TMEM is freed
    if (!done && lane == 0 && okall) tc::mbar_wait(mma_bar, 0, nullptr, tc::kDrainWaitNs);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, A_TMEM);
  }
}

// ------------------------------------------------------- grad_x, grad_f_out
// One CTA visit per token: the token's H record in shared memory, its threads
// over 8-channel vectors of all eight streams.  CTA 0 also finishes grad_b
// and grad_alpha from the mapping's per-tile partial sums in a fixed order.
__global__ void __launch_bounds__(ap8::B_NT) k_gx8(int64_t T, int64_t C,
                                                   const __nv_bfloat16* __restrict__ x,
                                                   const __nv_bfloat16* __restrict__ G,
                                                   const __nv_bfloat16* __restrict__ g,
                                                   const float* __restrict__ phiu,
                                                   const float* __restrict__ coef,
                                                   const float* __restrict__ part, int nparts,
                                                   __nv_bfloat16* __restrict__ gx,
                                                   __nv_bfloat16* __restrict__ gf,
                                                   float* __restrict__ grad_b,
                                                   float* __restrict__ grad_alpha, int ag) {
  using namespace ap8;
  using CF = Coef<N>;
  __shared__ float hs[CF::SIZE];
  __shared__ float wsum[4][M + 3];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (blockIdx.x == 0) {
    constexpr int NC = M + 3;
    for (int col = lane; col < NC; col += 32) {
      float s = 0.0f;
      for (int q = warp; q < nparts; q += 4) s += __ldg(part + (int64_t)q * CF::DZ_SIZE + col);
      wsum[warp][col] = s;
    }
    __syncthreads();
    for (int col = tid; col < NC; col += B_NT) {
      const float a = ((wsum[0][col] + wsum[1][col]) + wsum[2][col]) + wsum[3][col];
      if (col < M) grad_b[col] = a;
      else if (ag == 3) grad_alpha[col - M] = a;
      wsum[0][col] = a;
    }
    __syncthreads();
    if (ag != 3 && tid == 0) *grad_alpha = (wsum[0][M] + wsum[0][M + 1]) + wsum[0][M + 2];
  }
  const int64_t nv = C / 8;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    for (int e = tid; e < CF::SIZE; e += B_NT) hs[e] = __ldg(coef + t * CF::SIZE + e);
    __syncthreads();
    const float kappa = hs[CF::KAPPA];
    for (int64_t v = tid; v < nv; v += B_NT) {
      const int64_t c = v * 8;
      float Gv[N][8], gv[8];
#pragma unroll
      for (int i = 0; i < N; ++i)
        unpack8b(__ldcs(reinterpret_cast<const uint4*>(G + (t * N + i) * C + c)), Gv[i]);
      unpack8b(__ldcs(reinterpret_cast<const uint4*>(g + t * C + c)), gv);
      if (gf != nullptr) {
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float a = 0.0f;
#pragma unroll
          for (int i = 0; i < N; ++i) a = fmaf(hs[CF::POST + i], Gv[i][e], a);
          o[e] = a;
        }
        __stcs(reinterpret_cast<uint4*>(gf + t * C + c), pack8b(o));
      }
#pragma unroll 1
      for (int jj = 0; jj < N; ++jj) {
        float xv[8], o[8];
        unpack8b(__ldcs(reinterpret_cast<const uint4*>(x + (t * N + jj) * C + c)), xv);
        const float4* pu = reinterpret_cast<const float4*>(phiu + (t * N + jj) * C + c);
        const float4 p0 = __ldcs(pu), p1 = __ldcs(pu + 1);
        const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float a = fmaf(hs[CF::PRE + jj], gv[e], pv[e]);
#pragma unroll
          for (int i = 0; i < N; ++i) a = fmaf(hs[CF::RES + i * N + jj], Gv[i][e], a);
          o[e] = fmaf(-kappa, xv[e], a);
        }
        __stcs(reinterpret_cast<uint4*>(gx + (t * N + jj) * C + c), pack8b(o));
      }
    }
  }
}

// --------------------------------------------------------------- grad_phi
__global__ void __launch_bounds__(ap8::C_NT) k_gphi8(const __grid_constant__ CUtensorMap tm_x,
                                                     const __grid_constant__ CUtensorMap tm_u,
                                                     int64_t T, int64_t C, int ncb,
                                                     float* __restrict__ grad_phi, int* status,
                                                     uint64_t wait_ns) {
  using namespace ap8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C_DATA);  // full[2] empty[2] done fin
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C_NS + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + C_NS + s); };
  const uint32_t done_bar = tc::smem_u32(bars + 2 * C_NS);
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * C_NS + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int j = blockIdx.x / ncb, cb = blockIdx.x % ncb;
  const int c0 = cb * CB;
  const int ntt = (int)((T + TT - 1) / TT);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C_NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    tc::mbar_init(done_bar, 1);
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), C_TMEM);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto give_up = [&]() {
    *abort_flag = 1;
    flag_status(status, MHC_ERR_TIMEOUT);
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    const uint64_t pol_x = tc::policy_evict_first(), pol_u = tc::policy_evict_last();
    int issued = 0;
    for (int it = 0; it < ntt; ++it) {
      const int s = it % C_NS;
      if (it >= C_NS && !tc::mbar_wait(empty(s), ((uint32_t)(it / C_NS) & 1u) ^ 1u, abort_flag,
                                       wait_ns)) {
        give_up();
        break;
      }
      const uint32_t base = tc::smem_u32(smem + s * C_STAGE);
      tc::mbar_arrive_expect_tx(full(s), (uint32_t)C_STAGE);
      for (int a = 0; a < 2; ++a)
        tc::tma_load_3d(base + C_X_OFF + a * ATOM, &tm_x, full(s), c0 + 64 * a, j, it * TT, pol_x);
      for (int a = 0; a < 3; ++a)
        tc::tma_load_2d(base + C_U_OFF + a * ATOM, &tm_u, full(s), 64 * a, it * TT, pol_u);
      ++issued;
    }
    for (int it = (issued > C_NS ? issued - C_NS : 0); it < issued; ++it)
      tc::mbar_wait(full(it % C_NS), (uint32_t)(it / C_NS) & 1u, nullptr, tc::kDrainWaitNs);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    // D[k][m'] += sum over 16 tokens of X[tok][k] U[tok][m']: A = X^T (MN-major,
    // two 64-channel atoms), B = U (MN-major, three 64-column atoms)
    constexpr uint32_t idesc = tc::idesc_bf16(CB, NU, true, true);
    bool any = false;
    for (int it = 0; it < ntt; ++it) {
      const int s = it % C_NS;
      if (!tc::mbar_wait(full(s), (uint32_t)(it / C_NS) & 1u, abort_flag, wait_ns)) {
        give_up();
        break;
      }
      tc::tc_fence_after();
      const uint32_t base = tc::smem_u32(smem + s * C_STAGE);
#pragma unroll
      for (int k = 0; k < TT / 16; ++k) {
        const uint64_t da = tc::smem_desc(base + C_X_OFF + k * 2048, ATOM, 1024, tc::SWZ_128B);
        const uint64_t db = tc::smem_desc(base + C_U_OFF + k * 2048, ATOM, 1024, tc::SWZ_128B);
        tc::mma_bf16(tmem, da, db, idesc, (it | k) != 0 ? 1u : 0u);
      }
      any = true;
      tc::mma_commit(empty(s));
    }
    if (!*abort_flag) tc::mma_commit(done_bar);
    if (any) {
      tc::mma_commit(fin_bar);
      tc::mbar_wait(fin_bar, 0, nullptr, tc::kDrainWaitNs);
    }
  }
  // ---- epilogue: warp w holds phi rows (channels) 32w..32w+31 of this block
  bool ok = !*abort_flag && tc::mbar_wait(done_bar, 0, abort_flag, wait_ns);
  if (!ok && !*abort_flag) give_up();
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc::tc_fence_after();
    const int64_t c = (int64_t)c0 + 32 * warp + lane;
    float* dst = grad_phi + ((int64_t)j * C + c) * M;
    const uint32_t lb = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll 1
    for (int q = 0; q < M / 16; ++q) {
      float hi[16], lo[16];
      tc::tmem_ld16(lb + 16 * q, hi);
      tc::tmem_ld16(lb + TcRec8::LO + 16 * q, lo);
      tc::tmem_ld_wait();
      if (c < C) {
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(dst + 16 * q + e) =
              make_float4(hi[e] + lo[e], hi[e + 1] + lo[e + 1], hi[e + 2] + lo[e + 2],
                          hi[e + 3] + lo[e + 3]);
      }
    }
  }
  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C_TMEM);
  }
}

// ------------------------------------------------------------------ host
cudaError_t apply8_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_split,
                               const void* G, const void* g, const float* coef, const void* urec,
                               const float* part, int nparts, float* phiu, void* gx, void* gf,
                               float* gphi, float* gb, float* ga, int ag, int* st,
                               int64_t wait_ns, cudaStream_t s) {
  using namespace ap8;
  const uint64_t wl = tc::wait_limit(wait_ns);
  CUtensorMap mu, mx;
  // U rows [T][192] bf16, boxes of 64 columns x 128 tokens
  const uint64_t du[2] = {(uint64_t)NU, (uint64_t)T};
  const uint64_t su[1] = {(uint64_t)NU * 2};
  const uint32_t bu[2] = {64, TT};
  cudaError_t e = make_tmap_bf16(&mu, urec, 2, du, su, bu, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  // x [T][8][C] bf16: 64 channels of one stream x 128 tokens
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {64, 1, TT};
  e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;

  const int ntt = (int)((T + TT - 1) / TT);
  const int ncb_a = (int)((C + KB - 1) / KB);
  e = cudaFuncSetAttribute(k_phiu8, cudaFuncAttributeMaxDynamicSharedMemorySize, A_SMEM);
  if (e != cudaSuccess) return e;
  k_phiu8<<<(unsigned)((int64_t)ntt * N * ncb_a), A_NT, A_SMEM, s>>>(mu, (const __nv_bfloat16*)phi_split, T, C, ncb_a, phiu, st,
                                                                    wl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const int64_t grid_b = T < 148 * 8 ? T : 148 * 8;
  k_gx8<<<(unsigned)grid_b, B_NT, 0, s>>>(T, C, (const __nv_bfloat16*)x, (const __nv_bfloat16*)G,
                                          (const __nv_bfloat16*)g, phiu, coef, part, nparts,
                                          (__nv_bfloat16*)gx, (__nv_bfloat16*)gf, gb, ga, ag);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const int ncb_c = (int)((C + CB - 1) / CB);
  e = cudaFuncSetAttribute(k_gphi8, cudaFuncAttributeMaxDynamicSharedMemorySize, C_SMEM);
  if (e != cudaSuccess) return e;
  k_gphi8<<<(unsigned)(N * ncb_c), C_NT, C_SMEM, s>>>(mx, mu, T, C, ncb_c, gphi, st, wl);
  return cudaGetLastError();
}

}  // namespace mhc
