// k_dots_tc.cu -- the C-reductions of the backward mapping for wide stream
// buffers (bf16 activations): for every token t, summed over its C channels,
//
//   <G_i, x_j> (n*n pairs), <g, x_i> (n), <G_i, f_out> (n)
//
// (the reverse mode of the mixing and of the layer input and output maps;
// chatgpz.de explainer, section "Von Residualverbindungen zu
// Hyperverbindungen"; reportify.cn [19]-[21]).
//   n = 16: into the token's coefficient row at [288 + d] in the k_wide order
//           (d < 256: i = d / 16, j = d % 16; then <g, x_i>, then <G_i, f>),
//           where the backward epilogue of k_wide.cu reads them; the split
//           backward (training order) needs only <g, x_i>;
//   n = 8:  all 80 into rows [T][80] (<G_i, x_j> at i*8 + j, <G_i, f> at
//           64 + i, <g, x_j> at 72 + j), which the n = 8 mapping reads in its
//           MAP_BWD_DOTS mode.
//
// The n*n products <G_i, x_j> of a token are an n x n matrix product over the
// channels.  128 / n consecutive tokens' stream rows are 128 consecutive rows
// of grad_x_next and of x ([T*n][C] row-major), so one tcgen05 MMA (M = N =
// 128, K = 16 channels) of those two slabs produces all their products as the
// n x n diagonal blocks of D[128 x 128] (the off-diagonal blocks pair different
// tokens and are not read).  A CTA takes two slabs (two 128-column TMEM
// accumulators) and streams the channels in 64-channel chunks through a
// three-stage ring (TMA, 128-byte rows and swizzle); four CUDA-core warps take
// the vector products (<g, x_i>, <G_i, f_out>) from the same stages and then
// read the diagonal blocks out of TMEM.  Every wait is bounded; on timeout the
// kernel records MHC_ERR_TIMEOUT, drains what it issued, frees TMEM and
// returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

// Modes: DOTS_FULL16 (n = 16, all 288), DOTS_GX16 (n = 16, <g, x_i> only),
// DOTS_RED8 (n = 8, all 80).
enum DotsMode { DOTS_FULL16 = 0, DOTS_GX16 = 1, DOTS_RED8 = 2 };

template <int MODE> struct DotsCfg {
  static constexpr int N = MODE == DOTS_RED8 ? 8 : 16;
  static constexpr bool MMA = MODE != DOTS_GX16;    // <G_i, x_j> on the tensor cores
  static constexpr bool USE_G = MODE != DOTS_GX16;
  static constexpr bool USE_g = true;               // <g, x_i>
  static constexpr bool USE_f = MODE != DOTS_GX16;  // <G_i, f>
  static constexpr int TG = 128 / N;                // tokens per slab
  static constexpr int NG = 2;                      // slabs per CTA
  static constexpr int TC = TG * NG;                // tokens per CTA
  static constexpr int CH = 64;                     // channels per chunk: 128-byte rows
  static constexpr int SLAB = 128 * CH * 2;         // 16 KB
  static constexpr int ROWB = TC * CH * 2;          // g or f rows of the CTA's tokens
  static constexpr int X_OFF = 0;
  static constexpr int G_OFF = NG * SLAB;
  static constexpr int GG_OFF = 2 * NG * SLAB;      // grad_h_in rows
  static constexpr int F_OFF = GG_OFF + ROWB;       // f_out rows
  static constexpr int STAGE = F_OFF + ROWB;
  static constexpr int TX = NG * SLAB * (USE_G ? 2 : 1) + ROWB * ((USE_g ? 1 : 0) + (USE_f ? 1 : 0));
  static constexpr int NS = 3;
  static constexpr int DATA = NS * STAGE;
  static constexpr int SMEM = DATA + 1024 + 256;
  static constexpr int NT = 6 * 32;                 // TMA, MMA, four math warps
  static constexpr uint32_t TMEM_COLS = 256;
  // math thread: token tt (0..TC-1), streams SP*p .. SP*p + SP - 1
  static constexpr int TPT = 128 / TC;              // threads per token: 8 (n = 16), 4 (n = 8)
  static constexpr int SP = N / TPT;                // 2 streams per thread
  static_assert(STAGE % 1024 == 0 && SMEM <= 232448, "stage layout");
};

namespace {
// 16-byte piece p of row r of a tile stored with the 128-byte swizzle
__device__ __forceinline__ uint4 ld128sw(const uint8_t* tile, int r, int p) {
  return *reinterpret_cast<const uint4*>(tile + r * 128 + ((p ^ (r & 7)) << 4));
}
__device__ __forceinline__ void dot8(uint4 a, uint4 b, float& acc) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    acc = fmaf(__uint_as_float(wa[h] << 16), __uint_as_float(wb[h] << 16), acc);
    acc = fmaf(__uint_as_float(wa[h] & 0xffff0000u), __uint_as_float(wb[h] & 0xffff0000u), acc);
  }
}
}  // namespace

// rows: n = 16, [T][Coef<16>::SIZE] coefficient rows; n = 8, [T][80].
template <int MODE>
__global__ void __launch_bounds__(DotsCfg<MODE>::NT, 1) k_dots_tc(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_G,
    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_f, int64_t T,
    int64_t C, float* __restrict__ rows, int* status, uint64_t wait_ns) {
  using D = DotsCfg<MODE>;
  constexpr int N = D::N, NS = D::NS;
  // destination of token t's products: <G_i, x_j> at GX + i*N + j, <g, x_i> at
  // GV + i, <G_i, f> at GF + i in a row of RS floats
  constexpr int RS = N == 16 ? Coef<16>::SIZE : N * N + 2 * N;
  constexpr int GX = N == 16 ? Coef<16>::M : 0;
  constexpr int GV = N == 16 ? GX + N * N : N * N + N;
  constexpr int GF = N == 16 ? GX + N * N + N : N * N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + D::DATA);  // full[NS] empty[NS] done fin
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + NS + s); };
  const uint32_t done_bar = tc::smem_u32(bars + 2 * NS);
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * NS + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t0 = (int64_t)blockIdx.x * D::TC;
  const int nch = (int)((C + D::CH - 1) / D::CH);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), (D::MMA ? 1 : 0) + 4);  // the MMA commit + every math warp
    }
    tc::mbar_init(done_bar, 1);
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (D::MMA && warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), D::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = D::MMA ? *tmem_slot : 0u;
  auto give_up = [&]() {
    *abort_flag = 1;
    flag_status(status, MHC_ERR_TIMEOUT);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      const uint64_t pol = tc::policy_evict_first();
      int issued = 0;
      for (int cc = 0; cc < nch; ++cc) {
        const int s = cc % NS;
        if (cc >= NS && !tc::mbar_wait(empty(s), ((uint32_t)(cc / NS) & 1u) ^ 1u, abort_flag,
                                       wait_ns)) {
          give_up();
          break;
        }
        const uint32_t base = tc::smem_u32(smem + s * D::STAGE);
        const int c0 = cc * D::CH;
        tc::mbar_arrive_expect_tx(full(s), (uint32_t)D::TX);
        for (int gi = 0; gi < D::NG; ++gi) {
          const int r0 = (int)((t0 + gi * D::TG) * N);
          tc::tma_load_2d(base + D::X_OFF + gi * D::SLAB, &tm_x, full(s), c0, r0, pol);
          if constexpr (D::USE_G)
            tc::tma_load_2d(base + D::G_OFF + gi * D::SLAB, &tm_G, full(s), c0, r0, pol);
        }
        if constexpr (D::USE_g) tc::tma_load_2d(base + D::GG_OFF, &tm_g, full(s), c0, (int)t0, pol);
        if constexpr (D::USE_f) tc::tma_load_2d(base + D::F_OFF, &tm_f, full(s), c0, (int)t0, pol);
        ++issued;
      }
      for (int cc = (issued > NS ? issued - NS : 0); cc < issued; ++cc)
        tc::mbar_wait(full(cc % NS), (uint32_t)(cc / NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (D::MMA && lane == 0) {
      // D_gi[(tok, i)][(tok', j)] += sum over 16 channels of G[tok][i][c] x[tok'][j][c]:
      // both operands K-major (the channels), 128 rows each
      constexpr uint32_t idesc = tc::idesc_bf16(128, 128);
      bool any = false;
      for (int cc = 0; cc < nch; ++cc) {
        const int s = cc % NS;
        if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t base = tc::smem_u32(smem + s * D::STAGE);
#pragma unroll
        for (int gi = 0; gi < D::NG; ++gi)
#pragma unroll
          for (int k = 0; k < D::CH / 16; ++k) {
            const uint64_t a =
                tc::smem_desc(base + D::G_OFF + gi * D::SLAB + 32 * k, 16, 1024, tc::SWZ_128B);
            const uint64_t b =
                tc::smem_desc(base + D::X_OFF + gi * D::SLAB + 32 * k, 16, 1024, tc::SWZ_128B);
            tc::mma_bf16(tmem + (uint32_t)(gi * 128), a, b, idesc, (cc | k) != 0 ? 1u : 0u);
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
  } else {
    // ------------- the vector products; then the diagonal blocks out of TMEM
    const int tid = threadIdx.x - 64;
    const int tt = tid / D::TPT, p = tid % D::TPT;
    const int gi = tt / D::TG, r0 = (tt % D::TG) * N;
    float gx[D::SP], fG[D::SP];
#pragma unroll
    for (int h = 0; h < D::SP; ++h) gx[h] = fG[h] = 0.0f;
    for (int cc = 0; cc < nch; ++cc) {
      const int s = cc % NS;
      if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
        give_up();
        break;
      }
      const uint8_t* st = smem + s * D::STAGE;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if constexpr (D::USE_g) {
          const uint4 gv = ld128sw(st + D::GG_OFF, tt, q);
#pragma unroll
          for (int h = 0; h < D::SP; ++h)
            dot8(gv, ld128sw(st + D::X_OFF + gi * D::SLAB, r0 + D::SP * p + h, q), gx[h]);
        }
        if constexpr (D::USE_f) {
          const uint4 fv = ld128sw(st + D::F_OFF, tt, q);
#pragma unroll
          for (int h = 0; h < D::SP; ++h)
            dot8(fv, ld128sw(st + D::G_OFF + gi * D::SLAB, r0 + D::SP * p + h, q), fG[h]);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(empty(s));
    }
    const int64_t t = t0 + tt;
    bool ok = !*abort_flag;
    if (ok && t < T) {
      float* row = rows + t * RS;
#pragma unroll
      for (int h = 0; h < D::SP; ++h) {
        if constexpr (D::USE_g) row[GV + D::SP * p + h] = gx[h];
        if constexpr (D::USE_f) row[GF + D::SP * p + h] = fG[h];
      }
    }
    if constexpr (D::MMA) {
      ok = ok && tc::mbar_wait(done_bar, 0, abort_flag, wait_ns);
      if (!ok && !*abort_flag) give_up();
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        // TMEM lane l of slab g2 = (token l / N of the slab, stream i = l % N);
        // this warp's lanes 32 qd.. hold tokens 32 qd / N .. of each slab, whose
        // diagonal blocks sit at columns 32 qd .. 32 qd + 31
        tc::tc_fence_after();
        const int qd = warp & 3;
        const int i = lane % N, blk = lane / N;  // blk: which of this warp's tokens
#pragma unroll 1
        for (int g2 = 0; g2 < D::NG; ++g2) {
          float v0[16], v1[16];
          const uint32_t ta = tmem + (uint32_t)(g2 * 128 + 32 * qd) + ((uint32_t)(32 * qd) << 16);
          tc::tmem_ld16(ta, v0);
          tc::tmem_ld16(ta + 16, v1);
          tc::tmem_ld_wait();
          const int64_t tk = t0 + g2 * D::TG + 32 * qd / N + blk;
          // the block's N columns start at column N * blk of the 32 read (the
          // choice among the 32 / N blocks is a register select, no indexing)
          float w[N];
#pragma unroll
          for (int bb = 0; bb < 32 / N; ++bb)
#pragma unroll
            for (int e = 0; e < N; ++e) {
              const int c = N * bb + e;
              const float v = c < 16 ? v0[c % 16] : v1[c % 16];
              w[e] = bb == 0 ? v : (blk == bb ? v : w[e]);
            }
          if (tk < T) {
            float* row = rows + tk * RS + GX + i * N;
#pragma unroll
            for (int e = 0; e < N; e += 4)
              *reinterpret_cast<float4*>(row + e) = make_float4(w[e], w[e + 1], w[e + 2], w[e + 3]);
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (D::MMA && warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, D::TMEM_COLS);
  }
}

namespace {
template <int MODE>
cudaError_t launch_dots(int64_t T, int64_t C, const void* x, const void* G, const void* g,
                        const void* f, float* rows, int* st, int64_t wait_ns, cudaStream_t s) {
  using D = DotsCfg<MODE>;
  constexpr int N = D::N;
  CUtensorMap mx, mG, mg, mf;
  // x and grad_x_next as [T*n][C]: slabs of 128 rows
  const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T * N};
  const uint64_t s2[1] = {(uint64_t)C * 2};
  const uint32_t b2[2] = {D::CH, 128};
  cudaError_t e = make_tmap_bf16(&mx, x, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  // maps a mode does not read are copies of the x map (never dereferenced)
  mG = mx;
  mg = mx;
  mf = mx;
  if (D::USE_G) {
    e = make_tmap_bf16(&mG, G, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  // grad_h_in and f_out [T][C]: the CTA's token rows
  const uint64_t d1[2] = {(uint64_t)C, (uint64_t)T};
  const uint32_t b1[2] = {D::CH, D::TC};
  if (D::USE_g) {
    e = make_tmap_bf16(&mg, g, 2, d1, s2, b1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  if (D::USE_f) {
    e = make_tmap_bf16(&mf, f, 2, d1, s2, b1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(k_dots_tc<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM);
  if (e != cudaSuccess) return e;
  k_dots_tc<MODE><<<(unsigned)((T + D::TC - 1) / D::TC), D::NT, D::SMEM, s>>>(
      mx, mG, mg, mf, T, C, rows, st, tc::wait_limit(wait_ns));
  return cudaGetLastError();
}
}  // namespace

cudaError_t dots16_dispatch(bool full, int64_t T, int64_t C, const void* x, const void* G,
                            const void* g, const void* f, float* rows, int* st, int64_t wait_ns,
                            cudaStream_t s) {
  return full ? launch_dots<DOTS_FULL16>(T, C, x, G, g, f, rows, st, wait_ns, s)
              : launch_dots<DOTS_GX16>(T, C, x, G, g, f, rows, st, wait_ns, s);
}

cudaError_t dots8_red_dispatch(int64_t T, int64_t C, const void* x, const void* G, const void* g,
                               const void* f, float* red, int* st, int64_t wait_ns,
                               cudaStream_t s) {
  return launch_dots<DOTS_RED8>(T, C, x, G, g, f, red, st, wait_ns, s);
}

}  // namespace mhc
