// k_dots16_tc.cu -- the C-reductions of the n = 16 backward mapping (bf16
// activations): for every token t
//
//   <G_i, x_j> (256 pairs), <g, x_i> (16), <G_i, f_out> (16)
//
// summed over its C channels (the reverse mode of the mixing and of the layer
// input and output maps; chatgpz.de explainer, section "Von
// Residualverbindungen zu Hyperverbindungen"; reportify.cn [19]-[21]).  They go
// into the token's coefficient row at [288 + d] in the k_wide order (d < 256:
// i = d / 16, j = d % 16; then <g, x_i>, then <G_i, f>), where the backward
// epilogue of k_wide.cu reads them.
//
// The 256 products <G_i, x_j> of a token are a 16 x 16 matrix product over the
// channels.  Eight consecutive tokens' 16 stream rows are 128 consecutive rows
// of grad_x_next and of x ([T*16][C] row-major), so one tcgen05 MMA (M = N =
// 128, K = 16 channels) of those two slabs produces all eight tokens' products
// as the 16 x 16 diagonal blocks of D[128 x 128] (the off-diagonal blocks pair
// different tokens and are not read).  A CTA takes 16 tokens (two slabs, two
// 128-column TMEM accumulators) and streams the channels in 64-channel chunks
// through a three-stage ring (TMA, 128-byte rows and swizzle); four CUDA-core
// warps take <g, x_i> and <G_i, f_out> from the same stages and then read the
// diagonal blocks out of TMEM.  The split backward (training order) needs only
// <g, x_i>: no grad_x_next, no f_out, no MMA.  Every wait is bounded; on
// timeout the kernel records MHC_ERR_TIMEOUT, drains what it issued, frees TMEM
// and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

namespace d16 {
constexpr int N = 16;
constexpr int M = N * N + 2 * N;    // 288
constexpr int TG = 8;               // tokens per slab (8 x 16 rows = MMA M)
constexpr int NG = 2;               // slabs per CTA
constexpr int TC = TG * NG;         // 16 tokens per CTA
constexpr int CH = 64;              // channels per chunk: 128-byte rows
constexpr int SLAB = 128 * CH * 2;  // 16 KB
constexpr int ROWB = TC * CH * 2;   // g or f rows of the CTA's tokens: 2 KB
constexpr int X_OFF = 0;                          // x slabs
constexpr int G_OFF = NG * SLAB;                  // grad_x_next slabs
constexpr int GG_OFF = 2 * NG * SLAB;             // grad_h_in rows [16][64]
constexpr int F_OFF = GG_OFF + ROWB;              // f_out rows [16][64]
constexpr int STAGE = F_OFF + ROWB;               // 68 KB
constexpr int NS = 3;
constexpr int DATA = NS * STAGE;
constexpr int SMEM = DATA + 1024 + 256;
constexpr int NT = 6 * 32;          // TMA, MMA, four math warps
constexpr uint32_t TMEM_COLS = 256;
static_assert(STAGE % 1024 == 0 && SMEM <= 232448, "stage layout");
}  // namespace d16

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

template <bool FULL>
__global__ void __launch_bounds__(d16::NT, 1) k_dots16_tc(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_G,
    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_f, int64_t T,
    int64_t C, float* __restrict__ rows, int* status, uint64_t wait_ns) {
  using namespace d16;
  using CF = Coef<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DATA);  // full[NS] empty[NS] done fin
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + NS + s); };
  const uint32_t done_bar = tc::smem_u32(bars + 2 * NS);
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * NS + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t0 = (int64_t)blockIdx.x * TC;
  const int nch = (int)((C + CH - 1) / CH);
  constexpr uint32_t STAGE_TX = FULL ? STAGE : (uint32_t)(NG * SLAB + ROWB);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), (FULL ? 1 : 0) + 4);  // the MMA commit + every math warp
    }
    tc::mbar_init(done_bar, 1);
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (FULL && warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = FULL ? *tmem_slot : 0u;
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
        const uint32_t base = tc::smem_u32(smem + s * STAGE);
        const int c0 = cc * CH;
        tc::mbar_arrive_expect_tx(full(s), STAGE_TX);
        for (int gi = 0; gi < NG; ++gi) {
          const int r0 = (int)((t0 + gi * TG) * N);
          tc::tma_load_2d(base + X_OFF + gi * SLAB, &tm_x, full(s), c0, r0, pol);
          if constexpr (FULL) tc::tma_load_2d(base + G_OFF + gi * SLAB, &tm_G, full(s), c0, r0, pol);
        }
        tc::tma_load_2d(base + GG_OFF, &tm_g, full(s), c0, (int)t0, pol);
        if constexpr (FULL) tc::tma_load_2d(base + F_OFF, &tm_f, full(s), c0, (int)t0, pol);
        ++issued;
      }
      for (int cc = (issued > NS ? issued - NS : 0); cc < issued; ++cc)
        tc::mbar_wait(full(cc % NS), (uint32_t)(cc / NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (FULL && lane == 0) {
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
        const uint32_t base = tc::smem_u32(smem + s * STAGE);
#pragma unroll
        for (int gi = 0; gi < NG; ++gi)
#pragma unroll
          for (int k = 0; k < CH / 16; ++k) {
            const uint64_t a =
                tc::smem_desc(base + G_OFF + gi * SLAB + 32 * k, 16, 1024, tc::SWZ_128B);
            const uint64_t b =
                tc::smem_desc(base + X_OFF + gi * SLAB + 32 * k, 16, 1024, tc::SWZ_128B);
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
    // ------------------------- <g, x_i> and <G_i, f>; then the diagonal blocks
    // thread: token tt (0..15) of the CTA, streams 2p and 2p + 1
    const int tid = threadIdx.x - 64;
    const int tt = tid >> 3, p = tid & 7;
    const int gi = tt / TG, r0 = (tt % TG) * N;
    float gx[2] = {0.0f, 0.0f}, fG[2] = {0.0f, 0.0f};
    for (int cc = 0; cc < nch; ++cc) {
      const int s = cc % NS;
      if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
        give_up();
        break;
      }
      const uint8_t* st = smem + s * STAGE;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 gv = ld128sw(st + GG_OFF, tt, q);
#pragma unroll
        for (int h = 0; h < 2; ++h) dot8(gv, ld128sw(st + X_OFF + gi * SLAB, r0 + 2 * p + h, q), gx[h]);
        if constexpr (FULL) {
          const uint4 fv = ld128sw(st + F_OFF, tt, q);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            dot8(fv, ld128sw(st + G_OFF + gi * SLAB, r0 + 2 * p + h, q), fG[h]);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(empty(s));
    }
    const int64_t t = t0 + tt;
    bool ok = !*abort_flag;
    if (ok && t < T) {
      float* row = rows + t * CF::SIZE + M;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        row[256 + 2 * p + h] = gx[h];
        if constexpr (FULL) row[272 + 2 * p + h] = fG[h];
      }
    }
    if constexpr (FULL) {
      ok = ok && tc::mbar_wait(done_bar, 0, abort_flag, wait_ns);
      if (!ok && !*abort_flag) give_up();
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        // TMEM lane l of slab gi = (token 8 gi + l / 16, stream i = l % 16); this
        // warp's lanes 32 qd.. hold tokens 2 qd and 2 qd + 1 of each slab, whose
        // diagonal blocks sit at columns 32 qd .. 32 qd + 31
        tc::tc_fence_after();
        const int qd = warp & 3;
        const int i = lane & 15, hi = lane >> 4;
#pragma unroll 1
        for (int g2 = 0; g2 < NG; ++g2) {
          float v0[16], v1[16];
          const uint32_t ta = tmem + (uint32_t)(g2 * 128 + 32 * qd) + ((uint32_t)(32 * qd) << 16);
          tc::tmem_ld16(ta, v0);
          tc::tmem_ld16(ta + 16, v1);
          tc::tmem_ld_wait();
          const int64_t tk = t0 + g2 * TG + 2 * qd + hi;
          if (tk < T) {
            float* row = rows + tk * CF::SIZE + M + i * N;
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4*>(row + e) =
                  hi ? make_float4(v1[e], v1[e + 1], v1[e + 2], v1[e + 3])
                     : make_float4(v0[e], v0[e + 1], v0[e + 2], v0[e + 3]);
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (FULL && warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t dots16_dispatch(bool full, int64_t T, int64_t C, const void* x, const void* G,
                            const void* g, const void* f, float* rows, int* st, int64_t wait_ns,
                            cudaStream_t s) {
  using namespace d16;
  CUtensorMap mx, mG, mg, mf;
  // x and grad_x_next as [T*16][C]: 128-row slabs of eight tokens
  const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T * N};
  const uint64_t s2[1] = {(uint64_t)C * 2};
  const uint32_t b2[2] = {CH, 128};
  cudaError_t e = make_tmap_bf16(&mx, x, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  mG = mx;
  if (full) {
    e = make_tmap_bf16(&mG, G, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  // grad_h_in and f_out [T][C]: the CTA's 16 token rows
  const uint64_t d1[2] = {(uint64_t)C, (uint64_t)T};
  const uint32_t b1[2] = {CH, TC};
  e = make_tmap_bf16(&mg, g, 2, d1, s2, b1, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  mf = mg;
  if (full) {
    e = make_tmap_bf16(&mf, f, 2, d1, s2, b1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = (unsigned)((T + TC - 1) / TC);
  const uint64_t wl = tc::wait_limit(wait_ns);
  if (full) {
    e = cudaFuncSetAttribute(k_dots16_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    k_dots16_tc<true><<<grid, NT, SMEM, s>>>(mx, mG, mg, mf, T, C, rows, st, wl);
  } else {
    e = cudaFuncSetAttribute(k_dots16_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    k_dots16_tc<false><<<grid, NT, SMEM, s>>>(mx, mG, mg, mf, T, C, rows, st, wl);
  }
  return cudaGetLastError();
}

}  // namespace mhc
