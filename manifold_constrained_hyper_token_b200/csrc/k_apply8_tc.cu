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
// RMS-normalised projection; reportify.cn [19]-[21]).  At n = 8 the grad_phi
// accumulators of the channels a CTA covers do not fit beside the phi u
// accumulators in TMEM, so the two contractions run as two tensor-core kernels:
//
//   k_gxu8    grad_x and grad_f_out for (128-token tile, 32 channels of all 8
//             streams) items, one persistent CTA per SM: phi u as
//             D[128 x 256] = U[128 x 192] . PHI[192 x 256] (tcgen05, bf16
//             operands, fp32 in TMEM, two accumulators so that one item's MMAs
//             overlap the previous item's epilogue); the epilogue warps turn
//             8 tokens' rows of D around in shared memory and add the CUDA-core
//             terms from x, grad_x_next and grad_h_in, which they stage one
//             step ahead with 16-byte cp.async copies (4 lanes cover one
//             token's 64-byte row piece), so phi u never leaves the chip;
//   k_gphi8   grad_phi for 128 rows of phi: D[128 x 192] += X^T[128 x 128] .
//             U[128 x 192] over every token tile (tcgen05), then
//             grad_phi = D[:, m] + D[:, 96 + m]; the (block, tile) units are
//             split evenly over persistent CTAs, and k_gphi8_fin adds the
//             parts of blocks that two or more CTAs share;
//   k_bias8   grad_b and grad_alpha from the mapping's per-tile partial sums.
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
constexpr int CH = 16;                  // channels per block of the tiled phi^T copy
constexpr int NL = 2 * M;               // rows per block (80 high, 80 low)
constexpr int PHB = M * CH * 2;         // the 80 high rows of one block: 2.5 KB
// k_gxu8
constexpr int FS = 32;                  // channels per item (all 8 streams)
constexpr int FN = N * FS;              // MMA N: 256 columns, column 32 j + channel
constexpr int F_U_OFF = 0;              // U tile: three atoms (48 KB)
constexpr int F_P_OFF = 3 * ATOM;       // phi: 16 atoms (stream j, 16-channel half) of PHB
constexpr int F_W_OFF = F_P_OFF + 2 * N * PHB;  // the epilogue warps' areas
constexpr int NEPI = 8;                 // epilogue warps: two per TMEM lane quarter
constexpr int CK = 8;                   // tokens per epilogue step
constexpr int XTS = 260;                // row stride (floats) of the transpose buffer
constexpr int RS = (2 * N + 1) * 64;    // a token's staged rows: grad_x_next x 8, x x 8, grad_h_in
constexpr int RX = N * 64;              // offset of the x rows in them
constexpr int RG = 2 * N * 64;          // and of the grad_h_in row
constexpr int HS = 84;                  // H record in shared memory: res, pre, post, kappa
constexpr int SL_H = CK * RS;           // ring slot: [CK][RS] rows, then [CK][HS] records
constexpr int SLOT = SL_H + CK * HS * 4;
constexpr int NSLOT = 2;                // steps staged: the current one and the next
constexpr int W_RING = CK * XTS * 4;
constexpr int W_BYTES = W_RING + NSLOT * SLOT;
constexpr int F_DATA = F_W_OFF + 4 * W_BYTES;   // one area per lane quarter
constexpr int F_SMEM = F_DATA + 1024 + 128;
constexpr int F_NT = (2 + NEPI) * 32;   // TMA, MMA, epilogue x8
constexpr uint32_t F_TMEM = 512;
static_assert(F_P_OFF % 1024 == 0 && F_W_OFF % 1024 == 0, "operand alignment");
static_assert(W_BYTES % 16 == 0 && SLOT % 16 == 0 && W_RING % 16 == 0, "alignment");
static_assert((XTS * 4) % 128 == 16 && RS % 128 == 64 && (HS * 4) % 16 == 0, "bank spread");
// k_gphi8
constexpr int CB = 128;                 // phi rows (channels of one stream) per CTA (MMA M)
constexpr int C_X_OFF = 0;              // x tile [128 tokens][128 channels]: two atoms
constexpr int C_U_OFF = 2 * ATOM;       // U tile: three atoms
constexpr int C_STAGE = 5 * ATOM;       // 80 KB
constexpr int C_NS = 2;
constexpr int C_DATA = C_NS * C_STAGE;
constexpr int C_SMEM = C_DATA + 1024 + 128;
constexpr int C_NT = 6 * 32;            // TMA, MMA, four epilogue warps
constexpr uint32_t C_TMEM = 512;        // two accumulators of NU columns
constexpr int C_MAXGRID = 256;          // partial-sum slots are sized for this many CTAs
// k_bias8
constexpr int B_NT = 128;
static_assert(F_SMEM <= 232448 && C_SMEM <= 232448, "shared memory");
}  // namespace ap8

namespace {
// 16-byte asynchronous global -> shared copies (L2 only), in commit groups
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void cp_async_wait0() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
// wait until at most one committed group of this thread is still in flight
__device__ __forceinline__ void cp_async_wait1() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}
}  // namespace

// ------------------------------------------------------- grad_x, grad_f_out
// Items it = blockIdx.x + k * gridDim.x in (tile, 32-channel slice) order, so
// the CTAs work on neighbouring slices of the same token rows at any time.
// Warp 0 loads each item's U tile (when the tile changes) and the 16 phi atoms
// of its slice into single-buffered operands; warp 1 issues the MMAs into the
// item's accumulator (columns 256 (k & 1)..); warps 2..9 work in pairs, one
// pair per TMEM lane quarter, on its 32 tokens in four steps of 8 tokens,
// each warp of a pair on four of the eight streams.  A step's x, grad_x_next
// and grad_h_in rows and H records are copied into the pair's two-slot ring
// one step ahead (cp.async, 16 bytes per lane, 4 lanes per 64-byte row piece);
// the 8 tokens' D rows go through the pair's transpose buffer, and the lanes
// then work as 8 tokens x 4 groups of 8 channels.  A 64-thread named barrier
// orders the pair's shared buffers.
__global__ void __launch_bounds__(ap8::F_NT, 1) k_gxu8(
    const __grid_constant__ CUtensorMap tm_u, const __nv_bfloat16* __restrict__ phi_t, int64_t T,
    int64_t C, int nsl, int64_t nitems, const __nv_bfloat16* __restrict__ x,
    const __nv_bfloat16* __restrict__ G, const __nv_bfloat16* __restrict__ g,
    const float* __restrict__ coef, __nv_bfloat16* __restrict__ gx,
    __nv_bfloat16* __restrict__ gf, int* status, uint64_t wait_ns) {
  using namespace ap8;
  using CF = Coef<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  // op_full op_empty dfull[2] dempty[2] fin, the TMEM address, the abort flag
  // and the epilogue pairs' wait results
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + F_DATA);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* pair_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [4][2]
  const uint32_t op_full = tc::smem_u32(bars), op_empty = tc::smem_u32(bars + 1);
  auto dfull = [&](int d) { return tc::smem_u32(bars + 2 + d); };
  auto dempty = [&](int d) { return tc::smem_u32(bars + 4 + d); };
  const uint32_t fin_bar = tc::smem_u32(bars + 6);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nblk = (C + CH - 1) / CH;

  if (threadIdx.x == 0) {
    tc::mbar_init(op_full, 1);
    tc::mbar_init(op_empty, 1);
    for (int d = 0; d < 2; ++d) {
      tc::mbar_init(dfull(d), 1);
      tc::mbar_init(dempty(d), NEPI);
    }
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) tc::tma_prefetch_desc(&tm_u);
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), F_TMEM);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      const uint64_t pol = tc::policy_evict_last();  // U and phi are read by many CTAs
      int64_t prev_tile = -1;
      int li = 0;
      for (int64_t it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
        const int64_t tile = it / nsl;
        const int64_t q0 = (it % nsl) * (FS / CH);
        // the phi blocks past the last channel are not loaded (their columns
        // are not stored)
        const int nb = (int)(nblk - q0 < FS / CH ? nblk - q0 : FS / CH);
        if (li >= 1 && !tc::mbar_wait(op_empty, (uint32_t)(li - 1) & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        const bool new_u = tile != prev_tile;
        tc::mbar_arrive_expect_tx(op_full, (uint32_t)((new_u ? 3 * ATOM : 0) + nb * N * PHB));
        if (new_u)
          for (int a = 0; a < 3; ++a)
            tc::tma_load_2d(tc::smem_u32(smem + F_U_OFF + a * ATOM), &tm_u, op_full, 64 * a,
                            (int)(tile * TT), pol);
        for (int h = 0; h < nb; ++h)
          for (int j = 0; j < N; ++j)
            tc::bulk_load(tc::smem_u32(smem + F_P_OFF + (2 * j + h) * PHB),
                          phi_t + ((q0 + h) * N + j) * (NL * CH), PHB, op_full, pol);
        prev_tile = tile;
      }
      // every copy issued here has landed before the CTA can exit
      if (li > 0) tc::mbar_wait(op_full, (uint32_t)(li - 1) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      // D[tok][32 j + c] = sum over m' of U[tok][m'] PHI[m'][32 j + c]: K-steps
      // 0..4 take u_hi against phi rows 0..79, steps 6..10 u_lo against the
      // same rows (5 and 11 would only multiply U's zero padding).  PHI is
      // MN-major with the 32-byte swizzle: 16-channel atoms PHB bytes apart,
      // 8-row groups 256 apart.
      constexpr uint32_t idesc = tc::idesc_bf16(TT, FN, false, true);
      const uint32_t ub = tc::smem_u32(smem + F_U_OFF), pb = tc::smem_u32(smem + F_P_OFF);
      bool any = false;
      int li = 0;
      for (int64_t it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
        const int d = li & 1;
        if (li >= 2 &&
            !tc::mbar_wait(dempty(d), ((uint32_t)(li >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        if (!tc::mbar_wait(op_full, (uint32_t)li & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(d * FN);
        int issued = 0;
#pragma unroll
        for (int s = 0; s < NU / 16; ++s) {
          if (s == 5 || s == 11) continue;
          const int r = s < 5 ? s : s - 6;  // 16-row block of phi^T
          const uint64_t da =
              tc::smem_desc(ub + (s / 4) * ATOM + (s % 4) * 32, 16, 1024, tc::SWZ_128B);
          const uint64_t db = tc::smem_desc(pb + r * 16 * 32, PHB, 256, tc::SWZ_32B);
          tc::mma_bf16(dt, da, db, idesc, issued > 0 ? 1u : 0u);
          ++issued;
        }
        any = true;
        tc::mma_commit(op_empty);
        tc::mma_commit(dfull(d));
      }
      // every MMA issued here has finished before TMEM is freed
      if (any) {
        tc::mma_commit(fin_bar);
        tc::mbar_wait(fin_bar, 0, nullptr, tc::kDrainWaitNs);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // warps qd + 2 and qd + 6 (mod 4 = qd) share TMEM lane quarter qd, its
    // transpose buffer and its ring; warp half hw takes streams 4 hw .. 4 hw + 3
    const int ew = warp - 2;
    const int qd = warp & 3;             // TMEM lane quarter: tokens 32 qd .. 32 qd + 31
    const int hw = ew >> 2;
    const int pbar = 1 + qd;             // named barrier of the pair
    uint8_t* wbase = smem + F_W_OFF + qd * W_BYTES;
    float* xt = reinterpret_cast<float*>(wbase);
    const uint32_t ring = tc::smem_u32(wbase + W_RING);
    const int r = lane >> 2, q = lane & 3;  // token of the step, 8-channel group
    // this warp's share of a step's H records: chunks f = lane + 32 k
    // (k = 3 hw .. 3 hw + 2) of the 8 x 21 16-byte chunks (rows [0, 80) and
    // kappa of each token)
    int h_tok[3], h_src[3], h_dst[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int f = lane + 32 * (3 * hw + k);
      const int tk = f / 21, kk = f % 21;
      h_tok[k] = f < CK * 21 ? tk : CK;
      h_src[k] = tk * CF::SIZE + (kk < 20 ? 4 * kk : CF::KAPPA);
      h_dst[k] = SL_H + (tk * HS + 4 * kk) * 4;
    }
    // stage this warp's half of step s = (item (tile, slice), ci) into ring
    // slot s % 2: grad_x_next and x rows 4 hw .. 4 hw + 3 (and grad_h_in for
    // hw = 1) and a third of the H records
    auto stage = [&](int s, int tile, int sl, int ci) {
      if (tile >= 0) {
        const uint32_t dst = ring + (uint32_t)((s & 1) * SLOT);
        const int64_t tb = (int64_t)tile * TT + 32 * qd + CK * ci;
        const int64_t t = tb + r, c = (int64_t)sl * FS + 8 * q;
        if (t < T && c < C) {
          const uint32_t rd = dst + (uint32_t)(r * RS + 16 * q);
          const int64_t off = (t * N + 4 * hw) * C + c;
          const __nv_bfloat16* pG = G + off;
          const __nv_bfloat16* pX = x + off;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            cp_async16(rd + 64 * (4 * hw + i), pG + i * C);
            cp_async16(rd + RX + 64 * (4 * hw + i), pX + i * C);
          }
          if (hw == 1) cp_async16(rd + RG, g + t * C + c);
        }
        const float* hsrc = coef + tb * CF::SIZE;
#pragma unroll
        for (int k = 0; k < 3; ++k)
          if (h_tok[k] < CK && tb + h_tok[k] < T)
            cp_async16(dst + (uint32_t)h_dst[k], hsrc + h_src[k]);
      }
      cp_async_commit();
    };
    const int nit = (int)nitems, grid = (int)gridDim.x;
    int it = (int)blockIdx.x;
    int tile = it / nsl, sl = it - tile * nsl;
    stage(0, tile, sl, 0);
    int s = 0;
    bool ok = true;
    int li = 0;
    for (; it < nit && ok; it += grid, ++li) {
      const int d = li & 1;
      const int itn = it + grid;
      const int tilen = itn < nit ? itn / nsl : -1, sln = itn - (itn / nsl) * nsl;
      const int64_t c = (int64_t)sl * FS + 8 * q;
      const int64_t tile0 = (int64_t)tile * TT + 32 * qd;
      const uint32_t taddr = tmem + (uint32_t)(d * FN) + ((uint32_t)(32 * qd) << 16);
#pragma unroll 1
      for (int ci = 0; ci < 4; ++ci, ++s) {
        if (ci < 3) stage(s + 1, tile, sl, ci + 1);
        else stage(s + 1, tilen, sln, 0);
        const int64_t t = tile0 + CK * ci + r;
        const bool vld = t < T && c < C;
        if (ci == 0) {
          // both warps of the pair take the same decision
          bool okw = tc::mbar_wait(dfull(d), (uint32_t)(li >> 1) & 1u, abort_flag, wait_ns);
          okw = __all_sync(0xffffffffu, okw);
          if (!okw && !*abort_flag) give_up();
          if (lane == 0) pair_ok[2 * qd + hw] = okw ? 1 : 0;
          named_bar_sync(pbar, 64);
          ok = pair_ok[2 * qd] != 0 && pair_ok[2 * qd + 1] != 0;
          if (!ok) break;
          tc::tc_fence_after();
        }
        // this warp's 128 D columns of the step's 8 tokens (lanes 8 ci ..
        // 8 ci + 7 of the quarter) into the transpose buffer
        const int row = lane - CK * ci;
        const bool mine = row >= 0 && row < CK;
#pragma unroll 1
        for (int kb = 0; kb < 2; ++kb) {
          const int col = 128 * hw + 64 * kb;
          float v[4][16];
#pragma unroll
          for (int u = 0; u < 4; ++u) tc::tmem_ld16(taddr + col + 16 * u, v[u]);
          tc::tmem_ld_wait();
          if (mine) {
            float* dst = xt + row * XTS + col;
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                *reinterpret_cast<float4*>(dst + 16 * u + 4 * e) =
                    make_float4(v[u][4 * e], v[u][4 * e + 1], v[u][4 * e + 2], v[u][4 * e + 3]);
          }
        }
        if (ci == 3) {
          // the item's accumulator is free for the MMAs two items on
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(dempty(d));
        }
        cp_async_wait1();           // this warp's copies of the step
        named_bar_sync(pbar, 64);   // and the other warp's, and both halves of D
        const uint8_t* slot = wbase + W_RING + (s & 1) * SLOT;
        const uint8_t* rows = slot + r * RS + 16 * q;
        const float* hr = reinterpret_cast<const float*>(slot + SL_H) + r * HS;
        // acc[jj][p]: channels 2p, 2p + 1 of stream 4 hw + jj, from phi u
        uint64_t acc[4][4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float* a = xt + r * XTS + 32 * (4 * hw + jj) + 8 * q;
          const ulonglong2 a0 = *reinterpret_cast<const ulonglong2*>(a);
          const ulonglong2 a1 = *reinterpret_cast<const ulonglong2*>(a + 4);
          acc[jj][0] = a0.x;
          acc[jj][1] = a0.y;
          acc[jj][2] = a1.x;
          acc[jj][3] = a1.y;
        }
        {
          const uint4 gw = *reinterpret_cast<const uint4*>(rows + RG);
          const uint64_t gp[4] = {bf2_to_f2(gw.x), bf2_to_f2(gw.y), bf2_to_f2(gw.z),
                                  bf2_to_f2(gw.w)};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const float h = hr[CF::PRE + 4 * hw + jj];
            const uint64_t hh = f2pack(h, h);
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[jj][p] = f2fma(hh, gp[p], acc[jj][p]);
          }
        }
        uint64_t gfa[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < N; ++i) {
          const uint4 w = *reinterpret_cast<const uint4*>(rows + 64 * i);
          const uint64_t Gp[4] = {bf2_to_f2(w.x), bf2_to_f2(w.y), bf2_to_f2(w.z), bf2_to_f2(w.w)};
          if (hw == 0) {
            const float hpo = hr[CF::POST + i];
            const uint64_t hh = f2pack(hpo, hpo);
#pragma unroll
            for (int p = 0; p < 4; ++p) gfa[p] = f2fma(hh, Gp[p], gfa[p]);
          }
          const float4 h = *reinterpret_cast<const float4*>(hr + CF::RES + N * i + 4 * hw);
          const float hres[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint64_t hj = f2pack(hres[jj], hres[jj]);
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[jj][p] = f2fma(hj, Gp[p], acc[jj][p]);
          }
        }
        if (vld) {
          const float nk = -hr[M];
          const uint64_t kk = f2pack(nk, nk);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint4 xq = *reinterpret_cast<const uint4*>(rows + RX + 64 * (4 * hw + jj));
            const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
            uint32_t o[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) o[p] = f2_to_bf2(f2fma(kk, bf2_to_f2(xw[p]), acc[jj][p]));
            __stcs(reinterpret_cast<uint4*>(gx + (t * N + 4 * hw + jj) * C + c),
                   make_uint4(o[0], o[1], o[2], o[3]));
          }
          if (hw == 0 && gf != nullptr)
            __stcs(reinterpret_cast<uint4*>(gf + t * C + c),
                   make_uint4(f2_to_bf2(gfa[0]), f2_to_bf2(gfa[1]), f2_to_bf2(gfa[2]),
                              f2_to_bf2(gfa[3])));
        }
        named_bar_sync(pbar, 64);  // the transpose buffer and the slot are rewritten later
      }
      tile = tilen;
      sl = sln;
    }
    cp_async_wait0();
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, F_TMEM);
  }
}

// grad_b and grad_alpha: the mapping's per-tile partial sums in a fixed order
// (warp w adds partials w, w + 4, ...; then the four warps' sums in order).
__global__ void __launch_bounds__(ap8::B_NT) k_bias8(const float* __restrict__ part, int nparts,
                                                     float* __restrict__ grad_b,
                                                     float* __restrict__ grad_alpha, int ag) {
  using namespace ap8;
  using CF = Coef<N>;
  constexpr int NC = M + 3;
  __shared__ float wsum[4][NC];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
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

// --------------------------------------------------------------- grad_phi
// The (128-channel block of one stream, 128-token tile) units, block-major,
// are split evenly over the CTAs (a contiguous range each), so that every SM
// has the same number of tiles.  A CTA's range cuts into segments, one per
// block it touches; a segment accumulates D[128 x 192] += X^T U over its tiles
// (two TMEM accumulators, alternating, so one segment's epilogue overlaps the
// next segment's MMAs).  A segment that covers its whole block writes grad_phi;
// the first and last segments of a range can be parts of a block, and write
// the CTA's partial slots 0 and 1 instead, which k_gphi8_fin adds in CTA
// order.  The owner of unit u is the CTA b with lo_b <= u < lo_{b+1},
// lo_b = floor(b * units / grid).
__global__ void __launch_bounds__(ap8::C_NT, 1) k_gphi8(const __grid_constant__ CUtensorMap tm_x,
                                                        const __grid_constant__ CUtensorMap tm_u,
                                                        int64_t T, int64_t C, int ncb,
                                                        int64_t nunits,
                                                        float* __restrict__ grad_phi,
                                                        float* __restrict__ partial, int* status,
                                                        uint64_t wait_ns) {
  using namespace ap8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  // full[2] empty[2] dfull[2] dempty[2] fin
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C_DATA);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C_NS + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + C_NS + s); };
  auto dfull = [&](int d) { return tc::smem_u32(bars + 2 * C_NS + d); };
  auto dempty = [&](int d) { return tc::smem_u32(bars + 2 * C_NS + 2 + d); };
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * C_NS + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t ntt = (T + TT - 1) / TT;
  const int64_t lo = (int64_t)blockIdx.x * nunits / gridDim.x;
  const int64_t hi = ((int64_t)blockIdx.x + 1) * nunits / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C_NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    for (int d = 0; d < 2; ++d) {
      tc::mbar_init(dfull(d), 1);
      tc::mbar_init(dempty(d), 4);  // the four epilogue warps
    }
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      const uint64_t pol_x = tc::policy_evict_first(), pol_u = tc::policy_evict_last();
      int64_t k = 0;
      for (int64_t u = lo; u < hi; ++u, ++k) {
        const int s = (int)(k % C_NS);
        if (k >= C_NS && !tc::mbar_wait(empty(s), ((uint32_t)(k / C_NS) & 1u) ^ 1u, abort_flag,
                                        wait_ns)) {
          give_up();
          break;
        }
        const int64_t blk = u / ntt, tile = u % ntt;
        const int j = (int)(blk / ncb), c0 = (int)(blk % ncb) * CB;
        const uint32_t base = tc::smem_u32(smem + s * C_STAGE);
        tc::mbar_arrive_expect_tx(full(s), (uint32_t)C_STAGE);
        for (int a = 0; a < 2; ++a)
          tc::tma_load_3d(base + C_X_OFF + a * ATOM, &tm_x, full(s), c0 + 64 * a, j,
                          (int)(tile * TT), pol_x);
        for (int a = 0; a < 3; ++a)
          tc::tma_load_2d(base + C_U_OFF + a * ATOM, &tm_u, full(s), 64 * a, (int)(tile * TT),
                          pol_u);
      }
      // every copy issued here has landed before the CTA can exit
      for (int64_t q = (k > C_NS ? k - C_NS : 0); q < k; ++q)
        tc::mbar_wait(full((int)(q % C_NS)), (uint32_t)(q / C_NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    // D[k][m'] += sum over 16 tokens of X[tok][k] U[tok][m']: A = X^T (MN-major,
    // two 64-channel atoms), B = U (MN-major, three 64-column atoms)
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(CB, NU, true, true);
      bool any = false;
      int seg = 0;
      int64_t k = 0;
      for (int64_t u = lo; u < hi; ++u, ++k) {
        const int s = (int)(k % C_NS);
        const int64_t tile = u % ntt;
        const bool first = u == lo || tile == 0, last = u == hi - 1 || tile == ntt - 1;
        const int d = seg & 1;
        if (first && seg >= 2 &&
            !tc::mbar_wait(dempty(d), ((uint32_t)(seg >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        if (!tc::mbar_wait(full(s), (uint32_t)(k / C_NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t base = tc::smem_u32(smem + s * C_STAGE);
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk) {
          const uint64_t da = tc::smem_desc(base + C_X_OFF + kk * 2048, ATOM, 1024, tc::SWZ_128B);
          const uint64_t db = tc::smem_desc(base + C_U_OFF + kk * 2048, ATOM, 1024, tc::SWZ_128B);
          tc::mma_bf16(tmem + (uint32_t)(d * NU), da, db, idesc, (first && kk == 0) ? 0u : 1u);
        }
        any = true;
        tc::mma_commit(empty(s));
        if (last) {
          tc::mma_commit(dfull(d));
          ++seg;
        }
      }
      // every MMA issued here has finished before TMEM is freed
      if (any) {
        tc::mma_commit(fin_bar);
        tc::mbar_wait(fin_bar, 0, nullptr, tc::kDrainWaitNs);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // warp w holds phi rows (channels) 32 (w % 4).. of the segment's block
    const int q = warp & 3;
    const int64_t b0 = lo / ntt, b1 = hi > lo ? (hi - 1) / ntt : b0 - 1;
    bool ok = true;
    for (int64_t blk = b0; blk <= b1 && ok; ++blk) {
      const int si = (int)(blk - b0), d = si & 1;
      bool okw = tc::mbar_wait(dfull(d), (uint32_t)(si >> 1) & 1u, abort_flag, wait_ns);
      if (!okw && !*abort_flag) give_up();
      ok = __all_sync(0xffffffffu, okw);
      if (!ok) break;
      tc::tc_fence_after();
      const int64_t s_lo = blk * ntt > lo ? blk * ntt : lo;
      const int64_t s_hi = (blk + 1) * ntt < hi ? (blk + 1) * ntt : hi;
      const bool whole = s_lo == blk * ntt && s_hi == (blk + 1) * ntt;
      const int j = (int)(blk / ncb);
      const int64_t c = (blk % ncb) * CB + 32 * q + lane;
      float* dst = whole ? grad_phi + ((int64_t)j * C + c) * M
                         : partial + (((int64_t)blockIdx.x * 2 + (si == 0 ? 0 : 1)) * CB +
                                      32 * q + lane) * M;
      const uint32_t lb = tmem + (uint32_t)(d * NU) + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int qq = 0; qq < M / 16; ++qq) {
        float hv[16], lv[16];
        tc::tmem_ld16(lb + 16 * qq, hv);
        tc::tmem_ld16(lb + TcRec8::LO + 16 * qq, lv);
        tc::tmem_ld_wait();
        if (c < C) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(dst + 16 * qq + e) =
                make_float4(hv[e] + lv[e], hv[e + 1] + lv[e + 1], hv[e + 2] + lv[e + 2],
                            hv[e + 3] + lv[e + 3]);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(dempty(d));
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C_TMEM);
  }
}

// grad_phi rows of the blocks that several CTAs share: the CTAs' partial
// slots added in CTA order.  One CTA per block (it returns at once when one CTA
// covered the block), its threads along the rows' 16-byte pieces.
__global__ void __launch_bounds__(256) k_gphi8_fin(int64_t C, int ncb, int64_t ntt, int64_t nunits,
                                            int grid, const float* __restrict__ partial,
                                            float* __restrict__ grad_phi) {
  using namespace ap8;
  const int64_t blk = blockIdx.x;
  auto owner = [&](int64_t u) { return ((u + 1) * grid - 1) / nunits; };
  const int64_t bfirst = owner(blk * ntt), blast = owner((blk + 1) * ntt - 1);
  if (bfirst == blast) return;
  for (int e = threadIdx.x; e < CB * (M / 4); e += blockDim.x) {
    const int row = e / (M / 4), m = 4 * (e % (M / 4));
    const int64_t c = (blk % ncb) * CB + row;
    if (c >= C) continue;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int64_t b = bfirst; b <= blast; ++b) {
      const int64_t lo_b = b * nunits / grid;
      const int slot = lo_b / ntt == blk ? 0 : 1;
      const float4 v =
          *reinterpret_cast<const float4*>(partial + ((b * 2 + slot) * CB + row) * M + m);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    *reinterpret_cast<float4*>(grad_phi + ((blk / ncb) * C + c) * M + m) = acc;
  }
}

// ------------------------------------------------------------------ host
size_t apply8_tc_scratch_bytes() { return (size_t)ap8::C_MAXGRID * 2 * ap8::CB * ap8::M * 4; }

cudaError_t apply8_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_split,
                               const void* G, const void* g, const float* coef, const void* urec,
                               const float* part, int nparts, void* gx, void* gf, float* gphi,
                               float* gb, float* ga, int ag, float* gpart, int* st,
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

  const int64_t ntt = (T + TT - 1) / TT;
  const int nsl = (int)((C + FS - 1) / FS);
  const int64_t nitems = ntt * nsl;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid_a = nitems < nsm ? nitems : nsm;
  if (nitems > 0x7fffffff - grid_a) return cudaErrorInvalidValue;  // 32-bit item indices
  e = cudaFuncSetAttribute(k_gxu8, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM);
  if (e != cudaSuccess) return e;
  k_gxu8<<<(unsigned)grid_a, F_NT, F_SMEM, s>>>(
      mu, (const __nv_bfloat16*)phi_split, T, C, nsl, nitems, (const __nv_bfloat16*)x,
      (const __nv_bfloat16*)G, (const __nv_bfloat16*)g, coef, (__nv_bfloat16*)gx,
      (__nv_bfloat16*)gf, st, wl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  k_bias8<<<1, B_NT, 0, s>>>(part, nparts, gb, ga, ag);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const int ncb_c = (int)((C + CB - 1) / CB);
  const int64_t nunits_c = (int64_t)N * ncb_c * ntt;
  int grid_c = (int)(nunits_c < nsm ? nunits_c : nsm);
  if (grid_c > C_MAXGRID) grid_c = C_MAXGRID;
  e = cudaFuncSetAttribute(k_gphi8, cudaFuncAttributeMaxDynamicSharedMemorySize, C_SMEM);
  if (e != cudaSuccess) return e;
  k_gphi8<<<(unsigned)grid_c, C_NT, C_SMEM, s>>>(mx, mu, T, C, ncb_c, nunits_c, gphi, gpart, st,
                                                 wl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_gphi8_fin<<<(unsigned)(N * ncb_c), 256, 0, s>>>(C, ncb_c, ntt, nunits_c, grid_c, gpart,
                                                     gphi);
  return cudaGetLastError();
}

}  // namespace mhc
