// k_apply16_tc.cu -- second phase of the mHC backward for n = 16 streams with
// bf16 activations.  From the coefficient records of the n = 16 mapping
// (H_res, H_pre, H_post, kappa and u = alpha dz / r, fp32) it writes
//
//   grad_x[j][c]   = (phi u)[jC+c] + sum_i H_res[i][j] G[i][c] + H_pre[j] g[c] - kappa x[j][c]
//   grad_f_out[c]  = sum_i H_post[i] G[i][c]
//   grad_phi[k][m] = sum_t x_t[k] u_t[m]
//
// (reverse mode of the update equation of the chatgpz.de explainer and of the
// RMS-normalised projection; reportify.cn [19]-[21]), with the two contractions
// on the tensor cores:
//
//   k_urec16  u as bf16 rows [u_hi (288) | 0 (32) | u_lo (288) | 0 (32)]
//   k_phiu16  phi u: D[128 tok x 256 ch] = u_hi . phi_hi + u_lo . phi_hi over the
//             288 logits (tcgen05), one persistent CTA per SM walking
//             (token tile, stream, 256-channel block) items through a three-stage
//             ring; phi_hi comes from the tiled, pre-swizzled phi^T copy the
//             projection reads; two TMEM accumulators, so one item's epilogue
//             overlaps the next item's MMAs; fp32 scratch [T][16][C]
//   k_gx16    grad_x and grad_f_out from that scratch (CUDA cores, 8-byte vectors,
//             paired fp32 FMAs)
//   k_gphi16  grad_phi for 128 rows of phi: D[128 x 288] += X^T (u_hi + u_lo)
//             over every token tile (tcgen05), the (block, tile) units split
//             evenly over persistent CTAs; k_gphi16_fin adds the parts of
//             blocks that two or more CTAs share
//
// grad_b and grad_alpha come from the mapping's partial sums (k_wide.cu).  All
// sums run in a fixed order, so repeated calls give identical bits.  Waits are
// bounded; a wait that gives up records MHC_ERR_TIMEOUT, and the kernel drains
// what it issued, frees TMEM and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

namespace ap16 {
constexpr int N = 16;
constexpr int M = N * N + 2 * N;        // 288 logits
constexpr int MP = 320;                 // one half of a U row (288 + zero padding)
constexpr int NU = 2 * MP;              // 640
constexpr int TT = 128;                 // tokens per tile
constexpr int ATOM = 128 * 128;         // [128 rows][64 bf16], 128-byte swizzle: 16 KB
constexpr int CHB = 64;                 // channels per block of the tiled phi^T copy
constexpr int NL = 2 * M;               // rows per block (288 high, 288 low)
constexpr int PROW = CHB * 2;           // 128 bytes
// k_phiu16
constexpr int KB = 256;                 // channels per item (MMA N)
constexpr int NQ = KB / CHB;            // 4 phi blocks per item
constexpr int NB = MP / 64;             // 5 logit blocks of 64 per item
constexpr int PPIECE = 64 * PROW;       // 64 rows of one phi block: 8 KB
constexpr int S_UH = 0, S_UL = ATOM, S_P = 2 * ATOM;
constexpr int A_STAGE = 2 * ATOM + NQ * PPIECE;  // 64 KB
constexpr int A_NS = 3;
constexpr int XT = 36;                  // row stride (floats) of the transpose buffers
constexpr int A_XT_OFF = A_NS * A_STAGE;
constexpr int A_DATA = A_XT_OFF + 4 * 32 * XT * 4;
constexpr int A_SMEM = A_DATA + 1024 + 256;
constexpr int A_NT = 6 * 32;            // TMA, MMA, four epilogue warps
constexpr uint32_t A_TMEM = 512;        // two accumulators of 256 columns
// k_gphi16
constexpr int CB = 128;                 // phi rows (channels of one stream) per CTA
constexpr int G_X = 0;                  // x tile [128 tok][128 ch]: two atoms
constexpr int G_U = 2 * ATOM;           // one U half [128 tok][320]: five atoms
constexpr int G_STAGE = 7 * ATOM;       // 112 KB
constexpr int G_NS = 2;
constexpr int G_DATA = G_NS * G_STAGE;
constexpr int G_SMEM = G_DATA + 1024 + 128;
constexpr int G_NT = 6 * 32;
constexpr uint32_t G_TMEM = 512;
constexpr int G_MAXGRID = 256;          // partial-sum slots are sized for this many CTAs
static_assert(A_SMEM <= 232448 && G_SMEM <= 232448, "shared memory");
static_assert(A_STAGE % 1024 == 0 && A_XT_OFF % 1024 == 0, "stage alignment");
}  // namespace ap16

namespace {
// u (fp32, in the coefficient records) -> the bf16 U rows
__global__ void k_urec16(int64_t T, const float* __restrict__ coef,
                         __nv_bfloat16* __restrict__ urec) {
  using namespace ap16;
  using CF = Coef<N>;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // t * MP + m
  if (idx >= T * MP) return;
  const int64_t t = idx / MP;
  const int m = (int)(idx % MP);
  const float u = m < M ? __ldg(coef + t * CF::SIZE + CF::U + m) : 0.0f;
  const __nv_bfloat16 hi = __float2bfloat16_rn(u);
  urec[t * NU + m] = hi;
  urec[t * NU + MP + m] = __float2bfloat16_rn(u - __bfloat162float(hi));
}
}  // namespace

// ------------------------------------------------------------------ phi u
__global__ void __launch_bounds__(ap16::A_NT, 1) k_phiu16(
    const __grid_constant__ CUtensorMap tm_u, const __nv_bfloat16* __restrict__ phi_t, int64_t T,
    int64_t C, int ncb, int64_t nitems, float* __restrict__ phiu, int* status,
    uint64_t wait_ns) {
  using namespace ap16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  // full[3] empty[3] dfull[2] dempty[2] fin
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + A_DATA);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + A_NS + s); };
  auto dfull = [&](int d) { return tc::smem_u32(bars + 2 * A_NS + d); };
  auto dempty = [&](int d) { return tc::smem_u32(bars + 2 * A_NS + 2 + d); };
  const uint32_t fin_bar = tc::smem_u32(bars + 10);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nblk = (C + CHB - 1) / CHB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_NS; ++s) {
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
  if (warp == 0 && lane == 0) tc::tma_prefetch_desc(&tm_u);
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), A_TMEM);
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
  auto decode = [&](int64_t it, int64_t& t0, int& j, int& cb) {
    const int64_t per_tile = (int64_t)N * ncb;
    t0 = (it / per_tile) * TT;
    const int rem = (int)(it % per_tile);
    j = rem / ncb;
    cb = rem % ncb;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      const uint64_t pol = tc::policy_evict_last();  // U and phi are read by many CTAs
      int64_t g = 0;
      bool stop = false;
      for (int64_t it = blockIdx.x; it < nitems && !stop; it += gridDim.x) {
        int64_t t0;
        int j, cb;
        decode(it, t0, j, cb);
        const int64_t q0 = (int64_t)cb * NQ;
        const int nq = (int)(nblk - q0 < NQ ? nblk - q0 : NQ);
        for (int b = 0; b < NB; ++b, ++g) {
          const int s = (int)(g % A_NS);
          if (g >= A_NS &&
              !tc::mbar_wait(empty(s), ((uint32_t)(g / A_NS) & 1u) ^ 1u, abort_flag, wait_ns)) {
            give_up();
            stop = true;
            break;
          }
          const uint32_t st = tc::smem_u32(smem + s * A_STAGE);
          tc::mbar_arrive_expect_tx(full(s), (uint32_t)(2 * ATOM + nq * PPIECE));
          tc::tma_load_2d(st + S_UH, &tm_u, full(s), 64 * b, (int)t0, pol);
          tc::tma_load_2d(st + S_UL, &tm_u, full(s), MP + 64 * b, (int)t0, pol);
          for (int q = 0; q < nq; ++q)
            tc::bulk_load(st + S_P + q * PPIECE,
                          phi_t + (((q0 + q) * N + j) * NL + 64 * b) * (int64_t)CHB, PPIECE,
                          full(s), pol);
        }
      }
      // every copy issued here has landed before the CTA can exit
      for (int64_t k = (g > A_NS ? g - A_NS : 0); k < g; ++k)
        tc::mbar_wait(full((int)(k % A_NS)), (uint32_t)(k / A_NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      // D[tok][ch] += U[tok][m'] PHI[m'][ch]: A = U (K-major), B = the phi rows
      // (MN-major, 64-channel atoms PPIECE bytes apart, 8-row groups 1024 apart)
      constexpr uint32_t idesc = tc::idesc_bf16(TT, KB, false, true);
      bool any = false;
      int64_t g = 0;
      int li = 0;
      for (int64_t it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
        const int d = li & 1;
        if (li >= 2 &&
            !tc::mbar_wait(dempty(d), ((uint32_t)(li >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        bool ok = true;
        for (int b = 0; b < NB; ++b, ++g) {
          const int s = (int)(g % A_NS);
          if (!tc::mbar_wait(full(s), (uint32_t)(g / A_NS) & 1u, abort_flag, wait_ns)) {
            give_up();
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t st = tc::smem_u32(smem + s * A_STAGE);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ah = tc::smem_desc(st + S_UH + 32 * k, 16, 1024, tc::SWZ_128B);
            const uint64_t al = tc::smem_desc(st + S_UL + 32 * k, 16, 1024, tc::SWZ_128B);
            const uint64_t bd = tc::smem_desc(st + S_P + 2048 * k, PPIECE, 1024, tc::SWZ_128B);
            const uint32_t dt = tmem + (uint32_t)(d * KB);
            tc::mma_bf16(dt, ah, bd, idesc, (b | k) != 0 ? 1u : 0u);
            tc::mma_bf16(dt, al, bd, idesc, 1u);
          }
          any = true;
          tc::mma_commit(empty(s));
        }
        if (!ok) break;
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
    // warp w reads TMEM lanes 32(w % 4).. (tokens) and turns each 32 x 32 block
    // around in shared memory, so that 8 lanes store one token's 128 bytes
    const int qd = warp & 3;
    float* xt = reinterpret_cast<float*>(smem + A_XT_OFF) + qd * 32 * XT;
    const int rr = lane >> 3, cq = lane & 7;
    int li = 0;
    for (int64_t it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
      const int d = li & 1;
      bool ok = tc::mbar_wait(dfull(d), (uint32_t)(li >> 1) & 1u, abort_flag, wait_ns);
      if (!ok && !*abort_flag) give_up();
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc::tc_fence_after();
      int64_t t0;
      int j, cb;
      decode(it, t0, j, cb);
      const int64_t c0 = (int64_t)cb * KB;
      const uint32_t lb = tmem + (uint32_t)(d * KB) + ((uint32_t)(32 * qd) << 16);
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
        const int64_t c = c0 + 32 * q + 4 * cq;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + rr;
          const int64_t t = t0 + 32 * qd + r;
          const float4 val = *reinterpret_cast<const float4*>(xt + r * XT + 4 * cq);
          if (t < T && c < C) __stcg(reinterpret_cast<float4*>(phiu + (t * N + j) * C + c), val);
        }
        __syncwarp();
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
    tc::tmem_dealloc(tmem, A_TMEM);
  }
}

// ------------------------------------------------------- grad_x, grad_f_out
// One CTA visit per token: its coefficient record in shared memory, its
// threads over 4-channel vectors of all sixteen streams.  A thread keeps the
// sixteen output streams' sums as fp32 pairs, starting from phi u, and walks
// the input streams i once: H_res row i comes as four 16-byte shared-memory
// reads and each grad_x_next vector is widened once.  Per element the terms
// are added in the order phi u, H_pre g, H_res[0..15] G, -kappa x.
__global__ void __launch_bounds__(128, 4) k_gx16(int64_t T, int64_t C,
                                              const __nv_bfloat16* __restrict__ x,
                                              const __nv_bfloat16* __restrict__ G,
                                              const __nv_bfloat16* __restrict__ g,
                                              const float* __restrict__ phiu,
                                              const float* __restrict__ coef,
                                              __nv_bfloat16* __restrict__ gx,
                                              __nv_bfloat16* __restrict__ gf) {
  using namespace ap16;
  using CF = Coef<N>;
  static_assert(CF::RES % 4 == 0 && N % 4 == 0, "16-byte rows of H_res");
  __shared__ __align__(16) float hs[CF::SIZE];
  const int tid = threadIdx.x;
  const int64_t nv = C / 4;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    for (int e = tid; e < CF::SIZE; e += blockDim.x) hs[e] = __ldg(coef + t * CF::SIZE + e);
    __syncthreads();
    const float nk = -hs[CF::KAPPA];
    for (int64_t v = tid; v < nv; v += blockDim.x) {
      const int64_t c = v * 4;
      uint64_t acc[N][2];
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const ulonglong2 p =
            __ldcs(reinterpret_cast<const ulonglong2*>(phiu + (t * N + j) * C + c));
        acc[j][0] = p.x;
        acc[j][1] = p.y;
      }
      {
        const uint2 gw = __ldcs(reinterpret_cast<const uint2*>(g + t * C + c));
        const uint64_t gp[2] = {bf2_to_f2(gw.x), bf2_to_f2(gw.y)};
#pragma unroll
        for (int j = 0; j < N; ++j) {
          const uint64_t h = f2pack(hs[CF::PRE + j], hs[CF::PRE + j]);
          acc[j][0] = f2fma(h, gp[0], acc[j][0]);
          acc[j][1] = f2fma(h, gp[1], acc[j][1]);
        }
      }
      uint64_t gfa[2] = {0, 0};
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const uint2 w = __ldcs(reinterpret_cast<const uint2*>(G + (t * N + i) * C + c));
        const uint64_t Gp[2] = {bf2_to_f2(w.x), bf2_to_f2(w.y)};
        const uint64_t hpo = f2pack(hs[CF::POST + i], hs[CF::POST + i]);
        gfa[0] = f2fma(hpo, Gp[0], gfa[0]);
        gfa[1] = f2fma(hpo, Gp[1], gfa[1]);
#pragma unroll
        for (int q4 = 0; q4 < N / 4; ++q4) {
          const float4 h = *reinterpret_cast<const float4*>(hs + CF::RES + N * i + 4 * q4);
          const float hr[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t hh = f2pack(hr[k], hr[k]);
            acc[4 * q4 + k][0] = f2fma(hh, Gp[0], acc[4 * q4 + k][0]);
            acc[4 * q4 + k][1] = f2fma(hh, Gp[1], acc[4 * q4 + k][1]);
          }
        }
      }
      if (gf != nullptr)
        __stcs(reinterpret_cast<uint2*>(gf + t * C + c),
               make_uint2(f2_to_bf2(gfa[0]), f2_to_bf2(gfa[1])));
      const uint64_t kk = f2pack(nk, nk);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const uint2 xw = __ldcs(reinterpret_cast<const uint2*>(x + (t * N + j) * C + c));
        __stcs(reinterpret_cast<uint2*>(gx + (t * N + j) * C + c),
               make_uint2(f2_to_bf2(f2fma(kk, bf2_to_f2(xw.x), acc[j][0])),
                          f2_to_bf2(f2fma(kk, bf2_to_f2(xw.y), acc[j][1]))));
      }
    }
  }
}

// grad_phi for 128 rows of phi (128 channels of one stream) per (block, token
// tile) unit: D[128 x 288] += X^T (u_hi + u_lo), the u_hi half of a tile then
// its u_lo half through the stage ring.  The units, block-major, are split
// evenly over persistent CTAs (a contiguous range each); a range cuts into one
// segment per block it touches.  D (288 TMEM columns) is single: before a
// segment's first MMA the MMA warp waits for the previous segment's epilogue.
// A segment that covers its whole block writes grad_phi; the first and last
// segments of a range can be parts of a block and write the CTA's partial
// slots 0 and 1, which k_gphi16_fin adds in CTA order.
__global__ void __launch_bounds__(ap16::G_NT, 1) k_gphi16(const __grid_constant__ CUtensorMap tm_x,
                                                         const __grid_constant__ CUtensorMap tm_u,
                                                         int64_t T, int64_t C, int ncb,
                                                         int64_t nunits,
                                                         float* __restrict__ grad_phi,
                                                         float* __restrict__ partial,
                                                         int* status, uint64_t wait_ns) {
  using namespace ap16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  // full[2] empty[2] dfull dempty fin
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G_DATA);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * G_NS + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + G_NS + s); };
  const uint32_t dfull = tc::smem_u32(bars + 2 * G_NS);
  const uint32_t dempty = tc::smem_u32(bars + 2 * G_NS + 1);
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * G_NS + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t ntt = (T + TT - 1) / TT;
  const int64_t lo = (int64_t)blockIdx.x * nunits / gridDim.x;
  const int64_t hi = ((int64_t)blockIdx.x + 1) * nunits / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G_NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    tc::mbar_init(dfull, 1);
    tc::mbar_init(dempty, 4);  // the four epilogue warps
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), G_TMEM);
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
    const uint64_t pol_x = tc::policy_evict_normal(), pol_u = tc::policy_evict_last();
    int64_t g = 0;
    bool stop = false;
    for (int64_t u = lo; u < hi && !stop; ++u) {
      const int64_t blk = u / ntt, tile = u % ntt;
      const int j = (int)(blk / ncb), c0 = (int)(blk % ncb) * CB;
      for (int hh = 0; hh < 2; ++hh, ++g) {  // the u_hi half, then the u_lo half
        const int s = (int)(g % G_NS);
        if (g >= G_NS &&
            !tc::mbar_wait(empty(s), ((uint32_t)(g / G_NS) & 1u) ^ 1u, abort_flag, wait_ns)) {
          give_up();
          stop = true;
          break;
        }
        const uint32_t base = tc::smem_u32(smem + s * G_STAGE);
        tc::mbar_arrive_expect_tx(full(s), (uint32_t)G_STAGE);
        for (int a = 0; a < 2; ++a)
          tc::tma_load_3d(base + G_X + a * ATOM, &tm_x, full(s), c0 + 64 * a, j,
                          (int)(tile * TT), pol_x);
        for (int a = 0; a < 5; ++a)
          tc::tma_load_2d(base + G_U + a * ATOM, &tm_u, full(s), hh * MP + 64 * a,
                          (int)(tile * TT), pol_u);
      }
    }
    for (int64_t q = (g > G_NS ? g - G_NS : 0); q < g; ++q)
      tc::mbar_wait(full((int)(q % G_NS)), (uint32_t)(q / G_NS) & 1u, nullptr, tc::kDrainWaitNs);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    // D[k][m] += sum over 16 tokens of X[tok][k] U[tok][m]: A = X^T (MN-major,
    // two 64-channel atoms), B = U (MN-major): logit columns 0..127 (N = 128) and
    // 128..287 (N = 160) of the half, into D columns 0..127 and 128..287
    constexpr uint32_t id1 = tc::idesc_bf16(CB, 128, true, true);
    constexpr uint32_t id2 = tc::idesc_bf16(CB, 160, true, true);
    bool any = false, stop = false;
    int seg = 0;
    int64_t g = 0;
    for (int64_t u = lo; u < hi && !stop; ++u) {
      const int64_t tile = u % ntt;
      const bool first = u == lo || tile == 0, last = u == hi - 1 || tile == ntt - 1;
      if (first && seg >= 1 &&
          !tc::mbar_wait(dempty, ((uint32_t)(seg - 1) & 1u), abort_flag, wait_ns)) {
        give_up();
        break;
      }
      for (int hh = 0; hh < 2; ++hh, ++g) {
        const int s = (int)(g % G_NS);
        if (!tc::mbar_wait(full(s), (uint32_t)(g / G_NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          stop = true;
          break;
        }
        tc::tc_fence_after();
        const uint32_t base = tc::smem_u32(smem + s * G_STAGE);
#pragma unroll
        for (int k = 0; k < TT / 16; ++k) {
          const uint64_t da = tc::smem_desc(base + G_X + k * 2048, ATOM, 1024, tc::SWZ_128B);
          const uint64_t b1 = tc::smem_desc(base + G_U + k * 2048, ATOM, 1024, tc::SWZ_128B);
          const uint64_t b2 =
              tc::smem_desc(base + G_U + 2 * ATOM + k * 2048, ATOM, 1024, tc::SWZ_128B);
          const uint32_t acc = (first && hh == 0 && k == 0) ? 0u : 1u;
          tc::mma_bf16(tmem, da, b1, id1, acc);
          tc::mma_bf16(tmem + 128, da, b2, id2, acc);
        }
        any = true;
        tc::mma_commit(empty(s));
      }
      if (stop) break;
      if (last) {
        tc::mma_commit(dfull);
        ++seg;
      }
    }
    if (any) {
      tc::mma_commit(fin_bar);
      tc::mbar_wait(fin_bar, 0, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp >= 2) {
    // ----- epilogue: warp w holds phi rows (channels) 32(w % 4).. of the segment's block
    const int qd = warp & 3;
    const int64_t b0 = lo / ntt, b1 = hi > lo ? (hi - 1) / ntt : b0 - 1;
    bool ok = true;
    for (int64_t blk = b0; blk <= b1 && ok; ++blk) {
      const int si = (int)(blk - b0);
      bool okw = tc::mbar_wait(dfull, (uint32_t)si & 1u, abort_flag, wait_ns);
      if (!okw && !*abort_flag) give_up();
      ok = __all_sync(0xffffffffu, okw);
      if (!ok) break;
      tc::tc_fence_after();
      const int64_t s_lo = blk * ntt > lo ? blk * ntt : lo;
      const int64_t s_hi = (blk + 1) * ntt < hi ? (blk + 1) * ntt : hi;
      const bool whole = s_lo == blk * ntt && s_hi == (blk + 1) * ntt;
      const int j = (int)(blk / ncb);
      const int64_t c = (blk % ncb) * CB + 32 * qd + lane;
      float* dst = whole ? grad_phi + ((int64_t)j * C + c) * M
                         : partial + (((int64_t)blockIdx.x * 2 + (si == 0 ? 0 : 1)) * CB +
                                      32 * qd + lane) * M;
      const uint32_t lb = tmem + ((uint32_t)(32 * qd) << 16);
#pragma unroll 1
      for (int b16 = 0; b16 < M / 16; ++b16) {
        float v[16];
        tc::tmem_ld16(lb + 16 * b16, v);
        tc::tmem_ld_wait();
        if (c < C) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(dst + 16 * b16 + e) =
                make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(dempty);
    }
  }
  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, G_TMEM);
  }
}

// grad_phi rows of the blocks that several CTAs share: the CTAs' partial
// slots added in CTA order.  One CTA per block (it returns at once when one CTA
// covered the block), its threads along the rows' 16-byte pieces.
__global__ void __launch_bounds__(256) k_gphi16_fin(int64_t C, int ncb, int64_t ntt, int64_t nunits,
                                            int grid, const float* __restrict__ partial,
                                            float* __restrict__ grad_phi) {
  using namespace ap16;
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
size_t apply16_urec_bytes(int64_t T) { return (size_t)T * ap16::NU * 2; }
size_t apply16_gphi_part_bytes() { return (size_t)ap16::G_MAXGRID * 2 * ap16::CB * ap16::M * 4; }

cudaError_t apply16_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_t,
                                const void* G, const void* g, const float* coef,
                                const float* part, int nparts, void* urec, float* phiu, void* gx,
                                void* gf, float* gphi, float* gb, float* ga, int ag, int* st,
                                int64_t wait_ns, cudaStream_t s) {
  using namespace ap16;
  const uint64_t wl = tc::wait_limit(wait_ns);
  k_urec16<<<(unsigned)((T * MP + 255) / 256), 256, 0, s>>>(T, coef, (__nv_bfloat16*)urec);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mu, mx;
  const uint64_t du[2] = {(uint64_t)NU, (uint64_t)T};
  const uint64_t su[1] = {(uint64_t)NU * 2};
  const uint32_t bu[2] = {64, TT};
  e = make_tmap_bf16(&mu, urec, 2, du, su, bu, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {64, 1, TT};
  e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;

  const int64_t ntt = (T + TT - 1) / TT;
  const int ncb_a = (int)((C + KB - 1) / KB);
  const int64_t nitems = ntt * N * ncb_a;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid_a = nitems < nsm ? nitems : nsm;
  e = cudaFuncSetAttribute(k_phiu16, cudaFuncAttributeMaxDynamicSharedMemorySize, A_SMEM);
  if (e != cudaSuccess) return e;
  k_phiu16<<<(unsigned)grid_a, A_NT, A_SMEM, s>>>(mu, (const __nv_bfloat16*)phi_t, T, C, ncb_a,
                                                  nitems, phiu, st, wl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const int64_t grid_b = T < 148 * 8 ? T : 148 * 8;
  k_gx16<<<(unsigned)grid_b, 128, 0, s>>>(T, C, (const __nv_bfloat16*)x, (const __nv_bfloat16*)G,
                                          (const __nv_bfloat16*)g, phiu, coef,
                                          (__nv_bfloat16*)gx, (__nv_bfloat16*)gf);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const int ncb_c = (int)((C + CB - 1) / CB);
  const int64_t nunits_c = (int64_t)N * ncb_c * ntt;
  int grid_c = (int)(nunits_c < nsm ? nunits_c : nsm);
  if (grid_c > G_MAXGRID) grid_c = G_MAXGRID;
  // the partial slots reuse the phi u scratch (k_gx16 has read it by now)
  float* gpart = phiu;
  e = cudaFuncSetAttribute(k_gphi16, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
  if (e != cudaSuccess) return e;
  k_gphi16<<<(unsigned)grid_c, G_NT, G_SMEM, s>>>(mx, mu, T, C, ncb_c, nunits_c, gphi, gpart, st,
                                                  wl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_gphi16_fin<<<(unsigned)(N * ncb_c), 256, 0, s>>>(C, ncb_c, ntt, nunits_c, grid_c, gpart,
                                                      gphi);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return wide_bias_dispatch(part, nparts, gb, ga, ag, s);
}

}  // namespace mhc
