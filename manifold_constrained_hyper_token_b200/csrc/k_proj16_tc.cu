// k_proj16_tc.cu -- the logit projection of a wide stream buffer (n = 16, bf16
// activations) on the 5th-generation tensor cores: for every token
//
//   y[m] = sum_k x[k] phi[k][m]   (k = i*C + c over all 16 streams, m < 288)
//   ss   = sum_k x[k]^2
//
// the two C-reductions the mapping needs before its per-token epilogue (the
// RMS-normalised projection of the chatgpz.de explainer, section
// "Systemarbeit und Schulungsaufwand"; reportify.cn [17]-[19]).  The gates,
// Sinkhorn and, in the backward, the C-reductions against the gradients and
// the adjoint stay in k_wide.cu, which reads y and ss from the rows written
// here.
//
// One CTA = 128 tokens (the MMA M).  The k axis streams through a two-stage
// ring in chunks of (one stream i, 64 channels): the x tile [128 x 64] arrives
// by TMA with 128-byte rows and the 128-byte swizzle (the K-major A operand),
// and the matching 576 rows of phi^T -- the 288 logit columns split into a bf16
// high part and a bf16 low part (phi = hi + lo) -- arrive as one 72 KB bulk
// copy of a tiled, pre-swizzled copy of phi^T (the K-major B operand).  Per
// 16-channel K step four MMAs (M = 128, N = 144) add x . phi_hi and x . phi_lo
// for logit columns 0..143 and 144..287 into one fp32 accumulator
// D[128 x 288] in TMEM (columns 0..143 and 256..399), so y carries phi to
// ~16 bits; x is exact in bf16.
// Four CUDA-core warps take the sum of squares from the same x tiles and then
// move D out of TMEM.  Every wait is bounded; on timeout the kernel records
// MHC_ERR_TIMEOUT, drains what it issued, frees TMEM and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

namespace p16 {
constexpr int N = 16;
constexpr int M = N * N + 2 * N;      // 288 logits
constexpr int NL = 2 * M;             // 576 rows of the split phi^T
constexpr int NH = M / 2;             // MMA N: 144 logit columns per MMA
constexpr int TM = 128;               // tokens per CTA (MMA M)
constexpr int CH = 64;                // channels per chunk: 128-byte rows
constexpr int XBOX = TM * CH * 2;     // 16 KB
constexpr int PBLK = NL * CH * 2;     // 72 KB
constexpr int STAGE = XBOX + PBLK;    // 88 KB
constexpr int NS = 2;
constexpr int DATA = NS * STAGE;
constexpr int SMEM = DATA + 1024 + 256;
constexpr int NW = 6;                 // TMA, MMA, four math warps
constexpr int NT = NW * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D1_COL = 256;      // TMEM column of logit columns 144..287
static_assert(STAGE % 1024 == 0 && XBOX % 1024 == 0, "stage alignment");
static_assert(SMEM <= 232448, "shared memory");
}  // namespace p16

namespace {

// phi [K][288] fp32 (k = i*C + c) -> the tiled bf16 split of phi^T: block
// (chunk q of 64 channels, stream i) holds the 576 rows m (0..287 the high
// parts, 288..575 the bf16 rounding of the remainder) of 64 channels, 128 bytes
// per row, with the row's eight 16-byte pieces permuted by the 128-byte swizzle
// (piece p stored at p ^ (m & 7)).  Blocks run q-major, i-minor: the order the
// projection streams them.  Channels c >= C of the last chunk are zero.
__global__ void k_phi_split16(int64_t C, int64_t ncp, const float* __restrict__ phi,
                              __nv_bfloat16* __restrict__ out) {
  using namespace p16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // i * ncp + c
  if (idx >= (int64_t)N * ncp) return;
  const int64_t i = idx / ncp, c = idx % ncp;
  const int64_t q = c / CH;
  const int ci = (int)(c % CH), p = ci >> 3, e = ci & 7;
  __nv_bfloat16* blk = out + (q * N + i) * (int64_t)(NL * CH);
#pragma unroll 4
  for (int m = 0; m < M; ++m) {
    const float v = c < C ? __ldg(phi + (i * C + c) * M + m) : 0.0f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    const int m2 = M + m;
    blk[m * CH + ((p ^ (m & 7)) << 3) + e] = hi;
    blk[m2 * CH + ((p ^ (m2 & 7)) << 3) + e] = lo;
  }
}

}  // namespace

// rows: [T][ostride] fp32; the kernel writes y at [0, 288) and ss at [576].
__global__ void __launch_bounds__(p16::NT, 1) k_proj16_tc(
    const __grid_constant__ CUtensorMap tm_x, const __nv_bfloat16* __restrict__ phi_t, int64_t T,
    int64_t C, float* __restrict__ rows, int64_t ostride, int* status, uint64_t wait_ns) {
  using namespace p16;
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
  const int64_t t0 = (int64_t)blockIdx.x * TM;
  const int nq = (int)((C + CH - 1) / CH);
  const int nch = nq * N;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1 + 4);  // the MMA commit + every math warp
    }
    tc::mbar_init(done_bar, 1);
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) tc::tma_prefetch_desc(&tm_x);
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
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
      const uint64_t pol_stream = tc::policy_evict_first();
      const uint64_t pol_keep = tc::policy_evict_last();
      int issued = 0;
      for (int cc = 0; cc < nch; ++cc) {
        const int s = cc % NS;
        if (cc >= NS && !tc::mbar_wait(empty(s), ((uint32_t)(cc / NS) & 1u) ^ 1u, abort_flag,
                                       wait_ns)) {
          give_up();
          break;
        }
        const uint32_t base = tc::smem_u32(smem + s * STAGE);
        tc::mbar_arrive_expect_tx(full(s), STAGE);
        const int q = cc / N, i = cc % N;
        tc::tma_load_3d(base, &tm_x, full(s), q * CH, i, (int)t0, pol_stream);
        tc::bulk_load(base + XBOX, phi_t + (int64_t)cc * (NL * CH), PBLK, full(s), pol_keep);
        ++issued;
      }
      // every copy issued here has landed before the CTA can exit
      for (int cc = (issued > NS ? issued - NS : 0); cc < issued; ++cc)
        tc::mbar_wait(full(cc % NS), (uint32_t)(cc / NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(TM, NH);
      bool any = false;
      for (int cc = 0; cc < nch; ++cc) {
        const int s = cc % NS;
        if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t xb = tc::smem_u32(smem + s * STAGE);
        const uint32_t pb = xb + XBOX;
#pragma unroll
        for (int k = 0; k < CH / 16; ++k) {
          const uint64_t a = tc::smem_desc(xb + 32 * k, 16, 1024, tc::SWZ_128B);
#pragma unroll
          for (int part = 0; part < 4; ++part) {  // (hi, cols 0..143) (hi, 144..) (lo, 0..) (lo, 144..)
            const int half = part & 1;
            const uint64_t b =
                tc::smem_desc(pb + (uint32_t)(part * NH * 128) + 32 * k, 16, 1024, tc::SWZ_128B);
            tc::mma_bf16(tmem + (half ? D1_COL : 0u), a, b, idesc,
                         (cc | k | (part >> 1)) != 0 ? 1u : 0u);
          }
        }
        any = true;
        tc::mma_commit(empty(s));
      }
      if (!*abort_flag) tc::mma_commit(done_bar);
      // every MMA issued here has finished before TMEM is freed
      if (any) {
        tc::mma_commit(fin_bar);
        tc::mbar_wait(fin_bar, 0, nullptr, tc::kDrainWaitNs);
      }
    }
  } else {
    // ------------------------------------------- sum of squares, then the rows
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int tok = 32 * q + lane;     // row of the x tile
    float ss = 0.0f;
    for (int cc = 0; cc < nch; ++cc) {
      const int s = cc % NS;
      if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
        give_up();
        break;
      }
      const uint8_t* row = smem + s * STAGE + tok * 128;
#pragma unroll
      for (int p = 0; p < 8; ++p) {  // the row's 16-byte pieces in channel order
        const uint4 w = *reinterpret_cast<const uint4*>(row + ((p ^ (tok & 7)) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float a = __uint_as_float(ww[h] << 16), b = __uint_as_float(ww[h] & 0xffff0000u);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(empty(s));
    }
    bool ok = !*abort_flag && tc::mbar_wait(done_bar, 0, abort_flag, wait_ns);
    if (!ok && !*abort_flag) give_up();
    ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
    if (ok) {
      tc::tc_fence_after();
      const int64_t t = t0 + tok;
      float* out = rows + t * ostride;
      const uint32_t lb = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int b16 = 0; b16 < M / 16; ++b16) {
        float v[16];
        const int h = b16 >= NH / 16;  // logit columns 144.. sit at TMEM column D1_COL
        tc::tmem_ld16(lb + (h ? D1_COL + 16 * (b16 - NH / 16) : 16 * b16), v);
        tc::tmem_ld_wait();
        if (t < T) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(out + 16 * b16 + e) =
                make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      if (t < T) out[2 * M] = ss;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

size_t proj16_phi_bytes(int64_t C) {
  const int64_t nq = (C + p16::CH - 1) / p16::CH;
  return (size_t)nq * p16::N * p16::PBLK;
}

cudaError_t proj16_dispatch(int64_t T, int64_t C, const void* x, const float* phi, void* phi_t,
                            float* rows, int64_t ostride, int* st, int64_t wait_ns,
                            cudaStream_t s) {
  using namespace p16;
  const int64_t ncp = (C + CH - 1) / CH * CH;
  k_phi_split16<<<(unsigned)((N * ncp + 255) / 256), 256, 0, s>>>(C, ncp, phi,
                                                                   (__nv_bfloat16*)phi_t);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mx;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {CH, 1, TM};
  e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_proj16_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  k_proj16_tc<<<(unsigned)((T + TM - 1) / TM), NT, SMEM, s>>>(
      mx, (const __nv_bfloat16*)phi_t, T, C, rows, ostride, st, tc::wait_limit(wait_ns));
  return cudaGetLastError();
}

}  // namespace mhc
