// k_map_tc.cu -- per-token mapping on the 5th-generation tensor cores
// (bf16 activations, n = 4): the logit projection y = x . phi runs as
// tcgen05.mma (bf16 operands, fp32 accumulation in TMEM) while the CUDA cores
// take the sum of squares (and, for the backward, the C-reductions) from the
// same shared-memory tiles.  Sources: the fused RMSNorm / projection / gating
// operator of the chatgpz.de explainer (section "Systemarbeit und
// Schulungsaufwand") and reportify.cn [17]-[19], [21] (RMS applied after the
// projection, Sinkhorn and its custom backward in the same operator,
// recompute in the backward).
//
// One CTA = 128 tokens (the MMA M).  The token's n*C inputs stream through a
// TMA ring in chunks of 64 channels x 4 streams in the forward and split
// backward modes (128-byte rows and swizzle, two stages) and of 32 channels x 4
// streams in the full backward (64-byte rows; a TMA row piece narrower than 64
// bytes caps an SM's streaming rate): per stream an x tile [128 x CH] (the MMA A operand,
// K-major) and the matching rows of phi^T as a [48 x CH] B operand, whose 48
// rows are the
// 24 logit columns split into a bf16 high part and a bf16 low part
// (phi = hi + lo), so y = D[:, m] + D[:, 24 + m] carries phi to ~16 bits.
// x itself is bf16, so the products are exact and only the fp32
// accumulation order differs from the oracle.
//
// Split over channels: when one CTA per 128-token tile would leave SMs idle,
// the tile's chunks are cut into kp contiguous parts, one CTA each.  A part
// publishes its per-token sums (sum of squares, projection, C-reductions) as a
// 52-float record; the tile's last part to finish (an atomic count) adds the
// kp records in part order and runs the epilogue -- a fixed order, so repeated
// calls give identical bits.
//
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs, warps
// 2..9 (two per TMEM lane quarter, one per channel half) reduce the sum of
// squares -- and in the backward the 24 C-reductions <G_i, x_j>, <g, x_i>,
// <G_i, f> -- from the same stages, then run the per-token epilogue (gates,
// Sinkhorn, adjoint) with one thread per token; warp 10 stores x_next in the
// fused post-merge mode.  Every wait is bounded; on
// timeout the kernel records MHC_ERR_TIMEOUT, drains what it issued, frees
// TMEM and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

namespace tcmap {
constexpr int N = 4;
constexpr int M = N * N + 2 * N;     // 24 logits
constexpr int TM = 128;              // tokens per CTA (MMA M)
constexpr int NL = 48;               // MMA N: 24 high + 24 low logit columns
constexpr int NWARPS = 11;           // TMA, MMA, 8 math warps, TMA stores (MAP_POSTFWD)
constexpr int STORE_WARP = 10;
constexpr int NT = NWARPS * 32;
constexpr uint32_t TMEM_COLS = 64;
constexpr int KREC = 52;             // floats per part record: y[24] | ss | dots[24] | pad

// MAP_FWD: the forward mapping.  MAP_BWD: the backward's recompute with all
// 24 C-reductions.  MAP_BWD_SPLIT: the pre half of the backward in training
// order -- the post half already reduced <G_i, x_j> and <G_i, f_out> (the
// `red` input), so only x and grad_h_in are staged.  MAP_POSTFWD: layer l's
// post merge x_next = H_res x + H_post^T f_out fused with layer l+1's
// forward mapping of x_next (the math warps form x_next in the stage, the
// tensor cores project it, a store warp writes it out).
template <int MODE> struct Cfg {
  static constexpr bool FULLB = MODE == MAP_BWD;
  // channels per chunk: the forward modes and the split backward stream
  // 128-byte rows (half the row requests of 64-byte rows; the fused post merge
  // also stores every row it loads), the full backward 64-byte rows (its
  // stages hold four tensors).  Both forward modes use the same chunks, so
  // mhc_post_fused reproduces mhc_post -> mhc_pre bit for bit.
  static constexpr int CH = MODE == MAP_BWD ? 32 : 64;
  static constexpr int ROW = CH * 2;            // bytes per tile row = swizzle span
  static constexpr int XBOX = TM * CH * 2;      // one stream's x tile
  static constexpr int PBOX = NL * CH * 2;      // one stream's phi^T tile
  // pipeline stages (MAP_BWD stages 4 tensors; the 128-byte-row stages are twice as big)
  static constexpr int NS = FULLB || CH == 64 ? 2 : 4;
  static constexpr int X_OFF = 0;
  static constexpr int P_OFF = N * XBOX;
  static constexpr int G_OFF = P_OFF + N * PBOX;                 // grad_x_next tiles (MAP_BWD)
  static constexpr int GG_OFF = FULLB ? G_OFF + N * XBOX : G_OFF;  // grad_h_in tile
  static constexpr int F_OFF = GG_OFF + XBOX;                     // f_out tile (MAP_BWD)
  static constexpr int FN_OFF = G_OFF;                            // f_out tile (MAP_POSTFWD)
  static constexpr int STAGE = MODE == MAP_FWD ? G_OFF
                               : FULLB        ? F_OFF + XBOX
                               : MODE == MAP_BWD_SPLIT ? GG_OFF + XBOX
                                                       : FN_OFF + XBOX;
  static constexpr int DATA = NS * STAGE;
  static constexpr int SMEM = DATA + 1024 /*align*/ + 256 /*barriers, flags*/;
};
}  // namespace tcmap

// phi [K][24] fp32 -> phi^T split [48][K] bf16: rows 0..23 high parts, 24..47
// the bf16 rounding of the remainder.
__global__ void k_phi_split(int64_t K, const float* __restrict__ phi, __nv_bfloat16* __restrict__ out) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
#pragma unroll 4
  for (int m = 0; m < tcmap::M; ++m) {
    const float v = __ldg(phi + k * tcmap::M + m);
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    out[(int64_t)m * K + k] = hi;
    out[(int64_t)(tcmap::M + m) * K + k] = lo;
  }
}

cudaError_t phi_split_dispatch(int64_t K, const float* phi, void* phi_split, cudaStream_t s) {
  k_phi_split<<<(unsigned)((K + 255) / 256), 256, 0, s>>>(K, phi, (__nv_bfloat16*)phi_split);
  return cudaGetLastError();
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Row `tok`, 16-byte chunk `chunk` of a bf16 tile whose rows are ROW bytes
// and stored with the ROW-byte swizzle: 128-byte rows put chunk c at
// c ^ (tok & 7), 64-byte rows at c ^ ((tok >> 1) & 3), 32-byte rows at
// c ^ ((tok >> 2) & 1).
template <int ROW>
__device__ __forceinline__ int sw_off(int tok, int chunk) {
  static_assert(ROW == 32 || ROW == 64 || ROW == 128, "row width");
  const int phys = ROW == 128 ? chunk ^ (tok & 7)
                   : ROW == 64 ? chunk ^ ((tok >> 1) & 3)
                               : chunk ^ ((tok >> 2) & 1);
  return tok * ROW + phys * 16;
}
template <int ROW>
__device__ __forceinline__ uint4 ld_sw(const uint8_t* tile, int tok, int chunk) {
  return *reinterpret_cast<const uint4*>(tile + sw_off<ROW>(tok, chunk));
}
__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(tcmap::NT, 1) k_map_tc(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_phi,
    const __grid_constant__ CUtensorMap tm_G, const __grid_constant__ CUtensorMap tm_g,
    const __grid_constant__ CUtensorMap tm_f, int64_t T, int64_t C, int iters, float eps,
    int ck_period, const float* __restrict__ bias, const float* __restrict__ alpha_p, int ag,
    float* __restrict__ Hpre_o, float* __restrict__ Hpost_o, float* __restrict__ Hres_o,
    __nv_bfloat16* __restrict__ urec_o, float* __restrict__ hrec_o, float* __restrict__ part_o,
    const float* __restrict__ red_in, const float* __restrict__ hpost_in,
    const float* __restrict__ hres_in, int kp, float* __restrict__ kpart, int* __restrict__ kcnt,
    int* status, uint64_t wait_ns) {
  using namespace tcmap;
  using CFG = Cfg<MODE>;
  constexpr bool BWD = MODE == MAP_BWD || MODE == MAP_BWD_SPLIT;
  constexpr bool SPLIT = MODE == MAP_BWD_SPLIT;
  constexpr bool POST = MODE == MAP_POSTFWD;
  constexpr int NS = CFG::NS;
  constexpr int CH = CFG::CH, XBOX = CFG::XBOX, PBOX = CFG::PBOX, ROW = CFG::ROW;
  constexpr tc::Swz SWZ = ROW == 128 ? tc::SWZ_128B : (ROW == 64 ? tc::SWZ_64B : tc::SWZ_32B);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  // full[NS] empty[NS] done fin xready[NS] sdone
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + CFG::DATA);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * NS + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* bcast = reinterpret_cast<volatile int*>(tmem_slot + 2);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + NS + s); };
  const uint32_t done_bar = tc::smem_u32(bars + 2 * NS);
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * NS + 1);
  auto xready = [&](int s) { return tc::smem_u32(bars + 2 * NS + 2 + s); };
  const uint32_t sdone_bar = tc::smem_u32(bars + 3 * NS + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x / kp, part = blockIdx.x % kp;
  const int64_t t0 = (int64_t)tile * TM;
  const int nch_all = (int)((C + CH - 1) / CH);
  const int cbeg = (int)((int64_t)part * nch_all / kp);     // this part's chunks
  const int nch = (int)((int64_t)(part + 1) * nch_all / kp) - cbeg;
  const int64_t K = (int64_t)N * C;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(full(s), 1);
      // the MMA commit + one arrive per math warp; with the post merge fused,
      // the MMA commit + the store warp once its x_next stores read the stage
      tc::mbar_init(empty(s), POST ? 2 : 1 + 8);
      tc::mbar_init(xready(s), 8);  // (MAP_POSTFWD) every math warp wrote x_next
    }
    tc::mbar_init(done_bar, 1);
    tc::mbar_init(fin_bar, 1);
    tc::mbar_init(sdone_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_x);
    tc::tma_prefetch_desc(&tm_phi);
    if constexpr (BWD) tc::tma_prefetch_desc(&tm_g);
    if constexpr (BWD && !SPLIT) {
      tc::tma_prefetch_desc(&tm_G);
      tc::tma_prefetch_desc(&tm_f);
    }
    if constexpr (POST) {
      tc::tma_prefetch_desc(&tm_G);  // x_next (store)
      tc::tma_prefetch_desc(&tm_f);
    }
  }
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
        const uint32_t ph = (uint32_t)(cc / NS) & 1u;
        if (cc >= NS && !tc::mbar_wait(empty(s), ph ^ 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        const uint32_t base = tc::smem_u32(smem + s * CFG::STAGE);
        tc::mbar_arrive_expect_tx(full(s), CFG::STAGE);
        const int c0 = (cbeg + cc) * CH;
        for (int i = 0; i < N; ++i) {
          tc::tma_load_3d(base + CFG::X_OFF + i * XBOX, &tm_x, full(s), c0, i, (int)t0, pol_stream);
          tc::tma_load_3d(base + CFG::P_OFF + i * PBOX, &tm_phi, full(s), c0, i, 0, pol_keep);
          if constexpr (BWD && !SPLIT)
            tc::tma_load_3d(base + CFG::G_OFF + i * XBOX, &tm_G, full(s), c0, i, (int)t0,
                            pol_stream);
        }
        if constexpr (BWD) tc::tma_load_2d(base + CFG::GG_OFF, &tm_g, full(s), c0, (int)t0, pol_stream);
        if constexpr (BWD && !SPLIT)
          tc::tma_load_2d(base + CFG::F_OFF, &tm_f, full(s), c0, (int)t0, pol_stream);
        if constexpr (POST)
          tc::tma_load_2d(base + CFG::FN_OFF, &tm_f, full(s), c0, (int)t0, pol_stream);
        ++issued;
      }
      // drain: the last min(NS, issued) loads may still be landing if a consumer
      // gave up (after a normal run these waits return at once)
      for (int cc = (issued > NS ? issued - NS : 0); cc < issued; ++cc)
        tc::mbar_wait(full(cc % NS), (uint32_t)(cc / NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(TM, NL);
      bool any = false;
      for (int cc = 0; cc < nch; ++cc) {
        const int s = cc % NS;
        const uint32_t ph = (uint32_t)(cc / NS) & 1u;
        // with the post merge fused, the A operand is x_next, written by the math warps
        if (!tc::mbar_wait(POST ? xready(s) : full(s), ph, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t base = tc::smem_u32(smem + s * CFG::STAGE);
#pragma unroll
        for (int i = 0; i < N; ++i) {
#pragma unroll
          for (int kk = 0; kk < CH / 16; ++kk) {
            const uint64_t a = tc::smem_desc(base + CFG::X_OFF + i * XBOX + kk * 32, 16, 8 * ROW, SWZ);
            const uint64_t b = tc::smem_desc(base + CFG::P_OFF + i * PBOX + kk * 32, 16, 8 * ROW, SWZ);
            tc::mma_bf16(tmem, a, b, idesc, (cc | i | kk) != 0 ? 1u : 0u);
          }
        }
        any = true;
        tc::mma_commit(empty(s));
      }
      if (!*abort_flag) tc::mma_commit(done_bar);
      // every MMA issued here has finished before TMEM is freed, also when a
      // consumer gave up after done_bar was committed
      if (any) {
        tc::mma_commit(fin_bar);
        tc::mbar_wait(fin_bar, 0, nullptr, tc::kDrainWaitNs);
      }
    }
  } else if (warp == STORE_WARP) {
    // ------------------------------------------- x_next stores (MAP_POSTFWD)
    if (POST && lane == 0) {
      for (int cc = 0; cc < nch; ++cc) {
        const int s = cc % NS;
        if (!tc::mbar_wait(xready(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        const uint32_t base = tc::smem_u32(smem + s * CFG::STAGE);
#pragma unroll
        for (int i = 0; i < N; ++i)
          tc::tma_store_3d(&tm_G, base + CFG::X_OFF + i * XBOX, (cbeg + cc) * CH, i, (int)t0);
        tc::bulk_commit();
        tc::bulk_wait_read<0>();
        tc::mbar_arrive(empty(s));
      }
      tc::bulk_wait<0>();
      tc::mbar_arrive(sdone_bar);  // every stage read: its memory may be reused
    }
  } else {
    // -------------------------------------------------- CUDA-core reductions
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int h = (warp - 2) >> 2;     // channel half of each chunk
    const int tok = 32 * q + lane;
    float ss = 0.0f;
    // MAP_POSTFWD: this token's layer-l maps (the post merge's coefficients)
    float hr_in[POST ? N * N : 1], hp_in[POST ? N : 1];
    if constexpr (POST) {
      const bool tv = t0 + tok < T;
#pragma unroll
      for (int e = 0; e < N * N; ++e) hr_in[e] = tv ? __ldg(hres_in + (t0 + tok) * N * N + e) : 0.0f;
#pragma unroll
      for (int i = 0; i < N; ++i) hp_in[i] = tv ? __ldg(hpost_in + (t0 + tok) * N + i) : 0.0f;
    }
    float dots[BWD ? M : 1];
#pragma unroll
    for (int m = 0; m < (BWD ? M : 1); ++m) dots[m] = 0.0f;
    for (int cc = 0; cc < nch; ++cc) {
      const int s = cc % NS;
      const uint32_t ph = (uint32_t)(cc / NS) & 1u;
      if (!tc::mbar_wait(full(s), ph, abort_flag, wait_ns)) {
        give_up();
        break;
      }
      uint8_t* st = smem + s * CFG::STAGE;
#pragma unroll
      for (int qq = 0; qq < CH / 16; ++qq) {
        const int chunk = (CH / 16) * h + qq;
        if constexpr (POST) {
          // x_next[i] = sum_j H_res[i][j] x_j + H_post[i] f_out (the k_post order),
          // rounded to bf16 in place; the sum of squares is of the rounded values
          float xv[N][8], fv[8];
#pragma unroll
          for (int i = 0; i < N; ++i) bf16x8_to_f32(ld_sw<ROW>(st + CFG::X_OFF + i * XBOX, tok, chunk), xv[i]);
          bf16x8_to_f32(ld_sw<ROW>(st + CFG::FN_OFF, tok, chunk), fv);
#pragma unroll
          for (int i = 0; i < N; ++i) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float acc = hp_in[i] * fv[e];
#pragma unroll
              for (int j = 0; j < N; ++j) acc = fmaf(hr_in[i * N + j], xv[j][e], acc);
              o[e] = acc;
            }
            const uint4 w = make_uint4(pack_bf2(o[0], o[1]), pack_bf2(o[2], o[3]),
                                       pack_bf2(o[4], o[5]), pack_bf2(o[6], o[7]));
            *reinterpret_cast<uint4*>(st + CFG::X_OFF + i * XBOX + sw_off<ROW>(tok, chunk)) = w;
            float r[8];
            bf16x8_to_f32(w, r);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(r[e], r[e], ss);
          }
          continue;
        }
        float xv[N][8];
#pragma unroll
        for (int i = 0; i < N; ++i) {
          bf16x8_to_f32(ld_sw<ROW>(st + CFG::X_OFF + i * XBOX, tok, chunk), xv[i]);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss = fmaf(xv[i][e], xv[i][e], ss);
        }
        if constexpr (SPLIT) {
          float gv[8];
          bf16x8_to_f32(ld_sw<ROW>(st + CFG::GG_OFF, tok, chunk), gv);
#pragma unroll
          for (int i = 0; i < N; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) dots[N * N + i] = fmaf(gv[e], xv[i][e], dots[N * N + i]);
        } else if constexpr (BWD) {
          float gv[8], fv[8];
          bf16x8_to_f32(ld_sw<ROW>(st + CFG::GG_OFF, tok, chunk), gv);
          bf16x8_to_f32(ld_sw<ROW>(st + CFG::F_OFF, tok, chunk), fv);
#pragma unroll
          for (int i = 0; i < N; ++i) {
            float Gv[8];
            bf16x8_to_f32(ld_sw<ROW>(st + CFG::G_OFF + i * XBOX, tok, chunk), Gv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
#pragma unroll
              for (int j = 0; j < N; ++j) dots[i * N + j] = fmaf(Gv[e], xv[j][e], dots[i * N + j]);
              dots[N * N + i] = fmaf(gv[e], xv[i][e], dots[N * N + i]);
              dots[N * N + N + i] = fmaf(Gv[e], fv[e], dots[N * N + N + i]);
            }
          }
        }
      }
      if constexpr (POST) {
        tc::fence_proxy_async_smem();  // x_next visible to the MMA and the TMA store
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(xready(s));
      } else {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty(s));
      }
    }

    // all MMAs (and so all reads of the stage buffers) finished before the
    // stage memory is reused for the epilogue; with the post merge fused, the
    // x_next stores as well
    bool ok = !*abort_flag && tc::mbar_wait(done_bar, 0, abort_flag, wait_ns);
    if (POST && ok) ok = tc::mbar_wait(sdone_bar, 0, abort_flag, wait_ns);
    if (!ok && !*abort_flag) give_up();
    ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
    float* red_ss = reinterpret_cast<float*>(smem);       // [2][TM]
    float* red_dt = red_ss + 2 * TM;                      // [2][M][TM]
    float* dzs = red_dt + 2 * M * TM;                     // [M + 3][TM]
    float* ck = dzs + (M + 3) * TM;                       // checkpoints [nck][16][TM]
    // every math warp has finished reading its last stages before any of them
    // reuses the stage memory (the MMA finishing does not imply that)
    named_bar(1, 256);
    if (ok) {
      red_ss[h * TM + tok] = ss;
      if constexpr (BWD) {
#pragma unroll
        for (int m = 0; m < M; ++m) red_dt[(h * M + m) * TM + tok] = dots[m];
      }
    }
    named_bar(1, 256);
    // this CTA's sums for its chunks, per token (one thread per token)
    float sst = 0.0f, yr[M], dt[BWD ? M : 1];
    if (ok && h == 0) {
      tc::tc_fence_after();
      float d[NL];
      const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
      float v16[16];
      tc::tmem_ld16(lane_base + 0, v16);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) d[e] = v16[e];
      tc::tmem_ld16(lane_base + 16, v16);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) d[16 + e] = v16[e];
      tc::tmem_ld16(lane_base + 32, v16);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) d[32 + e] = v16[e];
      sst = red_ss[tok] + red_ss[TM + tok];
#pragma unroll
      for (int m = 0; m < M; ++m) yr[m] = d[m] + d[M + m];
      if constexpr (BWD) {
#pragma unroll
        for (int m = 0; m < M; ++m) dt[m] = red_dt[(0 * M + m) * TM + tok] + red_dt[(1 * M + m) * TM + tok];
      }
    }
    bool epi = ok;  // this CTA runs the per-token epilogue
    if (kp > 1) {
      // publish this part's sums and count it; the tile's last part adds the
      // kp records in part order
      if (ok && h == 0) {
        float rec[KREC];
#pragma unroll
        for (int m = 0; m < M; ++m) rec[m] = yr[m];
        rec[M] = sst;
#pragma unroll
        for (int m = 0; m < M; ++m) rec[M + 1 + m] = BWD ? dt[BWD ? m : 0] : 0.0f;
        rec[2 * M + 1] = rec[2 * M + 2] = rec[2 * M + 3] = 0.0f;
        float4* dst = reinterpret_cast<float4*>(kpart + (((int64_t)tile * kp + part) * TM + tok) * KREC);
#pragma unroll
        for (int e = 0; e < KREC / 4; ++e)
          __stcg(dst + e, make_float4(rec[4 * e], rec[4 * e + 1], rec[4 * e + 2], rec[4 * e + 3]));
      }
      __threadfence();
      named_bar(1, 256);
      if (threadIdx.x == 64) *bcast = ok ? atomicAdd(kcnt + tile, 1) : -1;
      named_bar(1, 256);
      epi = ok && *bcast == kp - 1;
      if (epi && h == 0) {
        __threadfence();
        sst = 0.0f;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          yr[m] = 0.0f;
          if constexpr (BWD) dt[m] = 0.0f;
        }
        for (int pp = 0; pp < kp; ++pp) {
          const float4* src =
              reinterpret_cast<const float4*>(kpart + (((int64_t)tile * kp + pp) * TM + tok) * KREC);
          float rec[KREC];
#pragma unroll
          for (int e = 0; e < KREC / 4; ++e) {
            const float4 v = __ldcg(src + e);
            rec[4 * e] = v.x; rec[4 * e + 1] = v.y; rec[4 * e + 2] = v.z; rec[4 * e + 3] = v.w;
          }
#pragma unroll
          for (int m = 0; m < M; ++m) yr[m] += rec[m];
          sst += rec[M];
          if constexpr (BWD) {
#pragma unroll
            for (int m = 0; m < M; ++m) dt[m] += rec[M + 1 + m];
          }
        }
      }
      if (epi && threadIdx.x == 64) kcnt[tile] = 0;  // ready for the next call
    }
    if (epi && h == 0) {
      // ------------------------------------------------- per-token epilogue
      const int64_t t = t0 + tok;
      const float r = sqrtf(sst / (float)K + eps);
      Alpha3 al;
      al.load(alpha_p, ag);
      float y[M], z[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        y[m] = yr[m] / r;
        z[m] = fmaf(al.at<N>(m), y[m], __ldg(bias + m));
      }
      float spre[N], spost[N];
#pragma unroll
      for (int i = 0; i < N; ++i) {
        spre[i] = sigmoidf_(z[i]);
        spost[i] = sigmoidf_(z[N + i]);
      }
      float H[N * N];
#pragma unroll
      for (int e = 0; e < N * N; ++e) H[e] = z[2 * N + e];
      if (t < T) {
        bool bad = !isfinite(r);
#pragma unroll
        for (int m = 0; m < M; ++m) bad |= !isfinite(z[m]);
        if (bad) flag_status(status, MHC_ERR_NONFINITE);
      }
      if constexpr (!BWD) {
        sk_forward<N>(H, iters);
        if (t < T) {
#pragma unroll
          for (int i = 0; i < N; ++i) {
            Hpre_o[t * N + i] = spre[i];
            Hpost_o[t * N + i] = 2.0f * spost[i];
          }
#pragma unroll
          for (int e = 0; e < N * N; e += 4)
            *reinterpret_cast<float4*>(Hres_o + t * N * N + e) =
                make_float4(H[e], H[e + 1], H[e + 2], H[e + 3]);
        }
      } else {
        sk_forward_ckpt<N>(H, iters, ck + tok, TM, ck_period);
        float dA[N * N], dz[M], dzres[N * N];
        // dL/dH_res and dL/dH_post: this CTA's C-reductions, or the post half's
        const float* rt = red_in + (t < T ? t : 0) * (N * N + N);
#pragma unroll
        for (int e = 0; e < N * N; ++e) dA[e] = SPLIT ? (t < T ? __ldg(rt + e) : 0.0f) : dt[e];
        sk_adjoint_ckpt<N>(dA, dzres, iters, ck + tok, TM, ck_period);
#pragma unroll
        for (int i = 0; i < N; ++i) {
          const float dpre = dt[N * N + i];
          const float dpost = SPLIT ? (t < T ? __ldg(rt + N * N + i) : 0.0f) : dt[N * N + N + i];
          dz[i] = dpre * spre[i] * (1.0f - spre[i]);
          dz[N + i] = dpost * 2.0f * spost[i] * (1.0f - spost[i]);
        }
#pragma unroll
        for (int e = 0; e < N * N; ++e) dz[2 * N + e] = dzres[e];
        float dzy[3] = {0.0f, 0.0f, 0.0f};  // dz . y over the pre, post, res logits
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const int grp = m < N ? 0 : (m < 2 * N ? 1 : 2);
          dzy[grp] = fmaf(dz[m], y[m], dzy[grp]);
        }
        const bool live = t < T;
        if (live) {
          float rec[TcRec::H_FLOATS];
#pragma unroll
          for (int e = 0; e < N * N; ++e) rec[TcRec::H_RES + e] = H[e];
#pragma unroll
          for (int i = 0; i < N; ++i) {
            rec[TcRec::H_PRE + i] = spre[i];
            rec[TcRec::H_POST + i] = 2.0f * spost[i];
          }
          rec[TcRec::H_KAPPA] =
              fmaf(al.a[2], dzy[2], fmaf(al.a[1], dzy[1], al.a[0] * dzy[0])) / ((float)K * r * r);
          rec[25] = rec[26] = rec[27] = 0.0f;
          float4* hd = reinterpret_cast<float4*>(hrec_o + t * TcRec::H_FLOATS);
#pragma unroll
          for (int e = 0; e < TcRec::H_FLOATS / 4; ++e)
            hd[e] = make_float4(rec[4 * e], rec[4 * e + 1], rec[4 * e + 2], rec[4 * e + 3]);
          float ar[3];
#pragma unroll
          for (int g = 0; g < 3; ++g) ar[g] = al.a[g] / r;
          uint32_t w[32];
#pragma unroll
          for (int m2 = 0; m2 < 12; ++m2) {
            const int g0 = 2 * m2 < N ? 0 : (2 * m2 < 2 * N ? 1 : 2);
            const int g1 = 2 * m2 + 1 < N ? 0 : (2 * m2 + 1 < 2 * N ? 1 : 2);
            const float u0 = ar[g0] * dz[2 * m2], u1 = ar[g1] * dz[2 * m2 + 1];
            const __nv_bfloat162 hi = __floats2bfloat162_rn(u0, u1);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(u0 - __low2float(hi), u1 - __high2float(hi));
            w[m2] = *reinterpret_cast<const uint32_t*>(&hi);
            w[16 + m2] = *reinterpret_cast<const uint32_t*>(&lo);
          }
#pragma unroll
          for (int m2 = 12; m2 < 16; ++m2) w[m2] = w[16 + m2] = 0u;
          uint4* ud = reinterpret_cast<uint4*>(urec_o + t * TcRec::U_ELEMS);
#pragma unroll
          for (int e = 0; e < 8; ++e) ud[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
#pragma unroll
        for (int m = 0; m < M; ++m) dzs[m * TM + tok] = live ? dz[m] : 0.0f;
#pragma unroll
        for (int g = 0; g < 3; ++g) dzs[(M + g) * TM + tok] = live ? dzy[g] : 0.0f;
      }
    }
    if constexpr (BWD) {
      named_bar(1, 256);
      if (epi && h == 0 && q == 0 && lane < M + 3) {
        // this tile's share of grad_b and the three grad_alpha sums, in token order
        float a = 0.0f;
        for (int k = 0; k < TM; ++k) a += dzs[lane * TM + k];
        part_o[(int64_t)tile * Coef<N>::DZ_SIZE + lane] = a;
      }
    }
  }

  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
static cudaError_t encode_maps(int mode, int64_t T, int64_t C, const void* x, const void* phiT,
                               const void* G, const void* g, const void* f, CUtensorMap* mx,
                               CUtensorMap* mp, CUtensorMap* mG, CUtensorMap* mg, CUtensorMap* mf) {
  using namespace tcmap;
  static_assert(Cfg<MAP_FWD>::CH == Cfg<MAP_POSTFWD>::CH &&
                    Cfg<MAP_FWD>::CH == Cfg<MAP_BWD_SPLIT>::CH,
                "one chunk width for the 128-byte-row modes");
  const bool wide = mode != MAP_BWD;  // 128-byte rows
  const uint32_t CH = wide ? Cfg<MAP_FWD>::CH : Cfg<MAP_BWD>::CH;
  const CUtensorMapSwizzle SW = wide ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {CH, 1, TM};
  cudaError_t e = make_tmap_bf16(mx, x, 3, dx, sx, bx, SW);
  if (e != cudaSuccess) return e;
  const uint64_t dp[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)NL};
  const uint32_t bp[3] = {CH, 1, NL};
  e = make_tmap_bf16(mp, phiT, 3, dp, sx, bp, SW);
  if (e != cudaSuccess) return e;
  // maps a mode does not read are copies of the x map (never dereferenced)
  *mG = *mx;
  *mg = *mx;
  *mf = *mx;
  const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T};
  const uint64_t s2[1] = {(uint64_t)C * 2};
  const uint32_t b2[2] = {CH, TM};
  if (mode != MAP_FWD && mode != MAP_POSTFWD) {
    e = make_tmap_bf16(mg, g, 2, d2, s2, b2, SW);
    if (e != cudaSuccess) return e;
  }
  if (mode == MAP_BWD) {
    e = make_tmap_bf16(mG, G, 3, dx, sx, bx, SW);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(mf, f, 2, d2, s2, b2, SW);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Smallest checkpoint period whose checkpoints fit beside the epilogue
// scratch in the freed stage memory.
static int ck_period_for(int iters, size_t stage_bytes) {
  using namespace tcmap;
  const size_t scratch = (size_t)(2 * TM + 2 * M * TM + (M + 3) * TM) * 4;
  const size_t per_ck = (size_t)N * N * TM * 4;
  const int max_ck = (int)((stage_bytes - scratch) / per_ck);  // >= 2 for the sizes used here
  const int steps = 2 * iters;
  int P = 1;
  while (steps / P + 1 > max_ck) ++P;
  return P;
}

size_t map_tc_phi_bytes(int64_t C) { return (size_t)tcmap::NL * tcmap::N * C * 2; }

static int map_device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Parts per 128-token tile.  The time of a launch is about
//   waves(kp) * (chunks per part + F),   waves(kp) = ceil(tiles * kp / SMs),
// where F = 8 chunks is a CTA's fixed cost (setup, pipeline fill and drain,
// the part records and their combine), measured at T = 16384, C = 7168: there
// one part per tile (one wave of 128 CTAs) beats eight parts (1024 CTAs).
// Small T is where the split pays: at T = 4096 one part per tile would leave
// 116 of 148 SMs idle.
static int map_tc_kp(int64_t T, int64_t C) {
  using namespace tcmap;
  const int64_t ntt = (T + TM - 1) / TM;
  constexpr int kModelCh = 32;  // the cost model counts 32-channel chunks
  const int nch = (int)((C + kModelCh - 1) / kModelCh);
  const int sms = map_device_sms();
  constexpr double kFixedChunks = 8.0;
  int kmax = nch / 4;
  if (kmax > 32) kmax = 32;
  if (kmax < 1) kmax = 1;
  int best = 1;
  double best_cost = 0.0;
  for (int kp = 1; kp <= kmax; ++kp) {
    const int64_t waves = (ntt * kp + sms - 1) / sms;
    const double cost = (double)waves * ((double)nch / kp + kFixedChunks);
    if (kp == 1 || cost < best_cost * 0.97) {  // a new split must win by 3 %
      best_cost = cost;
      best = kp;
    }
  }
  return best;
}

static size_t round256(size_t v) { return (v + 255) / 256 * 256; }

// Part records [tiles][kp][128][KREC] fp32 and per-tile counters; 0 when one
// CTA per tile fills the SMs.
size_t map_tc_scratch_bytes(int64_t T, int64_t C) {
  using namespace tcmap;
  const int kp = map_tc_kp(T, C);
  if (kp == 1) return 0;
  const int64_t ntt = (T + TM - 1) / TM;
  return round256((size_t)ntt * kp * TM * KREC * 4) + round256((size_t)ntt * 4);
}

template <int MODE>
static cudaError_t launch_map_tc(const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mG,
                                 const CUtensorMap& mg, const CUtensorMap& mf, int64_t T, int64_t C,
                                 int iters, float eps, const float* b, const float* alpha, int ag,
                                 float* Hpre, float* Hpost, float* Hres, void* urec, float* hrec,
                                 float* part, const float* red, void* kscratch, int* st,
                                 int64_t wait_ns, cudaStream_t s, const float* hpost_in = nullptr,
                                 const float* hres_in = nullptr) {
  using namespace tcmap;
  auto kern = k_map_tc<MODE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<MODE>::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t ntt = (T + TM - 1) / TM;
  const int kp = map_tc_kp(T, C);
  float* kpart = nullptr;
  int* kcnt = nullptr;
  if (kp > 1) {
    if (kscratch == nullptr) return cudaErrorInvalidValue;
    kpart = (float*)kscratch;
    kcnt = (int*)((char*)kscratch + round256((size_t)ntt * kp * TM * KREC * 4));
    // per-tile part counters start at zero (each tile's last part resets its own)
    e = cudaMemsetAsync(kcnt, 0, (size_t)ntt * sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = (unsigned)(ntt * kp);
  const int P = (MODE == MAP_BWD || MODE == MAP_BWD_SPLIT) ? ck_period_for(iters, Cfg<MODE>::DATA) : 1;
  kern<<<grid, NT, Cfg<MODE>::SMEM, s>>>(mx, mp, mG, mg, mf, T, C, iters, eps, P, b, alpha, ag, Hpre,
                                         Hpost, Hres, (__nv_bfloat16*)urec, hrec, part, red,
                                         hpost_in, hres_in, kp, kpart, kcnt, st,
                                         tc::wait_limit(wait_ns));
  return cudaGetLastError();
}

cudaError_t map_tc_dispatch(int mode, int64_t T, int64_t C, int iters, float eps, const void* x,
                            const float* phi, void* phi_split, const float* b, const float* alpha,
                            int ag,
                            float* Hpre, float* Hpost, float* Hres, const void* G, const void* g,
                            const void* f, const float* red, void* urec, float* hrec, float* part,
                            void* kscratch, int* st, int64_t wait_ns, cudaStream_t s) {
  using namespace tcmap;
  const int64_t K = (int64_t)N * C;
  k_phi_split<<<(unsigned)((K + 255) / 256), 256, 0, s>>>(K, phi, (__nv_bfloat16*)phi_split);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mp, mG, mg, mf;
  e = encode_maps(mode, T, C, x, phi_split, G, g, f, &mx, &mp, &mG, &mg, &mf);
  if (e != cudaSuccess) return e;
  switch (mode) {
    case MAP_FWD:
      return launch_map_tc<MAP_FWD>(mx, mp, mG, mg, mf, T, C, iters, eps, b, alpha, ag, Hpre, Hpost,
                                    Hres, nullptr, nullptr, nullptr, nullptr, kscratch, st, wait_ns, s);
    case MAP_BWD:
      return launch_map_tc<MAP_BWD>(mx, mp, mG, mg, mf, T, C, iters, eps, b, alpha, ag, nullptr,
                                    nullptr, nullptr, urec, hrec, part, nullptr, kscratch, st, wait_ns, s);
    case MAP_BWD_SPLIT:
      return launch_map_tc<MAP_BWD_SPLIT>(mx, mp, mG, mg, mf, T, C, iters, eps, b, alpha, ag, nullptr,
                                          nullptr, nullptr, urec, hrec, part, red, kscratch, st, wait_ns, s);
    default:
      return cudaErrorInvalidValue;
  }
}

// Layer l's post merge fused with layer l+1's forward mapping (bf16, n = 4):
// x_next = H_res x + H_post^T f_out is written once, and its RMS, projection
// onto phi_next, gates and Sinkhorn give layer l+1's maps.
cudaError_t post_map_tc_dispatch(int64_t T, int64_t C, int iters, float eps, const void* x,
                                 const void* f, const float* Hpost_in, const float* Hres_in,
                                 const float* phi_next, void* phi_split, const float* b_next,
                                 const float* alpha_next, int ag, void* x_next, float* Hpre,
                                 float* Hpost,
                                 float* Hres, void* kscratch, int* st, int64_t wait_ns,
                                 cudaStream_t s) {
  using namespace tcmap;
  const int64_t K = (int64_t)N * C;
  k_phi_split<<<(unsigned)((K + 255) / 256), 256, 0, s>>>(K, phi_next,
                                                          (__nv_bfloat16*)phi_split);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mp, mG, mg, mf;
  // the forward maps for x and phi, then x_next (store) and f_out
  e = encode_maps(MAP_POSTFWD, T, C, x, phi_split, nullptr, nullptr, nullptr, &mx, &mp, &mG, &mg,
                  &mf);
  if (e != cudaSuccess) return e;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {(uint32_t)Cfg<MAP_POSTFWD>::CH, 1, TM};
  e = make_tmap_bf16(&mG, x_next, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T};
  const uint64_t s2[1] = {(uint64_t)C * 2};
  const uint32_t b2[2] = {(uint32_t)Cfg<MAP_POSTFWD>::CH, TM};
  e = make_tmap_bf16(&mf, f, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  return launch_map_tc<MAP_POSTFWD>(mx, mp, mG, mg, mf, T, C, iters, eps, b_next, alpha_next, ag, Hpre,
                                    Hpost, Hres, nullptr, nullptr, nullptr, nullptr, kscratch, st,
                                    wait_ns, s, Hpost_in, Hres_in);
}

}  // namespace mhc
