// k_map8_tc.cu -- per-token mapping for n = 8 streams with bf16 activations:
// the logit projection y = x . phi (nC x 80) runs on the 5th-generation
// tensor cores (tcgen05.mma, bf16 operands, fp32 accumulation in TMEM); the
// sum of squares and, in the backward, the 80 C-reductions run on the CUDA
// cores from the same shared-memory stages.  Sources: the fused RMSNorm /
// projection / gating operator of the chatgpz.de explainer (section
// "Systemarbeit und Schulungsaufwand"), the n-stream buffer of section "Von
// Residualverbindungen zu Hyperverbindungen", and reportify.cn [17]-[19],
// [21], [26] (RMS applied after the projection, Sinkhorn and its custom
// backward in one operator, recompute, wider stream buffers).
//
// One CTA = 128 tokens (the MMA M).  The token's 8 C inputs stream through a
// TMA ring in chunks of 64 channels x 2 streams (128-byte rows, 128-byte
// swizzle; chunk cc covers channel group cc / 4 and streams 2 (cc % 4) and
// 2 (cc % 4) + 1): per stream an x tile [128 x 64] (the A operand, K-major,
// four K-steps of 16 channels) and, per 16 channels and stream, the rows of the
// bf16 split copy of phi^T as a [160 x 16] B operand -- the 80 logit columns'
// high parts, then their low parts (phi = hi + lo) -- so
// y = D[:, m] + D[:, 80 + m] carries phi to ~16 bits while x is exact.  The
// split copy is tiled and pre-swizzled, so a chunk's eight phi tiles (40 KB)
// arrive as four bulk copies.  The library's whole backward runs this kernel in
// the MAP_BWD_DOTS mode (only x staged, three stages): every C-reduction comes
// from the tensor-core reductions of k_dots_tc.cu.  The training-order
// backward runs the split mode: <G_i, x_j> and <G_i, f_out> from the post
// half, <g, x_j> here (grad_h_in staged with each chunk).
//
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs, warps
// 2..9 reduce: warp 2 + 4h + q covers token rows 32q..32q+31 and stream h of
// each chunk's pair, i.e. the sum of squares of streams h, h + 2, h + 4, h + 6
// and, in the split backward, <g, x_j> for those streams.  The h = 0 warps
// then run the per-token epilogue (gates, Sinkhorn and its adjoint) with one
// thread per token and write the same per-token records as the CUDA-core
// mapping plus the U rows of the n = 8 tensor-core apply.
// Every wait is bounded; on timeout the kernel records MHC_ERR_TIMEOUT,
// drains what it issued, frees TMEM and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
#include "tc_sm100.cuh"

namespace mhc {

namespace tcm8 {
constexpr int N = 8;
constexpr int M = N * N + 2 * N;     // 80 logits
constexpr int TM = 128;              // tokens per CTA (MMA M)
constexpr int NL = 2 * M;            // MMA N: 80 high + 80 low logit columns
constexpr int CH = 64;               // channels per chunk: 128-byte rows
constexpr int ROW = CH * 2;
constexpr int XBOX = TM * ROW;       // one stream's x (or grad_h_in) tile: 16 KB
constexpr int SPC = 2;               // streams per chunk
constexpr int PB = 16;               // channels per block of the tiled phi^T copy
constexpr int PROW = PB * 2;         // its 32-byte rows
constexpr int PBOX = NL * PROW;      // one (16-channel block, stream) phi^T tile: 5 KB
constexpr int NW = 10;
constexpr int NT = NW * 32;
constexpr uint32_t TMEM_COLS = 256;
// reductions per stream half: <G_i,x_j> 32, <G_i,f> 4, <g,x_j> 4 (the split
// backward fills only the last four)
constexpr int NDH = 4 * N + 4 + 4;

template <int MODE> struct Cfg {
  static_assert(MODE == MAP_FWD || MODE == MAP_BWD_SPLIT || MODE == MAP_BWD_DOTS, "mode");
  static constexpr bool BWD = MODE == MAP_BWD_SPLIT || MODE == MAP_BWD_DOTS;
  static constexpr bool STAGE_G = MODE == MAP_BWD_SPLIT;  // grad_h_in staged
  static constexpr int X_OFF = 0;                         // x tiles of the chunk's two streams
  // phi^T tiles: the one of 16-channel step k and stream s of the pair at 2k + s
  static constexpr int P_OFF = SPC * XBOX;
  static constexpr int GG_OFF = P_OFF + SPC * (CH / PB) * PBOX;  // grad_h_in (split backward)
  static constexpr int STAGE = STAGE_G ? GG_OFF + XBOX : GG_OFF;
  static constexpr int NS = STAGE_G ? 2 : 3;
  // the stages, reused after the chunk loop by the epilogue's reductions, dz
  // rows and per-token logits
  static constexpr int DATA = NS * STAGE;
  static_assert((2 * TM + 2 * NDH * TM + (M + 3) * TM + TM * (2 * M + 4)) * 4 <= DATA,
                "epilogue scratch");
  static_assert(STAGE % 1024 == 0 && GG_OFF % 1024 == 0, "128-byte swizzle atoms");
  static constexpr int SMEM = DATA + 1024 /*align*/ + 256 /*barriers, flags*/;
  static_assert(SMEM <= 232448, "shared memory");
};
}  // namespace tcm8

namespace {

__device__ __forceinline__ void unpack8(uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// 16-byte piece `c` (0..7) of token row `tok` of a [128 x 64] bf16 tile
// stored with the 128-byte swizzle.
__device__ __forceinline__ uint4 ld128sw(const uint8_t* tile, int tok, int c) {
  return *reinterpret_cast<const uint4*>(tile + tok * tcm8::ROW + ((c ^ (tok & 7)) << 4));
}

__device__ __forceinline__ void nbar8(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(tcm8::NT, 1) k_map8_tc(
    const __grid_constant__ CUtensorMap tm_x, const __nv_bfloat16* __restrict__ phi_t,
    const __grid_constant__ CUtensorMap tm_g, int64_t T, int64_t C, int iters, float eps,
    float* __restrict__ ck, const float* __restrict__ bias, const float* __restrict__ alpha_p,
    int ag,
    float* __restrict__ Hpre_o, float* __restrict__ Hpost_o, float* __restrict__ Hres_o,
    float* __restrict__ coef_o, __nv_bfloat16* __restrict__ urec_o, float* __restrict__ part_o,
    const float* __restrict__ red_in, int* status, uint64_t wait_ns) {
  using namespace tcm8;
  using CFG = Cfg<MODE>;
  using CF = Coef<N>;
  constexpr bool BWD = CFG::BWD;
  constexpr bool DOTS = MODE == MAP_BWD_DOTS;  // every C-reduction from red_in
  constexpr bool STAGE_G = CFG::STAGE_G;
  constexpr int NS = CFG::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + CFG::DATA);  // full[NS] empty[NS] done fin
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty = [&](int s) { return tc::smem_u32(bars + NS + s); };
  const uint32_t done_bar = tc::smem_u32(bars + 2 * NS);
  const uint32_t fin_bar = tc::smem_u32(bars + 2 * NS + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t0 = (int64_t)blockIdx.x * TM;
  const int nch = (int)((C + CH - 1) / CH) * (N / SPC);  // chunks: channel groups x stream pairs
  const int64_t K = (int64_t)N * C;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1 + 8);  // the MMA commit + every math warp
    }
    tc::mbar_init(done_bar, 1);
    tc::mbar_init(fin_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_x);
    if constexpr (STAGE_G) tc::tma_prefetch_desc(&tm_g);
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
        if (cc >= NS && !tc::mbar_wait(empty(s), ((uint32_t)(cc / NS) & 1u) ^ 1u, abort_flag,
                                       wait_ns)) {
          give_up();
          break;
        }
        const uint32_t base = tc::smem_u32(smem + s * CFG::STAGE);
        tc::mbar_arrive_expect_tx(full(s), CFG::STAGE);
        const int c0 = (cc >> 2) * CH, j0 = SPC * (cc & 3);
        // the chunk's phi^T tiles: for each of its four 16-channel blocks, the
        // tiles of streams j0 and j0 + 1 are one contiguous 10 KB piece of the
        // tiled copy, already in the 32-byte swizzled shared-memory order
        for (int k = 0; k < CH / PB; ++k)
          tc::bulk_load(base + CFG::P_OFF + SPC * k * PBOX,
                        phi_t + ((int64_t)((cc >> 2) * (CH / PB) + k) * N + j0) * (NL * PB),
                        SPC * PBOX, full(s), pol_keep);
        for (int i = 0; i < SPC; ++i)
          tc::tma_load_3d(base + CFG::X_OFF + i * XBOX, &tm_x, full(s), c0, j0 + i, (int)t0,
                          pol_stream);
        if constexpr (STAGE_G)
          tc::tma_load_2d(base + CFG::GG_OFF, &tm_g, full(s), c0, (int)t0, pol_stream);
        ++issued;
      }
      // every copy issued here has landed before the CTA can exit
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
        if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t base = tc::smem_u32(smem + s * CFG::STAGE);
#pragma unroll
        for (int i = 0; i < SPC; ++i) {
#pragma unroll
          for (int k = 0; k < CH / PB; ++k) {
            // A: x tile i, 16-channel step k (32 bytes into each 128-byte row);
            // B: the phi^T tile of block k and stream j0 + i
            const uint64_t a =
                tc::smem_desc(base + CFG::X_OFF + i * XBOX + 32 * k, 16, 8 * ROW, tc::SWZ_128B);
            const uint64_t bd = tc::smem_desc(base + CFG::P_OFF + (SPC * k + i) * PBOX, 16,
                                              8 * PROW, tc::SWZ_32B);
            tc::mma_bf16(tmem, a, bd, idesc, (cc | i | k) != 0 ? 1u : 0u);
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
    // -------------------------------------------------- CUDA-core reductions
    const int q = warp & 3;              // TMEM lane quarter this warp may read
    const int h = (warp - 2) >> 2;       // stream h of each chunk's pair (streams h, h + 2, ..)
    const int tok = 32 * q + lane;
    float ss = 0.0f;
    // split backward: <g, x_j> for j = 2p + h (p = chunk % 4) at [36 + p], the
    // layout of the reductions buffer below
    float dots[BWD ? NDH : 1];
#pragma unroll
    for (int e = 0; e < (BWD ? NDH : 1); ++e) dots[e] = 0.0f;
    bool run = true;
    for (int cc4 = 0; cc4 < nch && run; cc4 += N / SPC) {
#pragma unroll
      for (int p = 0; p < N / SPC; ++p) {
        const int cc = cc4 + p;
        const int s = cc % NS;
        if (!tc::mbar_wait(full(s), (uint32_t)(cc / NS) & 1u, abort_flag, wait_ns)) {
          give_up();
          run = false;
          break;
        }
        const uint8_t* st = smem + s * CFG::STAGE;
        const uint8_t* xt = st + CFG::X_OFF + h * XBOX;
#pragma unroll
        for (int c = 0; c < CH / 8; ++c) {  // the 8-channel pieces of the chunk
          float xv[8];
          unpack8(ld128sw(xt, tok, c), xv);
          if constexpr (STAGE_G) {
            float gv[8];
            unpack8(ld128sw(st + CFG::GG_OFF, tok, c), gv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              ss = fmaf(xv[e], xv[e], ss);
              dots[36 + p] = fmaf(gv[e], xv[e], dots[36 + p]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(xv[e], xv[e], ss);
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty(s));
      }
    }

    bool ok = !*abort_flag && tc::mbar_wait(done_bar, 0, abort_flag, wait_ns);
    if (!ok && !*abort_flag) give_up();
    ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
    // stage memory is reused below: every math warp has finished reading it
    nbar8(1, 256);
    float* red_ss = reinterpret_cast<float*>(smem);   // [2][TM]
    float* red_dt = red_ss + 2 * TM;                  // [2][NDH][TM]
    float* dzs = red_dt + 2 * NDH * TM;               // [M + 3][TM]
    constexpr int ZS = 2 * M + 4;                     // a token's z (M), then y / r (M)
    float* zs = dzs + (M + 3) * TM;                   // [TM][ZS]
    if (ok) {
      red_ss[h * TM + tok] = ss;
      if constexpr (BWD) {
#pragma unroll
        for (int e = 0; e < NDH; ++e) red_dt[(h * NDH + e) * TM + tok] = dots[e];
      }
    }
    nbar8(1, 256);
    if (ok && h == 0) {
      // ---------------------------------- the logits, one thread per token
      tc::tc_fence_after();
      const bool live = t0 + tok < T;
      const uint32_t lb = tmem + ((uint32_t)(32 * q) << 16);
      const float r = sqrtf((red_ss[tok] + red_ss[TM + tok]) / (float)K + eps);
      Alpha3 al;
      al.load(alpha_p, ag);
      float* zt = zs + tok * ZS;
      float zf[BWD ? 1 : M];  // the forward keeps its logits in registers
      bool bad = !isfinite(r);
      float lo16[16], hi16[16];
#pragma unroll
      for (int b16 = 0; b16 < M / 16; ++b16) {
        tc::tmem_ld16(lb + 16 * b16, hi16);
        tc::tmem_ld16(lb + M + 16 * b16, lo16);
        tc::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int m = 16 * b16 + e;
          const float yv = (hi16[e] + lo16[e]) / r;
          const float z = fmaf(al.at<N>(m), yv, __ldg(bias + m));
          bad |= !isfinite(z);
          if constexpr (BWD) {
            zt[m] = z;
            zt[M + m] = yv;
          } else {
            zf[m] = z;
          }
        }
      }
      if (live && bad) flag_status(status, MHC_ERR_NONFINITE);
      if constexpr (!BWD) {
        // the forward: gates and Sinkhorn in this thread's registers
        const int64_t t = t0 + tok;
        float H[N * N];
#pragma unroll
        for (int e = 0; e < N * N; ++e) H[e] = zf[2 * N + e];
        sk_forward<N>(H, iters);
        if (live) {
#pragma unroll
          for (int i = 0; i < N; i += 4) {
            *reinterpret_cast<float4*>(Hpre_o + t * N + i) =
                make_float4(sigmoidf_(zf[i]), sigmoidf_(zf[i + 1]), sigmoidf_(zf[i + 2]),
                            sigmoidf_(zf[i + 3]));
            *reinterpret_cast<float4*>(Hpost_o + t * N + i) = make_float4(
                2.0f * sigmoidf_(zf[N + i]), 2.0f * sigmoidf_(zf[N + i + 1]),
                2.0f * sigmoidf_(zf[N + i + 2]), 2.0f * sigmoidf_(zf[N + i + 3]));
          }
#pragma unroll
          for (int e = 0; e < N * N; e += 4)
            *reinterpret_cast<float4*>(Hres_o + t * N * N + e) =
                make_float4(H[e], H[e + 1], H[e + 2], H[e + 3]);
        }
      }
    }
    if constexpr (BWD) nbar8(1, 256);
    if (BWD && ok) {
      // ------------- gates, Sinkhorn and its adjoint: 8 lanes per token, lane
      // i on row i of H_res and on pre / post logit i; 4 tokens per warp, the
      // 8 math warps take the 128 tokens in 4 rounds
      const int i = lane & 7, sub = lane >> 3, mw = warp - 2;
      Alpha3 al;
      al.load(alpha_p, ag);
#pragma unroll 1
      for (int rd = 0; rd < TM / 32; ++rd) {
        const int tk = 32 * rd + 4 * mw + sub;
        const int64_t t = t0 + tk;
        const bool live = t < T;
        const float* zt = zs + tk * ZS;
        float a[N], sq[N];
#pragma unroll
        for (int j = 0; j < N; ++j) a[j] = zt[2 * N + N * i + j];
        const float spre = sigmoidf_(zt[i]), spost = sigmoidf_(zt[N + i]);
        skl_init<N>(a, iters);
        {
          // checkpoints: the iterate after every second normalisation (and the
          // start), row i of each at ckt + c * 64
          float* ckt = ck + (live ? t : 0) * ((int64_t)iters + 1) * N * N + N * i;
          auto ck_store = [&](int c) {
            if (live) {
              float4* d4 = reinterpret_cast<float4*>(ckt + (int64_t)c * N * N);
              d4[0] = make_float4(a[0], a[1], a[2], a[3]);
              d4[1] = make_float4(a[4], a[5], a[6], a[7]);
            }
          };
          auto ck_load = [&](int c) {
            if (live) {
              const float4* s4 = reinterpret_cast<const float4*>(ckt + (int64_t)c * N * N);
              const float4 v0 = s4[0], v1 = s4[1];
              a[0] = v0.x; a[1] = v0.y; a[2] = v0.z; a[3] = v0.w;
              a[4] = v1.x; a[5] = v1.y; a[6] = v1.z; a[7] = v1.w;
            } else {
#pragma unroll
              for (int j = 0; j < N; ++j) a[j] = 1.0f;
            }
          };
          ck_store(0);
          for (int qn = 1; qn <= 2 * iters; ++qn) {
            skl_step<N>(a, qn, sq);
            if ((qn & 1) == 0) ck_store(qn >> 1);
          }
          float H[N];
#pragma unroll
          for (int j = 0; j < N; ++j) H[j] = a[j];
          // dL/dH_res: <G_i, x_j> from the post half's reductions (split) or the
          // tensor-core reductions' rows (DOTS)
          constexpr int RSTRIDE = DOTS ? N * N + 2 * N : N * N + N;
          const float* rt = red_in + (live ? t : 0) * RSTRIDE;
          float g[N];
#pragma unroll
          for (int j = 0; j < N; ++j) g[j] = live ? __ldg(rt + N * i + j) : 0.0f;
          for (int step = 2 * iters; step >= 1; --step) {
            const int c = (step - 1) >> 1;
            ck_load(c);
            for (int qn = 2 * c + 1; qn < step; ++qn) skl_step<N>(a, qn, sq);
            skl_step<N>(a, step, sq);
            skl_adjoint_step<N>(a, sq, g, step);
          }
          ck_load(0);  // the exponentiated logits
          float dzres[N];
#pragma unroll
          for (int j = 0; j < N; ++j) dzres[j] = g[j] * a[j];
          // <g, x_i>: stream i was reduced by the warps of pair member i & 1 (split)
          const float dpre = DOTS ? (live ? __ldg(rt + N * N + N + i) : 0.0f)
                                  : red_dt[((i & 1) * NDH + 36 + (i >> 1)) * TM + tk];
          const float dpost = live ? __ldg(rt + N * N + i) : 0.0f;
          const float dzpre = dpre * spre * (1.0f - spre);
          const float dzpost = dpost * 2.0f * spost * (1.0f - spost);
          float pres = 0.0f;
#pragma unroll
          for (int j = 0; j < N; ++j) pres = fmaf(dzres[j], zt[M + 2 * N + N * i + j], pres);
          const float dzy0 = group_sum<N>(dzpre * zt[M + i]);
          const float dzy1 = group_sum<N>(dzpost * zt[M + N + i]);
          const float dzy2 = group_sum<N>(pres);
          const float r = sqrtf((red_ss[tk] + red_ss[TM + tk]) / (float)K + eps);
          const float ar0 = al.a[0] / r, ar1 = al.a[1] / r, ar2 = al.a[2] / r;
          if (live) {
            // the per-token record of the n = 8 apply: H_res | H_pre | H_post | u | kappa
            float* co = coef_o + t * CF::SIZE;
            float4* hr = reinterpret_cast<float4*>(co + CF::RES + N * i);
            hr[0] = make_float4(H[0], H[1], H[2], H[3]);
            hr[1] = make_float4(H[4], H[5], H[6], H[7]);
            co[CF::PRE + i] = spre;
            co[CF::POST + i] = 2.0f * spost;
            const float upre = ar0 * dzpre, upost = ar1 * dzpost;
            co[CF::U + i] = upre;
            co[CF::U + N + i] = upost;
            float ures[N];
#pragma unroll
            for (int j = 0; j < N; ++j) ures[j] = ar2 * dzres[j];
            float4* ur = reinterpret_cast<float4*>(co + CF::U + 2 * N + N * i);
            ur[0] = make_float4(ures[0], ures[1], ures[2], ures[3]);
            ur[1] = make_float4(ures[4], ures[5], ures[6], ures[7]);
            if (i == 0)
              co[CF::KAPPA] = fmaf(al.a[2], dzy2, fmaf(al.a[1], dzy1, al.a[0] * dzy0)) /
                              ((float)K * r * r);
            // the MMA operand row: u to ~16 bits as bf16 high and low parts,
            // [u_hi (80) | 0 (16) | u_lo (80) | 0 (16)]
            __nv_bfloat16* ud = urec_o + t * TcRec8::U_ELEMS;
            auto split = [&](float u, __nv_bfloat16& hi, __nv_bfloat16& lo) {
              hi = __float2bfloat16_rn(u);
              lo = __float2bfloat16_rn(u - __bfloat162float(hi));
            };
            __nv_bfloat16 h0, l0;
            split(upre, h0, l0);
            ud[i] = h0;
            ud[TcRec8::LO + i] = l0;
            split(upost, h0, l0);
            ud[N + i] = h0;
            ud[TcRec8::LO + N + i] = l0;
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int p2 = 0; p2 < 4; ++p2) {
              const __nv_bfloat162 hi = __floats2bfloat162_rn(ures[2 * p2], ures[2 * p2 + 1]);
              const __nv_bfloat162 lo = __floats2bfloat162_rn(ures[2 * p2] - __low2float(hi),
                                                              ures[2 * p2 + 1] - __high2float(hi));
              hw[p2] = *reinterpret_cast<const uint32_t*>(&hi);
              lw[p2] = *reinterpret_cast<const uint32_t*>(&lo);
            }
            *reinterpret_cast<uint4*>(ud + 2 * N + N * i) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(ud + TcRec8::LO + 2 * N + N * i) =
                make_uint4(lw[0], lw[1], lw[2], lw[3]);
            if (i < 2) {  // the zero padding after u_hi and after u_lo
              *reinterpret_cast<uint4*>(ud + M + 8 * i) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(ud + TcRec8::LO + M + 8 * i) = make_uint4(0, 0, 0, 0);
            }
          }
          dzs[i * TM + tk] = live ? dzpre : 0.0f;
          dzs[(N + i) * TM + tk] = live ? dzpost : 0.0f;
#pragma unroll
          for (int j = 0; j < N; ++j) dzs[(2 * N + N * i + j) * TM + tk] = live ? dzres[j] : 0.0f;
          if (i == 0) {
            dzs[M * TM + tk] = live ? dzy0 : 0.0f;
            dzs[(M + 1) * TM + tk] = live ? dzy1 : 0.0f;
            dzs[(M + 2) * TM + tk] = live ? dzy2 : 0.0f;
          }
        }
      }
    }
    if constexpr (BWD) {
      nbar8(1, 256);
      if (ok && h == 0 && tok < M + 3) {
        // this tile's share of grad_b and the three grad_alpha sums, in token order
        float a = 0.0f;
        for (int k = 0; k < TM; ++k) a += dzs[tok * TM + k];
        part_o[(int64_t)blockIdx.x * CF::DZ_SIZE + tok] = a;
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
namespace {
// phi [K][80] fp32 (k = j*C + c) -> the tiled bf16 split of phi^T the mapping
// and apply MMAs read: block (chunk q of 16 channels, stream j) holds the 160
// rows m (0..79 the high parts, 80..159 the bf16 rounding of the remainder) of
// 16 channels, 32 bytes per row, with the two 16-byte halves of rows whose bit
// 2 is set swapped -- the 32-byte swizzle of a 256-byte-aligned tile, so one
// bulk copy of a block (or of consecutive streams' blocks) lands in shared
// memory ready for the MMA.  The copy covers whole 64-channel groups (the
// mapping's chunks); channels c >= C are zero.
__global__ void k_phi_split8(int64_t C, int64_t ncp, const float* __restrict__ phi,
                             __nv_bfloat16* __restrict__ out) {
  using namespace tcm8;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // j * ncp + c
  if (idx >= (int64_t)N * ncp) return;
  const int64_t j = idx / ncp, c = idx % ncp;
  const int64_t q = c / PB;
  const int ci = (int)(c % PB), h = ci >> 3, e = ci & 7;
  __nv_bfloat16* blk = out + (q * N + j) * (NL * PB);
#pragma unroll 4
  for (int m = 0; m < M; ++m) {
    const float v = c < C ? __ldg(phi + (j * C + c) * M + m) : 0.0f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    const int m2 = M + m;
    blk[m * PB + ((h ^ ((m >> 2) & 1)) << 3) + e] = hi;
    blk[m2 * PB + ((h ^ ((m2 >> 2) & 1)) << 3) + e] = lo;
  }
}

template <int MODE>
cudaError_t launch_map8(const CUtensorMap& mx, const void* phi_t, const CUtensorMap& mg,
                        int64_t T, int64_t C,
                        int iters, float eps, const float* b, const float* alpha, int ag,
                        float* Hpre, float* Hpost, float* Hres, float* coef, void* urec,
                        float* part, const float* red, float* ck, int* st, int64_t wait_ns,
                        cudaStream_t s) {
  using namespace tcm8;
  auto kern = k_map8_tc<MODE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<MODE>::SMEM);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((T + TM - 1) / TM);
  kern<<<grid, NT, Cfg<MODE>::SMEM, s>>>(mx, (const __nv_bfloat16*)phi_t, mg, T, C, iters, eps,
                                          ck, b, alpha, ag,
                                          Hpre, Hpost, Hres, coef, (__nv_bfloat16*)urec, part,
                                          red, st, tc::wait_limit(wait_ns));
  return cudaGetLastError();
}
}  // namespace

size_t map8_ck_bytes(int64_t T, int iters) {
  return (size_t)T * ((size_t)iters + 1) * tcm8::N * tcm8::N * 4;
}

size_t map8_tc_phi_bytes(int64_t C) {
  const int64_t nblk = (C + tcm8::CH - 1) / tcm8::CH * (tcm8::CH / tcm8::PB);
  return (size_t)nblk * tcm8::N * tcm8::NL * tcm8::PB * 2;
}

cudaError_t map8_tc_dispatch(int mode, int64_t T, int64_t C, int iters, float eps, const void* x,
                             const float* phi, void* phi_split, const float* b,
                             const float* alpha, int ag, float* Hpre, float* Hpost, float* Hres,
                             const void* G, const void* g, const void* f, const float* red,
                             float* coef, void* urec, float* part, float* ck, int* st,
                             int64_t wait_ns, cudaStream_t s) {
  using namespace tcm8;
  const int64_t ncp = (C + CH - 1) / CH * CH;
  k_phi_split8<<<(unsigned)((N * ncp + 255) / 256), 256, 0, s>>>(C, ncp, phi,
                                                                  (__nv_bfloat16*)phi_split);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mg;
  const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {CH, 1, TM};
  e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, SW);
  if (e != cudaSuccess) return e;
  mg = mx;  // read only by the split backward (otherwise a copy, never dereferenced)
  if (mode == MAP_BWD_SPLIT) {
    const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T};
    const uint64_t s2[1] = {(uint64_t)C * 2};
    const uint32_t b2[2] = {CH, TM};
    e = make_tmap_bf16(&mg, g, 2, d2, s2, b2, SW);
    if (e != cudaSuccess) return e;
  }
  switch (mode) {
    case MAP_FWD:
      return launch_map8<MAP_FWD>(mx, phi_split, mg, T, C, iters, eps, b, alpha, ag, Hpre, Hpost,
                                  Hres, nullptr, nullptr, nullptr, nullptr, nullptr, st, wait_ns,
                                  s);
    case MAP_BWD_SPLIT:
      return launch_map8<MAP_BWD_SPLIT>(mx, phi_split, mg, T, C, iters, eps, b, alpha, ag, nullptr,
                                        nullptr, nullptr, coef, urec, part, red, ck, st, wait_ns,
                                        s);
    case MAP_BWD_DOTS:
      return launch_map8<MAP_BWD_DOTS>(mx, phi_split, mg, T, C, iters, eps, b, alpha, ag, nullptr,
                                       nullptr, nullptr, coef, urec, part, red, ck, st, wait_ns,
                                       s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace mhc
