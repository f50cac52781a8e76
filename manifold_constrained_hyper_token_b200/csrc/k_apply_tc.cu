// k_apply_tc.cu -- second phase of the mHC backward on the tensor cores
// (bf16 activations, n = 4).  From the per-token records of the mapping
// kernel (H_res, H_pre, H_post, u = alpha dz / r, kappa) it writes
//
//   grad_x[j][c]   = (phi u)[jC+c] + sum_i H_res[i][j] G[i][c] + H_pre[j] g[c] - kappa x[j][c]
//   grad_f_out[c]  = sum_i H_post[i] G[i][c]
//   grad_phi[k][m] = sum_t x_t[k] u_t[m]
//
// (reverse mode of the update equation of the chatgpz.de explainer and of the
// RMS-normalised projection; reportify.cn [19]-[21]).
//
// Work item = (channel slice of 32 channels x 4 streams = 128 rows of phi,
// token tile of 128 tokens).  Items are numbered slice-major and the 148 SMs
// take equal contiguous ranges of them (one persistent CTA per SM), so every
// SM streams the same number of bytes.  Per item:
//   MMA1  D1[tok][k] = U[tok][m'] x PHI[k][m']        (phi u for grad_x)
//   MMA2  D2[k][m'] += X[tok][k]^T x U[tok][m']        (grad_phi, over tokens)
// U holds u as a bf16 high part and low part (m' = 0..23 and 32..55), so
// MMA2 carries u to ~16 bits and x is exact; PHI holds phi's bf16 high part
// in both halves, so D1 = (u_hi + u_lo) . phi_hi -- phi u is a small term of
// grad_x.  X (TMA, 64-byte swizzle) is the MN-major A operand of MMA2; U is
// written by the epilogue threads with the 128-byte swizzle and serves as the
// K-major A of MMA1 and the MN-major B of MMA2.
//
// grad_phi: a CTA accumulates D2 in TMEM over the consecutive items of one
// slice ("segment") and flushes it at the segment's end.  A slice is covered
// by at most two CTAs; their two partials are added in a fixed order (first
// part + second part) by whichever finishes last, so the result does not
// depend on timing.  Waits are bounded; on timeout the kernel records
// MHC_ERR_TIMEOUT, drains, frees TMEM and returns.
#include "mhc_common.cuh"
#include "tc_sm100.cuh"

namespace mhc {

namespace tcap {
constexpr int N = 4;
constexpr int M = N * N + 2 * N;      // 24
constexpr int TT = 128;               // tokens per item (MMA1 M, MMA2 K)
constexpr int CS = 32;                // channels per slice
constexpr int KR = N * CS;            // 128 phi rows per slice (MMA2 M, MMA1 N)
constexpr int NU = 64;                // U width: 24 hi + 8 pad + 24 lo + 8 pad
constexpr int NWARPS = 10;
constexpr int NT = NWARPS * 32;
constexpr int XB = TT * CS * 2;       // one stream's x (or G) tile: 8 KB
constexpr int X_OFF = 0, G_OFF = N * XB, GG_OFF = 2 * N * XB;
constexpr int STAGE = GG_OFF + XB;    // 72 KB
constexpr int NS = 2;
constexpr int U_BYTES = TT * NU * 2;  // 16 KB
constexpr int PHI_BYTES = KR * NU * 2;  // 16 KB
constexpr int STAGES_OFF = 0;
constexpr int U_OFF = NS * STAGE;             // 147456
constexpr int PHI_OFF = U_OFF + 2 * U_BYTES;  // 180224
constexpr int XCH_OFF = PHI_OFF + PHI_BYTES;  // 196608: D2 exchange [KR][M] floats
constexpr int DATA = XCH_OFF + KR * M * 4;    // 208896
constexpr int SMEM = DATA + 1024 + 256;
constexpr uint32_t TMEM_COLS = 512;           // D1 x2 (256) + D2 (64)
constexpr uint32_t D2_COL = 256;
constexpr uint64_t WAIT_NS = 2000000000ull;
}  // namespace tcap

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void unpack8(uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// 16-byte chunk c of row r of a tile with 64-byte rows / 128-byte rows,
// stored with the matching TMA / UMMA swizzle.
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

struct ApplyArgs {
  int64_t T, C;
  int S;          // slices = ceil(C / 32)
  int NTT;        // token tiles = ceil(T / 128)
  int64_t items;  // S * NTT
  int64_t per;    // items per CTA
  const float* phi;     // [nC][24]
  const float* coef;    // [T][Coef<4>::SIZE]
  const float* part;    // bias / alpha partials of the mapping kernel
  int nparts;
  __nv_bfloat16* grad_x;
  __nv_bfloat16* grad_f;
  float* grad_phi;
  float* grad_b;
  float* grad_alpha;
  float* gphi_part;     // [S][2][KR][M]
  int* gphi_cnt;        // [S]
  int* status;
};

__global__ void __launch_bounds__(tcap::NT, 1) k_apply_tc(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_G,
    const __grid_constant__ CUtensorMap tm_g, const ApplyArgs a) {
  using namespace tcap;
  using CF = Coef<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DATA);
  // barrier slots
  enum { B_FULL = 0, B_SFREE = 2, B_UREADY = 4, B_UFREE = 6, B_D1READY = 8, B_D1FREE = 10,
         B_SEGREADY = 12, B_SEGDONE = 13, B_FIN = 14, NBARS = 15 };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* bcast = reinterpret_cast<int*>(tmem_slot + 2);
  auto bar = [&](int i) { return tc::smem_u32(bars + i); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t it0 = (int64_t)blockIdx.x * a.per;
  const int64_t it1 = (it0 + a.per < a.items) ? it0 + a.per : a.items;
  const int nit = (int)(it1 > it0 ? it1 - it0 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(B_FULL + s), 1);
      tc::mbar_init(bar(B_SFREE + s), 1 + 8);
      tc::mbar_init(bar(B_UREADY + s), 8);
      tc::mbar_init(bar(B_UFREE + s), 1);
      tc::mbar_init(bar(B_D1READY + s), 1);
      tc::mbar_init(bar(B_D1FREE + s), 8);
    }
    tc::mbar_init(bar(B_SEGREADY), 8);
    tc::mbar_init(bar(B_SEGDONE), 1);
    tc::mbar_init(bar(B_FIN), 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_x);
    tc::tma_prefetch_desc(&tm_G);
    tc::tma_prefetch_desc(&tm_g);
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
    flag_status(a.status, MHC_ERR_TIMEOUT);
  };
  auto item_slice = [&](int64_t it) { return (int)(it / a.NTT); };
  auto item_tile = [&](int64_t it) { return (int)(it % a.NTT); };
  auto seg_first = [&](int64_t it) { return it == it0 || item_tile(it) == 0; };
  auto seg_last = [&](int64_t it) { return it == it1 - 1 || item_tile(it) == a.NTT - 1; };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0 && nit > 0) {
      const uint64_t pol = tc::policy_evict_first();
      int issued = 0;
      for (int i = 0; i < nit; ++i) {
        const int s = i & 1;
        if (i >= 2 && !tc::mbar_wait(bar(B_SFREE + s), (uint32_t)((i >> 1) - 1) & 1u, abort_flag,
                                     WAIT_NS)) {
          give_up();
          break;
        }
        const int64_t it = it0 + i;
        const int c0 = item_slice(it) * CS;
        const int tt0 = item_tile(it) * TT;
        const uint32_t base = tc::smem_u32(smem + STAGES_OFF + s * STAGE);
        tc::mbar_arrive_expect_tx(bar(B_FULL + s), STAGE);
        for (int j = 0; j < N; ++j) {
          tc::tma_load_3d(base + X_OFF + j * XB, &tm_x, bar(B_FULL + s), c0, j, tt0, pol);
          tc::tma_load_3d(base + G_OFF + j * XB, &tm_G, bar(B_FULL + s), c0, j, tt0, pol);
        }
        tc::tma_load_2d(base + GG_OFF, &tm_g, bar(B_FULL + s), c0, tt0, pol);
        ++issued;
      }
      if (*abort_flag)
        for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i)
          tc::mbar_wait(bar(B_FULL + (i & 1)), (uint32_t)(i >> 1) & 1u, nullptr, WAIT_NS / 4);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0 && nit > 0) {
      constexpr uint32_t id1 = tc::idesc_bf16(TT, KR);                // K-major U x K-major PHI
      constexpr uint32_t id2 = tc::idesc_bf16(KR, NU, true, true);    // MN-major X x MN-major U
      const uint32_t phi_s = tc::smem_u32(smem + PHI_OFF);
      bool any = false;
      int seg = 0;
      for (int i = 0; i < nit; ++i) {
        const int64_t it = it0 + i;
        const int s = i & 1, b = i & 1;
        const uint32_t ph = (uint32_t)(i >> 1) & 1u;
        bool ok = tc::mbar_wait(bar(B_FULL + s), ph, abort_flag, WAIT_NS) &&
                  tc::mbar_wait(bar(B_UREADY + b), ph, abort_flag, WAIT_NS);
        if (ok && i >= 2) ok = tc::mbar_wait(bar(B_D1FREE + b), ph ^ 1u, abort_flag, WAIT_NS);
        const bool first = seg_first(it);
        if (ok && first) ok = tc::mbar_wait(bar(B_SEGREADY), (uint32_t)seg & 1u, abort_flag, WAIT_NS);
        if (!ok) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t xs = tc::smem_u32(smem + STAGES_OFF + s * STAGE + X_OFF);
        const uint32_t us = tc::smem_u32(smem + U_OFF + b * U_BYTES);
        // MMA1: D1[b] = U . PHI^T   (K = 64 over m', 128-byte swizzle, K-major)
#pragma unroll
        for (int k = 0; k < NU / 16; ++k) {
          const uint64_t da = tc::smem_desc(us + k * 32, 16, 1024, tc::SWZ_128B);
          const uint64_t db = tc::smem_desc(phi_s + k * 32, 16, 1024, tc::SWZ_128B);
          tc::mma_bf16(tmem + (uint32_t)(b * KR), da, db, id1, k > 0 ? 1u : 0u);
        }
        // MMA2: D2 += X^T . U   (K = 128 tokens; X MN-major 64-byte swizzle with the
        // four stream tiles 8 KB apart; U MN-major 128-byte swizzle)
#pragma unroll
        for (int k = 0; k < TT / 16; ++k) {
          const uint64_t da = tc::smem_desc(xs + k * 1024, XB, 512, tc::SWZ_64B);
          const uint64_t db = tc::smem_desc(us + k * 2048, U_BYTES, 1024, tc::SWZ_128B);
          tc::mma_bf16(tmem + D2_COL, da, db, id2, (first && k == 0) ? 0u : 1u);
        }
        any = true;
        tc::mma_commit(bar(B_D1READY + b));
        tc::mma_commit(bar(B_UFREE + b));
        tc::mma_commit(bar(B_SFREE + s));
        if (seg_last(it)) {
          tc::mma_commit(bar(B_SEGDONE));
          ++seg;
        }
      }
      if (*abort_flag && any) {
        tc::mma_commit(bar(B_FIN));
        tc::mbar_wait(bar(B_FIN), 0, nullptr, WAIT_NS / 4);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quarter
    const int h = (warp - 2) >> 2;    // channel half (16 of the slice's 32)
    const int tok = 32 * q + lane;    // token row within the tile / phi row in D2
    const int etid = threadIdx.x - 64;  // 0..255

    if (blockIdx.x == 0) {
      // grad_b / grad_alpha from the mapping kernel's per-CTA partials, in a fixed order
      float* wsum = reinterpret_cast<float*>(smem + XCH_OFF);
      const int ew = etid / 32;
      float sacc = 0.0f;
      if (lane <= M)
        for (int p = ew; p < a.nparts; p += 8) sacc += __ldg(a.part + (int64_t)p * CF::DZ_SIZE + lane);
      if (lane <= M) wsum[ew * (M + 1) + lane] = sacc;
      named_bar_sync(1, 256);
      if (etid <= M) {
        float acc = 0.0f;
        for (int w = 0; w < 8; ++w) acc += wsum[w * (M + 1) + etid];
        if (etid < M) a.grad_b[etid] = acc;
        else *a.grad_alpha = acc;
      }
      named_bar_sync(1, 256);
    }

    // PHI for a slice: row r = j*32 + c holds phi_hi[j*C + c0 + c][0..23] in m' 0..23
    // and again in m' 32..55 (zeros elsewhere), 128-byte swizzle.
    auto load_phi = [&](int slice) {
      uint8_t* ps = smem + PHI_OFF;
      for (int e = etid; e < KR * 8; e += 256) {
        const int r = e >> 3, chunk = e & 7;
        const int j = r / CS, cl = r % CS;
        const int64_t c = (int64_t)slice * CS + cl;
        const int m0 = (chunk & 3) * 8;
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int m = m0 + u;
          v[u] = (m < M && c < a.C) ? __ldg(a.phi + ((int64_t)j * a.C + c) * M + m) : 0.0f;
        }
        *reinterpret_cast<uint4*>(ps + sw128(r, chunk)) =
            make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_SEGREADY));
    };

    // coefficient record of token row `tok` of item i; writes this thread's half of
    // the U row (h = 0: u_hi, h = 1: u_lo) into U buffer i & 1.
    float hres[N * N], hpre[N], hpost[N], kap;      // for the item being finished
    float nres[N * N], npre[N], npost[N], nkap;     // for the item whose U was written
    auto write_u = [&](int i) {
      const int64_t it = it0 + i;
      const int64_t t = (int64_t)item_tile(it) * TT + tok;
      float rec[CF::SIZE];
      if (t < a.T) {
        const float4* src = reinterpret_cast<const float4*>(a.coef + t * CF::SIZE);
#pragma unroll
        for (int e = 0; e < CF::SIZE / 4; ++e) {
          const float4 v = __ldg(src + e);
          rec[4 * e] = v.x; rec[4 * e + 1] = v.y; rec[4 * e + 2] = v.z; rec[4 * e + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < CF::SIZE; ++e) rec[e] = 0.0f;
      }
#pragma unroll
      for (int e = 0; e < N * N; ++e) nres[e] = rec[CF::RES + e];
#pragma unroll
      for (int e = 0; e < N; ++e) {
        npre[e] = rec[CF::PRE + e];
        npost[e] = rec[CF::POST + e];
      }
      nkap = rec[CF::KAPPA];
      float uv[32];
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        float u = m < M ? rec[CF::U + m] : 0.0f;
        const float hi = __bfloat162float(__float2bfloat16_rn(u));
        uv[m] = h == 0 ? hi : u - hi;
      }
      const int b = i & 1;
      if (i >= 2 &&
          !tc::mbar_wait(bar(B_UFREE + b), (uint32_t)((i >> 1) - 1) & 1u, abort_flag, WAIT_NS)) {
        give_up();
        return;
      }
      uint8_t* us = smem + U_OFF + b * U_BYTES;
#pragma unroll
      for (int cch = 0; cch < 4; ++cch)
        *reinterpret_cast<uint4*>(us + sw128(tok, 4 * h + cch)) =
            make_uint4(pack2(uv[8 * cch], uv[8 * cch + 1]), pack2(uv[8 * cch + 2], uv[8 * cch + 3]),
                       pack2(uv[8 * cch + 4], uv[8 * cch + 5]), pack2(uv[8 * cch + 6], uv[8 * cch + 7]));
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_UREADY + b));
    };
    auto rotate = [&]() {
#pragma unroll
      for (int e = 0; e < N * N; ++e) hres[e] = nres[e];
#pragma unroll
      for (int e = 0; e < N; ++e) {
        hpre[e] = npre[e];
        hpost[e] = npost[e];
      }
      kap = nkap;
    };

    int seg = 0;
    if (nit > 0) {
      load_phi(item_slice(it0));
      write_u(0);
      rotate();
    }
    float* xch = reinterpret_cast<float*>(smem + XCH_OFF);
    // The loop never breaks: after a failed wait it keeps walking the items
    // without touching memory, so all eight warps meet every named barrier.
    for (int i = 0; i < nit; ++i) {
      const int64_t it = it0 + i;
      const int s = i & 1, b = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      if (i + 1 < nit && !*abort_flag) write_u(i + 1);
      bool live = !*abort_flag;
      if (live && (!tc::mbar_wait(bar(B_FULL + s), ph, abort_flag, WAIT_NS) ||
                   !tc::mbar_wait(bar(B_D1READY + b), ph, abort_flag, WAIT_NS))) {
        give_up();
        live = false;
      }
      tc::tc_fence_after();
      const int slice = item_slice(it);
      const int64_t t = (int64_t)item_tile(it) * TT + tok;
      const int64_t cbase = (int64_t)slice * CS + 16 * h;
      const uint8_t* st = smem + STAGES_OFF + s * STAGE;
      // G and g for this thread's 16 channels, all four streams
      float Gv[N][16], gv[16];
#pragma unroll
      for (int i2 = 0; i2 < N; ++i2) {
        float tmp[8];
        unpack8(*reinterpret_cast<const uint4*>(st + G_OFF + i2 * XB + sw64(tok, 2 * h)), tmp);
#pragma unroll
        for (int e = 0; e < 8; ++e) Gv[i2][e] = tmp[e];
        unpack8(*reinterpret_cast<const uint4*>(st + G_OFF + i2 * XB + sw64(tok, 2 * h + 1)), tmp);
#pragma unroll
        for (int e = 0; e < 8; ++e) Gv[i2][8 + e] = tmp[e];
      }
      {
        float tmp[8];
        unpack8(*reinterpret_cast<const uint4*>(st + GG_OFF + sw64(tok, 2 * h)), tmp);
#pragma unroll
        for (int e = 0; e < 8; ++e) gv[e] = tmp[e];
        unpack8(*reinterpret_cast<const uint4*>(st + GG_OFF + sw64(tok, 2 * h + 1)), tmp);
#pragma unroll
        for (int e = 0; e < 8; ++e) gv[8 + e] = tmp[e];
      }
      const bool tvalid = live && t < a.T;
      // grad_f_out
      if (tvalid) {
        float o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float acc = 0.0f;
#pragma unroll
          for (int i2 = 0; i2 < N; ++i2) acc = fmaf(hpost[i2], Gv[i2][e], acc);
          o[e] = acc;
        }
#pragma unroll
        for (int v8 = 0; v8 < 2; ++v8) {
          if (cbase + 8 * v8 < a.C) {
            uint4 pk = make_uint4(pack2(o[8 * v8], o[8 * v8 + 1]), pack2(o[8 * v8 + 2], o[8 * v8 + 3]),
                                  pack2(o[8 * v8 + 4], o[8 * v8 + 5]), pack2(o[8 * v8 + 6], o[8 * v8 + 7]));
            __stcs(reinterpret_cast<uint4*>(a.grad_f + t * a.C + cbase + 8 * v8), pk);
          }
        }
      }
      // grad_x, one output stream at a time
#pragma unroll
      for (int jj = 0; jj < N; ++jj) {
        float d1[16];
        if (live)
          tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * KR + jj * CS + 16 * h), d1);
        float xv[16];
        {
          float tmp[8];
          unpack8(*reinterpret_cast<const uint4*>(st + X_OFF + jj * XB + sw64(tok, 2 * h)), tmp);
#pragma unroll
          for (int e = 0; e < 8; ++e) xv[e] = tmp[e];
          unpack8(*reinterpret_cast<const uint4*>(st + X_OFF + jj * XB + sw64(tok, 2 * h + 1)), tmp);
#pragma unroll
          for (int e = 0; e < 8; ++e) xv[8 + e] = tmp[e];
        }
        if (live) tc::tmem_ld_wait();
        if (tvalid) {
          float o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float acc = fmaf(hpre[jj], gv[e], d1[e]);
#pragma unroll
            for (int i2 = 0; i2 < N; ++i2) acc = fmaf(hres[i2 * N + jj], Gv[i2][e], acc);
            o[e] = fmaf(-kap, xv[e], acc);
          }
#pragma unroll
          for (int v8 = 0; v8 < 2; ++v8) {
            if (cbase + 8 * v8 < a.C) {
              uint4 pk = make_uint4(pack2(o[8 * v8], o[8 * v8 + 1]), pack2(o[8 * v8 + 2], o[8 * v8 + 3]),
                                    pack2(o[8 * v8 + 4], o[8 * v8 + 5]), pack2(o[8 * v8 + 6], o[8 * v8 + 7]));
              __stcs(reinterpret_cast<uint4*>(a.grad_x + (t * N + jj) * a.C + cbase + 8 * v8), pk);
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0 && live) {
        tc::mbar_arrive(bar(B_D1FREE + b));
        tc::mbar_arrive(bar(B_SFREE + s));
      }
      rotate();

      if (seg_last(it)) {
        // ---- flush this segment's grad_phi rows
        if (live && !tc::mbar_wait(bar(B_SEGDONE), (uint32_t)seg & 1u, abort_flag, WAIT_NS)) {
          give_up();
          live = false;
        }
        tc::tc_fence_after();
        // D2 row tok (phi row j*32 + c of the slice); h = 0 reads m' 0..31 (u_hi),
        // h = 1 reads m' 32..63 (u_lo); the two halves meet in shared memory.
        float dd[16], dd2[16];
        if (live) {
          tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + D2_COL + 32 * h, dd);
          tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + D2_COL + 32 * h + 16, dd2);
          tc::tmem_ld_wait();
        }
        if (live && h == 1) {
#pragma unroll
          for (int m = 0; m < M; ++m) xch[tok * M + m] = m < 16 ? dd[m] : dd2[m - 16];
        }
        named_bar_sync(1, 256);
        const int j = tok / CS, cl = tok % CS;
        const int64_t c = (int64_t)slice * CS + cl;
        // part 0: this CTA holds the slice's first item; part 1: its last items
        const int part_idx = (it - item_tile(it) >= it0) ? 0 : 1;
        const bool whole = (it - item_tile(it) >= it0) && (it == (int64_t)slice * a.NTT + a.NTT - 1);
        float* dst_row = a.grad_phi + ((int64_t)j * a.C + c) * M;
        if (live && h == 0) {
          float sum[M];
#pragma unroll
          for (int m = 0; m < M; ++m) sum[m] = (m < 16 ? dd[m] : dd2[m - 16]) + xch[tok * M + m];
          if (whole) {
            if (c < a.C)
#pragma unroll
              for (int m = 0; m < M; ++m) dst_row[m] = sum[m];
          } else {
            float* pr = a.gphi_part + (((int64_t)slice * 2 + part_idx) * KR + tok) * M;
#pragma unroll
            for (int m = 0; m < M; ++m) __stcg(pr + m, sum[m]);
          }
        }
        if (!whole) {
          __threadfence();
          named_bar_sync(1, 256);
          if (etid == 0) *bcast = live ? atomicAdd(a.gphi_cnt + slice, 1) : -1;
          named_bar_sync(1, 256);
          if (*bcast == 1) {
            // both parts are in memory: add them in part order
            __threadfence();
            if (h == 0 && c < a.C) {
              const float* p0 = a.gphi_part + (((int64_t)slice * 2 + 0) * KR + tok) * M;
              const float* p1 = a.gphi_part + (((int64_t)slice * 2 + 1) * KR + tok) * M;
#pragma unroll
              for (int m = 0; m < M; ++m) dst_row[m] = __ldcg(p0 + m) + __ldcg(p1 + m);
            }
            if (etid == 0) a.gphi_cnt[slice] = 0;
          }
        }
        tc::tc_fence_before();
        named_bar_sync(1, 256);
        ++seg;
        if (i + 1 < nit && live) load_phi(item_slice(it + 1));
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
size_t apply_tc_scratch_bytes(int64_t C) {
  const int64_t S = (C + tcap::CS - 1) / tcap::CS;
  return (size_t)S * 2 * tcap::KR * tcap::M * 4 + (size_t)S * 4 + 256;
}

cudaError_t apply_tc_dispatch(int64_t T, int64_t C, const void* x, const float* phi, const void* G,
                              const void* g, const float* coef, const float* part, int nparts,
                              void* gx, void* gf, float* gphi, float* gb, float* ga,
                              void* scratch, int* st, cudaStream_t s) {
  using namespace tcap;
  int dev = 0, num_sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mG, mg;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {CS, 1, TT};
  e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&mG, G, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return e;
  const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T};
  const uint64_t s2[1] = {(uint64_t)C * 2};
  const uint32_t b2[2] = {CS, TT};
  e = make_tmap_bf16(&mg, g, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return e;

  ApplyArgs a;
  a.T = T;
  a.C = C;
  a.S = (int)((C + CS - 1) / CS);
  a.NTT = (int)((T + TT - 1) / TT);
  a.items = (int64_t)a.S * a.NTT;
  // at most one CTA per slice so that every slice meets at most two CTAs
  const int grid = a.S < num_sms ? a.S : num_sms;
  a.per = (a.items + grid - 1) / grid;
  a.phi = phi;
  a.coef = coef;
  a.part = part;
  a.nparts = nparts;
  a.grad_x = (__nv_bfloat16*)gx;
  a.grad_f = (__nv_bfloat16*)gf;
  a.grad_phi = gphi;
  a.grad_b = gb;
  a.grad_alpha = ga;
  a.gphi_part = (float*)scratch;
  a.gphi_cnt = (int*)((char*)scratch + (size_t)a.S * 2 * KR * M * 4);
  a.status = st;
  e = cudaFuncSetAttribute(k_apply_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  // slice counters start at zero (the combining CTA resets its counter too)
  e = cudaMemsetAsync(a.gphi_cnt, 0, (size_t)a.S * sizeof(int), s);
  if (e != cudaSuccess) return e;
  k_apply_tc<<<grid, NT, SMEM, s>>>(mx, mG, mg, a);
  return cudaGetLastError();
}

}  // namespace mhc
