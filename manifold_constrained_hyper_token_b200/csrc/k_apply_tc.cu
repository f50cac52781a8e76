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
// grad_x.  Everything an item reads arrives by TMA into one pipeline stage:
// the x, grad_x_next and grad_h_in tiles (64-byte swizzle, 64-byte L2 fills:
// the neighbouring half-lines belong to another slice that is read much
// later), the item's U rows as written by the mapping kernel (128-byte
// swizzle; the K-major A of MMA1 and the MN-major B of MMA2) and its H
// records (a contiguous bulk copy).  X is the MN-major A operand of MMA2.
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
constexpr int CS = 16;                // channels per slice: 32-byte rows, 32-byte swizzle
constexpr int KR = N * CS;            // 64 phi rows per slice (MMA2 M, MMA1 N)
constexpr int NU = 64;                // U width: 24 hi + 8 pad + 24 lo + 8 pad
constexpr int NEPI = 8;               // epilogue warps: 2 per TMEM lane quarter
constexpr int CPT = CS / (NEPI / 4);  // channels per epilogue thread (8)
constexpr int VPT = CPT / 8;          // 16-byte vectors per thread per stream row
constexpr int NWARPS = 2 + NEPI;
constexpr int NEPI_T = NEPI * 32;
constexpr int NT = NWARPS * 32;
constexpr int XB = TT * CS * 2;       // one stream's x (or G) tile: 4 KB
constexpr int X_OFF = 0, G_OFF = N * XB, GG_OFF = 2 * N * XB;
constexpr int U_OFF = GG_OFF + XB;              // 36864: U rows of the item, 16 KB
constexpr int U_BYTES = TT * NU * 2;
constexpr int H_OFF = U_OFF + U_BYTES;          // 53248: H records, 14 KB
constexpr int H_BYTES = TT * TcRec::H_BYTES;
constexpr int STAGE = 67584;                    // 66 KB, 1024-aligned
static_assert(H_OFF + H_BYTES <= STAGE, "stage layout");
constexpr int NS = 3;
constexpr int PHI_BYTES = KR * NU * 2;          // 8 KB
constexpr int PHI_OFF = NS * STAGE;             // 202752
constexpr int DATA = PHI_OFF + PHI_BYTES;       // 210944
constexpr int SMEM = DATA + 1024 + 256;
static_assert(KR * M * 4 <= H_BYTES, "the D2 exchange reuses a stage's H region");
constexpr uint32_t TMEM_COLS = 256;           // D1 x2 (2 x 64) + D2 (64)
constexpr uint32_t D2_COL = 2 * KR;
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
__device__ __forceinline__ int sw32(int r, int c) { return r * 32 + ((c ^ ((r >> 2) & 1)) << 4); }
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

struct ApplyArgs {
  int64_t T, C;
  int S;          // slices = ceil(C / 32)
  int NTT;        // token tiles = ceil(T / 128)
  int group;      // CTAs g*c .. g*c+g-1 take slices g*v .. g*v+g-1 of the same items
  int64_t items;  // (S / group) * NTT virtual items
  int64_t per;    // virtual items per CTA group
  const float* phi;     // [nC][24]
  const float* hrec;    // [T][TcRec::H_FLOATS]
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
    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_u,
    const __grid_constant__ CUtensorMap tm_gx, const __grid_constant__ CUtensorMap tm_gf,
    const ApplyArgs a) {
  using namespace tcap;
  using CF = Coef<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DATA);
  // barrier slots
  enum { B_FULL = 0, B_SFREE = NS, B_D1READY = 2 * NS, B_D1FREE = 2 * NS + 2,
         B_SEGREADY = 2 * NS + 4, B_SEGDONE = 2 * NS + 5, B_FIN = 2 * NS + 6, NBARS = 2 * NS + 7 };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* bcast = reinterpret_cast<int*>(tmem_slot + 2);
  auto bar = [&](int i) { return tc::smem_u32(bars + i); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Virtual item v = (virtual slice v / NTT, tile v % NTT).  The `group` CTAs
  // of a slot share the virtual items and take adjacent real slices, so the
  // group's 64-byte pieces of each row (group * 64 bytes in all) are requested
  // at about the same time and reach DRAM as one wide fetch (L2 fills of
  // group * 64 bytes).
  const int cta_slot = (int)(blockIdx.x / a.group);
  const int member = (int)(blockIdx.x % a.group);
  const int64_t it0 = (int64_t)cta_slot * a.per;
  const int64_t it1 = (it0 + a.per < a.items) ? it0 + a.per : a.items;
  const int nit = (int)(it1 > it0 ? it1 - it0 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(bar(B_FULL + s), 1);
      tc::mbar_init(bar(B_SFREE + s), 2);  // MMA commit + release after the stores drained
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(B_D1READY + b), 1);
      tc::mbar_init(bar(B_D1FREE + b), NEPI);
    }
    tc::mbar_init(bar(B_SEGREADY), NEPI);
    tc::mbar_init(bar(B_SEGDONE), 1);
    tc::mbar_init(bar(B_FIN), 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_x);
    tc::tma_prefetch_desc(&tm_G);
    tc::tma_prefetch_desc(&tm_g);
    tc::tma_prefetch_desc(&tm_u);
    tc::tma_prefetch_desc(&tm_gx);
    tc::tma_prefetch_desc(&tm_gf);
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
  auto item_slice = [&](int64_t it) {
    const int vs = (int)(it / a.NTT);
    return a.group * vs + member;
  };
  auto item_tile = [&](int64_t it) { return (int)(it % a.NTT); };
  auto seg_first = [&](int64_t it) { return it == it0 || item_tile(it) == 0; };
  auto seg_last = [&](int64_t it) { return it == it1 - 1 || item_tile(it) == a.NTT - 1; };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0 && nit > 0) {
      const uint64_t pol = tc::policy_evict_first();
      const uint64_t pol_keep = tc::policy_evict_last();  // records: read by every slice
      int issued = 0;
      for (int i = 0; i < nit; ++i) {
        const int s = i % NS;
        if (i >= NS && !tc::mbar_wait(bar(B_SFREE + s), (uint32_t)(i / NS - 1) & 1u, abort_flag,
                                      WAIT_NS)) {
          give_up();
          break;
        }
        const int64_t it = it0 + i;
        const int c0 = item_slice(it) * CS;
        const int tt0 = item_tile(it) * TT;
        const uint32_t base = tc::smem_u32(smem + s * STAGE);
        const int64_t nvalid = (a.T - tt0) < TT ? (a.T - tt0) : TT;
        const uint32_t hbytes = (uint32_t)nvalid * TcRec::H_BYTES;
        tc::mbar_arrive_expect_tx(bar(B_FULL + s), (uint32_t)U_OFF + (uint32_t)U_BYTES + hbytes);
        for (int j = 0; j < N; ++j) {
          tc::tma_load_3d(base + X_OFF + j * XB, &tm_x, bar(B_FULL + s), c0, j, tt0, pol);
          tc::tma_load_3d(base + G_OFF + j * XB, &tm_G, bar(B_FULL + s), c0, j, tt0, pol);
        }
        tc::tma_load_2d(base + GG_OFF, &tm_g, bar(B_FULL + s), c0, tt0, pol);
        tc::tma_load_2d(base + U_OFF, &tm_u, bar(B_FULL + s), 0, tt0, pol_keep);
        tc::bulk_load(base + H_OFF, a.hrec + (int64_t)tt0 * TcRec::H_FLOATS, hbytes, bar(B_FULL + s),
                      pol_keep);
        ++issued;
      }
      if (*abort_flag)
        for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
          tc::mbar_wait(bar(B_FULL + (i % NS)), (uint32_t)(i / NS) & 1u, nullptr, WAIT_NS / 4);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0 && nit > 0) {
      constexpr uint32_t id1 = tc::idesc_bf16(TT, KR);                // K-major U x K-major PHI
      constexpr uint32_t id2 = tc::idesc_bf16(KR, NU, true, true);    // MN-major X x MN-major U (M = 64)
      const uint32_t phi_s = tc::smem_u32(smem + PHI_OFF);
      bool any = false;
      int seg = 0;
      for (int i = 0; i < nit; ++i) {
        const int64_t it = it0 + i;
        const int s = i % NS, b = i & 1;
        const uint32_t sph = (uint32_t)(i / NS) & 1u, bph = (uint32_t)(i >> 1) & 1u;
        bool ok = tc::mbar_wait(bar(B_FULL + s), sph, abort_flag, WAIT_NS);
        if (ok && i >= 2) ok = tc::mbar_wait(bar(B_D1FREE + b), bph ^ 1u, abort_flag, WAIT_NS);
        const bool first = seg_first(it);
        if (ok && first) ok = tc::mbar_wait(bar(B_SEGREADY), (uint32_t)seg & 1u, abort_flag, WAIT_NS);
        if (!ok) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t xs = tc::smem_u32(smem + s * STAGE + X_OFF);
        const uint32_t us = tc::smem_u32(smem + s * STAGE + U_OFF);
        // MMA1: D1[b] = U . PHI^T   (K = 64 over m', 128-byte swizzle, K-major)
#pragma unroll
        for (int k = 0; k < NU / 16; ++k) {
          const uint64_t da = tc::smem_desc(us + k * 32, 16, 1024, tc::SWZ_128B);
          const uint64_t db = tc::smem_desc(phi_s + k * 32, 16, 1024, tc::SWZ_128B);
          tc::mma_bf16(tmem + (uint32_t)(b * KR), da, db, id1, k > 0 ? 1u : 0u);
        }
        // MMA2: D2 += X^T . U   (K = 128 tokens; X MN-major 32-byte swizzle with the
        // four stream tiles 4 KB apart; U MN-major 128-byte swizzle)
#pragma unroll
        for (int k = 0; k < TT / 16; ++k) {
          const uint64_t da = tc::smem_desc(xs + k * 512, XB, 256, tc::SWZ_32B);
          const uint64_t db = tc::smem_desc(us + k * 2048, U_BYTES, 1024, tc::SWZ_128B);
          tc::mma_bf16(tmem + D2_COL, da, db, id2, (first && k == 0) ? 0u : 1u);
        }
        any = true;
        tc::mma_commit(bar(B_D1READY + b));
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
    const int hq = (warp - 2) >> 2;   // channel group: channels CPT*hq .. CPT*hq+CPT-1 of the slice
    const int tok = 32 * q + lane;    // token row within the tile / phi row in D2
    const int etid = threadIdx.x - 64;  // 0 .. NEPI_T-1

    if (blockIdx.x == 0) {
      // grad_b / grad_alpha from the mapping kernel's per-CTA partials, in a fixed order
      float* wsum = reinterpret_cast<float*>(smem + PHI_OFF);  // before PHI is loaded
      const int ew = etid / 32;
      float sacc = 0.0f;
      if (lane <= M)
        for (int p = ew; p < a.nparts; p += NEPI) sacc += __ldg(a.part + (int64_t)p * CF::DZ_SIZE + lane);
      if (lane <= M) wsum[ew * (M + 1) + lane] = sacc;
      named_bar_sync(1, NEPI_T);
      if (etid <= M) {
        float acc = 0.0f;
        for (int w = 0; w < NEPI; ++w) acc += wsum[w * (M + 1) + etid];
        if (etid < M) a.grad_b[etid] = acc;
        else *a.grad_alpha = acc;
      }
      named_bar_sync(1, NEPI_T);
    }

    // PHI for a slice: row r = j*32 + c holds phi_hi[j*C + c0 + c][0..23] in m' 0..23
    // and again in m' 32..55 (zeros elsewhere), 128-byte swizzle.
    auto load_phi = [&](int slice) {
      uint8_t* ps = smem + PHI_OFF;
      for (int e = etid; e < KR * 8; e += NEPI_T) {
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

    int seg = 0;
    if (nit > 0) load_phi(item_slice(it0));
    // The loop never breaks: after a failed wait it keeps walking the items
    // without touching memory, so all eight warps meet every named barrier.
    for (int i = 0; i < nit; ++i) {
      const int64_t it = it0 + i;
      const int s = i % NS, b = i & 1;
      const uint32_t sph = (uint32_t)(i / NS) & 1u, bph = (uint32_t)(i >> 1) & 1u;
      bool live = !*abort_flag;
      if (live && (!tc::mbar_wait(bar(B_FULL + s), sph, abort_flag, WAIT_NS) ||
                   !tc::mbar_wait(bar(B_D1READY + b), bph, abort_flag, WAIT_NS))) {
        give_up();
        live = false;
      }
      live = __all_sync(0xffffffffu, live);  // TMEM loads below are warp-collective
      tc::tc_fence_after();
      const int slice = item_slice(it);
      uint8_t* st = smem + s * STAGE;
      // this token's H record
      float hres[N * N], hpre[N], hpost[N], kap;
      {
        const float4* hr = reinterpret_cast<const float4*>(st + H_OFF + tok * TcRec::H_BYTES);
        float rec[TcRec::H_FLOATS];
#pragma unroll
        for (int e = 0; e < TcRec::H_FLOATS / 4; ++e) {
          const float4 v = hr[e];
          rec[4 * e] = v.x; rec[4 * e + 1] = v.y; rec[4 * e + 2] = v.z; rec[4 * e + 3] = v.w;
        }
#pragma unroll
        for (int e = 0; e < N * N; ++e) hres[e] = rec[TcRec::H_RES + e];
#pragma unroll
        for (int e = 0; e < N; ++e) {
          hpre[e] = rec[TcRec::H_PRE + e];
          hpost[e] = rec[TcRec::H_POST + e];
        }
        kap = rec[TcRec::H_KAPPA];
      }
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int chunk = VPT * hq + v;            // 16-byte chunk of the 32-byte tile row
        // phi u of the four output streams for these 8 channels: four TMEM loads,
        // one wait (warp-collective: every lane takes part, whatever its token)
        float d1[N][8];
        if (live) {
#pragma unroll
          for (int jj = 0; jj < N; ++jj)
            tc::tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * KR + jj * CS + 8 * chunk),
                         d1[jj]);
        }
        float Gv[N][8], gv[8], xv[N][8];
#pragma unroll
        for (int i2 = 0; i2 < N; ++i2) {
          unpack8(*reinterpret_cast<const uint4*>(st + G_OFF + i2 * XB + sw32(tok, chunk)), Gv[i2]);
          unpack8(*reinterpret_cast<const uint4*>(st + X_OFF + i2 * XB + sw32(tok, chunk)), xv[i2]);
        }
        unpack8(*reinterpret_cast<const uint4*>(st + GG_OFF + sw32(tok, chunk)), gv);
        if (live) tc::tmem_ld_wait();
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float acc = 0.0f;
#pragma unroll
          for (int i2 = 0; i2 < N; ++i2) acc = fmaf(hpost[i2], Gv[i2][e], acc);
          o[e] = acc;
        }
        // grad_f_out replaces this thread's grad_h_in piece in the stage (the
        // same swizzled position), for the tile store below
        *reinterpret_cast<uint4*>(st + GG_OFF + sw32(tok, chunk)) =
            make_uint4(pack2(o[0], o[1]), pack2(o[2], o[3]), pack2(o[4], o[5]), pack2(o[6], o[7]));
#pragma unroll
        for (int jj = 0; jj < N; ++jj) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float acc = fmaf(hpre[jj], gv[e], d1[jj][e]);
#pragma unroll
            for (int i2 = 0; i2 < N; ++i2) acc = fmaf(hres[i2 * N + jj], Gv[i2][e], acc);
            o[e] = fmaf(-kap, xv[jj][e], acc);
          }
          // grad_x replaces this thread's x piece of stream jj in the stage
          *reinterpret_cast<uint4*>(st + X_OFF + jj * XB + sw32(tok, chunk)) =
              make_uint4(pack2(o[0], o[1]), pack2(o[2], o[3]), pack2(o[4], o[5]), pack2(o[6], o[7]));
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      const bool last = seg_last(it);
      if (lane == 0 && live) tc::mbar_arrive(bar(B_D1FREE + b));
      // Outputs are in the stage; once every warp has written its part, one
      // thread stores the item's tiles (clipped at T and C).  The stage is
      // released one item later, after those stores finished reading it.
      tc::fence_proxy_async_smem();
      named_bar_sync(1, NEPI_T);
      if (etid == 0 && live) {
        const int c0 = slice * CS, tt0 = item_tile(it) * TT;
        const uint32_t sb = tc::smem_u32(st);
#pragma unroll
        for (int jj = 0; jj < N; ++jj) tc::tma_store_3d(&tm_gx, sb + X_OFF + jj * XB, c0, jj, tt0);
        tc::tma_store_2d(&tm_gf, sb + GG_OFF, c0, tt0);
        tc::bulk_commit();
        if (i > 0) {
          tc::bulk_wait_read<1>();
          tc::mbar_arrive(bar(B_SFREE + (i - 1) % NS));
        }
      }

      if (last) {
        // ---- flush this segment's grad_phi rows.  Every warp has finished
        // reading this stage's H records before any overwrites them.
        named_bar_sync(1, NEPI_T);
        float* xch = reinterpret_cast<float*>(smem + s * STAGE + H_OFF);  // [KR][M]: the u_lo part
        if (live && !tc::mbar_wait(bar(B_SEGDONE), (uint32_t)seg & 1u, abort_flag, WAIT_NS)) {
          give_up();
          live = false;
        }
        live = __all_sync(0xffffffffu, live);
        tc::tc_fence_after();
        // D2 row tok (phi row j*32 + c of the slice): hq = 0 reads m' 0..31 (the
        // u_hi part), hq = 1 reads m' 32..63 (the u_lo part); they meet in smem.
        // D2 is an M = 64 accumulator: phi row 16q + l of the slice sits in lane
        // 32q + l (l < 16); lanes 16..31 of each quarter hold no row.
        float dd[32];
        if (live) {
          float t16[16];
          tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + D2_COL + 32 * hq, t16);
#pragma unroll
          for (int e = 0; e < 16; ++e) dd[e] = t16[e];
          tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + D2_COL + 32 * hq + 16, t16);
#pragma unroll
          for (int e = 0; e < 16; ++e) dd[16 + e] = t16[e];
          tc::tmem_ld_wait();
        }
        const int prow = 16 * q + lane;          // phi row of the slice held by this lane
        const bool has_row = lane < 16;
        if (live && hq == 1 && has_row) {
#pragma unroll
          for (int m = 0; m < M; ++m) xch[prow * M + m] = dd[m];
        }
        named_bar_sync(1, NEPI_T);
        const int j = prow / CS, cl = prow % CS;
        const int64_t c = (int64_t)slice * CS + cl;
        // part 0: this CTA holds the slice's first item; part 1: its last items
        const int part_idx = (it - item_tile(it) >= it0) ? 0 : 1;
        const bool whole = (it - item_tile(it) >= it0) && (item_tile(it) == a.NTT - 1);
        float* dst_row = a.grad_phi + ((int64_t)j * a.C + c) * M;
        if (live && hq == 0 && has_row) {
          float sum[M];
#pragma unroll
          for (int m = 0; m < M; ++m) sum[m] = dd[m] + xch[prow * M + m];
          if (whole) {
            if (c < a.C) {
#pragma unroll
              for (int m = 0; m < M; ++m) dst_row[m] = sum[m];
            }
          } else {
            float* pr = a.gphi_part + (((int64_t)slice * 2 + part_idx) * KR + prow) * M;
#pragma unroll
            for (int m = 0; m < M; ++m) __stcg(pr + m, sum[m]);
          }
        }
        if (!whole) {
          __threadfence();
          named_bar_sync(1, NEPI_T);
          if (etid == 0) *bcast = live ? atomicAdd(a.gphi_cnt + slice, 1) : -1;
          named_bar_sync(1, NEPI_T);
          if (*bcast == 1) {
            // both parts are in memory: add them in part order
            __threadfence();
            if (hq == 0 && has_row && c < a.C) {
              const float* p0 = a.gphi_part + (((int64_t)slice * 2 + 0) * KR + prow) * M;
              const float* p1 = a.gphi_part + (((int64_t)slice * 2 + 1) * KR + prow) * M;
#pragma unroll
              for (int m = 0; m < M; ++m) dst_row[m] = __ldcg(p0 + m) + __ldcg(p1 + m);
            }
            if (etid == 0) a.gphi_cnt[slice] = 0;
          }
        }
        tc::tc_fence_before();
        named_bar_sync(1, NEPI_T);
        ++seg;
        if (i + 1 < nit && live) load_phi(item_slice(it + 1));
      }
    }
  }

  if (warp >= 2 && threadIdx.x == 64) tc::bulk_wait<0>();  // the store thread's last tiles
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
                              const void* g, const void* urec, const float* hrec, const float* part,
                              int nparts, void* gx, void* gf, float* gphi, float* gb, float* ga,
                              void* scratch, int* st, cudaStream_t s) {
  using namespace tcap;
  int dev = 0, num_sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mG, mg, mu;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {CS, 1, TT};
  const int S = (int)((C + CS - 1) / CS);
  int group = 1;
  // A group of 4 requests 4 x 32 = 128 contiguous bytes of each row at about
  // the same time (measured: 32-byte rows 2.15 ms, 64 B 1.17 ms, 128 B 0.95 ms,
  // 256 B 0.98 ms at T = 16384, C = 7168).
  for (int gsz : {4, 2})
    if (S % gsz == 0 && num_sms >= gsz && group == 1) group = gsz;
  const CUtensorMapL2promotion promo = group == 4   ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                       : CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
  e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_32B, promo);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&mG, G, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_32B, promo);
  if (e != cudaSuccess) return e;
  const uint64_t d2[2] = {(uint64_t)C, (uint64_t)T};
  const uint64_t s2[1] = {(uint64_t)C * 2};
  const uint32_t b2[2] = {CS, TT};
  e = make_tmap_bf16(&mg, g, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_32B, promo);
  if (e != cudaSuccess) return e;
  const uint64_t du[2] = {(uint64_t)NU, (uint64_t)T};
  const uint64_t su[1] = {(uint64_t)NU * 2};
  const uint32_t bu[2] = {NU, TT};
  e = make_tmap_bf16(&mu, urec, 2, du, su, bu, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  CUtensorMap mgx, mgf;
  e = make_tmap_bf16(&mgx, gx, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_32B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&mgf, gf, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_32B);
  if (e != cudaSuccess) return e;

  ApplyArgs a;
  a.T = T;
  a.C = C;
  a.S = S;
  a.NTT = (int)((T + TT - 1) / TT);
  a.group = group;
  const int vslices = S / group;
  a.items = (int64_t)vslices * a.NTT;
  // at most one CTA group per virtual slice, so every slice meets at most two CTAs
  const int slots_max = num_sms / group;
  const int slots = vslices < slots_max ? vslices : slots_max;
  a.per = (a.items + slots - 1) / slots;
  const int grid = group * slots;
  a.phi = phi;
  a.hrec = hrec;
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
  k_apply_tc<<<grid, NT, SMEM, s>>>(mx, mG, mg, mu, mgx, mgf, a);
  return cudaGetLastError();
}

}  // namespace mhc
