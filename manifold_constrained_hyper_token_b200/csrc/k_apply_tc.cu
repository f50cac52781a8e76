// k_apply_tc.cu -- second phase of the mHC backward on the tensor cores
// (bf16 activations, n = 4).  From the per-token records of the mapping
// kernel (H_res, H_pre, H_post, kappa, and u = alpha dz / r as bf16 high and
// low parts) it writes
//
//   grad_x[j][c]   = (phi u)[jC+c] + sum_i H_res[i][j] G[i][c] + H_pre[j] g[c] - kappa x[j][c]
//   grad_f_out[c]  = sum_i H_post[i] G[i][c]
//   grad_phi[k][m] = sum_t x_t[k] u_t[m]
//
// (reverse mode of the update equation of the chatgpz.de explainer and of the
// RMS-normalised projection; reportify.cn [19]-[21]).
//
// Work item = (slice of 16 channels x 4 streams = 64 rows of phi, tile of 128
// tokens).  Per item:
//   MMA1  D1[tok][k] = U[tok][m'] x PHI[k][m']        phi u for grad_x (M=128, N=64)
//   MMA2  D2[k][m'] += X[tok][k]^T x U[tok][m']        grad_phi over tokens (M=64, N=64)
// U is [u_hi | 0 | u_lo | 0] (m' = 0..63); D1 = (u_hi + u_lo) . phi_hi, and
// D2's two halves add to x . u with u to ~16 bits (x is exact).
//
// Schedule ("lock-step"): every CTA owns P fixed slices for all token tiles
// and walks the tiles in order, so at any time all CTAs read the same 128
// token rows and together cover whole rows -- DRAM sees long runs instead of
// scattered 32-byte pieces.  The P grad_phi accumulators stay in TMEM for the
// whole kernel.  The E = S - P * grid leftover slices are spread item by item
// over the CTAs (round robin within each tile row); each such item flushes its
// own partial, and the last of a slice's NTT partials adds them in tile order.
// All sums are in a fixed order: repeated calls give identical bits.
//
// Everything an item reads arrives by TMA into one stage: x, grad_x_next and
// grad_h_in tiles (32-byte swizzle), the item's U rows (128-byte swizzle, the
// K-major A of MMA1 and the MN-major B of MMA2), its H records (bulk copy) and
// the phi rows of the slice from the bf16 split copy of phi^T (MN-major B of
// MMA1).  Outputs are written into the consumed x / grad_h_in tiles and stored
// with TMA.  Waits are bounded; on timeout the kernel records MHC_ERR_TIMEOUT,
// drains, frees TMEM and returns.
#include "mhc_common.cuh"
#include "mhc_dispatch.h"
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
constexpr int NWARPS = 2 + NEPI + 1;  // TMA loads, MMA, epilogue x8, TMA stores
constexpr int STORE_WARP = 2 + NEPI;
constexpr int NT = NWARPS * 32;
constexpr int NEPI_T = NEPI * 32;
constexpr int PMAX = 3;               // slices owned for all tiles (TMEM accumulators)
constexpr int XB = TT * CS * 2;       // one stream's x (or G) tile: 4 KB
constexpr int X_OFF = 0, G_OFF = N * XB, GG_OFF = 2 * N * XB;
constexpr int U_OFF = GG_OFF + XB;              // 36864: the item's U rows, 16 KB
constexpr int U_BYTES = TT * NU * 2;
constexpr int H_OFF = U_OFF + U_BYTES;          // 53248: H records, 14 KB
constexpr int H_BYTES = TT * TcRec::H_BYTES;
constexpr int PHI_OFF = H_OFF + H_BYTES;        // 67584: phi^T rows m = 0..31, 4 x 1 KB
constexpr int PHI_M = 32;
constexpr int PB = PHI_M * CS * 2;              // one stream's phi tile: 1 KB
constexpr int STAGE = PHI_OFF + N * PB;         // 71680 (70 KB)
constexpr int NS = 3;
constexpr int DATA = NS * STAGE;                // 215040
constexpr int XCH_OFF = DATA;                   // grad_phi row exchange [KR][M] floats, 6 KB
constexpr int MISC_OFF = XCH_OFF + KR * M * 4;  // barriers, flags, bias scratch
constexpr int MISC = 1280;
constexpr int SMEM = MISC_OFF + MISC + 1024;
static_assert(STAGE % 1024 == 0 && U_OFF % 1024 == 0, "stage alignment");
constexpr uint32_t TMEM_COLS = 512;             // D1 x2 | D2 primaries x PMAX | D2 extra
constexpr uint32_t D2_COL = 2 * KR;             // 128
constexpr uint32_t D2X_COL = D2_COL + PMAX * NU;  // 320
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
__device__ __forceinline__ void unpack_pairs(uint4 q, uint64_t (&v)[4]) {
  v[0] = bf2_to_f2(q.x);
  v[1] = bf2_to_f2(q.y);
  v[2] = bf2_to_f2(q.z);
  v[3] = bf2_to_f2(q.w);
}

// 16-byte chunk c of row r of a tile with 32-byte rows, 32-byte swizzle.
__device__ __forceinline__ int sw32(int r, int c) { return r * 32 + ((c ^ ((r >> 2) & 1)) << 4); }

struct ApplyArgs {
  int64_t T, C;
  int S;          // slices = ceil(C / 16)
  int NTT;        // token tiles = ceil(T / 128)
  int P;          // slices each CTA owns for all tiles (<= PMAX)
  int E;          // leftover slices, spread item by item
  int grid;       // CTAs
  const float* hrec;    // [T][TcRec::H_FLOATS]
  const float* part;    // bias / alpha partials of the mapping kernel
  int nparts;
  float* grad_phi;
  float* grad_b;
  float* grad_alpha;
  float* xpart;   // [E][NTT][KR][M] partials of the leftover slices
  int* xcnt;      // [E]
  int* status;
  int write_gf;   // 0: grad_f_out is not produced (pre half of the split backward)
  int ag;         // 3: grad_alpha per group (pre, post, res); else one shared alpha
  uint64_t wait_ns;  // limit of every wait on another warp's or the copy engine's progress
};

// Walks one CTA's items: for every tile t its P owned slices, then the
// leftover items of row t that fall to it (leftover slice k goes to CTA
// (t*E + k) mod grid).
struct ItemCursor {
  int t, p;       // p < P: owned slice p;  p >= P: leftover number p - P of this row
  __device__ __forceinline__ int first_extra(const ApplyArgs& a, int b) const {
    if (a.E == 0) return 0;
    int k0 = (int)(((int64_t)b - (int64_t)t * a.E) % a.grid);
    if (k0 < 0) k0 += a.grid;
    return k0;
  }
  __device__ __forceinline__ int extras(const ApplyArgs& a, int b) const {
    if (a.E == 0) return 0;
    const int k0 = first_extra(a, b);
    return k0 >= a.E ? 0 : (a.E - 1 - k0) / a.grid + 1;
  }
  __device__ __forceinline__ void skip_empty(const ApplyArgs& a, int b) {
    while (t < a.NTT && p >= a.P + extras(a, b)) {
      ++t;
      p = 0;
    }
  }
  __device__ __forceinline__ void start(const ApplyArgs& a, int b) {
    t = 0;
    p = 0;
    skip_empty(a, b);
  }
  __device__ __forceinline__ bool valid(const ApplyArgs& a) const { return t < a.NTT; }
  __device__ __forceinline__ void next(const ApplyArgs& a, int b) {
    ++p;
    skip_empty(a, b);
  }
  __device__ __forceinline__ bool is_extra(const ApplyArgs& a) const { return p >= a.P; }
  // leftover slice number (0..E-1) of a leftover item
  __device__ __forceinline__ int extra_k(const ApplyArgs& a, int b) const {
    return first_extra(a, b) + (p - a.P) * a.grid;
  }
  __device__ __forceinline__ int slice(const ApplyArgs& a, int b) const {
    return is_extra(a) ? a.P * a.grid + extra_k(a, b) : b * a.P + p;
  }
};

__global__ void __launch_bounds__(tcap::NT, 1) k_apply_tc(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_G,
    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_u,
    const __grid_constant__ CUtensorMap tm_phi, const __grid_constant__ CUtensorMap tm_gx,
    const __grid_constant__ CUtensorMap tm_gf, const ApplyArgs a) {
  using namespace tcap;
  using CF = Coef<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + MISC_OFF);
  enum { B_FULL = 0, B_SFREE = NS, B_OUTREADY = 2 * NS, B_D1READY = 3 * NS,
         B_D1FREE = 3 * NS + 2, B_XDONE = 3 * NS + 4, B_XFREE = 3 * NS + 5, B_DONE = 3 * NS + 6,
         B_FIN = 3 * NS + 7, NBARS = 3 * NS + 8 };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* bcast = reinterpret_cast<int*>(tmem_slot + 2);
  float* wsum = reinterpret_cast<float*>(smem + MISC_OFF + 256);  // [NEPI + 1][M + 3], bias sums
  float* xch = reinterpret_cast<float*>(smem + XCH_OFF);           // [KR][M], u_lo halves
  auto bar = [&](int i) { return tc::smem_u32(bars + i); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(bar(B_FULL + s), 1);
      tc::mbar_init(bar(B_SFREE + s), 2);     // MMA commit + store warp after its stores drained
      tc::mbar_init(bar(B_OUTREADY + s), NEPI);  // every epilogue warp wrote its outputs
    }
    for (int k = 0; k < 2; ++k) {
      tc::mbar_init(bar(B_D1READY + k), 1);
      tc::mbar_init(bar(B_D1FREE + k), NEPI);
    }
    tc::mbar_init(bar(B_XDONE), 1);
    tc::mbar_init(bar(B_XFREE), NEPI);
    tc::mbar_init(bar(B_DONE), 1);
    tc::mbar_init(bar(B_FIN), 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_x);
    tc::tma_prefetch_desc(&tm_G);
    tc::tma_prefetch_desc(&tm_g);
    tc::tma_prefetch_desc(&tm_u);
    tc::tma_prefetch_desc(&tm_phi);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      // x / G / g lines are shared with the neighbouring CTAs' slices a moment
      // later (normal priority); records and phi are read by every CTA (keep)
      const uint64_t pol = tc::policy_evict_normal();
      const uint64_t pol_keep = tc::policy_evict_last();
      int i = 0;
      ItemCursor cur;
      for (cur.start(a, b); cur.valid(a); cur.next(a, b), ++i) {
        const int s = i % NS;
        if (i >= NS && !tc::mbar_wait(bar(B_SFREE + s), (uint32_t)(i / NS - 1) & 1u, abort_flag,
                                      a.wait_ns)) {
          give_up();
          break;
        }
        const int c0 = cur.slice(a, b) * CS;
        const int tt0 = cur.t * TT;
        const uint32_t base = tc::smem_u32(smem + s * STAGE);
        const int64_t nvalid = (a.T - tt0) < TT ? (a.T - tt0) : TT;
        const uint32_t hbytes = (uint32_t)nvalid * TcRec::H_BYTES;
        tc::mbar_arrive_expect_tx(bar(B_FULL + s),
                                  (uint32_t)U_OFF + (uint32_t)U_BYTES + hbytes + (uint32_t)(N * PB));
        for (int j = 0; j < N; ++j) {
          tc::tma_load_3d(base + X_OFF + j * XB, &tm_x, bar(B_FULL + s), c0, j, tt0, pol);
          tc::tma_load_3d(base + G_OFF + j * XB, &tm_G, bar(B_FULL + s), c0, j, tt0, pol);
          tc::tma_load_3d(base + PHI_OFF + j * PB, &tm_phi, bar(B_FULL + s), c0, j, 0, pol_keep);
        }
        tc::tma_load_2d(base + GG_OFF, &tm_g, bar(B_FULL + s), c0, tt0, pol);
        tc::tma_load_2d(base + U_OFF, &tm_u, bar(B_FULL + s), 0, tt0, pol_keep);
        tc::bulk_load(base + H_OFF, a.hrec + (int64_t)tt0 * TcRec::H_FLOATS, hbytes, bar(B_FULL + s),
                      pol_keep);
      }
      // every copy issued here has landed before the CTA can exit (after a normal
      // run these waits return at once)
      for (int k = (i > NS ? i - NS : 0); k < i; ++k)
        tc::mbar_wait(bar(B_FULL + (k % NS)), (uint32_t)(k / NS) & 1u, nullptr, tc::kDrainWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      // MMA1: K-major U x MN-major phi tile;  MMA2: MN-major X x MN-major U (M = 64)
      constexpr uint32_t id1 = tc::idesc_bf16(TT, KR, false, true);
      constexpr uint32_t id2 = tc::idesc_bf16(KR, NU, true, true);
      bool any = false;
      int i = 0, nx = 0;
      ItemCursor cur;
      for (cur.start(a, b); cur.valid(a); cur.next(a, b), ++i) {
        const int s = i % NS, d = i & 1;
        const uint32_t sph = (uint32_t)(i / NS) & 1u, dph = (uint32_t)(i >> 1) & 1u;
        const bool extra = cur.is_extra(a);
        bool ok = tc::mbar_wait(bar(B_FULL + s), sph, abort_flag, a.wait_ns);
        if (ok && i >= 2) ok = tc::mbar_wait(bar(B_D1FREE + d), dph ^ 1u, abort_flag, a.wait_ns);
        if (ok && extra && nx > 0)
          ok = tc::mbar_wait(bar(B_XFREE), (uint32_t)(nx - 1) & 1u, abort_flag, a.wait_ns);
        if (!ok) {
          give_up();
          break;
        }
        tc::tc_fence_after();
        const uint32_t st = tc::smem_u32(smem + s * STAGE);
        // MMA1: D1[d] = U . PHI^T.  The phi tile holds rows m = 0..31 of the phi^T
        // split (phi_hi in 0..23); U's columns 24..31 and 56..63 are zero, so
        // K-steps 0,1 (u_hi) and 2,3 (u_lo) both read phi rows 0..31.
#pragma unroll
        for (int k = 0; k < NU / 16; ++k) {
          const uint64_t da = tc::smem_desc(st + U_OFF + k * 32, 16, 1024, tc::SWZ_128B);
          const uint64_t db = tc::smem_desc(st + PHI_OFF + (k & 1) * 512, PB, 256, tc::SWZ_32B);
          tc::mma_bf16(tmem + (uint32_t)(d * KR), da, db, id1, k > 0 ? 1u : 0u);
        }
        // MMA2: D2 += X^T . U over the 128 tokens
        const uint32_t d2 = extra ? D2X_COL : D2_COL + (uint32_t)(cur.p * NU);
        const bool fresh = extra || cur.t == 0;
#pragma unroll
        for (int k = 0; k < TT / 16; ++k) {
          const uint64_t da = tc::smem_desc(st + X_OFF + k * 512, XB, 256, tc::SWZ_32B);
          const uint64_t db = tc::smem_desc(st + U_OFF + k * 2048, U_BYTES, 1024, tc::SWZ_128B);
          tc::mma_bf16(tmem + d2, da, db, id2, (fresh && k == 0) ? 0u : 1u);
        }
        any = true;
        tc::mma_commit(bar(B_D1READY + d));
        tc::mma_commit(bar(B_SFREE + s));
        if (extra) {
          tc::mma_commit(bar(B_XDONE));
          ++nx;
        }
      }
      if (!*abort_flag) tc::mma_commit(bar(B_DONE));
      // every MMA issued here has finished before TMEM is freed
      if (any) {
        tc::mma_commit(bar(B_FIN));
        tc::mbar_wait(bar(B_FIN), 0, nullptr, tc::kDrainWaitNs);
      }
    }
  } else if (warp == STORE_WARP) {
    // ---------------------------------------------------------- TMA stores
    // Stores each item's output tiles once the epilogue has written them into
    // the stage, waits until the stores have read the stage, then releases it.
    if (lane == 0) {
      int i = 0;
      ItemCursor cur;
      for (cur.start(a, b); cur.valid(a); cur.next(a, b), ++i) {
        const int s = i % NS;
        if (!tc::mbar_wait(bar(B_OUTREADY + s), (uint32_t)(i / NS) & 1u, abort_flag, a.wait_ns)) {
          give_up();
          break;
        }
        const int c0 = cur.slice(a, b) * CS, tt0 = cur.t * TT;
        const uint32_t sb = tc::smem_u32(smem + s * STAGE);
#pragma unroll
        for (int jj = 0; jj < N; ++jj) tc::tma_store_3d(&tm_gx, sb + X_OFF + jj * XB, c0, jj, tt0);
        if (a.write_gf) tc::tma_store_2d(&tm_gf, sb + GG_OFF, c0, tt0);
        tc::bulk_commit();
        tc::bulk_wait_read<0>();
        tc::mbar_arrive(bar(B_SFREE + s));
      }
      tc::bulk_wait<0>();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quarter
    const int hq = (warp - 2) >> 2;   // channels 8*hq .. 8*hq+7 of the slice
    const int tok = 32 * q + lane;    // token row of the tile
    const int etid = threadIdx.x - 64;
    const int prow = 16 * q + lane;   // phi row of a slice held by this lane in an M=64 D2
    const bool has_row = lane < 16;

    if (b == 0) {
      // grad_b / grad_alpha from the mapping kernel's per-CTA partials, in a fixed order
      // columns: M dz sums, then dz . y over the pre, post and res logits
      constexpr int NC = M + 3;
      const int ew = etid / 32;
      float sacc = 0.0f;
      if (lane < NC)
        for (int p = ew; p < a.nparts; p += NEPI) sacc += __ldg(a.part + (int64_t)p * CF::DZ_SIZE + lane);
      if (lane < NC) wsum[ew * NC + lane] = sacc;
      named_bar_sync(1, NEPI_T);
      if (etid < NC) {
        float acc = 0.0f;
        for (int w = 0; w < NEPI; ++w) acc += wsum[w * NC + etid];
        wsum[NEPI * NC + etid] = acc;
        if (etid < M) a.grad_b[etid] = acc;
        else if (a.ag == 3) a.grad_alpha[etid - M] = acc;
      }
      named_bar_sync(1, NEPI_T);
      // one shared alpha: its gradient is the sum of the three group sums
      if (a.ag != 3 && etid == 0)
        *a.grad_alpha = (wsum[NEPI * NC + M] + wsum[NEPI * NC + M + 1]) + wsum[NEPI * NC + M + 2];
    }

    // Read one M = 64 grad_phi accumulator (phi row 16q + l in lane 32q + l,
    // l < 16) and write row sums u_hi part + u_lo part: hq = 0 holds m' 0..31,
    // hq = 1 m' 32..63; they meet in `xch`.  Returns through `out` for hq = 0.
    auto read_d2 = [&](uint32_t col, bool live, float* xch, float (&out)[M]) {
      float dd[32];
      if (live) {
        float t16[16];
        tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + col + 32 * hq, t16);
#pragma unroll
        for (int e = 0; e < 16; ++e) dd[e] = t16[e];
        tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + col + 32 * hq + 16, t16);
#pragma unroll
        for (int e = 0; e < 16; ++e) dd[16 + e] = t16[e];
        tc::tmem_ld_wait();
      }
      if (live && hq == 1 && has_row) {
#pragma unroll
        for (int m = 0; m < M; ++m) xch[prow * M + m] = dd[m];
      }
      tc::tc_fence_before();
      named_bar_sync(1, NEPI_T);
      if (live && hq == 0 && has_row) {
#pragma unroll
        for (int m = 0; m < M; ++m) out[m] = dd[m] + xch[prow * M + m];
      }
    };

    int i = 0, nx = 0;
    ItemCursor cur;
    // The loop never breaks: after a failed wait it keeps walking the items
    // without touching memory, so all eight warps meet every named barrier.
    for (cur.start(a, b); cur.valid(a); cur.next(a, b), ++i) {
      const int s = i % NS, d = i & 1;
      const uint32_t sph = (uint32_t)(i / NS) & 1u, dph = (uint32_t)(i >> 1) & 1u;
      bool live = !*abort_flag;
      if (live && !tc::mbar_wait(bar(B_FULL + s), sph, abort_flag, a.wait_ns)) {
        give_up();
        live = false;
      }
      const int slice = cur.slice(a, b);
      uint8_t* st = smem + s * STAGE;
      const int chunk = hq;  // 16-byte chunk of the 32-byte tile row
      // Everything but phi u comes from the stage: compute it while the MMA for
      // this item may still run, then add phi u from TMEM at the end.
      uint64_t acc[N][4];
      {
        uint64_t hres2[N * N], hpre2[N], hpost2[N], nkap2;
        {
          const float4* hr = reinterpret_cast<const float4*>(st + H_OFF + tok * TcRec::H_BYTES);
          float rec[TcRec::H_FLOATS];
#pragma unroll
          for (int e = 0; e < TcRec::H_FLOATS / 4; ++e) {
            const float4 v = hr[e];
            rec[4 * e] = v.x; rec[4 * e + 1] = v.y; rec[4 * e + 2] = v.z; rec[4 * e + 3] = v.w;
          }
#pragma unroll
          for (int e = 0; e < N * N; ++e)
            hres2[e] = f2pack(rec[TcRec::H_RES + e], rec[TcRec::H_RES + e]);
#pragma unroll
          for (int e = 0; e < N; ++e) {
            hpre2[e] = f2pack(rec[TcRec::H_PRE + e], rec[TcRec::H_PRE + e]);
            hpost2[e] = f2pack(rec[TcRec::H_POST + e], rec[TcRec::H_POST + e]);
          }
          nkap2 = f2pack(-rec[TcRec::H_KAPPA], -rec[TcRec::H_KAPPA]);
        }
        uint64_t Gp[N][4], gp[4];
#pragma unroll
        for (int i2 = 0; i2 < N; ++i2)
          unpack_pairs(*reinterpret_cast<const uint4*>(st + G_OFF + i2 * XB + sw32(tok, chunk)), Gp[i2]);
        unpack_pairs(*reinterpret_cast<const uint4*>(st + GG_OFF + sw32(tok, chunk)), gp);
        // grad_f_out = sum_i H_post[i] G_i; it replaces this thread's grad_h_in
        // piece in the stage (same swizzled position) for the tile store
        if (a.write_gf && live) {
          uint32_t w[4];
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            uint64_t f = f2pack(0.0f, 0.0f);
#pragma unroll
            for (int i2 = 0; i2 < N; ++i2) f = f2fma(hpost2[i2], Gp[i2][pr], f);
            w[pr] = f2_to_bf2(f);
          }
          *reinterpret_cast<uint4*>(st + GG_OFF + sw32(tok, chunk)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // grad_x_j without phi u: H_pre[j] g + sum_i H_res[i][j] G_i - kappa x_j
#pragma unroll
        for (int jj = 0; jj < N; ++jj) {
          uint64_t xp[4];
          unpack_pairs(*reinterpret_cast<const uint4*>(st + X_OFF + jj * XB + sw32(tok, chunk)), xp);
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            uint64_t v = f2fma(hpre2[jj], gp[pr], f2pack(0.0f, 0.0f));
#pragma unroll
            for (int i2 = 0; i2 < N; ++i2) v = f2fma(hres2[i2 * N + jj], Gp[i2][pr], v);
            acc[jj][pr] = f2fma(nkap2, xp[pr], v);
          }
        }
      }
      if (live && !tc::mbar_wait(bar(B_D1READY + d), dph, abort_flag, a.wait_ns)) {
        give_up();
        live = false;
      }
      live = __all_sync(0xffffffffu, live);  // the TMEM loads below are warp-collective
      tc::tc_fence_after();
      {
        // phi u of the four output streams for these 8 channels
        float d1[N][8];
        if (live) {
#pragma unroll
          for (int jj = 0; jj < N; ++jj)
            tc::tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(d * KR + jj * CS + 8 * chunk),
                         d1[jj]);
          tc::tmem_ld_wait();
        }
#pragma unroll
        for (int jj = 0; jj < N; ++jj) {
          uint32_t w[4];
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            float lo, hi;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[jj][pr]));
            w[pr] = pack2(lo + d1[jj][2 * pr], hi + d1[jj][2 * pr + 1]);
          }
          if (live)
            *reinterpret_cast<uint4*>(st + X_OFF + jj * XB + sw32(tok, chunk)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0 && live) tc::mbar_arrive(bar(B_D1FREE + d));
      // hand the outputs to the store warp (clipped at T and C by the TMA store)
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && live) tc::mbar_arrive(bar(B_OUTREADY + s));

      if (cur.is_extra(a)) {
        // ---- a leftover slice's item: flush its partial; the last of the
        // slice's NTT partials to arrive adds them in tile order.
        if (live && !tc::mbar_wait(bar(B_XDONE), (uint32_t)nx & 1u, abort_flag, a.wait_ns)) {
          give_up();
          live = false;
        }
        live = __all_sync(0xffffffffu, live);
        tc::tc_fence_after();
        float sum[M];
        read_d2(D2X_COL, live, xch, sum);
        if (lane == 0 && live) tc::mbar_arrive(bar(B_XFREE));
        const int k = cur.extra_k(a, b);
        if (live && hq == 0 && has_row) {
          float* pr = a.xpart + (((int64_t)k * a.NTT + cur.t) * KR + prow) * M;
#pragma unroll
          for (int m = 0; m < M; ++m) __stcg(pr + m, sum[m]);
        }
        __threadfence();
        named_bar_sync(1, NEPI_T);
        if (etid == 0) *bcast = live ? atomicAdd(a.xcnt + k, 1) : -1;
        named_bar_sync(1, NEPI_T);
        if (*bcast == a.NTT - 1) {
          __threadfence();
          const int j = prow / CS, cl = prow % CS;
          const int64_t c = (int64_t)slice * CS + cl;
          if (hq == 0 && has_row && c < a.C) {
            float acc[M];
#pragma unroll
            for (int m = 0; m < M; ++m) acc[m] = 0.0f;
            for (int t2 = 0; t2 < a.NTT; ++t2) {
              const float* pr = a.xpart + (((int64_t)k * a.NTT + t2) * KR + prow) * M;
#pragma unroll
              for (int m = 0; m < M; ++m) acc[m] += __ldcg(pr + m);
            }
            float* dst = a.grad_phi + ((int64_t)j * a.C + c) * M;
#pragma unroll
            for (int m = 0; m < M; ++m) dst[m] = acc[m];
          }
          if (etid == 0) a.xcnt[k] = 0;
        }
        named_bar_sync(1, NEPI_T);
        ++nx;
      }
    }

    // ---- the owned slices' grad_phi rows, accumulated over every tile
    bool live = !*abort_flag && tc::mbar_wait(bar(B_DONE), 0, abort_flag, a.wait_ns);
    if (!live && !*abort_flag) give_up();
    live = __all_sync(0xffffffffu, live);
    named_bar_sync(1, NEPI_T);
    tc::tc_fence_after();
    for (int p = 0; p < a.P; ++p) {
      float sum[M];
      read_d2(D2_COL + (uint32_t)(p * NU), live, xch, sum);
      const int slice = b * a.P + p;
      const int j = prow / CS, cl = prow % CS;
      const int64_t c = (int64_t)slice * CS + cl;
      if (live && hq == 0 && has_row && c < a.C) {
        float* dst = a.grad_phi + ((int64_t)j * a.C + c) * M;
#pragma unroll
        for (int m = 0; m < M; ++m) dst[m] = sum[m];
      }
      named_bar_sync(1, NEPI_T);
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
struct ApplyPlan {
  int S, NTT, P, E, grid;
};

static ApplyPlan apply_plan(int64_t T, int64_t C, int num_sms) {
  using namespace tcap;
  ApplyPlan pl;
  pl.S = (int)((C + CS - 1) / CS);
  pl.NTT = (int)((T + TT - 1) / TT);
  pl.grid = pl.S < num_sms ? pl.S : num_sms;
  pl.P = pl.S / pl.grid;
  if (pl.P > PMAX) pl.P = PMAX;
  pl.E = pl.S - pl.P * pl.grid;
  return pl;
}

static int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

size_t apply_tc_scratch_bytes(int64_t T, int64_t C) {
  const ApplyPlan pl = apply_plan(T, C, device_sms());
  return (size_t)pl.E * pl.NTT * tcap::KR * tcap::M * 4 + (size_t)pl.E * 4 + 256;
}

cudaError_t apply_tc_dispatch(int64_t T, int64_t C, const void* x, const void* phi_split,
                              const void* G, const void* g, const void* urec, const float* hrec,
                              const float* part, int nparts, void* gx, void* gf, float* gphi,
                              float* gb, float* ga, int ag, void* scratch, int* st,
                              int64_t wait_ns, cudaStream_t s) {
  using namespace tcap;
  const ApplyPlan pl = apply_plan(T, C, device_sms());
  CUtensorMap mx, mG, mg, mu, mp, mgx, mgf;
  // all CTAs read the same token rows at the same time: wide L2 fills
  const CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
  const uint64_t dx[3] = {(uint64_t)C, (uint64_t)N, (uint64_t)T};
  const uint64_t sx[2] = {(uint64_t)C * 2, (uint64_t)N * C * 2};
  const uint32_t bx[3] = {CS, 1, TT};
  cudaError_t e = make_tmap_bf16(&mx, x, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_32B, promo);
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
  // phi^T split [48][n][C] bf16: rows m = 0..31 of one stream's 16 channels
  const uint64_t dp[3] = {(uint64_t)C, (uint64_t)N, 48};
  const uint32_t bp[3] = {CS, 1, PHI_M};
  e = make_tmap_bf16(&mp, phi_split, 3, dp, sx, bp, CU_TENSOR_MAP_SWIZZLE_32B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&mgx, gx, 3, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_32B);
  if (e != cudaSuccess) return e;
  if (gf != nullptr) {
    e = make_tmap_bf16(&mgf, gf, 2, d2, s2, b2, CU_TENSOR_MAP_SWIZZLE_32B);
    if (e != cudaSuccess) return e;
  } else {
    mgf = mgx;  // never used: no grad_f_out store is issued
  }

  ApplyArgs a;
  a.T = T;
  a.C = C;
  a.S = pl.S;
  a.NTT = pl.NTT;
  a.P = pl.P;
  a.E = pl.E;
  a.grid = pl.grid;
  a.hrec = hrec;
  a.part = part;
  a.nparts = nparts;
  a.grad_phi = gphi;
  a.grad_b = gb;
  a.grad_alpha = ga;
  a.xpart = (float*)scratch;
  a.xcnt = (int*)((char*)scratch + (size_t)pl.E * pl.NTT * KR * M * 4);
  a.status = st;
  a.write_gf = gf != nullptr ? 1 : 0;
  a.ag = ag;
  a.wait_ns = tc::wait_limit(wait_ns);
  e = cudaFuncSetAttribute(k_apply_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  if (pl.E > 0) {
    // leftover-slice counters start at zero (the combining CTA resets its own)
    e = cudaMemsetAsync(a.xcnt, 0, (size_t)pl.E * sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  k_apply_tc<<<pl.grid, NT, SMEM, s>>>(mx, mG, mg, mu, mp, mgx, mgf, a);
  return cudaGetLastError();
}

}  // namespace mhc
