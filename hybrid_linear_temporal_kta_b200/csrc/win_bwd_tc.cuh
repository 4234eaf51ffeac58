// win_bwd_tc.cuh -- reverse mode of the frame-windowed softmax heads (SWA and DSWA) on the sm_100a
// tensor cores, bf16 in and out, fp32 accumulation.
//
// Operator: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar (SWA and DSWA paragraphs); the pages define only the forward. With P_ts = softmax over
// the visible keys of scale * q_t . k_s, the gradients of L = sum(dO * O) are
//   dP_ts = dO_t . v_s,   D_t = dO_t . o_t,   dS_ts = P_ts (dP_ts - D_t),
//   dQ_t = scale sum_s dS_ts k_s,   dK_s = scale sum_t dS_ts q_t,   dV_s = sum_t P_ts dO_t.
// P is rebuilt from the forward's row log-sum-exp (base 2): P_ts = 2^(scale log2(e) S_ts - lse_t).
//
// Three launches:
//   row_dot_kernel       D_t = dO_t . o_t (one warp per row).
//   win_bwd_dq_kernel    query-major: one CTA per 128-row query tile of a (frame, head, sequence);
//                        per key tile of the window S = Q K^T and dP = dO V^T (SS MMAs), the
//                        softmax warps write dS (bf16) over S in TMEM, then dQ += dS K (TS MMA).
//                        TMEM: S [0,128), dP [128,256), dQ [256,384).
//   win_bwd_dkv_kernel   key-major: one CTA per 128-key tile of a frame g; per query tile of the
//                        frames that see g (g, g + dil, ..., g + (W-1) dil), S^T = K Q^T and
//                        dP^T = V dO^T, the softmax warps write P^T over S^T and dS^T over dP^T,
//                        then dV += P^T dO and dK += dS^T Q (TS MMAs).
//                        TMEM: S^T [0,128), dP^T [128,256), dV [256,384), dK [384,512).
// Both kernels keep their fixed operands (Q and dO, or K and V) in shared memory and stream the
// other pair through a four-slot TMA ring, as the forward does. Every wait is bounded; on a
// timeout the CTA records it and unwinds to free its TMEM.
#pragma once

#include "kta_ptx.cuh"
#include "win_attn_tc.cuh"

namespace kta {

struct WinBwdParams {
  int B, P, F, Htot, H0;
  int W[2], dil[2];
  int n_t;               // 128-row tiles per frame
  int rows_b;            // rows per sequence (F * P)
  long long ld;          // row stride of q, k, v, o, dO, dq, dk, dv (elements)
  float scale, scale_log2;
  const float* lse;      // [B][Htot][rows_b]
  const float* Dt;       // [B][Htot][rows_b]
  __nv_bfloat16* out0;   // dq (dq kernel) or dk (dkv kernel), offset to the first head
  __nv_bfloat16* out1;   // dv (dkv kernel)
};

template <int D>
struct WinBwdSmem {
  static constexpr int BOX = 128 * 64 * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int NSLOT = 4;
  alignas(1024) uint8_t a[NBOX * BOX];          // dq: Q tile; dkv: K tile
  alignas(1024) uint8_t b[NBOX * BOX];          // dq: dO tile; dkv: V tile
  alignas(1024) uint8_t ring[NSLOT][NBOX * BOX];  // dq: K_i, V_i; dkv: Q_n, dO_n
  float st[2][2][128];                          // dkv: lse and D of a query tile's columns
  uint64_t bar_ab, full[NSLOT], empty[NSLOT], bar_s, bar_p, bar_o, bar_fin, bar_st[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t win_bwd_smem_bytes() {
  return sizeof(WinBwdSmem<D>) + 1024;
}

// D_t = dO_t . o_t for every row and head (bf16 in, fp32 out). One warp per (row, head).
template <int D>
__global__ void __launch_bounds__(256) row_dot_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      float* __restrict__ Dt, long long rows,
                                                      int rows_b, int H, long long ld) {
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows * H) return;
  const long long r = w / H;
  const int h = static_cast<int>(w % H);
  constexpr int E = D / 32;
  const __nv_bfloat16* a = o + r * ld + static_cast<long long>(h) * D + lane * E;
  const __nv_bfloat16* g = dout + r * ld + static_cast<long long>(h) * D + lane * E;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) acc = fmaf(__bfloat162float(a[e]), __bfloat162float(g[e]), acc);
#pragma unroll
  for (int s = 16; s; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    const long long b = r / rows_b, t = r % rows_b;
    Dt[(b * H + h) * rows_b + t] = acc;
  }
}

// Issue the 8 (D = 128) or 4 (D = 64) K-steps of X Y^T for two 128-row bf16 tiles in the
// two-box layout (SS form, both K-major).
template <int D>
__device__ __forceinline__ void bwd_issue_ss(uint32_t d_tmem, uint32_t x_base, uint32_t y_base) {
  constexpr int BOX = WinBwdSmem<D>::BOX;
  constexpr uint32_t ID = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
    mma_ss(d_tmem, smem_desc_sw128(x_base + off, 16, 1024), smem_desc_sw128(y_base + off, 16, 1024),
           ID, kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A_tmem (128 x 128, bf16 packed) * Y (128 rows x D, MN-major B operand).
template <int D>
__device__ __forceinline__ void bwd_issue_ts(uint32_t acc_tmem, uint32_t a_tmem, uint32_t y_base,
                                             bool first) {
  constexpr int BOX = WinBwdSmem<D>::BOX;
  constexpr uint32_t ID = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts(acc_tmem, a_tmem + kk * 8, smem_desc_sw128(y_base + kk * 16 * 128, BOX, 1024), ID,
           (!first || kk > 0) ? 1u : 0u);
}

// ---------------------------------------------------------------------------------- dQ
template <int D>
__global__ void __launch_bounds__(256, 1)
    win_bwd_dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                      const __grid_constant__ CUtensorMap tkm, const __grid_constant__ CUtensorMap tvm,
                      const WinBwdParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ uint8_t smem_raw[];
  WinBwdSmem<D>& sm = *reinterpret_cast<WinBwdSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int BOX = WinBwdSmem<D>::BOX, NBOX = WinBwdSmem<D>::NBOX, NSLOT = WinBwdSmem<D>::NSLOT;
  constexpr uint32_t TILE_BYTES = 128 * D * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: query tile qt of frame f (latest frames first), head h, sequence b
  int item = blockIdx.x;
  const int qt = item % p.n_t;
  item /= p.n_t;
  const int b = item % p.B;
  item /= p.B;
  const int h = item % p.Htot;
  item /= p.Htot;
  const int f = p.F - 1 - item;
  const int g = h >= p.H0 ? 1 : 0;
  const int W = p.W[g], dil = p.dil[g];
  const int hk = h;  // the K / V maps cover every head of the launch
  const CUtensorMap* tk = &tkm;
  const CUtensorMap* tv = &tvm;
  const int ntiles = win_num_tiles(f, p.P, W, dil);
  const int q_row0 = b * p.rows_b + f * p.P + qt * 128;
  const int nq = min(128, p.P - qt * 128);

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_ab, 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.bar_s, 1);
    mbar_init(&sm.bar_p, 128);
    mbar_init(&sm.bar_o, 1);
    mbar_init(&sm.bar_fin, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tdo);
      prefetch_tmap(tk);
      prefetch_tmap(tv);
      mbar_arrive_expect_tx(&sm.bar_ab, 2 * TILE_BYTES);
      for (int c = 0; c < NBOX; ++c) {
        tma_load_3d(sm.a + c * BOX, &tq, &sm.bar_ab, c * 64, h, q_row0);
        tma_load_3d(sm.b + c * BOX, &tdo, &sm.bar_ab, c * 64, h, q_row0);
      }
      int issued = 0;
      for (int n = 0; n < 2 * ntiles; ++n) {  // K_{n/2} (n even), V_{n/2} (n odd)
        if (*abort_flag) break;
        const int slot = n % NSLOT, use = n / NSLOT;
        int fr0, off, nv;
        win_tile(n >> 1, f, p.P, W, dil, fr0, off, nv);
        const int krow = (b * p.F + fr0) * p.P + off;
        if (use > 0 && !mbar_wait(&sm.empty[slot], (use - 1) & 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&sm.full[slot], TILE_BYTES);
        const CUtensorMap* tm = (n & 1) ? tv : tk;
        for (int c = 0; c < NBOX; ++c)
          tma_load_3d(sm.ring[slot] + c * BOX, tm, &sm.full[slot], c * 64, hk, krow);
        ++issued;
      }
      mbar_wait(&sm.bar_ab, 0);
      for (int n = issued - NSLOT > 0 ? issued - NSLOT : 0; n < issued; ++n)
        mbar_wait(&sm.full[n % NSLOT], (n / NSLOT) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t tS = sm.tmem_base, tP = sm.tmem_base + 128, tQ = sm.tmem_base + 256;
      const uint32_t a0 = smem_u32(sm.a), b0 = smem_u32(sm.b);
      bool ok = ntiles > 0 && mbar_wait(&sm.bar_ab, 0);
      auto issue_sp = [&](int i) {  // S = Q K_i^T, dP = dO V_i^T
        const int ks = (2 * i) % NSLOT, vs = (2 * i + 1) % NSLOT;
        const uint32_t ph = (i >> 1) & 1;
        if (!mbar_wait(&sm.full[ks], ph) || !mbar_wait(&sm.full[vs], ph)) return false;
        tc_fence_after();
        bwd_issue_ss<D>(tS, a0, smem_u32(sm.ring[ks]));
        bwd_issue_ss<D>(tP, b0, smem_u32(sm.ring[vs]));
        mma_commit(&sm.bar_s);
        mma_commit(&sm.empty[vs]);
        return true;
      };
      if (ok) ok = issue_sp(0);
      for (int i = 0; ok && i < ntiles; ++i) {
        if (*abort_flag || !mbar_wait(&sm.bar_p, i & 1)) { ok = false; break; }
        tc_fence_after();
        const int ks = (2 * i) % NSLOT;
        bwd_issue_ts<D>(tQ, tS, smem_u32(sm.ring[ks]), i == 0);  // dQ += dS K_i
        mma_commit(&sm.empty[ks]);
        if (i + 1 < ntiles && !issue_sp(i + 1)) { ok = false; break; }
      }
      if (ok) mma_commit(&sm.bar_o);
      if (!ok) *abort_flag = 1;
      mma_commit(&sm.bar_fin);
      mbar_wait(&sm.bar_fin, 0);
    }
  } else if (warp >= 4) {
    // softmax warps: thread <-> query row (TMEM lane)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = sm.tmem_base, tP = sm.tmem_base + 128, tQ = sm.tmem_base + 256;
    const long long si = (static_cast<long long>(b) * p.Htot + h) * p.rows_b + f * p.P + qt * 128 +
                         min(row, nq - 1);
    const float lse = p.lse[si], Dr = p.Dt[si];
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int i = 0; ok && i < ntiles; ++i) {
      int fr0, off, nv;
      win_tile(i, f, p.P, W, dil, fr0, off, nv);
      const bool got = !*abort_flag && mbar_wait(&sm.bar_s, i & 1);
      if (!__all_sync(0xffffffffu, got)) { *abort_flag = 1; ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rs[32], rp[32];
        tmem_ld32(tS + lane_off + 32 * c, rs);
        tmem_ld32(tP + lane_off + 32 * c, rp);
        tmem_wait_ld();
        tmem_ld_fence(rs);
        tmem_ld_fence(rp);
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = 32 * c + 2 * j;
          float d0 = ex2_approx(fmaf(__uint_as_float(rs[2 * j]), sl2, -lse)) *
                     (__uint_as_float(rp[2 * j]) - Dr);
          float d1 = ex2_approx(fmaf(__uint_as_float(rs[2 * j + 1]), sl2, -lse)) *
                     (__uint_as_float(rp[2 * j + 1]) - Dr);
          if (nv < 128) {
            d0 = col < nv ? d0 : 0.f;
            d1 = col + 1 < nv ? d1 : 0.f;
          }
          pk[j] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tS + lane_off + 16 * c, pk);  // dS over columns [0, 64) of S, already read
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_p);
    }
    const bool fin = ok && ntiles > 0 && mbar_wait(&sm.bar_o, 0);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      __nv_bfloat16* orow = p.out0 + static_cast<long long>(q_row0 + row) * p.ld + h * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tQ + lane_off + 32 * c, rr);
        tmem_wait_ld();
        tmem_ld_fence(rr);
        if (row < nq) {
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[j] = pack_bf16x2(__uint_as_float(rr[2 * j]) * p.scale, __uint_as_float(rr[2 * j + 1]) * p.scale);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
      }
    } else {
      *abort_flag = 1;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(sm.tmem_base, 512);
  }
}

// Query tiles that see key frame g: tile n covers frame g + (n / n_t) dil, rows from 128 (n % n_t).
__device__ __forceinline__ int dkv_num_tiles(int g, int F, int W, int dil, int n_t) {
  const int nf = min(W, (F - 1 - g) / dil + 1);
  return nf * n_t;
}

// ---------------------------------------------------------------------------------- dK, dV
template <int D>
__global__ void __launch_bounds__(256, 1)
    win_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                       const __grid_constant__ CUtensorMap tkm, const __grid_constant__ CUtensorMap tvm,
                       const WinBwdParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ uint8_t smem_raw[];
  WinBwdSmem<D>& sm = *reinterpret_cast<WinBwdSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int BOX = WinBwdSmem<D>::BOX, NBOX = WinBwdSmem<D>::NBOX, NSLOT = WinBwdSmem<D>::NSLOT;
  constexpr uint32_t TILE_BYTES = 128 * D * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: key tile kt of frame g, head h, sequence b
  int item = blockIdx.x;
  const int kt = item % p.n_t;
  item /= p.n_t;
  const int b = item % p.B;
  item /= p.B;
  const int h = item % p.Htot;
  item /= p.Htot;
  const int gfr = item;
  const int grp = h >= p.H0 ? 1 : 0;
  const int W = p.W[grp], dil = p.dil[grp];
  const int hk = h;
  const CUtensorMap* tk = &tkm;
  const CUtensorMap* tv = &tvm;
  const int ntiles = dkv_num_tiles(gfr, p.F, W, dil, p.n_t);
  const int k_row0 = b * p.rows_b + gfr * p.P + kt * 128;
  const int nk = min(128, p.P - kt * 128);

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_ab, 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.bar_s, 1);
    mbar_init(&sm.bar_p, 128);
    mbar_init(&sm.bar_o, 1);
    mbar_init(&sm.bar_fin, 1);
    mbar_init(&sm.bar_st[0], 128);
    mbar_init(&sm.bar_st[1], 128);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tdo);
      prefetch_tmap(tk);
      prefetch_tmap(tv);
      mbar_arrive_expect_tx(&sm.bar_ab, 2 * TILE_BYTES);
      for (int c = 0; c < NBOX; ++c) {
        tma_load_3d(sm.a + c * BOX, tk, &sm.bar_ab, c * 64, hk, k_row0);
        tma_load_3d(sm.b + c * BOX, tv, &sm.bar_ab, c * 64, hk, k_row0);
      }
      int issued = 0;
      for (int n = 0; n < 2 * ntiles; ++n) {  // Q_{n/2} (n even), dO_{n/2} (n odd)
        if (*abort_flag) break;
        const int slot = n % NSLOT, use = n / NSLOT;
        const int tile = n >> 1;
        const int fq = gfr + (tile / p.n_t) * dil;
        const int qrow = b * p.rows_b + fq * p.P + (tile % p.n_t) * 128;
        if (use > 0 && !mbar_wait(&sm.empty[slot], (use - 1) & 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&sm.full[slot], TILE_BYTES);
        const CUtensorMap* tm = (n & 1) ? &tdo : &tq;
        for (int c = 0; c < NBOX; ++c)
          tma_load_3d(sm.ring[slot] + c * BOX, tm, &sm.full[slot], c * 64, h, qrow);
        ++issued;
      }
      mbar_wait(&sm.bar_ab, 0);
      for (int n = issued - NSLOT > 0 ? issued - NSLOT : 0; n < issued; ++n)
        mbar_wait(&sm.full[n % NSLOT], (n / NSLOT) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t tS = sm.tmem_base, tP = sm.tmem_base + 128;
      const uint32_t tV = sm.tmem_base + 256, tK = sm.tmem_base + 384;
      const uint32_t a0 = smem_u32(sm.a), b0 = smem_u32(sm.b);
      bool ok = ntiles > 0 && mbar_wait(&sm.bar_ab, 0);
      auto issue_sp = [&](int n) {  // S^T = K Q_n^T, dP^T = V dO_n^T
        const int qs = (2 * n) % NSLOT, ds = (2 * n + 1) % NSLOT;
        const uint32_t ph = (n >> 1) & 1;
        if (!mbar_wait(&sm.full[qs], ph) || !mbar_wait(&sm.full[ds], ph)) return false;
        tc_fence_after();
        bwd_issue_ss<D>(tS, a0, smem_u32(sm.ring[qs]));
        bwd_issue_ss<D>(tP, b0, smem_u32(sm.ring[ds]));
        mma_commit(&sm.bar_s);
        return true;
      };
      if (ok) ok = issue_sp(0);
      for (int n = 0; ok && n < ntiles; ++n) {
        if (*abort_flag || !mbar_wait(&sm.bar_p, n & 1)) { ok = false; break; }
        tc_fence_after();
        const int qs = (2 * n) % NSLOT, ds = (2 * n + 1) % NSLOT;
        bwd_issue_ts<D>(tV, tS, smem_u32(sm.ring[ds]), n == 0);  // dV += P^T dO_n
        bwd_issue_ts<D>(tK, tP, smem_u32(sm.ring[qs]), n == 0);  // dK += dS^T Q_n
        mma_commit(&sm.empty[qs]);
        mma_commit(&sm.empty[ds]);
        if (n + 1 < ntiles && !issue_sp(n + 1)) { ok = false; break; }
      }
      if (ok) mma_commit(&sm.bar_o);
      if (!ok) *abort_flag = 1;
      mma_commit(&sm.bar_fin);
      mbar_wait(&sm.bar_fin, 0);
    }
  } else if (warp >= 4) {
    // softmax warps: thread <-> key row (TMEM lane); columns are query rows of the tile
    const int quad = warp & 3;
    const int krow = quad * 32 + lane;
    const int tid = threadIdx.x - 128;  // 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = sm.tmem_base, tP = sm.tmem_base + 128;
    const uint32_t tV = sm.tmem_base + 256, tK = sm.tmem_base + 384;
    const long long sb = (static_cast<long long>(b) * p.Htot + h) * p.rows_b;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int n = 0; ok && n < ntiles; ++n) {
      const int fq = gfr + (n / p.n_t) * dil;
      const int q0 = (n % p.n_t) * 128;
      const int nvq = min(128, p.P - q0);
      // this tile's column statistics into shared memory (one column per thread)
      float* sl = sm.st[n & 1][0];
      float* sd = sm.st[n & 1][1];
      {
        const long long si = sb + fq * p.P + q0 + min(tid, nvq - 1);
        sl[tid] = p.lse[si];
        sd[tid] = p.Dt[si];
      }
      mbar_arrive(&sm.bar_st[n & 1]);
      const bool got = !*abort_flag && mbar_wait(&sm.bar_st[n & 1], (n >> 1) & 1) &&
                       mbar_wait(&sm.bar_s, n & 1);
      if (!__all_sync(0xffffffffu, got)) { *abort_flag = 1; ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rs[32], rp[32];
        tmem_ld32(tS + lane_off + 32 * c, rs);
        tmem_ld32(tP + lane_off + 32 * c, rp);
        tmem_wait_ld();
        tmem_ld_fence(rs);
        tmem_ld_fence(rp);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = 32 * c + 2 * j;
          float p0 = ex2_approx(fmaf(__uint_as_float(rs[2 * j]), sl2, -sl[col]));
          float p1 = ex2_approx(fmaf(__uint_as_float(rs[2 * j + 1]), sl2, -sl[col + 1]));
          float d0 = p0 * (__uint_as_float(rp[2 * j]) - sd[col]);
          float d1 = p1 * (__uint_as_float(rp[2 * j + 1]) - sd[col + 1]);
          if (nvq < 128) {  // query rows past the frame's end
            p0 = col < nvq ? p0 : 0.f;
            p1 = col + 1 < nvq ? p1 : 0.f;
            d0 = col < nvq ? d0 : 0.f;
            d1 = col + 1 < nvq ? d1 : 0.f;
          }
          pk[j] = pack_bf16x2(p0, p1);
          dk[j] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tS + lane_off + 16 * c, pk);  // P^T over S^T
        tmem_st16(tP + lane_off + 16 * c, dk);  // dS^T over dP^T
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_p);
    }
    const bool fin = ok && ntiles > 0 && mbar_wait(&sm.bar_o, 0);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const long long orow = static_cast<long long>(k_row0 + krow) * p.ld + h * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = which ? tV : tK;
        __nv_bfloat16* dst_row = (which ? p.out1 : p.out0) + orow;
        const float mul = which ? 1.f : p.scale;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(src + lane_off + 32 * c, rr);
          tmem_wait_ld();
          tmem_ld_fence(rr);
          if (krow < nk) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              w[j] = pack_bf16x2(__uint_as_float(rr[2 * j]) * mul, __uint_as_float(rr[2 * j + 1]) * mul);
            uint4* dst = reinterpret_cast<uint4*>(dst_row + 32 * c);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
      }
    } else {
      *abort_flag = 1;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(sm.tmem_base, 512);
  }
}

}  // namespace kta
