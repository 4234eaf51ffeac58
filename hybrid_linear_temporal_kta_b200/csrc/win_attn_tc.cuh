// win_attn_tc.cuh -- frame-windowed softmax attention (SWA and DSWA) on the sm_100a tensor cores.
//
// Operator: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar. SWA: standard attention over a window of W whole frames ending at the query's frame.
// DSWA: the same window size with frames taken every dil-th step back (f, f-dil, ...).
//
// One CTA computes one tile of up to 128 query rows that lie in ONE frame (tiles restart at
// every frame start), so every row of the tile sees the same key frames and the only mask is a
// column bound on the last key tile of each key span. Key spans: for dil == 1 the W visible
// frames are adjacent and form one span; for dil > 1 each visible frame is its own span.
//
// Warp roles (192 threads, two CTAs per SM so one CTA's softmax overlaps the other's MMAs):
//   warp 0      TMA producer: Q once, then K_i and V_i tiles (128 keys x D, 128-byte swizzle).
//   warp 1      allocates 256 TMEM columns; one thread issues tcgen05.mma:
//               S = Q K_i^T (SS form, fp32 in TMEM cols [0,128)), then O += P_i V_i (TS form,
//               P_i read from TMEM where the softmax warps wrote it over S, V MN-major).
//   warps 2..5  softmax: thread <-> query row (TMEM lane). Row max, lazy rescale of O in TMEM
//               when the max grows by more than 2^8, P = exp2(S*scale*log2e - m) as bf16 into
//               TMEM, running row sum; epilogue O / l -> bf16 -> global.
// Every wait is bounded; on a timeout the CTA records it and unwinds to free its TMEM.
#pragma once

#include "kta_ptx.cuh"

namespace kta {

struct WinParams {
  int B;            // sequences
  int P;            // tokens per frame
  int Fq;           // query frames in this launch (sequence: F; streaming step: 1)
  int f_base;       // absolute frame index of query frame 0
  int n_qt;         // query tiles per frame = ceil(P / 128)
  int Htot;         // heads in this launch (group 0 then group 1)
  int H0;           // heads of group 0
  int W[2];         // window (frames) per group
  int dil[2];       // dilation per group
  int kh_off[2];    // head coordinate in the group's K/V map = h - kh_off[g]
  int kb_frames[2]; // frames per sequence in the group's K/V buffer
  int kmod[2];      // frame index modulus in the K/V buffer (ring slots; = F for a sequence)
  int q_rows_b;     // rows per sequence in the q / o buffers
  float scale_log2; // softmax scale * log2(e)
  __nv_bfloat16* o; // output, already offset to the launch's first head
  long long o_ld;   // output row stride in elements
};

__device__ __forceinline__ int win_num_tiles(int f, int P, int W, int dil) {
  if (dil == 1) {
    const int g0 = max(0, f - W + 1);
    return ((f - g0 + 1) * P + 127) / 128;
  }
  const int nsp = min(W, f / dil + 1);
  return nsp * ((P + 127) / 128);
}

// Key tile i of query frame f: first frame of its span, key offset from that frame's first
// token, and the number of valid keys (columns) in the tile. Spans are taken oldest first.
__device__ __forceinline__ void win_tile(int i, int f, int P, int W, int dil, int& frame0,
                                         int& off, int& nvalid) {
  if (dil == 1) {
    const int g0 = max(0, f - W + 1);
    const int len = (f - g0 + 1) * P;
    frame0 = g0;
    off = 128 * i;
    nvalid = min(128, len - off);
    return;
  }
  const int tp = (P + 127) / 128;
  const int nsp = min(W, f / dil + 1);
  const int j = i / tp, t = i % tp;
  frame0 = f - (nsp - 1 - j) * dil;
  off = 128 * t;
  nvalid = min(128, P - off);
}

template <int D>
struct WinSmem {
  static constexpr int BOX = 128 * 64 * 2;  // one 128-row x 64-column bf16 box, 16 KB
  static constexpr int NBOX = D / 64;
  alignas(1024) uint8_t q[NBOX * BOX];
  alignas(1024) uint8_t k[NBOX * BOX];
  alignas(1024) uint8_t v[NBOX * BOX];
  uint64_t bar_q, bar_kfull, bar_kempty, bar_vfull, bar_vempty, bar_s, bar_p, bar_pv, bar_fin;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t win_smem_bytes() {
  // +1024 for manual alignment of the dynamic shared memory base; at least 80 KB so that no
  // more than two CTAs (2 x 256 TMEM columns) share an SM.
  return sizeof(WinSmem<D>) + 1024 > 80 * 1024 ? sizeof(WinSmem<D>) + 1024 : 80 * 1024;
}

template <int D>
__global__ void __launch_bounds__(192, 2)
    win_attn_tc_kernel(const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk0,
                       const __grid_constant__ CUtensorMap tv0,
                       const __grid_constant__ CUtensorMap tk1,
                       const __grid_constant__ CUtensorMap tv1, const WinParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ uint8_t smem_raw[];
  WinSmem<D>& sm = *reinterpret_cast<WinSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int BOX = WinSmem<D>::BOX;
  constexpr int NBOX = WinSmem<D>::NBOX;
  constexpr uint32_t TILE_BYTES = 128 * D * 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: frames latest first (full windows first), then head, sequence, tile
  int item = blockIdx.x;
  const int qt = item % p.n_qt;
  item /= p.n_qt;
  const int b = item % p.B;
  item /= p.B;
  const int h = item % p.Htot;
  item /= p.Htot;
  const int f_local = p.Fq - 1 - item;
  const int f = f_local + p.f_base;
  const int g = h >= p.H0 ? 1 : 0;
  const int W = g ? p.W[1] : p.W[0];
  const int dil = g ? p.dil[1] : p.dil[0];
  const int hk = h - (g ? p.kh_off[1] : p.kh_off[0]);
  const int kbf = g ? p.kb_frames[1] : p.kb_frames[0];
  const int kmod = g ? p.kmod[1] : p.kmod[0];
  const CUtensorMap* tk = g ? &tk1 : &tk0;
  const CUtensorMap* tv = g ? &tv1 : &tv0;
  const int ntiles = win_num_tiles(f, p.P, W, dil);
  const int q_row0 = b * p.q_rows_b + f_local * p.P + qt * 128;
  const int nq = min(128, p.P - qt * 128);

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    mbar_init(&sm.bar_kfull, 1);
    mbar_init(&sm.bar_kempty, 1);
    mbar_init(&sm.bar_vfull, 1);
    mbar_init(&sm.bar_vempty, 1);
    mbar_init(&sm.bar_s, 1);
    mbar_init(&sm.bar_p, 128);
    mbar_init(&sm.bar_pv, 1);
    mbar_init(&sm.bar_fin, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tS = sm.tmem_base;        // S / P: columns [0, 128)
  const uint32_t tO = sm.tmem_base + 128;  // O: columns [128, 128 + D)
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(tk);
      prefetch_tmap(tv);
      mbar_arrive_expect_tx(&sm.bar_q, TILE_BYTES);
      for (int c = 0; c < NBOX; ++c) tma_load_3d(sm.q + c * BOX, &tq, &sm.bar_q, c * 64, h, q_row0);
      int k_issued = 0, v_issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        if (*abort_flag) break;
        int fr0, off, nv;
        win_tile(i, f, p.P, W, dil, fr0, off, nv);
        const int krow = (b * kbf + fr0 % kmod) * p.P + off;
        if (i > 0 && !mbar_wait(&sm.bar_kempty, (i - 1) & 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&sm.bar_kfull, TILE_BYTES);
        for (int c = 0; c < NBOX; ++c) tma_load_3d(sm.k + c * BOX, tk, &sm.bar_kfull, c * 64, hk, krow);
        ++k_issued;
        if (i > 0 && !mbar_wait(&sm.bar_vempty, (i - 1) & 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(&sm.bar_vfull, TILE_BYTES);
        for (int c = 0; c < NBOX; ++c) tma_load_3d(sm.v + c * BOX, tv, &sm.bar_vfull, c * 64, hk, krow);
        ++v_issued;
      }
      // Let the copies this thread started land before the CTA can exit (bounded waits).
      mbar_wait(&sm.bar_q, 0);
      if (k_issued > 0) mbar_wait(&sm.bar_kfull, (k_issued - 1) & 1);
      if (v_issued > 0) mbar_wait(&sm.bar_vfull, (v_issued - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t ID_O = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(sm.q), k_base = smem_u32(sm.k), v_base = smem_u32(sm.v);
      bool ok = mbar_wait(&sm.bar_q, 0);
      if (!ok) *abort_flag = 1;
      for (int i = 0; ok && i < ntiles; ++i) {
        if (*abort_flag) break;
        if (!mbar_wait(&sm.bar_kfull, i & 1)) { *abort_flag = 1; break; }
        // P_{i-1} lives in the S columns: S_i may only be written once PV_{i-1} has finished.
        if (i > 0 && !mbar_wait(&sm.bar_pv, (i - 1) & 1)) { *abort_flag = 1; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
          mma_ss(tS, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(k_base + off, 16, 1024),
                 ID_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.bar_s);
        mma_commit(&sm.bar_kempty);
        if (!mbar_wait(&sm.bar_p, i & 1)) { *abort_flag = 1; break; }
        if (!mbar_wait(&sm.bar_vfull, i & 1)) { *abort_flag = 1; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_ts(tO, tS + kk * 8, smem_desc_sw128(v_base + kk * 16 * 128, BOX, 1024), ID_O,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.bar_pv);
        mma_commit(&sm.bar_vempty);
      }
      // All MMAs issued by this thread are complete once bar_fin flips.
      mma_commit(&sm.bar_fin);
      mbar_wait(&sm.bar_fin, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      int fr0, off, nv;
      win_tile(i, f, p.P, W, dil, fr0, off, nv);
      const bool got = !*abort_flag && mbar_wait(&sm.bar_s, i & 1);
      if (!__all_sync(0xffffffffu, got)) { *abort_flag = 1; ok = false; break; }
      tc_fence_after();
      // pass 1: row maximum of the valid columns
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + lane_off + 32 * c, r);
        tmem_wait_ld();
        if (nv == 128) {
#pragma unroll
          for (int j = 0; j < 32; ++j) mx = fmaxf(mx, __uint_as_float(r[j]));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (32 * c + j < nv) mx = fmaxf(mx, __uint_as_float(r[j]));
        }
      }
      const float mnew = fmaxf(m, mx * sl2);
      if (i == 0) {
        m = mnew;
      } else {
        const bool need = mnew > m + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // O is stable here: S_i was issued only after PV_{i-1} completed.
          const float fac = need ? ex2_approx(m - mnew) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + 32 * c, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * fac);
            tmem_st32(tO + lane_off + 32 * c, r);
          }
          tmem_wait_st();
          if (need) {
            l *= fac;
            m = mnew;
          }
        }
      }
      // pass 2: P = exp2(S * scale * log2e - m) as bf16 pairs, written over S
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + lane_off + 32 * c, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = 32 * c + 2 * j;
          float p0 = ex2_approx(fmaf(__uint_as_float(r[2 * j]), sl2, -m));
          float p1 = ex2_approx(fmaf(__uint_as_float(r[2 * j + 1]), sl2, -m));
          if (nv < 128) {
            p0 = col < nv ? p0 : 0.f;
            p1 = col + 1 < nv ? p1 : 0.f;
          }
          ls += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + lane_off + 16 * c, pk);
      }
      l += ls;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_p);
    }
    // epilogue: O / l -> bf16 -> global (rows of this frame only)
    const bool fin = ok && ntiles > 0 && mbar_wait(&sm.bar_pv, (ntiles - 1) & 1);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      __nv_bfloat16* orow = p.o + static_cast<long long>(q_row0 + row) * p.o_ld + h * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + 32 * c, r);
        tmem_wait_ld();
        if (row < nq) {
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * inv, __uint_as_float(r[2 * j + 1]) * inv);
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
    tmem_dealloc(sm.tmem_base, 256);
  }
}

}  // namespace kta
