// gla_tc.cuh -- chunked gated linear attention with a vector forget gate on the sm_100a tensor
// cores (tcgen05 + TMEM), head dim 128, 64-token chunks; bf16 in / out, fp32 state and gates.
//
// Operator (paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar, GLA paragraph): S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = scale * q_t S_t, S key-major
// (d_k x d_v).
//
// Chunked form (exact algebra). Within a span of tokens [lo, hi) of a chunk, b_t is the cumulative
// log2 gate from the span start (a vector over key dims), m the span's middle token and S_0 the
// state entering the span. With Qs_t = q_t 2^{b_t - b_m} and Ks_s = k_s 2^{b_m - b_s}:
//   o_t   = scale [ Qs_t (diag(2^{b_m}) S_0) + sum_{s <= t} (Qs_t . Ks_s) v_s ]
//   S_end = diag(2^{b_end - b_m}) [ diag(2^{b_m}) S_0 + Ks^T V ].
// A span is normally the whole chunk. Qs and Ks carry factors above 1 on one side of m, so every
// chunk checks, per key dim, that |b_t - b_m| <= KTA_GLA_LIM (64 bits); if any dim fails, the chunk
// is processed as 16-token spans, and if one of those fails too, token by token (a span of one
// token has both factors exactly 1). All granularities are exact forms of the same recurrence:
// small gates cost time, never accuracy. log2 of a gate is clamped at -200 (alpha = 0 gives 0).
//
// The state lives in tensor memory transposed, S^T (d_v lanes x d_k columns, fp32), so that all
// three products are tcgen05 MMAs with M = d_v = 128:
//   read-out   O^T  = (S^T diag(2^{b_m}))_bf16 * Qs^T         (A from TMEM, B = Qs, N = 64 tokens)
//   intra      O^T += V^T * mask(Qs Ks^T)^T                   (A = V^T from smem, B = scores)
//   update     S^T += V^T * Ks                                 (N = 128 key dims)
// and the decays are column scalings of S^T applied between spans. The causal score block
// Qs Ks^T (64 x 64) is formed on warp-level mma.sync tiles. Rows outside the current span are zero
// in Qs and Ks, so the same MMAs serve every span size.
//
// Warp roles (384 threads, one CTA per SM, all 128 value columns of a (sequence, head, segment)):
//   warp 0       TMA producer: q, k, v (bf16, 128-byte swizzle) and alpha (fp32) of each chunk into
//                a two-stage ring.
//   warp 1       TMEM allocation; one thread issues the tcgen05 MMAs of every span.
//   warps 4..7   gate warps, thread <-> key dim: cumulative log2 gates, the range check and span
//                plan, Qs / Ks written into their own buffers (the raw chunk stays intact for finer
//                spans), the column factors, and the masked score block.
//   warps 8..11  state warps, thread <-> value column (TMEM lane): start state into TMEM, the
//                per-span column scaling of S^T (and its bf16 copy), the output rows, and the end
//                state.
// Sequence parallelism as in the warp-level kernel: segments of whole chunks; pass 1 (OUTPUT =
// false) writes each segment's end state from zero and its total log2 decay, the carry kernel
// folds them, pass 2 (OUTPUT = true) runs each segment from its start state and writes o.
// Every wait is bounded; on a timeout the CTA records it and unwinds to free its TMEM.
#pragma once

#include "kta_ptx.cuh"
#include "mma_sync.cuh"

namespace kta {

#ifndef KTA_GLA_LIM
#define KTA_GLA_LIM 64.0f
#endif

constexpr int GT_C = 64;                   // tokens per chunk
constexpr int GT_D = 128;                  // head dim
constexpr uint32_t GT_BOX = 64 * 128;      // 64 rows x 64 bf16 (128-byte rows), 8 KB
constexpr uint32_t GT_TILE = 2 * GT_BOX;   // 64 rows x 128 bf16

struct GlaTcParams {
  int N;                   // tokens per sequence in this call
  int H;                   // heads in this call
  int rows_b;              // rows per sequence in q / k / v / o / alpha
  int seg_len;             // tokens per segment (multiple of 64)
  int nseg;
  float scale;
  __nv_bfloat16* o;        // output, offset to the first head of the call
  long long ld;            // o row stride (elements)
  const float* S0;         // [B][H][D][D] key-major, or null
  float* S_out;            // [B][H][D][D], or null
  float* ws_S;             // [B*H][nseg][D][D] segment states (pass 1 writes, carry folds)
  float* ws_L;             // [B*H][nseg][D] segment total log2 decay
  int fold;                // 1: pass 2 folds the segment end states itself (no carry kernel ran)
};

constexpr int GT_FOLD_MAX = 3;  // most predecessor segments a pass-2 CTA folds itself

struct GlaTcSmem {
  alignas(1024) uint8_t q[2][GT_TILE];     // stage ring, TMA layout (two 64-column boxes)
  alignas(1024) uint8_t k[2][GT_TILE];
  alignas(1024) uint8_t v[2][GT_TILE];
  alignas(1024) uint8_t qs[GT_TILE];       // decayed operands of the current span
  alignas(1024) uint8_t ks[GT_TILE];
  alignas(1024) uint8_t ab[GT_BOX];        // masked scores [t][s] of the current span
  alignas(16) float alpha[2][GT_C][GT_D];  // stage ring, row-major
  float fac[2][GT_D];                      // per span parity: column factor applied before it
  float cend[2][GT_D];                     // per span parity: 2^{b_end - b_m}
  alignas(16) float bmv[GT_D];             // b_m of the current span, per key dim
  int rinfo[2][8];                         // per span parity: lo, hi, flags, stage, chunk
  alignas(16) __nv_bfloat16 otr[4][8][32]; // per state warp: 8 output rows x 32 values (transpose)
  alignas(128) __nv_bfloat16 ostage[GT_C][GT_D]; // a whole chunk's output rows for one TMA store
  uint64_t full[2], sfree[2], facrdy, opnd, opfree, sready, sdone, odone[2], ofree[2], fin;
  uint64_t gready;                         // a chunk's cumulative gates are in its alpha stage
  uint32_t tmem_base;
  int abort_flag;
};

enum : int { GT_LAST_OF_CHUNK = 1, GT_LAST_OF_SEG = 2 };

// Byte offset of element (row, col) of a 64-row x 128-column bf16 tile in the TMA 128-byte swizzle
// layout (two boxes of 64 columns; the 16-byte chunk index is XORed with row % 8).
__device__ __forceinline__ uint32_t gt_sw(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * GT_BOX + row * 128 +
                               ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

// Explicit shared-memory accesses by 32-bit shared address (the kernel's shared struct is reached
// through an aligned integer, so plain pointer accesses would compile to generic ones).
__device__ __forceinline__ float gt_lds_bf16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}
__device__ __forceinline__ void gt_sts_bf16(uint32_t a, float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(*reinterpret_cast<const uint16_t*>(&b)) : "memory");
}
__device__ __forceinline__ float gt_lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 gt_lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ void gt_sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
// All-of / any-of over the 128 gate threads (named barrier 1).
__device__ __forceinline__ bool gt_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

template <bool OUTPUT>
__global__ void __launch_bounds__(384, 1)
    gla_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap ta,
                  const __grid_constant__ CUtensorMap to, const GlaTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  GlaTcSmem& sm = *reinterpret_cast<GlaTcSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int t_begin = seg * p.seg_len;
  const int t_end = min(p.N, t_begin + p.seg_len);
  const int nchunk = (t_end - t_begin + GT_C - 1) / GT_C;
  const long long row_b = static_cast<long long>(b) * p.rows_b;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.sfree[s], 1);
      mbar_init(&sm.odone[s], 1);
      mbar_init(&sm.ofree[s], 4);
    }
    mbar_init(&sm.facrdy, 4);
    mbar_init(&sm.opnd, 4);
    mbar_init(&sm.opfree, 1);
    mbar_init(&sm.sready, 4);
    mbar_init(&sm.sdone, 1);
    mbar_init(&sm.fin, 1);
    mbar_init(&sm.gready, 4);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  // the decayed-operand and score buffers start at zero (rows outside a span must be zero)
  static_assert(offsetof(GlaTcSmem, ks) == offsetof(GlaTcSmem, qs) + GT_TILE &&
                    offsetof(GlaTcSmem, ab) == offsetof(GlaTcSmem, ks) + GT_TILE,
                "qs, ks and ab are contiguous");
  for (int u = threadIdx.x; u < static_cast<int>(2 * GT_TILE + GT_BOX) / 16; u += blockDim.x)
    reinterpret_cast<uint4*>(sm.qs)[u] = make_uint4(0, 0, 0, 0);
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort_flag = &sm.abort_flag;
  const uint32_t tS = sm.tmem_base;         // S^T fp32, columns [0, 128)
  const uint32_t tSb = sm.tmem_base + 128;  // bf16 copy of the scaled S^T, columns [128, 192)
  const uint32_t tO0 = sm.tmem_base + 256;  // O^T of even / odd spans, 64 columns each

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      prefetch_tmap(&ta);
      if (OUTPUT) prefetch_tmap(&tq);
      constexpr uint32_t BYTES = (OUTPUT ? 3 : 2) * GT_TILE + GT_C * GT_D * 4;
      int issued = 0;
      for (int c = 0; c < nchunk; ++c) {
        if (*abort_flag) break;
        const int s = c & 1, use = c >> 1;
        if (use > 0 && !mbar_wait(&sm.sfree[s], (use - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        const int row0 = static_cast<int>(row_b) + t_begin + c * GT_C;
        mbar_arrive_expect_tx(&sm.full[s], BYTES);
        for (int x = 0; x < 2; ++x) {
          if (OUTPUT) tma_load_3d(sm.q[s] + x * GT_BOX, &tq, &sm.full[s], x * 64, h, row0);
          tma_load_3d(sm.k[s] + x * GT_BOX, &tk, &sm.full[s], x * 64, h, row0);
          tma_load_3d(sm.v[s] + x * GT_BOX, &tv, &sm.full[s], x * 64, h, row0);
        }
        tma_load_3d(&sm.alpha[s][0][0], &ta, &sm.full[s], 0, h, row0);
        ++issued;
      }
      // the copies this thread started land before the CTA can exit (bounded waits)
      for (int c = issued - 2 > 0 ? issued - 2 : 0; c < issued; ++c)
        mbar_wait(&sm.full[c & 1], (c >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_R = idesc_bf16_f32(128, 64, 0, 0);   // S_bf16 (TMEM) x Qs^T
      constexpr uint32_t ID_I = idesc_bf16_f32(128, 64, 1, 0);   // V^T x scores^T
      constexpr uint32_t ID_U = idesc_bf16_f32(128, 128, 1, 1);  // V^T x Ks
      const uint32_t qs_a = smem_u32(sm.qs), ks_a = smem_u32(sm.ks), ab_a = smem_u32(sm.ab);
      bool ok = true;
      for (int R = 0; ok; ++R) {
        if (!mbar_wait(&sm.opnd, R & 1)) { ok = false; break; }
        const int lo = sm.rinfo[R & 1][0], hi = sm.rinfo[R & 1][1];
        const int flags = sm.rinfo[R & 1][2], s = sm.rinfo[R & 1][3];
        if (flags < 0) { ok = false; break; }  // the gate warps aborted
        if (!mbar_wait(&sm.sready, R & 1)) { ok = false; break; }
        const int ob = R & 1;
        if (OUTPUT && R >= 2 && !mbar_wait(&sm.ofree[ob], ((R - 2) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t v_a = smem_u32(sm.v[s]);
        const int k0 = lo >> 4, k1 = (hi - 1) >> 4;  // 16-token K steps the span touches
        if (OUTPUT) {
          const uint32_t tO = tO0 + 64 * ob;
#pragma unroll
          for (int kk = 0; kk < GT_D / 16; ++kk)
            mma_ts(tO, tSb + kk * 8,
                   smem_desc_sw128(qs_a + (kk >> 2) * GT_BOX + (kk & 3) * 32, 16, 1024), ID_R,
                   kk > 0 ? 1u : 0u);
          for (int kk = k0; kk <= k1; ++kk)
            mma_ss(tO, smem_desc_sw128(v_a + kk * 16 * 128, GT_BOX, 1024),
                   smem_desc_sw128(ab_a + kk * 32, 16, 1024), ID_I, 1u);
          mma_commit(&sm.odone[ob]);
        }
        for (int kk = k0; kk <= k1; ++kk)
          mma_ss(tS, smem_desc_sw128(v_a + kk * 16 * 128, GT_BOX, 1024),
                 smem_desc_sw128(ks_a + kk * 16 * 128, GT_BOX, 1024), ID_U, 1u);
        mma_commit(&sm.sdone);
        mma_commit(&sm.opfree);
        if (flags & GT_LAST_OF_CHUNK) mma_commit(&sm.sfree[s]);
        if (flags & GT_LAST_OF_SEG) break;
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&sm.fin);
      mbar_wait(&sm.fin, 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ gate warps (key dim kd)
    const int kd = threadIdx.x - 128;
    const int gw = warp - 4;
    float cend_prev = 1.f;
    int plo = 0, phi = 0;  // rows of the previous span in qs / ks
    int R = 0;
    bool ok = true;
    for (int c = 0; ok && c < nchunk; ++c) {
      const int s = c & 1;
      const int n = min(GT_C, t_end - t_begin - c * GT_C);
      if (!gt_all(!*abort_flag && mbar_wait(&sm.full[s], (c >> 1) & 1))) { ok = false; break; }
      // the state warps have replaced this chunk's alpha columns by the cumulative log2 gates
      if (!gt_all(!*abort_flag && mbar_wait(&sm.gready, c & 1))) { ok = false; break; }
      const uint32_t bcol = smem_u32(&sm.alpha[s][0][kd]);
      auto bt = [&](int t) { return gt_lds_f32(bcol + t * GT_D * 4); };
      // span plan: the whole chunk, 16-token spans, or single tokens. A span [lo, hi) with middle
      // m = lo + (hi - lo) / 2 passes when every |b_t - b_m| <= KTA_GLA_LIM; b is monotone, so the
      // largest deviation is at one of the span's ends.
      auto dev_ok = [&](int lo, int hi) {
        const float bm = bt(lo + ((hi - lo) >> 1));
        return !(fmaxf(bt(lo) - bm, bm - bt(hi - 1)) > KTA_GLA_LIM);
      };
      int span = GT_C;
      if (!gt_all(dev_ok(0, n))) {
        bool ok16 = true;
        for (int u = 0; u < n; u += 16) ok16 = ok16 && dev_ok(u, min(u + 16, n));
        span = gt_all(ok16) ? 16 : 1;
      }
      for (int lo = 0; ok && lo < n; lo += span) {
        const int hi = min(lo + span, n);
        const bool last_chunk = c == nchunk - 1, last_span = hi == n;
        // the MMAs of the previous span have read qs / ks / ab
        if (!gt_all(!*abort_flag && (R == 0 || mbar_wait(&sm.opfree, (R - 1) & 1)))) {
          ok = false;
          break;
        }
        const int mid = lo + ((hi - lo) >> 1);
        const float bl = lo > 0 ? bt(lo - 1) : 0.f, bm = bt(mid), be = bt(hi - 1);
        const float emid = ex2_approx(bm - bl), ce = ex2_approx(be - bm);
        sm.fac[R & 1][kd] = cend_prev * emid;
        sm.cend[R & 1][kd] = ce;
        cend_prev = ce;
        if (kd == 0) {
          sm.rinfo[R & 1][0] = lo;
          sm.rinfo[R & 1][1] = hi;
          sm.rinfo[R & 1][2] = (last_span ? GT_LAST_OF_CHUNK : 0) | (last_span && last_chunk ? GT_LAST_OF_SEG : 0);
          sm.rinfo[R & 1][3] = s;
          sm.rinfo[R & 1][4] = c;
        }
        // the state warps may scale S^T for this span while the operands are written
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.facrdy);
        // decayed operands, written as 16-byte chunks: thread i takes the 8 key dims of chunk
        // i % 16 in rows i / 16 + 8 j; rows of the previous span outside this one are cleared
        sm.bmv[kd] = bm;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        {
          // thread i takes the 8 key dims of 16-byte chunk i % 16 in rows i / 16 + 8 j; the
          // inputs of four rows are read before any of them is written, so that the reads overlap
          const int cc = kd & 15, r0t = kd >> 4;
          const uint4 bm0 = gt_lds128(smem_u32(&sm.bmv[cc * 8]));
          const uint4 bm1 = gt_lds128(smem_u32(&sm.bmv[cc * 8 + 4]));
          const float bmc[8] = {__uint_as_float(bm0.x), __uint_as_float(bm0.y), __uint_as_float(bm0.z),
                                __uint_as_float(bm0.w), __uint_as_float(bm1.x), __uint_as_float(bm1.y),
                                __uint_as_float(bm1.z), __uint_as_float(bm1.w)};
          const uint32_t a_base = smem_u32(&sm.alpha[s][0][cc * 8]);
          const uint32_t k_base = smem_u32(sm.k[s]), q_base = smem_u32(sm.q[s]);
          const uint32_t ks_base = smem_u32(sm.ks), qs_base = smem_u32(sm.qs);
#pragma unroll
          for (int j0 = 0; j0 < GT_C / 8; j0 += 4) {
            uint4 ga[4], gb[4], kr[4], qr[4];
            bool in[4], touch[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int t = r0t + 8 * (j0 + jj);
              in[jj] = t >= lo && t < hi;
              touch[jj] = in[jj] || (t >= plo && t < phi);
              ga[jj] = gb[jj] = kr[jj] = qr[jj] = make_uint4(0, 0, 0, 0);
              if (in[jj]) {
                const uint32_t off = gt_sw(t, cc * 8);
                ga[jj] = gt_lds128(a_base + t * GT_D * 4);
                gb[jj] = gt_lds128(a_base + t * GT_D * 4 + 16);
                kr[jj] = gt_lds128(k_base + off);
                if (OUTPUT) qr[jj] = gt_lds128(q_base + off);
              }
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              if (!touch[jj]) continue;
              const int t = r0t + 8 * (j0 + jj);
              const uint32_t off = gt_sw(t, cc * 8);
              uint4 kw = make_uint4(0, 0, 0, 0), qw = kw;
              if (in[jj]) {
                const float bb[8] = {__uint_as_float(ga[jj].x), __uint_as_float(ga[jj].y),
                                     __uint_as_float(ga[jj].z), __uint_as_float(ga[jj].w),
                                     __uint_as_float(gb[jj].x), __uint_as_float(gb[jj].y),
                                     __uint_as_float(gb[jj].z), __uint_as_float(gb[jj].w)};
                const uint32_t* kp = &kr[jj].x;
                uint32_t* ko = &kw.x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float d0 = bb[2 * e] - bmc[2 * e], d1 = bb[2 * e + 1] - bmc[2 * e + 1];
                  ko[e] = pack_bf16x2(__uint_as_float(kp[e] << 16) * ex2_approx(-d0),
                                      __uint_as_float(kp[e] & 0xffff0000u) * ex2_approx(-d1));
                }
                if (OUTPUT) {
                  const uint32_t* qp = &qr[jj].x;
                  uint32_t* qo = &qw.x;
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float d0 = bb[2 * e] - bmc[2 * e], d1 = bb[2 * e + 1] - bmc[2 * e + 1];
                    qo[e] = pack_bf16x2(__uint_as_float(qp[e] << 16) * ex2_approx(d0),
                                        __uint_as_float(qp[e] & 0xffff0000u) * ex2_approx(d1));
                  }
                }
              }
              gt_sts128(ks_base + off, kw);
              if (OUTPUT) gt_sts128(qs_base + off, qw);
            }
          }
        }
        plo = lo;
        phi = hi;
        if (OUTPUT) {
          asm volatile("bar.sync 2, 128;" ::: "memory");
          // masked scores of the span's query rows: A[t][s] = Qs_t . Ks_s for s <= t
          const int r0 = gw * 16;
          if (r0 < hi && r0 + 16 > lo) {
            uint32_t aq[GT_D / 16][4];
#pragma unroll
            for (int kk = 0; kk < GT_D / 16; ++kk)
              ldsm_x4(aq[kk], sm.qs + gt_sw(r0 + (lane & 15), kk * 16 + (lane >> 4) * 8));
            float sc[GT_C / 8][4];
#pragma unroll
            for (int nt = 0; nt < GT_C / 8; ++nt)
#pragma unroll
              for (int r = 0; r < 4; ++r) sc[nt][r] = 0.f;
#pragma unroll
            for (int np = 0; np < GT_C / 16; ++np) {
              if (np > gw) break;
#pragma unroll
              for (int kk = 0; kk < GT_D / 16; ++kk) {
                uint32_t bk[4];
                ldsm_x4(bk, sm.ks + gt_sw(np * 16 + (lane & 7) + (lane >> 4) * 8,
                                          kk * 16 + ((lane >> 3) & 1) * 8));
                mma16816(sc[2 * np], aq[kk], bk[0], bk[1]);
                mma16816(sc[2 * np + 1], aq[kk], bk[2], bk[3]);
              }
            }
            const int g4 = lane >> 2, t4 = lane & 3;
#pragma unroll
            for (int nt = 0; nt < GT_C / 8; ++nt) {
              const int col = nt * 8 + 2 * t4;
              const int ra = r0 + g4, rb = r0 + g4 + 8;
              const uint32_t wa = bf16x2(col <= ra ? sc[nt][0] : 0.f, col + 1 <= ra ? sc[nt][1] : 0.f);
              const uint32_t wb = bf16x2(col <= rb ? sc[nt][2] : 0.f, col + 1 <= rb ? sc[nt][3] : 0.f);
              *reinterpret_cast<uint32_t*>(sm.ab + (ra * 128 + (((col >> 3) ^ (ra & 7)) << 4) + ((col & 7) << 1))) = wa;
              *reinterpret_cast<uint32_t*>(sm.ab + (rb * 128 + (((col >> 3) ^ (rb & 7)) << 4) + ((col & 7) << 1))) = wb;
            }
          }
        }
        fence_proxy_async_smem();  // generic writes of qs / ks / ab -> the tensor core's reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.opnd);
        ++R;
      }
    }
    if (!ok) {
      // tell the MMA and state warps to stop: a span record with negative flags
      *abort_flag = 1;
      if (kd == 0) {
        sm.rinfo[R & 1][2] = -1;
        sm.rinfo[R & 1][0] = 0;
        sm.rinfo[R & 1][1] = 1;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.facrdy);
        mbar_arrive(&sm.opnd);
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------------ state warps (value vd)
    const int quad = warp & 3;
    const int vd = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    // Cumulative log2 gate of key dim vd over chunk cc, written over its alpha column (the stage
    // stays untouched by the producer until the chunk's MMAs are done); rows >= n: alpha = 1. Each
    // log2 gate is clamped to [-200, 0], so b_t never increases with t. The state warps do this
    // one chunk ahead of the gate warps, which wait for it on `gready`.
    float ltot = 0.f;
    auto cumsum = [&](int cc) {
      const int sc = cc & 1;
      const int n = min(GT_C, t_end - t_begin - cc * GT_C);
      const bool got = !*abort_flag && mbar_wait(&sm.full[sc], (cc >> 1) & 1);
      if (!__all_sync(0xffffffffu, got)) return false;
      const uint32_t bcol = smem_u32(&sm.alpha[sc][0][vd]);
      float acc = 0.f;
      for (int t = 0; t < GT_C; ++t) {
        const uint32_t a = bcol + t * GT_D * 4;
        acc += fmaxf(fminf(__log2f(t < n ? gt_lds_f32(a) : 1.f), 0.f), -200.f);
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(acc) : "memory");
      }
      ltot += acc;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.gready);
      return true;
    };
    int next_cum = 1;  // the next chunk whose gates are still raw
    bool ok = cumsum(0);
    if (!ok) *abort_flag = 1;
    // start state: S0 for a single segment, else the carry kernel's start of this segment, or
    // (fold) S_start(s+1) = 2^{L_s} S_start(s) + S_loc(s) over the predecessors, as the carry
    // kernel computes it
    const bool fold = OUTPUT && p.fold && p.nseg > 1;
    const float* S0b = p.S0 ? p.S0 + static_cast<long long>(bh) * GT_D * GT_D : nullptr;
    const float* Ss = !OUTPUT ? nullptr
                      : p.nseg > 1 && !fold ? p.ws_S + (static_cast<long long>(bh) * p.nseg + seg) * GT_D * GT_D
                                            : S0b;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = Ss ? __float_as_uint(Ss[(c4 * 32 + j) * GT_D + vd]) : 0u;
      if (fold) {
        for (int sp = 0; sp < seg && sp < GT_FOLD_MAX; ++sp) {
          const float* E = p.ws_S + (static_cast<long long>(bh) * p.nseg + sp) * GT_D * GT_D;
          const float* Lw = p.ws_L + (static_cast<long long>(bh) * p.nseg + sp) * GT_D;
          float e[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) e[j] = E[(c4 * 32 + j) * GT_D + vd];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            r[j] = __float_as_uint(fmaf(exp2f(Lw[c4 * 32 + j]), __uint_as_float(r[j]), e[j]));
        }
      }
      tmem_st32(tS + lane_off + 32 * c4, r);
    }
    tmem_wait_st();
    int R = 0, lo_prev = 0, hi_prev = 0, c_prev = 0;
    // All-of over the four state warps (named barrier 3), so that they take the same path.
    auto st_all = [&](bool v) {
      uint32_t r;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
          "bar.red.and.pred q, 3, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(r)
          : "r"(static_cast<uint32_t>(v))
          : "memory");
      return r != 0;
    };
    const bool store_lead = warp == 8 && lane == 0;  // issues the output TMA stores
    auto epilogue = [&](int Rq, int lo, int hi, int c) -> bool {
      const int ob = Rq & 1;
      const bool got = mbar_wait(&sm.odone[ob], (Rq >> 1) & 1);
      if (!st_all(got)) return false;
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(tO0 + 64 * ob + lane_off, *reinterpret_cast<uint32_t(*)[32]>(r));
      tmem_ld32(tO0 + 64 * ob + 32 + lane_off, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tmem_wait_ld();
      tmem_ld_fence(r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ofree[ob]);
      const int n = min(GT_C, t_end - t_begin - c * GT_C);
      if (lo == 0 && hi == n) {
        // the whole chunk: thread vd writes its value column of the 64 rows into the staging tile
        // (row-major, 256 bytes a row), then one thread stores the tile with the TMA unit (rows
        // past the sequence's end are outside the map and not written)
        if (store_lead) bulk_wait_read_all();  // the previous store has read the tile
        asm volatile("bar.sync 3, 128;" ::: "memory");
        const uint32_t col = smem_u32(&sm.ostage[0][vd]);
#pragma unroll
        for (int t = 0; t < GT_C; ++t) {
          const __nv_bfloat16 x = __float2bfloat16_rn(__uint_as_float(r[t]) * p.scale);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(col + t * GT_D * 2),
                       "h"(*reinterpret_cast<const uint16_t*>(&x))
                       : "memory");
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 3, 128;" ::: "memory");
        if (store_lead) {
          tma_store_4d(&to, &sm.ostage[0][0], 0, h, t_begin + c * GT_C, b);
          bulk_commit();
        }
        return true;
      }
      // a span inside the chunk: rows [lo, hi) of this warp's 32 value columns, eight rows at a
      // time through a small transpose buffer (each thread then stores 16 bytes of one row)
      __nv_bfloat16 (*tb)[32] = sm.otr[quad];
      const int tr = lane >> 2, tc = (lane & 3) * 8;
      __nv_bfloat16* obase = p.o + (row_b + t_begin + c * GT_C) * p.ld +
                             static_cast<long long>(h) * GT_D + quad * 32 + tc;
#pragma unroll
      for (int t0 = 0; t0 < GT_C; t0 += 8) {
        if (t0 + 8 <= lo || t0 >= hi) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) tb[j][lane] = __float2bfloat16_rn(__uint_as_float(r[t0 + j]) * p.scale);
        __syncwarp();
        const int t = t0 + tr;
        if (t >= lo && t < hi)
          *reinterpret_cast<uint4*>(obase + static_cast<long long>(t) * p.ld) =
              *reinterpret_cast<const uint4*>(&tb[tr][tc]);
        __syncwarp();
      }
      return true;
    };
    for (; ok; ++R) {
      const bool got = !*abort_flag && (R == 0 || mbar_wait(&sm.sdone, (R - 1) & 1)) &&
                       mbar_wait(&sm.facrdy, R & 1);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const int lo = sm.rinfo[R & 1][0], hi = sm.rinfo[R & 1][1];
      const int flags = sm.rinfo[R & 1][2], c = sm.rinfo[R & 1][4];
      if (flags < 0) { ok = false; break; }
      // S^T <- S^T diag(fac); bf16 copy for the read-out
      const float* fac = sm.fac[R & 1];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t r[32];
        tmem_ld32(tS + lane_off + 32 * c4, r);
        tmem_wait_ld();
        tmem_ld_fence(r);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * fac[c4 * 32 + j]);
        tmem_st32(tS + lane_off + 32 * c4, r);
        if (OUTPUT) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
          tmem_st16(tSb + lane_off + 16 * c4, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sready);
      // the next chunk's gates, before this warp's output rows, so that the gate warps can start it
      if (next_cum == c + 1 && next_cum < nchunk) {
        if (!cumsum(next_cum)) { ok = false; break; }
        ++next_cum;
      }
      if (OUTPUT && R > 0 && !epilogue(R - 1, lo_prev, hi_prev, c_prev)) { ok = false; break; }
      lo_prev = lo;
      hi_prev = hi;
      c_prev = c;
      if (flags & GT_LAST_OF_SEG) break;
    }
    if (ok && OUTPUT && !epilogue(R, lo_prev, hi_prev, c_prev)) ok = false;
    if (OUTPUT && store_lead) bulk_wait_all();  // the output stores are complete before exit
    if (ok && !OUTPUT) p.ws_L[(static_cast<long long>(bh) * p.nseg + seg) * GT_D + vd] = ltot;
    // end state of the segment: S^T diag(cend of the last span), written key-major
    const bool fin = ok && mbar_wait(&sm.sdone, R & 1);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      float* Sd = !OUTPUT ? p.ws_S + (static_cast<long long>(bh) * p.nseg + seg) * GT_D * GT_D
                  : (seg == p.nseg - 1 && p.S_out ? p.S_out + static_cast<long long>(bh) * GT_D * GT_D : nullptr);
      if (Sd) {
        const float* ce = sm.cend[R & 1];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t r[32];
          tmem_ld32(tS + lane_off + 32 * c4, r);
          tmem_wait_ld();
          tmem_ld_fence(r);
#pragma unroll
          for (int j = 0; j < 32; ++j) Sd[(c4 * 32 + j) * GT_D + vd] = __uint_as_float(r[j]) * ce[c4 * 32 + j];
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
