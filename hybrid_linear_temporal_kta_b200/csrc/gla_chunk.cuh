// gla_chunk.cuh -- chunked gated linear attention with a vector forget gate (bf16 in / out,
// fp32 state and gates), on warp-level bf16 tensor-core tiles.
//
// Operator (paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar, GLA paragraph): S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = scale * q_t S_t.
//
// Chunked form used here (exact algebra; spans of C tokens aligned to multiples of C from token
// 0). Let b_t = sum_{r <= t in span} log2 alpha_r (a vector over key dims), m = n/2 the span's
// middle token (n valid tokens), S_0 the state at the span start, and
//   Qi_t = q_t * 2^{b_t - b_m},   Ki_s = k_s * 2^{b_m - b_s}   (elementwise over key dims).
// Then
//   o_t   = scale * [ Qi_t (diag(2^{b_m}) S_0) + sum_{s <= t} (Qi_t . Ki_s) v_s ]
//   S_end = diag(2^{b_C - b_m}) [ diag(2^{b_m}) S_0 + Ki^T V ]
// so one pair of decayed operands (one exp2 each per element) serves the intra-chunk scores, the
// inter-chunk read-out and the state update.
//
// Gate range. Qi and Ki carry 2^{b_t - b_m} and 2^{b_m - b_s}, which exceed 1 on one side of the
// middle token; for gates near 0 they would leave the fp32 / bf16 range. So every span checks,
// per key dim, that |b_t - b_m| <= KTA_GLA_LIM (64 bits) for all its tokens. If any dim fails,
// the span is redone as sub-spans of 16 tokens (each with its own middle token), and a 16-token
// sub-span that still fails is redone token by token (n = 1: both factors are exactly 1). All
// three granularities are exact forms of the same recurrence, so the result is exact for every
// gate in [0, 1]; the finer levels only cost time (about 4x and 64x per affected chunk).
// log2 of a gate is clamped at -200 so that alpha = 0 gives a factor of 0, not a NaN.
// Sequence parallelism: the tokens of a sequence are split into segments of whole chunks.
//   pass 1 (OUTPUT = false): each segment's end state from a zero start, and its total log2 decay;
//   carry:                   S_start(0) = S0, S_start(s+1) = diag(2^{L_s}) S_start(s) + S_loc(s),
//                            one thread per state element, written over S_loc in the workspace;
//   pass 2 (OUTPUT = true):  each segment runs its chunks from S_start and writes o.
// The value dimension is split in BV = 64 column slices (columns of S are independent).
// CTA = 4 warps, three CTAs per SM. Warp w computes output rows [16w, 16w+16) of a chunk and state
// rows [w*D/4, (w+1)*D/4).
#pragma once

#include "kta_ptx.cuh"
#include "mma_sync.cuh"

namespace kta {

#ifndef KTA_GLA_LIM
#define KTA_GLA_LIM 64.0f
#endif

struct GlaParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* alpha;      // [B][rows][H][D]
  __nv_bfloat16* o;
  long long ld;            // q / k / v / o row stride (elements)
  int rows_b;              // rows per sequence in q / k / v / o / alpha
  int N;                   // tokens per sequence in this call
  int H;                   // heads in this call
  int seg_len;             // tokens per segment (multiple of C)
  int nseg;
  float scale;
  const float* S0;         // [B][H][D][D] key-major, or null
  float* S_out;            // [B][H][D][D], or null
  float* ws_S;             // [B*H][nseg][D][D] segment end states (pass 1)
  float* ws_L;             // [B*H][nseg][D] segment total log2 decay (pass 1)
  float* S_fold;           // carry kernel: also write the state after the last segment here
};

template <int D, int C>
struct GlaSmem {
  static constexpr int BV = 64;
  static constexpr int LDK = D + 8;   // padded rows: conflict-free ldmatrix
  static constexpr int LDV = BV + 8;
  __nv_bfloat16 q[C * LDK];   // raw q, then Qi
  __nv_bfloat16 k[C * LDK];   // raw k, then Ki
  __nv_bfloat16 v[C * LDV];
  __nv_bfloat16 s[D * LDV];   // bf16 copy of diag(2^{b_m}) S_0 (value slice)
  float emid[D];              // 2^{b_m}
  float cend[D];              // 2^{b_C - b_m}
};

template <int D, int C, bool OUTPUT>
__global__ void __launch_bounds__(128, 3) gla_chunk_kernel(const GlaParams p) {
  using SM = GlaSmem<D, C>;
  constexpr int BV = SM::BV, LDK = SM::LDK, LDV = SM::LDV;
  constexpr int RW = D / 4;           // state rows per warp
  constexpr int MT = RW / 16;         // m16 tiles of state per warp
  constexpr int NT = BV / 8;          // n8 tiles across the value slice
  constexpr int RT = C / 16;          // 16-row query tiles per chunk
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int seg = blockIdx.x, slice = blockIdx.y, bh = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  const int j0 = slice * BV;
  const int t_begin = seg * p.seg_len;
  const int t_end = min(p.N, t_begin + p.seg_len);
  const long long row_b = static_cast<long long>(b) * p.rows_b;

  // ---- state fragment registers: st[mt][nt][r] = S[row][j0 + col]
  float st[MT][NT][4];
  auto srow = [&](int mt, int r) { return warp * RW + mt * 16 + g4 + (r >= 2 ? 8 : 0); };
  auto scol = [&](int nt, int r) { return nt * 8 + 2 * t4 + (r & 1); };
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) st[mt][nt][r] = 0.f;

  if (OUTPUT) {
    // start state: S0 for a single segment, else the carry kernel's S_start of this segment
    const float* Ss = p.nseg > 1 ? p.ws_S + (static_cast<long long>(bh) * p.nseg + seg) * D * D
                                 : (p.S0 ? p.S0 + static_cast<long long>(bh) * D * D : nullptr);
    if (Ss) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) st[mt][nt][r] = Ss[srow(mt, r) * D + j0 + scol(nt, r)];
    }
  }
  float ltot = 0.f;  // this thread's key dim (tid < D): total log2 decay over the segment

  // Scale the state rows by 2^{b_m} (registers) and keep a bf16 copy for the inter-chunk product.
  auto prescale_and_publish = [&]() {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const float ea = sm.emid[srow(mt, 0)], eb = sm.emid[srow(mt, 2)];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        st[mt][nt][0] *= ea;
        st[mt][nt][1] *= ea;
        st[mt][nt][2] *= eb;
        st[mt][nt][3] *= eb;
        if (OUTPUT) {
          const int r0 = srow(mt, 0), c0 = scol(nt, 0);
          *reinterpret_cast<uint32_t*>(&sm.s[r0 * LDV + c0]) = bf16x2(st[mt][nt][0], st[mt][nt][1]);
          *reinterpret_cast<uint32_t*>(&sm.s[(r0 + 8) * LDV + c0]) = bf16x2(st[mt][nt][2], st[mt][nt][3]);
        }
      }
    }
  };

  // Spans: C tokens (level 0), 16-token sub-spans (level 1) or single tokens (level 2) when the
  // coarser span's decayed operands would leave the representable range. lvl_end[l] is where the
  // region handed down to level l ends.
  int lvl = 0;
  int lvl_end[3] = {t_end, t_end, t_end};
  for (int c0 = t_begin; c0 < t_end;) {
    const int span = lvl == 0 ? C : (lvl == 1 ? 16 : 1);
    const int n = min(span, min(t_end, lvl_end[lvl]) - c0);
    const int mid = n >> 1;
    // ---- load the span: q, k (OUTPUT only for q), v slice, alpha (rows >= n: zeros / alpha = 1)
    {
      constexpr int QCH = D / 8;  // 16-byte pieces per bf16 row
      for (int idx = tid; idx < C * QCH; idx += 128) {
        const int t = idx / QCH, c = (idx % QCH) * 8;
        const long long grow = row_b + c0 + min(t, n - 1);
        const int bytes = t < n ? 16 : 0;
        const long long off = grow * p.ld + static_cast<long long>(h) * D + c;
        if (OUTPUT) cp_async16(&sm.q[t * LDK + c], p.q + off, bytes);
        cp_async16(&sm.k[t * LDK + c], p.k + off, bytes);
      }
      constexpr int VCH = BV / 8;
      for (int idx = tid; idx < C * VCH; idx += 128) {
        const int t = idx / VCH, c = (idx % VCH) * 8;
        const long long grow = row_b + c0 + min(t, n - 1);
        cp_async16(&sm.v[t * LDV + c], p.v + grow * p.ld + static_cast<long long>(h) * D + j0 + c,
                   t < n ? 16 : 0);
      }
      cp_async_commit();
    }
    // gates of this thread's key column (rows >= n: alpha = 1), loaded straight into registers
    // while the copies above are in flight; bt[t] becomes the cumulative log2 gate below
    float bt[C];
    if (tid < D) {
      const float* ap = p.alpha + ((row_b + c0) * p.H + h) * D + tid;
#pragma unroll
      for (int t = 0; t < C; ++t) bt[t] = t < n ? __ldg(ap + static_cast<long long>(t) * p.H * D) : 1.f;
    }
    // ---- per key dim (thread tid < D owns column tid): the cumulative log2 gate b_t in
    // registers and the range check of the decayed operands against the middle token
    float bm = 0.f, acc = 0.f;
    bool in_range = true;
    if (tid < D) {
#pragma unroll
      for (int t = 0; t < C; ++t) {
        acc += fmaxf(__log2f(bt[t]), -200.f);
        bt[t] = acc;
      }
#pragma unroll
      for (int t = 0; t < C; ++t) bm = t == mid ? bt[t] : bm;
      float dev = 0.f;
#pragma unroll
      for (int t = 0; t < C; ++t) dev = fmaxf(dev, fabsf(bt[t] - bm));
      in_range = !(dev > KTA_GLA_LIM);
    }
    if (lvl < 2 && !__syncthreads_and(in_range ? 1 : 0)) {
      // redo this span at the next finer level (the copies above are simply overwritten)
      cp_async_wait_all();
      __syncthreads();
      const int next = (lvl == 0 && C > 16) ? 1 : 2;
      lvl_end[next] = c0 + n;
      if (lvl == 0 && next == 2) lvl_end[1] = c0 + n;
      lvl = next;
      continue;
    }
    cp_async_wait_all();
    __syncthreads();
    // the factors 2^{b_m}, 2^{b_C - b_m}, and the decayed operands of this thread's column,
    // Ki_t = k_t 2^{b_m - b_t} and Qi_t = q_t 2^{b_t - b_m}, written in place
    if (tid < D) {
      sm.emid[tid] = ex2_approx(bm);
      sm.cend[tid] = ex2_approx(acc - bm);
      ltot += acc;
#pragma unroll
      for (int t = 0; t < C; ++t) {
        const float dd = bt[t] - bm;
        sm.k[t * LDK + tid] = __float2bfloat16_rn(__bfloat162float(sm.k[t * LDK + tid]) * ex2_approx(-dd));
        if (OUTPUT)
          sm.q[t * LDK + tid] = __float2bfloat16_rn(__bfloat162float(sm.q[t * LDK + tid]) * ex2_approx(dd));
      }
    }
    __syncthreads();
    prescale_and_publish();
    __syncthreads();

    if (OUTPUT && warp < RT) {
      const int r0 = warp * 16;
      // intra-chunk scores A = Qi Ki^T, causal part only (key tiles up to this warp's rows)
      uint32_t aq[D / 16][4];
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) ldsm_x4(aq[kk], &sm.q[frag_a_rowmajor(lane, r0, kk * 16, LDK)]);
      float acc[C / 8][4];
#pragma unroll
      for (int nt = 0; nt < C / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[nt][r] = 0.f;
#pragma unroll
      for (int np = 0; np < C / 16; ++np) {
        if (np > warp) break;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t bk[4];
          ldsm_x4(bk, &sm.k[frag_b_nmajor(lane, np * 16, kk * 16, LDK)]);
          mma16816(acc[2 * np], aq[kk], bk[0], bk[1]);
          mma16816(acc[2 * np + 1], aq[kk], bk[2], bk[3]);
        }
      }
      // causal mask (s <= t) and conversion to bf16 A fragments
      uint32_t pa[C / 16][4];
#pragma unroll
      for (int nt = 0; nt < C / 8; ++nt) {
        const int col = nt * 8 + 2 * t4;
        const int ra = r0 + g4, rb = r0 + g4 + 8;
        const float x0 = col <= ra ? acc[nt][0] : 0.f;
        const float x1 = col + 1 <= ra ? acc[nt][1] : 0.f;
        const float x2 = col <= rb ? acc[nt][2] : 0.f;
        const float x3 = col + 1 <= rb ? acc[nt][3] : 0.f;
        pa[nt >> 1][(nt & 1) * 2 + 0] = bf16x2(x0, x1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = bf16x2(x2, x3);
      }
      float ov[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) ov[nt][r] = 0.f;
      // O = A V  (tokens up to this warp's rows)
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        if (kk > warp) break;
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t bv[4];
          ldsm_x4_t(bv, &sm.v[frag_b_kmajor(lane, kk * 16, np * 16, LDV)]);
          mma16816(ov[2 * np], pa[kk], bv[0], bv[1]);
          mma16816(ov[2 * np + 1], pa[kk], bv[2], bv[3]);
        }
      }
      // O += Qi diag(2^{b_m}) S_0
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t bs[4];
          ldsm_x4_t(bs, &sm.s[frag_b_kmajor(lane, kk * 16, np * 16, LDV)]);
          mma16816(ov[2 * np], aq[kk], bs[0], bs[1]);
          mma16816(ov[2 * np + 1], aq[kk], bs[2], bs[3]);
        }
      }
      // store rows < n
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int t = r0 + g4 + hr * 8;
        if (t < n) {
          __nv_bfloat16* orow = p.o + (row_b + c0 + t) * p.ld + static_cast<long long>(h) * D + j0;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            *reinterpret_cast<uint32_t*>(orow + nt * 8 + 2 * t4) =
                bf16x2(ov[nt][2 * hr] * p.scale, ov[nt][2 * hr + 1] * p.scale);
        }
      }
    }

    // ---- state update: S = diag(2^{b_C - b_m}) (diag(2^{b_m}) S + Ki^T V)  (all warps)
#pragma unroll
    for (int kk = 0; kk < C / 16; ++kk) {
      uint32_t bv[NT / 2][4];
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) ldsm_x4_t(bv[np], &sm.v[frag_b_kmajor(lane, kk * 16, np * 16, LDV)]);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t ak[4];
        ldsm_x4_t(ak, &sm.k[frag_a_kmajor(lane, warp * RW + mt * 16, kk * 16, LDK)]);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          mma16816(st[mt][2 * np], ak, bv[np][0], bv[np][1]);
          mma16816(st[mt][2 * np + 1], ak, bv[np][2], bv[np][3]);
        }
      }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const float ca = sm.cend[srow(mt, 0)], cb = sm.cend[srow(mt, 2)];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        st[mt][nt][0] *= ca;
        st[mt][nt][1] *= ca;
        st[mt][nt][2] *= cb;
        st[mt][nt][3] *= cb;
      }
    }
    __syncthreads();
    c0 += n;
    while (lvl > 0 && c0 >= lvl_end[lvl]) --lvl;
  }

  if (!OUTPUT) {
    float* Sl = p.ws_S + (static_cast<long long>(bh) * p.nseg + seg) * D * D;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) Sl[srow(mt, r) * D + j0 + scol(nt, r)] = st[mt][nt][r];
    if (slice == 0 && tid < D) p.ws_L[(static_cast<long long>(bh) * p.nseg + seg) * D + tid] = ltot;
  } else if (seg == p.nseg - 1 && p.S_out) {
    float* So = p.S_out + static_cast<long long>(bh) * D * D;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) So[srow(mt, r) * D + j0 + scol(nt, r)] = st[mt][nt][r];
  }
}

// Segment carry: for one (sequence, head) and one state element (i, j), walk the segments in
// order, replacing each segment's local end state by the state at its start:
//   S_start(0) = S0 (or 0),  S_start(s+1) = 2^{L_s[i]} S_start(s) + S_loc(s).
// All loads of a group of segments are issued before the dependent chain of FMAs.
template <int D>
__global__ void __launch_bounds__(128) gla_carry_kernel(const GlaParams p) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 128 + threadIdx.x;  // element index i * D + j
  if (e >= D * D) return;
  const int i = e / D;
  float cur = p.S0 ? p.S0[static_cast<long long>(bh) * D * D + e] : 0.f;
  float* S = p.ws_S + static_cast<long long>(bh) * p.nseg * D * D + e;
  const float* L = p.ws_L + static_cast<long long>(bh) * p.nseg * D + i;
  constexpr int G = 8;
  for (int s0 = 0; s0 < p.nseg; s0 += G) {
    float sl[G], dl[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const bool in = s0 + u < p.nseg;
      sl[u] = in ? S[static_cast<long long>(s0 + u) * D * D] : 0.f;
      dl[u] = in ? L[static_cast<long long>(s0 + u) * D] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < G; ++u) {
      if (s0 + u < p.nseg) {
        S[static_cast<long long>(s0 + u) * D * D] = cur;
        cur = fmaf(exp2f(dl[u]), cur, sl[u]);
      }
    }
  }
  if (p.S_fold) p.S_fold[static_cast<long long>(bh) * D * D + e] = cur;
}

}  // namespace kta
