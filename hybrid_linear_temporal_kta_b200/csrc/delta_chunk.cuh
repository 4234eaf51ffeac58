// delta_chunk.cuh -- chunked gated delta rule (bf16 in / out, fp32 state and gates) on
// warp-level bf16 tensor-core tiles.
//
// Operator: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar, the four update lines (v_old = M k, v_new = beta v + (1-beta) v_old,
// M = alpha M - v_old k^T + v_new k^T, o = M q). With the key-major state S = M^T (d_k x d_v)
// and row vectors this is  u_t = beta_t (v_t - k_t S_{t-1}),  S_t = alpha_t S_{t-1} + k_t^T u_t,
// o_t = scale * q_t S_t.
//
// Chunked form (derived by unrolling inside a chunk of C tokens; gamma_t = prod_{r<=t} alpha_r,
// gamma_{-1} = 1, S_0 the state at the chunk start):
//   (I + T) U = diag(beta) V - diag(beta_t gamma_{t-1}) K S_0,
//        T_ts = beta_t (gamma_{t-1} / gamma_s) (k_t . k_s)          for s < t
//   o_t   = scale * [ gamma_t q_t S_0 + sum_{s<=t} (gamma_t / gamma_s) (q_t . k_s) u_s ]
//   S_end = gamma_end S_0 + sum_s k_s^T (gamma_end / gamma_s) u_s
// (I + T) is unit lower triangular. Its four 16 x 16 diagonal blocks are inverted in fp32 by
// forward substitution; U follows by block forward substitution on the tensor cores:
//   U_i = X_ii (R_i - sum_{j<i} T_ij U_j).
// CTA = 4 warps over (sequence, head, value slice of BV = 32 columns); chunks in order, state in
// registers. Warp w owns value columns [8w, 8w+8) in the substitution, query rows [16w, 16w+16)
// of the output, and state rows [32w, 32w+32).
#pragma once

#include "mma_sync.cuh"

namespace kta {

struct DeltaParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* alpha;     // [B][rows][H]
  const float* beta;      // [B][rows][H]
  __nv_bfloat16* o;
  long long ld;
  int rows_b;
  int N;
  int H;
  float scale;
  const float* S0;        // [B][H][D][D] key-major, or null
  float* S_out;           // or null
};

template <int D>
struct DeltaSmem {
  static constexpr int C = 64;
  static constexpr int BV = 32;
  static constexpr int LDK = D + 8;
  static constexpr int LDV = BV + 8;
  static constexpr int LDC = C + 8;
  __nv_bfloat16 q[C * LDK];
  __nv_bfloat16 k[C * LDK];
  __nv_bfloat16 v[C * LDV];
  __nv_bfloat16 s[D * LDV];     // bf16 chunk-start state slice
  __nv_bfloat16 u[C * LDV];     // U (and the block right-hand sides while solving)
  __nv_bfloat16 ur[C * LDV];    // diag(gamma_end / gamma_s) U
  __nv_bfloat16 tb[C * LDC];    // T in bf16 (off-diagonal blocks are used)
  __nv_bfloat16 aq[C * LDC];    // (gamma_t / gamma_s) (q_t . k_s), s <= t
  __nv_bfloat16 xd[4][16 * 24]; // inverses of the 16 x 16 diagonal blocks of I + T
  float tf[C * (C + 1)];        // T in fp32 (diagonal blocks are inverted from it)
  float lg[C];                  // cumulative log2 alpha
  float beta[C];
};

template <int D>
__global__ void __launch_bounds__(128) delta_chunk_kernel(const DeltaParams p) {
  using SM = DeltaSmem<D>;
  constexpr int C = SM::C, BV = SM::BV, LDK = SM::LDK, LDV = SM::LDV, LDC = SM::LDC;
  constexpr int LDT = C + 1;
  constexpr int RW = D / 4, MT = RW / 16;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int slice = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int j0 = slice * BV;
  const long long row_b = static_cast<long long>(b) * p.rows_b;

  // state rows [warp*RW, +RW) x BV columns: st[mt][nt][r]
  float st[MT][BV / 8][4];
  auto srow = [&](int mt, int r) { return warp * RW + mt * 16 + g4 + (r >= 2 ? 8 : 0); };
  auto scol = [&](int nt, int r) { return nt * 8 + 2 * t4 + (r & 1); };
  const long long sb = static_cast<long long>(bh) * D * D;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < BV / 8; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r)
        st[mt][nt][r] = p.S0 ? p.S0[sb + srow(mt, r) * D + j0 + scol(nt, r)] : 0.f;

  auto write_state_smem = [&]() {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < BV / 8; ++nt) {
        const int r0 = srow(mt, 0), c0 = scol(nt, 0);
        *reinterpret_cast<uint32_t*>(&sm.s[r0 * LDV + c0]) = bf16x2(st[mt][nt][0], st[mt][nt][1]);
        *reinterpret_cast<uint32_t*>(&sm.s[(r0 + 8) * LDV + c0]) = bf16x2(st[mt][nt][2], st[mt][nt][3]);
      }
  };
  write_state_smem();

  for (int c0 = 0; c0 < p.N; c0 += C) {
    const int n = min(C, p.N - c0);
    // ---- load q, k (full head dim), v slice; gates
    {
      constexpr int QCH = D / 8;
      for (int idx = tid; idx < C * QCH; idx += 128) {
        const int t = idx / QCH, c = (idx % QCH) * 8;
        const long long grow = row_b + c0 + min(t, n - 1);
        const long long off = grow * p.ld + static_cast<long long>(h) * D + c;
        const int bytes = t < n ? 16 : 0;
        cp_async16(&sm.q[t * LDK + c], p.q + off, bytes);
        cp_async16(&sm.k[t * LDK + c], p.k + off, bytes);
      }
      constexpr int VCH = BV / 8;
      for (int idx = tid; idx < C * VCH; idx += 128) {
        const int t = idx / VCH, c = (idx % VCH) * 8;
        const long long grow = row_b + c0 + min(t, n - 1);
        cp_async16(&sm.v[t * LDV + c], p.v + grow * p.ld + static_cast<long long>(h) * D + j0 + c,
                   t < n ? 16 : 0);
      }
      if (warp == 0) {
        // cumulative log2 alpha over the chunk (two tokens per lane, warp scan); padding rows
        // have alpha = 1 and beta = 0.
        float a0 = 0.f, a1 = 0.f;
        const int t0 = 2 * lane, t1 = 2 * lane + 1;
        const long long r0 = (row_b + c0 + t0) * p.H + h, r1 = (row_b + c0 + t1) * p.H + h;
        if (t0 < n) { a0 = __log2f(p.alpha[r0]); sm.beta[t0] = p.beta[r0]; } else sm.beta[t0] = 0.f;
        if (t1 < n) { a1 = __log2f(p.alpha[r1]); sm.beta[t1] = p.beta[r1]; } else sm.beta[t1] = 0.f;
        float pair = a0 + a1;
        float incl = pair;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, incl, o2);
          if (lane >= o2) incl += y;
        }
        const float excl = incl - pair;
        sm.lg[t0] = excl + a0;
        sm.lg[t1] = excl + a0 + a1;
      }
      cp_async_wait_all();
    }
    __syncthreads();

    // ---- K K^T and Q K^T for query rows [16w, 16w+16): T (s < t) and decayed QK (s <= t)
    {
      const int r0 = warp * 16;
      uint32_t ak[D / 16][4], aqf[D / 16][4];
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        ldsm_x4(ak[kk], &sm.k[frag_a_rowmajor(lane, r0, kk * 16, LDK)]);
        ldsm_x4(aqf[kk], &sm.q[frag_a_rowmajor(lane, r0, kk * 16, LDK)]);
      }
      float kk_acc[C / 8][4], qk_acc[C / 8][4];
#pragma unroll
      for (int nt = 0; nt < C / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) kk_acc[nt][r] = qk_acc[nt][r] = 0.f;
#pragma unroll
      for (int np = 0; np < C / 16; ++np) {
        if (np > warp) break;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t bk[4];
          ldsm_x4(bk, &sm.k[frag_b_nmajor(lane, np * 16, kk * 16, LDK)]);
          mma16816(kk_acc[2 * np], ak[kk], bk[0], bk[1]);
          mma16816(kk_acc[2 * np + 1], ak[kk], bk[2], bk[3]);
          mma16816(qk_acc[2 * np], aqf[kk], bk[0], bk[1]);
          mma16816(qk_acc[2 * np + 1], aqf[kk], bk[2], bk[3]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < C / 8; ++nt) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = r0 + g4 + (r >= 2 ? 8 : 0);
          const int s = nt * 8 + 2 * t4 + (r & 1);
          const float lgt = sm.lg[t], lgs = sm.lg[s];
          const float lgp = t > 0 ? sm.lg[t - 1] : 0.f;
          const float tv = s < t ? sm.beta[t] * exp2f(lgp - lgs) * kk_acc[nt][r] : 0.f;
          const float av = s <= t ? exp2f(lgt - lgs) * qk_acc[nt][r] : 0.f;
          sm.tf[t * LDT + s] = tv;
          kk_acc[nt][r] = tv;
          qk_acc[nt][r] = av;
        }
        const int t = r0 + g4, s = nt * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(&sm.tb[t * LDC + s]) = bf16x2(kk_acc[nt][0], kk_acc[nt][1]);
        *reinterpret_cast<uint32_t*>(&sm.tb[(t + 8) * LDC + s]) = bf16x2(kk_acc[nt][2], kk_acc[nt][3]);
        *reinterpret_cast<uint32_t*>(&sm.aq[t * LDC + s]) = bf16x2(qk_acc[nt][0], qk_acc[nt][1]);
        *reinterpret_cast<uint32_t*>(&sm.aq[(t + 8) * LDC + s]) = bf16x2(qk_acc[nt][2], qk_acc[nt][3]);
      }
    }
    __syncthreads();

    // ---- invert diagonal block `warp` of I + T (lane c < 16 owns column c), fp32
    {
      const int base = warp * 16;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) x[r] = (r == lane) ? 1.f : 0.f;
#pragma unroll
      for (int r = 1; r < 16; ++r) {
        float acc = x[r];
#pragma unroll
        for (int s = 0; s < r; ++s) acc = fmaf(-sm.tf[(base + r) * LDT + base + s], x[s], acc);
        x[r] = acc;
      }
      if (lane < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) sm.xd[warp][r * 24 + lane] = __float2bfloat16_rn(x[r]);
      }
    }

    // ---- R = diag(beta) V - diag(beta_t gamma_{t-1}) K S_0 for value columns [8w, 8w+8)
    float racc[C / 16][4];
    {
#pragma unroll
      for (int mt = 0; mt < C / 16; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) racc[mt][r] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // B = S_0 rows [16kk, 16kk+16) x this warp's 8 value columns
        uint32_t bs[2];
        ldsm_x2_t(bs, &sm.s[frag_b_kmajor(lane, kk * 16, warp * 8, LDV)]);
#pragma unroll
        for (int mt = 0; mt < C / 16; ++mt) {
          uint32_t a[4];
          ldsm_x4(a, &sm.k[frag_a_rowmajor(lane, mt * 16, kk * 16, LDK)]);
          mma16816(racc[mt], a, bs[0], bs[1]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < C / 16; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = mt * 16 + g4 + (r >= 2 ? 8 : 0);
          const int col = warp * 8 + 2 * t4 + (r & 1);
          const float gp = t > 0 ? exp2f(sm.lg[t - 1]) : 1.f;
          const float bt = sm.beta[t];
          racc[mt][r] = bt * __bfloat162float(sm.v[t * LDV + col]) - bt * gp * racc[mt][r];
        }
    }
    __syncthreads();  // diagonal inverses visible to every warp

    // ---- block forward substitution for this warp's 8 value columns
#pragma unroll
    for (int i = 0; i < C / 16; ++i) {
      float y[4] = {racc[i][0], racc[i][1], racc[i][2], racc[i][3]};
#pragma unroll
      for (int j = 0; j < C / 16; ++j) {
        if (j >= i) break;
        uint32_t a[4], bu[2];
        ldsm_x4(a, &sm.tb[frag_a_rowmajor(lane, i * 16, j * 16, LDC)]);
        ldsm_x2_t(bu, &sm.u[frag_b_kmajor(lane, j * 16, warp * 8, LDV)]);
        float tmp[4] = {0.f, 0.f, 0.f, 0.f};
        mma16816(tmp, a, bu[0], bu[1]);
#pragma unroll
        for (int r = 0; r < 4; ++r) y[r] -= tmp[r];
      }
      // stage Y_i (bf16) in the U rows of block i, then U_i = X_ii Y_i
      const int t = i * 16 + g4, col = warp * 8 + 2 * t4;
      *reinterpret_cast<uint32_t*>(&sm.u[t * LDV + col]) = bf16x2(y[0], y[1]);
      *reinterpret_cast<uint32_t*>(&sm.u[(t + 8) * LDV + col]) = bf16x2(y[2], y[3]);
      __syncwarp();
      uint32_t a[4], by[2];
      ldsm_x4(a, &sm.xd[i][frag_a_rowmajor(lane, 0, 0, 24)]);
      ldsm_x2_t(by, &sm.u[frag_b_kmajor(lane, i * 16, warp * 8, LDV)]);
      float uo[4] = {0.f, 0.f, 0.f, 0.f};
      mma16816(uo, a, by[0], by[1]);
      __syncwarp();
      *reinterpret_cast<uint32_t*>(&sm.u[t * LDV + col]) = bf16x2(uo[0], uo[1]);
      *reinterpret_cast<uint32_t*>(&sm.u[(t + 8) * LDV + col]) = bf16x2(uo[2], uo[3]);
      __syncwarp();
    }
    __syncthreads();  // U complete

    // ---- scaled U for the state update: ur_s = (gamma_end / gamma_s) u_s
    for (int idx = tid; idx < C * BV; idx += 128) {
      const int t = idx / BV, c = idx % BV;
      const float r = exp2f(sm.lg[C - 1] - sm.lg[t]);
      sm.ur[t * LDV + c] = __float2bfloat16_rn(r * __bfloat162float(sm.u[t * LDV + c]));
    }

    // ---- outputs for rows [16w, 16w+16): gamma_t q_t S_0 + Aq U
    {
      const int r0 = warp * 16;
      float ov[BV / 8][4];
#pragma unroll
      for (int nt = 0; nt < BV / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) ov[nt][r] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, &sm.q[frag_a_rowmajor(lane, r0, kk * 16, LDK)]);
#pragma unroll
        for (int np = 0; np < BV / 16; ++np) {
          uint32_t bs[4];
          ldsm_x4_t(bs, &sm.s[frag_b_kmajor(lane, kk * 16, np * 16, LDV)]);
          mma16816(ov[2 * np], a, bs[0], bs[1]);
          mma16816(ov[2 * np + 1], a, bs[2], bs[3]);
        }
      }
      const float ga = exp2f(sm.lg[r0 + g4]), gb = exp2f(sm.lg[r0 + g4 + 8]);
#pragma unroll
      for (int nt = 0; nt < BV / 8; ++nt) {
        ov[nt][0] *= ga;
        ov[nt][1] *= ga;
        ov[nt][2] *= gb;
        ov[nt][3] *= gb;
      }
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        if (kk > warp) break;
        uint32_t a[4];
        ldsm_x4(a, &sm.aq[frag_a_rowmajor(lane, r0, kk * 16, LDC)]);
#pragma unroll
        for (int np = 0; np < BV / 16; ++np) {
          uint32_t bu[4];
          ldsm_x4_t(bu, &sm.u[frag_b_kmajor(lane, kk * 16, np * 16, LDV)]);
          mma16816(ov[2 * np], a, bu[0], bu[1]);
          mma16816(ov[2 * np + 1], a, bu[2], bu[3]);
        }
      }
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int t = r0 + g4 + hr * 8;
        if (t < n) {
          __nv_bfloat16* orow = p.o + (row_b + c0 + t) * p.ld + static_cast<long long>(h) * D + j0;
#pragma unroll
          for (int nt = 0; nt < BV / 8; ++nt)
            *reinterpret_cast<uint32_t*>(orow + nt * 8 + 2 * t4) =
                bf16x2(ov[nt][2 * hr] * p.scale, ov[nt][2 * hr + 1] * p.scale);
        }
      }
    }
    __syncthreads();  // ur complete; every read of s done

    // ---- state: S = gamma_end S + K^T Ur
    {
      const float gend = exp2f(sm.lg[C - 1]);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < BV / 8; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) st[mt][nt][r] *= gend;
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        uint32_t bu[BV / 16][4];
#pragma unroll
        for (int np = 0; np < BV / 16; ++np) ldsm_x4_t(bu[np], &sm.ur[frag_b_kmajor(lane, kk * 16, np * 16, LDV)]);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          uint32_t a[4];
          ldsm_x4_t(a, &sm.k[frag_a_kmajor(lane, warp * RW + mt * 16, kk * 16, LDK)]);
#pragma unroll
          for (int np = 0; np < BV / 16; ++np) {
            mma16816(st[mt][2 * np], a, bu[np][0], bu[np][1]);
            mma16816(st[mt][2 * np + 1], a, bu[np][2], bu[np][3]);
          }
        }
      }
    }
    __syncthreads();
    write_state_smem();
  }
  if (p.S_out) {
    float* So = p.S_out + sb;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < BV / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) So[srow(mt, r) * D + j0 + scol(nt, r)] = st[mt][nt][r];
  }
}

}  // namespace kta
