// bwd_f32.cuh -- reverse mode of the operator in fp32 on CUDA cores (the first correct backward
// path; the tensor-core backward is not built).
//
// Operators: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar (SWA, DSWA, GLA and the gated delta-rule equations). Given dO, the kernels compute the
// gradients of L = sum(dO * O):
//   softmax windows: p_ts = softmax_s(scale q_t . k_s) over the visible keys, o_t = sum_s p_ts v_s,
//     ds_ts = p_ts (dO_t . v_s - dO_t . o_t), dq_t = scale sum_s ds_ts k_s,
//     dk_s = scale sum_t ds_ts q_t, dv_s = sum_t p_ts dO_t;
//   GLA (S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = scale q_t S_t), with the state adjoint
//     G_t = scale q_t^T dO_t + diag(alpha_{t+1}) G_{t+1}: dq_t = scale S_t dO_t^T,
//     dk_t = G_t v_t^T, dv_t = k_t G_t, dalpha_t[i] = sum_j G_t[i][j] S_{t-1}[i][j];
//   delta rule (w_t = k_t S_{t-1}, u_t = beta_t (v_t - a_t w_t), a_t = 1 or alpha_t for the
//     decayed erase, S_t = alpha_t S_{t-1} + k_t^T u_t), with du_t = k_t G_t:
//     dq_t = scale S_t dO_t^T, dv_t = beta_t du_t, dbeta_t = du_t . (v_t - a_t w_t),
//     dk_t = G_t u_t^T - beta_t a_t S_{t-1} du_t^T,
//     dalpha_t = <G_t, S_{t-1}> (- beta_t du_t . w_t for the decayed erase),
//     G_{t-1} = alpha_t G_t - beta_t a_t k_t^T du_t;  dS_0 = the adjoint left after token 0.
#pragma once

#include "kta_ptx.cuh"

namespace kta {

struct SoftmaxBwdParams {
  int B, N, P, H, d;
  int W, dil;
  long long ld;      // row stride of q / k / v / dO / dq / dk / dv (elements)
  float scale;
  float* stats;      // [3][B][H][N]: row maximum m, 1 / l, dO_t . o_t
};

// Layout shared by the two softmax-backward kernels. A warp takes SB_R = 4 rows of one frame
// (a CTA of 4 warps takes 16), its lanes own DPL = d / 32 consecutive dims of every row, and the
// other side (keys or queries) is walked SB_K = 8 rows at a time, so one block is 4 x 8 = 32
// (row, other) pairs: lane l ends up owning pair (l / 8, l % 8).
constexpr int SB_R = 4, SB_K = 8, SB_ROWS_CTA = 16;

template <int DPL>
__device__ __forceinline__ void load_dims(const float* __restrict__ row, bool ok, float (&x)[DPL]) {
  if constexpr (DPL == 4) {
    const float4 u = ok ? __ldg(reinterpret_cast<const float4*>(row)) : make_float4(0.f, 0.f, 0.f, 0.f);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
  } else if constexpr (DPL == 2) {
    const float2 u = ok ? __ldg(reinterpret_cast<const float2*>(row)) : make_float2(0.f, 0.f);
    x[0] = u.x; x[1] = u.y;
  } else {
    x[0] = ok ? __ldg(row) : 0.f;
  }
}

template <int DPL>
__device__ __forceinline__ void store_dims(float* row, const float (&x)[DPL], float mul) {
  if constexpr (DPL == 4) {
    *reinterpret_cast<float4*>(row) = make_float4(x[0] * mul, x[1] * mul, x[2] * mul, x[3] * mul);
  } else if constexpr (DPL == 2) {
    *reinterpret_cast<float2*>(row) = make_float2(x[0] * mul, x[1] * mul);
  } else {
    row[0] = x[0] * mul;
  }
}

// 32 per-lane partial sums v[0..31] -> lane l returns the warp-wide sum of entry l (a butterfly
// reduce-scatter: five exchange steps, each halving the entries a lane keeps).
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool hi = lane & half;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = hi ? v[i] : v[i + half];
      const float keep = hi ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

__device__ __forceinline__ float group8_max(float x) {
#pragma unroll
  for (int o = 4; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float group8_sum(float x) {
#pragma unroll
  for (int o = 4; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// dq pass. Per warp: 4 query rows of frame f. Pass 1 recomputes each row's maximum m, sum l and
// output o (online softmax over the visible key frames, oldest first); pass 2 forms
// ds_ts = p_ts (dO_t . v_s - dO_t . o_t) and dq_t = scale sum_s ds_ts k_s. The statistics
// (m, 1/l, dO_t . o_t) go to p.stats for the key-major pass.
template <int DPL>
__global__ void __launch_bounds__(128) softmax_bwd_q_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ dout, float* __restrict__ dq, const SoftmaxBwdParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = (p.P + SB_ROWS_CTA - 1) / SB_ROWS_CTA;
  const int f = blockIdx.x / groups;
  const int i0 = (blockIdx.x % groups) * SB_ROWS_CTA + warp * SB_R;  // row within the frame
  if (i0 >= p.P) return;
  const int h = blockIdx.y, b = blockIdx.z;
  const int d = p.d;
  const long long rb = static_cast<long long>(b) * p.N;
  const long long col = static_cast<long long>(h) * d + lane * DPL;
  float qr[SB_R][DPL], dr[SB_R][DPL], acc[SB_R][DPL];
  float m[SB_R], l[SB_R];
#pragma unroll
  for (int r = 0; r < SB_R; ++r) {
    const bool ok = i0 + r < p.P;
    const long long row = (rb + static_cast<long long>(f) * p.P + i0 + (ok ? r : 0)) * p.ld + col;
    load_dims<DPL>(q + row, ok, qr[r]);
    load_dims<DPL>(dout + row, ok, dr[r]);
#pragma unroll
    for (int c = 0; c < DPL; ++c) acc[r][c] = 0.f;
    m[r] = -INFINITY;
    l[r] = 0.f;
  }
  const int my_r = lane >> 3, my_j = lane & 7;
  const int nfr = min(p.W, f / p.dil + 1);
  // ---- pass 1: m, l, o
  for (int jf = nfr - 1; jf >= 0; --jf) {
    const long long base = rb + static_cast<long long>(f - jf * p.dil) * p.P;
    for (int s0 = 0; s0 < p.P; s0 += SB_K) {
      float part[32];
#pragma unroll
      for (int j = 0; j < SB_K; ++j) {
        float kj[DPL];
        const bool ok = s0 + j < p.P;
        load_dims<DPL>(k + (base + (ok ? s0 + j : 0)) * p.ld + col, ok, kj);
#pragma unroll
        for (int r = 0; r < SB_R; ++r) {
          float x = 0.f;
#pragma unroll
          for (int c = 0; c < DPL; ++c) x = fmaf(qr[r][c], kj[c], x);
          part[r * SB_K + j] = x;
        }
      }
      const float dot = reduce_scatter32(part, lane);
      const float sc = s0 + my_j < p.P ? dot * p.scale : -INFINITY;
      const float mx = group8_max(sc);
      float mnew[SB_R], corr[SB_R];
#pragma unroll
      for (int r = 0; r < SB_R; ++r) {
        mnew[r] = fmaxf(m[r], __shfl_sync(0xffffffffu, mx, r * SB_K));
        corr[r] = expf(m[r] - mnew[r]);
      }
      float mine = mnew[0];
#pragma unroll
      for (int r = 1; r < SB_R; ++r) mine = my_r == r ? mnew[r] : mine;
      const float pr = expf(sc - mine);
      const float ps = group8_sum(pr);
#pragma unroll
      for (int r = 0; r < SB_R; ++r) {
        l[r] = fmaf(l[r], corr[r], __shfl_sync(0xffffffffu, ps, r * SB_K));
        m[r] = mnew[r];
#pragma unroll
        for (int c = 0; c < DPL; ++c) acc[r][c] *= corr[r];
      }
#pragma unroll
      for (int j = 0; j < SB_K; ++j) {
        float vj[DPL];
        const bool ok = s0 + j < p.P;
        load_dims<DPL>(v + (base + (ok ? s0 + j : 0)) * p.ld + col, ok, vj);
#pragma unroll
        for (int r = 0; r < SB_R; ++r) {
          const float pj = __shfl_sync(0xffffffffu, pr, r * SB_K + j);
#pragma unroll
          for (int c = 0; c < DPL; ++c) acc[r][c] = fmaf(pj, vj[c], acc[r][c]);
        }
      }
    }
  }
  float inv[SB_R], Dr[SB_R];
#pragma unroll
  for (int r = 0; r < SB_R; ++r) {
    inv[r] = 1.f / l[r];
    float x = 0.f;
#pragma unroll
    for (int c = 0; c < DPL; ++c) x = fmaf(dr[r][c], acc[r][c] * inv[r], x);
    Dr[r] = warp_sum(x);
  }
  if (lane < SB_R && i0 + lane < p.P) {
    float mm = m[0], ii = inv[0], dd = Dr[0];
#pragma unroll
    for (int r = 1; r < SB_R; ++r)
      if (lane == r) { mm = m[r]; ii = inv[r]; dd = Dr[r]; }
    const long long si = (static_cast<long long>(b) * p.H + h) * p.N +
                         static_cast<long long>(f) * p.P + i0 + lane;
    const long long plane = static_cast<long long>(p.B) * p.H * p.N;
    p.stats[si] = mm;
    p.stats[plane + si] = ii;
    p.stats[2 * plane + si] = dd;
  }
  float m_mine = m[0], inv_mine = inv[0], D_mine = Dr[0];
#pragma unroll
  for (int r = 1; r < SB_R; ++r)
    if (my_r == r) { m_mine = m[r]; inv_mine = inv[r]; D_mine = Dr[r]; }
  // ---- pass 2: ds and dq (acc is reused for dq)
#pragma unroll
  for (int r = 0; r < SB_R; ++r)
#pragma unroll
    for (int c = 0; c < DPL; ++c) acc[r][c] = 0.f;
  for (int jf = nfr - 1; jf >= 0; --jf) {
    const long long base = rb + static_cast<long long>(f - jf * p.dil) * p.P;
    for (int s0 = 0; s0 < p.P; s0 += SB_K) {
      float ps[32], pd[32], kk[SB_K][DPL];
#pragma unroll
      for (int j = 0; j < SB_K; ++j) {
        float vj[DPL];
        const bool ok = s0 + j < p.P;
        const long long row = (base + (ok ? s0 + j : 0)) * p.ld + col;
        load_dims<DPL>(k + row, ok, kk[j]);
        load_dims<DPL>(v + row, ok, vj);
#pragma unroll
        for (int r = 0; r < SB_R; ++r) {
          float x = 0.f, y = 0.f;
#pragma unroll
          for (int c = 0; c < DPL; ++c) {
            x = fmaf(qr[r][c], kk[j][c], x);
            y = fmaf(dr[r][c], vj[c], y);
          }
          ps[r * SB_K + j] = x;
          pd[r * SB_K + j] = y;
        }
      }
      const float dot = reduce_scatter32(ps, lane);
      const float dp = reduce_scatter32(pd, lane);
      const float ds = s0 + my_j < p.P
                           ? expf(dot * p.scale - m_mine) * inv_mine * (dp - D_mine) : 0.f;
#pragma unroll
      for (int j = 0; j < SB_K; ++j)
#pragma unroll
        for (int r = 0; r < SB_R; ++r) {
          const float g = __shfl_sync(0xffffffffu, ds, r * SB_K + j);
#pragma unroll
          for (int c = 0; c < DPL; ++c) acc[r][c] = fmaf(g, kk[j][c], acc[r][c]);
        }
    }
  }
#pragma unroll
  for (int r = 0; r < SB_R; ++r)
    if (i0 + r < p.P)
      store_dims<DPL>(dq + (rb + static_cast<long long>(f) * p.P + i0 + r) * p.ld + col, acc[r],
                      p.scale);
}

// dk / dv pass. Per warp: 4 key rows of frame g, visible to query frames g, g + dil, ...,
// g + (W-1) dil (those < F). For 8 queries at a time it forms S and dP for the 32 (key, query)
// pairs, p = exp(scale S - m) / l and ds = p (dP - dO . o) from the stored statistics, then
// dv_s += p dO_t and dk_s += scale ds q_t.
template <int DPL>
__global__ void __launch_bounds__(128) softmax_bwd_kv_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ dout, float* __restrict__ dk, float* __restrict__ dv,
    const SoftmaxBwdParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = (p.P + SB_ROWS_CTA - 1) / SB_ROWS_CTA;
  const int g = blockIdx.x / groups;
  const int i0 = (blockIdx.x % groups) * SB_ROWS_CTA + warp * SB_R;
  if (i0 >= p.P) return;
  const int h = blockIdx.y, b = blockIdx.z;
  const int d = p.d, F = p.N / p.P;
  const long long rb = static_cast<long long>(b) * p.N;
  const long long col = static_cast<long long>(h) * d + lane * DPL;
  float kr[SB_R][DPL], vr[SB_R][DPL], gk[SB_R][DPL], gv[SB_R][DPL];
#pragma unroll
  for (int r = 0; r < SB_R; ++r) {
    const bool ok = i0 + r < p.P;
    const long long row = (rb + static_cast<long long>(g) * p.P + i0 + (ok ? r : 0)) * p.ld + col;
    load_dims<DPL>(k + row, ok, kr[r]);
    load_dims<DPL>(v + row, ok, vr[r]);
#pragma unroll
    for (int c = 0; c < DPL; ++c) gk[r][c] = gv[r][c] = 0.f;
  }
  const int my_j = lane & 7;
  const long long plane = static_cast<long long>(p.B) * p.H * p.N;
  const float* sm = p.stats + (static_cast<long long>(b) * p.H + h) * p.N;
  for (int j = 0; j < p.W; ++j) {
    const int f = g + j * p.dil;
    if (f >= F) break;
    const long long fb = static_cast<long long>(f) * p.P;
    for (int t0 = 0; t0 < p.P; t0 += SB_K) {
      float ps[32], pd[32], qq[SB_K][DPL], dd[SB_K][DPL];
#pragma unroll
      for (int jj = 0; jj < SB_K; ++jj) {
        const bool ok = t0 + jj < p.P;
        const long long row = (rb + fb + (ok ? t0 + jj : 0)) * p.ld + col;
        load_dims<DPL>(q + row, ok, qq[jj]);
        load_dims<DPL>(dout + row, ok, dd[jj]);
#pragma unroll
        for (int r = 0; r < SB_R; ++r) {
          float x = 0.f, y = 0.f;
#pragma unroll
          for (int c = 0; c < DPL; ++c) {
            x = fmaf(kr[r][c], qq[jj][c], x);
            y = fmaf(vr[r][c], dd[jj][c], y);
          }
          ps[r * SB_K + jj] = x;
          pd[r * SB_K + jj] = y;
        }
      }
      const float dot = reduce_scatter32(ps, lane);
      const float dpv = reduce_scatter32(pd, lane);
      float pr = 0.f, ds = 0.f;
      if (t0 + my_j < p.P) {
        const long long si = fb + t0 + my_j;
        pr = expf(dot * p.scale - sm[si]) * sm[plane + si];
        ds = pr * (dpv - sm[2 * plane + si]);
      }
#pragma unroll
      for (int jj = 0; jj < SB_K; ++jj)
#pragma unroll
        for (int r = 0; r < SB_R; ++r) {
          const float pj = __shfl_sync(0xffffffffu, pr, r * SB_K + jj);
          const float gj = __shfl_sync(0xffffffffu, ds, r * SB_K + jj);
#pragma unroll
          for (int c = 0; c < DPL; ++c) {
            gv[r][c] = fmaf(pj, dd[jj][c], gv[r][c]);
            gk[r][c] = fmaf(gj, qq[jj][c], gk[r][c]);
          }
        }
    }
  }
#pragma unroll
  for (int r = 0; r < SB_R; ++r)
    if (i0 + r < p.P) {
      const long long row = (rb + static_cast<long long>(g) * p.P + i0 + r) * p.ld + col;
      store_dims<DPL>(dk + row, gk[r], p.scale);
      store_dims<DPL>(dv + row, gv[r], 1.f);
    }
}

constexpr int BWD_CK = 32;  // tokens between stored states in the linear-branch backward

struct LinBwdParams {
  const float *q, *k, *v, *alpha, *beta, *S0, *dout;
  float *dq, *dk, *dv, *dalpha, *dbeta, *dS0;
  long long ld;        // row stride of q / k / v / dO / dq / dk / dv (elements)
  int rows_b, N, H;
  float scale;
  int delta, erase_decayed;
  int seg_len, nseg;   // vector GLA: tokens per segment and segments per sequence
  int nck;             // delta rule: stored states per sequence = ceil(N / BWD_CK)
  float* ws;           // delta rule, per (sequence, head): states [nck][D][D], chunk
                       // [BWD_CK][D][D], u, w
  // vector GLA with nseg > 1 only, per (sequence, head, segment) [D][D] (key-major):
  const float* Sin;    // state before the segment's first token
  const float* Gin;    // adjoint entering the segment's last token from the right
};

template <int D>
__host__ __device__ constexpr long long lin_bwd_ws_floats(int nck) {
  return (static_cast<long long>(nck) + BWD_CK) * D * D + 2LL * BWD_CK * D;
}

// Segment summaries of the vector-GLA backward, one CTA of D threads per (segment, head,
// sequence), thread j owning column j. From a zero state over the segment's tokens [t0, t1):
//   E = the end state, c = prod_t alpha_t (all tokens), cx = prod_{t > t0} alpha_t,
//   R = the adjoint at t0 from the segment's own outputs (G_t = scale q_t^T dO_t +
//       diag(alpha_{t+1}) G_{t+1}, zero beyond t1 - 1).
// sum: per (sequence, head, segment) E [D][D], R [D][D], c [D], cx [D].
template <int D>
__global__ void __launch_bounds__(D) gla_bwd_summary_kernel(const LinBwdParams p, float* sum) {
  __shared__ float qv[D], kv[D], av[D];
  const int j = threadIdx.x;
  const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = seg * p.seg_len, t1 = min(p.N, t0 + p.seg_len);
  const long long rb = static_cast<long long>(b) * p.rows_b;
  float* E = sum + ((static_cast<long long>(b) * p.H + h) * p.nseg + seg) * (2LL * D * D + 2 * D);
  float* R = E + D * D;
  float* c = R + D * D;
  float* cx = c + D;
  float X[D];
#pragma unroll
  for (int i = 0; i < D; ++i) X[i] = 0.f;
  float cj = 1.f, cxj = 1.f;
  for (int t = t0; t < t1; ++t) {
    const long long r = (rb + t) * p.ld + static_cast<long long>(h) * D;
    __syncthreads();
    kv[j] = p.k[r + j];
    av[j] = p.alpha[((rb + t) * p.H + h) * D + j];
    const float vj = p.v[r + j];
    __syncthreads();
    cj *= av[j];
    if (t > t0) cxj *= av[j];
#pragma unroll
    for (int i = 0; i < D; ++i) X[i] = fmaf(av[i], X[i], kv[i] * vj);
  }
#pragma unroll
  for (int i = 0; i < D; ++i) E[i * D + j] = X[i];
  c[j] = cj;
  cx[j] = cxj;
#pragma unroll
  for (int i = 0; i < D; ++i) X[i] = 0.f;
  for (int t = t1 - 1; t >= t0; --t) {
    const long long r = (rb + t) * p.ld + static_cast<long long>(h) * D;
    __syncthreads();
    qv[j] = p.q[r + j];
    av[j] = p.alpha[((rb + t) * p.H + h) * D + j];
    const float dj = p.dout[r + j] * p.scale;
    __syncthreads();
    if (t > t0) {
#pragma unroll
      for (int i = 0; i < D; ++i) X[i] = av[i] * fmaf(qv[i], dj, X[i]);
    } else {
#pragma unroll
      for (int i = 0; i < D; ++i) X[i] = fmaf(qv[i], dj, X[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < D; ++i) R[i * D + j] = X[i];
}

// Carry across segments, one thread per (sequence, head, i, j) state element:
//   Sin_0 = S0, Sin_{s+1} = diag(c_s) Sin_s + E_s;
//   Gfirst_{last} = R_{last}, Gin_s = diag(alpha_{t1(s)}) Gfirst_{s+1} (0 for the last segment),
//   Gfirst_s = R_s + diag(cx_s) Gin_s;  dS0 = diag(alpha_0) Gfirst_0.
// Sin and Gin are written into p.Sin / p.Gin (cast from const: the launcher owns them).
template <int D>
__global__ void gla_bwd_carry_kernel(const LinBwdParams p, const float* __restrict__ sum,
                                     float* Sin, float* Gin) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<long long>(p.H) * D * D) return;
  const int b = blockIdx.y;
  const int h = static_cast<int>(e / (D * D)), i = static_cast<int>((e / D) % D),
            j = static_cast<int>(e % D);
  const long long bh = static_cast<long long>(b) * p.H + h;
  const long long rb = static_cast<long long>(b) * p.rows_b;
  const long long stride = 2LL * D * D + 2 * D;
  const float* base = sum + bh * p.nseg * stride;
  float S = p.S0 ? p.S0[bh * D * D + i * D + j] : 0.f;
  for (int s = 0; s < p.nseg; ++s) {
    Sin[(bh * p.nseg + s) * D * D + i * D + j] = S;
    const float* E = base + s * stride;
    S = fmaf(E[2 * D * D + i], S, E[i * D + j]);
  }
  float Gf = 0.f;
  for (int s = p.nseg - 1; s >= 0; --s) {
    const float* E = base + s * stride;
    float gin = 0.f;
    if (s < p.nseg - 1) {
      const long long t1 = static_cast<long long>(s + 1) * p.seg_len;
      gin = p.alpha[((rb + t1) * p.H + h) * D + i] * Gf;
    }
    Gin[(bh * p.nseg + s) * D * D + i * D + j] = gin;
    Gf = fmaf(E[2 * D * D + D + i], gin, E[D * D + i * D + j]);
  }
  if (p.dS0) p.dS0[bh * D * D + i * D + j] = p.alpha[(rb * p.H + h) * D + i] * Gf;
}

// Delta-rule backward (both erase forms), one CTA of D threads per (head, sequence). Thread j
// owns column j of the state in the forward passes (registers) and of the adjoint G (shared
// memory); for the row reductions (dq, dk, dalpha) thread i owns row i. States are checkpointed
// every BWD_CK tokens; each chunk is recomputed (its states, u and w kept in the workspace)
// before its reverse pass, which reads S_t and S_{t-1} rows from shared memory.
template <int D>
__global__ void __launch_bounds__(D) delta_bwd_f32_kernel(const LinBwdParams p) {
  extern __shared__ float bsm[];
  constexpr int LDG = D + 1;
  float* G = bsm;                 // [D][D + 1]
  float* Sx = G + D * LDG;        // [2][D][D + 1]: S_t and S_{t-1} in the reverse pass
  float* qv = Sx + 2 * D * LDG;   // q_t
  float* kv = qv + D;             // k_t
  float* vv = kv + D;             // v_t
  float* dv_ = vv + D;            // dO_t
  float* av = dv_ + D;            // alpha_t in av[0]
  float* du = av + D;             // du_t
  float* red = du + D;            // [2][D] block reductions
  const int j = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  const long long bh = static_cast<long long>(b) * p.H + h;
  float* ck = p.ws + bh * lin_bwd_ws_floats<D>(p.nck);
  float* buf = ck + static_cast<long long>(p.nck) * D * D;
  float* Ub = buf + static_cast<long long>(BWD_CK) * D * D;
  float* Wb = Ub + BWD_CK * D;
  const long long rb = static_cast<long long>(b) * p.rows_b;
  auto row_of = [&](int t) { return (rb + t) * p.ld + static_cast<long long>(h) * D; };
  auto gate_a = [&](int t) { return p.alpha[(rb + t) * p.H + h]; };
  auto gate_b = [&](int t) { return p.beta[(rb + t) * p.H + h]; };

  // one forward step of column j of S, given the token's vectors in shared memory
  float S[D];
  auto step = [&](int t, int tl, bool keep_uw) {
    const float a = av[0], be = gate_b(t), ae = p.erase_decayed ? a : 1.f;
    float w = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) w = fmaf(kv[i], S[i], w);
    const float u = be * (vv[j] - ae * w);
    if (keep_uw) {
      Ub[tl * D + j] = u;
      Wb[tl * D + j] = w;
    }
#pragma unroll
    for (int i = 0; i < D; ++i) S[i] = fmaf(a, S[i], kv[i] * u);
  };
  auto load_kva = [&](int t) {
    const long long r = row_of(t);
    kv[j] = p.k[r + j];
    vv[j] = p.v[r + j];
    av[j] = j == 0 ? gate_a(t) : 0.f;
  };

  // ---- forward: the state before every BWD_CK-th token
#pragma unroll
  for (int i = 0; i < D; ++i) S[i] = p.S0 ? p.S0[bh * D * D + i * D + j] : 0.f;
  for (int t = 0; t < p.N; ++t) {
    if (t % BWD_CK == 0) {
      float* c = ck + static_cast<long long>(t / BWD_CK) * D * D;
#pragma unroll
      for (int i = 0; i < D; ++i) c[i * D + j] = S[i];
    }
    __syncthreads();
    load_kva(t);
    __syncthreads();
    step(t, 0, false);
  }
  // ---- reverse, one chunk of BWD_CK tokens at a time
#pragma unroll
  for (int i = 0; i < D; ++i) G[i * LDG + j] = 0.f;
  for (int c = p.nck - 1; c >= 0; --c) {
    const int t0 = c * BWD_CK, t1 = min(p.N, t0 + BWD_CK);
    const float* cs = ck + static_cast<long long>(c) * D * D;
#pragma unroll
    for (int i = 0; i < D; ++i) S[i] = cs[i * D + j];
    for (int t = t0; t < t1; ++t) {  // recompute and keep the chunk's states
      __syncthreads();
      load_kva(t);
      __syncthreads();
      step(t, t - t0, true);
      float* st = buf + static_cast<long long>(t - t0) * D * D;
#pragma unroll
      for (int i = 0; i < D; ++i) st[i * D + j] = S[i];
    }
    __syncthreads();
    // rows of S_t and S_{t-1} are read from shared memory: S_{t1-1} is in registers
    float* cur = Sx;
    float* prv = Sx + D * LDG;
#pragma unroll
    for (int i = 0; i < D; ++i) cur[i * LDG + j] = S[i];
    for (int t = t1 - 1; t >= t0; --t) {
      const long long r = row_of(t);
      qv[j] = p.q[r + j];
      kv[j] = p.k[r + j];
      vv[j] = p.v[r + j];
      dv_[j] = p.dout[r + j];
      av[j] = j == 0 ? gate_a(t) : 0.f;
      const float* src = t == t0 ? cs : buf + static_cast<long long>(t - t0 - 1) * D * D;
      for (int i = 0; i < D; ++i) prv[i * LDG + j] = src[i * D + j];
      __syncthreads();
      const float* St = cur;
      const float* Sp = prv;
      // G_t: add the output term (column j)
#pragma unroll
      for (int i = 0; i < D; ++i) G[i * LDG + j] = fmaf(p.scale * qv[i], dv_[j], G[i * LDG + j]);
      __syncthreads();
      const float a = av[0], be = gate_b(t), ae = p.erase_decayed ? a : 1.f;
      const int tl = t - t0;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) acc = fmaf(kv[i], G[i * LDG + j], acc);
      du[j] = acc;
      p.dv[r + j] = be * acc;
      const float wj = Wb[tl * D + j];
      red[j] = acc * (vv[j] - ae * wj);                         // dbeta terms
      float dal = p.erase_decayed ? -be * acc * wj : 0.f;       // dalpha terms (column part)
      __syncthreads();
      const int i = j;
      float aq = 0.f, ak = 0.f, as = 0.f;
      for (int jj = 0; jj < D; ++jj) {
        aq = fmaf(St[i * LDG + jj], dv_[jj], aq);
        ak = fmaf(G[i * LDG + jj], Ub[tl * D + jj], ak);
        as = fmaf(Sp[i * LDG + jj], du[jj], as);
        dal = fmaf(G[i * LDG + jj], Sp[i * LDG + jj], dal);
      }
      p.dq[r + i] = p.scale * aq;
      p.dk[r + i] = ak - be * ae * as;
      red[D + j] = dal;
      __syncthreads();
      if (j < 32) {  // block sums of the dbeta and dalpha terms
        float sb = 0.f, sa = 0.f;
        for (int e = j; e < D; e += 32) {
          sb += red[e];
          sa += red[D + e];
        }
        for (int o2 = 16; o2; o2 >>= 1) {
          sb += __shfl_xor_sync(0xffffffffu, sb, o2);
          sa += __shfl_xor_sync(0xffffffffu, sa, o2);
        }
        if (j == 0) {
          p.dbeta[(rb + t) * p.H + h] = sb;
          p.dalpha[(rb + t) * p.H + h] = sa;
        }
      }
#pragma unroll
      for (int ii = 0; ii < D; ++ii)
        G[ii * LDG + j] = a * G[ii * LDG + j] - be * ae * kv[ii] * du[j];
      __syncthreads();
      float* tmp = cur;
      cur = prv;
      prv = tmp;
    }
  }
  if (p.dS0) {
#pragma unroll
    for (int i = 0; i < D; ++i) p.dS0[bh * D * D + i * D + j] = G[i * LDG + j];
  }
}

}  // namespace kta

namespace kta {

// Vector-GLA backward without stored states, one CTA of D threads per (segment, head, sequence),
// thread j owning column j of S (forward sweep) and of G (reverse sweep) in registers; row
// reductions go through a transposed copy in shared memory. The gate gradient uses the closed
// form of the log-gate derivative: with b_t = sum_{u <= t} log alpha_u, q enters as
// q_t * e^{b_t} and k as k_t * e^{-b_t}, so dL/db_t = q_t (.) dq_t - k_t (.) dk_t and
//   dalpha_u = (1 / alpha_u) sum_{t >= u} (q_t (.) dq_t - k_t (.) dk_t).
//   forward sweep (from the segment's entering state): S_t, dq_t = scale S_t dO_t^T, and
//     y_t = q_t (.) dq_t kept in `ybuf`;
//   reverse sweep (from the adjoint entering from the right): G_t += scale q_t^T dO_t,
//     dv_t = k_t G_t, dk_t = G_t v_t^T, the segment-local suffix X_t = sum_{t' >= t, in segment}
//     (y - k (.) dk) in fp64 (xbuf), then G <- diag(alpha_t) G;
//   ytot: per (sequence, head, segment) the segment's full sum X_{t0} (for the suffix carry).
// A segment that is the only one of its sequence writes dS0 = diag(alpha_0) G_0.
template <int D>
__global__ void __launch_bounds__(D) gla_bwd_sweep_kernel(const LinBwdParams p, float* ybuf,
                                                          double* xbuf, double* ytot) {
  extern __shared__ float gsm[];
  constexpr int LDT = D + 1;
  float* T = gsm;              // [D][D + 1] transposed state / adjoint
  float* qv = T + D * LDT;
  float* kv = qv + D;
  float* vv = kv + D;
  float* dv_ = vv + D;
  float* av = dv_ + D;
  const int j = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y, seg = blockIdx.z;
  const long long bh = static_cast<long long>(b) * p.H + h;
  const long long bhs = bh * p.nseg + seg;
  const int t0 = seg * p.seg_len, t1 = min(p.N, t0 + p.seg_len);
  const long long rb = static_cast<long long>(b) * p.rows_b;
  auto row_of = [&](int t) { return (rb + t) * p.ld + static_cast<long long>(h) * D; };
  auto load_vecs = [&](int t) {
    const long long r = row_of(t);
    qv[j] = p.q[r + j];
    kv[j] = p.k[r + j];
    vv[j] = p.v[r + j];
    dv_[j] = p.dout[r + j];
    av[j] = p.alpha[((rb + t) * p.H + h) * D + j];
  };
  // scratch rows of this sequence-head: token t of the sequence at (bh * N + t) * D
  float* yrow = ybuf + bh * static_cast<long long>(p.N) * D;
  double* xrow = xbuf + bh * static_cast<long long>(p.N) * D;

  float X[D];
  // ---- forward sweep: S column j, dq_t, y_t
  if (p.Sin) {
#pragma unroll
    for (int i = 0; i < D; ++i) X[i] = p.Sin[bhs * D * D + i * D + j];
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) X[i] = p.S0 ? p.S0[bh * D * D + i * D + j] : 0.f;
  }
  for (int t = t0; t < t1; ++t) {
    __syncthreads();
    load_vecs(t);
    __syncthreads();
    const float vj = vv[j];
#pragma unroll
    for (int i = 0; i < D; ++i) {
      X[i] = fmaf(av[i], X[i], kv[i] * vj);
      T[i * LDT + j] = X[i];
    }
    __syncthreads();
    const int i = j;
    float acc = 0.f;
#pragma unroll 8
    for (int jj = 0; jj < D; ++jj) acc = fmaf(T[i * LDT + jj], dv_[jj], acc);
    const float dqi = acc * p.scale;
    p.dq[row_of(t) + i] = dqi;
    yrow[static_cast<long long>(t) * D + i] = qv[i] * dqi;
  }
  // ---- reverse sweep: G column j, dv_t, dk_t, local suffix of the gate terms
  if (p.Gin) {
#pragma unroll
    for (int i = 0; i < D; ++i) X[i] = p.Gin[bhs * D * D + i * D + j];
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) X[i] = 0.f;
  }
  double suf = 0.0;  // thread j's key dim: sum over this segment's tokens >= t
  for (int t = t1 - 1; t >= t0; --t) {
    __syncthreads();
    load_vecs(t);
    __syncthreads();
    const float dj = dv_[j] * p.scale;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
      X[i] = fmaf(qv[i], dj, X[i]);
      acc = fmaf(kv[i], X[i], acc);
      T[i * LDT + j] = X[i];
    }
    p.dv[row_of(t) + j] = acc;
    __syncthreads();
    const int i = j;
    float dk = 0.f;
#pragma unroll 8
    for (int jj = 0; jj < D; ++jj) dk = fmaf(T[i * LDT + jj], vv[jj], dk);
    p.dk[row_of(t) + i] = dk;
    suf += static_cast<double>(yrow[static_cast<long long>(t) * D + i]) -
           static_cast<double>(kv[i]) * static_cast<double>(dk);
    xrow[static_cast<long long>(t) * D + i] = suf;
#pragma unroll
    for (int ii = 0; ii < D; ++ii) X[ii] *= av[ii];
  }
  ytot[bhs * D + j] = suf;
  if (p.dS0 && p.nseg == 1) {
    // X = diag(alpha_0) G_0 after the last step
#pragma unroll
    for (int i = 0; i < D; ++i) p.dS0[bh * D * D + i * D + j] = X[i];
  }
}

// dalpha_t[i] = (X_t[i] + sum of later segments' totals) / alpha_t[i], one thread per element of
// [B][N][H][D] (the later segments' totals are summed here: a handful per sequence-head).
template <int D>
__global__ void gla_bwd_dalpha_kernel(const LinBwdParams p, const double* __restrict__ xbuf,
                                      const double* __restrict__ ytot) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (e >= static_cast<long long>(p.N) * p.H * D) return;
  const int i = static_cast<int>(e % D);
  const int h = static_cast<int>((e / D) % p.H);
  const int t = static_cast<int>(e / (static_cast<long long>(D) * p.H));
  const long long bh = static_cast<long long>(b) * p.H + h;
  const int seg = t / p.seg_len;
  double x = xbuf[(bh * p.N + t) * D + i];
  for (int s = seg + 1; s < p.nseg; ++s) x += ytot[(bh * p.nseg + s) * D + i];
  const long long a = ((static_cast<long long>(b) * p.rows_b + t) * p.H + h) * D + i;
  p.dalpha[a] = static_cast<float>(x / static_cast<double>(p.alpha[a]));
}

}  // namespace kta
