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
};

// One warp per (query token, head, sequence): recompute the row's softmax statistics and
// output, then accumulate dq in registers and dk, dv with atomics.
__global__ void __launch_bounds__(128) softmax_bwd_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ dout, float* __restrict__ dq, float* dk, float* dv,
    const SoftmaxBwdParams p) {
  __shared__ float qs[4][128], dos[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const bool active = t < p.N;
  const int d = p.d;
  const long long rb = static_cast<long long>(b) * p.N;
  const long long qrow = (rb + (active ? t : 0)) * p.ld + static_cast<long long>(h) * d;
  for (int c = lane; c < d; c += 32) {
    qs[warp][c] = active ? q[qrow + c] : 0.f;
    dos[warp][c] = active ? dout[qrow + c] : 0.f;
  }
  __syncwarp();
  if (!active) return;
  const int f = t / p.P;
  const int nfr = p.dil == 1 ? min(p.W, f + 1) : min(p.W, f / p.dil + 1);
  // pass 1: row maximum m, normaliser l and output o (lanes over keys, then over dims)
  float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int jf = nfr - 1; jf >= 0; --jf) {
    const long long base = rb + static_cast<long long>(f - jf * p.dil) * p.P;
    for (int s0 = 0; s0 < p.P; s0 += 32) {
      const int s = s0 + lane;
      float sc = -INFINITY;
      if (s < p.P) {
        const float* kr = k + (base + s) * p.ld + static_cast<long long>(h) * d;
        float dot = 0.f;
        for (int c = 0; c < d; ++c) dot = fmaf(qs[warp][c], kr[c], dot);
        sc = dot * p.scale;
      }
      float mx = sc;
      for (int o2 = 16; o2; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      const float mnew = fmaxf(m, mx);
      const float corr = expf(m - mnew);
      const float pr = s < p.P ? expf(sc - mnew) : 0.f;
      float ps = pr;
      for (int o2 = 16; o2; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      l = l * corr + ps;
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] *= corr;
      const int nk = min(32, p.P - s0);
      for (int jj = 0; jj < nk; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, pr, jj);
        const float* vr = v + (base + s0 + jj) * p.ld + static_cast<long long>(h) * d;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (lane + 32 * c < d) acc[c] = fmaf(pj, vr[lane + 32 * c], acc[c]);
      }
      m = mnew;
    }
  }
  const float inv = 1.f / l;
  float dD = 0.f;  // dO_t . o_t
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (lane + 32 * c < d) dD = fmaf(dos[warp][lane + 32 * c], acc[c] * inv, dD);
  for (int o2 = 16; o2; o2 >>= 1) dD += __shfl_xor_sync(0xffffffffu, dD, o2);
  // pass 2: ds for every visible key; dq in registers, dk and dv by atomics
  float gq[4] = {0.f, 0.f, 0.f, 0.f};
  for (int jf = nfr - 1; jf >= 0; --jf) {
    const long long base = rb + static_cast<long long>(f - jf * p.dil) * p.P;
    for (int s0 = 0; s0 < p.P; s0 += 32) {
      const int s = s0 + lane;
      float pj = 0.f, ds = 0.f;
      if (s < p.P) {
        const float* kr = k + (base + s) * p.ld + static_cast<long long>(h) * d;
        const float* vr = v + (base + s) * p.ld + static_cast<long long>(h) * d;
        float dot = 0.f, dp = 0.f;
        for (int c = 0; c < d; ++c) {
          dot = fmaf(qs[warp][c], kr[c], dot);
          dp = fmaf(dos[warp][c], vr[c], dp);
        }
        pj = expf(dot * p.scale - m) * inv;
        ds = pj * (dp - dD);
      }
      const int nk = min(32, p.P - s0);
      for (int jj = 0; jj < nk; ++jj) {
        const float dsj = __shfl_sync(0xffffffffu, ds, jj) * p.scale;
        const float pjj = __shfl_sync(0xffffffffu, pj, jj);
        const long long kr = (base + s0 + jj) * p.ld + static_cast<long long>(h) * d;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int cc = lane + 32 * c;
          if (cc < d) {
            gq[c] = fmaf(dsj, k[kr + cc], gq[c]);
            atomicAdd(&dk[kr + cc], dsj * qs[warp][cc]);
            atomicAdd(&dv[kr + cc], pjj * dos[warp][cc]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (lane + 32 * c < d) dq[qrow + lane + 32 * c] = gq[c];
}

// Zero a [rows][H][d] head range of a [rows][ld] array (one thread per element).
__global__ void zero_rows_f32_kernel(float* x, long long rows, int Hd, long long ld) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e < rows * Hd) x[(e / Hd) * ld + e % Hd] = 0.f;
}

constexpr int BWD_CK = 32;  // tokens between stored states in the linear-branch backward

struct LinBwdParams {
  const float *q, *k, *v, *alpha, *beta, *S0, *dout;
  float *dq, *dk, *dv, *dalpha, *dbeta, *dS0;
  long long ld;        // row stride of q / k / v / dO / dq / dk / dv (elements)
  int rows_b, N, H;
  float scale;
  int delta, erase_decayed;
  int nck;             // stored states per (sequence, head) = ceil(N / BWD_CK)
  float* ws;           // per (sequence, head): states [nck][D][D], chunk [BWD_CK][D][D], u, w
};

template <int D>
__host__ __device__ constexpr long long lin_bwd_ws_floats(int nck) {
  return (static_cast<long long>(nck) + BWD_CK) * D * D + 2LL * BWD_CK * D;
}

// One CTA of D threads per (head, sequence). Thread j owns column j of the state in the
// forward passes (registers) and of the adjoint G (shared memory); for the row reductions
// (dq, dk, dalpha) thread i owns row i.
template <int D>
__global__ void __launch_bounds__(D) lin_bwd_f32_kernel(const LinBwdParams p) {
  extern __shared__ float bsm[];
  constexpr int LDG = D + 1;
  float* G = bsm;                 // [D][D + 1]
  float* qv = G + D * LDG;        // q_t
  float* kv = qv + D;             // k_t
  float* vv = kv + D;             // v_t
  float* dv_ = vv + D;            // dO_t
  float* av = dv_ + D;            // alpha_t (vector gate) or alpha_t in av[0]
  float* du = av + D;             // du_t (delta)
  float* red = du + D;            // [2][D] block reductions (delta)
  const int j = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  const long long bh = static_cast<long long>(b) * p.H + h;
  float* ck = p.ws + bh * lin_bwd_ws_floats<D>(p.nck);
  float* buf = ck + static_cast<long long>(p.nck) * D * D;
  float* Ub = buf + static_cast<long long>(BWD_CK) * D * D;
  float* Wb = Ub + BWD_CK * D;
  const long long rb = static_cast<long long>(b) * p.rows_b;
  auto row_of = [&](int t) { return (rb + t) * p.ld + static_cast<long long>(h) * D; };
  auto gate_a = [&](int t, int i) {
    return p.delta ? p.alpha[(rb + t) * p.H + h] : p.alpha[((rb + t) * p.H + h) * D + i];
  };
  auto gate_b = [&](int t) { return p.beta[(rb + t) * p.H + h]; };

  // one forward step of column j of S, given the token's vectors in shared memory
  float S[D];
  auto step = [&](int t, int tl, bool keep_uw) {
    if (p.delta) {
      const float a = av[0], be = gate_b(t), ae = p.erase_decayed ? a : 1.f;
      float w = 0.f;
#pragma unroll 8
      for (int i = 0; i < D; ++i) w = fmaf(kv[i], S[i], w);
      const float u = be * (vv[j] - ae * w);
      if (keep_uw) {
        Ub[tl * D + j] = u;
        Wb[tl * D + j] = w;
      }
#pragma unroll 8
      for (int i = 0; i < D; ++i) S[i] = fmaf(a, S[i], kv[i] * u);
    } else {
#pragma unroll 8
      for (int i = 0; i < D; ++i) S[i] = fmaf(av[i], S[i], kv[i] * vv[j]);
    }
  };
  auto load_kva = [&](int t) {
    const long long r = row_of(t);
    kv[j] = p.k[r + j];
    vv[j] = p.v[r + j];
    av[j] = p.delta ? (j == 0 ? gate_a(t, 0) : 0.f) : gate_a(t, j);
  };

  // ---- forward: the state before every BWD_CK-th token
#pragma unroll 8
  for (int i = 0; i < D; ++i) S[i] = p.S0 ? p.S0[bh * D * D + i * D + j] : 0.f;
  for (int t = 0; t < p.N; ++t) {
    if (t % BWD_CK == 0) {
      float* c = ck + static_cast<long long>(t / BWD_CK) * D * D;
#pragma unroll 8
      for (int i = 0; i < D; ++i) c[i * D + j] = S[i];
    }
    __syncthreads();
    load_kva(t);
    __syncthreads();
    step(t, 0, false);
  }
  // ---- reverse, one chunk of BWD_CK tokens at a time
#pragma unroll 8
  for (int i = 0; i < D; ++i) G[i * LDG + j] = 0.f;
  for (int c = p.nck - 1; c >= 0; --c) {
    const int t0 = c * BWD_CK, t1 = min(p.N, t0 + BWD_CK);
    const float* cs = ck + static_cast<long long>(c) * D * D;
#pragma unroll 8
    for (int i = 0; i < D; ++i) S[i] = cs[i * D + j];
    for (int t = t0; t < t1; ++t) {  // recompute and keep the chunk's states
      __syncthreads();
      load_kva(t);
      __syncthreads();
      step(t, t - t0, true);
      float* st = buf + static_cast<long long>(t - t0) * D * D;
#pragma unroll 8
      for (int i = 0; i < D; ++i) st[i * D + j] = S[i];
    }
    __syncthreads();
    for (int t = t1 - 1; t >= t0; --t) {
      const long long r = row_of(t);
      qv[j] = p.q[r + j];
      kv[j] = p.k[r + j];
      vv[j] = p.v[r + j];
      dv_[j] = p.dout[r + j];
      av[j] = p.delta ? (j == 0 ? gate_a(t, 0) : 0.f) : gate_a(t, j);
      __syncthreads();
      const float* St = buf + static_cast<long long>(t - t0) * D * D;
      const float* Sp = t == t0 ? cs : buf + static_cast<long long>(t - t0 - 1) * D * D;
      // G_t: add the output term (column j)
#pragma unroll 8
      for (int i = 0; i < D; ++i) G[i * LDG + j] = fmaf(p.scale * qv[i], dv_[j], G[i * LDG + j]);
      __syncthreads();
      if (!p.delta) {
        // column j: dv; row j: dq, dk, dalpha
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) acc = fmaf(kv[i], G[i * LDG + j], acc);
        p.dv[r + j] = acc;
        const int i = j;
        float aq = 0.f, ak = 0.f, aa = 0.f;
        for (int jj = 0; jj < D; ++jj) {
          aq = fmaf(St[i * D + jj], dv_[jj], aq);
          ak = fmaf(G[i * LDG + jj], vv[jj], ak);
          aa = fmaf(G[i * LDG + jj], Sp[i * D + jj], aa);
        }
        p.dq[r + i] = p.scale * aq;
        p.dk[r + i] = ak;
        p.dalpha[((rb + t) * p.H + h) * D + i] = aa;
        __syncthreads();
#pragma unroll 8
        for (int ii = 0; ii < D; ++ii) G[ii * LDG + j] *= av[ii];
      } else {
        const float a = av[0], be = gate_b(t), ae = p.erase_decayed ? a : 1.f;
        const int tl = t - t0;
        float acc = 0.f;
#pragma unroll 8
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
          aq = fmaf(St[i * D + jj], dv_[jj], aq);
          ak = fmaf(G[i * LDG + jj], Ub[tl * D + jj], ak);
          as = fmaf(Sp[i * D + jj], du[jj], as);
          dal = fmaf(G[i * LDG + jj], Sp[i * D + jj], dal);
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
#pragma unroll 8
        for (int ii = 0; ii < D; ++ii)
          G[ii * LDG + j] = a * G[ii * LDG + j] - be * ae * kv[ii] * du[j];
      }
      __syncthreads();
    }
  }
  if (p.dS0) {
#pragma unroll 8
    for (int i = 0; i < D; ++i) p.dS0[bh * D * D + i * D + j] = G[i * LDG + j];
  }
}

}  // namespace kta
