// simt_f32.cuh -- fp32 CUDA-core kernels: the fp32 reference mode of every branch.
//
// Same operator as the tensor-core path (paper-read "Kairos: A Native World Model Stack for
// Physical AI", section 2, second pillar: SWA, DSWA, GLA and the gated delta-rule equations),
// computed with fp32 FMAs and accurate expf so that results stay within 1e-4 of the fp64 oracle.
#pragma once

#include "kta_ptx.cuh"

namespace kta {

// Addressing shared by the softmax kernels: q / o rows (b, t) = b * q_rows_b + t for query token
// t of this launch; key rows of frame g, token s = (b * kb_frames + g % kmod) * P + s.
struct WinSimtParams {
  int B, P, Fq, f_base, Htot, H0;
  int W[2], dil[2], kh_off[2], kb_frames[2], kmod[2];
  int q_rows_b;
  long long q_ld, o_ld;   // q / o row strides (elements)
  long long k_ld[2];      // K / V row strides per group (elements)
  float scale;
  int d;
};

// One warp per (b, head, query token). Lanes take 32 keys at a time; online softmax in fp32.
__global__ void win_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k0,
                                    const float* __restrict__ v0, const float* __restrict__ k1,
                                    const float* __restrict__ v1, float* __restrict__ o,
                                    const WinSimtParams p) {
  __shared__ float qs[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + warp;  // query token within this launch
  const int h = blockIdx.y, b = blockIdx.z;
  const int nrows = p.Fq * p.P;
  const bool active = t < nrows;
  const int g = h >= p.H0 ? 1 : 0;
  const int W = g ? p.W[1] : p.W[0];
  const int dil = g ? p.dil[1] : p.dil[0];
  const float* K = g ? k1 : k0;
  const float* V = g ? v1 : v0;
  const int hk = h - (g ? p.kh_off[1] : p.kh_off[0]);
  const long long kld = g ? p.k_ld[1] : p.k_ld[0];
  const int kbf = g ? p.kb_frames[1] : p.kb_frames[0];
  const int kmod = g ? p.kmod[1] : p.kmod[0];
  const int d = p.d;
  const long long qrow = static_cast<long long>(b) * p.q_rows_b + (active ? t : 0);
  for (int c = lane; c < d; c += 32) qs[warp][c] = active ? q[qrow * p.q_ld + h * d + c] : 0.f;
  __syncwarp();
  if (!active) return;
  const int f = t / p.P + p.f_base;
  float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int nfr = dil == 1 ? min(W, f + 1) : min(W, f / dil + 1);
  for (int j = nfr - 1; j >= 0; --j) {  // oldest visible frame first
    const int fr = f - j * dil;
    const long long base = (static_cast<long long>(b) * kbf + fr % kmod) * p.P;
    for (int s0 = 0; s0 < p.P; s0 += 32) {
      const int s = s0 + lane;
      float sc = -INFINITY;
      if (s < p.P) {
        const float* kr = K + (base + s) * kld + hk * d;
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
        const float* vr = V + (base + s0 + jj) * kld + hk * d;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (lane + 32 * c < d) acc[c] = fmaf(pj, vr[lane + 32 * c], acc[c]);
      }
      m = mnew;
    }
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (lane + 32 * c < d) o[qrow * p.o_ld + h * d + lane + 32 * c] = acc[c] * inv;
}

struct RecF32Params {
  int B, N, H, d;
  long long ld;          // q / k / v / o row stride (elements)
  int rows_b;            // rows per sequence in q / k / v / o / gates
  float scale;
  const float* S0;       // [B][H][d][d] key-major or null
  float* S_out;          // [B][H][d][d] or null
  int erase_decayed;     // delta rule: 1 = decayed erase (GatedDeltaNet form)
};

// Vector-gated GLA, token by token. One CTA per (b, h); thread j owns column j of S (all key
// dims i in registers). S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = scale * q_t S_t.
template <int D>
__global__ void __launch_bounds__(D) gla_rec_f32_kernel(const float* __restrict__ q,
                                                        const float* __restrict__ k,
                                                        const float* __restrict__ v,
                                                        const float* __restrict__ alpha,
                                                        float* __restrict__ o,
                                                        const RecF32Params p) {
  __shared__ float qs[D], ks[D], as[D];
  const int j = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  float S[D];
  const long long sb = (static_cast<long long>(b) * p.H + h) * D * D;
#pragma unroll
  for (int i = 0; i < D; ++i) S[i] = p.S0 ? p.S0[sb + i * D + j] : 0.f;
  for (int t = 0; t < p.N; ++t) {
    const long long row = static_cast<long long>(b) * p.rows_b + t;
    qs[j] = q[row * p.ld + h * D + j];
    ks[j] = k[row * p.ld + h * D + j];
    as[j] = alpha[(row * p.H + h) * D + j];
    const float vj = v[row * p.ld + h * D + j];
    __syncthreads();
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
      S[i] = fmaf(as[i], S[i], ks[i] * vj);
      acc = fmaf(qs[i], S[i], acc);
    }
    o[row * p.ld + h * D + j] = acc * p.scale;
    __syncthreads();
  }
  if (p.S_out) {
#pragma unroll
    for (int i = 0; i < D; ++i) p.S_out[sb + i * D + j] = S[i];
  }
}

// Gated delta rule, the page's four lines token by token. Thread j owns column j of the
// key-major state S = M^T, i.e. row j of the page's M:
//   v_old = M k, v_new = beta v + (1-beta) v_old, M = alpha M - v_old k^T + v_new k^T, o = M q.
template <int D>
__global__ void __launch_bounds__(D) delta_rec_f32_kernel(const float* __restrict__ q,
                                                          const float* __restrict__ k,
                                                          const float* __restrict__ v,
                                                          const float* __restrict__ alpha,
                                                          const float* __restrict__ beta,
                                                          float* __restrict__ o,
                                                          const RecF32Params p) {
  __shared__ float qs[D], ks[D];
  const int j = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  float S[D];
  const long long sb = (static_cast<long long>(b) * p.H + h) * D * D;
#pragma unroll
  for (int i = 0; i < D; ++i) S[i] = p.S0 ? p.S0[sb + i * D + j] : 0.f;
  for (int t = 0; t < p.N; ++t) {
    const long long row = static_cast<long long>(b) * p.rows_b + t;
    qs[j] = q[row * p.ld + h * D + j];
    ks[j] = k[row * p.ld + h * D + j];
    const float a = alpha[row * p.H + h], be = beta[row * p.H + h];
    const float vj = v[row * p.ld + h * D + j];
    __syncthreads();
    float vold = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) vold = fmaf(S[i], ks[i], vold);
    const float vnew = be * vj + (1.f - be) * vold;
    float acc = 0.f;
    if (p.erase_decayed) {
      // S = alpha (S - beta v_old k^T) + beta v k^T
#pragma unroll
      for (int i = 0; i < D; ++i) {
        S[i] = a * (S[i] - be * vold * ks[i]) + be * vj * ks[i];
        acc = fmaf(S[i], qs[i], acc);
      }
    } else {
#pragma unroll
      for (int i = 0; i < D; ++i) {
        S[i] = a * S[i] - vold * ks[i] + vnew * ks[i];
        acc = fmaf(S[i], qs[i], acc);
      }
    }
    o[row * p.ld + h * D + j] = acc * p.scale;
    __syncthreads();
  }
  if (p.S_out) {
#pragma unroll
    for (int i = 0; i < D; ++i) p.S_out[sb + i * D + j] = S[i];
  }
}

// Y_m = A_m X_m (+ E_m) for m < gridDim.z, d x d fp32 row-major matrices: the composition of two
// affine state maps (a segment's transition applied to the state entering it, plus the state the
// segment builds from zero). A 32 x 32 output tile per CTA of 32 x 8 threads, both operands staged
// through shared memory in 32-wide K steps.
__global__ void __launch_bounds__(256) state_affine_kernel(const float* __restrict__ A,
                                                           const float* __restrict__ X,
                                                           const float* __restrict__ E,
                                                           float* __restrict__ Y, int d) {
  __shared__ float as[32][33], xs[32][33];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int col = blockIdx.x * 32 + tx, row0 = blockIdx.y * 32;
  const long long off = static_cast<long long>(blockIdx.z) * d * d;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < d; k0 += 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 8 * i;
      as[r][tx] = (row0 + r < d && k0 + tx < d) ? A[off + (row0 + r) * static_cast<long long>(d) + k0 + tx] : 0.f;
      xs[r][tx] = (k0 + r < d && col < d) ? X[off + (k0 + r) * static_cast<long long>(d) + col] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
      const float xv = xs[kk][tx];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(as[ty + 8 * i][kk], xv, acc[i]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + ty + 8 * i;
    if (r < d && col < d) {
      const long long e = off + static_cast<long long>(r) * d + col;
      Y[e] = acc[i] + (E ? E[e] : 0.f);
    }
  }
}

// T = diag(prod_t alpha_t) per (sequence, head): the transition of a vector-gated GLA run, whose
// end state is S_end = diag(prod_t alpha_t) S_start + S_loc (GLA paragraph: the gate scales the
// state row of each key dim once per token). alpha: [B][N][H][D] fp32; T: [B][H][D][D]. G token
// blocks per (sequence, head) each sum log2(alpha) per key dim into `part` ([B*H][G][D]); a
// second kernel adds the G partial sums in order and writes exp2 of the total on the diagonal.
template <int D>
__global__ void __launch_bounds__(D * 4) gla_transition_part_kernel(const float* __restrict__ alpha,
                                                                    float* __restrict__ part,
                                                                    int N, int H, int G) {
  // block (bh, blk): sum over its token block of log2(alpha) per key dim, clamped at -200
  // (a zero gate gives 0); four token groups per key dim, combined in a fixed order
  __shared__ float s[4][D];
  const int bh = blockIdx.x, blk = blockIdx.y, b = bh / H, h = bh % H;
  const int i = threadIdx.x % D, g = threadIdx.x / D;
  const int per = (N + G - 1) / G, t0 = blk * per, t1 = min(N, t0 + per);
  float acc = 0.f;
  for (int t = t0 + g; t < t1; t += 4)
    acc += fmaxf(__log2f(alpha[((static_cast<long long>(b) * N + t) * H + h) * D + i]), -200.f);
  s[g][i] = acc;
  __syncthreads();
  if (g == 0) part[(static_cast<long long>(bh) * G + blk) * D + i] = (s[0][i] + s[1][i]) + (s[2][i] + s[3][i]);
}

template <int D>
__global__ void __launch_bounds__(256) gla_transition_finish_kernel(const float* __restrict__ part,
                                                                    float* __restrict__ T, int G) {
  // the blocks' sums in block order, then the whole D x D matrix, zeros off the diagonal
  __shared__ float diag[D];
  const int bh = blockIdx.x;
  for (int i = threadIdx.x; i < D; i += 256) {
    float sum = 0.f;
    for (int u = 0; u < G; ++u) sum += part[(static_cast<long long>(bh) * G + u) * D + i];
    diag[i] = exp2f(sum);
  }
  __syncthreads();
  float4* Tb = reinterpret_cast<float4*>(T + static_cast<long long>(bh) * D * D);
  for (int e = threadIdx.x; e < D * D / 4; e += 256) {
    const int r = (4 * e) / D, c = (4 * e) % D;
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r >= c && r < c + 4) (&w.x)[r - c] = diag[r];
    Tb[e] = w;
  }
}

}  // namespace kta
