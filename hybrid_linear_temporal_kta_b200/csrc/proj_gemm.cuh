// proj_gemm.cuh -- the projections around the operator on the sm_100a tensor cores.
//
// Operator: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar, GLA paragraph: q_t = W_Q x_t, k_t = W_K x_t, v_t = W_V x_t, beta_t = sigmoid(W_beta x_t)
// (and the forget gate alpha_t, a sigmoid of a projection of x_t), and the layer's output
// projection of the mixed heads. All of them are one contraction Y = X W^T with X [M][K] and
// W [N][K] (bf16, both K-major), fp32 accumulation, and an epilogue that routes column ranges of
// Y to their own tensors (bf16, fp32, or sigmoid -> fp32).
//
// Persistent kernel, one CTA per SM (192 KB of shared memory, all 512 TMEM columns). Output tiles
// of 128 x 256 are taken in groups of 16 row blocks, column block by column block inside a group
// (pg_tile), so that each wave's slices of X and W are L2-resident. Warp roles (192 threads):
//   warp 0      TMA producer: per 64-wide K step, the X tile (128 x 64) and the W tile (256 x 64)
//               into a 4-stage ring (128-byte swizzle).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M = 128, N = 256, K = 16, SS form)
//               into one of two 256-column accumulators, alternating per tile.
//   warps 2..5  epilogue: thread <-> output row (TMEM lane), 32 columns per tcgen05.ld; while it
//               drains one accumulator the tensor core fills the other.
// Every wait is bounded; on a timeout the CTA records it and unwinds to free its TMEM.
#pragma once

#include "kta_ptx.cuh"

namespace kta {

constexpr int PG_BM = 128, PG_BN = 256, PG_BK = 64, PG_STAGES = 4, PG_MAXSEG = 8;
constexpr int PG_GROUP = 16;  // row blocks per raster group

// Tile t -> (row block, column block). Tiles go in groups of PG_GROUP row blocks; inside a group
// the column block is the slow index, so the CTAs of one wave share a few column blocks of W and
// the group's rows of X, both of which stay in L2 while the group runs.
__device__ __forceinline__ void pg_tile(int t, int n_mt, int n_nt, int& m0, int& n0) {
  const int per_group = PG_GROUP * n_nt;
  const int g = t / per_group, w = t % per_group;
  const int gm = min(PG_GROUP, n_mt - g * PG_GROUP);
  m0 = (g * PG_GROUP + w % gm) * PG_BM;
  n0 = (w / gm) * PG_BN;
}

struct ProjSeg {
  int c0, c1;       // columns [c0, c1) of Y
  void* dst;        // row r, column c -> dst[r * ld + (c - c0)]
  long long ld;     // elements
  int mode;         // 0 bf16, 1 sigmoid -> fp32, 2 fp32
  const float* bias;  // per column of the range (added before the sigmoid / rounding), or null
  int vec;          // dst and ld allow 16-byte vector stores of 8-column groups
};

struct ProjParams {
  int M, N, K;
  int nseg;
  ProjSeg seg[PG_MAXSEG];
};

struct ProjSmem {
  __nv_bfloat16 a[PG_STAGES][PG_BM * PG_BK];  // 16 KB per stage
  __nv_bfloat16 b[PG_STAGES][PG_BN * PG_BK];  // 32 KB per stage
  uint64_t full[PG_STAGES], empty[PG_STAGES];
  uint64_t acc_full[2], acc_empty[2], fin;
  uint32_t tmem_base;
  int abort_flag;
};

inline size_t proj_smem_bytes() { return sizeof(ProjSmem) + 1024; }

__device__ __forceinline__ float pg_sigmoid(float x) { return 1.f / (1.f + expf(-x)); }

// Store 32 accumulator columns [col0, col0 + 32) of one output row.
__device__ __forceinline__ void pg_store_chunk(const ProjParams& p, long long row, int col0,
                                               const uint32_t (&r)[32]) {
  int s = 0;
  while (s < p.nseg && !(col0 >= p.seg[s].c0 && col0 < p.seg[s].c1)) ++s;
  const bool whole = s < p.nseg && p.seg[s].vec && col0 + 32 <= p.seg[s].c1 &&
                     ((col0 - p.seg[s].c0) & 7) == 0;
  if (whole) {
    const ProjSeg& g = p.seg[s];
    const long long off = row * g.ld + (col0 - g.c0);
    float x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(r[e]);
    if (g.bias) {
      const float4* b4 = reinterpret_cast<const float4*>(g.bias + (col0 - g.c0));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 b = __ldg(b4 + j);
        x[4 * j] += b.x;
        x[4 * j + 1] += b.y;
        x[4 * j + 2] += b.z;
        x[4 * j + 3] += b.w;
      }
    }
    if (g.mode == 0) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.dst) + off);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[8 * j + 2 * e], x[8 * j + 2 * e + 1]);
          w[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.dst) + off);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float f[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] = g.mode == 1 ? pg_sigmoid(x[4 * j + e]) : x[4 * j + e];
        dst[j] = make_float4(f[0], f[1], f[2], f[3]);
      }
    }
    return;
  }
  // ragged: column by column (unrolled so that r stays in registers)
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int c = col0 + e;
    int t = 0;
    while (t < p.nseg && !(c >= p.seg[t].c0 && c < p.seg[t].c1)) ++t;
    if (c >= p.N || t == p.nseg) continue;
    const ProjSeg& g = p.seg[t];
    const long long off = row * g.ld + (c - g.c0);
    const float x = __uint_as_float(r[e]) + (g.bias ? g.bias[c - g.c0] : 0.f);
    if (g.mode == 0)
      static_cast<__nv_bfloat16*>(g.dst)[off] = __float2bfloat16_rn(x);
    else
      static_cast<float*>(g.dst)[off] = g.mode == 1 ? pg_sigmoid(x) : x;
  }
}

__global__ void __launch_bounds__(192, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                     const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  ProjSmem& sm = *reinterpret_cast<ProjSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr uint32_t STAGE_BYTES = (PG_BM + PG_BN) * PG_BK * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mt = (p.M + PG_BM - 1) / PG_BM, n_nt = (p.N + PG_BN - 1) / PG_BN;
  const int tiles = n_mt * n_nt;
  const int nk = (p.K + PG_BK - 1) / PG_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PG_STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.acc_full[x], 1);
      mbar_init(&sm.acc_empty[x], 128);
    }
    mbar_init(&sm.fin, 1);
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
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&ta);
      prefetch_tmap(&tb);
      long long it = 0;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        int m0, n0;
        pg_tile(t, n_mt, n_nt, m0, n0);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % PG_STAGES);
          const long long use = it / PG_STAGES;
          if (use > 0 && !mbar_wait(&sm.empty[s], static_cast<uint32_t>((use - 1) & 1))) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], STAGE_BYTES);
          tma_load_2d(sm.a[s], &ta, &sm.full[s], kb * PG_BK, m0);
          tma_load_2d(sm.b[s], &tb, &sm.full[s], kb * PG_BK, n0);
        }
      }
      // Let the copies this thread started land before the CTA can exit (bounded waits).
      for (long long i = it - PG_STAGES > 0 ? it - PG_STAGES : 0; i < it; ++i)
        mbar_wait(&sm.full[i % PG_STAGES], static_cast<uint32_t>((i / PG_STAGES) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID = idesc_bf16_f32(PG_BM, PG_BN, 0, 0);
      const uint32_t tbase = sm.tmem_base;
      long long it = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
        const int acc = lt & 1, use_acc = lt >> 1;
        if (*abort_flag) { ok = false; break; }
        if (use_acc > 0 && !mbar_wait(&sm.acc_empty[acc], (use_acc - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tbase + acc * PG_BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % PG_STAGES);
          if (!mbar_wait(&sm.full[s], static_cast<uint32_t>((it / PG_STAGES) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
          for (int kk = 0; kk < PG_BK / 16; ++kk)
            mma_ss(d, smem_desc_sw128(a0 + kk * 32, 16, 1024),
                   smem_desc_sw128(b0 + kk * 32, 16, 1024), ID, (kb | kk) ? 1u : 0u);
          mma_commit(&sm.empty[s]);
        }
        if (ok) mma_commit(&sm.acc_full[acc]);
      }
      if (!ok) *abort_flag = 1;
      // All MMAs issued by this thread are complete once fin flips.
      mma_commit(&sm.fin);
      mbar_wait(&sm.fin, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int lt = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1;
      if (*abort_flag || !mbar_wait(&sm.acc_full[acc], (lt >> 1) & 1)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int m0, n0;
      pg_tile(t, n_mt, n_nt, m0, n0);
      const long long row = m0 + quad * 32 + lane;
      const int ncols = min(PG_BN, p.N - n0);
#pragma unroll 1
      for (int c = 0; c < ncols; c += 32) {
        uint32_t r[32];
        tmem_ld32(sm.tmem_base + lane_base + acc * PG_BN + c, r);
        tmem_wait_ld();
        tmem_ld_fence(r);
        if (row < p.M) pg_store_chunk(p, row, n0 + c, r);
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[acc]);
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
