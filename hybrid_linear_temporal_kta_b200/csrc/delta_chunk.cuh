// delta_chunk.cuh -- chunked gated delta rule (bf16 in / out, fp32 state and gates) on
// warp-level bf16 tensor-core tiles, TMA-fed.
//
// Operator: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar, the four update lines (v_old = M k, v_new = beta v + (1-beta) v_old,
// M = alpha M - v_old k^T + v_new k^T, o = M q). With the key-major state S = M^T (d_k x d_v)
// and row vectors this is  u_t = beta_t (v_t - k_t S_{t-1}),  S_t = alpha_t S_{t-1} + k_t^T u_t,
// o_t = scale * q_t S_t.
//
// The decayed-erase reading (GatedDeltaNet's own update, the branch the page says it is based on)
// is u_t = beta_t (v_t - alpha_t k_t S_{t-1}); it changes only gamma_{t-1} -> gamma_t in T and W
// below (erase_decayed).
//
// Chunked form (derived by unrolling inside a chunk of C tokens; gamma_t = prod_{r<=t} alpha_r,
// gamma_{-1} = 1, S_0 the state at the chunk start, A = (I + T)^{-1} with the strictly lower
// triangular T_ts = beta_t (gamma_{t-1} / gamma_s) (k_t . k_s)):
//   U     = U' - W S_0,      U' = A diag(beta) V,      W = A diag(beta_t gamma_{t-1}) K
//   o_t   = scale * [ gamma_t q_t S_0 + sum_{s<=t} Aq_ts u_s ],  Aq_ts = (gamma_t/gamma_s)(q_t . k_s)
//   S_end = gamma_end S_0 + sum_s (gamma_end / gamma_s) k_s^T u_s
// Only the three products with S_0 depend on earlier chunks. Two kernels:
//   delta_prep_kernel (one CTA per chunk, all chunks at once): cumulative log2 gates, T and Aq,
//     the inverse of I + T (fp32 inverses of the 16 x 16 diagonal blocks, then block forward
//     substitution on the tensor cores) applied to [diag(beta gamma_prev) K | diag(beta) V].
//     Writes W [C][D], U'^T [D][C], Aq [C][C] (bf16) and the gates [C] (fp32) to a workspace.
//   delta_scan_kernel (one CTA per (value block, sequence, head), chunks in order): a producer
//     warp streams W, q, k, Aq, U'^T and the gates of the coming chunks into a ring of shared-
//     memory stages with TMA (128-byte swizzle); each pair of chain warps owns 16 value
//     columns, each warp half of the key dims of their state rows S^T (16 x D/2, fp32, in
//     registers), so the chunk-to-chunk chain stays in registers apart from one exchange of
//     partial sums inside the pair:
//       U^T = U'^T - S^T W^T,   S^T <- gamma_end S^T + (U^T diag(gamma_end / gamma)) K;
//     a pair of output warps per group takes S_0^T and U^T as bf16 fragments through shared
//     memory and forms o^T = (S_0^T q^T) diag(gamma) + U^T Aq^T off that chain.
#pragma once

#include "kta_ptx.cuh"
#include "mma_sync.cuh"

namespace kta {

constexpr int DELTA_C = 64;

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
  int nch;                // chunks per sequence
  int erase_decayed;      // 1: decayed erase (GatedDeltaNet form): gamma_{t-1} -> gamma_t in T, W
  __nv_bfloat16* ws_W;    // [B*H][nch][C][D]
  __nv_bfloat16* ws_U;    // [B*H][nch][D][C]   (U'^T)
  __nv_bfloat16* ws_A;    // [B*H][nch][C][C]
  float* ws_g;            // [B*H][nch][C]      cumulative log2 gates
};

// ------------------------------------------------------------------------------ prep kernel

template <int D>
struct DeltaPrepSmem {
  static constexpr int C = DELTA_C;
  static constexpr int LDK = D + 8;   // padded rows: conflict-free ldmatrix
  static constexpr int LDC = C + 8;
  union {
    __nv_bfloat16 q[C * LDK];   // raw q (until Q K^T is in registers)
    float tf[C * (C + 1)];      // then T in fp32
  };
  __nv_bfloat16 k[C * LDK];     // raw k, then W (in place)
  __nv_bfloat16 v[C * LDK];     // raw v, then U' (in place)
  __nv_bfloat16 tn[C * LDC];    // -T in bf16
  __nv_bfloat16 aq[C * LDC];    // Aq in bf16
  __nv_bfloat16 xd[4][16 * 24]; // inverses of the 16 x 16 diagonal blocks of I + T
  float lg[C];                  // cumulative log2 alpha
  float beta[C];
};

template <int D>
__global__ void __launch_bounds__(128, 3) delta_prep_kernel(const DeltaParams p) {
  using SM = DeltaPrepSmem<D>;
  constexpr int C = SM::C, LDK = SM::LDK, LDC = SM::LDC, LDT = C + 1;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int cidx = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int c0 = cidx * C;
  const int n = min(C, p.N - c0);
  const long long row_b = static_cast<long long>(b) * p.rows_b;

  // ---- q, k, v rows of the chunk (rows >= n zero-filled); gates
  {
    constexpr int QCH = D / 8;
    for (int idx = tid; idx < C * QCH; idx += 128) {
      const int t = idx / QCH, c = (idx % QCH) * 8;
      const long long grow = row_b + c0 + min(t, n - 1);
      const long long off = grow * p.ld + static_cast<long long>(h) * D + c;
      const int bytes = t < n ? 16 : 0;
      cp_async16(&sm.q[t * LDK + c], p.q + off, bytes);
      cp_async16(&sm.k[t * LDK + c], p.k + off, bytes);
      cp_async16(&sm.v[t * LDK + c], p.v + off, bytes);
    }
    if (warp == 0) {
      // cumulative log2 alpha over the chunk (two tokens per lane, warp scan); padding rows have
      // alpha = 1 and beta = 0.
      float a0 = 0.f, a1 = 0.f;
      const int t0 = 2 * lane, t1 = 2 * lane + 1;
      const long long r0 = (row_b + c0 + t0) * p.H + h, r1 = (row_b + c0 + t1) * p.H + h;
      if (t0 < n) { a0 = __log2f(p.alpha[r0]); sm.beta[t0] = p.beta[r0]; } else sm.beta[t0] = 0.f;
      if (t1 < n) { a1 = __log2f(p.alpha[r1]); sm.beta[t1] = p.beta[r1]; } else sm.beta[t1] = 0.f;
      const float pair = a0 + a1;
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

  // ---- K K^T and Q K^T for rows [16w, 16w+16): T (s < t) and Aq (s <= t)
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
    __syncthreads();  // every warp's q fragments are in registers: T may overwrite q
#pragma unroll
    for (int nt = 0; nt < C / 8; ++nt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = r0 + g4 + (r >= 2 ? 8 : 0);
        const int s = nt * 8 + 2 * t4 + (r & 1);
        const float lgt = sm.lg[t], lgs = sm.lg[s];
        // the erase term sees gamma_{t-1} (page form) or gamma_t (decayed erase)
        const float lgp = p.erase_decayed ? lgt : (t > 0 ? sm.lg[t - 1] : 0.f);
        const float tv = s < t ? sm.beta[t] * exp2f(lgp - lgs) * kk_acc[nt][r] : 0.f;
        const float av = s <= t ? exp2f(lgt - lgs) * qk_acc[nt][r] : 0.f;
        sm.tf[t * LDT + s] = tv;
        kk_acc[nt][r] = -tv;
        qk_acc[nt][r] = av;
      }
      const int t = r0 + g4, s = nt * 8 + 2 * t4;
      *reinterpret_cast<uint32_t*>(&sm.tn[t * LDC + s]) = bf16x2(kk_acc[nt][0], kk_acc[nt][1]);
      *reinterpret_cast<uint32_t*>(&sm.tn[(t + 8) * LDC + s]) = bf16x2(kk_acc[nt][2], kk_acc[nt][3]);
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
  __syncthreads();

  // ---- block forward substitution: Z_i = X_ii (R_i - sum_{j<i} T_ij Z_j) on the right-hand
  // sides R = [diag(beta_t gamma_{t-1}) K | diag(beta) V]; warp w owns D/2 of the 2D columns
  // (warps 0, 1: the K side -> W; warps 2, 3: the V side -> U'), in place over k / v.
  {
    constexpr int CW = D / 2, NTW = CW / 8;
    const bool kside = warp < 2;
    const int col0 = (warp & 1) * CW;
    __nv_bfloat16* buf = kside ? sm.k : sm.v;
#pragma unroll 1
    for (int i = 0; i < C / 16; ++i) {
      const int ta = i * 16 + g4, tb = ta + 8;
      const int pa = p.erase_decayed ? ta : ta - 1, pb = p.erase_decayed ? tb : tb - 1;
      const float fa = kside ? sm.beta[ta] * (pa >= 0 ? exp2f(sm.lg[pa]) : 1.f) : sm.beta[ta];
      const float fb = kside ? sm.beta[tb] * exp2f(sm.lg[pb]) : sm.beta[tb];
      float acc[NTW][4];
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
        const int col = col0 + nt * 8 + 2 * t4;
        const float2 ra = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&buf[ta * LDK + col]));
        const float2 rb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&buf[tb * LDK + col]));
        acc[nt][0] = fa * ra.x;
        acc[nt][1] = fa * ra.y;
        acc[nt][2] = fb * rb.x;
        acc[nt][3] = fb * rb.y;
      }
      for (int j = 0; j < i; ++j) {
        uint32_t a[4];
        ldsm_x4(a, &sm.tn[frag_a_rowmajor(lane, i * 16, j * 16, LDC)]);
#pragma unroll
        for (int np = 0; np < NTW / 2; ++np) {
          uint32_t bz[4];
          ldsm_x4_t(bz, &buf[frag_b_kmajor(lane, j * 16, col0 + np * 16, LDK)]);
          mma16816(acc[2 * np], a, bz[0], bz[1]);
          mma16816(acc[2 * np + 1], a, bz[2], bz[3]);
        }
      }
      // stage Y_i (bf16) over rows of block i (each lane rewrites the elements it read)
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
        const int col = col0 + nt * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(&buf[ta * LDK + col]) = bf16x2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t*>(&buf[tb * LDK + col]) = bf16x2(acc[nt][2], acc[nt][3]);
      }
      __syncwarp();
      uint32_t ax[4];
      ldsm_x4(ax, &sm.xd[i][frag_a_rowmajor(lane, 0, 0, 24)]);
      float z[NTW][4];
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) z[nt][r] = 0.f;
#pragma unroll
      for (int np = 0; np < NTW / 2; ++np) {
        uint32_t by[4];
        ldsm_x4_t(by, &buf[frag_b_kmajor(lane, i * 16, col0 + np * 16, LDK)]);
        mma16816(z[2 * np], ax, by[0], by[1]);
        mma16816(z[2 * np + 1], ax, by[2], by[3]);
      }
      __syncwarp();
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
        const int col = col0 + nt * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(&buf[ta * LDK + col]) = bf16x2(z[nt][0], z[nt][1]);
        *reinterpret_cast<uint32_t*>(&buf[tb * LDK + col]) = bf16x2(z[nt][2], z[nt][3]);
      }
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- workspace: W, U'^T, Aq, gates
  {
    const long long wsi = static_cast<long long>(bh) * p.nch + cidx;
    __nv_bfloat16* W = p.ws_W + wsi * C * D;
    constexpr int QCH = D / 8;
    for (int idx = tid; idx < C * QCH; idx += 128) {
      const int t = idx / QCH, c = (idx % QCH) * 8;
      *reinterpret_cast<uint4*>(&W[t * D + c]) = *reinterpret_cast<const uint4*>(&sm.k[t * LDK + c]);
    }
    __nv_bfloat16* A = p.ws_A + wsi * C * C;
    for (int idx = tid; idx < C * (C / 8); idx += 128) {
      const int t = idx / (C / 8), c = (idx % (C / 8)) * 8;
      *reinterpret_cast<uint4*>(&A[t * C + c]) = *reinterpret_cast<const uint4*>(&sm.aq[t * LDC + c]);
    }
    // U'^T: transposed 8 x 8 blocks of U' (ldmatrix.trans) into a [D][C] tile over the free q / T
    // region, its 16-byte pieces XOR-swizzled by row so that both the pair stores and the row
    // reads are conflict-free, then whole rows to the workspace
    static_assert(D * C * 2 <= sizeof(sm.q), "transpose tile");
    uint8_t* ut = reinterpret_cast<uint8_t*>(sm.q);
#pragma unroll
    for (int tb = 2 * warp; tb < 2 * warp + 2; ++tb) {
#pragma unroll
      for (int jb = 0; jb < D / 32; ++jb) {
        // matrix m = lane / 8 covers tokens 8 tb .. +7 and value columns 32 jb + 8 m .. +7; this
        // lane receives tokens 8 tb + 2 (lane % 4), +1 of value column 32 jb + 8 m + lane / 4
        uint32_t r[4];
        ldsm_x4_t(r, &sm.v[(8 * tb + (lane & 7)) * LDK + 32 * jb + 8 * (lane >> 3)]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int j = 32 * jb + 8 * m + (lane >> 2);
          *reinterpret_cast<uint32_t*>(ut + j * (C * 2) + ((tb ^ (j & 7)) << 4) + 4 * (lane & 3)) = r[m];
        }
      }
    }
    __syncthreads();
    __nv_bfloat16* U = p.ws_U + wsi * D * C;
    for (int idx = tid; idx < D * (C / 8); idx += 128) {
      const int j = idx / (C / 8), c = idx % (C / 8);
      *reinterpret_cast<uint4*>(&U[j * C + c * 8]) =
          *reinterpret_cast<const uint4*>(ut + j * (C * 2) + ((c ^ (j & 7)) << 4));
    }
    if (tid < C) p.ws_g[wsi * C + tid] = sm.lg[tid];
  }
}

// ------------------------------------------------------------------------------ scan kernel

// Byte offset of element (row, col) in a tile of ROWS rows x (64 * boxes) bf16 columns stored as
// boxes of [ROWS][64] with the TMA 128-byte swizzle (16-byte group index XOR row % 8).
template <int ROWS>
__device__ __forceinline__ uint32_t swz(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * (ROWS * 128) + row * 128 +
                               ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

template <int D, int VG, int NST>
struct DeltaScanSmem {
  static constexpr int C = DELTA_C;
  static constexpr int VB = 16 * VG;      // value columns per CTA (VG groups of 16)
  static constexpr int NCW = 2 * VG;      // chain warps: two per group (key-dim halves)
  static constexpr int NOW = 2 * VG;      // output warps: two per group (token halves)
  static constexpr int NBOX = D / 64;
  static constexpr int NKH = D / 32;      // k steps over a key-dim half
  static constexpr int NTP = C / 16;      // 16-token groups per chunk
  static constexpr int XCH = C / 8 * 4;   // floats a chain lane hands its partner per chunk
  struct alignas(1024) Stage {
    __nv_bfloat16 w[NBOX * C * 64];
    __nv_bfloat16 q[NBOX * C * 64];
    __nv_bfloat16 k[NBOX * C * 64];
    __nv_bfloat16 aq[C * 64];
    __nv_bfloat16 ut[VB * 64];
    float lg[C];
  };
  static constexpr uint32_t STAGE_TX =
      (3 * NBOX * C * 64 + C * 64 + VB * 64) * 2 + C * 4;  // bytes the TMA unit writes per stage
  Stage stage[NST];
  alignas(128) __nv_bfloat16 o[2][C * VB];  // output tiles [token][value column] for TMA stores
  float xch[2][NCW][XCH][32];   // partial sums of X exchanged within a chain pair (chunk parity)
  // chain -> output warps, by chunk parity: S_0^T as bf16 A fragments (per group, key half and
  // k step) and U^T as bf16 A fragments (per group and token group), one uint4 per lane
  uint4 hs[2][VG][2][NKH][32];
  uint4 hu[2][VG][NTP][32];
  int pair_ok[2][NCW];
  uint64_t full[NST];
  uint64_t empty[NST];
  uint64_t hfull[2];            // chain -> output warps: the chunk's S_0^T and U^T are written
  uint64_t hfree[2];            // output -> chain warps: read into registers
  uint64_t ofull[2];            // output warps -> producer: output tile written
  uint64_t ofree[2];            // producer -> output warps: output tile read by the TMA store
};

template <int D, int VG, int NST>
constexpr size_t delta_scan_smem_bytes() {
  return sizeof(DeltaScanSmem<D, VG, NST>) + 1024;  // + manual 1024-byte alignment
}

// Chain warp 2g + hk owns value columns [16g, 16g+16) of the CTA's block and key dims
// [hk D/2, (hk+1) D/2) of their state rows S^T. Per chunk the pair forms the key-dim partial sums
// of X = S^T W^T, swaps them through shared memory (one pair barrier), then each warp updates its
// own key-dim half of S^T. Output warp 2g + ho of the same group takes the chunk's S_0^T and U^T
// fragments from the chain pair through shared memory and forms the outputs of tokens
// [ho C/2, (ho+1) C/2): (S_0^T q^T) diag(gamma) + U^T Aq^T, off the chunk-to-chunk chain. The
// producer warp loads the stages and stores the output tiles (TMA).
template <int D, int VG, int NST>
__global__ void __launch_bounds__((4 * VG + 1) * 32, 1)
    delta_scan_kernel(const __grid_constant__ CUtensorMap tW, const __grid_constant__ CUtensorMap tQ,
                      const __grid_constant__ CUtensorMap tK, const __grid_constant__ CUtensorMap tA,
                      const __grid_constant__ CUtensorMap tU, const __grid_constant__ CUtensorMap tO,
                      const DeltaParams p) {
  using SM = DeltaScanSmem<D, VG, NST>;
  constexpr int C = SM::C, VB = SM::VB, NCW = SM::NCW, NOW = SM::NOW, NBOX = SM::NBOX;
  constexpr int DH = D / 2;               // key dims per chain warp
  constexpr int NKH = SM::NKH;            // k steps over a key-dim half
  constexpr int NTP = SM::NTP;            // 16-token groups per chunk
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int j0 = blockIdx.x * VB, bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], NCW + NOW);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.hfull[i], NCW);
      mbar_init(&sm.hfree[i], NOW);
      mbar_init(&sm.ofull[i], NOW);
      mbar_init(&sm.ofree[i], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW + NOW) {
    // ---- producer: one lane loads the stages and stores the output tiles
    if (lane == 0) {
      prefetch_tmap(&tW);
      prefetch_tmap(&tQ);
      prefetch_tmap(&tK);
      prefetch_tmap(&tA);
      prefetch_tmap(&tU);
      prefetch_tmap(&tO);
      auto store_out = [&](int j) -> bool {
        const int ob = j & 1;
        if (!mbar_wait(&sm.ofull[ob], (j >> 1) & 1)) return false;
        tma_store_4d(&tO, sm.o[ob], j0, h, j * C, b);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(&sm.ofree[ob]);
        return true;
      };
      bool good = true;
      for (int c = 0; c < p.nch && good; ++c) {
        const int s = c % NST;
        if (c >= NST && !mbar_wait(&sm.empty[s], ((c / NST) - 1) & 1)) break;
        typename SM::Stage& S = sm.stage[s];
        uint64_t* bar = &sm.full[s];
        mbar_arrive_expect_tx(bar, SM::STAGE_TX);
        const long long wsi = static_cast<long long>(bh) * p.nch + c;
        const int wrow = static_cast<int>(wsi * C);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx) {
          tma_load_2d(S.w + bx * C * 64, &tW, bar, bx * 64, wrow);
          tma_load_4d(S.q + bx * C * 64, &tQ, bar, bx * 64, h, c * C, b);
          tma_load_4d(S.k + bx * C * 64, &tK, bar, bx * 64, h, c * C, b);
        }
        tma_load_2d(S.aq, &tA, bar, 0, wrow);
        tma_load_2d(S.ut, &tU, bar, 0, static_cast<int>(wsi * D + j0));
        bulk_load(S.lg, p.ws_g + wsi * C, C * 4, bar);
        if (c >= 1) good = store_out(c - 1);
      }
      if (good && p.nch > 0) store_out(p.nch - 1);
      bulk_wait_all();
    }
    return;
  }

  // lane row / column offsets of the ldmatrix address patterns
  const int nm_r = (lane & 7) + (lane >> 4) * 8, nm_c = ((lane >> 3) & 1) * 8;  // B stored [n][k]
  const int km_r = (lane & 7) + ((lane >> 3) & 1) * 8, km_c = (lane >> 4) * 8;  // B stored [k][n]

  if (warp < NCW) {
    // ---- chain warps
    const int grp = warp >> 1, hk = warp & 1, mate = warp ^ 1;
    const int vr = 16 * grp + g4;           // this lane's value rows vr, vr + 8 (within the block)
    const int jv = j0 + vr;
    const int kb = hk * DH;                 // first key dim of this warp's half
    const long long sb = static_cast<long long>(bh) * D * D;
    // st[nt][r] = S^T[jv (+8 for r >= 2)][kb + 8 nt + 2 t4 + (r & 1)]
    float st[DH / 8][4];
#pragma unroll
    for (int nt = 0; nt < DH / 8; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r)
        st[nt][r] = p.S0 ? p.S0[sb + (kb + nt * 8 + 2 * t4 + (r & 1)) * D + jv + (r >= 2 ? 8 : 0)] : 0.f;

    bool failed = false;
    int c = 0;
    for (; c < p.nch; ++c) {
      const int s = c % NST, hb = c & 1;
      // the stage has landed, and the output warps have read the hand-over buffer of two chunks ago
      const bool ok = !failed && mbar_wait(&sm.full[s], (c / NST) & 1) &&
                      (c < 2 || mbar_wait(&sm.hfree[hb], ((c - 2) >> 1) & 1));
      float (*mine)[32] = sm.xch[hb][warp];
      float (*theirs)[32] = sm.xch[hb][mate];
      float xw[C / 8][4];
      const typename SM::Stage& S = sm.stage[s];
      const uint8_t* Wb = reinterpret_cast<const uint8_t*>(S.w);
      const uint8_t* Kb = reinterpret_cast<const uint8_t*>(S.k);
      const uint8_t* Ub = reinterpret_cast<const uint8_t*>(S.ut);
      if (ok) {
        // (a) this warp's half of S^T (the chunk's start state) as bf16 A fragments (k = key
        // dim), also handed to the output warps
        uint32_t sa[NKH][4];
#pragma unroll
        for (int kk = 0; kk < NKH; ++kk) {
          sa[kk][0] = bf16x2(st[2 * kk][0], st[2 * kk][1]);
          sa[kk][1] = bf16x2(st[2 * kk][2], st[2 * kk][3]);
          sa[kk][2] = bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
          sa[kk][3] = bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
          sm.hs[hb][grp][hk][kk][lane] = make_uint4(sa[kk][0], sa[kk][1], sa[kk][2], sa[kk][3]);
        }
        // (b) key-dim partial sums of X = S^T W^T (n = token); the B fragments of the next k step
        // are loaded while the current one's products issue
#pragma unroll
        for (int nt = 0; nt < C / 8; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) xw[nt][r] = 0.f;
        {
          uint32_t fw[2][NTP][4];
#pragma unroll
          for (int np = 0; np < NTP; ++np) ldsm_x4(fw[0][np], Wb + swz<C>(np * 16 + nm_r, kb + nm_c));
#pragma unroll
          for (int kk = 0; kk < NKH; ++kk) {
            const int cur = kk & 1;
            if (kk + 1 < NKH) {
#pragma unroll
              for (int np = 0; np < NTP; ++np)
                ldsm_x4(fw[cur ^ 1][np], Wb + swz<C>(np * 16 + nm_r, kb + (kk + 1) * 16 + nm_c));
            }
#pragma unroll
            for (int np = 0; np < NTP; ++np) {
              mma16816(xw[2 * np], sa[kk], fw[cur][np][0], fw[cur][np][1]);
              mma16816(xw[2 * np + 1], sa[kk], fw[cur][np][2], fw[cur][np][3]);
            }
          }
        }
        // hand the partner this warp's sums of X
#pragma unroll
        for (int nt = 0; nt < C / 8; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) mine[nt * 4 + r][lane] = xw[nt][r];
      }
      if (lane == 0) sm.pair_ok[hb][warp] = ok ? 1 : 0;
      named_bar_sync(2 + grp, 64);
      if (!ok || !sm.pair_ok[hb][mate]) break;  // the same decision in both warps of the pair

      // (c) U^T = U'^T - X  (value rows vr (+8), token columns)
#pragma unroll
      for (int nt = 0; nt < C / 8; ++nt) {
        const int tc = nt * 8 + 2 * t4;
        const float2 ua = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Ub + swz<VB>(vr, tc)));
        const float2 ub = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Ub + swz<VB>(vr + 8, tc)));
        xw[nt][0] = ua.x - (xw[nt][0] + theirs[nt * 4 + 0][lane]);
        xw[nt][1] = ua.y - (xw[nt][1] + theirs[nt * 4 + 1][lane]);
        xw[nt][2] = ub.x - (xw[nt][2] + theirs[nt * 4 + 2][lane]);
        xw[nt][3] = ub.y - (xw[nt][3] + theirs[nt * 4 + 3][lane]);
      }
      // (d) U^T as A fragments (k = token): plain (to the output warps, from one warp of the
      // pair) and scaled by gamma_end / gamma_s (for the state update)
      const float lgC = S.lg[C - 1];
      uint32_t ur[NTP][4];
#pragma unroll
      for (int kk = 0; kk < NTP; ++kk) {
        const int ta = 16 * kk + 2 * t4, tb = ta + 8;
        const float da0 = exp2f(lgC - S.lg[ta]), da1 = exp2f(lgC - S.lg[ta + 1]);
        const float db0 = exp2f(lgC - S.lg[tb]), db1 = exp2f(lgC - S.lg[tb + 1]);
        if (hk == 0)
          sm.hu[hb][grp][kk][lane] = make_uint4(bf16x2(xw[2 * kk][0], xw[2 * kk][1]),
                                                bf16x2(xw[2 * kk][2], xw[2 * kk][3]),
                                                bf16x2(xw[2 * kk + 1][0], xw[2 * kk + 1][1]),
                                                bf16x2(xw[2 * kk + 1][2], xw[2 * kk + 1][3]));
        ur[kk][0] = bf16x2(xw[2 * kk][0] * da0, xw[2 * kk][1] * da1);
        ur[kk][1] = bf16x2(xw[2 * kk][2] * da0, xw[2 * kk][3] * da1);
        ur[kk][2] = bf16x2(xw[2 * kk + 1][0] * db0, xw[2 * kk + 1][1] * db1);
        ur[kk][3] = bf16x2(xw[2 * kk + 1][2] * db0, xw[2 * kk + 1][3] * db1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.hfull[hb]);
      // (e) this warp's key dims of S^T = gamma_end S^T + Ur^T K  (n = key dim)
      const float gC = exp2f(lgC);
#pragma unroll
      for (int nt = 0; nt < DH / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) st[nt][r] *= gC;
      {
        uint32_t fk[2][NKH][4];
#pragma unroll
        for (int np = 0; np < NKH; ++np) ldsm_x4_t(fk[0][np], Kb + swz<C>(km_r, kb + np * 16 + km_c));
#pragma unroll
        for (int kk = 0; kk < NTP; ++kk) {
          const int cur = kk & 1;
          if (kk + 1 < NTP) {
#pragma unroll
            for (int np = 0; np < NKH; ++np)
              ldsm_x4_t(fk[cur ^ 1][np], Kb + swz<C>((kk + 1) * 16 + km_r, kb + np * 16 + km_c));
          }
#pragma unroll
          for (int np = 0; np < NKH; ++np) {
            mma16816(st[2 * np], ur[kk], fk[cur][np][0], fk[cur][np][1]);
            mma16816(st[2 * np + 1], ur[kk], fk[cur][np][2], fk[cur][np][3]);
          }
        }
      }
      // every read of the stage by this warp is done
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    if (p.S_out && c == p.nch) {
#pragma unroll
      for (int nt = 0; nt < DH / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r)
          p.S_out[sb + (kb + nt * 8 + 2 * t4 + (r & 1)) * D + jv + (r >= 2 ? 8 : 0)] = st[nt][r];
    }
    return;
  }

  // ---- output warps
  const int ow = warp - NCW;
  const int grp = ow >> 1, ho = ow & 1;
  const int vr = 16 * grp + g4;
  bool failed = false;
  for (int c = 0; c < p.nch && !failed; ++c) {
    const int s = c % NST, hb = c & 1;
    if (!mbar_wait(&sm.full[s], (c / NST) & 1) || !mbar_wait(&sm.hfull[hb], (c >> 1) & 1)) break;
    const typename SM::Stage& S = sm.stage[s];
    const uint8_t* Qb = reinterpret_cast<const uint8_t*>(S.q);
    const uint8_t* Ab = reinterpret_cast<const uint8_t*>(S.aq);
    // the chunk's start state S_0^T (both key halves) and U^T, as A fragments
    uint32_t sa[2 * NKH][4], ua[NTP][4];
#pragma unroll
    for (int kk = 0; kk < 2 * NKH; ++kk) {
      const uint4 x = sm.hs[hb][grp][kk / NKH][kk % NKH][lane];
      sa[kk][0] = x.x;
      sa[kk][1] = x.y;
      sa[kk][2] = x.z;
      sa[kk][3] = x.w;
    }
#pragma unroll
    for (int kk = 0; kk < NTP; ++kk) {
      const uint4 x = sm.hu[hb][grp][kk][lane];
      ua[kk][0] = x.x;
      ua[kk][1] = x.y;
      ua[kk][2] = x.z;
      ua[kk][3] = x.w;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.hfree[hb]);
    // (S_0^T q^T) for this warp's tokens [ho C/2, (ho+1) C/2) (n = token, k = key dim), the q
    // fragments of the next k step loaded while the current one's products issue
    constexpr int NPH = NTP / 2;            // 16-token groups per warp
    float ov[2 * NPH][4];
#pragma unroll
    for (int nt = 0; nt < 2 * NPH; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) ov[nt][r] = 0.f;
    {
      uint32_t fq[2][NPH][4];
#pragma unroll
      for (int np = 0; np < NPH; ++np)
        ldsm_x4(fq[0][np], Qb + swz<C>((ho * NPH + np) * 16 + nm_r, nm_c));
#pragma unroll
      for (int kk = 0; kk < 2 * NKH; ++kk) {
        const int cur = kk & 1;
        if (kk + 1 < 2 * NKH) {
#pragma unroll
          for (int np = 0; np < NPH; ++np)
            ldsm_x4(fq[cur ^ 1][np], Qb + swz<C>((ho * NPH + np) * 16 + nm_r, (kk + 1) * 16 + nm_c));
        }
#pragma unroll
        for (int np = 0; np < NPH; ++np) {
          mma16816(ov[2 * np], sa[kk], fq[cur][np][0], fq[cur][np][1]);
          mma16816(ov[2 * np + 1], sa[kk], fq[cur][np][2], fq[cur][np][3]);
        }
      }
    }
    // scale by gamma_t, then add U^T Aq^T (causal: token groups kk <= np)
#pragma unroll
    for (int nt = 0; nt < 2 * NPH; ++nt) {
      const int tc = (ho * NPH) * 16 + nt * 8 + 2 * t4;
      const float g0 = exp2f(S.lg[tc]), g1 = exp2f(S.lg[tc + 1]);
      ov[nt][0] *= g0;
      ov[nt][1] *= g1;
      ov[nt][2] *= g0;
      ov[nt][3] *= g1;
    }
#pragma unroll
    for (int npl = 0; npl < NPH; ++npl) {
      const int np = ho * NPH + npl;
      uint32_t fa[NTP][4];
#pragma unroll
      for (int kk = 0; kk < NTP; ++kk)
        if (kk <= np) ldsm_x4(fa[kk], Ab + swz<C>(np * 16 + nm_r, kk * 16 + nm_c));
#pragma unroll
      for (int kk = 0; kk < NTP; ++kk) {
        if (kk > np) break;
        mma16816(ov[2 * npl], ua[kk], fa[kk][0], fa[kk][1]);
        mma16816(ov[2 * npl + 1], ua[kk], fa[kk][2], fa[kk][3]);
      }
    }
    // every read of the stage by this warp is done
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
    // output tile [token][value column]: wait until the store of two chunks ago has read it
    const int obi = c & 1;
    if (c >= 2 && !mbar_wait(&sm.ofree[obi], ((c - 2) >> 1) & 1)) {
      failed = true;
      break;
    }
    __nv_bfloat16* ob = sm.o[obi];
#pragma unroll
    for (int nt = 0; nt < 2 * NPH; ++nt) {
      const int tc = (ho * NPH) * 16 + nt * 8 + 2 * t4;
      ob[tc * VB + vr] = __float2bfloat16_rn(ov[nt][0] * p.scale);
      ob[(tc + 1) * VB + vr] = __float2bfloat16_rn(ov[nt][1] * p.scale);
      ob[tc * VB + vr + 8] = __float2bfloat16_rn(ov[nt][2] * p.scale);
      ob[(tc + 1) * VB + vr + 8] = __float2bfloat16_rn(ov[nt][3] * p.scale);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.ofull[obi]);
  }
}

}  // namespace kta
