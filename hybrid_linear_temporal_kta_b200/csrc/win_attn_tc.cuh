// win_attn_tc.cuh -- frame-windowed softmax attention (SWA and DSWA) on the sm_100a tensor cores.
//
// Operator: paper-read "Kairos: A Native World Model Stack for Physical AI", section 2, second
// pillar. SWA: standard attention over a window of W whole frames ending at the query's frame.
// DSWA: the same window size with frames taken every dil-th step back (f, f-dil, ...).
//
// Query tiles of up to 128 rows lie in ONE frame (tiles restart at every frame start), so every
// row of a tile sees the same key frames and the only mask is a column bound on the last key tile
// of the window (or of each key span). For dil == 1 the W visible frames are adjacent and form
// one span; for dil > 1 with P a multiple of 8 the visible frames are packed into one sequence of
// keys whose tiles may straddle two frames (loaded as 8-row boxes from both), otherwise each
// visible frame is its own span.
//
// One CTA (one per SM: it holds all 512 TMEM columns) computes a PAIR of query tiles A and B of
// the same sequence, head and frame (launches too small to fill the GPU with pairs give each CTA
// one tile); both use every K / V tile, which is loaded once for the pair
// into a four-slot ring (K_0, V_0, K_1, V_1, ...; 128 keys x D, 128-byte swizzle), so the loads
// run a full key tile ahead of the tensor core. Warp roles (384 threads):
//   warp 0       TMA producer: Q_A and Q_B once, then the K / V ring.
//   warp 1       allocates TMEM (S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512)); one
//                thread issues tcgen05.mma in the order S_A(0) S_B(0) | PV_A(i) S_A(i+1) PV_B(i)
//                S_B(i+1) | ...: S = Q K^T (SS form), O += P V (TS form, P read from TMEM where
//                the softmax wrote it over S, V MN-major). MMAs of one thread run in issue order,
//                so S_X(i+1) overwrites P_X(i) only after PV_X(i) has read it, and the softmax of
//                S_X(i+1) finds O_X stable.
//   warp 2       with a key split (below), the second producer: the second half's K / V.
//   warp 3       idle after set-up.
//   warps 4..7   softmax of tile A; warps 8..11 softmax of tile B: thread <-> query row (TMEM
//                lane). Lazy rescale of O when the row max grows by more than 2^8; after the
//                first tile the exponentials P = exp2(S*scale*log2e - m) are taken against the
//                current m while the row max is formed (three-input max), and redone only when
//                the max grew past that bound, so the max is off the critical path. P goes to
//                TMEM as bf16 (scaling and row sums on packed fp32 pairs); one arrival per warp
//                hands P to the MMA thread (128 arrivals on one barrier serialise); epilogue
//                O / l -> bf16 -> the tile's Q buffer (free once its last product has run) ->
//                one TMA store of 32 rows per warp (rows past the frame are outside the map).
// While the softmax of one tile runs, the tensor core works on the other tile's products. A CTA
// left with a single query tile (a ragged last tile, or every tile of a launch too small for
// pairs) gives its two accumulators the two halves of that tile's key range instead and merges
// the two partial results (running maxima, sums and O) before the store.
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
  int pair;         // query tiles per CTA: 2 (tiles 2u, 2u+1) or 1 (small launches)
  int Htot;         // heads in this launch (group 0 then group 1)
  int H0;           // heads of group 0
  int W[2];         // window (frames) per group
  int dil[2];       // dilation per group
  int kh_off[2];    // head coordinate in the group's K/V map = h - kh_off[g]
  int kb_frames[2]; // frames per sequence in the group's K/V buffer
  int kmod[2];      // frame index modulus in the K/V buffer (ring slots; = F for a sequence)
  int span_mode[2]; // 1: the group's visible frames are not adjacent in its buffer (a ring of
                    // W slots), so each frame is its own span even with dil == 1
  int q_rows_b;     // rows per sequence in the q / o buffers
  float scale_log2; // softmax scale * log2(e)
  __nv_bfloat16* o; // output, already offset to the launch's first head
  long long o_ld;   // output row stride in elements
  int o_tma;        // 1: rows leave through the tile's Q buffer and TMA stores (map `to`)
  float* lse;       // optional [B][Htot][q_rows_b]: m + log2(l), the base-2 log-sum-exp of
                    // scale * log2(e) * S over each row's visible keys (null = not written)
};

// Work item `item` (a CTA index): frames latest first (full windows first), then head, sequence,
// tile pair.
struct WinItem {
  int pr, b, h, f_local;
};
__device__ __forceinline__ WinItem win_item(int item, const WinParams& p) {
  WinItem w;
  const int n_units = p.pair == 2 ? (p.n_qt + 1) >> 1 : p.n_qt;
  w.pr = item % n_units;  // first query tile: pr * p.pair
  item /= n_units;
  w.b = item % p.B;
  item /= p.B;
  w.h = item % p.Htot;
  item /= p.Htot;
  w.f_local = p.Fq - 1 - item;
  return w;
}

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

// Key tiles of the forward kernel. For dil > 1 with P a multiple of 8 the visible frames are
// packed: they form one sequence of nsp * P keys cut into 128-key tiles, so only the window's last
// tile is ragged (per-frame tiles would leave a ragged tile in every frame). A packed tile takes
// rows_a rows (a multiple of 8) from frame fr_a at row off_a and the rest from the first rows of
// frame fr_b, when that rest fits in one frame (always for P >= 120; shorter frames may need
// several, which the kernel's MF form loads box by box); nv keys of it are visible. Otherwise the
// tiles are win_tile's.
struct WinKTile {
  int fr_a, off_a, rows_a, fr_b, nv;
};
// (packed only where it saves tiles: with P = 880 the per-frame tiles are already as few). With
// `spans` (a dil == 1 window whose frames sit in a ring, not side by side) each frame is its own
// span as well, and the frames are packed whenever P is a multiple of 8: the packed tiles then
// start at the same keys as the tiles of the adjacent-frame layout, so results agree bit for bit.
__device__ __forceinline__ bool win_per_frame(int dil, bool spans) { return dil > 1 || spans; }
__device__ __forceinline__ bool win_packed(int f, int P, int W, int dil, bool spans) {
  if (!win_per_frame(dil, spans) || (P & 7) != 0) return false;
  if (dil == 1) return true;
  const int nsp = min(W, f / dil + 1);
  return (nsp * P + 127) / 128 < nsp * ((P + 127) / 128);
}
__device__ __forceinline__ int win_ktiles(int f, int P, int W, int dil, bool spans) {
  if (!win_per_frame(dil, spans)) return win_num_tiles(f, P, W, dil);
  const int nsp = min(W, f / dil + 1);
  if (!win_packed(f, P, W, dil, spans)) return nsp * ((P + 127) / 128);
  return (nsp * P + 127) / 128;
}
__device__ __forceinline__ WinKTile win_ktile(int i, int f, int P, int W, int dil, bool spans) {
  WinKTile t;
  if (!win_per_frame(dil, spans)) {
    win_tile(i, f, P, W, dil, t.fr_a, t.off_a, t.nv);
    t.rows_a = 128;
    t.fr_b = t.fr_a;
    return t;
  }
  const int nsp = min(W, f / dil + 1);
  if (!win_packed(f, P, W, dil, spans)) {
    // one frame per span, its own tiles
    const int tp = (P + 127) / 128;
    const int j = i / tp, tt = i % tp;
    t.fr_a = f - (nsp - 1 - j) * dil;
    t.off_a = 128 * tt;
    t.nv = min(128, P - t.off_a);
    t.rows_a = 128;
    t.fr_b = t.fr_a;
    return t;
  }
  const int v0 = 128 * i, j = v0 / P, o1 = v0 - j * P;
  t.fr_a = f - (nsp - 1 - j) * dil;
  t.off_a = o1;
  t.rows_a = min(128, P - o1);
  // rows past the window's last key come from any visible frame (finite data, masked by nv)
  t.fr_b = j + 1 < nsp ? t.fr_a + dil : t.fr_a;
  t.nv = min(128, nsp * P - v0);
  return t;
}

template <int D>
struct WinSmem {
  static constexpr int BOX = 128 * 64 * 2;  // one 128-row x 64-column bf16 box, 16 KB
  static constexpr int NBOX = D / 64;
  static constexpr int NSLOT = 4;           // K / V ring slots
  alignas(1024) uint8_t q[2][NBOX * BOX];
  alignas(1024) uint8_t kv[NSLOT][NBOX * BOX];
  uint64_t bar_q[2], full[NSLOT], empty[NSLOT], bar_s[2], bar_p[2], bar_o[2], bar_fin;
  float part_m[128], part_l[128];  // key split: row max and row sum of the second key half
  int part_ok[4];                  // key split: the second half's warps finished
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t win_smem_bytes() {
  return sizeof(WinSmem<D>) + 1024;  // + manual 1024-byte alignment of the dynamic base
}

// LSE: also store each row's base-2 log-sum-exp to p.lse (a separate instantiation, so that the
// plain forward's code is unchanged). MF: frames shorter than 120 keys with P a multiple of 8, so
// that a packed key tile may cross several frame boundaries (also a separate instantiation: the
// extra loader path, inlined or called, slowed the hot loops of the common form by 2-4 %).
template <int D, bool LSE = false, bool MF = false>
__global__ void __launch_bounds__(384, 1)
    win_attn_tc_kernel(const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk0,
                       const __grid_constant__ CUtensorMap tv0,
                       const __grid_constant__ CUtensorMap tk1,
                       const __grid_constant__ CUtensorMap tv1,
                       const __grid_constant__ CUtensorMap tk0s,
                       const __grid_constant__ CUtensorMap tv0s,
                       const __grid_constant__ CUtensorMap tk1s,
                       const __grid_constant__ CUtensorMap tv1s,
                       const __grid_constant__ CUtensorMap to, const WinParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ uint8_t smem_raw[];
  WinSmem<D>& sm = *reinterpret_cast<WinSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int BOX = WinSmem<D>::BOX;
  constexpr int NBOX = WinSmem<D>::NBOX;
  constexpr int NSLOT = WinSmem<D>::NSLOT;
  constexpr uint32_t TILE_BYTES = 128 * D * 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item
  const WinItem wi = win_item(blockIdx.x, p);
  const int pr = wi.pr, b = wi.b, h = wi.h, f_local = wi.f_local;
  const int f = f_local + p.f_base;
  const int g = h >= p.H0 ? 1 : 0;
  const int W = g ? p.W[1] : p.W[0];
  const int dil = g ? p.dil[1] : p.dil[0];
  const int hk = h - (g ? p.kh_off[1] : p.kh_off[0]);
  const int kbf = g ? p.kb_frames[1] : p.kb_frames[0];
  const int kmod = g ? p.kmod[1] : p.kmod[0];
  const CUtensorMap* tk = g ? &tk1 : &tk0;
  const CUtensorMap* tv = g ? &tv1 : &tv0;
  const CUtensorMap* tks = g ? &tk1s : &tk0s;  // 8-row boxes, for tiles that span two frames
  const CUtensorMap* tvs = g ? &tv1s : &tv0s;
  const bool spans = (g ? p.span_mode[1] : p.span_mode[0]) != 0;
  const int ntiles = win_ktiles(f, p.P, W, dil, spans);
  const bool has_b = p.pair == 2 && 2 * pr + 1 < p.n_qt;
  // A CTA with one query tile and at least two key tiles splits the key range instead: tile slot 0
  // takes key tiles [0, nA), slot 1 the rest for the same query rows, and the two partial softmax
  // results are merged before the output is written.
  const bool split = !has_b && ntiles >= 2;
  const int nA = split ? (ntiles + 1) / 2 : ntiles;
  const int nB = split ? ntiles - nA : (has_b ? ntiles : 0);
  const int q_row0 = b * p.q_rows_b + f_local * p.P + pr * p.pair * 128;  // tile A; B = +128

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q[0], 1);
    mbar_init(&sm.bar_q[1], 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.bar_s[x], 1);
      mbar_init(&sm.bar_p[x], 4);  // one arrival per softmax warp
      mbar_init(&sm.bar_o[x], 1);
    }
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

  if (warp == 0 || (warp == 2 && split)) {
    // ------------------------------------------------------------ TMA producer(s): warp 0 loads
    // Q and the K / V ring; with a key split, warp 0 loads the first half's K / V and warp 2 the
    // second's, so that neither half's next tiles wait behind the other's slot releases.
    if (lane == 0) {
      const int half = warp == 2 ? 1 : 0;
      prefetch_tmap(tk);
      prefetch_tmap(tv);
      if (half == 0) {
        prefetch_tmap(&tq);
        // Q_A first, then K_0 (below), then Q_B: the first product S_A(0) needs only Q_A and K_0
        mbar_arrive_expect_tx(&sm.bar_q[0], TILE_BYTES);
        for (int c = 0; c < NBOX; ++c)
          tma_load_3d(sm.q[0] + c * BOX, &tq, &sm.bar_q[0], c * 64, h, q_row0);
      }
      bool qb_issued = false;
      auto load_qb = [&]() {
        qb_issued = true;
        mbar_arrive_expect_tx(&sm.bar_q[1], TILE_BYTES);
        for (int c = 0; c < NBOX; ++c)
          tma_load_3d(sm.q[1] + c * BOX, &tq, &sm.bar_q[1], c * 64, h, q_row0 + 128);
      };
      int uses[NSLOT] = {0, 0, 0, 0};
      // load (key tile kt, V or K) into `slot` as that slot's next use
      auto load = [&](int kt, bool is_v, int slot) {
        const WinKTile t = win_ktile(kt, f, p.P, W, dil, spans);
        const int krow = (b * kbf + t.fr_a % kmod) * p.P + t.off_a;
        const int use = uses[slot];
        if (use > 0 && !mbar_wait(&sm.empty[slot], (use - 1) & 1)) { *abort_flag = 1; return false; }
        mbar_arrive_expect_tx(&sm.full[slot], TILE_BYTES);
        if (t.rows_a == 128) {
          const CUtensorMap* tm = is_v ? tv : tk;
          for (int c = 0; c < NBOX; ++c)
            tma_load_3d(sm.kv[slot] + c * BOX, tm, &sm.full[slot], c * 64, hk, krow);
        } else if (MF) {
          // a tile across one or more frame boundaries, in 8-row boxes (one 128-byte swizzle atom
          // each; P is a multiple of 8, so a box never straddles a frame). The boxes step through
          // the window's keys from row off_a of frame fr_a and move to the next visible frame,
          // dil frames on, at each frame's end; boxes past the window's last key repeat its final
          // rows (finite data, masked by nv).
          const CUtensorMap* tm = is_v ? tvs : tks;
          const int nsp = min(W, f / dil + 1);
          int jj = (128 * kt) / p.P, row = t.off_a, fslot = t.fr_a % kmod;
          for (int r = 0; r < 128; r += 8) {
            const int src = (b * kbf + fslot) * p.P + row;
            for (int c = 0; c < NBOX; ++c)
              tma_load_3d(sm.kv[slot] + c * BOX + r * 128, tm, &sm.full[slot], c * 64, hk, src);
            row += 8;
            if (row == p.P) {
              if (jj + 1 < nsp) {
                ++jj;
                row = 0;
                fslot += dil;
                while (fslot >= kmod) fslot -= kmod;
              } else {
                row = p.P - 8;
              }
            }
          }
        } else {
          // a tile across two frames, in 8-row boxes (one 128-byte swizzle atom each)
          const CUtensorMap* tm = is_v ? tvs : tks;
          const int krow_b = (b * kbf + t.fr_b % kmod) * p.P - t.rows_a;
          for (int c = 0; c < NBOX; ++c)
            for (int r = 0; r < 128; r += 8)
              tma_load_3d(sm.kv[slot] + c * BOX + r * 128, tm, &sm.full[slot], c * 64, hk,
                          r < t.rows_a ? krow + r : krow_b + r);
        }
        uses[slot] = use + 1;
        return true;
      };
      if (!split) {
        // load n: K_{n/2} (n even) or V_{n/2} (n odd), slot n % NSLOT
        for (int n = 0; n < 2 * ntiles; ++n) {
          if (*abort_flag || !load(n >> 1, n & 1, n % NSLOT)) break;
          if (n == 0 && has_b) load_qb();
        }
      } else {
        // this half's step i: K into slot `half`, V into slot 2 + `half`
        const int nh = half ? nB : nA, kt0 = half ? nA : 0;
        for (int i = 0; i < nh; ++i)
          if (*abort_flag || !load(kt0 + i, false, half) || !load(kt0 + i, true, 2 + half)) break;
      }
      // Let the copies this thread started land before the CTA can exit (bounded waits).
      if (half == 0) {
        mbar_wait(&sm.bar_q[0], 0);
        if (qb_issued) mbar_wait(&sm.bar_q[1], 0);
      }
      for (int sl = 0; sl < NSLOT; ++sl)
        if (uses[sl] > 0) mbar_wait(&sm.full[sl], (uses[sl] - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t ID_O = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t tbase = sm.tmem_base;
      const uint32_t q_base[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      auto issue_s = [&](int x, int slot) {
        const uint32_t k_base = smem_u32(sm.kv[slot]);
        const uint32_t qx = split ? q_base[0] : q_base[x];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
          mma_ss(tbase + 128 * x, smem_desc_sw128(qx + off, 16, 1024),
                 smem_desc_sw128(k_base + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.bar_s[x]);
      };
      auto issue_pv = [&](int x, int slot, bool first) {
        const uint32_t v_base = smem_u32(sm.kv[slot]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tbase + 256 + 128 * x, tbase + 128 * x + kk * 8,
                 smem_desc_sw128(v_base + kk * 16 * 128, BOX, 1024), ID_O,
                 (!first || kk > 0) ? 1u : 0u);
        mma_commit(&sm.bar_o[x]);
      };
      bool ok = mbar_wait(&sm.bar_q[0], 0) && ntiles > 0;
      if (!split) {
        if (ok && !mbar_wait(&sm.full[0], 0)) ok = false;
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          if (has_b) {
            if (!mbar_wait(&sm.bar_q[1], 0)) ok = false;
            tc_fence_after();
            if (ok) issue_s(1, 0);
          }
          mma_commit(&sm.empty[0]);
        }
        for (int i = 0; ok && i < ntiles; ++i) {
          const int vs = (2 * i + 1) % NSLOT;
          const uint32_t ph = (i >> 1) & 1;  // phase of both slots of tile i
          const bool more = i + 1 < ntiles;
          const int ks1 = (2 * i + 2) % NSLOT;
          const uint32_t ph1 = ((i + 1) >> 1) & 1;
          if (*abort_flag) { ok = false; break; }
          // The V tile of step i and the K tile of step i+1 landed long before P: check them first,
          // so that only the P handoff (an mbarrier wait costs ~200 cycles even when complete)
          // separates the softmax from the next MMAs.
          if (!mbar_wait(&sm.full[vs], ph) || (more && !mbar_wait(&sm.full[ks1], ph1))) {
            ok = false;
            break;
          }
          // tile A: PV_A(i), then S_A(i+1)
          if (!mbar_spin(&sm.bar_p[0], i & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(0, vs, i == 0);
          if (more) issue_s(0, ks1);
          // tile B: PV_B(i), then S_B(i+1)
          if (has_b) {
            if (!mbar_spin(&sm.bar_p[1], i & 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv(1, vs, i == 0);
          }
          mma_commit(&sm.empty[vs]);
          if (more) {
            if (has_b) issue_s(1, ks1);
            mma_commit(&sm.empty[ks1]);
          }
        }
      } else {
        // key split; slots: 0 = K of the first half, 1 = K of the second, 2 / 3 = their V
        if (ok && !(mbar_wait(&sm.full[0], 0) && mbar_wait(&sm.full[1], 0))) ok = false;
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          mma_commit(&sm.empty[0]);
          issue_s(1, 1);
          mma_commit(&sm.empty[1]);
        }
        for (int i = 0; ok && i < nA; ++i) {
          const uint32_t ph = i & 1, ph1 = (i + 1) & 1;
          const bool act_b = i < nB, more_a = i + 1 < nA, more_b = i + 1 < nB;
          if (*abort_flag) { ok = false; break; }
          // each operand is checked right before its own MMAs: the halves' loads run
          // independently, and a late K of one half must not hold back the other's PV
          if (!mbar_wait(&sm.full[2], ph) || !mbar_spin(&sm.bar_p[0], ph)) { ok = false; break; }
          tc_fence_after();
          issue_pv(0, 2, i == 0);
          mma_commit(&sm.empty[2]);
          if (more_a) {
            if (!mbar_wait(&sm.full[0], ph1)) { ok = false; break; }
            issue_s(0, 0);
            mma_commit(&sm.empty[0]);
          }
          if (act_b) {
            if (!mbar_wait(&sm.full[3], ph) || !mbar_spin(&sm.bar_p[1], ph)) { ok = false; break; }
            tc_fence_after();
            issue_pv(1, 3, i == 0);
            mma_commit(&sm.empty[3]);
            if (more_b) {
              if (!mbar_wait(&sm.full[1], ph1)) { ok = false; break; }
              issue_s(1, 1);
              mma_commit(&sm.empty[1]);
            }
          }
        }
      }
      if (!ok) *abort_flag = 1;
      // All MMAs issued by this thread are complete once bar_fin flips.
      mma_commit(&sm.bar_fin);
      mbar_wait(&sm.bar_fin, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue (tile x)
    const int x = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int xq = split ? 0 : x;                              // query tile of this slot
    const int nq = min(128, p.P - (p.pair * pr + xq) * 128);  // rows of this tile in the frame
    const int n_x = x ? nB : nA;                               // key tiles of this slot
    const int kt0 = split && x ? nA : 0;                       // its first key tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = sm.tmem_base + 128 * x;
    const uint32_t tO = sm.tmem_base + 256 + 128 * x;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = n_x > 0;
    for (int i = 0; ok && i < n_x; ++i) {
      const int nv = win_ktile(kt0 + i, f, p.P, W, dil, spans).nv;
      const bool got = !*abort_flag && mbar_wait(&sm.bar_s[x], i & 1);
      if (!__all_sync(0xffffffffu, got)) { *abort_flag = 1; ok = false; break; }
      tc_fence_after();
      // the whole S row in registers: four loads, one wait
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
      tmem_wait_ld();
      tmem_ld_fence(r);
      float mp[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) mp[u] = -INFINITY;
      const uint64_t sc2 = f32x2_pack(sl2, sl2);
      uint64_t lp2[2];
      // P = exp2(S * scale * log2e - mref) as bf16 pairs written over S (the scaling and the row
      // sums on packed fp32 pairs); with_max also forms the row maximum of a full tile (three-
      // input max, four partial maxima) alongside the exponentials
      auto exp_pass = [&](float mref, bool with_max) {
        const uint64_t nm2 = f32x2_pack(-mref, -mref);
        lp2[0] = f32x2_pack(0.f, 0.f);
        lp2[1] = f32x2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = 32 * c + 2 * j;
            if (with_max)
              mp[j & 3] = max3f(mp[j & 3], __uint_as_float(r[col]), __uint_as_float(r[col + 1]));
            float x0, x1;
            f32x2_unpack(ffma2(f32x2_pack(__uint_as_float(r[col]), __uint_as_float(r[col + 1])), sc2, nm2),
                         x0, x1);
            float p0 = ex2_approx(x0);
            float p1 = ex2_approx(x1);
            if (nv < 128) {
              p0 = col < nv ? p0 : 0.f;
              p1 = col + 1 < nv ? p1 : 0.f;
            }
            lp2[j & 1] = fadd2(lp2[j & 1], f32x2_pack(p0, p1));
            pk[j] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + lane_off + 16 * c, pk);
        }
      };
      // Lazy rescale: the reference m moves only when the row maximum grows by more than 2^8, so
      // for a full tile after the first the exponentials are taken against the current m while
      // the maximum is formed, and redone (rarely) when it grew by more than that.
      bool rescale = false;
      float fac = 1.0f;
      if (i > 0 && nv == 128) {
        exp_pass(m, true);
        const float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
        const float mnew = fmaxf(m, mx * sl2);
        const bool need = mnew > m + 8.0f;
        rescale = __any_sync(0xffffffffu, need);
        if (rescale) {
          if (need) {
            fac = ex2_approx(m - mnew);
            m = mnew;
          }
          tmem_wait_st();
          exp_pass(m, false);
        }
      } else {
        if (nv == 128) {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            mp[j & 3] = max3f(mp[j & 3], __uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
        } else {
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (j < nv) mp[j & 3] = fmaxf(mp[j & 3], __uint_as_float(r[j]));
        }
        const float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
        const float mnew = fmaxf(m, mx * sl2);
        if (i == 0) {
          m = mnew;
        } else {
          const bool need = mnew > m + 8.0f;
          rescale = __any_sync(0xffffffffu, need);
          if (need) {
            fac = ex2_approx(m - mnew);
            m = mnew;
          }
        }
        exp_pass(m, false);
      }
      float la, lb, lc, ld;
      f32x2_unpack(lp2[0], la, lb);
      f32x2_unpack(lp2[1], lc, ld);
      if (rescale) {
        // O is stable here: S_x(i) completed, and it runs after PV_x(i-1) on the tensor pipe.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ro[32];
          tmem_ld32(tO + lane_off + 32 * c, ro);
          tmem_wait_ld();
          tmem_ld_fence(ro);
#pragma unroll
          for (int j = 0; j < 32; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * fac);
          tmem_st32(tO + lane_off + 32 * c, ro);
        }
        l *= fac;
      }
      l += (la + lb) + (lc + ld);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_p[x]);
    }
    // epilogue: O / l -> bf16 -> global (rows of this frame only). With a key split the second
    // half hands its row max and row sum over through shared memory; its O stays in TMEM, where
    // the first half's thread of the same row (same TMEM lane quarter) reads it and merges.
    const bool active = x == 0 || has_b || split;
    if (active) {
      bool fin = ok && n_x > 0 && mbar_wait(&sm.bar_o[x], (n_x - 1) & 1);
      fin = __all_sync(0xffffffffu, fin);
      float mb = -INFINITY, lb = 0.f;
      if (split) {
        if (x == 1) {
          sm.part_m[row] = m;
          sm.part_l[row] = l;
          if (lane == 0) sm.part_ok[quad] = fin ? 1 : 0;
        }
        tc_fence_before();
        asm volatile("bar.sync 3, 256;" ::: "memory");
        if (x == 0) {
          fin = fin && sm.part_ok[quad] != 0;
          mb = sm.part_m[row];
          lb = sm.part_l[row];
        }
      }
      if (!fin) {
        *abort_flag = 1;
      } else if (!split || x == 0) {
        tc_fence_after();
        // merge factors of the two halves (fa = 1, fb = 0 without a split)
        const float mm = split ? fmaxf(m, mb) : m;
        const float fa = split ? ex2_approx(m - mm) : 1.f;
        const float fb = split ? ex2_approx(mb - mm) : 0.f;
        const float lt = split ? fa * l + fb * lb : l;
        const float inv = 1.0f / lt;
        const float ia = fa * inv, ib = fb * inv;
        if (LSE && row < nq)
          p.lse[(static_cast<long long>(b) * p.Htot + h) * p.q_rows_b + f_local * p.P +
                (p.pair * pr + x) * 128 + row] = mm + __log2f(lt);
        __nv_bfloat16* orow =
            p.o + static_cast<long long>(q_row0 + 128 * x + row) * p.o_ld + h * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(tO + lane_off + 32 * c, rr);
          tmem_wait_ld();
          tmem_ld_fence(rr);
          if (split) {
            uint32_t rb[32];
            tmem_ld32(tO + 128 + lane_off + 32 * c, rb);
            tmem_wait_ld();
            tmem_ld_fence(rb);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              rr[j] = __float_as_uint(__uint_as_float(rr[j]) * ia + __uint_as_float(rb[j]) * ib);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * inv);
          }
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[j] = pack_bf16x2(__uint_as_float(rr[2 * j]), __uint_as_float(rr[2 * j + 1]));
          if (p.o_tma) {
            // the row's 16-byte pieces go to the tile's Q buffer (free: its last reader, S_x,
            // completed before bar_o[x]) in the 128-byte swizzled layout of the output map
            uint8_t* srow = sm.q[x] + (c >> 1) * BOX + row * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(srow + ((((c & 1) * 4 + j) ^ (row & 7)) << 4)) =
                  make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          } else if (row < nq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
        if (p.o_tma) {
          // each warp stores its 32 rows (one box per 64 columns); rows past the frame fall
          // outside the map's token extent P and are not written
          fence_proxy_async_smem();
          __syncwarp();
          const int trow = (p.pair * pr + x) * 128 + quad * 32;
          if (lane == 0 && trow < p.P) {
            for (int cb = 0; cb < NBOX; ++cb)
              tma_store_5d(&to, sm.q[x] + cb * BOX + quad * 32 * 128, cb * 64, h, trow, f_local, b);
            bulk_commit();
            bulk_wait_read_all();
          }
        }
      }
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
