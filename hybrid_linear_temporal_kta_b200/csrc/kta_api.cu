// kta_api.cu -- the C ABI of libkta.so (declared in include/kta.h): argument validation, tensor
// map encoding, work decomposition and kernel launches for the Hybrid Linear Temporal Attention
// operator. All kernels of the library are compiled into this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "kta.h"
#include "kta_ptx.cuh"
#include "win_attn_tc.cuh"
#include "simt_f32.cuh"
#include "gla_chunk.cuh"
#include "gla_tc.cuh"
#include "delta_chunk.cuh"
#include "bwd_f32.cuh"
#include "proj_gemm.cuh"
#include "win_bwd_tc.cuh"

namespace {

using kta::WinParams;

thread_local std::string g_last_error;

kta_status fail(kta_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define KTA_CUDA(call)                                                                 \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(KTA_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));       \
  } while (0)

inline size_t elem_size(kta_dtype dt) { return dt == KTA_BF16 ? 2 : 4; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map over a token-major buffer: dim0 = d (contiguous), dim1 = heads (stride d),
// dim2 = rows (stride ld elements); box = 64 columns x 1 head x 128 rows, 128-byte swizzle,
// zero fill outside the tensor.
kta_status make_map(CUtensorMap* m, const void* base, int d, int heads, long long rows,
                    long long ld, int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(KTA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KTA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return KTA_OK;
}

// Tiled bf16 map of rank r (dims innermost first, byte strides of dims 1..r-1), 128-byte swizzle.
kta_status make_map_nd(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box,
                       CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(KTA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KTA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return KTA_OK;
}

// 3-D map (d, heads, rows) of a token-major buffer with a box of box_d x 1 x box_rows; bf16 with
// 128-byte swizzle or fp32 without swizzle.
kta_status make_map_box(CUtensorMap* m, const void* base, bool f32, int d, int heads, long long rows,
                        long long ld, int box_d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(KTA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const cuuint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * es, static_cast<cuuint64_t>(ld) * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  f32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KTA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return KTA_OK;
}

// ------------------------------------------------------------------------- per-device state

struct DeviceRes {
  struct Buf {
    void* ptr = nullptr;
    size_t bytes = 0;
  };
  std::map<cudaStream_t, Buf> ws;  // linear-attention workspace per stream (grown on demand)
  std::mutex mu;
};

DeviceRes& device_res(int dev) {
  static std::mutex mu;
  static std::map<int, DeviceRes*> m;
  std::lock_guard<std::mutex> lk(mu);
  auto it = m.find(dev);
  if (it == m.end()) it = m.emplace(dev, new DeviceRes()).first;
  return *it->second;
}

struct ThreadStreams {  // per host thread and device: the two streams of the hybrid fork
  cudaStream_t hi = nullptr;    // softmax heads: the device's highest stream priority
  cudaStream_t side = nullptr;  // linear heads: its lowest
  cudaEvent_t fork = nullptr, join_hi = nullptr, join = nullptr;
};

kta_status thread_streams(ThreadStreams** out) {
  thread_local std::map<int, ThreadStreams> m;
  int dev = 0;
  KTA_CUDA(cudaGetDevice(&dev));
  ThreadStreams& t = m[dev];
  if (!t.side) {
    int least = 0, greatest = 0;
    KTA_CUDA(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    KTA_CUDA(cudaStreamCreateWithPriority(&t.hi, cudaStreamNonBlocking, greatest));
    KTA_CUDA(cudaStreamCreateWithPriority(&t.side, cudaStreamNonBlocking, least));
    KTA_CUDA(cudaEventCreateWithFlags(&t.fork, cudaEventDisableTiming));
    KTA_CUDA(cudaEventCreateWithFlags(&t.join_hi, cudaEventDisableTiming));
    KTA_CUDA(cudaEventCreateWithFlags(&t.join, cudaEventDisableTiming));
  }
  *out = &t;
  return KTA_OK;
}

// Scratch for the chunked linear-attention kernels, one buffer per (device, CUDA stream): work on
// one stream runs in order, so a buffer is never in use by two calls at once, and calls on
// different streams never share one. It only grows (after that stream's earlier work is done).
kta_status workspace(size_t bytes, cudaStream_t st, void** out) {
  int dev = 0;
  KTA_CUDA(cudaGetDevice(&dev));
  DeviceRes& r = device_res(dev);
  std::lock_guard<std::mutex> lk(r.mu);
  DeviceRes::Buf& b = r.ws[st];
  if (b.bytes < bytes) {
    if (b.ptr) {
      KTA_CUDA(cudaStreamSynchronize(st));
      KTA_CUDA(cudaFree(b.ptr));
      b.ptr = nullptr;
      b.bytes = 0;
    }
    KTA_CUDA(cudaMalloc(&b.ptr, bytes));
    b.bytes = bytes;
  }
  *out = b.ptr;
  return KTA_OK;
}

// Raise a kernel's dynamic shared memory limit once per (kernel, device).
template <typename K>
kta_status set_smem_attr(K kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> done;
  int dev = 0;
  KTA_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  if (!done[key]) {
    KTA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)));
    done[key] = true;
  }
  return KTA_OK;
}

// ------------------------------------------------------------------------- tracing

struct TraceRec {
  const char* name;
  cudaEvent_t a, b;
};

struct TraceState {
  bool on = false;
  std::vector<TraceRec> recs;
};

TraceState& trace_state() {
  thread_local TraceState t;
  return t;
}

// Brackets one kernel launch with events on its stream while tracing is on.
struct TraceScope {
  TraceRec rec{nullptr, nullptr, nullptr};
  cudaStream_t st;
  TraceScope(const char* name, cudaStream_t s) : st(s) {
    TraceState& t = trace_state();
    if (!t.on) return;
    if (cudaEventCreate(&rec.a) != cudaSuccess || cudaEventCreate(&rec.b) != cudaSuccess) return;
    rec.name = name;
    cudaEventRecord(rec.a, st);
  }
  ~TraceScope() {
    if (!rec.name) return;
    cudaEventRecord(rec.b, st);
    trace_state().recs.push_back(rec);
  }
};

// ------------------------------------------------------------------------- softmax launches

struct WinGroup {
  int H = 0, W = 1, dil = 1;
  const void* k = nullptr;   // key buffer of the group (head coordinate = h - kh_off)
  const void* v = nullptr;
  long long k_ld = 0;        // row stride (elements)
  long long k_rows = 0;      // rows in the buffer
  int k_heads = 0;           // heads in one row of the buffer addressed by the map
  int kh_off = 0;
  int kb_frames = 0, kmod = 1;
  int span_mode = 0;         // 1: visible frames not adjacent in the buffer (a ring of W slots)
};

struct WinLaunch {
  int B = 0, P = 0, Fq = 0, f_base = 0, d = 0;
  kta_dtype dt = KTA_BF16;
  const void* q = nullptr;
  long long q_ld = 0;
  int q_rows_b = 0;
  void* o = nullptr;
  long long o_ld = 0;
  float scale = 1.f;
  float* lse = nullptr;      // optional row log-sum-exp output (bf16 tensor-core path only)
  WinGroup g[2];
};

template <int D>
kta_status launch_win_tc(const WinLaunch& L, cudaStream_t st) {
  const int Htot = L.g[0].H + L.g[1].H;
  CUtensorMap tq, tk0, tv0, tk1, tv1;
  kta_status s;
  if ((s = make_map(&tq, L.q, D, Htot, static_cast<long long>(L.B) * L.q_rows_b, L.q_ld))) return s;
  const WinGroup& g0 = L.g[0];
  const WinGroup& g1 = L.g[1].H > 0 ? L.g[1] : L.g[0];
  if ((s = make_map(&tk0, g0.k, D, g0.k_heads, g0.k_rows, g0.k_ld))) return s;
  if ((s = make_map(&tv0, g0.v, D, g0.k_heads, g0.k_rows, g0.k_ld))) return s;
  if ((s = make_map(&tk1, g1.k, D, g1.k_heads, g1.k_rows, g1.k_ld))) return s;
  if ((s = make_map(&tv1, g1.v, D, g1.k_heads, g1.k_rows, g1.k_ld))) return s;
  // 8-row boxes for the key tiles that span two frames of a dilated window (packed tiling)
  CUtensorMap tk0s = tk0, tv0s = tv0, tk1s = tk1, tv1s = tv1;
  const bool pk = L.P % 8 == 0;
  if (pk && (g0.dil > 1 || g0.span_mode) &&
      ((s = make_map(&tk0s, g0.k, D, g0.k_heads, g0.k_rows, g0.k_ld, 8)) ||
       (s = make_map(&tv0s, g0.v, D, g0.k_heads, g0.k_rows, g0.k_ld, 8))))
    return s;
  if (pk && (g1.dil > 1 || g1.span_mode) &&
      ((s = make_map(&tk1s, g1.k, D, g1.k_heads, g1.k_rows, g1.k_ld, 8)) ||
       (s = make_map(&tv1s, g1.v, D, g1.k_heads, g1.k_rows, g1.k_ld, 8))))
    return s;
  // output map (cols, heads, token of the frame, frame, sequence): a tile's rows past the frame
  // end lie outside the token extent P, so TMA stores of whole 32-row boxes never write them
  CUtensorMap to = tq;
  const bool o_tma = reinterpret_cast<uintptr_t>(L.o) % 16 == 0 && L.o_ld % 8 == 0;
  if (o_tma) {
    const cuuint64_t dO[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Htot),
                              static_cast<cuuint64_t>(L.P), static_cast<cuuint64_t>(L.Fq),
                              static_cast<cuuint64_t>(L.B)};
    const cuuint64_t sO[4] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L.o_ld) * 2,
                              static_cast<cuuint64_t>(L.P) * L.o_ld * 2,
                              static_cast<cuuint64_t>(L.q_rows_b) * L.o_ld * 2};
    const cuuint32_t bO[5] = {64, 1, 32, 1, 1};
    if ((s = make_map_nd(&to, L.o, 5, dO, sO, bO))) return s;
  }
  WinParams p{};
  p.o_tma = o_tma ? 1 : 0;
  p.B = L.B;
  p.P = L.P;
  p.Fq = L.Fq;
  p.f_base = L.f_base;
  p.n_qt = (L.P + 127) / 128;
  p.Htot = Htot;
  p.H0 = L.g[0].H;
  for (int i = 0; i < 2; ++i) {
    const WinGroup& g = L.g[i].H > 0 ? L.g[i] : L.g[0];
    p.W[i] = g.W;
    p.dil[i] = g.dil;
    p.kh_off[i] = g.kh_off;
    p.kb_frames[i] = g.kb_frames;
    p.kmod[i] = g.kmod;
    p.span_mode[i] = g.span_mode;
  }
  p.q_rows_b = L.q_rows_b;
  p.scale_log2 = L.scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(L.o);
  p.o_ld = L.o_ld;
  p.lse = L.lse;
  // one CTA per pair of query tiles of a (frame, head, sequence); one per tile when pairs would
  // leave SMs idle (a streaming step's single frame)
  const long long units = static_cast<long long>(L.Fq) * Htot * L.B;
  p.pair = units * ((p.n_qt + 1) / 2) >= 2 * 148 ? 2 : 1;
  const long long nblk = units * (p.pair == 2 ? (p.n_qt + 1) / 2 : p.n_qt);
  if (nblk <= 0) return KTA_OK;
  if (nblk > 0x7fffffffLL) return fail(KTA_ERR_UNSUPPORTED, "too many tiles (%lld)", nblk);
  const size_t smem = kta::win_smem_bytes<D>();
  // frames shorter than 120 keys (P a multiple of 8): a packed key tile may cross several frames
  const bool mf = pk && L.P < 120;
  auto kern = L.lse ? (mf ? kta::win_attn_tc_kernel<D, true, true> : kta::win_attn_tc_kernel<D, true, false>)
                    : (mf ? kta::win_attn_tc_kernel<D, false, true> : kta::win_attn_tc_kernel<D, false, false>);
  if ((s = set_smem_attr(kern, smem))) return s;
  {
    TraceScope ts("win_attn_tc", st);
    kern<<<static_cast<unsigned>(nblk), 384, smem, st>>>(tq, tk0, tv0, tk1, tv1, tk0s, tv0s, tk1s,
                                                         tv1s, to, p);
  }
  const cudaError_t le = cudaGetLastError();
  if (le != cudaSuccess) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, kta::win_attn_tc_kernel<D, false>);
    return fail(KTA_ERR_CUDA,
                "win_attn_tc launch failed: %s (grid %lld x 384, dyn smem %zu, regs %d, max threads "
                "%d, max dyn smem %d)",
                cudaGetErrorString(le), nblk, smem, fa.numRegs, fa.maxThreadsPerBlock,
                fa.maxDynamicSharedSizeBytes);
  }
  return KTA_OK;
}

kta_status launch_win_f32(const WinLaunch& L, cudaStream_t st) {
  kta::WinSimtParams p{};
  p.B = L.B;
  p.P = L.P;
  p.Fq = L.Fq;
  p.f_base = L.f_base;
  p.Htot = L.g[0].H + L.g[1].H;
  p.H0 = L.g[0].H;
  for (int i = 0; i < 2; ++i) {
    const WinGroup& g = L.g[i].H > 0 ? L.g[i] : L.g[0];
    p.W[i] = g.W;
    p.dil[i] = g.dil;
    p.kh_off[i] = g.kh_off;
    p.kb_frames[i] = g.kb_frames;
    p.kmod[i] = g.kmod;
    p.k_ld[i] = g.k_ld;
  }
  p.q_rows_b = L.q_rows_b;
  p.q_ld = L.q_ld;
  p.o_ld = L.o_ld;
  p.scale = L.scale;
  p.d = L.d;
  const WinGroup& g1 = L.g[1].H > 0 ? L.g[1] : L.g[0];
  dim3 grid((L.Fq * L.P + 3) / 4, p.Htot, L.B);
  if (grid.y > 65535 || grid.z > 65535) return fail(KTA_ERR_UNSUPPORTED, "too many heads/batches");
  {
    TraceScope ts("win_attn_f32", st);
    kta::win_attn_f32_kernel<<<grid, 128, 0, st>>>(
        static_cast<const float*>(L.q), static_cast<const float*>(L.g[0].k),
        static_cast<const float*>(L.g[0].v), static_cast<const float*>(g1.k),
        static_cast<const float*>(g1.v), static_cast<float*>(L.o), p);
  }
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

kta_status launch_win(const WinLaunch& L, cudaStream_t st) {
  if (L.g[0].H + L.g[1].H == 0 || L.Fq == 0) return KTA_OK;
  if (L.dt == KTA_F32) return launch_win_f32(L, st);
  if (L.d == 128) return launch_win_tc<128>(L, st);
  if (L.d == 64) return launch_win_tc<64>(L, st);
  return fail(KTA_ERR_UNSUPPORTED, "bf16 softmax branches need d in {64, 128} (got %d)", L.d);
}

// ------------------------------------------------------------------------- GLA launches

struct LinLaunch {
  int B = 0, N = 0, H = 0, d = 0, rows_b = 0, chunk = 64;
  kta_dtype dt = KTA_BF16;
  const void *q = nullptr, *k = nullptr, *v = nullptr;
  void* o = nullptr;
  long long ld = 0;
  const float* alpha = nullptr;
  const float* beta = nullptr;
  const float* S0 = nullptr;
  float* S_out = nullptr;
  float scale = 1.f;
  bool delta = false;
  bool erase_decayed = false;  // delta rule: decayed erase (GatedDeltaNet form)
  bool allow_segments = true;
  int cta_budget = 0;  // SMs the segment plan may fill (0: all of them)
  bool state_only = false;  // GLA: the end state only (state pass + carry fold, no outputs)
};

// Segment plan of the chunked GLA kernels: enough (segment, value slice, sequence-head) CTAs for
// one wave of three per SM, segments of whole chunks. ws_bytes is the workspace the state pass and
// the carry pass need (segment end states and total log2 decays; none for a single segment).
struct GlaPlan {
  int nseg = 1, seg_len = 0, slices = 1;
  bool tc = false;  // the tcgen05 kernel (d = 128, 64-token chunks)
  size_t ws_bytes = 0;
};

// SMs of the current device (148 on B200).
int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
      v = 148;
    n[dev] = v;
  }
  return n[dev];
}

template <int D, int C>
GlaPlan gla_plan(const LinLaunch& L) {
  using SM = kta::GlaSmem<D, C>;
  GlaPlan g;
  g.tc = D == kta::GT_D && C == kta::GT_C;
  g.slices = g.tc ? 1 : D / SM::BV;
  const long long base = static_cast<long long>(L.B) * L.H * g.slices;
  const int nchunks = (L.N + C - 1) / C;
  int nseg = 1;
  if (L.allow_segments) {
    // one wave: one CTA per SM (tcgen05 kernel) or three (warp-level kernel)
    const long long sms = L.cta_budget > 0 ? std::min(L.cta_budget, sm_count()) : sm_count();
    const long long slots = g.tc ? sms : 3LL * sms;
    const long long want = g.tc ? slots / base : (slots + base - 1) / base;
    nseg = static_cast<int>(std::min<long long>(std::max<long long>(want, 1), nchunks));
  }
  const int seg_chunks = (nchunks + nseg - 1) / nseg;
  g.seg_len = seg_chunks * C;
  g.nseg = (L.N + g.seg_len - 1) / g.seg_len;
  g.ws_bytes = g.nseg > 1 || L.state_only
                   ? static_cast<size_t>(L.B) * L.H * g.nseg * (size_t(D) * D + D) * 4
                   : 0;
  return g;
}

// The tcgen05 GLA kernels (d = 128, 64-token chunks): state pass, carry, output pass.
kta_status launch_gla_tc(const LinLaunch& L, const GlaPlan& g, void* ws, cudaStream_t st) {
  constexpr int D = kta::GT_D;
  if (static_cast<long long>(L.B) * L.H > 65535) return fail(KTA_ERR_UNSUPPORTED, "B*H > 65535");
  CUtensorMap tq, tk, tv, ta;
  const long long rows = static_cast<long long>(L.B) * L.rows_b;
  kta_status r;
  if ((r = make_map_box(&tq, L.q ? L.q : L.k, false, D, L.H, rows, L.ld, 64, kta::GT_C)) ||
      (r = make_map_box(&tk, L.k, false, D, L.H, rows, L.ld, 64, kta::GT_C)) ||
      (r = make_map_box(&tv, L.v, false, D, L.H, rows, L.ld, 64, kta::GT_C)) ||
      (r = make_map_box(&ta, L.alpha, true, D, L.H, rows, static_cast<long long>(L.H) * D, D,
                        kta::GT_C)))
    return r;
  // o: stores of whole 64-token chunks, [64 rows][128 values] unswizzled, per (head, sequence);
  // rows past N are outside the map
  CUtensorMap to = tq;
  if (!L.state_only) {
    const cuuint64_t dO[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L.H),
                              static_cast<cuuint64_t>(L.N), static_cast<cuuint64_t>(L.B)};
    const cuuint64_t sO[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L.ld) * 2,
                              static_cast<cuuint64_t>(L.rows_b) * L.ld * 2};
    const cuuint32_t bO[4] = {static_cast<cuuint32_t>(D), 1, static_cast<cuuint32_t>(kta::GT_C), 1};
    if ((r = make_map_nd(&to, L.o, 4, dO, sO, bO, CU_TENSOR_MAP_SWIZZLE_NONE))) return r;
  }
  kta::GlaTcParams p{};
  p.N = L.N;
  p.H = L.H;
  p.rows_b = L.rows_b;
  p.seg_len = g.seg_len;
  p.nseg = g.nseg;
  p.scale = L.scale;
  p.o = static_cast<__nv_bfloat16*>(L.o);
  p.ld = L.ld;
  p.S0 = L.S0;
  p.S_out = L.S_out;
  // A few segments: each output-pass CTA folds its predecessors' end states itself (reading at
  // most kta::GT_FOLD_MAX of them), which saves the carry launch.
  p.fold = g.nseg > 1 && g.nseg <= kta::GT_FOLD_MAX + 1 && !L.state_only ? 1 : 0;
  if (g.nseg > 1 || L.state_only) {
    p.ws_S = static_cast<float*>(ws);
    p.ws_L = p.ws_S + static_cast<size_t>(L.B) * L.H * g.nseg * D * D;
  }
  const size_t smem = sizeof(kta::GlaTcSmem) + 1024;
  if ((r = set_smem_attr(kta::gla_tc_kernel<false>, smem)) ||
      (r = set_smem_attr(kta::gla_tc_kernel<true>, smem)))
    return r;
  const dim3 grid(g.nseg, L.B * L.H);
  if (g.nseg > 1 || L.state_only) {
    {
      TraceScope ts("gla_tc_state", st);
      kta::gla_tc_kernel<false><<<grid, 384, smem, st>>>(tq, tk, tv, ta, to, p);
    }
    KTA_CUDA(cudaGetLastError());
    if (!p.fold) {
      kta::GlaParams pc{};  // the carry kernel folds the same workspace layout
      pc.S0 = L.S0;
      pc.nseg = g.nseg;
      pc.ws_S = p.ws_S;
      pc.ws_L = p.ws_L;
      pc.S_fold = L.state_only ? L.S_out : nullptr;
      {
        TraceScope ts("gla_carry", st);
        kta::gla_carry_kernel<D><<<dim3((D * D + 127) / 128, L.B * L.H), 128, 0, st>>>(pc);
      }
      KTA_CUDA(cudaGetLastError());
    }
  }
  if (L.state_only) return KTA_OK;
  {
    TraceScope ts("gla_tc_out", st);
    kta::gla_tc_kernel<true><<<grid, 384, smem, st>>>(tq, tk, tv, ta, to, p);
  }
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

// Launch the chunked GLA kernels of a plan with `ws` (ws_bytes of device memory, or null when
// the plan needs none) as the segment workspace.
template <int D, int C>
kta_status launch_gla_planned(const LinLaunch& L, const GlaPlan& g, void* ws, cudaStream_t st) {
  using SM = kta::GlaSmem<D, C>;
  if (g.tc) return launch_gla_tc(L, g, ws, st);
  if (static_cast<long long>(L.B) * L.H > 65535) return fail(KTA_ERR_UNSUPPORTED, "B*H > 65535");
  kta::GlaParams p{};
  p.q = static_cast<const __nv_bfloat16*>(L.q);
  p.k = static_cast<const __nv_bfloat16*>(L.k);
  p.v = static_cast<const __nv_bfloat16*>(L.v);
  p.alpha = L.alpha;
  p.o = static_cast<__nv_bfloat16*>(L.o);
  p.ld = L.ld;
  p.rows_b = L.rows_b;
  p.N = L.N;
  p.H = L.H;
  p.seg_len = g.seg_len;
  p.nseg = g.nseg;
  p.scale = L.scale;
  p.S0 = L.S0;
  p.S_out = L.state_only ? nullptr : L.S_out;
  p.S_fold = L.state_only ? L.S_out : nullptr;
  if (g.nseg > 1 || L.state_only) {
    // Every word the kernels read from the workspace is written earlier in the same call (the
    // state pass writes all segment states and decays, the carry pass rewrites them in place),
    // so nothing has to be cleared.
    p.ws_S = static_cast<float*>(ws);
    p.ws_L = p.ws_S + static_cast<size_t>(L.B) * L.H * g.nseg * D * D;
  }
  const size_t smem = sizeof(SM);
  kta_status sa;
  if ((sa = set_smem_attr(kta::gla_chunk_kernel<D, C, false>, smem)) ||
      (sa = set_smem_attr(kta::gla_chunk_kernel<D, C, true>, smem)))
    return sa;
  dim3 grid(g.nseg, g.slices, L.B * L.H);
  if (g.nseg > 1 || L.state_only) {
    {
      TraceScope ts("gla_chunk_state", st);
      kta::gla_chunk_kernel<D, C, false><<<grid, 128, smem, st>>>(p);
    }
    KTA_CUDA(cudaGetLastError());
    {
      TraceScope ts("gla_carry", st);
      kta::gla_carry_kernel<D><<<dim3((D * D + 127) / 128, L.B * L.H), 128, 0, st>>>(p);
    }
  }
  KTA_CUDA(cudaGetLastError());
  if (L.state_only) return KTA_OK;
  {
    TraceScope ts("gla_chunk_out", st);
    kta::gla_chunk_kernel<D, C, true><<<grid, 128, smem, st>>>(p);
  }
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

template <int D, int C>
kta_status launch_gla_chunk(const LinLaunch& L, cudaStream_t st) {
  const GlaPlan g = gla_plan<D, C>(L);
  void* ws = nullptr;
  if (g.ws_bytes) {
    kta_status s = workspace(g.ws_bytes, st, &ws);
    if (s) return s;
  }
  return launch_gla_planned<D, C>(L, g, ws, st);
}

template <int D>
kta_status launch_delta_chunk(const LinLaunch& L, cudaStream_t st) {
  constexpr int C = kta::DELTA_C, VG = 2, NST = 2;
  using PS = kta::DeltaPrepSmem<D>;
  using SS = kta::DeltaScanSmem<D, VG, NST>;
  const long long BH = static_cast<long long>(L.B) * L.H;
  if (BH > 65535) return fail(KTA_ERR_UNSUPPORTED, "B*H > 65535");
  const long long nch = (L.N + C - 1) / C;
  // workspace rows are addressed with 32-bit TMA coordinates
  if (BH * nch * D >= (1LL << 31)) return fail(KTA_ERR_UNSUPPORTED, "B*H*N too large for the delta workspace");
  kta::DeltaParams p{};
  p.q = static_cast<const __nv_bfloat16*>(L.q);
  p.k = static_cast<const __nv_bfloat16*>(L.k);
  p.v = static_cast<const __nv_bfloat16*>(L.v);
  p.alpha = L.alpha;
  p.beta = L.beta;
  p.o = static_cast<__nv_bfloat16*>(L.o);
  p.ld = L.ld;
  p.rows_b = L.rows_b;
  p.N = L.N;
  p.H = L.H;
  p.scale = L.scale;
  p.S0 = L.S0;
  p.S_out = L.S_out;
  p.nch = static_cast<int>(nch);
  p.erase_decayed = L.erase_decayed ? 1 : 0;
  const size_t units = static_cast<size_t>(BH) * nch;
  const size_t bytes = units * (static_cast<size_t>(C) * D * 2 * 2 + C * C * 2 + C * 4);
  void* ws = nullptr;
  kta_status s = workspace(bytes, st, &ws);
  if (s) return s;
  p.ws_W = static_cast<__nv_bfloat16*>(ws);
  p.ws_U = p.ws_W + units * C * D;
  p.ws_A = p.ws_U + units * D * C;
  p.ws_g = reinterpret_cast<float*>(p.ws_A + units * C * C);

  CUtensorMap tW, tQ, tK, tA, tU, tO;
  {
    const cuuint64_t dW[2] = {static_cast<cuuint64_t>(D), units * C};
    const cuuint64_t sW[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t bW[2] = {64, static_cast<cuuint32_t>(C)};
    if ((s = make_map_nd(&tW, p.ws_W, 2, dW, sW, bW))) return s;
    const cuuint64_t dA[2] = {static_cast<cuuint64_t>(C), units * C};
    const cuuint64_t sA[1] = {static_cast<cuuint64_t>(C) * 2};
    if ((s = make_map_nd(&tA, p.ws_A, 2, dA, sA, bW))) return s;
    const cuuint64_t dU[2] = {static_cast<cuuint64_t>(C), units * D};
    const cuuint32_t bU[2] = {64, static_cast<cuuint32_t>(SS::VB)};
    if ((s = make_map_nd(&tU, p.ws_U, 2, dU, sA, bU))) return s;
    // q, k: (key dim, head, row, sequence); rows past N read as zeros
    const cuuint64_t dQ[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L.H),
                              static_cast<cuuint64_t>(L.N), static_cast<cuuint64_t>(L.B)};
    const cuuint64_t sQ[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L.ld) * 2,
                              static_cast<cuuint64_t>(L.rows_b) * L.ld * 2};
    const cuuint32_t bQ[4] = {64, 1, static_cast<cuuint32_t>(C), 1};
    if ((s = make_map_nd(&tQ, L.q, 4, dQ, sQ, bQ))) return s;
    if ((s = make_map_nd(&tK, L.k, 4, dQ, sQ, bQ))) return s;
    // o: stores of [C tokens][VB value columns] tiles, unswizzled
    const cuuint32_t bO[4] = {static_cast<cuuint32_t>(SS::VB), 1, static_cast<cuuint32_t>(C), 1};
    if ((s = make_map_nd(&tO, L.o, 4, dQ, sQ, bO, CU_TENSOR_MAP_SWIZZLE_NONE))) return s;
  }
  const size_t smem_p = sizeof(PS), smem_s = kta::delta_scan_smem_bytes<D, VG, NST>();
  if ((s = set_smem_attr(kta::delta_prep_kernel<D>, smem_p))) return s;
  if ((s = set_smem_attr(kta::delta_scan_kernel<D, VG, NST>, smem_s))) return s;
  {
    TraceScope ts("delta_prep", st);
    kta::delta_prep_kernel<D><<<dim3(static_cast<unsigned>(nch), static_cast<unsigned>(BH)), 128,
                                smem_p, st>>>(p);
  }
  KTA_CUDA(cudaGetLastError());
  {
    TraceScope ts("delta_scan", st);
    kta::delta_scan_kernel<D, VG, NST>
        <<<dim3(D / SS::VB, static_cast<unsigned>(BH)), (SS::NCW + SS::NOW + 1) * 32, smem_s, st>>>(
            tW, tQ, tK, tA, tU, tO, p);
  }
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

template <int D>
kta_status launch_rec_f32(const LinLaunch& L, cudaStream_t st) {
  kta::RecF32Params p{};
  p.B = L.B;
  p.N = L.N;
  p.H = L.H;
  p.d = D;
  p.ld = L.ld;
  p.rows_b = L.rows_b;
  p.scale = L.scale;
  p.S0 = L.S0;
  p.S_out = L.S_out;
  p.erase_decayed = L.erase_decayed ? 1 : 0;
  if (L.B > 65535) return fail(KTA_ERR_UNSUPPORTED, "B > 65535");
  dim3 grid(L.H, L.B);
  TraceScope ts(L.delta ? "delta_rec_f32" : "gla_rec_f32", st);
  if (L.delta)
    kta::delta_rec_f32_kernel<D><<<grid, D, 0, st>>>(
        static_cast<const float*>(L.q), static_cast<const float*>(L.k),
        static_cast<const float*>(L.v), L.alpha, L.beta, static_cast<float*>(L.o), p);
  else
    kta::gla_rec_f32_kernel<D><<<grid, D, 0, st>>>(
        static_cast<const float*>(L.q), static_cast<const float*>(L.k),
        static_cast<const float*>(L.v), L.alpha, static_cast<float*>(L.o), p);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

kta_status launch_lin(const LinLaunch& L, cudaStream_t st) {
  if (L.H == 0 || L.N == 0) return KTA_OK;
  if (L.dt == KTA_F32) {
    if (L.d == 32) return launch_rec_f32<32>(L, st);
    if (L.d == 64) return launch_rec_f32<64>(L, st);
    return launch_rec_f32<128>(L, st);
  }
  if (L.delta) {
    if (L.d == 128) return launch_delta_chunk<128>(L, st);
    if (L.d == 64) return launch_delta_chunk<64>(L, st);
    return fail(KTA_ERR_UNSUPPORTED, "bf16 delta rule needs d in {64, 128} (got %d)", L.d);
  }
  if (L.d == 128) {
    if (L.chunk == 64) return launch_gla_chunk<128, 64>(L, st);
    if (L.chunk == 32) return launch_gla_chunk<128, 32>(L, st);
    return launch_gla_chunk<128, 16>(L, st);
  }
  if (L.d == 64) {
    if (L.chunk == 64) return launch_gla_chunk<64, 64>(L, st);
    if (L.chunk == 32) return launch_gla_chunk<64, 32>(L, st);
    return launch_gla_chunk<64, 16>(L, st);
  }
  return fail(KTA_ERR_UNSUPPORTED, "bf16 GLA needs d in {64, 128} (got %d)", L.d);
}

// ------------------------------------------------------------------------- validation

kta_status check_shape(const kta_shape& s) {
  if (s.B < 1 || s.F < 1 || s.P < 1) return fail(KTA_ERR_INVALID_ARG, "B, F, P must be >= 1");
  if (s.d != 32 && s.d != 64 && s.d != 128)
    return fail(KTA_ERR_UNSUPPORTED, "d must be 32, 64 or 128 (got %d)", s.d);
  if (s.dtype != KTA_BF16 && s.dtype != KTA_F32) return fail(KTA_ERR_INVALID_ARG, "bad dtype");
  const long long N = static_cast<long long>(s.F) * s.P;
  if (N >= (1LL << 31) || static_cast<long long>(s.B) * N >= (1LL << 31))
    return fail(KTA_ERR_UNSUPPORTED, "B*F*P must be < 2^31");
  return KTA_OK;
}

kta_status check_heads(int H, int ld_heads, const kta_shape& s) {
  if (H < 1 || ld_heads < H) return fail(KTA_ERR_INVALID_ARG, "need 1 <= H <= ld_heads");
  if ((static_cast<long long>(ld_heads) * s.d * elem_size(s.dtype)) % 16)
    return fail(KTA_ERR_ALIGNMENT, "row stride ld_heads*d*elem must be a multiple of 16 bytes");
  return KTA_OK;
}

kta_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return fail(KTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(p)) return fail(KTA_ERR_ALIGNMENT, "tensor pointer not 16-byte aligned");
  }
  return KTA_OK;
}

kta_status check_softmax_dtype(const kta_shape& s) {
  if (s.dtype == KTA_BF16 && s.d == 32)
    return fail(KTA_ERR_UNSUPPORTED, "bf16 softmax branches need d in {64, 128}");
  return KTA_OK;
}

WinLaunch seq_win_launch(const void* q, const void* k, const void* v, void* o, const kta_shape& s,
                         int ld_heads, float scale) {
  WinLaunch L;
  L.B = s.B;
  L.P = s.P;
  L.Fq = s.F;
  L.f_base = 0;
  L.d = s.d;
  L.dt = s.dtype;
  L.q = q;
  L.q_ld = static_cast<long long>(ld_heads) * s.d;
  L.q_rows_b = s.F * s.P;
  L.o = o;
  L.o_ld = L.q_ld;
  L.scale = scale;
  return L;
}

WinGroup seq_group(const void* k, const void* v, const kta_shape& s, int H, int Htot, int ld_heads,
                   int W, int dil) {
  WinGroup g;
  g.H = H;
  g.W = W;
  g.dil = dil;
  g.k = k;
  g.v = v;
  g.k_ld = static_cast<long long>(ld_heads) * s.d;
  g.k_rows = static_cast<long long>(s.B) * s.F * s.P;
  g.k_heads = Htot;
  g.kh_off = 0;
  g.kb_frames = s.F;
  g.kmod = s.F;
  return g;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

// =========================================================================== C ABI

extern "C" {

const char* kta_status_str(kta_status s) {
  switch (s) {
    case KTA_OK: return "KTA_OK";
    case KTA_ERR_INVALID_ARG: return "KTA_ERR_INVALID_ARG";
    case KTA_ERR_UNSUPPORTED: return "KTA_ERR_UNSUPPORTED";
    case KTA_ERR_ALIGNMENT: return "KTA_ERR_ALIGNMENT";
    case KTA_ERR_CUDA: return "KTA_ERR_CUDA";
    case KTA_ERR_TIMEOUT: return "KTA_ERR_TIMEOUT";
    case KTA_ERR_STATE: return "KTA_ERR_STATE";
  }
  return "KTA_ERR_UNKNOWN";
}

const char* kta_last_error(void) { return g_last_error.c_str(); }

int kta_version(void) { return KTA_VERSION; }

kta_status kta_swa_fwd(const void* q, const void* k, const void* v, void* o, kta_shape s, int H,
                       int ld_heads, int W, float scale, void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) || (r = check_ptrs({q, k, v, o})) ||
      (r = check_softmax_dtype(s)))
    return r;
  if (W < 1) return fail(KTA_ERR_INVALID_ARG, "W must be >= 1");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be > 0");
  WinLaunch L = seq_win_launch(q, k, v, o, s, ld_heads, scale);
  L.g[0] = seq_group(k, v, s, H, H, ld_heads, W, 1);
  return launch_win(L, as_stream(stream));
}

kta_status kta_dswa_fwd(const void* q, const void* k, const void* v, void* o, kta_shape s, int H,
                        int ld_heads, int W, int dil, float scale, void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) || (r = check_ptrs({q, k, v, o})) ||
      (r = check_softmax_dtype(s)))
    return r;
  if (W < 1 || dil < 1) return fail(KTA_ERR_INVALID_ARG, "W and dil must be >= 1");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be > 0");
  WinLaunch L = seq_win_launch(q, k, v, o, s, ld_heads, scale);
  L.g[0] = seq_group(k, v, s, H, H, ld_heads, W, dil);
  return launch_win(L, as_stream(stream));
}

static kta_status lin_common(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, float* S_out, void* o,
                             kta_shape s, int H, int ld_heads, int chunk, float scale, bool delta,
                             bool erase_decayed, void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) || (r = check_ptrs({q, k, v, o})))
    return r;
  if (!alpha || (delta && !beta)) return fail(KTA_ERR_INVALID_ARG, "null gate pointer");
  if (!aligned16(alpha) || (S0 && !aligned16(S0)) || (S_out && !aligned16(S_out)))
    return fail(KTA_ERR_ALIGNMENT, "gate / state pointers must be 16-byte aligned");
  if (chunk != 16 && chunk != 32 && chunk != 64)
    return fail(KTA_ERR_INVALID_ARG, "chunk must be 16, 32 or 64");
  if (!std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be finite");
  LinLaunch L;
  L.B = s.B;
  L.N = s.F * s.P;
  L.H = H;
  L.d = s.d;
  L.rows_b = L.N;
  L.chunk = chunk;
  L.dt = s.dtype;
  L.q = q;
  L.k = k;
  L.v = v;
  L.o = o;
  L.ld = static_cast<long long>(ld_heads) * s.d;
  L.alpha = alpha;
  L.beta = beta;
  L.S0 = S0;
  L.S_out = S_out;
  L.scale = scale;
  L.delta = delta;
  L.erase_decayed = erase_decayed;
  return launch_lin(L, as_stream(stream));
}

kta_status kta_gla_chunk_fwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* S0, float* S_out, void* o, kta_shape s, int H,
                             int ld_heads, int chunk, float scale, void* stream) {
  return lin_common(q, k, v, alpha, nullptr, S0, S_out, o, s, H, ld_heads, chunk, scale, false,
                    false, stream);
}

kta_status kta_gla_chunk_state(const void* k, const void* v, const float* alpha, const float* S0,
                               float* S_out, kta_shape s, int H, int ld_heads, int chunk,
                               void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) || (r = check_ptrs({k, v})))
    return r;
  if (s.dtype != KTA_BF16) return fail(KTA_ERR_UNSUPPORTED, "the end-state pass is built for bf16 only");
  if (!alpha || !S_out) return fail(KTA_ERR_INVALID_ARG, "null alpha or S_out");
  if (!aligned16(alpha) || (S0 && !aligned16(S0)) || !aligned16(S_out))
    return fail(KTA_ERR_ALIGNMENT, "gate / state pointers must be 16-byte aligned");
  if (chunk != 16 && chunk != 32 && chunk != 64)
    return fail(KTA_ERR_INVALID_ARG, "chunk must be 16, 32 or 64");
  LinLaunch L;
  L.B = s.B;
  L.N = s.F * s.P;
  L.H = H;
  L.d = s.d;
  L.rows_b = L.N;
  L.chunk = chunk;
  L.dt = s.dtype;
  L.k = k;
  L.v = v;
  L.ld = static_cast<long long>(ld_heads) * s.d;
  L.alpha = alpha;
  L.S0 = S0;
  L.S_out = S_out;
  L.state_only = true;
  return launch_lin(L, as_stream(stream));
}

kta_status kta_gla_delta_fwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, float* S_out, void* o,
                             kta_shape s, int H, int ld_heads, int chunk, float scale,
                             void* stream) {
  return lin_common(q, k, v, alpha, beta, S0, S_out, o, s, H, ld_heads, chunk, scale, true, false,
                    stream);
}

kta_status kta_gla_gdn_fwd(const void* q, const void* k, const void* v, const float* alpha,
                           const float* beta, const float* S0, float* S_out, void* o,
                           kta_shape s, int H, int ld_heads, int chunk, float scale,
                           void* stream) {
  return lin_common(q, k, v, alpha, beta, S0, S_out, o, s, H, ld_heads, chunk, scale, true, true,
                    stream);
}

static kta_status check_cfg(const kta_hybrid_cfg* c) {
  if (!c) return fail(KTA_ERR_INVALID_ARG, "null cfg");
  kta_status r;
  if ((r = check_shape(c->s))) return r;
  if (c->n_swa < 0 || c->n_dswa < 0 || c->n_gla < 0 || c->n_swa + c->n_dswa + c->n_gla < 1)
    return fail(KTA_ERR_INVALID_ARG, "head counts must be >= 0 with at least one head");
  if (c->n_swa + c->n_dswa > 0) {
    if ((r = check_softmax_dtype(c->s))) return r;
    if ((c->n_swa && c->W_swa < 1) || (c->n_dswa && (c->W_dswa < 1 || c->dil < 1)))
      return fail(KTA_ERR_INVALID_ARG, "windows and dilation must be >= 1");
    if (!(c->scale_softmax > 0.f) || !std::isfinite(c->scale_softmax))
      return fail(KTA_ERR_INVALID_ARG, "scale_softmax must be > 0");
  }
  if (c->n_gla > 0) {
    if (c->gla_delta < 0 || c->gla_delta > 2)
      return fail(KTA_ERR_INVALID_ARG, "gla_delta must be 0, 1 or 2");
    if (c->chunk != 16 && c->chunk != 32 && c->chunk != 64)
      return fail(KTA_ERR_INVALID_ARG, "chunk must be 16, 32 or 64");
    if (!std::isfinite(c->scale_gla)) return fail(KTA_ERR_INVALID_ARG, "scale_gla must be finite");
  }
  const int H = c->n_swa + c->n_dswa + c->n_gla;
  return check_heads(H, H, c->s);
}

// Softmax heads and linear heads of one hybrid call, forked from `st` onto the thread's two
// streams and joined back into it. The softmax stream has the higher priority, so the block
// scheduler dispatches every pending softmax CTA before a linear-head CTA: the linear heads fill
// the SMs that the softmax launch leaves free (its last wave) instead of taking SMs from it.
kta_status run_forked(const WinLaunch& W, const LinLaunch& L, cudaStream_t st) {
  ThreadStreams* ts = nullptr;
  kta_status r;
  if ((r = thread_streams(&ts))) return r;
  KTA_CUDA(cudaEventRecord(ts->fork, st));
  KTA_CUDA(cudaStreamWaitEvent(ts->hi, ts->fork, 0));
  KTA_CUDA(cudaStreamWaitEvent(ts->side, ts->fork, 0));
  const kta_status r_win = launch_win(W, ts->hi);
  const kta_status r_lin = launch_lin(L, ts->side);
  KTA_CUDA(cudaEventRecord(ts->join_hi, ts->hi));
  KTA_CUDA(cudaEventRecord(ts->join, ts->side));
  KTA_CUDA(cudaStreamWaitEvent(st, ts->join_hi, 0));
  KTA_CUDA(cudaStreamWaitEvent(st, ts->join, 0));
  return r_win ? r_win : r_lin;
}

static kta_status hybrid_common(const kta_hybrid_cfg* cfg, int f0, const void* q, const void* k,
                                const void* v, const float* alpha, const float* beta,
                                const float* S0, float* S_out, void* o, void* stream) {
  kta_status r;
  if ((r = check_cfg(cfg)) || (r = check_ptrs({q, k, v, o}))) return r;
  const kta_shape& s = cfg->s;
  if (f0 < 0 || f0 >= s.F) return fail(KTA_ERR_INVALID_ARG, "need 0 <= f0 < F (got f0 = %d)", f0);
  if (f0 > 0 && s.B != 1)
    return fail(KTA_ERR_UNSUPPORTED, "a query-frame offset f0 > 0 needs B == 1");
  const int H = cfg->n_swa + cfg->n_dswa + cfg->n_gla;
  if (cfg->n_gla > 0) {
    if (!alpha || (cfg->gla_delta && !beta)) return fail(KTA_ERR_INVALID_ARG, "null gate pointer");
    if (!aligned16(alpha)) return fail(KTA_ERR_ALIGNMENT, "alpha not 16-byte aligned");
  }
  const size_t es = elem_size(s.dtype);
  const long long ld = static_cast<long long>(H) * s.d;
  cudaStream_t st = as_stream(stream);

  WinLaunch W = seq_win_launch(q, k, v, o, s, H, cfg->scale_softmax);
  W.Fq = s.F - f0;  // query frames f0 .. F-1 of the key / value frames
  W.f_base = f0;
  W.q_rows_b = W.Fq * s.P;
  W.g[0] = seq_group(k, v, s, cfg->n_swa, cfg->n_swa + cfg->n_dswa, H, cfg->W_swa, 1);
  W.g[1] = seq_group(k, v, s, cfg->n_dswa, cfg->n_swa + cfg->n_dswa, H, cfg->W_dswa, cfg->dil);
  if (cfg->n_swa == 0) {  // DSWA heads only: make them group 0
    W.g[0] = W.g[1];
    W.g[1] = WinGroup();
  }

  LinLaunch L;
  L.B = s.B;
  L.N = (s.F - f0) * s.P;
  L.H = cfg->n_gla;
  L.d = s.d;
  L.rows_b = L.N;
  L.chunk = cfg->chunk;
  L.dt = s.dtype;
  const size_t hoff = static_cast<size_t>(cfg->n_swa + cfg->n_dswa) * s.d * es;
  L.q = static_cast<const char*>(q) + hoff;
  const size_t koff = static_cast<size_t>(f0) * s.P * ld * es;  // the query frames' keys
  L.k = static_cast<const char*>(k) + koff + hoff;
  L.v = static_cast<const char*>(v) + koff + hoff;
  L.o = static_cast<char*>(o) + hoff;
  L.ld = ld;
  L.alpha = alpha;
  L.beta = beta;
  L.scale = cfg->scale_gla;
  L.S0 = S0;
  L.S_out = S_out;
  L.delta = cfg->gla_delta != 0;
  L.erase_decayed = cfg->gla_delta == 2;

  const bool both = (cfg->n_swa + cfg->n_dswa) > 0 && cfg->n_gla > 0;
  if (!both) {
    if ((r = launch_win(W, st))) return r;
    return launch_lin(L, st);
  }
  return run_forked(W, L, st);
}

kta_status kta_hybrid_fwd(const kta_hybrid_cfg* cfg, const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta, void* o, void* stream) {
  return hybrid_common(cfg, 0, q, k, v, alpha, beta, nullptr, nullptr, o, stream);
}

kta_status kta_hybrid_fwd_window(const kta_hybrid_cfg* cfg, int f0, const void* q, const void* k,
                                 const void* v, const float* alpha, const float* beta,
                                 const float* S0, float* S_out, void* o, void* stream) {
  if ((S0 && !aligned16(S0)) || (S_out && !aligned16(S_out)))
    return fail(KTA_ERR_ALIGNMENT, "S0 / S_out not 16-byte aligned");
  return hybrid_common(cfg, f0, q, k, v, alpha, beta, S0, S_out, o, stream);
}

kta_status kta_gla_transition(const float* alpha, float* T, int B, int N, int H, int d,
                              void* stream) {
  if (!alpha || !T) return fail(KTA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || H <= 0 || N < 0) return fail(KTA_ERR_INVALID_ARG, "need B, H > 0 and N >= 0");
  if (static_cast<long long>(B) * H > 0x7fffffffLL)
    return fail(KTA_ERR_UNSUPPORTED, "too many sequences x heads");
  if (!aligned16(alpha) || !aligned16(T)) return fail(KTA_ERR_ALIGNMENT, "pointers not 16-byte aligned");
  if (d != 128 && d != 64 && d != 32) return fail(KTA_ERR_UNSUPPORTED, "d must be 32, 64 or 128 (got %d)", d);
  cudaStream_t st = as_stream(stream);
  // token blocks per (sequence, head): enough CTAs for every SM, at least ~32 tokens each
  const int G = static_cast<int>(std::max(1LL, std::min<long long>(
      (2LL * sm_count() + B * H - 1) / (static_cast<long long>(B) * H), (N + 31) / 32)));
  void* part = nullptr;
  kta_status r;
  if ((r = workspace(static_cast<size_t>(B) * H * G * d * sizeof(float), st, &part))) return r;
  const dim3 grid(static_cast<unsigned>(B * H), static_cast<unsigned>(G));
  float* pf = static_cast<float*>(part);
  {
    TraceScope ts("gla_transition", st);
    if (d == 128) {
      kta::gla_transition_part_kernel<128><<<grid, 512, 0, st>>>(alpha, pf, N, H, G);
      kta::gla_transition_finish_kernel<128><<<grid.x, 256, 0, st>>>(pf, T, G);
    } else if (d == 64) {
      kta::gla_transition_part_kernel<64><<<grid, 256, 0, st>>>(alpha, pf, N, H, G);
      kta::gla_transition_finish_kernel<64><<<grid.x, 256, 0, st>>>(pf, T, G);
    } else {
      kta::gla_transition_part_kernel<32><<<grid, 128, 0, st>>>(alpha, pf, N, H, G);
      kta::gla_transition_finish_kernel<32><<<grid.x, 256, 0, st>>>(pf, T, G);
    }
  }
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

kta_status kta_state_affine(const float* A, const float* X, const float* E, float* Y, int n, int d,
                            void* stream) {
  if (!A || !X || !Y) return fail(KTA_ERR_INVALID_ARG, "null pointer");
  if (n < 1 || d < 1 || d > 4096) return fail(KTA_ERR_INVALID_ARG, "need n >= 1 and 1 <= d <= 4096");
  if (Y == A || Y == X) return fail(KTA_ERR_INVALID_ARG, "Y must not alias A or X");
  cudaStream_t st = as_stream(stream);
  const dim3 grid((d + 31) / 32, (d + 31) / 32, n);
  TraceScope ts("state_affine", st);
  kta::state_affine_kernel<<<grid, dim3(32, 8), 0, st>>>(A, X, E, Y, d);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

// --------------------------------------------------------------------------- streaming

}  // extern "C"

struct kta_stream_s {
  kta_hybrid_cfg cfg;
  int device = 0;
  int64_t frame = 0;
  int R_swa = 0, R_dswa = 0;    // ring slots: a frame's keys and values go to slot f % R
  size_t es = 2;
  char* arena = nullptr;        // [header | swa k | swa v | dswa k | dswa v | state 0 | state 1]
  size_t arena_bytes = 0;
  size_t off_swa_k = 0, off_swa_v = 0, off_dswa_k = 0, off_dswa_v = 0, off_state[2] = {0, 0};
  size_t ring_swa_bytes = 0, ring_dswa_bytes = 0, state_bytes = 0;
  int cur = 0;
  uint32_t magic = 0x6b746131u;
};

namespace {

constexpr size_t kHeader = 256;

struct BlobHeader {
  uint32_t magic;
  uint32_t cur;
  int64_t frame;
  int32_t B, P, d, n_swa, n_dswa, n_gla, W_swa, W_dswa, dil, dtype, gla_delta;
};

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

std::mutex g_streams_mu;
std::map<const kta_stream_s*, bool> g_streams;  // live handles

kta_status valid_stream(kta_stream_t st) {
  std::lock_guard<std::mutex> lk(g_streams_mu);
  if (!st || !g_streams.count(st)) return fail(KTA_ERR_STATE, "invalid or destroyed stream handle");
  return KTA_OK;
}

// One frame's keys and values into the rings: up to four row-block copies (SWA k and v, DSWA k
// and v) in one launch, 16 bytes per thread and step. A copy takes heads [h0, h0+nh) of a frame
// ([B][P][H][d]) into ring slot `slot` ([B][RR][P][nh][d]).
struct RingCopy {
  const char* src = nullptr;
  char* dst = nullptr;
  long long src_seq = 0, dst_seq = 0;  // bytes between sequences
  int src_row = 0, dst_row = 0;        // bytes between rows
  int chunks = 0;                      // 16-byte pieces per row (nh * d * element size / 16)
};
constexpr int kRingRows = 16;  // rows per block
struct RingPutParams {
  RingCopy c[4];
  int B = 0, P = 0;
};

// Block (x, y): rows [16 x, 16 x + 16) of the frame batch (row = b * P + token) for copy y; 32-bit
// index arithmetic only.
__global__ void __launch_bounds__(256) ring_put_kernel(const RingPutParams p) {
  const RingCopy& c = p.c[blockIdx.y];
  const int rows = p.B * p.P;
  const int r0 = static_cast<int>(blockIdx.x) * kRingRows;
  const int n = min(kRingRows, rows - r0) * c.chunks;
  // eight pieces per thread in flight at once: all loads, then all stores
  for (int i0 = 0; i0 < n; i0 += 8 * 256) {
    uint4 v[8];
    long long dst[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * 256 + threadIdx.x;
      dst[u] = -1;
      if (i < n) {
        const int rr = i / c.chunks, ch = i - rr * c.chunks;
        const int r = r0 + rr, b = r / p.P, row = r - b * p.P;
        v[u] = *reinterpret_cast<const uint4*>(c.src + b * c.src_seq +
                                               static_cast<long long>(row) * c.src_row + ch * 16);
        dst[u] = b * c.dst_seq + static_cast<long long>(row) * c.dst_row + ch * 16;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (dst[u] >= 0) *reinterpret_cast<uint4*>(c.dst + dst[u]) = v[u];
  }
}

RingCopy ring_copy(const kta_stream_s* s, const void* src, char* ring, int h0, int nh, int RR,
                   int slot) {
  const kta_shape& sh = s->cfg.s;
  const int H = s->cfg.n_swa + s->cfg.n_dswa + s->cfg.n_gla;
  RingCopy c;
  c.src_row = static_cast<int>(static_cast<size_t>(H) * sh.d * s->es);
  c.dst_row = static_cast<int>(static_cast<size_t>(nh) * sh.d * s->es);
  c.src = static_cast<const char*>(src) + static_cast<size_t>(h0) * sh.d * s->es;
  c.dst = ring + static_cast<size_t>(slot) * sh.P * c.dst_row;
  c.src_seq = static_cast<long long>(sh.P) * c.src_row;
  c.dst_seq = static_cast<long long>(RR) * sh.P * c.dst_row;
  c.chunks = c.dst_row / 16;
  return c;
}

kta_status ring_put(const RingPutParams& rp, int ncopies, cudaStream_t st) {
  if (ncopies == 0) return KTA_OK;
  const long long rows = static_cast<long long>(rp.B) * rp.P;
  if (rows * 1024 > 0x7fffffffLL) return fail(KTA_ERR_UNSUPPORTED, "too many rows per frame batch");
  TraceScope ts("ring_put", st);
  const unsigned gx = static_cast<unsigned>((rows + kRingRows - 1) / kRingRows);
  ring_put_kernel<<<dim3(gx, static_cast<unsigned>(ncopies)), 256, 0, st>>>(rp);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

// ------------------------------------------------------------------------- backward (fp32)

kta_status bwd_f32_only(const kta_shape& s) {
  if (s.dtype != KTA_F32)
    return fail(KTA_ERR_UNSUPPORTED, "the backward is built for KTA_F32 (fp32 reference) only");
  return KTA_OK;
}

kta_status softmax_bwd_common(const void* q, const void* k, const void* v,
                                     const void* dout, void* dq, void* dk, void* dv, kta_shape s,
                                     int H, int ld_heads, int W, int dil, float scale,
                                     void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = bwd_f32_only(s)) || (r = check_heads(H, ld_heads, s)) ||
      (r = check_ptrs({q, k, v, dout, dq, dk, dv})))
    return r;
  if (W < 1 || dil < 1) return fail(KTA_ERR_INVALID_ARG, "W and dil must be >= 1");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be > 0");
  if (s.B > 65535 || H > 65535) return fail(KTA_ERR_UNSUPPORTED, "B and H must be <= 65535");
  cudaStream_t st = as_stream(stream);
  const long long N = static_cast<long long>(s.F) * s.P, ld = static_cast<long long>(ld_heads) * s.d;
  void* ws = nullptr;
  if ((r = workspace(static_cast<size_t>(3) * s.B * H * N * sizeof(float), st, &ws))) return r;
  kta::SoftmaxBwdParams p{};
  p.B = s.B;
  p.N = static_cast<int>(N);
  p.P = s.P;
  p.H = H;
  p.d = s.d;
  p.W = W;
  p.dil = dil;
  p.ld = ld;
  p.scale = scale;
  p.stats = static_cast<float*>(ws);
  const dim3 grid(static_cast<unsigned>(
                      s.F * ((s.P + kta::SB_ROWS_CTA - 1) / kta::SB_ROWS_CTA)), H, s.B);
  const float *fq = static_cast<const float*>(q), *fk = static_cast<const float*>(k),
              *fv = static_cast<const float*>(v), *fdo = static_cast<const float*>(dout);
  float *fdq = static_cast<float*>(dq), *fdk = static_cast<float*>(dk),
        *fdv = static_cast<float*>(dv);
  {
    TraceScope ts("softmax_bwd_q_f32", st);
    if (s.d == 128)
      kta::softmax_bwd_q_f32_kernel<4><<<grid, 128, 0, st>>>(fq, fk, fv, fdo, fdq, p);
    else if (s.d == 64)
      kta::softmax_bwd_q_f32_kernel<2><<<grid, 128, 0, st>>>(fq, fk, fv, fdo, fdq, p);
    else
      kta::softmax_bwd_q_f32_kernel<1><<<grid, 128, 0, st>>>(fq, fk, fv, fdo, fdq, p);
    KTA_CUDA(cudaGetLastError());
  }
  TraceScope ts("softmax_bwd_kv_f32", st);
  if (s.d == 128)
    kta::softmax_bwd_kv_f32_kernel<4><<<grid, 128, 0, st>>>(fq, fk, fv, fdo, fdk, fdv, p);
  else if (s.d == 64)
    kta::softmax_bwd_kv_f32_kernel<2><<<grid, 128, 0, st>>>(fq, fk, fv, fdo, fdk, fdv, p);
  else
    kta::softmax_bwd_kv_f32_kernel<1><<<grid, 128, 0, st>>>(fq, fk, fv, fdo, fdk, fdv, p);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

template <int D>
kta_status launch_lin_bwd(kta::LinBwdParams p, int B, cudaStream_t st) {
  const long long bh = static_cast<long long>(B) * p.H;
  if (p.delta) {
    // The delta rule's segment carry would need dense d x d transitions: one CTA per
    // (sequence, head), states checkpointed every BWD_CK tokens and recomputed per chunk.
    p.nck = (p.N + kta::BWD_CK - 1) / kta::BWD_CK;
    void* ws = nullptr;
    kta_status r = workspace(static_cast<size_t>(kta::lin_bwd_ws_floats<D>(p.nck)) * bh *
                                 sizeof(float), st, &ws);
    if (r) return r;
    p.ws = static_cast<float*>(ws);
    const size_t smem = (3 * static_cast<size_t>(D) * (D + 1) + 8 * D) * sizeof(float);
    if ((r = set_smem_attr(kta::delta_bwd_f32_kernel<D>, smem))) return r;
    TraceScope ts("delta_bwd_f32", st);
    kta::delta_bwd_f32_kernel<D><<<dim3(p.H, B), D, smem, st>>>(p);
    KTA_CUDA(cudaGetLastError());
    return KTA_OK;
  }
  // Vector GLA: segments of the sequence for about three CTAs per SM; a forward sweep and a
  // reverse sweep per segment from the carried state and adjoint.
  int nseg = 1;
  long long seg_len = p.N;
  if (bh < 3 * 148) {
    const long long want = std::max<long long>(1, 3 * 148 / bh);
    seg_len = ((p.N + want - 1) / want + kta::BWD_CK - 1) / kta::BWD_CK * kta::BWD_CK;
    nseg = static_cast<int>((p.N + seg_len - 1) / seg_len);
  }
  if (nseg == 1) seg_len = p.N;
  p.nseg = nseg;
  p.seg_len = static_cast<int>(seg_len);
  const long long bhs = bh * nseg;
  const long long sum_per = 2LL * D * D + 2 * D;
  const long long tokD = bh * p.N * D;
  // floats: ybuf, then (nseg > 1) summaries, Sin, Gin; doubles: xbuf, ytot
  const long long n_f = tokD + (nseg > 1 ? bhs * (sum_per + 2LL * D * D) : 0);
  const long long n_d = tokD + bhs * D;
  void* ws = nullptr;
  kta_status r = workspace(static_cast<size_t>(n_d) * 8 + static_cast<size_t>(n_f) * 4, st, &ws);
  if (r) return r;
  double* xbuf = static_cast<double*>(ws);
  double* ytot = xbuf + tokD;
  float* ybuf = reinterpret_cast<float*>(ytot + bhs * D);
  p.Sin = p.Gin = nullptr;
  if (nseg > 1) {
    float* sum = ybuf + tokD;
    float* Sin = sum + bhs * sum_per;
    float* Gin = Sin + bhs * D * D;
    {
      TraceScope ts("gla_bwd_summary_f32", st);
      kta::gla_bwd_summary_kernel<D><<<dim3(nseg, p.H, B), D, 0, st>>>(p, sum);
      KTA_CUDA(cudaGetLastError());
    }
    {
      TraceScope ts("gla_bwd_carry_f32", st);
      const long long n = static_cast<long long>(p.H) * D * D;
      kta::gla_bwd_carry_kernel<D><<<dim3(static_cast<unsigned>((n + 255) / 256), B), 256, 0, st>>>(
          p, sum, Sin, Gin);
      KTA_CUDA(cudaGetLastError());
    }
    p.Sin = Sin;
    p.Gin = Gin;
  }
  const size_t smem = (static_cast<size_t>(D) * (D + 1) + 5 * D) * sizeof(float);
  if ((r = set_smem_attr(kta::gla_bwd_sweep_kernel<D>, smem))) return r;
  {
    TraceScope ts("gla_bwd_f32", st);
    kta::gla_bwd_sweep_kernel<D><<<dim3(p.H, B, nseg), D, smem, st>>>(p, ybuf, xbuf, ytot);
    KTA_CUDA(cudaGetLastError());
  }
  TraceScope ts("gla_bwd_dalpha_f32", st);
  const long long n = static_cast<long long>(p.N) * p.H * D;
  kta::gla_bwd_dalpha_kernel<D><<<dim3(static_cast<unsigned>((n + 255) / 256), B), 256, 0, st>>>(
      p, xbuf, ytot);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

kta_status lin_bwd_common(const void* q, const void* k, const void* v, const float* alpha,
                                 const float* beta, const float* S0, const void* dout, void* dq,
                                 void* dk, void* dv, float* dalpha, float* dbeta, float* dS0,
                                 kta_shape s, int H, int ld_heads, float scale, bool delta,
                                 bool erase_decayed, void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = bwd_f32_only(s)) || (r = check_heads(H, ld_heads, s)) ||
      (r = check_ptrs({q, k, v, dout, dq, dk, dv})))
    return r;
  if (!alpha || !dalpha || (delta && (!beta || !dbeta)))
    return fail(KTA_ERR_INVALID_ARG, "null gate or gate-gradient pointer");
  if (!std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be finite");
  if (s.B > 65535 || H > 65535) return fail(KTA_ERR_UNSUPPORTED, "B and H must be <= 65535");
  const long long N = static_cast<long long>(s.F) * s.P;
  kta::LinBwdParams p{};
  p.q = static_cast<const float*>(q);
  p.k = static_cast<const float*>(k);
  p.v = static_cast<const float*>(v);
  p.alpha = alpha;
  p.beta = beta;
  p.S0 = S0;
  p.dout = static_cast<const float*>(dout);
  p.dq = static_cast<float*>(dq);
  p.dk = static_cast<float*>(dk);
  p.dv = static_cast<float*>(dv);
  p.dalpha = dalpha;
  p.dbeta = dbeta;
  p.dS0 = dS0;
  p.ld = static_cast<long long>(ld_heads) * s.d;
  p.rows_b = static_cast<int>(N);
  p.N = static_cast<int>(N);
  p.H = H;
  p.scale = scale;
  p.delta = delta ? 1 : 0;
  p.erase_decayed = erase_decayed ? 1 : 0;
  if (N == 0) return KTA_OK;
  cudaStream_t st = as_stream(stream);
  if (s.d == 32) return launch_lin_bwd<32>(p, s.B, st);
  if (s.d == 64) return launch_lin_bwd<64>(p, s.B, st);
  return launch_lin_bwd<128>(p, s.B, st);
}


template <int D>
kta_status launch_win_bwd_tc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             const kta_shape& s, int H, int ld_heads, int W, int dil, float scale,
                             cudaStream_t st) {
  const long long N = static_cast<long long>(s.F) * s.P;
  const long long rows = static_cast<long long>(s.B) * N;
  const long long ld = static_cast<long long>(ld_heads) * D;
  void* ws = nullptr;
  kta_status r;
  if ((r = workspace(static_cast<size_t>(s.B) * H * N * sizeof(float), st, &ws))) return r;
  float* Dt = static_cast<float*>(ws);
  {
    TraceScope ts("row_dot", st);
    const long long warps = rows * H;
    kta::row_dot_kernel<D><<<static_cast<unsigned>((warps + 7) / 8), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), Dt, rows,
        static_cast<int>(N), H, ld);
    KTA_CUDA(cudaGetLastError());
  }
  CUtensorMap tq, tdo, tk, tv;
  if ((r = make_map(&tq, q, D, H, rows, ld)) || (r = make_map(&tdo, dout, D, H, rows, ld)) ||
      (r = make_map(&tk, k, D, H, rows, ld)) || (r = make_map(&tv, v, D, H, rows, ld)))
    return r;
  kta::WinBwdParams p{};
  p.B = s.B;
  p.P = s.P;
  p.F = s.F;
  p.Htot = H;
  p.H0 = H;
  p.W[0] = p.W[1] = W;
  p.dil[0] = p.dil[1] = dil;
  p.n_t = (s.P + 127) / 128;
  p.rows_b = static_cast<int>(N);
  p.ld = ld;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse = lse;
  p.Dt = Dt;
  const long long nblk = static_cast<long long>(s.F) * H * s.B * p.n_t;
  if (nblk > 0x7fffffffLL) return fail(KTA_ERR_UNSUPPORTED, "too many tiles (%lld)", nblk);
  const size_t smem = kta::win_bwd_smem_bytes<D>();
  if ((r = set_smem_attr(kta::win_bwd_dq_kernel<D>, smem)) ||
      (r = set_smem_attr(kta::win_bwd_dkv_kernel<D>, smem)))
    return r;
  {
    p.out0 = static_cast<__nv_bfloat16*>(dq);
    p.out1 = nullptr;
    TraceScope ts("win_bwd_dq", st);
    kta::win_bwd_dq_kernel<D><<<static_cast<unsigned>(nblk), 256, smem, st>>>(tq, tdo, tk, tv, p);
    KTA_CUDA(cudaGetLastError());
  }
  p.out0 = static_cast<__nv_bfloat16*>(dk);
  p.out1 = static_cast<__nv_bfloat16*>(dv);
  TraceScope ts("win_bwd_dkv", st);
  kta::win_bwd_dkv_kernel<D><<<static_cast<unsigned>(nblk), 256, smem, st>>>(tq, tdo, tk, tv, p);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

}  // namespace

extern "C" {

kta_status kta_softmax_fwd_lse(const void* q, const void* k, const void* v, void* o, float* lse,
                               kta_shape s, int H, int ld_heads, int W, int dil, float scale,
                               void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) || (r = check_ptrs({q, k, v, o})) ||
      (r = check_softmax_dtype(s)))
    return r;
  if (s.dtype != KTA_BF16 || (s.d != 64 && s.d != 128))
    return fail(KTA_ERR_UNSUPPORTED, "the row log-sum-exp output needs bf16 and d in {64, 128}");
  if (!lse) return fail(KTA_ERR_INVALID_ARG, "null lse");
  if (W < 1 || dil < 1) return fail(KTA_ERR_INVALID_ARG, "W and dil must be >= 1");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be > 0");
  WinLaunch L = seq_win_launch(q, k, v, o, s, ld_heads, scale);
  L.g[0] = seq_group(k, v, s, H, H, ld_heads, W, dil);
  L.lse = lse;
  return launch_win(L, as_stream(stream));
}

kta_status kta_softmax_bwd_bf16(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                kta_shape s, int H, int ld_heads, int W, int dil, float scale,
                                void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) ||
      (r = check_ptrs({q, k, v, o, dout, dq, dk, dv})))
    return r;
  if (s.dtype != KTA_BF16 || (s.d != 64 && s.d != 128))
    return fail(KTA_ERR_UNSUPPORTED, "the tensor-core backward needs bf16 and d in {64, 128}");
  if (!lse) return fail(KTA_ERR_INVALID_ARG, "null lse");
  if (W < 1 || dil < 1) return fail(KTA_ERR_INVALID_ARG, "W and dil must be >= 1");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be > 0");
  cudaStream_t st = as_stream(stream);
  if (s.d == 128)
    return launch_win_bwd_tc<128>(q, k, v, o, lse, dout, dq, dk, dv, s, H, ld_heads, W, dil, scale, st);
  return launch_win_bwd_tc<64>(q, k, v, o, lse, dout, dq, dk, dv, s, H, ld_heads, W, dil, scale, st);
}

kta_status kta_proj_fwd(const void* x, const void* w, int M, int N, int K,
                        const kta_proj_seg* segs, int nseg, void* stream) {
  if (!x || !w || !segs) return fail(KTA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(w)) return fail(KTA_ERR_ALIGNMENT, "x and w must be 16-byte aligned");
  if (M < 1 || N < 1 || K < 1) return fail(KTA_ERR_INVALID_ARG, "M, N, K must be >= 1");
  if (K % 8) return fail(KTA_ERR_ALIGNMENT, "K must be a multiple of 8 (16-byte rows)");
  if (nseg < 1 || nseg > kta::PG_MAXSEG)
    return fail(KTA_ERR_INVALID_ARG, "nseg must be in [1, %d]", kta::PG_MAXSEG);
  kta::ProjParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.nseg = nseg;
  for (int i = 0; i < nseg; ++i) {
    const kta_proj_seg& g = segs[i];
    if (g.col_begin < 0 || g.col_end > N || g.col_begin >= g.col_end)
      return fail(KTA_ERR_INVALID_ARG, "segment %d: need 0 <= col_begin < col_end <= N", i);
    if (!g.dst) return fail(KTA_ERR_INVALID_ARG, "segment %d: null dst", i);
    if (g.mode < KTA_PROJ_BF16 || g.mode > KTA_PROJ_F32)
      return fail(KTA_ERR_INVALID_ARG, "segment %d: bad mode", i);
    if (g.ld < g.col_end - g.col_begin)
      return fail(KTA_ERR_INVALID_ARG, "segment %d: ld smaller than its width", i);
    for (int j = 0; j < i; ++j)
      if (g.col_begin < segs[j].col_end && segs[j].col_begin < g.col_end)
        return fail(KTA_ERR_INVALID_ARG, "segments %d and %d overlap", j, i);
    kta::ProjSeg& d = p.seg[i];
    d.c0 = g.col_begin;
    d.c1 = g.col_end;
    d.dst = g.dst;
    d.ld = g.ld;
    d.mode = g.mode;
    d.bias = g.bias;
    const long long esz = g.mode == KTA_PROJ_BF16 ? 2 : 4;
    d.vec = aligned16(g.dst) && (g.ld * esz) % 16 == 0 && (!g.bias || aligned16(g.bias));
  }
  CUtensorMap ta, tb;
  const cuuint64_t sK[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint64_t dA[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint32_t bA[2] = {kta::PG_BK, kta::PG_BM};
  const cuuint64_t dB[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
  const cuuint32_t bB[2] = {kta::PG_BK, kta::PG_BN};
  kta_status r;
  if ((r = make_map_nd(&ta, x, 2, dA, sK, bA)) || (r = make_map_nd(&tb, w, 2, dB, sK, bB)))
    return r;
  const size_t smem = kta::proj_smem_bytes();
  if ((r = set_smem_attr(kta::proj_gemm_kernel, smem))) return r;
  const long long tiles = static_cast<long long>((M + kta::PG_BM - 1) / kta::PG_BM) *
                          ((N + kta::PG_BN - 1) / kta::PG_BN);
  const int grid = static_cast<int>(std::min<long long>(tiles, sm_count()));
  cudaStream_t st = as_stream(stream);
  TraceScope ts("proj_gemm", st);
  kta::proj_gemm_kernel<<<grid, 192, smem, st>>>(ta, tb, p);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

kta_status kta_swa_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq,
                       void* dk, void* dv, kta_shape s, int H, int ld_heads, int W, float scale,
                       void* stream) {
  return softmax_bwd_common(q, k, v, dout, dq, dk, dv, s, H, ld_heads, W, 1, scale, stream);
}

kta_status kta_dswa_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq,
                        void* dk, void* dv, kta_shape s, int H, int ld_heads, int W, int dil,
                        float scale, void* stream) {
  return softmax_bwd_common(q, k, v, dout, dq, dk, dv, s, H, ld_heads, W, dil, scale, stream);
}

kta_status kta_gla_bwd(const void* q, const void* k, const void* v, const float* alpha,
                       const float* S0, const void* dout, void* dq, void* dk, void* dv,
                       float* dalpha, float* dS0, kta_shape s, int H, int ld_heads, float scale,
                       void* stream) {
  return lin_bwd_common(q, k, v, alpha, nullptr, S0, dout, dq, dk, dv, dalpha, nullptr, dS0, s, H,
                        ld_heads, scale, false, false, stream);
}

kta_status kta_gla_delta_bwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, const void* dout, void* dq,
                             void* dk, void* dv, float* dalpha, float* dbeta, float* dS0,
                             kta_shape s, int H, int ld_heads, float scale, int erase_decayed,
                             void* stream) {
  return lin_bwd_common(q, k, v, alpha, beta, S0, dout, dq, dk, dv, dalpha, dbeta, dS0, s, H,
                        ld_heads, scale, true, erase_decayed != 0, stream);
}

kta_status kta_stream_create(const kta_hybrid_cfg* cfg, kta_stream_t* out) {
  if (!out) return fail(KTA_ERR_INVALID_ARG, "null output handle");
  *out = nullptr;
  kta_hybrid_cfg c = *cfg;
  c.s.F = 1;
  kta_status r;
  if ((r = check_cfg(&c))) return r;
  kta_stream_s* s = new kta_stream_s();
  s->cfg = c;
  KTA_CUDA(cudaGetDevice(&s->device));
  s->es = elem_size(c.s.dtype);
  s->R_swa = c.n_swa ? c.W_swa : 0;
  s->R_dswa = c.n_dswa ? (c.W_dswa - 1) * c.dil + 1 : 0;
  const size_t frame_bytes_swa = static_cast<size_t>(c.s.P) * c.n_swa * c.s.d * s->es;
  const size_t frame_bytes_dswa = static_cast<size_t>(c.s.P) * c.n_dswa * c.s.d * s->es;
  s->ring_swa_bytes = round_up(static_cast<size_t>(c.s.B) * s->R_swa * frame_bytes_swa, 256);
  s->ring_dswa_bytes = round_up(static_cast<size_t>(c.s.B) * s->R_dswa * frame_bytes_dswa, 256);
  s->state_bytes = round_up(static_cast<size_t>(c.s.B) * c.n_gla * c.s.d * c.s.d * 4, 256);
  size_t off = kHeader;
  s->off_swa_k = off; off += s->ring_swa_bytes;
  s->off_swa_v = off; off += s->ring_swa_bytes;
  s->off_dswa_k = off; off += s->ring_dswa_bytes;
  s->off_dswa_v = off; off += s->ring_dswa_bytes;
  s->off_state[0] = off; off += s->state_bytes;
  s->off_state[1] = off; off += s->state_bytes;
  s->arena_bytes = off;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&s->arena), s->arena_bytes);
  if (e != cudaSuccess) {
    delete s;
    return fail(KTA_ERR_CUDA, "cudaMalloc of %zu stream bytes failed: %s", off, cudaGetErrorString(e));
  }
  e = cudaMemset(s->arena, 0, s->arena_bytes);
  if (e != cudaSuccess) {
    cudaFree(s->arena);
    delete s;
    return fail(KTA_ERR_CUDA, "cudaMemset failed: %s", cudaGetErrorString(e));
  }
  {
    std::lock_guard<std::mutex> lk(g_streams_mu);
    g_streams[s] = true;
  }
  *out = s;
  return KTA_OK;
}

kta_status kta_stream_step(kta_stream_t s, const void* q_f, const void* k_f, const void* v_f,
                           const float* alpha_f, const float* beta_f, void* o_f, void* stream) {
  kta_status r;
  if ((r = valid_stream(s)) || (r = check_ptrs({q_f, k_f, v_f, o_f}))) return r;
  const kta_hybrid_cfg& c = s->cfg;
  if (c.n_gla > 0 && (!alpha_f || (c.gla_delta && !beta_f)))
    return fail(KTA_ERR_INVALID_ARG, "null gate pointer");
  if (s->frame >= (1LL << 30)) return fail(KTA_ERR_STATE, "frame counter exhausted");
  int dev = 0;
  KTA_CUDA(cudaGetDevice(&dev));
  if (dev != s->device) return fail(KTA_ERR_STATE, "stream handle belongs to device %d", s->device);
  cudaStream_t st = as_stream(stream);
  const kta_shape& sh = c.s;
  const int H = c.n_swa + c.n_dswa + c.n_gla;
  const int f = static_cast<int>(s->frame);
  char* swa_k = s->arena + s->off_swa_k;
  char* swa_v = s->arena + s->off_swa_v;
  char* dswa_k = s->arena + s->off_dswa_k;
  char* dswa_v = s->arena + s->off_dswa_v;
  // 1. append this frame's keys and values to the rings (one gather launch; every ring row holds
  // a whole number of 16-byte pieces since d is 64 or 128)
  {
    RingPutParams rp;
    rp.B = sh.B;
    rp.P = sh.P;
    int nc = 0;
    if (c.n_swa) {
      const int slot = f % s->R_swa;
      rp.c[nc++] = ring_copy(s, k_f, swa_k, 0, c.n_swa, s->R_swa, slot);
      rp.c[nc++] = ring_copy(s, v_f, swa_v, 0, c.n_swa, s->R_swa, slot);
    }
    if (c.n_dswa) {
      const int slot = f % s->R_dswa;
      rp.c[nc++] = ring_copy(s, k_f, dswa_k, c.n_swa, c.n_dswa, s->R_dswa, slot);
      rp.c[nc++] = ring_copy(s, v_f, dswa_v, c.n_swa, c.n_dswa, s->R_dswa, slot);
    }
    if ((r = ring_put(rp, nc, st))) return r;
  }
  // 2. softmax heads: queries of this frame against the rings
  const bool has_win = c.n_swa + c.n_dswa > 0;
  WinLaunch W;
  if (has_win) {
    WinLaunch& L = W;
    L.B = sh.B;
    L.P = sh.P;
    L.Fq = 1;
    L.f_base = f;
    L.d = sh.d;
    L.dt = sh.dtype;
    L.q = q_f;
    L.q_ld = static_cast<long long>(H) * sh.d;
    L.q_rows_b = sh.P;
    L.o = o_f;
    L.o_ld = L.q_ld;
    L.scale = c.scale_softmax;
    int gi = 0;
    if (c.n_swa) {
      WinGroup& g = L.g[gi++];
      g.H = c.n_swa;
      g.W = c.W_swa;
      g.dil = 1;
      g.k = swa_k;
      g.v = swa_v;
      g.k_ld = static_cast<long long>(c.n_swa) * sh.d;
      g.k_rows = static_cast<long long>(sh.B) * s->R_swa * sh.P;
      g.k_heads = c.n_swa;
      g.kh_off = 0;
      g.kb_frames = s->R_swa;
      g.kmod = s->R_swa;
      g.span_mode = 1;  // the window's frames wrap around the ring
    }
    if (c.n_dswa) {
      WinGroup& g = L.g[gi++];
      g.H = c.n_dswa;
      g.W = c.W_dswa;
      g.dil = c.dil;
      g.k = dswa_k;
      g.v = dswa_v;
      g.k_ld = static_cast<long long>(c.n_dswa) * sh.d;
      g.k_rows = static_cast<long long>(sh.B) * s->R_dswa * sh.P;
      g.k_heads = c.n_dswa;
      g.kh_off = c.n_swa;
      g.kb_frames = s->R_dswa;
      g.kmod = s->R_dswa;
    }
  }
  // 3. GLA heads: this frame's tokens from the carried state (ping-pong state buffers)
  LinLaunch G;
  if (c.n_gla) {
    LinLaunch& L = G;
    L.B = sh.B;
    L.N = sh.P;
    L.H = c.n_gla;
    L.d = sh.d;
    L.rows_b = sh.P;
    L.chunk = c.chunk;
    L.dt = sh.dtype;
    const size_t hoff = static_cast<size_t>(c.n_swa + c.n_dswa) * sh.d * s->es;
    L.q = static_cast<const char*>(q_f) + hoff;
    L.k = static_cast<const char*>(k_f) + hoff;
    L.v = static_cast<const char*>(v_f) + hoff;
    L.o = static_cast<char*>(o_f) + hoff;
    L.ld = static_cast<long long>(H) * sh.d;
    L.alpha = alpha_f;
    L.beta = beta_f;
    L.S0 = reinterpret_cast<const float*>(s->arena + s->off_state[s->cur]);
    L.S_out = reinterpret_cast<float*>(s->arena + s->off_state[1 - s->cur]);
    L.scale = c.scale_gla;
    L.delta = c.gla_delta != 0;
    L.erase_decayed = c.gla_delta == 2;
    if (has_win) {
      // planned for the SMs that the softmax launch leaves free (its last wave's remainder)
      const long long units = static_cast<long long>(c.n_swa + c.n_dswa) * sh.B;
      const long long n_qt = (sh.P + 127) / 128;
      const long long nblk = units * (units * ((n_qt + 1) / 2) >= 2 * 148 ? (n_qt + 1) / 2 : n_qt);
      const long long sm = sm_count(), rem = nblk % sm;
      L.cta_budget = static_cast<int>(nblk < sm ? sm - nblk : (rem ? sm - rem : sm));
    }
  }
  if (has_win && c.n_gla)
    r = run_forked(W, G, st);
  else if (has_win)
    r = launch_win(W, st);
  else if (c.n_gla)
    r = launch_lin(G, st);
  if (r) return r;
  if (c.n_gla) s->cur = 1 - s->cur;
  s->frame += 1;
  return KTA_OK;
}

kta_status kta_stream_reset(kta_stream_t s, void* stream) {
  kta_status r;
  if ((r = valid_stream(s))) return r;
  KTA_CUDA(cudaMemsetAsync(s->arena, 0, s->arena_bytes, as_stream(stream)));
  s->frame = 0;
  s->cur = 0;
  return KTA_OK;
}

int64_t kta_stream_frame(kta_stream_t s) { return valid_stream(s) ? -1 : s->frame; }

size_t kta_stream_state_bytes(kta_stream_t s) { return valid_stream(s) ? 0 : s->arena_bytes; }

kta_status kta_stream_save(kta_stream_t s, void* dev_dst, void* stream) {
  kta_status r;
  if ((r = valid_stream(s))) return r;
  if (!dev_dst) return fail(KTA_ERR_INVALID_ARG, "null destination");
  cudaStream_t st = as_stream(stream);
  BlobHeader hd{};
  hd.magic = s->magic;
  hd.cur = static_cast<uint32_t>(s->cur);
  hd.frame = s->frame;
  const kta_hybrid_cfg& c = s->cfg;
  hd.B = c.s.B; hd.P = c.s.P; hd.d = c.s.d; hd.n_swa = c.n_swa; hd.n_dswa = c.n_dswa;
  hd.n_gla = c.n_gla; hd.W_swa = c.W_swa; hd.W_dswa = c.W_dswa; hd.dil = c.dil;
  hd.dtype = c.s.dtype; hd.gla_delta = c.gla_delta;
  KTA_CUDA(cudaMemcpyAsync(dev_dst, s->arena + kHeader, s->arena_bytes - kHeader,
                           cudaMemcpyDeviceToDevice, st));
  // The header goes last in the blob so that the arena copy above stays one contiguous copy.
  KTA_CUDA(cudaMemcpyAsync(static_cast<char*>(dev_dst) + (s->arena_bytes - kHeader), &hd, sizeof(hd),
                           cudaMemcpyHostToDevice, st));
  KTA_CUDA(cudaStreamSynchronize(st));
  return KTA_OK;
}

kta_status kta_stream_load(kta_stream_t s, const void* dev_src, void* stream) {
  kta_status r;
  if ((r = valid_stream(s))) return r;
  if (!dev_src) return fail(KTA_ERR_INVALID_ARG, "null source");
  cudaStream_t st = as_stream(stream);
  BlobHeader hd{};
  KTA_CUDA(cudaMemcpyAsync(&hd, static_cast<const char*>(dev_src) + (s->arena_bytes - kHeader),
                           sizeof(hd), cudaMemcpyDeviceToHost, st));
  KTA_CUDA(cudaStreamSynchronize(st));
  const kta_hybrid_cfg& c = s->cfg;
  if (hd.magic != s->magic || hd.B != c.s.B || hd.P != c.s.P || hd.d != c.s.d ||
      hd.n_swa != c.n_swa || hd.n_dswa != c.n_dswa || hd.n_gla != c.n_gla ||
      hd.W_swa != c.W_swa || hd.W_dswa != c.W_dswa || hd.dil != c.dil || hd.dtype != c.s.dtype ||
      hd.gla_delta != c.gla_delta || hd.frame < 0 || hd.cur > 1)
    return fail(KTA_ERR_STATE, "state blob does not match this stream's configuration");
  KTA_CUDA(cudaMemcpyAsync(s->arena + kHeader, dev_src, s->arena_bytes - kHeader,
                           cudaMemcpyDeviceToDevice, st));
  s->frame = hd.frame;
  s->cur = static_cast<int>(hd.cur);
  return KTA_OK;
}

kta_status kta_stream_destroy(kta_stream_t s) {
  kta_status r;
  if ((r = valid_stream(s))) return r;
  {
    std::lock_guard<std::mutex> lk(g_streams_mu);
    g_streams.erase(s);
  }
  s->magic = 0;
  cudaError_t e1 = cudaDeviceSynchronize();
  cudaError_t e2 = cudaFree(s->arena);
  delete s;
  if (e1 != cudaSuccess || e2 != cudaSuccess)
    return fail(KTA_ERR_CUDA, "stream teardown failed: %s",
                cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
  return KTA_OK;
}

// --------------------------------------------------------------------------- tracing

kta_status kta_trace_begin(void) {
  TraceState& t = trace_state();
  for (TraceRec& r : t.recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  t.recs.clear();
  t.on = true;
  return KTA_OK;
}

kta_status kta_trace_end(int* n, const char** names, int* launches, double* total_ms, int cap) {
  TraceState& t = trace_state();
  t.on = false;
  std::vector<const char*> keys;
  std::map<const char*, std::pair<int, double>> agg;
  kta_status st = KTA_OK;
  for (TraceRec& r : t.recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess && st == KTA_OK)
      st = fail(KTA_ERR_CUDA, "trace event read failed: %s", cudaGetErrorString(e));
    if (!agg.count(r.name)) keys.push_back(r.name);
    agg[r.name].first += 1;
    agg[r.name].second += ms;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  t.recs.clear();
  if (n) *n = static_cast<int>(keys.size());
  for (int i = 0; i < static_cast<int>(keys.size()) && i < cap; ++i) {
    if (names) names[i] = keys[i];
    if (launches) launches[i] = agg[keys[i]].first;
    if (total_ms) total_ms[i] = agg[keys[i]].second;
  }
  return st;
}

// --------------------------------------------------------------------------- diagnostics

kta_status kta_device_status(void* stream) {
  KTA_CUDA(cudaStreamSynchronize(as_stream(stream)));
  unsigned int word = 0;
  KTA_CUDA(cudaMemcpyFromSymbol(&word, kta::g_dev_error, sizeof(word)));
  if (word) {
    const unsigned int zero = 0;
    KTA_CUDA(cudaMemcpyToSymbol(kta::g_dev_error, &zero, sizeof(zero)));
    if (word & kta::DEVERR_WAIT_TIMEOUT)
      return fail(KTA_ERR_TIMEOUT, "a bounded device wait expired (code 0x%x)", word);
    return fail(KTA_ERR_CUDA, "device error word 0x%x", word);
  }
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

}  // extern "C"

namespace kta {
__global__ void wait_timeout_probe_kernel(long long budget) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  // Nobody arrives on `bar`: the bounded wait must give up after `budget` cycles.
  mbar_wait(&bar, 0, budget);
}
}  // namespace kta

extern "C" kta_status kta_selftest_wait_timeout(long long budget_cycles, void* stream) {
  if (budget_cycles < 1 || budget_cycles > (1LL << 31))
    return fail(KTA_ERR_INVALID_ARG, "budget must be in [1, 2^31] cycles");
  kta::wait_timeout_probe_kernel<<<1, 1, 0, as_stream(stream)>>>(budget_cycles);
  KTA_CUDA(cudaGetLastError());
  return KTA_OK;
}

// =========================================================================== no-allocation GLA
//
// kta_gla_chunk_fwd allocates its segment workspace with cudaMalloc the first time it needs it
// (and when a larger call needs more). Some callers cannot allocate device memory at call time:
// a real-time rollout loop that forbids allocation once it is running, or a process whose device
// memory is entirely held by another allocator's pool. kta_gla_chunk_fwd_noalloc serves them:
// the same kernels and segment plan, with the workspace in the fixed device array below instead.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kNoAllocMaxDevices = 64;

// Segment states and decays of the chunked GLA. Every device that loads the library holds this
// array until the process exits. Every call shares it and it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::once_flag g_noalloc_once[kNoAllocMaxDevices];
void* g_noalloc_ptr[kNoAllocMaxDevices];
cudaError_t g_noalloc_err[kNoAllocMaxDevices];

// Device address of the scratch array on the current device. Host code must not pass the
// symbol itself to a kernel (on the host it is only a stand-in); the address is looked up once
// per device, with that device current.
kta_status noalloc_scratch(void** out) {
  int dev = 0;
  KTA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(KTA_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kNoAllocMaxDevices - 1);
  std::call_once(g_noalloc_once[dev], [dev] {
    void* p = nullptr;
    g_noalloc_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_noalloc_ptr[dev] = p;
  });
  if (g_noalloc_err[dev] != cudaSuccess || !g_noalloc_ptr[dev])
    return fail(KTA_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed: %s",
                cudaGetErrorString(g_noalloc_err[dev]));
  *out = g_noalloc_ptr[dev];
  return KTA_OK;
}

// The segment plan and kernels of launch_gla_chunk, with the scratch array as the workspace.
template <int D, int C>
kta_status launch_gla_chunk_noalloc(const LinLaunch& L, cudaStream_t st) {
  const GlaPlan g = gla_plan<D, C>(L);
  if (g.ws_bytes > kNoAllocScratchBytes)
    return fail(KTA_ERR_UNSUPPORTED,
                "needs %zu bytes of scratch; the no-allocation variant has %zu (use "
                "kta_gla_chunk_fwd, or fewer sequences x heads per call)",
                g.ws_bytes, kNoAllocScratchBytes);
  void* ws = nullptr;
  if (g.ws_bytes) {
    kta_status r = noalloc_scratch(&ws);
    if (r) return r;
  }
  return launch_gla_planned<D, C>(L, g, ws, st);
}

}  // namespace

extern "C" kta_status kta_gla_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                                const float* alpha, const float* S0, float* S_out,
                                                void* o, kta_shape s, int H, int ld_heads,
                                                int chunk, float scale, void* stream) {
  kta_status r;
  if ((r = check_shape(s)) || (r = check_heads(H, ld_heads, s)) || (r = check_ptrs({q, k, v, o})))
    return r;
  if (!alpha) return fail(KTA_ERR_INVALID_ARG, "null gate pointer");
  if (!aligned16(alpha) || (S0 && !aligned16(S0)) || (S_out && !aligned16(S_out)))
    return fail(KTA_ERR_ALIGNMENT, "gate / state pointers must be 16-byte aligned");
  if (chunk != 16 && chunk != 32 && chunk != 64)
    return fail(KTA_ERR_INVALID_ARG, "chunk must be 16, 32 or 64");
  if (!std::isfinite(scale)) return fail(KTA_ERR_INVALID_ARG, "scale must be finite");
  if (s.dtype != KTA_BF16 || (s.d != 64 && s.d != 128))
    return fail(KTA_ERR_UNSUPPORTED,
                "the no-allocation variant covers the bf16 chunked kernel (d = 64 or 128)");
  LinLaunch L;
  L.B = s.B;
  L.N = s.F * s.P;
  L.H = H;
  L.d = s.d;
  L.rows_b = L.N;
  L.chunk = chunk;
  L.dt = s.dtype;
  L.q = q;
  L.k = k;
  L.v = v;
  L.o = o;
  L.ld = static_cast<long long>(ld_heads) * s.d;
  L.alpha = alpha;
  L.S0 = S0;
  L.S_out = S_out;
  L.scale = scale;
  cudaStream_t st = as_stream(stream);
  if (s.d == 128) {
    if (chunk == 64) return launch_gla_chunk_noalloc<128, 64>(L, st);
    if (chunk == 32) return launch_gla_chunk_noalloc<128, 32>(L, st);
    return launch_gla_chunk_noalloc<128, 16>(L, st);
  }
  if (chunk == 64) return launch_gla_chunk_noalloc<64, 64>(L, st);
  if (chunk == 32) return launch_gla_chunk_noalloc<64, 32>(L, st);
  return launch_gla_chunk_noalloc<64, 16>(L, st);
}
