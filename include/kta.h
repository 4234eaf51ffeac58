/*
 * kta.h -- C ABI of libkta.so: the Hybrid Linear Temporal Attention operator on B200 (sm_100a).
 *
 * Operator source: paper-read "Kairos: A Native World Model Stack for Physical AI"
 * (yingwang.github.io), section 2 "Method", second pillar: short-range sliding-window attention
 * (SWA), mid-range dilated sliding-window attention (DSWA), and global gated linear attention
 * (GLA, "based on GatedDeltaNet") whose state update is given there as four equations. The
 * ai-papers.net summary ("3-layer hybrid temporal architecture") and the secrett2633 review
 * ("Method & Key Results", the Delta Update Rule) describe the same three branches.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Tensors are row-major, token-major with heads interleaved: x[b][n][h][c] is at element
 *  offset ((b*N + n)*ld_heads + h)*d + c, i.e. the pages' (B, F*L, D) layout with D = H*d and
 *  L = P tokens per frame. N = F*P tokens, frames in time order, tokens of a frame contiguous.
 *  A call that serves heads [h0, h0+H) of a wider tensor receives pointers already offset by
 *  h0*d elements and ld_heads = the tensor's total head count; its H heads are computed.
 *  q, k, v, o use kta_shape.dtype (KTA_BF16: bf16, KTA_F32: fp32). Gates and states are fp32.
 *  o is written only for the computed heads; nothing else in o is touched.
 *
 *  Every pointer is a DEVICE pointer into memory the caller owns (cudaMalloc / torch). The
 *  library keeps no reference to it after the call's work has run. Work is enqueued on the
 *  CUDA stream passed as `stream` (a cudaStream_t; NULL = the legacy default stream) and the
 *  call returns without waiting for it.
 *
 *  Errors: every entry point returns kta_status. Argument, size and alignment errors are found
 *  before anything is enqueued and leave every output untouched. A launch failure returns
 *  KTA_ERR_CUDA; kta_last_error() gives a one-line description (per host thread). No entry point
 *  aborts, throws, or exits.
 *
 *  Supported sizes: d in {32, 64, 128}; bf16 softmax and chunk kernels need d in {64, 128};
 *  KTA_F32 runs every branch on fp32 CUDA cores (the fp32 reference mode). B, F, P >= 1;
 *  N = F*P < 2^31. Alignment: q, k, v, o 16-byte aligned; (ld_heads*d*elem) a multiple of 16.
 *
 *  Scales: softmax scores use `scale` (d^-1/2 is standard attention); GLA / delta outputs are
 *  multiplied by `scale` (1.0 gives the pages' o_t = S_t q_t, which has no scale).
 *
 *  Library scratch: the chunked GLA and delta-rule calls keep one device workspace per (device,
 *  CUDA stream) they run on, grown with cudaMalloc when a call needs more (after a
 *  cudaStreamSynchronize of that stream) and kept until the process exits. Calls on the same
 *  stream run in order; calls on different streams never share scratch. The gated delta rule
 *  needs about 40 KB per 64-token chunk and head.
 */
#ifndef KTA_H
#define KTA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KTA_VERSION 1

typedef enum {
  KTA_OK = 0,
  KTA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, W < 1, dil < 1, ...          */
  KTA_ERR_UNSUPPORTED = 2,  /* a valid request this build does not implement (e.g. d = 96)  */
  KTA_ERR_ALIGNMENT = 3,    /* pointer or row stride not 16-byte aligned                    */
  KTA_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed                          */
  KTA_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired                           */
  KTA_ERR_STATE = 6         /* handle misuse: destroyed handle, frame capacity exceeded      */
} kta_status;

typedef enum { KTA_BF16 = 0, KTA_F32 = 1 } kta_dtype;

/* Frame grid of one call: B sequences of F frames of P tokens, head dimension d. */
typedef struct {
  int B, F, P, d;
  kta_dtype dtype;
} kta_shape;

/* Human-readable name of a status code (static string). */
const char* kta_status_str(kta_status s);

/* Detail of the last failed call on this host thread ("" if none). */
const char* kta_last_error(void);

/* ABI version (KTA_VERSION of the build). */
int kta_version(void);

/*
 * SWA -- paper-read, section 2, second pillar, SWA paragraph: standard softmax attention inside
 * a window of L x window_size tokens. Query token t of frame f = t/P sees every key s of frames
 * f-W+1 .. f (the own frame in full, no later frame):
 *     o_t = sum_s softmax_s(scale * q_t . k_s) v_s.
 * q, k, v, o: [B][N][ld_heads][d] (H heads computed). W >= 1 frames (W >= F gives full
 * frame-causal attention).
 */
kta_status kta_swa_fwd(const void* q, const void* k, const void* v, void* o, kta_shape s,
                       int H, int ld_heads, int W, float scale, void* stream);

/*
 * DSWA -- paper-read, section 2, second pillar, DSWA paragraph: the SWA window size, with
 * frames taken every dil-th step: query frame f sees key frames f, f-dil, ..., f-(W-1)*dil.
 * When dil divides F this equals SWA on the page's reshape (B, F*L, D) -> (B*dil, F/dil*L, D)
 * with frame f in group f mod dil. dil = 1 is SWA.
 */
kta_status kta_dswa_fwd(const void* q, const void* k, const void* v, void* o, kta_shape s,
                        int H, int ld_heads, int W, int dil, float scale, void* stream);

/*
 * GLA with a vector forget gate -- paper-read, section 2, second pillar, GLA paragraph (a
 * fixed-size state updated once per token, gated forgetting):
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,     o_t = scale * q_t S_t
 * token-causal over the flattened token order, S is d x d fp32, key-major (S[i][j], i over key
 * dims). alpha: [B][N][H][d] fp32 in (0,1). S0: [B][H][d][d] initial state or NULL (= 0).
 * S_out: [B][H][d][d] final state or NULL. chunk in {16, 32, 64} (the token block of the
 * chunked form; results do not depend on it beyond rounding).
 * Gate range: every gate in [0, 1] is handled exactly. The bf16 chunked path scales q and k
 * by gate products taken from the middle token of each chunk; a chunk whose products would
 * leave the fp32 range (more than 64 bits of decay on one side of the middle token in some key
 * dim, i.e. gates far below ~0.25 on average) is recomputed as 16-token sub-chunks, and a
 * sub-chunk that still fails token by token. Small gates therefore cost time (about 4x per
 * affected chunk, 64x where single tokens are needed, e.g. exact zeros), never accuracy.
 */
kta_status kta_gla_chunk_fwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* S0, float* S_out, void* o, kta_shape s, int H,
                             int ld_heads, int chunk, float scale, void* stream);

/*
 * End state of a vector-gated GLA run, without its outputs -- the same recurrence as
 * kta_gla_chunk_fwd (paper-read, section 2, second pillar, GLA paragraph):
 *     S_end = diag(prod_t alpha_t) S0 + sum_t diag(prod_{u>t} alpha_u) k_t^T v_t.
 * k, v: [B][N][ld_heads][d] bf16 rows as in kta_gla_chunk_fwd (N = F * P, first of H heads at the
 * pointer); alpha [B][N][H][d] fp32; S0 (NULL = zero) and S_out [B][H][d][d] fp32 key-major.
 * Runs the chunked state pass and the segment fold only (no output pass), for callers that need
 * a run's state map and not its outputs (a sequence split's per-rank end state from zero).
 *  - bf16 only, d in {64, 128}, chunk in {16, 32, 64}; KTA_F32 returns KTA_ERR_UNSUPPORTED.
 *  - S_out must not be NULL; k, v, alpha, S0, S_out 16-byte aligned.
 *  - Same gate range, workspace and concurrency rules as kta_gla_chunk_fwd.
 */
kta_status kta_gla_chunk_state(const void* k, const void* v, const float* alpha, const float* S0,
                               float* S_out, kta_shape s, int H, int ld_heads, int chunk,
                               void* stream);

/*
 * kta_gla_chunk_fwd without any device allocation. The pages have no counterpart: this is a
 * service for callers that cannot allocate device memory while they run -- a real-time rollout
 * loop that forbids allocation once started, or a process whose device memory is entirely held
 * by another allocator's pool. kta_gla_chunk_fwd takes its segment workspace from a cache it
 * grows with cudaMalloc; this variant runs the same kernels and segment plan with the workspace
 * in a fixed 32 MiB array in device memory, which every GPU that loads the library holds until
 * the process exits. It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - bf16 only, d in {64, 128}; other arguments and results as kta_gla_chunk_fwd.
 *  - A call whose workspace would exceed 32 MiB (sequences x heads x segments x (d*d + d) x 4
 *    bytes) returns KTA_ERR_UNSUPPORTED with the size it needs, before anything is enqueued.
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *    with that device current); make that first call before any stream capture. With lazy
 *    module loading (the CUDA 12 default) that first call may also load the library's device
 *    code and so back the array with device memory: make one warm-up call before the region
 *    in which nothing may allocate. Later calls allocate nothing.
 *  - Every call shares the array and leaves its contents behind; each call writes all the
 *    scratch it reads before reading it, so nothing needs clearing. Calls that overlap on the
 *    GPU (for example on two streams) race on the array: serialise them.
 */
kta_status kta_gla_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                     const float* alpha, const float* S0, float* S_out, void* o,
                                     kta_shape s, int H, int ld_heads, int chunk, float scale,
                                     void* stream);

/*
 * Gated delta rule -- paper-read, section 2, second pillar, the four update equations:
 *     v_old = M_{t-1} k_t,   v_new = beta_t v_t + (1 - beta_t) v_old,
 *     M_t = alpha_t M_{t-1} - v_old k_t^T + v_new k_t^T,   o_t = scale * M_t q_t
 * with scalar alpha_t (forget gate) and beta_t per token and head: alpha, beta [B][N][H] fp32.
 * The page's M is d_v x d_k; S0 / S_out hold its transpose S = M^T, [B][H][d][d] key-major,
 * the same layout as kta_gla_chunk_fwd. NULL S0 = zero state.
 */
kta_status kta_gla_delta_fwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, float* S_out, void* o,
                             kta_shape s, int H, int ld_heads, int chunk, float scale,
                             void* stream);

/*
 * Gated delta rule with the erase term decayed too -- the GatedDeltaNet update, which the
 * paper-read's GLA paragraph names as the branch's basis:
 *     M_t = alpha_t M_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = scale * M_t q_t
 * (the page's four lines keep v_old k^T undecayed). It equals kta_gla_delta_fwd with beta
 * replaced by alpha * beta and v by v / alpha. Same arguments, layouts and errors as
 * kta_gla_delta_fwd.
 */
kta_status kta_gla_gdn_fwd(const void* q, const void* k, const void* v, const float* alpha,
                           const float* beta, const float* S0, float* S_out, void* o,
                           kta_shape s, int H, int ld_heads, int chunk, float scale,
                           void* stream);

/*
 * Hybrid layer. The pages say only that the three branches' outputs form one mixed temporal
 * representation; this ABI splits heads: heads [0, n_swa) are SWA (window W_swa), the next
 * n_dswa heads DSWA (window W_dswa, dilation dil), the last n_gla heads GLA (vector gate) or,
 * with gla_delta = 1, the gated delta rule (the page's form), with gla_delta = 2 its decayed-erase
 * form (kta_gla_gdn_fwd). Outputs are concatenated by head in o.
 * q, k, v, o: [B][N][H][d] with H = n_swa + n_dswa + n_gla. alpha: [B][N][n_gla][d] (vector
 * GLA) or [B][N][n_gla] (delta); beta: [B][N][n_gla] (delta only, else ignored).
 * The softmax and GLA branches run concurrently on internal streams forked from `stream` and
 * joined back into it before the call returns.
 */
typedef struct {
  kta_shape s;
  int n_swa, n_dswa, n_gla;
  int W_swa, W_dswa, dil;
  int chunk;
  int gla_delta;            /* 0: vector-gated GLA, 1: delta rule, 2: decayed-erase delta rule */
  float scale_softmax, scale_gla;
} kta_hybrid_cfg;

kta_status kta_hybrid_fwd(const kta_hybrid_cfg* cfg, const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta, void* o, void* stream);

/*
 * Projections around the operator -- paper-read, section 2, second pillar, GLA paragraph:
 * q_t = W_Q x_t, k_t = W_K x_t, v_t = W_V x_t, beta_t = sigmoid(W_beta x_t), the forget gate
 * alpha_t likewise a sigmoid of a projection of x_t, and the output projection of the mixed
 * heads. kta_proj_fwd computes Y = X W^T on the tensor cores:
 *   x: [M][K] bf16 (row-major), w: [N][K] bf16 (one row per output column, the layout of a
 *   linear layer's weight), fp32 accumulation. K % 8 == 0; x and w 16-byte aligned.
 * and writes column ranges of Y through `segs` (1..8 non-overlapping ranges; columns outside
 * every range are dropped): row r, column c of range s goes to dst_s[r * ld_s + (c - col_begin_s)]
 * as bf16 (KTA_PROJ_BF16), sigmoid(Y) in fp32 (KTA_PROJ_SIGMOID_F32) or Y in fp32 (KTA_PROJ_F32),
 * after adding bias_s[c - col_begin_s] when the range has a bias (fp32, device; NULL = none; a
 * gate's offset, e.g. one that keeps forget gates near 1, which the pages' bias-free
 * projections leave to the caller).
 * With W = [W_Q; W_K; W_V; W_alpha; W_beta] one call produces every input of kta_hybrid_fwd.
 * Outputs must not overlap x or w.
 */
typedef enum { KTA_PROJ_BF16 = 0, KTA_PROJ_SIGMOID_F32 = 1, KTA_PROJ_F32 = 2 } kta_proj_mode;

typedef struct {
  int col_begin, col_end;   /* columns [col_begin, col_end) of Y */
  void* dst;                /* device pointer */
  long long ld;             /* row stride of dst in elements (>= col_end - col_begin) */
  int mode;                 /* kta_proj_mode */
  const float* bias;        /* [col_end - col_begin] fp32 device array, or NULL */
} kta_proj_seg;

kta_status kta_proj_fwd(const void* x, const void* w, int M, int N, int K,
                        const kta_proj_seg* segs, int nseg, void* stream);

/*
 * Reverse mode (training). The pages define only the forward operators (paper-read, section 2,
 * second pillar); these entry points give the gradients of L = sum(dout * o) for the o of the
 * matching forward call, in fp32 on CUDA cores: s.dtype must be KTA_F32, else
 * KTA_ERR_UNSUPPORTED. Every tensor uses its forward layout (q, k, v, dout, dq, dk, dv:
 * [B][N][ld_heads][d]; heads [0, H) are read and written, other heads untouched). Gradients are
 * overwritten, not accumulated. Workspace, from the calling stream's cache: the softmax branches
 * 3 floats per (row, head); vector GLA N * d floats + N * d doubles per (sequence, head) plus
 * 2 d*d + 2 d + 2 d*d floats and d doubles per sequence segment; the delta rule
 * (ceil(N/32) + 32) * d * d + 64 * d floats per (sequence, head) (checkpointed states).
 *
 * kta_swa_bwd / kta_dswa_bwd: with p_ts the forward's softmax weights over the visible keys,
 *     ds_ts = p_ts (dout_t . v_s - dout_t . o_t),  dq_t = scale sum_s ds_ts k_s,
 *     dk_s = scale sum_t ds_ts q_t,                dv_s = sum_t p_ts dout_t.
 */
kta_status kta_swa_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq,
                       void* dk, void* dv, kta_shape s, int H, int ld_heads, int W, float scale,
                       void* stream);
kta_status kta_dswa_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq,
                        void* dk, void* dv, kta_shape s, int H, int ld_heads, int W, int dil,
                        float scale, void* stream);

/*
 * bf16 reverse mode of the softmax heads on the tensor cores (SWA: dil = 1; DSWA: dil > 1).
 * kta_softmax_fwd_lse is kta_dswa_fwd (bf16, d in {64, 128}) that also writes each query row's
 * base-2 log-sum-exp lse_t = log2(sum_s 2^(scale log2(e) q_t . k_s)) over its visible keys to
 * lse ([B][H][N] fp32, head-major). kta_softmax_bwd_bf16 takes that forward's q, k, v, o and
 * lse with dout and writes dq, dk, dv (bf16, the forward's layout; every computed row written)
 * by the formulas of kta_swa_bwd with P_ts = 2^(scale log2(e) q_t . k_s - lse_t), accumulating in
 * fp32. Workspace: B * H * N floats for dout_t . o_t, from the calling stream's cache.
 */
kta_status kta_softmax_fwd_lse(const void* q, const void* k, const void* v, void* o, float* lse,
                               kta_shape s, int H, int ld_heads, int W, int dil, float scale,
                               void* stream);
kta_status kta_softmax_bwd_bf16(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                kta_shape s, int H, int ld_heads, int W, int dil, float scale,
                                void* stream);

/*
 * kta_gla_bwd: gradients of kta_gla_chunk_fwd's output. With the state adjoint
 * G_t = scale q_t^T dout_t + diag(alpha_{t+1}) G_{t+1} (G after the last token = 0):
 *     dq_t = scale S_t dout_t^T,  dk_t = G_t v_t^T,  dv_t = k_t G_t,
 *     dalpha_t[i] = sum_j G_t[i][j] S_{t-1}[i][j],  dS0 = diag(alpha_1) G_1,
 * the gate gradient evaluated through its equal log-gate form
 * dalpha_t = (1/alpha_t) sum_{u >= t} (q_u (.) dq_u - k_u (.) dk_u) (sums in fp64; accuracy
 * degrades for gates near 0).
 * dalpha: [B][N][H][d] fp32 (required). S0 as in the forward or NULL; dS0: [B][H][d][d] or NULL.
 */
kta_status kta_gla_bwd(const void* q, const void* k, const void* v, const float* alpha,
                       const float* S0, const void* dout, void* dq, void* dk, void* dv,
                       float* dalpha, float* dS0, kta_shape s, int H, int ld_heads, float scale,
                       void* stream);

/*
 * kta_gla_delta_bwd: gradients of kta_gla_delta_fwd (erase_decayed = 0) or kta_gla_gdn_fwd
 * (erase_decayed = 1). In the key-major state S = M^T both read w_t = k_t S_{t-1},
 * u_t = beta_t (v_t - e_t w_t), S_t = alpha_t S_{t-1} + k_t^T u_t with e_t = 1 (the page's four
 * lines) or alpha_t (decayed erase). With du_t = k_t G_t:
 *     dv_t = beta_t du_t,  dbeta_t = du_t . (v_t - e_t w_t),
 *     dk_t = G_t u_t^T - beta_t e_t S_{t-1} du_t^T,  dq_t = scale S_t dout_t^T,
 *     dalpha_t = <G_t, S_{t-1}> (- beta_t du_t . w_t when decayed),
 *     G_{t-1} = alpha_t G_t - beta_t e_t k_t^T du_t,  dS0 = G_0.
 * dalpha, dbeta: [B][N][H] fp32 (required); S0 / dS0: [B][H][d][d] or NULL.
 */
kta_status kta_gla_delta_bwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, const void* dout, void* dq,
                             void* dk, void* dv, float* dalpha, float* dbeta, float* dS0,
                             kta_shape s, int H, int ld_heads, float scale, int erase_decayed,
                             void* stream);

/*
 * kta_hybrid_fwd for the query frames f0 .. F-1 of a longer key / value span: the building block
 * of a sequence split across devices (each holds a run of frames and receives from its
 * predecessors the K/V frames its windows reach back to, plus the GLA state at its first token).
 *   cfg->s.F = frames in k and v; q, o, alpha, beta cover the last F - f0 of them
 *   ([B][(F - f0)*P][...]), k and v all F ([B][F*P][H][d]). Window frames are numbered within
 *   k / v, so the span must start at the sequence's frame 0 or reach back at least
 *   max(W_swa - 1, (W_dswa - 1) * dil) frames before f0 (otherwise the first windows are cut).
 *   The GLA / delta heads run over the query frames' tokens from the state S0 ([B][n_gla][d][d]
 *   key-major fp32, NULL = zero) and write their end state to S_out (or NULL).
 *   f0 = 0 with NULL S0 and S_out is kta_hybrid_fwd. f0 > 0 needs B == 1.
 */
kta_status kta_hybrid_fwd_window(const kta_hybrid_cfg* cfg, int f0, const void* q, const void* k,
                                 const void* v, const float* alpha, const float* beta,
                                 const float* S0, float* S_out, void* o, void* stream);

/*
 * T = diag(prod_t alpha_t) for each sequence and head: the transition of a vector-gated GLA run
 * (paper-read, section 2, second pillar, GLA paragraph: S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,
 * so the state after the run is T S_start + S_loc). alpha: [B][N][H][d] fp32 gates of the run
 * (their own tensor, heads contiguous); T: [B][H][d][d] fp32, the full matrix, zeros off the
 * diagonal, ready for kta_state_affine. The product is formed as 2^(sum of log2 alpha) with
 * log2 clamped at -200 (a zero gate gives 0); N = 0 gives the identity. d in {32, 64, 128};
 * pointers 16-byte aligned. The caller owns both buffers.
 */
kta_status kta_gla_transition(const float* alpha, float* T, int B, int N, int H, int d,
                              void* stream);

/*
 * Y_m = A_m X_m + E_m for n row-major d x d fp32 matrices (E may be NULL): composes the affine
 * state maps of consecutive token runs. The GLA and delta-rule state after a run is
 * T S_start + S_loc, where S_loc is the run's end state from a zero start and T its transition
 * (the end state of the run started from the identity with v = 0), so the state entering run j
 * is obtained by folding the runs before it. Y must not alias A or X.
 */
kta_status kta_state_affine(const float* A, const float* X, const float* E, float* Y, int n, int d,
                            void* stream);

/*
 * Streaming rollout -- paper-read, section 2, third pillar: low-latency rolling prediction, one
 * frame at a time. A stream holds, per sequence, the GLA state and a ring of the last
 * W_swa frames (SWA heads) or (W_dswa-1)*dil+1 frames (DSWA heads) of k and v. Each step takes
 * one frame of P tokens ([B][P][H][d] q, k, v, o; alpha [B][P][n_gla](...)), appends its k, v to
 * the rings, and produces exactly the rows of that frame that kta_hybrid_fwd would produce for
 * the whole sequence. cfg->s.F is ignored. kta_stream_create allocates the rings and state on
 * the current CUDA device; nothing else is allocated by steps.
 */
typedef struct kta_stream_s* kta_stream_t;

kta_status kta_stream_create(const kta_hybrid_cfg* cfg, kta_stream_t* out);
kta_status kta_stream_step(kta_stream_t st, const void* q_f, const void* k_f, const void* v_f,
                           const float* alpha_f, const float* beta_f, void* o_f, void* stream);
/* Back to frame 0 with a zero state (enqueued on `stream`). */
kta_status kta_stream_reset(kta_stream_t st, void* stream);
/* Frames consumed so far. */
int64_t kta_stream_frame(kta_stream_t st);
/* Size of the opaque state blob written by kta_stream_save (rings + GLA state + counter). */
size_t kta_stream_state_bytes(kta_stream_t st);
/* Copy the state to / from device memory of kta_stream_state_bytes bytes (on `stream`). A
 * blob may be loaded into any stream created with an identical cfg. */
kta_status kta_stream_save(kta_stream_t st, void* dev_dst, void* stream);
kta_status kta_stream_load(kta_stream_t st, const void* dev_src, void* stream);
/* Frees the rings and state; synchronises the device first. */
kta_status kta_stream_destroy(kta_stream_t st);

/*
 * Device-side health. Every wait inside the library's kernels is bounded; a wait that runs out
 * records a code in a device error word and lets its kernel finish cleanly instead of hanging.
 * kta_device_status synchronises `stream`, returns KTA_ERR_TIMEOUT if such a code was recorded
 * since the last call (and clears it), KTA_ERR_CUDA on a pending CUDA error, else KTA_OK.
 */
kta_status kta_device_status(void* stream);

/*
 * Diagnostic: launches one thread that waits on a barrier nobody arrives at, with a budget of
 * `budget_cycles` SM clock cycles (1 .. 2^31), so that the bounded-wait path can be exercised
 * without hanging the GPU. The next kta_device_status(stream) must return KTA_ERR_TIMEOUT.
 */
kta_status kta_selftest_wait_timeout(long long budget_cycles, void* stream);

/*
 * Tracing. Between kta_trace_begin() and kta_trace_end(), every kernel the library launches from
 * this host thread is bracketed by a pair of CUDA events recorded on the stream it is launched
 * on. kta_trace_end synchronises those events and fills, for up to `cap` distinct kernels, the
 * kernel name (static string), its launch count and its summed device time in milliseconds;
 * *n receives the number of distinct kernels. Tracing adds two event records per launch.
 */
kta_status kta_trace_begin(void);
kta_status kta_trace_end(int* n, const char** names, int* launches, double* total_ms, int cap);

#ifdef __cplusplus
}
#endif

#endif /* KTA_H */
