/*
 * moe.h -- C ABI of libmoe_b200.so: forward pass of a Mixture-of-Experts
 * SwiGLU FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer (sources are web pages on the subject, cited by title and section):
 *
 *   logits  r = W_r x                     "FFN、SwiGLU 与 MoE" sec. 3; ops-transformer
 *                                          MoE walkthrough, MoEForward step 1 / 优化一
 *   gate    softmax + top-k renormalised  "FFN、SwiGLU 与 MoE" sec. 3 (example module)
 *           or sqrt(softplus(s)) raw,     "5A · MoE fine-grained" sec. 1 (DeepSeek-V4.1-Flash
 *           selection on s + bias/bias_vl  course): selection separated from weighting
 *   dispatch group tokens by expert,      ops-transformer walkthrough, MoEForward step 3,
 *           capacity drops in token order  坑一 (expert capacity)
 *   experts y = W_down[SiLU(W_gate x) * (W_up x)], optional +-clamp, optional shared
 *           expert                         "FFN、SwiGLU 与 MoE" sec. 2; "5A" sec. 1, 3
 *   combine out[t] = sum_j w_j y_j (+ shared)
 *                                          ops-transformer MoEForward step 4 (WeightedSum);
 *                                          Echo MoE quick reference, "Combine"
 *
 * Conventions for every entry point:
 *  - Pointers named in the argument lists are DEVICE pointers owned by the
 *    caller, unless documented as host.  The library allocates and frees no
 *    memory; scratch comes from the caller's workspace `ws`.
 *  - Tensors are dense row-major (last index fastest), 16-byte aligned.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Argument errors are detected on the host and returned
 *    synchronously, before anything is enqueued.  Device-side errors (a
 *    bounded wait inside a kernel that gave up) are recorded in the status
 *    word at the start of `ws`; read them with moe_check_device_status().
 *  - Nothing about a layer is kept between calls.  The library's only global
 *    state is a launch counter, the fixed scratch array of
 *    moe_dispatch_noalloc and, in the checked build, its violation counters.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* null pointer, bad size, k > E, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,    /* valid but not implemented (dtype combination, E too large) */
  MOE_ERR_WORKSPACE = 3,      /* ws_bytes smaller than the matching *_workspace_size() */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime call failed (launch error, no device) */
  MOE_ERR_DEVICE_TIMEOUT = 5  /* a kernel's bounded wait expired; results are invalid */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_NVFP4 = 2 } moe_dtype;

typedef enum {
  /* p = softmax(r) over all experts, top-k of p, divided by the selected sum
   * ("FFN、SwiGLU 与 MoE" sec. 3).  An optional per-expert bias is a router
   * LOGIT bias: r_e + bias[e] enters both the selection and the weights. */
  MOE_GATE_SOFTMAX_TOPK_RENORM = 0,
  /* selection: top-k of s_e + bias_vl[e] at image positions, s_e + bias[e]
   * elsewhere; multiplier: sqrt(softplus(s_e)) of the raw score, not
   * normalised ("5A · MoE fine-grained" sec. 1, 3). */
  MOE_GATE_SQRT_SOFTPLUS_RAW = 1,
  /* selection as in MOE_GATE_SQRT_SOFTPLUS_RAW (bias / bias_vl enter the
   * selection key only); multiplier: sigmoid(s_e) = 1 / (1 + e^-s_e) of the
   * raw score, not normalised.  ("กลยุทธ์การกำหนดเส้นทาง MoE: Top-K,
   * Expert-Choice และ Sigmoid Gating", blogdee.com: the sigmoid gives the
   * mixing weights of the selected experts; the selection rule and the
   * absence of renormalisation are this library's reading.) */
  MOE_GATE_SIGMOID_RAW = 2
} moe_gate;

typedef enum {
  MOE_CLAMP_PREACT = 0, /* clip g = W_gate x and u = W_up x to [-L, L], then SiLU(g) * u */
  MOE_CLAMP_OUTPUT = 1  /* clip h = SiLU(g) * u to [-L, L] */
} moe_clamp_mode;

/* Layer configuration.  The first five fields are the ops-transformer
 * walkthrough's MoEConfig ("MoE的核心思路" section). */
typedef struct {
  int num_experts;             /* E, 1..1024 */
  int top_k;                   /* k, 1..min(E, 16) */
  int expert_capacity;         /* C: max kept assignments per expert; 0 = unlimited */
  int hidden_dim;              /* D */
  int intermediate_dim;        /* F (routed experts) */
  int shared_intermediate_dim; /* F_s of the always-on shared expert; 0 = none */
  moe_gate gate;
  float swiglu_clamp;          /* L; 0 = no clamp */
  moe_clamp_mode clamp_mode;
  moe_dtype act_dtype;         /* x, router weights, shared-expert weights, x_perm and
                                  the SwiGLU hidden h: MOE_F32 or MOE_BF16 */
  moe_dtype expert_dtype;      /* routed expert weights: MOE_F32 (only with F32
                                  activations), MOE_BF16 or MOE_NVFP4 (BF16 activations) */
  moe_dtype out_dtype;         /* layer output: MOE_F32 or MOE_BF16.  The expert outputs
                                  y are always fp32, so the only rounding after the down
                                  projection is this final store (a bf16 store alone is
                                  up to 2^-8 relative) */
} MoEConfig;

/* Weights.  Matrices are in nn.Linear layout (out_features x in_features), so
 * the reduction dimension is the last one ("K-major").  NVFP4 matrices are
 * stored as two e2m1 codes per byte (even K index in the low nibble) plus one
 * e4m3 scale byte per 16 consecutive K elements: value = e2m1 * e4m3. */
typedef struct {
  const void *w_router;        /* [E, D] act dtype (no router bias) */
  const void *w_gate;          /* [E, F, D]   (NVFP4: uint8 [E, F, D/2]) */
  const void *w_up;            /* [E, F, D]   (NVFP4: uint8 [E, F, D/2]) */
  const void *w_down;          /* [E, D, F]   (NVFP4: uint8 [E, D, F/2]) */
  const void *s_gate;          /* NVFP4 only: e4m3 [E, F, D/16] */
  const void *s_up;            /* NVFP4 only: e4m3 [E, F, D/16] */
  const void *s_down;          /* NVFP4 only: e4m3 [E, D, F/16] */
  const void *sh_gate;         /* [F_s, D] act dtype (shared expert) */
  const void *sh_up;           /* [F_s, D] */
  const void *sh_down;         /* [D, F_s] */
  const float *bias;           /* [E] or NULL: softmax mode logit bias / sqrt and sigmoid modes selection bias */
  const float *bias_vl;        /* [E] or NULL: sqrt and sigmoid modes selection bias at image positions */
} MoEWeights;

/* ------------------------------------------------------------------ misc */

/* Human-readable name of a status code (static string). */
const char *moe_status_string(moe_status s);

/* Library version string (static). */
const char *moe_version(void);

/* C = ceil(T * k * cf / E) with cf = cf_num / cf_den, in exact integer
 * arithmetic (ops-transformer walkthrough, 坑一: capacity = S*top_k/E*1.2,
 * here rounded up).  Returns 0 (unlimited) when cf_num <= 0, -1 on bad input. */
int moe_expert_capacity(int T, int top_k, int num_experts, int cf_num, int cf_den);

/* Kernels launched by this library in this process so far (diagnostic). */
uint64_t moe_launch_count(void);

/* 1 in the checked build of this library (libmoe_b200_checked.so, built with
 * MOE_CHECKED), 0 otherwise.  In the checked build every kernel checks the
 * indices it reads from its inputs before using them -- row maps against the
 * token count, slot rows against T * k, expert offsets for a negative start or
 * a decrease -- and on a failed check skips the access (a row it cannot read
 * is left unwritten, a group with bad offsets does no work) and counts a
 * violation; nothing traps.  A substitute for a device memory checker. */
int moe_checked_build(void);

/* Violations the checked build's kernels counted since the last call, then
 * reset; always 0 in other builds.  Synchronises the current device. */
uint64_t moe_checked_violations(void);

/* Synchronises `stream`, then reads and clears the device status word at the
 * start of `ws` (any workspace passed to the calls above).  Returns MOE_OK or
 * MOE_ERR_DEVICE_TIMEOUT; MOE_ERR_CUDA if the stream reports an error. */
moe_status moe_check_device_status(void *ws, moe_stream_t stream);

/* Exercises the timeout path of the kernels' bounded waits: launches one
 * block that waits, with the same bounded wait the GEMM pipelines use, on an
 * mbarrier that nothing arrives on.  After the limit (2 s) it records
 * MOE_ERR_DEVICE_TIMEOUT in the status word of `ws` and returns normally, so
 * the context stays usable.  ws: >= 256 bytes.  For tests of the failure
 * path; nothing else calls it. */
moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, moe_stream_t stream);

/* ------------------------------------------------------------ stage 1: route */

/* Bytes of workspace moe_route_topk needs: its device status word, plus for
 * E > 32 with bf16 activations (the tensor-core router) the fp32 logit rows
 * [T, E rounded up to 32] it hands to its selection kernel. */
size_t moe_route_workspace_size(const MoEConfig *cfg, int T);

/* Router GEMM + gate + top-k for T tokens (a1-a2).
 *   x          [T, D] act dtype
 *   w->w_router, w->bias, w->bias_vl as in MoEWeights (other fields unused)
 *   image_mask [T] uint8 (nonzero = image position) or NULL; sqrt and sigmoid gates only
 *   topk_idx   [T, k] int32 out: selected experts, descending selection key,
 *              equal keys ordered by lower expert index
 *   topk_w     [T, k] float out: the multipliers (renormalised softmax, or raw
 *              sqrt(softplus(s)), or raw sigmoid(s))
 *   ws         >= moe_route_workspace_size(cfg, T) bytes (status word)
 * Logits are accumulated in fp32 (ops-transformer walkthrough, 坑三).  With
 * E <= 32 one kernel computes them (bf16: warp-level tensor-core MMAs on
 * 16-token groups; fp32 activations: CUDA-core FMA) and selects from shared
 * memory.  With bf16 activations and 32 < E <= 512 they are computed on the
 * 5th-generation tensor cores and each token's logit row is stored to the
 * route workspace, from which a second kernel selects. */
moe_status moe_route_topk(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                          const uint8_t *image_mask, int32_t *topk_idx, float *topk_w, void *ws,
                          size_t ws_bytes, moe_stream_t stream);

/* --------------------------------------------------------- stage 2: dispatch */

/* Bytes of workspace moe_dispatch needs for T tokens. */
size_t moe_dispatch_workspace_size(const MoEConfig *cfg, int T);

/* Histogram, scan, capacity and permute (a3-a5).  Assignment (t, j) with
 * expert e = topk_idx[t, j] gets position p = number of assignments of e
 * from tokens t' < t; it is kept iff C == 0 or p < C, and then lands in
 * row expert_offsets[e] + p of x_perm.
 *   expert_counts  [E] int32 out: assignments per expert before capacity
 *   expert_offsets [E+1] int32 out: prefix sums of the kept counts; R =
 *                  expert_offsets[E] rows are used (R <= T*k)
 *   slot_row       [T, k] int32 out: row of (t, j), or -1 if dropped
 *   row_token      [T*k] int32 out: token of each row (first R valid)
 *   row_weight     [T*k] float out: topk_w of each row (first R valid)
 *   x_perm         [T*k, D] act dtype out: x_perm[r] = x[row_token[r]], r < R;
 *                  or NULL: only the maps are built (moe_expert_gate_up can
 *                  gather the rows from x itself), and x may then be NULL
 *   ws             >= moe_dispatch_workspace_size(cfg, T) bytes
 * Deterministic: no global atomics; counts and rows are identical run to run. */
moe_status moe_dispatch(const MoEConfig *cfg, int T, const int32_t *topk_idx, const float *topk_w,
                        const void *x, int32_t *expert_counts, int32_t *expert_offsets,
                        int32_t *slot_row, int32_t *row_token, float *row_weight, void *x_perm,
                        void *ws, size_t ws_bytes, moe_stream_t stream);

/* Dispatch for callers that cannot allocate device memory on their call path
 * (a plugin inside an inference engine that offers no workspace, a serving
 * loop that may not call cudaMalloc, a program whose memory is all owned by
 * another allocator).  No counterpart on the pages: it is moe_dispatch with
 * the per-chunk histogram scratch taken from a fixed array inside the library
 * (MOE_DISPATCH_NOALLOC_MAX_SCRATCH_INTS int32, 1 MiB, held on every GPU that
 * loads the library until exit) instead of `ws`.  Same arguments, layouts and
 * results as moe_dispatch otherwise.
 *  - Returns MOE_ERR_UNSUPPORTED when ceil(T / 256) * E exceeds the limit,
 *    MOE_ERR_INVALID_ARG for a bad config or pointer, MOE_ERR_CUDA if the
 *    array's device address cannot be obtained.
 *  - The first call on a device looks up the array's address on that device
 *    (cudaGetSymbolAddress); make it before any stream capture.
 *  - All calls share the one array: calls that overlap on the GPU race and
 *    must be serialised by the caller.  No entry needs clearing between calls.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define MOE_DISPATCH_NOALLOC_MAX_SCRATCH_INTS 262144
moe_status moe_dispatch_noalloc(const MoEConfig *cfg, int T, const int32_t *topk_idx,
                                const float *topk_w, const void *x, int32_t *expert_counts,
                                int32_t *expert_offsets, int32_t *slot_row, int32_t *row_token,
                                float *row_weight, void *x_perm, moe_stream_t stream);

/* ---------------------------------------------------------- stage 3: experts */

/* Bytes of workspace moe_grouped_swiglu needs for up to `rows` rows. */
size_t moe_grouped_swiglu_workspace_size(const MoEConfig *cfg, int rows);
/* Bytes of workspace moe_expert_gate_up / moe_expert_down need (status word). */
size_t moe_expert_workspace_size(const MoEConfig *cfg);

/* Grouped gate/up GEMM with the SwiGLU epilogue (a6).  For every expert e and
 * row r in [expert_offsets[e], expert_offsets[e+1]), with A[r] the r-th input row:
 *   h[r, :] = SiLU(clip(A[r] W_gate[e]^T)) * clip(A[r] W_up[e]^T)
 * (clip per cfg->swiglu_clamp / clamp_mode), fp32 accumulation, stored in the
 * act dtype.  expert_offsets == NULL means one group of `rows` rows using
 * expert 0's weights.  `rows` bounds every offset (R <= rows).
 *   a, row_token  row_token == NULL: A = a, dense [rows, D] (x_perm).
 *                 Otherwise A[r] = a[row_token[r]] with a = x [a_rows, D] and
 *                 row_token the map from moe_dispatch: the rows are gathered
 *                 by the GEMM's own loads and no x_perm is needed.  On the
 *                 tensor-core path the gather issues one TMA copy per 4 rows x
 *                 64 columns, slower than moe_dispatch's gather plus a dense
 *                 A at large sizes; moe_forward uses the dense form.
 *   w_gate/w_up [E, F, D] in cfg->expert_dtype; s_gate/s_up NVFP4 scales or NULL
 *   h           [rows, F] out */
moe_status moe_expert_gate_up(const MoEConfig *cfg, int rows, const void *a, int a_rows,
                              const int32_t *row_token, const int32_t *expert_offsets, const void *w_gate,
                              const void *w_up, const void *s_gate, const void *s_up, void *h, void *ws,
                              size_t ws_bytes, moe_stream_t stream);

/* Grouped down GEMM with the routing-weight epilogue (a7):
 *   y[r, :] = row_weight[r] * (h[r] W_down[e]^T)   (row_weight NULL = 1)
 *   h      [rows, F] act dtype
 *   w_down [E, D, F] in cfg->expert_dtype; s_down NVFP4 scales or NULL
 *   y      [rows, D] float out */
moe_status moe_expert_down(const MoEConfig *cfg, int rows, const void *h,
                           const int32_t *expert_offsets, const void *w_down, const void *s_down,
                           const float *row_weight, void *y, void *ws, size_t ws_bytes,
                           moe_stream_t stream);

/* Both expert GEMMs: x_perm -> y_perm (float [rows, D]) through h held in `ws` (a6 + a7). */
moe_status moe_grouped_swiglu(const MoEConfig *cfg, int rows, const void *x_perm,
                              const int32_t *expert_offsets, const MoEWeights *w,
                              const float *row_weight, void *y_perm, void *ws, size_t ws_bytes,
                              moe_stream_t stream);

/* ---------------------------------------------------------- stage 4: combine */

/* out[t, :] = sum_{j=0..k-1, slot_row[t,j] >= 0} y_perm[slot_row[t, j], :]
 *             (+ shared_y[t, :] when shared_y != NULL)                  (a9)
 * y_perm [>= max slot_row + 1, D] float (rows already carry their weights),
 * shared_y [T, D] float or NULL, out [T, D] in cfg->out_dtype.  Sums in fp32
 * in the fixed order j = 0..k-1, then the shared term.  Deterministic. */
moe_status moe_combine(const MoEConfig *cfg, int T, const void *y_perm, const int32_t *slot_row,
                       const void *shared_y, void *out, moe_stream_t stream);

/* ------------------------------------------------------------- whole layer */

/* Bytes of workspace moe_forward needs for T tokens. */
size_t moe_workspace_size(const MoEConfig *cfg, int T);

/* The whole layer: route, dispatch, experts, shared expert, combine.
 *   x [T, D] act dtype, out [T, D] cfg->out_dtype; image_mask as in moe_route_topk
 *   topk_idx_out [T, k] int32 or NULL: copy of the routing decision
 *   expert_counts_out [E] int32 or NULL: assignments per expert before capacity
 *   ws: workspace of at least moe_workspace_size(cfg, T) bytes
 * No host synchronisation; per-expert counts never leave the device.  The
 * kept count of expert e is min(expert_counts_out[e], C) (all of it when
 * C = 0) and the layer drops T*k minus their sum.
 * Same kernels and results as the stage entry points called in order, with
 * two differences in operand format for NVFP4 experts whose gate/up reduction
 * length D is a multiple of 256:
 *   - the gate/up GEMM multiplies f16 operands (x rows scaled by a power of
 *     two each, expanded FP4 weights) instead of bf16 ones.  Both are exact,
 *     so g and u are identical whenever every element of a token row
 *     satisfies |x| >= max|row| * 2^-31 or x = 0;
 *   - when the down reduction length F is a multiple of 256 too and the
 *     SwiGLU clamp L is in (0, 255] (so |h| <= L^2 < 65504), h is stored in
 *     f16 rather than bf16 and the down GEMM multiplies in f16.  f16 rounds h
 *     more finely, so the output differs from the staged bf16-h result by
 *     less than bf16's rounding of h. */
moe_status moe_forward(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                       const uint8_t *image_mask, void *out, int32_t *topk_idx_out,
                       int32_t *expert_counts_out, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward with stage timing hooks (for profilers and benchmarks).
 * events: n_events CUDA event handles (cudaEvent_t, created by the caller;
 * NULL entries are skipped), recorded on `stream` at the stage boundaries:
 *   [0] before routing, [1] after routing (a1-a2), [2] after the dispatch
 *   maps (histogram, scan, row positions: a3-a4), [3] after the row gather
 *   into x_perm (a5), [4] after the expert gate/up GEMM (a6), [5] after the
 *   down GEMM (a7), [6] after the shared expert (a8), [7] after combine (a9).
 * Each interval brackets exactly the kernels of its stage, so the elapsed
 * time between events i and i+1 is that stage's device time.
 * n_events is 0 (then events may be NULL and this is moe_forward) or
 * MOE_STAGE_EVENTS; anything else is MOE_ERR_INVALID_ARG.  A failed event
 * record returns MOE_ERR_CUDA. */
#define MOE_STAGE_EVENTS 8
moe_status moe_forward_profiled(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                                const uint8_t *image_mask, void *out, int32_t *topk_idx_out,
                                int32_t *expert_counts_out, void *ws, size_t ws_bytes, moe_stream_t stream,
                                void *const *events, int n_events);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
