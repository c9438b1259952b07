// C ABI of libmoe_b200: argument checks, workspace layout and the order of
// the stage kernels.  Every compute step runs in the kernels of this library.
#include <limits.h>
#include <stdlib.h>

#include <atomic>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {

inline size_t act_size(const MoEConfig &c) { return c.act_dtype == MOE_F32 ? 4 : 2; }
inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
inline bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }

// Sequential carving of a workspace into 256-byte aligned pieces.  With a
// null base it only measures.
struct Carve {
  char *base;
  size_t off = 0;
  explicit Carve(void *b) : base((char *)b) {}
  template <class T>
  T *take(size_t n) {
    size_t o = align_up(off, 256);
    off = o + n * sizeof(T);
    return base ? (T *)(base + o) : nullptr;
  }
};

moe_status validate_cfg(const MoEConfig *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  const int E = c->num_experts, k = c->top_k;
  if (E < 1 || k < 1 || k > E || k > 16) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (c->expert_capacity < 0) return MOE_ERR_INVALID_ARG;
  if (c->hidden_dim <= 0 || c->intermediate_dim <= 0 || c->shared_intermediate_dim < 0)
    return MOE_ERR_INVALID_ARG;
  if (c->hidden_dim % 8 != 0) return MOE_ERR_UNSUPPORTED;  // 16-byte row vectors
  if (c->gate != MOE_GATE_SOFTMAX_TOPK_RENORM && c->gate != MOE_GATE_SQRT_SOFTPLUS_RAW &&
      c->gate != MOE_GATE_SIGMOID_RAW)
    return MOE_ERR_INVALID_ARG;
  if (!(c->swiglu_clamp >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (c->clamp_mode != MOE_CLAMP_PREACT && c->clamp_mode != MOE_CLAMP_OUTPUT) return MOE_ERR_INVALID_ARG;
  if (c->out_dtype != MOE_F32 && c->out_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->act_dtype == MOE_F32) {
    if (c->expert_dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
  } else if (c->act_dtype == MOE_BF16) {
    if (c->expert_dtype == MOE_NVFP4) {
      if (c->hidden_dim % 16 || c->intermediate_dim % 16) return MOE_ERR_UNSUPPORTED;
    } else if (c->expert_dtype != MOE_BF16) {
      return MOE_ERR_UNSUPPORTED;
    }
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status validate_tokens(const MoEConfig *c, int T) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)T * c->top_k > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// ---- expert-stage workspace: [status][bf16 expansion of NVFP4 weights]
// NVFP4 projections whose reduction length fits the tensor-core FP4 path read
// the packed weights directly; the others are expanded to bf16 first (gate and
// up together, then down into the same space).
struct ExpertWs {
  int *status;
  __nv_bfloat16 *wexp;
};
inline bool gate_up_direct(const MoEConfig &c) { return fp4_direct_ok(c, c.hidden_dim); }
inline bool down_direct(const MoEConfig &c) { return fp4_direct_ok(c, c.intermediate_dim); }
ExpertWs carve_expert(Carve &cv, const MoEConfig &c, bool with_status = true) {
  ExpertWs w;
  w.status = with_status ? cv.take<int>(kStatusBytes / sizeof(int)) : nullptr;
  w.wexp = nullptr;
  if (c.expert_dtype == MOE_NVFP4) {
    const size_t n = (size_t)c.num_experts * c.intermediate_dim * c.hidden_dim;
    const size_t need = gate_up_direct(c) ? (down_direct(c) ? 0 : n) : 2 * n;
    if (need) w.wexp = cv.take<__nv_bfloat16>(need);
  }
  return w;
}

// ---- gate/up and down with dtype handling (offsets == null: single group)
moe_status run_gate_up(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                       const int32_t *offsets, const void *wg, const void *wu, const void *sg, const void *su,
                       void *h, const ExpertWs &ws, cudaStream_t s) {
  MoEConfig cc = c;
  if (gate_up_direct(c))
    return launch_gate_up_fp4(c, rows, a, a_rows, row_token, offsets, wg, wu, sg, su, nullptr, h, ws.status, s);
  if (c.expert_dtype == MOE_NVFP4) {
    const long n = (long)c.num_experts * c.intermediate_dim * c.hidden_dim;
    moe_status st = launch_dequant_nvfp4(wg, sg, n, ws.wexp, s);
    if (st != MOE_OK) return st;
    st = launch_dequant_nvfp4(wu, su, n, ws.wexp + n, s);
    if (st != MOE_OK) return st;
    wg = ws.wexp;
    wu = ws.wexp + n;
    cc.expert_dtype = MOE_BF16;
  }
  if (tc_shapes_ok(cc, c.intermediate_dim))
    return launch_gate_up_tc(cc, rows, a, a_rows, row_token, offsets, wg, wu, c.intermediate_dim, h, ws.status, s);
  return launch_gate_up_simt(cc, rows, a, a_rows, row_token, offsets, wg, wu, c.intermediate_dim, h, s);
}

moe_status run_down(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                    const void *wd, const void *sd, const float *row_weight, void *y,
                    const ExpertWs &ws, cudaStream_t s) {
  MoEConfig cc = c;
  if (down_direct(c))
    return launch_down_fp4(c, rows, h, offsets, wd, sd, row_weight, (float *)y, ws.status, s);
  if (c.expert_dtype == MOE_NVFP4) {
    const long n = (long)c.num_experts * c.intermediate_dim * c.hidden_dim;
    moe_status st = launch_dequant_nvfp4(wd, sd, n, ws.wexp, s);
    if (st != MOE_OK) return st;
    wd = ws.wexp;
    cc.expert_dtype = MOE_BF16;
  }
  if (tc_shapes_ok(cc, c.intermediate_dim))
    return launch_down_tc(cc, rows, h, offsets, wd, c.intermediate_dim, row_weight, (float *)y, ws.status, s);
  return launch_down_simt(cc, rows, h, offsets, wd, c.intermediate_dim, row_weight, y, s);
}

// Both expert projections: x_perm -> h -> y, as two launches (gate/up, then down).
moe_status run_experts(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                       const int32_t *offsets, const void *wg, const void *wu, const void *wd, const void *sg,
                       const void *su, const void *sd, const float *row_weight, void *h, void *y,
                       const ExpertWs &ws, cudaStream_t s) {
  moe_status st = run_gate_up(c, rows, a, a_rows, row_token, offsets, wg, wu, sg, su, h, ws, s);
  if (st != MOE_OK) return st;
  return run_down(c, rows, h, offsets, wd, sd, row_weight, y, ws, s);
}

// NVTX ranges around the whole layer and each of its stages, so a timeline
// profiler shows which stage enqueued which kernels.  Without a profiler
// attached the calls return at once.  The destructor closes whatever is still
// open when a stage returns early.
struct NvtxStages {
  int depth = 0;
  void enter(const char *name) {
    nvtxRangePushA(name);
    ++depth;
  }
  void leave() {
    if (depth > 0) {
      nvtxRangePop();
      --depth;
    }
  }
  ~NvtxStages() {
    while (depth > 0) leave();
  }
};
const char *const kStageNames[MOE_STAGE_EVENTS - 1] = {"moe.route", "moe.dispatch_maps", "moe.gather",
                                                       "moe.gate_up", "moe.down", "moe.shared", "moe.combine"};

// The shared expert viewed as a one-expert layer of width F_s in the act dtype.
MoEConfig shared_cfg(const MoEConfig &c) {
  MoEConfig sc = c;
  sc.num_experts = 1;
  sc.top_k = 1;
  sc.intermediate_dim = c.shared_intermediate_dim;
  sc.expert_dtype = c.act_dtype;
  return sc;
}


// ---- whole-layer workspace
struct ForwardWs {
  int *status;
  int32_t *topk_idx, *counts, *offsets, *slot_row, *row_token, *chunk_cnt;
  float *topk_w, *row_weight, *row_scale, *route_logits;
  void *x_perm, *h, *y_perm, *sh_y;
  ExpertWs ex;
};
ForwardWs carve_forward(Carve &cv, const MoEConfig &c, int T) {
  ForwardWs w;
  const size_t Tk = (size_t)T * c.top_k, E = c.num_experts, D = c.hidden_dim;
  const size_t as = act_size(c);
  w.status = cv.take<int>(kStatusBytes / sizeof(int));
  w.topk_idx = cv.take<int32_t>(Tk);
  w.topk_w = cv.take<float>(Tk);
  w.counts = cv.take<int32_t>(E);
  w.offsets = cv.take<int32_t>(E + 1);
  w.slot_row = cv.take<int32_t>(Tk);
  w.row_token = cv.take<int32_t>(Tk);
  w.row_weight = cv.take<float>(Tk);
  w.row_scale = gate_up_direct(c) ? cv.take<float>(Tk) : nullptr;
  w.route_logits = cv.take<float>(route_scratch_floats(c, T));
  w.chunk_cnt = cv.take<int32_t>((size_t)num_chunks(T) * E);
  w.x_perm = cv.take<char>(Tk * D * as);
  size_t hrows = Tk * c.intermediate_dim;
  if ((size_t)T * c.shared_intermediate_dim > hrows) hrows = (size_t)T * c.shared_intermediate_dim;
  w.h = cv.take<char>(hrows * as);
  w.y_perm = cv.take<float>(Tk * D);
  w.sh_y = c.shared_intermediate_dim ? cv.take<float>((size_t)T * D) : nullptr;
  w.ex.status = w.status;
  w.ex.wexp = carve_expert(cv, c, false).wexp;  // NVFP4 expansion space, if any projection needs it
  return w;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: configuration not supported";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a kernel's bounded wait expired";
  }
  return "unknown moe_status";
}

const char *moe_version(void) { return "moe_b200 0.1 sm_100a"; }

int moe_expert_capacity(int T, int top_k, int num_experts, int cf_num, int cf_den) {
  if (T < 0 || top_k <= 0 || num_experts <= 0 || cf_den <= 0) return -1;
  if (cf_num <= 0) return 0;
  unsigned long long n = (unsigned long long)T * (unsigned)top_k * (unsigned)cf_num;
  unsigned long long d = (unsigned long long)num_experts * (unsigned)cf_den;
  unsigned long long q = (n + d - 1) / d;
  return q > (unsigned long long)INT_MAX ? INT_MAX : (int)q;
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_checked_build(void) { return kChecked ? 1 : 0; }

uint64_t moe_checked_violations(void) {
  return (uint64_t)violations_dispatch() + violations_combine() + violations_gemm_tc() + violations_gemm_fp4() +
         violations_gemm_simt();
}

moe_status moe_check_device_status(void *ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int host = 0;
  MOE_CUDA_TRY(cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, s));
  MOE_CUDA_TRY(cudaStreamSynchronize(s));
  if (host != kDevOk) {
    MOE_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(int), s));
    MOE_CUDA_TRY(cudaStreamSynchronize(s));
    return MOE_ERR_DEVICE_TIMEOUT;
  }
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ws || ws_bytes < kStatusBytes) return MOE_ERR_INVALID_ARG;
  return launch_wait_selftest((int *)ws, (cudaStream_t)stream);
}

size_t moe_route_workspace_size(const MoEConfig *cfg, int T) {
  if (validate_cfg(cfg) != MOE_OK || T < 0) return 0;
  Carve cv(nullptr);
  cv.take<int>(kStatusBytes / sizeof(int));
  cv.take<float>(route_scratch_floats(*cfg, T));
  return align_up(cv.off, 256);
}

moe_status moe_route_topk(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                          const uint8_t *image_mask, int32_t *topk_idx, float *topk_w, void *ws,
                          size_t ws_bytes, moe_stream_t stream) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if ((st = validate_tokens(cfg, T)) != MOE_OK) return st;
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_route_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  if (!w || !ok_ptr(x) || !ok_ptr(w->w_router) || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  Carve cv(ws);
  int *status = cv.take<int>(kStatusBytes / sizeof(int));
  float *scratch = cv.take<float>(route_scratch_floats(*cfg, T));
  return launch_route(*cfg, T, x, w->w_router, w->bias, w->bias_vl, image_mask, topk_idx, topk_w, status, scratch,
                      (cudaStream_t)stream);
}

size_t moe_dispatch_workspace_size(const MoEConfig *cfg, int T) {
  if (validate_cfg(cfg) != MOE_OK || T < 0) return 0;
  Carve cv(nullptr);
  cv.take<int>(kStatusBytes / sizeof(int));
  cv.take<int32_t>((size_t)num_chunks(T) * cfg->num_experts);
  return align_up(cv.off, 256);
}

moe_status moe_dispatch(const MoEConfig *cfg, int T, const int32_t *topk_idx, const float *topk_w,
                        const void *x, int32_t *expert_counts, int32_t *expert_offsets,
                        int32_t *slot_row, int32_t *row_token, float *row_weight, void *x_perm,
                        void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if ((st = validate_tokens(cfg, T)) != MOE_OK) return st;
  if (!expert_counts || !expert_offsets || !ws) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_w || !slot_row || !row_token || !row_weight ||
                (x_perm && (!ok_ptr(x) || !aligned16(x_perm)))))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_dispatch_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE;
  Carve cv(ws);
  cv.take<int>(kStatusBytes / sizeof(int));
  int32_t *chunk_cnt = cv.take<int32_t>((size_t)num_chunks(T) * cfg->num_experts);
  return launch_dispatch(*cfg, T, topk_idx, topk_w, x, expert_counts, expert_offsets, slot_row,
                         row_token, row_weight, x_perm, chunk_cnt, (cudaStream_t)stream);
}

size_t moe_expert_workspace_size(const MoEConfig *cfg) {
  if (validate_cfg(cfg) != MOE_OK) return 0;
  Carve cv(nullptr);
  carve_expert(cv, *cfg);
  return align_up(cv.off, 256);
}

size_t moe_grouped_swiglu_workspace_size(const MoEConfig *cfg, int rows) {
  if (validate_cfg(cfg) != MOE_OK || rows < 0) return 0;
  Carve cv(nullptr);
  carve_expert(cv, *cfg);
  cv.take<char>((size_t)rows * cfg->intermediate_dim * act_size(*cfg));
  return align_up(cv.off, 256);
}

// An expert weight matrix: 16-byte aligned data, plus its scales (also
// 16-byte aligned: TMA reads them) when NVFP4.
static bool ok_matrix(const MoEConfig *cfg, const void *w, const void *scales) {
  return ok_ptr(w) && (cfg->expert_dtype != MOE_NVFP4 || ok_ptr(scales));
}

moe_status moe_expert_gate_up(const MoEConfig *cfg, int rows, const void *a, int a_rows,
                              const int32_t *row_token, const int32_t *expert_offsets, const void *w_gate,
                              const void *w_up, const void *s_gate, const void *s_up, void *h, void *ws,
                              size_t ws_bytes, moe_stream_t stream) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if (rows < 0 || !ws || (row_token && a_rows <= 0)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_expert_workspace_size(cfg)) return MOE_ERR_WORKSPACE;
  if (rows == 0) return MOE_OK;
  if (!ok_ptr(a) || !ok_ptr(h)) return MOE_ERR_INVALID_ARG;
  if (!ok_matrix(cfg, w_gate, s_gate) || !ok_matrix(cfg, w_up, s_up)) return MOE_ERR_INVALID_ARG;
  Carve cv(ws);
  ExpertWs ew = carve_expert(cv, *cfg);
  return run_gate_up(*cfg, rows, a, row_token ? a_rows : rows, row_token, expert_offsets, w_gate, w_up, s_gate,
                     s_up, h, ew, (cudaStream_t)stream);
}

moe_status moe_expert_down(const MoEConfig *cfg, int rows, const void *h,
                           const int32_t *expert_offsets, const void *w_down, const void *s_down,
                           const float *row_weight, void *y, void *ws, size_t ws_bytes,
                           moe_stream_t stream) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if (rows < 0 || !ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_expert_workspace_size(cfg)) return MOE_ERR_WORKSPACE;
  if (rows == 0) return MOE_OK;
  if (!ok_ptr(h) || !ok_ptr(y)) return MOE_ERR_INVALID_ARG;
  if (!ok_matrix(cfg, w_down, s_down)) return MOE_ERR_INVALID_ARG;
  Carve cv(ws);
  ExpertWs ew = carve_expert(cv, *cfg);
  return run_down(*cfg, rows, h, expert_offsets, w_down, s_down, row_weight, y, ew,
                  (cudaStream_t)stream);
}

moe_status moe_grouped_swiglu(const MoEConfig *cfg, int rows, const void *x_perm,
                              const int32_t *expert_offsets, const MoEWeights *w,
                              const float *row_weight, void *y_perm, void *ws, size_t ws_bytes,
                              moe_stream_t stream) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if (rows < 0 || !ws || !w) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_grouped_swiglu_workspace_size(cfg, rows)) return MOE_ERR_WORKSPACE;
  if (rows == 0) return MOE_OK;
  if (!ok_ptr(x_perm) || !ok_ptr(y_perm)) return MOE_ERR_INVALID_ARG;
  if (!ok_matrix(cfg, w->w_gate, w->s_gate) || !ok_matrix(cfg, w->w_up, w->s_up) ||
      !ok_matrix(cfg, w->w_down, w->s_down))
    return MOE_ERR_INVALID_ARG;
  Carve cv(ws);
  ExpertWs ew = carve_expert(cv, *cfg);
  void *h = cv.take<char>((size_t)rows * cfg->intermediate_dim * act_size(*cfg));
  return run_experts(*cfg, rows, x_perm, rows, nullptr, expert_offsets, w->w_gate, w->w_up, w->w_down, w->s_gate,
                     w->s_up, w->s_down, row_weight, h, y_perm, ew, (cudaStream_t)stream);
}

moe_status moe_combine(const MoEConfig *cfg, int T, const void *y_perm, const int32_t *slot_row,
                       const void *shared_y, void *out, moe_stream_t stream) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if ((st = validate_tokens(cfg, T)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!ok_ptr(y_perm) || !slot_row || !ok_ptr(out)) return MOE_ERR_INVALID_ARG;
  if (shared_y && !aligned16(shared_y)) return MOE_ERR_INVALID_ARG;
  return launch_combine(*cfg, T, y_perm, slot_row, shared_y, out, (cudaStream_t)stream);
}

size_t moe_workspace_size(const MoEConfig *cfg, int T) {
  if (validate_cfg(cfg) != MOE_OK || T < 0 || validate_tokens(cfg, T) != MOE_OK) return 0;
  Carve cv(nullptr);
  carve_forward(cv, *cfg, T);
  return align_up(cv.off, 256);
}

static moe_status forward_impl(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                               const uint8_t *image_mask, void *out, int32_t *topk_idx_out,
                               int32_t *expert_counts_out, void *ws, size_t ws_bytes, moe_stream_t stream,
                               void *const *events) {
  moe_status st = validate_cfg(cfg);
  if (st != MOE_OK) return st;
  if ((st = validate_tokens(cfg, T)) != MOE_OK) return st;
  if (!w || !ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE;
  if (T == 0) {  // nothing to compute; the stage boundaries still get their events
    for (int e = 0; events && e < MOE_STAGE_EVENTS; ++e)
      if (events[e] && cudaEventRecord((cudaEvent_t)events[e], (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!ok_ptr(x) || !ok_ptr(out) || !ok_ptr(w->w_router)) return MOE_ERR_INVALID_ARG;
  if (!ok_matrix(cfg, w->w_gate, w->s_gate) || !ok_matrix(cfg, w->w_up, w->s_up) ||
      !ok_matrix(cfg, w->w_down, w->s_down))
    return MOE_ERR_INVALID_ARG;
  if (cfg->shared_intermediate_dim &&
      (!ok_ptr(w->sh_gate) || !ok_ptr(w->sh_up) || !ok_ptr(w->sh_down)))
    return MOE_ERR_INVALID_ARG;
  const MoEConfig &c = *cfg;
  cudaStream_t s = (cudaStream_t)stream;
  Carve cv(ws);
  ForwardWs f = carve_forward(cv, c, T);
  int32_t *idx = topk_idx_out ? topk_idx_out : f.topk_idx;
  int32_t *counts = expert_counts_out ? expert_counts_out : f.counts;
  const int rows = T * c.top_k;
  // stage boundary i: record events[i] when the caller asked for it
  NvtxStages nvtx;
  nvtx.enter("moe_forward");
  auto mark = [&](int i) -> moe_status {
    if (i > 0) nvtx.leave();
    if (i + 1 < MOE_STAGE_EVENTS) nvtx.enter(kStageNames[i]);
    if (events && events[i] && cudaEventRecord((cudaEvent_t)events[i], s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  };

  if ((st = mark(0)) != MOE_OK) return st;
  if ((st = launch_route(c, T, x, w->w_router, w->bias, w->bias_vl, image_mask, idx, f.topk_w, f.status,
                         f.route_logits, s)) != MOE_OK)
    return st;
  if ((st = mark(1)) != MOE_OK) return st;
  // the row maps (histogram, scan, positions), then the row gather
  if ((st = launch_dispatch(c, T, idx, f.topk_w, x, counts, f.offsets, f.slot_row, f.row_token, f.row_weight,
                            nullptr, f.chunk_cnt, s)) != MOE_OK)
    return st;
  if ((st = mark(2)) != MOE_OK) return st;
  // NVFP4 experts on the direct path: x_perm is gathered in f16 with a
  // power-of-two scale per row and the gate/up GEMM multiplies in f16
  const bool fp4_f16 = f.row_scale != nullptr;
  if (fp4_f16) st = launch_gather_f16(c, T, f.offsets, f.row_token, x, f.x_perm, f.row_scale, s);
  else st = launch_gather(c, T, f.offsets, f.row_token, x, f.x_perm, s);
  if (st != MOE_OK) return st;
  if ((st = mark(3)) != MOE_OK) return st;
  // with the SwiGLU clamp bounding |h| below 65504, h is kept in f16 and the
  // NVFP4 down projection multiplies in f16 too
  const bool h_f16 = fp4_f16 && down_direct(c) && h_fits_f16(c);
  if (fp4_f16) {
    st = launch_gate_up_fp4(c, rows, f.x_perm, rows, nullptr, f.offsets, w->w_gate, w->w_up, w->s_gate, w->s_up,
                            f.row_scale, f.h, f.ex.status, s, h_f16);
  } else {
    st = run_gate_up(c, rows, f.x_perm, rows, nullptr, f.offsets, w->w_gate, w->w_up, w->s_gate, w->s_up, f.h,
                     f.ex, s);
  }
  if (st != MOE_OK) return st;
  if ((st = mark(4)) != MOE_OK) return st;
  if (h_f16) st = launch_down_fp4(c, rows, f.h, f.offsets, w->w_down, w->s_down, f.row_weight, (float *)f.y_perm,
                                  f.ex.status, s, true);
  else st = run_down(c, rows, f.h, f.offsets, w->w_down, w->s_down, f.row_weight, f.y_perm, f.ex, s);
  if (st != MOE_OK) return st;
  if ((st = mark(5)) != MOE_OK) return st;
  if (c.shared_intermediate_dim) {
    const MoEConfig sc = shared_cfg(c);
    if ((st = run_experts(sc, T, x, T, nullptr, nullptr, w->sh_gate, w->sh_up, w->sh_down, nullptr, nullptr,
                          nullptr, nullptr, f.h, f.sh_y, f.ex, s)) != MOE_OK)
      return st;
  }
  if ((st = mark(6)) != MOE_OK) return st;
  if ((st = launch_combine(c, T, f.y_perm, f.slot_row, f.sh_y, out, s)) != MOE_OK) return st;
  return mark(7);
}

moe_status moe_forward(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                       const uint8_t *image_mask, void *out, int32_t *topk_idx_out,
                       int32_t *expert_counts_out, void *ws, size_t ws_bytes, moe_stream_t stream) {
  return forward_impl(cfg, T, x, w, image_mask, out, topk_idx_out, expert_counts_out, ws, ws_bytes, stream,
                      nullptr);
}

moe_status moe_forward_profiled(const MoEConfig *cfg, int T, const void *x, const MoEWeights *w,
                                const uint8_t *image_mask, void *out, int32_t *topk_idx_out,
                                int32_t *expert_counts_out, void *ws, size_t ws_bytes, moe_stream_t stream,
                                void *const *events, int n_events) {
  if (n_events != 0 && (n_events != MOE_STAGE_EVENTS || !events)) return MOE_ERR_INVALID_ARG;
  return forward_impl(cfg, T, x, w, image_mask, out, topk_idx_out, expert_counts_out, ws, ws_bytes, stream,
                      n_events ? events : nullptr);
}

}  // extern "C"
