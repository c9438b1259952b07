// Host-side launchers of the kernels (internal to libmoe_b200).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Tokens per dispatch chunk: the histogram and permute kernels work on
// chunks of this many consecutive tokens.
constexpr int kChunkTokens = 256;
inline int num_chunks(int T) { return (T + kChunkTokens - 1) / kChunkTokens; }

// route.cu ---------------------------------------------------------------
// Picks the tensor-core router (route_tc.cu) when route_tc_ok(c), else CUDA
// cores.  status: the workspace's device status word (bounded waits);
// scratch: route_scratch_floats(c, T) floats (null when that is 0).
moe_status launch_route(const MoEConfig &c, int T, const void *x, const void *w_router,
                        const float *bias, const float *bias_vl, const uint8_t *image_mask,
                        int32_t *topk_idx, float *topk_w, int *status, float *scratch, cudaStream_t s);

// route_tc.cu ------------------------------------------------------------
bool route_tc_ok(const MoEConfig &c);
// fp32 logit rows [T, E_pad] the tensor-core router stores for its selection pass
size_t route_scratch_floats(const MoEConfig &c, int T);
moe_status launch_route_tc(const MoEConfig &c, int T, const void *x, const void *w_router, const float *bias,
                           const float *bias_vl, const uint8_t *image_mask, int32_t *topk_idx, float *topk_w,
                           int *status, float *scratch, cudaStream_t s);

// dispatch.cu ------------------------------------------------------------
// chunk_cnt: [num_chunks(T), E] int32 scratch.  x_perm may be null: the row
// maps are built but no rows are copied.
moe_status launch_dispatch(const MoEConfig &c, int T, const int32_t *topk_idx, const float *topk_w,
                           const void *x, int32_t *expert_counts, int32_t *expert_offsets,
                           int32_t *slot_row, int32_t *row_token, float *row_weight, void *x_perm,
                           int32_t *chunk_cnt, cudaStream_t s);

// x_perm[r] = x[row_token[r]] for r < expert_offsets[E] (act dtype rows).
moe_status launch_gather(const MoEConfig &c, int T, const int32_t *expert_offsets, const int32_t *row_token,
                         const void *x, void *x_perm, cudaStream_t s);

// x_perm rows in f16, each scaled by a power of two (row_scale[r] = 2^-s_r),
// for the FP4 gate/up GEMM in f16 (bf16 activations only).
moe_status launch_gather_f16(const MoEConfig &c, int T, const int32_t *expert_offsets, const int32_t *row_token,
                             const void *x, void *x_perm, float *row_scale, cudaStream_t s);

// gemm_simt.cu -----------------------------------------------------------
// Grouped GEMMs on CUDA cores (fp32 FMA), any shape.  act: F32 or BF16 for
// activations and weights alike.
moe_status launch_gate_up_simt(const MoEConfig &c, int rows, const void *a, int a_rows,
                               const int32_t *row_token, const int32_t *offsets, const void *w_gate,
                               const void *w_up, int F, void *h, cudaStream_t s);
moe_status launch_down_simt(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                            const void *w_down, int F, const float *row_weight, void *y,
                            cudaStream_t s);

// gemm_tc.cu -------------------------------------------------------------
// Grouped GEMMs on tcgen05 tensor cores (bf16 in, fp32 accumulate).  Usable
// when tc_shapes_ok(): bf16 activations, D % 256 == 0, F % 128 == 0.
bool tc_shapes_ok(const MoEConfig &c, int F);
// A is dense [rows, D] when row_token is null; otherwise row r of A is
// a[row_token[r]] of a [a_rows, D] source (gathered by the GEMM's loads).
moe_status launch_gate_up_tc(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                             const int32_t *offsets, const void *w_gate, const void *w_up, int F, void *h,
                             int *status, cudaStream_t s);
moe_status launch_down_tc(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                          const void *w_down, int F, const float *row_weight, float *y, int *status,
                          cudaStream_t s);

// gemm_fp4.cu ------------------------------------------------------------
// The same projections with NVFP4 weights read in their packed form (codes
// and scales expanded to bf16 on chip).  Usable when fp4_direct_ok() for the
// projection's reduction length K (D for gate/up, F for down).
bool fp4_direct_ok(const MoEConfig &c, int K);
// row_scale non-null: `a` holds f16 rows scaled by 2^s_r (launch_gather_f16)
// and the MMAs run in f16; the epilogue multiplies g and u by row_scale[r].
// h_f16 (only with row_scale): h is stored in f16 instead of bf16.
moe_status launch_gate_up_fp4(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                              const int32_t *offsets, const void *w_gate, const void *w_up, const void *s_gate,
                              const void *s_up, const float *row_scale, void *h, int *status, cudaStream_t s,
                              bool h_f16 = false);
// h_f16: h is f16 (from launch_gate_up_fp4 with h_f16) and the MMAs run in f16.
moe_status launch_down_fp4(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                           const void *w_down, const void *s_down, const float *row_weight, float *y,
                           int *status, cudaStream_t s, bool h_f16 = false);
// The SwiGLU clamp bounds |h| within f16's range: |SiLU(g) u| <= L^2 with
// both pre-activations clipped, |h| <= L with h clipped; L <= 255 keeps
// either below 65504.
inline bool h_fits_f16(const MoEConfig &c) { return c.swiglu_clamp > 0.0f && c.swiglu_clamp <= 255.0f; }

// One block whose bounded wait never completes: records the timeout status.
moe_status launch_wait_selftest(int *status, cudaStream_t s);

// Violation counters of the checked build, one per file that checks (each
// returns its count and clears it; always 0 in other builds).
unsigned int violations_dispatch();
unsigned int violations_combine();
unsigned int violations_gemm_tc();
unsigned int violations_gemm_fp4();
unsigned int violations_gemm_simt();

// dequant.cu -------------------------------------------------------------
// n_elems values (a multiple of 16): packed [n/2] bytes + scales [n/16] -> bf16 [n].
moe_status launch_dequant_nvfp4(const void *packed, const void *scales, long n_elems, void *out,
                                cudaStream_t s);

// combine.cu -------------------------------------------------------------
moe_status launch_combine(const MoEConfig &c, int T, const void *y_perm, const int32_t *slot_row,
                          const void *shared_y, void *out, cudaStream_t s);

}  // namespace moe
