// Router GEMM + gate + top-k (one kernel).
//
// logits r = W_r x  ("FFN、SwiGLU 与 MoE" sec. 3; ops-transformer MoE walkthrough,
// 优化一), accumulated in fp32 (same walkthrough, 坑三).  Selection is a
// k-round warp argmax (partial selection, not a sort, as in the walkthrough's
// 优化二) with ties to the lower expert index.  Weights: renormalised softmax
// over the selected logits, or the raw sqrt(softplus(s)) gate with the
// selection bias kept out of the weight ("5A · MoE fine-grained" sec. 1, 3).
//
// Work split: each warp owns 4 tokens and sweeps the experts in chunks of 8.
// A lane accumulates 4 x 8 partial dot products over its slice of D, with the
// x loads of several 16-byte strides issued ahead; a 31-shuffle transpose
// reduction leaves lane l with dot product number l.  Logits go to shared
// memory, never to HBM, and the owning warp selects from there.  (Many
// experts with bf16 activations use the tensor-core router, route_tc.cu.)
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "route_select.cuh"

namespace moe {
namespace {

// Reduce a[32] across the warp: afterwards a[0] in lane l is the warp-wide sum
// of element l.
__device__ __forceinline__ float transpose_reduce32(float (&a)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = lane & s;
#pragma unroll
    for (int q = 0; q < s; ++q) {
      float send = upper ? a[q] : a[q + s];
      float keep = upper ? a[q + s] : a[q];
      a[q] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return a[0];
}

// Each warp owns kTokPerWarp tokens and sweeps the experts in chunks of
// kExpChunk = 32 / (kTokPerWarp * kParts).  Per pass over D the lanes first
// issue kAhead strides of 16-byte x loads for all of the warp's tokens (held
// in registers: several DRAM round trips in flight per lane), then reuse each
// W_r vector (L1/L2 resident) across those tokens.
template <typename TIn, int kTokPerWarp, int kParts, int kWarps, int kAhead>
__global__ void __launch_bounds__(kWarps * 32) route_kernel(int T, int D, int E, int k, int gate,
                                                           const TIn *__restrict__ x,
                                                           const TIn *__restrict__ wr,
                                                           const float *__restrict__ bias,
                                                           const float *__restrict__ bias_vl,
                                                           const uint8_t *__restrict__ image_mask,
                                                           int32_t *__restrict__ topk_idx,
                                                           float *__restrict__ topk_w) {
  extern __shared__ float logits[];  // [kTokPerBlock][E]
  constexpr int kExpChunk = 32 / (kTokPerWarp * kParts);
  static_assert(kExpChunk * kTokPerWarp * kParts == 32, "32 partial sums per lane");
  static_assert(kAhead % kParts == 0, "whole groups of parts per pass");
  constexpr int V = Vec16<TIn>::N;
  constexpr int kStride = 32 * V;     // elements covered by one warp-wide 16-byte load
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb = warp * kTokPerWarp;  // first token of this warp within the block
  const long t_base = (long)blockIdx.x * (kTokPerWarp * kWarps) + tb;

  // ---- phase 1: logits of this warp's tokens
  for (int e0 = 0; e0 < E; e0 += kExpChunk) {
    float acc[32];  // index ((i * kExpChunk + ee) * kParts + part)
#pragma unroll
    for (int q = 0; q < 32; ++q) acc[q] = 0.0f;
    for (int d0 = 0; d0 < D; d0 += kAhead * kStride) {
      Vec16<TIn> xv[kAhead][kTokPerWarp];
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const int d = d0 + u * kStride + lane * V;
#pragma unroll
        for (int i = 0; i < kTokPerWarp; ++i) {
          const long t = t_base + i;
          if (d < D && t < T) xv[u][i] = load16(x + t * D + d);
          else xv[u][i].v = {};
        }
      }
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const int part = u % kParts;
        const int d = d0 + u * kStride + lane * V;
        if (d < D) {
#pragma unroll
          for (int ee = 0; ee < kExpChunk; ++ee) {
            const int e = e0 + ee;
            if (e < E) {
              const Vec16<TIn> wv = load16(wr + (long)e * D + d);
#pragma unroll
              for (int v = 0; v < V; ++v) {
                const float wf = wv.get(v);
#pragma unroll
                for (int i = 0; i < kTokPerWarp; ++i) {
                  float &a = acc[(i * kExpChunk + ee) * kParts + part];
                  a = fmaf(xv[u][i].get(v), wf, a);
                }
              }
            }
          }
        }
      }
    }
    float r = transpose_reduce32(acc, lane);
#pragma unroll
    for (int off = 1; off < kParts; off <<= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    const int q = lane / kParts;
    const int i = q / kExpChunk, e = e0 + q % kExpChunk;
    if (lane % kParts == 0 && e < E) {
      if (gate == MOE_GATE_SOFTMAX_TOPK_RENORM && bias) r += bias[e];  // router logit bias
      logits[(tb + i) * E + e] = r;
    }
  }
  __syncwarp();

  for (int i = 0; i < kTokPerWarp; ++i) {
    const long t = t_base + i;
    if (t >= T) break;
    select_topk(logits + (tb + i) * E, t, E, k, gate, bias, bias_vl, image_mask, topk_idx, topk_w, lane);
  }
}

}  // namespace

template <typename TIn, int TPW, int PARTS, int WARPS, int AHEAD>
moe_status launch_route_t(const MoEConfig &c, int T, const void *x, const void *w_router, const float *bias,
                          const float *bias_vl, const uint8_t *image_mask, int32_t *topk_idx, float *topk_w,
                          cudaStream_t s) {
  constexpr int kTokPerBlock = TPW * WARPS;
  const int E = c.num_experts;
  const size_t smem = (size_t)kTokPerBlock * E * sizeof(float);
  const dim3 grid((T + kTokPerBlock - 1) / kTokPerBlock);
  auto kern = route_kernel<TIn, TPW, PARTS, WARPS, AHEAD>;
  if (smem > 48 * 1024)
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  kern<<<grid, WARPS * 32, smem, s>>>(T, c.hidden_dim, E, c.top_k, c.gate, (const TIn *)x, (const TIn *)w_router,
                                      bias, bias_vl, image_mask, topk_idx, topk_w);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_route(const MoEConfig &c, int T, const void *x, const void *w_router,
                        const float *bias, const float *bias_vl, const uint8_t *image_mask,
                        int32_t *topk_idx, float *topk_w, int *status, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (route_tc_ok(c)) return launch_route_tc(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, status, s);
  // CUDA cores: 4 tokens x 8 experts per lane and pass; 2-warp blocks keep
  // the grid several blocks per SM deep at a few thousand tokens
  if (c.act_dtype == MOE_F32)
    return launch_route_t<float, 4, 1, 2, 4>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, s);
  return launch_route_t<__nv_bfloat16, 4, 1, 2, 4>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w,
                                                   s);
}

}  // namespace moe
