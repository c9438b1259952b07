// Router GEMM + gate + top-k (one kernel).
//
// logits r = W_r x  ("FFN、SwiGLU 与 MoE" sec. 3; ops-transformer MoE walkthrough,
// 优化一), accumulated in fp32 (same walkthrough, 坑三).  Selection is a
// k-round warp argmax (partial selection, not a sort, as in the walkthrough's
// 优化二) with ties to the lower expert index.  Weights: renormalised softmax
// over the selected logits, or the raw sqrt(softplus(s)) gate with the
// selection bias kept out of the weight ("5A · MoE fine-grained" sec. 1, 3).
//
// Work split: a block of 8 warps; each warp owns TPW tokens and sweeps the
// experts in chunks of EC.  A lane accumulates TPW x EC x PARTS partial dot
// products over its slice of D with 16-byte loads, where PARTS interleaved
// partial sums (PARTS consecutive 32-lane strides of D) keep several loads in
// flight; TPW * EC * PARTS = 32, so a 31-shuffle transpose reduction leaves
// lane l with partial sum number l, and PARTS - 1 more shuffles finish it.
// This path serves many experts (TPW=4, EC=8, PARTS=1); few experts (E <= 32)
// use route_few_kernel.  Logits go to shared memory, never to HBM.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "route_select.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

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

// Few experts: one token per warp.  The warp first issues every 16-byte load
// of its x row slice (up to kXV vectors per lane held in registers, so one
// DRAM round trip per chunk of D), then walks the experts: independent L1/L2
// loads of W_r, fp32 FMAs, one warp reduction per expert.
constexpr int kFewWarps = 4;  // 128-thread blocks: three fit per SM at ~150 registers

template <typename TIn>
__global__ void __launch_bounds__(kFewWarps * 32) route_few_kernel(int T, int D, int E, int k, int gate,
                                                        const TIn *__restrict__ x, const TIn *__restrict__ wr,
                                                        const float *__restrict__ bias,
                                                        const float *__restrict__ bias_vl,
                                                        const uint8_t *__restrict__ image_mask,
                                                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
  extern __shared__ float logits[];  // [kFewWarps][E]
  constexpr int V = Vec16<TIn>::N;
  constexpr int kXV = 16;
  constexpr int kChunk = kXV * 32 * V;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long t = (long)blockIdx.x * kFewWarps + warp;
  if (t >= T) return;  // whole warp: no block-wide barrier follows
  float *lg = logits + warp * E;
  for (int c0 = 0; c0 < D; c0 += kChunk) {
    Vec16<TIn> xv[kXV];
#pragma unroll
    for (int j = 0; j < kXV; ++j) {
      const int d = c0 + j * 32 * V + lane * V;
      if (d < D) xv[j] = load16(x + t * D + d);
      else xv[j].v = {};
    }
    for (int e = 0; e < E; ++e) {
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < kXV; ++j) {
        const int d = c0 + j * 32 * V + lane * V;
        if (d < D) {
          Vec16<TIn> wv = load16(wr + (long)e * D + d);
#pragma unroll
          for (int v = 0; v < V; ++v) a = fmaf(xv[j].get(v), wv.get(v), a);
        }
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0) lg[e] = c0 == 0 ? a : lg[e] + a;
    }
  }
  __syncwarp();
  if (lane == 0 && gate == MOE_GATE_SOFTMAX_TOPK_RENORM && bias)
    for (int e = 0; e < E; ++e) lg[e] += bias[e];  // router logit bias
  __syncwarp();
  select_topk(lg, t, E, k, gate, bias, bias_vl, image_mask, topk_idx, topk_w, lane);
}

template <typename TIn, int kTokPerWarp, int kParts>
__global__ void __launch_bounds__(256) route_kernel(int T, int D, int E, int k, int gate,
                                                    const TIn *__restrict__ x,
                                                    const TIn *__restrict__ wr,
                                                    const float *__restrict__ bias,
                                                    const float *__restrict__ bias_vl,
                                                    const uint8_t *__restrict__ image_mask,
                                                    int32_t *__restrict__ topk_idx,
                                                    float *__restrict__ topk_w) {
  extern __shared__ float logits[];  // [kTokPerBlock][E]
  constexpr int kExpChunk = 32 / (kTokPerWarp * kParts);
  constexpr int kTokPerBlock = kTokPerWarp * kWarps;
  constexpr int V = Vec16<TIn>::N;
  constexpr int kStride = 32 * V;     // elements covered by one warp-wide 16-byte load
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb = warp * kTokPerWarp;  // first token of this warp within the block
  const long t_base = (long)blockIdx.x * kTokPerBlock + tb;

  // ---- phase 1: logits of this warp's tokens
  for (int e0 = 0; e0 < E; e0 += kExpChunk) {
    float acc[32];  // index ((i * kExpChunk + ee) * kParts + part)
#pragma unroll
    for (int q = 0; q < 32; ++q) acc[q] = 0.0f;
    for (int d0 = 0; d0 < D; d0 += kParts * kStride) {
#pragma unroll
      for (int part = 0; part < kParts; ++part) {
        const int d = d0 + part * kStride + lane * V;
        if (d < D) {
          Vec16<TIn> xv[kTokPerWarp];
#pragma unroll
          for (int i = 0; i < kTokPerWarp; ++i) {
            long t = t_base + i;
            if (t < T) xv[i] = load16(x + t * D + d);
            else xv[i].v = {};
          }
#pragma unroll
          for (int ee = 0; ee < kExpChunk; ++ee) {
            int e = e0 + ee;
            if (e < E) {
              Vec16<TIn> wv = load16(wr + (long)e * D + d);
#pragma unroll
              for (int v = 0; v < V; ++v) {
                float wf = wv.get(v);
#pragma unroll
                for (int i = 0; i < kTokPerWarp; ++i) {
                  float &a = acc[(i * kExpChunk + ee) * kParts + part];
                  a = fmaf(xv[i].get(v), wf, a);
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

template <typename TIn, int TPW, int PARTS>
moe_status launch_route_t(const MoEConfig &c, int T, const void *x, const void *w_router, const float *bias,
                          const float *bias_vl, const uint8_t *image_mask, int32_t *topk_idx, float *topk_w,
                          cudaStream_t s) {
  constexpr int kTokPerBlock = TPW * kWarps;
  const int E = c.num_experts;
  const size_t smem = (size_t)kTokPerBlock * E * sizeof(float);
  const dim3 grid((T + kTokPerBlock - 1) / kTokPerBlock);
  auto kern = route_kernel<TIn, TPW, PARTS>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  kern<<<grid, 256, smem, s>>>(T, c.hidden_dim, E, c.top_k, c.gate, (const TIn *)x, (const TIn *)w_router, bias,
                               bias_vl, image_mask, topk_idx, topk_w);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_route(const MoEConfig &c, int T, const void *x, const void *w_router,
                        const float *bias, const float *bias_vl, const uint8_t *image_mask,
                        int32_t *topk_idx, float *topk_w, int *status, float *scratch, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (route_tc_ok(c))
    return launch_route_tc(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, status, scratch, s);
  const int E = c.num_experts;
  if (E <= 32) {  // one token per warp, x row slice in registers
    const size_t smem = (size_t)kFewWarps * E * sizeof(float);
    const dim3 grid((T + kFewWarps - 1) / kFewWarps);
    if (c.act_dtype == MOE_F32)
      route_few_kernel<float><<<grid, kFewWarps * 32, smem, s>>>(T, c.hidden_dim, E, c.top_k, c.gate, (const float *)x,
                                                      (const float *)w_router, bias, bias_vl, image_mask,
                                                      topk_idx, topk_w);
    else
      route_few_kernel<__nv_bfloat16><<<grid, kFewWarps * 32, smem, s>>>(
          T, c.hidden_dim, E, c.top_k, c.gate, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w_router, bias,
          bias_vl, image_mask, topk_idx, topk_w);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
  }
  if (c.act_dtype == MOE_F32)
    return launch_route_t<float, 4, 1>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, s);
  return launch_route_t<__nv_bfloat16, 4, 1>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, s);
}

}  // namespace moe
