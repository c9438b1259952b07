// Router GEMM + gate + top-k (one kernel).
//
// logits r = W_r x  ("FFN、SwiGLU 与 MoE" sec. 3; ops-transformer MoE walkthrough,
// 优化一), accumulated in fp32 (same walkthrough, 坑三).  Selection is a
// k-round warp argmax (partial selection, not a sort, as in the walkthrough's
// 优化二) with ties to the lower expert index.  Weights: renormalised softmax
// over the selected logits, or the raw sqrt(softplus(s)) gate with the
// selection bias kept out of the weight ("5A · MoE fine-grained" sec. 1, 3).
//
// Work split: a block of 8 warps owns 32 consecutive tokens; each warp owns
// 4 of them.  For every chunk of 8 experts a lane accumulates 4x8 partial dot
// products over its slice of D (16-byte loads), then a 31-shuffle transpose
// reduction leaves lane l with the full dot product number l.  Logits go to
// shared memory, never to HBM.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kTokPerWarp = 4;
constexpr int kExpChunk = 8;     // kTokPerWarp * kExpChunk == 32
constexpr int kWarps = 8;
constexpr int kTokPerBlock = kTokPerWarp * kWarps;

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

template <typename TIn>
__global__ void __launch_bounds__(256) route_kernel(int T, int D, int E, int k, int gate,
                                                    const TIn *__restrict__ x,
                                                    const TIn *__restrict__ wr,
                                                    const float *__restrict__ bias,
                                                    const float *__restrict__ bias_vl,
                                                    const uint8_t *__restrict__ image_mask,
                                                    int32_t *__restrict__ topk_idx,
                                                    float *__restrict__ topk_w) {
  extern __shared__ float logits[];  // [kTokPerBlock][E]
  constexpr int V = Vec16<TIn>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb = warp * kTokPerWarp;              // first token of this warp within the block
  const long t_base = (long)blockIdx.x * kTokPerBlock + tb;

  // ---- phase 1: logits of this warp's 4 tokens
  for (int e0 = 0; e0 < E; e0 += kExpChunk) {
    float acc[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) acc[q] = 0.0f;
    for (int d = lane * V; d < D; d += 32 * V) {
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
            for (int i = 0; i < kTokPerWarp; ++i) acc[i * kExpChunk + ee] = fmaf(xv[i].get(v), wf, acc[i * kExpChunk + ee]);
          }
        }
      }
    }
    float r = transpose_reduce32(acc, lane);
    int i = lane / kExpChunk, e = e0 + lane % kExpChunk;
    if (e < E) {
      if (gate == MOE_GATE_SOFTMAX_TOPK_RENORM && bias) r += bias[e];  // router logit bias
      logits[(tb + i) * E + e] = r;
    }
  }
  __syncwarp();

  // ---- phase 2: top-k and weights, one token at a time per warp
  for (int i = 0; i < kTokPerWarp; ++i) {
    long t = t_base + i;
    if (t >= T) break;
    const float *lg = logits + (tb + i) * E;
    const float *sel_bias = nullptr;
    if (gate == MOE_GATE_SQRT_SOFTPLUS_RAW) {
      sel_bias = (bias_vl && image_mask && image_mask[t]) ? bias_vl : bias;
    }
    uint32_t removed = 0;  // bit j: expert lane + 32 j already selected
    int my_e = 0;
    float my_l = 0.0f;
    for (int r = 0; r < k; ++r) {
      float bk = -INFINITY;
      int be = E;
      for (int j = 0, e = lane; e < E; ++j, e += 32) {
        if (removed >> j & 1u) continue;
        float key = lg[e] + (sel_bias ? sel_bias[e] : 0.0f);
        if (key != key) key = -INFINITY;
        if (key > bk || (key == bk && e < be)) { bk = key; be = e; }
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        float ok = __shfl_xor_sync(0xffffffffu, bk, off);
        int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ok > bk || (ok == bk && oe < be)) { bk = ok; be = oe; }
      }
      if ((be & 31) == lane) removed |= 1u << (be >> 5);
      if (lane == r) { my_e = be; my_l = lg[be]; }
    }
    float w;
    if (gate == MOE_GATE_SOFTMAX_TOPK_RENORM) {
      float m = __shfl_sync(0xffffffffu, my_l, 0);   // the largest selected logit
      float ex = lane < k ? expf(my_l - m) : 0.0f;
      float sum = ex;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      w = ex / sum;
    } else {
      w = sqrtf(softplus_f32(my_l));
    }
    if (lane < k) {
      topk_idx[t * k + lane] = my_e;
      topk_w[t * k + lane] = w;
    }
  }
}

}  // namespace

moe_status launch_route(const MoEConfig &c, int T, const void *x, const void *w_router,
                        const float *bias, const float *bias_vl, const uint8_t *image_mask,
                        int32_t *topk_idx, float *topk_w, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int E = c.num_experts;
  size_t smem = (size_t)kTokPerBlock * E * sizeof(float);
  dim3 grid((T + kTokPerBlock - 1) / kTokPerBlock);
  if (c.act_dtype == MOE_F32) {
    auto kern = route_kernel<float>;
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<grid, 256, smem, s>>>(T, c.hidden_dim, E, c.top_k, c.gate, (const float *)x,
                                 (const float *)w_router, bias, bias_vl, image_mask, topk_idx, topk_w);
  } else {
    auto kern = route_kernel<__nv_bfloat16>;
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<grid, 256, smem, s>>>(T, c.hidden_dim, E, c.top_k, c.gate, (const __nv_bfloat16 *)x,
                                 (const __nv_bfloat16 *)w_router, bias, bias_vl, image_mask,
                                 topk_idx, topk_w);
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
