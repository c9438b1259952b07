// Warp-cooperative top-k selection of one token's router logits, shared by
// the CUDA-core and the tensor-core routers.
//
// k rounds of a warp argmax over the logits in shared memory (a partial
// selection, as the ops-transformer MoE walkthrough's 优化二 intends, without
// its heap); larger key first, equal keys to the lower expert index.  Keys:
// the logit in softmax mode (any router logit bias already added), the raw
// score plus bias (or bias_vl at image positions) in the sqrt and sigmoid
// modes.  Weights: the renormalised softmax of the selected logits,
// sqrt(softplus(s)), or sigmoid(s) ("FFN、SwiGLU 与 MoE" sec. 3; "5A · MoE
// fine-grained" sec. 1, 3; the blogdee.com routing-strategies page on
// Sigmoid Gating).
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

// Lane r (< k) holds the r-th selected expert and its logit: the weights
// (renormalised softmax over the selected logits, sqrt(softplus(s)) or
// sigmoid(s)) and the stores.
__device__ __forceinline__ void store_selection(long t, int k, int gate, int my_e, float my_l,
                                                int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                                int lane) {
  float w;
  if (gate == MOE_GATE_SOFTMAX_TOPK_RENORM) {
    float m = __shfl_sync(0xffffffffu, my_l, 0);  // the largest selected logit
    float ex = lane < k ? expf(my_l - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    w = ex / sum;
  } else if (gate == MOE_GATE_SIGMOID_RAW) {
    w = 1.0f / (1.0f + expf(-my_l));  // -> 0 and 1 at the ends, never NaN
  } else {
    w = sqrtf(softplus_f32(my_l));
  }
  if (lane < k) {
    topk_idx[t * k + lane] = my_e;
    topk_w[t * k + lane] = w;
  }
}

// Top-k of one token's logits (in shared memory) and its weights, by one warp:
// k rounds of a warp argmax (larger key first, equal keys to the lower expert).
__device__ __forceinline__ void select_topk(const float *lg, long t, int E, int k, int gate,
                                            const float *__restrict__ bias, const float *__restrict__ bias_vl,
                                            const uint8_t *__restrict__ image_mask, int32_t *__restrict__ topk_idx,
                                            float *__restrict__ topk_w, int lane) {
  const float *sel_bias = nullptr;
  if (gate != MOE_GATE_SOFTMAX_TOPK_RENORM) sel_bias = (bias_vl && image_mask && image_mask[t]) ? bias_vl : bias;
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
  store_selection(t, k, gate, my_e, my_l, topk_idx, topk_w, lane);
}

// The same selection with each lane's keys (experts lane + 32 j, j < NJ,
// E <= 32 NJ) computed once into registers, for many experts: the k rounds
// then compare registers instead of re-reading the logits and the bias.
// Same keys, same comparisons, same ties, same weights as select_topk.
template <int NJ>
__device__ __forceinline__ void select_topk_cached(const float *lg, long t, int E, int k, int gate,
                                                   const float *__restrict__ bias, const float *__restrict__ bias_vl,
                                                   const uint8_t *__restrict__ image_mask,
                                                   int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                                   int lane) {
  const float *sel_bias = nullptr;
  if (gate != MOE_GATE_SOFTMAX_TOPK_RENORM) sel_bias = (bias_vl && image_mask && image_mask[t]) ? bias_vl : bias;
  float key[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    float v = -INFINITY;
    if (e < E) {
      v = lg[e] + (sel_bias ? sel_bias[e] : 0.0f);
      if (v != v) v = -INFINITY;
    }
    key[j] = v;
  }
  uint32_t removed = 0;  // bit j: expert lane + 32 j already selected
  int my_e = 0;
  float my_l = 0.0f;
  for (int r = 0; r < k; ++r) {
    float bk = -INFINITY;
    int be = E;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !(removed >> j & 1u) && (key[j] > bk || (key[j] == bk && e < be))) {
        bk = key[j];
        be = e;
      }
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
  store_selection(t, k, gate, my_e, my_l, topk_idx, topk_w, lane);
}

}  // namespace moe
