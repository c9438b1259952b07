// Combine: the routing-weighted sum back to token order (+ the shared expert).
//
// ops-transformer MoE walkthrough, MoEForward step 4 (WeightedSum); Echo MoE
// quick reference, "Combine"; "FFN、SwiGLU 与 MoE" sec. 3 (y = sum_i p_i E_i(x)).
// The weights were applied in the down-projection epilogue, so here
//   out[t] = sum_{j=0..k-1, slot kept} y_perm[slot_row[t, j]]  (+ shared_y[t])
// summed in fp32 in that fixed order: deterministic, no atomics.
//
// One warp per token row, 16-byte vector loads of the fp32 expert outputs: a
// pure HBM stream of k (+1 shared) rows read and one row written per token.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

template <typename TOut>
__global__ void __launch_bounds__(256) combine_kernel(int T, int D, int k,
                                                      const float *__restrict__ y_perm,
                                                      const int32_t *__restrict__ slot_row,
                                                      const float *__restrict__ shared_y,
                                                      TOut *__restrict__ out) {
  constexpr int V = 4;  // four fp32 per 16-byte load
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    int rows[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) rows[j] = j < k ? slot_row[(long)t * k + j] : -1;
#pragma unroll 4
    for (int c = lane * V; c < D; c += 32 * V) {
      float acc[V];
#pragma unroll
      for (int v = 0; v < V; ++v) acc[v] = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < k && rows[j] >= 0) {
          Vec16<float> y = load16(y_perm + (long)rows[j] * D + c);
#pragma unroll
          for (int v = 0; v < V; ++v) acc[v] += y.get(v);
        }
      }
      if (shared_y) {
        Vec16<float> y = load16(shared_y + (long)t * D + c);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] += y.get(v);
      }
      if constexpr (sizeof(TOut) == 4) {
        Vec16<float> o;
#pragma unroll
        for (int v = 0; v < V; ++v) o.set(v, acc[v]);
        store16((float *)out + (long)t * D + c, o);
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
        uint2 o = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
        *reinterpret_cast<uint2 *>((__nv_bfloat16 *)out + (long)t * D + c) = o;
      }
    }
  }
}

}  // namespace

moe_status launch_combine(const MoEConfig &c, int T, const void *y_perm, const int32_t *slot_row,
                          const void *shared_y, void *out, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  int blocks = (T + 7) / 8;
  if (blocks > sms * 16) blocks = sms * 16;
  if (c.out_dtype == MOE_F32)
    combine_kernel<float><<<blocks, 256, 0, s>>>(T, c.hidden_dim, c.top_k, (const float *)y_perm,
                                                 slot_row, (const float *)shared_y, (float *)out);
  else
    combine_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(T, c.hidden_dim, c.top_k,
                                                         (const float *)y_perm, slot_row,
                                                         (const float *)shared_y,
                                                         (__nv_bfloat16 *)out);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
