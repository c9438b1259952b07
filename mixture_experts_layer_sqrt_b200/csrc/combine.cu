// Combine: the routing-weighted sum back to token order (+ the shared expert).
//
// ops-transformer MoE walkthrough, MoEForward step 4 (WeightedSum); Echo MoE
// quick reference, "Combine"; "FFN、SwiGLU 与 MoE" sec. 3 (y = sum_i p_i E_i(x)).
// The weights were applied in the down-projection epilogue, so here
//   out[t] = sum_{j=0..k-1, slot kept} y_perm[slot_row[t, j]]  (+ shared_y[t])
// summed in fp32 in that fixed order: deterministic, no atomics.
//
// One warp per token row, 16-byte streaming loads of the fp32 expert outputs:
// a pure HBM stream of k (+1 shared) rows read and one row written per token.
#include "common.cuh"
#include "kernels.h"

namespace moe {

MOE_VIOLATION_COUNTER(violations_combine)

namespace {

constexpr int kCombineThreads = 128;  // small blocks: every SM holds 16, so the last wave is even

// Streaming (evict-first) 16-byte load and store: y_perm and out are touched once.
__device__ __forceinline__ float4 ld_stream(const float *p) { return __ldcs(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ void st_stream(float *p, float4 v) { __stcs(reinterpret_cast<float4 *>(p), v); }

// kK > 0: the layer's top-k fixed at compile time (rows held in registers, the
// column loop unrolled with every row's load in flight); kK == 0: any k <= 16.
template <typename TOut, int kK>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(int T, int D, int k_rt, int max_row,
                                                                  const float *__restrict__ y_perm,
                                                                  const int32_t *__restrict__ slot_row,
                                                                  const float *__restrict__ shared_y,
                                                                  TOut *__restrict__ out) {
  constexpr int V = 4;  // four fp32 per 16-byte load
  constexpr int kMaxK = kK > 0 ? kK : 16;
  const int k = kK > 0 ? kK : k_rt;
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    // the token's k rows: lane j < k loads slot j, then every lane gets all of them
    int my_row = lane < k ? slot_row[(long)t * k + lane] : -1;
    if (kChecked && my_row >= max_row) {  // rows of y_perm: at most T * k
      note_violation();
      my_row = -1;
    }
    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);
#pragma unroll(kK > 0 && kK <= 4 ? 4 : 1)
    for (int c = lane * V; c < D; c += 32 * V) {
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j < k && rows[j] >= 0) {
          const float4 y = ld_stream(y_perm + (long)rows[j] * D + c);
          acc.x += y.x;
          acc.y += y.y;
          acc.z += y.z;
          acc.w += y.w;
        }
      }
      if (shared_y) {
        const float4 y = ld_stream(shared_y + (long)t * D + c);
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
      }
      if constexpr (sizeof(TOut) == 4) {
        st_stream((float *)out + (long)t * D + c, acc);
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 o = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
        *reinterpret_cast<uint2 *>((__nv_bfloat16 *)out + (long)t * D + c) = o;
      }
    }
  }
}

template <typename TOut>
void launch_combine_k(int k, int blocks, int T, int D, const float *y, const int32_t *slot_row, const float *sh,
                      TOut *out, cudaStream_t s) {
  switch (k) {
    case 1: combine_kernel<TOut, 1><<<blocks, kCombineThreads, 0, s>>>(T, D, k, T * k, y, slot_row, sh, out); break;
    case 2: combine_kernel<TOut, 2><<<blocks, kCombineThreads, 0, s>>>(T, D, k, T * k, y, slot_row, sh, out); break;
    case 4: combine_kernel<TOut, 4><<<blocks, kCombineThreads, 0, s>>>(T, D, k, T * k, y, slot_row, sh, out); break;
    case 6: combine_kernel<TOut, 6><<<blocks, kCombineThreads, 0, s>>>(T, D, k, T * k, y, slot_row, sh, out); break;
    case 8: combine_kernel<TOut, 8><<<blocks, kCombineThreads, 0, s>>>(T, D, k, T * k, y, slot_row, sh, out); break;
    default: combine_kernel<TOut, 0><<<blocks, kCombineThreads, 0, s>>>(T, D, k, T * k, y, slot_row, sh, out); break;
  }
}

}  // namespace

moe_status launch_combine(const MoEConfig &c, int T, const void *y_perm, const int32_t *slot_row,
                          const void *shared_y, void *out, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  constexpr int kWarpsPerBlock = kCombineThreads / 32;
  int blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > sms * 16) blocks = sms * 16;
  if (c.out_dtype == MOE_F32)
    launch_combine_k<float>(c.top_k, blocks, T, c.hidden_dim, (const float *)y_perm, slot_row,
                            (const float *)shared_y, (float *)out, s);
  else
    launch_combine_k<__nv_bfloat16>(c.top_k, blocks, T, c.hidden_dim, (const float *)y_perm, slot_row,
                                    (const float *)shared_y, (__nv_bfloat16 *)out, s);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
