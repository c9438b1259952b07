// NVFP4 (e2m1 codes + one e4m3 scale per 16 elements) -> bf16 expansion.
//
// The routed experts of the sqrt-softplus layer are stored in FP4 ("5A · MoE
// fine-grained" sec. 2: top-6 of 384 FP4 experts).  Every product
// e2m1 * e4m3 has at most 6 significant bits and lies within bf16's range, so
// the expansion is exact.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// e2m1 magnitude of code bits [2:0]: exponent bits [2:1] (bias 1), mantissa bit [0].
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  float mag = e == 0 ? 0.5f * (float)m : (float)(1u << (e - 1)) * (1.0f + 0.5f * (float)m);
  return (code & 8u) ? -mag : mag;
}

// One thread per 16-element block: 8 packed bytes + 1 scale byte -> 32 bytes of bf16.
__global__ void __launch_bounds__(256) dequant_nvfp4_kernel(long n_blocks,
                                                            const uint2 *__restrict__ packed,
                                                            const uint8_t *__restrict__ scales,
                                                            uint4 *__restrict__ out) {
  for (long b = (long)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks; b += (long)gridDim.x * blockDim.x) {
    uint2 p = packed[b];
    __nv_fp8_e4m3 sc;
    sc.__x = scales[b];
    const float s = (float)sc;
    uint32_t words[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t byte = ((i < 4 ? p.x : p.y) >> (8 * (i & 3))) & 0xFFu;
      float lo = e2m1_value(byte & 0xFu) * s, hi = e2m1_value(byte >> 4) * s;
      uint32_t blo = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
      uint32_t bhi = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
      words[i] = blo | (bhi << 16);
    }
    out[2 * b] = make_uint4(words[0], words[1], words[2], words[3]);
    out[2 * b + 1] = make_uint4(words[4], words[5], words[6], words[7]);
  }
}

}  // namespace

moe_status launch_dequant_nvfp4(const void *packed, const void *scales, long n_elems, void *out,
                                cudaStream_t s) {
  if (n_elems == 0) return MOE_OK;
  long nb = n_elems / 16;
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  long want = (nb + 255) / 256;
  int blocks = (int)(want < (long)sms * 16 ? want : (long)sms * 16);
  dequant_nvfp4_kernel<<<blocks, 256, 0, s>>>(nb, (const uint2 *)packed, (const uint8_t *)scales,
                                              (uint4 *)out);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
