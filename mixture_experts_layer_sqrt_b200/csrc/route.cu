// Router GEMM + gate + top-k (one kernel).
//
// logits r = W_r x  ("FFN、SwiGLU 与 MoE" sec. 3; ops-transformer MoE walkthrough,
// 优化一), accumulated in fp32 (same walkthrough, 坑三).  Selection is a
// k-round warp argmax (partial selection, not a sort, as in the walkthrough's
// 优化二) with ties to the lower expert index.  Weights: renormalised softmax
// over the selected logits, or the raw sqrt(softplus(s)) gate with the
// selection bias kept out of the weight ("5A · MoE fine-grained" sec. 1, 3).
//
// Work split: a block owns up to 16 consecutive tokens, whose x rows one
// thread brings into shared memory with bulk copies (a whole row per copy, all
// of the block's rows in flight at once).  16 warps then split the work four
// ways by token group and four ways by the reduction: warp w computes 4
// tokens x 8 experts over one interleaved quarter of D (a lane accumulates 32
// partial dot products, x from shared memory, each W_r vector from L1/L2 used
// for all 4 tokens), a 31-shuffle transpose reduction leaves lane l with
// partial sum number l, and the four quarters are added in a fixed order
// through shared memory.  Sixteen warps per SM keep enough independent
// instruction streams to hide the load and FMA latencies that left a
// four-warp version at 0.36 TB/s.  Logits go to shared memory, never to HBM,
// and the token group's first warp selects from there.  (Many experts with bf16 activations use the
// tensor-core router, route_tc.cu.)
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "route_select.cuh"
#include "tc_ptx.cuh"

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

constexpr int kTokPerWarp = 4;
constexpr int kExpChunk = 8;   // kTokPerWarp * kExpChunk = 32 partial sums per lane
constexpr int kDParts = 4;     // warps sharing a token group, each a quarter of D
constexpr uint64_t kRouteWaitNs = 2000000000ull;

// blockDim.x = 32 * groups * kDParts: warp w covers token group w % groups and
// D part w / groups.
template <typename TIn>
__global__ void __launch_bounds__(512) route_kernel(int T, int D, int E, int k, int gate, const TIn *__restrict__ x,
                                                    const TIn *__restrict__ wr, const float *__restrict__ bias,
                                                    const float *__restrict__ bias_vl,
                                                    const uint8_t *__restrict__ image_mask,
                                                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                                    int *status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int V = Vec16<TIn>::N;
  const int groups = (blockDim.x >> 5) / kDParts;
  const int tpb = kTokPerWarp * groups;
  TIn *xs = reinterpret_cast<TIn *>(smem);                                          // [tpb][D]
  float *part = reinterpret_cast<float *>(smem + (size_t)tpb * D * sizeof(TIn));    // [kDParts][tpb][kExpChunk]
  float *logits = part + kDParts * tpb * kExpChunk;                                  // [tpb][E]
  uint64_t *bar = reinterpret_cast<uint64_t *>(((uintptr_t)(logits + (size_t)tpb * E) + 15) & ~(uintptr_t)15);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp % groups, dp = warp / groups;
  const long t0 = (long)blockIdx.x * tpb;
  const int nt = (int)min((long)tpb, (long)T - t0);
  const uint32_t row_bytes = (uint32_t)D * sizeof(TIn);

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar, 1);
    ptx::fence_mbar_init();
    ptx::mbar_arrive_expect_tx(bar, row_bytes * nt);
    for (int i = 0; i < nt; ++i) ptx::bulk_load(xs + (size_t)i * D, x + (t0 + i) * D, row_bytes, bar);
  }
  __syncthreads();
  // every thread waits for the rows (bounded); a timeout is recorded and the
  // whole block leaves before any further barrier
  bool ok = ptx::mbar_try_wait(bar, 0);
  if (!ok) {
    const uint64_t ts = ptx::globaltimer_ns();
    while (!(ok = ptx::mbar_try_wait_sleep(bar, 0, ptx::kWaitHintNs)))
      if (ptx::globaltimer_ns() - ts > kRouteWaitNs) break;
  }
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0 && status) atomicExch(status, kDevTimeout);
    return;
  }

  const int tb = grp * kTokPerWarp;  // this warp's first token within the block
  for (int e0 = 0; e0 < E; e0 += kExpChunk) {
    float acc[32];  // index i * kExpChunk + ee
#pragma unroll
    for (int q = 0; q < 32; ++q) acc[q] = 0.0f;
    for (int d = (dp * 32 + lane) * V; d < D; d += kDParts * 32 * V) {
      Vec16<TIn> xv[kTokPerWarp];
#pragma unroll
      for (int i = 0; i < kTokPerWarp; ++i) {
        if (tb + i < nt) xv[i] = load16(xs + (size_t)(tb + i) * D + d);
        else xv[i].v = {};
      }
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
              float &a = acc[i * kExpChunk + ee];
              a = fmaf(xv[i].get(v), wf, a);
            }
          }
        }
      }
    }
    const float r = transpose_reduce32(acc, lane);  // lane l: token l / 8, expert e0 + l % 8
    part[(dp * tpb + tb) * kExpChunk + lane] = r;
    __syncthreads();
    if (dp == 0) {
      const int i = lane / kExpChunk, e = e0 + lane % kExpChunk;
      float sum = 0.0f;
#pragma unroll
      for (int q = 0; q < kDParts; ++q) sum += part[(q * tpb + tb) * kExpChunk + lane];  // fixed order
      if (e < E && tb + i < nt)
        logits[(tb + i) * E + e] = sum + ((gate == MOE_GATE_SOFTMAX_TOPK_RENORM && bias) ? bias[e] : 0.0f);
    }
    __syncthreads();
  }
  if (dp == 0)
    for (int i = 0; i < kTokPerWarp && tb + i < nt; ++i)
      select_topk(logits + (tb + i) * E, t0 + tb + i, E, k, gate, bias, bias_vl, image_mask, topk_idx, topk_w,
                  lane);
}

// bf16 activations, E <= 32: the logits on the tensor cores with the
// warp-level mma.sync (m16n8k16, bf16 in, fp32 accumulate), so the kernel is
// left with streaming x.  A block owns 8 tokens: one thread bulk-copies their
// x rows into shared memory (rows padded by 16 bytes so the fragment loads of
// the 8 rows fall in different banks), and 4 warps each take every fourth
// 16-wide step of D into two accumulator sets (alternate steps).  The 8
// partial sums per logit (4 warps x 2 sets) are added in a fixed order,
// which keeps each fp32 sum short, as the tensor-core router's split-K
// accumulators do.  Rows 8..15 of every MMA are zero.
constexpr int kMmaTok = 8;
constexpr int kMmaWarps = 4;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int NT>  // expert tiles of 8: ceil(E / 8)
__global__ void __launch_bounds__(32 * kMmaWarps) route_mma_kernel(int T, int D, int E, int k, int gate,
                                                                   const __nv_bfloat16 *__restrict__ x,
                                                                   const __nv_bfloat16 *__restrict__ wr,
                                                                   const float *__restrict__ bias,
                                                                   const float *__restrict__ bias_vl,
                                                                   const uint8_t *__restrict__ image_mask,
                                                                   int32_t *__restrict__ topk_idx,
                                                                   float *__restrict__ topk_w, int *status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int ld = D + 8;  // padded row length in bf16 (16 bytes of padding)
  __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(smem);                      // [kMmaTok][ld]
  float *part = reinterpret_cast<float *>(smem + (size_t)kMmaTok * ld * 2);         // [8 sums][kMmaTok][32]
  float *logits = part + 8 * kMmaTok * 32;                                           // [kMmaTok][E]
  uint64_t *bar = reinterpret_cast<uint64_t *>(((uintptr_t)(logits + kMmaTok * E) + 15) & ~(uintptr_t)15);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const long t0 = (long)blockIdx.x * kMmaTok;
  const int nt = (int)min((long)kMmaTok, (long)T - t0);
  const uint32_t row_bytes = (uint32_t)D * 2;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar, 1);
    ptx::fence_mbar_init();
    ptx::mbar_arrive_expect_tx(bar, row_bytes * nt);
    for (int i = 0; i < nt; ++i) ptx::bulk_load(xs + (size_t)i * ld, x + (t0 + i) * D, row_bytes, bar);
  }
  // rows past the last token read as zeros
  for (int i = nt + warp; i < kMmaTok; i += kMmaWarps)
    for (int j = lane * 8; j < D; j += 32 * 8) *reinterpret_cast<uint4 *>(xs + (size_t)i * ld + j) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  bool ok = ptx::mbar_try_wait(bar, 0);
  if (!ok) {
    const uint64_t ts = ptx::globaltimer_ns();
    while (!(ok = ptx::mbar_try_wait_sleep(bar, 0, ptx::kWaitHintNs)))
      if (ptx::globaltimer_ns() - ts > kRouteWaitNs) break;
  }
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0 && status) atomicExch(status, kDevTimeout);
    return;
  }

  float acc[2][NT][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[h][n][q] = 0.0f;
  const __nv_bfloat16 *xr = xs + (size_t)g * ld + 2 * c;
  // Steps are taken four at a time with every operand load of the four issued
  // before their MMAs (the W_r fragments come from L1/L2, so their latency has
  // to overlap); step j of the warp feeds accumulator set j & 1.
  constexpr int kAhead = 4;
  const int n_steps = (D / 16 - warp + kMmaWarps - 1) / kMmaWarps;  // this warp's 16-wide steps
  int j0 = 0;
  for (; j0 + kAhead <= n_steps; j0 += kAhead) {
    uint32_t a[kAhead][4], b[kAhead][NT][2];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int k0 = (warp + (j0 + u) * kMmaWarps) * 16;
      a[u][0] = *reinterpret_cast<const uint32_t *>(xr + k0);
      a[u][1] = 0u;  // rows 8..15
      a[u][2] = *reinterpret_cast<const uint32_t *>(xr + k0 + 8);
      a[u][3] = 0u;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int e = n * 8 + g;
        b[u][n][0] = b[u][n][1] = 0u;
        if (e < E) {
          const __nv_bfloat16 *wrow = wr + (long)e * D + k0 + 2 * c;
          b[u][n][0] = __ldg(reinterpret_cast<const unsigned int *>(wrow));
          b[u][n][1] = __ldg(reinterpret_cast<const unsigned int *>(wrow + 8));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u)
#pragma unroll
      for (int n = 0; n < NT; ++n) mma_bf16_16816(acc[u & 1][n], a[u], b[u][n][0], b[u][n][1]);  // j0 even: set = u & 1
  }
  for (int j = j0; j < n_steps; ++j) {  // the remaining steps, one at a time
    const int k0 = (warp + j * kMmaWarps) * 16;
    uint32_t a[4];
    a[0] = *reinterpret_cast<const uint32_t *>(xr + k0);
    a[1] = 0u;
    a[2] = *reinterpret_cast<const uint32_t *>(xr + k0 + 8);
    a[3] = 0u;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int e = n * 8 + g;
      uint32_t b0 = 0u, b1 = 0u;
      if (e < E) {
        const __nv_bfloat16 *wrow = wr + (long)e * D + k0 + 2 * c;
        b0 = __ldg(reinterpret_cast<const unsigned int *>(wrow));
        b1 = __ldg(reinterpret_cast<const unsigned int *>(wrow + 8));
      }
      if (j & 1) mma_bf16_16816(acc[1][n], a, b0, b1);
      else mma_bf16_16816(acc[0][n], a, b0, b1);
    }
  }
  // C fragment: d0, d1 = token g, experts n*8 + 2c, 2c + 1 (d2, d3: rows 8..15, unused)
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float *dst = part + ((warp * 2 + h) * kMmaTok + g) * 32 + n * 8 + 2 * c;
      dst[0] = acc[h][n][0];
      dst[1] = acc[h][n][1];
    }
  __syncthreads();
  for (int idx = threadIdx.x; idx < kMmaTok * E; idx += blockDim.x) {
    const int i = idx / E, e = idx - i * E;
    float sum = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) sum += part[(q * kMmaTok + i) * 32 + e];  // fixed order
    logits[i * E + e] = sum + ((gate == MOE_GATE_SOFTMAX_TOPK_RENORM && bias) ? bias[e] : 0.0f);
  }
  __syncthreads();
  for (int i = warp; i < nt; i += kMmaWarps)
    select_topk(logits + i * E, t0 + i, E, k, gate, bias, bias_vl, image_mask, topk_idx, topk_w, lane);
}

}  // namespace

// Token groups per block (4 tokens each): as many as keep a block's x rows
// within 160 KB of shared memory, at most 4 (16 warps).
template <typename TIn>
moe_status launch_route_t(const MoEConfig &c, int T, const void *x, const void *w_router, const float *bias,
                          const float *bias_vl, const uint8_t *image_mask, int32_t *topk_idx, float *topk_w,
                          int *status, cudaStream_t s) {
  const int E = c.num_experts, D = c.hidden_dim;
  const size_t row = (size_t)D * sizeof(TIn);
  int groups = (int)((160 * 1024) / (kTokPerWarp * row));
  if (groups > 4) groups = 4;
  if (groups < 1) return MOE_ERR_UNSUPPORTED;
  const int tpb = kTokPerWarp * groups;
  const size_t smem = (size_t)tpb * row + ((size_t)kDParts * tpb * kExpChunk + (size_t)tpb * E) * sizeof(float) + 32;
  auto kern = route_kernel<TIn>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const dim3 grid((unsigned)((T + tpb - 1) / tpb));
  kern<<<grid, 32 * groups * kDParts, smem, s>>>(T, D, E, c.top_k, c.gate, (const TIn *)x, (const TIn *)w_router, bias, bias_vl,
                                      image_mask, topk_idx, topk_w, status);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_route(const MoEConfig &c, int T, const void *x, const void *w_router,
                        const float *bias, const float *bias_vl, const uint8_t *image_mask,
                        int32_t *topk_idx, float *topk_w, int *status, float *scratch, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (route_tc_ok(c))
    return launch_route_tc(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, status, scratch, s);
  if (c.act_dtype == MOE_F32)
    return launch_route_t<float>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, status, s);
  if (c.num_experts <= 32 && c.hidden_dim % 16 == 0 && (size_t)kMmaTok * (c.hidden_dim + 8) * 2 <= 160 * 1024) {
    const int E = c.num_experts;
    const size_t smem = (size_t)kMmaTok * (c.hidden_dim + 8) * 2 + (8 * kMmaTok * 32 + (size_t)kMmaTok * E) * 4 + 32;
    auto kern = route_mma_kernel<4>;
    switch ((E + 7) / 8) {
      case 1: kern = route_mma_kernel<1>; break;
      case 2: kern = route_mma_kernel<2>; break;
      case 3: kern = route_mma_kernel<3>; break;
      default: break;
    }
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<(unsigned)((T + kMmaTok - 1) / kMmaTok), 32 * kMmaWarps, smem, s>>>(
        T, c.hidden_dim, E, c.top_k, c.gate, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w_router, bias,
        bias_vl, image_mask, topk_idx, topk_w, status);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
  }
  return launch_route_t<__nv_bfloat16>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, status, s);
}

}  // namespace moe
