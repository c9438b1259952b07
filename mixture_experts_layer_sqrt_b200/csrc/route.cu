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
// left with streaming x at HBM speed.  A block takes groups of 16 tokens (the
// MMA's 16 rows); a producer warp streams, per 512-wide slice of D, the
// group's 16 x rows and the E router rows into a ring of 4 stages (3 for
// E > 16) with one bulk copy per row issued by its own lane, rows padded by 16 bytes so that ldmatrix reads
// hit 8 different bank groups.  8 consumer warps each take every eighth
// 16-wide step of a slice into two accumulator sets (alternate steps).  A
// stage is released as soon as its reads are done, so the copies of the next
// slices, and of the next group, stay in flight while the tensor cores work.
// At the end of a group the 16 partial sums per logit (8 warps x 2 sets) are
// added in a fixed order, which keeps each fp32 sum short (the routing
// weights are held to 1e-5), and each consumer warp selects for two tokens.
// Rows of the last group past T repeat row T-1 and are never selected.
constexpr int kRGTok = 16;    // tokens per group (MMA rows)
constexpr int kRDC = 512;     // D per stage
template <int NT>
constexpr int route_stages() { return NT <= 2 ? 4 : 3; }  // ring depth within 227 KB of shared memory
constexpr int kRWarps = 8;    // consumer warps; one more warp produces
constexpr int kRRowBytes = (kRDC + 8) * 2;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_addr(p)));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t &r0, uint32_t &r1, const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(ptx::smem_addr(p)));
}

// Bounded wait; gives up at once when the block is aborting.  Waiters sleep
// on the barrier (a suspend-time hint) instead of spinning: measured the same
// (23-25 us for the Mixtral-shaped router either way) with fewer issue slots
// taken from the producer.
__device__ __forceinline__ bool route_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (*abort_flag) return false;
    if (ptx::mbar_try_wait_sleep(bar, parity, ptx::kWaitHintNs)) return true;
    if (ptx::globaltimer_ns() - t0 > kRouteWaitNs) {
      *abort_flag = 1;
      if (status) atomicExch(status, kDevTimeout);
      return false;
    }
  }
}

template <int NT>  // expert tiles of 8: ceil(E / 8)
constexpr size_t route_ring_smem() {
  return (size_t)route_stages<NT>() * (kRGTok + NT * 8) * kRRowBytes + (size_t)2 * kRWarps * kRGTok * NT * 8 * 4 +
         (size_t)kRGTok * NT * 8 * 4 + 2 * route_stages<NT>() * 8 + 16;
}

template <int NT>
__global__ void __launch_bounds__(32 * (kRWarps + 1), 1) route_ring_kernel(int T, int D, int E, int k, int gate,
                                                                     const __nv_bfloat16 *__restrict__ x,
                                                                     const __nv_bfloat16 *__restrict__ wr,
                                                                     const float *__restrict__ bias,
                                                                     const float *__restrict__ bias_vl,
                                                                     const uint8_t *__restrict__ image_mask,
                                                                     int32_t *__restrict__ topk_idx,
                                                                     float *__restrict__ topk_w, int *status) {
  constexpr int kRStages = route_stages<NT>();
  constexpr int ROWS = kRGTok + NT * 8;  // x rows, then router rows, per stage
  constexpr int STAGE = ROWS * kRRowBytes;
  constexpr int EP = NT * 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *stages = smem;
  float *part = reinterpret_cast<float *>(smem + kRStages * STAGE);  // [2 * kRWarps][kRGTok][EP]
  float *logits = part + 2 * kRWarps * kRGTok * EP;                   // [kRGTok][EP]
  uint64_t *full = reinterpret_cast<uint64_t *>(logits + kRGTok * EP);
  uint64_t *empty = full + kRStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kRStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = (T + kRGTok - 1) / kRGTok;
  const int nch = (D + kRDC - 1) / kRDC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kRWarps);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  // router rows E..EP-1 are never copied: zero them in every stage once
  for (int i = threadIdx.x; i < kRStages * (EP - E) * (kRRowBytes / 16); i += blockDim.x) {
    const int per = (EP - E) * (kRRowBytes / 16);
    const int s = i / per, r = (i % per) / (kRRowBytes / 16), c = i % (kRRowBytes / 16);
    *reinterpret_cast<uint4 *>(stages + s * STAGE + (kRGTok + E + r) * kRRowBytes + c * 16) = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  if (warp == kRWarps) {
    // ================================================= producer
    // lane 0 waits for a free stage and expects its bytes; the warp's lanes
    // then issue the row copies side by side (lane i: x row i, lanes 16..:
    // router rows), so no single thread serialises 16 + E copy issues.
    uint32_t it = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < G && ok; g += gridDim.x) {
      for (int c = 0; c < nch; ++c, ++it) {
        const int s = it % kRStages;
        bool got = true;
        if (lane == 0) got = route_wait(&empty[s], ((it / kRStages) & 1u) ^ 1u, abort_flag, status);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const int d0 = c * kRDC, len = min(kRDC, D - d0);
        const uint32_t bytes = (uint32_t)len * 2;
        uint8_t *st = stages + s * STAGE;
        if (lane == 0) ptx::mbar_arrive_expect_tx(&full[s], bytes * (uint32_t)(kRGTok + E));
        __syncwarp();
        for (int r = lane; r < kRGTok + E; r += 32) {
          const __nv_bfloat16 *src;
          if (r < kRGTok) src = x + min((long)g * kRGTok + r, (long)T - 1) * D + d0;
          else src = wr + (long)(r - kRGTok) * D + d0;
          ptx::bulk_load(st + r * kRRowBytes, src, bytes, &full[s]);
        }
      }
    }
    // every issued copy lands before the block's shared memory is released
    if (lane == 0) {
      const uint32_t n_drain = it < (uint32_t)kRStages ? it : (uint32_t)kRStages;
      for (uint32_t j = it - n_drain; j < it; ++j) {
        const uint64_t t0 = ptx::globaltimer_ns();
        while (!ptx::mbar_try_wait(&full[j % kRStages], (j / kRStages) & 1u))
          if (ptx::globaltimer_ns() - t0 > kRouteWaitNs / 10) break;
      }
    }
  } else {
    // ================================================= consumers
    float acc[2][NT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[h][n][q] = 0.0f;
    const int a_row = lane & 15, a_col = (lane >> 4) * 8;        // ldmatrix.x4 row addresses
    const int b_row = lane & 7, b_col = ((lane >> 3) & 1) * 8;   // ldmatrix.x2 (lanes 0-15 used)
    uint32_t it = 0;
    for (int g = blockIdx.x; g < G; g += gridDim.x) {
      for (int c = 0; c < nch; ++c, ++it) {
        const int s = it % kRStages;
        bool ok = true;
        if (lane == 0) ok = route_wait(&full[s], (it / kRStages) & 1u, abort_flag, status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
          const uint8_t *st = stages + s * STAGE;
          const int nk = min(kRDC, D - c * kRDC) / 16;
          for (int j = warp; j < nk; j += kRWarps) {
            uint32_t a[4];
            ldmatrix_x4(a, st + a_row * kRRowBytes + (j * 16 + a_col) * 2);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              uint32_t b0, b1;
              ldmatrix_x2(b0, b1, st + (kRGTok + n * 8 + b_row) * kRRowBytes + (j * 16 + b_col) * 2);
              if ((j / kRWarps) & 1) mma_bf16_16816(acc[1][n], a, b0, b1);
              else mma_bf16_16816(acc[0][n], a, b0, b1);
            }
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[s]);  // release-ordered after this warp's reads
      }
      // C fragment: d0, d1 = row lane / 4, columns 2 (lane % 4) + 0, 1; d2, d3 = row lane / 4 + 8
      const int r0 = lane >> 2, c0 = 2 * (lane & 3);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float *dst = part + ((warp * 2 + h) * kRGTok) * EP + n * 8 + c0;
          dst[r0 * EP] = acc[h][n][0];
          dst[r0 * EP + 1] = acc[h][n][1];
          dst[(r0 + 8) * EP] = acc[h][n][2];
          dst[(r0 + 8) * EP + 1] = acc[h][n][3];
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[h][n][q] = 0.0f;
        }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kRWarps) : "memory");
      for (int idx = threadIdx.x; idx < kRGTok * E; idx += 32 * kRWarps) {
        const int i = idx / E, e = idx - i * E;
        float sum = 0.0f;
#pragma unroll
        for (int q = 0; q < 2 * kRWarps; ++q) sum += part[(q * kRGTok + i) * EP + e];  // fixed order
        logits[i * EP + e] = sum + ((gate == MOE_GATE_SOFTMAX_TOPK_RENORM && bias) ? bias[e] : 0.0f);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kRWarps) : "memory");
      if (!*abort_flag)
        for (int i = warp; i < kRGTok; i += kRWarps) {
          const long t = (long)g * kRGTok + i;
          if (t < T) select_topk(logits + i * EP, t, E, k, gate, bias, bias_vl, image_mask, topk_idx, topk_w, lane);
        }
    }
  }
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
  if (c.num_experts <= 32 && c.hidden_dim % 16 == 0) {
    const int E = c.num_experts, NT = (E + 7) / 8;
    auto kern = route_ring_kernel<4>;
    size_t smem = route_ring_smem<4>();
    switch (NT) {
      case 1: kern = route_ring_kernel<1>; smem = route_ring_smem<1>(); break;
      case 2: kern = route_ring_kernel<2>; smem = route_ring_smem<2>(); break;
      case 3: kern = route_ring_kernel<3>; smem = route_ring_smem<3>(); break;
      default: break;
    }
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    int dev = 0, sms = 148, per_sm = 1;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * (kRWarps + 1), smem));
    if (per_sm < 1) per_sm = 1;
    const long groups = (T + kRGTok - 1) / kRGTok;
    const long cap = (long)sms * per_sm;
    kern<<<(unsigned)(groups < cap ? groups : cap), 32 * (kRWarps + 1), smem, s>>>(
        T, c.hidden_dim, E, c.top_k, c.gate, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w_router, bias,
        bias_vl, image_mask, topk_idx, topk_w, status);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
  }
  return launch_route_t<__nv_bfloat16>(c, T, x, w_router, bias, bias_vl, image_mask, topk_idx, topk_w, status, s);
}

}  // namespace moe
