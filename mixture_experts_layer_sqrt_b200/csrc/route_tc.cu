// Router GEMM + gate + top-k on the tensor cores (bf16 activations, 32 < E <= 512).
//
// logits r = W_r x ("FFN、SwiGLU 与 MoE" sec. 3; ops-transformer MoE walkthrough,
// 优化一) with fp32 accumulation (坑三), then the gate and a partial top-k
// selection (优化二) -- here without a heap and without writing the logits to
// HBM: the tensor-core kernel leaves them in an L2-resident scratch row per
// token and a second kernel selects each token's top-k with one warp (k rounds
// of a warp argmax) on every SM.  Softmax mode: weights
// are the renormalised softmax of the selected (optionally logit-biased)
// logits.  Sqrt mode: selection on s + bias / bias_vl, weights
// sqrt(softplus(s)) of the raw score ("5A · MoE fine-grained" sec. 1, 3).
//
// One CTA per 128 tokens and E_pad experts, 192 threads: warp 0 loads x
// (128 x 64) and the CTA's own W_r rows (E_pad x 64, in equal boxes of up
// to 128 rows) per k-block with TMA; warp 1 issues
// tcgen05.mma (M=128, N <= 256 per instruction, two instructions when
// E_pad > 256) into fp32 TMEM accumulators of E_pad columns -- up to four,
// fed by interleaved k-blocks and summed in a fixed order afterwards, which
// keeps each fp32 sum short.  Warps 2-5 then sum the accumulators of their
// tokens (TMEM lanes) and store the logit rows.  Selecting in this kernel
// leaves one thread per token, 4 warps per 128 tokens, on at most T / 128 SMs;
// the separate selection kernel (a warp per token) spreads it over the GPU.
// Measured at T = 8192: selecting in the epilogue with a register top-k took
// 120 us at E = 384 and 103 us at E = 128, against 90 us and 57 us here.
// All waits bounded.
#include "common.cuh"
#include "kernels.h"
#include "route_select.cuh"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace moe {
namespace {

constexpr int RBM = 128;
constexpr int RBK = 64;
constexpr int kRThreads = 192;
constexpr int kMaxEPad = 512;
constexpr int kMaxStages = 8;
constexpr uint64_t kRWaitNs = 2000000000ull;
constexpr uint64_t kRDrainNs = 200000000ull;

struct RParams {
  int T, D, E;
  int E_pad;  // expert columns of one CTA (a multiple of 16); CTA (x, y) covers [y * E_pad, (y + 1) * E_pad)
  int k, gate, stages, b_rows, w_box;  // W_r rows per stage, and per TMA box
  float *logits;  // [T, ld] fp32 out (router logit bias included in softmax mode)
  int ld;         // logit row stride: E_pad rounded up to whole 32-column chunks
  int n_acc;  // independent accumulators over interleaved k-blocks (shorter fp32 sums)
  uint32_t tmem_cols;
  const float *bias;
  int *status;
};

struct RSmem {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float bias[kMaxEPad];
};

__device__ __forceinline__ bool rwait(uint64_t *bar, uint32_t parity, RSmem &sm, int *status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait_sleep(bar, parity, ptx::kWaitHintNs)) return true;
    if (*(volatile int *)&sm.abort) return false;
    if (ptx::globaltimer_ns() - t0 > kRWaitNs) {
      *(volatile int *)&sm.abort = 1;
      atomicExch(status, kDevTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void rdrain(uint64_t *bar, uint32_t parity, int *status) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > kRDrainNs) {
      atomicExch(status, kDevTimeout);
      return;
    }
  }
}

__global__ void __launch_bounds__(kRThreads, 1)
    tc_route_topk(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, const RParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int a_bytes = RBM * RBK * 2;
  const int b_bytes = p.b_rows * RBK * 2;
  const int stage_bytes = a_bytes + b_bytes;
  RSmem &sm = *reinterpret_cast<RSmem *>(base + (size_t)p.stages * stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * RBM;
  const int e0 = blockIdx.y * p.E_pad;              // this CTA's first expert column
  const int e_cnt = min(p.E_pad, p.E - e0);         // of which real experts

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      ptx::mbar_init(&sm.full[s], 1);
      ptx::mbar_init(&sm.empty[s], 1);
    }
    ptx::mbar_init(&sm.acc_full, 1);
    ptx::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sm.tmem_base, p.tmem_cols);
    ptx::tmem_relinquish();
  }
  if (warp >= 2) {  // router logit bias (softmax mode), added before the logits are stored
    for (int e = threadIdx.x - 64; e < p.E; e += kRThreads - 64)
      sm.bias[e] = (p.bias && p.gate == MOE_GATE_SOFTMAX_TOPK_RENORM) ? p.bias[e] : 0.0f;
  }
  ptx::tc_fence_before();
  __syncwarp();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int k_blocks = p.D / RBK;
  const int n_boxes = p.b_rows / p.w_box;

  if (warp == 0) {
    if (lane == 0) {
      int last = -1;
      for (int kb = 0; kb < k_blocks; ++kb) {
        const int s = kb % p.stages;
        const uint32_t ph = (kb / p.stages) & 1u;
        if (!rwait(&sm.empty[s], ph ^ 1u, sm, p.status)) break;
        ptx::mbar_arrive_expect_tx(&sm.full[s], stage_bytes);
        uint8_t *a = base + (size_t)s * stage_bytes;
        ptx::tma_load_2d(a, &tmX, &sm.full[s], kb * RBK, m0);
        for (int j = 0; j < n_boxes; ++j)
          ptx::tma_load_2d(a + a_bytes + j * p.w_box * 128, &tmW, &sm.full[s], kb * RBK, e0 + j * p.w_box);
        last = kb;
      }
      // drain the copies still in flight (the last `stages` k-blocks)
      for (int kb = last - p.stages + 1; kb <= last; ++kb)
        if (kb >= 0) rdrain(&sm.full[kb % p.stages], (kb / p.stages) & 1u, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const int n0 = p.E_pad < 256 ? p.E_pad : 256;
      const int n1 = p.E_pad - n0;
      const uint32_t id0 = ptx::idesc_bf16_f32(RBM, n0);
      const uint32_t id1 = n1 > 0 ? ptx::idesc_bf16_f32(RBM, n1) : 0u;
      bool ok = true;
      for (int kb = 0; kb < k_blocks; ++kb) {
        const int s = kb % p.stages;
        const uint32_t ph = (kb / p.stages) & 1u;
        if (!rwait(&sm.full[s], ph, sm, p.status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_addr(base + (size_t)s * stage_bytes);
        const uint32_t b_addr = a_addr + a_bytes;
        const int acc = kb % p.n_acc;                       // k-block kb feeds accumulator kb mod n_acc
        const uint32_t d = tmem_base + (uint32_t)(acc * p.E_pad);
        const bool first = kb < p.n_acc;
#pragma unroll
        for (int k = 0; k < RBK / 16; ++k) {
          const uint64_t ad = ptx::desc_kmajor_sw128(a_addr + k * 32);
          ptx::mma_bf16(d, ad, ptx::desc_kmajor_sw128(b_addr + k * 32), id0, !(first && k == 0));
          if (n1 > 0)
            ptx::mma_bf16(d + 256, ad, ptx::desc_kmajor_sw128(b_addr + 256 * 128 + k * 32), id1,
                          !(first && k == 0));
        }
        ptx::mma_commit(&sm.empty[s]);
      }
      if (ok) ptx::mma_commit(&sm.acc_full);
      ptx::mma_commit(&sm.drain);
      rdrain(&sm.drain, 0, p.status);
    }
  } else {
    // ---- logit rows: one token (TMEM lane) per thread
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    bool ok = true;
    if (lane == 0) ok = rwait(&sm.acc_full, 0, sm, p.status);
    if (__shfl_sync(0xffffffffu, ok, 0)) {
      ptx::tc_fence_after();
      const bool live = row < p.T;
      float *dst = p.logits + (long)row * p.ld + e0;  // this CTA's columns [e0, e0 + E_pad) of the row
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16);
      for (int c = 0; c < p.E_pad; c += 32) {
        uint32_t v[32];
        float lsum[32];
        ptx::tmem_ld32(tbase + c, v);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) lsum[j] = __uint_as_float(v[j]);
        for (int a = 1; a < p.n_acc; ++a) {  // fixed order: accumulator 0, 1, ...
          ptx::tmem_ld32(tbase + a * p.E_pad + c, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) lsum[j] += __uint_as_float(v[j]);
        }
        if (live) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            if (c + j >= p.E_pad) break;  // the next CTA's columns
            const float *bb = sm.bias + e0 + c + j;
            float4 o;
            o.x = c + j < e_cnt ? lsum[j] + bb[0] : -INFINITY;
            o.y = c + j + 1 < e_cnt ? lsum[j + 1] + bb[1] : -INFINITY;
            o.z = c + j + 2 < e_cnt ? lsum[j + 2] + bb[2] : -INFINITY;
            o.w = c + j + 3 < e_cnt ? lsum[j + 3] + bb[3] : -INFINITY;
            *reinterpret_cast<float4 *>(dst + c + j) = o;
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// One warp per token: copy its logit row to shared memory, then select with
// each lane's keys cached in registers (NJ = keys per lane, E <= 32 NJ).
constexpr int kSelWarps = 8;
template <int NJ>
__global__ void __launch_bounds__(32 * kSelWarps) route_select_kernel(int T, int E, int ld, int k, int gate,
                                                                     const float *__restrict__ logits,
                                                                     const float *__restrict__ bias,
                                                                     const float *__restrict__ bias_vl,
                                                                     const uint8_t *__restrict__ image_mask,
                                                                     int32_t *__restrict__ topk_idx,
                                                                     float *__restrict__ topk_w) {
  extern __shared__ float rows[];  // [kSelWarps][ld]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *lg = rows + warp * ld;
  for (long t = (long)blockIdx.x * kSelWarps + warp; t < T; t += (long)gridDim.x * kSelWarps) {
    // all of the row's loads in flight at once (one L2 round trip, not NJ)
    const float *src = logits + t * ld;
    float v[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) v[j] = lane + 32 * j < E ? src[lane + 32 * j] : 0.0f;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (lane + 32 * j < E) lg[lane + 32 * j] = v[j];
    __syncwarp();
    select_topk_cached<NJ>(lg, t, E, k, gate, bias, bias_vl, image_mask, topk_idx, topk_w, lane);
    __syncwarp();
  }
}

}  // namespace

// Logit row stride of the tensor-core router: E padded to 16 (the MMA's N
// granularity), then to whole 32-column TMEM load chunks.
static int route_ld(int E) { return ((E + 15) / 16 * 16 + 31) / 32 * 32; }

size_t route_scratch_floats(const MoEConfig &c, int T) {
  return route_tc_ok(c) ? (size_t)T * route_ld(c.num_experts) : 0;
}

// Few experts: one CTA per 128 tokens leaves most SMs idle while it streams x,
// and the CUDA-core router (all SMs) is faster (measured 52 vs 84 us at E=8).
bool route_tc_ok(const MoEConfig &c) {
  return c.act_dtype == MOE_BF16 && c.num_experts > 32 && c.num_experts <= kMaxEPad && c.top_k <= 16 &&
         c.hidden_dim % RBK == 0 && tma_encode_fn() != nullptr;
}

moe_status launch_route_tc(const MoEConfig &c, int T, const void *x, const void *w_router, const float *bias,
                           const float *bias_vl, const uint8_t *image_mask, int32_t *topk_idx, float *topk_w,
                           int *status, float *scratch, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  RParams p;
  p.T = T;
  p.D = c.hidden_dim;
  p.E = c.num_experts;
  // Split the expert columns over 2-4 CTAs per 128 tokens when E allows it
  // (each part a multiple of 16) and the grid still fits in one wave: at a
  // few thousand tokens one CTA per 128 tokens would leave most SMs idle.
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int e_pad_all = (c.num_experts + 15) / 16 * 16;
  const long m_tiles = (T + RBM - 1) / RBM;
  int split = 1;
  for (int sp = 4; sp >= 2; --sp)
    if (e_pad_all % (16 * sp) == 0 && m_tiles * sp <= sms) {
      split = sp;
      break;
    }
  p.E_pad = e_pad_all / split;
  // W_r rows per stage: exactly this CTA's E_pad columns, in at most 8 equal
  // boxes of 128, 64, 32 or 16 rows (else 128-row boxes past E_pad, zero
  // filled beyond E), so that no CTA also loads its neighbour's rows.
  p.w_box = 0;
  for (int b = 128; b >= 16 && !p.w_box; b >>= 1)
    if (p.E_pad % b == 0 && p.E_pad / b <= 8) p.w_box = b;
  if (!p.w_box) p.w_box = 128;
  p.b_rows = (p.E_pad + p.w_box - 1) / p.w_box * p.w_box;
  p.k = c.top_k;
  p.gate = c.gate;
  p.n_acc = p.E_pad <= 128 ? 4 : (p.E_pad <= 256 ? 2 : 1);
  if (p.n_acc > p.D / RBK) p.n_acc = p.D / RBK;
  // the selection reads 32 columns at a time from every accumulator's start
  const uint32_t need = (uint32_t)((p.n_acc - 1) * p.E_pad + (p.E_pad + 31) / 32 * 32);
  uint32_t cols = 32;
  while (cols < need) cols <<= 1;
  p.tmem_cols = cols;
  p.bias = bias;
  p.logits = scratch;
  p.ld = route_ld(c.num_experts);
  p.status = status;
  const int stage_bytes = RBM * RBK * 2 + p.b_rows * RBK * 2;
  int stages = (192 * 1024) / stage_bytes;
  p.stages = stages > kMaxStages ? kMaxStages : stages;
  CUtensorMap tx, tw;
  if (!tma_map_bf16(&tx, x, 2, (uint64_t)p.D, (uint64_t)T, 1)) return MOE_ERR_CUDA;
  if (!tma_map_bf16(&tw, w_router, 2, (uint64_t)p.D, (uint64_t)p.E, 1, (uint32_t)p.w_box)) return MOE_ERR_CUDA;
  const size_t smem = 1024 + (size_t)p.stages * stage_bytes + sizeof(RSmem);
  const dim3 grid((unsigned)m_tiles, (unsigned)split);
  MOE_CUDA_TRY(cudaFuncSetAttribute(tc_route_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  tc_route_topk<<<grid, kRThreads, smem, s>>>(tx, tw, p);
  MOE_LAUNCH_CHECK();
  long sel_blocks = ((long)T + kSelWarps - 1) / kSelWarps;
  if (sel_blocks > (long)sms * 8) sel_blocks = (long)sms * 8;
  const bool sel = c.gate != MOE_GATE_SOFTMAX_TOPK_RENORM;  // softmax: the logit bias is already in the logits
  auto sel_kern = route_select_kernel<16>;  // up to 512 experts
  if (p.E <= 64) sel_kern = route_select_kernel<2>;
  else if (p.E <= 128) sel_kern = route_select_kernel<4>;
  else if (p.E <= 256) sel_kern = route_select_kernel<8>;
  sel_kern<<<(unsigned)sel_blocks, 32 * kSelWarps, (size_t)kSelWarps * p.ld * sizeof(float), s>>>(
      T, p.E, p.ld, p.k, p.gate, scratch, sel ? bias : nullptr, sel ? bias_vl : nullptr, image_mask, topk_idx,
      topk_w);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
