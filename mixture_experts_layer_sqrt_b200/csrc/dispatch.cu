// Dispatch: group assignments by expert in token order, apply the expert
// capacity, and gather the rows of x into expert-contiguous order.
//
// ops-transformer MoE walkthrough: MoEForward step 3 ("find the tokens routed
// to expert e; Gather") and 坑一 (tokens beyond the expert capacity are
// dropped); Echo MoE quick reference, "Dispatch".
//
// Four kernels, no atomics:
//   hist    one block per chunk of kChunkTokens tokens: per-chunk expert counts
//           (warp match groups into per-warp counter rows, then summed over
//           the warps) -> chunk_cnt[c][e]
//   scan    one block: per expert (a warp each), exclusive scan of chunk_cnt
//           over chunks (in place), total count, kept = min(count, C);
//           offsets = prefix of kept
//   maps    one block per chunk: the rank of each assignment among its
//           expert's assignments in token order (warp match + per-warp
//           running counters), -> slot_row, row_token, row_weight
//   gather  x_perm[r] = x[row_token[r]] with 16-byte vector copies
#include "common.cuh"
#include "kernels.h"

namespace moe {

MOE_VIOLATION_COUNTER(violations_dispatch)

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
static_assert(kChunkTokens == kWarps * 32, "one warp per 32 tokens of a chunk");

// Per-warp expert counts of the warp's 32 tokens (32 * k assignments): each
// round the lanes holding the same expert form a peer group
// (__match_any_sync) and the group's lowest lane adds the group's size to the
// warp's own counter row.  A row belongs to one warp and each round's leaders
// hold distinct experts, so no two lanes ever update one counter at once.
__device__ __forceinline__ void warp_expert_counts(long a0, long a_end, int E, int k,
                                                   const int32_t *__restrict__ topk_idx, int32_t *my, int lane) {
  for (long a = a0; a < a0 + 32L * k; a += 32) {
    long ai = a + lane;
    int e = ai < a_end ? topk_idx[ai] : -1;
    if (e >= E) e = -1;
    unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (__ffs(peers) - 1) == lane) my[e] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kThreads) hist_kernel(int T, int E, int k,
                                                        const int32_t *__restrict__ topk_idx,
                                                        int32_t *__restrict__ chunk_cnt) {
  extern __shared__ int32_t cnt[];  // [kWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * E; i += kThreads) cnt[i] = 0;
  __syncthreads();
  const long a0 = ((long)blockIdx.x * kChunkTokens + warp * 32) * k;
  warp_expert_counts(a0, min((long)T * k, a0 + 32L * k), E, k, topk_idx, cnt + warp * E, lane);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += cnt[w * E + e];
    chunk_cnt[(long)blockIdx.x * E + e] = c;
  }
}

// Block-wide exclusive scan of one int per thread (1024 threads).
__device__ int block_exclusive_scan(int v, int *warp_sums, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sums[lane];
    int wi = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += n;
    }
    warp_sums[lane] = wi - ws;  // exclusive prefix of warp sums
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  int r = warp_sums[warp] + incl - v;
  total = warp_sums[32];
  __syncthreads();
  return r;
}

// Per expert: exclusive scan of its chunk counts over the chunks (in place:
// chunk c's entry becomes the number of e's assignments in chunks < c), the
// total count, kept = min(count, C); then offsets = exclusive prefix of kept.
// One warp per expert walks the chunks 32 at a time (independent loads, a
// warp scan each); one block of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(int n_chunks, int E, int capacity,
                                                    int32_t *__restrict__ chunk_cnt,
                                                    int32_t *__restrict__ expert_counts,
                                                    int32_t *__restrict__ expert_offsets) {
  __shared__ int warp_sums[33];
  extern __shared__ int kept_s[];  // [E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = warp; e < E; e += 32) {
    int run = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < n_chunks ? chunk_cnt[(long)c * E + e] : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
      }
      if (c < n_chunks) chunk_cnt[(long)c * E + e] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      expert_counts[e] = run;
      kept_s[e] = (capacity > 0 && run > capacity) ? capacity : run;
    }
  }
  __syncthreads();
  int carry = 0;
  for (int e0 = 0; e0 < E; e0 += 1024) {
    const int e = e0 + threadIdx.x;
    const int kept = e < E ? kept_s[e] : 0;
    int total;
    int off = block_exclusive_scan(kept, warp_sums, total);
    if (e < E) expert_offsets[e] = carry + off;
    carry += total;
  }
  if (threadIdx.x == 0) expert_offsets[E] = carry;
}

__global__ void __launch_bounds__(kThreads) maps_kernel(int T, int E, int k, int capacity,
                                                        const int32_t *__restrict__ topk_idx,
                                                        const float *__restrict__ topk_w,
                                                        const int32_t *__restrict__ chunk_base,
                                                        const int32_t *__restrict__ expert_offsets,
                                                        int32_t *__restrict__ slot_row,
                                                        int32_t *__restrict__ row_token,
                                                        float *__restrict__ row_weight) {
  extern __shared__ int32_t run[];  // [kWarps][E]: running position per warp and expert
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t *my = run + warp * E;
  for (int i = threadIdx.x; i < kWarps * E; i += kThreads) run[i] = 0;
  __syncthreads();

  // assignments of this warp: tokens [tw, tw + 32), flat items [tw*k, (tw+32)*k)
  const long tw = (long)blockIdx.x * kChunkTokens + warp * 32;
  const long a0 = tw * k;
  const long a_end = min((long)T * k, a0 + 32L * k);
  // pass 1: per-warp counts per expert
  warp_expert_counts(a0, a_end, E, k, topk_idx, my, lane);
  __syncthreads();
  // warps' bases: chunk base + counts of the lower warps of this chunk
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int r = chunk_base[(long)blockIdx.x * E + e];
    for (int w = 0; w < kWarps; ++w) {
      int v = run[w * E + e];
      run[w * E + e] = r;
      r += v;
    }
  }
  __syncthreads();
  // pass 2: position of every assignment within its expert, in token order
  const unsigned lt = (1u << lane) - 1u;
  for (long a = a0; a < a0 + 32L * k; a += 32) {
    long ai = a + lane;
    int e = ai < a_end ? topk_idx[ai] : -1;
    if (e >= E) e = -1;
    unsigned peers = __match_any_sync(0xffffffffu, e);
    if (ai < a_end && e < 0) slot_row[ai] = -1;  // invalid expert index: treated as dropped
    if (e >= 0) {
      int pos = my[e] + __popc(peers & lt);
      if (capacity <= 0 || pos < capacity) {
        int row = expert_offsets[e] + pos;
        slot_row[ai] = row;
        row_token[row] = (int32_t)(ai / k);
        row_weight[row] = topk_w[ai];
      } else {
        slot_row[ai] = -1;
      }
    }
    __syncwarp();
    if (e >= 0 && (__ffs(peers) - 1) == lane) my[e] += __popc(peers);
    __syncwarp();
  }
}

// One warp per row: x_perm[r] = x[row_token[r]], lanes stride over 16-byte vectors.
template <typename TA>
__global__ void __launch_bounds__(256) gather_kernel(int max_rows, int D,
                                                     const int32_t *__restrict__ expert_offsets,
                                                     int E, const int32_t *__restrict__ row_token,
                                                     const TA *__restrict__ x, int src_rows,
                                                     TA *__restrict__ x_perm) {
  constexpr int V = Vec16<TA>::N;
  const int R = min(expert_offsets[E], max_rows);
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += warps) {
    const int tok = row_token[r];
    if (kChecked && (unsigned)tok >= (unsigned)src_rows) {  // whole warp: same row
      if (lane == 0) note_violation();
      continue;
    }
    const TA *src = x + (long)tok * D;
    TA *dst = x_perm + (long)r * D;
#pragma unroll 8
    for (int c = lane * V; c < D; c += 32 * V) store16(dst + c, load16(src + c));
  }
}

// x_perm in f16 with one power-of-two scale per row, for the FP4 gate/up GEMM
// that multiplies in f16: row r holds x[row_token[r]] * 2^s_r, with s_r chosen
// so that the row's largest magnitude lands in [2^14, 2^15), and
// row_scale[r] = 2^-s_r.  Scaling by a power of two is exact; a bf16 value v
// (8 significant bits) is then exact in f16 whenever |v| >= max|row| * 2^-31
// or v = 0, so the GEMM's products equal those of the bf16 operands.
__global__ void __launch_bounds__(256) gather_f16_kernel(int max_rows, int D,
                                                         const int32_t *__restrict__ expert_offsets, int E,
                                                         const int32_t *__restrict__ row_token,
                                                         const __nv_bfloat16 *__restrict__ x, int src_rows,
                                                         __half *__restrict__ x_perm, float *__restrict__ row_scale) {
  constexpr int V = 8;
  const int R = min(expert_offsets[E], max_rows);
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += warps) {
    const int tok = row_token[r];
    if (kChecked && (unsigned)tok >= (unsigned)src_rows) {  // whole warp: same row
      if (lane == 0) note_violation();
      continue;
    }
    const __nv_bfloat16 *src = x + (long)tok * D;
    float m = 0.0f;
#pragma unroll 8
    for (int c = lane * V; c < D; c += 32 * V) {
      const Vec16<__nv_bfloat16> v = load16(src + c);
#pragma unroll
      for (int j = 0; j < V; ++j) m = fmaxf(m, fabsf(v.get(j)));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    // s = 14 - floor(log2 m), from m's exponent field; zero, subnormal or
    // non-finite rows keep s in [-100, 100] so 2^s and 2^-s stay normal floats
    int s = 0;
    if (m > 0.0f) {
      s = 14 - ((int)((__float_as_uint(m) >> 23) & 255u) - 127);
      s = max(-100, min(100, s));
    }
    const float mul = __uint_as_float((uint32_t)(s + 127) << 23);
    __half *dst = x_perm + (long)r * D;
#pragma unroll 8
    for (int c = lane * V; c < D; c += 32 * V) {
      const Vec16<__nv_bfloat16> v = load16(src + c);
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __half2 h2 = __floats2half2_rn(v.get(2 * j) * mul, v.get(2 * j + 1) * mul);
        o[j] = *reinterpret_cast<uint32_t *>(&h2);
      }
      *reinterpret_cast<uint4 *>(dst + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (lane == 0) row_scale[r] = __uint_as_float((uint32_t)(127 - s) << 23);
  }
}

}  // namespace

moe_status launch_gather_f16(const MoEConfig &c, int T, const int32_t *expert_offsets, const int32_t *row_token,
                             const void *x, void *x_perm, float *row_scale, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (c.act_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  gather_f16_kernel<<<sms * 8, 256, 0, s>>>(T * c.top_k, c.hidden_dim, expert_offsets, c.num_experts, row_token,
                                            (const __nv_bfloat16 *)x, T, (__half *)x_perm, row_scale);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_dispatch(const MoEConfig &c, int T, const int32_t *topk_idx, const float *topk_w,
                           const void *x, int32_t *expert_counts, int32_t *expert_offsets,
                           int32_t *slot_row, int32_t *row_token, float *row_weight, void *x_perm,
                           int32_t *chunk_cnt, cudaStream_t s) {
  const int E = c.num_experts, k = c.top_k;
  const int nch = num_chunks(T);
  if (T == 0) {
    // still publish empty counts and offsets
    MOE_CUDA_TRY(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, s));
    MOE_CUDA_TRY(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s));
    return MOE_OK;
  }
  const size_t warp_rows_smem = (size_t)kWarps * E * sizeof(int32_t);  // <= 32 KB (E <= 1024)
  hist_kernel<<<nch, kThreads, warp_rows_smem, s>>>(T, E, k, topk_idx, chunk_cnt);
  MOE_LAUNCH_CHECK();
  scan_kernel<<<1, 1024, E * sizeof(int32_t), s>>>(nch, E, c.expert_capacity, chunk_cnt, expert_counts,
                                                   expert_offsets);
  MOE_LAUNCH_CHECK();
  const size_t maps_smem = warp_rows_smem;
  maps_kernel<<<nch, kThreads, maps_smem, s>>>(T, E, k, c.expert_capacity, topk_idx, topk_w, chunk_cnt,
                                               expert_offsets, slot_row, row_token, row_weight);
  MOE_LAUNCH_CHECK();
  if (!x_perm) return MOE_OK;  // maps only: the GEMM gathers the rows itself
  return launch_gather(c, T, expert_offsets, row_token, x, x_perm, s);
}

moe_status launch_gather(const MoEConfig &c, int T, const int32_t *expert_offsets, const int32_t *row_token,
                         const void *x, void *x_perm, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int max_rows = T * c.top_k, E = c.num_experts;
  if (c.act_dtype == MOE_F32) {
    gather_kernel<float><<<sms * 8, 256, 0, s>>>(max_rows, c.hidden_dim, expert_offsets, E, row_token,
                                                 (const float *)x, T, (float *)x_perm);
  } else {
    gather_kernel<__nv_bfloat16><<<sms * 8, 256, 0, s>>>(max_rows, c.hidden_dim, expert_offsets, E,
                                                         row_token, (const __nv_bfloat16 *)x, T,
                                                         (__nv_bfloat16 *)x_perm);
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
