// Grouped expert GEMMs on CUDA cores (fp32 FMA accumulation), any shape.
//
// Used for fp32 layers (the tensor cores' TF32 path cannot meet a 1e-5
// relative error) and for bf16 shapes the tensor-core kernel does not tile.
// Per expert e, rows [off[e], off[e+1]) of A are multiplied by expert e's
// weights ("FFN、SwiGLU 与 MoE" sec. 2: y = W_down[SiLU(W_gate x) * (W_up x)];
// ops-transformer MoE walkthrough 优化三: all experts' rows in one launch).
//
// Tiles are 64x64 outputs per block and never straddle two experts: the
// block's m-tile index is mapped to (expert, first row) by walking the
// per-expert tile counts ceil(rows_e / 64).  The grid carries the upper bound
// ceil(rows / 64) + E m-tiles; blocks past the real count exit at once.
#include "common.cuh"
#include "kernels.h"

namespace moe {

MOE_VIOLATION_COUNTER(violations_gemm_simt)

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename TIn, typename TOut, bool GATED>
__global__ void __launch_bounds__(256) grouped_gemm_simt(int rows, int K, int N,
                                                         const int32_t *__restrict__ offsets, int E,
                                                         const int32_t *__restrict__ row_token,
                                                         int src_rows, const TIn *__restrict__ A,
                                                         const TIn *__restrict__ B0,
                                                         const TIn *__restrict__ B1, float clamp,
                                                         int clamp_mode,
                                                         const float *__restrict__ row_weight,
                                                         TOut *__restrict__ out) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs0[BK][BN + 4];
  __shared__ float Bs1[GATED ? BK : 1][BN + 4];

  // ---- which expert and rows this block owns
  const int mt = blockIdx.x;
  int e = -1, m0 = 0, seg_end = 0;
  if (offsets == nullptr) {
    e = 0;
    m0 = mt * BM;
    seg_end = rows;
    if (m0 >= rows) return;
  } else {
    if (kChecked) {  // offsets must not start below 0 or decrease: otherwise no block does any work
      for (int ee = 0; ee < E; ++ee)
        if (offsets[ee] < 0 || offsets[ee + 1] < offsets[ee]) {
          if (threadIdx.x == 0 && mt == 0 && blockIdx.y == 0) note_violation();
          return;
        }
    }
    int acc = 0;
    for (int ee = 0; ee < E; ++ee) {
      int s0 = offsets[ee], s1 = offsets[ee + 1];
      int nt = (s1 - s0 + BM - 1) / BM;
      if (mt < acc + nt) {
        e = ee;
        m0 = s0 + (mt - acc) * BM;
        seg_end = s1;
        break;
      }
      acc += nt;
    }
    if (e < 0) return;
  }
  seg_end = min(seg_end, rows);
  const int n0 = blockIdx.y * BN;
  const TIn *Be0 = B0 + (long)e * N * K;
  const TIn *Be1 = GATED ? B1 + (long)e * N * K : nullptr;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc0[4][4] = {}, acc1[GATED ? 4 : 1][GATED ? 4 : 1] = {};

  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int q = 0; q < (BM * BK) / 256; ++q) {
      int idx = threadIdx.x + 256 * q;
      int r = idx / BK, kk = idx % BK;
      int gr = m0 + r, gk = k0 + kk;
      long ar = (gr < seg_end && row_token) ? (long)row_token[gr] : (long)gr;  // gathered A row
      bool a_ok = gr < seg_end && gk < K;
      if (kChecked && a_ok && row_token && (unsigned long)ar >= (unsigned long)src_rows) {
        if (kk == 0) note_violation();
        a_ok = false;
      }
      As[kk][r] = a_ok ? to_f32(A[ar * K + gk]) : 0.0f;
      int gn = n0 + r;
      Bs0[kk][r] = (gn < N && gk < K) ? to_f32(Be0[(long)gn * K + gk]) : 0.0f;
      if (GATED) Bs1[kk][r] = (gn < N && gk < K) ? to_f32(Be1[(long)gn * K + gk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b0[j] = Bs0[kk][tx + 16 * j];
        if (GATED) b1[j] = Bs1[kk][tx + 16 * j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (GATED) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int row = m0 + ty + 16 * i;
    if (row >= seg_end) continue;
    float rw = (!GATED && row_weight) ? row_weight[row] : 1.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int col = n0 + tx + 16 * j;
      if (col >= N) continue;
      float v;
      if (GATED) v = swiglu_h(acc0[i][j], acc1[i][j], clamp, clamp_mode);
      else v = acc0[i][j] * rw;
      out[(long)row * N + col] = from_f32<TOut>(v);
    }
  }
}

template <typename TIn, typename TOut, bool GATED>
void launch_one(int rows, int K, int N, const int32_t *offsets, int E, const int32_t *row_token, int src_rows,
                const void *A,
                const void *B0, const void *B1, float clamp, int clamp_mode,
                const float *row_weight, void *out, cudaStream_t s) {
  long mt = (rows + BM - 1) / BM + (offsets ? E : 0);
  dim3 grid((unsigned)mt, (N + BN - 1) / BN);
  grouped_gemm_simt<TIn, TOut, GATED><<<grid, 256, 0, s>>>(rows, K, N, offsets, E, row_token, src_rows,
                                                           (const TIn *)A,
                                                           (const TIn *)B0, (const TIn *)B1, clamp,
                                                           clamp_mode, row_weight, (TOut *)out);
}

}  // namespace

moe_status launch_gate_up_simt(const MoEConfig &c, int rows, const void *a, int a_rows,
                               const int32_t *row_token, const int32_t *offsets, const void *w_gate,
                               const void *w_up, int F, void *h, cudaStream_t s) {
  if (rows == 0) return MOE_OK;
  const int E = offsets ? c.num_experts : 1;
  if (c.act_dtype == MOE_F32)
    launch_one<float, float, true>(rows, c.hidden_dim, F, offsets, E, row_token, a_rows, a, w_gate, w_up,
                                   c.swiglu_clamp, c.clamp_mode, nullptr, h, s);
  else
    launch_one<__nv_bfloat16, __nv_bfloat16, true>(rows, c.hidden_dim, F, offsets, E, row_token, a_rows, a, w_gate,
                                                   w_up, c.swiglu_clamp, c.clamp_mode, nullptr, h, s);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_down_simt(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                            const void *w_down, int F, const float *row_weight, void *y,
                            cudaStream_t s) {
  if (rows == 0) return MOE_OK;
  const int E = offsets ? c.num_experts : 1;
  if (c.act_dtype == MOE_F32)
    launch_one<float, float, false>(rows, F, c.hidden_dim, offsets, E, nullptr, rows, h, w_down, nullptr, 0.0f, 0,
                                    row_weight, y, s);
  else
    launch_one<__nv_bfloat16, float, false>(rows, F, c.hidden_dim, offsets, E, nullptr, rows, h, w_down, nullptr,
                                            0.0f, 0, row_weight, y, s);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
