// Grouped expert GEMMs whose weights stay in NVFP4 (tcgen05 + TMEM + TMA).
//
// "5A · MoE fine-grained" sec. 2 keeps the routed experts of the
// sqrt-softplus layer in FP4: e2m1 codes with one e4m3 scale per 16 weights
// along the reduction axis.  Every product e2m1 * e4m3 has at most 6
// significant bits and lies in the range of bf16 and f16, so expanding a
// weight on chip gives exactly the operand an expanded copy would hold; the
// weights cross HBM once, at 4.5 bits each.
//
// The weights are the MMA's A operand and live in TMEM; the expert's tokens
// are the B operand (N columns) in shared memory:
//
//   gate/up (GATED):  D[128 x N] = [W_gate[e] rows f0..f0+63 ; W_up[e] rows
//                     f0..f0+63] . x_perm[rows r0..r0+N)^T, so TMEM lanes 0..63
//                     hold g and lanes 64..127 hold u of the same 64 h columns
//                     for N tokens; the epilogue forms h = SiLU(clip g) * clip u.
//   down:             D[128 x N] = W_down[e] rows d0..d0+127 . h[rows]^T, fp32
//                     out scaled by each row's routing weight.
//
// Why this shape: an expert's token count varies widely (the sqrt-softplus
// layer's experts get 25..336 of their 128 rows on average), and N can follow
// it in steps of 16, so the MMAs do almost no padded work and every weight is
// expanded once per tile of up to NMAX tokens, instead of once per 128-token
// tile with the tokens on the M side.  Converter warps write the expanded
// weights straight into TMEM (tcgen05.st): shared memory carries only the
// packed codes and the token rows, and the MMAs read only B from it.
//
// Roles (480 threads per CTA):
//   warp 0       token producer: the tile's token rows (boxes of 32 rows x 64
//                columns, or 4-row gathers through a row map) into a 4-stage
//                ring (the rows of an expert are read by all its weight
//                blocks, so they mostly come from L2).
//   warp 14      weight producer: the packed codes ([half][128 rows][16 B])
//                and scales of each k-block into a 16-stage ring.  Every
//                weight block is read once, from HBM, so this ring runs far
//                ahead (16 k-blocks, ~2 us of MMA work) to cover DRAM latency.
//   warp 1       TMEM owner; one thread issues the MMAs (A from a 4-stage TMEM
//                ring, B from the token ring) and commits stages back.  It
//                waits on one barrier per k-block: the converters arrive only
//                after the k-block's token rows have landed as well.
//   warps 2-5    epilogue: TMEM -> registers -> SwiGLU (u handed from the
//                upper lanes to the lower ones through shared memory) or
//                routing weight -> global stores; two accumulators of NMAX
//                columns overlap a tile's epilogue with the next tile's MMAs.
//   warps 6-13   converters: warp w expands the k-blocks of one parity
//                ((w - 6) / 4) for the 32 rows of its TMEM lane quarter
//                (w % 4), all 64 values of a row per k-block, so two k-blocks
//                are in flight per quarter.
//
// F16 (gate/up inside moe_forward): the token rows arrive as f16 scaled by a
// power of two per row (launch_gather_f16), the codes are expanded to f16,
// the MMAs run f16 x f16 -> fp32, and the epilogue undoes the row scale.  All
// three steps are exact, so the result equals the bf16 path's whenever the
// scaled activations are exact in f16.
//
// Tiles never straddle two experts.  An expert with n rows gets
// ceil(n / NMAX) token tiles of equal width (rounded up to 16); the tile list
// (expert-major, then token tile, then weight block) comes from
// expert_offsets on the device.  Every wait is bounded (2 s, then
// MOE_ERR_DEVICE_TIMEOUT in the status word and an orderly wind down).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace moe {

MOE_VIOLATION_COUNTER(violations_gemm_fp4)

namespace {

constexpr int BK = 64;                          // reduction values per k-block
constexpr int UMMA_K = 16;
constexpr int WM = 128;                         // weight rows per tile (MMA M, TMEM lanes)
constexpr int NMAX = 192;                       // token columns per tile at most (MMA N)
constexpr int NBOX = 32;                        // token rows per TMA box
constexpr int B_BYTES = NMAX * BK * 2;          // 24 KB of token rows per stage
constexpr int CODE_BYTES = WM * BK / 2;         // 4 KB: [half][row][16 B]
constexpr int SCL_BYTES = WM * 16;              // 2 KB: [row][16 B] (scales of 4 k-blocks)
constexpr int STAGES = 4;                       // token ring
constexpr int C_STAGES = 16;                    // weight (codes + scales) ring
constexpr int A_STAGES = 4;                     // expanded-weight ring in TMEM
constexpr int kConv = 8;                        // converter warps
constexpr int kConvPerBlock = kConv / 2;        // warps that expand one k-block (one per lane quarter)
constexpr int kWProducerWarp = 6 + kConv;       // the weight producer
constexpr int kThreads = 32 * (kWProducerWarp + 1);
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_COL0 = 2 * NMAX;           // TMEM: acc0 [0,192), acc1 [192,384), A ring [384,512)
constexpr int XPAD = 33;                        // exchange rows padded against bank conflicts
constexpr int MAX_E = 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s
static_assert(A_COL0 + A_STAGES * (BK / 2) == TMEM_COLS, "TMEM budget");
static_assert(NMAX % NBOX == 0 && NMAX % 32 == 0 && NMAX <= 256, "token tile");

struct Smem {
  uint64_t full[STAGES];       // token rows of the k-block landed
  uint64_t empty[STAGES];      // the MMAs reading the stage completed
  uint64_t c_full[C_STAGES];   // codes and scales of the k-block landed
  uint64_t c_empty[C_STAGES];  // the converters read them
  uint64_t a_full[A_STAGES];   // expanded weights of the k-block in TMEM (one arrival per lane quarter)
  uint64_t a_empty[A_STAGES];  // the MMAs reading them completed
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t x_full[2];          // gate/up epilogue: u of a chunk handed over (per warp pair)
  uint64_t x_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[MAX_E + 1];  // over the experts in `order`
  int order[MAX_E];           // experts by token-tile width, widest first
};

struct Params {
  int rows;                  // rows of the output (and of the token matrix unless gathered)
  const int32_t *row_token;  // gathered tokens: row r is src[row_token[r]]; null: dense
  int src_rows;
  int K;                     // reduction length (D for gate/up, F for down)
  int N;                     // output row length (F for gate/up, D for down)
  int E;
  int blocks;                // weight blocks per token tile (F/64 gated, D/128 down)
  const int32_t *offsets;    // [E+1] row offsets, or null: one group of `rows` rows
  void *out;                 // h (bf16) [rows, F] or y (fp32) [rows, D]
  const float *row_weight;   // down only, nullable
  float clamp;
  int clamp_mode;
  int *status;
  uint32_t hi_mul;           // 2^29, passed at run time so the multiply-add stays one instruction
  const float *row_scale;    // F16: 2^-s_r of each token row
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Smem &sm, int *status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait_sleep(bar, parity, ptx::kWaitHintNs)) return true;
    if (*(volatile int *)&sm.abort) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      *(volatile int *)&sm.abort = 1;
      atomicExch(status, kDevTimeout);
      return false;
    }
  }
}

// Used while winding down: copies and MMAs already issued must land first.
__device__ __forceinline__ void drain_bar(uint64_t *bar, uint32_t parity, int *status) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) {
      atomicExch(status, kDevTimeout);
      return;
    }
  }
}

// Warp-uniform wait: lane 0 polls, the outcome is broadcast to the warp.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, Smem &sm, int *status, int lane) {
  bool ok = true;
  if (lane == 0) ok = wait_bar(bar, parity, sm, status);
  return __shfl_sync(0xffffffffu, ok, 0);
}

__device__ __forceinline__ int seg_begin(const Params &p, int e) { return p.offsets ? p.offsets[e] : 0; }
__device__ __forceinline__ int seg_end(const Params &p, int e) {
  int v = p.offsets ? p.offsets[e + 1] : p.rows;
  return v < p.rows ? v : p.rows;
}

// Token tiling of an expert with n rows: tiles of `step` rows (a multiple of
// 16, at most NMAX), ceil(n / step) of them.
__device__ __forceinline__ int token_step(int n) {
  const int nt = (n + NMAX - 1) / NMAX;
  const int per = (n + nt - 1) / nt;
  return (per + 15) & ~15;
}

struct Tile {
  int e, blk;   // expert, weight block
  int r0;       // first token row
  int live;     // token rows of the tile (<= step)
  int n_mma;    // MMA N: live rounded up to 16
};

// Tile t: the largest position j with tile_start[j] <= t (empty experts share
// the next start), expert order[j].
__device__ __forceinline__ Tile decode_tile(const Params &p, const Smem &sm, int t) {
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (sm.tile_start[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int local = t - sm.tile_start[lo];
  const int e = sm.order[lo];
  const int b = seg_begin(p, e), n = seg_end(p, e) - b;
  const int step = token_step(n);
  const int nt = local / p.blocks;
  Tile r;
  r.e = e;
  r.blk = local - nt * p.blocks;
  r.r0 = b + nt * step;
  r.live = min(step, n - nt * step);
  r.n_mma = (r.live + 15) & ~15;
  return r;
}

// The i-th tile of this CTA: rounds of gridDim.x tiles, taken left to right in
// even rounds and right to left in odd ones; -1 past the end.
__device__ __forceinline__ int tile_of(int i, int total) {
  const int g = gridDim.x, b = blockIdx.x;
  const int t = i * g + ((i & 1) ? g - 1 - b : b);
  return t < total ? t : -1;
}

// e4m3 scale byte -> bf16x2 of (scale * 2^112), both halves.  The factor
// 2^112 undoes the exponent offset of the shifted codes below; every e4m3
// value times 2^112 is a normal bf16 with at most 4 significant bits.
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t b) {
  const uint32_t E = (b >> 3) & 15u, m = b & 7u;
  float v;
  if (E == 15u && m == 7u) v = __uint_as_float(0x7fc00000u);          // the NaN code
  else if (E) v = __uint_as_float(((E + 232u) << 23) | (m << 20));     // 2^(E-7) (1 + m/8) 2^112
  else v = (float)m * __uint_as_float(230u << 23);                     // m 2^-9 2^112
  if (b & 0x80u) v = -v;
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  return h | (h << 16);
}

// Eight e2m1 codes times one scale (from scale_bf16x2) -> four bf16x2 words.
// An e2m1 value in f16 has bits only in the sign (15) and in 14..9; moving
// 14..9 down by 3 bits with the sign kept gives the bf16 of the same value
// times 2^-112 (zero stays zero), and its product with the scaled e4m3 has
// at most 6 significant bits, so it is exact.  Words 0-1 re-bias with logic
// ops, words 2-3 with two integer multiply-adds (t >> 3 as the high word of
// t * 2^29) so that both pipes share the work.
__device__ __forceinline__ void expand_e2m1x8_bf16(uint32_t q, uint32_t scale2, uint32_t hi_mul, uint32_t *o) {
  uint32_t h[4];
  ptx::e2m1x8_to_f16x2(q, h);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t v;
    if (j < 2) {
      v = ((h[j] & 0x7FFF7FFFu) >> 3) | (h[j] & 0x80008000u);
    } else {
      const uint32_t t = h[j] & 0x7E007E00u;
      uint32_t sign;
      asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(sign) : "r"(t), "r"(0xFFFFFFFFu), "r"(h[j]));  // h - t
      asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(v) : "r"(t), "r"(hi_mul), "r"(sign));         // (t >> 3) + sign
    }
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&v),
                               *reinterpret_cast<const __nv_bfloat162 *>(&scale2));
    o[j] = *reinterpret_cast<uint32_t *>(&r);
  }
}

// e4m3 scale byte -> f16x2 of the scale, both halves (exact: e4m3 values are
// f16 numbers).
__device__ __forceinline__ uint32_t scale_f16x2(uint32_t b) {
  const uint32_t E = (b >> 3) & 15u, m = b & 7u;
  float v;
  if (E == 15u && m == 7u) v = __uint_as_float(0x7fc00000u);          // the NaN code
  else if (E) v = __uint_as_float(((E + 120u) << 23) | (m << 20));     // 2^(E-7) (1 + m/8)
  else v = (float)m * __uint_as_float(118u << 23);                     // m 2^-9
  if (b & 0x80u) v = -v;
  const uint32_t h = __half_as_ushort(__float2half_rn(v));
  return h | (h << 16);
}

// Eight e2m1 codes times one scale (from scale_f16x2) -> four f16x2 words;
// each product has at most 6 significant bits and lies in [2^-10, 2688]: exact.
__device__ __forceinline__ void expand_e2m1x8_f16(uint32_t q, uint32_t scale2, uint32_t *o) {
  uint32_t h[4];
  ptx::e2m1x8_to_f16x2(q, h);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&h[j]), *reinterpret_cast<const __half2 *>(&scale2));
    o[j] = *reinterpret_cast<uint32_t *>(&r);
  }
}

template <bool GATED, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    tc_fp4_gemm(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW0,
                const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmS0,
                const __grid_constant__ CUtensorMap tmS1, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *stage_b = base;                                   // STAGES x 24 KB (1024-aligned)
  uint8_t *stage_code = stage_b + STAGES * B_BYTES;          // C_STAGES x 4 KB
  uint8_t *stage_scl = stage_code + C_STAGES * CODE_BYTES;   // C_STAGES x 2 KB
  float *xbuf = reinterpret_cast<float *>(stage_scl + C_STAGES * SCL_BYTES);  // 2 pairs x 32 x XPAD
  uint32_t *lut = reinterpret_cast<uint32_t *>(xbuf + 2 * 32 * XPAD);
  Smem &sm = *reinterpret_cast<Smem *>(lut + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- setup: barriers, TMEM, scale table, tile schedule
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&sm.full[s], 1);
      ptx::mbar_init(&sm.empty[s], 1);
    }
    for (int s = 0; s < C_STAGES; ++s) {
      ptx::mbar_init(&sm.c_full[s], 1);
      ptx::mbar_init(&sm.c_empty[s], kConvPerBlock);
    }
    for (int s = 0; s < A_STAGES; ++s) {
      ptx::mbar_init(&sm.a_full[s], kConvPerBlock);
      ptx::mbar_init(&sm.a_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&sm.tmem_full[a], 1);
      ptx::mbar_init(&sm.tmem_empty[a], 4);
      ptx::mbar_init(&sm.x_full[a], 1);
      ptx::mbar_init(&sm.x_empty[a], 1);
    }
    ptx::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW0);
    ptx::prefetch_tmap(&tmS0);
    if (GATED) {
      ptx::prefetch_tmap(&tmW1);
      ptx::prefetch_tmap(&tmS1);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sm.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == 2) {
    // Schedule: experts ordered by token-tile width, widest first (a counting
    // sort over the widths 16..NMAX, stable in e), then tile_start[j] = sum
    // over positions j' < j of (token tiles of order[j']) * blocks.  The CTAs
    // take the tiles in snake order (tile_of), so the long tiles are spread
    // first and the short ones even out the end.
    bool bad = false;  // checked build: offsets must not decrease or start below 0
    int pos = 0;
    for (int w = NMAX / 16; w >= 0; --w) {  // width bucket: step / 16 (0: empty experts)
      for (int e0 = 0; e0 < p.E; e0 += 32) {
        const int e = e0 + lane;
        bool in = false;
        if (e < p.E) {
          if (kChecked && w == 0 && p.offsets && (p.offsets[e] < 0 || p.offsets[e + 1] < p.offsets[e])) bad = true;
          const int n = seg_end(p, e) - seg_begin(p, e);
          in = (n > 0 ? token_step(n) / 16 : 0) == w;
        }
        const unsigned m = __ballot_sync(0xffffffffu, in);
        if (in) sm.order[pos + __popc(m & ((1u << lane) - 1u))] = e;
        pos += __popc(m);
      }
    }
    __syncwarp();
    int carry = 0;
    for (int j0 = 0; j0 < p.E; j0 += 32) {
      const int j = j0 + lane;
      int v = 0;
      if (j < p.E) {
        const int e = sm.order[j];
        const int n = seg_end(p, e) - seg_begin(p, e);
        v = n > 0 ? (n + token_step(n) - 1) / token_step(n) * p.blocks : 0;
      }
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (j < p.E) sm.tile_start[j] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    const bool any_bad = kChecked && __any_sync(0xffffffffu, bad);
    if (any_bad) carry = 0;  // no tiles at all
    if (lane == 0) {
      sm.tile_start[p.E] = carry;
      if (any_bad && blockIdx.x == 0) note_violation();
    }
  }
  if (warp >= 6 && warp < kWProducerWarp) {
    for (int b = (int)threadIdx.x - 192; b < 256; b += 32 * kConv)
      lut[b] = F16 ? scale_f16x2((uint32_t)b) : scale_bf16x2((uint32_t)b);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int total_tiles = sm.tile_start[p.E];
  const int k_blocks = p.K / BK;
  constexpr int W_ROWS = GATED ? WM / 2 : WM;  // rows per weight tensor per tile

  if (warp == 0) {
    // ================================================= TMA producer
    // Dense tokens: lane 0 issues everything.  Gathered tokens: every lane
    // issues 4-row gathers of the tile's rows; lane 0 waits for the stage and
    // issues the rest.
    const bool gather = p.row_token != nullptr;
    if (gather || lane == 0) {
      uint32_t last_parity[STAGES];
      bool used[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) {
        used[s] = false;
        last_parity[s] = 0;
      }
      uint32_t it = 0;
      bool ok = true;
      for (int ti = 0, t; (t = tile_of(ti, total_tiles)) >= 0 && ok; ++ti) {
        const Tile tl = decode_tile(p, sm, t);
        const int n_box = (tl.n_mma + NBOX - 1) / NBOX;
        const uint32_t tx = gather ? tl.n_mma * BK * 2 : n_box * NBOX * BK * 2;
        int tok[2][4];
        if (gather) {
#pragma unroll
          for (int g = 0; g < 2; ++g)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = (lane + 32 * g) * 4 + i;  // token column of the tile
              tok[g][i] = j < tl.live ? p.row_token[tl.r0 + j] : p.src_rows;  // out of range: zero fill
            }
        }
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          bool got = true;
          if (lane == 0) got = wait_bar(&sm.empty[s], ph ^ 1u, sm, p.status);
          if (gather) got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          uint8_t *b = stage_b + s * B_BYTES;
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&sm.full[s], tx);
            if (!gather)
              for (int i = 0; i < n_box; ++i)
                ptx::tma_load_2d(b + i * NBOX * BK * 2, &tmX, &sm.full[s], kb * BK, tl.r0 + i * NBOX);
          }
          if (gather) {
            __syncwarp();
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int q4 = lane + 32 * g;  // 4-row group of the tile
              if (q4 * 4 < tl.n_mma)
                ptx::tma_gather4(b + q4 * 512, &tmX, &sm.full[s], kb * BK, tok[g][0], tok[g][1], tok[g][2],
                                 tok[g][3]);
            }
          }
          used[s] = true;
          last_parity[s] = ph;
        }
      }
      if (lane == 0) {
        for (int s = 0; s < STAGES; ++s)
          if (used[s]) drain_bar(&sm.full[s], last_parity[s], p.status);
      }
    }
  } else if (warp == kWProducerWarp) {
    // ================================================= weight producer
    if (lane == 0) {
      uint32_t last_parity[C_STAGES];
      bool used[C_STAGES];
#pragma unroll
      for (int s = 0; s < C_STAGES; ++s) {
        used[s] = false;
        last_parity[s] = 0;
      }
      uint32_t it = 0;
      bool ok = true;
      for (int ti = 0, t; (t = tile_of(ti, total_tiles)) >= 0 && ok; ++ti) {
        const Tile tl = decode_tile(p, sm, t);
        const int w0 = tl.blk * W_ROWS;  // first weight row of each weight tensor
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C_STAGES;
          const uint32_t ph = (it / C_STAGES) & 1u;
          if (!wait_bar(&sm.c_empty[s], ph ^ 1u, sm, p.status)) {
            ok = false;
            break;
          }
          uint8_t *code = stage_code + s * CODE_BYTES;
          uint8_t *scl = stage_scl + s * SCL_BYTES;
          ptx::mbar_arrive_expect_tx(&sm.c_full[s], CODE_BYTES + SCL_BYTES);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            ptx::tma_load_3d(code + h * (CODE_BYTES / 2), &tmW0, &sm.c_full[s], kb * (BK / 2) + h * 16, w0, tl.e);
            if (GATED)
              ptx::tma_load_3d(code + h * (CODE_BYTES / 2) + W_ROWS * 16, &tmW1, &sm.c_full[s],
                               kb * (BK / 2) + h * 16, w0, tl.e);
          }
          ptx::tma_load_3d(scl, &tmS0, &sm.c_full[s], (kb >> 2) * 16, w0, tl.e);
          if (GATED) ptx::tma_load_3d(scl + W_ROWS * 16, &tmS1, &sm.c_full[s], (kb >> 2) * 16, w0, tl.e);
          used[s] = true;
          last_parity[s] = ph;
        }
      }
      for (int s = 0; s < C_STAGES; ++s)
        if (used[s]) drain_bar(&sm.c_full[s], last_parity[s], p.status);
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      int i = 0;
      bool ok = true;
      for (int t; (t = tile_of(i, total_tiles)) >= 0 && ok; ++i) {
        const Tile tl = decode_tile(p, sm, t);
        const int acc = i & 1;
        if (!wait_bar(&sm.tmem_empty[acc], ((i >> 1) & 1u) ^ 1u, sm, p.status)) break;
        ptx::tc_fence_after();
        const uint32_t idesc = ptx::idesc_f32acc(!F16, WM, tl.n_mma);
        const uint32_t d_tmem = tmem_base + acc * NMAX;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const int as = it % A_STAGES;
          // a_full implies the token stage too: its converters waited for it
          if (!wait_bar(&sm.a_full[as], (it / A_STAGES) & 1u, sm, p.status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t b_addr = ptx::smem_addr(stage_b + s * B_BYTES);
          const uint32_t a_tmem = tmem_base + A_COL0 + as * (BK / 2);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t bd = ptx::desc_kmajor_sw128(b_addr + k * UMMA_K * 2);
            ptx::mma_f16_ts(d_tmem, a_tmem + k * (UMMA_K / 2), bd, idesc, (kb | k) != 0);
          }
          ptx::mma_commit(&sm.empty[s]);
          ptx::mma_commit(&sm.a_empty[as]);
        }
        if (!ok) break;
        ptx::mma_commit(&sm.tmem_full[acc]);
      }
      ptx::mma_commit(&sm.drain);  // all issued MMAs complete before TMEM is released
      drain_bar(&sm.drain, 0, p.status);
    }
  } else if (warp < 6) {
    // ================================================= epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    int i = 0;
    uint32_t xc = 0;  // exchange rounds so far (gate/up)
    for (int t; (t = tile_of(i, total_tiles)) >= 0; ++i) {
      const Tile tl = decode_tile(p, sm, t);
      const int acc = i & 1;
      if (!warp_wait(&sm.tmem_full[acc], (i >> 1) & 1u, sm, p.status, lane)) break;
      ptx::tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + acc * NMAX;
      bool ok = true;
      if (GATED) {
        // lanes 0..63 hold g, 64..127 u, of h columns f0 + (lane % 64)
        const int pair = q & 1;
        float *xb = xbuf + pair * 32 * XPAD;
        const int f = tl.blk * (WM / 2) + pair * 32 + lane;
        for (int c = 0; c < tl.n_mma && ok; c += 32, ++xc) {
          uint32_t v[32];
          ptx::tmem_ld32(tbase + c, v);
          ptx::tmem_ld_wait();
          if (q >= 2) {  // u: hand the chunk to the g warp of the same 32 columns
            if (!warp_wait(&sm.x_empty[pair], (xc & 1u) ^ 1u, sm, p.status, lane)) { ok = false; break; }
#pragma unroll
            for (int j = 0; j < 32; ++j) xb[lane * XPAD + j] = __uint_as_float(v[j]);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.x_full[pair]);
          } else {
            if (!warp_wait(&sm.x_full[pair], xc & 1u, sm, p.status, lane)) { ok = false; break; }
            float u[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) u[j] = xb[lane * XPAD + j];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.x_empty[pair]);
            __nv_bfloat16 *hcol = (__nv_bfloat16 *)p.out + f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c + j < tl.live) {
                const int row = tl.r0 + c + j;
                float g = __uint_as_float(v[j]), uu = u[j];
                if (F16) {
                  const float rs = p.row_scale[row];
                  g *= rs;
                  uu *= rs;
                }
                hcol[(long)row * p.N] = __float2bfloat16_rn(swiglu_h(g, uu, p.clamp, p.clamp_mode));
              }
            }
          }
        }
      } else {
        const int d = tl.blk * WM + q * 32 + lane;
        float *ycol = (float *)p.out + d;
        for (int c = 0; c < tl.n_mma; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(tbase + c, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c + j < tl.live) {
              const int row = tl.r0 + c + j;
              const float rw = p.row_weight ? p.row_weight[row] : 1.0f;
              ycol[(long)row * p.N] = __uint_as_float(v[j]) * rw;
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (!ok) break;
      if (lane == 0) ptx::mbar_arrive(&sm.tmem_empty[acc]);
    }
  } else {
    // ================================================= converters (warps 6..13)
    // Warp w: TMEM lane quarter q = w % 4 (weight rows 32q..32q+31) and the
    // k-blocks of parity (w - 6) / 4 in the common k-block sequence.  A
    // thread reads its row's 32 code bytes (two 16-byte halves; the rows of a
    // half lie 16 bytes apart: conflict-free) and four scales, releases the
    // weight stage, and writes 32 expanded words to 32 TMEM columns.
    const int q = warp & 3, par = (warp - 6) >> 2;
    const int r = q * 32 + lane;
    const uint32_t taddr0 = tmem_base + ((uint32_t)(q * 32) << 16) + A_COL0;
    uint32_t it = 0;
    bool ok = true;
    for (int ti = 0; tile_of(ti, total_tiles) >= 0 && ok; ++ti) {
      for (int kb = 0; kb < k_blocks; ++kb, ++it) {
        if ((int)(it & 1u) != par) continue;
        const int sc = it % C_STAGES;
        const int as = it % A_STAGES;
        bool got = true;
        if (lane == 0) {
          // the codes, a free TMEM stage, and the token rows the MMAs of this
          // k-block will read (so the MMA thread waits on a_full alone)
          got = wait_bar(&sm.c_full[sc], (it / C_STAGES) & 1u, sm, p.status) &&
                wait_bar(&sm.a_empty[as], ((it / A_STAGES) & 1u) ^ 1u, sm, p.status) &&
                wait_bar(&sm.full[it % STAGES], (it / STAGES) & 1u, sm, p.status);
        }
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint8_t *code = stage_code + sc * CODE_BYTES + r * 16;
        const uint4 c0 = *reinterpret_cast<const uint4 *>(code);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(code + CODE_BYTES / 2);
        const uint32_t s4 = *reinterpret_cast<const uint32_t *>(stage_scl + sc * SCL_BYTES + r * 16 + (kb & 3) * 4);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sm.c_empty[sc]);  // codes and scales are in registers
        const uint32_t qw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t sc2 = lut[(s4 >> (8 * (j >> 1))) & 0xFFu];  // 16 values per scale
          if (F16) expand_e2m1x8_f16(qw[j], sc2, w + 4 * j);
          else expand_e2m1x8_bf16(qw[j], sc2, p.hi_mul, w + 4 * j);
        }
        ptx::tmem_st32(taddr0 + as * (BK / 2), w);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sm.a_full[as]);
      }
    }
  }

  // ---- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * B_BYTES + (size_t)C_STAGES * (CODE_BYTES + SCL_BYTES) +
                              2 * 32 * XPAD * sizeof(float) + 256 * sizeof(uint32_t) + sizeof(Smem);
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// tokens: [rows, K] 16-bit (or the gather source); codes [E, Nw, K/2] bytes
// and scales [E, Nw, K/16] bytes for w0/s0 (and w1/s1 when gated).
template <bool GATED, bool F16>
moe_status launch_fp4(const Params &p, const void *x, const void *w0, const void *w1, const void *s0,
                      const void *s1, int Nw, cudaStream_t s) {
  CUtensorMap tx, tw0, tw1, ts0, ts1;
  const uint64_t K = (uint64_t)p.K;
  constexpr uint32_t W_ROWS = GATED ? WM / 2 : WM;
  if (!tma_map_bf16(&tx, x, 2, K, (uint64_t)(p.row_token ? p.src_rows : p.rows), 1, p.row_token ? 1 : NBOX))
    return MOE_ERR_CUDA;
  if (!tma_map_u8(&tw0, w0, K / 2, (uint64_t)Nw, (uint64_t)p.E, 16, W_ROWS)) return MOE_ERR_CUDA;
  if (!tma_map_u8(&ts0, s0, K / 16, (uint64_t)Nw, (uint64_t)p.E, 16, W_ROWS)) return MOE_ERR_CUDA;
  if (GATED) {
    if (!tma_map_u8(&tw1, w1, K / 2, (uint64_t)Nw, (uint64_t)p.E, 16, W_ROWS)) return MOE_ERR_CUDA;
    if (!tma_map_u8(&ts1, s1, K / 16, (uint64_t)Nw, (uint64_t)p.E, 16, W_ROWS)) return MOE_ERR_CUDA;
  } else {
    tw1 = tw0;
    ts1 = ts0;
  }
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  auto kern = tc_fp4_gemm<GATED, F16>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes));
  // every expert has at most ceil(rows_e / 16) / ... token tiles: bound by rows / 16 + E
  const long ub = ((long)(p.rows + NMAX - 1) / NMAX + (p.offsets ? p.E : 1)) * p.blocks;
  if (ub <= 0) return MOE_OK;
  const int grid = (int)(ub < sms ? ub : sms);
  kern<<<grid, kThreads, kSmemBytes, s>>>(tx, tw0, tw1, ts0, ts1, p);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace

bool fp4_direct_ok(const MoEConfig &c, int K) {
  // whole 16-byte TMA strides for the scale rows (K/16 bytes); 64-column h
  // blocks and 128-row W_down blocks
  return c.expert_dtype == MOE_NVFP4 && c.act_dtype == MOE_BF16 && K % 256 == 0 && c.hidden_dim % WM == 0 &&
         c.intermediate_dim % (WM / 2) == 0 && tma_encode_fn() != nullptr;
}

moe_status launch_gate_up_fp4(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                              const int32_t *offsets, const void *w_gate, const void *w_up, const void *s_gate,
                              const void *s_up, const float *row_scale, void *h, int *status, cudaStream_t s) {
  if (rows == 0) return MOE_OK;
  Params p;
  p.rows = rows;
  p.row_token = row_token;
  p.src_rows = row_token ? a_rows : rows;
  p.K = c.hidden_dim;
  p.N = c.intermediate_dim;
  p.E = offsets ? c.num_experts : 1;
  p.blocks = c.intermediate_dim / (WM / 2);
  p.offsets = offsets;
  p.out = h;
  p.row_weight = nullptr;
  p.clamp = c.swiglu_clamp;
  p.clamp_mode = c.clamp_mode;
  p.status = status;
  p.hi_mul = 1u << 29;
  p.row_scale = row_scale;
  if (row_scale) return launch_fp4<true, true>(p, a, w_gate, w_up, s_gate, s_up, c.intermediate_dim, s);
  return launch_fp4<true, false>(p, a, w_gate, w_up, s_gate, s_up, c.intermediate_dim, s);
}

moe_status launch_down_fp4(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                           const void *w_down, const void *s_down, const float *row_weight, float *y,
                           int *status, cudaStream_t s) {
  if (rows == 0) return MOE_OK;
  Params p;
  p.rows = rows;
  p.row_token = nullptr;
  p.src_rows = rows;
  p.K = c.intermediate_dim;
  p.N = c.hidden_dim;
  p.E = offsets ? c.num_experts : 1;
  p.blocks = c.hidden_dim / WM;
  p.offsets = offsets;
  p.out = y;
  p.row_weight = row_weight;
  p.clamp = 0.0f;
  p.clamp_mode = 0;
  p.status = status;
  p.hi_mul = 1u << 29;
  p.row_scale = nullptr;
  return launch_fp4<false, false>(p, h, w_down, nullptr, s_down, nullptr, c.hidden_dim, s);
}

}  // namespace moe
