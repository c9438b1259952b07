// Grouped expert GEMMs whose weights stay in NVFP4 (tcgen05 + TMEM + TMA).
//
// "5A · MoE fine-grained" sec. 2 keeps the routed experts of the
// sqrt-softplus layer in FP4: e2m1 codes with one e4m3 scale per 16 weights
// along the reduction axis.  Every product e2m1 * e4m3 has at most 6
// significant bits and lies in bf16's range, so expanding a weight to bf16 on
// chip gives exactly the operand the bf16 GEMM would read from an expanded
// copy; the weights cross HBM once, at 4.5 bits each.
//
//   gate/up (GATED):  D[128 x 256] accumulates x_perm[rows] . [W_gate[e] rows
//                     n0..n0+127 ; W_up[e] rows n0..n0+127]^T; TMEM columns
//                     0..127 hold g and 128..255 hold u of the same h columns.
//   down:             D[128 x 256] = h[rows] . W_down[e][n0..n0+255]^T, rows
//                     scaled by row_weight, fp32 out.
//
// The expansion runs on the CUDA cores (hardware e2m1 -> f16 conversion, an
// exponent re-bias to bf16, one bf16 multiply by the scale; or, for f16, the
// conversion and one f16 multiply) and is balanced between the integer-logic
// and the multiply-add pipes.  N = 256 keeps the MMAs' shared-memory operand
// traffic low; pairs of CTAs are not used because handing a converted
// half-tile to the peer CTA needs a cluster-scope release per k-block, which
// costs more than converting the whole tile locally.
//
// Three rings, because their data have different latencies and lifetimes:
//   A rows      (16 KB per k-block, 3 stages)  mostly L2 hits; held until the
//               MMAs that read them complete.
//   weights     (2 stages, from DRAM)  gate/up: 32 KB of codes in 128-byte
//               swizzled rows + 4 KB of scales per 4 k-blocks; down: 16 KB of
//               codes in 64-byte swizzled rows per 2 k-blocks, the 32 KB saved
//               holding the fp32 epilogue's staging.  Freed as soon as every
//               converter warp holds the bytes in registers.
//   converted B (32 KB per k-block, 3 stages)  written by the converters,
//               held until the MMAs that read it complete.
// With one shared A + weights ring released only after the MMA, gate/up took
// 1.55 ms on the sqrt-softplus layer; now 1.36-1.39.  The k-block period
// (~1200 cycles) is the MMA thread issuing its four MMAs (~740) plus waiting
// for A and for the slowest converter warp; deeper A or converted-B rings
// measured no faster.
//
// Roles (480 threads per CTA):
//   warp 0       TMA producer of A rows (128 x 64 per k-block; or a 4-row
//                gather per lane through a row map).
//   warp 1       TMEM owner; one thread issues the MMAs (A from its ring, B
//                from the converted ring) and commits both stages back.
//   warps 2-5    epilogue: TMEM -> registers -> SwiGLU or routing weight ->
//                global stores (fp32 y through 4 KB of shared memory per
//                warp, so that every store writes whole 128-byte row
//                segments); two 256-column accumulators overlap tiles.
//   warp 6       TMA producer of the packed codes and scales.
//   warps 7-14   converters: codes + scales -> swizzled 16-bit B tile, one
//                arrival per warp.
//
// F16 (inside moe_forward): for gate/up, A arrives as f16 rows pre-scaled by
// a power of two per row (launch_gather_f16), the codes are expanded to f16
// (e2m1 -> f16 needs no re-bias, so one conversion and one f16 multiply per
// pair of weights), the MMAs run f16 x f16 -> fp32, and the epilogue undoes
// the row scale.  All three steps are exact, so g and u equal the bf16
// path's bit for bit whenever the scaled activations are exact in f16.  When
// the SwiGLU clamp bounds |h| below f16's range the epilogue stores h in f16
// (10 fraction bits instead of bf16's 7) and the down projection runs in f16
// as well, without the bf16 re-bias and scale table.
//
// Tiles never straddle two experts; the tile list (expert-major, n-block,
// m-block) comes from expert_offsets on the device.  Every wait is bounded
// (2 s, then MOE_ERR_DEVICE_TIMEOUT in the status word and an orderly wind
// down).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace moe {

MOE_VIOLATION_COUNTER(violations_gemm_fp4)

namespace {

constexpr int BK = 64;                          // one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int TILE_M = 128;                     // rows per tile (TMEM lanes)
constexpr int FN = 256;                         // MMA N: B rows per k-block
constexpr int A_BYTES = TILE_M * BK * 2;        // 16 KB
constexpr int B_BYTES = FN * BK * 2;            // 32 KB
constexpr int SCL_BYTES = FN * 16;              // 4 KB of e4m3 scales (4 k-blocks)

// Per projection: gate/up keeps 4 k-blocks of codes per weight stage
// (128-byte rows); down takes 2 (64-byte rows) and spends the 32 KB saved on
// staging its fp32 epilogue through shared memory (whole-row stores).
template <bool GATED>
struct WCfg {
  static constexpr int KW = GATED ? 4 : 2;                 // k-blocks per weight stage
  static constexpr int W_ROW = KW * BK / 2;                // bytes of codes per B row per stage
  static constexpr int RAW_BYTES = FN * W_ROW;             // codes of a stage (swizzled rows)
  static constexpr int W_BYTES = RAW_BYTES + SCL_BYTES;
  static constexpr int STAGING = GATED ? 0 : 4 * 32 * 32 * 4;  // 4 epilogue warps x 32 x 32 fp32
};
constexpr int A_STAGES = 3;                     // A rows (mostly L2 hits)
constexpr int W_STAGES = 2;                     // codes + scales (DRAM)
constexpr int B_STAGES = 3;                     // converted B tiles
constexpr int kConv = 8;                        // converter warps
constexpr int kWProducer = 6;                   // the weight producer's warp
constexpr int kStagingOffset = 5120;            // epilogue staging, past Smem
constexpr int kConv0 = 7;                       // first converter warp
constexpr int kThreads = 32 * (kConv0 + kConv);
constexpr uint32_t TMEM_COLS = 512;             // 2 accumulators x FN
constexpr int MAX_E = 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s

struct Smem {
  uint64_t a_full[A_STAGES];   // A rows of the k-block landed
  uint64_t a_empty[A_STAGES];  // the MMAs reading them completed
  uint64_t w_full[W_STAGES];   // codes and scales landed
  uint64_t w_empty[W_STAGES];  // every converter warp holds them in registers
  uint64_t b_full[B_STAGES];   // converted B tile written
  uint64_t b_empty[B_STAGES];  // the MMAs reading it completed
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[MAX_E + 1];
};

struct Params {
  int rows;                  // rows of the output (and of A unless gathered)
  const int32_t *row_token;  // gathered A: row r of A is src[row_token[r]]; null: A is dense
  int src_rows;
  int K, N, E, n_tiles;
  const int32_t *offsets;    // [E+1] row offsets, or null: one group of `rows` rows
  void *out;                 // h (bf16) [rows, F] or y (fp32) [rows, D]
  const float *row_weight;   // down only, nullable
  float clamp;
  int clamp_mode;
  int *status;
  uint32_t hi_mul;           // 2^29, passed at run time so the multiply-add stays one
  const float *row_scale;    // F16 gate/up: 2^-s_r of each A row
  int h_f16;                 // F16 gate/up: store h in f16 (else bf16)
};

// Bounded wait.  The hand-offs on the k-block path (the MMA thread's A and B
// waits, the converters' weight and B-stage waits) spin: that path is a chain
// of hand-offs and a suspended waiter wakes late (measured: 5%).  Every other
// waiter (producers on a full ring, the epilogue for a whole tile) sleeps on
// the barrier with a suspend-time hint, so that it takes no issue slots from
// the converter warps.  The clock is read every 64 polls.
template <bool SPIN>
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Smem &sm, int *status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (SPIN ? ptx::mbar_try_wait(bar, parity) : ptx::mbar_try_wait_sleep(bar, parity, ptx::kWaitHintNs)) return true;
    if (SPIN && (n & 63u) != 0) continue;
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
template <bool SPIN>
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, Smem &sm, int *status, int lane) {
  bool ok = true;
  if (lane == 0) ok = wait_bar<SPIN>(bar, parity, sm, status);
  return __shfl_sync(0xffffffffu, ok, 0);
}

__device__ __forceinline__ int seg_begin(const Params &p, int e) { return p.offsets ? p.offsets[e] : 0; }
__device__ __forceinline__ int seg_end(const Params &p, int e) {
  int v = p.offsets ? p.offsets[e + 1] : p.rows;
  return v < p.rows ? v : p.rows;
}

struct Tile {
  int e, m0, end, n_blk;
};

// Largest e with tile_start[e] <= t (empty experts share the next start).
__device__ __forceinline__ Tile decode_tile(const Params &p, const Smem &sm, int t) {
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (sm.tile_start[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int local = t - sm.tile_start[lo];
  const int m_tiles = (sm.tile_start[lo + 1] - sm.tile_start[lo]) / p.n_tiles;
  Tile r;
  r.e = lo;
  r.n_blk = local / m_tiles;
  r.m0 = seg_begin(p, lo) + (local - r.n_blk * m_tiles) * TILE_M;
  r.end = seg_end(p, lo);
  return r;
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

// Eight e2m1 codes times one scale (from scale_bf16x2) -> eight bf16.  An
// e2m1 value in f16 has bits only in the sign (15) and in 14..9; moving
// 14..9 down by 3 bits with the sign kept gives the bf16 of the same value
// times 2^-112 (zero stays zero), and its product with the scaled e4m3 has
// at most 6 significant bits, so it is exact.  Words 0-1 re-bias with logic
// ops, words 2-3 with two integer multiply-adds (t >> 3 as the high word of
// t * 2^29) so that both pipes share the work.
__device__ __forceinline__ uint4 expand_e2m1x8(uint32_t q, uint32_t scale2, uint32_t hi_mul) {
  uint32_t h[4], o[4];
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
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// e4m3 scale byte -> f16x2 of the scale, both halves: the hardware e4m3 pair
// conversion of the byte twice (exact: every e4m3 value, subnormals and the
// NaN code included, is a normal f16 number or NaN).
__device__ __forceinline__ uint32_t scale_f16x2(uint32_t b) {
  uint32_t d;
  const uint16_t two = (uint16_t)(b * 0x0101u);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(two));
  return d;
}

// Eight e2m1 codes times one scale (from scale_f16x2) -> eight f16; each
// product has at most 6 significant bits and lies in [2^-10, 2688]: exact.
__device__ __forceinline__ uint4 expand_e2m1x8_f16(uint32_t q, uint32_t scale2) {
  uint32_t h[4], o[4];
  ptx::e2m1x8_to_f16x2(q, h);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&h[j]), *reinterpret_cast<const __half2 *>(&scale2));
    o[j] = *reinterpret_cast<uint32_t *>(&r);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool GATED, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    tc_fp4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmS0,
                const __grid_constant__ CUtensorMap tmS1, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *stage_a = base;                                  // A_STAGES x 16 KB (1024-aligned)
  uint8_t *stage_b = stage_a + A_STAGES * A_BYTES;          // B_STAGES x 32 KB
  uint8_t *stage_w = stage_b + B_STAGES * B_BYTES;          // W_STAGES x (32 KB codes + 4 KB scales)
  using WC = WCfg<GATED>;
  constexpr int KW = WC::KW, W_ROW = WC::W_ROW, RAW_BYTES = WC::RAW_BYTES, W_BYTES = WC::W_BYTES;
  uint32_t *lut = reinterpret_cast<uint32_t *>(stage_w + W_STAGES * W_BYTES);
  Smem &sm = *reinterpret_cast<Smem *>(stage_w + W_STAGES * W_BYTES + 1024);
  float *staging = reinterpret_cast<float *>(stage_w + W_STAGES * W_BYTES + 1024 + kStagingOffset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- setup: barriers, TMEM, scale table, tile schedule
  if (threadIdx.x == 0) {
    for (int s = 0; s < A_STAGES; ++s) {
      ptx::mbar_init(&sm.a_full[s], 1);
      ptx::mbar_init(&sm.a_empty[s], 1);
    }
    for (int s = 0; s < W_STAGES; ++s) {
      ptx::mbar_init(&sm.w_full[s], 1);
      ptx::mbar_init(&sm.w_empty[s], kConv);
    }
    for (int b = 0; b < B_STAGES; ++b) {
      ptx::mbar_init(&sm.b_full[b], kConv);
      ptx::mbar_init(&sm.b_empty[b], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&sm.tmem_full[a], 1);
      ptx::mbar_init(&sm.tmem_empty[a], 4);
    }
    ptx::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == kWProducer && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB0);
    ptx::prefetch_tmap(&tmS0);
    if (GATED) {
      ptx::prefetch_tmap(&tmB1);
      ptx::prefetch_tmap(&tmS1);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sm.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (warp == 2) {
    // tile_start[e] = sum over e' < e of ceil(rows_e' / TILE_M) * n_tiles
    int carry = 0;
    bool bad = false;  // checked build: offsets must not decrease or start below 0
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      int v = 0;
      if (e < p.E) {
        if (kChecked && p.offsets && (p.offsets[e] < 0 || p.offsets[e + 1] < p.offsets[e])) bad = true;
        const int n = seg_end(p, e) - seg_begin(p, e);
        v = n > 0 ? (n + TILE_M - 1) / TILE_M * p.n_tiles : 0;
      }
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (e < p.E) sm.tile_start[e] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    const bool any_bad = kChecked && __any_sync(0xffffffffu, bad);
    if (any_bad) carry = 0;  // no tiles at all
    if (lane == 0) {
      sm.tile_start[p.E] = carry;
      if (any_bad && blockIdx.x == 0) note_violation();
    }
  }
  if (!F16 && warp >= kConv0) {
    for (int b = (int)threadIdx.x - 32 * kConv0; b < 256; b += 32 * kConv) lut[b] = scale_bf16x2((uint32_t)b);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int total_tiles = sm.tile_start[p.E];
  const int k_blocks = p.K / BK;

  if (warp == 0) {
    // ================================================= TMA producer: A rows
    // Dense A: lane 0 issues the 128-row box.  Gathered A: each lane gathers
    // its 4 rows of the tile (one 4-row TMA gather per k-block).
    const bool gather = p.row_token != nullptr;
    if (gather || lane == 0) {
      uint32_t last_parity[A_STAGES];
      bool used[A_STAGES];
#pragma unroll
      for (int s = 0; s < A_STAGES; ++s) {
        used[s] = false;
        last_parity[s] = 0;
      }
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile(p, sm, t);
        int tok[4];
        if (gather) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = tl.m0 + lane * 4 + i;
            tok[i] = r < tl.end ? p.row_token[r] : p.src_rows;  // out of range: zero fill
          }
        }
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % A_STAGES;
          const uint32_t ph = (it / A_STAGES) & 1u;
          bool got = true;
          if (lane == 0) got = wait_bar<false>(&sm.a_empty[s], ph ^ 1u, sm, p.status);
          if (gather) got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          uint8_t *a = stage_a + s * A_BYTES;
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&sm.a_full[s], A_BYTES);
            if (!gather) ptx::tma_load_2d(a, &tmA, &sm.a_full[s], kb * BK, tl.m0);
          }
          if (gather) ptx::tma_gather4(a + lane * 512, &tmA, &sm.a_full[s], kb * BK, tok[0], tok[1], tok[2], tok[3]);
          used[s] = true;
          last_parity[s] = ph;
        }
      }
      if (lane == 0) {
        for (int s = 0; s < A_STAGES; ++s)
          if (used[s]) drain_bar(&sm.a_full[s], last_parity[s], p.status);
      }
    }
  } else if (warp == kWProducer) {
    // ================================================= TMA producer: weights
    // Per stage, four k-blocks: packed codes (256 B rows x 128 bytes, 128-byte
    // swizzle) and their scales (256 x 16 bytes).  The TMA's cost goes with
    // the rows it moves, so rows as wide as the swizzle allows, one stage per
    // four k-blocks; the converters free a stage as soon as they hold its
    // last k-block's bytes in registers.
    if (lane == 0) {
      uint32_t last_parity[W_STAGES];
      bool used[W_STAGES];
#pragma unroll
      for (int s = 0; s < W_STAGES; ++s) {
        used[s] = false;
        last_parity[s] = 0;
      }
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile(p, sm, t);
        const int n0 = GATED ? tl.n_blk * (FN / 2) : tl.n_blk * FN;
        const int n1 = GATED ? n0 : n0 + FN / 2;
        for (int kw = 0; kw < k_blocks / KW; ++kw, ++it) {
          const int s = it % W_STAGES;
          const uint32_t ph = (it / W_STAGES) & 1u;
          if (!wait_bar<false>(&sm.w_empty[s], ph ^ 1u, sm, p.status)) {
            ok = false;
            break;
          }
          uint8_t *raw = stage_w + s * W_BYTES;
          uint8_t *scl = raw + RAW_BYTES;
          ptx::mbar_arrive_expect_tx(&sm.w_full[s], W_BYTES);
          const int sx = (kw * KW >> 2) * 16;  // the scale box covers 4 k-blocks
          ptx::tma_load_3d(raw, &tmB0, &sm.w_full[s], kw * W_ROW, n0, tl.e);
          ptx::tma_load_3d(raw + RAW_BYTES / 2, GATED ? &tmB1 : &tmB0, &sm.w_full[s], kw * W_ROW, n1, tl.e);
          ptx::tma_load_3d(scl, &tmS0, &sm.w_full[s], sx, n0, tl.e);
          ptx::tma_load_3d(scl + SCL_BYTES / 2, GATED ? &tmS1 : &tmS0, &sm.w_full[s], sx, n1, tl.e);
          used[s] = true;
          last_parity[s] = ph;
        }
      }
      for (int s = 0; s < W_STAGES; ++s)
        if (used[s]) drain_bar(&sm.w_full[s], last_parity[s], p.status);
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = F16 ? ptx::idesc_f16_f32(TILE_M, FN) : ptx::idesc_bf16_f32(TILE_M, FN);
      uint32_t it = 0;
      int i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++i) {
        const int acc = i & 1;
        if (!wait_bar<false>(&sm.tmem_empty[acc], ((i >> 1) & 1u) ^ 1u, sm, p.status)) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % A_STAGES;
          const int sb = it % B_STAGES;
          if (!wait_bar<true>(&sm.a_full[s], (it / A_STAGES) & 1u, sm, p.status) ||
              !wait_bar<true>(&sm.b_full[sb], (it / B_STAGES) & 1u, sm, p.status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_addr(stage_a + s * A_BYTES);
          const uint32_t b_addr = ptx::smem_addr(stage_b + sb * B_BYTES);
          const uint32_t d_tmem = tmem_base + acc * FN;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = ptx::desc_kmajor_sw128(a_addr + k * UMMA_K * 2);
            const uint64_t bd = ptx::desc_kmajor_sw128(b_addr + k * UMMA_K * 2);
            ptx::mma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          ptx::mma_commit(&sm.a_empty[s]);
          ptx::mma_commit(&sm.b_empty[sb]);
        }
        if (!ok) break;
        ptx::mma_commit(&sm.tmem_full[acc]);
      }
      ptx::mma_commit(&sm.drain);  // all issued MMAs complete before TMEM is released
      drain_bar(&sm.drain, 0, p.status);
    }
  } else if (warp < 6) {
    // ================================================= epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    int i = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++i) {
      const Tile tl = decode_tile(p, sm, t);
      const int acc = i & 1;
      if (!warp_wait<false>(&sm.tmem_full[acc], (i >> 1) & 1u, sm, p.status, lane)) break;
      ptx::tc_fence_after();
      const int row = tl.m0 + q * 32 + lane;
      const bool live = row < tl.end;
      const uint32_t tbase = tmem_base + lane_addr + acc * FN;
      if (tl.m0 + q * 32 < tl.end) {  // warp-uniform: some row of this quarter is live
        if (GATED) {
          __nv_bfloat16 *hrow = (__nv_bfloat16 *)p.out + (long)row * p.N + tl.n_blk * (FN / 2);
          const float rs = (F16 && live) ? p.row_scale[row] : 1.0f;
#pragma unroll 1
          for (int c = 0; c < FN / 2; c += 32) {
            uint32_t g[32], u[32];
            ptx::tmem_ld32(tbase + c, g);
            ptx::tmem_ld32(tbase + FN / 2 + c, u);
            ptx::tmem_ld_wait();
            if (live) {
              uint32_t pk[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                float g0 = __uint_as_float(g[2 * j]), u0 = __uint_as_float(u[2 * j]);
                float g1 = __uint_as_float(g[2 * j + 1]), u1 = __uint_as_float(u[2 * j + 1]);
                if (F16) {
                  g0 *= rs;
                  u0 *= rs;
                  g1 *= rs;
                  u1 *= rs;
                }
                const float h0 = swiglu_h(g0, u0, p.clamp, p.clamp_mode);
                const float h1 = swiglu_h(g1, u1, p.clamp, p.clamp_mode);
                if (F16 && p.h_f16) {
                  __half2 f2 = __floats2half2_rn(h0, h1);
                  pk[j] = *reinterpret_cast<uint32_t *>(&f2);
                } else {
                  __nv_bfloat162 b2 = __floats2bfloat162_rn(h0, h1);
                  pk[j] = *reinterpret_cast<uint32_t *>(&b2);
                }
              }
              uint4 *dst = reinterpret_cast<uint4 *>(hrow + c);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
          }
        } else {
          // each 32 x 32 fp32 chunk through this warp's 4 KB of shared memory
          // (row r's 16-byte piece j at j ^ (r % 8)), so that every global
          // store writes four whole 128-byte row segments
          const float rw = (live && p.row_weight) ? p.row_weight[row] : 1.0f;
          float *stg = staging + q * 32 * 32;
          const int row0 = tl.m0 + q * 32;
          const int rr = lane >> 3, ff = lane & 7;
          const int ncol0 = tl.n_blk * FN;
#pragma unroll 1
          for (int c = 0; c < FN; c += 32) {
            uint32_t v[32];
            ptx::tmem_ld32(tbase + c, v);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4 *>(stg + lane * 32 + ((j ^ (lane & 7)) << 2)) =
                  make_float4(__uint_as_float(v[4 * j]) * rw, __uint_as_float(v[4 * j + 1]) * rw,
                              __uint_as_float(v[4 * j + 2]) * rw, __uint_as_float(v[4 * j + 3]) * rw);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + rr;
              const float4 val = *reinterpret_cast<const float4 *>(stg + r * 32 + ((ff ^ (r & 7)) << 2));
              if (row0 + r < tl.end)
                *reinterpret_cast<float4 *>((float *)p.out + (long)(row0 + r) * p.N + ncol0 + c + ff * 4) = val;
            }
            __syncwarp();
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sm.tmem_empty[acc]);
    }
  } else if (warp >= kConv0) {
    // ================================================= converters (kConv warps)
    // Per k-block 256 B rows x 4 groups of 16 codes, one e4m3 scale each:
    // thread ct takes group ct % 4 of rows ct / 4 + 64 j.  A group is one
    // 8-byte load of codes, one scale conversion and two 16-byte stores into
    // the swizzled tile (chunk c of row r at 16 * (c ^ (r % 8))); a warp's
    // stores cover 8 whole 128-byte rows, four wavefronts each, the minimum.
    // Codes of k-block kb: bytes 32 (kb % 4) .. +31 of each 128-byte row,
    // stored swizzled (16-byte chunk c of row r at chunk c ^ (r % 8)), so a
    // warp's 8 rows read different banks.  The weight stage is released once
    // its fourth k-block's bytes are in registers.
    constexpr int ROWS_PER_PASS = 32 * kConv / 4;
    constexpr int JOBS = FN / ROWS_PER_PASS;
    const int ct = (int)threadIdx.x - 32 * kConv0;
    const int g = ct & 3, r0 = ct >> 2;
    const int scl_off = RAW_BYTES + r0 * 16 + g;
    const int b_off0 = r0 * (BK * 2) + (((2 * g) ^ (r0 & 7)) << 4);
    const int b_off1 = r0 * (BK * 2) + (((2 * g + 1) ^ (r0 & 7)) << 4);
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < k_blocks; ++kb, ++it) {
        const uint32_t iw = it / KW;  // weight stages so far (every tile starts a stage: k_blocks % KW == 0)
        const int sw = iw % W_STAGES;
        const int sb = it % B_STAGES;
        const int kq = kb & (KW - 1);
        if (kq == 0 && !warp_wait<true>(&sm.w_full[sw], (iw / W_STAGES) & 1u, sm, p.status, lane)) {
          ok = false;
          break;
        }
        const uint8_t *w = stage_w + sw * W_BYTES;
        // the group's 16-byte chunk, swizzled as the TMA stored it
        const int chunk = 2 * kq + (g >> 1);
        const int raw_off = r0 * W_ROW + ((KW == 4 ? chunk ^ (r0 & 7) : chunk ^ ((r0 >> 1) & 3)) << 4) + (g & 1) * 8;
        uint2 qv[JOBS];
        uint32_t sc[JOBS];
#pragma unroll
        for (int j = 0; j < JOBS; ++j) {
          qv[j] = *reinterpret_cast<const uint2 *>(w + raw_off + j * ROWS_PER_PASS * W_ROW);
          sc[j] = w[scl_off + (kb & 3) * 4 + j * ROWS_PER_PASS * 16];
        }
        if (kq == KW - 1) {
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sm.w_empty[sw]);  // release-ordered after the loads above
        }
#pragma unroll
        for (int j = 0; j < JOBS; ++j) sc[j] = F16 ? scale_f16x2(sc[j]) : lut[sc[j]];
        if (!warp_wait<true>(&sm.b_empty[sb], ((it / B_STAGES) & 1u) ^ 1u, sm, p.status, lane)) {
          ok = false;
          break;
        }
        uint8_t *dst = stage_b + sb * B_BYTES;
#pragma unroll
        for (int j = 0; j < JOBS; ++j) {
          const int rb = j * ROWS_PER_PASS * (BK * 2);  // ROWS_PER_PASS % 8 == 0: the swizzle phase is kept
          *reinterpret_cast<uint4 *>(dst + b_off0 + rb) =
              F16 ? expand_e2m1x8_f16(qv[j].x, sc[j]) : expand_e2m1x8(qv[j].x, sc[j], p.hi_mul);
          *reinterpret_cast<uint4 *>(dst + b_off1 + rb) =
              F16 ? expand_e2m1x8_f16(qv[j].y, sc[j]) : expand_e2m1x8(qv[j].y, sc[j], p.hi_mul);
        }
        ptx::fence_proxy_async_smem();  // the MMA reads these stores through the async proxy
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sm.b_full[sb]);
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

template <bool GATED>
constexpr size_t fp4_smem_bytes() {
  return 1024 + (size_t)A_STAGES * A_BYTES + (size_t)B_STAGES * B_BYTES + (size_t)W_STAGES * WCfg<GATED>::W_BYTES +
         1024 + kStagingOffset + WCfg<GATED>::STAGING;
}
static_assert(sizeof(Smem) <= kStagingOffset, "the epilogue staging follows the barriers and tile list");
static_assert(fp4_smem_bytes<true>() <= 232448 && fp4_smem_bytes<false>() <= 232448, "shared memory per CTA");

// A: [rows, K] bf16 (or the gather source); codes [E, Nw, K/2] bytes and
// scales [E, Nw, K/16] bytes for b0/s0 (and b1/s1 when gated).
template <bool GATED, bool F16>
moe_status launch_fp4(const Params &p, const void *a, const void *b0, const void *b1, const void *s0,
                      const void *s1, int Nw, cudaStream_t s) {
  CUtensorMap ta, tb0, tb1, ts0, ts1;
  const uint64_t K = (uint64_t)p.K;
  if (!tma_map_bf16(&ta, a, 2, K, (uint64_t)(p.row_token ? p.src_rows : p.rows), 1, p.row_token ? 1 : TILE_M))
    return MOE_ERR_CUDA;
  constexpr int W_ROW = WCfg<GATED>::W_ROW;
  if (!tma_map_u8(&tb0, b0, K / 2, (uint64_t)Nw, (uint64_t)p.E, W_ROW, FN / 2, W_ROW)) return MOE_ERR_CUDA;
  if (!tma_map_u8(&ts0, s0, K / 16, (uint64_t)Nw, (uint64_t)p.E, 16, FN / 2)) return MOE_ERR_CUDA;
  if (GATED) {
    if (!tma_map_u8(&tb1, b1, K / 2, (uint64_t)Nw, (uint64_t)p.E, W_ROW, FN / 2, W_ROW)) return MOE_ERR_CUDA;
    if (!tma_map_u8(&ts1, s1, K / 16, (uint64_t)Nw, (uint64_t)p.E, 16, FN / 2)) return MOE_ERR_CUDA;
  } else {
    tb1 = tb0;
    ts1 = ts0;
  }
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  auto kern = tc_fp4_gemm<GATED, F16>;
  constexpr size_t kSmemBytes = fp4_smem_bytes<GATED>();
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes));
  const long ub = ((long)(p.rows + TILE_M - 1) / TILE_M + (p.offsets ? p.E : 0)) * p.n_tiles;  // tile bound
  if (ub <= 0) return MOE_OK;
  const int grid = (int)(ub < sms ? ub : sms);
  kern<<<grid, kThreads, kSmemBytes, s>>>(ta, tb0, tb1, ts0, ts1, p);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace

bool fp4_direct_ok(const MoEConfig &c, int K) {
  // whole 16-byte TMA strides for the scale rows (K/16 bytes); 128-column h
  // tiles and 256-column y tiles
  return c.expert_dtype == MOE_NVFP4 && c.act_dtype == MOE_BF16 && K % 256 == 0 && c.hidden_dim % FN == 0 &&
         c.intermediate_dim % (FN / 2) == 0 && tma_encode_fn() != nullptr;
}

moe_status launch_gate_up_fp4(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                              const int32_t *offsets, const void *w_gate, const void *w_up, const void *s_gate,
                              const void *s_up, const float *row_scale, void *h, int *status, cudaStream_t s,
                              bool h_f16) {
  if (rows == 0) return MOE_OK;
  Params p;
  p.rows = rows;
  p.row_token = row_token;
  p.src_rows = row_token ? a_rows : rows;
  p.K = c.hidden_dim;
  p.N = c.intermediate_dim;
  p.E = offsets ? c.num_experts : 1;
  p.n_tiles = c.intermediate_dim / (FN / 2);
  p.offsets = offsets;
  p.out = h;
  p.row_weight = nullptr;
  p.clamp = c.swiglu_clamp;
  p.clamp_mode = c.clamp_mode;
  p.status = status;
  p.hi_mul = 1u << 29;
  p.row_scale = row_scale;
  p.h_f16 = row_scale && h_f16 ? 1 : 0;
  if (row_scale) return launch_fp4<true, true>(p, a, w_gate, w_up, s_gate, s_up, c.intermediate_dim, s);
  return launch_fp4<true, false>(p, a, w_gate, w_up, s_gate, s_up, c.intermediate_dim, s);
}

moe_status launch_down_fp4(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                           const void *w_down, const void *s_down, const float *row_weight, float *y,
                           int *status, cudaStream_t s, bool h_f16) {
  if (rows == 0) return MOE_OK;
  Params p;
  p.rows = rows;
  p.row_token = nullptr;
  p.src_rows = rows;
  p.K = c.intermediate_dim;
  p.N = c.hidden_dim;
  p.E = offsets ? c.num_experts : 1;
  p.n_tiles = c.hidden_dim / FN;
  p.offsets = offsets;
  p.out = y;
  p.row_weight = row_weight;
  p.clamp = 0.0f;
  p.clamp_mode = 0;
  p.status = status;
  p.hi_mul = 1u << 29;
  p.row_scale = nullptr;
  p.h_f16 = 0;
  if (h_f16) return launch_fp4<false, true>(p, h, w_down, nullptr, s_down, nullptr, c.hidden_dim, s);
  return launch_fp4<false, false>(p, h, w_down, nullptr, s_down, nullptr, c.hidden_dim, s);
}

}  // namespace moe
