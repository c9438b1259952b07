// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "FFN、SwiGLU 与 MoE" sec. 2: y = W_down[SiLU(W_gate x) * (W_up x)]; the
// ops-transformer MoE walkthrough (优化三) packs every expert's rows into one
// irregular matmul launch.  Here one persistent kernel covers all experts:
//
//   gate/up (GATED):  for the rows of expert e, D[rows x 256] accumulates
//                     x_perm[rows] . [W_gate[e] rows n0..n0+127 ; W_up[e] rows n0..n0+127]^T,
//                     so TMEM columns 0..127 hold g and 128..255 hold u; the
//                     epilogue forms h = SiLU(clip g) * clip u and stores bf16.
//   down:             D[rows x 256] = h[rows] . W_down[e][n0..n0+255]^T; the
//                     epilogue scales row r by row_weight[r] and stores fp32.
//
// Two tile shapes:
//   single (PAIR=false)  one CTA per 128x256 tile: A 128x64 + B 256x64 per
//                        k-block, 4 stages, tcgen05.mma.cta_group::1 M=128.
//   pair   (PAIR=true)   a cluster of 2 CTAs per 256x256 tile: each CTA stages
//                        its own 128 rows of A and half of B (128x64 each), the
//                        leader issues tcgen05.mma.cta_group::2 M=256 and its
//                        commits arrive on both CTAs' barriers; each CTA's TMEM
//                        holds its 128 rows.  Half the operand bytes per SM
//                        and 6 stages.  Used when experts have many rows.
//
// Roles (192 threads per CTA):
//   warp 0      TMA producer into the stage ring guarded by mbarriers.
//   warp 1      TMEM owner; one thread (the leader's, for pairs) issues the
//               MMAs: 4 x K=16 per 64-wide k-block, then commits the stage
//               back to the producers; two 256-column fp32 accumulators let
//               the epilogue of tile i overlap the MMAs of tile i+1.
//   warps 2-5   epilogue: tcgen05.ld (one TMEM lane = one output row per
//               thread), fused SwiGLU or routing weight, global store (the
//               fp32 y through a 4 KB shared-memory stage per warp, so that
//               the stores are whole 128-byte row segments).
//
// Tiles never straddle two experts: expert e owns ceil(rows_e / tile_rows)
// m-blocks; the tile list (expert-major, then n-block, then m-block, so the
// CTAs in flight share weight tiles through L2) is derived on the device from
// expert_offsets, so the host never reads a count.  Rows past the expert's
// segment are computed from whatever lies there and never stored.
//
// Every wait is bounded: after kWaitLimitNs the waiting thread records
// MOE_ERR_DEVICE_TIMEOUT in the status word, raises the abort flag (in both
// CTAs of a pair) and every role winds down (copies and MMAs drained, TMEM
// freed) instead of hanging.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace moe {

MOE_VIOLATION_COUNTER(violations_gemm_tc)

namespace {

constexpr int BM = 128;          // rows per CTA (TMEM lanes)
constexpr int BN = 256;          // MMA N (accumulator columns)
constexpr int BK = 64;           // one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB
constexpr uint32_t TMEM_COLS = 2 * BN;       // two accumulators
constexpr int MAX_E = 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s
constexpr int kThreads = 192;
constexpr int kStagingOffset = 5120;  // past Smem, 1024-aligned; 4 warps x 4 KB

template <bool PAIR>
struct Cfg {
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;         // output rows per tile
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;         // B rows staged per CTA
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PAIR ? 6 : 4;
  static constexpr uint32_t TX_BYTES = PAIR ? 2 * STAGE_BYTES : STAGE_BYTES;  // per leader barrier phase
};

struct Smem {
  uint64_t full[6];
  uint64_t empty[6];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[MAX_E + 1];
};

static_assert(sizeof(Smem) <= kStagingOffset, "the epilogue staging follows the barriers and tile list");

struct Params {
  int rows;                  // rows of the output (and of A unless gathered)
  const int32_t *row_token;  // gathered A: row r of A is src[row_token[r]]; null: A is dense
  int src_rows;              // rows of the gather source
  int K;                     // reduction length
  int N;                     // output columns (F for gate/up, D for down)
  int E;                     // groups
  int n_tiles;               // output-column tiles per m-block
  const int32_t *offsets;    // [E+1] row offsets, or null: one group of `rows` rows
  void *out;                 // h (bf16) or y (fp32), [rows, N]
  const float *row_weight;   // down only, nullable
  float clamp;
  int clamp_mode;
  int *status;
};

template <bool PAIR>
__device__ __forceinline__ void raise_abort(Smem &sm, uint32_t rank) {
  *(volatile int *)&sm.abort = 1;
  if (PAIR) ptx::st_cluster_u32(ptx::map_to_rank(&sm.abort, rank ^ 1u), 1u);
}

// Bounded wait; false if the CTA is aborting (this thread may have started it).
// The stage ring's hand-offs (the producer waiting for a free stage, the MMA
// thread for a full one) spin: a stage's round trip (copy, MMA, completion,
// refill) is what bounds the k-block rate, and a suspended waiter woke ~350
// cycles late in every round trip (clock64 timeline of one CTA).  The
// epilogue, which waits a whole tile, sleeps on the barrier with a
// suspend-time hint.  The clock is read every 64 polls when spinning.
template <bool PAIR, bool SPIN = false>
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Smem &sm, int *status, uint32_t rank) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (SPIN ? ptx::mbar_try_wait(bar, parity) : ptx::mbar_try_wait_sleep(bar, parity, ptx::kWaitHintNs)) return true;
    if (SPIN && (n & 63u) != 0) continue;
    if (*(volatile int *)&sm.abort) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      raise_abort<PAIR>(sm, rank);
      atomicExch(status, kDevTimeout);
      return false;
    }
  }
}

// Bounded wait used while winding down: ignores the abort flag (copies and
// MMAs already issued must land before shared memory or TMEM is released).
__device__ __forceinline__ void drain_bar(uint64_t *bar, uint32_t parity, int *status) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) {
      atomicExch(status, kDevTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (ptx::globaltimer_ns() - t0 < ns) {
  }
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
__device__ __forceinline__ Tile decode_tile(const Params &p, const Smem &sm, int t, int tile_m) {
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (sm.tile_start[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int e = lo;
  const int local = t - sm.tile_start[e];
  const int m_tiles = (sm.tile_start[e + 1] - sm.tile_start[e]) / p.n_tiles;
  Tile r;
  r.e = e;
  r.n_blk = local / m_tiles;
  r.m0 = seg_begin(p, e) + (local - r.n_blk * m_tiles) * tile_m;
  r.end = seg_end(p, e);
  return r;
}

template <bool GATED, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const Params p) {
  using C = Cfg<PAIR>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // stage buffers first, 1024-byte aligned (the swizzle atoms need it)
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *stage_a = base;
  uint8_t *stage_b = base + C::STAGES * A_BYTES;
  Smem &sm = *reinterpret_cast<Smem *>(base + C::STAGES * C::STAGE_BYTES);
  // fp32 epilogue staging: 32 rows x 32 columns per epilogue warp
  float *staging = reinterpret_cast<float *>(base + C::STAGES * C::STAGE_BYTES + kStagingOffset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // tile-processing unit
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  // ---- setup: barriers, TMEM, tile schedule
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(&sm.full[s], 1);
      ptx::mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&sm.tmem_full[a], 1);
      ptx::mbar_init(&sm.tmem_empty[a], PAIR ? 8 : 4);  // epilogue warps of both CTAs
    }
    ptx::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB0);
    if (GATED) ptx::prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    if (PAIR) {
      ptx::tmem_alloc_pair(&sm.tmem_base, TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(&sm.tmem_base, TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  if (warp == 2) {
    // tile_start[e] = sum over e' < e of ceil(rows_e' / TILE_M) * n_tiles
    int carry = 0;
    bool bad = false;  // checked build: offsets must not decrease or start below 0
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      int v = 0;
      if (e < p.E) {
        int n = seg_end(p, e) - seg_begin(p, e);
        if (kChecked && p.offsets && (p.offsets[e] < 0 || p.offsets[e + 1] < p.offsets[e])) bad = true;
        v = n > 0 ? (n + C::TILE_M - 1) / C::TILE_M * p.n_tiles : 0;
      }
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, incl, off);
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
  ptx::tc_fence_before();
  __syncwarp();
  if (PAIR) ptx::cluster_sync();  // the peer's copies may target the leader's barriers from here on
  else __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int total_tiles = sm.tile_start[p.E];
  const int k_blocks = (p.K + BK - 1) / BK;

  if (warp == 0) {
    // ================================================= TMA producer (both CTAs)
    // Dense A: lane 0 issues everything.  Gathered A: every lane issues the
    // gather of its 4 rows of the 128-row tile; lane 0 waits for the stage,
    // expects the bytes and loads B.
    const bool gather = p.row_token != nullptr;
    if (gather || lane == 0) {
      uint32_t last_parity[C::STAGES];
      bool used[C::STAGES];
#pragma unroll
      for (int s = 0; s < C::STAGES; ++s) {
        used[s] = false;
        last_parity[s] = 0;
      }
      uint32_t it = 0;
      bool ok = true;
      for (int t = unit; t < total_tiles && ok; t += n_units) {
        const Tile tl = decode_tile(p, sm, t, C::TILE_M);
        int tok[4] = {0, 0, 0, 0};
        if (gather) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = tl.m0 + (int)rank * BM + lane * 4 + i;
            tok[i] = r < tl.end ? p.row_token[r] : p.src_rows;  // out of range: zero fill
          }
        }
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          bool got = true;
          if (lane == 0) got = wait_bar<PAIR, true>(&sm.empty[s], ph ^ 1u, sm, p.status, rank);
          if (gather) {
            got = __shfl_sync(0xffffffffu, got, 0);
            __syncwarp();
          }
          if (!got) { ok = false; break; }
          const int k0 = kb * BK;
          uint8_t *a = stage_a + s * A_BYTES;
          uint8_t *b = stage_b + s * C::B_BYTES;
          if (PAIR) {
            const uint32_t bar = ptx::map_to_rank(&sm.full[s], 0);   // the leader's barrier
            if (lane == 0) {
              if (leader) ptx::mbar_arrive_expect_tx(&sm.full[s], C::TX_BYTES);
              if (!gather) ptx::tma_load_2d_pair(a, &tmA, bar, k0, tl.m0 + (int)rank * BM);
              if (GATED) {
                ptx::tma_load_3d_pair(b, rank == 0 ? &tmB0 : &tmB1, bar, k0, tl.n_blk * (BN / 2), tl.e);
              } else {
                ptx::tma_load_3d_pair(b, &tmB0, bar, k0, tl.n_blk * BN + (int)rank * (BN / 2), tl.e);
              }
            }
            if (gather) ptx::tma_gather4_pair(a + lane * 512, &tmA, bar, k0, tok[0], tok[1], tok[2], tok[3]);
          } else {
            if (lane == 0) {
              ptx::mbar_arrive_expect_tx(&sm.full[s], C::TX_BYTES);
              if (!gather) ptx::tma_load_2d(a, &tmA, &sm.full[s], k0, tl.m0);
              if (GATED) {
                const int n0 = tl.n_blk * (BN / 2);
                ptx::tma_load_3d(b, &tmB0, &sm.full[s], k0, n0, tl.e);
                ptx::tma_load_3d(b + C::B_BYTES / 2, &tmB1, &sm.full[s], k0, n0, tl.e);
              } else {
                const int n0 = tl.n_blk * BN;
                ptx::tma_load_3d(b, &tmB0, &sm.full[s], k0, n0, tl.e);
                ptx::tma_load_3d(b + C::B_BYTES / 2, &tmB0, &sm.full[s], k0, n0 + BN / 2, tl.e);
              }
            }
            if (gather) ptx::tma_gather4(a + lane * 512, &tmA, &sm.full[s], k0, tok[0], tok[1], tok[2], tok[3]);
          }
          used[s] = true;
          last_parity[s] = ph;
        }
      }
      // drain: every issued copy has landed before shared memory is released.
      // The leader's barriers count both CTAs' bytes; a peer that stopped early
      // gives its last copies time to land.
      if (lane == 0) {
        if (leader) {
          for (int s = 0; s < C::STAGES; ++s)
            if (used[s]) drain_bar(&sm.full[s], last_parity[s], p.status);
        } else if (!ok) {
          spin_ns(1000000);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(C::TILE_M, BN);
      uint32_t it = 0;
      int i = 0;
      bool ok = true;
      for (int t = unit; t < total_tiles && ok; t += n_units, ++i) {
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1u;
        if (!wait_bar<PAIR>(&sm.tmem_empty[acc], aph ^ 1u, sm, p.status, rank)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!wait_bar<PAIR, true>(&sm.full[s], ph, sm, p.status, rank)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_addr(stage_a + s * A_BYTES);
          const uint32_t b_addr = ptx::smem_addr(stage_b + s * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = ptx::desc_kmajor_sw128(a_addr + k * UMMA_K * 2);
            const uint64_t bd = ptx::desc_kmajor_sw128(b_addr + k * UMMA_K * 2);
            if (PAIR) ptx::mma_bf16_pair(d_tmem, ad, bd, idesc, (kb | k) != 0);
            else ptx::mma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          if (PAIR) ptx::mma_commit_pair_mc(&sm.empty[s], 0x3);
          else ptx::mma_commit(&sm.empty[s]);
        }
        if (!ok) break;
        if (PAIR) ptx::mma_commit_pair_mc(&sm.tmem_full[acc], 0x3);
        else ptx::mma_commit(&sm.tmem_full[acc]);
      }
      // drain: all issued MMAs complete before TMEM is released
      if (PAIR) ptx::mma_commit_pair(&sm.drain);
      else ptx::mma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.status);
    }
  } else {
    // ================================================= epilogue (warps 2..5)
    const int q = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row_in_tile = (int)rank * BM + q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    int i = 0;
    for (int t = unit; t < total_tiles; t += n_units, ++i) {
      const Tile tl = decode_tile(p, sm, t, C::TILE_M);
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1u;
      // one lane waits; the decision is warp-uniform (tcgen05.ld needs the whole warp)
      bool ok = true;
      if (lane == 0) ok = wait_bar<PAIR>(&sm.tmem_full[acc], aph, sm, p.status, rank);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      ptx::tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + acc * BN;
      const int row = tl.m0 + row_in_tile;
      const bool live = row < tl.end;
      if (GATED) {
        const int ncol0 = tl.n_blk * (BN / 2);
        __nv_bfloat16 *hrow = (__nv_bfloat16 *)p.out + (long)row * p.N + ncol0;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], u[32];
          ptx::tmem_ld32(tbase + c, g);
          ptx::tmem_ld32(tbase + BN / 2 + c, u);
          ptx::tmem_ld_wait();
          if (live) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float h0 = swiglu_h(__uint_as_float(g[2 * j]), __uint_as_float(u[2 * j]), p.clamp, p.clamp_mode);
              float h1 = swiglu_h(__uint_as_float(g[2 * j + 1]), __uint_as_float(u[2 * j + 1]), p.clamp,
                                  p.clamp_mode);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(h0, h1);
              pk[j] = *reinterpret_cast<uint32_t *>(&b2);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(hrow + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      } else {
        // Each 32 x 32 fp32 chunk goes through this warp's 4 KB of shared
        // memory: lane r writes its row (16-byte piece j at j ^ (r % 8), four
        // wavefronts per 512 bytes), then every store instruction writes four
        // whole 128-byte row segments instead of 32 rows' 16-byte pieces.
        const int ncol0 = tl.n_blk * BN;
        const float rw = (live && p.row_weight) ? p.row_weight[row] : 1.0f;
        float *stg = staging + q * 32 * 32;
        const int row0 = tl.m0 + (int)rank * BM + q * 32;  // this warp's first row
        const int rr = lane >> 3, ff = lane & 7;            // read-back: row 4 i + rr, piece ff
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
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
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && !leader) ptx::mbar_arrive_cluster(ptx::map_to_rank(&sm.tmem_empty[acc], 0));
        else ptx::mbar_arrive(&sm.tmem_empty[acc]);
      }
    }
  }

  // ---- teardown
  ptx::tc_fence_before();
  __syncwarp();
  if (PAIR) ptx::cluster_sync();  // neither CTA leaves while the pair's copies, MMAs or arrivals are pending
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    if (PAIR) ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}


// ------------------------------------------------------------------ host
template <bool GATED, bool PAIR>
size_t smem_bytes() {
  return 1024 + (size_t)Cfg<PAIR>::STAGES * Cfg<PAIR>::STAGE_BYTES + kStagingOffset + 4 * 32 * 32 * sizeof(float);
}

template <bool GATED, bool PAIR>
moe_status launch_tc(const Params &p, const void *a, const void *b0, const void *b1, int Nw, cudaStream_t s) {
  // A: [rows, K]; B: [E, Nw, K] (rank 3 even for one group)
  CUtensorMap ta, tb0, tb1;
  if (!tma_map_bf16(&ta, a, 2, (uint64_t)p.K, (uint64_t)(p.row_token ? p.src_rows : p.rows), 1, p.row_token ? 1 : 128)) return MOE_ERR_CUDA;
  if (!tma_map_bf16(&tb0, b0, 3, (uint64_t)p.K, (uint64_t)Nw, (uint64_t)p.E)) return MOE_ERR_CUDA;
  if (GATED) {
    if (!tma_map_bf16(&tb1, b1, 3, (uint64_t)p.K, (uint64_t)Nw, (uint64_t)p.E)) return MOE_ERR_CUDA;
  } else {
    tb1 = tb0;
  }
  int dev = 0, sms = 148;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  MOE_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const size_t smem = smem_bytes<GATED, PAIR>();
  auto kern = tc_grouped_gemm<GATED, PAIR>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  constexpr int TM = Cfg<PAIR>::TILE_M;
  const long ub = ((long)(p.rows + TM - 1) / TM + (p.offsets ? p.E : 0)) * p.n_tiles;  // tile upper bound
  if (ub <= 0) return MOE_OK;
  if (!PAIR) {
    const int grid = (int)(ub < sms ? ub : sms);
    kern<<<grid, kThreads, smem, s>>>(ta, tb0, tb1, p);
  } else {
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    lc.attrs = attr;
    lc.numAttrs = 1;
    lc.gridDim = dim3(2);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &lc) != cudaSuccess || clusters <= 0) clusters = sms / 2;
    const long units = ub < clusters ? ub : clusters;
    lc.gridDim = dim3((unsigned)(2 * units));
    MOE_CUDA_TRY(cudaLaunchKernelEx(&lc, kern, ta, tb0, tb1, p));
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}


// Pairs pay off only when groups are so large that the padding of their last
// 256-row tile is negligible (measured under the power cap, extra padded rows
// cost more than the pair saves on operand traffic): gate/up from
// kPairRowsGated rows per group on average, down, with 3.5x longer tiles and
// fewer of them, from kPairRowsDown.  Both tile shapes compute the same
// result to fp32 rounding.
#ifndef MOE_PAIR_ROWS_GATED
#define MOE_PAIR_ROWS_GATED 2048
#endif
#ifndef MOE_PAIR_ROWS_DOWN
#define MOE_PAIR_ROWS_DOWN 768
#endif
constexpr long kPairRowsGated = MOE_PAIR_ROWS_GATED;
constexpr long kPairRowsDown = MOE_PAIR_ROWS_DOWN;
bool use_pair(int rows, int E, bool gated) { return rows >= (gated ? kPairRowsGated : kPairRowsDown) * E; }

// One thread waits on an mbarrier that nothing arrives on, with the bounded
// wait of the pipelines above: it gives up after kWaitLimitNs and records the
// timeout in the status word.
__global__ void wait_selftest_kernel(int *status) {
  __shared__ Smem sm;
  if (threadIdx.x != 0) return;
  sm.abort = 0;
  ptx::mbar_init(&sm.full[0], 1);
  ptx::fence_mbar_init();
  wait_bar<false>(&sm.full[0], 0, sm, status, 0);
}

}  // namespace

moe_status launch_wait_selftest(int *status, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

bool tc_shapes_ok(const MoEConfig &c, int F) {
  return c.act_dtype == MOE_BF16 && c.hidden_dim % BN == 0 && F % 128 == 0 && c.hidden_dim % BK == 0 &&
         tma_encode_fn() != nullptr;
}

moe_status launch_gate_up_tc(const MoEConfig &c, int rows, const void *a, int a_rows, const int32_t *row_token,
                             const int32_t *offsets, const void *w_gate, const void *w_up, int F, void *h,
                             int *status, cudaStream_t s) {
  if (rows == 0) return MOE_OK;
  Params p;
  p.rows = rows;
  p.row_token = row_token;
  p.src_rows = a_rows;
  p.K = c.hidden_dim;
  p.N = F;
  p.E = offsets ? c.num_experts : 1;
  p.n_tiles = F / (BN / 2);
  p.offsets = offsets;
  p.out = h;
  p.row_weight = nullptr;
  p.clamp = c.swiglu_clamp;
  p.clamp_mode = c.clamp_mode;
  p.status = status;
  if (use_pair(rows, p.E, true)) return launch_tc<true, true>(p, a, w_gate, w_up, F, s);
  return launch_tc<true, false>(p, a, w_gate, w_up, F, s);
}

moe_status launch_down_tc(const MoEConfig &c, int rows, const void *h, const int32_t *offsets,
                          const void *w_down, int F, const float *row_weight, float *y, int *status,
                          cudaStream_t s) {
  if (rows == 0) return MOE_OK;
  Params p;
  p.rows = rows;
  p.row_token = nullptr;
  p.src_rows = rows;
  p.K = F;
  p.N = c.hidden_dim;
  p.E = offsets ? c.num_experts : 1;
  p.n_tiles = c.hidden_dim / BN;
  p.offsets = offsets;
  p.out = y;
  p.row_weight = row_weight;
  p.clamp = 0.0f;
  p.clamp_mode = 0;
  p.status = status;
  if (use_pair(rows, p.E, false)) return launch_tc<false, true>(p, h, w_down, nullptr, c.hidden_dim, s);
  return launch_tc<false, false>(p, h, w_down, nullptr, c.hidden_dim, s);
}

}  // namespace moe
