// Per-expert FFN on the kept rows as a grouped GEMM on the 5th-generation tensor cores.
//
//   up:   h[s]      = act(x_perm[s] . W1_e^T)     [rows of e] x [d_ff, d_model]^T
//   down: y_perm[s] = h[s] . W2_e^T               [rows of e] x [d_model, d_ff]^T
//
// h is stored in the operand type of the second product: bf16, or fp16 when W2 is given
// in fp16 (11 instead of 8 significant bits for h; A and B of one MMA always share a
// type).  y_perm is fp32.
//
// Experts are the feed-forward sub-networks of the sparsely-gated MoE layer (Shazeer et
// al., "Schlüsselbegriffe"); each runs only on the rows routed to it ("Methode": no
// computation where G(x)_i = 0).  Expert e owns permuted rows [offsets[e], offsets[e+1]).
//
// Kernel design (one CTA per SM, persistent):
//   warp 0      TMA producer: A tile [128 x 64] and B tile [BN x 64] per k-block into a
//               4-stage ring of 128-byte-swizzled shared-memory buffers.
//   warp 1      TMEM owner and MMA issuer: one thread issues tcgen05.mma (M=128, N=BN,
//               K=16) into one of two TMEM accumulators (2 x 256 fp32 columns), and
//               tcgen05.commit releases smem stages and hands finished accumulators on.
//   warps 2-17  epilogue: tcgen05.ld of the accumulator (each warp reads its 32-lane
//               quarter and every fourth 32-column chunk), activation, rounding to
//               bf16/fp16 (or fp32 as is), stores of the rows that belong to the expert
//               (a ragged tail is masked).  Four warps per lane quarter split a 256-column
//               accumulator evenly (two chunks each) and keep a ragged tile, whose rows
//               all sit in the first quarters, from serialising on few warps; the GELU
//               epilogue of the up-projection is latency-bound, and four warps per SM
//               sub-partition measured 1.2% faster on the whole expert FFN than three.
// Tiles are (expert, m-tile, n-tile) with n innermost: CTAs running at the same time share
// the A rows of an m-tile through L2 while each streams a different weight tile (measured
// 1.5-3.5% faster than m innermost on the five workloads).
// Rows past an expert's end that a 128-row tile reads belong to the next expert or lie
// past the buffer (TMA fills those with zeros); they only feed masked output rows.
// No cross-CTA waits; every mbarrier wait is bounded and an expired wait sets
// kErrTimeout, drains this CTA's in-flight copies and MMAs and frees TMEM.
#include <cudaTypedefs.h>

#include <map>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace gg {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 16;  // 4 per TMEM lane quarter (96 registers a thread, no spills)
constexpr int EPI_SUBS = EPI_WARPS / 4;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES_MAX = 256 * BK * 2;   // 32 KB
constexpr int MAX_GROUPS = 1024;
constexpr int TMEM_COLS = 512;              // two accumulators of up to 256 columns
constexpr int STAGE_BYTES = A_BYTES + B_BYTES_MAX;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;  // 192 KB
// CTA pairs load half of each B box, so the same ring holds 6 stages of 32 KB
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_STAGE_BYTES = A_BYTES + B_BYTES_MAX / 2;
static_assert(PAIR_STAGES * PAIR_STAGE_BYTES <= RING_BYTES, "pair ring fits the ring");
static_assert(2 * PAIR_STAGES + 5 <= 28, "barriers fit their 256 bytes with the flags");
constexpr int SMEM_BYTES = 1024 /*align slack*/ + RING_BYTES + 256 /*barriers, flags*/ +
                           4 * (MAX_GROUPS + 1 + 40);

// Epilogue output modes.
constexpr int OUT_BF16 = 0;  // act, bf16
constexpr int OUT_F16 = 1;   // act, fp16
constexpr int OUT_F32 = 2;   // fp32
constexpr int OUT_COMBINE = 3;  // fp32 times the gate, into the token's row of y (k = 1)
constexpr int OUT_COMBINE_BF16 = 4;  // as OUT_COMBINE, y in bf16 (the scaled fp32 rounded)
constexpr int OUT_COMBINE_ADD = 5;   // fp32 times the gate, added in memory into the token's
                                     // row of y (k = 2; y zeroed by the up-projection)
// 16-byte vectors of a zeroing chunk: two per epilogue thread
constexpr int ZERO_CHUNK_VECS = EPI_WARPS * 32 * 2;

struct Args {
  const int32_t* offsets;
  int E;
  int N;         // output columns (d_ff for up, d_model for down)
  int K;         // contraction (d_model for up, d_ff for down)
  int bn;        // N tile: 256, 128 or 64 (divides N)
  int n_tiles;   // N / bn
  int64_t rows_cap;
  void* out;
  int act;       // 0 none, 1 ReLU, 2 GELU
  int out_mode;  // OUT_*
  int ab_f16;    // operand type of A and B: 1 fp16, 0 bf16
  const int32_t* perm_src;  // OUT_COMBINE*: assignment t*comb_k + j of each permuted row
  int comb_k;               // OUT_COMBINE*: assignments per token
  const float* gate;        // OUT_COMBINE*: gate of each assignment
  const int32_t* slot_pos;  // OUT_COMBINE*: permuted row of each token, < 0 when dropped
  const int32_t* gather_src;  // non-null: A row s is row gather_src[s] / gather_k of the
  int gather_k;               // A tensor (the token rows x), gathered by the TMA itself
  void* pre;                  // OUT_BF16 / OUT_F16 with an activation: also store the
                              // pre-activation there (same type and layout as out), or null
  int w_mod;                  // row group g multiplies weight block g % w_mod (w_mod >= E:
                              // group g uses block g)
  float4* zero_out;           // non-null: the epilogue threads also zero zero_out[0, zero_vecs)
  int64_t zero_vecs;          // (16-byte vectors), one chunk per CTA and tile
  int* err;
};

struct Tile {
  int e, mt, nt, row0, valid;
};

// Tile L of the (expert, m-tile, n-tile) list, m-tiles of bm rows: row0 is the tile's
// first permuted row, valid its rows that belong to the expert (>= 1).
__device__ __forceinline__ Tile decode_tile(int L, const int* tp, const Args& a, int bm) {
  // expert: the largest e with tp[e] * n_tiles <= L
  int lo = 0, hi = a.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tp[mid] * a.n_tiles <= L) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.e = lo;
  const int local = L - tp[lo] * a.n_tiles;
  t.mt = local / a.n_tiles;
  t.nt = local - t.mt * a.n_tiles;
  const int r0 = __ldg(a.offsets + lo), r1 = __ldg(a.offsets + lo + 1);
  t.row0 = r0 + t.mt * bm;
  t.valid = min(bm, r1 - t.row0);
  return t;
}

template <int ACT>
__device__ __forceinline__ float epi_act(float z) {
  if (ACT == 1) return fmaxf(z, 0.0f);
  if (ACT == 2) return 0.5f * z * (1.0f + erf_as7126(z * 0.70710678118654752f));
  return z;
}

// One warp's share of a finished accumulator: its 32 rows (one per lane), the 32-column
// chunks sub*32 + 32*EPI_SUBS*i of the tile; rows outside the expert are not stored.
template <int MODE, int ACT>
__device__ __forceinline__ void epilogue_rows(const Args& a, uint32_t tbase, int64_t oidx, int sub,
                                              bool row_ok, float scale) {
  for (int c = sub * 32; c < a.bn; c += 32 * EPI_SUBS) {
    uint32_t v[32];
    tmem_ld32(tbase + c, v);
    tmem_ld_wait();
    if (!row_ok) continue;
    if (MODE == OUT_COMBINE_BF16) {
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        pk[j] = pack_bf16x2(scale * __uint_as_float(v[2 * j]), scale * __uint_as_float(v[2 * j + 1]));
      uint16_t* dst = static_cast<uint16_t*>(a.out) + oidx + c;  // 64-byte aligned
      st_global_v8(dst, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
      st_global_v8(dst + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
    } else if (MODE == OUT_COMBINE_ADD) {
      // the token's other assignment adds its row too: the two in-memory adds onto the
      // zeroed row commute, so y does not depend on which lands first
      float* dst = static_cast<float*>(a.out) + oidx + c;  // 128-byte aligned
#pragma unroll
      for (int j = 0; j < 8; ++j)
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 4 * j),
                     "f"(__fmul_rn(scale, __uint_as_float(v[4 * j]))),
                     "f"(__fmul_rn(scale, __uint_as_float(v[4 * j + 1]))),
                     "f"(__fmul_rn(scale, __uint_as_float(v[4 * j + 2]))),
                     "f"(__fmul_rn(scale, __uint_as_float(v[4 * j + 3])))
                     : "memory");
    } else if (MODE == OUT_F32 || MODE == OUT_COMBINE) {
      float* dst = static_cast<float*>(a.out) + oidx + c;  // 128-byte aligned
      if (MODE == OUT_COMBINE) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(scale * __uint_as_float(v[j]));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        st_global_v8(dst + 8 * j, v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3], v[8 * j + 4],
                     v[8 * j + 5], v[8 * j + 6], v[8 * j + 7]);
    } else {
      uint32_t pk[16];
      if (a.pre != nullptr) {  // the pre-activation, for the backward pass
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float z0 = __uint_as_float(v[2 * j]), z1 = __uint_as_float(v[2 * j + 1]);
          pk[j] = MODE == OUT_F16 ? pack_f16x2(z0, z1) : pack_bf16x2(z0, z1);
        }
        uint16_t* pdst = static_cast<uint16_t*>(a.pre) + oidx + c;  // 64-byte aligned
        st_global_v8(pdst, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
        st_global_v8(pdst + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float x0, x1;
        if (ACT == 2) {
          gelu2_as7126(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]), x0, x1);
        } else {
          x0 = epi_act<ACT>(__uint_as_float(v[2 * j]));
          x1 = epi_act<ACT>(__uint_as_float(v[2 * j + 1]));
        }
        pk[j] = MODE == OUT_F16 ? pack_f16x2(x0, x1) : pack_bf16x2(x0, x1);
      }
      uint16_t* dst = static_cast<uint16_t*>(a.out) + oidx + c;  // 64-byte aligned
      st_global_v8(dst, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
      st_global_v8(dst + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
    }
  }
}

// PAIR = false: one CTA per SM, 128-row tiles, tcgen05 cta_group::1.
// PAIR = true: clusters of two CTAs on the two SMs of a pair share 256-row tiles
// (tcgen05 cta_group::2, M = 256): CTA rank r loads rows [row0 + 128 r, +128) of A and
// rows [n0 + r bn/2, +bn/2) of the B tile into its own shared memory, with the copies of
// both CTAs completing on the rank-0 CTA's full barrier; one thread of rank 0 issues the
// MMAs and commits their completion to both CTAs' barriers; each CTA's epilogue reads its
// own 128 TMEM lanes and both arrive on rank 0's accumulator-empty barrier.  Each SM then
// streams half of the B tile per k-block instead of all of it.
template <bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // stage s: A tile at ring + s * SB, then the B tile
  constexpr int NST = PAIR ? PAIR_STAGES : STAGES;        // stages of the ring
  constexpr int SB = PAIR ? PAIR_STAGE_BYTES : STAGE_BYTES;  // bytes of one stage
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES);
  // bars: full[NST], empty[NST], tfull[2], tempty[2], drain
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + NST);
  const uint32_t tfull0 = smem_u32(bars + 2 * NST);
  const uint32_t tempty0 = smem_u32(bars + 2 * NST + 2);
  const uint32_t drain = smem_u32(bars + 2 * NST + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NST + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* scratch = reinterpret_cast<int*>(smem + RING_BYTES + 256);
  int* tp = scratch + 40;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  constexpr int TBM = PAIR ? 2 * BM : BM;  // rows of one tile (of the pair)
  const int first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int stride = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, PAIR ? 2 * EPI_WARPS : EPI_WARPS);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
      tmem_relinquish();
    }
  }
  grid_dep_wait();  // offsets and A come from the previous kernels on the stream
  grid_dep_launch();
  const bool ok = block_tile_prefix(a.offsets, a.E, a.rows_cap, TBM, tp, scratch);
  if (!ok && threadIdx.x == 0 && rank == 0) set_error(a.err, kErrOffsets);
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = ok ? tp[a.E] * a.n_tiles : 0;
  const int kblocks = a.K / BK;
  const int b_rows = PAIR ? a.bn / 2 : a.bn;  // rows of the B tile this CTA loads
  const uint32_t b_bytes = static_cast<uint32_t>(b_rows) * BK * 2;
  const uint32_t stage_tx = (PAIR ? 2u : 1u) * (A_BYTES + b_bytes);  // bytes per full phase
  // the full barrier every copy of a stage completes on: rank 0's in a pair
  auto full_bar = [&](int stage) -> uint32_t {
    return PAIR ? mapa_shared(full0 + 8 * stage, 0) : full0 + 8 * stage;
  };

  if (warp == 0 && a.gather_src != nullptr) {
    // ------------------------------------------------- TMA producer, gathered A rows
    // The A operand of permuted row s is token row gather_src[s] / gather_k of x: lane l
    // fetches rows 4l .. 4l+3 of this CTA's 128 rows with one tile::gather4 per k-block
    // (the same 512 bytes a tiled load of the permuted rows would place there).  Rows
    // past the expert's end repeat its last row; they only feed masked output rows.
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_par = 0;
    bool aborted = false;
    int cur_row0 = -1;
    int g0 = 0, g1 = 0, g2 = 0, g3 = 0;
    for (int L = first; L < total && !aborted; L += stride) {
      const Tile t = decode_tile(L, tp, a, TBM);
      if (t.row0 != cur_row0) {  // n-tiles of one m-tile are consecutive: gather once
        cur_row0 = t.row0;
        const int last = t.valid - 1;
        const int r = static_cast<int>(rank) * BM + 4 * lane;
        g0 = __ldg(a.gather_src + t.row0 + min(r + 0, last)) / a.gather_k;
        g1 = __ldg(a.gather_src + t.row0 + min(r + 1, last)) / a.gather_k;
        g2 = __ldg(a.gather_src + t.row0 + min(r + 2, last)) / a.gather_k;
        g3 = __ldg(a.gather_src + t.row0 + min(r + 3, last)) / a.gather_k;
      }
      const int brow = (t.e % a.w_mod) * a.N + t.nt * a.bn + static_cast<int>(rank) * b_rows;
      for (int kb = 0; kb < kblocks; ++kb) {
        int okw = 1;
        if (lane == 0) okw = mbar_wait(empty0 + 8 * stage, phase ^ 1, s_abort) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, okw, 0)) {
          aborted = true;
          break;
        }
        uint8_t* st = ring + stage * SB;
        const uint32_t fb = full_bar(stage);
        if (lane == 0 && rank == 0) mbar_arrive_expect_tx(full0 + 8 * stage, stage_tx);
        __syncwarp();
        if constexpr (PAIR) {
          tma_gather4_2d_pair(smem_u32(st) + 512u * lane, &tmA, fb, kb * BK, g0, g1, g2, g3);
          if (lane == 0) tma_load_2d_pair(smem_u32(st + A_BYTES), &tmB, fb, kb * BK, brow);
        } else {
          tma_gather4_2d(smem_u32(st) + 512u * lane, &tmA, fb, kb * BK, g0, g1, g2, g3);
          if (lane == 0) tma_load_2d(smem_u32(st + A_BYTES), &tmB, fb, kb * BK, brow);
        }
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == NST) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (aborted && lane == 0) {
      set_error(a.err, kErrTimeout);
      *s_abort = 1;
      // let every copy this warp started land before the CTA releases its smem (a pair's
      // second CTA cannot watch rank 0's barrier: it waits out a fixed drain time)
      if (rank == 0) {
        for (int s = 0; s < NST; ++s)
          if (armed & (1u << s)) mbar_wait(full0 + 8 * s, (armed_par >> s) & 1, nullptr, kDrainLimitNs);
      } else {
        const unsigned long long t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < kDrainLimitNs / 4) __nanosleep(1000);
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool aborted = false;
      for (int L = first; L < total && !aborted; L += stride) {
        const Tile t = decode_tile(L, tp, a, TBM);
        const int brow = (t.e % a.w_mod) * a.N + t.nt * a.bn + static_cast<int>(rank) * b_rows;
        const int arow = t.row0 + static_cast<int>(rank) * BM;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, s_abort)) {
            aborted = true;
            break;
          }
          uint8_t* st = ring + stage * SB;
          const uint32_t fb = full_bar(stage);
          if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * stage, stage_tx);
          if constexpr (PAIR) {
            tma_load_2d_pair(smem_u32(st), &tmA, fb, kb * BK, arow);
            tma_load_2d_pair(smem_u32(st + A_BYTES), &tmB, fb, kb * BK, brow);
          } else {
            tma_load_2d(smem_u32(st), &tmA, fb, kb * BK, arow);
            tma_load_2d(smem_u32(st + A_BYTES), &tmB, fb, kb * BK, brow);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (aborted) {
        set_error(a.err, kErrTimeout);
        *s_abort = 1;
        // let every copy this thread started land before the CTA releases its smem
        if (rank == 0) {
          for (int s = 0; s < NST; ++s)
            if (armed & (1u << s)) mbar_wait(full0 + 8 * s, (armed_par >> s) & 1, nullptr, kDrainLimitNs);
        } else {
          const unsigned long long t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < kDrainLimitNs / 4) __nanosleep(1000);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_f32acc(TBM, a.bn, a.ab_f16 ? kFmtF16 : kFmtBF16);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool aborted = false;
      for (int L = first; L < total && !aborted; L += stride) {
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1, s_abort)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, s_abort)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(ring + stage * SB);
          const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if constexpr (PAIR)
              tc_mma_pair_f16kind(d_tmem, sdesc_k128(a0 + kk * 32), sdesc_k128(b0 + kk * 32), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma_f16kind(d_tmem, sdesc_k128(a0 + kk * 32), sdesc_k128(b0 + kk * 32), idesc,
                             (kb | kk) != 0 ? 1u : 0u);
          }
          if constexpr (PAIR) {  // both CTAs' stages are free once these MMAs are done
            tc_commit_pair(mapa_shared(empty0 + 8 * stage, 0));
            tc_commit_pair(mapa_shared(empty0 + 8 * stage, 1));
          } else {
            tc_commit(empty0 + 8 * stage);
          }
          if (++stage == NST) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        if constexpr (PAIR) {
          tc_commit_pair(mapa_shared(tfull0 + 8 * acc, 0));
          tc_commit_pair(mapa_shared(tfull0 + 8 * acc, 1));
        } else {
          tc_commit(tfull0 + 8 * acc);
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (aborted) {
        set_error(a.err, kErrTimeout);
        *s_abort = 1;
        // wait for the MMAs already issued before TMEM is freed
        if constexpr (PAIR) tc_commit_pair(mapa_shared(drain, 0));
        else tc_commit(drain);
        mbar_wait(drain, 0, nullptr, kDrainLimitNs);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;               // TMEM lane quarter this warp may read
    const int sub = (warp - 2) >> 2;      // which 32-column chunks: sub*32 + 128*i
    const int mode = a.out_mode * 3 + a.act;
    const bool combine = a.out_mode == OUT_COMBINE || a.out_mode == OUT_COMBINE_BF16 ||
                         a.out_mode == OUT_COMBINE_ADD;
    // zeroing of zero_out: chunk blockIdx.x + i * gridDim.x after this CTA's i-th tile,
    // the chunks left after its last tile at the end
    int64_t zc = blockIdx.x;
    const int64_t zchunks = a.zero_out != nullptr
                                ? (a.zero_vecs + ZERO_CHUNK_VECS - 1) / ZERO_CHUNK_VECS : 0;
    auto zero_chunk = [&]() {
      const int64_t v0 = zc * ZERO_CHUNK_VECS + (warp - 2) * 64 + lane * 2;
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (v0 + u < a.zero_vecs) a.zero_out[v0 + u] = make_float4(0.f, 0.f, 0.f, 0.f);
      zc += gridDim.x;
    };
    if (a.out_mode == OUT_COMBINE || a.out_mode == OUT_COMBINE_BF16) {
      // y = 0 for tokens whose only assignment was dropped (no tile writes them); done
      // while the first tile's operands stream in
      const int row_vec = a.out_mode == OUT_COMBINE ? a.N / 4 : a.N / 8;  // 16-byte vectors
      const int ew = warp - 2;
      const int64_t gstride = static_cast<int64_t>(gridDim.x) * EPI_WARPS * 32;
      for (int64_t b = (static_cast<int64_t>(blockIdx.x) * EPI_WARPS + ew) * 32; b < a.rows_cap;
           b += gstride) {
        const bool drop = b + lane < a.rows_cap && __ldg(a.slot_pos + b + lane) < 0;
        uint32_t m = __ballot_sync(0xffffffffu, drop);
        while (m) {
          const int j = __ffs(m) - 1;
          m &= m - 1;
          float4* row = reinterpret_cast<float4*>(static_cast<uint8_t*>(a.out) + (b + j) * row_vec * 16);
          for (int v = lane; v < row_vec; v += 32) row[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    const uint32_t tempty_peer0 = PAIR ? mapa_shared(tempty0, 0) : tempty0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int L = first; L < total; L += stride) {
      const Tile t = decode_tile(L, tp, a, TBM);
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, s_abort)) {
        if (lane == 0) set_error(a.err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const int r = q * 32 + lane;
      const int crow = static_cast<int>(rank) * BM + r;  // row within the (pair's) tile
      bool row_ok = crow < t.valid;
      int64_t orow = t.row0 + crow;
      float scale = 1.0f;
      if (combine && row_ok) {
        // the permuted row's assignment a = t*comb_k + j: y[t] gets g_a * (h W2^T)[row]
        const int asg = __ldg(a.perm_src + orow);
        if (asg < 0 || asg >= a.rows_cap) {
          set_error(a.err, kErrSlot);  // not a permutation written by the permute step
          row_ok = false;
        } else {
          scale = __ldg(a.gate + asg);
          orow = asg / a.comb_k;
        }
      }
      const int64_t oidx = orow * a.N + t.nt * a.bn;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256;
      // a warp none of whose rows belong to the expert skips the tile
      if (__any_sync(0xffffffffu, row_ok)) {
        switch (mode) {
          case OUT_BF16 * 3 + 1: epilogue_rows<OUT_BF16, 1>(a, tbase, oidx, sub, row_ok, scale); break;
          case OUT_BF16 * 3 + 2: epilogue_rows<OUT_BF16, 2>(a, tbase, oidx, sub, row_ok, scale); break;
          case OUT_F16 * 3 + 1: epilogue_rows<OUT_F16, 1>(a, tbase, oidx, sub, row_ok, scale); break;
          case OUT_F16 * 3 + 2: epilogue_rows<OUT_F16, 2>(a, tbase, oidx, sub, row_ok, scale); break;
          case OUT_COMBINE * 3 + 0: epilogue_rows<OUT_COMBINE, 0>(a, tbase, oidx, sub, row_ok, scale); break;
          case OUT_COMBINE_BF16 * 3 + 0: epilogue_rows<OUT_COMBINE_BF16, 0>(a, tbase, oidx, sub, row_ok, scale); break;
          case OUT_COMBINE_ADD * 3 + 0: epilogue_rows<OUT_COMBINE_ADD, 0>(a, tbase, oidx, sub, row_ok, scale); break;
          default: epilogue_rows<OUT_F32, 0>(a, tbase, oidx, sub, row_ok, scale); break;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // relaxed: the accumulator's TMEM reads are complete (tcgen05.wait::ld) and the
        // MMA thread reads none of this warp's global stores
        if constexpr (PAIR) mbar_arrive_cluster_relaxed(tempty_peer0 + 8 * acc);
        else mbar_arrive_relaxed(tempty0 + 8 * acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
      if (zc < zchunks) zero_chunk();
    }
    while (zc < zchunks) zero_chunk();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // a pair's CTAs leave together: rank 0's MMAs read the other CTA's shared memory and
  // the other CTA's epilogue arrives on rank 0's barriers
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gg

// ------------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_2b(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, int f16) {
  auto encode = get_encode_fn();
  if (encode == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                      2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int pick_bn(int N) {
  if (N % 256 == 0) return 256;
  if (N % 128 == 0) return 128;
  return 64;
}

// Experts with at least this many rows on average (T*k / E, counted before capacity
// drops) run on CTA pairs (256-row tiles, cta_group::2).  Near 256 rows a good share of
// the experts spill into a second, mostly empty 256-row tile (the two-level workload's
// experts hold 195-331 rows: its expert FFN took 116.7 us on pairs, 111.6 us on 128-row
// tiles); from 512 on that share is small.
constexpr int64_t kPairMinRowsPerExpert = 512;

// Clusters of two CTAs of grouped_gemm_tc_kernel<true> that fit on the device at once (a
// persistent grid larger than that would serialise), looked up once per context.
static int max_active_pairs(const LaunchCtx& c) {
  static std::mutex mu;
  static std::map<unsigned long long, int> cache;
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) != cudaSuccess) return c.num_sms / 2;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(ctx);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (c.num_sms / 2));
  cfg.blockDim = dim3(gg::THREADS);
  cfg.dynamicSmemBytes = gg::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gg::grouped_gemm_tc_kernel<true>, &cfg) != cudaSuccess ||
      n <= 0)
    n = c.num_sms / 2;
  if (n > c.num_sms / 2) n = c.num_sms / 2;
  cache[ctx] = n;
  return n;
}

// A: the permuted rows [rows_cap, K], or with gather_src the token rows [a_rows, K] that
// permuted row s reads at row gather_src[s] / gather_k.
static cudaError_t launch_one(const void* A, int64_t rows_cap, int K, const void* B, int E, int N,
                              int ab_f16, void* out, int out_mode, const int32_t* offsets, int act,
                              const LaunchCtx& c, const int32_t* perm_src = nullptr,
                              const float* gate = nullptr, const int32_t* slot_pos = nullptr,
                              const int32_t* gather_src = nullptr, int gather_k = 1,
                              int64_t a_rows = 0, void* pre = nullptr, int w_count = 0,
                              int comb_k = 1, void* zero_out = nullptr, int64_t zero_bytes = 0) {
  const int bn = pick_bn(N);
  const int wb = w_count > 0 ? w_count : E;  // weight blocks of B
  const bool pair = rows_cap >= kPairMinRowsPerExpert * E;
  CUtensorMap tmA, tmB;
  if (gather_src != nullptr) {
    // one-row boxes for tile::gather4
    if (a_rows <= 0 || !make_tmap_2b(&tmA, A, static_cast<uint64_t>(a_rows), K, 1, ab_f16))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_2b(&tmA, A, static_cast<uint64_t>(rows_cap), K, gg::BM, ab_f16)) {
    return cudaErrorInvalidValue;
  }
  // a pair's CTA loads half of each B tile
  if (!make_tmap_2b(&tmB, B, static_cast<uint64_t>(wb) * N, K, pair ? bn / 2 : bn, ab_f16))
    return cudaErrorInvalidValue;
  gg::Args a;
  a.offsets = offsets;
  a.E = E;
  a.N = N;
  a.K = K;
  a.bn = bn;
  a.n_tiles = N / bn;
  a.rows_cap = rows_cap;
  a.out = out;
  a.act = act;
  a.out_mode = out_mode;
  a.ab_f16 = ab_f16;
  a.perm_src = perm_src;
  a.gate = gate;
  a.slot_pos = slot_pos;
  a.gather_src = gather_src;
  a.gather_k = gather_k;
  a.pre = pre;
  a.w_mod = wb;
  a.comb_k = comb_k;
  a.zero_out = static_cast<float4*>(zero_out);
  a.zero_vecs = zero_out != nullptr ? zero_bytes / 16 : 0;
  a.err = c.err;
  // upper bound of the tile count: sum_e ceil(n_e / bm) <= rows_cap / bm + E
  const int tbm = pair ? 2 * gg::BM : gg::BM;
  const int64_t max_tiles = (rows_cap / tbm + E) * static_cast<int64_t>(a.n_tiles);
  if (pair) {
    cudaError_t e = ensure_smem_limit(gg::grouped_gemm_tc_kernel<true>, gg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int64_t pairs_cap = max_active_pairs(c);
    const int pairs = static_cast<int>(max_tiles < pairs_cap ? max_tiles : pairs_cap);
    if (pairs <= 0) return cudaSuccess;
    return launch_kernel_pairs(gg::grouped_gemm_tc_kernel<true>, dim3(2 * pairs), dim3(gg::THREADS),
                               gg::SMEM_BYTES, c, tmA, tmB, a);
  }
  const int grid = static_cast<int>(max_tiles < c.num_sms ? max_tiles : c.num_sms);
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = ensure_smem_limit(gg::grouped_gemm_tc_kernel<false>, gg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(gg::grouped_gemm_tc_kernel<false>, dim3(grid), dim3(gg::THREADS),
                       gg::SMEM_BYTES, c, tmA, tmB, a);
}

// The up-projection h = act(A . W1^T): A is x_perm, or the token rows x gathered by the
// TMA through gather_src (no x_perm).
// zero_out / zero_bytes: a buffer (16-byte multiple) the epilogue threads also zero.
static cudaError_t launch_up(const FfnProblem& p, const LaunchCtx& c, void* zero_out = nullptr,
                             int64_t zero_bytes = 0) {
  const int hf = p.hidden_f16 ? 1 : 0;
  const int mode = hf ? gg::OUT_F16 : gg::OUT_BF16;
  if (p.gather_src != nullptr)
    return launch_one(p.x, p.rows_cap, p.d, p.w1, p.E, p.f, 0, p.h, mode, p.offsets, p.act, c,
                      nullptr, nullptr, nullptr, p.gather_src, p.k, p.x_rows, p.u, p.w_count, 1,
                      zero_out, zero_bytes);
  return launch_one(p.x_perm, p.rows_cap, p.d, p.w1, p.E, p.f, 0, p.h, mode, p.offsets, p.act, c,
                    nullptr, nullptr, nullptr, nullptr, 1, 0, p.u, p.w_count, 1, zero_out,
                    zero_bytes);
}

cudaError_t launch_ffn_combine_bf16(const FfnProblem& p, const int32_t* perm_src,
                                    const int32_t* slot_pos, const float* gate, void* y,
                                    const LaunchCtx& c) {
  if (p.E > gg::MAX_GROUPS) return cudaErrorInvalidValue;
  const int hf = p.hidden_f16 ? 1 : 0;
  if (p.k == 2) {
    // y = 0 by the up-projection's epilogue threads (one 16 KB chunk per CTA and tile, in
    // time with the tensor-core work), then each kept row added into its token's row
    if (p.y_bf16) return cudaErrorInvalidValue;
    const int64_t y_bytes = p.rows_cap / 2 * p.d * 4;
    cudaError_t e = launch_up(p, c, y, y_bytes);
    if (e != cudaSuccess) return e;
    return launch_one(p.h, p.rows_cap, p.f, p.w2, p.E, p.d, hf, y, gg::OUT_COMBINE_ADD, p.offsets,
                      0, c, perm_src, gate, slot_pos, nullptr, 1, 0, nullptr, 0, 2);
  }
  if (p.k != 1) return cudaErrorInvalidValue;
  cudaError_t e = launch_up(p, c);
  if (e != cudaSuccess) return e;
  return launch_one(p.h, p.rows_cap, p.f, p.w2, p.E, p.d, hf, y,
                    p.y_bf16 ? gg::OUT_COMBINE_BF16 : gg::OUT_COMBINE, p.offsets, 0, c, perm_src,
                    gate, slot_pos);
}

cudaError_t launch_ffn_bf16(const FfnProblem& p, const LaunchCtx& c) {
  if (p.E > gg::MAX_GROUPS) return cudaErrorInvalidValue;
  const int hf = p.hidden_f16 ? 1 : 0;
  cudaError_t e = launch_up(p, c);
  if (e != cudaSuccess) return e;
  return launch_one(p.h, p.rows_cap, p.f, p.w2, p.E, p.d, hf, p.y_perm, gg::OUT_F32, p.offsets, 0, c,
                    nullptr, nullptr, nullptr, nullptr, 1, 0, nullptr, p.w_count);
}

}  // namespace moe

// ------------------------------------------------------------- erf self-check

namespace moe {
__global__ void erf_check_kernel(const float* __restrict__ x, float* __restrict__ fast,
                                 float* __restrict__ ref, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    fast[i] = erf_as7126(x[i]);
    ref[i] = erff(x[i]);
  }
}

// the GELU epilogue's paired evaluation on (z[2i], z[2i+1]); an odd last value is paired
// with itself
__global__ void gelu_check_kernel(const float* __restrict__ z, float* __restrict__ fast,
                                  float* __restrict__ ref, int64_t n) {
  const int64_t pairs = (n + 1) / 2;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pairs;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j0 = 2 * i, j1 = 2 * i + 1 < n ? 2 * i + 1 : 2 * i;
    float g0, g1;
    gelu2_as7126(z[j0], z[j1], g0, g1);
    fast[j0] = g0;
    ref[j0] = gelu_exact(z[j0]);
    if (j1 != j0) {
      fast[j1] = g1;
      ref[j1] = gelu_exact(z[j1]);
    }
  }
}
}  // namespace moe

extern "C" moe_status moe_erf_check(const float* x, float* fast, float* ref, int64_t n,
                                    moe_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !fast || !ref))) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  moe::erf_check_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                          reinterpret_cast<cudaStream_t>(stream)>>>(x, fast, ref, n);
  moe::set_last_launch_count(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_gelu_check(const float* z, float* fast, float* ref, int64_t n,
                                     moe_stream_t stream) {
  if (n < 0 || (n > 0 && (!z || !fast || !ref))) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  int64_t blocks = ((n + 1) / 2 + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  moe::gelu_check_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                           reinterpret_cast<cudaStream_t>(stream)>>>(z, fast, ref, n);
  moe::set_last_launch_count(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
