// Backward pass of the sparsely-gated MoE layer (bf16 layers).
//
// The loss whose gradients are formed is L = sum(dy * y) + w_importance * CV(Importance)^2
// + w_load * CV(Load)^2 (Shazeer et al., "Load-Balancing-Losses": the auxiliary losses
// scale the squared coefficient of variation of Importance and of Load; "Fragen": the
// gate values of the chosen experts keep continuous derivatives, so gradients flow
// through the gating network although the top-k choice is discrete).  The choice of
// experts and the capacity drop pass no gradient; the noise draws are inputs.
//
// Steps, in the order they run:
//   pad offsets    per expert a run of its rows rounded up to 64 (poff), so that the
//                  ragged contraction over an expert's rows in the weight gradients reads
//                  whole 64-row blocks with zeros past the expert's end
//   combine bwd    d_o[p] = G_tj dy[t] at the padded row p of each kept assignment
//                  (padding rows zero), dgate[t, j] = <dy[t], y_perm[slot]>
//   dgrad down     du = (d_o . W2_e) * act'(u)  (tensor cores; W2_e read N-major)
//   wgrad down     dW2_e = d_o_e^T . h_e        (tensor cores; both operands MN-major,
//                                                the contraction runs over the rows)
//   dgrad up       dx_perm = du . W1_e          (tensor cores; W1_e read N-major)
//   wgrad up       dW1_e = du_e^T . x_perm_e
//   unpermute      dx[t] = sum_j dx_perm[slot(t, j)]
//   loss grads     dImportance, dLoad of the CV^2 terms
//   gate bwd       per token: scores gradient through Softmax(KeepTopK) (or the full
//                  softmax of the Switch gate), the Importance term, and for noisy gating
//                  the Load term through P(x, i) = Phi((l_i - kth_excluding(H, k, i)) /
//                  Softplus(z_i)) and the noise scale: dl [T, E], dz [T, E]
//   router         dx += dl . W_g (+ dz . W_noise); dW_g = dl^T . x; dW_noise = dz^T . x;
//                  dbias = sum_t dl   (fp32 SIMT products with a fixed-order split of
//                  the token contraction, so results are reproducible)
#include <cudaTypedefs.h>

#include <map>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace bw {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 12;
constexpr int EPI_SUBS = EPI_WARPS / 4;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES_MAX = 256 * BK * 2;   // 32 KB
constexpr int CHUNK = 64 * BK * 2;          // one MN-major TMA box: 64 rows of 64 elements
constexpr int MAX_GROUPS = 1024;
constexpr int TMEM_COLS = 512;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES_MAX;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
// CTA pairs (cta_group::2, 256-row tiles): each CTA holds its 128 rows of A and half of
// the B columns, so a stage is 32 KB and six of them fill the same ring
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_STAGE_BYTES = A_BYTES + B_BYTES_MAX / 2;
static_assert(PAIR_STAGES * PAIR_STAGE_BYTES <= RING_BYTES, "pair ring fits the ring");
static_assert(2 * PAIR_STAGES + 5 <= 28, "barriers fit their 256 bytes with the flags");
constexpr int SMEM_BYTES = 1024 + RING_BYTES + 256 + 4 * (MAX_GROUPS + 1 + 40);

enum Mode { DGRAD_DOWN = 0, DGRAD_UP = 1, WGRAD = 2 };

struct Args {
  int mode;
  int E;
  const int32_t* offsets;  // [E+1] kept rows of each expert (unpadded)
  const int32_t* poff;     // [E+1] the same rows, each expert's run padded to 64
  int M;                   // WGRAD: rows of each expert's weight gradient
  int N;                   // output columns
  int K;                   // DGRAD: contraction length
  int bn, n_tiles, m_tiles;  // m_tiles: WGRAD m-tiles per expert
  int64_t rows_cap;        // T*k
  void* out;
  const uint16_t* u;       // DGRAD_DOWN: pre-activations [rows_cap, N], 16-bit
  int u_f16;               // u is fp16 (else bf16)
  int act;                 // DGRAD_DOWN: 1 ReLU, 2 GELU
  int ab_f16;              // operand type: 1 fp16, 0 bf16
  int* err;
};

// DGRAD: m-tiles of tbm (128, or 256 for a pair) padded rows per expert; WGRAD: m_tiles
// per expert.  tp[e] = tiles before expert e (times n_tiles later).  Checks poff.  Every
// thread must call it.
__device__ bool bwd_tile_prefix(const Args& a, int* tp, int* scratch, int tbm) {
  if (threadIdx.x == 0) {
    tp[0] = 0;
    scratch[33] = 0;
  }
  __syncthreads();
  int carry = 0;
  for (int base = 0; base < a.E; base += blockDim.x) {
    const int e = base + threadIdx.x;
    int v = 0;
    if (e < a.E) {
      if (a.mode == WGRAD) {
        v = a.m_tiles;
      } else {
        const int p0 = a.poff[e], p1 = a.poff[e + 1];
        if (p0 < 0 || p1 < p0 || (p1 - p0) % 64 != 0 || p1 > a.rows_cap + 64LL * a.E)
          scratch[33] = 1;
        else
          v = (p1 - p0 + tbm - 1) / tbm;
      }
    }
    int tot;
    const int incl = block_incl_scan(v, scratch, &tot);
    if (e < a.E) tp[e + 1] = carry + incl;
    carry += tot;
  }
  __syncthreads();
  return scratch[33] == 0;
}

struct BTile {
  int e, mt, nt;
};

__device__ __forceinline__ BTile bwd_decode(int L, const int* tp, const Args& a) {
  int lo = 0, hi = a.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tp[mid] * a.n_tiles <= L) lo = mid; else hi = mid - 1;
  }
  BTile t;
  t.e = lo;
  const int local = L - tp[lo] * a.n_tiles;
  t.mt = local / a.n_tiles;
  t.nt = local - t.mt * a.n_tiles;
  return t;
}

__device__ __forceinline__ int bwd_kblocks(const Args& a, int e) {
  if (a.mode == WGRAD) return (__ldg(a.poff + e + 1) - __ldg(a.poff + e)) / BK;
  return a.K / BK;
}

// the derivative of the activation for ReLU (1) and identity (0); GELU pairs take
// gelu_grad2_as7126
__device__ __forceinline__ float act_grad(float u, int act) {
  if (act == 1) return u > 0.0f ? 1.0f : 0.0f;
  return 1.0f;
}

__device__ __forceinline__ float u16_to_float(uint16_t v, int f16) {
  if (f16) return __half2float(__ushort_as_half(v));
  return __bfloat162float(__ushort_as_bfloat16(v));
}

// PAIR = false: one CTA per SM, 128-row tiles (tcgen05 cta_group::1).
// PAIR = true: clusters of two CTAs share 256-row tiles (cta_group::2, M = 256): rank r
// loads rows [128 r, +128) of the tile's A (dgrad: padded expert rows; wgrad: weight
// rows, as two 64-column MN-major chunks) and B chunks [r bn/128, (r+1) bn/128) of the
// tile's bn columns, all completing on rank 0's full barrier; one thread of rank 0 issues
// the MMAs and commits to both CTAs' barriers; each CTA's epilogue reads its own 128 TMEM
// lanes and arrives on rank 0's accumulator-empty barrier.
template <bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int NST = PAIR ? PAIR_STAGES : STAGES;
  constexpr int SB = PAIR ? PAIR_STAGE_BYTES : STAGE_BYTES;
  constexpr int TBM = PAIR ? 2 * BM : BM;
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES);
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
  const bool wgrad = a.mode == WGRAD;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
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
  grid_dep_wait();
  grid_dep_launch();
  const bool ok = bwd_tile_prefix(a, tp, scratch, TBM);
  if (!ok && threadIdx.x == 0 && rank == 0) set_error(a.err, kErrOffsets);
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = ok ? tp[a.E] * a.n_tiles : 0;
  const int b_chunks = (PAIR ? a.bn / 2 : a.bn) / 64;  // B chunks this CTA loads
  const int b_chunk0 = static_cast<int>(rank) * b_chunks;
  const uint32_t b_bytes = static_cast<uint32_t>(b_chunks) * CHUNK;
  const uint32_t a_bytes = wgrad ? 2u * CHUNK : static_cast<uint32_t>(A_BYTES);
  const uint32_t stage_tx = (PAIR ? 2u : 1u) * (a_bytes + b_bytes);  // bytes per full phase
  // the full barrier every copy of a stage completes on: rank 0's in a pair
  auto full_bar = [&](int stage) -> uint32_t {
    return PAIR ? mapa_shared(full0 + 8 * stage, 0) : full0 + 8 * stage;
  };
  auto load = [&](uint32_t dst, const CUtensorMap* m, uint32_t fb, int c0, int c1) {
    if constexpr (PAIR) tma_load_2d_pair(dst, m, fb, c0, c1);
    else tma_load_2d(dst, m, fb, c0, c1);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool aborted = false;
      for (int L = first; L < total && !aborted; L += stride) {
        const BTile t = bwd_decode(L, tp, a);
        const int kblocks = bwd_kblocks(a, t.e);
        const int p0 = __ldg(a.poff + t.e), r0 = __ldg(a.offsets + t.e);
        const int m0 = t.mt * TBM + static_cast<int>(rank) * BM;  // this CTA's first row
        const int n0 = t.nt * a.bn + 64 * b_chunk0;                // this CTA's first column
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, s_abort)) {
            aborted = true;
            break;
          }
          const uint32_t st = smem_u32(ring + stage * SB);
          const uint32_t fb = full_bar(stage);
          if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * stage, stage_tx);
          if (wgrad) {
            // A: the padded rows p0 + 64 kb .. (contraction) x columns m0 .. (M)
            for (int c = 0; c < 2; ++c) load(st + c * CHUNK, &tmA, fb, m0 + 64 * c, p0 + kb * BK);
            // B: the unpadded rows r0 + 64 kb .. x columns n0 .. (N)
            for (int c = 0; c < b_chunks; ++c)
              load(st + A_BYTES + c * CHUNK, &tmB, fb, n0 + 64 * c, r0 + kb * BK);
          } else {
            // A: 128 padded rows, 64 contraction columns (K-major)
            load(st, &tmA, fb, kb * BK, p0 + m0);
            // B: weight rows e*K + 64 kb .. (contraction) x columns n0 .. (N-major)
            for (int c = 0; c < b_chunks; ++c)
              load(st + A_BYTES + c * CHUNK, &tmB, fb, n0 + 64 * c, t.e * a.K + kb * BK);
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
        // let every copy this thread started land before the CTA releases its smem (a
        // pair's second CTA cannot watch rank 0's barrier: it waits out a fixed drain time)
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
      const uint32_t idesc = idesc_f32acc_major(TBM, a.bn, a.ab_f16 ? kFmtF16 : kFmtBF16, wgrad, true);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool aborted = false;
      for (int L = first; L < total && !aborted; L += stride) {
        const BTile t = bwd_decode(L, tp, a);
        const int kblocks = bwd_kblocks(a, t.e);
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
            const uint64_t ad = wgrad ? sdesc_mn128(a0 + kk * 2048, CHUNK) : sdesc_k128(a0 + kk * 32);
            if constexpr (PAIR)
              tc_mma_pair_f16kind(d_tmem, ad, sdesc_mn128(b0 + kk * 2048, CHUNK), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma_f16kind(d_tmem, ad, sdesc_mn128(b0 + kk * 2048, CHUNK), idesc,
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
        // also with no k-block: the epilogue writes zeros
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
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const uint32_t tempty_peer0 = PAIR ? mapa_shared(tempty0, 0) : tempty0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int L = first; L < total; L += stride) {
      const BTile t = bwd_decode(L, tp, a);
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, s_abort)) {
        if (lane == 0) set_error(a.err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const int r = q * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256;
      const int col0 = t.nt * a.bn;
      if (wgrad) {
        const int m = t.mt * TBM + static_cast<int>(rank) * BM + r;
        const bool any = bwd_kblocks(a, t.e) > 0;
        float* dst_row = static_cast<float*>(a.out) +
                         (static_cast<int64_t>(t.e) * a.M + m) * a.N + col0;
        for (int c = sub * 32; c < a.bn; c += 32 * EPI_SUBS) {
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (m >= a.M) continue;
          if (!any) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0u;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_global_v8(dst_row + c + 8 * j, v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3],
                         v[8 * j + 4], v[8 * j + 5], v[8 * j + 6], v[8 * j + 7]);
        }
      } else {
        const int p0 = __ldg(a.poff + t.e), p1 = __ldg(a.poff + t.e + 1);
        const int r0 = __ldg(a.offsets + t.e), r1 = __ldg(a.offsets + t.e + 1);
        const int i = t.mt * TBM + static_cast<int>(rank) * BM + r;  // row in the padded run
        const bool kept = i < r1 - r0;
        const bool pad = !kept && i < p1 - p0;
        const int64_t s = r0 + i;            // unpadded row of a kept one
        for (int c = sub * 32; c < a.bn; c += 32 * EPI_SUBS) {
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (a.mode == DGRAD_DOWN) {
            if (!kept && !pad) continue;
            uint32_t pk[16];
            if (kept) {
              const uint4* up = reinterpret_cast<const uint4*>(a.u + s * a.N + col0 + c);
              uint32_t uw[16];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint4 w4 = __ldg(up + j);
                uw[4 * j] = w4.x; uw[4 * j + 1] = w4.y; uw[4 * j + 2] = w4.z; uw[4 * j + 3] = w4.w;
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float u0 = u16_to_float(static_cast<uint16_t>(uw[j] & 0xFFFFu), a.u_f16);
                const float u1 = u16_to_float(static_cast<uint16_t>(uw[j] >> 16), a.u_f16);
                float g0, g1;
                if (a.act == 2) {
                  gelu_grad2_as7126(u0, u1, g0, g1);
                } else {
                  g0 = act_grad(u0, a.act);
                  g1 = act_grad(u1, a.act);
                }
                pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * g0, __uint_as_float(v[2 * j + 1]) * g1);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) pk[j] = 0u;  // padding rows of du are zero
            }
            uint16_t* dst = static_cast<uint16_t*>(a.out) + (p0 + static_cast<int64_t>(i)) * a.N +
                            col0 + c;
            st_global_v8(dst, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            st_global_v8(dst + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
          } else {  // DGRAD_UP: dx_perm at the unpadded row
            if (!kept) continue;
            float* dst = static_cast<float*>(a.out) + s * a.N + col0 + c;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_global_v8(dst + 8 * j, v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3],
                           v[8 * j + 4], v[8 * j + 5], v[8 * j + 6], v[8 * j + 7]);
          }
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
    }
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

}  // namespace bw

// ------------------------------------------------------------ small backward kernels

// poff[e] = 64 * sum_{e' < e} ceil(n_e' / 64) for the kept rows n_e of offsets.
__global__ void pad_offsets_kernel(const int32_t* __restrict__ offsets, int E, int64_t rows_cap,
                                   int32_t* __restrict__ poff, int* err) {
  extern __shared__ int psm[];
  int* scratch = psm;       // 40
  int* tp = psm + 40;       // E + 1
  grid_dep_wait();
  grid_dep_launch();
  const bool ok = block_tile_prefix(offsets, E, rows_cap, 64, tp, scratch);
  if (!ok) {
    if (threadIdx.x == 0) set_error(err, kErrOffsets);
    for (int e = threadIdx.x; e <= E; e += blockDim.x) poff[e] = 0;
    return;
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) poff[e] = 64 * tp[e];
}

// One warp per token: d_o[padded row] = G_tj dy[t] (16-bit) for each kept assignment and
// dgate[t, j] = <dy[t], y_perm[slot]> (0 for a dropped one), summed in a fixed order.
__global__ void __launch_bounds__(256)
    combine_bwd_kernel(const float* __restrict__ dy, const float* __restrict__ y_perm,
                       const int32_t* __restrict__ slot_pos, const int32_t* __restrict__ topk_idx,
                       const float* __restrict__ gate, const int32_t* __restrict__ offsets,
                       const int32_t* __restrict__ poff, uint16_t* __restrict__ d_o, int d_o_f16,
                       float* __restrict__ dgate, int64_t T, int k, int E, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  grid_dep_wait();
  grid_dep_launch();
  if (t >= T) return;
  const float4* dyr = reinterpret_cast<const float4*>(dy + t * d);
  for (int j = 0; j < k; ++j) {
    const int s = slot_pos[t * k + j];
    const int e = topk_idx[t * k + j];
    if (s < 0 || e < 0 || e >= E) {
      if (lane == 0) dgate[t * k + j] = 0.0f;
      continue;
    }
    const float g = gate[t * k + j];
    const int64_t p = poff[e] + (s - offsets[e]);
    const float4* yr = reinterpret_cast<const float4*>(y_perm + static_cast<int64_t>(s) * d);
    uint2* orow = reinterpret_cast<uint2*>(d_o + p * d);
    float dot = 0.0f;
    for (int v = lane; v < d / 4; v += 32) {
      const float4 a4 = __ldg(dyr + v), y4 = __ldg(yr + v);
      dot = fmaf(a4.x, y4.x, dot);
      dot = fmaf(a4.y, y4.y, dot);
      dot = fmaf(a4.z, y4.z, dot);
      dot = fmaf(a4.w, y4.w, dot);
      orow[v] = d_o_f16 ? make_uint2(pack_f16x2(g * a4.x, g * a4.y), pack_f16x2(g * a4.z, g * a4.w))
                        : make_uint2(pack_bf16x2(g * a4.x, g * a4.y), pack_bf16x2(g * a4.z, g * a4.w));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) dgate[t * k + j] = dot;
  }
}

// Zeroes the padding rows [poff[e] + n_e, poff[e+1]) of a padded 16-bit row buffer
// [*, d]: one block per expert.
__global__ void pad_zero_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff,
                                uint16_t* __restrict__ buf, int d) {
  const int e = blockIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  const int64_t a = poff[e] + (offsets[e + 1] - offsets[e]);
  const int64_t b = poff[e + 1];
  uint4* p = reinterpret_cast<uint4*>(buf + a * d);
  const int64_t n = (b - a) * d / 8;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) p[i] = make_uint4(0, 0, 0, 0);
}

// One warp per token: dx[t] = sum_j dx_perm[slot(t, j)] over the kept assignments, in
// the order j = 0 .. k-1 (0 for a token with none).
__global__ void __launch_bounds__(256)
    unpermute_kernel(const float* __restrict__ dx_perm, const int32_t* __restrict__ slot_pos,
                     float* __restrict__ dx, int64_t T, int k, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  grid_dep_wait();
  grid_dep_launch();
  if (t >= T) return;
  float4* out = reinterpret_cast<float4*>(dx + t * d);
  for (int v = lane; v < d / 4; v += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int s = slot_pos[t * k + j];
      if (s < 0) continue;
      const float4 r = __ldg(reinterpret_cast<const float4*>(dx_perm + static_cast<int64_t>(s) * d) + v);
      acc.x += r.x; acc.y += r.y; acc.z += r.z; acc.w += r.w;
    }
    out[v] = acc;
  }
}

// d CV(v)^2 / dv_i = 2 (v_i - m) / (n m^2) - 2 var / (n m^3), population variance, times
// the loss weight; one block, sums in index order.  losses[0] += w * CV^2 when given.
__global__ void cv2_grad_kernel(const float* __restrict__ v, int n, float w, float* __restrict__ grad,
                                float* losses, int which) {
  __shared__ float s_m, s_var;
  grid_dep_wait();
  grid_dep_launch();
  if (threadIdx.x == 0) {
    double sum = 0.0;
    for (int i = 0; i < n; ++i) sum += v[i];
    const double m = sum / n;
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += (v[i] - m) * (v[i] - m);
    s_m = static_cast<float>(m);
    s_var = static_cast<float>(ss / n);
    if (losses) losses[which] = static_cast<float>(w * (ss / n) / (m * m));
  }
  __syncthreads();
  const float m = s_m, var = s_var;
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    grad[i] = w * (2.0f * (v[i] - m) / (n * m * m) - 2.0f * var / (n * m * m * m));
}

// Softplus(z) as the router computes it, and its derivative sigmoid(z).
// Gate backward, one thread per token over its E score columns.  Every [E, T] array is
// read and written at e * T + t, so a warp's 32 tokens touch 128 contiguous bytes.
//   dgate [T, k]: gradient of L with respect to each chosen gate (from combine_bwd)
//   dimp [E] (or null): the Importance loss gradient, added to every chosen gate's
//   lg [E, T]: the forward's clean logits x.W_g (+ bias)
//   noisy gating: sw [E, T] Softplus(x.W_noise) and hw [E, T] the noisy scores H, both as
//   the forward computed them, the noise [T, E], and dload [E] (or null): the Load loss
//   gradient
// Writes dl [E, T] (gradient of the clean logits) and, for noisy gating, dz [E, T]
// (gradient of x.W_noise).  topk_gate holds the forward's gates: the chosen experts'
// Softmax(KeepTopK) values, or for the Switch gate their full-softmax values.
__global__ void __launch_bounds__(128)
    gate_bwd_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_gate,
                    const float* __restrict__ dgate, const float* __restrict__ dimp,
                    const float* __restrict__ lg, const float* __restrict__ sw,
                    const float* __restrict__ hw, const float* __restrict__ noise,
                    const float* __restrict__ dload, float* __restrict__ dl, float* __restrict__ dz,
                    int64_t T, int E, int k, int noisy, int renorm) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  if (t >= T) return;
  // the chosen experts (k <= 8), their gates G_j and gradients dg_j; S = sum_j G_j dg_j
  int ci[8];
  float cg[8], cd[8];
  float S = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ci[j] = -1;
    cg[j] = cd[j] = 0.0f;
    if (j < k) {
      ci[j] = topk_idx[t * k + j];
      cg[j] = topk_gate[t * k + j];
      cd[j] = dgate[t * k + j] + (dimp ? dimp[ci[j]] : 0.0f);
      S += cg[j] * cd[j];
    }
  }
  // Softmax(KeepTopK): d score_e = G_e (dg_e - S) at the chosen experts, 0 elsewhere
  auto keep_part = [&](int e) {
    float v = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (ci[j] == e) v = cg[j] * (cd[j] - S);
    return v;
  };
  if (!noisy) {
    if (renorm) {
      for (int e = 0; e < E; ++e) dl[e * T + t] = keep_part(e);
    } else {
      // Switch gate: p = softmax over all logits; d score_e = p_e (dp_e - S) with dp
      // nonzero only at the chosen experts, where p_e = G_e
      float m = -INFINITY;
      for (int e = 0; e < E; ++e) m = fmaxf(m, lg[e * T + t]);
      float z = 0.0f;
      for (int e = 0; e < E; ++e) z += expf(lg[e * T + t] - m);
      for (int e = 0; e < E; ++e) {
        float v = -(expf(lg[e * T + t] - m) / z) * S;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (ci[j] == e) v += cg[j] * cd[j];
        dl[e * T + t] = v;
      }
    }
    return;
  }
  // noisy gating: the scores are H = l + n Softplus(z), so far d score = dH; Softplus'(z)
  // = sigmoid(z) = 1 - exp(-Softplus(z))
  const float* nrow = noise + t * E;
  if (dload == nullptr) {
    for (int e = 0; e < E; ++e) {
      const float dH = keep_part(e);
      dl[e * T + t] = dH;
      dz[e * T + t] = dH * nrow[e] * -expm1f(-sw[e * T + t]);
    }
    return;
  }
  // kth_excluding(H, k, i) is the (k+1)-th largest H when H_i is among the k largest
  // (H_i >= the k-th largest value), else the k-th largest, ranked by (-H, index): one
  // pass keeps the k+1 largest (k <= 8) in ascending expert order, so an equal later value
  // never displaces an earlier one
  float tv[9];
  int ti[9];
#pragma unroll
  for (int j = 0; j < 9; ++j) {
    tv[j] = -INFINITY;
    ti[j] = 0;
  }
  for (int e = 0; e < E; ++e) {
    float cv = hw[e * T + t];
    int cix = e;
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      if (j <= k && cv > tv[j]) {
        const float sv = tv[j];
        const int si = ti[j];
        tv[j] = cv;
        ti[j] = cix;
        cv = sv;
        cix = si;
      }
    }
  }
  float hk = tv[0], hk1 = tv[1];
  int pk = ti[0], pk1 = ti[1];
#pragma unroll
  for (int j = 1; j < 9; ++j)
    if (j == k) {
      hk = tv[j - 1];
      pk = ti[j - 1];
      hk1 = tv[j];
      pk1 = ti[j];
    }
  // P(x, e) = Phi(zeta), zeta = (l_e - kth_excluding) / Softplus(z_e): its gradient goes to
  // l_e, to Softplus(z_e), and to H at the entry kth_excluding picked (pk or pk1), whose
  // totals are gathered first
  float to_pk = 0.0f, to_pk1 = 0.0f;
  for (int e = 0; e < E; ++e) {
    const float sp = sw[e * T + t];
    const bool top = hw[e * T + t] >= hk;
    const float zeta = (lg[e * T + t] - (top ? hk1 : hk)) / sp;
    const float g = dload[e] * 0.3989422804014327f * expf(-0.5f * zeta * zeta);
    if (top) to_pk1 -= g / sp;
    else to_pk -= g / sp;
  }
  for (int e = 0; e < E; ++e) {
    const float sp = sw[e * T + t];
    const bool top = hw[e * T + t] >= hk;
    const float zeta = (lg[e * T + t] - (top ? hk1 : hk)) / sp;
    const float g = dload[e] * 0.3989422804014327f * expf(-0.5f * zeta * zeta);
    const float dH = keep_part(e) + (e == pk ? to_pk : 0.0f) + (e == pk1 ? to_pk1 : 0.0f);
    dz[e * T + t] = (dH * nrow[e] - g * zeta / sp) * -expm1f(-sp);
    dl[e * T + t] = dH + g / sp;
  }
}

// ------------------------------------------------------------- router products
//
// The router's gradients from dl (and dz) [R, T] (R = E, or 2E with dz below dl):
//   dx[t, n]  += sum_r A[r, t] B[r, n],  B = W_g (rows r < E) and W_noise (rows E..2E-1)
//   dW[r, n]   = sum_t A[r, t] x[t, n]   (dW_g, dW_noise)
//   dbias[e]   = sum_t dl[e, t]
// SIMT fp32 arithmetic on coalesced tiles: every operand row is read along its contiguous
// dimension.

namespace rx {
constexpr int TT = 32, TN = 256, TR = 32, THREADS = 256;
}

// dx += A^T B over a 32-token x 256-column tile per block, r in chunks of 32; each thread
// holds 8 tokens x 4 columns.
__global__ void __launch_bounds__(rx::THREADS)
    router_dx_kernel(const float* __restrict__ A, const __nv_bfloat16* __restrict__ B0,
                     const __nv_bfloat16* __restrict__ B1, int E, int R, int64_t T, int d,
                     float* __restrict__ dx) {
  __shared__ __align__(16) float sA[rx::TR][rx::TT];
  __shared__ __align__(16) __nv_bfloat16 sB[rx::TR][rx::TN];
  const int tid = threadIdx.x, tx = tid & 63, ty = tid >> 6;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * rx::TT;
  const int n0 = blockIdx.y * rx::TN;
  grid_dep_wait();
  grid_dep_launch();
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int r0 = 0; r0 < R; r0 += rx::TR) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // A tile: 32 rows x 32 tokens, along the tokens
      const int idx = tid + i * rx::THREADS, r = idx >> 5, tt = idx & 31;
      sA[r][tt] = (r0 + r < R && t0 + tt < T) ? __ldg(A + (r0 + r) * T + t0 + tt) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // B tile: 32 rows x 256 columns, 8 columns per load
      const int idx = tid + i * rx::THREADS, r = idx >> 5, c8 = (idx & 31) * 8;
      const int row = r0 + r, col = n0 + c8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row < R && col < d) {
        const __nv_bfloat16* src = row < E ? B0 + static_cast<int64_t>(row) * d
                                           : B1 + static_cast<int64_t>(row - E) * d;
        v = __ldg(reinterpret_cast<const uint4*>(src + col));
      }
      *reinterpret_cast<uint4*>(&sB[r][c8]) = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < rx::TR; ++r) {
      const float4 a0 = *reinterpret_cast<const float4*>(&sA[r][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sA[r][ty * 8 + 4]);
      const uint2 bb = *reinterpret_cast<const uint2*>(&sB[r][tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[4] = {__uint_as_float(bb.x << 16), __uint_as_float(bb.x & 0xFFFF0000u),
                          __uint_as_float(bb.y << 16), __uint_as_float(bb.y & 0xFFFF0000u)};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int n = n0 + tx * 4;
  if (n >= d) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + ty * 8 + i;
    if (t >= T) break;
    float4* p = reinterpret_cast<float4*>(dx + t * d + n);
    float4 v = *p;
    v.x += acc[i][0];
    v.y += acc[i][1];
    v.z += acc[i][2];
    v.w += acc[i][3];
    *p = v;
  }
}

namespace rw {
constexpr int TT = 64, TN = 256, THREADS = 128;
}

// part[z][r][n] = sum over the tokens of chunk z of A[r, t] x[t, n] for the block's RG rows
// of A (from blockIdx.y * RG) and 256 columns (two per thread); the chunk's tokens pass
// through shared memory 64 at a time, A transposed there so that a token's RG values are
// read as float4s.
template <int RG>
__global__ void __launch_bounds__(rw::THREADS)
    router_wgrad_kernel(const float* __restrict__ A, int R, int64_t T,
                        const __nv_bfloat16* __restrict__ x, int d, int64_t tchunk,
                        float* __restrict__ part) {
  __shared__ __align__(16) float sA[rw::TT][RG + 4];
  const int tid = threadIdx.x;
  const int n = blockIdx.x * rw::TN + 2 * tid;
  const int r0 = blockIdx.y * RG;
  const int64_t lo = static_cast<int64_t>(blockIdx.z) * tchunk;
  const int64_t hi = min(T, lo + tchunk);
  grid_dep_wait();
  grid_dep_launch();
  float acc0[RG], acc1[RG];
#pragma unroll
  for (int r = 0; r < RG; ++r) acc0[r] = acc1[r] = 0.0f;
  const bool col_ok = n < d;
  for (int64_t t0 = lo; t0 < hi; t0 += rw::TT) {
    for (int idx = tid; idx < RG * rw::TT; idx += rw::THREADS) {
      const int r = idx / rw::TT, tt = idx % rw::TT;
      sA[tt][r] = (r0 + r < R && t0 + tt < hi) ? __ldg(A + (r0 + r) * T + t0 + tt) : 0.0f;
    }
    __syncthreads();
    const int nt = static_cast<int>(min(static_cast<int64_t>(rw::TT), hi - t0));
#pragma unroll 4
    for (int tt = 0; tt < nt; ++tt) {
      float x0 = 0.0f, x1 = 0.0f;
      if (col_ok) {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(x + (t0 + tt) * d + n));
        x0 = __uint_as_float(v << 16);
        x1 = __uint_as_float(v & 0xFFFF0000u);
      }
#pragma unroll
      for (int r = 0; r < RG; r += 4) {
        const float4 a = *reinterpret_cast<const float4*>(&sA[tt][r]);
        acc0[r] = fmaf(a.x, x0, acc0[r]);
        acc1[r] = fmaf(a.x, x1, acc1[r]);
        acc0[r + 1] = fmaf(a.y, x0, acc0[r + 1]);
        acc1[r + 1] = fmaf(a.y, x1, acc1[r + 1]);
        acc0[r + 2] = fmaf(a.z, x0, acc0[r + 2]);
        acc1[r + 2] = fmaf(a.z, x1, acc1[r + 2]);
        acc0[r + 3] = fmaf(a.w, x0, acc0[r + 3]);
        acc1[r + 3] = fmaf(a.w, x1, acc1[r + 3]);
      }
    }
    __syncthreads();
  }
  if (!col_ok) return;
#pragma unroll
  for (int r = 0; r < RG; ++r)
    if (r0 + r < R)
      *reinterpret_cast<float2*>(part + (static_cast<int64_t>(blockIdx.z) * R + r0 + r) * d + n) =
          make_float2(acc0[r], acc1[r]);
}

// dW_g[r, n] (r < E) and dW_noise[r - E, n] (r >= E) = sum_z part[z][r][n], z in order.
__global__ void sum_router_wgrad_kernel(const float* __restrict__ part, int chunks, int E, int R,
                                        int d, float* __restrict__ dwg, float* __restrict__ dwn) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  if (i >= static_cast<int64_t>(R) * d) return;
  float s = 0.0f;
  for (int z = 0; z < chunks; ++z) s += part[static_cast<int64_t>(z) * R * d + i];
  const int64_t r = i / d;
  if (r < E) dwg[i] = s;
  else dwn[i - static_cast<int64_t>(E) * d] = s;
}

// out[e] = sum_t A[e, t] for a row-major [E, T] matrix: one block per row, each thread a
// fixed strided subset in order, then a fixed tree over the block.
__global__ void __launch_bounds__(256)
    rowsum_kernel(const float* __restrict__ A, int64_t T, float* __restrict__ out) {
  const float* row = A + static_cast<int64_t>(blockIdx.x) * T;
  grid_dep_wait();
  grid_dep_launch();
  float s = 0.0f;
  for (int64_t t = threadIdx.x; t < T; t += 256) s += __ldg(row + t);
  s = block_sum_fixed<256>(s);
  if (threadIdx.x == 0) out[blockIdx.x] = s;
}

// ------------------------------------------------------------------ host side

namespace {

int pick_bn_bwd(int N) {
  if (N % 256 == 0) return 256;
  if (N % 128 == 0) return 128;
  return 64;
}

// 2-D tensor map of 16-bit elements over [rows, cols] with a [box_rows x 64] box.
bool tmap16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, int f16) {
  return make_tmap_2b(m, base, static_cast<uint64_t>(rows), static_cast<uint64_t>(cols),
                      static_cast<uint32_t>(box_rows), f16);
}

// Clusters of two CTAs of bwd_gemm_kernel<true> that fit on the device at once, looked up
// once per context.
int bwd_max_active_pairs(const LaunchCtx& c) {
  static std::mutex mu;
  static std::map<unsigned long long, int> cache;
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) != cudaSuccess) return c.num_sms / 2;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(ctx);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (c.num_sms / 2));
  cfg.blockDim = dim3(bw::THREADS);
  cfg.dynamicSmemBytes = bw::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, bw::bwd_gemm_kernel<true>, &cfg) != cudaSuccess || n <= 0)
    n = c.num_sms / 2;
  if (n > c.num_sms / 2) n = c.num_sms / 2;
  cache[ctx] = n;
  return n;
}

// Experts with at least this many rows on average (T*k / E) run their products on CTA
// pairs (256-row tiles), as the forward pass does.
constexpr int64_t kBwdPairMinRowsPerExpert = 256;

// One product: pairs when the experts are large enough, B's bn columns split into whole
// 64-column chunks per CTA, and (weight gradients) the M rows into 256-row tiles.  Sets
// a.m_tiles for the weight gradients.  prows: rows of the padded layout.
cudaError_t launch_bwd_gemm(bw::Args a, const CUtensorMap& tmA, const CUtensorMap& tmB,
                            int64_t prows, const LaunchCtx& c) {
  const bool wg = a.mode == bw::WGRAD;
  const bool pair = a.bn >= 128 && a.rows_cap >= kBwdPairMinRowsPerExpert * a.E &&
                    (!wg || a.M % (2 * bw::BM) == 0);
  const int tbm = pair ? 2 * bw::BM : bw::BM;
  if (wg) a.m_tiles = (a.M + tbm - 1) / tbm;
  const int64_t max_tiles = wg ? static_cast<int64_t>(a.E) * a.m_tiles * a.n_tiles
                               : (prows / tbm + a.E) * static_cast<int64_t>(a.n_tiles);
  if (pair) {
    cudaError_t e = ensure_smem_limit(bw::bwd_gemm_kernel<true>, bw::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int64_t cap = bwd_max_active_pairs(c);
    const int pairs = static_cast<int>(max_tiles < cap ? max_tiles : cap);
    if (pairs <= 0) return cudaSuccess;
    return launch_kernel_pairs(bw::bwd_gemm_kernel<true>, dim3(2 * pairs), dim3(bw::THREADS),
                               bw::SMEM_BYTES, c, tmA, tmB, a);
  }
  const int grid = static_cast<int>(max_tiles < c.num_sms ? max_tiles : c.num_sms);
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = ensure_smem_limit(bw::bwd_gemm_kernel<false>, bw::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(bw::bwd_gemm_kernel<false>, dim3(grid), dim3(bw::THREADS), bw::SMEM_BYTES,
                       c, tmA, tmB, a);
}

}  // namespace

int64_t backward_padded_rows(int64_t rows_cap, int E) { return rows_cap + 64LL * E; }

cudaError_t launch_backward(const BackwardProblem& p, const LaunchCtx& c) {
  const int64_t n = p.T * p.k;
  const int64_t prows = backward_padded_rows(n, p.E);
  const int d = p.d, f = p.f, E = p.E;
  const int w2f16 = p.hidden_f16;
  cudaError_t e;
  // ---- padded row ranges
  e = launch_kernel(pad_offsets_kernel, dim3(1), dim3(1024), (E + 1 + 40) * sizeof(int), c,
                    p.offsets, E, n, p.poff, c.err);
  if (e != cudaSuccess) return e;
  // ---- combine backward: d_o (padded, in W2's type) and dgate
  e = launch_kernel(pad_zero_kernel, dim3(E), dim3(256), 0, c, static_cast<const int32_t*>(p.offsets),
                    static_cast<const int32_t*>(p.poff), static_cast<uint16_t*>(p.d_o), d);
  if (e != cudaSuccess) return e;
  e = launch_kernel(combine_bwd_kernel, dim3(static_cast<unsigned>((p.T + 7) / 8)), dim3(256), 0, c,
                    p.dy, p.y_perm, p.slot_pos, p.topk_idx, p.topk_gate, p.offsets,
                    static_cast<const int32_t*>(p.poff), static_cast<uint16_t*>(p.d_o), w2f16, p.dgate,
                    p.T, p.k, E, d);
  if (e != cudaSuccess) return e;

  // ---- expert products on the tensor cores
  {  // du = (d_o . W2_e) * act'(u): M = padded rows, N = f, K = d; W2 [E, d, f] as [E*d, f]
    bw::Args a = {};
    a.mode = bw::DGRAD_DOWN; a.E = E; a.offsets = p.offsets; a.poff = p.poff;
    a.N = f; a.K = d; a.bn = pick_bn_bwd(f); a.n_tiles = f / a.bn; a.rows_cap = n;
    a.out = p.du; a.u = static_cast<const uint16_t*>(p.u); a.u_f16 = p.hidden_f16; a.act = p.act;
    a.ab_f16 = w2f16; a.err = c.err;
    CUtensorMap tA, tB;
    if (!tmap16(&tA, p.d_o, prows, d, bw::BM, w2f16) ||
        !tmap16(&tB, p.w2, static_cast<int64_t>(E) * d, f, 64, w2f16))
      return cudaErrorInvalidValue;
    e = launch_bwd_gemm(a, tA, tB, prows, c);
    if (e != cudaSuccess) return e;
  }
  {  // dW2_e = d_o_e^T . h_e: M = d, N = f, contraction over the expert's rows
    bw::Args a = {};
    a.mode = bw::WGRAD; a.E = E; a.offsets = p.offsets; a.poff = p.poff;
    a.M = d; a.N = f; a.bn = pick_bn_bwd(f); a.n_tiles = f / a.bn;
    a.rows_cap = n; a.out = p.dw2; a.ab_f16 = w2f16; a.err = c.err;
    CUtensorMap tA, tB;
    if (!tmap16(&tA, p.d_o, prows, d, 64, w2f16) || !tmap16(&tB, p.h, n, f, 64, w2f16))
      return cudaErrorInvalidValue;
    e = launch_bwd_gemm(a, tA, tB, prows, c);
    if (e != cudaSuccess) return e;
  }
  {  // dx_perm = du . W1_e: M = padded rows, N = d, K = f; W1 [E, f, d] as [E*f, d]
    bw::Args a = {};
    a.mode = bw::DGRAD_UP; a.E = E; a.offsets = p.offsets; a.poff = p.poff;
    a.N = d; a.K = f; a.bn = pick_bn_bwd(d); a.n_tiles = d / a.bn; a.rows_cap = n;
    a.out = p.dx_perm; a.ab_f16 = 0; a.err = c.err;
    CUtensorMap tA, tB;
    if (!tmap16(&tA, p.du, prows, f, bw::BM, 0) ||
        !tmap16(&tB, p.w1, static_cast<int64_t>(E) * f, d, 64, 0))
      return cudaErrorInvalidValue;
    e = launch_bwd_gemm(a, tA, tB, prows, c);
    if (e != cudaSuccess) return e;
  }
  {  // dW1_e = du_e^T . x_perm_e: M = f, N = d
    bw::Args a = {};
    a.mode = bw::WGRAD; a.E = E; a.offsets = p.offsets; a.poff = p.poff;
    a.M = f; a.N = d; a.bn = pick_bn_bwd(d); a.n_tiles = d / a.bn;
    a.rows_cap = n; a.out = p.dw1; a.ab_f16 = 0; a.err = c.err;
    CUtensorMap tA, tB;
    if (!tmap16(&tA, p.du, prows, f, 64, 0) || !tmap16(&tB, p.x_perm, n, d, 64, 0))
      return cudaErrorInvalidValue;
    e = launch_bwd_gemm(a, tA, tB, prows, c);
    if (e != cudaSuccess) return e;
  }
  e = launch_kernel(unpermute_kernel, dim3(static_cast<unsigned>((p.T + 7) / 8)), dim3(256), 0, c,
                    static_cast<const float*>(p.dx_perm), p.slot_pos, p.dx, p.T, p.k, d);
  if (e != cudaSuccess) return e;

  // ---- auxiliary loss gradients
  if (p.w_importance != 0.0f) {
    e = launch_kernel(cv2_grad_kernel, dim3(1), dim3(256), 0, c, p.importance, E, p.w_importance,
                      p.dimp, p.losses, 0);
    if (e != cudaSuccess) return e;
  }
  if (p.w_load != 0.0f) {
    e = launch_kernel(cv2_grad_kernel, dim3(1), dim3(256), 0, c, p.load, E, p.w_load, p.dload,
                      p.losses, 1);
    if (e != cudaSuccess) return e;
  }
  // ---- router: gate backward from the forward's scores, then the parameter gradients
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* wg = static_cast<const __nv_bfloat16*>(p.w_gate);
  const __nv_bfloat16* wn = static_cast<const __nv_bfloat16*>(p.w_noise);
  e = launch_kernel(gate_bwd_kernel, dim3(static_cast<unsigned>((p.T + 127) / 128)), dim3(128), 0, c,
                    p.topk_idx, p.topk_gate, static_cast<const float*>(p.dgate),
                    static_cast<const float*>(p.w_importance != 0.0f ? p.dimp : nullptr), p.lg, p.sw,
                    p.hw, p.noise, static_cast<const float*>(p.w_load != 0.0f ? p.dload : nullptr),
                    p.dl, p.dz, p.T, E, p.k, p.noisy, p.renorm);
  if (e != cudaSuccess) return e;
  // A = dl (and dz below it): R rows of [T]
  const int R = p.noisy ? 2 * E : E;
  const float* A = p.dl;
  // dx += A^T [W_g; W_noise]
  e = launch_kernel(router_dx_kernel,
                    dim3(static_cast<unsigned>((p.T + rx::TT - 1) / rx::TT), (d + rx::TN - 1) / rx::TN),
                    dim3(rx::THREADS), 0, c, A, wg, wn, E, R, p.T, d, p.dx);
  if (e != cudaSuccess) return e;
  // [dW_g; dW_noise] = A x, as partial sums over token chunks summed in chunk order
  {
    const int rg = R <= 8 ? 8 : R <= 16 ? 16 : 32;
    const int gx = (d + rw::TN - 1) / rw::TN, gy = (R + rg - 1) / rg;
    int64_t chunks = (2LL * c.num_sms + gx * gy - 1) / (gx * gy);
    const int64_t by_cap = p.part_cap / (static_cast<int64_t>(R) * d);
    const int64_t by_t = (p.T + rw::TT - 1) / rw::TT;
    if (chunks > by_cap) chunks = by_cap;
    if (chunks > by_t) chunks = by_t;
    if (chunks < 1) chunks = 1;
    int64_t tchunk = (p.T + chunks - 1) / chunks;
    tchunk = (tchunk + rw::TT - 1) / rw::TT * rw::TT;
    chunks = (p.T + tchunk - 1) / tchunk;
    const dim3 grid(gx, gy, static_cast<unsigned>(chunks));
    switch (rg) {
      case 8: e = launch_kernel(router_wgrad_kernel<8>, grid, dim3(rw::THREADS), 0, c, A, R, p.T, x, d, tchunk, p.part); break;
      case 16: e = launch_kernel(router_wgrad_kernel<16>, grid, dim3(rw::THREADS), 0, c, A, R, p.T, x, d, tchunk, p.part); break;
      default: e = launch_kernel(router_wgrad_kernel<32>, grid, dim3(rw::THREADS), 0, c, A, R, p.T, x, d, tchunk, p.part); break;
    }
    if (e != cudaSuccess) return e;
    const int64_t nout = static_cast<int64_t>(R) * d;
    e = launch_kernel(sum_router_wgrad_kernel, dim3(static_cast<unsigned>((nout + 255) / 256)), dim3(256), 0,
                      c, static_cast<const float*>(p.part), static_cast<int>(chunks), E, R, d, p.dw_gate,
                      p.dw_noise);
    if (e != cudaSuccess) return e;
  }
  if (p.dbias) {
    e = launch_kernel(rowsum_kernel, dim3(E), dim3(256), 0, c, static_cast<const float*>(p.dl), p.T,
                      p.dbias);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace moe
