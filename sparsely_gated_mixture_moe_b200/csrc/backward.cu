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

// DGRAD: m-tiles of 128 padded rows per expert; WGRAD: m_tiles per expert.  tp[e] = tiles
// before expert e (times n_tiles later).  Checks poff.  Every thread must call it.
__device__ bool bwd_tile_prefix(const Args& a, int* tp, int* scratch) {
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
          v = (p1 - p0 + BM - 1) / BM;
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

__global__ void __launch_bounds__(THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* scratch = reinterpret_cast<int*>(smem + RING_BYTES + 256);
  int* tp = scratch + 40;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool wgrad = a.mode == WGRAD;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, EPI_WARPS);
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
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  grid_dep_wait();
  grid_dep_launch();
  const bool ok = bwd_tile_prefix(a, tp, scratch);
  if (!ok && threadIdx.x == 0) set_error(a.err, kErrOffsets);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = ok ? tp[a.E] * a.n_tiles : 0;
  const int b_chunks = a.bn / 64;
  const uint32_t b_bytes = static_cast<uint32_t>(b_chunks) * CHUNK;
  const uint32_t a_bytes = wgrad ? 2u * CHUNK : static_cast<uint32_t>(A_BYTES);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool aborted = false;
      for (int L = blockIdx.x; L < total && !aborted; L += gridDim.x) {
        const BTile t = bwd_decode(L, tp, a);
        const int kblocks = bwd_kblocks(a, t.e);
        const int p0 = __ldg(a.poff + t.e), r0 = __ldg(a.offsets + t.e);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, s_abort)) {
            aborted = true;
            break;
          }
          const uint32_t st = smem_u32(ring + stage * STAGE_BYTES);
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, a_bytes + b_bytes);
          if (wgrad) {
            // A: the padded rows p0 + 64 kb .. (contraction) x columns mt*128 .. (M)
            for (int c = 0; c < 2; ++c)
              tma_load_2d(st + c * CHUNK, &tmA, fb, t.mt * BM + 64 * c, p0 + kb * BK);
            // B: the unpadded rows r0 + 64 kb .. x columns nt*bn .. (N)
            for (int c = 0; c < b_chunks; ++c)
              tma_load_2d(st + A_BYTES + c * CHUNK, &tmB, fb, t.nt * a.bn + 64 * c, r0 + kb * BK);
          } else {
            // A: 128 padded rows, 64 contraction columns (K-major)
            tma_load_2d(st, &tmA, fb, kb * BK, p0 + t.mt * BM);
            // B: weight rows e*K + 64 kb .. (contraction) x columns nt*bn .. (N-major)
            for (int c = 0; c < b_chunks; ++c)
              tma_load_2d(st + A_BYTES + c * CHUNK, &tmB, fb, t.nt * a.bn + 64 * c,
                          t.e * a.K + kb * BK);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (aborted) {
        set_error(a.err, kErrTimeout);
        *s_abort = 1;
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(full0 + 8 * s, (armed_par >> s) & 1, nullptr, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_f32acc_major(BM, a.bn, a.ab_f16 ? kFmtF16 : kFmtBF16, wgrad, true);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool aborted = false;
      for (int L = blockIdx.x; L < total && !aborted; L += gridDim.x) {
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
          const uint32_t a0 = smem_u32(ring + stage * STAGE_BYTES);
          const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = wgrad ? sdesc_mn128(a0 + kk * 2048, CHUNK) : sdesc_k128(a0 + kk * 32);
            tc_mma_f16kind(d_tmem, ad, sdesc_mn128(b0 + kk * 2048, CHUNK), idesc,
                           (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty0 + 8 * stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        tc_commit(tfull0 + 8 * acc);  // also with no k-block: the epilogue writes zeros
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (aborted) {
        set_error(a.err, kErrTimeout);
        *s_abort = 1;
        tc_commit(drain);
        mbar_wait(drain, 0, nullptr, kDrainLimitNs);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
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
        const int m = t.mt * BM + r;
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
        const int i = t.mt * BM + r;         // row within the expert's padded run
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
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
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
__device__ __forceinline__ float bwd_softplus(float z) {
  return fmaxf(z, 0.0f) + log1pf(__expf(-fabsf(z)));
}
__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + __expf(-z)); }

// Gate backward, one thread per token, over the E score columns of its row.
//   dgate [T, k]: gradient of L with respect to each chosen gate (from combine_bwd)
//   dimp [E] (or null): the Importance loss gradient, added to every chosen gate's
//   logits [T, E]: the clean logits x.W_g (+ bias); zlog [T, E]: x.W_noise (noisy)
//   dload [E] (or null): the Load loss gradient
// Writes dl [T, E] (gradient of the clean logits) and, for noisy gating, dz [T, E]
// (gradient of x.W_noise).  The gates of the forward pass are topk_gate (the chosen
// experts' Softmax(KeepTopK) values, or for the Switch gate the full-softmax values).
__global__ void __launch_bounds__(128)
    gate_bwd_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_gate,
                    const float* __restrict__ dgate, const float* __restrict__ dimp,
                    const float* __restrict__ logits, const float* __restrict__ zlog,
                    const float* __restrict__ noise, const float* __restrict__ dload,
                    float* __restrict__ dl, float* __restrict__ dz, int64_t T, int E, int k,
                    int noisy, int renorm) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  if (t >= T) return;
  const float* lrow = logits + t * E;
  float* dlr = dl + t * E;
  float* dzr = noisy ? dz + t * E : nullptr;
  for (int e = 0; e < E; ++e) dlr[e] = 0.0f;
  // chosen gates and their gradients
  float S = 0.0f;
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[t * k + j];
    const float dg = dgate[t * k + j] + (dimp ? dimp[e] : 0.0f);
    S += topk_gate[t * k + j] * dg;
  }
  const bool full = !noisy && !renorm;
  if (full) {
    // Switch gate: p = softmax over all logits; d score_e = p_e (dp_e - S), dp nonzero
    // only at the chosen experts
    float m = -INFINITY;
    for (int e = 0; e < E; ++e) m = fmaxf(m, lrow[e]);
    float z = 0.0f;
    for (int e = 0; e < E; ++e) z += expf(lrow[e] - m);
    for (int e = 0; e < E; ++e) dlr[e] = -(expf(lrow[e] - m) / z) * S;
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[t * k + j];
      const float dg = dgate[t * k + j] + (dimp ? dimp[e] : 0.0f);
      dlr[e] += topk_gate[t * k + j] * dg;
    }
  } else {
    // Softmax(KeepTopK): d score_i = G_i (dg_i - S) at the chosen experts
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[t * k + j];
      const float dg = dgate[t * k + j] + (dimp ? dimp[e] : 0.0f);
      dlr[e] = topk_gate[t * k + j] * (dg - S);
    }
  }
  if (!noisy) return;
  // noisy gating: the scores are H = l + n * Softplus(z); dlr holds dH so far
  const float* zrow = zlog + t * E;
  const float* nrow = noise + t * E;
  if (dload != nullptr) {
    // kth_excluding(H, k, i) is the (k+1)-th largest H when H_i is among the k largest
    // (H_i >= the k-th largest value), else the k-th largest, ranked by (-H, index):
    // one pass keeps the k+1 largest (k <= 8) in ascending expert order, so an equal
    // later value never displaces an earlier one
    float tv[9];
    int ti[9];
    for (int j = 0; j <= k; ++j) {
      tv[j] = -INFINITY;
      ti[j] = 0;
    }
    for (int e = 0; e < E; ++e) {
      float cv = lrow[e] + nrow[e] * bwd_softplus(zrow[e]);
      int ci = e;
      for (int j = 0; j <= k; ++j) {
        if (cv > tv[j]) {
          const float sv = tv[j];
          const int si = ti[j];
          tv[j] = cv;
          ti[j] = ci;
          cv = sv;
          ci = si;
        }
      }
    }
    const float hk = tv[k - 1], hk1 = tv[k];
    const int pk = ti[k - 1], pk1 = ti[k];
    // P(x, e) = Phi(zeta), zeta = (l_e - kth_excluding) / Softplus(z_e): its gradient goes
    // to l_e, to Softplus(z_e), and to H at the entry kth_excluding picked; the dH part
    // is gathered first, since any entry may receive it
    for (int e = 0; e < E; ++e) {
      const float sp = bwd_softplus(zrow[e]);
      const float He = lrow[e] + nrow[e] * sp;
      const bool top = He >= hk;
      const float zeta = (lrow[e] - (top ? hk1 : hk)) / sp;
      const float g = dload[e] * 0.3989422804014327f * expf(-0.5f * zeta * zeta);
      dlr[top ? pk1 : pk] += -g / sp;   // dH at the picked entry
      dzr[e] = -g * zeta / sp;          // d Softplus(z_e), times sigmoid(z_e) below
    }
    for (int e = 0; e < E; ++e) {
      const float sp = bwd_softplus(zrow[e]);
      const float He = lrow[e] + nrow[e] * sp;
      const bool top = He >= hk;
      const float zeta = (lrow[e] - (top ? hk1 : hk)) / sp;
      const float g = dload[e] * 0.3989422804014327f * expf(-0.5f * zeta * zeta);
      const float dH = dlr[e];
      dzr[e] = (dH * nrow[e] + dzr[e]) * sigmoidf_(zrow[e]);
      dlr[e] = dH + g / sp;
    }
  } else {
    for (int e = 0; e < E; ++e) dzr[e] = dlr[e] * nrow[e] * sigmoidf_(zrow[e]);
  }
}

// ---------------------------------------------------- strided SIMT products (router)
//
// C(m, n) (+)= sum_k A(m, k) B(n, k) with arbitrary element strides, fp32 accumulation;
// A and B bf16 or fp32.  blockIdx.z splits the contraction into `splits` runs whose
// partial results go to C + z * M * N (contiguous [M, N]) when splits > 1, to be summed
// in order by sum_partials_kernel.
namespace sr {
constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256;
}

template <typename TA, typename TB>
__device__ __forceinline__ float ldf(const TA* p, int64_t i);
template <>
__device__ __forceinline__ float ldf<float, float>(const float* p, int64_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16, __nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

template <typename TA, typename TB>
__global__ void __launch_bounds__(sr::THREADS)
    sgemm_strided_kernel(const TA* __restrict__ A, int64_t sam, int64_t sak, const TB* __restrict__ B,
                         int64_t sbn, int64_t sbk, float* __restrict__ C, int64_t scm, int64_t scn,
                         int M, int N, int64_t K, int64_t kchunk, int accumulate) {
  __shared__ float As[sr::BK][sr::BM + 4];
  __shared__ float Bs[sr::BK][sr::BN + 4];
  const int tid = threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  const int m0 = blockIdx.x * sr::BM, n0 = blockIdx.y * sr::BN;
  const int64_t k_lo = blockIdx.z * kchunk;
  const int64_t k_hi = min(K, k_lo + kchunk);
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (int64_t k0 = k_lo; k0 < k_hi; k0 += sr::BK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * sr::THREADS;
      const int r = idx & 63, kk = idx >> 6;   // 64 rows x 16 k
      const int64_t kc = k0 + kk;
      As[kk][r] = (m0 + r < M && kc < k_hi) ? ldf<TA, TA>(A, (m0 + r) * sam + kc * sak) : 0.0f;
      Bs[kk][r] = (n0 + r < N && kc < k_hi) ? ldf<TB, TB>(B, (n0 + r) * sbn + kc * sbk) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < sr::BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const bool partial = gridDim.z > 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      if (partial) {
        C[(static_cast<int64_t>(blockIdx.z) * M + m) * N + n] = acc[i][j];
      } else {
        float* c = C + m * scm + n * scn;
        *c = accumulate ? *c + acc[i][j] : acc[i][j];
      }
    }
  }
}

// out(m, n) (+)= sum_z part[z][m][n], z in order.
__global__ void sum_partials_kernel(const float* __restrict__ part, int splits, int M, int N,
                                    float* __restrict__ C, int64_t scm, int64_t scn, int accumulate) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  if (i >= static_cast<int64_t>(M) * N) return;
  float s = 0.0f;
  for (int z = 0; z < splits; ++z) s += part[static_cast<int64_t>(z) * M * N + i];
  const int64_t m = i / N, n = i - m * N;
  float* c = C + m * scm + n * scn;
  *c = accumulate ? *c + s : s;
}

// Column sums of a row-major [T, E] fp32 matrix in token order: out[e] = sum_t v[t, e].
__global__ void colsum_kernel(const float* __restrict__ v, int64_t T, int E, float* __restrict__ out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  if (e >= E) return;
  float s = 0.0f;
  for (int64_t t = 0; t < T; ++t) s += v[t * E + e];
  out[e] = s;
}

// Adds a per-column bias to a row-major [T, E] matrix.
__global__ void add_bias_kernel(float* __restrict__ v, int64_t T, int E, const float* __restrict__ b) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  if (i < T * E) v[i] += b[i % E];
}

// ------------------------------------------------------------------ host side

namespace {

template <typename TA, typename TB>
cudaError_t sgemm_strided(const TA* A, int64_t sam, int64_t sak, const TB* B, int64_t sbn, int64_t sbk,
                          float* C, int64_t scm, int64_t scn, int M, int N, int64_t K, int accumulate,
                          float* part, int64_t part_cap, const LaunchCtx& c) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const int gm = (M + sr::BM - 1) / sr::BM, gn = (N + sr::BN - 1) / sr::BN;
  // split the contraction when the output has few tiles, so that the grid fills the GPU
  int splits = 1;
  while (static_cast<int64_t>(gm) * gn * splits < 2 * c.num_sms && K / (splits * 2) >= 256 &&
         static_cast<int64_t>(splits * 2) * M * N <= part_cap)
    splits *= 2;
  int64_t kchunk = (K + splits - 1) / splits;
  kchunk = (kchunk + sr::BK - 1) / sr::BK * sr::BK;
  cudaError_t e = launch_kernel(sgemm_strided_kernel<TA, TB>, dim3(gm, gn, splits), dim3(sr::THREADS), 0,
                                c, A, sam, sak, B, sbn, sbk, splits > 1 ? part : C, scm, scn, M, N, K,
                                kchunk, accumulate);
  if (e != cudaSuccess || splits == 1) return e;
  const int64_t n = static_cast<int64_t>(M) * N;
  return launch_kernel(sum_partials_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0,
                       c, static_cast<const float*>(part), splits, M, N, C, scm, scn, accumulate);
}

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

cudaError_t launch_bwd_gemm(const bw::Args& a, const CUtensorMap& tmA, const CUtensorMap& tmB,
                            int64_t max_tiles, const LaunchCtx& c) {
  const int grid = static_cast<int>(max_tiles < c.num_sms ? max_tiles : c.num_sms);
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = ensure_smem_limit(bw::bwd_gemm_kernel, bw::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(bw::bwd_gemm_kernel, dim3(grid), dim3(bw::THREADS), bw::SMEM_BYTES, c, tmA,
                       tmB, a);
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
    e = launch_bwd_gemm(a, tA, tB, (prows / bw::BM + E) * static_cast<int64_t>(a.n_tiles), c);
    if (e != cudaSuccess) return e;
  }
  {  // dW2_e = d_o_e^T . h_e: M = d, N = f, contraction over the expert's rows
    bw::Args a = {};
    a.mode = bw::WGRAD; a.E = E; a.offsets = p.offsets; a.poff = p.poff;
    a.M = d; a.N = f; a.bn = pick_bn_bwd(f); a.n_tiles = f / a.bn; a.m_tiles = (d + bw::BM - 1) / bw::BM;
    a.rows_cap = n; a.out = p.dw2; a.ab_f16 = w2f16; a.err = c.err;
    CUtensorMap tA, tB;
    if (!tmap16(&tA, p.d_o, prows, d, 64, w2f16) || !tmap16(&tB, p.h, n, f, 64, w2f16))
      return cudaErrorInvalidValue;
    e = launch_bwd_gemm(a, tA, tB, static_cast<int64_t>(E) * a.m_tiles * a.n_tiles, c);
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
    e = launch_bwd_gemm(a, tA, tB, (prows / bw::BM + E) * static_cast<int64_t>(a.n_tiles), c);
    if (e != cudaSuccess) return e;
  }
  {  // dW1_e = du_e^T . x_perm_e: M = f, N = d
    bw::Args a = {};
    a.mode = bw::WGRAD; a.E = E; a.offsets = p.offsets; a.poff = p.poff;
    a.M = f; a.N = d; a.bn = pick_bn_bwd(d); a.n_tiles = d / a.bn; a.m_tiles = (f + bw::BM - 1) / bw::BM;
    a.rows_cap = n; a.out = p.dw1; a.ab_f16 = 0; a.err = c.err;
    CUtensorMap tA, tB;
    if (!tmap16(&tA, p.du, prows, f, 64, 0) || !tmap16(&tB, p.x_perm, n, d, 64, 0))
      return cudaErrorInvalidValue;
    e = launch_bwd_gemm(a, tA, tB, static_cast<int64_t>(E) * a.m_tiles * a.n_tiles, c);
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
  // ---- router: recompute the logits (and x.W_noise), gate backward, parameter grads
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* wg = static_cast<const __nv_bfloat16*>(p.w_gate);
  const __nv_bfloat16* wn = static_cast<const __nv_bfloat16*>(p.w_noise);
  e = sgemm_strided(x, d, 1, wg, d, 1, p.logits, E, 1, static_cast<int>(p.T), E, d, 0, p.part,
                    p.part_cap, c);
  if (e != cudaSuccess) return e;
  if (p.bias) {
    const int64_t m = p.T * E;
    e = launch_kernel(add_bias_kernel, dim3(static_cast<unsigned>((m + 255) / 256)), dim3(256), 0, c,
                      p.logits, p.T, E, p.bias);
    if (e != cudaSuccess) return e;
  }
  if (p.noisy) {
    e = sgemm_strided(x, d, 1, wn, d, 1, p.zlog, E, 1, static_cast<int>(p.T), E, d, 0, p.part,
                      p.part_cap, c);
    if (e != cudaSuccess) return e;
  }
  e = launch_kernel(gate_bwd_kernel, dim3(static_cast<unsigned>((p.T + 127) / 128)), dim3(128), 0, c,
                    p.topk_idx, p.topk_gate, static_cast<const float*>(p.dgate),
                    static_cast<const float*>(p.w_importance != 0.0f ? p.dimp : nullptr),
                    static_cast<const float*>(p.logits), static_cast<const float*>(p.zlog), p.noise,
                    static_cast<const float*>(p.w_load != 0.0f ? p.dload : nullptr), p.dl, p.dz, p.T,
                    E, p.k, p.noisy, p.renorm);
  if (e != cudaSuccess) return e;
  // dx += dl . W_g: A = dl [T, E], B(n, e) = W_g[e, n]
  e = sgemm_strided(static_cast<const float*>(p.dl), E, 1, wg, 1, d, p.dx, d, 1, static_cast<int>(p.T),
                    d, E, 1, p.part, p.part_cap, c);
  if (e != cudaSuccess) return e;
  // dW_g[e, :] = sum_t dl[t, e] x[t, :]
  e = sgemm_strided(static_cast<const float*>(p.dl), 1, E, x, 1, d, p.dw_gate, d, 1, E, d, p.T, 0,
                    p.part, p.part_cap, c);
  if (e != cudaSuccess) return e;
  if (p.dbias) {
    e = launch_kernel(colsum_kernel, dim3((E + 127) / 128), dim3(128), 0, c,
                      static_cast<const float*>(p.dl), p.T, E, p.dbias);
    if (e != cudaSuccess) return e;
  }
  if (p.noisy) {
    e = sgemm_strided(static_cast<const float*>(p.dz), E, 1, wn, 1, d, p.dx, d, 1, static_cast<int>(p.T),
                      d, E, 1, p.part, p.part_cap, c);
    if (e != cudaSuccess) return e;
    e = sgemm_strided(static_cast<const float*>(p.dz), 1, E, x, 1, d, p.dw_noise, d, 1, E, d, p.T, 0,
                      p.part, p.part_cap, c);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace moe
