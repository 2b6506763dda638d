// fp32 path of the per-expert FFN (and of the router product): a ragged grouped product
// on the FP32 pipes, out[r, n] = act(sum_k A[r, k] * B_g[n, k]) for the rows r of group
// g, where A row r is A[a_idx[r] / a_div] when a row index a_idx is given (the token rows
// gathered by the permutation's perm_src) and A[r] otherwise.  fp32 inputs with fp32
// accumulation meet the fp32 tolerance that TF32 tensor-core products would miss.  Small
// problems only: the bf16 path is the fast one.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace sg {
constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256;
constexpr int MAX_GROUPS = 1024;
}  // namespace sg

__global__ void __launch_bounds__(sg::THREADS)
    sgemm_grouped_kernel(const float* __restrict__ A, const float* __restrict__ B,
                         float* __restrict__ out, const int32_t* __restrict__ offsets,
                         int groups, int64_t rows_cap, int N, int K, int act,
                         const int32_t* __restrict__ a_idx, int a_div, int* err) {
  __shared__ float As[sg::BK][sg::BM + 4];
  __shared__ float Bs[sg::BK][sg::BN + 4];
  __shared__ int tp[sg::MAX_GROUPS + 1];
  __shared__ int scratch[40];
  const int tid = threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();

  int g = 0;
  int64_t row0, row_end;
  if (offsets == nullptr) {
    row0 = static_cast<int64_t>(blockIdx.x) * sg::BM;
    row_end = rows_cap;
    if (row0 >= row_end) return;
  } else {
    if (!block_tile_prefix(offsets, groups, rows_cap, sg::BM, tp, scratch)) {
      if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) set_error(err, kErrOffsets);
      return;
    }
    const int L = blockIdx.x;
    if (L >= tp[groups]) return;
    int lo = 0, hi = groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tp[mid] <= L) lo = mid; else hi = mid - 1;
    }
    g = lo;
    row0 = offsets[g] + static_cast<int64_t>(L - tp[g]) * sg::BM;
    row_end = offsets[g + 1];
  }
  const float* Bg = B + static_cast<int64_t>(g) * N * K;
  const int n0 = blockIdx.y * sg::BN;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  // source row in A of each of the tile's rows this thread loads (rows tid/16 + 16 i)
  int64_t src[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t ar = row0 + ((tid + i * sg::THREADS) >> 4);
    src[i] = ar;
    if (a_idx != nullptr && ar < row_end) src[i] = a_idx[ar] / a_div;
  }

  for (int k0 = 0; k0 < K; k0 += sg::BK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * sg::THREADS;
      const int r = idx >> 4, kk = idx & 15;
      const int64_t ar = row0 + r;
      const int kc = k0 + kk;
      As[kk][r] = (ar < row_end && kc < K) ? A[src[i] * K + kc] : 0.0f;
      const int bn = n0 + r;
      Bs[kk][r] = (bn < N && kc < K) ? Bg[static_cast<int64_t>(bn) * K + kc] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < sg::BK; ++kk) {
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
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = row0 + ty * 4 + i;
    if (r >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cidx = n0 + tx * 4 + j;
      if (cidx < N) out[r * N + cidx] = apply_act(acc[i][j], act);
    }
  }
}

cudaError_t launch_sgemm_grouped(const float* A, const float* B, float* out,
                                 const int32_t* offsets, int groups, int64_t rows_cap, int N,
                                 int K, int act, const LaunchCtx& c, const int32_t* a_idx,
                                 int a_div) {
  if (groups > sg::MAX_GROUPS) return cudaErrorInvalidValue;
  const int64_t mt = offsets ? rows_cap / sg::BM + groups : (rows_cap + sg::BM - 1) / sg::BM;
  if (mt <= 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(mt), static_cast<unsigned>((N + sg::BN - 1) / sg::BN));
  return launch_kernel(sgemm_grouped_kernel, grid, dim3(sg::THREADS), 0, c, A, B, out, offsets,
                       groups, rows_cap, N, K, act, a_idx, a_div, c.err);
}

cudaError_t launch_ffn_f32(const FfnProblem& p, const LaunchCtx& c) {
  const bool gather = p.gather_src != nullptr;
  cudaError_t e = launch_sgemm_grouped(static_cast<const float*>(gather ? p.x : p.x_perm),
                                       static_cast<const float*>(p.w1), static_cast<float*>(p.h),
                                       p.offsets, p.E, p.rows_cap, p.f, p.d, p.act, c,
                                       p.gather_src, p.k);
  if (e != cudaSuccess) return e;
  return launch_sgemm_grouped(static_cast<const float*>(p.h), static_cast<const float*>(p.w2),
                              static_cast<float*>(p.y_perm), p.offsets, p.E, p.rows_cap, p.d, p.f, 0, c);
}

}  // namespace moe
