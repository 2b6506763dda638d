// Gate-weighted combine (un-permute): y[t] = sum_j G_{t,j} * y_perm[slot_pos[t*k + j]].
//
// The layer output of Shazeer et al. ("Methode"): y = sum_i G(x)_i E_i(x), with only the
// k chosen experts contributing and a dropped assignment (slot_pos = -1) adding nothing.
// y_perm is fp32 for both layer dtypes (the expert outputs leave the tensor cores as fp32
// accumulators); y is fp32, or bf16 when asked for (each fp32 sum rounded once).  One
// warp per token; each lane handles 4-value vectors of the row, gathers the k expert rows
// and accumulates in fp32 in the order j = 0 .. k-1.
#include "common.cuh"
#include "internal.h"

namespace moe {

// Four consecutive values of a row: loads from fp32, stores to fp32 (16 bytes) or bf16
// (8 bytes, round to nearest even).
template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float (&v)[4]) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  __device__ static void store(void* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <>
struct Vec<__nv_bfloat16> {
  __device__ static void store(void* p, const float (&v)[4]) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
  }
};
constexpr int kCombineWarps = 8;

template <typename OUT>
__global__ void __launch_bounds__(kCombineWarps * 32)
    combine_kernel(const float* __restrict__ y_perm, const int32_t* __restrict__ slot_pos,
                   const float* __restrict__ gate, OUT* __restrict__ y, int64_t T_, int k, int d,
                   int* err) {
  using T = float;
  constexpr int V = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kCombineWarps + warp;
  grid_dep_wait();
  grid_dep_launch();
  if (t >= T_) return;
  const int64_t nrows = T_ * k;
  int slot[8];
  float g[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    slot[j] = -1;
    g[j] = 0.0f;
    if (j < k) {
      const int s = slot_pos[t * k + j];
      if (s >= 0 && s < nrows) {
        slot[j] = s;
        g[j] = gate[t * k + j];
      } else if (s != -1 && lane == 0) {
        set_error(err, kErrSlot);
      }
    }
  }
  const int nv = d / V;
  // four vectors per lane per step so that several loads per slot are in flight
  int v = lane;
  for (; v + 96 < nv; v += 128) {
    float acc[4][V];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int i = 0; i < V; ++i) acc[u][i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (slot[j] >= 0) {
        const T* src = y_perm + static_cast<int64_t>(slot[j]) * d + v * V;
        float r[4][V];
#pragma unroll
        for (int u = 0; u < 4; ++u) Vec<T>::load(src + u * 32 * V, r[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int i = 0; i < V; ++i) acc[u][i] = fmaf(g[j], r[u][i], acc[u][i]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) Vec<OUT>::store(y + t * d + (v + u * 32) * V, acc[u]);
  }
  for (; v < nv; v += 32) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (slot[j] >= 0) {
        float r[V];
        Vec<T>::load(y_perm + static_cast<int64_t>(slot[j]) * d + v * V, r);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(g[j], r[i], acc[i]);
      }
    }
    Vec<OUT>::store(y + t * d + v * V, acc);
  }
}

cudaError_t launch_combine(const CombineProblem& p, const LaunchCtx& c) {
  const int64_t blocks = (p.T + kCombineWarps - 1) / kCombineWarps;
  if (blocks == 0) return cudaSuccess;
  if (p.y_bf16)
    return launch_kernel(combine_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(blocks)),
                         dim3(kCombineWarps * 32), 0, c, static_cast<const float*>(p.y_perm),
                         p.slot_pos, p.gate, static_cast<__nv_bfloat16*>(p.y), p.T, p.k, p.d,
                         c.err);
  return launch_kernel(combine_kernel<float>, dim3(static_cast<unsigned>(blocks)),
                       dim3(kCombineWarps * 32), 0, c, static_cast<const float*>(p.y_perm),
                       p.slot_pos, p.gate, static_cast<float*>(p.y), p.T, p.k, p.d, c.err);
}

}  // namespace moe
