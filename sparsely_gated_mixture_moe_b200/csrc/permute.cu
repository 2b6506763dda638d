// Capacity truncation and stable permutation of the token->expert assignments.
//
// Dispatch gathers each expert's tokens (Switch Transformer, switch_routing: the expert
// loop "needs a gather").  Assignment a = t*k + j goes to expert e = topk_idx[a].  Rows
// are ordered by expert, and within an expert by ascending a (a stable counting sort);
// only the first C assignments of an expert are kept (capacity factor, "moe paper models"
// Table 2), the rest are dropped (slot_pos = -1).
//
// Three kernels, no atomics on global memory and no cross-block waits:
//   count    block b counts its chunk of 2048 assignments per expert (shared-memory
//            histogram) -> blk[b][e]
//   scan     one block: per expert an exclusive scan over the chunks (blk[b][e] becomes
//            the number of earlier assignments of e), counts[e], kept[e] = min(count, C),
//            and offsets = exclusive scan of kept
//   scatter  block b ranks its chunk stably (warp match + per-warp prefix), writes
//            slot_pos / perm_src and copies the kept token rows into x_perm with 16-byte
//            vector loads and stores
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace pm {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int PER_WARP = kPermChunk / WARPS;  // 256 assignments per warp, 8 rounds of 32
constexpr int SCAN_THREADS = 1024;
}  // namespace pm

int64_t permute_blocks(int64_t n) { return (n + kPermChunk - 1) / kPermChunk; }

__global__ void __launch_bounds__(pm::THREADS)
    perm_count_kernel(const int32_t* __restrict__ idx, int64_t n, int E, int32_t* __restrict__ blk,
                      int* err) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermChunk;
  for (int i = threadIdx.x; i < kPermChunk; i += blockDim.x) {
    const int64_t a = base + i;
    if (a >= n) break;
    const int e = idx[a];
    if (e < 0 || e >= E) {
      set_error(err, kErrExpertIndex);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    blk[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

__global__ void __launch_bounds__(pm::SCAN_THREADS)
    perm_scan_kernel(int32_t* __restrict__ blk, int nblk, int E, int64_t C,
                     int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  extern __shared__ int kept[];  // [E]
  __shared__ int scratch[40];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      const int64_t i = static_cast<int64_t>(b) * E + e;
      const int cnt = blk[i];
      blk[i] = run;
      run += cnt;
    }
    counts[e] = run;
    kept[e] = (C >= 0 && run > C) ? static_cast<int>(C) : run;
  }
  __syncthreads();
  int carry = 0;
  for (int base = 0; base < E; base += blockDim.x) {
    const int e = base + threadIdx.x;
    const int v = e < E ? kept[e] : 0;
    int tot;
    const int incl = block_incl_scan(v, scratch, &tot);
    if (e < E) offsets[e] = carry + incl - v;
    carry += tot;
  }
  if (threadIdx.x == 0) offsets[E] = carry;
}

template <int VEC_BYTES>
__device__ __forceinline__ void copy_row(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                         int row_bytes, int lane) {
  const int nv = row_bytes / 16;
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  int v = lane;
  for (; v + 96 < nv; v += 128) {
    const uint4 a0 = __ldg(s + v), a1 = __ldg(s + v + 32), a2 = __ldg(s + v + 64),
                a3 = __ldg(s + v + 96);
    d[v] = a0;
    d[v + 32] = a1;
    d[v + 64] = a2;
    d[v + 96] = a3;
  }
  for (; v < nv; v += 32) d[v] = __ldg(s + v);
}

__global__ void __launch_bounds__(pm::THREADS)
    perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t n, int k, int E, int64_t C,
                        const int32_t* __restrict__ blk, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ perm_src, int32_t* __restrict__ slot_pos,
                        const uint8_t* __restrict__ x, uint8_t* __restrict__ x_perm,
                        int row_bytes) {
  extern __shared__ int wbase[];  // [WARPS][E]: running rank base of each warp per expert
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermChunk + warp * pm::PER_WARP;

  for (int i = threadIdx.x; i < pm::WARPS * E; i += blockDim.x) wbase[i] = 0;
  __syncthreads();
  // per-warp histogram of this warp's 256 assignments
  for (int r = 0; r < pm::PER_WARP / 32; ++r) {
    const int64_t a = base + r * 32 + lane;
    int e = (a < n) ? idx[a] : -1;
    if (e < 0 || e >= E) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt_mask) == 0) wbase[warp * E + e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan over the warps, offset by the chunk's rank base from the scan kernel
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = blk[static_cast<int64_t>(blockIdx.x) * E + e];
    for (int w = 0; w < pm::WARPS; ++w) {
      const int c = wbase[w * E + e];
      wbase[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // ranks in assignment order: warp-major, then round, then lane
  for (int r = 0; r < pm::PER_WARP / 32; ++r) {
    const int64_t a = base + r * 32 + lane;
    int e = (a < n) ? idx[a] : -1;
    if (e < 0 || e >= E) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    int slot = -1;
    if (e >= 0) {
      const int rank = wbase[warp * E + e] + __popc(peers & lt_mask);
      if (C < 0 || rank < C) slot = offsets[e] + rank;
    }
    __syncwarp();
    if (e >= 0 && (peers & lt_mask) == 0) wbase[warp * E + e] += __popc(peers);
    if (a < n) {
      slot_pos[a] = slot;
      if (slot >= 0) perm_src[slot] = static_cast<int32_t>(a);
    }
    // copy the kept rows of this round, one row per warp step
    uint32_t kept = __ballot_sync(0xffffffffu, slot >= 0);
    while (kept) {
      const int src_lane = __ffs(kept) - 1;
      kept &= kept - 1;
      const int s = __shfl_sync(0xffffffffu, slot, src_lane);
      const int64_t t = (base + r * 32 + src_lane) / k;
      copy_row<16>(x + t * row_bytes, x_perm + static_cast<int64_t>(s) * row_bytes, row_bytes, lane);
    }
    __syncwarp();
  }
}

cudaError_t launch_permute(const PermuteProblem& p, const LaunchCtx& c) {
  const int64_t nblk = permute_blocks(p.n);
  if (nblk == 0) return cudaSuccess;
  const size_t hist_smem = static_cast<size_t>(p.E) * 4;
  perm_count_kernel<<<static_cast<unsigned>(nblk), pm::THREADS, hist_smem, c.stream>>>(
      p.topk_idx, p.n, p.E, p.blk, c.err);
  ++*c.launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  perm_scan_kernel<<<1, pm::SCAN_THREADS, hist_smem, c.stream>>>(p.blk, static_cast<int>(nblk), p.E,
                                                                 p.C, p.counts, p.offsets);
  ++*c.launches;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t wsmem = static_cast<size_t>(pm::WARPS) * p.E * 4;
  if (wsmem > 48 * 1024) {
    e = cudaFuncSetAttribute(perm_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(wsmem));
    if (e != cudaSuccess) return e;
  }
  perm_scatter_kernel<<<static_cast<unsigned>(nblk), pm::THREADS, wsmem, c.stream>>>(
      p.topk_idx, p.n, p.k, p.E, p.C, p.blk, p.offsets, p.perm_src, p.slot_pos,
      static_cast<const uint8_t*>(p.x), static_cast<uint8_t*>(p.x_perm), p.d * p.esize);
  ++*c.launches;
  return cudaGetLastError();
}

}  // namespace moe
