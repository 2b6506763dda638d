// Capacity truncation and stable permutation of the token->expert assignments.
//
// Dispatch gathers each expert's tokens (Switch Transformer, switch_routing: the expert
// loop "needs a gather").  Assignment a = t*k + j goes to expert e = topk_idx[a].  Rows
// are ordered by expert, and within an expert by ascending a (a stable counting sort);
// only the first C assignments of an expert are kept (capacity factor, "moe paper models"
// Table 2), the rest are dropped (slot_pos = -1).
//
// Four kernels, no atomics on global memory and no cross-block waits:
//   count    block b counts its chunk of 2048 assignments per expert (shared-memory
//            histogram) -> blk[b][e]
//   scan     one block: per expert an exclusive scan over the chunks (blk[b][e] becomes
//            the number of earlier assignments of e), counts[e], kept[e] = min(count, C),
//            and offsets = exclusive scan of kept
//   scatter  block b ranks its chunk stably (warp match + per-warp prefix) and writes
//            slot_pos / perm_src
//   gather   x_perm[s] = x[perm_src[s] / k] for every kept row s < offsets[E]: one warp
//            per row, 16-byte vectors, a grid of several blocks per SM so that enough
//            loads are in flight to stream at HBM rate
#include <mutex>

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

__global__ void __launch_bounds__(pm::THREADS)
    perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t n, int k, int E, int64_t C,
                        const int32_t* __restrict__ blk, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ perm_src, int32_t* __restrict__ slot_pos) {
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
    __syncwarp();
  }
}

constexpr int kGatherWarps = 8;

__global__ void __launch_bounds__(kGatherWarps * 32)
    perm_gather_kernel(const int32_t* __restrict__ perm_src, const int32_t* __restrict__ offsets,
                       int E, int k, const uint8_t* __restrict__ x, uint8_t* __restrict__ x_perm,
                       int row_bytes) {
  const int lane = threadIdx.x & 31;
  const int n_kept = __ldg(offsets + E);
  const int nv = row_bytes >> 4;
  const int warps = gridDim.x * kGatherWarps;
  for (int s = blockIdx.x * kGatherWarps + (threadIdx.x >> 5); s < n_kept; s += warps) {
    const int64_t t = __ldg(perm_src + s) / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + t * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(s) * row_bytes);
    int v = lane;
    for (; v + 96 < nv; v += 128) {
      const uint4 a0 = __ldg(src + v), a1 = __ldg(src + v + 32), a2 = __ldg(src + v + 64),
                  a3 = __ldg(src + v + 96);
      dst[v] = a0;
      dst[v + 32] = a1;
      dst[v + 64] = a2;
      dst[v + 96] = a3;
    }
    for (; v < nv; v += 32) dst[v] = __ldg(src + v);
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
      p.topk_idx, p.n, p.k, p.E, p.C, p.blk, p.offsets, p.perm_src, p.slot_pos);
  ++*c.launches;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // enough warps for every row when the grid allows, capped at 16 blocks per SM
  int64_t gblocks = (p.n + kGatherWarps - 1) / kGatherWarps;
  const int64_t cap = static_cast<int64_t>(c.num_sms) * 16;
  if (gblocks > cap) gblocks = cap;
  perm_gather_kernel<<<static_cast<unsigned>(gblocks), kGatherWarps * 32, 0, c.stream>>>(
      p.perm_src, p.offsets, p.E, p.k, static_cast<const uint8_t*>(p.x),
      static_cast<uint8_t*>(p.x_perm), p.d * p.esize);
  ++*c.launches;
  return cudaGetLastError();
}

}  // namespace moe

// ------------------------------------------------------------------------------------
// moe_permute without a caller-provided workspace, for callers that cannot allocate
// device memory.  Its per-chunk, per-expert counts live in a fixed array in the
// library's own device memory instead of in `ws`.

namespace moe {

// Every device that loads libmoe holds this array until the process exits.
static __device__ __align__(256) int32_t g_permute_scratch[MOE_NOALLOC_SCRATCH_BYTES / 4];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_permute_scratch on the current device.  In host code the name
// g_permute_scratch is only a host-side stand-in, so the address is looked up once per
// device, with that device current, and cached.
cudaError_t scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}
}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                          const void* x, int32_t* counts, int32_t* offsets,
                                          int32_t* perm_src, int32_t* slot_pos, void* x_perm,
                                          moe_stream_t stream) {
  using namespace moe;
  moe_status st = check_config_host(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->T == 0) {
    const size_t E = static_cast<size_t>(cfg->E);
    if (cudaMemsetAsync(counts, 0, E * 4, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, (E + 1) * 4, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    set_last_launch_count(0);
    return MOE_OK;
  }
  if (!topk_idx || !x || !perm_src || !slot_pos || !x_perm) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u))
    return MOE_ERR_INVALID_ARG;
  const int64_t n = cfg->T * cfg->k;
  // the scratch holds one int32 per (2048-assignment chunk, expert)
  if (permute_blocks(n) * cfg->E * 4 > static_cast<int64_t>(MOE_NOALLOC_SCRATCH_BYTES))
    return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  LaunchCtx c;
  int launches = 0;
  void* scratch = nullptr;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      scratch_address(dev, &scratch) != cudaSuccess)
    return MOE_ERR_CUDA;
  c.stream = s;
  c.err = nullptr;  // no error word: out-of-range expert indices are dropped unreported
  c.launches = &launches;
  PermuteProblem p;
  p.n = n;
  p.k = cfg->k;
  p.E = cfg->E;
  p.d = cfg->d_model;
  p.esize = cfg->dtype == MOE_BF16 ? 2 : 4;
  p.C = capacity_host(cfg);
  p.topk_idx = topk_idx;
  p.x = x;
  p.counts = counts;
  p.offsets = offsets;
  p.perm_src = perm_src;
  p.slot_pos = slot_pos;
  p.x_perm = x_perm;
  p.blk = static_cast<int32_t*>(scratch);  // fully rewritten by the count kernel each call
  if (launch_permute(p, c) != cudaSuccess) return MOE_ERR_CUDA;
  set_last_launch_count(launches);
  return MOE_OK;
}
