// Capacity truncation and stable permutation of the token->expert assignments.
//
// Dispatch gathers each expert's tokens (Switch Transformer, switch_routing: the expert
// loop "needs a gather").  Assignment a = t*k + j goes to expert e = topk_idx[a].  Rows
// are ordered by expert, and within an expert by ascending a (a stable counting sort);
// only the first C assignments of an expert are kept (capacity factor, "moe paper models"
// Table 2), the rest are dropped (slot_pos = -1).
//
// Three kernels, no cross-block waits:
//   count+scan  block b counts its chunk of 256 assignments per expert (shared-memory
//               histogram) into blk[b][e]; the last block to finish (a ticket counter)
//               turns blk into per-chunk rank bases with a segmented scan over the chunks,
//               writes counts[e], kept[e] = min(count, C) and offsets (exclusive scan of
//               kept), and resets the ticket
//   scatter     block b ranks its chunk stably (warp match + per-warp prefix) and writes
//               slot_pos / perm_src
//   gather      x_perm[s] = x[perm_src[s] / k] for every kept row s < offsets[E]: one warp
//               per row, 16-byte vectors, a grid of several blocks per SM so that enough
//               loads are in flight to stream at HBM rate
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace pm {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
static_assert(kPermChunk == THREADS, "one assignment per thread per chunk");
}  // namespace pm

int64_t permute_blocks(int64_t n) { return (n + kPermChunk - 1) / kPermChunk; }

// Shared memory of perm_count_scan_kernel: hist[E] and, for the scan, seg[2][256] and
// kept[E] ints.
static size_t count_scan_smem(int E) { return (static_cast<size_t>(E) * 2 + 512 + 64) * 4; }

__global__ void __launch_bounds__(pm::THREADS)
    perm_count_scan_kernel(const int32_t* __restrict__ idx, int64_t n, int E, int64_t C,
                           int32_t* __restrict__ blk, int32_t* __restrict__ counts,
                           int32_t* __restrict__ offsets, int32_t* ticket, int* err) {
  extern __shared__ int sm[];
  int* hist = sm;                 // [E]
  int* seg = hist + E;            // [256] segment sums, then segment bases
  int* kept = seg + 512;          // [E]
  int* scratch = kept + E;        // [40]
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int nblk = gridDim.x;
  for (int e = tid; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t a = static_cast<int64_t>(blockIdx.x) * kPermChunk + tid;
  if (a < n) {
    const int e = idx[a];
    if (e < 0 || e >= E) set_error(err, kErrExpertIndex);
    else atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) blk[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(ticket, 1) == nblk - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last block: per expert, exclusive scan of blk[.][e] over the chunks.  With
  // E < 256 several threads share an expert, each owning a contiguous run of chunks.
  int tpe = 1;
  while (tpe * 2 * E <= pm::THREADS) tpe *= 2;
  const int len = (nblk + tpe - 1) / tpe;
  for (int e0 = 0; e0 < E; e0 += pm::THREADS / tpe) {
    const int e = e0 + tid % (pm::THREADS / tpe);
    const int part = tid / (pm::THREADS / tpe);
    const bool act = (tid % (pm::THREADS / tpe)) < (pm::THREADS / tpe) && e < E && part < tpe;
    const int b0 = part * len, b1 = min(nblk, b0 + len);
    int sum = 0;
    if (act)
      for (int b = b0; b < b1; ++b) sum += __ldcg(blk + static_cast<int64_t>(b) * E + e);
    if (act) seg[part * (pm::THREADS / tpe) + (e - e0)] = sum;
    __syncthreads();
    if (act && part == 0) {
      int run = 0;
      for (int q = 0; q < tpe; ++q) {
        const int v = seg[q * (pm::THREADS / tpe) + (e - e0)];
        seg[256 + q * (pm::THREADS / tpe) + (e - e0)] = run;
        run += v;
      }
      counts[e] = run;
      kept[e] = (C >= 0 && run > C) ? static_cast<int>(C) : run;
    }
    __syncthreads();
    if (act) {
      int run = seg[256 + part * (pm::THREADS / tpe) + (e - e0)];
      for (int b = b0; b < b1; ++b) {
        const int64_t i = static_cast<int64_t>(b) * E + e;
        const int c = __ldcg(blk + i);
        blk[i] = run;
        run += c;
      }
    }
    __syncthreads();
  }
  int carry = 0;
  for (int base = 0; base < E; base += blockDim.x) {
    const int e = base + tid;
    const int v = e < E ? kept[e] : 0;
    int tot;
    const int incl = block_incl_scan(v, scratch, &tot);
    if (e < E) offsets[e] = carry + incl - v;
    carry += tot;
  }
  if (tid == 0) {
    offsets[E] = carry;
    *ticket = 0;  // ready for the next call
  }
}

__global__ void __launch_bounds__(pm::THREADS)
    perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t n, int E, int64_t C,
                        const int32_t* __restrict__ blk, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ perm_src, int32_t* __restrict__ slot_pos) {
  extern __shared__ int wbase[];  // [WARPS][E]: rank base of each warp per expert
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int64_t a = static_cast<int64_t>(blockIdx.x) * kPermChunk + threadIdx.x;

  for (int i = threadIdx.x; i < pm::WARPS * E; i += blockDim.x) wbase[i] = 0;
  __syncthreads();
  int e = (a < n) ? idx[a] : -1;
  if (e < 0 || e >= E) e = -1;
  const uint32_t peers = __match_any_sync(0xffffffffu, e);
  if (e >= 0 && (peers & lt_mask) == 0) wbase[warp * E + e] = __popc(peers);
  __syncthreads();
  // exclusive scan over the warps, offset by the chunk's rank base from the scan
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = blk[static_cast<int64_t>(blockIdx.x) * E + x];
    for (int w = 0; w < pm::WARPS; ++w) {
      const int c = wbase[w * E + x];
      wbase[w * E + x] = run;
      run += c;
    }
  }
  __syncthreads();
  // ranks in assignment order: warp, then lane
  int slot = -1;
  if (e >= 0) {
    const int rank = wbase[warp * E + e] + __popc(peers & lt_mask);
    if (C < 0 || rank < C) slot = offsets[e] + rank;
  }
  if (a < n) {
    slot_pos[a] = slot;
    if (slot >= 0) perm_src[slot] = static_cast<int32_t>(a);
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
  cudaError_t e = cudaSuccess;
  const size_t cs_smem = count_scan_smem(p.E);
  if (cs_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(perm_count_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(cs_smem));
    if (e != cudaSuccess) return e;
  }
  perm_count_scan_kernel<<<static_cast<unsigned>(nblk), pm::THREADS, cs_smem, c.stream>>>(
      p.topk_idx, p.n, p.E, p.C, p.blk, p.counts, p.offsets, p.ticket, c.err);
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
      p.topk_idx, p.n, p.E, p.C, p.blk, p.offsets, p.perm_src, p.slot_pos);
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
  // the scratch holds a 256-byte counter block, then one int32 per (chunk, expert)
  if (256 + permute_blocks(n) * cfg->E * 4 > static_cast<int64_t>(MOE_NOALLOC_SCRATCH_BYTES))
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
  // the ticket must start at zero: clear it (a call cut short could have left it set);
  // the per-chunk counts are fully rewritten by the count kernel each call
  p.ticket = static_cast<int32_t*>(scratch);
  p.blk = static_cast<int32_t*>(scratch) + 64;
  if (cudaMemsetAsync(p.ticket, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_permute(p, c) != cudaSuccess) return MOE_ERR_CUDA;
  set_last_launch_count(launches);
  return MOE_OK;
}
