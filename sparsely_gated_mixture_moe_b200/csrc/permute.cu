// Capacity truncation and stable permutation of the token->expert assignments.
//
// Dispatch gathers each expert's tokens (Switch Transformer, switch_routing: the expert
// loop "needs a gather").  Assignment a = t*k + j goes to expert e = topk_idx[a].  Rows
// are ordered by expert, and within an expert by ascending a (a stable counting sort);
// only the first C assignments of an expert are kept (capacity factor, "moe paper models"
// Table 2), the rest are dropped (slot_pos = -1).
//
// One launch when every block of its grid can be resident at once (perm_fused_kernel,
// below), else three kernels with no cross-block waits:
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
// With x_perm null only the index arrays are written (no row copy): the expert FFN then
// gathers the token rows itself (moe_expert_ffn_gather).
#include <map>
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
// Ints of the per-chunk count array the workspace must hold: the three-kernel path uses
// ceil(n / 256) chunks of 256 assignments by E experts, the one-launch path at most
// ceil(n / 128) chunks by E rounded up to a multiple of 4.
int64_t permute_count_ints(int64_t n, int E) {
  const int64_t three = permute_blocks(n) * E;
  const int64_t fused = (n + 127) / 128 * ((E + 3) & ~3);
  return three > fused ? three : fused;
}

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
  grid_dep_wait();
  grid_dep_launch();
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
  grid_dep_wait();
  grid_dep_launch();
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
  grid_dep_wait();
  grid_dep_launch();
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

// ------------------------------------------------------------------ one-launch path
//
// The same counting sort in one launch with one grid barrier.  The n assignments are
// split into nchunks chunks of `chunk` (<= 1024, a multiple of 32) consecutive
// assignments, one per block of 1024 threads; all blocks are resident at once (the grid
// never exceeds what the occupancy query says fits).
//   phase 1  the block ranks its chunk stably (warp match + per-warp prefix, kept in
//            registers and shared memory) and writes its per-expert counts to row c of
//            blk [nchunks][Ep] (Ep = E rounded up to a multiple of 4, the padding zeroed,
//            so that phase 2 reads the rows as 16-byte vectors)
//   barrier
//   phase 2  the block sums column e of blk over the rows below its chunk (its rank base)
//            and over all rows (the expert's count), reading whole rows (a warp reads
//            512 contiguous bytes), scans min(count, C) into offsets (block 0
//            writes counts and offsets), writes slot_pos and perm_src for its chunk, and
//            copies its kept rows x[a / k] -> x_perm[slot] (16-byte vectors, two rows
//            per warp in flight).  Every block redoes the small column sums itself, so
//            no second scan pass or flag is needed.
// The barrier is an arrival counter in the workspace with a bounded wait (1 s, then the
// timeout bit and an early exit); the last block to leave resets it and the exit counter.
namespace pf {
constexpr int THREADS = 1024;
constexpr int WARPS = THREADS / 32;
}  // namespace pf

static size_t fused_smem(int E) {
  return (8 * pf::THREADS + static_cast<size_t>(pf::WARPS) * E + 3 * static_cast<size_t>(E) +
          pf::THREADS + 64) * 4;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier over all blocks of the grid (all resident).  Arrivals accumulate in *ctr over
// the launch; the barrier is complete once *ctr reaches `target`.  Gives up after the
// wait limit: sets the timeout bit and *s_abort.  Every thread must call it.
__device__ bool grid_barrier(int* ctr, int target, int* err, volatile int* s_abort) {
  __syncthreads();
  if (threadIdx.x == 0 && *s_abort == 0) {
    __threadfence();
    atomicAdd(ctr, 1);
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_gpu(ctr) < target) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        set_error(err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
  return *s_abort == 0;
}

__global__ void __launch_bounds__(pf::THREADS, 1)
    perm_fused_kernel(const int32_t* __restrict__ idx, int64_t n, int E, int64_t C, int k,
                      int chunk, int nchunks, int32_t* blk, int32_t* __restrict__ counts,
                      int32_t* __restrict__ offsets, int32_t* __restrict__ perm_src,
                      int32_t* __restrict__ slot_pos, const uint8_t* __restrict__ x,
                      uint8_t* __restrict__ x_perm, int row_bytes, int32_t* sync, int* err) {
  extern __shared__ __align__(16) int fsm[];
  int4* red = reinterpret_cast<int4*>(fsm);  // [2][THREADS]: column-sum partials
  int* wbase = fsm + 8 * pf::THREADS;   // [WARPS][E]: per-warp rank bases
  int* s_pre = wbase + pf::WARPS * E;   // [E]: rank base of this chunk
  int* s_tot = s_pre + E;               // [E]: assignments per expert
  int* s_off = s_tot + E;               // [E]: offsets
  int* s_slot = s_off + E;              // [THREADS]: slot of each assignment of the chunk
  int* scratch = s_slot + pf::THREADS;  // [64]
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int c = blockIdx.x;
  const int64_t a0 = static_cast<int64_t>(c) * chunk;
  const int cn = static_cast<int>(min(static_cast<int64_t>(chunk), n - a0));  // > 0
  const int nw = (chunk + 31) >> 5;  // warps holding assignments
  if (tid == 0) s_abort = 0;
  for (int i = tid; i < nw * E; i += pf::THREADS) wbase[i] = 0;
  grid_dep_wait();
  grid_dep_launch();
  __syncthreads();

  // ---- phase 1: stable ranks within the chunk, chunk counts to blk[e][c]
  const int64_t a = a0 + tid;
  int e = -1;
  uint32_t peers = 0;
  if (warp < nw) {  // uniform across the warp
    if (tid < cn) {
      e = idx[a];
      if (e < 0 || e >= E) {
        set_error(err, kErrExpertIndex);
        e = -1;
      }
    }
    peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt_mask) == 0) wbase[warp * E + e] = __popc(peers);
  }
  __syncthreads();
  const int Ep = (E + 3) & ~3;  // row length of blk
  for (int xe = tid; xe < Ep; xe += pf::THREADS) {
    int run = 0;
    if (xe < E)
      for (int w = 0; w < nw; ++w) {
        const int v = wbase[w * E + xe];
        wbase[w * E + xe] = run;
        run += v;
      }
    blk[static_cast<int64_t>(c) * Ep + xe] = run;
  }
  const bool ok = grid_barrier(sync, nchunks, err, &s_abort);

  // ---- phase 2: rank bases, counts, offsets; slot_pos, perm_src and rows of this chunk
  if (ok) {
    // thread (row group rg, column quad q) sums rows rg, rg + RG, ... of its four columns;
    // then the first row group adds up the RG partials (integer sums: any order is exact)
    const int NQ = Ep >> 2;
    const int4* rows = reinterpret_cast<const int4*>(blk);
    for (int qb = 0; qb < NQ; qb += pf::THREADS) {
      const int nqb = min(NQ - qb, pf::THREADS);
      const int RG = pf::THREADS / nqb;
      const int q = qb + tid % nqb, rg = tid / nqb;
      int4 pre = make_int4(0, 0, 0, 0), tot = make_int4(0, 0, 0, 0);
      if (rg < RG) {
#pragma unroll 4
        for (int r = rg; r < nchunks; r += RG) {
          const int4 v = __ldcg(rows + static_cast<int64_t>(r) * NQ + q);
          tot.x += v.x;
          tot.y += v.y;
          tot.z += v.z;
          tot.w += v.w;
          if (r < c) {
            pre.x += v.x;
            pre.y += v.y;
            pre.z += v.z;
            pre.w += v.w;
          }
        }
      }
      red[tid] = pre;
      red[pf::THREADS + tid] = tot;
      __syncthreads();
      if (tid < nqb) {
        int4 P = make_int4(0, 0, 0, 0), S = make_int4(0, 0, 0, 0);
        for (int g = 0; g < RG; ++g) {
          const int4 a = red[g * nqb + tid], b = red[pf::THREADS + g * nqb + tid];
          P.x += a.x;
          P.y += a.y;
          P.z += a.z;
          P.w += a.w;
          S.x += b.x;
          S.y += b.y;
          S.z += b.z;
          S.w += b.w;
        }
        const int e4 = 4 * (qb + tid);
        if (e4 < E) {
          s_pre[e4] = P.x;
          s_tot[e4] = S.x;
        }
        if (e4 + 1 < E) {
          s_pre[e4 + 1] = P.y;
          s_tot[e4 + 1] = S.y;
        }
        if (e4 + 2 < E) {
          s_pre[e4 + 2] = P.z;
          s_tot[e4 + 2] = S.z;
        }
        if (e4 + 3 < E) {
          s_pre[e4 + 3] = P.w;
          s_tot[e4 + 3] = S.w;
        }
      }
      __syncthreads();
    }
    int carry = 0;
    for (int base = 0; base < E; base += pf::THREADS) {
      const int xe = base + tid;
      const int tot = xe < E ? s_tot[xe] : 0;
      const int kv = (C >= 0 && tot > C) ? static_cast<int>(C) : tot;
      int sum;
      const int incl = block_incl_scan(kv, scratch, &sum);
      if (xe < E) {
        s_off[xe] = carry + incl - kv;
        if (c == 0) {
          counts[xe] = tot;
          offsets[xe] = carry + incl - kv;
        }
      }
      carry += sum;
    }
    if (c == 0 && tid == 0) offsets[E] = carry;
    __syncthreads();
    if (tid < cn) {
      int slot = -1;
      if (e >= 0) {
        const int rank = s_pre[e] + wbase[warp * E + e] + __popc(peers & lt_mask);
        if (C < 0 || rank < C) slot = s_off[e] + rank;
      }
      slot_pos[a] = slot;
      if (slot >= 0) perm_src[slot] = static_cast<int32_t>(a);
      s_slot[tid] = slot;
    }
    __syncthreads();
    // the chunk's kept rows, in assignment order; warp w takes assignments w, w + 32, ...
    // (nothing to copy when only the index arrays are asked for)
    const int nv = row_bytes >> 4;
    for (int i = warp; x_perm != nullptr && i < cn; i += 2 * pf::WARPS) {
      const int i2 = i + pf::WARPS;
      const int sl1 = s_slot[i];
      const int sl2 = i2 < cn ? s_slot[i2] : -1;
      if (sl1 < 0 && sl2 < 0) continue;
      const int64_t t1 = (a0 + i) / k, t2 = (a0 + i2) / k;
      const uint4* src1 = reinterpret_cast<const uint4*>(x + t1 * row_bytes);
      const uint4* src2 = reinterpret_cast<const uint4*>(x + (sl2 >= 0 ? t2 : t1) * row_bytes);
      uint4* dst1 = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(sl1 >= 0 ? sl1 : 0) * row_bytes);
      uint4* dst2 = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(sl2 >= 0 ? sl2 : 0) * row_bytes);
      int v = lane;
      for (; v + 32 < nv; v += 64) {
        const uint4 p0 = __ldg(src1 + v), p1 = __ldg(src1 + v + 32);
        const uint4 q0 = __ldg(src2 + v), q1 = __ldg(src2 + v + 32);
        if (sl1 >= 0) {
          dst1[v] = p0;
          dst1[v + 32] = p1;
        }
        if (sl2 >= 0) {
          dst2[v] = q0;
          dst2[v + 32] = q1;
        }
      }
      for (; v < nv; v += 32) {
        const uint4 p0 = __ldg(src1 + v), q0 = __ldg(src2 + v);
        if (sl1 >= 0) dst1[v] = p0;
        if (sl2 >= 0) dst2[v] = q0;
      }
    }
  }

  // ---- the last block to leave resets both counters for the next call
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(sync + 1, 1) == nchunks - 1) {
      atomicExch(sync, 0);
      atomicExch(sync + 1, 0);
    }
  }
}

// The grid barrier with a target no block reaches (one more arrival than blocks): every
// block's wait expires, sets the timeout bit and returns; the last block out resets the
// counters.  Used by moe_wait_timeout_check.
__global__ void barrier_timeout_check_kernel(int32_t* sync, int* err) {
  __shared__ int s_abort;
  grid_dep_wait();
  grid_dep_launch();
  if (threadIdx.x == 0) s_abort = 0;
  __syncthreads();
  grid_barrier(sync, static_cast<int>(gridDim.x) + 1, err, &s_abort);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(sync + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(sync, 0);
      atomicExch(sync + 1, 0);
    }
  }
}

cudaError_t launch_wait_timeout_check(int32_t* sync, int* err, const LaunchCtx& c) {
  return launch_kernel(barrier_timeout_check_kernel, dim3(2), dim3(32), 0, c, sync, err);
}

// Chunking for the one-launch path: returns the number of chunks (= blocks) and sets
// *chunk, or returns 0 when the chunks would exceed 1024 assignments or the blocks would
// not all fit on the GPU at once.
static int fused_chunks(const PermuteProblem& p, const LaunchCtx& c, size_t smem, int* chunk) {
  if (p.sync == nullptr) return 0;
  if (smem > 48 * 1024 &&
      ensure_smem_limit(perm_fused_kernel, static_cast<int>(smem)) != cudaSuccess)
    return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, perm_fused_kernel, pf::THREADS,
                                                    smem) != cudaSuccess)
    return 0;
  const int64_t cap = static_cast<int64_t>(per_sm) * c.num_sms;
  // at least 128 assignments per chunk, at most one chunk per resident block
  int64_t g = (p.n + 127) / 128;
  if (g > cap) g = cap;
  if (g < 1) return 0;
  int64_t ch = (p.n + g - 1) / g;
  ch = (ch + 31) / 32 * 32;
  if (ch > pf::THREADS) return 0;
  *chunk = static_cast<int>(ch);
  return static_cast<int>((p.n + ch - 1) / ch);
}

cudaError_t launch_permute(const PermuteProblem& p, const LaunchCtx& c) {
  const int64_t nblk = permute_blocks(p.n);
  if (nblk == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  const size_t f_smem = fused_smem(p.E);
  int chunk = 0;
  const int nchunks = fused_chunks(p, c, f_smem, &chunk);
  if (nchunks > 0) {
    return launch_kernel(perm_fused_kernel, dim3(nchunks), dim3(pf::THREADS), f_smem, c,
                         p.topk_idx, p.n, p.E, p.C, p.k, chunk, nchunks, p.blk, p.counts,
                         p.offsets, p.perm_src, p.slot_pos, static_cast<const uint8_t*>(p.x),
                         static_cast<uint8_t*>(p.x_perm), p.d * p.esize, p.sync, c.err);
  }
  const size_t cs_smem = count_scan_smem(p.E);
  if (cs_smem > 48 * 1024) {
    e = ensure_smem_limit(perm_count_scan_kernel, static_cast<int>(cs_smem));
    if (e != cudaSuccess) return e;
  }
  e = launch_kernel(perm_count_scan_kernel, dim3(static_cast<unsigned>(nblk)), dim3(pm::THREADS),
                    cs_smem, c, p.topk_idx, p.n, p.E, p.C, p.blk, p.counts, p.offsets, p.ticket,
                    c.err);
  if (e != cudaSuccess) return e;
  const size_t wsmem = static_cast<size_t>(pm::WARPS) * p.E * 4;
  if (wsmem > 48 * 1024) {
    e = ensure_smem_limit(perm_scatter_kernel, static_cast<int>(wsmem));
    if (e != cudaSuccess) return e;
  }
  e = launch_kernel(perm_scatter_kernel, dim3(static_cast<unsigned>(nblk)), dim3(pm::THREADS),
                    wsmem, c, p.topk_idx, p.n, p.E, p.C, static_cast<const int32_t*>(p.blk),
                    static_cast<const int32_t*>(p.offsets), p.perm_src, p.slot_pos);
  if (e != cudaSuccess || p.x_perm == nullptr) return e;
  // enough warps for every row when the grid allows, capped at 16 blocks per SM
  int64_t gblocks = (p.n + kGatherWarps - 1) / kGatherWarps;
  const int64_t cap = static_cast<int64_t>(c.num_sms) * 16;
  if (gblocks > cap) gblocks = cap;
  return launch_kernel(perm_gather_kernel, dim3(static_cast<unsigned>(gblocks)),
                       dim3(kGatherWarps * 32), 0, c, static_cast<const int32_t*>(p.perm_src),
                       static_cast<const int32_t*>(p.offsets), p.E, p.k,
                       static_cast<const uint8_t*>(p.x), static_cast<uint8_t*>(p.x_perm),
                       p.d * p.esize);
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
std::mutex g_scratch_mu;
std::map<unsigned long long, void*> g_scratch_addr;  // context id -> device address

// Device address of g_permute_scratch in the current context.  In host code the name
// g_permute_scratch is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per context (the context current on this thread, i.e. the
// current device's), and cached under the context's unique id: a context that replaces
// an earlier one (after cudaDeviceReset, say) gets its own lookup.
cudaError_t scratch_address(void** out) {
  unsigned long long ctx = 0;
  cudaError_t e = current_context_id(&ctx);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  auto it = g_scratch_addr.find(ctx);
  if (it == g_scratch_addr.end()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    it = g_scratch_addr.emplace(ctx, p).first;
  }
  *out = it->second;
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
  if (!topk_idx || !perm_src || !slot_pos || (x_perm && !x)) return MOE_ERR_INVALID_ARG;
  if (x_perm && ((reinterpret_cast<uintptr_t>(x) & 15u) ||
                 (reinterpret_cast<uintptr_t>(x_perm) & 15u)))
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
      scratch_address(&scratch) != cudaSuccess)
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
  p.sync = nullptr;  // always the three-kernel path here
  if (cudaMemsetAsync(p.ticket, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_permute(p, c) != cudaSuccess) return MOE_ERR_CUDA;
  set_last_launch_count(launches);
  return MOE_OK;
}
