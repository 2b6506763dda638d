// Device helpers shared by the kernels of libmoe: error bits, bounded mbarrier waits,
// TMA loads, tcgen05 (5th-generation tensor core) MMA / TMEM wrappers, shared-memory
// matrix descriptors and a block-wide scan.  sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device error word bits (mirror MOE_DEVERR_* in include/moe.h).
constexpr int kErrExpertIndex = 1;
constexpr int kErrOffsets = 2;
constexpr int kErrSlot = 4;
constexpr int kErrTimeout = 8;

// A wait on an mbarrier gives up after this long; normal waits last microseconds.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s
constexpr unsigned long long kDrainLimitNs = 100000000ull;  // 0.1 s for teardown drains

// Programmatic dependent launch.  grid_dep_wait: block until the kernel that precedes this
// one on the stream has completed and its memory operations are visible (returns at once
// when the launch did not allow an early start).  grid_dep_launch: let the next kernel on
// the stream be scheduled now; it still waits in its own grid_dep_wait.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void set_error(int* err, int bits) {
  if (err != nullptr) atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (TMA / tensor core) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with parity `parity` of `bar` has completed.  Returns false
// (without having seen the phase) once `limit_ns` has passed or, when `abort_flag` is
// given, once another thread of the CTA has raised it.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          const volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// --------------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load global -> this CTA's shared memory, completion signalled
// as transaction bytes on `bar`.  x is the innermost (contiguous) coordinate in
// elements; callers keep x * element size a multiple of 16 bytes.  No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Four rows of a 2-D tensor, each one box of [1 row x box-width columns] at column x,
// gathered into consecutive rows of this CTA's shared memory (TMA tile::gather4); rows
// r0..r3 may be any rows of the tensor, in any order.  The tensor map's box is one row
// high.  With 128-byte swizzling the rows land where a tiled load of rows (dst / 128)
// mod 8 ... of a 1024-byte-aligned tile would put them, so a 4-row group at a 512-byte
// offset of such a tile fits the tile's layout.  No multicast.
__device__ __forceinline__ void tma_gather4_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                               int x, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

// ----------------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   holder_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit inputs (both bf16 or both fp16, as the
// instruction descriptor says), fp32 accumulation, one CTA.
__device__ __forceinline__ void tc_mma_f16kind(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f16 with A and B of one 16-bit type (both K-major)
// and fp32 D.  bits 4-5 D format (1 = f32), 7-9 A format and 10-12 B format (0 = fp16,
// 1 = bf16; always equal here), 15/16 A/B major (0 = K-major), 17-22 N >> 3, 24-28 M >> 4.
constexpr uint32_t kFmtF16 = 0;
constexpr uint32_t kFmtBF16 = 1;
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, uint32_t ab_fmt) {
  return (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor of a K-major operand tile written by TMA with
// 128-byte swizzling: rows of 64 bf16 (128 B), 8-row groups 1024 B apart, tile base
// 1024-byte aligned.  Advancing K by 16 elements inside the 128-byte row adds 32 bytes
// to the start address.
//   bits 0-13 start >> 4, 16-29 leading offset >> 4 (unused here), 32-45 stride offset
//   >> 4 (1024 B), 46-47 version (1), 61-63 layout (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc_k128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Shared-memory matrix descriptor of an MN-major operand tile written by TMA with 128-byte
// swizzling (the operand's M or N index is the contiguous one, as for a row-major [K, N]
// weight read as B = W^T): the tile is a run of chunks of 64 MN-elements, each chunk
// [K rows x 128 B] from one TMA box, K rows 128 B apart, 8-row groups 1024 B apart
// (stride offset), chunks `chunk_bytes` apart (leading offset).  Advancing K by 16 rows
// adds 2048 bytes to the start address.
__device__ __forceinline__ uint64_t sdesc_mn128(uint32_t saddr, uint32_t chunk_bytes) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((chunk_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// idesc_f32acc with the major order of each operand: bit 15 set when A is M-major, bit 16
// when B is N-major.
__host__ __device__ constexpr uint32_t idesc_f32acc_major(int M, int N, uint32_t ab_fmt, bool a_mn,
                                                          bool b_mn) {
  return idesc_f32acc(M, N, ab_fmt) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u);
}

// Each thread of the warp reads 32 consecutive fp32 columns of its own TMEM lane
// (the warp's lane quarter is fixed by its warp index modulo 4).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// As tmem_ld32, 8 consecutive columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
// As tmem_ld32, 16 consecutive columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------- CTA pairs (clusters of two CTAs)
//
// The two CTAs of a cluster share one tensor-core product of M = 256 rows
// (tcgen05 cta_group::2): each holds half of A (its 128 rows) and half of B in its own
// shared memory and gets its 128 rows of D in its own TMEM.  Every tcgen05 instruction of
// a kernel that does this uses cta_group::2.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address in the shared::cluster window of the object at shared::cta address `addr` in the
// cluster's CTA of rank `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Barrier over all threads of both CTAs of the cluster (release / acquire).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (possibly the peer CTA's).
// Arrivals that order nothing before them (relaxed), for a barrier whose waiter needs only
// the arrival: an accumulator handed back to the MMA thread after tcgen05.wait::ld (the
// TMEM reads have completed; nothing the waiter does reads the epilogue's global
// stores).  A release arrival would hold the warp until its earlier global stores are
// performed.
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

// As tma_load_2d, into this CTA's shared memory, with completion signalled on `bar`, a
// shared::cluster address that may be the peer CTA's mbarrier.  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// As tma_gather4_2d, with completion signalled on a shared::cluster mbarrier address that
// may be the peer CTA's.  No multicast.
__device__ __forceinline__ void tma_gather4_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                    uint32_t bar, int x, int r0, int r1, int r2,
                                                    int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::"
      "complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

// TMEM allocation shared by the pair: a warp of the same index in each CTA runs it.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive once on the mbarrier at shared::cluster address `bar` (this CTA's or the peer's)
// when every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// D[tmem] (+)= A * B^T over the pair: M = 256 (128 rows of A and D in each CTA), B split
// by N between the CTAs; the descriptors name the same shared-memory offsets in both.
__device__ __forceinline__ void tc_mma_pair_f16kind(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// --------------------------------------------------------------------- utilities

// One 32-byte store of 8 words (the address 32-byte aligned): a whole L2 sector per
// thread, where two 16-byte stores would each write half of one.
__device__ __forceinline__ void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t a4, uint32_t a5, uint32_t a6,
                                             uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0),
               "r"(a1), "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Sum of one value per thread over a block of NT threads (a multiple of 32) in a fixed
// order: a butterfly within each warp, then the warps' sums in warp order by thread 0.
// The result is returned to thread 0 only.  Every thread of the block must call it.
template <int NT>
__device__ __forceinline__ float block_sum_fixed(float v) {
  __shared__ float warp_sums[NT / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.0f;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) s += warp_sums[w];
  }
  return s;
}

// erf by Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
// erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2), t = 1 / (1 + p x),
// x >= 0, |error| <= 1.5e-7 (odd extension for x < 0).  About a third of the
// instructions of a full-accuracy erf.  Used for the GELU epilogue (its results are
// rounded to 16 bits) and for the normal CDF of the Load estimate (summed in fp32).
// The reciprocal and 2^x are the approximate PTX instructions with subnormals flushed:
// t lies in (0, 1] and exp(-x^2) only underflows where the product no longer changes
// the result, and the flushed forms skip the range fix-ups (measured 2.4% faster on
// the GELU up-projection).
__device__ __forceinline__ float erf_as7126(float x) {
  const float ax = fabsf(x);
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, ax, 1.0f)));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  float e;  // exp(-x^2) = 2^(-x^2 log2(e))
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(ax * (-1.4426950408889634f * ax)));
  const float y = 1.0f - poly * e;
  return copysignf(y, x);
}

// Pairs of fp32 values in one 64-bit register for the packed f32x2 arithmetic of
// sm_100 (fma/mul .rn.f32x2: two IEEE fp32 operations, each rounded as the scalar one,
// per instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_splat(float c) { return f2_pack(c, c); }
__device__ __forceinline__ float rcp_ftz(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_ftz(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU of two values, z Phi(z) = (z/2) (1 + erf(z / sqrt 2)), with erf by Abramowitz &
// Stegun 7.1.26 exactly as erf_as7126 evaluates it, every multiply-add done on both
// values by one f32x2 instruction.  The polynomial is carried negated (its coefficients'
// signs flipped, an exact operation), so 1 - poly exp(-x^2) is one fused multiply-add;
// the last step is (z/2) + (z/2) erf, one rounding instead of two.
__device__ __forceinline__ void gelu2_as7126(float z0, float z1, float& g0, float& g1) {
  const uint64_t z = f2_pack(z0, z1);
  float x0, x1;
  f2_unpack(f2_mul(z, f2_splat(0.70710678118654752f)), x0, x1);
  const uint64_t ax = f2_pack(fabsf(x0), fabsf(x1));
  float d0, d1;
  f2_unpack(f2_fma(f2_splat(0.3275911f), ax, f2_splat(1.0f)), d0, d1);
  const uint64_t t = f2_pack(rcp_ftz(d0), rcp_ftz(d1));
  uint64_t np = f2_fma(f2_splat(-1.061405429f), t, f2_splat(1.453152027f));
  np = f2_fma(np, t, f2_splat(-1.421413741f));
  np = f2_fma(np, t, f2_splat(0.284496736f));
  np = f2_fma(np, t, f2_splat(-0.254829592f));
  np = f2_mul(np, t);
  float q0, q1;  // -x^2 log2(e)
  f2_unpack(f2_mul(ax, f2_mul(ax, f2_splat(-1.4426950408889634f))), q0, q1);
  float y0, y1;  // 1 - poly exp(-x^2), in [0, 1]
  f2_unpack(f2_fma(np, f2_pack(ex2_ftz(q0), ex2_ftz(q1)), f2_splat(1.0f)), y0, y1);
  const uint64_t hz = f2_mul(z, f2_splat(0.5f));
  f2_unpack(f2_fma(hz, f2_pack(copysignf(y0, x0), copysignf(y1, x1)), hz), g0, g1);
}

// GELU'(u) = Phi(u) + u phi(u) for two values, on f32x2 pairs like gelu2_as7126: with
// x = u / sqrt 2, erf(x) = 1 - poly(t) exp(-x^2) (A&S 7.1.26) and phi(u) =
// exp(-u^2 / 2) / sqrt(2 pi) take the same exponential, computed once.
__device__ __forceinline__ void gelu_grad2_as7126(float u0, float u1, float& g0, float& g1) {
  const uint64_t u = f2_pack(u0, u1);
  float x0, x1;
  f2_unpack(f2_mul(u, f2_splat(0.70710678118654752f)), x0, x1);
  const uint64_t ax = f2_pack(fabsf(x0), fabsf(x1));
  float d0, d1;
  f2_unpack(f2_fma(f2_splat(0.3275911f), ax, f2_splat(1.0f)), d0, d1);
  const uint64_t t = f2_pack(rcp_ftz(d0), rcp_ftz(d1));
  uint64_t np = f2_fma(f2_splat(-1.061405429f), t, f2_splat(1.453152027f));
  np = f2_fma(np, t, f2_splat(-1.421413741f));
  np = f2_fma(np, t, f2_splat(0.284496736f));
  np = f2_fma(np, t, f2_splat(-0.254829592f));
  np = f2_mul(np, t);
  float q0, q1;  // -x^2 log2(e) = -(u^2 / 2) log2(e)
  f2_unpack(f2_mul(ax, f2_mul(ax, f2_splat(-1.4426950408889634f))), q0, q1);
  const uint64_t e = f2_pack(ex2_ftz(q0), ex2_ftz(q1));
  float y0, y1;
  f2_unpack(f2_fma(np, e, f2_splat(1.0f)), y0, y1);
  const uint64_t Phi = f2_fma(f2_pack(copysignf(y0, x0), copysignf(y1, x1)), f2_splat(0.5f),
                              f2_splat(0.5f));
  f2_unpack(f2_fma(f2_mul(u, f2_splat(0.3989422804014327f)), e, Phi), g0, g1);
}

__device__ __forceinline__ float gelu_exact(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}

__device__ __forceinline__ float apply_act(float z, int act) {
  // act: 0 none, 1 ReLU, 2 GELU (exact erf form)
  if (act == 1) return fmaxf(z, 0.0f);
  if (act == 2) return gelu_exact(z);
  return z;
}

// Inclusive scan of one int per thread across the block; every thread must call it.
// `scratch` holds at least 33 ints.  Returns the inclusive prefix; *total gets the sum.
__device__ __forceinline__ int block_incl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    scratch[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int before = warp > 0 ? scratch[warp - 1] : 0;
  const int tot = scratch[nwarps - 1];
  __syncthreads();
  *total = tot;
  return v + before;
}

// Per-group tile prefix for a ragged grouped product: tp[g] = sum over groups g' < g of
// ceil((offsets[g'+1] - offsets[g']) / bm), tp[G] = total.  Also checks the offsets
// are non-decreasing within [0, rows_cap]; returns false (on every thread) otherwise.
// Every thread must call it.  tp holds G+1 ints, scratch 34 ints.
__device__ __forceinline__ bool block_tile_prefix(const int* __restrict__ offsets, int G,
                                                  int64_t rows_cap, int bm, int* tp,
                                                  int* scratch) {
  if (threadIdx.x == 0) {
    tp[0] = 0;
    scratch[33] = 0;
  }
  __syncthreads();
  int carry = 0;
  for (int base = 0; base < G; base += blockDim.x) {
    const int g = base + threadIdx.x;
    int v = 0;
    if (g < G) {
      const int a = offsets[g], b = offsets[g + 1];
      if (a < 0 || b < a || static_cast<int64_t>(b) > rows_cap) {
        scratch[33] = 1;
      } else {
        v = (b - a + bm - 1) / bm;
      }
    }
    int tot;
    const int incl = block_incl_scan(v, scratch, &tot);
    if (g < G) tp[g + 1] = carry + incl;
    carry += tot;
  }
  __syncthreads();
  return scratch[33] == 0;
}

}  // namespace moe
