// Host-side launchers shared by the translation units of libmoe.  Each launcher queues
// its kernels on `stream`, adds the number of launches to *launches and returns the
// CUDA error of the last launch (cudaSuccess on success).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#include "moe.h"

namespace moe {

struct LaunchCtx {
  cudaStream_t stream;
  int num_sms;
  int* err;       // device error word
  int* launches;  // host counter
};

// Unique id of the CUDA context current on this thread (cuCtxGetId), initialising the
// device's primary context first if need be.  Ids are never reused within a process, so
// state cached per context (a looked-up symbol address, a raised kernel attribute) is
// never taken for a context that replaced it, e.g. after cudaDeviceReset.
cudaError_t current_context_id(unsigned long long* id);

// Raises a kernel's dynamic shared-memory limit to at least `bytes` in the current
// context, calling cudaFuncSetAttribute only the first time a larger limit is needed
// there (the attribute outlives the call; repeating it on every launch only costs host
// time).
template <typename... KArgs>
cudaError_t ensure_smem_limit(void (*kernel)(KArgs...), int bytes) {
  static std::mutex mu;
  static std::map<std::pair<unsigned long long, const void*>, int> limit;
  unsigned long long ctx = 0;
  cudaError_t e = current_context_id(&ctx);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(ctx, reinterpret_cast<const void*>(kernel));
  const auto it = limit.find(key);
  if (it != limit.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) limit[key] = bytes;
  return e;
}

// Every kernel of the library is launched with programmatic stream serialisation: the
// launch may start while the previous kernel on the stream is still running, and the
// kernel's grid_dep_wait() (at its top, before any global-memory access) blocks until
// that kernel has completed and its writes are visible.  Only the prologue (barrier
// init, TMEM allocation, descriptor prefetch) overlaps the previous kernel's tail.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          const LaunchCtx& c, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  ++*c.launches;
  return e;
}

// As launch_kernel, for a kernel whose CTAs run in clusters of two (grid.x even): the two
// CTAs of a cluster are co-scheduled on a pair of SMs and share a tensor-core product.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_pairs(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                const LaunchCtx& c, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  ++*c.launches;
  return e;
}

// ---- route -----------------------------------------------------------------------
struct RouteProblem {
  int64_t T;
  int d, E, k;
  int noisy, renorm;
  int hier = 0, groups = 0, k_primary = 0;  // hierarchical gating: w_gate has groups + E rows
  const void* x;
  const void* w_gate;
  const void* w_noise;
  const float* noise;
  const float* bias;
  int32_t* topk_idx;
  float* topk_gate;
  uint8_t* near_tie;
  float* importance;  // may be null
  float* load;        // may be null
  float* partials;    // workspace: [route_blocks][2][E]
  float* logits_ws;   // fp32 path only: [T][E] ([T][groups + E] for hierarchical gating)
  float* nz_ws;       // fp32 path only: [T][E]
  float* lw = nullptr;  // bf16 path: clean logits (+ bias), and for noisy gating Softplus
  float* sw = nullptr;  // (x.W_noise) and noisy scores H, each [E][T], and the k-th /
  float* hw = nullptr;  // (k+1)-th noisy scores [2][T] of each token; written for noisy
  float* kw = nullptr;  // gating with Importance/Load, or always with store_scores
  bool store_scores = false;  // the training forward keeps them for the backward
};
int route_blocks(int64_t T);
cudaError_t launch_route_bf16(const RouteProblem& p, const LaunchCtx& c);
cudaError_t launch_route_f32(const RouteProblem& p, const LaunchCtx& c);

// ---- permute ---------------------------------------------------------------------
constexpr int kPermChunk = 256;  // assignments per permute block (one per thread)
struct PermuteProblem {
  int64_t n;  // T*k assignments
  int k, E, d, esize;
  int64_t C;  // capacity, < 0: none
  const int32_t* topk_idx;
  const void* x;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm_src;
  int32_t* slot_pos;
  void* x_perm;
  int32_t* blk;     // workspace [nblk][E]
  int32_t* ticket;  // workspace counter, zero between calls
  int32_t* sync;    // two workspace counters, zero between calls, for the one-launch
                    // path (null: always use the three-kernel path)
};
int64_t permute_blocks(int64_t n);
int64_t permute_count_ints(int64_t n, int E);
cudaError_t launch_permute(const PermuteProblem& p, const LaunchCtx& c);
cudaError_t launch_wait_timeout_check(int32_t* sync, int* err, const LaunchCtx& c);

// ---- expert FFN ------------------------------------------------------------------
struct FfnProblem {
  int64_t rows_cap;  // T*k
  int d, f, E, act;  // act: 1 ReLU, 2 GELU
  int hidden_f16;    // bf16 path: h stored in fp16 and w2 given in fp16
  const void* x_perm;  // permuted rows, or null when gather_src is given
  const void* x = nullptr;              // token rows [x_rows, d] (gather mode)
  const int32_t* gather_src = nullptr;  // permuted row s reads x[gather_src[s] / k]
  int64_t x_rows = 0;
  int k = 1;
  void* u = nullptr;                    // bf16 path: also store the pre-activations [rows, f]
  const int32_t* offsets;
  const void* w1;
  const void* w2;
  void* h;
  void* y_perm;
  int y_bf16 = 0;  // fused combine (k = 1): y in bf16
  int w_count = 0;  // > 0: E row groups over w_count weight blocks, group g using g % w_count
};
cudaError_t launch_ffn_bf16(const FfnProblem& p, const LaunchCtx& c);
cudaError_t launch_ffn_f32(const FfnProblem& p, const LaunchCtx& c);
// bf16 expert FFN whose down-projection forms y itself instead of y_perm.  k = 1: it
// writes y[t] = gate[t] * row (its epilogue also zeroes the rows of dropped tokens); y in
// fp32, or bf16 with p.y_bf16.  k = 2 (fp32 y): the up-projection's epilogue threads zero
// y and the down-projection adds gate * row into its token's row in memory.
cudaError_t launch_ffn_combine_bf16(const FfnProblem& p, const int32_t* perm_src,
                                    const int32_t* slot_pos, const float* gate, void* y,
                                    const LaunchCtx& c);

// fp32 SIMT grouped product out[r, n] = act(sum_k A'[r, k] B_g[n, k]) for the rows r of
// each group g (offsets, or a single group of `rows` rows when offsets is null), where
// A'[r] = A[a_idx[r] / a_div] when a_idx is given, else A[r].
cudaError_t launch_sgemm_grouped(const float* A, const float* B, float* out,
                                 const int32_t* offsets, int groups, int64_t rows_cap, int N,
                                 int K, int act, const LaunchCtx& c,
                                 const int32_t* a_idx = nullptr, int a_div = 1);

// ---- combine ---------------------------------------------------------------------
struct CombineProblem {
  int64_t T;
  int k, d;
  const void* y_perm;
  const int32_t* slot_pos;
  const float* gate;
  void* y;
  int y_bf16 = 0;  // y in bf16 (each fp32 sum rounded once), else fp32
};
cudaError_t launch_combine(const CombineProblem& p, const LaunchCtx& c);

// ---- backward --------------------------------------------------------------------
// Everything moe_backward launches; the buffers come from the training state and the
// backward workspace (see moe_api.cu for their layout).
struct BackwardProblem {
  int64_t T;
  int d, f, E, k, act;  // act: 1 ReLU, 2 GELU
  int noisy, renorm, hidden_f16;
  float w_importance, w_load;
  // forward inputs and saved forward state
  const void* x;
  const void* w_gate;
  const void* w_noise;
  const float* noise;
  const float* bias;
  const void* w1;
  const void* w2;
  const int32_t* topk_idx;
  const float* topk_gate;
  const float* importance;
  const float* load;
  const int32_t* offsets;
  const int32_t* slot_pos;
  const void* x_perm;
  const void* u;
  const void* h;
  const float* y_perm;
  const float* dy;
  // outputs
  float* dx;
  float* dw_gate;
  float* dw_noise;
  float* dbias;
  float* dw1;
  float* dw2;
  float* dgate;
  float* losses;  // [2] or null: w_importance CV^2 and w_load CV^2
  // workspace
  int32_t* poff;
  void* d_o;      // [T*k + 64 E, d] 16-bit
  void* du;       // [T*k + 64 E, f] bf16
  float* dx_perm; // [T*k, d]
  // the router's scores kept by the training forward, [E, T]: clean logits (+ bias),
  // and for noisy gating Softplus(x.W_noise) and the noisy scores H
  const float* lg;
  const float* sw;
  const float* hw;
  float* dl;      // [E, T]; for noisy gating dz [E, T] follows it (dz = dl + E T)
  float* dz;
  float* dimp;    // [E]
  float* dload;   // [E]
  float* part;    // split-contraction partial sums
  int64_t part_cap;
};
int64_t backward_padded_rows(int64_t rows_cap, int E);
cudaError_t launch_backward(const BackwardProblem& p, const LaunchCtx& c);

// ---- weight preparation ----------------------------------------------------------
cudaError_t launch_bf16_to_f16(const void* src, void* dst, int64_t n, int32_t* n_inexact,
                               const LaunchCtx& c);

// ---- host helpers shared by the entry points (moe_api.cu) ------------------------
moe_status check_config_host(const moe_config* cfg);  // MOE_OK / INVALID_ARG / UNSUPPORTED
int64_t capacity_host(const moe_config* cfg);         // C, or -1 for no limit
void set_last_launch_count(int32_t n);

// ---- tensor maps -----------------------------------------------------------------
// 2-D tensor map of 2-byte elements (bf16, or fp16 when f16 != 0) over a row-major
// [rows, cols] matrix with a box of [box_rows, 64 columns] and 128-byte swizzling;
// out-of-range elements read as zero.
bool make_tmap_2b(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, int f16);
inline bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows) {
  return make_tmap_2b(map, base, rows, cols, box_rows, 0);
}

}  // namespace moe
