// bf16 -> fp16 re-encoding of weight tensors (for fp16 hidden activations, whose
// second product needs W2 in the same 16-bit type as h).
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                                   int64_t n, int32_t* n_inexact) {
  grid_dep_wait();
  grid_dep_launch();
  int inexact = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = __bfloat162float(src[i]);
    const __half h = __float2half_rn(v);
    dst[i] = h;
    inexact += (__half2float(h) != v) ? 1 : 0;
  }
  if (n_inexact != nullptr) {
    for (int o = 16; o > 0; o >>= 1) inexact += __shfl_down_sync(0xffffffffu, inexact, o);
    if ((threadIdx.x & 31) == 0 && inexact) atomicAdd(n_inexact, inexact);
  }
}

cudaError_t launch_bf16_to_f16(const void* src, void* dst, int64_t n, int32_t* n_inexact,
                               const LaunchCtx& c) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(c.num_sms) * 16;
  if (blocks > cap) blocks = cap;
  return launch_kernel(bf16_to_f16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, c,
                       static_cast<const __nv_bfloat16*>(src), static_cast<__half*>(dst), n,
                       n_inexact);
}

}  // namespace moe
