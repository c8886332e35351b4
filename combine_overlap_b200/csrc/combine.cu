// combine.cu -- step (d) as a stand-alone kernel: the weighted reduction over
// all tokens after the expert GEMMs have finished (the sequential mode, and the
// moe_combine entry point).  One warp per token, 16-byte vector loads of the k
// expert-output rows, fp32 accumulation in slot order, 16-byte stores.
#include "kernels.h"
#include "combine.cuh"

namespace moe {

// skip (optional): tokens whose arrive word has TOKEN_DONE set were already
// combined by the persistent kernel's consumers and are left alone.
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                      const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ gate, int T, int d,
                                                      int k, __nv_bfloat16* __restrict__ out,
                                                      const uint32_t* __restrict__ skip) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    if (skip && (skip[t] & TOKEN_DONE)) continue;
    combine_token_warp(y, row_of, gate, t, d, k, out, lane);
  }
}

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* row_of, const float* gate,
                           int T, int d, int k, __nv_bfloat16* out, int num_sms, cudaStream_t s,
                           const uint32_t* skip) {
  const int grid = max(1, min(cdiv(T, 8), num_sms * 8));
  return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, s, y, row_of, gate, T, d, k, out, skip);
}

}  // namespace moe
