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

// The home rank's combine of the expert-parallel return: one warp per token waits
// (bounded, system-scope acquire) until the owners have landed the token's k rows
// and bumped its arrival word to k, then combines exactly as combine_kernel does
// (the same per-token routine, so the same bits as the one-GPU layer) and zeroes
// the arrival word for the next call.  A wait that runs out records
// MOE_ERR_TIMEOUT in *status (first error wins) and ends every other wait.
__global__ void __launch_bounds__(256) home_combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                           uint32_t* __restrict__ arrive,
                                                           const int32_t* __restrict__ row_of,
                                                           const float* __restrict__ gate, int T,
                                                           int d, int k,
                                                           __nv_bfloat16* __restrict__ out,
                                                           uint32_t* status, uint64_t timeout_ns) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const volatile uint32_t* abort = status;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    int ok = 1;
    if (lane == 0) {
      if (ld_acquire_sys(&arrive[t]) < (uint32_t)k) {
        const uint64_t deadline = globaltimer() + timeout_ns;
        uint32_t ns = 32;
        while (ld_acquire_sys(&arrive[t]) < (uint32_t)k) {
          if (*abort) { ok = 0; break; }
          if (globaltimer() > deadline) {
            atomicCAS(status, 0u, 4u);   // MOE_ERR_TIMEOUT
            ok = 0;
            break;
          }
          __nanosleep(ns);
          if (ns < 1024) ns <<= 1;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) continue;
    (void)ld_acquire_sys(&arrive[t]);   // every lane's reads of the rows come after the arrival
    combine_token_warp(y, row_of, gate, t, d, k, out, lane);
    __syncwarp();
    if (lane == 0) arrive[t] = 0u;
  }
}

cudaError_t launch_home_combine(const __nv_bfloat16* y, uint32_t* arrive, const int32_t* row_of,
                                const float* gate, int T, int d, int k, __nv_bfloat16* out,
                                uint32_t* status, uint64_t timeout_ns, int num_sms, cudaStream_t s) {
  const int grid = max(1, min(cdiv(T, 8), num_sms * 8));
  return launch_pdl(home_combine_kernel, dim3(grid), dim3(256), 0, s, y, arrive, row_of, gate, T, d, k,
                    out, status, timeout_ns);
}

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* row_of, const float* gate,
                           int T, int d, int k, __nv_bfloat16* out, int num_sms, cudaStream_t s,
                           const uint32_t* skip) {
  const int grid = max(1, min(cdiv(T, 8), num_sms * 8));
  return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, s, y, row_of, gate, T, d, k, out, skip);
}

}  // namespace moe
