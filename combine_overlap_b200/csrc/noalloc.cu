// noalloc.cu -- moe_permute_noalloc: the expert-contiguous permutation for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc on the path where they permute tokens: a
// runtime that has already handed all device memory to its own pool, code that
// runs while a CUDA graph is being built around it, or a plug-in host that owns
// every allocation.  moe_permute needs a caller-provided workspace for its
// per-block histograms and scan bases; this variant takes that scratch from a
// fixed array compiled into the library instead, so the caller only passes the
// inputs and outputs.
//
// The scratch is one file-scope __device__ array of PERMUTE_NOALLOC_SCRATCH_BYTES
// (a little over 4 MiB), present on every GPU that loads the library until the
// process exits.  In host code the array's name is only a host-side stand-in,
// never a device address, so its device address is looked up with
// cudaGetSymbolAddress (with that device current) and cached per device and per
// CUDA context: after cudaDeviceReset the device gets a new primary context, in
// which the library's module (and so the array) may sit at another address, and
// the first call in the new context looks it up again.
#include "kernels.h"
#include "../../include/moe.h"

#include <cuda.h>
#include <mutex>
#include <string.h>

namespace {

using namespace moe;

constexpr int NOALLOC_MAX_T = 65536;
constexpr int NOALLOC_MAX_BLK = (NOALLOC_MAX_T + ROUTE_TOK - 1) / ROUTE_TOK;   // 2048
constexpr size_t HDR_BYTES = 512;   // Status + Sync, padded to 512 bytes
constexpr size_t CNT_BYTES = (size_t)MAX_E * sizeof(int32_t);   // counts when the caller passes none
constexpr size_t HIST_BYTES = (size_t)NOALLOC_MAX_BLK * MAX_E * sizeof(int32_t);
constexpr size_t PERMUTE_NOALLOC_SCRATCH_BYTES = HDR_BYTES + CNT_BYTES + 2 * HIST_BYTES;

static_assert(sizeof(Status) + sizeof(Sync) <= HDR_BYTES, "header does not fit");

// Shared by every call on a device; holds whatever the last call left in it.
static __device__ __align__(256) unsigned char g_permute_scratch[PERMUTE_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mutex;
void* g_scratch_ptr[MAX_DEVICES] = {nullptr};
CUcontext g_scratch_ctx[MAX_DEVICES] = {nullptr};   // the context g_scratch_ptr[dev] belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current driver context (null if the runtime has not made
// one current yet).  The driver entry point is looked up once through the
// runtime, so the library needs no link against libcuda.
cudaError_t current_context(CUcontext* ctx) {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return cudaErrorNotSupported;
    fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn(ctx) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of g_permute_scratch on the current device (looked up on the
// first call on that device, and again whenever the device's context changed,
// e.g. after cudaDeviceReset; cached otherwise).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  CUcontext ctx = nullptr;
  // cudaGetSymbolAddress makes the device's primary context current if none is,
  // so the context is read after it on a miss
  if (current_context(&ctx) == cudaSuccess && ctx && g_scratch_ptr[dev] && ctx == g_scratch_ctx[dev]) {
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_permute_scratch);
  if (e != cudaSuccess) return e;
  if (!p) return cudaErrorInvalidSymbol;
  e = current_context(&ctx);
  if (e != cudaSuccess) return e;
  g_scratch_ptr[dev] = p;
  g_scratch_ctx[dev] = ctx;
  *out = p;
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline moe_status fail(cudaError_t e) {
  record_cuda_error(e);
  return MOE_ERR_CUDA;
}

}  // namespace

extern "C" size_t moe_permute_noalloc_scratch_bytes(void) { return PERMUTE_NOALLOC_SCRATCH_BYTES; }

extern "C" moe_status moe_permute_noalloc(const void* x, int T, int d, int E, int k,
                                          const int32_t* topk_idx, int32_t* counts,
                                          int32_t* offsets, int32_t* perm, int32_t* row_of,
                                          void* x_perm, void* stream) {
  if (T < 1 || E < 1 || k < 1 || k > E || d < 1) return MOE_ERR_INVALID;
  if (E > MAX_E || k > MAX_K || d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (T > NOALLOC_MAX_T) return MOE_ERR_UNSUPPORTED;   // beyond the fixed scratch
  const void* req[] = {x, topk_idx, offsets, perm, row_of, x_perm};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID;
  if (counts && !aligned16(counts)) return MOE_ERR_INVALID;

  void* base = nullptr;
  if (const cudaError_t e = scratch_address(&base); e != cudaSuccess) return fail(e);
  char* s = static_cast<char*>(base);
  const int nblk = route_blocks(T);
  Work w;
  memset(&w, 0, sizeof(w));
  w.status = reinterpret_cast<Status*>(s);
  w.sync = reinterpret_cast<Sync*>(s + sizeof(Status));
  w.blk_hist = reinterpret_cast<int32_t*>(s + HDR_BYTES + CNT_BYTES);
  w.blk_base = reinterpret_cast<int32_t*>(s + HDR_BYTES + CNT_BYTES + HIST_BYTES);
  // the plan kernel always stores counts: into the caller's buffer, else the scratch
  w.counts = counts ? counts : reinterpret_cast<int32_t*>(s + HDR_BYTES);
  w.offsets = offsets;
  w.perm = perm;
  w.row_of = row_of;
  // Nothing in the scratch has to start at zero: the histogram kernel writes
  // every block's counts, the plan kernel writes the bases, counts and status.
  int nsm = 0, dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return fail(e);
  if (const cudaError_t e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
      e != cudaSuccess)
    return fail(e);
  CostModel cm;
  cm.mma_flops_per_sm = 1.0f;
  cm.copy_bytes_per_sm = 1.0f;
  cm.hbm_bytes = 1.0f;
  cm.max_consumers = 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_hist(topk_idx, T, E, k, w.blk_hist, st);
  if (e == cudaSuccess) e = launch_plan(w, nblk, nullptr, T, BN2, BN1, E, k, nsm, 1, 1, 1, 1, 1, cm, st);
  if (e == cudaSuccess) e = launch_scatter(topk_idx, T, E, k, w.blk_base, perm, row_of, nullptr, st);
  if (e == cudaSuccess)
    e = launch_gather(static_cast<const __nv_bfloat16*>(x), row_of, T, d, k,
                      static_cast<__nv_bfloat16*>(x_perm), nsm, st);
  if (e != cudaSuccess) return fail(e);
  return MOE_OK;
}
