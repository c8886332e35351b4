// kernels.h -- internal launch functions of libmoe_b200.so (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include "common.cuh"

#include <utility>

namespace moe {

// Launch with programmatic stream serialization (the kernel calls pdl_trigger /
// pdl_wait), so its launch overlaps the tail of the previous kernel on `s`.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// route.cu
// arrive / ready_q (optional): per-token counters the route kernel zeroes.
cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx,
                         float* topk_gate, int32_t* blk_hist, uint32_t* arrive_or_null,
                         uint32_t* ready_q_or_null, cudaStream_t s);
cudaError_t launch_hist(const int32_t* topk_idx, int T, int E, int k, int32_t* blk_hist,
                        cudaStream_t s);
cudaError_t launch_colsum(const int32_t* blk_hist, int nblk, int E, int32_t* counts,
                          cudaStream_t s);
// Plan: counts/offsets (from blk_hist when nblk > 0, else from `offsets_in`),
// per-block scatter bases, expert priority order, band table, tile counts,
// zeroed sync counters and the producer/consumer split.
// G = row bands per MMA tile (1: 128-row tiles; 2: 256-row tiles), cg = CTAs per
// tile (consumer CTAs come in whole tiles' CTAs).
cudaError_t launch_plan(const Work& w, int nblk, const int32_t* offsets_in, int T, int d, int f,
                        int E, int k, int num_sms, int consumer_hint, int mgb, int G, int cg,
                        int join, const CostModel& cm, cudaStream_t s);
// With a plan (w.bands etc. set), also fills w.tok_band, GEMM1's gather indices.
cudaError_t launch_scatter(const int32_t* topk_idx, int T, int E, int k, const int32_t* blk_base,
                           int32_t* perm, int32_t* row_of, const Work* plan, cudaStream_t s);
// Expert-parallel owner plan: the owner's received rows (source rank major, then
// local expert) are planned as W*El segments (local expert e, source s), each a
// contiguous run of rows with one destination; bands and tiles follow the
// remote-first order.  recv_base[s]: home row of the first row source s sent.
struct EpPlanIn {
  int W, rank, El, N;
  int recv_base[MAX_W];
};
cudaError_t launch_plan_ep(const Work& w, const int32_t* recv_counts, const EpPlanIn& in, int d,
                           int f, int num_sms, int consumer_hint, int mgb, int G, int cg, int join,
                           const CostModel& cm, cudaStream_t s);
// Home side of the expert-parallel return: waits (bounded) for each token's k rows
// to arrive, combines them exactly as launch_combine does, and zeroes its arrival
// word; a wait that runs out sets *status to MOE_ERR_TIMEOUT (if it was 0).
cudaError_t launch_home_combine(const __nv_bfloat16* y, uint32_t* arrive, const int32_t* row_of,
                                const float* gate, int T, int d, int k, __nv_bfloat16* out,
                                uint32_t* status, uint64_t timeout_ns, int num_sms, cudaStream_t s);

// x_perm[row_of[p]] = x[p / k] for every slot p < T*k (token-major copy).
cudaError_t launch_gather(const __nv_bfloat16* x, const int32_t* row_of, int T, int d, int k,
                          __nv_bfloat16* x_perm, int num_sms, cudaStream_t s);

// combine.cu
// skip (optional): arrive words; tokens flagged TOKEN_DONE are not recomputed.
cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* row_of, const float* gate,
                           int T, int d, int k, __nv_bfloat16* out, int num_sms, cudaStream_t s,
                           const uint32_t* skip = nullptr);

// ffn.cu
enum : int { PH_G1 = 1, PH_G2 = 2, PH_CONS = 4 };

struct FfnArgs {
  Work w;
  const __nv_bfloat16* x_perm;   // A operand of GEMM1 (tiled path)
  const __nv_bfloat16* x;        // token rows for GEMM1's gathered A path
  const int32_t* tok_band;       // [bands][BM] token of each band row (gathered path)
  int gather;                    // GEMM1's A rows from x instead of x_perm: 1 TMA gather4,
                                 // 2 cp.async by extra gather warps (single CTAs)
  __nv_bfloat16* h;              // GEMM1 output / GEMM2 A operand
  __nv_bfloat16* y;              // GEMM2 output
  const void* W1; const void* W3; const void* W2;
  const float* gate;             // [T][k] (consumer role)
  __nv_bfloat16* out;            // [T][d] (consumer role)
  int R, T, d, f, E, k;
  int V;                         // tile variant: 1 one CTA per 128-row tile, 2 a CTA pair per
                                 // 256-row tile (cta_group::2), 3 one CTA per 256-row tile
  int phase;                     // PH_* bits
  int join;                      // producers join the combine when the tile queue drains
  int side;                      // side combine warps (MOE_SCHED_SIDE_COMBINE, single CTAs):
                                 // the CTA whose GEMM2 tile completes a band hands the band's
                                 // arrivals to two extra warps, which also combine ready
                                 // tokens while the tiles run; consumers take no band tickets
  int mgb;
  int b_atoms;                   // single CTA: weight maps are 4-D, one box carries all 64-column atoms
  uint32_t flags;
  uint64_t timeout_ns;
  int n_units;                   // planning units in w.tile_start1 / w.group_start: E on one
                                 // GPU, (local expert, source rank) segments for an EP owner
  // Expert-parallel owner (ep != 0): the consumer role returns each finished band to
  // its home rank instead of combining: the band's rows are copied to
  // ep_home_y[rank] at the combine plan's row (w.band_dest), then the arrival word
  // of each row's token (ep_slot[row] / k) is bumped in ep_home_arrive[rank].
  int ep;
  const int32_t* ep_slot;        // [rows] home slot p = t*k + j of each owner row
  void* ep_home_y[MAX_W];        // [R_home][d] bf16 return buffer of each home rank
  uint32_t* ep_home_arrive[MAX_W];  // [T_home] arrival words of each home rank
};

size_t ffn_smem_bytes();
// CTAs the persistent kernel runs with for tile variant V; also sets the
// kernel's shared-memory attribute for the current device.
cudaError_t ffn_grid(int V, int* grid);

// The CUDA error behind the calling thread's latest MOE_ERR_CUDA (api.cu).
void record_cuda_error(cudaError_t e);
cudaError_t last_cuda_error();
cudaError_t launch_ffn(const FfnArgs& a, int grid, cudaStream_t s);

}  // namespace moe
