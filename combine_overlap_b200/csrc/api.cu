// api.cu -- the C ABI of libmoe_b200.so (declared in include/moe.h): argument
// checks, the workspace carve-up and the launch sequence of each entry point.
#include "kernels.h"
#include "../../include/moe.h"

#include <stdint.h>
#include <string.h>

#include <vector>

namespace moe {
namespace {
// The CUDA error behind the calling thread's latest MOE_ERR_CUDA.
thread_local cudaError_t g_last_cuda = cudaSuccess;
}  // namespace
void record_cuda_error(cudaError_t e) { g_last_cuda = e; }
cudaError_t last_cuda_error() { return g_last_cuda; }
}  // namespace moe

namespace {

using namespace moe;

constexpr size_t ALIGN = 256;

inline size_t up(size_t v) { return (v + ALIGN - 1) & ~(ALIGN - 1); }

// Workspace regions.  The status block sits at offset 0 so moe_get_status can
// find it without the shape.  The routing part depends on (T, E, k) only and is
// all moe_route / moe_permute need; the plan part adds the band tables; the
// last part holds the permuted activations and the expert intermediates.
struct Layout {
  size_t status, sync, stamps, blk_hist, blk_base, counts, offsets, topk_idx, topk_gate, perm, row_of, arrive, ready_q;
  size_t routing_end;
  size_t sorted_e, band_start, tile_start1, bands, band_done1, band_done2, groups, group_start,
      tok_band, expert_rank, band_dest, g2_start;
  size_t plan_end;
  size_t x_perm, h, y;
  size_t total;
};

Layout layout(int T, int d, int f, int E, int k) {
  Layout L;
  const size_t R = (size_t)T * k;
  const size_t nblk = (size_t)route_blocks(T);
  const size_t mb = (size_t)max_bands((int)R, E);
  size_t o = 0;
  L.status = o; o = up(o + sizeof(Status));
  L.sync = o; o = up(o + sizeof(Sync));
  L.stamps = o; o = up(o + ((size_t)STAMP_CTAS * NSTAMP + (size_t)STAMP_BANDS * 4) * 8);
  L.blk_hist = o; o = up(o + nblk * E * 4);
  L.blk_base = o; o = up(o + nblk * E * 4);
  L.counts = o; o = up(o + (size_t)E * 4);
  L.offsets = o; o = up(o + (size_t)(E + 1) * 4);
  L.topk_idx = o; o = up(o + R * 4);
  L.topk_gate = o; o = up(o + R * 4);
  L.perm = o; o = up(o + R * 4);
  L.row_of = o; o = up(o + R * 4);
  L.arrive = o; o = up(o + (size_t)T * 4);
  L.ready_q = o; o = up(o + (size_t)T * 4);
  L.routing_end = o;
  L.sorted_e = o; o = up(o + (size_t)E * 4);
  L.band_start = o; o = up(o + (size_t)(E + 1) * 4);
  L.tile_start1 = o; o = up(o + (size_t)(E + 1) * 4);
  L.bands = o; o = up(o + mb * sizeof(Band));
  L.band_done1 = o; o = up(o + mb * 4);
  L.band_done2 = o; o = up(o + mb * 4);
  L.groups = o; o = up(o + mb * sizeof(Group));
  L.group_start = o; o = up(o + (size_t)(E + 1) * 4);
  L.tok_band = o; o = up(o + mb * BM * 4);
  L.expert_rank = o; o = up(o + (size_t)E * 4);
  L.g2_start = o; o = up(o + (size_t)(E + 1) * 4);
  L.band_dest = o; o = up(o + mb * sizeof(int2));
  L.plan_end = o;
  L.x_perm = o; o = up(o + R * d * 2);
  L.h = o; o = up(o + R * f * 2);
  L.y = o; o = up(o + R * d * 2);
  L.total = o;
  return L;
}

// Band-table capacity of a layout (the band_dest region holds one int2 per band).
int max_bands_of(const Layout& L) { return (int)((L.plan_end - L.band_dest) / sizeof(int2)); }

template <class T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

Work work_from(void* ws, const Layout& L, bool plan, bool acts) {
  Work w;
  memset(&w, 0, sizeof(w));
  w.status = at<Status>(ws, L.status);
  w.sync = at<Sync>(ws, L.sync);
  w.stamps = at<unsigned long long>(ws, L.stamps);
  w.blk_hist = at<int32_t>(ws, L.blk_hist);
  w.blk_base = at<int32_t>(ws, L.blk_base);
  w.counts = at<int32_t>(ws, L.counts);
  w.offsets = at<int32_t>(ws, L.offsets);
  w.topk_idx = at<int32_t>(ws, L.topk_idx);
  w.topk_gate = at<float>(ws, L.topk_gate);
  w.perm = at<int32_t>(ws, L.perm);
  w.row_of = at<int32_t>(ws, L.row_of);
  w.arrive = at<uint32_t>(ws, L.arrive);
  w.ready_q = at<uint32_t>(ws, L.ready_q);
  if (plan) {
    w.sorted_e = at<int32_t>(ws, L.sorted_e);
    w.band_start = at<int32_t>(ws, L.band_start);
    w.tile_start1 = at<int32_t>(ws, L.tile_start1);
    w.bands = at<Band>(ws, L.bands);
    w.band_done1 = at<uint32_t>(ws, L.band_done1);
    w.band_done2 = at<uint32_t>(ws, L.band_done2);
    w.groups = at<Group>(ws, L.groups);
    w.group_start = at<int32_t>(ws, L.group_start);
    w.tok_band = at<int32_t>(ws, L.tok_band);
    w.expert_rank = at<int32_t>(ws, L.expert_rank);
    w.g2_start = at<int32_t>(ws, L.g2_start);
    // the combine plan exists only for an expert-parallel owner (set by its entry)
  }
  if (acts) {
    w.x_perm = at<__nv_bfloat16>(ws, L.x_perm);
    w.h = at<__nv_bfloat16>(ws, L.h);
    w.y = at<__nv_bfloat16>(ws, L.y);
  }
  return w;
}

// Shape checks: MOE_ERR_INVALID for meaningless shapes, MOE_ERR_UNSUPPORTED for
// valid MoE shapes outside what the kernels tile.
moe_status check_route_shape(int T, int E, int k) {
  if (T < 1 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID;
  if (E > MAX_E || k > MAX_K) return MOE_ERR_UNSUPPORTED;
  if ((long long)T * k > (1LL << 30)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_shape(int T, int d, int f, int E, int k) {
  moe_status s = check_route_shape(T, E, k);
  if (s != MOE_OK) return s;
  if (d < 1 || f < 1) return MOE_ERR_INVALID;
  if (d % BN2 != 0 || f % BN1 != 0) return MOE_ERR_UNSUPPORTED;
  if ((long long)T * k * (d > f ? d : f) >= (1LL << 40)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
inline bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

int sms_cache[64] = {0};

inline moe_status cuda_fail(cudaError_t e) {
  moe::record_cuda_error(e);
  return MOE_ERR_CUDA;
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64 && sms_cache[dev] > 0) return sms_cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) sms_cache[dev] = n;
  return n;
}

// Per-SM throughputs for the split cost model (the search starts at one dedicated
// consumer CTA group; see choose_consumers), from B200 measurements: a
// producer SM sustains about 1/148 of ~1.2 PFLOP/s of bf16 MMA inside this kernel
// (power-capped), one consumer SM moves about 30 GB/s of combine traffic (bulk
// reads of expert rows plus output stores), HBM ~6.5 TB/s.
CostModel default_cost_model() {
  CostModel cm;
  cm.mma_flops_per_sm = 1.2e15f / 148.0f;
  cm.copy_bytes_per_sm = 30.0e9f;
  cm.hbm_bytes = 6.5e12f;
  cm.max_consumers = 32;
  return cm;
}

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : cuda_fail(e); }

// Tile variant (FfnArgs::V).  A CTA pair (V = 2: 256-row tiles, cta_group::2) or
// a single CTA with two 128-row MMAs per K step (V = 3: 256-row tiles) streams a
// third less operand data per FLOP than a single CTA with 128-row tiles (V = 1),
// but a 256-row tile wastes more masked rows when experts are small, a pair
// couples two SMs' loads, and V = 3 gives up the accumulator double-buffering.
// Measured on B200, one variant per process (alternating two kernels step by
// step penalises the pair): V = 3 is 4-9 % faster than V = 1 from 256 rows per
// expert up (T=2048-32768 at d_ff = 2048, the fine-grained and imbalanced
// layers) and 6-8 % faster than pairs on the Mixtral-shaped layer; at 64 rows
// per expert V = 1 is 4 % faster.  So V = 3 when T*k/E >= 256, else V = 1.
// Flags force a variant (MOE_SCHED_ONE_CTA before MOE_SCHED_CTA_PAIR before
// MOE_SCHED_WIDE_CTA).
int choose_variant(int T, int f, int E, int k, unsigned flags) {
  (void)f;
  if (flags & MOE_SCHED_ONE_CTA) return 1;
  if (flags & MOE_SCHED_CTA_PAIR) return 2;
  if (flags & MOE_SCHED_WIDE_CTA) return 3;
  return (long long)T * k >= 256LL * E ? 3 : 1;
}

inline int bands_per_tile(int V) { return V == 1 ? 1 : 2; }
inline int ctas_per_tile(int V) { return V == 2 ? 2 : 1; }

#define MOE_TRY(expr)                                   \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_);        \
  } while (0)

}  // namespace

extern "C" {

size_t moe_workspace_size(int T, int d, int f, int E, int k) {
  if (check_shape(T, d, f, E, k) != MOE_OK) return 0;
  return layout(T, d, f, E, k).total;
}

int moe_tile_variant(int T, int f, int E, int k, unsigned flags) {
  if (T < 1 || f < 1 || E < 1 || k < 1) return 0;
  return choose_variant(T, f, E, k, flags);
}

int moe_last_cuda_error(void) { return (int)moe::last_cuda_error(); }

const char* moe_cuda_error_string(int code) {
  return cudaGetErrorString(static_cast<cudaError_t>(code));
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "a bounded device wait ran out";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int moe_num_sms(void) { return device_sms(); }

moe_status moe_route(const float* logits, int T, int E, int k, int32_t* topk_idx,
                     float* topk_gate, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  moe_status s = check_route_shape(T, E, k);
  if (s != MOE_OK) return s;
  if (!ok_ptr(logits) || !ok_ptr(topk_idx) || !ok_ptr(topk_gate) || !ok_opt(counts))
    return MOE_ERR_INVALID;
  // any shape's full workspace covers the routing part; d/f do not matter here
  const Layout L = layout(T, BN2, BN1, E, k);
  if (!ws || !aligned16(ws) || ws_bytes < L.routing_end) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Work w = work_from(ws, L, false, false);
  MOE_TRY(launch_route(logits, T, E, k, topk_idx, topk_gate, w.blk_hist, nullptr, nullptr, st));
  if (counts) MOE_TRY(launch_colsum(w.blk_hist, route_blocks(T), E, counts, st));
  return MOE_OK;
}

moe_status moe_permute(const void* x, int T, int d, int E, int k, const int32_t* topk_idx,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of,
                       void* x_perm, void* ws, size_t ws_bytes, void* stream) {
  moe_status s = check_route_shape(T, E, k);
  if (s != MOE_OK) return s;
  if (d < 1) return MOE_ERR_INVALID;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!ok_ptr(x) || !ok_ptr(topk_idx) || !ok_ptr(offsets) || !ok_ptr(perm) || !ok_ptr(row_of) ||
      !ok_ptr(x_perm) || !ok_opt(counts))
    return MOE_ERR_INVALID;
  const Layout L = layout(T, BN2, BN1, E, k);
  if (!ws || !aligned16(ws) || ws_bytes < L.routing_end) return MOE_ERR_WORKSPACE;
  const int nsm = device_sms();
  if (nsm <= 0) return cuda_fail(cudaErrorInvalidDevice);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Work w = work_from(ws, L, false, false);
  if (counts) w.counts = counts;
  w.offsets = offsets;
  w.perm = perm;
  w.row_of = row_of;
  const int nblk = route_blocks(T);
  MOE_TRY(launch_hist(topk_idx, T, E, k, w.blk_hist, st));
  MOE_TRY(launch_plan(w, nblk, nullptr, T, BN2, BN1, E, k, nsm, 1, 1, 1, 1, 1, default_cost_model(), st));
  MOE_TRY(launch_scatter(topk_idx, T, E, k, w.blk_base, perm, row_of, nullptr, st));
  MOE_TRY(launch_gather(static_cast<const __nv_bfloat16*>(x), row_of, T, d, k,
                        static_cast<__nv_bfloat16*>(x_perm), nsm, st));
  return MOE_OK;
}

moe_status moe_grouped_ffn(const void* x_perm, const int32_t* offsets, int T, int d, int f, int E,
                           int k, const void* W1, const void* W3, const void* W2, void* h, void* y,
                           unsigned flags, void* ws, size_t ws_bytes, void* stream) {
  moe_status s = check_shape(T, d, f, E, k);
  if (s != MOE_OK) return s;
  if (!ok_ptr(x_perm) || !ok_ptr(offsets) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
      !ok_ptr(y) || !ok_opt(h))
    return MOE_ERR_INVALID;
  constexpr unsigned tile_flags = MOE_SCHED_ONE_CTA | MOE_SCHED_CTA_PAIR | MOE_SCHED_WIDE_CTA |
                                  MOE_SCHED_B_PER_ATOM | MOE_SCHED_FULL_TILES |
                                  MOE_SCHED_INTERLEAVE | MOE_SCHED_EVICT_FIRST | MOE_SCHED_EXP_SILU;
  if (flags & ~tile_flags) return MOE_ERR_INVALID;
  const Layout L = layout(T, d, f, E, k);
  if (!ws || !aligned16(ws) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const int V = choose_variant(T, f, E, k, flags);
  int grid = 0;
  MOE_TRY(ffn_grid(V, &grid));
  if (grid <= ctas_per_tile(V)) return cuda_fail(cudaErrorInvalidConfiguration);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Work w = work_from(ws, L, true, true);
  MOE_TRY(launch_plan(w, 0, offsets, T, d, f, E, k, grid, 1, 1, bands_per_tile(V), ctas_per_tile(V),
                      1, default_cost_model(), st));
  FfnArgs a;
  memset(&a, 0, sizeof(a));
  a.w = w;
  a.x_perm = static_cast<const __nv_bfloat16*>(x_perm);
  a.h = h ? static_cast<__nv_bfloat16*>(h) : w.h;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.W1 = W1; a.W3 = W3; a.W2 = W2;
  a.R = T * k; a.T = T; a.d = d; a.f = f; a.E = E; a.k = k;
  a.n_units = E;
  a.V = V;
  a.phase = PH_G1 | PH_G2;
  a.join = 0;
  a.mgb = 1;
  a.flags = flags;
  a.timeout_ns = 2000000000ull;
  MOE_TRY(launch_ffn(a, grid, st));
  return MOE_OK;
}

moe_status moe_combine(const void* y, const int32_t* row_of, const float* topk_gate, int T, int d,
                       int k, void* out, void* stream) {
  if (T < 1 || d < 1 || k < 1) return MOE_ERR_INVALID;
  if (k > MAX_K || d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!ok_ptr(y) || !ok_ptr(row_of) || !ok_ptr(topk_gate) || !ok_ptr(out)) return MOE_ERR_INVALID;
  const int nsm = device_sms();
  if (nsm <= 0) return cuda_fail(cudaErrorInvalidDevice);
  return cuda_status(launch_combine(static_cast<const __nv_bfloat16*>(y), row_of, topk_gate, T, d, k,
                                    static_cast<__nv_bfloat16*>(out), nsm,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_forward(const moe_layer_args* args, moe_mode mode, void* ws, size_t ws_bytes,
                             void* stream) {
  if (!args) return MOE_ERR_INVALID;
  const moe_layer_args& A = *args;
  moe_status s = check_shape(A.T, A.d, A.f, A.E, A.k);
  if (s != MOE_OK) return s;
  if (mode != MOE_MODE_SEQUENTIAL && mode != MOE_MODE_OVERLAPPED) return MOE_ERR_INVALID;
  // identity experts read no weights: W1, W3, W2 may then be NULL
  const bool identity = (A.flags & MOE_DBG_IDENTITY_EXPERTS) != 0;
  auto ok_w = [&](const void* p) { return identity ? ok_opt(p) : ok_ptr(p); };
  if (!ok_ptr(A.x) || !ok_ptr(A.logits) || !ok_w(A.W1) || !ok_w(A.W3) || !ok_w(A.W2) ||
      !ok_ptr(A.out) || !ok_opt(A.topk_idx) || !ok_opt(A.topk_gate) || !ok_opt(A.counts) ||
      !ok_opt(A.offsets) || !ok_opt(A.perm))
    return MOE_ERR_INVALID;
  if (A.consumer_sms < 0 || A.mgb < 0 || A.timeout_us < 0) return MOE_ERR_INVALID;
  const Layout L = layout(A.T, A.d, A.f, A.E, A.k);
  if (!ws || !aligned16(ws) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const int nsm = device_sms();
  // MOE_SCHED_GATHER_A: GEMM1 gathers its A rows from x with TMA gather4 instead
  // of reading x_perm (no x_perm pass, but 32 gather instructions per k-block);
  // 128-row gathers only, so not with V = 3
  // MOE_SCHED_GATHER_LSU: the same, by extra warps with cp.async (single CTAs only)
  const int gather_a = (A.flags & MOE_DBG_IDENTITY_EXPERTS) ? 0
                       : (A.flags & MOE_SCHED_GATHER_LSU) ? 2
                       : (A.flags & MOE_SCHED_GATHER_A) ? 1 : 0;
  const int V = choose_variant(A.T, A.f, A.E, A.k, A.flags);
  if (gather_a == 2 && V == 2) return MOE_ERR_UNSUPPORTED;
  // MOE_SCHED_SIDE_COMBINE: side combine warps in every producer CTA (single CTAs;
  // CTA pairs keep the ticketed consumer protocol); exclusive with the LSU gather,
  // which uses the same extra warps
  const bool side_flag = (A.flags & MOE_SCHED_SIDE_COMBINE) != 0;
  if (side_flag && gather_a == 2) return MOE_ERR_UNSUPPORTED;
  const int side = (side_flag && V != 2 && mode == MOE_MODE_OVERLAPPED) ? 1 : 0;
  int grid = 0;
  MOE_TRY(ffn_grid(V, &grid));
  if (nsm <= 1 || grid <= ctas_per_tile(V)) return cuda_fail(cudaErrorInvalidConfiguration);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Work w = work_from(ws, L, true, true);
  if (!gather_a) w.tok_band = nullptr;   // GEMM1's gather indices exist only on that path
  if (A.topk_idx) w.topk_idx = A.topk_idx;
  if (A.topk_gate) w.topk_gate = A.topk_gate;
  if (A.counts) w.counts = A.counts;
  if (A.offsets) w.offsets = A.offsets;
  if (A.perm) w.perm = A.perm;
  const int T = A.T, d = A.d, f = A.f, E = A.E, k = A.k, R = T * k;
  const int mgb = A.mgb > 0 ? A.mgb : 1;
  const int nblk = route_blocks(T);
  MOE_TRY(launch_route(A.logits, T, E, k, w.topk_idx, w.topk_gate, w.blk_hist, w.arrive, w.ready_q, st));
  const int join = (A.flags & MOE_SCHED_NO_JOIN) ? 0 : 1;
  // with side warps no SM is a dedicated consumer unless the caller asks for some
  const int consumer_hint = (side && A.consumer_sms == 0) ? -1 : A.consumer_sms;
  MOE_TRY(launch_plan(w, nblk, nullptr, T, d, f, E, k, grid, consumer_hint, mgb, bands_per_tile(V),
                      ctas_per_tile(V), join,
                      default_cost_model(), st));
  // Default: a gather kernel writes x_perm and GEMM1 reads it with tiled TMA loads.
  MOE_TRY(launch_scatter(w.topk_idx, T, E, k, w.blk_base, w.perm, w.row_of, gather_a ? &w : nullptr, st));
  if (!gather_a)
    MOE_TRY(launch_gather(static_cast<const __nv_bfloat16*>(A.x), w.row_of, T, d, k, w.x_perm, nsm, st));
  if (identity) {
    // identity experts: y = x_perm, so the combine reads the permuted rows directly
    if (A.ev_ffn_begin) MOE_TRY(cudaEventRecord(static_cast<cudaEvent_t>(A.ev_ffn_begin), st));
    if (A.ev_ffn_end) MOE_TRY(cudaEventRecord(static_cast<cudaEvent_t>(A.ev_ffn_end), st));
    MOE_TRY(launch_combine(w.x_perm, w.row_of, w.topk_gate, T, d, k,
                           static_cast<__nv_bfloat16*>(A.out), nsm, st));
    return MOE_OK;
  }
  FfnArgs a;
  memset(&a, 0, sizeof(a));
  a.w = w;
  a.x_perm = w.x_perm;
  a.x = static_cast<const __nv_bfloat16*>(A.x);
  a.tok_band = w.tok_band;
  a.gather = gather_a;
  a.h = w.h;
  a.y = w.y;
  a.W1 = A.W1; a.W3 = A.W3; a.W2 = A.W2;
  a.gate = w.topk_gate;
  a.out = static_cast<__nv_bfloat16*>(A.out);
  a.R = R; a.T = T; a.d = d; a.f = f; a.E = E; a.k = k;
  a.n_units = E;
  a.V = V;
  a.mgb = mgb;
  a.flags = A.flags;
  a.timeout_ns = (A.timeout_us > 0 ? (uint64_t)A.timeout_us : 2000000ull) * 1000ull;
  if (A.ev_ffn_begin) MOE_TRY(cudaEventRecord(static_cast<cudaEvent_t>(A.ev_ffn_begin), st));
  if (mode == MOE_MODE_OVERLAPPED) {
    a.phase = PH_G1 | PH_G2 | PH_CONS;
    a.join = join;
    a.side = side;
    MOE_TRY(launch_ffn(a, grid, st));
    if (A.ev_ffn_end) MOE_TRY(cudaEventRecord(static_cast<cudaEvent_t>(A.ev_ffn_end), st));
    // Consumers stop once the GEMM work is done; a full-occupancy combine pass
    // finishes every token they did not (same arithmetic, so the same bits).
    MOE_TRY(launch_combine(w.y, w.row_of, w.topk_gate, T, d, k, a.out, nsm, st, w.arrive));
  } else {
    a.phase = PH_G1;
    MOE_TRY(launch_ffn(a, grid, st));
    a.phase = PH_G2;
    MOE_TRY(launch_ffn(a, grid, st));
    if (A.ev_ffn_end) MOE_TRY(cudaEventRecord(static_cast<cudaEvent_t>(A.ev_ffn_end), st));
    MOE_TRY(launch_combine(w.y, w.row_of, w.topk_gate, T, d, k, a.out, nsm, st));
  }
  return MOE_OK;
}

size_t moe_ep_owner_workspace_size(int N, int d, int f, int El, int W) {
  if (N < 0 || d < 1 || f < 1 || El < 1 || W < 1 || W > MAX_W || (long long)El * W > MAX_E) return 0;
  if (d % BN2 != 0 || f % BN1 != 0) return 0;
  if ((long long)N * (d > f ? d : f) >= (1LL << 40)) return 0;
  // rows N (k = 1), planning units W * El
  return layout(N > 0 ? N : 1, d, f, El * W, 1).total;
}

moe_status moe_ep_owner_forward(const moe_ep_owner_args* args, moe_mode mode, void* ws,
                                size_t ws_bytes, void* stream) {
  if (!args) return MOE_ERR_INVALID;
  const moe_ep_owner_args& A = *args;
  if (A.W < 1 || A.rank < 0 || A.rank >= A.W || A.El < 1 || A.N < 0 || A.d < 1 || A.f < 1 ||
      A.k < 1)
    return MOE_ERR_INVALID;
  if (A.W > MAX_W || (long long)A.El * A.W > MAX_E || A.k > MAX_K) return MOE_ERR_UNSUPPORTED;
  if (A.d % BN2 != 0 || A.f % BN1 != 0) return MOE_ERR_UNSUPPORTED;
  if ((long long)A.N * (A.d > A.f ? A.d : A.f) >= (1LL << 40)) return MOE_ERR_UNSUPPORTED;
  if (mode != MOE_MODE_SEQUENTIAL && mode != MOE_MODE_OVERLAPPED) return MOE_ERR_INVALID;
  if (A.consumer_sms < 0 || A.mgb < 0 || A.timeout_us < 0) return MOE_ERR_INVALID;
  if (!ok_ptr(A.x_recv) || !ok_ptr(A.slot_recv) || !ok_ptr(A.recv_counts) || !ok_ptr(A.W1) ||
      !ok_ptr(A.W3) || !ok_ptr(A.W2))
    return MOE_ERR_INVALID;
  for (int r = 0; r < A.W; ++r) {
    if (!ok_ptr(A.home_y[r]) || !A.home_arrive[r] || (reinterpret_cast<uintptr_t>(A.home_arrive[r]) & 3u))
      return MOE_ERR_INVALID;
    if (A.recv_base[r] < 0) return MOE_ERR_INVALID;
  }
  const int U = A.El * A.W;
  const Layout L = layout(A.N > 0 ? A.N : 1, A.d, A.f, U, 1);
  if (!ws || !aligned16(ws) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const int nsm = device_sms();
  int V = choose_variant(A.N > 0 ? A.N : 1, A.f, U, 1, A.flags);
  int grid = 0;
  MOE_TRY(ffn_grid(V, &grid));
  if (nsm <= 1 || grid <= ctas_per_tile(V)) return cuda_fail(cudaErrorInvalidConfiguration);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Work w = work_from(ws, L, true, true);
  w.band_dest = at<int2>(ws, L.band_dest);
  w.tok_band = nullptr;
  w.expert_rank = nullptr;
  const int mgb = A.mgb > 0 ? A.mgb : 1;
  const int join = (A.flags & MOE_SCHED_NO_JOIN) ? 0 : 1;
  EpPlanIn in;
  memset(&in, 0, sizeof(in));
  in.W = A.W; in.rank = A.rank; in.El = A.El; in.N = A.N;
  for (int r = 0; r < A.W; ++r) in.recv_base[r] = A.recv_base[r];
  MOE_TRY(launch_plan_ep(w, A.recv_counts, in, A.d, A.f, grid, A.consumer_sms, mgb, bands_per_tile(V),
                         ctas_per_tile(V), join, default_cost_model(), st));
  if (A.N == 0) return MOE_OK;   // nothing received: no tile, no row to return
  FfnArgs a;
  memset(&a, 0, sizeof(a));
  a.w = w;
  a.x_perm = static_cast<const __nv_bfloat16*>(A.x_recv);
  a.h = w.h;
  a.y = w.y;
  a.W1 = A.W1; a.W3 = A.W3; a.W2 = A.W2;
  a.R = A.N; a.T = A.N; a.d = A.d; a.f = A.f; a.E = A.El; a.k = A.k;
  a.n_units = U;
  a.V = V;
  a.mgb = mgb;
  a.flags = A.flags & ~(MOE_SCHED_GATHER_A | MOE_DBG_IDENTITY_EXPERTS);
  a.timeout_ns = (A.timeout_us > 0 ? (uint64_t)A.timeout_us : 2000000ull) * 1000ull;
  a.ep = 1;
  a.ep_slot = A.slot_recv;
  for (int r = 0; r < A.W; ++r) {
    a.ep_home_y[r] = A.home_y[r];
    a.ep_home_arrive[r] = A.home_arrive[r];
  }
  if (mode == MOE_MODE_OVERLAPPED) {
    a.phase = PH_G1 | PH_G2 | PH_CONS;
    a.join = join;
    MOE_TRY(launch_ffn(a, grid, st));
  } else {
    // the baseline: expert compute, then the whole return as a separate pass
    a.phase = PH_G1;
    MOE_TRY(launch_ffn(a, grid, st));
    a.phase = PH_G2;
    MOE_TRY(launch_ffn(a, grid, st));
    a.phase = PH_CONS;
    a.join = 1;
    MOE_TRY(launch_ffn(a, grid, st));
  }
  return MOE_OK;
}

moe_status moe_ep_home_combine(const void* home_y, uint32_t* arrive, const int32_t* row_of,
                               const float* topk_gate, int T, int d, int k, void* out,
                               uint32_t* status, int timeout_us, void* stream) {
  if (T < 1 || d < 1 || k < 1 || timeout_us < 0) return MOE_ERR_INVALID;
  if (k > MAX_K || d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!ok_ptr(home_y) || !ok_ptr(arrive) || !ok_ptr(row_of) || !ok_ptr(topk_gate) || !ok_ptr(out) ||
      !status || (reinterpret_cast<uintptr_t>(status) & 3u))
    return MOE_ERR_INVALID;
  const int nsm = device_sms();
  if (nsm <= 0) return cuda_fail(cudaErrorInvalidDevice);
  const uint64_t tmo = (timeout_us > 0 ? (uint64_t)timeout_us : 2000000ull) * 1000ull;
  return cuda_status(launch_home_combine(static_cast<const __nv_bfloat16*>(home_y), arrive, row_of,
                                         topk_gate, T, d, k, static_cast<__nv_bfloat16*>(out), status,
                                         tmo, nsm, static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_debug_plan(void* ws, int N, int d, int f, int El, int W, void* stream,
                             int32_t* host_out, int max_bands) {
  if (!ws || !aligned16(ws) || !host_out || max_bands < 1) return MOE_ERR_INVALID;
  if (moe_ep_owner_workspace_size(N, d, f, El, W) == 0) return MOE_ERR_INVALID;
  MOE_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  const Layout L = layout(N > 0 ? N : 1, d, f, El * W, 1);
  const int mb = max_bands < max_bands_of(L) ? max_bands : max_bands_of(L);
  MOE_TRY(cudaMemcpy(host_out, static_cast<char*>(ws) + L.band_dest, (size_t)mb * sizeof(int2),
                     cudaMemcpyDeviceToHost));
  return MOE_OK;
}

moe_status moe_debug_band_stamps(void* ws, void* stream, uint64_t* host_out, int max_bands) {
  if (!ws || !aligned16(ws) || !host_out || max_bands < 1) return MOE_ERR_INVALID;
  MOE_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  const Layout L = layout(1, BN2, BN1, 1, 1);
  const int n = max_bands < STAMP_BANDS ? max_bands : STAMP_BANDS;
  MOE_TRY(cudaMemcpy(host_out, static_cast<char*>(ws) + L.stamps + (size_t)STAMP_CTAS * NSTAMP * 8,
                     (size_t)n * 4 * 8, cudaMemcpyDeviceToHost));
  return MOE_OK;
}

moe_status moe_debug_stamps(void* ws, void* stream, uint64_t* host_out, int max_ctas, int* n_ctas) {
  if (!ws || !aligned16(ws) || !host_out || max_ctas < 1) return MOE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY(cudaStreamSynchronize(st));
  const Layout L = layout(1, BN2, BN1, 1, 1);   // the stamps sit at a shape-independent offset
  const int n = max_ctas < STAMP_CTAS ? max_ctas : STAMP_CTAS;
  MOE_TRY(cudaMemcpy(host_out, static_cast<char*>(ws) + L.stamps, (size_t)n * NSTAMP * 8,
                     cudaMemcpyDeviceToHost));
  if (n_ctas) {
    int g = 0;
    for (int i = 0; i < n; ++i) g += host_out[(size_t)i * NSTAMP] != 0;
    *n_ctas = g;
  }
  return MOE_OK;
}

moe_status moe_debug_tokens_combined(const void* ws, int T, int d, int f, int E, int k, void* stream,
                                     int* n_combined) {
  if (!ws || !aligned16(ws) || !n_combined) return MOE_ERR_INVALID;
  moe_status s = check_shape(T, d, f, E, k);
  if (s != MOE_OK) return s;
  MOE_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  const Layout L = layout(T, d, f, E, k);
  std::vector<uint32_t> words((size_t)T);
  MOE_TRY(cudaMemcpy(words.data(), static_cast<const char*>(ws) + L.arrive, (size_t)T * 4,
                     cudaMemcpyDeviceToHost));
  int n = 0;
  for (uint32_t v : words) n += (v & TOKEN_DONE) ? 1 : 0;
  *n_combined = n;
  return MOE_OK;
}

moe_status moe_get_status(void* ws, void* stream, int* consumer_sms, int* n_bands) {
  if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY(cudaStreamSynchronize(st));
  Status h;
  MOE_TRY(cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost));
  if (consumer_sms) *consumer_sms = h.consumer_sms;
  if (n_bands) *n_bands = h.n_bands;
  if (h.code == ST_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (h.code == ST_INVALID) return MOE_ERR_INVALID;
  return h.code == ST_OK ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
