// route.cu -- steps (a) routing and (b) expert-contiguous permutation, plus the
// per-call plan (band table, tile counts, producer/consumer split).
//
// Routing follows "Fine-grained Computation-Communication Overlap via
// Tile-level Signaling and Scheduling for Mixture-of-Experts", Section 2.1
// (top-k experts per token, gate weights); the permutation is that paper's
// Section 3.2.1 row layout on one GPU (rows grouped by expert, no pad rows), and
// the tile order is its Section 3.2.2 schedule rule (ii): experts with more rows
// first, each expert's tiles contiguous.  The split follows "Weave" (arXiv
// 2609.21483), Abstract: once routing is known, a cost model sizes the
// communication (here: combine) and computation worker groups.
#include "kernels.h"

#include <float.h>

namespace moe {

// ------------------------------------------------------------------ route ---
// A warp ranks RT_W tokens in lockstep (their shuffle chains interleave); a block
// of ROUTE_TOK / RT_W warps takes ROUTE_TOK tokens.  Lane l holds logits of
// experts l, l+32, ... (E <= 256).  k rounds of a warp arg-max under the order
// (logit desc, id asc); after round j, lane j keeps slot j's expert and logit.
// Lane j then forms w_j = exp(l_j - l_0) in double, every lane sums the w_j in
// slot order, and lane j writes slot j and adds its expert to the block's
// histogram (blk_hist[b][e], no global atomics: the plan kernel scans the
// per-block counts, so ranks come out deterministic).
constexpr int RT_W = 4;
constexpr int ROUTE_THREADS = ROUTE_TOK / RT_W * 32;

__global__ void __launch_bounds__(ROUTE_THREADS) route_kernel(const float* __restrict__ logits,
                                                              int T, int E, int k,
                                                              int32_t* __restrict__ topk_idx,
                                                              float* __restrict__ topk_gate,
                                                              int32_t* __restrict__ blk_hist,
                                                              uint32_t* __restrict__ arrive,
                                                              uint32_t* __restrict__ ready_q) {
  pdl_trigger();
  pdl_wait();
  __shared__ int hist[MAX_E];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int tb = blockIdx.x * ROUTE_TOK + warp * RT_W;
  const int nv = (E + 31) >> 5;
  float v[RT_W][8];
  uint32_t used[RT_W];
#pragma unroll
  for (int q = 0; q < RT_W; ++q) {
    used[q] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      const bool ok = tb + q < T && i < nv && e < E;
      v[q][i] = ok ? __ldg(logits + (size_t)(tb + q) * E + e) : -FLT_MAX;
      if (!(i < nv && e < E)) used[q] |= 1u << i;
    }
  }
  int my_e[RT_W];
  float my_v[RT_W], vmax[RT_W];
#pragma unroll
  for (int q = 0; q < RT_W; ++q) { my_e[q] = 0; my_v[q] = 0.0f; vmax[q] = 0.0f; }
  for (int j = 0; j < k; ++j) {
    float bv[RT_W];
    int be[RT_W];
#pragma unroll
    for (int q = 0; q < RT_W; ++q) {
      bv[q] = -FLT_MAX;
      be[q] = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (!(used[q] & (1u << i)) && (v[q][i] > bv[q] || (v[q][i] == bv[q] && e < be[q]))) {
          bv[q] = v[q][i];
          be[q] = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int q = 0; q < RT_W; ++q) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv[q], off);
        const int oe = __shfl_xor_sync(0xffffffffu, be[q], off);
        if (ov > bv[q] || (ov == bv[q] && oe < be[q])) { bv[q] = ov; be[q] = oe; }
      }
    }
#pragma unroll
    for (int q = 0; q < RT_W; ++q) {
      if ((be[q] & 31) == lane) used[q] |= 1u << (be[q] >> 5);
      if (lane == j) { my_e[q] = be[q]; my_v[q] = bv[q]; }
      if (j == 0) vmax[q] = bv[q];
    }
  }
  // gates: lane j < k forms w_j = exp(l_j - l_0) in double; the sum runs in slot
  // order; lane j writes slot j
#pragma unroll
  for (int q = 0; q < RT_W; ++q) {
    const int t = tb + q;
    const double wj = lane < k ? exp((double)my_v[q] - (double)vmax[q]) : 0.0;
    double ssum = 0.0;
    for (int j = 0; j < k; ++j) ssum += __shfl_sync(0xffffffffu, wj, j);
    if (t < T) {
      if (lane < k) {
        topk_idx[(size_t)t * k + lane] = my_e[q];
        topk_gate[(size_t)t * k + lane] = (float)(wj / ssum);
        atomicAdd(&hist[my_e[q]], 1);
      }
      if (lane == 0) {
        if (arrive) arrive[t] = 0u;
        if (ready_q) ready_q[t] = 0u;
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) blk_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx,
                         float* topk_gate, int32_t* blk_hist, uint32_t* arrive, uint32_t* ready_q,
                         cudaStream_t s) {
  return launch_pdl(route_kernel, dim3(route_blocks(T)), dim3(ROUTE_THREADS), 0, s, logits, T, E,
                    k, topk_idx, topk_gate, blk_hist, arrive, ready_q);
}

__global__ void colsum_kernel(const int32_t* __restrict__ blk_hist, int nblk, int E,
                              int32_t* __restrict__ counts) {
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  int s = 0;
  for (int b = 0; b < nblk; ++b) s += blk_hist[(size_t)b * E + e];
  counts[e] = s;
}

cudaError_t launch_colsum(const int32_t* blk_hist, int nblk, int E, int32_t* counts, cudaStream_t s) {
  return launch_pdl(colsum_kernel, dim3(cdiv(E, 256)), dim3(256), 0, s, blk_hist, nblk, E, counts);
}

// Per-block expert histogram of given top-k ids (moe_permute's entry, where the
// routing came from the caller rather than route_kernel).  An id outside [0, E)
// is not counted; the plan kernel sees the short total and records ST_INVALID.
__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ topk_idx, int T,
                                                   int E, int k, int32_t* __restrict__ blk_hist) {
  pdl_trigger();
  pdl_wait();
  __shared__ int hist[MAX_E];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const long p0 = (long)blockIdx.x * ROUTE_TOK * k;
  const long p1 = (long)min(T, (int)(blockIdx.x + 1) * ROUTE_TOK) * k;
  for (long p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = topk_idx[p];
    if ((unsigned)e < (unsigned)E) atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) blk_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

cudaError_t launch_hist(const int32_t* topk_idx, int T, int E, int k, int32_t* blk_hist,
                        cudaStream_t s) {
  return launch_pdl(hist_kernel, dim3(route_blocks(T)), dim3(256), 0, s, topk_idx, T, E, k, blk_hist);
}

// ------------------------------------------------------------------- plan ---
// Producer/consumer split (the Weave-style spatial scheduler): choose the number
// C of CTAs (a multiple of cg, the CTAs per tile, from `cmin`) that consume from
// the start instead of running GEMM2, minimising the modelled layer tail
//   t(C) = t2 + max(0, Bc - C * beta * t2) / min(S * beta, beta_hbm),
//   t2   = F2 / ((S - C) * phi)
// F2 = GEMM2 FLOPs (the part the combine can overlap), Bc = combine bytes (every
// routed row read once, every output row written once): C dedicated consumers
// combine during GEMM2, and whatever is left is combined by all S CTAs once the
// GEMM queue is empty (producers join).  Deterministic: same counts, same C.
// The search starts at one CTA group (cmin = cg): paired step-by-step timings on
// B200 of every benchmark layer put C = 0 behind C = 1 on all of them (by 0-5 %),
// and C = 1 within noise of the best fixed C; the model's trade-off then decides
// whether more consumers pay.
// Run by one warp: lane l evaluates candidates C = cmin + (l + 32 i) cg; the pick is
// the smallest C whose modelled time is within a relative 1e-9 of the minimum.
__device__ int choose_consumers(int S, int cg, int cmin, long long R, int T, int d, int f,
                                const CostModel& cm, int lane) {
  const double F2 = 2.0 * (double)R * f * d;
  const double Bc = 2.0 * (double)R * d + 2.0 * (double)T * d;
  const double drain = fmin((double)S * cm.copy_bytes_per_sm, (double)cm.hbm_bytes);
  const int cmax = min(cm.max_consumers, S - cg);
  auto model = [&](int C) {
    const double t2 = F2 / ((double)(S - C) * cm.mma_flops_per_sm);
    const double left = fmax(0.0, Bc - (double)C * cm.copy_bytes_per_sm * t2);
    return t2 + left / drain;
  };
  double my_t = 1e300;
  int my_c = 0x7fffffff;
  for (int C = cmin + lane * cg; C <= cmax; C += 32 * cg) {
    const double t = model(C);
    if (t < my_t) { my_t = t; my_c = C; }
  }
  double tmin = my_t;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) tmin = fmin(tmin, __shfl_xor_sync(0xffffffffu, tmin, off));
  int pick = my_t <= tmin * (1.0 + 1e-9) ? my_c : 0x7fffffff;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) pick = min(pick, __shfl_xor_sync(0xffffffffu, pick, off));
  return pick == 0x7fffffff ? cmin : pick;
}

__host__ __device__ inline int n_items_for(int nb, int mgb) {
  if (mgb <= 1 || nb <= 2) return nb;
  return 2 + cdiv(nb - 2, mgb);
}

// One warp: exclusive scan in place of a[0..n), n <= 256 (8 values per lane);
// returns the total.
__device__ int warp_scan_smem(int* a, int n, int lane) {
  int v[8];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = lane * 8 + i;
    v[i] = idx < n ? a[idx] : 0;
    sum += v[i];
  }
  int inc = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += t;
  }
  int run = inc - sum;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = lane * 8 + i;
    if (idx < n) a[idx] = run;
    run += v[i];
  }
  return __shfl_sync(0xffffffffu, inc, 31);
}

// The tile plan shared by the one-GPU plan and the expert-parallel owner plan.
// U planning units (experts; or an owner's (local expert, source rank) segments)
// in priority order sorted[0..U); unit u has cnt[u] rows from row row0[u],
// computes with expert unit_e[u] (null: u itself) and, for an owner, returns to
// rank dest[u] at home row home0[u] (null on one GPU).  Writes the per-unit
// band/group/GEMM1-tile starts, the status block (`code`, the consumer split, the
// counts) and a zeroed sync block; with w.bands set also the band and group
// tables, the combine plan (w.band_dest) and zeroed band counters.
__device__ void plan_tables(const Work& w, int U, const int* cnt, const int* row0,
                            const int* unit_e, const int* dest, const int* home0,
                            const int* sorted, uint32_t code, long long R, int T, int d, int f,
                            int num_sms, int consumer_hint, int mgb, int G, int cg, int join,
                            const CostModel& cm) {
  const int lag = num_sms;   // GEMM1 tiles between a unit's last one and its GEMM2 block
  (void)join;                // producers join the combine or not: either way the search
                             // starts at one dedicated consumer group
  __shared__ int bstart[MAX_E + 1];
  __shared__ int gstart[MAX_E + 1];
  __shared__ int t1start[MAX_E + 1];
  __shared__ int totals[3];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NT1 = f / BN1, NT2 = d / BN2;
  // bands, groups and GEMM1 tiles of the units in priority order, prefix-summed
  for (int s2 = tid; s2 < U; s2 += blockDim.x) {
    const int bands = cdiv(cnt[sorted[s2]], BM);
    const int groups = cdiv(bands, G);
    bstart[s2] = bands;
    gstart[s2] = groups;
    t1start[s2] = groups * NT1;
  }
  __syncthreads();
  if (warp < 3) {
    int* arr = warp == 0 ? bstart : (warp == 1 ? gstart : t1start);
    const int total = warp_scan_smem(arr, U, lane);
    if (lane == 0) { arr[U] = total; totals[warp] = total; }
  }
  __syncthreads();
  const int nb = totals[0], ng = totals[1], nt1 = totals[2];
  if (w.bands) {
    for (int s2 = tid; s2 <= U; s2 += blockDim.x) {
      w.band_start[s2] = bstart[s2];
      w.group_start[s2] = gstart[s2];
      w.tile_start1[s2] = t1start[s2];
    }
    // The interleaved queue (MOE_SCHED_INTERLEAVE): GEMM1 tiles in their order, with
    // unit s's block of GEMM2 tiles inserted once `lag` more GEMM1 tiles have been
    // handed out after unit s's last one (so its GEMM1 tiles are likely stored by
    // the time its GEMM2 tiles are taken).  Insertion points never decrease, so the
    // blocks keep the priority order; g2_start[s] is block s's queue position.
    if (w.g2_start) {
      for (int s2 = tid; s2 < U; s2 += blockDim.x)
        w.g2_start[s2] = min(t1start[s2 + 1] + lag, nt1) + gstart[s2] * NT2;
      if (tid == 0) w.g2_start[U] = nt1 + ng * NT2;
    }
  }
  // the split: warp 0 evaluates the model for one candidate C per lane
  __shared__ int c_pick;
  if (warp == 0) {
    const int cmin = cg;   // at least one dedicated consumer group (measured: see choose_consumers)
    const int C = consumer_hint != 0 ? consumer_hint : choose_consumers(num_sms, cg, cmin, R, T, d, f, cm, lane);
    if (lane == 0) c_pick = C;
  }
  for (int i = tid; i < (int)(sizeof(Sync) / 4); i += blockDim.x) reinterpret_cast<uint32_t*>(w.sync)[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    const int cmin = cg;
    int C = c_pick;
    if (C < 0) {
      C = 0;                                    // no dedicated consumers (side combine warps)
    } else {
      C = cg * cdiv(C, cg);                     // consumers come in whole CTA groups
      C = max(cmin, min(C, num_sms - cg));      // and leave at least one producer group
    }
    Status st;
    st.code = code;
    st.consumer_sms = C;
    st.n_bands = nb;
    st.n_tiles1 = nt1;
    st.n_tiles2 = ng * NT2;
    st.where = W_NONE;
    st.n_items = n_items_for(nb, mgb);
    st.n_groups = ng;
    *w.status = st;
  }
  if (w.bands == nullptr) return;   // permutation only: no tile plan wanted
  for (int s = tid; s < U; s += blockDim.x) {
    w.sorted_e[s] = sorted[s];
    if (w.expert_rank) w.expert_rank[sorted[s]] = s;
  }
  __syncthreads();
  for (int s = tid; s < U; s += blockDim.x) {
    const int u = sorted[s];
    const int e = unit_e ? unit_e[u] : u;
    const int b0 = bstart[s], nbe = bstart[s + 1] - b0;
    for (int i = 0; i < nbe; ++i) {
      Band bd;
      bd.expert = e;
      bd.row0 = row0[u] + i * BM;
      bd.rows = min(BM, cnt[u] - i * BM);
      bd.pad = 0;
      w.bands[b0 + i] = bd;
      if (w.band_dest && dest) w.band_dest[b0 + i] = make_int2(dest[u], home0[u] + i * BM);
    }
    const int g0 = gstart[s], nge = gstart[s + 1] - g0;
    for (int i = 0; i < nge; ++i) {
      Group gr;
      gr.expert = e;
      gr.band0 = b0 + i * G;
      gr.row0 = row0[u] + i * G * BM;
      gr.rows = min(G * BM, cnt[u] - i * G * BM);
      w.groups[g0 + i] = gr;
    }
  }
  for (int i = tid; i < nb; i += blockDim.x) { w.band_done1[i] = 0u; w.band_done2[i] = 0u; }
  if (w.tok_band) {
    int4* tb = reinterpret_cast<int4*>(w.tok_band);
    for (int i = tid; i < nb * (BM / 4); i += blockDim.x) tb[i] = make_int4(0, 0, 0, 0);
  }
}

__global__ void __launch_bounds__(1024) plan_kernel(Work w, int nblk, const int32_t* offsets_in,
                                                    int T, int d, int f, int E, int k, int num_sms,
                                                    int consumer_hint, int mgb, int G, int cg,
                                                    int join, CostModel cm) {
  pdl_trigger();
  pdl_wait();
  __shared__ int cnt[MAX_E];
  __shared__ int offs[MAX_E + 1];
  __shared__ int sorted[MAX_E];
  __shared__ int part[1024];        // [g][e]: rows' sums of chunk g, then its exclusive base
  __shared__ int bad_in;            // caller-supplied offsets were not a valid scan
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) bad_in = 0;
  __syncthreads();
  // Counts and per-block scatter bases.  Thread (g, e) = (tid / E, tid % E) owns
  // expert e over the contiguous chunk g of route blocks, so a warp's loads and
  // stores cover consecutive experts of the same rows (coalesced).
  const int NG = nblk > 0 ? (int)blockDim.x / E : 0;    // chunks (E <= 256 <= blockDim)
  const int chunk = NG > 0 ? cdiv(nblk, NG) : 0;
  const int g = tid / E, ge = tid - g * E;
  const bool owner = nblk > 0 && g < NG;
  const int cb0 = owner ? min(nblk, g * chunk) : 0, cb1 = owner ? min(nblk, cb0 + chunk) : 0;
  const int32_t* __restrict__ bh = w.blk_hist;
  if (nblk > 0) {
    // 8 independent loads in flight per thread
    int sum = 0, b = cb0;
    for (; b + 8 <= cb1; b += 8) {
      int hv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) hv[u] = bh[(size_t)(b + u) * E + ge];
#pragma unroll
      for (int u = 0; u < 8; ++u) sum += hv[u];
    }
    for (; b < cb1; ++b) sum += bh[(size_t)b * E + ge];
    if (owner) part[tid] = sum;
    __syncthreads();
    // per expert, an exclusive scan over the NG chunks: a warp per expert, each
    // lane a run of cpl chunks (a sum, a shuffle scan of the sums, the prefixes)
    const int nwarps = (int)(blockDim.x >> 5);
    const int cpl = cdiv(NG, 32);
    for (int e = warp; e < E; e += nwarps) {
      const int c0 = lane * cpl, c1 = min(NG, c0 + cpl);
      int sum = 0;
      for (int c = c0; c < c1; ++c) sum += part[c * E + e];
      int inc = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += t;
      }
      int run = inc - sum;
      for (int c = c0; c < c1; ++c) {
        const int v = part[c * E + e];
        part[c * E + e] = run;
        run += v;
      }
      if (lane == 31) cnt[e] = inc;
    }
  } else {
    // caller-supplied offsets (moe_grouped_ffn): they must start at 0, never
    // decrease and end at most at T*k, or no row is planned and ST_INVALID is
    // recorded (no tile would stay inside the row buffers otherwise)
    for (int e = tid; e < E; e += blockDim.x) {
      cnt[e] = offsets_in[e + 1] - offsets_in[e];
      if (cnt[e] < 0) bad_in = 1;
    }
    if (tid == 0 && (offsets_in[0] != 0 || offsets_in[E] > T * k)) bad_in = 1;
    __syncthreads();
    if (bad_in)
      for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  }
  __syncthreads();
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) offs[e] = cnt[e];
    __syncwarp();
    const int total = warp_scan_smem(offs, E, lane);
    if (lane == 0) offs[E] = total;
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) {
    if (e < E) w.counts[e] = cnt[e];
    w.offsets[e] = offs[e];
  }
  if (owner) {
    int32_t* __restrict__ bb = w.blk_base;
    int run = offs[ge] + part[tid];
    int b = cb0;
    for (; b + 8 <= cb1; b += 8) {
      int hv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) hv[u] = bh[(size_t)(b + u) * E + ge];
#pragma unroll
      for (int u = 0; u < 8; ++u) { bb[(size_t)(b + u) * E + ge] = run; run += hv[u]; }
    }
    for (; b < cb1; ++b) {
      const int hcount = bh[(size_t)b * E + ge];
      bb[(size_t)b * E + ge] = run;
      run += hcount;
    }
  }
  // expert priority: rows descending, id ascending (rank by comparison count)
  for (int e = tid; e < E; e += blockDim.x) {
    int r = 0;
    for (int o = 0; o < E; ++o) r += (cnt[o] > cnt[e]) || (cnt[o] == cnt[e] && o < e);
    sorted[r] = e;
  }
  __syncthreads();
  // ids from the caller (nblk > 0 and no route kernel before us) that fell outside
  // [0, E) were not counted: the total comes up short of T*k
  const long long R = offs[E];
  const uint32_t code = (bad_in || (nblk > 0 && R != (long long)T * k)) ? ST_INVALID : ST_OK;
  plan_tables(w, E, cnt, offs, nullptr, nullptr, nullptr, sorted, code, R, T, d, f, num_sms,
              consumer_hint, mgb, G, cg, join, cm);
}

cudaError_t launch_plan(const Work& w, int nblk, const int32_t* offsets_in, int T, int d, int f,
                        int E, int k, int num_sms, int consumer_hint, int mgb, int G, int cg,
                        int join, const CostModel& cm, cudaStream_t s) {
  return launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, s, w, nblk, offsets_in, T, d, f, E, k, num_sms,
                    consumer_hint, mgb, G, cg, join, cm);
}

// ------------------------------------------------------------ owner plan ---
// The expert-parallel owner's plan ("Fine-grained Computation-Communication
// Overlap via Tile-level Signaling and Scheduling for Mixture-of-Experts",
// Section 3.2): the rows it received arrive source rank major, then local expert
// ascending, each source's rows in its own (slot) order, so the rows of local
// expert e from source s are one contiguous run -- a segment.  Planning units are
// the W*El segments:
//  * remote-owner-aligned layout (Section 3.2.1): a segment's rows all return to
//    one rank, and bands never straddle two segments, so every band has a single
//    destination (the paper pads each run to a band boundary with zero rows; here
//    the last band of a run is masked instead, as every expert's last band is);
//  * remote-first schedule (Section 3.2.2): every remote segment before any local
//    one; remote segments by their expert's remote band count, descending (ties:
//    lower expert), an expert's segments together in source order; then the local
//    segments by expert;
//  * combine plan (Section 3.2.3): per band, the home rank and the row in the
//    home's return buffer (its dispatch order) where the band's first row goes.
__global__ void __launch_bounds__(1024) plan_ep_kernel(Work w, const int32_t* __restrict__ recv_counts,
                                                       EpPlanIn in, int d, int f, int num_sms,
                                                       int consumer_hint, int mgb, int G, int cg,
                                                       int join, CostModel cm) {
  pdl_trigger();
  pdl_wait();
  __shared__ int cnt[MAX_E];        // per segment u = e * W + s
  __shared__ int row0[MAX_E];
  __shared__ int unit_e[MAX_E];
  __shared__ int dest[MAX_E];
  __shared__ int home0[MAX_E];
  __shared__ int sorted[MAX_E];
  __shared__ int rbands[MAX_E];     // remote bands per local expert
  __shared__ int bad;
  const int tid = threadIdx.x;
  const int W = in.W, El = in.El, U = W * El;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int u = tid; u < U; u += blockDim.x) {
    const int e = u / W, src = u - e * W;
    const int c = recv_counts[src * El + e];
    if (c < 0) bad = 1;
    cnt[u] = c;
    unit_e[u] = e;
    dest[u] = src;
  }
  __syncthreads();
  if (tid == 0) {
    // segment starts in the received rows (source major, expert ascending) and in
    // the home's return buffer (recv_base[s] + the source's rows of earlier experts)
    long long run = 0;
    for (int src = 0; src < W; ++src) {
      int within = 0;
      for (int e = 0; e < El; ++e) {
        const int u = e * W + src;
        row0[u] = (int)run + within;
        home0[u] = in.recv_base[src] + within;
        within += cnt[u];
      }
      run += within;
    }
    if (run != (long long)in.N) bad = 1;
  }
  __syncthreads();
  if (bad)
    for (int u = tid; u < U; u += blockDim.x) cnt[u] = 0;
  for (int e = tid; e < El; e += blockDim.x) {
    int rb = 0;
    for (int src = 0; src < W; ++src)
      if (src != in.rank) rb += cdiv(cnt[e * W + src], BM);
    rbands[e] = rb;
  }
  __syncthreads();
  // rank of each segment under (local?, remote bands desc, expert asc, source asc)
  for (int u = tid; u < U; u += blockDim.x) {
    const int e = u / W, src = u - e * W;
    const bool loc = src == in.rank;
    int r = 0;
    for (int v = 0; v < U; ++v) {
      const int e2 = v / W, s2 = v - e2 * W;
      const bool loc2 = s2 == in.rank;
      bool before;
      if (loc2 != loc) before = !loc2;                          // remote segments first
      else if (!loc && rbands[e2] != rbands[e]) before = rbands[e2] > rbands[e];
      else if (e2 != e) before = e2 < e;
      else before = s2 < src;
      r += before;
    }
    sorted[r] = u;
  }
  __syncthreads();
  plan_tables(w, U, cnt, row0, unit_e, dest, home0, sorted, bad ? ST_INVALID : ST_OK,
              bad ? 0 : in.N, bad ? 1 : in.N, d, f, num_sms, consumer_hint, mgb, G, cg, join, cm);
}

cudaError_t launch_plan_ep(const Work& w, const int32_t* recv_counts, const EpPlanIn& in, int d,
                           int f, int num_sms, int consumer_hint, int mgb, int G, int cg, int join,
                           const CostModel& cm, cudaStream_t s) {
  return launch_pdl(plan_ep_kernel, dim3(1), dim3(1024), 0, s, w, recv_counts, in, d, f, num_sms,
                    consumer_hint, mgb, G, cg, join, cm);
}

// ---------------------------------------------------------------- scatter ---
// Block b owns the slots of route block b (tokens [b*ROUTE_TOK, (b+1)*ROUTE_TOK))
// and walks them in ascending order, 256 at a time.  Within a warp, __match_any_sync gives
// each slot's rank among earlier lanes with the same expert; per-warp counts in
// shared memory give the rank among earlier warps; a running count per expert
// carries across chunks.  row = (expert's offset + earlier blocks' count, from
// the plan) + rank inside the block -- a stable counting sort.
__global__ void __launch_bounds__(256) scatter_kernel(const int32_t* __restrict__ topk_idx, int T,
                                                      int E, int k, const int32_t* __restrict__ blk_base,
                                                      int32_t* __restrict__ perm,
                                                      int32_t* __restrict__ row_of,
                                                      const int32_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ band_start,
                                                      const int32_t* __restrict__ expert_rank,
                                                      int32_t* __restrict__ tok_band) {
  pdl_trigger();
  pdl_wait();
  __shared__ int running[MAX_E];
  __shared__ int wcnt[8][MAX_E];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += 256) running[e] = 0;
  for (int i = threadIdx.x; i < 8 * MAX_E; i += 256) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const long p0 = (long)blockIdx.x * ROUTE_TOK * k;
  const long p1 = (long)min(T, (int)(blockIdx.x + 1) * ROUTE_TOK) * k;
  const int* base = blk_base + (size_t)blockIdx.x * E;
  const uint32_t lt = (1u << lane) - 1u;
  for (long c = p0; c < p1; c += 256) {
    const long p = c + threadIdx.x;
    const bool in_block = p < p1;
    int e = in_block ? topk_idx[p] : -1;
    // an id outside [0, E) (a caller's bad input) gets no row: row_of = -1
    const bool valid = in_block && (unsigned)e < (unsigned)E;
    if (!valid) e = -1;
    if (in_block && !valid) row_of[p] = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & lt);
    if (valid && rank_w == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (valid) {
      int pre = running[e];
      for (int w2 = 0; w2 < warp; ++w2) pre += wcnt[w2][e];
      const int r = base[e] + pre + rank_w;
      perm[r] = (int32_t)p;
      row_of[p] = r;
      if (tok_band) {
        const int pos = r - offsets[e];
        tok_band[(size_t)(band_start[expert_rank[e]] + pos / BM) * BM + pos % BM] = (int32_t)(p / k);
      }
    }
    __syncthreads();
    for (int e2 = threadIdx.x; e2 < E; e2 += 256) {
      int add = 0;
      for (int w2 = 0; w2 < 8; ++w2) { add += wcnt[w2][e2]; wcnt[w2][e2] = 0; }
      running[e2] += add;
    }
    __syncthreads();
  }
}

cudaError_t launch_scatter(const int32_t* topk_idx, int T, int E, int k, const int32_t* blk_base,
                           int32_t* perm, int32_t* row_of, const Work* plan, cudaStream_t s) {
  const bool tb = plan && plan->tok_band;
  return launch_pdl(scatter_kernel, dim3(route_blocks(T)), dim3(256), 0, s, topk_idx, T, E, k, blk_base,
                    perm, row_of, (const int32_t*)(tb ? plan->offsets : nullptr),
                    (const int32_t*)(tb ? plan->band_start : nullptr),
                    (const int32_t*)(tb ? plan->expert_rank : nullptr), (tb ? plan->tok_band : nullptr));
}

// ----------------------------------------------------------------- gather ---
// x_perm[row_of[t*k + j]] = x[t] for every slot: token-major, so each x row is
// read from memory once and written to its k expert rows (a row-major walk of
// x_perm would re-read x[t] k times, from DRAM once x outgrows L2).  One warp per
// token; 4 x 16-byte vectors per lane in flight, then k stores of each.
__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ x,
                                                     const int32_t* __restrict__ row_of, int T,
                                                     int dv, int k, uint4* __restrict__ x_perm) {
  const unsigned R = (unsigned)T * (unsigned)k;   // rows of x_perm; row_of = -1 marks none
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  constexpr int U = 4;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    const int my_row = lane < k ? row_of[(size_t)t * k + lane] : 0;
    int rows[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    const uint4* src = x + (size_t)t * dv;
    for (int v0 = 0; v0 < dv; v0 += 32 * U) {
      uint4 buf[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < dv) buf[u] = __ldcs(src + v);
      }
#pragma unroll
      for (int j = 0; j < MAX_K; ++j) {
        if (j < k && (unsigned)rows[j] < R) {
          uint4* dst = x_perm + (size_t)rows[j] * dv;
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < dv) dst[v] = buf[u];
          }
        }
      }
    }
  }
}

cudaError_t launch_gather(const __nv_bfloat16* x, const int32_t* row_of, int T, int d, int k,
                          __nv_bfloat16* x_perm, int num_sms, cudaStream_t s) {
  const int grid = max(1, min(cdiv(T, 8), num_sms * 8));
  return launch_pdl(gather_kernel, dim3(grid), dim3(256), 0, s, reinterpret_cast<const uint4*>(x),
                    row_of, T, d / 8, k, reinterpret_cast<uint4*>(x_perm));
}

}  // namespace moe
