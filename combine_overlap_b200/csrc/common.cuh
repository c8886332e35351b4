// common.cuh -- shared constants, workspace layout and sm_100a PTX helpers for
// the MoE layer kernels (libmoe_b200.so).  Everything here is written for
// B200 (sm_100a): TMA tensor copies, mbarriers, tcgen05 MMA with TMEM
// accumulators, and release/acquire flags in global memory.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- tiling ---
constexpr int BM = 128;         // rows per row band (= MMA M, = TMEM lanes)
constexpr int BK = 64;          // K elements per pipeline stage (128 B of bf16; 256-row
                                // single-CTA tiles use 32, see Cfg in ffn.cu)
constexpr int BN1 = 128;        // h columns per GEMM1 tile (accumulates W1 and W3: 256 TMEM cols)
constexpr int BN2 = 256;        // y columns per GEMM2 tile
constexpr int NSTAGE = 4;       // smem pipeline depth
constexpr int ACC_COLS = 256;   // TMEM columns per accumulator; two accumulators
constexpr int TMEM_COLS = 512;
constexpr int A_STAGE_BYTES = BM * BK * 2;          // 16 KiB
constexpr int B_BOX_BYTES = BK * 64 * 2;            // one 64x64 bf16 box, 8 KiB
constexpr int B_STAGE_BYTES = 4 * B_BOX_BYTES;      // 32 KiB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int FFN_THREADS = 320;                    // warp0 TMA, warp1 MMA, warps2-9 epilogue
constexpr int SCHED_DEPTH = 4;

constexpr int ROUTE_TOK = 32;   // tokens per route / scatter block
constexpr int STAMP_CTAS = 256; // debug timestamps: at most this many CTAs ...
constexpr int NSTAMP = 8;       // ... times this many 64-bit words each
constexpr int STAMP_BANDS = 2048;  // debug per-band stamps: at most this many bands x 4 words
constexpr int MAX_E = 256;
constexpr uint32_t TOKEN_DONE = 0x80000000u;   // arrive[t] flag: a consumer combined token t
constexpr int MAX_K = 8;
constexpr int MAX_W = 8;        // ranks of an expert-parallel group

// ----------------------------------------------------------------- status ---
// ST_INVALID: a caller-supplied expert id outside [0, E) (moe_permute); ST_TIMEOUT: a
// bounded device wait ran out.
enum : uint32_t { ST_OK = 0, ST_INVALID = 1, ST_TIMEOUT = 4 };
// where a wait ran out (Status::where)
enum : uint32_t {
  W_NONE = 0, W_SCHED_EMPTY = 1, W_SCHED_FULL = 2, W_STAGE_EMPTY = 3, W_STAGE_FULL = 4,
  W_TMEM_EMPTY = 5, W_TMEM_FULL = 6, W_BAND1 = 7, W_BAND2 = 8, W_DRAIN = 9,
  W_CONS_EMPTY = 10, W_CONS_FULL = 11, W_CONS_QUEUE = 12, W_CONS_IDLE = 13,
  W_SIDE_QUEUE = 14, W_SIDE_IDLE = 15
};

struct Status {
  uint32_t code;
  int32_t consumer_sms;
  int32_t n_bands;
  int32_t n_tiles1;
  int32_t n_tiles2;
  uint32_t where;
  int32_t n_items;
  int32_t n_groups;    // producer tile rows: groups of 1 or 2 consecutive bands of one expert
};

struct Sync {          // zeroed by the plan kernel on every call
  uint32_t q1, q2;      // GEMM1 tiles, GEMM2 tiles taken (MOE_SCHED_INTERLEAVE: q1 counts
                        // the one interleaved queue)
  uint32_t pad0[30];    // the producer queues get a 128-byte line of their own, apart from
                        // the consumers' counters
  uint32_t qc;          // consumer band items taken
  uint32_t rq_alloc;    // ready-token queue: entries allocated
  uint32_t rq_head;     // ready-token queue: entries claimed for combining
  uint32_t prod_done;   // CTAs that have left the producer role
  uint32_t pad1[28];
};
static_assert(sizeof(Sync) == 256, "two 128-byte lines");

struct Band {          // one row band: up to BM rows of one expert
  int32_t expert, row0, rows, pad;
};

// A producer row group: the 1 or 2 consecutive bands of one expert that one MMA
// tile covers (128-row or 256-row tiles).
struct Group {
  int32_t expert, band0, row0, rows;   // rows: valid rows over the whole group
};

// Cost-model constants for the producer/consumer split (per SM throughputs).
struct CostModel {
  float mma_flops_per_sm;   // sustained bf16 dense FLOP/s of one producer SM
  float copy_bytes_per_sm;  // combine bytes/s one consumer SM sustains
  float hbm_bytes;          // device HBM bytes/s ceiling
  int max_consumers;
};

// Device pointers into one workspace buffer (layout from ws_layout on the host).
struct Work {
  int32_t* topk_idx;    // [R]
  float* topk_gate;     // [R]
  int32_t* blk_hist;    // [nblk][E]
  int32_t* blk_base;    // [nblk][E]
  int32_t* counts;      // [E]
  int32_t* offsets;     // [E+1]
  int32_t* perm;        // [R]
  int32_t* row_of;      // [R]
  int32_t* tok_band;    // [max_bands][BM] token of each row of each band (0 past the
                        // band's rows): GEMM1's gather indices, 512 aligned bytes per band
  int32_t* expert_rank; // [E] position of expert e in the priority order
  __nv_bfloat16* x_perm;  // [R][d]
  __nv_bfloat16* h;       // [R][f]
  __nv_bfloat16* y;       // [R][d]
  Band* bands;          // [max_bands]
  int32_t* sorted_e;    // [E]   experts by rows desc, id asc
  int32_t* band_start;  // [E+1] first band of the s-th sorted expert
  int32_t* tile_start1; // [E+1] first GEMM1 tile of the s-th sorted expert
  Group* groups;        // [max_bands] producer row groups in priority order
  int32_t* group_start; // [E+1] first group of the s-th sorted expert
  int32_t* g2_start;    // [E+1] MOE_SCHED_INTERLEAVE: position in the interleaved queue of
                        // the s-th unit's first GEMM2 tile ([E]: the queue's length)
  uint32_t* band_done1; // [max_bands] GEMM1 tiles finished per band
  uint32_t* band_done2; // [max_bands] GEMM2 tiles finished per band
  uint32_t* arrive;     // [T] rows of token t that have arrived; TOKEN_DONE set once out[t]
                        // is written by a consumer
  uint32_t* ready_q;    // [T] tokens whose k rows all arrived (t + 1; 0 = entry not yet written)
  int2* band_dest;      // [max_bands] expert-parallel owner: (home rank, home row of the band's
                        // first row) -- the combine plan; null on one GPU
  Sync* sync;
  Status* status;
  unsigned long long* stamps;  // [STAMP_CTAS][NSTAMP] debug timestamps (MOE_DBG_TIMESTAMPS),
                               // then [STAMP_BANDS][4] per consumed band
};

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline int max_bands(int R, int E) { return R / BM + E; }
__host__ __device__ inline int route_blocks(int T) { return cdiv(T, ROUTE_TOK); }

// --------------------------------------------------- programmatic launch ---
// Every kernel of a layer call lets the next one launch as soon as all of its
// own blocks are running (launch_dependents), and waits for the previous grid
// to complete and flush (wait) before touching any of its outputs, so only the
// launch latency between kernels is hidden, never a data dependence.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------ PTX helpers ---
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// An L2 cache policy that marks the lines a store writes as first to evict.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte global store with an L2 cache policy.
__device__ __forceinline__ void st_global_v4_policy(void* ptr, uint4 v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;"
               :: "l"(ptr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy) : "memory");
}

// System-scope release add and acquire load: arrival words that another GPU's
// kernel (or, on one GPU, another rank's kernel) writes or reads over NVLink.
__device__ __forceinline__ void red_release_sys_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.sys.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// mbarrier -------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
               :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase completed, false when `deadline` (globaltimer
// ns) passed or `abort` became non-zero first.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline,
                                          const volatile uint32_t* abort) {
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++n & 1023u) == 0) {
      if (globaltimer() > deadline || *abort) return false;
    }
  }
  return true;
}

// TMA ------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Untiled bulk copy global -> shared (no multicast): `bytes` (multiple of 16),
// both addresses 16-byte aligned; completes `bytes` of transaction on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Four rows (coordinates y0..y3) of a 2-D tensor, 64 columns from x, into 4
// consecutive 128-byte smem rows (the tensor map's box is one row high).
__device__ __forceinline__ void tma_gather4(void* dst, const void* tmap, uint64_t* bar, int x,
                                           int y0, int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

// 16-byte copy global -> shared through L2 only (the load/store path, generic proxy).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Arrive on `bar` once all of this thread's earlier cp.async copies have completed
// (the arrival is not counted up front: the barrier's count includes it).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// tcgen05 --------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
               :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive once on `bar` when all prior tcgen05.mma of this thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Clusters (CTA pairs) ---------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory offset in CTA `cta` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(cta));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t cluster_addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};"
               :: "r"(cluster_addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA load whose completion is counted on the pair leader's mbarrier (`bar_cluster`
// is a shared::cluster address, possibly in the other CTA).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* tmap, uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(bar_cluster), "r"(c0), "r"(c1) : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const void* tmap, uint32_t bar_cluster,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

__device__ __forceinline__ void tma_gather4_pair(void* dst, const void* tmap, uint32_t bar_cluster,
                                                int x, int y0, int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      :: "r"(smem_u32(dst)), "l"(tmap), "r"(bar_cluster), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A * B over a CTA pair (M = 256: 128 rows of A and half of B's N
// from each CTA's shared memory, same offsets); issued by the pair's leader.
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
               :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive once on `bar` (same offset) in every CTA of `mask` when this thread's
// prior pair MMAs have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               :: "r"(smem_u32(bar)), "h"(mask) : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format, version 1), 128-byte swizzle.
//   K-major tile (rows of 128 B, 8-row atoms 1024 B apart): lbo unused, sbo = 1024.
//   MN-major tile (64-element MN atoms `lbo` bytes apart, 8-row K groups
//   `sbo` bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                 // descriptor version for tcgen05
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

// The same with 64-byte swizzle: a K-major tile of 64-byte rows (32 bf16 of K),
// 8-row atoms `sbo` = 512 bytes apart; lbo unused.
__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                 // descriptor version for tcgen05
  d |= (uint64_t)4 << 61;                 // SWIZZLE_64B
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4)                        // D format: f32
       | (1u << 7)                        // A format: bf16
       | (1u << 10)                       // B format: bf16
       | ((b_mn_major ? 1u : 0u) << 16)   // B major-ness
       | ((uint32_t)(N >> 3) << 17)
       | ((uint32_t)(M >> 4) << 24);
}

}  // namespace moe
