// ffn.cu -- steps (c1), (c2), (d), (e): the persistent grouped SwiGLU expert
// FFN on tcgen05 tensor cores, its per-row-band ready signals, and the consumer
// role that combines each row band as soon as it is ready.
//
// Design source: "Fine-grained Computation-Communication Overlap via Tile-level
// Signaling and Scheduling for Mixture-of-Experts" (arXiv 2607.19539):
//   Section 3.3.1 -- one persistent kernel covers every expert's tiles; each
//     work item pairs an expert with a tile coordinate; the epilogue stores the
//     tile, fences, then publishes a ready signal.
//   Section 3.3.2 -- the consumer's unit of work is a row band (BM rows by the
//     full output width), optionally x (= mgb) bands per item, first and last
//     items one band each.
//   Section 3.3.3 -- producer and consumer own disjoint SMs.
//   Section 3.2.2 -- tile order: experts with more rows first, each expert's
//     tiles contiguous; all tiles of a band before the next band (GEMM2).
// and "Weave" (arXiv 2609.21483), Abstract: the split is chosen per call from
// the routing counts, and worker groups are coordinated so SMs do not idle --
// here consumer CTAs help with GEMM1 first, and producer CTAs join the combine
// once the GEMM tile queue is empty.
//
// B200 mapping (differs from the paper's A100 CUTLASS/NVSHMEM kernels):
//   * one launch of one CTA per SM (V = 1, 3: a cooperative launch; V = 2: a
//     cluster launch of as many pairs as can be resident at once), each CTA
//     taking tiles from an atomic work queue in priority order instead of a
//     fixed stride;
//   * per CTA: warp 0 = tile scheduler + TMA producer, warp 1 = TMEM allocator
//     + single-thread tcgen05.mma issuer, warps 2-9 = epilogue (TMEM -> registers
//     -> bf16 -> global, two warps per TMEM lane quadrant), a 192 KB smem operand
//     ring and two 256-column TMEM accumulators;
//   * three tile variants V, chosen per call by the host: V = 1, one CTA per
//     128-row tile; V = 2, a cluster pair per 256-row tile with tcgen05
//     cta_group::2 -- the leader issues the MMAs, each CTA loads its 128 rows of
//     A and half of B (no multicast), work items are mirrored into the peer over
//     DSMEM, and an expert's odd last band runs as an M=128 half tile; V = 3, one
//     CTA per 256-row tile as two 128-row MMAs per K step into its two
//     accumulators.  V = 1 and 2 alternate the accumulators between tiles, so the
//     epilogue of one tile overlaps the main loop of the next; single CTAs read
//     their weight tiles with one 4-D TMA copy per operand;
//   * GEMM1 tile: 128 or 256 rows x 128 h-columns; one N=256 MMA accumulates
//     x*W1 and x*W3 side by side (the B tile holds the W1 and W3 column blocks),
//     and the epilogue applies silu(a)*b;  GEMM2 tile: 128 or 256 rows x 256
//     y-columns;
//   * A (x_perm or h) is K-major, W is stored [K][N] (N-major): both are read
//     by TMA with 128-byte swizzle and fed to tcgen05 as K-major / MN-major
//     operands, so the weights need no repacking;
//   * signals are counters per row band (GEMM1 tiles done, GEMM2 tiles done,
//     2 per tile) published with red.release and polled with ld.acquire; every
//     wait is bounded and reports MOE_ERR_TIMEOUT through the status block.
#include "kernels.h"
#include "combine.cuh"
#include "../../include/moe.h"

#include <cuda.h>
#include <stddef.h>

namespace moe {

enum : int { K_END = 0, K_G1 = 1, K_G2 = 2 };

constexpr int CONS_SLOTS = 16;    // at most this many tokens in flight per consumer CTA
constexpr int MAX_NST = 6;        // pipeline depth of the CTA-pair variant
constexpr int STAGE_AREA = 196608;  // shared memory of the operand ring (and the consumer's slots)

// Tile variants, V:
//   V = 1  one CTA per 128x256 tile (A: 128 rows, B: all 256 columns);
//   V = 2  a CTA pair per 256x256 tile with tcgen05 cta_group::2 (each CTA: 128
//          rows of A and 128 columns of B);
//   V = 3  one CTA per 256x256 tile, as two 128-row MMAs (two A boxes, one B
//          stage) into its two accumulators.
// V = 2 and V = 3 stream 32 KB of operands per 128x256x64 of MMA work, V = 1 48 KB.
// A stage holds BK = 64 elements of K: A rows of 128 bytes in the 128-byte swizzle.
// (The roles also take BK = 32 -- 64-byte A rows in the 64-byte swizzle -- which
// gives V = 3 six stages of 32 KB instead of three of 64 KB.  Measured on B200 it
// was 10-12 % slower on every V = 3 layer, and a V = 3 ring of two 64 KB stages
// 16-22 % slower than three, so three stages of 64 KB it is.)
template <int V>
struct Cfg {
  static_assert(V >= 1 && V <= 3, "tile variant");
  static constexpr int CTAS = V == 2 ? 2 : 1;                      // CTAs per tile
  static constexpr int BANDS = V == 1 ? 1 : 2;                     // row bands per tile
  static constexpr int ABOX = V == 3 ? 2 : 1;                      // 128-row A boxes per CTA
  static constexpr int NBOX = V == 2 ? 2 : 4;                      // 64-column B boxes per CTA
  static constexpr int BK = 64;                                    // K elements per stage
  static constexpr int A_ROW = BK * 2;                             // bytes of an A row (swizzle span)
  static constexpr int A_BYTES = BM * A_ROW;                       // one 128-row A box
  static constexpr int B_BOX = BK * 64 * 2;                        // one 64-column B atom
  static constexpr int STAGE = ABOX * A_BYTES + NBOX * B_BOX;
  static constexpr int NST = STAGE_AREA / STAGE;
  static_assert(NST <= MAX_NST && NST * STAGE == STAGE_AREA, "stage ring must fill the area");
  static_assert(BK % 16 == 0 && (A_ROW == 64 || A_ROW == 128), "A rows of one swizzle span");
};

// 16-byte aligned: the pair leader copies items into its peer's ring with 16-byte
// distributed-shared-memory stores.
struct __align__(16) Item {
  int kind, group, nt, expert, row0, rows, band0, pad;   // rows: valid rows of the whole group
};

constexpr int EPI_WARPS = FFN_THREADS / 32 - 2;   // warps 2.. : two per TMEM lane quadrant
constexpr int OSTAGE_ROW = 80;                    // staged bytes per row: 64 of data + 16 of pad

constexpr int SIDE_RING = 64;   // completed bands a CTA's side warps may have pending
constexpr int SIDE_TOK = 2;     // ready tokens a side warp claims at a time

struct SmemCtl {
  uint64_t full[MAX_NST];        // operands of a stage landed (pair: counted on the leader)
  uint64_t empty[MAX_NST];       // the MMAs reading a stage finished
  uint64_t tfull[2];             // accumulator ready for the epilogue
  uint64_t tempty[2];            // accumulator drained by every epilogue warp (pair: on the leader)
  uint64_t sfull[SCHED_DEPTH];   // a work item is in the ring slot
  uint64_t sempty[SCHED_DEPTH];  // every role read the slot (pair: on the leader)
  uint64_t epi_done[2];          // per accumulator: this CTA's epilogue warps stored the tile
  uint64_t mma_done;
  uint64_t cfull[CONS_SLOTS];    // consumer ring: a token's k expert rows landed in the slot
  uint64_t cempty[CONS_SLOTS];   // consumer ring: the slot's token is reduced and stored
  uint64_t gbar[2];              // a GEMM1 tile's gather indices landed (two items in flight)
  Item ring[SCHED_DEPTH];
  int4 gidx[2][2 * BM / 4];      // token of each row of a GEMM1 tile (up to 256 rows)
  uint32_t tmem_base;
  int item;
  int ok;
  int cn;                        // tokens completed by the current band
  int ctok[BM];                  // ... and which,
  int crow[BM][MAX_K];           // ... their k expert rows
  float cgate[BM][MAX_K];        // ... and their k gates (staged once, read by every warp)
  // side combine warps: bands this CTA completed, waiting for their arrivals (one
  // writer, the publishing thread; the side warps claim entries with a CAS on bhead)
  int bring[SIDE_RING];
  int bhead, btail;
  int prod_left;                 // producer warps (TMA, MMA, epilogue) still in their roles
  // epilogue: per warp, 32 rows x 32 bf16 columns on their way to global memory
  alignas(16) uint8_t ostage[EPI_WARPS][32 * OSTAGE_ROW];
};

static_assert(offsetof(SmemCtl, ring) % 16 == 0, "ring items must be 16-byte aligned");
static_assert(sizeof(Item) == 32, "an item is two 16-byte stores");

size_t ffn_smem_bytes() { return 1024 + (size_t)STAGE_AREA + sizeof(SmemCtl); }
static_assert(1024 + STAGE_AREA + sizeof(SmemCtl) <= 227 * 1024, "over the 227 KB per-CTA limit");

// Weight-tile bytes of one stage of variant V (the whole B share of a CTA).
template <int V>
__device__ __forceinline__ constexpr int NBOX_BYTES() { return Cfg<V>::NBOX * Cfg<V>::B_BOX; }

__device__ __forceinline__ void set_error(Status* st, uint32_t where) {
  if (atomicCAS(&st->code, (uint32_t)ST_OK, (uint32_t)ST_TIMEOUT) == (uint32_t)ST_OK) {
    st->where = where;
  }
}

// Bounded mbarrier wait (acquire at cluster scope when `cluster`, for phases that
// the other CTA of a pair completes); `abort` (may be null) ends it early once
// any CTA has recorded an error.
template <bool cluster = false>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                         const volatile uint32_t* abort) {
  auto test = [&]() { return cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (test()) return true;
  const uint64_t deadline = globaltimer() + timeout_ns;
  uint32_t n = 0;
  while (!test()) {
    if ((++n & 255u) == 0u) {
      if (globaltimer() > deadline) return false;
      if (abort && *abort) return false;
    }
  }
  return true;
}

// Bounded poll of a release-published counter.
__device__ __forceinline__ bool wait_count(const uint32_t* p, uint32_t target, uint64_t timeout_ns,
                                           const volatile uint32_t* abort) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t deadline = globaltimer() + timeout_ns;
  uint32_t ns = 32;
  while (ld_acquire(p) < target) {
    if (globaltimer() > deadline || *abort) return false;
    __nanosleep(ns);
    if (ns < 1024) ns <<= 1;
  }
  return true;
}

__device__ __forceinline__ Item make_item(int kind, int group, int nt, const Group& gr) {
  Item it;
  it.kind = kind;
  it.group = group;
  it.nt = nt;
  it.expert = gr.expert;
  it.row0 = gr.row0;
  it.rows = gr.rows;
  it.band0 = gr.band0;
  it.pad = 0;
  return it;
}

// GEMM1 tile t: experts in priority order; inside an expert, column-block major
// (every row group of one 128-column block of W1/W3, then the next), so the
// weight slice in use stays in L2 while every group of the expert reads it.
__device__ Item decode_g1(const Work& w, int t, int E) {
  int lo = 0, hi = E;  // tile_start1[lo] <= t < tile_start1[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (w.tile_start1[mid] <= t) lo = mid; else hi = mid;
  }
  const int g0 = w.group_start[lo];
  const int nge = w.group_start[lo + 1] - g0;
  const int local = t - w.tile_start1[lo];
  const int group = g0 + local % nge;
  return make_item(K_G1, group, local / nge, w.groups[group]);
}

// GEMM2 tile t: group-major (all column blocks of a row group, then the next), so
// row bands complete -- and can be combined -- in priority order.
__device__ Item decode_g2(const Work& w, int t, int NT2) {
  const int group = t / NT2;
  return make_item(K_G2, group, t % NT2, w.groups[group]);
}

// Position t of the interleaved queue (MOE_SCHED_INTERLEAVE): unit s's GEMM2 block
// occupies [g2_start[s], g2_start[s] + its GEMM2 tiles); every other position is
// the next GEMM1 tile.  Blocks do not overlap and their starts never decrease.
__device__ Item decode_mixed(const Work& w, int t, int U, int NT2) {
  int lo = -1, hi = U;   // the last block with g2_start <= t is lo (-1: none)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (w.g2_start[mid] <= t) lo = mid; else hi = mid;
  }
  int g2_before = 0;     // GEMM2 tiles at positions before t
  if (lo >= 0) {
    const int n2b = (w.group_start[lo + 1] - w.group_start[lo]) * NT2;
    const int off = t - w.g2_start[lo];
    if (off < n2b) return decode_g2(w, w.group_start[lo] * NT2 + off, NT2);
    g2_before = w.group_start[lo + 1] * NT2;
  }
  return decode_g1(w, t - g2_before, U);
}

__device__ __forceinline__ void item_range(int item, int nb, int mgb, int& b0, int& b1) {
  if (mgb <= 1 || nb <= 2) { b0 = item; b1 = item + 1; return; }
  const int nmid = cdiv(nb - 2, mgb);
  if (item == 0) { b0 = 0; b1 = 1; }
  else if (item <= nmid) { b0 = 1 + (item - 1) * mgb; b1 = min(b0 + mgb, nb - 1); }
  else { b0 = nb - 1; b1 = nb; }
}

__device__ __forceinline__ float silu_mul(float a, float b) {
  return __fdividef(a, 1.0f + __expf(-a)) * b;
}

// silu(a) * b through one special-function op: silu(a) = a * sigmoid(a) and
// sigmoid(a) = (1 + tanh(a / 2)) / 2, with the hardware tanh approximation
// (tanh.approx.f32, relative error about 2^-11).  The GEMM1 epilogue runs two
// special-function ops per h element with the exp form (silu_mul above) and is
// bound by them; measured on B200 the tanh form makes the layer 1-2.6 % faster.
// Its error is below the bf16 rounding of h except for a below about -4, where
// 1 + tanh(a/2) cancels and silu(a) -- already under 0.08 in size -- carries an
// absolute error of a few 1e-4 times |a|; MOE_SCHED_EXP_SILU keeps the exp form.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_mul_tanh(float a, float b) {
  const float ha = 0.5f * a;
  return fmaf(ha, tanh_approx(ha), ha) * b;
}

// A CTA pair's row group of one band only (an expert's last, odd band) runs as
// a half tile: an M=128 cta_group::2 MMA, each CTA supplying 64 rows of A, at
// half the tensor time of the M=256 tile whose second band would be all masked.
// Its accumulator holds, in each CTA, 64 rows x N/2 columns twice: TMEM lanes
// 0-63 the columns that the leader's B half supplies, lanes 64-127 (the same 64
// rows) the peer's.  (The gathered-A path keeps full tiles, as does
// MOE_SCHED_FULL_TILES.)
template <int V>
__device__ __forceinline__ bool half_tile(const Item& it, const FfnArgs& a) {
  return V == 2 && !a.gather && !(a.flags & MOE_SCHED_FULL_TILES) && it.rows <= BM;
}

// This CTA's rows of a row group: CTA `rank` of a pair owns band band0+rank (in
// a half tile, rows 64*rank.. of band0); a single CTA owns the whole group (V = 3:
// up to two bands, band0 and band0+1).
struct MyRows {
  int row0, rows, band;
};

template <int V>
__device__ __forceinline__ MyRows my_rows(const Item& it, uint32_t rank, bool half) {
  MyRows m;
  if (V == 3) {
    m.row0 = it.row0;
    m.rows = min(2 * BM, it.rows);
    m.band = it.band0;
    return m;
  }
  const int h = half ? BM / 2 : BM;
  m.row0 = it.row0 + (int)rank * h;
  m.rows = min(h, max(0, it.rows - (int)rank * h));
  m.band = it.band0 + (half ? 0 : (int)rank);
  return m;
}

// Band counters: each tile adds 2 to its band's counter (1 from each CTA of a
// half tile), so a band is complete at twice its tile count.
constexpr uint32_t BAND_UNIT = 2;

// Arrive on a barrier that lives in the pair leader (local when this CTA leads).
template <int V>
__device__ __forceinline__ void arrive_leader(uint64_t* bar, uint32_t rank) {
  if (V != 2 || rank == 0) mbar_arrive(bar);
  else mbar_arrive_remote(mapa_shared(smem_u32(bar), 0));
}

// ---------------------------------------------------------------- scheduler ---
// The work-item scheduler of a CTA (a single CTA, or a pair's leader): takes the
// next item from the atomic queues and publishes it in the item ring (the leader
// also writes it into its peer's ring over distributed shared memory); a pair's
// peer reads it from its own ring.  One thread runs it.
struct Sched {
  int slot;
  uint32_t sph;
  bool g1, g2;
  bool interleave;
  unsigned long long* stamp;   // per-CTA debug stamps, or null
};

template <int V>
__device__ bool sched_next(Sched& sc, Item& it, const FfnArgs& a, SmemCtl* ctl, uint32_t rank,
                           int n1, int n2, const volatile uint32_t* abort) {
  const Work& w = a.w;
  const int NT2 = a.d / BN2;
  const uint64_t tmo = a.timeout_ns;
  const bool leader = V != 2 || rank == 0;
  if (leader) {
    it.kind = K_END;
    if (*abort) sc.g1 = sc.g2 = false;
    if (sc.interleave && sc.g1) {
      const int t = (int)atomicAdd(&w.sync->q1, 1u);
      if (t < n1 + n2) it = decode_mixed(w, t, a.n_units, NT2);
      else {
        sc.g1 = sc.g2 = false;
        if (sc.stamp) sc.stamp[1] = globaltimer();
      }
    }
    if (!sc.interleave && it.kind == K_END && sc.g1) {
      const int t = (int)atomicAdd(&w.sync->q1, 1u);
      if (t < n1) it = decode_g1(w, t, a.n_units);
      else {
        sc.g1 = false;
        if (sc.stamp) sc.stamp[1] = globaltimer();
      }
    }
    if (!sc.interleave && it.kind == K_END && sc.g2) {
      const int t = (int)atomicAdd(&w.sync->q2, 1u);
      if (t < n2) it = decode_g2(w, t, NT2); else sc.g2 = false;
    }
    if (!wait_bar<V == 2>(&ctl->sempty[sc.slot], sc.sph ^ 1u, tmo, abort)) { set_error(w.status, W_SCHED_EMPTY); return false; }
    ctl->ring[sc.slot] = it;
    if (V == 2) {
      const uint4* src = reinterpret_cast<const uint4*>(&it);
      const uint32_t dst = mapa_shared(smem_u32(&ctl->ring[sc.slot]), 1);
      st_cluster_v4(dst, src[0]);
      st_cluster_v4(dst + 16, src[1]);
      mbar_arrive_remote(mapa_shared(smem_u32(&ctl->sfull[sc.slot]), 1));
    }
    mbar_arrive(&ctl->sfull[sc.slot]);
  } else {
    if (!wait_bar<true>(&ctl->sfull[sc.slot], sc.sph, tmo, abort)) { set_error(w.status, W_SCHED_FULL); return false; }
    it = ctl->ring[sc.slot];
    arrive_leader<V>(&ctl->sempty[sc.slot], rank);
  }
  if (++sc.slot == SCHED_DEPTH) { sc.slot = 0; sc.sph ^= 1u; }
  return true;
}

// ------------------------------------------------------------ TMA producer ---
// A single CTA, or the pair leader: takes work items from the atomic queues and puts
// them in the ring (the leader also writes them into its peer's ring over
// distributed shared memory).  The peer reads items from its own ring.  Each CTA
// then loads its own 128 rows of A and its share of B for every k-block; in a
// pair the loads count on the leader's `full` barrier.
// V = 3 loads two 128-row A boxes (one when the group holds a single band).
// GEMM1's A rows are gathered straight from x (a.gather, V = 1 and 2): the
// tile's 128 token indices (one aligned 512-byte row of tok_band) are
// bulk-copied into shared memory one work item ahead, and each k-block's A tile
// is 32 TMA gather4 loads of 4 token rows x 64 columns into the same swizzled
// layout a tiled load gives.
template <int V>
__device__ void role_tma(const CUtensorMap* tm_a1, const CUtensorMap* tm_w1,
                         const CUtensorMap* tm_w3, const CUtensorMap* tm_a2,
                         const CUtensorMap* tm_w2, const FfnArgs& a, SmemCtl* ctl,
                         uint8_t* smem, uint32_t rank, bool run_g1, bool run_g2, int n1, int n2,
                         const volatile uint32_t* abort) {
  using C = Cfg<V>;
  const Work& w = a.w;
  const int NT1 = a.f / BN1;
  const uint64_t tmo = a.timeout_ns;
  const bool leader = V != 2 || rank == 0;
  int stage = 0;
  uint32_t ph = 0;
  uint32_t pending = 0, pend_par = 0;   // stages with an issued fill, and its parity
  uint32_t gph = 0;                     // parity of the next wait on gbar[0], gbar[1]
  uint32_t gpend = 0;                   // index copies issued and not yet waited, per buffer
  bool g1 = run_g1, g2 = run_g2;
  bool ok = true;
  const bool stamp = (a.flags & MOE_DBG_TIMESTAMPS) && blockIdx.x < STAMP_CTAS;
  unsigned long long* my_stamps = w.stamps + (size_t)blockIdx.x * NSTAMP;
  unsigned long long n_g1 = 0, n_g2 = 0;

  // With MOE_SCHED_INTERLEAVE (and both GEMMs in this launch) one queue hands out
  // GEMM1 and GEMM2 tiles interleaved, in the order the plan fixed (decode_mixed):
  // a GEMM2 tile comes a grid's worth of GEMM1 tiles after the last GEMM1 tile of
  // its unit, so every GEMM1 tile it waits on sits earlier in the queue and was
  // taken by a resident CTA (no deadlock), and is most likely stored already.
  Sched sc{0, 0u, g1, g2, (a.flags & MOE_SCHED_INTERLEAVE) && g1 && g2, stamp ? my_stamps : nullptr};
  auto next_item = [&](Item& it) -> bool { return sched_next<V>(sc, it, a, ctl, rank, n1, n2, abort); };
  // Does this CTA gather indices for the item?  (GEMM1, gathered path, own rows)
  auto gathers = [&](const Item& it) {
    return a.gather == 1 && it.kind == K_G1 && my_rows<V>(it, rank, false).rows > 0;
  };
  auto fetch_indices = [&](const Item& it, int buf) {
    if (!gathers(it)) return;
    const MyRows m = my_rows<V>(it, rank, false);
    fence_proxy_async_shared();   // earlier generic reads of this buffer come first
    gpend |= 1u << buf;
    mbar_arrive_expect_tx(&ctl->gbar[buf], BM * 4);
    bulk_load(&ctl->gidx[buf][0], a.tok_band + (size_t)m.band * BM, BM * 4, &ctl->gbar[buf]);
  };

  Item cur;
  int buf = 0;
  if (!next_item(cur)) ok = false;
  else fetch_indices(cur, buf);
  while (ok && cur.kind != K_END) {
    Item nxt;
    if (!next_item(nxt)) break;
    fetch_indices(nxt, buf ^ 1);
    const bool is1 = cur.kind == K_G1;
    if (is1) ++n_g1; else ++n_g2;
    const bool half = half_tile<V>(cur, a);
    const MyRows m = my_rows<V>(cur, rank, half);
    const bool two = V == 3 && m.rows > BM;   // V = 3: the group's second band is present
    const bool gat = a.gather == 1 && is1;
    if (gat && m.rows > 0) {
      if (!wait_bar(&ctl->gbar[buf], (gph >> buf) & 1u, tmo, abort)) { set_error(w.status, W_STAGE_FULL); break; }
      gph ^= 1u << buf;
      gpend &= ~(1u << buf);
    }
    if (!is1 && m.rows > 0) {
      // GEMM2 reads this CTA's h rows: every GEMM1 column block of its band must be stored.
      if (!wait_count(&w.band_done1[m.band], BAND_UNIT * (uint32_t)NT1, tmo, abort) ||
          (two && !wait_count(&w.band_done1[m.band + 1], BAND_UNIT * (uint32_t)NT1, tmo, abort))) {
        set_error(w.status, W_BAND1);
        break;
      }
      fence_proxy_async_global();  // generic-proxy stores -> async-proxy (TMA) loads
    }
    const int nk = (is1 ? a.d : a.f) / C::BK;
    for (int kb = 0; kb < nk; ++kb) {
      if (!wait_bar<V == 2>(&ctl->empty[stage], ph ^ 1u, tmo, abort)) { set_error(w.status, W_STAGE_EMPTY); ok = false; break; }
      uint8_t* sa = smem + (size_t)stage * C::STAGE;
      uint8_t* sb = sa + C::ABOX * C::A_BYTES;
      uint64_t* fb = &ctl->full[stage];
      const uint32_t fbl = V == 2 ? mapa_shared(smem_u32(fb), 0) : 0u;
      // a pair's leader expects both CTAs' bytes; V = 3 without a second band
      // loads one A box; GEMM1 A rows copied by the gather warps are not TMA bytes
      const bool lsu = is1 && a.gather == 2;
      if (leader)
        mbar_arrive_expect_tx(fb, lsu ? NBOX_BYTES<V>() :
                                  C::CTAS * C::STAGE - (V == 3 && !two ? C::A_BYTES : 0));
      // A: 128 rows x 64 columns of x_perm (tiled) or of x (gathered); h for GEMM2
      if (lsu) {
        // (the gather warps copy these A rows)
      } else if (gat) {
#pragma unroll 8
        for (int q = 0; q < BM / 4; ++q) {
          const int4 tk = m.rows > 0 ? ctl->gidx[buf][q] : make_int4(0, 0, 0, 0);
          if (V != 2) tma_gather4(sa + q * 4 * C::A_ROW, tm_a1, fb, kb * C::BK, tk.x, tk.y, tk.z, tk.w);
          else tma_gather4_pair(sa + q * 4 * C::A_ROW, tm_a1, fbl, kb * C::BK, tk.x, tk.y, tk.z, tk.w);
        }
      } else if (V != 2) {
        tma_load_2d(sa, is1 ? tm_a1 : tm_a2, fb, kb * C::BK, m.row0);
        if (two) tma_load_2d(sa + C::A_BYTES, is1 ? tm_a1 : tm_a2, fb, kb * C::BK, m.row0 + BM);
      } else {
        tma_load_2d_pair(sa, is1 ? tm_a1 : tm_a2, fbl, kb * C::BK, m.row0);
      }
      // B: 64-column atoms of W1/W3 (GEMM1) or W2 (GEMM2), K-rows kb*C::BK.., each
      // atom BK K rows x 128 B, atom after atom (the MMA's leading-byte offset)
      if (V != 2 && a.b_atoms) {
        // 4-D maps {64 columns, K, atom, expert}: one copy per operand
        const int k0 = kb * C::BK;
        if (is1) {
          tma_load_4d(sb, tm_w1, fb, 0, k0, cur.nt * (BN1 / 64), cur.expert);
          tma_load_4d(sb + 2 * C::B_BOX, tm_w3, fb, 0, k0, cur.nt * (BN1 / 64), cur.expert);
        } else {
          tma_load_4d(sb, tm_w2, fb, 0, k0, cur.nt * (BN2 / 64), cur.expert);
        }
      } else if (V != 2) {
        if (is1) {
          tma_load_3d(sb, tm_w1, fb, cur.nt * BN1, kb * C::BK, cur.expert);
          tma_load_3d(sb + C::B_BOX, tm_w1, fb, cur.nt * BN1 + 64, kb * C::BK, cur.expert);
          tma_load_3d(sb + 2 * C::B_BOX, tm_w3, fb, cur.nt * BN1, kb * C::BK, cur.expert);
          tma_load_3d(sb + 3 * C::B_BOX, tm_w3, fb, cur.nt * BN1 + 64, kb * C::BK, cur.expert);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tma_load_3d(sb + q * C::B_BOX, tm_w2, fb, cur.nt * BN2 + q * 64, kb * C::BK, cur.expert);
        }
      } else {
        if (is1 && half) {
          // half tile: each CTA's B half is [W1 | W3] of one 64-column atom (the
          // leader's the first, the peer's the second), so every accumulator
          // lane holds matching W1 and W3 columns
          const int n0 = cur.nt * BN1 + (int)rank * 64;
          tma_load_3d_pair(sb, tm_w1, fbl, n0, kb * C::BK, cur.expert);
          tma_load_3d_pair(sb + C::B_BOX, tm_w3, fbl, n0, kb * C::BK, cur.expert);
        } else if (is1) {
          // B columns [0,128) of the N=256 MMA come from the leader (W1), [128,256) from the peer (W3)
          const CUtensorMap* tw = rank == 0 ? tm_w1 : tm_w3;
          tma_load_3d_pair(sb, tw, fbl, cur.nt * BN1, kb * C::BK, cur.expert);
          tma_load_3d_pair(sb + C::B_BOX, tw, fbl, cur.nt * BN1 + 64, kb * C::BK, cur.expert);
        } else {
          const int n0 = cur.nt * BN2 + (int)rank * 128;
          tma_load_3d_pair(sb, tm_w2, fbl, n0, kb * C::BK, cur.expert);
          tma_load_3d_pair(sb + C::B_BOX, tm_w2, fbl, n0 + 64, kb * C::BK, cur.expert);
        }
      }
      pending |= 1u << stage;
      pend_par = (pend_par & ~(1u << stage)) | (ph << stage);
      if (++stage == C::NST) { stage = 0; ph ^= 1u; }
    }
    cur = nxt;
    buf ^= 1;
  }
  // Index copies issued for items that were not processed must land too.
  for (int b = 0; b < 2; ++b)
    if (gpend & (1u << b)) wait_bar(&ctl->gbar[b], (gph >> b) & 1u, tmo, nullptr);
  // Never leave with a copy still landing in shared memory.  A CTA alone (and a
  // pair leader) waits the last fill of each stage; a pair's peer, whose copies
  // count on the leader, waits until the MMAs released each stage, and if that
  // never comes (an aborted call), for a fixed 100 us.
  bool drained = true;
  for (int s = 0; s < C::NST; ++s) {
    if (!(pending & (1u << s))) continue;
    const uint32_t par = (pend_par >> s) & 1u;
    if (leader) drained &= wait_bar<V == 2>(&ctl->full[s], par, tmo, nullptr);
    else drained &= wait_bar<true>(&ctl->empty[s], par, tmo, abort);
  }
  if (!drained) {
    const uint64_t until = globaltimer() + 100000ull;
    while (globaltimer() < until) __nanosleep(1000);
  }
  if (stamp) { my_stamps[4] = n_g1; my_stamps[5] = n_g2; }
}

// ---------------------------------------------------- TMA producer, gathered ---
// The producer of single-CTA tiles (V = 1, 3) whose GEMM1 A rows are gathered
// straight from x (MOE_SCHED_GATHER_A), run by the whole of warp 0: lane 0
// schedules items, waits on the ring and loads the weight tiles (and GEMM2's h
// rows) exactly as role_tma does, and all 32 lanes issue the GEMM1 A gathers --
// lane l the TMA tile::gather4 of rows 4l..4l+3 of each 128-row band of the tile
// (one instruction per lane per band and k-block, instead of 32 or 64 from one
// thread).  The tile's token indices (1 or 2 aligned 512-byte rows of tok_band)
// are bulk-copied into shared memory one work item ahead.
template <int V>
__device__ void role_tma_gathered(const CUtensorMap* tm_a1, const CUtensorMap* tm_w1,
                                  const CUtensorMap* tm_w3, const CUtensorMap* tm_a2,
                                  const CUtensorMap* tm_w2, const FfnArgs& a, SmemCtl* ctl,
                                  uint8_t* smem, bool run_g1, bool run_g2, int n1, int n2,
                                  const volatile uint32_t* abort) {
  static_assert(V != 2, "CTA pairs gather from one thread (role_tma)");
  using C = Cfg<V>;
  const Work& w = a.w;
  const int lane = threadIdx.x & 31;
  const int NT1 = a.f / BN1;
  const uint64_t tmo = a.timeout_ns;
  const bool stamp = (a.flags & MOE_DBG_TIMESTAMPS) && blockIdx.x < STAMP_CTAS;
  unsigned long long* my_stamps = w.stamps + (size_t)blockIdx.x * NSTAMP;
  Sched sc{0, 0u, run_g1, run_g2, (a.flags & MOE_SCHED_INTERLEAVE) && run_g1 && run_g2,
           stamp ? my_stamps : nullptr};
  int stage = 0;
  uint32_t ph = 0;
  uint32_t pending = 0, pend_par = 0;   // (lane 0) stages with an issued fill, and its parity
  uint32_t gph = 0;                     // parity of the next wait on gbar[0], gbar[1]
  uint32_t gpend = 0;                   // (lane 0) index copies issued and not yet waited
  unsigned long long n_g1 = 0, n_g2 = 0;
  // lane 0 takes the next item; every lane gets it
  auto next_item = [&](Item& it) -> bool {
    int okf = 1;
    if (lane == 0) okf = sched_next<V>(sc, it, a, ctl, 0u, n1, n2, abort) ? 1 : 0;
    okf = __shfl_sync(0xffffffffu, okf, 0);
    int* p = reinterpret_cast<int*>(&it);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(Item) / 4); ++i) p[i] = __shfl_sync(0xffffffffu, p[i], 0);
    return okf != 0;
  };
  // bands of the item this CTA computes (V = 3: 1 or 2)
  auto n_bands = [&](const Item& it) { return (V == 3 && it.rows > BM) ? 2 : 1; };
  auto fetch_indices = [&](const Item& it, int buf) {
    if (lane != 0 || it.kind != K_G1 || it.rows <= 0) return;
    const uint32_t bytes = (uint32_t)(n_bands(it) * BM * 4);   // consecutive bands: one copy
    fence_proxy_async_shared();   // earlier generic reads of this buffer come first
    gpend |= 1u << buf;
    mbar_arrive_expect_tx(&ctl->gbar[buf], bytes);
    bulk_load(&ctl->gidx[buf][0], a.tok_band + (size_t)it.band0 * BM, bytes, &ctl->gbar[buf]);
  };

  bool ok = true;
  Item cur;
  int buf = 0;
  if (!next_item(cur)) ok = false;
  else fetch_indices(cur, buf);
  while (ok && cur.kind != K_END) {
    Item nxt;
    if (!next_item(nxt)) break;
    fetch_indices(nxt, buf ^ 1);
    const bool is1 = cur.kind == K_G1;
    if (is1) ++n_g1; else ++n_g2;
    const int nb = n_bands(cur);
    int okw = 1;
    if (is1 && cur.rows > 0) {
      // every lane reads the indices: every lane waits for them
      okw = wait_bar(&ctl->gbar[buf], (gph >> buf) & 1u, tmo, abort) ? 1 : 0;
      okw = __all_sync(0xffffffffu, okw);
      gph ^= 1u << buf;
      if (lane == 0) gpend &= ~(1u << buf);
    } else if (!is1 && lane == 0) {
      // GEMM2 reads the group's h rows: every GEMM1 column block of its bands stored
      okw = (wait_count(&w.band_done1[cur.band0], BAND_UNIT * (uint32_t)NT1, tmo, abort) &&
             (nb < 2 || wait_count(&w.band_done1[cur.band0 + 1], BAND_UNIT * (uint32_t)NT1, tmo, abort)))
                ? 1 : 0;
      if (okw) fence_proxy_async_global();   // generic-proxy stores -> async-proxy (TMA) loads
    }
    okw = __shfl_sync(0xffffffffu, okw, 0);
    if (!okw) { if (lane == 0) set_error(w.status, is1 ? W_STAGE_FULL : W_BAND1); break; }
    // this lane's token rows of each band (4 per band)
    int4 tk[2] = {make_int4(0, 0, 0, 0), make_int4(0, 0, 0, 0)};
    if (is1)
      for (int b = 0; b < nb; ++b) tk[b] = ctl->gidx[buf][b * (BM / 4) + lane];
    const int nk = (is1 ? a.d : a.f) / C::BK;
    for (int kb = 0; kb < nk; ++kb) {
      int oks = 1;
      if (lane == 0) {
        oks = wait_bar(&ctl->empty[stage], ph ^ 1u, tmo, abort) ? 1 : 0;
        if (oks) mbar_arrive_expect_tx(&ctl->full[stage], C::STAGE - (nb < 2 ? (C::ABOX - 1) * C::A_BYTES : 0));
        else set_error(w.status, W_STAGE_EMPTY);
      }
      oks = __shfl_sync(0xffffffffu, oks, 0);   // (a warp shuffle orders lane 0's expect first)
      if (!oks) { ok = false; break; }
      uint8_t* sa = smem + (size_t)stage * C::STAGE;
      uint8_t* sb = sa + C::ABOX * C::A_BYTES;
      uint64_t* fb = &ctl->full[stage];
      if (is1) {
        for (int b = 0; b < nb; ++b)
          tma_gather4(sa + b * C::A_BYTES + lane * 4 * C::A_ROW, tm_a1, fb, kb * C::BK, tk[b].x, tk[b].y,
                      tk[b].z, tk[b].w);
      }
      if (lane == 0) {
        if (!is1) {
          tma_load_2d(sa, tm_a2, fb, kb * C::BK, cur.row0);
          if (nb == 2) tma_load_2d(sa + C::A_BYTES, tm_a2, fb, kb * C::BK, cur.row0 + BM);
        }
        const int k0 = kb * C::BK;
        if (a.b_atoms) {
          if (is1) {
            tma_load_4d(sb, tm_w1, fb, 0, k0, cur.nt * (BN1 / 64), cur.expert);
            tma_load_4d(sb + 2 * C::B_BOX, tm_w3, fb, 0, k0, cur.nt * (BN1 / 64), cur.expert);
          } else {
            tma_load_4d(sb, tm_w2, fb, 0, k0, cur.nt * (BN2 / 64), cur.expert);
          }
        } else if (is1) {
          tma_load_3d(sb, tm_w1, fb, cur.nt * BN1, k0, cur.expert);
          tma_load_3d(sb + C::B_BOX, tm_w1, fb, cur.nt * BN1 + 64, k0, cur.expert);
          tma_load_3d(sb + 2 * C::B_BOX, tm_w3, fb, cur.nt * BN1, k0, cur.expert);
          tma_load_3d(sb + 3 * C::B_BOX, tm_w3, fb, cur.nt * BN1 + 64, k0, cur.expert);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tma_load_3d(sb + q * C::B_BOX, tm_w2, fb, cur.nt * BN2 + q * 64, k0, cur.expert);
        }
        pending |= 1u << stage;
        pend_par = (pend_par & ~(1u << stage)) | (ph << stage);
      }
      if (++stage == C::NST) { stage = 0; ph ^= 1u; }
    }
    __syncwarp();
    cur = nxt;
    buf ^= 1;
  }
  if (lane == 0) {
    // index copies issued for items that were not processed must land too, and
    // no copy may still be landing in shared memory when the CTA leaves
    for (int b = 0; b < 2; ++b)
      if (gpend & (1u << b)) wait_bar(&ctl->gbar[b], (gph >> b) & 1u, tmo, nullptr);
    bool drained = true;
    for (int s2 = 0; s2 < C::NST; ++s2)
      if (pending & (1u << s2)) drained &= wait_bar(&ctl->full[s2], (pend_par >> s2) & 1u, tmo, nullptr);
    if (!drained) {
      const uint64_t until = globaltimer() + 100000ull;
      while (globaltimer() < until) __nanosleep(1000);
    }
    if (stamp) { my_stamps[4] = n_g1; my_stamps[5] = n_g2; }
  }
  __syncwarp();
}

// ------------------------------------------- GEMM1 A rows, load/store path ---
// MOE_SCHED_GATHER_LSU (single CTAs): GW extra warps copy every GEMM1 k-block's
// A rows straight from x into the stage with 16-byte cp.async, in the swizzled
// layout a tiled TMA load gives -- rows of A_ROW bytes (CPR 16-byte chunks), chunk
// c of row r at r*A_ROW + ((c ^ ((r*A_ROW >> 7) & (CPR-1))) << 4), the 128- or
// 64-byte swizzle -- so x_perm is never written and the TMA thread loads the
// weights only.  Thread t copies chunk t % CPR of rows t / CPR, t / CPR + NT / CPR,
// ... (each warp instruction: 32 / CPR rows of A_ROW contiguous bytes).  The
// warps walk the item ring like the MMA and epilogue warps; for every k-block of
// every item each thread waits (through lane 0) for the stage to be free, issues
// its copies (GEMM1 only: GEMM2's A rows come by TMA) and arrives on the stage's
// full barrier with cp.async.mbarrier.arrive.noinc -- the arrival happens when its
// copies have landed, so the warps never block on them.  The MMA thread, after it
// waits on the full barrier, fences the generic proxy (these writes) against the
// async proxy (its operand reads).
template <int V, int GW>
__device__ void role_gather_lsu(const FfnArgs& a, SmemCtl* ctl, uint8_t* smem, int gw, int lane,
                                const volatile uint32_t* abort) {
  using C = Cfg<V>;
  const Work& w = a.w;
  const uint64_t tmo = a.timeout_ns;
  constexpr int NT = GW * 32;                  // copying threads
  constexpr int CPR = C::A_ROW / 16;           // 16-byte chunks per A row
  constexpr int RSTEP = NT / CPR;              // rows per pass of all threads
  constexpr int ROWS = C::ABOX * BM;           // A rows of a k-block
  const int gt = gw * 32 + lane;
  const int c = gt % CPR;
  const size_t row_bytes = (size_t)a.d * 2;
  const char* x = reinterpret_cast<const char*>(a.x);
  int slot = 0, stage = 0;
  uint32_t sph = 0, ph = 0;
  bool ok = true;
  while (ok) {
    if (!__all_sync(0xffffffffu, wait_bar(&ctl->sfull[slot], sph, tmo, abort))) {
      if (lane == 0 && gw == 0) set_error(w.status, W_SCHED_FULL);
      break;
    }
    const Item it = ctl->ring[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->sempty[slot]);
    if (++slot == SCHED_DEPTH) { slot = 0; sph ^= 1u; }
    if (it.kind == K_END) break;
    const bool is1 = it.kind == K_G1;
    const int nk = (is1 ? a.d : a.f) / C::BK;
    // rows to copy: the group's bands (V = 3 without a second band: the first 128)
    const int nrows = (V == 3 && it.rows > BM) ? 2 * BM : BM;
    const int32_t* tok = a.tok_band + (size_t)it.band0 * BM;   // 0 past the bands' rows
    for (int kb = 0; kb < nk; ++kb) {
      int okw = 1;
      if (lane == 0) okw = wait_bar(&ctl->empty[stage], ph ^ 1u, tmo, abort) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) {
        if (lane == 0 && gw == 0) set_error(w.status, W_STAGE_EMPTY);
        ok = false;
        break;
      }
      if (is1) {
        uint8_t* sa = smem + (size_t)stage * C::STAGE;
        const size_t col = (size_t)kb * C::BK * 2 + (size_t)c * 16;
#pragma unroll 4
        for (int r = gt / CPR; r < ROWS; r += RSTEP) {
          if (r >= nrows) break;
          const int t = __ldg(tok + r);
          const int sw = ((r * C::A_ROW) >> 7) & (CPR - 1);
          cp_async16(sa + r * C::A_ROW + ((c ^ sw) << 4), x + (size_t)t * row_bytes + col);
        }
        cp_async_arrive_noinc(&ctl->full[stage]);   // arrives when these copies landed
      } else {
        mbar_arrive(&ctl->full[stage]);
      }
      if (++stage == C::NST) { stage = 0; ph ^= 1u; }
    }
  }
  cp_async_wait<0>();   // never leave with copies landing in shared memory
}

// --------------------------------------------------------------- MMA issuer ---
// MMA descriptor of an A box at `saddr` (plus the K offset of the MMA step): K-major
// rows of A_ROW bytes in the matching swizzle, 8-row atoms 8 * A_ROW bytes apart.
// B (MN-major) is always 128-byte K rows, 64-column atoms B_BOX bytes apart.
template <int V>
__device__ __forceinline__ uint64_t a_desc(uint32_t saddr) {
  if constexpr (Cfg<V>::A_ROW == 64) return smem_desc_sw64(saddr, 16, 8 * 64);
  else return smem_desc_sw128(saddr, 16, 8 * 128);
}

// One thread (a single CTA's, or the pair leader's) issues every MMA.
// V = 1, 2: one accumulator per tile, alternating, so the epilogue of tile i
// overlaps the main loop of tile i+1.  V = 3: both accumulators per tile, acc b
// taking band b's 128 rows (A box b) against the same B stage; tile i+1's first
// MMAs into acc 0 wait only for acc 0 of tile i to be drained, acc 1 for acc 1.
template <int V>
__device__ void role_mma(const FfnArgs& a, SmemCtl* ctl, uint8_t* smem, uint32_t tmem_base,
                         const volatile uint32_t* abort) {
  using C = Cfg<V>;
  const uint64_t tmo = a.timeout_ns;
  constexpr uint32_t idesc_full = idesc_bf16_f32(BM * C::CTAS, 256, true);
  constexpr uint32_t idesc_half = idesc_bf16_f32(BM, 256, true);   // V == 2 only
  int stage = 0, slot = 0, acc = 0;
  uint32_t ph = 0, sph = 0, aph = 0;
  const bool lsu = a.gather == 2;
  while (true) {
    if (!wait_bar(&ctl->sfull[slot], sph, tmo, abort)) { set_error(a.w.status, W_SCHED_FULL); break; }
    const Item it = ctl->ring[slot];
    mbar_arrive(&ctl->sempty[slot]);
    if (++slot == SCHED_DEPTH) { slot = 0; sph ^= 1u; }
    if (it.kind == K_END) break;
    const int nk = (it.kind == K_G1 ? a.d : a.f) / C::BK;
    bool ok = true;
    if (V == 3) {
      const bool two = it.rows > BM;
      // acc b's 4 MMAs of one k-block from stage `st`
      auto issue = [&](int b, int st, int kb) {
        const uint32_t sa = smem_u32(smem + (size_t)st * C::STAGE);
        const uint32_t sb = sa + C::ABOX * C::A_BYTES;
        const uint32_t dt = tmem_base + (uint32_t)(b * ACC_COLS);
#pragma unroll
        for (int ks = 0; ks < C::BK / 16; ++ks) {
          const uint64_t ad = a_desc<V>(sa + b * C::A_BYTES + ks * 32);
          const uint64_t bd = smem_desc_sw128(sb + ks * 2048, C::B_BOX, 1024);
          tc_mma_f16(dt, ad, bd, idesc_full, (kb | ks) != 0 ? 1u : 0u);
        }
      };
      // both accumulators' phases advance every tile, a one-band group's too
      auto acc_free = [&](int b) {
        if (!wait_bar(&ctl->tempty[b], aph ^ 1u, tmo, abort)) { set_error(a.w.status, W_TMEM_EMPTY); return false; }
        tc_fence_after();
        return true;
      };
      for (int kb = 0; kb < nk && ok; ++kb) {
        if (!wait_bar(&ctl->full[stage], ph, tmo, abort)) { set_error(a.w.status, W_STAGE_FULL); ok = false; break; }
        if (lsu) fence_proxy_async_shared();   // the gather warps' generic-proxy writes
        tc_fence_after();
        for (int b = 0; b < 2; ++b) {
          if (kb == 0 && !acc_free(b)) { ok = false; break; }
          if (b == 1 && !two) continue;
          issue(b, stage, kb);
        }
        if (!ok) break;
        tc_commit(&ctl->empty[stage]);
        if (++stage == C::NST) { stage = 0; ph ^= 1u; }
      }
      if (!ok) break;
      tc_commit(&ctl->tfull[0]);
      tc_commit(&ctl->tfull[1]);
      aph ^= 1u;
      continue;
    }
    if (!wait_bar<V == 2>(&ctl->tempty[acc], aph ^ 1u, tmo, abort)) { set_error(a.w.status, W_TMEM_EMPTY); break; }
    tc_fence_after();
    const uint32_t dt = tmem_base + (uint32_t)(acc * ACC_COLS);
    const uint32_t idesc = half_tile<V>(it, a) ? idesc_half : idesc_full;
    for (int kb = 0; kb < nk; ++kb) {
      if (!wait_bar<V == 2>(&ctl->full[stage], ph, tmo, abort)) { set_error(a.w.status, W_STAGE_FULL); ok = false; break; }
      if (lsu) fence_proxy_async_shared();   // the gather warps' generic-proxy writes
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)stage * C::STAGE);
      const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
      for (int ks = 0; ks < C::BK / 16; ++ks) {
        const uint64_t ad = a_desc<V>(sa + ks * 32);
        const uint64_t bd = smem_desc_sw128(sb + ks * 2048, C::B_BOX, 1024);
        if (V != 2) tc_mma_f16(dt, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
        else tc_mma_f16_pair(dt, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
      }
      // frees the smem stage (in both CTAs of a pair) once these MMAs finish
      if (V != 2) tc_commit(&ctl->empty[stage]);
      else tc_commit_pair(&ctl->empty[stage], (uint16_t)0x3);
      if (++stage == C::NST) { stage = 0; ph ^= 1u; }
    }
    if (!ok) break;
    // accumulator ready for the epilogue (of both CTAs of a pair)
    if (V != 2) tc_commit(&ctl->tfull[acc]);
    else tc_commit_pair(&ctl->tfull[acc], (uint16_t)0x3);
    acc ^= 1;
    if (acc == 0) aph ^= 1u;
  }
  // Wait for every MMA this thread issued before TMEM can be released.
  if (V != 2) tc_commit(&ctl->mma_done);
  else tc_commit_pair(&ctl->mma_done, (uint16_t)0x1);
  wait_bar(&ctl->mma_done, 0u, tmo, nullptr);
}

// ----------------------------------------------------------------- epilogue ---
static_assert(EPI_WARPS == 8, "the epilogue splits each accumulator's columns between two warps");

// This warp's 32 TMEM lanes of one accumulator, columns [c0, c1) (multiples of
// 32) -> registers -> bf16 -> global memory, rows `row` of the lanes whose
// `valid` is set (the warp's lanes hold consecutive rows):
//   GEMM1: h[row][col0 + c] = silu(acc[c]) * acc[nc + c] (nc = 128 for a full
//          tile, 64 for a half tile's lane half),
//   GEMM2: y[row][col0 + c] = acc[c] (nc = 256, or 128 in a half tile).
// Each 32-column chunk (64 bytes per row) goes through the warp's staging tile
// in shared memory, so that a store instruction writes 8 rows x 64 contiguous
// bytes instead of 32 rows x 16.
// GEMM1's h rows are read back by TMA (async proxy) in other CTAs: the caller
// fences them (fence.proxy.async) after releasing the accumulator and before
// the tile is published.
__device__ __forceinline__ void store_chunk(uint8_t* ost, const uint32_t (&pk)[16], int lane,
                                            unsigned vmask, __nv_bfloat16* base_row0,
                                            size_t ld, int col, bool evict_first, uint64_t pol) {
#pragma unroll
  for (int v = 0; v < 4; ++v)
    *reinterpret_cast<uint4*>(ost + lane * OSTAGE_ROW + v * 16) =
        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
  __syncwarp();
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int r = (lane >> 2) + 8 * v;            // row of the warp this lane writes
    const uint4 val = *reinterpret_cast<const uint4*>(ost + r * OSTAGE_ROW + (lane & 3) * 16);
    if ((vmask >> r) & 1u) {
      uint4* dst = reinterpret_cast<uint4*>(base_row0 + (size_t)r * ld + col + (lane & 3) * 8);
      if (evict_first) st_global_v4_policy(dst, val, pol);
      else *dst = val;
    }
  }
  __syncwarp();
}

__device__ __forceinline__ void drain_acc(const FfnArgs& a, int kind, uint32_t tb, size_t row,
                                          bool valid, int nc, int col0, int c0, int c1,
                                          uint8_t* ost) {
  const int lane = threadIdx.x & 31;
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  const size_t row0 = row - (size_t)lane;         // the warp's first row
  const bool ef = (a.flags & MOE_SCHED_EVICT_FIRST) != 0;
  const uint64_t pol = ef ? l2_policy_evict_first() : 0ull;
  if (kind == K_G1) {
    __nv_bfloat16* base = a.h + row0 * a.f + col0;
#pragma unroll 1
    for (int c = c0 / 32; c < c1 / 32; ++c) {
      uint32_t ra[32], rb[32];
      tmem_ld32(tb + c * 32, ra);
      tmem_ld32(tb + nc + c * 32, rb);
      tmem_ld_wait();
      uint32_t pk[16];
      if (!(a.flags & MOE_SCHED_EXP_SILU)) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(silu_mul_tanh(__uint_as_float(ra[2 * i]), __uint_as_float(rb[2 * i])),
                              silu_mul_tanh(__uint_as_float(ra[2 * i + 1]), __uint_as_float(rb[2 * i + 1])));
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(silu_mul(__uint_as_float(ra[2 * i]), __uint_as_float(rb[2 * i])),
                              silu_mul(__uint_as_float(ra[2 * i + 1]), __uint_as_float(rb[2 * i + 1])));
      }
      store_chunk(ost, pk, lane, vmask, base, (size_t)a.f, c * 32, ef, pol);
    }
  } else {
    __nv_bfloat16* base = a.y + row0 * a.d + col0;
#pragma unroll 1
    for (int c = c0 / 32; c < c1 / 32; ++c) {
      uint32_t rr[32];
      tmem_ld32(tb + c * 32, rr);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(rr[2 * i]), __uint_as_float(rr[2 * i + 1]));
      store_chunk(ost, pk, lane, vmask, base, (size_t)a.d, c * 32, ef, pol);
    }
  }
}

// Publish a stored band tile: fence, then add `units` to the band's counter with
// release semantics (skipped for band 0's GEMM1 tiles under MOE_DBG_SKIP_FLAG_BAND).
__device__ __forceinline__ void publish_band(const FfnArgs& a, int kind, int band, uint32_t units) {
  if ((a.flags & MOE_DBG_SKIP_FLAG_BAND) && kind == K_G1 && band == 0) return;
  __threadfence();
  red_release_add(kind == K_G1 ? &a.w.band_done1[band] : &a.w.band_done2[band], units);
}

// The arrivals of a completed band: every row's token gets one more of its k rows
// (acq_rel, so the rows' stores are seen by whoever sees the count); the row that
// brings a token to k appends it to the ready queue (st.release of t + 1 into an
// allocated entry).  Threads lane, lane + nl, ... take the band's rows.
__device__ void band_arrivals(const FfnArgs& a, int band, int lane, int nl) {
  const Work& w = a.w;
  const Band bd = w.bands[band];
  const int k = a.k;
  for (int r = lane; r < bd.rows; r += nl) {
    const int t = w.perm[bd.row0 + r] / k;
    if (atom_acq_rel_add(&w.arrive[t], 1u) == (uint32_t)(k - 1)) {
      const uint32_t e = atomicAdd(&w.sync->rq_alloc, 1u);
      __threadfence();
      st_release(&w.ready_q[e], (uint32_t)t + 1u);
    }
  }
}

// Publish a stored GEMM2 tile with side combine warps: the counter is bumped with a
// returning acq_rel atomic, so the CTA whose tile completes the band knows it (and
// has acquired every other tile's stores); it hands the band to its side warps
// through the shared-memory ring, or, with the ring full, does the arrivals itself.
__device__ __forceinline__ void publish_g2_side(const FfnArgs& a, SmemCtl* ctl, int band, uint32_t units) {
  __threadfence();
  const uint32_t full = BAND_UNIT * (uint32_t)(a.d / BN2);
  if (atom_acq_rel_add(&a.w.band_done2[band], units) + units != full) return;
  volatile int* vt = &ctl->btail;
  volatile int* vh = &ctl->bhead;
  const int tl = *vt;
  if (tl - *vh < SIDE_RING) {
    ctl->bring[tl % SIDE_RING] = band;
    __threadfence_block();   // the entry before the tail that exposes it
    *vt = tl + 1;
  } else {
    band_arrivals(a, band, 0, 1);
  }
}

// Eight warps per CTA; warp w reads TMEM lanes [32q, 32q+32) with q = w mod 4,
// i.e. rows 32q.. of each accumulator's 128 rows, and half of the accumulator's
// columns, hc = (w - 2) / 4.  Stores are masked to the band's valid rows; then
// the tile is published on the band's counter.
template <int V>
__device__ void role_epilogue(const FfnArgs& a, SmemCtl* ctl, uint32_t tmem_base, uint32_t rank,
                              int warp, int lane, const volatile uint32_t* abort) {
  const Work& w = a.w;
  const uint64_t tmo = a.timeout_ns;
  const int q = warp & 3;                 // TMEM lane quadrant this warp may read
  const int hc = (warp - 2) >> 2;         // which half of the columns
  const int row = q * 32 + lane;
  int slot = 0, acc = 0;
  uint32_t sph = 0, aph = 0, eph = 0;   // eph: one parity bit per accumulator
  while (true) {
    // Every lane waits; the warp proceeds only if all lanes saw the phase, so a
    // timeout never splits the warp before the .sync.aligned TMEM loads.
    bool ok = __all_sync(0xffffffffu, wait_bar<V == 2>(&ctl->sfull[slot], sph, tmo, abort));
    if (!ok) { if (lane == 0) set_error(w.status, W_SCHED_FULL); break; }
    const Item it = ctl->ring[slot];
    __syncwarp();
    if (lane == 0) arrive_leader<V>(&ctl->sempty[slot], rank);
    if (++slot == SCHED_DEPTH) { slot = 0; sph ^= 1u; }
    if (it.kind == K_END) break;
    const int col0 = it.kind == K_G1 ? it.nt * BN1 : it.nt * BN2;
    const int ncf = it.kind == K_G1 ? BN1 : BN2;   // columns a full tile stores
    if (V == 3) {
      // acc b holds band0+b: rows it.row0 + 128 b + row
      for (int b = 0; b < 2 && ok; ++b) {
        ok = __all_sync(0xffffffffu, wait_bar(&ctl->tfull[b], aph, tmo, abort));
        if (!ok) { if (lane == 0) set_error(w.status, W_TMEM_FULL); break; }
        tc_fence_after();
        const int rb = min(BM, max(0, it.rows - b * BM));
        if (rb > 0)
          drain_acc(a, it.kind, tmem_base + (uint32_t)(b * ACC_COLS) + ((uint32_t)(q * 32) << 16),
                    (size_t)(it.row0 + b * BM + row), row < rb, ncf, col0, hc * ncf / 2,
                    (hc + 1) * ncf / 2, ctl->ostage[warp - 2]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->tempty[b]);   // accumulator may be overwritten
        if (it.kind == K_G1) fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->epi_done[b]);  // this warp's rows of band b are stored
      }
      if (!ok) break;
      aph ^= 1u;
      // publish both bands once the epilogue warps stored them (each epi_done phase
      // holds one tile's arrivals: a warp can run at most one tile ahead)
      if (warp == 2 && lane == 0) {
        for (int b = 0; b < 2; ++b) {
          const bool stored = wait_bar(&ctl->epi_done[b], (eph >> b) & 1u, tmo, abort);
          if (!stored) { set_error(w.status, W_DRAIN); break; }
          if (it.rows <= b * BM) continue;
          if (a.side && it.kind == K_G2) publish_g2_side(a, ctl, it.band0 + b, BAND_UNIT);
          else publish_band(a, it.kind, it.band0 + b, BAND_UNIT);
        }
      }
      eph ^= 3u;
      __syncwarp();
      continue;
    }
    ok = __all_sync(0xffffffffu, wait_bar<V == 2>(&ctl->tfull[acc], aph, tmo, abort));
    if (!ok) { if (lane == 0) set_error(w.status, W_TMEM_FULL); break; }
    tc_fence_after();
    const bool half = half_tile<V>(it, a);
    const MyRows m = my_rows<V>(it, rank, half);
    const uint32_t tb = tmem_base + (uint32_t)(acc * ACC_COLS) + ((uint32_t)(q * 32) << 16);
    // full tile: lane `row` is row `row`, all N columns; half tile: lane `row` is
    // row row % 64, and the N/2 columns of the B half row / 64 supplied (GEMM1:
    // h columns nt*128 + 64*ch + [0,64) from accumulator columns [0,64) and
    // [64,128); GEMM2: y columns nt*256 + 128*ch + [0,128))
    const int r = half ? (row & (BM / 2 - 1)) : row;
    const int ch = half ? (row >> 6) : 0;
    const int nc = half ? ncf / 2 : ncf;
    drain_acc(a, it.kind, tb, (size_t)(m.row0 + r), r < m.rows, nc, col0 + ch * nc, hc * nc / 2,
              (hc + 1) * nc / 2, ctl->ostage[warp - 2]);
    tc_fence_before();
    __syncwarp();
    const int my_acc = acc;
    if (lane == 0) arrive_leader<V>(&ctl->tempty[my_acc], rank);   // accumulator may be overwritten
    if (it.kind == K_G1) fence_proxy_async_global();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->epi_done[my_acc]);            // this warp's rows are stored
    acc ^= 1;
    if (acc == 0) aph ^= 1u;
    // Publish the tile: one thread waits (bounded) for this CTA's epilogue
    // warps' stores of the tile, then fences and bumps its band's counter with
    // release semantics.  A warp can run at most one tile ahead, and consecutive
    // tiles use different accumulators, so each epi_done phase holds one tile's
    // arrivals only.  A half tile's band is published by both CTAs (even one with
    // no valid rows), one unit each.
    if (warp == 2 && lane == 0) {
      const bool stored = wait_bar(&ctl->epi_done[my_acc], (eph >> my_acc) & 1u, tmo, abort);
      if (!stored) set_error(w.status, W_DRAIN);
      else if (a.side && it.kind == K_G2 && m.rows > 0) publish_g2_side(a, ctl, m.band, BAND_UNIT);
      else if (half || m.rows > 0) publish_band(a, it.kind, m.band, half ? BAND_UNIT / 2 : BAND_UNIT);
    }
    eph ^= 1u << my_acc;
    __syncwarp();
  }
}

// ----------------------------------------------------------------- consumer ---
// The return step.  A consuming CTA repeatedly takes whichever work is ready:
//  * BAND: the next combine item (row bands in priority order, [TLS] 3.3.2), once
//    all its bands are flagged -- claimed only then, so nobody blocks on it.
//    Every thread takes one row and bumps its token's arrival counter (acq_rel);
//    the thread that brings it to k appends the token to the ready queue
//    (st.release of t+1 into an allocated entry).
//  * COMBINE: up to S ready tokens from the queue.  Their k expert rows are
//    streamed into a shared-memory slot ring with cp.async.bulk by one thread,
//    and warps 1.. each reduce a column slice of every token in fp32, slot order
//    (the arithmetic of combine_token_warp, so both modes agree bit for bit),
//    storing out[t] with 16-byte stores.
// Splitting arrival from reduction lets every consuming CTA share the tokens
// that the last bands complete, instead of one CTA per band.  Consumers work only
// while GEMM work remains (dedicated consumers during GEMM2, producers that
// finished early during its last wave); once every CTA has left the producer
// role they stop, and a full-occupancy combine pass after this kernel handles
// every token not flagged TOKEN_DONE.
// If one token's rows do not fit the staging area, warps fall back to
// combine_token_warp straight from global memory.
enum : int { C_IDLE = 0, C_BAND = 1, C_COMBINE = 2, C_DONE = 3, C_ERROR = 4 };

__device__ void role_consumer(const FfnArgs& a, SmemCtl* ctl, uint8_t* smem, int nb, int n_items,
                              const volatile uint32_t* abort) {
  const Work& w = a.w;
  const uint32_t NT2 = (uint32_t)(a.d / BN2);
  const int k = a.k, d = a.d, dv = d >> 3;
  const uint32_t T = (uint32_t)a.T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NTHREADS = (int)blockDim.x;
  const int NWARPS = NTHREADS / 32;
  const int NCW = NWARPS - 1;                             // reducing warps
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const uint32_t tok_bytes = row_bytes * (uint32_t)k;
  int S = (int)((size_t)STAGE_AREA / tok_bytes);
  if (S > CONS_SLOTS) S = CONS_SLOTS;
  const int chunk = S >= 1 ? S : NWARPS;                  // tokens per COMBINE
  uint32_t base = 0;                                      // tokens this CTA reduced so far
  uint32_t pend = 0, pend_par = 0;                        // issuer: slots with a copy issued
  unsigned long long n_bands_done = 0;
  const bool stamp_on = (a.flags & MOE_DBG_TIMESTAMPS) != 0;
  uint64_t idle_since = 0;
  int my_item = -1;                                       // thread 0: band ticket held, not yet processed
  // thread 0: band tickets may remain (none with side warps: the producers' CTAs
  // do every band's arrivals)
  bool items_left = !a.side;
  while (true) {
    // ---- thread 0 decides what to do next.  Band items and queue entries are
    // taken with fetch-and-add tickets (no CAS contention at the tail).  A CTA
    // holding a band ticket waits for that band, combining already-queued
    // tokens meanwhile; once every band ticket is taken, CTAs take queue tickets
    // and wait for their entries -- every entry will be written, because every
    // band still to come is held by a CTA that waits only on the producers.
    if (threadIdx.x == 0) {
      int act = C_IDLE, arg0 = 0, arg1 = 0;
      if (*abort) act = C_ERROR;
      // Once every CTA has left the producer role the GEMM work is over: stop, and
      // leave what is not combined yet to the full-occupancy combine pass that
      // follows this kernel.
      else if (ld_relaxed(&w.sync->prod_done) >= gridDim.x) act = C_DONE;
      if (act == C_IDLE && my_item < 0 && items_left) {
        const int t = (int)atomicAdd(&w.sync->qc, 1u);
        if (t < n_items) my_item = t; else items_left = false;
      }
      if (act == C_IDLE && my_item >= 0) {
        int b0, b1;
        item_range(my_item, nb, a.mgb, b0, b1);
        bool ready = true;
        for (int b = b0; b < b1 && ready; ++b) ready = ld_acquire(&w.band_done2[b]) >= BAND_UNIT * NT2;
        if (ready) {
          act = C_BAND; arg0 = b0; arg1 = b1;
          my_item = -1;
        } else {
          // meanwhile: tokens already in the queue (allocated entries only)
          const uint32_t h = ld_relaxed(&w.sync->rq_head);
          const uint32_t al = ld_relaxed(&w.sync->rq_alloc);
          if (h < al) {
            const uint32_t n = min(al - h, (uint32_t)chunk);
            if (atomicCAS(&w.sync->rq_head, h, h + n) == h) { act = C_COMBINE; arg0 = (int)h; arg1 = (int)n; }
          }
        }
      } else if (act == C_IDLE) {
        const uint32_t h = atomicAdd(&w.sync->rq_head, (uint32_t)chunk);
        if (h >= T) act = C_DONE;
        else { act = C_COMBINE; arg0 = (int)h; arg1 = (int)min((uint32_t)chunk, T - h); }
      }
      if (act == C_IDLE) {
        const uint64_t now = globaltimer();
        if (idle_since == 0) idle_since = now;
        else if (now - idle_since > a.timeout_ns) { set_error(w.status, W_CONS_IDLE); act = C_ERROR; }
      } else {
        idle_since = 0;
      }
      ctl->item = act;
      ctl->ok = arg0;
      ctl->cn = arg1;
    }
    __syncthreads();
    const int act = ctl->item, arg0 = ctl->ok, arg1 = ctl->cn;
    __syncthreads();   // everyone has read the decision before thread 0 rewrites it
    if (act == C_DONE || act == C_ERROR) break;
    if (act == C_IDLE) {
      if (threadIdx.x == 0) __nanosleep(200);
      continue;
    }
    if (act == C_BAND) {
      for (int b = arg0; b < arg1; ++b) {
        const bool bstamp = stamp_on && b < STAMP_BANDS && threadIdx.x == 0;
        unsigned long long* bs = w.stamps + (size_t)STAMP_CTAS * NSTAMP + (size_t)b * 4;
        if (bstamp) { bs[0] = globaltimer(); bs[3] = blockIdx.x; }
        const Band bd = w.bands[b];
        unsigned long long completed = 0;
        for (int r = threadIdx.x; r < bd.rows; r += NTHREADS) {
          const int t = w.perm[bd.row0 + r] / k;
          if (atom_acq_rel_add(&w.arrive[t], 1u) == (uint32_t)(k - 1)) {
            const uint32_t e = atomicAdd(&w.sync->rq_alloc, 1u);
            __threadfence();
            st_release(&w.ready_q[e], (uint32_t)t + 1u);
            ++completed;
          }
        }
        ++n_bands_done;
        if (bstamp) { bs[1] = globaltimer(); bs[2] = completed; }
      }
      __syncthreads();
      continue;
    }
    // ---- C_COMBINE: queue entries [arg0, arg0 + arg1)
    if (threadIdx.x == 0) ctl->cn = 0;
    __syncthreads();
    bool got = true;
    if (threadIdx.x < arg1) {
      // The entry is (or will be) written by some band's arrivals.  Spin, bounded;
      // give up once the GEMM work is over (that token is then combined by the
      // pass after this kernel).
      uint32_t* q = &w.ready_q[arg0 + threadIdx.x];
      uint32_t v = ld_acquire(q);
      const uint64_t deadline = globaltimer() + a.timeout_ns;
      while (v == 0u && !*abort) {
        if (ld_relaxed(&w.sync->prod_done) >= gridDim.x) break;
        if (globaltimer() > deadline) { set_error(w.status, W_CONS_QUEUE); got = false; break; }
        __nanosleep(64);
        v = ld_acquire(q);
      }
      if (v != 0u) {
        const int t = (int)v - 1;
        const int i = atomicAdd(&ctl->cn, 1);
        ctl->ctok[i] = t;
        for (int j = 0; j < k; ++j) {
          ctl->crow[i][j] = w.row_of[(size_t)t * k + j];
          ctl->cgate[i][j] = a.gate[(size_t)t * k + j];
        }
      }
    }
    if (!__syncthreads_and(got)) break;
    const int n = ctl->cn;
    if (S < 1) {
      for (int i = warp; i < n; i += NWARPS)
        combine_token_warp(a.y, w.row_of, a.gate, ctl->ctok[i], d, k, a.out, lane);
    } else if (warp == 0) {
      if (lane == 0) {
        fence_proxy_async_global();   // y rows were stored by other SMs' generic stores
        for (int i = 0; i < n; ++i) {
          const uint32_t g = base + (uint32_t)i;
          const int s = (int)(g % (uint32_t)S);
          const uint32_t ph = (g / (uint32_t)S) & 1u;
          if (!wait_bar(&ctl->cempty[s], ph ^ 1u, a.timeout_ns, abort)) { set_error(w.status, W_CONS_EMPTY); break; }
          uint8_t* dst = smem + (size_t)s * tok_bytes;
          mbar_arrive_expect_tx(&ctl->cfull[s], tok_bytes);
          for (int j = 0; j < k; ++j)
            bulk_load(dst + (size_t)j * row_bytes, a.y + (size_t)ctl->crow[i][j] * d, row_bytes,
                      &ctl->cfull[s]);
          pend |= 1u << s;
          pend_par = (pend_par & ~(1u << s)) | (ph << s);
        }
      }
    } else {
      // Every reducing warp takes every token in order (a slice of its columns),
      // so each warp waits each slot's phases in order -- an mbarrier parity wait
      // cannot tell two phases apart.
      const int cw = warp - 1;
      for (int i = 0; i < n; ++i) {
        const uint32_t g = base + (uint32_t)i;
        const int s = (int)(g % (uint32_t)S);
        const uint32_t ph = (g / (uint32_t)S) & 1u;
        if (!__all_sync(0xffffffffu, wait_bar(&ctl->cfull[s], ph, a.timeout_ns, abort))) {
          if (lane == 0) set_error(w.status, W_CONS_FULL);
          break;
        }
        const int t = ctl->ctok[i];
        float gt[MAX_K];
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) gt[j] = j < k ? ctl->cgate[i][j] : 0.0f;
        const uint4* src = reinterpret_cast<const uint4*>(smem + (size_t)s * tok_bytes);
        uint4* ov = reinterpret_cast<uint4*>(a.out) + (size_t)t * dv;
        for (int v = cw * 32 + lane; v < dv; v += NCW * 32) {
          float acc[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
          for (int j = 0; j < MAX_K; ++j) {
            if (j < k) {
              float f[8];
              bf16x8_to_f32(src[(size_t)j * dv + v], f);
#pragma unroll
              for (int q = 0; q < 8; ++q) acc[q] = fmaf(gt[j], f[q], acc[q]);
            }
          }
          ov[v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                             pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->cempty[s]);
      }
    }
    base += (uint32_t)n;
    __syncthreads();
    // every warp's slice of these tokens is stored: mark them combined
    if (threadIdx.x < n) atomicOr(&w.arrive[ctl->ctok[threadIdx.x]], TOKEN_DONE);
    __syncthreads();
  }
  // Never leave with a bulk copy still landing in shared memory.
  if (threadIdx.x == 0)
    for (int s = 0; s < S; ++s)
      if (pend & (1u << s)) wait_bar(&ctl->cfull[s], (pend_par >> s) & 1u, a.timeout_ns, nullptr);
  if (threadIdx.x == 0 && stamp_on && blockIdx.x < STAMP_CTAS)
    w.stamps[(size_t)blockIdx.x * NSTAMP + 6] = n_bands_done;
}

// ------------------------------------------------------------ side warps ---
// MOE_SCHED_SIDE_COMBINE: the consumer work of [TLS] Section 3.3.3 spread over two
// extra warps in every producer CTA instead of a partition of whole SMs, so that no
// SM gives up tensor-core time for it.  A side warp repeatedly takes, in this order:
//  * a band its CTA completed (the ring filled by publish_g2_side): the band's
//    arrivals, 32 rows at a time;
//  * up to SIDE_TOK tokens of the ready queue, claimed only where entries are
//    already allocated (never waiting for future bands): each token is combined
//    straight from global memory by the warp (the combine kernel's routine, so the
//    same bits) and flagged TOKEN_DONE;
// and leaves as soon as its CTA's producer warps have all left their roles.  The CTA then joins the consumer role (without band tickets) if joining
// is on; the combine pass after the kernel finishes any token left.
enum : int { S_IDLE = 0, S_BAND = 1, S_COMBINE = 2, S_EXIT = 3, S_RETRY = 4 };

__device__ void role_side(const FfnArgs& a, SmemCtl* ctl, int lane, const volatile uint32_t* abort) {
  const Work& w = a.w;
  volatile int* vh = &ctl->bhead;
  volatile int* vt = &ctl->btail;
  volatile int* vl = &ctl->prod_left;
  uint64_t idle_since = 0;
  uint32_t nap = 64;
  while (true) {
    int act = S_IDLE, arg = 0, n = 0;
    if (lane == 0) {
      if (*abort) {
        act = S_EXIT;
      } else {
        const int hd = *vh, tl = *vt;
        if (*vl == 0) {
          // The CTA's producers are done: leave at once, so that the CTA's exit (and
          // with the last CTA, the kernel's end) waits for nothing here.  Bands
          // still in the ring and tokens not combined go to the combine pass.
          act = S_EXIT;
        } else if (hd < tl) {
          __threadfence_block();   // the entry after the tail that exposed it
          const int b = ctl->bring[hd % SIDE_RING];   // read before the claim frees the slot
          if (atomicCAS(&ctl->bhead, hd, hd + 1) == hd) { act = S_BAND; arg = b; }
          else act = S_RETRY;
        } else {
          const uint32_t h = ld_relaxed(&w.sync->rq_head);
          const uint32_t al = ld_relaxed(&w.sync->rq_alloc);
          if (h < al) {
            const uint32_t m = min(al - h, (uint32_t)SIDE_TOK);
            if (atomicCAS(&w.sync->rq_head, h, h + m) == h) { act = S_COMBINE; arg = (int)h; n = (int)m; }
            else act = S_RETRY;
          }
        }
      }
      // Idle for long stretches is normal (no band completes during GEMM1); the
      // producers' own waits are bounded, so their exit ends this loop.  The limit
      // here is a backstop only.
      if (act == S_IDLE) {
        const uint64_t now = globaltimer();
        if (idle_since == 0) idle_since = now;
        else if (now - idle_since > 4 * a.timeout_ns) { set_error(w.status, W_SIDE_IDLE); act = S_EXIT; }
      } else if (act != S_RETRY) {
        idle_since = 0;
        nap = 64;
      }
    }
    act = __shfl_sync(0xffffffffu, act, 0);
    arg = __shfl_sync(0xffffffffu, arg, 0);
    n = __shfl_sync(0xffffffffu, n, 0);
    if (act == S_EXIT) break;
    if (act == S_RETRY) continue;
    if (act == S_IDLE) {
      if (lane == 0) {
        __nanosleep(nap);
        if (nap < 2048) nap <<= 1;
      }
      __syncwarp();
      continue;
    }
    if (act == S_BAND) {
      __threadfence();   // the publishing thread's acquire of the band's tiles comes first
      band_arrivals(a, arg, lane, 32);
      __syncwarp();
      continue;
    }
    // S_COMBINE: queue entries [arg, arg + n), allocated, so written soon if not yet;
    // a token not reached before the producers are done is left to the combine pass
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      if (i > 0 && *vl == 0) break;
      uint32_t* q = &w.ready_q[arg + i];
      int got = 1;
      if (lane == 0) {
        uint32_t v = ld_acquire(q);
        const uint64_t deadline = globaltimer() + a.timeout_ns;
        while (v == 0u) {
          if (*abort) { got = 0; break; }
          if (globaltimer() > deadline) { set_error(w.status, W_SIDE_QUEUE); got = 0; break; }
          __nanosleep(32);
          v = ld_acquire(q);
        }
      }
      ok = __shfl_sync(0xffffffffu, got, 0) != 0;
      if (!ok) break;
      const int t = (int)ld_acquire(q) - 1;   // every lane: the token's rows are stored before
      if (a.k <= 4) combine_token_warp_u<4, 3>(a.y, w.row_of, a.gate, t, a.d, a.k, a.out, lane);
      else combine_token_warp_u<MAX_K, 2>(a.y, w.row_of, a.gate, t, a.d, a.k, a.out, lane);
      __syncwarp();
      if (lane == 0) atomicOr(&w.arrive[t], TOKEN_DONE);
    }
    if (!ok) break;
  }
}

// ------------------------------------------------------------- EP return ---
// The consumer role of an expert-parallel owner: the return all-to-all of "Fine-
// grained Computation-Communication Overlap via Tile-level Signaling and
// Scheduling for Mixture-of-Experts", fused into the persistent kernel
// (Sections 3.3.2-3.3.3).  A consuming CTA takes the next segment item (mgb row
// bands; the first and last items one band each) by ticket, waits (bounded) until
// every band of it is flagged, and moves each band -- its rows are contiguous on
// both sides -- into its home rank's return buffer at the combine plan's row,
// with 16-byte loads and stores (no TMA, no loads from the home's memory).  It
// then fences at system scope and adds 1 to the home's arrival word of each row's
// token with a system-scope release, so the home can combine a token as soon as
// its k rows have landed.  Unlike the one-GPU combine, consumers keep going until
// every item is returned: nothing is left for a later pass.
__device__ void role_return(const FfnArgs& a, SmemCtl* ctl, int nb, int n_items,
                            const volatile uint32_t* abort) {
  const Work& w = a.w;
  const uint32_t NT2 = (uint32_t)(a.d / BN2);
  const int dv = a.d >> 3;
  const int k = a.k;
  constexpr int U = 4;   // 16-byte vectors in flight per thread
  while (true) {
    if (threadIdx.x == 0) {
      int act = C_DONE, b0 = 0, b1 = 0;
      if (*abort) act = C_ERROR;
      else {
        const int t = (int)atomicAdd(&w.sync->qc, 1u);
        if (t < n_items) {
          item_range(t, nb, a.mgb, b0, b1);
          bool ok = true;
          for (int b = b0; b < b1 && ok; ++b)
            ok = wait_count(&w.band_done2[b], BAND_UNIT * NT2, a.timeout_ns, abort);
          if (ok) act = C_BAND;
          else { set_error(w.status, W_CONS_QUEUE); act = C_ERROR; }
        }
      }
      ctl->item = act;
      ctl->ok = b0;
      ctl->cn = b1;
    }
    __syncthreads();
    const int act = ctl->item, b0 = ctl->ok, b1 = ctl->cn;
    __syncthreads();
    if (act != C_BAND) break;
    for (int b = b0; b < b1; ++b) {
      const Band bd = w.bands[b];
      const int2 dst = w.band_dest[b];
      const uint4* src = reinterpret_cast<const uint4*>(a.y) + (size_t)bd.row0 * dv;
      uint4* home = reinterpret_cast<uint4*>(a.ep_home_y[dst.x]) + (size_t)dst.y * dv;
      const size_t n = (size_t)bd.rows * dv;
      for (size_t i0 = threadIdx.x; i0 < n; i0 += (size_t)blockDim.x * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const size_t i = i0 + (size_t)u * blockDim.x;
          if (i < n) v[u] = __ldcg(src + i);   // y rows were stored by other SMs: read through L2
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const size_t i = i0 + (size_t)u * blockDim.x;
          if (i < n) home[i] = v[u];
        }
      }
    }
    __threadfence_system();   // the rows reach the home before any arrival below
    __syncthreads();
    for (int b = b0; b < b1; ++b) {
      const Band bd = w.bands[b];
      uint32_t* arrive = a.ep_home_arrive[w.band_dest[b].x];
      for (int r = threadIdx.x; r < bd.rows; r += (int)blockDim.x)
        red_release_sys_add(&arrive[a.ep_slot[bd.row0 + r] / k], 1u);
    }
    if (threadIdx.x == 0 && (a.flags & MOE_DBG_TIMESTAMPS) && blockIdx.x < STAMP_CTAS)
      w.stamps[(size_t)blockIdx.x * NSTAMP + 6] += (unsigned long long)(b1 - b0);
    __syncthreads();
  }
}

// ------------------------------------------------------------------- kernel ---
// XW: extra warps, 0 or 2: they copy GEMM1's A rows from x (a.gather == 2,
// MOE_SCHED_GATHER_LSU) or are side combine warps (a.side).
template <int V, int XW>
__global__ void __launch_bounds__(FFN_THREADS + 32 * XW, 1)
ffn_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_w1,
           const __grid_constant__ CUtensorMap tm_w3, const __grid_constant__ CUtensorMap tm_a2,
           const __grid_constant__ CUtensorMap tm_w2, const FfnArgs a) {
  constexpr int GW0 = FFN_THREADS / 32;         // first extra warp
  const int GW = (XW > 0 && a.gather == 2) ? XW : 0;   // gather warps
  const bool side = XW > 0 && a.side != 0 && a.gather != 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + (size_t)STAGE_AREA);
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int CTAS = Cfg<V>::CTAS;
  const uint32_t rank = V == 2 ? cluster_ctarank() : 0u;

  // prologue (touches nothing the previous kernel writes): barriers, TMEM, descriptors
  if (threadIdx.x == 0) {
    // a stage is full after the TMA thread's expected bytes and, with gather warps, one
    // arrival per gather thread
    for (int i = 0; i < MAX_NST; ++i) { mbar_init(&ctl->full[i], 1 + 32 * GW); mbar_init(&ctl->empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&ctl->tfull[i], 1); mbar_init(&ctl->tempty[i], EPI_WARPS * CTAS); }
    for (int i = 0; i < SCHED_DEPTH; ++i) {
      mbar_init(&ctl->sfull[i], 1);
      // MMA + epilogue (+ gather warps); a pair adds the peer's TMA + epilogue
      mbar_init(&ctl->sempty[i], (1 + EPI_WARPS + GW) * CTAS);
    }
    mbar_init(&ctl->epi_done[0], EPI_WARPS);
    mbar_init(&ctl->epi_done[1], EPI_WARPS);
    mbar_init(&ctl->mma_done, 1);
    mbar_init(&ctl->gbar[0], 1);
    mbar_init(&ctl->gbar[1], 1);
    for (int i = 0; i < CONS_SLOTS; ++i) { mbar_init(&ctl->cfull[i], 1); mbar_init(&ctl->cempty[i], (int)(blockDim.x / 32) - 1); }
    ctl->bhead = 0;
    ctl->btail = 0;
    ctl->prod_left = GW0;
    mbar_fence_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a1); tma_prefetch_desc(&tm_w1); tma_prefetch_desc(&tm_w3);
    tma_prefetch_desc(&tm_a2); tma_prefetch_desc(&tm_w2);
  }
  if (warp == 1) {
    if (V != 2) tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    else tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
    tc_fence_before();
  }
  __syncthreads();
  if (V == 2) cluster_sync();   // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  pdl_wait();   // the plan and the operands of the previous kernels are complete from here on
  Status* st = a.w.status;
  const volatile uint32_t* abort = &st->code;
  const int n1 = st->n_tiles1, n2 = st->n_tiles2, nb = st->n_bands, n_items = st->n_items;
  // consumer CTAs come in whole tiles' CTAs (the plan rounds C to a multiple of cg).
  // With GEMM2 tiles interleaved (MOE_SCHED_INTERLEAVE), bands complete from early
  // on, so the consumers are a partition of their own from the start (the paper's
  // disjoint SM subsets); otherwise no band completes before the GEMM1 queue
  // drains, and the consumers help with GEMM1 until then.
  const bool consumer_cta = (a.phase & PH_CONS) && (int)blockIdx.x < st->consumer_sms;
  const bool interleaved = (a.phase & PH_G1) && (a.phase & PH_G2) && (a.flags & MOE_SCHED_INTERLEAVE);
  const bool run_g1 = (a.phase & PH_G1) && !(consumer_cta && interleaved);
  const bool run_g2 = (a.phase & PH_G2) && !consumer_cta;
  const bool do_consume = (a.phase & PH_CONS) && (consumer_cta || a.join);
  const bool stamp = (a.flags & MOE_DBG_TIMESTAMPS) && blockIdx.x < STAMP_CTAS;
  unsigned long long* my_stamps = a.w.stamps + (size_t)blockIdx.x * NSTAMP;
  if (stamp && threadIdx.x == 0) {
    my_stamps[0] = globaltimer();
    for (int i = 1; i < NSTAMP; ++i) my_stamps[i] = 0;
    my_stamps[7] = rank;
  }
  __syncthreads();

  if (run_g1 || run_g2) {
    if (warp == 0) {
      bool warp_wide = false;
      if constexpr (V != 2) {
        if (a.gather == 1) {
          role_tma_gathered<V>(&tm_a1, &tm_w1, &tm_w3, &tm_a2, &tm_w2, a, ctl, smem, run_g1, run_g2, n1,
                               n2, abort);
          warp_wide = true;
        }
      }
      if (!warp_wide && lane == 0)
        role_tma<V>(&tm_a1, &tm_w1, &tm_w3, &tm_a2, &tm_w2, a, ctl, smem, rank, run_g1, run_g2, n1, n2,
                    abort);
    } else if (warp == 1) {
      if (lane == 0 && rank == 0) role_mma<V>(a, ctl, smem, tmem_base, abort);
    } else if (warp < GW0) {
      role_epilogue<V>(a, ctl, tmem_base, rank, warp, lane, abort);
    } else if constexpr (XW > 0 && V != 2) {
      if (GW > 0) role_gather_lsu<V, XW>(a, ctl, smem, warp - GW0, lane, abort);
      else if (side) role_side(a, ctl, lane, abort);
    }
    __syncwarp();
    if (side && warp < GW0 && lane == 0) {
      __threadfence_block();   // this warp's ring entries before its exit
      atomicSub(&ctl->prod_left, 1);
    }
  }
  __syncthreads();
  if (stamp && threadIdx.x == 0) my_stamps[2] = globaltimer();
  if (threadIdx.x == 0 && (a.phase & PH_CONS)) atomicAdd(&a.w.sync->prod_done, 1u);
  // A pair's peer may still be read by the leader's MMAs until the leader is
  // done; nobody reuses the operand ring before both CTAs finished producing.
  if (V == 2) cluster_sync();
  if (do_consume) {
    if (a.ep) role_return(a, ctl, nb, n_items, abort);
    else role_consumer(a, ctl, smem, nb, n_items, abort);
  }
  __syncthreads();
  if (stamp && threadIdx.x == 0) my_stamps[3] = globaltimer();
  if (V == 2) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (V != 2) tmem_dealloc(tmem_base, TMEM_COLS);
    else tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------- launch ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 tensor of `rank` dims (innermost first), box of 64 x rows (x 1), 128-B swizzle.
// bf16, rank 2 or 3: box `inner` x `box_rows` (x 1); the swizzle spans the box's
// inner bytes (128 or 64).
static bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                   const cuuint64_t* strides_bytes, cuuint32_t inner, cuuint32_t box_rows) {
  EncodeTiledFn fn = get_encode();
  if (!fn) return false;
  cuuint32_t box[3] = {inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = inner * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
            strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 weights as 4-D {64, K, atoms, E}: box 64 x `bk` x `atoms` x 1, 128-B swizzle.
static bool encode4(CUtensorMap* m, const void* base, const cuuint64_t* dims,
                    const cuuint64_t* strides_bytes, cuuint32_t bk, cuuint32_t atoms) {
  EncodeTiledFn fn = get_encode();
  if (!fn) return false;
  cuuint32_t box[4] = {64, bk, atoms, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides_bytes,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
constexpr int MAX_DEV = 64;
constexpr int XW_WARPS = 2;   // extra warps: gather (MOE_SCHED_GATHER_LSU) or side combine
// index of (V, with extra warps): 0-2 plain V = 1..3, 3 V = 1 + XW, 4 V = 3 + XW
int g_configured[5][MAX_DEV] = {{0}};
int g_grid[5][MAX_DEV] = {{0}};

inline int kernel_slot(int V, int gw) { return gw ? (V == 1 ? 3 : 4) : V - 1; }

template <int V, int GW>
cudaError_t configure(int dev) {
  if (dev < 0 || dev >= MAX_DEV) return cudaErrorInvalidDevice;
  const int ks = kernel_slot(V, GW);
  if (g_configured[ks][dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(ffn_kernel<V, GW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ffn_smem_bytes());
  if (e != cudaSuccess) return e;
  int nsm = 0;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  int grid = nsm;
  if (V == 2) {
    // as many CTA pairs as can be resident at once (one CTA per SM)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nsm & ~1));
    cfg.blockDim = dim3(FFN_THREADS);
    cfg.dynamicSmemBytes = ffn_smem_bytes();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, ffn_kernel<2, 0>, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    grid = 2 * min(clusters, nsm / 2);
  }
  g_grid[ks][dev] = grid;
  g_configured[ks][dev] = 1;
  return cudaSuccess;
}

cudaError_t configure_variant(int V, int gw, int dev) {
  if (gw) {
    if (V == 1) return configure<1, XW_WARPS>(dev);
    if (V == 3) return configure<3, XW_WARPS>(dev);
    return cudaErrorInvalidValue;   // CTA pairs have no extra-warp kernel
  }
  switch (V) {
    case 1: return configure<1, 0>(dev);
    case 2: return configure<2, 0>(dev);
    case 3: return configure<3, 0>(dev);
  }
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t ffn_grid(int V, int* grid) {
  *grid = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = configure_variant(V, 0, dev);
  if (e != cudaSuccess) return e;
  *grid = g_grid[kernel_slot(V, 0)][dev];
  return cudaSuccess;
}

cudaError_t launch_ffn(const FfnArgs& a, int grid, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int gw = (a.gather == 2 || a.side) ? XW_WARPS : 0;
  if (gw && a.V == 2) return cudaErrorInvalidValue;   // CTA pairs have no extra-warp kernel
  e = configure_variant(a.V, gw, dev);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_a1, tm_w1, tm_w3, tm_a2, tm_w2;
  const cuuint64_t R = (cuuint64_t)a.R, d = (cuuint64_t)a.d, f = (cuuint64_t)a.f, E = (cuuint64_t)a.E;
  // K elements per stage of this variant: the A boxes' inner extent (and swizzle
  // span) and the weight boxes' K rows
  const cuuint32_t bk = a.V == 3 ? Cfg<3>::BK : a.V == 2 ? Cfg<2>::BK : Cfg<1>::BK;
  if (a.gather == 1) {
    // token rows of x, boxes one row high for gather4
    const cuuint64_t dims[2] = {d, (cuuint64_t)a.T}, st[1] = {d * 2};
    if (!encode(&tm_a1, a.x, 2, dims, st, bk, 1)) return cudaErrorInvalidValue;
  } else {
    const cuuint64_t dims[2] = {d, R}, st[1] = {d * 2};
    if (!encode(&tm_a1, a.x_perm, 2, dims, st, bk, BM)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {f, R}, st[1] = {f * 2};
    if (!encode(&tm_a2, a.h, 2, dims, st, bk, BM)) return cudaErrorInvalidValue;
  }
  // Single CTAs (V = 1, 3) read the weights through 4-D maps {64 columns, K,
  // 64-column atom, expert} with the atom stride 128 B, so that one box holds
  // all the atoms of the CTA's tile, atom after atom: 2-3 copies per k-block
  // instead of 5 (measured faster).  CTA pairs take 2 atoms per CTA and per operand through
  // the 3-D maps {columns, K, expert}, one box per atom (a 4-D copy there
  // measured slower), as do single CTAs if the driver refuses the 4-D maps.
  FfnArgs args = a;
  args.b_atoms = 0;
  if (a.V != 2 && !(a.flags & MOE_SCHED_B_PER_ATOM)) {
    const cuuint64_t d1[4] = {64, d, f / 64, E}, s1[3] = {f * 2, 128, d * f * 2};
    const cuuint64_t d2[4] = {64, f, d / 64, E}, s2[3] = {d * 2, 128, f * d * 2};
    args.b_atoms = encode4(&tm_w1, a.W1, d1, s1, bk, 2) && encode4(&tm_w3, a.W3, d1, s1, bk, 2) &&
                   encode4(&tm_w2, a.W2, d2, s2, bk, 4);
  }
  if (!args.b_atoms) {
    const cuuint64_t dims[3] = {f, d, E}, st[2] = {f * 2, d * f * 2};
    if (!encode(&tm_w1, a.W1, 3, dims, st, 64, bk)) return cudaErrorInvalidValue;
    if (!encode(&tm_w3, a.W3, 3, dims, st, 64, bk)) return cudaErrorInvalidValue;
    const cuuint64_t dims2[3] = {d, f, E}, st2[2] = {d * 2, f * d * 2};
    if (!encode(&tm_w2, a.W2, 3, dims2, st2, 64, bk)) return cudaErrorInvalidValue;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(FFN_THREADS + 32 * gw);
  cfg.dynamicSmemBytes = ffn_smem_bytes();
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  if (a.V == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // launch overlaps the previous kernel's tail; the kernel waits before its plan reads
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  } else {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.numAttrs = 1;
  }
  cfg.attrs = attr;
  if (gw) {
    if (a.V == 3) return cudaLaunchKernelEx(&cfg, ffn_kernel<3, XW_WARPS>, tm_a1, tm_w1, tm_w3, tm_a2, tm_w2, args);
    return cudaLaunchKernelEx(&cfg, ffn_kernel<1, XW_WARPS>, tm_a1, tm_w1, tm_w3, tm_a2, tm_w2, args);
  }
  if (a.V == 2) return cudaLaunchKernelEx(&cfg, ffn_kernel<2, 0>, tm_a1, tm_w1, tm_w3, tm_a2, tm_w2, args);
  if (a.V == 3) return cudaLaunchKernelEx(&cfg, ffn_kernel<3, 0>, tm_a1, tm_w1, tm_w3, tm_a2, tm_w2, args);
  return cudaLaunchKernelEx(&cfg, ffn_kernel<1, 0>, tm_a1, tm_w1, tm_w3, tm_a2, tm_w2, args);
}

}  // namespace moe
