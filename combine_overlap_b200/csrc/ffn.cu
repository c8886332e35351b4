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
//   * one launch of one CTA per SM (cooperative launch: all CTAs co-resident),
//     each CTA taking tiles from an atomic work queue in priority order instead
//     of a fixed stride;
//   * per CTA: warp 0 = tile scheduler + TMA producer, warp 1 = TMEM allocator
//     + single-thread tcgen05.mma issuer, warps 2-5 = epilogue (TMEM -> registers
//     -> bf16 -> global), 4-stage smem ring, two 256-column TMEM accumulators so
//     the epilogue of one tile overlaps the main loop of the next;
//   * GEMM1 tile: 128 rows x 128 h-columns; one N=256 MMA accumulates x*W1 and
//     x*W3 side by side (the B tile holds the W1 and W3 column blocks), and the
//     epilogue applies silu(a)*b;  GEMM2 tile: 128 rows x 256 y-columns;
//   * A (x_perm or h) is K-major, W is stored [K][N] (N-major): both are read
//     by TMA with 128-byte swizzle and fed to tcgen05 as K-major / MN-major
//     operands, so the weights need no repacking;
//   * signals are counters per row band (GEMM1 tiles done, GEMM2 tiles done)
//     published with red.release and polled with ld.acquire; every wait is
//     bounded and reports MOE_ERR_TIMEOUT through the status block.
#include "kernels.h"
#include "combine.cuh"
#include "../../include/moe.h"

#include <cuda.h>

namespace moe {

enum : int { K_END = 0, K_G1 = 1, K_G2 = 2 };

constexpr int CONS_SLOTS = 16;   // at most this many tokens in flight per consumer CTA

struct Item {
  int kind, band, nt, expert, row0, rows, pad0, pad1;
};

struct SmemCtl {
  uint64_t full[NSTAGE];
  uint64_t empty[NSTAGE];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t sfull[SCHED_DEPTH];
  uint64_t sempty[SCHED_DEPTH];
  uint64_t epi_done[2];   // per accumulator: the four epilogue warps stored the tile
  uint64_t mma_done;
  uint64_t cfull[CONS_SLOTS];    // consumer ring: a token's k expert rows landed in the slot
  uint64_t cempty[CONS_SLOTS];   // consumer ring: the slot's token is reduced and stored
  Item ring[SCHED_DEPTH];
  uint32_t tmem_base;
  int item;
  int ok;
  int cn;                        // tokens completed by the current band
  int ctok[BM];                  // ... and which
};

size_t ffn_smem_bytes() { return 1024 + (size_t)NSTAGE * STAGE_BYTES + sizeof(SmemCtl); }

__device__ __forceinline__ void set_error(Status* st, uint32_t where) {
  if (atomicCAS(&st->code, (uint32_t)ST_OK, (uint32_t)ST_TIMEOUT) == (uint32_t)ST_OK) {
    st->where = where;
  }
}

// Bounded mbarrier wait; `abort` (may be null) ends it early once any CTA has
// recorded an error.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                         const volatile uint32_t* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = globaltimer() + timeout_ns;
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
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

__device__ __forceinline__ Item make_item(int kind, int band, int nt, const Band& bd) {
  Item it;
  it.kind = kind;
  it.band = band;
  it.nt = nt;
  it.expert = bd.expert;
  it.row0 = bd.row0;
  it.rows = bd.rows;
  it.pad0 = it.pad1 = 0;
  return it;
}

// GEMM1 tile t: experts in priority order; inside an expert, column-block major
// (all row bands of one 128-column block of W1/W3, then the next), so the
// weights slice in use stays in L2 while every band of the expert reads it.
__device__ Item decode_g1(const Work& w, int t, int E) {
  int lo = 0, hi = E;  // tile_start1[lo] <= t < tile_start1[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (w.tile_start1[mid] <= t) lo = mid; else hi = mid;
  }
  const int b0 = w.band_start[lo];
  const int nbe = w.band_start[lo + 1] - b0;
  const int local = t - w.tile_start1[lo];
  const int band = b0 + local % nbe;
  return make_item(K_G1, band, local / nbe, w.bands[band]);
}

// GEMM2 tile t: band-major (all column blocks of a band, then the next band), so
// bands complete -- and can be combined -- in priority order.
__device__ Item decode_g2(const Work& w, int t, int NT2) {
  const int band = t / NT2;
  return make_item(K_G2, band, t % NT2, w.bands[band]);
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

// ------------------------------------------------------------ TMA producer ---
__device__ void role_tma(const CUtensorMap* tm_a1, const CUtensorMap* tm_w1,
                         const CUtensorMap* tm_w3, const CUtensorMap* tm_a2,
                         const CUtensorMap* tm_w2, const FfnArgs& a, SmemCtl* ctl,
                         uint8_t* smem, bool run_g1, bool run_g2, int n1, int n2,
                         const volatile uint32_t* abort) {
  const Work& w = a.w;
  const int NT1 = a.f / BN1, NT2 = a.d / BN2;
  const uint64_t tmo = a.timeout_ns;
  int stage = 0, slot = 0;
  uint32_t ph = 0, sph = 0;
  uint32_t pending = 0, pend_par = 0;   // stages with an issued fill, and its parity
  bool g1 = run_g1, g2 = run_g2;
  while (true) {
    Item it;
    it.kind = K_END;
    if (*abort) g1 = g2 = false;
    if (g1) {
      const int t = (int)atomicAdd(&w.sync->q1, 1u);
      if (t < n1) it = decode_g1(w, t, a.E); else g1 = false;
    }
    if (it.kind == K_END && g2) {
      const int t = (int)atomicAdd(&w.sync->q2, 1u);
      if (t < n2) it = decode_g2(w, t, NT2); else g2 = false;
    }
    if (!wait_bar(&ctl->sempty[slot], sph ^ 1u, tmo, abort)) { set_error(w.status, W_SCHED_EMPTY); break; }
    ctl->ring[slot] = it;
    mbar_arrive(&ctl->sfull[slot]);
    if (++slot == SCHED_DEPTH) { slot = 0; sph ^= 1u; }
    if (it.kind == K_END) break;
    const bool is1 = it.kind == K_G1;
    if (!is1) {
      // GEMM2 reads h rows of this band: every GEMM1 column block must be stored.
      if (!wait_count(&w.band_done1[it.band], (uint32_t)NT1, tmo, abort)) {
        set_error(w.status, W_BAND1);
        break;
      }
      fence_proxy_async_global();  // generic-proxy stores -> async-proxy (TMA) loads
    }
    const int nk = (is1 ? a.d : a.f) / BK;
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      if (!wait_bar(&ctl->empty[stage], ph ^ 1u, tmo, abort)) { set_error(w.status, W_STAGE_EMPTY); ok = false; break; }
      uint8_t* sa = smem + (size_t)stage * STAGE_BYTES;
      uint8_t* sb = sa + A_STAGE_BYTES;
      uint64_t* fb = &ctl->full[stage];
      mbar_arrive_expect_tx(fb, STAGE_BYTES);
      if (is1) {
        tma_load_2d(sa, tm_a1, fb, kb * BK, it.row0);
        tma_load_3d(sb, tm_w1, fb, it.nt * BN1, kb * BK, it.expert);
        tma_load_3d(sb + B_BOX_BYTES, tm_w1, fb, it.nt * BN1 + 64, kb * BK, it.expert);
        tma_load_3d(sb + 2 * B_BOX_BYTES, tm_w3, fb, it.nt * BN1, kb * BK, it.expert);
        tma_load_3d(sb + 3 * B_BOX_BYTES, tm_w3, fb, it.nt * BN1 + 64, kb * BK, it.expert);
      } else {
        tma_load_2d(sa, tm_a2, fb, kb * BK, it.row0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_3d(sb + q * B_BOX_BYTES, tm_w2, fb, it.nt * BN2 + q * 64, kb * BK, it.expert);
      }
      pending |= 1u << stage;
      pend_par = (pend_par & ~(1u << stage)) | (ph << stage);
      if (++stage == NSTAGE) { stage = 0; ph ^= 1u; }
    }
    if (!ok) break;
  }
  // Never leave with a copy still landing in shared memory.
  for (int s = 0; s < NSTAGE; ++s)
    if (pending & (1u << s)) wait_bar(&ctl->full[s], (pend_par >> s) & 1u, tmo, nullptr);
}

// --------------------------------------------------------------- MMA issuer ---
__device__ void role_mma(const FfnArgs& a, SmemCtl* ctl, uint8_t* smem, uint32_t tmem_base,
                         const volatile uint32_t* abort) {
  const uint64_t tmo = a.timeout_ns;
  constexpr uint32_t idesc = idesc_bf16_f32(BM, 256, true);
  int stage = 0, slot = 0, acc = 0;
  uint32_t ph = 0, sph = 0, aph = 0;
  while (true) {
    if (!wait_bar(&ctl->sfull[slot], sph, tmo, abort)) { set_error(a.w.status, W_SCHED_FULL); break; }
    const Item it = ctl->ring[slot];
    mbar_arrive(&ctl->sempty[slot]);
    if (++slot == SCHED_DEPTH) { slot = 0; sph ^= 1u; }
    if (it.kind == K_END) break;
    if (!wait_bar(&ctl->tempty[acc], aph ^ 1u, tmo, abort)) { set_error(a.w.status, W_TMEM_EMPTY); break; }
    tc_fence_after();
    const uint32_t dt = tmem_base + (uint32_t)(acc * ACC_COLS);
    const int nk = (it.kind == K_G1 ? a.d : a.f) / BK;
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      if (!wait_bar(&ctl->full[stage], ph, tmo, abort)) { set_error(a.w.status, W_STAGE_FULL); ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)stage * STAGE_BYTES);
      const uint32_t sb = sa + A_STAGE_BYTES;
#pragma unroll
      for (int ks = 0; ks < BK / 16; ++ks) {
        const uint64_t ad = smem_desc_sw128(sa + ks * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(sb + ks * 2048, B_BOX_BYTES, 1024);
        tc_mma_f16(dt, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
      }
      tc_commit(&ctl->empty[stage]);  // frees the smem stage once these MMAs finish
      if (++stage == NSTAGE) { stage = 0; ph ^= 1u; }
    }
    if (!ok) break;
    tc_commit(&ctl->tfull[acc]);      // accumulator ready for the epilogue
    acc ^= 1;
    if (acc == 0) aph ^= 1u;
  }
  // Wait for every MMA this thread issued before TMEM can be released.
  tc_commit(&ctl->mma_done);
  wait_bar(&ctl->mma_done, 0u, tmo, nullptr);
}

// ----------------------------------------------------------------- epilogue ---
__device__ void role_epilogue(const FfnArgs& a, SmemCtl* ctl, uint32_t tmem_base, int warp,
                              int lane, const volatile uint32_t* abort) {
  const Work& w = a.w;
  const uint64_t tmo = a.timeout_ns;
  const int q = warp & 3;                 // TMEM lane quadrant this warp may read
  const int row = q * 32 + lane;
  int slot = 0, acc = 0;
  uint32_t sph = 0, aph = 0, eph = 0;   // eph: one parity bit per accumulator
  while (true) {
    // Every lane waits; the warp proceeds only if all lanes saw the phase, so a
    // timeout never splits the warp before the .sync.aligned TMEM loads.
    bool ok = __all_sync(0xffffffffu, wait_bar(&ctl->sfull[slot], sph, tmo, abort));
    if (!ok) { if (lane == 0) set_error(w.status, W_SCHED_FULL); break; }
    const Item it = ctl->ring[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->sempty[slot]);
    if (++slot == SCHED_DEPTH) { slot = 0; sph ^= 1u; }
    if (it.kind == K_END) break;
    ok = __all_sync(0xffffffffu, wait_bar(&ctl->tfull[acc], aph, tmo, abort));
    if (!ok) { if (lane == 0) set_error(w.status, W_TMEM_FULL); break; }
    tc_fence_after();
    const uint32_t tb = tmem_base + (uint32_t)(acc * ACC_COLS) + ((uint32_t)(q * 32) << 16);
    const bool valid = row < it.rows;
    if (it.kind == K_G1) {
      uint4* dst = reinterpret_cast<uint4*>(a.h + (size_t)(it.row0 + row) * a.f + it.nt * BN1);
#pragma unroll 1
      for (int c = 0; c < BN1 / 32; ++c) {
        uint32_t ra[32], rb[32];
        tmem_ld32(tb + c * 32, ra);
        tmem_ld32(tb + BN1 + c * 32, rb);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(silu_mul(__uint_as_float(ra[2 * i]), __uint_as_float(rb[2 * i])),
                              silu_mul(__uint_as_float(ra[2 * i + 1]), __uint_as_float(rb[2 * i + 1])));
        if (valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      fence_proxy_async_global();   // h is read back by TMA in other CTAs
    } else {
      uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)(it.row0 + row) * a.d + it.nt * BN2);
#pragma unroll 1
      for (int c = 0; c < BN2 / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tb + c * 32, r);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        if (valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    const int my_acc = acc;
    if (lane == 0) {
      mbar_arrive(&ctl->tempty[my_acc]);    // accumulator may be overwritten
      mbar_arrive(&ctl->epi_done[my_acc]);  // this warp's rows of the tile are stored
    }
    acc ^= 1;
    if (acc == 0) aph ^= 1u;
    // Publish the tile: one thread waits (bounded) for all four epilogue warps'
    // stores of this tile, then fences and bumps the band's counter with release
    // semantics.  A warp can run at most one tile ahead, and consecutive tiles
    // use different accumulators, so each epi_done phase holds one tile's
    // arrivals only.
    if (warp == 2 && lane == 0) {
      const bool stored = wait_bar(&ctl->epi_done[my_acc], (eph >> my_acc) & 1u, tmo, abort);
      const bool skip = (a.flags & MOE_DBG_SKIP_FLAG_BAND) && it.kind == K_G2 && it.band == 0;
      if (!stored) set_error(w.status, W_DRAIN);
      else if (!skip) {
        __threadfence();
        red_release_add(it.kind == K_G1 ? &w.band_done1[it.band] : &w.band_done2[it.band], 1u);
      }
    }
    eph ^= 1u << my_acc;
    __syncwarp();
  }
}

// ----------------------------------------------------------------- consumer ---
// All CTAs that consume take combine items (row bands in priority order) from a
// shared atomic counter.  For a ready band:
//   1. every thread takes one row of the band and bumps its token's arrival
//      counter (acq_rel); the thread that brings it to k records the token, whose
//      k expert rows are now all stored (published by the earlier arrivals);
//   2. thread 0 streams each recorded token's k rows of y into a ring of shared-
//      memory slots with cp.async.bulk (the GEMM staging buffers are idle by
//      now), so up to CONS_SLOTS tokens' rows are in flight per SM;
//   3. warps 1-5 reduce a slot in fp32, slot order, and store out[t] with 16-byte
//      stores -- the same arithmetic as combine_token_warp, so both modes agree
//      bit for bit.  Each slot has one owning warp (see below).
// If one token's rows do not fit the staging area, the warps fall back to
// combine_token_warp straight from global memory.
__device__ void role_consumer(const FfnArgs& a, SmemCtl* ctl, uint8_t* smem, int nb, int n_items,
                              const volatile uint32_t* abort) {
  const Work& w = a.w;
  const int NT2 = a.d / BN2;
  const int k = a.k, d = a.d, dv = d >> 3;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NWARPS = FFN_THREADS / 32;
  constexpr int NCW = NWARPS - 1;                         // reducing warps
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const uint32_t tok_bytes = row_bytes * (uint32_t)k;
  int S = (int)((size_t)NSTAGE * STAGE_BYTES / tok_bytes);
  if (S > CONS_SLOTS) S = CONS_SLOTS;
  if (S > NCW) S -= S % NCW;   // slots split evenly over the reducing warps
  uint32_t base = 0;                                      // tokens this CTA reduced so far
  uint32_t pend = 0, pend_par = 0;                        // issuer: slots with a copy issued
  while (true) {
    if (threadIdx.x == 0) ctl->item = *abort ? -1 : (int)atomicAdd(&w.sync->qc, 1u);
    __syncthreads();
    const int item = ctl->item;
    if (item < 0 || item >= n_items) break;
    int b0, b1;
    item_range(item, nb, a.mgb, b0, b1);
    bool ok = true;
    for (int b = b0; b < b1; ++b) {
      if (threadIdx.x == 0) {
        const bool ready = wait_count(&w.band_done2[b], (uint32_t)NT2, a.timeout_ns, abort);
        if (!ready) set_error(w.status, W_BAND2);
        ctl->ok = ready ? 1 : 0;
        ctl->cn = 0;
      }
      __syncthreads();
      if (!ctl->ok) { ok = false; break; }
      const Band bd = w.bands[b];
      for (int r = threadIdx.x; r < bd.rows; r += FFN_THREADS) {
        const int t = w.perm[bd.row0 + r] / k;
        if (atom_acq_rel_add(&w.arrive[t], 1u) == (uint32_t)(k - 1)) ctl->ctok[atomicAdd(&ctl->cn, 1)] = t;
      }
      __syncthreads();
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
            const int t = ctl->ctok[i];
            uint8_t* dst = smem + (size_t)s * tok_bytes;
            mbar_arrive_expect_tx(&ctl->cfull[s], tok_bytes);
            for (int j = 0; j < k; ++j) {
              const int r = w.row_of[(size_t)t * k + j];
              bulk_load(dst + (size_t)j * row_bytes, a.y + (size_t)r * d, row_bytes, &ctl->cfull[s]);
            }
            pend |= 1u << s;
            pend_par = (pend_par & ~(1u << s)) | (ph << s);
          }
        }
      } else {
        // Slot s belongs to warp 1 + s % NCW alone, which takes that slot's tokens in
        // order, so it never waits on a slot's phase before the previous phase has
        // completed (an mbarrier parity wait cannot tell phases two apart).
        const int cw = warp - 1;
        for (int i = 0; i < n; ++i) {
          const uint32_t g = base + (uint32_t)i;
          const int s = (int)(g % (uint32_t)S);
          if (s % NCW != cw) continue;
          const uint32_t ph = (g / (uint32_t)S) & 1u;
          if (!__all_sync(0xffffffffu, wait_bar(&ctl->cfull[s], ph, a.timeout_ns, abort))) {
            if (lane == 0) set_error(w.status, W_CONS_FULL);
            break;
          }
          const int t = ctl->ctok[i];
          float gt[MAX_K];
#pragma unroll
          for (int j = 0; j < MAX_K; ++j) gt[j] = j < k ? a.gate[(size_t)t * k + j] : 0.0f;
          const uint4* src = reinterpret_cast<const uint4*>(smem + (size_t)s * tok_bytes);
          uint4* ov = reinterpret_cast<uint4*>(a.out) + (size_t)t * dv;
          for (int v = lane; v < dv; v += 32) {
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
    }
    if (!ok) break;
    __syncthreads();
  }
  // Never leave with a bulk copy still landing in shared memory.
  if (threadIdx.x == 0)
    for (int s = 0; s < S; ++s)
      if (pend & (1u << s)) wait_bar(&ctl->cfull[s], (pend_par >> s) & 1u, a.timeout_ns, nullptr);
}

// ------------------------------------------------------------------- kernel ---
__global__ void __launch_bounds__(FFN_THREADS, 1)
ffn_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_w1,
           const __grid_constant__ CUtensorMap tm_w3, const __grid_constant__ CUtensorMap tm_a2,
           const __grid_constant__ CUtensorMap tm_w2, const FfnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + (size_t)NSTAGE * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Status* st = a.w.status;
  const volatile uint32_t* abort = &st->code;
  const int n1 = st->n_tiles1, n2 = st->n_tiles2, nb = st->n_bands, n_items = st->n_items;
  const bool consumer_cta = (a.phase & PH_CONS) && (int)blockIdx.x < st->consumer_sms;
  const bool run_g1 = (a.phase & PH_G1) != 0;
  const bool run_g2 = (a.phase & PH_G2) && !consumer_cta;
  const bool do_consume = (a.phase & PH_CONS) && (consumer_cta || a.join);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) { mbar_init(&ctl->full[i], 1); mbar_init(&ctl->empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&ctl->tfull[i], 1); mbar_init(&ctl->tempty[i], 4); }
    for (int i = 0; i < SCHED_DEPTH; ++i) { mbar_init(&ctl->sfull[i], 1); mbar_init(&ctl->sempty[i], 5); }
    mbar_init(&ctl->epi_done[0], 4);
    mbar_init(&ctl->epi_done[1], 4);
    mbar_init(&ctl->mma_done, 1);
    for (int i = 0; i < CONS_SLOTS; ++i) { mbar_init(&ctl->cfull[i], 1); mbar_init(&ctl->cempty[i], 1); }
    mbar_fence_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a1); tma_prefetch_desc(&tm_w1); tma_prefetch_desc(&tm_w3);
    tma_prefetch_desc(&tm_a2); tma_prefetch_desc(&tm_w2);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  if (run_g1 || run_g2) {
    if (warp == 0) {
      if (lane == 0) role_tma(&tm_a1, &tm_w1, &tm_w3, &tm_a2, &tm_w2, a, ctl, smem, run_g1, run_g2, n1, n2, abort);
    } else if (warp == 1) {
      if (lane == 0) role_mma(a, ctl, smem, tmem_base, abort);
    } else {
      role_epilogue(a, ctl, tmem_base, warp, lane, abort);
    }
    __syncwarp();
  }
  __syncthreads();
  if (do_consume) role_consumer(a, ctl, smem, nb, n_items, abort);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
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
static bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                   const cuuint64_t* strides_bytes, cuuint32_t box_rows) {
  EncodeTiledFn fn = get_encode();
  if (!fn) return false;
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
            strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_ffn(const FfnArgs& a, int grid, cudaStream_t s) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = ffn_smem_bytes();
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  CUtensorMap tm_a1, tm_w1, tm_w3, tm_a2, tm_w2;
  const cuuint64_t R = (cuuint64_t)a.R, d = (cuuint64_t)a.d, f = (cuuint64_t)a.f, E = (cuuint64_t)a.E;
  {
    const cuuint64_t dims[2] = {d, R}, st[1] = {d * 2};
    if (!encode(&tm_a1, a.x_perm, 2, dims, st, BM)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {f, d, E}, st[2] = {f * 2, d * f * 2};
    if (!encode(&tm_w1, a.W1, 3, dims, st, 64)) return cudaErrorInvalidValue;
    if (!encode(&tm_w3, a.W3, 3, dims, st, 64)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {f, R}, st[1] = {f * 2};
    if (!encode(&tm_a2, a.h, 2, dims, st, BM)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {d, f, E}, st[2] = {d * 2, f * d * 2};
    if (!encode(&tm_w2, a.W2, 3, dims, st, 64)) return cudaErrorInvalidValue;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(FFN_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, ffn_kernel, tm_a1, tm_w1, tm_w3, tm_a2, tm_w2, a);
}

}  // namespace moe
