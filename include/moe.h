/*
 * moe.h -- C ABI of libmoe_b200.so: one Mixture-of-Experts layer on a B200
 * (sm_100a), with the gate-weighted combine overlapped with the expert GEMM at
 * tile granularity.
 *
 * The method is the one of "Fine-grained Computation-Communication Overlap via
 * Tile-level Signaling and Scheduling for Mixture-of-Experts" (arXiv 2607.19539)
 * on a single GPU: a persistent rank-wide expert GEMM (the producer, Section
 * 3.3.1) publishes a ready signal per output tile from its epilogue; a small
 * partition of SMs (the consumer, Sections 3.3.2-3.3.3) performs the return step
 * -- here the gate-weighted unpermute/combine back to token order, standing in
 * for the return all-to-all -- as tiles become ready.  The producer/consumer SM
 * split is chosen per call from the routing counts by a small cost model, as in
 * "Weave: Fine-Grained Dynamic SM Scheduling in an MoE Megakernel for
 * Compute-Communication Overlap" (arXiv 2609.21483), Abstract.
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless stated otherwise; the caller allocates
 *    and owns every buffer, including the workspace.  The library allocates no
 *    device memory.
 *  - bf16 = bfloat16 bit patterns (2 bytes); matrices are dense row-major.
 *    Every device pointer must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void*.  Calls are asynchronous on it
 *    and never synchronise the host, except moe_get_status.
 *  - Buffers must hold the sizes each entry point states: the library sees
 *    pointers only and cannot check them (the Python binding checks tensor
 *    shapes before calling).
 *  - Argument errors return at once, before any launch, with MOE_ERR_INVALID or
 *    MOE_ERR_UNSUPPORTED; a launch failure returns MOE_ERR_CUDA, and
 *    moe_last_cuda_error names the CUDA error behind it.  Errors found on the
 *    device (a bounded wait that ran out) are written to the status block in
 *    the workspace and read back by moe_get_status.  Kernels never trap and
 *    every wait inside them is bounded.
 *  - Preconditions: 1 <= T; 1 <= k <= min(E, 8); E <= 256; d % 256 == 0;
 *    f % 128 == 0; logits finite.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,      /* bad argument (null pointer, bad size, misaligned)    */
  MOE_ERR_UNSUPPORTED = 2,  /* valid MoE shape the library does not handle        */
  MOE_ERR_CUDA = 3,         /* a CUDA call failed                                  */
  MOE_ERR_TIMEOUT = 4,      /* a bounded device wait ran out (see moe_get_status)  */
  MOE_ERR_WORKSPACE = 5     /* workspace missing or smaller than moe_workspace_size */
} moe_status;

typedef enum {
  /* route -> permute -> GEMM1 (all SMs) -> GEMM2 (all SMs) -> combine, each a
   * separate launch: the conventional non-overlapped path (paper Section 4.1.3,
   * the baseline that runs expert compute and the return step one after the
   * other). */
  MOE_MODE_SEQUENTIAL = 0,
  /* route -> permute -> one persistent launch in which producer CTAs run the
   * GEMM tiles and consumer CTAs combine each row band as soon as its tiles are
   * flagged ready (paper Sections 3.3.1-3.3.3). */
  MOE_MODE_OVERLAPPED = 1
} moe_mode;

/* Debug flags (moe_layer_args.flags). */
#define MOE_DBG_SKIP_FLAG_BAND 0x1u  /* the producer never publishes that the first row
                                        band's GEMM1 tiles are stored, so the GEMM2 tile that
                                        reads those h rows waits until its bound runs out:
                                        exercises MOE_ERR_TIMEOUT without a GPU fault */
#define MOE_SCHED_NO_JOIN      0x2u  /* producer CTAs do not join the combine after the
                                        GEMM tile queue drains (dedicated consumers only) */
#define MOE_DBG_TIMESTAMPS     0x8u  /* the persistent kernel records per-CTA globaltimer
                                        stamps, read back with moe_debug_stamps */
#define MOE_SCHED_GATHER_A     0x10u /* GEMM1 gathers its A rows from x with TMA gather4
                                        (4 rows per instruction) instead of reading the
                                        permuted copy x_perm, which is then not written:
                                        single CTAs issue the gathers from all 32 lanes of
                                        the producer warp, CTA pairs from one thread */
#define MOE_SCHED_ONE_CTA      0x4u  /* force 128-row MMA tiles on single CTAs          */
#define MOE_SCHED_CTA_PAIR     0x20u /* force 256-row MMA tiles on CTA pairs (tcgen05
                                        cta_group::2); an expert's odd last row band runs
                                        as a 128-row half tile.  Without a tile flag the
                                        call picks 256-row tiles on single CTAs
                                        (MOE_SCHED_WIDE_CTA) when T*k/E >= 256, else
                                        128-row tiles (measured on B200).  ONE_CTA wins
                                        over CTA_PAIR, CTA_PAIR over WIDE_CTA */
#define MOE_SCHED_B_PER_ATOM   0x40u /* single-CTA tiles load each 64-column atom of the
                                        weight tiles with a TMA copy of its own (3-D maps),
                                        as CTA pairs always do, instead of one 4-D copy
                                        carrying all the atoms of the tile */
#define MOE_SCHED_FULL_TILES   0x80u /* CTA pairs run an expert's odd last row band as a
                                        full 256-row tile (half of it masked) instead of a
                                        128-row half tile (M=128 cta_group::2 MMA) */
#define MOE_DBG_IDENTITY_EXPERTS 0x200u /* every expert is the identity map (y = x_perm):
                                        the call runs route, permute and the combine only,
                                        in either mode, so out[t] = bf16(sum_j g_j x[t])
                                        checks those steps apart from the GEMMs; W1, W3
                                        and W2 are not read and may be NULL */
#define MOE_SCHED_INTERLEAVE   0x400u /* GEMM2 tiles interleave with GEMM1 tiles: a
                                        scheduler takes the next GEMM2 tile (in priority
                                        order) as soon as every GEMM1 tile of its row group
                                        is stored, and GEMM1 tiles otherwise, so row bands
                                        complete throughout the launch; dedicated consumer
                                        CTAs then skip GEMM1.  Default: every CTA takes
                                        GEMM1 tiles until that queue is empty before any
                                        GEMM2 tile.  Same bits */
#define MOE_SCHED_EXP_SILU     0x4000u /* GEMM1's epilogue computes silu(a) = a / (1 +
                                        exp(-a)) (two special-function ops per element)
                                        instead of the default a/2 (1 + tanh(a/2)) with the
                                        hardware tanh approximation (one op; other bits in
                                        h, within the same bound of the oracle) */
#define MOE_SCHED_GATHER_LSU   0x8000u /* single-CTA tiles: two extra warps copy GEMM1's
                                        A rows from x with 16-byte cp.async into the
                                        swizzled operand layout (x_perm is not written);
                                        the TMA loads the weights only.  Same bits.  With
                                        CTA pairs: MOE_ERR_UNSUPPORTED */
#define MOE_SCHED_SIDE_COMBINE 0x1000u /* overlapped mode, single-CTA tiles: two extra
                                        warps in every producer CTA do the combine while
                                        the tiles run -- the CTA whose GEMM2 tile
                                        completes a row band hands them its arrivals,
                                        and they combine ready tokens from global
                                        memory -- and no SM is a dedicated consumer
                                        unless consumer_sms asks for some.  Same bits.
                                        With CTA pairs: no effect.  With
                                        MOE_SCHED_GATHER_LSU: MOE_ERR_UNSUPPORTED */
#define MOE_SCHED_EVICT_FIRST  0x800u /* the epilogue stores h and y with an L2
                                        evict-first policy (they compete with the weights
                                        for L2).  Same bits */
#define MOE_SCHED_WIDE_CTA     0x100u /* force 256-row MMA tiles on single CTAs: two
                                        128-row MMAs per K step share one B stage and
                                        fill the CTA's two accumulators (an expert's odd
                                        last band uses the first only) */

typedef struct {
  int T, d, f, E, k;        /* tokens, d_model, d_ff, experts, top-k                */
  const void* x;            /* [T][d] bf16 tokens                                   */
  const float* logits;      /* [T][E] fp32 gate logits                              */
  const void* W1;           /* [E][d][f] bf16 gate projection                       */
  const void* W3;           /* [E][d][f] bf16 up projection                         */
  const void* W2;           /* [E][f][d] bf16 down projection                       */
  void* out;                /* [T][d] bf16 layer output                             */
  /* Optional outputs (NULL = kept only in the workspace): */
  int32_t* topk_idx;        /* [T][k] selected experts, by logit desc then id asc   */
  float* topk_gate;         /* [T][k] softmax over the selected logits              */
  int32_t* counts;          /* [E] routed rows per expert                           */
  int32_t* offsets;         /* [E+1] exclusive prefix sum of counts                 */
  int32_t* perm;            /* [T*k] routed row r -> source slot p = t*k + j        */
  int consumer_sms;         /* overlapped mode: 0 = cost model; > 0 = this many (rounded
                               up to whole CTA pairs under MOE_SCHED_CTA_PAIR)       */
  int mgb;                  /* row bands per consumer item (paper's x), >= 1; 0 = 1 */
  unsigned flags;           /* MOE_DBG_* / MOE_SCHED_* bits                         */
  int timeout_us;           /* bound on each device wait; 0 = default (2 s)         */
  /* Optional timing hooks (cudaEvent_t as void*, NULL = none): recorded on the
   * stream just before the first and just after the last expert-FFN launch,
   * i.e. around the one persistent kernel (overlapped mode; it also runs the
   * overlapped part of the combine) or around GEMM1 and GEMM2 (sequential mode).
   * The combine pass that follows (the remainder, or the full combine) is
   * outside the span.  A recorded event separates the launches on either side,
   * so their programmatic overlap is lost while the hooks are in use. */
  void* ev_ffn_begin;
  void* ev_ffn_end;
} moe_layer_args;

/* Bytes of device workspace moe_layer_forward, moe_route, moe_permute and
 * moe_grouped_ffn need for this shape (one buffer serves all of them).  0 on
 * an invalid shape. */
size_t moe_workspace_size(int T, int d, int f, int E, int k);

/* Step (a), routing (paper Section 2.1, "Routing"): per token the k largest
 * logits, ordered by logit descending then expert id ascending (ties to the
 * lower id); gates g_j = softmax over the k selected logits.
 * logits [T][E] fp32 -> topk_idx [T][k] int32, topk_gate [T][k] fp32.
 * counts [E] int32 (optional, NULL to skip): routed rows per expert. */
moe_status moe_route(const float* logits, int T, int E, int k,
                     int32_t* topk_idx, float* topk_gate, int32_t* counts,
                     void* ws, size_t ws_bytes, void* stream);

/* Step (b), permutation into expert-contiguous order (paper Section 3.2.1,
 * remote-owner-aligned row layout, one owner per expert on one GPU, no pad
 * rows): counts, offsets (exclusive scan), and a stable order -- the rows of
 * expert e are its slots p = t*k + j in ascending p.
 * perm [T*k]: row r -> slot p; row_of [T*k]: slot p -> row r;
 * x_perm [T*k][d] bf16: x_perm[r] = x[perm[r] / k].
 * counts [E] and offsets [E+1] are outputs (offsets required, counts optional).
 * Every topk_idx value must lie in [0, E).  An id outside that range (e.g. -1
 * for a dropped token) is skipped rather than indexed with: its slot gets
 * row_of = -1 and no row, offsets[E] comes out below T*k (perm past offsets[E]
 * is left unwritten), and the status block records MOE_ERR_INVALID, which
 * moe_get_status(ws, ...) returns. */
moe_status moe_permute(const void* x, int T, int d, int E, int k, const int32_t* topk_idx,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of,
                       void* x_perm, void* ws, size_t ws_bytes, void* stream);

/* Steps (c1)+(c2) alone, the grouped SwiGLU expert FFN on permuted rows (paper
 * Section 3.3.1, one persistent kernel covering all experts): for expert e and
 * rows r in [offsets[e], offsets[e+1]):
 *   h[r] = bf16(silu(x_perm[r] W1_e) * (x_perm[r] W3_e)),  y[r] = bf16(h[r] W2_e)
 * (fp32 accumulation).  x_perm [R][d], y [R][d] bf16, R = offsets[E] <= T*k;
 * h [R][f] bf16 is written to the caller's buffer if non-NULL, else kept in the
 * workspace.  offsets must start at 0, never decrease and end at most at T*k;
 * otherwise nothing is computed and moe_get_status returns MOE_ERR_INVALID.
 * flags: 0, or MOE_SCHED_ONE_CTA / MOE_SCHED_CTA_PAIR / MOE_SCHED_WIDE_CTA /
 * MOE_SCHED_B_PER_ATOM / MOE_SCHED_FULL_TILES (tile variant), MOE_SCHED_INTERLEAVE,
 * MOE_SCHED_EVICT_FIRST, MOE_SCHED_EXP_SILU; any other bit is MOE_ERR_INVALID. */
moe_status moe_grouped_ffn(const void* x_perm, const int32_t* offsets, int T, int d, int f,
                           int E, int k, const void* W1, const void* W3, const void* W2,
                           void* h, void* y, unsigned flags, void* ws, size_t ws_bytes,
                           void* stream);

/* Step (d) alone, the weighted reduction (paper Section 2.1, "Weighted reduction
 * (scale)"): out[t] = bf16( sum_{j<k} g[t][j] * y[row_of[t*k+j]] ), fp32 in slot
 * order.  y [T*k][d] bf16, row_of [T*k], topk_gate [T][k] -> out [T][d] bf16.
 * Every row_of value must lie in [0, T*k) (as moe_permute writes it when all
 * expert ids are in range); the kernel reads y[row_of[p]] without a check. */
moe_status moe_combine(const void* y, const int32_t* row_of, const float* topk_gate,
                       int T, int d, int k, void* out, void* stream);

/* moe_permute for callers that cannot allocate device memory.  The paper has no
 * counterpart to this entry point; it exists for callers such as a runtime that
 * has already handed all device memory to its own pool, a plug-in host that owns
 * every allocation, or code that must not call cudaMalloc where it permutes.
 * Same arguments, outputs and results as moe_permute, minus the workspace: the
 * per-block histograms and scan bases live in one fixed array inside the library
 * (moe_permute_noalloc_scratch_bytes() bytes, a little over 4 MiB), which every
 * GPU that loads the library holds until the process exits.  This call allocates
 * nothing and calls no allocating routine.
 *  - Limits: T <= 65536 (MOE_ERR_UNSUPPORTED above that), E <= 256, k <= 8,
 *    d % 8 == 0; counts may be NULL.
 *  - An expert id outside [0, E) is skipped as in moe_permute (row_of = -1, no
 *    row); with no status block to record it in, the sign is offsets[E] < T*k.
 *  - The first call on a device looks up the array's device address (with that
 *    device current) and caches it for that device's CUDA context; make that
 *    first call before any stream capture.  After cudaDeviceReset (a new
 *    context) the next call looks the address up again, and so is again a
 *    first call.
 *  - Every call on a device shares the one array and leaves its contents behind;
 *    nothing in it needs to start at zero.  Calls whose work overlaps on the GPU
 *    (e.g. on two streams at once) race on the array: order them on one stream. */
moe_status moe_permute_noalloc(const void* x, int T, int d, int E, int k,
                               const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                               int32_t* perm, int32_t* row_of, void* x_perm, void* stream);

/* Size in bytes of the fixed scratch array moe_permute_noalloc uses. */
size_t moe_permute_noalloc_scratch_bytes(void);

/* The whole layer, steps (a)-(e).  Both modes give bit-identical outputs. */
moe_status moe_layer_forward(const moe_layer_args* args, moe_mode mode,
                             void* ws, size_t ws_bytes, void* stream);

/* ---- Expert parallelism: the fused return ---------------------------------
 * W ranks; rank o owns the local experts [o*El, (o+1)*El) of E = W*El.  Each
 * home rank routes and permutes its own tokens (moe_route, moe_permute); its
 * routed rows, grouped by expert and so by owner, are dispatched to the owners
 * (an all-to-all outside this library, e.g. NCCL) together with each row's home
 * slot p = t*k + j.  The owner runs moe_ep_owner_forward: the paper's rank-wide
 * persistent expert GEMM (Section 3.3.1) whose consumer partition returns every
 * finished row band straight into its home rank's return buffer (the return
 * all-to-all, fused: Sections 3.2.1-3.2.3 and 3.3.2-3.3.3).  Each home then runs
 * moe_ep_home_combine.  The result is bit-identical to moe_layer_forward on the
 * home's tokens with every expert local.
 *
 * The owner only STORES into home buffers (16-byte stores and system-scope
 * release adds; no loads from them, no TMA), so home_y / home_arrive may be
 * another GPU's memory mapped into this one (CUDA IPC, symmetric memory); on one
 * GPU they are plain device pointers of W virtual ranks. */
#define MOE_MAX_EP_RANKS 8

typedef struct {
  int W;                     /* ranks, 1..MOE_MAX_EP_RANKS                           */
  int rank;                  /* this owner's rank o                                  */
  int N;                     /* rows received                                        */
  int d, f, El, k;           /* d_model, d_ff, local experts (W*El <= 256), top-k    */
  const void* x_recv;        /* [N][d] bf16: source rank major, then local expert
                                ascending, each source's rows in its own order       */
  const int32_t* slot_recv;  /* [N] home slot p = t*k + j of each received row       */
  const int32_t* recv_counts;/* [W][El] device: rows from source s for local expert e */
  const void* W1;            /* [El][d][f] bf16, this owner's experts                */
  const void* W3;            /* [El][d][f] bf16                                      */
  const void* W2;            /* [El][f][d] bf16                                      */
  int recv_base[MOE_MAX_EP_RANKS];  /* per source s: row, in s's return buffer (its
                                       dispatch order), of the first row s sent here */
  void* home_y[MOE_MAX_EP_RANKS];   /* per rank: return buffer [T_s*k][d] bf16, in the
                                       home's permutation order (rows of x_perm)     */
  uint32_t* home_arrive[MOE_MAX_EP_RANKS]; /* per rank: arrival words [T_s], zero
                                       before the first call                         */
  int consumer_sms;          /* 0 = cost model; > 0 = this many return CTAs          */
  int mgb;                   /* row bands per middle return segment (paper's x); 0 = 1 */
  unsigned flags;            /* MOE_SCHED_* bits (tile variant, NO_JOIN, INTERLEAVE,
                                EVICT_FIRST); MOE_DBG_TIMESTAMPS                      */
  int timeout_us;            /* bound on each device wait; 0 = 2 s                   */
} moe_ep_owner_args;

/* Workspace bytes moe_ep_owner_forward needs (0 on an invalid shape). */
size_t moe_ep_owner_workspace_size(int N, int d, int f, int El, int W);

/* The owner side of one expert-parallel MoE layer.  Plan (on the device, from
 * recv_counts): the (local expert, source) segments of the received rows are the
 * planning units -- every row band has one destination; remote segments are
 * scheduled first, experts with more remote bands first (Section 3.2.2); the
 * combine plan gives each band its home rank and home row (Section 3.2.3).
 * OVERLAPPED: one persistent launch; consumer CTAs (consumer_sms, or the cost
 * model; producers join once the tile queue drains) wait for each segment's
 * bands, copy them into home_y[s] at the planned row and add 1 per row to
 * home_arrive[s][p / k].  SEQUENTIAL: GEMM1, GEMM2, then the whole return as a
 * separate pass (the baseline).  Both modes store the same bytes.
 * Errors: argument errors at once; a device wait that runs out is reported by
 * moe_get_status(ws, ...); recv_counts that do not sum to N give MOE_ERR_INVALID
 * there (nothing is computed). */
moe_status moe_ep_owner_forward(const moe_ep_owner_args* args, moe_mode mode, void* ws,
                                size_t ws_bytes, void* stream);

/* The home side: for every token t, waits (bounded by timeout_us; 0 = 2 s) until
 * arrive[t] == k, then out[t] = bf16( sum_j g[t][j] * home_y[row_of[t*k+j]] ) in
 * fp32, slot order (moe_combine's arithmetic), and zeroes arrive[t] for the next
 * call.  status: a device word, 0 on entry; a wait that runs out sets it to
 * MOE_ERR_TIMEOUT and ends the other waits (that token's out row is not
 * written).  home_y [T*k][d] bf16, arrive [T], row_of [T*k], topk_gate [T][k]. */
moe_status moe_ep_home_combine(const void* home_y, uint32_t* arrive, const int32_t* row_of,
                               const float* topk_gate, int T, int d, int k, void* out,
                               uint32_t* status, int timeout_us, void* stream);

/* Debug aid: synchronises `stream` and copies the combine plan of the last
 * moe_ep_owner_forward on `ws` (same N, d, f, El, W) into host_out: per row band
 * in schedule order, (home rank, home row of the band's first row) -- 2 int32
 * each; host_out holds max_bands pairs. */
moe_status moe_ep_debug_plan(void* ws, int N, int d, int f, int El, int W, void* stream,
                             int32_t* host_out, int max_bands);

/* Synchronises `stream`, then reads the status block the last call left in `ws`.
 * Returns MOE_OK or the device-side error (MOE_ERR_TIMEOUT).  Host outputs may be
 * NULL: consumer_sms = the consumer SM count used (cost model or hint),
 * n_bands = row bands (tiles of 128 rows) over all experts. */
moe_status moe_get_status(void* ws, void* stream, int* consumer_sms, int* n_bands);

/* Debug aid: synchronises `stream` and copies the per-CTA stamps of the last
 * persistent-kernel launch made with MOE_DBG_TIMESTAMPS into host_out
 * (n_ctas x 8 uint64: [0] start, [1] GEMM1 queue drained, [2] producer role done,
 * [3] consumer role done (all globaltimer ns), [4] GEMM1 tiles, [5] GEMM2 tiles,
 * [6] consumer bands, [7] cluster rank).  *n_ctas = CTAs of that launch (<= 256);
 * host_out must hold max_ctas x 8 values. */
moe_status moe_debug_stamps(void* ws, void* stream, uint64_t* host_out, int max_ctas, int* n_ctas);

/* Debug aid, same launch: per consumed row band b < min(max_bands, 2048), 4 uint64:
 * [0] band ready (globaltimer ns), [1] band combined, [2] tokens it completed,
 * [3] consuming CTA.  host_out must hold max_bands x 4 values. */
moe_status moe_debug_band_stamps(void* ws, void* stream, uint64_t* host_out, int max_bands);

/* Debug aid: synchronises `stream` and sets *n_combined to the number of tokens of
 * the last overlapped layer call on `ws` (shape T, d, f, E, k as in that call) that
 * the persistent kernel combined itself -- the rest were left to the combine pass
 * after it.  Reads T arrival words from the workspace. */
moe_status moe_debug_tokens_combined(const void* ws, int T, int d, int f, int E, int k, void* stream,
                                     int* n_combined);

/* Static English description of a status code. */
const char* moe_status_string(moe_status s);

/* The MMA tile variant moe_layer_forward and moe_grouped_ffn use for this
 * shape and these flags (a host query, no device work): 1 = 128-row tiles on
 * single CTAs, 2 = 256-row tiles on CTA pairs (cta_group::2), 3 = 256-row tiles
 * on single CTAs; 0 for a non-positive size. */
int moe_tile_variant(int T, int f, int E, int k, unsigned flags);

/* The cudaError_t value behind the calling thread's most recent MOE_ERR_CUDA
 * from any entry point (a launch refused, a device fault surfacing at a launch
 * or synchronisation, a failed copy); 0 (cudaSuccess) if none so far.  Not
 * cleared by later successful calls. */
int moe_last_cuda_error(void);

/* Static description of a cudaError_t value (from moe_last_cuda_error). */
const char* moe_cuda_error_string(int code);

/* The number of SMs the persistent kernels use on the current device (a host
 * query, cached per device). */
int moe_num_sms(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
