/*
 * moe_oracle.h -- CPU reference ("oracle") for one Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library under
 * combine_overlap_b200/) may include, link or call this code; only the tests, the
 * smoke check and the CPU-baseline leg of the benchmark do.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes is the plain definition of the layer in
 * "Fine-grained Computation-Communication Overlap via Tile-level Signaling and
 * Scheduling for Mixture-of-Experts" (arXiv 2607.19539), Section 2.1
 * (Mixture-of-Experts Architectures): the router picks top-k experts per token
 * from a probability distribution, each expert is a feed-forward sub-layer, and
 * the layer output is the gate-weighted sum of the selected experts' outputs.
 * The paper's method (Section 3) changes only the schedule, not that result
 * (Section 4.4, Correctness Analysis).  The expert form (SwiGLU, no bias), the
 * softmax over the selected logits, the tie rule and the bf16 storage of the
 * intermediates are readings the paper leaves open; each is stated beside the
 * function that takes it.
 *
 * Arithmetic: fp32 on bf16-rounded operands.  bf16 values are passed as their
 * 16-bit patterns (uint16_t); bf16 rounding is round-to-nearest-even.
 *
 * Every function returns 0 on success and a negative number on a bad argument.
 * All buffers are host memory owned by the caller.
 *
 * Parity pins (see tests/test_oracle_pins.py): every function here is pinned
 * by brute force, closed forms, library routines or invariants; none is
 * "parity unpinned".
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Number of OpenMP threads the oracle uses for the expert and combine loops
 * (1 = single-threaded).  Returns the value now in force. */
int oracle_set_threads(int nthreads);
int oracle_get_threads(void);

/* Router (Section 2.1): for each token t, the k experts with the largest logits,
 * ordered by logit descending then expert id ascending (ties go to the lower id;
 * +0.0 and -0.0 compare equal).  Gates: softmax over the k selected logits,
 * g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), computed in double, stored fp32.
 * logits [T][E] fp32 -> topk_idx [T][k] int32, topk_gate [T][k] fp32.
 * Precondition: finite logits; 1 <= k <= E. */
int oracle_route(const float* logits, int T, int E, int k,
                 int32_t* topk_idx, float* topk_gate);

/* Expert-contiguous permutation (Section 3.2.1 row layout, single-rank reading:
 * one owner group per expert, no padding).  Slot p = t*k + j.
 * counts[e] = #{p : idx[p] == e}; offsets = exclusive prefix sum (E+1 entries);
 * within an expert, slots appear in ascending p (a stable counting sort).
 * perm[r] = p for routed row r; row_of[p] = r. */
int oracle_permute(const int32_t* topk_idx, int T, int E, int k,
                   int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of);

/* x_perm[r] = x[perm[r] / k]  (bf16 rows of d elements). */
int oracle_gather(const uint16_t* x, int T, int d, int k,
                  const int32_t* perm, uint16_t* x_perm);

/* One expert's SwiGLU FFN on one row (the expert sub-layer of Section 2.1):
 *   a_c = sum_i x_i W1[i][c],  b_c = sum_i x_i W3[i][c]   (fp32, i ascending)
 *   h_c = bf16( silu(a_c) * b_c ),  silu(a) = a / (1 + exp(-a))  (fp32)
 *   y_n = bf16( sum_c h_c W2[c][n] )                      (fp32, c ascending)
 * W1, W3: [d][f] bf16; W2: [f][d] bf16 (already offset to the expert).
 * If fp32_h != 0, h is kept in fp32 (no bf16 rounding) -- the "fp32
 * intermediates" variant.  y_row: d bf16 values. */
int oracle_ffn_row(const uint16_t* x_row, int d, int f,
                   const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                   int fp32_h, uint16_t* y_row);

/* The grouped expert step over the permuted rows: for expert e and every row r
 * in [offsets[e], offsets[e+1]), y[r] = FFN_e(x_perm[r]).
 * W1, W3: [E][d][f]; W2: [E][f][d].  identity != 0 replaces every expert by the
 * identity map (y = x_perm; requires nothing of W). */
int oracle_expert_ffn(const uint16_t* x_perm, const int32_t* offsets, int E, int d, int f,
                      const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                      int fp32_h, int identity, uint16_t* y);

/* Weighted reduction "scale" (Section 2.1 step 5):
 *   out[t] = bf16( sum_{j=0..k-1} g_{t,j} * y[row_of[t*k+j]] )  fp32, slot order. */
int oracle_combine(const uint16_t* y, const int32_t* row_of, const float* topk_gate,
                   int T, int d, int k, uint16_t* out);

/* The whole layer: route -> permute -> gather -> experts -> combine.
 * Optional outputs (topk_idx, topk_gate, counts, offsets, perm) may be NULL. */
int oracle_moe_forward(const uint16_t* x, const float* logits,
                       const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                       int T, int d, int f, int E, int k, int fp32_h, int identity,
                       uint16_t* out, int32_t* topk_idx, float* topk_gate,
                       int32_t* counts, int32_t* offsets, int32_t* perm);

/* Definition path, token by token, with no permutation: for each listed token t,
 * out_rows[i] = bf16( sum_j g_{t,j} * FFN_{e_{t,j}}(x_t) ), using the given
 * routing.  Used to check sampled tokens of large layers. */
int oracle_moe_tokens(const uint16_t* x, const int32_t* topk_idx, const float* topk_gate,
                      const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                      int T, int d, int f, int E, int k, int fp32_h, int identity,
                      const int32_t* tokens, int n_tokens, uint16_t* out_rows);

/* bf16 helpers exposed for the tests (round-to-nearest-even, NaN kept quiet). */
uint16_t oracle_f32_to_bf16(float v);
float    oracle_bf16_to_f32(uint16_t h);

#ifdef __cplusplus
}
#endif
#endif /* MOE_ORACLE_H */
