/*
 * moe_oracle.cpp -- plain CPU reference for one Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline).  See moe_oracle.h
 * for the definitions and the readings taken where the paper is silent.
 *
 * The code is deliberately direct: each function is the definition written out
 * with loops, in the order the definition states, with no blocking, fusion or
 * reordering.  OpenMP, when enabled, only splits independent rows or tokens
 * across threads; every row's arithmetic is the same single-threaded sequence.
 *
 * ORACLE_MUTANT (compile-time, tests only) plants one known mistake so that the
 * pin tests can show they catch it.  0 (the default) is the oracle itself.
 */
#include "moe_oracle.h"

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>
#include <algorithm>

#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

static int g_threads = 1;

extern "C" int oracle_set_threads(int nthreads) {
  if (nthreads < 1) nthreads = 1;
#ifdef _OPENMP
  g_threads = nthreads;
#else
  g_threads = 1;
#endif
  return g_threads;
}

extern "C" int oracle_get_threads(void) { return g_threads; }

/* ---- bf16 <-> fp32 (round to nearest, ties to even) ---------------------- */

extern "C" uint16_t oracle_f32_to_bf16(float v) {
  uint32_t u;
  std::memcpy(&u, &v, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0) {
    return (uint16_t)((u >> 16) | 0x0040u);  /* quiet NaN, sign kept */
  }
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

extern "C" float oracle_bf16_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float v;
  std::memcpy(&v, &u, 4);
  return v;
}

static inline float bf(uint16_t h) { return oracle_bf16_to_f32(h); }
static inline uint16_t to_bf(float v) { return oracle_f32_to_bf16(v); }

/* ---- Router --------------------------------------------------------------- */

/* a beats b: larger logit, or equal logit and lower expert id. */
static inline bool beats(float la, int ea, float lb, int eb) {
#if ORACLE_MUTANT == 2
  if (la == lb) return ea > eb;          /* planted: ties go to the higher id */
#endif
  if (la > lb) return true;
  if (la < lb) return false;
  return ea < eb;
}

extern "C" int oracle_route(const float* logits, int T, int E, int k,
                            int32_t* topk_idx, float* topk_gate) {
  if (!logits || !topk_idx || !topk_gate || T < 0 || E < 1 || k < 1 || k > E) return -1;
  std::vector<int> chosen(k);
  std::vector<double> w(k);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    /* Selection: k passes, each takes the best expert not yet chosen. */
    std::vector<char> used(E, 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (used[e]) continue;
        if (best < 0 || beats(l[e], e, l[best], best)) best = e;
      }
      used[best] = 1;
      chosen[j] = best;
    }
    /* Softmax over the selected logits, in double. */
    double m = (double)l[chosen[0]];
    double s = 0.0;
    for (int j = 0; j < k; ++j) {
      w[j] = std::exp((double)l[chosen[j]] - m);
#if ORACLE_MUTANT == 1
      if (j < k - 1 || k == 1) s += w[j];  /* planted: last term dropped */
#else
      s += w[j];
#endif
    }
    for (int j = 0; j < k; ++j) {
      topk_idx[(size_t)t * k + j] = chosen[j];
      topk_gate[(size_t)t * k + j] = (float)(w[j] / s);
    }
  }
  return 0;
}

/* ---- Permutation (stable counting sort by expert) ------------------------- */

extern "C" int oracle_permute(const int32_t* topk_idx, int T, int E, int k,
                              int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of) {
  if (!topk_idx || !counts || !offsets || !perm || !row_of || T < 0 || E < 1 || k < 1) return -1;
  const long P = (long)T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (long p = 0; p < P; ++p) {
    int e = topk_idx[p];
    if (e < 0 || e >= E) return -2;
    counts[e] += 1;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> next(offsets, offsets + E);
#if ORACLE_MUTANT == 6
  for (long p = P - 1; p >= 0; --p) {      /* planted: descending p inside an expert */
#else
  for (long p = 0; p < P; ++p) {
#endif
    int e = topk_idx[p];
    int r = next[e]++;
    perm[r] = (int32_t)p;
    row_of[p] = r;
  }
  return 0;
}

extern "C" int oracle_gather(const uint16_t* x, int T, int d, int k,
                             const int32_t* perm, uint16_t* x_perm) {
  if (!x || !perm || !x_perm || T < 0 || d < 1 || k < 1) return -1;
  const long R = (long)T * k;
  for (long r = 0; r < R; ++r) {
    long t = perm[r] / k;
    std::memcpy(x_perm + r * (size_t)d, x + t * (size_t)d, sizeof(uint16_t) * (size_t)d);
  }
  return 0;
}

/* ---- Expert FFN ----------------------------------------------------------- */

static inline float silu(float a) {
#if ORACLE_MUTANT == 7
  return a / (1.0f + std::exp(a));         /* planted: sign of the exponent */
#else
  return a / (1.0f + std::exp(-a));
#endif
}

extern "C" int oracle_ffn_row(const uint16_t* x_row, int d, int f,
                              const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                              int fp32_h, uint16_t* y_row) {
  if (!x_row || !W1 || !W3 || !W2 || !y_row || d < 1 || f < 1) return -1;
  std::vector<float> a(f, 0.0f), b(f, 0.0f), h(f);
  for (int i = 0; i < d; ++i) {
    const float xi = bf(x_row[i]);
    const uint16_t* w1 = W1 + (size_t)i * f;
    const uint16_t* w3 = W3 + (size_t)i * f;
    for (int c = 0; c < f; ++c) {
      a[c] += xi * bf(w1[c]);
      b[c] += xi * bf(w3[c]);
    }
  }
  for (int c = 0; c < f; ++c) {
#if ORACLE_MUTANT == 3
    float v = silu(b[c]) * a[c];           /* planted: gate and up swapped */
#else
    float v = silu(a[c]) * b[c];
#endif
    h[c] = fp32_h ? v : bf(to_bf(v));
  }
  std::vector<float> y(d, 0.0f);
  for (int c = 0; c < f; ++c) {
    const float hc = h[c];
#if ORACLE_MUTANT == 4
    for (int n = 0; n < d; ++n) y[n] += hc * bf(W2[(size_t)n * f + c]);  /* planted: W2 transposed */
#else
    const uint16_t* w2 = W2 + (size_t)c * d;
    for (int n = 0; n < d; ++n) y[n] += hc * bf(w2[n]);
#endif
  }
  for (int n = 0; n < d; ++n) y_row[n] = to_bf(y[n]);
  return 0;
}

extern "C" int oracle_expert_ffn(const uint16_t* x_perm, const int32_t* offsets, int E, int d, int f,
                                 const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                                 int fp32_h, int identity, uint16_t* y) {
  if (!x_perm || !offsets || !y || E < 1 || d < 1 || f < 1) return -1;
  if (!identity && (!W1 || !W3 || !W2)) return -1;
  const long R = offsets[E];
  /* Row r's expert: the e with offsets[e] <= r < offsets[e+1]. */
  std::vector<int32_t> expert_of(R > 0 ? R : 1);
  for (int e = 0; e < E; ++e)
    for (long r = offsets[e]; r < offsets[e + 1]; ++r) expert_of[r] = e;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(g_threads) reduction(|:bad)
  for (long r = 0; r < R; ++r) {
    const uint16_t* xr = x_perm + (size_t)r * d;
    uint16_t* yr = y + (size_t)r * d;
    if (identity) {
      std::memcpy(yr, xr, sizeof(uint16_t) * (size_t)d);
      continue;
    }
    const int e = expert_of[r];
    const size_t wsz = (size_t)d * f;
    bad |= oracle_ffn_row(xr, d, f, W1 + e * wsz, W3 + e * wsz, W2 + e * wsz, fp32_h, yr) != 0;
  }
  return bad ? -3 : 0;
}

/* ---- Combine -------------------------------------------------------------- */

static void combine_token(const uint16_t* y, const int32_t* row_of, const float* topk_gate,
                          long t, int d, int k, uint16_t* out_row) {
  for (int n = 0; n < d; ++n) {
    float acc = 0.0f;
    for (int j = 0; j < k; ++j) {
#if ORACLE_MUTANT == 5
      const float g = topk_gate[t * k];     /* planted: slot 0's gate for every slot */
#else
      const float g = topk_gate[t * k + j];
#endif
      const long r = row_of[t * k + j];
      acc += g * bf(y[(size_t)r * d + n]);
    }
    out_row[n] = to_bf(acc);
  }
}

extern "C" int oracle_combine(const uint16_t* y, const int32_t* row_of, const float* topk_gate,
                              int T, int d, int k, uint16_t* out) {
  if (!y || !row_of || !topk_gate || !out || T < 0 || d < 1 || k < 1) return -1;
#pragma omp parallel for schedule(static) num_threads(g_threads)
  for (long t = 0; t < T; ++t) combine_token(y, row_of, topk_gate, t, d, k, out + (size_t)t * d);
  return 0;
}

/* ---- Whole layer ---------------------------------------------------------- */

extern "C" int oracle_moe_forward(const uint16_t* x, const float* logits,
                                  const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                                  int T, int d, int f, int E, int k, int fp32_h, int identity,
                                  uint16_t* out, int32_t* topk_idx, float* topk_gate,
                                  int32_t* counts, int32_t* offsets, int32_t* perm) {
  if (!x || !logits || !out || T < 0 || d < 1 || f < 1 || E < 1 || k < 1 || k > E) return -1;
  const long R = (long)T * k;
  std::vector<int32_t> idx(R), cnt(E), off(E + 1), pm(R), rof(R);
  std::vector<float> gate(R);
  int rc = oracle_route(logits, T, E, k, idx.data(), gate.data());
  if (rc) return rc;
  rc = oracle_permute(idx.data(), T, E, k, cnt.data(), off.data(), pm.data(), rof.data());
  if (rc) return rc;
  std::vector<uint16_t> xp((size_t)R * d), y((size_t)R * d);
  rc = oracle_gather(x, T, d, k, pm.data(), xp.data());
  if (rc) return rc;
  rc = oracle_expert_ffn(xp.data(), off.data(), E, d, f, W1, W3, W2, fp32_h, identity, y.data());
  if (rc) return rc;
  rc = oracle_combine(y.data(), rof.data(), gate.data(), T, d, k, out);
  if (rc) return rc;
  if (topk_idx) std::memcpy(topk_idx, idx.data(), sizeof(int32_t) * R);
  if (topk_gate) std::memcpy(topk_gate, gate.data(), sizeof(float) * R);
  if (counts) std::memcpy(counts, cnt.data(), sizeof(int32_t) * E);
  if (offsets) std::memcpy(offsets, off.data(), sizeof(int32_t) * (E + 1));
  if (perm) std::memcpy(perm, pm.data(), sizeof(int32_t) * R);
  return 0;
}

extern "C" int oracle_moe_tokens(const uint16_t* x, const int32_t* topk_idx, const float* topk_gate,
                                 const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                                 int T, int d, int f, int E, int k, int fp32_h, int identity,
                                 const int32_t* tokens, int n_tokens, uint16_t* out_rows) {
  if (!x || !topk_idx || !topk_gate || !tokens || !out_rows || d < 1 || f < 1 || E < 1 || k < 1)
    return -1;
  if (!identity && (!W1 || !W3 || !W2)) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(g_threads) reduction(|:bad)
  for (int i = 0; i < n_tokens; ++i) {
    const long t = tokens[i];
    if (t < 0 || t >= T) { bad = 1; continue; }
    const uint16_t* xt = x + (size_t)t * d;
    std::vector<uint16_t> yj((size_t)k * d);
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[t * k + j];
      if (e < 0 || e >= E) { bad = 1; break; }
      if (identity) {
        std::memcpy(&yj[(size_t)j * d], xt, sizeof(uint16_t) * (size_t)d);
      } else {
        const size_t wsz = (size_t)d * f;
        bad |= oracle_ffn_row(xt, d, f, W1 + e * wsz, W3 + e * wsz, W2 + e * wsz, fp32_h,
                              &yj[(size_t)j * d]) != 0;
      }
    }
    if (bad) continue;
    uint16_t* o = out_rows + (size_t)i * d;
    for (int n = 0; n < d; ++n) {
      float acc = 0.0f;
      for (int j = 0; j < k; ++j) acc += topk_gate[t * k + j] * bf(yj[(size_t)j * d + n]);
      o[n] = to_bf(acc);
    }
  }
  return bad ? -3 : 0;
}
