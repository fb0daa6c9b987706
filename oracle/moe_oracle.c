/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for one
 * Occult-style mixture-of-experts layer.  TEST INFRASTRUCTURE ONLY: the
 * product library never links, loads or calls this file; only the tests,
 * the smoke check and the benchmark's CPU-baseline leg do.
 *
 * Sources (cited by page title and section/figure):
 *   [Occult]   "Occult: Optimizing Collaborative Communication across Experts
 *               for Accelerated Parallel MoE Training and Inference" -- TL;DR,
 *               Abstract, Figure 2 (three all-to-all strategies), Figure 4
 *               (ORI/SFD/EPD token states guided by BRIMs), Figure 5 (the two
 *               BRIMs and their dimensions).
 *   [Coupling] "Expert Coupling in MoE Pretraining: Reducing All-to-All
 *               Overhead with Correlated Placement and Token Shuffling" --
 *               Abstract (top-k routing, once-per-GPU dispatch, correlated
 *               placement from co-selected expert pairs).
 *
 * Arithmetic: every floating-point quantity is computed in double precision
 * (the pages fix no precision).  Inputs that arrive as float32 or bfloat16
 * are widened exactly to double before use.  Loops follow the definitions
 * one term at a time: no blocking, fusion or reordering.
 *
 * Readings taken where the pages are silent (each one is listed, with its
 * reason, in the design notes of the repository):
 *   R1  BRIM entries are row positions (-1 = not sent); one entry drives both
 *       the gather into SFD and the scatter back out of it ("bidirectional").
 *   R2  Rows inside an SFD segment and inside an EPD group are in ascending
 *       ORI-token order (stable compaction).
 *   R3  Top-k compares raw logits; equal logits go to the lower expert id;
 *       output order is descending score.
 *   R4  Gate weights: softmax over all E logits then gather (renorm = 0), or
 *       softmax over the k selected logits (renorm = 1).
 *   R5  The gate weight is applied on the expert side, before the per-rank
 *       pre-reduce (intra-collaboration), so one return row per (token,rank)
 *       carries sum_j w_j * FFN_j(x).
 *   R6  C_T counts every SFD row, including rows whose destination rank is
 *       the token's own source rank; "remote" rows use the contiguous token
 *       sharding src(t) = floor(t * R / T).
 *   R7  Shared experts are not dispatched; they see ORI rows with weight 1
 *       and are added after the routed combine.
 *   R8  Placement slot q = slot_of[e]; rank(e) = q / L, loc(e) = q % L;
 *       EPD groups are laid out in slot order.
 *   R9  Routing-score-based collaboration pruning keeps, per token, the first
 *       m distinct ranks met along its descending-score expert list (so the
 *       ranks of its highest-scoring experts), drops every assignment on any
 *       other rank (expert id -1 = empty slot), and rescales the kept gate
 *       weights so that their sum equals the sum before pruning.
 *   R10 An expert id of -1 in a top-k list is an empty slot: it is sent
 *       nowhere and contributes nothing.  Any other id outside [0, E) is an
 *       error.
 *   R11 The backward pass is the exact derivative of the layer output for
 *       fixed expert choices: the top-k selection is piecewise constant and
 *       passes no gradient; the gate weights pass theirs through the softmax
 *       variant of R4.  It is defined for unpruned routing.
 *   R12 A weight gradient sums, over every (token, slot) routed to that
 *       expert in ascending token order, the outer products of that row;
 *       shared experts take every token with weight 1.
 *   R13-R15 Token shuffling across layers: see the section of that name
 *       below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_DT_F32 0
#define ORACLE_DT_BF16 1
#define ORACLE_DT_F64 2

/* Exact widening of one stored element to double.  bfloat16 is the upper
 * half of an IEEE binary32, so widening is a 16-bit left shift of the bits. */
static double widen(const void* base, size_t i, int dt) {
  if (dt == ORACLE_DT_F64) return ((const double*)base)[i];
  if (dt == ORACLE_DT_F32) return (double)((const float*)base)[i];
  uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static size_t esize(int dt) {
  return dt == ORACLE_DT_BF16 ? 2 : dt == ORACLE_DT_F32 ? 4 : 8;
}

int oracle_abi_version(void) { return 1; }

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------
 * Routing: each token picks k of E experts [Coupling, Abstract: "each token
 * is routed to k of these experts"]; top-2/4/6/8 appear in [Occult, Fig. 3].
 * Selection by reading R3, weights by reading R4.
 *   logits  float32 [T,E]
 *   idx     int32   [T,k]  (descending score)
 *   w       double  [T,k]
 * ---------------------------------------------------------------------- */
int oracle_route(const float* logits, int T, int E, int k, int renorm,
                 int32_t* idx, double* w) {
  if (T < 0 || E < 1 || k < 1 || k > E) return -1;
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    /* k rounds of "best remaining expert": larger logit wins, and on an
     * equal logit the lower id wins. */
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        int taken = 0;
        for (int i = 0; i < j; ++i)
          if (idx[(size_t)t * k + i] == e) taken = 1;
        if (taken) continue;
        if (best < 0 || l[e] > l[best]) best = e; /* ties keep the lower id */
      }
      idx[(size_t)t * k + j] = best;
    }
    /* softmax, stabilised by the row maximum (a no-op in exact arithmetic) */
    double m = (double)l[0];
    for (int e = 1; e < E; ++e)
      if ((double)l[e] > m) m = (double)l[e];
    double denom = 0.0;
    if (renorm) {
      for (int j = 0; j < k; ++j) denom += exp((double)l[idx[(size_t)t * k + j]] - m);
    } else {
      for (int e = 0; e < E; ++e) denom += exp((double)l[e] - m);
    }
    for (int j = 0; j < k; ++j)
      w[(size_t)t * k + j] = exp((double)l[idx[(size_t)t * k + j]] - m) / denom;
  }
  return 0;
}

/* ------------------------------------------------------------------------
 * BRIM construction [Occult, Fig. 5; Fig. 4; TL;DR "all-to-all budget C_T"].
 *   BRIM_0 : int32 [R, T]      rank x ORI token  -> SFD row or -1
 *   BRIM_1 : int32 [L, cap]    local expert x SFD row -> EPD row or -1
 *            (cap = T * min(k, R) is the row stride; columns >= C_T unused)
 *   sfd_token [cap]  : SFD row -> ORI token (inverse of BRIM_0)
 *   sfd_off  [R+1]   : start of each rank's SFD segment; sfd_off[R] = C_T
 *   epd_off  [E+1]   : start of each slot's EPD group (slot order, R8)
 *   epd_sfd  [T*k]   : EPD row -> SFD row (inverse of BRIM_1)
 *   epd_gate [T*k]   : EPD row -> gate weight of that (token, expert) pair
 * "Each token is sent once per destination device" [Coupling, Abstract;
 * Occult, Fig. 2 third strategy].  Ordering by reading R2.
 * ---------------------------------------------------------------------- */
int oracle_brim(const int32_t* idx, const double* w, int T, int k,
                const int32_t* slot_of, int E, int R,
                int32_t* brim0, int32_t* sfd_token, int32_t* sfd_off,
                int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                double* epd_gate, int32_t* c_t) {
  if (R < 1 || E % R != 0 || k < 1 || k > E || T < 0) return -1;
  const int L = E / R;
  const int kr = k < R ? k : R;
  const size_t cap = (size_t)T * kr;

  /* hit(t, r): does token t select at least one expert held by rank r? */
  char* hit = (char*)calloc((size_t)T * R + 1, 1);
  if (!hit) return -2;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      if (e == -1) continue; /* empty slot (R10) */
      if (e < 0 || e >= E) { free(hit); return -3; }
      hit[(size_t)t * R + slot_of[e] / L] = 1;
    }

  /* n_r = number of tokens sent to rank r; sfd_off = exclusive prefix. */
  sfd_off[0] = 0;
  for (int r = 0; r < R; ++r) {
    int n = 0;
    for (int t = 0; t < T; ++t) n += hit[(size_t)t * R + r];
    sfd_off[r + 1] = sfd_off[r] + n;
  }
  *c_t = sfd_off[R];

  /* BRIM_0[r][t] = sfd_off[r] + #{t' < t : hit(t', r)}, else -1. */
  for (int r = 0; r < R; ++r) {
    int seen = 0;
    for (int t = 0; t < T; ++t) {
      if (hit[(size_t)t * R + r]) {
        int s = sfd_off[r] + seen;
        brim0[(size_t)r * T + t] = s;
        sfd_token[s] = t;
        ++seen;
      } else {
        brim0[(size_t)r * T + t] = -1;
      }
    }
  }

  /* c_q = number of tokens that selected the expert placed at slot q. */
  int32_t* expert_at_slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  if (!expert_at_slot) { free(hit); return -2; }
  for (int e = 0; e < E; ++e) expert_at_slot[slot_of[e]] = e;
  epd_off[0] = 0;
  for (int q = 0; q < E; ++q) {
    int c = 0, e = expert_at_slot[q];
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j)
        if (idx[(size_t)t * k + j] == e) ++c;
    epd_off[q + 1] = epd_off[q] + c;
  }

  /* every BRIM_1 entry starts as "no expert" */
  for (size_t i = 0; i < (size_t)L * cap; ++i) brim1[i] = -1;

  /* p = epd_off[slot(e)] + #{t' < t : e in idx[t']};
   * BRIM_1[loc(e)][BRIM_0[rank(e)][t]] = p. */
  int32_t* seen_e = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!seen_e) { free(hit); free(expert_at_slot); return -2; }
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      if (e == -1) continue;
      int q = slot_of[e];
      int r = q / L, l = q % L;
      int p = epd_off[q] + seen_e[e];
      seen_e[e] += 1;
      int s = brim0[(size_t)r * T + t];
      brim1[(size_t)l * cap + s] = p;
      epd_sfd[p] = s;
      epd_gate[p] = w[(size_t)t * k + j];
    }
  }
  free(seen_e);
  free(expert_at_slot);
  free(hit);
  return 0;
}

/* ------------------------------------------------------------------------
 * Row gathers of the dispatch [Occult, Fig. 4: ORI -> SFD -> EPD].
 * Rows are copied byte for byte (row_bytes each).
 * ---------------------------------------------------------------------- */
void oracle_gather_rows(const void* src, size_t row_bytes, const int32_t* index,
                        int n_rows, void* dst) {
  for (int i = 0; i < n_rows; ++i)
    memcpy((char*)dst + (size_t)i * row_bytes,
           (const char*)src + (size_t)index[i] * row_bytes, row_bytes);
}

/* ------------------------------------------------------------------------
 * One SwiGLU expert applied to one row a[d] (double):
 *   g_i = sum_c Wg[i][c] a_c,  u_i = sum_c Wu[i][c] a_c  (i < f)
 *   h_i = silu(g_i) * u_i,     silu(z) = z / (1 + exp(-z))
 *   o_c = sum_i Wd[c][i] h_i   (c < d)
 * Wg, Wu are [f, d]; Wd is [d, f]; all in dtype wdt.  h is scratch [f].
 * The expert's FFN is the "sparse matrix multiplication" stage of the
 * pipeline [Occult, TL;DR]; SwiGLU is the configured expert kind.
 * kind 1 = IDENTITY: o = a (a test expert with no weights).
 * ---------------------------------------------------------------------- */
static void expert_row(int kind, const double* a, const void* Wg, const void* Wu,
                       const void* Wd, int wdt, int d, int f, double* h, double* o) {
  if (kind == 1) {
    for (int c = 0; c < d; ++c) o[c] = a[c];
    return;
  }
  for (int i = 0; i < f; ++i) {
    double g = 0.0, u = 0.0;
    for (int c = 0; c < d; ++c) {
      g += widen(Wg, (size_t)i * d + c, wdt) * a[c];
      u += widen(Wu, (size_t)i * d + c, wdt) * a[c];
    }
    double silu = g / (1.0 + exp(-g));
    h[i] = silu * u;
  }
  for (int c = 0; c < d; ++c) {
    double acc = 0.0;
    for (int i = 0; i < f; ++i) acc += widen(Wd, (size_t)c * f + i, wdt) * h[i];
    o[c] = acc;
  }
}

/* Public single-row expert, used by the oracle's own self-checks. */
void oracle_expert_row(int kind, const double* a, const void* Wg, const void* Wu,
                       const void* Wd, int wdt, int d, int f, double* o) {
  double* h = (double*)malloc(sizeof(double) * (size_t)(f > 0 ? f : 1));
  expert_row(kind, a, Wg, Wu, Wd, wdt, d, f, h, o);
  free(h);
}

/* ------------------------------------------------------------------------
 * Dense definition of the layer output, with no BRIM anywhere:
 *   Y[t] = sum_j w[t][j] * FFN_{idx[t][j]}(X[t]) + sum_s FFN_shared_s(X[t])
 * for the tokens listed in `tokens` (n_tok of them; NULL = all T).
 *   X    [T, d] dtype xdt
 *   Wg,Wu [E, f, d], Wd [E, d, f] dtype wdt (expert-id order)
 *   Sg,Su [S, fs, d], Sd [S, d, fs] (S = 0 allowed)
 *   Y    [n_tok, d] double
 * ---------------------------------------------------------------------- */
int oracle_dense_layer(const void* X, int xdt, int T, int d,
                       const int32_t* idx, const double* w, int k,
                       const void* Wg, const void* Wu, const void* Wd, int wdt,
                       int E, int f, int kind,
                       const void* Sg, const void* Su, const void* Sd, int S, int fs,
                       const int32_t* tokens, int n_tok, double* Y) {
  if (d < 1 || T < 0 || k < 1) return -1;
  if (tokens == NULL) n_tok = T;
  const size_t wg_stride = (size_t)f * d, wd_stride = (size_t)d * f;
  const size_t sg_stride = (size_t)fs * d, sd_stride = (size_t)d * fs;
  const size_t es = esize(wdt);
  int bad = 0;
#pragma omp parallel
  {
    int hmax = f > fs ? f : fs;
    double* a = (double*)malloc(sizeof(double) * (size_t)d);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
#pragma omp for schedule(dynamic, 1)
    for (int n = 0; n < n_tok; ++n) {
      int t = tokens ? tokens[n] : n;
      double* y = Y + (size_t)n * d;
      if (t < 0 || t >= T) { bad = 1; continue; }
      for (int c = 0; c < d; ++c) a[c] = widen(X, (size_t)t * d + c, xdt);
      for (int c = 0; c < d; ++c) y[c] = 0.0;
      for (int j = 0; j < k; ++j) {
        int e = idx[(size_t)t * k + j];
        if (e == -1) continue; /* empty slot (R10) */
        if (e < 0 || e >= E) { bad = 1; continue; }
        expert_row(kind, a, (const char*)Wg + e * wg_stride * es,
                   (const char*)Wu + e * wg_stride * es,
                   (const char*)Wd + e * wd_stride * es, wdt, d, f, h, o);
        for (int c = 0; c < d; ++c) y[c] += w[(size_t)t * k + j] * o[c];
      }
      for (int s = 0; s < S; ++s) {
        expert_row(0, a, (const char*)Sg + s * sg_stride * es, (const char*)Su + s * sg_stride * es,
                   (const char*)Sd + s * sd_stride * es, wdt, d, fs, h, o);
        for (int c = 0; c < d; ++c) y[c] += o[c];
      }
    }
    free(a); free(o); free(h);
  }
  return bad ? -3 : 0;
}

/* ------------------------------------------------------------------------
 * The layer the Occult way [Occult, Fig. 4 and Fig. 5; Abstract,
 * intra-collaboration], one step after another on the BRIMs built by
 * oracle_brim():
 *   1. dispatch  X_sfd[s] = X[sfd_token[s]]            (ORI -> SFD)
 *   2. re-index  X_epd[p] = X_sfd[epd_sfd[p]]          (SFD -> EPD)
 *   3. experts   O_epd[p] = epd_gate[p] * FFN_{x(p)}(X_epd[p]), where x(p)
 *                is the expert placed at the slot whose EPD group holds p
 *   4. pre-reduce (intra-collaboration, one return row per SFD row)
 *                Y_sfd[s] = sum over l ascending, BRIM_1[l][s] >= 0, of
 *                           O_epd[BRIM_1[l][s]]
 *   5. combine   Y[t] = sum over r ascending, BRIM_0[r][t] >= 0, of
 *                       Y_sfd[BRIM_0[r][t]]
 *   6. shared    Y[t] += sum over s ascending of FFN_shared_s(X[t])
 * All in double.  Outputs Y_sfd [C_T, d], Y [T, d] (double).
 * ---------------------------------------------------------------------- */
int oracle_occult_layer(const void* X, int xdt, int T, int d,
                        const int32_t* slot_of, int E, int R, int k,
                        const int32_t* brim0, const int32_t* sfd_token,
                        const int32_t* brim1, const int32_t* epd_off,
                        const int32_t* epd_sfd, const double* epd_gate, int c_t,
                        const void* Wg, const void* Wu, const void* Wd, int wdt,
                        int f, int kind,
                        const void* Sg, const void* Su, const void* Sd, int S, int fs,
                        double* Y_sfd, double* Y) {
  if (R < 1 || E % R != 0) return -1;
  const int L = E / R;
  const int kr = k < R ? k : R;
  const size_t cap = (size_t)T * kr;
  const size_t tk = (size_t)T * k;
  const size_t es = esize(wdt);

  double* X_sfd = (double*)malloc(sizeof(double) * ((size_t)c_t * d + 1));
  double* X_epd = (double*)malloc(sizeof(double) * (tk * d + 1));
  double* O_epd = (double*)malloc(sizeof(double) * (tk * d + 1));
  int32_t* expert_at_slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  if (!X_sfd || !X_epd || !O_epd || !expert_at_slot) {
    free(X_sfd); free(X_epd); free(O_epd); free(expert_at_slot);
    return -2;
  }
  for (int e = 0; e < E; ++e) expert_at_slot[slot_of[e]] = e;

  /* 1. ORI -> SFD */
  for (int s = 0; s < c_t; ++s)
    for (int c = 0; c < d; ++c)
      X_sfd[(size_t)s * d + c] = widen(X, (size_t)sfd_token[s] * d + c, xdt);
  /* 2. SFD -> EPD */
  for (size_t p = 0; p < (size_t)epd_off[E]; ++p)
    for (int c = 0; c < d; ++c)
      X_epd[p * d + c] = X_sfd[(size_t)epd_sfd[p] * d + c];
  /* 3. expert compute, one EPD group (slot) after another; with empty slots
   *    (R10) only the first epd_off[E] EPD rows exist */
  const size_t n_epd = (size_t)epd_off[E];
#pragma omp parallel
  {
    double* h = (double*)malloc(sizeof(double) * (size_t)(f > 0 ? f : 1));
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
    for (long long pp = 0; pp < (long long)n_epd; ++pp) {
      size_t p = (size_t)pp;
      int q = 0;
      while (!(epd_off[q] <= (int)p && (int)p < epd_off[q + 1])) ++q;
      int e = expert_at_slot[q];
      expert_row(kind, X_epd + p * d, (const char*)Wg + (size_t)e * f * d * es,
                 (const char*)Wu + (size_t)e * f * d * es,
                 (const char*)Wd + (size_t)e * d * f * es, wdt, d, f, h, o);
      for (int c = 0; c < d; ++c) O_epd[p * d + c] = epd_gate[p] * o[c];
    }
    free(h); free(o);
  }
  /* 4. intra-collaboration pre-reduce: one return row per SFD row */
  for (int s = 0; s < c_t; ++s) {
    for (int c = 0; c < d; ++c) Y_sfd[(size_t)s * d + c] = 0.0;
    for (int l = 0; l < L; ++l) {
      int p = brim1[(size_t)l * cap + s];
      if (p < 0) continue;
      for (int c = 0; c < d; ++c) Y_sfd[(size_t)s * d + c] += O_epd[(size_t)p * d + c];
    }
  }
  /* 5. combine back into ORI order */
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < d; ++c) Y[(size_t)t * d + c] = 0.0;
    for (int r = 0; r < R; ++r) {
      int s = brim0[(size_t)r * T + t];
      if (s < 0) continue;
      for (int c = 0; c < d; ++c) Y[(size_t)t * d + c] += Y_sfd[(size_t)s * d + c];
    }
  }
  /* 6. shared experts on ORI rows, weight 1 */
  if (S > 0) {
#pragma omp parallel
    {
      double* a = (double*)malloc(sizeof(double) * (size_t)d);
      double* h = (double*)malloc(sizeof(double) * (size_t)(fs > 0 ? fs : 1));
      double* o = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
      for (int t = 0; t < T; ++t) {
        for (int c = 0; c < d; ++c) a[c] = widen(X, (size_t)t * d + c, xdt);
        for (int s = 0; s < S; ++s) {
          expert_row(0, a, (const char*)Sg + (size_t)s * fs * d * es,
                     (const char*)Su + (size_t)s * fs * d * es,
                     (const char*)Sd + (size_t)s * d * fs * es, wdt, d, fs, h, o);
          for (int c = 0; c < d; ++c) Y[(size_t)t * d + c] += o[c];
        }
      }
      free(a); free(h); free(o);
    }
  }
  free(X_sfd); free(X_epd); free(O_epd); free(expert_at_slot);
  return 0;
}

/* ------------------------------------------------------------------------
 * Routing-score-based collaboration pruning [Occult, TL;DR: two pruning
 * schemes, routing-score-based and similarity-based, minimise the all-to-all
 * budget C_T; Abstract: collaboration pruning controllably minimises the
 * cost], by reading R9.  In place on idx [T,k] (descending score) and
 * w [T,k]:
 *   keep = the first m distinct ranks met walking j = 0 .. k-1
 *   for j with rank(idx[t][j]) not in keep: idx = -1, w = 0
 *   kept w_j *= (sum_j w_j before) / (sum of kept w_j)
 * m >= the number of distinct ranks leaves the token unchanged.
 * ---------------------------------------------------------------------- */
int oracle_prune(int32_t* idx, double* w, int T, int k, const int32_t* slot_of, int E, int R,
                 int m) {
  if (R < 1 || E % R != 0 || m < 1) return -1;
  const int L = E / R;
  int32_t* keep = (int32_t*)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
  if (!keep) return -2;
  for (int t = 0; t < T; ++t) {
    int32_t* id = idx + (size_t)t * k;
    double* wt = w + (size_t)t * k;
    int n_keep = 0;
    for (int j = 0; j < k; ++j) {
      if (id[j] == -1) continue;
      int r = slot_of[id[j]] / L, known = 0;
      for (int i = 0; i < n_keep; ++i)
        if (keep[i] == r) known = 1;
      if (!known && n_keep < m) keep[n_keep++] = r;
    }
    double before = 0.0, kept = 0.0;
    for (int j = 0; j < k; ++j) before += wt[j];
    for (int j = 0; j < k; ++j) {
      if (id[j] == -1) continue;
      int r = slot_of[id[j]] / L, in = 0;
      for (int i = 0; i < n_keep; ++i)
        if (keep[i] == r) in = 1;
      if (in) {
        kept += wt[j];
      } else {
        id[j] = -1;
        wt[j] = 0.0;
      }
    }
    if (kept > 0.0)
      for (int j = 0; j < k; ++j)
        if (id[j] != -1) wt[j] = wt[j] * before / kept;
  }
  free(keep);
  return 0;
}

/* ------------------------------------------------------------------------
 * Dispatched-row counter for a placement [Coupling, Abstract: a dispatcher
 * that sends each token to each GPU once; Occult, Fig. 2].
 *   per_rank[r] = #{t : token t selects an expert held by rank r}
 *   total       = sum_r per_rank[r]                    (= C_T)
 *   remote      = #{(t, r) sent : r != floor(t * R / T)}   (reading R6)
 * ---------------------------------------------------------------------- */
int oracle_count_dispatched(const int32_t* idx, int T, int k, const int32_t* slot_of,
                            int E, int R, int32_t* per_rank, int64_t* total,
                            int64_t* remote) {
  if (R < 1 || E % R != 0) return -1;
  const int L = E / R;
  for (int r = 0; r < R; ++r) per_rank[r] = 0;
  *total = 0;
  *remote = 0;
  for (int t = 0; t < T; ++t) {
    int src = (int)(((int64_t)t * R) / T);
    for (int r = 0; r < R; ++r) {
      int sent = 0;
      for (int j = 0; j < k; ++j) {
        int e = idx[(size_t)t * k + j];
        if (e != -1 && slot_of[e] / L == r) sent = 1;
      }
      if (!sent) continue;
      per_rank[r] += 1;
      *total += 1;
      if (r != src) *remote += 1;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------
 * Expert co-activation pair histogram [Coupling, Abstract: expert pairs
 * selected together by tokens; Occult, Abstract: "collaborated" experts].
 *   H[a][b] (a != b) = #{t : a and b both in idx[t]}  (symmetric)
 *   H[a][a]          = #{t : a in idx[t]}
 * accumulate = 0 clears H first.
 * ---------------------------------------------------------------------- */
void oracle_coact_histogram(const int32_t* idx, int T, int k, int E, uint32_t* H,
                            int accumulate) {
  if (!accumulate)
    for (size_t i = 0; i < (size_t)E * E; ++i) H[i] = 0;
  for (int t = 0; t < T; ++t)
    for (int a = 0; a < E; ++a)
      for (int b = 0; b < E; ++b) {
        int has_a = 0, has_b = 0;
        for (int j = 0; j < k; ++j) {
          if (idx[(size_t)t * k + j] == a) has_a = 1;
          if (idx[(size_t)t * k + j] == b) has_b = 1;
        }
        if (has_a && has_b) H[(size_t)a * E + b] += 1;
      }
}

/* ------------------------------------------------------------------------
 * Correlated placement, greedy [Coupling, Abstract: experts often selected
 * together go on the same GPU; Occult, TL;DR: expert-placement rescheduling].
 * The pages name no algorithm; this greedy is the plainest one:
 *   repeat for rank r = 0 .. R-1:
 *     seed = unplaced expert with the largest H[a][a] (ties -> lower id)
 *     while the rank holds fewer than L experts:
 *       add the unplaced b maximising sum_{a in rank} H[a][b]
 *       (ties -> larger H[b][b], then lower id)
 *   slots inside a rank follow insertion order.
 * H is uint32 [E, E]; slot_of receives the placement.
 * ---------------------------------------------------------------------- */
int oracle_place_greedy(const uint32_t* H, int E, int R, int32_t* slot_of) {
  if (R < 1 || E % R != 0) return -1;
  const int L = E / R;
  char* placed = (char*)calloc((size_t)E, 1);
  int32_t* members = (int32_t*)malloc(sizeof(int32_t) * (size_t)L);
  if (!placed || !members) { free(placed); free(members); return -2; }
  for (int r = 0; r < R; ++r) {
    int n = 0;
    int seed = -1;
    for (int a = 0; a < E; ++a) {
      if (placed[a]) continue;
      if (seed < 0 || H[(size_t)a * E + a] > H[(size_t)seed * E + seed]) seed = a;
    }
    members[n++] = seed;
    placed[seed] = 1;
    slot_of[seed] = r * L + 0;
    while (n < L) {
      int best = -1;
      uint64_t best_score = 0;
      for (int b = 0; b < E; ++b) {
        if (placed[b]) continue;
        uint64_t score = 0;
        for (int i = 0; i < n; ++i) score += H[(size_t)members[i] * E + b];
        int better = 0;
        if (best < 0) better = 1;
        else if (score > best_score) better = 1;
        else if (score == best_score &&
                 H[(size_t)b * E + b] > H[(size_t)best * E + best]) better = 1;
        if (better) { best = b; best_score = score; }
      }
      slot_of[best] = r * L + n;
      members[n++] = best;
      placed[best] = 1;
    }
  }
  free(placed);
  free(members);
  return 0;
}


/* ------------------------------------------------------------------------
 * Backward pass (readings R11, R12).  The forward of one (token, expert)
 * row is, with a = X[t] and gate weight w:
 *     g = Wg a,  u = Wu a,  h_i = silu(g_i) u_i,  o = Wd h,  out = w o
 * so for an upstream gradient dy = dL/d(out):
 *     dL/dw     = <dy, o>
 *     dh        = w Wd^T dy
 *     dg_i      = dh_i u_i silu'(g_i),  silu'(z) = s (1 + z (1 - s)), s = 1/(1+e^-z)
 *     du_i      = dh_i silu(g_i)
 *     dL/da     = Wg^T dg + Wu^T du
 *     dL/dWd    = w dy h^T,  dL/dWg = dg a^T,  dL/dWu = du a^T
 * The identity expert (kind 1) has o = a: dL/dw = <dy, a>, dL/da = w dy.
 *
 * row_backward() fills h, dg, du (each [f]) and returns dL/dw; da (if not
 * NULL) receives dL/da, and dw_abs (if not NULL) the sum of the absolute
 * values of the terms of dL/dw (sum_i |(Wd^T dy)_i h_i|), the magnitude its
 * rounding error scales with.  Weights are one expert's Wg,Wu [f,d], Wd [d,f].
 * ---------------------------------------------------------------------- */
static double row_backward(int kind, const double* a, const double* dy, double w,
                           const void* Wg, const void* Wu, const void* Wd, int wdt,
                           int d, int f, double* h, double* dg, double* du, double* da,
                           double* dw_abs) {
  double abs_sum = 0.0; /* sum of |terms| of dL/dw: its condition magnitude */
  if (kind == 1) {
    double dw = 0.0;
    for (int c = 0; c < d; ++c) {
      dw += dy[c] * a[c];
      abs_sum += fabs(dy[c] * a[c]);
    }
    if (da)
      for (int c = 0; c < d; ++c) da[c] = w * dy[c];
    if (dw_abs) *dw_abs = abs_sum;
    return dw;
  }
  double dw = 0.0;
  for (int i = 0; i < f; ++i) {
    double g = 0.0, u = 0.0;
    for (int c = 0; c < d; ++c) {
      g += widen(Wg, (size_t)i * d + c, wdt) * a[c];
      u += widen(Wu, (size_t)i * d + c, wdt) * a[c];
    }
    double s = 1.0 / (1.0 + exp(-g));
    double silu = g * s;
    h[i] = silu * u;
    double wd_dy = 0.0; /* (Wd^T dy)_i */
    for (int c = 0; c < d; ++c) wd_dy += widen(Wd, (size_t)c * f + i, wdt) * dy[c];
    dw += wd_dy * h[i]; /* <dy, Wd h> summed by i */
    abs_sum += fabs(wd_dy * h[i]);
    double dh = w * wd_dy;
    dg[i] = dh * u * s * (1.0 + g * (1.0 - s));
    du[i] = dh * silu;
  }
  if (da)
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int i = 0; i < f; ++i)
        acc += widen(Wg, (size_t)i * d + c, wdt) * dg[i] + widen(Wu, (size_t)i * d + c, wdt) * du[i];
      da[c] = acc;
    }
  if (dw_abs) *dw_abs = abs_sum;
  return dw;
}

/* ------------------------------------------------------------------------
 * Dense backward of the layer (no BRIM anywhere), the derivative of
 * oracle_dense_layer() for an upstream gradient dY [T, d] (double):
 *   dX[t]    = sum_j dL/da of row (t, j) + sum_s dL/da of shared row (t, s)
 *   dW[t][j] = dL/dw of row (t, j)                     (0 for an empty slot)
 *   dW_abs[t][j] = the sum of |terms| of dW[t][j]        (its condition magnitude)
 * for the tokens in `tokens` (NULL = all T; outputs [n_tok, d], [n_tok, k],
 * [n_tok, k]; any of them may be NULL).
 * Weight gradients, each optional (NULL = not computed), over ALL T tokens:
 *   dWg, dWu [n_exp, f, d], dWd [n_exp, d, f] for the experts listed in
 *   `experts` (n_exp of them), and dSg, dSu [S, fs, d], dSd [S, d, fs].
 * ---------------------------------------------------------------------- */
int oracle_dense_layer_backward(const void* X, int xdt, int T, int d,
                                const int32_t* idx, const double* w, int k,
                                const void* Wg, const void* Wu, const void* Wd, int wdt,
                                int E, int f, int kind,
                                const void* Sg, const void* Su, const void* Sd, int S, int fs,
                                const double* dY, const int32_t* tokens, int n_tok,
                                double* dX, double* dW, double* dW_abs,
                                const int32_t* experts, int n_exp,
                                double* dWg, double* dWu, double* dWd,
                                double* dSg, double* dSu, double* dSd) {
  if (d < 1 || T < 0 || k < 1) return -1;
  if (tokens == NULL) n_tok = T;
  const size_t wg_stride = (size_t)f * d, wd_stride = (size_t)d * f;
  const size_t sg_stride = (size_t)fs * d, sd_stride = (size_t)d * fs;
  const size_t es = esize(wdt);
  const int hmax = (f > fs ? f : fs) > 0 ? (f > fs ? f : fs) : 1;
  int bad = 0;

  /* 1. per-token input gradient and gate-weight gradient */
  if (dX || dW || dW_abs) {
#pragma omp parallel
    {
      double* a = (double*)malloc(sizeof(double) * (size_t)d);
      double* da = (double*)malloc(sizeof(double) * (size_t)d);
      double* h = (double*)malloc(sizeof(double) * (size_t)hmax);
      double* dg = (double*)malloc(sizeof(double) * (size_t)hmax);
      double* du = (double*)malloc(sizeof(double) * (size_t)hmax);
#pragma omp for schedule(dynamic, 1)
      for (int n = 0; n < n_tok; ++n) {
        int t = tokens ? tokens[n] : n;
        if (t < 0 || t >= T) { bad = 1; continue; }
        const double* dy = dY + (size_t)t * d;
        for (int c = 0; c < d; ++c) a[c] = widen(X, (size_t)t * d + c, xdt);
        if (dX)
          for (int c = 0; c < d; ++c) dX[(size_t)n * d + c] = 0.0;
        for (int j = 0; j < k; ++j) {
          int e = idx[(size_t)t * k + j];
          if (dW) dW[(size_t)n * k + j] = 0.0;
          if (dW_abs) dW_abs[(size_t)n * k + j] = 0.0;
          if (e == -1) continue;
          if (e < 0 || e >= E) { bad = 1; continue; }
          double g_abs = 0.0;
          double g = row_backward(kind, a, dy, w[(size_t)t * k + j],
                                  (const char*)Wg + e * wg_stride * es,
                                  (const char*)Wu + e * wg_stride * es,
                                  (const char*)Wd + e * wd_stride * es, wdt, d, f, h, dg, du,
                                  dX ? da : NULL, &g_abs);
          if (dW) dW[(size_t)n * k + j] = g;
          if (dW_abs) dW_abs[(size_t)n * k + j] = g_abs;
          if (dX)
            for (int c = 0; c < d; ++c) dX[(size_t)n * d + c] += da[c];
        }
        if (dX)
          for (int s = 0; s < S; ++s) {
            row_backward(0, a, dy, 1.0, (const char*)Sg + s * sg_stride * es,
                         (const char*)Su + s * sg_stride * es, (const char*)Sd + s * sd_stride * es,
                         wdt, d, fs, h, dg, du, da, NULL);
            for (int c = 0; c < d; ++c) dX[(size_t)n * d + c] += da[c];
          }
      }
      free(a); free(da); free(h); free(dg); free(du);
    }
  }

  /* 2. weight gradients: for each listed expert (then each shared expert),
   *    gather its rows (t ascending, then slot j), compute each row's h, dg,
   *    du, then sum the outer products entry by entry in row order. */
  int n_w = (dWg || dWu || dWd) && kind == 0 ? n_exp : 0;
  int n_s = (dSg || dSu || dSd) ? S : 0;
  for (int q = 0; q < n_w + n_s; ++q) {
    int shared = q >= n_w;
    int e = shared ? q - n_w : experts[q];
    int ff = shared ? fs : f;
    if (!shared && (e < 0 || e >= E)) { bad = 1; continue; }
    const char* g_w = shared ? (const char*)Sg + e * sg_stride * es : (const char*)Wg + e * wg_stride * es;
    const char* u_w = shared ? (const char*)Su + e * sg_stride * es : (const char*)Wu + e * wg_stride * es;
    const char* d_w = shared ? (const char*)Sd + e * sd_stride * es : (const char*)Wd + e * wd_stride * es;
    double* og = shared ? (dSg ? dSg + (size_t)e * sg_stride : NULL) : (dWg ? dWg + (size_t)q * wg_stride : NULL);
    double* ou = shared ? (dSu ? dSu + (size_t)e * sg_stride : NULL) : (dWu ? dWu + (size_t)q * wg_stride : NULL);
    double* od = shared ? (dSd ? dSd + (size_t)e * sd_stride : NULL) : (dWd ? dWd + (size_t)q * wd_stride : NULL);
    /* the rows of this expert */
    int n_rows = 0;
    int32_t* row_t = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T * (shared ? 1 : k) : 1));
    double* row_w = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T * (shared ? 1 : k) : 1));
    for (int t = 0; t < T; ++t) {
      if (shared) { row_t[n_rows] = t; row_w[n_rows++] = 1.0; continue; }
      for (int j = 0; j < k; ++j)
        if (idx[(size_t)t * k + j] == e) { row_t[n_rows] = t; row_w[n_rows++] = w[(size_t)t * k + j]; }
    }
    size_t nr = (size_t)(n_rows > 0 ? n_rows : 1);
    double* A = (double*)malloc(sizeof(double) * nr * d);
    double* H = (double*)malloc(sizeof(double) * nr * ff);
    double* DG = (double*)malloc(sizeof(double) * nr * ff);
    double* DU = (double*)malloc(sizeof(double) * nr * ff);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
      double* a = A + (size_t)r * d;
      for (int c = 0; c < d; ++c) a[c] = widen(X, (size_t)row_t[r] * d + c, xdt);
      row_backward(0, a, dY + (size_t)row_t[r] * d, row_w[r], g_w, u_w, d_w, wdt, d, ff,
                   H + (size_t)r * ff, DG + (size_t)r * ff, DU + (size_t)r * ff, NULL, NULL);
    }
#pragma omp parallel for schedule(static)
    for (int i = 0; i < ff; ++i)
      for (int c = 0; c < d; ++c) {
        double sg = 0.0, su = 0.0, sd = 0.0;
        for (int r = 0; r < n_rows; ++r) {
          double ac = A[(size_t)r * d + c];
          sg += DG[(size_t)r * ff + i] * ac;
          su += DU[(size_t)r * ff + i] * ac;
          sd += row_w[r] * dY[(size_t)row_t[r] * d + c] * H[(size_t)r * ff + i];
        }
        if (og) og[(size_t)i * d + c] = sg;
        if (ou) ou[(size_t)i * d + c] = su;
        if (od) od[(size_t)c * ff + i] = sd;
      }
    free(row_t); free(row_w); free(A); free(H); free(DG); free(DU);
  }
  return bad ? -3 : 0;
}

/* ------------------------------------------------------------------------
 * Routing backward (reading R11): the gradient of the logits from the
 * gradient of the k gate weights, the selection held fixed.  With q the
 * normalised probabilities of R4 -- over all E logits (renorm = 0) or over
 * the k selected ones (renorm = 1, q_e = 0 for the others) -- each gate is
 * w_j = q_{idx_j}, and
 *     dw_j / dl_e = w_j (delta(e, idx_j) - q_e)   for e in the softmax set,
 *                   0                              otherwise,
 *     dL/dl_e     = sum_j dL/dw_j * dw_j / dl_e.
 * The gates are recomputed from the logits (double).  Empty slots (-1)
 * carry no gradient.  dlogits [T, E] double.
 * ---------------------------------------------------------------------- */
int oracle_route_backward(const float* logits, int T, int E, int k, int renorm,
                          const int32_t* idx, const double* dw, double* dlogits) {
  if (T < 0 || E < 1 || k < 1 || k > E) return -1;
  double* q = (double*)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    const int32_t* id = idx + (size_t)t * k;
    double m = (double)l[0];
    for (int e = 1; e < E; ++e)
      if ((double)l[e] > m) m = (double)l[e];
    for (int e = 0; e < E; ++e) {
      int in_set = !renorm;
      for (int j = 0; j < k; ++j)
        if (id[j] == e) in_set = 1;
      q[e] = in_set ? exp((double)l[e] - m) : 0.0;
    }
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += q[e];
    for (int e = 0; e < E; ++e) q[e] /= z;
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) {
        if (id[j] < 0) continue;
        double wj = q[id[j]];
        double jac = wj * ((id[j] == e ? 1.0 : 0.0) - q[e]); /* q_e = 0 off the set */
        acc += dw[(size_t)t * k + j] * jac;
      }
      dlogits[(size_t)t * E + e] = acc;
    }
  }
  free(q);
  return 0;
}

/* ------------------------------------------------------------------------
 * Token shuffling across layers ("Expert Coupling in MoE Pretraining",
 * Abstract: the experts a token selects at one layer predict those it
 * selects at the next; token shuffling moves each token to the GPU predicted
 * to hold its next-layer experts).  Readings R13-R15.
 *
 *   R13 The inter-layer statistic is the pair histogram of a calibration
 *       batch: H[a][b] = #tokens that select expert a at layer l and expert b
 *       at layer l+1 (empty slots, -1, count nothing).
 *   R14 The affinity of layer-l expert a to rank r is
 *       A[a][r] = sum over the layer-(l+1) experts b held by rank r of H[a][b];
 *       a token's predicted rank is the r maximising sum_j A[idx_l[t][j]][r]
 *       (ties -> lower r); a token whose scores are all zero keeps its
 *       contiguous home floor(t * R / T).
 *   R15 The served-locally share counts token-expert assignments of layer l+1
 *       whose expert sits on the token's home rank; the shuffle itself is the
 *       stable reordering of tokens by home rank (a BRIM_0 over one
 *       "expert" per rank).
 * ---------------------------------------------------------------------- */
void oracle_interlayer_histogram(const int32_t* idx_a, const int32_t* idx_b, int T, int k, int E,
                                 uint32_t* H, int accumulate) {
  if (!accumulate)
    for (size_t i = 0; i < (size_t)E * E; ++i) H[i] = 0;
  for (int t = 0; t < T; ++t)
    for (int i = 0; i < k; ++i) {
      int a = idx_a[(size_t)t * k + i];
      if (a < 0 || a >= E) continue;
      for (int j = 0; j < k; ++j) {
        int b = idx_b[(size_t)t * k + j];
        if (b < 0 || b >= E) continue;
        H[(size_t)a * E + b] += 1;
      }
    }
}

int oracle_rank_affinity(const uint32_t* H, int E, const int32_t* slot_of_b, int R,
                         uint64_t* A) {
  if (R < 1 || E % R != 0) return -1;
  const int L = E / R;
  for (int a = 0; a < E; ++a)
    for (int r = 0; r < R; ++r) {
      uint64_t s = 0;
      for (int b = 0; b < E; ++b)
        if (slot_of_b[b] / L == r) s += H[(size_t)a * E + b];
      A[(size_t)a * R + r] = s;
    }
  return 0;
}

void oracle_predict_home(const int32_t* idx_a, int T, int k, int E, const uint64_t* A, int R,
                         int32_t* home) {
  for (int t = 0; t < T; ++t) {
    int best = -1;
    uint64_t best_score = 0;
    for (int r = 0; r < R; ++r) {
      uint64_t s = 0;
      for (int j = 0; j < k; ++j) {
        int a = idx_a[(size_t)t * k + j];
        if (a >= 0 && a < E) s += A[(size_t)a * R + r];
      }
      if (best < 0 || s > best_score) { best = r; best_score = s; } /* ties keep the lower r */
    }
    home[t] = best_score > 0 ? best : (int32_t)(((int64_t)t * R) / T);
  }
}

/* out[0] = assignments of layer-l+1 experts held by the token's home rank,
 * out[1] = all assignments (slots that are not empty).  home == NULL means
 * the contiguous home floor(t * R / T). */
int oracle_count_local(const int32_t* idx, int T, int k, const int32_t* slot_of, int E, int R,
                       const int32_t* home, int64_t* out) {
  if (R < 1 || E % R != 0) return -1;
  const int L = E / R;
  out[0] = out[1] = 0;
  for (int t = 0; t < T; ++t) {
    int h = home ? home[t] : (int)(((int64_t)t * R) / T);
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) continue;
      out[1] += 1;
      if (slot_of[e] / L == h) out[0] += 1;
    }
  }
  return 0;
}
