/*
 * CPU oracle for head-aware paged attention (SegPagedAttention).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library.  It shares no code,
 * header, table or constant with the CUDA path.
 *
 * What it computes is the plain definition the method must reproduce: dense
 * attention over the full causal context with an explicit per-head visibility
 * mask, accumulated in fp64.  The method's claim is that evaluating each head
 * over only the tokens it stores gives this same result ("SegPagedAttention
 * runtime design", §4: verify_against_dense compares against a dense + mask
 * baseline and asks for cosine > 0.99998).
 *
 * Head kinds ("SegPagedAttention runtime design", §1 and §3; "RedKnot head
 * classification", the four-kind table):
 *   GLOBAL reads the whole causal prefix; DENSE reads the whole prefix as well
 *   (its RoPE re-alignment belongs to KV reuse, not to attention);
 *   LOCAL reads only the first `sink` tokens of the sequence and the `window`
 *   most recent tokens;
 *   RETRIEVAL has the whole prefix as candidates but keeps only its top-p
 *   important tokens, fetched page by page (the four-kind table; runtime
 *   design, closing summary: retrieval heads fetch pages on demand).  Reading
 *   taken: importance is given per block of `block` consecutive positions
 *   [i*block, (i+1)*block) (one page of the cache); the head keeps the sink and
 *   the recent window like a LOCAL head plus the smallest set of blocks, taken
 *   in decreasing order of importance (ties: lower block first), whose
 *   importance reaches the fraction top_p of the total over the candidate
 *   blocks (those holding a position >= sink); top_p >= 1 keeps every block,
 *   top_p <= 0 none.  Sums run in fp64 in that order.
 * Readings where the pages are silent: the recent window counts the query's
 * own position (positions p-window+1 .. p); sinks are absolute positions
 * 0 .. sink-1 of the sequence; an overlap of sink and window is a plain union.
 *
 * Parity pins: O1 is checked in the tests against a brute-force enumeration of
 * the visible set, against ordinary causal attention for GLOBAL heads, and
 * against closed forms (window 1, equal keys).  See tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Kind codes of this file only: 0 global, 1 local, 2 dense, 3 retrieval. */
#define ORACLE_GLOBAL 0
#define ORACLE_LOCAL 1
#define ORACLE_DENSE 2
#define ORACLE_RETRIEVAL 3

/* Does query position p see key position j?  Causal for every kind; a local
 * head additionally needs j among the first `sink` positions or among the
 * `window` most recent positions ending at p; a retrieval head sees those and
 * every position of a kept block (sel[j / block] != 0). */
static int oracle_sees(int kind, int64_t sink, int64_t window, const uint8_t* sel, int64_t block, int64_t p,
                       int64_t j) {
  if (j > p) return 0;
  if (kind == ORACLE_GLOBAL || kind == ORACLE_DENSE) return 1;
  if ((j < sink) || (j >= p - window + 1)) return 1;
  return kind == ORACLE_RETRIEVAL && sel[j / block] != 0;
}

/*
 * Blocks a retrieval head keeps (the reading in the header above).
 *   L, block   context length and block size (positions per block; the page size)
 *   sink       the head's sink; blocks entirely inside [0, sink) are not candidates
 *   top_p      fraction of the candidates' total importance to reach
 *   mass       [ceil(L / block)] non-negative importance of each block
 *   sel        [ceil(L / block)] out: 1 for a kept block, else 0
 * Returns the number of kept blocks, or -1 for a negative or non-finite mass.
 */
int64_t oracle_retrieval_select(int64_t L, int64_t block, int64_t sink, float top_p, const float* mass,
                                uint8_t* sel) {
  const int64_t n = (L + block - 1) / block;
  int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
  uint8_t* taken = (uint8_t*)calloc((size_t)(n > 0 ? n : 1), 1);
  int64_t nc = 0;
  for (int64_t i = 0; i < n; ++i) {
    sel[i] = 0;
    if (!(mass[i] >= 0.0f) || isinf(mass[i])) {
      free(order);
      free(taken);
      return -1;
    }
  }
  /* candidates in decreasing importance, ties by lower index: repeated selection of the largest */
  for (;;) {
    int64_t best = -1;
    for (int64_t i = 0; i < n; ++i) {
      if (taken[i] || (i + 1) * block <= sink) continue;
      if (best < 0 || mass[i] > mass[best]) best = i;
    }
    if (best < 0) break;
    taken[best] = 1;
    order[nc++] = best;
  }
  double total = 0.0;
  for (int64_t k = 0; k < nc; ++k) total += (double)mass[order[k]];
  int64_t keep = nc;
  if (top_p <= 0.0f) {
    keep = 0;
  } else if (top_p < 1.0f) {
    const double target = (double)top_p * total;
    double run = 0.0;
    for (int64_t k = 0; k <= nc; ++k) {
      if (run >= target) {
        keep = k;
        break;
      }
      if (k < nc) run += (double)mass[order[k]];
    }
  }
  for (int64_t k = 0; k < keep; ++k) sel[order[k]] = 1;
  free(order);
  free(taken);
  return keep;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * One query row against the dense K/V of its kv-head (the definition itself):
 * scores s_j = scale * <q, k_j> over the visible j, m = max_j s_j,
 * e_j = exp(s_j - m), O = sum_j e_j v_j / sum_j e_j, LSE = m + ln sum_j e_j.
 * `s` and `vis` are scratch of L entries.  Returns 0, or -1 if the position
 * lies outside [0, L) or the row sees nothing.
 */
static int oracle_one_row(int64_t d, const double* qr, int64_t p, int64_t L, const double* k,
                          const double* v, int kind, int64_t sink, int64_t window, const uint8_t* sel,
                          int64_t block, double scale, double* o, double* lse, double* s, char* vis) {
  if (p < 0 || p >= L) return -1;
  double m = -INFINITY;
  int64_t nvis = 0;
  for (int64_t j = 0; j < L; ++j) {
    vis[j] = (char)oracle_sees(kind, sink, window, sel, block, p, j);
    if (!vis[j]) continue;
    double acc = 0.0;
    for (int64_t t = 0; t < d; ++t) acc += qr[t] * k[j * d + t];
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
    ++nvis;
  }
  if (nvis == 0) return -1;
  double denom = 0.0;
  for (int64_t t = 0; t < d; ++t) o[t] = 0.0;
  for (int64_t j = 0; j < L; ++j) {
    if (!vis[j]) continue;
    const double e = exp(s[j] - m);
    denom += e;
    for (int64_t t = 0; t < d; ++t) o[t] += e * v[j * d + t];
  }
  for (int64_t t = 0; t < d; ++t) o[t] /= denom;
  *lse = m + log(denom);
  return 0;
}

/*
 * Attention of n_rows query rows of one (sequence, query-head) against the
 * dense K/V of its kv-head.
 *   q    [n_rows][d]   fp64, post-RoPE queries
 *   pos  [n_rows]      absolute position p of each query row
 *   k, v [L][d]        dense keys / values of the kv-head, positions 0 .. L-1
 *   out  [n_rows][d]   O = sum_j e_j v_j / sum_j e_j over visible j
 *   lse  [n_rows]      m + ln sum_j e_j,  e_j = exp(s_j - m), m = max_j s_j
 *   sel, block  retrieval heads: kept blocks (oracle_retrieval_select) and
 *               the block size; ignored (may be NULL / 0) for other kinds
 * Scores are s_j = scale * <q, k_j>.  Returns 0, or -1 if a row sees nothing
 * or a position lies outside [0, L).  Rows run in parallel (OpenMP).
 */
int oracle_attention_rows(int64_t n_rows, int64_t d, const double* q, const int64_t* pos,
                          int64_t L, const double* k, const double* v, int kind,
                          int64_t sink, int64_t window, const uint8_t* sel, int64_t block,
                          double scale, double* out, double* lse) {
  int bad = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    char* vis = (char*)malloc((size_t)(L > 0 ? L : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      if (oracle_one_row(d, q + r * d, pos[r], L, k, v, kind, sink, window, sel, block, scale, out + r * d,
                         lse + r, s, vis) != 0) {
#pragma omp atomic write
        bad = 1;
      }
    }
    free(s);
    free(vis);
  }
  return bad ? -1 : 0;
}

/*
 * The same computation for rows of many (sequence, kv-head) groups in one
 * parallel loop, so that a batch of small groups (a decode step: a handful
 * of rows per group) keeps every host core busy.  Row r uses group
 * group_of[r]: its dense K/V k[g], v[g] ([L[g]][d]) and its policy kind[g],
 * sink[g], window[g] (retrieval: kept blocks sel[g], block size block[g]).
 * Each row's arithmetic is oracle_one_row, exactly as in
 * oracle_attention_rows.  Returns 0, or -1 as oracle_attention_rows.
 */
int oracle_attention_batch(int64_t n_rows, int64_t d, const double* q, const int64_t* pos,
                           const int64_t* group_of, int64_t n_groups, const int64_t* L,
                           const double* const* k, const double* const* v, const int* kind,
                           const int64_t* sink, const int64_t* window, const uint8_t* const* sel,
                           const int64_t* block, double scale, double* out, double* lse) {
  int bad = 0;
  int64_t lmax = 1;
  for (int64_t g = 0; g < n_groups; ++g)
    if (L[g] > lmax) lmax = L[g];
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)lmax);
    char* vis = (char*)malloc((size_t)lmax);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      const int64_t g = group_of[r];
      if (g < 0 || g >= n_groups ||
          oracle_one_row(d, q + r * d, pos[r], L[g], k[g], v[g], kind[g], sink[g], window[g], sel[g],
                         block[g], scale, out + r * d, lse + r, s, vis) != 0) {
#pragma omp atomic write
        bad = 1;
      }
    }
    free(s);
    free(vis);
  }
  return bad ? -1 : 0;
}

/*
 * Which positions of a (sequence, kv-head) the cache must keep so that every
 * query of a call with queries at positions q0 .. L-1 finds its visible keys:
 * the union of the queries' visible sets ("SegPagedAttention runtime design",
 * §3: build_segpaged_cache keeps only the tokens a local head can see).
 * mask[j] = 1 if position j is kept.  Returns the number kept.  sel / block as in
 * oracle_attention_rows.
 */
int64_t oracle_stored_mask(int kind, int64_t sink, int64_t window, const uint8_t* sel, int64_t block,
                           int64_t L, int64_t q0, uint8_t* mask) {
  int64_t n = 0;
  for (int64_t j = 0; j < L; ++j) {
    uint8_t keep = 0;
    for (int64_t p = q0; p < L && !keep; ++p) keep = (uint8_t)oracle_sees(kind, sink, window, sel, block, p, j);
    mask[j] = keep;
    n += keep;
  }
  return n;
}

/*
 * Number of (query, key) pairs a call evaluates: sum over query positions
 * q0 .. L-1 of the size of the visible set.  Used for the visible-FLOP ledger
 * (4 * d FLOPs per pair: QK^T and PV, a multiply and an add each).
 */
int64_t oracle_visible_pairs(int kind, int64_t sink, int64_t window, const uint8_t* sel, int64_t block,
                             int64_t L, int64_t q0) {
  int64_t n = 0;
  for (int64_t p = q0; p < L; ++p)
    for (int64_t j = 0; j <= p; ++j) n += oracle_sees(kind, sink, window, sel, block, p, j);
  return n;
}

/*
 * FP8 E4M3 codes for KV pages quantised with a per-layer scale (the pages
 * say only that the system works with FP8 quantisation; the plainest
 * reading is a per-layer scale, code = round(x * inv_scale), value =
 * code * scale).  E4M3 as defined by the OCP 8-bit floating point format:
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite magnitude 448 = 1.75 * 2^8, subnormals
 * m * 2^-9.  Encoding rounds to nearest, ties to even, and saturates finite
 * values to +-448.  The product x * inv_scale is formed in fp32 (the
 * precision in which the GPU takes the same decision).
 */
static double oracle_e4m3_value(uint8_t c) {
  const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return sgn ? -mag : mag;
}

static uint8_t oracle_e4m3_encode_f32(float xf) {
  const double x = (double)xf;
  if (x != x) return 0x7F;
  const uint8_t sgn = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0;
  const double a = fabs(x);
  if (a >= 448.0) return sgn | 0x7E;
  /* The values of codes 0 .. 0x7E increase with the code: find the first
   * code whose value is >= a, then take the nearer of it and the code below
   * (a tie goes to the even code). */
  int lo = 0, hi = 0x7E;
  while (lo < hi) {
    const int mid = (lo + hi) / 2;
    if (oracle_e4m3_value((uint8_t)mid) >= a) hi = mid;
    else lo = mid + 1;
  }
  uint8_t best = (uint8_t)lo;
  if (lo > 0) {
    const double up = oracle_e4m3_value((uint8_t)lo) - a, down = a - oracle_e4m3_value((uint8_t)(lo - 1));
    if (down < up || (down == up && ((lo - 1) & 1) == 0)) best = (uint8_t)(lo - 1);
  }
  return sgn | best;
}

/* codes[i] = E4M3 code of fp32(x[i] * inv_scale) (x[i] given as float). */
void oracle_e4m3_encode(int64_t n, const float* x, float inv_scale, uint8_t* codes) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode_f32(x[i] * inv_scale);
}

/* values[i] = value of codes[i] times scale, in fp64. */
void oracle_e4m3_decode(int64_t n, const uint8_t* codes, double scale, double* values) {
  for (int64_t i = 0; i < n; ++i) values[i] = oracle_e4m3_value(codes[i]) * scale;
}

/*
 * Attention mass per block: the scoring pass that gives a RETRIEVAL head its
 * importance.  The pages leave the scoring rule open; the reading taken is
 * the head's own attention mass per page (four-kind table, retrieval row:
 * the important tokens are the ones the head attends to).  For the query at
 * the last position p = L - 1 of a sequence, over its whole causal context
 * [0, L), in fp64:
 *   s_hj = scale * q_h . k_j,  a_hj = exp(s_hj - max_j s_hj) / sum_j exp(s_hj - max_j s_hj)
 *   mass_i = (1 / g) * sum_h sum_{j in [i*block, min((i+1)*block, L))} a_hj
 * i.e. the softmax probability each of the kv-head's g q-heads puts on block
 * i, averaged over the group.  q [g][d], k [L][d]; mass [ceil(L / block)] out.
 * Returns 0, or -1 for sizes < 1.
 */
int oracle_block_mass(int64_t g, int64_t d, const double* q, int64_t L, const double* k, double scale,
                      int64_t block, double* mass) {
  if (g < 1 || d < 1 || L < 1 || block < 1) return -1;
  const int64_t nb = (L + block - 1) / block;
  for (int64_t i = 0; i < nb; ++i) mass[i] = 0.0;
  double* a = (double*)malloc((size_t)L * sizeof(double));
  if (!a) return -1;
  for (int64_t h = 0; h < g; ++h) {
    const double* qh = q + h * d;
    double m = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
      double acc = 0.0;
      for (int64_t t = 0; t < d; ++t) acc += qh[t] * k[j * d + t];
      a[j] = scale * acc;
      if (a[j] > m) m = a[j];
    }
    double z = 0.0;
    for (int64_t j = 0; j < L; ++j) {
      a[j] = exp(a[j] - m);
      z += a[j];
    }
    for (int64_t j = 0; j < L; ++j) mass[j / block] += a[j] / z / (double)g;
  }
  free(a);
  return 0;
}
