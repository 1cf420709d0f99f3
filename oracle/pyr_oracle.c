/*
 * CPU oracle for hierarchical (pyramid) top-K key-block selection followed by
 * causal block-sparse attention. TEST INFRASTRUCTURE ONLY: the tests, the
 * smoke check and the benchmark's CPU-baseline leg call it; the product path
 * never does.
 *
 * Plain, slow and written for reading: double accumulation, no blocking, no
 * fusion, one function per step of the method. It shares no code, header or
 * table with the CUDA library.
 *
 * What it computes (sources):
 *   PISA abstract (peercurrent record, the PISA paragraph): keys are pooled
 *     into a coarse-to-fine hierarchy of O(log N) levels; selection starts at
 *     the coarsest level; at each level LogSumExp scoring is applied to a
 *     bounded candidate set and the survivors' children become the next
 *     level's candidates, until the finest level is reached.
 *   PHBA summary (paperlayer.ai, A.1.2 "Routing metadata kernels"): block
 *     centroids are the average of the block's key rows; routes go only to
 *     strictly preceding blocks and unavailable route slots hold -1.
 *   PHBA summary (3.1 "Top-K block routing", A.1.3 "Query-tile fused sparse
 *     forward kernel"): the current block is always attended with local
 *     causal attention; attention over the routed blocks is an online-softmax
 *     merge equal to one softmax over the union of the attended keys, and the
 *     forward pass also writes the log-sum-exp.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes):
 *   - pooling operator: arithmetic mean; node (l, m) covers level-0 blocks
 *     [m 2^l, min((m+1) 2^l, nb)); levels l = 0 .. L, L = ceil(log2 nb);
 *   - node score for query block i:
 *       S = ln sum_{rows r of block i (all heads of the kv group)}
 *               exp(q_r . kbar / sqrt(d)) + ln n_valid,
 *     where kbar and n_valid are the mean and token count of the node's
 *     causally valid part (its blocks < i); nodes starting at or after i are
 *     never candidates;
 *   - the walk starts at s0 = smallest level with at most `cap` nodes, all of
 *     whose valid nodes are candidates (equivalent to starting at the root,
 *     because every level above s0 has at most cap/2 nodes); each level > 0
 *     keeps min(cap/2, #candidates) nodes, level 0 keeps min(topk, #cand);
 *     ties go to the lower node index; survivors expand to their existing,
 *     valid children {2m, 2m+1};
 *   - idx lists the kept level-0 blocks ascending, padded with -1; the
 *     current (diagonal) block is not listed and is always attended;
 *   - gap = min over scored levels of (score of last kept - score of first
 *     dropped), +inf when a level drops nothing.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int B, Hq, Hkv; /* batch, query heads, kv heads (Hq % Hkv == 0) */
  int N;          /* key/value length */
  int Nq;         /* query rows; row t sits at position q_offset + t */
  int q_offset;
  int d;          /* head dim */
  int b;          /* block size (keys per block, query rows per block) */
  int topk, cap;  /* final K and per-level candidate cap */
  int dtype;      /* 0 = fp32, 1 = bf16, 2 = fp64 (oracle only: finite-difference pins) */
} ora_shape;

enum { ORA_OK = 0, ORA_EINVAL = 1, ORA_EBADIDX = 2 };

/* ---- element access ---------------------------------------------------- */

static double elem(const void* base, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)base)[i];
  if (dtype == 2) return ((const double*)base)[i];
  uint32_t u = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---- pyramid geometry --------------------------------------------------- */

static int64_t num_blocks(const ora_shape* s) { return ((int64_t)s->N + s->b - 1) / s->b; }

/* L = ceil(log2 nb): the number of pooling steps above level 0. */
static int top_level(int64_t nb) {
  int L = 0;
  while (((int64_t)1 << L) < nb) L++;
  return L;
}

static int64_t level_nodes(int64_t nb, int l) { return (nb + ((int64_t)1 << l) - 1) >> l; }

static int64_t level_offset(int64_t nb, int l) {
  int64_t off = 0;
  for (int k = 0; k < l; k++) off += level_nodes(nb, k);
  return off;
}

int ora_num_levels(const ora_shape* s) { return top_level(num_blocks(s)) + 1; }

int64_t ora_num_nodes(const ora_shape* s) {
  int64_t nb = num_blocks(s), P = 0;
  for (int l = 0; l <= top_level(nb); l++) P += level_nodes(nb, l);
  return P;
}

/* tokens in level-0 blocks [j0, j1) */
static int64_t tokens_in(const ora_shape* s, int64_t j0, int64_t j1) {
  int64_t t0 = j0 * s->b, t1 = j1 * s->b;
  if (t1 > s->N) t1 = s->N;
  return t1 > t0 ? t1 - t0 : 0;
}

int64_t ora_first_qblock(const ora_shape* s) { return s->q_offset / s->b; }

int64_t ora_num_qblocks(const ora_shape* s) {
  return (s->q_offset + s->Nq - 1) / s->b - s->q_offset / s->b + 1;
}

/* ---- step 1: key pyramid (mean pooling) -------------------------------- */

/*
 * Pyramid of one (batch, kv head) unit, level-major, level 0 first:
 * out[(level_offset(l) + m) * d + e] = mean of the keys under node (l, m).
 * Level 0 is the per-block mean of the key rows (PHBA centroids); a node at
 * level l > 0 is the token-weighted mean of the level-0 blocks it covers,
 * which equals the mean of all of its keys.
 */
static void pyramid_unit(const ora_shape* s, const void* K, int64_t unit, double* out) {
  const int d = s->d;
  const int64_t nb = num_blocks(s);
  const int L = top_level(nb);
  const int64_t kbase = unit * (int64_t)s->N * d;
  for (int64_t j = 0; j < nb; j++) {
    const int64_t t0 = j * s->b, t1 = (j + 1) * s->b < s->N ? (j + 1) * s->b : s->N;
    for (int e = 0; e < d; e++) {
      double acc = 0.0;
      for (int64_t t = t0; t < t1; t++) acc += elem(K, s->dtype, kbase + t * d + e);
      out[j * d + e] = acc / (double)(t1 - t0);
    }
  }
  for (int l = 1; l <= L; l++) {
    const int64_t off = level_offset(nb, l), n = level_nodes(nb, l);
    for (int64_t m = 0; m < n; m++) {
      const int64_t j0 = m << l, j1 = ((m + 1) << l) < nb ? ((m + 1) << l) : nb;
      const double cnt = (double)tokens_in(s, j0, j1);
      for (int e = 0; e < d; e++) {
        double acc = 0.0;
        for (int64_t j = j0; j < j1; j++) acc += (double)tokens_in(s, j, j + 1) * out[j * d + e];
        out[(off + m) * d + e] = acc / cnt;
      }
    }
  }
}

/* Pyramids of the listed units: out is [nunits][P][d]. */
int ora_pyramid(const ora_shape* s, const void* K, int nunits, const int32_t* units, double* out) {
  if (!s || !K || !units || !out || s->d <= 0 || s->b <= 0 || s->N <= 0) return ORA_EINVAL;
  const int64_t P = ora_num_nodes(s);
#pragma omp parallel for schedule(dynamic)
  for (int u = 0; u < nunits; u++) pyramid_unit(s, K, units[u], out + (int64_t)u * P * s->d);
  return ORA_OK;
}

/* ---- step 2: LogSumExp score of one node for one query block ----------- */

/* Query rows of query block i for kv head hk of batch bi: every row of the
 * G heads that share hk whose position lies in block i. */
static int gather_rows(const ora_shape* s, const void* Q, int64_t bi, int64_t hk, int64_t i, double* rows) {
  const int G = s->Hq / s->Hkv, d = s->d;
  int64_t p0 = i * s->b, p1 = (i + 1) * s->b;
  if (p0 < s->q_offset) p0 = s->q_offset;
  if (p1 > s->q_offset + s->Nq) p1 = s->q_offset + s->Nq;
  int nr = 0;
  for (int g = 0; g < G; g++) {
    const int64_t hq = hk * G + g;
    for (int64_t p = p0; p < p1; p++) {
      const int64_t base = ((bi * s->Hq + hq) * (int64_t)s->Nq + (p - s->q_offset)) * d;
      for (int e = 0; e < d; e++) rows[(int64_t)nr * d + e] = elem(Q, s->dtype, base + e);
      nr++;
    }
  }
  return nr;
}

/*
 * Score of node (l, m) for query block i, given the unit's pyramid.
 * Returns 0 and writes *score, *nvalid when the node has a valid part,
 * 1 when it lies entirely at or after block i (not a candidate).
 */
static int node_score(const ora_shape* s, const double* pyr, const double* rows, int nr, int64_t i, int l,
                      int64_t m, double* kbar, double* score, double* nvalid) {
  const int d = s->d;
  const int64_t nb = num_blocks(s);
  const int64_t j0 = m << l;
  int64_t j1 = ((m + 1) << l) < nb ? ((m + 1) << l) : nb;
  if (j0 >= i) return 1;
  if (j1 <= i) {
    const double* mean = pyr + (level_offset(nb, l) + m) * d;
    for (int e = 0; e < d; e++) kbar[e] = mean[e];
  } else {
    /* the node straddles block i: mean over its valid blocks [j0, i) only */
    j1 = i;
    const double cnt = (double)tokens_in(s, j0, j1);
    for (int e = 0; e < d; e++) {
      double acc = 0.0;
      for (int64_t j = j0; j < j1; j++) acc += (double)tokens_in(s, j, j + 1) * pyr[j * d + e];
      kbar[e] = acc / cnt;
    }
  }
  const double n = (double)tokens_in(s, j0, j1);
  const double scale = 1.0 / sqrt((double)d);
  double mx = -INFINITY;
  double* x = (double*)malloc(sizeof(double) * (size_t)(nr > 0 ? nr : 1));
  for (int r = 0; r < nr; r++) {
    double dot = 0.0;
    for (int e = 0; e < d; e++) dot += rows[(int64_t)r * d + e] * kbar[e];
    x[r] = dot * scale;
    if (x[r] > mx) mx = x[r];
  }
  double sum = 0.0;
  for (int r = 0; r < nr; r++) sum += exp(x[r] - mx);
  free(x);
  *score = mx + log(sum) + log(n);
  *nvalid = n;
  return 0;
}

/* Public: score of node (level, m) for (unit, relative query block u). */
int ora_node_score(const ora_shape* s, const void* Q, const double* pyr_unit, int32_t unit, int64_t u, int level,
                   int64_t m, double* score, double* nvalid) {
  if (!s || !Q || !pyr_unit || !score || !nvalid) return ORA_EINVAL;
  const int64_t bi = unit / s->Hkv, hk = unit % s->Hkv;
  const int64_t i = ora_first_qblock(s) + u;
  const int G = s->Hq / s->Hkv;
  double* rows = (double*)malloc(sizeof(double) * (size_t)G * s->b * s->d);
  double* kbar = (double*)malloc(sizeof(double) * (size_t)s->d);
  const int nr = gather_rows(s, Q, bi, hk, i, rows);
  const int rc = node_score(s, pyr_unit, rows, nr, i, level, m, kbar, score, nvalid);
  free(rows);
  free(kbar);
  if (rc) {
    *score = -INFINITY;
    *nvalid = 0.0;
  }
  return rc ? 3 : ORA_OK;
}

/* ---- step 3: coarse-to-fine walk --------------------------------------- */

typedef struct {
  int64_t m;
  double score;
} cand_t;

/* descending score; equal scores: lower node index first */
static int before(const cand_t* a, const cand_t* b) {
  if (a->score != b->score) return a->score > b->score;
  return a->m < b->m;
}

static void sort_candidates(cand_t* c, int n) {
  for (int k = 1; k < n; k++) {
    cand_t v = c[k];
    int p = k - 1;
    while (p >= 0 && before(&v, &c[p])) {
      c[p + 1] = c[p];
      p--;
    }
    c[p + 1] = v;
  }
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Selection variants of the PHAROS page ("Four mechanisms powering PHAROS"),
 * all off by default (a zeroed struct or NULL gives the plain walk above):
 *   budget     depth-sounding budget allocation (DBA): token budgets differ
 *              across heads. budget[unit] (unit = batch * Hkv + kv head) is
 *              the number of level-0 blocks that unit's walk keeps, clamped
 *              to [0, topk]; NULL: topk - fcf_extra for every unit. The page
 *              derives budgets from attention-head entropy but gives no
 *              formula, so the budgets are an input.
 *   fcf_tau,   fog-gate confidence fallback (FCF): the budget grows when
 *   fcf_extra  confidence is low. Confidence is the walk's smallest margin
 *              between the last kept and the first dropped candidate over the
 *              levels above 0 and at the level-0 budget boundary; when it is
 *              below fcf_tau, level 0 keeps min(budget + fcf_extra, topk).
 *              fcf_extra = 0: off.
 *   rcg_lambda range-light cross-level guidance (RCG): coarse-level scores
 *              guide the finer levels. Candidates are ranked by
 *              R = S + rcg_lambda * R(parent), R = S at the start level;
 *              0: off (rank by S).
 */
typedef struct {
  const int32_t* budget; /* [B * Hkv] or NULL */
  double fcf_tau;
  int fcf_extra;
  double rcg_lambda;
} ora_select_opts;

/* Levels a trace holds: the start level s0 (the finest level with at most cap
 * nodes) down to 0. */
int ora_trace_levels(const ora_shape* s) {
  const int64_t nb = num_blocks(s);
  int s0 = 0;
  while (level_nodes(nb, s0) > s->cap) s0++;
  return s0 + 1;
}

/* Entries per trace level: the most nodes any level keeps. */
int ora_trace_width(const ora_shape* s) { return s->cap / 2 > s->topk ? s->cap / 2 : s->topk; }

/*
 * Selection for (unit, query block i). Writes idx[0..topk) (ascending, -1
 * padded), *gap, and, when ncand is given, the number of candidates scored at
 * each level (ncand[l], l = 0..L; zero for levels not scored). When trace is
 * given ([s0 + 1][ora_trace_width] entries), row s0 - l lists the nodes kept at
 * level l, best first, then -1.
 * start_level < 0 starts at s0; otherwise at the given level (used by tests
 * to check that starting at the root gives the same answer).
 * gap is the smallest margin of any decision the walk took: last kept minus
 * first dropped at every level that dropped a candidate (at the level-0
 * boundary actually used) and, when FCF could change the result, the distance
 * between the confidence and fcf_tau.
 */
static void select_one(const ora_shape* s, const void* Q, const double* pyr, int64_t unit, int64_t i, int start_level,
                       const ora_select_opts* opt, int32_t* idx, double* gap, int32_t* ncand, int32_t* trace) {
  const int d = s->d, G = s->Hq / s->Hkv;
  const int64_t nb = num_blocks(s);
  const int L = top_level(nb);
  const int64_t bi = unit / s->Hkv, hk = unit % s->Hkv;
  double* rows = (double*)malloc(sizeof(double) * (size_t)G * s->b * d);
  double* kbar = (double*)malloc(sizeof(double) * (size_t)d);
  const int nr = gather_rows(s, Q, bi, hk, i, rows);
  const int extra = opt ? opt->fcf_extra : 0;
  const double lambda = opt ? opt->rcg_lambda : 0.0;
  int base = (opt && opt->budget) ? opt->budget[unit] : s->topk - extra;
  if (base < 0) base = 0;
  if (base > s->topk) base = s->topk;

  int s0 = 0;
  while (level_nodes(nb, s0) > s->cap) s0++;
  if (start_level >= 0) s0 = start_level > L ? L : start_level;
  const int tw = ora_trace_width(s);
  if (trace)
    for (int k = 0; k < (s0 + 1) * tw; k++) trace[k] = -1;

  /* candidate lists hold at most max(cap, n_s0) nodes; score is the ranking
   * score R, parent the parent's R (0 at the start level) */
  int64_t room = level_nodes(nb, s0);
  if (room < s->cap) room = s->cap;
  if (room < 2) room = 2;
  cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)room * 2);
  cand_t* next = (cand_t*)malloc(sizeof(cand_t) * (size_t)room * 2);
  double* parent = (double*)malloc(sizeof(double) * (size_t)room * 2);
  double* next_parent = (double*)malloc(sizeof(double) * (size_t)room * 2);
  int nc = 0;
  for (int64_t m = 0; m < level_nodes(nb, s0); m++)
    if ((m << s0) < i) {
      parent[nc] = 0.0;
      cand[nc++].m = m;
    }

  if (ncand)
    for (int l = 0; l <= L; l++) ncand[l] = 0;
  double g = INFINITY;    /* smallest decision margin */
  double conf = INFINITY; /* smallest margin above level 0 (FCF confidence) */
  for (int k = 0; k < s->topk; k++) idx[k] = -1;

  for (int l = s0; l >= 0; l--) {
    for (int c = 0; c < nc; c++) {
      double nv, sc;
      node_score(s, pyr, rows, nr, i, l, cand[c].m, kbar, &sc, &nv);
      cand[c].score = sc + lambda * parent[c];
    }
    if (ncand) ncand[l] = nc;
    sort_candidates(cand, nc);
    int keep;
    if (l > 0) {
      const int want = s->cap / 2;
      keep = nc < want ? nc : want;
      if (keep < nc && keep > 0) {
        const double gl = cand[keep - 1].score - cand[keep].score;
        if (gl < g) g = gl;
        if (gl < conf) conf = gl;
      }
    } else {
      const int keep_base = nc < base ? nc : base;
      keep = keep_base;
      if (extra > 0) {
        double c0 = conf;
        if (keep_base < nc && keep_base > 0) {
          const double gb = cand[keep_base - 1].score - cand[keep_base].score;
          if (gb < c0) c0 = gb;
        }
        int wide = base + extra < s->topk ? base + extra : s->topk;
        if (wide > nc) wide = nc;
        if (c0 < opt->fcf_tau) keep = wide;
        if (wide != keep_base) {
          /* the fallback decision changes the result: its margin counts */
          const double gt = fabs(c0 - opt->fcf_tau);
          if (gt < g) g = gt;
        }
      }
      if (keep < nc && keep > 0) {
        const double gl = cand[keep - 1].score - cand[keep].score;
        if (gl < g) g = gl;
      }
    }
    if (trace)
      for (int k = 0; k < keep; k++) trace[(s0 - l) * tw + k] = (int32_t)cand[k].m;
    if (l == 0) {
      for (int k = 0; k < keep; k++) idx[k] = (int32_t)cand[k].m;
      qsort(idx, (size_t)keep, sizeof(int32_t), cmp_i32);
      break;
    }
    const int64_t nchild = level_nodes(nb, l - 1);
    int nn = 0;
    for (int k = 0; k < keep; k++)
      for (int64_t ch = 2 * cand[k].m; ch <= 2 * cand[k].m + 1; ch++)
        if (ch < nchild && (ch << (l - 1)) < i) {
          next_parent[nn] = cand[k].score;
          next[nn++].m = ch;
        }
    cand_t* t = cand;
    cand = next;
    next = t;
    double* tp = parent;
    parent = next_parent;
    next_parent = tp;
    nc = nn;
  }
  *gap = g;
  free(cand);
  free(next);
  free(parent);
  free(next_parent);
  free(rows);
  free(kbar);
}

/*
 * Selection for a list of items. Item k is (slot[k], qb[k]): slot indexes
 * units[] and pyr ([nunits][P][d], the pyramids of those units, as written
 * by ora_pyramid); qb is the query block relative to the first query block.
 * opt: the PHAROS variants (NULL: plain walk); opt->budget is indexed by the
 * global unit id units[slot]. idx: [nitems][topk]; gap: [nitems] (nullable);
 * ncand: [nitems][L+1] (nullable); trace: [nitems][levels][width] with
 * levels = s0 + 1 of the walk's start level (ora_trace_levels unless
 * start_level is given) and width = ora_trace_width (nullable).
 */
int ora_select_ex(const ora_shape* s, const void* Q, const double* pyr, int nunits, const int32_t* units, int nitems,
                  const int32_t* slot, const int64_t* qb, int start_level, const ora_select_opts* opt, int32_t* idx,
                  double* gap, int32_t* ncand, int32_t* trace) {
  if (!s || !Q || !pyr || !units || !slot || !qb || !idx) return ORA_EINVAL;
  if (s->cap < 2 || s->cap % 2 || s->topk < 0 || s->Hq % s->Hkv) return ORA_EINVAL;
  if (opt && (opt->fcf_extra < 0 || opt->fcf_tau != opt->fcf_tau || opt->rcg_lambda != opt->rcg_lambda))
    return ORA_EINVAL;
  const int64_t P = ora_num_nodes(s);
  const int nl = ora_num_levels(s);
  const int64_t nqb = ora_num_qblocks(s);
  int tl = ora_trace_levels(s);
  if (start_level >= 0) tl = (start_level > nl - 1 ? nl - 1 : start_level) + 1;
  const int64_t tstride = (int64_t)tl * ora_trace_width(s);
  for (int k = 0; k < nitems; k++)
    if (slot[k] < 0 || slot[k] >= nunits || qb[k] < 0 || qb[k] >= nqb) return ORA_EINVAL;
#pragma omp parallel for schedule(dynamic)
  for (int k = 0; k < nitems; k++) {
    double gk;
    const int64_t i = ora_first_qblock(s) + qb[k];
    select_one(s, Q, pyr + (int64_t)slot[k] * P * s->d, units[slot[k]], i, start_level, opt,
               idx + (int64_t)k * s->topk, &gk, ncand ? ncand + (int64_t)k * nl : NULL,
               trace ? trace + k * tstride : NULL);
    if (gap) gap[k] = gk;
  }
  return ORA_OK;
}

/* The plain walk (no PHAROS variant, no trace). */
int ora_select(const ora_shape* s, const void* Q, const double* pyr, int nunits, const int32_t* units, int nitems,
               const int32_t* slot, const int64_t* qb, int start_level, int32_t* idx, double* gap,
               int32_t* ncand) {
  return ora_select_ex(s, Q, pyr, nunits, units, nitems, slot, qb, start_level, NULL, idx, gap, ncand, NULL);
}

/* ---- step 4: causal block-sparse attention ----------------------------- */

/*
 * Output and log-sum-exp of the listed query rows. Row r (flat index
 * (bi*Hq + hq)*Nq + t) at position p = q_offset + t in query block i attends
 * to every key of the blocks idx[bi][hq/G][i - first][*] (entries < 0
 * skipped) and to the keys of block i at positions <= p, with one softmax
 * over that union at scale 1/sqrt(d). With dense != 0 it attends to every
 * key at position <= p instead (plain causal attention).
 * idx: [B][Hkv][nqb][topk]. O: [nrows][d]; lse: [nrows] (natural log).
 * Returns ORA_EBADIDX if a listed block is not strictly before i or repeats.
 */
/*
 * Rows of attention. With M > 0 the prefix states take part too (PHBA
 * prefix-state branch, below): PK, PV are [B*Hkv][nb][M][d] and Qs (NULL: Q)
 * is the query the state slots are scored with.
 */
static int attend_rows(const ora_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx, int nrows,
                       const int64_t* rows, int dense, const void* Qs, int M, const double* PK, const double* PV,
                       double* O, double* lse) {
  const int d = s->d, G = s->Hq / s->Hkv;
  const int64_t nqb = ora_num_qblocks(s), first = ora_first_qblock(s), nb = num_blocks(s);
  const double scale = 1.0 / sqrt((double)d);
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int r = 0; r < nrows; r++) {
    const int64_t t = rows[r] % s->Nq, bh = rows[r] / s->Nq;
    const int64_t bi = bh / s->Hq, hq = bh % s->Hq, hk = hq / G;
    const int64_t p = s->q_offset + t, i = p / s->b;
    const int64_t qbase = rows[r] * d, kvbase = (bi * s->Hkv + hk) * (int64_t)s->N * d;
    /* the attended key positions, in any order; with states, the attended state blocks */
    int64_t cap_keys = dense ? p + 1 : (int64_t)(s->topk + 1) * s->b;
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap_keys);
    int64_t* sblk = (int64_t*)malloc(sizeof(int64_t) * (size_t)(s->topk + 1));
    int64_t nk = 0, ns = 0;
    if (dense) {
      for (int64_t k = 0; k <= p; k++) keys[nk++] = k;
    } else {
      const int32_t* row_idx = idx + ((bi * s->Hkv + hk) * nqb + (i - first)) * s->topk;
      for (int k = 0; k < s->topk; k++) {
        const int64_t j = row_idx[k];
        if (j < 0) continue;
        int rep = 0;
        for (int k2 = 0; k2 < k; k2++) rep |= (row_idx[k2] == j);
        if (j >= i || rep) {
          bad = 1;
          continue;
        }
        for (int64_t x = j * s->b; x < (j + 1) * s->b && x < s->N; x++) keys[nk++] = x;
        if (M > 0 && j >= 1) sblk[ns++] = j; /* the prefix state aligned with routed block j */
      }
      for (int64_t x = i * s->b; x <= p; x++) keys[nk++] = x;
      if (M > 0 && i >= 1) sblk[ns++] = i; /* the current block's prefix state */
    }
    const int64_t nslot = ns * M;
    double* sc = (double*)malloc(sizeof(double) * (size_t)(nk + nslot + 1));
    double mx = -INFINITY;
    for (int64_t k = 0; k < nk; k++) {
      double dot = 0.0;
      for (int e = 0; e < d; e++) dot += elem(Q, s->dtype, qbase + e) * elem(K, s->dtype, kvbase + keys[k] * d + e);
      sc[k] = dot * scale;
      if (sc[k] > mx) mx = sc[k];
    }
    const void* qs = Qs ? Qs : Q;
    const int64_t sbase = (bi * s->Hkv + hk) * nb * (int64_t)M * d;
    for (int64_t c = 0; c < nslot; c++) {
      const double* key = PK + sbase + (sblk[c / M] * M + c % M) * d;
      double dot = 0.0;
      for (int e = 0; e < d; e++) dot += elem(qs, s->dtype, qbase + e) * key[e];
      sc[nk + c] = dot * scale;
      if (sc[nk + c] > mx) mx = sc[nk + c];
    }
    double sum = 0.0;
    for (int64_t k = 0; k < nk + nslot; k++) sum += exp(sc[k] - mx);
    const double l = mx + log(sum);
    for (int e = 0; e < d; e++) O[(int64_t)r * d + e] = 0.0;
    for (int64_t k = 0; k < nk; k++) {
      const double w = exp(sc[k] - l);
      for (int e = 0; e < d; e++) O[(int64_t)r * d + e] += w * elem(V, s->dtype, kvbase + keys[k] * d + e);
    }
    for (int64_t c = 0; c < nslot; c++) {
      const double w = exp(sc[nk + c] - l);
      const double* val = PV + sbase + (sblk[c / M] * M + c % M) * d;
      for (int e = 0; e < d; e++) O[(int64_t)r * d + e] += w * val[e];
    }
    lse[r] = l;
    free(sc);
    free(keys);
    free(sblk);
  }
  return bad ? ORA_EBADIDX : ORA_OK;
}

int ora_attend(const ora_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx, int nrows,
               const int64_t* rows, int dense, double* O, double* lse) {
  if (!s || !Q || !K || !V || !rows || !O || !lse || (!dense && !idx)) return ORA_EINVAL;
  return attend_rows(s, Q, K, V, idx, nrows, rows, dense, NULL, 0, NULL, NULL, O, lse);
}

/* ---- PHBA prefix-state branch ----------------------------------------- */
/*
 * PHBA summary, 2.2 "Gated slot memory", 3.2 "Prefix-state construction" and
 * A.1.1: gated recurrences build a prefix-key and a prefix-value state of M
 * slots each; the state stored immediately before a block summarises only the
 * causal context before it; the key and the value recurrence share one
 * slot-wise retention gate and one write gate; the recurrence starts from a
 * zero state at the start of a sequence.
 * Reading (the summary prints no formula): with state-branch key k_t, value
 * v_t, retention a_t[s] and write w_t[s] of token t (slot s = 0 .. M-1),
 *   SK[s] <- a_t[s] SK[s] + w_t[s] k_t,    SV[s] <- a_t[s] SV[s] + w_t[s] v_t,
 * from SK = SV = 0 before position 0, token by token; the prefix state of key
 * block j is (SK, SV) after the tokens at positions < j b, so block 0's is
 * zero. Written here as that plain sequential recurrence in double.
 */
static void prefix_states_unit(const ora_shape* s, int M, const void* Ks, const void* V, const float* A,
                               const float* W, int64_t unit, double* PK, double* PV) {
  const int d = s->d;
  double* SK = (double*)calloc((size_t)M * d, sizeof(double));
  double* SV = (double*)calloc((size_t)M * d, sizeof(double));
  const int64_t xbase = unit * (int64_t)s->N * d, gbase = unit * (int64_t)s->N * M;
  for (int64_t t = 0; t < s->N; t++) {
    if (t % s->b == 0) {
      const int64_t j = t / s->b;
      memcpy(PK + j * M * d, SK, sizeof(double) * (size_t)M * d);
      memcpy(PV + j * M * d, SV, sizeof(double) * (size_t)M * d);
    }
    for (int m = 0; m < M; m++) {
      const double a = A[gbase + t * M + m], w = W[gbase + t * M + m];
      for (int e = 0; e < d; e++) {
        SK[m * d + e] = a * SK[m * d + e] + w * elem(Ks, s->dtype, xbase + t * d + e);
        SV[m * d + e] = a * SV[m * d + e] + w * elem(V, s->dtype, xbase + t * d + e);
      }
    }
  }
  free(SK);
  free(SV);
}

/*
 * Prefix states of the listed units: PK, PV [nunits][nb][M][d] (double).
 * Ks (state-branch keys) and V: [B][Hkv][N][d] in s->dtype; A (retention)
 * and W (write): [B][Hkv][N][M] float32.
 */
int ora_prefix_states(const ora_shape* s, int M, const void* Ks, const void* V, const float* A, const float* W,
                      int nunits, const int32_t* units, double* PK, double* PV) {
  if (!s || !Ks || !V || !A || !W || !units || !PK || !PV || M <= 0) return ORA_EINVAL;
  const int64_t per = num_blocks(s) * (int64_t)M * s->d;
#pragma omp parallel for schedule(dynamic)
  for (int u = 0; u < nunits; u++) prefix_states_unit(s, M, Ks, V, A, W, units[u], PK + u * per, PV + u * per);
  return ORA_OK;
}

/*
 * PHBA summary, 3.3 "Online-softmax token-state attention" and A.1.3: the
 * output is one softmax over the exact tokens (the routed blocks and the
 * current block up to the query's position) and the prefix-state slots: the
 * current block's prefix state and the prefix state aligned with each routed
 * block. Token scores use the (rotated) query and keys, state scores the raw
 * query against the raw state keys; the values are V and the value states.
 * Readings: a slot's score is qs . PK[slot] / sqrt(d), the token branch's
 * scale; a block whose causal prefix is empty (block 0) brings no state (the
 * PrefixValid flag of PHBA A.1.2); Qs NULL means the state branch uses Q (the
 * rotation of the pages' models is outside this library).
 * PK, PV: [B*Hkv][nb][M][d] double, as ora_prefix_states writes for all units.
 */
int ora_attend_states(const ora_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx, int nrows,
                      const int64_t* rows, const void* Qs, int M, const double* PK, const double* PV, double* O,
                      double* lse) {
  if (!s || !Q || !K || !V || !idx || !rows || !O || !lse || M < 0 || (M > 0 && (!PK || !PV))) return ORA_EINVAL;
  return attend_rows(s, Q, K, V, idx, nrows, rows, 0, Qs, M, PK, PV, O, lse);
}

/* ---- backward: block-major route metadata and gradients ----------------- */
/*
 * PHBA summary, A.1.2 "Routing metadata kernels": for the backward pass the
 * query-centric routes are re-expressed block-major: per key block, the
 * contiguous range of the query rows that route to it, formed by counting the
 * assignments per block, prefix-summing the counts and scattering the ids.
 * Route indices are non-differentiable.
 * PHBA summary, A.1.4 "Sparse backward kernel": the block-major schedule
 * enumerates, for each key block, the query rows that attend it; scores and
 * probabilities are recomputed from the log-sum-exp instead of being stored.
 *
 * Readings: rho lists query-block indices qb (the row index into idx, all G
 * heads of the kv group implied), ascending within each key block's range;
 * the diagonal block (always attended) is not listed, as in idx. Gradients
 * are those of the scalar sum_t dO_t . O_t with respect to Q, K and V, with
 * the routes held fixed; O and the log-sum-exp are recomputed here in double.
 */

/* offset[0..nb], rho[0..offset[nb]) for one (batch, kv head) unit. */
int ora_route_invert(const ora_shape* s, const int32_t* idx, int32_t unit, int32_t* offset, int32_t* rho) {
  if (!s || !idx || !offset || !rho) return ORA_EINVAL;
  const int64_t nb = num_blocks(s), nqb = ora_num_qblocks(s), first = ora_first_qblock(s);
  const int32_t* u = idx + (int64_t)unit * nqb * s->topk;
  /* count the assignments per key block */
  for (int64_t j = 0; j <= nb; j++) offset[j] = 0;
  for (int64_t q = 0; q < nqb; q++)
    for (int k = 0; k < s->topk; k++) {
      const int64_t j = u[q * s->topk + k];
      if (j < 0) continue;
      int rep = 0;
      for (int k2 = 0; k2 < k; k2++) rep |= (u[q * s->topk + k2] == j);
      if (j >= first + q || rep) return ORA_EBADIDX;
      offset[j + 1]++;
    }
  /* prefix sums give each block a contiguous range */
  for (int64_t j = 0; j < nb; j++) offset[j + 1] += offset[j];
  /* scatter the query blocks in ascending order */
  int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nb > 0 ? nb : 1));
  for (int64_t j = 0; j < nb; j++) fill[j] = offset[j];
  for (int64_t q = 0; q < nqb; q++)
    for (int k = 0; k < s->topk; k++) {
      const int64_t j = u[q * s->topk + k];
      if (j >= 0) rho[fill[j]++] = (int32_t)q;
    }
  free(fill);
  return ORA_OK;
}

/* The attended key positions of one query row (routed blocks, then the
 * diagonal block up to the row's position), as in ora_attend. */
static int64_t row_keys(const ora_shape* s, const int32_t* idx, int dense, int64_t row, int64_t* keys, int* bad) {
  const int G = s->Hq / s->Hkv;
  const int64_t nqb = ora_num_qblocks(s), first = ora_first_qblock(s);
  const int64_t t = row % s->Nq, bh = row / s->Nq;
  const int64_t bi = bh / s->Hq, hq = bh % s->Hq, hk = hq / G;
  const int64_t p = s->q_offset + t, i = p / s->b;
  int64_t nk = 0;
  if (dense) {
    for (int64_t k = 0; k <= p; k++) keys[nk++] = k;
    return nk;
  }
  const int32_t* row_idx = idx + ((bi * s->Hkv + hk) * nqb + (i - first)) * s->topk;
  for (int k = 0; k < s->topk; k++) {
    const int64_t j = row_idx[k];
    if (j < 0) continue;
    int rep = 0;
    for (int k2 = 0; k2 < k; k2++) rep |= (row_idx[k2] == j);
    if (j >= i || rep) {
      *bad = 1;
      continue;
    }
    for (int64_t x = j * s->b; x < (j + 1) * s->b && x < s->N; x++) keys[nk++] = x;
  }
  for (int64_t x = i * s->b; x <= p; x++) keys[nk++] = x;
  return nk;
}

/* For one query row: P_k, and dS_k = P_k (dO . v_k - dO . O) over its keys. */
static void row_grad(const ora_shape* s, const void* Q, const void* K, const void* V, const void* dO, int64_t row,
                     const int64_t* keys, int64_t nk, double* P, double* dS) {
  const int d = s->d, G = s->Hq / s->Hkv;
  const int64_t bh = row / s->Nq, bi = bh / s->Hq, hk = (bh % s->Hq) / G;
  const int64_t qbase = row * d, kvbase = (bi * s->Hkv + hk) * (int64_t)s->N * d;
  const double scale = 1.0 / sqrt((double)d);
  double mx = -INFINITY;
  for (int64_t k = 0; k < nk; k++) {
    double dot = 0.0;
    for (int e = 0; e < d; e++) dot += elem(Q, s->dtype, qbase + e) * elem(K, s->dtype, kvbase + keys[k] * d + e);
    P[k] = dot * scale;
    if (P[k] > mx) mx = P[k];
  }
  double sum = 0.0;
  for (int64_t k = 0; k < nk; k++) sum += exp(P[k] - mx);
  const double lse = mx + log(sum);
  double D = 0.0; /* dO . O with O = sum_k P_k v_k */
  for (int64_t k = 0; k < nk; k++) {
    P[k] = exp(P[k] - lse);
    double dp = 0.0;
    for (int e = 0; e < d; e++) dp += elem(dO, s->dtype, qbase + e) * elem(V, s->dtype, kvbase + keys[k] * d + e);
    dS[k] = dp;
    D += P[k] * dp;
  }
  for (int64_t k = 0; k < nk; k++) dS[k] = P[k] * (dS[k] - D);
}

/* dQ for the listed flat query rows ((b*Hq + hq)*Nq + t): dQ_t = sum_k dS_k k_k / sqrt(d). */
int ora_attend_bwd_q(const ora_shape* s, const void* Q, const void* K, const void* V, const void* dO,
                     const int32_t* idx, int nrows, const int64_t* rows, int dense, double* dQ) {
  if (!s || !Q || !K || !V || !dO || !rows || !dQ || (!dense && !idx)) return ORA_EINVAL;
  const int d = s->d, G = s->Hq / s->Hkv;
  const double scale = 1.0 / sqrt((double)d);
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int r = 0; r < nrows; r++) {
    const int64_t p = s->q_offset + rows[r] % s->Nq;
    const int64_t cap_keys = dense ? p + 1 : (int64_t)(s->topk + 1) * s->b;
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap_keys);
    double* P = (double*)malloc(sizeof(double) * (size_t)cap_keys);
    double* dS = (double*)malloc(sizeof(double) * (size_t)cap_keys);
    const int64_t nk = row_keys(s, idx, dense, rows[r], keys, &bad);
    row_grad(s, Q, K, V, dO, rows[r], keys, nk, P, dS);
    const int64_t bh = rows[r] / s->Nq, bi = bh / s->Hq, hk = (bh % s->Hq) / G;
    const int64_t kvbase = (bi * s->Hkv + hk) * (int64_t)s->N * d;
    for (int e = 0; e < d; e++) {
      double acc = 0.0;
      for (int64_t k = 0; k < nk; k++) acc += dS[k] * elem(K, s->dtype, kvbase + keys[k] * d + e);
      dQ[(int64_t)r * d + e] = acc * scale;
    }
    free(dS);
    free(P);
    free(keys);
  }
  return bad ? ORA_EBADIDX : ORA_OK;
}

/* dK and dV of the listed key blocks (entries unit * nb + j): every query row of
 * every head of the kv group whose keys include a position of block j contributes
 * dK_x += dS_x q_t / sqrt(d) and dV_x += P_x dO_t. Output [nblk][b][d]; positions
 * at or beyond N stay zero. */
int ora_attend_bwd_kv(const ora_shape* s, const void* Q, const void* K, const void* V, const void* dO,
                      const int32_t* idx, int nblk, const int64_t* blocks, int dense, double* dK, double* dV) {
  if (!s || !Q || !K || !V || !dO || !blocks || !dK || !dV || (!dense && !idx)) return ORA_EINVAL;
  const int d = s->d, G = s->Hq / s->Hkv, b = s->b;
  const int64_t nb = num_blocks(s), nqb = ora_num_qblocks(s), first = ora_first_qblock(s);
  const double scale = 1.0 / sqrt((double)d);
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int n = 0; n < nblk; n++) {
    const int64_t unit = blocks[n] / nb, j = blocks[n] % nb;
    const int64_t bi = unit / s->Hkv, hk = unit % s->Hkv;
    double* gk = dK + (int64_t)n * b * d;
    double* gv = dV + (int64_t)n * b * d;
    for (int64_t x = 0; x < (int64_t)b * d; x++) gk[x] = gv[x] = 0.0;
    const int64_t cap_keys = dense ? s->N : (int64_t)(s->topk + 1) * b;
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap_keys);
    double* P = (double*)malloc(sizeof(double) * (size_t)cap_keys);
    double* dS = (double*)malloc(sizeof(double) * (size_t)cap_keys);
    for (int64_t q = 0; q < nqb; q++) {
      const int64_t i = first + q;
      /* does query block i attend block j? (the diagonal always; otherwise through its routes) */
      int uses = dense ? (i >= j) : (i == j);
      if (!dense && i > j)
        for (int k = 0; k < s->topk; k++) uses |= (idx[((unit * nqb) + q) * s->topk + k] == j);
      if (!uses) continue;
      for (int gg = 0; gg < G; gg++) {
        const int64_t hq = hk * G + gg;
        for (int64_t p = (i * b > s->q_offset ? i * b : s->q_offset); p < (i + 1) * b && p < s->q_offset + s->Nq; p++) {
          const int64_t row = (bi * s->Hq + hq) * s->Nq + (p - s->q_offset);
          const int64_t nk = row_keys(s, idx, dense, row, keys, &bad);
          row_grad(s, Q, K, V, dO, row, keys, nk, P, dS);
          for (int64_t k = 0; k < nk; k++) {
            if (keys[k] / b != j) continue;
            const int64_t x = keys[k] - j * b;
            for (int e = 0; e < d; e++) {
              gk[x * d + e] += dS[k] * elem(Q, s->dtype, row * d + e) * scale;
              gv[x * d + e] += P[k] * elem(dO, s->dtype, row * d + e);
            }
          }
        }
      }
    }
    free(dS);
    free(P);
    free(keys);
  }
  return bad ? ORA_EBADIDX : ORA_OK;
}
