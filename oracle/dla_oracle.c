/*
 * dla_oracle.c -- plain, slow, token-by-token fp64 CPU oracle of the
 * Dynamic Linear Attention (DLA) forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library and neither side
 * imports the other.
 *
 * What it computes (per (batch, head) stream, in fp64; f32 and bf16 inputs are
 * widened exactly):
 *
 *   - per-token state v_t phi(k_t)^T with phi = elu + 1
 *       ("Dynamic Linear Attention | Chlience Paper Archive", section 5.1,
 *        the per-token state s_t; stored transposed as [d_v][d_k]);
 *   - token score r_t = 1 - cos(k_t, k_{t-1}) on the raw keys, r_0 = 0, and a
 *     token joins the open segment only when r_t < tau and r_{t-1} < tau
 *       (ai-feeds.com "Dynamic Linear Attention" summary, section
 *        "信息感知的动态状态合并": two consecutive low-information tokens are
 *        merged; Chlience section 5.1: b_t = 1 opens a new state, b_t = 0 adds
 *        s_t to the current state);
 *   - a time-ordered cache of at most C states (open one included); when a
 *     boundary seals the open state and C states are sealed, the adjacent
 *     sealed pair with the smallest Ward loss
 *         n_i n_j / (n_i + n_j) * || mu_i - mu_j ||^2,   mu = z / n,
 *     z = sum of phi(k), is merged into the left one (earlier timestamp kept),
 *     ties to the leftmost pair
 *       (Chlience section 5.2, capacity-bounded memory and the merge update
 *        S <- S + S', n <- n + n'; ai-feeds "容量受限的内存建模": adjacent
 *        pair with least merge loss, merged state keeps the earlier timestamp;
 *        Chlience Corollary 1: the Ward term is the within-block scatter);
 *   - readout o_t = sum_i lambda_{t,i} S_i phi(q_t) over the states present at
 *     t (after the merge at t, open state including token t), with
 *     lambda_{t,i} = softmax_i( phi(q_t) . mu_i / sqrt(d_k) )
 *       (Chlience section 5.3, reading from bounded states).
 *
 * The information policy (the pages' own criteria, Chlience section 5.1 and
 * section 5.2) decides and merges on the states themselves:
 *   - I_t = || N(s_t) - N(S) ||_F / ( || N(S) ||_F + eps ), with s_t the
 *     per-token state v_t phi(k_t)^T, S the open state before token t and
 *     N(X) = X / sqrt(mean of the entries of X^2 + eps) (RMSNorm over the
 *     whole d_v x d_k state, no gain), eps = 1e-6 in both places;
 *   - b_t = [I_t >= tau]; the first token of a stream has no open state to
 *     compare with, so it opens one, with I_0 = 0;
 *   - each state keeps the sum of the scores of its tokens (I-bar); at
 *     capacity the adjacent sealed pair with the least information density
 *     (I-bar_i + I-bar_{i+1}) / (n_i + n_{i+1}) is merged (leftmost on ties)
 *     and the sums add.
 *
 * The unbounded policy, DLA(I) (the ablation row "Mamba-2 + DLA(I)" of the
 * Chlience page's ablation table: dynamic merging without the capacity-bounded
 * memory), takes the same decisions and readout with no capacity at all:
 * every segment stays a state of its own and nothing is ever merged.
 *
 * The fixed-bucket policy (Chlience section 2 and section 5.4, Log-Linear
 * Attention's Fenwick buckets) keeps a binary-counter list of blocks over
 * [0, t-1]; token t reads the blocks plus {t} with the same softmax, then {t}
 * is pushed and the two newest blocks are merged while their sizes are equal.
 *
 * Readings where the pages are silent (applied identically by the CUDA path):
 *   r_0 = 0 (no predecessor); a zero-norm key gives cos = 0 (r = 1);
 *   "below tau" is strict; C counts the open state, so a merge fires only at a
 *   boundary when C sealed states exist; order within a token is
 *   decide -> merge -> add v phi(k)^T -> read out.
 *
 * Arithmetic order (fixed so that r_t is bit-identical on both sides): dot
 * products and squared norms are summed sequentially over the index, with no
 * fused multiply-add (build with -ffp-contract=off), and
 * cos = dot / (sqrt(|a|^2) * sqrt(|b|^2)).  z is summed token by token.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_F64 2

#define OR_POLICY_DLA 0
#define OR_POLICY_FENWICK 1
#define OR_POLICY_INFO 2
#define OR_POLICY_UNBOUNDED 3

/* RMSNorm epsilon and the information score's denominator epsilon. */
#define OR_INFO_EPS 1e-6

typedef struct {
  double *S; /* [dv][dk] sum of v phi(k)^T */
  double *z; /* [dk] sum of phi(k) */
  int64_t n;
  int64_t ts;
  double info; /* sum of the information scores of its tokens (information policy) */
} ostate;

typedef struct {
  int nsealed;
  int cap_sealed;
  ostate *sealed; /* time order */
  int has_open;
  ostate open;
  double *prev_k;
  double prev_r;
  int64_t t;
} ohead;

typedef struct {
  int nheads, dk, dv, C, policy, want_S;
  ohead *heads;
} oracle;

static double widen(const void *p, int dtype, size_t i) {
  if (dtype == OR_F32) return (double)((const float *)p)[i];
  if (dtype == OR_F64) return ((const double *)p)[i];
  uint32_t b = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &b, sizeof f);
  return (double)f;
}

/* phi = elu + 1: x + 1 for x > 0, exp(x) for x <= 0. */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

static void st_alloc(ostate *s, int dk, int dv, int want_S) {
  s->S = want_S ? (double *)calloc((size_t)dv * dk, sizeof(double)) : NULL;
  s->z = (double *)calloc((size_t)dk, sizeof(double));
  s->n = 0;
  s->ts = 0;
  s->info = 0.0;
}

static void st_zero(ostate *s, int dk, int dv) {
  if (s->S) memset(s->S, 0, sizeof(double) * (size_t)dv * dk);
  memset(s->z, 0, sizeof(double) * (size_t)dk);
  s->n = 0;
  s->ts = 0;
  s->info = 0.0;
}

static void st_copy(ostate *dst, const ostate *src, int dk, int dv) {
  if (dst->S && src->S) memcpy(dst->S, src->S, sizeof(double) * (size_t)dv * dk);
  memcpy(dst->z, src->z, sizeof(double) * (size_t)dk);
  dst->n = src->n;
  dst->ts = src->ts;
  dst->info = src->info;
}

/* left <- left + right (S, z, n, info); left keeps its timestamp. */
static void st_absorb(ostate *left, const ostate *right, int dk, int dv) {
  if (left->S && right->S)
    for (size_t i = 0; i < (size_t)dv * dk; i++) left->S[i] = left->S[i] + right->S[i];
  for (int i = 0; i < dk; i++) left->z[i] = left->z[i] + right->z[i];
  left->n = left->n + right->n;
  left->info = left->info + right->info;
}

/* Room for one more sealed state (the unbounded policy grows its list). */
static void ensure_room(ohead *hd, int dk, int dv, int want_S) {
  if (hd->nsealed < hd->cap_sealed) return;
  int cap = hd->cap_sealed * 2;
  hd->sealed = (ostate *)realloc(hd->sealed, sizeof(ostate) * (size_t)cap);
  for (int i = hd->cap_sealed; i < cap; i++) st_alloc(&hd->sealed[i], dk, dv, want_S);
  hd->cap_sealed = cap;
}

/* Ward loss n_a n_b / (n_a + n_b) * sum_i (z_a[i]/n_a - z_b[i]/n_b)^2. */
static double ward(const ostate *a, const ostate *b, int dk) {
  double na = (double)a->n, nb = (double)b->n;
  double f = (na * nb) / (na + nb);
  double s = 0.0;
  for (int i = 0; i < dk; i++) {
    double diff = a->z[i] / na - b->z[i] / nb;
    s = s + diff * diff;
  }
  return f * s;
}

/* r = 1 - cos(a, b); zero norm gives cos = 0. */
static double score(const double *a, const double *b, int dk) {
  double dot = 0.0, na = 0.0, nb = 0.0;
  for (int i = 0; i < dk; i++) dot = dot + a[i] * b[i];
  for (int i = 0; i < dk; i++) na = na + a[i] * a[i];
  for (int i = 0; i < dk; i++) nb = nb + b[i] * b[i];
  if (na == 0.0 || nb == 0.0) return 1.0;
  return 1.0 - dot / (sqrt(na) * sqrt(nb));
}

/* Information score of a token against the open state S ([dv][dk]):
 * || N(v u^T) - N(S) ||_F / (|| N(S) ||_F + eps), N = RMSNorm over all entries. */
static double info_score(const double *vv, const double *u, const double *S, int dk, int dv) {
  double cnt = (double)dk * (double)dv;
  double ss = 0.0, sS = 0.0;
  for (int a = 0; a < dv; a++)
    for (int c = 0; c < dk; c++) {
      double x = vv[a] * u[c];
      ss = ss + x * x;
    }
  for (size_t i = 0; i < (size_t)dv * dk; i++) sS = sS + S[i] * S[i];
  double rs = sqrt(ss / cnt + OR_INFO_EPS), rS = sqrt(sS / cnt + OR_INFO_EPS);
  double diff = 0.0, norm = 0.0;
  for (int a = 0; a < dv; a++)
    for (int c = 0; c < dk; c++) {
      double ns = (vv[a] * u[c]) / rs, nS = S[(size_t)a * dk + c] / rS;
      diff = diff + (ns - nS) * (ns - nS);
      norm = norm + nS * nS;
    }
  return sqrt(diff) / (sqrt(norm) + OR_INFO_EPS);
}

/* Information density of the union of two adjacent states. */
static double density(const ostate *a, const ostate *b) {
  return (a->info + b->info) / ((double)a->n + (double)b->n);
}

oracle *dla_oracle_new(int nheads, int dk, int dv, int C, int policy, int want_S) {
  oracle *o = (oracle *)calloc(1, sizeof(oracle));
  o->nheads = nheads;
  o->dk = dk;
  o->dv = dv;
  o->C = C;
  o->policy = policy;
  /* the information policy decides on the states themselves */
  o->want_S = policy == OR_POLICY_INFO ? 1 : want_S;
  want_S = o->want_S;
  o->heads = (ohead *)calloc((size_t)nheads, sizeof(ohead));
  int cap = policy == OR_POLICY_FENWICK ? 64 : (policy == OR_POLICY_UNBOUNDED ? 16 : C);
  for (int h = 0; h < nheads; h++) {
    ohead *hd = &o->heads[h];
    hd->cap_sealed = cap;
    hd->sealed = (ostate *)calloc((size_t)cap, sizeof(ostate));
    for (int i = 0; i < cap; i++) st_alloc(&hd->sealed[i], dk, dv, want_S);
    st_alloc(&hd->open, dk, dv, want_S);
    hd->prev_k = (double *)calloc((size_t)dk, sizeof(double));
  }
  return o;
}

void dla_oracle_free(oracle *o) {
  if (!o) return;
  for (int h = 0; h < o->nheads; h++) {
    ohead *hd = &o->heads[h];
    for (int i = 0; i < hd->cap_sealed; i++) {
      free(hd->sealed[i].S);
      free(hd->sealed[i].z);
    }
    free(hd->sealed);
    free(hd->open.S);
    free(hd->open.z);
    free(hd->prev_k);
  }
  free(o->heads);
  free(o);
}

typedef struct {
  oracle *o;
  int head_lo, head_hi, T;
  double tau;
  int dtype;
  const void *q, *k, *v; /* [nrun][T][d] */
  double *out;           /* [nrun][T][dv] or NULL */
  const uint8_t *out_mask; /* [T]: read out only where set (NULL: every token) */
  uint8_t *boundary;     /* [nrun][T] or NULL */
  int32_t *merge_t, *merge_i, *merge_count; /* [nrun][cap], [nrun] */
  int cap;
  int32_t *live; /* [nrun][T] live states read by token t, or NULL */
  double *margins; /* [nrun][3]: min |score - tau|, min relative gap of the merge
                      criterion (Ward loss or density), #exact ties */
  double *score;   /* [nrun][T] decision score of each token (r_t or I_t), or NULL */
  /* forced merges (NULL: argmin): each capacity merge of head r takes the
   * next entry (t, i) of force_t / force_i [nrun][fcap] (force_count [nrun]
   * entries) instead of the argmin; excess [nrun] receives the largest
   * relative excess (l_i - l_min) / l_min of a forced pair's criterion over
   * the minimum (0 for the minimum itself, +inf when the list does not match
   * the capacity merges, i.e. a wrong token, an index out of range, or an
   * entry left over or missing) */
  const int32_t *force_t, *force_i, *force_count;
  int fcap;
  double *excess;
  int next;        /* work counter */
  pthread_mutex_t mu;
} job;

static void record_merge(job *J, int r, int64_t t, int i) {
  int32_t c = J->merge_count[r];
  if (c < J->cap) {
    J->merge_t[(size_t)r * J->cap + c] = (int32_t)t;
    J->merge_i[(size_t)r * J->cap + c] = i;
  }
  J->merge_count[r] = c + 1;
}

/* Forced mode: the pair the capacity merge at token t takes.  `best` is the
 * argmin and `bl` its criterion; crit(i) gives pair i's criterion.  Updates
 * the head's forced-list position *fk and largest excess *ex. */
static int forced_pair(job *J, int r, int *fk, int64_t t, int best, double bl, int npairs,
                       double (*crit)(const ohead *, int, int), const ohead *hd, int dk,
                       double *ex) {
  int k = (*fk)++;
  const int32_t *ft = J->force_t + (size_t)r * J->fcap;
  const int32_t *fi = J->force_i + (size_t)r * J->fcap;
  if (k >= J->force_count[r] || k >= J->fcap || (int64_t)ft[k] != t || fi[k] < 0 ||
      fi[k] >= npairs) {
    *ex = INFINITY;
    return best;
  }
  int i = fi[k];
  double l = crit(hd, i, dk);
  double e = l == bl ? 0.0 : (bl > 0.0 ? (l - bl) / bl : INFINITY);
  if (e > *ex) *ex = e;
  return i;
}

static double crit_ward(const ohead *hd, int i, int dk) {
  return ward(&hd->sealed[i], &hd->sealed[i + 1], dk);
}

static double crit_density(const ohead *hd, int i, int dk) {
  (void)dk;
  return density(&hd->sealed[i], &hd->sealed[i + 1]);
}

/* Forced mode, at the end of a head's run: every forced entry was used. */
static void forced_close(job *J, int r, int fk, double ex) {
  if (fk != J->force_count[r]) ex = INFINITY;
  if (ex > J->excess[r] || ex != ex) J->excess[r] = ex;
}

/* Readout: lambda = softmax(phi(q).mu/sqrt(dk)) over states; o = sum lambda S p. */
static void readout(const oracle *o, ostate *const *st, int m, const double *p, double *out) {
  int dk = o->dk, dv = o->dv;
  double *a = (double *)malloc(sizeof(double) * (size_t)m);
  double amax = -INFINITY;
  for (int i = 0; i < m; i++) {
    double dot = 0.0;
    for (int c = 0; c < dk; c++) {
      double mu = st[i]->z[c] / (double)st[i]->n;
      dot = dot + p[c] * mu;
    }
    a[i] = dot / sqrt((double)dk);
    if (a[i] > amax) amax = a[i];
  }
  double den = 0.0;
  for (int i = 0; i < m; i++) {
    a[i] = exp(a[i] - amax);
    den = den + a[i];
  }
  for (int r = 0; r < dv; r++) out[r] = 0.0;
  for (int i = 0; i < m; i++) {
    double lam = a[i] / den;
    for (int r = 0; r < dv; r++) {
      double acc = 0.0;
      for (int c = 0; c < dk; c++) acc = acc + st[i]->S[(size_t)r * dk + c] * p[c];
      out[r] = out[r] + lam * acc;
    }
  }
  free(a);
}

/* The dynamic policy, and without its capacity merges the unbounded one. */
static void run_head_dla(job *J, int r) {
  oracle *o = J->o;
  int dk = o->dk, dv = o->dv, C = o->C, T = J->T;
  const int unbounded = o->policy == OR_POLICY_UNBOUNDED;
  ohead *hd = &o->heads[J->head_lo + r];
  int lst_cap = unbounded ? hd->cap_sealed : C;
  double *kk = (double *)malloc(sizeof(double) * dk);
  double *u = (double *)malloc(sizeof(double) * dk);
  double *p = (double *)malloc(sizeof(double) * dk);
  double *vv = (double *)malloc(sizeof(double) * dv);
  ostate **lst = (ostate **)malloc(sizeof(ostate *) * (size_t)(lst_cap + 1));
  double min_rm = INFINITY, min_gap = INFINITY, ties = 0.0;
  int fk = 0;
  double fex = 0.0;
  for (int tl = 0; tl < T; tl++) {
    size_t base = ((size_t)r * T + tl) * dk;
    for (int c = 0; c < dk; c++) kk[c] = widen(J->k, J->dtype, base + c);
    for (int c = 0; c < dk; c++) u[c] = phi(kk[c]);
    double rt = hd->t == 0 ? 0.0 : score(kk, hd->prev_k, dk);
    if (J->score) J->score[(size_t)r * T + tl] = rt;
    if (hd->t > 0) {
      double mrg = fabs(rt - J->tau);
      if (mrg < min_rm) min_rm = mrg;
    }
    int join = hd->t > 0 && rt < J->tau && hd->prev_r < J->tau;
    if (J->boundary) J->boundary[(size_t)r * T + tl] = (uint8_t)(!join);
    if (!join) {
      if (hd->has_open) {
        if (unbounded) {
          ensure_room(hd, dk, dv, o->want_S);
          if (hd->cap_sealed > lst_cap) {
            lst_cap = hd->cap_sealed;
            lst = (ostate **)realloc(lst, sizeof(ostate *) * (size_t)(lst_cap + 1));
          }
        }
        st_copy(&hd->sealed[hd->nsealed], &hd->open, dk, dv);
        hd->nsealed++;
      }
      if (!unbounded && hd->nsealed == C) {
        int best = 0;
        double bl = ward(&hd->sealed[0], &hd->sealed[1], dk);
        double second = INFINITY;
        for (int i = 1; i < C - 1; i++) {
          double l = ward(&hd->sealed[i], &hd->sealed[i + 1], dk);
          if (l < bl) {
            second = bl;
            bl = l;
            best = i;
          } else if (l < second) {
            second = l;
          }
        }
        if (second == bl) ties += 1.0;
        else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;
        if (J->force_count)
          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_ward, hd, dk, &fex);
        st_absorb(&hd->sealed[best], &hd->sealed[best + 1], dk, dv);
        /* drop best+1: rotate its buffers to the end of the list */
        ostate tmp = hd->sealed[best + 1];
        for (int i = best + 1; i < hd->nsealed - 1; i++) hd->sealed[i] = hd->sealed[i + 1];
        hd->sealed[hd->nsealed - 1] = tmp;
        hd->nsealed--;
        record_merge(J, r, hd->t, best);
      }
      st_zero(&hd->open, dk, dv);
      hd->open.ts = hd->t;
      hd->has_open = 1;
    }
    if (J->out) {
      size_t vb = ((size_t)r * T + tl) * dv;
      for (int c = 0; c < dv; c++) vv[c] = widen(J->v, J->dtype, vb + c);
      for (int a = 0; a < dv; a++)
        for (int c = 0; c < dk; c++)
          hd->open.S[(size_t)a * dk + c] = hd->open.S[(size_t)a * dk + c] + vv[a] * u[c];
    }
    for (int c = 0; c < dk; c++) hd->open.z[c] = hd->open.z[c] + u[c];
    hd->open.n = hd->open.n + 1;
    int m = 0;
    for (int i = 0; i < hd->nsealed; i++) lst[m++] = &hd->sealed[i];
    lst[m++] = &hd->open;
    if (J->live) J->live[(size_t)r * T + tl] = m;
    if (J->out && (!J->out_mask || J->out_mask[tl])) {
      for (int c = 0; c < dk; c++) p[c] = phi(widen(J->q, J->dtype, base + c));
      readout(o, lst, m, p, J->out + ((size_t)r * T + tl) * dv);
    }
    for (int c = 0; c < dk; c++) hd->prev_k[c] = kk[c];
    hd->prev_r = rt;
    hd->t = hd->t + 1;
  }
  if (J->margins) {
    double *mg = J->margins + (size_t)r * 3;
    if (min_rm < mg[0]) mg[0] = min_rm;
    if (min_gap < mg[1]) mg[1] = min_gap;
    mg[2] += ties;
  }
  if (J->force_count) forced_close(J, r, fk, fex);
  free(kk);
  free(u);
  free(p);
  free(vv);
  free(lst);
}

static void run_head_info(job *J, int r) {
  oracle *o = J->o;
  int dk = o->dk, dv = o->dv, C = o->C, T = J->T;
  ohead *hd = &o->heads[J->head_lo + r];
  double *u = (double *)malloc(sizeof(double) * dk);
  double *p = (double *)malloc(sizeof(double) * dk);
  double *vv = (double *)malloc(sizeof(double) * dv);
  ostate **lst = (ostate **)malloc(sizeof(ostate *) * (size_t)(C + 1));
  double min_im = INFINITY, min_gap = INFINITY, ties = 0.0;
  int fk = 0;
  double fex = 0.0;
  for (int tl = 0; tl < T; tl++) {
    size_t base = ((size_t)r * T + tl) * dk;
    size_t vb = ((size_t)r * T + tl) * dv;
    for (int c = 0; c < dk; c++) u[c] = phi(widen(J->k, J->dtype, base + c));
    for (int c = 0; c < dv; c++) vv[c] = widen(J->v, J->dtype, vb + c);
    double it = 0.0;
    int join = 0;
    if (hd->has_open) {
      it = info_score(vv, u, hd->open.S, dk, dv);
      double mrg = fabs(it - J->tau);
      if (mrg < min_im) min_im = mrg;
      join = it < J->tau;
    }
    if (J->score) J->score[(size_t)r * T + tl] = it;
    if (J->boundary) J->boundary[(size_t)r * T + tl] = (uint8_t)(!join);
    if (!join) {
      if (hd->has_open) {
        st_copy(&hd->sealed[hd->nsealed], &hd->open, dk, dv);
        hd->nsealed++;
      }
      if (hd->nsealed == C) {
        int best = 0;
        double bl = density(&hd->sealed[0], &hd->sealed[1]);
        double second = INFINITY;
        for (int i = 1; i < C - 1; i++) {
          double l = density(&hd->sealed[i], &hd->sealed[i + 1]);
          if (l < bl) {
            second = bl;
            bl = l;
            best = i;
          } else if (l < second) {
            second = l;
          }
        }
        if (second == bl) ties += 1.0;
        else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;
        if (J->force_count)
          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_density, hd, dk, &fex);
        st_absorb(&hd->sealed[best], &hd->sealed[best + 1], dk, dv);
        ostate tmp = hd->sealed[best + 1];
        for (int i = best + 1; i < hd->nsealed - 1; i++) hd->sealed[i] = hd->sealed[i + 1];
        hd->sealed[hd->nsealed - 1] = tmp;
        hd->nsealed--;
        record_merge(J, r, hd->t, best);
      }
      st_zero(&hd->open, dk, dv);
      hd->open.ts = hd->t;
      hd->has_open = 1;
    }
    for (int a = 0; a < dv; a++)
      for (int c = 0; c < dk; c++)
        hd->open.S[(size_t)a * dk + c] = hd->open.S[(size_t)a * dk + c] + vv[a] * u[c];
    for (int c = 0; c < dk; c++) hd->open.z[c] = hd->open.z[c] + u[c];
    hd->open.n = hd->open.n + 1;
    hd->open.info = hd->open.info + it;
    int m = 0;
    for (int i = 0; i < hd->nsealed; i++) lst[m++] = &hd->sealed[i];
    lst[m++] = &hd->open;
    if (J->live) J->live[(size_t)r * T + tl] = m;
    if (J->out && (!J->out_mask || J->out_mask[tl])) {
      for (int c = 0; c < dk; c++) p[c] = phi(widen(J->q, J->dtype, base + c));
      readout(o, lst, m, p, J->out + ((size_t)r * T + tl) * dv);
    }
    hd->prev_r = it;
    hd->t = hd->t + 1;
  }
  if (J->margins) {
    double *mg = J->margins + (size_t)r * 3;
    if (min_im < mg[0]) mg[0] = min_im;
    if (min_gap < mg[1]) mg[1] = min_gap;
    mg[2] += ties;
  }
  if (J->force_count) forced_close(J, r, fk, fex);
  free(u);
  free(p);
  free(vv);
  free(lst);
}

static void run_head_fenwick(job *J, int r) {
  oracle *o = J->o;
  int dk = o->dk, dv = o->dv, T = J->T;
  ohead *hd = &o->heads[J->head_lo + r];
  double *u = (double *)malloc(sizeof(double) * dk);
  double *p = (double *)malloc(sizeof(double) * dk);
  double *vv = (double *)malloc(sizeof(double) * dv);
  ostate **lst = (ostate **)malloc(sizeof(ostate *) * (size_t)(hd->cap_sealed + 1));
  for (int tl = 0; tl < T; tl++) {
    size_t base = ((size_t)r * T + tl) * dk;
    for (int c = 0; c < dk; c++) u[c] = phi(widen(J->k, J->dtype, base + c));
    if (J->boundary) J->boundary[(size_t)r * T + tl] = 1;
    /* {t} is the open bucket; {t-1} was pushed and carried at the end of t-1. */
    st_zero(&hd->open, dk, dv);
    hd->open.ts = hd->t;
    hd->has_open = 1;
    if (J->out) {
      size_t vb = ((size_t)r * T + tl) * dv;
      for (int c = 0; c < dv; c++) vv[c] = widen(J->v, J->dtype, vb + c);
      for (int a = 0; a < dv; a++)
        for (int c = 0; c < dk; c++) hd->open.S[(size_t)a * dk + c] = vv[a] * u[c];
    }
    for (int c = 0; c < dk; c++) hd->open.z[c] = u[c];
    hd->open.n = 1;
    int m = 0;
    for (int i = 0; i < hd->nsealed; i++) lst[m++] = &hd->sealed[i];
    lst[m++] = &hd->open;
    if (J->live) J->live[(size_t)r * T + tl] = m;
    if (J->out && (!J->out_mask || J->out_mask[tl])) {
      for (int c = 0; c < dk; c++) p[c] = phi(widen(J->q, J->dtype, base + c));
      readout(o, lst, m, p, J->out + ((size_t)r * T + tl) * dv);
    }
    /* push {t}; carry while the two newest blocks have equal size.  The
     * merged buckets are first read by token t+1, so the trace records t+1. */
    st_copy(&hd->sealed[hd->nsealed], &hd->open, dk, dv);
    hd->nsealed++;
    while (hd->nsealed >= 2 && hd->sealed[hd->nsealed - 1].n == hd->sealed[hd->nsealed - 2].n) {
      int left = hd->nsealed - 2;
      st_absorb(&hd->sealed[left], &hd->sealed[left + 1], dk, dv);
      hd->nsealed--;
      record_merge(J, r, hd->t + 1, left);
    }
    hd->t = hd->t + 1;
  }
  free(u);
  free(p);
  free(vv);
  free(lst);
}

static void *worker(void *arg) {
  job *J = (job *)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int r = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (r >= J->head_hi - J->head_lo) break;
    if (J->o->policy == OR_POLICY_DLA || J->o->policy == OR_POLICY_UNBOUNDED) run_head_dla(J, r);
    else if (J->o->policy == OR_POLICY_INFO) run_head_info(J, r);
    else run_head_fenwick(J, r);
  }
  return NULL;
}

/* Run T tokens for heads [head_lo, head_hi).  Inputs are [nrun][T][d] in
 * `dtype`; outputs (all optional) are indexed by the run-local head r.
 * `out` needs the oracle created with want_S = 1; with `out_mask` the readout
 * runs only at tokens whose mask entry is set (states are updated at every
 * token either way); `score` receives each token's decision score.  The
 * information policy needs v even without outputs.  With force_count
 * (dynamic and information policies) the capacity merges take the pairs of
 * the given list instead of the argmin (see job.force_t); the decisions that
 * open states do not depend on merges, so they are unchanged.  Returns 0 on
 * success. */
int dla_oracle_run_forced(oracle *o, int head_lo, int head_hi, int T, double tau, int dtype,
                          const void *q, const void *k, const void *v, double *out,
                          const uint8_t *out_mask, uint8_t *boundary, int32_t *merge_t,
                          int32_t *merge_i, int32_t *merge_count, int cap, int32_t *live,
                          double *margins, double *score, const int32_t *force_t,
                          const int32_t *force_i, const int32_t *force_count, int fcap,
                          double *excess, int nthreads) {
  if (!o || head_lo < 0 || head_hi > o->nheads || head_lo > head_hi || T < 0) return 1;
  if (out && (!o->want_S || !q || !v)) return 2;
  if (o->policy == OR_POLICY_INFO && !v) return 2;
  if (!k) return 3;
  if (force_count && (!force_t || !force_i || !excess || fcap < 0 ||
                      o->policy == OR_POLICY_FENWICK || o->policy == OR_POLICY_UNBOUNDED))
    return 4;
  job J;
  memset(&J, 0, sizeof J);
  J.o = o;
  J.head_lo = head_lo;
  J.head_hi = head_hi;
  J.T = T;
  J.tau = tau;
  J.dtype = dtype;
  J.q = q;
  J.k = k;
  J.v = v;
  J.out = out;
  J.out_mask = out_mask;
  J.boundary = boundary;
  J.merge_t = merge_t;
  J.merge_i = merge_i;
  J.merge_count = merge_count;
  J.cap = cap;
  J.live = live;
  J.margins = margins;
  J.score = score;
  J.force_t = force_t;
  J.force_i = force_i;
  J.force_count = force_count;
  J.fcap = fcap;
  J.excess = excess;
  int nrun = head_hi - head_lo;
  int32_t *mc_local = NULL;
  if (!merge_count) {
    mc_local = (int32_t *)calloc((size_t)(nrun > 0 ? nrun : 1), sizeof(int32_t));
    J.merge_count = mc_local;
    J.cap = 0;
  }
  pthread_mutex_init(&J.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrun) nthreads = nrun > 0 ? nrun : 1;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  for (int i = 0; i < nthreads; i++) pthread_create(&th[i], NULL, worker, &J);
  for (int i = 0; i < nthreads; i++) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J.mu);
  free(mc_local);
  return 0;
}

/* Same, taking every capacity merge's pair from the argmin. */
int dla_oracle_run_scored(oracle *o, int head_lo, int head_hi, int T, double tau, int dtype,
                          const void *q, const void *k, const void *v, double *out,
                          const uint8_t *out_mask, uint8_t *boundary, int32_t *merge_t,
                          int32_t *merge_i, int32_t *merge_count, int cap, int32_t *live,
                          double *margins, double *score, int nthreads) {
  return dla_oracle_run_forced(o, head_lo, head_hi, T, tau, dtype, q, k, v, out, out_mask,
                               boundary, merge_t, merge_i, merge_count, cap, live, margins, score,
                               NULL, NULL, NULL, 0, NULL, nthreads);
}

/* Same, without the per-token scores. */
int dla_oracle_run_masked(oracle *o, int head_lo, int head_hi, int T, double tau, int dtype,
                          const void *q, const void *k, const void *v, double *out,
                          const uint8_t *out_mask, uint8_t *boundary, int32_t *merge_t,
                          int32_t *merge_i, int32_t *merge_count, int cap, int32_t *live,
                          double *margins, int nthreads) {
  return dla_oracle_run_scored(o, head_lo, head_hi, T, tau, dtype, q, k, v, out, out_mask,
                               boundary, merge_t, merge_i, merge_count, cap, live, margins, NULL,
                               nthreads);
}

/* Same, reading out at every token. */
int dla_oracle_run(oracle *o, int head_lo, int head_hi, int T, double tau, int dtype,
                   const void *q, const void *k, const void *v, double *out,
                   uint8_t *boundary, int32_t *merge_t, int32_t *merge_i,
                   int32_t *merge_count, int cap, int32_t *live, double *margins,
                   int nthreads) {
  return dla_oracle_run_masked(o, head_lo, head_hi, T, tau, dtype, q, k, v, out, NULL, boundary,
                               merge_t, merge_i, merge_count, cap, live, margins, nthreads);
}

/* Live states of one head in time order (sealed..., open).  Returns m and
 * fills up to `maxm` entries: S [m][dv][dk] (if non-NULL and kept), z
 * [m][dk], n [m], ts [m], info [m] (score sums); plus prev_r and t. */
int dla_oracle_state_info(const oracle *o, int head, int maxm, double *S, double *z, int64_t *n,
                          int64_t *ts, double *info, double *prev_r, int64_t *t) {
  if (!o || head < 0 || head >= o->nheads) return -1;
  const ohead *hd = &o->heads[head];
  int m = hd->nsealed + (hd->has_open ? 1 : 0);
  int dk = o->dk, dv = o->dv;
  for (int i = 0; i < m && i < maxm; i++) {
    const ostate *s = i < hd->nsealed ? &hd->sealed[i] : &hd->open;
    if (S && s->S) memcpy(S + (size_t)i * dv * dk, s->S, sizeof(double) * (size_t)dv * dk);
    if (z) memcpy(z + (size_t)i * dk, s->z, sizeof(double) * (size_t)dk);
    if (n) n[i] = s->n;
    if (ts) ts[i] = s->ts;
    if (info) info[i] = s->info;
  }
  if (prev_r) *prev_r = hd->prev_r;
  if (t) *t = hd->t;
  return m;
}

/* Same, without the score sums. */
int dla_oracle_state(const oracle *o, int head, int maxm, double *S, double *z, int64_t *n,
                     int64_t *ts, double *prev_r, int64_t *t) {
  return dla_oracle_state_info(o, head, maxm, S, z, n, ts, NULL, prev_r, t);
}
