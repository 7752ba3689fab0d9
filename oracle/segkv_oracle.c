/*
 * segkv_oracle.c -- plain fp64 CPU oracle for head-wise segmented paged attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline may load this library.  It shares no code, header or table with the CUDA
 * library under head_wise_sparse_b200/csrc and includes none of its files.
 *
 * What it computes (the method, "RedKnot" pages: zhichai.net news item "What Happened",
 * item 3 SegPagedAttention; hysenlabs.com write-up "The Three Core Mechanisms in Detail",
 * third mechanism):
 *   - every (layer, KV head) owns its own page list; a "global" head keeps the whole
 *     causal context, a "local" head keeps only a sliding window of W tokens, stored in a
 *     ring of R pages (item 1 of the same news item: global heads see full context,
 *     local heads a sliding window);
 *   - attention for every head runs over that head's own pages; the result equals plain
 *     masked softmax attention with an explicit per-head visibility row.
 *
 * Readings taken where the pages are silent:
 *   visibility of a query at position p:  global  k <= p;   local  p - W < k <= p;
 *   query head h reads KV head h / G (G = Hq / Hkv, contiguous groups);
 *   lse = natural log of the sum of exp(scale * q.k) over visible keys;
 *   page allocation: every slot touched by an append that is unallocated, or whose page is
 *   shared with another sequence, takes the next id of the caller's free list, in the
 *   order (sequence in call order, KV head ascending, logical page ascending); a shared
 *   page's content is copied into the new page first (copy on write); a global head maps
 *   logical page lp to slot lp, a local head to slot lp mod R and keeps only the last R
 *   logical pages ending at the call's last token;
 *   fork (hysenlabs.com write-up, "Experimental Features and Current Limitations": a shared
 *   KV manager with forks and copy-on-write append): an empty sequence takes a copy of
 *   another's page-table rows in every layer and its length; the pages become shared.
 *
 * Arithmetic: bf16 inputs are widened exactly to double; everything after that is fp64;
 * exp/log are the host libm's.  Outputs are never rounded.
 *
 * Every pin of this file lives in tests/test_oracle_pins.py (closed forms, a library
 * routine, brute force and hand-worked page tables).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_OUT_OF_PAGES 3
#define ORC_ERR_NOT_RESIDENT 4 /* a visible token is not (or no longer) stored */

typedef struct {
  int layers, hq, hkv, d, page, window, ring, max_seqs, max_seq_len, num_pages;
  int max_lp;
  uint8_t *cls;       /* [layers][hkv] 1 = global, 0 = local */
  int32_t *free_list; /* [num_pages] */
  int32_t cursor;
  int32_t *pt;   /* page table [layers][max_seqs][hkv][max_lp], -1 = unallocated */
  int32_t *len;  /* tokens appended so far [layers][max_seqs] */
  int64_t *tag;  /* per physical page: which (layer, head, logical page) it holds */
  int32_t *ref;  /* per physical page: page-table slots pointing at it */
  uint16_t *kpool, *vpool; /* [num_pages][page][d] bf16 bits */
} orc_t;

/* A page holds one logical page of one (layer, head); sequences that share it (after a
 * fork) share that content, so the tag leaves the sequence out. */
static int64_t make_tag(const orc_t *o, int layer, int seq, int head, int lp) {
  (void)seq;
  return ((int64_t)layer * o->hkv + head) * (int64_t)o->max_lp + lp;
}

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

orc_t *orc_create(int layers, int hq, int hkv, int d, int page, int window, int ring, int max_seqs,
                  int max_seq_len, int num_pages, const uint8_t *cls, const int32_t *free_list) {
  if (layers < 1 || hkv < 1 || hq < hkv || hq % hkv || d < 1 || page < 1 || window < 1 || ring < 1 ||
      max_seqs < 1 || max_seq_len < 1 || num_pages < 1)
    return NULL;
  orc_t *o = (orc_t *)calloc(1, sizeof(orc_t));
  o->layers = layers; o->hq = hq; o->hkv = hkv; o->d = d; o->page = page; o->window = window;
  o->ring = ring; o->max_seqs = max_seqs; o->max_seq_len = max_seq_len; o->num_pages = num_pages;
  o->max_lp = (max_seq_len + page - 1) / page;
  o->cls = (uint8_t *)malloc((size_t)layers * hkv);
  memcpy(o->cls, cls, (size_t)layers * hkv);
  o->free_list = (int32_t *)malloc(sizeof(int32_t) * (size_t)num_pages);
  memcpy(o->free_list, free_list, sizeof(int32_t) * (size_t)num_pages);
  size_t npt = (size_t)layers * max_seqs * hkv * o->max_lp;
  o->pt = (int32_t *)malloc(sizeof(int32_t) * npt);
  for (size_t i = 0; i < npt; ++i) o->pt[i] = -1;
  o->len = (int32_t *)calloc((size_t)layers * max_seqs, sizeof(int32_t));
  o->tag = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_pages);
  for (int i = 0; i < num_pages; ++i) o->tag[i] = -1;
  o->ref = (int32_t *)calloc((size_t)num_pages, sizeof(int32_t));
  o->kpool = (uint16_t *)calloc((size_t)num_pages * page * d, sizeof(uint16_t));
  o->vpool = (uint16_t *)calloc((size_t)num_pages * page * d, sizeof(uint16_t));
  return o;
}

void orc_destroy(orc_t *o) {
  if (!o) return;
  free(o->cls); free(o->free_list); free(o->pt); free(o->len); free(o->tag); free(o->ref);
  free(o->kpool); free(o->vpool); free(o);
}

const int32_t *orc_page_table(const orc_t *o) { return o->pt; }
int orc_max_lp(const orc_t *o) { return o->max_lp; }
int orc_cursor(const orc_t *o) { return o->cursor; }
int orc_seq_len(const orc_t *o, int layer, int seq) { return o->len[(size_t)layer * o->max_seqs + seq]; }

static int32_t *pt_row(const orc_t *o, int layer, int seq, int head) {
  return o->pt + (((size_t)layer * o->max_seqs + seq) * o->hkv + head) * o->max_lp;
}

/* Slot of logical page lp for a head: a global head stores lp at slot lp, a local head in
 * a ring of R slots. */
static int slot_of(const orc_t *o, int global, int lp) { return global ? lp : lp % o->ring; }

/*
 * Append tokens [start[b], start[b] + count[b]) of sequence seq_ids[b] to every KV head of
 * `layer`.  k_new / v_new are varlen-packed bf16 bits [sum(count), hkv, d], sequences in
 * call order.  Step 1 allocates pages, step 2 stores the tokens each head keeps.
 */
int orc_append(orc_t *o, int layer, int nseq, const int32_t *seq_ids, const int32_t *start,
               const int32_t *count, const uint16_t *k_new, const uint16_t *v_new) {
  const int P = o->page, R = o->ring, H = o->hkv, D = o->d;
  if (layer < 0 || layer >= o->layers) return ORC_ERR_ARG;
  for (int b = 0; b < nseq; ++b) {
    int s = seq_ids[b];
    if (s < 0 || s >= o->max_seqs || count[b] < 0) return ORC_ERR_ARG;
    if (start[b] != o->len[(size_t)layer * o->max_seqs + s]) return ORC_ERR_ARG;
    if (start[b] + count[b] > o->max_seq_len) return ORC_ERR_ARG;
    for (int c = 0; c < b; ++c)
      if (seq_ids[c] == s) return ORC_ERR_ARG;
  }
  /* step 1: page allocation, sequences in call order, heads ascending, pages ascending */
  for (int b = 0; b < nseq; ++b) {
    if (count[b] == 0) continue;
    const int s = seq_ids[b], first = start[b], last = start[b] + count[b] - 1;
    for (int h = 0; h < H; ++h) {
      const int global = o->cls[layer * H + h];
      int lp0 = first / P;
      const int lp1 = last / P;
      if (!global && lp1 - R + 1 > lp0) lp0 = lp1 - R + 1;
      int32_t *row = pt_row(o, layer, s, h);
      for (int lp = lp0; lp <= lp1; ++lp) {
        int slot = slot_of(o, global, lp);
        const int32_t old = row[slot];
        if (old < 0 || o->ref[old] > 1) {
          if (o->cursor >= o->num_pages) return ORC_ERR_OUT_OF_PAGES;
          const int32_t fresh = o->free_list[o->cursor++];
          if (old >= 0) { /* copy on write: the other sequences keep the old page */
            const size_t bytes = sizeof(uint16_t) * (size_t)P * D;
            memcpy(o->kpool + (size_t)fresh * P * D, o->kpool + (size_t)old * P * D, bytes);
            memcpy(o->vpool + (size_t)fresh * P * D, o->vpool + (size_t)old * P * D, bytes);
            o->ref[old]--;
          }
          row[slot] = fresh;
          o->ref[fresh] = 1;
        }
        o->tag[row[slot]] = make_tag(o, layer, s, h, lp);
      }
    }
  }
  /* step 2: store every token the head keeps */
  size_t tok = 0;
  for (int b = 0; b < nseq; ++b) {
    const int s = seq_ids[b], first = start[b], last = start[b] + count[b] - 1;
    for (int pos = first; pos <= last; ++pos, ++tok) {
      const int lp = pos / P;
      for (int h = 0; h < H; ++h) {
        const int global = o->cls[layer * H + h];
        if (!global && lp < last / P - R + 1) continue; /* the ring would overwrite it */
        const int32_t phys = pt_row(o, layer, s, h)[slot_of(o, global, lp)];
        const size_t dst = ((size_t)phys * P + pos % P) * D;
        const size_t src = (tok * H + h) * D;
        memcpy(o->kpool + dst, k_new + src, sizeof(uint16_t) * D);
        memcpy(o->vpool + dst, v_new + src, sizeof(uint16_t) * D);
      }
    }
    o->len[(size_t)layer * o->max_seqs + s] = count[b] > 0 ? last + 1 : first;
  }
  return ORC_OK;
}

/* Fork: the empty sequence dst takes src's page-table rows and length in every layer; every
 * page it now points at gains a reference. */
int orc_fork(orc_t *o, int src, int dst) {
  if (src < 0 || dst < 0 || src >= o->max_seqs || dst >= o->max_seqs || src == dst) return ORC_ERR_ARG;
  for (int l = 0; l < o->layers; ++l)
    if (o->len[(size_t)l * o->max_seqs + dst] != 0) return ORC_ERR_ARG;
  for (int l = 0; l < o->layers; ++l) {
    for (int h = 0; h < o->hkv; ++h) {
      const int32_t *a = pt_row(o, l, src, h);
      int32_t *b = pt_row(o, l, dst, h);
      for (int i = 0; i < o->max_lp; ++i) {
        b[i] = a[i];
        if (a[i] >= 0) o->ref[a[i]]++;
      }
    }
    o->len[(size_t)l * o->max_seqs + dst] = o->len[(size_t)l * o->max_seqs + src];
  }
  return ORC_OK;
}

/* Read token `pos` of (layer, seq, head) through page table and pool.  Returns NULL when
 * the token is not resident (never written, skipped by the ring, or overwritten). */
static const uint16_t *read_token(const orc_t *o, const uint16_t *pool, int layer, int seq, int head,
                                  int pos) {
  if (pos < 0 || pos >= o->len[(size_t)layer * o->max_seqs + seq]) return NULL;
  const int global = o->cls[layer * o->hkv + head];
  const int lp = pos / o->page;
  const int32_t phys = pt_row(o, layer, seq, head)[slot_of(o, global, lp)];
  if (phys < 0 || phys >= o->num_pages) return NULL;
  if (o->tag[phys] != make_tag(o, layer, seq, head, lp)) return NULL;
  return pool + ((size_t)phys * o->page + pos % o->page) * o->d;
}

typedef struct {
  const orc_t *o;
  int layer, nseq;
  const int32_t *seq_ids, *q_start, *q_len, *q_off; /* q_off: first packed row of each seq */
  const uint16_t *q;
  double scale;
  double *out, *lse;
  uint64_t *row_count; /* per (packed token, q head) */
  const int64_t *rows; /* work rows: packed token * hq + q head */
  int64_t nrows;
  int64_t next;
  pthread_mutex_t mu;
  int err;
} job_t;

/* One query row: explicit visibility row, fp64 scores, softmax, weighted sum of V. */
static int one_row(job_t *j, int64_t r, uint8_t *vis, double *x) {
  const orc_t *o = j->o;
  const int D = o->d, G = o->hq / o->hkv;
  const int64_t tok = r / o->hq;
  const int hqi = (int)(r % o->hq);
  int b = 0;
  while (b + 1 < j->nseq && j->q_off[b + 1] <= tok) ++b;
  const int seq = j->seq_ids[b];
  const int p = j->q_start[b] + (int)(tok - j->q_off[b]);
  const int kvh = hqi / G;
  const int global = o->cls[j->layer * o->hkv + kvh];
  const int L = o->len[(size_t)j->layer * o->max_seqs + seq];
  if (p >= L) return ORC_ERR_ARG;
  /* visibility row over every position the sequence has */
  int nvis = 0;
  for (int k = 0; k < L; ++k) {
    vis[k] = global ? (k <= p) : (k <= p && k > p - o->window);
    nvis += vis[k];
  }
  const uint16_t *qr = j->q + (size_t)r * D;
  double m = -INFINITY;
  for (int k = 0; k < L; ++k) {
    if (!vis[k]) continue;
    const uint16_t *kr = read_token(o, o->kpool, j->layer, seq, kvh, k);
    if (!kr) return ORC_ERR_NOT_RESIDENT;
    double acc = 0.0;
    for (int dd = 0; dd < D; ++dd) acc += bf16_to_double(qr[dd]) * bf16_to_double(kr[dd]);
    x[k] = j->scale * acc;
    if (x[k] > m) m = x[k];
  }
  double z = 0.0;
  for (int k = 0; k < L; ++k)
    if (vis[k]) z += exp(x[k] - m);
  double *orow = j->out + (size_t)r * D;
  for (int dd = 0; dd < D; ++dd) orow[dd] = 0.0;
  for (int k = 0; k < L; ++k) {
    if (!vis[k]) continue;
    const uint16_t *vr = read_token(o, o->vpool, j->layer, seq, kvh, k);
    if (!vr) return ORC_ERR_NOT_RESIDENT;
    const double w = exp(x[k] - m) / z;
    for (int dd = 0; dd < D; ++dd) orow[dd] += w * bf16_to_double(vr[dd]);
  }
  j->lse[r] = m + log(z);
  j->row_count[r] = (uint64_t)nvis;
  return ORC_OK;
}

static void *worker(void *arg) {
  job_t *j = (job_t *)arg;
  const int cap = j->o->max_seq_len;
  uint8_t *vis = (uint8_t *)malloc((size_t)cap);
  double *x = (double *)malloc(sizeof(double) * (size_t)cap);
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int64_t i = j->next;
    j->next += 16;
    int err = j->err;
    pthread_mutex_unlock(&j->mu);
    if (i >= j->nrows || err) break;
    int64_t e = i + 16 < j->nrows ? i + 16 : j->nrows;
    for (; i < e; ++i) {
      int rc = one_row(j, j->rows ? j->rows[i] : i, vis, x);
      if (rc) {
        pthread_mutex_lock(&j->mu);
        j->err = rc;
        pthread_mutex_unlock(&j->mu);
        break;
      }
    }
  }
  free(vis);
  free(x);
  return NULL;
}

/*
 * Attention for query rows of `layer`.  Queries of sequence b sit at positions
 * [q_start[b], q_start[b] + q_len[b]); q is varlen-packed bf16 bits [sum(q_len), hq, d].
 * If rows == NULL every (token, q head) row is computed; otherwise only rows[i]
 * (= packed token * hq + q head).  out [.., d] and lse are indexed by row id, so they
 * must span sum(q_len) * hq rows either way.  counts [nseq][hq] accumulates |visible|.
 * Decode is the same call with q_len = 1.
 */
int orc_attention(const orc_t *o, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start,
                  const int32_t *q_len, const uint16_t *q, double scale, const int64_t *rows, int64_t nrows,
                  double *out, double *lse, uint64_t *counts, int nthreads) {
  if (layer < 0 || layer >= o->layers || nseq < 1) return ORC_ERR_ARG;
  int32_t *q_off = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nseq + 1));
  q_off[0] = 0;
  for (int b = 0; b < nseq; ++b) {
    if (seq_ids[b] < 0 || seq_ids[b] >= o->max_seqs || q_len[b] < 0 || q_start[b] < 0) {
      free(q_off);
      return ORC_ERR_ARG;
    }
    q_off[b + 1] = q_off[b] + q_len[b];
  }
  const int64_t total = (int64_t)q_off[nseq] * o->hq;
  job_t j;
  memset(&j, 0, sizeof(j));
  j.o = o; j.layer = layer; j.nseq = nseq; j.seq_ids = seq_ids; j.q_start = q_start; j.q_len = q_len;
  j.q_off = q_off; j.q = q; j.scale = scale; j.out = out; j.lse = lse;
  j.rows = rows; j.nrows = rows ? nrows : total;
  j.row_count = (uint64_t *)calloc((size_t)(total > 0 ? total : 1), sizeof(uint64_t));
  pthread_mutex_init(&j.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, &j);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  pthread_mutex_destroy(&j.mu);
  if (!j.err && counts) {
    for (int64_t i = 0; i < j.nrows; ++i) {
      const int64_t r = rows ? rows[i] : i;
      const int64_t tok = r / o->hq;
      int b = 0;
      while (b + 1 < nseq && q_off[b + 1] <= tok) ++b;
      counts[(size_t)b * o->hq + r % o->hq] += j.row_count[r];
    }
  }
  free(j.row_count);
  free(q_off);
  return j.err;
}

/*
 * Longest-processing-time-first work list.  An item is (sequence b in call order, KV
 * head h, query tile t); a tile holds `tile_pos` consecutive query positions of all G
 * query heads of h.  Its cost is the number of `bn`-aligned key tiles that intersect
 * [lo, q_last], with lo = 0 for a global head and max(0, q_first - W + 1) for a local one.
 * Items are ordered by cost descending, equal costs by item index ascending.
 * items_out receives n rows of (b, h, t, cost); returns n, or -1 if cap is too small.
 */
typedef struct { int32_t b, h, t, cost; int64_t idx; } lpt_item;

static int lpt_cmp(const void *pa, const void *pb) {
  const lpt_item *a = (const lpt_item *)pa, *b = (const lpt_item *)pb;
  if (a->cost != b->cost) return a->cost > b->cost ? -1 : 1;
  return a->idx < b->idx ? -1 : (a->idx > b->idx);
}

int64_t orc_lpt_items(int nseq, const int32_t *q_start, const int32_t *q_len, int hkv, const uint8_t *cls,
                      int window, int tile_pos, int bn, int32_t *items_out, int64_t cap) {
  int64_t n = 0;
  for (int b = 0; b < nseq; ++b) n += (int64_t)hkv * ((q_len[b] + tile_pos - 1) / tile_pos);
  if (n > cap) return -1;
  lpt_item *it = (lpt_item *)malloc(sizeof(lpt_item) * (size_t)(n > 0 ? n : 1));
  int64_t i = 0;
  for (int b = 0; b < nseq; ++b)
    for (int h = 0; h < hkv; ++h)
      for (int t = 0; t * tile_pos < q_len[b]; ++t) {
        const int q_first = q_start[b] + t * tile_pos;
        int q_last = q_start[b] + (t + 1) * tile_pos - 1;
        if (q_last > q_start[b] + q_len[b] - 1) q_last = q_start[b] + q_len[b] - 1;
        int lo = cls[h] ? 0 : q_first - window + 1;
        if (lo < 0) lo = 0;
        it[i].b = b; it[i].h = h; it[i].t = t; it[i].idx = i;
        it[i].cost = q_last / bn - lo / bn + 1;
        ++i;
      }
  qsort(it, (size_t)n, sizeof(lpt_item), lpt_cmp);
  for (i = 0; i < n; ++i) {
    items_out[4 * i + 0] = it[i].b;
    items_out[4 * i + 1] = it[i].h;
    items_out[4 * i + 2] = it[i].t;
    items_out[4 * i + 3] = it[i].cost;
  }
  free(it);
  return n;
}

/*
 * Attention as a router (zhichai.net news item "What Happened", item 2 and its body: dense
 * FFN only on the top-k tokens by attention score, an identity path for the rest;
 * hysenlabs.com write-up, "The Three Core Mechanisms in Detail", second mechanism:
 * token-level importance scores decide which tokens enter the FFN).  The pages do not
 * define the score; the reading taken here is the attention mass a token receives:
 *   score[j] = sum over query heads h and over the call's queries i of sequence b that
 *              see j of  softmax_h(i)[j] = exp(scale q_{i,h}.k_j - lse_{i,h}),
 * for every token j of the call's own query range (the tokens whose FFN rows are being
 * routed).  Each query row is computed as in one_row (explicit visibility row, fp64
 * scores, its own lse); its weights are then added to the scores of the keys in range.
 * scores: fp64 [sum(q_len)], packed like q.
 */
typedef struct {
  job_t base;
  double **acc; /* per worker: fp64 [sum(q_len)] */
  int next_worker;
} router_job_t;

static int router_row(job_t *j, int64_t r, uint8_t *vis, double *x, double *acc) {
  const orc_t *o = j->o;
  const int D = o->d, G = o->hq / o->hkv;
  const int64_t tok = r / o->hq;
  const int hqi = (int)(r % o->hq);
  int b = 0;
  while (b + 1 < j->nseq && j->q_off[b + 1] <= tok) ++b;
  const int seq = j->seq_ids[b];
  const int p = j->q_start[b] + (int)(tok - j->q_off[b]);
  const int kvh = hqi / G;
  const int global = o->cls[j->layer * o->hkv + kvh];
  const int L = o->len[(size_t)j->layer * o->max_seqs + seq];
  if (p >= L) return ORC_ERR_ARG;
  for (int k = 0; k < L; ++k) vis[k] = global ? (k <= p) : (k <= p && k > p - o->window);
  const uint16_t *qr = j->q + (size_t)r * D;
  double m = -INFINITY;
  for (int k = 0; k < L; ++k) {
    if (!vis[k]) continue;
    const uint16_t *kr = read_token(o, o->kpool, j->layer, seq, kvh, k);
    if (!kr) return ORC_ERR_NOT_RESIDENT;
    double s = 0.0;
    for (int dd = 0; dd < D; ++dd) s += bf16_to_double(qr[dd]) * bf16_to_double(kr[dd]);
    x[k] = j->scale * s;
    if (x[k] > m) m = x[k];
  }
  double z = 0.0;
  for (int k = 0; k < L; ++k)
    if (vis[k]) z += exp(x[k] - m);
  const double lse = m + log(z);
  const int k_lo = j->q_start[b], k_hi = j->q_start[b] + j->q_len[b] - 1;
  for (int k = k_lo; k <= k_hi && k < L; ++k)
    if (vis[k]) acc[j->q_off[b] + (k - k_lo)] += exp(x[k] - lse);
  return ORC_OK;
}

static void *router_worker(void *arg) {
  router_job_t *rj = (router_job_t *)arg;
  job_t *j = &rj->base;
  pthread_mutex_lock(&j->mu);
  double *acc = rj->acc[rj->next_worker++];
  pthread_mutex_unlock(&j->mu);
  const int cap = j->o->max_seq_len;
  uint8_t *vis = (uint8_t *)malloc((size_t)cap);
  double *x = (double *)malloc(sizeof(double) * (size_t)cap);
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int64_t i = j->next;
    j->next += 16;
    int err = j->err;
    pthread_mutex_unlock(&j->mu);
    if (i >= j->nrows || err) break;
    int64_t e = i + 16 < j->nrows ? i + 16 : j->nrows;
    for (; i < e; ++i) {
      int rc = router_row(j, i, vis, x, acc);
      if (rc) {
        pthread_mutex_lock(&j->mu);
        j->err = rc;
        pthread_mutex_unlock(&j->mu);
        break;
      }
    }
  }
  free(vis);
  free(x);
  return NULL;
}

int orc_router_scores(const orc_t *o, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start,
                      const int32_t *q_len, const uint16_t *q, double scale, double *scores, int nthreads) {
  if (layer < 0 || layer >= o->layers || nseq < 1) return ORC_ERR_ARG;
  int32_t *q_off = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nseq + 1));
  q_off[0] = 0;
  for (int b = 0; b < nseq; ++b) {
    if (seq_ids[b] < 0 || seq_ids[b] >= o->max_seqs || q_len[b] < 0 || q_start[b] < 0) {
      free(q_off);
      return ORC_ERR_ARG;
    }
    q_off[b + 1] = q_off[b] + q_len[b];
  }
  const int64_t T = q_off[nseq];
  if (nthreads < 1) nthreads = 1;
  router_job_t rj;
  memset(&rj, 0, sizeof(rj));
  job_t *j = &rj.base;
  j->o = o; j->layer = layer; j->nseq = nseq; j->seq_ids = seq_ids; j->q_start = q_start; j->q_len = q_len;
  j->q_off = q_off; j->q = q; j->scale = scale; j->nrows = T * o->hq;
  pthread_mutex_init(&j->mu, NULL);
  rj.acc = (double **)malloc(sizeof(double *) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) rj.acc[t] = (double *)calloc((size_t)(T > 0 ? T : 1), sizeof(double));
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, router_worker, &rj);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  pthread_mutex_destroy(&j->mu);
  for (int64_t i = 0; i < T; ++i) {
    double s = 0.0;
    for (int t = 0; t < nthreads; ++t) s += rj.acc[t][i];
    scores[i] = s;
  }
  for (int t = 0; t < nthreads; ++t) free(rj.acc[t]);
  free(rj.acc);
  free(q_off);
  return j->err;
}
