/*
 * sep_oracle.c -- plain, slow, fp64 CPU oracle for Sep-Attention and the
 * four-block SepCache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or helper with the CUDA library, and the CUDA library never calls it.
 *
 * What each routine follows (pages cited by title and section):
 *   - kept set of query i:  {j <= i : j < a  or  is_sep[j]  or  i - j < n}
 *     "HKUDS047: SepLLM ..." study, section "SepAttention"
 *     (build_prefill_mask: separator columns, initial columns, local
 *     triangular window, AND with the lower-triangular causal mask), and the
 *     jieyibu.net explainer, section 1.2 (binary mask M; masked scores are
 *     set to -inf before softmax).
 *   - scores are scaled dot products q.k; softmax over the kept set; output
 *     is the softmax-weighted sum of v (same explainer, section 1.2).
 *   - four-block cache (initial / separator cache capped at s, oldest
 *     evicted / past-window buffer that keeps only separators when flushed /
 *     local window w): xugj520 article, section 3.3 table; the KV-manager
 *     steps of the HKUDS047 study, section "KV Cache Manager" (select the
 *     separators of the old window, accumulate them onto the old separators,
 *     keep the last sep_cache_size of them).
 *
 * Readings taken where the pages leave a step open (each is also listed in
 * the design notes): a counts initial tokens (kept set j < a); the window
 * is 0 <= i-j < n, so n counts the query itself; scale defaults to
 * 1/sqrt(D); query head h uses kv head h / (Hq/Hkv); lse is the natural log
 * of the softmax denominator over the scaled scores; the past buffer is
 * flushed when it holds more than `past` rows, and all of it is flushed.
 *
 *   - positional-encoding shifting for streaming: the keys kept in the cache
 *     are stored before their position is encoded, and the rotary encoding
 *     of a Llama model is applied at each step with the rows' positions
 *     inside the cache ("HKUDS047: SepLLM ..." study, section on the three
 *     versions: the streaming setting needs positional-encoding shifting;
 *     section "Streaming-SepLLM": the Llama positional-encoding-shifting
 *     module).  The rotary encoding itself is not spelled out on the pages;
 *     the reading taken is the rotate-half form used by Llama models: for
 *     i < D/2 the pair (x_i, x_{i+D/2}) turns by pos * theta^(-2i/D).
 *
 * Arithmetic is fp64 throughout, from the exact input values (fp32 inputs
 * widen exactly; bf16 inputs are the top 16 bits of an fp32).  Threads only
 * split independent rows / sequences; each row's arithmetic is sequential.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* element loaders: dtype 0 = fp32, 1 = bf16 (raw 16-bit patterns), 2 = fp64 */
static double elem(const void* base, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)base)[i];
  if (dtype == 2) return ((const double*)base)[i];
  uint32_t u = ((uint32_t)((const uint16_t*)base)[i]) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------------ */
/* a tiny thread pool: dynamic chunks of an index range               */
/* ------------------------------------------------------------------ */
typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end, int tid);
typedef struct {
  range_fn fn;
  void* ctx;
  int64_t n, chunk;
  int64_t next; /* atomic */
  int tid;
} pool_t;
typedef struct {
  pool_t* p;
  int tid;
} worker_arg;

static void* worker(void* arg) {
  worker_arg* w = (worker_arg*)arg;
  pool_t* p = w->p;
  for (;;) {
    int64_t b = __atomic_fetch_add(&p->next, p->chunk, __ATOMIC_RELAXED);
    if (b >= p->n) break;
    int64_t e = b + p->chunk < p->n ? b + p->chunk : p->n;
    p->fn(p->ctx, b, e, w->tid);
  }
  return NULL;
}

static void parallel_for(int64_t n, int64_t chunk, int nthreads, range_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pool_t p = {fn, ctx, n, chunk < 1 ? 1 : chunk, 0, 0};
  pthread_t th[256];
  worker_arg args[256];
  for (int t = 0; t < nthreads; ++t) {
    args[t].p = &p;
    args[t].tid = t;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, &args[t]);
  worker(&args[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------ */
/* separator flags and the index list                                  */
/* ------------------------------------------------------------------ */

/* is_sep[t] = 1 iff ids[t] is one of the separator ids
 * (HKUDS047 study, section "SepAttention": token_id in separator_token_ids). */
int oracle_flags_from_ids(const int32_t* ids, int64_t n_tok, const int32_t* sep_ids, int n_sep,
                          uint8_t* is_sep) {
  for (int64_t t = 0; t < n_tok; ++t) {
    uint8_t f = 0;
    for (int k = 0; k < n_sep; ++k)
      if (ids[t] == sep_ids[k]) f = 1;
    is_sep[t] = f;
  }
  return 0;
}

/* prefix[b][j] = number of separators among positions < j (j = 0..S);
 * idx[b][k] = position of the k-th separator, in increasing order, then -1;
 * count[b] = prefix[b][S]. */
int oracle_build_index(const uint8_t* is_sep, int B, int S, int32_t* prefix, int32_t* idx,
                       int32_t* count) {
  for (int b = 0; b < B; ++b) {
    const uint8_t* f = is_sep + (int64_t)b * S;
    int32_t* pre = prefix + (int64_t)b * (S + 1);
    int32_t* ix = idx + (int64_t)b * S;
    int32_t c = 0;
    pre[0] = 0;
    for (int j = 0; j < S; ++j) {
      if (f[j]) ix[c++] = j;
      pre[j + 1] = c;
    }
    for (int k = c; k < S; ++k) ix[k] = -1;
    count[b] = c;
  }
  return 0;
}

/* the kept predicate of one (query i, key j) pair */
static int kept(const uint8_t* sep_row, int a, int n, int64_t i, int64_t j) {
  if (j > i) return 0; /* causal */
  return (j < a) || sep_row[j] || (i - j < n);
}

/* ------------------------------------------------------------------ */
/* kept-pair counts (retention statistics)                             */
/* ------------------------------------------------------------------ */
typedef struct {
  const uint8_t* sep_row;
  int S, a, n;
  int64_t* partial; /* per thread */
} count_ctx;

static void count_rows(void* vctx, int64_t begin, int64_t end, int tid) {
  count_ctx* c = (count_ctx*)vctx;
  int64_t acc = 0;
  for (int64_t i = begin; i < end; ++i)
    for (int64_t j = 0; j <= i; ++j) acc += kept(c->sep_row, c->a, c->n, i, j);
  c->partial[tid] += acc;
}

/* kept_pairs[b] = number of (i, j) pairs of sequence b that one head keeps,
 * counted by testing every causal pair. */
int oracle_count_pairs(const uint8_t* is_sep, int B, int S, int a, int n, int64_t* kept_pairs,
                       int nthreads) {
  for (int b = 0; b < B; ++b) {
    int64_t partial[256] = {0};
    count_ctx c = {is_sep + (int64_t)b * S, S, a, n, partial};
    parallel_for(S, 64, nthreads, count_rows, &c);
    int64_t tot = 0;
    for (int t = 0; t < 256; ++t) tot += partial[t];
    kept_pairs[b] = tot;
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* explicit-mask attention over the kept set                           */
/* ------------------------------------------------------------------ */

/* softmax attention of one query row over an explicit list of key rows:
 *   s_t = scale * sum_d q[d] k_t[d];  m = max s;  l = sum exp(s_t - m);
 *   out[d] = sum_t exp(s_t - m) v_t[d] / l;  lse = m + ln l. */
static void attend_list(const double* q, const void* k, const void* v, int dtype,
                        const int64_t* krow, int64_t nk, int D, double scale, double* sc,
                        double* out, double* lse) {
  double m = -INFINITY;
  for (int64_t t = 0; t < nk; ++t) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += q[d] * elem(k, dtype, krow[t] * D + d);
    s *= scale;
    sc[t] = s;
    if (s > m) m = s;
  }
  double l = 0.0;
  for (int64_t t = 0; t < nk; ++t) {
    sc[t] = exp(sc[t] - m); /* unnormalised weight of key t */
    l += sc[t];
  }
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int64_t t = 0; t < nk; ++t)
    for (int d = 0; d < D; ++d) out[d] += sc[t] * elem(v, dtype, krow[t] * D + d);
  for (int d = 0; d < D; ++d) out[d] /= l;
  *lse = m + log(l);
}

typedef struct {
  const void *q, *k, *v;
  int dtype;
  const uint8_t* is_sep;
  int B, Hq, Hkv, S, D, a, n;
  double scale;
  const int64_t* rows;
  double *out, *lse;
  int64_t** scratch_rows; /* per thread, S entries */
  double** scratch_sc;    /* per thread, S entries */
} prefill_ctx;

static void prefill_range(void* vctx, int64_t begin, int64_t end, int tid) {
  prefill_ctx* c = (prefill_ctx*)vctx;
  int G = c->Hq / c->Hkv;
  int D = c->D;
  double qd[512];
  int64_t* krow = c->scratch_rows[tid];
  double* sc = c->scratch_sc[tid];
  for (int64_t r = begin; r < end; ++r) {
    int64_t id = c->rows[r];
    int64_t i = id % c->S;
    int64_t bh = id / c->S;
    int64_t h = bh % c->Hq;
    int64_t b = bh / c->Hq;
    int64_t g = h / G; /* contiguous query-head groups */
    const uint8_t* sep_row = c->is_sep + b * c->S;
    for (int d = 0; d < D; ++d) qd[d] = elem(c->q, c->dtype, id * D + d);
    int64_t kv_base = (b * c->Hkv + g) * c->S; /* row index of key 0 */
    int64_t nk = 0;
    for (int64_t j = 0; j <= i; ++j)
      if (kept(sep_row, c->a, c->n, i, j)) krow[nk++] = kv_base + j;
    attend_list(qd, c->k, c->v, c->dtype, krow, nk, D, c->scale, sc, c->out + r * D, c->lse + r);
  }
}

/* Sep-Attention prefill rows.  q [B,Hq,S,D], k/v [B,Hkv,S,D], is_sep [B,S].
 * rows[r] = (b*Hq + h)*S + i selects the query rows to compute;
 * out [nrows, D] and lse [nrows] are fp64.  scale <= 0 means 1/sqrt(D). */
int oracle_prefill_rows(const void* q, const void* k, const void* v, int dtype,
                        const uint8_t* is_sep, int B, int Hq, int Hkv, int S, int D, int a, int n,
                        double scale, const int64_t* rows, int64_t nrows, double* out, double* lse,
                        int nthreads) {
  if (D > 512 || Hkv <= 0 || Hq % Hkv != 0) return -1;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  int64_t* srows[256];
  double* ssc[256];
  for (int t = 0; t < nthreads; ++t) {
    srows[t] = (int64_t*)malloc(sizeof(int64_t) * (size_t)S);
    ssc[t] = (double*)malloc(sizeof(double) * (size_t)S);
  }
  prefill_ctx c = {q,  k, v, dtype, is_sep, B,     Hq,  Hkv,  S,     D,  a,
                   n, scale, rows, out, lse, srows, ssc};
  parallel_for(nrows, 16, nthreads, prefill_range, &c);
  for (int t = 0; t < nthreads; ++t) {
    free(srows[t]);
    free(ssc[t]);
  }
  return 0;
}

/* Attention of Hq query heads over L key rows each (decode over a cache
 * whose retained rows the caller lists): q [Hq,D], k/v [Hkv,L,D];
 * out [Hq,D], lse [Hq] in fp64.  scale <= 0 means 1/sqrt(D). */
int oracle_attend(const void* q, const void* k, const void* v, int dtype, int Hq, int Hkv, int L,
                  int D, double scale, double* out, double* lse) {
  if (D > 512 || Hkv <= 0 || Hq % Hkv != 0 || L < 1) return -1;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  int G = Hq / Hkv;
  double qd[512];
  int64_t* krow = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
  double* sc = (double*)malloc(sizeof(double) * (size_t)L);
  for (int h = 0; h < Hq; ++h) {
    int g = h / G;
    for (int d = 0; d < D; ++d) qd[d] = elem(q, dtype, (int64_t)h * D + d);
    for (int t = 0; t < L; ++t) krow[t] = (int64_t)g * L + t;
    attend_list(qd, k, v, dtype, krow, L, D, scale, sc, out + (int64_t)h * D, lse + h);
  }
  free(krow);
  free(sc);
  return 0;
}

/* ------------------------------------------------------------------ */
/* the four-block SepCache state machine                               */
/* ------------------------------------------------------------------ */
typedef struct {
  int32_t* pos;
  uint8_t* flag;
  int n;
} blk;

static void blk_push(blk* x, int32_t p, uint8_t f) {
  x->pos[x->n] = p;
  x->flag[x->n] = f;
  x->n++;
}

/* Simulate T tokens of B independent sequences; flags [T,B].
 * Per token t with separator flag f (xugj520 article, section 3.3 table):
 *   1. while the initial cache holds fewer than a tokens, t joins it;
 *      otherwise t joins the local window, and when the window then holds
 *      more than w tokens its oldest token moves to the back of the past
 *      window;
 *   2. when the past window then holds more than `past` tokens it is
 *      flushed: its separators are appended to the separator cache, which
 *      keeps only its last s entries (oldest evicted), and the past window
 *      empties.
 * After the token at step snap_steps[k] the cache I|S|P|L is written to
 * snap_pos/snap_flag [nsnap,B,cap] (-1 / 0 padded) and the block sizes to
 * snap_counts [nsnap,B,4] = (|I|,|S|,|P|,|L|).  flushed [T,B] (optional)
 * marks the steps whose token triggered a flush.  snap_steps ascending.
 *
 * mode bits, the KV manager's switches and its compression condition
 * ("HKUDS047: SepLLM ..." study, section "KV Cache Manager": the
 * SEP_ACCUMULATION and USE_MAX_SEP_CACHE branches of the compression step,
 * and compression when the sequence exceeds cache_size):
 *   1  no accumulation: a flush keeps only the separators of the flushed
 *      past window (the old separator cache is dropped), newest s of them;
 *   2  no maximum on the separator cache: separators are never evicted; the
 *      s rows are its capacity, and a flush that would need more sets
 *      overflowed[b] and keeps the newest s;
 *   4  total-length trigger: flush when |I|+|S|+|P|+|L| > a+s+past+w instead
 *      of when |P| > past (the same once |S| = s).
 * overflowed [B] (optional) receives the mode-2 overflow flag. */
int oracle_sepcache_simulate(const uint8_t* flags, int B, int64_t T, int a, int s, int past, int w,
                             const int64_t* snap_steps, int nsnap, int cap, int32_t* snap_pos,
                             uint8_t* snap_flag, int32_t* snap_counts, uint8_t* flushed, int mode,
                             uint8_t* overflowed) {
  if (a < 0 || s < 0 || past < 0 || w < 1 || (mode & ~7) != 0) return -1;
  /* under the total-length trigger the past window holds up to past + s */
  int capI = a + 1, capS = s + 1, capP = past + s + 2, capL = w + 2;
  int32_t* bufp = (int32_t*)malloc(sizeof(int32_t) * (size_t)(capI + capS + capP + capL) * 2);
  uint8_t* buff = (uint8_t*)malloc((size_t)(capI + capS + capP + capL) * 2);
  for (int k = 0; k < nsnap; ++k)
    for (int b = 0; b < B; ++b)
      for (int r = 0; r < cap; ++r) {
        snap_pos[((int64_t)k * B + b) * cap + r] = -1;
        snap_flag[((int64_t)k * B + b) * cap + r] = 0;
      }
  int rc = 0;
  for (int b = 0; b < B && rc == 0; ++b) {
    int32_t* p0 = bufp;
    uint8_t* f0 = buff;
    blk I = {p0, f0, 0};
    blk Sb = {p0 + capI, f0 + capI, 0};
    blk P = {p0 + capI + capS, f0 + capI + capS, 0};
    blk L = {p0 + capI + capS + capP, f0 + capI + capS + capP, 0};
    /* scratch for the flush candidates */
    int32_t* cp = p0 + capI + capS + capP + capL;
    uint8_t* cf = f0 + capI + capS + capP + capL;
    int ks = 0;
    for (int64_t t = 0; t < T; ++t) {
      uint8_t f = flags[t * B + b];
      int did_flush = 0;
      /* 1. place the token */
      if (I.n < a) {
        blk_push(&I, (int32_t)t, f);
      } else {
        blk_push(&L, (int32_t)t, f);
        if (L.n > w) {
          blk_push(&P, L.pos[0], L.flag[0]);
          memmove(L.pos, L.pos + 1, sizeof(int32_t) * (size_t)(L.n - 1));
          memmove(L.flag, L.flag + 1, (size_t)(L.n - 1));
          L.n--;
        }
      }
      /* 2. flush the past window when it overflows (or the whole cache,
       *    under the total-length trigger) */
      int over = (mode & 4) ? (I.n + Sb.n + P.n + L.n > a + s + past + w) : (P.n > past);
      if (over) {
        int nc = 0;
        if (!(mode & 1))
          for (int r = 0; r < Sb.n; ++r) {
            cp[nc] = Sb.pos[r];
            cf[nc] = Sb.flag[r];
            nc++;
          }
        for (int r = 0; r < P.n; ++r)
          if (P.flag[r]) {
            cp[nc] = P.pos[r];
            cf[nc] = P.flag[r];
            nc++;
          }
        int keep = nc < s ? nc : s;
        if ((mode & 2) && nc > s && overflowed) overflowed[b] = 1;
        Sb.n = 0;
        for (int r = nc - keep; r < nc; ++r) blk_push(&Sb, cp[r], cf[r]);
        P.n = 0;
        did_flush = 1;
      }
      if (flushed) flushed[t * B + b] = (uint8_t)did_flush;
      /* invariant of the budget contract: never above a+s+past+w */
      if (I.n + Sb.n + P.n + L.n > a + s + past + w) rc = -2;
      while (ks < nsnap && snap_steps[ks] < t) ks++;
      while (ks < nsnap && snap_steps[ks] == t) {
        int64_t base = ((int64_t)ks * B + b) * cap;
        int r = 0;
        blk* order[4] = {&I, &Sb, &P, &L};
        for (int q = 0; q < 4; ++q)
          for (int e = 0; e < order[q]->n; ++e) {
            if (r < cap) {
              snap_pos[base + r] = order[q]->pos[e];
              snap_flag[base + r] = order[q]->flag[e];
            }
            r++;
          }
        if (r > cap) rc = -3;
        int32_t* cnt = snap_counts + ((int64_t)ks * B + b) * 4;
        cnt[0] = I.n;
        cnt[1] = Sb.n;
        cnt[2] = P.n;
        cnt[3] = L.n;
        ks++;
      }
    }
  }
  free(bufp);
  free(buff);
  return rc;
}

/* ------------------------------------------------------------------ */
/* rotary position encoding and the position-shifted decode            */
/* ------------------------------------------------------------------ */

/* Rotate each of the nrows rows of x [nrows, D] to the position pos[r]:
 * for i < D/2, with phi = pos[r] * theta^(-2i/D),
 *   out_i       = x_i cos(phi) - x_{i+D/2} sin(phi)
 *   out_{i+D/2} = x_{i+D/2} cos(phi) + x_i sin(phi)
 * i.e. the complex number x_i + j x_{i+D/2} times exp(j phi).  fp64 out. */
int oracle_rope(const void* x, int dtype, int64_t nrows, int D, const int64_t* pos, double theta,
                double* out) {
  if (D < 2 || D % 2 != 0 || !(theta > 0.0)) return -1;
  int half = D / 2;
  for (int64_t r = 0; r < nrows; ++r) {
    for (int i = 0; i < half; ++i) {
      double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
      double phi = (double)pos[r] * inv_freq;
      double c = cos(phi), sn = sin(phi);
      double a = elem(x, dtype, r * D + i);
      double b = elem(x, dtype, r * D + i + half);
      out[r * D + i] = a * c - b * sn;
      out[r * D + i + half] = b * c + a * sn;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* Sep-Attention backward                                              */
/* ------------------------------------------------------------------ */
/* Gradients of L = sum_{b,h,i,d} out[b,h,i,d] * dout[b,h,i,d] with respect
 * to q, k, v, where out is the Sep-Attention of the prefill (kept set of row
 * i: {j <= i : j < a or is_sep[j] or i - j < n}; the training use of the
 * sparse attention, "HKUDS047: SepLLM ..." study, section on the three
 * versions: Training-SepLLM).  For each row i over its kept keys j:
 *   s_j = scale q_i.k_j,  p_j = exp(s_j - m) / sum_t exp(s_t - m),
 *   out_i = sum_j p_j v_j,  delta_i = dout_i . out_i,
 *   dv_j += p_j dout_i,  ds_j = p_j (dout_i . v_j - delta_i),
 *   dq_i += scale sum_j ds_j k_j,  dk_j += scale ds_j q_i.
 * (the chain rule through the softmax: d s_j = p_j (d p-term - sum_t p_t d p-term)).
 * q, dout [B,Hq,S,D]; k, v [B,Hkv,S,D] (dtype 0 fp32, 1 bf16 bits, 2 fp64;
 * dout has its own dtype); dq [B,Hq,S,D], dk, dv [B,Hkv,S,D] fp64 out.
 * Threads split (b, kv head) units; every query head of a group runs in the
 * same thread, so its dk/dv sums are race-free. */
typedef struct {
  const void *q, *k, *v, *dout;
  int dtype, dtype_o;
  const uint8_t* is_sep;
  int B, Hq, Hkv, S, D, a, n;
  double scale;
  double *dq, *dk, *dv;
} bwd_ctx;

static void bwd_range(void* vctx, int64_t begin, int64_t end, int tid) {
  (void)tid;
  bwd_ctx* c = (bwd_ctx*)vctx;
  int G = c->Hq / c->Hkv, D = c->D, S = c->S;
  int64_t* krow = (int64_t*)malloc(sizeof(int64_t) * (size_t)S);
  double* p = (double*)malloc(sizeof(double) * (size_t)S);
  double qd[512], od[512], go[512];
  for (int64_t u = begin; u < end; ++u) {
    int64_t b = u / c->Hkv, g = u % c->Hkv;
    const uint8_t* sep_row = c->is_sep + b * S;
    int64_t kv_base = (b * c->Hkv + g) * (int64_t)S;
    for (int64_t h = g * G; h < (g + 1) * G; ++h) {
      int64_t qrow0 = (b * c->Hq + h) * (int64_t)S;
      for (int64_t i = 0; i < S; ++i) {
        int64_t qi = qrow0 + i;
        for (int d = 0; d < D; ++d) {
          qd[d] = elem(c->q, c->dtype, qi * D + d);
          go[d] = elem(c->dout, c->dtype_o, qi * D + d);
        }
        int64_t nk = 0;
        for (int64_t j = 0; j <= i; ++j)
          if (kept(sep_row, c->a, c->n, i, j)) krow[nk++] = kv_base + j;
        double m = -INFINITY;
        for (int64_t t = 0; t < nk; ++t) {
          double s = 0.0;
          for (int d = 0; d < D; ++d) s += qd[d] * elem(c->k, c->dtype, krow[t] * D + d);
          s *= c->scale;
          p[t] = s;
          if (s > m) m = s;
        }
        double l = 0.0;
        for (int64_t t = 0; t < nk; ++t) {
          p[t] = exp(p[t] - m);
          l += p[t];
        }
        for (int d = 0; d < D; ++d) od[d] = 0.0;
        for (int64_t t = 0; t < nk; ++t) {
          p[t] /= l;
          for (int d = 0; d < D; ++d) od[d] += p[t] * elem(c->v, c->dtype, krow[t] * D + d);
        }
        double delta = 0.0;
        for (int d = 0; d < D; ++d) delta += go[d] * od[d];
        double* dqi = c->dq + qi * D;
        for (int64_t t = 0; t < nk; ++t) {
          double dp = 0.0;
          for (int d = 0; d < D; ++d) dp += go[d] * elem(c->v, c->dtype, krow[t] * D + d);
          double ds = p[t] * (dp - delta);
          double* dkj = c->dk + krow[t] * D;
          double* dvj = c->dv + krow[t] * D;
          for (int d = 0; d < D; ++d) {
            dvj[d] += p[t] * go[d];
            dkj[d] += c->scale * ds * qd[d];
            dqi[d] += c->scale * ds * elem(c->k, c->dtype, krow[t] * D + d);
          }
        }
      }
    }
  }
  free(krow);
  free(p);
}

int oracle_prefill_backward(const void* q, const void* k, const void* v, int dtype,
                            const void* dout, int dtype_o, const uint8_t* is_sep, int B, int Hq,
                            int Hkv, int S, int D, int a, int n, double scale, double* dq,
                            double* dk, double* dv, int nthreads) {
  if (D > 512 || Hkv <= 0 || Hq % Hkv != 0 || S < 1 || n < 1 || a < 0) return -1;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  if (nthreads < 1) nthreads = 1;
  memset(dq, 0, sizeof(double) * (size_t)B * Hq * S * D);
  memset(dk, 0, sizeof(double) * (size_t)B * Hkv * S * D);
  memset(dv, 0, sizeof(double) * (size_t)B * Hkv * S * D);
  bwd_ctx c = {q, k, v, dout, dtype, dtype_o, is_sep, B, Hq, Hkv, S, D, a, n, scale, dq, dk, dv};
  parallel_for((int64_t)B * Hkv, 1, nthreads, bwd_range, &c);
  return 0;
}
