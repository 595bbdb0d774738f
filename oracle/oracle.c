/*
 * oracle.c -- FP64 CPU reference for attention over a KV cache.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the test suite, the smoke check and the
 * benchmark's CPU-baseline leg, never by the library.  Shares no code with
 * the CUDA path.  The definition it implements, and the pages it follows, are
 * stated in oracle.h.
 *
 * Structure: one work unit per query row.  For a row the visible cell set is
 * built once (ascending cell order), then for every query head the logits are
 * formed, the max is taken, and the weighted sum is accumulated in ascending
 * cell order.  Threads take rows from a shared counter.
 */
#define _GNU_SOURCE
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

static int g_mutation = 0;
void oracle_set_mutation(int m) { g_mutation = m; }
int  oracle_get_mutation(void)  { return g_mutation; }

/* Planted mistakes (only the mutation tests set these). */
enum {
    MUT_NONE = 0,
    MUT_ALIBI_BEFORE_SOFTCAP = 1,  /* transform order reversed                 */
    MUT_SINK_NOT_IN_SUM = 2,       /* sink only in the max, not in L           */
    MUT_ALIBI_SIGN = 3,            /* +slope*|dpos| instead of -slope*|dpos|   */
    MUT_NAN_DROPPED = 4,           /* max ignores NaN logits (fmax semantics)  */
    MUT_EMPTY_ROW_NAN = 5,         /* exp(-inf - -inf) left unguarded          */
    MUT_GQA_MODULO = 6,            /* g = h % Hkv instead of floor(h / G)      */
    MUT_NO_DEDUP = 7,              /* duplicate selections counted again       */
    MUT_MASK_NARROWED = 8,         /* mask clamped to the F16 range            */
    MUT_INVALID_CLAMPED = 9,       /* invalid selections clamped into range    */
    MUT_SCALE_AFTER_CAP = 10,      /* scale applied after the softcap          */
    MUT_NEG_INF_MASK_ADDED = 11,   /* -inf mask cell added, not excluded       */
    MUT_CAUSAL_STRICT = 12,        /* cell_pos < row_pos (drops the diagonal)  */
    MUT_SEQ_IGNORED = 13,          /* sequence filter not applied              */
    MUT_K_D_REVERSED = 14,         /* score reads k[c,g,D-1-d]                 */
    MUT_CELL_POS_NO_BEGIN = 15,    /* default cell position c, not c - begin   */
    MUT_ROW_POS_NO_MINUS1 = 16,    /* default row position end - begin         */
    MUT_POS_FROM_CLIPPED = 17,     /* default positions from the clipped range */
};

static int n_online_cores(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* ---- visibility --------------------------------------------------------- */

static int32_t row_begin_of(const oracle_problem *p, int r) {
    int32_t b = p->row_begin ? p->row_begin[r] : 0;
    if (g_mutation == MUT_POS_FROM_CLIPPED && b < 0) b = 0;
    return b;
}
static int32_t row_end_of(const oracle_problem *p, int r) {
    int32_t e = p->row_end ? p->row_end[r] : p->n_cells;
    if (g_mutation == MUT_POS_FROM_CLIPPED && e > p->n_cells) e = p->n_cells;
    return e;
}
/* Default positions (cell c at c - begin, the row at end - begin - 1) come
 * from the range as the caller gave it; only visibility clips it to the cache. */
static int64_t row_pos_of(const oracle_problem *p, int r) {
    if (p->row_pos) return p->row_pos[r];
    if (g_mutation == MUT_ROW_POS_NO_MINUS1) return (int64_t)row_end_of(p, r) - row_begin_of(p, r);
    return (int64_t)row_end_of(p, r) - row_begin_of(p, r) - 1;
}
static int64_t cell_pos_of(const oracle_problem *p, int r, int32_t c) {
    if (p->cell_pos) return p->cell_pos[c];
    if (g_mutation == MUT_CELL_POS_NO_BEGIN) return (int64_t)c;
    return (int64_t)c - row_begin_of(p, r);
}

static int cmp_i32(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Distinct valid entries of one selection list, ascending.  Returns count. */
static int32_t compact_list(const int32_t *list, int32_t n_sel, int32_t n_cells,
                            int32_t *out) {
    int32_t n = 0;
    for (int32_t i = 0; i < n_sel; ++i) {
        int32_t e = list[i];
        if (g_mutation == MUT_INVALID_CLAMPED) {
            if (e < 0) e = 0;
            if (e >= n_cells) e = n_cells - 1;
        }
        if (e >= 0 && e < n_cells) out[n++] = e;
    }
    qsort(out, (size_t)n, sizeof(int32_t), cmp_i32);
    if (g_mutation == MUT_NO_DEDUP) return n;
    int32_t m = 0;
    for (int32_t i = 0; i < n; ++i)
        if (m == 0 || out[i] != out[m - 1]) out[m++] = out[i];
    return m;
}

/* Visible cells of row r, ascending; returns count.  cells must hold
 * max(n_cells, n_sel) entries. */
static int32_t visible_cells(const oracle_problem *p, int r, int32_t *cells) {
    if (p->sel)
        return compact_list(p->sel + (int64_t)r * p->sel_stride_row, p->n_sel,
                            p->n_cells, cells);
    int32_t b = row_begin_of(p, r), e = row_end_of(p, r), n = 0;
    if (b < 0) b = 0;
    if (e > p->n_cells) e = p->n_cells;
    int64_t rp = row_pos_of(p, r);
    for (int32_t c = b; c < e; ++c) {
        if (p->cell_seq && p->row_seq && g_mutation != MUT_SEQ_IGNORED &&
            p->cell_seq[c] != p->row_seq[r])
            continue;
        if (p->causal) {
            int64_t cp = cell_pos_of(p, r, c);
            if (g_mutation == MUT_CAUSAL_STRICT ? !(cp < rp) : !(cp <= rp)) continue;
        }
        if (p->mask && g_mutation != MUT_NEG_INF_MASK_ADDED) {
            float mv = p->mask[(int64_t)r * p->mask_stride_row + c];
            if (isinf(mv) && mv < 0) continue;
        }
        cells[n++] = c;
    }
    return n;
}

/* ---- logits -------------------------------------------------------------- */

static double logit(const oracle_problem *p, int r, int h, int g, int32_t c) {
    const double *q = p->q + (int64_t)r * p->q_stride_row + (int64_t)h * p->q_stride_head;
    const double *k = p->k + (int64_t)c * p->kv_stride_cell + (int64_t)g * p->kv_stride_head;
    const int D = p->head_dim;
    double dot = 0.0;
    for (int d = 0; d < D; ++d)
        dot += q[d] * k[g_mutation == MUT_K_D_REVERSED ? D - 1 - d : d];

    double x = p->scale * dot;
    double alibi = 0.0;
    if (p->alibi_slopes) {
        int64_t dp = row_pos_of(p, r) - cell_pos_of(p, r, c);
        double dist = (double)(dp < 0 ? -dp : dp);
        alibi = (double)p->alibi_slopes[h] * (g_mutation == MUT_ALIBI_SIGN ? dist : -dist);
    }
    if (g_mutation == MUT_ALIBI_BEFORE_SOFTCAP) {
        x += alibi;
        if (p->softcap > 0) x = p->softcap * tanh(x / p->softcap);
    } else if (g_mutation == MUT_SCALE_AFTER_CAP) {
        x = dot;
        if (p->softcap > 0) x = p->softcap * tanh(x / p->softcap);
        x = p->scale * x + alibi;
    } else {
        /* softcap first, then ALiBi (HartsyInference #910, flash_attn_f32.cu fix) */
        if (p->softcap > 0) x = p->softcap * tanh(x / p->softcap);
        x += alibi;
    }
    if (p->mask && !p->sel) {
        float mv = p->mask[(int64_t)r * p->mask_stride_row + c];
        if (g_mutation == MUT_MASK_NARROWED) {
            if (mv > 65504.0f) mv = 65504.0f;
            if (mv < -65504.0f) mv = -65504.0f;
        }
        x += (double)mv;   /* F32 bias widened, never narrowed (#910) */
    }
    return x;
}

/* ---- one row ------------------------------------------------------------- */

typedef struct {
    const oracle_problem *p;
    double *out;
    int n_slices;              /* 0: plain definition; >0: split form       */
    atomic_int next_row;
} job_t;

typedef struct {
    int32_t *cells;
    double *x;                 /* logits of the visible cells               */
    double *acc;               /* head_dim accumulator                      */
} scratch_t;

static void fill(double *o, int D, double v) { for (int d = 0; d < D; ++d) o[d] = v; }

/* Plain definition for one (row, head). */
static void row_head_plain(const oracle_problem *p, int r, int h, const int32_t *cells,
                           int32_t nv, scratch_t *s, double *o) {
    const int D = p->head_dim;
    const int G = p->n_head_q / p->n_head_kv;
    const int g = (g_mutation == MUT_GQA_MODULO) ? h % p->n_head_kv : h / G;

    int any_nan = 0;
    for (int32_t i = 0; i < nv; ++i) {
        s->x[i] = logit(p, r, h, g, cells[i]);
        if (isnan(s->x[i])) any_nan = 1;
    }
    double sigma = p->sinks ? (double)p->sinks[h] : -INFINITY;
    if (isnan(sigma)) any_nan = 1;
    if (g_mutation == MUT_NAN_DROPPED) any_nan = 0;
    if (any_nan) { fill(o, D, NAN); return; }

    double M = sigma;
    for (int32_t i = 0; i < nv; ++i)
        if (g_mutation == MUT_NAN_DROPPED ? (s->x[i] > M) : (s->x[i] > M)) M = s->x[i];

    if (g_mutation != MUT_EMPTY_ROW_NAN) {
        if (isinf(M) && M < 0) { fill(o, D, 0.0); return; }
        if (nv == 0 && isfinite(sigma)) { fill(o, D, 0.0); return; }
    }

    double L = 0.0;
    fill(s->acc, D, 0.0);
    for (int32_t i = 0; i < nv; ++i) {
        if (g_mutation == MUT_NAN_DROPPED && isnan(s->x[i])) continue;
        double w = exp(s->x[i] - M);
        L += w;
        const double *v = p->v + (int64_t)cells[i] * p->kv_stride_cell +
                          (int64_t)g * p->kv_stride_head;
        for (int d = 0; d < D; ++d) s->acc[d] += w * v[d];
    }
    if (g_mutation != MUT_SINK_NOT_IN_SUM) L += exp(sigma - M);  /* 0 when sigma = -inf */
    for (int d = 0; d < D; ++d) o[d] = s->acc[d] / L;
}

/* Split form for one (row, head): cut [begin, end) into n_slices pieces on a
 * 32-cell grid, reduce each piece to (m, l, o), fold in slice order with the
 * sink.  Mirrors the plain definition exactly up to FP64 rounding order.   */
static void row_head_split(const oracle_problem *p, int r, int h, int n_slices,
                           const int32_t *cells, int32_t nv, scratch_t *s, double *o) {
    const int D = p->head_dim;
    const int G = p->n_head_q / p->n_head_kv;
    const int g = h / G;
    int32_t b = row_begin_of(p, r), e = row_end_of(p, r);
    if (b < 0) b = 0;
    if (e > p->n_cells) e = p->n_cells;
    int64_t len = e > b ? (int64_t)e - b : 0;
    int64_t chunks = (len + 31) / 32;

    double *ms = (double *)malloc(sizeof(double) * (size_t)n_slices * (size_t)(D + 2));
    double *ls = ms + n_slices;
    double *os = ls + n_slices;

    int32_t ci = 0;   /* cursor into the ascending visible list */
    for (int sl = 0; sl < n_slices; ++sl) {
        int64_t c0 = b + 32 * ((chunks * sl) / n_slices);
        int64_t c1 = b + 32 * ((chunks * (sl + 1)) / n_slices);
        if (c1 > e) c1 = e;
        double *osl = os + (int64_t)sl * D;
        /* visible cells of this slice */
        int32_t i0 = ci;
        while (ci < nv && cells[ci] < c1) ++ci;
        int32_t i1 = ci;
        (void)c0;
        double m = -INFINITY;
        int nan_seen = 0;
        for (int32_t i = i0; i < i1; ++i) {
            s->x[i] = logit(p, r, h, g, cells[i]);
            if (isnan(s->x[i])) nan_seen = 1;
            else if (s->x[i] > m) m = s->x[i];
        }
        if (nan_seen) m = NAN;
        double mu = (isinf(m) && m < 0) ? 0.0 : m;   /* guard exp(-inf - -inf) */
        double l = 0.0;
        fill(osl, D, 0.0);
        for (int32_t i = i0; i < i1; ++i) {
            double w = exp(s->x[i] - mu);
            l += w;
            const double *v = p->v + (int64_t)cells[i] * p->kv_stride_cell +
                              (int64_t)g * p->kv_stride_head;
            for (int d = 0; d < D; ++d) osl[d] += w * v[d];
        }
        ms[sl] = m;
        ls[sl] = l;
    }

    double sigma = p->sinks ? (double)p->sinks[h] : -INFINITY;
    int any_nan = isnan(sigma);
    double M = sigma;
    for (int sl = 0; sl < n_slices; ++sl) {
        if (isnan(ms[sl])) any_nan = 1;
        else if (ms[sl] > M) M = ms[sl];
    }
    if (any_nan) { fill(o, D, NAN); free(ms); return; }
    if (isinf(M) && M < 0) { fill(o, D, 0.0); free(ms); return; }
    double L = exp(sigma - M);
    fill(s->acc, D, 0.0);
    for (int sl = 0; sl < n_slices; ++sl) {
        double f = exp(ms[sl] - M);          /* 0 for an empty slice */
        L += ls[sl] * f;
        for (int d = 0; d < D; ++d) s->acc[d] += os[(int64_t)sl * D + d] * f;
    }
    for (int d = 0; d < D; ++d) o[d] = s->acc[d] / L;
    free(ms);
}

static void *worker(void *arg) {
    job_t *job = (job_t *)arg;
    const oracle_problem *p = job->p;
    int32_t cap = p->n_cells > p->n_sel ? p->n_cells : p->n_sel;
    if (cap < 1) cap = 1;
    scratch_t s;
    s.cells = (int32_t *)malloc(sizeof(int32_t) * (size_t)cap);
    s.x = (double *)malloc(sizeof(double) * (size_t)cap);
    s.acc = (double *)malloc(sizeof(double) * (size_t)p->head_dim);
    for (;;) {
        int r = atomic_fetch_add(&job->next_row, 1);
        if (r >= p->n_rows) break;
        int32_t nv = visible_cells(p, r, s.cells);
        for (int h = 0; h < p->n_head_q; ++h) {
            double *o = job->out + ((int64_t)r * p->n_head_q + h) * p->head_dim;
            if (job->n_slices > 0) row_head_split(p, r, h, job->n_slices, s.cells, nv, &s, o);
            else row_head_plain(p, r, h, s.cells, nv, &s, o);
        }
    }
    free(s.cells); free(s.x); free(s.acc);
    return NULL;
}

static int validate(const oracle_problem *p) {
    if (!p || !p->q || !p->k || !p->v) return -1;
    if (p->n_rows < 0 || p->n_cells < 0 || p->head_dim <= 0) return -1;
    if (p->n_head_kv <= 0 || p->n_head_q <= 0 || p->n_head_q % p->n_head_kv) return -1;
    if (p->sel && p->n_sel < 0) return -1;
    return 0;
}

static int run(const oracle_problem *p, double *out, int n_threads, int n_slices) {
    if (validate(p)) return -1;
    if (n_threads <= 0) n_threads = n_online_cores();
    if (n_threads > p->n_rows) n_threads = p->n_rows > 0 ? p->n_rows : 1;
    job_t job;
    job.p = p; job.out = out; job.n_slices = n_slices;
    atomic_init(&job.next_row, 0);
    if (n_threads == 1) { worker(&job); return 0; }
    pthread_t *t = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i) pthread_create(&t[i], NULL, worker, &job);
    for (int i = 0; i < n_threads; ++i) pthread_join(t[i], NULL);
    free(t);
    return 0;
}

int oracle_attn(const oracle_problem *p, double *out, int n_threads) {
    return run(p, out, n_threads, 0);
}

int oracle_attn_split(const oracle_problem *p, int n_slices, double *out, int n_threads) {
    if (!p || p->sel || n_slices < 1) return -1;
    return run(p, out, n_threads, n_slices);
}

int oracle_select_compact(const int32_t *sel, int64_t sel_stride_row, int32_t n_rows,
                          int32_t n_sel, int32_t n_cells,
                          int32_t *sorted_out, int32_t *count_out) {
    if (!sel || !sorted_out || !count_out || n_sel < 0 || n_rows < 0) return -1;
    int32_t *tmp = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_sel > 0 ? n_sel : 1));
    for (int32_t r = 0; r < n_rows; ++r) {
        int32_t n = compact_list(sel + (int64_t)r * sel_stride_row, n_sel, n_cells, tmp);
        int32_t *dst = sorted_out + (int64_t)r * n_sel;
        for (int32_t i = 0; i < n_sel; ++i) dst[i] = i < n ? tmp[i] : -1;
        count_out[r] = n;
    }
    free(tmp);
    return 0;
}
