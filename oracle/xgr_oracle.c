/*
 * xgr_oracle.c -- plain, slow, obviously-correct CPU oracle for the xGR
 * beam-decode hot path.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library, and it does not
 * include or call anything from it.
 *
 * Sources (page titles and sections; the pages are summaries, they print no
 * formulas, so each function states the plain definition it follows):
 *   [xGR]  "xGR: Efficient Generative Recommendation Serving at Scale"
 *          2.1 xAttention -- "Separate KV cache" (Shared prompt cache computed
 *              once, Unshared cache of generated tokens), "Token-granular
 *              management", "Staged computation" (Shared, Unshared, Merging by
 *              OnlineSoftmax), "In-place updates" (direct indices, no
 *              write-before-read hazard).
 *          2.2 xBeam -- "Valid-path constraint" (masks from a pre-built
 *              vocabulary of valid items, dense early / sparse later),
 *              "Early sort termination" (global min-heap, a branch stops once
 *              its next log-prob is below the heap minimum).
 *
 * Arithmetic: everything is fp64, except the cumulative-score add of the
 * log-prob selection mode, which is by definition one IEEE fp32
 * round-to-nearest-even add (the selection contract is bit-exact on fp32
 * log-prob inputs).  Build without -ffast-math.
 *
 * Parity pins: see tests/test_oracle_*.py (closed forms, a library special
 * case, brute force on tiny inputs, split+merge invariant, three selection
 * algorithms that must agree, end-to-end enumeration of all items).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_INDEX (-2)   /* an ancestry slot or token outside its range */
#define ORC_ERR_NAN (-3)     /* a NaN score among the candidates */
#define ORC_ERR_ALLOC (-4)

/* bf16 -> fp64, exact: a bf16 is the upper half of an fp32. */
static double bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* Attention: one query row against an explicit list of keys/values.        */
/*   s_j = (q . k_j) * scale,  m = max_j s_j,  l = sum_j exp(s_j - m),      */
/*   O = sum_j exp(s_j - m) v_j / l,  LSE = m + ln l.                       */
/* The full (unsplit) softmax: xGR 2.1 "Staged computation" states that the */
/* Shared/Unshared/Merging stages compute this same attention.              */
/* ------------------------------------------------------------------------ */
static void attend_row(int D, const uint16_t *q, int n, const uint16_t *const *krow,
                       const uint16_t *const *vrow, double scale, double *s,
                       double *out, double *lse)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += bf16(q[d]) * bf16(krow[j][d]);
        s[j] = acc * scale;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) l += exp(s[j] - m);
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        double p = exp(s[j] - m);
        for (int d = 0; d < D; ++d) out[d] += p * bf16(vrow[j][d]);
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
    *lse = m + log(l);
}

/* Contiguous keys: q [n_q][D], k, v [n][D] (bf16 bits); out [n_q][D], lse [n_q]. */
int orc_attend(int n_q, int D, const uint16_t *q, int n, const uint16_t *k,
               const uint16_t *v, double scale, double *out, double *lse)
{
    const uint16_t **kr = malloc(sizeof(*kr) * (size_t)(n > 0 ? n : 1));
    const uint16_t **vr = malloc(sizeof(*vr) * (size_t)(n > 0 ? n : 1));
    double *s = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!kr || !vr || !s) { free(kr); free(vr); free(s); return ORC_ERR_ALLOC; }
    for (int j = 0; j < n; ++j) { kr[j] = k + (size_t)j * D; vr[j] = v + (size_t)j * D; }
    for (int i = 0; i < n_q; ++i)
        attend_row(D, q + (size_t)i * D, n, kr, vr, scale, s, out + (size_t)i * D, lse + i);
    free(kr); free(vr); free(s);
    return ORC_OK;
}

/*
 * Attention of one request at decode step s (xGR 2.1).
 * Key set of live beam b, query head h, kv head g = h / (Hq/Hkv):
 *   the shared prompt  ks[g][0..P)          (computed once at prefill)
 *   the request suffix kx[g][0..X)          (X may be 0)
 *   the beam's own generated tokens, one per step i = 0..s, read token by
 *   token from the Unshared pool at slot anc[b][i] of step i:
 *       kpool[i][anc[b][i]][g]
 * Layouts (bf16 bits): q [BW][Hq][D]; ks, vs [Hkv][P][D]; kx, vx [Hkv][X][D];
 * kpool, vpool [S][BW][Hkv][D]; anc[b * anc_stride + i].
 * Output rows of beams b >= n_live are dead: O = 0, LSE = -inf.
 * beam_ids (optional): compute only these n_ids beams; output row i (and
 * query row i of q) then belongs to beam beam_ids[i].  NULL: all BW beams.
 */
int orc_decode_attention(int BW, int Hq, int Hkv, int D, int s, int n_live,
                         const uint16_t *q,
                         const uint16_t *ks, const uint16_t *vs, int P,
                         const uint16_t *kx, const uint16_t *vx, int X,
                         const uint16_t *kpool, const uint16_t *vpool,
                         const int32_t *anc, int anc_stride,
                         const int32_t *beam_ids, int n_ids,
                         double *out, double *lse)
{
    const int n_beams = beam_ids ? n_ids : BW;
    const int G = Hq / Hkv;
    const double scale = 1.0 / sqrt((double)D);
    const int n = P + X + s + 1;
    int err = ORC_OK;

    for (int bi = 0; bi < n_beams; ++bi) {
        const int b = beam_ids ? beam_ids[bi] : bi;
        if (b < 0 || b >= BW) return ORC_ERR_INDEX;
        if (b >= n_live) continue;
        for (int i = 0; i <= s; ++i) {
            int slot = anc[(size_t)b * anc_stride + i];
            if (slot < 0 || slot >= BW) err = ORC_ERR_INDEX;
        }
    }
    if (err) return err;

#pragma omp parallel
    {
        const uint16_t **kr = malloc(sizeof(*kr) * (size_t)n);
        const uint16_t **vr = malloc(sizeof(*vr) * (size_t)n);
        double *sc = malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 4)
        for (int row = 0; row < n_beams * Hq; ++row) {
            const int bi = row / Hq, h = row % Hq, g = h / G;
            const int b = beam_ids ? beam_ids[bi] : bi;
            double *o = out + (size_t)row * D;
            if (b >= n_live) {
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                lse[row] = -INFINITY;
                continue;
            }
            int j = 0;
            for (int t = 0; t < P; ++t, ++j) {
                kr[j] = ks + ((size_t)g * P + t) * D;
                vr[j] = vs + ((size_t)g * P + t) * D;
            }
            for (int t = 0; t < X; ++t, ++j) {
                kr[j] = kx + ((size_t)g * X + t) * D;
                vr[j] = vx + ((size_t)g * X + t) * D;
            }
            for (int i = 0; i <= s; ++i, ++j) {
                const int slot = anc[(size_t)b * anc_stride + i];
                kr[j] = kpool + (((size_t)i * BW + slot) * Hkv + g) * D;
                vr[j] = vpool + (((size_t)i * BW + slot) * Hkv + g) * D;
            }
            attend_row(D, q + (size_t)row * D, n, kr, vr, scale, sc, o, lse + row);
        }
        free(kr); free(vr); free(sc);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Valid-path masks (xGR 2.2 "Valid-path constraint").                      */
/* The valid next tokens of a prefix p = (t_0..t_{s-1}) are                 */
/*   { item[s] : item[0..s-1] == p },  sorted ascending, without repeats.    */
/* ------------------------------------------------------------------------ */

/* Brute force: scan every item.  out must hold V entries; returns the count. */
int orc_next_tokens_scan(const int32_t *items, int64_t N, int L, int V,
                         const int32_t *prefix, int s, int32_t *out)
{
    uint8_t *flag = calloc((size_t)V, 1);
    if (!flag) return ORC_ERR_ALLOC;
    for (int64_t n = 0; n < N; ++n) {
        const int32_t *it = items + n * L;
        int match = 1;
        for (int i = 0; i < s; ++i)
            if (it[i] != prefix[i]) { match = 0; break; }
        if (match) flag[it[s]] = 1;
    }
    int c = 0;
    for (int t = 0; t < V; ++t)
        if (flag[t]) out[c++] = t;
    free(flag);
    return c;
}

/* lexicographic order of two L-token items */
static int lex_cmp(const int32_t *a, const int32_t *b, int len)
{
    for (int i = 0; i < len; ++i) {
        if (a[i] < b[i]) return -1;
        if (a[i] > b[i]) return 1;
    }
    return 0;
}

static int g_sort_L;
static int item_cmp(const void *x, const void *y)
{
    return lex_cmp((const int32_t *)x, (const int32_t *)y, g_sort_L);
}

/* Sort the item list lexicographically, in place (library qsort). */
void orc_sort_items(int32_t *items, int64_t N, int L)
{
    g_sort_L = L;
    qsort(items, (size_t)N, sizeof(int32_t) * (size_t)L, item_cmp);
}

/* In a lexicographically sorted list the items that start with p form one
 * contiguous range; find it by binary search, then read item[s] along it (the
 * range is sorted by item[s], so repeats are adjacent).  Returns the count. */
int orc_next_tokens_sorted(const int32_t *sorted, int64_t N, int L,
                           const int32_t *prefix, int s, int32_t *out)
{
    int64_t lo = 0, hi = N;              /* first item with item[0..s) >= p */
    while (lo < hi) {
        int64_t mid = lo + (hi - lo) / 2;
        if (lex_cmp(sorted + mid * L, prefix, s) < 0) lo = mid + 1; else hi = mid;
    }
    int64_t end = lo, top = N;           /* first item with item[0..s) > p */
    while (end < top) {
        int64_t mid = end + (top - end) / 2;
        if (lex_cmp(sorted + mid * L, prefix, s) <= 0) end = mid + 1; else top = mid;
    }
    int c = 0;
    for (int64_t n = lo; n < end; ++n) {
        int32_t t = sorted[n * L + s];
        if (c == 0 || out[c - 1] != t) out[c++] = t;
    }
    return c;
}

/* Dense mask of the first step: bit t%32 of word t/32 (LSB first) is set when
 * some item starts with token t.  bits has ceil(V/32) words. */
void orc_mask_dense(const int32_t *items, int64_t N, int L, int V, uint32_t *bits)
{
    memset(bits, 0, sizeof(uint32_t) * (size_t)((V + 31) / 32));
    for (int64_t n = 0; n < N; ++n) {
        int32_t t = items[n * L];
        bits[t >> 5] |= 1u << (t & 31);
    }
}

/* Sparse mask of step s >= 1 for n_rows beams: row r's valid next tokens (of
 * prefix prefixes[r][0..s)) when live[r] != 0, else an empty row.  CSR in row
 * order with row_ptr[0] = 0; cols needs cap entries.  Returns nnz or -1 when
 * cap is too small. */
int64_t orc_mask_csr(const int32_t *sorted, int64_t N, int L, int V, int s, int n_rows,
                     const int32_t *prefixes, int prefix_stride, const uint8_t *live,
                     int64_t *row_ptr, int32_t *cols, int64_t cap)
{
    int32_t *buf = malloc(sizeof(int32_t) * (size_t)V);
    if (!buf) return -1;
    row_ptr[0] = 0;
    for (int r = 0; r < n_rows; ++r) {
        int c = 0;
        if (live[r]) c = orc_next_tokens_sorted(sorted, N, L, prefixes + (size_t)r * prefix_stride, s, buf);
        if (row_ptr[r] + c > cap) { free(buf); return -1; }
        memcpy(cols + row_ptr[r], buf, sizeof(int32_t) * (size_t)c);
        row_ptr[r + 1] = row_ptr[r] + c;
    }
    free(buf);
    return row_ptr[n_rows];
}

/* ------------------------------------------------------------------------ */
/* Beam selection (xGR 2.2; readings: candidates are (live beam b, valid     */
/* token t), score = cum[b] + logprob[b][t]; keep the best BW under the      */
/* total order  higher score first, then lower parent b, then lower t).      */
/* ------------------------------------------------------------------------ */

typedef struct { float key; int32_t b, t; } cand32;
typedef struct { double key; int32_t b, t; } cand64;

/* total order: negative when x ranks before y */
static int rank32(const cand32 *x, const cand32 *y)
{
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    if (x->b != y->b) return x->b < y->b ? -1 : 1;
    if (x->t != y->t) return x->t < y->t ? -1 : 1;
    return 0;
}
static int cmp32(const void *x, const void *y) { return rank32(x, y); }

static int cmp64(const void *px, const void *py)
{
    const cand64 *x = px, *y = py;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    if (x->b != y->b) return x->b < y->b ? -1 : 1;
    if (x->t != y->t) return x->t < y->t ? -1 : 1;
    return 0;
}

/* The fp32 score of the log-prob mode: one fp32 add; -0.0 is written as +0.0
 * (IEEE compares them equal, so the tie-break decides, and the stored value
 * is canonical). */
static float score32(float cum, float lp)
{
    float k = cum + lp;
    if (k == 0.0f) k = 0.0f;
    return k;
}

/* binary min-heap on the total order whose root is the WORST kept candidate */
static void heap_down(cand32 *h, int n, int i)
{
    for (;;) {
        int l = 2 * i + 1, r = l + 1, w = i;
        if (l < n && rank32(&h[l], &h[w]) > 0) w = l;
        if (r < n && rank32(&h[r], &h[w]) > 0) w = r;
        if (w == i) return;
        cand32 tmp = h[i]; h[i] = h[w]; h[w] = tmp;
        i = w;
    }
}
static void heap_up(cand32 *h, int i)
{
    while (i > 0) {
        int p = (i - 1) / 2;
        if (rank32(&h[i], &h[p]) <= 0) return;
        cand32 tmp = h[i]; h[i] = h[p]; h[p] = tmp;
        i = p;
    }
}

/*
 * Log-prob mode.  lp [BW][V] fp32; cum [BW] fp32; the valid tokens of live
 * beam b are cols[row_ptr[b]..row_ptr[b+1]) (for the dense first step the
 * caller passes the set bits as one CSR row).  method:
 *   0  flat definition: sort every candidate, keep the first BW;
 *   1  two stages: each beam keeps its top-K, then the union is cut to BW;
 *   2  the page's early-terminating form: each beam's candidates in sorted
 *      order feed one global min-heap of size BW whose root is the worst kept
 *      candidate; a beam stops at its first candidate that does not beat the
 *      root (all later ones of that beam are worse).
 * Outputs (rank order, slot = rank): parent, token, cum_out [BW]; slots past
 * the number of candidates get -1, -1, -inf.  Returns n_out or an error.
 */
int orc_select_logprob(int BW, int K, int V, int n_live, const float *cum, const float *lp,
                       const int64_t *row_ptr, const int32_t *cols, int method,
                       int32_t *parent, int32_t *token, float *cum_out)
{
    int64_t total = 0;
    for (int b = 0; b < n_live; ++b) total += row_ptr[b + 1] - row_ptr[b];
    cand32 *all = malloc(sizeof(cand32) * (size_t)(total > 0 ? total : 1));
    if (!all) return ORC_ERR_ALLOC;
    int64_t c = 0;
    for (int b = 0; b < n_live; ++b)
        for (int64_t e = row_ptr[b]; e < row_ptr[b + 1]; ++e) {
            int32_t t = cols[e];
            if (t < 0 || t >= V) { free(all); return ORC_ERR_INDEX; }
            float x = lp[(size_t)b * V + t];
            if (isnan(x) || isnan(cum[b])) { free(all); return ORC_ERR_NAN; }
            all[c].key = score32(cum[b], x);
            all[c].b = b;
            all[c].t = t;
            ++c;
        }

    cand32 *best = NULL;
    int64_t n_best = 0;
    if (method == 0) {
        qsort(all, (size_t)total, sizeof(cand32), cmp32);
        best = all;
        n_best = total < BW ? total : BW;
    } else if (method == 1) {
        cand32 *kept = malloc(sizeof(cand32) * (size_t)(total > 0 ? total : 1));
        if (!kept) { free(all); return ORC_ERR_ALLOC; }
        int64_t nk = 0, off = 0;
        for (int b = 0; b < n_live; ++b) {
            int64_t nb = row_ptr[b + 1] - row_ptr[b];
            qsort(all + off, (size_t)nb, sizeof(cand32), cmp32);
            int64_t keep = nb < K ? nb : K;
            memcpy(kept + nk, all + off, sizeof(cand32) * (size_t)keep);
            nk += keep;
            off += nb;
        }
        qsort(kept, (size_t)nk, sizeof(cand32), cmp32);
        memcpy(all, kept, sizeof(cand32) * (size_t)nk);
        free(kept);
        best = all;
        n_best = nk < BW ? nk : BW;
    } else {
        cand32 *heap = malloc(sizeof(cand32) * (size_t)(BW > 0 ? BW : 1));
        if (!heap) { free(all); return ORC_ERR_ALLOC; }
        int hn = 0;
        int64_t off = 0;
        for (int b = 0; b < n_live; ++b) {
            int64_t nb = row_ptr[b + 1] - row_ptr[b];
            qsort(all + off, (size_t)nb, sizeof(cand32), cmp32);   /* beam's list, best first */
            for (int64_t e = 0; e < nb; ++e) {
                cand32 *x = all + off + e;
                if (hn < BW) {
                    heap[hn] = *x;
                    heap_up(heap, hn);
                    ++hn;
                } else if (rank32(x, &heap[0]) < 0) {
                    heap[0] = *x;
                    heap_down(heap, hn, 0);
                } else {
                    break;   /* early termination of this branch */
                }
            }
            off += nb;
        }
        qsort(heap, (size_t)hn, sizeof(cand32), cmp32);
        memcpy(all, heap, sizeof(cand32) * (size_t)hn);
        free(heap);
        best = all;
        n_best = hn;
    }
    for (int i = 0; i < BW; ++i) {
        if (i < n_best) {
            parent[i] = best[i].b;
            token[i] = best[i].t;
            cum_out[i] = best[i].key;
        } else {
            parent[i] = -1;
            token[i] = -1;
            cum_out[i] = -INFINITY;
        }
    }
    free(all);
    return (int)n_best;
}

/*
 * Logits mode, fp64 throughout: lp[b][t] = logits[b][t] - ln sum_u exp(logits[b][u])
 * over the FULL vocabulary (masking comes after normalisation), score =
 * cum[b] + lp[b][t] with cum the fp64 path sum; flat sort, keep BW.
 * lse_out [BW] receives the row log-sum-exp of every live row.
 */
int orc_select_logits(int BW, int V, int n_live, const double *cum, const float *logits,
                      const int64_t *row_ptr, const int32_t *cols,
                      int32_t *parent, int32_t *token, double *cum_out, double *lse_out)
{
    int64_t total = 0;
    for (int b = 0; b < n_live; ++b) total += row_ptr[b + 1] - row_ptr[b];
    cand64 *all = malloc(sizeof(cand64) * (size_t)(total > 0 ? total : 1));
    if (!all) return ORC_ERR_ALLOC;
    int64_t c = 0;
    for (int b = 0; b < n_live; ++b) {
        const float *x = logits + (size_t)b * V;
        double m = -INFINITY;
        for (int t = 0; t < V; ++t) {
            if (isnan(x[t])) { free(all); return ORC_ERR_NAN; }
            if ((double)x[t] > m) m = x[t];
        }
        double l = 0.0;
        for (int t = 0; t < V; ++t) l += exp((double)x[t] - m);
        double lse = m + log(l);
        lse_out[b] = lse;
        for (int64_t e = row_ptr[b]; e < row_ptr[b + 1]; ++e) {
            int32_t t = cols[e];
            if (t < 0 || t >= V) { free(all); return ORC_ERR_INDEX; }
            all[c].key = cum[b] + ((double)x[t] - lse);
            all[c].b = b;
            all[c].t = t;
            ++c;
        }
    }
    qsort(all, (size_t)total, sizeof(cand64), cmp64);
    int64_t n_best = total < BW ? total : BW;
    for (int i = 0; i < BW; ++i) {
        if (i < n_best) {
            parent[i] = all[i].b;
            token[i] = all[i].t;
            cum_out[i] = all[i].key;
        } else {
            parent[i] = -1;
            token[i] = -1;
            cum_out[i] = -INFINITY;
        }
    }
    free(all);
    return (int)n_best;
}
