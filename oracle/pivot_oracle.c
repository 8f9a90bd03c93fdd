/*
 * PIVOT query-group indexer -- CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * statement of what the indexer computes.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline / reference legs may load it.  It shares
 * no code, header, table or helper with the CUDA library, and the CUDA
 * library never calls it.
 *
 * Source: "PIVOT: Efficient Query-Group Indexing for Token-Level Sparse
 * Attention" (arXiv 2607.24593) as described on the pages "PIVOT explained --
 * from paper to working code in 10 minutes" (sections "How It Works" and
 * "Show Me The Code") and the paper's abstract.  All arithmetic is fp64 on
 * the bf16 input values (decoded exactly); selection is a full sort.
 *
 * Readings of the pages taken here (the pages are silent or disagree):
 *  - Groups: g consecutive queries starting at 0, g, 2g, ...; the last group
 *    may be partial and its proxy is the mean over its actual members
 *    ("Show Me The Code", the g_start/g_end loop).
 *  - Proxy: the mean of the members' queries, accumulated in fp64 in member
 *    order (exact for bf16 inputs of ordinary range), divided by the member
 *    count in fp64 and rounded to fp32 (round to nearest even): the fp32 mean
 *    is the scan operand.  Option proxy_bf16 rounds that mean once more, to
 *    bf16, and scans with the bf16 value instead (what a scan that feeds the
 *    mean to the tensor cores as a single bf16 operand computes).
 *  - Causality: a query at position pos sees keys j < pos (the listing scans
 *    k_h[:pos]).
 *  - Refine: ONE proxy scan per group over j < last, last = the largest
 *    member position (the sketch's "ONE scan instead of g scans" together
 *    with the listing's per-member prefix), candidate set C = top-min(Kc,last)
 *    of the proxy scores; member pos keeps V = {j in C : j < pos}, re-scores V
 *    with its own query and keeps top-min(top_k, |V|).
 *  - The listing's own Refine (mode 2, kept to measure the difference the
 *    reading above makes): every member re-runs the proxy scan over its own
 *    prefix j < pos, takes C_pos = top-min(Kc, pos) of it, re-scores C_pos
 *    with its own query and keeps top-min(top_k, |C_pos|) ("Show Me The
 *    Code", pivot_refine: the scan k_h[:pos] inside the member loop).
 *  - Reuse: the proxy's top-min(top_k, s) over keys j < s (s = group start,
 *    strictly causal for every member; group 0 gets nothing), shared by all
 *    members.
 *  - Dense: per query, top-min(top_k, pos) of q_pos . k_j over j < pos
 *    (the indexer that PIVOT replaces, section "The Problem").
 *  - Ties break toward the lower key index; an output row is the selected
 *    index set in ascending index order, padded with -1.
 *  - Scores are the unscaled dot products q . k (the 1/sqrt(D) factor of the
 *    demo belongs to the downstream attention only).
 *  - Decode: one group per sequence = the g queries of one multi-token
 *    prediction step at positions n_b .. n_b+g-1; the sequence's cache holds
 *    n_b + g keys (abstract: "the queries decoded together in one MTP step").
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    double s;   /* score */
    int32_t j;  /* key index */
} scored_t;

static double bf16_val(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp32 -> bf16, round to nearest, ties to even (finite inputs). */
static uint16_t bf16_round(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/* Order of the selection: larger score first, then lower index. */
static int by_score_then_index(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int by_index(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static double dot(const uint16_t *a, const uint16_t *b, int d)
{
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += bf16_val(a[c]) * bf16_val(b[c]);
    return acc;
}

/* Proxy query: mean of the n member rows (see the reading above).  p
 * receives the scan operand (the fp32 mean, or its bf16 rounding when
 * proxy_bf16), p32 / pb (nullable) the fp32 mean and its bf16 rounding. */
static void proxy_of(const uint16_t *const *rows, int n, int d, int proxy_bf16,
                     double *p, float *p32, uint16_t *pb)
{
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int m = 0; m < n; ++m) acc += bf16_val(rows[m][c]);
        float mean = (float)(acc / (double)n);
        uint16_t b = bf16_round(mean);
        p[c] = proxy_bf16 ? bf16_val(b) : (double)mean;
        if (p32) p32[c] = mean;
        if (pb) pb[c] = b;
    }
}

/* Scan score of the proxy against one key row. */
static double proxy_dot(const double *p, const uint16_t *k, int d)
{
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += p[c] * bf16_val(k[c]);
    return acc;
}

/*
 * Keep the K best of v[0..n) (score desc, index asc), write them in ascending
 * index order to idx/sc (padded to width with -1 / NaN), and the scores of
 * ranks K and K+1 to edge (NaN where that rank does not exist).  v is
 * reordered.  Returns K.
 */
static int select_top(scored_t *v, int n, int K, int width, int32_t *idx, double *sc, double *edge)
{
    if (K > n) K = n;
    if (K < 0) K = 0;
    qsort(v, (size_t)n, sizeof *v, by_score_then_index);
    if (edge) {
        edge[0] = (K >= 1) ? v[K - 1].s : NAN;
        edge[1] = (n > K && K >= 1) ? v[K].s : NAN;
    }
    qsort(v, (size_t)K, sizeof *v, by_index);
    for (int t = 0; t < width; ++t) {
        if (idx) idx[t] = (t < K) ? v[t].j : -1;
        if (sc) sc[t] = (t < K) ? v[t].s : NAN;
    }
    return K;
}

/*
 * One group.  mq[m] = query row of member m (m < nm), mpos[m] its position;
 * key j is at kbase + j*kstride.  s = first member position (Reuse bound),
 * last = largest member position (Refine scan bound).  Output rows for
 * members m < g (rows m >= nm are padding: -1).
 */
static int one_group(const uint16_t *const *mq, const int32_t *mpos, int nm, int g,
                     const uint16_t *kbase, long kstride, int d, int s, int last,
                     int top_k, int Kc, int mode, int proxy_bf16,
                     int32_t *out, double *out_sc, double *edge,
                     int32_t *cand, double *cand_edge, float *proxy32, uint16_t *proxyb,
                     double *mcand_edge)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)d);
    int bound = (mode == 1) ? s : last;
    scored_t *sig = (scored_t *)malloc(sizeof(scored_t) * (size_t)(bound > 0 ? bound : 1));
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)(Kc > 0 ? Kc : 1));
    if (!p || !sig || !v) { free(p); free(sig); free(v); return -1; }

    proxy_of(mq, nm, d, proxy_bf16, p, proxy32, proxyb);
    for (int j = 0; j < bound; ++j) {
        sig[j].s = proxy_dot(p, kbase + (long)j * kstride, d);
        sig[j].j = j;
    }

    for (int m = 0; m < g; ++m) {
        for (int t = 0; t < top_k; ++t) {
            out[(long)m * top_k + t] = -1;
            if (out_sc) out_sc[(long)m * top_k + t] = NAN;
        }
        if (edge) { edge[2 * m] = NAN; edge[2 * m + 1] = NAN; }
    }
    if (cand) for (int t = 0; t < Kc; ++t) cand[t] = -1;
    if (cand_edge) { cand_edge[0] = NAN; cand_edge[1] = NAN; }
    if (mcand_edge) for (int m = 0; m < 2 * g; ++m) mcand_edge[m] = NAN;

    if (mode == 1) {
        /* Reuse: the proxy's top-k over j < s, shared by every member. */
        int32_t *row = (int32_t *)malloc(sizeof(int32_t) * (size_t)top_k);
        double *rsc = (double *)malloc(sizeof(double) * (size_t)top_k);
        double e2[2];
        select_top(sig, bound, top_k, top_k, row, rsc, e2);
        for (int m = 0; m < nm; ++m) {
            memcpy(out + (long)m * top_k, row, sizeof(int32_t) * (size_t)top_k);
            if (out_sc) memcpy(out_sc + (long)m * top_k, rsc, sizeof(double) * (size_t)top_k);
            if (edge) { edge[2 * m] = e2[0]; edge[2 * m + 1] = e2[1]; }
        }
        free(row); free(rsc);
    } else if (mode == 2) {
        /* The listing's Refine: a proxy scan over each member's own prefix. */
        scored_t *own = (scored_t *)malloc(sizeof(scored_t) * (size_t)(bound > 0 ? bound : 1));
        int32_t *C = (int32_t *)malloc(sizeof(int32_t) * (size_t)(Kc > 0 ? Kc : 1));
        for (int m = 0; m < nm; ++m) {
            int pos = mpos[m];
            memcpy(own, sig, sizeof(scored_t) * (size_t)pos);
            int nC = select_top(own, pos, Kc, Kc, C, NULL, mcand_edge ? mcand_edge + 2 * m : NULL);
            for (int t = 0; t < nC; ++t) {
                v[t].j = C[t];
                v[t].s = dot(mq[m], kbase + (long)C[t] * kstride, d);
            }
            select_top(v, nC, top_k, top_k, out + (long)m * top_k,
                       out_sc ? out_sc + (long)m * top_k : NULL, edge ? edge + 2 * m : NULL);
        }
        free(own); free(C);
    } else {
        /* Refine: candidate set from the one proxy scan, then per-member re-score. */
        int32_t *C = (int32_t *)malloc(sizeof(int32_t) * (size_t)(Kc > 0 ? Kc : 1));
        int nC = select_top(sig, bound, Kc, Kc, C, NULL, cand_edge);
        if (cand) memcpy(cand, C, sizeof(int32_t) * (size_t)Kc);
        for (int m = 0; m < nm; ++m) {
            int nv = 0;
            for (int t = 0; t < nC; ++t) {
                if (C[t] < mpos[m]) {
                    v[nv].j = C[t];
                    v[nv].s = dot(mq[m], kbase + (long)C[t] * kstride, d);
                    ++nv;
                }
            }
            select_top(v, nv, top_k, top_k, out + (long)m * top_k,
                       out_sc ? out_sc + (long)m * top_k : NULL, edge ? edge + 2 * m : NULL);
        }
        free(C);
    }
    free(p); free(sig); free(v);
    return 0;
}

/*
 * Prefill PIVOT for a list of (group, head) units.
 * q, k: bf16 bits [L, H, d].  mode 0 = Refine, 1 = Reuse, 2 = the listing's
 * per-member-scan Refine (cand / cand_edge are not written in mode 2).
 * proxy_bf16 = 0: scan with the fp32 mean (the method); 1: with its bf16
 * rounding (the variant).
 * Per unit u: out [g, top_k] (member m = position i*g + m), out_sc [g, top_k]
 * (nullable), edge [g, 2] (nullable), cand [Kc] (nullable), cand_edge [2]
 * (nullable), proxy32 [d] fp32 mean (nullable), proxyb [d] its bf16 rounding
 * (nullable), mcand_edge [g, 2] (nullable; mode 2 only): each member's own
 * Kc-th and (Kc+1)-th proxy scores over its prefix.  Returns 0, or -1 on bad
 * arguments.
 */
int oracle_prefill_units(const uint16_t *q, const uint16_t *k, int L, int H, int d,
                         int g, int top_k, int Kc, int mode, int proxy_bf16,
                         int n_units, const int32_t *unit_group, const int32_t *unit_head,
                         int32_t *out, double *out_sc, double *edge,
                         int32_t *cand, double *cand_edge, float *proxy32, uint16_t *proxyb,
                         double *mcand_edge)
{
    if (L < 1 || H < 1 || d < 1 || g < 1 || top_k < 1 || Kc < top_k || mode < 0 || mode > 2 ||
        proxy_bf16 < 0 || proxy_bf16 > 1)
        return -1;
    int G = (L + g - 1) / g;
    const uint16_t **mq = (const uint16_t **)malloc(sizeof(*mq) * (size_t)g);
    int32_t *mpos = (int32_t *)malloc(sizeof(int32_t) * (size_t)g);
    int rc = 0;
    for (int u = 0; u < n_units && rc == 0; ++u) {
        int i = unit_group[u], h = unit_head[u];
        if (i < 0 || i >= G || h < 0 || h >= H) { rc = -1; break; }
        int s = i * g, e = s + g < L ? s + g : L, nm = e - s;
        for (int m = 0; m < nm; ++m) {
            mq[m] = q + ((long)(s + m) * H + h) * d;
            mpos[m] = s + m;
        }
        rc = one_group(mq, mpos, nm, g, k + (long)h * d, (long)H * d, d, s, e - 1,
                       top_k, Kc, mode, proxy_bf16,
                       out + (long)u * g * top_k,
                       out_sc ? out_sc + (long)u * g * top_k : NULL,
                       edge ? edge + (long)u * g * 2 : NULL,
                       cand ? cand + (long)u * Kc : NULL,
                       cand_edge ? cand_edge + (long)u * 2 : NULL,
                       proxy32 ? proxy32 + (long)u * d : NULL,
                       proxyb ? proxyb + (long)u * d : NULL,
                       mcand_edge ? mcand_edge + (long)u * g * 2 : NULL);
    }
    free(mq); free(mpos);
    return rc;
}

/*
 * Dense indexer for a list of (position, head) units: top-min(top_k, pos) of
 * q_pos . k_j over j < pos.  out [n_units, top_k], out_sc/edge nullable.
 */
int oracle_dense_units(const uint16_t *q, const uint16_t *k, int L, int H, int d, int top_k,
                       int n_units, const int32_t *unit_pos, const int32_t *unit_head,
                       int32_t *out, double *out_sc, double *edge)
{
    if (L < 1 || H < 1 || d < 1 || top_k < 1) return -1;
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)L);
    if (!v) return -1;
    for (int u = 0; u < n_units; ++u) {
        int pos = unit_pos[u], h = unit_head[u];
        if (pos < 0 || pos >= L || h < 0 || h >= H) { free(v); return -1; }
        const uint16_t *qp = q + ((long)pos * H + h) * d;
        for (int j = 0; j < pos; ++j) {
            v[j].s = dot(qp, k + ((long)j * H + h) * d, d);
            v[j].j = j;
        }
        select_top(v, pos, top_k, top_k, out + (long)u * top_k,
                   out_sc ? out_sc + (long)u * top_k : NULL, edge ? edge + 2L * u : NULL);
    }
    free(v);
    return 0;
}

/*
 * Decode PIVOT for a list of (sequence, head) units (modes and proxy_bf16 as
 * in oracle_prefill_units).
 * q: bf16 bits [B, g, H, d]; kcache: bf16 bits [cu[B], H, d]; sequence b's
 * keys are cache rows cu[b] .. cu[b+1]-1 and it holds n_b + g of them, so
 * n_b = cu[b+1] - cu[b] - g.  Member i sits at position n_b + i.
 * Outputs per unit as in oracle_prefill_units.
 */
int oracle_decode_units(const uint16_t *q, const uint16_t *kcache, const int32_t *cu,
                        int B, int H, int d, int g, int top_k, int Kc, int mode, int proxy_bf16,
                        int n_units, const int32_t *unit_seq, const int32_t *unit_head,
                        int32_t *out, double *out_sc, double *edge,
                        int32_t *cand, double *cand_edge, float *proxy32, uint16_t *proxyb)
{
    if (B < 1 || H < 1 || d < 1 || g < 1 || top_k < 1 || Kc < top_k || mode < 0 || mode > 2 ||
        proxy_bf16 < 0 || proxy_bf16 > 1)
        return -1;
    const uint16_t **mq = (const uint16_t **)malloc(sizeof(*mq) * (size_t)g);
    int32_t *mpos = (int32_t *)malloc(sizeof(int32_t) * (size_t)g);
    int rc = 0;
    for (int u = 0; u < n_units && rc == 0; ++u) {
        int b = unit_seq[u], h = unit_head[u];
        if (b < 0 || b >= B || h < 0 || h >= H) { rc = -1; break; }
        int n_b = cu[b + 1] - cu[b] - g;
        if (n_b < 0) { rc = -1; break; }
        for (int m = 0; m < g; ++m) {
            mq[m] = q + (((long)b * g + m) * H + h) * d;
            mpos[m] = n_b + m;
        }
        rc = one_group(mq, mpos, g, g, kcache + ((long)cu[b] * H + h) * d, (long)H * d, d,
                       n_b, n_b + g - 1, top_k, Kc, mode, proxy_bf16,
                       out + (long)u * g * top_k,
                       out_sc ? out_sc + (long)u * g * top_k : NULL,
                       edge ? edge + (long)u * g * 2 : NULL,
                       cand ? cand + (long)u * Kc : NULL,
                       cand_edge ? cand_edge + (long)u * 2 : NULL,
                       proxy32 ? proxy32 + (long)u * d : NULL,
                       proxyb ? proxyb + (long)u * d : NULL, NULL);
    }
    free(mq); free(mpos);
    return rc;
}

/*
 * The sparse attention that consumes the index rows ("Show Me The Code", the
 * demo after pivot_refine): for query row r and head h, with the valid
 * indices J of its row (entries >= 0; -1 is padding),
 *     s_j = (q . k_j) * d^-1/2,   w = softmax(s) over J,   out = sum_j w_j v_j,
 * all in fp64 on the bf16 inputs.  A row without a valid index (position 0)
 * gets zeros, as the demo leaves out[0].  Prefill (cu == NULL): q, k, v are
 * [R, H, d] and index j is key row j.  Decode (cu != NULL): q is [R, H, d]
 * with R = B*g (row r is member r % g of sequence r / g), k and v are the
 * packed cache [rows, H, d] and index j of sequence b is cache row cu[b] + j.
 * idx [R, H, top_k] int32; out [R, H, d] fp64.  Returns 0, or -1 on bad
 * arguments.
 */
int oracle_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *idx,
                            const int32_t *cu, int R, int H, int d, int g, int top_k, double *out)
{
    if (R < 1 || H < 1 || d < 1 || top_k < 1 || (cu && g < 1)) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)top_k);
    if (!s) return -1;
    const double scale = 1.0 / sqrt((double)d);
    for (int r = 0; r < R; ++r) {
        long base = cu ? (long)cu[r / g] : 0;
        for (int h = 0; h < H; ++h) {
            const int32_t *row = idx + ((long)r * H + h) * top_k;
            const uint16_t *qr = q + ((long)r * H + h) * d;
            double *o = out + ((long)r * H + h) * d;
            double m = -INFINITY;
            int any = 0;
            for (int t = 0; t < top_k; ++t) {
                if (row[t] < 0) continue;
                s[t] = dot(qr, k + ((base + row[t]) * H + h) * (long)d, d) * scale;
                if (s[t] > m) m = s[t];
                any = 1;
            }
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            if (!any) continue;
            double z = 0.0;
            for (int t = 0; t < top_k; ++t) {
                if (row[t] < 0) continue;
                double w = exp(s[t] - m);
                z += w;
                const uint16_t *vr = v + ((base + row[t]) * H + h) * (long)d;
                for (int c = 0; c < d; ++c) o[c] += w * bf16_val(vr[c]);
            }
            for (int c = 0; c < d; ++c) o[c] /= z;
        }
    }
    free(s);
    return 0;
}
