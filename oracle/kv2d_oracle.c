/*
 * kv2d_oracle.c -- plain, slow, fp64 CPU oracle for MosaicKV-style dynamic
 * two-dimensional KV-cache compression and decode attention over the
 * compressed segments.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Sources followed (page title, section / figure):
 *   [MosaicKV] "MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
 *       Compression" (pith.science summary of arXiv 2607.00760):
 *       Core claim -- importance is identified per element of every KV vector
 *       and a compression strategy is chosen per KV-cache segment;
 *       Fig. 5 -- segment partitioning and compression-strategy generation;
 *       Fig. 6 -- Stage-1 keeps the top important elements of each KV vector,
 *       packed KV format, flexible KV encoding, packed sparse attention;
 *       Fig. 7 / Sec. 5.3 -- PackedAttention computes attention directly on
 *       the packed compressed segments during decode.
 *   [Kara] "KARA: Efficient Reasoning LLM Serving via Sliding-Window KV Cache
 *       Compression" (pith.science review of arXiv 2607.01237):
 *       "What carries the argument" -- token importance is the attention
 *       accumulated from all queries of a recent observation window;
 *       periodic compression of the trailing region every fixed number of
 *       decode steps.
 *
 * The pages give no formulas for the scores, the error proxy, the selection
 * rule or the byte layout.  Every reading taken where they are silent is
 * stated at the function that implements it.  Floating point is fp64
 * throughout; every sum runs sequentially in the order written, and the file
 * is compiled with -ffp-contract=off so that no multiply-add is fused.
 *
 * Parity status: every function here is pinned by tests that do not call
 * this file's own arithmetic twice (closed forms, invariants, brute force
 * and special cases that reduce to textbook attention).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t d;       /* head dimension                                   */
    int32_t G;       /* query heads per KV head                          */
    int32_t S;       /* segment length (tokens)                          */
    int32_t W;       /* observation-window queries                       */
    int32_t r;       /* tokens kept by TOK / BOTH                        */
    int32_t c;       /* channels kept per key vector by CH / BOTH        */
    double beta;     /* byte budget as a fraction of the FULL bytes      */
    double scale;    /* softmax scale                                    */
    int32_t chunk_len;     /* Token2Chunk: longest chunk (tokens); 0 = off */
    int32_t chunk_budget;  /* Token2Chunk: tokens chunks may add per segment */
} orc_params;

enum { ORC_FULL = 0, ORC_TOK = 1, ORC_CH = 2, ORC_BOTH = 3 };
enum { ORC_OK = 0, ORC_INFEASIBLE = 2 };

/* ---------------------------------------------------------------- fp16 */

/* IEEE binary16 bit pattern -> exact double. */
double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = (m == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* ------------------------------------------------------ step 1: a_d */

/* Element-importance weights of one (sequence, KV head) unit:
 * a[d] = mean over the G*W window query rows of |q[row][d]|
 * ([MosaicKV] Core claim: importance of each element of a KV vector; the
 * mean is taken over the window queries of all G query heads that share the
 * KV head, so there is one a per KV head). */
void orc_win_stats(const orc_params* p, const double* qw, double* a)
{
    int rows = p->G * p->W;
    for (int k = 0; k < p->d; ++k) {
        double acc = 0.0;
        for (int row = 0; row < rows; ++row)
            acc += fabs(qw[(int64_t)row * p->d + k]);
        a[k] = acc / (double)rows;
    }
}

/* -------------------------------------------- steps 2-3: lse and s_t */

/* Token importance from the observation window ([Kara] "What carries the
 * argument": attention accumulated from all queries of the window).
 * The region holds keys r0..T-1 (K has T-r0 rows).  Window row
 * rho = g*W + i is the query at position p_i = T-W+i and sees the keys
 * r0 <= t <= p_i (causal).  Readings: the softmax of a row is normalised
 * over the scored region only (keys already compressed are no longer dense);
 * s_t is the SUM over rows of the softmax weight given to key t.
 *   l[rho][t] = scale * q_rho . k_t
 *   lse[rho]  = log sum_{t=r0}^{p_i} exp(l[rho][t])
 *   s[t]      = sum_{rho : t <= p_i} exp(l[rho][t] - lse[rho])
 * Returns 0, or -1 when W exceeds the region. */
int orc_score(const orc_params* p, int T, int r0, const double* K,
              const double* qw, double* lse, double* s)
{
    int n = T - r0;
    if (p->W > n || p->W <= 0) return -1;
    double* l = (double*)malloc(sizeof(double) * (size_t)n);
    if (!l) return -1;
    for (int t = 0; t < n; ++t) s[t] = 0.0;
    for (int g = 0; g < p->G; ++g) {
        for (int i = 0; i < p->W; ++i) {
            int row = g * p->W + i;
            int last = T - p->W + i;          /* p_i, absolute position  */
            int nvis = last - r0 + 1;         /* keys r0..p_i            */
            const double* q = qw + (int64_t)row * p->d;
            double mx = -INFINITY;
            for (int t = 0; t < nvis; ++t) {
                const double* k = K + (int64_t)t * p->d;
                double dot = 0.0;
                for (int x = 0; x < p->d; ++x) dot += q[x] * k[x];
                l[t] = p->scale * dot;
                if (l[t] > mx) mx = l[t];
            }
            double sum = 0.0;
            for (int t = 0; t < nvis; ++t) sum += exp(l[t] - mx);
            double lz = mx + log(sum);
            lse[row] = lz;
            for (int t = 0; t < nvis; ++t) s[t] += exp(l[t] - lz);
        }
    }
    free(l);
    return 0;
}

/* ---------------------------------------- step 4: channel top-c, g_t */

/* Per-key-vector channel selection ([MosaicKV] Fig. 6, Stage-1: keep the top
 * important elements of each vector; applied to key vectors, values of kept
 * tokens stay whole).  e[t][x] = |K[t][x]| * a[x].  C_t = the c channels of
 * largest e, ties to the lower channel, written ascending.  g[t] is the
 * share of the row's element importance that the dropped channels carry:
 *   g = (sum_{x not in C_t} e) / (sum_x e), both sums ascending in x,
 *   g = 0 when the denominator is 0.
 * The SVD rotation of Fig. 6 is not applied. */
void orc_channel(const orc_params* p, int n, const double* K, const double* a,
                 uint8_t* cidx, double* g)
{
    int d = p->d, c = p->c;
    double* e = (double*)malloc(sizeof(double) * (size_t)d);
    unsigned char* sel = (unsigned char*)malloc((size_t)d);
    for (int t = 0; t < n; ++t) {
        const double* k = K + (int64_t)t * d;
        for (int x = 0; x < d; ++x) { e[x] = fabs(k[x]) * a[x]; sel[x] = 0; }
        /* c rounds of "take the largest remaining, lowest index on ties". */
        for (int j = 0; j < c; ++j) {
            int best = -1;
            for (int x = 0; x < d; ++x) {
                if (sel[x]) continue;
                if (best < 0 || e[x] > e[best]) best = x;
            }
            sel[best] = 1;
        }
        int w = 0;
        for (int x = 0; x < d; ++x)
            if (sel[x]) cidx[(int64_t)t * c + w++] = (uint8_t)x;
        double tot = 0.0, drop = 0.0;
        for (int x = 0; x < d; ++x) {
            tot += e[x];
            if (!sel[x]) drop += e[x];
        }
        g[t] = (tot > 0.0) ? drop / tot : 0.0;
    }
    free(e);
    free(sel);
}

/* ------------------------------------- step 5: top-r and error proxy */

/* R_j: the r tokens of one segment with the largest s, ties to the lower
 * token, written ascending as segment-relative indices. */
void orc_topr(const orc_params* p, const double* s_seg, uint8_t* tidx)
{
    int S = p->S, r = p->r;
    unsigned char* sel = (unsigned char*)calloc((size_t)S, 1);
    for (int j = 0; j < r; ++j) {
        int best = -1;
        for (int t = 0; t < S; ++t) {
            if (sel[t]) continue;
            if (best < 0 || s_seg[t] > s_seg[best]) best = t;
        }
        sel[best] = 1;
    }
    int w = 0;
    for (int t = 0; t < S; ++t)
        if (sel[t]) tidx[w++] = (uint8_t)t;
    free(sel);
}

/* Token2Chunk variant of R_j ([Kara] "What carries the argument": high-score
 * tokens are endpoints of candidate flexible chunks, the best kept under a
 * length cap and a budget; free parameters: max chunk length gamma and
 * chunk budget alpha).  The page gives no equations; the reading taken
 * keeps exactly r tokens (so the TOK / BOTH byte layout does not change):
 *   1. core: the r - alpha tokens with the largest s, ties to the lower t;
 *   2. candidates: every gap between consecutive core positions a < b with
 *      b - a - 1 >= 1 and b - a + 1 <= gamma; its merit is the sum of s over
 *      the gap (fp64, ascending t);
 *   3. candidates by (merit desc, a asc) are filled while their gap fits the
 *      remaining budget (a gap that does not fit is skipped);
 *   4. budget left over goes to the best tokens not yet kept, by (s desc,
 *      t asc).
 * Written ascending as segment-relative indices. */
void orc_topr_chunks(const orc_params* p, const double* s_seg, uint8_t* tidx)
{
    int S = p->S, r = p->r, a = p->chunk_budget, gamma = p->chunk_len;
    unsigned char* sel = (unsigned char*)calloc((size_t)S, 1);
    int* order = (int*)malloc(sizeof(int) * (size_t)S);
    /* all tokens by (s desc, t asc): repeated maximum search */
    unsigned char* used = (unsigned char*)calloc((size_t)S, 1);
    for (int k = 0; k < S; ++k) {
        int best = -1;
        for (int t = 0; t < S; ++t) {
            if (used[t]) continue;
            if (best < 0 || s_seg[t] > s_seg[best]) best = t;
        }
        used[best] = 1;
        order[k] = best;
    }
    for (int k = 0; k < r - a; ++k) sel[order[k]] = 1;
    /* candidate gaps between consecutive core positions */
    int nc = 0;
    int* ca = (int*)malloc(sizeof(int) * (size_t)S);
    int* cg = (int*)malloc(sizeof(int) * (size_t)S);
    double* cm = (double*)malloc(sizeof(double) * (size_t)S);
    int prev = -1;
    for (int t = 0; t < S; ++t) {
        if (!sel[t]) continue;
        if (prev >= 0 && t - prev - 1 >= 1 && t - prev + 1 <= gamma) {
            double m = 0.0;
            for (int x = prev + 1; x < t; ++x) m += s_seg[x];
            ca[nc] = prev;
            cg[nc] = t - prev - 1;
            cm[nc] = m;
            ++nc;
        }
        prev = t;
    }
    /* by (merit desc, start asc): selection sort */
    for (int i = 0; i < nc; ++i) {
        int best = i;
        for (int k = i + 1; k < nc; ++k)
            if (cm[k] > cm[best] || (cm[k] == cm[best] && ca[k] < ca[best])) best = k;
        int ta = ca[i], tg = cg[i];
        double tm = cm[i];
        ca[i] = ca[best]; cg[i] = cg[best]; cm[i] = cm[best];
        ca[best] = ta; cg[best] = tg; cm[best] = tm;
    }
    int rem = a;
    for (int i = 0; i < nc; ++i) {
        if (cg[i] > rem) continue;
        for (int x = ca[i] + 1; x <= ca[i] + cg[i]; ++x) sel[x] = 1;
        rem -= cg[i];
    }
    for (int k = 0; k < S && rem > 0; ++k) {
        if (sel[order[k]]) continue;
        sel[order[k]] = 1;
        --rem;
    }
    int w = 0;
    for (int t = 0; t < S; ++t)
        if (sel[t]) tidx[w++] = (uint8_t)t;
    free(sel);
    free(order);
    free(used);
    free(ca);
    free(cg);
    free(cm);
}

/* Error proxy of the four strategies of one segment, read as LOST ATTENTION
 * MASS (the pages name a per-segment choice but define no criterion):
 * a dropped token loses all of its mass s_t; a kept token whose key keeps
 * only C_t loses s_t * g_t.  Sums run in ascending token order.
 *   E_FULL = 0
 *   E_TOK  = sum_{t not in R} s_t
 *   E_CH   = sum_t s_t * g_t
 *   E_BOTH = E_TOK + (sum_{t in R} s_t * g_t)   (inner sum from 0.0)   */
void orc_segment_errors(const orc_params* p, const double* s_seg,
                        const double* g_seg, const uint8_t* tidx, double* E)
{
    int S = p->S, r = p->r;
    unsigned char* kept = (unsigned char*)calloc((size_t)S, 1);
    for (int j = 0; j < r; ++j) kept[tidx[j]] = 1;
    double etok = 0.0, ech = 0.0, ekept = 0.0;
    for (int t = 0; t < S; ++t)
        if (!kept[t]) etok += s_seg[t];
    for (int t = 0; t < S; ++t) ech += s_seg[t] * g_seg[t];
    for (int t = 0; t < S; ++t)
        if (kept[t]) ekept += s_seg[t] * g_seg[t];
    E[ORC_FULL] = 0.0;
    E[ORC_TOK] = etok;
    E[ORC_CH] = ech;
    E[ORC_BOTH] = etok + ekept;
    free(kept);
}

/* ------------------------------------------- step 6: packed bytes */

static int64_t pad16(int64_t x) { return (x + 15) / 16 * 16; }

/* Payload bytes of one segment in the packed layout of orc_pack_segment;
 * every section is padded to 16 bytes.  These bytes, indices and padding
 * included, are what the budget counts. */
int64_t orc_segment_bytes(const orc_params* p, int strategy)
{
    int64_t S = p->S, d = p->d, r = p->r, c = p->c;
    switch (strategy) {
    case ORC_FULL: return S * d * 2 + S * d * 2;
    case ORC_TOK:  return pad16(r) + r * d * 2 + r * d * 2;
    case ORC_CH:   return pad16(S * c) + pad16(S * c * 2) + S * d * 2;
    case ORC_BOTH: return pad16(r) + pad16(r * c) + pad16(r * c * 2) + r * d * 2;
    }
    return -1;
}

/* ------------------------------------------------- step 7: the hull */

/* Lower convex hull of the four (bytes, E) options of one segment.  Options
 * are visited by (bytes, id) ascending; an option no better than the last
 * hull point is skipped; an option with the same bytes as the last hull
 * point replaces it; the last point is popped while it lies on or above the
 * chord from the point before it to the new option.  Each product and
 * difference below is rounded once, in the order written.
 * Outputs: verts[0..nv) strategy ids along the hull (bytes ascending,
 * E strictly descending); for step k = 1..nv-1, dbytes[k-1] and
 * eff[k-1] = (E_{k-1} - E_k) / dbytes.  Returns nv. */
int orc_hull(const orc_params* p, const double* E, int32_t* verts,
             double* eff, int64_t* dbytes)
{
    int order[4] = {0, 1, 2, 3};
    int64_t b[4];
    for (int k = 0; k < 4; ++k) b[k] = orc_segment_bytes(p, k);
    /* insertion sort by (bytes, id) */
    for (int i = 1; i < 4; ++i) {
        int v = order[i], j = i - 1;
        while (j >= 0 && (b[order[j]] > b[v] ||
                          (b[order[j]] == b[v] && order[j] > v))) {
            order[j + 1] = order[j];
            --j;
        }
        order[j + 1] = v;
    }
    int h[4], nh = 0;
    h[nh++] = order[0];
    for (int i = 1; i < 4; ++i) {
        int o = order[i];
        int last = h[nh - 1];
        if (E[o] >= E[last]) continue;            /* dominated           */
        if (b[o] == b[last]) { h[nh - 1] = o; continue; }
        while (nh >= 2) {
            int A = h[nh - 2], B = h[nh - 1];
            double lhs = (E[A] - E[B]) * (double)(b[o] - b[B]);
            double rhs = (E[B] - E[o]) * (double)(b[B] - b[A]);
            if (lhs <= rhs) --nh; else break;
        }
        h[nh++] = o;
    }
    for (int k = 0; k < nh; ++k) verts[k] = h[k];
    for (int k = 1; k < nh; ++k) {
        dbytes[k - 1] = b[h[k]] - b[h[k - 1]];
        eff[k - 1] = (E[h[k - 1]] - E[h[k]]) / (double)dbytes[k - 1];
    }
    return nh;
}

/* --------------------------------------------- step 8: the budget */

/* Byte budget of one unit for the nseg segments of one compression call:
 * floor(beta * (nseg * FULL_bytes)), one fp64 rounding then the floor. */
int64_t orc_budget_bytes(const orc_params* p, int nseg)
{
    int64_t full = orc_segment_bytes(p, ORC_FULL);
    return (int64_t)floor(p->beta * (double)((int64_t)nseg * full));
}

typedef struct { double eff; int32_t seg, step; int64_t db; } orc_upg;

static int upg_cmp(const void* x, const void* y)
{
    const orc_upg* u = (const orc_upg*)x;
    const orc_upg* v = (const orc_upg*)y;
    if (u->eff > v->eff) return -1;
    if (u->eff < v->eff) return 1;
    if (u->seg != v->seg) return u->seg < v->seg ? -1 : 1;
    if (u->step != v->step) return u->step < v->step ? -1 : 1;
    return 0;
}

/* Budgeted choice of one strategy per segment (reading: the greedy
 * convex-hull solution of the multiple-choice knapsack).  beta >= 1 keeps
 * every segment FULL.  Otherwise every segment starts at its cheapest hull
 * point; if those bytes exceed the budget the call is infeasible; the hull
 * steps of all segments are then applied in (eff desc, segment asc, step
 * asc) order while each fits the remaining bytes, stopping at the first that
 * does not.  verts/nv/eff/dbytes are per segment with stride 4/1/3/3.
 * Writes strat[nseg] and *used; returns ORC_OK or ORC_INFEASIBLE. */
int orc_budget(const orc_params* p, int nseg, const int32_t* nv,
               const int32_t* verts, const double* eff, const int64_t* dbytes,
               int32_t* strat, int64_t* used)
{
    int64_t Bu = orc_budget_bytes(p, nseg);
    if (p->beta >= 1.0) {
        for (int j = 0; j < nseg; ++j) strat[j] = ORC_FULL;
        *used = (int64_t)nseg * orc_segment_bytes(p, ORC_FULL);
        return ORC_OK;
    }
    int64_t base = 0;
    for (int j = 0; j < nseg; ++j) base += orc_segment_bytes(p, verts[4 * j]);
    if (base > Bu) { *used = 0; return ORC_INFEASIBLE; }
    int nu = 0;
    for (int j = 0; j < nseg; ++j) nu += nv[j] - 1;
    orc_upg* list = (orc_upg*)malloc(sizeof(orc_upg) * (size_t)(nu > 0 ? nu : 1));
    int w = 0;
    for (int j = 0; j < nseg; ++j)
        for (int k = 1; k < nv[j]; ++k) {
            list[w].eff = eff[3 * j + k - 1];
            list[w].seg = j;
            list[w].step = k;
            list[w].db = dbytes[3 * j + k - 1];
            ++w;
        }
    qsort(list, (size_t)nu, sizeof(orc_upg), upg_cmp);
    int32_t* level = (int32_t*)calloc((size_t)(nseg > 0 ? nseg : 1), sizeof(int32_t));
    int64_t rem = Bu - base;
    for (int i = 0; i < nu; ++i) {
        if (list[i].db > rem) break;
        rem -= list[i].db;
        level[list[i].seg] = list[i].step;
    }
    int64_t tot = 0;
    for (int j = 0; j < nseg; ++j) {
        strat[j] = verts[4 * j + level[j]];
        tot += orc_segment_bytes(p, strat[j]);
    }
    *used = tot;
    free(list);
    free(level);
    return ORC_OK;
}

/* ------------------------------------------------ step 9: packing */

/* Packed layout of one segment (the pages name a packed KV format and a
 * flexible encoding but give no layout; this one is chosen so that every
 * section starts on 16 bytes).  K16/V16 are the segment's S rows of d fp16
 * bit patterns; tidx is R_j (ascending, segment-relative); cidx_all holds
 * C_t for all S tokens.  Sections, each zero-padded to 16 bytes:
 *   FULL : K[S][d] | V[S][d]
 *   TOK  : tidx[r] | K[r][d] | V[r][d]
 *   CH   : cidx[S][c] | Kval[S][c] | V[S][d]
 *   BOTH : tidx[r] | cidx[r][c] | Kval[r][c] | V[r][d]
 * Kval[t][j] = K[t][cidx[t][j]].  Returns the bytes written. */
int64_t orc_pack_segment(const orc_params* p, int strategy,
                         const uint16_t* K16, const uint16_t* V16,
                         const uint8_t* tidx, const uint8_t* cidx_all,
                         uint8_t* out)
{
    int S = p->S, d = p->d, r = p->r, c = p->c;
    int64_t nb = orc_segment_bytes(p, strategy);
    memset(out, 0, (size_t)nb);
    uint8_t* o = out;
    int ntok = (strategy == ORC_TOK || strategy == ORC_BOTH) ? r : S;
    int tok[256];
    for (int j = 0; j < ntok; ++j)
        tok[j] = (strategy == ORC_TOK || strategy == ORC_BOTH) ? tidx[j] : j;
    if (strategy == ORC_TOK || strategy == ORC_BOTH) {
        memcpy(o, tidx, (size_t)r);
        o += pad16(r);
    }
    if (strategy == ORC_FULL || strategy == ORC_TOK) {
        for (int j = 0; j < ntok; ++j)
            memcpy(o + (int64_t)j * d * 2, K16 + (int64_t)tok[j] * d, (size_t)d * 2);
        o += (int64_t)ntok * d * 2;
    } else {
        for (int j = 0; j < ntok; ++j)
            memcpy(o + (int64_t)j * c, cidx_all + (int64_t)tok[j] * c, (size_t)c);
        o += pad16((int64_t)ntok * c);
        uint16_t* kv = (uint16_t*)o;
        for (int j = 0; j < ntok; ++j)
            for (int x = 0; x < c; ++x) {
                int ch = cidx_all[(int64_t)tok[j] * c + x];
                kv[(int64_t)j * c + x] = K16[(int64_t)tok[j] * d + ch];
            }
        o += pad16((int64_t)ntok * c * 2);
    }
    for (int j = 0; j < ntok; ++j)
        memcpy(o + (int64_t)j * d * 2, V16 + (int64_t)tok[j] * d, (size_t)d * 2);
    o += (int64_t)ntok * d * 2;
    return (int64_t)(o - out);
}

/* ----------------------------------------- whole compression of a unit */

/* Compresses the nseg complete segments of the region [r0, T) of one unit
 * (K16/V16: the region's rows as fp16 bits; Kd: the same keys as doubles;
 * qw: the G*W window rows as doubles).  a_in / s_in may be NULL (computed
 * here in fp64) or given (the "fed" mode that checks the selection steps on
 * another implementation's scores).  Outputs (caller-sized):
 *   a[d], lse[G*W], s[T-r0], g[nseg*S], cidx[nseg*S*c], tidx[nseg*r],
 *   E[nseg*4], strat[nseg], offs[nseg] (payload offsets from arena_base),
 *   arena (appended at arena_base), *used (bytes written).
 * Returns ORC_OK, ORC_INFEASIBLE or -1 (bad arguments). */
int orc_compress_unit(const orc_params* p, int T, int r0,
                      const uint16_t* K16, const uint16_t* V16,
                      const double* Kd, const double* qw,
                      const double* a_in, const double* s_in,
                      double* a, double* lse, double* s, double* g,
                      uint8_t* cidx, uint8_t* tidx, double* E, int32_t* strat,
                      int64_t* offs, uint8_t* arena, int64_t arena_base,
                      int64_t* used)
{
    int S = p->S, d = p->d;
    int nseg = (T - r0) / S;
    if (a_in) memcpy(a, a_in, sizeof(double) * (size_t)d);
    else orc_win_stats(p, qw, a);
    if (s_in) {
        memcpy(s, s_in, sizeof(double) * (size_t)(T - r0));
        for (int i = 0; i < p->G * p->W; ++i) lse[i] = NAN;
    } else if (orc_score(p, T, r0, Kd, qw, lse, s) != 0) {
        return -1;
    }
    orc_channel(p, nseg * S, Kd, a, cidx, g);
    int32_t* nv = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nseg + 1));
    int32_t* verts = (int32_t*)malloc(sizeof(int32_t) * 4 * (size_t)(nseg + 1));
    double* eff = (double*)malloc(sizeof(double) * 3 * (size_t)(nseg + 1));
    int64_t* db = (int64_t*)malloc(sizeof(int64_t) * 3 * (size_t)(nseg + 1));
    for (int j = 0; j < nseg; ++j) {
        if (p->chunk_len > 0)
            orc_topr_chunks(p, s + (int64_t)j * S, tidx + (int64_t)j * p->r);
        else
            orc_topr(p, s + (int64_t)j * S, tidx + (int64_t)j * p->r);
        orc_segment_errors(p, s + (int64_t)j * S, g + (int64_t)j * S,
                           tidx + (int64_t)j * p->r, E + 4 * (int64_t)j);
        nv[j] = orc_hull(p, E + 4 * (int64_t)j, verts + 4 * j, eff + 3 * j, db + 3 * j);
    }
    int st = orc_budget(p, nseg, nv, verts, eff, db, strat, used);
    if (st == ORC_OK) {
        int64_t off = arena_base;
        for (int j = 0; j < nseg; ++j) {
            offs[j] = off;
            off += orc_pack_segment(p, strat[j], K16 + (int64_t)j * S * d,
                                    V16 + (int64_t)j * S * d,
                                    tidx + (int64_t)j * p->r,
                                    cidx + (int64_t)j * S * p->c, arena + off);
        }
    }
    free(nv);
    free(verts);
    free(eff);
    free(db);
    return st;
}

/* ----------------------------------------------- step 10: decode */

/* Attention of the G query heads of one unit over its compressed segments
 * and its dense tail ([MosaicKV] Sec. 5.3: attention runs directly on the
 * packed segments).  Readings: dropped channels contribute nothing to q.k
 * (no rescaling); dropped tokens are left out of the softmax; all kept
 * tokens keep their whole value vector.
 *   logit = scale * q . k           (FULL, TOK, dense tail)
 *   logit = scale * sum_j q[cidx_j] * Kval_j   (CH, BOTH)
 *   out[g] = sum_t softmax(logit)_t * v_t
 * arena + offs[j] holds segment j with strategy strat[j]; Kt/Vt are the
 * n_tail dense rows as doubles; q is [G][d]; out is [G][d]. */
void orc_decode(const orc_params* p, int nseg, const uint8_t* arena,
                const int64_t* offs, const int32_t* strat, int n_tail,
                const double* Kt, const double* Vt, const double* q,
                double* out)
{
    int S = p->S, d = p->d, r = p->r, c = p->c, G = p->G;
    int64_t ntot = (int64_t)nseg * S + n_tail;
    double* logit = (double*)malloc(sizeof(double) * (size_t)(ntot > 0 ? ntot : 1));
    double* vrows = (double*)malloc(sizeof(double) * (size_t)(ntot > 0 ? ntot : 1) * d);
    for (int g = 0; g < G; ++g) {
        const double* qg = q + (int64_t)g * d;
        int64_t n = 0;
        for (int j = 0; j < nseg; ++j) {
            const uint8_t* seg = arena + offs[j];
            int st = strat[j];
            int ntok = (st == ORC_TOK || st == ORC_BOTH) ? r : S;
            const uint8_t* sec = seg;
            if (st == ORC_TOK || st == ORC_BOTH) sec += pad16(r);
            const uint8_t* vsec;
            for (int t = 0; t < ntok; ++t) {
                double dot = 0.0;
                if (st == ORC_FULL || st == ORC_TOK) {
                    const uint8_t* krow = sec + (int64_t)t * d * 2;
                    for (int x = 0; x < d; ++x) {
                        uint16_t h = (uint16_t)(krow[2 * x] | (krow[2 * x + 1] << 8));
                        dot += qg[x] * orc_half_to_double(h);
                    }
                } else {
                    const uint8_t* ci = sec + (int64_t)t * c;
                    const uint8_t* kv = sec + pad16((int64_t)ntok * c) + (int64_t)t * c * 2;
                    for (int x = 0; x < c; ++x) {
                        uint16_t h = (uint16_t)(kv[2 * x] | (kv[2 * x + 1] << 8));
                        dot += qg[ci[x]] * orc_half_to_double(h);
                    }
                }
                logit[n + t] = p->scale * dot;
            }
            if (st == ORC_FULL || st == ORC_TOK)
                vsec = sec + (int64_t)ntok * d * 2;
            else
                vsec = sec + pad16((int64_t)ntok * c) + pad16((int64_t)ntok * c * 2);
            for (int t = 0; t < ntok; ++t)
                for (int x = 0; x < d; ++x) {
                    const uint8_t* vb = vsec + ((int64_t)t * d + x) * 2;
                    vrows[(n + t) * d + x] = orc_half_to_double((uint16_t)(vb[0] | (vb[1] << 8)));
                }
            n += ntok;
        }
        for (int t = 0; t < n_tail; ++t) {
            double dot = 0.0;
            for (int x = 0; x < d; ++x) dot += qg[x] * Kt[(int64_t)t * d + x];
            logit[n + t] = p->scale * dot;
            for (int x = 0; x < d; ++x) vrows[(n + t) * d + x] = Vt[(int64_t)t * d + x];
        }
        n += n_tail;
        double mx = -INFINITY;
        for (int64_t t = 0; t < n; ++t) if (logit[t] > mx) mx = logit[t];
        double z = 0.0;
        for (int64_t t = 0; t < n; ++t) z += exp(logit[t] - mx);
        for (int x = 0; x < d; ++x) out[(int64_t)g * d + x] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            double w = exp(logit[t] - mx) / z;
            for (int x = 0; x < d; ++x) out[(int64_t)g * d + x] += w * vrows[t * d + x];
        }
    }
    free(logit);
    free(vrows);
}

/* ------------------------------ decode-time token selection (stage 2) */

/* [MosaicKV] Fig. 6 caption: "stage 2" (sequence compression) runs in the
 * decode stage before each attention layer; Sec. 5.3: PackedAttention
 * performs sequence compression and attention in each layer of the decode
 * stage; Fig. 8: token selection rates of 6.25% and 12.5%.  The pages give no
 * rule, so these readings are taken:
 *   - candidates are the tokens the packed segments keep (S for FULL / CH, r
 *     for TOK / BOTH), slot j*S + i for token i of segment j; the dense tail
 *     [comp_end, T) is always attended;
 *   - the score of a candidate is the largest over the G query heads of its
 *     logit, scale * q_g . k (the stored key: whole for FULL / TOK, its kept
 *     channels for CH / BOTH), so one selection serves the heads that share
 *     the KV head;
 *   - the rate rho counts tokens of the compressed context:
 *     n_sel = min(candidates, ceil(rho * nseg * S));
 *   - the n_sel largest scores are kept, ties to the lower slot;
 *   - attention then runs over the kept candidates and the dense tail, the
 *     others leaving the softmax. */

/* Key of candidate i of segment j as doubles (dropped channels 0). */
static void orc_candidate_key(const orc_params* p, const uint8_t* seg, int st, int i, double* k)
{
    int S = p->S, d = p->d, r = p->r, c = p->c;
    int ntok = (st == ORC_TOK || st == ORC_BOTH) ? r : S;
    const uint8_t* sec = seg + ((st == ORC_TOK || st == ORC_BOTH) ? pad16(r) : 0);
    for (int x = 0; x < d; ++x) k[x] = 0.0;
    if (st == ORC_FULL || st == ORC_TOK) {
        const uint8_t* krow = sec + (int64_t)i * d * 2;
        for (int x = 0; x < d; ++x)
            k[x] = orc_half_to_double((uint16_t)(krow[2 * x] | (krow[2 * x + 1] << 8)));
    } else {
        const uint8_t* ci = sec + (int64_t)i * c;
        const uint8_t* kv = sec + pad16((int64_t)ntok * c) + (int64_t)i * c * 2;
        for (int x = 0; x < c; ++x)
            k[ci[x]] = orc_half_to_double((uint16_t)(kv[2 * x] | (kv[2 * x + 1] << 8)));
    }
}

/* score[j*S + i] = max_g scale * q_g . k_{j,i} for every candidate, -inf for
 * slots past a segment's kept tokens.  Returns the number of candidates. */
int64_t orc_select_scores(const orc_params* p, int nseg, const uint8_t* arena, const int64_t* offs,
                          const int32_t* strat, const double* q, double* score)
{
    int S = p->S, d = p->d, G = p->G;
    double* k = (double*)malloc(sizeof(double) * (size_t)d);
    int64_t ncand = 0;
    for (int j = 0; j < nseg; ++j) {
        int st = strat[j];
        int ntok = (st == ORC_TOK || st == ORC_BOTH) ? p->r : S;
        for (int i = 0; i < S; ++i) {
            double best = -INFINITY;
            if (i < ntok) {
                orc_candidate_key(p, arena + offs[j], st, i, k);
                for (int g = 0; g < G; ++g) {
                    double dot = 0.0;
                    for (int x = 0; x < d; ++x) dot += q[(int64_t)g * d + x] * k[x];
                    double l = p->scale * dot;
                    if (l > best) best = l;
                }
                ++ncand;
            }
            score[(int64_t)j * S + i] = best;
        }
    }
    free(k);
    return ncand;
}

/* Tokens to keep at rate rho for nseg segments and ncand candidates. */
int64_t orc_select_count(const orc_params* p, int nseg, int64_t ncand, double rho)
{
    double want = ceil(rho * (double)((int64_t)nseg * p->S));
    int64_t n = (int64_t)want;
    if (want >= (double)ncand) n = ncand;
    return n < 0 ? 0 : n;
}

/* sel[slot] = 1 for the n_sel largest finite scores, ties to the lower
 * slot (a plain repeated maximum search). */
void orc_select_tokens(int64_t nslots, const double* score, int64_t n_sel, uint8_t* sel)
{
    for (int64_t s = 0; s < nslots; ++s) sel[s] = 0;
    for (int64_t n = 0; n < n_sel; ++n) {
        int64_t arg = -1;
        for (int64_t s = 0; s < nslots; ++s) {
            if (sel[s] || score[s] == -INFINITY) continue;
            if (arg < 0 || score[s] > score[arg]) arg = s;
        }
        if (arg < 0) break;
        sel[arg] = 1;
    }
}

/* Attention of the G heads over the selected candidates and the dense tail:
 * per head, softmax over that set of logits scale * q_g . k, output the
 * weighted sum of the value rows. */
void orc_decode_select(const orc_params* p, int nseg, const uint8_t* arena, const int64_t* offs,
                       const int32_t* strat, const uint8_t* sel, int n_tail, const double* Kt,
                       const double* Vt, const double* q, double* out)
{
    int S = p->S, d = p->d, r = p->r, c = p->c, G = p->G;
    int64_t cap = (int64_t)nseg * S + n_tail;
    double* logit = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
    double* vrows = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1) * d);
    double* k = (double*)malloc(sizeof(double) * (size_t)d);
    for (int g = 0; g < G; ++g) {
        const double* qg = q + (int64_t)g * d;
        int64_t n = 0;
        for (int j = 0; j < nseg; ++j) {
            int st = strat[j];
            int ntok = (st == ORC_TOK || st == ORC_BOTH) ? r : S;
            const uint8_t* seg = arena + offs[j];
            const uint8_t* sec = seg + ((st == ORC_TOK || st == ORC_BOTH) ? pad16(r) : 0);
            const uint8_t* vsec = (st == ORC_FULL || st == ORC_TOK)
                                      ? sec + (int64_t)ntok * d * 2
                                      : sec + pad16((int64_t)ntok * c) + pad16((int64_t)ntok * c * 2);
            for (int i = 0; i < ntok; ++i) {
                if (!sel[(int64_t)j * S + i]) continue;
                orc_candidate_key(p, seg, st, i, k);
                double dot = 0.0;
                for (int x = 0; x < d; ++x) dot += qg[x] * k[x];
                logit[n] = p->scale * dot;
                for (int x = 0; x < d; ++x) {
                    const uint8_t* vb = vsec + ((int64_t)i * d + x) * 2;
                    vrows[n * d + x] = orc_half_to_double((uint16_t)(vb[0] | (vb[1] << 8)));
                }
                ++n;
            }
        }
        for (int t = 0; t < n_tail; ++t) {
            double dot = 0.0;
            for (int x = 0; x < d; ++x) dot += qg[x] * Kt[(int64_t)t * d + x];
            logit[n] = p->scale * dot;
            for (int x = 0; x < d; ++x) vrows[n * d + x] = Vt[(int64_t)t * d + x];
            ++n;
        }
        for (int x = 0; x < d; ++x) out[(int64_t)g * d + x] = 0.0;
        if (n == 0) continue;
        double mx = -INFINITY;
        for (int64_t t = 0; t < n; ++t) if (logit[t] > mx) mx = logit[t];
        double z = 0.0;
        for (int64_t t = 0; t < n; ++t) z += exp(logit[t] - mx);
        for (int64_t t = 0; t < n; ++t) {
            double w = exp(logit[t] - mx) / z;
            for (int x = 0; x < d; ++x) out[(int64_t)g * d + x] += w * vrows[t * d + x];
        }
    }
    free(k);
    free(logit);
    free(vrows);
}
