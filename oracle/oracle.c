/*
 * Oracle for zigzag context-parallel causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the package entry's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header or table
 * with the CUDA library.
 *
 * Everything is written from the definitions, in double precision, with no
 * blocking, fusion or reordering beyond what the definition states:
 *
 *  - Context parallelism shards Q, K and V along the sequence; rank i keeps
 *    Q_i and attends it against its own K_i,V_i and then every other rank's
 *    K_j,V_j, after which the partial attentions are combined
 *    (Accelerate "Context Parallel" concept guide, "So how does it work?",
 *    the pseudocode block).
 *  - The sequence length must be divisible by 2*cp (NeMo "Hierarchical
 *    Context Parallel Skill", "Required constraints"); the 2*cp chunks are
 *    paired head/tail so rank r owns chunks r and 2*cp-1-r.
 *  - All-gather visits the K/V shards in rank order after one gather; ring
 *    ("all-to-all") rotation receives the neighbour's shard cp-1 times
 *    (concept guide, "all-to-all vs all-gather").
 *  - "combine" is read as the exact log-sum-exp merge, the only combination
 *    under which the sharded result equals unsharded attention.
 *
 * Layouts: attention tensors are [BH][S][D] (batch and head flattened),
 * original token order unless a function says "shard order".  doc_start is a
 * per-original-position array: the first original position of the document
 * holding that token (all zeros for the plain causal mask).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1

/* ------------------------------------------------------------------------ */
/* Plan                                                                      */
/* ------------------------------------------------------------------------ */

/* Original position of local token t (0 <= t < 2C) of virtual rank r: the
 * first C local tokens are chunk r, the next C are chunk 2cp-1-r. */
static int64_t orc_orig_of_local(int64_t C, int64_t cp, int64_t r, int64_t t)
{
    int64_t chunk = (t < C) ? r : (2 * cp - 1 - r);
    return chunk * C + (t % C);
}

/* Document start for every original position, from cu_seqlens (num_docs+1
 * offsets, cu[0]=0, cu[num_docs]=S).  num_docs == 0 means one document. */
int orc_doc_start(int32_t S, int32_t num_docs, const int32_t *cu, int32_t *ds_orig)
{
    if (num_docs <= 0) {
        for (int32_t i = 0; i < S; ++i) ds_orig[i] = 0;
        return ORC_OK;
    }
    if (cu[0] != 0 || cu[num_docs] != S) return ORC_EINVAL;
    for (int32_t d = 0; d < num_docs; ++d) {
        if (cu[d + 1] <= cu[d]) return ORC_EINVAL;
        for (int32_t i = cu[d]; i < cu[d + 1]; ++i) ds_orig[i] = cu[d];
    }
    return ORC_OK;
}

/*
 * The zigzag shard plan.
 *   perm[r*2C + t]  = original index of local token t of rank r.  Sequence-level
 *                     sharding (per_doc = 0): rank r holds chunk r, then chunk
 *                     2cp-1-r of the whole sequence.  Per-document sharding
 *                     (per_doc = 1): every document is cut into 2cp equal
 *                     chunks and rank r holds, document after document, its
 *                     chunk r followed by its chunk 2cp-1-r (each document's
 *                     length must be a multiple of 2cp).
 *   inv_perm[o]     = shard position of original index o
 *   src[r*cp + s]   = K/V shard visited by rank r at step s:
 *                     s (all-gather, rank order) or (r - s) mod cp (ring,
 *                     receiving from the left neighbour each step); step 0
 *                     is the local shard under the ring order.
 *   doc_start[p]    = doc start (original coordinates) of token perm[p]
 *   rank_cu_off[r]  = offset of rank r's list in rank_cu; rank_cu_off[cp] =
 *                     total entries.  rank r's list holds the local offsets
 *                     where a segment starts, then 2C: sequence-level, local 0,
 *                     the chunk boundary C and every document start inside its
 *                     chunks; per-document, the start of each of its chunks
 *                     (two per document).
 *   pairs[r]        = number of unmasked (q, k) pairs whose query is on rank r;
 *                     causal: the query at o sees keys ds(o) .. o, raised to
 *                     max(ds(o), o - W + 1) under a sliding window W > 0
 *                     (window 0: no window); without the causal mask
 *                     (causal = 0) it sees its whole document, ds(o) ..
 *                     de(o) - 1 (window: only 0 is accepted then)
 * Returns ORC_EINVAL on a bad configuration.
 */
int orc_plan(int32_t S, int32_t cp, int32_t rotate, int32_t num_docs, const int32_t *cu,
             int32_t window, int32_t causal, int32_t per_doc, int32_t *perm, int32_t *inv_perm,
             int32_t *src, int32_t *doc_start, int32_t *rank_cu_off, int32_t *rank_cu,
             int64_t *pairs)
{
    if (cp < 1 || S <= 0 || S % (2 * cp) != 0 || window < 0) return ORC_EINVAL;
    if (!causal && window != 0) return ORC_EINVAL;
    if (rotate != 0 && rotate != 1) return ORC_EINVAL;
    if (per_doc && num_docs < 1) return ORC_EINVAL;
    int64_t C = S / (2 * cp);
    int32_t *ds_orig = (int32_t *)malloc(sizeof(int32_t) * (size_t)S);
    if (!ds_orig) return ORC_EINVAL;
    if (orc_doc_start(S, num_docs, cu, ds_orig) != ORC_OK) { free(ds_orig); return ORC_EINVAL; }
    if (per_doc)
        for (int64_t d = 0; d < num_docs; ++d)
            if ((cu[d + 1] - cu[d]) % (2 * cp) != 0) { free(ds_orig); return ORC_EINVAL; }

    int32_t n = 0;   /* entries written to rank_cu */
    if (!per_doc) {
        for (int64_t r = 0; r < cp; ++r)
            for (int64_t t = 0; t < 2 * C; ++t) {
                int64_t o = orc_orig_of_local(C, cp, r, t);
                perm[r * 2 * C + t] = (int32_t)o;
                inv_perm[o] = (int32_t)(r * 2 * C + t);
            }
    } else {
        /* rank r's local tokens, appended document by document: its chunk r, then
         * its chunk 2cp-1-r; each appended chunk starts a segment */
        for (int64_t r = 0; r < cp; ++r) {
            rank_cu_off[r] = n;
            int64_t t = 0;
            for (int64_t d = 0; d < num_docs; ++d) {
                int64_t len = (cu[d + 1] - cu[d]) / (2 * cp);
                int64_t chunks[2] = {r, 2 * cp - 1 - r};
                for (int h = 0; h < 2; ++h) {
                    rank_cu[n++] = (int32_t)t;
                    for (int64_t w = 0; w < len; ++w, ++t) {
                        int64_t o = cu[d] + chunks[h] * len + w;
                        perm[r * 2 * C + t] = (int32_t)o;
                        inv_perm[o] = (int32_t)(r * 2 * C + t);
                    }
                }
            }
            rank_cu[n++] = (int32_t)(2 * C);
        }
        rank_cu_off[cp] = n;
    }
    for (int64_t r = 0; r < cp; ++r)
        for (int64_t s = 0; s < cp; ++s)
            src[r * cp + s] = (int32_t)(rotate == 0 ? s : ((r - s) % cp + cp) % cp);
    for (int64_t p = 0; p < S; ++p) doc_start[p] = ds_orig[perm[p]];

    for (int64_t r = 0; r < cp; ++r) {
        if (!per_doc) rank_cu_off[r] = n;
        int64_t cnt = 0;
        for (int64_t t = 0; t < 2 * C; ++t) {
            int64_t o = perm[r * 2 * C + t];
            int is_start = (t == 0) || (t == C) || (ds_orig[o] == o);
            if (!per_doc && is_start) rank_cu[n++] = (int32_t)t;
            int64_t first = ds_orig[o];
            if (window > 0 && o - window + 1 > first) first = o - window + 1;
            int64_t last = o;
            if (!causal) { /* the end of o's document: the next document's start, or S */
                last = S - 1;
                for (int64_t d = 0; d < num_docs; ++d)
                    if (cu[d] > o) { last = cu[d] - 1; break; }
            }
            cnt += last - first + 1; /* keys first..last are unmasked */
        }
        if (!per_doc) rank_cu[n++] = (int32_t)(2 * C);
        pairs[r] = cnt;
    }
    if (!per_doc) rank_cu_off[cp] = n;
    free(ds_orig);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Attention by the definition                                               */
/* ------------------------------------------------------------------------ */

/* mask(q, k) for original positions: the query at q sees the keys
 * ds_orig[q] <= k <= lk_orig[q].  Causal: lk_orig[q] = q; without the causal
 * mask: the last key of q's document (S - 1 with one document).  ds_orig[q] is
 * q's document start, raised to q - W + 1 under a sliding window of W keys. */
static int orc_mask(const int32_t *ds_orig, const int32_t *lk_orig, int64_t q, int64_t k)
{
    return k <= lk_orig[q] && k >= ds_orig[q];
}

/*
 * One query row against an explicit key set, by the definition:
 *   LSE = ln sum_k exp(scale * q.k),   O = sum_k exp(scale*q.k - LSE) v_k
 * over the keys in keys[0..nk) that the mask admits.  No admitted key gives
 * LSE = -inf and O = 0.  q_vec/o are D-vectors; kmat/vmat are the head's
 * [S][D] arrays in original order; keys are original positions.
 */
static void orc_row(int64_t D, double scale, const double *q_vec, int64_t q_orig,
                    const double *kmat, const double *vmat, const int64_t *keys, int64_t nk,
                    const int32_t *ds_orig, const int32_t *lk_orig, double *sc, double *o,
                    double *lse)
{
    double m = -INFINITY;
    for (int64_t i = 0; i < nk; ++i) {
        int64_t k = keys[i];
        if (!orc_mask(ds_orig, lk_orig, q_orig, k)) { sc[i] = -INFINITY; continue; }
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += q_vec[d] * kmat[k * D + d];
        sc[i] = scale * dot;
        if (sc[i] > m) m = sc[i];
    }
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; return; }
    double l = 0.0;
    for (int64_t i = 0; i < nk; ++i) {
        if (sc[i] == -INFINITY) continue;
        double w = exp(sc[i] - m);
        l += w;
        const double *v = vmat + keys[i] * D;
        for (int64_t d = 0; d < D; ++d) o[d] += w * v[d];
    }
    for (int64_t d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
}

/*
 * Unsharded attention for selected rows.  rows[i] = bh*S + q (original q).
 * GQA: query head h of batch b reads KV head h / (Hq/Hkv) of batch b.
 * Output o[i][D], lse[i].  Keys visited: 0..lk_orig[q] (the mask trims the rest).
 */
int orc_fwd_rows(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, double scale,
                 const double *q, const double *k, const double *v, const int32_t *ds_orig,
                 const int32_t *lk_orig, int64_t nrows, const int64_t *rows, double *o,
                 double *lse)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return ORC_EINVAL;
    int64_t g = Hq / Hkv;
    int64_t err = 0;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)S);
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)S);
        if (!sc || !keys) {
#pragma omp atomic write
            err = 1;
        } else {
            for (int64_t t = 0; t < S; ++t) keys[t] = t;
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < nrows; ++i) {
                int64_t bh = rows[i] / S, qi = rows[i] % S;
                int64_t b = bh / Hq, h = bh % Hq;
                int64_t bkv = b * Hkv + h / g;
                orc_row(D, scale, q + (bh * S + qi) * D, qi, k + bkv * (int64_t)S * D,
                        v + bkv * (int64_t)S * D, keys, (int64_t)lk_orig[qi] + 1, ds_orig, lk_orig,
                        sc, o + i * D, lse + i);
            }
        }
        free(sc);
        free(keys);
    }
    (void)B;
    return err ? ORC_EINVAL : ORC_OK;
}

/* Unsharded attention over every row: o[BH][S][D], lse[BH][S] (original order). */
int orc_fwd(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, double scale,
            const double *q, const double *k, const double *v, const int32_t *ds_orig,
            const int32_t *lk_orig, double *o, double *lse)
{
    int64_t n = (int64_t)B * Hq * S;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
    if (!rows) return ORC_EINVAL;
    for (int64_t i = 0; i < n; ++i) rows[i] = i;
    int rc = orc_fwd_rows(B, Hq, Hkv, S, D, scale, q, k, v, ds_orig, lk_orig, n, rows, o, lse);
    free(rows);
    return rc;
}

/*
 * The per-(rank, step) partial of the shard loop: Q_r (the 2C rows of rank r)
 * against K_j, V_j (the 2C keys of rank j).  Inputs are in ORIGINAL order;
 * the rank's tokens are located through perm.  Output o_part[BH][2C][D] and
 * lse_part[BH][2C] for rank r's local rows (shard order within the rank).
 */
int orc_partial(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, int32_t cp,
                double scale, const double *q, const double *k, const double *v,
                const int32_t *ds_orig, const int32_t *lk_orig, const int32_t *perm, int32_t r,
                int32_t j, double *o_part, double *lse_part)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || S % (2 * cp) != 0) return ORC_EINVAL;
    int64_t g = Hq / Hkv, n2c = S / cp, BH = (int64_t)B * Hq;
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)n2c);
    if (!keys) return ORC_EINVAL;
    for (int64_t t = 0; t < n2c; ++t) keys[t] = perm[(int64_t)j * n2c + t];
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)n2c);
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < BH * n2c; ++i) {
            int64_t bh = i / n2c, t = i % n2c;
            int64_t b = bh / Hq, h = bh % Hq, bkv = b * Hkv + h / g;
            int64_t qi = perm[(int64_t)r * n2c + t];
            orc_row(D, scale, q + (bh * S + qi) * D, qi, k + bkv * (int64_t)S * D,
                    v + bkv * (int64_t)S * D, keys, n2c, ds_orig, lk_orig, sc, o_part + i * D,
                    lse_part + i);
        }
        free(sc);
    }
    free(keys);
    return ORC_OK;
}

/*
 * The backward of one (rank, step) unit: rank r's queries (its 2C rows) against
 * shard j's keys (its 2C rows), by the explicit-P formula with P taken from the
 * final LSE and D_q = sum_d dO*O from the final O (the row's own forward is not
 * redone).  Inputs in ORIGINAL order, the rank's and the shard's tokens located
 * through perm.  Outputs in local shard order: dq_part[B*Hq][2C][D] for rank
 * r's rows, dk_part / dv_part[B*Hkv][2C][D] for shard j's rows.  Summed over
 * the steps (dQ_r) and over the ranks (dK_j, dV_j) they are the gradients of
 * the unsharded attention.
 */
int orc_bwd_partial(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, int32_t cp,
                    double scale, const double *q, const double *k, const double *v,
                    const double *o, const double *lse, const double *dout,
                    const int32_t *ds_orig, const int32_t *lk_orig, const int32_t *perm, int32_t r,
                    int32_t j, double *dq_part, double *dk_part, double *dv_part)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || cp < 1 || S % (2 * cp) != 0 || r < 0 || r >= cp || j < 0 ||
        j >= cp)
        return ORC_EINVAL;
    int64_t g = Hq / Hkv, n2c = S / cp, SD = (int64_t)S * D;
    memset(dq_part, 0, sizeof(double) * (size_t)((int64_t)B * Hq * n2c * D));
    memset(dk_part, 0, sizeof(double) * (size_t)((int64_t)B * Hkv * n2c * D));
    memset(dv_part, 0, sizeof(double) * (size_t)((int64_t)B * Hkv * n2c * D));
    /* one KV head per task: its dK/dV rows collect over the group's query heads */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bkv = 0; bkv < (int64_t)B * Hkv; ++bkv) {
        int64_t b = bkv / Hkv, hk = bkv % Hkv;
        const double *kh = k + bkv * SD, *vh = v + bkv * SD;
        double *dkh = dk_part + bkv * n2c * D, *dvh = dv_part + bkv * n2c * D;
        for (int64_t h = hk * g; h < (hk + 1) * g; ++h) {
            int64_t bh = b * Hq + h;
            for (int64_t t = 0; t < n2c; ++t) {
                int64_t qi = perm[(int64_t)r * n2c + t];
                const double *qv = q + (bh * S + qi) * D, *ov = o + (bh * S + qi) * D;
                const double *dov = dout + (bh * S + qi) * D;
                double *dqv = dq_part + (bh * n2c + t) * D;
                double L = lse[bh * S + qi], Dq = 0.0;
                for (int64_t d = 0; d < D; ++d) Dq += dov[d] * ov[d];
                for (int64_t u = 0; u < n2c; ++u) {
                    int64_t kk = perm[(int64_t)j * n2c + u];
                    if (kk < ds_orig[qi] || kk > lk_orig[qi]) continue;
                    const double *kv = kh + kk * D, *vv = vh + kk * D;
                    double dot = 0.0, dP = 0.0;
                    for (int64_t d = 0; d < D; ++d) { dot += qv[d] * kv[d]; dP += dov[d] * vv[d]; }
                    double P = exp(scale * dot - L);
                    double dS = P * (dP - Dq);
                    for (int64_t d = 0; d < D; ++d) {
                        dvh[u * D + d] += P * dov[d];
                        dqv[d] += scale * dS * kv[d];
                        dkh[u * D + d] += scale * dS * qv[d];
                    }
                }
            }
        }
    }
    return ORC_OK;
}

/*
 * combine(): fold n_parts partial (O, LSE) pairs, in the given order, into one.
 * For the running pair (O_a, L_a) and the next (O_b, L_b):
 *   m = max(L_a, L_b); if m = -inf the result stays (0, -inf); otherwise
 *   w_x = exp(L_x - m), L = m + ln(w_a + w_b), O = (w_a O_a + w_b O_b)/(w_a + w_b).
 * o_parts[n_parts][rows][D], lse_parts[n_parts][rows].
 */
void orc_lse_merge(int64_t rows, int32_t D, int32_t n_parts, const double *o_parts,
                   const double *lse_parts, double *o_out, double *lse_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        double L = -INFINITY;
        double *o = o_out + i * D;
        for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
        for (int32_t p = 0; p < n_parts; ++p) {
            double Lb = lse_parts[(int64_t)p * rows + i];
            const double *ob = o_parts + ((int64_t)p * rows + i) * D;
            double m = L > Lb ? L : Lb;
            if (m == -INFINITY) continue;
            double wa = (L == -INFINITY) ? 0.0 : exp(L - m);
            double wb = (Lb == -INFINITY) ? 0.0 : exp(Lb - m);
            for (int32_t d = 0; d < D; ++d) o[d] = (wa * o[d] + wb * ob[d]) / (wa + wb);
            L = m + log(wa + wb);
        }
        lse_out[i] = L;
    }
}

/* ------------------------------------------------------------------------ */
/* Backward by the explicit-P formula                                        */
/* ------------------------------------------------------------------------ */

/*
 * Gradients of the attention output given the upstream gradient dO, using the
 * final LSE:  P = exp(scale q.k - LSE_q),  Dq = sum_d dO_q O_q,
 *   dV_k += P dO_q,  dP = dO_q . v_k,  dS = P (dP - Dq),
 *   dQ_q += scale dS k_k,  dK_k += scale dS q_q
 * summed over every admitted (q, k); for GQA dK/dV sum over the query heads
 * of the group.  o/lse are the oracle's own forward results.  All arrays in
 * original order; dq [B*Hq][S][D], dk/dv [B*Hkv][S][D].
 */
int orc_bwd(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, double scale,
            const double *q, const double *k, const double *v, const double *o,
            const double *lse, const double *dout, const int32_t *ds_orig,
            const int32_t *lk_orig, double *dq, double *dk, double *dv)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return ORC_EINVAL;
    int64_t g = Hq / Hkv, SD = (int64_t)S * D;
    memset(dq, 0, sizeof(double) * (size_t)((int64_t)B * Hq * SD));
    memset(dk, 0, sizeof(double) * (size_t)((int64_t)B * Hkv * SD));
    memset(dv, 0, sizeof(double) * (size_t)((int64_t)B * Hkv * SD));
    /* one KV head per task: its dK/dV collect over the group's query heads */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bkv = 0; bkv < (int64_t)B * Hkv; ++bkv) {
        int64_t b = bkv / Hkv, hk = bkv % Hkv;
        const double *kh = k + bkv * SD, *vh = v + bkv * SD;
        double *dkh = dk + bkv * SD, *dvh = dv + bkv * SD;
        for (int64_t h = hk * g; h < (hk + 1) * g; ++h) {
            int64_t bh = b * Hq + h;
            for (int64_t qi = 0; qi < S; ++qi) {
                const double *qv = q + (bh * S + qi) * D, *ov = o + (bh * S + qi) * D;
                const double *dov = dout + (bh * S + qi) * D;
                double *dqv = dq + (bh * S + qi) * D;
                double L = lse[bh * S + qi], Dq = 0.0;
                for (int64_t d = 0; d < D; ++d) Dq += dov[d] * ov[d];
                for (int64_t kk = ds_orig[qi]; kk <= lk_orig[qi]; ++kk) {
                    const double *kv = kh + kk * D, *vv = vh + kk * D;
                    double dot = 0.0, dP = 0.0;
                    for (int64_t d = 0; d < D; ++d) { dot += qv[d] * kv[d]; dP += dov[d] * vv[d]; }
                    double P = exp(scale * dot - L);
                    double dS = P * (dP - Dq);
                    for (int64_t d = 0; d < D; ++d) {
                        dvh[kk * D + d] += P * dov[d];
                        dqv[d] += scale * dS * kv[d];
                        dkh[kk * D + d] += scale * dS * qv[d];
                    }
                }
            }
        }
    }
    return ORC_OK;
}

/*
 * dK, dV for selected keys only (keys_sel[i] = bkv*S + k, original k), from the
 * oracle's own forward results o / lse of every row (the arrays orc_fwd
 * writes): the same sum as orc_bwd, restricted to the selected keys,
 *   dV_k = sum_q P_qk dO_q,  dK_k = scale sum_q P_qk (dO_q.v_k - dO_q.O_q) q_q,
 * over the rows q that admit key k, in every query head of the group.  Each row's O and
 * LSE are read, not recomputed, so a key costs O(S D) instead of a forward per
 * row.
 */
int orc_bwd_dkv_keys_fwd(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, double scale,
                         const double *q, const double *k, const double *v, const double *o,
                         const double *lse, const double *dout, const int32_t *ds_orig,
                         const int32_t *lk_orig, int64_t nkeys, const int64_t *keys_sel,
                         double *dk, double *dv)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return ORC_EINVAL;
    int64_t g = Hq / Hkv, SD = (int64_t)S * D;
    for (int64_t i = 0; i < nkeys; ++i)
        if (keys_sel[i] < 0 || keys_sel[i] >= (int64_t)B * Hkv * S) return ORC_EINVAL;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nkeys; ++i) {
        int64_t bkv = keys_sel[i] / S, kk = keys_sel[i] % S;
        int64_t b = bkv / Hkv, hk = bkv % Hkv;
        const double *kv = k + bkv * SD + kk * D, *vv = v + bkv * SD + kk * D;
        double *dkv = dk + i * D, *dvv = dv + i * D;
        for (int64_t d = 0; d < D; ++d) { dkv[d] = 0.0; dvv[d] = 0.0; }
        for (int64_t h = hk * g; h < (hk + 1) * g; ++h) {
            int64_t bh = b * Hq + h;
            for (int64_t qi = 0; qi < S; ++qi) {
                if (!orc_mask(ds_orig, lk_orig, qi, kk)) continue;
                const double *qv = q + (bh * S + qi) * D, *ov = o + (bh * S + qi) * D;
                const double *dov = dout + (bh * S + qi) * D;
                double Dq = 0.0, dot = 0.0, dP = 0.0;
                for (int64_t d = 0; d < D; ++d) {
                    Dq += dov[d] * ov[d];
                    dot += qv[d] * kv[d];
                    dP += dov[d] * vv[d];
                }
                double P = exp(scale * dot - lse[bh * S + qi]);
                double dS = P * (dP - Dq);
                for (int64_t d = 0; d < D; ++d) {
                    dvv[d] += P * dov[d];
                    dkv[d] += scale * dS * qv[d];
                }
            }
        }
    }
    return ORC_OK;
}

/*
 * dQ for selected rows only (rows[i] = bh*S + q), each from its own forward:
 * the row's LSE and O are recomputed by the definition first.
 */
int orc_bwd_dq_rows(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, double scale,
                    const double *q, const double *k, const double *v, const double *dout,
                    const int32_t *ds_orig, const int32_t *lk_orig, int64_t nrows,
                    const int64_t *rows, double *dq)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return ORC_EINVAL;
    int64_t g = Hq / Hkv, SD = (int64_t)S * D;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)S);
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)S);
        double *orow = (double *)malloc(sizeof(double) * (size_t)D);
        for (int64_t t = 0; t < S; ++t) keys[t] = t;
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t bh = rows[i] / S, qi = rows[i] % S;
            int64_t b = bh / Hq, h = bh % Hq, bkv = b * Hkv + h / g;
            const double *qv = q + (bh * S + qi) * D, *dov = dout + (bh * S + qi) * D;
            const double *kh = k + bkv * SD, *vh = v + bkv * SD;
            double L;
            orc_row(D, scale, qv, qi, kh, vh, keys, (int64_t)lk_orig[qi] + 1, ds_orig, lk_orig, sc,
                    orow, &L);
            double Dq = 0.0;
            for (int64_t d = 0; d < D; ++d) Dq += dov[d] * orow[d];
            double *dqv = dq + i * D;
            for (int64_t d = 0; d < D; ++d) dqv[d] = 0.0;
            for (int64_t kk = ds_orig[qi]; kk <= lk_orig[qi]; ++kk) {
                double dot = 0.0, dP = 0.0;
                for (int64_t d = 0; d < D; ++d) { dot += qv[d] * kh[kk * D + d]; dP += dov[d] * vh[kk * D + d]; }
                double P = exp(scale * dot - L);
                double dS = P * (dP - Dq);
                for (int64_t d = 0; d < D; ++d) dqv[d] += scale * dS * kh[kk * D + d];
            }
        }
        free(sc); free(keys); free(orow);
    }
    return ORC_OK;
}

/*
 * dK and dV for selected keys only (keys_sel[i] = bkv*S + k).  Every query row
 * that admits the key (rows k .. end of its document, in every query head of
 * the group) contributes; each such row's LSE and Dq come from its own
 * forward by the definition, computed here.
 */
int orc_bwd_dkv_keys(int32_t B, int32_t Hq, int32_t Hkv, int32_t S, int32_t D, double scale,
                     const double *q, const double *k, const double *v, const double *dout,
                     const int32_t *ds_orig, const int32_t *lk_orig, int64_t nkeys,
                     const int64_t *keys_sel,
                     double *dk, double *dv)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return ORC_EINVAL;
    int64_t g = Hq / Hkv, SD = (int64_t)S * D;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)S);
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)S);
        double *orow = (double *)malloc(sizeof(double) * (size_t)D);
        for (int64_t t = 0; t < S; ++t) keys[t] = t;
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nkeys; ++i) {
            int64_t bkv = keys_sel[i] / S, kk = keys_sel[i] % S;
            int64_t b = bkv / Hkv, hk = bkv % Hkv;
            const double *kh = k + bkv * SD, *vh = v + bkv * SD;
            double *dkv = dk + i * D, *dvv = dv + i * D;
            for (int64_t d = 0; d < D; ++d) { dkv[d] = 0.0; dvv[d] = 0.0; }
            for (int64_t h = hk * g; h < (hk + 1) * g; ++h) {
                int64_t bh = b * Hq + h;
                for (int64_t qi = 0; qi < S; ++qi) {
                    if (!orc_mask(ds_orig, lk_orig, qi, kk)) continue;
                    const double *qv = q + (bh * S + qi) * D, *dov = dout + (bh * S + qi) * D;
                    double L;
                    orc_row(D, scale, qv, qi, kh, vh, keys, (int64_t)lk_orig[qi] + 1, ds_orig,
                            lk_orig, sc, orow, &L);
                    double Dq = 0.0, dot = 0.0, dP = 0.0;
                    for (int64_t d = 0; d < D; ++d) {
                        Dq += dov[d] * orow[d];
                        dot += qv[d] * kh[kk * D + d];
                        dP += dov[d] * vh[kk * D + d];
                    }
                    double P = exp(scale * dot - L);
                    double dS = P * (dP - Dq);
                    for (int64_t d = 0; d < D; ++d) {
                        dvv[d] += P * dov[d];
                        dkv[d] += scale * dS * qv[d];
                    }
                }
            }
        }
        free(sc); free(keys); free(orow);
    }
    return ORC_OK;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
