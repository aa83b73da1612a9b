/*
 * Oracle for the absorbed, top-k masked MLA decode step of DeepSeek-V3.2-Exp.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, fp64 statement of
 * what the decode step computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or helper with the CUDA library, and the CUDA library never calls it.
 *
 * Source pages (DeepSeek-V3.2-Exp atlas, inference/model.py rev 87e509a2e5a1):
 *   "Query-key similarity" (decode): the MQA-decode excerpt, model.py 590-606,
 *       S_i = Q~^C_i c^KV^T + Q^R_i k^R^T, times softmax_scale (596-597);
 *   "Softmax": A[b,i,t,s] = exp(S~[b,i,t,s]) / sum_u exp(S~[b,i,t,u]);
 *   "Apply value weights": O_i = O~_i W_UV,i (model.py 606);
 *   the index mask of the decode excerpt: a -inf row with 0 scattered at the
 *       indexer's top-k positions, shared by every head (model.py 601-602).
 *
 * Definition computed, for each batch row b and head h, with
 *   T_b = { topk_idx[b,k] : 0 <= topk_idx[b,k] < end_pos[b] }  (a set: a
 *   repeated index is scattered once, so it counts once):
 *   1. q_lat[c]  = sum_{d<Dn} q_nope[b,h,d] * wkv_b[h, d, c]          (absorb)
 *   2. s[t]      = scale * ( sum_{c<Dl} q_lat[c] * kv[b,t,c]
 *                          + sum_{r<Dr} q_pe[b,h,r] * pe[b,t,r] )   t in T_b
 *   3. w[t]      = exp(s[t] - m) / sum_{u in T_b} exp(s[u] - m),  m = max s
 *      (positions outside T_b carry score -inf, hence weight exactly 0)
 *   4. o_lat[c]  = sum_{t in T_b} w[t] * kv[b,t,c]                   (mix)
 *   5. out[b,h,e]= sum_{c<Dl} o_lat[c] * wkv_b[h, Dn + e, c]         (W_UV)
 *
 * Every product and sum is taken in double precision from the exact values of
 * the inputs: no intermediate is rounded to a narrower type.  Subtracting m in
 * step 3 leaves the exact value unchanged.
 *
 * A row whose T_b is empty has no finite score; this oracle returns out = 0
 * and lse = -inf for it (the pages' torch code would produce NaN there).
 *
 * Layouts (row-major, element strides in brackets):
 *   q_nope [B, H, Dn]      q_pe [B, H, Dr]
 *   kv     [B, S_max, Dl]  pe   [B, S_max, Dr]   (batch row b uses cache slot b)
 *   wkv_b  [H, Dn + Dv, Dl]   rows 0..Dn-1 of a head are W_UK, rows Dn.. W_UV
 *   end_pos [B] int32, topk_idx [B, K] int32
 * Dense inputs are given either as bfloat16 bit patterns (uint16) or as double,
 * selected by `in_bf16`; a bfloat16 value widens to double exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of one input element to double. */
static double load_elem(const void *base, size_t i, int in_bf16)
{
    if (in_bf16) {
        uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return ((const double *)base)[i];
}

/*
 * Sorted list of the distinct selected positions of one batch row.
 * Returns the count; positions are written to `list` (capacity end_pos).
 * `mark` is scratch of at least end_pos bytes.
 */
static int selected_positions(const int32_t *idx_row, int K, int end_pos,
                              unsigned char *mark, int32_t *list)
{
    int n = 0;
    if (end_pos <= 0)
        return 0;
    memset(mark, 0, (size_t)end_pos);
    for (int k = 0; k < K; ++k) {
        int32_t t = idx_row[k];
        if (t >= 0 && t < end_pos)
            mark[t] = 1;
    }
    for (int t = 0; t < end_pos; ++t)
        if (mark[t])
            list[n++] = t;
    return n;
}

/*
 * The decode step for the batch rows listed in `rows` (n_rows entries; each a
 * batch index in [0, B)).  Output r corresponds to batch row rows[r].
 *
 * Row b reads the cached latents and rotary keys of slot cache_slot[b] when
 * cache_slot is given (kv [n_slots, S_max, Dl], pe [n_slots, S_max, Dr]),
 * else of slot b (n_slots = B).  With one row per query position of a
 * sequence, a slot per sequence and end_pos = s + 1 (the causal bound), this
 * is the "MHA prefill" branch of the page "Queries" (model.py 574-589) in
 * absorbed form: a row whose slot is outside [0, n_slots) has no valid
 * position.
 *
 * Outputs (any optional one may be NULL):
 *   out    [n_rows, H, Dv]      required
 *   lse    [n_rows, H]          log sum_{t in T_b} exp(s[t])  (natural log)
 *   q_lat  [n_rows, H, Dl]      step 1
 *   o_lat  [n_rows, H, Dl]      step 4
 *   w_full [n_rows, H, S_max]   step 3 spread over cache positions: w[t] for
 *                               t in T_b, exactly 0.0 everywhere else
 * Returns 0, or -1 on bad sizes or failed scratch allocation.
 */
int oracle_mla_sparse_decode_f64(
    const void *q_nope, const void *q_pe, const void *kv, const void *pe,
    const void *wkv_b, int in_bf16,
    const int32_t *end_pos, const int32_t *topk_idx, double scale,
    int B, int K, int S_max, int H, int Dn, int Dr, int Dl, int Dv,
    const int32_t *rows, int n_rows, const int32_t *cache_slot, int n_slots,
    double *out, double *lse, double *q_lat, double *o_lat, double *w_full)
{
    if (B < 0 || K < 0 || S_max < 0 || H <= 0 || Dn <= 0 || Dr < 0 ||
        Dl <= 0 || Dv <= 0 || n_rows < 0 || out == NULL)
        return -1;
    for (int r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= B)
            return -1;

    /* Selected set T_b of every requested row (distinct, ascending). */
    int32_t **sel = (int32_t **)calloc((size_t)n_rows + 1, sizeof *sel);
    int *nsel = (int *)calloc((size_t)n_rows + 1, sizeof *nsel);
    unsigned char *mark = (unsigned char *)malloc((size_t)S_max + 1);
    int fail = (sel == NULL || nsel == NULL || mark == NULL);
    for (int r = 0; r < n_rows && !fail; ++r) {
        int b = rows[r];
        int ep = end_pos[b];
        if (ep > S_max)
            ep = S_max; /* positions past the cache do not exist */
        if (cache_slot && (cache_slot[b] < 0 || cache_slot[b] >= n_slots))
            ep = 0;     /* no such sequence: nothing is selected */
        sel[r] = (int32_t *)malloc(sizeof(int32_t) * ((size_t)(ep > 0 ? ep : 0) + 1));
        if (sel[r] == NULL) {
            fail = 1;
            break;
        }
        nsel[r] = selected_positions(topk_idx + (size_t)b * K, K, ep, mark, sel[r]);
    }
    free(mark);

    const int Dqk = Dn + Dv; /* rows of one head in wkv_b */
    if (!fail) {
#pragma omp parallel for collapse(2) schedule(dynamic)
        for (int r = 0; r < n_rows; ++r) {
            for (int h = 0; h < H; ++h) {
                const int b = rows[r];
                const int n = nsel[r];
                const size_t slot = cache_slot ? (size_t)(n > 0 ? cache_slot[b] : 0) : (size_t)b;
                const int32_t *T = sel[r];
                double *ql = (double *)malloc(sizeof(double) * (size_t)Dl);
                double *ol = (double *)malloc(sizeof(double) * (size_t)Dl);
                double *s = (double *)malloc(sizeof(double) * ((size_t)n + 1));
                double *w = (double *)malloc(sizeof(double) * ((size_t)n + 1));
                if (!ql || !ol || !s || !w) {
                    /* leave a recognisable result rather than crash */
                    for (int e = 0; e < Dv; ++e)
                        out[((size_t)r * H + h) * Dv + e] = NAN;
                    free(ql); free(ol); free(s); free(w);
                    continue;
                }

                /* 1. absorb: q_lat[c] = sum_d q_nope[b,h,d] * W_UK[h,d,c] */
                for (int c = 0; c < Dl; ++c)
                    ql[c] = 0.0;
                for (int d = 0; d < Dn; ++d) {
                    double qd = load_elem(q_nope, ((size_t)b * H + h) * Dn + d, in_bf16);
                    size_t wrow = ((size_t)h * Dqk + d) * Dl;
                    for (int c = 0; c < Dl; ++c)
                        ql[c] += qd * load_elem(wkv_b, wrow + c, in_bf16);
                }

                /* 2. scores over the selected positions, scale applied after
                 *    the latent and rotary parts are summed */
                double m = -INFINITY;
                for (int j = 0; j < n; ++j) {
                    int t = T[j];
                    size_t kvrow = (slot * S_max + t) * Dl;
                    size_t perow = (slot * S_max + t) * Dr;
                    double acc_lat = 0.0, acc_rope = 0.0;
                    for (int c = 0; c < Dl; ++c)
                        acc_lat += ql[c] * load_elem(kv, kvrow + c, in_bf16);
                    for (int rr = 0; rr < Dr; ++rr)
                        acc_rope += load_elem(q_pe, ((size_t)b * H + h) * Dr + rr, in_bf16) *
                                    load_elem(pe, perow + rr, in_bf16);
                    s[j] = (acc_lat + acc_rope) * scale;
                    if (s[j] > m)
                        m = s[j];
                }

                /* 3. softmax over T_b (masked positions: exp(-inf) = 0) */
                double denom = 0.0;
                for (int j = 0; j < n; ++j) {
                    w[j] = exp(s[j] - m);
                    denom += w[j];
                }
                for (int j = 0; j < n; ++j)
                    w[j] /= denom;

                /* 4. mix the cached latents */
                for (int c = 0; c < Dl; ++c)
                    ol[c] = 0.0;
                for (int j = 0; j < n; ++j) {
                    size_t kvrow = (slot * S_max + T[j]) * Dl;
                    for (int c = 0; c < Dl; ++c)
                        ol[c] += w[j] * load_elem(kv, kvrow + c, in_bf16);
                }

                /* 5. value-up: out[e] = sum_c o_lat[c] * W_UV[h,e,c] */
                for (int e = 0; e < Dv; ++e) {
                    size_t wrow = ((size_t)h * Dqk + Dn + e) * Dl;
                    double acc = 0.0;
                    for (int c = 0; c < Dl; ++c)
                        acc += ol[c] * load_elem(wkv_b, wrow + c, in_bf16);
                    out[((size_t)r * H + h) * Dv + e] = acc;
                }

                if (lse)
                    lse[(size_t)r * H + h] = (n > 0) ? m + log(denom) : -INFINITY;
                if (q_lat)
                    memcpy(q_lat + ((size_t)r * H + h) * Dl, ql, sizeof(double) * (size_t)Dl);
                if (o_lat)
                    memcpy(o_lat + ((size_t)r * H + h) * Dl, ol, sizeof(double) * (size_t)Dl);
                if (w_full) {
                    double *wf = w_full + ((size_t)r * H + h) * S_max;
                    for (int t = 0; t < S_max; ++t)
                        wf[t] = 0.0;
                    for (int j = 0; j < n; ++j)
                        wf[T[j]] = w[j];
                }
                free(ql); free(ol); free(s); free(w);
            }
        }
    }

    for (int r = 0; r < n_rows; ++r)
        if (sel)
            free(sel[r]);
    free(sel);
    free(nsel);
    return fail ? -1 : 0;
}

/*
 * Output projection (model.py 607-608, atlas page "Attention update"): the
 * head outputs of a row, flattened to n_in = H * Dv values, are projected to
 * the model width by wo (a Linear layer, weight [dim, n_in], no bias on the
 * pages):
 *   delta[b, n] = sum_{k < n_in} x[b, k] * wo[n, k]
 * in double precision from the exact input values.  x [B, n_in], wo
 * [dim, n_in] row-major, given as bfloat16 bit patterns or as double
 * (in_bf16).  Rows `rows[0..n_rows)` of x are computed; result r is row
 * rows[r], written to delta[r * dim .. r * dim + dim).  Returns 0, or -1 for
 * a row index out of range.
 */
int oracle_output_projection_f64(const void *x, const void *wo, int in_bf16, int B, int n_in, int dim,
                                 const int32_t *rows, int n_rows, double *delta)
{
    for (int r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= B)
            return -1;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int n = 0; n < dim; ++n) {
        for (int r = 0; r < n_rows; ++r) {
            const size_t xrow = (size_t)rows[r] * n_in, wrow = (size_t)n * n_in;
            double acc = 0.0;
            for (int k = 0; k < n_in; ++k)
                acc += load_elem(x, xrow + k, in_bf16) * load_elem(wo, wrow + k, in_bf16);
            delta[(size_t)r * dim + n] = acc;
        }
    }
    return 0;
}

/* Number of OpenMP threads the oracle's parallel loop will use. */
int oracle_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
