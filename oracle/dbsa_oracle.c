/*
 * dbsa_oracle.c -- plain, slow, obviously correct CPU oracle for the DBSA
 * attention engine.  TEST INFRASTRUCTURE ONLY: it is loaded by tests/,
 * by __graft_entry__.smoke() and by the cpu_baseline leg of bench.py, and
 * by nothing on the product path.  It shares no code, header, table or
 * constant generator with the CUDA library (many_shot_icl_b200/csrc).
 *
 * Source of truth: the paper-notes page "Efficient Many-Shot In-Context
 * Learning with Dynamic Block-Sparse Attention" (ACL 2025), cited below as
 * [DBSA notes] with the section it falls in:
 *   - §Stage 1 (block-sparse streaming attention encoding), items 1-4
 *   - §Stage 2 (dynamic demonstration selection and answer generation),
 *     items 1-4
 *   - §Configuration parameters (50 demos per block, random grouping,
 *     previous 2 blocks, 30 % retrieval)
 *   - §Ablations › sparse attention patterns (Full / Sink+Prev+Self /
 *     Sink+Self / Self only)
 *
 * Everything is evaluated in fp64 from the exact input values (bf16 or
 * fp32 inputs are handed over as float arrays, which hold them exactly).
 * No blocking, no fusion, no reordering: every output row is computed on
 * its own from its explicit boolean mask row.
 *
 * Readings of points the page leaves open:
 *   - positions are token positions (not demo indices), 0..T-1 in Stage 1
 *     and 0..T'-1 over the gathered tokens in Stage 2;
 *   - query / tail tokens continue after the gathered cache: T' + u;
 *   - RoPE is the rotate-half form, w_i = theta^(-2i/d), no frequency remap;
 *   - softmax scale 1/sqrt(d) unless a scale is given;
 *   - q-head h reads kv-head floor(h / (Hq/Hkv));
 *   - the sink / previous-j / self parts are a set union, clamped at b_1.
 *
 * Parity pins (tests/test_oracle_pins.py) tie every function below to
 * brute force, closed forms, invariants and torch's fp64 SDPA.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Mask patterns of [DBSA notes] §Ablations › sparse attention patterns. */
enum {
    ORC_PATTERN_SINK_PREV_SELF = 0, /* the DBSA pattern (§Stage 1, item 2) */
    ORC_PATTERN_FULL = 1,           /* full causal attention */
    ORC_PATTERN_SINK_SELF = 2,      /* sink + causal self */
    ORC_PATTERN_SELF = 3            /* causal self only */
};

/* ----------------------------------------------------------------------- */
/* [DBSA notes] §Stage 1, item 1: split the n demonstrations into n/k blocks
 * of k demonstrations each.  Output: token offsets offs[0..nb] with
 * offs[0] = 0 and block b covering tokens [offs[b], offs[b+1]).  When k does
 * not divide n, the last block holds the remaining demonstrations.
 * Returns nb, or -1 on bad arguments. */
int32_t orc_group_blocks(const int32_t *demo_len, int32_t n_demos, int32_t k,
                         int32_t *offs)
{
    if (n_demos <= 0 || k <= 0) return -1;
    int32_t nb = (n_demos + k - 1) / k;
    offs[0] = 0;
    for (int32_t b = 0; b < nb; ++b) {
        int64_t total = offs[b];
        for (int32_t m = b * k; m < (b + 1) * k && m < n_demos; ++m) {
            if (demo_len[m] < 1) return -1;
            total += demo_len[m];
        }
        if (total > INT32_MAX) return -1;
        offs[b + 1] = (int32_t)total;
    }
    return nb;
}

/* The block that holds token t: the b with offs[b] <= t < offs[b+1]. */
static int32_t block_of(const int32_t *offs, int32_t nb, int64_t t)
{
    for (int32_t b = 0; b < nb; ++b)
        if (t >= offs[b] && t < offs[b + 1]) return b;
    return -1;
}

/* [DBSA notes] §Stage 1, item 2 (and §Ablations for the other patterns):
 * may the token at position t attend to the token at position s?
 * Blocks are 0-indexed here, so block 0 is the page's b_1 (the sink). */
int32_t orc_stage1_allowed(const int32_t *offs, int32_t nb, int32_t j,
                           int32_t pattern, int64_t t, int64_t s)
{
    if (s > t) return 0; /* causal */
    int32_t bt = block_of(offs, nb, t);
    int32_t bs = block_of(offs, nb, s);
    if (bt < 0 || bs < 0) return 0;
    int is_sink = (bs == 0);
    int is_self = (bs == bt);
    int is_prev = (bs >= bt - j) && (bs < bt);
    switch (pattern) {
    case ORC_PATTERN_SINK_PREV_SELF: return is_sink || is_prev || is_self;
    case ORC_PATTERN_FULL: return 1;
    case ORC_PATTERN_SINK_SELF: return is_sink || is_self;
    case ORC_PATTERN_SELF: return is_self;
    default: return 0;
    }
}

/* Rotary position embedding in the rotate-half form, applied to one
 * d-vector at position pos: for i < d/2, with w_i = theta^(-2i/d),
 *   y_i       = x_i cos(pos w_i) - x_{i+d/2} sin(pos w_i)
 *   y_{i+d/2} = x_{i+d/2} cos(pos w_i) + x_i sin(pos w_i).
 * [DBSA notes] §Stage 1, item 3 (applied at sequential positions) and
 * §Stage 2, item 3 (re-applied at fresh positions). */
void orc_rope(const double *x, int32_t d, double pos, double theta, double *y)
{
    int32_t h = d / 2;
    for (int32_t i = 0; i < h; ++i) {
        double w = pow(theta, -2.0 * (double)i / (double)d);
        double a = pos * w;
        double c = cos(a), s = sin(a);
        y[i] = x[i] * c - x[i + h] * s;
        y[i + h] = x[i + h] * c + x[i] * s;
    }
}

/* Softmax-weighted sum over an explicit key list, in fp64:
 *   z_n = scale * (qr . kr_n), p = softmax(z) (max subtracted), out = sum p_n v_n.
 * kr is [n][d] (already rotated), v is [n][d]. */
static void attend(const double *qr, const double *kr, const double *v,
                   int64_t n, int32_t d, double scale, double *out)
{
    double *z = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double zmax = -INFINITY;
    for (int64_t m = 0; m < n; ++m) {
        double acc = 0.0;
        for (int32_t e = 0; e < d; ++e) acc += qr[e] * kr[m * d + e];
        z[m] = acc * scale;
        if (z[m] > zmax) zmax = z[m];
    }
    double l = 0.0;
    for (int64_t m = 0; m < n; ++m) {
        z[m] = exp(z[m] - zmax);
        l += z[m];
    }
    for (int32_t e = 0; e < d; ++e) out[e] = 0.0;
    for (int64_t m = 0; m < n; ++m)
        for (int32_t e = 0; e < d; ++e) out[e] += (z[m] / l) * v[m * d + e];
    free(z);
}

/* ----------------------------------------------------------------------- */
/* Stage 1 ([DBSA notes] §Stage 1, items 2-3), for an explicit list of output
 * rows (head, token).  Inputs are token-major: q [T][Hq][d], k and v
 * [T][Hkv][d], all pre-RoPE.  For each requested row (h, t):
 *   mask row M[t][s] for every s in [0, T)      (orc_stage1_allowed)
 *   q' = R(t) q_t,  k'_s = R(s) k_s             (orc_rope)
 *   out = softmax over allowed s of scale q'.k'_s, applied to v_s.
 * out is [nrows][d].  scale <= 0 means 1/sqrt(d).  Returns 0, or -1 on a
 * bad argument. */
int32_t orc_stage1_rows(int32_t Hq, int32_t Hkv, int32_t d, double theta,
                        double scale, int32_t j, int32_t pattern,
                        const float *q, const float *k, const float *v,
                        int64_t T, const int32_t *offs, int32_t nb,
                        const int32_t *row_head, const int64_t *row_tok,
                        int64_t nrows, double *out, int32_t nthreads)
{
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || d % 2 != 0) return -1;
    if (offs[0] != 0 || offs[nb] != T) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int32_t g = Hq / Hkv;
    int32_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int32_t h = row_head[r];
        int64_t t = row_tok[r];
        if (h < 0 || h >= Hq || t < 0 || t >= T) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        int32_t c = h / g;
        /* explicit boolean mask row */
        unsigned char *mask = (unsigned char *)malloc((size_t)T);
        int64_t n = 0;
        for (int64_t s = 0; s < T; ++s) {
            mask[s] = (unsigned char)orc_stage1_allowed(offs, nb, j, pattern, t, s);
            n += mask[s];
        }
        double *x = (double *)malloc((size_t)d * sizeof(double));
        double *qr = (double *)malloc((size_t)d * sizeof(double));
        double *kr = (double *)malloc((size_t)(n > 0 ? n : 1) * d * sizeof(double));
        double *vv = (double *)malloc((size_t)(n > 0 ? n : 1) * d * sizeof(double));
        for (int32_t e = 0; e < d; ++e) x[e] = q[(t * Hq + h) * d + e];
        orc_rope(x, d, (double)t, theta, qr);
        int64_t m = 0;
        for (int64_t s = 0; s < T; ++s) {
            if (!mask[s]) continue;
            for (int32_t e = 0; e < d; ++e) x[e] = k[(s * Hkv + c) * d + e];
            orc_rope(x, d, (double)s, theta, kr + m * d);
            for (int32_t e = 0; e < d; ++e) vv[m * d + e] = v[(s * Hkv + c) * d + e];
            ++m;
        }
        attend(qr, kr, vv, n, d, scale, out + r * d);
        free(mask); free(x); free(qr); free(kr); free(vv);
    }
    return bad ? -1 : 0;
}

/* ----------------------------------------------------------------------- */
/* [DBSA notes] §Stage 2, items 2-3: the gathered cache of one query is the
 * concatenation, in the given order, of the token ranges [offs[b],
 * offs[b+1]) of the selected blocks sel[0..m); sel[0] must be the sink
 * (block 0) and no block may repeat.  Gathered token number p (0-based)
 * takes the fresh position p.  If map is not NULL it receives, per gathered
 * token, the pair (cache row, fresh position).  Returns T' (the number of
 * gathered tokens) or -1 if the selection is invalid. */
int64_t orc_stage2_gather_map(const int32_t *offs, int32_t nb,
                              const int32_t *sel, int32_t m, int32_t *map)
{
    if (m < 1 || sel[0] != 0) return -1;
    for (int32_t a = 0; a < m; ++a) {
        if (sel[a] < 0 || sel[a] >= nb) return -1;
        for (int32_t b = 0; b < a; ++b)
            if (sel[b] == sel[a]) return -1;
    }
    int64_t p = 0;
    for (int32_t a = 0; a < m; ++a) {
        for (int64_t s = offs[sel[a]]; s < offs[sel[a] + 1]; ++s) {
            if (map) {
                map[2 * p] = (int32_t)s;
                map[2 * p + 1] = (int32_t)p;
            }
            ++p;
        }
    }
    return p;
}

/* Stage 2 ([DBSA notes] §Stage 2, items 3-4) for one query and an explicit
 * list of output rows (h, u).
 *   kc, vc      : pre-RoPE cache, head-major [Hkv][cap][d]
 *   q_new       : the n_new newest query tokens, [n_new][Hq][d], pre-RoPE
 *   k_tail/v_tail: the query's own tokens so far, [tail_len][Hkv][d],
 *                 pre-RoPE; the last n_new of them belong to q_new.
 * Row (h, u) is query token u, i.e. tail token tu = tail_len - n_new + u at
 * position T' + tu.  Its keys are every gathered token (cache row from the
 * gather map, rotated at its fresh position) and the tail tokens u' <= tu
 * (rotated at T' + u').  out is [nrows][d].  Returns 0 or -1. */
int32_t orc_stage2_rows(int32_t Hq, int32_t Hkv, int32_t d, double theta,
                        double scale, const float *kc, const float *vc,
                        int64_t cap, const int32_t *offs, int32_t nb,
                        const int32_t *sel, int32_t m, const float *q_new,
                        int32_t n_new, const float *k_tail,
                        const float *v_tail, int32_t tail_len,
                        const int32_t *row_head, const int32_t *row_u,
                        int32_t nrows, double *out, int32_t nthreads)
{
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || d % 2 != 0) return -1;
    if (n_new < 1 || tail_len < n_new || offs[nb] > cap) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int32_t g = Hq / Hkv;
    int64_t Tg = orc_stage2_gather_map(offs, nb, sel, m, NULL);
    if (Tg < 0) return -1;
    int32_t *map = (int32_t *)malloc((size_t)(Tg > 0 ? Tg : 1) * 2 * sizeof(int32_t));
    orc_stage2_gather_map(offs, nb, sel, m, map);
    int32_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int32_t r = 0; r < nrows; ++r) {
        int32_t h = row_head[r], u = row_u[r];
        if (h < 0 || h >= Hq || u < 0 || u >= n_new) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        int32_t c = h / g;
        int32_t tu = tail_len - n_new + u;
        int64_t n = Tg + tu + 1; /* explicit key list: gathered ++ tail[0..tu] */
        double *x = (double *)malloc((size_t)d * sizeof(double));
        double *qr = (double *)malloc((size_t)d * sizeof(double));
        double *kr = (double *)malloc((size_t)n * d * sizeof(double));
        double *vv = (double *)malloc((size_t)n * d * sizeof(double));
        for (int32_t e = 0; e < d; ++e) x[e] = q_new[((int64_t)u * Hq + h) * d + e];
        orc_rope(x, d, (double)(Tg + tu), theta, qr);
        for (int64_t p = 0; p < Tg; ++p) {
            int64_t row = map[2 * p];
            for (int32_t e = 0; e < d; ++e) x[e] = kc[((int64_t)c * cap + row) * d + e];
            orc_rope(x, d, (double)map[2 * p + 1], theta, kr + p * d);
            for (int32_t e = 0; e < d; ++e) vv[p * d + e] = vc[((int64_t)c * cap + row) * d + e];
        }
        for (int32_t w = 0; w <= tu; ++w) {
            int64_t p = Tg + w;
            for (int32_t e = 0; e < d; ++e) x[e] = k_tail[((int64_t)w * Hkv + c) * d + e];
            orc_rope(x, d, (double)(Tg + w), theta, kr + p * d);
            for (int32_t e = 0; e < d; ++e) vv[p * d + e] = v_tail[((int64_t)w * Hkv + c) * d + e];
        }
        attend(qr, kr, vv, n, d, scale, out + (int64_t)r * d);
        free(x); free(qr); free(kr); free(vv);
    }
    free(map);
    return bad ? -1 : 0;
}

/* Number of allowed keys of every Stage-1 row t, from the explicit mask
 * (used by the pins and to count algorithmic work). cnt is [T]. */
void orc_stage1_allowed_counts(const int32_t *offs, int32_t nb, int32_t j,
                               int32_t pattern, int64_t T, int64_t *cnt)
{
    for (int64_t t = 0; t < T; ++t) {
        int64_t n = 0;
        for (int64_t s = 0; s <= t; ++s) n += orc_stage1_allowed(offs, nb, j, pattern, t, s);
        cnt[t] = n;
    }
}
