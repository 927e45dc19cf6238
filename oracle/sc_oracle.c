/*
 * sc_oracle.c -- plain, slow, CPU reference for the stochastic-computing (SC)
 * bipolar XNOR matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator
 * with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [PAYN]  "Precision As You Need: Stochastic Computing Is a Dense Adaptive
 *           Quantizer" (paper-notes page), key design 1 (the C-hat equation,
 *           C-BSG, Sobol-8 cumulative indicator table K[b,l] = 1[r_l <= b]),
 *           key design 2 (row statistics and thresholds), key design 3
 *           (early termination, cost linear in the stream length).
 *   [VIT]   "scmp_vit" README, section "Why it works" (scale = abs_max_row/127,
 *           enable-signal count over a Sobol prefix).
 *   [KBAND] "feat(mp): per-group (K-band) stream lengths on the contraction
 *           axis", sections "How the banding works", "Guards", "Tooling".
 *
 * Readings taken where the pages leave a step open (the plainest reading the
 * rest of the pages supports):
 *   - Sobol: first dimension, direction numbers v_k = 2^-k, natural
 *     (non-Gray) order; r_l = u_l * 2^p + 1, so a full period of K[b,.]
 *     holds exactly b ones.
 *   - C-BSG: operand A (the row operand) streams K[a, l]; operand B keeps two
 *     enable-gated counters, one advanced on A's ones and one on A's zeros,
 *     and emits K[b, counter].
 *   - Quantisation: s = amax / 127 in IEEE fp32, x = nearbyintf(v / s)
 *     (round half to even), clamped to [-127, 127]; level = x + 2^(p-1).
 *     amax == 0 gives s = 0 and every level 2^(p-1).
 *   - Decode constant q_dec is a parameter (2^(p-1) by default); the decode is
 *     evaluated in long double from the exact integer counts and rounded once
 *     to fp32.
 *   - Rung of a row = number of thresholds tau_k with g~ >= tau_k, where
 *     g~ = g / max over the group (fp32 division); a group max <= 0 gives
 *     g~ = 0.
 *   - Fraction-based fixed MP ("scmp_vit" README, the MP flags): units (rows,
 *     or whole (batch, head) matrices ranked within sets of consecutive
 *     groups) are ordered by their statistic, largest first, ties to the lower
 *     index, NaN counted as -inf; the units of rung k and above are the first
 *     floor(n * T_k + 1/2) of that order, T_k = f_k + ... + f_{K-1} summed in
 *     that order in double (all n for k = 0).
 *   - K-band tilt: raw[b][k] = L_k (1 + t (2b - (B-1)) / (B-1)), floored, the
 *     deficit handed back one unit at a time to the bands with the largest
 *     lost fraction (ties to the lower band); a rung whose tilted maximum
 *     would pass the ceiling stays untilted.
 *
 * Every routine below is written for a reader checking it against the pages,
 * not for speed: the matmul simulates each bitstream bit by bit.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_TABLE 3
#define ORC_ERR_NONFINITE 4

#define ORC_MAX_PREC 8
#define ORC_MAX_PREC_Q (1 << ORC_MAX_PREC)

/* ------------------------------------------------------------------------ */
/* Sobol-8 sequence and the cumulative indicator table  [PAYN key design 1]  */
/* ------------------------------------------------------------------------ */

/* First Sobol dimension: u_l is the XOR of the direction numbers
 * v_k = 2^-k over the set bits k-1 of the point's index.  In natural order
 * the index of point l is l; in Gray-code order (the order in which the
 * Antonov-Saleev recurrence emits the points, one direction number XOR-ed
 * in per step) it is g(l) = l XOR (l >> 1).  Kept as integers scaled by 2^p,
 * so V_k = 2^(p-k).  Output r_l = u_l * 2^p + 1 for l = 0 .. 2^p - 1. */
static void sobol_first_dim(int sc_prec, int gray, int32_t *r_out)
{
    const int Q = 1 << sc_prec;
    int32_t V[ORC_MAX_PREC + 1];
    for (int k = 1; k <= sc_prec; ++k) V[k] = 1 << (sc_prec - k);
    for (int l = 0; l < Q; ++l) {
        const int idx = gray ? (l ^ (l >> 1)) : l;
        int32_t u = 0;
        for (int k = 1; k <= sc_prec; ++k)
            if ((idx >> (k - 1)) & 1) u ^= V[k];
        r_out[l] = u + 1;
    }
}

int orc_sobol_r(int sc_prec, int32_t *r_out)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !r_out) return ORC_ERR_ARG;
    sobol_first_dim(sc_prec, 0, r_out);
    return ORC_OK;
}

/* The same points in Gray-code order. */
int orc_sobol_r_gray(int sc_prec, int32_t *r_out)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !r_out) return ORC_ERR_ARG;
    sobol_first_dim(sc_prec, 1, r_out);
    return ORC_OK;
}

/* K[b][l] = 1[r_l <= b] for levels b = 0 .. 2^p and positions l < 2^p.
 * K is laid out [(2^p + 1) x 2^p], row b. */
/* Seed-bank variants ("scmp_vit" README, the Sobol-seed bank: the default
 * sequence, its antithetic, alternative seeds): the sequence's integer
 * points u_l = r_l - 1 are XOR-ed with a digital shift s (a permutation of
 * the period for s < 2^p), and the antithetic variant takes 1 - u, i.e.
 * r'_l = 2^p - (u_l XOR s); otherwise r'_l = (u_l XOR s) + 1. */
static int sobol_r_variant(int sc_prec, int gray, uint32_t shift, int antithetic, int32_t *r_out)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !r_out) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    if (shift >= (uint32_t)Q) return ORC_ERR_ARG;
    sobol_first_dim(sc_prec, gray, r_out);
    for (int l = 0; l < Q; ++l) {
        const int32_t u = (r_out[l] - 1) ^ (int32_t)shift;
        r_out[l] = antithetic ? Q - u : u + 1;
    }
    return ORC_OK;
}

int orc_sobol_r_variant(int sc_prec, uint32_t shift, int antithetic, int32_t *r_out)
{
    return sobol_r_variant(sc_prec, 0, shift, antithetic, r_out);
}

static int indicator_variant(int sc_prec, int gray, uint32_t shift, int antithetic, uint8_t *K)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !K) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    int32_t r[1 << ORC_MAX_PREC];
    int st = sobol_r_variant(sc_prec, gray, shift, antithetic, r);
    if (st != ORC_OK) return st;
    for (int b = 0; b <= Q; ++b)
        for (int l = 0; l < Q; ++l)
            K[(size_t)b * Q + l] = (uint8_t)(r[l] <= b);
    return ORC_OK;
}

int orc_indicator_variant(int sc_prec, uint32_t shift, int antithetic, uint8_t *K)
{
    return indicator_variant(sc_prec, 0, shift, antithetic, K);
}

int orc_indicator(int sc_prec, uint8_t *K)
{
    return indicator_variant(sc_prec, 0, 0, 0, K);
}

/* Indicator table of an arbitrary sequence of integer points u_l in
 * [0, 2^p) (one sequence of a per-index Sobol pool, "scmp_vit" README:
 * the Sobol pool of a contraction width D and precision p): r_l = u_l + 1,
 * K[b][l] = 1[r_l <= b].  The points must be a permutation of [0, 2^p) so
 * that a full period of K[b, .] holds exactly b ones; otherwise
 * ORC_ERR_TABLE. */
int orc_indicator_points(int sc_prec, const int32_t *u, uint8_t *K)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !u || !K) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    char seen[1 << ORC_MAX_PREC];
    memset(seen, 0, sizeof(seen));
    for (int l = 0; l < Q; ++l) {
        if (u[l] < 0 || u[l] >= Q || seen[u[l]]) return ORC_ERR_TABLE;
        seen[u[l]] = 1;
    }
    for (int b = 0; b <= Q; ++b)
        for (int l = 0; l < Q; ++l)
            K[(size_t)b * Q + l] = (uint8_t)(u[l] + 1 <= b);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Symmetric quantisation  [VIT "Why it works"; PAYN flowchart]               */
/* ------------------------------------------------------------------------ */

/* x is [rows x cols] row-major with row stride ld.  axis 0: one scale per
 * row, levels[r][c]; axis 1: one scale per column, levels written transposed
 * as levels[c][r] so that the contraction index is contiguous.
 * Returns ORC_ERR_NONFINITE (and still fills the outputs) when an input is
 * not finite. */
int orc_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld,
                 int axis, int sc_prec, uint8_t *levels, float *scales)
{
    if (!x || !levels || !scales || rows < 0 || cols < 0 || ld < cols) return ORC_ERR_ARG;
    if (sc_prec < 2 || sc_prec > ORC_MAX_PREC || (axis != 0 && axis != 1)) return ORC_ERR_ARG;
    const int half = 1 << (sc_prec - 1);          /* 2^(p-1) */
    const int qmax = half - 1;                    /* 127 for p = 8 */
    const int64_t n_vec = axis == 0 ? rows : cols;   /* one scale per vector */
    const int64_t len = axis == 0 ? cols : rows;
    int status = ORC_OK;
    for (int64_t v = 0; v < n_vec; ++v) {
        float amax = 0.0f;
        for (int64_t e = 0; e < len; ++e) {
            float val = axis == 0 ? x[v * ld + e] : x[e * ld + v];
            if (!isfinite(val)) status = ORC_ERR_NONFINITE;
            float m = fabsf(val);
            if (m > amax) amax = m;
        }
        float s = amax / (float)qmax;             /* IEEE fp32 division */
        scales[v] = s;
        for (int64_t e = 0; e < len; ++e) {
            float val = axis == 0 ? x[v * ld + e] : x[e * ld + v];
            long xi = 0;
            if (s > 0.0f && isfinite(val)) {
                float q = val / s;                /* IEEE fp32 division */
                xi = lrintf(nearbyintf(q));       /* round half to even */
                if (xi > qmax) xi = qmax;
                if (xi < -qmax) xi = -qmax;
            }
            levels[v * len + e] = (uint8_t)(xi + half);
        }
    }
    return status;
}

/* Per-(row, chunk) quantisation [KBAND "Summary": the contraction axis is
 * partitioned into bands of whole quantisation chunks].  x is [rows x cols]
 * row-major with row stride ld and cols = n_chunks * chunk; every chunk of
 * every row is quantised on its own exactly as orc_quantize quantises a row:
 * scales[r][c] = max_{e in chunk c} |x[r][e]| / qmax, levels[r][e].
 * Returns ORC_ERR_NONFINITE (and still fills the outputs) when an input is
 * not finite. */
int orc_quantize_chunked(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t chunk,
                         int sc_prec, uint8_t *levels, float *scales)
{
    if (!x || !levels || !scales || rows < 0 || cols < 1 || ld < cols) return ORC_ERR_ARG;
    if (chunk < 1 || cols % chunk != 0) return ORC_ERR_ARG;
    if (sc_prec < 2 || sc_prec > ORC_MAX_PREC) return ORC_ERR_ARG;
    const int half = 1 << (sc_prec - 1);
    const int qmax = half - 1;
    const int64_t n_chunks = cols / chunk;
    int status = ORC_OK;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < n_chunks; ++c) {
            const float *xc = x + r * ld + c * chunk;
            uint8_t *lc = levels + r * cols + c * chunk;
            float amax = 0.0f;
            for (int64_t e = 0; e < chunk; ++e) {
                if (!isfinite(xc[e])) status = ORC_ERR_NONFINITE;
                float m = fabsf(xc[e]);
                if (m > amax) amax = m;
            }
            float s = amax / (float)qmax;
            scales[r * n_chunks + c] = s;
            for (int64_t e = 0; e < chunk; ++e) {
                long xi = 0;
                if (s > 0.0f && isfinite(xc[e])) {
                    float q = xc[e] / s;
                    xi = lrintf(nearbyintf(q));
                    if (xi > qmax) xi = qmax;
                    if (xi < -qmax) xi = -qmax;
                }
                lc[e] = (uint8_t)(xi + half);
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* Row statistic and rung  [PAYN key design 2]                                */
/* ------------------------------------------------------------------------ */

/* mode 0: g_i = max_j |x_ij| (||Q_i||_inf, ||X_i||_inf);
 * mode 1: g_i = max_j x_ij   (max_j A_ij for the attention map). */
int orc_row_stat(const float *x, int64_t rows, int64_t cols, int64_t ld, int mode, float *stat)
{
    if (!x || !stat || rows < 0 || cols < 1 || (mode != 0 && mode != 1)) return ORC_ERR_ARG;
    for (int64_t i = 0; i < rows; ++i) {
        float g = mode == 0 ? 0.0f : x[i * ld];
        for (int64_t j = 0; j < cols; ++j) {
            float v = x[i * ld + j];
            float m = mode == 0 ? fabsf(v) : v;
            if (m > g) g = m;
        }
        stat[i] = g;
    }
    return ORC_OK;
}

/* Normalise g by its group maximum and threshold.  stat is [batch][rows]; the
 * group is one batch entry.  tau holds n_rungs - 1 thresholds, descending. */
int orc_assign_rungs(const float *stat, int64_t rows, int64_t batch,
                     const float *tau, int n_rungs, int32_t *rung)
{
    if (!stat || !rung || rows < 0 || batch < 0 || n_rungs < 1) return ORC_ERR_ARG;
    if (n_rungs > 1 && !tau) return ORC_ERR_ARG;
    for (int k = 1; k + 1 < n_rungs; ++k)
        if (!(tau[k] <= tau[k - 1])) return ORC_ERR_ARG;
    for (int64_t g = 0; g < batch; ++g) {
        const float *s = stat + g * rows;
        float gmax = 0.0f;
        int have = 0;
        for (int64_t i = 0; i < rows; ++i)
            if (!have || s[i] > gmax) { gmax = s[i]; have = 1; }
        for (int64_t i = 0; i < rows; ++i) {
            float gt = gmax > 0.0f ? s[i] / gmax : 0.0f;   /* fp32 division */
            int k = 0;
            for (int t = 0; t + 1 < n_rungs; ++t)
                if (gt >= tau[t]) ++k;
            rung[g * rows + i] = k;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Fraction-based fixed MP  ["scmp_vit" README, MP flags]                     */
/* ------------------------------------------------------------------------ */

/* A unit (a row, or a head's whole matrix) holds level k for a given fraction
 * f_k of the units, the longest level going to the largest statistic.  The
 * number of units at rung k or above is floor(n * T_k + 1/2) with
 * T_k = f_k + f_{k+1} + ... + f_{K-1} (double, summed in that order); rung 0
 * takes every unit. */
static int64_t frac_units_at_or_above(const double *frac, int n_rungs, int k, int64_t n)
{
    if (k == 0) return n;
    double t = 0.0;
    for (int j = k; j < n_rungs; ++j) t += frac[j];
    return (int64_t)floor((double)n * t + 0.5);
}

/* the unit order: statistic descending, NaN counted as -inf, ties by index */
static const float *g_rank_keys;
static int cmp_rank(const void *pa, const void *pb)
{
    const int64_t a = *(const int64_t *)pa, b = *(const int64_t *)pb;
    float va = g_rank_keys[a], vb = g_rank_keys[b];
    if (isnan(va)) va = -INFINITY;
    if (isnan(vb)) vb = -INFINITY;
    if (va > vb) return -1;
    if (va < vb) return 1;
    return a < b ? -1 : (a > b ? 1 : 0);
}

/* Ranks n keys and writes each unit's rung. */
static void frac_rank_rungs(const float *keys, int64_t n, const double *frac, int n_rungs,
                            int32_t *unit_rung)
{
    int64_t *order = (int64_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int64_t));
    for (int64_t i = 0; i < n; ++i) order[i] = i;
    g_rank_keys = keys;
    qsort(order, (size_t)n, sizeof(int64_t), cmp_rank);
    for (int64_t r = 0; r < n; ++r) {
        int k = 0;
        for (int kk = 1; kk < n_rungs; ++kk)
            if (r < frac_units_at_or_above(frac, n_rungs, kk, n)) k = kk;
        unit_rung[order[r]] = k;
    }
    free(order);
}

/* stat is [batch][rows].  set_size == 0: the rows of each batch entry are the
 * units.  set_size > 0: each batch entry is one unit with statistic
 * max_i stat[g][i] (per-head |Q|.amax), ranked within consecutive sets of
 * set_size entries, and all its rows take its rung.  frac[k] is the fraction
 * for rung k (ascending length); each >= 0, summing to 1 within 1e-6. */
int orc_assign_fraction(const float *stat, int64_t rows, int64_t batch, int64_t set_size,
                        const double *frac, int n_rungs, int32_t *rung)
{
    if (!stat || !rung || !frac || rows < 0 || batch < 0 || n_rungs < 1) return ORC_ERR_ARG;
    if (set_size < 0 || (set_size > 0 && batch % set_size != 0)) return ORC_ERR_ARG;
    double sum = 0.0;
    for (int k = 0; k < n_rungs; ++k) {
        if (!(frac[k] >= 0.0)) return ORC_ERR_ARG;
        sum += frac[k];
    }
    if (fabs(sum - 1.0) > 1e-6) return ORC_ERR_ARG;
    if (set_size == 0) {
        for (int64_t g = 0; g < batch; ++g)
            frac_rank_rungs(stat + g * rows, rows, frac, n_rungs, rung + g * rows);
        return ORC_OK;
    }
    float *keys = (float *)malloc((size_t)set_size * sizeof(float));
    int32_t *unit_rung = (int32_t *)malloc((size_t)set_size * sizeof(int32_t));
    for (int64_t s0 = 0; s0 < batch; s0 += set_size) {
        for (int64_t u = 0; u < set_size; ++u) {
            const float *st = stat + (s0 + u) * rows;
            float m = -INFINITY;             /* the head's statistic: max over its rows */
            for (int64_t i = 0; i < rows; ++i)
                if (st[i] > m) m = st[i];
            keys[u] = m;
        }
        frac_rank_rungs(keys, set_size, frac, n_rungs, unit_rung);
        for (int64_t u = 0; u < set_size; ++u)
            for (int64_t i = 0; i < rows; ++i) rung[(s0 + u) * rows + i] = unit_rung[u];
    }
    free(keys);
    free(unit_rung);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* One C-BSG bipolar XNOR count, bit by bit  [PAYN key design 1]             */
/* ------------------------------------------------------------------------ */

/* Streams of length L for levels a (operand A) and b (operand B).  A's bit l
 * is K[a][l].  B's bit is drawn from K[b][.] through one of two enable-gated
 * counters: the one-counter when A's bit is 1, the zero-counter otherwise.
 * Returns the number of positions where the two bits agree (XNOR = 1). */
static int64_t cbsg_count(const uint8_t *KA, const uint8_t *KB, int Q, int a, int b, int L)
{
    const uint8_t *ka = KA + (size_t)a * Q;
    const uint8_t *kb = KB + (size_t)b * Q;
    int n_one = 0, n_zero = 0;
    int64_t agree = 0;
    for (int l = 0; l < L; ++l) {
        int za = ka[l];
        int zb;
        if (za) { zb = kb[n_one]; ++n_one; }
        else    { zb = kb[n_zero]; ++n_zero; }
        agree += 1 - (za ^ zb);
    }
    return agree;
}

/* Unipolar AND mode ("scmp_vit" README, the comp matmul's unipolar quant
 * mode; "Precision As You Need", the AND gate of unipolar SC).  A level v
 * (bipolar code v = x + 2^(p-1)) is read as sign-magnitude: sign(x) and the
 * unipolar stream of magnitude level 2|x| on the same table, i.e.
 * P(1) = |x| / 2^(p-1).  A's bit l is K[2|x_a|][l]; B keeps one enable-gated
 * counter, advanced on A's ones only, and emits K[2|x_b|][counter] there
 * (at A's zeros the AND is 0 whatever B emits).  Returns
 * sign(x_a) sign(x_b) * #{l < L : A_l AND B_l}. */
static int64_t and_count_signed(const uint8_t *KA, const uint8_t *KB, int Q, int a, int b, int L)
{
    const int half = Q / 2;
    const int xa = a - half, xb = b - half;
    const int ma = 2 * (xa < 0 ? -xa : xa), mb = 2 * (xb < 0 ? -xb : xb);
    if (ma > Q || mb > Q) return 0;   /* out of the code range: no stream */
    const uint8_t *ka = KA + (size_t)ma * Q;
    const uint8_t *kb = KB + (size_t)mb * Q;
    int n_one = 0;
    int64_t both = 0;
    for (int l = 0; l < L; ++l) {
        if (ka[l]) {
            both += kb[n_one];
            ++n_one;
        }
    }
    const int sgn = ((xa < 0) != (xb < 0)) ? -1 : 1;
    return sgn * both;
}

int64_t orc_and_count(int sc_prec, int a, int b, int L, int64_t *out)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !out) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    if (a < 0 || a > Q || b < 0 || b > Q || L < 0 || L > Q) return ORC_ERR_ARG;
    uint8_t *K = (uint8_t *)malloc((size_t)(Q + 1) * Q);
    if (!K) return ORC_ERR_ARG;
    orc_indicator(sc_prec, K);
    *out = and_count_signed(K, K, Q, a, b, L);
    free(K);
    return ORC_OK;
}

int64_t orc_cbsg_count(int sc_prec, int a, int b, int L)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC) return -1;
    const int Q = 1 << sc_prec;
    if (a < 0 || a > Q || b < 0 || b > Q || L < 0 || L > Q) return -1;
    uint8_t *K = (uint8_t *)malloc((size_t)(Q + 1) * Q);
    if (!K) return -1;
    orc_indicator(sc_prec, K);
    int64_t c = cbsg_count(K, K, Q, a, b, L);
    free(K);
    return c;
}

/* Bit-by-bit counts for every level pair at one stream length:
 * out[a * (2^p + 1) + b] for a, b = 0 .. 2^p. */
int orc_cbsg_table(int sc_prec, int L, int32_t *out)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !out) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    if (L < 0 || L > Q) return ORC_ERR_ARG;
    uint8_t *K = (uint8_t *)malloc((size_t)(Q + 1) * Q);
    if (!K) return ORC_ERR_ARG;
    orc_indicator(sc_prec, K);
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int a = 0; a <= Q; ++a)
        for (int b = 0; b <= Q; ++b)
            out[(size_t)a * (Q + 1) + b] = (int32_t)cbsg_count(K, K, Q, a, b, L);
    free(K);
    return ORC_OK;
}

/* The bit streams themselves, for inspection: za[l], zb[l] for l < L. */
int orc_cbsg_streams(int sc_prec, int a, int b, int L, uint8_t *za, uint8_t *zb)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC || !za || !zb) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    if (a < 0 || a > Q || b < 0 || b > Q || L < 0 || L > Q) return ORC_ERR_ARG;
    uint8_t *K = (uint8_t *)malloc((size_t)(Q + 1) * Q);
    if (!K) return ORC_ERR_ARG;
    orc_indicator(sc_prec, K);
    int n_one = 0, n_zero = 0;
    for (int l = 0; l < L; ++l) {
        za[l] = K[(size_t)a * Q + l];
        if (za[l]) zb[l] = K[(size_t)b * Q + n_one++];
        else       zb[l] = K[(size_t)b * Q + n_zero++];
    }
    free(K);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* The SC matmul, bit by bit, with the decode  [PAYN key designs 1 and 3;     */
/* KBAND "How the banding works"]                                            */
/* ------------------------------------------------------------------------ */

/* Problem: `batch` independent groups; per group A levels [M x D], B levels
 * [N x D] (contraction index contiguous), scales a_s [M], b_s [N], rung [M].
 * Without bands row i runs at L = ladder[rung_i] over all of D.  With bands
 * (band_len != NULL) D = n_bands * chunk_d and contraction index d lies in
 * band d / chunk_d, which runs at band_len[band * n_rungs + rung_i].
 *
 * sel: n_sel triples (g, i, j); when sel is NULL every output is computed and
 * n_sel must be batch*M*N (outputs then in [g][i][j] order).
 * counts: [n_sel][n_bands_eff] agreement counts (n_bands_eff = 1 without
 * bands).  out: [n_sel] fp32 decode.  steps: total simulated XNORs.
 *
 * Decode: C_ij = s_i s_j q_dec^2 * sum_bands (2 count_b / L_b - D_b), in long
 * double, rounded once to fp32.  With band_scales (bands of whole
 * quantisation chunks, one chunk per band) a_s is [batch][M][n_bands] and
 * b_s [batch][N][n_bands] and every band carries its own scales:
 * C_ij = q_dec^2 * sum_bands s_ib s_jb (2 count_b / L_b - D_b).
 * b_shift / b_antithetic select a seed-bank variant of the second operand's
 * sequence (orc_sobol_r_variant); the first operand keeps the default.
 * gray: the first Sobol dimension in Gray-code order for both operands.
 * pool (n_pool sequences of 2^p integer points each, a per-index Sobol pool,
 * "scmp_vit" README: one pool per contraction width and precision):
 * contraction index d streams both of its operands from sequence
 * d mod n_pool; each sequence must be a permutation of [0, 2^p).  A pool
 * excludes gray and the seed-bank variants. */
static int matmul_impl(int sc_prec, double q_dec,
                       int64_t batch, int64_t M, int64_t N, int64_t D,
                       const uint8_t *a_lv, const float *a_s,
                       const uint8_t *b_lv, const float *b_s,
                       const int32_t *rung, const int32_t *ladder, int n_rungs,
                       const int32_t *band_len, int n_bands, int64_t chunk_d,
                       int64_t n_sel, const int64_t *sel,
                       int32_t *counts, float *out, int64_t *steps, int n_threads,
                       int band_scales, int unipolar, uint32_t b_shift, int b_antithetic,
                       int gray, const int32_t *pool, int n_pool, int memo)
{
    if (sc_prec < 1 || sc_prec > ORC_MAX_PREC) return ORC_ERR_ARG;
    if (batch < 0 || M < 0 || N < 0 || D < 1 || n_rungs < 1 || !ladder) return ORC_ERR_ARG;
    if (!a_lv || !a_s || !b_lv || !b_s || !rung || !out) return ORC_ERR_ARG;
    const int Q = 1 << sc_prec;
    for (int k = 0; k < n_rungs; ++k)
        if (ladder[k] < 1 || ladder[k] > Q) return ORC_ERR_TABLE;
    int nb = 1;
    if (band_len) {
        if (n_bands < 1 || n_bands > 64 || chunk_d < 1 || (int64_t)n_bands * chunk_d != D)
            return ORC_ERR_TABLE;
        for (int i = 0; i < n_bands * n_rungs; ++i)
            if (band_len[i] < 1 || band_len[i] > Q) return ORC_ERR_TABLE;
        nb = n_bands;
    }
    if (band_scales && !band_len) return ORC_ERR_ARG;
    if (!sel && n_sel != batch * M * N) return ORC_ERR_ARG;
    if (pool && (n_pool < 1 || gray || b_shift || b_antithetic)) return ORC_ERR_ARG;

    /* Streams: without a pool one sequence for every contraction index (the
     * first Sobol dimension in natural or Gray-code order; B may take a
     * seed-bank variant of it).  With a pool of n_pool sequences, index d
     * streams both operands from sequence d mod n_pool. */
    const int nK = pool ? n_pool : 1;
    uint8_t **KA = (uint8_t **)calloc((size_t)nK, sizeof(uint8_t *));
    uint8_t **KB = (uint8_t **)calloc((size_t)nK, sizeof(uint8_t *));
    int table_bad = !KA || !KB;
    for (int q = 0; q < nK && !table_bad; ++q) {
        KA[q] = (uint8_t *)malloc((size_t)(Q + 1) * Q);
        if (!KA[q]) { table_bad = ORC_ERR_ARG; break; }
        if (pool) {
            const int st = orc_indicator_points(sc_prec, pool + (size_t)q * Q, KA[q]);
            if (st != ORC_OK) { table_bad = st; break; }
            KB[q] = KA[q];
        } else {
            indicator_variant(sc_prec, gray, 0, 0, KA[q]);
            KB[q] = KA[q];
            if (b_shift || b_antithetic) {
                KB[q] = (uint8_t *)malloc((size_t)(Q + 1) * Q);
                if (!KB[q] || indicator_variant(sc_prec, gray, b_shift, b_antithetic, KB[q]) != ORC_OK) {
                    table_bad = ORC_ERR_ARG;
                    break;
                }
            }
        }
    }
    if (table_bad) {
        for (int q = 0; KA && KB && q < nK; ++q) {
            if (KB[q] && KB[q] != KA[q]) free(KB[q]);
            free(KA[q]);
        }
        free(KA);
        free(KB);
        return table_bad == ORC_ERR_TABLE ? ORC_ERR_TABLE : ORC_ERR_ARG;
    }

    /* memo: the count of every level pair (a, b) for every (sequence, length)
     * in use, each one simulated bit by bit by the same routine the loop
     * below calls; a count depends on (sequence, a, b, L) only, so a table
     * entry stands for the simulation of that quadruple. */
    const int W = Q + 1;
    int32_t **memo_tab = NULL;
    int memo_fail = 0;
    if (memo) {
        memo_tab = (int32_t **)calloc((size_t)nK * W, sizeof(int32_t *));
        if (!memo_tab) memo_fail = 1;
        for (int64_t d = 0; d < D && !memo_fail; ++d) {
            const int q = (int)(d % nK);
            const int bb = band_len ? (int)(d / chunk_d) : 0;
            for (int k = 0; k < n_rungs && !memo_fail; ++k) {
                const int L = band_len ? band_len[bb * n_rungs + k] : ladder[k];
                if (memo_tab[(size_t)q * W + L]) continue;
                int32_t *T = (int32_t *)malloc((size_t)W * W * sizeof(int32_t));
                if (!T) { memo_fail = 1; break; }
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
                for (int a = 0; a <= Q; ++a)
                    for (int b = 0; b <= Q; ++b)
                        T[(size_t)a * W + b] = (int32_t)(unipolar ? and_count_signed(KA[q], KB[q], Q, a, b, L)
                                                                  : cbsg_count(KA[q], KB[q], Q, a, b, L));
                memo_tab[(size_t)q * W + L] = T;
            }
        }
    }

    int bad = memo_fail;
    int64_t total_steps = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : total_steps) reduction(| : bad)
#endif
    for (int64_t s = 0; s < n_sel; ++s) {
        int64_t g, i, j;
        if (sel) { g = sel[3 * s]; i = sel[3 * s + 1]; j = sel[3 * s + 2]; }
        else { g = s / (M * N); i = (s / N) % M; j = s % N; }
        if (g < 0 || g >= batch || i < 0 || i >= M || j < 0 || j >= N) { bad = 1; continue; }
        const uint8_t *ar = a_lv + (g * M + i) * D;
        const uint8_t *br = b_lv + (g * N + j) * D;
        const int k = rung[g * M + i];
        if (k < 0 || k >= n_rungs) { bad = 1; continue; }
        int64_t cnt[64];
        int64_t len[64];
        int64_t dlen[64];
        for (int bb = 0; bb < nb; ++bb) {
            cnt[bb] = 0;
            len[bb] = band_len ? band_len[bb * n_rungs + k] : ladder[k];
            dlen[bb] = band_len ? chunk_d : D;
        }
        for (int64_t d = 0; d < D; ++d) {
            const int bb = band_len ? (int)(d / chunk_d) : 0;
            const int L = (int)len[bb];
            const int q = (int)(d % nK);
            const int a = ar[d], b = br[d];
            if (a > Q || b > Q) { bad = 1; continue; }
            if (memo) {
                const int32_t *T = memo_tab ? memo_tab[(size_t)q * W + L] : NULL;
                if (!T) { bad = 1; continue; }
                cnt[bb] += T[(size_t)a * W + b];
            } else {
                cnt[bb] += unipolar ? and_count_signed(KA[q], KB[q], Q, a, b, L)
                                    : cbsg_count(KA[q], KB[q], Q, a, b, L);
            }
            total_steps += L;
        }
        long double acc = 0.0L;
        for (int bb = 0; bb < nb; ++bb) {
            if (counts) counts[s * nb + bb] = (int32_t)cnt[bb];
            /* bipolar: 2 count / L - D (XNOR agreement); unipolar: the signed
             * AND count over L estimates sum_d |x_a x_b| / 2^(2(p-1)) */
            long double term = unipolar
                ? (long double)cnt[bb] / (long double)len[bb]
                : 2.0L * (long double)cnt[bb] / (long double)len[bb] - (long double)dlen[bb];
            if (band_scales)
                term *= (long double)a_s[(g * M + i) * nb + bb] * (long double)b_s[(g * N + j) * nb + bb];
            acc += term;
        }
        long double v;
        if (band_scales)
            v = (long double)q_dec * (long double)q_dec * acc;
        else
            v = (long double)a_s[g * M + i] * (long double)b_s[g * N + j]
                * (long double)q_dec * (long double)q_dec * acc;
        out[s] = (float)v;
    }
    if (memo_tab) {
        for (size_t e = 0; e < (size_t)nK * W; ++e) free(memo_tab[e]);
        free(memo_tab);
    }
    for (int q = 0; q < nK; ++q) {
        if (KB[q] != KA[q]) free(KB[q]);
        free(KA[q]);
    }
    free(KA);
    free(KB);
    if (steps) *steps = total_steps;
    return bad ? ORC_ERR_ARG : ORC_OK;
}

int orc_matmul(int sc_prec, double q_dec,
               int64_t batch, int64_t M, int64_t N, int64_t D,
               const uint8_t *a_lv, const float *a_s,
               const uint8_t *b_lv, const float *b_s,
               const int32_t *rung, const int32_t *ladder, int n_rungs,
               const int32_t *band_len, int n_bands, int64_t chunk_d,
               int64_t n_sel, const int64_t *sel,
               int32_t *counts, float *out, int64_t *steps, int n_threads, int band_scales,
               int unipolar, uint32_t b_shift, int b_antithetic, int gray, const int32_t *pool,
               int n_pool)
{
    return matmul_impl(sc_prec, q_dec, batch, M, N, D, a_lv, a_s, b_lv, b_s, rung, ladder,
                       n_rungs, band_len, n_bands, chunk_d, n_sel, sel, counts, out, steps,
                       n_threads, band_scales, unipolar, b_shift, b_antithetic, gray, pool, n_pool,
                       0);
}

/* orc_matmul with every count read from a table of the bit-by-bit counts of
 * all level pairs at each length in use (filled before the loop by the same
 * stream simulation), so that full-size problems finish in seconds.  Same
 * arguments, outputs and decode as orc_matmul; the tests pin the two equal. */
int orc_matmul_memo(int sc_prec, double q_dec,
                    int64_t batch, int64_t M, int64_t N, int64_t D,
                    const uint8_t *a_lv, const float *a_s,
                    const uint8_t *b_lv, const float *b_s,
                    const int32_t *rung, const int32_t *ladder, int n_rungs,
                    const int32_t *band_len, int n_bands, int64_t chunk_d,
                    int64_t n_sel, const int64_t *sel,
                    int32_t *counts, float *out, int64_t *steps, int n_threads, int band_scales,
                    int unipolar, uint32_t b_shift, int b_antithetic, int gray,
                    const int32_t *pool, int n_pool)
{
    return matmul_impl(sc_prec, q_dec, batch, M, N, D, a_lv, a_s, b_lv, b_s, rung, ladder,
                       n_rungs, band_len, n_bands, chunk_d, n_sel, sel, counts, out, steps,
                       n_threads, band_scales, unipolar, b_shift, b_antithetic, gray, pool, n_pool,
                       1);
}

/* ------------------------------------------------------------------------ */
/* K-band straight-line tilt  [KBAND "Tooling", "Guards"]                    */
/* ------------------------------------------------------------------------ */

/* out[b * n_rungs + k] = length of rung k in band b.  Each rung keeps the
 * identity sum_b out[b][k] = n_bands * ladder[k].  tilt = 0 gives the parent
 * ladder in every band. */
int orc_kband_tilt(const int32_t *ladder, int n_rungs, int n_bands, double tilt,
                   int ceiling, int32_t *out)
{
    if (!ladder || !out || n_rungs < 1 || n_bands < 1 || ceiling < 1) return ORC_ERR_ARG;
    if (!(tilt > -1.0 && tilt < 1.0)) return ORC_ERR_ARG;
    for (int k = 0; k < n_rungs; ++k)
        if (ladder[k] < 1 || ladder[k] > ceiling) return ORC_ERR_TABLE;
    for (int k = 0; k < n_rungs; ++k) {
        const int64_t Lk = ladder[k];
        const int64_t target = (int64_t)n_bands * Lk;
        double raw[64];
        if (n_bands > 64) return ORC_ERR_ARG;
        double top = 0.0;
        for (int b = 0; b < n_bands; ++b) {
            double pos = n_bands > 1 ? (2.0 * b - (n_bands - 1)) / (double)(n_bands - 1) : 0.0;
            raw[b] = (double)Lk * (1.0 + tilt * pos);
            if (raw[b] > top) top = raw[b];
        }
        if (top > (double)ceiling) {           /* this rung cannot be tilted */
            for (int b = 0; b < n_bands; ++b) out[b * n_rungs + k] = (int32_t)Lk;
            continue;
        }
        int64_t sum = 0;
        double frac[64];
        for (int b = 0; b < n_bands; ++b) {
            double f = floor(raw[b]);
            out[b * n_rungs + k] = (int32_t)f;
            frac[b] = raw[b] - f;
            sum += (int64_t)f;
        }
        int64_t deficit = target - sum;        /* never negative: floors */
        int used[64] = {0};
        for (int64_t u = 0; u < deficit; ++u) {
            int best = -1;
            for (int b = 0; b < n_bands; ++b) {
                if (used[b]) continue;
                if (best < 0 || frac[b] > frac[best]) best = b;
            }
            if (best < 0) return ORC_ERR_TABLE;
            used[best] = 1;
            out[best * n_rungs + k] += 1;
        }
        for (int b = 0; b < n_bands; ++b)
            if (out[b * n_rungs + k] < 1 || out[b * n_rungs + k] > ceiling) return ORC_ERR_TABLE;
    }
    return ORC_OK;
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
