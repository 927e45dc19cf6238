// sc_api.cu -- host side of the C ABI: validation, table construction, dispatch.
//
// Every entry point validates its arguments before anything is enqueued, so a
// rejected call launches nothing and writes nothing ("feat(mp): per-group
// (K-band) stream lengths on the contraction axis", "Guards": failures must
// surface as errors, never as a wrong number).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>

#include "sc_internal.cuh"

namespace scb {

static thread_local char g_err[512] = "";

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

void clear_error() { g_err[0] = '\0'; }

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n;
}

int max_optin_smem() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    return n;
}

}  // namespace scb

using namespace scb;

#define ARG_FAIL(...)              \
    do {                           \
        set_error(__VA_ARGS__);    \
        return SC_ERR_ARG;         \
    } while (0)
#define TABLE_FAIL(...)            \
    do {                           \
        set_error(__VA_ARGS__);    \
        return SC_ERR_TABLE;       \
    } while (0)

extern "C" const char *sc_last_error(void) { return g_err; }

extern "C" const char *sc_version(void) { return "sc_b200 0.1 (sm_100a)"; }

// ---------------------------------------------------------------------------
// K-band tilt ("Tooling": straight-line tilt, floor, largest-lost-fraction
// first; "Guards": a band length above the ceiling is rejected; the top rung
// cannot be tilted when the parent already sits at the ceiling).
// ---------------------------------------------------------------------------
extern "C" int sc_kband_tilt(const int32_t *ladder, int n_rungs, int n_bands, double tilt,
                             int ceiling, int32_t *out) {
    clear_error();
    if (!ladder || !out) ARG_FAIL("sc_kband_tilt: null pointer");
    if (n_rungs < 1 || n_rungs > SC_MAX_RUNGS) ARG_FAIL("sc_kband_tilt: n_rungs %d", n_rungs);
    if (n_bands < 1 || n_bands > SC_MAX_BANDS) ARG_FAIL("sc_kband_tilt: n_bands %d", n_bands);
    if (!(tilt > -1.0 && tilt < 1.0)) ARG_FAIL("sc_kband_tilt: tilt must lie in (-1, 1)");
    if (ceiling < 1) ARG_FAIL("sc_kband_tilt: ceiling %d", ceiling);
    for (int k = 0; k < n_rungs; ++k)
        if (ladder[k] < 1 || ladder[k] > ceiling)
            TABLE_FAIL("sc_kband_tilt: ladder[%d] = %d outside [1, %d]", k, ladder[k], ceiling);
    std::vector<int32_t> res((size_t)n_bands * n_rungs);
    for (int k = 0; k < n_rungs; ++k) {
        const int64_t Lk = ladder[k];
        std::vector<double> raw(n_bands);
        double hi = -1.0;
        for (int b = 0; b < n_bands; ++b) {
            const double slope = n_bands > 1 ? (2.0 * b - (n_bands - 1)) / (double)(n_bands - 1) : 0.0;
            raw[b] = (double)Lk * (1.0 + tilt * slope);
            hi = std::max(hi, raw[b]);
        }
        if (hi > (double)ceiling) {  // no band can be lengthened: keep the parent
            for (int b = 0; b < n_bands; ++b) res[(size_t)b * n_rungs + k] = (int32_t)Lk;
            continue;
        }
        // floor every band, then return the lost units one at a time
        std::vector<int> order(n_bands);
        std::vector<double> lost(n_bands);
        int64_t spent = 0;
        for (int b = 0; b < n_bands; ++b) {
            const double f = floor(raw[b]);
            res[(size_t)b * n_rungs + k] = (int32_t)f;
            lost[b] = raw[b] - f;
            spent += (int64_t)f;
            order[b] = b;
        }
        std::stable_sort(order.begin(), order.end(),
                         [&](int x, int y) { return lost[x] > lost[y]; });
        const int64_t give = (int64_t)n_bands * Lk - spent;
        if (give < 0 || give > n_bands) TABLE_FAIL("sc_kband_tilt: apportionment failed");
        for (int64_t u = 0; u < give; ++u) res[(size_t)order[u] * n_rungs + k] += 1;
        for (int b = 0; b < n_bands; ++b) {
            const int32_t v = res[(size_t)b * n_rungs + k];
            if (v < 1 || v > ceiling)
                TABLE_FAIL("sc_kband_tilt: band %d rung %d length %d outside [1, %d]", b, k, v,
                           ceiling);
        }
    }
    memcpy(out, res.data(), res.size() * sizeof(int32_t));
    return SC_OK;
}

// ---------------------------------------------------------------------------
// Tables ("Precision As You Need", key design 1)
// ---------------------------------------------------------------------------
static int bit_reverse(int v, int bits) {
    int r = 0;
    for (int i = 0; i < bits; ++i) r |= ((v >> i) & 1) << (bits - 1 - i);
    return r;
}

static void free_table_memory(sc_table *t) {
    void **ptrs[] = {(void **)&t->d_C,    (void **)&t->d_CA,     (void **)&t->d_len,
                     (void **)&t->d_len_idx, (void **)&t->d_Aw,  (void **)&t->d_Ct8,
                     (void **)&t->d_Pk,   (void **)&t->d_pk_off, (void **)&t->d_Pmap,
                     (void **)&t->d_E,    (void **)&t->d_e_off,  (void **)&t->d_Cpool,
                     (void **)&t->d_AwU,  (void **)&t->d_PkU,    (void **)&t->d_pku_off,
                     (void **)&t->d_PmapU, (void **)&t->d_EU,    (void **)&t->d_eu_off,
                     (void **)&t->d_ErowU};
    for (void **p : ptrs) {
        cudaFree(*p);
        *p = nullptr;
    }
}

static int build_table(int sc_prec, const int32_t *ladder, int n_rungs, const int32_t *band_len,
                       int n_bands, int64_t chunk_d, int64_t contraction_d, uint32_t b_shift,
                       int b_antithetic, int order, const int32_t *pool, int n_pool, sc_table **out);

extern "C" int sc_build_table(int sc_prec, const int32_t *ladder, int n_rungs,
                              const int32_t *band_len, int n_bands, int64_t chunk_d,
                              int64_t contraction_d, sc_table **out) {
    return build_table(sc_prec, ladder, n_rungs, band_len, n_bands, chunk_d, contraction_d, 0u, 0,
                       SC_ORDER_NATURAL, nullptr, 0, out);
}

extern "C" int sc_build_table_variant(int sc_prec, const int32_t *ladder, int n_rungs,
                                      const int32_t *band_len, int n_bands, int64_t chunk_d,
                                      int64_t contraction_d, uint32_t b_shift, int b_antithetic,
                                      sc_table **out) {
    return build_table(sc_prec, ladder, n_rungs, band_len, n_bands, chunk_d, contraction_d, b_shift,
                       b_antithetic, SC_ORDER_NATURAL, nullptr, 0, out);
}

extern "C" int sc_build_table_seq(int sc_prec, const int32_t *ladder, int n_rungs,
                                  const int32_t *band_len, int n_bands, int64_t chunk_d,
                                  int64_t contraction_d, int order, const int32_t *pool, int n_pool,
                                  sc_table **out) {
    return build_table(sc_prec, ladder, n_rungs, band_len, n_bands, chunk_d, contraction_d, 0u, 0,
                       order, pool, n_pool, out);
}

static int build_table(int sc_prec, const int32_t *ladder, int n_rungs, const int32_t *band_len,
                       int n_bands, int64_t chunk_d, int64_t contraction_d, uint32_t b_shift,
                       int b_antithetic, int order, const int32_t *pool, int n_pool, sc_table **out) {
    clear_error();
    if (!out) ARG_FAIL("sc_build_table: out is null");
    *out = nullptr;
    if (sc_prec < 2 || sc_prec > SC_MAX_PREC) ARG_FAIL("sc_build_table: sc_prec %d", sc_prec);
    if (b_shift >= (1u << sc_prec))
        ARG_FAIL("sc_build_table: shift %u outside [0, 2^sc_prec)", b_shift);
    if (b_antithetic != 0 && b_antithetic != 1)
        ARG_FAIL("sc_build_table: antithetic %d is not 0 or 1", b_antithetic);
    if (order != SC_ORDER_NATURAL && order != SC_ORDER_GRAY)
        ARG_FAIL("sc_build_table: order %d", order);
    if (pool && (n_pool < 1 || order != SC_ORDER_NATURAL))
        ARG_FAIL("sc_build_table: a pool needs n_pool >= 1 and the natural order");
    if (!pool && n_pool != 0) ARG_FAIL("sc_build_table: n_pool %d without a pool", n_pool);
    if (pool) {  // every sequence a permutation of the period
        const int Qp = 1 << sc_prec;
        std::vector<char> seen(Qp);
        for (int q = 0; q < n_pool; ++q) {
            std::fill(seen.begin(), seen.end(), 0);
            for (int l = 0; l < Qp; ++l) {
                const int32_t u = pool[(size_t)q * Qp + l];
                if (u < 0 || u >= Qp || seen[u])
                    TABLE_FAIL("sc_build_table: pool sequence %d is not a permutation of [0, %d) "
                               "(point %d = %d)", q, Qp, l, u);
                seen[u] = 1;
            }
        }
    }
    if (!ladder) ARG_FAIL("sc_build_table: ladder is null");
    if (n_rungs < 1 || n_rungs > SC_MAX_RUNGS) ARG_FAIL("sc_build_table: n_rungs %d", n_rungs);
    const int Q = 1 << sc_prec;
    for (int k = 0; k < n_rungs; ++k) {
        if (ladder[k] < 1 || ladder[k] > Q)
            TABLE_FAIL("sc_build_table: ladder[%d] = %d outside [1, %d]", k, ladder[k], Q);
        if (k > 0 && ladder[k] <= ladder[k - 1])
            TABLE_FAIL("sc_build_table: ladder is not strictly ascending at %d", k);
    }
    if (band_len) {
        if (n_bands < 1 || n_bands > SC_MAX_BANDS) ARG_FAIL("sc_build_table: n_bands %d", n_bands);
        if (chunk_d < 1) ARG_FAIL("sc_build_table: chunk_d %lld", (long long)chunk_d);
        if (contraction_d != (int64_t)n_bands * chunk_d)
            TABLE_FAIL("sc_build_table: contraction_d %lld != n_bands * chunk_d = %lld",
                       (long long)contraction_d, (long long)n_bands * chunk_d);
        for (int k = 0; k < n_rungs; ++k) {
            int64_t sum = 0;
            for (int b = 0; b < n_bands; ++b) {
                const int32_t v = band_len[(size_t)b * n_rungs + k];
                if (v < 1 || v > Q)
                    TABLE_FAIL("sc_build_table: band %d rung %d length %d above the ceiling %d "
                               "or below 1", b, k, v, Q);
                sum += v;
            }
            if (sum != (int64_t)n_bands * ladder[k])
                TABLE_FAIL("sc_build_table: rung %d breaks the iso-compute identity "
                           "(sum over bands %lld != %d * %d)", k, (long long)sum, n_bands,
                           ladder[k]);
        }
    }

    sc_table *t = new sc_table();
    t->sc_prec = sc_prec;
    t->Q = Q;
    t->n_rungs = n_rungs;
    t->n_bands = band_len ? n_bands : 0;
    t->chunk_d = band_len ? chunk_d : 0;
    t->contraction_d = band_len ? contraction_d : 0;
    for (int k = 0; k < n_rungs; ++k) t->ladder[k] = ladder[k];
    const int nb = band_len ? n_bands : 1;
    std::vector<int32_t> lens((size_t)nb * n_rungs);
    for (int b = 0; b < nb; ++b)
        for (int k = 0; k < n_rungs; ++k)
            lens[(size_t)b * n_rungs + k] = band_len ? band_len[(size_t)b * n_rungs + k] : ladder[k];
    if (band_len) t->band_len = lens;
    t->lengths = lens;
    std::sort(t->lengths.begin(), t->lengths.end());
    t->lengths.erase(std::unique(t->lengths.begin(), t->lengths.end()), t->lengths.end());
    t->len_idx.resize(lens.size());
    for (size_t i = 0; i < lens.size(); ++i)
        t->len_idx[i] = (int32_t)(std::lower_bound(t->lengths.begin(), t->lengths.end(), lens[i]) -
                                  t->lengths.begin());

    // Sobol-8, first dimension: r_l - 1 is the bit reversal of the point's
    // index, l in natural order, l XOR (l >> 1) in Gray-code order (first
    // operand).  The second operand's points u_l = r_l - 1 may be shifted
    // (u XOR s) and mirrored (antithetic: 2^p - u).
    t->b_shift = b_shift;
    t->b_antithetic = b_antithetic;
    t->order = order;
    const bool variant = b_shift != 0 || b_antithetic != 0;
    std::vector<int> rA(Q), r(Q);
    for (int l = 0; l < Q; ++l) {
        const int u = bit_reverse(order == SC_ORDER_GRAY ? (l ^ (l >> 1)) : l, sc_prec);
        rA[l] = u + 1;
        const int us = u ^ (int)b_shift;
        r[l] = b_antithetic ? Q - us : us + 1;
    }
    const int W = Q + 1;
    auto prefix_counts = [&](const std::vector<int> &seq) {
        std::vector<uint16_t> T((size_t)W * W);
        for (int b = 0; b <= Q; ++b) {
            int acc = 0;
            T[(size_t)b * W] = 0;
            for (int n = 1; n <= Q; ++n) {
                acc += seq[n - 1] <= b;
                T[(size_t)b * W + n] = (uint16_t)acc;
            }
        }
        return T;
    };
    const std::vector<uint16_t> C = prefix_counts(r);     // second operand (B)
    const std::vector<uint16_t> CA = variant ? prefix_counts(rA) : C;  // first operand (A)
    // Folded expansions per distinct length: P_L[b, j] = number of the
    // positions m < L at fold distance j = |2m - (L-1)| / 2 with r_m <= b.
    const int nl = (int)t->lengths.size();
    std::vector<int32_t> Aw((size_t)nl * W);
    std::vector<uint8_t> Pk, Pmap((size_t)nl * W * PMAP_STRIDE, 0);
    t->pk_off.resize(nl);
    for (int u = 0; u < nl; ++u) {
        const int L = t->lengths[u];
        const int F = (L + 1) / 2, f16 = (F + 15) & ~15, cpd = f16 / 16;
        // A operand: (w, sign, L - n) of every level
        for (int a = 0; a <= Q; ++a) {
            const int n = CA[(size_t)a * W + L];
            const int lo = std::min(n, L - n);
            const int w = (L - 2 * lo + 1) / 2;  // 0 when 2n == L
            const int neg = 2 * n < L ? 1 : 0;
            Aw[(size_t)u * W + a] = w | (neg << 9) | ((L - n) << 16);
        }
        // B operand: per chunk of 16 folded positions, its stream positions
        // in the order they switch on (ascending threshold r_m)
        t->pk_off[u] = (int64_t)Pk.size();
        Pk.resize(Pk.size() + (size_t)cpd * PK_ROWS * 16, 0);
        uint8_t *tab = &Pk[t->pk_off[u]];
        for (int jc = 0; jc < cpd; ++jc) {
            std::vector<int> pos;
            for (int m = 0; m < L; ++m)
                if (abs(2 * m - (L - 1)) / 2 / 16 == jc) pos.push_back(m);
            std::sort(pos.begin(), pos.end(), [&](int x, int y) { return r[x] < r[y]; });
            if ((int)pos.size() > PK_ROWS - 1) {
                set_error("sc_build_table: internal error (chunk of %d positions)", (int)pos.size());
                delete t;
                return SC_ERR_TABLE;
            }
            uint8_t *ct = tab + (size_t)jc * PK_ROWS * 16;
            for (int c = 1; c < PK_ROWS; ++c) {  // row c: the first c positions on
                memcpy(ct + c * 16, ct + (c - 1) * 16, 16);
                if (c <= (int)pos.size()) ct[c * 16 + abs(2 * pos[c - 1] - (L - 1)) / 2 - 16 * jc] += 1;
            }
            for (int b = 0; b <= Q; ++b) {
                int cls = 0;
                for (int m : pos) cls += r[m] <= b;
                Pmap[((size_t)u * W + b) * PMAP_STRIDE + jc] = (uint8_t)cls;
            }
        }
        // construction check: table row of the class = the folded row itself
        for (int b = 0; b <= Q; ++b) {
            std::vector<int> row(f16, 0);
            for (int m = 0; m < L; ++m) row[abs(2 * m - (L - 1)) / 2] += r[m] <= b;
            for (int j = 0; j < f16; ++j) {
                const int jc = j / 16, cls = Pmap[((size_t)u * W + b) * PMAP_STRIDE + jc];
                if (tab[((size_t)jc * PK_ROWS + cls) * 16 + j % 16] != row[j]) {
                    set_error("sc_build_table: internal error (chunk table of length %d)", L);
                    delete t;
                    return SC_ERR_TABLE;
                }
            }
        }
    }

    // Unipolar AND mode (sign-magnitude streams of magnitude level 2|x|, B
    // drawn by one enable-gated counter at A's ones): the signed count of one
    // (a, b) is sgn_a sgn_b C_B[2|x_b|][n], n = C_A[2|x_a|][L], i.e. the
    // contraction over the L stream positions of the thermometer
    // sgn_a 1[m < n] (A) with sgn_b K_B[2|x_b|, m] (B).  A: (n, sign) per level
    // (no row constant); B: per chunk of 16 positions, 17 classes of each
    // sign (rows c and 17 + c: the first c positions in threshold order on,
    // +1 or -1), the map giving the row for every level; CUDA-core rows: the
    // count table per (sign of a, n) row, E_u[row][b], and the row of every
    // level a.
    std::vector<int32_t> AwU((size_t)nl * W);
    std::vector<uint8_t> PkU, PmapU((size_t)nl * W * PMAP_STRIDE, 0);
    std::vector<uint16_t> EU, ErowU((size_t)nl * 256, 0);
    t->pku_off.resize(nl);
    t->eu_off.resize(nl);
    {
        const int half = Q / 2;
        for (int u = 0; u < nl; ++u) {
            const int L = t->lengths[u];
            const int l16 = (L + 15) & ~15, cpd = l16 / 16;
            for (int a = 0; a <= Q; ++a) {
                const int x = a - half, mag = 2 * std::abs(x);
                const int n = CA[(size_t)std::min(mag, Q) * W + L];
                AwU[(size_t)u * W + a] = n | ((x < 0 ? 1 : 0) << 9);
                if (a <= 255) ErowU[(size_t)u * 256 + a] = (uint16_t)(n + (x < 0 ? L + 1 : 0));
            }
            t->pku_off[u] = (int64_t)PkU.size();
            PkU.resize(PkU.size() + (size_t)cpd * PK_ROWS * 16, 0);
            uint8_t *tab = &PkU[t->pku_off[u]];
            for (int jc = 0; jc < cpd; ++jc) {
                std::vector<int> pos;
                for (int m = 16 * jc; m < std::min(16 * jc + 16, L); ++m) pos.push_back(m);
                std::sort(pos.begin(), pos.end(), [&](int x, int y) { return r[x] < r[y]; });
                uint8_t *ct = tab + (size_t)jc * PK_ROWS * 16;
                for (int c = 1; c <= 16; ++c) {
                    memcpy(ct + c * 16, ct + (c - 1) * 16, 16);
                    memcpy(ct + (17 + c) * 16, ct + (16 + c) * 16, 16);
                    if (c <= (int)pos.size()) {
                        ct[c * 16 + pos[c - 1] - 16 * jc] = 0x01;
                        ct[(17 + c) * 16 + pos[c - 1] - 16 * jc] = 0xFF;
                    }
                }
                for (int b = 0; b <= Q; ++b) {
                    const int x = b - half, mag = std::min(2 * std::abs(x), Q);
                    int cls = 0;
                    for (int m : pos) cls += r[m] <= mag;
                    PmapU[((size_t)u * W + b) * PMAP_STRIDE + jc] = (uint8_t)(cls + (x < 0 ? 17 : 0));
                }
            }
            // construction check: the class row of every level is sgn_b K_B[2|x_b|, m]
            for (int b = 0; b <= Q; ++b) {
                const int x = b - half, mag = std::min(2 * std::abs(x), Q);
                for (int m = 0; m < l16; ++m) {
                    const int want = m < L && r[m] <= mag ? (x < 0 ? 0xFF : 0x01) : 0;
                    const int jc = m / 16, cls = PmapU[((size_t)u * W + b) * PMAP_STRIDE + jc];
                    if (tab[((size_t)jc * PK_ROWS + cls) * 16 + m % 16] != want) {
                        set_error("sc_build_table: internal error (unipolar table of length %d)", L);
                        delete t;
                        return SC_ERR_TABLE;
                    }
                }
            }
            t->eu_off[u] = (int64_t)EU.size();
            EU.resize(EU.size() + (size_t)2 * (L + 1) * 256, 0);
            uint16_t *et = &EU[t->eu_off[u]];
            for (int sa = 0; sa < 2; ++sa)
                for (int n = 0; n <= L; ++n)
                    for (int b = 0; b <= std::min(Q, 255); ++b) {
                        const int x = b - half, mag = std::min(2 * std::abs(x), Q);
                        const int v = (int)C[(size_t)mag * W + n] * ((sa != 0) != (x < 0) ? -1 : 1);
                        et[((size_t)sa * (L + 1) + n) * 256 + b] = (uint16_t)(int16_t)v;
                    }
        }
    }

    // transposed byte copy of C for the CUDA-core small-row path: levels are
    // uint8 so b <= 255, and C[b][n] <= min(b, n) fits a byte
    std::vector<uint8_t> Ct8((size_t)W * 256, 0);
    for (int n = 0; n <= Q; ++n)
        for (int b = 0; b <= std::min(Q, 255); ++b) Ct8[(size_t)n * 256 + b] = (uint8_t)CA[(size_t)b * W + n];

    // count table per length for the CUDA-core leftover-row path:
    // E_L[n][b] = (L - n) + C[b][n] - C[b][L - n], n = C[a][L] in [0, L]
    std::vector<uint16_t> E;
    t->e_off.resize(nl);
    for (int u = 0; u < nl; ++u) {
        const int L = t->lengths[u];
        t->e_off[u] = (int64_t)E.size();
        E.resize(E.size() + (size_t)(L + 1) * 256, 0);
        uint16_t *tab = &E[t->e_off[u]];
        for (int n = 0; n <= L; ++n)
            for (int b = 0; b <= std::min(Q, 255); ++b)
                tab[(size_t)n * 256 + b] =
                    (uint16_t)((L - n) + C[(size_t)b * W + n] - C[(size_t)b * W + (L - n)]);
    }

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        delete t;
        return cuda_fail(e, "sc_build_table: cudaGetDevice");
    }
    t->device = dev;
    struct Up {
        void **dst;
        const void *src;
        size_t bytes;
    } ups[] = {
        {(void **)&t->d_C, C.data(), C.size() * sizeof(uint16_t)},
        {(void **)&t->d_len, lens.data(), lens.size() * sizeof(int32_t)},
        {(void **)&t->d_len_idx, t->len_idx.data(), t->len_idx.size() * sizeof(int32_t)},
        {(void **)&t->d_Aw, Aw.data(), Aw.size() * sizeof(int32_t)},
        {(void **)&t->d_Ct8, Ct8.data(), Ct8.size()},
        {(void **)&t->d_Pk, Pk.data(), Pk.size()},
        {(void **)&t->d_pk_off, t->pk_off.data(), t->pk_off.size() * sizeof(int64_t)},
        {(void **)&t->d_Pmap, Pmap.data(), Pmap.size()},
        {(void **)&t->d_AwU, AwU.data(), AwU.size() * sizeof(int32_t)},
        {(void **)&t->d_PkU, PkU.data(), PkU.size()},
        {(void **)&t->d_pku_off, t->pku_off.data(), t->pku_off.size() * sizeof(int64_t)},
        {(void **)&t->d_PmapU, PmapU.data(), PmapU.size()},
        {(void **)&t->d_EU, EU.data(), EU.size() * sizeof(uint16_t)},
        {(void **)&t->d_eu_off, t->eu_off.data(), t->eu_off.size() * sizeof(int64_t)},
        {(void **)&t->d_ErowU, ErowU.data(), ErowU.size() * sizeof(uint16_t)},
        {(void **)&t->d_E, E.data(), E.size() * sizeof(uint16_t)},
        {(void **)&t->d_e_off, t->e_off.data(), t->e_off.size() * sizeof(int64_t)},
    };
    if (variant) {
        e = cudaMalloc((void **)&t->d_CA, CA.size() * sizeof(uint16_t));
        if (e == cudaSuccess)
            e = cudaMemcpy(t->d_CA, CA.data(), CA.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            free_table_memory(t);
            delete t;
            return cuda_fail(e, "sc_build_table: device upload");
        }
    }
    if (pool) {
        // prefix counts of every pool sequence, levels b <= 255, uint8
        std::vector<uint8_t> Cp((size_t)n_pool * 256 * W, 0);
        for (int q = 0; q < n_pool; ++q) {
            const int32_t *u = pool + (size_t)q * Q;
            for (int b = 0; b <= std::min(Q, 255); ++b) {
                uint8_t *row = &Cp[((size_t)q * 256 + b) * W];
                int acc = 0;
                for (int n = 1; n <= Q; ++n) {
                    acc += u[n - 1] + 1 <= b;
                    row[n] = (uint8_t)acc;
                }
            }
        }
        t->n_pool = n_pool;
        e = cudaMalloc((void **)&t->d_Cpool, Cp.size());
        if (e == cudaSuccess) e = cudaMemcpy(t->d_Cpool, Cp.data(), Cp.size(), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            free_table_memory(t);
            delete t;
            return cuda_fail(e, "sc_build_table: device upload");
        }
    }
    for (auto &u : ups) {
        e = cudaMalloc(u.dst, u.bytes);
        if (e == cudaSuccess) e = cudaMemcpy(*u.dst, u.src, u.bytes, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            free_table_memory(t);
            delete t;
            return cuda_fail(e, "sc_build_table: device upload");
        }
    }
    *out = t;
    return SC_OK;
}

extern "C" int sc_table_destroy(sc_table *t) {
    clear_error();
    if (!t) return SC_OK;
    int cur = 0;
    cudaGetDevice(&cur);
    if (t->device >= 0 && t->device != cur) cudaSetDevice(t->device);
    free_table_memory(t);
    if (t->device >= 0 && t->device != cur) cudaSetDevice(cur);
    delete t;
    return SC_OK;
}

extern "C" int sc_table_info(const sc_table *t, int *sc_prec, int *n_rungs, int *n_bands,
                             int64_t *chunk_d, int64_t *contraction_d) {
    clear_error();
    if (!t) ARG_FAIL("sc_table_info: table is null");
    if (sc_prec) *sc_prec = t->sc_prec;
    if (n_rungs) *n_rungs = t->n_rungs;
    if (n_bands) *n_bands = t->n_bands;
    if (chunk_d) *chunk_d = t->chunk_d;
    if (contraction_d) *contraction_d = t->contraction_d;
    return SC_OK;
}

// ---------------------------------------------------------------------------
// Quantise, assign rows
// ---------------------------------------------------------------------------
extern "C" int sc_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                           int64_t batch_stride, int axis, int sc_prec, int stat_mode,
                           uint8_t *levels, float *scales, float *stat, int32_t *dev_status,
                           void *stream) {
    clear_error();
    if (rows < 0 || cols < 0 || batch < 0) ARG_FAIL("sc_quantize: negative size");
    if (axis != 0 && axis != 1) ARG_FAIL("sc_quantize: axis %d", axis);
    if (sc_prec < 2 || sc_prec > SC_MAX_PREC) ARG_FAIL("sc_quantize: sc_prec %d", sc_prec);
    if (stat_mode != SC_STAT_AMAX && stat_mode != SC_STAT_ROWMAX)
        ARG_FAIL("sc_quantize: stat_mode %d", stat_mode);
    if (stat && axis != 0) ARG_FAIL("sc_quantize: the row statistic needs axis 0");
    if (rows == 0 || cols == 0 || batch == 0) return SC_OK;
    if (!x || !levels || !scales) ARG_FAIL("sc_quantize: null pointer");
    if (ld < cols) ARG_FAIL("sc_quantize: ld %lld < cols %lld", (long long)ld, (long long)cols);
    if (batch > 1 && batch_stride < (rows - 1) * ld + cols)
        ARG_FAIL("sc_quantize: batch_stride %lld overlaps entries", (long long)batch_stride);
    return launch_quantize(x, rows, cols, ld, batch, batch_stride, axis, sc_prec, stat_mode, levels,
                           scales, stat, dev_status, (cudaStream_t)stream);
}

extern "C" int sc_quantize_chunked(const float *x, int64_t rows, int64_t cols, int64_t ld,
                                   int64_t batch, int64_t batch_stride, int64_t chunk, int sc_prec,
                                   int stat_mode, uint8_t *levels, float *scales, float *stat,
                                   int32_t *dev_status, void *stream) {
    clear_error();
    if (rows < 0 || cols < 0 || batch < 0) ARG_FAIL("sc_quantize_chunked: negative size");
    if (chunk < 1) ARG_FAIL("sc_quantize_chunked: chunk %lld", (long long)chunk);
    if (cols % chunk) ARG_FAIL("sc_quantize_chunked: chunk %lld does not divide cols %lld",
                               (long long)chunk, (long long)cols);
    if (sc_prec < 2 || sc_prec > SC_MAX_PREC) ARG_FAIL("sc_quantize_chunked: sc_prec %d", sc_prec);
    if (stat_mode != SC_STAT_AMAX && stat_mode != SC_STAT_ROWMAX)
        ARG_FAIL("sc_quantize_chunked: stat_mode %d", stat_mode);
    if (rows == 0 || cols == 0 || batch == 0) return SC_OK;
    if (!x || !levels || !scales) ARG_FAIL("sc_quantize_chunked: null pointer");
    if (ld < cols) ARG_FAIL("sc_quantize_chunked: ld %lld < cols %lld", (long long)ld, (long long)cols);
    if (batch > 1 && batch_stride < (rows - 1) * ld + cols)
        ARG_FAIL("sc_quantize_chunked: batch_stride %lld overlaps entries", (long long)batch_stride);
    return launch_quantize_chunked(x, rows, cols, ld, batch, batch_stride, chunk, sc_prec, stat_mode,
                                   levels, scales, stat, dev_status, (cudaStream_t)stream);
}

extern "C" int sc_assign_rows(const float *stat, int64_t rows, int64_t batch, const float *tau,
                              int n_rungs, int32_t *rung, int32_t *perm, int32_t *rung_offsets,
                              void *stream) {
    clear_error();
    if (rows < 0 || batch < 0) ARG_FAIL("sc_assign_rows: negative size");
    if (rows > INT32_MAX) ARG_FAIL("sc_assign_rows: rows %lld too large", (long long)rows);
    if (n_rungs < 1 || n_rungs > SC_MAX_RUNGS) ARG_FAIL("sc_assign_rows: n_rungs %d", n_rungs);
    if (n_rungs > 1 && !tau) ARG_FAIL("sc_assign_rows: tau is null");
    for (int k = 0; k + 1 < n_rungs; ++k)
        if (!(tau[k] == tau[k]) || (k > 0 && !(tau[k] <= tau[k - 1])))
            ARG_FAIL("sc_assign_rows: tau must be non-increasing (tau[%d])", k);
    if (batch == 0) return SC_OK;
    if (!rung || !perm || !rung_offsets) ARG_FAIL("sc_assign_rows: null output");
    if (rows > 0 && !stat) ARG_FAIL("sc_assign_rows: stat is null");
    return launch_assign_rows(stat, rows, batch, tau, n_rungs, rung, perm, rung_offsets,
                              (cudaStream_t)stream);
}

extern "C" int sc_assign_fraction(const float *stat, int64_t rows, int64_t batch, int64_t set_size,
                                  const double *fractions, int n_rungs, int32_t *rung,
                                  int32_t *perm, int32_t *rung_offsets, void *stream) {
    clear_error();
    if (rows < 0 || batch < 0) ARG_FAIL("sc_assign_fraction: negative size");
    if (rows > INT32_MAX) ARG_FAIL("sc_assign_fraction: rows %lld too large", (long long)rows);
    if (n_rungs < 1 || n_rungs > SC_MAX_RUNGS) ARG_FAIL("sc_assign_fraction: n_rungs %d", n_rungs);
    if (!fractions) ARG_FAIL("sc_assign_fraction: fractions is null");
    if (set_size < 0 || (set_size > 0 && batch % set_size != 0))
        ARG_FAIL("sc_assign_fraction: set_size %lld must divide batch %lld", (long long)set_size,
                 (long long)batch);
    if (set_size > INT32_MAX) ARG_FAIL("sc_assign_fraction: set_size too large");
    double sum = 0.0;
    for (int k = 0; k < n_rungs; ++k) {
        if (!(fractions[k] >= 0.0) || isinf(fractions[k]))
            ARG_FAIL("sc_assign_fraction: fraction %d is not a finite value >= 0", k);
        sum += fractions[k];
    }
    if (fabs(sum - 1.0) > 1e-6) ARG_FAIL("sc_assign_fraction: fractions sum to %.9g, not 1", sum);
    if (batch == 0) return SC_OK;
    if (!rung || !perm || !rung_offsets) ARG_FAIL("sc_assign_fraction: null output");
    if (rows > 0 && !stat) ARG_FAIL("sc_assign_fraction: stat is null");
    // units at rung k or above: floor(n T_k + 1/2), T_k = f_k + ... + f_{K-1}
    const int64_t n = set_size > 0 ? set_size : rows;
    int32_t n_at[SC_MAX_RUNGS];
    for (int k = 0; k < n_rungs; ++k) {
        if (k == 0) {
            n_at[k] = (int32_t)n;
            continue;
        }
        double t = 0.0;
        for (int j = k; j < n_rungs; ++j) t += fractions[j];
        n_at[k] = (int32_t)floor((double)n * t + 0.5);
    }
    return launch_assign_fraction(stat, rows, batch, set_size, n_at, n_rungs, rung, perm,
                                  rung_offsets, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Matmul
// ---------------------------------------------------------------------------
extern "C" int sc_matmul(const sc_matmul_desc *d, const uint8_t *a_lv, const float *a_s,
                         const uint8_t *b_lv, const float *b_s, const int32_t *rung,
                         const int32_t *perm, const int32_t *rung_offsets, const sc_table *t,
                         float *out, int32_t *counts, int32_t *dev_status, void *stream) {
    clear_error();
    if (!d) ARG_FAIL("sc_matmul: desc is null");
    if (!t) ARG_FAIL("sc_matmul: table is null");
    if (d->M < 0 || d->N < 0 || d->batch < 0 || d->D < 1) ARG_FAIL("sc_matmul: bad sizes");
    if (d->M > INT32_MAX || d->N > INT32_MAX || d->D > INT32_MAX)
        ARG_FAIL("sc_matmul: a size exceeds 2^31 - 1");
    if (d->op != SC_OP_LINEAR && d->op != SC_OP_QK && d->op != SC_OP_AV)
        ARG_FAIL("sc_matmul: op %d", d->op);
    if (d->engine != SC_ENGINE_AUTO && d->engine != SC_ENGINE_GATHER && d->engine != SC_ENGINE_TC)
        ARG_FAIL("sc_matmul: engine %d", d->engine);
    if (!(d->q_dec >= 0.0) || isinf(d->q_dec)) ARG_FAIL("sc_matmul: q_dec must be finite and >= 0");
    if (d->scales != SC_SCALES_ROW && d->scales != SC_SCALES_BAND)
        ARG_FAIL("sc_matmul: scales %d", d->scales);
    if (d->mode != SC_MODE_BIPOLAR && d->mode != SC_MODE_UNIPOLAR) ARG_FAIL("sc_matmul: mode %d", d->mode);
    if (d->workspace_bytes < 0) ARG_FAIL("sc_matmul: workspace_bytes < 0");
    if (reinterpret_cast<uintptr_t>(d->workspace) & 255u)
        ARG_FAIL("sc_matmul: workspace is not 256-byte aligned");
    if (d->scales == SC_SCALES_BAND && t->n_bands == 0)
        ARG_FAIL("sc_matmul: per-band scales need a K-band table");
    if (t->n_bands > 0) {
        if (d->op != SC_OP_LINEAR)
            TABLE_FAIL("sc_matmul: K-band tables apply to linear ops only (QK/AV contract over "
                       "head_dim and have no band dispatch)");
        if (d->D != t->contraction_d)
            TABLE_FAIL("sc_matmul: table priced at width %lld (%d bands x %lld) used with D = %lld",
                       (long long)t->contraction_d, t->n_bands, (long long)t->chunk_d,
                       (long long)d->D);
    }
    // int32 counts: a count never exceeds D * 2^sc_prec
    if ((double)d->D * (double)t->Q > 2147483647.0) ARG_FAIL("sc_matmul: D too large for int32 counts");
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev != t->device)
        TABLE_FAIL("sc_matmul: table lives on device %d, current device is %d", t->device, dev);
    if (d->M == 0 || d->N == 0 || d->batch == 0) return SC_OK;
    if (!a_lv || !a_s || !b_lv || !b_s || !rung || !out) ARG_FAIL("sc_matmul: null pointer");
    const double q = d->q_dec > 0.0 ? d->q_dec : (double)(1 << (t->sc_prec - 1));

    int engine = d->engine;
    if (engine == SC_ENGINE_AUTO) engine = tc_supports(*d, *t) ? SC_ENGINE_TC : SC_ENGINE_GATHER;
    if (engine == SC_ENGINE_TC) {
        if (!tc_supports(*d, *t)) {
            set_error("sc_matmul: the tensor-core engine does not support this problem");
            return SC_ERR_UNSUPPORTED;
        }
        if (!perm || !rung_offsets) ARG_FAIL("sc_matmul: the tensor-core engine needs perm and rung_offsets");
        return launch_tc(*d, q, a_lv, a_s, b_lv, b_s, rung, perm, rung_offsets, *t, out, counts,
                         dev_status, (cudaStream_t)stream);
    }
    return launch_gather(*d, q, a_lv, a_s, b_lv, b_s, rung, *t, out, counts, dev_status,
                         (cudaStream_t)stream);
}

extern "C" int64_t sc_prepare_b_bytes(const sc_matmul_desc *d, const sc_table *t) {
    clear_error();
    if (!d || !t) {
        set_error("sc_prepare_b_bytes: null pointer");
        return -SC_ERR_ARG;
    }
    return tc_prepare_b_bytes(*d, *t);
}

extern "C" int sc_prepare_b(const sc_matmul_desc *d, const uint8_t *b_lv, const sc_table *t,
                            sc_bprep **out, void *stream) {
    clear_error();
    if (!out) ARG_FAIL("sc_prepare_b: out is null");
    *out = nullptr;
    if (!d || !t || !b_lv) ARG_FAIL("sc_prepare_b: null pointer");
    if (d->N < 1 || d->D < 1 || d->batch < 1) ARG_FAIL("sc_prepare_b: bad sizes");
    if (d->N > INT32_MAX || d->D > INT32_MAX) ARG_FAIL("sc_prepare_b: a size exceeds 2^31 - 1");
    if (d->mode != SC_MODE_BIPOLAR && d->mode != SC_MODE_UNIPOLAR) ARG_FAIL("sc_prepare_b: mode %d", d->mode);
    if (t->n_bands > 0 && d->D != t->contraction_d)
        TABLE_FAIL("sc_prepare_b: table priced at width %lld used with D = %lld",
                   (long long)t->contraction_d, (long long)d->D);
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev != t->device)
        TABLE_FAIL("sc_prepare_b: table lives on device %d, current device is %d", t->device, dev);
    return tc_prepare_b(*d, b_lv, *t, out, (cudaStream_t)stream);
}

extern "C" int sc_selftest_wait_limit(int32_t *dev_status, int64_t limit_cycles, void *stream) {
    clear_error();
    if (!dev_status) ARG_FAIL("sc_selftest_wait_limit: dev_status is null");
    if (limit_cycles < 1 || limit_cycles > (int64_t)1 << 34)
        ARG_FAIL("sc_selftest_wait_limit: limit %lld outside [1, 2^34] cycles", (long long)limit_cycles);
    return launch_wait_limit_selftest(dev_status, limit_cycles, (cudaStream_t)stream);
}

extern "C" int sc_bprep_destroy(sc_bprep *prep) {
    clear_error();
    return tc_bprep_destroy(prep);
}

extern "C" int sc_matmul_engine(const sc_matmul_desc *d, const sc_table *t) {
    clear_error();
    if (!d || !t) {
        set_error("sc_matmul_engine: null pointer");
        return -SC_ERR_ARG;
    }
    if (d->engine == SC_ENGINE_GATHER) return SC_ENGINE_GATHER;
    const bool tc = tc_supports(*d, *t);
    if (d->engine == SC_ENGINE_TC) {
        if (tc) return SC_ENGINE_TC;
        set_error("sc_matmul_engine: the tensor-core engine does not support this problem");
        return -SC_ERR_UNSUPPORTED;
    }
    if (d->engine != SC_ENGINE_AUTO) {
        set_error("sc_matmul_engine: engine %d", d->engine);
        return -SC_ERR_ARG;
    }
    return tc ? SC_ENGINE_TC : SC_ENGINE_GATHER;
}

extern "C" int64_t sc_matmul_workspace_bytes(const sc_matmul_desc *d, const sc_table *t) {
    const int e = sc_matmul_engine(d, t);
    if (e < 0) return e;
    return e == SC_ENGINE_TC ? tc_workspace_bytes(*d, *t) : 0;
}

extern "C" int sc_matmul_launches(const sc_matmul_desc *d, const sc_table *t) {
    const int e = sc_matmul_engine(d, t);
    if (e < 0) return e;
    if (d->M == 0 || d->N == 0 || d->batch == 0) return 0;
    return e == SC_ENGINE_TC ? tc_launch_count(*d, *t) : 1;
}
