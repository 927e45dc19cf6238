/*
 * sc.h -- C ABI of the B200 (sm_100a) stochastic-computing bipolar XNOR matmul.
 *
 * The library computes, for every output of C = A * B, the stochastic-computing
 * (SC) estimate described in "Precision As You Need: Stochastic Computing Is a
 * Dense Adaptive Quantizer" (paper-notes page, key design 1, the C-hat
 * equation):
 *
 *     C_ij = s^A_i s^B_j q_dec^2 ( 2/L_i * sum_l sum_d XNOR(z^A_idl, z^B_jdl) - D )
 *
 * where both operands are symmetrically quantised to sc_prec-bit levels
 * ("scmp_vit" README, "Why it works": scale = abs_max / 127), each level b
 * selects its bitstream from the Sobol-8 cumulative indicator table
 * K[b,l] = 1[r_l <= b], the second operand's stream is generated conditionally
 * on the first (C-BSG), and row i runs for L_i bits, its length chosen from a
 * ladder by thresholding a normalised row statistic (key design 2) with early
 * termination (key design 3).  Optionally the contraction axis is split into
 * bands that run each rung at its own length ("feat(mp): per-group (K-band)
 * stream lengths on the contraction axis", "How the banding works").
 *
 * Conventions for every entry point:
 *   - Pointers marked (device) are device memory owned by the caller; pointers
 *     marked (host) are host memory owned by the caller and only read during
 *     the call.  The library keeps no reference to caller memory after return.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Work is enqueued asynchronously; nothing synchronises the host
 *     except sc_build_table / sc_table_destroy (which allocate / free).
 *   - Arguments are validated on the host before anything is enqueued.  On an
 *     error no kernel is launched and nothing is written.
 *   - Return value: an SC_* status.  sc_last_error() gives a message for the
 *     last failing call on the calling thread.
 *   - Problems found on the device (a non-finite input, a level outside the
 *     table) are OR-ed into *dev_status (device int32, caller-owned, caller
 *     zeroes it); read it after synchronising.  Kernels never trap.
 *   - Layouts are dense row-major; "levels" are uint8 with the contraction
 *     index contiguous.
 *   - The library runs on the device that is current when it is called.
 */
#ifndef SC_B200_H
#define SC_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define SC_OK 0
#define SC_ERR_ARG 1          /* bad pointer, size, enum or unsorted threshold      */
#define SC_ERR_UNSUPPORTED 2  /* valid request the library does not implement       */
#define SC_ERR_TABLE 3        /* table / band / ceiling / width mismatch             */
#define SC_ERR_NONFINITE 4    /* reported through dev_status (SC_DEV_NONFINITE)      */
#define SC_ERR_CUDA 5         /* a CUDA runtime call failed                          */

/* bits OR-ed into *dev_status by kernels */
#define SC_DEV_NONFINITE 0x1   /* an input value was NaN or infinite                 */
#define SC_DEV_LEVEL_RANGE 0x2 /* a level was above 2^sc_prec (clamped; output unspecified) */
#define SC_DEV_WAIT_LIMIT 0x4  /* an internal bounded wait gave up (kernel returned) */

/* row statistic g_i ("Precision As You Need", key design 2) */
#define SC_STAT_AMAX 0    /* g_i = max_j |x_ij|  (||Q_i||_inf, ||X_i||_inf)       */
#define SC_STAT_ROWMAX 1  /* g_i = max_j x_ij    (max_j A_ij of an attention map) */

/* operator kind; K-band tables are rejected on QK and AV ("Guards") */
#define SC_OP_LINEAR 0
#define SC_OP_QK 1
#define SC_OP_AV 2

/* quantisation scales the decode applies (sc_matmul_desc.scales) */
#define SC_SCALES_ROW 0   /* one scale per row of A and per row/column of B     */
#define SC_SCALES_BAND 1  /* one scale per (row, band): bands are whole
                           * quantisation chunks ("feat(mp) ... K-band",
                           * "Summary"); needs a K-band table               */

/* stream arithmetic (sc_matmul_desc.mode) */
#define SC_MODE_BIPOLAR 0   /* bipolar XNOR with the two-counter C-BSG            */
#define SC_MODE_UNIPOLAR 1  /* unipolar AND of sign-magnitude streams ("scmp_vit"
                             * README, the comp matmul's unipolar quant mode):
                             * level v = x + 2^(p-1) streams magnitude level
                             * 2|x|, B keeps one enable-gated counter advanced
                             * at A's ones; counts are signed, and
                             * out = s^A s^B q_dec^2 sum_b count_b / L_b.  The
                             * CUDA-core engine only (the tensor-core engine
                             * reports SC_ERR_UNSUPPORTED).                      */

/* count engine */
#define SC_ENGINE_AUTO 0    /* library choice                                      */
#define SC_ENGINE_GATHER 1  /* CUDA cores: prefix-count table gathers              */
#define SC_ENGINE_TC 2      /* tcgen05 int8 tensor cores: exact folded contraction  */

#define SC_MAX_PREC 8
#define SC_MAX_RUNGS 8
#define SC_MAX_BANDS 64

typedef struct sc_table sc_table; /* opaque, library-owned, device-resident */
typedef struct sc_bprep sc_bprep; /* opaque: a static second operand prepared for the
                                   * tensor-core engine (sc_prepare_b)             */

/* Problem description for sc_matmul.  Per group g (0 <= g < batch):
 *   A levels  a_lv[g][M][D], scales a_s[g][M], rungs rung[g][M]
 *   B levels  b_lv[g][N][D], scales b_s[g][N]
 *   output    out[g][M][N] (fp32)
 * With scales == SC_SCALES_BAND the scales are a_s[g][M][n_bands] and
 * b_s[g][N][n_bands] (n_bands of the table).
 * The product is C = A * B^T over the level matrices as laid out above, i.e.
 * B is supplied with its contraction index contiguous. */
typedef struct sc_matmul_desc {
    int64_t M, N, D;  /* per-group sizes; M, N >= 0, D >= 1                    */
    int64_t batch;    /* number of independent groups, >= 0                    */
    int32_t op;       /* SC_OP_*                                               */
    int32_t engine;   /* SC_ENGINE_*                                           */
    double q_dec;     /* decode constant q in C-hat; 0 selects 2^(sc_prec-1)   */
    int32_t scales;   /* SC_SCALES_*                                           */
    int32_t mode;     /* SC_MODE_*                                             */
    void *workspace;  /* (device, nullable, 256-byte aligned) scratch the
                       * call may use; with K-bands on the tensor-core engine,
                       * at least one slice of fp64 band sums (see
                       * sc_matmul_workspace_bytes) lets the kernel keep its
                       * running sums there (160-column tiles, bands split
                       * into segments across CTA pairs) instead of in tensor
                       * memory; when D is not a multiple of 16 it can also
                       * hold the levels in 16-byte rows (aligned loads).
                       * Contents on return are unspecified; calls that may
                       * overlap must not share one workspace.                 */
    int64_t workspace_bytes; /* size of workspace, >= 0                        */
    const sc_bprep *b_prep;  /* NULL, or the second operand prepared once by
                              * sc_prepare_b for this problem and table (a
                              * layer's static weight): the tensor-core kernel
                              * then copies its B tiles instead of building
                              * them; b_lv and b_s must still be the levels and
                              * scales it was prepared from.                   */
} sc_matmul_desc;

/* Message for the last failing call on this thread ("" if none). */
const char *sc_last_error(void);

/* Library version string. */
const char *sc_version(void);

/* sc_kband_tilt -- straight-line tilt of a ladder across n_bands contraction
 * bands ("feat(mp): per-group (K-band) stream lengths on the contraction axis",
 * "Tooling": lengths tilted linearly, rounded down so the identity is never
 * overspent, single units handed back largest-lost-fraction first; tilt 0
 * reproduces the parent).  Host only; launches nothing.
 *   ladder        (host) n_rungs lengths, ascending, each in [1, ceiling]
 *   tilt          slope in (-1, 1): raw[b][k] = L_k (1 + tilt (2b-(B-1))/(B-1))
 *   ceiling       largest allowed length (2^sc_prec); a rung whose tilted
 *                 maximum would exceed it keeps the parent length in every band
 *   band_len_out  (host) [n_bands][n_rungs] result; sum_b = n_bands * L_k
 * Errors: SC_ERR_ARG (pointers, n_bands outside [1, SC_MAX_BANDS], |tilt|>=1),
 *         SC_ERR_TABLE (ladder above ceiling, a band length below 1). */
int sc_kband_tilt(const int32_t *ladder, int n_rungs, int n_bands, double tilt, int ceiling,
                  int32_t *band_len_out);

/* sc_build_table -- build the device-resident stream tables once per layer
 * ("Precision As You Need", key design 1: the Sobol-8 cumulative indicator
 * table is generated once at layer load and stays resident; any stream length
 * is a prefix slice of it).  Synchronous; allocates device memory on the
 * current device.
 *   sc_prec        bits per level, 2..8 (Q = 2^sc_prec positions per period)
 *   ladder         (host) n_rungs stream lengths, strictly ascending, in [1, Q]
 *   band_len       (host) NULL, or [n_bands][n_rungs] per-(band, rung) lengths
 *   n_bands, chunk_d, contraction_d
 *                  with band_len: contraction_d == n_bands * chunk_d is the
 *                  only D the table may be used with ("Guards": a table priced
 *                  at another chunk_d or width is rejected); each band length
 *                  in [1, Q]; sum_b band_len[b][k] == n_bands * ladder[k]
 *                  (iso-compute identity).  Without band_len they are ignored.
 *   out            receives the table; release it with sc_table_destroy.
 * Errors: SC_ERR_ARG, SC_ERR_TABLE (ladder order, ceiling, identity, width),
 *         SC_ERR_CUDA (allocation / copy failed; nothing is leaked). */
int sc_build_table(int sc_prec, const int32_t *ladder, int n_rungs, const int32_t *band_len,
                   int n_bands, int64_t chunk_d, int64_t contraction_d, sc_table **out);

/* sc_build_table_variant -- sc_build_table with a seed-bank variant of the
 * second operand's sequence ("scmp_vit" README, Sobol-seed bank: the default
 * sequence, its antithetic, alternative seeds on the K side).  The first
 * operand keeps the default sequence r_l = u_l + 1 (u_l the bit reversal of
 * l); the second uses u'_l = u_l XOR b_shift and
 *     r'_l = 2^sc_prec - u'_l   (b_antithetic = 1)   or   u'_l + 1   (0),
 * a permutation of the period, so its full-period streams still hold exactly
 * their level's ones.  A's stream is K_A[a, .], B's is drawn from K_B[b, .]
 * by the same two enable-gated counters.  b_shift in [0, 2^sc_prec),
 * b_antithetic 0 or 1; (0, 0) is sc_build_table.  Errors as sc_build_table. */
int sc_build_table_variant(int sc_prec, const int32_t *ladder, int n_rungs,
                           const int32_t *band_len, int n_bands, int64_t chunk_d,
                           int64_t contraction_d, uint32_t b_shift, int b_antithetic,
                           sc_table **out);

/* Order of the built-in Sobol sequence (sc_build_table_seq). */
#define SC_ORDER_NATURAL 0  /* point l = XOR of the direction numbers over the bits of l        */
#define SC_ORDER_GRAY 1     /* point l = the same over the bits of l XOR (l >> 1): the order in
                             * which the Gray-code (Antonov-Saleev) recurrence emits them      */

/* sc_build_table_seq -- sc_build_table with another Sobol sequence ("scmp_vit"
 * README: the SNG of a (contraction width, precision) pair is taken from a
 * cached Sobol pool, _CFG_CACHE[(D, sc_prec)], shared by every op of that
 * width, e.g. the 16 per-head D = 64 comp matmuls and the block's QK).
 *   order    SC_ORDER_NATURAL or SC_ORDER_GRAY: the first Sobol dimension in
 *            that order, for both operands (used when pool is NULL).
 *   pool     (host) NULL, or n_pool sequences of 2^sc_prec integer points
 *            each, int32 [n_pool][2^sc_prec] (e.g. the first 2^sc_prec points
 *            of dimensions 1..n_pool of a Sobol generator, times 2^sc_prec):
 *            contraction index d streams BOTH operands from sequence
 *            d mod n_pool, thresholds r_l = u_l + 1, K[b, l] = 1[r_l <= b].
 *            Every sequence must be a permutation of [0, 2^sc_prec) (so that a
 *            full period of K[b, .] holds b ones): SC_ERR_TABLE otherwise.
 *            With a pool, order must be SC_ORDER_NATURAL.  Pool tables take
 *            n_pool * 256 * 257 bytes of device memory; sc_matmul runs them
 *            on the CUDA-core engine (SC_ENGINE_AUTO picks it;
 *            SC_ENGINE_TC reports SC_ERR_UNSUPPORTED).
 * Other arguments and errors as sc_build_table. */
int sc_build_table_seq(int sc_prec, const int32_t *ladder, int n_rungs, const int32_t *band_len,
                       int n_bands, int64_t chunk_d, int64_t contraction_d, int order,
                       const int32_t *pool, int n_pool, sc_table **out);

/* Free a table (synchronous).  NULL is accepted. */
int sc_table_destroy(sc_table *table);

/* Table properties, for callers and tests. */
int sc_table_info(const sc_table *table, int *sc_prec, int *n_rungs, int *n_bands,
                  int64_t *chunk_d, int64_t *contraction_d);

/* sc_quantize -- symmetric per-row or per-column quantisation to levels, with
 * the row statistic ("scmp_vit" README, "Why it works": scale = abs_max / 127;
 * "Precision As You Need" flowchart: PTQ symmetric integer scaling; key
 * design 2 for the statistic).  For each vector v (a row when axis == 0, a
 * column when axis == 1) of each batch entry:
 *     s_v   = max|x_v| / (2^(sc_prec-1) - 1)       (IEEE fp32 division)
 *     x_int = clamp(rint(x / s_v), -(2^(p-1)-1), 2^(p-1)-1)   (fp32 division,
 *             round half to even; s_v == 0 gives x_int = 0)
 *     level = x_int + 2^(sc_prec-1)
 *   x        (device) fp32, batch entries of [rows x cols], row stride ld >= cols,
 *            batch_stride elements between entries (>= rows * ld)
 *   axis     0: levels[b][rows][cols], scales[b][rows];
 *            1: levels[b][cols][rows] (transposed, contraction contiguous), scales[b][cols]
 *   stat_mode SC_STAT_AMAX or SC_STAT_ROWMAX; stat (device, nullable)
 *            [b][rows] receives g_i (only with axis == 0)
 *   levels, scales (device) outputs as above, dense.
 *   dev_status (device, nullable) receives SC_DEV_NONFINITE on NaN/Inf input;
 *            outputs for such vectors are then unspecified.
 * Errors: SC_ERR_ARG. */
int sc_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                int64_t batch_stride, int axis, int sc_prec, int stat_mode, uint8_t *levels,
                float *scales, float *stat, int32_t *dev_status, void *stream);

/* sc_quantize_chunked -- symmetric quantisation with one scale per (row,
 * chunk of `chunk` contiguous columns), for K-bands whose bands are whole
 * quantisation chunks ("feat(mp) ... K-band", "Summary"; the per-chunk rule is
 * that of sc_quantize: "scmp_vit" README, "Why it works").  For row r and chunk
 * c of each batch entry, over x[r][c*chunk .. (c+1)*chunk):
 *     s_rc  = max|x| / (2^(sc_prec-1) - 1)        (IEEE fp32 division)
 *     level = clamp(rint(x / s_rc), -(2^(p-1)-1), 2^(p-1)-1) + 2^(sc_prec-1)
 * and the row statistic g_r (SC_STAT_*) is taken over the whole row.
 *   x        (device) fp32, batch entries of [rows x cols], row stride ld >= cols,
 *            batch_stride elements between entries (>= rows * ld)
 *   chunk    >= 1, divides cols
 *   levels   (device) out, levels[b][rows][cols]
 *   scales   (device) out, scales[b][rows][cols / chunk]
 *   stat     (device, nullable) out, [b][rows]
 *   dev_status (device, nullable) receives SC_DEV_NONFINITE on NaN/Inf input.
 * Errors: SC_ERR_ARG. */
int sc_quantize_chunked(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                        int64_t batch_stride, int64_t chunk, int sc_prec, int stat_mode,
                        uint8_t *levels, float *scales, float *stat, int32_t *dev_status,
                        void *stream);

/* sc_assign_rows -- rung of every row and the rung-sorted row order
 * ("Precision As You Need", key design 2: g~_i = g_i / max over the group,
 * thresholds tau_1 >= ... >= tau_{K-1}; "feat(mp) ... K-band", "How the banding
 * works": rows are grouped by rung index).  Per group (one batch entry):
 *     g~_i   = g_i / max_i g_i  (fp32 division; 0 when the max is <= 0)
 *     rung_i = #{k : g~_i >= tau_k}
 *     perm   = rows sorted by rung, stably (ascending row index within a rung)
 *   stat          (device) [batch][rows]
 *   tau           (host) n_rungs - 1 thresholds, non-increasing (may be NULL if
 *                 n_rungs == 1)
 *   rung          (device) [batch][rows] out
 *   perm          (device) [batch][rows] out
 *   rung_offsets  (device) [batch][n_rungs + 1] out: rows of rung k are
 *                 perm[offsets[k] .. offsets[k+1])
 * Errors: SC_ERR_ARG (including tau not sorted descending). */
int sc_assign_rows(const float *stat, int64_t rows, int64_t batch, const float *tau, int n_rungs,
                   int32_t *rung, int32_t *perm, int32_t *rung_offsets, void *stream);

/* sc_assign_fraction -- fraction-based fixed mixed precision: each rung holds
 * a given fraction of the units, the longest rung the largest statistic
 * ("scmp_vit" README, MP flags: per input row on linears, per attention row
 * on AV, per head on QK with the metric |Q|.amax).  Units are ordered by
 * their statistic descending, NaN counted as -inf, ties to the lower index;
 * with n units, rung k or above goes to the first
 *     n_k = floor(n * T_k + 1/2),  T_k = f_k + f_{k+1} + ... + f_{K-1}
 * units of that order (T_k summed left to right in double; n_0 = n).
 *   stat          (device) [batch][rows] row statistic (sc_quantize's stat)
 *   set_size      0: the rows of each batch entry are the units;
 *                 > 0: each batch entry (a head's matrix) is one unit with
 *                 statistic max_i stat[g][i] (NaN ignored), ranked within
 *                 consecutive sets of set_size entries; all its rows take
 *                 its rung.  set_size must divide batch.
 *   fractions     (host) n_rungs values f_k >= 0 for rung k (ascending
 *                 length), summing to 1 within 1e-6
 *   rung, perm, rung_offsets  (device) out, as sc_assign_rows (perm is the
 *                 stable rung-sorted row order of each batch entry)
 * Errors: SC_ERR_ARG; SC_ERR_UNSUPPORTED for batch > 65535. */
int sc_assign_fraction(const float *stat, int64_t rows, int64_t batch, int64_t set_size,
                       const double *fractions, int n_rungs, int32_t *rung, int32_t *perm,
                       int32_t *rung_offsets, void *stream);

/* sc_matmul -- the SC bipolar XNOR matmul with C-BSG streams, per-row stream
 * lengths with early termination, optional K-bands, and the decode
 * ("Precision As You Need", key designs 1 and 3; "feat(mp) ... K-band", "How
 * the banding works").  For output (i, j) of group g, with row rung k = rung_i
 * and, for contraction index d, length L = ladder[k] (or band_len[d/chunk_d][k]):
 *     count_b = sum_{d in band b} sum_{l < L} XNOR(K[a_id, l], z^B_jd,l)
 * where z^B is drawn from K[b_jd, .] by two enable-gated counters (one
 * advanced on A's ones, one on A's zeros), and
 *     out_ij  = s^A_i s^B_j q_dec^2 * sum_b (2 count_b / L_b - D_b)
 * (with SC_SCALES_BAND: q_dec^2 * sum_b s^A_ib s^B_jb (2 count_b / L_b - D_b);
 * with SC_MODE_UNIPOLAR the signed AND counts and count_b / L_b in place of
 * 2 count_b / L_b - D_b)
 * evaluated from the exact integer counts in fp64 and rounded once to fp32.
 *   desc           sizes, op, engine, q_dec (see sc_matmul_desc)
 *   a_lv, a_s      (device) A levels / scales
 *   b_lv, b_s      (device) B levels / scales
 *   rung, perm, rung_offsets (device) from sc_assign_rows (rung values must be
 *                  < the table's n_rungs)
 *   table          from sc_build_table; its sc_prec sets the level range; with
 *                  bands, desc->D must equal the table's contraction_d and
 *                  desc->op must be SC_OP_LINEAR; SC_SCALES_BAND needs bands
 *   out            (device) fp32 [batch][M][N]
 *   counts         (device, nullable) int32 [batch][n_bands_eff][M][N] exact
 *                  agreement counts (n_bands_eff = n_bands, or 1 without bands)
 *   dev_status     (device, nullable) receives SC_DEV_LEVEL_RANGE if a level
 *                  exceeds 2^sc_prec; it is clamped to 2^sc_prec so that no
 *                  table is read out of range, and the outputs are unspecified
 * Errors: SC_ERR_ARG, SC_ERR_TABLE, SC_ERR_UNSUPPORTED, SC_ERR_CUDA (launch). */
int sc_matmul(const sc_matmul_desc *desc, const uint8_t *a_lv, const float *a_s,
              const uint8_t *b_lv, const float *b_s, const int32_t *rung, const int32_t *perm,
              const int32_t *rung_offsets, const sc_table *table, float *out, int32_t *counts,
              int32_t *dev_status, void *stream);

/* sc_prepare_b -- prepare a static second operand (a linear layer's weight,
 * "Precision As You Need", key design 1: the tables are built once per layer
 * load; the weight's streams are as static as the tables) for the
 * tensor-core engine: the B operand rows sgn/K-table rows of every level
 * b_jd, for every stream length the table can give a row (each ladder
 * length, or each band's lengths), are written once into device memory in
 * the exact shared-memory layout of the kernel's pipeline stages.  sc_matmul
 * with desc->b_prep set then fills each stage with one bulk copy instead of
 * gathering it.  Asynchronous on stream; allocates device memory (the size
 * sc_prepare_b_bytes gives) on the current device.
 *   desc     the problem it will be used with (M is ignored; N, D, batch, op,
 *            mode, engine, workspace as in the sc_matmul calls): the
 *            preparation fits the wide-tile kernels (no bands, or K-bands
 *            with a workspace of at least one slice), N > 64.
 *   b_lv     (device) B levels [batch][N][D] as sc_matmul takes them
 *   table    the table of the sc_matmul calls
 *   out      receives the handle; release it with sc_bprep_destroy
 * Errors: SC_ERR_ARG; SC_ERR_UNSUPPORTED when the problem runs another
 *         kernel (gather engine, N <= 64, bands without a workspace, a pool);
 *         SC_ERR_CUDA (allocation).  sc_matmul rejects a b_prep made for
 *         another problem or table (SC_ERR_ARG). */
int sc_prepare_b(const sc_matmul_desc *desc, const uint8_t *b_lv, const sc_table *table,
                 sc_bprep **out, void *stream);

/* Device bytes sc_prepare_b allocates for this problem, or minus an SC_ERR_*
 * status.  Host only. */
int64_t sc_prepare_b_bytes(const sc_matmul_desc *desc, const sc_table *table);

/* Free a prepared operand (synchronises the device first).  NULL is accepted. */
int sc_bprep_destroy(sc_bprep *prep);

/* sc_selftest_wait_limit -- exercise the bounded wait every tensor-core
 * kernel uses on its pipeline barriers, alone (the pages have no
 * counterpart: it checks this library's failure reporting).  One thread
 * waits, for at most limit_cycles SM clocks (1 .. 2^34), on a barrier that
 * nothing arrives at, then ORs SC_DEV_WAIT_LIMIT into *dev_status (device,
 * caller-owned) as a kernel whose wait expired does; the kernel returns and
 * the context stays usable.  Asynchronous on stream.  Errors: SC_ERR_ARG,
 * SC_ERR_CUDA. */
int sc_selftest_wait_limit(int32_t *dev_status, int64_t limit_cycles, void *stream);

/* sc_matmul_engine -- the engine sc_matmul would run for this problem and
 * table (resolves SC_ENGINE_AUTO).  Host only; launches nothing.
 * Returns SC_ENGINE_GATHER or SC_ENGINE_TC, or minus an SC_ERR_* status
 * (SC_ERR_UNSUPPORTED when the requested engine cannot run the problem). */
int sc_matmul_engine(const sc_matmul_desc *desc, const sc_table *table);

/* sc_matmul_workspace_bytes -- workspace bytes sc_matmul can use for this
 * problem and table on the tensor-core engine (0 on the gather engine, and 0
 * when there are no K-bands and D is a multiple of 16).
 *   With K-bands the workspace first holds S slices of fp64 running band
 *   sums (batch * M * N each, 256-byte aligned), S the number of segments
 *   each tile's bands are split into so that CTA pairs share the work evenly
 *   (a divisor of the band count), then a small array of counters.  A
 *   smaller workspace is valid: the call uses the largest S whose slices
 *   fit, and below one slice it runs the tensor-memory variant (64-column
 *   tiles).
 *   When D is not a multiple of 16 (and no prepared second operand is
 *   given), it then holds both operands' levels copied into rows of
 *   round16(D) bytes with a zero tail (batch * M and batch * N rows, each
 *   block 256-byte aligned), which the kernels read with aligned loads; the
 *   copy is made in every call, before the count, and is skipped when the
 *   workspace is too small for it (the kernels then read the caller's rows).
 *   Host only.  Returns the byte count, or minus an SC_ERR_* status. */
int64_t sc_matmul_workspace_bytes(const sc_matmul_desc *desc, const sc_table *table);

/* sc_matmul_static_ws -- sc_matmul with a library-owned scratch buffer in
 * place of a caller workspace.  The source pages have no counterpart to this
 * entry point.  It serves callers that cannot allocate device memory: code
 * running where a cudaMalloc is not allowed or not wanted (inside a
 * framework's memory pool that owns all device memory, a process that must
 * not grow its footprint after start-up, or a plugin without an allocator
 * handle).
 *   Arguments, layouts, ownership and errors as sc_matmul, except:
 *   desc->workspace must be NULL and desc->workspace_bytes 0.  The call then
 *   uses a fixed SC_STATIC_WS_BYTES buffer (a file-scope device array of the
 *   library, one per device, present from the moment the library's device
 *   code is loaded until the process exits; the call allocates nothing).
 *   Scratch is needed only by K-band problems on the tensor-core engine
 *   (fp64 running band sums); widths D that are not a multiple of 16 also
 *   use it, when it has room after the sums, for 16-byte level rows.  The call is rejected with SC_ERR_UNSUPPORTED,
 *   before anything is enqueued, when ONE slice of those sums
 *   (batch * M * N * 8 bytes, 256-byte aligned) plus the segment counters
 *   does not fit the buffer; otherwise it runs, splitting each tile's bands
 *   into as many segments as the buffer holds (possibly fewer than
 *   sc_matmul_workspace_bytes asks for: full fc2, 4112 x 1024 outputs, runs
 *   with one segment, i.e. unsplit, at a different speed from a call given
 *   the preferred workspace).
 *   The first call on a device looks up the buffer's device address (once
 *   per device, retried on the next call if the lookup failed); make that
 *   first call outside any stream capture.
 *   Races: every call on a device uses the same buffer and the buffer keeps
 *   the last call's contents.  Calls that can overlap in time (different
 *   streams, or different host threads without ordering) give unspecified
 *   results; issue them on one stream per device or order them otherwise. */
#define SC_STATIC_WS_BYTES (64LL << 20)
int sc_matmul_static_ws(const sc_matmul_desc *desc, const uint8_t *a_lv, const float *a_s,
                        const uint8_t *b_lv, const float *b_s, const int32_t *rung,
                        const int32_t *perm, const int32_t *rung_offsets, const sc_table *table,
                        float *out, int32_t *counts, int32_t *dev_status, void *stream);

/* sc_matmul_launches -- how many kernels sc_matmul launches for this
 * problem and table (0 for an empty problem).  Host only; launches nothing.
 * Lets a caller count device work (e.g. one CUDA graph node per launch).
 * Returns the count, or minus an SC_ERR_* status as sc_matmul_engine. */
int sc_matmul_launches(const sc_matmul_desc *desc, const sc_table *table);

#ifdef __cplusplus
}
#endif

#endif /* SC_B200_H */
