// sc_internal.cuh -- shared definitions of the CUDA library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/sc.h"

// Device-resident stream tables built once per layer by sc_build_table.
//
// C[b][n]  = #{l < n : r_l <= b}, the prefix counts of the Sobol-8 cumulative
//            indicator table K[b, l] = 1[r_l <= b] (levels b = 0..Q,
//            n = 0..Q), uint16.
// For every distinct stream length L used by the table (the ladder, or every
// band length) the tensor-core engine uses the folded form of one C-BSG count
// (derived from the two enable-gated counters):
//     count(a, b, L) = (L - n_a) + sgn_a * sum_{j < w_a} P_L[b, j]
// with n_a = C[a][L] (ones in A's stream), the enable window
// [min(n_a, L-n_a), max(n_a, L-n_a)) folded about the stream centre into
// w_a = ceil(|2 n_a - L| / 2) positions, sgn_a = sign(2 n_a - L), and
// P_L[b, j] = sum of K[b, m] over the (one or two) positions m < L whose
// distance to the centre folds to j.  F_L = ceil(L / 2) folded positions.
struct sc_table {
    int sc_prec = 0;
    int Q = 0;
    int n_rungs = 0;
    int n_bands = 0;          // 0: no bands
    int64_t chunk_d = 0;
    int64_t contraction_d = 0;
    int32_t ladder[SC_MAX_RUNGS] = {0};
    std::vector<int32_t> band_len;     // [n_bands][n_rungs] (host copy)
    std::vector<int32_t> lengths;      // distinct lengths
    std::vector<int32_t> len_idx;      // [max(n_bands,1)][n_rungs] -> index into lengths
    int device = -1;

    // second operand's sequence: digital shift and antithetic (seed bank);
    // tables of the first operand (n = C_A[a][L]) use the default sequence
    uint32_t b_shift = 0;
    int b_antithetic = 0;
    int order = 0;                     // SC_ORDER_*: built-in sequence order (both operands)
    // per-index Sobol pool: contraction index d streams both operands from
    // sequence d mod n_pool (0: no pool); prefix counts of every sequence,
    // d_Cpool[s][b][n] = C_s[b][n] for levels b <= 255 (uint8: C <= b)
    int n_pool = 0;
    uint8_t *d_Cpool = nullptr;        // [n_pool][256][Q+1]

    // device memory.  Without a variant C_A == C_B and d_CA is null.
    uint16_t *d_C = nullptr;           // [(Q+1)*(Q+1)] prefix counts C_B[b][n]
    uint16_t *d_CA = nullptr;          // [(Q+1)*(Q+1)] C_A[a][n], only with a variant
    int32_t *d_len = nullptr;          // [max(n_bands,1)][n_rungs] lengths
    int32_t *d_len_idx = nullptr;      // [max(n_bands,1)][n_rungs]
    // Per length, the A operand of level a is sgn_a x [1 (w_a times), 0, ...]
    // over the F16 folded positions: d_Aw[u][a] = w | neg << 9 | (L - n) << 16
    // with neg = 1 when sgn_a = -1 (2 n < L).  Chunk jc (16 folded positions)
    // of that row is one of 34 patterns: t = clamp(w - 16 jc, 0, 16) ones of
    // sign sgn, which the kernel builds itself.
    int32_t *d_Aw = nullptr;           // [n_lengths][Q+1]: w | neg << 9 | (L - n) << 16
    uint8_t *d_Ct8 = nullptr;          // [(Q+1)][256]: Ct8[n][a] = C_A[a][n], a <= min(Q, 255)
    // The B operand of level b is P_L[b, .].  Chunk jc of it covers the
    // stream positions folding to [16 jc, 16 jc + 16), at most 32 of them;
    // as b grows they switch on one at a time (in the order of their
    // thresholds r_m), so the chunk takes at most 33 values: row c of the
    // chunk's table is the chunk with the first c of its positions on, and
    // the class map gives c = #{positions of the chunk with r_m <= b}.
    std::vector<int64_t> pk_off;       // byte offset of each length's chunk tables in d_Pk
    uint8_t *d_Pk = nullptr;           // per length: [cpd][PK_ROWS][16] bytes
    int64_t *d_pk_off = nullptr;       // device copy of pk_off
    uint8_t *d_Pmap = nullptr;         // [n_lengths][Q+1][PMAP_STRIDE]: class of chunk jc for level b
    // The same for the unipolar AND mode over the L stream positions (chunks
    // of 16 positions, K bytes per index round16(L)): d_AwU[u][a] = n | neg << 9
    // (n = C_A[2|x_a|][L], no row constant), chunk tables of 34 rows (17
    // classes of each sign), class maps; for the CUDA-core rows the signed
    // count tables E_u[(neg_a, n)][b] (int16 bit patterns) and the row of
    // every level a.
    int32_t *d_AwU = nullptr;          // [n_lengths][Q+1]
    std::vector<int64_t> pku_off;
    uint8_t *d_PkU = nullptr;          // per length: [cpd][PK_ROWS][16]
    int64_t *d_pku_off = nullptr;
    uint8_t *d_PmapU = nullptr;        // [n_lengths][Q+1][PMAP_STRIDE]
    std::vector<int64_t> eu_off;
    uint16_t *d_EU = nullptr;          // per length: [2 (L + 1)][256]
    int64_t *d_eu_off = nullptr;
    uint16_t *d_ErowU = nullptr;       // [n_lengths][256]: row of E_u for level a
    // E_L[n][b] = (L - n) + C[b][n] - C[b][L - n] (the count of one (a, b)
    // pair with n = C[a][L]) for n in [0, L], b in [0, 255]: CUDA-core path.
    std::vector<int64_t> e_off;
    uint16_t *d_E = nullptr;           // concatenated [L+1][256] tables
    int64_t *d_e_off = nullptr;
};

// A static second operand prepared for the tensor-core engine (sc_prepare_b):
// for every (band, rung) slot, group, column tile, CTA of the pair and
// pipeline stage, the stage's B tile in the kernel's shared-memory layout
// (BPREP_BLOCK bytes apart; the tile's own columns at the start).
struct sc_bprep {
    int64_t N = 0, D = 0, batch = 0;
    int mode = 0;
    const sc_table *table = nullptr;
    int n_ntiles = 0, tile_w = 0;
    std::vector<int64_t> slot_off;     // [max(n_bands,1) * n_rungs] byte offsets
    int64_t bytes = 0;
    uint8_t *d_buf = nullptr;
    int64_t *d_slot_off = nullptr;
    int device = -1;
};

// Rows of one chunk table of the B operand: bipolar classes 0..32, or the
// unipolar mode's 17 classes of each sign; bytes per row of a class map
// (one byte per chunk, up to 16 chunks of the unipolar mode).
constexpr int PK_ROWS = 34;
constexpr int PMAP_STRIDE = 16;

namespace scb {

void set_error(const char *fmt, ...);
void clear_error();

inline int cuda_fail(cudaError_t e, const char *what) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return SC_ERR_CUDA;
}

int sm_count();
int max_optin_smem();

// launchers (sc_kernels.cu)
int launch_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                    int64_t batch_stride, int axis, int sc_prec, int stat_mode, uint8_t *levels,
                    float *scales, float *stat, int32_t *dev_status, cudaStream_t stream);
int launch_quantize_chunked(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                            int64_t batch_stride, int64_t chunk, int sc_prec, int stat_mode,
                            uint8_t *levels, float *scales, float *stat, int32_t *dev_status,
                            cudaStream_t stream);
int launch_assign_fraction(const float *stat, int64_t rows, int64_t batch, int64_t set_size,
                           const int32_t *n_at, int n_rungs, int32_t *rung, int32_t *perm,
                           int32_t *rung_offsets, cudaStream_t stream);
int launch_assign_rows(const float *stat, int64_t rows, int64_t batch, const float *tau,
                       int n_rungs, int32_t *rung, int32_t *perm, int32_t *rung_offsets,
                       cudaStream_t stream);
int launch_gather(const sc_matmul_desc &d, double q_dec, const uint8_t *a_lv, const float *a_s,
                  const uint8_t *b_lv, const float *b_s, const int32_t *rung, const sc_table &t,
                  float *out, int32_t *counts, int32_t *dev_status, cudaStream_t stream);
// sc_tc.cu
int launch_tc(const sc_matmul_desc &d, double q_dec, const uint8_t *a_lv, const float *a_s,
              const uint8_t *b_lv, const float *b_s, const int32_t *rung, const int32_t *perm,
              const int32_t *rung_offsets, const sc_table &t, float *out, int32_t *counts,
              int32_t *dev_status, cudaStream_t stream);
bool tc_supports(const sc_matmul_desc &d, const sc_table &t);
int tc_prepare_b(const sc_matmul_desc &d, const uint8_t *b_lv, const sc_table &t, sc_bprep **out,
                 cudaStream_t stream);
int64_t tc_prepare_b_bytes(const sc_matmul_desc &d, const sc_table &t);
int tc_bprep_destroy(sc_bprep *prep);
int launch_wait_limit_selftest(int32_t *dev_status, int64_t limit_cycles, cudaStream_t stream);
int tc_launch_count(const sc_matmul_desc &d, const sc_table &t);  // kernels launch_tc launches
int64_t tc_workspace_bytes(const sc_matmul_desc &d, const sc_table &t);  // fp64 sums, bands only
int64_t tc_workspace_min_bytes(const sc_matmul_desc &d, const sc_table &t);  // one slice of sums

// Rows of a rung that the tensor-core engine leaves to the CUDA cores: the
// last, partial 128-row tile of a rung goes to the tensor cores only when it
// holds at least this many rows (F16 = folded length rounded up to 16).
// Contraction bytes per index of the tensor-core operands: the folded
// length ceil(L/2) (bipolar) or L (unipolar), rounded up to 16.
__host__ __device__ inline int kbytes_of(int L, bool unipolar) {
    return unipolar ? ((L + 15) & ~15) : ((((L + 1) / 2) + 15) & ~15);
}

__host__ __device__ inline int tc_min_rows(int f16) {
    const int t = f16 / 8;
    return t < 2 ? 2 : t;
}

}  // namespace scb
