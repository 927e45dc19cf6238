// sc_tc_dev.cuh -- tcgen05 (5th-generation tensor core) count engine for
// sm_100a: the kernel and its device helpers.  Every variant is instantiated
// in its own translation unit (sc_tc_k_*.cu) so that they compile in
// parallel; sc_tc.cu holds the host launcher, the preparation of static
// second operands and the CUDA-core leftover-row kernel.
//
// Exact dense reformulation of the C-BSG bipolar XNOR count
// ("Precision As You Need", key design 1: A streams K[a, l]; B is drawn from
// K[b, .] through two enable-gated counters).  For one (i, j, d) with
// n = C[a][L] ones in A's stream,
//     count = C[b][n] + (L - n) - C[b][L - n]
//           = (L - n) + sgn(2n - L) * #{m in [lo, L - lo) : K[b, m] = 1},
// lo = min(n, L - n): a +-1 window centred on the stream.  Folding the window
// about its centre (positions m and L-1-m share the fold index
// j = |2m - (L-1)| / 2) gives
//     count = (L - n) + sum_{j < F} U[a, j] * P_L[b, j],   F = ceil(L / 2),
//     U[a, j] = sgn * 1[j < w_a] in {-1, 0, 1},  P_L[b, j] in {0, 1, 2},
// so a row of C is an int8 contraction of length D * F plus the row constant
// R_i = sum_d (L - n_{a_id}).  This is one MAC per two stream bits, and the
// contraction runs on the tensor cores with `tcgen05.mma.kind::i8`
// (s32 accumulators in tensor memory), which is exact.  In the unipolar AND
// mode the signed count sgn_a sgn_b C[2|x_b|][n] (n = C[2|x_a|][L]) is the
// contraction over the L stream positions of the thermometer sgn_a 1[m < n]
// with sgn_b K[2|x_b|, m]: the same kernel with L bytes per index.
//
// Kernel layout: for N > 64, clusters of two CTAs on two SMs run one
// `cta_group::2` MMA of M = 256 rows (128 per SM) x N <= 160 columns; each
// SM expands its own 128 rows of A and half of the N columns of B.  For
// N <= 64 every CTA runs `cta_group::1` MMAs of M = 128 alone.  Per CTA:
//   warps 0-3 (and 12-15)  epilogue: tcgen05.ld of this SM's accumulator
//               rows, decode C = s_i s_j q^2 (2 count - D L) / L, store
//   warps 4-7   A producers: one thread per row builds its U chunks from
//               (w, sgn) of each level and writes them into a tensor-memory
//               ring with tcgen05.st (the MMA reads A from tensor memory)
//   warps 8-10  B producers: one thread per column copies P_L chunks from
//               replicated per-chunk tables into this SM's share of the
//               K-major UMMA B tile -- or, with a prepared operand, one lane
//               bulk-copies whole stages and another relays their arrival
//   warp  11    in the MMA's first CTA, one thread issues the MMAs and the
//               commits
// Work items are (group, rung, row tile of the rung-sorted rows, column tile
// [, band segment]); every row of an item runs the same stream length, so
// early termination is real: an item costs D * K(L) per MAC lane.
// All waits on mbarriers are bounded; on expiry the kernel records
// SC_DEV_WAIT_LIMIT, drains its own MMAs and copies, frees tensor memory and
// returns.
#pragma once
#include <stdint.h>

#include "sc_internal.cuh"

namespace scb {
namespace tcd {

constexpr int TM = 128;                    // rows per CTA (TMEM lanes)
constexpr int PM = 2 * TM;                 // rows per pair tile (UMMA M = 256)
constexpr int TNMAX = 160;                 // max columns per pair tile (UMMA N, multiple of 32)
constexpr int BC = TNMAX / 2;              // B columns staged per CTA
// Pipeline stages: SKB contraction bytes per stage (SKB/32 UMMA K-steps, one
// barrier round trip each).  Every wait and every tcgen05.mma has a fixed
// cost of a few hundred cycles in this kernel, so stages are as deep as
// tensor memory allows: 256 bytes without bands, 128 with bands.
// 256-byte stages (8 MMAs of K = 32 per barrier round trip) in a 3-slot ring
// (no bands, bands with workspace sums, the one-CTA kernel): every stage
// costs the MMA warp a fixed ~200 cycles besides its MMAs, so stages are as
// deep as tensor memory allows (128-byte stages in a 6-slot ring, the same
// bytes in flight, measured 10-40 % slower)
constexpr int SK_PLAIN = 256, SK_BANDS = 256;
constexpr int TN_SINGLE = 64;  // column tiles of the one-CTA (M = 128) kernel
constexpr int RING_PLAIN = 3, RING_BANDS = 4;
constexpr int MAX_STAGES = 4;
constexpr int B_RING_BYTES = 60 * 1024;    // B ring: 3 x 80 x 256 (pair) or 4 x 32 x 256 (bands in TMEM)
static_assert(RING_PLAIN * BC * SK_PLAIN <= B_RING_BYTES, "B ring");
// Tensor memory (512 columns x 128 lanes of 32 bits per SM):
//   no bands: accumulators [0, 160) and [160, 320), A ring of 3 x 64 at 320;
//   bands:    accumulators [0, 64) and [64, 128), fp64 running sum (two
//             columns per output) at [128, 256), A ring of 4 x 64 at 256.
constexpr int TNMAX_BANDS = 64;
static_assert(RING_BANDS * (TNMAX_BANDS / 2) * SK_BANDS <= B_RING_BYTES, "B ring (bands)");
constexpr uint32_t SUM_COL = 2 * TNMAX_BANDS;
constexpr int MMA_BATCH = 1;  // ring stages per round of MMA issue (< ring)
static_assert(MMA_BATCH >= 1 && MMA_BATCH < RING_PLAIN, "MMA batch below the ring depth");
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_EPI_WARPS = 4;            // warps 0-3; without bands also warps 12-15
constexpr int MAX_EPI_WARPS = 8;
constexpr int NUM_A_WARPS = 4;
constexpr int NUM_B_WARPS = 3;             // 96 threads: one B column each
constexpr int A_WARP0 = NUM_EPI_WARPS;                 // 4
constexpr int B_WARP0 = A_WARP0 + NUM_A_WARPS;         // 8
constexpr int MMA_WARP = B_WARP0 + NUM_B_WARPS;        // 11
constexpr int THREADS = (MMA_WARP + 1) * 32;           // 384 with bands
constexpr int THREADS_PLAIN = THREADS + NUM_EPI_WARPS * 32;  // 512: a second epilogue warp per quadrant
constexpr int B_THREADS = NUM_B_WARPS * 32;            // 96
static_assert(B_THREADS >= BC, "one B column per producer thread");
constexpr uint32_t READY_ARRIVALS = NUM_A_WARPS + NUM_B_WARPS;  // local producers per stage
constexpr long long WAIT_LIMIT_CYCLES = 1LL << 32;     // ~2 s
// Operand tables in shared memory, every 16-byte entry replicated 8 times
// (entry e, replica k at (8 e + k) * 16; lane l reads replica l % 8), so the 8
// lanes of a shared-memory wavefront hit 8 different 16-byte bank groups
// whatever entries they read.
constexpr int REP = 8;
constexpr int MAX_CPD = 16;   // 16-byte chunks per index (bipolar F16 <= 128, unipolar round16(L) <= 256)
constexpr int PTAB_BYTES = MAX_CPD * PK_ROWS * REP * 16;  // B chunk tables: 69,632 B
constexpr int PMAP_BYTES = 257 * PMAP_STRIDE;      // B class maps: one 16-byte row per level
constexpr int UPAT_ROWS = 34;                      // A chunk patterns: +t (rows 0-16), -t (17-33)
constexpr int UTAB_BYTES = UPAT_ROWS * REP * 16;   // 4,352 B
constexpr int UMAX = 2048;             // (group, rung) units per launch
// Balanced deal of the work items: launches of at most BAL_MAX items whose
// units (clusters, or CTAs) get at most PLIST_MAX items each sort the items
// by their stage count and deal them out in snake order.
constexpr int BAL_MAX = 2048;
constexpr int PLIST_MAX = 64;
constexpr uint32_t BAL_COST_MAX = (1u << 20) - 1;  // stage counts beyond it tie
constexpr uint32_t BAL_ITEM_STAGES = 4;            // an item's fixed cost, in stages

static_assert(2 * TNMAX + RING_PLAIN * SK_PLAIN / 4 <= TMEM_COLS, "TMEM budget (no bands)");
static_assert(RING_PLAIN * TN_SINGLE * SK_PLAIN <= B_RING_BYTES, "B ring (single)");
static_assert(2 * TN_SINGLE + RING_PLAIN * SK_PLAIN / 4 <= TMEM_COLS, "TMEM budget (single)");
static_assert(TN_SINGLE <= NUM_B_WARPS * 32, "one B column per producer thread (single)");
static_assert(SUM_COL + 2 * TNMAX_BANDS + RING_BANDS * SK_BANDS / 4 <= TMEM_COLS, "TMEM budget (bands)");
static_assert(RING_PLAIN <= MAX_STAGES && RING_BANDS <= MAX_STAGES, "ring slots");

struct TcArgs {
    int64_t M, N, D, batch;
    const uint8_t *a_lv;
    const float *a_s;
    const uint8_t *b_lv;
    const float *b_s;
    int64_t lda, ldb;          // bytes between level rows of A and of B (D, or D padded to 16)
    const int32_t *perm;
    const int32_t *offs;       // [batch][n_rungs + 1]
    const uint8_t *Pk;         // B chunk tables, [cpd][PK_ROWS][16] per length
    const int64_t *pk_off;     // byte offset of each length's chunk tables
    const uint8_t *Pmap;       // [n_lengths][Q+1][8]: class of chunk jc for level b
    const int32_t *Aw;         // [n_lengths][Q+1]: w | neg << 8 | (L - n) << 16
    int32_t len[SC_MAX_RUNGS];  // stream length per rung
    int32_t lidx[SC_MAX_RUNGS]; // table index per rung
    int n_rungs, Q;
    int n_bands;               // 0: one band covering D
    int64_t chunk_d;           // band width
    const int32_t *blen;       // [n_bands][n_rungs] band lengths (device)
    const int32_t *blidx;      // [n_bands][n_rungs] table index of each band length
    int band_scales;           // a_s [.][M][n_bands], b_s [.][N][n_bands]: one scale per (row, band)
    int acc_stride;            // TMEM columns per accumulator buffer (160, or 96 with bands)
    int ring;                  // pipeline ring slots
    int bslot;                 // bytes of one B stage on one SM (tile columns / 2 x stage bytes)
    uint32_t ring_col;         // TMEM column of the A ring
    int n_ntiles, tile_w;      // column tiles of tile_w (multiple of 32, <= acc_stride) columns
    int64_t g_begin;           // first group of this launch
    int n_groups;              // groups in this launch (n_groups * n_rungs <= UMAX)
    double q2d;
    float *out;
    int32_t *counts;
    int32_t *dev_status;
    double *gsum;              // bands on wide tiles: fp64 running sums [ksplit][batch][M][N]
    int ksplit;                // band segments per tile (1: an item walks all bands)
    int64_t part_stride;       // elements between the segments' partial sums (batch M N)
    int32_t *tile_cnt;         // per (tile, CTA, epilogue warp): segments finished
    const uint8_t *bprep;      // prepared B stages (sc_prepare_b), or null: build B on chip
    const int64_t *bprep_off;  // [max(n_bands,1) * n_rungs] byte offset of each slot's stages
    int balance;               // deal items by cost (see BAL_MAX) instead of round robin
};

// bytes between two prepared B stages (one CTA's half of a 160-column tile,
// 256-byte stages); a stage's own columns (chalf) come first
constexpr int BPREP_BLOCK = BC * SK_PLAIN;
constexpr int BPREP_PREFETCH = 4;  // stages fetched into L2 ahead of their copy

struct RowInfo {
    int64_t obase; // offset of (row, first column of the tile) in out, -1 for a padding row
    double fd;     // s^A_i q^2 (band decode; s^A_ib q^2 with per-band scales)
    int R;         // row constant sum_{d in band} (L - n)
    float f;       // s^A_i q^2 / L (single band)
};

struct __align__(16) Smem {
    uint8_t bring[B_RING_BYTES];  // B stages: slot s at s * BC * SKB
    uint8_t ptab[PTAB_BYTES];
    uint8_t utab[UTAB_BYTES];
    uint8_t pmap[PMAP_BYTES];
    uint32_t epi[MAX_EPI_WARPS][32][33];   // per-warp 32 x 32 transpose of accumulator values
    RowInfo rowinfo[2][TM];     // per item (parity): written by the A producers
    float sbw[MAX_EPI_WARPS][TNMAX];  // per epilogue warp: column scales s^B_j of the tile
    int32_t aw[SC_MAX_RUNGS][257];
    int32_t awb[257];          // (urow, L - n) of the current band's length (A producers)
    int32_t ubase[UMAX + 1];   // exclusive prefix of work items over units (group, rung)
    int32_t urow0[UMAX];       // per unit: its first position in the rung-sorted order
    int32_t ucnt[UMAX];        // per unit: its rows
    int32_t plist[PLIST_MAX];  // balanced deal: this unit's item ids in order
    int nplist;                // their number, or -1: round robin (item pair + j * n_pairs)
    uint64_t ready[MAX_STAGES];  // this CTA's producers (+ on the first CTA the second CTA's relay)
    uint64_t empty[MAX_STAGES];  // both CTAs: multicast MMA commit
    uint64_t acc_full[2];      // both CTAs: multicast MMA commit
    uint64_t acc_empty[2];     // first CTA: both SMs' epilogue warps arrive
    uint64_t rinfo_full[2];    // local: A producers -> epilogue
    uint64_t rinfo_empty[2];   // local: epilogue -> A producers
    uint64_t bgrp;             // local: B producer warps (table reloads)
    uint64_t bfull[MAX_STAGES];  // local: bulk copy of a prepared B stage landed
    uint64_t agrp;             // local: A producer warps (table reloads)
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget");

// ---- PTX wrappers ----------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}

// Arrive on the barrier at the same shared-memory offset in CTA `rank` of
// the cluster.  Relaxed: every caller has already completed what the arrive
// announces (tcgen05.wait::st / wait::ld for tensor memory, the async-proxy
// fence for shared-memory stores, a local acquire of the producers' barrier),
// so a release at cluster scope would only add a full memory drain (~850
// cycles measured) to every pipeline stage.
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t *bar, uint32_t rank) {
    asm volatile(
        "{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_addr(bar)),
        "r"(rank)
        : "memory");
}

// try_wait with a suspend-time hint: a waiting warp sleeps until the phase
// completes instead of spinning.  Acquire at CTA scope, as for any barrier
// in this kernel: a phase that a remote arrive or a multicast commit
// completes publishes no generic-proxy data that the waiter reads (operands
// and accumulators are ordered by the tcgen05 fences around the waits), and
// a cluster-scope acquire costs hundreds of cycles on every wait.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false if the
// kernel is aborting (another role gave up) or the limit expired.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          long long limit = WAIT_LIMIT_CYCLES) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - t0 > limit || it > (1u << 30)) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Warp-uniform bounded wait: every lane of the calling warp gets the same
// answer, so the warp stays converged for the .sync.aligned instructions that
// follow even when the kernel is aborting.
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

// Prepared B stages: one bulk copy global -> this CTA's shared memory per
// stage, completing on a local barrier that expects its bytes; plus a hint
// that brings later stages into L2 (no multicast anywhere).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand, no swizzle: core matrices of 8 rows x 16 bytes stored as
// 128 contiguous bytes; LBO = distance between K-adjacent core matrices,
// SBO = distance between 8-row groups.  Descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
           ((uint64_t)(sbo >> 4) << 32) | (1ull << 46);
}

// kind::i8 instruction descriptor: D s32, A s8, B s8, both K-major.
__device__ __forceinline__ uint32_t make_idesc(int m, int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

// MMA with A from tensor memory and B from shared memory.  CG = 2 (pair):
// both SMs' A at the same address, each SM holding N/2 rows of B at the same
// offset, D in both SMs' TMEM (M = 256); CG = 1: one SM, M = 128.
template <int CG>
__device__ __forceinline__ void mma_i8_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                          uint32_t accumulate) {
    if constexpr (CG == 2) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
            "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
            "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

// Commit the outstanding MMAs to the barrier at this offset: CG = 2, in both
// CTAs of the pair (multicast); CG = 1, in this CTA.
template <int CG>
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    if constexpr (CG == 2) {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
            "[%0], %1;" ::"r"(smem_addr(bar)),
            "h"((uint16_t)3)
            : "memory");
    } else {
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_addr(bar))
                     : "memory");
    }
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- work items ------------------------------------------------------------
// Items are ordered (rung, group, 256-row tile, column tile); cluster c takes
// items c, c + clusters, ...  Every role of both CTAs walks the same sequence.
// A rung's last, partial row tile is a tensor-core item only when it holds
// at least tc_min_rows(F16) rows; smaller remainders go to small_rows_kernel.
__device__ __forceinline__ int f16_of(int L) { return kbytes_of(L, false); }

template <bool UNI, int CG>
__device__ __forceinline__ int unit_items(const TcArgs &p, int cnt, int k) {
    constexpr int TR = CG * TM;  // rows per tile
    const int rem = cnt % TR;
    const int tiles = cnt / TR + (rem >= tc_min_rows(kbytes_of(p.len[k], UNI)) ? 1 : 0);
    return tiles * p.n_ntiles * p.ksplit;
}

// Locates work items among units; ubase (shared memory) holds the first item
// id of every unit and ubase[U] the total.  Targets only grow, so the search
// for the unit holding item `target` (the last u with ubase[u] <= target)
// starts at the previous unit: O(log U) shared-memory reads per item.
struct Walker {
    int u = 0;
};

__device__ __forceinline__ bool walker_seek(const int32_t *ubase, int U, Walker &w, int64_t target) {
    if (target >= ubase[U]) return false;
    int lo = w.u, hi = U;  // ubase[lo] <= target < ubase[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ubase[mid] <= target) lo = mid;
        else hi = mid;
    }
    w.u = lo;
    return true;
}

// The j-th work item of unit `pair`: entry j of its balanced list when the
// launch deals items by cost, else item pair + j * n_pairs.  Returns false
// past the unit's last item; w is left on the item's (group, rung) unit.
__device__ __forceinline__ bool sched_item(const int32_t *plist, int nplist, const int32_t *ubase, int U,
                                           int64_t pair, int64_t n_pairs, int j, Walker &w, int64_t &id) {
    if (nplist >= 0) {
        if (j >= nplist) return false;
        id = plist[j];
        w.u = 0;  // a balanced list is not in increasing order
    } else {
        id = pair + (int64_t)j * n_pairs;
    }
    return walker_seek(ubase, U, w, id);
}

struct Item {
    int64_t g;
    int k;
    int row0;                  // start in perm of this CTA's 128 rows
    int rows;                  // valid rows of this CTA (0..128)
    int n0, nw, nvalid;        // pair column tile: start, MMA width (mult. of 32), valid columns
    int c0, chalf;             // this CTA's B columns: n0 + c0 .. + chalf (chalf = nw / 2)
    int b_lo, b_hi, seg;       // bands [b_lo, b_hi): segment seg of the tile's bands
    int64_t tile;              // tile index in the launch (items / ksplit)
};

template <int CG>
__device__ __forceinline__ Item make_item(const TcArgs &p, const Smem &sm, const Walker &w,
                                          int64_t id, int rank) {
    Item it;
    // item ids of a launch fit 32 bits (the unit prefix is int32).  Within a
    // unit the items run row tile, column tile, band segment (a tile's
    // segments are consecutive items, dealt to different pairs); with
    // prepared B stages they run column tile, segment, row tile instead, so
    // that the pairs running at the same time read the same B stages
    // through L2 (measured: half the DRAM reads of the fc2 count).
    const int local = (int)id - sm.ubase[w.u];
    const int per_mt = p.n_ntiles * p.ksplit;                // items per row tile
    const int nmt = (sm.ubase[w.u + 1] - sm.ubase[w.u]) / per_mt;  // row tiles of the unit
    int mt, r;
    if (p.bprep) {
        mt = nmt == 1 ? 0 : local % nmt;
        r = nmt == 1 ? local : local / nmt;                  // column tile x segments + segment
    } else {
        mt = local / per_mt;
        r = local - mt * per_mt;
    }
    if (p.ksplit == 1) {
        it.seg = 0;
        it.b_lo = 0;
        it.b_hi = p.n_bands > 0 ? p.n_bands : 1;
    } else {
        it.seg = r % p.ksplit;
        const int per = p.n_bands / p.ksplit;
        it.b_lo = it.seg * per;
        it.b_hi = it.b_lo + per;
    }
    const int nt = p.ksplit == 1 ? r : r / p.ksplit;
    // the tile's index in the launch (its segments share one counter)
    it.tile = sm.ubase[w.u] / p.ksplit + nt * nmt + mt;
    it.k = w.u / p.n_groups;  // units run rung-major: a pair's items mostly share L
    it.g = p.g_begin + w.u % p.n_groups;
    const int row0 = sm.urow0[w.u], cnt = sm.ucnt[w.u];  // cached at kernel start
    if constexpr (CG == 2) {
        const int pair_rows = min(PM, cnt - mt * PM);
        // a partial tile's rows are split between the two CTAs in whole warps
        // (32 TMEM lanes), as evenly as possible, so that the producer and
        // epilogue warps left without a valid row can skip their work
        const int h0 = min(TM, 32 * ((pair_rows + 63) / 64));
        it.row0 = row0 + mt * PM + (rank ? h0 : 0);
        it.rows = rank ? max(pair_rows - h0, 0) : min(pair_rows, h0);
    } else {
        it.row0 = row0 + mt * TM;
        it.rows = min(TM, cnt - mt * TM);
    }
    it.n0 = nt * p.tile_w;
    it.nvalid = (int)min((int64_t)p.tile_w, p.N - it.n0);
    it.nw = (it.nvalid + 31) & ~31;
    it.chalf = it.nw / CG;  // this CTA's B columns
    it.c0 = rank * it.chalf;
    return it;
}

// Position in the pipeline ring: slot and the parity of its current use.
struct RingPos {
    int slot = 0;
    uint32_t ph = 0;
};

__device__ __forceinline__ void ring_next(RingPos &r, int ring) {
    if (++r.slot == ring) {
        r.slot = 0;
        r.ph ^= 1u;
    }
}

// One band of an item: contraction indices [d_lo, d_hi) at stream length L.
struct Band {
    int L, F16, lidx, n_stages;
    int64_t d_lo, d_hi;
};

template <int SKB, bool UNI>
__device__ __forceinline__ Band band_of(const TcArgs &p, const Item &it, int b) {
    Band bd;
    if (p.n_bands == 0) {
        bd.L = p.len[it.k];
        bd.lidx = p.lidx[it.k];
        bd.d_lo = 0;
        bd.d_hi = p.D;
    } else {
        bd.L = __ldg(p.blen + b * p.n_rungs + it.k);
        bd.lidx = __ldg(p.blidx + b * p.n_rungs + it.k);
        bd.d_lo = (int64_t)b * p.chunk_d;
        bd.d_hi = bd.d_lo + p.chunk_d;
    }
    bd.F16 = kbytes_of(bd.L, UNI);  // contraction bytes per index
    bd.n_stages = (int)(((bd.d_hi - bd.d_lo) * bd.F16 + SKB - 1) / SKB);
    return bd;
}

// 16 levels of one row starting at d0.  Bytes at or past D read as 0 on
// the byte path; the word paths may return the bytes that follow up to cap
// (the bytes readable from the row's start, >= D), which the
// tensor-core producers ignore (their dead contraction indices contribute
// nothing).  A window that is not 16-byte aligned is read as two aligned
// 16-byte words and funnel-shifted, as long as both lie within cap; rows
// padded to a multiple of 16 bytes (cap = the padded stride) are always
// read with one aligned load.
__device__ __forceinline__ uint4 load_levels16_cap(const uint8_t *row, int64_t d0, int64_t D, int64_t cap) {
    if (row == nullptr || d0 >= D) return make_uint4(0, 0, 0, 0);
    const uintptr_t addr = reinterpret_cast<uintptr_t>(row + d0);
    const uint32_t k = (uint32_t)(addr & 15u);
    if (d0 + 16 <= cap && k == 0) return __ldg(reinterpret_cast<const uint4 *>(addr));
    if (d0 + 32 - (int64_t)k <= cap) {
        const uint4 *base = reinterpret_cast<const uint4 *>(addr - k);
        const uint4 lo = __ldg(base), hi = __ldg(base + 1);
        const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        const uint32_t q = k >> 2, r = 8u * (k & 3u);
        uint32_t x[5];
#pragma unroll
        for (int j = 0; j < 5; ++j)  // x[j] = w[q + j], q in 0..3
            x[j] = q == 0 ? w[j] : (q == 1 ? w[j + 1] : (q == 2 ? w[j + 2] : w[j + 3]));
        return make_uint4(__funnelshift_r(x[0], x[1], r), __funnelshift_r(x[1], x[2], r),
                          __funnelshift_r(x[2], x[3], r), __funnelshift_r(x[3], x[4], r));
    }
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int64_t d = d0 + u;
        const uint32_t v = d < D ? (uint32_t)__ldg(row + d) : 0u;
        w[u >> 2] |= v << (8 * (u & 3));
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// The same with cap = D: bytes at or past D always read as 0.
__device__ __forceinline__ uint4 load_levels16(const uint8_t *row, int64_t d0, int64_t D) {
    return load_levels16_cap(row, d0, D, D);
}

// Level u (compile-time after unrolling) of a 16-level window.
__device__ __forceinline__ int lv_byte(const uint4 &c, int u) {
    const uint32_t w = (u >> 2) == 0 ? c.x : ((u >> 2) == 1 ? c.y : ((u >> 2) == 2 ? c.z : c.w));
    return (int)((w >> (8 * (u & 3))) & 0xffu);
}


// Contraction indices per level window of a producer: a whole number of
// stages always covers a whole number of windows.
template <int SKB>
__host__ __device__ constexpr int win_of() { return SKB >= 512 ? 32 : 16; }

// Level u (compile-time after unrolling) of a window of 16 * NW levels.
template <int NW>
__device__ __forceinline__ int lv_byte_w(const uint4 (&c)[NW], int u) {
    return lv_byte(c[u >> 4], u & 15);
}

// Canonical no-swizzle K-major offset of (row r, 16-byte chunk q) in a stage
// that is SKB bytes deep: 8-row groups of SKB/16 core matrices of 128 bytes.
template <int SKB>
__device__ __forceinline__ uint32_t op_offset(int r, int q) {
    return (uint32_t)((r >> 3) * (SKB / 16) * 128 + q * 128 + (r & 7) * 16);
}

// Producer warp's "stage filled" signal: on the first CTA of the pair a local
// arrive, on the second a cluster arrive on the first CTA's barrier (the MMA
// issuer waits for the producers of both SMs on one barrier).
template <int CG>
__device__ __forceinline__ void ready_arrive(uint64_t *bar) {
    if (CG == 1 || cluster_rank() == 0) mbar_arrive(bar);
    else mbar_arrive_cluster(bar, 0);
}

// ---- replicated tables ------------------------------------------------------
// n_entries 16-byte entries of src staged with every entry repeated REP
// times (see REP); threads t of nt share the copy.
__device__ __forceinline__ void stage_replicated(uint8_t *dst, const uint8_t *src, int n_entries, int t,
                                                 int nt) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    for (int e = t; e < n_entries * REP; e += nt)
        *reinterpret_cast<uint4 *>(dst + (size_t)e * 16) = __ldg(s4 + e / REP);
}

// The 34 chunk patterns of the A operand, replicated: row t (0..16) holds
// +1 in its first t bytes, row 17 + t holds -1 (0xff) there.
__device__ __forceinline__ void stage_u_patterns(uint8_t *dst, int t, int nt) {
    for (int e = t; e < UPAT_ROWS * REP * 4; e += nt) {
        const int row = e / (REP * 4), word = e % 4;
        const int ones = row < 17 ? row : row - 17;
        const uint32_t sgn = row < 17 ? 0x01010101u : 0xffffffffu;
        const int k = ones - 4 * word;  // bytes of this word inside the pattern
        const uint32_t mask = k >= 4 ? 0xffffffffu : (k <= 0 ? 0u : (0xffffffffu >> (32 - 8 * k)));
        reinterpret_cast<uint32_t *>(dst)[e] = sgn & mask;
    }
}

// Bounded barrier among the n_warps warps of one producer group: the n-th
// call waits for phase n of bar.
__device__ __forceinline__ bool group_sync(uint64_t *bar, uint32_t &n, volatile int *abort_flag) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = wait_warp(bar, n & 1u, abort_flag);
    ++n;
    return ok;
}

// ---- producers, specialised on the stage depth SKB and the number of 16-byte
// chunks per contraction index (CPD = F16 / 16) so that every level byte,
// fold offset and stage offset below is a compile-time constant.  A stage is
// SKB/16 chunks; a window of 16 contraction indices is 16 * CPD chunks.

// A: one thread per row of this CTA (= TMEM lane).  The U row of level a is
// sgn_a x [1 (w_a times), 0, ...]; its chunk jc is the staged pattern with
// t = clamp(w_a - 16 jc, 0, 16) bytes of that sign (zeros for a dead
// contraction index), so a 16-byte chunk costs one add-min-max and one
// conflict-free shared-memory load.  A stage goes to tensor memory in
// 32-column pieces (8 chunks each).
template <int SKB, int CPD, int CG>
__device__ __forceinline__ bool produce_a(const TcArgs &p, Smem &sm, const Band &bd,
                                          const int32_t *aw, const uint8_t *row, bool a_ok,
                                          const uint8_t *tab, uint32_t lane_base, RingPos &rp,
                                          int &Rsum, volatile int *abort_flag, bool &range_bad,
                                          bool has_pre, uint4 pre) {
    constexpr int CH = SKB / 16;                  // chunks per stage
    constexpr int WIN = win_of<SKB>(), NW = WIN / 16;
    constexpr int SPW = WIN * CPD / CH;           // stages per window
    static_assert((WIN * CPD) % CH == 0, "stage boundaries at window boundaries");
    if (!__any_sync(0xffffffffu, a_ok)) {
        // no valid row in this warp: its lanes of the ring are left as they
        // are (the outputs of padding rows are never stored); the warp still
        // takes every slot in order, so that its arrivals stay in phase
        for (int s = 0; s < bd.n_stages; ++s) {
            if (!wait_warp(&sm.empty[rp.slot], rp.ph ^ 1u, abort_flag)) return false;
            __syncwarp();
            if ((threadIdx.x & 31) == 0) ready_arrive<CG>(&sm.ready[rp.slot]);
            ring_next(rp, p.ring);
        }
        return true;
    }
    uint4 nxt[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k)  // the first window may have been loaded ahead (next-item prefetch)
        nxt[k] = (has_pre && k == 0) ? pre : load_levels16_cap(row, bd.d_lo + 16 * k, bd.d_hi, p.lda);
    int s = 0;
    for (int64_t d0 = bd.d_lo; s < bd.n_stages; d0 += WIN) {
        uint4 cur[NW];
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            cur[k] = nxt[k];
            nxt[k] = load_levels16_cap(row, d0 + WIN + 16 * k, bd.d_hi, p.lda);
        }
        const int nlive = a_ok ? (int)min((int64_t)WIN, bd.d_hi - d0) : 0;
#pragma unroll
        for (int t = 0; t < SPW; ++t) {
            if (s >= bd.n_stages) break;
#pragma unroll
            for (int h = 0; h < CH / 8; ++h) {
                uint32_t v[32];
                const uint8_t *rowp = tab;
                int w = 0;
                int last_dr = -1;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int c = t * CH + h * 8 + q, dr = c / CPD, jc = c % CPD;
                    if (dr != last_dr) {  // compile-time after unrolling
                        last_dr = dr;
                        int a = lv_byte_w(cur, dr);
                        if (a > p.Q) {
                            a = p.Q;
                            range_bad = true;
                        }
                        const int32_t e = aw[a];
                        const bool live = dr < nlive;
                        w = live ? (e & 0x1ff) : 0;
                        rowp = tab + ((e >> 9) & 1) * (17 * REP * 16);
                        // an index whose chunks straddle two pieces is counted once
                        if (live && jc == 0) Rsum += e >> 16;
                    }
                    const int tt = __viaddmin_s32_relu(w, -16 * jc, 16);  // clamp(w - 16 jc, 0, 16)
                    const uint4 x = *reinterpret_cast<const uint4 *>(rowp + tt * (REP * 16));
                    v[4 * q] = x.x;
                    v[4 * q + 1] = x.y;
                    v[4 * q + 2] = x.z;
                    v[4 * q + 3] = x.w;
                }
                if (h == 0) {
                    if (!wait_warp(&sm.empty[rp.slot], rp.ph ^ 1u, abort_flag)) return false;
                    tc_fence_after();
                }
                tmem_st32(lane_base + p.ring_col + (uint32_t)(rp.slot * (SKB / 4) + h * 32), v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) ready_arrive<CG>(&sm.ready[rp.slot]);
            ++s;
            ring_next(rp, p.ring);
        }
    }
    return true;
}

// B: one column of this CTA's half of the pair tile per thread; per
// contraction index one 8-byte load of the level's class map, then each
// 16-byte chunk jc is row class[jc] of chunk jc's staged table.
// The levels row of the B column a producer thread fills for an item (null
// when the thread has no valid column), and the thread's group and column.
__device__ __forceinline__ const uint8_t *b_column(const TcArgs &p, const Item &it, int bt, int nbt, int ch,
                                                   int &G, int &grp, int &bc) {
    // G thread groups share each column, group g filling the 8-chunk pieces h
    // with h % G == g of every stage: as many groups as the threads cover
    // (each group at least one thread per column) and the pieces allow
    G = max(1, min(min(3, ch / 8), nbt / max(it.chalf, 1)));
    const int span = nbt / G;
    grp = bt / span;
    bc = bt - grp * span;
    const bool c_ok = bc < it.chalf && grp < G;
    const int col = it.c0 + bc;  // within the tile
    return (c_ok && col < it.nvalid) ? p.b_lv + (it.g * p.N + it.n0 + col) * p.ldb : nullptr;
}

template <int SKB, int CPD, int CG>
__device__ __forceinline__ bool produce_b(const TcArgs &p, Smem &sm, const Item &it, const Band &bd,
                                          int bt, int nbt, RingPos &rpos, volatile int *abort_flag,
                                          bool &range_bad, bool has_pre, uint4 pre) {
    constexpr int CH = SKB / 16;
    constexpr int WIN = win_of<SKB>(), NW = WIN / 16;
    constexpr int SPW = WIN * CPD / CH;
    int G, grp, bc;
    const uint8_t *rp = b_column(p, it, bt, nbt, CH, G, grp, bc);
    const uint8_t *tab = sm.ptab + (threadIdx.x & (REP - 1)) * 16;
    const bool c_ok = bc < it.chalf && grp < G;
    const uint32_t off = op_offset<SKB>(bc, 0);
    const int qmax = p.Q;
    uint4 nx[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k)  // the first window may have been loaded ahead (next-item prefetch)
        nx[k] = (has_pre && k == 0) ? pre : load_levels16_cap(rp, bd.d_lo + 16 * k, bd.d_hi, p.ldb);
    int s = 0;
    for (int64_t d0 = bd.d_lo; s < bd.n_stages; d0 += WIN) {
        uint4 lv[NW];
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            lv[k] = nx[k];
            nx[k] = load_levels16_cap(rp, d0 + WIN + 16 * k, bd.d_hi, p.ldb);
        }
#pragma unroll
        for (int t = 0; t < SPW; ++t) {
            if (s >= bd.n_stages) break;
            if (!wait_warp(&sm.empty[rpos.slot], rpos.ph ^ 1u, abort_flag)) return false;
            if (c_ok) {
                uint8_t *sb = sm.bring + rpos.slot * p.bslot;
#pragma unroll
                for (int h = 0; h < CH / 8; ++h) {
                    if (h % G != grp) continue;
                    uint4 x[8];
                    int last_dr = -1;
                    uint4 cls = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int c = t * CH + h * 8 + q, dr = c / CPD, jc = c % CPD;
                        if (dr != last_dr) {
                            last_dr = dr;
                            int b = lv_byte_w(lv, dr);
                            if (b > qmax) {
                                range_bad = true;
                                b = qmax;
                            }
                            if constexpr (CPD <= 8) {
                                const uint2 c2 = *reinterpret_cast<const uint2 *>(sm.pmap + b * PMAP_STRIDE);
                                cls = make_uint4(c2.x, c2.y, 0, 0);
                            } else {
                                cls = *reinterpret_cast<const uint4 *>(sm.pmap + b * PMAP_STRIDE);
                            }
                        }
                        const uint32_t cw = jc < 4 ? cls.x : (jc < 8 ? cls.y : (jc < 12 ? cls.z : cls.w));
                        const int k = (int)((cw >> (8 * (jc & 3))) & 0xffu);
                        x[q] = *reinterpret_cast<const uint4 *>(tab + (jc * PK_ROWS + k) * (REP * 16));
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4 *>(sb + off + (h * 8 + q) * 128) = x[q];
                }
            }
            fence_async_smem();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) ready_arrive<CG>(&sm.ready[rpos.slot]);
            ++s;
            ring_next(rpos, p.ring);
        }
    }
    return true;
}

// chunks per index: 1..8 bipolar (F16 <= 128), 1..16 unipolar (round16(L) <= 256)
#define SC_CPD_DISPATCH(cpd, CALL)           \
    if constexpr (UNI) {                     \
        switch (cpd) {                       \
            case 1: ok = CALL(1); break;     \
            case 2: ok = CALL(2); break;     \
            case 3: ok = CALL(3); break;     \
            case 4: ok = CALL(4); break;     \
            case 5: ok = CALL(5); break;     \
            case 6: ok = CALL(6); break;     \
            case 7: ok = CALL(7); break;     \
            case 8: ok = CALL(8); break;     \
            case 9: ok = CALL(9); break;     \
            case 10: ok = CALL(10); break;   \
            case 11: ok = CALL(11); break;   \
            case 12: ok = CALL(12); break;   \
            case 13: ok = CALL(13); break;   \
            case 14: ok = CALL(14); break;   \
            case 15: ok = CALL(15); break;   \
            default: ok = CALL(16); break;   \
        }                                    \
    } else {                                 \
        switch (cpd) {                       \
            case 1: ok = CALL(1); break;     \
            case 2: ok = CALL(2); break;     \
            case 3: ok = CALL(3); break;     \
            case 4: ok = CALL(4); break;     \
            case 5: ok = CALL(5); break;     \
            case 6: ok = CALL(6); break;     \
            case 7: ok = CALL(7); break;     \
            default: ok = CALL(8); break;    \
        }                                    \
    }


// GSUM (with bands): the fp64 running sum over bands lives in a global
// workspace laid out like the output instead of in tensor memory, so the
// kernel keeps the wide tiles, the 16-warp layout and the epilogue of the
// no-band kernel.
// UNI: the unipolar AND mode (thermometer of n = C_A[2|x_a|][L] ones against
// sgn_b K_B[2|x_b|, .] over the L stream positions; out = s s q^2 count / L).
// CG: CTAs per MMA -- 2, a cluster of two CTAs on two SMs issuing
// cta_group::2 MMAs of M = 256 (launched with a cluster dimension of 2); 1,
// each CTA alone with M = 128 (tiles of at most 64 columns).
template <int SKB, bool BANDS, bool BSCALE = false, bool GSUM = false, bool UNI = false, int CG = 2>
__global__ void __launch_bounds__(BANDS && !GSUM ? THREADS : THREADS_PLAIN, 1)
    tc_kernel(const __grid_constant__ TcArgs p) {
    constexpr bool PLAIN = !BANDS;
    constexpr bool WIDE = !BANDS || GSUM;  // 16 warps, 8 epilogue warps
    static_assert(BANDS || !BSCALE, "per-band scales need bands");
    static_assert(BANDS || !GSUM, "the workspace sum needs bands");
    constexpr int NT = WIDE ? THREADS_PLAIN : THREADS;
    // epilogue warps 0-3 and, in the 16-warp variants, 12-15 (two per TMEM
    // lane quadrant); B producers: warps 8-10.  (Warps 12-15 as B producers,
    // two threads per column, measured slower: the epilogue then lags.)
    constexpr int EPI = WIDE ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS;
    constexpr int NBW = NUM_B_WARPS;
    constexpr int NBT = NBW * 32;
    // the leftover-row kernel that follows reads nothing this kernel writes:
    // let it start on SMs as soon as this kernel's CTAs leave them
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &sm.abort_flag;
    const int rank = CG == 2 ? (int)cluster_rank() : 0;
    // the unit that takes work items: a cluster of two CTAs, or one CTA
    const int64_t pair = CG == 2 ? cluster_id() : blockIdx.x;
    const int64_t n_pairs = CG == 2 ? cluster_count() : gridDim.x;
    const int nb = p.n_bands > 0 ? p.n_bands : 1;

    // the A operand's chunk patterns (the same for every length)
    stage_u_patterns(sm.utab, threadIdx.x, NT);
    // per-rung (w, sgn, L - n) tables of the ladder lengths (no bands)
    for (int i = threadIdx.x; i < p.n_rungs * (p.Q + 1); i += NT) {
        const int k = i / (p.Q + 1), a = i % (p.Q + 1);
        sm.aw[k][a] = __ldg(p.Aw + (int64_t)p.lidx[k] * (p.Q + 1) + a);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < MAX_STAGES; ++s) {
            // the first CTA's ready counts the producer warps of both SMs
            // producer warps of every SM of the MMA: A warps and B warps, or
            // A warps and one relay arrival per SM with prepared B stages
            mbar_init(&sm.ready[s], CG * (NUM_A_WARPS + (p.bprep ? 1 : NBW)));
            mbar_init(&sm.empty[s], 1);
            mbar_init(&sm.bfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], CG * EPI);  // every epilogue warp of the MMA's SMs
            mbar_init(&sm.rinfo_full[b], NUM_A_WARPS);
            mbar_init(&sm.rinfo_empty[b], EPI);
        }
        mbar_init(&sm.bgrp, NBW);
        mbar_init(&sm.agrp, NUM_A_WARPS);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        if constexpr (CG == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_addr(&sm.tmem_base)),
                         "r"(TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_addr(&sm.tmem_base)),
                         "r"(TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    // items per unit, then an exclusive prefix over units (warp 0)
    const int U = p.n_groups * p.n_rungs;
    for (int u = threadIdx.x; u < U; u += NT) {
        const int64_t g = p.g_begin + u % p.n_groups;
        const int k = u / p.n_groups;
        const int32_t *o = p.offs + g * (p.n_rungs + 1);
        const int o0 = __ldg(o + k), cnt = max(__ldg(o + k + 1) - o0, 0);
        sm.urow0[u] = o0;
        sm.ucnt[u] = cnt;
        sm.ubase[u + 1] = unit_items<UNI, CG>(p, cnt, k);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int u0 = 0; u0 < U; u0 += 32) {
            const int u = u0 + lane;
            int v = u < U ? sm.ubase[u + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (u < U) sm.ubase[u + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) sm.ubase[0] = 0;
    }
    // both CTAs of the pair: barriers initialised and tensor memory allocated
    // before any cross-CTA arrive or MMA
    if (CG == 2) cluster_sync();
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int32_t *ubase = sm.ubase;

    // Balanced deal (see BAL_MAX): every CTA sorts the launch's items by
    // their stage count, largest first, ties in item order (which keeps
    // together the items that read the same prepared B stages), with the B
    // ring as scratch before any producer writes it; unit `pair` then takes
    // the sorted positions pair, 2P - 1 - pair, 2P + pair, ... (snake order),
    // so that every unit's total is close to the mean.
    {
        const int T = ubase[U];
        const bool bal = p.balance && T > 0 && T <= BAL_MAX && (T + n_pairs - 1) / n_pairs <= PLIST_MAX;
        if (bal) {
            uint32_t *key = reinterpret_cast<uint32_t *>(sm.bring);
            int32_t *scost = reinterpret_cast<int32_t *>(sm.bring + BAL_MAX * sizeof(uint32_t));
            const int nseg = p.ksplit;
            for (int e = threadIdx.x; e < p.n_rungs * nseg; e += NT) {  // stages per (rung, segment)
                const int k = e / nseg, sg = e % nseg;
                int b_lo = 0, b_hi = 1;
                if (p.n_bands > 0) {
                    const int per = p.n_bands / nseg;
                    b_lo = sg * per;
                    b_hi = b_lo + per;
                }
                Item tk{};
                tk.k = k;
                int64_t c = 0;
                for (int b = b_lo; b < b_hi; ++b) c += band_of<SKB, UNI>(p, tk, b).n_stages;
                scost[e] = (int32_t)min(c, (int64_t)BAL_COST_MAX);
            }
            __syncthreads();
            int T2 = 1;
            while (T2 < T) T2 <<= 1;
            for (int i = threadIdx.x; i < T2; i += NT) {
                uint32_t kv = 0xFFFFFFFFu;  // padding sorts last
                if (i < T) {
                    Walker w;
                    walker_seek(ubase, U, w, i);
                    const Item it = make_item<CG>(p, sm, w, i, 0);
                    const uint32_t c = min((uint32_t)scost[it.k * nseg + it.seg] + BAL_ITEM_STAGES,
                                           (uint32_t)BAL_COST_MAX);
                    kv = ((uint32_t)(BAL_COST_MAX - c) << 11) | (uint32_t)i;
                }
                key[i] = kv;
            }
            __syncthreads();
            for (int kk = 2; kk <= T2; kk <<= 1) {  // bitonic sort, ascending
                for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                    for (int i = threadIdx.x; i < T2; i += NT) {
                        const int ixj = i ^ jj;
                        if (ixj > i) {
                            const uint32_t a = key[i], b = key[ixj];
                            if ((a > b) == ((i & kk) == 0)) {
                                key[i] = b;
                                key[ixj] = a;
                            }
                        }
                    }
                    __syncthreads();
                }
            }
            if (threadIdx.x == 0) {
                int n = 0;
                for (int64_t r = 0; r * n_pairs < T; ++r) {
                    const int64_t pos = r * n_pairs + ((r & 1) ? n_pairs - 1 - pair : pair);
                    if (pos < T) sm.plist[n++] = (int32_t)(key[pos] & 0x7FFu);
                }
                sm.nplist = n;
            }
        } else if (threadIdx.x == 0) {
            sm.nplist = -1;
        }
        __syncthreads();
    }
    const int32_t *plist = sm.plist;
    const int nplist = sm.nplist;
    bool range_bad = false;

    // Every role walks the same items and, per item, the same bands; the
    // accumulator buffers and row-info slots alternate per (item, band).
    if (warp >= A_WARP0 && warp < B_WARP0) {
        // ================= A producers: U rows into the TMEM ring =================
        const int quad = warp & 3;
        const int r = quad * 32 + lane;                     // row of this CTA = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        Walker wk;
        RingPos rp;
        uint32_t acc_count = 0, n_gsync = 0;
        int loaded = -1;
        bool ok = true;
        // items run software-pipelined: the next item's entry of the row
        // order is loaded before this item's stages, its first window of
        // levels after them, so that an item starts without waiting on memory
        int j = 0;
        int64_t id = 0;
        bool have = sched_item(plist, nplist, ubase, U, pair, n_pairs, j, wk, id);
        Item it{};
        int64_t orow = -1;
        bool has_pre = false;
        uint4 pre = make_uint4(0, 0, 0, 0);
        if (have) {
            it = make_item<CG>(p, sm, wk, id, rank);
            if (r < it.rows) orow = it.g * p.M + __ldg(p.perm + it.g * p.M + it.row0 + r);
        }
        while (ok && have) {
            int64_t nid = 0;
            Walker nwk = wk;
            const bool nhave = sched_item(plist, nplist, ubase, U, pair, n_pairs, j + 1, nwk, nid);
            Item nit{};
            int64_t norow = -1;
            if (nhave) {
                nit = make_item<CG>(p, sm, nwk, nid, rank);
                if (r < nit.rows) norow = nit.g * p.M + __ldg(p.perm + nit.g * p.M + nit.row0 + r);
            }
            const bool a_ok = r < it.rows;
            const uint8_t *row = a_ok ? p.a_lv + orow * p.lda : nullptr;
            float sa = (a_ok && !BSCALE) ? __ldg(p.a_s + orow) : 0.0f;
            for (int b = it.b_lo; b < it.b_hi; ++b, ++acc_count) {
                const Band bd = band_of<SKB, UNI>(p, it, b);
                const int cpd = bd.F16 >> 4;
                if (p.n_bands > 0 && bd.lidx != loaded) {
                    // with bands, stage this length's (w, sign, L - n) map
                    if (!group_sync(&sm.agrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    for (int a = r; a <= p.Q; a += NUM_A_WARPS * 32)
                        sm.awb[a] = __ldg(p.Aw + (int64_t)bd.lidx * (p.Q + 1) + a);
                    if (!group_sync(&sm.agrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    loaded = bd.lidx;
                }
                const int32_t *aw = p.n_bands > 0 ? sm.awb : sm.aw[it.k];
                const uint8_t *tab = sm.utab + (lane & (REP - 1)) * 16;
                int Rsum = 0;  // row constant sum_{d in band} (L - n_{a_id})
                const bool use_pre = has_pre && b == it.b_lo;
#define SC_A_CALL(C)                                                                              \
    produce_a<SKB, C, CG>(p, sm, bd, aw, row, a_ok, tab, lane_base, rp, Rsum, abort_flag, range_bad, \
                          use_pre, pre)
                SC_CPD_DISPATCH(cpd, SC_A_CALL)
#undef SC_A_CALL
                if (!ok) break;
                if (b == it.b_hi - 1) {  // the next item's first window, ahead
                    has_pre = nhave && norow >= 0;
                    if (has_pre) {
                        const Band nbd = band_of<SKB, UNI>(p, nit, nit.b_lo);
                        pre = load_levels16_cap(p.a_lv + norow * p.lda, nbd.d_lo, nbd.d_hi, p.lda);
                    }
                }
                // publish this row's constant and factors for the epilogue
                const int buf = acc_count & 1;
                if (!wait_warp(&sm.rinfo_empty[buf], ((acc_count >> 1) & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                RowInfo ri;
                ri.obase = a_ok ? orow * p.N + it.n0 : -1;
                if (BSCALE) sa = a_ok ? __ldg(p.a_s + orow * nb + b) : 0.0f;
                ri.fd = (double)sa * p.q2d;
                ri.R = Rsum;
                ri.f = a_ok ? (float)((double)sa * p.q2d / (double)bd.L) : 0.0f;
                sm.rowinfo[buf][r] = ri;
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.rinfo_full[buf]);
            }
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            it = nit;
            orow = norow;
            wk = nwk;
            id = nid;
            have = nhave;
            ++j;
        }
    } else if (warp >= B_WARP0 && warp < MMA_WARP && p.bprep) {
        // ============ prepared B: bulk copies of whole stages, relayed to the MMA ============
        // lane 0 of warp 8 issues the copies (each after its slot is free),
        // lane 0 of warp 9 waits for them to land and signals "ready"
        if (lane == 0 && (warp == B_WARP0 || warp == B_WARP0 + 1)) {
            const bool issuer = warp == B_WARP0;
            Walker wk;
            RingPos rpos;
            bool ok = true;
            int pend_ph[MAX_STAGES];  // issuer: parity of the copy in flight per slot, or -1
            for (int i = 0; i < MAX_STAGES; ++i) pend_ph[i] = -1;
            int64_t id = 0;
            for (int j = 0; ok && sched_item(plist, nplist, ubase, U, pair, n_pairs, j, wk, id); ++j) {
                const Item it = make_item<CG>(p, sm, wk, id, rank);
                const int nt = it.n0 / p.tile_w;
                const uint32_t bytes = (uint32_t)(it.chalf * SKB);
                for (int b = it.b_lo; ok && b < it.b_hi; ++b) {
                    const Band bd = band_of<SKB, UNI>(p, it, b);
                    const int slot_u = (p.n_bands > 0 ? b : 0) * p.n_rungs + it.k;
                    const uint8_t *src0 =
                        p.bprep + __ldg(p.bprep_off + slot_u) +
                        ((int64_t)((it.g * p.n_ntiles + nt) * 2 + rank) * bd.n_stages) * BPREP_BLOCK;
                    if (issuer)
                        for (int s = 0; s < min(BPREP_PREFETCH, bd.n_stages); ++s)
                            prefetch_l2(src0 + (int64_t)s * BPREP_BLOCK, bytes);
                    for (int s = 0; s < bd.n_stages; ++s) {
                        if (issuer) {
                            if (!mbar_wait(&sm.empty[rpos.slot], rpos.ph ^ 1u, abort_flag)) {
                                ok = false;
                                break;
                            }
                            if (s + BPREP_PREFETCH < bd.n_stages)
                                prefetch_l2(src0 + (int64_t)(s + BPREP_PREFETCH) * BPREP_BLOCK, bytes);
                            mbar_expect_tx(&sm.bfull[rpos.slot], bytes);
                            bulk_copy_g2s(sm.bring + rpos.slot * p.bslot, src0 + (int64_t)s * BPREP_BLOCK,
                                          bytes, &sm.bfull[rpos.slot]);
                            pend_ph[rpos.slot] = (int)rpos.ph;
                        } else {
                            if (!mbar_wait(&sm.bfull[rpos.slot], rpos.ph, abort_flag)) {
                                ok = false;
                                break;
                            }
                            ready_arrive<CG>(&sm.ready[rpos.slot]);
                        }
                        ring_next(rpos, p.ring);
                    }
                }
                if (*abort_flag) break;
            }
            if (issuer) {
                // every copy this CTA issued has landed before its shared
                // memory can be released (bounded, even when aborting)
                for (int sl = 0; sl < MAX_STAGES; ++sl) {
                    if (pend_ph[sl] < 0) continue;
                    const long long t0 = clock64();
                    while (!mbar_try_wait(&sm.bfull[sl], (uint32_t)pend_ph[sl])) {
                        if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
                            *abort_flag = 1;
                            break;
                        }
                    }
                }
            }
        }
    } else if (warp >= B_WARP0 && warp < MMA_WARP) {
        // ================= B producers: P_L rows into shared-memory tiles =================
        const int bt = threadIdx.x - B_WARP0 * 32;  // 0..NBT-1
        Walker wk;
        RingPos rpos;
        uint32_t n_gsync = 0;
        int loaded = -1;
        bool ok = true;
        bool has_pre = false;
        uint4 pre = make_uint4(0, 0, 0, 0);
        int64_t id = 0;
        for (int j = 0; ok && sched_item(plist, nplist, ubase, U, pair, n_pairs, j, wk, id); ++j) {
            const Item it = make_item<CG>(p, sm, wk, id, rank);
            for (int b = it.b_lo; b < it.b_hi; ++b) {
                const Band bd = band_of<SKB, UNI>(p, it, b);
                const int cpd = bd.F16 >> 4;
                if (bd.lidx != loaded) {
                    // stage this length's chunk tables (replicated) and class maps
                    if (!group_sync(&sm.bgrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    stage_replicated(sm.ptab, p.Pk + __ldg(p.pk_off + bd.lidx), cpd * PK_ROWS, bt, NBT);
                    {
                        const uint4 *src =
                            reinterpret_cast<const uint4 *>(p.Pmap + (int64_t)bd.lidx * (p.Q + 1) * PMAP_STRIDE);
                        for (int e = bt; e <= p.Q; e += NBT)
                            reinterpret_cast<uint4 *>(sm.pmap)[e] = __ldg(src + e);
                    }
                    if (!group_sync(&sm.bgrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    loaded = bd.lidx;
                }
                const bool use_pre = has_pre && b == it.b_lo;
#define SC_B_CALL(C) \
    produce_b<SKB, C, CG>(p, sm, it, bd, bt, NBT, rpos, abort_flag, range_bad, use_pre, pre)
                SC_CPD_DISPATCH(cpd, SC_B_CALL)
#undef SC_B_CALL
                if (!ok) break;
                if (b == it.b_hi - 1) {  // the next item's first window of this column, ahead
                    Walker nwk = wk;
                    int64_t nid = 0;
                    has_pre = sched_item(plist, nplist, ubase, U, pair, n_pairs, j + 1, nwk, nid);
                    if (has_pre) {
                        const Item nit = make_item<CG>(p, sm, nwk, nid, rank);
                        const Band nbd = band_of<SKB, UNI>(p, nit, nit.b_lo);
                        int G, grp, bc;
                        const uint8_t *nrp = b_column(p, nit, bt, NBT, SKB / 16, G, grp, bc);
                        pre = load_levels16_cap(nrp, nbd.d_lo, nbd.d_hi, p.ldb);
                    }
                }
            }
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
        }
    } else if (warp == MMA_WARP) {
        Walker wk;
        RingPos rp;
        uint32_t acc_count = 0;
        bool ok = true;
        if (rank == 1) {
            // second CTA: its producers signal the first CTA directly
        } else {
            // ================= MMA issuer (first CTA of the pair) =================
            int64_t id = 0;
            for (int j = 0; ok && sched_item(plist, nplist, ubase, U, pair, n_pairs, j, wk, id); ++j) {
                const Item it = make_item<CG>(p, sm, wk, id, rank);
                const uint32_t idesc = make_idesc(CG * TM, it.nw);
                for (int b = it.b_lo; ok && b < it.b_hi; ++b, ++acc_count) {
                    const int n_stages = band_of<SKB, UNI>(p, it, b).n_stages;
                    const int buf = acc_count & 1;
                    const uint32_t aph = (acc_count >> 1) & 1u;
                    if (!wait_warp(&sm.acc_empty[buf], aph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tacc = tmem + (uint32_t)(buf * p.acc_stride);
                    // Stages are taken in batches of MMA_BATCH: wait until they
                    // are filled (both SMs), then issue all their MMAs back to back.
                    for (int s = 0; s < n_stages;) {
                        const int nbat = min(MMA_BATCH, n_stages - s);
                        RingPos q = rp;
                        for (int i = 0; i < nbat; ++i, ring_next(q, p.ring)) {
                            if (!wait_warp(&sm.ready[q.slot], q.ph, abort_flag)) {
                                ok = false;
                                break;
                            }
                        }
                        if (!ok) break;
                        tc_fence_after();
                        if (lane == 0) {
                            q = rp;
                            for (int i = 0; i < nbat; ++i, ring_next(q, p.ring)) {
                                const uint32_t a0 = tmem + p.ring_col + (uint32_t)(q.slot * (SKB / 4));
                                const uint32_t b0 = smem_addr(sm.bring + q.slot * p.bslot);
#pragma unroll
                                for (int kk = 0; kk < SKB / 32; ++kk) {
                                    const uint64_t db = make_desc(b0 + kk * 256, 128, (SKB / 16) * 128);
                                    mma_i8_ts<CG>(tacc, a0 + kk * 8, db, idesc,
                                                   (s + i > 0 || kk > 0) ? 1u : 0u);
                                }
                                mma_commit<CG>(&sm.empty[q.slot]);
                            }
                        }
                        __syncwarp();
                        for (int i = 0; i < nbat; ++i) ring_next(rp, p.ring);
                        s += nbat;
                    }
                    if (!ok) break;
                    if (lane == 0) mma_commit<CG>(&sm.acc_full[buf]);
                    __syncwarp();
                }
            }
            // drain: every MMA issued for the pair has completed before tensor
            // memory is freed (waited for even when aborting; bounded all the same)
            if (lane == 0) mma_commit<CG>(&sm.drain);
            __syncwarp();
            const long long t0 = clock64();
            while (!mbar_try_wait(&sm.drain, 0)) {
                if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
                    *abort_flag = 1;
                    break;
                }
            }
        }
    } else {
        // ================= epilogue (warps 0-3, and 12-15 without bands) =================
        // Each warp owns 32 TMEM lanes (rows) of its quadrant warp % 4; the
        // two warps of a quadrant take alternate 32-column blocks.  Per block: one
        // tcgen05.ld of 32 x 32 counts, a shared-memory transpose, then lane =
        // column and the warp walks the 32 rows, so every store instruction
        // writes 128 contiguous bytes of one output row.  Row constants,
        // factors and output rows come from the A producers (rowinfo).
        // With bands, each band's decode (2 count_b - D_b L_b) / L_b is added
        // to an fp64 running sum kept in tensor memory (two 32-bit columns per
        // output, at SUM_COL) and the last band writes the output.
        const int quad = warp & 3, esub = warp >> 2 == 3 ? 1 : 0, eslot = quad + 4 * esub;
        constexpr int CSTEP = WIDE ? 64 : 32;  // column-block stride of one warp
        uint32_t(*stg)[33] = sm.epi[eslot];
        float *sbw = sm.sbw[eslot];
        const uint32_t lane_quad = (uint32_t)(quad * 32) << 16;
        const uint32_t tsum = tmem + lane_quad + SUM_COL;
        Walker wk;
        uint32_t acc_count = 0;
        bool ok = true;
        int64_t id = 0;
        for (int j = 0; ok && sched_item(plist, nplist, ubase, U, pair, n_pairs, j, wk, id); ++j) {
            const Item it = make_item<CG>(p, sm, wk, id, rank);
            // column scales s^B_j of this tile (per-warp copy)
            __syncwarp();
            if (!BSCALE)
                for (int c = lane; c < it.nw; c += 32)
                    sbw[c] = c < it.nvalid ? __ldg(p.b_s + it.g * p.N + it.n0 + c) : 0.0f;
            __syncwarp();
            for (int b = it.b_lo; b < it.b_hi; ++b, ++acc_count) {
                const Band bd = band_of<SKB, UNI>(p, it, b);
                if (BSCALE) {
                    // this band's column scales s^B_jb
                    __syncwarp();
                    for (int c = lane; c < it.nw; c += 32)
                        sbw[c] = c < it.nvalid ? __ldg(p.b_s + (it.g * p.N + it.n0 + c) * nb + b) : 0.0f;
                    __syncwarp();
                }
                const int buf = acc_count & 1;
                const uint32_t aph = (acc_count >> 1) & 1u;
                if (!wait_warp(&sm.rinfo_full[buf], aph, abort_flag) ||
                    !wait_warp(&sm.acc_full[buf], aph, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const RowInfo *ri = sm.rowinfo[buf] + quad * 32;
                const uint32_t tbase = tmem + lane_quad + (uint32_t)(buf * p.acc_stride);
                // a warp whose 32 rows are all padding has nothing to store
                const int nw_live = __any_sync(0xffffffffu, ri[lane].obase >= 0) ? it.nw : 0;
                if constexpr (PLAIN) {
                    const float DL = (float)(p.D * (int64_t)bd.L);
                    for (int c0 = 32 * esub; c0 < nw_live; c0 += CSTEP) {
                        uint32_t v[32];
                        tmem_ld32(tbase + c0, v);
#pragma unroll
                        for (int u = 0; u < 32; ++u) stg[lane][u] = v[u];
                        __syncwarp();
                        const bool col_ok = c0 + lane < it.nvalid;
                        const float sb = sbw[c0 + lane];
                        float *outc = p.out + c0 + lane;
                        int32_t *cntc = p.counts ? p.counts + c0 + lane : nullptr;
#pragma unroll
                        for (int r8 = 0; r8 < 32; r8 += 8) {
                            // eight rows at a time: all shared-memory reads, then the stores
                            int64_t ob[8];
                            int cnt[8];
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                ob[i] = ri[r8 + i].obase;
                                cnt[i] = (int)stg[r8 + i][lane] + ri[r8 + i].R;
                                f[i] = ri[r8 + i].f;
                            }
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                if (col_ok && ob[i] >= 0) {
                                    outc[ob[i]] = UNI ? ((float)cnt[i] * f[i]) * sb
                                                      : ((2.0f * (float)cnt[i] - DL) * f[i]) * sb;
                                    if (cntc) cntc[ob[i]] = cnt[i];
                                }
                            }
                        }
                        __syncwarp();
                    }
                } else if constexpr (GSUM) {
                    // lane = column after the transpose; per row the band's term
                    // (2 count_b - D_b L_b) / L_b (times q^2 s^A_ib s^B_jb with
                    // per-band scales) is added to the fp64 sum of that output in
                    // the workspace; the last band writes the output instead.
                    // Each thread revisits the same outputs in every band, so its
                    // own program order orders the sum's reads and writes.
                    // With the tile's bands split in segments (ksplit > 1), each
                    // segment's last band writes its partial sum to its own
                    // slice of the workspace; the warp of the last segment to
                    // finish (counted per tile, CTA and warp) adds the slices in
                    // segment order and writes the output.
                    const bool first = b == it.b_lo, last = b == it.b_hi - 1;
                    const bool split = p.ksplit > 1;
                    const int64_t DbL = (bd.d_hi - bd.d_lo) * (int64_t)bd.L;
                    const double Ld = (double)bd.L;
                    for (int c0 = 32 * esub; c0 < nw_live; c0 += CSTEP) {
                        uint32_t v[32];
                        tmem_ld32(tbase + c0, v);
#pragma unroll
                        for (int u = 0; u < 32; ++u) stg[lane][u] = v[u];
                        __syncwarp();
                        const bool col_ok = c0 + lane < it.nvalid;
                        const double sb = (double)sbw[c0 + lane];
                        float *outc = p.out + c0 + lane;
                        double *sumc = p.gsum + it.seg * p.part_stride + c0 + lane;
                        int32_t *cntc =
                            p.counts ? p.counts + ((it.g * nb + b) - it.g) * p.M * p.N + c0 + lane : nullptr;
                        // the earlier bands' sums of 8 rows at a time, every load of a
                        // group issued before any is used: their latencies overlap
                        // (the sums have often left L2 since the previous band)
#pragma unroll
                        for (int r0 = 0; r0 < 32; r0 += 8) {
                            double prev[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int64_t ob = ri[r0 + u].obase;
                                prev[u] = (!first && col_ok && ob >= 0) ? sumc[ob] : 0.0;
                            }
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int row = r0 + u;
                                const int64_t ob = ri[row].obase;
                                if (col_ok && ob >= 0) {
                                    const int cnt = (int)stg[row][lane] + ri[row].R;
                                    if (cntc) cntc[ob] = cnt;
                                    double term = (double)(UNI ? (int64_t)cnt : 2LL * cnt - DbL) / Ld;
                                    if (BSCALE) term *= ri[row].fd * sb;
                                    const double acc = prev[u] + term;
                                    if (last && !split)
                                        outc[ob] = BSCALE ? (float)acc : (float)(acc * ri[row].fd * sb);
                                    else
                                        sumc[ob] = acc;
                                }
                            }
                        }
                        __syncwarp();
                    }
                    if (last && split && nw_live > 0) {
                        __threadfence();  // this lane's partial sums, before the count
                        __syncwarp();
                        int done = 0;
                        int32_t *ctr = p.tile_cnt + (it.tile * 2 + rank) * MAX_EPI_WARPS + eslot;
                        if (lane == 0) done = atomicAdd(ctr, 1) + 1;
                        done = __shfl_sync(0xffffffffu, done, 0);
                        if (done == p.ksplit) {
                            __threadfence();  // the other segments' partial sums, after the count
                            if (lane == 0) *ctr = 0;  // ready for the next launch
                            for (int c0 = 32 * esub; c0 < nw_live; c0 += CSTEP) {
                                const bool col_ok = c0 + lane < it.nvalid;
                                const double sb = (double)sbw[c0 + lane];
                                float *outc = p.out + c0 + lane;
                                const double *sum0 = p.gsum + c0 + lane;
#pragma unroll 4
                                for (int row = 0; row < 32; ++row) {
                                    const int64_t ob = ri[row].obase;
                                    if (col_ok && ob >= 0) {
                                        double acc = __ldcg(sum0 + ob);
                                        for (int sgm = 1; sgm < p.ksplit; ++sgm)
                                            acc += __ldcg(sum0 + sgm * p.part_stride + ob);
                                        outc[ob] = BSCALE ? (float)acc : (float)(acc * ri[row].fd * sb);
                                    }
                                }
                            }
                        }
                    }
                } else {
                    const bool last = b == it.b_hi - 1;
                    constexpr bool bscale = BSCALE;
                    const RowInfo me = ri[lane];
                    const int64_t DbL = (bd.d_hi - bd.d_lo) * (int64_t)bd.L;
                    const double Ld = (double)bd.L;
                    for (int c0 = 0; c0 < nw_live; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tbase + c0, v);
                        const bool col_ok = c0 + lane < it.nvalid;
                        if (p.counts) {
#pragma unroll
                            for (int u = 0; u < 32; ++u) stg[lane][u] = v[u];
                            __syncwarp();
                            // counts[g][b][i][j] = counts + (g nb + b - g) M N + obase
                            int32_t *cntc = p.counts + ((it.g * nb + b) - it.g) * p.M * p.N + c0 + lane;
#pragma unroll 8
                            for (int row = 0; row < 32; ++row) {
                                const int64_t ob = ri[row].obase;
                                if (col_ok && ob >= 0) cntc[ob] = (int)stg[row][lane] + ri[row].R;
                            }
                            __syncwarp();
                        }
                        float fo[32];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t s[32];
                            if (b > it.b_lo) {
                                tmem_ld32(tsum + (uint32_t)(2 * (c0 + 16 * h)), s);
                            } else {
#pragma unroll
                                for (int e = 0; e < 32; ++e) s[e] = 0u;
                            }
#pragma unroll
                            for (int uu = 0; uu < 16; ++uu) {
                                const int u = 16 * h + uu;
                                const int cnt = (int)v[u] + me.R;
                                double acc = __hiloint2double((int)s[2 * uu + 1], (int)s[2 * uu]);
                                // per-band scales: q^2 s^A_ib s^B_jb weighs each band's
                                // term; otherwise the row scales multiply the sum
                                if (bscale) {
                                    acc += (double)(UNI ? (int64_t)cnt : 2LL * cnt - DbL) / Ld *
                                           (me.fd * (double)sbw[c0 + u]);
                                } else {
                                    acc += (double)(UNI ? (int64_t)cnt : 2LL * cnt - DbL) / Ld;
                                }
                                if (last) {
                                    fo[u] = bscale ? (float)acc : (float)(acc * me.fd * (double)sbw[c0 + u]);
                                } else {
                                    s[2 * uu] = (uint32_t)__double2loint(acc);
                                    s[2 * uu + 1] = (uint32_t)__double2hiint(acc);
                                }
                            }
                            if (!last) tmem_st32(tsum + (uint32_t)(2 * (c0 + 16 * h)), s);
                        }
                        if (last) {
#pragma unroll
                            for (int u = 0; u < 32; ++u) stg[lane][u] = __float_as_uint(fo[u]);
                            __syncwarp();
                            float *outc = p.out + c0 + lane;
#pragma unroll 8
                            for (int row = 0; row < 32; ++row) {
                                const int64_t ob = ri[row].obase;
                                if (col_ok && ob >= 0) outc[ob] = __uint_as_float(stg[row][lane]);
                            }
                            __syncwarp();
                        }
                    }
                    if (!last) tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (CG == 2) mbar_arrive_cluster(&sm.acc_empty[buf], 0);
                    else mbar_arrive(&sm.acc_empty[buf]);
                    mbar_arrive(&sm.rinfo_empty[buf]);
                }
            }
        }
    }

    // both CTAs: all MMAs drained, no cross-CTA traffic outstanding
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();
    else __syncthreads();
    tc_fence_after();
    if (warp == 0)
    {
        if constexpr (CG == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(TMEM_COLS)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(TMEM_COLS)
                         : "memory");
    }
    if (threadIdx.x == 0 && sm.abort_flag && p.dev_status) atomicOr(p.dev_status, SC_DEV_WAIT_LIMIT);
    if (range_bad && p.dev_status) atomicOr(p.dev_status, SC_DEV_LEVEL_RANGE);
}


using TcKernelFn = void (*)(TcArgs);
// one getter per instantiated variant (defined in sc_tc_k_*.cu)
TcKernelFn tc_kernel_plain();
TcKernelFn tc_kernel_single();       // one CTA per MMA (M = 128), no bands, tiles <= 64 columns
TcKernelFn tc_kernel_single_uni();
TcKernelFn tc_kernel_plain_uni();
TcKernelFn tc_kernel_bands();
TcKernelFn tc_kernel_bands_bs();
TcKernelFn tc_kernel_bands_uni();
TcKernelFn tc_kernel_bands_bs_uni();
TcKernelFn tc_kernel_bands_ws();
TcKernelFn tc_kernel_bands_ws_bs();
TcKernelFn tc_kernel_bands_ws_uni();
TcKernelFn tc_kernel_bands_ws_bs_uni();

}  // namespace tcd
}  // namespace scb
