// sc_tc.cu -- tcgen05 (5th-generation tensor core) count engine for sm_100a.
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
// (s32 accumulators in tensor memory), which is exact.
//
// Kernel layout: clusters of two CTAs on two SMs run one `cta_group::2` MMA
// of M = 256 rows (128 per SM) x N <= 192 columns; each SM expands its own
// 128 rows of A and half of the N columns of B.  Per CTA (12 warps):
//   warps 0-3   epilogue: tcgen05.ld of this SM's accumulator rows, decode
//               C = s_i s_j q^2 (2 count - D L) / L, store
//   warps 4-7   A producers: one thread per row computes its U bytes from
//               (w, sgn) of each level and writes them into a tensor-memory
//               ring with tcgen05.st (the MMA reads A from tensor memory)
//   warps 8-10  B producers: one thread per column copies P_L row slices from
//               a compressed, replicated shared-memory table into this SM's
//               half of the K-major UMMA B tile
//   warp  11    in the pair's first CTA, one thread issues the MMAs for both
//               SMs and the multicast commits
// Work items are (group, rung, 256-row tile of the rung-sorted rows, column
// tile); every row of an item runs the same stream length, so early
// termination is real: an item costs D * ceil(L/2) per MAC lane.
// All waits on mbarriers are bounded; on expiry the kernel records
// SC_DEV_WAIT_LIMIT, drains its own MMAs, frees tensor memory and returns.
#include <stdint.h>

#include "sc_internal.cuh"

namespace scb {

namespace {

constexpr int TM = 128;                    // rows per CTA (TMEM lanes)
constexpr int PM = 2 * TM;                 // rows per pair tile (UMMA M = 256)
constexpr int TNMAX = 160;                 // max columns per pair tile (UMMA N, multiple of 32)
constexpr int BC = TNMAX / 2;              // B columns staged per CTA
// Pipeline stages: SKB contraction bytes per stage (SKB/32 UMMA K-steps, one
// barrier round trip each).  Every wait and every tcgen05.mma has a fixed
// cost of a few hundred cycles in this kernel, so stages are as deep as
// tensor memory allows: 256 bytes without bands, 128 with bands.
constexpr int SK_PLAIN = 256, SK_BANDS = 256, SK_NARROW = 512;
constexpr int TN_NARROW = 64;  // column tiles of at most 64: 512-byte stages
constexpr int RING_PLAIN = 3, RING_BANDS = 4;
constexpr int MAX_STAGES = 4;
constexpr int B_RING_BYTES = 60 * 1024;    // B ring: 3 x 80 x 256 or 4 x 80 x 128 bytes
static_assert(RING_PLAIN * BC * SK_PLAIN <= B_RING_BYTES, "B ring");
// Tensor memory (512 columns x 128 lanes of 32 bits per SM):
//   no bands: accumulators [0, 160) and [160, 320), A ring of 3 x 64 at 320;
//   bands:    accumulators [0, 64) and [64, 128), fp64 running sum (two
//             columns per output) at [128, 256), A ring of 4 x 64 at 256.
constexpr int TNMAX_BANDS = 64;
static_assert(RING_BANDS * (TNMAX_BANDS / 2) * SK_BANDS <= B_RING_BYTES, "B ring (bands)");
constexpr uint32_t SUM_COL = 2 * TNMAX_BANDS;
#ifndef SC_MMA_BATCH
#define SC_MMA_BATCH 1
#endif
constexpr int MMA_BATCH = SC_MMA_BATCH;  // ring stages per round of MMA issue (< ring)
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
constexpr int PTAB_BYTES = 48 * 1024;  // compressed P_L, replicated (see stage_table)
constexpr int UTAB_BYTES = 37120;      // compressed U_L: 257 rows x 9 entries x 16 B at rep 1
constexpr int UMAX = 2048;             // (group, rung) units per launch

static_assert(2 * TNMAX + RING_PLAIN * SK_PLAIN / 4 <= TMEM_COLS, "TMEM budget (no bands)");
static_assert(2 * TN_NARROW + RING_PLAIN * SK_NARROW / 4 <= TMEM_COLS, "TMEM budget (narrow)");
static_assert(RING_PLAIN * (TN_NARROW / 2) * SK_NARROW <= B_RING_BYTES, "B ring (narrow)");
static_assert(SUM_COL + 2 * TNMAX_BANDS + RING_BANDS * SK_BANDS / 4 <= TMEM_COLS, "TMEM budget (bands)");
static_assert(RING_PLAIN <= MAX_STAGES && RING_BANDS <= MAX_STAGES, "ring slots");

struct TcArgs {
    int64_t M, N, D, batch;
    const uint8_t *a_lv;
    const float *a_s;
    const uint8_t *b_lv;
    const float *b_s;
    const int32_t *perm;
    const int32_t *offs;       // [batch][n_rungs + 1]
    const uint8_t *Pc;         // compressed P_L tables, [L+1][F16] each
    const int64_t *pc_off;     // byte offset of each length's table
    const uint8_t *rho;        // [n_lengths][256]: rho = C[b][L]
    const int32_t *Aw;         // [n_lengths][Q+1]: urow | (L - n) << 16
    const uint8_t *Uc;         // compressed U_L tables, [2F+1][F16] each
    const int64_t *uc_off;     // byte offset of each length's U table
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
};

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
    uint8_t rho[256];
    uint32_t epi[MAX_EPI_WARPS][32][33];   // per-warp 32 x 32 transpose of accumulator values
    RowInfo rowinfo[2][TM];     // per item (parity): written by the A producers
    float sbw[MAX_EPI_WARPS][TNMAX];  // per epilogue warp: column scales s^B_j of the tile
    int32_t aw[SC_MAX_RUNGS][257];
    int32_t awb[257];          // (urow, L - n) of the current band's length (A producers)
    int32_t ubase[UMAX + 1];   // exclusive prefix of work items over units (group, rung)
    uint64_t ready[MAX_STAGES];  // this CTA's producers (+ on the first CTA the second CTA's relay)
    uint64_t empty[MAX_STAGES];  // both CTAs: multicast MMA commit
    uint64_t acc_full[2];      // both CTAs: multicast MMA commit
    uint64_t acc_empty[2];     // first CTA: both SMs' epilogue warps arrive
    uint64_t rinfo_full[2];    // local: A producers -> epilogue
    uint64_t rinfo_empty[2];   // local: epilogue -> A producers
    uint64_t bgrp;             // local: B producer warps (table reloads)
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
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - t0 > WAIT_LIMIT_CYCLES || it > (1u << 30)) {
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

// Pair MMA: A from tensor memory (both SMs, same address), B from shared
// memory (each SM holds N/2 rows at the same offset), D in both SMs' TMEM.
__device__ __forceinline__ void mma_i8_ts_pair(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Commit the pair's outstanding MMAs to the barrier at this offset in both CTAs.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(smem_addr(bar)),
        "h"((uint16_t)3)
        : "memory");
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
__device__ __forceinline__ int f16_of(int L) { return (((L + 1) / 2) + 15) & ~15; }

__device__ __forceinline__ int unit_items(const TcArgs &p, int cnt, int k) {
    const int rem = cnt % PM;
    const int tiles = cnt / PM + (rem >= tc_min_rows(f16_of(p.len[k])) ? 1 : 0);
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

__device__ __forceinline__ Item make_item(const TcArgs &p, const int32_t *ubase, const Walker &w,
                                          int64_t id, int rank) {
    Item it;
    const int64_t local = id - ubase[w.u];
    // consecutive items are the band segments of one tile, dealt to
    // different pairs
    const int64_t tl = local / p.ksplit;
    it.seg = (int)(local % p.ksplit);
    it.tile = id / p.ksplit;
    {
        const int per = (p.n_bands > 0 ? p.n_bands : 1) / p.ksplit;
        it.b_lo = it.seg * per;
        it.b_hi = it.b_lo + per;
    }
    const int mt = (int)(tl / p.n_ntiles);
    const int nt = (int)(tl % p.n_ntiles);
    it.k = w.u / p.n_groups;  // units run rung-major: a pair's items mostly share L
    it.g = p.g_begin + w.u % p.n_groups;
    const int32_t *o = p.offs + it.g * (p.n_rungs + 1);
    const int row0 = __ldg(o + it.k), cnt = max(__ldg(o + it.k + 1) - row0, 0);
    const int pair_rows = min(PM, cnt - mt * PM);
    // a partial tile's rows are split between the two CTAs in whole warps
    // (32 TMEM lanes), as evenly as possible, so that the producer and
    // epilogue warps left without a valid row can skip their work
    const int h0 = min(TM, 32 * ((pair_rows + 63) / 64));
    it.row0 = row0 + mt * PM + (rank ? h0 : 0);
    it.rows = rank ? max(pair_rows - h0, 0) : min(pair_rows, h0);
    it.n0 = nt * p.tile_w;
    it.nvalid = (int)min((int64_t)p.tile_w, p.N - it.n0);
    it.nw = (it.nvalid + 31) & ~31;
    it.chalf = it.nw / 2;
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

template <int SKB>
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
    bd.F16 = f16_of(bd.L);
    bd.n_stages = (int)(((bd.d_hi - bd.d_lo) * bd.F16 + SKB - 1) / SKB);
    return bd;
}

// 16 levels of one row starting at d0, bytes at or past D read as 0.  A row
// that is not 16-byte aligned (odd D) is read as two aligned 16-byte words
// and funnel-shifted, as long as both words lie inside the row; only the
// last window of such a row falls back to byte loads.
__device__ __forceinline__ uint4 load_levels16(const uint8_t *row, int64_t d0, int64_t D) {
    if (row == nullptr || d0 >= D) return make_uint4(0, 0, 0, 0);
    const uintptr_t addr = reinterpret_cast<uintptr_t>(row + d0);
    const uint32_t k = (uint32_t)(addr & 15u);
    if (d0 + 16 <= D && k == 0) return __ldg(reinterpret_cast<const uint4 *>(addr));
    if (d0 + 32 - (int64_t)k <= D) {
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

// Level u (compile-time after unrolling) of a 16-level window.
__device__ __forceinline__ int lv_byte(const uint4 &c, int u) {
    const uint32_t w = (u >> 2) == 0 ? c.x : ((u >> 2) == 1 ? c.y : ((u >> 2) == 2 ? c.z : c.w));
    return (int)((w >> (8 * (u & 3))) & 0xffu);
}


// Contraction indices per level window of a producer: a whole number of
// stages always covers a whole number of windows.
template <int SKB>
__host__ __device__ constexpr int win_of() { return SKB >= SK_NARROW ? 32 : 16; }

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
__device__ __forceinline__ void ready_arrive(uint64_t *bar) {
    if (cluster_rank() == 0) mbar_arrive(bar);
    else mbar_arrive_cluster(bar, 0);
}

// ---- replicated tables ------------------------------------------------------
// A compressed table of `rows` rows x cpd 16-byte entries is staged with
// every entry repeated rep times: entry (row, jc, k) at (row * rs + jc * rep
// + k) * 16, and lane l reads replica l % rep.  With rep = 8 the 8 lanes of a
// shared-memory wavefront hit 8 different 16-byte bank groups whatever rows
// they read; with rep < 8 the row stride is padded by one entry so that rows
// do not alias onto the same banks.
__device__ __forceinline__ int pick_rep(int rows, int cpd, int cap_bytes, int &rs) {
    int rep = 8;
    for (;;) {
        rs = cpd * rep + (rep < 8 ? 1 : 0);
        if (rep == 1 || rows * rs * 16 <= cap_bytes) return rep;
        rep >>= 1;
    }
}

__device__ __forceinline__ void stage_table(uint8_t *dst, const uint8_t *src, int rows, int cpd,
                                            int rep, int rs, int t, int nt) {
    const int per_row = cpd * rep, n = rows * per_row;
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    for (int e = t; e < n; e += nt) {
        const int row = e / per_row, rem = e - row * per_row;
        *reinterpret_cast<uint4 *>(dst + (size_t)(row * rs + rem) * 16) = __ldg(s4 + row * cpd + rem / rep);
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
// row urow(a) of the staged compressed table (zeros for a dead contraction
// index), so a 16-byte chunk costs one shared-memory load.  A stage goes to
// tensor memory in 32-column pieces (8 chunks each).
template <int SKB, int CPD>
__device__ __forceinline__ bool produce_a(const TcArgs &p, Smem &sm, const Band &bd,
                                          const int32_t *aw, const uint8_t *row, bool a_ok,
                                          const uint8_t *tab, int rs16, int rep16,
                                          uint32_t lane_base, RingPos &rp, int &Rsum,
                                          volatile int *abort_flag, bool &range_bad) {
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
            if ((threadIdx.x & 31) == 0) ready_arrive(&sm.ready[rp.slot]);
            ring_next(rp, p.ring);
        }
        return true;
    }
    uint4 nxt[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) nxt[k] = load_levels16(row, bd.d_lo + 16 * k, bd.d_hi);
    int s = 0;
    for (int64_t d0 = bd.d_lo; s < bd.n_stages; d0 += WIN) {
        uint4 cur[NW];
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            cur[k] = nxt[k];
            nxt[k] = load_levels16(row, d0 + WIN + 16 * k, bd.d_hi);
        }
        const int nlive = a_ok ? (int)min((int64_t)WIN, bd.d_hi - d0) : 0;
#pragma unroll
        for (int t = 0; t < SPW; ++t) {
            if (s >= bd.n_stages) break;
#pragma unroll
            for (int h = 0; h < CH / 8; ++h) {
                uint32_t v[32];
                const uint8_t *rowp = tab;
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
                        rowp = tab + (live ? (e & 0xffff) : 0) * rs16;
                        // an index whose chunks straddle two pieces is counted once
                        if (live && jc == 0) Rsum += e >> 16;
                    }
                    const uint4 x = *reinterpret_cast<const uint4 *>(rowp + jc * rep16);
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
            if ((threadIdx.x & 31) == 0) ready_arrive(&sm.ready[rp.slot]);
            ++s;
            ring_next(rp, p.ring);
        }
    }
    return true;
}

// B: one column of this CTA's half of the pair tile per thread; each 16-byte
// chunk is a slice of row rho = C[b][L] of the staged compressed P_L table.
template <int SKB, int CPD>
__device__ __forceinline__ bool produce_b(const TcArgs &p, Smem &sm, const Item &it, const Band &bd,
                                          int bt, int rep, int rs16, RingPos &rpos,
                                          volatile int *abort_flag, bool &range_bad) {
    constexpr int CH = SKB / 16;
    constexpr int WIN = win_of<SKB>(), NW = WIN / 16;
    constexpr int SPW = WIN * CPD / CH;
    const int rep16 = rep * 16;
    // narrow tiles: G thread groups share each column, group g filling the
    // 8-chunk pieces h with h % G == g of every stage
    const int G = it.chalf > 48 ? 1 : (it.chalf > 32 ? 2 : min(3, CH / 8));
    const int span = B_THREADS / G, grp = bt / span, bc = bt - grp * span;
    const uint8_t *tab = sm.ptab + (bc & (rep - 1)) * 16;
    const bool c_ok = bc < it.chalf && grp < G;
    const int col = it.c0 + bc;  // within the pair tile
    const uint8_t *rp = (c_ok && col < it.nvalid) ? p.b_lv + (it.g * p.N + it.n0 + col) * p.D : nullptr;
    const uint32_t off = op_offset<SKB>(bc, 0);
    const int qmax = p.Q;
    uint4 nx[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) nx[k] = load_levels16(rp, bd.d_lo + 16 * k, bd.d_hi);
    int s = 0;
    for (int64_t d0 = bd.d_lo; s < bd.n_stages; d0 += WIN) {
        uint4 lv[NW];
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            lv[k] = nx[k];
            nx[k] = load_levels16(rp, d0 + WIN + 16 * k, bd.d_hi);
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
                    const uint8_t *rowp = tab;
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
                            rowp = tab + (int)sm.rho[b] * rs16;
                        }
                        x[q] = *reinterpret_cast<const uint4 *>(rowp + jc * rep16);
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4 *>(sb + off + (h * 8 + q) * 128) = x[q];
                }
            }
            fence_async_smem();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) ready_arrive(&sm.ready[rpos.slot]);
            ++s;
            ring_next(rpos, p.ring);
        }
    }
    return true;
}

#define SC_CPD_DISPATCH(cpd, CALL) \
    switch (cpd) {                 \
        case 1: ok = CALL(1); break; \
        case 2: ok = CALL(2); break; \
        case 3: ok = CALL(3); break; \
        case 4: ok = CALL(4); break; \
        case 5: ok = CALL(5); break; \
        case 6: ok = CALL(6); break; \
        case 7: ok = CALL(7); break; \
        default: ok = CALL(8); break; \
    }


// GSUM (with bands): the fp64 running sum over bands lives in a global
// workspace laid out like the output instead of in tensor memory, so the
// kernel keeps the wide tiles, the 16-warp layout and the epilogue of the
// no-band kernel.
template <int SKB, bool BANDS, bool BSCALE = false, bool GSUM = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(BANDS && !GSUM ? THREADS : THREADS_PLAIN, 1)
    tc_kernel(const __grid_constant__ TcArgs p) {
    constexpr bool PLAIN = !BANDS;
    constexpr bool WIDE = !BANDS || GSUM;  // 16 warps, 8 epilogue warps
    static_assert(BANDS || !BSCALE, "per-band scales need bands");
    static_assert(BANDS || !GSUM, "the workspace sum needs bands");
    constexpr int NT = WIDE ? THREADS_PLAIN : THREADS;
    constexpr int EPI = WIDE ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS;
    // the leftover-row kernel that follows reads nothing this kernel writes:
    // let it start on SMs as soon as this kernel's CTAs leave them
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &sm.abort_flag;
    const int rank = (int)cluster_rank();
    const int64_t pair = cluster_id(), n_pairs = cluster_count();
    const int nb = p.n_bands > 0 ? p.n_bands : 1;

    // per-rung (w, sgn, L - n) tables of the ladder lengths (no bands)
    for (int i = threadIdx.x; i < p.n_rungs * (p.Q + 1); i += NT) {
        const int k = i / (p.Q + 1), a = i % (p.Q + 1);
        sm.aw[k][a] = __ldg(p.Aw + (int64_t)p.lidx[k] * (p.Q + 1) + a);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < MAX_STAGES; ++s) {
            // the first CTA's ready counts the producer warps of both SMs
            mbar_init(&sm.ready[s], 2 * READY_ARRIVALS);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 2 * EPI);  // every epilogue warp of both SMs
            mbar_init(&sm.rinfo_full[b], NUM_A_WARPS);
            mbar_init(&sm.rinfo_empty[b], EPI);
        }
        mbar_init(&sm.bgrp, NUM_B_WARPS);
        mbar_init(&sm.agrp, NUM_A_WARPS);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&sm.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    // items per unit, then an exclusive prefix over units (warp 0)
    const int U = p.n_groups * p.n_rungs;
    for (int u = threadIdx.x; u < U; u += NT) {
        const int64_t g = p.g_begin + u % p.n_groups;
        const int k = u / p.n_groups;
        const int32_t *o = p.offs + g * (p.n_rungs + 1);
        sm.ubase[u + 1] = unit_items(p, max(__ldg(o + k + 1) - __ldg(o + k), 0), k);
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
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int32_t *ubase = sm.ubase;
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
        int loaded = -1, rep = 8, rs = 0;
        bool ok = true;
        for (int64_t id = pair; ok && walker_seek(ubase, U, wk, id); id += n_pairs) {
            const Item it = make_item(p, ubase, wk, id, rank);
            const bool a_ok = r < it.rows;
            const uint8_t *row = nullptr;
            int64_t orow = -1;
            float sa = 0.0f;
            if (a_ok) {
                orow = it.g * p.M + __ldg(p.perm + it.g * p.M + it.row0 + r);
                row = p.a_lv + orow * p.D;
                if (!BSCALE) sa = __ldg(p.a_s + orow);
            }
            for (int b = it.b_lo; b < it.b_hi; ++b, ++acc_count) {
                const Band bd = band_of<SKB>(p, it, b);
                const int cpd = bd.F16 >> 4;
                if (bd.lidx != loaded) {
                    // stage the compressed U_L (replicated) and, with bands,
                    // this length's (urow, L - n) map
                    const int rows = 2 * ((bd.L + 1) / 2) + 1;
                    rep = pick_rep(rows, cpd, UTAB_BYTES, rs);
                    if (!group_sync(&sm.agrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    stage_table(sm.utab, p.Uc + __ldg(p.uc_off + bd.lidx), rows, cpd, rep, rs, r,
                                NUM_A_WARPS * 32);
                    if (p.n_bands > 0)
                        for (int a = r; a <= p.Q; a += NUM_A_WARPS * 32)
                            sm.awb[a] = __ldg(p.Aw + (int64_t)bd.lidx * (p.Q + 1) + a);
                    if (!group_sync(&sm.agrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    loaded = bd.lidx;
                }
                const int32_t *aw = p.n_bands > 0 ? sm.awb : sm.aw[it.k];
                const uint8_t *tab = sm.utab + (lane & (rep - 1)) * 16;
                int Rsum = 0;  // row constant sum_{d in band} (L - n_{a_id})
#define SC_A_CALL(C)                                                                              \
    produce_a<SKB, C>(p, sm, bd, aw, row, a_ok, tab, rs * 16, rep * 16, lane_base, rp, Rsum, abort_flag, \
                 range_bad)
                SC_CPD_DISPATCH(cpd, SC_A_CALL)
#undef SC_A_CALL
                if (!ok) break;
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
        }
    } else if (warp >= B_WARP0 && warp < MMA_WARP) {
        // ================= B producers: P_L rows into shared-memory tiles =================
        const int bt = threadIdx.x - B_WARP0 * 32;  // 0..B_THREADS-1
        Walker wk;
        RingPos rpos;
        uint32_t n_gsync = 0;
        int loaded = -1, rep = 8, rs = 0;
        bool ok = true;
        for (int64_t id = pair; ok && walker_seek(ubase, U, wk, id); id += n_pairs) {
            const Item it = make_item(p, ubase, wk, id, rank);
            for (int b = it.b_lo; b < it.b_hi; ++b) {
                const Band bd = band_of<SKB>(p, it, b);
                const int cpd = bd.F16 >> 4;
                if (bd.lidx != loaded) {
                    // stage the compressed P_L (replicated) and the rho map for this length
                    rep = pick_rep(bd.L + 1, cpd, PTAB_BYTES, rs);
                    if (!group_sync(&sm.bgrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    stage_table(sm.ptab, p.Pc + __ldg(p.pc_off + bd.lidx), bd.L + 1, cpd, rep, rs, bt,
                                B_THREADS);
                    for (int e = bt; e < 256; e += B_THREADS)
                        sm.rho[e] = __ldg(p.rho + (int64_t)bd.lidx * 256 + e);
                    if (!group_sync(&sm.bgrp, n_gsync, abort_flag)) {
                        ok = false;
                        break;
                    }
                    loaded = bd.lidx;
                }
#define SC_B_CALL(C) produce_b<SKB, C>(p, sm, it, bd, bt, rep, rs * 16, rpos, abort_flag, range_bad)
                SC_CPD_DISPATCH(cpd, SC_B_CALL)
#undef SC_B_CALL
                if (!ok) break;
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
            for (int64_t id = pair; ok && walker_seek(ubase, U, wk, id); id += n_pairs) {
                const Item it = make_item(p, ubase, wk, id, rank);
                const uint32_t idesc = make_idesc(PM, it.nw);
                for (int b = it.b_lo; ok && b < it.b_hi; ++b, ++acc_count) {
                    const int n_stages = band_of<SKB>(p, it, b).n_stages;
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
                                    mma_i8_ts_pair(tacc, a0 + kk * 8, db, idesc,
                                                   (s + i > 0 || kk > 0) ? 1u : 0u);
                                }
                                mma_commit_pair(&sm.empty[q.slot]);
                            }
                        }
                        __syncwarp();
                        for (int i = 0; i < nbat; ++i) ring_next(rp, p.ring);
                        s += nbat;
                    }
                    if (!ok) break;
                    if (lane == 0) mma_commit_pair(&sm.acc_full[buf]);
                    __syncwarp();
                }
            }
            // drain: every MMA issued for the pair has completed before tensor
            // memory is freed (waited for even when aborting; bounded all the same)
            if (lane == 0) mma_commit_pair(&sm.drain);
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
        for (int64_t id = pair; ok && walker_seek(ubase, U, wk, id); id += n_pairs) {
            const Item it = make_item(p, ubase, wk, id, rank);
            // column scales s^B_j of this tile (per-warp copy)
            __syncwarp();
            if (!BSCALE)
                for (int c = lane; c < it.nw; c += 32)
                    sbw[c] = c < it.nvalid ? __ldg(p.b_s + it.g * p.N + it.n0 + c) : 0.0f;
            __syncwarp();
            for (int b = it.b_lo; b < it.b_hi; ++b, ++acc_count) {
                const Band bd = band_of<SKB>(p, it, b);
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
                                    outc[ob[i]] = ((2.0f * (float)cnt[i] - DL) * f[i]) * sb;
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
#pragma unroll 4
                        for (int row = 0; row < 32; ++row) {
                            const int64_t ob = ri[row].obase;
                            if (col_ok && ob >= 0) {
                                const int cnt = (int)stg[row][lane] + ri[row].R;
                                if (cntc) cntc[ob] = cnt;
                                double term = (double)(2LL * cnt - DbL) / Ld;
                                if (BSCALE) term *= ri[row].fd * sb;
                                const double acc = first ? term : sumc[ob] + term;
                                if (last && !split)
                                    outc[ob] = BSCALE ? (float)acc : (float)(acc * ri[row].fd * sb);
                                else
                                    sumc[ob] = acc;
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
                                    acc += (double)(2LL * cnt - DbL) / Ld * (me.fd * (double)sbw[c0 + u]);
                                } else {
                                    acc += (double)(2LL * cnt - DbL) / Ld;
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
                    mbar_arrive_cluster(&sm.acc_empty[buf], 0);
                    mbar_arrive(&sm.rinfo_empty[buf]);
                }
            }
        }
    }

    // both CTAs: all MMAs drained, no cross-CTA traffic outstanding
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    if (threadIdx.x == 0 && sm.abort_flag && p.dev_status) atomicOr(p.dev_status, SC_DEV_WAIT_LIMIT);
    if (range_bad && p.dev_status) atomicOr(p.dev_status, SC_DEV_LEVEL_RANGE);
}

// ---------------------------------------------------------------------------
// CUDA-core path for the rows a rung leaves over after its tensor-core tiles
// (fewer than tc_min_rows rows; typically the few outlier rows of an
// attention head that sit on the long rungs).  Each block first lists the
// leftover rows of its launch's units (group, rung) in shared memory (an
// exclusive prefix over units); one warp then takes one item = (leftover
// row, block of 32 * CPL columns), lane l owning columns l + 32 c.  CPL
// (1..5) is chosen per N so that the blocks waste the fewest lanes.  Per
// contraction index the count of (i, j, d) is
//     E_L[n][b] = (L - n) + C[b][n] - C[b][L - n],  n = C[a][L],
// one 16-bit load (through L1) from the per-length count table, whose rows
// are 256 levels wide so that the 32 lanes of a gather (one n, 32 columns' b)
// fall in one 512-byte row; n comes from the transposed byte copy Ct8[n][b]
// of the prefix counts.
// ---------------------------------------------------------------------------
constexpr int SR_THREADS = 256;
constexpr int SR_WARPS = SR_THREADS / 32;
constexpr int SR_DS = 64;            // contraction indices staged per round
constexpr int SR_MAX_CPL = 5;        // columns per lane, at most
constexpr int SR_UMAX = UMAX;        // units per launch

struct SmallArgs {
    int64_t M, N, D, batch;
    const uint8_t *a_lv;
    const float *a_s;
    const uint8_t *b_lv;
    const float *b_s;
    const int32_t *perm;
    const int32_t *offs;
    const uint8_t *Ct8;  // [(Q+1)][256]: Ct8[n][b] = C[b][n]
    const uint16_t *E;   // count tables E_L[n][b] per length
    const int64_t *e_off;
    int32_t len[SC_MAX_RUNGS];
    int32_t lidx[SC_MAX_RUNGS];
    int n_rungs, Q;
    int n_bands;         // 0: one band covering D
    int64_t chunk_d;
    const int32_t *blen; // [n_bands][n_rungs] band lengths (device)
    const int32_t *blidx;// [n_bands][n_rungs] table index of each band length
    int band_scales;     // a_s [.][M][n_bands], b_s [.][N][n_bands]
    int n_cb;            // column blocks of 32 * CPL columns
    int64_t g_begin;     // first group of this launch
    int n_groups;        // groups in this launch (n_groups * n_rungs <= SR_UMAX)
    double q2d;
    float *out;
    int32_t *counts;
    int32_t *dev_status;
};

struct SmallSmem {
    int32_t lbase[SR_UMAX + 1];   // exclusive prefix of leftover rows over units
    int32_t lfirst[SR_UMAX];      // position in perm of each unit's first leftover row
    uint16_t nst[SR_WARPS][SR_DS];// per warp: n = C[a][L] of the staged contraction indices
    int32_t wsum[SR_WARPS];       // block scan: per-warp totals
};

template <int SR_CPL>
__global__ void __launch_bounds__(SR_THREADS) small_rows_kernel(const __grid_constant__ SmallArgs p) {
    constexpr int SR_COLS = 32 * SR_CPL;
    __shared__ SmallSmem sm;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    uint16_t *nst = sm.nst[warp];
    bool range_bad = false;
    // leftover rows per unit and their exclusive prefix: each thread takes a
    // run of consecutive units, then one block-wide scan of the run totals
    const int U = p.n_groups * p.n_rungs;
    const int per = (U + SR_THREADS - 1) / SR_THREADS;
    const int u_lo = min(t * per, U), u_hi = min(u_lo + per, U);
    int run = 0;
    for (int u = u_lo; u < u_hi; ++u) {
        const int k = u / p.n_groups;  // rung-major: see the item loop
        const int64_t g = p.g_begin + u % p.n_groups;
        const int32_t *o = p.offs + g * (p.n_rungs + 1);
        const int o0 = __ldg(o + k), cnt = max(__ldg(o + k + 1) - o0, 0);
        const int r = cnt % PM;
        const bool small = r > 0 && r < tc_min_rows(f16_of(p.len[k]));
        sm.lbase[u + 1] = small ? r : 0;  // per-unit count for now
        sm.lfirst[u] = o0 + cnt - r;
        run += small ? r : 0;
    }
    // inclusive scan of the run totals over the block
    int v = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) sm.wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < SR_WARPS ? sm.wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < SR_WARPS; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        if (lane < SR_WARPS) sm.wsum[lane] = w;
    }
    __syncthreads();
    // this thread's units: exclusive prefix from the run base
    int base = v - run + (warp > 0 ? sm.wsum[warp - 1] : 0);
    for (int u = u_lo; u < u_hi; ++u) {
        const int c = sm.lbase[u + 1];
        sm.lbase[u + 1] = base + c;
        base += c;
    }
    if (t == 0) sm.lbase[0] = 0;
    __syncthreads();
    const int64_t n_items = (int64_t)sm.lbase[U] * p.n_cb;
    const int nb = p.n_bands > 0 ? p.n_bands : 1;
    const int64_t gw = (int64_t)blockIdx.x * SR_WARPS + warp, nw = (int64_t)gridDim.x * SR_WARPS;
    for (int64_t item = gw; item < n_items; item += nw) {
        const int R = (int)(item / p.n_cb);
        const int cb = (int)(item - (int64_t)R * p.n_cb);
        // unit holding leftover row R: the last u with lbase[u] <= R
        int lo = 0, hi = U;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (sm.lbase[mid] <= R) lo = mid;
            else hi = mid;
        }
        const int u = lo;
        // units run rung-major, so the warps of a block, which take
        // consecutive items, mostly share one length and its count table
        const int k = u / p.n_groups;
        const int64_t g = p.g_begin + u % p.n_groups;
        const int L = p.len[k];
        const int64_t orow = g * p.M + __ldg(p.perm + g * p.M + sm.lfirst[u] + (R - sm.lbase[u]));
        const uint8_t *arow = p.a_lv + orow * p.D;
        // lane owns columns cb * SR_COLS + lane + 32 c, c < SR_CPL
        int64_t jc[SR_CPL];
        bool okc[SR_CPL];
        const uint8_t *bp[SR_CPL];
        float sbc[SR_CPL];
#pragma unroll
        for (int c = 0; c < SR_CPL; ++c) {
            jc[c] = (int64_t)cb * SR_COLS + lane + 32 * c;
            okc[c] = jc[c] < p.N;
            bp[c] = okc[c] ? p.b_lv + (g * p.N + jc[c]) * p.D : nullptr;
            sbc[c] = okc[c] && !p.band_scales ? __ldg(p.b_s + g * p.N + jc[c]) : 0.0f;
        }
        const double fd = p.band_scales ? p.q2d : (double)__ldg(p.a_s + orow) * p.q2d;
        double dec[SR_CPL];
#pragma unroll
        for (int c = 0; c < SR_CPL; ++c) dec[c] = 0.0;
        for (int band = 0; band < nb; ++band) {
            const int Lb = p.n_bands > 0 ? __ldg(p.blen + band * p.n_rungs + k) : L;
            const int64_t d_lo = p.n_bands > 0 ? band * p.chunk_d : 0;
            const int64_t d_hi = p.n_bands > 0 ? d_lo + p.chunk_d : p.D;
            const int lx = p.n_bands > 0 ? __ldg(p.blidx + band * p.n_rungs + k) : p.lidx[k];
            const uint8_t *ctL = p.Ct8 + Lb * 256;
            const uint16_t *EL = p.E + __ldg(p.e_off + lx);
            int acc[SR_CPL];
#pragma unroll
            for (int c = 0; c < SR_CPL; ++c) acc[c] = 0;
            for (int64_t d0 = d_lo; d0 < d_hi; d0 += SR_DS) {
                const int ds = (int)min((int64_t)SR_DS, d_hi - d0);
                // the first 16 B levels of every column of the lane are loaded
                // before the A row is staged (the two latencies overlap); later
                // ones one round ahead
                uint4 lv[SR_CPL];
#pragma unroll
                for (int c = 0; c < SR_CPL; ++c) lv[c] = load_levels16(bp[c], d0, d_hi);
                __syncwarp();
#pragma unroll
                for (int dd = lane; dd < SR_DS; dd += 32) {
                    int n = 0;
                    if (dd < ds) {
                        int a = __ldg(arow + d0 + dd);
                        if (a > p.Q) {
                            a = p.Q;
                            range_bad = true;
                        }
                        n = __ldg(ctL + a);
                    }
                    nst[dd] = (uint16_t)n;
                }
                __syncwarp();
                for (int dd0 = 0; dd0 < ds; dd0 += 16) {
                    uint4 lvn[SR_CPL];
#pragma unroll
                    for (int c = 0; c < SR_CPL; ++c)
                        lvn[c] = dd0 + 16 < ds ? load_levels16(bp[c], d0 + dd0 + 16, d_hi)
                                               : make_uint4(0, 0, 0, 0);
                    if (p.Q < 255) {  // levels above 2^sc_prec are clamped and flagged
#pragma unroll
                        for (int c = 0; c < SR_CPL; ++c)
#pragma unroll
                            for (int uu = 0; uu < 16; ++uu) range_bad |= lv_byte(lv[c], uu) > p.Q;
                    }
#pragma unroll
                    for (int uu = 0; uu < 16; ++uu) {
                        if (dd0 + uu >= ds) break;
                        const uint16_t *er = EL + nst[dd0 + uu] * 256;
#pragma unroll
                        for (int c = 0; c < SR_CPL; ++c) acc[c] += (int)__ldg(er + min(lv_byte(lv[c], uu), p.Q));
                    }
#pragma unroll
                    for (int c = 0; c < SR_CPL; ++c) lv[c] = lvn[c];
                }
            }
            if (p.n_bands == 0) {
                // single band: fp32 decode, same arithmetic as the tensor-core epilogue
                const float DL = (float)(p.D * (int64_t)L);
                const float f = (float)(fd / (double)L);
#pragma unroll
                for (int c = 0; c < SR_CPL; ++c) {
                    if (okc[c]) {
                        const int cnt = acc[c];
                        p.out[orow * p.N + jc[c]] = ((2.0f * (float)cnt - DL) * f) * sbc[c];
                        if (p.counts) p.counts[orow * p.N + jc[c]] = cnt;
                    }
                }
            } else {
                const int64_t DbL = (d_hi - d_lo) * (int64_t)Lb;
                // per-band scales weigh each band's term by q^2 s^A_ib s^B_jb
                const double fab = p.band_scales ? fd * (double)__ldg(p.a_s + orow * nb + band) : 1.0;
#pragma unroll
                for (int c = 0; c < SR_CPL; ++c) {
                    const int cnt = acc[c];
                    const double term = (double)(2LL * cnt - DbL) / (double)Lb;
                    if (p.band_scales)
                        dec[c] += okc[c] ? term * (fab * (double)__ldg(p.b_s + (g * p.N + jc[c]) * nb + band)) : 0.0;
                    else
                        dec[c] += term;
                    if (okc[c] && p.counts)
                        p.counts[((g * nb + band) * p.M + (orow - g * p.M)) * p.N + jc[c]] = cnt;
                }
            }
        }
        if (p.n_bands > 0) {
#pragma unroll
            for (int c = 0; c < SR_CPL; ++c)
                if (okc[c])
                    p.out[orow * p.N + jc[c]] =
                        p.band_scales ? (float)dec[c] : (float)(dec[c] * fd * (double)sbc[c]);
        }
    }
    if (range_bad && p.dev_status) atomicOr(p.dev_status, SC_DEV_LEVEL_RANGE);
    // launched as a programmatic dependent of tc_kernel: finish only after it
    // has, so that later work on the stream sees both kernels complete
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

bool device_is_sm100() {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    return major == 10 && minor == 0;
}

}  // namespace

bool tc_supports(const sc_matmul_desc &d, const sc_table &t) {
    if (t.n_bands > SC_MAX_BANDS) return false;
    if (d.mode != SC_MODE_BIPOLAR) return false;  // the folded tables are the bipolar count's
    if (d.batch > (int64_t)1 << 40) return false;
    return device_is_sm100();
}

// Workspace of the wide-tile band kernel: ksplit slices of fp64 running sums
// (one per output each), then the per-(tile, CTA, epilogue warp) counters of
// finished band segments.  A tile's bands are split into ksplit segments so
// that there are at least about four items per CTA pair (a divisor of the
// band count; 1 when the tiles alone are enough).
namespace {
int64_t tile_bound(const sc_matmul_desc &d, const sc_table &t) {
    const int64_t n_nt = (d.N + TNMAX - 1) / TNMAX;
    return d.batch * ((d.M + PM - 1) / PM + t.n_rungs) * n_nt;
}
int64_t counter_bytes(const sc_matmul_desc &d, const sc_table &t) {
    return ((tile_bound(d, t) * 2 * MAX_EPI_WARPS * (int64_t)sizeof(int32_t)) + 255) & ~255LL;
}
int64_t part_bytes(const sc_matmul_desc &d) {
    return ((d.batch * d.M * d.N * (int64_t)sizeof(double)) + 255) & ~255LL;
}
int preferred_ksplit(const sc_matmul_desc &d, const sc_table &t) {
    const int64_t n_nt = (d.N + TNMAX - 1) / TNMAX;
    const int64_t tiles = d.batch * ((d.M + PM - 1) / PM) * n_nt;
    const int64_t want = 4 * (int64_t)(sm_count() / 2);
    int s = 1;
    for (int c = 1; c <= t.n_bands; ++c) {
        if (t.n_bands % c) continue;
        s = c;
        if (tiles * c >= want) break;
    }
    return s;
}
}  // namespace

int64_t tc_workspace_bytes(const sc_matmul_desc &d, const sc_table &t) {
    if (t.n_bands == 0) return 0;
    return preferred_ksplit(d, t) * part_bytes(d) + counter_bytes(d, t);
}

int64_t tc_workspace_min_bytes(const sc_matmul_desc &d, const sc_table &t) {
    if (t.n_bands == 0) return 0;
    return part_bytes(d) + counter_bytes(d, t);
}

// tc_kernel and small_rows_kernel each run in launches of at most
// UMAX / n_rungs groups.
int tc_launch_count(const sc_matmul_desc &d, const sc_table &t) {
    const int64_t gpl = UMAX / t.n_rungs, sr_gpl = SR_UMAX / t.n_rungs;
    return (int)((d.batch + gpl - 1) / gpl + (d.batch + sr_gpl - 1) / sr_gpl);
}

int launch_tc(const sc_matmul_desc &d, double q_dec, const uint8_t *a_lv, const float *a_s,
              const uint8_t *b_lv, const float *b_s, const int32_t *rung, const int32_t *perm,
              const int32_t *rung_offsets, const sc_table &t, float *out, int32_t *counts,
              int32_t *dev_status, cudaStream_t stream) {
    (void)rung;
    TcArgs p;
    p.M = d.M;
    p.N = d.N;
    p.D = d.D;
    p.batch = d.batch;
    p.a_lv = a_lv;
    p.a_s = a_s;
    p.b_lv = b_lv;
    p.b_s = b_s;
    p.perm = perm;
    p.offs = rung_offsets;
    p.Pc = t.d_Pc;
    p.pc_off = t.d_pc_off;
    p.rho = t.d_rho;
    p.Aw = t.d_Aw;
    p.Uc = t.d_Uc;
    p.uc_off = t.d_uc_off;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) {
        p.len[k] = k < t.n_rungs ? t.ladder[k] : 1;
        p.lidx[k] = k < t.n_rungs ? t.len_idx[k] : 0;
    }
    p.n_rungs = t.n_rungs;
    p.Q = t.Q;
    p.n_bands = t.n_bands;
    p.chunk_d = t.n_bands > 0 ? t.chunk_d : d.D;
    p.blen = t.d_len;
    p.blidx = t.d_len_idx;
    p.band_scales = d.scales == SC_SCALES_BAND;
    // Kernel variant: with bands two accumulators and the fp64 running sum
    // share tensor memory (128-byte stages); without bands 256-byte stages
    // and tiles up to 160 columns, or, when N <= 64, 512-byte stages and
    // 64-column accumulators (the stage depth the tensor memory leaves).
    // With bands and a workspace for the fp64 running sums, the wide-tile
    // layout of the no-band kernel (GSUM).
    // the largest segment count (a divisor of the bands, up to the preferred
    // one) whose partial sums fit the workspace given
    int ksplit = 0;
    if (t.n_bands > 0 && d.workspace) {
        const int pref = preferred_ksplit(d, t);
        for (int c = 1; c <= pref; ++c)
            if (t.n_bands % c == 0 && c * part_bytes(d) + counter_bytes(d, t) <= d.workspace_bytes)
                ksplit = c;
    }
    const bool gsum = ksplit > 0;
    const bool banded = t.n_bands > 0 && !gsum;
    const bool narrow = !banded && !gsum && d.N <= TN_NARROW;
    const int tn = banded ? TNMAX_BANDS : (narrow ? TN_NARROW : TNMAX);
    p.acc_stride = tn;
    p.ring = banded ? RING_BANDS : RING_PLAIN;
    p.ring_col = banded ? SUM_COL + 2 * TNMAX_BANDS : 2 * tn;
    p.bslot = (tn / 2) * (banded ? SK_BANDS : (narrow ? SK_NARROW : SK_PLAIN));
    p.gsum = gsum ? static_cast<double *>(d.workspace) : nullptr;
    p.ksplit = gsum ? ksplit : 1;
    p.part_stride = d.batch * d.M * d.N;
    p.tile_cnt = gsum ? reinterpret_cast<int32_t *>(static_cast<uint8_t *>(d.workspace) +
                                                   ksplit * part_bytes(d))
                      : nullptr;
    if (gsum && ksplit > 1) {
        cudaError_t me = cudaMemsetAsync(p.tile_cnt, 0, (size_t)counter_bytes(d, t), stream);
        if (me != cudaSuccess) return cuda_fail(me, "sc_matmul tc: counter reset");
    }
    // column tiles: as few as possible, each a multiple of 32 columns
    p.n_ntiles = (int)((d.N + tn - 1) / tn);
    {
        const int64_t per = (d.N + p.n_ntiles - 1) / p.n_ntiles;
        p.tile_w = (int)((per + 31) & ~31LL);
    }
    p.q2d = q_dec * q_dec;
    p.out = out;
    p.counts = counts;
    p.dev_status = dev_status;
    const size_t smem = sizeof(Smem) + 1024;
    void (*kern)(TcArgs) =
        gsum     ? (p.band_scales ? tc_kernel<SK_PLAIN, true, true, true> : tc_kernel<SK_PLAIN, true, false, true>)
        : banded ? (p.band_scales ? tc_kernel<SK_BANDS, true, true> : tc_kernel<SK_BANDS, true>)
        : narrow ? tc_kernel<SK_NARROW, false>
                 : tc_kernel<SK_PLAIN, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "sc_matmul tc: smem attribute");
    // groups are processed in launches of at most UMAX / n_rungs groups
    const int64_t gpl = UMAX / t.n_rungs;
    for (int64_t g0 = 0; g0 < d.batch; g0 += gpl) {
        p.g_begin = g0;
        p.n_groups = (int)(d.batch - g0 < gpl ? d.batch - g0 : gpl);
        // upper bound on work items: every rung could own a partial row tile
        const int64_t rows_tiles = (int64_t)p.n_groups * ((d.M + PM - 1) / PM + t.n_rungs);
        int64_t pairs = sm_count() / 2;
        if (pairs > rows_tiles * p.n_ntiles) pairs = rows_tiles * p.n_ntiles;
        if (pairs < 1) pairs = 1;
        kern<<<(unsigned)(2 * pairs), banded ? THREADS : THREADS_PLAIN, smem, stream>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "sc_matmul tc launch");
    }

    SmallArgs q;
    q.M = d.M;
    q.N = d.N;
    q.D = d.D;
    q.batch = d.batch;
    q.a_lv = a_lv;
    q.a_s = a_s;
    q.b_lv = b_lv;
    q.b_s = b_s;
    q.perm = perm;
    q.offs = rung_offsets;
    q.Ct8 = t.d_Ct8;
    q.E = t.d_E;
    q.e_off = t.d_e_off;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) q.lidx[k] = p.lidx[k];
    q.blidx = t.d_len_idx;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) q.len[k] = p.len[k];
    q.n_rungs = t.n_rungs;
    q.Q = t.Q;
    q.n_bands = t.n_bands;
    q.chunk_d = p.chunk_d;
    q.blen = t.d_len;
    q.band_scales = p.band_scales;
    // columns per lane: the fewest lane slots ceil(N / 32c) * c, ties to the wider block
    int cpl = 1;
    for (int c = 2; c <= SR_MAX_CPL; ++c) {
        const int64_t slots = (d.N + 32 * c - 1) / (32 * c) * c;
        if (slots <= (d.N + 32 * cpl - 1) / (32 * cpl) * cpl) cpl = c;
    }
    q.n_cb = (int)((d.N + 32 * cpl - 1) / (32 * cpl));
    void (*sr_kern)(SmallArgs) = cpl == 1 ? small_rows_kernel<1>
                               : cpl == 2 ? small_rows_kernel<2>
                               : cpl == 3 ? small_rows_kernel<3>
                               : cpl == 4 ? small_rows_kernel<4>
                                          : small_rows_kernel<5>;
    q.q2d = q_dec * q_dec;
    q.out = out;
    q.counts = counts;
    q.dev_status = dev_status;
    // leftover rows, in launches of at most SR_UMAX / n_rungs groups; the
    // grid covers an upper bound of (tc_min_rows - 1) leftover rows per unit
    const int64_t sr_gpl = SR_UMAX / t.n_rungs;
    for (int64_t g0 = 0; g0 < d.batch; g0 += sr_gpl) {
        q.g_begin = g0;
        q.n_groups = (int)(d.batch - g0 < sr_gpl ? d.batch - g0 : sr_gpl);
        int64_t max_rows = 0;
        for (int k = 0; k < t.n_rungs; ++k) {
            const int f16 = (((t.ladder[k] + 1) / 2) + 15) & ~15;
            max_rows += tc_min_rows(f16) - 1;
        }
        const int64_t sr_items = (int64_t)q.n_groups * max_rows * q.n_cb;
        int64_t sr_grid = (int64_t)sm_count() * 2;  // one wave at 2 blocks per SM
        if (sr_grid > (sr_items + SR_WARPS - 1) / SR_WARPS) sr_grid = (sr_items + SR_WARPS - 1) / SR_WARPS;
        if (sr_grid < 1) sr_grid = 1;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3((unsigned)sr_grid);
        cfg.blockDim = dim3(SR_THREADS);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, sr_kern, q);
        if (e != cudaSuccess) return cuda_fail(e, "sc_matmul small rows launch");
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "sc_matmul small rows launch");
    }
    return SC_OK;
}

}  // namespace scb
