// sc_tc.cu -- host launcher of the tensor-core count engine (sc_tc_dev.cuh,
// instantiated in sc_tc_k_*.cu) and the CUDA-core kernel for the rows a rung
// leaves over after its tensor-core tiles.
#include <stdint.h>

#include "sc_tc_dev.cuh"

namespace scb {

using namespace tcd;

namespace {

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
    int64_t ld;          // bytes between level rows (both operands): D, or D padded to 16
    const uint8_t *a_lv;
    const float *a_s;
    const uint8_t *b_lv;
    const float *b_s;
    const int32_t *perm;
    const int32_t *offs;
    const uint8_t *Ct8;  // [(Q+1)][256]: Ct8[n][b] = C[b][n]
    const uint16_t *E;   // count tables E_L[n][b] per length
    const int64_t *e_off;
    int unipolar;        // SC_MODE_UNIPOLAR: signed tables E_u[row][b], row of level a from ErowU
    int tile_rows;       // rows of the tensor-core kernel's tiles (its leftovers come here)
    const uint16_t *ErowU;  // [n_lengths][256]
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

template <int SR_CPL, bool UNI>
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
        const int r = cnt % p.tile_rows;
        const bool small = r > 0 && r < tc_min_rows(kbytes_of(p.len[k], UNI));
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
        const uint8_t *arow = p.a_lv + orow * p.ld;
        // lane owns columns cb * SR_COLS + lane + 32 c, c < SR_CPL
        int64_t jc[SR_CPL];
        bool okc[SR_CPL];
        const uint8_t *bp[SR_CPL];
        float sbc[SR_CPL];
#pragma unroll
        for (int c = 0; c < SR_CPL; ++c) {
            jc[c] = (int64_t)cb * SR_COLS + lane + 32 * c;
            okc[c] = jc[c] < p.N;
            bp[c] = okc[c] ? p.b_lv + (g * p.N + jc[c]) * p.ld : nullptr;
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
            // bipolar: row n = C_A[a][L] of E_L; unipolar: row (sign, n) of E_u
            const uint8_t *ctL = p.Ct8 + Lb * 256;
            const uint16_t *erow = UNI ? p.ErowU + lx * 256 : nullptr;
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
                        n = UNI ? (int)__ldg(erow + min(a, 255)) : (int)__ldg(ctL + a);
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
                        for (int c = 0; c < SR_CPL; ++c) {
                            const uint16_t v = __ldg(er + min(lv_byte(lv[c], uu), p.Q));
                            acc[c] += UNI ? (int)(int16_t)v : (int)v;  // unipolar counts are signed
                        }
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
                        p.out[orow * p.N + jc[c]] = UNI ? ((float)cnt * f) * sbc[c]
                                                               : ((2.0f * (float)cnt - DL) * f) * sbc[c];
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
                    const double term = (double)(UNI ? (int64_t)cnt : 2LL * cnt - DbL) / (double)Lb;
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

// The bounded wait of the tensor-core kernel, alone: one thread waits, with
// the given limit, on a barrier that nothing arrives at, then reports
// SC_DEV_WAIT_LIMIT as the kernel does when a wait expires.
__global__ void wait_limit_selftest_kernel(int32_t *dev_status, long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit) && abort_flag && dev_status)
        atomicOr(dev_status, SC_DEV_WAIT_LIMIT);
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
    if (t.n_pool > 0) return false;  // one folded table set per length, not per contraction index
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

// the largest segment count (a divisor of the bands, up to the preferred
// one) whose partial sums fit the workspace given; 0: none fits (or no bands)
int chosen_ksplit(const sc_matmul_desc &d, const sc_table &t) {
    int ksplit = 0;
    if (t.n_bands > 0 && d.workspace) {
        const int pref = preferred_ksplit(d, t);
        for (int c = 1; c <= pref; ++c)
            if (t.n_bands % c == 0 && c * part_bytes(d) + counter_bytes(d, t) <= d.workspace_bytes)
                ksplit = c;
    }
    return ksplit;
}

// Level rows padded to 16 bytes.  When D is not a multiple of 16 every
// 16-level window of a row is unaligned, and its two-word load and shift
// measured a quarter of the attention AV count kernel's time (257-byte rows);
// when the workspace has room after the band sums, the call first copies
// both operands' levels into rows of round16(D) bytes (zero tail) and the
// kernels read those with one aligned load per window.
int64_t padded_ld(const sc_matmul_desc &d) { return (d.D + 15) & ~15LL; }
int64_t round256(int64_t x) { return (x + 255) & ~255LL; }
int64_t pad_region_bytes(const sc_matmul_desc &d) {
    const int64_t ld = padded_ld(d);
    return round256(d.batch * d.M * ld) + round256(d.batch * d.N * ld);
}
int64_t sums_region_bytes(const sc_matmul_desc &d, const sc_table &t, int ksplit) {
    return ksplit > 0 ? round256(ksplit * part_bytes(d) + counter_bytes(d, t)) : 0;
}
// byte offset of the padded levels in the workspace, or -1: no padding
int64_t pad_offset(const sc_matmul_desc &d, const sc_table &t) {
    if (d.D % 16 == 0 || !d.workspace || d.b_prep) return -1;
    const int64_t off = sums_region_bytes(d, t, chosen_ksplit(d, t));
    return off + pad_region_bytes(d) <= d.workspace_bytes ? off : -1;
}

// Copies rows of D level bytes into rows of ld = round16(D) bytes with a
// zero tail, one aligned 16-byte store per thread and chunk; the source is
// read with aligned 16-byte words where they lie inside [src, end), else byte
// by byte.
__global__ void pad_levels_kernel(const uint8_t *__restrict__ src, int64_t rows, int64_t D, int64_t ld,
                                  uint8_t *__restrict__ dst) {
    const int64_t cpr = ld / 16;
    const int64_t n = rows * cpr;
    const uint8_t *end = src + rows * D;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / cpr, c = i - r * cpr;
        const int64_t d0 = 16 * c;
        const int nv = (int)(D - d0 < 16 ? D - d0 : 16);  // >= 1: d0 < D
        const uint8_t *sp = src + r * D + d0;
        const uintptr_t addr = reinterpret_cast<uintptr_t>(sp);
        const uint32_t k = (uint32_t)(addr & 15u);
        const uint8_t *base = sp - k;
        uint32_t w[4];
        if (base >= src && base + 32 <= end) {
            const uint4 lo = __ldg(reinterpret_cast<const uint4 *>(base));
            const uint4 hi = __ldg(reinterpret_cast<const uint4 *>(base) + 1);
            const uint32_t x8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            const uint32_t q = k >> 2, sh = 8u * (k & 3u);
            uint32_t x[5];
#pragma unroll
            for (int j = 0; j < 5; ++j)  // x[j] = x8[q + j], q in 0..3
                x[j] = q == 0 ? x8[j] : (q == 1 ? x8[j + 1] : (q == 2 ? x8[j + 2] : x8[j + 3]));
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = __funnelshift_r(x[j], x[j + 1], sh);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = 0u;
            for (int u = 0; u < nv; ++u) w[u >> 2] |= (uint32_t)__ldg(sp + u) << (8 * (u & 3));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // zero the bytes at or past D
            const int b = nv - 4 * j;
            if (b <= 0) w[j] = 0u;
            else if (b < 4) w[j] &= (1u << (8 * b)) - 1u;
        }
        *reinterpret_cast<uint4 *>(dst + r * ld + d0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

int launch_pad_levels(const uint8_t *src, int64_t rows, int64_t D, int64_t ld, uint8_t *dst,
                      cudaStream_t stream) {
    const int64_t n = rows * (ld / 16);
    int64_t grid = (n + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    pad_levels_kernel<<<(unsigned)grid, 256, 0, stream>>>(src, rows, D, ld, dst);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_matmul tc: level padding launch");
}
}  // namespace

namespace {
bool runs_wide_kernel(const sc_matmul_desc &d, const sc_table &t) {
    if (d.engine == SC_ENGINE_GATHER || !tc_supports(d, t)) return false;
    if (d.N <= TN_SINGLE) return false;  // the one-CTA kernel
    if (t.n_bands > 0)                   // bands: the wide tiles need a workspace slice
        return d.workspace && d.workspace_bytes >= part_bytes(d) + counter_bytes(d, t);
    return true;
}
}  // namespace

int64_t tc_workspace_bytes(const sc_matmul_desc &d, const sc_table &t) {
    const int64_t sums = t.n_bands > 0 ? round256(preferred_ksplit(d, t) * part_bytes(d) + counter_bytes(d, t)) : 0;
    const int64_t pad = (d.D % 16 != 0 && !d.b_prep) ? pad_region_bytes(d) : 0;
    return sums + pad;
}

int64_t tc_workspace_min_bytes(const sc_matmul_desc &d, const sc_table &t) {
    if (t.n_bands == 0) return 0;
    return part_bytes(d) + counter_bytes(d, t);
}

// tc_kernel and small_rows_kernel each run in launches of at most
// UMAX / n_rungs groups.
int tc_launch_count(const sc_matmul_desc &d, const sc_table &t) {
    const int64_t gpl = UMAX / t.n_rungs, sr_gpl = SR_UMAX / t.n_rungs;
    const int pads = pad_offset(d, t) >= 0 ? 2 : 0;  // the two level-padding copies
    return (int)((d.batch + gpl - 1) / gpl + (d.batch + sr_gpl - 1) / sr_gpl) + pads;
}

// ---------------------------------------------------------------------------
// Prepared second operand (sc_prepare_b): the B stages of the wide-tile pair
// kernels (160-column tiles, 256-byte stages, one CTA's 80 columns per
// stage) written once, in the shared-memory layout the B producers would
// build, for every (band, rung) slot of the table.
// ---------------------------------------------------------------------------
namespace {

struct WideTiling {
    int n_ntiles, tile_w;
};

WideTiling wide_tiling(int64_t N) {
    WideTiling w;
    w.n_ntiles = (int)((N + TNMAX - 1) / TNMAX);
    const int64_t per = (N + w.n_ntiles - 1) / w.n_ntiles;
    w.tile_w = (int)((per + 31) & ~31LL);
    return w;
}

// stages of one slot: contraction width x bytes per index, in 256-byte stages
int slot_stages(const sc_table &t, int64_t D, int slot, bool uni) {
    const int nb = t.n_bands > 0 ? t.n_bands : 1;
    (void)nb;
    const int k = slot % t.n_rungs;
    const int L = t.n_bands > 0 ? t.band_len[slot] : t.ladder[k];
    const int64_t width = t.n_bands > 0 ? t.chunk_d : D;
    return (int)((width * kbytes_of(L, uni) + SK_PLAIN - 1) / SK_PLAIN);
}

struct PrepArgs {
    const uint8_t *b_lv;
    int64_t N, D, batch;
    int Q, n_ntiles, tile_w, n_stages, kpi;  // kpi: contraction bytes per index
    int64_t d_lo, d_hi;                      // this slot's contraction indices
    const uint8_t *Pk;                       // this length's chunk tables
    const uint8_t *Pmap;                     // this length's class maps [Q+1][PMAP_STRIDE]
    uint8_t *dst;                            // this slot's stages
};

// One thread per 16-byte chunk of one slot's stages: chunk (column bc of the
// CTA's half, chunk q of the stage) of block (g, column tile, CTA h, stage s).
__global__ void __launch_bounds__(256) prep_b_kernel(const PrepArgs a) {
    constexpr int QPS = SK_PLAIN / 16;  // chunks per column per stage
    const int64_t per_block = (int64_t)BC * QPS;
    const int64_t total = a.batch * a.n_ntiles * 2 * (int64_t)a.n_stages * per_block;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = e / per_block;
        const int rem = (int)(e - blk * per_block);
        const int bc = rem / QPS, q = rem % QPS;
        const int s = (int)(blk % a.n_stages);
        const int64_t t2 = blk / a.n_stages;
        const int h = (int)(t2 % 2);
        const int nt = (int)((t2 / 2) % a.n_ntiles);
        const int64_t g = t2 / 2 / a.n_ntiles;
        const int64_t n0 = (int64_t)nt * a.tile_w;
        const int nvalid = (int)min((int64_t)a.tile_w, a.N - n0);
        const int chalf = ((nvalid + 31) & ~31) / 2;
        const int64_t kb = (int64_t)s * SK_PLAIN + 16 * q;  // contraction byte in the slot
        const int64_t d = a.d_lo + kb / a.kpi;
        const int jc = (int)((kb % a.kpi) / 16);
        const int64_t col = n0 + (int64_t)h * chalf + bc;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (bc < chalf && bc + h * chalf < nvalid && d < a.d_hi) {
            int lv = a.b_lv[(g * a.N + col) * a.D + d];
            lv = min(lv, a.Q);
            const int cls = a.Pmap[lv * PMAP_STRIDE + jc];
            v = *reinterpret_cast<const uint4 *>(a.Pk + (jc * PK_ROWS + cls) * 16);
        }
        *reinterpret_cast<uint4 *>(a.dst + blk * BPREP_BLOCK + op_offset<SK_PLAIN>(bc, q)) = v;
    }
}

// The kernel variant sc_matmul would run: whether it is a wide-tile pair
// kernel that can take prepared B stages.
bool runs_wide_kernel(const sc_matmul_desc &d, const sc_table &t);

}  // namespace

int64_t tc_prepare_b_bytes(const sc_matmul_desc &d, const sc_table &t) {
    if (!runs_wide_kernel(d, t)) return -SC_ERR_UNSUPPORTED;
    const WideTiling w = wide_tiling(d.N);
    const bool uni = d.mode == SC_MODE_UNIPOLAR;
    const int n_slots = (t.n_bands > 0 ? t.n_bands : 1) * t.n_rungs;
    int64_t bytes = 0;
    for (int u = 0; u < n_slots; ++u)
        bytes += d.batch * w.n_ntiles * 2 * (int64_t)slot_stages(t, d.D, u, uni) * BPREP_BLOCK;
    return bytes;
}

int tc_prepare_b(const sc_matmul_desc &d, const uint8_t *b_lv, const sc_table &t, sc_bprep **out,
                 cudaStream_t stream) {
    const int64_t bytes = tc_prepare_b_bytes(d, t);
    if (bytes < 0) {
        set_error("sc_prepare_b: the problem does not run the wide-tile tensor-core kernel (gather "
                  "engine, N <= 64, a pool, or bands without a workspace of one slice)");
        return SC_ERR_UNSUPPORTED;
    }
    const WideTiling w = wide_tiling(d.N);
    const bool uni = d.mode == SC_MODE_UNIPOLAR;
    const int n_slots = (t.n_bands > 0 ? t.n_bands : 1) * t.n_rungs;
    sc_bprep *bp = new sc_bprep();
    bp->N = d.N;
    bp->D = d.D;
    bp->batch = d.batch;
    bp->mode = d.mode;
    bp->table = &t;
    bp->n_ntiles = w.n_ntiles;
    bp->tile_w = w.tile_w;
    bp->bytes = bytes;
    bp->slot_off.resize(n_slots);
    int64_t off = 0;
    for (int u = 0; u < n_slots; ++u) {
        bp->slot_off[u] = off;
        off += d.batch * w.n_ntiles * 2 * (int64_t)slot_stages(t, d.D, u, uni) * BPREP_BLOCK;
    }
    cudaGetDevice(&bp->device);
    cudaError_t e = cudaMalloc((void **)&bp->d_buf, (size_t)bytes);
    if (e == cudaSuccess) e = cudaMalloc((void **)&bp->d_slot_off, n_slots * sizeof(int64_t));
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(bp->d_slot_off, bp->slot_off.data(), n_slots * sizeof(int64_t),
                            cudaMemcpyHostToDevice, stream);
    for (int u = 0; e == cudaSuccess && u < n_slots; ++u) {
        const int k = u % t.n_rungs, band = u / t.n_rungs;
        const int lidx = t.len_idx[u];
        PrepArgs a;
        a.b_lv = b_lv;
        a.N = d.N;
        a.D = d.D;
        a.batch = d.batch;
        a.Q = t.Q;
        a.n_ntiles = w.n_ntiles;
        a.tile_w = w.tile_w;
        a.n_stages = slot_stages(t, d.D, u, uni);
        a.kpi = kbytes_of(t.n_bands > 0 ? t.band_len[u] : t.ladder[k], uni);
        a.d_lo = t.n_bands > 0 ? (int64_t)band * t.chunk_d : 0;
        a.d_hi = t.n_bands > 0 ? a.d_lo + t.chunk_d : d.D;
        a.Pk = (uni ? t.d_PkU : t.d_Pk) + (uni ? t.pku_off[lidx] : t.pk_off[lidx]);
        a.Pmap = (uni ? t.d_PmapU : t.d_Pmap) + (int64_t)lidx * (t.Q + 1) * PMAP_STRIDE;
        a.dst = bp->d_buf + bp->slot_off[u];
        prep_b_kernel<<<sm_count() * 8, 256, 0, stream>>>(a);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        tc_bprep_destroy(bp);
        return cuda_fail(e, "sc_prepare_b");
    }
    *out = bp;
    return SC_OK;
}

int tc_bprep_destroy(sc_bprep *bp) {
    if (!bp) return SC_OK;
    int cur = 0;
    cudaGetDevice(&cur);
    if (bp->device >= 0 && bp->device != cur) cudaSetDevice(bp->device);
    cudaDeviceSynchronize();  // no kernel may still read the stages
    cudaFree(bp->d_buf);
    cudaFree(bp->d_slot_off);
    if (bp->device >= 0 && bp->device != cur) cudaSetDevice(cur);
    delete bp;
    return SC_OK;
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
    const bool uni = d.mode == SC_MODE_UNIPOLAR;
    p.Pk = uni ? t.d_PkU : t.d_Pk;
    p.pk_off = uni ? t.d_pku_off : t.d_pk_off;
    p.Pmap = uni ? t.d_PmapU : t.d_Pmap;
    p.Aw = uni ? t.d_AwU : t.d_Aw;
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
    const int ksplit = chosen_ksplit(d, t);
    const bool gsum = ksplit > 0;
    // levels padded to 16-byte rows in the workspace, after the band sums
    p.lda = p.ldb = d.D;
    const int64_t poff = pad_offset(d, t);
    if (poff >= 0 && d.batch * (d.M + d.N) > 0) {
        const int64_t ld = padded_ld(d);
        uint8_t *pa = static_cast<uint8_t *>(d.workspace) + poff;
        uint8_t *pb = pa + round256(d.batch * d.M * ld);
        int rc = d.batch * d.M > 0 ? launch_pad_levels(a_lv, d.batch * d.M, d.D, ld, pa, stream) : SC_OK;
        if (rc != SC_OK) return rc;
        rc = d.batch * d.N > 0 ? launch_pad_levels(b_lv, d.batch * d.N, d.D, ld, pb, stream) : SC_OK;
        if (rc != SC_OK) return rc;
        a_lv = pa;
        b_lv = pb;
        p.a_lv = a_lv;
        p.b_lv = b_lv;
        p.lda = p.ldb = ld;
    }
    const bool banded = t.n_bands > 0 && !gsum;
    // N <= 64 (attention AV): one CTA per MMA (M = 128 rows, 64-column
    // tiles) so that the few rows a rung holds per group waste half as many
    // MMA rows as in a 256-row pair tile
    const bool single = !banded && !gsum && d.N <= TN_SINGLE;
    const int cg = single ? 1 : 2;
    const int tn = banded ? TNMAX_BANDS : (single ? TN_SINGLE : TNMAX);
    p.acc_stride = tn;
    p.ring = banded ? RING_BANDS : RING_PLAIN;
    p.ring_col = banded ? SUM_COL + 2 * TNMAX_BANDS : 2 * tn;
    p.bslot = (tn / cg) * (banded ? SK_BANDS : SK_PLAIN);
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
    p.bprep = nullptr;
    p.bprep_off = nullptr;
    // deal items by cost with bands, whose segments differ in stage count
    // (tilted band lengths: round robin left fc2's CTAs busy 71 % of the
    // kernel, 93 % dealt by cost), and with a prepared second operand, whose
    // items restage no tables when the lengths mix (fraction-based fc1 on
    // four lengths: count call 1.09 -> 1.01 ms); otherwise items of a rung
    // cost the same and the rung-major order keeps each pair on one length
    p.balance = (t.n_bands > 0 || d.b_prep) ? 1 : 0;
    if (d.b_prep) {
        const sc_bprep &bp = *d.b_prep;
        if (single || banded || bp.table != &t || bp.N != d.N || bp.D != d.D ||
            bp.batch != d.batch || bp.mode != d.mode || bp.n_ntiles != p.n_ntiles ||
            bp.tile_w != p.tile_w) {
            set_error("sc_matmul: b_prep was prepared for another problem, table or kernel");
            return SC_ERR_ARG;
        }
        p.bprep = bp.d_buf;
        p.bprep_off = bp.d_slot_off;
    }
    const size_t smem = sizeof(Smem) + 1024;
    const bool bs = p.band_scales != 0;
    TcKernelFn kern;
    if (gsum)
        kern = bs ? (uni ? tc_kernel_bands_ws_bs_uni() : tc_kernel_bands_ws_bs())
                  : (uni ? tc_kernel_bands_ws_uni() : tc_kernel_bands_ws());
    else if (banded)
        kern = bs ? (uni ? tc_kernel_bands_bs_uni() : tc_kernel_bands_bs())
                  : (uni ? tc_kernel_bands_uni() : tc_kernel_bands());
    else if (single)
        kern = uni ? tc_kernel_single_uni() : tc_kernel_single();
    else
        kern = uni ? tc_kernel_plain_uni() : tc_kernel_plain();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "sc_matmul tc: smem attribute");
    // groups are processed in launches of at most UMAX / n_rungs groups
    const int64_t gpl = UMAX / t.n_rungs;
    for (int64_t g0 = 0; g0 < d.batch; g0 += gpl) {
        p.g_begin = g0;
        p.n_groups = (int)(d.batch - g0 < gpl ? d.batch - g0 : gpl);
        // upper bound on work items: every rung could own a partial row tile
        const int64_t tr = (int64_t)cg * TM;
        const int64_t rows_tiles = (int64_t)p.n_groups * ((d.M + tr - 1) / tr + t.n_rungs);
        int64_t units = sm_count() / cg;  // CTA pairs, or CTAs
        if (units > rows_tiles * p.n_ntiles) units = rows_tiles * p.n_ntiles;
        if (units < 1) units = 1;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(cg * units));
        cfg.blockDim = dim3(banded ? THREADS : THREADS_PLAIN);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = cg == 2 ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, kern, p);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "sc_matmul tc launch");
    }

    SmallArgs q;
    q.M = d.M;
    q.N = d.N;
    q.D = d.D;
    q.ld = p.lda;  // == p.ldb
    q.batch = d.batch;
    q.a_lv = a_lv;
    q.a_s = a_s;
    q.b_lv = b_lv;
    q.b_s = b_s;
    q.perm = perm;
    q.offs = rung_offsets;
    q.Ct8 = t.d_Ct8;
    q.E = uni ? t.d_EU : t.d_E;
    q.e_off = uni ? t.d_eu_off : t.d_e_off;
    q.unipolar = uni ? 1 : 0;
    q.tile_rows = cg * TM;
    q.ErowU = t.d_ErowU;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) q.lidx[k] = p.lidx[k];
    q.blidx = t.d_len_idx;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) q.len[k] = p.len[k];
    q.n_rungs = t.n_rungs;
    q.Q = t.Q;
    q.n_bands = t.n_bands;
    q.chunk_d = p.chunk_d;
    q.blen = t.d_len;
    q.band_scales = p.band_scales;
    // columns per lane: the fewest lane slots ceil(N / 32c) * c; ties go to
    // the wider block (each item stages its row's counts once), except for
    // long contractions, where narrower blocks give more items to run at once
    int cpl = 1;
    for (int c = 2; c <= SR_MAX_CPL; ++c) {
        const int64_t slots = (d.N + 32 * c - 1) / (32 * c) * c;
        const int64_t best = (d.N + 32 * cpl - 1) / (32 * cpl) * cpl;
        if (slots < best || (slots == best && d.D <= 128)) cpl = c;
    }
    q.n_cb = (int)((d.N + 32 * cpl - 1) / (32 * cpl));
    void (*sr_kern)(SmallArgs) =
        uni ? (cpl == 1 ? small_rows_kernel<1, true>
               : cpl == 2 ? small_rows_kernel<2, true>
               : cpl == 3 ? small_rows_kernel<3, true>
               : cpl == 4 ? small_rows_kernel<4, true>
                          : small_rows_kernel<5, true>)
            : (cpl == 1 ? small_rows_kernel<1, false>
               : cpl == 2 ? small_rows_kernel<2, false>
               : cpl == 3 ? small_rows_kernel<3, false>
               : cpl == 4 ? small_rows_kernel<4, false>
                          : small_rows_kernel<5, false>);
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
            max_rows += tc_min_rows(kbytes_of(t.ladder[k], uni)) - 1;
        }
        const int64_t sr_items = (int64_t)q.n_groups * max_rows * q.n_cb;
        int64_t sr_grid = (int64_t)sm_count() * 3;  // one wave at 3 blocks per SM (the register limit)
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

namespace scb {
int launch_wait_limit_selftest(int32_t *dev_status, int64_t limit_cycles, cudaStream_t stream) {
    wait_limit_selftest_kernel<<<1, 32, 0, stream>>>(dev_status, (long long)limit_cycles);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_selftest_wait_limit launch");
}
}  // namespace scb
