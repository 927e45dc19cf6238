// sc_kernels.cu -- quantise + row statistic, rung assignment with the
// rung-sorted row order, and the CUDA-core (table-gather) count engine.
#include <math.h>

#include "sc_internal.cuh"

namespace scb {

// ---------------------------------------------------------------------------
// Quantisation ("scmp_vit" README, "Why it works": scale = abs_max / 127;
// "Precision As You Need" flowchart: PTQ symmetric integer scaling).
// x_int = clamp(rint(x / s), -qmax, qmax) with IEEE fp32 division and round
// half to even; level = x_int + 2^(p-1).
// ---------------------------------------------------------------------------
// rint(v / s) is taken from the product v * rs, rs = 1/s rounded to nearest:
// for |v / s| <= 128 the product differs from the IEEE quotient by less than
// 2.3e-5 (two roundings of 2^-24 relative each, plus half an ulp of the
// quotient), so both round to the same integer unless the product lies
// within 1e-4 of a half-integer; only then is the quotient computed.
__device__ __forceinline__ uint8_t quant_level(float v, float s, float rs, int half, int qmax) {
    int xi = 0;
    if (s > 0.0f && isfinite(v)) {
        float q = v * rs;
        // (a non-finite product, from a subnormal s, also takes the quotient)
        if (!(fabsf(q - floorf(q) - 0.5f) >= 1.0e-4f)) q = __fdiv_rn(v, s);
        xi = __float2int_rn(q);
        xi = min(max(xi, -qmax), qmax);
    }
    return (uint8_t)(xi + half);
}

// quant_level for a row known to be finite with s > 0 (no per-element checks).
__device__ __forceinline__ uint32_t quant_level_finite(float v, float s, float rs, int half, int qmax) {
    float q = v * rs;
    if (!(fabsf(q - floorf(q) - 0.5f) >= 1.0e-4f)) q = __fdiv_rn(v, s);
    int xi = __float2int_rn(q);
    xi = min(max(xi, -qmax), qmax);
    return (uint32_t)(xi + half);
}

// One warp per row: pass 1 finds max|x| (and max x for the AV statistic),
// pass 2 re-reads the row (L1/L2 resident) and writes the levels.
__global__ void __launch_bounds__(256) quant_rows_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
    int64_t bstride, int half, int qmax, int stat_mode, uint8_t *__restrict__ levels,
    float *__restrict__ scales, float *__restrict__ stat, int32_t *dev_status) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows * batch;
         w += warps_total) {
        const int64_t bi = w / rows, r = w - bi * rows;
        const float *xr = x + bi * bstride + r * ld;
        float amax = 0.0f, vmax = -INFINITY;
        bool bad = false;
        for (int64_t c = lane; c < cols; c += 32) {
            const float v = __ldg(xr + c);
            bad |= !isfinite(v);
            amax = fmaxf(amax, fabsf(v));
            vmax = fmaxf(vmax, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        }
        bad = __any_sync(0xffffffffu, bad);
        const float s = __fdiv_rn(amax, (float)qmax), rs = __frcp_rn(s);
        uint8_t *lr = levels + w * cols;
        for (int64_t c = lane; c < cols; c += 32) lr[c] = quant_level(__ldg(xr + c), s, rs, half, qmax);
        if (lane == 0) {
            scales[w] = s;
            if (stat) stat[w] = stat_mode == SC_STAT_AMAX ? amax : vmax;
            if (bad && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
        }
    }
}

// Rows of any width and alignment that fit in registers (cols <= 32 NV): one
// warp per row, lane l holding x[l + 32 k]; every load of the row is issued
// before the reduction, and the levels are written from the registers.
template <int NV>
__global__ void __launch_bounds__(256) quant_rows_reg_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
    int64_t bstride, int half, int qmax, int stat_mode, uint8_t *__restrict__ levels,
    float *__restrict__ scales, float *__restrict__ stat, int32_t *dev_status) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    bool bad_any = false;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows * batch;
         w += warps_total) {
        const int64_t bi = w / rows, r = w - bi * rows;
        const float *xr = x + bi * bstride + r * ld;
        float v[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int64_t c = lane + 32 * k;
            v[k] = c < cols ? __ldg(xr + c) : 0.0f;
        }
        float amax = 0.0f, vmax = -INFINITY;
        bool bad = false;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            if (lane + 32 * k < cols) {
                bad |= !isfinite(v[k]);
                amax = fmaxf(amax, fabsf(v[k]));
                vmax = fmaxf(vmax, v[k]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        }
        bad = __any_sync(0xffffffffu, bad);
        const float s = __fdiv_rn(amax, (float)qmax), rs = __frcp_rn(s);
        uint8_t *lr = levels + w * cols;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int64_t c = lane + 32 * k;
            if (c < cols) lr[c] = quant_level(v[k], s, rs, half, qmax);
        }
        if (lane == 0) {
            scales[w] = s;
            if (stat) stat[w] = stat_mode == SC_STAT_AMAX ? amax : vmax;
        }
        bad_any |= bad;
    }
    if (bad_any && lane == 0 && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
}

// Vectorised variant for rows that fit in registers: G lanes per row, each
// holding NV float4 (cols <= 4 * G * NV, cols % 4 == 0, 16-byte aligned rows).
// One global read per element, four levels stored as one 32-bit word.
template <int G, int NV>
__global__ void __launch_bounds__(256) quant_rows_vec_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
    int64_t bstride, int half, int qmax, int stat_mode, uint8_t *__restrict__ levels,
    float *__restrict__ scales, float *__restrict__ stat, int32_t *dev_status) {
    constexpr int RPW = 32 / G;  // rows per warp
    const int lane = threadIdx.x & 31;
    const int sub = lane / G, gl = lane % G;
    const int64_t total = rows * batch;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t c4 = cols >> 2;
    const bool dense = bstride == rows * ld;
    bool bad_any = false;
    for (int64_t w0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW;
         w0 < total; w0 += warps_total * RPW) {
        const int64_t w = w0 + sub;
        const bool live = w < total;
        // row w of the flattened batch: batches packed back to back need no
        // division (the common case); otherwise split w into (batch, row)
        int64_t xoff;
        if (dense) {
            xoff = live ? w * ld : 0;
        } else {
            const int64_t bi = live ? w / rows : 0, r = live ? w - bi * rows : 0;
            xoff = bi * bstride + r * ld;
        }
        const float4 *xr = reinterpret_cast<const float4 *>(x + xoff);
        float4 v[NV];
        // max |x| as the integer max of the sign-cleared bit patterns: equal
        // to the float max for finite values, and any inf or NaN sorts above
        // every finite value, which flags the row
        uint32_t abits = 0u;
        float vmax = -INFINITY;
        const bool rowmax = stat_mode != SC_STAT_AMAX;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int64_t c = gl + (int64_t)k * G;
            if (live && c < c4) {
                v[k] = __ldg(xr + c);
                abits = max(abits, max(max(__float_as_uint(v[k].x) & 0x7fffffffu,
                                           __float_as_uint(v[k].y) & 0x7fffffffu),
                                       max(__float_as_uint(v[k].z) & 0x7fffffffu,
                                           __float_as_uint(v[k].w) & 0x7fffffffu)));
                if (rowmax) vmax = fmaxf(vmax, fmaxf(fmaxf(v[k].x, v[k].y), fmaxf(v[k].z, v[k].w)));
            }
        }
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) {
            abits = max(abits, __shfl_xor_sync(0xffffffffu, abits, o, G));
            if (rowmax) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o, G));
        }
        const bool bad = abits >= 0x7f800000u;
        const float amax = __uint_as_float(abits);
        const float s = __fdiv_rn(amax, (float)qmax), rs = __frcp_rn(s);
        const bool fast = !bad && s > 0.0f;
        if (live) {
            uint32_t *lr = reinterpret_cast<uint32_t *>(levels + w * cols);
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                const int64_t c = gl + (int64_t)k * G;
                if (c >= c4) continue;
                if (fast)
                    lr[c] = quant_level_finite(v[k].x, s, rs, half, qmax) |
                            (quant_level_finite(v[k].y, s, rs, half, qmax) << 8) |
                            (quant_level_finite(v[k].z, s, rs, half, qmax) << 16) |
                            (quant_level_finite(v[k].w, s, rs, half, qmax) << 24);
                else
                    lr[c] = (uint32_t)quant_level(v[k].x, s, rs, half, qmax) |
                            ((uint32_t)quant_level(v[k].y, s, rs, half, qmax) << 8) |
                            ((uint32_t)quant_level(v[k].z, s, rs, half, qmax) << 16) |
                            ((uint32_t)quant_level(v[k].w, s, rs, half, qmax) << 24);
            }
            if (gl == 0) {
                scales[w] = s;
                if (stat) stat[w] = stat_mode == SC_STAT_AMAX ? amax : vmax;
            }
        }
        bad_any |= bad;
    }
    if (__any_sync(0xffffffffu, bad_any) && lane == 0 && dev_status)
        atomicOr(dev_status, SC_DEV_NONFINITE);
}

// Long rows (512 < cols <= 1024 NV, cols % 4 == 0, 16-byte aligned rows):
// one block of 256 threads per row, thread t holding float4 t + 256 k of it
// in registers; the row's max |x| (and max x) is reduced through shared
// memory, then the levels are written from the registers, four per 32-bit
// store.  One global read per element (the one-warp kernel above reads a
// row twice with scalar loads).
template <int NV>
__global__ void __launch_bounds__(256) quant_rows_block_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
    int64_t bstride, int half, int qmax, int stat_mode, uint8_t *__restrict__ levels,
    float *__restrict__ scales, float *__restrict__ stat, int32_t *dev_status) {
    __shared__ uint32_t red_a[8];
    __shared__ float red_v[8];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t total = rows * batch;
    const int64_t c4 = cols >> 2;
    const bool rowmax = stat_mode != SC_STAT_AMAX;
    bool bad_any = false;
    for (int64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const int64_t bi = w / rows, r = w - bi * rows;
        const float4 *xr = reinterpret_cast<const float4 *>(x + bi * bstride + r * ld);
        float4 v[NV];
        // max |x| as the integer max of the sign-cleared bit patterns (see
        // quant_rows_vec_kernel): any inf or NaN flags the row
        uint32_t abits = 0u;
        float vmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int64_t c = tid + (int64_t)k * 256;
            if (c < c4) {
                v[k] = __ldg(xr + c);
                abits = max(abits, max(max(__float_as_uint(v[k].x) & 0x7fffffffu,
                                           __float_as_uint(v[k].y) & 0x7fffffffu),
                                       max(__float_as_uint(v[k].z) & 0x7fffffffu,
                                           __float_as_uint(v[k].w) & 0x7fffffffu)));
                if (rowmax) vmax = fmaxf(vmax, fmaxf(fmaxf(v[k].x, v[k].y), fmaxf(v[k].z, v[k].w)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            abits = max(abits, __shfl_xor_sync(0xffffffffu, abits, o));
            if (rowmax) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        }
        if (lane == 0) {
            red_a[wid] = abits;
            red_v[wid] = vmax;
        }
        __syncthreads();
        abits = red_a[0];
        vmax = red_v[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            abits = max(abits, red_a[i]);
            vmax = fmaxf(vmax, red_v[i]);
        }
        __syncthreads();  // red_* are reused by the next row
        const bool bad = abits >= 0x7f800000u;
        const float amax = __uint_as_float(abits);
        const float s = __fdiv_rn(amax, (float)qmax), rs = __frcp_rn(s);
        const bool fast = !bad && s > 0.0f;
        uint32_t *lr = reinterpret_cast<uint32_t *>(levels + w * cols);
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int64_t c = tid + (int64_t)k * 256;
            if (c >= c4) continue;
            if (fast)
                lr[c] = quant_level_finite(v[k].x, s, rs, half, qmax) |
                        (quant_level_finite(v[k].y, s, rs, half, qmax) << 8) |
                        (quant_level_finite(v[k].z, s, rs, half, qmax) << 16) |
                        (quant_level_finite(v[k].w, s, rs, half, qmax) << 24);
            else
                lr[c] = (uint32_t)quant_level(v[k].x, s, rs, half, qmax) |
                        ((uint32_t)quant_level(v[k].y, s, rs, half, qmax) << 8) |
                        ((uint32_t)quant_level(v[k].z, s, rs, half, qmax) << 16) |
                        ((uint32_t)quant_level(v[k].w, s, rs, half, qmax) << 24);
        }
        if (tid == 0) {
            scales[w] = s;
            if (stat) stat[w] = stat_mode == SC_STAT_AMAX ? amax : vmax;
        }
        bad_any |= bad;
    }
    if (bad_any && tid == 0 && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
}

// Per-column quantisation of short columns (rows <= 8 RPT): block (32, 8)
// owns 32 columns of one batch entry, thread (tx, ty) holding rows ty + 8 k
// of column tx in registers; the column maxima are reduced through shared
// memory, the levels go through a shared-memory tile (one padded row per
// column) and are written out column by column, consecutive threads on
// consecutive bytes.  One global read per element.
template <int RPT>
__global__ void __launch_bounds__(256) quant_cols_reg_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t bstride, int half,
    int qmax, uint8_t *__restrict__ levels, float *__restrict__ scales, int32_t *dev_status) {
    constexpr int TR = 8 * RPT + 4;  // tile row pitch (bytes): the rows, padded against bank conflicts
    __shared__ float red[8][33];
    __shared__ __align__(16) uint8_t tile[32][TR];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int64_t bi = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * 32;
    const int64_t c = c0 + tx;
    const float *xb = x + bi * bstride;
    const bool col_ok = c < cols;
    float v[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int64_t r = ty + 8 * k;
        v[k] = (col_ok && r < rows) ? __ldg(xb + r * ld + c) : 0.0f;
    }
    float amax = 0.0f;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        bad |= !isfinite(v[k]);
        amax = fmaxf(amax, fabsf(v[k]));
    }
    red[ty][tx] = amax;
    bad = __syncthreads_or(bad);
    if (ty == 0) {
        float m = red[0][tx];
        for (int k = 1; k < 8; ++k) m = fmaxf(m, red[k][tx]);
        red[0][tx] = __fdiv_rn(m, (float)qmax);
        if (col_ok) scales[bi * cols + c] = red[0][tx];
    }
    if (bad && tx == 0 && ty == 0 && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
    __syncthreads();
    const float sc = red[0][tx], rs = __frcp_rn(sc);
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int r = ty + 8 * k;
        if (r < rows) tile[tx][r] = quant_level(v[k], sc, rs, half, qmax);
    }
    __syncthreads();
    uint8_t *lb = levels + bi * cols * rows;
    const int ncol = (int)(cols - c0 < 32 ? cols - c0 : 32);
    const int total = ncol * (int)rows;
    for (int i = ty * 32 + tx; i < total; i += 256) {
        const int cc = i / (int)rows, r = i - cc * (int)rows;
        lb[(c0 + cc) * rows + r] = tile[cc][r];
    }
}

// Per-column quantisation with a transposed write: block (32, 8) owns 32
// columns of one batch entry; pass 1 reduces max|x| per column, pass 2 walks
// 32-row tiles and writes levels[c][r] through a shared-memory transpose so
// that both the fp32 reads and the byte writes are coalesced.
__global__ void __launch_bounds__(256) quant_cols_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t bstride, int half,
    int qmax, uint8_t *__restrict__ levels, float *__restrict__ scales, int32_t *dev_status) {
    __shared__ float red[8][33];
    __shared__ uint8_t tile[32][33];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int64_t bi = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * 32;
    const int64_t c = c0 + tx;
    const float *xb = x + bi * bstride;
    float amax = 0.0f;
    bool bad = false;
    if (c < cols) {
        // eight independent rows per thread in flight
        int64_t r = ty;
        for (; r + 56 < rows; r += 64) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = __ldg(xb + (r + 8 * k) * ld + c);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                bad |= !isfinite(v[k]);
                amax = fmaxf(amax, fabsf(v[k]));
            }
        }
        for (; r < rows; r += 8) {
            const float v = __ldg(xb + r * ld + c);
            bad |= !isfinite(v);
            amax = fmaxf(amax, fabsf(v));
        }
    }
    red[ty][tx] = amax;
    bad = __syncthreads_or(bad);
    if (ty == 0) {
        float m = red[0][tx];
        for (int k = 1; k < 8; ++k) m = fmaxf(m, red[k][tx]);
        red[0][tx] = __fdiv_rn(m, (float)qmax);
        if (c < cols) scales[bi * cols + c] = red[0][tx];
    }
    if (bad && tx == 0 && ty == 0 && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
    __syncthreads();
    const float s = red[0][tx], rs = __frcp_rn(s);
    uint8_t *lb = levels + bi * cols * rows;
    for (int64_t r0 = 0; r0 < rows; r0 += 32) {
        for (int k = ty; k < 32; k += 8) {
            const int64_t r = r0 + k;
            tile[tx][k] = (c < cols && r < rows) ? quant_level(__ldg(xb + r * ld + c), s, rs, half, qmax)
                                                 : (uint8_t)half;
        }
        __syncthreads();
        for (int k = ty; k < 32; k += 8) {
            const int64_t cc = c0 + k, r = r0 + tx;
            if (cc < cols && r < rows) lb[cc * rows + r] = tile[k][tx];
        }
        __syncthreads();
    }
}

int launch_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                    int64_t batch_stride, int axis, int sc_prec, int stat_mode, uint8_t *levels,
                    float *scales, float *stat, int32_t *dev_status, cudaStream_t stream) {
    const int half = 1 << (sc_prec - 1), qmax = half - 1;
    const int64_t bs = batch > 1 ? batch_stride : rows * ld;
    // float4 rows and packed 4-level stores: aligned input rows, 4-byte
    // aligned level rows
    const bool v4 = axis == 0 && cols % 4 == 0 && ld % 4 == 0 &&
                    (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (bs % 4 == 0 || batch == 1) &&
                    (reinterpret_cast<uintptr_t>(levels) & 3u) == 0;
    const bool vec_ok = v4 && cols <= 512;
    const bool block_ok = v4 && cols > 512 && cols <= 8192;
    if (block_ok) {
        int64_t blocks = rows * batch;
        const int64_t cap = (int64_t)sm_count() * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
#define SC_QB_ARGS x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status
        if (cols <= 1024)
            quant_rows_block_kernel<1><<<(unsigned)blocks, 256, 0, stream>>>(SC_QB_ARGS);
        else if (cols <= 2048)
            quant_rows_block_kernel<2><<<(unsigned)blocks, 256, 0, stream>>>(SC_QB_ARGS);
        else if (cols <= 4096)
            quant_rows_block_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(SC_QB_ARGS);
        else
            quant_rows_block_kernel<8><<<(unsigned)blocks, 256, 0, stream>>>(SC_QB_ARGS);
#undef SC_QB_ARGS
    } else if (vec_ok) {
        const int64_t cap = (int64_t)sm_count() * 8;
        auto grid_for = [&](int rpw) {
            int64_t b = (rows * batch + 8 * rpw - 1) / (8 * rpw);
            return (unsigned)(b > cap ? cap : (b < 1 ? 1 : b));
        };
        // 4 float4 per lane: the per-row reductions and scale are spread
        // over 16 elements per lane
        if (cols <= 32)
            quant_rows_vec_kernel<2, 4><<<grid_for(16), 256, 0, stream>>>(
                x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status);
        else if (cols <= 64)
            quant_rows_vec_kernel<4, 4><<<grid_for(8), 256, 0, stream>>>(
                x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status);
        else if (cols <= 128)
            quant_rows_vec_kernel<8, 4><<<grid_for(4), 256, 0, stream>>>(
                x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status);
        else if (cols <= 256)
            quant_rows_vec_kernel<16, 4><<<grid_for(2), 256, 0, stream>>>(
                x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status);
        else
            quant_rows_vec_kernel<32, 4><<<grid_for(1), 256, 0, stream>>>(
                x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status);
    } else if (axis == 0) {
        const int64_t warps = rows * batch;
        int64_t blocks = (warps + 7) / 8;
        const int64_t cap = (int64_t)sm_count() * 16;
        if (blocks > cap) blocks = cap;
#define SC_QR_ARGS x, rows, cols, ld, batch, bs, half, qmax, stat_mode, levels, scales, stat, dev_status
        if (cols <= 128)
            quant_rows_reg_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(SC_QR_ARGS);
        else if (cols <= 256)
            quant_rows_reg_kernel<8><<<(unsigned)blocks, 256, 0, stream>>>(SC_QR_ARGS);
        else if (cols <= 384)
            quant_rows_reg_kernel<12><<<(unsigned)blocks, 256, 0, stream>>>(SC_QR_ARGS);
        else if (cols <= 512)
            quant_rows_reg_kernel<16><<<(unsigned)blocks, 256, 0, stream>>>(SC_QR_ARGS);
        else
            quant_rows_kernel<<<(unsigned)blocks, 256, 0, stream>>>(SC_QR_ARGS);
#undef SC_QR_ARGS
    } else {
        if (batch > 65535) {
            set_error("sc_quantize: batch %lld too large for per-column mode", (long long)batch);
            return SC_ERR_UNSUPPORTED;
        }
        dim3 grid((unsigned)((cols + 31) / 32), (unsigned)batch);
        if (rows <= 8 * 40)  // short columns (AV's V: 257 rows) held in registers
            quant_cols_reg_kernel<40><<<grid, dim3(32, 8), 0, stream>>>(x, rows, cols, ld, bs, half, qmax,
                                                                      levels, scales, dev_status);
        else
            quant_cols_kernel<<<grid, dim3(32, 8), 0, stream>>>(x, rows, cols, ld, bs, half, qmax,
                                                              levels, scales, dev_status);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_quantize launch");
}

// ---------------------------------------------------------------------------
// Per-(row, chunk) quantisation for K-bands whose bands are whole quantisation
// chunks ("feat(mp) ... K-band", "Summary"); each chunk follows the per-row
// rule above, the row statistic is taken over the whole row.
// ---------------------------------------------------------------------------
// One warp per row; the warp walks the row's chunks with a chunk held in
// registers (NV float4 per lane, chunk <= 128 NV, chunk % 4 == 0, 16-byte
// aligned rows and chunks) and loads the next chunk before quantising the
// current one.
template <int NV>
__device__ __forceinline__ void load_chunk(float4 (&v)[NV], const float4 *xc, int64_t c4, int lane) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int64_t e = (int64_t)k * 32 + lane;
        v[k] = e < c4 ? __ldg(xc + e) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
}

template <int NV>
__global__ void __launch_bounds__(256) quant_chunks_vec_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
    int64_t bstride, int64_t chunk, int half, int qmax, int stat_mode, uint8_t *__restrict__ levels,
    float *__restrict__ scales, float *__restrict__ stat, int32_t *dev_status) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t nc = cols / chunk, c4 = chunk >> 2;
    const bool rowmax = stat_mode != SC_STAT_AMAX;
    bool bad_any = false;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows * batch;
         w += warps_total) {
        const int64_t bi = w / rows, r = w - bi * rows;
        const float4 *xr = reinterpret_cast<const float4 *>(x + bi * bstride + r * ld);
        uint32_t *lr = reinterpret_cast<uint32_t *>(levels + w * cols);
        float *sr = scales + w * nc;
        float4 cur[NV], nxt[NV];
        load_chunk<NV>(cur, xr, c4, lane);
        uint32_t row_bits = 0u;
        float row_max = -INFINITY;
        for (int64_t c = 0; c < nc; ++c) {
            if (c + 1 < nc) load_chunk<NV>(nxt, xr + (c + 1) * c4, c4, lane);
            uint32_t abits = 0u;
            float vmax = -INFINITY;
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                if ((int64_t)k * 32 + lane < c4) {
                    abits = max(abits, max(max(__float_as_uint(cur[k].x) & 0x7fffffffu,
                                               __float_as_uint(cur[k].y) & 0x7fffffffu),
                                           max(__float_as_uint(cur[k].z) & 0x7fffffffu,
                                               __float_as_uint(cur[k].w) & 0x7fffffffu)));
                    if (rowmax)
                        vmax = fmaxf(vmax, fmaxf(fmaxf(cur[k].x, cur[k].y), fmaxf(cur[k].z, cur[k].w)));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                abits = max(abits, __shfl_xor_sync(0xffffffffu, abits, o));
                if (rowmax) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
            }
            // integer max of sign-cleared bits: any inf or NaN sorts above
            // every finite value and flags the chunk
            const bool bad = abits >= 0x7f800000u;
            const float s = __fdiv_rn(__uint_as_float(abits), (float)qmax), rs = __frcp_rn(s);
            const bool fast = !bad && s > 0.0f;
            uint32_t *lc = lr + c * c4;
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                const int64_t e = (int64_t)k * 32 + lane;
                if (e >= c4) continue;
                if (fast)
                    lc[e] = quant_level_finite(cur[k].x, s, rs, half, qmax) |
                            (quant_level_finite(cur[k].y, s, rs, half, qmax) << 8) |
                            (quant_level_finite(cur[k].z, s, rs, half, qmax) << 16) |
                            (quant_level_finite(cur[k].w, s, rs, half, qmax) << 24);
                else
                    lc[e] = (uint32_t)quant_level(cur[k].x, s, rs, half, qmax) |
                            ((uint32_t)quant_level(cur[k].y, s, rs, half, qmax) << 8) |
                            ((uint32_t)quant_level(cur[k].z, s, rs, half, qmax) << 16) |
                            ((uint32_t)quant_level(cur[k].w, s, rs, half, qmax) << 24);
            }
            if (lane == 0) sr[c] = s;
            row_bits = max(row_bits, abits);
            row_max = fmaxf(row_max, vmax);
            bad_any |= bad;
#pragma unroll
            for (int k = 0; k < NV; ++k) cur[k] = nxt[k];
        }
        if (lane == 0 && stat) stat[w] = rowmax ? row_max : __uint_as_float(row_bits);
    }
    if (bad_any && lane == 0 && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
}

// Any chunk width or alignment: one warp per row, two passes per chunk (the
// second re-reads the chunk from L1 / L2).
__global__ void __launch_bounds__(256) quant_chunks_kernel(
    const float *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
    int64_t bstride, int64_t chunk, int half, int qmax, int stat_mode, uint8_t *__restrict__ levels,
    float *__restrict__ scales, float *__restrict__ stat, int32_t *dev_status) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t nc = cols / chunk;
    bool bad_any = false;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows * batch;
         w += warps_total) {
        const int64_t bi = w / rows, r = w - bi * rows;
        const float *xr = x + bi * bstride + r * ld;
        uint8_t *lr = levels + w * cols;
        float row_amax = 0.0f, row_max = -INFINITY;
        for (int64_t c = 0; c < nc; ++c) {
            const float *xc = xr + c * chunk;
            float amax = 0.0f, vmax = -INFINITY;
            bool bad = false;
            for (int64_t e = lane; e < chunk; e += 32) {
                const float v = __ldg(xc + e);
                bad |= !isfinite(v);
                amax = fmaxf(amax, fabsf(v));
                vmax = fmaxf(vmax, v);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
            }
            bad_any |= __any_sync(0xffffffffu, bad);
            const float s = __fdiv_rn(amax, (float)qmax), rs = __frcp_rn(s);
            for (int64_t e = lane; e < chunk; e += 32)
                lr[c * chunk + e] = quant_level(__ldg(xc + e), s, rs, half, qmax);
            if (lane == 0) scales[w * nc + c] = s;
            row_amax = fmaxf(row_amax, amax);
            row_max = fmaxf(row_max, vmax);
        }
        if (lane == 0 && stat) stat[w] = stat_mode == SC_STAT_AMAX ? row_amax : row_max;
    }
    if (bad_any && lane == 0 && dev_status) atomicOr(dev_status, SC_DEV_NONFINITE);
}

int launch_quantize_chunked(const float *x, int64_t rows, int64_t cols, int64_t ld, int64_t batch,
                            int64_t batch_stride, int64_t chunk, int sc_prec, int stat_mode,
                            uint8_t *levels, float *scales, float *stat, int32_t *dev_status,
                            cudaStream_t stream) {
    const int64_t bs = batch > 1 ? batch_stride : rows * ld;
    const int64_t nc = cols / chunk;
    // Without the row statistic and with packed rows, every chunk is a row of
    // a [rows * nc][chunk] matrix with the same level and scale layout.
    if (!stat && ld == cols && bs == rows * cols)
        return launch_quantize(x, rows * nc, chunk, chunk, batch, rows * cols, 0, sc_prec, stat_mode,
                               levels, scales, nullptr, dev_status, stream);
    const int half = 1 << (sc_prec - 1), qmax = half - 1;
    const bool vec_ok = chunk % 4 == 0 && ld % 4 == 0 && (bs % 4 == 0 || batch == 1) &&
                        (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && chunk <= 1024;
    int64_t blocks = (rows * batch + 7) / 8;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
#define SC_QC_ARGS x, rows, cols, ld, batch, bs, chunk, half, qmax, stat_mode, levels, scales, stat, dev_status
    if (vec_ok && chunk <= 128)
        quant_chunks_vec_kernel<1><<<(unsigned)blocks, 256, 0, stream>>>(SC_QC_ARGS);
    else if (vec_ok && chunk <= 256)
        quant_chunks_vec_kernel<2><<<(unsigned)blocks, 256, 0, stream>>>(SC_QC_ARGS);
    else if (vec_ok && chunk <= 512)
        quant_chunks_vec_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(SC_QC_ARGS);
    else if (vec_ok)
        quant_chunks_vec_kernel<8><<<(unsigned)blocks, 256, 0, stream>>>(SC_QC_ARGS);
    else
        quant_chunks_kernel<<<(unsigned)blocks, 256, 0, stream>>>(SC_QC_ARGS);
#undef SC_QC_ARGS
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_quantize_chunked launch");
}

// ---------------------------------------------------------------------------
// Rung assignment and rung-sorted order ("Precision As You Need", key design
// 2; "feat(mp) ... K-band", "How the banding works": rows grouped by rung).
// One block per group.  The sort is a stable counting sort: ranks inside a
// 1024-row chunk come from warp ballots, chunks are taken in row order.
// ---------------------------------------------------------------------------
struct TauArg {
    float tau[SC_MAX_RUNGS];
};

// GIVEN: the rungs are already in `rung` (fraction-based MP) and only the
// histogram and the rung-sorted order are built.
template <bool GIVEN>
__global__ void __launch_bounds__(1024) assign_rows_kernel(const float *__restrict__ stat,
                                                           int64_t rows, TauArg ta, int n_rungs,
                                                           int32_t *__restrict__ rung,
                                                           int32_t *__restrict__ perm,
                                                           int32_t *__restrict__ offsets) {
    __shared__ float wmax[32];
    __shared__ int hist[SC_MAX_RUNGS];
    __shared__ int base[SC_MAX_RUNGS];
    __shared__ int wcount[32][SC_MAX_RUNGS];
    __shared__ float s_gmax;
    const int64_t g = blockIdx.x;
    const float *st = stat + g * rows;
    int32_t *rg = rung + g * rows;
    int32_t *pm = perm + g * rows;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;

    float m = -INFINITY;
    if (!GIVEN)
        for (int64_t i = tid; i < rows; i += blockDim.x) m = fmaxf(m, st[i]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[wid] = m;
    if (tid < SC_MAX_RUNGS) hist[tid] = 0;
    __syncthreads();
    if (tid == 0) {
        float mm = wmax[0];
        for (int k = 1; k < nw; ++k) mm = fmaxf(mm, wmax[k]);
        s_gmax = mm;
    }
    __syncthreads();
    const float gmax = s_gmax;
    auto rung_of = [&](float v) {
        const float gt = gmax > 0.0f ? __fdiv_rn(v, gmax) : 0.0f;
        int k = 0;
        for (int t = 0; t + 1 < n_rungs; ++t) k += (gt >= ta.tau[t]) ? 1 : 0;
        return k;
    };
    int k_first = -1;  // rung of row tid, kept for the first pass of the sort
    for (int64_t i = tid; i < rows; i += blockDim.x) {
        int k;
        if (GIVEN) {
            k = rg[i];
        } else {
            k = rung_of(st[i]);
            rg[i] = k;
        }
        if (i == tid) k_first = k;
        atomicAdd(&hist[k], 1);
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int k = 0; k < n_rungs; ++k) {
            offsets[g * (n_rungs + 1) + k] = acc;
            base[k] = acc;
            acc += hist[k];
        }
        offsets[g * (n_rungs + 1) + n_rungs] = acc;
    }
    __syncthreads();
    for (int64_t c0 = 0; c0 < rows; c0 += blockDim.x) {
        const int64_t i = c0 + tid;
        const int k = i < rows ? (c0 == 0 ? k_first : rg[i]) : -1;
        int rank = 0;
        for (int kk = 0; kk < n_rungs; ++kk) {
            const unsigned mask = __ballot_sync(0xffffffffu, k == kk);
            if (k == kk) rank = __popc(mask & ((1u << lane) - 1u));
            if (lane == 0) wcount[wid][kk] = __popc(mask);
        }
        __syncthreads();
        if (k >= 0) {
            int before = base[k];
            for (int w = 0; w < wid; ++w) before += wcount[w][k];
            pm[before + rank] = (int32_t)i;
        }
        __syncthreads();
        if (tid < n_rungs) {
            int tot = 0;
            for (int w = 0; w < nw; ++w) tot += wcount[w][tid];
            base[tid] += tot;
        }
        __syncthreads();
    }
}

int launch_assign_rows(const float *stat, int64_t rows, int64_t batch, const float *tau,
                       int n_rungs, int32_t *rung, int32_t *perm, int32_t *rung_offsets,
                       cudaStream_t stream) {
    if (batch > 2147483647LL) {
        set_error("sc_assign_rows: batch too large");
        return SC_ERR_UNSUPPORTED;
    }
    TauArg ta;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) ta.tau[k] = (k + 1 < n_rungs) ? tau[k] : 0.0f;
    // one block per group, as many threads as rows (rounded to warps, at most
    // 1024): small groups leave room for several blocks per SM
    const int threads = (int)(rows >= 1024 ? 1024 : (rows < 64 ? 64 : (rows + 31) / 32 * 32));
    assign_rows_kernel<false><<<(unsigned)batch, threads, 0, stream>>>(stat, rows, ta, n_rungs, rung,
                                                                      perm, rung_offsets);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_assign_rows launch");
}

// ---------------------------------------------------------------------------
// Fraction-based fixed MP ("scmp_vit" README, MP flags): each length holds a
// given fraction of the units (rows, or whole (batch, head) matrices), the
// longest length going to the largest statistic.  Units are ordered by their
// statistic descending, NaN counted as -inf, ties to the lower index; the
// units of rung k and above are the first n_k of that order (n_k computed on
// the host from the fractions).  The rank of a unit is the number of units
// before it in that order.
// ---------------------------------------------------------------------------
struct FracArg {
    int32_t n_at[SC_MAX_RUNGS];  // n_at[k]: units at rung k or above (n_at[0] = all)
};

__device__ __forceinline__ float rank_key(float v) { return isnan(v) ? -INFINITY : v; }

__device__ __forceinline__ int rung_of_rank(int64_t rank, const FracArg &fa, int n_rungs) {
    int k = 0;
    for (int kk = 1; kk < n_rungs; ++kk) k += rank < fa.n_at[kk] ? 1 : 0;
    return k;
}

constexpr int FR_THREADS = 256, FR_TILE = 2048;

// Rows ranked within their group: block (x, g) ranks rows x*256 .. of group g
// against every row of the group, staged through shared memory.
__global__ void __launch_bounds__(FR_THREADS) frac_rank_rows_kernel(const float *__restrict__ stat,
                                                                    int64_t rows, FracArg fa,
                                                                    int n_rungs,
                                                                    int32_t *__restrict__ rung) {
    __shared__ float tile[FR_TILE];
    const int64_t g = blockIdx.y;
    const float *st = stat + g * rows;
    const int64_t i = (int64_t)blockIdx.x * FR_THREADS + threadIdx.x;
    const float ki = i < rows ? rank_key(st[i]) : 0.0f;
    int64_t rank = 0;
    for (int64_t t0 = 0; t0 < rows; t0 += FR_TILE) {
        const int tn = (int)min((int64_t)FR_TILE, rows - t0);
        __syncthreads();
        for (int t = threadIdx.x; t < tn; t += FR_THREADS) tile[t] = rank_key(st[t0 + t]);
        __syncthreads();
        if (i < rows) {
            int c = 0;
            for (int t = 0; t < tn; ++t) {
                const float kj = tile[t];
                c += (kj > ki || (kj == ki && t0 + t < i)) ? 1 : 0;
            }
            rank += c;
        }
    }
    if (i < rows) rung[g * rows + i] = rung_of_rank(rank, fa, n_rungs);
}

// Whole groups (heads) ranked within sets of set_size consecutive groups by
// their statistic max_i stat[g][i]; block (x, g) writes rows x*256 .. of g.
__global__ void __launch_bounds__(FR_THREADS) frac_rank_heads_kernel(const float *__restrict__ stat,
                                                                     int64_t rows, int64_t set_size,
                                                                     FracArg fa, int n_rungs,
                                                                     int32_t *__restrict__ rung) {
    __shared__ float wred[FR_THREADS / 32];
    __shared__ int64_t s_rank;
    const int64_t g = blockIdx.y, s0 = g - g % set_size;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    auto head_key = [&](int64_t h) {  // max over the head's rows (NaN ignored), then the key
        const float *st = stat + h * rows;
        float m = -INFINITY;
        for (int64_t r = threadIdx.x; r < rows; r += FR_THREADS) m = fmaxf(m, st[r]);
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        __syncthreads();
        if (lane == 0) wred[wid] = m;
        __syncthreads();
        float mm = wred[0];
        for (int w = 1; w < FR_THREADS / 32; ++w) mm = fmaxf(mm, wred[w]);
        return rank_key(mm);
    };
    const float kg = head_key(g);
    int64_t rank = 0;
    for (int64_t h = s0; h < s0 + set_size; ++h) {
        if (h == g) continue;
        const float kh = head_key(h);
        rank += (kh > kg || (kh == kg && h < g)) ? 1 : 0;
    }
    if (threadIdx.x == 0) s_rank = rank;
    __syncthreads();
    const int k = rung_of_rank(s_rank, fa, n_rungs);
    const int64_t i = (int64_t)blockIdx.x * FR_THREADS + threadIdx.x;
    if (i < rows) rung[g * rows + i] = k;
}

int launch_assign_fraction(const float *stat, int64_t rows, int64_t batch, int64_t set_size,
                           const int32_t *n_at, int n_rungs, int32_t *rung, int32_t *perm,
                           int32_t *rung_offsets, cudaStream_t stream) {
    if (batch > 65535) {
        set_error("sc_assign_fraction: batch %lld too large", (long long)batch);
        return SC_ERR_UNSUPPORTED;
    }
    FracArg fa;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) fa.n_at[k] = k < n_rungs ? n_at[k] : 0;
    if (rows > 0) {
        const dim3 grid((unsigned)((rows + FR_THREADS - 1) / FR_THREADS), (unsigned)batch);
        if (set_size == 0)
            frac_rank_rows_kernel<<<grid, FR_THREADS, 0, stream>>>(stat, rows, fa, n_rungs, rung);
        else
            frac_rank_heads_kernel<<<grid, FR_THREADS, 0, stream>>>(stat, rows, set_size, fa,
                                                                   n_rungs, rung);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "sc_assign_fraction rank launch");
    }
    TauArg ta;
    for (int k = 0; k < SC_MAX_RUNGS; ++k) ta.tau[k] = 0.0f;
    const int threads = (int)(rows >= 1024 ? 1024 : (rows < 64 ? 64 : (rows + 31) / 32 * 32));
    assign_rows_kernel<true><<<(unsigned)batch, threads, 0, stream>>>(stat, rows, ta, n_rungs, rung,
                                                                     perm, rung_offsets);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_assign_fraction launch");
}

// ---------------------------------------------------------------------------
// CUDA-core count engine.  One C-BSG count has the closed form
//     count(a, b, L) = C[b][n] + (L - n) - C[b][L - n],   n = C[a][L],
// which follows from the two enable-gated counters: at A's n ones B emits its
// first n bits, at A's L - n zeros its first L - n bits
// ("Precision As You Need", key design 1).  The prefix-count table C lives in
// shared memory; every (i, j, d) costs two gathers, whatever L is.
// Block tile 32 rows x 64 columns, 256 threads with 2 x 4 outputs each,
// contraction staged 32 at a time; persistent over tiles.
// ---------------------------------------------------------------------------
constexpr int GM = 32, GN = 64, GK = 32, GTHREADS = 256;

struct GatherArgs {
    int64_t M, N, D, batch;
    const uint8_t *a_lv;
    const float *a_s;
    const uint8_t *b_lv;
    const float *b_s;
    const int32_t *rung;
    const uint16_t *C;
    const uint16_t *CA;  // first operand's prefix counts (a variant of B's sequence), or null: C
    const uint8_t *Cpool;  // per-index pool: [n_pool][256][Q+1] prefix counts, index d uses d mod n_pool
    int n_pool;            // 0: no pool
    const int32_t *len;  // [n_bands_eff][n_rungs]
    int Q, n_rungs, n_bands_eff;
    int64_t chunk_d;     // band width (D when there are no bands)
    int band_scales;     // scales are [.][n_bands_eff]: one per (row, band)
    int unipolar;        // sign-magnitude AND streams (SC_MODE_UNIPOLAR)
    double q2;
    float *out;
    int32_t *counts;
    int32_t *dev_status;
    int64_t tiles_m, tiles_n;
};

__global__ void __launch_bounds__(GTHREADS, 1) gather_kernel(GatherArgs p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int W = p.Q + 1;
    uint16_t *sC = reinterpret_cast<uint16_t *>(smem);
    const size_t c_bytes = (((size_t)W * W * 2) + 15) & ~(size_t)15;
    uint32_t *sNM = reinterpret_cast<uint32_t *>(smem + c_bytes);        // [GM][GK] n | (L-n)<<16
    uint32_t *sB = sNM + GM * GK;                                         // [GK][GN/4] packed b
    int *sR = reinterpret_cast<int *>(sB + GK * (GN / 4));               // [GM] row constant
    int *sL = sR + GM;                                                    // [GM] L of row (band)
    int *sRung = sL + GM;                                                 // [GM]
    const int tid = threadIdx.x;

    for (int i = tid; i < W * W; i += GTHREADS) sC[i] = p.C[i];
    const int ty = tid / 16, tx = tid % 16;   // rows 2ty, 2ty+1; cols 4tx..4tx+3
    const int64_t tiles_per_g = p.tiles_m * p.tiles_n;
    const int64_t total = tiles_per_g * p.batch;
    bool range_bad = false;

    for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int64_t g = tile / tiles_per_g;
        const int64_t tm = (tile - g * tiles_per_g) / p.tiles_n;
        const int64_t tn = tile - g * tiles_per_g - tm * p.tiles_n;
        const int64_t i0 = tm * GM, j0 = tn * GN;
        const uint8_t *A = p.a_lv + (g * p.M) * p.D;
        const uint8_t *B = p.b_lv + (g * p.N) * p.D;
        __syncthreads();  // previous tile done with shared buffers (and sC loaded)
        if (tid < GM) {
            const int64_t i = i0 + tid;
            int k = i < p.M ? p.rung[g * p.M + i] : 0;
            if (k < 0 || k >= p.n_rungs) {
                range_bad = true;
                k = k < 0 ? 0 : p.n_rungs - 1;
            }
            sRung[tid] = k;
        }
        double dec[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) dec[r][c] = 0.0;

        for (int band = 0; band < p.n_bands_eff; ++band) {
            const int64_t d_lo = (int64_t)band * p.chunk_d;
            const int64_t d_hi = min(d_lo + p.chunk_d, p.D);
            __syncthreads();
            if (tid < GM) {
                sR[tid] = 0;
                sL[tid] = p.len[band * p.n_rungs + sRung[tid]];
            }
            int acc[2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = 0;
            for (int64_t d0 = d_lo; d0 < d_hi; d0 += GK) {
                const int kw = (int)min((int64_t)GK, d_hi - d0);
                __syncthreads();
                // stage A as (n, L - n) per (row, d) and B levels packed 4 columns per word
                for (int e = tid; e < GM * GK; e += GTHREADS) {
                    const int r = e / GK, dd = e % GK;
                    const int64_t i = i0 + r;
                    uint32_t nm = 0;
                    if (i < p.M && dd < kw) {
                        int a = A[i * p.D + d0 + dd];
                        if (a > p.Q) {
                            range_bad = true;
                            a = p.Q;
                        }
                        const int L = sL[r];
                        // pool: this index's sequence, rows of 256 levels
                        const uint8_t *Cq = p.n_pool ? p.Cpool + (size_t)((d0 + dd) % p.n_pool) * 256 * W : nullptr;
                        if (p.unipolar) {
                            // n = A's ones among L (magnitude level 2|x|), sign in bit 16
                            const int x = a - (p.Q >> 1);
                            const int ia = (2 * abs(x)) * W + L;
                            // magnitude level 256 (x = -128, never quantised) has every
                            // threshold below it: C[256][n] = n
                            const int n = Cq ? (2 * abs(x) > 255 ? L : (int)__ldg(Cq + 2 * abs(x) * W + L))
                                             : (p.CA ? (int)__ldg(p.CA + ia) : (int)sC[ia]);
                            nm = (uint32_t)n | ((x < 0 ? 1u : 0u) << 16);
                        } else {
                            const int n = Cq ? (int)__ldg(Cq + min(a, 255) * W + L)
                                             : (p.CA ? (int)__ldg(p.CA + a * W + L) : (int)sC[a * W + L]);
                            nm = (uint32_t)n | ((uint32_t)(L - n) << 16);
                            atomicAdd(&sR[r], L - n);
                        }
                    }
                    sNM[r * GK + dd] = nm;
                }
                for (int e = tid; e < GK * (GN / 4); e += GTHREADS) {
                    const int dd = e / (GN / 4), q4 = e % (GN / 4);
                    uint32_t packed = 0;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int64_t j = j0 + q4 * 4 + u;
                        int b = 0;
                        if (j < p.N && dd < kw) {
                            b = B[j * p.D + d0 + dd];
                            if (b > p.Q) {
                                range_bad = true;
                                b = p.Q;
                            }
                        }
                        packed |= (uint32_t)b << (8 * u);
                    }
                    sB[dd * (GN / 4) + q4] = packed;
                }
                __syncthreads();
                if (p.n_pool) {
                    // per-index pool: the index's prefix counts from global memory
                    const int half = p.Q >> 1;
                    for (int dd = 0; dd < kw; ++dd) {
                        const uint8_t *Cq = p.Cpool + (size_t)((d0 + dd) % p.n_pool) * 256 * W;
                        const uint32_t nm0 = sNM[(2 * ty) * GK + dd];
                        const uint32_t nm1 = sNM[(2 * ty + 1) * GK + dd];
                        const uint32_t b4 = sB[dd * (GN / 4) + tx];
                        const int n0 = nm0 & 0xffff, n1 = nm1 & 0xffff;
                        if (p.unipolar) {
                            const bool neg0 = (nm0 >> 16) != 0, neg1 = (nm1 >> 16) != 0;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int xb = (int)((b4 >> (8 * c)) & 0xff) - half;
                                const int mb = 2 * abs(xb);
                                const uint8_t *row = Cq + min(mb, 255) * W;
                                const int v0 = mb > 255 ? n0 : __ldg(row + n0);
                                const int v1 = mb > 255 ? n1 : __ldg(row + n1);
                                acc[0][c] += ((xb < 0) != neg0) ? -v0 : v0;
                                acc[1][c] += ((xb < 0) != neg1) ? -v1 : v1;
                            }
                        } else {
                            const int m0 = nm0 >> 16, m1 = nm1 >> 16;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint8_t *row = Cq + (int)((b4 >> (8 * c)) & 0xff) * W;
                                acc[0][c] += (int)__ldg(row + n0) - (int)__ldg(row + m0);
                                acc[1][c] += (int)__ldg(row + n1) - (int)__ldg(row + m1);
                            }
                        }
                    }
                } else if (p.unipolar) {
                    // signed AND count: B's first n bits, n = A's ones,
                    // C[2|x_b|][n] with the sign of x_a x_b
                    const int half = p.Q >> 1;
                    for (int dd = 0; dd < kw; ++dd) {
                        const uint32_t nm0 = sNM[(2 * ty) * GK + dd];
                        const uint32_t nm1 = sNM[(2 * ty + 1) * GK + dd];
                        const uint32_t b4 = sB[dd * (GN / 4) + tx];
                        const int n0 = nm0 & 0xffff, n1 = nm1 & 0xffff;
                        const bool neg0 = (nm0 >> 16) != 0, neg1 = (nm1 >> 16) != 0;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int xb = (int)((b4 >> (8 * c)) & 0xff) - half;
                            const int row = (2 * abs(xb)) * W;
                            const int v0 = sC[row + n0], v1 = sC[row + n1];
                            acc[0][c] += ((xb < 0) != neg0) ? -v0 : v0;
                            acc[1][c] += ((xb < 0) != neg1) ? -v1 : v1;
                        }
                    }
                } else {
                    for (int dd = 0; dd < kw; ++dd) {
                        const uint32_t nm0 = sNM[(2 * ty) * GK + dd];
                        const uint32_t nm1 = sNM[(2 * ty + 1) * GK + dd];
                        const uint32_t b4 = sB[dd * (GN / 4) + tx];
                        const int n0 = nm0 & 0xffff, m0 = nm0 >> 16, n1 = nm1 & 0xffff, m1 = nm1 >> 16;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int row = ((b4 >> (8 * c)) & 0xff) * W;
                            acc[0][c] += (int)sC[row + n0] - (int)sC[row + m0];
                            acc[1][c] += (int)sC[row + n1] - (int)sC[row + m1];
                        }
                    }
                }
            }
            __syncthreads();
            const int64_t Db = d_hi - d_lo;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int rr = 2 * ty + r;
                const int64_t i = i0 + rr;
                const int L = sL[rr];
                const int R = sR[rr];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int64_t j = j0 + 4 * tx + c;
                    const int cnt = acc[r][c] + R;
                    if (i < p.M && j < p.N) {
                        if (p.counts)
                            p.counts[((g * p.n_bands_eff + band) * p.M + i) * p.N + j] = cnt;
                        double term = p.unipolar ? (double)cnt / (double)L
                                                 : (double)(2LL * cnt - Db * (int64_t)L) / (double)L;
                        if (p.band_scales)
                            term *= (double)p.a_s[(g * p.M + i) * p.n_bands_eff + band] *
                                    (double)p.b_s[(g * p.N + j) * p.n_bands_eff + band];
                        dec[r][c] += term;
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int64_t i = i0 + 2 * ty + r;
            if (i >= p.M) continue;
            const double sa = p.band_scales ? 0.0 : (double)p.a_s[g * p.M + i];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t j = j0 + 4 * tx + c;
                if (j < p.N)
                    p.out[(g * p.M + i) * p.N + j] =
                        p.band_scales ? (float)(p.q2 * dec[r][c])
                                      : (float)(sa * (double)p.b_s[g * p.N + j] * p.q2 * dec[r][c]);
            }
        }
    }
    if (range_bad && p.dev_status) atomicOr(p.dev_status, SC_DEV_LEVEL_RANGE);
}

int launch_gather(const sc_matmul_desc &d, double q_dec, const uint8_t *a_lv, const float *a_s,
                  const uint8_t *b_lv, const float *b_s, const int32_t *rung, const sc_table &t,
                  float *out, int32_t *counts, int32_t *dev_status, cudaStream_t stream) {
    GatherArgs p;
    p.M = d.M;
    p.N = d.N;
    p.D = d.D;
    p.batch = d.batch;
    p.a_lv = a_lv;
    p.a_s = a_s;
    p.b_lv = b_lv;
    p.b_s = b_s;
    p.rung = rung;
    p.C = t.d_C;
    p.CA = t.d_CA;
    p.Cpool = t.d_Cpool;
    p.n_pool = t.n_pool;
    p.len = t.d_len;
    p.Q = t.Q;
    p.n_rungs = t.n_rungs;
    p.n_bands_eff = t.n_bands > 0 ? t.n_bands : 1;
    p.chunk_d = t.n_bands > 0 ? t.chunk_d : d.D;
    p.band_scales = d.scales == SC_SCALES_BAND;
    p.unipolar = d.mode == SC_MODE_UNIPOLAR;
    p.q2 = q_dec * q_dec;
    p.out = out;
    p.counts = counts;
    p.dev_status = dev_status;
    p.tiles_m = (d.M + GM - 1) / GM;
    p.tiles_n = (d.N + GN - 1) / GN;
    const int W = t.Q + 1;
    const size_t c_bytes = (((size_t)W * W * 2) + 15) & ~(size_t)15;
    const size_t smem = c_bytes + (size_t)GM * GK * 4 + (size_t)GK * (GN / 4) * 4 + 3 * GM * 4;
    cudaError_t e = cudaFuncSetAttribute(gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "sc_matmul gather: smem attribute");
    int64_t total = p.tiles_m * p.tiles_n * p.batch;
    int64_t grid = (int64_t)sm_count();
    if (grid > total) grid = total;
    gather_kernel<<<(unsigned)grid, GTHREADS, smem, stream>>>(p);
    e = cudaGetLastError();
    return e == cudaSuccess ? SC_OK : cuda_fail(e, "sc_matmul gather launch");
}

}  // namespace scb
