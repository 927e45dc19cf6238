// sc_static_ws.cu -- sc_matmul with a library-owned, statically sized scratch
// buffer instead of a caller workspace.  The source pages have no counterpart
// to this entry point: it is a convenience of this library for callers that
// cannot allocate device memory.
//
// It serves callers that cannot allocate device memory (code inside a
// framework that owns every device allocation, or a process that must not
// grow its footprint after start-up).  The scratch is one file-scope
// __device__ array per device (present from the moment the module is loaded
// until the process exits, never allocated by the call); its address is
// looked up on the first call on each device and kept once the lookup has
// succeeded (a failed lookup is retried by the next call).  Every call on a
// device uses the same array, so calls that may overlap in time (different
// streams, or different host threads) race on it: callers serialise them,
// e.g. by issuing all of them on one stream per device.
#include <mutex>

#include "sc_internal.cuh"

namespace scb {
namespace {

static __device__ __align__(256) unsigned char g_static_ws[SC_STATIC_WS_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mutex[MAX_DEVICES];
void *g_addr[MAX_DEVICES];  // null until a lookup on that device has succeeded

}  // namespace
}  // namespace scb

extern "C" int sc_matmul_static_ws(const sc_matmul_desc *desc, const uint8_t *a_lv,
                                   const float *a_s, const uint8_t *b_lv, const float *b_s,
                                   const int32_t *rung, const int32_t *perm,
                                   const int32_t *rung_offsets, const sc_table *table, float *out,
                                   int32_t *counts, int32_t *dev_status, void *stream) {
    using namespace scb;
    clear_error();
    if (!desc || !table) {
        set_error("sc_matmul_static_ws: desc or table is null");
        return SC_ERR_ARG;
    }
    if (desc->workspace || desc->workspace_bytes) {
        set_error("sc_matmul_static_ws: the descriptor must not name a workspace");
        return SC_ERR_ARG;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "sc_matmul_static_ws: cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEVICES) {
        set_error("sc_matmul_static_ws: device %d out of range", dev);
        return SC_ERR_UNSUPPORTED;
    }
    void *scratch = nullptr;
    {
        // the host-side name of the array is not a device address: ask the
        // runtime for this device's copy, with the device current
        std::lock_guard<std::mutex> lock(g_mutex[dev]);
        if (!g_addr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_static_ws);
            if (e != cudaSuccess) return cuda_fail(e, "sc_matmul_static_ws: scratch address");
            g_addr[dev] = p;
        }
        scratch = g_addr[dev];
    }
    sc_matmul_desc d = *desc;
    d.workspace = scratch;
    d.workspace_bytes = SC_STATIC_WS_BYTES;
    // the wide-tile band kernel fits if one slice of band sums does (it then
    // splits the bands into as many segments as the buffer holds)
    const int eng = sc_matmul_engine(&d, table);
    if (eng < 0) return -eng;
    const int64_t need = eng == SC_ENGINE_TC ? tc_workspace_min_bytes(d, *table) : 0;
    if (need > SC_STATIC_WS_BYTES) {
        set_error("sc_matmul_static_ws: the problem needs %lld bytes of scratch, the static buffer "
                  "holds %lld",
                  (long long)need, (long long)SC_STATIC_WS_BYTES);
        return SC_ERR_UNSUPPORTED;
    }
    return sc_matmul(&d, a_lv, a_s, b_lv, b_s, rung, perm, rung_offsets, table, out, counts,
                     dev_status, stream);
}
