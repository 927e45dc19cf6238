// sc_tc_k_bands_ws.cu -- instantiation of one variant of the tensor-core count
// kernel (see sc_tc_dev.cuh); kept apart so that the variants compile in
// parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands_ws(bool band_scales) {
    return band_scales ? tc_kernel<SK_PLAIN, true, true, true> : tc_kernel<SK_PLAIN, true, false, true>;
}

}  // namespace tcd
}  // namespace scb
