// sc_tc_k_bands.cu -- instantiation of one variant of the tensor-core count
// kernel (see sc_tc_dev.cuh); kept apart so that the variants compile in
// parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands(bool band_scales) {
    return band_scales ? tc_kernel<SK_BANDS, true, true> : tc_kernel<SK_BANDS, true>;
}

}  // namespace tcd
}  // namespace scb
