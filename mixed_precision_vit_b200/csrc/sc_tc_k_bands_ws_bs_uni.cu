// sc_tc_k_bands_ws_bs_uni.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): as bands_ws_bs, unipolar AND mode.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands_ws_bs_uni() { return tc_kernel<SK_PLAIN, true, true, true, true>; }

}  // namespace tcd
}  // namespace scb
