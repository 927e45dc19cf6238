// sc_tc_k_bands_ws_uni.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): as bands_ws, unipolar AND mode.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands_ws_uni() { return tc_kernel<SK_PLAIN, true, false, true, true>; }

}  // namespace tcd
}  // namespace scb
