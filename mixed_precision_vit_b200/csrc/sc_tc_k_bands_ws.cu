// sc_tc_k_bands_ws.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): K-bands, fp64 band sums in the caller workspace.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands_ws() { return tc_kernel<SK_PLAIN, true, false, true>; }

}  // namespace tcd
}  // namespace scb
