// sc_tc_k_single_uni.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): as single, unipolar AND mode.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_single_uni() { return tc_kernel<SK_PLAIN, false, false, false, true, 1>; }

}  // namespace tcd
}  // namespace scb
