// sc_tc_k_narrow_uni.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): as narrow, unipolar AND mode.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_narrow_uni() { return tc_kernel<SK_NARROW, false, false, false, true>; }

}  // namespace tcd
}  // namespace scb
