// sc_tc_k_narrow.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): no bands, 512-byte stages, tiles of up to 64 columns.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_narrow() { return tc_kernel<SK_NARROW, false>; }

}  // namespace tcd
}  // namespace scb
