// sc_tc_k_plain.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): no bands, 256-byte stages, tiles of up to 160 columns.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_plain() { return tc_kernel<SK_PLAIN, false>; }

}  // namespace tcd
}  // namespace scb
