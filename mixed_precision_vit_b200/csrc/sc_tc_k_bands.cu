// sc_tc_k_bands.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): K-bands, fp64 band sums in tensor memory.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands() { return tc_kernel<SK_BANDS, true>; }

}  // namespace tcd
}  // namespace scb
