// sc_tc_k_bands_bs.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): as bands, one scale per (row, band).  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_bands_bs() { return tc_kernel<SK_BANDS, true, true>; }

}  // namespace tcd
}  // namespace scb
