// sc_tc_k_narrow.cu -- instantiation of one variant of the tensor-core count
// kernel (see sc_tc_dev.cuh); kept apart so that the variants compile in
// parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_narrow() { return tc_kernel<SK_NARROW, false>; }

}  // namespace tcd
}  // namespace scb
