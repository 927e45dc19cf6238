// sc_tc_k_plain.cu -- instantiation of one variant of the tensor-core count
// kernel (see sc_tc_dev.cuh); kept apart so that the variants compile in
// parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_plain() { return tc_kernel<SK_PLAIN, false>; }

}  // namespace tcd
}  // namespace scb
