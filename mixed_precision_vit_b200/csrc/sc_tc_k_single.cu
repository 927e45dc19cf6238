// sc_tc_k_single.cu -- one instantiation of the tensor-core count kernel
// (sc_tc_dev.cuh): one CTA per MMA (M = 128), no bands, 256-byte stages, tiles of up to 64 columns.  Each variant sits in its own unit so that
// the variants compile in parallel.
#include "sc_tc_dev.cuh"

namespace scb {
namespace tcd {

TcKernelFn tc_kernel_single() { return tc_kernel<SK_PLAIN, false, false, false, false, 1>; }

}  // namespace tcd
}  // namespace scb
