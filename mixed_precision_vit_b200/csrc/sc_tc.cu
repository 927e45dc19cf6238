// sc_tc.cu -- tcgen05 tensor-core count engine (placeholder until implemented).
#include "sc_internal.cuh"

namespace scb {

bool tc_supports(const sc_matmul_desc &, const sc_table &) { return false; }

int launch_tc(const sc_matmul_desc &, double, const uint8_t *, const float *, const uint8_t *,
              const float *, const int32_t *, const int32_t *, const int32_t *, const sc_table &,
              float *, int32_t *, int32_t *, cudaStream_t) {
    set_error("sc_matmul: tensor-core engine not available in this build");
    return SC_ERR_UNSUPPORTED;
}

}  // namespace scb
