// layer_t1.cu -- fused single-token layer forward (both projections in one
// launch).  Not built yet: the general path serves T = 1.
#include "common.cuh"

namespace bitsmoe {

uint64_t layer_fused_t1_workspace(const bitsmoe_plan*, const bitsmoe_plan*) { return 0; }

int layer_forward_fused_t1(const bitsmoe_proj_io**, const uint16_t*, const int32_t*, const float*, void*, uint64_t,
                           int32_t*, cudaStream_t, bool* used) {
    *used = false;
    return BITSMOE_OK;
}

}  // namespace bitsmoe
