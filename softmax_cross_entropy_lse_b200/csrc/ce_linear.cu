// Fused-linear cross-entropy (Z = H W^T never stored). Placeholder entry
// points until the tensor-core kernels land.
#include "ce_b200.h"
#include "ce_linear.h"

extern "C" {

size_t linear_ce_workspace_size(int64_t, int64_t, int64_t, int) { return 0; }

ce_status linear_ce_forward(const void*, int64_t, const void*, int64_t, const void*,
                            ce_index_dtype, int64_t, int64_t, int64_t, float, int64_t,
                            float*, float*, void*, size_t, void*) {
    return CE_ENOTSUP;
}

size_t linear_ce_backward_workspace_size(int64_t, int64_t, int64_t, int) { return 0; }

ce_status linear_ce_backward(const float*, int64_t, const void*, int64_t, const void*, int64_t,
                             const void*, ce_index_dtype, const float*, int64_t, int64_t,
                             int64_t, float, int64_t, void*, ce_dtype, void*, ce_dtype, void*,
                             size_t, void*) {
    return CE_ENOTSUP;
}

}  // extern "C"
