// Internal interface of the fused-linear cross-entropy translation unit.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ceb {
unsigned int* error_word();
int device_sms(int num_sms);
}  // namespace ceb
