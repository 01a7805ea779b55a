// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "../../include/w4a16.h"

namespace w4a16 {

// W4A16_OK if the current device is an sm_100 part this library was built for,
// W4A16_ERR_UNSUPPORTED otherwise (including "no CUDA device").
int check_device();

// Streaming multiprocessors of the current device (0 if unknown).
int sm_count();

}  // namespace w4a16
