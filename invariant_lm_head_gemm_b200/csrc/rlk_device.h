// rlk_device.h -- the library's device check, shared by its source files.
#pragma once

#include "rlk.h"

namespace rlk {

// RLK_OK when the current CUDA device is compute capability 10.0 (its SM
// count in *num_sms), RLK_ERR_UNSUPPORTED_DEVICE when there is no such
// device, RLK_ERR_CUDA when a query fails.
rlk_status current_device_supported(int* num_sms);

}  // namespace rlk
