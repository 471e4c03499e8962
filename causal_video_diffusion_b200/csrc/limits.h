// limits.h -- the device-side wait limit shared by every kernel's launch parameters.
#pragma once

#include <cstdint>

namespace unstep {

// Default limit of every device-side wait: no legitimate wait of these kernels lasts this long.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace unstep
