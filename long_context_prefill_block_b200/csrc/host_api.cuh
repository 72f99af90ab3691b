// Host-side helpers shared by the files that implement the C ABI (api.cu,
// gate_noalloc.cu). Nothing here is visible outside libmoba.so.
#pragma once

#include "common.cuh"
#include "moba.h"

namespace moba {

// Checks the parameters and fills the launch sizes: the one place that
// decides which parameters the library accepts.
moba_status validate(const moba_params* p, Dims& dm);

// Device address of the per-device status word on the current device, or
// nullptr if it cannot be looked up.
int* status_word();

}  // namespace moba
