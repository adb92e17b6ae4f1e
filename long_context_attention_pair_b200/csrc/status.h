// Status codes shared by the C ABI and the kernels.
#pragma once
#include "atflash.h"

// A kernel whose bounded wait ran out writes ATFLASH_DEVICE_TIMEOUT_BASE + site
// into the device status word (first writer wins); the host maps any value at
// or above the base to ATFLASH_ERR_TIMEOUT.
#define ATFLASH_DEVICE_TIMEOUT_BASE 1000
