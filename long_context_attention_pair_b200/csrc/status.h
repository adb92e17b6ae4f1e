// Status codes shared by the C ABI and the kernels.
#pragma once
#include "atflash.h"

// A kernel whose bounded wait ran out writes ATFLASH_DEVICE_TIMEOUT_BASE + site
// into the device status word (first writer wins); the host maps any value at
// or above the base to ATFLASH_ERR_TIMEOUT.
#define ATFLASH_DEVICE_TIMEOUT_BASE 1000
// A paged decode that met a page index past its block-table row, or a page id
// outside the pool, writes this value (first writer wins); the host maps it to
// ATFLASH_ERR_BAD_PAGE.
#define ATFLASH_DEVICE_BAD_PAGE 2000

// Waits that only let a CTA's own copies and tensor-core work finish before it
// exits (after a pipeline wait has given up) use at least this limit, so that a
// short pipeline limit never frees TMEM or shared memory under work in flight.
#define ATFLASH_DRAIN_FLOOR_NS 200000000ull
#ifdef __CUDACC__
__host__ __device__ inline unsigned long long atflash_drain_limit_ns(unsigned long long pipeline_limit_ns) {
    return pipeline_limit_ns > ATFLASH_DRAIN_FLOOR_NS ? pipeline_limit_ns : ATFLASH_DRAIN_FLOOR_NS;
}
#endif
