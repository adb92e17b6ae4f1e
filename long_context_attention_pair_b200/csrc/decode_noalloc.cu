// Decode entry point that allocates nothing.
//
// atflash_decode needs a scratch buffer for the per-split softmax states
// (max, sum and un-normalised output of every split of every query head) and
// asks the caller for it.  Some callers cannot allocate device memory when they
// call us: a serving loop that must never enter the CUDA allocator once it is
// running (cudaMalloc can synchronise the device and stall other streams), or
// a plugin whose host framework owns every byte of device memory and offers
// it no allocation hook.  atflash_decode_noalloc serves them: the scratch is a
// fixed array in this file, reserved on every GPU that loads the library and
// kept until the process exits.  The caller still passes inputs and outputs.
//
// Limits and rules of use:
//  - the split states must fit in ATFLASH_NOALLOC_SCRATCH_BYTES; larger
//    problems are rejected with ATFLASH_ERR_WORKSPACE before anything runs;
//  - the array is part of the library's device image, so every process that
//    loads the library holds its 32 MiB on every GPU it uses, whether or not it
//    ever calls this entry point;
//  - every call on a device shares the one array, so two calls whose work
//    overlaps on the GPU (different streams without ordering between them)
//    race on it; calls queued on one stream are ordered and safe;
//  - the first call on a device looks up the array's device address once
//    (with that device current) and keeps it; make that first call before any
//    stream capture begins, and do not reset the device (cudaDeviceReset)
//    after it, since the kept address would then be stale.
// Arguments are checked by the same code as atflash_decode's (decode_check), so
// both reject the same arguments with the same status.  The array keeps the
// last call's contents.  Nothing in it needs to start at zero: the split kernel
// writes every state the merge kernel reads.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"

namespace atf {
namespace {

constexpr size_t kScratchBytes = ATFLASH_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must be a multiple of 256 bytes");

// Device-side scratch.  In host code this name is only a handle: its address
// here is NOT a device address, so it is never passed to a kernel directly.
static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

std::mutex g_mu;
float *g_dev_ptr[64];  // device address of the array, per device ordinal

// Device address of the array on the current device (looked up once per device).
int scratch_on_current_device(float **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATFLASH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_ptr[dev]) {
        float *ptr = nullptr;
        if (cudaGetSymbolAddress((void **)&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return ATFLASH_ERR_CUDA;
        g_dev_ptr[dev] = ptr;
    }
    *out = g_dev_ptr[dev];
    return ATFLASH_OK;
}

}  // namespace
}  // namespace atf

using namespace atf;

extern "C" int atflash_decode_noalloc(const void *q, const void *kcache, const void *vcache,
                                      const int32_t *seqlens, void *out, int B, int Hq, int Hkv, int64_t Nmax,
                                      int D, double rope_base, double k_window, int kcache_rotated, int kv_layout,
                                      int in_dtype, int out_dtype, cudaStream_t stream) {
    if (!q || !kcache || !vcache || !seqlens || !out) return ATFLASH_ERR_INVALID_ARG;
    double theta[kMaxPairs];
    int rc = theta_from_base(D, rope_base, theta);
    if (rc != ATFLASH_OK) return rc;
    size_t need = 0;
    rc = decode_check(q, kcache, vcache, seqlens, out, B, Hq, Hkv, Nmax, D, theta, k_window, kcache_rotated,
                      kv_layout, in_dtype, out_dtype, &need);
    if (rc != ATFLASH_OK) return rc;
    if (need > kScratchBytes) return ATFLASH_ERR_WORKSPACE;
    float *scratch = nullptr;
    if ((rc = scratch_on_current_device(&scratch)) != ATFLASH_OK) return rc;
    return decode_run(q, kcache, vcache, seqlens, out, B, Hq, Hkv, Nmax, D, theta, k_window, kcache_rotated,
                      kv_layout, in_dtype, out_dtype, scratch, stream);
}
