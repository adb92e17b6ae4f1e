// Internal interfaces between the C ABI (api.cu) and the kernel launchers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "status.h"

namespace atf {

constexpr int kMaxPairs = 128;  // D <= 256

// Host-side window math (window.cpp).  theta_r = base^(-2r/D),
// lambda_r = 2*pi/theta_r, w_r = floor(k*lambda_r) clamped to N-1.
int window_table(int D, double base, double k, int64_t N, int64_t *w);
int pruned_terms(int64_t N, int D, double base, double k, atflash_terms *out);
void theta_table(int D, double base, double *theta);
bool theta_valid(int D, const double *theta);
int window_table_theta(int D, const double *theta, double k, int64_t N, int64_t *w);
int pruned_terms_theta(int64_t N, int D, const double *theta, double k, atflash_terms *out);

// Programmatic dependent launch (sm_90 and later).  A kernel launched with
// launch_dependent() may be scheduled while the previous kernel in the stream
// still runs; it must call pdl_wait() before it touches anything that kernel
// writes (the wait returns once the previous kernel has completed and its
// memory operations are visible; in a kernel launched without the attribute it
// returns at once).  pdl_allow_dependents() lets the dependent launch begin
// before the calling kernel ends.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
static inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                           cudaStream_t s, Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
#endif

// Per-call constants shared by every kernel of one call.
struct WindowParams {
    int H;                      // D/2 pairs
    int32_t w[kMaxPairs];       // per-pair window, clamped to N-1 (non-decreasing in r)
    double theta[kMaxPairs];    // theta_r in fp64 (RoPE angles are reduced in fp64)
};

struct Problem {
    int B, Hq, Hkv, D;
    int64_t N;
};

// RoPE pre-pass: rotate q and k once per token into the layouts the prefill
// kernels read.  bf16 path: packed [b*H+h][D/16][N][16] bf16, pair-interleaved
// (element 2j of chunk c is x~_{8c+j}, element 2j+1 is x~_{8c+j+D/2}).
// fp32 path: [b*H+h][N][D] fp32 pair-interleaved.
// cu (device, nseq + 1 entries) != nullptr: the token axis holds several
// sequences and each token is rotated by its position within its sequence.
cudaError_t launch_rope_pack_bf16(const void *x, void *y, int B, int64_t N, int Hx, int D,
                                  const WindowParams &wp, cudaStream_t s, const int32_t *cu = nullptr,
                                  int nseq = 0);
cudaError_t launch_rope_pack_f32(const void *x, void *y, int B, int64_t N, int Hx, int D,
                                 const WindowParams &wp, cudaStream_t s);

// Exact fp32 CUDA-core prefill over pre-rotated fp32 Q~/K~.
cudaError_t launch_prefill_simt_f32(const float *qt, const float *kt, const float *v, void *out, int out_f32,
                                    float *lse, const Problem &p, const WindowParams &wp, cudaStream_t s);

// tcgen05 prefill over the packed bf16 Q~/K~ and the caller's bf16 V.
// cu_seqlens (device, B + 1 entries) != nullptr: q/k/v/out and the packed
// Q~/K~ hold a batch of `total` tokens packed along the token axis; p.N is the
// longest sequence.  block_mask (device, [B][Hkv][T][T] uint8, T = ceil(N/128))
// != nullptr: token-level block selection (not with cu_seqlens).
cudaError_t launch_prefill_tc(const void *qpack, const void *kpack, const void *v, void *out, int out_f32,
                              float *lse, const Problem &p, const WindowParams &wp, int *status,
                              uint64_t wait_limit_ns, cudaStream_t s, const int32_t *cu_seqlens = nullptr,
                              int64_t total = 0, const uint8_t *block_mask = nullptr);

// A paged KV cache: keys i*page_size.. of sequence b are in pool page
// block_table[b*max_pages + i]; page_size is a multiple of 64.
struct PagedKV {
    const int32_t *block_table;  // device, [B][max_pages]
    int max_pages, page_size, num_pages;
};

// Rows that see at most 128 keys, recomputed in fp32 on CUDA cores from the
// caller's un-rotated bf16 q, k, v after the tensor-core kernel (short_rows.cu):
// the first 128-row tile of every sequence, or with a block mask every query
// tile whose mask row selects no earlier key tile.  Overwrites those rows of out
// (and lse).  q/k/v/out/lse/cu_seqlens/block_mask as for launch_prefill_tc, with
// the caller's natural q, k instead of the packed ones.
cudaError_t launch_short_rows_prefill(const void *q, const void *k, const void *v, void *out, int out_f32,
                                      float *lse, const Problem &p, const WindowParams &wp, int *status,
                                      cudaStream_t s, const int32_t *cu_seqlens = nullptr, int64_t total = 0,
                                      const uint8_t *block_mask = nullptr);
// The same for a bf16 decode: every sequence of at most 128 tokens, recomputed
// in fp32 after the merge (any cache layout, contiguous or paged).
cudaError_t launch_short_rows_decode(const void *q, const void *kc, const void *vc, const int32_t *seqlens,
                                     void *out, int out_f32, int krot, int layout, const Problem &p,
                                     const WindowParams &wp, int *status, cudaStream_t s,
                                     const PagedKV *paged = nullptr);

// Split-KV decode + merge.
int decode_split_keys(int B, int Hkv, int64_t Nmax);
int decode_num_splits(int B, int Hkv, int64_t Nmax);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int D);

cudaError_t launch_decode_tc(const void *q, const void *kc, const void *vc, const int32_t *seqlens, int krot,
                             int layout, const Problem &p, const WindowParams &wp, float *workspace, int split_keys,
                             int nsplit, int *status, uint64_t limit_ns, cudaStream_t s,
                             const PagedKV *paged = nullptr);

// theta_r = base^(-2r/D) into theta (D/2 entries) after the base-taking calls'
// checks (even D in 2..256, base > 1); ATFLASH_ERR_INVALID_ARG otherwise.
int theta_from_base(int D, double base, double *theta);

// atflash_decode in two halves (api.cu): decode_check validates the arguments
// exactly as atflash_decode does and reports the scratch bytes the call needs;
// decode_run builds the window table and launches into a workspace of at least
// that size.  theta: host table of D/2 frequencies.
int decode_check(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out, int B,
                 int Hq, int Hkv, int64_t Nmax, int D, const double *theta, double k_window, int kcache_rotated,
                 int kv_layout, int in_dtype, int out_dtype, size_t *need);
int decode_run(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out, int B,
               int Hq, int Hkv, int64_t Nmax, int D, const double *theta, double k_window, int kcache_rotated,
               int kv_layout, int in_dtype, int out_dtype, float *workspace, cudaStream_t stream);

// Device status word of the current device (bounded waits record timeouts
// here) and the wait limit in nanoseconds.
int *device_status_word();
uint64_t wait_limit_ns();
// One CTA whose bounded wait on an mbarrier that nothing completes runs out.
cudaError_t launch_selftest_wait(int *status, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_decode(const void *q, const void *kc, const void *vc, const int32_t *seqlens, void *out,
                          int out_f32, int in_f32, int krot, int layout, const Problem &p,
                          const WindowParams &wp, float *workspace, cudaStream_t s,
                          const PagedKV *paged = nullptr);

// Driver entry point for cuTensorMapEncodeTiled (resolved once, no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace atf
