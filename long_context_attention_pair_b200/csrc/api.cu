// C ABI of libatflash.so (declared in include/atflash.h): argument checks,
// the fp64 window table, workspace carving and the kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace atf {

// Device status word: kernels whose bounded wait ran out record it here.
__device__ int g_device_status;

static std::mutex g_mu;
static int *g_status_ptr[64];
static cudaMemPool_t g_pool[64];

int *device_status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    return g_status_ptr[dev];
}

// Stream-ordered pool for the scratch of atflash_prefill (kept cached: no
// release back to the driver between calls).
static cudaMemPool_t scratch_pool() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_pool[dev]) {
        cudaMemPoolProps props;
        memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
        uint64_t keep = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        g_pool[dev] = pool;
    }
    return g_pool[dev];
}

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Limit of every pipeline wait in the kernels: ATFLASH_WAIT_LIMIT_MS at first
// use (default 2000 ms), changed by atflash_set_wait_limit_ms.
static std::atomic<uint64_t> g_wait_limit_ns{0};

uint64_t wait_limit_ns() {
    uint64_t v = g_wait_limit_ns.load();
    if (v) return v;
    const char *e = getenv("ATFLASH_WAIT_LIMIT_MS");
    double ms = e ? atof(e) : 2000.0;
    if (!(ms > 0)) ms = 2000.0;
    uint64_t want = (uint64_t)(ms * 1e6);
    if (want == 0) want = 1;
    uint64_t expected = 0;
    g_wait_limit_ns.compare_exchange_strong(expected, want);
    return g_wait_limit_ns.load();
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_window_args(int D, double base, double k) {
    if (D < 2 || D > 2 * kMaxPairs || (D & 1) || !(base > 1.0) || isnan(k) || k < 0.0)
        return ATFLASH_ERR_INVALID_ARG;
    return ATFLASH_OK;
}

static int check_shape(int B, int Hq, int Hkv, int64_t N) {
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0 || N > INT32_MAX) return ATFLASH_ERR_INVALID_ARG;
    if ((int64_t)B * Hq > 65535 || (int64_t)B * Hkv * 8 > INT32_MAX) return ATFLASH_ERR_INVALID_ARG;
    return ATFLASH_OK;
}

static int check_theta_args(int D, const double *theta, double k) {
    if (!theta_valid(D, theta) || isnan(k) || k < 0.0) return ATFLASH_ERR_INVALID_ARG;
    return ATFLASH_OK;
}

static int fill_window_theta(WindowParams &wp, int D, const double *theta, double k, int64_t N) {
    int64_t w[kMaxPairs];
    int rc = window_table_theta(D, theta, k, N, w);
    if (rc != ATFLASH_OK) return rc;
    memset(&wp, 0, sizeof(wp));
    wp.H = D / 2;
    for (int r = 0; r < D / 2; ++r) {
        wp.w[r] = (int32_t)w[r];  // <= N-1 <= INT32_MAX
        wp.theta[r] = theta[r];
    }
    return ATFLASH_OK;
}

static size_t prefill_ws(int B, int Hq, int Hkv, int64_t N, int D, int in_dtype) {
    const size_t es = (in_dtype == ATFLASH_F32) ? 4 : 2;
    return align256((size_t)B * Hq * N * D * es) + align256((size_t)B * Hkv * N * D * es);
}

// theta_r = base^(-2r/D) after the same checks as the base-taking calls.
int theta_from_base(int D, double base, double *theta) {
    const int rc = check_window_args(D, base, 0.0);
    if (rc == ATFLASH_OK) theta_table(D, base, theta);
    return rc;
}

// atflash_decode's argument checks; on success the scratch it needs (need) is
// known but not yet checked.  Shared by atflash_decode and the entry point that
// allocates nothing, so that both reject the same arguments the same way.
int decode_check(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out, int B,
                 int Hq, int Hkv, int64_t Nmax, int D, const double *theta, double k_window, int kcache_rotated,
                 int kv_layout, int in_dtype, int out_dtype, size_t *need) {
    if (!q || !kcache || !vcache || !seqlens || !out) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, Nmax);
    if (rc != ATFLASH_OK) return rc;
    if ((rc = check_theta_args(D, theta, k_window)) != ATFLASH_OK) return rc;
    if (kcache_rotated != 0 && kcache_rotated != 1) return ATFLASH_ERR_INVALID_ARG;
    if (kv_layout != ATFLASH_KV_HND && kv_layout != ATFLASH_KV_NHD && kv_layout != ATFLASH_KV_PACKED)
        return ATFLASH_ERR_INVALID_ARG;
    if (kv_layout == ATFLASH_KV_PACKED && !kcache_rotated) return ATFLASH_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATFLASH_ERR_UNSUPPORTED;
    if ((in_dtype != ATFLASH_F32 && in_dtype != ATFLASH_BF16) ||
        (out_dtype != ATFLASH_F32 && out_dtype != ATFLASH_BF16))
        return ATFLASH_ERR_UNSUPPORTED;
    if (Hq / Hkv > 16) return ATFLASH_ERR_UNSUPPORTED;
    if (kv_layout == ATFLASH_KV_PACKED && in_dtype != ATFLASH_BF16) return ATFLASH_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out))
        return ATFLASH_ERR_ALIGNMENT;
    *need = decode_workspace_bytes(B, Hq, Hkv, Nmax, D);
    return ATFLASH_OK;
}

// The decode after decode_check, into a workspace of at least its `need` bytes.
int decode_run(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out, int B,
               int Hq, int Hkv, int64_t Nmax, int D, const double *theta, double k_window, int kcache_rotated,
               int kv_layout, int in_dtype, int out_dtype, float *workspace, cudaStream_t stream) {
    WindowParams wp;
    int rc = fill_window_theta(wp, D, theta, k_window, Nmax);
    if (rc != ATFLASH_OK) return rc;
    Problem p{B, Hq, Hkv, D, Nmax};
    cudaError_t e = launch_decode(q, kcache, vcache, seqlens, out, out_dtype == ATFLASH_F32,
                                  in_dtype == ATFLASH_F32, kcache_rotated, kv_layout, p, wp, workspace, stream);
    return e == cudaSuccess ? ATFLASH_OK : ATFLASH_ERR_CUDA;
}

static int decode_impl(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out,
                       int B, int Hq, int Hkv, int64_t Nmax, int D, const double *theta, double k_window,
                       int kcache_rotated, int kv_layout, int in_dtype, int out_dtype, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
    size_t need = 0;
    int rc = decode_check(q, kcache, vcache, seqlens, out, B, Hq, Hkv, Nmax, D, theta, k_window, kcache_rotated,
                          kv_layout, in_dtype, out_dtype, &need);
    if (rc != ATFLASH_OK) return rc;
    if (!workspace || workspace_bytes < need) return ATFLASH_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return ATFLASH_ERR_ALIGNMENT;
    return decode_run(q, kcache, vcache, seqlens, out, B, Hq, Hkv, Nmax, D, theta, k_window, kcache_rotated,
                      kv_layout, in_dtype, out_dtype, static_cast<float *>(workspace), stream);
}

}  // namespace atf

using namespace atf;

extern "C" {

const char *atflash_status_string(int status) {
    switch (status) {
        case ATFLASH_OK: return "ok";
        case ATFLASH_ERR_INVALID_ARG: return "invalid argument";
        case ATFLASH_ERR_UNSUPPORTED: return "unsupported head dim or dtype";
        case ATFLASH_ERR_WORKSPACE: return "workspace missing or too small";
        case ATFLASH_ERR_CUDA: return "CUDA runtime or launch error";
        case ATFLASH_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
        case ATFLASH_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case ATFLASH_ERR_BAD_PAGE: return "a paged decode met a page index outside its block table or pool";
        default: return "unknown status";
    }
}

int atflash_version(void) { return 100; }

int atflash_window_table(int D, double rope_base, double k_window, int64_t N, int64_t *w_out) {
    if (!w_out) return ATFLASH_ERR_INVALID_ARG;
    return window_table(D, rope_base, k_window, N, w_out);
}

int atflash_pruned_terms(int64_t N, int D, double rope_base, double k_window, atflash_terms *out) {
    return pruned_terms(N, D, rope_base, k_window, out);
}

int atflash_theta_table(int D, double rope_base, double *theta_out) {
    if (!theta_out) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_window_args(D, rope_base, 0.0);
    if (rc != ATFLASH_OK) return rc;
    theta_table(D, rope_base, theta_out);
    return ATFLASH_OK;
}

int atflash_window_table_theta(int D, const double *theta, double k_window, int64_t N, int64_t *w_out) {
    if (!w_out) return ATFLASH_ERR_INVALID_ARG;
    return window_table_theta(D, theta, k_window, N, w_out);
}

int atflash_pruned_terms_theta(int64_t N, int D, const double *theta, double k_window, atflash_terms *out) {
    return pruned_terms_theta(N, D, theta, k_window, out);
}

size_t atflash_prefill_workspace_bytes(int B, int Hq, int Hkv, int64_t N, int D, int in_dtype) {
    if (check_shape(B, Hq, Hkv, N) != ATFLASH_OK || D < 2 || D > 2 * kMaxPairs || (D & 1)) return 0;
    if (in_dtype != ATFLASH_F32 && in_dtype != ATFLASH_BF16) return 0;
    return prefill_ws(B, Hq, Hkv, N, D, in_dtype);
}

static int check_prefill_common(int B, int Hq, int Hkv, int64_t N, int D, const double *theta, double k,
                                int in_dtype, int out_dtype) {
    int rc = check_shape(B, Hq, Hkv, N);
    if (rc != ATFLASH_OK) return rc;
    if ((rc = check_theta_args(D, theta, k)) != ATFLASH_OK) return rc;
    if ((in_dtype != ATFLASH_F32 && in_dtype != ATFLASH_BF16) ||
        (out_dtype != ATFLASH_F32 && out_dtype != ATFLASH_BF16))
        return ATFLASH_ERR_UNSUPPORTED;
    if (in_dtype == ATFLASH_BF16 && D != 64 && D != 128) return ATFLASH_ERR_UNSUPPORTED;
    return ATFLASH_OK;
}

static int run_prefill_packed(const void *qt, const void *kt, const void *v, void *out, int B, int Hq, int Hkv,
                              int64_t N, int D, const double *theta, double k, int in_dtype, int out_dtype,
                              float *lse, cudaStream_t stream, const uint8_t *block_mask = nullptr) {
    WindowParams wp;
    int rc = fill_window_theta(wp, D, theta, k, N);
    if (rc != ATFLASH_OK) return rc;
    Problem p{B, Hq, Hkv, D, N};
    const int out_f32 = (out_dtype == ATFLASH_F32);
    cudaError_t e;
    if (in_dtype == ATFLASH_BF16) {
        int *status = device_status_word();
        if (!status) return ATFLASH_ERR_CUDA;
        e = launch_prefill_tc(qt, kt, v, out, out_f32, lse, p, wp, status, wait_limit_ns(), stream, nullptr, 0,
                              block_mask);
    } else {
        e = launch_prefill_simt_f32((const float *)qt, (const float *)kt, (const float *)v, out, out_f32, lse, p,
                                    wp, stream);
    }
    return e == cudaSuccess ? ATFLASH_OK : ATFLASH_ERR_CUDA;
}

static int run_rope_pack(const void *x, void *y, int B, int64_t N, int H, int D, const double *theta,
                         int in_dtype, cudaStream_t stream) {
    WindowParams wp;
    memset(&wp, 0, sizeof(wp));
    wp.H = D / 2;
    for (int r = 0; r < D / 2; ++r) wp.theta[r] = theta[r];
    cudaError_t e = (in_dtype == ATFLASH_BF16) ? launch_rope_pack_bf16(x, y, B, N, H, D, wp, stream)
                                               : launch_rope_pack_f32(x, y, B, N, H, D, wp, stream);
    return e == cudaSuccess ? ATFLASH_OK : ATFLASH_ERR_CUDA;
}

// The rows that see at most 128 keys, recomputed in fp32 from the caller's
// un-rotated bf16 inputs after the tensor-core prefill (see short_rows.cu).
static int run_short_rows(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv, int64_t N,
                          int D, const double *theta, double k_window, int out_dtype, float *lse,
                          cudaStream_t stream, const int32_t *cu_seqlens = nullptr, int64_t total = 0,
                          const uint8_t *block_mask = nullptr) {
    WindowParams wp;
    int rc = fill_window_theta(wp, D, theta, k_window, N);
    if (rc != ATFLASH_OK) return rc;
    int *status = device_status_word();
    if (!status) return ATFLASH_ERR_CUDA;
    Problem p{B, Hq, Hkv, D, N};
    cudaError_t e = launch_short_rows_prefill(q, k, v, out, out_dtype == ATFLASH_F32, lse, p, wp, status, stream,
                                              cu_seqlens, total, block_mask);
    return e == cudaSuccess ? ATFLASH_OK : ATFLASH_ERR_CUDA;
}

size_t atflash_rope_pack_bytes(int B, int64_t N, int H, int D, int in_dtype) {
    if (check_shape(B, H, H, N) != ATFLASH_OK || D < 2 || D > 2 * kMaxPairs || (D & 1)) return 0;
    if (in_dtype == ATFLASH_BF16) return (D == 64 || D == 128) ? (size_t)B * H * N * D * 2 : 0;
    if (in_dtype == ATFLASH_F32) return (size_t)B * H * N * D * 4;
    return 0;
}

static int rope_pack_impl(const void *x, void *y, int B, int64_t N, int H, int D, const double *theta,
                          int in_dtype, cudaStream_t stream) {
    if (!x || !y) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_shape(B, H, H, N);
    if (rc != ATFLASH_OK) return rc;
    if ((rc = check_theta_args(D, theta, 0.0)) != ATFLASH_OK) return rc;
    if (in_dtype != ATFLASH_F32 && in_dtype != ATFLASH_BF16) return ATFLASH_ERR_UNSUPPORTED;
    if (in_dtype == ATFLASH_BF16 && D != 64 && D != 128) return ATFLASH_ERR_UNSUPPORTED;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(y) & 255u)) return ATFLASH_ERR_ALIGNMENT;
    return run_rope_pack(x, y, B, N, H, D, theta, in_dtype, stream);
}

// theta_r = base^(-2r/D) for the calls that take a RoPE base (validated first).
struct BaseTheta {
    double theta[kMaxPairs];
    int rc;
    BaseTheta(int D, double base) : rc(check_window_args(D, base, 0.0)) {
        if (rc == ATFLASH_OK) theta_table(D, base, theta);
    }
};

int atflash_rope_pack(const void *x, void *y, int B, int64_t N, int H, int D, double rope_base, int in_dtype,
                      cudaStream_t stream) {
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return rope_pack_impl(x, y, B, N, H, D, bt.theta, in_dtype, stream);
}

int atflash_rope_pack_theta(const void *x, void *y, int B, int64_t N, int H, int D, const double *theta,
                            int in_dtype, cudaStream_t stream) {
    return rope_pack_impl(x, y, B, N, H, D, theta, in_dtype, stream);
}

static int prefill_packed_impl(const void *qpack, const void *kpack, const void *v, void *out, int B, int Hq,
                               int Hkv, int64_t N, int D, const double *theta, double k_window, int in_dtype,
                               int out_dtype, float *lse, cudaStream_t stream) {
    int rc = check_prefill_common(B, Hq, Hkv, N, D, theta, k_window, in_dtype, out_dtype);
    if (rc != ATFLASH_OK) return rc;
    if ((reinterpret_cast<uintptr_t>(qpack) & 255u) || (reinterpret_cast<uintptr_t>(kpack) & 255u) ||
        !aligned16(v) || !aligned16(out))
        return ATFLASH_ERR_ALIGNMENT;
    return run_prefill_packed(qpack, kpack, v, out, B, Hq, Hkv, N, D, theta, k_window, in_dtype, out_dtype, lse,
                              stream);
}

int atflash_prefill_packed(const void *qpack, const void *kpack, const void *v, void *out, int B, int Hq,
                           int Hkv, int64_t N, int D, double rope_base, double k_window, int in_dtype,
                           int out_dtype, float *lse, cudaStream_t stream) {
    if (!qpack || !kpack || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return prefill_packed_impl(qpack, kpack, v, out, B, Hq, Hkv, N, D, bt.theta, k_window, in_dtype, out_dtype,
                               lse, stream);
}

int atflash_prefill_packed_theta(const void *qpack, const void *kpack, const void *v, void *out, int B, int Hq,
                                 int Hkv, int64_t N, int D, const double *theta, double k_window, int in_dtype,
                                 int out_dtype, float *lse, cudaStream_t stream) {
    if (!qpack || !kpack || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    return prefill_packed_impl(qpack, kpack, v, out, B, Hq, Hkv, N, D, theta, k_window, in_dtype, out_dtype, lse,
                               stream);
}

static int prefill_ex_impl(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                           int64_t N, int D, const double *theta, double k_window, int in_dtype, int out_dtype,
                           float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !k || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_prefill_common(B, Hq, Hkv, N, D, theta, k_window, in_dtype, out_dtype);
    if (rc != ATFLASH_OK) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATFLASH_ERR_ALIGNMENT;
    const size_t need = prefill_ws(B, Hq, Hkv, N, D, in_dtype);
    if (!workspace || workspace_bytes < need) return ATFLASH_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATFLASH_ERR_ALIGNMENT;
    const size_t es = (in_dtype == ATFLASH_F32) ? 4 : 2;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *qt = ws;
    void *kt = ws + align256((size_t)B * Hq * N * D * es);
    if ((rc = run_rope_pack(q, qt, B, N, Hq, D, theta, in_dtype, stream)) != ATFLASH_OK) return rc;
    if ((rc = run_rope_pack(k, kt, B, N, Hkv, D, theta, in_dtype, stream)) != ATFLASH_OK) return rc;
    rc = run_prefill_packed(qt, kt, v, out, B, Hq, Hkv, N, D, theta, k_window, in_dtype, out_dtype, lse, stream);
    if (rc != ATFLASH_OK || in_dtype != ATFLASH_BF16) return rc;
    return run_short_rows(q, k, v, out, B, Hq, Hkv, N, D, theta, k_window, out_dtype, lse, stream);
}

static int prefill_sparse_impl(const void *q, const void *k, const void *v, const uint8_t *block_mask, void *out,
                               int B, int Hq, int Hkv, int64_t N, int D, const double *theta, double k_window,
                               int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
    int rc = check_prefill_common(B, Hq, Hkv, N, D, theta, k_window, ATFLASH_BF16, out_dtype);
    if (rc != ATFLASH_OK) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATFLASH_ERR_ALIGNMENT;
    const size_t need = prefill_ws(B, Hq, Hkv, N, D, ATFLASH_BF16);
    if (!workspace || workspace_bytes < need) return ATFLASH_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATFLASH_ERR_ALIGNMENT;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *qt = ws;
    void *kt = ws + align256((size_t)B * Hq * N * D * 2);
    if ((rc = run_rope_pack(q, qt, B, N, Hq, D, theta, ATFLASH_BF16, stream)) != ATFLASH_OK) return rc;
    if ((rc = run_rope_pack(k, kt, B, N, Hkv, D, theta, ATFLASH_BF16, stream)) != ATFLASH_OK) return rc;
    rc = run_prefill_packed(qt, kt, v, out, B, Hq, Hkv, N, D, theta, k_window, ATFLASH_BF16, out_dtype, lse, stream,
                            block_mask);
    if (rc != ATFLASH_OK) return rc;
    return run_short_rows(q, k, v, out, B, Hq, Hkv, N, D, theta, k_window, out_dtype, lse, stream, nullptr, 0,
                          block_mask);
}

int atflash_prefill_sparse(const void *q, const void *k, const void *v, const uint8_t *block_mask, void *out,
                           int B, int Hq, int Hkv, int64_t N, int D, double rope_base, double k_window,
                           int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    if (!q || !k || !v || !out || !block_mask) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return prefill_sparse_impl(q, k, v, block_mask, out, B, Hq, Hkv, N, D, bt.theta, k_window, out_dtype, lse,
                               workspace, workspace_bytes, stream);
}

int atflash_prefill_sparse_theta(const void *q, const void *k, const void *v, const uint8_t *block_mask,
                                 void *out, int B, int Hq, int Hkv, int64_t N, int D, const double *theta,
                                 double k_window, int out_dtype, float *lse, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !k || !v || !out || !block_mask) return ATFLASH_ERR_INVALID_ARG;
    return prefill_sparse_impl(q, k, v, block_mask, out, B, Hq, Hkv, N, D, theta, k_window, out_dtype, lse,
                               workspace, workspace_bytes, stream);
}

static int short_rows_impl(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                           int64_t N, int D, const double *theta, double k_window, int out_dtype, float *lse,
                           cudaStream_t stream) {
    if (!q || !k || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_prefill_common(B, Hq, Hkv, N, D, theta, k_window, ATFLASH_BF16, out_dtype);
    if (rc != ATFLASH_OK) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATFLASH_ERR_ALIGNMENT;
    return run_short_rows(q, k, v, out, B, Hq, Hkv, N, D, theta, k_window, out_dtype, lse, stream);
}

int atflash_prefill_short_rows(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                               int64_t N, int D, double rope_base, double k_window, int out_dtype, float *lse,
                               cudaStream_t stream) {
    if (!q || !k || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return short_rows_impl(q, k, v, out, B, Hq, Hkv, N, D, bt.theta, k_window, out_dtype, lse, stream);
}

int atflash_prefill_short_rows_theta(const void *q, const void *k, const void *v, void *out, int B, int Hq,
                                     int Hkv, int64_t N, int D, const double *theta, double k_window, int out_dtype,
                                     float *lse, cudaStream_t stream) {
    return short_rows_impl(q, k, v, out, B, Hq, Hkv, N, D, theta, k_window, out_dtype, lse, stream);
}

int atflash_prefill_ex(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                       int64_t N, int D, double rope_base, double k_window, int in_dtype, int out_dtype,
                       float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !k || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return prefill_ex_impl(q, k, v, out, B, Hq, Hkv, N, D, bt.theta, k_window, in_dtype, out_dtype, lse, workspace,
                           workspace_bytes, stream);
}

int atflash_prefill_theta(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                          int64_t N, int D, const double *theta, double k_window, int in_dtype, int out_dtype,
                          float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    return prefill_ex_impl(q, k, v, out, B, Hq, Hkv, N, D, theta, k_window, in_dtype, out_dtype, lse, workspace,
                           workspace_bytes, stream);
}

int atflash_prefill(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv, int64_t N,
                    int D, double rope_base, double k_window, cudaStream_t stream) {
    if (!q || !k || !v || !out) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, N);
    if (rc != ATFLASH_OK) return rc;
    if ((rc = check_window_args(D, rope_base, k_window)) != ATFLASH_OK) return rc;
    if (D != 64 && D != 128) return ATFLASH_ERR_UNSUPPORTED;
    const size_t need = prefill_ws(B, Hq, Hkv, N, D, ATFLASH_BF16);
    cudaMemPool_t pool = scratch_pool();
    if (!pool) return ATFLASH_ERR_CUDA;
    void *ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, need, pool, stream) != cudaSuccess) return ATFLASH_ERR_CUDA;
    rc = atflash_prefill_ex(q, k, v, out, B, Hq, Hkv, N, D, rope_base, k_window, ATFLASH_BF16, ATFLASH_BF16,
                            nullptr, ws, need, stream);
    cudaFreeAsync(ws, stream);
    return rc;
}

static int check_varlen(int B, int Hq, int Hkv, int64_t max_seqlen, int64_t total, int D, const double *theta,
                        double k, int out_dtype) {
    int rc = check_shape(B, Hq, Hkv, max_seqlen);
    if (rc != ATFLASH_OK) return rc;
    if (total < 1 || total > INT32_MAX || max_seqlen > total) return ATFLASH_ERR_INVALID_ARG;
    if ((rc = check_theta_args(D, theta, k)) != ATFLASH_OK) return rc;
    if (D != 64 && D != 128) return ATFLASH_ERR_UNSUPPORTED;
    if (out_dtype != ATFLASH_F32 && out_dtype != ATFLASH_BF16) return ATFLASH_ERR_UNSUPPORTED;
    return ATFLASH_OK;
}

size_t atflash_prefill_varlen_workspace_bytes(int Hq, int Hkv, int64_t total, int D) {
    if (Hq < 1 || Hkv < 1 || total < 1 || total > INT32_MAX || (D != 64 && D != 128)) return 0;
    return align256((size_t)Hq * total * D * 2) + align256((size_t)Hkv * total * D * 2);
}

static int prefill_varlen_impl(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens,
                               int B, int64_t max_seqlen, int64_t total, int Hq, int Hkv, int D, const double *theta,
                               double k_window, int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
    if (!q || !k || !v || !out || !cu_seqlens) return ATFLASH_ERR_INVALID_ARG;
    int rc = check_varlen(B, Hq, Hkv, max_seqlen, total, D, theta, k_window, out_dtype);
    if (rc != ATFLASH_OK) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATFLASH_ERR_ALIGNMENT;
    const size_t need = atflash_prefill_varlen_workspace_bytes(Hq, Hkv, total, D);
    void *owned = nullptr;
    if (!workspace) {  // no caller workspace: take it from the library's stream-ordered pool
        cudaMemPool_t pool = scratch_pool();
        if (!pool) return ATFLASH_ERR_CUDA;
        if (cudaMallocFromPoolAsync(&owned, need, pool, stream) != cudaSuccess) return ATFLASH_ERR_CUDA;
        workspace = owned;
    } else if (workspace_bytes < need) {
        return ATFLASH_ERR_WORKSPACE;
    } else if (reinterpret_cast<uintptr_t>(workspace) & 255u) {
        return ATFLASH_ERR_ALIGNMENT;
    }
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *qt = ws;
    void *kt = ws + align256((size_t)Hq * total * D * 2);
    WindowParams wp;
    rc = fill_window_theta(wp, D, theta, k_window, max_seqlen);
    cudaError_t e = cudaSuccess;
    int *status = device_status_word();
    if (rc == ATFLASH_OK && !status) rc = ATFLASH_ERR_CUDA;
    if (rc == ATFLASH_OK) {
        e = launch_rope_pack_bf16(q, qt, 1, total, Hq, D, wp, stream, cu_seqlens, B);
        if (e == cudaSuccess) e = launch_rope_pack_bf16(k, kt, 1, total, Hkv, D, wp, stream, cu_seqlens, B);
        Problem p{B, Hq, Hkv, D, max_seqlen};
        if (e == cudaSuccess)
            e = launch_prefill_tc(qt, kt, v, out, out_dtype == ATFLASH_F32, lse, p, wp, status, wait_limit_ns(),
                                  stream, cu_seqlens, total);
        if (e == cudaSuccess)
            e = launch_short_rows_prefill(q, k, v, out, out_dtype == ATFLASH_F32, lse, p, wp, status, stream,
                                          cu_seqlens, total);
        if (e != cudaSuccess) rc = ATFLASH_ERR_CUDA;
    }
    if (owned) cudaFreeAsync(owned, stream);
    return rc;
}

int atflash_prefill_varlen(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens, int B,
                           int64_t max_seqlen, int64_t total, int Hq, int Hkv, int D, double rope_base,
                           double k_window, int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    if (!q || !k || !v || !out || !cu_seqlens) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return prefill_varlen_impl(q, k, v, out, cu_seqlens, B, max_seqlen, total, Hq, Hkv, D, bt.theta, k_window,
                               out_dtype, lse, workspace, workspace_bytes, stream);
}

int atflash_prefill_varlen_theta(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens,
                                 int B, int64_t max_seqlen, int64_t total, int Hq, int Hkv, int D,
                                 const double *theta, double k_window, int out_dtype, float *lse, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
    return prefill_varlen_impl(q, k, v, out, cu_seqlens, B, max_seqlen, total, Hq, Hkv, D, theta, k_window,
                               out_dtype, lse, workspace, workspace_bytes, stream);
}

size_t atflash_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int D) {
    if (check_shape(B, Hq, Hkv, Nmax) != ATFLASH_OK || (D != 64 && D != 128)) return 0;
    return decode_workspace_bytes(B, Hq, Hkv, Nmax, D);
}

static int decode_paged_impl(const void *q, const void *kpages, const void *vpages, const int32_t *block_table,
                             const int32_t *seqlens, void *out, int B, int Hq, int Hkv, int max_pages, int num_pages,
                             int page_size, int D, const double *theta, double k_window, int kcache_rotated,
                             int kv_layout, int out_dtype, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    if (!q || !kpages || !vpages || !block_table || !seqlens || !out) return ATFLASH_ERR_INVALID_ARG;
    if (max_pages < 1 || num_pages < 1 || page_size < 64 || page_size % 64 != 0) return ATFLASH_ERR_INVALID_ARG;
    const int64_t Nmax = (int64_t)max_pages * page_size;
    int rc = check_shape(B, Hq, Hkv, Nmax);
    if (rc != ATFLASH_OK) return rc;
    if ((int64_t)num_pages * Hkv * (D / 16) > INT32_MAX) return ATFLASH_ERR_INVALID_ARG;
    if ((rc = check_theta_args(D, theta, k_window)) != ATFLASH_OK) return rc;
    if (kcache_rotated != 0 && kcache_rotated != 1) return ATFLASH_ERR_INVALID_ARG;
    if (kv_layout != ATFLASH_KV_NHD && kv_layout != ATFLASH_KV_PACKED) return ATFLASH_ERR_INVALID_ARG;
    if (kv_layout == ATFLASH_KV_PACKED && !kcache_rotated) return ATFLASH_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATFLASH_ERR_UNSUPPORTED;
    if (out_dtype != ATFLASH_F32 && out_dtype != ATFLASH_BF16) return ATFLASH_ERR_UNSUPPORTED;
    if (Hq / Hkv > 16) return ATFLASH_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(kpages) || !aligned16(vpages) || !aligned16(out)) return ATFLASH_ERR_ALIGNMENT;
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, Nmax, D);
    if (!workspace || workspace_bytes < need) return ATFLASH_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return ATFLASH_ERR_ALIGNMENT;
    WindowParams wp;
    if ((rc = fill_window_theta(wp, D, theta, k_window, Nmax)) != ATFLASH_OK) return rc;
    Problem p{B, Hq, Hkv, D, Nmax};
    PagedKV pk{block_table, max_pages, page_size, num_pages};
    cudaError_t e = launch_decode(q, kpages, vpages, seqlens, out, out_dtype == ATFLASH_F32, 0, kcache_rotated,
                                  kv_layout, p, wp, static_cast<float *>(workspace), stream, &pk);
    return e == cudaSuccess ? ATFLASH_OK : ATFLASH_ERR_CUDA;
}

int atflash_decode_paged(const void *q, const void *kpages, const void *vpages, const int32_t *block_table,
                         const int32_t *seqlens, void *out, int B, int Hq, int Hkv, int max_pages, int num_pages,
                         int page_size, int D, double rope_base, double k_window, int kcache_rotated, int kv_layout,
                         int out_dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !kpages || !vpages || !block_table || !seqlens || !out) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return decode_paged_impl(q, kpages, vpages, block_table, seqlens, out, B, Hq, Hkv, max_pages, num_pages,
                             page_size, D, bt.theta, k_window, kcache_rotated, kv_layout, out_dtype, workspace,
                             workspace_bytes, stream);
}

int atflash_decode_paged_theta(const void *q, const void *kpages, const void *vpages, const int32_t *block_table,
                               const int32_t *seqlens, void *out, int B, int Hq, int Hkv, int max_pages,
                               int num_pages, int page_size, int D, const double *theta, double k_window,
                               int kcache_rotated, int kv_layout, int out_dtype, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream) {
    return decode_paged_impl(q, kpages, vpages, block_table, seqlens, out, B, Hq, Hkv, max_pages, num_pages,
                             page_size, D, theta, k_window, kcache_rotated, kv_layout, out_dtype, workspace,
                             workspace_bytes, stream);
}

int atflash_decode(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out,
                   int B, int Hq, int Hkv, int64_t Nmax, int D, double rope_base, double k_window,
                   int kcache_rotated, int kv_layout, int in_dtype, int out_dtype, void *workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !kcache || !vcache || !seqlens || !out) return ATFLASH_ERR_INVALID_ARG;
    BaseTheta bt(D, rope_base);
    if (bt.rc != ATFLASH_OK) return bt.rc;
    return decode_impl(q, kcache, vcache, seqlens, out, B, Hq, Hkv, Nmax, D, bt.theta, k_window, kcache_rotated,
                       kv_layout, in_dtype, out_dtype, workspace, workspace_bytes, stream);
}

int atflash_decode_theta(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *out,
                         int B, int Hq, int Hkv, int64_t Nmax, int D, const double *theta, double k_window,
                         int kcache_rotated, int kv_layout, int in_dtype, int out_dtype, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
    return decode_impl(q, kcache, vcache, seqlens, out, B, Hq, Hkv, Nmax, D, theta, k_window, kcache_rotated,
                       kv_layout, in_dtype, out_dtype, workspace, workspace_bytes, stream);
}

int atflash_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return ATFLASH_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return ATFLASH_ERR_CUDA;
    if (clear) {
        int z = 0;
        if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(int)) != cudaSuccess) return ATFLASH_ERR_CUDA;
    }
    if (v >= ATFLASH_DEVICE_BAD_PAGE) return ATFLASH_ERR_BAD_PAGE;
    return v >= ATFLASH_DEVICE_TIMEOUT_BASE ? ATFLASH_ERR_TIMEOUT : ATFLASH_OK;
}

int atflash_set_wait_limit_ms(double ms) {
    if (!(ms > 0.0) || ms > 60000.0) return ATFLASH_ERR_INVALID_ARG;
    uint64_t v = (uint64_t)(ms * 1e6);
    if (v == 0) v = 1;
    g_wait_limit_ns.store(v);
    return ATFLASH_OK;
}

int atflash_selftest_wait_timeout(double limit_ms, cudaStream_t stream) {
    if (!(limit_ms > 0.0) || limit_ms > 10000.0) return ATFLASH_ERR_INVALID_ARG;
    int *status = device_status_word();
    if (!status) return ATFLASH_ERR_CUDA;
    uint64_t v = (uint64_t)(limit_ms * 1e6);
    if (v == 0) v = 1;
    return launch_selftest_wait(status, v, stream) == cudaSuccess ? ATFLASH_OK : ATFLASH_ERR_CUDA;
}

}  // extern "C"
