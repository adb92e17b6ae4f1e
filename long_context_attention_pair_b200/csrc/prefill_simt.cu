// Exact fp32 CUDA-core prefill (the fp32-input path).  Reads the fp32
// pair-interleaved Q~/K~ written by the RoPE pre-pass and the caller's fp32 V.
//
// Per cell (n, m <= n): the kept pairs at distance d = n - m are exactly the
// suffix r >= r*(d) = min{r : w_r >= d} because w_r is non-decreasing in r
// ("The idea": the window grows with the pair's wavelength), so the score is
// (1/sqrt(D)) * sum_{r >= r*(d)} t_r(n, m); an empty suffix scores 0.
// Online softmax in fp32 with expf.  One warp = 32 query rows; keys staged
// through shared memory 32 at a time.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace atf {

constexpr int kSimtRows = 32;

// r*(d): first pair whose window reaches distance d (H when none does).
__device__ __forceinline__ int first_kept_pair(const int *w, int H, int64_t d) {
    int lo = 0, hi = H;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)w[mid] >= d) hi = mid; else lo = mid + 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kSimtRows) prefill_simt_f32_kernel(
    const float *__restrict__ qt, const float *__restrict__ kt, const float *__restrict__ v, void *out, int out_f32,
    float *lse, int64_t N, int Hq, int Hkv, int D, const __grid_constant__ WindowParams wp) {
    extern __shared__ float sm[];
    const int H = D / 2;
    float *sq = sm;                    // [D][32]  rotated query rows (transposed)
    float *sacc = sq + D * kSimtRows;  // [D][32]  output accumulators
    float *sk = sacc + D * kSimtRows;  // [32][D]  rotated keys of the tile
    float *sv = sk + kSimtRows * D;    // [32][D]  values of the tile
    int *sw = reinterpret_cast<int *>(sv + kSimtRows * D);  // [H]
    const int bh = blockIdx.y;
    const int b = bh / Hq, hq = bh % Hq, g = hq / (Hq / Hkv);
    const int lane = threadIdx.x;
    const int64_t n0 = (int64_t)blockIdx.x * kSimtRows;
    const int64_t n = n0 + lane;
    for (int r = lane; r < H; r += kSimtRows) sw[r] = wp.w[r];
    for (int d = 0; d < D; ++d) {
        sq[d * kSimtRows + lane] = (n < N) ? qt[((size_t)bh * N + n) * D + d] : 0.f;
        sacc[d * kSimtRows + lane] = 0.f;
    }
    const float scale = rsqrtf((float)D);
    float mrun = -INFINITY, lrun = 0.f;
    const int64_t kend = (n0 + kSimtRows < N) ? n0 + kSimtRows : N;
    for (int64_t m0 = 0; m0 < kend; m0 += kSimtRows) {
        __syncthreads();
        const int64_t mk = m0 + lane;
        for (int d = 0; d < D; ++d) {
            sk[lane * D + d] = (mk < N) ? kt[((size_t)((int64_t)b * Hkv + g) * N + mk) * D + d] : 0.f;
            sv[lane * D + d] = (mk < N) ? v[((size_t)((int64_t)b * N + mk) * Hkv + g) * D + d] : 0.f;
        }
        __syncthreads();
        if (n < N) {
            for (int j = 0; j < kSimtRows; ++j) {
                const int64_t m = m0 + j;
                if (m > n) break;
                const int rs = first_kept_pair(sw, H, n - m);
                float s = 0.f;
                for (int r = rs; r < H; ++r)
                    s += sq[(2 * r) * kSimtRows + lane] * sk[j * D + 2 * r] +
                         sq[(2 * r + 1) * kSimtRows + lane] * sk[j * D + 2 * r + 1];
                s *= scale;
                const float mnew = fmaxf(mrun, s);
                const float alpha = expf(mrun - mnew);
                const float p = expf(s - mnew);
                lrun = lrun * alpha + p;
                for (int d = 0; d < D; ++d)
                    sacc[d * kSimtRows + lane] = sacc[d * kSimtRows + lane] * alpha + p * sv[j * D + d];
                mrun = mnew;
            }
        }
    }
    if (n >= N) return;
    const float inv = 1.f / lrun;
    const size_t o = ((size_t)((int64_t)b * N + n) * Hq + hq) * D;
    for (int d = 0; d < D; ++d) {
        float val = sacc[d * kSimtRows + lane] * inv;
        if (out_f32) reinterpret_cast<float *>(out)[o + d] = val;
        else reinterpret_cast<__nv_bfloat16 *>(out)[o + d] = __float2bfloat16_rn(val);
    }
    if (lse) lse[((size_t)b * Hq + hq) * N + n] = mrun + logf(lrun);
}

cudaError_t launch_prefill_simt_f32(const float *qt, const float *kt, const float *v, void *out, int out_f32,
                                    float *lse, const Problem &p, const WindowParams &wp, cudaStream_t s) {
    size_t smem = (size_t)4 * p.D * kSimtRows * sizeof(float) + kMaxPairs * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(prefill_simt_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((p.N + kSimtRows - 1) / kSimtRows), (unsigned)(p.B * p.Hq));
    prefill_simt_f32_kernel<<<grid, kSimtRows, smem, s>>>(qt, kt, v, out, out_f32, lse, p.N, p.Hq, p.Hkv, p.D,
                                                          wp);
    return cudaGetLastError();
}

}  // namespace atf
