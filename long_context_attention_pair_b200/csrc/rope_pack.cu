// RoPE pre-pass of the prefill: every query and key vector is rotated exactly
// once (rotate-half RoPE, "The idea": each frequency pair (r, r+D/2) is
// rotated by position * theta_r) and written in the layout the attention
// kernels read.
//
// Angles are reduced modulo 2*pi in fp64 (position * theta_r reaches 1e6 rad
// at 1M tokens, far beyond fp32) and only the reduced angle goes to sincosf.
//
// bf16 layout ("packed"): [b*H + h][c][n][16] with c = 0..D/16-1; element 2j
// of chunk c is x~_{8c+j}, element 2j+1 is x~_{8c+j+D/2}.  A chunk therefore
// holds 8 complete frequency pairs in 32 contiguous bytes per token, which is
// one K-step (16 bf16) of the tensor-core contraction; permuting the
// contraction axis the same way for Q and K leaves every dot product intact.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace atf {

constexpr int kRopePos = 32;  // positions per block

__device__ __forceinline__ float2 rope_cos_sin(int64_t n, double theta) {
    double turns = (double)n * theta * 0.15915494309189533576888376337251;  // 1/(2*pi)
    turns -= rint(turns);
    float a = (float)(turns * 6.283185307179586476925286766559);
    float s, c;
    sincosf(a, &s, &c);
    return make_float2(c, s);
}

// Position of token n of a batch packed along the token axis: n minus the start
// of its sequence (cu[s] <= n < cu[s+1]); the token's own index without cu.
__device__ __forceinline__ int64_t token_position(int64_t n, const int32_t *cu, int nseq) {
    if (!cu) return n;
    int lo = 0, hi = nseq;  // largest s with cu[s] <= n
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)cu[mid] <= n) lo = mid; else hi = mid;
    }
    return n - (int64_t)cu[lo];
}

template <int D>
__global__ void __launch_bounds__(256) rope_pack_bf16_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             __nv_bfloat16 *__restrict__ y, int64_t N, int Hx,
                                                             const __grid_constant__ WindowParams wp,
                                                             const int32_t *__restrict__ cu, int nseq) {
    constexpr int H = D / 2;
    constexpr int C = D / 16;
    __shared__ float2 cs[H][kRopePos];
    __shared__ int64_t pos[kRopePos];
    const int b = blockIdx.y;
    const int64_t n0 = (int64_t)blockIdx.x * kRopePos;
    if (threadIdx.x < kRopePos) pos[threadIdx.x] = token_position(n0 + threadIdx.x, cu, nseq);
    __syncthreads();
    for (int e = threadIdx.x; e < H * kRopePos; e += blockDim.x) {
        int r = e / kRopePos, p = e % kRopePos;
        cs[r][p] = (n0 + p < N) ? rope_cos_sin(pos[p], wp.theta[r]) : make_float2(1.f, 0.f);
    }
    __syncthreads();
    const int p = threadIdx.x & 31;
    const int64_t n = n0 + p;
    if (n >= N) return;
    for (int item = threadIdx.x >> 5; item < Hx * C; item += blockDim.x >> 5) {
        const int h = item / C, c = item % C;
        const __nv_bfloat16 *src = x + ((size_t)((int64_t)b * N + n) * Hx + h) * D;
        uint4 lo = *reinterpret_cast<const uint4 *>(src + 8 * c);
        uint4 hi = *reinterpret_cast<const uint4 *>(src + H + 8 * c);
        const uint32_t a[4] = {lo.x, lo.y, lo.z, lo.w};
        const uint32_t bb[4] = {hi.x, hi.y, hi.z, hi.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float xa = (j & 1) ? bf16hi(a[j >> 1]) : bf16lo(a[j >> 1]);
            float xb = (j & 1) ? bf16hi(bb[j >> 1]) : bf16lo(bb[j >> 1]);
            float2 t = cs[8 * c + j][p];
            o[j] = pack_bf16x2(xa * t.x - xb * t.y, xb * t.x + xa * t.y);
        }
        __nv_bfloat16 *dst = y + (((size_t)((int64_t)b * Hx + h) * C + c) * N + n) * 16;
        reinterpret_cast<uint4 *>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4 *>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// fp32 variant for the exact CUDA-core path: y[(b*H + h)*N + n][2r] = x~_r,
// [2r+1] = x~_{r+D/2}; any even D <= 256.
__global__ void __launch_bounds__(256) rope_pack_f32_kernel(const float *__restrict__ x, float *__restrict__ y,
                                                            int64_t N, int Hx, int D,
                                                            const __grid_constant__ WindowParams wp) {
    __shared__ float2 cs[kMaxPairs][kRopePos];
    const int H = D / 2;
    const int b = blockIdx.y;
    const int64_t n0 = (int64_t)blockIdx.x * kRopePos;
    for (int e = threadIdx.x; e < H * kRopePos; e += blockDim.x) {
        int r = e / kRopePos, p = e % kRopePos;
        cs[r][p] = (n0 + p < N) ? rope_cos_sin(n0 + p, wp.theta[r]) : make_float2(1.f, 0.f);
    }
    __syncthreads();
    const int p = threadIdx.x & 31;
    const int64_t n = n0 + p;
    if (n >= N) return;
    for (int item = threadIdx.x >> 5; item < Hx * H; item += blockDim.x >> 5) {
        const int h = item / H, r = item % H;
        const float *src = x + ((size_t)((int64_t)b * N + n) * Hx + h) * D;
        float xa = src[r], xb = src[r + H];
        float2 t = cs[r][p];
        float *dst = y + ((size_t)((int64_t)b * Hx + h) * N + n) * D + 2 * r;
        dst[0] = xa * t.x - xb * t.y;
        dst[1] = xb * t.x + xa * t.y;
    }
}

cudaError_t launch_rope_pack_bf16(const void *x, void *y, int B, int64_t N, int Hx, int D,
                                  const WindowParams &wp, cudaStream_t s, const int32_t *cu, int nseq) {
    dim3 grid((unsigned)((N + kRopePos - 1) / kRopePos), (unsigned)B);
    if (D == 128)
        rope_pack_bf16_kernel<128><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)x, (__nv_bfloat16 *)y, N, Hx, wp,
                                                        cu, nseq);
    else if (D == 64)
        rope_pack_bf16_kernel<64><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)x, (__nv_bfloat16 *)y, N, Hx, wp, cu,
                                                       nseq);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_rope_pack_f32(const void *x, void *y, int B, int64_t N, int Hx, int D,
                                 const WindowParams &wp, cudaStream_t s) {
    dim3 grid((unsigned)((N + kRopePos - 1) / kRopePos), (unsigned)B);
    rope_pack_f32_kernel<<<grid, 256, 0, s>>>((const float *)x, (float *)y, N, Hx, D, wp);
    return cudaGetLastError();
}

}  // namespace atf
