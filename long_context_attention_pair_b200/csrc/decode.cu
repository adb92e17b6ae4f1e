// Split-KV windowed decode, CUDA-core version (fp32 caches; the bf16 path is
// the tensor-core kernel in decode_tc.cu): one query token per sequence over a
// contiguous cache ("Numbers"/"Using the ports": the window is a
// condition on which K elements are loaded).
//
// Kernel 1 (grid splits x Hkv x B): each CTA owns kSplitKeys consecutive cache
// rows of one (sequence, KV head) and all G = Hq/Hkv query heads that read it.
// For a key at distance d = L-1-m only the pairs r >= r*(d) are kept, so only
// those K elements are loaded; each kept pair is rotated at load (unless the
// cache already holds rotated keys) and dotted with the G rotated queries.
// Each warp keeps an online-softmax state per head; the CTA folds its four
// warps' states and writes one partial (max, sum, acc[D]) per head.
// Kernel 2 merges the partial states of all splits (log-sum-exp).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace atf {

constexpr int kDecodeWarps = 4;
constexpr int kMaxGroup = 16;  // query heads per KV head

// Keys per split: a multiple of 64 (one TMA stage of the tensor-core kernel)
// between 256 and 4096, chosen so that the (sequence, KV head, split) CTAs come
// close to, without passing, a whole number of waves of that kernel's 148 SMs x
// 3 resident CTAs: a last wave that is mostly empty streams at a fraction of
// the HBM bandwidth.
int decode_split_keys(int B, int Hkv, int64_t Nmax) {
    constexpr int64_t kSlots = 148 * 3, kUnit = 64, kMinUnits = 4, kMaxUnits = 64;
    const int64_t units = (Nmax + kUnit - 1) / kUnit;  // stages per (sequence, KV head)
    const int64_t pairs = (int64_t)B * Hkv;
    const int64_t waves = (pairs * units + kSlots * kMaxUnits - 1) / (kSlots * kMaxUnits);
    int64_t splits = waves * kSlots / pairs;  // per (sequence, KV head)
    if (splits < 1) splits = 1;
    int64_t per = (units + splits - 1) / splits;
    per = per < kMinUnits ? kMinUnits : (per > kMaxUnits ? kMaxUnits : per);
    return (int)(per * kUnit);
}

int decode_num_splits(int B, int Hkv, int64_t Nmax) {
    const int sk = decode_split_keys(B, Hkv, Nmax);
    return (int)((Nmax + sk - 1) / sk);
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int D) {
    return (size_t)B * Hq * decode_num_splits(B, Hkv, Nmax) * (D + 2) * sizeof(float);
}

__device__ __forceinline__ float2 dec_cos_sin(int64_t n, double theta) {
    double turns = (double)n * theta * 0.15915494309189533576888376337251;
    turns -= rint(turns);
    float a = (float)(turns * 6.283185307179586476925286766559);
    float s, c;
    sincosf(a, &s, &c);
    return make_float2(c, s);
}

__device__ __forceinline__ float ld_elem(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

__device__ __forceinline__ int dec_first_kept_pair(const int *w, int H, int64_t d) {
    int lo = 0, hi = H;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)w[mid] >= d) hi = mid; else lo = mid + 1;
    }
    return lo;
}

template <typename T, int D>
__global__ void __launch_bounds__(32 * kDecodeWarps) decode_split_kernel(
    const T *__restrict__ q, const T *__restrict__ kc, const T *__restrict__ vc, const int32_t *__restrict__ seqlens,
    float *__restrict__ ws, int Hq, int Hkv, int64_t Nmax, int krot, int nhd, int split_keys, int nsplit,
    const __grid_constant__ WindowParams wp) {
    constexpr int H = D / 2;
    constexpr int PPL = H / 32;  // pairs per lane
    constexpr int DPL = D / 32;  // value dims per lane
    __shared__ float sq[kMaxGroup][D];
    __shared__ int sw[H];
    __shared__ float red_m[kDecodeWarps][kMaxGroup], red_l[kDecodeWarps][kMaxGroup];
    __shared__ float red_acc[kDecodeWarps][kMaxGroup][D];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t L = seqlens[b];
    const int64_t s0 = (int64_t)split * split_keys;
    const int64_t s1 = (s0 + split_keys < L) ? s0 + split_keys : L;
    for (int r = tid; r < H; r += blockDim.x) sw[r] = wp.w[r];
    for (int e = tid; e < G * H; e += blockDim.x) {
        const int j = e / H, r = e % H;
        const size_t qo = ((size_t)b * Hq + (size_t)g * G + j) * D;
        const float x = ld_elem(q, qo + r), y = ld_elem(q, qo + r + H);
        const float2 t = dec_cos_sin(L - 1, wp.theta[r]);
        sq[j][r] = x * t.x - y * t.y;
        sq[j][r + H] = y * t.x + x * t.y;
    }
    __syncthreads();
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
    float mrun[kMaxGroup], lrun[kMaxGroup], acc[kMaxGroup][DPL];
#pragma unroll
    for (int j = 0; j < kMaxGroup; ++j) {
        mrun[j] = -INFINITY;
        lrun[j] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[j][e] = 0.f;
    }
    // HND: [B][Hkv][Nmax][D]; NHD: [B][Nmax][Hkv][D].
    const size_t head_base = nhd ? ((size_t)b * Nmax * Hkv + g) * D : ((size_t)b * Hkv + g) * (size_t)Nmax * D;
    const size_t key_stride = nhd ? (size_t)Hkv * D : (size_t)D;
    for (int64_t m = s0 + warp; m < s1; m += kDecodeWarps) {
        const int rs = dec_first_kept_pair(sw, H, (L - 1) - m);
        const size_t ko = head_base + (size_t)m * key_stride;
        float part[kMaxGroup];
#pragma unroll
        for (int j = 0; j < kMaxGroup; ++j) part[j] = 0.f;
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
            const int r = lane + 32 * i;
            if (r >= rs) {
                float ka = ld_elem(kc, ko + r), kb = ld_elem(kc, ko + r + H);
                if (!krot) {
                    const float2 t = dec_cos_sin(m, wp.theta[r]);
                    const float ra = ka * t.x - kb * t.y, rb = kb * t.x + ka * t.y;
                    ka = ra;
                    kb = rb;
                }
#pragma unroll
                for (int j = 0; j < kMaxGroup; ++j)
                    if (j < G) part[j] += sq[j][r] * ka + sq[j][r + H] * kb;
            }
        }
        float vv[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) vv[e] = ld_elem(vc, ko + lane + 32 * e);
#pragma unroll
        for (int j = 0; j < kMaxGroup; ++j) {
            if (j < G) {
                float s = part[j];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                s *= scale_log2;
                const float mnew = fmaxf(mrun[j], s);
                const float alpha = exp2f(mrun[j] - mnew);
                const float p = exp2f(s - mnew);
                lrun[j] = lrun[j] * alpha + p;
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[j][e] = acc[j][e] * alpha + p * vv[e];
                mrun[j] = mnew;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxGroup; ++j) {
        if (j < G) {
            if (lane == 0) {
                red_m[warp][j] = mrun[j];
                red_l[warp][j] = lrun[j];
            }
#pragma unroll
            for (int e = 0; e < DPL; ++e) red_acc[warp][j][lane + 32 * e] = acc[j][e];
        }
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += blockDim.x) {
        const int j = e / D, d = e % D;
        float M = -INFINITY;
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, red_m[w][j]);
        float l = 0.f, a = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < kDecodeWarps; ++w) {
                if (red_l[w][j] > 0.f) {
                    const float f = exp2f(red_m[w][j] - M);
                    l += red_l[w][j] * f;
                    a += red_acc[w][j][d] * f;
                }
            }
        }
        float *dst = ws + (((size_t)b * Hq + (size_t)g * G + j) * nsplit + split) * (D + 2);
        if (d == 0) {
            dst[0] = M;
            dst[1] = l;
        }
        dst[2 + d] = a;
    }
}

// Merge the per-split states (m in log2 units, l, unnormalised acc) of one
// (sequence, query head) into the output row.  A block takes a slice of
// kMergeDims output dims: it forms the max and the weighted sum over all splits
// (block-wide reductions), then kMergeParts thread groups accumulate interleaved
// splits for its dims and add their parts through shared memory.  The grid
// (query heads x sequences x dim slices) keeps enough split states in flight to
// hide memory latency.
constexpr int kMergeDims = 32;
constexpr int kMergeParts = 8;
constexpr int kMergeThreads = kMergeDims * kMergeParts;

__device__ __forceinline__ float block_reduce(float v, bool is_max, float *red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, v, off);
        v = is_max ? fmaxf(v, o) : v + o;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = (lane < (int)(blockDim.x >> 5)) ? red[lane] : (is_max ? -INFINITY : 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, v, off);
        v = is_max ? fmaxf(v, o) : v + o;
    }
    return v;
}

__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const float *__restrict__ ws, void *out,
                                                                     int out_f32, int Hq, int nsplit, int D) {
    __shared__ float red[32];
    __shared__ float part_acc[kMergeParts][kMergeDims];
    // Launched as a dependent of the split kernel: wait for its states.
    pdl_wait();
    pdl_allow_dependents();
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const float *base = ws + ((size_t)b * Hq + h) * nsplit * (D + 2);
    float mx = -INFINITY;
    for (int s = tid; s < nsplit; s += kMergeThreads) {
        const float *st = base + (size_t)s * (D + 2);
        if (st[1] > 0.f) mx = fmaxf(mx, st[0]);
    }
    const float M = block_reduce(mx, true, red);
    float ls = 0.f;
    for (int s = tid; s < nsplit; s += kMergeThreads) {
        const float *st = base + (size_t)s * (D + 2);
        if (st[1] > 0.f) ls += st[1] * exp2f(st[0] - M);
    }
    const float Lsum = block_reduce(ls, false, red);
    const int part = tid / kMergeDims, dl = tid % kMergeDims;
    const int d = blockIdx.z * kMergeDims + dl;
    float a = 0.f;
#pragma unroll 8
    for (int s = part; s < nsplit; s += kMergeParts) {
        const float *st = base + (size_t)s * (D + 2);
        const float l = st[1];
        if (l > 0.f) a += st[2 + d] * exp2f(st[0] - M);
    }
    part_acc[part][dl] = a;
    __syncthreads();
    if (tid < kMergeDims) {
        float acc = 0.f;
#pragma unroll
        for (int pp = 0; pp < kMergeParts; ++pp) acc += part_acc[pp][tid];
        const float val = acc / Lsum;
        const size_t o = ((size_t)b * Hq + h) * D + d;
        if (out_f32) reinterpret_cast<float *>(out)[o] = val;
        else reinterpret_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(val);
    }
}

cudaError_t launch_decode(const void *q, const void *kc, const void *vc, const int32_t *seqlens, void *out,
                          int out_f32, int in_f32, int krot, int layout, const Problem &p, const WindowParams &wp,
                          float *workspace, cudaStream_t s, const PagedKV *paged) {
    const int nhd = (layout == ATFLASH_KV_NHD);
    const int split_keys = decode_split_keys(p.B, p.Hkv, p.N);
    const int nsplit = decode_num_splits(p.B, p.Hkv, p.N);
    cudaError_t e;
    if (!in_f32) {
        int *status = device_status_word();
        if (!status) return cudaErrorUnknown;
        e = launch_decode_tc(q, kc, vc, seqlens, krot, layout, p, wp, workspace, split_keys, nsplit, status,
                             wait_limit_ns(), s, paged);
    } else {
        if (layout == ATFLASH_KV_PACKED || paged) return cudaErrorInvalidValue;  // bf16 caches only
        dim3 grid((unsigned)nsplit, (unsigned)p.Hkv, (unsigned)p.B);
        dim3 block(32 * kDecodeWarps);
        if (p.D == 128)
            decode_split_kernel<float, 128><<<grid, block, 0, s>>>((const float *)q, (const float *)kc,
                                                                   (const float *)vc, seqlens, workspace, p.Hq,
                                                                   p.Hkv, p.N, krot, nhd, split_keys, nsplit, wp);
        else if (p.D == 64)
            decode_split_kernel<float, 64><<<grid, block, 0, s>>>((const float *)q, (const float *)kc,
                                                                  (const float *)vc, seqlens, workspace, p.Hq,
                                                                  p.Hkv, p.N, krot, nhd, split_keys, nsplit, wp);
        else
            return cudaErrorInvalidValue;
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    // The merge and the short decode rows are launched as programmatic dependents,
    // so that their launch overlaps the tail of the kernel before them.
    e = launch_dependent(decode_merge_kernel, dim3((unsigned)p.Hq, (unsigned)p.B, (unsigned)(p.D / kMergeDims)),
                         dim3(kMergeThreads), 0, s, (const float *)workspace, out, out_f32, p.Hq, nsplit, p.D);
    if (e != cudaSuccess || in_f32) return e;
    // bf16 caches: sequences of at most 128 tokens again in fp32 (the fp32 path is exact already).
    int *status = device_status_word();
    if (!status) return cudaErrorUnknown;
    return launch_short_rows_decode(q, kc, vc, seqlens, out, out_f32, krot, layout, p, wp, status, s, paged);
}

}  // namespace atf
