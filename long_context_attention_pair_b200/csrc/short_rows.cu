// Rows that see at most 128 keys, recomputed exactly in fp32 on CUDA cores.
//
// The tensor-core kernels round the rotated queries and keys to bf16 (the
// tcgen05 / mma.sync operands) and the probabilities P to bf16 (the P.V
// operand).  Over a long row those roundings average out.  A row that sees only
// a handful of keys is a weighted mean of a handful of values, so one rounded
// score moves it by up to about 1e-2 (seeded sweeps: rows with 4-16 keys reach
// 1.06e-2; rows with more than 128 keys stay below 4e-3).  Such rows are few
// and cheap, so this kernel computes them again after the tensor-core kernels,
// from the caller's un-rotated inputs, by the method's plain definition
// ("ATFlash — Per-RoPE-Wavelength Attention Windows", "The idea"): rotate-half
// RoPE with the angle position * theta_r reduced mod 2*pi in fp64, the score as
// the sum over the pairs kept at the cell's distance (n - m <= w_r) scaled by
// 1/sqrt(D), a two-pass softmax and P.V, all in fp32.  It overwrites the rows'
// output (and log-sum-exp).
//
// Which rows:
//   prefill           the first 128-row tile of every sequence (row n sees n+1 keys);
//   block selection   every query tile whose mask selects no earlier key tile
//                     (its rows see only their own tile; every other row sees
//                     at least 129 keys);
//   decode            every sequence of at most 128 tokens.
//
// A CTA takes up to 32 rows: 32 consecutive positions of one query head
// (prefill), or the G query heads of one KV head at the decode position.  Keys
// are staged 32 at a time, rotated, as fp32 columns [dim][key]; scores go to
// shared memory, then the softmax, then P.V with the values staged the same way.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace atf {
namespace sr {

constexpr int kTile = 128;                     // query / key tile of the prefill kernel
constexpr int kRows = 32;                      // rows per work item
constexpr int kKeys = 32;                      // keys staged per pass
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRowsPerWarp = kRows / kWarps;   // 4

// Where the keys and values live.  Element offsets are in bf16 units.
struct Src {
    const __nv_bfloat16 *k, *v;
    int k_layout;        // ATFLASH_KV_HND, ATFLASH_KV_NHD or ATFLASH_KV_PACKED
    int v_layout;        // ATFLASH_KV_HND or ATFLASH_KV_NHD
    int rotated;         // keys stored rotated (packed, or a pre-rotated cache)
    int64_t ntok;        // tokens per batch entry along the token axis
    int Hkv;
    const int32_t *block_table;  // paged pool when not null
    int max_pages, page_size, num_pages;
};

struct Args {
    const __nv_bfloat16 *q;
    Src kv;
    void *out;
    int out_f32;
    float *lse;            // prefill only: [bz][Hq][ntok]
    int Hq, Hkv, G;
    int64_t N;             // prefill: longest sequence; decode: Nmax
    const int32_t *cu;     // varlen prefill: sequence b is tokens cu[b] .. cu[b+1]-1
    int64_t total;
    const uint8_t *block_mask;  // block-selected prefill: [B][Hkv][T][T]
    int num_qt;
    const int32_t *seqlens;     // decode
    int *status;                // device status word (bad page ids)
};

__device__ __forceinline__ float2 sr_cos_sin(int64_t pos, double theta) {
    double turns = (double)pos * theta * 0.15915494309189533576888376337251;  // 1/(2*pi)
    turns -= rint(turns);
    float s, c;
    sincosf((float)(turns * 6.283185307179586476925286766559), &s, &c);
    return make_float2(c, s);
}

// Page holding token t of sequence b, or -1 (recorded in the status word) when
// the index is past the block table row or the id is outside the pool.
__device__ __forceinline__ int sr_page(const Src &s, int b, int64_t t, int *status) {
    const int64_t pi = t / s.page_size;
    const int page = pi < s.max_pages ? s.block_table[(size_t)b * s.max_pages + pi] : -1;
    if (page < 0 || page >= s.num_pages) {
        atomicCAS(status, 0, ATFLASH_DEVICE_BAD_PAGE);
        return -1;
    }
    return page;
}

// Offset of token t's D-vector of KV head kvh in a natural layout or a page; -1 for a bad page.
template <int D>
__device__ __forceinline__ int64_t sr_row(const Src &s, int layout, int b, int kvh, int64_t t, int *status) {
    if (s.block_table) {
        const int page = sr_page(s, b, t, status);
        if (page < 0) return -1;
        return (((int64_t)page * s.page_size + t % s.page_size) * s.Hkv + kvh) * D;
    }
    if (layout == ATFLASH_KV_HND) return (((int64_t)b * s.Hkv + kvh) * s.ntok + t) * D;
    return (((int64_t)b * s.ntok + t) * s.Hkv + kvh) * D;
}

// Stored (k_r, k_{r+D/2}) of token t, rotated to position `pos` unless stored rotated.
template <int D>
__device__ __forceinline__ float2 sr_key_pair(const Src &s, int b, int kvh, int64_t t, int64_t pos, int r,
                                              double theta, int *status) {
    constexpr int H = D / 2, C = D / 16;
    float x, y;
    if (s.k_layout == ATFLASH_KV_PACKED) {
        int64_t o;
        if (s.block_table) {
            const int page = sr_page(s, b, t, status);
            if (page < 0) return make_float2(0.f, 0.f);
            o = ((((int64_t)page * s.Hkv + kvh) * C + r / 8) * s.page_size + t % s.page_size) * 16 + 2 * (r % 8);
        } else {
            o = ((((int64_t)b * s.Hkv + kvh) * C + r / 8) * s.ntok + t) * 16 + 2 * (r % 8);
        }
        x = __bfloat162float(s.k[o]);
        y = __bfloat162float(s.k[o + 1]);
    } else {
        const int64_t o = sr_row<D>(s, s.k_layout, b, kvh, t, status);
        if (o < 0) return make_float2(0.f, 0.f);
        x = __bfloat162float(s.k[o + r]);
        y = __bfloat162float(s.k[o + r + H]);
    }
    if (s.rotated) return make_float2(x, y);
    const float2 cs = sr_cos_sin(pos, theta);
    return make_float2(x * cs.x - y * cs.y, y * cs.x + x * cs.y);
}

// kDecode = false: grid (candidate query tiles, work items, B*Hkv); a work item is
// (32-row slice, query head of the group), one per CTA (gridDim.y = 4G).  Dense and
// ragged launches take only query tile 0; block-selected launches every query tile,
// and a CTA whose tile keeps an earlier key tile exits after scanning the mask row.
// kDecode = true: grid (1, 1, B*Hkv); the rows are the group's query heads.
template <int D, bool kDecode>
__global__ void __launch_bounds__(kThreads) short_rows_kernel(const __grid_constant__ Args a,
                                                              const __grid_constant__ WindowParams wp) {
    constexpr int H = D / 2;
    constexpr int DW = D / 32;  // output dims per lane
    extern __shared__ float smem[];
    float *sQ = smem;                 // [kRows][D] rotated queries
    float *sKV = sQ + kRows * D;      // [D][kKeys] rotated keys, later [kKeys][D] values
    float *sS = sKV + kKeys * D;      // [kRows][kTile] scores, then probabilities
    __shared__ int sw[kMaxPairs];
    __shared__ float s_l[kRows], s_m[kRows];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z / a.Hkv, kvh = blockIdx.z % a.Hkv;
    const float scale = rsqrtf((float)D);
    for (int r = tid; r < H; r += kThreads) sw[r] = wp.w[r];

    // Rows of this CTA: positions (prefill) or heads (decode), keys [key_lo, key_hi].
    int64_t seq_len = 0, tokbase = 0, n0 = 0;
    int bz = b;
    if constexpr (kDecode) {
        // A programmatic dependent of the merge, whose output rows it overwrites;
        // every CTA waits, so that this kernel never completes before the merge.
        pdl_wait();
        seq_len = a.seqlens[b];
        if (seq_len < 1 || seq_len > kTile || seq_len > a.N) return;
    } else {
        seq_len = a.N;
        if (a.cu) {
            const int64_t t0 = a.cu[b], t1 = a.cu[b + 1];
            seq_len = (t0 >= 0 && t1 >= t0 && t1 <= a.total) ? t1 - t0 : 0;
            tokbase = seq_len > 0 ? t0 : 0;
            if (seq_len > a.N) seq_len = a.N;  // rows beyond max_seqlen are not computed
            bz = 0;
        }
        const int qt = blockIdx.x;
        n0 = (int64_t)qt * kTile;
        if (n0 >= seq_len) return;
        if (a.block_mask) {
            // A query tile whose mask selects an earlier key tile has rows of >= 129 keys.
            const uint8_t *row = a.block_mask + (((size_t)b * a.Hkv + kvh) * a.num_qt + qt) * (size_t)a.num_qt;
            int any = 0;
            for (int j = tid; j < qt; j += kThreads) any |= row[j];
            if (__syncthreads_or(any)) return;
        }
    }

    const int items = kDecode ? 1 : 4 * a.G;
    for (int item = blockIdx.y; item < items; item += gridDim.y) {
        int hq = 0, nrows;
        int64_t n_lo = 0, key_lo, key_hi;
        if constexpr (kDecode) {
            nrows = a.G;
            key_lo = 0;
            key_hi = seq_len - 1;
        } else {
            const int slice = item % 4;
            hq = kvh * a.G + item / 4;
            n_lo = n0 + kRows * slice;
            int64_t n_hi = n_lo + kRows - 1;
            if (n_hi > seq_len - 1) n_hi = seq_len - 1;
            if (n_lo > n_hi) continue;  // uniform over the CTA
            nrows = (int)(n_hi - n_lo + 1);
            key_lo = n0;
            key_hi = n_hi;
        }
        const int nkeys = (int)(key_hi - key_lo + 1);  // <= 128
        const int nchunks = (nkeys + kKeys - 1) / kKeys;
        __syncthreads();  // the previous item is done with shared memory

        // Rotated queries, fp32.
        for (int e = tid; e < kRows * H; e += kThreads) {
            const int row = e / H, r = e % H;
            float xr = 0.f, xh = 0.f;
            if (row < nrows) {
                int64_t qo, pos;
                if constexpr (kDecode) {
                    qo = ((int64_t)b * a.Hq + kvh * a.G + row) * D;
                    pos = seq_len - 1;
                } else {
                    qo = (((int64_t)bz * a.kv.ntok + tokbase + n_lo + row) * a.Hq + hq) * D;
                    pos = n_lo + row;
                }
                const float x = __bfloat162float(a.q[qo + r]), y = __bfloat162float(a.q[qo + r + H]);
                const float2 cs = sr_cos_sin(pos, wp.theta[r]);
                xr = x * cs.x - y * cs.y;
                xh = y * cs.x + x * cs.y;
            }
            sQ[row * D + r] = xr;
            sQ[row * D + r + H] = xh;
        }

        // Scores: the pairs kept at each cell's distance, in fp32.
        for (int kc = 0; kc < nchunks; ++kc) {
            __syncthreads();
            for (int e = tid; e < kKeys * H; e += kThreads) {
                const int j = e % kKeys, r = e / kKeys;
                const int64_t m = key_lo + kc * kKeys + j;
                float2 kp = make_float2(0.f, 0.f);
                if (m <= key_hi) kp = sr_key_pair<D>(a.kv, bz, kvh, tokbase + m, m, r, wp.theta[r], a.status);
                sKV[r * kKeys + j] = kp.x;
                sKV[(r + H) * kKeys + j] = kp.y;
            }
            __syncthreads();
#pragma unroll
            for (int rr = 0; rr < kRowsPerWarp; ++rr) {
                const int row = warp * kRowsPerWarp + rr;
                if (row >= nrows) break;
                const int64_t pos = kDecode ? seq_len - 1 : n_lo + row;
                const int64_t m = key_lo + kc * kKeys + lane;
                float s = -INFINITY;
                if (m <= key_hi && m <= pos) {
                    const int64_t d = pos - m;
                    const float *qr = sQ + row * D;
                    float acc = 0.f;
#pragma unroll 8
                    for (int r = 0; r < H; ++r)
                        if (d <= (int64_t)sw[r])
                            acc = fmaf(qr[r], sKV[r * kKeys + lane], fmaf(qr[r + H], sKV[(r + H) * kKeys + lane], acc));
                    s = acc * scale;  // an empty sum scores 0
                }
                sS[row * kTile + kc * kKeys + lane] = s;
            }
        }
        __syncwarp();

        // Softmax of each row (two passes: max, then exp and sum).
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int row = warp * kRowsPerWarp + rr;
            if (row >= nrows) break;
            float *srow = sS + row * kTile;
            float mx = -INFINITY;
            for (int idx = lane; idx < nchunks * kKeys; idx += 32) mx = fmaxf(mx, srow[idx]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            float l = 0.f;
            for (int idx = lane; idx < nchunks * kKeys; idx += 32) {
                const float sv = srow[idx];
                const float p = (sv == -INFINITY) ? 0.f : expf(sv - mx);
                srow[idx] = p;
                l += p;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
            if (lane == 0) {
                s_l[row] = l;
                s_m[row] = mx;
            }
        }

        // P.V, values staged as [key][dim].
        float o[kRowsPerWarp][DW];
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr)
#pragma unroll
            for (int e = 0; e < DW; ++e) o[rr][e] = 0.f;
        for (int kc = 0; kc < nchunks; ++kc) {
            __syncthreads();
            for (int e = tid; e < kKeys * D; e += kThreads) {
                const int j = e / D, dd = e % D;
                const int64_t m = key_lo + kc * kKeys + j;
                float val = 0.f;
                if (m <= key_hi) {
                    const int64_t vo = sr_row<D>(a.kv, a.kv.v_layout, bz, kvh, tokbase + m, a.status);
                    if (vo >= 0) val = __bfloat162float(a.kv.v[vo + dd]);
                }
                sKV[j * D + dd] = val;
            }
            __syncthreads();
#pragma unroll
            for (int rr = 0; rr < kRowsPerWarp; ++rr) {
                const int row = warp * kRowsPerWarp + rr;
                if (row >= nrows) break;
                const float *prow = sS + row * kTile + kc * kKeys;
#pragma unroll 4
                for (int j = 0; j < kKeys; ++j) {
                    const float p = prow[j];
#pragma unroll
                    for (int e = 0; e < DW; ++e) o[rr][e] = fmaf(p, sKV[j * D + lane + 32 * e], o[rr][e]);
                }
            }
        }

        // Output rows (and log-sum-exp).
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int row = warp * kRowsPerWarp + rr;
            if (row >= nrows) break;
            const float inv = 1.f / s_l[row];
            int64_t oo;
            if constexpr (kDecode) oo = ((int64_t)b * a.Hq + kvh * a.G + row) * D;
            else oo = (((int64_t)bz * a.kv.ntok + tokbase + n_lo + row) * a.Hq + hq) * D;
#pragma unroll
            for (int e = 0; e < DW; ++e) {
                const float val = o[rr][e] * inv;
                if (a.out_f32) reinterpret_cast<float *>(a.out)[oo + lane + 32 * e] = val;
                else reinterpret_cast<__nv_bfloat16 *>(a.out)[oo + lane + 32 * e] = __float2bfloat16_rn(val);
            }
            if (!kDecode && a.lse && lane == 0)
                a.lse[((int64_t)bz * a.Hq + hq) * a.kv.ntok + tokbase + n_lo + row] = s_m[row] + logf(s_l[row]);
        }
    }
}

template <int D, bool kDecode>
static cudaError_t launch(const Args &a, const WindowParams &wp, dim3 grid, cudaStream_t s) {
    const int smem = (kRows * D + kKeys * D + kRows * kTile) * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(short_rows_kernel<D, kDecode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    if constexpr (kDecode) {
        // After the merge, as its programmatic dependent.
        return launch_dependent(short_rows_kernel<D, kDecode>, grid, dim3(kThreads), smem, s, a, wp);
    } else {
        short_rows_kernel<D, kDecode><<<grid, kThreads, smem, s>>>(a, wp);
        return cudaGetLastError();
    }
}

}  // namespace sr

cudaError_t launch_short_rows_prefill(const void *q, const void *k, const void *v, void *out, int out_f32,
                                      float *lse, const Problem &p, const WindowParams &wp, int *status,
                                      cudaStream_t s, const int32_t *cu_seqlens, int64_t total,
                                      const uint8_t *block_mask) {
    if (cu_seqlens && block_mask) return cudaErrorInvalidValue;
    sr::Args a{};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.kv.k = static_cast<const __nv_bfloat16 *>(k);
    a.kv.v = static_cast<const __nv_bfloat16 *>(v);
    a.kv.k_layout = a.kv.v_layout = ATFLASH_KV_NHD;
    a.kv.rotated = 0;
    a.kv.ntok = cu_seqlens ? total : p.N;
    a.kv.Hkv = p.Hkv;
    a.out = out;
    a.out_f32 = out_f32;
    a.lse = lse;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.Hq / p.Hkv;
    a.N = p.N;
    a.cu = cu_seqlens;
    a.total = total;
    a.block_mask = block_mask;
    a.num_qt = (int)((p.N + sr::kTile - 1) / sr::kTile);
    a.status = status;
    const unsigned z = (unsigned)(p.B * p.Hkv);
    const dim3 grid((unsigned)(block_mask ? a.num_qt : 1), (unsigned)(4 * a.G), z);
    if (p.D == 128) return sr::launch<128, false>(a, wp, grid, s);
    if (p.D == 64) return sr::launch<64, false>(a, wp, grid, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_short_rows_decode(const void *q, const void *kc, const void *vc, const int32_t *seqlens,
                                     void *out, int out_f32, int krot, int layout, const Problem &p,
                                     const WindowParams &wp, int *status, cudaStream_t s, const PagedKV *paged) {
    sr::Args a{};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.kv.k = static_cast<const __nv_bfloat16 *>(kc);
    a.kv.v = static_cast<const __nv_bfloat16 *>(vc);
    a.kv.k_layout = layout;
    // Packed K goes with HND values in a contiguous cache and with natural pages.
    a.kv.v_layout = (layout == ATFLASH_KV_PACKED) ? (paged ? ATFLASH_KV_NHD : ATFLASH_KV_HND) : layout;
    a.kv.rotated = (layout == ATFLASH_KV_PACKED) ? 1 : krot;
    a.kv.ntok = p.N;
    a.kv.Hkv = p.Hkv;
    if (paged) {
        a.kv.block_table = paged->block_table;
        a.kv.max_pages = paged->max_pages;
        a.kv.page_size = paged->page_size;
        a.kv.num_pages = paged->num_pages;
    }
    a.out = out;
    a.out_f32 = out_f32;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.Hq / p.Hkv;
    a.N = p.N;
    a.seqlens = seqlens;
    a.status = status;
    if (a.G > sr::kRows) return cudaErrorInvalidValue;
    const dim3 grid(1, 1, (unsigned)(p.B * p.Hkv));
    if (p.D == 128) return sr::launch<128, true>(a, wp, grid, s);
    if (p.D == 64) return sr::launch<64, true>(a, wp, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace atf
