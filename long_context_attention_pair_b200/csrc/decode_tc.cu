// Split-KV windowed decode on tensor cores (bf16 caches).
//
// One CTA = one split of one (sequence, KV head): the 16 keys of a consumer
// warp are the M rows of mma.sync m16n8k16 tiles and the G = Hq/Hkv query
// heads their N columns (tiles of 8 heads).  The
// method ("ATFlash — Per-RoPE-Wavelength Attention Windows", "The idea" and
// "Numbers": the window is a condition on which K elements are loaded):
// for a key at distance d = L-1-m only pairs r >= r*(d) are kept, so
//   - the producer warp streams 64-key stages with TMA, loading for K only the
//     8-pair chunks that some key of the stage keeps, and all of V;
//   - each consumer warp takes 16 keys of a stage: ldmatrix puts complete
//     frequency pairs (r, r+D/2) of one key into one thread, which rotates them
//     (unless the cache is pre-rotated) and zeroes the pairs its key prunes;
//   - S^T = K~ Q~^T, the online softmax and O^T += V^T P^T stay in registers.
// The contraction order inside a K-step is [8 low-half dims, 8 high-half dims]
// for both Q~ and K~, so every dot product is unchanged.
//
// Angles (rotation at load only): the producer writes, per stage, the base
// angle stage_start*theta_r reduced mod 2*pi, from a 64-bit fixed-point turn
// count: theta_r/(2*pi) as a fraction of 2^64, times the integer position,
// wraps modulo 2^64 = whole turns, so the reduction is exact integer
// arithmetic (the fraction carries fp64's precision of theta_r).  A key at
// offset i adds i*theta_r (i < 64) in fp32, reduces once more and takes
// sin/cos on [-pi, pi].
//
// Packed cache (ATFLASH_KV_PACKED): K already rotated and stored as the RoPE
// pre-pass writes it, [B*Hkv][D/16][Nmax][16] with 8 frequency pairs per 32-byte
// chunk.  A pruned chunk of 64 keys is then 2 KB of HBM that is never fetched.
// In the natural layouts a key's pruned dims are a prefix of each half-row; the
// copy fetches each half in 32-byte (16-dim) boxes from the first 32-byte sector
// that some key of the stage keeps.  That saves shared-memory fills and consumer
// work but no DRAM traffic: every half-row keeps its lowest-frequency sector, and
// the memory system brings a 128-byte half-row in whole once any of its sectors
// is read (measured: the whole cache per launch).  The 2 KB of one chunk
// of a stage are contiguous, so the copy views them as 16 rows of 128 bytes
// (4 keys per row, SWIZZLE_128B) rather than 64 rows of 32 bytes: a quarter of
// the TMA row requests, which bound the producer otherwise.  That view needs
// Nmax % 4 == 0 (whole rows per chunk); other lengths keep the 32-byte rows.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace atf {
namespace dtc {

constexpr int kStageKeys = 64;
constexpr int kWarpsPerStage = 4;                   // 16 keys per consumer warp
constexpr int kGroups = 1;                          // groups consume stages round-robin
constexpr int kConsumers = kWarpsPerStage * kGroups;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct Cfg {
    // Two stages per CTA and three CTAs per SM (69 KB of dynamic shared memory each,
    // plus at most 3 KB of static tables and the 1 KB the hardware reserves per CTA):
    // more consumer warps to hide latency, as many bytes in flight as three stages at
    // two.  The rotated queries are kept as bf16 (the MMA operand) so that three fit.
    static constexpr int kStages = 2;
    static constexpr int H = D / 2;
    static constexpr int C = D / 16;                   // chunks of 8 pairs
    // K stage: packed [c][64 keys][32 B] (SW128 as 16 rows of 128 B, or SW32), natural
    // [half][D/32 16-dim groups][64 keys][32 B] SW32.
    static constexpr int KBytes = C * 2 * 1024;
    static constexpr int VBytes = (D / 64) * 8192;     // [D/64][64 keys][64 dims] bf16, SW128
    static constexpr int OffK = 0;
    static constexpr int OffV = OffK + kStages * KBytes;
    static constexpr int OffBase = OffV + kStages * VBytes;      // [stage][H] float
    static constexpr int OffQ = OffBase + kStages * H * 4;       // [16][D] bf16, rotated queries
    static constexpr int OffBar = OffQ + 16 * D * 2;
    static constexpr int Total = OffBar + 256;
    static constexpr int Request = Total + 1024;
    static_assert(3 * (Request + 3072 + 1024) <= 233472, "three CTAs must fit the SM's 228 KB");
};

constexpr int kMaxStages = 8;
struct Bars {
    uint64_t full[kMaxStages], empty[kMaxStages];
    int abort_flag;
};

// r*(d) as d shrinks: keys of later stages are nearer the query, so the first
// kept pair only moves down; amortised O(1) per stage.
__device__ __forceinline__ int walk_down(const int *w, int r, int d) {
    while (r > 0 && w[r - 1] >= d) --r;
    return r;
}
// The walks' starting points: r*(d) = the smallest r with w_r >= d (H when none),
// by bisection (the windows do not decrease in r).  Walking down from H instead
// took up to H dependent shared-memory reads before a CTA's first stage.
__device__ __forceinline__ int first_kept_pair(const int *w, int H, int d) {
    int lo = 0, hi = H;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (w[mid] >= d) hi = mid; else lo = mid + 1;
    }
    return lo;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &d0, uint32_t &d1, uint32_t &d2, uint32_t &d3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &d0, uint32_t &d1, uint32_t &d2, uint32_t &d3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
                 : "r"(addr));
}
// 8x8 transpose of a b16 matrix held one row pair per thread (thread t: row t/4,
// columns 2(t%4), 2(t%4)+1); afterwards thread t holds row t/4 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two bf16 values as one register (lo in the low half).
__device__ __forceinline__ uint32_t bf16_pair(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// Rotate the two pairs held in (lo, hi) = (dims r|r+1 of the low half, dims
// r+H|r+1+H) of one key, and zero a pair whose window the key exceeds.
__device__ __forceinline__ void rotate_pairs(uint32_t &lo, uint32_t &hi, float c0, float s0, float c1, float s1,
                                             bool keep0, bool keep1) {
    const float a0 = bf16lo(lo), a1 = bf16hi(lo), b0 = bf16lo(hi), b1 = bf16hi(hi);
    float x0 = a0 * c0 - b0 * s0, y0 = b0 * c0 + a0 * s0;
    float x1 = a1 * c1 - b1 * s1, y1 = b1 * c1 + a1 * s1;
    if (!keep0) x0 = y0 = 0.f;
    if (!keep1) x1 = y1 = 0.f;
    lo = pack_bf16x2(x0, x1);
    hi = pack_bf16x2(y0, y1);
}
__device__ __forceinline__ void mask_pairs(uint32_t &lo, uint32_t &hi, bool keep0, bool keep1) {
    const uint32_t m = (keep0 ? 0x0000FFFFu : 0u) | (keep1 ? 0xFFFF0000u : 0u);
    lo &= m;
    hi &= m;
}

// Three CTAs per SM for groups of up to 8 heads (160 threads each, at most 128
// registers per thread); larger groups keep the registers their accumulators need.
// kPaged: K and V live in pages of page_size tokens (a multiple of the 64-key
// stage), page block_table[b * max_pages + i] holding keys i*page_size.. of
// sequence b; the maps index pages along their outermost axis.
// NT: tiles of 8 query heads (a GQA group of G <= 8 heads takes one tile, up to 16 two).
template <int D, bool kPacked, bool kPaged, int NT>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 3 : 1) decode_tc_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const void *q_,
    const int32_t *__restrict__ seqlens, float *__restrict__ ws, int Hq, int Hkv, int nhd, int krot, int split_keys,
    int nsplit, const __grid_constant__ WindowParams wp, int *status, uint64_t limit_ns,
    const int32_t *__restrict__ block_table, int max_pages, int page_size, int num_pages, int k_rows128) {
    using F = Cfg<D>;
    constexpr int H = F::H, C = F::C;
    constexpr int kStages = F::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + F::OffK;
    uint8_t *sV = smem + F::OffV;
    float *sBase = reinterpret_cast<float *>(smem + F::OffBase);
    __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(smem + F::OffQ);
    Bars *bars = reinterpret_cast<Bars *>(smem + F::OffBar);
    __shared__ int sw[kMaxPairs];
    __shared__ float sTheta[kMaxPairs];
    __shared__ uint64_t sTurn[kMaxPairs];  // theta_r / (2*pi) in units of 2^-64 turns
    __shared__ float2 sRot8[kMaxPairs];    // (cos, sin) of 8 * theta_r (rotation at load)

    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(q_);
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t L = seqlens[b];
    const int64_t s0 = (int64_t)split * split_keys;
    const int64_t s1 = (s0 + split_keys < L) ? s0 + split_keys : L;
    const int nstage = (s1 > s0) ? (int)((s1 - s0 + kStageKeys - 1) / kStageKeys) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], kWarpsPerStage);
        }
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    for (int r = threadIdx.x; r < H; r += kThreads) {
        sw[r] = wp.w[r];
        sTheta[r] = (float)wp.theta[r];
        // theta_r <= pi (base tables: <= 1), so the fraction is at most 2^63 and fits the integer.
        sTurn[r] = __double2ull_rn(wp.theta[r] * (0.15915494309189533576888376337251 * 18446744073709551616.0));
        if (!kPacked && !krot) {
            double s8, c8;
            sincos(8.0 * wp.theta[r], &s8, &c8);
            sRot8[r] = make_float2((float)c8, (float)s8);
        }
    }
    // Rotated queries at position L-1 (fp64 angle reduction), rows >= G are zero.
    for (int e = threadIdx.x; e < 16 * H; e += kThreads) {
        const int j = e / H, r = e % H;
        float xr = 0.f, xh = 0.f;
        if (j < G) {
            const size_t qo = ((size_t)b * Hq + (size_t)g * G + j) * D;
            const float a = __bfloat162float(q[qo + r]), c = __bfloat162float(q[qo + r + H]);
            double turns = (double)(L - 1) * wp.theta[r] * 0.15915494309189533576888376337251;
            turns -= rint(turns);
            float sn, cs;
            sincosf((float)(turns * 6.283185307179586476925286766559), &sn, &cs);
            xr = a * cs - c * sn;
            xh = c * cs + a * sn;
        }
        // Rounded once to bf16 here: the MMA's B operand.
        sQ[j * D + r] = __float2bfloat16_rn(xr);
        sQ[j * D + r + H] = __float2bfloat16_rn(xh);
    }
    __syncthreads();
    pdl_allow_dependents();  // the merge may be scheduled now; it waits for this grid to complete
    WaitCtl wc{&bars->abort_flag, status, limit_ns, 20};

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        int last[kMaxStages];
        for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        // Only a rotation at load needs the stage base angles.
        const bool rotate = !kPacked && !krot;
        // r*(d) of the stage's nearest key: stages move towards the query, so the
        // first kept pair only moves down (amortised O(1) per stage).
        int r_near = first_kept_pair(sw, H, (int)((L - 1) - (s0 + kStageKeys - 1 < s1 ? s0 + kStageKeys - 1 : s1 - 1)));
        for (int it = 0; it < nstage && ok; ++it) {
            const int st = it % kStages;
            const int64_t k0 = s0 + (int64_t)it * kStageKeys;
            int64_t k1 = k0 + kStageKeys - 1;
            if (k1 > s1 - 1) k1 = s1 - 1;
            r_near = walk_down(sw, r_near, (int)((L - 1) - k1));  // nearest key keeps the most
            const int c_lo = r_near >> 3;
            if (!(ok = mbar_wait_warp(&bars->empty[st], ((it / kStages) & 1) ^ 1, wc))) break;
            if (rotate) {
                for (int r = lane; r < H; r += 32) {
                    // Turns of k0 * theta_r modulo 1, as a signed fraction of 2^64 in [-1/2, 1/2).
                    const int64_t t = (int64_t)((uint64_t)k0 * sTurn[r]);
                    sBase[st * H + r] = (float)t * 3.4061215800865545e-19f;  // 2*pi / 2^64
                }
            }
            __syncwarp();
            if (lane == 0) {
                // Natural layouts: 16-dim groups g >= g_lo of both halves (32-byte sectors).
                constexpr int NG = H / 16;  // 16-dim groups per half
                const int g_lo = c_lo >> 1;
                const uint32_t kbytes =
                    kPacked ? (uint32_t)(C - c_lo) * 2048u : (uint32_t)(2 * (NG - g_lo)) * 2048u;
                const uint32_t bytes = kbytes + (uint32_t)F::VBytes;
                mbar_expect_tx(&bars->full[st], bytes);
                uint8_t *kst = sK + st * F::KBytes;
                if constexpr (kPaged) {
                    // A stage never straddles a page (page_size is a multiple of 64).  A
                    // page index past the table row or an id outside the pool is reported
                    // in the device status word and becomes -1, which the maps treat as
                    // out of bounds (zero fill, no access).
                    const int64_t pi = k0 / page_size;
                    int page = pi < max_pages ? block_table[(size_t)b * max_pages + pi] : -1;
                    if (page < 0 || page >= num_pages) {
                        atomicCAS(status, 0, ATFLASH_DEVICE_BAD_PAGE);
                        page = -1;
                    }
                    const int kk = (int)(k0 % page_size);
                    if (kPacked) {
                        // Pages hold a multiple of 64 keys, so the 128-byte row view always applies.
                        for (int c = c_lo; c < C; ++c)
                            tma_load_3d(kst + c * 2048, &tm_k, &bars->full[st], 0, kk / 4, (page * Hkv + g) * C + c);
                    } else {
                        for (int hf = 0; hf < 2; ++hf)
                            for (int gg = g_lo; gg < NG; ++gg)
                                tma_load_4d(kst + (hf * NG + gg) * 2048, &tm_k, &bars->full[st], hf * H + 16 * gg, g,
                                            kk, page);
                    }
                    for (int gi = 0; gi < D / 64; ++gi)
                        tma_load_4d(sV + st * F::VBytes + gi * 8192, &tm_v, &bars->full[st], 64 * gi, g, kk, page);
                } else if (kPacked) {
                    const int ky = k_rows128 ? (int)(k0 / 4) : (int)k0;
                    for (int c = c_lo; c < C; ++c)
                        tma_load_3d(kst + c * 2048, &tm_k, &bars->full[st], 0, ky, (b * Hkv + g) * C + c);
                } else {
                    // 64 keys x 16 dims per box, SWIZZLE_32B.
                    for (int hf = 0; hf < 2; ++hf)
                        for (int gg = g_lo; gg < NG; ++gg) {
                            uint8_t *dst = kst + (hf * NG + gg) * 2048;
                            const int x = hf * H + 16 * gg;
                            if (nhd) tma_load_4d(dst, &tm_k, &bars->full[st], x, g, (int)k0, b);
                            else tma_load_3d(dst, &tm_k, &bars->full[st], x, (int)k0, b * Hkv + g);
                        }
                }
                if constexpr (!kPaged) {
                    for (int gi = 0; gi < D / 64; ++gi) {
                        uint8_t *dst = sV + st * F::VBytes + gi * 8192;
                        if (nhd) tma_load_4d(dst, &tm_v, &bars->full[st], 64 * gi, g, (int)k0, b);
                        else tma_load_3d(dst, &tm_v, &bars->full[st], 64 * gi, (int)k0, b * Hkv + g);
                    }
                }
            }
            __syncwarp();
            last[st] = it;
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < kStages; ++s) {
                if (last[s] < 0) continue;
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bars->full[s], (last[s] / kStages) & 1))
                    if (globaltimer_ns() - t0 > atflash_drain_limit_ns(limit_ns)) break;
            }
        }
    } else {
        // ----------------------------------------------------------- consumers
        // Keys are the M rows of mma.sync m16n8k16 and the query heads of the group
        // its N columns (NT tiles of 8 heads): S^T = K~ Q~^T and O^T += V^T P^T.  A
        // group has at most 16 heads, so no head rows are padded beyond the tile.
        // Thread (gq, tq) = (lane / 4, lane % 4) holds S^T of keys gq and gq + 8 and
        // of heads 8t + 2tq, 8t + 2tq + 1 of head tile t.
        const int gq = lane >> 2, tq = lane & 3;
        // Q~^T B-fragments per chunk and head tile (head 8t + gq): elements
        // k = 2tq, 2tq+1 and k = 8+2tq, 9+2tq of the chunk's contraction order.
        uint32_t qb[C][NT][2];
#pragma unroll
        for (int c = 0; c < C; ++c) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const __nv_bfloat16 *qrow = sQ + (8 * t + gq) * D;
                if (kPacked) {
                    // k-order of a packed chunk: (pair 8c + k/2, component k%2).
                    const int pa = 8 * c + tq, pb = pa + 4;
                    qb[c][t][0] = bf16_pair(qrow[pa], qrow[pa + H]);
                    qb[c][t][1] = bf16_pair(qrow[pb], qrow[pb + H]);
                } else {
                    // k-order [dims 8c..8c+7, dims H+8c..H+8c+7]: two adjacent bf16 per register.
                    const int lo = 8 * c + 2 * tq, hi = H + 8 * c + 2 * tq;
                    qb[c][t][0] = *reinterpret_cast<const uint32_t *>(qrow + lo);
                    qb[c][t][1] = *reinterpret_cast<const uint32_t *>(qrow + hi);
                }
            }
        }
        const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
        // O^T accumulators: dims 16dg + gq (e = 0, 1) and 16dg + gq + 8 (e = 2, 3),
        // heads 8t + 2tq (e even) and 8t + 2tq + 1 (e odd).
        float o[D / 16][NT][4];
#pragma unroll
        for (int i = 0; i < D / 16; ++i)
#pragma unroll
            for (int t = 0; t < NT; ++t) o[i][t][0] = o[i][t][1] = o[i][t][2] = o[i][t][3] = 0.f;
        // Running max (log2 units) and this thread's part of the sum, per head 8t + 2tq + hh.
        float m_run[NT][2], l_run[NT][2];
#pragma unroll
        for (int t = 0; t < NT; ++t) m_run[t][0] = m_run[t][1] = -INFINITY, l_run[t][0] = l_run[t][1] = 0.f;
        const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
        bool ok = true;
        // Positions fit in int32 (Nmax <= 2^31 - 1).  Walk pointers for r*(d) of the
        // stage's nearest key, this warp's nearest key and this warp's farthest key.
        const int Lq = (int)L - 1;
        const int grp = warp / kWarpsPerStage, wq = warp % kWarpsPerStage;
        int r_stage = H, r_warp = H, r_keep = H;
        if (grp < nstage) {
            // Start the walks at this warp's first stage.
            const int k0 = (int)s0 + grp * kStageKeys, kw0 = k0 + 16 * wq, kend = (int)s1 - 1;
            r_stage = first_kept_pair(sw, H, Lq - (k0 + kStageKeys - 1 < kend ? k0 + kStageKeys - 1 : kend));
            r_warp = first_kept_pair(sw, H, Lq - (kw0 + 15 < kend ? kw0 + 15 : kend));
            r_keep = first_kept_pair(sw, H, Lq - kw0);
        }
        for (int it = grp; it < nstage && ok; it += kGroups) {
            const int st = it % kStages;
            const int k0 = (int)s0 + it * kStageKeys;
            const int kw0 = k0 + 16 * wq;  // this warp's first key
            if (!(ok = mbar_wait_warp(&bars->full[st], (it / kStages) & 1, wc))) break;
            const int kend = (int)s1 - 1;
            const int kw1 = (kw0 + 15 < kend) ? kw0 + 15 : kend;
            const int k1 = (k0 + kStageKeys - 1 < kend) ? k0 + kStageKeys - 1 : kend;
            r_stage = walk_down(sw, r_stage, Lq - k1);
            const int c_stage = r_stage >> 3;
            float sacc[NT][4], sodd[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[t][e] = sodd[t][e] = 0.f;
            if (kw0 < (int)s1) {
                r_warp = walk_down(sw, r_warp, Lq - kw1);
                r_keep = walk_down(sw, r_keep, Lq - kw0);
                const int c_warp = r_warp >> 3;
                // Distances of this thread's keys kw0 + gq and kw0 + gq + 8.
                const int da = Lq - (kw0 + gq), db = da - 8;
                const float fa = (float)(16 * wq + gq);
                const uint32_t kst = sKa + st * F::KBytes;
                const int mi = lane >> 3, ri = lane & 7;
                const int c_keep = (r_keep + 7) >> 3;
                // ldmatrix x4 of a chunk gives, per thread, b0 = key gq / first 8 k,
                // b1 = key gq / last 8 k, b2 = key gq+8 / first 8 k, b3 = key gq+8 /
                // last 8 k; the A fragment of the 16 keys is (b0, b2, b1, b3).
                if constexpr (kPacked) {
                    const int c_begin = c_warp > c_stage ? c_warp : c_stage;
                    // All of this warp's K fragments first (independent shared-memory loads in
                    // flight together), then the masks and the MMAs.
                    uint32_t kb[C][4];
                    // Matrix mi of the x4 load: keys +8*(mi>>1), bytes 16*(mi&1) of each key's 32.
                    const int key = 16 * wq + 8 * (mi >> 1) + ri;
                    // 128-byte rows (4 keys each, SWIZZLE_128B: 16-byte unit ^= row & 7), or
                    // 32-byte rows (one key each, SWIZZLE_32B: unit bit 0 ^= key bit 2).
                    const uint32_t koff =
                        (kPaged || k_rows128)
                            ? (uint32_t)((key >> 2) * 128 + ((((key & 3) * 2 + (mi & 1)) ^ ((key >> 2) & 7)) << 4))
                            : (uint32_t)(key * 32 + ((16 * (mi & 1)) ^ ((key & 4) << 2)));
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        if (c < c_begin) continue;
                        ldsm_x4(kst + c * 2048 + koff, kb[c][0], kb[c][1], kb[c][2], kb[c][3]);
                    }
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        if (c < c_begin) continue;
                        // Chunks from c_keep on are kept by every key of this warp: no masking.
                        const bool masked = c < c_keep;
                        uint32_t a[4] = {kb[c][0], kb[c][2], kb[c][1], kb[c][3]};
                        if (masked) {
                            const int p0 = 8 * c + tq, p1 = p0 + 4;
                            const int w0 = sw[p0], w1 = sw[p1];
                            a[0] = (da <= w0) ? a[0] : 0u;
                            a[2] = (da <= w1) ? a[2] : 0u;
                            a[1] = (db <= w0) ? a[1] : 0u;
                            a[3] = (db <= w1) ? a[3] : 0u;
                        }
                        // Two independent accumulation chains (chunk parity).
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            if (c & 1) mma16816(sodd[t], a, qb[c][t][0], qb[c][t][1]);
                            else mma16816(sacc[t], a, qb[c][t][0], qb[c][t][1]);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        if (c < (c_warp > c_stage ? c_warp : c_stage)) continue;
                        const bool masked = c < c_keep;
                        uint32_t b0, b1, b2, b3;
                        // 16-dim groups of 64 keys x 32 B (SWIZZLE_32B: 16-byte unit ^= key bit 2);
                        // matrix mi: keys +8*(mi>>1), dims (mi&1)*H + 8c .. +8 of each key, i.e.
                        // unit c&1 of group c>>1 of half mi&1.
                        const int key = 16 * wq + 8 * (mi >> 1) + ri;
                        const uint32_t addr = kst + ((mi & 1) * (H / 16) + (c >> 1)) * 2048 + key * 32 +
                                              ((((uint32_t)c & 1u) ^ (((uint32_t)key >> 2) & 1u)) << 4);
                        ldsm_x4(addr, b0, b1, b2, b3);
                        const int p0 = 8 * c + 2 * tq, p1 = p0 + 1;
                        const int w0 = sw[p0], w1 = sw[p1];
                        const bool ka0 = da <= w0, ka1 = da <= w1, kb0 = db <= w0, kb1 = db <= w1;
                        if (krot) {
                            if (masked) {
                                mask_pairs(b0, b1, ka0, ka1);
                                mask_pairs(b2, b3, kb0, kb1);
                            }
                        } else {
                            const float th0 = sTheta[p0], th1 = sTheta[p1];
                            const float base0 = sBase[st * H + p0], base1 = sBase[st * H + p1];
                            // Key gq's angles reduced to [-pi, pi] and sin/cos taken; key gq+8
                            // sits 8 positions later: its (cos, sin) is key gq's rotated by the
                            // fixed 8*theta_r (angle addition, 4 FMAs instead of a sincos).
                            float ang[2] = {fmaf(fa, th0, base0), fmaf(fa, th1, base1)};
                            float cs[4], sn[4];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const float turns = rintf(ang[u] * 0.15915494309189533577f);
                                const float x = fmaf(-turns, 6.283185307179586477f, ang[u]);
                                __sincosf(x, &sn[u], &cs[u]);
                            }
                            const float2 e0 = sRot8[p0], e1 = sRot8[p1];
                            cs[2] = fmaf(cs[0], e0.x, -sn[0] * e0.y);
                            sn[2] = fmaf(sn[0], e0.x, cs[0] * e0.y);
                            cs[3] = fmaf(cs[1], e1.x, -sn[1] * e1.y);
                            sn[3] = fmaf(sn[1], e1.x, cs[1] * e1.y);
                            rotate_pairs(b0, b1, cs[0], sn[0], cs[1], sn[1], ka0, ka1);
                            rotate_pairs(b2, b3, cs[2], sn[2], cs[3], sn[3], kb0, kb1);
                        }
                        const uint32_t a[4] = {b0, b2, b1, b3};
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            if (c & 1) mma16816(sodd[t], a, qb[c][t][0], qb[c][t][1]);
                            else mma16816(sacc[t], a, qb[c][t][0], qb[c][t][1]);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc[t][e] += sodd[t][e];
            }
            // Online softmax over this warp's 16 keys, per head: the thread's two keys,
            // then the 8 row groups (lanes with the same tq).
            float x[NT][4];
            float alpha[NT][2];
            bool rescale = false;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = kw0 + gq + 8 * (e >> 1);
                    const float v = (key < (int)s1) ? sacc[t][e] * scale_log2 : -INFINITY;
                    x[t][e] = v;
                    tmax[e & 1] = fmaxf(tmax[e & 1], v);
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    tmax[hh] = fmaxf(tmax[hh], __shfl_xor_sync(0xffffffffu, tmax[hh], 4));
                    tmax[hh] = fmaxf(tmax[hh], __shfl_xor_sync(0xffffffffu, tmax[hh], 8));
                    tmax[hh] = fmaxf(tmax[hh], __shfl_xor_sync(0xffffffffu, tmax[hh], 16));
                    const bool need = tmax[hh] > m_run[t][hh] + kRescaleThreshold;
                    const float m_new = need ? tmax[hh] : m_run[t][hh];
                    alpha[t][hh] = need ? fast_exp2(m_run[t][hh] - m_new) : 1.f;
                    rescale |= need;
                    m_run[t][hh] = m_new;
                }
            }
            uint32_t pb[NT][2];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float mref0 = m_run[t][0] == -INFINITY ? 0.f : m_run[t][0];
                const float mref1 = m_run[t][1] == -INFINITY ? 0.f : m_run[t][1];
                const float p0 = fast_exp2(x[t][0] - mref0), p1 = fast_exp2(x[t][1] - mref1);
                const float p2 = fast_exp2(x[t][2] - mref0), p3 = fast_exp2(x[t][3] - mref1);
                l_run[t][0] = l_run[t][0] * alpha[t][0] + (p0 + p2);
                l_run[t][1] = l_run[t][1] * alpha[t][1] + (p1 + p3);
                // P^T (keys x heads) into the B fragment of O^T += V^T P^T: an 8x8
                // transpose per key half turns (key gq; heads 2tq, 2tq+1) into
                // (head gq; keys 2tq, 2tq+1).
                pb[t][0] = movmatrix_trans(pack_bf16x2(p0, p1));
                pb[t][1] = movmatrix_trans(pack_bf16x2(p2, p3));
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int i = 0; i < D / 16; ++i)
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        o[i][t][0] *= alpha[t][0];
                        o[i][t][1] *= alpha[t][1];
                        o[i][t][2] *= alpha[t][0];
                        o[i][t][3] *= alpha[t][1];
                    }
            }
            if (kw0 < (int)s1) {
                // O^T += V^T P^T: V rows = this warp's 16 keys, SW128 rows of 64 dims.
                // ldmatrix.trans matrix mi: keys 8*(mi&1).., dims 16dg + 8*(mi>>1)..; the
                // A fragment (dims x keys) of 16 dims is (v0, v2, v1, v3).
                const uint32_t vst = sVa + st * F::VBytes;
                const int mi = lane >> 3, ri = lane & 7;
                const int vkey = 16 * wq + 8 * (mi & 1) + ri;
#pragma unroll
                for (int dg = 0; dg < D / 16; ++dg) {
                    const int d0 = 16 * dg + 8 * (mi >> 1);
                    const uint32_t addr = vst + (d0 / 64) * 8192 + vkey * 128 + ((((d0 & 63) >> 3) ^ (vkey & 7)) << 4);
                    uint32_t v0, v1, v2, v3;
                    ldsm_x4_t(addr, v0, v1, v2, v3);
                    if (kw0 + 15 >= (int)s1) {
                        // Rows past the sequence end may hold anything: P is 0 there, and
                        // 0 * (non-finite) must not reach O.  v0, v2: keys 2tq, 2tq+1; v1, v3: +8.
                        const int kk = kw0 + 2 * tq, se = (int)s1;
                        const uint32_t m01 = (kk < se ? 0x0000FFFFu : 0u) | (kk + 1 < se ? 0xFFFF0000u : 0u);
                        const uint32_t m89 = (kk + 8 < se ? 0x0000FFFFu : 0u) | (kk + 9 < se ? 0xFFFF0000u : 0u);
                        v0 &= m01;
                        v1 &= m89;
                        v2 &= m01;
                        v3 &= m89;
                    }
                    const uint32_t a[4] = {v0, v2, v1, v3};
#pragma unroll
                    for (int t = 0; t < NT; ++t) mma16816(o[dg][t], a, pb[t][0], pb[t][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[st]);
        }
        // Row sums across the 8 row groups, then fold the four warps through shared memory.
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                l_run[t][hh] += __shfl_xor_sync(0xffffffffu, l_run[t][hh], 4);
                l_run[t][hh] += __shfl_xor_sync(0xffffffffu, l_run[t][hh], 8);
                l_run[t][hh] += __shfl_xor_sync(0xffffffffu, l_run[t][hh], 16);
            }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers));  // consumers only: stages are drained
        float *red = reinterpret_cast<float *>(smem);  // reuse the K/V stages: [warp][16 heads][D+2]
        float *mine = red + (size_t)warp * 16 * (D + 2);
#pragma unroll
        for (int i = 0; i < D / 16; ++i)
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int h0 = 8 * t + 2 * tq, d = 16 * i + gq;
                mine[h0 * (D + 2) + 2 + d] = o[i][t][0];
                mine[(h0 + 1) * (D + 2) + 2 + d] = o[i][t][1];
                mine[h0 * (D + 2) + 2 + d + 8] = o[i][t][2];
                mine[(h0 + 1) * (D + 2) + 2 + d + 8] = o[i][t][3];
            }
        if (gq == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int h0 = 8 * t + 2 * tq;
                mine[h0 * (D + 2)] = m_run[t][0];
                mine[h0 * (D + 2) + 1] = l_run[t][0];
                mine[(h0 + 1) * (D + 2)] = m_run[t][1];
                mine[(h0 + 1) * (D + 2) + 1] = l_run[t][1];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers));
        for (int e = threadIdx.x; e < G * D; e += 32 * kConsumers) {
            const int j = e / D, d = e % D;
            float M = -INFINITY;
            for (int wv = 0; wv < kConsumers; ++wv) {
                const float *st = red + ((size_t)wv * 16 + j) * (D + 2);
                if (st[1] > 0.f) M = fmaxf(M, st[0]);
            }
            float l = 0.f, a = 0.f;
            for (int wv = 0; wv < kConsumers; ++wv) {
                const float *st = red + ((size_t)wv * 16 + j) * (D + 2);
                if (st[1] > 0.f) {
                    const float f = fast_exp2(st[0] - M);
                    l += st[1] * f;
                    a += st[2 + d] * f;
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
}

}  // namespace dtc

static cudaError_t make_map_bf16(CUtensorMap *map, const void *base, int rank, const cuuint64_t *dims,
                                 const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return cudaErrorNotSupported;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_decode_tc(const void *q, const void *kc, const void *vc, const int32_t *seqlens, int krot,
                             int layout, const Problem &p, const WindowParams &wp, float *workspace, int split_keys,
                             int nsplit, int *status, uint64_t limit_ns, cudaStream_t s, const PagedKV *paged) {
    CUtensorMap tk, tv;
    const cuuint64_t Dd = (cuuint64_t)p.D, Nm = (cuuint64_t)p.N, Hk = (cuuint64_t)p.Hkv, Bb = (cuuint64_t)p.B;
    const int nhd = (layout == ATFLASH_KV_NHD);
    const bool packed = (layout == ATFLASH_KV_PACKED);
    // Packed K chunks as 128-byte rows: always for pages (a multiple of 64 keys),
    // for a contiguous cache when every chunk holds whole rows.
    const int rows128 = packed && (paged || (p.N % 4) == 0) ? 1 : 0;
    cudaError_t e;
    if (paged) {
        // Pools: V [num_pages][page_size][Hkv][D]; K the same (natural, rotated or
        // not) or packed [num_pages][Hkv][D/16][page_size][16].
        const cuuint64_t P = (cuuint64_t)paged->page_size, NP = (cuuint64_t)paged->num_pages;
        cuuint64_t dv[4] = {Dd, Hk, P, NP};
        cuuint64_t sv[3] = {Dd * 2, Hk * Dd * 2, P * Hk * Dd * 2};
        cuuint32_t boxv[4] = {64, 1, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tv, vc, 4, dv, sv, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
        if (packed) {
            // One chunk of a page: P keys x 32 B contiguous, viewed as P/4 rows of 128 B.
            cuuint64_t dk[3] = {64, P / 4, NP * Hk * (Dd / 16)};
            cuuint64_t sk[2] = {128, P * 32};
            cuuint32_t boxk[3] = {64, dtc::kStageKeys / 4, 1};
            if ((e = make_map_bf16(&tk, kc, 3, dk, sk, boxk, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
        } else {
            cuuint32_t boxk[4] = {16, 1, dtc::kStageKeys, 1};
            if ((e = make_map_bf16(&tk, kc, 4, dv, sv, boxk, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
        }
    } else if (packed) {
        // K: [B*Hkv*D/16][Nmax][16] packed chunks; V: [B][Hkv][Nmax][D].
        if (rows128) {
            cuuint64_t dk[3] = {64, Nm / 4, Bb * Hk * (Dd / 16)};
            cuuint64_t sk[2] = {128, Nm * 32};
            cuuint32_t boxk[3] = {64, dtc::kStageKeys / 4, 1};
            if ((e = make_map_bf16(&tk, kc, 3, dk, sk, boxk, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
        } else {
            cuuint64_t dk[3] = {16, Nm, Bb * Hk * (Dd / 16)};
            cuuint64_t sk[2] = {32, Nm * 32};
            cuuint32_t boxk[3] = {16, dtc::kStageKeys, 1};
            if ((e = make_map_bf16(&tk, kc, 3, dk, sk, boxk, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
        }
        cuuint64_t dims[3] = {Dd, Nm, Bb * Hk};
        cuuint64_t str[2] = {Dd * 2, Nm * Dd * 2};
        cuuint32_t boxv[3] = {64, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tv, vc, 3, dims, str, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    } else if (nhd) {
        cuuint64_t dims[4] = {Dd, Hk, Nm, Bb};
        cuuint64_t str[3] = {Dd * 2, Hk * Dd * 2, Nm * Hk * Dd * 2};
        cuuint32_t boxk[4] = {16, 1, dtc::kStageKeys, 1}, boxv[4] = {64, 1, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tk, kc, 4, dims, str, boxk, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
        if ((e = make_map_bf16(&tv, vc, 4, dims, str, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    } else {
        cuuint64_t dims[3] = {Dd, Nm, Bb * Hk};
        cuuint64_t str[2] = {Dd * 2, Nm * Dd * 2};
        cuuint32_t boxk[3] = {16, dtc::kStageKeys, 1}, boxv[3] = {64, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tk, kc, 3, dims, str, boxk, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
        if ((e = make_map_bf16(&tv, vc, 3, dims, str, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    }
    dim3 grid((unsigned)nsplit, (unsigned)p.Hkv, (unsigned)p.B);
    const int32_t *bt = paged ? paged->block_table : nullptr;
    const int maxp = paged ? paged->max_pages : 0, psz = paged ? paged->page_size : 0;
    const int npool = paged ? paged->num_pages : 0;
#define ATF_DEC_TC_NT(DD, PK, PG, NT)                                                                          \
    do {                                                                                                       \
        const int smem = dtc::Cfg<DD>::Request;                                                                \
        if ((e = cudaFuncSetAttribute(dtc::decode_tc_kernel<DD, PK, PG, NT>,                                  \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)      \
            return e;                                                                                          \
        if ((e = cudaFuncSetAttribute(dtc::decode_tc_kernel<DD, PK, PG, NT>,                                  \
                                      cudaFuncAttributePreferredSharedMemoryCarveout, 100)) != cudaSuccess)    \
            return e;                                                                                          \
        dtc::decode_tc_kernel<DD, PK, PG, NT><<<grid, dtc::kThreads, smem, s>>>(                              \
            tk, tv, q, seqlens, workspace, p.Hq, p.Hkv, nhd, krot, split_keys, nsplit, wp, status, limit_ns,  \
            bt, maxp, psz, npool, rows128);                                                                    \
    } while (0)
#define ATF_DEC_TC(DD, PK, PG)                                                                                 \
    do {                                                                                                       \
        if (p.Hq / p.Hkv <= 8) ATF_DEC_TC_NT(DD, PK, PG, 1);                                                   \
        else ATF_DEC_TC_NT(DD, PK, PG, 2);                                                                     \
    } while (0)
    if (p.D == 128) {
        if (paged) {
            if (packed) ATF_DEC_TC(128, true, true); else ATF_DEC_TC(128, false, true);
        } else {
            if (packed) ATF_DEC_TC(128, true, false); else ATF_DEC_TC(128, false, false);
        }
    } else {
        if (paged) {
            if (packed) ATF_DEC_TC(64, true, true); else ATF_DEC_TC(64, false, true);
        } else {
            if (packed) ATF_DEC_TC(64, true, false); else ATF_DEC_TC(64, false, false);
        }
    }
#undef ATF_DEC_TC
#undef ATF_DEC_TC_NT
    return cudaGetLastError();
}

}  // namespace atf
