// Split-KV windowed decode on tensor cores (bf16 caches).
//
// One CTA = one split of one (sequence, KV head): its G = Hq/Hkv query heads
// are the M rows (padded to 16) of mma.sync m16n8k16 tiles, keys are N.  The
// method ("ATFlash — Per-RoPE-Wavelength Attention Windows", "The idea" and
// "Numbers": the window is a condition on which K elements are loaded):
// for a key at distance d = L-1-m only pairs r >= r*(d) are kept, so
//   - the producer warp streams 64-key stages with TMA, loading for K only the
//     8-pair chunks that some key of the stage keeps, and all of V;
//   - each consumer warp takes 16 keys of a stage: ldmatrix puts complete
//     frequency pairs (r, r+D/2) of one key into one thread, which rotates them
//     (unless the cache is pre-rotated) and zeroes the pairs its key prunes;
//   - S = Q~ K~^T, the online softmax and O += P V stay in registers.
// The contraction order inside a K-step is [8 low-half dims, 8 high-half dims]
// for both Q~ and K~, so every dot product is unchanged.
//
// Angles: the producer writes, per stage, the base angle stage_start*theta_r
// reduced mod 2*pi in fp64; a key at offset i adds i*theta_r (i < 64) in fp32,
// reduces once more and takes sin/cos on [-pi, pi].
//
// Packed cache (ATFLASH_KV_PACKED): K already rotated and stored as the RoPE
// pre-pass writes it, [B*Hkv][D/16][Nmax][16] with 8 frequency pairs per 32-byte
// chunk.  A pruned chunk of 64 keys is then 2 KB of HBM that is never fetched;
// in the natural layouts a key's pruned dims are a short prefix of each 128-byte
// half and HBM's access granularity fetches them anyway.
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
    static constexpr int kStages = 3;
    static constexpr int H = D / 2;
    static constexpr int C = D / 16;                   // chunks of 8 pairs
    static constexpr int KBytes = C * 2 * 1024;        // [c][half][64 keys][8 dims] bf16
    static constexpr int VBytes = (D / 64) * 8192;     // [D/64][64 keys][64 dims] bf16, SW128
    static constexpr int OffK = 0;
    static constexpr int OffV = OffK + kStages * KBytes;
    static constexpr int OffBase = OffV + kStages * VBytes;      // [stage][H] float
    static constexpr int OffQ = OffBase + kStages * H * 4;       // [16][D] float, rotated queries
    static constexpr int OffBar = OffQ + 16 * D * 4;
    static constexpr int Total = OffBar + 256;
    static constexpr int Request = Total + 1024;
};

constexpr int kMaxStages = 8;
struct Bars {
    uint64_t full[kMaxStages], empty[kMaxStages];
    int abort_flag;
};

__device__ __forceinline__ int first_kept_pair(const int *w, int H, int64_t d) {
    int lo = 0, hi = H;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)w[mid] >= d) hi = mid; else lo = mid + 1;
    }
    return lo;
}

// r*(d) as d shrinks: keys of later stages are nearer the query, so the first
// kept pair only moves down; amortised O(1) per stage.
__device__ __forceinline__ int walk_down(const int *w, int r, int d) {
    while (r > 0 && w[r - 1] >= d) --r;
    return r;
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
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// The natural-layout kernel (rotation at load) is asked for two CTAs per SM, which
// lets the compiler use more registers than its default; the packed kernel keeps
// the default, which measured faster.
// kPaged: K and V live in pages of page_size tokens (a multiple of the 64-key
// stage), page block_table[b * max_pages + i] holding keys i*page_size.. of
// sequence b; the maps index pages along their outermost axis.
template <int D, bool kPacked, bool kPaged>
__global__ void __launch_bounds__(kThreads, kPacked ? 0 : 2) decode_tc_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const void *q_,
    const int32_t *__restrict__ seqlens, float *__restrict__ ws, int Hq, int Hkv, int nhd, int krot, int split_keys,
    int nsplit, const __grid_constant__ WindowParams wp, int *status, uint64_t limit_ns,
    const int32_t *__restrict__ block_table, int max_pages, int page_size, int num_pages) {
    using F = Cfg<D>;
    constexpr int H = F::H, C = F::C;
    constexpr int kStages = F::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + F::OffK;
    uint8_t *sV = smem + F::OffV;
    float *sBase = reinterpret_cast<float *>(smem + F::OffBase);
    float *sQ = reinterpret_cast<float *>(smem + F::OffQ);
    Bars *bars = reinterpret_cast<Bars *>(smem + F::OffBar);
    __shared__ int sw[kMaxPairs];
    __shared__ float sTheta[kMaxPairs];

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
        sQ[j * D + r] = xr;
        sQ[j * D + r + H] = xh;
    }
    __syncthreads();
    WaitCtl wc{&bars->abort_flag, status, limit_ns, 20};

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        int last[kMaxStages];
        for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
        for (int it = 0; it < nstage && ok; ++it) {
            const int st = it % kStages;
            const int64_t k0 = s0 + (int64_t)it * kStageKeys;
            int64_t k1 = k0 + kStageKeys - 1;
            if (k1 > s1 - 1) k1 = s1 - 1;
            const int c_lo = first_kept_pair(sw, H, (L - 1) - k1) >> 3;  // nearest key keeps the most
            if (!(ok = mbar_wait_warp(&bars->empty[st], ((it / kStages) & 1) ^ 1, wc))) break;
            for (int r = lane; r < H; r += 32) {
                double turns = (double)k0 * wp.theta[r] * 0.15915494309189533576888376337251;
                turns -= rint(turns);
                sBase[st * H + r] = (float)(turns * 6.283185307179586476925286766559);
            }
            __syncwarp();
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)(C - c_lo) * 2048u + (uint32_t)F::VBytes;
                mbar_expect_tx(&bars->full[st], bytes);
                uint8_t *kst = sK + st * F::KBytes;
                if constexpr (kPaged) {
                    // A stage never straddles a page (page_size is a multiple of 64).  A
                    // page index past the table row or an id outside the pool becomes -1,
                    // which the maps treat as out of bounds (zero fill, no access).
                    const int64_t pi = k0 / page_size;
                    int page = pi < max_pages ? block_table[(size_t)b * max_pages + pi] : -1;
                    if (page < 0 || page >= num_pages) page = -1;
                    const int kk = (int)(k0 % page_size);
                    if (kPacked) {
                        for (int c = c_lo; c < C; ++c)
                            tma_load_3d(kst + c * 2048, &tm_k, &bars->full[st], 0, kk, (page * Hkv + g) * C + c);
                    } else {
                        for (int c = c_lo; c < C; ++c)
                            for (int hf = 0; hf < 2; ++hf)
                                tma_load_4d(kst + (2 * c + hf) * 1024, &tm_k, &bars->full[st], hf * H + 8 * c, g, kk,
                                            page);
                    }
                    for (int gi = 0; gi < D / 64; ++gi)
                        tma_load_4d(sV + st * F::VBytes + gi * 8192, &tm_v, &bars->full[st], 64 * gi, g, kk, page);
                } else if (kPacked) {
                    for (int c = c_lo; c < C; ++c)
                        tma_load_3d(kst + c * 2048, &tm_k, &bars->full[st], 0, (int)k0, (b * Hkv + g) * C + c);
                } else {
                    for (int c = c_lo; c < C; ++c)
                        for (int hf = 0; hf < 2; ++hf) {
                            uint8_t *dst = kst + (2 * c + hf) * 1024;
                            const int x = hf * H + 8 * c;
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
        const int gq = lane >> 2, tq = lane & 3;  // mma fragment row group / column pair
        // Q~ A-fragments per chunk: k-order [dims 8c..8c+7, dims H+8c..H+8c+7].
        uint32_t qa[C][4];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (kPacked) {
                // k-order of a packed chunk: (pair 8c+e/2, component e%2).
                const int pa = 8 * c + tq, pb = pa + 4;
                qa[c][0] = pack_bf16x2(sQ[gq * D + pa], sQ[gq * D + pa + H]);
                qa[c][1] = pack_bf16x2(sQ[(gq + 8) * D + pa], sQ[(gq + 8) * D + pa + H]);
                qa[c][2] = pack_bf16x2(sQ[gq * D + pb], sQ[gq * D + pb + H]);
                qa[c][3] = pack_bf16x2(sQ[(gq + 8) * D + pb], sQ[(gq + 8) * D + pb + H]);
            } else {
                const int lo = 8 * c + 2 * tq, hi = H + 8 * c + 2 * tq;
                qa[c][0] = pack_bf16x2(sQ[gq * D + lo], sQ[gq * D + lo + 1]);
                qa[c][1] = pack_bf16x2(sQ[(gq + 8) * D + lo], sQ[(gq + 8) * D + lo + 1]);
                qa[c][2] = pack_bf16x2(sQ[gq * D + hi], sQ[gq * D + hi + 1]);
                qa[c][3] = pack_bf16x2(sQ[(gq + 8) * D + hi], sQ[(gq + 8) * D + hi + 1]);
            }
        }
        const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
        float o[D / 8][4];
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows gq, gq+8
        const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
        bool ok = true;
        // Positions fit in int32 (Nmax <= 2^31 - 1).  Walk pointers for r*(d) of the
        // stage's nearest key, this warp's nearest key and this warp's farthest key.
        const int Lq = (int)L - 1;
        int r_stage = H, r_warp = H, r_keep = H;
        const int grp = warp / kWarpsPerStage, wq = warp % kWarpsPerStage;
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
            float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            float sodd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            if (kw0 < (int)s1) {
                r_warp = walk_down(sw, r_warp, Lq - kw1);
                r_keep = walk_down(sw, r_keep, Lq - kw0);
                const int c_warp = r_warp >> 3;
                // Keys of this thread's fragments: n-tile 0 -> kw0 + gq, n-tile 1 -> kw0 + 8 + gq.
                const int da = Lq - (kw0 + gq), db = da - 8;
                const float fa = (float)(16 * wq + gq), fb = fa + 8.f;
                const uint32_t kst = sKa + st * F::KBytes;
                const int mi = lane >> 3, ri = lane & 7;
                const int c_keep = (r_keep + 7) >> 3;
                if constexpr (kPacked) {
                    const int c_begin = c_warp > c_stage ? c_warp : c_stage;
                    // All of this warp's K fragments first (independent shared-memory loads in
                    // flight together), then the masks and the MMAs.
                    uint32_t kb[C][4];
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        if (c < c_begin) continue;
                        // 64 keys x 32 B per chunk, SWIZZLE_32B; matrix mi: keys +8*(mi>>1), bytes 16*(mi&1).
                        const int key = 16 * wq + 8 * (mi >> 1) + ri;
                        ldsm_x4(kst + c * 2048 + key * 32 + ((16 * (mi & 1)) ^ ((key & 4) << 2)), kb[c][0], kb[c][1],
                                kb[c][2], kb[c][3]);
                    }
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        if (c < c_begin) continue;
                        // Chunks from c_keep on are kept by every key of this warp: no masking.
                        const bool masked = c < c_keep;
                        uint32_t b0 = kb[c][0], b1 = kb[c][1], b2 = kb[c][2], b3 = kb[c][3];
                        if (masked) {
                            const int p0 = 8 * c + tq, p1 = p0 + 4;
                            const int w0 = sw[p0], w1 = sw[p1];
                            b0 = (da <= w0) ? b0 : 0u;
                            b1 = (da <= w1) ? b1 : 0u;
                            b2 = (db <= w0) ? b2 : 0u;
                            b3 = (db <= w1) ? b3 : 0u;
                        }
                        // Two independent accumulation chains (chunk parity).
                        if (c & 1) {
                            mma16816(sodd[0], qa[c], b0, b1);
                            mma16816(sodd[1], qa[c], b2, b3);
                        } else {
                            mma16816(sacc[0], qa[c], b0, b1);
                            mma16816(sacc[1], qa[c], b2, b3);
                        }
                    }
                } else {
                    for (int c = (c_warp > c_stage ? c_warp : c_stage); c < C; ++c) {
                        const bool masked = c < c_keep;
                        uint32_t b0, b1, b2, b3;
                        if (kPacked) {
                            // 64 keys x 32 B per chunk, SWIZZLE_32B; matrix mi: keys +8*(mi>>1), bytes 16*(mi&1).
                            const int key = 16 * wq + 8 * (mi >> 1) + ri;
                            ldsm_x4(kst + c * 2048 + key * 32 + ((16 * (mi & 1)) ^ ((key & 4) << 2)), b0, b1, b2, b3);
                            if (masked) {
                                const int p0 = 8 * c + tq, p1 = p0 + 4;
                                const int w0 = sw[p0], w1 = sw[p1];
                                b0 = (da <= w0) ? b0 : 0u;
                                b1 = (da <= w1) ? b1 : 0u;
                                b2 = (db <= w0) ? b2 : 0u;
                                b3 = (db <= w1) ? b3 : 0u;
                            }
                        } else {
                            const uint32_t addr = kst + (2 * c + (mi & 1)) * 1024 + (16 * wq + 8 * (mi >> 1) + ri) * 16;
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
                                float ang[4] = {fmaf(fa, th0, base0), fmaf(fa, th1, base1), fmaf(fb, th0, base0),
                                                fmaf(fb, th1, base1)};
                                float cs[4], sn[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const float turns = rintf(ang[u] * 0.15915494309189533577f);
                                    const float x = fmaf(-turns, 6.283185307179586477f, ang[u]);
                                    __sincosf(x, &sn[u], &cs[u]);
                                }
                                rotate_pairs(b0, b1, cs[0], sn[0], cs[1], sn[1], ka0, ka1);
                                rotate_pairs(b2, b3, cs[2], sn[2], cs[3], sn[3], kb0, kb1);
                            }
                        }
                        // Two independent accumulation chains (chunk parity).
                        if (c & 1) {
                            mma16816(sodd[0], qa[c], b0, b1);
                            mma16816(sodd[1], qa[c], b2, b3);
                        } else {
                            mma16816(sacc[0], qa[c], b0, b1);
                            mma16816(sacc[1], qa[c], b2, b3);
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sacc[0][e] += sodd[0][e];
                    sacc[1][e] += sodd[1][e];
                }
            }
            // Online softmax over this warp's 16 keys; rows gq (sacc[.][0..1]) and gq+8 ([2..3]).
            float x[2][4];
            float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = kw0 + 8 * nt + 2 * tq + (e & 1);
                    const float v = (key < (int)s1) ? sacc[nt][e] * scale_log2 : -INFINITY;
                    x[nt][e] = v;
                    tmax[e >> 1] = fmaxf(tmax[e >> 1], v);
                }
            float alpha[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xffffffffu, tmax[rr], 1));
                tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xffffffffu, tmax[rr], 2));
                const bool need = tmax[rr] > m_run[rr] + kRescaleThreshold;
                const float m_new = need ? tmax[rr] : m_run[rr];
                alpha[rr] = need ? fast_exp2(m_run[rr] - m_new) : 1.f;
                m_run[rr] = m_new;
            }
            float p[2][4];
            const float mref[2] = {m_run[0] == -INFINITY ? 0.f : m_run[0], m_run[1] == -INFINITY ? 0.f : m_run[1]};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) p[nt][e] = fast_exp2(x[nt][e] - mref[e >> 1]);
            l_run[0] = l_run[0] * alpha[0] + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
            l_run[1] = l_run[1] * alpha[1] + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
            if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int i = 0; i < D / 8; ++i) {
                    o[i][0] *= alpha[0];
                    o[i][1] *= alpha[0];
                    o[i][2] *= alpha[1];
                    o[i][3] *= alpha[1];
                }
            }
            uint32_t pa[4];
            pa[0] = pack_bf16x2(p[0][0], p[0][1]);
            pa[1] = pack_bf16x2(p[0][2], p[0][3]);
            pa[2] = pack_bf16x2(p[1][0], p[1][1]);
            pa[3] = pack_bf16x2(p[1][2], p[1][3]);
            if (kw0 < (int)s1) {
                // O += P V: V rows = this warp's 16 keys, SW128 rows of 64 dims.
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
                        // 0 * (non-finite) must not reach O.  b0b1: keys 2tq, 2tq+1; b2b3: +8.
                        const int kk = kw0 + 2 * tq, se = (int)s1;
                        const uint32_t m01 = (kk < se ? 0x0000FFFFu : 0u) | (kk + 1 < se ? 0xFFFF0000u : 0u);
                        const uint32_t m89 = (kk + 8 < se ? 0x0000FFFFu : 0u) | (kk + 9 < se ? 0xFFFF0000u : 0u);
                        v0 &= m01;
                        v1 &= m89;
                        v2 &= m01;
                        v3 &= m89;
                    }
                    mma16816(o[2 * dg], pa, v0, v1);
                    mma16816(o[2 * dg + 1], pa, v2, v3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[st]);
        }
        // Full row sums across the quad, then fold the four warps through shared memory.
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
            l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers));  // consumers only: stages are drained
        float *red = reinterpret_cast<float *>(smem);  // reuse the K/V stages: [warp][16][D+2]
        float *mine = red + (size_t)warp * 16 * (D + 2);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            const int col = 8 * i + 2 * tq;
            mine[gq * (D + 2) + 2 + col] = o[i][0];
            mine[gq * (D + 2) + 3 + col] = o[i][1];
            mine[(gq + 8) * (D + 2) + 2 + col] = o[i][2];
            mine[(gq + 8) * (D + 2) + 3 + col] = o[i][3];
        }
        if (tq == 0) {
            mine[gq * (D + 2)] = m_run[0];
            mine[gq * (D + 2) + 1] = l_run[0];
            mine[(gq + 8) * (D + 2)] = m_run[1];
            mine[(gq + 8) * (D + 2) + 1] = l_run[1];
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
            cuuint64_t dk[3] = {16, P, NP * Hk * (Dd / 16)};
            cuuint64_t sk[2] = {32, P * 32};
            cuuint32_t boxk[3] = {16, dtc::kStageKeys, 1};
            if ((e = make_map_bf16(&tk, kc, 3, dk, sk, boxk, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
        } else {
            cuuint32_t boxk[4] = {8, 1, dtc::kStageKeys, 1};
            if ((e = make_map_bf16(&tk, kc, 4, dv, sv, boxk, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess) return e;
        }
    } else if (packed) {
        // K: [B*Hkv*D/16][Nmax][16] packed chunks; V: [B][Hkv][Nmax][D].
        cuuint64_t dk[3] = {16, Nm, Bb * Hk * (Dd / 16)};
        cuuint64_t sk[2] = {32, Nm * 32};
        cuuint32_t boxk[3] = {16, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tk, kc, 3, dk, sk, boxk, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
        cuuint64_t dims[3] = {Dd, Nm, Bb * Hk};
        cuuint64_t str[2] = {Dd * 2, Nm * Dd * 2};
        cuuint32_t boxv[3] = {64, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tv, vc, 3, dims, str, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    } else if (nhd) {
        cuuint64_t dims[4] = {Dd, Hk, Nm, Bb};
        cuuint64_t str[3] = {Dd * 2, Hk * Dd * 2, Nm * Hk * Dd * 2};
        cuuint32_t boxk[4] = {8, 1, dtc::kStageKeys, 1}, boxv[4] = {64, 1, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tk, kc, 4, dims, str, boxk, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess) return e;
        if ((e = make_map_bf16(&tv, vc, 4, dims, str, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    } else {
        cuuint64_t dims[3] = {Dd, Nm, Bb * Hk};
        cuuint64_t str[2] = {Dd * 2, Nm * Dd * 2};
        cuuint32_t boxk[3] = {8, dtc::kStageKeys, 1}, boxv[3] = {64, dtc::kStageKeys, 1};
        if ((e = make_map_bf16(&tk, kc, 3, dims, str, boxk, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess) return e;
        if ((e = make_map_bf16(&tv, vc, 3, dims, str, boxv, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    }
    dim3 grid((unsigned)nsplit, (unsigned)p.Hkv, (unsigned)p.B);
    const int32_t *bt = paged ? paged->block_table : nullptr;
    const int maxp = paged ? paged->max_pages : 0, psz = paged ? paged->page_size : 0;
    const int npool = paged ? paged->num_pages : 0;
#define ATF_DEC_TC(DD, PK, PG)                                                                                 \
    do {                                                                                                       \
        const int smem = dtc::Cfg<DD>::Request;                                                                \
        if ((e = cudaFuncSetAttribute(dtc::decode_tc_kernel<DD, PK, PG>,                                      \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)      \
            return e;                                                                                          \
        dtc::decode_tc_kernel<DD, PK, PG><<<grid, dtc::kThreads, smem, s>>>(                                  \
            tk, tv, q, seqlens, workspace, p.Hq, p.Hkv, nhd, krot, split_keys, nsplit, wp, status, limit_ns,  \
            bt, maxp, psz, npool);                                                                             \
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
    return cudaGetLastError();
}

}  // namespace atf
