// Windowed causal RoPE prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Method ("ATFlash — Per-RoPE-Wavelength Attention Windows", sections "The
// idea" and "Porting to something else"): the query-key contraction axis is a
// sum over frequency pairs; pair r's term is kept only while n - m <= w_r.
// Inside one (query tile, key tile) the distance spans [d_min, d_max], so
//   pairs r <  r_lo   = r*(d_min) are pruned for every cell   -> never loaded,
//   pairs r >= r_full = r*(d_max) are kept for every cell     -> dense MMA,
//   pairs in [r_lo, r_full) are kept for some cells           -> exact per-cell fix-up,
// where r*(d) = min{r : w_r >= d}.  The online softmax is untouched.
//
// Data: Q~ and K~ come pre-rotated and packed by the RoPE pre-pass
// ([bh][D/16][N][16] bf16, 8 pairs per 32-byte chunk, pair-interleaved), V is
// the caller's [B][N][Hkv][D] bf16.  One K-step of the MMA (16 bf16) is one
// chunk = 8 complete pairs, so the dense contraction over pairs >= 8*floor(r_lo/8)
// is a run of whole K-steps; the < 8 fully-pruned pairs at the start of the
// first loaded chunk are zeroed in shared memory before the MMA reads it, and
// the boundary pairs are subtracted per cell where n - m > w_r.
//
// CTA = one (batch*query head, 128-row query tile); 6 warps:
//   warp 0      TMA producer (Q~ once; K~ chunks and V per key tile, 2 stages)
//   warp 1      TMEM owner and MMA issuer (S = Q~ K~^T into one of two TMEM
//               S buffers, O += P V into TMEM O); zeroes pruned pairs
//   warps 2..5  softmax: one TMEM lane quarter (32 query rows) each; fix-up,
//               causal mask, online softmax in the log2 domain, O rescale,
//               P (bf16) to shared memory; epilogue O / l.
// Every mbarrier wait is bounded in time; on expiry the CTA records
// ATFLASH_ERR_TIMEOUT in the device status word, drains its tensor-core work
// and in-flight copies, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace atf {

namespace tc {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kChunkBytes = kBN * 32;  // 128 rows x 16 bf16 (one K-step)

template <int D>
struct Layout {
    static constexpr int C = D / 16;                  // chunks (K-steps) of the QK contraction
    static constexpr int QBytes = C * kChunkBytes;
    static constexpr int KBytes = C * kChunkBytes;
    static constexpr int VBytes = (D / 64) * 16384;   // 128 keys x 64 dims x 2 B per group
    static constexpr int PBytes = 2 * 16384;          // 128 rows x 128 keys bf16, two 64-key groups
    static constexpr int OffQ = 0;
    static constexpr int OffK = OffQ + QBytes;
    static constexpr int OffV = OffK + kStages * KBytes;
    static constexpr int OffP = OffV + kStages * VBytes;
    static constexpr int OffCtl = OffP + PBytes;
    static constexpr int CtlBytes = 2048;
    static constexpr int Total = OffCtl + CtlBytes;
    // At least ~114 KB so that one CTA (and its 512 TMEM columns) owns an SM.
    static constexpr int Request = (Total + 1024 > 120 * 1024) ? Total + 1024 : 120 * 1024;
};

struct Ctl {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full, o_ready, drain;
    uint32_t tmem_base;
    int abort_flag;
    int w[kMaxPairs];
};

// Byte offset of 32-bit word `word` (0..7) of row `row` in a 128 x 32 B chunk
// written by TMA with SWIZZLE_32B (16-byte unit index bit 0 ^= address bit 7).
__device__ __forceinline__ uint32_t sw32_off(int row, int word) {
    return (uint32_t)row * 32u + (((uint32_t)word * 4u) ^ (((uint32_t)row & 4u) << 2));
}

__device__ __forceinline__ int first_kept(const int *w, int H, int64_t d) {
    int lo = 0, hi = H;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)w[mid] >= d) hi = mid; else lo = mid + 1;
    }
    return lo;
}

struct Band {
    int r_lo, r_full;
};
__device__ __forceinline__ Band tile_band(const int *w, int H, int64_t n0, int64_t m0) {
    int64_t dmin = n0 - (m0 + kBN - 1);
    if (dmin < 0) dmin = 0;
    const int64_t dmax = n0 + kBM - 1 - m0;
    Band b;
    b.r_lo = first_kept(w, H, dmin);
    b.r_full = first_kept(w, H, dmax);
    return b;
}

__device__ __forceinline__ bool wait_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ WindowParams wp,
                      void *out, int out_f32, float *lse, int64_t N, int Hq, int Hkv, int *status,
                      uint64_t limit_ns) {
    using L = Layout<D>;
    constexpr int C = L::C;
    constexpr int H = D / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::OffQ;
    uint8_t *sK = smem + L::OffK;
    uint8_t *sV = smem + L::OffV;
    uint8_t *sP = smem + L::OffP;
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + L::OffCtl);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_qt = (int)((N + kBM - 1) / kBM);
    const int qt = num_qt - 1 - (int)blockIdx.x;  // longest query tiles first
    const int bh = blockIdx.y;
    const int b = bh / Hq, hq = bh % Hq, kvh = hq / (Hq / Hkv);
    const int64_t n0 = (int64_t)qt * kBM;
    const int nkt = qt + 1;  // key tiles 0..qt (causal)

    if (threadIdx.x == 0) {
        mbar_init(&ctl->q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->k_full[s], 1);
            mbar_init(&ctl->k_empty[s], 1 + 4);
            mbar_init(&ctl->v_full[s], 1);
            mbar_init(&ctl->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ctl->s_full[s], 1);
            mbar_init(&ctl->s_free[s], 4);
        }
        mbar_init(&ctl->p_full, 4);
        mbar_init(&ctl->o_ready, 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
    }
    for (int r = threadIdx.x; r < H; r += kThreads) ctl->w[r] = wp.w[r];
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int *w = ctl->w;
    WaitCtl wc{&ctl->abort_flag, status, limit_ns, 0};

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int last_k[kStages] = {-1, -1}, last_v[kStages] = {-1, -1};
            mbar_expect_tx(&ctl->q_full, L::QBytes);
            for (int c = 0; c < C; ++c)
                tma_load_3d(sQ + c * kChunkBytes, &tm_q, &ctl->q_full, 0, (int)n0, bh * C + c);
            bool ok = true;
            for (int j = 0; j < nkt && ok; ++j) {
                const int st = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                const int64_t m0 = (int64_t)j * kBN;
                const Band bd = tile_band(w, H, n0, m0);
                const int ca = bd.r_lo >> 3;
                wc.site = 1;
                if (!(ok = mbar_wait(&ctl->k_empty[st], ph ^ 1, wc))) break;
                mbar_expect_tx(&ctl->k_full[st], (uint32_t)(C - ca) * kChunkBytes);
                for (int c = ca; c < C; ++c)
                    tma_load_3d(sK + st * L::KBytes + c * kChunkBytes, &tm_k, &ctl->k_full[st], 0, (int)m0,
                                (b * Hkv + kvh) * C + c);
                last_k[st] = j;
                wc.site = 2;
                if (!(ok = mbar_wait(&ctl->v_empty[st], ph ^ 1, wc))) break;
                mbar_expect_tx(&ctl->v_full[st], L::VBytes);
                for (int gidx = 0; gidx < D / 64; ++gidx)
                    tma_load_4d(sV + st * L::VBytes + gidx * 16384, &tm_v, &ctl->v_full[st], gidx * 64, kvh,
                                (int)m0, b);
                last_v[st] = j;
            }
            if (!ok) {
                // Let every copy this thread started land before the CTA exits.
                wait_drain(&ctl->q_full, 0, limit_ns);
                for (int s = 0; s < kStages; ++s) {
                    if (last_k[s] >= 0) wait_drain(&ctl->k_full[s], (last_k[s] >> 1) & 1, limit_ns);
                    if (last_v[s] >= 0) wait_drain(&ctl->v_full[s], (last_v[s] >> 1) & 1, limit_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
        const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
        const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
        bool ok = true;
        wc.site = 3;
        ok = mbar_wait_warp(&ctl->q_full, 0, wc);
        auto issue_pv = [&](int jj) -> bool {
            const int st = jj & 1;
            wc.site = 4;
            if (!mbar_wait_warp(&ctl->v_full[st], (jj >> 1) & 1, wc)) return false;
            wc.site = 5;
            if (!mbar_wait_warp(&ctl->p_full, jj & 1, wc)) return false;
            if (lane == 0) {
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < kBN / 16; ++t) {
                    // A = P keys [16t, 16t+16): K-major SW128, 64-key groups 16 KB apart.
                    const uint64_t da = smem_desc(sPa + (t >> 2) * 16384 + (t & 3) * 32, 16, 1024, kSwizzle128B);
                    // B = V rows [16t, 16t+16): MN-major SW128, 64-dim groups 16 KB apart.
                    const uint64_t db =
                        smem_desc(sVa + st * L::VBytes + t * 2048, 16384, 1024, kSwizzle128B);
                    umma_bf16_ss(tmem + 256, da, db, idesc_pv, (jj > 0 || t > 0) ? 1u : 0u);
                }
                umma_commit(&ctl->o_ready);
                umma_commit(&ctl->v_empty[st]);
            }
            __syncwarp();
            return true;
        };
        for (int j = 0; j < nkt && ok; ++j) {
            const int st = j & 1, sb = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            const Band bd = tile_band(w, H, (int64_t)qt * kBM, (int64_t)j * kBN);
            const int ca = bd.r_lo >> 3;
            wc.site = 6;
            if (!(ok = mbar_wait_warp(&ctl->k_full[st], ph, wc))) break;
            if ((bd.r_lo & 7) && ca < C) {
                // Pairs [8*ca, r_lo) are pruned for every cell of this tile: zero them
                // in the landed K~ chunk so the dense MMA over whole chunks skips them.
                uint8_t *chunk = sK + st * L::KBytes + ca * kChunkBytes;
                for (int row = lane; row < kBN; row += 32)
                    for (int p = 8 * ca; p < bd.r_lo; ++p)
                        *reinterpret_cast<uint32_t *>(chunk + sw32_off(row, p & 7)) = 0u;
                fence_proxy_async_smem();
            }
            __syncwarp();
            wc.site = 7;
            if (!(ok = mbar_wait_warp(&ctl->s_free[sb], ph ^ 1, wc))) break;
            if (lane == 0) {
                tc_fence_after();
                for (int c = ca; c < C; ++c) {
                    const uint64_t da = smem_desc(sQa + c * kChunkBytes, 16, 256, kSwizzle32B);
                    const uint64_t db = smem_desc(sKa + st * L::KBytes + c * kChunkBytes, 16, 256, kSwizzle32B);
                    umma_bf16_ss(tmem + sb * 128, da, db, idesc_qk, c > ca ? 1u : 0u);
                }
                umma_commit(&ctl->s_full[sb]);
                umma_commit(&ctl->k_empty[st]);
            }
            __syncwarp();
            if (j > 0 && !(ok = issue_pv(j - 1))) break;
        }
        if (ok) ok = issue_pv(nkt - 1);
    } else {
        // ------------------------------------------------------------- softmax
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int64_t n = n0 + row;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
        float mrun = -INFINITY, lrun = 0.f;
        wc.site = 11;
        bool ok = mbar_wait_warp(&ctl->q_full, 0, wc);  // Q~ rows are read for the boundary fix-up
        for (int j = 0; j < nkt && ok; ++j) {
            const int st = j & 1, sb = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            const int64_t m0 = (int64_t)j * kBN;
            const Band bd = tile_band(w, H, n0, m0);
            float s[kBN];
            wc.site = 8;
            if (!(ok = mbar_wait_warp(&ctl->s_full[sb], ph, wc))) break;
            tc_fence_after();
            if ((bd.r_lo >> 3) < C) {
#pragma unroll
                for (int cc = 0; cc < kBN / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tl + sb * 128 + cc * 32, r);
                    tmem_ld_wait(r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < kBN; ++i) s[i] = 0.f;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->s_free[sb]);
            // Boundary pairs: the dense MMA included them; remove them from the
            // cells where the distance exceeds the pair's window.
            if (bd.r_lo < bd.r_full) {
                wc.site = 12;  // the K~ chunk landed long ago; this orders its TMA writes before our reads
                if (!(ok = mbar_wait_warp(&ctl->k_full[st], ph, wc))) break;
            }
            for (int r = bd.r_lo; r < bd.r_full; ++r) {
                const int64_t lim = n - m0 - (int64_t)w[r];  // cells jj < lim have n - m > w_r
                if (lim > 0) {
                    const uint32_t qw = *reinterpret_cast<const uint32_t *>(sQ + (r >> 3) * kChunkBytes +
                                                                            sw32_off(row, r & 7));
                    const float qa = bf16lo(qw), qb = bf16hi(qw);
                    const uint8_t *kch = sK + st * L::KBytes + (r >> 3) * kChunkBytes;
#pragma unroll
                    for (int jj = 0; jj < kBN; ++jj) {
                        if (jj < lim) {
                            const uint32_t kw = *reinterpret_cast<const uint32_t *>(kch + sw32_off(jj, r & 7));
                            s[jj] -= qa * bf16lo(kw) + qb * bf16hi(kw);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->k_empty[st]);
            // Causal mask (diagonal tile only), scale to log2 units, running max.
            float mx = mrun;
#pragma unroll
            for (int jj = 0; jj < kBN; ++jj) {
                float x = s[jj] * scale_log2;
                if (m0 + jj > n) x = -INFINITY;
                s[jj] = x;
                mx = fmaxf(mx, x);
            }
            const float alpha = fast_exp2(mrun - mx);
            float rs = 0.f;
#pragma unroll
            for (int jj = 0; jj < kBN; ++jj) {
                const float p = fast_exp2(s[jj] - mx);
                s[jj] = p;
                rs += p;
            }
            lrun = lrun * alpha + rs;
            mrun = mx;
            if (j > 0) {
                wc.site = 9;
                if (!(ok = mbar_wait_warp(&ctl->o_ready, (j - 1) & 1, wc))) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(tl + 256 + cc * 32, r);
                        tmem_ld_wait(r);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st_32x32b_x32(tl + 256 + cc * 32, r);
                    }
                    tmem_st_wait();
                }
            }
            // P (bf16) to shared memory, K-major SW128: 64-key groups of 16 KB, 128 B rows.
#pragma unroll
            for (int kk = 0; kk < kBN / 8; ++kk) {
                uint4 v4;
                v4.x = pack_bf16x2(s[kk * 8 + 0], s[kk * 8 + 1]);
                v4.y = pack_bf16x2(s[kk * 8 + 2], s[kk * 8 + 3]);
                v4.z = pack_bf16x2(s[kk * 8 + 4], s[kk * 8 + 5]);
                v4.w = pack_bf16x2(s[kk * 8 + 6], s[kk * 8 + 7]);
                const uint32_t off = (uint32_t)(kk >> 3) * 16384u + (uint32_t)row * 128u +
                                     ((((uint32_t)kk & 7u) ^ ((uint32_t)row & 7u)) << 4);
                *reinterpret_cast<uint4 *>(sP + off) = v4;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->p_full);
        }
        if (ok) {
            wc.site = 10;
            ok = mbar_wait_warp(&ctl->o_ready, (nkt - 1) & 1, wc);
        }
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / lrun;
            const size_t o = ((size_t)((int64_t)b * N + n) * Hq + hq) * D;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tl + 256 + cc * 32, r);
                tmem_ld_wait(r);
                if (n < N) {
                    if (out_f32) {
                        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + o + cc * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                                 __uint_as_float(r[4 * i + 2]) * inv,
                                                 __uint_as_float(r[4 * i + 3]) * inv);
                    } else {
                        uint4 *dst =
                            reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(out) + o + cc * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(
                                pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv, __uint_as_float(r[8 * i + 1]) * inv),
                                pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv),
                                pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv),
                                pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv));
                    }
                }
            }
            if (lse && n < N) lse[((size_t)b * Hq + hq) * N + n] = (mrun + __log2f(lrun)) * 0.69314718055994531f;
        }
    }

    // Teardown: every tensor-core operation must be complete before TMEM is freed.
    __syncthreads();
    if (warp == 1) {
        if (lane == 0) {
            umma_commit(&ctl->drain);
            wait_drain(&ctl->drain, 0, limit_ns);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace tc

static cudaError_t make_map(CUtensorMap *map, void *base, int rank, const cuuint64_t *dims,
                            const cuuint64_t *strides_bytes, const cuuint32_t *box, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return cudaErrorNotSupported;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, base, dims, strides_bytes, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_prefill_tc(const void *qpack, const void *kpack, const void *v, void *out, int out_f32,
                              float *lse, const Problem &p, const WindowParams &wp, int *status,
                              uint64_t wait_limit_ns, cudaStream_t s) {
    const int C = p.D / 16;
    CUtensorMap tq, tk, tv;
    {
        cuuint64_t dims[3] = {16, (cuuint64_t)p.N, (cuuint64_t)p.B * p.Hq * C};
        cuuint64_t str[2] = {32, (cuuint64_t)p.N * 32};
        cuuint32_t box[3] = {16, tc::kBM, 1};
        cudaError_t e = make_map(&tq, const_cast<void *>(qpack), 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B);
        if (e != cudaSuccess) return e;
    }
    {
        cuuint64_t dims[3] = {16, (cuuint64_t)p.N, (cuuint64_t)p.B * p.Hkv * C};
        cuuint64_t str[2] = {32, (cuuint64_t)p.N * 32};
        cuuint32_t box[3] = {16, tc::kBN, 1};
        cudaError_t e = make_map(&tk, const_cast<void *>(kpack), 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B);
        if (e != cudaSuccess) return e;
    }
    {
        cuuint64_t dims[4] = {(cuuint64_t)p.D, (cuuint64_t)p.Hkv, (cuuint64_t)p.N, (cuuint64_t)p.B};
        cuuint64_t str[3] = {(cuuint64_t)p.D * 2, (cuuint64_t)p.Hkv * p.D * 2, (cuuint64_t)p.N * p.Hkv * p.D * 2};
        cuuint32_t box[4] = {64, 1, tc::kBN, 1};
        cudaError_t e = make_map(&tv, const_cast<void *>(v), 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
    }
    const int num_qt = (int)((p.N + tc::kBM - 1) / tc::kBM);
    dim3 grid((unsigned)num_qt, (unsigned)(p.B * p.Hq));
    cudaError_t e;
    if (p.D == 128) {
        const int smem = tc::Layout<128>::Request;
        e = cudaFuncSetAttribute(tc::prefill_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        tc::prefill_tc_kernel<128><<<grid, tc::kThreads, smem, s>>>(tq, tk, tv, wp, out, out_f32, lse, p.N, p.Hq,
                                                                    p.Hkv, status, wait_limit_ns);
    } else if (p.D == 64) {
        const int smem = tc::Layout<64>::Request;
        e = cudaFuncSetAttribute(tc::prefill_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        tc::prefill_tc_kernel<64><<<grid, tc::kThreads, smem, s>>>(tq, tk, tv, wp, out, out_f32, lse, p.N, p.Hq,
                                                                   p.Hkv, status, wait_limit_ns);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace atf
