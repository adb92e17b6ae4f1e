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
// first loaded chunk are zeroed in shared memory before the MMA reads them,
// and the boundary pairs are subtracted per cell where n - m > w_r.
//
// CTA = one 128-row query tile of TWO query heads of the same GQA group: both
// heads read the same K/V tiles at the same distances, so they share every
// load, every pruned-chunk decision and every boundary pair, while their two
// softmax warps ping-pong with the tensor core.  20 warps:
//   warps 0-7 / 8-15 softmax of head 0 / head 1: warp 4 hc + q4 of a head takes
//                    TMEM lane quarter q4 (32 query rows) and S columns
//                    [64 hc, 64 hc + 64) of the key tile; the two warps of a row
//                    exchange their partial row maxima once per tile (and their
//                    partial sums at the end).  Boundary fix-up, causal mask,
//                    online softmax in the log2 domain, P (bf16) into TMEM, O
//                    rescale (only when the running max grows by more than 2^8)
//                    and the epilogue, each on the warp's half of the columns
//   warp 16          TMA producer (Q~ once; K~ chunks and V per key tile)
//   warp 17          TMEM owner and QK issuer: S_h = Q~_h K~^T (smem x smem)
//   warp 18          zeroes the fully-pruned pairs of the first loaded K~ chunk
//                    and stages the tile's boundary pairs as fp32 for the fix-up
//   warp 19          PV issuer: O_h += P_h V (P from TMEM, V from smem)
// For D = 64 with no pair pruned anywhere the launcher takes the one-head form
// instead: 8 warps (softmax 0-3 over whole rows, then producer, QK, fix-up,
// PV), 256 TMEM columns and two K/V stages, so that two CTAs share an SM.
// TMEM columns: as in Cfg below.
// Every mbarrier wait is bounded in time; on expiry the CTA records
// ATFLASH_ERR_TIMEOUT in the device status word, lets its copies land, drains
// its tensor-core work, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace atf {

namespace tc {

constexpr int kBM = 128;
constexpr int kBN = 128;
// NH query heads per CTA (2: one CTA per SM, the heads share every K/V tile; 1:
// two CTAs per SM, which run out of phase so one CTA's exp2 pass overlaps the
// other's loads, waits and stores).  CH softmax warps share each row's 128
// columns (2: with window pruning, where the boundary subtraction and the
// shorter per-warp passes pay for a per-tile exchange of partial row maxima;
// 1: whole rows, which measured faster without pruning).  Warps: 4*NH*CH
// softmax, then producer, QK issuer, fix-up and PV issuer.  Registers: every
// thread gets LaunchRegs at launch; the four other warps drop to OtherRegs and
// the softmax warps rise to SoftRegs, which must fit the launch's total
// (checked here and, against the compiled kernel, at launch).
template <int NH, int CH>
struct Warps {
    static constexpr int Soft = 4 * NH * CH;
    static constexpr int Threads = 32 * (Soft + 4);
    static constexpr int Producer = Soft, Mma = Soft + 1, Fix = Soft + 2, Pv = Soft + 3;
    static constexpr int LaunchRegs = 65536 / (Threads * (3 - NH)) / 8 * 8;
    static constexpr int OtherRegs = (NH == 2 && CH == 1) ? 96 : 56;
    static constexpr int SoftRegs = CH == 2 ? 104 : 200;
    static_assert(NH == 2 || CH == 1, "the one-head form keeps whole rows");
    static_assert(32 * Soft * SoftRegs + 128 * OtherRegs <= Threads * LaunchRegs, "register split exceeds the launch");
};
constexpr uint32_t kChunkBytes = kBN * 32;  // 128 rows x 16 bf16 (one K-step)
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8
// Boundary pairs whose key values the fix-up warp stages per tile (fp32, two
// keys per 16 bytes); a tile with more boundary pairs handles the rest directly
// from the K~ chunk.
constexpr int kMaxStagedPairs = 8;

template <int D, int NH>
struct Cfg {
    static constexpr int C = D / 16;                  // K-steps of the QK contraction
    static constexpr int KS = (D == 64 && NH == 2) ? 3 : 2;  // K~ stages
    static constexpr int VS = KS;                     // V stages
    static constexpr int QBytes = C * kChunkBytes;    // one query tile
    static constexpr int KBytes = C * kChunkBytes;
    static constexpr int VBytes = (D / 64) * 16384;   // 128 keys x 64 dims x 2 B per group
    static constexpr int OffQ = 0;                    // NH query tiles
    static constexpr int OffK = OffQ + NH * QBytes;
    static constexpr int OffV = OffK + KS * KBytes;
    static constexpr int OffBnd = OffV + VS * VBytes;                 // [KS][kMaxStagedPairs][64] float4
    static constexpr int BndBytes = kMaxStagedPairs * 64 * 16;
    static constexpr int OffCtl = OffBnd + KS * BndBytes;
    static constexpr int CtlBytes = 6144;
    static constexpr int Total = OffCtl + CtlBytes;
    static constexpr int Request = Total + 1024;
    // TMEM, two heads: D = 64: S0 [0,128), S1 [128,256), O0, O1 [256,384), P0, P1 [384,512).
    //                  D = 128: one S [0,128) shared by the two heads in turn, P0 [128,192),
    //                  P1 [192,256), O0 [256,384), O1 [384,512).
    //       one head (D = 64 only): S [0,128), O [128,192), P [192,256) of a 256-column
    //                  allocation, so that two CTAs share the SM's 512 columns.
    // Either way S_t is free again as soon as softmax t has read it into registers.
    static_assert(NH == 2 || D == 64, "one head per CTA is laid out for D = 64");
    static constexpr uint32_t TmemCols = NH == 2 ? 512 : 256;
    static constexpr uint32_t TmemO0 = NH == 2 ? 256 : 128, TmemO1 = 256 + D;
    static constexpr bool SharedS = (D == 128);
    static constexpr uint32_t TmemS0 = 0, TmemS1 = SharedS ? 0 : 128;
    static constexpr uint32_t TmemP0 = NH == 1 ? 192 : (SharedS ? 128 : 384), TmemP1 = SharedS ? 192 : 448;
};

template <int KS, int VS>
struct Ctl {
    uint64_t q_full;
    uint64_t k_full[KS], k_ready[KS], k_empty[KS];
    uint64_t v_full[VS], v_empty[VS];
    uint64_t s_full[2], s_read[2], p_full[2], o_done[2];
    uint64_t drain;
    uint64_t xbar[2][4];             // (head, lane quarter): both column halves have posted
    uint32_t tmem_base;
    int abort_flag;
    int w[kMaxPairs];
    float xval[2][4][2][2][32];      // (head, quarter, tile parity, column half, lane)
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

// The band of key tile j as j advances: both distances shrink by kBN per tile,
// so r_lo and r_full only move down; each step is amortised O(1) instead of a
// binary search on the critical path.
struct BandWalk {
    int r_lo, r_full;
    __device__ __forceinline__ void init(const int *w, int H, int64_t n0) {
        const Band b = tile_band(w, H, n0, 0);
        r_lo = b.r_lo;
        r_full = b.r_full;
    }
    __device__ __forceinline__ Band at(const int *w, int64_t n0, int64_t m0) {
        int64_t dmin = n0 - (m0 + kBN - 1);
        if (dmin < 0) dmin = 0;
        const int64_t dmax = n0 + kBM - 1 - m0;
        while (r_lo > 0 && (int64_t)w[r_lo - 1] >= dmin) --r_lo;
        while (r_full > 0 && (int64_t)w[r_full - 1] >= dmax) --r_full;
        Band b;
        b.r_lo = r_lo;
        b.r_full = r_full;
        return b;
    }
};

// The key tiles a CTA visits, in order: all of 0..qt, or under a token-level
// block selection the tiles whose mask entry is set, the diagonal tile qt always
// (every query keeps at least the causal prefix of its own tile).  Every warp
// walks the same sequence; pipeline stages and phases count visited tiles.
template <bool kMasked>
struct KeyTiles {
    const uint8_t *row;  // mask entries of this CTA's (sequence, KV head, query tile)
    int qt;
    __device__ __forceinline__ int from(int j) const {
        if constexpr (kMasked) {
            while (j < qt && row[j] == 0) ++j;
        }
        return j;
    }
    __device__ __forceinline__ int first() const { return from(0); }
    __device__ __forceinline__ int after(int j) const { return from(j + 1); }
};

__device__ __forceinline__ bool wait_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// kVarlen: the batch is packed along the token axis (q, k, v, out [total][H][D],
// packed Q~/K~ [H][D/16][total][16]); sequence b holds tokens cu[b]..cu[b+1]-1
// and N is the longest sequence.  Otherwise q/k/v/out are [B][N][H][D].
// kMasked: token-level block selection, block_mask [B][Hkv][T][T] (T query /
// key tiles of 128), entry (b, g, i, j) != 0 keeps key tile j for query tile i.
template <int D, bool kVarlen, int NH, bool kMasked, int CH>
__global__ void __launch_bounds__(Warps<NH, CH>::Threads, 3 - NH)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ WindowParams wp,
                      void *out, int out_f32, float *lse, int64_t N, int Hq, int Hkv, int *status,
                      uint64_t limit_ns, const int32_t *cu_seqlens, int64_t total, const uint8_t *block_mask) {
    using F = Cfg<D, NH>;
    using W = Warps<NH, CH>;
    constexpr int kThreads = W::Threads;
    constexpr int kWarpProducer = W::Producer, kWarpMma = W::Mma, kWarpFix = W::Fix, kWarpPv = W::Pv;
    constexpr uint32_t kTmemCols = F::TmemCols;
    constexpr int C = F::C;
    constexpr int H = D / 2;
    constexpr int KS = F::KS, VS = F::VS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + F::OffQ;
    uint8_t *sK = smem + F::OffK;
    uint8_t *sV = smem + F::OffV;
    float4 *sBnd = reinterpret_cast<float4 *>(smem + F::OffBnd);
    Ctl<KS, VS> *ctl = reinterpret_cast<Ctl<KS, VS> *>(smem + F::OffCtl);
    static_assert(sizeof(Ctl<KS, VS>) <= F::CtlBytes, "control block outgrew its space");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_qt = (int)((N + kBM - 1) / kBM);
    const int qt = num_qt - 1 - (int)blockIdx.x;  // longest query tiles first
    const int G = Hq / Hkv;
    const int pairs_per_group = (G + NH - 1) / NH;
    const int b = blockIdx.y / (Hkv * pairs_per_group);
    const int rem = blockIdx.y % (Hkv * pairs_per_group);
    const int kvh = rem / pairs_per_group;
    const int hp = rem % pairs_per_group;
    const int h0 = kvh * G + NH * hp;
    const bool two = NH == 2 && (2 * hp + 1) < G;  // a second head of the group shares this CTA
    const int nwg = two ? 2 : 1;
    const int64_t n0 = (int64_t)qt * kBM;
    const int nkt = qt + 1;  // key tiles 0..qt (causal)
    KeyTiles<kMasked> tiles;
    tiles.qt = qt;
    tiles.row = kMasked ? block_mask + (((size_t)b * Hkv + kvh) * num_qt + qt) * (size_t)num_qt : nullptr;
    // Where this CTA's sequence lives: first token on the token axis, valid rows,
    // batch coordinate of the tensor maps, rows per batch of out / lse.
    int64_t tokbase = 0, seq_len = N, nrows = N;
    int bz = b;
    if constexpr (kVarlen) {
        const int64_t t0 = cu_seqlens[b], t1 = cu_seqlens[b + 1];
        // A malformed table selects no rows (every write below stays inside [0, total)).
        seq_len = (t0 >= 0 && t1 >= t0 && t1 <= total) ? t1 - t0 : 0;
        tokbase = seq_len > 0 ? t0 : 0;
        nrows = total;
        bz = 0;
        if (n0 >= seq_len) return;  // this sequence has fewer query tiles (whole CTA, before any barrier)
    }

    if (threadIdx.x == 0) {
        mbar_init(&ctl->q_full, 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(&ctl->k_full[s], 1);
            mbar_init(&ctl->k_ready[s], 1);
            mbar_init(&ctl->k_empty[s], 1 + 4 * CH * nwg);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&ctl->v_full[s], 1);
            mbar_init(&ctl->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ctl->s_full[s], 1);
            mbar_init(&ctl->s_read[s], 4 * CH);
            mbar_init(&ctl->p_full[s], 4 * CH);
            mbar_init(&ctl->o_done[s], 1);
        }
        mbar_init(&ctl->drain, 2);  // one commit from each issuing warp
        for (int t = 0; t < 2; ++t)
            for (int q = 0; q < 4; ++q) mbar_init(&ctl->xbar[t][q], CH);
        ctl->abort_flag = 0;
        fence_mbar_init();
    }
    for (int r = threadIdx.x; r < H; r += kThreads) ctl->w[r] = wp.w[r];
    if (warp == kWarpMma) {
        tmem_alloc(&ctl->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int *w = ctl->w;
    WaitCtl wc{&ctl->abort_flag, status, limit_ns, 0};

    // Register split (Warps): two heads, split rows: 640 threads at 96 registers
    // (61440); the last warpgroup (producer, MMA, fix-up, PV) drops to 56 and the
    // four softmax warpgroups rise to 104: 128 x 56 + 512 x 104 = 60416.  Two
    // heads, whole rows: 384 threads at 168 (64512); 128 x 96 + 256 x 200 = 63488.
    // One head (two CTAs per SM): 256 threads at 128 (32768); 128 x 56 + 128 x 200.
    if (warp >= W::Soft) setmaxnreg_dec<W::OtherRegs>();
    if (warp == kWarpProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int last_k[KS], last_v[VS];
            for (int s = 0; s < KS; ++s) last_k[s] = -1;
            for (int s = 0; s < VS; ++s) last_v[s] = -1;
            mbar_expect_tx(&ctl->q_full, (uint32_t)(nwg * F::QBytes));
            for (int t = 0; t < nwg; ++t)
                for (int c = 0; c < C; ++c)
                    tma_load_3d(sQ + t * F::QBytes + c * kChunkBytes, &tm_q, &ctl->q_full, 0, (int)(tokbase + n0),
                                (bz * Hq + h0 + t) * C + c);
            bool ok = true;
            BandWalk bw;
            bw.init(w, H, n0);
            for (int it = 0, j = tiles.first(); j < nkt && ok; ++it, j = tiles.after(j)) {
                const int ks = it % KS, vs = it % VS;
                const int64_t m0 = (int64_t)j * kBN;
                const int ca = bw.at(w, n0, m0).r_lo >> 3;
                wc.site = 1;
                if (!(ok = mbar_wait(&ctl->k_empty[ks], ((it / KS) & 1) ^ 1, wc))) break;
                mbar_expect_tx(&ctl->k_full[ks], (uint32_t)(C - ca) * kChunkBytes);
                for (int c = ca; c < C; ++c)
                    tma_load_3d(sK + ks * F::KBytes + c * kChunkBytes, &tm_k, &ctl->k_full[ks], 0,
                                (int)(tokbase + m0), (bz * Hkv + kvh) * C + c);
                last_k[ks] = it;
                wc.site = 2;
                if (!(ok = mbar_wait(&ctl->v_empty[vs], ((it / VS) & 1) ^ 1, wc))) break;
                mbar_expect_tx(&ctl->v_full[vs], F::VBytes);
                for (int gidx = 0; gidx < D / 64; ++gidx)
                    tma_load_4d(sV + vs * F::VBytes + gidx * 16384, &tm_v, &ctl->v_full[vs], gidx * 64, kvh,
                                (int)(tokbase + m0), bz);
                last_v[vs] = it;
            }
            if (!ok) {
                // Let every copy this thread started land before the CTA exits.
                const uint64_t drain_ns = atflash_drain_limit_ns(limit_ns);
                wait_drain(&ctl->q_full, 0, drain_ns);
                for (int s = 0; s < KS; ++s)
                    if (last_k[s] >= 0) wait_drain(&ctl->k_full[s], (last_k[s] / KS) & 1, drain_ns);
                for (int s = 0; s < VS; ++s)
                    if (last_v[s] >= 0) wait_drain(&ctl->v_full[s], (last_v[s] / VS) & 1, drain_ns);
            }
        }
    } else if (warp == kWarpFix) {
        // ------------------------- pruned-pair zeroing and boundary staging
        bool ok = true;
        BandWalk bw;
        bw.init(w, H, n0);
        for (int it = 0, j = tiles.first(); j < nkt && ok; ++it, j = tiles.after(j)) {
            const int ks = it % KS;
            const Band bd = bw.at(w, n0, (int64_t)j * kBN);
            const int r_lo = bd.r_lo;
            const int ca = r_lo >> 3;
            wc.site = 3;
            if (!(ok = mbar_wait_warp(&ctl->k_full[ks], (it / KS) & 1, wc))) break;
            // Boundary pairs r_lo + b: key values of keys (2i, 2i+1) as
            // (k_r[2i], k_r[2i+1], k_{r+H}[2i], k_{r+H}[2i+1]) in fp32.
            const int nb = min(bd.r_full - r_lo, kMaxStagedPairs);
            float4 *bst = sBnd + ks * (kMaxStagedPairs * 64);
            for (int e = lane; e < nb * 64; e += 32) {
                const int bi = e >> 6, i = e & 63, r = r_lo + bi;
                const uint8_t *kch = sK + ks * F::KBytes + (r >> 3) * kChunkBytes;
                const uint32_t w0 = *reinterpret_cast<const uint32_t *>(kch + sw32_off(2 * i, r & 7));
                const uint32_t w1 = *reinterpret_cast<const uint32_t *>(kch + sw32_off(2 * i + 1, r & 7));
                bst[e] = make_float4(bf16lo(w0), bf16lo(w1), bf16hi(w0), bf16hi(w1));
            }
            if ((r_lo & 7) && ca < C) {
                // Pairs [8*ca, r_lo) are pruned for every cell of this tile: zero them
                // in the landed K~ chunk so the dense MMA over whole chunks skips them.
                // Lane -> (row, word) with consecutive lanes on consecutive words.
                uint8_t *chunk = sK + ks * F::KBytes + ca * kChunkBytes;
                const int z = r_lo & 7;
#pragma unroll 4
                for (int e = lane; e < kBN * 8; e += 32)
                    if ((e & 7) < z) *reinterpret_cast<uint32_t *>(chunk + sw32_off(e >> 3, e & 7)) = 0u;
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->k_ready[ks]);
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------- QK issuer
        // tcgen05.mma issue returns only once the tensor pipe has taken the
        // instruction, so a warp that issued PV could not start the next QK
        // early; QK and PV therefore have an issuing warp each.
        const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
        const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
        wc.site = 4;
        bool ok = mbar_wait_warp(&ctl->q_full, 0, wc);
        auto issue_qk = [&](int t, int ks, int ca) {
            if (lane == 0) {
                tc_fence_after();
                for (int c = ca; c < C; ++c) {
                    const uint64_t da = smem_desc(sQa + t * F::QBytes + c * kChunkBytes, 16, 256, kSwizzle32B);
                    const uint64_t db = smem_desc(sKa + ks * F::KBytes + c * kChunkBytes, 16, 256, kSwizzle32B);
                    umma_bf16_ss(tmem + (t ? F::TmemS1 : F::TmemS0), da, db, idesc_qk, c > ca ? 1u : 0u);
                }
                umma_commit(&ctl->s_full[t]);
            }
            __syncwarp();
        };
        BandWalk bw;
        bw.init(w, H, n0);
        for (int it = 0, j = tiles.first(); j < nkt && ok; ++it, j = tiles.after(j)) {
            const int ks = it % KS;
            const int ca = bw.at(w, n0, (int64_t)j * kBN).r_lo >> 3;
            wc.site = 7;
            if (!(ok = mbar_wait_warp(&ctl->k_ready[ks], (it / KS) & 1, wc))) break;
            // S_0(j) once its columns are free: read by head 0 (own buffer) or by
            // head 1 (buffer shared by the two heads); S_1(j) likewise.
            wc.site = 13;
            if (it > 0) {
                uint64_t *free_bar = (F::SharedS && two) ? &ctl->s_read[1] : &ctl->s_read[0];
                if (!(ok = mbar_wait_warp(free_bar, (it - 1) & 1, wc))) break;
            }
            issue_qk(0, ks, ca);
            if (two) {
                if (F::SharedS) {
                    if (!(ok = mbar_wait_warp(&ctl->s_read[0], it & 1, wc))) break;
                } else if (it > 0) {
                    if (!(ok = mbar_wait_warp(&ctl->s_read[1], (it - 1) & 1, wc))) break;
                }
                issue_qk(1, ks, ca);
            }
            if (lane == 0) umma_commit(&ctl->k_empty[ks]);
            __syncwarp();
        }
    } else if (warp == kWarpPv) {
        // ------------------------------------------------------- PV issuer
        const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
        const uint32_t sVa = smem_u32(sV);
        bool ok = true;
        for (int it = 0, j = tiles.first(); j < nkt && ok; ++it, j = tiles.after(j)) {
            const int vs = it % VS;
            wc.site = 5;
            if (!(ok = mbar_wait_warp(&ctl->v_full[vs], (it / VS) & 1, wc))) break;
            for (int t = 0; t < nwg && ok; ++t) {
                wc.site = 6;
                if (!(ok = mbar_wait_warp(&ctl->p_full[t], it & 1, wc))) break;
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t o_col = t ? F::TmemO1 : F::TmemO0;
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk) {
                        // A = P_t keys [16kk, 16kk+16): 8 TMEM columns of bf16 pairs.
                        // B = V rows [16kk, 16kk+16): MN-major SW128, 64-dim groups 16 KB apart.
                        const uint64_t db = smem_desc(sVa + vs * F::VBytes + kk * 2048, 16384, 1024, kSwizzle128B);
                        umma_bf16_ts(tmem + o_col, tmem + (t ? F::TmemP1 : F::TmemP0) + kk * 8, db, idesc_pv,
                                     (it > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&ctl->o_done[t]);
                }
                __syncwarp();
            }
            if (ok && lane == 0) umma_commit(&ctl->v_empty[vs]);
            __syncwarp();
        }
    } else if (warp < W::Soft) {
        // ------------------------------------------------------------- softmax
        setmaxnreg_inc<W::SoftRegs>();
        constexpr int kCols = kBN / CH;    // S columns per warp
        constexpr int kOCols = D / CH;     // O columns per warp (rescale, epilogue)
        const int t = warp / (4 * CH);     // which head of the pair
        if (t < nwg) {
            const int q4 = warp & 3, hc = (warp >> 2) % CH;
            const int c0 = hc * kCols;     // this warp's first column of the key tile
            const int row = q4 * 32 + lane;
            const int64_t n = n0 + row;
            const int hq = h0 + t;
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            const uint32_t tS = tmem + (t ? F::TmemS1 : F::TmemS0) + lane_off + c0;
            const uint32_t tP = tmem + (t ? F::TmemP1 : F::TmemP0) + lane_off + c0 / 2;
            const uint32_t tO = tmem + (t ? F::TmemO1 : F::TmemO0) + lane_off + hc * kOCols;
            const uint8_t *sQt = sQ + t * F::QBytes;
            const float scale_log2 = 1.4426950408889634f * rsqrtf((float)D);
            // The two warps of a row post partial values here (parity of the tile
            // count: a slot is rewritten only after the partner has passed the
            // next exchange, hence has read it).
            uint64_t *xbar = &ctl->xbar[t][q4];
            float m_used = -INFINITY, lrun = 0.f;
            wc.site = 8;
            bool ok = mbar_wait_warp(&ctl->q_full, 0, wc);  // Q~ rows are read for the boundary fix-up
            BandWalk bw;
            bw.init(w, H, n0);
            int it = 0;  // key tiles visited
            for (int j = tiles.first(); j < nkt && ok; ++it, j = tiles.after(j)) {
                const int ks = it % KS;
                const int64_t m0 = (int64_t)j * kBN;
                const Band bd = bw.at(w, n0, m0);
                float s[kCols];
                wc.site = 9;
                if (!(ok = mbar_wait_warp(&ctl->s_full[t], it & 1, wc))) break;
                tc_fence_after();
                if ((bd.r_lo >> 3) < C) {
                    // One load of the warp's columns; two of 64 for a whole row in the
                    // one-head kernel (launched with 128 registers).  Both measured faster
                    // than loads of 32 columns.
                    if constexpr (kCols == 64) {
                        uint32_t ra[64];
                        tmem_ld_32x32b_x64(tS, ra);
                        tmem_ld_wait(ra);
#pragma unroll
                        for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(ra[i]);
                    } else if constexpr (NH == 2) {
                        uint32_t ra[128];
                        tmem_ld_32x32b_x128(tS, ra);
                        tmem_ld_wait(ra);
#pragma unroll
                        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(ra[i]);
                    } else {
                        uint32_t ra[64], rb[64];
                        tmem_ld_32x32b_x64(tS + 0, ra);
                        tmem_ld_32x32b_x64(tS + 64, rb);
                        tmem_ld_wait(ra);
                        tmem_ld_wait(rb);
#pragma unroll
                        for (int i = 0; i < 64; ++i) {
                            s[i] = __uint_as_float(ra[i]);
                            s[64 + i] = __uint_as_float(rb[i]);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kCols; ++i) s[i] = 0.f;
                }
                // S is in registers: the MMA may reuse its columns.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->s_read[t]);
                // Boundary pairs: the dense MMA included them; remove them from the
                // cells whose distance exceeds the pair's window (jj < n - m0 - w_r).
                if (bd.r_lo < bd.r_full) {
                    // The fix-up warp has staged this tile's boundary pairs.  This wait is
                    // skipped on tiles without boundary pairs; it is never a phase off:
                    // S(j) was waited for above and its MMA waited for this phase, and
                    // the stage's next phase needs this warp to release the stage first.
                    wc.site = 10;
                    if (!(ok = mbar_wait_warp(&ctl->k_ready[ks], (it / KS) & 1, wc))) break;
                    const float4 *bst = sBnd + ks * (kMaxStagedPairs * 64);
                    for (int r = bd.r_lo; r < bd.r_full; ++r) {
                        const int lim = (int)(n - m0 - (int64_t)w[r]);  // cells jj < lim drop pair r
                        const int lim_max = __reduce_max_sync(0xffffffffu, lim);
                        if (lim_max <= c0) continue;  // none of this warp's columns
                        const uint32_t qw =
                            *reinterpret_cast<const uint32_t *>(sQt + (r >> 3) * kChunkBytes + sw32_off(row, r & 7));
                        const float2 qa2 = make_float2(bf16lo(qw), bf16lo(qw));
                        const float2 qb2 = make_float2(bf16hi(qw), bf16hi(qw));
                        if (r - bd.r_lo < kMaxStagedPairs) {
                            const float4 *kb = bst + (r - bd.r_lo) * 64;
                            // One predicated loop per 32-column block: a separate copy for the
                            // blocks every row of the warp prunes in full measured slower (the
                            // larger correction code cost more than the saved compares).
#pragma unroll
                            for (int cc = 0; cc < kCols / 32; ++cc) {
                                if (c0 + 32 * cc < lim_max) {
#pragma unroll
                                    for (int i = 0; i < 16; ++i) {
                                        const int jl = 32 * cc + 2 * i, jj = c0 + jl;
                                        const float4 kv = kb[jj / 2];
                                        const float2 t = fma2(qa2, make_float2(kv.x, kv.y),
                                                              mul2(qb2, make_float2(kv.z, kv.w)));
                                        if (jj < lim) s[jl] -= t.x;
                                        if (jj + 1 < lim) s[jl + 1] -= t.y;
                                    }
                                }
                            }
                        } else {
                            // More boundary pairs than staged: read the K~ chunk directly.
                            const float qa = qa2.x, qb = qb2.x;
                            const uint8_t *kch = sK + ks * F::KBytes + (r >> 3) * kChunkBytes;
#pragma unroll
                            for (int cc = 0; cc < kCols / 32; ++cc) {
                                if (c0 + 32 * cc < lim_max) {
#pragma unroll
                                    for (int i = 0; i < 32; ++i) {
                                        const int jl = 32 * cc + i, jj = c0 + jl;
                                        if (jj < lim) {
                                            const uint32_t kw =
                                                *reinterpret_cast<const uint32_t *>(kch + sw32_off(jj, r & 7));
                                            s[jl] -= qa * bf16lo(kw) + qb * bf16hi(kw);
                                        }
                                    }
                                }
                            }
                        }
                    }
                    __syncwarp();  // every lane is done with this stage's staged keys
                }
                if (lane == 0) mbar_arrive(&ctl->k_empty[ks]);
                // Causal mask on the diagonal tile; row max of the raw scores (4 chains
                // of 3-input max); the 1/sqrt(D) * log2(e) scale is folded into the exp.
                if (j == qt) {
#pragma unroll
                    for (int jl = 0; jl < kCols; ++jl)
                        if (c0 + jl > row) s[jl] = -INFINITY;
                }
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < kCols; jj += 8) {
                    mx0 = max3(mx0, s[jj], s[jj + 1]);
                    mx1 = max3(mx1, s[jj + 2], s[jj + 3]);
                    mx2 = max3(mx2, s[jj + 4], s[jj + 5]);
                    mx3 = max3(mx3, s[jj + 6], s[jj + 7]);
                }
                float raw_max = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
                if constexpr (CH == 2) {
                    // The row's maximum over both column halves, so that both warps take
                    // the same running max (P of one row must share it).
                    float *slot = ctl->xval[t][q4][it & 1][0];
                    slot[hc * 32 + lane] = raw_max;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(xbar);
                    wc.site = 13;
                    if (!(ok = mbar_wait_warp(xbar, it & 1, wc))) break;
                    raw_max = fmaxf(raw_max, slot[(hc ^ 1) * 32 + lane]);
                }
                const float tile_max = raw_max * scale_log2;
                // Keep the previous (stale) max unless the row max grew by more than
                // 2^8: the final O / l uses the same max, so the result is exact.
                const bool need = tile_max > m_used + kRescaleThreshold;
                const float m_new = need ? tile_max : m_used;
                const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;
                m_used = m_new;
                // P = exp2(s * scale - m) as bf16 pairs; S registers die as P is produced.
                const float2 mneg = make_float2(-m_used, -m_used);
                const float2 sc2 = make_float2(scale_log2, scale_log2);
                float2 l0 = make_float2(0.f, 0.f), l1 = make_float2(0.f, 0.f);
                uint32_t pk[kCols / 2];
#pragma unroll
                for (int i = 0; i < kCols / 2; i += 2) {
                    float2 xa = fma2(make_float2(s[2 * i], s[2 * i + 1]), sc2, mneg);
                    float2 xb = fma2(make_float2(s[2 * i + 2], s[2 * i + 3]), sc2, mneg);
                    xa.x = fast_exp2(xa.x);
                    xa.y = fast_exp2(xa.y);
                    xb.x = fast_exp2(xb.x);
                    xb.y = fast_exp2(xb.y);
                    l0 = add2(l0, xa);
                    l1 = add2(l1, xb);
                    pk[i] = pack_bf16x2(xa.x, xa.y);
                    pk[i + 1] = pack_bf16x2(xb.x, xb.y);
                }
                // Rescale O only when some row's max grew past the threshold (rare).
                // PV_t(j-1) must also be done reading P_t before it is overwritten.
                const bool rescale = (it > 0) && __any_sync(0xffffffffu, need);
                if (it > 0) {
                    wc.site = 11;
                    if (!(ok = mbar_wait_warp(&ctl->o_done[t], (it - 1) & 1, wc))) break;
                    tc_fence_after();
                }
                if (rescale) {
#pragma unroll 1
                    for (int cc = 0; cc < kOCols / 32; ++cc) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(tO + cc * 32, r);
                        tmem_ld_wait(r);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st_32x32b_x32(tO + cc * 32, r);
                    }
                }
                // This warp's part of P_t (bf16 pairs of its columns).
#pragma unroll
                for (int cc = 0; cc < kCols / 64; ++cc)
                    tmem_st_32x32b_x32(tP + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * cc]));
                tmem_st_wait();
                const float2 ls = add2(l0, l1);
                lrun = lrun * alpha + (ls.x + ls.y);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->p_full[t]);
            }
            if (ok) {
                wc.site = 12;
                ok = mbar_wait_warp(&ctl->o_done[t], (it - 1) & 1, wc);
            }
            if constexpr (CH == 2) {
                // The row's sum over both column halves (one more exchange).
                if (ok) {
                    float *slot = ctl->xval[t][q4][it & 1][0];
                    slot[hc * 32 + lane] = lrun;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(xbar);
                    wc.site = 13;
                    ok = mbar_wait_warp(xbar, it & 1, wc);
                    if (ok) lrun += slot[(hc ^ 1) * 32 + lane];
                }
            }
            if (ok) {
                tc_fence_after();
                const float inv = 1.f / lrun;
                const size_t o = ((size_t)((int64_t)bz * nrows + tokbase + n) * Hq + hq) * D + hc * kOCols;
#pragma unroll
                for (int cc = 0; cc < kOCols / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tO + cc * 32, r);
                    tmem_ld_wait(r);
                    if (n < seq_len) {
                        if (out_f32) {
                            float4 *dst =
                                reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + o + cc * 32);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv,
                                                     __uint_as_float(r[4 * i + 1]) * inv,
                                                     __uint_as_float(r[4 * i + 2]) * inv,
                                                     __uint_as_float(r[4 * i + 3]) * inv);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(out) + o +
                                                                   cc * 32);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                dst[i] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv,
                                                                __uint_as_float(r[8 * i + 1]) * inv),
                                                    pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv,
                                                                __uint_as_float(r[8 * i + 3]) * inv),
                                                    pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv,
                                                                __uint_as_float(r[8 * i + 5]) * inv),
                                                    pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv,
                                                                __uint_as_float(r[8 * i + 7]) * inv));
                        }
                    }
                }
                if (lse && hc == 0 && n < seq_len)
                    lse[((size_t)bz * Hq + hq) * nrows + tokbase + n] = (m_used + __log2f(lrun)) * 0.69314718055994531f;
            }
        }
    }

    // Teardown: every tensor-core operation must be complete before TMEM is freed.
    __syncthreads();
    if (warp == kWarpPv && lane == 0) umma_commit(&ctl->drain);
    if (warp == kWarpMma) {
        if (lane == 0) {
            umma_commit(&ctl->drain);
            wait_drain(&ctl->drain, 0, atflash_drain_limit_ns(limit_ns));
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
                              uint64_t wait_limit_ns, cudaStream_t s, const int32_t *cu_seqlens, int64_t total,
                              const uint8_t *block_mask) {
    const int C = p.D / 16;
    const bool varlen = cu_seqlens != nullptr;
    const bool masked = block_mask != nullptr;
    if (varlen && masked) return cudaErrorInvalidValue;
    // Token axis of the maps: N per batch entry, or the whole packed batch.
    const cuuint64_t T = varlen ? (cuuint64_t)total : (cuuint64_t)p.N;
    const cuuint64_t NB = varlen ? 1 : (cuuint64_t)p.B;
    CUtensorMap tq, tk, tv;
    {
        cuuint64_t dims[3] = {16, T, NB * p.Hq * C};
        cuuint64_t str[2] = {32, T * 32};
        cuuint32_t box[3] = {16, tc::kBM, 1};
        cudaError_t e = make_map(&tq, const_cast<void *>(qpack), 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B);
        if (e != cudaSuccess) return e;
    }
    {
        cuuint64_t dims[3] = {16, T, NB * p.Hkv * C};
        cuuint64_t str[2] = {32, T * 32};
        cuuint32_t box[3] = {16, tc::kBN, 1};
        cudaError_t e = make_map(&tk, const_cast<void *>(kpack), 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B);
        if (e != cudaSuccess) return e;
    }
    {
        cuuint64_t dims[4] = {(cuuint64_t)p.D, (cuuint64_t)p.Hkv, T, NB};
        cuuint64_t str[3] = {(cuuint64_t)p.D * 2, (cuuint64_t)p.Hkv * p.D * 2, T * p.Hkv * p.D * 2};
        cuuint32_t box[4] = {64, 1, tc::kBN, 1};
        cudaError_t e = make_map(&tv, const_cast<void *>(v), 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
    }
    const int num_qt = (int)((p.N + tc::kBM - 1) / tc::kBM);
    const int G = p.Hq / p.Hkv;
    cudaError_t e;
#define ATF_PREFILL_TC_M(DD, VL, NHH, MK, CHH)                                                                   \
    do {                                                                                                         \
        const int smem = tc::Cfg<DD, NHH>::Request;                                                             \
        dim3 grid((unsigned)num_qt, (unsigned)(p.B * p.Hkv * ((G + NHH - 1) / NHH)));                          \
        e = cudaFuncSetAttribute(tc::prefill_tc_kernel<DD, VL, NHH, MK, CHH>,                                        \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);                             \
        if (e != cudaSuccess) return e;                                                                          \
        /* The in-kernel register split assumes this launch count: refuse to run otherwise. */                  \
        cudaFuncAttributes fa;                                                                                   \
        if ((e = cudaFuncGetAttributes(&fa, tc::prefill_tc_kernel<DD, VL, NHH, MK, CHH>)) != cudaSuccess) return e;  \
        if (fa.numRegs != tc::Warps<NHH, CHH>::LaunchRegs) return cudaErrorInvalidConfiguration;                      \
        tc::prefill_tc_kernel<DD, VL, NHH, MK, CHH><<<grid, tc::Warps<NHH, CHH>::Threads, smem, s>>>(                     \
            tq, tk, tv, wp, out, out_f32, lse, p.N, p.Hq, p.Hkv, status, wait_limit_ns, cu_seqlens, total,       \
            block_mask);                                                                                         \
    } while (0)
    // Block-selected launches (never varlen) take their own instantiations, so that
    // the dense kernels' code is what it was.
#define ATF_PREFILL_TC(DD, VL, NHH, CHH)                                                                         \
    do {                                                                                                         \
        if constexpr (!VL) {                                                                                     \
            if (masked) {                                                                                        \
                ATF_PREFILL_TC_M(DD, false, NHH, true, CHH);                                                     \
                break;                                                                                           \
            }                                                                                                    \
        }                                                                                                        \
        ATF_PREFILL_TC_M(DD, VL, NHH, false, CHH);                                                               \
    } while (0)
    // No pair pruned anywhere (k = inf, or windows covering the longest sequence).
    const bool unpruned = (int64_t)wp.w[0] >= p.N - 1;
    if (p.D == 128) {
        // Two heads per CTA; each row split between two softmax warps only with pruning
        // (without it the whole-row form measured faster).
        if (unpruned) {
            if (varlen) ATF_PREFILL_TC(128, true, 2, 1); else ATF_PREFILL_TC(128, false, 2, 1);
        } else {
            if (varlen) ATF_PREFILL_TC(128, true, 2, 2); else ATF_PREFILL_TC(128, false, 2, 2);
        }
    } else if (p.D == 64) {
        // Unpruned: one head per CTA, two CTAs per SM measured faster (no boundary work
        // to share between heads).  With pruning, two heads per CTA share every K~
        // tile's zeroing and boundary staging, with split rows.
        if (unpruned) {
            if (varlen) ATF_PREFILL_TC(64, true, 1, 1); else ATF_PREFILL_TC(64, false, 1, 1);
        } else {
            if (varlen) ATF_PREFILL_TC(64, true, 2, 2); else ATF_PREFILL_TC(64, false, 2, 2);
        }
    } else {
        return cudaErrorInvalidValue;
    }
#undef ATF_PREFILL_TC
#undef ATF_PREFILL_TC_M
    return cudaGetLastError();
}

}  // namespace atf
