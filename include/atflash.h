/*
 * atflash.h — C ABI of the B200 (sm_100a) per-RoPE-wavelength windowed
 * attention library (libatflash.so).
 *
 * The method ("ATFlash — Per-RoPE-Wavelength Attention Windows",
 * gh.bsm-lab.com/ATFlash/ATFlash-Kernel, section "The idea"; arXiv 2608.02947
 * abstract): in causal attention with rotate-half RoPE, the query-key score is
 * a sum over D/2 frequency pairs, pair r = dims (r, r + D/2), rotated by
 * position * theta_r with theta_r = base^(-2r/D).  The term of pair r is kept
 * only while the distance n - m <= w_r = floor(k * lambda_r), lambda_r =
 * 2*pi/theta_r; the kept terms feed an unchanged softmax and P.V product.
 * k = +INFINITY keeps every term (plain causal RoPE attention).  A cell whose
 * every pair is pruned scores 0 (the empty sum); no key is dropped.
 *
 * Conventions shared by every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, unless a
 *    call says otherwise.  They must stay valid until the work queued on
 *    `stream` has finished.  The library keeps no reference after returning.
 *  - GPU calls are asynchronous on `stream` (0 = legacy default stream).
 *  - Every call validates its arguments first and returns a status < 0 with
 *    nothing launched when they are invalid.  ATFLASH_OK (0) means the work
 *    was queued.  Faults inside a queued kernel surface as CUDA errors on the
 *    stream; a kernel whose bounded internal wait ran out records
 *    ATFLASH_ERR_TIMEOUT, read back with atflash_device_status().
 *  - Softmax scale is 1/sqrt(D).  Query head h reads KV head h / (Hq / Hkv).
 *  - Positions: prefill queries and keys sit at 0..N-1; a decode query of
 *    sequence b sits at seqlens[b]-1 and attends cache rows 0..seqlens[b]-1.
 *  - w_r is computed once on the host in fp64 and never in fp32.
 */
#ifndef ATFLASH_H
#define ATFLASH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t. */
typedef struct CUstream_st *cudaStream_t;

/* Status codes. */
#define ATFLASH_OK 0
#define ATFLASH_ERR_INVALID_ARG (-1) /* null pointer, non-positive size, Hq % Hkv != 0, NaN or
                                        negative k, base <= 1, N beyond 2^31-1 */
#define ATFLASH_ERR_UNSUPPORTED (-2) /* a head dim or dtype combination with no kernel */
#define ATFLASH_ERR_WORKSPACE (-3)   /* workspace missing or smaller than required */
#define ATFLASH_ERR_CUDA (-4)        /* a CUDA runtime/driver call or launch failed */
#define ATFLASH_ERR_TIMEOUT (-5)     /* a kernel's bounded wait ran out (device status) */
#define ATFLASH_ERR_ALIGNMENT (-6)   /* a pointer is not 16-byte aligned */
#define ATFLASH_ERR_BAD_PAGE (-7)    /* a paged decode met a page index past its block-table row or a
                                        page id outside the pool (device status) */

/* Element types of tensors passed to the GPU calls. */
#define ATFLASH_F32 0
#define ATFLASH_BF16 1

/* KV-cache layouts accepted by atflash_decode. */
#define ATFLASH_KV_HND 0 /* [B][Hkv][Nmax][D]: one contiguous block per (sequence, KV head) */
#define ATFLASH_KV_NHD 1 /* [B][Nmax][Hkv][D]: token-major, the prefill's k/v layout */
#define ATFLASH_KV_PACKED 2 /* K pre-rotated in atflash_rope_pack's bf16 layout [B*Hkv][D/16][Nmax][16]
                               (8 frequency pairs per 32-byte chunk); V as [B][Hkv][Nmax][D].
                               Pruned chunks are contiguous, so they are never fetched from HBM. */

/* Text of a status code (static storage, never NULL). */
const char *atflash_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int atflash_version(void);

/*
 * Per-pair window table ("The idea": w_r = k * lambda_r, kept while n - m <= w_r).
 *   D         head dim, even, 2..256
 *   rope_base RoPE base (> 1)
 *   k_window  k >= 0, or +INFINITY for no window
 *   N         sequence length (>= 1); entries are clamped to N - 1
 *   w_out     HOST array of D/2 int64 written with min(floor(k*lambda_r), N-1)
 * Host only; no device work.
 */
int atflash_window_table(int D, double rope_base, double k_window, int64_t N, int64_t *w_out);

/* Counts of query-key inner-product terms of ONE (sequence, head) over the
 * causal triangle of N positions.  A pair-term is one (n, m, r) with m <= n;
 * a dim-term is one of its two products (so dims = 2 x pairs). */
typedef struct {
    uint64_t total;      /* (D/2) * N(N+1)/2 pair-terms */
    uint64_t kept;       /* pair-terms with n - m <= w_r */
    uint64_t pruned;     /* total - kept */
    uint64_t total_dims; /* 2 * total */
    uint64_t kept_dims;  /* 2 * kept */
} atflash_terms;

/*
 * Input-independent closed-form count of kept and pruned terms (arXiv
 * 2608.02947 abstract: "the reduction rate is input-independent, with a
 * closed form"; README "The idea": "you know the cost before running").
 * kept = sum_r (W_r + 1)(2N - W_r)/2 with W_r = min(w_r, N - 1).
 * Host only; `out` is a HOST pointer.
 */
int atflash_pruned_terms(int64_t N, int D, double rope_base, double k_window, atflash_terms *out);

/*
 * Windowed causal RoPE prefill, bf16 in and out (the spec call).
 *   q    [B][N][Hq][D]  bf16, un-rotated queries, row-major
 *   k, v [B][N][Hkv][D] bf16, un-rotated keys, values
 *   out  [B][N][Hq][D]  bf16, written
 *   D in {64, 128}; B, Hq, Hkv, N >= 1; Hq % Hkv == 0; N <= 2^31 - 1.
 * Scratch (rotated Q and K, atflash_prefill_workspace_bytes()) is taken from
 * a stream-ordered pool owned by the library and returned on `stream`; use
 * atflash_prefill_ex with a caller workspace to avoid that.
 * All pointers 16-byte aligned.
 */
int atflash_prefill(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                    int64_t N, int D, double rope_base, double k_window, cudaStream_t stream);

/* Device scratch bytes atflash_prefill_ex needs (0 on invalid arguments). */
size_t atflash_prefill_workspace_bytes(int B, int Hq, int Hkv, int64_t N, int D, int in_dtype);

/*
 * Prefill with explicit dtypes, optional log-sum-exp and a caller workspace.
 *   in_dtype  ATFLASH_BF16: tensor-core path (tcgen05, bf16 operands, fp32
 *             accumulate), D in {64, 128}.
 *             ATFLASH_F32: exact fp32 CUDA-core path, any even D in 2..256.
 *   out_dtype ATFLASH_BF16 or ATFLASH_F32 (out's element type).
 *   lse       NULL, or [B][Hq][N] fp32 device array written with the natural
 *             log-sum-exp of each row's scaled scores.
 *   workspace device buffer of >= atflash_prefill_workspace_bytes(...) bytes,
 *             256-byte aligned; owned by the caller, free for reuse once the
 *             call's work on `stream` has finished.
 */
int atflash_prefill_ex(const void *q, const void *k, const void *v, void *out, int B, int Hq,
                       int Hkv, int64_t N, int D, double rope_base, double k_window, int in_dtype,
                       int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/*
 * Accuracy of short rows.  The tensor-core path rounds the rotated queries and
 * keys, and the probabilities P, to bf16.  Over a row that sees few keys those
 * roundings do not average out (seeded sweeps measured errors up to 1.06e-2 on
 * rows of 4-16 keys, against below 4e-3 on rows of more than 128 keys), so
 * every bf16 call recomputes, after its tensor-core kernel, each row that sees
 * at most 128 keys in fp32 on CUDA cores from the un-rotated inputs, by the
 * method's plain definition ("The idea": RoPE, the per-pair window, softmax,
 * P.V), and overwrites that row's output and log-sum-exp: the first 128-row
 * tile of every prefill sequence, every query tile of a block selection whose
 * mask selects no earlier key tile, and every decode sequence of at most 128
 * tokens.
 *
 * atflash_prefill_short_rows is that step on its own, for callers that run
 * atflash_rope_pack + atflash_prefill_packed themselves: same q, k, v (the
 * un-rotated bf16 inputs), out, out_dtype, lse, shapes and errors as
 * atflash_prefill_ex with in_dtype ATFLASH_BF16; queue it after the packed
 * prefill on the same stream.  The three calls together give the same bits as
 * atflash_prefill_ex.
 */
int atflash_prefill_short_rows(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                               int64_t N, int D, double rope_base, double k_window, int out_dtype, float *lse,
                               cudaStream_t stream);

/*
 * Windowed prefill on top of a token-level block selection ("Abstract": token-
 * level selection such as MInference's is orthogonal to the frequency-level
 * window, which can be applied on top of it).
 *   block_mask  DEVICE uint8 [B][Hkv][T][T], T = ceil(N / 128), read during the
 *               call (stream order), owned by the caller.  Entry (b, g, i, j) != 0
 *               makes key tile j (keys 128j .. 128j+127) visible to query tile i
 *               (queries 128i .. 128i+127) for every query head of KV head g.
 *               The diagonal tile j == i is always visible (each query keeps the
 *               causal prefix of its own tile, so no row is empty); entries with
 *               j > i cover only future keys and are ignored.
 * Query n attends key m iff m <= n and m is visible; the window prunes pair
 * terms of the visible cells exactly as atflash_prefill_ex, and invisible keys
 * take no part in the softmax.  q, k, v bf16 (the tensor-core path, D in
 * {64, 128}); out, out_dtype, lse, workspace and errors as atflash_prefill_ex
 * (block_mask NULL: ATFLASH_ERR_INVALID_ARG).
 */
int atflash_prefill_sparse(const void *q, const void *k, const void *v, const uint8_t *block_mask, void *out,
                           int B, int Hq, int Hkv, int64_t N, int D, double rope_base, double k_window,
                           int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/*
 * RoPE pre-pass on its own: rotate x [B][N][H][D] (positions 0..N-1) once and
 * write the layout atflash_prefill_packed reads.
 *   in_dtype ATFLASH_BF16: y is [B*H][D/16][N][16] bf16 ("packed"): chunk c
 *            holds pairs 8c..8c+7 of each token as (x~_r, x~_{r+D/2})
 *            interleaved, one 32-byte tensor-core K-step per token; D in {64, 128}.
 *            ATFLASH_F32: y is [B*H][N][D] fp32, pair-interleaved; even D <= 256.
 *   y must hold atflash_rope_pack_bytes(B, N, H, D, in_dtype) bytes, 256-byte aligned.
 * Angles position * theta_r are reduced modulo 2*pi in fp64.
 */
int atflash_rope_pack(const void *x, void *y, int B, int64_t N, int H, int D, double rope_base, int in_dtype,
                      cudaStream_t stream);
size_t atflash_rope_pack_bytes(int B, int64_t N, int H, int D, int in_dtype);

/*
 * Windowed attention over already rotated, packed queries and keys (outputs of
 * atflash_rope_pack with the same in_dtype, B, N, D and rope_base).  Same
 * semantics, layouts of v/out/lse and constraints as atflash_prefill_ex, except
 * that the short-row step (see "Accuracy of short rows") is not part of this
 * call: it needs the un-rotated inputs, so queue atflash_prefill_short_rows
 * after it on the same stream to get atflash_prefill_ex's bits (bf16).
 */
int atflash_prefill_packed(const void *qpack, const void *kpack, const void *v, void *out, int B, int Hq,
                           int Hkv, int64_t N, int D, double rope_base, double k_window, int in_dtype,
                           int out_dtype, float *lse, cudaStream_t stream);

/*
 * Windowed prefill of a ragged batch packed along the token axis (the
 * "variable-length" form): sequence b is tokens cu_seqlens[b] ..
 * cu_seqlens[b+1]-1, each with its own positions 0..len_b-1 and its own causal
 * attention; no token attends across a sequence boundary.  Same method,
 * window and numerics as atflash_prefill ("The idea"; the window is applied
 * per sequence with n - m measured inside the sequence).
 *   q          [total][Hq][D] bf16, un-rotated;  k, v  [total][Hkv][D] bf16.
 *   out        [total][Hq][D], bf16 (out_dtype ATFLASH_BF16) or fp32.
 *   cu_seqlens device int32 [B+1]: cu[0] = 0, non-decreasing, cu[B] = total.
 *              A sequence whose entries break these rules gets no output rows.
 *   max_seqlen host value >= every sequence length (grid size and window
 *              clamp); rows of longer sequences beyond it are not computed.
 *   D in {64, 128}; Hq % Hkv == 0.
 *   lse        NULL, or [Hq][total] fp32 (natural log-sum-exp per row).
 *   workspace  NULL (the library takes atflash_prefill_varlen_workspace_bytes
 *              from its stream-ordered pool for the call), or a caller buffer
 *              of at least that size, 256-byte aligned.
 * Errors: ATFLASH_ERR_INVALID_ARG (null pointer, shapes, total < max_seqlen),
 * ATFLASH_ERR_UNSUPPORTED (D, out_dtype), ATFLASH_ERR_ALIGNMENT,
 * ATFLASH_ERR_WORKSPACE; nothing is launched on error.
 */
int atflash_prefill_varlen(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens, int B,
                           int64_t max_seqlen, int64_t total, int Hq, int Hkv, int D, double rope_base,
                           double k_window, int out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);
size_t atflash_prefill_varlen_workspace_bytes(int Hq, int Hkv, int64_t total, int D);

/*
 * Decode over a paged KV cache (the layout serving engines keep): pages of
 * page_size tokens in one pool; keys i*page_size .. (i+1)*page_size-1 of
 * sequence b are in page block_table[b*max_pages + i].  Same method, window,
 * numerics, q/out layouts and splits as atflash_decode (bf16 caches only).
 *   page_size   a multiple of 64 (one 64-key TMA stage never straddles a page).
 *   kv_layout   ATFLASH_KV_NHD: kpages and vpages [num_pages][page_size][Hkv][D]
 *               bf16 (K rotated iff kcache_rotated);
 *               ATFLASH_KV_PACKED: kpages [num_pages][Hkv][D/16][page_size][16]
 *               bf16, rotated, in the packed chunk layout (kcache_rotated = 1),
 *               vpages as for NHD.
 *   block_table device int32 [B][max_pages]; seqlens device int32 [B],
 *               1 <= seqlens[b] <= max_pages*page_size.  A page index past
 *               the row or an id outside [0, num_pages) is an error found on
 *               the device: the kernel records ATFLASH_ERR_BAD_PAGE in the
 *               device status word (atflash_device_status) and reads zeros in
 *               its place, so that sequence's output is not valid.
 *   workspace   >= atflash_decode_workspace_bytes(B, Hq, Hkv,
 *               max_pages*page_size, D) bytes, 16-byte aligned.
 * Errors as atflash_decode, plus ATFLASH_ERR_INVALID_ARG for page_size,
 * max_pages, num_pages or kv_layout.
 */
int atflash_decode_paged(const void *q, const void *kpages, const void *vpages, const int32_t *block_table,
                         const int32_t *seqlens, void *out, int B, int Hq, int Hkv, int max_pages, int num_pages,
                         int page_size, int D, double rope_base, double k_window, int kcache_rotated, int kv_layout,
                         int out_dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Device scratch bytes atflash_decode needs (0 on invalid arguments): one split
 * state of D + 2 floats per (sequence, query head, split).  A split is 256 to
 * 4096 keys, a multiple of 64, chosen so that the B * Hkv * splits CTAs come
 * close to, without passing, a whole number of waves of 148 SMs x 3 CTAs. */
size_t atflash_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int D);

/*
 * Windowed decode: one query token per sequence over a contiguous KV cache
 * (README "Numbers"/"Using the ports": the window is one more condition on
 * which K elements are loaded).  Split-KV: each CTA streams one slice of one
 * sequence's cache, loading only the K dims kept at that slice's distances,
 * and a second kernel merges the slices' softmax states.  The merge (and, for
 * bf16 caches, the fp32 short-row step) is launched on `stream` as a
 * programmatic dependent of the kernel before it; the call captures into a
 * CUDA graph as one chain.
 *   q              [B][Hq][D]        un-rotated query of each sequence
 *   kcache, vcache keys (un-rotated unless kcache_rotated) and values, in
 *                  kv_layout ATFLASH_KV_HND [B][Hkv][Nmax][D] or
 *                  ATFLASH_KV_NHD [B][Nmax][Hkv][D]
 *   seqlens        [B] int32 device array, 1 <= seqlens[b] <= Nmax; the query
 *                  of sequence b sits at position seqlens[b] - 1
 *   out            [B][Hq][D] written (out_dtype)
 *   kcache_rotated 0: keys are rotated on load; 1: keys already rotated
 *                  (required by ATFLASH_KV_PACKED, which is bf16 only)
 *   in_dtype       element type of q, kcache, vcache (ATFLASH_BF16 or ATFLASH_F32)
 *   workspace      device buffer of >= atflash_decode_workspace_bytes(...) bytes
 *   D in {64, 128}.
 */
int atflash_decode(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                   void *out, int B, int Hq, int Hkv, int64_t Nmax, int D, double rope_base,
                   double k_window, int kcache_rotated, int kv_layout, int in_dtype, int out_dtype,
                   void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Scaled RoPE: the calls below take the per-pair frequencies theta_r as a HOST
 * table of D/2 fp64 values instead of a base, for models whose configuration
 * rescales the RoPE frequencies ("Porting to something else" derives the window
 * table from the model's RoPE configuration, rope_scaling included).  Both the
 * rotation (angle position * theta_r) and the window (w_r = floor(k * 2*pi /
 * theta_r)) use the table.  The table must be finite, in (0, pi], and
 * non-increasing in r (so that the pairs kept at any distance are a suffix of
 * the pairs); otherwise ATFLASH_ERR_INVALID_ARG.  The library reads the table
 * during the call only.  Every other argument, layout and error is that of the
 * base-taking call of the same name; a table equal to atflash_theta_table's
 * gives bit-identical results to that call.
 */
/* theta_out (HOST, D/2 fp64) = base^(-2r/D), the table the base-taking calls use. */
int atflash_theta_table(int D, double rope_base, double *theta_out);
int atflash_window_table_theta(int D, const double *theta, double k_window, int64_t N, int64_t *w_out);
int atflash_pruned_terms_theta(int64_t N, int D, const double *theta, double k_window, atflash_terms *out);
int atflash_rope_pack_theta(const void *x, void *y, int B, int64_t N, int H, int D, const double *theta,
                            int in_dtype, cudaStream_t stream);
int atflash_prefill_theta(const void *q, const void *k, const void *v, void *out, int B, int Hq, int Hkv,
                          int64_t N, int D, const double *theta, double k_window, int in_dtype, int out_dtype,
                          float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream);
int atflash_prefill_sparse_theta(const void *q, const void *k, const void *v, const uint8_t *block_mask,
                                 void *out, int B, int Hq, int Hkv, int64_t N, int D, const double *theta,
                                 double k_window, int out_dtype, float *lse, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream);
int atflash_prefill_short_rows_theta(const void *q, const void *k, const void *v, void *out, int B, int Hq,
                                     int Hkv, int64_t N, int D, const double *theta, double k_window, int out_dtype,
                                     float *lse, cudaStream_t stream);
/* qpack/kpack written by atflash_rope_pack_theta with the same table. */
int atflash_prefill_packed_theta(const void *qpack, const void *kpack, const void *v, void *out, int B, int Hq,
                                 int Hkv, int64_t N, int D, const double *theta, double k_window, int in_dtype,
                                 int out_dtype, float *lse, cudaStream_t stream);
int atflash_decode_theta(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                         void *out, int B, int Hq, int Hkv, int64_t Nmax, int D, const double *theta,
                         double k_window, int kcache_rotated, int kv_layout, int in_dtype, int out_dtype,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream);
int atflash_prefill_varlen_theta(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens,
                                 int B, int64_t max_seqlen, int64_t total, int Hq, int Hkv, int D,
                                 const double *theta, double k_window, int out_dtype, float *lse, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream);
int atflash_decode_paged_theta(const void *q, const void *kpages, const void *vpages, const int32_t *block_table,
                               const int32_t *seqlens, void *out, int B, int Hq, int Hkv, int max_pages,
                               int num_pages, int page_size, int D, const double *theta, double k_window,
                               int kcache_rotated, int kv_layout, int out_dtype, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream);

/*
 * Decode that allocates nothing (no counterpart in the paper; an addition of
 * this library).  For callers that cannot allocate device memory at the call
 * site, e.g. a serving loop that must never enter the CUDA allocator once it
 * is running, or a plugin whose host framework owns all device memory.  Same
 * arguments and results as atflash_decode, without the workspace: the split
 * states live in a fixed device array of ATFLASH_NOALLOC_SCRATCH_BYTES that
 * every GPU loading the library reserves until the process exits.
 *   Returns ATFLASH_ERR_WORKSPACE, launching nothing, when the problem needs
 *   more than that (atflash_decode_workspace_bytes() > the limit).
 *   The array is part of the library's device image: every process that loads
 *   the library holds these 32 MiB on every GPU it uses, whether or not it
 *   calls this entry point.
 *   Arguments are checked exactly as atflash_decode checks them (same status
 *   for the same bad argument).
 *   Every call on a device shares the array: calls whose work overlaps on the
 *   GPU race; calls on one stream are ordered.  The first call on a device
 *   looks up the array's address with that device current and keeps it; make
 *   it before any stream capture begins, and do not reset the device
 *   (cudaDeviceReset) after it.
 */
#define ATFLASH_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int atflash_decode_noalloc(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                           void *out, int B, int Hq, int Hkv, int64_t Nmax, int D, double rope_base,
                           double k_window, int kcache_rotated, int kv_layout, int in_dtype, int out_dtype,
                           cudaStream_t stream);

/*
 * Device status word of the current device: ATFLASH_OK, ATFLASH_ERR_TIMEOUT
 * when a kernel's bounded wait ran out, or ATFLASH_ERR_BAD_PAGE when a paged
 * decode met a bad page index, since the last clear (the first such event is
 * kept).  Synchronises the device.  clear != 0 resets the word.
 */
int atflash_device_status(int clear);

/*
 * Limit, in milliseconds, of every pipeline wait (an mbarrier wait between the
 * warps of a CTA) in the kernels launched after this call; initially
 * ATFLASH_WAIT_LIMIT_MS from the environment, else 2000.  When a wait runs out
 * the CTA records ATFLASH_ERR_TIMEOUT in the device status word, lets its own
 * copies and tensor-core work finish (those waits use at least 200 ms) and
 * exits; its output is then incomplete.  Returns ATFLASH_ERR_INVALID_ARG unless
 * 0 < ms <= 60000.  Not part of the method; it exists to bound failures.
 */
int atflash_set_wait_limit_ms(double ms);

/*
 * Failure-detection self-test: launches one CTA on `stream` that waits, with
 * the bounded wait the kernels use, on an mbarrier that nothing completes, for
 * `limit_ms` milliseconds (0 < limit_ms <= 10000), then records
 * ATFLASH_ERR_TIMEOUT in the device status word and returns.  The call itself
 * returns ATFLASH_OK once launched; read the outcome with
 * atflash_device_status.  Not part of the method.
 */
int atflash_selftest_wait_timeout(double limit_ms, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATFLASH_H */
