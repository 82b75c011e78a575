/*
 * lsa.h — C ABI of liblsa.so: indexed sparse attention over a GQA KV cache on
 * NVIDIA B200 (sm_100a).
 *
 * One decode step, per sequence b and KV head h (Joint Subspace Sparse
 * Attention for Efficient Long-Context Decoding, Fig. 1 and Key contributions):
 *   q_bar[b,h]  = mean of the projected queries qt[b,i] of h's query group
 *   s[b,h,t]    = q_bar[b,h] . kt[b,t,h]            for every cached t
 *   S[b,h]      = top-B positions of s[b,h,:]       (ties: lower position)
 *   out[b,i]    = softmax attention of q[b,i] over K/V rows S[b,h], read in
 *                 place from the [T, hkv, d] cache (no gather copy)
 * optionally coarse-to-fine over block centroids first (LongCat Sparse
 * Attention: Taming the Lightning via Streaming-aware Hierarchical Cross-Layer
 * Indexing, Abstract, strategy (3) Hierarchical Indexing), plus the prefill
 * indexer (the same scoring and top-B for every query row of a prefill, causal)
 * and prefill indexed attention.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers, owned by the caller. The library
 *     never allocates, frees or synchronizes; every call enqueues its kernels on
 *     `stream` (a cudaStream_t passed as void*, NULL = legacy default stream)
 *     and returns at once.
 *   - Arguments are validated on the host before anything is launched; a
 *     validation failure returns a negative lsa_status and launches nothing.
 *   - Pointers must be 16-byte aligned and tensors densely packed, row-major,
 *     in the layouts given below. bf16 tensors are passed as lsa_bf16 (raw
 *     16-bit storage of bfloat16 values).
 *   - GQA grouping: query head i belongs to KV head i / G, G = hq / hkv.
 *   - Index sets are int32, strictly ascending, padded at the end with -1 when
 *     fewer than B candidates exist. NaN scores mark non-candidates.
 *   - Supported sizes: r in {16, 32, 64, 128}; d in {64, 128, 256};
 *     1 <= hkv, hkv * r <= 4096; G = hq / hkv in {1, 2, 4, 8, 16};
 *     1 <= T <= 2^31 - 1; 1 <= B <= 65536 (the attention entries
 *     lsa_indexed_attn, lsa_indexed_attn_paged and lsa_indexed_attn_noalloc,
 *     which only read index sets, and lsa_workspace_size accept B <= 2^24, so
 *     that one index set can cover a whole cache). Other sizes return
 *     LSA_ERR_UNSUPPORTED.
 *   - Errors found on the device (an index outside [-1, T), a bounded wait that
 *     ran out) are OR-ed into a status word at the start of the workspace;
 *     read it with lsa_read_device_status. Kernels never trap.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LSA_API __attribute__((visibility("default")))
#else
#define LSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int lsa_status;
enum {
    LSA_OK = 0,
    LSA_ERR_ARG = -1,         /* null pointer, non-positive size, hq % hkv != 0 */
    LSA_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
    LSA_ERR_SHAPE = -3,       /* inconsistent sizes (e.g. q_start + nq > T) */
    LSA_ERR_WORKSPACE = -4,   /* workspace missing, misaligned (256 B) or too small */
    LSA_ERR_CUDA = -5,        /* a CUDA launch failed (cudaGetLastError) */
    LSA_ERR_TIMEOUT = -6,     /* reserved: device-side bounded wait ran out (status word) */
    LSA_ERR_UNSUPPORTED = -7, /* sizes outside the supported set above */
    LSA_ERR_SCRATCH = -8      /* sizes need more than the fixed scratch of
                                 lsa_indexed_attn_noalloc holds */
};

/* Bits of the device status word (lsa_read_device_status). */
enum {
    LSA_DEV_OK = 0,
    LSA_DEV_BAD_INDEX = 1,    /* an index outside [-1, T) was skipped */
    LSA_DEV_TIMEOUT = 2       /* a bounded wait ran out; outputs are incomplete */
};

typedef uint16_t lsa_bf16;
typedef uint8_t lsa_fp8_e4m3;   /* OCP FP8 E4M3 storage (1 byte per value) */

/* Problem sizes. batch sequences, hq query heads, hkv KV heads, head dim d,
 * scoring-subspace rank r (the projected-key cache width), cache length T. */
typedef struct lsa_dims {
    int batch, hq, hkv, d, r, T;
} lsa_dims;

/* Library version (major * 10000 + minor * 100 + patch). */
LSA_API int lsa_version(void);

/* Human-readable name of a status code. Never NULL. */
LSA_API const char* lsa_status_string(lsa_status s);

/* Bytes of workspace needed by lsa_topk, lsa_indexed_attn and lsa_decode_step
 * for these sizes. blk = tokens per block and nblk_keep = blocks kept in
 * coarse-to-fine mode; pass 0, 0 for flat scoring. Returns 0 for invalid
 * sizes. The workspace must be 256-byte aligned and zero-filled before its
 * first use (e.g. cudaMemsetAsync); every completed call leaves its internal
 * counters at zero again, so it is reusable without re-zeroing. Calls that
 * share one workspace must not overlap on the GPU (one stream, or ordered). */
LSA_API size_t lsa_workspace_size(const lsa_dims* dims, int B, int blk, int nblk_keep);

/* Group-mean candidate scoring (JSSA, Fig. 1; Fig. 2a "channel budget r").
 *   qt     [batch, hq, r]      bf16  projected queries
 *   kt     [batch, T, hkv, r]  bf16  projected-key cache
 *   scores [batch, hkv, T]     fp32  out: q_bar[b,h] . kt[b,t,h]
 * q_bar is the mean of the group's projected queries; the group sum is formed
 * in fp32, the dot product accumulates in fp32, and the result is divided by G
 * (exact when G is a power of two). Integer-valued inputs give exact scores. */
LSA_API lsa_status lsa_score(const lsa_dims* dims, const lsa_bf16* qt, const lsa_bf16* kt,
                     float* scores, void* stream);

/* Top-B selection per row (JSSA, Fig. 1 "select the top-B token positions").
 *   scores [batch * hkv, T] fp32   one row per (b, h); NaN = not a candidate
 *   idx    [batch * hkv, B] int32  out: the B positions with the largest
 *          scores, ties broken toward the lower position, ascending, -1 padded
 * ws may be NULL (ws_bytes 0); if given, its status word is not touched.
 * -0.0 and +0.0 compare equal. Deterministic: identical inputs give identical
 * outputs. */
LSA_API lsa_status lsa_topk(const lsa_dims* dims, const float* scores, int B, int32_t* idx,
                    void* ws, size_t ws_bytes, void* stream);

/* Gather-free indexed attention (JSSA, Key contributions; Fig. 1).
 *   q    [batch, hq, d]      bf16
 *   k, v [batch, T, hkv, d]  bf16  the standard GQA KV cache, read in place
 *   idx  [batch, hkv, B]     int32 per-KV-head index sets (-1 entries skipped)
 *   out  [batch, hq, d]      bf16  out: softmax(scale * q . K[S]) V[S], fp32
 *                                  accumulation, rounded to nearest even
 * Entries outside [-1, T) are skipped and set LSA_DEV_BAD_INDEX. A head whose
 * set is empty gets a zero output. ws: lsa_workspace_size(dims, B, 0, 0). */
LSA_API lsa_status lsa_indexed_attn(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* k,
                            const lsa_bf16* v, const int32_t* idx, int B, float scale,
                            lsa_bf16* out, void* ws, size_t ws_bytes, void* stream);

/* Bytes of the fixed per-device scratch buffer of lsa_indexed_attn_noalloc. */
#define LSA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* lsa_indexed_attn without a workspace, for callers that cannot allocate
 * device memory where they make the call: a host thread that must not call
 * cudaMalloc/cudaFree (both can synchronize the whole device and stall other
 * streams), or code inside a framework that owns all device memory and hands
 * out no scratch. The papers have no counterpart of this call; it is a
 * deployment convenience around the same attention kernel.
 * Arguments, supported sizes and results are those of lsa_indexed_attn,
 * except:
 *   - The split-softmax partials and merge counters live in one buffer of
 *     LSA_NOALLOC_SCRATCH_BYTES per device inside liblsa.so. The library
 *     allocates nothing: no cudaMalloc, no cudaFree, no allocating routine.
 *   - Sizes that need more than that buffer return LSA_ERR_SCRATCH and launch
 *     nothing. Every size with
 *       batch * hkv * (4 + G * ceil(B / 64) * (d + 2) * 4) + 768
 *         <= LSA_NOALLOC_SCRATCH_BYTES
 *     is accepted (batch 4, hkv 8, G 4, d 128, B 2048 needs at most 2.2 MB);
 *     larger ones often fit as well, since the split uses fewer slots.
 *   - dev_status: NULL, or a caller-owned device int32 (4-byte aligned) into
 *     which the LSA_DEV_* bits are OR-ed; the caller zeroes it.
 *   - The first call on each device (the device current at the call) does a
 *     one-time setup: it looks up the buffer's device address, zero-fills the
 *     buffer on `stream` and waits for `stream`. Make that first call before
 *     any stream capture begins; a first call on a capturing stream returns
 *     LSA_ERR_CUDA and enqueues nothing. The setup is kept for the life of
 *     the process and is not redone after cudaDeviceReset (which reloads the
 *     library's device image elsewhere): do not call this entry point on a
 *     device after resetting it.
 *   - Only the merge counters at the start of the buffer must be zero when a
 *     call starts; the setup zeroes them and every completed call leaves
 *     them at zero. The partials need no initial value.
 *   - All calls on one device share the buffer, so calls that overlap on the
 *     GPU (unordered streams, concurrent host threads) race and produce wrong
 *     outputs. Order them, e.g. on one stream. */
LSA_API lsa_status lsa_indexed_attn_noalloc(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* k,
                                    const lsa_bf16* v, const int32_t* idx, int B, float scale,
                                    lsa_bf16* out, int32_t* dev_status, void* stream);

/* One whole decode step: scoring, top-B and indexed attention (JSSA, Fig. 1).
 *   q [batch, hq, d], qt [batch, hq, r], k/v [batch, T, hkv, d],
 *   kt [batch, T, hkv, r]: as above.
 *   centroids  NULL for flat scoring; else [batch, ceil(T/blk), hkv, r] bf16
 *              block centroids (lsa_block_centroids) for coarse-to-fine mode:
 *              score the centroids, keep the nblk_keep best blocks (ties: the
 *              lower block), score the tokens of those blocks, take the top B
 *              (LongCat Sparse Attention, Abstract, strategy (3)).
 *   idx_out    NULL, or [batch, hkv, B] int32 to receive the index sets.
 *   out        [batch, hq, d] bf16.
 * Selection inside the step ranks the group-sum scores (G times the mean),
 * which orders positions exactly as the mean does. */
LSA_API lsa_status lsa_decode_step(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* qt,
                           const lsa_bf16* k, const lsa_bf16* v, const lsa_bf16* kt,
                           const lsa_bf16* centroids, int blk, int nblk_keep, int B,
                           float scale, int32_t* idx_out, lsa_bf16* out,
                           void* ws, size_t ws_bytes, void* stream);

/* FP8 projected-key cache (JSSA, Fig. 10: the projected-key cache may be held
 * in FP8 while the KV cache and the attention stay in BF16). lsa_score and the
 * flat-mode lsa_decode_step with kt [batch, T, hkv, r] stored as OCP FP8 E4M3,
 * which halves the bytes the scorer streams. Every E4M3 value converts to fp32
 * exactly, so scores and index sets equal those of a bf16 cache holding the
 * same values (e.g. integers of magnitude at most 16, or multiples of 4 up to
 * 32). r must be 64 and hkv one of 4, 8, 16, 32; other sizes return
 * LSA_ERR_UNSUPPORTED. Workspace: lsa_workspace_size(dims, B, 0, 0). */
LSA_API lsa_status lsa_score_fp8(const lsa_dims* dims, const lsa_bf16* qt, const lsa_fp8_e4m3* kt,
                                 float* scores, void* stream);

LSA_API lsa_status lsa_decode_step_fp8(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* qt,
                                       const lsa_bf16* k, const lsa_bf16* v, const lsa_fp8_e4m3* kt, int B,
                                       float scale, int32_t* idx_out, lsa_bf16* out, void* ws,
                                       size_t ws_bytes, void* stream);

/* Block centroids for coarse-to-fine scoring (LongCat Sparse Attention,
 * Abstract, strategy (3); Latent Sparse Attention, summary: queries score
 * clusters instead of every key).
 *   kt        [batch, T, hkv, r]           bf16
 *   centroids [batch, ceil(T/blk), hkv, r] bf16  out: sum of the block's
 *             (up to blk) projected keys, fp32 sum rounded to nearest even
 * blk in [1, 4096]. Blocks start at t = 0; the last one may be partial. */
LSA_API lsa_status lsa_block_centroids(const lsa_dims* dims, const lsa_bf16* kt, int blk,
                               lsa_bf16* centroids, void* stream);

/* ---- Paged KV cache, page size 1 ("Their 42x decode speedup never compiled
 * on my GPU", What their numbers claim: the release's serving configurations
 * pin a KV page size of 1, one token per page, which token-level index sets
 * need). K and V live in pools k_pool / v_pool [nslots, hkv, d] bf16, and
 * page_table [batch, T] int32 gives the pool slot of logical position t of
 * sequence b. The index sets stay logical positions; attention reads row
 * (page_table[b, t], h) of the pools in place. A slot outside [0, nslots)
 * for a selected position is skipped and sets LSA_DEV_BAD_INDEX. The
 * projected-key cache kt stays contiguous [batch, T, hkv, r]. nslots >= 1,
 * page_table 16-byte aligned. Workspace: lsa_workspace_size(dims, B, 0, 0). */
LSA_API lsa_status lsa_indexed_attn_paged(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* k_pool,
                                          const lsa_bf16* v_pool, int nslots, const int32_t* page_table,
                                          const int32_t* idx, int B, float scale, lsa_bf16* out, void* ws,
                                          size_t ws_bytes, void* stream);

/* lsa_decode_step (flat scoring) with the KV cache in paged pools. */
LSA_API lsa_status lsa_decode_step_paged(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* qt,
                                         const lsa_bf16* k_pool, const lsa_bf16* v_pool, int nslots,
                                         const int32_t* page_table, const lsa_bf16* kt, int B, float scale,
                                         int32_t* idx_out, lsa_bf16* out, void* ws, size_t ws_bytes,
                                         void* stream);

/* Cross-layer index reuse (LongCat Sparse Attention, Abstract, strategy (2)
 * Cross-Layer Indexing: one layer's index sets serve the consecutive layers)
 * needs no entry of its own: pass the idx that lsa_decode_step (idx_out) or
 * lsa_topk produced for one layer to lsa_indexed_attn / lsa_indexed_attn_paged
 * with the next layers' q, k and v. */

/* ---- Scoring preparation (JSSA, Fig. 9: the key projection that fills the
 * projected-key cache; Fig. 1: keys and the group's queries are scored in a
 * shared low-dimensional subspace). Every basis P[j] holds r vectors of length
 * d; row i of x uses basis i / G with G = H / nbases:
 *   y[b, t, i, c] = sum_e P[i / G, c, e] * x[b, t, i, e]
 * accumulated in fp32 on the tensor cores and rounded to nearest even once.
 * Keys: x = k [batch, T, hkv, d], H = nbases = hkv, y = kt.
 * Queries: x = q viewed as [batch, 1, hq, d] (T = 1, t0 = 0, n = 1),
 *          nbases = hkv, y = qt viewed as [batch, 1, hq, r].
 * (One basis per layer: nbases = 1.) */
typedef struct lsa_proj_dims {
    int batch, T, H, d, r, nbases;
} lsa_proj_dims;

/* Project rows t0 .. t0 + n - 1 of every sequence (0 <= t0, n >= 0,
 * t0 + n <= T; n = 0 does nothing); other rows of y are left untouched.
 *   x [batch, T, H, d] bf16   P [nbases, r, d] bf16   y [batch, T, H, r] bf16
 * Sizes: H % nbases == 0; d a multiple of 16 with d in {16, 32} or
 * 64 <= d <= 256; r a multiple of 16 in [16, 128]; batch * T < 2^31; other
 * sizes return LSA_ERR_UNSUPPORTED (d = 256 with r above 80 does not fit the
 * staging buffers). x, P, y 16-byte aligned.
 * dev_status: NULL, or a caller-owned device int32 into which LSA_DEV_TIMEOUT
 * is OR-ed if a bounded wait ran out. The call allocates nothing. */
LSA_API lsa_status lsa_project(const lsa_proj_dims* dims, const lsa_bf16* x, const lsa_bf16* P, int t0,
                               int n, lsa_bf16* y, int32_t* dev_status, void* stream);

/* lsa_project with an FP8 E4M3 output (JSSA, Fig. 10: the projected-key cache
 * held in FP8): each fp32 projection rounds to nearest even E4M3, saturated to
 * +-448. y [batch, T, H, r] lsa_fp8_e4m3. */
LSA_API lsa_status lsa_project_fp8(const lsa_proj_dims* dims, const lsa_bf16* x, const lsa_bf16* P, int t0,
                                   int n, lsa_fp8_e4m3* y, int32_t* dev_status, void* stream);

/* Incremental block centroids (LongCat Sparse Attention, Abstract, strategy
 * (3)): for every sequence and KV head, add the projected keys of positions
 * t0 .. t0 + n - 1 to the centroid of their block, in position order,
 * rounding the sum to bf16 after every add:
 *   centroids[b, t / blk, h, :] <- bf16(centroids[b, t / blk, h, :] + kt[b, t, h, :])
 *   kt [batch, T, hkv, r] bf16 (dims.T = capacity), centroids [batch, ceil(T/blk), hkv, r]
 * Starting from zeros and adding a block's tokens gives lsa_block_centroids'
 * value whenever the partial sums are exact in bf16 (e.g. small integers).
 * 0 <= t0, n >= 0, t0 + n <= T, blk in [1, 4096]. */
LSA_API lsa_status lsa_update_centroids(const lsa_dims* dims, const lsa_bf16* kt, int blk, int t0, int n,
                                        lsa_bf16* centroids, void* stream);

/* Bytes of workspace for lsa_prefill_index / lsa_prefill_attn (one workspace
 * serves both; calls that share it must not overlap on the GPU). The attention
 * merge counters in it must be zero before the first lsa_prefill_attn (zero-fill
 * the workspace once); every completed call leaves them at zero. Returns 0 for
 * invalid sizes (batch != 1, nq < 1). */
LSA_API size_t lsa_prefill_workspace_size(const lsa_dims* dims, int nq, int B);

/* Prefill indexer (LongCat Sparse Attention, Abstract: the Lightning Indexer's
 * dense O(L^2) scoring; JSSA, Fig. 1 for the group-mean query): for each of nq
 * query rows at absolute positions q_start .. q_start + nq - 1, score every
 * key t <= p with the row's group mean and take the top B (causal).
 *   dims.batch must be 1; dims.T = cache length (the queries' own keys are in
 *   the cache, so q_start + nq <= T).
 *   qt  [nq, hq, r]   bf16     kt [T, hkv, r] bf16
 *   idx [nq, hkv, B]  int32    out, ascending, -1 padded (rows with p+1 < B)
 * The group mean is rounded to bf16 for the tensor-core contraction (exact when
 * it is a multiple of 2^-k representable in bf16, e.g. integer inputs).
 * Limits: T <= 2^18 (the per-row output bitmap lives in shared memory; larger
 * caches return LSA_ERR_UNSUPPORTED). ws: lsa_prefill_workspace_size(dims, nq,
 * B) bytes, 256-byte aligned, no initial value needed (its buffers are written
 * before they are read); about 3.26 GiB for nq = 4096, T = 128K, B = 2048. */
LSA_API lsa_status lsa_prefill_index(const lsa_dims* dims, const lsa_bf16* qt, int nq, int q_start,
                             const lsa_bf16* kt, int B, int32_t* idx,
                             void* ws, size_t ws_bytes, void* stream);

/* Prefill indexed attention: lsa_indexed_attn for each of nq query rows, the
 * G heads of a KV head sharing that row's index set.
 *   q [nq, hq, d], k/v [T, hkv, d], idx [nq, hkv, B], out [nq, hq, d]. */
LSA_API lsa_status lsa_prefill_attn(const lsa_dims* dims, const lsa_bf16* q, int nq,
                            const lsa_bf16* k, const lsa_bf16* v, const int32_t* idx, int B,
                            float scale, lsa_bf16* out, void* ws, size_t ws_bytes, void* stream);

/* Enqueue a copy of the workspace's device status word into *host_flags
 * (pinned or pageable host memory); synchronize `stream` before reading it. */
LSA_API lsa_status lsa_read_device_status(const void* ws, int32_t* host_flags, void* stream);

/* Enqueue a reset of the workspace's device status word to LSA_DEV_OK. */
LSA_API lsa_status lsa_clear_device_status(void* ws, void* stream);

/* Test hook: nanoseconds of device time after which a device-side wait gives
 * up and sets LSA_DEV_TIMEOUT (default 2e9; 0 = give up at the first failed
 * probe; negative restores the default). It affects only launches enqueued
 * after the call. Process-wide. */
LSA_API void lsa_debug_set_wait_limit(long long ns);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
