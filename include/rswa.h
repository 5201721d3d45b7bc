/*
 * rswa.h -- C ABI of librswa.so: R-SWA / SR-SWA decode attention on B200 (sm_100a).
 *
 * Reference Sliding Window Attention (R-SWA): every query attends to a static
 * reference prefix of m tokens (all page visual tokens plus the prompt, never
 * evicted) and to a ring buffer holding the last n generated tokens, so the KV
 * cache holds L_m + min(n, T) tokens after T generated tokens
 *   ("百度Unlimited OCR" paper summary, lshu.cn/news/33052, §二.1 核心设计逻辑
 *    and §二.2 数学与KV缓存优势).
 * SR-SWA, its sparse successor, cuts the prefix into 32-token blocks, scores
 * each block against the query with a low-dimensional index projection, runs
 * a 1.5-entmax over the scores, keeps the top-16 blocks and adds log(prob) of
 * each kept block as a bias inside the attention softmax
 *   (Unlimited-OCR-2 SR-SWA explainer, nxmr.cn/news/162408, 稀疏路由 steps 1-4).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers into caller-owned memory, 16-byte
 *   aligned, dense row-major in the layouts given. The library never
 *   allocates device memory on a call and never keeps a pointer after a call
 *   returns (kernels may still be running on `stream`).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call only enqueues work on it and returns; nothing synchronises
 *   except rswa_check_status.
 * - bf16 = IEEE bfloat16 bit pattern (2 bytes); f32 = IEEE binary32.
 * - Host-side validation runs before any launch. On failure the call returns
 *   a non-zero rswa_status, launches nothing, and rswa_last_error() describes
 *   the problem. Values that live in device memory (prefix_len, wp, fill,
 *   blk_idx) are range-checked inside the kernels: an out-of-range value is
 *   skipped (its rows are not read) and RSWA_DEVICE_* bits are OR-ed into the
 *   status word of the workspace (or of `status` for rswa_append), which
 *   rswa_check_status reads back. No kernel traps.
 * - Outputs are f32. lse is the natural-log log-sum-exp of the scores a query
 *   attended to (-inf if it attended to nothing; out is then 0).
 * - Layout: per (sequence, head) every K/V row of head_dim 128 bf16 is 256
 *   contiguous bytes, and a sequence's rows for one head are contiguous, so a
 *   32-token block of one head is one 8 KiB run of memory.
 */
#ifndef RSWA_H
#define RSWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RSWA_API __attribute__((visibility("default")))
#else
#define RSWA_API
#endif

typedef enum {
  RSWA_OK = 0,
  RSWA_ERR_INVALID = 1,      /* bad argument (null pointer, size, alignment, too-small workspace) */
  RSWA_ERR_UNSUPPORTED = 2,  /* valid but not built for (head_dim != 128, too many blocks, ...) */
  RSWA_ERR_CUDA = 3,         /* a CUDA runtime call failed; see rswa_last_error() */
  RSWA_ERR_DEVICE_CHECK = 5  /* returned by rswa_check_status when a device-side check tripped */
} rswa_status;

/* Bits of the device status word. */
#define RSWA_DEVICE_BAD_PREFIX_LEN 0x1 /* prefix_len[b] < 0 or > prefix_cap: sequence skipped        */
#define RSWA_DEVICE_BAD_RING_STATE 0x2 /* wp[b] not in [0, n) or fill[b] not in [0, n]: ring skipped */
#define RSWA_DEVICE_BAD_BLOCK_IDX 0x4  /* blk_idx entry >= number of prefix blocks: entry skipped    */
#define RSWA_DEVICE_WAIT_TIMEOUT 0x8   /* a bounded pipeline wait gave up (the output is not valid)  */
#define RSWA_DEVICE_PIPELINE 0x10      /* a pipeline stage held an unexpected tile (output not valid) */

typedef struct {
  int32_t batch;      /* B: sequences                                                   */
  int32_t heads;      /* H: attention heads (query heads == KV heads), 1..128            */
  int32_t head_dim;   /* D: must be 128                                                  */
  int32_t ring;       /* n: ring slots per (sequence, head), 1..1024 (the pages use 128) */
  int64_t prefix_cap; /* cap: rows allocated per (sequence, head) in the prefix K/V      */
} rswa_dims;

/* Operation codes for rswa_workspace_bytes. */
#define RSWA_OP_DECODE 1        /* rswa_decode, rswa_decode_fp8, rswa_decode_append          */
#define RSWA_OP_SRSWA_DECODE 2  /* srswa_decode, srswa_decode_fp8, srswa_decode_append
                                   (any topk in 1..32)                                      */
#define RSWA_OP_ROUTE 3         /* srswa_route, srswa_route_tokens (256 bytes)               */
#define RSWA_OP_PREFILL 4       /* rswa_prefill (256 bytes); srswa_prefill: srswa_prefill_workspace_bytes */
#define RSWA_OP_SRSWA_ROUTED 5  /* srswa_decode_routed, srswa_step (any topk in 1..32)       */

/* Message of the last failed call on this host thread ("" if none). */
RSWA_API const char* rswa_last_error(void);

/* Library ABI version (incremented when entry points are added or changed): 2 adds the
 * FP8 prefix, the fused decode step and the SR-SWA chunked prefill to version 1; 3 adds
 * the page2d rotary encoding (rswa_rope_page2d, rswa_append_rope); 4 the FP8 ring
 * (rswa_append_fp8, rswa_decode_fp8kv, srswa_decode_fp8kv), the fused router
 * (srswa_decode_routed, srswa_step) and the wait-timeout test hook; 5 the fused steps
 * with the page2d encoding (rswa_decode_append_rope, srswa_step_rope). */
RSWA_API int32_t rswa_version(void);

/*
 * Bytes of device workspace `op` needs for these dims. The workspace holds a
 * status word, per-(sequence, head) completion counters and split-KV
 * partials. It must be zero-filled once before its first use; every call that
 * completes leaves the counters at zero again, so it can be reused by later
 * calls on the same stream. Calls that share a workspace must not overlap in
 * time (use one workspace per stream). Returns 0 for invalid dims.
 */
RSWA_API size_t rswa_workspace_bytes(const rswa_dims* dims, int32_t op);

/*
 * Synchronises `stream`, reads the workspace's device status word into
 * *device_status (may be NULL) and clears it. Returns RSWA_OK if it was zero,
 * RSWA_ERR_DEVICE_CHECK otherwise, RSWA_ERR_CUDA if the copy failed.
 * If RSWA_DEVICE_WAIT_TIMEOUT is set, CTAs that gave up may have left completion
 * counters behind, so all ws_bytes of the workspace are zero-filled again (its
 * initial state) and it can be reused; otherwise only the status word is cleared.
 * Also accepts the `status` pointer given to rswa_append (ws_bytes >= 4).
 */
RSWA_API rswa_status rswa_check_status(void* workspace, size_t ws_bytes, int32_t* device_status, void* stream);

/*
 * Test hook for the bounded-wait path (failure detection without a GPU fault; the
 * pages have no counterpart). Every pipeline wait of the decode kernels gives up after
 * a time limit (2 s by default), sets RSWA_DEVICE_WAIT_TIMEOUT, lets its CTA's copies
 * in flight land (bounded by the same limit) and ends the CTA, so the call returns and
 * the CUDA context stays usable. This call arms, for the NEXT decode-family call made
 * by the calling host thread only (rswa_decode*, srswa_decode*, srswa_prefill,
 * rswa_decode_noalloc; consumed by that call even if it fails validation):
 *   drop_tile     : >= 0: CTA 0 neither arms nor fills the shared-memory stage of its
 *                   CTA-local tile number drop_tile, so that tile's bounded wait runs
 *                   out (no copy is in flight for it); -1: nothing dropped.
 *   wait_limit_ns : the wait limit for that call, in [1e3, 1e10] ns.
 * Returns RSWA_ERR_INVALID for values out of range. Not for production use.
 */
RSWA_API rswa_status rswa_test_arm_wait_timeout(int32_t drop_tile, int64_t wait_limit_ns);

/*
 * Ring append (one generated token per sequence).
 * The new token's K and V overwrite ring slot wp[b] of every head of sequence
 * b, then wp[b] <- (wp[b] + 1) mod n and fill[b] <- min(fill[b] + 1, n);
 * slot_out[b] (nullable) receives the slot written.
 *   (SR-SWA explainer, 环形缓冲: the newest token overwrites the oldest slot in
 *    place and the write pointer advances cyclically; "百度 Unlimited OCR 深度实战"
 *    tutorial, chenxutan.com/d/4055.html, §3.3.2: a window of at most n K/V.)
 * ring_k, ring_v : bf16 [B][H][n][D], updated in place.
 * k_new, v_new   : bf16 [B][H][D].
 * wp, fill       : int32 [B], updated in place. The ring's valid slots are the
 *                  fill[b] most recently written: (wp - fill + i) mod n, i < fill.
 * slot_out       : int32 [B] or NULL.
 * status         : int32 device word or NULL; RSWA_DEVICE_BAD_RING_STATE is
 *                  OR-ed in (and the sequence left untouched) if wp[b] is out of range.
 */
RSWA_API rswa_status rswa_append(const rswa_dims* dims, void* ring_k, void* ring_v, const void* k_new, const void* v_new,
                        int32_t* wp, int32_t* fill, int32_t* slot_out, int32_t* status, void* stream);

/*
 * R-SWA decode: for every (b, h), one query attends to prefix rows
 * [0, prefix_len[b]) and to the ring's valid slots (which, after this step's
 * rswa_append, include the query's own token):
 *   out[b][h] = softmax(scale * q K^T) V over that key set.
 *   (paper summary §二.1; tutorial §2.2.1 and §3.3.1.)
 * Split-KV flash decoding: each CTA streams 32-row K/V tiles through a shared-
 * memory pipeline filled by bulk async copies, keeps an online softmax, and
 * the last CTA of a (b, h) merges the partials by log-sum-exp.
 * q              : bf16 [B][H][D]
 * pk, pv         : bf16 [B][H][prefix_cap][D]
 * prefix_len     : int32 [B], each in [0, prefix_cap]
 * ring_k, ring_v : bf16 [B][H][n][D];  wp, fill : int32 [B] (as after rswa_append)
 * scale          : softmax scale (1/sqrt(D) in the model)
 * out            : f32 [B][H][D];  lse : f32 [B][H] or NULL
 * workspace      : zero-initialised device buffer of rswa_workspace_bytes(dims, RSWA_OP_DECODE) bytes
 */
RSWA_API rswa_status rswa_decode(const rswa_dims* dims, const void* q, const void* pk, const void* pv,
                        const int32_t* prefix_len, const void* ring_k, const void* ring_v, const int32_t* wp,
                        const int32_t* fill, float scale, float* out, float* lse, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * R-SWA chunked prefill: for every (b, h) and output-side query i in [0, T),
 *   out[b][h][i] = softmax(scale q_i K^T) V over the prefix rows [0, prefix_len[b])
 *                  and the chunk's outputs j with i - n < j <= i
 * (the most recent n outputs including itself). Positions j < 0 belong to a
 * previous chunk: they are read from the ring when one is given (position -r
 * is the r-th most recently written slot, (wp - r) mod n, present if r <= fill).
 *   (tutorial §3.3.1: reference positions always visible, only the most recent
 *    n output positions visible; paper summary §二.1.)
 * Tensor cores: tcgen05.mma with TMEM accumulators, operands staged by TMA.
 * T              : chunk length, >= 1
 * q, k_out, v_out: bf16 [B][H][T][D]  (the chunk's queries and its own keys/values)
 * pk, pv         : bf16 [B][H][prefix_cap][D];  prefix_len : int32 [B]
 * ring_k, ring_v : bf16 [B][H][n][D], wp, fill : int32 [B]; all four NULL when there is
 *                  no previous chunk (then write_ring must be 0)
 * out            : f32 [B][H][T][D];  lse : f32 [B][H][T] or NULL
 * write_ring     : 1 = afterwards leave ring/wp/fill as if the T outputs had been
 *                  appended in order with rswa_append (launched after the attention)
 * workspace      : zero-initialised, rswa_workspace_bytes(dims, RSWA_OP_PREFILL) bytes (status word)
 * Unsupported: B*H*T or B*H*prefix_cap or B*H*n at or above 2^31 rows.
 */
RSWA_API rswa_status rswa_prefill(const rswa_dims* dims, int32_t T, const void* q, const void* k_out, const void* v_out,
                                  const void* pk, const void* pv, const int32_t* prefix_len, void* ring_k, void* ring_v,
                                  int32_t* wp, int32_t* fill, float scale, float* out, float* lse, int32_t write_ring,
                                  void* workspace, size_t ws_bytes, void* stream);

/*
 * SR-SWA block index keys (run once per prefix, not per step): the prefix is
 * cut into 32-token blocks and a block's index key is the mean of its tokens'
 * index keys (a partial last block averages its valid tokens; blocks past
 * the prefix are written as zero).
 *   (SR-SWA explainer, 稀疏路由 step 1: sparse_block_size 32.)
 * k_idx : bf16 [B][prefix_cap][32] per-token index keys
 * kbar  : f32 [B][ceil(prefix_cap / 32)][32]
 */
RSWA_API rswa_status srswa_index_pool(const rswa_dims* dims, const void* k_idx, const int32_t* prefix_len, float* kbar,
                             void* stream);

/*
 * SR-SWA router, one route per sequence shared by all heads:
 *   z_c  = idx_scale * <q_idx[b], kbar[b][c]>   for the NB = ceil(prefix_len/32) prefix blocks
 *   p    = 1.5-entmax(z / 2), solved exactly (sort-based threshold) in fp32
 *   blk_idx[b] = the topk blocks by z, descending, equal scores to the smaller index;
 *                -1 past NB when NB < topk
 *   blk_logp   = ln p of each selected block (-inf where p = 0 or padded)
 *   (SR-SWA explainer, 稀疏路由 steps 2-4 and 偏置融合; top-16 = sparse_topk_blocks.)
 * Ring-window tokens are not candidates.
 * q_idx    : f32 [B][32]
 * kbar     : f32 [B][ceil(prefix_cap / 32)][32] from srswa_index_pool
 * topk     : 1..32
 * blk_idx  : int32 [B][topk];  blk_logp : f32 [B][topk]
 * probs    : f32 [B][ceil(prefix_cap / 32)] or NULL (zero past NB)
 * tau      : f32 [B] or NULL: the threshold of the x = z/2 problem
 * workspace: zero-initialised, rswa_workspace_bytes(dims, RSWA_OP_ROUTE) bytes (status word)
 * One thread-block cluster of ceil(ceil(prefix_cap / 32) / 1024) CTAs per sequence scores
 * the blocks; the CTAs exchange their maxima and hand the first CTA, through distributed
 * shared memory, the blocks with z > max z - 2 (plus their sorted top-32 when the sequence
 * has fewer than topk such blocks); the first CTA ranks them and solves the threshold.
 * Unsupported: ceil(prefix_cap / 32) > 8192.
 */
RSWA_API rswa_status srswa_route(const rswa_dims* dims, const float* q_idx, const float* kbar, const int32_t* prefix_len,
                        float idx_scale, int32_t topk, int32_t* blk_idx, float* blk_logp, float* probs, float* tau,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * SR-SWA gathered-block decode: for every (b, h) the query reads only the
 * selected blocks and the ring. A token of selected block c scores
 * scale * q.k + blk_logp[b][i]; ring tokens score scale * q.k; entries with
 * blk_idx < 0 or blk_logp = -inf are skipped.
 *   (SR-SWA explainer, "三者合起来": a fixed local window plus a fixed number of
 *    remote reference blocks per decoding step.)
 * Arguments as rswa_decode, plus blk_idx int32 [B][topk], blk_logp f32 [B][topk],
 * topk in 1..32. workspace: rswa_workspace_bytes(dims, RSWA_OP_SRSWA_DECODE).
 */
RSWA_API rswa_status srswa_decode(const rswa_dims* dims, const void* q, const void* pk, const void* pv,
                         const int32_t* prefix_len, const int32_t* blk_idx, const float* blk_logp, int32_t topk,
                         const void* ring_k, const void* ring_v, const int32_t* wp, const int32_t* fill, float scale,
                         float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * rswa_decode for callers that cannot allocate device memory (no
 * counterpart on the pages; this is an interface convenience).
 * Some callers cannot call cudaMalloc: code inside an allocator-free serving
 * loop, plugins that only receive raw pointers from a host engine owning all
 * allocations, or paths that must not touch a caching allocator. This entry
 * point computes exactly what rswa_decode computes (same arguments minus the
 * workspace), taking its scratch (status word, completion counters, split
 * partials) from a 4 MiB array of static device memory inside the library,
 * which every GPU that loads the library holds until the process exits. It
 * calls no cudaMalloc/cudaFree and no allocating library routine.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture on the device. The address is kept for the
 *   life of the process: do not use this entry point across a reset of the
 *   device (cudaDeviceReset) or after its primary context was destroyed.
 * - Every call shares the one array per device: calls whose work overlaps on
 *   the GPU (other streams, other threads) race and give wrong results.
 *   Serialise them, e.g. on one stream.
 * - Each call first zeroes the status word and completion counters it uses.
 * - status: int32 device word or NULL; if given, it receives this call's
 *   RSWA_DEVICE_* bits (copied, not OR-ed).
 * - The split-KV work is planned to fit the 4 MiB (it may use fewer splits
 *   than rswa_decode would); dims that do not fit even with one split (more
 *   than about a million (sequence, head) pairs) are rejected with
 *   RSWA_ERR_UNSUPPORTED.
 */
RSWA_API rswa_status rswa_decode_noalloc(const rswa_dims* dims, const void* q, const void* pk, const void* pv,
                                         const int32_t* prefix_len, const void* ring_k, const void* ring_v,
                                         const int32_t* wp, const int32_t* fill, float scale, float* out, float* lse,
                                         int32_t* status, void* stream);

/*
 * One decode step in one launch: rswa_append followed by rswa_decode (respectively
 * srswa_decode), fused. This step's token joins the key set straight from k_new / v_new
 * (its own key, as after an append), the oldest slot of a full ring is left out, the
 * token is written into ring slot wp[b] (slot_out[b] <- wp[b]), and wp / fill advance
 * as rswa_append advances them once the launch has read them. Same results as the two
 * calls; one kernel boundary fewer per step.
 * Arguments: those of rswa_append and rswa_decode (srswa_decode), with the ring, wp and
 * fill writable. workspace: rswa_workspace_bytes(dims, RSWA_OP_DECODE) (resp.
 * RSWA_OP_SRSWA_DECODE), zero-initialised; bytes 128..131 of its status area hold the
 * launch's completion counter (its last CTA advances wp / fill), left at zero.
 * A sequence whose wp / fill are out of range is flagged (RSWA_DEVICE_BAD_RING_STATE)
 * and left untouched, its ring read as empty and its new token not attended.
 */
RSWA_API rswa_status rswa_decode_append(const rswa_dims* dims, const void* q, const void* k_new, const void* v_new,
                                        const void* pk, const void* pv, const int32_t* prefix_len, void* ring_k,
                                        void* ring_v, int32_t* wp, int32_t* fill, int32_t* slot_out, float scale,
                                        float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

RSWA_API rswa_status srswa_decode_append(const rswa_dims* dims, const void* q, const void* k_new, const void* v_new,
                                         const void* pk, const void* pv, const int32_t* prefix_len,
                                         const int32_t* blk_idx, const float* blk_logp, int32_t topk, void* ring_k,
                                         void* ring_v, int32_t* wp, int32_t* fill, int32_t* slot_out, float scale,
                                         float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * SR-SWA decode with the router fused into the gathered-block attention: srswa_route
 * followed by srswa_decode in ONE launch (SR-SWA explainer, 稀疏路由 steps 2-4 and
 * "三者合起来": the router picks the remote blocks that the attention then reads).
 * Same route as srswa_route (blk_idx, blk_logp, tau as there; probs is not produced) and
 * the same attention output as srswa_decode over that route. Inside the launch every
 * warp first scores slices of 64 blocks (z = idx_scale <q_idx, kbar_c>) and publishes
 * each slice sorted; one CTA per sequence then merges the slices' candidates, solves the
 * exact 1.5-entmax threshold and publishes the top-k; meanwhile the attention warps
 * stream the ring (which needs no route) and wait, bounded, for their sequence's route
 * before they read the routed blocks. The CTAs of the launch wait on one another, so the
 * grid is sized to one resident wave of the kernel: do not run two of these launches
 * concurrently on one GPU (their waits would run out: RSWA_DEVICE_WAIT_TIMEOUT).
 * Arguments: srswa_decode's, with q_idx f32 [B][32], kbar f32 [B][ceil(prefix_cap/32)][32]
 * (srswa_index_pool), idx_scale, and blk_idx int32 [B][topk], blk_logp f32 [B][topk],
 * tau f32 [B] or NULL as OUTPUTS. workspace: rswa_workspace_bytes(dims,
 * RSWA_OP_SRSWA_ROUTED) bytes, zero-initialised; each launch leaves its counters at zero.
 * Unsupported: ceil(prefix_cap / 32) > 8192.
 */
RSWA_API rswa_status srswa_decode_routed(const rswa_dims* dims, const void* q, const float* q_idx, const float* kbar,
                                         float idx_scale, int32_t topk, const void* pk, const void* pv,
                                         const int32_t* prefix_len, const void* ring_k, const void* ring_v,
                                         const int32_t* wp, const int32_t* fill, float scale, int32_t* blk_idx,
                                         float* blk_logp, float* tau, float* out, float* lse, void* workspace,
                                         size_t ws_bytes, void* stream);

/*
 * The whole SR-SWA decode step in one launch: the ring append of rswa_decode_append and
 * the fused router + gathered attention of srswa_decode_routed. Results equal rswa_append,
 * srswa_route and srswa_decode called in turn. Arguments: those of srswa_decode_routed
 * plus k_new, v_new (bf16 [B][H][D]) and slot_out (int32 [B] or NULL), with ring_k,
 * ring_v, wp and fill updated in place as by rswa_append.
 */
RSWA_API rswa_status srswa_step(const rswa_dims* dims, const void* q, const void* k_new, const void* v_new,
                                const float* q_idx, const float* kbar, float idx_scale, int32_t topk, const void* pk,
                                const void* pv, const int32_t* prefix_len, void* ring_k, void* ring_v, int32_t* wp,
                                int32_t* fill, int32_t* slot_out, float scale, int32_t* blk_idx, float* blk_logp,
                                float* tau, float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * SR-SWA chunked prefill. The pages size prefill memory by a
 * per-token router score tensor of about [tokens, context/32] (serving notes,
 * --max-prefill-tokens), i.e. every output-side token of a chunk is routed by itself;
 * the rule is the decode router's (srswa_route). Reading adopted: query i of a chunk of
 * T outputs attends to its own top-k routed prefix blocks (bias ln p) and to the outputs
 * j with i - n < j <= i (bias 0); positions j < 0 come from the previous chunk's ring, as
 * in rswa_prefill.
 *
 * srswa_route_tokens: srswa_route for T router queries per sequence.
 *   q_idx    : f32 [B][T][32];  kbar : f32 [B][ceil(prefix_cap / 32)][32]
 *   blk_idx  : int32 [B][T][topk];  blk_logp : f32 [B][T][topk]
 *   workspace: >= 256 bytes (status word).  Unsupported: B * T > 65535.
 * srswa_prefill: the attention of the chunk's T queries (T <= 8192).
 *   q, k_out, v_out : bf16 [B][H][T][D] (the chunk's queries and output K/V)
 *   pk, pv, prefix_len : as srswa_decode;  blk_idx / blk_logp from srswa_route_tokens
 *   ring_k, ring_v, wp, fill : the previous chunk's ring, or all NULL for the first chunk
 *   out : f32 [B][H][T][D];  lse : f32 [B][H][T] or NULL
 *   workspace: srswa_prefill_workspace_bytes(dims, T) bytes, zero-initialised once
 *   (status word, grouping scratch, and the band part's lse when lse is NULL).
 * The routed blocks and the band are disjoint key sets, so the softmax over their union is
 * the log-sum-exp merge of one over each: the band and ring part of every query runs on the
 * tcgen05 prefill kernel (as rswa_prefill, prefix left out); the chunk's queries are grouped
 * by the set of blocks their routes select, and each group of up to 128 queries runs, per
 * head, as one 128-row tcgen05 tile against its blocks (passes of 16 blocks) with a per-
 * (query, block) bias ln p, merged into the band result. P is rounded to bf16 for the P.V
 * product, as in rswa_prefill. Route entries naming a block past prefix_len are flagged
 * (RSWA_DEVICE_BAD_BLOCK_IDX) and attend to nothing.
 */
RSWA_API rswa_status srswa_route_tokens(const rswa_dims* dims, int32_t T, const float* q_idx, const float* kbar,
                                        const int32_t* prefix_len, float idx_scale, int32_t topk, int32_t* blk_idx,
                                        float* blk_logp, void* workspace, size_t ws_bytes, void* stream);

RSWA_API size_t srswa_prefill_workspace_bytes(const rswa_dims* dims, int32_t T);

RSWA_API rswa_status srswa_prefill(const rswa_dims* dims, int32_t T, const void* q, const void* k_out,
                                   const void* v_out, const void* pk, const void* pv, const int32_t* prefix_len,
                                   const int32_t* blk_idx, const float* blk_logp, int32_t topk, const void* ring_k,
                                   const void* ring_v, const int32_t* wp, const int32_t* fill, float scale,
                                   float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * FP8 prefix cache (the Unlimited-OCR technical analysis page, "Unlimited-OCR：突破32768
 * 上下文限制的视觉语言模型技术解析", lists quantised KV-cache compression among its memory
 * measures, 内存使用效率 / KV缓存压缩, without fixing a format; the format below is this
 * library's reading). The prefix K and V are stored
 * as OCP FP8 E4M3 codes (bias 7, 3 mantissa bits, subnormals, largest finite 448, no
 * infinities) with one f32 scale per (sequence, head, 32-token block) for K and one
 * for V; an element is code value * scale. The ring stays bf16.
 *
 * rswa_quantize_prefix: for every (b, h) and block c with 32c < prefix_len[b],
 *   scale = amax / 448 over the block's valid rows and all D dims (1 if amax = 0),
 *   code  = E4M3(x / scale), round to nearest even, saturating at +-448,
 * both steps in f32. Rows of a partial block past prefix_len get code 0; blocks past
 * prefix_len are not written.
 * pk, pv       : bf16 [B][H][prefix_cap][D]
 * pk8, pv8     : uint8 codes [B][H][prefix_cap][D] (caller-owned, written)
 * k_scale, v_scale : f32 [B][H][ceil(prefix_cap / 32)] (written)
 * status       : int32 device word or NULL (RSWA_DEVICE_BAD_PREFIX_LEN)
 * Errors: host validation as rswa_decode; nothing is launched on error.
 */
RSWA_API rswa_status rswa_quantize_prefix(const rswa_dims* dims, const void* pk, const void* pv,
                                          const int32_t* prefix_len, uint8_t* pk8, uint8_t* pv8, float* k_scale,
                                          float* v_scale, int32_t* status, void* stream);

/*
 * rswa_decode over an FP8 prefix: prefix rows are read as codes (128 B per row per
 * head) and their block scales; the ring as bf16. Same key set, arguments and
 * workspace (RSWA_OP_DECODE) as rswa_decode, with pk8 / pv8 / k_scale / v_scale in
 * place of pk / pv. Streams half the prefix bytes of the bf16 call.
 */
RSWA_API rswa_status rswa_decode_fp8(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                                     const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                                     const void* ring_k, const void* ring_v, const int32_t* wp, const int32_t* fill,
                                     float scale, float* out, float* lse, void* workspace, size_t ws_bytes,
                                     void* stream);

/*
 * srswa_decode over an FP8 prefix: the routed blocks are read as codes and scales, the
 * ring as bf16. Arguments and workspace (RSWA_OP_SRSWA_DECODE) as srswa_decode, with
 * pk8 / pv8 / k_scale / v_scale in place of pk / pv.
 */
RSWA_API rswa_status srswa_decode_fp8(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                                      const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                                      const int32_t* blk_idx, const float* blk_logp, int32_t topk, const void* ring_k,
                                      const void* ring_v, const int32_t* wp, const int32_t* fill, float scale,
                                      float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * FP8 ring (the KV-cache quantisation above extended to the ring): the ring K and V are
 * stored as E4M3 codes [B][H][n][D] with one f32 scale per row [B][H][n] for K and one
 * for V. The ring is written one token at a time, so each written row is quantised on its
 * own: scale = amax over its D dims / 448 (1 if 0), code = E4M3(x / scale), nearest even,
 * saturating, both in f32 (the prefix rule with a one-row block).
 *
 * rswa_append_fp8: rswa_append into an FP8 ring (same wp / fill / slot_out / status rules).
 * rswa_decode_fp8kv / srswa_decode_fp8kv: rswa_decode_fp8 / srswa_decode_fp8 reading the
 *   ring as codes and row scales; workspace as rswa_decode (srswa_decode).
 */
RSWA_API rswa_status rswa_append_fp8(const rswa_dims* dims, uint8_t* ring_k8, uint8_t* ring_v8, float* ring_kscale,
                                     float* ring_vscale, const void* k_new, const void* v_new, int32_t* wp,
                                     int32_t* fill, int32_t* slot_out, int32_t* status, void* stream);

RSWA_API rswa_status rswa_decode_fp8kv(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                                       const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                                       const uint8_t* ring_k8, const uint8_t* ring_v8, const float* ring_kscale,
                                       const float* ring_vscale, const int32_t* wp, const int32_t* fill, float scale,
                                       float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

RSWA_API rswa_status srswa_decode_fp8kv(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                                        const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                                        const int32_t* blk_idx, const float* blk_logp, int32_t topk,
                                        const uint8_t* ring_k8, const uint8_t* ring_v8, const float* ring_kscale,
                                        const float* ring_vscale, const int32_t* wp, const int32_t* fill, float scale,
                                        float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * page2d rotary position encoding (Unlimited-OCR-2 SR-SWA explainer, 2D 位置编码: two
 * rotary axes, sparse_rope_mode page2d; the token axis carries the token's offset inside
 * its page, the page axis (page_mod: 2) the page number). The pages give no constants;
 * this library's reading:
 *   - pair i (i < D/2) couples dims i and i + D/2 (the LLaMA family's half split) and is
 *     turned by angle a_i:  y_i = x_i cos a_i - x_{i+D/2} sin a_i,
 *                           y_{i+D/2} = x_{i+D/2} cos a_i + x_i sin a_i;
 *   - a_i = pos * base^(-2i/D), pos = page[r] when i mod page_mod == page_mod - 1 (the
 *     page axis), else tok_pos[r] (the token axis); page_mod 0 = token axis only (plain
 *     1-D rotary encoding); base = 10000 in the model family;
 *   - angles and their cos / sin in fp64, cos / sin rounded to f32, the rotation in f32
 *     (one product and one FMA per output), the result rounded to bf16 (nearest even):
 *     within 2^-22 (|x_i| + |x_{i+D/2}|) plus half a bf16 step of the exact rotation.
 * Keys are stored encoded (the prefix and the ring hold encoded keys); values and the
 * router's index keys are not encoded.
 *
 * rswa_rope_page2d: encodes `rows` tokens of q (and of k) in one launch.
 *   rows       : R >= 0; one token per row. R = 0 launches nothing and accepts NULL
 *                buffers (after the checks of heads, head_dim, base and page_mod)
 *   q, q_out   : bf16 [R][heads][head_dim]; q_out may be q (in place)
 *   k, k_out   : bf16 [R][heads][head_dim], or both NULL; k_out may be k
 *   tok_pos, page : int32 [R] device arrays, any values
 *   heads 1..128; head_dim a multiple of 16 in [16, 256]; base finite > 0; page_mod >= 0
 *   No device-side checks; nothing is launched on a host-side error.
 *
 * rswa_append_rope: rswa_append of this step's token with its key encoded on the way
 * into the ring, and its query encoded into q_out, in one launch (head_dim 128).
 *   Arguments of rswa_append, plus q, q_out : bf16 [B][H][D] (q_out may be q) and
 *   tok_pos, page : int32 [B] (this step's token positions), base, page_mod. q_out is
 *   written whatever the ring state; a sequence with wp / fill out of range is flagged
 *   and its ring left untouched, as in rswa_append.
 * A decode step with the encoding: rswa_decode_append_rope or srswa_step_rope (one launch,
 * below); or rswa_append_rope, then srswa_route + srswa_decode (or rswa_decode) on q_out.
 */
RSWA_API rswa_status rswa_rope_page2d(int64_t rows, int32_t heads, int32_t head_dim, const void* q, void* q_out,
                                      const void* k, void* k_out, const int32_t* tok_pos, const int32_t* page,
                                      double base, int32_t page_mod, void* stream);

RSWA_API rswa_status rswa_append_rope(const rswa_dims* dims, void* ring_k, void* ring_v, const void* k_new,
                                      const void* v_new, int32_t* wp, int32_t* fill, int32_t* slot_out, const void* q,
                                      void* q_out, const int32_t* tok_pos, const int32_t* page, double base,
                                      int32_t page_mod, int32_t* status, void* stream);

/*
 * The fused decode steps with the page2d encoding inside the same launch: this step's
 * query is encoded where the attention loads it, and its key where the step appends it
 * (into ring slot wp[b] and into the step's key set); values are not encoded. Results are
 * bit-identical to rswa_rope_page2d (or rswa_append_rope) on q and k_new followed by
 * rswa_decode_append (resp. srswa_step) on the encoded rows: the same fp64 angles, the
 * same f32 cos / sin and the same f32 rotation rounded to bf16. The router (srswa_step_rope)
 * reads q_idx, which is not encoded.
 *   rope : host pointer to an rswa_rope (read during the call only):
 *          tok_pos, page : int32 device arrays [batch], this step's positions (any values;
 *                          4-byte aligned, read on the device)
 *          base          : finite > 0;  page_mod : >= 0 (as rswa_rope_page2d)
 *   The other arguments, the workspace and the error behaviour are those of
 *   rswa_decode_append (resp. srswa_step); head_dim 128. A sequence whose ring state is
 *   out of range is flagged and not appended, and its query is still encoded.
 */
typedef struct rswa_rope {
  const int32_t* tok_pos;
  const int32_t* page;
  double base;
  int32_t page_mod;
} rswa_rope;

RSWA_API rswa_status rswa_decode_append_rope(const rswa_dims* dims, const rswa_rope* rope, const void* q,
                                             const void* k_new, const void* v_new, const void* pk, const void* pv,
                                             const int32_t* prefix_len, void* ring_k, void* ring_v, int32_t* wp,
                                             int32_t* fill, int32_t* slot_out, float scale, float* out, float* lse,
                                             void* workspace, size_t ws_bytes, void* stream);

RSWA_API rswa_status srswa_step_rope(const rswa_dims* dims, const rswa_rope* rope, const void* q, const void* k_new,
                                     const void* v_new, const float* q_idx, const float* kbar, float idx_scale,
                                     int32_t topk, const void* pk, const void* pv, const int32_t* prefix_len,
                                     void* ring_k, void* ring_v, int32_t* wp, int32_t* fill, int32_t* slot_out,
                                     float scale, int32_t* blk_idx, float* blk_logp, float* tau, float* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RSWA_H */
