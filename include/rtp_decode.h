/*
 * rtp_decode.h -- C ABI of the RTPurbo decode-step sparse attention library
 * (librtp.so, CUDA, sm_100a).
 *
 * The operation (sources: "Full Attention Strikes Back" / RTPurbo -- the
 * paper review on dongryeollee1.github.io, section Method: "Adaptive sparse
 * attention" (s_h(m,n) = (W^Q_h q^pre_m)^T (W^K_h k^pre_n),
 * S_h(m) = Top-P(s_h(m,.), p)) and "Hardware-aware top-p decoding kernel"
 * (histogram threshold where the cumulative mass reaches p_top, block mask,
 * block-sparse decode); the aitrends.kr summary, items 2 and 5 (softmax
 * attention over S_h(m); block-sparse attention with a cross-split reduce)):
 *
 * For every sequence b and query head h of one decode step:
 *   local head (head_kind[h] == 0): exact softmax attention of q_rope[b,h]
 *     over cache positions [0, min(sink,L)) U [max(0, L-window), L);
 *   retrieval head (head_kind[h] == 1):
 *     q_idx = Wq_idx[h] . q_pre[b,h] (16 values, fp32),
 *     s_n   = q_idx . k_idx[b, kv(h), n] for every cached n < L,
 *     keep the smallest set of tokens whose softmax(s/4) mass reaches p[b],
 *     taking tokens in order of decreasing s, equal scores toward the lower
 *     index; p[b] >= 1 keeps every token;
 *     widen the kept tokens to whole 64-token blocks [64j, 64j+64) n [0, L);
 *     exact softmax attention of q_rope[b,h] over those positions.
 *   Attention logits are q.k / sqrt(128); kv(h) = h / (Hq / Hkv) (GQA).
 *
 * Conventions
 *   - Every tensor pointer is DEVICE memory owned by the caller unless marked
 *     host.  bf16 tensors are passed as uint16_t bit patterns.  Strides are
 *     the dense row-major strides of the stated shapes.  The bf16 tensors and
 *     `out` must be 16-byte aligned (else RTP_ERR_UNSUPPORTED): the caches
 *     are read by TMA / bulk copies.
 *   - The library allocates no memory.  Scratch lives in a caller-allocated
 *     device workspace of rtp_workspace_size() bytes.  Zero-fill it once
 *     after allocation (cudaMemset); every call leaves it ready for the next.
 *   - Work is enqueued on `stream` (a cudaStream_t); nothing synchronises the
 *     host.  Calls that share a workspace must be ordered on the GPU.
 *   - Errors the host can see (null pointers, unsupported sizes, a small
 *     workspace) return a status and enqueue nothing.  Errors only the device
 *     can see (a seq_len outside [1, capacity], p <= 0 or NaN, a page id
 *     outside [0, num_pages), a wait that timed out) set a status word in the
 *     workspace, the affected sequence's outputs are not written (bad seq_len,
 *     bad p) or unspecified (bad page id, timeout), and rtp_get_status()
 *     reports it.
 *   - No C++ exception crosses this interface.
 */
#ifndef RTP_DECODE_H
#define RTP_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rtp_status {
    RTP_OK = 0,
    RTP_ERR_NULL = 1,          /* a required pointer is NULL */
    RTP_ERR_SHAPE = 2,         /* inconsistent sizes (e.g. Hq % Hkv != 0, capacity not a multiple of 64) */
    RTP_ERR_UNSUPPORTED = 3,   /* head_dim != 128, idx_dim != 16, block_size != 64, GQA group > 8, ... */
    RTP_ERR_WORKSPACE = 4,     /* workspace missing or smaller than rtp_workspace_size() */
    RTP_ERR_CUDA = 5,          /* a CUDA launch or query failed */
    RTP_ERR_DEVICE_INPUT = 6,  /* device-side: bad seq_len, p or page id (see rtp_get_status) */
    RTP_ERR_TIMEOUT = 7,       /* device-side: a bounded wait inside a kernel gave up */
    RTP_ERR_SCRATCH_LIMIT = 8  /* rtp_decode_step_noalloc: the sizes need more than RTP_NOALLOC_SCRATCH_BYTES */
} rtp_status;

/*
 * Optional diagnostic outputs (device pointers; any may be NULL).  Entries are
 * indexed by b * num_q_heads + h and written for retrieval heads only.
 */
typedef struct rtp_debug {
    float* tau;              /* [B*Hq] the k*-th kept score s (fp32) */
    int32_t* kstar;          /* [B*Hq] number of kept tokens k* */
    int32_t* kept_blocks;    /* [B*Hq] number of kept 64-token blocks */
    float* smax;             /* [B*Hq] largest index score s */
    double* Z;               /* [B*Hq] sum over n < L of exp((s_n - smax)/4) */
    uint32_t* block_bitmap;  /* [B*Hq*words], words = ceil(ceil(capacity/64)/32); bit j%32 of word j/32 = block j kept */
    /* [48] debug trace, zeroed by the caller before the call.
     * 0-15: latest %globaltimer ns over CTAs of: 0 first CTA start, 1 group decision done,
     *   2 local-head output done, 3 block lists final, 4 retrieval attention done, 5 CTA end,
     *   6 group decision started, 7 streaming shares assigned, 8-11 selection steps done
     *   (local select / refine passes 2-4), 12 block marks done, 13 retrieval kernel started,
     *   14 first selection pass and digits done, 15 retrieval attention started.
     * 16-40: sums over CTAs of one thread's SM cycles (or counts) by phase; the Python
     *   binding's TRACE_SUMS names them in order (slots 22 and 23 are %globaltimer events:
     *   first index tile consumed, last streaming share done).
     * 43-47: latest %globaltimer ns over CTAs of: 43 a group decision reduced its
     *   buckets, 44 ... decided its heads' modes, 46 an index split took its ticket,
     *   47 an index split reduced its scores (41, 42 and 45 unused). */
    unsigned long long* trace;
} rtp_debug;

/*
 * Sizes and layout of one call.
 *   batch, num_q_heads (Hq), num_kv_heads (Hkv): Hq % Hkv == 0, Hq/Hkv in
 *     {1, 2, 4, 8}, batch <= 1024, Hq <= 128, Hkv <= 64, batch x (KV heads
 *     with a retrieval head) <= 4096, and fewer than 2^31 cache rows of 128
 *     (batch x Hkv x max_seq_len, or num_pages x Hkv x 64).
 *   head_dim must be 128, idx_dim 16, block_size 64.
 *   max_seq_len: per-sequence capacity in tokens, a multiple of 64.
 *     Contiguous layout: caches are [batch, Hkv, max_seq_len, dim].
 *     Paged layout (block_table != NULL): caches are [num_pages, Hkv, 64, dim]
 *     and max_seq_len must equal max_blocks_per_seq * 64.
 *   block_table: device int32 [batch, max_blocks_per_seq], page id of each
 *     64-token block of each sequence, or NULL for the contiguous layout.
 *   workspace / workspace_bytes: caller-allocated device scratch.
 *   debug: host pointer to an rtp_debug of device pointers, or NULL.
 *   timing_events / n_timing_events: optional host array of cudaEvent_t
 *     handles (created by the caller).  When n_timing_events >=
 *     RTP_TIMING_EVENTS the call records, on `stream`, event 0 just before
 *     its first kernel (index scores + local heads), event 1 between it and
 *     the second kernel (exact select + retrieval heads; absent when no head
 *     is a retrieval head) and event 2 after the last kernel (external event
 *     nodes when the stream is being captured into a CUDA graph).
 */
enum { RTP_TIMING_EVENTS = 3 };

typedef struct rtp_dims {
    int32_t batch, num_q_heads, num_kv_heads;
    int32_t head_dim, idx_dim, block_size;
    int32_t max_seq_len;
    const int32_t* block_table;
    int32_t max_blocks_per_seq, num_pages;
    void* workspace;
    size_t workspace_bytes;
    const rtp_debug* debug;
    void* const* timing_events;
    int32_t n_timing_events;
} rtp_dims;

/*
 * Bytes of device workspace rtp_decode_step needs for these sizes and this
 * head split (head_kind is a HOST array of num_q_heads bytes, 1 = retrieval,
 * 0 = local: the score scratch and the per-head state scale with the number
 * of retrieval heads, so the size depends on the split, not on the sizes
 * alone).  Returns 0 if the sizes are invalid or unsupported.
 */
size_t rtp_workspace_size(const rtp_dims* dims, const uint8_t* head_kind);

/*
 * One decode step (see the top of this file).
 *   q_pre     [B, Hq, 128]  bf16  pre-RoPE query (indexer input)
 *   q_rope    [B, Hq, 128]  bf16  RoPE'd query (attention input)
 *   k_idx     [B, Hkv, cap, 16] or paged [pages, Hkv, 64, 16]   bf16 index keys W^K k^pre
 *   k_cache   [B, Hkv, cap, 128] or paged [pages, Hkv, 64, 128] bf16 RoPE'd keys
 *   v_cache   same layout as k_cache, bf16 values
 *   Wq_idx    [Hq, 16, 128] bf16 indexer query projections (rows of local heads unused)
 *   seq_lens  [B] int32, 1 <= L <= cap (device)
 *   head_kind [Hq] uint8, HOST memory: 1 = retrieval head, 0 = local head.
 *             (A host array, where a device array would match the rest: the
 *             head split is fixed per layer by offline calibration, and the
 *             host needs it to size the grids and the workspace exactly, so
 *             the call reads it without a device-to-host copy.)
 *   p         [B] fp32 top-p mass per sequence, in (0, 1]; >= 1 keeps all tokens (device)
 *   window, sink: local heads' sliding window and sink sizes, >= 0, window + sink >= 1
 *   out       [B, Hq, 128] bf16 (round to nearest even)
 *   stream    cudaStream_t to enqueue on (NULL = legacy default stream)
 * Rows no head may read (rows >= L; for KV heads without retrieval heads,
 * rows outside the sink and window) never enter the arithmetic, whatever they
 * hold (NaN included).  They may still be copied into shared memory as part
 * of a 64-row tile that also holds readable rows, so the whole capacity
 * (contiguous) or whole pages (paged) must be allocated.
 */
rtp_status rtp_decode_step(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                           const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                           const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                           const float* p, int32_t window, int32_t sink, uint16_t* out, void* stream);

/*
 * rtp_decode_step_ring -- the decode step for a model whose local KV heads
 * keep only their sink and sliding window (review, Method: "Adaptive sparse
 * attention": local heads attend to a sink and a window, so they need no
 * long-context cache; Insight 1: most heads are local).  Local heads of KV
 * heads that serve no retrieval head read their keys and values from rings
 * instead of k_cache / v_cache; every other read is rtp_decode_step's.
 *
 * Ring layout, per sequence b and KV head g (rows of 128 bf16):
 *   rows 0 .. 63      : positions 0 .. 63 (the sink, 64 >= sink);
 *   rows 64 .. 63 + W : position n >= 64 in row 64 + (n mod W).
 * Writing positions in order, each new one overwrites the one W places
 * before it, so after L tokens the ring holds [0, min(64, L)) and
 * [max(64, L - W), L); W (ring_W) must be a multiple of 64 and >= window.
 *
 * Arguments are those of rtp_decode_step, plus
 *   k_ring, v_ring : device bf16 [batch, num_kv_heads, 64 + ring_W, 128],
 *     16-byte aligned (rows of KV heads with retrieval heads are not read).
 *   ring_W : the window region's rows, a multiple of 64, >= window.
 * Rows of k_cache / v_cache for KV heads without retrieval heads are not read.
 * Returns RTP_ERR_NULL for a NULL ring, RTP_ERR_SHAPE for ring_W not a
 * multiple of 64 or below window (or below 64) or sink > 64; otherwise as
 * rtp_decode_step (same workspace size).
 */
rtp_status rtp_decode_step_ring(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                const uint16_t* k_ring, const uint16_t* v_ring, int32_t ring_W,
                                const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                                const float* p, int32_t window, int32_t sink, uint16_t* out, void* stream);

/*
 * rtp_ring_write -- write the key and value rows of new tokens of the local-
 * only KV heads into their rings (the layout of rtp_decode_step_ring: rows
 * 0 .. 63 hold positions 0 .. 63, position n >= 64 goes to row 64 + n mod W).
 * The result is that of writing the tokens t = 0 .. num_new-1 of each
 * sequence in order: a token whose row a later token of the same call also
 * takes is not written.
 *   dims     : batch, num_kv_heads, head_dim 128, block_size 64 (other fields
 *              unused).
 *   k_new, v_new : device bf16 [batch, num_kv_heads, num_new, 128] (RoPE'd
 *              keys, values), 16-byte aligned.
 *   pos      : device int32 [batch], position of each sequence's first new token.
 *   ring_W   : the rings' window rows, a multiple of 64.
 *   k_ring, v_ring : device bf16 [batch, num_kv_heads, 64 + ring_W, 128],
 *              16-byte aligned; owned by the caller.
 *   device_status : optional device uint32, set to RTP_ERR_DEVICE_INPUT for a
 *              negative position (that sequence is skipped).
 * Returns RTP_ERR_NULL / RTP_ERR_SHAPE / RTP_ERR_UNSUPPORTED before anything
 * is enqueued, RTP_ERR_CUDA if the launch failed, else RTP_OK (num_new = 0:
 * nothing is enqueued).
 */
rtp_status rtp_ring_write(const rtp_dims* dims, const uint16_t* k_new, const uint16_t* v_new, const int32_t* pos,
                          int32_t num_new, int32_t ring_W, uint16_t* k_ring, uint16_t* v_ring,
                          uint32_t* device_status, void* stream);

/*
 * rtp_decode_step_topk -- the decode step with the static top-k selection in
 * place of dynamic top-p: every retrieval head keeps its min(topk, L) best
 * tokens under the order (score descending, token index ascending), widened
 * to 64-token blocks, and attends over them exactly as rtp_decode_step does.
 * Local heads are unchanged.  This is the fixed-budget variant that the
 * paper's experiments compare against (review on dongryeollee1.github.io,
 * Experiments: the static top-k baseline at k = 4096; Method, "Insight 3":
 * a fixed budget against a query-dependent one).
 *
 * Arguments are those of rtp_decode_step, with p replaced by
 *   topk: tokens kept per retrieval head, >= 1 (the same for every sequence
 *     and head); topk >= L keeps every block of that sequence, topk = 1 keeps
 *     the block of the best-scoring token (lowest index among equal maxima).
 * Returns RTP_ERR_SHAPE for topk < 1; every other check, the workspace and
 * the error behaviour are those of rtp_decode_step (same workspace size).
 */
rtp_status rtp_decode_step_topk(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                                int32_t topk, int32_t window, int32_t sink, uint16_t* out, void* stream);

/*
 * Synchronises `stream`, returns the first device-side error recorded in the
 * workspace since the last call to this function (RTP_OK if none) and clears
 * it.  For tests and debugging; it blocks the host.
 */
rtp_status rtp_get_status(const rtp_dims* dims, void* stream);

/*
 * rtp_decode_step_noalloc -- the same decode step as rtp_decode_step, for
 * callers that must not allocate device memory.  (No counterpart in the
 * paper: it is a packaging variant of the library, not part of the method.)
 *
 * Who needs it: code that runs where cudaMalloc is off limits -- a plugin
 * inside an inference engine whose memory pool owns all device memory and
 * whose budget leaves nothing for a private allocation, or a caller on a hot
 * loop that cannot afford cudaMalloc's implicit device-wide synchronisation.
 * Such a caller cannot hand rtp_decode_step a workspace, so this entry point
 * uses a scratch array compiled into the library instead.
 *
 * Arguments are those of rtp_decode_step, except:
 *   dims->workspace and dims->workspace_bytes are ignored;
 *   device_status: optional DEVICE uint32; after the step, on `stream`, it
 *     receives this call's device-side status (0 = none, otherwise an
 *     rtp_status such as RTP_ERR_DEVICE_INPUT).  NULL = not reported.
 *     rtp_get_status() does not see these calls.
 * Scratch and its limit: one static device array of RTP_NOALLOC_SCRATCH_BYTES
 *   (64 MiB), held on every GPU that loads the library until the process
 *   exits.  Sizes whose rtp_workspace_size() exceeds it are rejected with
 *   RTP_ERR_SCRATCH_LIMIT before anything is enqueued.
 * Allocation: none -- no cudaMalloc, cudaFree or allocating library call.
 *   The call enqueues one cudaMemsetAsync (clearing the part of the scratch
 *   that the kernels expect at zero, since the array keeps whatever the
 *   previous call left), the kernels, and, with device_status, one 4-byte
 *   device-to-device cudaMemcpyAsync.
 * Set-up: every call looks up the array's device address in the current
 *   device's context (cudaGetSymbolAddress, with that device current), so a
 *   context that was reset and made again is followed.  The first call in a
 *   context also loads the library's kernels into it: make that first call
 *   outside any stream capture.  A failed lookup returns RTP_ERR_CUDA and
 *   enqueues nothing.
 * Host-side errors (RTP_ERR_NULL, _SHAPE, _UNSUPPORTED, _SCRATCH_LIMIT,
 *   a failed lookup or tensor-map encoding) return before anything is
 *   enqueued, as for rtp_decode_step.
 * Concurrency: every call on a device shares the one array.  Calls whose
 *   work overlaps on the GPU (different streams without ordering between
 *   them) race on it and produce wrong results; order them on one stream.
 */
#define RTP_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

rtp_status rtp_decode_step_noalloc(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                   const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                   const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                                   const float* p, int32_t window, int32_t sink, uint16_t* out,
                                   uint32_t* device_status, void* stream);

/*
 * rtp_index_append -- write the retrieval keys of new tokens into the index
 * cache that rtp_decode_step reads (the step before the decode hot path).
 *
 * Source: "Full Attention Strikes Back" (RTPurbo) review, Method: "Adaptive
 * sparse attention": the retrieval key k^idx_n = W^K k^pre_n, a rank-16
 * projection of the pre-RoPE key kept as a 16-dim bf16 cache; W^K is per KV
 * head under GQA.
 *
 * For every sequence b < batch, KV head g < num_kv_heads and new token
 * t < num_new:
 *     k_idx row (b, g, pos[b] + t) = bf16( W^K[g] (16 x 128) . k_pre[b, g, t] )
 * each of the 16 entries the fp64 sum, in index order, of the 128 exact
 * products of bf16 values, rounded once to bf16 (round to nearest even).
 *
 *   dims     : batch, num_kv_heads, head_dim 128, idx_dim 16, block_size 64,
 *              max_seq_len (the cache capacity, a multiple of 64) and, for a
 *              paged cache, block_table / max_blocks_per_seq / num_pages as for
 *              rtp_decode_step.  num_q_heads, workspace, debug and timing
 *              fields are not used.
 *   k_pre    : device bf16 [batch, num_kv_heads, num_new, 128], 16-byte aligned.
 *   Wk_idx   : device bf16 [num_kv_heads, 16, 128], 16-byte aligned.
 *   pos      : device int32 [batch]: the cache row of each sequence's first
 *              new token (its current length, for an append).
 *   num_new  : new tokens per sequence (0: nothing is enqueued).
 *   k_idx    : device bf16 index cache, contiguous [batch, num_kv_heads,
 *              max_seq_len, 16] or paged [num_pages, num_kv_heads, 64, 16]
 *              (page id = block_table[b, n / 64]), 8-byte aligned; only the
 *              rows above are written.  Owned by the caller.
 *   device_status : optional device uint32: a row outside [0, max_seq_len)
 *              or a page id outside [0, num_pages) is skipped and sets it to
 *              RTP_ERR_DEVICE_INPUT if it was 0.  NULL: not reported.
 *   stream   : the cudaStream_t the kernel is enqueued on.
 * Returns RTP_OK, or RTP_ERR_NULL / RTP_ERR_SHAPE / RTP_ERR_UNSUPPORTED
 * (unaligned k_pre, Wk_idx or k_idx, sizes beyond the limits of rtp_dims) before
 * anything is enqueued, or RTP_ERR_CUDA if the launch failed.
 */
rtp_status rtp_index_append(const rtp_dims* dims, const uint16_t* k_pre, const uint16_t* Wk_idx, const int32_t* pos,
                            int32_t num_new, uint16_t* k_idx, uint32_t* device_status, void* stream);

/*
 * rtp_kv_append -- the KV-cache write of new tokens with the index-cache
 * append in the same kernel: the key and value rows that rtp_decode_step's
 * attention reads and the index rows its scoring reads, from one read of the
 * new pre-RoPE keys.
 *
 * Source: review, Method: "Adaptive sparse attention" (the indexer projects
 * pre-RoPE keys, the attention uses RoPE'd keys) and Insight 2 (RoPE rotates
 * each frequency pair by an angle proportional to the position).
 *
 * For every sequence b, KV head g and new token t, at cache row n = pos[b] + t:
 *     k_idx row (b, g, n)   = as rtp_index_append
 *     k_cache row (b, g, n) = bf16( RoPE_n(k_pre[b, g, t]) )
 *     v_cache row (b, g, n) = v_new[b, g, t]   (bits copied)
 * RoPE_n rotates the pairs (i, i + 64), i < 64 (rotate-half pairing), by the
 * caller's angle table row n:
 *     y_i = k_i cos[n][i] - k_{i+64} sin[n][i],  y_{i+64} = k_{i+64} cos[n][i] + k_i sin[n][i]
 * each computed as one fp64 fused multiply-add onto the other (exact)
 * product, then rounded to bf16 (round to nearest even).  The table carries
 * the model's own RoPE (base, scaling); the kernels never compute angles.
 *
 *   dims, k_pre, Wk_idx, pos, num_new, k_idx, device_status, stream: as
 *              rtp_index_append.
 *   v_new    : device bf16 [batch, num_kv_heads, num_new, 128], 16-byte aligned.
 *   rope_cos, rope_sin : device fp32 [max_seq_len, 64], 16-byte aligned; row n
 *              holds cos and sin of the angles of cache position n.
 *   k_cache, v_cache : device bf16 caches in rtp_decode_step's layout
 *              (contiguous [batch, num_kv_heads, max_seq_len, 128] or paged
 *              [num_pages, num_kv_heads, 64, 128]), 16-byte aligned; only the
 *              rows above are written.  Owned by the caller.
 * A row or page id out of range is skipped in all three caches (and reported
 * through device_status).  Returns the codes of rtp_index_append; also
 * RTP_ERR_NULL for a NULL k_cache, v_cache, v_new or table, and
 * RTP_ERR_UNSUPPORTED for one that is not 16-byte aligned.
 */
rtp_status rtp_kv_append(const rtp_dims* dims, const uint16_t* k_pre, const uint16_t* v_new, const uint16_t* Wk_idx,
                         const float* rope_cos, const float* rope_sin, const int32_t* pos, int32_t num_new,
                         uint16_t* k_idx, uint16_t* k_cache, uint16_t* v_cache, uint32_t* device_status,
                         void* stream);

/*
 * rtp_prefill -- prefill attention of a chunk of num_q queries per sequence,
 * the method's other workload: retrieval heads attend densely and causally,
 * local heads only to their sink and sliding window.
 *
 * Source: review "RTPurbo" on dongryeollee1.github.io, Method: "Adaptive
 * sparse attention" (in prefill the retrieval heads keep full attention and
 * the local heads a sink and a sliding window); Experiments, efficiency (the
 * prefill speedups over dense attention); aitrends.kr summary, efficiency
 * paragraph.
 *
 * For every sequence b, query head h and query t < num_q, at position
 * m = pos[b] + t (the cache already holds the keys and values of positions
 * 0 .. pos[b] + num_q - 1, these queries' own included):
 *   retrieval head (head_kind[h] == 1): positions [0, m];
 *   local head     (head_kind[h] == 0): [0, min(sink, m + 1)) U
 *                                       [max(0, m + 1 - window), m + 1);
 *   out[b, h, t] = softmax_n(q[b, h, t] . k_n / sqrt(128)) . v_n over those
 *   positions (the decode step's position sets at length L = m + 1).
 *
 *   dims      : batch, num_q_heads, num_kv_heads, head_dim 128, block_size 64,
 *               max_seq_len and the paged fields as for rtp_decode_step
 *               (idx_dim, workspace, debug and timing fields are not used).
 *   q         : device bf16 [B, Hq, num_q, 128], RoPE'd queries, 16-byte aligned.
 *   k_cache, v_cache : the decode step's caches (contiguous or paged), 16-byte aligned.
 *   head_kind : HOST uint8 [Hq], 1 = retrieval head, 0 = local head.
 *   pos       : device int32 [B], position of each sequence's first query.
 *   num_q     : queries per sequence, 0 <= num_q <= max_seq_len (0: nothing is enqueued).
 *   window, sink : the local heads' window and sink, >= 0, window + sink >= 1.
 *   out       : device bf16 [B, Hq, num_q, 128], 16-byte aligned (round to nearest even).
 *   device_status : optional device uint32, set to RTP_ERR_DEVICE_INPUT (if 0) for a
 *               sequence with pos[b] < 0 or pos[b] + num_q > max_seq_len (its outputs are
 *               not written) or a page id out of range (its outputs are unspecified), and
 *               to RTP_ERR_TIMEOUT if a bounded wait in the kernel gave up.
 *   stream    : the cudaStream_t the kernel is enqueued on.
 * Cache rows no query may read are never part of the arithmetic, whatever they hold.
 * Kernel: tcgen05 MMAs with tensor-memory accumulators and TMA-fed K/V tiles;
 * RTP_PREFILL_TC=0 in the environment (read at every call) selects the
 * warp-level MMA kernel instead (the same results within rounding).
 * Returns RTP_OK, or RTP_ERR_NULL / RTP_ERR_SHAPE / RTP_ERR_UNSUPPORTED before anything is
 * enqueued, or RTP_ERR_CUDA if the tensor maps or the launch failed.
 */
rtp_status rtp_prefill(const rtp_dims* dims, const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                       const uint8_t* head_kind, const int32_t* pos, int32_t num_q, int32_t window, int32_t sink,
                       uint16_t* out, uint32_t* device_status, void* stream);

/* Static string naming a status code. */
const char* rtp_status_string(rtp_status status);

#ifdef __cplusplus
}
#endif

#endif /* RTP_DECODE_H */
