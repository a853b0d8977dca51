/*
 * flint.h -- C ABI of libflint.so: Flint attention on a B200 (sm_100a).
 *   - decode: one step for batch 1 or a batch of paged requests
 *     (flint_qk_norm_rope, flint_kv_append, flint_attn_decode), all 49 layers
 *     of a token in one launch (flint_attn_stack, flint_attn_stack_noalloc)
 *     or as 49 dependent launches (flint_attn_layers_serial); bf16 or E4M3
 *     caches;
 *   - prefill of a prompt (flint_prefill_qk_norm_rope, flint_prefill_attn);
 *   - context-parallel decode across GPUs (flint_attn_decode_partial,
 *     flint_merge_partials).
 *
 * Model facts the operations follow (page title, section):
 *   - "Day-0 Support for Flint on vLLM" (hnkhoi.com/news/1467), "Model
 *     architecture": 49 layers; 35 attend a 513-token sliding window with
 *     RoPE, 14 attend the full context with no positional encoding; only the
 *     14 keep KV for the whole sequence; learned attention sinks; GQA with 32
 *     query and 4 KV heads; per-head Q/K RMSNorm.
 *   - "Recursive Flint" model JSON (studiotvai.com/api/models/flint.json):
 *     `architecture` "GQA 4 KV x 128" (head_dim 128), `maxContext` 262144,
 *     `kvCacheGiBPerRequest` (checked by flint_kv_bytes).
 *   - "Day-0 Support for Flint on vLLM" (newruntime.com), "What happened":
 *     BF16 KV cache; fused normalization, rotary-position and cache
 *     operations; a low-latency decode path for small batches; "Why it
 *     matters": one Blackwell GPU, tensor parallelism 1.
 * The pages print no formulas.  Definitions adopted here:
 *   score_j = q_h . K_j / sqrt(128); out_h = sum_j e^(score_j - M) V_j /
 *   (sum_j e^(score_j - M) + e^(sink_h - M)), M = max(max_j score_j, sink_h):
 *   the sink logit joins the softmax but carries no value.  Query head h reads
 *   KV head h / 8.  A window layer at position t attends max(0, t-512) .. t.
 *   RMSNorm: y = x * w / sqrt(mean(x^2) + eps).  RoPE: rotate-half over all
 *   128 dims, pairs (i, i+64), angle t * theta^(-2i/128), absolute position.
 *
 * Conventions for every call:
 *   - Device pointers are CUDA device memory owned by the caller; host
 *     pointers are read during the call only.  The library allocates no
 *     memory and never synchronises; work is queued on `stream` (a
 *     cudaStream_t, NULL = legacy default stream) and runs asynchronously.
 *   - bf16 tensors are passed as uint16_t bit patterns.  All shapes are
 *     row-major and densely packed unless a stride says otherwise; every
 *     device pointer must be 16-byte aligned.
 *   - Errors found on the host (bad pointer, shape, size, index) return
 *     synchronously with nothing queued: FLINT_ERR_INVALID_ARG or
 *     FLINT_ERR_UNSUPPORTED.  A failed launch returns FLINT_ERR_CUDA.  The
 *     detail of the last error on the calling thread is in flint_last_error().
 *   - Problems found on the device (a paged block id out of range, a pipeline
 *     wait that ran past its time limit) are written to *dev_err as a
 *     flint_status value if dev_err is not NULL (first error wins; the caller
 *     zeroes it).  No kernel traps or spins without a limit.
 */
#ifndef FLINT_H
#define FLINT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLINT_NUM_Q_HEADS 32
#define FLINT_NUM_KV_HEADS 4
#define FLINT_HEAD_DIM 128
#define FLINT_WINDOW 513          /* sliding-window length (tokens) */
#define FLINT_BLOCK_SIZE 64       /* paged-cache block length (tokens) */
#define FLINT_MAX_CONTEXT 262144  /* "maxContext" of the model JSON */
#define FLINT_MAX_BATCH 64        /* requests per flint_attn_decode launch */
#define FLINT_MAX_LAYERS 49       /* layers per flint_attn_stack call */
#define FLINT_CP_PARTIAL_FLOATS 4160  /* 32*128 + 32 + 32: one context-parallel partial */
#define FLINT_MAX_CP_PARTS 1024       /* partials per flint_merge_partials call */
#define FLINT_NOALLOC_SCRATCH_BYTES (4u << 20)  /* flint_attn_stack_noalloc's fixed scratch */

typedef enum {
    FLINT_OK = 0,
    FLINT_ERR_INVALID_ARG = 1,
    FLINT_ERR_UNSUPPORTED = 2,
    FLINT_ERR_WORKSPACE = 3,
    FLINT_ERR_CUDA = 4,
    FLINT_ERR_TIMEOUT = 5
} flint_status;

typedef enum {
    FLINT_KV_CONTIGUOUS = 0, /* K/V [B][capacity][4][128]; position t in slot t     */
    FLINT_KV_RING = 1,       /* K/V [B][513][4][128]; position t in slot t mod 513   */
    FLINT_KV_PAGED = 2       /* K/V [num_blocks][64][4][128]; position t in block
                                block_table[b][t / 64], row t mod 64                 */
} flint_kv_layout;

typedef enum {
    FLINT_KV_BF16 = 0,       /* one bf16 per cached value */
    FLINT_KV_FP8_E4M3 = 1    /* one byte per value: an OCP E4M3 code of value / scale
                                ("Recursive Flint" model JSON, the fp8 column of
                                kvCacheGiBPerRequest; the format is this library's
                                reading: the pages give only the byte count) */
} flint_kv_dtype;

/* One layer's KV cache for a batch of requests.  k and v are device buffers
 * of identical geometry, with elements of the given dtype (the geometry below
 * counts elements, so an E4M3 row of 4 x 128 values is 512 bytes). */
typedef struct {
    void* k;
    void* v;
    int32_t layout;              /* flint_kv_layout */
    int32_t capacity;            /* CONTIGUOUS: slots per request; RING: 513; PAGED: 0 */
    int64_t req_stride;          /* CONTIGUOUS/RING: elements between requests
                                    (0 = capacity*4*128); multiple of 8 */
    const int32_t* block_table;  /* PAGED: device int32 [B][max_blocks_per_req] */
    int32_t max_blocks_per_req;  /* PAGED */
    int32_t block_size;          /* PAGED: must be 64 */
    int32_t num_blocks;          /* PAGED: blocks in the pool */
    int32_t dtype;               /* flint_kv_dtype; 0 (bf16) for zero-filled structs */
    float k_scale[4];            /* FP8_E4M3: per KV head, stored code = e4m3(k / k_scale)
                                    rounded to nearest even, saturated at +-448, with
                                    the division in float32; value read = code * k_scale */
    float v_scale[4];            /* FP8_E4M3: the same for v */
} flint_kv_cache;

/* One layer of one decoded token, for flint_attn_stack (batch 1). */
typedef struct {
    const uint16_t* q_raw;   /* bf16 [32][128], before norm/RoPE */
    const uint16_t* k_raw;   /* bf16 [4][128] */
    const uint16_t* v_raw;   /* bf16 [4][128], appended as is */
    const uint16_t* w_q;     /* bf16 [128] RMSNorm weight for q (shared by heads) */
    const uint16_t* w_k;     /* bf16 [128] RMSNorm weight for k */
    const float* sinks;      /* fp32 [32] sink logits */
    flint_kv_cache cache;    /* this layer's cache (request 0 only) */
    int32_t window;          /* 0 = full context, 513 = sliding window */
    int32_t rope;            /* 1 = apply RoPE (window layers), 0 = NoPE */
} flint_layer;

/* Short English name of a status code (static storage). */
const char* flint_status_string(flint_status s);

/* Detail of the last error returned on the calling thread ("" if none). */
const char* flint_last_error(void);

/* KV-cache bytes per request of a model with n_full full-context layers and
 * n_window window layers at context ctx_len: every token of a full layer, and
 * min(ctx_len, window) tokens of a window layer, each 2*4*128 values of
 * elem_bytes bytes ("Recursive Flint" model JSON, kvCacheGiBPerRequest).
 * Pure host arithmetic; returns 0 for negative arguments. */
uint64_t flint_kv_bytes(int64_t ctx_len, int32_t n_full, int32_t n_window,
                        int32_t window, int32_t elem_bytes);

/* Per-head Q/K RMSNorm, optional RoPE, optional KV append for B requests
 * ("Model architecture": per-head Q/K RMSNorm, RoPE on window layers;
 * "What happened": fused normalization, rotary-position and cache ops).
 *   q_raw  bf16 [B][32][128], k_raw bf16 [B][4][128]          (device, in)
 *   v_raw  bf16 [B][4][128] (device, in); only read when cache != NULL
 *   w_q, w_k  bf16 [128] (device, in); the norm weight, shared by all heads
 *   pos    host int32 [B]: absolute position of each request's new token
 *   eps    RMSNorm epsilon (1e-6); theta  RoPE base (10000)
 *   apply_rope  0 or 1
 *   q_out  fp32 [B][32][128] (device, out) or NULL
 *   k_out  bf16 [B][4][128]  (device, out) or NULL: k after norm/RoPE,
 *          rounded to nearest even
 *   cache  NULL, or the cache to append k (as in k_out) and v_raw to, at
 *          position pos[b] (slot per the layout; PAGED reads block_table on
 *          the device, an out-of-range block id skips the write and sets
 *          *dev_err = FLINT_ERR_INVALID_ARG)
 * B in [1, FLINT_MAX_BATCH]. */
flint_status flint_qk_norm_rope(const uint16_t* q_raw, const uint16_t* k_raw,
                                const uint16_t* v_raw, const uint16_t* w_q,
                                const uint16_t* w_k, const int32_t* pos, int32_t B,
                                float eps, double theta, int32_t apply_rope,
                                float* q_out, uint16_t* k_out,
                                const flint_kv_cache* cache, int32_t* dev_err,
                                void* stream);

/* Bit-exact append of already final k, v (bf16 [B][4][128], device) at host
 * positions pos[B] of `cache` ("Model architecture": only full layers keep
 * the whole sequence, window layers keep a 513-slot ring).  Untouched slots
 * are not written.  Same device-side error rule as flint_qk_norm_rope. */
flint_status flint_kv_append(const uint16_t* k, const uint16_t* v, const int32_t* pos,
                             int32_t B, const flint_kv_cache* cache, int32_t* dev_err,
                             void* stream);

/* Bytes of device workspace for flint_attn_decode / flint_attn_stack with
 * n_problems (requests, or layers) on num_ctas CTAs (0 = one per SM): room
 * for the full split plan, 4096 + 768 * 16640 bytes (12.8 MB).  A call also
 * runs with less, down to 4096 + (CTAs + n_problems) * 16640 bytes, with a
 * coarser run-time balancing queue; below that it returns
 * FLINT_ERR_WORKSPACE.  The workspace holds split partials, per-problem
 * arrival counters, a grid-barrier word, the merge-ticket word (whose upper
 * bits count launches), per-partial ready flags and the queue head; it must be
 * zero-filled before its first use, and every call that completes without a
 * device error leaves it ready for the next call (arrival counters and queue
 * head back at zero, flags tagged with the launch count).
 * After a device error, zero it again.  Calls that share a workspace must not
 * overlap in time.  Returns 0 for invalid arguments. */
size_t flint_attn_workspace_bytes(int32_t n_problems, int32_t num_ctas);

/* Split-KV flash-decode over a batch of B requests of one layer: q already
 * normed (and roped).  The new token is already in the cache; request b
 * attends positions [max(0, L_b - window), L_b) (window 513) or [0, L_b)
 * (window 0), L_b = seq_lens[b].  What it computes is the attention of
 * "Day-0 Support for Flint on vLLM" (hnkhoi.com), "Model architecture": GQA
 * with 32 query over 4 KV heads of 128 dims, a learned sink logit per query
 * head that joins the softmax without a value, and either a 513-token window
 * or the whole context; the batch-1 decode at 100,000 tokens it serves is the
 * one of the same page on newruntime.com, "What happened".
 *   q         bf16 or fp32 [B][32][128] (device); q_is_fp32 selects
 *   cache     any layout; RING requires window == 513 and capacity 513
 *   seq_lens  HOST int32 [B], 1 <= L_b <= FLINT_MAX_CONTEXT (and <= capacity
 *             for CONTIGUOUS, <= max_blocks_per_req*64 for PAGED); the split
 *             plan is built from them on the host
 *   sinks     fp32 [32] (device), shared by the batch; -INFINITY drops a sink
 *   out       fp32 [B][32][128] (device)
 *   workspace device, >= flint_attn_workspace_bytes(B, num_ctas) bytes
 *   num_ctas  0 = one CTA per SM (the tuned default)
 * B in [1, FLINT_MAX_BATCH].  Result is deterministic run to run for a given
 * workspace size and num_ctas: queued chunks have fixed bounds, whichever CTA
 * takes them, and partials are merged in a fixed order.  A PAGED block id
 * outside [0, num_blocks) is never handed to a load: that tile is skipped, the
 * output is meaningless, and *dev_err = FLINT_ERR_INVALID_ARG.  A pipeline
 * wait that runs past its time limit sets *dev_err = FLINT_ERR_TIMEOUT; the
 * kernel then lets its copies in flight land and returns (zero the workspace
 * before the next call). */
flint_status flint_attn_decode(const void* q, int32_t q_is_fp32,
                               const flint_kv_cache* cache, const int32_t* seq_lens,
                               int32_t B, const float* sinks, int32_t window,
                               float* out, void* workspace, size_t ws_bytes,
                               int32_t num_ctas, int32_t* dev_err, void* stream);

/* One decoded token through n_layers attention layers in ONE launch: for each
 * layer, per-head Q/K RMSNorm (+RoPE if layer.rope), append of k and v_raw at
 * position pos, and decode attention over the layer's window, all scheduled
 * together across the GPU (the layers are independent problems here).  The
 * layer stack is Flint's ("Day-0 Support for Flint on vLLM", hnkhoi.com,
 * "Model architecture"): 49 layers, 35 with a 513-token window and RoPE, 14
 * over the full context without positional encoding, each with per-head Q/K
 * RMSNorm and sinks; the norm, rotary and cache steps fused with attention
 * follow the same page on newruntime.com, "What happened".
 *   layers    HOST array [n_layers], 1 <= n_layers <= FLINT_MAX_LAYERS;
 *             window layers usually RING caches, full layers CONTIGUOUS
 *   pos       position of the new token (context pos + 1 after the append)
 *   out       fp32 [n_layers][32][128] (device)
 *   workspace >= flint_attn_workspace_bytes(n_layers, num_ctas) bytes */
flint_status flint_attn_stack(const flint_layer* layers, int32_t n_layers, int32_t pos,
                              float eps, double theta, float* out, void* workspace,
                              size_t ws_bytes, int32_t num_ctas, int32_t* dev_err,
                              void* stream);

/* The same n_layers layers of one token as flint_attn_stack, run as n_layers
 * serially dependent launches, one layer each, as a model whose layers feed
 * one another must run them.  Each launch after the first is a programmatic
 * dependent of the one before (CUDA programmatic dependent launch): its launch
 * and on-chip set-up overlap the previous layer's tail, and it waits for the
 * previous launch to complete before it touches any memory.  The layers here
 * are independent problems (the synthetic dependence is the ordering), so the
 * outputs equal flint_attn_stack's up to rounding order.  No counterpart
 * kernel in the pages: their serving path launches per-layer kernels ("Day-0
 * Support for Flint on vLLM", newruntime.com, "What happened": the kernel
 * count per forward step).  Arguments, workspace and errors as
 * flint_attn_stack; the workspace is reused by every layer in turn. */
flint_status flint_attn_layers_serial(const flint_layer* layers, int32_t n_layers,
                                      int32_t pos, float eps, double theta, float* out,
                                      void* workspace, size_t ws_bytes, int32_t num_ctas,
                                      int32_t* dev_err, void* stream);

/* flint_attn_stack without a workspace argument, for callers that cannot
 * allocate device memory (a runtime that owns all of it through its own pool,
 * a plug-in handed buffers but no allocator).  No counterpart in the paper: it
 * changes where the scratch lives, not what is computed; the results are
 * those of flint_attn_stack.
 *   Scratch: the library holds one FLINT_NOALLOC_SCRATCH_BYTES array in the
 *   device memory of every device its device code is loaded on, until the
 *   process exits.  Calls whose smallest workspace,
 *   4096 + (CTAs + n_layers) * 16640 bytes, exceeds it are refused with
 *   FLINT_ERR_WORKSPACE; CTAs counts the CTAs a launch uses, num_ctas (0: one
 *   per SM) but never more than the device has SMs.  49 layers fit with up to
 *   202 CTAs, so on a device of 202 SMs or fewer (a 148-SM B200) no call is
 *   refused for its size.  The scratch is
 *   below flint_attn_workspace_bytes, so the run-time balancing queue is
 *   coarser than with a full workspace (same results up to rounding order).
 *   Set-up: the first call on a device, with that device current, looks up the
 *   scratch's address; make it before any stream capture.  The address
 *   belongs to the device's CUDA context: after a device reset the first call
 *   looks it up again, and must again come before any capture.
 *   Sharing: every call on a device uses the same scratch, which keeps the last
 *   call's contents; each call clears the counters it needs on `stream` first.
 *   Calls that overlap on the GPU (other streams, other threads) race.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 * Other arguments, errors and the append are those of flint_attn_stack. */
flint_status flint_attn_stack_noalloc(const flint_layer* layers, int32_t n_layers,
                                      int32_t pos, float eps, double theta, float* out,
                                      int32_t num_ctas, int32_t* dev_err, void* stream);

/* Prefill, step 1: per-head Q/K RMSNorm, optional RoPE and the cache write
 * for the T tokens of one prompt at positions 0 .. T-1, with nothing cached
 * before it (the 8,192-token prefill of "Day-0 Support for Flint on vLLM",
 * newruntime.com, "What happened"; norm and RoPE as in flint_qk_norm_rope,
 * token t at position t).
 *   q_raw  bf16 [T][32][128], k_raw / v_raw bf16 [T][4][128]   (device, in)
 *   w_q, w_k  bf16 [128] (device, in)
 *   q_out  bf16 [T][32][128] (device, out): q after norm/RoPE, rounded to
 *          nearest even (prefill activations are bf16), or NULL
 *   k_out  bf16 [T][4][128]  (device, out): k after norm/RoPE, rounded to
 *          nearest even (the cache value), or NULL
 *   v_out  fp16 [T][4][128]  (device, out): v_raw converted to fp16 (nearest,
 *          saturating at +-65504; exact for bf16 values in the fp16 normal
 *          range), the v operand of flint_prefill_attn, or NULL
 *   cache  NULL, or the cache of this one request (request 0 of a
 *          CONTIGUOUS / RING cache, row 0 of a PAGED block table): token t
 *          goes to slot t (ring: t % 513, and only the last 513 tokens are
 *          written); an E4M3 cache gets the codes of flint_qk_norm_rope.
 * Arithmetic in float32 as in flint_qk_norm_rope (the angles formed and
 * rounded from double), except that the sum of squares runs in another order
 * and the reciprocal square root is the hardware's (within 2 ulp): q and k
 * may differ from flint_qk_norm_rope's by one bf16 ulp where a value lies
 * next to a rounding boundary.
 * T in [1, FLINT_MAX_CONTEXT]; T must fit the cache (contiguous capacity,
 * block table).  Every pointer 16-byte aligned.  Errors as for
 * flint_qk_norm_rope; the kernel streams the tokens through shared memory,
 * and a copy wait that runs past its time limit sets *dev_err =
 * FLINT_ERR_TIMEOUT. */
flint_status flint_prefill_qk_norm_rope(const uint16_t* q_raw, const uint16_t* k_raw,
                                        const uint16_t* v_raw, const uint16_t* w_q,
                                        const uint16_t* w_k, int32_t T, float eps,
                                        double theta, int32_t apply_rope, uint16_t* q_out,
                                        uint16_t* k_out, uint16_t* v_out,
                                        const flint_kv_cache* cache, int32_t* dev_err,
                                        void* stream);

/* Prefill, step 2: causal attention of a T-token prompt over itself, with the
 * head's sink ("Model architecture": GQA 32/4, learned sinks, 513-token
 * windows on the RoPE layers, full context on the NoPE layers).  Query row t
 * of head h attends the keys of positions max(0, t - window + 1) .. t
 * (window > 0) or 0 .. t of KV head h / 8, as flint_attn_decode does for the
 * token at position t with L = t + 1:
 *   out[t][h] = sum_j e^(s_j - M) v[j] / (sum_j e^(s_j - M) + e^(sink_h - M)),
 *   s_j = q[t][h] . k[j] / sqrt(128), M = max(max_j s_j, sink_h).
 *   q  bf16 [T][32][128], k  bf16 [T][4][128], v  fp16 [T][4][128] (device,
 *      in; flint_prefill_qk_norm_rope's q_out, k_out and v_out)
 *   sinks  fp32 [32] (device, in); window  0 or FLINT_WINDOW
 *   out  fp32 [T][32][128] (device, out)
 * T in [1, FLINT_MAX_CONTEXT].  Products on tensor-core MMAs (tcgen05) with
 * fp32 accumulation: q.k in bf16, p.v in fp16 (p rounded to fp16 after an
 * fp32 softmax).  A pipeline wait that runs past
 * its time limit sets *dev_err = FLINT_ERR_TIMEOUT (dev_err may be NULL). */
flint_status flint_prefill_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                int32_t T, const float* sinks, int32_t window, float* out,
                                int32_t* dev_err, void* stream);

/* Context-parallel decode, step 1 (multi-GPU split-KV of a full layer: each
 * rank owns a range of the layer's tokens; the pages serve on one GPU, so
 * this follows the split-KV arithmetic of flint_attn_decode).  The attention
 * of q over tokens [0, seq_lens[b]) of this rank's `cache` (no window, no
 * sink), returned unnormalised so that the ranks' results can be merged:
 *   partials  fp32 [B][FLINT_CP_PARTIAL_FLOATS] (device, out): for request b,
 *             O [32][128], then m [32], then l [32], with scores in log2
 *             units (s'_j = q_h . k_j / sqrt(128) * log2(e)):
 *             l_h = sum_j 2^(s'_j - m_h), O_h = sum_j 2^(s'_j - m_h) v_j (up
 *             to rounding order), where m_h is the reference the kernel
 *             scaled by: its running maximum, which moves only by steps of
 *             more than 8, so max_j s'_j - 8 <= m_h <= max_j s'_j.  The triple
 *             is defined up to the common factor 2^m_h.
 * Other arguments, the workspace and errors as flint_attn_decode. */
flint_status flint_attn_decode_partial(const void* q, int32_t q_is_fp32,
                                       const flint_kv_cache* cache, const int32_t* seq_lens,
                                       int32_t B, float* partials, void* workspace,
                                       size_t ws_bytes, int32_t num_ctas, int32_t* dev_err,
                                       void* stream);

/* Context-parallel decode, step 2: the log-sum-exp merge of n_parts partials
 * per request (the ranks' flint_attn_decode_partial results after an
 * all-gather) with the head's sink logit, as flint_attn_decode folds its own
 * split partials:  M = max(sink_h log2(e), max_r m_r),
 *   out_h = sum_r 2^(m_r - M) O_r / (2^(sink_h log2(e) - M) + sum_r 2^(m_r - M) l_r).
 *   partials  fp32 [n_parts][B][FLINT_CP_PARTIAL_FLOATS] (device, in)
 *   sinks     fp32 [32] (device, in);  out  fp32 [B][32][128] (device, out)
 * n_parts in [1, FLINT_MAX_CP_PARTS], B in [1, FLINT_MAX_BATCH].  A partial
 * with m = -inf (no tokens) contributes nothing; a head with no token in any
 * partial and a sink of -inf (M = -inf) gets the output 0. */
flint_status flint_merge_partials(const float* partials, int32_t n_parts, int32_t B,
                                  const float* sinks, float* out, void* stream);

/* The split planner behind both attention calls (pure host code, exposed for
 * tests).  Work is n_segs segments (one per problem, all four KV heads
 * together) of seg_tiles[s] 32-token tiles; it is cut into items (segment, tile range)
 * laid over num_ctas CTAs so that tiles + item_cost per item are level.
 * Outputs: item_seg/item_t0/item_t1 [max_items], cta_begin [num_ctas+1]
 * (items of CTA c are cta_begin[c] .. cta_begin[c+1]-1; the items of one
 * segment are consecutive).  Returns the item count, or -1 on bad
 * arguments / too many items. */
int32_t flint_plan_items(const int32_t* seg_tiles, int32_t n_segs, int32_t num_ctas,
                         int32_t item_cost, int32_t* item_seg, int32_t* item_t0,
                         int32_t* item_t1, int32_t* cta_begin, int32_t max_items);

/* The full plan of one attention launch (pure host code, exposed for tests):
 * when there are at least 64 tiles per CTA, the static plan of
 * flint_plan_items over the first ~80 % of every segment of at least 64
 * tiles (smaller ones stay whole), plus a queue of chunks that
 * cut the remaining tails, in guided sizes (ceil(remaining tiles / num_ctas),
 * at least 8), which CTAs claim at run time once their static lists are done.
 * Coarser queues (chunks of at least 16 or 32 tiles, never above an eighth
 * of a CTA's share), then none, are used when max_items is too small; with
 * fewer than 64 tiles per CTA the plan is static only.
 * Outputs: item_seg/item_t0/item_t1 [max_items], sorted by (segment, t0);
 * order [max_items] and cta_begin [num_ctas + 1]: the static items of CTA c
 * are order[cta_begin[c] .. cta_begin[c+1]-1] and the queue is
 * order[cta_begin[num_ctas] .. n-1].  Returns n, the item count, or -1 on bad
 * arguments / no plan within max_items. */
int32_t flint_plan_split(const int32_t* seg_tiles, int32_t n_segs, int32_t num_ctas,
                         int32_t item_cost, int32_t max_items, int32_t* item_seg,
                         int32_t* item_t0, int32_t* item_t1, int32_t* order,
                         int32_t* cta_begin);

#ifdef __cplusplus
}
#endif

#endif /* FLINT_H */
