/*
 * dec.h - C ABI of the batched single-token decoder step (B200, sm_100a).
 *
 * One call of dec_step advances B independent streams of a pre-norm
 * transformer decoder by one token each: embedding (+ learned position),
 * per layer pre-norm, fused Q/K/V projection, KV-cache append, causal
 * self-attention over the stream's cache, output projection and residual,
 * (Whisper) cross-attention over precomputed encoder K/V, the FFN, and the
 * final norm with the tied LM head and the greedy argmax.
 *
 * Sources (docs.rs source pages), cited by crate, file and item:
 *   [wa-dec]  whisper-apr 0.3.3 src/model/decoder_generated.rs
 *   [wa-cuda] whisper-apr 0.3.0 src/cuda/impl_generated.rs
 *   [focr]    franken_ocr 0.8.0 src/native_engine/decoder_qwen2.rs
 *   [cera]    cera 0.5.4 src/model/whisper.rs
 *   [q8]      lattice-inference 0.4.0 src/forward/cpu_q8.rs
 *
 * Conventions for every entry point:
 *   - Pointers documented "host" are read during the call only; pointers
 *     documented "device" must be CUDA device memory on the handle's device
 *     and stay valid until the work queued on `stream` has run.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - All argument checks run before any work is queued; a call that returns
 *     an error other than DEC_ECUDA has changed no state.
 *   - A handle is not thread-safe: serialise calls on one handle.
 *   - dec_last_error(h) returns a message for the last failed call on h.
 */
#ifndef DEC_H
#define DEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dec_status {
    DEC_OK = 0,
    DEC_EINVAL = 1,     /* null pointer, bad shape, bad config, duplicate slot */
    DEC_ERANGE = 2,     /* token >= vocab, position outside the position table */
    DEC_EOVERFLOW = 3,  /* cache_lens[b] + 1 > max_cache_len (cache full) */
    DEC_ESTATE = 4,     /* cache_lens[b] differs from the slot's length, slot not prefilled */
    DEC_ENOMEM = 5,     /* device or pinned host allocation failed */
    DEC_ECUDA = 6,      /* a CUDA call failed; the message names it */
    DEC_ETIMEOUT = 7    /* a bounded device wait gave up (reported by dec_sync) */
} dec_status;

enum { DEC_FAMILY_WHISPER = 0, DEC_FAMILY_QWEN2 = 1 };
enum { DEC_PROJ_F32 = 0, DEC_PROJ_W8A8 = 1, DEC_PROJ_W8A32 = 2 };

#define DEC_MAX_BATCH 128

/*
 * Model and capacity description.
 *   family      DEC_FAMILY_WHISPER: LayerNorm with bias, learned positions,
 *               self- and cross-attention, GELU(tanh) FFN, all projections
 *               biased ([cera] `decode_step_into`).
 *               DEC_FAMILY_QWEN2: RMSNorm, NEOX RoPE, SwiGLU MLP, bias on
 *               q/k/v only ([focr] `qwen2_decode_step`).
 *   head_dim    must be 64; d_model = n_heads * 64.
 *   d_ff        FFN width, a multiple of 16 (16-byte int8 weight loads).
 *   max_pos     whisper: rows of the learned position table (positions must
 *               be < max_pos); qwen2: exclusive bound on positions (RoPE table rows).
 *   enc_len     whisper: encoder rows attended by cross-attention; 0 for qwen2.
 *   proj_fmt    DEC_PROJ_F32 (f32 weights), DEC_PROJ_W8A8 (int8 weights and
 *               int8 per-row activations, int32 accumulation; qwen2 only) or
 *               DEC_PROJ_W8A32 (int8 weights, f32 activations; whisper only).
 *   norm_eps    1e-5 (LayerNorm) / 1e-6 (RMSNorm) in the configs of the pages.
 *   rope_theta  RoPE base (qwen2), e.g. 1e6.
 *   max_slots   number of independent streams the handle holds caches for.
 *   max_cache_len  rows per stream and layer in the self-attention cache.
 *   n_kv_heads  K/V heads (grouped-query attention, qwen2 only; [focr] native kv-lane
 *               mapping: query head h reads K/V head h / (n_heads / n_kv_heads));
 *               must divide n_heads; 0 means one K/V head per query head. The K and
 *               V projections are [n_kv_heads * 64, d] and the caches hold n_kv_heads
 *               heads.
 *   kv_page_rows  0: each slot owns max_cache_len rows of self-attention cache.
 *               16, 32 or 64: a paged cache ([wa-dec] `PagedDecoderKVCache`,
 *               `forward_one_paged`): a pool of kv_pages pages of that many rows
 *               (per layer, K and V) shared by all slots through a page table; a slot
 *               takes pages as it grows (dec_step, dec_prefill, dec_kv_append) and
 *               returns them when it is prefilled again, shortened by dec_kv_append,
 *               released (dec_release_slot) or reset. A call that would need more
 *               pages than are free returns DEC_ENOMEM before any work.
 *               max_cache_len still bounds each slot's length.
 *   kv_pages    pages in the pool (kv_page_rows > 0).
 *   head_fmt    DEC_HEAD_EXACT: the tied head on the f32 embedding (three-digit
 *               exact-integer split, 3 bytes per weight). DEC_HEAD_INT8_REFINE
 *               ([focr] `LmHead` int8 arm, `got_lm_head`: int8 per-row head, then an
 *               exact re-score of the best candidates): coarse logits from the
 *               embedding's per-row int8 quantisation (1 byte per weight), then every
 *               token whose coarse logit is within a proven error bound of the row's
 *               best is re-scored with the exact head's arithmetic. The greedy pick
 *               equals the exact head's pick; the returned logits are exact for those
 *               candidates and coarse (within the bound) elsewhere.
 */
enum { DEC_HEAD_EXACT = 0, DEC_HEAD_INT8_REFINE = 1 };
typedef struct dec_config {
    int32_t family;
    int32_t n_layers;
    int32_t d_model;
    int32_t n_heads;
    int32_t head_dim;
    int32_t d_ff;
    int32_t vocab;
    int32_t max_pos;
    int32_t enc_len;
    int32_t proj_fmt;
    float norm_eps;
    float rope_theta;
    int32_t max_slots;
    int32_t max_cache_len;
    int32_t head_fmt;
    int32_t n_kv_heads;
    int32_t kv_page_rows;
    int32_t kv_pages;
} dec_config;

/*
 * One projection y = x W^T (+ b), W [out, in] row-major (PyTorch layout), host memory.
 *   w      float when proj_fmt == DEC_PROJ_F32, int8_t (codes in [-127, 127]) otherwise
 *   scale  per-output-row f32 scale s_n of the int8 formats (W_nk = s_n q_nk); NULL for f32
 *   bias   f32 [out] or NULL (must be NULL exactly where the family has no bias)
 */
typedef struct dec_proj {
    const void* w;
    const float* scale;
    const float* bias;
} dec_proj;

/*
 * One layer's weights (host). Whisper uses norm1 (self-attn LN), q/k/v/o,
 * norm2 (cross-attn LN), xq/xk/xv/xo, norm3 (FFN LN), fc1 [d_ff, d], fc2 [d, d_ff].
 * Qwen2 uses norm1 (input RMSNorm weight), q/k/v/o, norm2 (post-attention RMSNorm
 * weight), gate and up [d_ff, d], down [d, d_ff]. Unused members are ignored.
 */
typedef struct dec_layer_weights {
    const float* norm1_w;
    const float* norm1_b;
    dec_proj q, k, v, o;
    const float* norm2_w;
    const float* norm2_b;
    dec_proj xq, xk, xv, xo;
    const float* norm3_w;
    const float* norm3_b;
    dec_proj fc1, fc2;
    dec_proj gate, up, down;
} dec_layer_weights;

/*
 * Model weights (host). tok_emb [vocab, d] f32 is both the embedding and the
 * tied LM head ([focr] module doc: tied embeddings; [cera] proj_w). pos_emb
 * [max_pos, d] f32 for whisper, NULL for qwen2. final_w / final_b: final norm
 * (final_b NULL for RMSNorm). layers: [n_layers].
 */
typedef struct dec_weights {
    const float* tok_emb;
    const float* pos_emb;
    const float* final_w;
    const float* final_b;
    const dec_layer_weights* layers;
} dec_weights;

typedef struct dec_handle dec_handle;

/*
 * Validate cfg, copy and pack all weights into device memory on the current
 * CUDA device, and allocate every KV cache and workspace once ([wa-dec]
 * `DecoderScratch`: per-token buffers allocated once). The caller may free
 * its weight buffers after the call. On error *out is NULL and nothing leaks;
 * the message is available from dec_last_error(NULL) on the same thread.
 * Besides the packed weights the handle keeps, for the tensor-core paths:
 * the embedding as three int8 digit planes plus row scales (3 bytes per
 * element, for the LM head) and, for qwen2, row-permuted copies of the
 * q|k|v and gate/up panels.
 * Numerics: W8A8 products are exact int32 sums on every path; the LM head is
 * computed from exact-integer products of three-digit splits of its f32
 * operands (error below 2^-22 of each row's largest element per operand);
 * f32 and W8A32 projections of batches of 8 or more may run on TF32 tensor
 * cores with split operands (three / two products). A stream's logits never
 * depend on the other streams of the batch for the head and W8A8 layers, and
 * for f32 / W8A32 layers not within batches below 8 or within batches of 8+.
 */
dec_status dec_create(const dec_config* cfg, const dec_weights* w, dec_handle** out);

/* Free everything the handle owns. Synchronises the device first. NULL is a no-op. */
dec_status dec_destroy(dec_handle* h);

/* Message of the last failed call on h (or, when h is NULL, of the last failed
 * dec_create or handle-less call on this thread). Never NULL; "" when there was
 * no error. */
const char* dec_last_error(const dec_handle* h);

/*
 * Reset stream `slot` and run `n_tokens` tokens (host int32) at positions
 * 0..n_tokens-1 through the decoder, filling its self-attention cache
 * ([focr] `forward_prefill_seed`: the prompt in one forward that seeds the
 * cache). The prompt runs in chunks of up to 128 rows (dec_set_prefill_chunk):
 * each chunk is one step whose projections are m = chunk contractions on the
 * tensor-core paths and whose attention is causal per row; only the last row
 * goes through the head. Whisper: `enc_hidden` (device f32 [enc_len, d]) is
 * required; cross-attention K and V are computed from it once per layer
 * ([cera] `precompute_cross_attention`: K = enc Wk^T + bk, V = enc Wv^T + bv).
 * Qwen2: enc_hidden must be NULL. n_tokens may be 0 (cross K/V only).
 * last_logits (device f32 [vocab] or NULL) receives the last row's logits;
 * the last row's argmax becomes the slot's greedy continuation token.
 */
dec_status dec_prefill(dec_handle* h, int32_t slot, const int32_t* tokens, int32_t n_tokens,
                       const float* enc_hidden, float* last_logits, void* stream);

/*
 * Per-phase device timing ([wa-dec] `forward_probed`: where a decode step's
 * time goes). While enabled, every dec_step / dec_step_host runs uncaptured
 * with a CUDA event after each phase; dec_phase_times then gives, for the most
 * recent step, each phase's device time in ms with its layer (-1 outside the
 * layers) and kind, in launch order. Programmatic dependent launch does not
 * overlap kernels across the events, so the phases sum to more than a captured
 * step. dec_phase_times synchronises on the step's last event; *n receives the
 * phase count (entries beyond cap are not written).
 */
enum {
    DEC_PHASE_EMBED = 1, DEC_PHASE_QKV = 2, DEC_PHASE_SELF_ATTN = 3, DEC_PHASE_O = 4,
    DEC_PHASE_CROSS_Q = 5, DEC_PHASE_CROSS_ATTN = 6, DEC_PHASE_CROSS_O = 7,
    DEC_PHASE_FFN_UP = 8, DEC_PHASE_FFN_DOWN = 9, DEC_PHASE_HEAD = 10
};
dec_status dec_set_phase_timing(dec_handle* h, int32_t enabled);
dec_status dec_phase_times(dec_handle* h, int32_t cap, float* ms, int32_t* layer, int32_t* kind, int32_t* n);

/* Prompt rows per prefill step, 1..128 (default 128). A W8A8 model gives the same
 * bits for every chunk size; f32 / W8A32 projections switch to the split-TF32
 * tensor-core path from 8 rows on. */
dec_status dec_set_prefill_chunk(dec_handle* h, int32_t rows);

/*
 * Write rows [start_pos, start_pos + n_rows) of every layer's self-attention
 * K and V for `slot` and set the slot length to start_pos + n_rows
 * ([focr] `Qwen2KvCache::seed`). k and v are device f32 [n_layers, n_rows,
 * kv heads * 64], token-major (already rotated K for qwen2). Requires
 * start_pos <= the slot's current length (no holes). Rows are copied bit for bit.
 * Whisper slots still need dec_prefill (n_tokens may be 0) for cross K/V.
 */
dec_status dec_kv_append(dec_handle* h, int32_t slot, int32_t start_pos, int32_t n_rows,
                         const float* k, const float* v, void* stream);

/*
 * One decode step over `batch` streams.
 *   slots       host int32 [batch], distinct slot ids, or NULL for 0..batch-1
 *   tokens      host int32 [batch] input tokens, or NULL to feed each slot its
 *               own previous greedy pick (set by the last dec_step/dec_prefill
 *               on that slot; DEC_ESTATE if it has none)
 *   positions   host int32 [batch]: learned-position row (whisper) or RoPE
 *               position (qwen2) of the new token ([focr] batched step:
 *               positions passed explicitly so the caller stays in charge)
 *   cache_lens  host int32 [batch]: must equal each slot's current length
 *               ([cera] `decode_step_into` checks seq_len == pos); the new
 *               K/V row is written at that row and attention covers rows
 *               0..cache_lens[b]; on success each slot's length grows by one
 *   logits      device f32 [batch, vocab] or NULL (not written)
 *   argmax      device int32 [batch] or NULL: greedy pick, lowest index on ties
 *               ([focr] `argmax`)
 * Queues the work on `stream` and returns without synchronising.
 */
dec_status dec_step(dec_handle* h, int32_t batch, const int32_t* slots, const int32_t* tokens,
                    const int32_t* positions, const int32_t* cache_lens, float* logits,
                    int32_t* argmax, void* stream);

/*
 * dec_step with host result buffers: queues the step, copies logits (host f32
 * [batch, vocab] or NULL) and argmax (host int32 [batch] or NULL) back, and
 * synchronises `stream` before returning. Host buffers may be pageable;
 * pinned buffers copy faster.
 */
dec_status dec_step_host(dec_handle* h, int32_t batch, const int32_t* slots,
                         const int32_t* tokens, const int32_t* positions,
                         const int32_t* cache_lens, float* logits_host, int32_t* argmax_host,
                         void* stream);

/*
 * Each listed slot's greedy continuation token (the argmax of its most recent
 * dec_prefill last row or dec_step row) into host `tokens` [n]. Synchronises
 * `stream`; DEC_ESTATE for a slot with no continuation yet, DEC_ETIMEOUT (and
 * the handle becomes failed) when a bounded device wait gave up.
 */
dec_status dec_next_tokens(dec_handle* h, int32_t n, const int32_t* slots, int32_t* tokens, void* stream);

/* The configuration the handle was created with. */
dec_status dec_get_config(const dec_handle* h, dec_config* out);

/*
 * Greedy generation for many requests with continuous batching ([focr]
 * `BatchScheduler::run`, `generate_greedy_batched`). Requests are admitted in
 * order whenever one of min(max_active, max_slots, DEC_MAX_BATCH) slots is
 * free: the prompt is prefilled and its last row's argmax is the first token.
 * Every iteration then advances all admitted streams by one token with one
 * dec_step. A stream retires after emitting `eos` (which is kept in its
 * output) or `max_new` tokens, or when its next row would overflow the cache
 * or the position range; its slot is refilled from the queue before the next
 * step. A stream's tokens are those it would get alone (the step's per-stream
 * arithmetic does not depend on the batch). A retired stream's slot is released
 * (dec_release_slot), so a paged cache returns its pages to the pool at once.
 *   reqs        host [n_reqs]; prompt host int32 [n_prompt] (n_prompt >= 1);
 *               enc_hidden device f32 [enc_len, d] for whisper, NULL for qwen2
 *   tokens_out  host int32 [n_reqs, stride]: request r's tokens in row r
 *   n_out       host int32 [n_reqs]: tokens written per request
 * Synchronises `stream` once per step. Uses (and overwrites) slots
 * 0..min(max_active, max_slots) - 1 of the handle.
 */
typedef struct dec_request {
    const int32_t* prompt;
    int32_t n_prompt;
    int32_t max_new;
    int32_t eos;               /* stop token, or -1 for none */
    const float* enc_hidden;
} dec_request;
dec_status dec_generate(dec_handle* h, const dec_request* reqs, int32_t n_reqs, int32_t max_active,
                        int32_t* tokens_out, int32_t stride, int32_t* n_out, void* stream);

/* Empty `slot`: its length becomes 0 and, with a paged cache, its pages return to the
 * pool. The slot needs dec_prefill or dec_kv_append before its next step. */
dec_status dec_release_slot(dec_handle* h, int32_t slot);

/* Free pages in the paged cache's pool (0 for a dense cache). */
dec_status dec_kv_pages_free(const dec_handle* h, int32_t* pages);

/* Current length (cached rows) of `slot` as tracked by the handle. */
dec_status dec_slot_len(const dec_handle* h, int32_t slot, int32_t* len);

/*
 * Copy rows [start, start + n) of layer `layer`'s self-attention K and V of
 * `slot` into device buffers k_out, v_out (f32 [n, kv heads * 64], token-major).
 * Rows at or beyond the slot length hold whatever was last written there.
 */
dec_status dec_kv_read(dec_handle* h, int32_t slot, int32_t layer, int32_t start, int32_t n,
                       float* k_out, float* v_out, void* stream);

/* Copy the residual stream after the last layer of the most recent dec_step
 * (before the final norm), f32 [batch, d_model], into device `out`. */
dec_status dec_hidden(dec_handle* h, float* out, int32_t batch, void* stream);

/*
 * Parity bisection ([wa-dec] `forward_traced`: per-layer hidden states for
 * comparison against a reference). While `buf` is not NULL, every dec_step /
 * dec_step_host also copies the residual stream leaving each layer (after its
 * FFN residual add, before the next layer's norm) into device `buf` as f32
 * [n_layers, batch, d_model] for that step's batch; `buf` must hold
 * n_layers * batch * d_model floats for every later step's batch (the caller
 * owns it; it must stay valid while set). NULL turns tracing off. Traced steps
 * run as their own captured graphs (one extra device-to-device copy per layer).
 * dec_prefill's prompt chunks are not traced.
 */
dec_status dec_set_layer_trace(dec_handle* h, float* buf);

/*
 * Synchronise `stream` and report device-side failures: DEC_ETIMEOUT when a
 * bounded wait inside one of the handle's kernels gave up (a copy that never
 * landed; lattice-inference-style fail-closed reporting instead of a hang). The
 * kernel that gave up returned early, so that step's results are not valid.
 * From then on the handle is failed: dec_step, dec_step_host, dec_prefill and
 * dec_kv_append return DEC_ETIMEOUT without queueing work until dec_reset.
 * dec_step_host checks the status word itself (it synchronises anyway).
 */
dec_status dec_sync(dec_handle* h, void* stream);

/*
 * Recover a failed handle: synchronise the device, clear the status word and
 * every arrival counter and argmax key the kernels share across launches, and
 * empty every slot (its cache contents are no longer trusted; prefill or
 * dec_kv_append it again). The wait limit and the weights are kept.
 */
dec_status dec_reset(dec_handle* h);

/*
 * Limit of every bounded device wait of this handle's kernels, in nanoseconds
 * (0: the default of one second). Synchronous (writes the handle's status block).
 */
dec_status dec_set_wait_limit(dec_handle* h, uint64_t ns);

/*
 * Test hooks for the failure path; no fault is ever raised on the device.
 *   dec_debug_inject(h, DEC_INJECT_DROP_ATTN_COPY, 1): in every later step the
 *     first self-attention CTA of layer 0 announces its first K/V tile on its
 *     mbarrier but issues no copy, so its bounded wait runs out (after the
 *     handle's wait limit) and the step reports DEC_ETIMEOUT; such steps run
 *     without CUDA-graph capture. Value 0 switches it off.
 *   dec_debug_fail_alloc(n): the n-th device or pinned-host allocation made by
 *     the next dec_create on the calling thread fails, which must return
 *     DEC_ENOMEM with everything already allocated freed; 0 switches it off.
 */
enum { DEC_INJECT_DROP_ATTN_COPY = 1 };
dec_status dec_debug_inject(dec_handle* h, int32_t what, int32_t value);
void dec_debug_fail_alloc(int32_t nth);

/* Number of kernels one step of the most recent dec_step / dec_step_host call
 * launches (the kernel nodes of its captured CUDA graph), or -1 when that step's
 * launch sequence could not be captured. Host-only; never blocks. */
dec_status dec_step_kernels(const dec_handle* h, int32_t* kernels);

/*
 * Kernel-level entry points (no handle). They run one kernel of the step on
 * caller-provided device buffers, for testing each kernel on its own.
 */

/*
 * Split-K decode attention over head-first caches ([focr] `decode_attn_head`:
 * s_j = q . k_j / 8, max-subtracted softmax, sum_j p_j v_j; a row whose
 * softmax sum is not finite and positive gives zeros, [q8] full-attention step).
 *   q        device f32 [batch, n_heads, 64]
 *   k, v     device f32 [batch, n_heads, ld, 64] (head-first, ld rows per head),
 *            16-byte aligned
 *   lens     device int32 [batch]: keys attended per stream (rows 0..lens[b]-1),
 *            0 <= lens[b] <= ld; lens[b] == 0 gives zeros
 *   tiles_per_split  64-key tiles per CTA of a row: 0 splits every row alike
 *            (the split count minimising waves x tiles per CTA); a positive value
 *            fixes each row's split boundaries from its own length, as the decode
 *            step does (dec_attention_plan gives a handle's value); at most 32
 *            splits over ld rows (DEC_EINVAL otherwise)
 *   out      device f32 [batch, n_heads, 64]
 *   workspace device scratch of at least dec_attention_workspace_size(batch,
 *            n_heads, ld) bytes, 16-byte aligned; its first
 *            batch * n_heads int32 must be zero before the first call (each call
 *            leaves them zero again)
 * Errors set dec_last_error(NULL).
 */
size_t dec_attention_workspace_size(int32_t batch, int32_t n_heads, int32_t ld);
dec_status dec_attention(const float* q, const float* k, const float* v, const int32_t* lens,
                         int32_t batch, int32_t n_heads, int32_t ld, int32_t tiles_per_split, float* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Tiles per split of a handle's self-attention (cross = 0) or cross-attention
 * (cross = 1, whisper) launches in dec_step, for timing the step's own launch
 * shape through dec_attention. Host-only. */
dec_status dec_attention_plan(const dec_handle* h, int32_t cross, int32_t* tiles_per_split);

/*
 * Allocation-free variant of dec_attention, for callers that cannot allocate
 * device memory themselves: code that runs under a host framework whose allocator
 * owns the whole device and hands plug-ins no workspace, or latency-critical
 * paths where cudaMalloc's implicit device synchronisation is not acceptable.
 * (It has no counterpart in the pages; it is an interface convenience only.)
 * Same arguments as dec_attention with tiles_per_split = 0, minus the workspace,
 * and the same launch, hence the same output bits: the split-K scratch lives in
 * one fixed array of about 8.9 MB inside this library, which every GPU that loads
 * the library holds until the process exits.
 * Limits: batch * n_heads <= 1024 (DEC_EINVAL otherwise, message from
 * dec_last_error(NULL)). Every call looks up that array's device address
 * (cudaGetSymbolAddress) with the calling thread's current device; make the first
 * call on a device before any stream capture (it may load the module). Every call
 * clears the status word and the arrival counters it needs (cudaMemsetAsync on
 * `stream`) and shares the one array, which keeps the last call's contents: calls
 * that overlap on the GPU (different streams, no ordering) race on it. A bounded
 * device wait that gives up (about a second) leaves `out` undefined; it is noted in
 * the array's status word only and not reported by this call. It allocates nothing.
 */
dec_status dec_attention_noalloc(const float* q, const float* k, const float* v, const int32_t* lens,
                                 int32_t batch, int32_t n_heads, int32_t ld, float* out, void* stream);

/*
 * int8 x int8 -> int32 dot products acc[m, n] = sum_k xq[m, k] * wq[n, k]
 * (the accumulator of [focr] `gemv_i8_bias_prequant`). xq device int8 [m, kdim],
 * wq device int8 [n, kdim], acc device int32 [m, n]; kdim a multiple of 16,
 * 1 <= m <= 64, xq and wq 16-byte aligned. `path` selects the kernel the decode
 * step uses for that batch size: DEC_I8_PATH_DP4A (CUDA cores, dp4a, batches
 * below 8) or DEC_I8_PATH_TCGEN05 (tcgen05.mma kind::i8 with TMEM accumulators,
 * batches of 8 or more; this path allocates its split-K scratch with
 * cudaMallocAsync on `stream` and frees it after the launch). Errors set
 * dec_last_error(NULL).
 */
enum { DEC_I8_PATH_DP4A = 0, DEC_I8_PATH_TCGEN05 = 1 };
dec_status dec_i8_dot(const int8_t* xq, const int8_t* wq, int32_t m, int32_t n, int32_t kdim, int32_t path,
                      int32_t* acc, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DEC_H */
