/*
 * minikv.h -- C ABI of libminikv.so: the MiniKV hot path on NVIDIA B200 (sm_100a).
 *
 * MiniKV ("MiniKV: Pushing the Limits of LLM Inference via 2-Bit
 * Layer-Discriminative KV Cache") keeps, per layer, only the keys that earned
 * the most attention from the last W prompt queries, stores them in 2 bits, and
 * attends over that cache during decoding.  The pages that describe it give the
 * ideas, not the formulas:
 *   - abstract: a 2-bit, layer-discriminative KV cache, with CUDA kernels made
 *     compatible with FlashAttention;
 *   - gptget.net summary of arXiv 2411.18077, section 方法论 / 方法详解:
 *     sub-channel (per-channel) key quantization, per-token value quantization,
 *     a compact cache layout, and "selective flash attention" done by a second
 *     kernel;
 *   - same page, glossary 术语表 "adaptive KV": keep the KV states that matter;
 *   - pre.notesum.ai LongBench table, "MiniKV Pyramid" rows: a keep budget that
 *     differs by layer.
 * The calls below are this library's reading of those steps.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers, owned by the caller.  The library
 *     never allocates, frees or keeps them.  fp16 values are passed as uint16_t
 *     bit patterns (IEEE binary16).  Tensors are contiguous, row-major.
 *   - Work is queued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and runs asynchronously.  No call synchronizes the device.
 *   - Return value: MINIKV_OK (0) or a negative MINIKV_ERR_* code.  On error
 *     nothing was queued, the cache descriptor is unchanged, and
 *     minikv_last_error_string() (per host thread) says why.  A device fault, if
 *     any, surfaces at the caller's next synchronization; kernels never trap.
 *   - Head size D must be 128.  Query head h reads KV head h / (Hq / Hkv)
 *     (grouped-query attention with contiguous groups).
 */
#ifndef MINIKV_H
#define MINIKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MINIKV_API __attribute__((visibility("default")))
#else
#define MINIKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MINIKV_OK                0
#define MINIKV_ERR_INVALID_ARG  -1  /* null pointer, bad shape, W > keep, ... */
#define MINIKV_ERR_UNSUPPORTED  -2  /* D != 128, G not 32/64/128, ...        */
#define MINIKV_ERR_CAPACITY     -3  /* the packed cache would exceed `cap`     */
#define MINIKV_ERR_CUDA         -4  /* a CUDA launch or attribute call failed  */

/*
 * Packed 2-bit cache of ONE layer, for B sequences x Hkv KV heads.
 * Device arrays (caller-allocated; minikv_cache_bytes/minikv_cache_bind carve
 * them from one buffer):
 *   k_codes, v_codes [B, Hkv, cap, D/16] uint32: packed token t holds 16 codes
 *       per word; code of channel 16w+i sits in bits 2i..2i+1 of word w.
 *   k_scale, k_zero  [B, Hkv, cap/G, D] fp16: one (scale, zero) per key channel
 *       per group of G consecutive packed tokens (groups start at token 0).
 *   v_scale, v_zero  [B, Hkv, cap, D/Gv] fp16: one (scale, zero) per token per
 *       block of Gv consecutive value channels.
 *   k_res, v_res     [B, Hkv, R+G, D] fp16: ring of the newest tokens, kept in
 *       fp16; logical residual token i (0 = oldest) is in slot
 *       (res_start + i) mod (R+G).
 * Host-side state: n_packed packed tokens (a multiple of G), n_res residual
 * tokens, ring origin res_start.  Calls update it synchronously when they
 * queue their work.
 *   - Uniform batch (seq == NULL): one state for every sequence and head.
 *   - Ragged batch (seq != NULL, see minikv_cache_set_ragged): seq is a HOST
 *     array [B][3] = (n_packed, n_res, res_start) per sequence, owned by the
 *     caller and kept alive while the cache is used; the three scalars are then
 *     not read.  Sequences of one batch may hold different numbers of packed
 *     and residual tokens (unequal prompts, unequal budgets).
 *   - Device-resident state (dseq != NULL, see minikv_cache_set_device_state):
 *     the per-sequence state lives in a DEVICE array [B][4] = (n_packed,
 *     n_res, res_start, status); kernels read and advance it, the host fields
 *     are not read, and a decode step queues the same launches whatever the
 *     lengths, so a caller can capture steps in a CUDA graph and replay them.
 * Dequantized value of a code c: c * scale + zero.
 */
typedef struct minikv_cache {
    int B, Hkv, D, G, Gv, R, cap;
    uint32_t *k_codes, *v_codes;
    uint16_t *k_scale, *k_zero;
    uint16_t *v_scale, *v_zero;
    uint16_t *k_res, *v_res;
    int n_packed, n_res, res_start;
    int *seq;
    int *dseq;
} minikv_cache;

/* Most sequences a ragged batch may hold. */
#define MINIKV_MAX_RAGGED_SEQS 256

/* Bytes of device memory one layer's cache needs (each array 256-byte aligned),
 * or 0 if the shape is invalid. */
MINIKV_API size_t minikv_cache_bytes(int B, int Hkv, int D, int G, int Gv, int R, int cap);

/* Fill *c with the shape, point its arrays into `base` (a device buffer of at
 * least minikv_cache_bytes(...) bytes, 256-byte aligned) and reset the state to
 * empty (uniform batch, seq = NULL).  Touches no device memory. */
MINIKV_API int minikv_cache_bind(minikv_cache *c, void *base, size_t bytes,
                      int B, int Hkv, int D, int G, int Gv, int R, int cap);

/*
 * minikv_cache_set_ragged -- give each sequence of the batch its own length.
 * Source: none on the pages (they state no batching rule); serving batches
 * prompts of unequal length, so each sequence keeps its own packed and
 * residual counts.
 *   seq: HOST array of 3*B ints, caller-owned, alive while the cache is used;
 *   every sequence is reset to empty (0, 0, 0).  seq = NULL turns the cache
 *   back into a uniform batch, also empty.  Touches no device memory.
 * Afterwards minikv_quant_pack / minikv_evict_pack set every sequence (same
 * length for all), minikv_quant_pack_seq / minikv_evict_pack_seq set one, and
 * the decode calls step every sequence from its own state.
 * Errors: INVALID_ARG (null cache), UNSUPPORTED (B > MINIKV_MAX_RAGGED_SEQS).
 */
MINIKV_API int minikv_cache_set_ragged(minikv_cache *c, int *seq);

/*
 * minikv_cache_set_device_state -- keep the per-sequence state on the GPU.
 * Source: none on the pages; decode steps whose launches do not depend on the
 * host's view of the lengths can be captured once in a CUDA graph and
 * replayed every step, which removes the per-call host cost.
 *   dseq: DEVICE array of 4*B int32, 16-byte aligned, caller-owned, alive while
 *   the cache is used: (n_packed, n_res, res_start, status) per sequence.  It
 *   is zero-filled on `stream` (every sequence empty).  dseq = NULL returns to
 *   host-side state (also empty).
 * In this mode the loaders (minikv_quant_pack, minikv_evict_pack and their
 * _seq forms) write the loaded rows' state into dseq from their kernel, and
 * each decode call runs one launch configuration fixed by the cache's shape:
 * the kernel reads the state, splits this step's packed tokens over its CTAs,
 * and writes every sequence's next state once all its CTAs have read the
 * current one (minikv_decode_attn_static reads and advances the same state).  A step whose flush would pass `cap` leaves that
 * sequence's state unchanged (its new token is not kept) and sets its status
 * word to 1; the host learns it by reading dseq.  Capacity is therefore not
 * checked on the host in this mode.
 * Errors: INVALID_ARG (null cache, misaligned dseq), UNSUPPORTED
 * (B > MINIKV_MAX_RAGGED_SEQS), CUDA (the fill could not be queued).
 */
MINIKV_API int minikv_cache_set_device_state(minikv_cache *c, int *dseq, void *stream);

/*
 * minikv_quant_pack -- load a fresh compacted sequence into the cache.
 * Source: summary page, 方法论 (sub-channel key quantization, per-token value
 * quantization, compact layout); the fp16 residual of the newest tokens.
 *   k, v      [B, Hkv, n_tokens, D] fp16, the kept tokens in position order.
 * Split: with N = n_tokens, the newest r tokens stay fp16, r = R + (N-R) mod G
 * if N >= R, else r = N; the oldest N - r (a multiple of G) are quantized:
 *   keys  : per channel over each group of G tokens; values: per token over
 *           each block of Gv channels;
 *   mn = min x, mx = max x (a zero extreme counts as +0);
 *   scale = fp16_rn(fp32(mx - mn) / 3), zero = mn;
 *   code = 0 if scale == 0, else clamp(rint((x - zero) / scale), 0, 3) in fp32
 *   (IEEE round-to-nearest-even at every step).
 * The cache state becomes n_packed = N - r, n_res = r, res_start = 0.
 * Errors: INVALID_ARG (null, n_tokens < 0), CAPACITY (N - r > cap),
 * UNSUPPORTED (shape).
 */
MINIKV_API int minikv_quant_pack(minikv_cache *c, const uint16_t *k, const uint16_t *v,
                      int n_tokens, void *stream);

/*
 * minikv_quant_pack_seq -- minikv_quant_pack for sequence b of a ragged cache
 * only: k, v [Hkv, n_tokens, D] fp16 become sequence b's kept tokens (same
 * split and quantizer); seq[b] = (n_tokens - r, r, 0).  Other sequences are
 * untouched.
 * Errors: as minikv_quant_pack; INVALID_ARG also if the cache is neither
 * ragged nor device-state, or b is outside [0, B).
 */
MINIKV_API int minikv_quant_pack_seq(minikv_cache *c, int b, const uint16_t *k, const uint16_t *v,
                                     int n_tokens, void *stream);

/*
 * minikv_select_prefill -- "selective flash attention" over the prompt.
 * Source: summary page, 方法详解, third bullet (selective flash attention by a
 * second kernel); abstract (FlashAttention compatibility).
 *   q [B, Hq, T, D], k, v [B, Hkv, T, D] fp16.
 *   o [B, Hq, T, D] fp16: o_i = sum_{j<=i} softmax_j(sm_scale * q_i.k_j) v_j.
 *   scores [B, Hkv, T] fp32: scores[j] = sum over the Hq/Hkv query heads of the
 *       KV head and over the last W rows i in [T-W, T) of the softmax
 *       probability P[i, j] (0 where j > i).
 * Pass 1 is a causal flash-attention forward on the tcgen05 tensor cores
 * (128-row query tiles, operands brought in by TMA) that also records the row
 * log-sum-exp of the window rows in `ws`; pass 2 (the second kernel) recomputes
 * the window rows' probabilities from it and sums them per key.
 *   sm_scale > 0 (the usual 1/sqrt(D)).
 *   ws: device scratch of minikv_workspace_size(MINIKV_OP_SELECT_PREFILL, ...)
 *       bytes, no initial contents required; it also holds the call's status
 *       word (minikv_select_prefill_status).
 * Errors: INVALID_ARG (null, W < 1, W > T, Hq % Hkv, sm_scale <= 0, ws too
 * small), UNSUPPORTED (D != 128), CUDA (tensor-map encoding or launch failed).
 */
MINIKV_API int minikv_select_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          int B, int Hq, int Hkv, int T, int D, int W, float sm_scale,
                          uint16_t *o, float *scores, void *ws, size_t ws_bytes,
                          void *stream);

/*
 * minikv_select_prefill_status -- did the last minikv_select_prefill on this
 * workspace finish its work?  The flash-attention pass waits on its own copies
 * and tensor-core operations with bounded waits; if a wait gives up (a copy
 * that never lands), the CTA drains what it started, skips its outputs and
 * sets bit 0 of a status word in `ws`, instead of hanging or trapping.
 * minikv_select_prefill clears the word on its stream before its kernels.
 * Source: none on the pages (failure reporting of this library).
 *   ws, ws_bytes, B, Hq, W: as passed to that minikv_select_prefill.
 *   *status (host): 0 = every CTA finished; bit 0 = a bounded wait expired, the
 *   call's o / scores are not valid.
 * Queues a 4-byte device-to-host copy on `stream` and synchronizes the stream.
 * Errors: INVALID_ARG (null, shape, ws smaller than the call's), CUDA.
 */
MINIKV_API int minikv_select_prefill_status(const void *ws, size_t ws_bytes, int B, int Hq, int W, void *stream,
                                            unsigned *status);

/*
 * minikv_topk_evict -- adaptive KV: keep the tokens that matter.
 * Source: summary page, glossary 术语表 "adaptive KV" (keep KV states by
 * importance); notesum LongBench table, "MiniKV Pyramid" (the caller picks
 * `keep` per layer).
 *   scores [B, Hkv, T] fp32 (from minikv_select_prefill); k, v [B, Hkv, T, D].
 *   If keep >= T every position is kept (n = T).  Otherwise (W <= keep) the
 *   window [T-W, T) is kept, plus the keep-W positions j < T-W with the highest
 *   scores; equal scores go to the lower index.  n = min(keep, T).
 *   idx [B, Hkv, n] int32: kept positions, ascending.
 *   k_kept, v_kept [B, Hkv, n, D] fp16: rows k[idx], v[idx] (exact copies).
 *   ws: minikv_workspace_size(MINIKV_OP_TOPK_EVICT, ...) bytes (may be 0).
 * Errors: INVALID_ARG (null, keep < 1, W > keep < T).
 */
MINIKV_API int minikv_topk_evict(const float *scores, const uint16_t *k, const uint16_t *v,
                      int B, int Hkv, int T, int D, int W, int keep,
                      int32_t *idx, uint16_t *k_kept, uint16_t *v_kept,
                      void *ws, size_t ws_bytes, void *stream);

/*
 * minikv_evict_pack -- minikv_topk_evict followed by minikv_quant_pack in one
 * call, without the fp16 copy of the kept rows in between.
 * Source: the same passages as the two calls it fuses (glossary "adaptive KV";
 * 方法论, the compact 2-bit layout): keep by importance, then quantize what is
 * kept.
 *   scores [B, Hkv, T] fp32, k, v [B, Hkv, T, D] fp16 (the prompt), as for
 *   minikv_topk_evict; idx [B, Hkv, n] int32 receives the kept positions
 *   (n = min(keep, T), ascending).  The kept rows are read straight from k and
 *   v and packed into *c exactly as minikv_quant_pack(c, k[idx], v[idx], n)
 *   would pack them (same codes, scales, zeros and residual, bit for bit);
 *   the cache state is reset the same way.
 *   B, Hkv must match the cache.  No workspace.
 * Errors: INVALID_ARG (null, misaligned, keep < 1, W > keep < T, B/Hkv differ
 * from the cache), UNSUPPORTED (D != 128, bad cache shape), CAPACITY (the
 * packed part would exceed cap).
 */
MINIKV_API int minikv_evict_pack(const float *scores, const uint16_t *k, const uint16_t *v,
                      int B, int Hkv, int T, int D, int W, int keep,
                      int32_t *idx, minikv_cache *c, void *stream);

/*
 * minikv_evict_pack_seq -- minikv_evict_pack of ONE prompt (scores [Hkv, T],
 * k, v [Hkv, T, D], idx [Hkv, min(keep, T)]) into sequence b of a ragged
 * cache; T and keep are this prompt's own.  Other sequences are untouched.
 * Errors: as minikv_evict_pack; INVALID_ARG also if the cache is neither
 * ragged nor device-state, or b is outside [0, B).
 */
MINIKV_API int minikv_evict_pack_seq(const float *scores, const uint16_t *k, const uint16_t *v,
                                     int Hkv, int T, int D, int W, int keep, int32_t *idx,
                                     minikv_cache *c, int b, void *stream);

/*
 * minikv_decode_attn -- one decoding step of one layer over the 2-bit cache.
 * Source: abstract ("specialized CUDA kernels ... compatible with
 * FlashAttention"); summary page, 方法论 (the compact 2-bit layout it reads).
 *   q [B, Hq, D] fp16; k_new, v_new [B, Hkv, D] fp16 (this step's token).
 *   out [B, Hq, D] fp16.
 * 1. Append (k_new, v_new) as the newest residual token.
 * 2. out_h = sum_t softmax_t(sm_scale * q_h . kappa_t) nu_t over all packed
 *    tokens (dequantized in registers) and all residual tokens, new one
 *    included.  Flash-decoding: the tokens are split across CTAs and the
 *    partial softmax states are merged by the last CTA of each KV head.
 * 3. If the residual now holds R+G tokens, its oldest G are quantized (same
 *    rules as minikv_quant_pack) into key group n_packed/G: n_packed += G,
 *    n_res -= G.
 * On a ragged cache every step runs per sequence, from and into its own state
 * (one launch for the whole batch; the split of packed tokens over CTAs
 * follows the actual per-sequence lengths).
 *   ws: minikv_workspace_size(MINIKV_OP_DECODE_ATTN, B, Hq, Hkv, cap + R + G, D, 0)
 *       bytes, ZERO-FILLED before its first use; every call leaves it ready for
 *       the next (its arrival counters return to zero).  Calls that share one
 *       ws must not overlap on the GPU.
 * Errors: INVALID_ARG (null, Hq % Hkv, ws too small), CAPACITY (a flush would
 * exceed cap), UNSUPPORTED (D != 128, Gv != D, G not 32/64/128, more than 4
 * query heads per KV head).
 */
MINIKV_API int minikv_decode_attn(minikv_cache *c, const uint16_t *q, const uint16_t *k_new,
                       const uint16_t *v_new, int Hq, float sm_scale, uint16_t *out,
                       void *ws, size_t ws_bytes, void *stream);

/*
 * minikv_decode_attn_mass -- minikv_decode_attn that also accumulates, per
 * cached token, the attention mass the step gave it (H2O-style scores).
 * Source: summary page, 实验设计 (experiments), which names H2O -- eviction by
 * accumulated attention -- among the methods MiniKV is compared with; the
 * per-KV-head sum over the query heads of the group follows the window score
 * of minikv_select_prefill.
 *   Arguments, output `out`, cache update and errors as minikv_decode_attn, plus:
 *   mass [B, Hkv, cap + R + G] fp32, caller-owned, 4-byte aligned, updated in
 *       place: for every token t the step attends to,
 *         mass[b, kvh, t] += sum over the Hq/Hkv query heads h of KV head kvh
 *                            of softmax_t(sm_scale * q_h . kappa_t),
 *       where t numbers the tokens in the order they entered the cache: the
 *       n_packed packed tokens first (t = 0 .. n_packed-1), then the residual,
 *       oldest first, the new token last (t = n_packed + n_res, counted before
 *       this step's flush).  A flush keeps every token's t.  Entries from
 *       n_packed + n_res + 1 on are not touched.  Each step adds exactly Hq/Hkv
 *       to the sum over t (up to fp32 rounding).
 *   ws: minikv_workspace_size(MINIKV_OP_DECODE_ATTN_MASS, B, Hq, Hkv,
 *       cap + R + G, D, 0) bytes, zero-filled before first use, reusable like
 *       the workspace of minikv_decode_attn.
 * Two kernels are queued: the decode kernel, which also stores each token's
 * log2 score per query head in ws, and a pass that turns them into
 * probabilities with the merged softmax state and adds them to `mass`.
 * Choosing tokens to drop by `mass` is left to the caller.
 * Errors: those of minikv_decode_attn; INVALID_ARG also for a null or
 * misaligned `mass`.
 */
MINIKV_API int minikv_decode_attn_mass(minikv_cache *c, const uint16_t *q, const uint16_t *k_new,
                                       const uint16_t *v_new, int Hq, float sm_scale, uint16_t *out,
                                       float *mass, void *ws, size_t ws_bytes, void *stream);

/*
 * minikv_decode_attn_static -- minikv_decode_attn without a caller workspace.
 * The paper has no counterpart to this call; it exists for callers that may
 * not allocate device memory: hosts whose device memory is entirely planned by
 * their own allocator or pool (a cudaMalloc behind its back would break its
 * accounting and budget) and latency-critical loops where cudaMalloc is not
 * allowed because it can synchronize the device.
 * Same arguments, semantics, results and errors as minikv_decode_attn, minus
 * `ws`: the scratch is a fixed 8 MiB array inside the library's device module,
 * held by every GPU that loads the library until the process exits.  A step
 * whose scratch need is larger fails with MINIKV_ERR_UNSUPPORTED and queues
 * nothing; minikv_decode_attn with a caller workspace has no such limit.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, that device current); make it before any stream
 * capture.  All calls share the array: calls whose GPU work overlaps race on
 * it.  Each call clears the array's arrival counters on `stream` first.  No
 * call allocates or frees device memory.  `stream` must belong to the current
 * device (the array's address is the current device's); otherwise the call
 * fails with MINIKV_ERR_INVALID_ARG and queues nothing.
 */
MINIKV_API int minikv_decode_attn_static(minikv_cache *c, const uint16_t *q, const uint16_t *k_new,
                                         const uint16_t *v_new, int Hq, float sm_scale, uint16_t *out,
                                         void *stream);

#define MINIKV_OP_SELECT_PREFILL 1
#define MINIKV_OP_TOPK_EVICT     2
#define MINIKV_OP_DECODE_ATTN    3
#define MINIKV_OP_DECODE_ATTN_MASS 4

/*
 * minikv_decode_plan -- how the next minikv_decode_attn (or _mass, _static)
 * call on this cache state splits its work.  Host logic only: touches no
 * device memory and launches nothing; without a GPU it assumes 148 SMs.
 * The work list: for each (sequence, KV head) unit in order,
 * ceil((n_res + 1) / 5) residual items of up to 5 fp16 tokens (the new token
 * included), then n_packed / 32 packed items of 32 tokens.  It is cut into
 * one contiguous range per CTA at equal steps of a weight: 8 per packed
 * item, 7 per residual item, plus a boundary weight before each unit's first
 * item, chosen per call from 128, 256, 512, 896, 1280 and 2^20 by a cost
 * model of the slowest CTA (2^20 gives one CTA per unit when units are few).
 *   *ctas: CTAs that take a range (at most one per SM).
 *   *boundary_weight: the boundary weight of the cut (640 for a cache with
 *     device-resident state, whose CTAs cut the list themselves on the GPU).
 *   first_items: if n_first > 0, at least *ctas + 1 entries: the first item of
 *     each CTA's range, then the number of items.  Not written for a cache
 *     with device-resident state.
 * The answer depends only on the cache's shape and state (and the SM count).
 * Errors: INVALID_ARG (null, bad cache, n_first too small), UNSUPPORTED (as
 * for minikv_decode_attn: B*Hkv or the item count too large).
 */
MINIKV_API int minikv_decode_plan(const minikv_cache *c, int *ctas, int *boundary_weight, int *first_items,
                                  int n_first);

/* Scratch bytes an op needs.  For MINIKV_OP_DECODE_ATTN and
 * MINIKV_OP_DECODE_ATTN_MASS pass the cache capacity plus R+G as T (the most
 * tokens a step can attend to). */
MINIKV_API size_t minikv_workspace_size(int op, int B, int Hq, int Hkv, int T, int D, int W);

/*
 * minikv_set_deterministic -- choose how the decode calls spread their work
 * inside a CTA (process-wide; takes effect at the next decode call).
 *   on = 0 (default): the 16 warps of a CTA claim 32-token items from a
 *     shared counter, so a warp that the scheduler favours takes more.  Which
 *     warp sums which items then varies from run to run, and so does the fp32
 *     rounding of the sums: two identical calls may give fp16 outputs that
 *     differ by about one unit in the last place of the largest outputs
 *     (5e-4 for outputs below 1), a quarter of the 2e-3 tolerance.
 *   on = 1: warp w of a CTA takes items w, w + 16, w + 32, .. of its range.
 *     Identical calls give bit-identical outputs; the step can be slower when
 *     warps progress unevenly.
 * The cache contents (packed codes, scales, residual rows) are bit-identical
 * in both modes.  Returns MINIKV_OK.
 */
MINIKV_API int minikv_set_deterministic(int on);

/* Why the last failing call on this host thread failed ("" if none). */
MINIKV_API const char *minikv_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* MINIKV_H */
