/*
 * duo_attn.h -- C ABI of the B200 (sm_100a) DuoAttention hybrid-GQA
 * attention library (libduoattn.so).
 *
 * What is computed (DuoAttention Laguna Adapter model card, sections Summary
 * and Why It Works; Laguna sliding-window articles; Laguna-XS-2.1 cookbook,
 * section 1): each KV head of a layer is
 *   - a full-context head: the query at position i attends to every key
 *     j <= i, and the cache keeps every token;
 *   - a streaming head: the query attends to keys j <= i with j < sink or
 *     j > i - recent (sink 64, recent 256 on the pages), and the cache keeps
 *     only those: `sink` fixed slots plus a ring of `recent` slots;
 *   - on a sliding-window layer (window > 0, 512 on the pages) every head
 *     attends to keys i - window < j <= i and keeps a ring of `window` slots.
 * Query head h reads KV head h / (num_q_heads / num_kv_heads).  Scores are
 * softmax_scale * q.k; an optional per-query-head sink logit (not scaled)
 * joins the softmax denominator with a zero value vector, and the exported
 * log-sum-exp (natural log) includes it.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     keeps no pointer after the call returns and allocates no device memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream; a non-negative return only means the work
 *     was enqueued.
 *   - bf16 tensors are dense row-major with the shapes given; every tensor
 *     pointer must be 16-byte aligned.
 *   - Arguments are checked on the host before anything is launched; a call
 *     that returns an error has launched nothing and written nothing.
 *     Conditions that only the device can see (cache capacity overflow, a
 *     bounded wait that expired) set a device status word that
 *     duo_get_device_status() returns.
 *   - Supported geometry: head_dim 128, num_q_heads / num_kv_heads == 6,
 *     num_kv_heads <= 64, sequence positions below 2^30.
 */
#ifndef DUO_ATTN_H
#define DUO_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DUO_API __attribute__((visibility("default")))
#else
#define DUO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return and status codes. */
#define DUO_OK 0
#define DUO_ERR_INVALID_ARG (-1) /* NULL / misaligned pointer, bad size or range   */
#define DUO_ERR_UNSUPPORTED (-2) /* geometry outside what the kernels implement     */
#define DUO_ERR_CUDA (-3)        /* a CUDA runtime call or a launch failed          */
#define DUO_ERR_WORKSPACE (-4)   /* decode workspace NULL or smaller than required  */
#define DUO_ERR_TIMEOUT (-5)     /* device: a bounded wait inside a kernel expired  */
#define DUO_ERR_CAPACITY (-6)    /* device: an append ran past the full-cache capacity */
#define DUO_ERR_DEVICE (-7)      /* the current device is not sm_100 (B200)          */

/* One attention layer.
 *   window > 0 : sliding-window layer; full_mask, sink and recent are ignored.
 *   window == 0: DuoAttention layer; full_mask[g] == 1 marks KV head g as a
 *                full-context head, 0 as a streaming head (sink + recent).
 * full_mask is a HOST array [num_kv_heads]; sink_logit is a DEVICE array
 * [num_q_heads] of fp32 logits, or NULL for none. */
typedef struct {
    int32_t batch;          /* B >= 1                                        */
    int32_t num_q_heads;    /* Hq (48 on the pages)                          */
    int32_t num_kv_heads;   /* Hkv (8 on the pages); Hq == 6 * Hkv           */
    int32_t head_dim;       /* D, must be 128                                */
    int32_t sink;           /* streaming heads: sink tokens kept (64), >= 0  */
    int32_t recent;         /* streaming heads: recent tokens kept (256), >= 1 */
    int32_t window;         /* 0, or the sliding window (512), <= 8192       */
    float softmax_scale;    /* > 0, usually 1/sqrt(D)                        */
    const uint8_t *full_mask;  /* host [Hkv]                                 */
    const float *sink_logit;   /* device [Hq] fp32, or NULL                  */
} duo_params;

/* A layer's KV cache (all device memory, bf16, caller-owned).
 * Let n_full = number of full heads (0 on a sliding layer), n_ring =
 * Hkv - n_full, and ring_slots = sink + recent (Duo layer) or window
 * (sliding layer).  Head g's slot in either array is its rank among the
 * heads of its kind (the number of same-kind heads with a lower index).
 *   full_k, full_v : [B][n_full][capacity][D]  (may be NULL if n_full == 0)
 *   strm_k, strm_v : [B][n_ring][ring_slots][D] (may be NULL if n_ring == 0)
 *                    slots 0..sink-1 hold positions 0..sink-1; slots
 *                    sink..ring_slots-1 form the ring of recent tokens.
 *   seq_len        : device int32 [B], tokens appended so far.
 *   ring_head      : device int32 [B], ring slot (0..ring_slots-sink-1,
 *                    relative to the first ring slot) that the next ring
 *                    write goes to.  It advances once per appended position
 *                    >= sink.  Any starting value is allowed.
 * The valid ring slots are the min(max(seq_len - sink, 0), ring size) slots
 * written last, i.e. those just before ring_head, cyclically. */
typedef struct {
    void *full_k;
    void *full_v;
    int64_t capacity;       /* rows per full head, >= the longest sequence  */
    void *strm_k;
    void *strm_v;
    int32_t *seq_len;
    int32_t *ring_head;
} duo_cache;

/* Optional output gate of the attention (Laguna's gated attention output:
 * the Laguna attention article "深入理解Laguna的注意力机制", section on
 * attention output gating, and the Laguna XS 2.1 sliding-window article,
 * section on the g_proj output gate).  The normalised attention output of
 * query head h is multiplied by sigmoid(g) before it is rounded and stored:
 *   DUO_GATE_PER_ELEMENT  one g per (query head, channel), laid out like out;
 *   DUO_GATE_PER_HEAD     one g per query head, broadcast over the channels,
 *                         laid out like out without its last dimension
 *                         (prefill [B][L][Hq], decode [B][Hq]).
 * g is the model's gate projection output (bf16, device, 16-byte aligned);
 * computing it is not part of this library.  The pages do not name the gate's
 * activation: sigmoid is this library's reading.  The log-sum-exp output is
 * not gated.  A NULL duo_gate pointer, or mode DUO_GATE_NONE, means no gate. */
typedef enum {
    DUO_GATE_NONE = 0,
    DUO_GATE_PER_ELEMENT = 1,
    DUO_GATE_PER_HEAD = 2
} duo_gate_mode;

typedef struct {
    int32_t mode;           /* duo_gate_mode                                 */
    const void *values;     /* device bf16 gate pre-activations              */
} duo_gate;

/* Appends n_new tokens to every sequence of the cache.
 * k, v: device bf16 [B][n_new][Hkv][D] (token-major, as a K/V projection
 * writes them).  For each sequence b and token t the position is
 * p = seq_len[b] + t; a full head writes row p of its full cache; a
 * streaming / sliding head writes slot p if p < sink, else the ring slot the
 * sequential rule gives, and only tokens that would still be in the ring
 * after all n_new appends are written (the result equals n_new one-token
 * appends).  Afterwards seq_len[b] += n_new and ring_head advances.
 * On a layer with full heads, an append that would take seq_len[b] past
 * capacity stops there: the positions below capacity are appended, the rest
 * are dropped for every head, seq_len[b] becomes capacity, and
 * DUO_ERR_CAPACITY is set on the device (duo_get_device_status).
 * Defined by the DuoAttention card, section Summary (sink and
 * recent sizes) and section Why It Works (what each head keeps). */
DUO_API int duo_kv_append(const duo_params *params, const duo_cache *cache, const void *k,
                  const void *v, int32_t n_new, void *stream);

/* Bytes of device workspace duo_attn_prefill uses for dynamic work-tile
 * scheduling (the same for every layer). */
DUO_API size_t duo_prefill_workspace_bytes(void);

/* Query/key preparation fused into the append (Laguna attention article
 * "深入理解Laguna的注意力机制", section on YaRN dynamic RoPE: the
 * full-attention layers' rope parameters; Laguna XS 2.1 sliding-window
 * article, section on its attention optimisations: RMSNorm of the queries and
 * keys before the rotary embedding).  Per head row x of D = 128 channels:
 *   y = x / sqrt(mean(x^2) + rms_eps) * w        (w: the norm weight, or 1)
 *   then the rotary embedding at the token's cache position p, rotating the
 *   pairs (y[i], y[i + 64]), i < 64, by the angle p * inv_freq[i]:
 *   out[i]      = (y[i] cos a - y[i + 64] sin a) * attention_factor
 *   out[i + 64] = (y[i + 64] cos a + y[i] sin a) * attention_factor
 * inv_freq follows YaRN ("NTK-by-parts"): with base theta and D = 128,
 * f_i = theta^(-2i/D); dimensions that turn more than beta_fast times over
 * original_max_position keep f_i, those that turn fewer than beta_slow times
 * use f_i / rope_factor, and a linear ramp over the dimension index blends the
 * two in between (bounds floor / ceil of D ln(original_max_position /
 * (2 pi beta)) / (2 ln theta)).  rope_factor = 1 gives plain RoPE.  The
 * pages' full-attention values: theta 500000, factor 64, original 4096,
 * beta_fast 64, beta_slow 1, attention_factor 1.  Which half-pairing the
 * rotation uses, and the norm epsilon, are not on the pages: the (i, i + 64)
 * pairing and eps 1e-6 are this library's readings. */
typedef struct {
    float rope_theta;
    float rope_factor;
    int32_t original_max_position;
    float beta_fast;
    float beta_slow;
    float attention_factor;
    float rms_eps;
    const void *q_norm_weight;  /* device bf16 [D], or NULL for unit weight */
    const void *k_norm_weight;  /* device bf16 [D], or NULL for unit weight */
} duo_qk_prep;

/* duo_kv_append with the query/key preparation above fused in: for each
 * sequence b and token t (position p = seq_len[b] + t), every head row of q
 * [B][n_new][Hq][D] and k [B][n_new][Hkv][D] is normalised and rotated IN
 * PLACE (so that duo_attn_prefill / duo_attn_decode read the prepared
 * tensors), and the prepared k with v is appended exactly as duo_kv_append
 * appends it.  Results are rounded to bf16 once, after the rotation.  Errors
 * as duo_kv_append; a NULL prep, a non-positive theta, rope_factor < 1,
 * original_max_position < 1, beta_slow <= 0, beta_fast < beta_slow or
 * rms_eps < 0 is DUO_ERR_INVALID_ARG. */
DUO_API int duo_kv_append_prep(const duo_params *params, const duo_cache *cache,
                               const duo_qk_prep *prep, void *q, void *k, const void *v,
                               int32_t n_new, void *stream);

/* Prefill attention over a sequence that starts at position 0 (empty cache).
 * q: device bf16 [B][L][Hq][D]; k, v: device bf16 [B][L][Hkv][D]; L = seq_len.
 * out: device bf16 [B][L][Hq][D].  lse: device fp32 [B][Hq][L] (natural-log
 * log-sum-exp of the row's scores, sink term included) or NULL.
 * Query i of head h attends to the keys its KV head's rule allows (full:
 * j <= i; streaming: j < sink or i - recent < j <= i; sliding:
 * i - window < j <= i).  Computed with tcgen05 tensor cores (bf16 inputs,
 * fp32 accumulation, probabilities rounded to bf16 before the PV product).
 * workspace: NULL, or device memory of at least duo_prefill_workspace_bytes()
 * bytes, 16-byte aligned, owned by the caller; its contents need not be
 * initialised (the call zeroes it on the stream).  With a workspace the
 * persistent CTAs claim work tiles from a counter in it (balanced when the
 * heads' costs differ); without one they take a fixed stride of the list.
 * Calls that may run at the same time need separate workspaces.  A smaller
 * or misaligned workspace returns DUO_ERR_WORKSPACE.
 * gate: NULL or an output gate (see duo_gate; values [B][L][Hq][D] or
 * [B][L][Hq]).
 * The cache is not touched: call duo_kv_append(n_new = L) to fill it. */
DUO_API int duo_attn_prefill(const duo_params *params, const void *q, const void *k, const void *v,
                     int32_t seq_len, void *out, float *lse, void *workspace,
                     size_t workspace_bytes, const duo_gate *gate, void *stream);

/* Bytes of device workspace duo_attn_decode needs for this layer when no
 * sequence holds more than max_seq_len tokens.  Returns 0 on invalid params. */
DUO_API size_t duo_decode_workspace_bytes(const duo_params *params, int32_t max_seq_len);

/* One-token decode against the cache: the query of sequence b sits at
 * position seq_len[b] - 1 (append its K/V first).
 * q: device bf16 [B][Hq][D]; out: device bf16 [B][Hq][D]; lse: device fp32
 * [B][Hq] or NULL.  max_seq_len bounds every seq_len[b] (it sizes the split
 * of long caches into parallel pieces; a sequence longer than it is an error
 * the device cannot report, so pass a true bound).  workspace: device memory
 * of at least duo_decode_workspace_bytes(params, max_seq_len) bytes, 256-byte
 * aligned, contents need not be initialised.  A full head reads its seq_len
 * rows, a ring head only its valid sink and ring slots (at most
 * sink + recent or window).  A sequence with seq_len 0 gives out = 0 and
 * lse = -inf (or the sink logit when one is given).
 * gate: NULL or an output gate (see duo_gate; values [B][Hq][D] or [B][Hq]),
 * applied in the split merge. */
DUO_API int duo_attn_decode(const duo_params *params, const duo_cache *cache, const void *q,
                    int32_t max_seq_len, void *out, float *lse, void *workspace,
                    size_t workspace_bytes, const duo_gate *gate, void *stream);

/* Bytes of device workspace duo_attn_decode_block needs (0 on invalid
 * arguments or q_len outside [1, 2^30]). */
DUO_API size_t duo_decode_block_workspace_bytes(const duo_params *params, int32_t q_len,
                                                int32_t max_seq_len);

/* Block decode: q_len query tokens per sequence against the cache as it
 * stands BEFORE they are appended -- the verify pass of block speculative
 * decoding (Laguna-XS-2.1 cookbook, section 3.1 DFlash: the target checks a
 * drafted block in one forward pass and keeps the tokens it accepts), and, for
 * long blocks, chunked prefill: a prompt chunk that continues cached tokens.
 * Query t of sequence b sits at position i = seq_len[b] + t and attends to
 * the keys its head's rule allows at i: cached ones (a full head every cached
 * row; a ring head its sink slots and the ring slots holding a position
 * j > i - recent, resp. window) and the block's own keys u <= t under the same
 * rule, read from k_new / v_new.  The cache is not modified: append the
 * accepted tokens with duo_kv_append afterwards (rejected draft tokens never
 * reach the ring, which could not take them back; a prompt chunk is appended
 * whole, after this call, before the next chunk).
 * Blocks of up to 8 tokens run as one split kernel over the cache (the
 * block's keys ride on each head's last split) and a merge.  Longer blocks run
 * the prefill kernel twice, over the cached keys and over the block's own
 * keys, and fold the two by their log-sum-exps.
 * q: device bf16 [B][q_len][Hq][D]; k_new, v_new: [B][q_len][Hkv][D];
 * out: [B][q_len][Hq][D]; lse: fp32 [B][q_len][Hq] or NULL.  max_seq_len
 * bounds every seq_len[b] (the cached length, without the block).
 * workspace: >= duo_decode_block_workspace_bytes(params, q_len, max_seq_len)
 * bytes, 256-byte aligned, contents need not be initialised (it holds the
 * split partials, or for long blocks the two halves' outputs, and work-item
 * counters that the call zeroes on the stream; calls that may run at the same
 * time need separate workspaces).  gate: NULL or an output gate (values
 * [B][q_len][Hq][D] or [B][q_len][Hq]).  q_len outside [1, 2^30] is
 * DUO_ERR_UNSUPPORTED; other errors as duo_attn_decode. */
DUO_API int duo_attn_decode_block(const duo_params *params, const duo_cache *cache, const void *q,
                                  const void *k_new, const void *v_new, int32_t q_len,
                                  int32_t max_seq_len, void *out, float *lse, void *workspace,
                                  size_t workspace_bytes, const duo_gate *gate, void *stream);

/* duo_attn_decode without a caller workspace, for callers that cannot
 * allocate device memory at call time (an engine plugin that must not
 * allocate inside its execute hook, a server with a fixed memory budget, a
 * latency-critical loop that cannot afford cudaMalloc's device-wide
 * synchronisation).  The pages have no counterpart: this is an interface
 * convenience, not part of the method.
 * The split partials live in a 16 MiB array inside the library, reserved on
 * every GPU that loads it until the process exits; the call allocates
 * nothing.  The first call on a device looks up that array's address, so make
 * it before any stream capture begins; the address is cached per device and
 * does not survive cudaDeviceReset (do not call this after resetting a device
 * in the same process).  A layer whose
 * duo_decode_workspace_bytes exceeds 16 MiB returns DUO_ERR_WORKSPACE with
 * nothing launched.  All calls on a device share the array: calls whose
 * kernels may overlap on the GPU (different streams or threads) race, so
 * issue them on one stream.  Arguments, outputs and errors otherwise as
 * duo_attn_decode. */
DUO_API int duo_attn_decode_static(const duo_params *params, const duo_cache *cache, const void *q,
                                   int32_t max_seq_len, void *out, float *lse,
                                   const duo_gate *gate, void *stream);

/* KV-cache accounting for one layer (host arithmetic only, no device access).
 * The DuoAttention card (sections Benefits and Changes In This Submission)
 * measures KV-cache size and active KV-cache utilisation of the static Duo
 * cache; this gives those numbers for the layout above:
 *   duo_bytes        = B * (n_full * capacity + n_ring * ring_slots) * D * 2 B * 2 (K and V)
 *   full_cache_bytes = B * num_kv_heads * capacity * D * 2 B * 2 (every head keeps all tokens)
 *   active_bytes     = bytes of duo_bytes that hold a valid token when every sequence
 *                      holds seq_len tokens (full heads: min(seq_len, capacity) rows;
 *                      ring heads: min(seq_len, ring_slots) slots)
 *   utilization      = active_bytes / duo_bytes (0 when duo_bytes is 0)
 * Returns DUO_OK, or DUO_ERR_INVALID_ARG for bad params, capacity < 0,
 * seq_len < 0 or a NULL out. */
typedef struct {
    uint64_t duo_bytes;
    uint64_t full_cache_bytes;
    uint64_t active_bytes;
    double utilization;
} duo_cache_stats;

DUO_API int duo_cache_bytes(const duo_params *params, int64_t capacity, int64_t seq_len,
                            duo_cache_stats *out);

/* Reads and clears the device status word of the current device after
 * synchronising `stream`: DUO_OK, DUO_ERR_TIMEOUT or DUO_ERR_CAPACITY (the
 * first error any kernel recorded since the last read), or DUO_ERR_CUDA. */
DUO_API int duo_get_device_status(void *stream);

/* Short English text for a return or status code (static storage). */
DUO_API const char *duo_status_string(int code);

/* Text of the last host-side error on the calling thread (static storage of
 * that thread; "" if none). */
DUO_API const char *duo_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DUO_ATTN_H */
