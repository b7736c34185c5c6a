/*
 * sepattn.h -- C ABI of the Sep-Attention / SepCache library (B200, sm_100a).
 *
 * Sep-Attention is causal softmax attention in which query i attends to key
 * j only when j <= i and (j < a, or token j is a separator, or i - j < n).
 * Definition: "HKUDS047: SepLLM ..." study, section "SepAttention"
 * (build_prefill_mask: separator columns, initial columns, local triangular
 * window, AND the lower-triangular causal mask) and the jieyibu.net SepLLM
 * explainer, section 1.2 (binary mask M; masked scores are -inf before the
 * softmax).  The four-block KV cache (initial / separator cache capped at s
 * evicting the oldest / past window that keeps only separators when flushed
 * / local window w) follows the xugj520 SepLLM article, section 3.3 table,
 * and the KV-manager steps of the HKUDS047 study, section "KV Cache Manager".
 *
 * Conventions shared by every call:
 *  - All pointers are DEVICE pointers unless a parameter says "host".
 *    All memory is owned by the caller; no call allocates or frees memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *    Calls only enqueue work on it; none synchronises, except
 *    sep_device_status() and sepcache_status(), which say so.
 *  - Return value: SEP_OK (0) or a negative SEP_E* code.  On an error
 *    return nothing was enqueued.
 *  - dtype codes: SEP_F32 (fp32) and SEP_BF16 (bfloat16).
 *  - Layouts are row-major with the last dimension contiguous:
 *      q, out [B, Hq, S, D];  k, v [B, Hkv, S, D];  lse [B, Hq, S] fp32;
 *      is_sep [B, S] uint8 in {0,1};  query head h reads kv head
 *      h / (Hq / Hkv) (contiguous groups).
 *  - a counts the initial tokens kept (positions 0..a-1); n counts the
 *    window including the query itself (keys with 0 <= i - j < n).
 *  - scale <= 0 selects 1/sqrt(D).  lse is the natural log of the softmax
 *    denominator over the scaled scores.
 */
#ifndef SEPATTN_H
#define SEPATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SEP_OK 0
#define SEP_EINVAL (-1)  /* bad size / parameter (also the budget rules below) */
#define SEP_EDTYPE (-2)  /* unsupported dtype or head_dim for this call */
#define SEP_EALIGN (-3)  /* a pointer is not 16-byte aligned */
#define SEP_ECUDA (-4)   /* a CUDA launch or runtime call failed */
#define SEP_EDEVICE (-5) /* a kernel reported an error in a status word */
#define SEP_ENULL (-6)   /* a required pointer is NULL */
#define SEP_ETOOBIG (-7) /* sizes exceed the fixed scratch of sep_attn_decode_noalloc */

#define SEP_F32 0
#define SEP_BF16 1

/* Human-readable name of a status code (static string). */
const char* sep_strerror(int status);

/* Library ABI version (major * 100 + minor). */
int sep_version(void);

/* ---------------------------------------------------------------------- */
/* Separator flags and index lists                                          */
/* ---------------------------------------------------------------------- */

/* is_sep[t] = 1 iff ids[t] is one of sep_ids[0..n_sep_ids) (HKUDS047 study,
 * sections "Separator Tokens" and "SepAttention": token_id in
 * separator_token_ids).  ids: int32 [n_tok]; sep_ids: HOST int32 array,
 * 1 <= n_sep_ids <= 32; is_sep: uint8 [n_tok].  n_tok = 0 is a no-op. */
int sep_flags_from_ids(const int32_t* ids, int64_t n_tok, const int32_t* sep_ids, int n_sep_ids,
                       uint8_t* is_sep, void* stream);

/* Per-sequence prefix-scan compaction of the separator flags (the
 * separator index lists used to gather separator rows).  The flags are the
 * separator columns of the Sep-Attention mask ("HKUDS047: SepLLM ..." study,
 * section "SepAttention": build_prefill_mask marks every column whose token
 * is a separator; jieyibu.net explainer, section 1.2), so these lists name
 * exactly the keys that every later query keeps beyond its window.
 *   prefix [B, S+1]: prefix[b][j] = number of separators among positions < j
 *   idx    [B, S]  : positions of the separators of sequence b in increasing
 *                    order, then -1 up to S
 *   count  [B]     : prefix[b][S]
 * B >= 1, S >= 1.  Results are exact integers. */
int sep_build_index(const uint8_t* is_sep, int B, int S, int32_t* prefix, int32_t* idx,
                    int32_t* count, void* stream);

/* sep_flags_from_ids followed by sep_build_index in one launch: ids int32
 * [B, S] -> is_sep uint8 [B, S] (written), prefix [B, S+1], idx [B, S],
 * count [B], with the same results as the two calls.  sep_ids: HOST int32
 * array, 1 <= n_sep_ids <= 32.  B >= 1, S >= 1. */
int sep_build_index_from_ids(const int32_t* ids, int B, int S, const int32_t* sep_ids,
                             int n_sep_ids, uint8_t* is_sep, int32_t* prefix, int32_t* idx,
                             int32_t* count, void* stream);

/* Kept (query, key) pairs of one head of each sequence (the retention
 * statistics of the HKUDS047 study, section "Forward Input Wrapper").
 * prefix: from sep_build_index; kept_pairs: int64 [B]. a >= 0, n >= 1. */
int sep_count_pairs(const int32_t* prefix, int B, int S, int a, int n, int64_t* kept_pairs,
                    void* stream);

/* ---------------------------------------------------------------------- */
/* Prefill / training forward                                               */
/* ---------------------------------------------------------------------- */

/* Workspace bytes sep_attn_prefill needs for these sizes (bf16: 256 bytes
 * of head, which hold the attention kernel's work-item counter, then room
 * for the compacted initial+separator K and V rows of every (b, kv head),
 * i.e. two buffers of k's size; fp32: 256 bytes). */
size_t sep_attn_prefill_workspace(int B, int Hq, int Hkv, int S, int D, int dtype);

/* Sep-Attention over whole sequences ("HKUDS047: SepLLM ..." study, section
 * "SepAttention": build_prefill_mask = (separator columns | initial columns |
 * local triangular window) AND the causal lower triangle; jieyibu.net
 * explainer, section 1.2: scores outside the mask are -inf before the
 * softmax):
 *   out[b,h,i,:] = sum_{j in K_i} softmax_j(scale * q_i . k_j) v_j,
 *   K_i = { j <= i : j < a or is_sep[b,j] or i - j < n },
 *   lse[b,h,i]  = ln sum_{j in K_i} exp(scale * q_i . k_j).
 * q, k, v, out: dtype elements in the layouts above; lse: fp32 (may be NULL).
 * is_sep, prefix, idx: the flags and their sep_build_index results.
 * dtype SEP_BF16 requires D in {64, 128} and runs on tcgen05 tensor cores
 * (fp32 accumulation); dtype SEP_F32 requires D in {32, 64, 128} and runs
 * in exact fp32 FMA arithmetic.  Constraints: B, Hq, Hkv, S >= 1,
 * Hq % Hkv == 0, a >= 0, n >= 1; pointers 16-byte aligned; workspace of at
 * least sep_attn_prefill_workspace() bytes, 256-byte aligned, contents
 * arbitrary.  Calls that share a workspace must not overlap on the GPU. */
int sep_attn_prefill(const void* q, const void* k, const void* v, int dtype, const uint8_t* is_sep,
                     const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S, int D,
                     int a, int n, float scale, void* out, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream);

/* Sep-Attention backward (the training use of the sparse attention:
 * "HKUDS047: SepLLM ..." study, section on the three versions,
 * Training-SepLLM).  Gradients of sum(out * dout) with respect to q, k, v
 * through sep_attn_prefill's attention (same kept set, scale and query-head
 * grouping): per kept pair (i, j), with p_ij the forward probability rebuilt
 * from lse and delta_i = dout_i . out_i,
 *   dv_j += p_ij dout_i,  ds_ij = p_ij (dout_i . v_j - delta_i),
 *   dk_j += scale ds_ij q_i,  dq_i += scale ds_ij k_j
 * (dk, dv summed over the query heads of each kv head).
 * q, out, dout, dq: [B, Hq, S, D]; k, v, dk, dv: [B, Hkv, S, D]; lse
 * [B, Hq, S] fp32 from sep_attn_prefill; is_sep, prefix, idx as for the
 * prefill.  dtype SEP_BF16 only (fp32 accumulation; SEP_EDTYPE otherwise),
 * D in {64, 128}.  workspace: sep_attn_backward_workspace() bytes, 256-byte
 * aligned, contents arbitrary (the call clears what it needs); calls sharing
 * it must not overlap on the GPU.  Every output element is written.  The
 * call's five kernels overlap one another's set-up on the stream
 * (programmatic launches), but its first launch starts only after earlier
 * work on `stream` has completed, and its last one ends only after all of
 * the call's work, so stream order holds as for any call. */
size_t sep_attn_backward_workspace(int B, int Hq, int Hkv, int S, int D);
int sep_attn_backward(const void* q, const void* k, const void* v, const void* out,
                      const float* lse, const void* dout, int dtype, const uint8_t* is_sep,
                      const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S,
                      int D, int a, int n, float scale, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Streaming decode over the four-block SepCache                            */
/* ---------------------------------------------------------------------- */

/* Block sizes: a initial tokens, s separator-cache entries, `past` past-
 * window entries, w local-window entries; capacity c = a + s + past + w
 * (the KV-manager budget rules of the HKUDS047 study, section "Streaming
 * parameter constraints": init >= 0, local > 0; SepLLM needs s > 0, and s =
 * 0 with past = 0 is the StreamingLLM special case). */
typedef struct {
  int32_t a, s, past, w;
  int32_t mode; /* 0, or a sum of the SEP_CACHE_* variant bits below */
} sep_cache_cfg;

/* Variants of the KV manager's compression step ("HKUDS047: SepLLM ..."
 * study, section "KV Cache Manager": the SEP_ACCUMULATION and
 * USE_MAX_SEP_CACHE switches, and compression once the sequence exceeds
 * cache_size).  Mode 0 is the default: separators accumulate, the separator
 * cache keeps its newest s, and the past window is flushed when it holds
 * more than `past` tokens. */
#define SEP_CACHE_NO_ACCUMULATION 1 /* a flush keeps only the flushed past window's
                                       separators (newest s); the old ones are dropped */
#define SEP_CACHE_UNBOUNDED_SEPS 2  /* separators are never evicted: s is the block's
                                       capacity, and a flush that needs more sets
                                       SEP_CACHE_ESEPS in the status word (the newest s
                                       stay).  The page's list without a maximum simply
                                       grows; a device cache has a fixed capacity, so a
                                       caller gets those semantics by sizing s for the
                                       whole stream (at least its separator count), and
                                       this bit then only reports a cache sized too
                                       small */
#define SEP_CACHE_TOTAL_TRIGGER 4   /* flush when the whole cache holds more than
                                       a+s+past+w tokens (the past window may then hold
                                       up to past+s); the same as the default once the
                                       separator cache is full */

/* Cache state.  Every pointer is device memory inside one caller-owned
 * buffer laid out by sepcache_carve().  Rows of each (layer, b, kv head)
 * are stored in increasing position order: initial | separator | past |
 * local, cap = c + 1 rows (one spare row holds the newest token between
 * sepcache_append and sepcache_compact).  A flush compacts the surviving
 * rows in place (each moves to a row at or below its own, in order). */
typedef struct {
  void* k;           /* [layers][B][Hkv][cap][D] dtype */
  void* v;           /* [layers][B][Hkv][cap][D] dtype */
  int32_t* pos;      /* [B][cap]  token position of each row, -1 when empty */
  uint8_t* flag;     /* [B][cap]  separator flag of each row */
  int32_t* counts;   /* [B][4]    rows in blocks I, S, P, L */
  int32_t* plan;     /* [B][cap+8] this step's slot / flush / buffers / move list */
  int64_t* step;     /* [B]       tokens appended so far */
  int32_t* status;   /* [1]       0, or SEP_CACHE_E* bits set by a kernel */
  float* rope;       /* [rope_rows][D/2][2] cos, sin of slot r at frequency i (fp32) */
  int32_t layers, B, Hkv, D, dtype, cap;
  sep_cache_cfg cfg;
  float rope_theta;  /* 0: keys are stored encoded; > 0: see sepcache_set_rope */
  int32_t rope_rows; /* max(cap, 65) */
} sepcache;

#define SEP_CACHE_EOVERFLOW 1 /* a step found more rows than the capacity */
#define SEP_CACHE_ESTATE 2    /* corrupt block counts */
#define SEP_CACHE_ESEPS 4     /* SEP_CACHE_UNBOUNDED_SEPS: more separators than s rows */

/* Bytes of the single buffer holding a cache (256-byte aligned pieces). */
size_t sepcache_bytes(sep_cache_cfg cfg, int layers, int B, int Hkv, int D, int dtype);

/* Fill *cache with pointers into `buffer` (device, >= sepcache_bytes(),
 * 256-byte aligned) and the sizes.  Host-only; enqueues nothing.
 * Validation: a >= 0, s >= 0, past >= 0, w >= 1, mode bits in 0..7, D in {64, 128},
 * dtype in {SEP_F32, SEP_BF16}, layers, B, Hkv >= 1. */
int sepcache_carve(sepcache* cache, void* buffer, size_t bytes, sep_cache_cfg cfg, int layers,
                   int B, int Hkv, int D, int dtype);

/* Positional-encoding shifting for streaming (HKUDS047 study, section on
 * the three versions: the streaming setting needs positional-encoding
 * shifting; section "Streaming-SepLLM": the Llama positional-encoding-
 * shifting module).  With theta > 0 the cache holds keys BEFORE their
 * rotary encoding, and every decode call (sep_attn_decode, _noalloc, _step)
 * encodes each retained key at its slot r inside the cache (0 .. len-1, the
 * order I | S | P | L) and the query at len-1, the newest token's slot:
 * for i < D/2 the pair (x_i, x_{i+D/2}) turns by r * theta^(-2i/D)
 * (rotate-half form, as in Llama models; Llama-3 uses theta = 500000).  So
 * positions never exceed the capacity however long the stream runs.  Keys
 * passed to sepcache_append / _ingest / _decode_step and q passed to the
 * decode calls must then be un-encoded; values are never encoded.  Fills the
 * cache's cos / sin table (fp32, rounded from fp64) on `stream` and records
 * theta in *cache.  theta = 0 switches the shifting off (keys stored already
 * encoded, the default after sepcache_carve).  Errors: SEP_EINVAL for theta
 * < 0, not finite, or in (0, 1]. */
int sepcache_set_rope(sepcache* cache, float theta, void* stream);

/* Reset to the empty state (no tokens; status 0). */
int sepcache_init(const sepcache* cache, void* stream);

/* Append one token to every sequence at `layer`: k_new, v_new [B, Hkv, D].
 * At layer 0 this also advances the shared block bookkeeping by one token
 * using is_sep_new [B] (uint8): the token joins the initial block while it
 * holds fewer than a tokens, else the local window, whose oldest token
 * moves to the past window when it holds more than w; when the past window
 * then holds more than `past` tokens this step is a flush step (xugj520
 * article, section 3.3).  is_sep_new is ignored at layers > 0.  Per step:
 * append(layer 0) must come first, then for every layer append -> compact
 * -> decode; the next step starts after all layers have been compacted. */
int sepcache_append(const sepcache* cache, int layer, const void* k_new, const void* v_new,
                    const uint8_t* is_sep_new, void* stream);

/* Apply this step's flush to `layer` ("HKUDS047: SepLLM ..." study, section
 * "KV Cache Manager": the compression step; xugj520 article, section 3.3
 * table: the past window keeps only its separators, which join the
 * separator cache, and that cache evicts its oldest entries beyond s): the
 * separators of the past window join the separator cache, which keeps its
 * newest s entries, the past window empties and the local window slides
 * down.  The surviving rows (found by an
 * order-preserving warp-ballot stream compaction at layer 0's append) move
 * in place, in ascending order, each to a row at or below its own.  A no-op
 * on steps without a flush. */
int sepcache_compact(const sepcache* cache, int layer, void* stream);

/* Prompt ingestion (bulk append): put the T tokens of a prompt into an EMPTY
 * cache in one call per layer, with the same result as T calls of
 * sepcache_append (and sepcache_compact) -- the prefill of the prompt then
 * hands over to streaming decode (the study's prefill / decode split; the
 * cache's block rules as in sepcache_append, xugj520 article section 3.3).
 * k, v: the prompt's keys and values [B, Hkv, T, D] in the cache dtype (the
 * layout sep_attn_prefill reads); is_sep [B, T], prefix [B, T+1] and idx
 * [B, T] from sep_build_index of the prompt, read at layer 0, which also
 * writes the block bookkeeping (step becomes T).  Layers 0..layers-1 in
 * order.  A sequence whose cache is not empty is left unchanged and the
 * cache status word gets SEP_CACHE_ESTATE.  Errors: SEP_EINVAL (T < 1, bad
 * layer or cache), SEP_ENULL, SEP_EALIGN (k, v not 16-byte aligned). */
int sepcache_ingest(const sepcache* cache, int layer, const void* k, const void* v,
                    const uint8_t* is_sep, const int32_t* prefix, const int32_t* idx, int T,
                    void* stream);

/* One whole decode step of `layer` in a single launch per layer (plus, at
 * layer 0, the bookkeeping launch): the same result as sepcache_append(layer,
 * k_new, v_new, is_sep_new) -> sepcache_compact(layer) -> sep_attn_decode(
 * layer, q, ...).  Each decode CTA writes the new token's row; on a flush
 * step the CTAs of a (sequence, kv head) load the surviving rows from their
 * old places and compact them in place (the first CTA of the pair while it
 * loads its share, the second, whose destinations may be the first one's
 * sources, once the first has loaded everything).  Same arguments as those
 * calls; is_sep_new is read at layer 0 only.  Layers are stepped in order
 * 0..layers-1 each token. */
int sep_attn_decode_step(const sepcache* cache, int layer, const void* q, const void* k_new,
                         const void* v_new, const uint8_t* is_sep_new, int Hq, float scale,
                         void* out, float* lse, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Workspace bytes sep_attn_decode needs (split-K partials and counters). */
size_t sep_attn_decode_workspace(const sepcache* cache, int Hq);

/* Attention of the newest token over the retained rows of `layer` (the
 * streaming decode over the four cache blocks: xugj520 article, section 3.3
 * table; jieyibu.net explainer, section 1.3: the query attends over the
 * initial, separator, past-window and local-window rows only; the softmax is
 * that of sep_attn_prefill restricted to those rows):
 * q [B, Hq, D] (cache dtype), out [B, Hq, D] (cache dtype), lse [B, Hq]
 * fp32 (may be NULL).  Hq % Hkv == 0 and Hq / Hkv <= 8.  workspace: at least
 * sep_attn_decode_workspace() bytes, zero-filled before its first use (the
 * kernel leaves its counters at zero); calls sharing a workspace must not
 * overlap on the GPU. */
int sep_attn_decode(const sepcache* cache, int layer, const void* q, int Hq, float scale, void* out,
                    float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Decode for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a library convenience.  Some callers cannot pass a
 * workspace -- a plug-in that a host framework calls with only the tensors
 * of the call (the framework owns every device allocation), or a serving
 * loop whose device memory is fully reserved for its KV pool, where a new
 * cudaMalloc would fail or stall the device.  Same arguments and result as
 * sep_attn_decode, without the workspace: the split-K partials and tickets
 * live in a fixed scratch array inside the library (about 4.1 MiB, held by
 * every GPU that loads the library until the process exits).
 * Only an fp32 cache with more than 8 splits of 64 rows (a+s+past+w+1 >
 * 512) merges its splits through that array; bf16 caches and smaller fp32
 * caches merge inside a thread-block cluster and do not use it.  For the
 * fp32 case the limits are B * Hq * ceil((a+s+past+w+1) / 64) <= 8192 and
 * B * Hkv <= 4096; larger sizes return SEP_ETOOBIG before anything is
 * enqueued.  In that case the first call on a device looks up the array's
 * device address (with that device current); make that first call before
 * any stream capture, and do not use this entry point on a device after
 * cudaDeviceReset.  Each such call clears the tickets on `stream` before
 * its kernel.  No call allocates.  All calls share the array, so calls that
 * overlap on the GPU (other streams, other threads) race on it. */
int sep_attn_decode_noalloc(const sepcache* cache, int layer, const void* q, int Hq, float scale,
                            void* out, float* lse, void* stream);

/* Mask-based generation: the decode of the generate mask ("HKUDS047:
 * SepLLM ..." study, section "SepAttention": build_generate_mask applies the
 * prefill mask's rule to a query of length 1), over a full KV history with
 * no row evicted.  The newest token of each sequence, at position T - 1,
 * attends over k, v [B, Hkv, S, D] (rows 0 .. T-1 hold the history) with
 * the kept set of its row
 *   { j <= T-1 : j < a  or  is_sep[j]  or  T-1-j < n },
 * read as the initial rows [0, min(a, lo)), the separators in
 * [min(a, lo), lo) taken from idx, and the window [lo, T), lo = max(0, T-n).
 * q [B, Hq, D] and out [B, Hq, D] in dtype; lse [B, Hq] fp32 (may be NULL).
 * prefix [B, S+1], idx [B, S]: sep_build_index of the flags [B, S] (flags at
 * positions >= T are never used).  scale <= 0 means 1/sqrt(D).  Same query
 * head grouping and limits as sep_attn_decode (Hq/Hkv in {1, 2, 4, 8}),
 * D in {64, 128}, 1 <= T <= S, a >= 0, n >= 1.  bf16 runs on warp-level
 * tensor cores with the rows gathered by 16-byte asynchronous copies (no
 * workspace: may be NULL); fp32 runs the exact FMA kernel and needs
 * sep_attn_decode_masked_workspace() bytes, zero-filled before first use,
 * 16-byte aligned; calls sharing it must not overlap on the GPU. */
size_t sep_attn_decode_masked_workspace(int B, int Hq, int Hkv, int S, int D);
int sep_attn_decode_masked(const void* q, const void* k, const void* v, int dtype,
                           const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv,
                           int S, int T, int D, int a, int n, float scale, void* out, float* lse,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, copy the cache status word to *host_status (host)
 * and return SEP_EDEVICE if it is nonzero, SEP_OK otherwise. */
int sepcache_status(const sepcache* cache, int32_t* host_status, void* stream);

/* Synchronise `stream` and report the library's device-side error bits
 * (a bounded wait inside a kernel that timed out sets them); clear them when
 * `clear` is nonzero.  Returns SEP_EDEVICE when any bit was set. */
int sep_device_status(int32_t* host_bits, int clear, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SEPATTN_H */
