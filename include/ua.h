/*
 * ua.h -- C ABI of libua, the B200 (sm_100a) Universal Attention hot path.
 *
 * Universal Attention (UA) is causal RoPE softmax attention whose logits carry an
 * additive, content-aware decay bias Lambda, plus the inference-time self-pruning of
 * the KV cache that Lambda drives.  Sources: "A Self-Pruning Transformer: Extreme
 * KV-Cache Compression with Universal Attention" -- paperlayer.ai summary (§3 causal
 * softmax attention and the FoX additive forget gate; §4 and §4.1 the three decay
 * mechanisms and their geometric mean; §4.2 threshold-p eviction and the training
 * kernels; App. C decay applied inside a fused online softmax; App. H the missing
 * fused dynamic cache manager) and the ai4snews synopsis of the same paper (Fig. 1
 * caption: L2-normalised keys, sigmoid output gate, geometric mean -> log space ->
 * causal accumulation; the veto property; the eviction paragraph).
 *
 * The pages fix the structure, not the formulas.  This library computes, per KV head:
 *   khat_j     = k_j / max(||k_j||, 1e-12)                   (keys L2-normalised)
 *   r_q(l)     = softplus(a_q[l])      query-aware rate
 *   r_k(j)     = softplus(a_k[j])      key-aware rate
 *   r_sim(l,j) = softplus(alpha * <khat_l, khat_j> + beta)   similarity rate (pre-RoPE keys)
 *   D[l,j]     = (r_q(l) r_k(j) r_sim(l,j))^(1/3)            geometric mean (veto: any 0 -> 0)
 *   Lambda_ij  = -sum_{l=j+1..i} D[l,j]                      (Lambda_ii = 0, never positive)
 *   O_i        = softmax_{j<=i}(scale * RoPE(q_i).RoPE(khat_j) + Lambda_ij) V  (.) sigmoid(G_i)
 * RoPE pairs element m with m + d/2 ("rotate half"), frequency theta^(-2m/d), position =
 * token index.  Query head h uses KV head h / (H/Hkv); a_q, a_k, alpha and beta belong
 * to the KV head, so the G query heads of a group share one Lambda.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers to caller-owned memory; the library never
 *     allocates or frees, and launches asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Nothing synchronises except ua_get_device_status.
 *   - Tensors are dense, row-major, innermost dimension last, with the shapes written
 *     beside each argument.  "act" means the activation dtype of the call: float32 for
 *     UA_F32, bfloat16 for UA_BF16.  Decay logits and parameters are always float32.
 *   - Every pointer must be 16-byte aligned (256-byte for the workspace) and address at
 *     least the elements its shape implies: the library cannot see a buffer's extent, so an
 *     undersized one is read or written past its end (the Python binding checks extents and
 *     element types before calling).
 *   - Host-detectable errors (NULL pointer, bad shape, unsupported head_dim, misaligned
 *     pointer, workspace too small) return a status before anything is launched and leave
 *     all outputs untouched.  Device-detectable errors (cache capacity exceeded) set a
 *     device status word read back by ua_get_device_status; the affected outputs are then
 *     unspecified.  No kernel traps.
 */
#ifndef UA_H_
#define UA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UA_OK = 0,
    UA_ERR_INVALID_ARG = 1,   /* NULL pointer, non-positive size, H % Hkv != 0, ... */
    UA_ERR_UNSUPPORTED = 2,   /* head_dim / group size / dtype outside what is compiled */
    UA_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte (workspace: 256-byte) aligned */
    UA_ERR_WORKSPACE = 4,     /* workspace smaller than the size query returned */
    UA_ERR_CAPACITY = 5,      /* a cache would exceed its capacity (device status bit) */
    UA_ERR_CUDA = 6,          /* a CUDA runtime call failed (launch error, ...) */
    UA_ERR_TIMEOUT = 7,       /* a bounded device-side wait gave up (device status bit) */
    UA_ERR_RANGE = 8          /* reserved: a softmax row normaliser out of range (no path
                                 raises it; the tensor-core forward recomputes such rows) */
} ua_status;

typedef enum { UA_F32 = 0, UA_BF16 = 1 } ua_dtype;

/* Variant bits: the ablations of "A Self-Pruning Transformer: Extreme KV-Cache Compression
 * with Universal Attention" (paperlayer.ai summary, §5.4 with Table 3 and App. E with
 * Table 6; ai4snews synopsis, interpretation paragraph).  0 is the method itself.
 *   UA_VAR_NO_QUERY_DECAY / UA_VAR_NO_KEY_DECAY / UA_VAR_NO_SIM_DECAY switch one decay
 *     mechanism off; the decay rate is then the geometric mean of the rates left on,
 *     D = (product of the n active rates)^(1/n).  Switching all three off is
 *     UA_ERR_INVALID_ARG.
 *   UA_VAR_QUERY_NORM RMS-normalises every query head before RoPE (Qwen3-style query norm
 *     with unit gain): q' = q / sqrt(mean(q^2) + 1e-6).  Keys keep their L2 normalisation.
 *   UA_VAR_PER_HEAD_DECAY (prefill calls only) gives every query head its own decay: a_q, a_k
 *     are [B,T,H], alpha, beta [H], and b_final / lambda_dbg have H heads ([B,H,T] / [B,H,T,T]).
 *     The pages decide retention "head by head" (summary §4.2) without saying whether a head is
 *     a query or a KV head; with per-query-head rates, query head h is exactly multi-head UA over
 *     its group's shared keys and values, so the library repeats each KV head's keys and values
 *     for the G heads of its group (inside the workspace), runs the per-KV-head path with one
 *     decay unit per query head (G times the decay work), and sums dk, dv over the copies.  The
 *     matching decode uses a cache of H heads filled from the repeated keys and values (each
 *     query head evicts on its own bias); ua_decode_step takes no per-head bit.
 * Any other bit is UA_ERR_INVALID_ARG. */
#define UA_VAR_NO_QUERY_DECAY 1
#define UA_VAR_NO_KEY_DECAY 2
#define UA_VAR_NO_SIM_DECAY 4
#define UA_VAR_QUERY_NORM 8
#define UA_VAR_PER_HEAD_DECAY 16

/* Decode-step flag: defer compaction (see ua_decode_step). */
#define UA_DECODE_DEFER_COMPACT 256

/* Problem shape of a prefill call.  d (head_dim) must be 64 or 128; H % Hkv == 0 and
 * H / Hkv in {1, 2, 3, 4, 8}; T >= 1. */
typedef struct {
    int B, T, H, Hkv, d;
    float scale;          /* logit scale, usually 1/sqrt(d); multiplies only QK^T */
    double rope_theta;    /* RoPE base, e.g. 500000 */
    ua_dtype dtype;       /* activation dtype of q, k, v, g, o (and gradients) */
    int variant;          /* UA_VAR_* bits, 0 = Universal Attention as published */
    float prune_p;        /* chunked pruned prefill threshold p in [0, 1]; 0 = dense prefill
                             (see ua_prefill_fwd); must be 0 for the backward */
} ua_shape;

/* ------------------------------------------------------------------ prefill forward
 * Decay construction (§4, §4.1, Fig. 1) and biased causal attention with the decay
 * applied inside the online softmax (App. C).  Lambda is never written to HBM except
 * through the optional debug output.
 *
 * ua_prefill_workspace_size: bytes of device scratch ua_prefill_fwd needs for `shape`
 * (rotated queries and keys, rates and the per-query-tile column prefixes of the decay).
 */
ua_status ua_prefill_workspace_size(const ua_shape* shape, size_t* bytes);

/* q, g: [B,T,H,d] act;  k, v: [B,T,Hkv,d] act;  a_q, a_k: [B,T,Hkv] f32;
 * alpha, beta: [Hkv] f32.
 * Outputs: o [B,T,H,d] act (required);
 *          lse [B,H,T] f32 natural-log row normaliser of the biased logits (or NULL);
 *          b_final [B,Hkv,T] f32 = Lambda_{T-1,j}, the initial per-pair cache bias (or NULL);
 *          lambda_dbg [B,Hkv,T,T] f32 full Lambda, zero above the diagonal (or NULL;
 *          allowed only for T <= 1024).
 * ws / ws_bytes: device workspace of at least ua_prefill_workspace_size bytes; its
 * contents are scratch (overwritten).
 *
 * Paths: bf16 problems with d = 64 or 128 and H/Hkv <= 4 run on the tensor cores (tcgen05/
 * TMEM/TMA).  That path shifts every softmax row by the a-priori bound scale*||q_i|| (the keys
 * are unit vectors and Lambda <= 0, so no logit exceeds it; one shift per 16-row quarter and
 * KV group) instead of a running maximum.  A row whose true maximum lies far below that shift
 * (large query norms: only possible when scale*||q|| exceeds ~20) shows it in its shifted row
 * sum; every row whose sum falls below 2^-60 is listed and recomputed exactly afterwards, with a
 * running maximum, from the same bf16 operands (k_fwd_fix: about T x 128 decay evaluations per
 * listed row, plus, when b_final is not requested, one exact column sweep of the row's (batch,
 * KV head)).  UA_ERR_RANGE is therefore never raised by this path.  The same path skips
 * the softmax and PV work of every 128 x 128 (query tile, key tile) whose decay prefix
 * makes all its probabilities underflow to exactly 0 in fp32 (Lambda only decreases down a
 * key column, so the prefix above the tile bounds the whole tile).  When b_final is requested
 * the decay of such a tile is still evaluated (b_final stays exact); when b_final is NULL the
 * tile is skipped entirely.  Either way every requested output is identical to the unskipped
 * computation (see ua_prefill_tile_stats).  The tensor-core path computes the
 * three-rate geometric mean only; it takes UA_VAR_QUERY_NORM, but a shape with a decay
 * mechanism switched off runs the SIMT path.  All other problems, and every call that asks
 * for lambda_dbg, run the fp32 SIMT path, which uses a running maximum.
 *
 * Chunked pruned prefill (shape->prune_p = p > 0; paperlayer.ai summary §5: prefill pruning
 * proceeds in chunks of 128 tokens): before the chunk that starts at token c (c a multiple of
 * 128), every pair j < c whose bias Lambda_{c-1,j} is below log p is evicted, and the rows of
 * that chunk and of every later one attend over the surviving pairs and their own chunk only
 * (the biases themselves are unchanged).  b_final and lambda_dbg are the same as for the dense
 * prefill, so filling a cache with b_final and compacting it at p keeps exactly the pairs that
 * survive the last chunk; o and lse change.  Key tiles evicted as a whole are skipped. */
ua_status ua_prefill_fwd(const ua_shape* shape, const void* q, const void* k, const void* v,
                         const void* g, const float* a_q, const float* a_k, const float* alpha,
                         const float* beta, void* o, float* lse, float* b_final, float* lambda_dbg,
                         void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ allocation-free forward
 * No counterpart on the pages: this is a deployment convenience of this library.
 * Same computation and arguments as ua_prefill_fwd, minus lambda_dbg and the workspace.
 * For callers that cannot allocate device memory (a plug-in inside a host application that
 * owns the whole GPU memory pool, or a caller that cannot afford cudaMalloc's latency and
 * synchronisation): the scratch lives in a fixed 32 MiB array inside the library, which
 * every device that loads the library keeps until the process exits.
 *   - Problems whose ua_prefill_workspace_size exceeds ua_prefill_noalloc_max_scratch()
 *     (32 MiB; e.g. one 4096-token sequence of the 1B shape fits) return UA_ERR_WORKSPACE.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (different streams,
 *     without ordering between them) race on it and give undefined results.  Serialise them.
 *   - Nothing is allocated or freed; no state carries over between calls (every byte of the
 *     scratch a call reads was written earlier in the same call). */
ua_status ua_prefill_fwd_noalloc(const ua_shape* shape, const void* q, const void* k, const void* v,
                                 const void* g, const float* a_q, const float* a_k, const float* alpha,
                                 const float* beta, void* o, float* lse, float* b_final, void* stream);

/* Size in bytes of the array ua_prefill_fwd_noalloc uses (the largest workspace it serves). */
size_t ua_prefill_noalloc_max_scratch(void);

/* ------------------------------------------------------------------ prefill tile statistics
 * No counterpart on the pages: a measurement aid for the tile skipping described at
 * ua_prefill_fwd.  Synchronises `stream` and reports, for the most recent ua_prefill_fwd
 * (without lambda_dbg) that used workspace `ws` for `shape`, the number of causal
 * 128 x 128 tiles, B*Hkv*n*(n+1)/2 with n = ceil(T/128), in *tiles, and how many of them
 * skipped the softmax in *skipped.  Problems that run the fp32 SIMT path report
 * *skipped = 0.  Not available for the allocation-free entry point. */
ua_status ua_prefill_tile_stats(const ua_shape* shape, const void* ws, size_t ws_bytes,
                                unsigned long long* tiles, unsigned long long* skipped, void* stream);

/* Likewise for the exact row recomputation described at ua_prefill_fwd: synchronises `stream`
 * and reports in *rows how many (row, query head) pairs the most recent tensor-core
 * ua_prefill_fwd that used `ws` for `shape` listed as out of its softmax shift's range and
 * recomputed.  0 for problems that run the fp32 SIMT path. */
ua_status ua_prefill_fixed_rows(const ua_shape* shape, const void* ws, size_t ws_bytes,
                                unsigned long long* rows, void* stream);

/* ------------------------------------------------------------------ prefill backward
 * Gradient of sum(dO * O) with respect to every input of ua_prefill_fwd (the backward of
 * the custom training kernels, §4.2 and App. H; the decay is recomputed, not stored,
 * App. C).  Needs the forward's o and lse (natural-log row normalisers); b_final may be NULL
 * and is not read (the decay prefixes are recomputed).  d_o: [B,T,H,d] act.
 * Outputs: dq, dg [B,T,H,d] act; dk, dv [B,T,Hkv,d] act; da_q, da_k [B,T,Hkv] f32;
 * dalpha, dbeta [Hkv] f32 (summed over the batch).  All outputs are overwritten; the result
 * is deterministic (no atomics).  bf16 problems with d = 64 (H/Hkv <= 4) or d = 128
 * (H/Hkv <= 3) of the three-rate method (the query norm allowed) run on the tensor cores: the
 * decay prefixes above every 32-row step, a key-major pass that accumulates dv and the rotated
 * key gradient in TMEM and stores the bf16 dZ / dX tiles of the causal band, and tensor-core
 * GEMMs for the query and similarity gradients (the workspace holds the band: about
 * (G+1) * 2 bytes per causal pair and KV head).  Similarities are formed from the same bf16 unit
 * keys as the tensor-core forward (whose row normalisers the probabilities are divided by).  The
 * band below each 128-key tile's last 32-row step whose probabilities can be nonzero is skipped
 * exactly: Lambda only decreases down a key's column, so once s|q|(1 + 2^-6) - lse - Pb falls
 * below -88 (the exp2 then flushes to 0) for every row of a step and every step below, its dZ,
 * dLambda and dX contributions are exact zeros (the workspace still holds the whole band).  Other
 * problems run as fp32 SIMT kernels.
 * Training is dense: a shape with prune_p != 0 is UA_ERR_INVALID_ARG. */
ua_status ua_prefill_bwd_workspace_size(const ua_shape* shape, size_t* bytes);

ua_status ua_prefill_bwd(const ua_shape* shape, const void* q, const void* k, const void* v,
                         const void* g, const float* a_q, const float* a_k, const float* alpha,
                         const float* beta, const void* o, const float* lse, const float* b_final,
                         const void* d_o, void* dq, void* dk, void* dv, void* dg, float* da_q,
                         float* da_k, float* dalpha, float* dbeta, void* ws, size_t ws_bytes,
                         void* stream);

/* No counterpart on the pages: a measurement aid for the exact underflow skipping described at
 * ua_prefill_bwd.  Synchronises `stream` and reports, for the most recent ua_prefill_bwd that
 * used workspace `ws` for `shape`, the 32-row steps of the causal band (per KV head and batch:
 * key tile kt meets steps 4kt .. 4*ceil(T/128)-1) in *steps, and how many of them the key-major
 * pass walked in *walked (the rest hold no nonzero probability).  Problems that run the fp32
 * SIMT backward report *walked = *steps.  prune_p != 0 is UA_ERR_INVALID_ARG. */
ua_status ua_prefill_bwd_band_stats(const ua_shape* shape, const void* ws, size_t ws_bytes,
                                    unsigned long long* steps, unsigned long long* walked, void* stream);

/* ------------------------------------------------------------------ self-pruning cache
 * One cache per (batch, KV head), structure of arrays, `capacity` slots each; slot s of
 * (b, h) lives at index (b*Hkv + h)*capacity + s.  Slots [0, n_kept[b,h]) are live, in
 * ascending token order.  The cache element type follows `dtype` (f32 or bf16).
 *   khat  [B,Hkv,cap,d]  normalised key (pre-RoPE), pair-interleaved: element 2m holds
 *                        component m and element 2m+1 component m + d/2 (the two components
 *                        one RoPE frequency rotates together).  The similarity rate uses it as
 *                        is; the attention logit rotates it by the slot's pos on the fly, so
 *                        no rotated copy is stored (2*d*elt + 12 bytes per slot)
 *   v     [B,Hkv,cap,d]  value
 *   bias  [B,Hkv,cap]    f32 running log-bias b_j (= Lambda_{t,j} at the current row t)
 *   rk    [B,Hkv,cap]    f32 key-aware rate softplus(a_k[j])
 *   pos   [B,Hkv,cap]    int32 token position
 *   n_kept [B,Hkv]       int32 live slot count
 * The pages keep a scalar bias per cached pair and evict a pair once exp(b_j) < p; b_j
 * only decreases, so an evicted pair never returns (§4.2; ai4snews eviction paragraph). */
typedef struct {
    int B, Hkv, d, capacity;
    ua_dtype dtype;
    int kv_rep;           /* cache heads per KV head of the keys and values the cache is filled and
                             stepped with: k, v of ua_cache_fill and the decode steps have Hkv / kv_rep
                             heads, cache head h reading head h / kv_rep.  0 or 1: one each.  With
                             per-query-head decay (UA_VAR_PER_HEAD_DECAY) the cache keeps one head per
                             query head (Hkv = H, kv_rep = G), each with its own biases and evictions */
    void* khat;
    void* v;
    float* bias;
    float* rk;
    int32_t* pos;
    int32_t* n_kept;
    /* Paged storage (optional; page_table == NULL: one contiguous region of `capacity` slots per
     * cache, as above).  Otherwise khat, v, bias, rk and pos are a pool of pool_pages pages of
     * page_size slots each (khat, v [pool_pages*page_size, d]; the others [pool_pages*page_size]),
     * and slot s of cache u = b*Hkv + h lives in page page_table[u*max_pages + s/page_size] at
     * offset s % page_size.  page_size: a power of two, 128 <= page_size <= 2^20;
     * capacity == max_pages*page_size; pool_pages*page_size < 2^31.  The caller owns the table:
     * before a call, every slot the call may touch (slots [0, n_kept) and, for a decode step, the
     * append slot n_kept) must lie in a page with an id in [0, pool_pages); the kernels check every
     * id they use and, on one outside that range, raise UA_ERR_INVALID_ARG in the device status
     * and skip the access (the call's outputs are then unspecified).  After a compaction, the pages
     * past ceil(n_kept/page_size) hold no live pair and may be handed to other caches.  This is
     * the pages' missing dynamic cache manager (summary App. H) in its plainest form: a pruned
     * cache occupies pages for its live pairs only, not a reserved region of its longest length. */
    int page_size, max_pages, pool_pages;
    const int32_t* page_table;
} ua_cache;

/* Load a prefill into the cache: slot t <- token t for t < T (khat, v from k and v; bias =
 * b_final; rk = softplus(a_k); pos = t) and n_kept = T.  Requires T <= capacity.
 * k, v: [B,T,Hkv/kv_rep,d] act; a_k [B,T,Hkv] f32; b_final [B,Hkv,T] f32. */
ua_status ua_cache_fill(const ua_cache* cache, int T, const void* k, const void* v,
                        const float* a_k, const float* b_final, double rope_theta, void* stream);

/* Stable in-place compaction of every (b, KV head) cache.  A slot survives when
 * keep[b,h,s] != 0 (keep: [B,Hkv,cap] uint8) or, with keep == NULL, when bias >= log p.
 * Survivors keep their relative order.  kept_idx (optional, [B,Hkv,cap] int32) receives
 * the old slot of each survivor in its new order; entries past the new n_kept are left
 * untouched. */
ua_status ua_cache_compact(const ua_cache* cache, const uint8_t* keep, float p,
                           int32_t* kept_idx, void* stream);

/* One decode step for all B sequences, the new token sitting at position pos_t:
 *   1. each live pair j takes the new row's decay, b_j -= D[t,j];
 *   2. it is evicted when b_j < log p (exp(b_j) < p); p = 0 evicts nothing;
 *   3. the H query heads attend over the survivors plus the new token (bias 0) with
 *      logits scale * RoPE(q, pos_t).RoPE(khat_j, pos_j) + b_j, and the result is gated by
 *      sigmoid(g);
 *   4. survivors are compacted stably in place and the new token is appended (b = 0).
 * All in one pass over the cache.  q, g: [B,H,d] act; k, v: [B,Hkv,d] act;
 * a_q, a_k: [B,Hkv] f32; alpha, beta [Hkv] f32; o: [B,H,d] act (required).
 * evict_bits (optional, [B,Hkv,ceil(cap/32)] uint32): bit s set when pre-step slot s was
 * evicted (all words are written).  kept_idx (optional, [B,Hkv,cap] int32): pre-step
 * slot of each survivor in new order, then -1 for the appended token.
 * flags: UA_VAR_* bits, which must equal the variant of the prefill that filled the cache
 * (0 = the method itself; the cache stores softplus(a_k) whatever the variant), plus
 * optionally UA_DECODE_DEFER_COMPACT: step 4 then moves nothing.  Every pair stays in its slot
 * with its updated bias, the new token is appended at slot n_kept, and evicted pairs (b < log p,
 * which never rises again) are left in place, excluded from attention by their bias, until a
 * ua_cache_compact(p) removes them; evict_bits then marks every pair with b < log p and
 * kept_idx (if given) holds s at slot s.  The outputs and the compacted cache are those of the
 * step-by-step compaction; deferring trades the per-step moves for cache slots.  Every cache call requires capacity <= 2^20 slots
 * (UA_ERR_UNSUPPORTED otherwise).  If a cache is full (no pair evicted and n_kept == capacity)
 * the step sets UA_ERR_CAPACITY in the device status word and that cache is left as it
 * was after compaction, without the new token. */
ua_status ua_decode_step(const ua_cache* cache, int H, const void* q, const void* k,
                         const void* v, const void* g, const float* a_q, const float* a_k,
                         const float* alpha, const float* beta, int pos_t, float p, float scale,
                         double rope_theta, void* o, uint32_t* evict_bits, int32_t* kept_idx,
                         int flags, void* stream);

/* ------------------------------------------------------------------ split decode step
 * The same step as ua_decode_step with UA_DECODE_DEFER_COMPACT (set or not in flags), for long
 * caches: a cache of n live slots is walked by several CTAs at once instead of by one -- bf16
 * caches by min(S, ceil(n / 256)) CTAs over slices of whole 128-slot tiles, S (at most 64) chosen
 * on the host from the number of caches and their capacity; fp32 caches by min(16, ceil(n / 512))
 * CTAs over slices of whole 32-slot words (the pages' App. H asks for fused,
 * specialised kernels for the pruned cache; a single CTA per cache leaves most of the GPU idle
 * when B * Hkv is small and the caches long).  Each CTA updates its slots' biases in place and
 * leaves a partial softmax state in the workspace; the last one to finish merges them with the
 * new token, gates, writes o and appends the token at slot n.  evict_bits and kept_idx follow the
 * deferred-compaction rules of ua_decode_step; evicted pairs stay until ua_cache_compact.
 * ws: device workspace of ua_decode_workspace_size bytes (256-byte aligned).  Zero it once before
 * its first use (and again after using it for anything else): its first 4 x B x Hkv bytes are
 * per-cache arrival counters, which every step leaves zero, so consecutive steps need no memset
 * between their kernels (a counter found already at the grid's size raises UA_ERR_INVALID_ARG in
 * the device status).  Calls that share a workspace must not overlap on the GPU.
 * bf16 caches run on the tensor cores: per 128-entry tile one tcgen05 product gives every
 * entry's similarity and G logits (the new key and the rotated queries enter as bf16 high parts
 * plus residuals), a thread per entry turns them into the decay, the bias, the eviction and the
 * probabilities, and a second product accumulates the weighted values in TMEM; the softmax shift
 * starts at the new token's logit and is raised (with the accumulated values rescaled) whenever
 * a tile exceeds it by more than 16, so any query norm is computed.  fp32 caches run the same
 * step on the CUDA cores. */
ua_status ua_decode_workspace_size(const ua_cache* cache, int H, size_t* bytes);
ua_status ua_decode_step_split(const ua_cache* cache, int H, const void* q, const void* k, const void* v,
                               const void* g, const float* a_q, const float* a_k, const float* alpha,
                               const float* beta, int pos_t, float p, float scale, double rope_theta, void* o,
                               uint32_t* evict_bits, int32_t* kept_idx, int flags, void* ws, size_t ws_bytes,
                               void* stream);

/* ------------------------------------------------------------------ status
 * Synchronises `stream`, returns the device status word accumulated since the last call
 * (0 = no error, else a ua_status code) in *code, and clears it. */
ua_status ua_get_device_status(void* stream, int* code);

/* ------------------------------------------------------------------ bounded waits
 * No counterpart on the pages: a robustness aid.  Every device-side wait of the tensor-core
 * kernels (an mbarrier phase, another CTA's published decay prefix) gives up after a limit of
 * %globaltimer nanoseconds, records UA_ERR_TIMEOUT in the device status word and tears the CTA
 * down (abort flag, a 10 ms pause for copies in flight, TMEM freed), so a stuck wait can never
 * hang the GPU.  ua_set_wait_limit_ns sets that limit on the current device (synchronously, for
 * every later launch; UA_WAIT_LIMIT_DEFAULT_NS = 2 s, far above any legitimate wait).  A limit
 * of 0 makes every wait that has to spin give up at its first check: that exercises the timeout
 * path, after which the outputs of the call are unspecified; restore the default afterwards. */
#define UA_WAIT_LIMIT_DEFAULT_NS 2000000000ull
ua_status ua_set_wait_limit_ns(unsigned long long ns);

/* ------------------------------------------------------------------ kernel timing
 * Optional tracing for measurement: while enabled, every libua kernel launch is bracketed
 * by two CUDA events recorded on its stream (about a microsecond of overhead per launch; at
 * most 8192 launches are recorded between resets).  ua_profile_read synchronises on the
 * recorded events and returns, per kernel name, the number of launches and their summed
 * duration in milliseconds; it returns UA_ERR_CAPACITY if launches were dropped.  `name`
 * points to a static string owned by the library. */
typedef struct {
    const char* name;
    int launches;
    double total_ms;
} ua_kernel_time;

ua_status ua_profile_enable(int enable);
ua_status ua_profile_reset(void);
ua_status ua_profile_read(ua_kernel_time* out, int max_entries, int* n_entries);

/* Static, human-readable name of a status code. */
const char* ua_status_string(ua_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
int ua_version(void);

#ifdef __cplusplus
}
#endif

#endif /* UA_H_ */
