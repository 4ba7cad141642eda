/*
 * lowram.h — C ABI of a B200 (sm_100a) library for decode-time attention over a
 * LowRAM-compressed KV cache.
 *
 * What the library computes (one "unit" = one sequence b, one layer l, one KV head):
 *
 *   1. Chunk scoring.  The N prefill tokens of a unit are split into chunks of C tokens.
 *      Each live chunk c is scored against the step's queries:
 *          s_c = sum_{j in group} q_j . kbar_{l,c} / sqrt(d_h),  kbar_{l,c} = abar_c . B_l
 *      where abar_c is the chunk's mean coefficient row (the chunk key summary).
 *      Sources: "LowRAM: Low-Rank Keys and Amortised Values for Composable KV Cache
 *      Compression at Test-Time" (arXiv 2611.07025 abstract: only a selected subset of KV
 *      pairs is reconstructed per step); rit.work "lowram-kv-cache-compression", section
 *      "Значения предсказывают, ключи раскладывают по общему базису" (the context is split
 *      into fragments and the ones that fit the current query are chosen).  The pages do not
 *      define the summary or the score; the mean-key reading is this library's.
 *   2. Top-k selection of the k highest-scoring live chunks (ties go to the lower chunk id).
 *   3. Key rebuild from the cross-layer low-rank form, for the selected chunks only:
 *          khat_t = sigma_t * a_t . B_l
 *      a_t is the token's coefficient row, shared by the G layers of a layer group; B_l is the
 *      layer's slice of the group basis ("LowRAM Compresses KV Cache Asymmetrically",
 *      section "Cross-Layer Low-Rank Key Compression"; rit.work post: keys via xKV with a
 *      common basis for adjacent layers).  sigma_t is the per-token int8 scale, else 1.
 *   4. Value rebuild with the per-head predictor and the stored residuals:
 *          vhat_t = W2 . silu(W1 . khat_t) (+ rho_t * delta_t if token t is flagged)
 *      ("LowRAM Compresses KV Cache Asymmetrically", section "Core Mechanism: Predict
 *      Values and Keep Difficult Residuals": Vhat = f(K), delta = V - Vhat kept for the
 *      worst-predicted tokens).  rho_t is the residual's int8 scale, else 1.
 *   5. GQA attention of each query head j of the unit over the rebuilt tokens of the
 *      selected chunks plus the uncompressed tail of tokens generated after prefill:
 *          o_j = softmax_t(q_j . k_t / sqrt(d_h)) . v_t
 *      ("OjaKV", section 3 "预备知识：低秩注意力", the attention equations; the raw tail:
 *      rit.work post, same section as in step 1).
 *
 * Layouts: all arrays are row-major, last index contiguous.  Symbols: B batch, L layers,
 * G layers per group, Hkv KV heads, Hq query heads (g = Hq/Hkv per KV head), d head dim,
 * r rank, h predictor hidden width, N compressed tokens, C chunk size, nC = N/C chunks,
 * nL live chunks per (b, group, KV head) (nL = nC without eviction), T tail capacity.
 * Query head j belongs to KV head j / g.
 *
 * Error behaviour: every entry point returns a lowram_status.  Argument and shape checks
 * run on the host before anything is launched and return LOWRAM_EINVAL with no side
 * effect.  A CUDA error becomes LOWRAM_ECUDA; lowram_last_error_string() gives the CUDA
 * runtime's text for the calling thread.  Kernels never trap: a device-side check that
 * fails records an error word that lowram_cache_validate() turns into LOWRAM_ECORRUPT.
 */
#ifndef LOWRAM_H
#define LOWRAM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lowram_stream; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  LOWRAM_OK = 0,
  LOWRAM_EINVAL = 1,        /* bad argument, shape or pointer; nothing was launched */
  LOWRAM_ENOMEM = 2,        /* a device allocation failed (create only) */
  LOWRAM_ECUDA = 3,         /* a CUDA runtime call or launch failed */
  LOWRAM_EUNSUPPORTED = 4,  /* the shapes are valid but no kernel in this build handles them */
  LOWRAM_ECORRUPT = 5,      /* lowram_cache_validate found an inconsistent index table */
  LOWRAM_ETIMEOUT = 6       /* a kernel gave up a bounded wait and returned early */
} lowram_status;

typedef enum {
  LOWRAM_F32 = 0,  /* fp32 storage and fp32 arithmetic everywhere */
  LOWRAM_BF16 = 1  /* bf16 storage; tensor-core products with fp32 accumulation */
} lowram_dtype;

typedef enum {
  LOWRAM_STORE_NATIVE = 0, /* coefficients and residuals stored in the config dtype */
  LOWRAM_STORE_INT8 = 1    /* int8 coefficients and residuals with one fp16 scale per row
                              ("LowRAM Compresses KV Cache Asymmetrically", section
                              "Composition with Quantization and Eviction").  Needs BF16. */
} lowram_store;

/* Shapes of one compressed cache.  Constraints checked by lowram_cache_create:
 * n_layers % group == 0, n_q_heads % n_kv_heads == 0, n_ctx % chunk == 0,
 * 1 <= top_k <= n_live <= n_ctx/chunk, rank <= group*head_dim, chunk <= 32767,
 * n_q_heads/n_kv_heads <= 16, head_dim <= 256, rank <= 512, mlp_hidden <= 1024,
 * n_ctx/chunk <= 8192, tail_cap <= 4096. */
typedef struct {
  int32_t batch;       /* B */
  int32_t n_layers;    /* L */
  int32_t group;       /* G: layers sharing one coefficient matrix */
  int32_t n_kv_heads;  /* Hkv */
  int32_t n_q_heads;   /* Hq */
  int32_t head_dim;    /* d */
  int32_t rank;        /* r */
  int32_t mlp_hidden;  /* h */
  int32_t n_ctx;       /* N compressed (prefill) tokens per sequence */
  int32_t chunk;       /* C */
  int32_t top_k;       /* k chunks selected per unit and step */
  int32_t tail_cap;    /* T: capacity of the raw tail per (b, l, KV head) */
  int32_t n_live;      /* nL: live chunks per (b, group, KV head) */
  int32_t dtype;       /* lowram_dtype */
  int32_t store;       /* lowram_store */
} lowram_config;

/* Source arrays of a compressed cache, all DEVICE pointers, read by lowram_cache_create
 * (which copies them; the caller keeps ownership and may free them once the create
 * stream has reached the copy).  "dt" is fp32 (LOWRAM_F32) or bf16 (LOWRAM_BF16).
 *
 *   coeff      [B][L/G][Hkv][nL*C][r]  dt, or int8 with STORE_INT8.  Rows of live chunks
 *                                      only, chunk after chunk in ascending chunk id.
 *   coeff_scale[B][L/G][Hkv][nL*C]     fp16 per-row scale (STORE_INT8), else NULL.
 *   basis      [L][Hkv][r][d]          dt.  B_l, the layer's slice of the group basis.
 *   w1         [L][Hkv][h][d]          dt.  Predictor first layer (out x in), no bias.
 *   w2         [L][Hkv][d][h]          dt.  Predictor second layer (out x in), no bias.
 *   summary    [B][L/G][Hkv][nL][r]    dt (bf16 with STORE_INT8).  abar: the mean of the
 *                                      chunk's (dequantised) coefficient rows.
 *   slot       [B][L/G][Hkv][nC]       int16: storage slot of chunk c, or -1 if evicted.
 *                                      NULL means no eviction (slot[c] = c, nL = nC).
 *                                      Live slots are 0..nL-1 in ascending chunk id.
 *   res_ptr    [B][L][Hkv][nL+1]       int32 global record offsets: records of slot s of a
 *                                      unit are [res_ptr[s], res_ptr[s+1]).  Non-decreasing.
 *   res_pos    [R]                     uint16 token offset of the record inside its chunk,
 *                                      strictly increasing within a chunk, < C.
 *   res_val    [R][d]                  dt, or int8 with STORE_INT8.  delta rows.
 *   res_scale  [R]                     fp16 per-record scale (STORE_INT8), else NULL.
 *   tail_k     [B][L][Hkv][T][d]       dt (bf16 with STORE_INT8).  Raw tail keys.
 *   tail_v     [B][L][Hkv][T][d]       dt (bf16 with STORE_INT8).  Raw tail values.
 *   tail_len   [B]                     int32, 0 <= tail_len[b] <= T.
 * Every pointer must be 16-byte aligned. */
typedef struct {
  const void* coeff;
  const void* coeff_scale;
  const void* basis;
  const void* w1;
  const void* w2;
  const void* summary;
  const int16_t* slot;
  const int32_t* res_ptr;
  const uint16_t* res_pos;
  const void* res_val;
  const void* res_scale;
  const void* tail_k;
  const void* tail_v;
  const int32_t* tail_len;
  int64_t n_records; /* R: total residual records (length of res_pos/res_val/res_scale) */
} lowram_cache_src;

typedef struct lowram_cache lowram_cache; /* opaque; owns its device memory */

/* Byte accounting of a cache (host only). */
typedef struct {
  uint64_t coeff;       /* coefficient rows (+ their scales) */
  uint64_t basis;       /* per-layer bases */
  uint64_t predictor;   /* W1 and W2 */
  uint64_t summary;     /* chunk key summaries */
  uint64_t residual;    /* residual rows, positions, scales and CSR offsets */
  uint64_t index;       /* eviction slot map */
  uint64_t tail;        /* raw tail keys and values (+ lengths) */
  uint64_t total;       /* sum of the above: the compressed cache */
  uint64_t dense_equiv; /* M_KV * B for the same N (at 2 bytes per scalar for BF16 and
                           int8 stores, 4 for F32) plus the same raw tail */
} lowram_bytes;

/* Execution path of lowram_decode_attn.  There is one product path per shape: AUTO takes the
 * tcgen05 kernel for every BF16 shape it serves and the CUDA-core kernel for the rest (every
 * LOWRAM_F32 cache, and BF16 shapes the tensor-core kernel does not serve).  SIMT and TC only
 * pin that choice.  SIMT on a cache AUTO would serve on tensor cores is a DIAGNOSTIC: a
 * second, independent implementation (fp32 arithmetic, about 100x slower) that tests use to
 * cross-check the tensor-core kernel; it is not a second backend to deploy. */
typedef enum {
  LOWRAM_PATH_AUTO = 0,  /* the product path: tensor cores when the shapes allow, else CUDA cores */
  LOWRAM_PATH_SIMT = 1,  /* CUDA-core kernel (any shapes; the only one for LOWRAM_F32; for BF16
                            shapes the tensor cores serve, a diagnostic cross-check) */
  LOWRAM_PATH_TC = 2     /* tcgen05 tensor-core kernel; LOWRAM_EUNSUPPORTED if shapes don't fit */
} lowram_path;

/* Dense KV-cache bytes M_KV * B = 2 * L * Hkv * d * N * s * B ("LowRAM Compresses KV Cache
 * Asymmetrically", section "Core Mechanism", the M_KV formula).  Host only; returns 0 if an
 * argument is negative. */
uint64_t lowram_dense_kv_bytes(int32_t n_layers, int32_t n_kv_heads, int32_t head_dim,
                               int64_t n_ctx, int32_t bytes_per_scalar, int32_t batch);

/* Byte accounting of a cache with these shapes and n_records residual records, without
 * creating it (host only; for capacity planning).  has_slot says whether an eviction slot
 * map is stored (only when n_live < n_ctx/chunk).  Returns EINVAL for a bad config. */
lowram_status lowram_config_bytes(const lowram_config* cfg, int64_t n_records, int32_t has_slot,
                                  lowram_bytes* out);

/* Copy a compressed cache into memory the cache object owns, derive the folded predictor
 * weights W1' = W1 . B_l^T per (layer, KV head) (an exact rewrite: W1 . khat = W1' . a), and
 * allocate the per-call scratch for up to cfg->batch sequences and all layers.
 * Stream-ordered on `stream`; the object is usable on that stream immediately.
 * Returns EINVAL for bad shapes or NULL/unaligned pointers, ENOMEM if allocation fails. */
lowram_status lowram_cache_create(const lowram_config* cfg, const lowram_cache_src* src,
                                  lowram_cache** out, lowram_stream stream);

/* Free everything the cache owns (synchronises the device first).  NULL is a no-op. */
void lowram_cache_destroy(lowram_cache* cache);

/* Decode-time attention for layers [layer0, layer0 + n_layers) of every sequence.
 *   q   [n_layers][B][Hq][d]  dt, DEVICE.  One decode query per sequence per layer.
 *   out [n_layers][B][Hq][d]  dt, DEVICE.  o_j of step 5.
 *   sel [n_layers][B][Hkv][k] int32, DEVICE, may be NULL: the selected chunk ids of each
 *                             unit in ascending order.
 * Runs steps 1-5 on `stream`: no host synchronisation and no allocation.  One cache must
 * not be used by two streams at the same time (the scratch is shared).  Returns EINVAL
 * for a bad layer range or NULL q/out, EUNSUPPORTED if `path` cannot serve the shapes. */
lowram_status lowram_decode_attn(lowram_cache* cache, int32_t layer0, int32_t n_layers,
                                 const void* q, void* out, int32_t* sel, int32_t path,
                                 lowram_stream stream);

/* Steps 1-2 alone: chunk scores and the top-k selection.
 *   scores [n_layers][B][Hkv][nC] fp32, DEVICE, may be NULL: s_c, -inf for evicted chunks.
 *   sel    [n_layers][B][Hkv][k]  int32, DEVICE, may be NULL (ids ascending). */
lowram_status lowram_select_chunks(lowram_cache* cache, int32_t layer0, int32_t n_layers,
                                   const void* q, float* scores, int32_t* sel,
                                   lowram_stream stream);

/* Same as lowram_decode_attn with HOST buffers q_host/out_host/sel_host (sel may be NULL):
 * copies q to the device, decodes, copies the results back and synchronises `stream`.
 * Pinned host memory makes the copies asynchronous; pageable memory works too.  The decode
 * runs on device buffers the cache owns, so the first call for a layer range captures it
 * into a CUDA graph (on a stream of the cache's own) and later calls replay the graph; a
 * re-pack drops it, stage events (lowram_cache_set_stage_events) bypass it, and if capture
 * fails the calls stay eager. */
lowram_status lowram_decode_attn_host(lowram_cache* cache, int32_t layer0, int32_t n_layers,
                                      const void* q_host, void* out_host, int32_t* sel_host,
                                      lowram_stream stream);

/* Byte accounting of a created cache (host only, no device access): the live arrays.  Room a
 * re-pack keeps for later chunks (lowram_cache_view's spare_chunks, and the spare record
 * rows after each unit's records) is allocated in addition and not counted here. */
lowram_status lowram_cache_bytes(const lowram_cache* cache, lowram_bytes* out);

/* Device-side consistency check of the index tables (slot map, CSR offsets, record
 * positions, tail lengths) and of the error word left by earlier kernels.  Synchronises
 * `stream`.  Returns ECORRUPT if a table is inconsistent, ETIMEOUT if an earlier kernel
 * reported a bounded wait that ran out, EINVAL if an earlier lowram_cache_append found a
 * full tail (and dropped that token), OK otherwise; the error word is cleared. */
lowram_status lowram_cache_validate(lowram_cache* cache, lowram_stream stream);

/* Optional timing hook: when events != NULL, lowram_decode_attn records events[0] before
 * its first kernel, events[1] after steps 1-2 and the tail, events[2] after the chunk
 * attention kernel and events[3] after the combine, all on the call's stream.  The events
 * are cudaEvent_t handles owned by the caller; pass NULL to switch the hook off. */
lowram_status lowram_cache_set_stage_events(lowram_cache* cache, void* const* events);

/* Number of kernels the last lowram_decode_attn call on this cache launched. */
int32_t lowram_cache_last_launches(const lowram_cache* cache);

/* Which path the last lowram_decode_attn call on this cache ran (a lowram_path value). */
int32_t lowram_cache_last_path(const lowram_cache* cache);

/* ------------------------------------------------------------- decode-loop upkeep
 *
 * Tokens generated after prefill stay uncompressed in the raw tail (rit.work
 * "lowram-kv-cache-compression": generated tokens are kept raw).  When every sequence's
 * tail holds at least one chunk, lowram_cache_repack compresses the oldest chunk of the
 * tail with the cache's basis and predictor.  The pages name no moment for this; the
 * library's reading: one chunk of C tokens at a time, encoded by the steps of
 * lowram_encode below, appended after the existing chunks. */

/* The arrays the cache owns, as a read-only view (DEVICE pointers; slot is NULL when
 * nothing is evicted), and its current config.  Layouts are those of lowram_cache_src except
 * that each (b, group, KV head) / (b, l, KV head) keeps room for *spare_chunks more chunks:
 * unit strides of (nL + S) * C coefficient rows (and scales), nL + S summaries, nL + S + 1
 * CSR offsets and nC + S slot entries, S = *spare_chunks (0 until a re-pack adds room).
 * After a re-pack the records of each unit are followed by spare record rows, so n_records
 * counts allocated rows, not live records.  While *spare_chunks is 0 the view is exactly a
 * lowram_cache_src (lowram_decode_attn_static and lowram_cache_create accept it); with
 * spare room the chunk arrays are strided and those entry points do not.  Valid until the
 * next lowram_cache_repack or lowram_cache_destroy.  Host only. */
lowram_status lowram_cache_view(const lowram_cache* cache, lowram_config* cfg, lowram_cache_src* src,
                                int32_t* spare_chunks);

/* Append one decode step's key and value to every (layer, sequence, KV head) tail:
 *   k_new, v_new [L][B][Hkv][d], the tail's element type (dt; bf16 with STORE_INT8),
 *   DEVICE, 16-byte aligned.
 * Writes tail[b][l][h][tail_len[b]] and then adds 1 to tail_len[b].  A sequence whose tail
 * is full (tail_len[b] == T) is left unchanged and its token dropped; the error word
 * records it and lowram_cache_validate then returns LOWRAM_EINVAL.  Needs
 * head_dim * element size to be a multiple of 16 (EUNSUPPORTED otherwise).
 * Stream-ordered: two small kernels, no allocation, no host synchronisation. */
lowram_status lowram_cache_append(lowram_cache* cache, const void* k_new, const void* v_new,
                                  lowram_stream stream);

/* Re-pack the oldest C tail tokens of every (sequence, layer, KV head) into one new chunk.
 * The new chunk is encoded as lowram_encode encodes a context of C tokens (steps 1-6 below,
 * with n_resid residual records per (b, l, KV head) for this chunk, 0 <= n_resid <= C),
 * appended after the existing chunks (slot nL when the cache evicts: a new live chunk),
 * and the tail shifts down by C (tail_len[b] -= C).  Afterwards n_ctx grows by C and
 * n_live by 1; residual records are re-laid in unit order (b, l, KV head), a unit's old
 * records first.
 * Requires every tail_len[b] >= C (EINVAL otherwise), tail_cap >= chunk, and the shapes
 * lowram_encode supports (EUNSUPPORTED otherwise).
 * SYNCHRONOUS: it reads the tail lengths to the host and returns after the stream has
 * finished.  When the cache has room for one more chunk per unit (and for the new records
 * after each unit's last ones), the new chunk is written in place; otherwise the arrays are
 * re-laid into new allocations with room for max(4, nL / 16) more chunks per unit and as
 * many spare records per unit as this call keeps per chunk (device memory peaks at about
 * twice the cache during that copy; the old arrays are freed).  A cache created from
 * caller arrays gets its room at its first re-pack.  On any error the cache is left as it
 * was.  Meant to run once every C decode steps. */
lowram_status lowram_cache_repack(lowram_cache* cache, int32_t n_resid, lowram_stream stream);

/* Dense decode attention over an UNCOMPRESSED bf16 KV cache, the baseline a compressed cache
 * is compared with: every cached token is attended, o_j = softmax_t(q_j . k_t / sqrt(d)) v_t
 * ("OjaKV", section 3, attention), and the cache holds M_KV = 2 L Hkv d N s bytes per
 * sequence ("LowRAM Compresses KV Cache Asymmetrically", section "Core Mechanism").
 *   k, v [B][L][Hkv][S][d] bf16, DEVICE, 16-byte aligned;
 *   q, out [L][B][Hq][d] bf16, DEVICE.  All L layers in one call, stream-ordered.
 * Needs head_dim % 8 == 0, head_dim <= 256, Hq/Hkv <= 16; returns EINVAL otherwise.
 * d = 128 with Hq/Hkv in {1, 2, 4, 8, 16} and a 16-byte aligned q runs on tcgen05 tensor
 * cores (probabilities rounded to bf16 for the P.V product, fp32 accumulation); other
 * shapes on CUDA cores (fp32 throughout).  The tensor-core kernel's waits are bounded: if
 * one runs out (it does not in normal operation) that unit's outputs are written as NaN. */
lowram_status lowram_dense_decode_attn(int32_t batch, int32_t n_layers, int32_t n_kv_heads,
                                       int32_t n_q_heads, int32_t head_dim, int64_t seq_len,
                                       const void* k, const void* v, const void* q, void* out,
                                       lowram_stream stream);

/* Decode-time attention with no device allocation at all, for callers that cannot call
 * cudaMalloc on their decode path (an engine that reserves all device memory for its own
 * pool, a runtime that forbids allocation after start-up, a thread capturing a CUDA graph
 * in a mode that rejects allocation calls).  The pages have no counterpart of this entry
 * point; it is a deployment variant of lowram_decode_attn.
 *
 * It reads the compressed cache straight from the caller's DEVICE arrays `src` (layouts of
 * lowram_cache_src, no copy, no cache object), runs the CUDA-core decode kernels for layers
 * [layer0, layer0 + n_layers) and writes out / sel exactly like lowram_decode_attn (q, out,
 * sel: DEVICE, layouts as there).  All scratch -- the folded W1' of the requested layers,
 * the projected queries, the selection, the split partials and an error word -- lives in
 * one static device array of 16 MiB inside the library, which every GPU that loads the
 * library holds until the process exits.
 *
 * Limits and behaviour:
 *  - A call whose scratch exceeds 16 MiB is rejected with LOWRAM_EINVAL and a message giving
 *    the bytes needed (for the 32K Llama-shaped cache: one to three layers per call fit).
 *  - It calls no cudaMalloc, cudaFree or allocating library routine.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (once per device, with that device current); make that first call
 *    before any stream capture.
 *  - Every call shares the array, which keeps the last call's contents (the error word is
 *    cleared at the start of each call): calls that overlap on the GPU -- on two streams,
 *    or on the same device from two threads -- race and must be serialised by the caller.
 *  - Stream-ordered on `stream`, no host synchronisation; same error codes as
 *    lowram_decode_attn. */
lowram_status lowram_decode_attn_static(const lowram_config* cfg, const lowram_cache_src* src,
                                        int32_t layer0, int32_t n_layers, const void* q,
                                        void* out, int32_t* sel, lowram_stream stream);

/* ------------------------------------------------------------- context-sharded decode
 *
 * One sequence's context split by chunk over P shards, usually one per GPU, so that a context
 * too long for one GPU's memory (or bandwidth) is decoded by several ("LowRAM Compresses KV
 * Cache Asymmetrically", section "Why Peak Throughput Can Improve by 5x": decode is bound by
 * moving the KV cache, also between GPUs).  Shard s is an ordinary cache created from the
 * chunk ids [off_s, off_s + nC_s) of every (sequence, layer group, KV head): its coefficient
 * rows, scales, summaries and those chunks' residual records, its chunk ids local (global id =
 * off_s + local id); every shard holds the same weights, and only the shard with the newest
 * tokens has a non-empty raw tail (tail_len = 0 elsewhere).  Each shard needs nC_s >= top_k
 * live chunks.  One decode step:
 *   1. every shard: lowram_shard_candidates -> its own top k as (score, global chunk id);
 *   2. the caller gathers every shard's candidates on every shard, in ascending off_s order
 *      (an all-gather; the library itself does not communicate);
 *   3. every shard: lowram_shard_partial -> the k best of all candidates by (descending score,
 *      ascending global id) -- exactly the unsharded selection, since a chunk among the k
 *      best overall has fewer than k better chunks in its own shard -- then attention of each
 *      query head over the selected chunks the shard holds plus its raw tail, unnormalised;
 *   4. the caller gathers the shards' partials; lowram_merge_partials gives the output:
 *      o_j = sum_s w_s y_{s,j} / sum_s w_s l_{s,j},  w_s = 2^(m_{s,j} - max_s m_{s,j}).
 * The result equals lowram_decode_attn on the whole cache up to floating-point regrouping.
 * Shapes: those the tensor-core path serves (EUNSUPPORTED otherwise). */

/* Phase 1 on one shard for layers [layer0, layer0 + n_layers):
 *   q          [n_layers][B][Hq][d] dt, DEVICE (the same queries on every shard);
 *   cand_score [n_layers][B][Hkv][k] fp32, DEVICE: the scores of the shard's own k best chunks;
 *   cand_id    [n_layers][B][Hkv][k] int32, DEVICE: their global ids (chunk_offset + local id),
 *              ascending.
 * Also leaves in the cache's scratch what phase 2 needs (the projected queries and the raw
 * tail's partial softmax): lowram_shard_partial must be the next call on this cache that
 * writes its scratch (no decode, selection or re-pack in between).  Stream-ordered, no
 * allocation, no host synchronisation.  EINVAL for a bad range, NULL pointer or negative
 * offset. */
lowram_status lowram_shard_candidates(lowram_cache* shard, int32_t layer0, int32_t n_layers, const void* q,
                                      int32_t chunk_offset, float* cand_score, int32_t* cand_id,
                                      lowram_stream stream);

/* Phase 2 on one shard, after every shard's candidates were gathered:
 *   cand_score / cand_id [n_shards][n_layers][B][Hkv][k] (shards in ascending chunk_offset);
 *   partial [n_layers][B][Hq][d + 2] fp32, DEVICE: per query head j, m_j (the largest logit
 *           in log2 units: q.k / sqrt(d) * log2(e)), l_j = sum_t 2^(logit_t - m_j) and
 *           y_j[d] = sum_t 2^(logit_t - m_j) v_t over the shard's selected tokens and tail
 *           (m_j = -inf, l_j = 0, y_j = 0 when the shard holds none of them);
 *   sel     [n_layers][B][Hkv][k] int32, DEVICE, may be NULL: the global selection, ascending.
 * EINVAL unless it follows lowram_shard_candidates for the same layers on this cache, or when
 * n_shards < 1 or n_shards * top_k > 1024.  Stream-ordered, no allocation or synchronisation. */
lowram_status lowram_shard_partial(lowram_cache* shard, int32_t layer0, int32_t n_layers, int32_t chunk_offset,
                                   int32_t n_shards, const float* cand_score, const int32_t* cand_id,
                                   float* partial, int32_t* sel, lowram_stream stream);

/* Merge of the shards' partial records: partials [n_parts][n_rows][head_dim + 2] fp32 (rows
 * laid out as lowram_shard_partial writes them), out [n_rows][head_dim] in out_dtype
 * (LOWRAM_F32 or LOWRAM_BF16), DEVICE.  EINVAL for bad sizes.  Stream-ordered. */
lowram_status lowram_merge_partials(int32_t n_parts, int64_t n_rows, int32_t head_dim, const float* partials,
                                    int32_t out_dtype, void* out, lowram_stream stream);

/* ---------------------------------------------------------- reuse of rebuilt chunks
 *
 * Consecutive decode steps select mostly the same chunks; each step can reuse what an earlier
 * one rebuilt (rit.work "lowram-kv-cache-compression", section "Значения предсказывают, ключи
 * раскладывают по общему базису").  A store keeps, per (sequence, layer, KV head, chunk), the
 * chunk's rebuilt values vhat_t = W2 silu(W1 khat_t) + delta_t (bf16, C x d = 32 KB at C = d =
 * 128); a hit attends over them, scoring the keys from the stored coefficients as usual, and
 * skips the predictor.  Policy (this library's; the pages give none): `capacity` entries filled
 * first-in first-out; per decode call at most `fill_cap` of its misses are admitted, in unit
 * order ((layer, KV head, sequence), sequence fastest), each unit's in ascending chunk id; hits
 * are decided against the store as it was before the call.  The results equal those of
 * lowram_decode_attn up to floating-point rounding (the stored values are rounded to bf16).
 * Costs: a miss as lowram_decode_attn; a hit reads the chunk's coefficients and its stored
 * values (2 x 32 KB) and runs no predictor; a fill rebuilds the chunk's values once more
 * (tensor cores) and writes them.  Shapes: bf16 native stores, head_dim 128, mlp_hidden 256,
 * rank 64 or 128, chunk 128, 4 or 8 query heads per KV head, top_k <= 32. */
typedef struct lowram_reuse lowram_reuse; /* opaque; owns its device memory */
typedef struct {
  uint64_t hits, misses, fills;  /* cumulative chunk counts over the store's decode calls */
} lowram_reuse_counts;

/* A store for `cache` with `capacity` entries (1 <= capacity <= 2^30; capacity * 32 KB at C = d
 * = 128, plus a table of 4 bytes per chunk slot of the cache), admitting at most
 * fill_cap <= capacity misses per call.
 * Stream-ordered.  EINVAL for bad sizes, EUNSUPPORTED for shapes without a reuse path, ENOMEM;
 * *out is NULL after any error.  The store is tied to the cache as it is now: after a lowram_cache_repack the store's calls
 * return EINVAL (make a new one).  Destroy the store before the cache. */
lowram_status lowram_reuse_create(lowram_cache* cache, int32_t capacity, int32_t fill_cap, lowram_reuse** out,
                                  lowram_stream stream);
void lowram_reuse_destroy(lowram_reuse* store); /* synchronises the device first; NULL is a no-op */

/* lowram_decode_attn for layers [layer0, layer0 + n_layers) through the store (q, out, sel as
 * there), updating it.  Stream-ordered, no allocation, no host synchronisation.  A store must
 * not be used by two streams at the same time, nor its cache by another call in between the
 * kernels of this one. */
lowram_status lowram_decode_attn_reuse(lowram_reuse* store, int32_t layer0, int32_t n_layers, const void* q,
                                       void* out, int32_t* sel, lowram_stream stream);

/* The cumulative hit / miss / fill counts (synchronises `stream`). */
lowram_status lowram_reuse_counts_get(lowram_reuse* store, lowram_reuse_counts* out, lowram_stream stream);

/* Read-only DEVICE view of the store (valid until lowram_reuse_destroy): table [B][L][Hkv]
 * [table_stride] int32 (the entry holding chunk slot s of (b, l, KV head), or -1), owner
 * [capacity] int64 (the table index an entry serves, or -1) and entries [capacity][C][d] bf16. */
lowram_status lowram_reuse_view(const lowram_reuse* store, const int32_t** table, const int64_t** owner,
                                const void** entries, int64_t* table_stride);

/* ---------------------------------------------------------------- prefill-side encoder
 *
 * lowram_encode: dense keys and values -> the compressed arrays lowram_cache_create takes
 * (no eviction: pass slot = NULL there), with a GIVEN basis and predictor (no fitting).
 * Steps, per sequence b, layer group, KV head and chunk of C tokens:
 *   1. coefficients a_t = (1/G) sum_{l in group} k_{l,t} . B_l^T, the least-squares fit of
 *      the group's keys on its stacked basis when every B_l has orthonormal rows
 *      ("LowRAM Compresses KV Cache Asymmetrically", section "Cross-Layer Low-Rank Key
 *      Compression"; the caller must pass such a basis -- for another one the result is
 *      the average of the per-layer projections, not the least-squares fit);
 *   2. storage: bf16 (STORE_NATIVE), or int8 with a per-row fp16 scale = max|a| / 127
 *      rounded to fp16 and codes round-half-even(a / scale) clamped to +-127 (STORE_INT8;
 *      same section, "Composition with Quantization and Eviction");
 *   3. summary: the mean of the chunk's stored (dequantised) coefficient rows, bf16;
 *   4. per layer: vhat_t = W2 silu(W1 khat_t) with khat_t the key rebuilt from the STORED
 *      coefficients, delta_t = v_t - vhat_t ("Core Mechanism: Predict Values and Keep
 *      Difficult Residuals");
 *   5. residual flags: the n_resid tokens of each (b, l, KV head) with the largest
 *      |delta_t|_2 (float32), ties to the lower token index;
 *   6. records: unit by unit in the order (b, l, KV head), chunk by chunk, ascending token
 *      offset; unit u's records are [u * n_resid, (u + 1) * n_resid).
 *
 * Arguments (DEVICE pointers, 16-byte aligned, row-major):
 *   keys, values [B][L][Hkv][N][d] bf16;  basis [L][Hkv][r][d], w1 [L][Hkv][h][d],
 *   w2 [L][Hkv][d][h] bf16 (the same arrays a cache is then created with);
 *   dst->coeff [B][L/G][Hkv][N][r] bf16 or int8, dst->coeff_scale [B][L/G][Hkv][N] fp16
 *   (STORE_INT8, else NULL), dst->summary [B][L/G][Hkv][nC][r] bf16,
 *   dst->res_ptr [B][L][Hkv][nC+1] int32, dst->res_pos [B*L*Hkv*n_resid] uint16,
 *   dst->res_val [B*L*Hkv*n_resid][d] bf16 or int8, dst->res_scale [B*L*Hkv*n_resid] fp16
 *   (STORE_INT8, else NULL);  workspace: at least lowram_encode_workspace_bytes(cfg) bytes.
 *   The caller owns every buffer.  cfg->n_live must equal n_ctx / chunk; top_k, tail_cap
 *   and n_q_heads are not used.
 * Supported shapes: dtype BF16, head_dim 128, mlp_hidden 256, rank 64 or 128, chunk 64 or
 * 128, 0 <= n_resid <= n_ctx, B*L*Hkv*n_resid < 2^31; LOWRAM_EUNSUPPORTED otherwise.
 * Stream-ordered on `stream`, no allocation, no host synchronisation. */
typedef struct {
  void* coeff;
  void* coeff_scale;
  void* summary;
  int32_t* res_ptr;
  uint16_t* res_pos;
  void* res_val;
  void* res_scale;
} lowram_encode_dst;

/* Workspace bytes lowram_encode needs for cfg (0 if cfg is invalid).  Host only. */
uint64_t lowram_encode_workspace_bytes(const lowram_config* cfg);

lowram_status lowram_encode(const lowram_config* cfg, int32_t n_resid, const void* keys,
                            const void* values, const void* basis, const void* w1,
                            const void* w2, const lowram_encode_dst* dst, void* workspace,
                            uint64_t workspace_bytes, lowram_stream stream);

/* ------------------------------------------------------------------- test hooks
 *
 * For tests of the failure paths only; a deployment never calls these.  They make a failure
 * happen on the host side (an allocation reported as failed) or make a bounded wait in a
 * kernel run out early; neither faults, traps or hangs the GPU.  The pages have no
 * counterpart. */

/* Limit, in SM clock cycles, of the main-loop waits of the tensor-core chunk-attention kernel
 * in later lowram_decode_attn calls on this cache; cycles <= 0 restores the default (about
 * one second).  A wait that runs out raises the kernel's error word and abort flag: every
 * warp of that CTA stops, the CTA waits (with the default limit) for the copies and MMAs it
 * has already issued, frees its tensor memory and returns, so the context stays usable.  The
 * call's outputs are then meaningless and lowram_cache_validate returns LOWRAM_ETIMEOUT.  A
 * limit of a few cycles makes the first wait that is not already satisfied run out.
 * Drops the graph lowram_decode_attn_host keeps.  EINVAL for a NULL cache. */
lowram_status lowram_debug_set_wait_limit(lowram_cache* cache, int64_t cycles);

/* Inject one allocation failure: the next `after` device allocations made by
 * lowram_cache_create or lowram_cache_repack succeed and the one after them fails as if
 * cudaMalloc had run out of memory (those calls then return LOWRAM_ENOMEM, leaving no
 * allocation behind; a failed re-pack leaves the cache as it was).  One-shot: the hook is
 * off again after the failure.  after < 0 switches it off.  Process-wide; not meant for
 * concurrent use. */
void lowram_debug_fail_alloc(int32_t after);

const char* lowram_status_string(lowram_status status);
const char* lowram_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* LOWRAM_H */
