/*
 * duo.h -- C ABI of the B200 (sm_100a) hybrid-head KV attention library.
 *
 * The operation is DuoAttention's deployment path ("DuoAttention: Efficient
 * Long-Context LLM Inference with Retrieval and Streaming Heads", arXiv 2410.10819,
 * as explained on the paper-graph-ui page, section "Deployment Architecture"):
 * each KV head of a layer is either a retrieval head, which keeps every token and
 * attends with the causal mask, or a streaming head, which keeps only the first S
 * "attention sink" tokens plus the W most recent tokens and attends with the
 * Lambda-shaped mask ("The Full and Streaming Attention Masks").
 *
 * Conventions shared by every call
 * ---------------------------------
 * Notation: B batch, Hq query heads, Hkv KV heads, G = Hq / Hkv, d head_dim,
 * S sinks, W recent window, len = tokens already in a layer's cache, n = tokens in
 * one call.  Query head h reads KV head h / G (contiguous GQA grouping); the cache
 * is kept per KV head, so no K/V row is ever repeated per query head.
 *
 * Mask: query at absolute position i sees key j iff j <= i and, for a streaming
 * head, (j < S or i - j < W).  W counts the query's own token, so a streaming
 * head holds exactly S + W tokens once len >= S + W, and W >= 1.
 *
 * Tensors are dense, row-major, device-resident, 16-byte aligned, in the dtype
 * chosen at creation (bf16 or fp32):
 *     decode q, out   [B][Hq][d]          decode lse   [B][Hq]      (fp32)
 *     prefill q, out  [B][n][Hq][d]       prefill lse  [B][n][Hq]   (fp32)
 *     k, v            [B][n][Hkv][d]
 * lse is the natural log of the sum of exp(scaled logits) over the visible keys.
 * Heads keep the caller's order; the library groups retrieval and streaming heads
 * internally through index tables, so no weight permutation is needed.
 *
 * Ownership: the caller owns every device buffer, the cache storage included
 * (one buffer of duo_cache_bytes() bytes, 256-byte aligned).  The handle owns only
 * host metadata.  No pointer is kept beyond the call that receives it, except the
 * cache buffer, which must outlive the handle.
 *
 * Ordering: calls are asynchronous on the given CUDA stream (NULL = legacy default
 * stream).  Calls on one handle must be ordered on one stream (or externally
 * synchronised): they share the cache's scratch space.  A handle is not thread-safe.
 *
 * Errors: every argument is checked, and every fallible host step of a call (tensor
 * map encoding, kernel attributes) is done, before its first launch; on such an error
 * nothing is launched and the cache (lengths included) is unchanged.  A launch that
 * fails returns DUO_ERR_CUDA.  len always describes what the cache holds: it advances
 * exactly when the launch that writes the new rows was accepted.  Each call writes the
 * cache in its last launch, so a call that fails leaves it unchanged -- except
 * duo_append_decode on its two-launch path, whose token stays appended (len advanced)
 * when the attention launch after the append fails.  Conditions detected on the device
 * (a bounded wait that ran out) are latched in a status word and reported by
 * duo_get_device_status().
 */
#ifndef DUO_H
#define DUO_H

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

typedef struct duo_cache duo_cache; /* opaque host handle */

typedef enum {
  DUO_OK = 0,
  DUO_ERR_INVALID = 1,     /* bad argument (NULL, range, alignment, shape)      */
  DUO_ERR_CAPACITY = 2,    /* the call would grow a layer past max_len          */
  DUO_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed              */
  DUO_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (device status)   */
  DUO_ERR_UNSUPPORTED = 5  /* valid request this build does not implement       */
} duo_status;

typedef enum { DUO_BF16 = 0, DUO_FP32 = 1 } duo_dtype;

/* Storage of retrieval-head K/V.  DUO_KV_INT4_G128: 4-bit asymmetric codes, one
 * group per token row of a head (head_dim must be 128), fp16 scale and zero per
 * group: scale = fp16((max-min)/15), zero = fp16(min), code = clamp(rint((x - zero)
 * / scale), 0, 15) in fp32, element 2t in the low nibble of byte t, value =
 * code*scale + zero.  DUO_KV_FP8_E4M3: 8-bit floating point codes (OCP E4M3: bias 7,
 * 3 mantissa bits, largest finite 448), one fp32 scale per token row of a head (head_dim
 * 128): scale = max|x| / 448, code = x / scale rounded to the nearest E4M3 value (ties
 * to even, held at +-448), value = code * scale ("Integration with Existing
 * Optimizations": 8-bit KV).  Both: bf16 only; caches of these formats are filled with
 * duo_append_kv / duo_append_decode and read by decode (pre-fill of them is
 * DUO_ERR_UNSUPPORTED).  Streaming heads always keep the working dtype. */
typedef enum { DUO_KV_SAME = 0, DUO_KV_INT4_G128 = 1, DUO_KV_FP8_E4M3 = 2 } duo_kv_fmt;

typedef struct {
  int batch;           /* B >= 1                                               */
  int q_heads;         /* Hq, a multiple of kv_heads; 0 means kv_heads (MHA)   */
  duo_dtype dtype;     /* activations and K/V                                  */
  duo_kv_fmt retr_fmt; /* retrieval-head storage                               */
  float softmax_scale; /* logit scale; 0 means 1/sqrt(head_dim)                */
} duo_opts;            /* NULL opts = {1, 0, DUO_BF16, DUO_KV_SAME, 0}         */

/*
 * Bytes of device memory a cache needs: the per-layer K/V arrays (retrieval heads
 * [B][H_r][max_len][d], streaming heads [B][H_s][S+W][d]; the KV memory
 * (H_r L + H_s (S+R)) d of "Decoding Procedure" at L = max_len) plus scratch for
 * split-KV decode partials and the pre-fill staging of streaming heads.
 * Returns 0 when the arguments are invalid (same checks as duo_cache_create).
 */
DUO_API size_t duo_cache_bytes(int layers, int kv_heads, int head_dim, const uint8_t *retrieval_head_mask, int S, int W,
                       int64_t max_len, const duo_opts *opts);

/*
 * Creates a cache handle over caller-owned device memory ("Deployment
 * Architecture": two KV caches per layer, pre-allocated).
 *   layers, kv_heads      >= 1; kv_heads <= 128
 *   head_dim              64 or 128
 *   retrieval_head_mask   host [layers][kv_heads], 1 = retrieval, 0 = streaming
 *                         (the binarised gates of "Optimization-Based Retrieval
 *                         Head Identification"); copied, not kept
 *   S >= 0, W >= 1        sinks and recent window of streaming heads
 *   max_len >= 1          capacity of every retrieval head, in tokens
 *   dev_buf, dev_bytes    device buffer of >= duo_cache_bytes() bytes, 256-byte
 *                         aligned; it is zero-filled by the first call that
 *                         launches work
 * No device work happens here.  *out receives the handle.
 */
DUO_API duo_status duo_cache_create(int layers, int kv_heads, int head_dim, const uint8_t *retrieval_head_mask, int S,
                            int W, int64_t max_len, const duo_opts *opts, void *dev_buf, size_t dev_bytes,
                            duo_cache **out);

/* Frees the host handle only; the caller frees dev_buf.  NULL is a no-op. */
DUO_API void duo_cache_destroy(duo_cache *cache);

/*
 * Appends n >= 1 tokens (positions len .. len+n-1) of one layer ("Decoding
 * Procedure", step 4: update both caches).  Retrieval heads store every row
 * (INT4-quantised when configured).  Streaming heads store position p in slot p
 * when p < S, else in ring slot S + (p mod W), which evicts position p - W; of an
 * n-token append only the sinks and the last min(n, W) positions are written
 * (earlier ones would be evicted within the same call).
 *   k, v   device [B][n][Hkv][d]
 * DUO_ERR_CAPACITY if len + n > max_len.
 */
DUO_API duo_status duo_append_kv(duo_cache *cache, int layer, const void *k, const void *v, int n, void *cuda_stream);

/*
 * Chunked pre-fill of one layer ("Chunked Pre-filling", Figure 5 right): the n
 * queries at positions len .. len+n-1 attend to the layer's cache plus the
 * chunk itself -- causal mask for retrieval heads, Lambda mask for streaming heads
 * -- and the chunk is then appended as by duo_append_kv.  Launches: the staging copy
 * of the streaming heads' history (when there is any), the attention (cached positions
 * from the cache, the chunk's own keys from k and v), then the append.
 *   q, out  device [B][n][Hq][d];  k, v device [B][n][Hkv][d]
 *   lse     device [B][n][Hq] fp32, or NULL
 * DUO_ERR_UNSUPPORTED for an INT4 retrieval cache.
 */
DUO_API duo_status duo_prefill_chunk(duo_cache *cache, int layer, const void *q, const void *k, const void *v, int n,
                             void *out, float *lse, void *cuda_stream);

/*
 * Single-token decode attention of one layer ("Decoding Procedure", steps 2, 3
 * and 5): the query of the newest token, at position len-1, attends to every
 * cached token of its retrieval head, or to the sinks and ring of its streaming
 * head.  The token must have been appended first (it attends to itself).
 *   q, out  device [B][Hq][d];  lse device [B][Hq] fp32, or NULL
 * With INT4 or FP8 retrieval heads (bf16, head_dim 128) the streaming heads and the
 * retrieval heads are two launches on the stream; each writes only its own heads' rows
 * of out and lse.
 * DUO_ERR_INVALID if the layer is empty.
 */
DUO_API duo_status duo_decode_attention(duo_cache *cache, int layer, const void *q, void *out, float *lse,
                                void *cuda_stream);

/*
 * duo_append_kv of one token followed by duo_decode_attention, as one call: k, v
 * device [B][1][Hkv][d] (the token at position len), q / out / lse as for
 * duo_decode_attention ("Decoding Procedure", steps 2-4, in the order of reading R6).
 * For bf16 caches with head_dim 128 (not INT4 or FP8) and batch 1 it is one launch: the decode
 * kernel writes the token's rows into the cache itself, each by the CTA that then reads
 * the tile holding it; other caches get the append launch, then the decode launches
 * (the faster choice measured).  The cache afterwards holds exactly what duo_append_kv
 * would have written, and len advances by one.  On the two-launch path, a failure of
 * the attention launch after the append was accepted returns DUO_ERR_CUDA with the
 * token appended and len advanced (outputs not written).
 * DUO_ERR_CAPACITY if len + 1 > max_len.
 */
DUO_API duo_status duo_append_decode(duo_cache *cache, int layer, const void *q, const void *k, const void *v,
                                     void *out, float *lse, void *cuda_stream);

/* Tokens in a layer's cache (host value, no synchronisation). */
DUO_API duo_status duo_cache_len(const duo_cache *cache, int layer, int64_t *len);

/*
 * KV memory of the configured cache at sequence length L, in bytes of K plus V:
 * *retained = what the hybrid cache keeps, (H_r L + H_s min(L, S+W)) d per layer
 * ("Decoding Procedure"), INT4 codes and scale/zero counted when configured;
 * *full = what full attention would keep in the working dtype, 2 D H L d elements
 * ("The Core Problem").  Either pointer may be NULL.
 */
DUO_API duo_status duo_kv_bytes(const duo_cache *cache, int64_t L, uint64_t *retained, uint64_t *full);

/*
 * Position held by a cache slot of one KV head, from the host's bookkeeping
 * (no device access): retrieval heads hold position `slot` iff slot < len;
 * streaming heads follow the slot rule of duo_append_kv.  *pos = -1 when empty.
 */
DUO_API duo_status duo_debug_slot_position(const duo_cache *cache, int layer, int kv_head, int slot, int64_t *pos);

/*
 * Device address and size of one storage array of a layer, for inspection and
 * tests (no device access).  which:
 *   DUO_REGION_RETR_K / _RETR_V   retrieval heads [B][H_r][cap][row], row = d
 *                                 elements, or d/2 code bytes for INT4, d for FP8
 *   DUO_REGION_RETR_KSZ / _VSZ    INT4: [B][H_r][cap][2] fp16 (scale, zero);
 *                                 FP8: [B][H_r][cap] fp32 scale
 *   DUO_REGION_STRM_K / _STRM_V   streaming heads [B][H_s][S+W][d]
 * Heads of a kind are in increasing KV-head order.  *cap receives the token stride
 * of retrieval arrays (max_len rounded up to a multiple of 256).  Any output
 * pointer may be NULL.  An array with no heads reports 0 bytes.
 */
typedef enum {
  DUO_REGION_RETR_K = 0,
  DUO_REGION_RETR_V = 1,
  DUO_REGION_RETR_KSZ = 2,
  DUO_REGION_RETR_VSZ = 3,
  DUO_REGION_STRM_K = 4,
  DUO_REGION_STRM_V = 5
} duo_region;
DUO_API duo_status duo_debug_region(const duo_cache *cache, int layer, duo_region which, void **ptr, uint64_t *bytes,
                                    int64_t *cap);

/*
 * Synchronises `cuda_stream`, reads and clears the device status word.
 * DUO_ERR_TIMEOUT if a kernel's bounded wait ran out since the last check.
 */
DUO_API duo_status duo_get_device_status(duo_cache *cache, void *cuda_stream);

/*
 * duo_decode_attention for callers that cannot allocate device memory when they
 * decode -- for instance a serving runtime whose device memory belongs to a pool it
 * sized once at start-up (every further cudaMalloc fails or fragments that pool), or
 * a caller with a fixed memory budget that must not grow while it runs.  The paper has
 * no counterpart: this is a property of the library, not of the method.
 *
 * Same arguments, layouts and result as duo_decode_attention.  It calls no cudaMalloc,
 * cudaFree or allocating library routine and does not use the scratch area of the
 * cache buffer: the split-KV partial results and merge tickets go to one 4 MiB array
 * of static device memory that every GPU which loads this library holds until the
 * process exits.  The tickets are cleared (cudaMemsetAsync on `cuda_stream`) at every
 * call; the rest of the array keeps the previous call's contents, so calls that
 * overlap on the GPU (other streams, other threads) race and must be ordered by the
 * caller.  The first call on each device looks up the array's device address with
 * cudaGetSymbolAddress, with that device current, and keeps it for the life of the
 * process; make that first call before any stream capture.  After cudaDeviceReset on
 * a device the kept address is stale: do not call this entry point on that device again
 * in the same process.
 * Limits: bf16 caches with head_dim 128, not INT4 or FP8, at most 16 query heads per KV head
 * (else DUO_ERR_UNSUPPORTED).  The partials of B*kv_heads heads must fit the array at
 * one CTA: B*kv_heads*G*(head_dim+4)*4 bytes <= 4 MiB less the tickets, else
 * DUO_ERR_CAPACITY; larger head counts still fit but run on fewer CTAs.  The refusal is
 * kept even though a single CTA would need no scratch: such a cache would decode on one
 * SM, over a hundred times slower than duo_decode_attention, and the caller should know
 * the size is past what this entry point serves.
 */
DUO_API duo_status duo_decode_attention_static_scratch(duo_cache *cache, int layer, const void *q, void *out,
                                                       float *lse, void *cuda_stream);

/*
 * ---- Paged pool of sequences: ragged batching ----
 *
 * Sequences of different lengths share one caller-owned buffer (the pages name batched
 * serving, and how the dual cache fits paged memory management, as open questions:
 * "Critical Assessment").  Retrieval heads keep K/V in pages of 128 tokens: page p of
 * layer l is [H_r(l)][128][d] and holds the same 128 positions of one sequence for all
 * of the layer's retrieval heads; a sequence's logical page i is physical page
 * table[slot][i] on every layer (a block table in the buffer, kept by the library).
 * Streaming heads keep their sinks + ring per sequence slot, [slot][H_s][S+W][d], with
 * the slot rule of duo_append_kv.  The host keeps every sequence's length per layer.
 * bf16, head_dim 128, retrieval format DUO_KV_SAME, at most 16 query heads per KV head
 * (else DUO_ERR_UNSUPPORTED).  Sequences are filled with duo_pool_append_kv and decoded
 * with duo_pool_decode_step; pre-fill attention over a pool is not provided.  Calls on
 * one pool must be ordered on one stream.  Errors follow the cache's contract: checked
 * before any launch, lengths follow what the cache holds.
 */
typedef struct duo_pool duo_pool;

/* Bytes of the pool buffer: max_seqs sequence slots, num_pages pages per layer, every
 * sequence at most max_len tokens.  0 for invalid arguments. */
DUO_API size_t duo_pool_bytes(int layers, int kv_heads, int head_dim, const uint8_t *retrieval_head_mask, int S, int W,
                              int max_seqs, int64_t max_len, int64_t num_pages, const duo_opts *opts);

/* Creates a pool over caller-owned device memory (>= duo_pool_bytes(), 256-byte
 * aligned; the first launching call clears it).  opts->batch is ignored.  No device
 * work happens here. */
DUO_API duo_status duo_pool_create(int layers, int kv_heads, int head_dim, const uint8_t *retrieval_head_mask, int S,
                                   int W, int max_seqs, int64_t max_len, int64_t num_pages, const duo_opts *opts,
                                   void *dev_buf, size_t dev_bytes, duo_pool **out);
DUO_API void duo_pool_destroy(duo_pool *pool); /* host handle only */

/* Opens a sequence in a free slot (*seq), length 0 on every layer; its sink / ring rows
 * are cleared on `cuda_stream`.  DUO_ERR_CAPACITY when every slot is open. */
DUO_API duo_status duo_pool_open(duo_pool *pool, void *cuda_stream, int *seq);
/* Closes a sequence: its pages return to the pool, its slot can be opened again. */
DUO_API duo_status duo_pool_close(duo_pool *pool, int seq);
DUO_API duo_status duo_pool_len(const duo_pool *pool, int seq, int layer, int64_t *len);
DUO_API duo_status duo_pool_free_pages(const duo_pool *pool, int64_t *pages);

/* Appends n >= 1 tokens (k, v [n][Hkv][d]) to one sequence on one layer, as
 * duo_append_kv does for a cache: every retrieval row into the sequence's pages (new
 * pages are taken from the pool; the rest of a page the call opens is cleared), sinks and
 * the last min(n, W) positions into the ring.  DUO_ERR_CAPACITY past max_len or when
 * the pool has too few free pages. */
DUO_API duo_status duo_pool_append_kv(duo_pool *pool, int layer, int seq, const void *k, const void *v, int n,
                                      void *cuda_stream);

/*
 * One decode step of a ragged batch: for each of the nseq listed sequences (host array
 * `seqs`, distinct, open) and each layer layer0 .. layer0+nlayers-1, append the token
 * (k, v [nlayers][nseq][Hkv][d]) at the sequence's length, then attend with its query
 * (q [nlayers][nseq][Hq][d]) over that layer's cache ("Decoding Procedure", steps 2-5),
 * writing out [nlayers][nseq][Hq][d] and lse [nlayers][nseq][Hq] (fp32, or NULL).  Two
 * launches whatever nlayers and nseq: the append of every (layer, sequence, KV head),
 * then one tcgen05 decode over all of them, each sequence at its own length.  Several
 * layers in one call serve callers that hold the queries of those layers together (in
 * a model, layer l+1's query depends on layer l's output, so a model step makes one call
 * per layer).  A listed sequence must have the same length on every listed layer.
 * nseq <= 128, nlayers * nseq <= 1024.  DUO_ERR_CAPACITY past max_len or without free
 * pages; as for duo_append_decode, a failed attention launch leaves the tokens appended.
 */
DUO_API duo_status duo_pool_decode_step(duo_pool *pool, int layer0, int nlayers, int nseq, const int *seqs,
                                        const void *q, const void *k, const void *v, void *out, float *lse,
                                        void *cuda_stream);

/* Physical page of a sequence's logical page (host bookkeeping, for inspection). */
DUO_API duo_status duo_pool_page(const duo_pool *pool, int seq, int logical_page, int *physical_page);
/* Device address and size of a layer's page array (DUO_REGION_RETR_K / _V,
 * [pages][H_r][128][d]) or streaming array (DUO_REGION_STRM_K / _V, [slots][H_s][S+W][d]). */
DUO_API duo_status duo_pool_region(const duo_pool *pool, int layer, duo_region which, void **ptr, uint64_t *bytes);
/* Synchronises `cuda_stream`, reads and clears the pool's device status word. */
DUO_API duo_status duo_pool_device_status(duo_pool *pool, void *cuda_stream);

/*
 * Gated mixed attention of the identification phase ("Gate Parameterization"): over
 * whole sequences (positions 0..L-1, no cache), the output of every query head of KV
 * head g is
 *     alpha[g] * full_attn + (1 - alpha[g]) * streaming_attn
 * with full_attn under the causal mask and streaming_attn under the Lambda mask of
 * sinks S and window W ("The Full and Streaming Attention Masks"; same mask reading as
 * the cache calls).  Training the gates is not part of this library.
 *   q, out   device [B][L][Hq][d];  k, v  device [B][L][Hkv][d]  (dtype bf16 or fp32)
 *   alpha    device [Hkv] fp32, one gate per KV head (values outside [0, 1] are used
 *            as given)
 *   softmax_scale  0 means 1/sqrt(head_dim)
 * Two launches on `cuda_stream`, both reading q, k and v where they are (no copy, no
 * scratch): the causal term is written to `out`, then the Lambda term is computed and
 * each row of `out` becomes alpha * out + (1 - alpha) * streaming.  Arguments are
 * checked before any launch (DUO_ERR_INVALID).
 */
DUO_API duo_status duo_gated_attention(const void *q, const void *k, const void *v, int batch, int seq_len,
                                       int q_heads, int kv_heads, int head_dim, duo_dtype dtype, const float *alpha,
                                       int S, int W, float softmax_scale, void *out, void *cuda_stream);

/*
 * Test controls of the host-side bookkeeping, process-wide and not thread-safe (tests
 * only; the paper has no counterpart).
 *   dry_run     1: no call touches a device -- the first-use clear of a cache buffer and
 *               every kernel launch are skipped and reported as accepted -- so that
 *               argument checks, lengths and the error contract above can be exercised
 *               on a machine without a GPU; 0: normal operation.
 *   fail_after  >= 0: the launch attempt number fail_after + 1, counted from this call,
 *               is not made and reports a launch failure (the call returns
 *               DUO_ERR_CUDA); -1: off.
 * DUO_ERR_INVALID for other values.
 */
DUO_API duo_status duo_debug_launch_controls(int dry_run, int64_t fail_after);

/*
 * Test control of the device-side timeout path, process-wide (tests only; the paper has
 * no counterpart).  on = 1: every bf16 tensor-core decode of a contiguous cache
 * (duo_decode_attention, duo_append_decode, and the streaming heads of an INT4 or FP8
 * layer) makes its softmax warps wait first for a barrier that nothing arrives at.  That
 * bounded wait runs out after about 2 s; the kernel latches DUO_ERR_TIMEOUT in the
 * cache's status word (read by duo_get_device_status), every role of every CTA stops
 * waiting, drains its copies and products and exits, and the call's outputs are
 * undefined.  The CUDA context stays usable.  on = 0: normal operation.
 * DUO_ERR_INVALID for other values.
 */
DUO_API duo_status duo_debug_device_stall(int on);

/* Static description of a status code. */
DUO_API const char *duo_status_str(duo_status status);

#ifdef __cplusplus
}
#endif

#endif /* DUO_H */
