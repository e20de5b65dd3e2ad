/*
 * hca.h -- C ABI of libhca: Heavily Compressed Attention (HCA) on sm_100a.
 *
 * The operation (sources are two pages about ERNIE-5.5-Flash-Base):
 *   [news 二.1]     "280B总参数、14B激活！百度开源文心5.5 Flash Base" (aitest123.com),
 *                   section 二.1 "Latent-Gated Sparse Attention": an HCA layer stores one
 *                   cache entry per 128 tokens and attends only to those entries plus a
 *                   window of the most recent uncompressed tokens.
 *   [analysis 1]    "百度 ERNIE 5.5 Flash Base 完整解析" (communeify.com), architecture item 1
 *                   (HCA): 128 consecutive tokens become one entry, the layer attends to all
 *                   compressed history entries and a short window of recent raw tokens, and
 *                   its heads are 512 wide.
 *   [gate]          both pages, "Low-Rank Gated Attention" paragraph: the attention output
 *                   is multiplied by a learned gate.
 *
 * Readings where the pages are silent: mean pooling over the tokens present in a block;
 * window = the last `window` tokens up to and including the query; compressed entry j is
 * visible to position t iff (j+1)*block <= t+1-window (blocks that end before the window);
 * one softmax over both key sets; the gate arrives already passed through the sigmoid.
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned DEVICE memory unless stated; the library allocates
 *     nothing, keeps no global state between calls (the one exception is the fixed
 *     scratch array behind hca_attn_decode_noalloc, below), and never frees caller memory.
 *   - Layouts are dense row-major with head_dim innermost:
 *       Q, O        [batch, seqlen, hq,  head_dim]
 *       K, V        [batch, seqlen, hkv, head_dim]
 *       cache pools [num_pages, page_entries, hkv, head_dim]
 *     Element type is desc->dtype (HCA_BF16 or HCA_F32) for all of them; LSE is float32.
 *   - The bf16 tensor-core paths read and write through TMA and vector accesses: Q, K, V, O,
 *     the cache pools and the gate must start on a 16-byte boundary (HCA_EINVAL otherwise).
 *     Prefill writes O with 32-byte stores when O starts on a 32-byte boundary (faster;
 *     same result).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and the
 *     call returns before it runs. The return value reports argument validation and
 *     launch failures only. Kernels that meet an out-of-range page id or a cache holding
 *     fewer entries than a query needs skip that access and OR a bit into *cache->err_word
 *     (if non-NULL); the caller reads it after synchronising.
 *   - No entry point throws across the ABI or aborts the process.
 */
#ifndef HCA_H_
#define HCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t, declared here so this header needs no CUDA header. */
typedef struct CUstream_st* hca_stream_t;

typedef enum {
  HCA_OK = 0,
  HCA_EINVAL = -1,        /* NULL pointer, negative size, inconsistent shapes */
  HCA_EUNSUPPORTED = -2,  /* valid HCA problem that this build has no kernel for */
  HCA_ENOSPACE = -3,      /* cache pages or workspace too small for the request */
  HCA_ECUDA = -4          /* a CUDA runtime/driver call failed (launch, tensor map) */
} hca_status;

typedef enum { HCA_BF16 = 0, HCA_F32 = 1 } hca_dtype;

/* Bits OR-ed into *hca_cache.err_word by kernels. */
#define HCA_ERR_PAGE_RANGE 1   /* a page-table entry outside [0, num_pages) was skipped */
#define HCA_ERR_CACHE_SHORT 2  /* a query needed more entries than n_entries[b] holds */
#define HCA_ERR_TIMEOUT 4      /* a kernel gave up waiting on one of its own pipeline stages
                                  (bits 8 and up then name the stage); outputs are invalid */
#define HCA_ERR_CTX_RANGE 8    /* decode: a ctx_len[b] outside [1, seqlen] was clamped into it */

/* Problem description. Plain data filled by the caller; copied by value into launches. */
typedef struct {
  int32_t batch;       /* sequences in the call (prefill: b; decode: number of sequences) */
  int32_t seqlen;      /* prefill: tokens per sequence T. decode: largest context length in
                          the batch (bounds the split count and the workspace size) */
  int32_t hq;          /* query heads (64 in the pages' model) */
  int32_t hkv;         /* key/value heads; hq % hkv == 0; query head h reads kv head h*hkv/hq */
  int32_t head_dim;    /* 512 in [analysis 1] */
  int32_t block;       /* tokens pooled into one entry: 128 in [news 二.1] */
  int32_t window;      /* raw tokens each query sees, itself included (reading: 128) */
  float scale;         /* softmax scale applied to q.k (reading: 1/sqrt(head_dim)) */
  int32_t dtype;       /* hca_dtype of Q, K, V, O, the pools, the ring and the gate */
  int32_t decode_splits; /* decode only: key-range splits per sequence, 0 = automatic */
  const void* gate;    /* optional gate G (post-sigmoid), dtype as above; NULL = no gate.
                          Set through hca_set_gate. */
  int64_t gate_strides[3]; /* element strides of G: prefill [batch, token, head];
                              decode [sequence, unused, head]; head_dim is contiguous */
} hca_desc;

/* Element format of the compressed pools (hca_cache.pool_format). */
typedef enum {
  HCA_POOL_NATIVE = 0,  /* the pools hold desc->dtype elements */
  HCA_POOL_E4M3 = 1     /* 8-bit cache of [serve fp8]: one e4m3 code per element */
} hca_pool_format;

/* [serve fp8]: the communeify.com page ("百度 ERNIE 5.5 Flash Base 完整解析"), section
 * "本地部署與推論實戰指南" item 3, serves the model with an 8-bit KV cache
 * (`--kv-cache-dtype fp8`). Readings where it is silent: the compressed pools are what is
 * stored in 8 bits (the raw window ring stays in desc->dtype); the element format is e4m3
 * of the OCP 8-bit floating-point specification (bias 7, subnormals, no infinities, largest
 * finite 448); one float32 scale per pool: stored code = e4m3(entry / scale), value read
 * back = value(code) * scale. */

/* Paged compressed-KV cache. Entry j of sequence b lives in pool row
 *   page_table[b * max_pages + j / page_entries] * page_entries + j % page_entries. */
typedef struct {
  void* kc_pool;              /* [num_pages, page_entries, hkv, head_dim] */
  void* vc_pool;              /* same shape */
  const int32_t* page_table;  /* device [batch, max_pages] */
  int32_t* n_entries;         /* device [batch]; hca_compress stores first_block + n_blocks */
  int32_t page_entries;       /* entries per page; the bf16 kernels need a multiple of 128 */
  int32_t max_pages;          /* columns of page_table */
  int32_t num_pages;          /* pages in each pool */
  int32_t* err_word;          /* optional device int32 error bits (HCA_ERR_*), may be NULL */
  int32_t pool_format;        /* hca_pool_format; 0 (native) for a zero-initialised struct */
  float k_scale;              /* HCA_POOL_E4M3: Kc value = value(code) * k_scale (finite, > 0) */
  float v_scale;              /* HCA_POOL_E4M3: Vc value = value(code) * v_scale (finite, > 0) */
} hca_cache;

/* ABI version of this header (bumped on any layout change of the structs above). */
#define HCA_ABI_VERSION 2
int32_t hca_abi_version(void);

/* Human-readable name of a status code. Static string, never NULL. */
const char* hca_status_string(int32_t status);

/* Attach (gate != NULL) or detach (gate == NULL) the output gate of [gate].
 * Host-only: writes d->gate and d->gate_strides; no device work. `strides` (3 elements)
 * may be NULL only when gate is NULL.
 * Returns HCA_EINVAL for d == NULL or a non-NULL gate without strides. */
int32_t hca_set_gate(hca_desc* d, const void* gate, const int64_t* strides);

/* Block compression of [news 二.1] / [analysis 1] (mean pooling, the reading above).
 * For every sequence b < d->batch and block j in [first_block, first_block + n_blocks):
 *   Kc[j] = mean of K rows of tokens [j*block, min((j+1)*block, d->seqlen)), same for V,
 * accumulated in float32 and rounded once to d->dtype, stored into the cache pools at the
 * row the page table gives; then n_entries[b] = first_block + n_blocks.
 * An HCA_POOL_E4M3 cache ([serve fp8]) stores instead the code e4m3(mean / scale): the
 * float32 mean divided by k_scale (Kc) or v_scale (Vc) in float32, rounded to the nearest
 * e4m3 value (ties to even) with magnitudes of 448 and more stored as 448. Pool rows are
 * then hkv * head_dim bytes.
 * K, V point at the first token of block `first_block` of sequence 0; the token rows of
 * sequence b start `b * batch_stride_tokens` token rows later (prefill: batch_stride_tokens
 * = seqlen with K advanced by first_block*block rows; a decode ring of `block` slots:
 * batch_stride_tokens = block).
 * Errors: HCA_EINVAL (NULL pointer, n_blocks < 0, first_block < 0, a block starting at or
 * past seqlen), HCA_ENOSPACE (first_block + n_blocks > max_pages * page_entries),
 * HCA_EUNSUPPORTED (head_dim not a multiple of 8), HCA_ECUDA. An HCA_POOL_E4M3 cache also
 * gives HCA_EINVAL for a scale that is not finite and positive, and an unknown pool_format
 * gives HCA_EINVAL on every entry point. */
int32_t hca_compress(const hca_desc* d, const void* K, const void* V,
                     int64_t batch_stride_tokens, int32_t first_block, int32_t n_blocks,
                     const hca_cache* cache, hca_stream_t stream);

/* Decode-step update of the raw window ([news 二.1]: the last `window` raw tokens are
 * attended as they are; the decode path keeps them in a ring, token u in slot u % window).
 * For every sequence b < d->batch the new token, at position t = ctx_len[b] - 1:
 *   ring_k[b, t % window] = new_k[b],   ring_v[b, t % window] = new_v[b]
 *   new_k, new_v    [batch, hkv, head_dim]          d->dtype, contiguous
 *   ring_k, ring_v  [batch, window, hkv, head_dim]  d->dtype, contiguous
 *   ctx_len         device int32 [batch], as passed to hca_attn_decode (clamped into
 *                   [1, seqlen] the same way, so both agree on the slot)
 * One launch for both rows of every sequence; run it before hca_attn_decode of the step
 * (and before hca_compress of a block the token completes).
 * Errors: HCA_EINVAL (NULL pointer, a pointer not 16-byte aligned), HCA_EUNSUPPORTED
 * (hkv * head_dim * element size not a multiple of 16 bytes), HCA_ECUDA. */
int32_t hca_ring_append(const hca_desc* d, const void* new_k, const void* new_v,
                        const int32_t* ctx_len, void* ring_k, void* ring_v,
                        hca_stream_t stream);

/* HCA prefill attention of [news 二.1] / [analysis 1] with the optional gate of [gate].
 * For every sequence b, position t < seqlen and head h:
 *   keys  = compressed entries j < n_c(t) of sequence b, then raw tokens u in
 *           [max(0, t-window+1), t];  n_c(t) = max(0, floor((t+1-window)/block))
 *   O[b,t,h] = softmax(scale * q . keys) . values  (one softmax over both sets)
 *   O[b,t,h] *= G[b,t,h] when a gate is attached
 *   lse[b,t,h] = natural log of the softmax denominator incl. the max (if lse != NULL)
 *   dbg_mask[(b*seqlen+t)*3 + {0,1,2}] = (n_c(t), window lo, window hi) (if non-NULL)
 * Compressed entries are read from `cache` (hca_compress must have written them); an
 * HCA_POOL_E4M3 cache gives HCA_EUNSUPPORTED here and in the backward (the 8-bit cache
 * serves decode).
 * Kernels: bf16 -> tcgen05/TMEM tensor-core kernels (need head_dim 512, hkv 1, hq in
 * {8,16,32,64,128}, window <= 128, page_entries % 128 == 0, batch*seqlen*hq and
 * num_pages*page_entries below 2^31). hq >= 16 runs on clusters of two CTAs sharing the
 * 2-SM UMMA (each SM loads half of every K/V tile; needs (batch*seqlen + 256)*hq below
 * 2^31, else the one-CTA kernel runs); hq = 8 on one CTA per tile. f32 -> CUDA-core kernel
 * (head_dim % 32 == 0, head_dim <= 512, any block/window).
 * Errors: HCA_EINVAL, HCA_EUNSUPPORTED, HCA_ECUDA. */
int32_t hca_attn_prefill(const hca_desc* d, const void* Q, const void* K, const void* V,
                         const hca_cache* cache, void* O, float* lse, int32_t* dbg_mask,
                         hca_stream_t stream);

/* Prefill of a contiguous range of query positions: the operation of hca_attn_prefill for
 * positions q_pos0 .. q_pos0 + d->seqlen - 1 of every sequence, with the key/value tokens
 * given as a range too. It serves chunked prefill and the split of one long sequence's
 * query rows over several GPUs (each GPU holds its own rows plus a window-1 token halo).
 *   Q, O     [batch, d->seqlen, hq, head_dim]   rows of positions q_pos0 + t
 *   lse      [batch, d->seqlen, hq];  dbg_mask [batch, d->seqlen, 3] (values are positions)
 *   gate     rows aligned with Q (token stride over the d->seqlen rows)
 *   K, V     [batch, kv_len, hkv, head_dim]     rows of positions kv_pos0 + u; they must
 *            cover every window: kv_pos0 <= max(0, q_pos0 - window + 1) and
 *            kv_pos0 + kv_len >= q_pos0 + d->seqlen
 *   cache    compressed entries by absolute block index (entry j = block j of the sequence)
 * hca_attn_prefill(d, ...) is hca_attn_prefill_range(d, 0, 0, d->seqlen, ...).
 * Kernels and support as hca_attn_prefill (also needs batch * kv_len below 2^31 for bf16).
 * Errors: HCA_EINVAL (also: negative positions, K/V rows that miss a window),
 * HCA_EUNSUPPORTED, HCA_ECUDA. */
int32_t hca_attn_prefill_range(const hca_desc* d, int32_t q_pos0, int32_t kv_pos0,
                               int32_t kv_len, const void* Q, const void* K, const void* V,
                               const hca_cache* cache, void* O, float* lse, int32_t* dbg_mask,
                               hca_stream_t stream);

/* Bytes of device workspace hca_attn_prefill_backward needs for d (0 if d is invalid). */
size_t hca_prefill_backward_workspace_bytes(const hca_desc* d);

/* Gradients of hca_attn_prefill for the training context of the pages ([analysis infra 3]:
 * the communeify.com page, section "33.5T 預訓練資料工程與分散式訓練基礎設施" item 3, quotes
 * the backward kernel of this operator; the pages print no formulas, so these are the exact
 * derivatives of the forward definition above). Given the forward's inputs, its lse and
 * the output gradient dO, per row (b, t, h) with visible keys k_i and values v_i,
 * p_i = exp(scale q.k_i - lse) and the ungated output O_pre = sum_i p_i v_i:
 *   dG  = dO * O_pre                          (the gate's gradient; gate attached only)
 *   dO' = dO * G (dO without a gate),  Delta = dO' . O_pre,  dp_i = dO' . v_i
 *   ds_i = p_i (dp_i - Delta),  dq = scale sum_i ds_i k_i
 *   dk_i += scale ds_i q,  dv_i += p_i dO'     (summed over every row that sees key i)
 * and each token of block j receives 1/count_j of the gradient of entry j (the entry is the
 * mean of its block's count_j tokens), on top of its window gradient.
 *   Q, dO, dQ, dG  [batch, seqlen, hq, head_dim];  K, V, dK, dV [batch, seqlen, hkv, head_dim]
 *   lse [batch, seqlen, hq] float32 (natural log, as hca_attn_prefill writes it)
 *   cache: the compressed entries the forward used (hca_compress of K, V)
 *   dG must be non-NULL exactly when d->gate is attached (G > 0, as a sigmoid is).
 * O_pre is recomputed in float32 from Q, K, V and lse rather than read from the stored
 * output: a bf16 output carries 2^-9 of |O| of rounding, which Delta (a sum over head_dim
 * of dO' * O_pre) and dG would inherit.
 * dQ, dK, dV, dG are written (not accumulated), in d->dtype. workspace: device memory of
 * hca_prefill_backward_workspace_bytes(d) bytes, 16-byte aligned, contents ignored.
 * Kernels: bf16 with head_dim 512, hkv 1, window <= 128, hq <= 128 -> the contractions on
 * tcgen05 tensor cores (groups of 1024 query positions: the scores, dP, P and dS of a group
 * are held in the workspace, P, dS and dO * G enter the products as bf16 pairs hi + lo);
 * otherwise (float32, other shapes) CUDA cores with float32 arithmetic (head_dim % 32 == 0,
 * head_dim <= 512). batch * seqlen * hq below 2^31. The bf16 path's 16-byte alignment rule
 * applies to its tensors.
 * Errors: HCA_EINVAL, HCA_EUNSUPPORTED, HCA_ENOSPACE, HCA_ECUDA. */
int32_t hca_attn_prefill_backward(const hca_desc* d, const void* Q, const void* K,
                                  const void* V, const hca_cache* cache,
                                  const float* lse, const void* dO, void* dQ, void* dK,
                                  void* dV, void* dG, void* workspace, size_t workspace_bytes,
                                  hca_stream_t stream);

/* The output gate from the attention layer's low-rank query latent ([news 二.1] and
 * [analysis 1], "Low-Rank Gated Attention": the gate is computed from the query latent, a
 * quarter of the hidden width, instead of the hidden state). Reading: one gate value per
 * output element,
 *   G[r, h, e] = sigmoid(sum_i q_lat[r, i] W_g[i, h * head_dim + e]),
 * for the d->batch * d->seqlen rows r of q_lat [rows, latent] (bf16) and W_g
 * [latent, hq * head_dim] (bf16); G [rows, hq, head_dim] bf16 -- the layout hca_set_gate
 * expects. Runs as one tcgen05 GEMM with the sigmoid in its epilogue.
 * Errors: HCA_EINVAL, HCA_EUNSUPPORTED (f32; latent or hq * head_dim not a multiple of 8),
 * HCA_ECUDA. */
int32_t hca_gate_from_latent(const hca_desc* d, const void* q_lat, const void* W_g,
                             int32_t latent, void* G, hca_stream_t stream);

/* The layer's attention output with Virtual Head Attention ([news 二.1] and [analysis 1],
 * "Virtual Head Attention": after the attention computation, a light cross-head low-rank
 * mixing with an identity skip), then the gate of d if attached. Reading, per position p
 * (d->batch * d->seqlen positions) and column e:
 *   z_r = sum_g B[g, r] O[p, g, e],   out[p, h, e] = (O[p, h, e] + sum_r A[h, r] z_r) * G[p, h, e]
 *   O, out  [batch, seqlen, hq, head_dim] in d->dtype: O the heads' ungated attention outputs
 *           (hca_attn_prefill / hca_attn_decode run with no gate attached)
 *   A, B    [hq, rank] float32 device arrays, 0 <= rank <= 16 (rank 0: the gate alone)
 * Errors: HCA_EINVAL, HCA_EUNSUPPORTED (rank > 16, hq > 128, head_dim % 4 or > 512),
 * HCA_ECUDA. */
int32_t hca_vha_gate(const hca_desc* d, const void* O, const float* A, const float* B,
                     int32_t rank, void* out, hca_stream_t stream);

/* Bytes of device workspace hca_attn_decode needs for `d` (split partials of O, max and
 * sum). 0 if d is invalid. */
size_t hca_decode_workspace_bytes(const hca_desc* d);

/* One HCA decode step for d->batch sequences ([news 二.1]; the query is the newest token).
 *   Q        [batch, hq, head_dim]   query of the new token of each sequence
 *   ctx_len  device int32 [batch]    context length including the new token; the query
 *                                    position is t = ctx_len - 1, 1 <= ctx_len <= seqlen;
 *                                    a value outside is clamped into that range and sets
 *                                    HCA_ERR_CTX_RANGE in *cache->err_word
 *   ring_k/v [batch, window, hkv, head_dim]  raw tokens; token u sits in slot u % window
 *   O        [batch, hq, head_dim];  lse [batch, hq] float32 (optional)
 * Keys are exactly the prefill key set of position t. The key list is cut into splits
 * (d->decode_splits, 0 = automatic), each split writes float32 partial (O, max, sum) into
 * `workspace`, and a merge kernel combines them, applies the gate and casts.
 * Kernels: bf16 -> tcgen05/TMEM kernel (head_dim 512, hkv 1, hq <= 64, window <= 128,
 * page_entries % 128 == 0, num_pages*page_entries below 2^31); f32 -> CUDA-core kernel.
 * An HCA_POOL_E4M3 cache ([serve fp8]; bf16 only, same shape limits) runs the 8-bit
 * kernel: the compressed keys enter q.k as e4m3 codes (the query is carried exactly as two
 * e4m3 parts per element with a power-of-two scale per head), the compressed values are
 * widened to f16 (exact), the scales apply in float32, and the raw window runs in bf16 as
 * above; the result is that of the decode above over the dequantised entries
 * value(code) * scale. The same holds for hca_attn_decode_partial and
 * hca_attn_decode_noalloc.
 * Errors: HCA_EINVAL, HCA_EUNSUPPORTED, HCA_ENOSPACE (workspace_bytes too small),
 * HCA_ECUDA. */
int32_t hca_attn_decode(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                        const hca_cache* cache, const void* ring_k, const void* ring_v,
                        void* O, float* lse, void* workspace, size_t workspace_bytes,
                        hca_stream_t stream);

/* hca_ring_append and hca_attn_decode in one call ([news 二.1]): the new token's rows
 * new_k, new_v [batch, hkv, head_dim] go into ring slot (ctx_len[b] - 1) % window (ctx_len
 * clamped as hca_attn_decode clamps it), then the decode step runs over the updated rings.
 * The bf16 tensor-core kernels write the two rows from the CTA that reads the window, just
 * before it reads it, so the step needs no separate launch; other paths run the two calls.
 * Arguments and errors as hca_attn_decode, plus HCA_EINVAL for a NULL or not 16-byte
 * aligned new_k / new_v. A block the new token completes is compressed after this call
 * (its entry is not visible to the token's own query). */
int32_t hca_attn_decode_append(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                               const hca_cache* cache, const void* new_k, const void* new_v,
                               void* ring_k, void* ring_v, void* O, float* lse,
                               void* workspace, size_t workspace_bytes, hca_stream_t stream);

/* Bytes of one decode partial result for d (bf16 paths; 0 if d is invalid or f32). */
size_t hca_decode_partial_bytes(const hca_desc* d);

/* One decode step over a part of every sequence's key list, for splitting a long context
 * over several GPUs ([news 二.1]: the keys are the compressed entries and the window; one
 * softmax over all of them is the same as a log-sum-exp combination of softmaxes over
 * disjoint parts). The part is the visible compressed entries j with
 * entry_begin <= j < entry_end (entry_begin a multiple of 128), plus the raw window when
 * with_window != 0. Instead of O it writes, into `partial` (hca_decode_partial_bytes(d)
 * bytes of device memory, 16-byte aligned), float32 data laid out as
 *   ml [batch, hq, 2]   (m, l), padded to a multiple of 4 floats, then
 *   o  [batch, hq, head_dim]
 * with s_i = scale * q . k_i * log2(e) over the part's keys: l = sum_i 2^(s_i - m) and
 * o = sum_i 2^(s_i - m) v_i for a reference m near max_i s_i. A part holding no key has
 * l = 0 (m and o are then unspecified). No gate is applied. workspace: as for
 * hca_attn_decode; hca_decode_workspace_bytes(d) bytes always suffice (a part that fits one
 * split per sequence needs none).
 * Errors: HCA_EINVAL (also: entry_begin not a multiple of 128, entry_end < entry_begin),
 * HCA_EUNSUPPORTED (f32, or shapes the bf16 decode does not run), HCA_ENOSPACE, HCA_ECUDA. */
int32_t hca_attn_decode_partial(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                                const hca_cache* cache, const void* ring_k, const void* ring_v,
                                int32_t entry_begin, int32_t entry_end, int32_t with_window,
                                void* partial, void* workspace, size_t workspace_bytes,
                                hca_stream_t stream);

/* The decode output from n_parts partial results of disjoint key parts that together make
 * up each sequence's key set (part k at parts + k * part_stride bytes, each laid out as
 * above): per sequence and head, M = max m_k over the parts with l_k > 0,
 *   O = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k,
 * times the gate of d if attached, rounded to bf16; lse (optional, [batch, hq] float32)
 * = (M + log2 sum_k 2^(m_k - M) l_k) ln 2. At least one part of every sequence must hold a
 * key. part_stride: a multiple of 16, at least hca_decode_partial_bytes(d) when n_parts > 1.
 * Errors: HCA_EINVAL, HCA_EUNSUPPORTED (f32, head_dim != 512, hq > 64), HCA_ECUDA. */
int32_t hca_decode_merge(const hca_desc* d, const void* parts, int32_t n_parts,
                         int64_t part_stride, void* O, float* lse, hca_stream_t stream);

/* Bytes of device memory the library keeps for hca_attn_decode_noalloc (64 MiB). */
#define HCA_DECODE_NOALLOC_SCRATCH_BYTES (64u << 20)

/* hca_attn_decode without a caller-provided workspace. The pages have no counterpart to
 * this entry point: it exists for callers that cannot give the library device memory --
 * their memory is owned by another allocator (a framework's caching pool, or a serving
 * engine that reserves all of HBM at start-up), or their decode loop must not call the CUDA
 * allocator, whose cudaMalloc/cudaFree can synchronise the device.
 * Same arguments and results as hca_attn_decode minus workspace/workspace_bytes, bf16 only.
 * The split partials go to a fixed HCA_DECODE_NOALLOC_SCRATCH_BYTES array inside the
 * library, allocated on every GPU that loads the library's device code and held until the
 * process exits. It allocates nothing, and calls no cudaMalloc or cudaFree.
 *   - The first call on a device looks up the array's device address (once per device, with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; nothing in it needs
 *     to start at zero. Calls whose work overlaps on the GPU (different streams or host
 *     threads) race on it: serialise them.
 * Errors: as hca_attn_decode; HCA_ENOSPACE when the partials this call needs
 * (hca_decode_workspace_bytes(d)) exceed HCA_DECODE_NOALLOC_SCRATCH_BYTES;
 * HCA_EUNSUPPORTED for f32 (its kernel needs no workspace: call hca_attn_decode). */
int32_t hca_attn_decode_noalloc(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                                const hca_cache* cache, const void* ring_k, const void* ring_v,
                                void* O, float* lse, hca_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HCA_H_ */
