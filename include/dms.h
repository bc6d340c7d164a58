/*
 * dms.h -- C ABI of libdms: the inference hot path of Dynamic Memory
 * Sparsification (DMS), learned per-head KV-cache eviction with delayed
 * eviction, for one NVIDIA B200 (sm_100a).
 *
 * Sources the operations follow (cited by title and section):
 *  [DMS-Qwen3] "基于 DMS 的 KV Cache 压缩实战：为 Qwen3-8B 训练驱逐适配器
 *              (Model-Optimizer 实验模块)", an article on NVIDIA
 *              Model-Optimizer's experimental/dms module: sections "DMS 工作原理"
 *              (delayed eviction), "驱逐决策的两种来源与两种粒度" (decision
 *              sources and granularity, Qwen3ConfigDMS table), "注意力实现"
 *              (training score_mod; inference with a paged KV cache), "高级选项"
 *              (chunked prefill, cache preallocation), "当前限制" (limits).
 *  [FastDMS]   the FastDMS announcement post: the compact-KV speed table and the
 *              table of serving subsystems DMS changes (prefill kernel, decode
 *              kernel, split-K attention scoring).
 *
 * Conventions shared by every entry point
 *  - Shapes: B batch, T prompt length, Hq query heads, Hkv KV heads
 *    (g = Hq / Hkv query heads share KV head hq / g), D head_dim, w window,
 *    P block (page) size.  Arrays are dense, row-major, token-major:
 *    q[B,T,Hq,D], k/v[B,T,Hkv,D], o[B,T,Hq,D], h[B,T,hidden]; decode drops T.
 *  - Memory: every pointer named "device" is CUDA device memory owned by the
 *    caller.  The library never allocates device memory: the cache lives in a
 *    caller buffer sized by dms_cache_bytes.  Inputs are borrowed until the work
 *    queued on `stream` completes; outputs are written asynchronously on
 *    `stream` (a cudaStream_t passed as void*, NULL = legacy default stream).
 *  - Errors: entry points return DMS_OK (0) or a negative DMS_ERR_* code after
 *    synchronous host-side checks; nothing is launched when a check fails.
 *    Conditions only the device can see (page pool exhausted) set bits of a
 *    sticky device status word, skip the affected writes and never trap; read
 *    it with dms_cache_status.  After a status bit is set the cache contents are
 *    unspecified until dms_cache_reset.
 *  - All calls on one cache must be issued on one stream (or ordered by the
 *    caller); calls on different caches are independent.
 *  - Launch overlap: the decode step kernels, the rotary / decision-neuron
 *    pass and the compaction kernels are programmatic dependents of the
 *    kernel before them on the stream: they may start while it runs and read
 *    none of the caller's inputs before it has completed.  A decode step
 *    kernel may read its cache's own state (counts, plans, page tables) and
 *    request its first pages earlier, when the launch before it is this
 *    library's for another cache or layer, or the same step's rotary pass;
 *    so the cache's buffer must be written by nothing but this library.
 *  - q, k, v and o (prefill and decode) are read and written as 16-byte
 *    vectors: their base pointers must be 16-byte aligned (DMS_ERR_INVALID
 *    otherwise).
 */
#ifndef DMS_H
#define DMS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DMS_API __attribute__((visibility("default")))
#else
#define DMS_API
#endif

/* ---- return codes ---------------------------------------------------------- */
#define DMS_OK 0
#define DMS_ERR_INVALID (-1) /* bad descriptor, argument, pointer or size       */
#define DMS_ERR_STATE (-2)   /* call not allowed in the cache's current state   */
#define DMS_ERR_CUDA (-3)    /* a CUDA runtime call failed                      */
#define DMS_ERR_NOMEM (-4)   /* caller buffer smaller than dms_cache_bytes      */
#define DMS_ERR_SCRATCH_LIMIT (-5) /* the cache's worst-case split-K partials do not
                                      fit the fixed scratch of
                                      dms_decode_attention_noalloc              */

/* ---- device status bits (sticky, read by dms_cache_status) ---------------- */
#define DMS_ST_POOL_EXHAUSTED 1 /* a page was needed and the pool had none     */
#define DMS_ST_CAPACITY 2       /* a slot index exceeded the per-head capacity */
#define DMS_ST_TIMEOUT 4        /* a bounded device wait gave up               */
#define DMS_ST_SPLIT_LIMIT 8    /* FLAT decode: a CTA's share of the slots met
                                   more heads than its table holds (thousands
                                   of heads of very different lengths); use
                                   DMS_DECODE_CLUSTER for such a cache         */

/* ---- enumerations ------------------------------------------------------------ */
enum dms_dtype { DMS_F32 = 0, DMS_BF16 = 1, DMS_FP8_E4M3 = 2 };
/* [DMS-Qwen3] "驱逐决策的两种来源与两种粒度": dms_alpha_per is head or layer. */
enum dms_alpha_per { DMS_ALPHA_PER_HEAD = 0, DMS_ALPHA_PER_LAYER = 1 };
/* Source of the decision logit: the separate adapter (RMSNorm + Linear over the
 * pre-attention hidden state, dms_separate_alpha=True), the last neuron of
 * each key / of the first query head of each GQA group (separate_alpha=False),
 * or an importance score (the KVzap-linear page: one Linear from the hidden
 * state to one score per KV head, no normalisation; a token scoring below the
 * threshold is pruned, the most recent tokens kept -- the DMS rule with
 * window = that number of recent tokens, e.g. 128). */
enum dms_alpha_source {
  DMS_ALPHA_PROJ = 0,
  DMS_ALPHA_KEY_NEURON = 1,
  DMS_ALPHA_QUERY_NEURON = 2,
  DMS_ALPHA_SCORE_LINEAR = 3
};

/* Decode attention kernels.  CLUSTER: one thread-block cluster per (b, h)
 * (cluster size from 8 down to 1 as B * Hkv grows), partials combined on chip.
 * FLAT: one CTA per SM over a balanced list of every head's slots, partials
 * combined by the last CTA to finish a head (for heads of very different
 * lengths).  AUTO picks CLUSTER; FLAT falls back to CLUSTER for shapes it does
 * not stage. */
enum dms_decode_kernel { DMS_DECODE_AUTO = 0, DMS_DECODE_CLUSTER = 1, DMS_DECODE_FLAT = 2 };

/* ---- cache descriptor ---------------------------------------------------------
 * Mirrors the DMS configuration record ([DMS-Qwen3], Qwen3ConfigDMS table):
 * window_size (512), paged_attention_block_size (256, must be below the
 * window), alpha_scale (100), disable_eviction, alpha_per, preallocate_for_tokens
 * (4096), plus the attention-layer shape and the pool size.
 * Constraints (else DMS_ERR_INVALID): all sizes > 0; block % 16 == 0;
 * window > block; num_q_heads % num_kv_heads == 0; head_dim in {64, 128};
 * act_dtype in {F32, BF16}; kv_dtype == act_dtype, or FP8_E4M3 with BF16
 * activations; max_positions <= 1 << 20; pool_pages covers the preallocation. */
typedef struct dms_cache_desc {
  int num_layers;       /* layers held by this cache (L)                        */
  int batch;            /* sequences (B)                                        */
  int num_q_heads;      /* Hq                                                   */
  int num_kv_heads;     /* Hkv                                                  */
  int head_dim;         /* D                                                    */
  int hidden;           /* hidden size read by the adapter (PROJ source)        */
  int window;           /* w: sliding window of delayed eviction                */
  int block;            /* P: page (block) size in tokens                       */
  int max_positions;    /* tokens per sequence the cache can ever hold (T+steps)*/
  int prealloc_tokens;  /* pages for this many tokens per (layer, b, head) are
                           granted at allocation                               */
  int pool_pages;       /* pages in the shared pool (all layers, heads)         */
  int act_dtype;        /* dtype of q, k, v, o, hidden, norm/proj weights       */
  int kv_dtype;         /* dtype of stored pages                                */
  int alpha_per;        /* enum dms_alpha_per                                   */
  int alpha_source;     /* enum dms_alpha_source                                */
  float alpha_scale;    /* multiplies the raw logit (100)                       */
  float rms_eps;        /* RMSNorm epsilon of the adapter (1e-6)                */
  int disable_eviction; /* nonzero: every decision is "keep" (vanilla model)    */
  int decode_kernel;    /* enum dms_decode_kernel: how a decode step splits the
                           attention over the SMs (0: chosen from the shape)  */
  int decision_shift;   /* which token's decision marks token t for eviction
                           ([DMS-Qwen3] "注意力实现": the training path shifts
                           the decision logits by one position; the operators
                           of the page are garbled, so both directions exist):
                             0  token t's own decision (default);
                            +1  token t-1's decision: the logits shifted right
                                by one, token 0 padded with "keep";
                            -1  token t+1's decision: a token's decision marks
                                the token before it, so the newest token is
                                unmarked until the next one arrives        */
} dms_cache_desc;

/* Fill `desc` with the defaults of the DMS configuration record: window 512,
 * block 256, alpha_scale 100, prealloc 4096, per-head decisions, adapter source,
 * rms_eps 1e-6, eviction enabled.  Shape fields are set to 0 (caller fills). */
DMS_API void dms_cache_desc_default(dms_cache_desc* desc);

/* Opaque host handle. */
typedef struct dms_cache dms_cache;

/* Byte offsets of the cache's arrays inside the caller's device buffer, for
 * inspection (tests, debuggers).  All int32 unless noted.
 *   pos        [L,B]             tokens appended per sequence
 *   count      [L,B,Hkv]         retained slots per head
 *   npages     [L,B,Hkv]         pages owned per head
 *   page_table [L,B,Hkv,maxp]    page ids (-1 = none)
 *   slot_pos   [L,B,Hkv,cap]     token position held by each slot
 *   ring       [L,B,Hkv,w]       slot of the token at position p (index p % w)
 *                                in bits 0..30, its evict decision in bit 31
 *   k_pool/v_pool [pool_pages,P,D] page contents in kv_dtype
 *   k_scale/v_scale [pool_pages]  fp32 page scales (FP8 only)
 *   status, next_page             int32 scalars                              */
typedef struct dms_cache_layout {
  size_t total_bytes;
  size_t status, next_page, pos, count, npages, page_table, slot_pos, ring;
  size_t k_pool, v_pool, k_scale, v_scale;
  int max_pages_per_head; /* maxp = ceil(max_positions / P) */
  int slot_capacity;      /* cap = maxp * P                 */
  int prealloc_pages;     /* pages granted per head at allocation */
  int first_free_page;    /* L*B*Hkv*prealloc_pages          */
} dms_cache_layout;

/* ---- decision-logit parameters ----------------------------------------------
 * [DMS-Qwen3] "驱逐决策的两种来源与两种粒度":
 *   PROJ:    alpha[b,h,t] = (W_h . RMSNorm_gamma(h_t) + bias_h) * alpha_scale - offset[b,h]
 *            RMSNorm_gamma(x)_i = x_i / sqrt(mean(x^2) + rms_eps) * gamma_i
 *   *_NEURON: alpha = x[D-1] * alpha_scale - offset[b,h], x the key of head h
 *            (KEY) or the query of head h*g (QUERY); that element is then set
 *            to zero in the caller's k (or q) before the rotary embedding.
 *   SCORE_LINEAR: alpha[b,h,t] = offset[b,h] - (W_h . h_t + bias_h), the offset
 *            holding the pruning threshold (-4 on the KVzap page): a token whose
 *            score is below it is marked; norm_weight is not read.
 *   Layer granularity: every head takes head 0's logit.
 *   [DMS-Qwen3] "Gumbel 噪声与可微门控": at inference a token is evicted iff
 *   alpha > 0 (alpha == 0 keeps), and never when disable_eviction is set. */
typedef struct dms_decide_params {
  /* PROJ: hidden, norm_weight and proj_weight are read as 16-byte vectors and
   * must be 16-byte aligned (DMS_ERR_INVALID otherwise). */
  const void* hidden;      /* device [B,T,hidden] (decode: [B,hidden]), act dtype; PROJ, SCORE_LINEAR */
  const void* norm_weight; /* device gamma [hidden], act dtype; PROJ only (not read by SCORE_LINEAR) */
  const void* proj_weight; /* device W [Hkv,hidden], act dtype; PROJ, SCORE_LINEAR        */
  const void* proj_bias;   /* device [Hkv] act dtype, or NULL                             */
  const float* offset;     /* device fp32 offset[b*offset_batch_stride + h]               */
  int offset_batch_stride; /* 0 (one offset per head) or Hkv (per sequence and head)      */
} dms_decide_params;

/* ---- prefill -------------------------------------------------------------------
 * T prompt tokens for every sequence of one layer, at positions T0 .. T0+T-1
 * where T0 is the number of tokens the layer already holds.  A prompt may be
 * prefilled in several calls (chunked prefill, [DMS-Qwen3] "高级选项": the
 * prompt split into fixed-size chunks, 4096 tokens by default): each call's
 * queries attend to the keys the cache holds, as stored (FP8 pages decoded),
 * plus the call's own keys, under the mask below, so with bf16/fp32 pages the
 * chunks' outputs equal one prefill of the whole prompt.  Prefill calls may
 * follow each other until the layer's first decode step; after it a prefill
 * is DMS_ERR_STATE ([DMS-Qwen3] "当前限制": prefill-then-generate; reset the
 * cache for a new prompt).  A call with T0 > 0 needs bf16 activations and a
 * GQA group Hq/Hkv that is a power of two up to 16 (else DMS_ERR_INVALID), and
 * T0 + T <= max_positions.  In order, on `stream`:
 *  1. decision logits alpha[B,Hkv,T] (when `decide` is non-NULL; else `alpha`
 *     is read as an input);
 *  2. for neuron sources the decision element is zeroed in place, then, when
 *     rope tables are given, q and k are rotated in place (half-split rotary
 *     embedding; token t at position t);
 *  3. the append rule is replayed for t = 0..T-1 in parallel ([DMS-Qwen3]
 *     "推理模式", delayed eviction: a token marked for eviction stays while it
 *     is inside the window; the token entering overwrites its slot in place,
 *     else the next free slot is used and the block table grows by one page);
 *     the survivors are written to the pages ([FastDMS]: the prefill kernel
 *     streams surviving K/V into compact storage; FP8 pages are quantised after
 *     eviction, scale = max |x| / 448 over the page's rows);
 *  4. DMS-masked attention: query i sees key j iff j <= i and (i - j < w or
 *     alpha_j <= 0); o = softmax(q k^T / sqrt(D)) v over those keys, computed
 *     from the unquantised k, v.
 * Page grants of one call go to (b, h) in row-major order from one ascending
 * counter. */
typedef struct dms_prefill_args {
  int seq_len;              /* T, 1 <= T <= min(max_positions, 262144 = 2^18)
                               (DMS_ERR_INVALID otherwise)                         */
  void* q;                  /* device [B,T,Hq,D] act dtype (rotated in place)     */
  void* k;                  /* device [B,T,Hkv,D] act dtype (rotated/zeroed in place) */
  const void* v;            /* device [B,T,Hkv,D] act dtype                        */
  void* o;                  /* device [B,T,Hq,D] act dtype, output                 */
  float* alpha;             /* device [B,Hkv,T] fp32: output, or input if decide==NULL */
  const dms_decide_params* decide; /* host struct, or NULL                         */
  const float* rope_cos;    /* device [max_positions, D/2] fp32, or NULL           */
  const float* rope_sin;    /* device [max_positions, D/2] fp32, or NULL           */
} dms_prefill_args;

/* ---- decode step -----------------------------------------------------------------
 * One new token per sequence for one layer, at position t = pos[layer, b]:
 * decision logit, rotary embedding, append with in-place reuse of the slot of
 * token t - w when that token was marked for eviction (else a new slot; a new
 * page whenever the slot starts one), then attention of the g query heads of
 * each KV head over that head's retained slots [0, count), split across the
 * SMs and merged with a log-sum-exp combine ([FastDMS], attention scoring:
 * split-K grouped compact decode attention over variable-length per-head live
 * spans).  FP8 pages: when the new row's max |x| / 448 exceeds the page scale,
 * the page's rows are re-encoded at the larger scale before the row is written.
 * bf16 and FP8 pages take one launch per step with DMS_DECODE_AUTO or
 * DMS_DECODE_CLUSTER (FP8 with DMS_DECODE_FLAT: an append launch, then the
 * attention), plus the neuron / rotary pass when it applies. */
typedef struct dms_decode_args {
  void* q;                  /* device [B,Hq,D] act dtype (rotated in place)  */
  void* k;                  /* device [B,Hkv,D] act dtype (rotated in place) */
  const void* v;            /* device [B,Hkv,D] act dtype                    */
  void* o;                  /* device [B,Hq,D] act dtype, output             */
  float* alpha;             /* device [B,Hkv] fp32: output, or input if decide==NULL */
  const dms_decide_params* decide; /* host struct, or NULL                   */
  const float* rope_cos;    /* device tables as in dms_prefill_args, or NULL */
  const float* rope_sin;
} dms_decode_args;

/* ---- entry points ----------------------------------------------------------------- */

/* Device bytes a cache with this descriptor needs (pool, tables, scratch).
 * Returns DMS_ERR_INVALID on a bad descriptor. */
DMS_API int dms_cache_bytes(const dms_cache_desc* desc, size_t* dev_bytes);

/* Create a cache inside `dev_mem` (device, >= dms_cache_bytes bytes, 256-byte
 * aligned, owned by the caller and not freed by the library) and initialise it
 * on `stream` (preallocated pages granted row-major over (layer, b, head, page)).
 * On success *out receives a host handle to release with dms_cache_free. */
DMS_API int dms_cache_alloc(const dms_cache_desc* desc, void* dev_mem, size_t bytes, void* stream,
                    dms_cache** out);

/* Release the host handle (the device buffer stays the caller's). NULL is a no-op. */
DMS_API int dms_cache_free(dms_cache* cache);

/* Empty every layer for a new set of sequences ([DMS-Qwen3] "当前限制": the
 * cache must be reset between independent sequences). Clears the status word. */
DMS_API int dms_cache_reset(dms_cache* cache, void* stream);

/* Offsets of the cache's arrays in the caller buffer. */
DMS_API int dms_cache_get_layout(const dms_cache* cache, dms_cache_layout* layout);

/* ---- state export -----------------------------------------------------------------
 * Host copies of one layer's cache state ([DMS-Qwen3], inference mode with the
 * paged KV cache: what the append rule maintains).  Every pointer is a
 * caller-owned host buffer of the size given (B = batch, H = num_kv_heads,
 * maxp and cap from dms_cache_get_layout, w = window), or NULL to skip it:
 *   pos        [B]            tokens appended so far per sequence
 *   count      [B,H]          retained slots per head
 *   npages     [B,H]          pages owned per head
 *   page_table [B,H,maxp]     page ids (-1 past npages)
 *   slot_pos   [B,H,cap]      position held by each slot (entries past count undefined)
 *   ring       [B,H,w]        slot of position t at t % w, bit 31 = its eviction decision */
typedef struct dms_cache_view {
  int* pos;
  int* count;
  int* npages;
  int* page_table;
  int* slot_pos;
  int* ring;
} dms_cache_view;

/* Copy layer `layer`'s state into `out` after the work already on `stream`
 * (synchronises the stream).  DMS_ERR_INVALID for a bad handle or layer,
 * DMS_ERR_CUDA if a copy fails. */
DMS_API int dms_cache_export(dms_cache* cache, int layer, dms_cache_view* out, void* stream);

/* Read the sticky device status word (DMS_ST_* bits).  Synchronises `stream`. */
DMS_API int dms_cache_status(dms_cache* cache, void* stream, int* status);

/* Decision logits alone, for T tokens of every sequence (no cache state is
 * touched): PROJ reads decide->hidden [B,T,hidden]; neuron sources read (and
 * zero) the decision element of `neuron_src` ([B,T,Hkv,D] keys or [B,T,Hq,D]
 * queries).  alpha: device [B,Hkv,T] fp32 output. */
DMS_API int dms_decide(dms_cache* cache, int seq_len, const dms_decide_params* decide, void* neuron_src,
               float* alpha, void* stream);

/* Prefill T tokens into layer `layer` (0 <= layer < L) after the tokens it
 * already holds; see dms_prefill_args.  Equivalent to dms_prefill_compact
 * followed by dms_prefill_attention. */
DMS_API int dms_prefill(dms_cache* cache, int layer, const dms_prefill_args* args, void* stream);

/* Steps 1-3 of dms_prefill: decision logits, neuron zeroing / rotation, and the
 * compaction of the tokens into the layer's pages ([FastDMS] prefill kernel),
 * continuing from the layer's state.  Leaves the position-sorted list of kept
 * tokens (and, for a later chunk, the keys and values of the last w positions
 * before it) in the cache's scratch for dms_prefill_attention; that scratch is
 * shared by the layers, so the attention must follow before another layer's
 * compaction.  DMS_ERR_STATE after the layer's first decode step. */
DMS_API int dms_prefill_compact(dms_cache* cache, int layer, const dms_prefill_args* args, void* stream);

/* Step 4 of dms_prefill: the DMS-masked attention of the call's tokens.  Must
 * follow dms_prefill_compact of the same layer and length, with no other
 * layer's compaction in between (else DMS_ERR_STATE); reads args->q, k, v (as
 * rotated by the compaction) and writes args->o. */
DMS_API int dms_prefill_attention(dms_cache* cache, int layer, const dms_prefill_args* args, void* stream);

/* One decode step of layer `layer` after its prefill; DMS_ERR_STATE before the
 * prefill or when max_positions tokens are already held. */
DMS_API int dms_decode_step(dms_cache* cache, int layer, const dms_decode_args* args, void* stream);

/* One decode step of the layers [layer, layer + num_layers) in one launch of
 * the attention kernel (one thread-block cluster per (layer, b, h)), for a
 * stack whose layers do not feed each other within a step -- the same result
 * as dms_decode_step on each layer in turn (page grants in (layer, b, h)
 * order).  Every array of `args` holds the num_layers layers back to back:
 * q/o [L',B,Hq,D], k/v [L',B,Hkv,D], alpha [L',B,Hkv]; with decision
 * parameters, hidden [L',B,hidden], norm_weight [L',hidden], proj_weight
 * [L',Hkv,hidden], proj_bias [L',Hkv] (or NULL) and offset [L',B,Hkv] (batch
 * stride Hkv) or [L',Hkv] (batch stride 0).  bf16 or FP8 pages
 * (DMS_ERR_INVALID for fp32 pages); every layer of the range must be
 * prefilled and hold the same number of tokens (else DMS_ERR_STATE). */
DMS_API int dms_decode_step_layers(dms_cache* cache, int layer, int num_layers, const dms_decode_args* args,
                                   void* stream);

/* First half of dms_decode_step: decision logit, rotation and the append of
 * the new token ([FastDMS] decode kernel), plus the work list of the attention.
 * The token's position is read on the device, so the call may be captured in a
 * CUDA graph; `o` is not used. */
DMS_API int dms_decode_append(dms_cache* cache, int layer, const dms_decode_args* args, void* stream);

/* Second half of dms_decode_step: split-K grouped attention of q [B,Hq,D] over
 * each head's retained slots, written to o [B,Hq,D] (act dtype).  Must follow a
 * dms_decode_append of the same layer (else DMS_ERR_STATE). */
DMS_API int dms_decode_attention(dms_cache* cache, int layer, const void* q, void* o, void* stream);

/* dms_decode_attention without touching any scratch memory of the caller.
 * The pages have no counterpart of this call: it exists for embedding the
 * library in callers that cannot set aside device memory for the split-K
 * partials -- e.g. an engine whose device memory is handed out by its own
 * fixed pool at start-up and whose decode loop must never reach cudaMalloc
 * (cudaMalloc can synchronise the device and can fail once the pool owns the
 * memory).  Same arguments as dms_decode_attention, and the same result within the
 * decode attention tolerance (it runs another kernel, k_decode_attn, whose
 * splits and merge order differ, so the two are not bit-identical); the partial
 * results of the splits live instead in one fixed array of device memory that
 * the library holds (4 MiB per GPU that loads the library, kept until exit).
 * fp32 caches need no partials: their attention runs one CTA per query head,
 * with no limit and nothing shared.
 *  - Limit (bf16 and FP8 pages): the cache's worst case of split-K scratch, one int per (b, h) for
 *    the per-head arrival counters (rounded up to 256 bytes) plus
 *    items_cap * (Hq/Hkv) * (head_dim + 2) * 4 bytes of partials with
 *    items_cap = max(B * Hkv * ceil(max_positions / block), 640) + B * Hkv,
 *    must fit in 4 MiB; otherwise DMS_ERR_SCRATCH_LIMIT and nothing is launched.
 *  - The first call on a device looks up the array's device address with that
 *    device current (no allocation); make that first call before any stream
 *    capture.
 *  - Every call shares the one array, which keeps the last call's contents.
 *    Each call clears the per-head counters on `stream` before its kernel (the
 *    partials need no clearing: each is written before it is read).  Calls
 *    that overlap on the GPU (on different streams, or on different caches of
 *    the same device without ordering) race on the array and give wrong
 *    results; order them. */
DMS_API int dms_decode_attention_noalloc(dms_cache* cache, int layer, const void* q, void* o, void* stream);

/* ---- training mode (forward) ------------------------------------------------------
 * [DMS-Qwen3] "Gumbel 噪声与可微门控" and "注意力实现": while the eviction
 * adapter is trained, decisions are soft.  Both calls use only the cache's
 * shape (B, Hq, Hkv, D, window) and none of its state.
 *
 * dms_train_gate: for each of the B*Hkv rows of T tokens, l = (alpha + noise)
 * / tau (tau = 0.1 on the page; noise drawn by the caller, NULL for none),
 * prob = sigmoid(l), hard = 1 if l > 0 else 0 -- the forward value of the
 * straight-through decision (prob > 0.5) - prob + prob -- and the eviction
 * penalty of the attention, taken from the logits shifted right by one
 * position: penalty[t] = logsigmoid(-l[t-1]) = log(1 - prob[t-1]),
 * penalty[0] = 0.  alpha, noise, prob, hard, penalty: device [B,Hkv,T] fp32.
 * DMS_ERR_INVALID for a null pointer, T <= 0 or tau not positive and finite.
 *
 * dms_train_attention: the soft-gated attention of the training score_mod:
 * query i and key j <= i score q.k / sqrt(D), plus penalty[b,h,j] when j is
 * outside the window (i - j >= w); causal violations (mask value -50000) carry
 * no weight; o = softmax(scores) v over every key, on the tensor cores.
 * q/o [B,T,Hq,D], k/v [B,T,Hkv,D] bf16 (16-byte aligned), penalty [B,Hkv,T]
 * fp32.  Needs bf16 activations and Hq/Hkv a power of two up to 16
 * (DMS_ERR_INVALID otherwise). */
DMS_API int dms_train_gate(dms_cache* cache, int seq_len, const float* alpha, const float* noise, float tau,
                           float* prob, float* hard, float* penalty, void* stream);
DMS_API int dms_train_attention(dms_cache* cache, int seq_len, const void* q, const void* k, const void* v,
                                const float* penalty, void* o, void* stream);

/* Self-check of the device failure path (the pages have no counterpart): one
 * thread waits, with the same bounded wait every kernel of the library uses,
 * on a shared-memory barrier that nothing ever completes, gives up after
 * `tries` tries (1 <= tries <= 2^24, each try suspends the thread for a few
 * microseconds at most) and sets DMS_ST_TIMEOUT in the cache's status word, as
 * a kernel whose tile never arrives would.  Nothing is left in flight and the
 * context stays usable; dms_cache_reset clears the bit.  For tests of a
 * caller's error handling. */
DMS_API int dms_selftest_wait_timeout(dms_cache* cache, int tries, void* stream);

/* Tokens appended so far to `layer` (host-side counter, no device access). */
DMS_API int dms_cache_positions(const dms_cache* cache, int layer);

#ifdef __cplusplus
}
#endif

#endif /* DMS_H */
