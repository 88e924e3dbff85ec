/*
 * kvc.h -- C ABI of libkvc, a B200 (sm_100a) paged KV cache for streaming
 * visual-geometry transformers: per-frame, frame-causal attention of a new
 * frame's tokens over a bounded paged cache, plus the cache maintenance around
 * it (page-aligned append, sliding-window eviction with pinned scale frames,
 * keyframe skip-append, FP8 quantisation, importance-scored compression).
 *
 * Sources, cited by page title and section:
 *   [GCT]  "How GCTStream Implements Streaming 3D Reconstruction with KV Cache"
 *   [LBM]  "Can LingBot-Map Achieve 20 FPS Streaming 3D Reconstruction?"
 *   [SCV]  StreamCacheVGGT (cross-layer consistency scoring + hybrid compression)
 *   [IVG]  "InfiniteVGGT: Visual Geometry Grounded Transformer for Endless Streams"
 *   [XSV]  "XStreamVGGT: Extremely Memory-Efficient Streaming Vision Geometry
 *          Grounded Transformer with KV Cache Compression" (abstract)
 *
 * Conventions for every call:
 *   - Device pointers are caller-owned and must stay valid until the cache's
 *     stream has executed the call. Host pointers are read or written before
 *     the call returns.
 *   - Q, K, V and O are token-major [T, H, D] tensors (T = tokens_per_frame,
 *     H = num_heads, D = head_dim), densely packed, in the configured I/O dtype
 *     (fp32 or bf16). D*element_size must be a multiple of 16 bytes and device
 *     pointers 16-byte aligned.
 *   - The library allocates all device memory (page pools, page tables,
 *     scratch) in kvc_create and nothing afterwards, so cache memory is
 *     constant for the life of a stream ([GCT] Sliding Window Eviction: O(1)
 *     memory).
 *   - Calls enqueue work on the cache's stream and return without waiting for
 *     the GPU, except kvc_page_table, kvc_token_meta, kvc_last_merge,
 *     kvc_export_pages, kvc_step_host and kvc_synchronize, which synchronise
 *     (the cache's stream and its internal copy streams).
 *   - Errors are status codes; kvc_last_error() gives a message. A status other
 *     than KVC_OK leaves the cache state unchanged unless stated otherwise.
 *     A device-side failure (a bounded wait that gave up, an exhausted page
 *     pool) is latched in a device error word and reported by the next
 *     synchronising call as KVC_ERR_TIMEOUT or KVC_ERR_DEVICE; the CUDA
 *     context stays usable.
 *   - A kvc_cache is not thread-safe; use one per thread or serialise.
 */
#ifndef KVC_H_
#define KVC_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVC_VERSION 1

/* Every entry point is exported with default visibility; internals stay hidden. */
#if defined(__GNUC__)
#define KVC_API __attribute__((visibility("default")))
#else
#define KVC_API
#endif

typedef enum {
  KVC_OK = 0,
  KVC_ERR_ARG = 1,          /* invalid argument or unsupported shape */
  KVC_ERR_OOM = 2,          /* device allocation failed in kvc_create */
  KVC_ERR_CUDA = 3,         /* a CUDA runtime call failed */
  KVC_ERR_STATE = 4,        /* call out of order (e.g. attend with nothing pending) */
  KVC_ERR_BUDGET = 5,       /* protected tokens exceed the keep tier */
  KVC_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up */
  KVC_ERR_DEVICE = 7,       /* device-side consistency check failed */
  KVC_ERR_UNSUPPORTED = 8   /* configuration valid but not implemented on this path */
} kvc_status;

typedef enum { KVC_F32 = 0, KVC_BF16 = 1, KVC_FP8_E4M3 = 2 } kvc_dtype;

/* Cache configuration; all fields are read once by kvc_create.
 *
 * Eviction ([LBM] Sliding-Window Eviction Strategy; [GCT] Sliding Window
 * Eviction): with window_frames = W > 0 the committed cache of each layer is
 * the first scale_frames = S committed frames plus the last W committed frames.
 *
 * Compression ([SCV] sections 2.1-2.2): with budget_tokens = B > 0 (and
 * window_frames <= 0) kvc_compress keeps floor(keep_frac * B) tokens, merges
 * the next B - floor(keep_frac * B) into kept tokens and drops the rest
 * whenever a layer holds more than B committed tokens.
 */
typedef struct {
  int32_t num_layers;           /* independent per-layer caches */
  int32_t num_heads;            /* H */
  int32_t head_dim;             /* D */
  int32_t tokens_per_frame;     /* T (e.g. 1004 = 37*27 patches + 1 camera + 4 register) */
  int32_t num_special_tokens;   /* leading camera/register tokens of each frame (protected) */
  int32_t page_size;            /* P tokens per page; each frame starts on a fresh page */
  int32_t window_frames;        /* W; <= 0: no sliding window */
  int32_t scale_frames;         /* S pinned first frames */
  int32_t io_dtype;             /* kvc_dtype of Q, K, V, O: KVC_F32 or KVC_BF16 */
  int32_t kv_dtype;             /* storage: same as io_dtype, or KVC_FP8_E4M3 with bf16 I/O */
  float softmax_scale;          /* logits = softmax_scale * q . k */
  int32_t budget_tokens;        /* B; 0: no compression */
  float keep_frac;              /* keep tier fraction (0.6) */
  float lambda_;                /* consistency weight lambda (0.5) */
  int32_t rank_window;          /* layers in the rank window (5) */
  int32_t residual_dim;         /* R, columns of the residual given to kvc_compress */
  int32_t protect_first_frame;  /* 1: every token of frame 0 is always kept */
  int32_t max_frames;           /* cap on cached frames when W <= 0 and B == 0 */
  int32_t kv_splits;            /* s > 0: the tensor-core attention cuts each head's KV
                                   sequence into about s pieces (merged in the kernel);
                                   0 = automatic (the pieces that fill the SMs) */
  int32_t diversity_budget;     /* K > 0: rolling diversity-pruned memory, K kept tokens per
                                   head per layer besides the first frame (see kvc_attend) */
  int32_t special_frames;       /* > 0 (window mode only): cross-frame special tokens, see
                                   kvc_attend; the evicted frames whose special tokens stay */
  int32_t fp8_dim_adaptive;     /* 1 with kv_dtype FP8 (D = 64, P = 16): dimension-adaptive
                                   scales, see kvc_append_frame; 0: one scale per (page, head) */
  int32_t model_heads;          /* heads of the caller's Q/K/V/O tensors; 0 = num_heads. With
                                   model_heads > num_heads the cache holds the head range below
                                   (bf16 window caches on the tensor-core path only) */
  int32_t head_begin;           /* first of the num_heads consecutive model heads the cache
                                   holds: kvc_append_frame reads that slice of [T, model_heads, D]
                                   K and V, kvc_attend reads the slice of Q and writes the same
                                   slice of O (other heads of O untouched) */
  int32_t reserved[2];          /* must be zero */
} kvc_config;

/* Cache statistics ([GCT] Cache Monitoring: occupancy, memory use, eviction status). */
typedef struct {
  int64_t tokens;               /* committed tokens in the layer */
  int64_t pages_used;           /* pages held (committed + pending) */
  int64_t pages_total;          /* pool pages of the layer */
  int64_t pool_bytes;           /* device bytes of the layer's page pool */
  int64_t high_water_pages;     /* max pages ever held at once by the layer */
  int64_t frames_appended;      /* kvc_append_frame calls on the layer */
  int64_t frames_committed;     /* keyframes committed */
  int64_t frames_skipped;       /* non-keyframes released after attention */
  int64_t frames_evicted;       /* frames removed by the sliding window */
  int64_t compress_events;      /* compressions performed */
  int64_t device_error;         /* latched device error word (0 = none) */
  int64_t kernel_launches;      /* kernels this cache has launched (all layers) */
} kvc_info;

typedef struct kvc_cache kvc_cache;

/* Create a cache on the current CUDA device. `stream` is a cudaStream_t (NULL:
 * the legacy default stream) on which all later work is enqueued. Allocates the
 * page pools sized for the configuration (window: (S + W + 1) frames of pages
 * per layer; budget: 2*ceil(B/P) + (ceil(B/T) + 2) frames of pages), page
 * tables and scratch, and zero-fills them. On success *out owns everything;
 * release with kvc_destroy. Errors: KVC_ERR_ARG (bad config; also sizes past
 * the index range: more than 2^30 pages per layer, more than 2^31 - 1 pool
 * rows of P slots per head over all layers on the tensor-core path, a frame
 * (tokens x model heads x head_dim) or a page (P x heads x head_dim) of 2^29 elements
 * or more, or a field above its cap: 65,536 layers, heads or page size,
 * 2^24 tokens per frame or frames of window, scale or max_frames), KVC_ERR_OOM. */
KVC_API kvc_status kvc_create(const kvc_config* cfg, void* stream, kvc_cache** out);

/* Synchronise the stream and free everything the cache owns. NULL is a no-op. */
KVC_API kvc_status kvc_destroy(kvc_cache* c);

/* Change the stream used by later calls (work already enqueued stays on the old one:
 * synchronise it first if later work must follow it). Errors: KVC_ERR_ARG (NULL cache). */
KVC_API kvc_status kvc_set_stream(kvc_cache* c, void* stream);

/* Empty every layer (page tables, free lists, rank history, counters) between
 * videos, keeping the pool memory ([GCT] Cache Initialization and Cleanup,
 * clean_kv_cache). Stream-ordered. Errors: KVC_ERR_ARG (NULL cache), KVC_ERR_CUDA. */
KVC_API kvc_status kvc_reset(kvc_cache* c);

/* Page-aligned append of frame `frame_idx` to `layer` ([LBM] Page-Aligned
 * Tensor Layout; [GCT] AggregatorStream with Paged KV Cache). The device
 * allocates ceil(T/P) lowest-free pages and writes k_dev, v_dev ([T, H, D],
 * io dtype) into them as pool layout [page][head][slot][dim]; slots past T in
 * the last page are zero. With kv_dtype FP8 each (page, head) block of K and V
 * is quantised with its own absmax scale: scale = fp32(amax / 448), code =
 * E4M3 round-to-nearest-even saturating of fp32(x / scale) ([XSV] abstract).
 * With fp8_dim_adaptive ([XSV] abstract: dimension-adaptive KV quantisation, read as
 * KIVI's keys per channel and values per token) the same rule applies to each channel of
 * K (a scale per (page, head, channel)) and each token of V (a scale per (page, head,
 * slot)); the per-(page, head) scale arrays then hold the largest of a block's scales.
 * The frame is *pending* until kvc_attend: `is_keyframe` = 0 makes attention
 * release it afterwards ([GCT] Selective Frame Caching with Skip Append).
 * Frame indices must increase per layer. Errors: KVC_ERR_STATE if a frame is
 * already pending on the layer. */
KVC_API kvc_status kvc_append_frame(kvc_cache* c, int32_t layer, int32_t frame_idx,
                            const void* k_dev, const void* v_dev, int32_t is_keyframe);

/* kvc_append_frame for every layer at once: k_devs[l], v_devs[l] (host arrays of
 * num_layers device pointers) hold layer l's [T, H, D] K and V. One page-allocation
 * launch and one append launch cover up to 64 layers, so the frame's whole K/V write is
 * a single HBM-bound kernel. Same semantics, layout and errors as kvc_append_frame
 * applied to each layer; nothing is appended unless every layer can take the frame. */
KVC_API kvc_status kvc_append_frame_all(kvc_cache* c, int32_t frame_idx, const void* const* k_devs,
                                        const void* const* v_devs, int32_t is_keyframe);

/* Frame attention of the pending frame's queries q_dev [T, H, D] over every
 * token of `layer` (committed + pending), writing o_dev [T, H, D]:
 * O[i,h] = sum_j softmax_j(softmax_scale * q_i . k_j) v_j, no mask
 * ([GCT] Frame-by-Frame Causal Processing; [IVG] Causal Attention). Then the
 * pending frame is committed (keyframe; frames outside the first S and last W
 * committed are evicted and their pages freed) or released (non-keyframe).
 * With special_frames > 0 an evicted frame keeps its special tokens ([GCT] Special
 * Token Persistence): its first ceil(num_special_tokens / P) pages stay in the page
 * table, trimmed to those tokens (other slots zeroed), and later frames attend to them;
 * beyond special_frames such frames the oldest one's pages are freed. A non-keyframe
 * keeps nothing.
 * bf16 with D = 64 runs on tcgen05 tensor cores (fp32 accumulation); fp32 I/O
 * runs fp32 FMA arithmetic. With FP8 storage the tensor cores take Q as f16: each query
 * row is first multiplied by the power of two that puts its largest magnitude in
 * [2^14, 2^15) (and its logits by the inverse), so every finite bf16 query is accepted
 * and none overflows. On every path the logits are formed and exponentiated in fp32:
 * while |softmax_scale * q . k| stays far below 2^20 the softmax keeps its full
 * resolution; logits of 2^24 and beyond (where fp32 cannot tell logits one unit apart)
 * are outside the supported range and may give non-finite outputs.
 * Errors: KVC_ERR_ARG (bad layer, NULL or non-16-byte-aligned Q or O), KVC_ERR_STATE
 * (nothing pending on the layer), KVC_ERR_CUDA (a launch failed). */
KVC_API kvc_status kvc_attend(kvc_cache* c, int32_t layer, const void* q_dev, void* o_dev);

/* kvc_attend on every layer, in layer order: q_devs[l] and o_devs[l] are layer l's
 * [T, H, D] queries and outputs (each 16-byte aligned), and every layer must have a
 * pending frame. The results, page tables and counters are those of the per-layer
 * calls. On the tensor cores (bf16 or FP8 storage, D = 64, P = 16) the layers'
 * attention runs in one launch per 32 layers (after the rolling memory's pruning of
 * every layer, itself one launch); otherwise (fp32, other head dims or page sizes) the
 * call is the per-layer loop.
 * Errors: KVC_ERR_ARG (NULL or misaligned pointers), KVC_ERR_STATE (a layer without a
 * pending frame; nothing is attended then). */
KVC_API kvc_status kvc_attend_all(kvc_cache* c, const void* const* q_devs, void* const* o_devs);

/* The joint scale-frame phase ([GCT] Scale-Frame Phase): the first n_frames frames of a
 * stream, processed together with bidirectional attention. q_dev, k_dev, v_dev and o_dev
 * are [n_frames * T, H, D] (frame-major, io dtype). Frames 0 .. n_frames-1 are appended
 * and committed (as kvc_append_frame with is_keyframe = 1), then all n_frames * T
 * queries attend over all of their tokens with no mask; the causal frame-by-frame phase
 * continues with frame n_frames. 1 <= n_frames <= max(1, scale_frames). Errors:
 * KVC_ERR_ARG (pointers, alignment, frame count, more than 2^31 - 1 elements in Q),
 * KVC_ERR_STATE (the layer is not empty, a token budget or per-head page lists). */
KVC_API kvc_status kvc_scale_phase(kvc_cache* c, int32_t layer, int32_t n_frames, const void* q_dev,
                                   const void* k_dev, const void* v_dev, void* o_dev);

/* Importance scoring and, when the committed cache of `layer` holds more than
 * B tokens, keep/merge/drop compression ([SCV] 2.1.1-2.1.4, 2). Must follow
 * kvc_attend of the same frame; within a frame layers are scored in ascending
 * order (the rank history covers the last rank_window layers of this frame and
 * is reset when a new frame starts). residual_dev [T, R] fp32 gives the raw
 * score s_i = fp32(sqrt(sum_c r_ic^2)), the squares summed in fp64 (each lane of a
 * warp sums 32 consecutive channels in ascending order, then the 32 lane sums are
 * added in lane order). Scores:
 * rank R (s descending, ties lower slot), sigma from the population variance
 * of R/(T-1) over the window, Cons = max(0, 1 - sigma sqrt(12)),
 * s_hat = fp32(s (1 + lambda Cons)) evaluated in fp64. Compression: protected
 * tokens (frame 0 if protect_first_frame, and the first num_special_tokens of
 * every frame) are kept; the others by s_hat descending (ties lower id) fill
 * the keep tier; the next B - floor(keep_frac B) are each merged into the kept
 * non-protected token of highest full-key cosine (ties lower id) as a
 * count-weighted mean rounded once to bf16; the rest are dropped; kept tokens
 * are rewritten in ascending id into the lowest free pages. *fired_out (host,
 * may be NULL) receives 1 when a compression ran. bf16 caches only.
 * Errors: KVC_ERR_ARG (B == 0 or NULL residual), KVC_ERR_STATE (order),
 * KVC_ERR_BUDGET (protected tokens exceed the keep tier). */
KVC_API kvc_status kvc_compress(kvc_cache* c, int32_t layer, const float* residual_dev, int32_t* fired_out);

/* kvc_compress on every layer of the frame just attended: residual_devs[l] is layer l's
 * [T, R] fp32 residual (device); fired_out (host, num_layers int32, may be NULL) receives
 * per layer 1 when a compression ran. Results, page tables and metadata are those of
 * kvc_compress on layers 0, 1, ... in order. Every layer is scored first, in order (the
 * CLCES rank window spans layers); the layers over budget are then compressed side by side
 * on the cache's side streams (each with its own scratch), joined back into the cache's
 * stream before the call returns. kvc_last_raw_scores afterwards gives the last layer's
 * raw scores. Errors: those of kvc_compress (the first one met); KVC_ERR_ARG for a NULL
 * array or residual. An error in the scoring leaves every layer uncompressed; an error in
 * one layer's compression (e.g. KVC_ERR_BUDGET) does not stop the other layers over
 * budget, which are compressed as usual: fired_out tells which were. */
KVC_API kvc_status kvc_compress_all(kvc_cache* c, const float* const* residual_devs, int32_t* fired_out);

/* Synchronise and copy the page table of `layer` to host: rows of 4 int32
 * (owner, page_in_owner, phys_page, valid_tokens) in cache order; owner is the
 * frame index, or -1 for pages written by compaction. Writes at most
 * `capacity` rows; *n_rows receives the full count. `info` (may be NULL)
 * receives the layer's statistics. Errors: KVC_ERR_ARG (bad layer), KVC_ERR_CUDA,
 * and a device-side failure latched earlier (KVC_ERR_TIMEOUT, KVC_ERR_DEVICE). */
KVC_API kvc_status kvc_page_table(kvc_cache* c, int32_t layer, int32_t* rows_host, int32_t capacity,
                          int32_t* n_rows, kvc_info* info);

/* Synchronise and copy per-token metadata of `layer` in cache order: token id
 * (frame * T + slot), merge count, and enhanced score s_hat. Any output pointer
 * may be NULL; at most `capacity` tokens are written and *n_out receives the full count.
 * Errors: KVC_ERR_ARG (bad layer), KVC_ERR_UNSUPPORTED (no token budget: no metadata),
 * KVC_ERR_STATE (per-head page lists), KVC_ERR_DEVICE (a page-table row outside the
 * pool), KVC_ERR_CUDA, and a device-side failure latched earlier. */
KVC_API kvc_status kvc_token_meta(kvc_cache* c, int32_t layer, int64_t* ids_host, int32_t* counts_host,
                          float* shat_host, int32_t capacity, int32_t* n_out);

/* Synchronise and copy the raw scores s_i (fp32, one per token slot of the frame) that
 * the last kvc_compress call computed from its residual ([SCV] 2.1.1: the L2 norm of the
 * FFN residual), for inspection. s_host: host array of `capacity` >= tokens_per_frame
 * floats; *n_out receives tokens_per_frame. Errors: KVC_ERR_ARG (budget_tokens is 0,
 * capacity too small), KVC_ERR_STATE (nothing scored yet). */
KVC_API kvc_status kvc_last_raw_scores(kvc_cache* c, float* s_host, int32_t capacity, int32_t* n_out);

/* Synchronise and copy the (source id, target id) pairs of the last
 * compression of `layer`, in ascending source id. At most `capacity` pairs are written;
 * *n_out receives the full count. Errors: KVC_ERR_ARG (bad layer, budget_tokens is 0),
 * KVC_ERR_CUDA. */
KVC_API kvc_status kvc_last_merge(kvc_cache* c, int32_t layer, int64_t* src_host, int64_t* dst_host,
                          int32_t capacity, int32_t* n_out);

/* Synchronise and copy the raw pool contents of page-table rows
 * [first_row, first_row + n_rows) of `layer`: K and V pages as stored
 * ([H][P][D] per page, storage dtype; FP8: codes), and for FP8 the per-(page,
 * head) scales [n_rows][H] fp32 (scale pointers may be NULL otherwise). Errors:
 * KVC_ERR_ARG (bad layer, rows outside the page table), KVC_ERR_STATE (per-head page
 * lists), KVC_ERR_CUDA, and a device-side failure latched earlier. */
KVC_API kvc_status kvc_export_pages(kvc_cache* c, int32_t layer, int32_t first_row, int32_t n_rows,
                            void* k_host, void* v_host, float* k_scale_host, float* v_scale_host);

/* Dimension-adaptive FP8 scales of page-table rows [first_row, first_row + n_rows) of
 * `layer`: k_chan_host [n_rows][H][D] (K, per channel) and v_tok_host [n_rows][H][P] (V,
 * per slot; 0 for slots without a token). Host buffers owned by the caller. Synchronises.
 * Errors: KVC_ERR_STATE (not dimension-adaptive FP8), KVC_ERR_ARG (range, pointers). */
KVC_API kvc_status kvc_export_fp8_group_scales(kvc_cache* c, int32_t layer, int32_t first_row, int32_t n_rows,
                                               float* k_chan_host, float* v_tok_host);

/* One whole frame step of `layer` from HOST buffers: copy q, k, v [T, H, D]
 * host -> device, append, attend (+ commit/evict), copy O device -> host,
 * and wait for the copy. Pinned host memory gives full copy bandwidth. Caches that hold
 * a head range (model_heads > num_heads) are refused with KVC_ERR_ARG. Errors: those of
 * kvc_append_frame and kvc_attend, KVC_ERR_ARG (a NULL host buffer), KVC_ERR_CUDA (a
 * copy), and a device-side failure latched by this or an earlier step. */
KVC_API kvc_status kvc_step_host(kvc_cache* c, int32_t layer, int32_t frame_idx, int32_t is_keyframe,
                         const void* q_host, const void* k_host, const void* v_host, void* o_host);

/* The same step without waiting: enqueues the upload of Q, K, V (on an internal copy
 * stream), append + attend (on the cache's stream) and the download of O (on a second
 * internal copy stream), then returns. Two consecutive steps use different staging
 * buffers, so one step's copies overlap the neighbouring steps' compute; the streams are
 * ordered by events. The host buffers must be pinned for the copies to overlap, must stay
 * unchanged (q, k, v) and unread (o) until a synchronising call (kvc_synchronize, or any
 * call documented to synchronise) returns. The pages define no host interface; this is
 * the streaming form of kvc_step_host. Errors as for kvc_step_host; device-side errors
 * appear at the next synchronising call. */
KVC_API kvc_status kvc_step_host_async(kvc_cache* c, int32_t layer, int32_t frame_idx, int32_t is_keyframe,
                                       const void* q_host, const void* k_host, const void* v_host,
                                       void* o_host);

/* ---- Rolling diversity-pruned memory (diversity_budget = K > 0; [IVG] Building Blocks,
 * Step-by-step recipe). Requires bf16 I/O and storage, head_dim 64, page_size 16, no
 * window, no token budget, and at most 2,048 candidate slots per head:
 * (ceil(K / 16) + ceil(T / 16)) * 16 <= 2048 (T = tokens_per_frame; kvc_create returns
 * KVC_ERR_ARG otherwise). Every head keeps its own tokens: the first frame appended
 * to a layer is its immutable anchor (all heads); each later frame joins the candidates,
 * and kvc_attend first prunes each head to its Top-K candidates by diversity score
 * (negative cosine of the L2-normalised key to the mean normalised candidate key; ties to
 * the lower token id; fp64), then attends over anchor + kept. is_keyframe must be 1. */

/* Per-layer budgets (tokens per head), each in [1, diversity_budget], from the next
 * pruning on ([IVG] layer-wise adaptive budgets: the caller turns the layers' mean
 * diversities into budgets, e.g. floor(L * k * softmax(mean / tau)) for an average k;
 * diversity_budget is the largest budget a layer can take, as it sizes the pools).
 * budgets: host array of num_layers values. Errors: KVC_ERR_ARG, KVC_ERR_STATE (not in
 * this mode). */
KVC_API kvc_status kvc_set_layer_budgets(kvc_cache* c, const int32_t* budgets, int32_t n);

/* Layer-wise adaptive budgets computed by the library ([IVG] Layer-wise adaptive budgets:
 * each layer's share of the total budget is a softmax, with temperature tau, of the
 * layers' mean diversity). From every layer's last pruning, mean_l = (the heads' fp64
 * score sums, in head order) / (H x candidates), p = softmax(mean / tau) in fp64 and
 * budget_l = floor(L * k_avg * p_l), clamped to [1, diversity_budget] (a layer keeps at
 * least one token besides the anchor, and no more than its pool holds; the page states
 * neither bound). tau <= 0 gives every layer k_avg (clamped likewise). The budgets apply
 * from the next pruning, as with kvc_set_layer_budgets; budgets_out (host, num_layers
 * values) may be NULL. Synchronises. Errors: KVC_ERR_ARG (k_avg < 1, tau NaN),
 * KVC_ERR_STATE (not in this mode, or a layer never pruned). */
KVC_API kvc_status kvc_adapt_layer_budgets(kvc_cache* c, double tau, int32_t k_avg, int32_t* budgets_out);

/* The pruning step alone ([IVG] Step-by-step recipe: prune, then attend): scores every
 * head's candidates (kept tokens + the pending frame) and keeps each head's Top-K; the
 * pending frame stays pending for kvc_attend, which then only attends. Enqueued on the
 * cache's stream. Errors: KVC_ERR_ARG (bad layer), KVC_ERR_STATE (not in this mode, or
 * no frame pending); calling it twice prunes once. */
KVC_API kvc_status kvc_prune(kvc_cache* c, int32_t layer);

/* kvc_prune on every layer that has a pending frame, in one launch per run of up to 32
 * consecutive such layers (the layers' candidate sets and budgets may differ); layers
 * without a pending frame are left alone. Errors: KVC_ERR_STATE (not a rolling cache). */
KVC_API kvc_status kvc_prune_all(kvc_cache* c);

/* Mean diversity score of the layer's last pruning over all heads' candidates (fp64:
 * per head the scores summed in blocks of 32 consecutive candidates in ascending token
 * id, then the block sums in order; then the heads in order, divided by H * candidates).
 * Synchronises. Errors: KVC_ERR_STATE if the layer was never pruned. */
KVC_API kvc_status kvc_layer_diversity(kvc_cache* c, int32_t layer, double* mean_out);

/* Token ids (frame * T + slot) that head `head` of `layer` attends, in cache order
 * (anchor, then the kept tokens in ascending id, then a pending frame). ids_out: host
 * array of `capacity` entries; *n_out receives the count. Synchronises. Errors:
 * KVC_ERR_ARG (capacity too small), KVC_ERR_STATE (not in this mode). */
KVC_API kvc_status kvc_head_tokens(kvc_cache* c, int32_t layer, int32_t head, int64_t* ids_out, int32_t capacity,
                                   int32_t* n_out);

/* Wait for all work of the cache and report any latched device error. */
KVC_API kvc_status kvc_synchronize(kvc_cache* c);

/* Message for the last failing call on `c` (never NULL). */
KVC_API const char* kvc_last_error(const kvc_cache* c);

/* Name of a status code. */
KVC_API const char* kvc_status_string(kvc_status s);

/* KVC_VERSION of the built library. */
KVC_API int32_t kvc_version(void);

/* Frame attention for callers that cannot allocate device memory: code running
 * inside a CUDA-graph capture it does not own, embedded runtimes without a device
 * allocator, plug-ins whose host process forbids allocation after start-up. The pages
 * have no counterpart to this call; it exists only for such callers.
 *
 * Computes the same attention as kvc_attend, with the same tensor-core kernel, over
 * caller-owned buffers: q_dev and o_dev [tokens, num_heads, 64] bf16; k_pool_dev and
 * v_pool_dev [pool_pages][num_heads][16][64] bf16 (the layout kvc_append_frame writes);
 * page_table_dev int32 [n_pages][4] device rows (phys_page, 0, 0, valid_tokens) listing
 * the pages to attend in any order, each with 1..16 valid leading slots (slots past
 * valid_tokens must hold zeros in both K and V, as kvc_append_frame writes them). head_dim must be 64 and page_size 16; kv_splits >= 1 splits
 * the KV sequence across CTAs. Enqueued on `stream`; nothing is allocated or freed.
 *
 * Split partials live in one file-scope device array of 544 partial tiles (128 query
 * rows x 64 dims fp32 + one log-sum-exp per row) and 16,384 counters (18.17 MB in all)
 * that every GPU loading the library holds until the process exits. With kv_splits = s
 * the kernel runs G = ceil(num_heads * n / R) groups of Q = ceil(ceil(tokens / 128) / 2)
 * CTAs, n = ceil(n_pages / 8) KV tiles and R = ceil(n / s); when a head's tiles fall into
 * more than one group, the call needs 4 * G * Q partial tiles, and calls needing more
 * than 544 (or more than 16,384 counters: num_heads * ceil(tokens / 128) * 4) are
 * rejected with KVC_ERR_ARG. The first
 * call on a device looks the array's device address up (cudaGetSymbolAddress); make
 * that first call before any stream capture. All calls share the array: calls whose
 * kernels overlap on the GPU race on it. Nothing in it needs to start at zero. A wait in
 * the kernel that gives up (bounded) ends the kernel without an error report here.
 * Errors: KVC_ERR_ARG (shapes, alignment, sizes beyond the array, a softmax_scale
 * that is not positive and finite, pools of more than 2^31 - 1 rows of 16 slots per
 * head), KVC_ERR_CUDA. */
KVC_API kvc_status kvc_attend_paged_noalloc(const void* q_dev, void* o_dev, const void* k_pool_dev,
                                            const void* v_pool_dev, int64_t pool_pages,
                                            const int32_t* page_table_dev, int32_t n_pages, int32_t tokens,
                                            int32_t num_heads, int32_t head_dim, int32_t page_size,
                                            float softmax_scale, int32_t kv_splits, void* stream);

/* Test hooks for failure handling, tested without any GPU fault:
 *   kvc_debug_fail_allocs(n): the n-th next device allocation inside
 *     kvc_create reports failure (n = 0 disables), which must surface as
 *     KVC_ERR_OOM with nothing leaked.
 *   kvc_debug_bounded_wait(c, timeout_us): launches one kernel that waits on a
 *     device flag nobody sets, with the given bound; the wait gives up, the
 *     kernel records KVC_ERR_TIMEOUT in the device error word and returns,
 *     which kvc_synchronize then reports. */
KVC_API kvc_status kvc_debug_fail_allocs(int32_t n);
KVC_API kvc_status kvc_debug_bounded_wait(kvc_cache* c, int32_t timeout_us);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H_ */
