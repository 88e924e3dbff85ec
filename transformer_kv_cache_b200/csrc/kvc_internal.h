// kvc_internal.h -- host-side state of a kvc_cache and the launchers of every kernel.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>
#include <climits>
#include <vector>

#include "kvc.h"

namespace kvc {

// Launch with programmatic stream serialization: the kernel may start launching while the
// previous kernel of the stream finishes. Every kernel launched this way calls
// griddep_wait() (sm100_ptx.cuh) before it touches global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// A committed frame's pages are a contiguous run of entries in the layer's page list.
struct FrameRec {
  int32_t frame = -1;
  int32_t first_entry = 0;
  int32_t n_entries = 0;
};

struct LayerHost {
  int32_t n_entries = 0;          // entries in the device page list (block + frames + pending)
  int32_t block_entries = 0;      // leading entries written by compaction (owner -1)
  int64_t block_tokens = 0;
  std::vector<FrameRec> frames;   // committed frames after the block, in cache order
  std::vector<FrameRec> retained; // evicted frames whose special-token pages stay, oldest first
  bool has_pending = false;
  bool pending_key = false;
  FrameRec pending;
  int32_t last_frame = -1;
  int64_t tokens = 0;             // committed tokens
  int64_t high_water = 0;
  int64_t appended = 0, committed = 0, skipped = 0, evicted = 0, compressions = 0;
  bool seen_frame0 = false;       // frame 0 committed (its tokens are protected)
  int64_t protected_tokens = 0;   // committed protected tokens (compression)
  int32_t last_merge_n = 0;
  int32_t scored_frame = -1;      // frame whose residual was last scored on this layer
  // rolling diversity-pruned memory (one page list per head, all heads the same shape)
  int32_t anchor_pages = 0;       // pages of the first frame (immutable)
  int32_t mut_pages = 0;          // pages of the kept tokens (ascending id)
  int32_t pend_pages = 0;         // pages of the frame appended and not yet pruned
  int64_t mut_tokens = 0;
  int64_t cand_count = 0;         // candidates of the last pruning (per head)
  bool has_anchor = false;
  bool bm_alt = false;            // the layer's current free bitmap is Cache::bitmap_alt
};

// Device page-table entry: x = physical page, y = owner frame (-1: compaction block),
// z = page index within the owner, w = valid tokens in the page.
using Entry = int4;

struct Cache {
  kvc_config cfg{};
  cudaStream_t stream = nullptr;
  int device = 0;
  int sm_count = 148;
  int ppf = 0;                      // pages per frame
  int model_heads = 0;              // heads of the caller's tensors (the cache holds a range of them)
  int head0 = 0;                    // first model head the cache holds
  int pool_pages = 0;               // pages per layer
  int bitmap_words = 0;
  size_t elem_io = 4, elem_kv = 4;  // bytes
  size_t page_elems = 0;            // H * P * D
  size_t page_bytes_kv = 0;         // one tensor (K or V) page
  // device memory (one allocation each, all layers)
  uint8_t* k_pool = nullptr;        // [layers][pool_pages][H][P][D]
  uint8_t* v_pool = nullptr;
  float* k_scale = nullptr;         // FP8: [layers][pool_pages][H]
  float* v_scale = nullptr;
  Entry* entries = nullptr;         // [layers][pool_pages]
  uint32_t* bitmap = nullptr;       // [layers][bitmap_words]
  uint32_t* bitmap_alt = nullptr;   // [layers][bitmap_words]: the other buffer of the fused append
  int* d_err = nullptr;             // [0] error word, [1] a flag nobody sets
  // compression metadata, budget mode only: [layers][pool_pages][P]
  int64_t* tok_id = nullptr;
  int32_t* tok_cnt = nullptr;
  float* tok_shat = nullptr;
  // compression scratch: kCmpSets sets of cmp_scratch_bytes each; set 0 also holds the
  // raw scores and the merge records that kvc_last_raw_scores and kvc_last_merge read.
  // kvc_compress_all compresses layers on the side streams, set i on stream i.
  static constexpr int kCmpSets = 4;
  void* cmp_scratch = nullptr;
  size_t cmp_scratch_bytes = 0;
  cudaStream_t cmp_stream[kCmpSets] = {nullptr, nullptr, nullptr, nullptr};
  cudaEvent_t cmp_fork = nullptr;
  cudaEvent_t cmp_join[kCmpSets] = {nullptr, nullptr, nullptr, nullptr};
  // attention split scratch (partial O and log-sum-exp)
  float* k_chan = nullptr;          // dimension-adaptive FP8: [layer][page][head][D] K channel scales
  float* v_tok = nullptr;           // dimension-adaptive FP8: [layer][page][head][P] V token scales
  float* part_o = nullptr;
  float* part_lse = nullptr;
  int* split_cnt = nullptr;         // [H][q_tiles][4] attention piece counters (zero between launches)
  size_t part_rows = 0;             // capacity in 128-row partial tiles
  // host-buffer steps: two staging slots so that one step's copies overlap another's
  // compute; uploads and downloads run on their own streams, ordered by events
  uint8_t* stage_q[2] = {nullptr, nullptr};
  uint8_t* stage_k[2] = {nullptr, nullptr};
  uint8_t* stage_v[2] = {nullptr, nullptr};
  uint8_t* stage_o[2] = {nullptr, nullptr};
  cudaStream_t copy_up = nullptr, copy_down = nullptr;
  cudaEvent_t ev_up[2] = {nullptr, nullptr};      // slot's inputs uploaded
  cudaEvent_t ev_done[2] = {nullptr, nullptr};    // slot's step computed
  cudaEvent_t ev_down[2] = {nullptr, nullptr};    // slot's output downloaded
  int host_slot = 0;
  // tensor maps of each layer's K and V pools (bf16 tensor-core path)
  std::vector<CUtensorMap> tmap_k, tmap_v;
  bool tc_path = false;
  std::vector<LayerHost> L;
  std::string last_error;
  // rank history of the frame being scored (compression): [rank_window][T] int32
  int32_t* rank_hist = nullptr;
  int32_t hist_frame = -1;
  int32_t hist_next_layer = 0;
  std::vector<int> hist_layers;     // layers scored so far in the current frame
  int64_t launches = 0;             // kernels launched by this cache
  // rolling diversity-pruned memory: sub-layer (layer, head) = index layer * H + head owns
  // its own page list, bitmap and pool region of pool_pages single-head pages
  bool per_head = false;
  std::vector<int32_t> layer_budget;
  double* div_sums = nullptr;       // [layers][H] fp64 score sums of the last pruning
  long long* div_cand = nullptr;    // [layers] candidates of the last pruning (for the budgets)
  int32_t* div_budget = nullptr;    // [layers] budgets computed on the device
};

}  // namespace kvc

// The opaque handle of the C ABI is the host-side cache state.
struct kvc_cache : public kvc::Cache {};

namespace kvc {
// The current free-page bitmap of a layer (shared pages): the fused append writes the next
// bitmap into the layer's other buffer and switches to it.
inline uint32_t* layer_free_bitmap(Cache* c, int layer) {
  return (c->L[layer].bm_alt ? c->bitmap_alt : c->bitmap) + static_cast<size_t>(layer) * c->bitmap_words;
}
}  // namespace kvc

namespace kvc {

// ------------------------------------------------------------------ launchers
// Batched calls cover up to kMaxBatchLayers layers per launch (arrays passed by value).
constexpr int kMaxBatchLayers = 64;
struct LayerStarts {
  int first_layer;
  int start[kMaxBatchLayers];     // first page-table entry of the new frame, per layer of the batch
};
struct AppendBatch {
  const void* k[kMaxBatchLayers];
  const void* v[kMaxBatchLayers];
};

// Page-table manager (one CTA).
cudaError_t launch_mgr_alloc(cudaStream_t s, Entry* entries, uint32_t* bitmap, int words, int pool_pages,
                             int start, int n_new, int owner, int valid_full, int valid_last, int* err);
cudaError_t launch_mgr_alloc_layers(cudaStream_t s, Entry* entries_all, uint32_t* bitmap_all, int words,
                                    int pool_pages, const LayerStarts& starts, int n_lists, int n_new, int owner,
                                    int valid_full, int valid_last, int* err, int group = 1);
cudaError_t launch_mgr_remove(cudaStream_t s, Entry* entries, uint32_t* bitmap, int n_entries, int a, int b,
                              int* err);
// Trim entries [first, first + n_pages) to the first `keep` tokens: zero the other slots of
// every head (K and V) and set the entries' valid counts.
cudaError_t launch_trim_pages(cudaStream_t s, uint8_t* k_pool_layer, uint8_t* v_pool_layer, Entry* entries, int first,
                              int n_pages, int keep, int H, int P, int row_bytes);
cudaError_t launch_debug_wait(cudaStream_t s, int* flag, int* err, long long timeout_ns);

// Append (same dtype in and out): K, V [T,H,D] -> pages of entries [0, n_pages).
cudaError_t launch_append(cudaStream_t s, int elem_bytes, const void* k, const void* v, void* k_pool,
                          void* v_pool, const Entry* entries, int n_pages, int T, int H, int D, int P,
                          int* err = nullptr);
// Batched append of one frame to layers [starts.first_layer, + n_layers): pools and
// entries are the all-layer bases (pool_pages pages per layer).
cudaError_t launch_append_layers(cudaStream_t s, int elem_bytes, const AppendBatch& in, const LayerStarts& starts,
                                 int n_layers, void* k_pool_all, void* v_pool_all, const Entry* entries_all,
                                 int pool_pages, int n_pages, int T, int H, int D, int P, int* err = nullptr);
// Allocation and append of one frame in one launch (kvc_append.cu): for layers
// [starts.first_layer, + n_layers), the n_pages lowest free pages of each layer's current
// bitmap (bm_alt when the layer's bit of alt_mask is set, else bm_main; `words` words per
// layer) are written as entries [start, start + n_pages) with the given owner, the next
// bitmap goes to the layer's other buffer, and the frame's K/V are copied in. The caller
// then switches each layer to its other bitmap buffer.
bool append_alloc_fusable(int elem_bytes, int H, int D, int P);
// src_tok_bytes: bytes between consecutive tokens of the sources (0: H * D * elem_bytes,
// the cache holds every head); the source pointers then point at the first held head.
// n_frames > 1 (one layer's joint phase): frames owner .. owner + n_frames - 1, their
// sources T tokens apart, entries from starts.start[b] on in frame order.
cudaError_t launch_append_alloc_layers(cudaStream_t s, int elem_bytes, const AppendBatch& in,
                                       const LayerStarts& starts, unsigned long long alt_mask, int n_layers,
                                       void* k_pool_all, void* v_pool_all, Entry* entries_all, uint32_t* bm_main,
                                       uint32_t* bm_alt, int words, int pool_pages, int n_pages, int T, int H, int D,
                                       int P, int owner, int* err, long long src_tok_bytes = 0,
                                       int n_frames = 1);
cudaError_t launch_append_fp8_layers(cudaStream_t s, const AppendBatch& in, const LayerStarts& starts, int n_layers,
                                     uint8_t* k_pool_all, uint8_t* v_pool_all, float* k_scale_all,
                                     float* v_scale_all, const Entry* entries_all, int pool_pages, int n_pages, int T,
                                     int H, int D, int P, float* k_chan_all = nullptr, float* v_tok_all = nullptr);
// Append with FP8 E4M3 absmax quantisation per (page, head); bf16 input.
cudaError_t launch_append_fp8(cudaStream_t s, const void* k, const void* v, uint8_t* k_pool, uint8_t* v_pool,
                              float* k_scale, float* v_scale, const Entry* entries, int n_pages, int T, int H,
                              int D, int P, float* k_chan = nullptr, float* v_tok = nullptr);

// SIMT attention (fp32 arithmetic) over pages [0, n_pages) of a layer.
cudaError_t launch_attn_simt(cudaStream_t s, int io_dtype, int kv_dtype, const void* q, void* o,
                             const void* k_pool, const void* v_pool, const float* k_scale, const float* v_scale,
                             const Entry* entries, int n_pages, int T, int H, int D, int P, float softmax_scale);

// Tensor-core attention (bf16 or FP8 storage, D = 64).
struct TcAttnArgs {
  const void* q;
  void* o;
  const Entry* entries;
  int n_pages, T, H, P;
  long long page_base;              // first pool page of the layer (layer * pool_pages)
  long long pool_rows;              // rows (pages x heads x P) of the pool tensor maps
  float softmax_scale;
  int splits;                       // 0: choose automatically
  const CUtensorMap* tmap_k;
  const CUtensorMap* tmap_v;
  const float* k_scale;             // FP8 only
  const float* v_scale;
  bool fp8;
  float* part_o;
  float* part_lse;
  size_t part_rows;
  int sm_count;
  int* err;
  int head_pages;                   // > 0: one page list per head, head h's pages at
                                    // entries + h * head_pages, pool page index page_base +
                                    // h * head_pages + phys (single-head pages)
  const float* k_chan = nullptr;    // dimension-adaptive FP8 scales (FP8 kernel), or null
  const float* v_tok = nullptr;
  int q_heads = 0;                  // heads of the Q and O tensors (0: H); the kernel reads and
  int head0 = 0;                    // writes heads [head0, head0 + H) of them (bf16 kernel)
  int* split_cnt = nullptr;         // [H][q_tiles][4] zeroed counters (bf16 kernel): the
                                    // piece of a unit that finishes last merges, no combine
                                    // launch
  bool strict_splits = false;       // bf16: fail (cudaErrorInvalidValue) rather than use fewer
                                    // pieces when the requested split count's partials do not fit
};
// Returns the number of kernels launched through *launched.
cudaError_t launch_attn_tc(cudaStream_t s, const TcAttnArgs& a, int* splits_used, int* launched);

// Several layers in one launch of the bf16 tensor-core kernel: base carries what the layers
// share (T, H, P, the pool tensor maps, scratch, counters for n x H heads, head_pages); each
// layer its queries, outputs, page list and first pool page. At most kMaxAttnLayers layers.
constexpr int kMaxAttnLayers = 32;
struct LayerAttn {
  const void* q;
  void* o;
  const Entry* entries;
  long long page_base;
  int n_pages;
  int n_tiles;                      // set by the launcher
  int pos0;                         // first step of the layer in the flattened sweep (launcher)
  int pad;
};
struct AttnLayers {
  int n;
  int pad;
  LayerAttn l[kMaxAttnLayers];
};
cudaError_t launch_attn_tc_layers(cudaStream_t s, const TcAttnArgs& base, const LayerAttn* layers, int n,
                                  int* launched);

// Schedule of the bf16 tensor-core attention (kvc_attn_tc.cu): units are (layer, head,
// pair of 128-row query tiles); groups of q_pairs CTAs sweep R consecutive (layer, head,
// 128-slot KV tile) steps each; a unit's pieces (at most max_pieces) are merged in the
// kernel through part_tiles 128-row partial tiles and [layers x H][q_tiles][4] counters.
// n_pages[l] are the layers' page counts (per head for per-head page lists); n_tiles[l]
// and pos0[l] (the layer's first step) are written for each layer.
struct AttnPlan {
  int q_tiles, q_pairs, R, groups, grid, max_pieces;
  long long steps;                  // layers x H x their KV tiles
  size_t part_tiles;
};
bool plan_attn_bf16(int T, int H, const int* n_pages, int n_layers, int P, int sm_count, int kv_splits,
                    size_t part_tiles, bool strict, AttnPlan* out, int* n_tiles, int* pos0);

// Split counters the bf16 kernel needs for T query rows and H heads.
inline size_t attn_counter_count(long long T, int H) { return static_cast<size_t>(H) * ((T + 127) / 128) * 4; }

// Runs a set-up step (a kernel attribute, which applies per device) once for each device
// it is called on, with that device current; thread-safe; a failed step is retried on the
// next call.
constexpr int kMaxAttrDevices = 64;
struct PerDeviceOnce {
  std::mutex mu;
  bool done[kMaxAttrDevices] = {};
  template <typename F>
  cudaError_t run(F&& fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxAttrDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev]) return cudaSuccess;
    e = fn();
    if (e == cudaSuccess) done[dev] = true;
    return e;
  }
};

// Tensor map for a pool: rows of D elements, box of P rows.
bool encode_pool_tmap(CUtensorMap* map, void* base, size_t rows, int D, int P, int elem_bytes, bool swizzle128);

// Merge targets (kvc_cos_tc.cu): for each of n_src source keys, the index of the eligible
// target key of highest fp64 cosine (lowest index on ties), screened on the tensor cores.
cudaError_t launch_merge_targets(cudaStream_t s, const __nv_bfloat16* ks, const __nv_bfloat16* ke,
                                 const double* ns, const double* ne, const float* inv_ns, const float* inv_ne,
                                 int n_src, int n_elig, int HD, float* top_v, int32_t* top_j, int tiles_n,
                                 int32_t* target, int* err, int* launched);

// Rolling diversity-pruned memory (kvc_diversity.cu).
cudaError_t launch_append_heads(cudaStream_t s, const AppendBatch& in, int first_layer, const LayerStarts& starts,
                                int n_layers, void* k_pool, void* v_pool, const Entry* entries_all,
                                int64_t* tok_id_all, int pool_pages, int n_pages, int T, int H, int D, int P,
                                int frame);
int diversity_prune_max_candidates();
// Pruning of n consecutive layers of a rolling memory in one launch (blockIdx.y = layer):
// the bases are layer 0's (entries, pools, free bitmaps, token ids, score sums of its
// sub-layers); each layer's candidates are the entries [first_cand_entry,
// first_cand_entry + n_cand_entries) of every head's list, of which keep are kept.
constexpr int kMaxPruneLayers = 32;
struct PruneLayerArgs {
  int first_cand_entry, n_cand_entries, keep;
};
struct PruneLayer {
  int first, n_entries, keep, B;
};
struct PruneBatch {
  long long entries_stride, pool_stride, tok_stride, bitmap_stride;
  int sums_stride, pad;
  PruneLayer l[kMaxPruneLayers];
};
cudaError_t launch_diversity_prune_layers(cudaStream_t s, Entry* entries_base, void* k_base, void* v_base,
                                          uint32_t* bitmap_base, int words, int64_t* tok_base, int pool_pages,
                                          const PruneLayerArgs* layers, int n, int H, int D, int P,
                                          double* sums_base, int* err);

// Layer-wise adaptive budgets of the rolling memory: budget_l = clamp(floor(L * k *
// softmax(mean_l / tau)), 1, cap) from the layers' per-head score sums and candidate counts.
cudaError_t launch_layer_budgets(cudaStream_t s, const double* sums, const long long* cand, int L, int H, double tau,
                                 int k, int cap, int32_t* out);

// Compression kernels.
cudaError_t launch_score(cudaStream_t s, const float* residual, int T, int R, int layer_slot, int n_hist,
                         int32_t* rank_hist, int window, float lam, float* shat_out);
}  // namespace kvc
