// kvc_abi.cu -- the extern "C" entry points of libkvc (declared in include/kvc.h).
//
// Host code here validates arguments, keeps the per-layer bookkeeping that decides *what*
// happens (how many pages a frame takes, which frame the sliding window evicts, whether
// compression fires) and enqueues the kernels that do it on the device: the page-table
// manager picks the physical pages and moves entries, the append / attention kernels move
// and combine the data. Nothing on this path computes on the CPU.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

using namespace kvc;

namespace {

int g_fail_allocs = 0;  // test hook: the n-th next allocation in kvc_create fails

cudaError_t dev_alloc(void** p, size_t bytes) {
  *p = nullptr;
  if (g_fail_allocs > 0 && --g_fail_allocs == 0) return cudaErrorMemoryAllocation;
  if (bytes == 0) bytes = 16;
  return cudaMalloc(p, bytes);
}

template <typename T>
cudaError_t dev_alloc_t(T** p, size_t bytes) {
  void* v = nullptr;
  cudaError_t e = dev_alloc(&v, bytes);
  *p = static_cast<T*>(v);
  return e;
}

// Piece counters of the attention kernel, for the largest query count (a frame, or the
// joint phase's S frames) and the heads of the most layers one launch takes.
size_t split_cnt_count(const kvc_config& g) {
  const long long rows = static_cast<long long>(g.tokens_per_frame) * std::max(1, g.scale_frames);
  return attn_counter_count(rows, g.num_heads * std::min(g.num_layers, kMaxAttnLayers));
}

void free_all(kvc_cache* c) {
  void* ptrs[] = {c->k_pool,     c->v_pool,     c->k_scale,    c->v_scale,    c->entries,    c->bitmap,
                  c->d_err,      c->tok_id,     c->tok_cnt,    c->tok_shat,   c->cmp_scratch, c->part_o,
                  c->part_lse,   c->stage_q[0], c->stage_k[0], c->stage_v[0], c->stage_o[0], c->stage_q[1],
                  c->stage_k[1], c->stage_v[1], c->stage_o[1], c->rank_hist, c->div_sums, c->split_cnt,
                  c->k_chan,     c->v_tok,      c->bitmap_alt, c->div_cand, c->div_budget};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  for (int i = 0; i < 2; ++i) {
    if (c->ev_up[i]) cudaEventDestroy(c->ev_up[i]);
    if (c->ev_done[i]) cudaEventDestroy(c->ev_done[i]);
    if (c->ev_down[i]) cudaEventDestroy(c->ev_down[i]);
  }
  if (c->copy_up) cudaStreamDestroy(c->copy_up);
  if (c->copy_down) cudaStreamDestroy(c->copy_down);
  for (int i = 0; i < kvc_cache::kCmpSets; ++i) {
    if (c->cmp_stream[i]) cudaStreamDestroy(c->cmp_stream[i]);
    if (c->cmp_join[i]) cudaEventDestroy(c->cmp_join[i]);
  }
  if (c->cmp_fork) cudaEventDestroy(c->cmp_fork);
}

kvc_status fail(kvc_cache* c, kvc_status s, const char* msg) {
  if (c) c->last_error = msg;
  return s;
}

kvc_status cuda_fail(kvc_cache* c, cudaError_t e, const char* where) {
  if (c) {
    c->last_error = std::string(where) + ": " + cudaGetErrorString(e);
  }
  return KVC_ERR_CUDA;
}

size_t dtype_bytes(int dt) { return dt == KVC_F32 ? 4 : (dt == KVC_BF16 ? 2 : 1); }

// A layer's page list (in per-head mode: head 0's).
Entry* layer_entries(kvc_cache* c, int layer) {
  return c->entries + static_cast<size_t>(layer) * (c->per_head ? c->cfg.num_heads : 1) * c->pool_pages;
}
uint32_t* layer_bitmap(kvc_cache* c, int layer) {
  return c->per_head ? c->bitmap + static_cast<size_t>(layer) * c->bitmap_words : layer_free_bitmap(c, layer);
}
uint8_t* layer_pool(kvc_cache* c, uint8_t* pool, int layer) {
  return pool + static_cast<size_t>(layer) * c->pool_pages * c->page_bytes_kv;
}
// Dimension-adaptive FP8 group scales of a layer (per = D for K channels, P for V tokens).
float* layer_group_scales(kvc_cache* c, float* sc, int layer, int per) {
  return sc ? sc + static_cast<size_t>(layer) * c->pool_pages * c->cfg.num_heads * per : nullptr;
}
float* layer_scale(kvc_cache* c, float* sc, int layer) {
  return sc ? sc + static_cast<size_t>(layer) * c->pool_pages * c->cfg.num_heads : nullptr;
}

kvc_status check_device_error(kvc_cache* c) {
  int err = 0;
  cudaError_t e = cudaMemcpy(&err, c->d_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "reading the device error word");
  if (err == DERR_TIMEOUT) return fail(c, KVC_ERR_TIMEOUT, "a bounded device-side wait gave up");
  if (err != 0) return fail(c, KVC_ERR_DEVICE, "device-side consistency check failed (error word set)");
  return KVC_OK;
}

kvc_status sync_and_check(kvc_cache* c) {
  cudaError_t e = cudaStreamSynchronize(c->copy_up);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->copy_down);
  if (e != cudaSuccess) return cuda_fail(c, e, "cudaStreamSynchronize");
  return check_device_error(c);
}

bool valid_layer(kvc_cache* c, int layer) { return layer >= 0 && layer < c->cfg.num_layers; }

// Remove page-table entries [a, b) of a layer (frees their pages, closes the gap).
kvc_status remove_entries(kvc_cache* c, int layer, int a, int b) {
  LayerHost& L = c->L[layer];
  cudaError_t e = launch_mgr_remove(c->stream, layer_entries(c, layer), layer_bitmap(c, layer), L.n_entries, a, b,
                                    c->d_err);
  if (e != cudaSuccess) return cuda_fail(c, e, "page-table remove");
  c->launches++;
  const int n = b - a;
  L.n_entries -= n;
  for (FrameRec& f : L.frames)
    if (f.first_entry >= b) f.first_entry -= n;
  for (FrameRec& f : L.retained)
    if (f.first_entry >= b) f.first_entry -= n;
  return KVC_OK;
}

// Pages of a frame that hold its special tokens (the first num_special_tokens tokens).
int special_pages(const kvc_config& g) {
  return g.special_frames > 0 ? (std::min(g.num_special_tokens, g.tokens_per_frame) + g.page_size - 1) / g.page_size
                              : 0;
}

// Evict a committed frame ([GCT] Sliding Window Eviction). With special-token persistence
// ([GCT] Special Token Persistence) its first special_pages() pages stay where they are,
// trimmed to the special tokens; beyond special_frames retained frames the oldest goes.
kvc_status evict_frame(kvc_cache* c, int layer, const FrameRec& f) {
  const kvc_config& g = c->cfg;
  LayerHost& L = c->L[layer];
  const int sp = special_pages(g);
  if (sp == 0) {
    L.tokens -= g.tokens_per_frame;
    return remove_entries(c, layer, f.first_entry, f.first_entry + f.n_entries);
  }
  const int ns = std::min(g.num_special_tokens, g.tokens_per_frame);
  cudaError_t e = launch_trim_pages(c->stream, layer_pool(c, c->k_pool, layer), layer_pool(c, c->v_pool, layer),
                                    layer_entries(c, layer), f.first_entry, sp, ns, g.num_heads, g.page_size,
                                    static_cast<int>(g.head_dim * c->elem_kv));
  if (e != cudaSuccess) return cuda_fail(c, e, "special-token trim");
  c->launches++;
  if (f.n_entries > sp) {
    kvc_status st = remove_entries(c, layer, f.first_entry + sp, f.first_entry + f.n_entries);
    if (st != KVC_OK) return st;
  }
  FrameRec r = f;
  r.n_entries = sp;
  L.retained.push_back(r);
  L.tokens -= g.tokens_per_frame - ns;
  if (static_cast<int>(L.retained.size()) > g.special_frames) {
    const FrameRec old = L.retained.front();
    L.retained.erase(L.retained.begin());
    L.tokens -= ns;
    return remove_entries(c, layer, old.first_entry, old.first_entry + old.n_entries);
  }
  return KVC_OK;
}

}  // namespace

namespace kvc {
// Budget-mode helpers live in kvc_compress.cu.
kvc_status compress_layer(kvc_cache* c, int layer, const float* residual, int32_t* fired);
kvc_status compress_all_layers(kvc_cache* c, const float* const* residuals, int32_t* fired);
kvc_status init_token_meta(kvc_cache* c, int layer, int first_entry, int n_pages, int frame);
kvc_status init_token_meta_layers(kvc_cache* c, const LayerStarts& st, int n_layers, int n_pages, int frame);
size_t compress_scratch_bytes(const kvc_config& cfg, int pool_pages);
}  // namespace kvc

extern "C" {

int32_t kvc_version(void) { return KVC_VERSION; }

const char* kvc_status_string(kvc_status s) {
  switch (s) {
    case KVC_OK: return "KVC_OK";
    case KVC_ERR_ARG: return "KVC_ERR_ARG";
    case KVC_ERR_OOM: return "KVC_ERR_OOM";
    case KVC_ERR_CUDA: return "KVC_ERR_CUDA";
    case KVC_ERR_STATE: return "KVC_ERR_STATE";
    case KVC_ERR_BUDGET: return "KVC_ERR_BUDGET";
    case KVC_ERR_TIMEOUT: return "KVC_ERR_TIMEOUT";
    case KVC_ERR_DEVICE: return "KVC_ERR_DEVICE";
    case KVC_ERR_UNSUPPORTED: return "KVC_ERR_UNSUPPORTED";
  }
  return "KVC_STATUS_UNKNOWN";
}

const char* kvc_last_error(const kvc_cache* c) { return c ? c->last_error.c_str() : "null cache"; }

kvc_status kvc_debug_fail_allocs(int32_t n) {
  g_fail_allocs = n < 0 ? 0 : n;
  return KVC_OK;
}

kvc_status kvc_create(const kvc_config* cfg, void* stream, kvc_cache** out) {
  if (!cfg || !out) return KVC_ERR_ARG;
  *out = nullptr;
  const kvc_config& g = *cfg;
  for (int i = 0; i < 2; ++i)
    if (g.reserved[i] != 0) return KVC_ERR_ARG;
  // a head range of the caller's tensors: bf16 window caches on the tensor-core path
  const int mh = g.model_heads > 0 ? g.model_heads : g.num_heads;
  if (g.model_heads < 0 || g.model_heads > (1 << 16) || g.head_begin < 0 || g.num_heads < 1 ||
      g.head_begin > mh - g.num_heads)
    return KVC_ERR_ARG;
  if (mh != g.num_heads &&
      (g.io_dtype != KVC_BF16 || g.kv_dtype != KVC_BF16 || g.head_dim != 64 || g.page_size != 16 ||
       g.window_frames <= 0 || g.budget_tokens > 0 || g.diversity_budget > 0))
    return KVC_ERR_ARG;
  if (g.fp8_dim_adaptive != 0 &&
      (g.fp8_dim_adaptive != 1 || g.kv_dtype != KVC_FP8_E4M3 || g.head_dim != 64 || g.page_size != 16))
    return KVC_ERR_ARG;
  if (g.special_frames < 0 || g.special_frames > (1 << 20) ||
      (g.special_frames > 0 && (g.window_frames <= 0 || g.budget_tokens > 0 || g.diversity_budget > 0)))
    return KVC_ERR_ARG;
  // the size caps keep every page count and row index below in range of int
  const bool dims_ok = g.num_layers >= 1 && g.num_heads >= 1 && g.tokens_per_frame >= 1 && g.page_size >= 1 &&
                       g.num_layers <= (1 << 16) && g.num_heads <= (1 << 16) && g.tokens_per_frame <= (1 << 24) &&
                       g.page_size <= (1 << 16) && g.window_frames <= (1 << 24) && g.scale_frames <= (1 << 24) &&
                       g.max_frames <= (1 << 24) &&
                       g.num_special_tokens >= 0 && g.num_special_tokens <= g.tokens_per_frame &&
                       g.scale_frames >= 0 && g.budget_tokens >= 0 &&
                       (g.head_dim == 16 || g.head_dim == 32 || g.head_dim == 64 || g.head_dim == 128);
  if (!dims_ok) return KVC_ERR_ARG;
  if (g.io_dtype != KVC_F32 && g.io_dtype != KVC_BF16) return KVC_ERR_ARG;
  if (!(g.kv_dtype == g.io_dtype || (g.kv_dtype == KVC_FP8_E4M3 && g.io_dtype == KVC_BF16))) return KVC_ERR_ARG;
  if (g.kv_dtype == KVC_FP8_E4M3 && g.page_size * g.head_dim > 2048) return KVC_ERR_ARG;
  if (!(g.softmax_scale > 0.f) || !std::isfinite(g.softmax_scale)) return KVC_ERR_ARG;
  if (g.window_frames > 0 && g.budget_tokens > 0) return KVC_ERR_ARG;
  if (g.budget_tokens > 0) {
    if (g.kv_dtype != KVC_BF16 || !(g.keep_frac > 0.f && g.keep_frac <= 1.f) || g.rank_window < 1 ||
        g.rank_window > 32 || g.tokens_per_frame > 12288 ||
        g.residual_dim < 1 || !(g.lambda_ >= 0.f) || g.budget_tokens > (1 << 24))
      return KVC_ERR_ARG;
  }
  if (g.diversity_budget < 0) return KVC_ERR_ARG;
  if (g.diversity_budget > 0) {
    // rolling diversity-pruned memory: bf16 tensor-core path, no window, no token budget;
    // a head's candidates (kept pages + one frame) fit the pruning kernel's shared memory
    const long long frame_pages = (g.tokens_per_frame + g.page_size - 1) / g.page_size;
    const long long kept_pages = (static_cast<long long>(g.diversity_budget) + g.page_size - 1) / g.page_size;
    if (g.io_dtype != KVC_BF16 || g.kv_dtype != KVC_BF16 || g.head_dim != 64 || g.page_size != 16 ||
        g.num_heads > kMaxBatchLayers ||
        g.window_frames > 0 || g.budget_tokens > 0 ||
        (kept_pages + frame_pages) * g.page_size > diversity_prune_max_candidates())
      return KVC_ERR_ARG;
  } else if (g.window_frames <= 0 && g.budget_tokens == 0 && g.max_frames < 1) {
    return KVC_ERR_ARG;
  }
  if (g.kv_splits < 0) return KVC_ERR_ARG;

  const int T = g.tokens_per_frame, P = g.page_size, H = g.num_heads, D = g.head_dim;
  const int ppf = (T + P - 1) / P;
  long long pool_pages;
  if (g.diversity_budget > 0) {
    // per head: the anchor frame, the kept pages and one pending frame (pruning compacts
    // the kept tokens in place)
    const long long kp = (static_cast<long long>(g.diversity_budget) + P - 1) / P;
    pool_pages = 2LL * ppf + kp + 1;
  } else if (g.window_frames > 0) {
    pool_pages = (static_cast<long long>(g.scale_frames) + g.window_frames + 1) * ppf +
                 static_cast<long long>(g.special_frames) * special_pages(g);
  } else if (g.budget_tokens > 0) {
    const long long B = g.budget_tokens;
    pool_pages = 2 * ((B + P - 1) / P) + ((B + T - 1) / T + 2) * ppf;
  } else {
    pool_pages = (static_cast<long long>(g.max_frames) + 1) * ppf;
  }
  // page counts are ints on the device; the tensor-core path addresses the pools by an int
  // row index (pages x heads x P rows over all layers)
  const long long pool_rows_all = static_cast<long long>(g.num_layers) * pool_pages * H * P;
  const bool tc_shape = g.io_dtype == KVC_BF16 && (g.kv_dtype == KVC_BF16 || g.kv_dtype == KVC_FP8_E4M3) &&
                        D == 64 && P == 16;
  if (pool_pages > (1LL << 30) || (tc_shape && pool_rows_all > INT_MAX)) return KVC_ERR_ARG;
  // a frame's and a page's elements, and the append kernels' work items (2 per page and
  // head of every layer, up to 64 threads each), are ints
  const long long model_heads = g.model_heads > 0 ? g.model_heads : H;
  if (static_cast<long long>(T) * model_heads * D * 4 > INT_MAX ||
      static_cast<long long>(P) * H * D * 4 > INT_MAX ||
      static_cast<long long>(g.num_layers) * ppf * H * 2 * 64 > INT_MAX)
    return KVC_ERR_ARG;

  kvc_cache* c = new (std::nothrow) kvc_cache();
  if (!c) return KVC_ERR_OOM;
  c->cfg = g;
  c->stream = static_cast<cudaStream_t>(stream);
  cudaGetDevice(&c->device);
  cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device);
  c->ppf = ppf;
  c->model_heads = g.model_heads > 0 ? g.model_heads : H;
  c->head0 = g.head_begin;
  c->per_head = g.diversity_budget > 0;
  if (c->per_head) c->layer_budget.assign(g.num_layers, g.diversity_budget);
  c->pool_pages = static_cast<int>(pool_pages);
  c->bitmap_words = (c->pool_pages + 31) / 32;
  c->elem_io = dtype_bytes(g.io_dtype);
  c->elem_kv = dtype_bytes(g.kv_dtype);
  if ((D * c->elem_io) % 16 != 0) {
    delete c;
    return KVC_ERR_ARG;
  }
  // pages hold all heads ([page][head][slot][dim]), or one head per sub-layer
  c->page_elems = static_cast<size_t>(c->per_head ? 1 : H) * P * D;
  c->page_bytes_kv = c->page_elems * c->elem_kv;
  const size_t L = g.num_layers;
  const size_t NS = c->per_head ? L * H : L;   // page lists (sub-layers)
  const size_t frame_bytes = static_cast<size_t>(T) * H * D * c->elem_io;
  c->tc_path = tc_shape;
  const int q_tiles = (T + 127) / 128;
  // partial tiles: 16 per (query tile, head), and at least 8 per SM (a split unit's pieces
  // take 4 per CTA of the groups that cut it)
  c->part_rows = std::max(static_cast<size_t>(q_tiles) * H * 16, static_cast<size_t>(8) * std::max(1, c->sm_count));

  cudaError_t e = cudaSuccess;
  auto A = [&](cudaError_t r) {
    if (e == cudaSuccess) e = r;
  };
  A(dev_alloc_t(&c->k_pool, NS * c->pool_pages * c->page_bytes_kv));
  A(dev_alloc_t(&c->v_pool, NS * c->pool_pages * c->page_bytes_kv));
  if (g.kv_dtype == KVC_FP8_E4M3) {
    A(dev_alloc_t(&c->k_scale, L * c->pool_pages * H * sizeof(float)));
    if (g.fp8_dim_adaptive) {
      A(dev_alloc_t(&c->k_chan, L * c->pool_pages * H * D * sizeof(float)));
      A(dev_alloc_t(&c->v_tok, L * c->pool_pages * H * P * sizeof(float)));
    }
    A(dev_alloc_t(&c->v_scale, L * c->pool_pages * H * sizeof(float)));
  }
  A(dev_alloc_t(&c->entries, NS * c->pool_pages * sizeof(Entry)));
  A(dev_alloc_t(&c->bitmap, NS * c->bitmap_words * sizeof(uint32_t)));
  if (!c->per_head) A(dev_alloc_t(&c->bitmap_alt, NS * c->bitmap_words * sizeof(uint32_t)));
  if (c->per_head) {
    A(dev_alloc_t(&c->tok_id, NS * c->pool_pages * P * sizeof(int64_t)));
    A(dev_alloc_t(&c->div_sums, NS * sizeof(double)));
    A(dev_alloc_t(&c->div_cand, L * sizeof(long long)));
    A(dev_alloc_t(&c->div_budget, L * sizeof(int32_t)));
  }
  A(dev_alloc_t(&c->d_err, 4 * sizeof(int)));
  if (c->tc_path) {
    A(dev_alloc_t(&c->part_o, c->part_rows * 128 * 64 * sizeof(float)));
    A(dev_alloc_t(&c->part_lse, c->part_rows * 128 * sizeof(float)));
    A(dev_alloc_t(&c->split_cnt, split_cnt_count(g) * sizeof(int)));
  }
  for (int i = 0; i < 2; ++i) {
    A(dev_alloc_t(&c->stage_q[i], frame_bytes));
    A(dev_alloc_t(&c->stage_k[i], frame_bytes));
    A(dev_alloc_t(&c->stage_v[i], frame_bytes));
    A(dev_alloc_t(&c->stage_o[i], frame_bytes));
  }
  A(cudaStreamCreateWithFlags(&c->copy_up, cudaStreamNonBlocking));
  A(cudaStreamCreateWithFlags(&c->copy_down, cudaStreamNonBlocking));
  for (int i = 0; i < 2; ++i) {
    A(cudaEventCreateWithFlags(&c->ev_up[i], cudaEventDisableTiming));
    A(cudaEventCreateWithFlags(&c->ev_done[i], cudaEventDisableTiming));
    A(cudaEventCreateWithFlags(&c->ev_down[i], cudaEventDisableTiming));
  }
  if (g.budget_tokens > 0) {
    const size_t slots = L * c->pool_pages * P;
    A(dev_alloc_t(&c->tok_id, slots * sizeof(int64_t)));
    A(dev_alloc_t(&c->tok_cnt, slots * sizeof(int32_t)));
    A(dev_alloc_t(&c->tok_shat, slots * sizeof(float)));
    A(dev_alloc_t(&c->rank_hist, static_cast<size_t>(g.rank_window) * T * sizeof(int32_t)));
    c->cmp_scratch_bytes = compress_scratch_bytes(g, c->pool_pages);
    A(dev_alloc(&c->cmp_scratch, c->cmp_scratch_bytes * kvc_cache::kCmpSets));
    for (int i = 0; i < kvc_cache::kCmpSets; ++i) {
      A(cudaStreamCreateWithFlags(&c->cmp_stream[i], cudaStreamNonBlocking));
      A(cudaEventCreateWithFlags(&c->cmp_join[i], cudaEventDisableTiming));
    }
    A(cudaEventCreateWithFlags(&c->cmp_fork, cudaEventDisableTiming));
  }
  if (e != cudaSuccess) {
    free_all(c);
    delete c;
    cudaGetLastError();
    return KVC_ERR_OOM;
  }
  // zero everything once so masked slots and unused pages never hold non-finite bytes
  A(cudaMemsetAsync(c->k_pool, 0, NS * c->pool_pages * c->page_bytes_kv, c->stream));
  A(cudaMemsetAsync(c->v_pool, 0, NS * c->pool_pages * c->page_bytes_kv, c->stream));
  if (c->k_scale) A(cudaMemsetAsync(c->k_scale, 0, L * c->pool_pages * H * sizeof(float), c->stream));
  if (c->v_scale) A(cudaMemsetAsync(c->v_scale, 0, L * c->pool_pages * H * sizeof(float), c->stream));
  if (c->k_chan) A(cudaMemsetAsync(c->k_chan, 0, L * c->pool_pages * H * D * sizeof(float), c->stream));
  if (c->v_tok) A(cudaMemsetAsync(c->v_tok, 0, L * c->pool_pages * H * P * sizeof(float), c->stream));
  A(cudaMemsetAsync(c->entries, 0, NS * c->pool_pages * sizeof(Entry), c->stream));
  A(cudaMemsetAsync(c->bitmap, 0, NS * c->bitmap_words * sizeof(uint32_t), c->stream));
  if (c->bitmap_alt) A(cudaMemsetAsync(c->bitmap_alt, 0, NS * c->bitmap_words * sizeof(uint32_t), c->stream));
  if (c->per_head) {
    A(cudaMemsetAsync(c->tok_id, 0xff, NS * c->pool_pages * P * sizeof(int64_t), c->stream));
    A(cudaMemsetAsync(c->div_sums, 0, NS * sizeof(double), c->stream));
  }
  A(cudaMemsetAsync(c->d_err, 0, 4 * sizeof(int), c->stream));
  if (c->split_cnt) A(cudaMemsetAsync(c->split_cnt, 0, split_cnt_count(g) * sizeof(int), c->stream));
  if (g.budget_tokens > 0) {
    const size_t slots = L * c->pool_pages * P;
    A(cudaMemsetAsync(c->tok_id, 0, slots * sizeof(int64_t), c->stream));
    A(cudaMemsetAsync(c->tok_cnt, 0, slots * sizeof(int32_t), c->stream));
    A(cudaMemsetAsync(c->tok_shat, 0, slots * sizeof(float), c->stream));
  }
  A(cudaStreamSynchronize(c->stream));
  if (e != cudaSuccess) {
    free_all(c);
    delete c;
    cudaGetLastError();
    return KVC_ERR_CUDA;
  }
  if (c->tc_path) {
    c->tmap_k.resize(1);
    c->tmap_v.resize(1);
    const size_t rows = L * c->pool_pages * H * P;
    const bool fp8 = g.kv_dtype == KVC_FP8_E4M3;
    if (!encode_pool_tmap(&c->tmap_k[0], c->k_pool, rows, D, P, fp8 ? 1 : 2, !fp8) ||
        !encode_pool_tmap(&c->tmap_v[0], c->v_pool, rows, D, P, fp8 ? 1 : 2, !fp8)) {
      free_all(c);
      delete c;
      return KVC_ERR_CUDA;
    }
  }
  c->L.assign(g.num_layers, LayerHost());
  *out = c;
  return KVC_OK;
}

kvc_status kvc_destroy(kvc_cache* c) {
  if (!c) return KVC_OK;
  cudaStreamSynchronize(c->copy_up);
  cudaStreamSynchronize(c->stream);
  cudaStreamSynchronize(c->copy_down);
  free_all(c);
  delete c;
  return KVC_OK;
}

kvc_status kvc_set_stream(kvc_cache* c, void* stream) {
  if (!c) return KVC_ERR_ARG;
  c->stream = static_cast<cudaStream_t>(stream);
  return KVC_OK;
}

kvc_status kvc_reset(kvc_cache* c) {
  if (!c) return KVC_ERR_ARG;
  const size_t L = c->cfg.num_layers;
  const size_t NS = c->per_head ? L * c->cfg.num_heads : L;
  cudaError_t e = cudaMemsetAsync(c->entries, 0, NS * c->pool_pages * sizeof(Entry), c->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->bitmap, 0, NS * c->bitmap_words * sizeof(uint32_t), c->stream);
  if (e == cudaSuccess && c->bitmap_alt)
    e = cudaMemsetAsync(c->bitmap_alt, 0, NS * c->bitmap_words * sizeof(uint32_t), c->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->d_err, 0, 4 * sizeof(int), c->stream);
  if (e == cudaSuccess && c->split_cnt)   // a launch that gave up may have left a count behind
    e = cudaMemsetAsync(c->split_cnt, 0, split_cnt_count(c->cfg) * sizeof(int), c->stream);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_reset");
  c->L.assign(c->cfg.num_layers, LayerHost());
  c->hist_frame = -1;
  c->hist_next_layer = 0;
  c->hist_layers.clear();
  return KVC_OK;
}

// ---------------------------------------------------------- rolling diversity-pruned memory
// Sub-layer (layer, head) = layer * H + head: its own page list, bitmap and pool region.
// The first frame appended to a layer is the anchor; a later frame is pending until
// kvc_attend prunes every head's candidates (kept pages + the frame's pages) to its
// Top-K ("InfiniteVGGT" explainer, Step-by-step recipe: prune, then attend).
// One frame into layers [l0, l0 + nl) (nl <= kMaxBatchLayers): one allocation launch for
// every head of every layer, one append launch.
kvc_status div_append_layers(kvc_cache* c, int l0, int nl, int frame_idx, const void* const* k_devs,
                             const void* const* v_devs) {
  const kvc_config& g = c->cfg;
  const int n = c->ppf, T = g.tokens_per_frame, P = g.page_size, H = g.num_heads;
  for (int b = 0; b < nl; ++b)
    if (c->L[l0 + b].n_entries + n > c->pool_pages) return fail(c, KVC_ERR_STATE, "kvc_append_frame: page pool full");
  LayerStarts st{};
  AppendBatch in{};
  st.first_layer = l0 * H;
  for (int b = 0; b < nl; ++b) {
    st.start[b] = c->L[l0 + b].n_entries;
    in.k[b] = k_devs[b];
    in.v[b] = v_devs[b];
  }
  cudaError_t e = launch_mgr_alloc_layers(c->stream, c->entries, c->bitmap, c->bitmap_words, c->pool_pages, st,
                                          nl * H, n, frame_idx, P, T - (n - 1) * P, c->d_err, H);
  if (e != cudaSuccess) return cuda_fail(c, e, "page allocation");
  c->launches++;
  e = launch_append_heads(c->stream, in, l0, st, nl, c->k_pool, c->v_pool, c->entries, c->tok_id, c->pool_pages, n, T,
                          H, g.head_dim, P, frame_idx);
  if (e != cudaSuccess) return cuda_fail(c, e, "append");
  c->launches++;
  for (int b = 0; b < nl; ++b) {
    LayerHost& L = c->L[l0 + b];
    if (!L.has_anchor) {
      L.anchor_pages = n;
      L.has_anchor = true;
    } else {
      L.pend_pages = n;
    }
    L.has_pending = true;
    L.pending_key = true;
    L.n_entries += n;
    L.high_water = std::max<int64_t>(L.high_water, L.n_entries);
    L.appended++;
    L.last_frame = frame_idx;
  }
  return KVC_OK;
}

// Scores every head's candidates and keeps its Top-K, for the layers [l0, l0 + n) that
// have a pending frame: each run of consecutive such layers (up to kMaxPruneLayers) in one
// launch.
kvc_status div_prune_layers(kvc_cache* c, int l0, int n) {
  const kvc_config& g = c->cfg;
  const int T = g.tokens_per_frame, P = g.page_size, H = g.num_heads;
  for (int l = l0; l < l0 + n;) {
    if (c->L[l].pend_pages == 0) {
      ++l;
      continue;
    }
    PruneLayerArgs args[kMaxPruneLayers];
    int m = 0;
    while (l + m < l0 + n && m < kMaxPruneLayers && c->L[l + m].pend_pages > 0) {
      const LayerHost& L = c->L[l + m];
      const int64_t cand = L.mut_tokens + T;
      args[m].first_cand_entry = L.anchor_pages;
      args[m].n_cand_entries = L.mut_pages + L.pend_pages;
      args[m].keep = static_cast<int>(std::min<int64_t>(c->layer_budget[l + m], cand));
      ++m;
    }
    // the kept tokens are compacted in place into the first ceil(keep / P) candidate
    // pages; the other candidate pages are freed by the kernel
    const size_t sub0 = static_cast<size_t>(l) * H * c->pool_pages;
    cudaError_t e = launch_diversity_prune_layers(
        c->stream, c->entries + sub0, c->k_pool + sub0 * c->page_bytes_kv, c->v_pool + sub0 * c->page_bytes_kv,
        c->bitmap + static_cast<size_t>(l) * H * c->bitmap_words, c->bitmap_words, c->tok_id + sub0 * P,
        c->pool_pages, args, m, H, g.head_dim, P, c->div_sums + static_cast<size_t>(l) * H, c->d_err);
    if (e != cudaSuccess) return cuda_fail(c, e, "diversity pruning");
    c->launches++;
    for (int b = 0; b < m; ++b) {
      LayerHost& L = c->L[l + b];
      const int keep = args[b].keep;
      L.n_entries = L.anchor_pages + (keep + P - 1) / P;
      L.mut_pages = (keep + P - 1) / P;
      L.cand_count = L.mut_tokens + T;
      L.mut_tokens = keep;
      L.pend_pages = 0;
      L.compressions++;
    }
    l += m;
  }
  return KVC_OK;
}

kvc_status div_prune(kvc_cache* c, int layer) { return div_prune_layers(c, layer, 1); }

kvc_status div_attend(kvc_cache* c, int layer, const void* q_dev, void* o_dev) {
  kvc_status st = div_prune(c, layer);
  if (st != KVC_OK) return st;
  LayerHost& L = c->L[layer];
  const kvc_config& g = c->cfg;
  const int T = g.tokens_per_frame, P = g.page_size, H = g.num_heads;
  const size_t sub0 = static_cast<size_t>(layer) * H * c->pool_pages;
  cudaError_t e;
  TcAttnArgs a{};
  a.q = q_dev;
  a.o = o_dev;
  a.entries = c->entries + sub0;
  a.n_pages = L.n_entries;
  a.T = T;
  a.H = H;
  a.P = P;
  a.page_base = static_cast<long long>(sub0);
  a.pool_rows = static_cast<long long>(g.num_layers) * H * c->pool_pages * P;
  a.softmax_scale = g.softmax_scale;
  a.splits = g.kv_splits;
  a.tmap_k = &c->tmap_k[0];
  a.tmap_v = &c->tmap_v[0];
  a.fp8 = false;
  a.part_o = c->part_o;
  a.part_lse = c->part_lse;
  a.part_rows = c->part_rows;
  a.split_cnt = c->split_cnt;
  a.sm_count = c->sm_count;
  a.err = c->d_err;
  a.head_pages = c->pool_pages;
  int launched = 0;
  e = launch_attn_tc(c->stream, a, nullptr, &launched);
  c->launches += launched;
  if (e != cudaSuccess) return cuda_fail(c, e, "attention launch");
  L.has_pending = false;
  L.committed++;
  L.tokens = static_cast<int64_t>(T) + L.mut_tokens;
  return KVC_OK;
}

kvc_status kvc_append_frame(kvc_cache* c, int32_t layer, int32_t frame_idx, const void* k_dev, const void* v_dev,
                            int32_t is_keyframe) {
  if (!c) return KVC_ERR_ARG;
  if (!valid_layer(c, layer) || !k_dev || !v_dev || frame_idx < 0)
    return fail(c, KVC_ERR_ARG, "kvc_append_frame: bad layer, pointer or frame index");
  if ((reinterpret_cast<uintptr_t>(k_dev) | reinterpret_cast<uintptr_t>(v_dev)) & 15)
    return fail(c, KVC_ERR_ARG, "kvc_append_frame: K and V must be 16-byte aligned");
  LayerHost& L = c->L[layer];
  if (L.has_pending) return fail(c, KVC_ERR_STATE, "kvc_append_frame: a frame is already pending on this layer");
  if (frame_idx <= L.last_frame) return fail(c, KVC_ERR_STATE, "kvc_append_frame: frame indices must increase");
  if (c->per_head) {
    if (!is_keyframe) return fail(c, KVC_ERR_ARG, "kvc_append_frame: every frame is a candidate in this mode");
    return div_append_layers(c, layer, 1, frame_idx, &k_dev, &v_dev);
  }
  const kvc_config& g = c->cfg;
  const int n = c->ppf;
  int used = 0;
  used = L.n_entries;
  if (used + n > c->pool_pages) return fail(c, KVC_ERR_STATE, "kvc_append_frame: page pool full");
  const int T = g.tokens_per_frame, P = g.page_size;
  Entry* E = layer_entries(c, layer);
  cudaError_t e;
  if (g.kv_dtype != KVC_FP8_E4M3 && append_alloc_fusable(static_cast<int>(c->elem_kv), g.num_heads, g.head_dim, P)) {
    // allocation and copy in one launch; the layer moves to its other bitmap buffer
    // (with a head range, the sources start at the first held head; tokens are model_heads
    // rows apart)
    const size_t head_off = static_cast<size_t>(c->head0) * g.head_dim * c->elem_kv;
    AppendBatch in{};
    in.k[0] = static_cast<const uint8_t*>(k_dev) + head_off;
    in.v[0] = static_cast<const uint8_t*>(v_dev) + head_off;
    LayerStarts st{};
    st.first_layer = layer;
    st.start[0] = L.n_entries;
    e = launch_append_alloc_layers(c->stream, static_cast<int>(c->elem_kv), in, st, L.bm_alt ? 1ull : 0ull, 1,
                                   c->k_pool, c->v_pool, c->entries, c->bitmap, c->bitmap_alt, c->bitmap_words,
                                   c->pool_pages, n, T, g.num_heads, g.head_dim, P, frame_idx, c->d_err,
                                   static_cast<long long>(c->model_heads) * g.head_dim * c->elem_kv);
    if (e != cudaSuccess) return cuda_fail(c, e, "append");
    c->launches++;
    L.bm_alt = !L.bm_alt;
  } else {
    e = launch_mgr_alloc(c->stream, E, layer_bitmap(c, layer), c->bitmap_words, c->pool_pages, L.n_entries, n,
                         frame_idx, P, T - (n - 1) * P, c->d_err);
    if (e != cudaSuccess) return cuda_fail(c, e, "page allocation");
    c->launches++;
  }
  if (g.kv_dtype == KVC_FP8_E4M3) {
    e = launch_append_fp8(c->stream, k_dev, v_dev, layer_pool(c, c->k_pool, layer), layer_pool(c, c->v_pool, layer),
                          layer_scale(c, c->k_scale, layer), layer_scale(c, c->v_scale, layer), E + L.n_entries, n, T,
                          g.num_heads, g.head_dim, P, layer_group_scales(c, c->k_chan, layer, g.head_dim),
                          layer_group_scales(c, c->v_tok, layer, P));
    if (e != cudaSuccess) return cuda_fail(c, e, "append");
    c->launches++;
  } else if (!append_alloc_fusable(static_cast<int>(c->elem_kv), g.num_heads, g.head_dim, P)) {
    e = launch_append(c->stream, static_cast<int>(c->elem_kv), k_dev, v_dev, layer_pool(c, c->k_pool, layer),
                      layer_pool(c, c->v_pool, layer), E + L.n_entries, n, T, g.num_heads, g.head_dim, P, c->d_err);
    if (e != cudaSuccess) return cuda_fail(c, e, "append");
    c->launches++;
  }
  if (g.budget_tokens > 0) {
    kvc_status st = init_token_meta(c, layer, L.n_entries, n, frame_idx);
    if (st != KVC_OK) return st;
  }
  L.pending.frame = frame_idx;
  L.pending.first_entry = L.n_entries;
  L.pending.n_entries = n;
  L.has_pending = true;
  L.pending_key = is_keyframe != 0;
  L.n_entries += n;
  L.high_water = std::max<int64_t>(L.high_water, L.n_entries);
  L.appended++;
  L.last_frame = frame_idx;
  return KVC_OK;
}

kvc_status kvc_append_frame_all(kvc_cache* c, int32_t frame_idx, const void* const* k_devs,
                                const void* const* v_devs, int32_t is_keyframe) {
  if (!c) return KVC_ERR_ARG;
  const kvc_config& g = c->cfg;
  if (!k_devs || !v_devs || frame_idx < 0) return fail(c, KVC_ERR_ARG, "kvc_append_frame_all: bad argument");
  if (c->per_head) {
    // one page list per head (all layers checked first)
    if (!is_keyframe) return fail(c, KVC_ERR_ARG, "kvc_append_frame_all: every frame is a candidate in this mode");
    for (int l = 0; l < g.num_layers; ++l) {
      if (!k_devs[l] || !v_devs[l] ||
          ((reinterpret_cast<uintptr_t>(k_devs[l]) | reinterpret_cast<uintptr_t>(v_devs[l])) & 15))
        return fail(c, KVC_ERR_ARG, "kvc_append_frame_all: K and V must be non-null and 16-byte aligned");
      if (c->L[l].has_pending || frame_idx <= c->L[l].last_frame)
        return fail(c, KVC_ERR_STATE, "kvc_append_frame_all: a layer cannot take the frame");
      if (c->L[l].n_entries + c->ppf > c->pool_pages)
        return fail(c, KVC_ERR_STATE, "kvc_append_frame_all: page pool full");
    }
    for (int l0 = 0; l0 < g.num_layers; l0 += kMaxBatchLayers) {
      const int nl = std::min(kMaxBatchLayers, g.num_layers - l0);
      kvc_status st = div_append_layers(c, l0, nl, frame_idx, k_devs + l0, v_devs + l0);
      if (st != KVC_OK) return st;
    }
    return KVC_OK;
  }
  const int n = c->ppf;
  for (int l = 0; l < g.num_layers; ++l) {
    if (!k_devs[l] || !v_devs[l] ||
        ((reinterpret_cast<uintptr_t>(k_devs[l]) | reinterpret_cast<uintptr_t>(v_devs[l])) & 15))
      return fail(c, KVC_ERR_ARG, "kvc_append_frame_all: K and V must be non-null and 16-byte aligned");
    const LayerHost& L = c->L[l];
    if (L.has_pending) return fail(c, KVC_ERR_STATE, "kvc_append_frame_all: a frame is already pending");
    if (frame_idx <= L.last_frame) return fail(c, KVC_ERR_STATE, "kvc_append_frame_all: frame indices must increase");
    if (L.n_entries + n > c->pool_pages) return fail(c, KVC_ERR_STATE, "kvc_append_frame_all: page pool full");
  }
  const int T = g.tokens_per_frame, P = g.page_size;
  for (int l0 = 0; l0 < g.num_layers; l0 += kMaxBatchLayers) {
    const int nl = std::min(kMaxBatchLayers, g.num_layers - l0);
    LayerStarts st{};
    AppendBatch in{};
    st.first_layer = l0;
    const size_t head_off = static_cast<size_t>(c->head0) * g.head_dim * c->elem_kv;
    for (int b = 0; b < nl; ++b) {
      st.start[b] = c->L[l0 + b].n_entries;
      in.k[b] = static_cast<const uint8_t*>(k_devs[l0 + b]) + head_off;
      in.v[b] = static_cast<const uint8_t*>(v_devs[l0 + b]) + head_off;
    }
    cudaError_t e;
    if (g.kv_dtype != KVC_FP8_E4M3 && append_alloc_fusable(static_cast<int>(c->elem_kv), g.num_heads, g.head_dim, P)) {
      // allocation and copy of every layer of the batch in one launch
      unsigned long long alt = 0;
      for (int b = 0; b < nl; ++b)
        if (c->L[l0 + b].bm_alt) alt |= 1ull << b;
      e = launch_append_alloc_layers(c->stream, static_cast<int>(c->elem_kv), in, st, alt, nl, c->k_pool, c->v_pool,
                                     c->entries, c->bitmap, c->bitmap_alt, c->bitmap_words, c->pool_pages, n, T,
                                     g.num_heads, g.head_dim, P, frame_idx, c->d_err,
                                     static_cast<long long>(c->model_heads) * g.head_dim * c->elem_kv);
      if (e != cudaSuccess) return cuda_fail(c, e, "append (all layers)");
      c->launches++;
      for (int b = 0; b < nl; ++b) c->L[l0 + b].bm_alt = !c->L[l0 + b].bm_alt;
      if (g.budget_tokens > 0) {
        kvc_status ms = init_token_meta_layers(c, st, nl, n, frame_idx);
        if (ms != KVC_OK) return ms;
      }
      continue;
    }
    // FP8 storage or pages too large for the fused kernel: never on the fused path, so every
    // layer is still on its first bitmap buffer
    e = launch_mgr_alloc_layers(c->stream, c->entries, c->bitmap, c->bitmap_words, c->pool_pages, st, nl,
                                n, frame_idx, P, T - (n - 1) * P, c->d_err);
    if (e != cudaSuccess) return cuda_fail(c, e, "page allocation (all layers)");
    c->launches++;
    if (g.kv_dtype == KVC_FP8_E4M3)
      e = launch_append_fp8_layers(c->stream, in, st, nl, c->k_pool, c->v_pool, c->k_scale, c->v_scale, c->entries,
                                   c->pool_pages, n, T, g.num_heads, g.head_dim, P, c->k_chan, c->v_tok);
    else
      e = launch_append_layers(c->stream, static_cast<int>(c->elem_kv), in, st, nl, c->k_pool, c->v_pool, c->entries,
                               c->pool_pages, n, T, g.num_heads, g.head_dim, P, c->d_err);
    if (e != cudaSuccess) return cuda_fail(c, e, "append (all layers)");
    c->launches++;
    if (g.budget_tokens > 0) {
      kvc_status ms = init_token_meta_layers(c, st, nl, n, frame_idx);
      if (ms != KVC_OK) return ms;
    }
  }
  for (int l = 0; l < g.num_layers; ++l) {
    LayerHost& L = c->L[l];
    L.pending.frame = frame_idx;
    L.pending.first_entry = L.n_entries;
    L.pending.n_entries = n;
    L.has_pending = true;
    L.pending_key = is_keyframe != 0;
    L.n_entries += n;
    L.high_water = std::max<int64_t>(L.high_water, L.n_entries);
    L.appended++;
    L.last_frame = frame_idx;
  }
  return KVC_OK;
}

// Attention of Tq query rows over every page of the layer's list (shared pages).
kvc_status attend_layer(kvc_cache* c, int layer, const void* q_dev, void* o_dev, int Tq) {
  const kvc_config& g = c->cfg;
  const int P = g.page_size, H = g.num_heads, D = g.head_dim;
  const LayerHost& L = c->L[layer];
  Entry* E = layer_entries(c, layer);
  cudaError_t e;
  if (c->tc_path) {
    TcAttnArgs a{};
    a.q = q_dev;
    a.o = o_dev;
    a.entries = E;
    a.n_pages = L.n_entries;
    a.T = Tq;
    a.H = H;
    a.P = P;
    a.page_base = static_cast<long long>(layer) * c->pool_pages;
    a.pool_rows = static_cast<long long>(g.num_layers) * c->pool_pages * H * P;
    a.softmax_scale = g.softmax_scale;
    a.splits = g.kv_splits;
    a.tmap_k = &c->tmap_k[0];
    a.tmap_v = &c->tmap_v[0];
    a.fp8 = g.kv_dtype == KVC_FP8_E4M3;
    a.q_heads = c->model_heads;
    a.head0 = c->head0;
    a.k_scale = c->k_scale;
    a.v_scale = c->v_scale;
    a.k_chan = c->k_chan;
    a.v_tok = c->v_tok;
    a.part_o = c->part_o;
    a.part_lse = c->part_lse;
    a.part_rows = c->part_rows;
    a.split_cnt = c->split_cnt;
    a.sm_count = c->sm_count;
    a.err = c->d_err;
    int launched = 0;
    e = launch_attn_tc(c->stream, a, nullptr, &launched);
    c->launches += launched;
  } else {
    e = launch_attn_simt(c->stream, g.io_dtype, g.kv_dtype, q_dev, o_dev, layer_pool(c, c->k_pool, layer),
                         layer_pool(c, c->v_pool, layer), layer_scale(c, c->k_scale, layer),
                         layer_scale(c, c->v_scale, layer), E, L.n_entries, Tq, H, D, P, g.softmax_scale);
    if (e == cudaSuccess) c->launches++;
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "attention launch");
  return KVC_OK;
}

kvc_status commit_layer(kvc_cache* c, int layer);

kvc_status kvc_attend(kvc_cache* c, int32_t layer, const void* q_dev, void* o_dev) {
  if (!c) return KVC_ERR_ARG;
  if (!valid_layer(c, layer) || !q_dev || !o_dev) return fail(c, KVC_ERR_ARG, "kvc_attend: bad layer or pointer");
  if ((reinterpret_cast<uintptr_t>(q_dev) | reinterpret_cast<uintptr_t>(o_dev)) & 15)
    return fail(c, KVC_ERR_ARG, "kvc_attend: Q and O must be 16-byte aligned");
  LayerHost& L = c->L[layer];
  if (!L.has_pending) return fail(c, KVC_ERR_STATE, "kvc_attend: no frame pending on this layer");
  if (c->per_head) return div_attend(c, layer, q_dev, o_dev);
  kvc_status ast = attend_layer(c, layer, q_dev, o_dev, c->cfg.tokens_per_frame);
  if (ast != KVC_OK) return ast;
  return commit_layer(c, layer);
}

// After a layer's attention: commit the pending frame and evict past the window, or
// release a skipped frame.
kvc_status commit_layer(kvc_cache* c, int layer) {
  const kvc_config& g = c->cfg;
  const int T = g.tokens_per_frame;
  LayerHost& L = c->L[layer];
  if (L.pending_key) {
    L.frames.push_back(L.pending);
    L.tokens += T;
    L.committed++;
    if (g.budget_tokens > 0) {
      const bool first = L.pending.frame == 0 && g.protect_first_frame;
      L.protected_tokens += first ? T : std::min(g.num_special_tokens, T);
    }
    if (g.window_frames > 0) {
      const size_t S = static_cast<size_t>(g.scale_frames), W = static_cast<size_t>(g.window_frames);
      while (L.frames.size() > S + W) {
        const FrameRec f = L.frames[S];
        L.frames.erase(L.frames.begin() + S);
        kvc_status st = evict_frame(c, layer, f);
        if (st != KVC_OK) return st;
        L.evicted++;
      }
    }
  } else {
    kvc_status st = remove_entries(c, layer, L.pending.first_entry, L.pending.first_entry + L.pending.n_entries);
    if (st != KVC_OK) return st;
    L.skipped++;
  }
  L.has_pending = false;
  return KVC_OK;
}

// Every layer's pending frame attended, as kvc_attend on each layer in order. On the
// tensor-core path (bf16 or E4M3 storage) the layers go through one launch per
// kMaxAttnLayers layers (one sweep over every layer's (head, KV tile) steps: no per-layer
// launch cost or tail); the commits follow, layer by layer.
kvc_status kvc_attend_all(kvc_cache* c, const void* const* q_devs, void* const* o_devs) {
  if (!c) return KVC_ERR_ARG;
  const kvc_config& g = c->cfg;
  if (!q_devs || !o_devs) return fail(c, KVC_ERR_ARG, "kvc_attend_all: NULL pointer array");
  for (int l = 0; l < g.num_layers; ++l) {
    if (!q_devs[l] || !o_devs[l] ||
        ((reinterpret_cast<uintptr_t>(q_devs[l]) | reinterpret_cast<uintptr_t>(o_devs[l])) & 15))
      return fail(c, KVC_ERR_ARG, "kvc_attend_all: Q and O must be non-null and 16-byte aligned");
    if (!c->L[l].has_pending) return fail(c, KVC_ERR_STATE, "kvc_attend_all: a layer has no pending frame");
  }
  const bool fp8 = g.kv_dtype == KVC_FP8_E4M3;
  const bool batch = c->tc_path && g.num_layers > 1 && !(fp8 && c->per_head);
  if (batch) {
    if (c->per_head) {
      // the pruning comes first: the page counts the attention sees are the pruned ones
      kvc_status st = div_prune_layers(c, 0, g.num_layers);
      if (st != KVC_OK) return st;
    }
  }
  if (!batch) {
    for (int l = 0; l < g.num_layers; ++l) {
      kvc_status st = kvc_attend(c, l, q_devs[l], o_devs[l]);
      if (st != KVC_OK) return st;
    }
    return KVC_OK;
  }
  const int T = g.tokens_per_frame, P = g.page_size, H = g.num_heads;
  TcAttnArgs a{};
  a.T = T;
  a.H = H;
  a.P = P;
  a.pool_rows = static_cast<long long>(g.num_layers) * c->pool_pages * H * P;
  a.softmax_scale = g.softmax_scale;
  a.splits = g.kv_splits;
  a.tmap_k = &c->tmap_k[0];
  a.tmap_v = &c->tmap_v[0];
  a.fp8 = fp8;
  a.k_scale = c->k_scale;
  a.v_scale = c->v_scale;
  a.k_chan = c->k_chan;
  a.v_tok = c->v_tok;
  a.q_heads = c->model_heads;
  a.head0 = c->head0;
  a.part_o = c->part_o;
  a.part_lse = c->part_lse;
  a.part_rows = c->part_rows;
  a.split_cnt = c->split_cnt;
  a.sm_count = c->sm_count;
  a.err = c->d_err;
  a.head_pages = c->per_head ? c->pool_pages : 0;
  for (int l0 = 0; l0 < g.num_layers; l0 += kMaxAttnLayers) {
    const int n = std::min(kMaxAttnLayers, g.num_layers - l0);
    LayerAttn la[kMaxAttnLayers];
    for (int b = 0; b < n; ++b) {
      const int l = l0 + b;
      la[b] = LayerAttn{};
      la[b].q = q_devs[l];
      la[b].o = o_devs[l];
      la[b].n_pages = c->L[l].n_entries;
      if (c->per_head) {
        const size_t sub0 = static_cast<size_t>(l) * H * c->pool_pages;
        la[b].entries = c->entries + sub0;
        la[b].page_base = static_cast<long long>(sub0);
      } else {
        la[b].entries = layer_entries(c, l);
        la[b].page_base = static_cast<long long>(l) * c->pool_pages;
      }
    }
    int launched = 0;
    cudaError_t e = launch_attn_tc_layers(c->stream, a, la, n, &launched);
    c->launches += launched;
    if (e != cudaSuccess) return cuda_fail(c, e, "attention launch (layers)");
  }
  for (int l = 0; l < g.num_layers; ++l) {
    LayerHost& L = c->L[l];
    if (c->per_head) {
      L.has_pending = false;
      L.committed++;
      L.tokens = static_cast<int64_t>(T) + L.mut_tokens;
    } else {
      kvc_status st = commit_layer(c, l);
      if (st != KVC_OK) return st;
    }
  }
  return KVC_OK;
}

kvc_status kvc_scale_phase(kvc_cache* c, int32_t layer, int32_t n_frames, const void* q_dev, const void* k_dev,
                           const void* v_dev, void* o_dev) {
  if (!c) return KVC_ERR_ARG;
  const kvc_config& g = c->cfg;
  if (!valid_layer(c, layer) || !q_dev || !k_dev || !v_dev || !o_dev || n_frames < 1 ||
      n_frames > std::max(1, g.scale_frames))
    return fail(c, KVC_ERR_ARG, "kvc_scale_phase: bad layer, pointer or frame count (1..scale_frames)");
  if ((reinterpret_cast<uintptr_t>(q_dev) | reinterpret_cast<uintptr_t>(k_dev) | reinterpret_cast<uintptr_t>(v_dev) |
       reinterpret_cast<uintptr_t>(o_dev)) & 15)
    return fail(c, KVC_ERR_ARG, "kvc_scale_phase: Q, K, V and O must be 16-byte aligned");
  if (c->per_head || g.budget_tokens > 0)
    return fail(c, KVC_ERR_STATE, "kvc_scale_phase: not with a token budget or per-head page lists");
  // the kernels index the n*T query rows' elements with ints
  if (static_cast<long long>(n_frames) * g.tokens_per_frame * c->model_heads * g.head_dim > INT_MAX)
    return fail(c, KVC_ERR_ARG, "kvc_scale_phase: more than 2^31 - 1 query elements");
  LayerHost& L = c->L[layer];
  if (L.n_entries != 0 || L.has_pending || L.last_frame >= 0)
    return fail(c, KVC_ERR_STATE, "kvc_scale_phase: the joint phase starts an empty layer");
  // frames 0 .. n-1 appended and committed, then all n*T queries over all of them
  const size_t frame_bytes = static_cast<size_t>(g.tokens_per_frame) * c->model_heads * g.head_dim * c->elem_io;
  const int n = c->ppf;
  if (L.n_entries + n_frames * n > c->pool_pages)
    return fail(c, KVC_ERR_STATE, "kvc_scale_phase: page pool full");
  if (g.kv_dtype != KVC_FP8_E4M3 &&
      append_alloc_fusable(static_cast<int>(c->elem_kv), g.num_heads, g.head_dim, g.page_size)) {
    // the n frames' allocation and copy in one launch (page g of frame f is the
    // (f * pages_per_frame + g)-th free page, as n appends in order would take it)
    const size_t head_off = static_cast<size_t>(c->head0) * g.head_dim * c->elem_kv;
    AppendBatch in{};
    in.k[0] = static_cast<const uint8_t*>(k_dev) + head_off;
    in.v[0] = static_cast<const uint8_t*>(v_dev) + head_off;
    LayerStarts st{};
    st.first_layer = layer;
    st.start[0] = L.n_entries;
    cudaError_t e = launch_append_alloc_layers(
        c->stream, static_cast<int>(c->elem_kv), in, st, L.bm_alt ? 1ull : 0ull, 1, c->k_pool, c->v_pool,
        c->entries, c->bitmap, c->bitmap_alt, c->bitmap_words, c->pool_pages, n, g.tokens_per_frame, g.num_heads,
        g.head_dim, g.page_size, 0, c->d_err, static_cast<long long>(c->model_heads) * g.head_dim * c->elem_kv,
        n_frames);
    if (e != cudaSuccess) return cuda_fail(c, e, "append (joint phase)");
    c->launches++;
    L.bm_alt = !L.bm_alt;
    for (int f = 0; f < n_frames; ++f) {
      FrameRec r;
      r.frame = f;
      r.first_entry = L.n_entries;
      r.n_entries = n;
      L.frames.push_back(r);
      L.n_entries += n;
      L.tokens += g.tokens_per_frame;
      L.appended++;
      L.committed++;
    }
    L.high_water = std::max<int64_t>(L.high_water, L.n_entries);
    L.last_frame = n_frames - 1;
    return attend_layer(c, layer, q_dev, o_dev, n_frames * g.tokens_per_frame);
  }
  for (int f = 0; f < n_frames; ++f) {
    kvc_status st = kvc_append_frame(c, layer, f, static_cast<const uint8_t*>(k_dev) + f * frame_bytes,
                                     static_cast<const uint8_t*>(v_dev) + f * frame_bytes, 1);
    if (st != KVC_OK) return st;
    L.frames.push_back(L.pending);
    L.tokens += g.tokens_per_frame;
    L.committed++;
    L.has_pending = false;
  }
  return attend_layer(c, layer, q_dev, o_dev, n_frames * g.tokens_per_frame);
}

kvc_status kvc_compress(kvc_cache* c, int32_t layer, const float* residual_dev, int32_t* fired_out) {
  if (!c) return KVC_ERR_ARG;
  if (fired_out) *fired_out = 0;
  if (!valid_layer(c, layer)) return fail(c, KVC_ERR_ARG, "kvc_compress: bad layer");
  if (c->cfg.budget_tokens <= 0) return fail(c, KVC_ERR_ARG, "kvc_compress: budget_tokens is 0");
  if (!residual_dev) return fail(c, KVC_ERR_ARG, "kvc_compress: residual is NULL");
  return compress_layer(c, layer, residual_dev, fired_out);
}

kvc_status kvc_compress_all(kvc_cache* c, const float* const* residual_devs, int32_t* fired_out) {
  if (!c) return KVC_ERR_ARG;
  const kvc_config& g = c->cfg;
  if (g.budget_tokens <= 0) return fail(c, KVC_ERR_ARG, "kvc_compress_all: budget_tokens is 0");
  if (!residual_devs) return fail(c, KVC_ERR_ARG, "kvc_compress_all: NULL residual array");
  for (int l = 0; l < g.num_layers; ++l) {
    if (fired_out) fired_out[l] = 0;
    if (!residual_devs[l]) return fail(c, KVC_ERR_ARG, "kvc_compress_all: a residual is NULL");
  }
  return compress_all_layers(c, residual_devs, fired_out);
}

kvc_status kvc_page_table(kvc_cache* c, int32_t layer, int32_t* rows_host, int32_t capacity, int32_t* n_rows,
                          kvc_info* info) {
  if (!c) return KVC_ERR_ARG;
  if (!valid_layer(c, layer)) return fail(c, KVC_ERR_ARG, "kvc_page_table: bad layer");
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  LayerHost& L = c->L[layer];
  const int n = L.n_entries;
  if (n_rows) *n_rows = n;
  if (rows_host && capacity > 0 && n > 0) {
    std::vector<Entry> tmp(n);
    cudaError_t e = cudaMemcpy(tmp.data(), layer_entries(c, layer), n * sizeof(Entry), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(c, e, "kvc_page_table copy");
    const int m = std::min(n, capacity);
    for (int i = 0; i < m; ++i) {
      rows_host[4 * i + 0] = tmp[i].y;
      rows_host[4 * i + 1] = tmp[i].z;
      rows_host[4 * i + 2] = tmp[i].x;
      rows_host[4 * i + 3] = tmp[i].w;
    }
  }
  if (info) {
    int derr = 0;
    cudaMemcpy(&derr, c->d_err, sizeof(int), cudaMemcpyDeviceToHost);
    info->tokens = L.tokens;
    info->pages_used = L.n_entries;
    info->pages_total = c->pool_pages;
    info->pool_bytes = static_cast<int64_t>(c->pool_pages) * c->page_bytes_kv * 2;
    info->high_water_pages = L.high_water;
    info->frames_appended = L.appended;
    info->frames_committed = L.committed;
    info->frames_skipped = L.skipped;
    info->frames_evicted = L.evicted;
    info->compress_events = L.compressions;
    info->device_error = derr;
    info->kernel_launches = c->launches;
  }
  return KVC_OK;
}

kvc_status kvc_token_meta(kvc_cache* c, int32_t layer, int64_t* ids_host, int32_t* counts_host, float* shat_host,
                          int32_t capacity, int32_t* n_out) {
  if (c && c->per_head) return fail(c, KVC_ERR_STATE, "not available with per-head page lists");
  if (!c) return KVC_ERR_ARG;
  if (!valid_layer(c, layer)) return fail(c, KVC_ERR_ARG, "kvc_token_meta: bad layer");
  if (!c->tok_id) return fail(c, KVC_ERR_UNSUPPORTED, "kvc_token_meta: token metadata exists in budget mode only");
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  LayerHost& L = c->L[layer];
  const int n = L.n_entries;
  std::vector<Entry> ent(n);
  if (n > 0 &&
      cudaMemcpy(ent.data(), layer_entries(c, layer), n * sizeof(Entry), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(c, KVC_ERR_CUDA, "kvc_token_meta copy");
  const int P = c->cfg.page_size;
  const size_t base = static_cast<size_t>(layer) * c->pool_pages * P;
  std::vector<int64_t> ids(static_cast<size_t>(c->pool_pages) * P);
  std::vector<int32_t> cnt(ids.size());
  std::vector<float> sh(ids.size());
  cudaError_t e = cudaMemcpy(ids.data(), c->tok_id + base, ids.size() * sizeof(int64_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess)
    e = cudaMemcpy(cnt.data(), c->tok_cnt + base, cnt.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(sh.data(), c->tok_shat + base, sh.size() * sizeof(float), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_token_meta copy");
  int k = 0;
  for (int i = 0; i < n; ++i) {
    if (ent[i].x < 0 || ent[i].x >= c->pool_pages || ent[i].w < 0 || ent[i].w > P)
      return fail(c, KVC_ERR_DEVICE, "kvc_token_meta: page-table row outside the pool");
    for (int s = 0; s < ent[i].w; ++s, ++k) {
      if (k >= capacity) continue;
      const size_t slot = static_cast<size_t>(ent[i].x) * P + s;
      if (ids_host) ids_host[k] = ids[slot];
      if (counts_host) counts_host[k] = cnt[slot];
      if (shat_host) shat_host[k] = sh[slot];
    }
  }
  if (n_out) *n_out = k;
  return KVC_OK;
}

kvc_status kvc_export_pages(kvc_cache* c, int32_t layer, int32_t first_row, int32_t n_rows, void* k_host,
                            void* v_host, float* k_scale_host, float* v_scale_host) {
  if (c && c->per_head) return fail(c, KVC_ERR_STATE, "not available with per-head page lists");
  if (!c) return KVC_ERR_ARG;
  if (!valid_layer(c, layer)) return fail(c, KVC_ERR_ARG, "kvc_export_pages: bad layer");
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  LayerHost& L = c->L[layer];
  if (first_row < 0 || n_rows < 0 || first_row > L.n_entries || n_rows > L.n_entries - first_row)
    return fail(c, KVC_ERR_ARG, "kvc_export_pages: row range outside the page table");
  std::vector<Entry> ent(n_rows);
  if (n_rows > 0 && cudaMemcpy(ent.data(), layer_entries(c, layer) + first_row, n_rows * sizeof(Entry),
                               cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(c, KVC_ERR_CUDA, "kvc_export_pages copy");
  const int H = c->cfg.num_heads;
  for (int i = 0; i < n_rows; ++i) {
    const size_t phys = ent[i].x;
    const size_t off = phys * c->page_bytes_kv;
    if (k_host)
      cudaMemcpy(static_cast<uint8_t*>(k_host) + i * c->page_bytes_kv, layer_pool(c, c->k_pool, layer) + off,
                 c->page_bytes_kv, cudaMemcpyDeviceToHost);
    if (v_host)
      cudaMemcpy(static_cast<uint8_t*>(v_host) + i * c->page_bytes_kv, layer_pool(c, c->v_pool, layer) + off,
                 c->page_bytes_kv, cudaMemcpyDeviceToHost);
    if (k_scale_host && c->k_scale)
      cudaMemcpy(k_scale_host + static_cast<size_t>(i) * H, layer_scale(c, c->k_scale, layer) + phys * H,
                 H * sizeof(float), cudaMemcpyDeviceToHost);
    if (v_scale_host && c->v_scale)
      cudaMemcpy(v_scale_host + static_cast<size_t>(i) * H, layer_scale(c, c->v_scale, layer) + phys * H,
                 H * sizeof(float), cudaMemcpyDeviceToHost);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_export_pages");
  return KVC_OK;
}

kvc_status kvc_export_fp8_group_scales(kvc_cache* c, int32_t layer, int32_t first_row, int32_t n_rows,
                                       float* k_chan_host, float* v_tok_host) {
  if (!c) return KVC_ERR_ARG;
  if (!c->k_chan) return fail(c, KVC_ERR_STATE, "kvc_export_fp8_group_scales: not dimension-adaptive FP8");
  if (!valid_layer(c, layer) || !k_chan_host || !v_tok_host)
    return fail(c, KVC_ERR_ARG, "kvc_export_fp8_group_scales: bad argument");
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  LayerHost& L = c->L[layer];
  if (first_row < 0 || n_rows < 0 || first_row > L.n_entries || n_rows > L.n_entries - first_row)
    return fail(c, KVC_ERR_ARG, "kvc_export_fp8_group_scales: row range outside the page table");
  std::vector<Entry> ent(n_rows);
  if (n_rows > 0 && cudaMemcpy(ent.data(), layer_entries(c, layer) + first_row, n_rows * sizeof(Entry),
                               cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(c, KVC_ERR_CUDA, "kvc_export_fp8_group_scales copy");
  const size_t H = c->cfg.num_heads, D = c->cfg.head_dim, P = c->cfg.page_size;
  const float* kc = layer_group_scales(c, c->k_chan, layer, static_cast<int>(D));
  const float* vt = layer_group_scales(c, c->v_tok, layer, static_cast<int>(P));
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < n_rows && e == cudaSuccess; ++i) {
    const size_t phys = ent[i].x;
    e = cudaMemcpy(k_chan_host + i * H * D, kc + phys * H * D, H * D * sizeof(float), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess)
      e = cudaMemcpy(v_tok_host + i * H * P, vt + phys * H * P, H * P * sizeof(float), cudaMemcpyDeviceToHost);
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_export_fp8_group_scales");
  return KVC_OK;
}

kvc_status kvc_step_host_async(kvc_cache* c, int32_t layer, int32_t frame_idx, int32_t is_keyframe,
                               const void* q_host, const void* k_host, const void* v_host, void* o_host) {
  if (!c) return KVC_ERR_ARG;
  if (!q_host || !k_host || !v_host || !o_host) return fail(c, KVC_ERR_ARG, "kvc_step_host: NULL host buffer");
  if (c->model_heads != c->cfg.num_heads)
    return fail(c, KVC_ERR_ARG, "kvc_step_host: host-buffer steps take caches that hold every head");
  const kvc_config& g = c->cfg;
  const size_t bytes = static_cast<size_t>(g.tokens_per_frame) * g.num_heads * g.head_dim * c->elem_io;
  const int b = c->host_slot;
  // upload once the step that last used this slot has consumed its inputs
  cudaError_t e = cudaStreamWaitEvent(c->copy_up, c->ev_done[b], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->stage_q[b], q_host, bytes, cudaMemcpyHostToDevice, c->copy_up);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->stage_k[b], k_host, bytes, cudaMemcpyHostToDevice, c->copy_up);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->stage_v[b], v_host, bytes, cudaMemcpyHostToDevice, c->copy_up);
  if (e == cudaSuccess) e = cudaEventRecord(c->ev_up[b], c->copy_up);
  // compute after the upload, and after this slot's previous output has left the device
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->stream, c->ev_up[b], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->stream, c->ev_down[b], 0);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_step_host upload");
  kvc_status st = kvc_append_frame(c, layer, frame_idx, c->stage_k[b], c->stage_v[b], is_keyframe);
  if (st != KVC_OK) return st;
  st = kvc_attend(c, layer, c->stage_q[b], c->stage_o[b]);
  if (st != KVC_OK) return st;
  e = cudaEventRecord(c->ev_done[b], c->stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->copy_down, c->ev_done[b], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(o_host, c->stage_o[b], bytes, cudaMemcpyDeviceToHost, c->copy_down);
  if (e == cudaSuccess) e = cudaEventRecord(c->ev_down[b], c->copy_down);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_step_host download");
  c->host_slot = b ^ 1;
  return KVC_OK;
}

kvc_status kvc_step_host(kvc_cache* c, int32_t layer, int32_t frame_idx, int32_t is_keyframe, const void* q_host,
                         const void* k_host, const void* v_host, void* o_host) {
  kvc_status st = kvc_step_host_async(c, layer, frame_idx, is_keyframe, q_host, k_host, v_host, o_host);
  if (st != KVC_OK) return st;
  return sync_and_check(c);
}

kvc_status kvc_set_layer_budgets(kvc_cache* c, const int32_t* budgets, int32_t n) {
  if (!c) return KVC_ERR_ARG;
  if (!c->per_head) return fail(c, KVC_ERR_STATE, "kvc_set_layer_budgets: not a diversity-pruned cache");
  if (!budgets || n != c->cfg.num_layers) return fail(c, KVC_ERR_ARG, "kvc_set_layer_budgets: one budget per layer");
  for (int l = 0; l < n; ++l)
    if (budgets[l] < 1 || budgets[l] > c->cfg.diversity_budget)
      return fail(c, KVC_ERR_ARG, "kvc_set_layer_budgets: budgets must lie in [1, diversity_budget]");
  c->layer_budget.assign(budgets, budgets + n);
  return KVC_OK;
}

kvc_status kvc_prune(kvc_cache* c, int32_t layer) {
  if (!c) return KVC_ERR_ARG;
  if (!c->per_head) return fail(c, KVC_ERR_STATE, "kvc_prune: not a diversity-pruned cache");
  if (!valid_layer(c, layer)) return fail(c, KVC_ERR_ARG, "kvc_prune: bad layer");
  if (!c->L[layer].has_pending) return fail(c, KVC_ERR_STATE, "kvc_prune: no frame pending on this layer");
  return div_prune(c, layer);
}

kvc_status kvc_prune_all(kvc_cache* c) {
  if (!c) return KVC_ERR_ARG;
  if (!c->per_head) return fail(c, KVC_ERR_STATE, "kvc_prune_all: not a diversity-pruned cache");
  return div_prune_layers(c, 0, c->cfg.num_layers);
}

kvc_status kvc_adapt_layer_budgets(kvc_cache* c, double tau, int32_t k_avg, int32_t* budgets_out) {
  if (!c) return KVC_ERR_ARG;
  if (!c->per_head) return fail(c, KVC_ERR_STATE, "kvc_adapt_layer_budgets: not a diversity-pruned cache");
  if (k_avg < 1 || !(tau == tau)) return fail(c, KVC_ERR_ARG, "kvc_adapt_layer_budgets: k_avg must be >= 1");
  const kvc_config& g = c->cfg;
  std::vector<long long> cand(g.num_layers);
  for (int l = 0; l < g.num_layers; ++l) {
    cand[l] = c->L[l].cand_count;
    if (cand[l] == 0) return fail(c, KVC_ERR_STATE, "kvc_adapt_layer_budgets: every layer must have been pruned");
  }
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  cudaError_t e = cudaMemcpy(c->div_cand, cand.data(), cand.size() * sizeof(long long), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = launch_layer_budgets(c->stream, c->div_sums, c->div_cand, g.num_layers, g.num_heads, tau, k_avg,
                             g.diversity_budget, c->div_budget);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_adapt_layer_budgets");
  c->launches++;
  std::vector<int32_t> b(g.num_layers);
  e = cudaStreamSynchronize(c->stream);
  if (e == cudaSuccess) e = cudaMemcpy(b.data(), c->div_budget, b.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_adapt_layer_budgets copy");
  c->layer_budget = b;
  if (budgets_out) std::copy(b.begin(), b.end(), budgets_out);
  return KVC_OK;
}

kvc_status kvc_layer_diversity(kvc_cache* c, int32_t layer, double* mean_out) {
  if (!c) return KVC_ERR_ARG;
  if (!c->per_head) return fail(c, KVC_ERR_STATE, "kvc_layer_diversity: not a diversity-pruned cache");
  if (!valid_layer(c, layer) || !mean_out) return fail(c, KVC_ERR_ARG, "kvc_layer_diversity: bad argument");
  const LayerHost& L = c->L[layer];
  if (L.cand_count == 0) return fail(c, KVC_ERR_STATE, "kvc_layer_diversity: the layer was never pruned");
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  const int H = c->cfg.num_heads;
  std::vector<double> sums(H);
  cudaError_t e = cudaMemcpy(sums.data(), c->div_sums + static_cast<size_t>(layer) * H, H * sizeof(double),
                             cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_layer_diversity copy");
  double tot = 0.0;
  for (int h = 0; h < H; ++h) tot += sums[h];       // heads in order
  *mean_out = tot / static_cast<double>(static_cast<int64_t>(H) * L.cand_count);
  return KVC_OK;
}

kvc_status kvc_head_tokens(kvc_cache* c, int32_t layer, int32_t head, int64_t* ids_out, int32_t capacity,
                           int32_t* n_out) {
  if (!c) return KVC_ERR_ARG;
  if (!c->per_head) return fail(c, KVC_ERR_STATE, "kvc_head_tokens: not a diversity-pruned cache");
  if (!valid_layer(c, layer) || head < 0 || head >= c->cfg.num_heads || !ids_out || !n_out)
    return fail(c, KVC_ERR_ARG, "kvc_head_tokens: bad argument");
  kvc_status st = sync_and_check(c);
  if (st != KVC_OK) return st;
  const int P = c->cfg.page_size;
  const size_t sub = (static_cast<size_t>(layer) * c->cfg.num_heads + head) * c->pool_pages;
  const int n = c->L[layer].n_entries;
  std::vector<Entry> ent(n);
  std::vector<int64_t> ids(static_cast<size_t>(c->pool_pages) * P);
  cudaError_t e = n ? cudaMemcpy(ent.data(), c->entries + sub, n * sizeof(Entry), cudaMemcpyDeviceToHost) : cudaSuccess;
  if (e == cudaSuccess)
    e = cudaMemcpy(ids.data(), c->tok_id + sub * P, ids.size() * sizeof(int64_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_head_tokens copy");
  int m = 0;
  for (int i = 0; i < n; ++i) {
    if (ent[i].x < 0 || ent[i].x >= c->pool_pages || ent[i].w < 0 || ent[i].w > P)
      return fail(c, KVC_ERR_DEVICE, "kvc_head_tokens: page-table row outside the pool");
    for (int s = 0; s < ent[i].w; ++s) {
      if (m >= capacity) return fail(c, KVC_ERR_ARG, "kvc_head_tokens: capacity too small");
      ids_out[m++] = ids[static_cast<size_t>(ent[i].x) * P + s];
    }
  }
  *n_out = m;
  return KVC_OK;
}

kvc_status kvc_synchronize(kvc_cache* c) {
  if (!c) return KVC_ERR_ARG;
  return sync_and_check(c);
}

kvc_status kvc_debug_bounded_wait(kvc_cache* c, int32_t timeout_us) {
  if (!c || timeout_us < 0) return KVC_ERR_ARG;
  cudaError_t e = launch_debug_wait(c->stream, c->d_err + 1, c->d_err, static_cast<long long>(timeout_us) * 1000);
  if (e != cudaSuccess) return cuda_fail(c, e, "kvc_debug_bounded_wait");
  c->launches++;
  return KVC_OK;
}

}  // extern "C"
