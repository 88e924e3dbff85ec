// kvc_noalloc.cu -- paged frame attention for callers that cannot allocate device memory.
//
// kvc_attend needs scratch for the KV pieces it merges (partial outputs, log-sum-exps and
// piece counters), which a cache allocates once in kvc_create. Some callers cannot call
// cudaMalloc at all: code that runs inside a CUDA-graph capture it does not own,
// allocator-less embedded runtimes, or plug-ins whose host process forbids device
// allocations after start-up. For them, kvc_attend_paged_noalloc runs the same tensor-core
// attention kernel over caller-owned pools and page table, keeping its scratch in one fixed
// file-scope device array.
//
// The array is part of the loaded module: every GPU that loads libkvc holds
// kNoAllocScratchBytes of it until the process exits. Its device address is looked up
// once per device (cudaGetSymbolAddress, with that device current) on the first call made
// on that device; make that first call before any stream capture. All calls share the
// array and it keeps the last call's contents: each call clears the piece counters (they
// must start at zero) with cudaMemsetAsync on its stream; the partials need no clearing
// (every partial a call reads was written by the same call). Calls whose kernels overlap on
// the GPU (different streams, or different host threads) race on the array: serialise them.
#include <cuda_bf16.h>

#include <climits>
#include <cmath>
#include <mutex>

#include "kvc_internal.h"

namespace kvc {
namespace {

// Partial tiles of 128 query rows x 64 dims (fp32) plus one log-sum-exp per row, and the
// piece counters ([heads][128-row query tiles][4] ints).
constexpr size_t kNoAllocTiles = 544;
constexpr size_t kNoAllocCounters = 16384;
constexpr size_t kNoAllocPartFloats = kNoAllocTiles * 128 * 64;
constexpr size_t kNoAllocLseFloats = kNoAllocTiles * 128;
constexpr size_t kNoAllocFloats = kNoAllocPartFloats + kNoAllocLseFloats + kNoAllocCounters;
constexpr size_t kNoAllocScratchBytes = kNoAllocFloats * sizeof(float);

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];
static_assert(sizeof(g_noalloc_scratch) == kNoAllocScratchBytes, "scratch size");

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_addr[kMaxDevices] = {nullptr};
int g_sm_count[kMaxDevices] = {0};

// Host code cannot use g_noalloc_scratch's name as a device address: look the address up
// once per device, with that device current.
cudaError_t scratch_for_current_device(float** scratch, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_sm_count[dev] = n;
  }
  *scratch = g_scratch_addr[dev];
  *sms = g_sm_count[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace kvc

extern "C" kvc_status kvc_attend_paged_noalloc(const void* q_dev, void* o_dev, const void* k_pool_dev,
                                               const void* v_pool_dev, int64_t pool_pages,
                                               const int32_t* page_table_dev, int32_t n_pages,
                                               int32_t tokens, int32_t num_heads, int32_t head_dim,
                                               int32_t page_size, float softmax_scale, int32_t kv_splits,
                                               void* stream) {
  using namespace kvc;
  if (!q_dev || !o_dev || !k_pool_dev || !v_pool_dev || !page_table_dev) return KVC_ERR_ARG;
  if (head_dim != 64 || page_size != 16 || tokens < 1 || num_heads < 1 || n_pages < 1 || pool_pages < 1 ||
      !(softmax_scale > 0.f) || !std::isfinite(softmax_scale) || kv_splits < 1)
    return KVC_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(q_dev) | reinterpret_cast<uintptr_t>(o_dev) |
       reinterpret_cast<uintptr_t>(k_pool_dev) | reinterpret_cast<uintptr_t>(v_pool_dev) |
       reinterpret_cast<uintptr_t>(page_table_dev)) & 15)
    return KVC_ERR_ARG;
  // pool rows (pages x heads x slots) index the tensor maps as int: reject pools past that
  // without forming an overflowing product
  if (pool_pages > INT_MAX / (static_cast<long long>(num_heads) * page_size)) return KVC_ERR_ARG;
  if (attn_counter_count(tokens, num_heads) > kNoAllocCounters) return KVC_ERR_ARG;
  float* scratch = nullptr;
  int sms = 0;
  if (scratch_for_current_device(&scratch, &sms) != cudaSuccess) return KVC_ERR_CUDA;
  // the requested split count as the kernel runs it; one whose partials exceed the array
  // is rejected
  AttnPlan plan;
  int n_tiles = 0, pos0 = 0;
  if (!plan_attn_bf16(tokens, num_heads, &n_pages, 1, page_size, sms, kv_splits, kNoAllocTiles, true, &plan,
                      &n_tiles, &pos0))
    return KVC_ERR_ARG;
  CUtensorMap tk, tv;
  const size_t rows = static_cast<size_t>(pool_pages) * num_heads * page_size;
  if (!encode_pool_tmap(&tk, const_cast<void*>(k_pool_dev), rows, head_dim, page_size, 2, true) ||
      !encode_pool_tmap(&tv, const_cast<void*>(v_pool_dev), rows, head_dim, page_size, 2, true))
    return KVC_ERR_CUDA;
  int* counters = reinterpret_cast<int*>(scratch + kNoAllocPartFloats + kNoAllocLseFloats);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(counters, 0, attn_counter_count(tokens, num_heads) * sizeof(int), s) != cudaSuccess)
    return KVC_ERR_CUDA;
  TcAttnArgs a{};
  a.q = q_dev;
  a.o = o_dev;
  a.entries = reinterpret_cast<const Entry*>(page_table_dev);
  a.n_pages = n_pages;
  a.T = tokens;
  a.H = num_heads;
  a.P = page_size;
  a.page_base = 0;
  a.pool_rows = static_cast<long long>(rows);
  a.softmax_scale = softmax_scale;
  a.splits = kv_splits;
  a.tmap_k = &tk;
  a.tmap_v = &tv;
  a.fp8 = false;
  a.part_o = scratch;
  a.part_lse = scratch + kNoAllocPartFloats;
  a.part_rows = kNoAllocTiles;
  a.split_cnt = counters;
  a.strict_splits = true;
  a.sm_count = sms;
  a.err = nullptr;   // no error word: a wait that gives up ends the kernel without a report
  cudaError_t e = launch_attn_tc(s, a, nullptr, nullptr);
  return e == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}
