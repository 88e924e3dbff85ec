// kvc_manager.cu -- device-side page-table manager: lowest-free page allocation and
// in-place removal of page-table ranges, each as one stream-ordered single-CTA kernel.
//
// Paging follows "How GCTStream Implements Streaming 3D Reconstruction with KV Cache"
// (AggregatorStream with Paged KV Cache) and "Can LingBot-Map Achieve 20 FPS" (Page-Aligned
// Tensor Layout: a frame's K/V go straight into page-aligned storage). Which physical page
// a frame receives is not stated there; this manager always hands out the lowest free page
// ids in ascending order, so the page table is a deterministic function of the call
// sequence and can be compared bit for bit.
#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {

constexpr int kMgrThreads = 1024;

__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (kMgrThreads / 32)) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int warp_base = (warp > 0) ? s_warp[warp - 1] : 0;
  *total = s_warp[kMgrThreads / 32 - 1];
  int excl = warp_base + x - v;
  __syncthreads();
  return excl;
}

// Allocate the n_new lowest free pages of a pool and write page-table entries
// [start, start + n_new): (phys, owner, index, valid), valid = valid_full except the
// last page, which gets valid_last. Pages are marked used in the bitmap.
// One CTA per page list of a batch: list (first_layer + blockIdx.x) of the pools starting
// at `entries` / `bitmap` (strides pool_pages entries and `words` bitmap words per list);
// `group` consecutive lists share one start (the heads of a layer with per-head lists).
__global__ void __launch_bounds__(kMgrThreads) mgr_alloc_kernel(Entry* entries_all, uint32_t* bitmap_all, int words,
                                                                 int pool_pages, LayerStarts starts, int group,
                                                                 int n_new, int owner, int valid_full, int valid_last,
                                                                 int* err) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int s_warp[32];
  const int layer = starts.first_layer + blockIdx.x;
  Entry* entries = entries_all + static_cast<size_t>(layer) * pool_pages;
  uint32_t* bitmap = bitmap_all + static_cast<size_t>(layer) * words;
  const int start = starts.start[blockIdx.x / group];
  int found = 0;
  for (int chunk = 0; chunk < words && found < n_new; chunk += kMgrThreads) {
    const int w = chunk + threadIdx.x;
    uint32_t freebits = 0;
    if (w < words) {
      uint32_t used = bitmap[w];
      uint32_t valid_mask = 0xffffffffu;
      const int first = w * 32;
      if (first + 32 > pool_pages) {
        const int nv = pool_pages - first;
        valid_mask = nv <= 0 ? 0u : (nv >= 32 ? 0xffffffffu : ((1u << nv) - 1u));
      }
      freebits = ~used & valid_mask;
    }
    int total;
    const int excl = block_exclusive_scan(__popc(freebits), s_warp, &total);
    int r = found + excl;
    uint32_t taken = 0;
    uint32_t m = freebits;
    while (m && r < n_new) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int page = w * 32 + bit;
      const int valid = (r == n_new - 1) ? valid_last : valid_full;
      entries[start + r] = make_int4(page, owner, r, valid);
      taken |= 1u << bit;
      ++r;
    }
    if (taken) bitmap[w] |= taken;
    found += total;
    __syncthreads();
  }
  if (threadIdx.x == 0 && found < n_new) latch_error(err, DERR_POOL);
}

// Release the pages of entries [a, b) and close the gap: entries [b, n) move to [a, ...).
// The move runs in chunks of the block size with a barrier between the reads and the
// writes of each chunk; destinations are always below every not-yet-read source, so the
// in-place move is safe.
__global__ void __launch_bounds__(kMgrThreads) mgr_remove_kernel(Entry* entries, uint32_t* bitmap, int n, int a,
                                                                  int b, int* err) {
  griddep_wait();
  griddep_launch_dependents();
  for (int i = a + threadIdx.x; i < b; i += kMgrThreads) {
    const int page = entries[i].x;
    const uint32_t bit = 1u << (page & 31);
    const uint32_t old = atomicAnd(&bitmap[page >> 5], ~bit);
    if (!(old & bit)) latch_error(err, DERR_BOUNDS);
  }
  __syncthreads();
  const int tail = n - b;
  for (int base = 0; base < tail; base += kMgrThreads) {
    const int i = base + threadIdx.x;
    Entry v = make_int4(0, 0, 0, 0);
    if (i < tail) v = entries[b + i];
    __syncthreads();
    if (i < tail) entries[a + i] = v;
    __syncthreads();
  }
}

// Waits on a flag that nothing sets, bounded by timeout_ns of %globaltimer, then records
// a timeout in the error word and returns (the failure-handling test for bounded waits).
__global__ void debug_wait_kernel(volatile int* flag, int* err, long long timeout_ns) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const uint64_t t0 = globaltimer_ns();
  while (*flag == 0) {
    if (static_cast<long long>(globaltimer_ns() - t0) > timeout_ns) {
      latch_error(err, DERR_TIMEOUT);
      return;
    }
    __nanosleep(1000);
  }
}

cudaError_t launch_mgr_alloc(cudaStream_t s, Entry* entries, uint32_t* bitmap, int words, int pool_pages,
                             int start, int n_new, int owner, int valid_full, int valid_last, int* err) {
  LayerStarts st{};
  st.first_layer = 0;
  st.start[0] = start;
  return launch_pdl(mgr_alloc_kernel, dim3(1), dim3(kMgrThreads), 0, s,
                    entries, bitmap, words, pool_pages, st, 1, n_new, owner, valid_full, valid_last, err);
}

cudaError_t launch_mgr_alloc_layers(cudaStream_t s, Entry* entries_all, uint32_t* bitmap_all, int words,
                                    int pool_pages, const LayerStarts& starts, int n_lists, int n_new, int owner,
                                    int valid_full, int valid_last, int* err, int group) {
  return launch_pdl(mgr_alloc_kernel, dim3(n_lists), dim3(kMgrThreads), 0, s,
                    entries_all, bitmap_all, words, pool_pages, starts, group, n_new, owner, valid_full, valid_last,
                    err);
}

cudaError_t launch_mgr_remove(cudaStream_t s, Entry* entries, uint32_t* bitmap, int n_entries, int a, int b,
                              int* err) {
  return launch_pdl(mgr_remove_kernel, dim3(1), dim3(kMgrThreads), 0, s,
                    entries, bitmap, n_entries, a, b, err);
}

// One 16-byte chunk per thread over (page, head, slot past the kept tokens, chunk) for K
// and V; the first thread of each page writes its valid count.
__global__ void trim_pages_kernel(uint8_t* k_pool, uint8_t* v_pool, Entry* entries, int first, int n_pages, int keep,
                                  int H, int P, int chunks) {
  griddep_wait();
  griddep_launch_dependents();
  const long long per_tensor = static_cast<long long>(n_pages) * H * P * chunks;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < 2 * per_tensor;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const bool is_v = idx >= per_tensor;
    long long r = is_v ? idx - per_tensor : idx;
    const int ch = static_cast<int>(r % chunks);
    r /= chunks;
    const int slot = static_cast<int>(r % P);
    r /= P;
    const int h = static_cast<int>(r % H);
    const int j = static_cast<int>(r / H);
    const int kept = min(P, keep - j * P);
    const int page = entries[first + j].x;
    if (slot >= kept) {
      uint4* dst = reinterpret_cast<uint4*>((is_v ? v_pool : k_pool) +
                                            ((static_cast<long long>(page) * H + h) * P + slot) * chunks * 16);
      dst[ch] = make_uint4(0, 0, 0, 0);
    }
    if (!is_v && h == 0 && slot == 0 && ch == 0) entries[first + j].w = kept;
  }
}

cudaError_t launch_trim_pages(cudaStream_t s, uint8_t* k_pool_layer, uint8_t* v_pool_layer, Entry* entries, int first,
                              int n_pages, int keep, int H, int P, int row_bytes) {
  if (row_bytes % 16 != 0 || n_pages < 1 || keep < 1 || keep > n_pages * P) return cudaErrorInvalidValue;
  const int chunks = row_bytes / 16;
  const long long total = 2LL * n_pages * H * P * chunks;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 1184) blocks = 1184;
  return launch_pdl(trim_pages_kernel, dim3(static_cast<int>(blocks)), dim3(threads), 0, s,
                    k_pool_layer, v_pool_layer, entries, first, n_pages, keep, H, P, chunks);
}

cudaError_t launch_debug_wait(cudaStream_t s, int* flag, int* err, long long timeout_ns) {
  debug_wait_kernel<<<1, 32, 0, s>>>(flag, err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace kvc
