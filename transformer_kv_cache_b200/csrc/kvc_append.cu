// kvc_append.cu -- page-aligned append of one frame's K and V, optionally with FP8 E4M3
// absmax quantisation per (page, head).
//
// Layout ("Can LingBot-Map Achieve 20 FPS", Page-Aligned Tensor Layout): the caller's
// token-major [T, H, D] tensors are written straight into pool pages laid out as
// [page][head][slot][dim], so each (page, head) block is P*D contiguous elements: one
// TMA box for attention. Slot j of the frame goes to page j / P, offset j % P; slots past
// T in the frame's last page are written as zeros so masked columns never hold garbage.
//
// HBM-bound: every byte is read once and written once with 16-byte vector accesses,
// iterated in destination order so stores are fully coalesced and each source row of
// D elements is read by consecutive threads.
#include <cuda_bf16.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {

constexpr int kBulkAppendMaxSmem = 96 * 1024;   // two pages staged per CTA

// One thread per destination row of one tensor: (layer of the batch, tensor, page, head,
// slot), slots fastest, so a warp writes 32 consecutive rows of a (page, head) block. The
// thread decodes its indices and reads the page entry once, then moves the row 8 chunks
// of 16 bytes at a time, all 8 loads issued before their stores. Slots past T get zeros.
__global__ void append_kernel(AppendBatch in, LayerStarts starts, int n_layers, uint4* k_pool_all, uint4* v_pool_all,
                              const Entry* __restrict__ entries_all, int pool_pages, int n_pages, int T, int H,
                              int chunks_per_row, int P) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int kGroup = 8;
  const long long rows_per_tensor = static_cast<long long>(n_pages) * H * P;
  const long long total = 2 * rows_per_tensor * n_layers;
  const long long page_chunks = static_cast<long long>(H) * P * chunks_per_row;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int bl = static_cast<int>(idx / (2 * rows_per_tensor));
    long long r = idx - static_cast<long long>(bl) * 2 * rows_per_tensor;
    const bool is_v = r >= rows_per_tensor;
    if (is_v) r -= rows_per_tensor;
    const int slot = static_cast<int>(r % P);
    r /= P;
    const int h = static_cast<int>(r % H);
    const int g = static_cast<int>(r / H);
    const int tok = g * P + slot;
    const long long layer = starts.first_layer + bl;
    const int phys = __ldg(&entries_all[layer * pool_pages + starts.start[bl] + g].x);
    const uint4* src = static_cast<const uint4*>(is_v ? in.v[bl] : in.k[bl]) +
                       (static_cast<long long>(tok) * H + h) * chunks_per_row;
    uint4* dst = (is_v ? v_pool_all : k_pool_all) + (layer * pool_pages + phys) * page_chunks +
                 (static_cast<long long>(h) * P + slot) * chunks_per_row;
    for (int c0 = 0; c0 < chunks_per_row; c0 += kGroup) {
      uint4 val[kGroup];
#pragma unroll
      for (int c = 0; c < kGroup; ++c)
        if (c0 + c < chunks_per_row) val[c] = tok < T ? __ldg(src + c0 + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < kGroup; ++c)
        if (c0 + c < chunks_per_row) dst[c0 + c] = val[c];
    }
  }
}

// One CTA per (layer of the batch, tensor, page). A page's P tokens x H heads x D dims
// are contiguous in the source ([T][H][D]) and in the pool ([head][slot][dim]), so the
// CTA brings them in with one bulk copy, transposes 16-byte chunks in shared memory
// (tokens past T become zeros) and writes the page out with one bulk copy: every HBM
// byte moves in large contiguous transfers. The load wait is bounded (error word).
__global__ void __launch_bounds__(256) append_bulk_kernel(AppendBatch in, LayerStarts starts, int n_layers,
                                                          uint8_t* k_pool_all, uint8_t* v_pool_all,
                                                          const Entry* __restrict__ entries_all, int pool_pages,
                                                          int n_pages, int T, int H, int row_bytes, int P, int* err) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const int page_bytes = P * H * row_bytes;
  uint4* src_s = reinterpret_cast<uint4*>(sm);                 // [slot][head][chunk]
  uint4* dst_s = reinterpret_cast<uint4*>(sm + page_bytes);    // [head][slot][chunk]
  const int g = blockIdx.x % n_pages;
  const int tensor = (blockIdx.x / n_pages) & 1;
  const int bl = blockIdx.x / (2 * n_pages);
  const int ntok = min(P, T - g * P);
  const long long layer = starts.first_layer + bl;
  const uint8_t* src = static_cast<const uint8_t*>(tensor ? in.v[bl] : in.k[bl]) + static_cast<long long>(g) * page_bytes;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(ntok * H * row_bytes));
    bulk_load(src_s, src, static_cast<uint32_t>(ntok * H * row_bytes), &bar);
  }
  const int phys = __ldg(&entries_all[layer * pool_pages + starts.start[bl] + g].x);
  uint8_t* dst = (tensor ? v_pool_all : k_pool_all) + (layer * pool_pages + phys) * static_cast<long long>(page_bytes);
  if (!mbar_wait_bounded(&bar, 0, &abort_flag, err)) return;
  const int chunks = row_bytes / 16;
  for (int i = threadIdx.x; i < page_bytes / 16; i += blockDim.x) {
    const int q = i % chunks;
    const int r = i / chunks;
    const int slot = r % P, h = r / P;
    dst_s[i] = slot < ntok ? src_s[(slot * H + h) * chunks + q] : make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_shared();
  __syncthreads();
  if (threadIdx.x == 0) {
    bulk_store(dst, dst_s, static_cast<uint32_t>(page_bytes));
    bulk_store_wait_all();
  }
}

// Allocation fused into the append: the same CTA per (layer of the batch, tensor, page g)
// as append_bulk_kernel, which first finds its physical page itself, as the g-th free page
// (lowest first) of the layer's current bitmap. The current bitmap is only read in this
// kernel, so every CTA sees the same free set; the CTA of page 0 of K writes the next
// bitmap (the current one with the frame's pages marked used) into the layer's other
// bitmap buffer, each K CTA writes its page-table entry, and the host switches the layer to
// the other buffer. No CTA waits on another. A pool without enough free pages latches
// DERR_POOL; the CTAs whose page is missing copy nothing. Several frames of one layer (the
// joint scale-frame phase) take consecutive ranks: page g of frame f is the
// (f * n_pages + g)-th free page, so the result equals n single-frame appends in order.
__device__ __forceinline__ uint32_t free_bits(const uint32_t* bm, int w, int words, int pool_pages) {
  if (w >= words) return 0u;
  uint32_t valid = 0xffffffffu;
  const int nv = pool_pages - w * 32;
  if (nv < 32) valid = nv <= 0 ? 0u : ((1u << nv) - 1u);
  return ~bm[w] & valid;
}

__global__ void __launch_bounds__(256) append_alloc_bulk_kernel(AppendBatch in, LayerStarts starts,
                                                                unsigned long long alt_mask, int n_layers,
                                                                uint8_t* k_pool_all, uint8_t* v_pool_all,
                                                                Entry* entries_all, uint32_t* bm_main,
                                                                uint32_t* bm_alt, int words, int pool_pages,
                                                                int n_pages, int T, int H, int row_bytes, int P,
                                                                int owner, int* err, long long src_tok_bytes,
                                                                int n_frames) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  __shared__ int s_phys;
  __shared__ int s_warp[8];
  const int page_bytes = P * H * row_bytes;
  uint4* src_s = reinterpret_cast<uint4*>(sm);                 // [slot][head][chunk]
  uint4* dst_s = reinterpret_cast<uint4*>(sm + page_bytes);    // [head][slot][chunk]
  // CTA (layer of the batch, frame of the batch, tensor, page of the frame); the frame's
  // page g is the (f * n_pages + g)-th lowest free page of its layer
  const int g = blockIdx.x % n_pages;
  const int tensor = (blockIdx.x / n_pages) & 1;
  const int fb_idx = blockIdx.x / (2 * n_pages);
  const int f = fb_idx % n_frames;
  const int bl = fb_idx / n_frames;
  const int rank = f * n_pages + g;
  const int total_pages = n_frames * n_pages;
  const int ntok = min(P, T - g * P);
  const long long layer = starts.first_layer + bl;
  const bool on_alt = (alt_mask >> bl) & 1ull;
  const uint32_t* cur = (on_alt ? bm_alt : bm_main) + layer * words;
  uint32_t* next = (on_alt ? bm_main : bm_alt) + layer * words;
  // a token's H rows are contiguous in the source; tokens are src_tok_bytes apart (more than
  // H rows when the cache holds a range of the caller's heads)
  const int tok_bytes = H * row_bytes;
  const uint8_t* src = static_cast<const uint8_t*>(tensor ? in.v[bl] : in.k[bl]) +
                       (static_cast<long long>(f) * T + static_cast<long long>(g) * P) * src_tok_bytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    s_phys = -1;
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(ntok * tok_bytes));
    if (src_tok_bytes == tok_bytes) {
      bulk_load(src_s, src, static_cast<uint32_t>(ntok * tok_bytes), &bar);
    } else {
      for (int t = 0; t < ntok; ++t)
        bulk_load(reinterpret_cast<uint8_t*>(src_s) + t * tok_bytes, src + t * src_tok_bytes,
                  static_cast<uint32_t>(tok_bytes), &bar);
    }
  }
  if (warp == 0) {
    // the rank-th free page: word popcounts scanned 32 words at a time
    int found = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const uint32_t fb = free_bits(cur, w0 + lane, words, pool_pages);
      const int cnt = __popc(fb);
      int x = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const int before = found + x - cnt;
      const unsigned hit = __ballot_sync(0xffffffffu, rank >= before && rank < found + x);
      if (hit) {
        if (lane == __ffs(hit) - 1) s_phys = (w0 + lane) * 32 + static_cast<int>(__fns(fb, 0, rank - before + 1));
        break;
      }
      found += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  if (tensor == 0 && rank == 0) {
    // the next bitmap: the n_frames * n_pages lowest free pages marked used
    int found = 0;
    for (int w0 = 0; w0 < words; w0 += 256) {
      const int w = w0 + threadIdx.x;
      const uint32_t fb = free_bits(cur, w, words, pool_pages);
      const int cnt = __popc(fb);
      int x = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) s_warp[warp] = x;
      __syncthreads();
      int wbase = 0, total = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        wbase += i < warp ? s_warp[i] : 0;
        total += s_warp[i];
      }
      int r = found + wbase + x - cnt;
      uint32_t m = fb, taken = 0;
      while (m && r < total_pages) {
        const uint32_t bit = m & (0u - m);
        taken |= bit;
        m ^= bit;
        ++r;
      }
      if (w < words) next[w] = cur[w] | taken;
      found += total;
      __syncthreads();
    }
    if (threadIdx.x == 0 && found < total_pages) latch_error(err, DERR_POOL);
  }
  __syncthreads();
  const int phys = s_phys;
  if (phys < 0) {
    // no free page: the copy is dropped (DERR_POOL latched above), the load drained
    mbar_wait_drain(&bar, 0, err);
    return;
  }
  if (tensor == 0 && threadIdx.x == 0) {
    const int valid = g == n_pages - 1 ? T - (n_pages - 1) * P : P;
    entries_all[layer * pool_pages + starts.start[bl] + rank] = make_int4(phys, owner + f, g, valid);
  }
  uint8_t* dst = (tensor ? v_pool_all : k_pool_all) + (layer * pool_pages + phys) * static_cast<long long>(page_bytes);
  if (!mbar_wait_bounded(&bar, 0, &abort_flag, err)) return;
  const int chunks = row_bytes / 16;
  for (int i = threadIdx.x; i < page_bytes / 16; i += blockDim.x) {
    const int q = i % chunks;
    const int rr = i / chunks;
    const int slot = rr % P, h = rr / P;
    dst_s[i] = slot < ntok ? src_s[(slot * H + h) * chunks + q] : make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_shared();
  __syncthreads();
  if (threadIdx.x == 0) {
    bulk_store(dst, dst_s, static_cast<uint32_t>(page_bytes));
    bulk_store_wait_all();
  }
}

// Two fp32 values -> two E4M3 codes, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// One warp per (layer of the batch, page, head, tensor). The block of valid tokens x D
// dims is reduced to its absolute maximum; scale = fp32(amax / 448) with an IEEE-rounded
// division; each code is the E4M3 rounding of the IEEE-rounded fp32 quotient x / scale; an
// all-zero block has scale 0 and codes 0 ("XStreamVGGT" abstract: KV cache quantisation;
// OCP FP8 E4M3). Requires D % 8 == 0 and P * D <= 32 * 64.
// Dimension-adaptive (k_chan_all != nullptr; D = 64, P = 16): the same quantisation per
// channel of K (a scale per (page, head, channel), into k_chan_all) and per token of V (a
// scale per (page, head, slot), into v_tok_all); the page's scale is the largest of them.
// A lane then holds the 8-dim chunk lane % 8 of slots lane / 8 + 4k, k < 4: a channel's
// maximum reduces over the four lanes of its chunk, a token's over the eight of its slot.
__global__ void append_fp8_kernel(AppendBatch in, LayerStarts starts, int n_layers, uint8_t* k_pool_all,
                                  uint8_t* v_pool_all, float* k_scale_all, float* v_scale_all, float* k_chan_all,
                                  float* v_tok_all, const Entry* __restrict__ entries_all, int pool_pages,
                                  int n_pages, int T, int H, int D, int P) {
  griddep_wait();
  griddep_launch_dependents();
  const int warps_per_block = blockDim.x / 32;
  const int gw = blockIdx.x * warps_per_block + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const int per_layer = n_pages * H * 2;
  if (gw >= per_layer * n_layers) return;
  const int bl = gw / per_layer;
  const int item = gw % per_layer;
  const int tensor = item % 2;
  const int ph = item / 2;
  const int h = ph % H;
  const int g = ph / H;
  const long long layer = starts.first_layer + bl;
  const long long phys = layer * pool_pages + __ldg(&entries_all[layer * pool_pages + starts.start[bl] + g].x);
  const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(tensor ? in.v[bl] : in.k[bl]);
  uint8_t* dst = (tensor ? v_pool_all : k_pool_all) + (phys * H + h) * P * D;
  float* sc = (tensor ? v_scale_all : k_scale_all) + phys * H + h;
  const int vec_per_row = D / 8;
  const int n_vec = P * vec_per_row;     // 8-element groups in the block
  // each lane handles groups lane, lane + 32, ... (at most 8 for P*D <= 2048)
  float x[8][8];
  int nmine = 0;
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int v = lane + 32 * k;
    if (v < n_vec) {
      const int slot = v / vec_per_row, c = v % vec_per_row;
      const int tok = g * P + slot;
      if (tok < T) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + (static_cast<long long>(tok) * H + h) * D) + c);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          x[k][2 * e] = f.x;
          x[k][2 * e + 1] = f.y;
          amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[k][e] = 0.f;
      }
      nmine = k + 1;
    }
  }
  if (k_chan_all) {
    // dimension-adaptive: D = 64, P = 16, four groups per lane
    float gs[8];                                  // K: per dim of the chunk; V: per group k
    if (tensor == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float m = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) m = fmaxf(m, fabsf(x[k][e]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        gs[e] = m > 0.f ? __fdiv_rn(m, 448.0f) : 0.f;
      }
      if (lane < 8) {
        float4* cs = reinterpret_cast<float4*>(k_chan_all + (phys * H + h) * D + 8 * lane);
        cs[0] = make_float4(gs[0], gs[1], gs[2], gs[3]);
        cs[1] = make_float4(gs[4], gs[5], gs[6], gs[7]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float m = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(x[k][e]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        gs[k] = m > 0.f ? __fdiv_rn(m, 448.0f) : 0.f;
        if ((lane & 7) == 0) v_tok_all[(phys * H + h) * P + (lane >> 3) + 4 * k] = gs[k];
      }
    }
    float pm = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (tensor == 0 || e < 4) pm = fmaxf(pm, gs[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
    if (lane == 0) *sc = pm;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float s0 = tensor == 0 ? gs[2 * e] : gs[k], s1 = tensor == 0 ? gs[2 * e + 1] : gs[k];
        const float a = s0 > 0.f ? __fdiv_rn(x[k][2 * e], s0) : 0.f;
        const float b = s1 > 0.f ? __fdiv_rn(x[k][2 * e + 1], s1) : 0.f;
        w[e] = e4m3x2(a, b);
      }
      reinterpret_cast<uint2*>(dst)[lane + 32 * k] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
    }
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
  if (lane == 0) *sc = scale;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (k < nmine) {
      const int v = lane + 32 * k;
      uint2 packed = make_uint2(0, 0);
      if (scale > 0.f) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = e4m3x2(__fdiv_rn(x[k][2 * e], scale), __fdiv_rn(x[k][2 * e + 1], scale));
        packed.x = w[0] | (w[1] << 16);
        packed.y = w[2] | (w[3] << 16);
      }
      reinterpret_cast<uint2*>(dst)[v] = packed;
    }
  }
}

cudaError_t launch_append_layers(cudaStream_t s, int elem_bytes, const AppendBatch& in, const LayerStarts& starts,
                                 int n_layers, void* k_pool_all, void* v_pool_all, const Entry* entries_all,
                                 int pool_pages, int n_pages, int T, int H, int D, int P, int* err) {
  const int chunks_per_row = D * elem_bytes / 16;
  if (chunks_per_row < 1) return cudaErrorInvalidValue;
  const int page_bytes = P * H * D * elem_bytes;
  if (2 * page_bytes <= kBulkAppendMaxSmem) {
    // bulk copies through shared memory: the K/V tensors and pools are 16-byte aligned and
    // every transfer is a whole number of 16-byte rows
    static PerDeviceOnce attr;
    cudaError_t e = attr.run([] {
      return cudaFuncSetAttribute(append_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kBulkAppendMaxSmem);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(append_bulk_kernel, dim3(2 * n_layers * n_pages), dim3(256), static_cast<size_t>(2 * page_bytes),
                      s, in, starts, n_layers, static_cast<uint8_t*>(k_pool_all), static_cast<uint8_t*>(v_pool_all),
                      entries_all, pool_pages, n_pages, T, H, D * elem_bytes, P, err);
  }
  const long long total = 2LL * n_layers * n_pages * H * P;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(append_kernel, dim3(static_cast<int>(blocks)), dim3(threads), 0, s, in, starts, n_layers,
                    static_cast<uint4*>(k_pool_all), static_cast<uint4*>(v_pool_all), entries_all, pool_pages, n_pages,
                    T, H, chunks_per_row, P);
}

cudaError_t launch_append_fp8_layers(cudaStream_t s, const AppendBatch& in, const LayerStarts& starts, int n_layers,
                                     uint8_t* k_pool_all, uint8_t* v_pool_all, float* k_scale_all,
                                     float* v_scale_all, const Entry* entries_all, int pool_pages, int n_pages, int T,
                                     int H, int D, int P, float* k_chan_all, float* v_tok_all) {
  if (k_chan_all && (D != 64 || P != 16 || !v_tok_all)) return cudaErrorInvalidValue;
  const int items = n_layers * n_pages * H * 2;
  const int warps = 8;
  return launch_pdl(append_fp8_kernel, dim3((items + warps - 1) / warps), dim3(warps * 32), 0, s, in, starts,
                    n_layers, k_pool_all, v_pool_all, k_scale_all, v_scale_all, k_chan_all, v_tok_all, entries_all,
                    pool_pages, n_pages, T, H, D, P);
}

bool append_alloc_fusable(int elem_bytes, int H, int D, int P) {
  return D * elem_bytes % 16 == 0 && 2 * P * H * D * elem_bytes <= kBulkAppendMaxSmem;
}

cudaError_t launch_append_alloc_layers(cudaStream_t s, int elem_bytes, const AppendBatch& in,
                                       const LayerStarts& starts, unsigned long long alt_mask, int n_layers,
                                       void* k_pool_all, void* v_pool_all, Entry* entries_all, uint32_t* bm_main,
                                       uint32_t* bm_alt, int words, int pool_pages, int n_pages, int T, int H, int D,
                                       int P, int owner, int* err, long long src_tok_bytes, int n_frames) {
  if (!append_alloc_fusable(elem_bytes, H, D, P) || n_frames < 1) return cudaErrorInvalidValue;
  if (src_tok_bytes == 0) src_tok_bytes = static_cast<long long>(H) * D * elem_bytes;
  if (src_tok_bytes % 16) return cudaErrorInvalidValue;
  static PerDeviceOnce attr;
  cudaError_t e = attr.run([] {
    return cudaFuncSetAttribute(append_alloc_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kBulkAppendMaxSmem);
  });
  if (e != cudaSuccess) return e;
  const int page_bytes = P * H * D * elem_bytes;
  return launch_pdl(append_alloc_bulk_kernel, dim3(2 * n_layers * n_frames * n_pages), dim3(256),
                    static_cast<size_t>(2 * page_bytes), s, in, starts, alt_mask, n_layers,
                    static_cast<uint8_t*>(k_pool_all), static_cast<uint8_t*>(v_pool_all), entries_all, bm_main, bm_alt,
                    words, pool_pages, n_pages, T, H, D * elem_bytes, P, owner, err, src_tok_bytes, n_frames);
}

cudaError_t launch_append(cudaStream_t s, int elem_bytes, const void* k, const void* v, void* k_pool,
                          void* v_pool, const Entry* entries, int n_pages, int T, int H, int D, int P, int* err) {
  AppendBatch in{};
  in.k[0] = k;
  in.v[0] = v;
  LayerStarts st{};
  st.first_layer = 0;
  st.start[0] = 0;
  return launch_append_layers(s, elem_bytes, in, st, 1, k_pool, v_pool, entries, 0, n_pages, T, H, D, P, err);
}

cudaError_t launch_append_fp8(cudaStream_t s, const void* k, const void* v, uint8_t* k_pool, uint8_t* v_pool,
                              float* k_scale, float* v_scale, const Entry* entries, int n_pages, int T, int H,
                              int D, int P, float* k_chan, float* v_tok) {
  AppendBatch in{};
  in.k[0] = k;
  in.v[0] = v;
  LayerStarts st{};
  st.first_layer = 0;
  st.start[0] = 0;
  return launch_append_fp8_layers(s, in, st, 1, k_pool, v_pool, k_scale, v_scale, entries, 0, n_pages, T, H, D, P,
                                  k_chan, v_tok);
}

}  // namespace kvc
