// kvc_diversity.cu -- the rolling diversity-pruned memory ("InfiniteVGGT" explainer page,
// Building Blocks and Step-by-step recipe): every head keeps its own tokens, the first
// frame is an immutable anchor, and each later frame's tokens join the head's candidates,
// of which the Top-K by diversity score are kept.
//
// Layout: sub-layer (layer, head) = layer * H + head owns a page list, a free bitmap and a
// pool region of single-head pages [page][slot][dim] (bf16, P = 16, D = 64), so the
// attention kernel reads head h's pages through its own page list. The page manager's
// kernels serve the sub-layers exactly as they serve layers.
//
// Scores follow the definition in fp64 with a fixed evaluation order, so the kept sets
// match an fp64 reference bit for bit: |k| = sqrt of the squares summed over ascending
// dims; k_hat = k / |k| (0 for a zero key); mu = sum of k_hat over the candidates in
// ascending token id (the direction of the mean); score = -(k_hat . mu) / |mu| with both
// sums over ascending dims; each step one IEEE operation (explicitly rounded intrinsics,
// no contraction).
#include <cuda_bf16.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {
namespace {

constexpr int kDivThreads = 512;
constexpr int kDivD = 64;

// One 16-byte chunk per thread-iteration over (head, page, slot, chunk) of one frame, for
// K and for V; also the token ids of the frame's slots (-1 past T).
__global__ void append_heads_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* k_pool,
                                    uint4* v_pool, const Entry* __restrict__ entries_layer, int64_t* tok_id_layer,
                                    int pool_pages, int start, int n_pages, int T, int H, int P, int chunks,
                                    long long frame_base) {
  const long long per_tensor = static_cast<long long>(H) * n_pages * P * chunks;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < 2 * per_tensor;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const bool is_v = idx >= per_tensor;
    long long r = is_v ? idx - per_tensor : idx;
    const int c = static_cast<int>(r % chunks);
    r /= chunks;
    const int slot = static_cast<int>(r % P);
    r /= P;
    const int g = static_cast<int>(r % n_pages);
    const int h = static_cast<int>(r / n_pages);
    const long long sub = static_cast<long long>(h) * pool_pages;
    const int phys = __ldg(&entries_layer[sub + start + g].x);
    const int tok = g * P + slot;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (tok < T) val = __ldg(&(is_v ? v : k)[(static_cast<long long>(tok) * H + h) * chunks + c]);
    const long long dst = ((sub + phys) * P + slot) * chunks + c;
    (is_v ? v_pool : k_pool)[dst] = val;
    if (!is_v && c == 0) tok_id_layer[(sub + phys) * P + slot] = tok < T ? frame_base + tok : -1;
  }
}

// One CTA per head of the layer. Candidates: the slots of page-list entries
// [first, first + n_entries) of the head (the kept pages, then the new frame's pages),
// in ascending token id. Keeps the `keep` best by (score descending, id ascending),
// writes them in ascending id into the head's pages at entries [new_entry, ...), zeroes
// the tail slots of the last new page, and stores the head's score sum (ascending id).
__global__ void __launch_bounds__(kDivThreads) diversity_prune_kernel(
    const Entry* __restrict__ entries_layer, const __nv_bfloat16* __restrict__ k_pool,
    const __nv_bfloat16* __restrict__ v_pool, __nv_bfloat16* k_pool_w, __nv_bfloat16* v_pool_w, int64_t* tok_id_layer,
    int pool_pages, int first, int n_entries, int new_entry, int keep, int P, double* sums_layer, int* err) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int h = blockIdx.x;
  const long long sub = static_cast<long long>(h) * pool_pages;
  const Entry* E = entries_layer + sub;
  __shared__ int s_off[1025];
  __shared__ double s_mu[kDivD];
  __shared__ double s_mnorm;
  __shared__ int s_n;
  __shared__ int s_warp[32];
  // candidate slots (offset of each entry's first candidate: one thread, <= 1024 entries)
  if (threadIdx.x == 0) {
    int o = 0;
    for (int e = 0; e < n_entries; ++e) {
      s_off[e] = o;
      o += E[first + e].w;
    }
    s_off[n_entries] = o;
    s_n = o;
  }
  __syncthreads();
  const int N = s_n;
  int32_t* c_slot = reinterpret_cast<int32_t*>(sm);                      // [N] pool slot within the head
  double* c_norm = reinterpret_cast<double*>(sm + ((static_cast<size_t>(N) * 4 + 15) & ~size_t(15)));
  double* c_score = c_norm + N;
  int64_t* c_id = reinterpret_cast<int64_t*>(c_score + N);
  int32_t* c_keep = reinterpret_cast<int32_t*>(c_id + N);
  for (int e = threadIdx.x; e < n_entries; e += blockDim.x) {
    const Entry en = E[first + e];
    for (int s = 0; s < en.w; ++s) {
      const int i = s_off[e] + s;
      c_slot[i] = en.x * P + s;
      c_id[i] = tok_id_layer[(sub + en.x) * P + s];
    }
  }
  __syncthreads();
  auto krow = [&](int i) { return k_pool + (sub * P + c_slot[i]) * kDivD; };
  // norms: squares summed over ascending dims
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const __nv_bfloat16* kr = krow(i);
    double acc = 0.0;
    for (int d = 0; d < kDivD; ++d) {
      const double x = static_cast<double>(__bfloat162float(kr[d]));
      acc = __dadd_rn(acc, __dmul_rn(x, x));
    }
    c_norm[i] = __dsqrt_rn(acc);
  }
  __syncthreads();
  // mu_d: normalised keys summed over ascending candidates (one thread per dim)
  if (threadIdx.x < kDivD) {
    const int d = threadIdx.x;
    double mu = 0.0;
    for (int i = 0; i < N; ++i) {
      const double n = c_norm[i];
      const double kh = n > 0.0 ? __ddiv_rn(static_cast<double>(__bfloat162float(krow(i)[d])), n) : 0.0;
      mu = __dadd_rn(mu, kh);
    }
    s_mu[d] = mu;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double m2 = 0.0;
    for (int d = 0; d < kDivD; ++d) m2 = __dadd_rn(m2, __dmul_rn(s_mu[d], s_mu[d]));
    s_mnorm = __dsqrt_rn(m2);
  }
  __syncthreads();
  const double mnorm = s_mnorm;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    double sc = 0.0;
    const double n = c_norm[i];
    if (mnorm > 0.0) {
      const __nv_bfloat16* kr = krow(i);
      double dot = 0.0;
      for (int d = 0; d < kDivD; ++d) {
        const double kh = n > 0.0 ? __ddiv_rn(static_cast<double>(__bfloat162float(kr[d])), n) : 0.0;
        dot = __dadd_rn(dot, __dmul_rn(kh, s_mu[d]));
      }
      sc = -__ddiv_rn(dot, mnorm);
    }
    c_score[i] = sc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < N; ++i) s = __dadd_rn(s, c_score[i]);
    sums_layer[h] = s;
  }
  // rank by counting: (score descending, id ascending) is a strict total order
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const double si = c_score[i];
    const int64_t ii = c_id[i];
    int r = 0;
    for (int j = 0; j < N; ++j) {
      const double sj = c_score[j];
      r += (sj > si) || (sj == si && c_id[j] < ii);
    }
    c_keep[i] = r < keep;
  }
  __syncthreads();
  // compaction: kept candidates in ascending id (= candidate order) into the new pages
  int base = 0;
  for (int chunk = 0; chunk < N; chunk += blockDim.x) {
    const int i = chunk + threadIdx.x;
    const int f = i < N ? c_keep[i] : 0;
    int x = f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const int pos = base + (warp > 0 ? s_warp[warp - 1] : 0) + x - f;
    const int total = s_warp[nw - 1];
    if (f) {
      if (pos >= keep) latch_error(err, DERR_BOUNDS);
      else {
        const int phys = E[new_entry + pos / P].x;
        const long long dst = (sub + phys) * P + pos % P;
        const long long src = sub * P + c_slot[i];
        const uint4* ks = reinterpret_cast<const uint4*>(k_pool + src * kDivD);
        const uint4* vs = reinterpret_cast<const uint4*>(v_pool + src * kDivD);
        uint4* kd = reinterpret_cast<uint4*>(k_pool_w + dst * kDivD);
        uint4* vd = reinterpret_cast<uint4*>(v_pool_w + dst * kDivD);
#pragma unroll
        for (int q = 0; q < kDivD / 8; ++q) {
          kd[q] = ks[q];
          vd[q] = vs[q];
        }
        tok_id_layer[dst] = c_id[i];
      }
    }
    base += total;
    __syncthreads();
  }
  // the last new page's slots past the kept count: zero K and V, no token
  const int n_new = (keep + P - 1) / P;
  const int tail0 = keep, tail1 = n_new * P;
  for (int t = tail0 + static_cast<int>(threadIdx.x); t < tail1; t += blockDim.x) {
    const int phys = E[new_entry + t / P].x;
    const long long dst = (sub + phys) * P + t % P;
    uint4* kd = reinterpret_cast<uint4*>(k_pool_w + dst * kDivD);
    uint4* vd = reinterpret_cast<uint4*>(v_pool_w + dst * kDivD);
#pragma unroll
    for (int q = 0; q < kDivD / 8; ++q) {
      kd[q] = make_uint4(0, 0, 0, 0);
      vd[q] = make_uint4(0, 0, 0, 0);
    }
    tok_id_layer[dst] = -1;
  }
}

}  // namespace

size_t diversity_prune_smem(int n_cand) {
  const size_t a = (static_cast<size_t>(n_cand) * 4 + 15) & ~size_t(15);
  return a + static_cast<size_t>(n_cand) * (8 + 8 + 8 + 4);
}

cudaError_t launch_append_heads(cudaStream_t s, const void* k, const void* v, void* k_pool, void* v_pool,
                                const Entry* entries_layer, int64_t* tok_id_layer, int pool_pages, int start,
                                int n_pages, int T, int H, int D, int P, int frame) {
  const int chunks = D * 2 / 16;
  const long long total = 2LL * H * n_pages * P * chunks;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  append_heads_kernel<<<static_cast<int>(blocks), threads, 0, s>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_pool),
      static_cast<uint4*>(v_pool), entries_layer, tok_id_layer, pool_pages, start, n_pages, T, H, P, chunks,
      static_cast<long long>(frame) * T);
  return cudaGetLastError();
}

cudaError_t launch_diversity_prune(cudaStream_t s, Entry* entries_layer, const void* k_pool, const void* v_pool,
                                   void* k_pool_w, void* v_pool_w, int64_t* tok_id_layer, int pool_pages,
                                   int first_cand_entry, int n_cand_entries, int new_entry, int keep, int H, int D,
                                   int P, double* sums_layer, int* err) {
  if (D != kDivD || n_cand_entries > 1024) return cudaErrorInvalidValue;
  const int n_max = n_cand_entries * P;
  const size_t smem = diversity_prune_smem(n_max);
  // dynamic plus static shared memory above 48 KB needs the opt-in limit raised
  static size_t attr = 0;
  if (smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(diversity_prune_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  diversity_prune_kernel<<<H, kDivThreads, smem, s>>>(
      entries_layer, static_cast<const __nv_bfloat16*>(k_pool), static_cast<const __nv_bfloat16*>(v_pool),
      static_cast<__nv_bfloat16*>(k_pool_w), static_cast<__nv_bfloat16*>(v_pool_w), tok_id_layer, pool_pages,
      first_cand_entry, n_cand_entries, new_entry, keep, P, sums_layer, err);
  return cudaGetLastError();
}

}  // namespace kvc
