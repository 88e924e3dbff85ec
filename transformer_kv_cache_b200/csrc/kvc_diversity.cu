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
// Scores follow the definition in fp64, each step one IEEE operation (explicitly rounded
// intrinsics, no contraction), in the order a parallel evaluation takes: every sum over the
// 64 dims (the squares of |k|, the dot k_hat . mu, the squares of |mu|) in 8 blocks of 8
// consecutive dims, then the block sums; k_hat = k * RN(1 / |k|) (0 for a zero key);
// mu = the sum of k_hat over the candidates (the direction of the mean) and a head's score
// total in blocks of 32 consecutive candidates in ascending token id, then the block sums;
// score = -(k_hat . mu) / |mu|. Any other correct fp64 order differs from this one only
// within the rounding bound of these sums, so kept sets agree with an fp64 reference except
// among candidates whose scores tie within that bound.
#include <cuda_bf16.h>

#include <climits>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {
namespace {

constexpr int kDivD = 64;

// One frame into the per-head pages of a batch of layers: eight lanes per (layer, slot,
// head) row of 64 dims, one 16-byte chunk each, heads next (so a warp loads four heads of a
// slot, 512 contiguous bytes, and writes four whole 128-byte rows). A slot past T gets zeros
// and token id -1. The page-table entries [start, start + n_pages) of every head were just
// written by the allocator.
__global__ void __launch_bounds__(256) append_heads_kernel(AppendBatch in, int first_layer, LayerStarts starts,
                                                           int n_layers, uint4* k_pool, uint4* v_pool,
                                                           const Entry* __restrict__ entries_all,
                                                           int64_t* tok_id_all, int pool_pages, int n_pages, int T,
                                                           int H, int P, long long frame_base) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int kChunks = kDivD / 8;              // 16-byte chunks per row
  const int slots = n_pages * P;
  const long long total = static_cast<long long>(n_layers) * slots * H * kChunks;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int q = static_cast<int>(idx % kChunks);
    const long long r = idx / kChunks;
    const int h = static_cast<int>(r % H);
    const long long rt = r / H;
    const int t = static_cast<int>(rt % slots);
    const int b = static_cast<int>(rt / slots);
    const long long sub = (static_cast<long long>(first_layer + b) * H + h) * pool_pages;
    const int phys = __ldg(&entries_all[sub + starts.start[b] + t / P].x);
    const long long dst = ((sub + phys) * P + t % P) * kChunks + q;
    uint4 kc = make_uint4(0, 0, 0, 0), vc = make_uint4(0, 0, 0, 0);
    if (t < T) {
      const long long src = (static_cast<long long>(t) * H + h) * kChunks + q;
      kc = __ldg(static_cast<const uint4*>(in.k[b]) + src);
      vc = __ldg(static_cast<const uint4*>(in.v[b]) + src);
    }
    k_pool[dst] = kc;
    v_pool[dst] = vc;
    if (q == 0) tok_id_all[(sub + phys) * P + t % P] = t < T ? frame_base + t : -1;
  }
}

// ------------------------------------------------------------------ pruning
// One cluster of kPruneCluster CTAs per head. The head's candidates are the valid slots
// of its page-list entries [first, first + n_entries) (the kept pages, then the new
// frame's pages), in ascending token id; CTA r of the cluster owns candidates
// [r * B, r * B + B) (B a multiple of the 32-candidate block, so every block of a sum
// over candidates lies in one CTA) and stages their K and V rows in shared memory first.
// Each CTA publishes its blocks' partial sums of the normalised keys, then its scores, in
// its own shared memory; after a cluster barrier the others read them (distributed shared
// memory), and every CTA selects the Top-K itself. The kept candidates are written in
// place, in ascending id, over the slots of the first ceil(kept / P) candidate entries
// (every CTA's reads of the pool precede the first barrier); the pages of the remaining
// candidate entries go back to the head's free bitmap.
constexpr int kPruneCluster = 8;
constexpr int kPruneThreads = 512;
constexpr int kCandBlock = 32;          // candidates per block of every sum over candidates
constexpr int kDimBlock = 8;            // dims per block of every sum over the dims
constexpr int kPruneMaxB = 256;         // candidates per CTA (2,048 per head)
constexpr int kKRowStride = kDivD + 8;  // bf16 per staged key row: 144 bytes spread the banks
constexpr int kBins = 2048;             // selection histogram over [-1, 1]

struct PruneLayout {
  uint32_t sc_all, bsum_own, bsum_all, ssum_own, ssum_all, krow, vrow, rcp, score, id, slot, pos, page, hist, sbin,
      bucket, kflag, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

__host__ __device__ inline PruneLayout prune_layout(int n_max, int B, int n_entries) {
  PruneLayout l;
  const size_t nblk = static_cast<size_t>((n_max + kCandBlock - 1) / kCandBlock);
  const size_t b = static_cast<size_t>(B), bb = b / kCandBlock, n = static_cast<size_t>(n_max);
  size_t o = 0;
  auto take = [&o](size_t bytes) {
    const uint32_t r = static_cast<uint32_t>(o);
    o += align16(bytes);
    return r;
  };
  l.sc_all = take((n + 1) * 8);           // one spare: pairs are read 16 bytes at a time
  l.bsum_own = take(bb * kDivD * 8);
  // the block sums of all CTAs are dead once mu is known: the selection reuses their space
  const size_t sel_bytes = align16(kBins * 4) + align16(n * 2) + align16(n * 4) + align16(n);
  const size_t bsum_bytes = nblk * kDivD * 8;
  l.bsum_all = take(bsum_bytes > sel_bytes ? bsum_bytes : sel_bytes);
  l.hist = l.bsum_all;
  l.sbin = l.hist + static_cast<uint32_t>(align16(kBins * 4));
  l.bucket = l.sbin + static_cast<uint32_t>(align16(n * 2));
  l.kflag = l.bucket + static_cast<uint32_t>(align16(n * 4));
  l.ssum_own = take(bb * 8);
  l.ssum_all = take(nblk * 8);
  l.krow = take(b * kKRowStride * 2);
  l.vrow = take(b * kDivD * 2);
  l.rcp = take(b * 8);
  l.score = take(b * 8);
  l.id = take(b * 8);
  l.slot = take(b * 4);
  l.pos = take(b * 4);
  l.page = take(static_cast<size_t>(n_entries) * 4);
  l.total = static_cast<uint32_t>(o);
  return l;
}

__device__ __forceinline__ double bf16_lo(uint32_t w) { return static_cast<double>(__uint_as_float(w << 16)); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return static_cast<double>(__uint_as_float(w & 0xffff0000u)); }

// One 8-dim block of a sum over the dims, from 8 bf16 values (ascending):
// part = sum of x * x, or of (x * r) * m[d]
__device__ __forceinline__ double block_sq(const uint4 u) {
  const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
  double part = 0.0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const double a = bf16_lo(wv[j]), b = bf16_hi(wv[j]);
    part = __dadd_rn(part, __dmul_rn(a, a));
    part = __dadd_rn(part, __dmul_rn(b, b));
  }
  return part;
}
// m is read from shared memory at every use (volatile): the mean's 64 components kept in
// registers across the candidate loop would not fit beside the rest of the kernel.
__device__ __forceinline__ double block_dot(const uint4 u, double r, const volatile double* m) {
  const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
  double part = 0.0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    part = __dadd_rn(part, __dmul_rn(__dmul_rn(bf16_lo(wv[j]), r), m[2 * j]));
    part = __dadd_rn(part, __dmul_rn(__dmul_rn(bf16_hi(wv[j]), r), m[2 * j + 1]));
  }
  return part;
}

// Monotone histogram bin of a score in [-1, 1] (clamped): a higher bin means a higher score.
__device__ __forceinline__ int score_bin(double s) {
  const double t = (s + 1.0) * (kBins / 2);
  return t >= kBins - 1 ? kBins - 1 : (t > 0.0 ? static_cast<int>(t) : 0);
}

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Exclusive prefix sum of one value per thread over the CTA; every thread calls it.
__device__ int cta_scan_excl(int x, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int v = warp_incl_scan(x);
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_incl_scan(lane < nw ? s_warp[lane] : 0);
    s_warp[lane] = w;
  }
  __syncthreads();
  const int r = v - x + (warp > 0 ? s_warp[warp - 1] : 0);
  *total = s_warp[nw - 1];
  __syncthreads();
  return r;
}

// Layers of one launch: blockIdx.y selects the layer, whose bases are the launch's plus
// blockIdx.y strides, and whose candidate entries, budget and per-CTA candidate count
// (B) are its row of the table.
__global__ void __cluster_dims__(kPruneCluster, 1, 1) __launch_bounds__(kPruneThreads, 2) diversity_prune_kernel(
    Entry* entries_base, __nv_bfloat16* k_base, __nv_bfloat16* v_base, uint32_t* bitmap_base, int words,
    int64_t* tok_base, int pool_pages, int P, double* sums_base, int* err, const __grid_constant__ PruneBatch pb) {
  griddep_wait();
  griddep_launch_dependents();
  const long long y = blockIdx.y;
  Entry* entries_layer = entries_base + y * pb.entries_stride;
  __nv_bfloat16* k_pool = k_base + y * pb.pool_stride;
  __nv_bfloat16* v_pool = v_base + y * pb.pool_stride;
  uint32_t* bitmap_layer = bitmap_base + y * pb.bitmap_stride;
  int64_t* tok_id_layer = tok_base + y * pb.tok_stride;
  double* sums_layer = sums_base + y * pb.sums_stride;
  const int first = pb.l[y].first, n_entries = pb.l[y].n_entries, keep = pb.l[y].keep, B = pb.l[y].B;
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ int s_warp[32];
  __shared__ double s_mu[kDivD];
  __shared__ double s_mnorm;
  __shared__ int s_sel, s_above, s_cnt, s_bcnt;
  const int rank = static_cast<int>(cluster_ctarank());
  const int h = blockIdx.x / kPruneCluster;
  const int tid = threadIdx.x;
  const long long sub = static_cast<long long>(h) * pool_pages;
  Entry* E = entries_layer + sub;
  const PruneLayout lay = prune_layout(n_entries * P, B, n_entries);
  double* sc_all = reinterpret_cast<double*>(sm + lay.sc_all);          // [N] every candidate's score
  double* bsum_own = reinterpret_cast<double*>(sm + lay.bsum_own);      // [B/32][D] published
  double* bsum_all = reinterpret_cast<double*>(sm + lay.bsum_all);      // [blocks][D]
  double* ssum_own = reinterpret_cast<double*>(sm + lay.ssum_own);      // [B/32] published
  double* ssum_all = reinterpret_cast<double*>(sm + lay.ssum_all);      // [blocks] (CTA 0)
  __nv_bfloat16* krow = reinterpret_cast<__nv_bfloat16*>(sm + lay.krow);  // [B][kKRowStride]
  uint4* vrow = reinterpret_cast<uint4*>(sm + lay.vrow);                // [B][8]
  double* rcp = reinterpret_cast<double*>(sm + lay.rcp);                // [B] RN(1 / |k|), 0 for |k| = 0
  double* score = reinterpret_cast<double*>(sm + lay.score);            // [B] published
  int64_t* ids = reinterpret_cast<int64_t*>(sm + lay.id);               // [B] token ids
  int* slot = reinterpret_cast<int*>(sm + lay.slot);                    // [B] pool slot within the head
  int* pos = reinterpret_cast<int*>(sm + lay.pos);                      // [B] kept position, or -1
  int* page = reinterpret_cast<int*>(sm + lay.page);                    // [n_entries] physical pages
  int* s_hist = reinterpret_cast<int*>(sm + lay.hist);                  // [kBins] (after mu)
  uint16_t* sbin = reinterpret_cast<uint16_t*>(sm + lay.sbin);          // [N] histogram bin
  int* bucket = reinterpret_cast<int*>(sm + lay.bucket);                // [N] the threshold bin's members
  uint8_t* kflag = sm + lay.kflag;                                      // [N] kept
  const int bpc = B / kCandBlock;                                       // blocks per CTA

  // candidate offsets of the entries (one entry per thread) and the own candidates' slots
  int w = 0, x = 0;
  if (tid < n_entries) {
    const Entry en = E[first + tid];
    w = en.w;
    x = en.x;
    page[tid] = x;
  }
  int N;
  const int o = cta_scan_excl(w, s_warp, &N);
  const int c0 = rank * B;
  const int nl = max(0, min(N, c0 + B) - c0);
  for (int s = 0; s < w; ++s) {
    const int i = o + s - c0;
    if (i >= 0 && i < nl) slot[i] = x * P + s;
  }
  if (rank == 0 && tid == 0 && N < keep) latch_error(err, DERR_BOUNDS);
  __syncthreads();
  // own K and V rows and token ids into shared memory: every read of the pool happens here
  for (int it = tid; it < nl * 16; it += blockDim.x) {
    const int li = it >> 4, q = it & 15;
    const long long src = sub * P + slot[li];
    if (q < 8) cp_async16(krow + li * kKRowStride + q * 8, k_pool + src * kDivD + q * 8);
    else cp_async16(vrow + li * 8 + q - 8, v_pool + src * kDivD + (q - 8) * 8);
    if (q == 0) cp_async8(ids + li, tok_id_layer + src);
  }
  cp_async_wait_all();
  __syncthreads();
  // |k| (a sum over the dims in 8-dim blocks) and its reciprocal
#pragma unroll 1
  for (int li = tid; li < nl; li += blockDim.x) {
    const uint4* kr = reinterpret_cast<const uint4*>(krow + li * kKRowStride);
    double acc = 0.0;
#pragma unroll
    for (int hq = 0; hq < kDivD / kDimBlock; hq += 4) {   // four blocks in flight, added in order
      double part[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) part[q] = block_sq(kr[hq + q]);
#pragma unroll
      for (int q = 0; q < 4; ++q) acc = __dadd_rn(acc, part[q]);
    }
    const double n = __dsqrt_rn(acc);
    rcp[li] = n > 0.0 ? __ddiv_rn(1.0, n) : 0.0;
  }
  __syncthreads();
  // own blocks' sums of k_hat = k * rcp, ascending within the block
  const int nb_own = (nl + kCandBlock - 1) / kCandBlock;
  for (int it = tid; it < nb_own * kDivD; it += blockDim.x) {
    const int j = it / kDivD, d = it % kDivD;
    const int i0 = j * kCandBlock, n = min(nl - i0, kCandBlock);
    const __nv_bfloat16* kc = krow + i0 * kKRowStride + d;
    double sum = 0.0;
#pragma unroll 8
    for (int t = 0; t < kCandBlock; ++t)
      if (t < n)
        sum = __dadd_rn(sum, __dmul_rn(static_cast<double>(__bfloat162float(kc[t * kKRowStride])), rcp[i0 + t]));
    bsum_own[j * kDivD + d] = sum;
  }
  __syncwarp();
  cluster_arrive_release();
  cluster_wait_acquire();
  // every block's partial sums, read from the CTA that owns it (all loads in flight first)
  const int nblk = (N + kCandBlock - 1) / kCandBlock;
  {
    constexpr int kMaxIt = kPruneCluster * kPruneMaxB / kCandBlock * (kDivD / 2) / kPruneThreads;
    uint64_t u[kMaxIt][2];
#pragma unroll
    for (int k = 0; k < kMaxIt; ++k) {
      const int it = tid + k * kPruneThreads;
      if (it < nblk * (kDivD / 2)) {
        const int b = it / (kDivD / 2), d2 = it % (kDivD / 2);
        ld_cluster_v2u64(cluster_map(smem_u32(bsum_own + (b % bpc) * kDivD + 2 * d2), b / bpc), u[k][0], u[k][1]);
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxIt; ++k) {
      const int it = tid + k * kPruneThreads;
      if (it < nblk * (kDivD / 2)) {
        bsum_all[2 * it] = __longlong_as_double(static_cast<long long>(u[k][0]));
        bsum_all[2 * it + 1] = __longlong_as_double(static_cast<long long>(u[k][1]));
      }
    }
  }
  __syncthreads();
  // mu: the block sums in ascending block order; |mu|^2 a sum over the dims in 8-dim blocks
  if (tid < kDivD) {
    double m = 0.0;
    for (int b = 0; b < nblk; ++b) m = __dadd_rn(m, bsum_all[b * kDivD + tid]);
    s_mu[tid] = m;
  }
  __syncthreads();
  if (tid < kDivD / kDimBlock) {
    double part = 0.0;
#pragma unroll
    for (int d = 0; d < kDimBlock; ++d) {
      const double m = s_mu[tid * kDimBlock + d];
      part = __dadd_rn(part, __dmul_rn(m, m));
    }
    double acc = __shfl_sync(0xffu, part, 0, 8);
    acc = __dadd_rn(0.0, acc);
#pragma unroll
    for (int q = 1; q < kDivD / kDimBlock; ++q) acc = __dadd_rn(acc, __shfl_sync(0xffu, part, q, 8));
    if (tid == 0) s_mnorm = __dsqrt_rn(acc);
  }
  __syncthreads();
  const double mnorm = s_mnorm;
  // scores -(k_hat . mu) / |mu| (the dot a sum over the dims in 8-dim blocks)
#pragma unroll 1
  for (int li = tid; li < nl; li += blockDim.x) {
    double sc = 0.0;
    if (mnorm > 0.0) {
      const uint4* kr = reinterpret_cast<const uint4*>(krow + li * kKRowStride);
      const double r = rcp[li];
      double dot = 0.0;
#pragma unroll
      for (int hq = 0; hq < kDivD / kDimBlock; hq += 4) {
        double part[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) part[q] = block_dot(kr[hq + q], r, s_mu + (hq + q) * kDimBlock);
#pragma unroll
        for (int q = 0; q < 4; ++q) dot = __dadd_rn(dot, part[q]);
      }
      sc = -__ddiv_rn(dot, mnorm);
    }
    score[li] = sc;
  }
  __syncthreads();
  for (int j = tid; j < nb_own; j += blockDim.x) {
    const int i1 = min(nl, (j + 1) * kCandBlock);
    double sum = 0.0;
    for (int li = j * kCandBlock; li < i1; ++li) sum = __dadd_rn(sum, score[li]);
    ssum_own[j] = sum;
  }
  __syncwarp();
  cluster_arrive_release();
  cluster_wait_acquire();
  // every candidate's score (pairs of 16 bytes; B is even, so a pair never spans two CTAs);
  // CTA 0 also the score block sums
  {
    constexpr int kMaxIt = kPruneCluster * kPruneMaxB / 2 / kPruneThreads;
    uint64_t u[kMaxIt][2];
    const int npair = (N + 1) / 2;
#pragma unroll
    for (int k = 0; k < kMaxIt; ++k) {
      const int it = tid + k * kPruneThreads;
      if (it < npair) {
        const int i = 2 * it;
        ld_cluster_v2u64(cluster_map(smem_u32(score + i % B), i / B), u[k][0], u[k][1]);
      }
    }
    double sb = 0.0;
    if (rank == 0 && tid < nblk)
      sb = __longlong_as_double(
          static_cast<long long>(ld_cluster_u64(cluster_map(smem_u32(ssum_own + tid % bpc), tid / bpc))));
#pragma unroll
    for (int k = 0; k < kMaxIt; ++k) {
      const int it = tid + k * kPruneThreads;
      if (it < npair) {
        sc_all[2 * it] = __longlong_as_double(static_cast<long long>(u[k][0]));
        sc_all[2 * it + 1] = __longlong_as_double(static_cast<long long>(u[k][1]));
      }
    }
    if (rank == 0 && tid < nblk) ssum_all[tid] = sb;
  }
  __syncthreads();
  __syncwarp();
  cluster_arrive_release();   // this CTA reads no other CTA's shared memory any more

  // Top-K by (score descending, id ascending): a histogram of monotone score bins finds the
  // bin that holds the kk-th best; candidates in higher bins are kept, and the members of
  // that bin are ranked exactly among themselves (ties to the lower id).
  const int kk = keep < N ? keep : N;
  if (kk >= N) {
    for (int i = tid; i < N; i += blockDim.x) kflag[i] = 1;
  } else {
    for (int b = tid; b < kBins; b += blockDim.x) s_hist[b] = 0;
    if (tid == 0) s_bcnt = 0;
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x) {
      const int b = score_bin(sc_all[i]);
      sbin[i] = static_cast<uint16_t>(b);
      atomicAdd(&s_hist[b], 1);
    }
    __syncthreads();
    // thread t holds bins 2047 - 4t down to 2044 - 4t
    constexpr int kPer = kBins / kPruneThreads;
    int c[kPer], lsum = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      c[k] = s_hist[kBins - 1 - kPer * tid - k];
      lsum += c[k];
    }
    int tot;
    int acc = cta_scan_excl(lsum, s_warp, &tot);
    if (acc < kk && kk <= acc + lsum) {
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        if (acc < kk && kk <= acc + c[k]) {
          s_sel = kBins - 1 - kPer * tid - k;
          s_above = acc;
          s_cnt = c[k];
        }
        acc += c[k];
      }
    }
    __syncthreads();
    const int sel = s_sel, rem = kk - s_above, cnt = s_cnt;
    for (int i = tid; i < N; i += blockDim.x) {
      const int b = sbin[i];
      kflag[i] = b > sel;
      if (b == sel) bucket[atomicAdd(&s_bcnt, 1)] = i;
    }
    __syncthreads();
    if (tid == 0 && s_bcnt != cnt) latch_error(err, DERR_BOUNDS);
    for (int m = tid; m < cnt; m += blockDim.x) {
      const int a = bucket[m];
      const double sa = sc_all[a];
      int r = 0;
      for (int m2 = 0; m2 < cnt; ++m2) {
        const int b = bucket[m2];
        const double sbv = sc_all[b];
        r += (sbv > sa) || (sbv == sa && b < a);
      }
      kflag[a] = r < rem;
    }
    __syncthreads();
  }
  // positions: kept candidates numbered in ascending id (contiguous chunks per thread)
  {
    const int ch = (N + blockDim.x - 1) / blockDim.x;
    const int i0 = min(N, tid * ch), i1 = min(N, i0 + ch);
    int n_kept = 0;
    for (int i = i0; i < i1; ++i) n_kept += kflag[i];
    int tot;
    int p = cta_scan_excl(n_kept, s_warp, &tot);
    if (tid == 0 && tot != kk) latch_error(err, DERR_BOUNDS);
    for (int i = i0; i < i1; ++i) {
      const bool kept = kflag[i];
      if (i >= c0 && i < c0 + nl) pos[i - c0] = kept ? p : -1;
      p += kept;
    }
  }
  __syncthreads();
  // kept position p goes to slot p % P of candidate entry first + p / P
  uint4* kd = reinterpret_cast<uint4*>(k_pool);
  uint4* vd = reinterpret_cast<uint4*>(v_pool);
  for (int it = tid; it < nl * 16; it += blockDim.x) {
    const int li = it >> 4, q = it & 15;
    const int p = pos[li];
    if (p < 0) continue;
    if (p >= kk) {
      latch_error(err, DERR_BOUNDS);
      continue;
    }
    const long long dst = (sub + page[p / P]) * P + p % P;
    if (q < 8) kd[dst * 8 + q] = reinterpret_cast<const uint4*>(krow + li * kKRowStride)[q];
    else vd[dst * 8 + q - 8] = vrow[li * 8 + q - 8];
    if (q == 0) tok_id_layer[dst] = ids[li];
  }
  const int n_new = (kk + P - 1) / P;
  if (rank == kPruneCluster - 1) {
    // the last kept page's slots past the kept count: zero K and V, no token
    for (int it = tid; it < (n_new * P - kk) * 16; it += blockDim.x) {
      const int t = kk + (it >> 4), q = it & 15;
      const long long dst = (sub + page[t / P]) * P + t % P;
      if (q < 8) kd[dst * 8 + q] = make_uint4(0, 0, 0, 0);
      else vd[dst * 8 + q - 8] = make_uint4(0, 0, 0, 0);
      if (q == 0) tok_id_layer[dst] = -1;
    }
  }
  if (rank == 0) {
    // the kept pages' entries (owner -1: compaction), the other candidate pages freed
    uint32_t* bitmap = bitmap_layer + static_cast<long long>(h) * words;
    for (int e = tid; e < n_entries; e += blockDim.x) {
      int* en = reinterpret_cast<int*>(E + first + e);
      if (e < n_new) {
        en[1] = -1;
        en[2] = e;
        en[3] = min(P, kk - e * P);
      } else {
        const uint32_t bit = 1u << (page[e] & 31);
        const uint32_t old = atomicAnd(&bitmap[page[e] >> 5], ~bit);
        if (!(old & bit)) latch_error(err, DERR_BOUNDS);
      }
    }
    if (tid == 0) {
      double t = 0.0;
      for (int b = 0; b < nblk; ++b) t = __dadd_rn(t, ssum_all[b]);
      sums_layer[h] = t;
    }
  }
  __syncwarp();
  cluster_wait_acquire();     // no CTA leaves while another may still read its shared memory
}

}  // namespace

cudaError_t launch_append_heads(cudaStream_t s, const AppendBatch& in, int first_layer, const LayerStarts& starts,
                                int n_layers, void* k_pool, void* v_pool, const Entry* entries_all,
                                int64_t* tok_id_all, int pool_pages, int n_pages, int T, int H, int D, int P,
                                int frame) {
  if (D != kDivD) return cudaErrorInvalidValue;
  const long long total = static_cast<long long>(n_layers) * n_pages * P * H * (kDivD / 8);
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  return launch_pdl(append_heads_kernel, dim3(static_cast<int>(blocks)), dim3(threads), 0, s,
                    in, first_layer, starts, n_layers, static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool),
                    entries_all, tok_id_all, pool_pages, n_pages, T, H, P, static_cast<long long>(frame) * T);
}

int diversity_prune_max_candidates() { return kPruneCluster * kPruneMaxB; }

cudaError_t launch_diversity_prune_layers(cudaStream_t s, Entry* entries_base, void* k_base, void* v_base,
                                          uint32_t* bitmap_base, int words, int64_t* tok_base, int pool_pages,
                                          const PruneLayerArgs* layers, int n, int H, int D, int P,
                                          double* sums_base, int* err) {
  if (D != kDivD || n < 1 || n > kMaxPruneLayers) return cudaErrorInvalidValue;
  PruneBatch pb{};
  pb.entries_stride = static_cast<long long>(H) * pool_pages;
  pb.pool_stride = static_cast<long long>(H) * pool_pages * P * kDivD;
  pb.tok_stride = static_cast<long long>(H) * pool_pages * P;
  pb.bitmap_stride = static_cast<long long>(H) * words;
  pb.sums_stride = H;
  size_t smem = 0;
  for (int l = 0; l < n; ++l) {
    const int n_max = layers[l].n_cand_entries * P;
    if (layers[l].n_cand_entries < 1 || layers[l].n_cand_entries > kPruneThreads || layers[l].keep < 1 ||
        n_max > kPruneCluster * kPruneMaxB)
      return cudaErrorInvalidValue;
    int B = (n_max + kPruneCluster - 1) / kPruneCluster;
    B = (B + kCandBlock - 1) / kCandBlock * kCandBlock;
    pb.l[l].first = layers[l].first_cand_entry;
    pb.l[l].n_entries = layers[l].n_cand_entries;
    pb.l[l].keep = layers[l].keep;
    pb.l[l].B = B;
    smem = std::max(smem, static_cast<size_t>(prune_layout(n_max, B, layers[l].n_cand_entries).total));
  }
  // opt in once per device for the largest layout any call can need
  static PerDeviceOnce attr;
  cudaError_t e = attr.run([] {
    const size_t most = prune_layout(kPruneCluster * kPruneMaxB, kPruneMaxB, kPruneThreads).total;
    return cudaFuncSetAttribute(diversity_prune_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(most));
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(diversity_prune_kernel, dim3(H * kPruneCluster, n), dim3(kPruneThreads), smem, s, entries_base,
                    static_cast<__nv_bfloat16*>(k_base), static_cast<__nv_bfloat16*>(v_base), bitmap_base, words,
                    tok_base, pool_pages, P, sums_base, err, pb);
}

// Layer-wise adaptive budgets ("InfiniteVGGT" explainer, Layer-wise adaptive budgets): from
// each layer's mean diversity of its last pruning (the heads' fp64 score sums in head order
// over H x candidates), p = softmax(mean / tau) over the layers in fp64 and
// budget_l = floor(L * k * p_l), clamped to [1, cap] (a layer keeps at least one token and
// at most what its pool holds); tau <= 0 gives every layer k. One warp.
__global__ void layer_budget_kernel(const double* __restrict__ sums, const long long* __restrict__ cand, int L,
                                    int H, double tau, int k, int cap, int32_t* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x;
  auto mean_of = [&](int l) {
    double tot = 0.0;
    for (int h = 0; h < H; ++h) tot = __dadd_rn(tot, sums[static_cast<long long>(l) * H + h]);
    return __ddiv_rn(tot, static_cast<double>(static_cast<long long>(H) * cand[l]));
  };
  if (tau <= 0.0) {
    for (int l = lane; l < L; l += 32) out[l] = min(max(k, 1), cap);
    return;
  }
  double zmax = -INFINITY;
  for (int l = lane; l < L; l += 32) zmax = fmax(zmax, __ddiv_rn(mean_of(l), tau));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zmax = fmax(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
  // the denominator: the layers' exponentials summed in layer order by lane 0
  double den = 0.0;
  if (lane == 0)
    for (int l = 0; l < L; ++l) den = __dadd_rn(den, exp(__ddiv_rn(mean_of(l), tau) - zmax));
  den = __shfl_sync(0xffffffffu, den, 0);
  for (int l = lane; l < L; l += 32) {
    const double p = __ddiv_rn(exp(__ddiv_rn(mean_of(l), tau) - zmax), den);
    const double b = floor(__dmul_rn(static_cast<double>(L) * static_cast<double>(k), p));
    out[l] = static_cast<int32_t>(fmin(fmax(b, 1.0), static_cast<double>(cap)));
  }
}

cudaError_t launch_layer_budgets(cudaStream_t s, const double* sums, const long long* cand, int L, int H, double tau,
                                 int k, int cap, int32_t* out) {
  return launch_pdl(layer_budget_kernel, dim3(1), dim3(32), 0, s, sums, cand, L, H, tau, k, cap, out);
}

}  // namespace kvc
