// kvc_compress.cu -- importance scoring and keep / merge / drop compression (budget mode).
//
// Scoring follows the StreamCacheVGGT page, sections 2.1.1-2.1.4: the raw score of a token
// is the L2 norm of its FFN residual; at every layer the frame's tokens are ranked by it
// (0 = largest); over a window of the last W layers of the same frame the normalised ranks
// R/(N-1) have a population standard deviation sigma, compared with the uniform-null
// spread 1/sqrt(12): Cons = max(0, 1 - sigma*sqrt(12)); s_hat = s * (1 + lambda * Cons).
// The rank history is kept per frame and reset when a new frame starts.
//
// Compression follows section 2 of that page (keep the core, merge the middle into the
// core, drop the rest); sizes, the merge rule and the protected set follow the budgeted
// workload's statement: keep floor(keep_frac * B) tokens (protected ones first), merge the
// next B - floor(keep_frac * B) into the kept non-protected token of highest full-key
// cosine as count-weighted means, drop the remainder, then rewrite the kept tokens in
// ascending id into fresh pages.
//
// Every step whose result is an integer (ranks, tiers, targets) or a stored value is
// computed in fp64 with the operation order written next to it, so the results match an
// fp64 reference bit for bit; the fp64 helpers below use explicitly rounded intrinsics so
// the compiler cannot contract them into fused multiply-adds.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {

namespace {

constexpr int kCosTile = 128;    // targets per tile of the merge-target screen

struct Scratch {
  int64_t* ids;
  float* shat;
  int32_t* slot;
  int32_t* cnt;
  uint8_t* prot;
  int32_t* page_off;   // first position of each page-table entry's tokens
  int32_t* keep;
  int32_t* elig;
  int32_t* merge;
  int32_t* counts;     // [0] N, [1] keep, [2] elig, [3] merge; [8..11] tier thresholds
  int32_t* target;     // index into elig, per merge source
  int32_t* order;      // merge sources sorted by (target, source)
  int32_t* bucket;     // [n_keep + 1]: sources of target e are order[bucket[e] .. bucket[e+1])
  int64_t* src_base;   // per entry of `order`: pool element offset of the source's (page, slot)
  int32_t* src_cnt;    // per entry of `order`: the source's count
  int32_t* cursor;     // [n_keep]
  __nv_bfloat16* ks;   // full keys of the merge sources [n_merge][H*D]
  __nv_bfloat16* ke;   // full keys of the eligible targets [n_keep][H*D]
  double* ns;          // fp64 key norms
  double* ne;
  float* inv_ns;       // fp32 inverse norms for the screen
  float* inv_ne;
  float* top_v;        // four best screened cosines per (source, target tile)
  int32_t* top_j;
  float* s_raw;        // raw scores of the frame being scored [T]
  float* s_raw_all;    // raw scores of every layer of the frame [layers][T] (kvc_compress_all)
  int64_t* last_src;   // [layers][merge cap]
  int64_t* last_dst;
};

struct Caps {
  size_t n_max, n_keep, n_merge, hd, tiles;
};

Caps caps_of(const kvc_config& g) {
  Caps c;
  const size_t B = g.budget_tokens;
  c.n_max = B + g.tokens_per_frame;
  c.n_keep = static_cast<size_t>(std::floor(static_cast<double>(g.keep_frac) * static_cast<double>(B)));
  if (c.n_keep < 1) c.n_keep = 1;
  c.n_merge = B > c.n_keep ? B - c.n_keep : 1;
  c.hd = static_cast<size_t>(g.num_heads) * g.head_dim;
  c.tiles = (c.n_keep + kCosTile - 1) / kCosTile;
  return c;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Lays out the scratch regions; with base == nullptr only the total size is computed.
size_t carve(const kvc_config& g, uint8_t* base, Scratch* s) {
  const Caps c = caps_of(g);
  size_t off = 0;
  auto take = [&](size_t bytes) -> uint8_t* {
    uint8_t* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  Scratch t;
  t.ids = reinterpret_cast<int64_t*>(take(c.n_max * 8));
  t.shat = reinterpret_cast<float*>(take(c.n_max * 4));
  t.slot = reinterpret_cast<int32_t*>(take(c.n_max * 4));
  t.cnt = reinterpret_cast<int32_t*>(take(c.n_max * 4));
  t.prot = take(c.n_max);
  t.page_off = reinterpret_cast<int32_t*>(take(c.n_max * 4));
  t.keep = reinterpret_cast<int32_t*>(take(c.n_max * 4));
  t.elig = reinterpret_cast<int32_t*>(take(c.n_max * 4));
  t.merge = reinterpret_cast<int32_t*>(take(c.n_max * 4));
  t.counts = reinterpret_cast<int32_t*>(take(16 * 4));
  t.target = reinterpret_cast<int32_t*>(take(c.n_merge * 4));
  t.order = reinterpret_cast<int32_t*>(take(c.n_merge * 4));
  t.bucket = reinterpret_cast<int32_t*>(take((c.n_keep + 1) * 4));
  t.src_base = reinterpret_cast<int64_t*>(take(c.n_merge * 8));
  t.src_cnt = reinterpret_cast<int32_t*>(take(c.n_merge * 4));
  t.cursor = reinterpret_cast<int32_t*>(take(c.n_keep * 4));
  t.ks = reinterpret_cast<__nv_bfloat16*>(take(c.n_merge * c.hd * 2));
  t.ke = reinterpret_cast<__nv_bfloat16*>(take(c.n_keep * c.hd * 2));
  t.ns = reinterpret_cast<double*>(take(c.n_merge * 8));
  t.ne = reinterpret_cast<double*>(take(c.n_keep * 8));
  t.inv_ns = reinterpret_cast<float*>(take(c.n_merge * 4));
  t.inv_ne = reinterpret_cast<float*>(take(c.n_keep * 4));
  t.top_v = reinterpret_cast<float*>(take(c.n_merge * c.tiles * 16));
  t.top_j = reinterpret_cast<int32_t*>(take(c.n_merge * c.tiles * 16));
  t.s_raw = reinterpret_cast<float*>(take(static_cast<size_t>(g.tokens_per_frame) * 4));
  t.s_raw_all = reinterpret_cast<float*>(take(static_cast<size_t>(g.num_layers) * g.tokens_per_frame * 4));
  t.last_src = reinterpret_cast<int64_t*>(take(static_cast<size_t>(g.num_layers) * c.n_merge * 8));
  t.last_dst = reinterpret_cast<int64_t*>(take(static_cast<size_t>(g.num_layers) * c.n_merge * 8));
  if (s) *s = t;
  return off;
}

// fp64 -> bf16, round to nearest even, one rounding (written from the format's
// definition: 8 significant bits, subnormal quantum 2^-133, overflow to infinity).
__device__ __forceinline__ __nv_bfloat16 f64_to_bf16_rne(double x) {
  // bf16 normal range (biased fp64 exponent 897..1150): round the 52 fraction bits to 7,
  // to nearest even, on the bit pattern; a carry may raise the exponent (1151 = overflow)
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  const int ex = static_cast<int>((b >> 52) & 0x7FF);
  if (ex >= 897 && ex <= 1150) {
    const unsigned long long r = (b + 0x0FFFFFFFFFFFull + ((b >> 45) & 1ull)) & ~0x1FFFFFFFFFFFull;
    if (((r >> 52) & 0x7FF) > 1150) return __float2bfloat16_rn(x > 0 ? INFINITY : -INFINITY);
    return __float2bfloat16_rn(static_cast<float>(__longlong_as_double(static_cast<long long>(r))));   // exact
  }
  if (x == 0.0 || isnan(x) || isinf(x)) return __float2bfloat16_rn(static_cast<float>(x));
  int e = ilogb(x);                    // |x| in [2^e, 2^(e+1))
  int qe = e - 7;                      // quantum of 8 significant bits
  if (qe < -133) qe = -133;
  const double y = ldexp(rint(ldexp(x, -qe)), qe);   // exact scaling; rint = ties to even
  if (fabs(y) > 3.3895313892515355e38) return __float2bfloat16_rn(y > 0 ? INFINITY : -INFINITY);
  return __float2bfloat16_rn(static_cast<float>(y));  // y is a bf16 value: exact
}

// ------------------------------------------------------------------ scoring
// s_i = fp32(sqrt(sum_c r_ic^2)); the squares (exact in fp64) are summed per block of 32
// consecutive channels in ascending c, then the block sums in ascending block order. One
// warp per token: lane b sums block b (its 32 channels are 8 float4 loads), lane 0 adds
// the block sums in order; for more than 32 blocks the warp repeats per 32 blocks.
__device__ __forceinline__ void residual_norm_rows(const float* __restrict__ r, int T, int R, float* __restrict__ s_out) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const float* x = r + static_cast<long long>(row) * R;
  const int nb = (R + 31) / 32;
  double acc = 0.0;
  for (int b0 = 0; b0 < nb; b0 += 32) {
    const int b = b0 + lane;
    double blk = 0.0;
    if (b < nb) {
      const int c0 = b * 32, n = min(32, R - c0);
      if (n == 32 && (R & 3) == 0 && (reinterpret_cast<uintptr_t>(r) & 15) == 0) {
        float v[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 f = __ldg(reinterpret_cast<const float4*>(x + c0) + q);
          v[4 * q] = f.x;
          v[4 * q + 1] = f.y;
          v[4 * q + 2] = f.z;
          v[4 * q + 3] = f.w;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const double y = static_cast<double>(v[c]);
          blk = __dadd_rn(blk, __dmul_rn(y, y));
        }
      } else {
        for (int c = 0; c < n; ++c) {
          const double y = static_cast<double>(__ldg(x + c0 + c));
          blk = __dadd_rn(blk, __dmul_rn(y, y));
        }
      }
    }
    const int nin = min(32, nb - b0);
    for (int q = 0; q < nin; ++q) {
      const double pq = __shfl_sync(0xffffffffu, blk, q);
      acc = __dadd_rn(acc, pq);
    }
  }
  if (lane == 0) s_out[row] = __double2float_rn(__dsqrt_rn(acc));
}
__global__ void residual_norm_kernel(const float* __restrict__ r, int T, int R, float* __restrict__ s_out) {
  residual_norm_rows(r, T, R, s_out);
}
// Every layer of a frame in one launch, blockIdx.y the layer.
struct ResidualBatch {
  const float* r[kMaxBatchLayers];
};
__global__ void residual_norm_layers_kernel(const __grid_constant__ ResidualBatch rb, int T, int R,
                                            float* __restrict__ s_all) {
  residual_norm_rows(rb.r[blockIdx.y], T, R, s_all + static_cast<long long>(blockIdx.y) * T);
}

// Ranks of the frame's T tokens (s descending, ties to the lower slot), stored in the
// history slot of this layer; then, over the window layers in `mask`, the population
// variance of the normalised ranks gives Cons and s_hat, written next to the tokens.
// Eight lanes per token (every token's lanes read all T scores from shared memory, each
// counting every eighth, then a shuffle sum); a token's Cons needs only its own ranks, so
// the CTAs are independent. kClcesTokens tokens per 128-thread CTA.
constexpr int kClcesTokens = 16;
__global__ void __launch_bounds__(128) clces_kernel(const float* __restrict__ s, int T, int32_t* hist, int slot,
                                                     uint32_t mask, int n_win, float lam,
                                                     const Entry* __restrict__ frame_pages, int P,
                                                     float* __restrict__ tok_shat_layer) {
  extern __shared__ float s_sm[];
  for (int i = threadIdx.x; i < T; i += blockDim.x) s_sm[i] = s[i];
  __syncthreads();
  const int sub = threadIdx.x & 7;
  const int i = blockIdx.x * kClcesTokens + static_cast<int>(threadIdx.x >> 3);
  int r = 0;
  if (i < T) {
    const float si = s_sm[i];
    for (int j = sub; j < T; j += 8) {
      const float sj = s_sm[j];
      r += (sj > si) || (sj == si && j < i);
    }
  }
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 4);
  if (i >= T || sub != 0) return;
  hist[slot * T + i] = r;
  const double sqrt12 = __dsqrt_rn(12.0);
  const double lamd = static_cast<double>(lam);
  {
    long long sr = 0, sr2 = 0;
    for (int k = 0; k < 32; ++k) {
      if (mask & (1u << k)) {
        const long long v = hist[k * T + i];
        sr += v;
        sr2 += v * v;
      }
    }
    const long long Dv = static_cast<long long>(n_win) * sr2 - sr * sr;
    const double sigma = __ddiv_rn(__dsqrt_rn(static_cast<double>(Dv)),
                                   __dmul_rn(static_cast<double>(n_win), static_cast<double>(T - 1)));
    double cons = __dsub_rn(1.0, __dmul_rn(sigma, sqrt12));
    if (cons < 0.0) cons = 0.0;
    const double w = __dmul_rn(static_cast<double>(s_sm[i]), __dadd_rn(1.0, __dmul_rn(lamd, cons)));
    const int g = i / P;
    const int phys = frame_pages[g].x;
    tok_shat_layer[static_cast<long long>(phys) * P + (i % P)] = __double2float_rn(w);
  }
}

// CLCES of every layer of a frame in one launch (layers scored in order in one call): a
// CTA carries its kClcesTokens tokens through the layers in order, keeping their ranks of
// the last RW layers in shared memory, since a token's Cons needs only its own ranks. The
// arithmetic per (layer, token) is clces_kernel's (ranks by counting, integer window sums,
// the same fp64 operations).
// kStaged: every layer's scores are staged in shared memory at once (n_layers * T floats),
// with kClcesStagedTokens tokens per 64-thread CTA (twice the CTAs); otherwise one layer's
// scores at a time.
constexpr int kClcesStagedTokens = 8;
template <bool kStaged>
__global__ void __launch_bounds__(128) clces_layers_kernel(const float* __restrict__ s_all, int T, int n_layers,
                                                            int RW, float lam, const Entry* __restrict__ entries_all,
                                                            LayerStarts fr, int pool_pages, int P,
                                                            float* __restrict__ tok_shat_all) {
  extern __shared__ float s_sm[];
  constexpr int kTok = kStaged ? kClcesStagedTokens : kClcesTokens;
  __shared__ int rk[32][kTok];                  // [layer % RW][token of the CTA]
  const int sub = threadIdx.x & 7, tl = static_cast<int>(threadIdx.x >> 3);
  const int i = blockIdx.x * kTok + tl;
  const double sqrt12 = __dsqrt_rn(12.0);
  const double lamd = static_cast<double>(lam);
  if (kStaged) {
    const long long n = static_cast<long long>(n_layers) * T;
    for (long long j = threadIdx.x; j < n; j += blockDim.x) s_sm[j] = s_all[j];
    __syncthreads();
  }
  for (int l = 0; l < n_layers; ++l) {
    const float* s_l = s_sm;
    if (kStaged) {
      s_l = s_sm + static_cast<long long>(l) * T;
    } else {
      __syncthreads();                          // the previous layer's scores are no longer read
      const float* s = s_all + static_cast<long long>(l) * T;
      for (int j = threadIdx.x; j < T; j += blockDim.x) s_sm[j] = s[j];
      __syncthreads();
    }
    int r = 0;
    if (i < T) {
      const float si = s_l[i];
      for (int j = sub; j < T; j += 8) {
        const float sj = s_l[j];
        r += (sj > si) || (sj == si && j < i);
      }
    }
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 4);
    if (i < T && sub == 0) {
      rk[l % RW][tl] = r;
      const int w0 = max(0, l - RW + 1);
      const int n_win = l - w0 + 1;
      long long sr = 0, sr2 = 0;
      for (int k = w0; k <= l; ++k) {
        const long long v = rk[k % RW][tl];
        sr += v;
        sr2 += v * v;
      }
      const long long Dv = static_cast<long long>(n_win) * sr2 - sr * sr;
      const double sigma = __ddiv_rn(__dsqrt_rn(static_cast<double>(Dv)),
                                     __dmul_rn(static_cast<double>(n_win), static_cast<double>(T - 1)));
      double cons = __dsub_rn(1.0, __dmul_rn(sigma, sqrt12));
      if (cons < 0.0) cons = 0.0;
      const double w = __dmul_rn(static_cast<double>(s_l[i]), __dadd_rn(1.0, __dmul_rn(lamd, cons)));
      const long long lay = static_cast<long long>(l) * pool_pages;
      const int phys = entries_all[lay + fr.start[l] + i / P].x;
      tok_shat_all[(lay + phys) * P + (i % P)] = __double2float_rn(w);
    }
  }
}

// Metadata of a freshly appended frame: id = frame * T + slot, count 1, score 0.
__global__ void meta_init_kernel(int64_t* tok_id, int32_t* tok_cnt, float* tok_shat, const Entry* pages, int n_pages,
                                 int P, int T, int frame) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pages * P) return;
  const int g = idx / P, s = idx % P;
  const int tok = g * P + s;
  const long long phys = pages[g].x;
  const long long k = phys * P + s;
  tok_id[k] = tok < T ? static_cast<int64_t>(frame) * T + tok : -1;
  tok_cnt[k] = tok < T ? 1 : 0;
  tok_shat[k] = 0.f;
}

// The same for a batch of layers, blockIdx.y the layer of the batch (st.first_layer + y),
// its new entries starting at st.start[y].
__global__ void meta_init_layers_kernel(int64_t* tok_id_all, int32_t* tok_cnt_all, float* tok_shat_all,
                                        const Entry* entries_all, LayerStarts st, int pool_pages, int n_pages, int P,
                                        int T, int frame) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pages * P) return;
  const int layer = st.first_layer + static_cast<int>(blockIdx.y);
  const size_t base = static_cast<size_t>(layer) * pool_pages * P;
  const Entry* pages = entries_all + static_cast<size_t>(layer) * pool_pages + st.start[blockIdx.y];
  const int g = idx / P, s = idx % P;
  const int tok = g * P + s;
  const size_t k = base + static_cast<size_t>(pages[g].x) * P + s;
  tok_id_all[k] = tok < T ? static_cast<int64_t>(frame) * T + tok : -1;
  tok_cnt_all[k] = tok < T ? 1 : 0;
  tok_shat_all[k] = 0.f;
}

// Exclusive scan of v over the CTA (blockDim.x a multiple of 32, at most 1024); *total
// receives the CTA-wide sum. s_warp holds 32 ints.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
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
  const int excl = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
  *total = s_warp[nw - 1];
  __syncthreads();
  return excl;
}

// ------------------------------------------------------------------ tiering
// Flatten the cache into position order (page-table order, valid slots only; positions
// ascend with token id) with the metadata each later step needs: a one-CTA scan of the
// entries' valid counts gives each entry's first position, then one thread per slot.
__global__ void __launch_bounds__(1024) page_offsets_kernel(const Entry* __restrict__ entries, int n_entries,
                                                             Scratch sc) {
  __shared__ int s_warp[32];
  int base = 0;
  for (int chunk = 0; chunk < n_entries; chunk += blockDim.x) {
    const int e = chunk + threadIdx.x;
    const int v = e < n_entries ? entries[e].w : 0;
    int total;
    const int excl = cta_exclusive_scan(v, s_warp, &total);
    if (e < n_entries) sc.page_off[e] = base + excl;
    base += total;
  }
  if (threadIdx.x == 0) sc.counts[0] = base;
}

__global__ void gather_meta_kernel(const Entry* __restrict__ entries, int n_entries, int P,
                                   const int64_t* __restrict__ tok_id, const int32_t* __restrict__ tok_cnt,
                                   const float* __restrict__ tok_shat, int T, int specials, int protect_first,
                                   Scratch sc) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_entries * P) return;
  const int e = idx / P, sl = idx % P;
  const Entry en = entries[e];
  if (sl >= en.w) return;
  const int pos = sc.page_off[e] + sl;
  const long long k = static_cast<long long>(en.x) * P + sl;
  const int64_t id = tok_id[k];
  sc.ids[pos] = id;
  sc.shat[pos] = tok_shat[k];
  sc.cnt[pos] = tok_cnt[k];
  sc.slot[pos] = static_cast<int32_t>(k);
  const int64_t frame = id / T, tslot = id % T;
  sc.prot[pos] = (tslot < specials) || (protect_first && frame == 0);
}

// Order of the non-protected tokens by (s_hat descending, id ascending): positions ascend
// with id, so (key, position) with the key below is a strict total order.
__device__ __forceinline__ uint32_t desc_key(float f) {
  // maps larger floats to smaller unsigned keys (total order on finite values)
  uint32_t u = __float_as_uint(f);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~u;
}

// The k-th smallest (key, position) pair of the non-protected tokens for k = k1 and
// k = k2, by MSB-first radix selection on the 32-bit key (8 bits per pass); positions
// break ties, so the pair is fixed by the key value v and how many tokens of key v (in
// position order) come before it. Writes, per k: counts[8 + 2q] = v and counts[9 + 2q]
// = that number (a token of key v is among the k smallest iff its index among the
// non-protected tokens of key v is below it). k <= 0 selects nothing, k >= the number
// of non-protected tokens selects everything.
__global__ void __launch_bounds__(1024) tier_select_kernel(Scratch sc, int N, int k1, int k2) {
  __shared__ int hist[2][256];
  __shared__ uint32_t s_prefix[2];
  __shared__ int s_krem[2];
  __shared__ int s_np;
  __shared__ int s_warp[32];
  int np_local = 0;
  for (int i = threadIdx.x; i < N; i += blockDim.x) np_local += !sc.prot[i];
  int n_np;
  cta_exclusive_scan(np_local, s_warp, &n_np);
  if (threadIdx.x == 0) {
    s_np = n_np;
    s_prefix[0] = s_prefix[1] = 0u;
    s_krem[0] = k1;
    s_krem[1] = k2;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 512; b += blockDim.x) hist[b >> 8][b & 255] = 0;
    __syncthreads();
    const uint32_t hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    const uint32_t p0 = s_prefix[0], p1 = s_prefix[1];
    for (int base = 0; base < N; base += blockDim.x) {
      const int i = base + threadIdx.x;
      bool np = false;
      uint32_t key = 0;
      if (i < N) {
        np = !sc.prot[i];
        key = desc_key(sc.shat[i]);
      }
      const int digit = (key >> shift) & 255;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const bool in = np && ((key & hi_mask) == ((q ? p1 : p0) & hi_mask));
        const uint32_t act = __ballot_sync(0xffffffffu, in);
        if (in) {
          // one shared atomic per distinct digit of the warp
          const uint32_t peers = __match_any_sync(act, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[q][digit], __popc(peers));
        }
      }
    }
    __syncthreads();
    if (warp < 2) {
      const int q = warp;
      const int kr = s_krem[q];
      // lane owns digits [8 lane, 8 lane + 8)
      int c8[8], sum = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        c8[d] = hist[q][lane * 8 + d];
        sum += c8[d];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int before = incl - sum;
      int found = -1, krem_new = 0;
      if (kr >= 1 && before < kr && kr <= incl) {
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          if (found < 0 && kr <= before + c8[d]) {
            found = lane * 8 + d;
            krem_new = kr - before;
          }
          before += c8[d];
        }
      }
      if (found >= 0) {
        s_prefix[q] |= static_cast<uint32_t>(found) << shift;
        s_krem[q] = krem_new;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x < 2) {
    const int q = threadIdx.x;
    const int k = q ? k2 : k1;
    uint32_t v = s_prefix[q];
    int need = s_krem[q];
    if (k <= 0) {
      v = 0u;                 // nothing is below key 0 and no index is below 0
      need = 0;
    } else if (k >= s_np) {
      v = 0xFFFFFFFFu;        // everything: every key is <= v, every index below N
      need = 0x7fffffff;
    }
    sc.counts[8 + 2 * q] = static_cast<int32_t>(v);
    sc.counts[9 + 2 * q] = need;
  }
}

// Tier lists in position order: keep (protected, or among the n_keep_other smallest
// (key, position) pairs), eligible targets (kept, not protected) and merge sources (the
// next n_merge). Each thread walks a contiguous range of positions three times: counts of
// the threshold keys (two scans give each token its index among the non-protected tokens
// of those keys), counts per list (three scans give the list offsets), then the writes.
__global__ void __launch_bounds__(1024) tier_lists_kernel(Scratch sc, int N) {
  __shared__ int s_warp[32];
  const uint32_t v1 = static_cast<uint32_t>(sc.counts[8]), v2 = static_cast<uint32_t>(sc.counts[10]);
  const int need1 = sc.counts[9], need2 = sc.counts[11];
  const int ch = (N + blockDim.x - 1) / blockDim.x;
  const int i0 = min(N, static_cast<int>(threadIdx.x) * ch), i1 = min(N, i0 + ch);
  int c1 = 0, c2 = 0;
  for (int i = i0; i < i1; ++i) {
    const bool p = sc.prot[i];
    const uint32_t key = desc_key(sc.shat[i]);
    c1 += !p && key == v1;
    c2 += !p && key == v2;
  }
  int tot;
  const int b1 = cta_exclusive_scan(c1, s_warp, &tot);
  const int b2 = cta_exclusive_scan(c2, s_warp, &tot);
  // flags of position i given the running indices among the threshold keys
  auto flags = [&](int i, int& r1, int& r2, int (&f)[3]) {
    const bool p = sc.prot[i];
    const uint32_t key = desc_key(sc.shat[i]);
    const bool e1 = !p && key == v1, e2 = !p && key == v2;
    const bool lt1 = !p && (key < v1 || (e1 && r1 < need1));
    const bool lt2 = !p && (key < v2 || (e2 && r2 < need2));
    r1 += e1;
    r2 += e2;
    f[0] = p || lt1;
    f[1] = lt1;
    f[2] = !lt1 && lt2;
  };
  int n[3] = {0, 0, 0};
  {
    int r1 = b1, r2 = b2, f[3];
    for (int i = i0; i < i1; ++i) {
      flags(i, r1, r2, f);
      n[0] += f[0];
      n[1] += f[1];
      n[2] += f[2];
    }
  }
  int off[3], total[3];
#pragma unroll
  for (int q = 0; q < 3; ++q) off[q] = cta_exclusive_scan(n[q], s_warp, &total[q]);
  int* lists[3] = {sc.keep, sc.elig, sc.merge};
  {
    int r1 = b1, r2 = b2, f[3];
    for (int i = i0; i < i1; ++i) {
      flags(i, r1, r2, f);
#pragma unroll
      for (int q = 0; q < 3; ++q)
        if (f[q]) lists[q][off[q]++] = i;
    }
  }
  if (threadIdx.x == 0) {
    sc.counts[1] = total[0];
    sc.counts[2] = total[1];
    sc.counts[3] = total[2];
  }
}

// Tier selection and tier lists in one CTA with the candidates' keys and protected flags
// staged in shared memory once (N <= kTierSmemMax): the same MSB-first radix selection as
// tier_select_kernel and the same position-order scans as tier_lists_kernel, without their
// repeated global reads, which bound those kernels by load latency.
constexpr int kTierSmemMax = 40960;
__global__ void __launch_bounds__(1024) tier_kernel(Scratch sc, int N, int k1, int k2) {
  extern __shared__ __align__(16) uint8_t tier_sm[];
  uint32_t* key_s = reinterpret_cast<uint32_t*>(tier_sm);
  uint8_t* prot_s = tier_sm + static_cast<size_t>(N) * 4;
  __shared__ int hist[2][256];
  __shared__ uint32_t s_prefix[2];
  __shared__ int s_krem[2];
  __shared__ int s_np;
  __shared__ int s_warp[32];
  int np_local = 0;
#pragma unroll 4
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const uint8_t pr = sc.prot[i];
    key_s[i] = desc_key(sc.shat[i]);
    prot_s[i] = pr;
    np_local += !pr;
  }
  int n_np;
  cta_exclusive_scan(np_local, s_warp, &n_np);   // its barriers also publish the staged arrays
  if (threadIdx.x == 0) {
    s_np = n_np;
    s_prefix[0] = s_prefix[1] = 0u;
    s_krem[0] = k1;
    s_krem[1] = k2;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 512; b += blockDim.x) hist[b >> 8][b & 255] = 0;
    __syncthreads();
    const uint32_t hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    const uint32_t p0 = s_prefix[0], p1 = s_prefix[1];
    for (int base = 0; base < N; base += blockDim.x) {
      const int i = base + threadIdx.x;
      bool np = false;
      uint32_t key = 0;
      if (i < N) {
        np = !prot_s[i];
        key = key_s[i];
      }
      const int digit = (key >> shift) & 255;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const bool in = np && ((key & hi_mask) == ((q ? p1 : p0) & hi_mask));
        const uint32_t act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const uint32_t peers = __match_any_sync(act, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[q][digit], __popc(peers));
        }
      }
    }
    __syncthreads();
    if (warp < 2) {
      const int q = warp;
      const int kr = s_krem[q];
      int c8[8], sum = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        c8[d] = hist[q][lane * 8 + d];
        sum += c8[d];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int before = incl - sum;
      int found = -1, krem_new = 0;
      if (kr >= 1 && before < kr && kr <= incl) {
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          if (found < 0 && kr <= before + c8[d]) {
            found = lane * 8 + d;
            krem_new = kr - before;
          }
          before += c8[d];
        }
      }
      if (found >= 0) {
        s_prefix[q] |= static_cast<uint32_t>(found) << shift;
        s_krem[q] = krem_new;
      }
    }
    __syncthreads();
  }
  __shared__ uint32_t s_v[2];
  __shared__ int s_need[2];
  if (threadIdx.x < 2) {
    const int q = threadIdx.x;
    const int k = q ? k2 : k1;
    uint32_t v = s_prefix[q];
    int need = s_krem[q];
    if (k <= 0) {
      v = 0u;
      need = 0;
    } else if (k >= s_np) {
      v = 0xFFFFFFFFu;
      need = 0x7fffffff;
    }
    s_v[q] = v;
    s_need[q] = need;
    sc.counts[8 + 2 * q] = static_cast<int32_t>(v);
    sc.counts[9 + 2 * q] = need;
  }
  __syncthreads();
  // the three lists, each thread a contiguous range of positions
  const uint32_t v1 = s_v[0], v2 = s_v[1];
  const int need1 = s_need[0], need2 = s_need[1];
  const int ch = (N + blockDim.x - 1) / blockDim.x;
  const int i0 = min(N, static_cast<int>(threadIdx.x) * ch), i1 = min(N, i0 + ch);
  int c1 = 0, c2 = 0;
  for (int i = i0; i < i1; ++i) {
    const bool pr = prot_s[i];
    const uint32_t key = key_s[i];
    c1 += !pr && key == v1;
    c2 += !pr && key == v2;
  }
  int tot;
  const int b1 = cta_exclusive_scan(c1, s_warp, &tot);
  const int b2 = cta_exclusive_scan(c2, s_warp, &tot);
  auto flags = [&](int i, int& r1, int& r2, int (&f)[3]) {
    const bool pr = prot_s[i];
    const uint32_t key = key_s[i];
    const bool e1 = !pr && key == v1, e2 = !pr && key == v2;
    const bool lt1 = !pr && (key < v1 || (e1 && r1 < need1));
    const bool lt2 = !pr && (key < v2 || (e2 && r2 < need2));
    r1 += e1;
    r2 += e2;
    f[0] = pr || lt1;
    f[1] = lt1;
    f[2] = !lt1 && lt2;
  };
  int n[3] = {0, 0, 0};
  {
    int r1 = b1, r2 = b2, f[3];
    for (int i = i0; i < i1; ++i) {
      flags(i, r1, r2, f);
      n[0] += f[0];
      n[1] += f[1];
      n[2] += f[2];
    }
  }
  int off[3], total[3];
#pragma unroll
  for (int q = 0; q < 3; ++q) off[q] = cta_exclusive_scan(n[q], s_warp, &total[q]);
  int* lists[3] = {sc.keep, sc.elig, sc.merge};
  {
    int r1 = b1, r2 = b2, f[3];
    for (int i = i0; i < i1; ++i) {
      flags(i, r1, r2, f);
#pragma unroll
      for (int q = 0; q < 3; ++q)
        if (f[q]) lists[q][off[q]++] = i;
    }
  }
  if (threadIdx.x == 0) {
    sc.counts[1] = total[0];
    sc.counts[2] = total[1];
    sc.counts[3] = total[2];
  }
}

// ------------------------------------------------------------------ merge targets
// Full H*D keys of listed tokens (the stored bf16 values), their fp64 norms and fp32
// inverse norms.
__global__ void gather_keys_kernel(const int32_t* __restrict__ list, const int32_t* __restrict__ count, int cap,
                                   const int32_t* __restrict__ slot, const __nv_bfloat16* __restrict__ k_pool,
                                   int H, int P, int D, __nv_bfloat16* __restrict__ out, double* __restrict__ norms,
                                   float* __restrict__ inv_norms) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int n = min(*count, cap);
  if (w >= n) return;
  const int pos = list[w];
  const long long k = slot[pos];
  const long long phys = k / P, s = k % P;
  const int HD = H * D;
  double acc = 0.0;
  for (int c = lane; c < HD; c += 32) {
    const int h = c / D, d = c % D;
    const __nv_bfloat16 xb = k_pool[((phys * H + h) * P + s) * D + d];
    out[static_cast<long long>(w) * HD + c] = xb;
    const double x = static_cast<double>(__bfloat162float(xb));
    acc = fma(x, x, acc);
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const double n = sqrt(acc);
    norms[w] = n;
    inv_norms[w] = static_cast<float>(1.0 / n);
  }
}

// Merge sources grouped by target, each group in ascending source index: counts per
// target, their exclusive scan (the group offsets), a scatter, then a sort of every group
// (groups are small). One CTA; every step is deterministic.
__global__ void __launch_bounds__(1024) merge_group_kernel(Scratch sc, int n_src, int n_elig, int H, int P, int D) {
  __shared__ int s_warp[32];
  for (int e = threadIdx.x; e <= n_elig; e += blockDim.x) sc.bucket[e] = 0;
  for (int e = threadIdx.x; e < n_elig; e += blockDim.x) sc.cursor[e] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n_src; i += blockDim.x) atomicAdd(&sc.bucket[sc.target[i] + 1], 1);
  __syncthreads();
  {
    // group ends: an inclusive scan of the counts, contiguous ranges per thread
    const int ch = (n_elig + blockDim.x - 1) / blockDim.x;
    const int e0 = min(n_elig, static_cast<int>(threadIdx.x) * ch), e1 = min(n_elig, e0 + ch);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += sc.bucket[e + 1];
    int total;
    int run = cta_exclusive_scan(local, s_warp, &total);
    for (int e = e0; e < e1; ++e) {
      run += sc.bucket[e + 1];
      sc.bucket[e + 1] = run;                                // inclusive: end of group e
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_src; i += blockDim.x) {
    const int e = sc.target[i];
    sc.order[sc.bucket[e] + atomicAdd(&sc.cursor[e], 1)] = i;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_elig; e += blockDim.x) {
    const int b = sc.bucket[e], n = sc.bucket[e + 1] - b;
    for (int x = 1; x < n; ++x) {                          // insertion sort of the group
      const int v = sc.order[b + x];
      int y = x - 1;
      while (y >= 0 && sc.order[b + y] > v) {
        sc.order[b + y + 1] = sc.order[b + y];
        --y;
      }
      sc.order[b + y + 1] = v;
    }
  }
  __syncthreads();
  for (int q = threadIdx.x; q < n_src; q += blockDim.x) {
    const int pos = sc.merge[sc.order[q]];
    const long long k = sc.slot[pos];
    sc.src_base[q] = ((k / P) * H * P + k % P) * D;
    sc.src_cnt[q] = sc.cnt[pos];
  }
}

// merge_group_kernel with its counting sort in shared memory (group ends, cursors and the
// grouped order; n_src + 2 n_elig + 1 ints <= kGroupSmemInts), written to the scratch once
// at the end: the global version is bound by the latency of its atomics and of the
// insertion sort's global accesses.
constexpr int kGroupSmemInts = 53248;
__global__ void __launch_bounds__(1024) merge_group_smem_kernel(Scratch sc, int n_src, int n_elig, int H, int P,
                                                                int D) {
  extern __shared__ __align__(16) int grp_sm[];
  int* bucket = grp_sm;                    // [n_elig + 1]
  int* cursor = bucket + n_elig + 1;       // [n_elig]
  int* order = cursor + n_elig;            // [n_src]
  __shared__ int s_warp[32];
  for (int e = threadIdx.x; e <= n_elig; e += blockDim.x) bucket[e] = 0;
  for (int e = threadIdx.x; e < n_elig; e += blockDim.x) cursor[e] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n_src; i += blockDim.x) atomicAdd(&bucket[sc.target[i] + 1], 1);
  __syncthreads();
  {
    const int ch = (n_elig + blockDim.x - 1) / blockDim.x;
    const int e0 = min(n_elig, static_cast<int>(threadIdx.x) * ch), e1 = min(n_elig, e0 + ch);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += bucket[e + 1];
    int total;
    int run = cta_exclusive_scan(local, s_warp, &total);
    for (int e = e0; e < e1; ++e) {
      run += bucket[e + 1];
      bucket[e + 1] = run;                                   // inclusive: end of group e
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_src; i += blockDim.x) {
    const int e = sc.target[i];
    order[bucket[e] + atomicAdd(&cursor[e], 1)] = i;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_elig; e += blockDim.x) {
    const int b = bucket[e], n = bucket[e + 1] - b;
    for (int x = 1; x < n; ++x) {                          // insertion sort of the group
      const int v = order[b + x];
      int y = x - 1;
      while (y >= 0 && order[b + y] > v) {
        order[b + y + 1] = order[b + y];
        --y;
      }
      order[b + y + 1] = v;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= n_elig; e += blockDim.x) sc.bucket[e] = bucket[e];
  for (int q = threadIdx.x; q < n_src; q += blockDim.x) {
    const int o = order[q];
    sc.order[q] = o;
    const int pos = sc.merge[o];
    const long long k = sc.slot[pos];
    sc.src_base[q] = ((k / P) * H * P + k % P) * D;
    sc.src_cnt[q] = sc.cnt[pos];
  }
}

// For every eligible target with at least one source: acc = c_j x_j, then acc += c_m x_m
// for its sources in ascending id, all in fp64; x_j = bf16(acc / sum of counts), for
// every dimension of K and V; the count becomes the sum. Sources are read before any
// target is written because no token is both. A thread takes 8 consecutive dims of one
// head row (16-byte loads of the target and of each source, 8 accumulators).
__global__ void __launch_bounds__(256) merge_apply_kernel(Scratch sc, int cap_src, int cap_elig,
                                                          __nv_bfloat16* k_pool, __nv_bfloat16* v_pool, int H, int P,
                                                          int D) {
  const int e = blockIdx.x;
  const int n_elig = min(sc.counts[2], cap_elig);
  if (e >= n_elig) return;
  const int begin = sc.bucket[e], end = sc.bucket[e + 1];
  if (begin == end) return;
  const int jpos = sc.elig[e];
  const long long kj = sc.slot[jpos];
  const long long bj = ((kj / P) * H * P + kj % P) * D;
  const int cj = sc.cnt[jpos];
  int tot = cj;
  for (int q = begin; q < end; ++q) tot += sc.src_cnt[q];
  const double dtot = static_cast<double>(tot);
  const int chunks = H * D / 8;                     // 8-dim chunks of one tensor's row
  for (int ch = threadIdx.x; ch < 2 * chunks; ch += blockDim.x) {
    const bool is_v = ch >= chunks;
    __nv_bfloat16* pool = is_v ? v_pool : k_pool;
    const int cc = (is_v ? ch - chunks : ch) * 8;
    const long long off = static_cast<long long>(cc / D) * P * D + cc % D;
    const uint4 tj = *reinterpret_cast<const uint4*>(pool + bj + off);
    const __nv_bfloat16* tv = reinterpret_cast<const __nv_bfloat16*>(&tj);
    double acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      acc[k] = __dmul_rn(static_cast<double>(cj), static_cast<double>(__bfloat162float(tv[k])));
    for (int q = begin; q < end; ++q) {
      const uint4 xm = *reinterpret_cast<const uint4*>(pool + sc.src_base[q] + off);
      const __nv_bfloat16* xv = reinterpret_cast<const __nv_bfloat16*>(&xm);
      const double cm = static_cast<double>(sc.src_cnt[q]);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        acc[k] = __dadd_rn(acc[k], __dmul_rn(cm, static_cast<double>(__bfloat162float(xv[k]))));
    }
    uint4 o;
    __nv_bfloat16* ov = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
    for (int k = 0; k < 8; ++k) ov[k] = f64_to_bf16_rne(__ddiv_rn(acc[k], dtot));
    *reinterpret_cast<uint4*>(pool + bj + off) = o;
  }
  if (threadIdx.x == 0) sc.cnt[jpos] = tot;
}

__global__ void record_merges_kernel(Scratch sc, int cap_src, int64_t* last_src, int64_t* last_dst) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = min(sc.counts[3], cap_src);
  if (i >= n) return;
  last_src[i] = sc.ids[sc.merge[i]];
  last_dst[i] = sc.ids[sc.elig[sc.target[i]]];
}

// Rewrite kept tokens, in position (= id) order, into the freshly allocated pages:
// K, V (one warp per token, 16-byte rows) and the metadata; tail slots are zeroed.
__global__ void compact_kernel(Scratch sc, int cap_keep, const Entry* __restrict__ new_pages, int n_new_pages,
                               __nv_bfloat16* k_pool, __nv_bfloat16* v_pool, int64_t* tok_id, int32_t* tok_cnt,
                               float* tok_shat, int H, int P, int D) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int n_keep = min(sc.counts[1], cap_keep);
  if (w >= n_new_pages * P) return;
  const long long nphys = new_pages[w / P].x;
  const int ns = w % P;
  const long long nk = nphys * P + ns;
  const int chunks = D / 8;   // 16-byte chunks per head row
  if (w < n_keep) {
    const int pos = sc.keep[w];
    const long long ok = sc.slot[pos];
    const long long ophys = ok / P, os = ok % P;
    for (int c = lane; c < H * chunks; c += 32) {
      const int h = c / chunks, q = c % chunks;
      const long long src = ((ophys * H + h) * P + os) * D + q * 8;
      const long long dst = ((nphys * H + h) * P + ns) * D + q * 8;
      *reinterpret_cast<uint4*>(k_pool + dst) = *reinterpret_cast<const uint4*>(k_pool + src);
      *reinterpret_cast<uint4*>(v_pool + dst) = *reinterpret_cast<const uint4*>(v_pool + src);
    }
    if (lane == 0) {
      tok_id[nk] = sc.ids[pos];
      tok_cnt[nk] = sc.cnt[pos];
      tok_shat[nk] = sc.shat[pos];
    }
  } else {
    for (int c = lane; c < H * chunks; c += 32) {
      const int h = c / chunks, q = c % chunks;
      const long long dst = ((nphys * H + h) * P + ns) * D + q * 8;
      *reinterpret_cast<uint4*>(k_pool + dst) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(v_pool + dst) = make_uint4(0, 0, 0, 0);
    }
    if (lane == 0) {
      tok_id[nk] = -1;
      tok_cnt[nk] = 0;
      tok_shat[nk] = 0.f;
    }
  }
}

__global__ void check_counts_kernel(const int32_t* counts, int n, int keep, int elig, int merge, int* err) {
  if (counts[0] != n || counts[1] != keep || counts[2] != elig || counts[3] != merge) latch_error(err, DERR_BOUNDS);
}

}  // namespace

size_t compress_scratch_bytes(const kvc_config& cfg, int pool_pages) { return carve(cfg, nullptr, nullptr); }

kvc_status init_token_meta(kvc_cache* c, int layer, int first_entry, int n_pages, int frame) {
  const int P = c->cfg.page_size;
  const size_t base = static_cast<size_t>(layer) * c->pool_pages * P;
  const Entry* pages = c->entries + static_cast<size_t>(layer) * c->pool_pages + first_entry;
  const int n = n_pages * P;
  meta_init_kernel<<<(n + 255) / 256, 256, 0, c->stream>>>(c->tok_id + base, c->tok_cnt + base, c->tok_shat + base,
                                                           pages, n_pages, P, c->cfg.tokens_per_frame, frame);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    c->last_error = std::string("token metadata: ") + cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  c->launches++;
  return KVC_OK;
}

kvc_status init_token_meta_layers(kvc_cache* c, const LayerStarts& st, int n_layers, int n_pages, int frame) {
  const int P = c->cfg.page_size;
  const int n = n_pages * P;
  meta_init_layers_kernel<<<dim3((n + 255) / 256, n_layers), 256, 0, c->stream>>>(
      c->tok_id, c->tok_cnt, c->tok_shat, c->entries, st, c->pool_pages, n_pages, P, c->cfg.tokens_per_frame, frame);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    c->last_error = std::string("token metadata: ") + cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  c->launches++;
  return KVC_OK;
}

// Scratch set i (of kCmpSets); the raw scores and the merge records always live in set 0.
Scratch scratch_set(kvc_cache* c, int i) {
  Scratch s0, si;
  uint8_t* base = static_cast<uint8_t*>(c->cmp_scratch);
  carve(c->cfg, base, &s0);
  carve(c->cfg, base + static_cast<size_t>(i) * c->cmp_scratch_bytes, &si);
  si.s_raw = s0.s_raw;
  si.last_src = s0.last_src;
  si.last_dst = s0.last_dst;
  return si;
}

// Scoring of the frame just committed on `layer` (raw score, CLCES rank, s_hat), on the
// cache's stream with scratch set 0. Layers of a frame come in ascending order.
kvc_status score_layer(kvc_cache* c, int layer, const float* residual) {
  const kvc_config& g = c->cfg;
  LayerHost& L = c->L[layer];
  if (L.has_pending || L.frames.empty() || L.frames.back().frame != L.last_frame) {
    c->last_error = "kvc_compress: call after kvc_attend of the frame, before the next append";
    return KVC_ERR_STATE;
  }
  const int t = L.last_frame;
  if (L.scored_frame == t) {
    c->last_error = "kvc_compress: this layer's frame was already scored";
    return KVC_ERR_STATE;
  }
  // rank history of the current frame: layers must come in ascending order
  if (c->hist_frame != t) {
    c->hist_frame = t;
    c->hist_next_layer = 0;
    c->hist_layers.clear();
  }
  if (layer < c->hist_next_layer) {
    c->last_error = "kvc_compress: layers of a frame must be scored in ascending order";
    return KVC_ERR_STATE;
  }
  const Scratch sc = scratch_set(c, 0);
  const int T = g.tokens_per_frame, P = g.page_size;
  const int RW = g.rank_window;
  const size_t lay_slots = static_cast<size_t>(layer) * c->pool_pages * P;
  Entry* E = c->entries + static_cast<size_t>(layer) * c->pool_pages;
  cudaStream_t s = c->stream;
  cudaError_t e = cudaSuccess;
  auto ok = [&]() {
    cudaError_t r = cudaGetLastError();
    if (r != cudaSuccess && e == cudaSuccess) e = r;
    c->launches++;
  };

  // ---- scoring of the frame just committed
  c->hist_layers.push_back(layer);
  uint32_t mask = 0;
  int n_win = 0;
  for (int l : c->hist_layers)
    if (l > layer - RW && l <= layer) {
      mask |= 1u << (l % RW);
      ++n_win;
    }
  residual_norm_kernel<<<(T * 32 + 255) / 256, 256, 0, s>>>(residual, T, g.residual_dim, sc.s_raw);
  ok();
  const FrameRec& fr = L.frames.back();
  clces_kernel<<<(T + kClcesTokens - 1) / kClcesTokens, 128, T * sizeof(float), s>>>(sc.s_raw, T, c->rank_hist, layer % RW, mask, n_win, g.lambda_,
                                                  E + fr.first_entry, P, c->tok_shat + lay_slots);
  ok();
  c->hist_next_layer = layer + 1;
  L.scored_frame = t;
  if (e != cudaSuccess) {
    c->last_error = std::string("kvc_compress scoring: ") + cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  return KVC_OK;
}

// Compression of a layer over its budget, on stream s with scratch set sc (no other
// compression may use sc meanwhile). Host checks come before any launch.
kvc_status compress_body(kvc_cache* c, int layer, cudaStream_t s, const Scratch& sc, int32_t* fired) {
  const kvc_config& g = c->cfg;
  LayerHost& L = c->L[layer];
  const Caps cp = caps_of(g);
  const int T = g.tokens_per_frame, P = g.page_size, H = g.num_heads, D = g.head_dim;
  const size_t lay_slots = static_cast<size_t>(layer) * c->pool_pages * P;
  Entry* E = c->entries + static_cast<size_t>(layer) * c->pool_pages;
  cudaError_t e = cudaSuccess;
  auto ok = [&]() {
    cudaError_t r = cudaGetLastError();
    if (r != cudaSuccess && e == cudaSuccess) e = r;
    c->launches++;
  };
  // a failed launch stops the sequence: later kernels index by the tier lists and the page
  // entries that the failed one was to write
  auto fail = [&]() {
    c->last_error = std::string("kvc_compress: ") + cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  };
  const int B = g.budget_tokens;
  const int N = static_cast<int>(L.tokens);
  const int n_keep = static_cast<int>(cp.n_keep);
  const int n_merge_cap = B - n_keep;
  const int n_prot = static_cast<int>(L.protected_tokens);
  if (n_prot > n_keep) {
    c->last_error = "kvc_compress: protected tokens exceed the keep tier";
    return KVC_ERR_BUDGET;
  }
  const int n_keep_other = n_keep - n_prot;
  int n_merge = std::min(n_merge_cap, N - n_keep);
  if (n_keep_other == 0) n_merge = 0;   // no eligible target: the merge tier is dropped
  __nv_bfloat16* kp = reinterpret_cast<__nv_bfloat16*>(c->k_pool) + static_cast<size_t>(layer) * c->pool_pages * c->page_elems;
  __nv_bfloat16* vp = reinterpret_cast<__nv_bfloat16*>(c->v_pool) + static_cast<size_t>(layer) * c->pool_pages * c->page_elems;

  page_offsets_kernel<<<1, 1024, 0, s>>>(E, L.n_entries, sc);
  ok();
  gather_meta_kernel<<<(L.n_entries * P + 255) / 256, 256, 0, s>>>(E, L.n_entries, P, c->tok_id + lay_slots,
                                                                     c->tok_cnt + lay_slots,
                                        c->tok_shat + lay_slots, T, g.num_special_tokens, g.protect_first_frame, sc);
  ok();
  if (N <= kTierSmemMax) {
    static PerDeviceOnce attr;
    cudaError_t ea = attr.run([] {
      return cudaFuncSetAttribute(tier_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTierSmemMax * 5);
    });
    if (ea != cudaSuccess && e == cudaSuccess) e = ea;
    tier_kernel<<<1, 1024, static_cast<size_t>(N) * 5, s>>>(sc, N, n_keep_other, n_keep_other + n_merge);
    ok();
  } else {
    tier_select_kernel<<<1, 1024, 0, s>>>(sc, N, n_keep_other, n_keep_other + n_merge);
    ok();
    tier_lists_kernel<<<1, 1024, 0, s>>>(sc, N);
    ok();
  }
  check_counts_kernel<<<1, 1, 0, s>>>(sc.counts, N, n_keep, n_keep_other, n_merge, c->d_err);
  ok();
  if (e != cudaSuccess) return fail();
  const int HD = H * D;
  int64_t* lsrc = sc.last_src + static_cast<size_t>(layer) * cp.n_merge;
  int64_t* ldst = sc.last_dst + static_cast<size_t>(layer) * cp.n_merge;
  if (n_merge > 0) {
    gather_keys_kernel<<<(n_merge * 32 + 255) / 256, 256, 0, s>>>(sc.merge, sc.counts + 3, static_cast<int>(cp.n_merge),
                                                                   sc.slot, kp, H, P, D, sc.ks, sc.ns, sc.inv_ns);
    ok();
    gather_keys_kernel<<<(n_keep_other * 32 + 255) / 256, 256, 0, s>>>(
        sc.elig, sc.counts + 2, static_cast<int>(cp.n_keep), sc.slot, kp, H, P, D, sc.ke, sc.ne, sc.inv_ne);
    ok();
    // merge targets: tensor-core screen, fp64 decision among the screened candidates
    int launched = 0;
    cudaError_t r = launch_merge_targets(s, sc.ks, sc.ke, sc.ns, sc.ne, sc.inv_ns, sc.inv_ne, n_merge, n_keep_other,
                                         HD, sc.top_v, sc.top_j, static_cast<int>(cp.tiles), sc.target, c->d_err,
                                         &launched);
    if (r != cudaSuccess && e == cudaSuccess) e = r;
    c->launches += launched;
    if (n_merge + 2 * n_keep_other + 1 <= kGroupSmemInts) {
      static PerDeviceOnce attr;
      cudaError_t ea = attr.run([] {
        return cudaFuncSetAttribute(merge_group_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kGroupSmemInts * 4);
      });
      if (ea != cudaSuccess && e == cudaSuccess) e = ea;
      merge_group_smem_kernel<<<1, 1024, static_cast<size_t>(n_merge + 2 * n_keep_other + 1) * 4, s>>>(
          sc, n_merge, n_keep_other, H, P, D);
    } else {
      merge_group_kernel<<<1, 1024, 0, s>>>(sc, n_merge, n_keep_other, H, P, D);
    }
    ok();
    merge_apply_kernel<<<n_keep_other, 256, 0, s>>>(sc, static_cast<int>(cp.n_merge), static_cast<int>(cp.n_keep),
                                                    kp, vp, H, P, D);
    ok();
    record_merges_kernel<<<(n_merge + 255) / 256, 256, 0, s>>>(sc, static_cast<int>(cp.n_merge), lsrc, ldst);
    ok();
  }
  if (e != cudaSuccess) return fail();
  // compaction into the lowest free pages, then release every old page
  const int n_old = L.n_entries;
  const int n_new = (n_keep + P - 1) / P;
  if (n_old + n_new > c->pool_pages) {
    c->last_error = "kvc_compress: page pool too small for compaction";
    return KVC_ERR_STATE;
  }
  e = launch_mgr_alloc(s, E, layer_free_bitmap(c, layer), c->bitmap_words, c->pool_pages, n_old, n_new, -1, P,
                       n_keep - (n_new - 1) * P, c->d_err);
  c->launches++;
  if (e != cudaSuccess) return fail();
  compact_kernel<<<(n_new * P * 32 + 255) / 256, 256, 0, s>>>(sc, static_cast<int>(cp.n_keep), E + n_old, n_new, kp, vp,
                                                              c->tok_id + lay_slots, c->tok_cnt + lay_slots,
                                                              c->tok_shat + lay_slots, H, P, D);
  ok();
  if (e != cudaSuccess) return fail();
  e = launch_mgr_remove(s, E, layer_free_bitmap(c, layer), n_old + n_new, 0, n_old, c->d_err);
  c->launches++;
  if (e != cudaSuccess) return fail();
  L.n_entries = n_new;
  L.frames.clear();
  L.block_entries = n_new;
  L.block_tokens = n_keep;
  L.tokens = n_keep;
  L.compressions++;
  L.last_merge_n = n_merge;
  L.high_water = std::max<int64_t>(L.high_water, n_old + n_new);
  if (fired) *fired = 1;
  return KVC_OK;
}

// Every layer of the frame scored in two launches (raw scores, then CLCES of all layers),
// with the results of score_layer on layers 0, 1, ... in order; kvc_last_raw_scores then
// gives the last layer's raw scores. Used when every layer is at the same frame and none of
// its layers has been scored yet; otherwise the layers are scored one by one.
kvc_status score_all_layers(kvc_cache* c, const float* const* residuals) {
  const kvc_config& g = c->cfg;
  const int nl = g.num_layers;
  const int t = c->L[0].last_frame;
  bool batch = nl <= kMaxBatchLayers && g.rank_window <= 32 && !(c->hist_frame == t && c->hist_next_layer > 0);
  for (int l = 0; l < nl && batch; ++l) {
    const LayerHost& L = c->L[l];
    if (L.last_frame != t || L.has_pending || L.frames.empty() || L.frames.back().frame != t || L.scored_frame == t)
      batch = false;
  }
  if (!batch) {
    for (int l = 0; l < nl; ++l) {
      kvc_status st = score_layer(c, l, residuals[l]);
      if (st != KVC_OK) return st;
    }
    return KVC_OK;
  }
  const Scratch sc = scratch_set(c, 0);
  const int T = g.tokens_per_frame, P = g.page_size;
  ResidualBatch rb{};
  LayerStarts fr{};
  for (int l = 0; l < nl; ++l) {
    rb.r[l] = residuals[l];
    fr.start[l] = c->L[l].frames.back().first_entry;
  }
  cudaStream_t s = c->stream;
  residual_norm_layers_kernel<<<dim3((T * 32 + 255) / 256, nl), 256, 0, s>>>(rb, T, g.residual_dim, sc.s_raw_all);
  cudaError_t e = cudaGetLastError();
  c->launches++;
  if (e == cudaSuccess) {
    const size_t staged = static_cast<size_t>(nl) * T * sizeof(float);
    constexpr size_t kStagedMax = 200 * 1024;
    if (staged <= kStagedMax) {
      static PerDeviceOnce attr;
      e = attr.run([] {
        return cudaFuncSetAttribute(clces_layers_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kStagedMax));
      });
      if (e == cudaSuccess)
        clces_layers_kernel<true><<<(T + kClcesStagedTokens - 1) / kClcesStagedTokens, 8 * kClcesStagedTokens, staged,
                                    s>>>(sc.s_raw_all, T, nl, g.rank_window, g.lambda_, c->entries, fr,
                                         c->pool_pages, P, c->tok_shat);
    } else {
      clces_layers_kernel<false><<<(T + kClcesTokens - 1) / kClcesTokens, 8 * kClcesTokens, T * sizeof(float), s>>>(
          sc.s_raw_all, T, nl, g.rank_window, g.lambda_, c->entries, fr, c->pool_pages, P, c->tok_shat);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    c->launches++;
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(sc.s_raw, sc.s_raw_all + static_cast<size_t>(nl - 1) * T, static_cast<size_t>(T) * sizeof(float),
                        cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) {
    c->last_error = std::string("kvc_compress_all scoring: ") + cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  c->hist_frame = t;
  c->hist_layers.clear();
  for (int l = 0; l < nl; ++l) {
    c->hist_layers.push_back(l);
    c->L[l].scored_frame = t;
  }
  c->hist_next_layer = nl;
  return KVC_OK;
}

kvc_status compress_layer(kvc_cache* c, int layer, const float* residual, int32_t* fired) {
  kvc_status st = score_layer(c, layer, residual);
  if (st != KVC_OK) return st;
  if (c->L[layer].tokens <= c->cfg.budget_tokens) return KVC_OK;
  return compress_body(c, layer, c->stream, scratch_set(c, 0), fired);
}

// Every layer scored in ascending order on the cache's stream (the CLCES rank window
// spans layers), then the layers over budget compressed side by side: layer k of them on
// side stream k mod kCmpSets with scratch set k mod kCmpSets, forked from and joined back
// into the cache's stream. A layer's compression reads and writes only that layer's pages,
// page table, token metadata and free bitmap, so the layers are independent.
kvc_status compress_all_layers(kvc_cache* c, const float* const* residuals, int32_t* fired) {
  const kvc_config& g = c->cfg;
  for (int l = 0; l < g.num_layers; ++l)
    if (fired) fired[l] = 0;
  kvc_status sst = score_all_layers(c, residuals);
  if (sst != KVC_OK) return sst;
  std::vector<int> todo;
  for (int l = 0; l < g.num_layers; ++l)
    if (c->L[l].tokens > g.budget_tokens) todo.push_back(l);
  const int n = static_cast<int>(todo.size());
  if (n == 0) return KVC_OK;
  const int sets = std::min(n, static_cast<int>(kvc_cache::kCmpSets));
  cudaError_t e = cudaEventRecord(c->cmp_fork, c->stream);
  for (int i = 0; i < sets && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(c->cmp_stream[i], c->cmp_fork, 0);
  if (e != cudaSuccess) {
    c->last_error = std::string("kvc_compress_all fork: ") + cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  kvc_status first = KVC_OK;
  for (int k = 0; k < n; ++k) {
    const int i = k % sets;
    kvc_status st = compress_body(c, todo[k], c->cmp_stream[i], scratch_set(c, i), fired ? &fired[todo[k]] : nullptr);
    if (st != KVC_OK && first == KVC_OK) first = st;
  }
  // join every side stream back, whatever happened above
  for (int i = 0; i < sets; ++i) {
    cudaError_t r = cudaEventRecord(c->cmp_join[i], c->cmp_stream[i]);
    if (r == cudaSuccess) r = cudaStreamWaitEvent(c->stream, c->cmp_join[i], 0);
    if (r != cudaSuccess && e == cudaSuccess) e = r;
  }
  if (e != cudaSuccess && first == KVC_OK) {
    c->last_error = std::string("kvc_compress_all join: ") + cudaGetErrorString(e);
    first = KVC_ERR_CUDA;
  }
  return first;
}

}  // namespace kvc

extern "C" kvc_status kvc_last_merge(kvc_cache* c, int32_t layer, int64_t* src_host, int64_t* dst_host,
                                     int32_t capacity, int32_t* n_out) {
  if (!c) return KVC_ERR_ARG;
  if (n_out) *n_out = 0;
  if (layer < 0 || layer >= c->cfg.num_layers) {
    c->last_error = "kvc_last_merge: bad layer";
    return KVC_ERR_ARG;
  }
  if (c->cfg.budget_tokens <= 0) {
    c->last_error = "kvc_last_merge: budget_tokens is 0";
    return KVC_ERR_ARG;
  }
  cudaError_t e = cudaStreamSynchronize(c->stream);
  if (e != cudaSuccess) {
    c->last_error = cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  kvc::Scratch sc;
  kvc::carve(c->cfg, static_cast<uint8_t*>(c->cmp_scratch), &sc);
  const kvc::Caps cp = kvc::caps_of(c->cfg);
  const int n = c->L[layer].last_merge_n;
  const int m = std::min(n, capacity);
  if (m > 0) {
    if (src_host)
      e = cudaMemcpy(src_host, sc.last_src + static_cast<size_t>(layer) * cp.n_merge, m * 8, cudaMemcpyDeviceToHost);
    if (dst_host && e == cudaSuccess)
      e = cudaMemcpy(dst_host, sc.last_dst + static_cast<size_t>(layer) * cp.n_merge, m * 8, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
      c->last_error = std::string("kvc_last_merge copy: ") + cudaGetErrorString(e);
      return KVC_ERR_CUDA;
    }
  }
  if (n_out) *n_out = n;
  return KVC_OK;
}

extern "C" kvc_status kvc_last_raw_scores(kvc_cache* c, float* s_host, int32_t capacity, int32_t* n_out) {
  if (!c) return KVC_ERR_ARG;
  if (n_out) *n_out = 0;
  const int T = c->cfg.tokens_per_frame;
  if (c->cfg.budget_tokens <= 0 || !s_host || capacity < T) {
    c->last_error = "kvc_last_raw_scores: budget_tokens is 0, or no host array of tokens_per_frame floats";
    return KVC_ERR_ARG;
  }
  if (c->hist_layers.empty() && c->hist_frame < 0) {
    c->last_error = "kvc_last_raw_scores: nothing scored yet";
    return KVC_ERR_STATE;
  }
  kvc::Scratch sc;
  kvc::carve(c->cfg, static_cast<uint8_t*>(c->cmp_scratch), &sc);
  cudaError_t e = cudaStreamSynchronize(c->stream);
  if (e == cudaSuccess) e = cudaMemcpy(s_host, sc.s_raw, static_cast<size_t>(T) * sizeof(float), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    c->last_error = cudaGetErrorString(e);
    return KVC_ERR_CUDA;
  }
  if (n_out) *n_out = T;
  return KVC_OK;
}
