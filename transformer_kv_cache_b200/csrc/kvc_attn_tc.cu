// kvc_attn_tc.cu -- frame attention over the paged bf16 cache on sm_100a tensor cores.
//
// Computes O[i, h] = sum_j softmax_j(scale * q_i . k_j) v_j for the T queries of the new
// frame over every valid slot of the layer's page list ("How GCTStream ...",
// Frame-by-Frame Causal Processing; "InfiniteVGGT" explainer, Causal Attention) without
// materialising the score matrix, as a flash-attention pipeline built for Blackwell. Each
// CTA owns one 128-row query tile of one head and a range of 64-slot KV tiles (4 pages):
//
//   warp 0 (one lane)   TMA producer: per KV tile the 4 pages of K and of V, each
//                       page-head block one 2-D box, into a ring of 128-byte-swizzled
//                       stages. Pages past the end of the list are read past the end of the
//                       pool, which TMA fills with zeros.
//   warp 1              MMA issuer (the warp waits, one elected lane issues): S = Q K^T
//                       (tcgen05.mma kind::f16, M=128, N=64, A = Q read from TMEM) into
//                       TMEM, then O' += P [V | 1] (M=128, N=80, A = P read from TMEM,
//                       B = the V tile as an MN-major operand followed by a constant block
//                       of ones), so accumulator column 64 carries the row sum of P.
//   warps 2..5          softmax, thread = query row = TMEM lane. First each thread stores
//                       its row of Q into TMEM (so S reads only K from shared memory);
//                       then per KV tile, 64 columns:
//                       x = s*c - m with packed f32x2 FMAs, P = 2^x on the MUFU, its upper
//                       halves taken as the bf16 pairs the MMA consumes (one byte permute
//                       per pair) and written back to TMEM (tcgen05.st); no per-element sum
//                       (the MMA makes it from the same bf16 P). The next tile's S is
//                       loaded from TMEM while this tile's P store is in flight.
//
// Online softmax with lazy rescaling: the reference max m of a row only moves when a
// tile's P would exceed 2^8; the common case costs a bf16x2 max over the packed P and no
// fp32 max at all. When a row's reference moves (the first tile, or a
// new maximum), the exact fp32 tile max is taken and O' (including the row-sum column) is
// rescaled in TMEM. The result is exact up to rounding after the final division by the
// row sum.
//
// Partial pages need no per-column mask: slots past a page's valid count hold K = V = 0
// (the append and compaction kernels write zeros there), so each scores exactly 0, adds
// nothing to O and 2^-m to the row sum; that amount is tracked per row and taken out.
//
// P is double-buffered in TMEM so a tile's softmax never waits for the previous tile's
// P.V product. TMEM (256 columns): S [0,64), P0 [64,96), P1 [96,128), O' [128,208),
// Q [208,240). Two CTAs fit per SM. The KV sequence can be split across CTAs; partial outputs carry the
// log2-sum-exp, and the split CTA of a query tile that finishes last merges them (a
// separate combine kernel does it where no split counters are given). Every barrier wait is bounded: on
// timeout the CTA records KVC_ERR_TIMEOUT in the error word, drains its own copies and
// MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kvc_attn_common.cuh"

namespace kvc {
namespace tc {
constexpr int kBM = 128;                      // query rows per CTA
constexpr int kBN = 64;                       // KV slots per tile
constexpr int kHD = 64;                       // head dim (one 128-byte swizzle row)
constexpr int kON = kHD + 16;                 // O' columns: O plus the row-sum block
constexpr int kStages = 4;
constexpr int kTileBytes = kBN * kHD * 2;     // 8 KB (K or V tile)
constexpr int kOnesBytes = kBN * kHD * 2;     // 8 KB block of bf16 ones
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;
constexpr int kColS = 0, kColP = 64, kColO = 128, kColQ = 208;   // Q: 32 columns of bf16 pairs
constexpr float kPMax = 256.0f;               // a P above 2^8 moves the row's reference max
constexpr size_t kSmemBytes = 1024 + 2 * kStages * kTileBytes + kOnesBytes + 256;
}  // namespace tc

// Barrier over the softmax warps only (named barrier 1; barrier 0 is __syncthreads).
__device__ __forceinline__ void softmax_warps_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Merge one query row's split partials: O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M)
// (M the largest lse), splits in ascending order. Partials were written by other CTAs of
// this launch and are read through L2: half rows (32 dims) of up to four splits at a time
// are copied (cp.async, every row's copies in flight together) into `stage`, the CTA's
// K/V stage buffers, dead once the last P.V product has completed; with two splits both
// halves come in one round. Each thread reads only its own row, whose eight 16-byte
// chunks per half sit XOR-swizzled by the row so that neighbouring rows use other banks.
__device__ __forceinline__ void merge_split_row(const TcParams& p, uint8_t* stage, int h, int qt, int r, int row) {
  constexpr int kHalf = tc::kHD / 2;                  // dims per pass
  constexpr int kSlot = tc::kBM * kHalf * 4;          // 16 KB: one split's half rows
  constexpr int kSlots = 4;                           // the 64 KB of K/V stages
  constexpr int kKeep = 8;                            // lse values kept in registers
  const long long pi0 = static_cast<long long>(h) * p.splits * p.q_tiles + qt;
  auto lse_at = [&](int s) { return __ldcg(p.part_lse + (pi0 + static_cast<long long>(s) * p.q_tiles) * tc::kBM + r); };
  auto part_at = [&](int s, int half) {
    return p.part_o + ((pi0 + static_cast<long long>(s) * p.q_tiles) * tc::kBM + r) * tc::kHD + half * kHalf;
  };
  // copy a half row into slot j / read chunk c of slot j
  auto stage_in = [&](int j, const float* src) {
    uint8_t* dst = stage + j * kSlot + r * kHalf * 4;
#pragma unroll
    for (int c = 0; c < 8; ++c) cp_async16(dst + ((c ^ (r & 7)) << 4), src + 4 * c);
  };
  auto accumulate = [&](float (&a)[kHalf], int j, float w) {
    const uint8_t* rowp = stage + j * kSlot + r * kHalf * 4;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 f = *reinterpret_cast<const float4*>(rowp + ((c ^ (r & 7)) << 4));
      a[4 * c + 0] = fmaf(w, f.x, a[4 * c + 0]);
      a[4 * c + 1] = fmaf(w, f.y, a[4 * c + 1]);
      a[4 * c + 2] = fmaf(w, f.z, a[4 * c + 2]);
      a[4 * c + 3] = fmaf(w, f.w, a[4 * c + 3]);
    }
  };
  uint4* out = reinterpret_cast<uint4*>(p.out + (static_cast<long long>(row) * p.H + h) * tc::kHD);
  auto store_half = [&](const float (&a)[kHalf], int half, float inv) {
#pragma unroll
    for (int v = 0; v < kHalf / 8; ++v) {
      uint4 q;
      q.x = pack_bf16(a[8 * v + 0] * inv, a[8 * v + 1] * inv);
      q.y = pack_bf16(a[8 * v + 2] * inv, a[8 * v + 3] * inv);
      q.z = pack_bf16(a[8 * v + 4] * inv, a[8 * v + 5] * inv);
      q.w = pack_bf16(a[8 * v + 6] * inv, a[8 * v + 7] * inv);
      out[half * (kHalf / 8) + v] = q;
    }
  };
  const bool one_round = p.splits <= kSlots / 2;
  if (one_round)                                      // both halves of every split, issued first
    for (int s = 0; s < p.splits; ++s) {
      stage_in(2 * s, part_at(s, 0));
      stage_in(2 * s + 1, part_at(s, 1));
    }
  float lr[kKeep];
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < kKeep; ++k) {
    lr[k] = k < p.splits ? lse_at(k) : -INFINITY;
    M = fmaxf(M, lr[k]);
  }
  for (int s = kKeep; s < p.splits; ++s) M = fmaxf(M, lse_at(s));
  float ws = 0.f;
#pragma unroll
  for (int k = 0; k < kKeep; ++k)
    if (k < p.splits) ws += exp2f(lr[k] - M);
  for (int s = kKeep; s < p.splits; ++s) ws += exp2f(lse_at(s) - M);
  const float inv = 1.f / ws;
  auto weight = [&](int s) {
    float l = 0.f;
#pragma unroll
    for (int k = 0; k < kKeep; ++k)
      if (k == s) l = lr[k];
    return exp2f((s < kKeep ? l : lse_at(s)) - M);
  };
  if (one_round) {
    cp_async_wait_all();
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      float a[kHalf];
#pragma unroll
      for (int k = 0; k < kHalf; ++k) a[k] = 0.f;
      for (int s = 0; s < p.splits; ++s) accumulate(a, 2 * s + half, weight(s));
      store_half(a, half, inv);
    }
    return;
  }
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float a[kHalf];
#pragma unroll
    for (int k = 0; k < kHalf; ++k) a[k] = 0.f;
    for (int s0 = 0; s0 < p.splits; s0 += kSlots) {
      const int ns = min(kSlots, p.splits - s0);
      for (int j = 0; j < ns; ++j) stage_in(j, part_at(s0 + j, half));
      cp_async_wait_all();
      for (int j = 0; j < ns; ++j) accumulate(a, j, weight(s0 + j));
    }
    store_half(a, half, inv);
  }
}

template <int P, bool kPerHead>
__global__ void __launch_bounds__(tc::kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const TcParams p) {
  griddep_wait();
  griddep_launch_dependents();
  using namespace tc;
  constexpr int kPPT = kBN / P;               // pages per KV tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* k_s = smem;
  uint8_t* v_s = k_s + kStages * kTileBytes;
  uint8_t* ones_s = v_s + kStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ones_s + kOnesBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStages;
  uint64_t* kv_empty = v_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_full + 2;              // [2] one per P buffer
  uint64_t* pv_done = s_full + 4;             // [2] one per P buffer
  uint64_t* mma_final = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x % p.q_tiles;
  const int rest = blockIdx.x / p.q_tiles;
  const int split = rest % p.splits;
  const int h = rest / p.splits;
  const int tile0 = split * p.tiles_per_split;
  const int tile1 = min(tile0 + p.tiles_per_split, p.total_tiles);
  const int n_tiles = tile1 - tile0;
  // page list and pool rows of this head: shared pages [page][head][slot] or, with
  // per-head page lists, single-head pages of head h's pool region
  const long long hp = kPerHead ? static_cast<long long>(h) * p.head_pages : 0;
  const Entry* ent = kPerHead ? p.entries + hp : p.entries;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 4);                       // the four softmax warps stored Q in TMEM
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  // the constant ones block (every element 1.0, so the swizzle does not matter), made
  // visible to the tensor core's operand reads
  for (int i = threadIdx.x; i < kOnesBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(ones_s)[i] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (n_tiles > 0) {
    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------------------- TMA producer
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
        int last[kStages];
#pragma unroll
        for (int i = 0; i < kStages; ++i) last[i] = -1;
        for (int j = 0; j < n_tiles; ++j) {
          const int st = j % kStages;
          if (j >= kStages && !mbar_wait_bounded(&kv_empty[st], ((j / kStages) - 1) & 1, abort_flag, p.err)) break;
          const int gt = tile0 + j;
          int row[kPPT];
#pragma unroll
          for (int g = 0; g < kPPT; ++g) {
            const int idx = gt * kPPT + g;
            // pages past the list end are read past the end of the pool: TMA fills zeros
            if (kPerHead)
              row[g] = idx < p.n_pages ? static_cast<int>((p.page_base + hp + __ldg(&ent[idx].x)) * P) : p.pool_rows;
            else
              row[g] = idx < p.n_pages ? static_cast<int>(((p.page_base + __ldg(&ent[idx].x)) * p.H + h) * P)
                                       : p.pool_rows;
          }
          mbar_arrive_expect_tx(&k_full[st], kTileBytes);
#pragma unroll
          for (int g = 0; g < kPPT; ++g)
            tma_load_2d(k_s + st * kTileBytes + g * P * 128, &tmap_k, &k_full[st], 0, row[g]);
          mbar_arrive_expect_tx(&v_full[st], kTileBytes);
#pragma unroll
          for (int g = 0; g < kPPT; ++g)
            tma_load_2d(v_s + st * kTileBytes + g * P * 128, &tmap_v, &v_full[st], 0, row[g]);
          last[st] = j;
        }
        // drain: every copy this CTA issued has landed before shared memory is released
#pragma unroll
        for (int i = 0; i < kStages; ++i) {
          if (last[i] >= 0) {
            mbar_wait_drain(&k_full[i], (last[i] / kStages) & 1, p.err);
            mbar_wait_drain(&v_full[i], (last[i] / kStages) & 1, p.err);
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      // the whole warp runs the loop and waits; one elected lane issues the MMAs and
      // commits (the warp stays converged)
      const uint32_t idesc_s = idesc_f16kind(1, kBM, kBN, 0, 0);
      const uint32_t idesc_o = idesc_f16kind(1, kBM, kON, 0, 1);
      const uint32_t tS = tmem + kColS, tP = tmem + kColP, tO = tmem + kColO, tQ = tmem + kColQ;
      const uint32_t k_addr = smem_u32(k_s), v_addr = smem_u32(v_s);
      const uint32_t ones_addr = smem_u32(ones_s);
      const bool leader = elect_one();
      bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(q_full, 0, abort_flag, p.err) &&
                                            mbar_wait_bounded(&k_full[0], 0, abort_flag, p.err));
      if (ok) {
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)
            mma_ts(tS, tQ + kk * 8, sw128_desc(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0);
          mma_commit(s_full);
        }
        __syncwarp();
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        if (j + 1 < n_tiles) {
          const int st1 = (j + 1) % kStages;
          const uint32_t ph1 = ((j + 1) / kStages) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_free, j & 1, abort_flag, p.err) &&
                                           mbar_wait_bounded(&k_full[st1], ph1, abort_flag, p.err)))
            break;
          tc_fence_after();
          const uint32_t kb = k_addr + st1 * kTileBytes;
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk)
              mma_ts(tS, tQ + kk * 8, sw128_desc(kb + kk * 32, 16, 1024), idesc_s, kk > 0);
            mma_commit(s_full);
          }
          __syncwarp();
        }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&p_full[j & 1], (j >> 1) & 1, abort_flag, p.err) &&
                                         mbar_wait_bounded(&v_full[st], ph, abort_flag, p.err)))
          break;
        tc_fence_after();
        const uint32_t vb = v_addr + st * kTileBytes;
        const uint32_t lbo = ones_addr - vb;
        const uint32_t pa = tP + (j & 1) * (kBN / 2);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts(tO, pa + kk * 8, sw128_desc(vb + kk * 2048, lbo, 1024), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&pv_done[j & 1]);
          mma_commit(&kv_empty[st]);
        }
        __syncwarp();
      }
      if (leader) mma_commit(mma_final);
      __syncwarp();
      mbar_wait_drain(mma_final, 0, p.err);
    } else {
      // ------------------------------------------------------------------ softmax warps
      const int wq = warp & 3;                      // TMEM lane quadrant this warp may access
      const int r = wq * 32 + lane;                 // query row within the tile
      const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t tS = tmem + kColS + lane_off, tP = tmem + kColP + lane_off, tO = tmem + kColO + lane_off;
      {
        // this row of Q into TMEM (the A operand of S = Q K^T): 64 bf16 = 32 packed columns
        uint32_t qv[32];
        const int row = qt * kBM + r;
        if (row < p.T) {
          const uint4* src = reinterpret_cast<const uint4*>(p.q + (static_cast<long long>(row) * p.H + h) * kHD);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 w = __ldg(src + v);
            qv[4 * v] = w.x;
            qv[4 * v + 1] = w.y;
            qv[4 * v + 2] = w.z;
            qv[4 * v + 3] = w.w;
          }
        } else {
#pragma unroll
          for (int v = 0; v < 32; ++v) qv[v] = 0u;
        }
        tmem_st32(tmem + kColQ + lane_off, qv);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full);
      }
      const float c = p.scale_log2;
      float m = -INFINITY;       // reference max (log2 domain) of the row
      float masked = 0.f;        // row-sum share of zero-padded slots, rescaled like O'
      bool ok = true;
      // valid-slot counts of the next KV tile's pages, loaded one tile ahead
      int vnext[kPPT];
#pragma unroll
      for (int g = 0; g < kPPT; ++g) {
        const int idx = tile0 * kPPT + g;
        vnext[g] = idx < p.n_pages ? __ldg(&ent[idx].w) : 0;
      }
      // S of the current tile lives in registers; the next tile's S is loaded while this
      // tile's P store is in flight
      uint32_t s[2][32];
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, 0, abort_flag, p.err))) ok = false;
      if (ok) {
        tc_fence_after();
        tmem_ld32(tS + 0, s[0]);
        tmem_ld32(tS + 32, s[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        int n_masked = 0;
#pragma unroll
        for (int g = 0; g < kPPT; ++g) n_masked += P - vnext[g];
        if (j + 1 < n_tiles) {
#pragma unroll
          for (int g = 0; g < kPPT; ++g) {
            const int idx = (tile0 + j + 1) * kPPT + g;
            vnext[g] = idx < p.n_pages ? __ldg(&ent[idx].w) : 0;
          }
        }
        // P = 2^(s*c - m): exponent pairs with one packed FMA, two MUFU ex2, one bf16 pack;
        // a bf16x2 max over the packed P tells whether any exponent exceeded 2^8 (or the
        // reference was unset), in which case the row's reference max moves (slow path)
        uint32_t pb[kBN / 2];
        uint32_t mxb = 0u;
        {
          const uint64_t c2 = pk2(c, c), nm2 = pk2(-m, -m);
#pragma unroll
          for (int i = 0; i < kBN / 2; ++i) {
            float x0, x1;
            up2(fma2_pair(s[(2 * i) / 32][(2 * i) % 32], s[(2 * i + 1) / 32][(2 * i + 1) % 32], c2, nm2), x0, x1);
            pb[i] = bf16x2_trunc(ex2(x0), ex2(x1));
            mxb = max_bf16x2(mxb, pb[i]);
          }
        }
        const bool move = (j == 0) || fmaxf(bf16lo(mxb), bf16hi(mxb)) > kPMax;
        if (__any_sync(0xffffffffu, move)) {
          // slow path (first tile or a new maximum): exact fp32 tile max for the rows that
          // move their reference; rescale O' and the masked share by 2^(m_old - m_new)
          float ta = -INFINITY, tb = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < kBN; cc += 4) {
            ta = max3(ta, __uint_as_float(s[cc / 32][cc % 32]), __uint_as_float(s[cc / 32][cc % 32 + 1]));
            tb = max3(tb, __uint_as_float(s[cc / 32][cc % 32 + 2]), __uint_as_float(s[cc / 32][cc % 32 + 3]));
          }
          const float m_new = move ? fmaxf(ta, tb) * c : m;
          const bool resc = move && j > 0;
          if (__any_sync(0xffffffffu, resc)) {
            // O' row *= f; the previous tile's P.V must have landed
            if (!__all_sync(0xffffffffu,
                            mbar_wait_bounded(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, p.err))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float f = resc ? ex2(m - m_new) : 1.0f;
            masked *= f;
#pragma unroll
            for (int q4 = 0; q4 < kON / 16; ++q4) {
              uint32_t oc[16];
              tmem_ld16(tO + q4 * 16, oc);
              tmem_ld_wait();
#pragma unroll
              for (int d = 0; d < 16; ++d) oc[d] = __float_as_uint(__uint_as_float(oc[d]) * f);
              tmem_st16(tO + q4 * 16, oc);
            }
          }
          m = m_new;
          const uint64_t c2 = pk2(c, c), nm2 = pk2(-m, -m);
#pragma unroll
          for (int i = 0; i < kBN / 2; ++i) {
            float x0, x1;
            up2(fma2_pair(s[(2 * i) / 32][(2 * i) % 32], s[(2 * i + 1) / 32][(2 * i + 1) % 32], c2, nm2), x0, x1);
            pb[i] = bf16x2_trunc(ex2(x0), ex2(x1));
          }
        }
        if (n_masked) {
          // each zero-padded slot scored 0 and contributed exactly bf16(2^-m) to the sum
          masked += static_cast<float>(n_masked) * bf16lo(bf16x2_trunc(ex2(-m), 0.f));
        }
        // P buffer j & 1 was last read by the P.V product of tile j - 2
        if (j >= 2) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(&pv_done[j & 1], ((j - 2) >> 1) & 1, abort_flag, p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st32(tP + (j & 1) * (kBN / 2), pb);
        // tcgen05.ld/st are .sync.aligned: every branch around them is kept warp-uniform
        const bool more = j + 1 < n_tiles;
        if (more) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, (j + 1) & 1, abort_flag, p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_ld32(tS + 0, s[0]);
          tmem_ld32(tS + 32, s[1]);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[j & 1]);
        if (more) {
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
      }
      const int jl = n_tiles - 1;
      if (__all_sync(0xffffffffu, ok && mbar_wait_bounded(&pv_done[jl & 1], (jl >> 1) & 1, abort_flag, p.err))) {
        tc_fence_after();
        uint32_t o0[32], o1[32], ls[16];
        tmem_ld32(tO, o0);
        tmem_ld32(tO + 32, o1);
        tmem_ld16(tO + 64, ls);
        tmem_ld_wait();
        const float l = __uint_as_float(ls[0]) - masked;
        const float inv = 1.f / l;
        const int row = qt * kBM + r;
        if (p.splits == 1) {
          if (row < p.T) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<long long>(row) * p.H + h) * kHD);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(o0[8 * v + 0]) * inv, __uint_as_float(o0[8 * v + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(o0[8 * v + 2]) * inv, __uint_as_float(o0[8 * v + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(o0[8 * v + 4]) * inv, __uint_as_float(o0[8 * v + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(o0[8 * v + 6]) * inv, __uint_as_float(o0[8 * v + 7]) * inv);
              dst[v] = w;
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(o1[8 * v + 0]) * inv, __uint_as_float(o1[8 * v + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(o1[8 * v + 2]) * inv, __uint_as_float(o1[8 * v + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(o1[8 * v + 4]) * inv, __uint_as_float(o1[8 * v + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(o1[8 * v + 6]) * inv, __uint_as_float(o1[8 * v + 7]) * inv);
              dst[4 + v] = w;
            }
          }
        } else {
          const long long pi = (static_cast<long long>(h) * p.splits + split) * p.q_tiles + qt;
          float4* dst = reinterpret_cast<float4*>(p.part_o + (pi * kBM + r) * kHD);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o0[4 * v + 0]) * inv, __uint_as_float(o0[4 * v + 1]) * inv,
                                 __uint_as_float(o0[4 * v + 2]) * inv, __uint_as_float(o0[4 * v + 3]) * inv);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[8 + v] = make_float4(__uint_as_float(o1[4 * v + 0]) * inv, __uint_as_float(o1[4 * v + 1]) * inv,
                                     __uint_as_float(o1[4 * v + 2]) * inv, __uint_as_float(o1[4 * v + 3]) * inv);
          p.part_lse[pi * kBM + r] = m + __log2f(l);
        }
      }
      if (p.splits > 1 && p.split_cnt) {
        // the split CTA that finishes a (query tile, head) last merges every split's
        // partial (threadfence-then-count: each partial is visible before its count)
        __shared__ int s_last;
        __threadfence();
        softmax_warps_sync();
        if (warp == 2 && lane == 0) s_last = atomicAdd(&p.split_cnt[h * p.q_tiles + qt], 1) == p.splits - 1;
        softmax_warps_sync();
        if (s_last) {
          __threadfence();
          const int row = qt * kBM + r;
          if (row < p.T) merge_split_row(p, k_s, h, qt, r, row);
          if (warp == 2 && lane == 0) p.split_cnt[h * p.q_tiles + qt] = 0;   // ready for the next launch
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge split partials: O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M). One warp per
// (row, head): lane s (and s + 32) loads split s's log-sum-exp, so the maximum and the
// weights take one round of loads and warp shuffles; then each lane accumulates two of
// the 64 dims over the splits, four partial rows in flight at a time (up to 64 splits).
__global__ void combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                               __nv_bfloat16* __restrict__ out, int T, int H, int q_tiles, int splits) {
  griddep_wait();
  griddep_launch_dependents();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= T * H) return;
  const int t = gw / H, h = gw % H;
  const int qt = t / tc::kBM, r = t % tc::kBM;
  const long long pi0 = static_cast<long long>(h) * splits * q_tiles + qt;
  auto row_of = [&](int s) { return (pi0 + static_cast<long long>(s) * q_tiles) * tc::kBM + r; };
  const float l0 = lane < splits ? __ldg(&part_lse[row_of(lane)]) : -INFINITY;
  const float l1 = lane + 32 < splits ? __ldg(&part_lse[row_of(lane + 32)]) : -INFINITY;
  float M = fmaxf(l0, l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = lane < splits ? exp2f(l0 - M) : 0.f;
  const float w1 = lane + 32 < splits ? exp2f(l1 - M) : 0.f;
  float ws = w0 + w1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
  for (int s = 0; s < splits; ++s) {
    const float w = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
    const float2 o = __ldg(reinterpret_cast<const float2*>(part_o + row_of(s) * tc::kHD) + lane);
    a0 = fmaf(w, o.x, a0);
    a1 = fmaf(w, o.y, a1);
  }
  const float inv = 1.f / ws;
  reinterpret_cast<__nv_bfloat162*>(out + (static_cast<long long>(t) * H + h) * tc::kHD)[lane] =
      __floats2bfloat162_rn(a0 * inv, a1 * inv);
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool encode_pool_tmap(CUtensorMap* map, void* base, size_t rows, int D, int P, int elem_bytes, bool swizzle128) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * elem_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(P)};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt =
      elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(map, dt, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool encode_q_tmap(CUtensorMap* map, const void* q, int T, int H) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(tc::kHD), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(tc::kHD) * 2, static_cast<cuuint64_t>(H) * tc::kHD * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(tc::kHD), 1, static_cast<cuuint32_t>(tc::kBM)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Pick the number of KV splits. Cost of a split count, in units of one KV tile of a CTA
// that shares its SM: waves x (fixed cost of a CTA + tiles per CTA), where a CTA alone on
// its SM (at most one per SM in the whole launch) runs a tile in about 0.84 of the time,
// plus a cost per split (the partials written and merged). Fixed cost and split cost:
// 8 and 2 tiles for the bf16 kernel, whose last split CTA merges (measured on 24-, 272- and
// 1,146-tile caches); 4 and 0.25 (+ 0.5 for the combine launch) for the FP8 kernel, one CTA
// per SM. Among counts within 1% of the best cost the fewest splits win.
int choose_splits(int units, int tiles, int slots, bool fp8) {
  const double cta_cost = fp8 ? 4.0 : 8.0;
  const int max_s = tiles < 64 ? tiles : 64;
  double cost[65];
  double best_cost = 1e30;
  for (int s = 1; s <= max_s; ++s) {
    cost[s] = 1e30;
    const int tps = (tiles + s - 1) / s;
    if ((tiles + tps - 1) / tps != s) continue;        // the same as a smaller split count
    const long long ctas = static_cast<long long>(units) * s;
    const long long waves = (ctas + slots - 1) / slots;
    const double per_tile = !fp8 && 2 * ctas <= slots ? 0.84 : 1.0;
    const double split_cost = s == 1 ? 0.0 : fp8 ? 0.5 + 0.25 * s : 2.0 * s;
    cost[s] = static_cast<double>(waves) * (cta_cost + tps) * per_tile + split_cost;
    if (cost[s] < best_cost) best_cost = cost[s];
  }
  for (int s = 1; s <= max_s; ++s)
    if (cost[s] <= best_cost * 1.01) return s;
  return 1;
}

cudaError_t launch_attn_tc(cudaStream_t s, const TcAttnArgs& a, int* splits_used, int* launched) {
  if (launched) *launched = 0;
  if (a.P != 16 || (a.fp8 && a.head_pages)) return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!a.fp8 && !attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(tc::kSmemBytes));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(tc::kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  CUtensorMap tq;
  if (!encode_q_tmap(&tq, a.q, a.T, a.H)) return cudaErrorInvalidValue;
  const int q_tiles = (a.T + tc::kBM - 1) / tc::kBM;
  const int total_tiles = (a.n_pages * a.P + tc::kBN - 1) / tc::kBN;
  // a CTA of the bf16 kernel takes one query tile (two CTAs per SM); a CTA of the FP8
  // kernel takes two (one CTA per SM)
  const int units = a.fp8 ? ((q_tiles + 1) / 2) * a.H : q_tiles * a.H;
  const int slots = a.fp8 ? a.sm_count : 2 * a.sm_count;
  const int part_units = q_tiles * a.H;       // 128-row partial tiles per split
  int splits = a.splits > 0 ? a.splits : choose_splits(units, total_tiles, slots, a.fp8);
  if (splits > total_tiles) splits = total_tiles;
  if (splits > 64) splits = 64;                  // the combine takes up to 64 partials per row
  int tps = (total_tiles + splits - 1) / splits;
  splits = (total_tiles + tps - 1) / tps;
  if (splits > 1 && static_cast<size_t>(part_units) * splits > a.part_rows) {
    // not enough partial scratch: fall back to as many splits as fit
    splits = static_cast<int>(a.part_rows / part_units);
    if (splits < 1) splits = 1;
    tps = (total_tiles + splits - 1) / splits;
    splits = (total_tiles + tps - 1) / tps;
  }
  TcParams prm;
  prm.q = static_cast<const __nv_bfloat16*>(a.q);
  prm.k_scale = a.k_scale;
  prm.v_scale = a.v_scale;
  prm.entries = a.entries;
  prm.n_pages = a.n_pages;
  prm.T = a.T;
  prm.H = a.H;
  prm.q_tiles = q_tiles;
  prm.splits = splits;
  prm.tiles_per_split = tps;
  prm.total_tiles = total_tiles;
  prm.page_base = a.page_base;
  prm.pool_rows = static_cast<int>(a.pool_rows);
  prm.scale_log2 = static_cast<float>(static_cast<double>(a.softmax_scale) * 1.4426950408889634);
  prm.out = static_cast<__nv_bfloat16*>(a.o);
  prm.part_o = a.part_o;
  prm.part_lse = a.part_lse;
  prm.err = a.err;
  prm.head_pages = a.head_pages;
  prm.k_chan = a.fp8 ? a.k_chan : nullptr;
  prm.v_tok = a.fp8 ? a.v_tok : nullptr;
  // the last split CTA merges when a merge is one copy round per half row (up to four
  // splits); with more, a separate combine launch is faster (measured at 9 splits)
  prm.split_cnt = a.fp8 || splits > 4 ? nullptr : a.split_cnt;
  const int grid = units * splits;
  cudaError_t e;
  if (a.fp8) {
    e = launch_attn_fp8_kernel(s, tq, *a.tmap_k, *a.tmap_v, prm, grid);
  } else {
    if (a.head_pages)
      e = launch_pdl(attn_tc_kernel<16, true>, dim3(grid), dim3(tc::kThreads), tc::kSmemBytes, s, tq, *a.tmap_k,
                     *a.tmap_v, prm);
    else
      e = launch_pdl(attn_tc_kernel<16, false>, dim3(grid), dim3(tc::kThreads), tc::kSmemBytes, s, tq, *a.tmap_k,
                     *a.tmap_v, prm);
  }
  if (e != cudaSuccess) return e;
  if (launched) *launched = 1;
  if (splits > 1 && !prm.split_cnt) {
    const long long warps = static_cast<long long>(a.T) * a.H;
    const int threads = 256;
    e = launch_pdl(combine_kernel, dim3(static_cast<int>((warps * 32 + threads - 1) / threads)), dim3(threads), 0, s,
                   a.part_o, a.part_lse, static_cast<__nv_bfloat16*>(a.o), a.T, a.H, q_tiles, splits);
    if (launched) *launched = 2;
  }
  if (splits_used) *splits_used = splits;
  return e;
}

}  // namespace kvc
