// kvc_attn_tc.cu -- frame attention over the paged bf16 cache on sm_100a tensor cores.
//
// Computes O[i, h] = sum_j softmax_j(scale * q_i . k_j) v_j for the T queries of the new
// frame over every valid slot of the layer's page list ("How GCTStream ...",
// Frame-by-Frame Causal Processing; "InfiniteVGGT" explainer, Causal Attention) without
// materialising the score matrix, as a flash-attention pipeline built for Blackwell:
//
//   warp 0 (one lane)   TMA producer: the CTA's 128x64 query tile once, then per KV tile
//                       the 128/P pages of K and of V, each page-head block one 2-D box
//                       into a 128-byte-swizzled stage (ring of kStages stages).
//   warp 1 (one lane)   MMA issuer: S = Q K^T (tcgen05.mma kind::f16, M=128, N=128,
//                       4 K-steps of 16) into TMEM; O += P V with P read from TMEM
//                       (M=128, N=64, 8 K-steps) and V as an MN-major operand.
//   warps 2..9          softmax: two warps per TMEM lane quadrant, thread = query row =
//                       TMEM lane, each warp of a pair owning 64 of the tile's 128
//                       columns; S half-row to registers (tcgen05.ld), row max
//                       exchanged with the partner warp through shared memory, online
//                       max with lazy
//                       rescaling (the running reference max only moves when the tile max
//                       exceeds it by 2^8, which keeps the result exact after the final
//                       normalisation), P = 2^(s - m) as bf16 back into TMEM (tcgen05.st),
//                       the warp's 32 O columns rescaled in TMEM when the max moves.
//
// Partial pages need no per-column mask: slots past a page's valid count hold K = V = 0
// (the append and compaction kernels write zeros there, and pages past the end of the
// list are read out of bounds so TMA fills zeros), so each scores exactly 0, adds nothing
// to O and exactly 2^-m to the row sum, which is subtracted once per tile.
//
// TMEM (256 columns): S [0,128), P [128,192) (bf16 pairs), O [192,256). Two CTAs fit per
// SM (TMEM 2 x 256 columns, shared memory 2 x ~85 KB, 96 registers per thread), which puts
// four softmax warps on every SM sub-partition and lets one CTA's MMAs overlap the
// other's softmax. The KV sequence can be split across CTAs; partial outputs carry the
// log2-sum-exp and a combine kernel merges them. Every barrier wait is bounded: on
// timeout the CTA records KVC_ERR_TIMEOUT in the error word, drains its own copies and
// MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {
namespace tc {
constexpr int kBM = 128;                      // query rows per CTA
constexpr int kBN = 128;                      // KV slots per tile
constexpr int kHD = 64;                       // head dim (one 128-byte swizzle row)
constexpr int kStages = 2;
constexpr int kTileBytes = kBN * kHD * 2;     // 16 KB
constexpr int kQBytes = kBM * kHD * 2;        // 16 KB
constexpr int kThreads = 320;                 // producer, MMA, 8 softmax warps
constexpr int kTmemCols = 256;
constexpr int kColS = 0, kColP = 128, kColO = 192;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kPolyCols = 0;                  // of each warp's 64 columns, exponentiated on the FMA pipe
                                              // (0: measured fastest; the MUFU is not the limit)                 // of each warp's 64 columns, exponentiated on the FMA pipe
constexpr size_t kSmemBytes = 1024 + kQBytes + 2 * kStages * kTileBytes + 256 + 2 * 2 * kBM * 4;
}  // namespace tc

struct TcParams {
  const Entry* entries;
  int n_pages, T, H;
  int q_tiles, splits, tiles_per_split, total_tiles;
  long long page_base;          // layer * pool_pages: first pool page of the layer
  int pool_rows;                // rows of the pool tensor maps (a row index past the end reads zeros)
  float scale_log2;
  __nv_bfloat16* out;
  float* part_o;
  float* part_lse;
  int* err;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 3-input max (sm_100a)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe for x <= 8 (lazy rescaling bounds the exponent): x is split as
// n + f with n = round(x) (adding and subtracting 1.5 * 2^23) and |f| <= 1/2; 2^f comes
// from a degree-3 polynomial whose coefficients were fitted for this kernel (relative
// minimax on [-1/2, 1/2], max relative error 7.6e-5, far below the 2^-9 rounding of P to
// bf16); 2^n is applied by adding n to the exponent field. Inputs below -125 are clamped
// so the result stays a normal number. Used for the last kPolyCols columns of a half.
__device__ __forceinline__ float exp2_poly(float x) {
  constexpr float kC0 = 0.9999281764030457f, kC1 = 0.6932609677314758f, kC2 = 0.2426096349954605f,
                  kC3 = 0.055170949548482895f, kMagic = 12582912.0f;
  x = fmaxf(x, -125.f);
  const float t = x + kMagic;
  const float n = t - kMagic;
  const float f = x - n;
  float q = fmaf(kC3, f, kC2);
  q = fmaf(q, f, kC1);
  q = fmaf(q, f, kC0);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

// Wait without the abort shortcut, used only to drain a CTA's own in-flight work.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, int* err) {
  volatile int never = 0;
  mbar_wait_bounded(bar, parity, &never, err);
}

template <int P>
__global__ void __launch_bounds__(tc::kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const TcParams p) {
  using namespace tc;
  constexpr int kPPT = kBN / P;               // pages per KV tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;
  uint8_t* k_s = smem + kQBytes;
  uint8_t* v_s = k_s + kStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(v_s + kStages * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStages;
  uint64_t* kv_empty = v_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = s_full + 3;
  uint64_t* mma_final = s_full + 4;
  uint64_t* xchg = s_full + 5;                // [4] one per TMEM lane quadrant (softmax warp pair)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xchg + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(bars + 32);   // [2 parity][2 halves][128 rows] row values

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x % p.q_tiles;
  const int rest = blockIdx.x / p.q_tiles;
  const int split = rest % p.splits;
  const int h = rest / p.splits;
  const int tile0 = split * p.tiles_per_split;
  const int tile1 = min(tile0 + p.tiles_per_split, p.total_tiles);
  const int n_tiles = tile1 - tile0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(p_full, 8);
    for (int i = 0; i < 4; ++i) mbar_init(&xchg[i], 64);
    mbar_init(pv_done, 1);
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
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
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
        mbar_arrive_expect_tx(q_full, kQBytes);
        tma_load_3d(q_s, &tmap_q, q_full, 0, h, qt * kBM);
        int last[kStages];
#pragma unroll
        for (int i = 0; i < kStages; ++i) last[i] = -1;
        for (int j = 0; j < n_tiles; ++j) {
          const int st = j % kStages;
          if (j >= kStages && !mbar_wait_bounded(&kv_empty[st], ((j / kStages) - 1) & 1, abort_flag, p.err)) break;
          const int gt = tile0 + j;
          uint8_t* kd = k_s + st * kTileBytes;
          uint8_t* vd = v_s + st * kTileBytes;
          mbar_arrive_expect_tx(&k_full[st], kTileBytes);
#pragma unroll
          for (int g = 0; g < kPPT; ++g) {
            const int idx = gt * kPPT + g;
            // pages past the list end are read past the end of the pool: TMA fills zeros
            const int row = idx < p.n_pages ? static_cast<int>(((p.page_base + __ldg(&p.entries[idx].x)) * p.H + h) * P)
                                            : p.pool_rows;
            tma_load_2d(kd + g * P * 128, &tmap_k, &k_full[st], 0, row);
          }
          mbar_arrive_expect_tx(&v_full[st], kTileBytes);
#pragma unroll
          for (int g = 0; g < kPPT; ++g) {
            const int idx = gt * kPPT + g;
            const int row = idx < p.n_pages ? static_cast<int>(((p.page_base + __ldg(&p.entries[idx].x)) * p.H + h) * P)
                                            : p.pool_rows;
            tma_load_2d(vd + g * P * 128, &tmap_v, &v_full[st], 0, row);
          }
          last[st] = j;
        }
        // drain: every copy this CTA issued has landed before shared memory is released
        mbar_wait_drain(q_full, 0, p.err);
#pragma unroll
        for (int i = 0; i < kStages; ++i) {
          if (last[i] >= 0) {
            mbar_wait_drain(&k_full[i], (last[i] / kStages) & 1, p.err);
            mbar_wait_drain(&v_full[i], (last[i] / kStages) & 1, p.err);
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------------------- MMA issuer
        const uint32_t idesc_s = idesc_f16kind(1, kBM, kBN, 0, 0);
        const uint32_t idesc_o = idesc_f16kind(1, kBM, kHD, 0, 1);
        const uint32_t tS = tmem + kColS, tP = tmem + kColP, tO = tmem + kColO;
        const uint32_t q_addr = smem_u32(q_s), k_addr = smem_u32(k_s), v_addr = smem_u32(v_s);
        bool ok = mbar_wait_bounded(q_full, 0, abort_flag, p.err) &&
                  mbar_wait_bounded(&k_full[0], 0, abort_flag, p.err);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)
            mma_ss(tS, sw128_desc(q_addr + kk * 32, 16, 1024), sw128_desc(k_addr + kk * 32, 16, 1024), idesc_s,
                   kk > 0);
          mma_commit(s_full);
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int st = j % kStages;
          const uint32_t ph = (j / kStages) & 1;
          if (j + 1 < n_tiles) {
            const int st1 = (j + 1) % kStages;
            const uint32_t ph1 = ((j + 1) / kStages) & 1;
            if (!mbar_wait_bounded(s_free, j & 1, abort_flag, p.err)) break;
            if (!mbar_wait_bounded(&k_full[st1], ph1, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t kb = k_addr + st1 * kTileBytes;
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk)
              mma_ss(tS, sw128_desc(q_addr + kk * 32, 16, 1024), sw128_desc(kb + kk * 32, 16, 1024), idesc_s,
                     kk > 0);
            mma_commit(s_full);
          }
          if (!mbar_wait_bounded(p_full, j & 1, abort_flag, p.err)) break;
          if (!mbar_wait_bounded(&v_full[st], ph, abort_flag, p.err)) break;
          tc_fence_after();
          const uint32_t vb = v_addr + st * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts(tO, tP + kk * 8, sw128_desc(vb + kk * 2048, 8192, 1024), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pv_done);
          mma_commit(&kv_empty[st]);
        }
        // drain: all MMAs of this CTA complete before TMEM is released
        mma_commit(mma_final);
        mbar_wait_drain(mma_final, 0, p.err);
      }
    } else {
      // ------------------------------------------------------------------ softmax warps
      // Eight warps. Warp w may only access TMEM lane quadrant w % 4 (its 32 query rows);
      // the two warps sharing a quadrant split each 128-column S tile into halves of 64
      // and exchange per-row maxima through shared memory (mbarrier xchg[quadrant]).
      constexpr int kHalf = kBN / 2;
      constexpr int kPPH = kPPT / 2;               // pages per column half
      const int wq = warp & 3;
      const int hf = (warp - 2) >> 2;
      const int r = wq * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t tS = tmem + kColS + hf * kHalf + lane_off;
      const uint32_t tP = tmem + kColP + hf * (kHalf / 2) + lane_off;
      const uint32_t tO = tmem + kColO + hf * (kHD / 2) + lane_off;
      const float c = p.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      // valid-slot counts of this half's pages of the next KV tile, loaded one tile ahead
      int vnext[kPPH];
#pragma unroll
      for (int g = 0; g < kPPH; ++g) {
        const int idx = tile0 * kPPT + hf * kPPH + g;
        vnext[g] = idx < p.n_pages ? __ldg(&p.entries[idx].w) : 0;
      }
      for (int j = 0; j < n_tiles; ++j) {
        // invalid slots hold K = V = 0, so they score 0 and add exactly 2^-m to the row
        // sum and nothing to O: count them and take them out of the sum below
        int n_masked = 0;
#pragma unroll
        for (int g = 0; g < kPPH; ++g) n_masked += P - vnext[g];
        if (j + 1 < n_tiles) {
#pragma unroll
          for (int g = 0; g < kPPH; ++g) {
            const int idx = (tile0 + j + 1) * kPPT + hf * kPPH + g;
            vnext[g] = idx < p.n_pages ? __ldg(&p.entries[idx].w) : 0;
          }
        }
        // tcgen05.ld/st are .sync.aligned: every branch around them is kept warp-uniform
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, j & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[2][32];
        tmem_ld32(tS + 0, s[0]);
        tmem_ld32(tS + 32, s[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < kHalf; cc += 8) {
          mxa = max3(mxa, __uint_as_float(s[cc / 32][cc % 32 + 0]), __uint_as_float(s[cc / 32][cc % 32 + 1]));
          mxb = max3(mxb, __uint_as_float(s[cc / 32][cc % 32 + 2]), __uint_as_float(s[cc / 32][cc % 32 + 3]));
          mxc = max3(mxc, __uint_as_float(s[cc / 32][cc % 32 + 4]), __uint_as_float(s[cc / 32][cc % 32 + 5]));
          mxd = max3(mxd, __uint_as_float(s[cc / 32][cc % 32 + 6]), __uint_as_float(s[cc / 32][cc % 32 + 7]));
        }
        float mx = fmaxf(fmaxf(mxa, mxb), fmaxf(mxc, mxd));
        // row max of the whole tile: swap halves with the partner warp
        red[((j & 1) * 2 + hf) * kBM + r] = mx;
        mbar_arrive(&xchg[wq]);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&xchg[wq], j & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        mx = fmaxf(mx, red[((j & 1) * 2 + (1 - hf)) * kBM + r]);
        const float mx_s = mx * c;
        float m_new = m;
        bool rescale = false;
        if (j == 0) {
          m_new = mx_s;
        } else if (mx_s > m + kRescaleLog2) {
          m_new = mx_s;
          rescale = true;
        }
        // P = 2^(s*c - m) in scalar fp32: the first kHalf - kPolyCols columns on the MUFU
        // ex2, the last kPolyCols with the FMA-pipe polynomial; each pair is summed into
        // four independent accumulators and packed to bf16 right away.
        const float nm = -m_new;
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
        uint32_t pk[kHalf / 2];
#pragma unroll
        for (int cc = 0; cc < kHalf; cc += 2) {
          float x0 = fmaf(__uint_as_float(s[cc / 32][cc % 32]), c, nm);
          float x1 = fmaf(__uint_as_float(s[cc / 32][cc % 32 + 1]), c, nm);
          if (cc >= kHalf - kPolyCols) {
            x0 = exp2_poly(x0);
            x1 = exp2_poly(x1);
          } else {
            x0 = ex2(x0);
            x1 = ex2(x1);
          }
          if ((cc / 2) & 1) {
            acc2 += x0;
            acc3 += x1;
          } else {
            acc0 += x0;
            acc1 += x1;
          }
          pk[cc / 2] = pack_bf16(x0, x1);
        }
        float rs = (acc0 + acc1) + (acc2 + acc3);
        if (n_masked) rs -= static_cast<float>(n_masked) * ex2(nm);
        if (j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, (j - 1) & 1, abort_flag, p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, rescale)) {
          // this warp's 32 O columns *= 2^(m_old - m_new); rows that keep their reference
          // max scale by 1 (the branch is warp-uniform)
          const float corr = rescale ? ex2(m - m_new) : 1.0f;
          l *= corr;
#pragma unroll
          for (int q4 = 0; q4 < kHD / 32; ++q4) {
            uint32_t oc[16];
            tmem_ld16(tO + q4 * 16, oc);
            tmem_ld_wait();
#pragma unroll
            for (int d = 0; d < 16; ++d) oc[d] = __float_as_uint(__uint_as_float(oc[d]) * corr);
            tmem_st16(tO + q4 * 16, oc);
          }
        }
        m = m_new;
        l += rs;
        tmem_st32(tP, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      // row sum of the two halves, then the epilogue writes this warp's 32 columns
      if (ok) {
        red[((n_tiles & 1) * 2 + hf) * kBM + r] = l;
        mbar_arrive(&xchg[wq]);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&xchg[wq], n_tiles & 1, abort_flag, p.err));
        if (ok) l += red[((n_tiles & 1) * 2 + (1 - hf)) * kBM + r];
      }
      if (__all_sync(0xffffffffu, ok && mbar_wait_bounded(pv_done, (n_tiles - 1) & 1, abort_flag, p.err))) {
        tc_fence_after();
        uint32_t o0[32];
        tmem_ld32(tO, o0);
        tmem_ld_wait();
        const float inv = 1.f / l;
        const int row = qt * kBM + r;
        if (p.splits == 1) {
          if (row < p.T) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<long long>(row) * p.H + h) * kHD + hf * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(o0[8 * v + 0]) * inv, __uint_as_float(o0[8 * v + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(o0[8 * v + 2]) * inv, __uint_as_float(o0[8 * v + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(o0[8 * v + 4]) * inv, __uint_as_float(o0[8 * v + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(o0[8 * v + 6]) * inv, __uint_as_float(o0[8 * v + 7]) * inv);
              dst[v] = w;
            }
          }
        } else {
          const long long pi = (static_cast<long long>(h) * p.splits + split) * p.q_tiles + qt;
          float4* dst = reinterpret_cast<float4*>(p.part_o + (pi * kBM + r) * kHD + hf * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o0[4 * v + 0]) * inv, __uint_as_float(o0[4 * v + 1]) * inv,
                                 __uint_as_float(o0[4 * v + 2]) * inv, __uint_as_float(o0[4 * v + 3]) * inv);
          if (hf == 0) p.part_lse[pi * kBM + r] = m + __log2f(l);
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
// (row, head); lane covers two of the 64 dims.
__global__ void combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                               __nv_bfloat16* __restrict__ out, int T, int H, int q_tiles, int splits) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= T * H) return;
  const int t = gw / H, h = gw % H;
  const int qt = t / tc::kBM, r = t % tc::kBM;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) {
    const long long pi = (static_cast<long long>(h) * splits + s) * q_tiles + qt;
    M = fmaxf(M, part_lse[pi * tc::kBM + r]);
  }
  float a0 = 0.f, a1 = 0.f, ws = 0.f;
  for (int s = 0; s < splits; ++s) {
    const long long pi = (static_cast<long long>(h) * splits + s) * q_tiles + qt;
    const float w = exp2f(part_lse[pi * tc::kBM + r] - M);
    const float2 o = reinterpret_cast<const float2*>(part_o + (pi * tc::kBM + r) * tc::kHD)[lane];
    a0 = fmaf(w, o.x, a0);
    a1 = fmaf(w, o.y, a1);
    ws += w;
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

// Pick the number of KV splits: fewest waves x tiles-per-CTA over two resident CTAs per SM.
int choose_splits(int units, int tiles, int slots) {
  int best = 1;
  double best_cost = 1e30;
  const int max_s = tiles < 64 ? tiles : 64;
  for (int s = 1; s <= max_s; ++s) {
    const int tps = (tiles + s - 1) / s;
    const int s_eff = (tiles + tps - 1) / tps;
    const long long ctas = static_cast<long long>(units) * s_eff;
    const long long waves = (ctas + slots - 1) / slots;
    // combine traffic grows with the split count: charge it lightly
    const double cost = static_cast<double>(waves) * tps * (1.0 + 0.004 * s_eff);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s_eff;
    }
  }
  return best;
}

cudaError_t launch_attn_tc(cudaStream_t s, const TcAttnArgs& a, int* splits_used, int* launched) {
  if (launched) *launched = 0;
  if (a.P != 16 || a.fp8) return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(tc::kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  CUtensorMap tq;
  if (!encode_q_tmap(&tq, a.q, a.T, a.H)) return cudaErrorInvalidValue;
  const int q_tiles = (a.T + tc::kBM - 1) / tc::kBM;
  const int total_tiles = (a.n_pages * a.P + tc::kBN - 1) / tc::kBN;
  const int units = q_tiles * a.H;
  int splits = a.splits > 0 ? a.splits : choose_splits(units, total_tiles, 2 * a.sm_count);
  if (splits > total_tiles) splits = total_tiles;
  int tps = (total_tiles + splits - 1) / splits;
  splits = (total_tiles + tps - 1) / tps;
  if (splits > 1 && static_cast<size_t>(units) * splits > a.part_rows) {
    // not enough partial scratch: fall back to as many splits as fit
    splits = static_cast<int>(a.part_rows / units);
    if (splits < 1) splits = 1;
    tps = (total_tiles + splits - 1) / splits;
    splits = (total_tiles + tps - 1) / tps;
  }
  TcParams prm;
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
  const int grid = units * splits;
  attn_tc_kernel<16><<<grid, tc::kThreads, tc::kSmemBytes, s>>>(tq, *a.tmap_k, *a.tmap_v, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (launched) *launched = 1;
  if (splits > 1) {
    const long long warps = static_cast<long long>(a.T) * a.H;
    const int threads = 256;
    combine_kernel<<<static_cast<int>((warps * 32 + threads - 1) / threads), threads, 0, s>>>(
        a.part_o, a.part_lse, static_cast<__nv_bfloat16*>(a.o), a.T, a.H, q_tiles, splits);
    e = cudaGetLastError();
    if (launched) *launched = 2;
  }
  if (splits_used) *splits_used = splits;
  return e;
}

}  // namespace kvc
