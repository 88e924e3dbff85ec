// kvc_attn_fp8.cu -- frame attention over the paged FP8 E4M3 cache on sm_100a tensor cores.
//
// Same attention as kvc_attn_tc.cu ("How GCTStream ...", Frame-by-Frame Causal
// Processing) over K/V stored as E4M3 codes with one absmax scale per (page, head)
// ("XStreamVGGT" abstract: KV cache quantisation). The tensor cores multiply f16
// operands (kind::f16 needs both operands of one type), so each KV tile is widened in
// shared memory right after it lands. One CTA per SM owns two 128-row query tiles of one
// head, so every converted KV tile serves 256 query rows:
//
//   warps 0, 10         converters, one half of each 64-slot KV tile (2 of its 4 pages)
//                       each: lane 0 loads the half's K and V code blocks (1 KB per page
//                       and tensor) by TMA into the warp's own three-stage ring; the warp
//                       turns every code pair into an f16 pair with the hardware E4M3
//                       conversion (exact) and writes it as a 128-byte-swizzled MMA operand.
//                       K codes stay unscaled; each V pair is multiplied by the page's V
//                       scale over the CTA's largest V scale of the head.
//   warps 1, 11         MMA issuers, one per query tile (so the two tiles' pipelines do not
//                       wait on each other; the warp waits, one elected lane issues): per
//                       KV tile S = Q K^T (M=128, N=64, A = Q read from TMEM) and
//                       O' += P [V | 1] (M=128, N=80), f16 inputs, fp32 accumulation in
//                       TMEM (512 columns: 256 per query tile).
//   warps 2..5, 6..9    softmax of query tile 0 and 1: each thread first widens its row of
//                       Q bf16 -> f16 into TMEM; then as in the bf16 kernel (one thread per
//                       row, 64 columns per tile, lazy rescaling, row sum from the ones
//                       column), with P packed as f16. The K scale of a page multiplies the
//                       logit factor of its 16 columns, so Q K^T runs on exact decoded codes.
//
// The epilogue multiplies by the V reference scale. Rounding V times s_page / s_ref to f16
// is the only extra rounding of an operand (relative 2^-11). The query row is held in f16
// after an exact power-of-two scaling into f16's range (the row's logit factor carries the
// inverse), so every finite bf16 query is taken. Slots past a page's valid count score
// -inf in the tiles that have them, so they take no weight. Every barrier wait is bounded.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "kvc_attn_common.cuh"

namespace kvc {
namespace tc8 {
constexpr int kBM = 128, kBN = 64, kHD = 64, kON = kHD + 16;
constexpr int kGroups = 2;                    // query tiles per CTA
constexpr int kCodeStages = 3;                // code staging ring of each converter
constexpr int kStages = 4;                    // converted f16 operand ring
constexpr int kHalfCodeBytes = (kBN / 2) * kHD;   // 2 KB: a converter's half tile of one tensor
constexpr int kConvBytes = kBN * kHD * 2;     // 8 KB f16 tile
constexpr int kOnesBytes = kBN * kHD * 2;
constexpr int kThreads = 384;                 // 12 warps
constexpr int kConvThreads = 64;              // warps 0 and 10
constexpr int kTmemCols = 512;
constexpr int kGroupCols = 256;               // TMEM columns per query tile
constexpr int kColS = 0, kColP = 64, kColO = 128, kColQ = 208;   // per query tile
constexpr float kPMax = 256.0f;
constexpr size_t kCodesBytes = 2 * kCodeStages * 2 * kHalfCodeBytes;
constexpr size_t kSmemBytes =
    1024 + 2 * kStages * kConvBytes + kOnesBytes + kCodesBytes + 512;
}  // namespace tc8

__device__ __forceinline__ uint32_t f16x2_of_e4m3x2(uint32_t code_pair) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(static_cast<uint16_t>(code_pair)));
  return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t max_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float f16lo(uint32_t v) { return __half2float(__ushort_as_half(static_cast<uint16_t>(v))); }
__device__ __forceinline__ float f16hi(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<uint16_t>(v >> 16)));
}
__device__ __forceinline__ uint32_t f16x2_splat(float x) { return pack_f16(x, x); }

// Page-table entry idx of the layer, or (-1, 0, 0, 0) past the end of the list.
__device__ __forceinline__ int4 page_entry(const TcParams& p, int idx) {
  return idx < p.n_pages ? __ldg(&p.entries[idx]) : make_int4(-1, 0, 0, 0);
}
// Scale of (physical page, head), 0 for the past-the-end sentinel.
__device__ __forceinline__ float page_scale(const TcParams& p, const float* sc, int phys, int h) {
  return phys >= 0 ? __ldg(&sc[(p.page_base + phys) * p.H + h]) : 0.f;
}

// Dimension-adaptive scales a converter lane needs for one tile: for each of its half's two
// pages, the K scales of its 8-dim chunk and the page's K scale, and the V scales of its
// rows r0 + 4i (slot r0 + 4 (i mod 4) of page i / 4). Zero for the past-the-end page.
struct DaScales {
  float kc[2][8];
  float ks[2];
  float vt[8];
};
__device__ __forceinline__ void load_da_scales(const TcParams& p, int phys_lane, int h, int r0, int c0, DaScales& d) {
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int phys = __shfl_sync(0xffffffffu, phys_lane, g);
    if (phys >= 0) {
      const long long base = (p.page_base + phys) * p.H + h;
      const float4 a = __ldg(reinterpret_cast<const float4*>(p.k_chan + base * 64 + 8 * c0));
      const float4 b = __ldg(reinterpret_cast<const float4*>(p.k_chan + base * 64 + 8 * c0) + 1);
      d.kc[g][0] = a.x; d.kc[g][1] = a.y; d.kc[g][2] = a.z; d.kc[g][3] = a.w;
      d.kc[g][4] = b.x; d.kc[g][5] = b.y; d.kc[g][6] = b.z; d.kc[g][7] = b.w;
      d.ks[g] = __ldg(&p.k_scale[base]);
#pragma unroll
      for (int i = 0; i < 4; ++i) d.vt[4 * g + i] = __ldg(&p.v_tok[base * 16 + r0 + 4 * i]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) d.kc[g][e] = 0.f;
      d.ks[g] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) d.vt[4 * g + i] = 0.f;
    }
  }
}

template <int P, bool kDA>
__global__ void __launch_bounds__(tc8::kThreads, 1)
    attn_fp8_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const TcParams p) {
  griddep_wait();
  griddep_launch_dependents();
  using namespace tc8;
  constexpr int kPPT = kBN / P;               // pages per KV tile
  constexpr int kPPH = kPPT / 2;              // pages per converter half
  static_assert(kPPT % 2 == 0, "a KV tile splits into two halves of whole pages");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ck_s = smem;                                 // converted K tiles [kStages]
  uint8_t* cv_s = ck_s + kStages * kConvBytes;          // converted V tiles [kStages]
  uint8_t* ones_s = cv_s + kStages * kConvBytes;
  uint8_t* codes = ones_s + kOnesBytes;                 // [converter][kCodeStages][K, V][half tile]
  uint64_t* bars = reinterpret_cast<uint64_t*>(codes + kCodesBytes);
  uint64_t* q_ready = bars;                             // [kGroups] Q of the tile stored in TMEM
  uint64_t* ref_ready = bars + kGroups;                 // V reference scale written
  uint64_t* c8_full = ref_ready + 1;                    // [converter][kCodeStages]
  uint64_t* kc_full = c8_full + 2 * kCodeStages;        // [kStages] both halves converted
  uint64_t* kv_empty = kc_full + kStages;               // [kStages]
  uint64_t* s_full = kv_empty + kStages;                // [kGroups]
  uint64_t* s_free = s_full + kGroups;                  // [kGroups]
  uint64_t* p_full = s_free + kGroups;                  // [kGroups][2]
  uint64_t* pv_done = p_full + 2 * kGroups;             // [kGroups][2]
  uint64_t* mma_final = pv_done + 2 * kGroups;          // [kGroups]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + kGroups);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sref = reinterpret_cast<float*>(tmem_slot + 2);   // V reference scale

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = (p.q_tiles + 1) / 2;
  const int qp = blockIdx.x % pairs;
  const int rest = blockIdx.x / pairs;
  const int split = rest % p.splits;
  const int h = rest / p.splits;
  const int ngroups = (2 * qp + 1 < p.q_tiles) ? 2 : 1;  // the last pair may hold one tile
  const int tile0 = split * p.tiles_per_split;
  const int tile1 = min(tile0 + p.tiles_per_split, p.total_tiles);
  const int n_tiles = tile1 - tile0;

  if (threadIdx.x == 0) {
    mbar_init(&q_ready[0], 4);
    mbar_init(&q_ready[1], 4);
    mbar_init(ref_ready, 1);
    for (int i = 0; i < 2 * kCodeStages; ++i) mbar_init(&c8_full[i], 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kc_full[i], kConvThreads);
      mbar_init(&kv_empty[i], ngroups);                 // one commit per query tile's issuer
    }
    for (int g = 0; g < kGroups; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], 4);
      mbar_init(&p_full[2 * g], 4);
      mbar_init(&p_full[2 * g + 1], 4);
      mbar_init(&pv_done[2 * g], 1);
      mbar_init(&pv_done[2 * g + 1], 1);
      mbar_init(&mma_final[g], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < kOnesBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(ones_s)[i] = make_uint4(0x3c003c00u, 0x3c003c00u, 0x3c003c00u, 0x3c003c00u);
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
    if (warp == 0 || warp == 10) {
      // ------------------------------------------------ converters (TMA in lane 0 each)
      const int ci = warp == 0 ? 0 : 1;                 // half of every KV tile: pages 2ci, 2ci+1
      const int gl = ci * kPPH + (lane & (kPPH - 1));   // page of the tile tracked by lanes 0..kPPH-1
      uint64_t* c8f = c8_full + ci * kCodeStages;
      uint8_t* my_codes = codes + ci * (kCodeStages * 2 * kHalfCodeBytes);
      // V reference scale: the largest V scale of the head over this CTA's pages (both
      // converters compute the same value)
      float mv = 0.f;
#pragma unroll 4
      for (int idx = tile0 * kPPT + lane; idx < min(tile1 * kPPT, p.n_pages); idx += 32)
        mv = fmaxf(mv, page_scale(p, p.v_scale, __ldg(&p.entries[idx].x), h));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
      if (mv == 0.f) mv = 1.f;                          // all-zero pages: any reference works
      const float iv = 1.f / mv;
      if (ci == 0 && lane == 0) {
        *sref = mv;
        mbar_arrive(ref_ready);
      }
      // physical page gl of tiles ahead and its V scale; each value loaded in iteration j
      // is first used in iteration j + 1
      const int pq0 = page_entry(p, tile0 * kPPT + gl).x;
      int pq1 = page_entry(p, (tile0 + 1) * kPPT + gl).x;
      int pq2 = page_entry(p, (tile0 + 2) * kPPT + gl).x;
      int pq4n = page_entry(p, (tile0 + 3) * kPPT + gl).x;
      float vsn = page_scale(p, p.v_scale, pq0, h);
      DaScales dan;                                     // dimension-adaptive scales of the next tile
      if (kDA) load_da_scales(p, pq0, h, lane >> 3, lane & 7, dan);
#define KVC_FP8_ISSUE(t, phys)                                                                      \
  do {                                                                                              \
    const int st_ = (t) % kCodeStages;                                                              \
    uint8_t* kc_ = my_codes + st_ * 2 * kHalfCodeBytes;                                             \
    if (lane == 0) mbar_arrive_expect_tx(&c8f[st_], 2 * kHalfCodeBytes);                            \
    __syncwarp();                                                                                   \
    if (lane < kPPH) {                                                                              \
      const int row_ = (phys) >= 0 ? static_cast<int>(((p.page_base + (phys)) * p.H + h) * P) : p.pool_rows; \
      tma_load_2d(kc_ + lane * P * kHD, &tmap_k, &c8f[st_], 0, row_);                               \
      tma_load_2d(kc_ + kHalfCodeBytes + lane * P * kHD, &tmap_v, &c8f[st_], 0, row_);              \
    }                                                                                               \
  } while (0)
      if (lane == 0) {
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
      }
      static_assert(kCodeStages == 3, "the issue distance below is three tiles");
      KVC_FP8_ISSUE(0, pq0);
      if (n_tiles > 1) KVC_FP8_ISSUE(1, pq1);
      if (n_tiles > 2) KVC_FP8_ISSUE(2, pq2);
      int issued = min(n_tiles, kCodeStages);
      bool ok = true;
      // this converter's rows of the tile: 32 ci + (lane >> 3) + 4 i, i < 8, chunk lane & 7
      // of 8 dims; in the swizzled f16 tile the chunk moves to chunk ^ (row & 7)
      const int r0 = lane >> 3, c0 = lane & 7;
      const int src_off = r0 * kHD + c0 * 8;
      const int dst_base = ci * 32 * 128;
      const int dst_even = dst_base + r0 * 128 + ((c0 ^ r0) << 4);
      const int dst_odd = dst_base + r0 * 128 + ((c0 ^ r0 ^ 4) << 4);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kStages;
        const int cs = j % kCodeStages;
        const float fvj = vsn * iv;                     // V factor of page gl of tile j
        const int pq3 = pq4n;                           // page gl of tile j + 3
        vsn = page_scale(p, p.v_scale, pq1, h);         // tile j + 1
        pq4n = page_entry(p, (tile0 + j + 4) * kPPT + gl).x;
        uint32_t rv[kPPH];
#pragma unroll
        for (int g = 0; g < kPPH; ++g) rv[g] = f16x2_splat(__shfl_sync(0xffffffffu, fvj, g));
        // dimension-adaptive factors of tile j: K chunk scale over the page's K scale (the
        // page's logit factor carries the rest), V token scale over the V reference
        uint32_t kf[2][4], rvr[8];
        if (kDA) {
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const float inv = dan.ks[g] > 0.f ? 1.f / dan.ks[g] : 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) kf[g][e] = pack_f16(dan.kc[g][2 * e] * inv, dan.kc[g][2 * e + 1] * inv);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) rvr[i] = f16x2_splat(dan.vt[i] * iv);
          load_da_scales(p, pq1, h, lane >> 3, lane & 7, dan);   // tile j + 1
        }
        // converted stage st is free once the MMAs of tile j - kStages have completed
        if (j >= kStages &&
            !__all_sync(0xffffffffu, mbar_wait_bounded(&kv_empty[st], ((j / kStages) - 1) & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&c8f[cs], (j / kCodeStages) & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        const uint8_t* ksrc = my_codes + cs * 2 * kHalfCodeBytes + src_off;
        const uint8_t* vsrc = ksrc + kHalfCodeBytes;
        uint8_t* kdst = ck_s + st * kConvBytes;
        uint8_t* vdst = cv_s + st * kConvBytes;
#pragma unroll
        for (int i = 0; i < kBN / 8; ++i) {             // local row (lane >> 3) + 4 i, page i / 4
          const uint2 kc = *reinterpret_cast<const uint2*>(ksrc + i * 4 * kHD);
          const uint2 vc = *reinterpret_cast<const uint2*>(vsrc + i * 4 * kHD);
          uint4 ko, vo;
          ko.x = f16x2_of_e4m3x2(kc.x);
          ko.y = f16x2_of_e4m3x2(kc.x >> 16);
          ko.z = f16x2_of_e4m3x2(kc.y);
          ko.w = f16x2_of_e4m3x2(kc.y >> 16);
          if (kDA) {
            ko.x = hmul2(ko.x, kf[i >> 2][0]);
            ko.y = hmul2(ko.y, kf[i >> 2][1]);
            ko.z = hmul2(ko.z, kf[i >> 2][2]);
            ko.w = hmul2(ko.w, kf[i >> 2][3]);
          }
          const uint32_t vr = kDA ? rvr[i] : rv[i >> 2];
          vo.x = hmul2(f16x2_of_e4m3x2(vc.x), vr);
          vo.y = hmul2(f16x2_of_e4m3x2(vc.x >> 16), vr);
          vo.z = hmul2(f16x2_of_e4m3x2(vc.y), vr);
          vo.w = hmul2(f16x2_of_e4m3x2(vc.y >> 16), vr);
          const int off = i * 512 + ((i & 1) ? dst_odd : dst_even);
          *reinterpret_cast<uint4*>(kdst + off) = ko;
          *reinterpret_cast<uint4*>(vdst + off) = vo;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&kc_full[st]);
        __syncwarp();
        // code stage cs has been read by the whole warp: refill it with tile j + 3
        if (j + kCodeStages < n_tiles) {
          KVC_FP8_ISSUE(j + kCodeStages, pq3);
          ++issued;
        }
        pq1 = pq2;
        pq2 = pq3;
      }
#undef KVC_FP8_ISSUE
      // drain: the last code load issued into each stage has landed before the CTA exits
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < kCodeStages; ++i)
          if (issued > i) {
            const int t = i + kCodeStages * ((issued - 1 - i) / kCodeStages);
            mbar_wait_drain(&c8f[i], (t / kCodeStages) & 1, p.err);
          }
      }
    } else if (warp == 1 || warp == 11) {
      const int g = warp == 1 ? 0 : 1;
      if (g < ngroups) {
        // ---------------------------- MMA issuer of query tile g (one elected lane issues)
        const uint32_t idesc_s = idesc_f16kind(0, kBM, kBN, 0, 0);
        const uint32_t idesc_o = idesc_f16kind(0, kBM, kON, 0, 1);
        const uint32_t k_addr = smem_u32(ck_s), v_addr = smem_u32(cv_s);
        const uint32_t ones_addr = smem_u32(ones_s);
        const uint32_t tS = tmem + g * kGroupCols + kColS, tP = tmem + g * kGroupCols + kColP;
        const uint32_t tO = tmem + g * kGroupCols + kColO, tQ = tmem + g * kGroupCols + kColQ;
        const bool leader = elect_one();
        bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&q_ready[g], 0, abort_flag, p.err) &&
                                              mbar_wait_bounded(&kc_full[0], 0, abort_flag, p.err));
        if (ok) {
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk)
              mma_ts(tS, tQ + kk * 8, sw128_desc(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0);
            mma_commit(&s_full[g]);
          }
          __syncwarp();
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int st = j % kStages;
          if (j + 1 < n_tiles) {
            const int st1 = (j + 1) % kStages;
            if (!__all_sync(0xffffffffu,
                            mbar_wait_bounded(&kc_full[st1], ((j + 1) / kStages) & 1, abort_flag, p.err) &&
                                mbar_wait_bounded(&s_free[g], j & 1, abort_flag, p.err)))
              break;
            tc_fence_after();
            const uint32_t kb = k_addr + st1 * kConvBytes;
            if (leader) {
#pragma unroll
              for (int kk = 0; kk < kHD / 16; ++kk)
                mma_ts(tS, tQ + kk * 8, sw128_desc(kb + kk * 32, 16, 1024), idesc_s, kk > 0);
              mma_commit(&s_full[g]);
            }
            __syncwarp();
          }
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(&p_full[2 * g + (j & 1)], (j >> 1) & 1, abort_flag, p.err)))
            break;
          tc_fence_after();
          const uint32_t vb = v_addr + st * kConvBytes;
          const uint32_t lbo = ones_addr - vb;
          const uint32_t pa = tP + (j & 1) * (kBN / 2);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
              mma_ts(tO, pa + kk * 8, sw128_desc(vb + kk * 2048, lbo, 1024), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&pv_done[2 * g + (j & 1)]);
            mma_commit(&kv_empty[st]);
          }
          __syncwarp();
        }
        if (leader) mma_commit(&mma_final[g]);
        __syncwarp();
        mbar_wait_drain(&mma_final[g], 0, p.err);
      }
    } else if (((warp - 2) >> 2) < ngroups) {
      // ------------------------------------------------------------------ softmax warps
      const int g = (warp - 2) >> 2;                     // query tile of this warp
      const int qt = 2 * qp + g;
      const int wq = warp & 3;
      const int r = wq * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t tbase = tmem + g * kGroupCols + lane_off;
      const uint32_t tS = tbase + kColS, tP = tbase + kColP, tO = tbase + kColO;
      uint64_t* my_s_full = &s_full[g];
      uint64_t* my_s_free = &s_free[g];
      uint64_t* my_p_full = &p_full[2 * g];
      uint64_t* my_pv_done = &pv_done[2 * g];
      // this row of Q, bf16 -> f16, into TMEM: the A operand of S. The row is first scaled
      // by a power of two 2^e that brings its largest magnitude into [2^14, 2^15), so no
      // finite bf16 query overflows f16 and small rows keep their bits; the logit factor of
      // the row carries 2^-e, which makes the scaling exact (e is clamped to [-120, 100] so
      // that factor stays a normal fp32 number)
      float row_fac = 1.f;
      {
        uint32_t qv[32];
        const int row = qt * kBM + r;
        if (row < p.T) {
          const uint4* src = reinterpret_cast<const uint4*>(p.q + (static_cast<long long>(row) * p.H + h) * kHD);
          uint4 w[8];
          float qmax = 0.f;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            w[v] = __ldg(src + v);
            qmax = max3(qmax, fabsf(bf16lo(w[v].x)), fabsf(bf16hi(w[v].x)));
            qmax = max3(qmax, fabsf(bf16lo(w[v].y)), fabsf(bf16hi(w[v].y)));
            qmax = max3(qmax, fabsf(bf16lo(w[v].z)), fabsf(bf16hi(w[v].z)));
            qmax = max3(qmax, fabsf(bf16lo(w[v].w)), fabsf(bf16hi(w[v].w)));
          }
          int e = 0;
          if (qmax > 0.f) {
            int ex;
            frexpf(qmax, &ex);                            // qmax in [2^(ex-1), 2^ex)
            e = min(100, max(-120, 15 - ex));
          }
          row_fac = ldexpf(1.f, -e);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            qv[4 * v] = pack_f16(ldexpf(bf16lo(w[v].x), e), ldexpf(bf16hi(w[v].x), e));
            qv[4 * v + 1] = pack_f16(ldexpf(bf16lo(w[v].y), e), ldexpf(bf16hi(w[v].y), e));
            qv[4 * v + 2] = pack_f16(ldexpf(bf16lo(w[v].z), e), ldexpf(bf16hi(w[v].z), e));
            qv[4 * v + 3] = pack_f16(ldexpf(bf16lo(w[v].w), e), ldexpf(bf16hi(w[v].w), e));
          }
        } else {
#pragma unroll
          for (int v = 0; v < 32; ++v) qv[v] = 0u;
        }
        tmem_st32(tbase + kColQ, qv);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_ready[g]);
      }
      bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(ref_ready, 0, abort_flag, p.err));
      const float vref = ok ? *sref : 1.f;
      float m = -INFINITY;
      // Lanes 0..3 hold page g = lane of the current tile (K scale, valid slots) and the
      // entry of the next tile, loaded one tile ahead; every lane reads them by shuffle.
      // Pages past the list have scale 0 and no valid slots.
      const int gl = lane & 3;
      int4 en = page_entry(p, tile0 * kPPT + gl);
      float ksj = page_scale(p, p.k_scale, en.x, h);
      int vj = en.w;
      en = page_entry(p, (tile0 + 1) * kPPT + gl);
      uint32_t s[2][32];
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(my_s_full, 0, abort_flag, p.err));
      if (ok) {
        tc_fence_after();
        tmem_ld32(tS + 0, s[0]);
        tmem_ld32(tS + 32, s[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(my_s_free);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        int n_masked = 0;
        float cg[kPPT];            // logit factor per page: log2(e) x softmax scale x K scale
        int vpg[kPPT];             // valid slots per page
#pragma unroll
        for (int pg = 0; pg < kPPT; ++pg) {
          vpg[pg] = __shfl_sync(0xffffffffu, vj, pg);
          n_masked += P - vpg[pg];
          // a zero-scale page (all-zero K, or past the list) gets a tiny positive factor: its
          // valid scores are 0 either way, and its masked -inf scores stay -inf
          cg[pg] = fmaxf((p.scale_log2 * row_fac) * __shfl_sync(0xffffffffu, ksj, pg), 1e-30f);
        }
        if (n_masked) {
          // slots past a page's valid count (and pages past the list end) take no weight
#pragma unroll
          for (int cc = 0; cc < kBN; ++cc)
            if ((cc % P) >= vpg[cc / P]) s[cc / 32][cc % 32] = __float_as_uint(-INFINITY);
        }
        if (j + 1 < n_tiles) {
          ksj = page_scale(p, p.k_scale, en.x, h);
          vj = en.w;
          en = page_entry(p, (tile0 + j + 2) * kPPT + gl);
        }
        uint32_t pb[kBN / 2];
        uint32_t mxb = 0u;
        {
          const uint64_t nm2 = pk2(-m, -m);
#pragma unroll
          for (int pg = 0; pg < kPPT; ++pg) {
            const uint64_t c2 = pk2(cg[pg], cg[pg]);
#pragma unroll
            for (int i = pg * (P / 2); i < (pg + 1) * (P / 2); ++i) {
              float x0, x1;
              up2(fma2_pair(s[(2 * i) / 32][(2 * i) % 32], s[(2 * i + 1) / 32][(2 * i + 1) % 32], c2, nm2), x0,
                  x1);
              pb[i] = pack_f16(ex2(x0), ex2(x1));
              mxb = max_f16x2(mxb, pb[i]);
            }
          }
        }
        const bool move = (j == 0) || fmaxf(f16lo(mxb), f16hi(mxb)) > kPMax;
        if (__any_sync(0xffffffffu, move)) {
          // exact row maximum of the scaled logits: per page, the largest raw score times
          // the page's (non-negative) factor
          float mt = -INFINITY;
#pragma unroll
          for (int pg = 0; pg < kPPT; ++pg) {
            float ta = -INFINITY, tb = -INFINITY;
#pragma unroll
            for (int cc = pg * P; cc < (pg + 1) * P; cc += 4) {
              ta = max3(ta, __uint_as_float(s[cc / 32][cc % 32]), __uint_as_float(s[cc / 32][cc % 32 + 1]));
              tb = max3(tb, __uint_as_float(s[cc / 32][cc % 32 + 2]), __uint_as_float(s[cc / 32][cc % 32 + 3]));
            }
            mt = fmaxf(mt, fmaxf(ta, tb) * cg[pg]);
          }
          const float m_new = move ? (mt == -INFINITY ? (m == -INFINITY ? 0.f : m) : mt) : m;
          const bool resc = move && j > 0;
          if (__any_sync(0xffffffffu, resc)) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&my_pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag,
                                                            p.err))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float f = resc ? ex2(m - m_new) : 1.0f;
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
          const uint64_t nm2 = pk2(-m, -m);
#pragma unroll
          for (int pg = 0; pg < kPPT; ++pg) {
            const uint64_t c2 = pk2(cg[pg], cg[pg]);
#pragma unroll
            for (int i = pg * (P / 2); i < (pg + 1) * (P / 2); ++i) {
              float x0, x1;
              up2(fma2_pair(s[(2 * i) / 32][(2 * i) % 32], s[(2 * i + 1) / 32][(2 * i + 1) % 32], c2, nm2), x0,
                  x1);
              pb[i] = pack_f16(ex2(x0), ex2(x1));
            }
          }
        }
        if (j >= 2) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(&my_pv_done[j & 1], ((j - 2) >> 1) & 1, abort_flag,
                                                          p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st32(tP + (j & 1) * (kBN / 2), pb);
        const bool more = j + 1 < n_tiles;
        if (more) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(my_s_full, (j + 1) & 1, abort_flag, p.err))) {
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
        if (lane == 0) mbar_arrive(&my_p_full[j & 1]);
        if (more) {
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(my_s_free);
        }
      }
      const int jl = n_tiles - 1;
      if (__all_sync(0xffffffffu, ok && mbar_wait_bounded(&my_pv_done[jl & 1], (jl >> 1) & 1, abort_flag, p.err))) {
        tc_fence_after();
        uint32_t o0[32], o1[32], ls[16];
        tmem_ld32(tO, o0);
        tmem_ld32(tO + 32, o1);
        tmem_ld16(tO + 64, ls);
        tmem_ld_wait();
        const float l = __uint_as_float(ls[0]);
        const float inv = vref / l;
        const int row = qt * kBM + r;
        if (p.splits == 1) {
          if (row < p.T) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<long long>(row) * p.H + h) * kHD);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const uint32_t* src = v < 4 ? &o0[8 * v] : &o1[8 * (v - 4)];
              uint4 w;
              w.x = pack_bf16(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv);
              w.y = pack_bf16(__uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv);
              w.z = pack_bf16(__uint_as_float(src[4]) * inv, __uint_as_float(src[5]) * inv);
              w.w = pack_bf16(__uint_as_float(src[6]) * inv, __uint_as_float(src[7]) * inv);
              dst[v] = w;
            }
          }
        } else {
          const long long pi = (static_cast<long long>(h) * p.splits + split) * p.q_tiles + qt;
          float4* dst = reinterpret_cast<float4*>(p.part_o + (pi * kBM + r) * kHD);
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const uint32_t* src = v < 8 ? &o0[4 * v] : &o1[4 * (v - 8)];
            dst[v] = make_float4(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv,
                                 __uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv);
          }
          p.part_lse[pi * kBM + r] = m + __log2f(l);
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

cudaError_t launch_attn_fp8_kernel(cudaStream_t s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                   const TcParams& prm, int grid) {
  static PerDeviceOnce attr;
  cudaError_t e = attr.run([] {
    cudaError_t r = cudaFuncSetAttribute(attn_fp8_kernel<16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(tc8::kSmemBytes));
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(attn_fp8_kernel<16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(tc8::kSmemBytes));
    return r;
  });
  if (e != cudaSuccess) return e;
  if (prm.k_chan)
    return launch_pdl(attn_fp8_kernel<16, true>, dim3(grid), dim3(tc8::kThreads), tc8::kSmemBytes, s, tq, tk, tv, prm);
  return launch_pdl(attn_fp8_kernel<16, false>, dim3(grid), dim3(tc8::kThreads), tc8::kSmemBytes, s, tq, tk, tv, prm);
}

}  // namespace kvc
