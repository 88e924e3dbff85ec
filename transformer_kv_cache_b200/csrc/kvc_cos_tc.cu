// kvc_cos_tc.cu -- merge-target search of the keep / merge / drop compression: for every
// merge source, the eligible kept token of highest full-key cosine ("StreamCacheVGGT",
// section 2: merge the middle tier into the most similar kept token).
//
// The decision is taken in fp64, as the definition is written; the tensor cores only
// narrow the search:
//
//   screen  one CTA per 256 sources x 256 targets (two M=128, N=256 accumulators filling
//           TMEM, so each key byte brought from L2 feeds 128 multiply-adds): the bf16 keys
//           (stored values, exact) of both sides go through tcgen05 (K = H*D, fp32
//           accumulation in TMEM); the epilogue scales each dot product by the two fp32
//           inverse norms and keeps the four largest approximate cosines of the tile per
//           source.
//   refine  one warp per source: M = the largest screened value over all tiles; every
//           target whose screened value is within kMargin of M is re-evaluated in fp64,
//           and where a tile's fourth value is itself within the margin, all targets of
//           that tile are. The fp64 argmax (lowest index on ties) is the target.
//
// Bound: each bf16 product is exact in fp32; the fp32 accumulation of 1024 products in
// any order and grouping adds at most (1024 + 64) * 2^-23 * sum|a_i b_i| <= 1.3e-4
// * |a| |b|, and the inverse norms and two scalings add a few 2^-24 relative. The
// screened cosine is therefore within 1.4e-4 of the fp64 one, and any target whose fp64
// cosine can be the maximum has a screened value >= M - 2.8e-4 > M - kMargin.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {
namespace cs {
constexpr int kBM = 128;                           // sources per accumulator (MMA M)
constexpr int kMT = 2;                             // accumulators per CTA: 256 sources
constexpr int kBN = 256;                           // targets per CTA (MMA N)
constexpr int kBK = 64;                            // key dims per stage
constexpr int kStages = 3;
constexpr int kBoxBytes = 128 * kBK * 2;           // one TMA box: 128 rows x 64 dims (16 KB)
constexpr int kATileBytes = kMT * kBoxBytes;       // 256 source rows
constexpr int kBTileBytes = 2 * kBoxBytes;         // 256 target rows
constexpr int kThreads = 384;                      // TMA, MMA, 2 idle, 8 epilogue warps
constexpr int kTmemCols = 512;
constexpr size_t kSmemBytes = 1024 + kStages * (kATileBytes + kBTileBytes) + kBN * 4 + 256;
constexpr float kMargin = 0.0009765625f;           // 2^-10
}  // namespace cs

// Screened cosines: warp 0 lane 0 issues TMA loads, warp 1 lane 0 issues the MMAs, warps
// 4..11 run the epilogue (one source row per thread; warps 4..7 the first accumulator,
// 8..11 the second).
__global__ void __launch_bounds__(cs::kThreads, 1)
    cos_screen_kernel(const __grid_constant__ CUtensorMap tmap_s, const __grid_constant__ CUtensorMap tmap_e,
                      const float* __restrict__ inv_ns, const float* __restrict__ inv_ne, int n_src, int n_elig,
                      int HD, float* __restrict__ top_v, int32_t* __restrict__ top_j, int tiles_n, int* err) {
  using namespace cs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                                   // sources [kStages][256 rows]
  uint8_t* b_s = smem + kStages * kATileBytes;           // targets [kStages][256 rows]
  float* inv_e_s = reinterpret_cast<float*>(b_s + kStages * kBTileBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(inv_e_s + kBN);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * kBN, s0 = blockIdx.y * (kMT * kBM);
  const int nk = (HD + kBK - 1) / kBK;                  // dims past HD read as zeros

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmap_s);
      tma_prefetch_desc(&tmap_e);
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % kStages;
        if (kb >= kStages && !mbar_wait_bounded(&empty[st], ((kb / kStages) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&full[st], kATileBytes + kBTileBytes);
        tma_load_2d(a_s + st * kATileBytes, &tmap_s, &full[st], kb * kBK, s0);
        tma_load_2d(a_s + st * kATileBytes + kBoxBytes, &tmap_s, &full[st], kb * kBK, s0 + 128);
        tma_load_2d(b_s + st * kBTileBytes, &tmap_e, &full[st], kb * kBK, e0);
        tma_load_2d(b_s + st * kBTileBytes + kBoxBytes, &tmap_e, &full[st], kb * kBK, e0 + 128);
        issued = kb + 1;
      }
      // the last load issued into each stage has landed before the CTA exits
      volatile int never = 0;
      for (int i = 0; i < kStages; ++i)
        if (issued > i) {
          const int kb = i + kStages * ((issued - 1 - i) / kStages);
          mbar_wait_bounded(&full[i], (kb / kStages) & 1, &never, err);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16kind(1, kBM, kBN, 0, 0);
      const uint32_t a_addr = smem_u32(a_s), b_addr = smem_u32(b_s);
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % kStages;
        if (!mbar_wait_bounded(&full[st], (kb / kStages) & 1, abort_flag, err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt)
            mma_ss(tmem + mt * kBN, sw128_desc(a_addr + st * kATileBytes + mt * kBoxBytes + kk * 32, 16, 1024),
                   sw128_desc(b_addr + st * kBTileBytes + kk * 32, 16, 1024), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[st]);
      }
      mma_commit(acc_full);
      volatile int never = 0;
      mbar_wait_bounded(acc_full, 0, &never, err);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 128;                   // 0..255
    inv_e_s[et] = e0 + et < n_elig ? inv_ne[e0 + et] : 0.f;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const int mt = (warp - 4) >> 2;                     // accumulator of this warp
    const int wq = warp & 3;                            // its TMEM lane quadrant
    const int row = wq * 32 + lane;
    const int i = s0 + mt * kBM + row;
    const float inv_s = i < n_src ? inv_ns[i] : 0.f;
    float t0 = -INFINITY, t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
    int j0 = 0x7fffffff, j1 = 0x7fffffff, j2 = 0x7fffffff, j3 = 0x7fffffff;
    if (__all_sync(0xffffffffu, mbar_wait_bounded(acc_full, 0, abort_flag, err))) {
      tc_fence_after();
      const uint32_t taddr = tmem + mt * kBN + (static_cast<uint32_t>(wq * 32) << 16);
#pragma unroll 1
      for (int q = 0; q < kBN / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(taddr + q * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = q * 32 + c;
          const float x = __uint_as_float(v[c]) * inv_s * inv_e_s[col];
          // ascending j with strict comparisons: equal values keep the lower index first
          if (e0 + col < n_elig && x > t3) {
            const int j = e0 + col;
            if (x > t2) {
              t3 = t2;
              j3 = j2;
              if (x > t1) {
                t2 = t1;
                j2 = j1;
                if (x > t0) {
                  t1 = t0;
                  j1 = j0;
                  t0 = x;
                  j0 = j;
                } else {
                  t1 = x;
                  j1 = j;
                }
              } else {
                t2 = x;
                j2 = j;
              }
            } else {
              t3 = x;
              j3 = j;
            }
          }
        }
      }
    }
    if (i < n_src) {
      const long long o = (static_cast<long long>(i) * tiles_n + blockIdx.x) * 4;
      *reinterpret_cast<float4*>(top_v + o) = make_float4(t0, t1, t2, t3);
      *reinterpret_cast<int4*>(top_j + o) = make_int4(j0, j1, j2, j3);
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

// fp64 cosine of source row i and target row j over HD bf16 dims (8 per lane per step),
// reduced across the warp; every lane returns the same value.
__device__ __forceinline__ double cos_f64(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                                          int HD, double na, double nb, int lane) {
  double acc = 0.0;
  for (int c = lane * 8; c < HD; c += 256) {
    const uint4 x = *reinterpret_cast<const uint4*>(a + c);
    const uint4 y = *reinterpret_cast<const uint4*>(b + c);
    const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* yb = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fx = __bfloat1622float2(xa[e]), fy = __bfloat1622float2(yb[e]);
      acc = fma(static_cast<double>(fx.x), static_cast<double>(fy.x), acc);
      acc = fma(static_cast<double>(fx.y), static_cast<double>(fy.y), acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc / (nb * na);
}

__global__ void cos_refine_kernel(const float* __restrict__ top_v, const int32_t* __restrict__ top_j, int tiles_n,
                                  const __nv_bfloat16* __restrict__ ks, const __nv_bfloat16* __restrict__ ke,
                                  const double* __restrict__ ns, const double* __restrict__ ne, int n_src, int n_elig,
                                  int HD, int32_t* __restrict__ target) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (i >= n_src) return;
  const int nt = (n_elig + cs::kBN - 1) / cs::kBN;
  const float* tv = top_v + static_cast<long long>(i) * tiles_n * 4;
  const int32_t* tj = top_j + static_cast<long long>(i) * tiles_n * 4;
  float M = -INFINITY;
  for (int t = lane; t < nt; t += 32) M = fmaxf(M, tv[4 * t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float thr = M - cs::kMargin;
  const __nv_bfloat16* a = ks + static_cast<long long>(i) * HD;
  const double na = ns[i];
  double bv = -INFINITY;
  int bj = 0x7fffffff;
  auto consider = [&](int j) {
    if (j < 0 || j >= n_elig) return;                  // unfilled slots of a short tile
    const double cv = cos_f64(a, ke + static_cast<long long>(j) * HD, HD, na, ne[j], lane);
    if (cv > bv || (cv == bv && j < bj)) {
      bv = cv;
      bj = j;
    }
  };
  for (int base = 0; base < nt; base += 32) {
    const int t = base + lane;
    float v4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    int j4[4] = {0, 0, 0, 0};
    if (t < nt) {
      const float4 vv = *reinterpret_cast<const float4*>(tv + 4 * t);
      const int4 jj = *reinterpret_cast<const int4*>(tj + 4 * t);
      v4[0] = vv.x; v4[1] = vv.y; v4[2] = vv.z; v4[3] = vv.w;
      j4[0] = jj.x; j4[1] = jj.y; j4[2] = jj.z; j4[3] = jj.w;
    }
    // a tile whose fourth value is within the margin may hide more candidates: all of it
    const bool exhaustive = v4[3] >= thr;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t m = __ballot_sync(0xffffffffu, !exhaustive && v4[q] >= thr);
      while (m) {
        const int src = __ffs(m) - 1;
        m &= m - 1;
        consider(__shfl_sync(0xffffffffu, j4[q], src));
      }
    }
    uint32_t em = __ballot_sync(0xffffffffu, exhaustive);
    while (em) {
      const int src = __ffs(em) - 1;
      em &= em - 1;
      const int j_end = min((base + src + 1) * cs::kBN, n_elig);
      for (int j = (base + src) * cs::kBN; j < j_end; ++j) consider(j);
    }
  }
  if (lane == 0) target[i] = bj < n_elig ? bj : 0;   // only after an aborted screen
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// rows x HD bf16 matrix, box of 64 dims x 128 rows, 128-byte swizzle; rows past `rows`
// read as zeros.
static bool encode_keys_tmap(CUtensorMap* map, const void* base, int rows, int HD) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(HD), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(HD) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(cs::kBK), static_cast<cuuint32_t>(cs::kBM)};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_merge_targets(cudaStream_t s, const __nv_bfloat16* ks, const __nv_bfloat16* ke,
                                 const double* ns, const double* ne, const float* inv_ns, const float* inv_ne,
                                 int n_src, int n_elig, int HD, float* top_v, int32_t* top_j, int tiles_n,
                                 int32_t* target, int* err, int* launched) {
  *launched = 0;
  if (n_src <= 0 || n_elig <= 0) return cudaSuccess;
  if (HD % 8 != 0 || (n_elig + cs::kBN - 1) / cs::kBN > tiles_n) return cudaErrorInvalidValue;
  static PerDeviceOnce attr;
  cudaError_t ea = attr.run([] {
    return cudaFuncSetAttribute(cos_screen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(cs::kSmemBytes));
  });
  if (ea != cudaSuccess) return ea;
  CUtensorMap ts, te;
  if (!encode_keys_tmap(&ts, ks, n_src, HD) || !encode_keys_tmap(&te, ke, n_elig, HD)) return cudaErrorInvalidValue;
  dim3 grid((n_elig + cs::kBN - 1) / cs::kBN, (n_src + cs::kMT * cs::kBM - 1) / (cs::kMT * cs::kBM));
  cos_screen_kernel<<<grid, cs::kThreads, cs::kSmemBytes, s>>>(ts, te, inv_ns, inv_ne, n_src, n_elig, HD, top_v,
                                                               top_j, tiles_n, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int threads = 256;
  cos_refine_kernel<<<(n_src * 32 + threads - 1) / threads, threads, 0, s>>>(top_v, top_j, tiles_n, ks, ke, ns, ne,
                                                                            n_src, n_elig, HD, target);
  e = cudaGetLastError();
  *launched = e == cudaSuccess ? 2 : 1;
  return e;
}

}  // namespace kvc
