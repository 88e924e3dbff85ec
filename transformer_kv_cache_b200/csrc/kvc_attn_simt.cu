// kvc_attn_simt.cu -- frame attention over the paged cache with fp32 FMA arithmetic.
//
// O[i, h] = sum_j softmax_j(scale * q_i . k_j) v_j over every valid slot of the layer's
// page list ("How GCTStream ...", Frame-by-Frame Causal Processing: the new frame's
// queries attend to the cached frames and to themselves, no mask). Used for fp32 caches,
// where bf16/tf32 tensor cores cannot hold a 1e-4 tolerance, and for head sizes outside
// the tensor-core kernel. One thread owns one query row of one head and runs an online
// softmax; each page's (head) block is staged once in shared memory for the CTA's rows.
#include <cuda_bf16.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {

constexpr int kSimtRows = 128;

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
__device__ __forceinline__ float e4m3_to_f(uint8_t c) {
  // OCP FP8 E4M3: sign, 4-bit exponent (bias 7), 3-bit mantissa; subnormals m * 2^-9
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  const float v = (e == 0) ? ldexpf(static_cast<float>(m), -9) : ldexpf(static_cast<float>(8 + m), e - 10);
  return s ? -v : v;
}

template <typename TIO>
__device__ __forceinline__ void st_f(TIO* p, float v);
template <>
__device__ __forceinline__ void st_f<float>(float* p, float v) {
  *p = v;
}
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// KV storage kinds: 0 = fp32, 1 = bf16, 2 = FP8 E4M3 codes with per-(page, head) scale.
template <typename TIO, int KV, int D>
__global__ void __launch_bounds__(kSimtRows) attn_simt_kernel(const TIO* __restrict__ q, TIO* __restrict__ o,
                                                               const void* __restrict__ k_pool,
                                                               const void* __restrict__ v_pool,
                                                               const float* __restrict__ k_scale,
                                                               const float* __restrict__ v_scale,
                                                               const Entry* __restrict__ entries, int n_pages,
                                                               int T, int H, int P, float scale_log2) {
  extern __shared__ float sm[];
  float* ks = sm;            // [P][D]
  float* vs = sm + P * D;    // [P][D]
  const int h = blockIdx.y;
  const int row = blockIdx.x * kSimtRows + threadIdx.x;
  const bool active = row < T;
  float qv[D];
#pragma unroll
  for (int d = 0; d < D; ++d) qv[d] = active ? ld_f<TIO>(q + (static_cast<long long>(row) * H + h) * D + d) : 0.f;
  float acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) acc[d] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int pg = 0; pg < n_pages; ++pg) {
    const Entry e = entries[pg];
    const int phys = e.x, valid = e.w;
    __syncthreads();
    const long long base = (static_cast<long long>(phys) * H + h) * P * D;
    for (int i = threadIdx.x; i < valid * D; i += kSimtRows) {
      float kx, vx;
      if (KV == 0) {
        kx = static_cast<const float*>(k_pool)[base + i];
        vx = static_cast<const float*>(v_pool)[base + i];
      } else if (KV == 1) {
        kx = __bfloat162float(static_cast<const __nv_bfloat16*>(k_pool)[base + i]);
        vx = __bfloat162float(static_cast<const __nv_bfloat16*>(v_pool)[base + i]);
      } else {
        const float sk = k_scale[static_cast<long long>(phys) * H + h];
        const float sv = v_scale[static_cast<long long>(phys) * H + h];
        kx = e4m3_to_f(static_cast<const uint8_t*>(k_pool)[base + i]) * sk;
        vx = e4m3_to_f(static_cast<const uint8_t*>(v_pool)[base + i]) * sv;
      }
      ks[i] = kx;
      vs[i] = vx;
    }
    __syncthreads();
    for (int j = 0; j < valid; ++j) {
      float z = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) z = fmaf(qv[d], ks[j * D + d], z);
      z *= scale_log2;
      const float m_new = fmaxf(m, z);
      const float corr = exp2f(m - m_new);
      const float p = exp2f(z - m_new);
      l = l * corr + p;
#pragma unroll
      for (int d = 0; d < D; ++d) acc[d] = fmaf(acc[d], corr, p * vs[j * D + d]);
      m = m_new;
    }
  }
  if (!active) return;
  const float inv = 1.f / l;
#pragma unroll
  for (int d = 0; d < D; ++d) st_f<TIO>(o + (static_cast<long long>(row) * H + h) * D + d, acc[d] * inv);
}

template <typename TIO, int KV>
static cudaError_t launch_simt_d(cudaStream_t s, const void* q, void* o, const void* kp, const void* vp,
                                 const float* ks, const float* vs, const Entry* entries, int n_pages, int T, int H,
                                 int D, int P, float scale_log2) {
  dim3 grid((T + kSimtRows - 1) / kSimtRows, H);
  const size_t smem = 2 * static_cast<size_t>(P) * D * sizeof(float);
  switch (D) {
#define KVC_CASE(DD)                                                                                          \
  case DD:                                                                                                    \
    if (smem > 48 * 1024)                                                                                     \
      cudaFuncSetAttribute(attn_simt_kernel<TIO, KV, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                           static_cast<int>(smem));                                                           \
    attn_simt_kernel<TIO, KV, DD><<<grid, kSimtRows, smem, s>>>(static_cast<const TIO*>(q), static_cast<TIO*>(o), \
                                                                kp, vp, ks, vs, entries, n_pages, T, H, P,    \
                                                                scale_log2);                                  \
    break;
    KVC_CASE(16)
    KVC_CASE(32)
    KVC_CASE(64)
    KVC_CASE(128)
#undef KVC_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(cudaStream_t s, int io_dtype, int kv_dtype, const void* q, void* o,
                             const void* k_pool, const void* v_pool, const float* k_scale, const float* v_scale,
                             const Entry* entries, int n_pages, int T, int H, int D, int P, float softmax_scale) {
  const float scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  if (io_dtype == KVC_F32 && kv_dtype == KVC_F32)
    return launch_simt_d<float, 0>(s, q, o, k_pool, v_pool, k_scale, v_scale, entries, n_pages, T, H, D, P,
                                   scale_log2);
  if (io_dtype == KVC_BF16 && kv_dtype == KVC_BF16)
    return launch_simt_d<__nv_bfloat16, 1>(s, q, o, k_pool, v_pool, k_scale, v_scale, entries, n_pages, T, H, D,
                                           P, scale_log2);
  if (io_dtype == KVC_BF16 && kv_dtype == KVC_FP8_E4M3)
    return launch_simt_d<__nv_bfloat16, 2>(s, q, o, k_pool, v_pool, k_scale, v_scale, entries, n_pages, T, H, D,
                                           P, scale_log2);
  return cudaErrorInvalidValue;
}

}  // namespace kvc
