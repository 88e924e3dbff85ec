// kvc_attn_common.cuh -- parameters and device helpers shared by the tensor-core attention
// kernels (bf16 and FP8 storage).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {

struct TcParams {
  const __nv_bfloat16* q;       // [T][H][D] queries
  const float* k_scale;         // FP8 storage only: per (pool page, head) scales
  const float* v_scale;
  const Entry* entries;
  int n_pages, T, H;
  int q_tiles, splits, tiles_per_split, total_tiles;
  int q_pairs;                  // bf16 kernel: query-tile pairs (one per CTA of a group)
  int out_heads, head0;         // bf16 kernel: heads of Q and O; the cache's head h is head0 + h
  long long page_base;          // layer * pool_pages: first pool page of the layer
  int pool_rows;                // rows of the pool tensor maps (a row index past the end reads zeros)
  float scale_log2;
  __nv_bfloat16* out;
  float* part_o;
  float* part_lse;
  int* err;
  int head_pages;               // > 0: per-head page lists (see TcAttnArgs)
  int* split_cnt;               // [H][q_tiles][4] zeroed counters: the piece that counts last merges (bf16 kernel)
  const float* k_chan;          // dimension-adaptive FP8: [pool page][head][64] K channel scales
  const float* v_tok;           // dimension-adaptive FP8: [pool page][head][16] V token scales
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

// ---- packed arithmetic used by the softmax
__device__ __forceinline__ uint64_t fma2_pair(uint32_t s0, uint32_t s1, uint64_t c2, uint64_t nm2) {
  uint64_t x, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(s0), "r"(s1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(x), "l"(c2), "l"(nm2));
  return r;
}
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void up2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Upper halves of two fp32 values as a bf16 pair (truncation toward zero), one byte
// permute; P is consumed by the MMA and summed by it from the same bf16 values, so the
// truncation's common scale cancels in O / l.
__device__ __forceinline__ uint32_t bf16x2_trunc(float lo, float hi) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(__float_as_uint(lo)), "r"(__float_as_uint(hi)));
  return r;
}

// True in exactly one lane of a converged warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}" : "=r"(pred));
  return pred != 0;
}



// FP8 E4M3 storage variant (kvc_attn_fp8.cu): same parameters, the query map of the bf16
// kernel, pool maps over the code bytes (box 64 B x P rows, no swizzle).
cudaError_t launch_attn_fp8_kernel(cudaStream_t s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                   const TcParams& prm, int grid);

}  // namespace kvc
