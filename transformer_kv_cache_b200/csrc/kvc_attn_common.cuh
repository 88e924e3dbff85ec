// kvc_attn_common.cuh -- parameters and device helpers of the tensor-core attention kernel
// (bf16 and FP8 E4M3 storage).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvc_internal.h"
#include "sm100_ptx.cuh"

namespace kvc {

struct TcParams {
  const float* k_scale;         // E4M3 storage: [pool page][head] K and V scales
  const float* v_scale;
  int T, H;
  int q_tiles;                  // 128-row query tiles
  int splits;                   // most pieces of one unit (head, query-tile pair)
  int tiles_per_split;          // R: steps (128-slot KV tiles) per group of CTAs
  int total_tiles;              // steps of all layers
  int q_pairs;                  // query-tile pairs (one per CTA of a group)
  int out_heads, head0;         // heads of Q and O; the cache's head h is head0 + h
  int pool_rows;                // rows of the pool tensor maps (a row index past the end reads zeros)
  float scale_log2;
  float* part_o;
  float* part_lse;
  int* err;
  int head_pages;               // > 0: per-head page lists (see TcAttnArgs)
  int* split_cnt;               // [layer x H][q_tiles][4] zeroed counters: the piece that counts last merges
  const float* k_chan;          // dimension-adaptive E4M3: [pool page][head][64] K channel scales
  const float* v_tok;           // dimension-adaptive E4M3: [pool page][head][16] V token scales
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


}  // namespace kvc
