// kvc_attn_tc.cu -- frame attention over the paged cache (bf16 or FP8 E4M3 storage) on
// sm_100a tensor cores.
//
// Computes O[i, h] = sum_j softmax_j(scale * q_i . k_j) v_j for the T queries of the new
// frame over every valid slot of the layer's page list ("How GCTStream ...",
// Frame-by-Frame Causal Processing; "InfiniteVGGT" explainer, Causal Attention) without
// materialising the score matrix, as a flash-attention pipeline built for Blackwell.
//
// Work decomposition. A unit is one head and one pair of 128-row query tiles (256 query
// rows). The KV sequence of a head is cut into 128-slot tiles (8 pages). The launch is
// persistent: CTAs form groups of q_pairs CTAs (one per query-tile pair), and group g sweeps
// the contiguous range [g*R, (g+1)*R) of the flattened (head, KV tile) sequence, so every
// CTA of a group reads the same K/V tiles at about the same time and the group's other
// CTAs find them in L2. A range may end inside a head and the next group continue it: the
// pieces of a unit are merged by the piece that finishes last (partial outputs carry their
// log2-sum-exp), so no separate combine launch is needed.
//
// Roles of a CTA (384 threads for bf16 storage, one CTA per SM, all 512 TMEM columns;
// warpgroup 0 gives up registers to the two softmax warpgroups with setmaxnreg):
//   warp 0 (one lane)   TMA producer: per KV tile the 8 page-head blocks of K and of V
//                       (128-byte swizzled) into a 5-stage ring. Pages past the end of the
//                       list are read past the end of the pool, which TMA fills with zeros.
//   warps 1, 2          MMA issuers of query tile 0 and 1 (the warp waits, one elected lane
//                       issues), per 64-slot half of a KV tile: S = Q K^T (tcgen05.mma
//                       kind::f16, M=128, N=64, A = Q read from TMEM, B = the K half in
//                       shared memory) and O' += P [V | 1] (M=128, N=80, A = P from TMEM,
//                       B = the V half as an MN-major operand followed by a block of
//                       ones), so column 64 of O' is the exact row sum of the bf16 P used.
//   warps 4-7, 8-11     softmax of query tile 0 and 1 (thread = query row = TMEM lane):
//                       first the row of Q into TMEM, then per half the 64 scores from
//                       TMEM, P = 2^(s*c - m) for 6 of every 8 column pairs on the MUFU
//                       and for 2 on the FMA pipe (a cubic in the fraction, the integer
//                       part added to the exponent field), interleaved, rounded to bf16
//                       pairs and written over the first 32 columns of the half's own S
//                       buffer.
//
// TMEM per query tile (248 of 256 columns): Q (32: bf16 pairs), the mask product's A
// operand (8), two S buffers (64 each;
// half u uses buffer u & 1, and its P goes over the buffer's first 32 columns once its S is
// in registers), O' (80). The issuer keeps S one half ahead of the softmax: after the P.V
// product of half u it issues S of half u + 2 into the same buffer (one issuer's MMAs run
// in order, so the product has read P before S overwrites it). A softmax warp then finds
// the next S computed when it finishes a half, and each half costs it one wait (S ready)
// and one arrive (P ready).
//
// Online softmax with lazy rescaling: the reference max m of a row only moves when a
// half's P would exceed 2^8 (the exact fp32 max of the half, from 3-input max
// instructions, is compared with m + 8). When a row's reference moves (the first half of a
// piece, or a new maximum), O' (with its row-sum column) is rescaled by 2^(m_old - m_new)
// after the previous half's P.V has completed.
//
// Partial pages: slots past a page's valid count hold K = V = 0 (the append and compaction
// kernels write zeros there); pages past the end of the list are read as zeros. Such slots
// must take no weight. With bf16 storage S carries the mask itself: one more K=16 MMA per
// S tile adds 1 x bias, where the A operand is a TMEM block holding 1 in each row's first
// element and the B operand a per-stage, per-half shared-memory block (64 slots x 16 bf16,
// 32-byte swizzle) holding -2^100 for masked slots and 0 elsewhere. The TMA producer keeps
// these blocks current from the page entries it already loads, rewriting only the rows
// whose state changes (none between two full tiles). A masked score is then about
// -2^100 x the logit factor and its P rounds to 0 (2^-126 on the FMA-pipe path, as for a
// -inf score), so the softmax needs no page metadata. With E4M3 storage the per-page logit
// factors can be tiny, so the softmax sets those scores to -inf from the stage metadata.
//
// E4M3 storage ("XStreamVGGT" abstract: KV cache quantisation; codes with one absmax scale
// per (page, head), or per K channel and V token with the dimension-adaptive scales). The
// tensor cores multiply f16 operands (kind::f16 takes one type for A and B), so the CTA has a
// fourth warpgroup (512 threads): the TMA producer loads each KV tile's codes into a 3-stage
// code ring, and warps 12-15, one per sub-partition, each widen a quarter of the tile (32
// rows of K and V) into the 4-stage f16 operand ring with the exact E4M3 -> f16 conversion.
// K codes stay unscaled: the page's K scale multiplies the logit factor of the page's 16
// columns in the softmax. V codes are multiplied by the page's V scale over the piece's V
// reference (the largest V scale of its pages, which keeps every product in f16 range) and
// the epilogue multiplies O by that reference; this rounding of V to f16 (relative 2^-11)
// is the only extra rounding of an operand. Each Q row is scaled into f16 by the power of
// two that brings its largest magnitude into [2^14, 2^15), the row's logit factor carrying
// the inverse. P is rounded to f16. The converters also write each tile's page metadata
// (valid slots, K scales, V reference) next to the stage, which the softmax reads after the
// stage's K barrier.
//
// Every barrier wait is bounded: on timeout the CTA records KVC_ERR_TIMEOUT in the error
// word, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kvc_attn_common.cuh"

namespace kvc {
namespace tc {
constexpr int kBM = 128;                      // query rows per query tile
constexpr int kQT = 2;                        // query tiles per CTA
constexpr int kBN = 128;                      // KV slots per TMA stage
constexpr int kBH = 64;                       // KV slots per S tile (half a stage)
constexpr int kHD = 64;                       // head dim (one 128-byte swizzle row)
constexpr int kStages = 5;
constexpr int kON = kHD + 16;                 // O' columns: O plus the row-sum block
constexpr int kTileBytes = kBN * kHD * 2;     // 16 KB (K or V tile)
constexpr int kHalfBytes = kBH * kHD * 2;     // 8 KB: rows of one half (a multiple of the 1 KB swizzle atom)
constexpr int kOnesBytes = kHalfBytes;        // bf16 ones: the row-sum block of the B operand of P.V
constexpr int kThreads = 384;                 // 3 warpgroups
constexpr int kRegsLow = 56, kRegsHigh = 224;  // after the split: 128 x 56 + 256 x 224 <= 384 x 168
constexpr int kTmemCols = 512;
// TMEM columns of query tile i, from 256 i: Q (bf16 pairs), the A operand of the mask
// product (8 columns: 1 in each row's first element), S buffers 0 and 1 (fp32; P as bf16
// pairs over the first 32 columns of its buffer), O' (fp32)
constexpr int kColQ = 0, kColQb = 32, kColS = 40, kColO = 168;
__host__ __device__ constexpr int col_base(int i) { return 256 * i; }
constexpr float kLog2PMax = 8.0f;             // a P above 2^8 moves the row's reference max
constexpr int kPolyPer8 = 2;                  // of every 8 column pairs, the 2^x on the FMA pipe
// bf16 storage: per stage and half, the B operand of the mask product (64 slots x 16 bf16,
// 32-byte rows: the slot's bias in its first element, 0 or kMaskBias)
constexpr int kBiasHalfBytes = kBH * 32;
constexpr uint16_t kMaskBias = 0xF180;        // bf16 -2^100
constexpr size_t kSmemBytes = 1024 + 2 * kStages * kTileBytes + kOnesBytes + kStages * 2 * kBiasHalfBytes + 512;
// E4M3 storage: a fourth warpgroup widens the codes of each KV tile into the f16 operand
// ring; the codes land by TMA in a ring of their own
constexpr int kThreads8 = 512;
constexpr int kStages8 = 4;                   // f16 operand stages
constexpr int kCodeStages = 3;                // code stages (K and V codes of one KV tile)
constexpr int kCodeTileBytes = kBN * kHD;     // 8 KB: one tensor's codes of a KV tile
constexpr int kRegsConv = 96, kRegsHigh8 = 176;  // 128 x 56 + 256 x 176 + 128 x 96 <= 512 x 128
constexpr int kMetaBytes = kStages8 * (8 + 8 + 1) * 4;   // per operand stage: the tile's page metadata
constexpr size_t kSmemBytes8 =
    1024 + 2 * kStages8 * kTileBytes + kOnesBytes + 2 * kCodeStages * kCodeTileBytes + kMetaBytes + 512;
// storage modes of the kernel
constexpr int kBf16 = 0, kE4m3 = 1, kE4m3Da = 2;   // bf16; E4M3 + page scales; + dimension-adaptive
}  // namespace tc

// ---- the FMA-pipe exponential
// 2^x for a pair: x clamped below at -126, x = n + f with n = rint(x) (the 1.5 * 2^23 shift)
// and f in [-0.5, 0.5]; 2^f = 1 + f (c1 + f (c2 + f c3)), a cubic fitted for this kernel by
// iteratively reweighted least squares on the relative error (at most 1.02e-4, against the
// 2^-9 of the bf16 rounding P takes next); 2^n is added to the exponent field. No upper
// clamp: the softmax only evaluates x = s*c - m <= 8 (the reference max m is at most 8
// below any score it weights).
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t exp2_fma_pair(uint64_t x2) {
  constexpr float kShift = 12582912.0f;       // 1.5 * 2^23
  float x0, x1;
  up2(x2, x0, x1);
  const uint64_t xc = pk2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = add2(xc, pk2(kShift, kShift));
  const uint64_t fr = sub2(xc, sub2(t, pk2(kShift, kShift)));
  uint64_t q = fma2(pk2(0.05500858277082443f, 0.05500858277082443f), fr,
                    pk2(0.24221037328243256f, 0.24221037328243256f));
  q = fma2(q, fr, pk2(0.6932829022407532f, 0.6932829022407532f));
  q = fma2(q, fr, pk2(1.0f, 1.0f));
  float q0, q1, t0, t1;
  up2(q, q0, q1);
  up2(t, t0, t1);
  return pk2(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
             __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// ---- E4M3 codes
// Two E4M3 codes (low byte first) as an f16 pair, exactly (every E4M3 value is an f16 value).
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

// One S tile of P for a row: pb[i] = pair of 2^(s*c - m) for columns 2i, 2i+1, rounded to
// nearest bf16 (or f16). c is the logit factor of the pair's group of N / 2 / NQ pairs
// (NQ = 1: one factor; for E4M3 storage one per page, which carries the page's K scale).
// Of every 8 pairs the last kPoly go to the FMA pipe and the others to the MUFU, and every
// pair is finished (exponent, packing) in one pass, so MUFU instructions are spread through
// the row's FMA and ALU work instead of queueing behind one another.
template <bool kF16, int N, int NQ>
__device__ __forceinline__ void tile_p(const uint32_t (&s)[N], const float (&cq)[NQ], float m,
                                       uint32_t (&pb)[N / 2]) {
  constexpr int kPoly = tc::kPolyPer8;
  constexpr int kPairsPerQ = N / 2 / NQ;
  const uint64_t nm2 = pk2(-m, -m);
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const uint64_t c2 = pk2(cq[i / kPairsPerQ], cq[i / kPairsPerQ]);
    const uint64_t x2 = fma2_pair(s[2 * i], s[2 * i + 1], c2, nm2);
    uint64_t y2;
    if ((i & 7) >= 8 - kPoly) {
      y2 = exp2_fma_pair(x2);
    } else {
      float x0, x1;
      up2(x2, x0, x1);
      y2 = pk2(ex2(x0), ex2(x1));
    }
    float y0, y1;
    up2(y2, y0, y1);
    pb[i] = kF16 ? pack_f16(y0, y1) : pack_bf16(y0, y1);
  }
}

// Largest of a row's 64 scores as a tree of 3-input max instructions (depth 4), so the
// row's maximum does not wait on one long dependent chain.
__device__ __forceinline__ float row_max64(const uint32_t (&s)[tc::kBH]) {
  float a[22];
#pragma unroll
  for (int i = 0; i < 21; ++i)
    a[i] = max3(__uint_as_float(s[3 * i]), __uint_as_float(s[3 * i + 1]), __uint_as_float(s[3 * i + 2]));
  a[21] = __uint_as_float(s[63]);
  float b[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) b[i] = max3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[7] = a[21];
  return max3(max3(b[0], b[1], b[2]), max3(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}
// Largest scaled score of a row with one logit factor per 16-slot page (E4M3 storage): the
// page's largest raw score times its factor (factors are positive).
__device__ __forceinline__ float row_max64_pages(const uint32_t (&s)[tc::kBH], const float (&cq)[4]) {
  float r = -INFINITY;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t* t = &s[16 * q];
    const float a = max3(__uint_as_float(t[0]), __uint_as_float(t[1]), __uint_as_float(t[2]));
    const float b = max3(__uint_as_float(t[3]), __uint_as_float(t[4]), __uint_as_float(t[5]));
    const float c = max3(__uint_as_float(t[6]), __uint_as_float(t[7]), __uint_as_float(t[8]));
    const float d = max3(__uint_as_float(t[9]), __uint_as_float(t[10]), __uint_as_float(t[11]));
    const float e = max3(__uint_as_float(t[12]), __uint_as_float(t[13]), __uint_as_float(t[14]));
    const float pm = max3(max3(a, b, c), max3(d, e, __uint_as_float(t[15])), -INFINITY);
    r = fmaxf(r, pm * cq[q]);
  }
  return r;
}

// Register split between warpgroups (every warp of a warpgroup executes the same one).
template <int N>
__device__ __forceinline__ void reg_dealloc() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void reg_alloc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// The schedule of one CTA: group g sweeps [g*R, min((g+1)*R, steps)) of the flattened
// (layer, head, KV tile) sequence (layer l's steps start at lt.l[l].pos0) for query-tile
// pair qp. next_piece() cuts the range at head (and so layer) boundaries.
struct Sweep {
  int pos, end, l;
};
__device__ __forceinline__ bool next_piece(Sweep& sw, const AttnLayers& lt, int H, int& l, int& h, int& t0,
                                           int& t1) {
  if (sw.pos >= sw.end) return false;
  while (sw.l + 1 < lt.n && sw.pos >= lt.l[sw.l + 1].pos0) ++sw.l;
  const int nt = lt.l[sw.l].n_tiles;
  const int rel = sw.pos - lt.l[sw.l].pos0;
  l = sw.l;
  h = rel / nt;
  t0 = rel - h * nt;
  t1 = min(nt, t0 + (sw.end - sw.pos));
  sw.pos += t1 - t0;
  return true;
}

// Epilogue of one warp's 32 query rows of a piece (O = oscale O' / l, oscale the V reference
// scale of E4M3 storage, else 1). Single-piece units store bf16 O directly; otherwise every piece stores its normalised partial and log2-sum-exp, counts
// itself on the warp's counter, and the piece that counts last merges. Only a group's
// first and last piece can belong to a unit of several pieces (the pieces between them are
// whole heads), so a partial lives in the slot of (its group, first or last piece of the
// group): a piece that starts where its group starts takes the first slot. The merge is
// O = sum_k 2^(lse_k - M) O_k / sum_k 2^(lse_k - M), M the largest lse, over the unit's
// pieces in order (its own from registers, the others through L2). Only warp-level
// synchronisation is used, so a warp that gave up on a wait cannot hold another here.
__device__ __forceinline__ void store_piece(const TcParams& p, const LayerAttn& la, int lay, int wg, int wq, int lane,
                                            int h, int qp, int g, const uint32_t (&o0)[32], const uint32_t (&o1)[32],
                                            float l, float m, float oscale) {
  using namespace tc;
  const int r = wq * 32 + lane;
  const int qtile = 2 * qp + wg;
  const int row = qtile * kBM + r;
  const float inv = oscale / l;
  const int n_tiles = la.n_tiles, R = p.tiles_per_split;
  const int g_first = (la.pos0 + h * n_tiles) / R;
  const int g_last = (la.pos0 + h * n_tiles + n_tiles - 1) / R;
  const int npieces = g_last - g_first + 1;
  const int hh = lay * p.H + h;                 // the unit's head among all layers' heads
  uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(la.o) +
                                        (static_cast<long long>(row) * p.out_heads + p.head0 + h) * kHD);
  if (npieces == 1) {
    if (row < p.T) {
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint32_t* src = v < 4 ? &o0[8 * v] : &o1[8 * (v - 4)];
        uint4 w;
        w.x = pack_bf16(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv);
        w.y = pack_bf16(__uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv);
        w.z = pack_bf16(__uint_as_float(src[4]) * inv, __uint_as_float(src[5]) * inv);
        w.w = pack_bf16(__uint_as_float(src[6]) * inv, __uint_as_float(src[7]) * inv);
        out[v] = w;
      }
    }
    return;
  }
  if (qtile >= p.q_tiles) return;           // the pair's second tile is past the queries
  // piece k of the unit is in group g_first + k; only the first can start inside its group
  const bool starts_inside = la.pos0 + h * n_tiles > g_first * R;
  auto slot_row = [&](int k) {
    const long long slot = 2LL * (g_first + k) + (k == 0 && starts_inside ? 1 : 0);
    return (slot * p.q_pairs + qp) * (kQT * kBM) + wg * kBM + r;
  };
  const int me = g - g_first;
  const float lse_me = m + __log2f(l);
  {
    float4* dst = reinterpret_cast<float4*>(p.part_o + slot_row(me) * kHD);
#pragma unroll
    for (int v = 0; v < 8; ++v)
      dst[v] = make_float4(__uint_as_float(o0[4 * v + 0]) * inv, __uint_as_float(o0[4 * v + 1]) * inv,
                           __uint_as_float(o0[4 * v + 2]) * inv, __uint_as_float(o0[4 * v + 3]) * inv);
#pragma unroll
    for (int v = 0; v < 8; ++v)
      dst[8 + v] = make_float4(__uint_as_float(o1[4 * v + 0]) * inv, __uint_as_float(o1[4 * v + 1]) * inv,
                               __uint_as_float(o1[4 * v + 2]) * inv, __uint_as_float(o1[4 * v + 3]) * inv);
    p.part_lse[slot_row(me)] = lse_me;
  }
  // threadfence-then-count: each partial is visible before its count
  __threadfence();
  __syncwarp();
  const int cidx = ((hh * p.q_tiles + qtile) << 2) + wq;
  int last = 0;
  if (lane == 0) last = atomicAdd(&p.split_cnt[cidx], 1) == npieces - 1;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  if (row < p.T) {
    // pieces in ascending order whichever piece merges, so the result does not depend on
    // which finished last (its own partial enters at its place, with the values it stored)
    float M = lse_me;
    for (int k = 0; k < npieces; ++k)
      if (k != me) M = fmaxf(M, __ldcg(p.part_lse + slot_row(k)));
    float acc[kHD];
#pragma unroll
    for (int d = 0; d < kHD; ++d) acc[d] = 0.f;
    float ws = 0.f;
    for (int k = 0; k < npieces; ++k) {
      if (k == me) {
        const float w = exp2f(lse_me - M);
        ws += w;
#pragma unroll
        for (int d = 0; d < 32; ++d) {
          acc[d] = fmaf(w, __uint_as_float(o0[d]) * inv, acc[d]);
          acc[32 + d] = fmaf(w, __uint_as_float(o1[d]) * inv, acc[32 + d]);
        }
        continue;
      }
      const float w = exp2f(__ldcg(p.part_lse + slot_row(k)) - M);
      ws += w;
      const float4* src = reinterpret_cast<const float4*>(p.part_o + slot_row(k) * kHD);
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        const float4 f = __ldcg(src + v);
        acc[4 * v + 0] = fmaf(w, f.x, acc[4 * v + 0]);
        acc[4 * v + 1] = fmaf(w, f.y, acc[4 * v + 1]);
        acc[4 * v + 2] = fmaf(w, f.z, acc[4 * v + 2]);
        acc[4 * v + 3] = fmaf(w, f.w, acc[4 * v + 3]);
      }
    }
    const float iw = 1.f / ws;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint4 w;
      w.x = pack_bf16(acc[8 * v + 0] * iw, acc[8 * v + 1] * iw);
      w.y = pack_bf16(acc[8 * v + 2] * iw, acc[8 * v + 3] * iw);
      w.z = pack_bf16(acc[8 * v + 4] * iw, acc[8 * v + 5] * iw);
      w.w = pack_bf16(acc[8 * v + 6] * iw, acc[8 * v + 7] * iw);
      out[v] = w;
    }
  }
  if (lane == 0) p.split_cnt[cidx] = 0;   // ready for the next launch
}

// kPrefetch (bf16 only): each piece's epilogue loads the next piece's Q rows before its
// last wait and stores them in TMEM right after reading O', so the next piece's S starts
// while this piece's outputs are stored; chosen for launches with many pieces per CTA.
template <int P, bool kPerHead, int kMode, bool kPrefetch = false>
__global__ void __launch_bounds__(kMode == tc::kBf16 ? tc::kThreads : tc::kThreads8, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                   const TcParams p, const __grid_constant__ AttnLayers lt) {
  griddep_wait();
  griddep_launch_dependents();
  using namespace tc;
  constexpr bool kF8 = kMode != kBf16;        // E4M3 codes, widened to f16 operands
  constexpr bool kDA = kMode == kE4m3Da;
  constexpr int kS = kF8 ? kStages8 : kStages;   // operand stages
  constexpr int kPPT = kBN / P;               // pages per KV tile (TMA stage)
  constexpr int kPPH = kBH / P;               // pages per half (S tile)
  static_assert(P == 16, "16-slot pages: a 64-slot half holds 4 of them");
  static_assert(!kF8 || !kPerHead, "E4M3 storage: one page list per layer");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* k_s = smem;                                   // [stage][128 rows][128 B]
  uint8_t* v_s = k_s + kS * kTileBytes;
  uint8_t* ones_s = v_s + kS * kTileBytes;               // after every V stage: a positive offset
  uint8_t* bias_s = ones_s + kOnesBytes;                 // bf16: [stage][half][64 slots][32 B]
  uint8_t* codes = bias_s + (kF8 ? 0 : kS * 2 * kBiasHalfBytes);   // E4M3: [code stage][K, V][128 rows][64 B]
  // E4M3, per operand stage (written by the converters with the tile's K, read by the
  // softmax): the valid slots and K scales of the tile's 8 pages, the piece's V reference
  int* meta_valid = reinterpret_cast<int*>(codes + (kF8 ? 2 * kCodeStages * kCodeTileBytes : 0));   // [kS][8]
  float* meta_ks = reinterpret_cast<float*>(meta_valid + (kF8 ? kS * 8 : 0));                       // [kS][8]
  float* meta_vref = meta_ks + (kF8 ? kS * 8 : 0);                                                  // [kS]
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta_vref + (kF8 ? kS : 0));
  uint64_t* k_full = bars;
  uint64_t* v_full = k_full + kS;
  uint64_t* kv_empty = v_full + kS;           // both issuers done with the stage
  // Per query tile i ([i], or [2 i + b] for S buffer b). Every wait is on a phase at most
  // one ahead of the last one the waiter saw complete (a parity wait cannot tell two
  // phases apart), which is why P and the piece's end have their own barriers:
  uint64_t* q_ready = kv_empty + kS;          // Q in TMEM (the 4 softmax warps)
  uint64_t* s_full = q_ready + 2;             // S buffer computed
  uint64_t* p_full = s_full + 4;              // P in S buffer b (the 4 softmax warps)
  uint64_t* pv_done = p_full + 4;             // a P.V product complete (rescale: S of half u
                                              // complete implies P.V of half u - 2 complete)
  uint64_t* o_full = pv_done + 2;             // the piece's last P.V complete
  uint64_t* o_free = o_full + 2;              // O' read by the epilogue (the 4 softmax warps)
  uint64_t* mma_final = o_free + 2;
  uint64_t* code_full = mma_final + 2;        // E4M3: a code stage landed
  uint64_t* code_empty = code_full + kCodeStages;   // E4M3: a code stage read (the 4 converters)
  uint64_t* vref_bar = code_empty + kCodeStages;    // E4M3: [piece & 1] partial V maxima written
  float* vref_part = reinterpret_cast<float*>(vref_bar + 2);   // [piece & 1][converter]
  uint64_t* bias_pack = reinterpret_cast<uint64_t*>(vref_part + 8);   // bf16: [stage] valid slots its mask rows hold
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bias_pack + kS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qp = blockIdx.x % p.q_pairs;
  const int g = blockIdx.x / p.q_pairs;
  const int HT = p.total_tiles;                 // steps of all layers
  const int R = p.tiles_per_split;
  const Sweep sweep0{min(g * R, HT), min(g * R + R, HT), 0};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kS; ++i) {
      mbar_init(&k_full[i], kF8 ? 4 : 1);       // E4M3: the 4 converter warps
      mbar_init(&v_full[i], kF8 ? 4 : 1);
      mbar_init(&kv_empty[i], kQT);
    }
    for (int i = 0; i < kQT; ++i) {
      mbar_init(&q_ready[i], 4);
      mbar_init(&s_full[2 * i], 1);
      mbar_init(&s_full[2 * i + 1], 1);
      mbar_init(&p_full[2 * i], 4);
      mbar_init(&p_full[2 * i + 1], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 4);
      mbar_init(&mma_final[i], 1);
    }
    if (kF8) {
      for (int i = 0; i < kCodeStages; ++i) {
        mbar_init(&code_full[i], 1);
        mbar_init(&code_empty[i], 4);
      }
      mbar_init(&vref_bar[0], 4);
      mbar_init(&vref_bar[1], 4);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  // the constant ones block (every element 1.0, so the swizzle does not matter), made
  // visible to the tensor core's operand reads
  const uint32_t one2 = kF8 ? 0x3c003c00u : 0x3f803f80u;
  for (int i = threadIdx.x; i < kOnesBytes / 16; i += (kF8 ? kThreads8 : kThreads))
    reinterpret_cast<uint4*>(ones_s)[i] = make_uint4(one2, one2, one2, one2);
  if (!kF8) {
    // every slot of every stage starts unmasked (all pages full)
    for (int i = threadIdx.x; i < kS * 2 * kBiasHalfBytes / 16; i += kThreads)
      reinterpret_cast<uint4*>(bias_s)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < kS; i += kThreads) {
      uint64_t full = 0;                          // every page P valid slots, packed 5 bits a page
      for (int q = 0; q < kPPT; ++q) full |= static_cast<uint64_t>(P) << (5 * q);
      bias_pack[i] = full;
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0) {
    reg_dealloc<kRegsLow>();
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      // bf16: the K and V tiles into the operand ring; E4M3: their codes into the code ring
      constexpr int kRing = kF8 ? kCodeStages : kS;
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      int last[kRing];
#pragma unroll
      for (int i = 0; i < kRing; ++i) last[i] = -1;
      int jg = 0;
      bool ok = true;
      Sweep sw = sweep0;
      int lay, h, t0, t1;
      while (ok && next_piece(sw, lt, p.H, lay, h, t0, t1)) {
        const LayerAttn& la = lt.l[lay];
        const long long hp = kPerHead ? static_cast<long long>(h) * p.head_pages : 0;
        const Entry* ent = kPerHead ? la.entries + hp : la.entries;
        const int n_pages = la.n_pages;
        const long long page_base = la.page_base;
        // physical page of each page of the next tile (past the list: -1) and, packed 5 bits
        // a page, their valid slots (past the list: 0)
        int phys_next[kPPT];
        uint64_t vpack_next = 0;
#pragma unroll
        for (int q = 0; q < kPPT; ++q) {
          const int idx = t0 * kPPT + q;
          const int4 en = idx < n_pages ? __ldg(&ent[idx]) : make_int4(-1, 0, 0, 0);
          phys_next[q] = en.x;
          vpack_next |= static_cast<uint64_t>(min(max(en.w, 0), P)) << (5 * q);
        }
        for (int t = t0; t < t1; ++t, ++jg) {
          const int st = jg % kRing;
          int row[kPPT];
          const uint64_t vpack = vpack_next;
#pragma unroll
          for (int q = 0; q < kPPT; ++q) {
            if (kPerHead)
              row[q] = phys_next[q] >= 0 ? static_cast<int>((page_base + hp + phys_next[q]) * P) : p.pool_rows;
            else
              row[q] = phys_next[q] >= 0 ? static_cast<int>(((page_base + phys_next[q]) * p.H + h) * P) : p.pool_rows;
          }
          if (t + 1 < t1) {
            vpack_next = 0;
#pragma unroll
            for (int q = 0; q < kPPT; ++q) {
              const int idx = (t + 1) * kPPT + q;
              const int4 en = idx < n_pages ? __ldg(&ent[idx]) : make_int4(-1, 0, 0, 0);
              phys_next[q] = en.x;
              vpack_next |= static_cast<uint64_t>(min(max(en.w, 0), P)) << (5 * q);
            }
          }
          uint64_t* free_bar = kF8 ? &code_empty[st] : &kv_empty[st];
          if (jg >= kRing && !mbar_wait_bounded(free_bar, ((jg / kRing) - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          if (kF8) {
            uint8_t* cb = codes + st * 2 * kCodeTileBytes;
            mbar_arrive_expect_tx(&code_full[st], 2 * kCodeTileBytes);
#pragma unroll
            for (int q = 0; q < kPPT; ++q) tma_load_2d(cb + q * P * kHD, &tmap_k, &code_full[st], 0, row[q]);
#pragma unroll
            for (int q = 0; q < kPPT; ++q)
              tma_load_2d(cb + kCodeTileBytes + q * P * kHD, &tmap_v, &code_full[st], 0, row[q]);
          } else {
            // the stage's mask rows: slot j of page q is masked (bias kMaskBias) iff j >= its
            // valid count. The stage remembers the counts its rows hold (packed as the tile's
            // are), and only rows whose state changes are written: nothing for a full tile
            // after a full tile. Both 16-byte halves of a row start with the bias, so the
            // 32-byte swizzle cannot move it out of the element the product reads.
            const uint64_t held = bias_pack[st];
            if (vpack != held) {
              for (int q = 0; q < kPPT; ++q) {
                const int vo = static_cast<int>((held >> (5 * q)) & 31u);
                const int vn = static_cast<int>((vpack >> (5 * q)) & 31u);
                if (vo != vn) {
                  uint8_t* rows = bias_s + (st * 2 + q / kPPH) * kBiasHalfBytes + (q % kPPH) * P * 32;
                  const uint16_t val = vn < vo ? kMaskBias : 0;
                  for (int j = min(vo, vn); j < max(vo, vn); ++j) {
                    *reinterpret_cast<uint16_t*>(rows + j * 32) = val;
                    *reinterpret_cast<uint16_t*>(rows + j * 32 + 16) = val;
                  }
                }
              }
              bias_pack[st] = vpack;
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            mbar_arrive_expect_tx(&k_full[st], kTileBytes);
#pragma unroll
            for (int q = 0; q < kPPT; ++q)
              tma_load_2d(k_s + st * kTileBytes + q * P * 128, &tmap_k, &k_full[st], 0, row[q]);
            mbar_arrive_expect_tx(&v_full[st], kTileBytes);
#pragma unroll
            for (int q = 0; q < kPPT; ++q)
              tma_load_2d(v_s + st * kTileBytes + q * P * 128, &tmap_v, &v_full[st], 0, row[q]);
          }
          last[st] = jg;
        }
      }
      // drain: every copy this CTA issued has landed before shared memory is released
#pragma unroll
      for (int i = 0; i < kRing; ++i) {
        if (last[i] >= 0) {
          if (kF8) {
            mbar_wait_drain(&code_full[i], (last[i] / kRing) & 1, p.err);
          } else {
            mbar_wait_drain(&k_full[i], (last[i] / kRing) & 1, p.err);
            mbar_wait_drain(&v_full[i], (last[i] / kRing) & 1, p.err);
          }
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    reg_dealloc<kRegsLow>();
    // ------------------------------------------------------------------ MMA issuer of query tile i
    // Halves are numbered globally (uu = 2 * KV tile + half); half uu uses S buffer uu & 1.
    const int i = warp - 1;
    const uint32_t fmt = kF8 ? 0u : 1u;         // operand type: f16 or bf16
    const uint32_t idesc_s = idesc_f16kind(fmt, kBM, kBH, 0, 0);
    const uint32_t idesc_o = idesc_f16kind(fmt, kBM, kON, 0, 1);
    const uint32_t tb = tmem + col_base(i);
    const uint32_t k_addr = smem_u32(k_s), v_addr = smem_u32(v_s), ones_addr = smem_u32(ones_s);
    const uint32_t bias_addr = smem_u32(bias_s);
    const bool leader = elect_one();
    int ub = 0, pc = 0;                           // first half of the piece; pieces done
    // S of half uu (u: its index in the piece) into buffer uu & 1. Issued after the P.V
    // product of half uu - 2 (which read its P from this buffer): this issuer's MMAs run in
    // order, so that product has read P before S overwrites it.
    auto issue_s = [&](int uu, int u) -> bool {
      const int jj = uu >> 1, hb = uu & 1, st = jj % kS;
      bool w = true;
      if (hb == 0) w = mbar_wait_bounded(&k_full[st], (jj / kS) & 1, abort_flag, p.err);
      if (u == 0) w = w && mbar_wait_bounded(&q_ready[i], pc & 1, abort_flag, p.err);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      if (leader) {
        const uint32_t kb = k_addr + st * kTileBytes + hb * kHalfBytes;
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk)
          mma_ts(tb + kColS + hb * kBH, tb + kColQ + kk * 8, sw128_desc(kb + kk * 32, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        // bf16: + 1 x the slots' bias (0, or -2^100 for slots past a page's valid count)
        if (!kF8) mma_ts(tb + kColS + hb * kBH, tb + kColQb, sw32_desc(bias_addr + (st * 2 + hb) * kBiasHalfBytes, 256),
                         idesc_s, 1u);
        mma_commit(&s_full[2 * i + hb]);
      }
      __syncwarp();
      return true;
    };
    // O' += P [V | 1] for half uu; the first half of a piece overwrites O' once the previous
    // piece's epilogue has read it
    auto issue_pv = [&](int uu, int u, bool last) -> bool {
      const int jj = uu >> 1, hb = uu & 1, st = jj % kS;
      bool w = mbar_wait_bounded(&p_full[2 * i + hb], jj & 1, abort_flag, p.err);
      if (hb == 0) w = w && mbar_wait_bounded(&v_full[st], (jj / kS) & 1, abort_flag, p.err);
      if (u == 0 && pc > 0) w = w && mbar_wait_bounded(&o_free[i], (pc - 1) & 1, abort_flag, p.err);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      if (leader) {
        const uint32_t vb = v_addr + st * kTileBytes + hb * kHalfBytes;
        const uint32_t lbo = ones_addr - vb;      // the N block after V: the ones
#pragma unroll
        for (int kk = 0; kk < kBH / 16; ++kk)
          mma_ts(tb + kColO, tb + kColS + hb * kBH + kk * 8, sw128_desc(vb + kk * 2048, lbo, 1024), idesc_o,
                 (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&pv_done[i]);
        if (last) mma_commit(&o_full[i]);
      }
      __syncwarp();
      return true;
    };
    // the stage of half uu's KV tile is released after its second half's P.V (committed
    // after the next S, off the path from P.V to that S)
    auto release = [&](int uu) {
      if (leader && (uu & 1)) mma_commit(&kv_empty[(uu >> 1) % kS]);
      __syncwarp();
    };
    bool ok = true;
    Sweep sw = sweep0;
    int lay, h, t0, t1;
    while (ok && next_piece(sw, lt, p.H, lay, h, t0, t1)) {
      const int nh = 2 * (t1 - t0);
      ok = issue_s(ub, 0) && issue_s(ub + 1, 1);
      for (int u = 0; ok && u < nh; ++u) {
        if (!issue_pv(ub + u, u, u + 1 == nh)) ok = false;
        else if (u + 2 < nh && !issue_s(ub + u + 2, u + 2)) ok = false;
        else release(ub + u);
      }
      ub += nh;
      ++pc;
    }
    if (leader) mma_commit(&mma_final[i]);
    __syncwarp();
    mbar_wait_drain(&mma_final[i], 0, p.err);
  } else if (warp < 4) {
    reg_dealloc<kRegsLow>();                       // warp 3 only gives up registers
  } else if (!kF8 || warp < 12) {
    reg_alloc<kF8 ? kRegsHigh8 : kRegsHigh>();
    // ------------------------------------------------------------------ softmax warps
    const int wg = (warp - 4) >> 2;               // query tile of the pair
    const int wq = warp & 3;                      // TMEM lane quadrant this warp may access
    const uint32_t tb = tmem + col_base(wg) + (static_cast<uint32_t>(wq * 32) << 16);
    const float c = p.scale_log2;
    const int row = (2 * qp + wg) * kBM + wq * 32 + lane;
    int ub = 0, pc = 0;
    bool ok = true;
    [[maybe_unused]] bool q_stored = false;   // kPrefetch: this piece's Q is already in TMEM
    Sweep sw = sweep0;
    int lay, h, t0, t1;
    while (ok && next_piece(sw, lt, p.H, lay, h, t0, t1)) {
      const int nh = 2 * (t1 - t0);
      const LayerAttn& la = lt.l[lay];
      float row_fac = 1.f;       // E4M3: 2^-e of the query row's scaling into f16
      bool have_q = false;
      if constexpr (kPrefetch) have_q = q_stored;
      if (!have_q) {
        // this row of Q (zeros past the last query) into TMEM, the A operand of S; the S
        // products of the previous piece, its only readers, have completed (their S was read)
        uint32_t qv[32];
        if (row < p.T) {
          const uint4* src =
              reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(la.q) +
                                             (static_cast<long long>(row) * p.out_heads + p.head0 + h) * kHD);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 w = __ldg(src + v);
            qv[4 * v] = w.x;
            qv[4 * v + 1] = w.y;
            qv[4 * v + 2] = w.z;
            qv[4 * v + 3] = w.w;
          }
          if (kF8) {
            // f16 operands: the row is scaled by the power of two 2^e that brings its largest
            // magnitude into [2^14, 2^15), so no finite bf16 query overflows f16 and small
            // rows keep their bits; the row's logit factor carries 2^-e, which makes the
            // scaling exact (e is clamped to [-120, 100] so that factor stays a normal float)
            float qmax = 0.f;
#pragma unroll
            for (int v = 0; v < 32; ++v) qmax = max3(qmax, fabsf(bf16lo(qv[v])), fabsf(bf16hi(qv[v])));
            int e = 0;
            if (qmax > 0.f) {
              int ex;
              frexpf(qmax, &ex);                  // qmax in [2^(ex-1), 2^ex)
              e = min(100, max(-120, 15 - ex));
            }
            row_fac = ldexpf(1.f, -e);
#pragma unroll
            for (int v = 0; v < 32; ++v) qv[v] = pack_f16(ldexpf(bf16lo(qv[v]), e), ldexpf(bf16hi(qv[v]), e));
          }
        } else {
#pragma unroll
          for (int v = 0; v < 32; ++v) qv[v] = 0u;
        }
        tmem_st32(tb + kColQ, qv);
        if (!kF8) {
          // A operand of the mask product: 1 in the row's first element
          const uint32_t qb[8] = {0x3f80u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          tmem_st8(tb + kColQb, qb);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_ready[wg]);
      }
      if constexpr (kPrefetch) q_stored = false;
      float m = -INFINITY;       // reference max (log2 domain) of the row
      float vref = 1.f;          // E4M3: the piece's V reference
      for (int u = 0; u < nh; ++u) {
        const int uu = ub + u, hb = uu & 1, jj = uu >> 1;
        int vcur[kPPH];
        float cq[kF8 ? kPPH : 1];                 // logit factor (per page for E4M3)
        bool partial = false;
        if constexpr (kF8) {
          // the half's 4 pages from the stage's metadata, which the converters wrote before
          // they released the tile's K (the wait makes their writes visible; the stage is
          // not refilled before this tile's P.V products, which need this half's P)
          const int st = jj % kS;
          if (hb == 0 &&
              !__all_sync(0xffffffffu, mbar_wait_bounded(&k_full[st], (jj / kS) & 1, abort_flag, p.err))) {
            ok = false;
            break;
          }
          const int4 v4 = *reinterpret_cast<const int4*>(&meta_valid[st * 8 + 4 * hb]);
          const float4 ks4 = *reinterpret_cast<const float4*>(&meta_ks[st * 8 + 4 * hb]);
          vref = meta_vref[st];
          vcur[0] = v4.x;
          vcur[1] = v4.y;
          vcur[2] = v4.z;
          vcur[3] = v4.w;
          partial = min(min(v4.x, v4.y), min(v4.z, v4.w)) < P;
          // a zero-scale page (all-zero K, or past the list) gets a tiny positive factor:
          // its valid scores are 0 either way, and its masked -inf scores stay -inf
          const float crow = c * row_fac;
          cq[0] = fmaxf(crow * ks4.x, 1e-30f);
          cq[1] = fmaxf(crow * ks4.y, 1e-30f);
          cq[2] = fmaxf(crow * ks4.z, 1e-30f);
          cq[3] = fmaxf(crow * ks4.w, 1e-30f);
        } else {
          // bf16: slots past a page's valid count were masked inside S by the mask product
          cq[0] = c;
        }
        uint32_t s[kBH];
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[2 * wg + hb], jj & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_ld32(tb + kColS + hb * kBH, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld32(tb + kColS + hb * kBH + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld_wait();
        if (kF8 && partial) {
          // E4M3: slots past a page's valid count (and pages past the list end) take no weight
#pragma unroll
          for (int cc = 0; cc < kBH; ++cc)
            if ((cc % P) >= vcur[cc / P]) s[cc] = __float_as_uint(-INFINITY);
        }
        // exact fp32 max of the half; the row's reference max moves when some P would exceed
        // 2^8 (or on the first half of a piece); O' is then rescaled by 2^(m_old - m_new)
        // once the previous half's P.V has completed
        float tm;
        if constexpr (kF8) tm = row_max64_pages(s, cq);
        else tm = row_max64(s) * c;
        const bool move = (u == 0) || tm > m + kLog2PMax;
        if (__any_sync(0xffffffffu, move)) {
          const float m_new = move ? (tm == -INFINITY ? (m == -INFINITY ? 0.f : m) : tm) : m;
          const bool resc = move && u > 0 && m_new != m;
          if (__any_sync(0xffffffffu, resc)) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&pv_done[wg], (uu - 1) & 1, abort_flag, p.err))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float f = resc ? ex2(m - m_new) : 1.0f;
#pragma unroll
            for (int q4 = 0; q4 < kON / 16; ++q4) {
              uint32_t oc[16];
              tmem_ld16(tb + kColO + q4 * 16, oc);
              tmem_ld_wait();
#pragma unroll
              for (int d = 0; d < 16; ++d) oc[d] = __float_as_uint(__uint_as_float(oc[d]) * f);
              tmem_st16(tb + kColO + q4 * 16, oc);
            }
          }
          m = m_new;
        }
        uint32_t pb[kBH / 2];
        tile_p<kF8>(s, cq, m, pb);
        // P over the first 32 columns of this half's S buffer, whose S is in registers; the
        // buffer is not written again before this P's product has read it (tcgen05.ld/st are
        // .sync.aligned: every branch around them is warp-uniform)
        tmem_st32(tb + kColS + hb * kBH, pb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[2 * wg + hb]);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      [[maybe_unused]] bool has_next = false;
      [[maybe_unused]] uint32_t qn[32];
      if constexpr (kPrefetch && !kF8) {
        Sweep swn = sw;
        int layn, hn, t0n, t1n;
        has_next = next_piece(swn, lt, p.H, layn, hn, t0n, t1n);
        if (has_next) {
          if (row < p.T) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(lt.l[layn].q) +
                                                              (static_cast<long long>(row) * p.out_heads + p.head0 + hn) * kHD);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const uint4 w = __ldg(src + v);
              qn[4 * v] = w.x;
              qn[4 * v + 1] = w.y;
              qn[4 * v + 2] = w.z;
              qn[4 * v + 3] = w.w;
            }
          } else {
#pragma unroll
            for (int v = 0; v < 32; ++v) qn[v] = 0u;
          }
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&o_full[wg], pc & 1, abort_flag, p.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32(tb + kColO, o0);
      tmem_ld32(tb + kColO + 32, o1);
      const uint32_t lsum = tmem_ld1(tb + kColO + 64);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[wg]);
      if constexpr (kPrefetch && !kF8) {
        if (has_next) {
          // the next piece's Q: every S product of this piece has completed (its S was read)
          tmem_st32(tb + kColQ, qn);
          const uint32_t qb[8] = {0x3f80u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          tmem_st8(tb + kColQb, qb);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&q_ready[wg]);
          q_stored = true;
        }
      }
      // E4M3: V was divided by the piece's V reference
      store_piece(p, la, lay, wg, wq, lane, h, qp, g, o0, o1, __uint_as_float(lsum), m, kF8 ? vref : 1.f);
      ub += nh;
      ++pc;
    }
  } else if constexpr (kF8) {
    reg_dealloc<kRegsConv>();
    // ------------------------------------------------------------------ E4M3 converters
    // Converter cw widens rows [32 cw, 32 cw + 32) of every KV tile (pages 2 cw and 2 cw + 1):
    // lane (r0, c0) = (lane >> 3, lane & 7) takes rows 32 cw + r0 + 4 i (i < 8), 8-code chunk
    // c0, stored at chunk c0 ^ (row & 7) of the 128-byte-swizzled f16 row. K codes stay
    // unscaled (the page's K scale is in the softmax's logit factor); V codes are multiplied
    // by the page's V scale over the piece's V reference (the largest V scale of its pages).
    // Dimension-adaptive scales: K also by its channel scale over the page's K scale, V by its
    // token scale instead of the page's.
    const int cw = warp - 12;
    const int r0 = lane >> 3, c0 = lane & 7;
    const int src_off = (32 * cw + r0) * kHD + 8 * c0;
    const int dst_even = (32 * cw + r0) * 128 + ((c0 ^ r0) << 4);
    const int dst_odd = (32 * cw + r0) * 128 + ((c0 ^ r0 ^ 4) << 4);
    int jg = 0, pc = 0;
    bool ok = true;
    Sweep sw = sweep0;
    int lay, h, t0, t1;
    while (ok && next_piece(sw, lt, p.H, lay, h, t0, t1)) {
      const LayerAttn& la = lt.l[lay];
      const Entry* ent = la.entries;
      const int n_pages = la.n_pages;
      const long long page_base = la.page_base;
      // V reference of the piece: each converter takes a quarter of its pages, 16 loads in
      // flight per lane, and the four partial maxima meet in shared memory
      float mv = 0.f;
      {
        const int i0 = t0 * kPPT, i1 = min(t1 * kPPT, n_pages);
        const int span = (i1 - i0 + 3) / 4;
        const int a0 = i0 + cw * span, a1 = min(i1, a0 + span);
        for (int base = a0; base < a1; base += 32 * 16) {
          int ph[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int idx = base + 32 * k + lane;
            ph[k] = idx < a1 ? __ldg(&ent[idx].x) : -1;
          }
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (ph[k] >= 0) mv = fmaxf(mv, __ldg(&p.v_scale[(page_base + ph[k]) * p.H + h]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
        const int b = pc & 1;
        if (lane == 0) {
          vref_part[4 * b + cw] = mv;
          mbar_arrive(&vref_bar[b]);
        }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&vref_bar[b], (pc >> 1) & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        mv = fmaxf(fmaxf(vref_part[4 * b], vref_part[4 * b + 1]), fmaxf(vref_part[4 * b + 2], vref_part[4 * b + 3]));
        if (mv == 0.f) mv = 1.f;                  // all-zero pages: any reference works
      }
      const float iv = 1.f / mv;
      // this converter's two pages of tile t (every lane loads both): physical page and
      // valid slots, one tile ahead
      auto entry_of = [&](int t, int gg) -> int2 {
        const int idx = t * kPPT + 2 * cw + gg;
        if (t < t1 && idx < n_pages) {
          const int4 e = __ldg(&ent[idx]);
          return make_int2(e.x, e.w);
        }
        return make_int2(-1, 0);
      };
      int2 en_next[2] = {entry_of(t0, 0), entry_of(t0, 1)};
      for (int t = t0; ok && t < t1; ++t, ++jg) {
        const int st = jg % kS, cs = jg % kCodeStages;
        const int ph[2] = {en_next[0].x, en_next[1].x};
        const int nv[2] = {en_next[0].y, en_next[1].y};
        en_next[0] = entry_of(t + 1, 0);
        en_next[1] = entry_of(t + 1, 1);
        // f16 factors of this tile: vr[gg] per page, or per row (and per K chunk) for the
        // dimension-adaptive scales; the pages' K scales for the softmax
        uint32_t vr[kDA ? 8 : 2];
        uint32_t kf[kDA ? 2 : 1][4];
        float ksp[2];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const long long base = (page_base + ph[gg]) * p.H + h;
          ksp[gg] = ph[gg] >= 0 ? __ldg(&p.k_scale[base]) : 0.f;
          if (!kDA) {
            const float vs = ph[gg] >= 0 ? __ldg(&p.v_scale[base]) : 0.f;
            vr[gg] = pack_f16(vs * iv, vs * iv);
          } else {
            float kc[8], vt[4];
            const float ks = ksp[gg];
#pragma unroll
            for (int e = 0; e < 8; ++e) kc[e] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) vt[e] = 0.f;
            if (ph[gg] >= 0) {
              const float4 a = __ldg(reinterpret_cast<const float4*>(p.k_chan + base * kHD + 8 * c0));
              const float4 b = __ldg(reinterpret_cast<const float4*>(p.k_chan + base * kHD + 8 * c0) + 1);
              kc[0] = a.x; kc[1] = a.y; kc[2] = a.z; kc[3] = a.w;
              kc[4] = b.x; kc[5] = b.y; kc[6] = b.z; kc[7] = b.w;
#pragma unroll
              for (int e = 0; e < 4; ++e) vt[e] = __ldg(&p.v_tok[base * P + r0 + 4 * e]);
            }
            const float inv = ks > 0.f ? 1.f / ks : 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) kf[kDA ? gg : 0][e] = pack_f16(kc[2 * e] * inv, kc[2 * e + 1] * inv);
#pragma unroll
            for (int e = 0; e < 4; ++e) vr[kDA ? 4 * gg + e : 0] = pack_f16(vt[e] * iv, vt[e] * iv);
          }
        }
        // the operand stage is free once both query tiles' products of tile jg - kS are done
        if (jg >= kS &&
            !__all_sync(0xffffffffu, mbar_wait_bounded(&kv_empty[st], ((jg / kS) - 1) & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&code_full[cs], (jg / kCodeStages) & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          meta_ks[st * 8 + 2 * cw] = ksp[0];
          meta_ks[st * 8 + 2 * cw + 1] = ksp[1];
          meta_valid[st * 8 + 2 * cw] = nv[0];
          meta_valid[st * 8 + 2 * cw + 1] = nv[1];
          if (cw == 0) meta_vref[st] = mv;
        }
        const uint8_t* ksrc = codes + cs * 2 * kCodeTileBytes + src_off;
        const uint8_t* vsrc = ksrc + kCodeTileBytes;
        uint8_t* kdst = k_s + st * kTileBytes;
        uint8_t* vdst = v_s + st * kTileBytes;
#pragma unroll
        for (int i = 0; i < 8; ++i) {             // row 32 cw + r0 + 4 i: page i / 4 of the two
          const uint2 kc = *reinterpret_cast<const uint2*>(ksrc + i * 4 * kHD);
          uint4 ko;
          ko.x = f16x2_of_e4m3x2(kc.x);
          ko.y = f16x2_of_e4m3x2(kc.x >> 16);
          ko.z = f16x2_of_e4m3x2(kc.y);
          ko.w = f16x2_of_e4m3x2(kc.y >> 16);
          if (kDA) {
            ko.x = hmul2(ko.x, kf[kDA ? i >> 2 : 0][0]);
            ko.y = hmul2(ko.y, kf[kDA ? i >> 2 : 0][1]);
            ko.z = hmul2(ko.z, kf[kDA ? i >> 2 : 0][2]);
            ko.w = hmul2(ko.w, kf[kDA ? i >> 2 : 0][3]);
          }
          *reinterpret_cast<uint4*>(kdst + i * 512 + ((i & 1) ? dst_odd : dst_even)) = ko;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&k_full[st]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint2 vc = *reinterpret_cast<const uint2*>(vsrc + i * 4 * kHD);
          const uint32_t f = vr[kDA ? i : i >> 2];
          uint4 vo;
          vo.x = hmul2(f16x2_of_e4m3x2(vc.x), f);
          vo.y = hmul2(f16x2_of_e4m3x2(vc.x >> 16), f);
          vo.z = hmul2(f16x2_of_e4m3x2(vc.y), f);
          vo.w = hmul2(f16x2_of_e4m3x2(vc.y >> 16), f);
          *reinterpret_cast<uint4*>(vdst + i * 512 + ((i & 1) ? dst_odd : dst_even)) = vo;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&v_full[st]);
          mbar_arrive(&code_empty[cs]);
        }
      }
      ++pc;
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

// Queries [T][H][64] bf16 as a 3-D map; one box is 128 rows of one head (128-byte swizzle),
// rows past T read as zeros.
// Schedule of the bf16 kernel over one or more layers. R = steps per group; groups of
// q_pairs CTAs. Automatic: as many groups as fill the SMs (one CTA each); with
// kv_splits = s > 0, about s pieces per head of the largest layer. Split units need
// 2 x groups x q_pairs x 2 partial tiles (a group's first and last piece); when more than
// part_tiles, R doubles (fewer groups) until they fit, unless `strict`, in which case the
// plan fails.
bool plan_attn_bf16(int T, int H, const int* n_pages, int n_layers, int P, int sm_count, int kv_splits,
                    size_t part_tiles, bool strict, AttnPlan* out, int* n_tiles, int* pos0) {
  if (T < 1 || H < 1 || n_layers < 1 || P < 1 || sm_count < 1) return false;
  AttnPlan a{};
  a.q_tiles = (T + tc::kBM - 1) / tc::kBM;
  a.q_pairs = (a.q_tiles + 1) / 2;
  long long steps = 0;
  int max_nt = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (n_pages[l] < 1) return false;
    n_tiles[l] = static_cast<int>((static_cast<long long>(n_pages[l]) * P + tc::kBN - 1) / tc::kBN);
    pos0[l] = static_cast<int>(steps);
    steps += static_cast<long long>(H) * n_tiles[l];
    max_nt = std::max(max_nt, n_tiles[l]);
    if (steps > (1LL << 30)) return false;
  }
  a.steps = steps;
  long long R;
  if (kv_splits > 0) {
    R = (max_nt + kv_splits - 1) / kv_splits;
  } else {
    const long long groups = std::max(1, sm_count / a.q_pairs);
    R = (steps + groups - 1) / groups;
  }
  if (R < 1) R = 1;
  for (;;) {
    const long long groups = (steps + R - 1) / R;
    int max_pieces = 1;
    for (int l = 0; l < n_layers; ++l)
      for (int h = 0; h < H; ++h) {
        const long long s0 = pos0[l] + static_cast<long long>(h) * n_tiles[l];
        max_pieces = std::max(max_pieces, static_cast<int>((s0 + n_tiles[l] - 1) / R - s0 / R + 1));
      }
    const long long need = max_pieces > 1 ? 2 * groups * a.q_pairs * tc::kQT : 0;
    if (need <= static_cast<long long>(part_tiles) || strict) {
      if (need > static_cast<long long>(part_tiles)) return false;
      a.R = static_cast<int>(R);
      a.groups = static_cast<int>(groups);
      a.max_pieces = max_pieces;
      a.grid = a.groups * a.q_pairs;
      a.part_tiles = static_cast<size_t>(need);
      *out = a;
      return true;
    }
    R *= 2;
  }
}

namespace {
template <int kMode>
cudaError_t launch_mode(cudaStream_t s, bool per_head, bool prefetch, dim3 grid, const TcParams& prm,
                        const TcAttnArgs& a, const AttnLayers& lt) {
  constexpr bool kF8 = kMode != tc::kBf16;
  const int threads = kF8 ? tc::kThreads8 : tc::kThreads;
  const size_t smem = kF8 ? tc::kSmemBytes8 : tc::kSmemBytes;
  if constexpr (kF8) {
    if (per_head) return cudaErrorInvalidValue;
  } else {
    if (per_head && prefetch)
      return launch_pdl(attn_tc_kernel<16, true, kMode, true>, grid, dim3(threads), smem, s, *a.tmap_k, *a.tmap_v,
                        prm, lt);
    if (per_head)
      return launch_pdl(attn_tc_kernel<16, true, kMode>, grid, dim3(threads), smem, s, *a.tmap_k, *a.tmap_v, prm, lt);
    if (prefetch)
      return launch_pdl(attn_tc_kernel<16, false, kMode, true>, grid, dim3(threads), smem, s, *a.tmap_k, *a.tmap_v,
                        prm, lt);
  }
  return launch_pdl(attn_tc_kernel<16, false, kMode>, grid, dim3(threads), smem, s, *a.tmap_k, *a.tmap_v, prm, lt);
}

cudaError_t launch_layers(cudaStream_t s, const TcAttnArgs& a, const LayerAttn* layers, int n, int* splits_used,
                          int* launched) {
  if (n < 1 || n > kMaxAttnLayers) return cudaErrorInvalidValue;
  if (a.P != 16 || (a.fp8 && a.head_pages)) return cudaErrorInvalidValue;
  if (a.fp8 && (!a.k_scale || !a.v_scale || (a.k_chan != nullptr) != (a.v_tok != nullptr)))
    return cudaErrorInvalidValue;
  const int qh = a.q_heads > 0 ? a.q_heads : a.H;
  if (a.head0 < 0 || a.head0 + a.H > qh) return cudaErrorInvalidValue;
  static PerDeviceOnce attr;
  cudaError_t e = attr.run([] {
    const int b = static_cast<int>(tc::kSmemBytes), f = static_cast<int>(tc::kSmemBytes8);
    const cudaFuncAttribute at = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t r = cudaFuncSetAttribute(attn_tc_kernel<16, false, tc::kBf16>, at, b);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(attn_tc_kernel<16, true, tc::kBf16>, at, b);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(attn_tc_kernel<16, false, tc::kBf16, true>, at, b);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(attn_tc_kernel<16, true, tc::kBf16, true>, at, b);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(attn_tc_kernel<16, false, tc::kE4m3>, at, f);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(attn_tc_kernel<16, false, tc::kE4m3Da>, at, f);
    return r;
  });
  if (e != cudaSuccess) return e;
  AttnLayers lt{};
  lt.n = n;
  int np[kMaxAttnLayers], nt[kMaxAttnLayers], p0[kMaxAttnLayers];
  for (int l = 0; l < n; ++l) {
    // the softmax warps read Q rows and write O rows with 16-byte accesses
    if ((reinterpret_cast<uintptr_t>(layers[l].q) | reinterpret_cast<uintptr_t>(layers[l].o)) & 15)
      return cudaErrorInvalidValue;
    np[l] = layers[l].n_pages;
  }
  AttnPlan pl;
  if (!plan_attn_bf16(a.T, a.H, np, n, a.P, a.sm_count, a.splits, a.part_rows, a.strict_splits, &pl, nt, p0))
    return cudaErrorInvalidValue;
  if (pl.max_pieces > 1 && !a.split_cnt) return cudaErrorInvalidValue;
  for (int l = 0; l < n; ++l) {
    lt.l[l] = layers[l];
    lt.l[l].n_tiles = nt[l];
    lt.l[l].pos0 = p0[l];
  }
  TcParams prm{};
  prm.T = a.T;
  prm.H = a.H;
  prm.q_tiles = pl.q_tiles;
  prm.q_pairs = pl.q_pairs;
  prm.splits = pl.max_pieces;
  prm.tiles_per_split = pl.R;
  prm.total_tiles = static_cast<int>(pl.steps);
  prm.pool_rows = static_cast<int>(a.pool_rows);
  prm.scale_log2 = static_cast<float>(static_cast<double>(a.softmax_scale) * 1.4426950408889634);
  prm.part_o = a.part_o;
  prm.part_lse = a.part_lse;
  prm.err = a.err;
  prm.head_pages = a.head_pages;
  prm.split_cnt = a.split_cnt;
  prm.out_heads = qh;
  prm.head0 = a.head0;
  prm.k_scale = a.k_scale;
  prm.v_scale = a.v_scale;
  prm.k_chan = a.k_chan;
  prm.v_tok = a.v_tok;
  const dim3 grid(pl.grid);
  // the Q prefetch pays where a CTA sweeps many pieces: several layers or per-head lists
  const bool prefetch = n > 1 || a.head_pages > 0;
  if (!a.fp8) e = launch_mode<tc::kBf16>(s, a.head_pages > 0, prefetch, grid, prm, a, lt);
  else if (a.k_chan) e = launch_mode<tc::kE4m3Da>(s, false, false, grid, prm, a, lt);
  else e = launch_mode<tc::kE4m3>(s, false, false, grid, prm, a, lt);
  if (e != cudaSuccess) return e;
  if (launched) *launched = 1;
  if (splits_used) *splits_used = pl.max_pieces;
  return cudaSuccess;
}
}  // namespace

cudaError_t launch_attn_tc_layers(cudaStream_t s, const TcAttnArgs& base, const LayerAttn* layers, int n,
                                  int* launched) {
  if (launched) *launched = 0;
  return launch_layers(s, base, layers, n, nullptr, launched);
}

cudaError_t launch_attn_tc(cudaStream_t s, const TcAttnArgs& a, int* splits_used, int* launched) {
  if (launched) *launched = 0;
  LayerAttn one{};
  one.q = a.q;
  one.o = a.o;
  one.entries = a.entries;
  one.page_base = a.page_base;
  one.n_pages = a.n_pages;
  return launch_layers(s, a, &one, 1, splits_used, launched);
}

}  // namespace kvc
