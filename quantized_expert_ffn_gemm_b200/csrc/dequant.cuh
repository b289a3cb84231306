// On-the-fly dequantization of Q2 / Q3 blocks into fp16 MMA operands.
//
// The expert matmul dequantizes low-bit block weights during the multiply ("Two-Day Port, 8x
// Faster Prefill: Strata Engine Benchmarked", "Where Strata Is Fast: Not Magic, but Logistics",
// MMQ paragraph). Block formats (stand-in): 32 weights, fp16 scale d; Q2 w = d(c-2), Q3 w = d(c-4).
//
// Plane layout (include/moe_ffn.h): in each 32-bit little-endian word of the 2-bit plane (16
// weights), weight 2i+h (i = 0..7, h = 0..1) sits at bits 16h+2i. Masking bits 2p..2p+1 of both
// 16-bit halves (p = 0..3) and OR-ing in the fp16 exponent pattern of M_p = 2^(10-2p) (whose ulp
// is 2^-2p) gives the half2 (M_p + c_2i, M_p + c_2i+1) exactly; shifting the word right by 8
// gives pairs 4..7 the same way. Subtracting M_p + q0 is exact (small integers), and one fp16
// multiply by d rounds d(c - q0) once (exact for Q2; Q3 codes 1 and 7 round d*(+-3) to nearest).
//
// Q4 (4-bit codes, w = d(c-8)): per block four words, word q (weights 8q..8q+7) holding weight
// 8q+2i+h (i = 0..3, h = 0..1) at bits 16h+4i. Pairs 0 and 1 sit at bits 0-3 and 4-7 of both
// halves: masked and OR-ed with M = 1024 (ulp 1) and M = 64 (ulp 2^-4) they give M + c exactly;
// the word shifted right by 8 gives pairs 2 and 3 the same way. (M + c) - (M + 8) = c - 8 is exact
// and one fp16 multiply by d rounds d(c - 8) once.
//
// Q3: the 1-bit plane holds, per block, one word with bit 2 of weight 16q+2i+h at bit 16h+8q+i.
// The word pre-shifted so that pair i of half-block q lands on bits i+2 / 18+i, masked and OR-ed
// with M_h = 2^(10-i) (ulp 2^-i), is (M_h + 4 hi) exactly; (x_lo - (M_p + 4 + M_h)) + x_hi =
// c - 4 exactly (each intermediate is representable), then times d.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace moe {

__device__ __forceinline__ __half2 h2bits(uint32_t b) {
  __half2 r;
  *reinterpret_cast<uint32_t *>(&r) = b;
  return r;
}
__device__ __forceinline__ uint32_t bits_h2(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// fp16 bit patterns of M_p = 1024, 256, 64, 16 replicated in both halves
__device__ __forceinline__ uint32_t dq_magic(int p) {
  return p == 0 ? 0x64006400u : p == 1 ? 0x5C005C00u : p == 2 ? 0x54005400u : 0x4C004C00u;
}
// M_p + 2
__device__ __forceinline__ uint32_t dq2_sub(int p) {
  return p == 0 ? 0x64026402u : p == 1 ? 0x5C085C08u : p == 2 ? 0x54205420u : 0x4C804C80u;
}
// M_h(i) = 2^(10-i)
__device__ __forceinline__ uint32_t dq3_hmag(int i) {
  switch (i) {
    case 0: return 0x64006400u;
    case 1: return 0x60006000u;
    case 2: return 0x5C005C00u;
    case 3: return 0x58005800u;
    case 4: return 0x54005400u;
    case 5: return 0x50005000u;
    case 6: return 0x4C004C00u;
    default: return 0x48004800u;
  }
}
// M_(i mod 4) + 4 + M_h(i)
__device__ __forceinline__ uint32_t dq3_sub(int i) {
  switch (i) {
    case 0: return 0x68026802u;
    case 1: return 0x62086208u;
    case 2: return 0x5D105D10u;
    case 3: return 0x58A058A0u;
    case 4: return 0x64446444u;
    case 5: return 0x5C905C90u;
    case 6: return 0x55405540u;
    default: return 0x4F004F00u;
  }
}

// Pair j (weights 2j, 2j+1; j = 0..7, a compile-time constant in callers) of a Q2 word w, times d;
// w8 = w >> 8.
__device__ __forceinline__ uint32_t dq2_pair(uint32_t w, uint32_t w8, int j, __half2 d2) {
  const int p = j & 3;
  const uint32_t src = (j < 4) ? w : w8;
  const uint32_t t = (src & (0x00030003u << (2 * p))) | dq_magic(p);
  return bits_h2(__hmul2_rn(__hsub2_rn(h2bits(t), h2bits(dq2_sub(p))), d2));
}

// One Q2 word (16 weights) -> 8 half2 in natural K order (out[j] = weights 2j, 2j+1), times d.
__device__ __forceinline__ void dq2_word(uint32_t w, __half2 d2, uint32_t out[8]) {
  const uint32_t w8 = w >> 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) out[j] = dq2_pair(w, w8, j, d2);
}

// Same pairs without the scale: (c - 2) exactly, for callers that apply d afterwards.
__device__ __forceinline__ void dq2_word_noscale(uint32_t w, uint32_t out[8]) {
  const uint32_t w8 = w >> 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int p = j & 3;
    const uint32_t src = (j < 4) ? w : w8;
    const uint32_t t = (src & (0x00030003u << (2 * p))) | dq_magic(p);
    out[j] = bits_h2(__hsub2_rn(h2bits(t), h2bits(dq2_sub(p))));
  }
}

// Pair j of a Q3 half-block (see dq3_word): w8 = w >> 8, hs = the hi word shifted for the half
// (q ? hw >> 6 : hw << 2).
__device__ __forceinline__ uint32_t dq3_pair(uint32_t w, uint32_t w8, uint32_t hs, int j, __half2 d2) {
  const int p = j & 3;
  const uint32_t src = (j < 4) ? w : w8;
  const uint32_t tl = (src & (0x00030003u << (2 * p))) | dq_magic(p);
  const uint32_t th = (hs & (0x00010001u << (j + 2))) | dq3_hmag(j);
  const __half2 v = __hadd2_rn(__hsub2_rn(h2bits(tl), h2bits(dq3_sub(j))), h2bits(th));
  return bits_h2(__hmul2_rn(v, d2));
}

// One Q3 half-block: low-plane word w (16 weights) and the block's hi word `hw`, q = which half
// (0: weights 0..15 of the block, 1: weights 16..31). out[j] = weights 2j, 2j+1, times d.
__device__ __forceinline__ void dq3_word(uint32_t w, uint32_t hw, int q, __half2 d2, uint32_t out[8]) {
  const uint32_t w8 = w >> 8;
  const uint32_t hs = q ? (hw >> 6) : (hw << 2);
#pragma unroll
  for (int j = 0; j < 8; ++j) out[j] = dq3_pair(w, w8, hs, j, d2);
}

// Pair j (0..3) of a Q4 word w (8 weights), times d; w8 = w >> 8.
__device__ __forceinline__ uint32_t dq4_pair(uint32_t w, uint32_t w8, int j, __half2 d2) {
  const uint32_t src = (j < 2) ? w : w8;
  const bool hi = j & 1;  // bits 4-7 (magic 64) or 0-3 (magic 1024)
  const uint32_t t = (src & (hi ? 0x00F000F0u : 0x000F000Fu)) | (hi ? 0x54005400u : 0x64006400u);
  return bits_h2(__hmul2_rn(__hsub2_rn(h2bits(t), h2bits(hi ? 0x54805480u : 0x64086408u)), d2));  // - (M + 8)
}

// One Q4 word (8 weights) -> 4 half2 in natural K order (out[j] = weights 2j, 2j+1), times d.
__device__ __forceinline__ void dq4_word(uint32_t w, __half2 d2, uint32_t out[4]) {
  const uint32_t w8 = w >> 8;
#pragma unroll
  for (int j = 0; j < 4; ++j) out[j] = dq4_pair(w, w8, j, d2);
}

}  // namespace moe
