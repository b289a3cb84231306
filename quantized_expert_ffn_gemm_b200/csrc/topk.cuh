// Warp top-k over fp32 logits (lower expert index wins ties, slots in descending order, softmax
// over the selected set) and the grouping of selected (token, slot) pairs by distinct expert.
#pragma once

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------- top-k within one warp

// order-preserving 32-bit key of an fp32 logit (NaN sorts lowest, -0 == +0)
__device__ __forceinline__ uint32_t logit_key(float f) {
  if (f != f) return 0u;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of E logits (l[0..E) in shared or global memory) by one warp. Writes idx[0..k) and
// w[0..k). Rounds of: per-lane best among untaken candidates (ascending index scan, strict >,
// so the lower index wins a tie inside a lane), warp max of the key, then warp min of the index
// among lanes holding that key. Lane j keeps the winner of round j, so the k selections end up
// spread over lanes 0..k-1 and the softmax over the set is one warp reduction.
__device__ __forceinline__ void topk_finish(float my_val, int my_idx, int k, int32_t *idx, float *w) {
  const int lane = threadIdx.x & 31;
  const float l0 = __shfl_sync(0xffffffffu, my_val, 0);
  const float ev = (lane < k) ? expf(my_val - l0) : 0.0f;
  const float z = warp_sum(ev);
  if (lane < k) {
    idx[lane] = my_idx;
    w[lane] = ev / z;
  }
}

// 64-bit code ordering candidates: larger logit first, equal logits -> lower expert index first
__device__ __forceinline__ unsigned long long topk_code(float v, int e) {
  return ((unsigned long long)logit_key(v) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)e);
}
__device__ __forceinline__ float key_to_logit(uint32_t key) {
  const uint32_t u = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(u);
}

// bitonic network: 16 codes into descending order (compile-time indices, registers only)
__device__ __forceinline__ void sort16_desc(unsigned long long c[16]) {
#pragma unroll
  for (int size = 2; size <= 16; size <<= 1) {
#pragma unroll
    for (int stride = size / 2; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = c[i], b = c[j];
          const bool sw = desc ? (a < b) : (a > b);
          c[i] = sw ? b : a;
          c[j] = sw ? a : b;
        }
      }
    }
  }
}

// warp-wide bitonic networks on 64-bit codes (one code per lane, shuffles only)
__device__ __forceinline__ unsigned long long cmax64(unsigned long long a, unsigned long long b) { return a > b ? a : b; }
__device__ __forceinline__ unsigned long long cmin64(unsigned long long a, unsigned long long b) { return a < b ? a : b; }

// How many of the first n (<= 32) codes of s exceed v: with distinct codes, v's position in
// descending order. Every lane reads all n from shared memory (broadcast reads, independent of one
// another), so ranking a warp's worth of codes costs about one pass over them instead of the
// dependent stages of a sorting network.
__device__ __forceinline__ int rank_desc32(const unsigned long long *s, int n, unsigned long long v) {
  int r0 = 0, r1 = 0;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    r0 += (j < n && s[j] > v) ? 1 : 0;
    r1 += (j + 1 < n && s[j + 1] > v) ? 1 : 0;
  }
  return r0 + r1;
}

// sort the warp's 32 codes into descending lane order
__device__ __forceinline__ unsigned long long warp_sort32_desc(unsigned long long v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool keep_max = (((lane & size) == 0) == ((lane & stride) == 0));
      v = keep_max ? cmax64(v, o) : cmin64(v, o);
    }
  }
  return v;
}

// lanes 0-15 hold a descending list, lanes 16-31 another list in ascending order (a bitonic
// sequence): merge into descending lane order (lanes 0-15 then hold the top 16 of both)
__device__ __forceinline__ unsigned long long warp_merge32_desc(unsigned long long v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
    v = ((lane & stride) == 0) ? cmax64(v, o) : cmin64(v, o);
  }
  return v;
}

// E <= 512: lane L holds experts L, L+32, ... sorted; each round the warp takes the best head
// (max key, then min index) and the winning lane shifts its list by one.
// l_out (optional): receives logit + bias for every expert, stored as soon as it is formed.
template <int PER_LANE>
static __device__ void warp_topk(const float *l, const float *bias, int E, int k, int32_t *idx, float *w,
                                 float *l_out = nullptr) {
  static_assert(PER_LANE == 16, "16 candidates per lane");
  const int lane = threadIdx.x & 31;
  unsigned long long c[16];
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {  // all loads first, then the codes (and the stores)
    const int e = lane + 32 * i;
    v[i] = (e < E) ? l[e] + (bias ? bias[e] : 0.0f) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int e = lane + 32 * i;
    c[i] = (e < E) ? topk_code(v[i], e) : 0ull;
    if (l_out && e < E) l_out[e] = v[i];
  }
  sort16_desc(c);
  float my_val = -INFINITY;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t hk = (uint32_t)(c[0] >> 32);
    const uint32_t m = __reduce_max_sync(0xffffffffu, hk);
    const uint32_t lo = (hk == m) ? (uint32_t)c[0] : 0u;
    const uint32_t win = __reduce_max_sync(0xffffffffu, lo);  // max of (~index) = lowest index
    const bool is_win = (hk == m) && ((uint32_t)c[0] == win);
#pragma unroll
    for (int i = 0; i < 15; ++i) c[i] = is_win ? c[i + 1] : c[i];
    c[15] = is_win ? 0ull : c[15];
    if (lane == j) {
      my_val = key_to_logit(m);
      my_idx = (int)(0xFFFFFFFFu - win);
    }
  }
  topk_finish(my_val, my_idx, k, idx, w);
}

// generic E (up to kMaxE) from shared memory: lanes rescan their strided candidates each round
static __device__ void warp_topk_generic(const float *l, const float *bias, int E, int k, int32_t *idx, float *w,
                                  uint32_t *taken_words /* smem, E/32 words, zeroed */) {
  const int lane = threadIdx.x & 31;
  float my_val = -INFINITY;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;
    int bi = 0x7fffffff;
    float bv = -INFINITY;
    for (int e = lane; e < E; e += 32) {
      if ((taken_words[e >> 5] >> (e & 31)) & 1u) continue;
      const float v = l[e] + (bias ? bias[e] : 0.0f);
      const uint32_t kk = logit_key(v);
      if (kk > bk || bi == 0x7fffffff) { bk = kk; bi = e; bv = v; }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bi == 0x7fffffff ? 0u : bk);
    const uint32_t cand = (bi != 0x7fffffff && bk == m) ? (uint32_t)bi : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if ((uint32_t)bi == win) taken_words[bi >> 5] |= 1u << (bi & 31);
    __syncwarp();
    const float wv = __shfl_sync(0xffffffffu, bv, (int)(win & 31u));
    if (lane == j) { my_val = wv; my_idx = (int)win; }
  }
  topk_finish(my_val, my_idx, k, idx, w);
}

// ---------------------------------------------------------------- decode units
// Group the T*k selected (token, slot) pairs by distinct expert, in order of first appearance
// (token-major), plus the always-on shared expert as the last unit. Uses every thread of the
// block (all of them must call it): an expert -> first-pair table built with atomicMin, a ballot
// prefix to number the first pairs, then one pass over the pairs fills the records.
struct UnitScratch {
  int first_of[kMaxE];                    // expert -> first pair index choosing it
  int unit_of[kDecodeMaxT * kMaxK];       // pair -> unit (valid at first pairs)
  int mask[kDecodeMaxT * kMaxK + 1];
  float w[kDecodeMaxT * kMaxK + 1][8];
  int expert[kDecodeMaxT * kMaxK + 1];
  int nu;
};

static __device__ void build_units(const int32_t *sidx, const float *sw, int T, int k, int E, int has_shared,
                                   DecUnit *units, int *n_units_out, UnitScratch &us) {
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31;
  const int P = T * k;
  for (int e = tid; e < E; e += nthr) us.first_of[e] = 0x7fffffff;
  __syncthreads();
  for (int p = tid; p < P; p += nthr) atomicMin(&us.first_of[sidx[p]], p);
  __syncthreads();
  if (tid < 32) {  // number the first pairs in pair order
    int nu = 0;
    for (int base = 0; base < P; base += 32) {
      const int p = base + lane;
      const bool lead = (p < P) && us.first_of[sidx[p]] == p;
      const unsigned bal = __ballot_sync(0xffffffffu, lead);
      if (lead) us.unit_of[p] = nu + __popc(bal & ((1u << lane) - 1u));
      nu += __popc(bal);
    }
    if (lane == 0) us.nu = nu;
  }
  __syncthreads();
  const int nu = us.nu, total = nu + (has_shared ? 1 : 0);
  for (int i = tid; i < total * 8; i += nthr) {
    const int u = i >> 3, c = i & 7;
    us.w[u][c] = (u == nu) ? (c < T ? 1.0f : 0.0f) : 0.0f;
    if (c == 0) {
      us.mask[u] = (u == nu) ? (1 << T) - 1 : 0;
      if (u == nu) us.expert[u] = 0;
    }
  }
  __syncthreads();
  for (int p = tid; p < P; p += nthr) {  // each (unit, token) is hit once: an expert appears once per token
    const int u = us.unit_of[us.first_of[sidx[p]]], t = p / k;
    us.expert[u] = sidx[p];
    atomicOr(&us.mask[u], 1 << t);
    us.w[u][t] = sw[p];
  }
  __syncthreads();
  for (int u = tid; u < total; u += nthr) {
    DecUnit d;
    d.expert = us.expert[u];
    d.set = (u == nu) ? 1 : 0;
    d.mask = us.mask[u];
    d.xrow0 = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) d.w[c] = us.w[u][c];
    units[u] = d;
  }
  if (tid == 0) *n_units_out = total;
  __syncthreads();
}

}  // namespace moe
