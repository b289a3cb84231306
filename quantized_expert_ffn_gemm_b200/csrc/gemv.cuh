// Dequant-GEMV building blocks for 1-8 activation columns (decode / MTP verify): a warp owns 16
// weight rows; lane (g, t) holds rows g and g+8 and a 64-weight slice of each 256-wide K step
// (one 16-byte code load per row per step for the 2-bit plane, two for the 4-bit plane); each
// code word is dequantized to fp16 pairs and fed to mma.sync m16n8k16 with the activation
// columns as the 8 MMA columns (fp32 accumulate). QT is the block format: 2 (Q2), 3 (Q3), 4 (Q4).
// Activations are staged in shared memory as fp16, each 64-element chunk followed by 16 halves of
// padding and columns a multiple of 64 plus 4 halves apart, so the fragment loads of the four K
// slices and eight columns hit distinct banks and a lane's loads within a chunk are one base
// address plus compile-time offsets. Each MMA's four A registers are dequantized right before it.
#pragma once

#include "common.cuh"
#include "dequant.cuh"

namespace moe {

constexpr int kStepK = 256;       // K covered by one warp step (4 lanes x 64 weights)

// bytes of the code plane per weight row of K weights: 2-bit plane K/4, 4-bit plane K/2
__host__ __device__ constexpr int code_row_bytes(int qt, int K) { return qt == 4 ? K / 2 : K / 4; }

__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// shared-memory position of activation element k of a column (column stride added by the caller):
// 64-element chunk ch starts at 80 ch
__device__ __forceinline__ int xs_pos(int k) { return k + 16 * (k >> 6); }
// column stride (halves) of a staged column of K elements: the padded length rounded up to 64,
// plus 4
__host__ __device__ constexpr int xs_stride(int K) { return ((K + K / 4 + 63) & ~63) + 4; }

// word i (0..3) of a 16-byte fragment, by selects (no local-memory indexing)
__device__ __forceinline__ uint32_t sel4(const uint4 &v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

struct MatView {
  const uint8_t *codes;
  const uint8_t *hibits;
  const uint16_t *scales;
  int K;
};

// matrix `which` (0 gate, 1 up, 2 down) of expert `expert` in set `set` (0 routed, 1 shared); scalar
// selects only, so the kernel-parameter structs are never copied to local memory
__device__ __forceinline__ MatView mat_sel(const moe_expert_set &r, const moe_expert_set &sh, int set, int which,
                                           int expert) {
#define MOE_SEL(field)                                                                                  \
  (which == 0 ? (set ? sh.gate.field : r.gate.field)                                                    \
              : which == 1 ? (set ? sh.up.field : r.up.field) : (set ? sh.down.field : r.down.field))
  const uint8_t *codes = MOE_SEL(codes);
  const uint8_t *hib = MOE_SEL(hibits);
  const uint16_t *sc = MOE_SEL(scales);
  const int rows = MOE_SEL(rows), K = MOE_SEL(K), qt = MOE_SEL(qtype);
#undef MOE_SEL
  MatView v;
  const size_t row0 = (size_t)expert * rows;
  v.codes = codes + row0 * code_row_bytes(qt, K);
  v.hibits = hib ? hib + row0 * (K / 8) : nullptr;
  v.scales = sc + row0 * (K / 32);
  v.K = K;
  return v;
}

__device__ __forceinline__ MatView mat_of(const moe_qmat &m, int expert) {
  MatView v;
  const size_t row0 = (size_t)expert * m.rows;
  v.codes = m.codes + row0 * code_row_bytes(m.qtype, m.K);
  v.hibits = m.hibits ? m.hibits + row0 * (m.K / 8) : nullptr;
  v.scales = m.scales + row0 * (m.K / 32);
  v.K = m.K;
  return v;
}

// one lane's share of a 16-row x 256-wide K step: the code bytes of rows g and g+8 (16 each for the
// 2-bit plane; 32 for the 4-bit plane, the second 16 in w0b / w1b), their two block scales, and
// (Q3) the two blocks' hi-bit words
struct StepFrag {
  uint4 w0, w1;
  uint4 w0b, w1b;
  uint32_t d0, d1;
  uint2 h0, h1;
};

template <int QT>
__device__ __forceinline__ void load_step(StepFrag &f, const MatView &m, int r0, int step, bool valid) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int k0 = step * kStepK + 64 * t;
  const bool ok = valid && k0 < m.K;
  const size_t rs = (size_t)code_row_bytes(QT, m.K), ss = (size_t)m.K / 32, hs = (size_t)m.K / 8;
  const size_t co = (size_t)code_row_bytes(QT, k0);
  const size_t ra = (size_t)(r0 + g), rb = (size_t)(r0 + g + 8);
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  f.w0 = ok ? __ldcs(reinterpret_cast<const uint4 *>(m.codes + ra * rs + co)) : z4;
  f.w1 = ok ? __ldcs(reinterpret_cast<const uint4 *>(m.codes + rb * rs + co)) : z4;
  if (QT == 4) {
    f.w0b = ok ? __ldcs(reinterpret_cast<const uint4 *>(m.codes + ra * rs + co) + 1) : z4;
    f.w1b = ok ? __ldcs(reinterpret_cast<const uint4 *>(m.codes + rb * rs + co) + 1) : z4;
  }
  f.d0 = ok ? __ldcs(reinterpret_cast<const uint32_t *>(m.scales + ra * ss + k0 / 32)) : 0u;
  f.d1 = ok ? __ldcs(reinterpret_cast<const uint32_t *>(m.scales + rb * ss + k0 / 32)) : 0u;
  if (QT == 3) {
    f.h0 = ok ? __ldcs(reinterpret_cast<const uint2 *>(m.hibits + ra * hs + k0 / 8)) : make_uint2(0, 0);
    f.h1 = ok ? __ldcs(reinterpret_cast<const uint2 *>(m.hibits + rb * hs + k0 / 8)) : make_uint2(0, 0);
  }
}

// load_step with the two MMA row halves from different matrices: MMA row g is row ra of ma and
// MMA row g+8 is row rb of mb (gate row and up row of one feature), both for lane group g
template <int QT>
__device__ __forceinline__ void load_step_pair(StepFrag &f, const MatView &ma, int ra, const MatView &mb, int rb,
                                               int step, bool valid) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  const int k0 = step * kStepK + 64 * t;
  const bool ok = valid && k0 < ma.K;
  const size_t rs = (size_t)code_row_bytes(QT, ma.K), ss = (size_t)ma.K / 32, hs = (size_t)ma.K / 8;
  const size_t co = (size_t)code_row_bytes(QT, k0);
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  f.w0 = ok ? __ldcs(reinterpret_cast<const uint4 *>(ma.codes + (size_t)ra * rs + co)) : z4;
  f.w1 = ok ? __ldcs(reinterpret_cast<const uint4 *>(mb.codes + (size_t)rb * rs + co)) : z4;
  if (QT == 4) {
    f.w0b = ok ? __ldcs(reinterpret_cast<const uint4 *>(ma.codes + (size_t)ra * rs + co) + 1) : z4;
    f.w1b = ok ? __ldcs(reinterpret_cast<const uint4 *>(mb.codes + (size_t)rb * rs + co) + 1) : z4;
  }
  f.d0 = ok ? __ldcs(reinterpret_cast<const uint32_t *>(ma.scales + (size_t)ra * ss + k0 / 32)) : 0u;
  f.d1 = ok ? __ldcs(reinterpret_cast<const uint32_t *>(mb.scales + (size_t)rb * ss + k0 / 32)) : 0u;
  if (QT == 3) {
    f.h0 = ok ? __ldcs(reinterpret_cast<const uint2 *>(ma.hibits + (size_t)ra * hs + k0 / 8)) : make_uint2(0, 0);
    f.h1 = ok ? __ldcs(reinterpret_cast<const uint2 *>(mb.hibits + (size_t)rb * hs + k0 / 8)) : make_uint2(0, 0);
  }
}

// dequantize the fragment (zero codes with zero scales give zero weights) and run the step's 16
// MMAs; B fragments come from the lane's column in shared memory when `bok`, else zero. kbase (a
// multiple of 64) starts the lane's 64 weights, which lie in one staged chunk.
template <int QT>
__device__ __forceinline__ void mma_step(float acc[4], float acc2[4], const StepFrag &f, const __half *xcol, int kbase,
                                         bool bok) {
  const __half *xb = xcol + xs_pos(kbase);
  auto bfrag = [&](int off, uint32_t &b0, uint32_t &b1) {
    b0 = 0u;
    b1 = 0u;
    if (bok) {
      const uint2 bv = *reinterpret_cast<const uint2 *>(xb + off);
      b0 = bv.x;
      b1 = bv.y;
    }
  };
  if constexpr (QT == 4) {  // eight 8-weight words per row: word wq in block wq/4, two MMAs per word
#pragma unroll
    for (int wq = 0; wq < 8; ++wq) {
      const int blk = wq >> 2;
      const uint32_t w0 = blk ? sel4(f.w0b, wq & 3) : sel4(f.w0, wq & 3);
      const uint32_t w1 = blk ? sel4(f.w1b, wq & 3) : sel4(f.w1, wq & 3);
      const uint32_t w08 = w0 >> 8, w18 = w1 >> 8;
      const __half2 dd0 = __half2half2(__ushort_as_half((uint16_t)(f.d0 >> (16 * blk))));
      const __half2 dd1 = __half2half2(__ushort_as_half((uint16_t)(f.d1 >> (16 * blk))));
#pragma unroll
      for (int mm = 0; mm < 2; ++mm) {
        const uint32_t a[4] = {dq4_pair(w0, w08, 2 * mm, dd0), dq4_pair(w1, w18, 2 * mm, dd1),
                               dq4_pair(w0, w08, 2 * mm + 1, dd0), dq4_pair(w1, w18, 2 * mm + 1, dd1)};
        uint32_t b0, b1;
        bfrag(8 * wq + 4 * mm, b0, b1);
        mma16816(mm ? acc2 : acc, a, b0, b1);
      }
    }
  } else {
#pragma unroll
    for (int wq = 0; wq < 4; ++wq) {  // word wq: block wq/2, half q = wq%2
      const int blk = wq >> 1, q = wq & 1;
      const uint32_t w0 = sel4(f.w0, wq), w1 = sel4(f.w1, wq);
      const uint32_t w08 = w0 >> 8, w18 = w1 >> 8;
      const __half2 dd0 = __half2half2(__ushort_as_half((uint16_t)(f.d0 >> (16 * blk))));
      const __half2 dd1 = __half2half2(__ushort_as_half((uint16_t)(f.d1 >> (16 * blk))));
      uint32_t hs0 = 0u, hs1 = 0u;
      if (QT == 3) {
        const uint32_t h0 = blk ? f.h0.y : f.h0.x, h1 = blk ? f.h1.y : f.h1.x;
        hs0 = q ? (h0 >> 6) : (h0 << 2);
        hs1 = q ? (h1 >> 6) : (h1 << 2);
      }
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {  // MMA 4*wq + mm: pairs 2mm, 2mm+1 of this word
        uint32_t a[4];
        if (QT == 3) {
          a[0] = dq3_pair(w0, w08, hs0, 2 * mm, dd0);
          a[1] = dq3_pair(w1, w18, hs1, 2 * mm, dd1);
          a[2] = dq3_pair(w0, w08, hs0, 2 * mm + 1, dd0);
          a[3] = dq3_pair(w1, w18, hs1, 2 * mm + 1, dd1);
        } else {
          a[0] = dq2_pair(w0, w08, 2 * mm, dd0);
          a[1] = dq2_pair(w1, w18, 2 * mm, dd1);
          a[2] = dq2_pair(w0, w08, 2 * mm + 1, dd0);
          a[3] = dq2_pair(w1, w18, 2 * mm + 1, dd1);
        }
        uint32_t b0, b1;
        bfrag(16 * wq + 4 * mm, b0, b1);
        mma16816((mm & 1) ? acc2 : acc, a, b0, b1);
      }
    }
  }
}

// Half of a step: a 16-row x 128-wide K slice, lane (g, t) holding the 32-weight block
// kbase..kbase+31 (kbase = slice start + 32 t) of rows g and g+8: two code words per row (four
// for the 4-bit plane, the last two in w0b / w1b), one scale per row, and (Q3) one hi word per
// row. Same pair decoder and MMA-K order as mma_step.
struct HalfFrag {
  uint2 w0, w1;
  uint2 w0b, w1b;
  uint16_t d0, d1;
  uint32_t h0, h1;
};

template <int QT>
__device__ __forceinline__ void mma_half_step(float acc[4], float acc2[4], const HalfFrag &f, const __half *xcol,
                                              int kbase, bool bok) {
  const __half *xb = xcol + xs_pos(kbase);  // kbase: a multiple of 32; its 32 weights lie in one chunk
  auto bfrag = [&](int off, uint32_t &b0, uint32_t &b1) {
    b0 = 0u;
    b1 = 0u;
    if (bok) {
      const uint2 bv = *reinterpret_cast<const uint2 *>(xb + off);
      b0 = bv.x;
      b1 = bv.y;
    }
  };
  const __half2 dd0 = __half2half2(__ushort_as_half(f.d0));
  const __half2 dd1 = __half2half2(__ushort_as_half(f.d1));
  if constexpr (QT == 4) {
#pragma unroll
    for (int wq = 0; wq < 4; ++wq) {
      const uint2 a0 = (wq >> 1) ? f.w0b : f.w0, a1 = (wq >> 1) ? f.w1b : f.w1;
      const uint32_t w0 = (wq & 1) ? a0.y : a0.x, w1 = (wq & 1) ? a1.y : a1.x;
      const uint32_t w08 = w0 >> 8, w18 = w1 >> 8;
#pragma unroll
      for (int mm = 0; mm < 2; ++mm) {
        const uint32_t a[4] = {dq4_pair(w0, w08, 2 * mm, dd0), dq4_pair(w1, w18, 2 * mm, dd1),
                               dq4_pair(w0, w08, 2 * mm + 1, dd0), dq4_pair(w1, w18, 2 * mm + 1, dd1)};
        uint32_t b0, b1;
        bfrag(8 * wq + 4 * mm, b0, b1);
        mma16816(mm ? acc2 : acc, a, b0, b1);
      }
    }
  } else {
#pragma unroll
    for (int wq = 0; wq < 2; ++wq) {
      const uint32_t w0 = wq ? f.w0.y : f.w0.x, w1 = wq ? f.w1.y : f.w1.x;
      const uint32_t w08 = w0 >> 8, w18 = w1 >> 8;
      uint32_t hs0 = 0u, hs1 = 0u;
      if (QT == 3) {
        hs0 = wq ? (f.h0 >> 6) : (f.h0 << 2);
        hs1 = wq ? (f.h1 >> 6) : (f.h1 << 2);
      }
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        uint32_t a[4];
        if (QT == 3) {
          a[0] = dq3_pair(w0, w08, hs0, 2 * mm, dd0);
          a[1] = dq3_pair(w1, w18, hs1, 2 * mm, dd1);
          a[2] = dq3_pair(w0, w08, hs0, 2 * mm + 1, dd0);
          a[3] = dq3_pair(w1, w18, hs1, 2 * mm + 1, dd1);
        } else {
          a[0] = dq2_pair(w0, w08, 2 * mm, dd0);
          a[1] = dq2_pair(w1, w18, 2 * mm, dd1);
          a[2] = dq2_pair(w0, w08, 2 * mm + 1, dd0);
          a[3] = dq2_pair(w1, w18, 2 * mm + 1, dd1);
        }
        uint32_t b0, b1;
        bfrag(16 * wq + 4 * mm, b0, b1);
        mma16816((mm & 1) ? acc2 : acc, a, b0, b1);
      }
    }
  }
}

// a lane's HalfFrag straight from global memory: rows r0+g and r0+g+8 of m, the 32-weight block
// starting at K offset kk (a multiple of 32)
template <int QT>
__device__ __forceinline__ void load_half(HalfFrag &f, const MatView &m, int r0, int kk) {
  const int g = (threadIdx.x & 31) >> 2;
  const size_t rs = (size_t)code_row_bytes(QT, m.K), ss = (size_t)m.K / 32, hs = (size_t)m.K / 8;
  const size_t ra = (size_t)(r0 + g), rb = ra + 8;
  if (QT == 4) {
    const uint4 c0 = __ldcs(reinterpret_cast<const uint4 *>(m.codes + ra * rs + kk / 2));
    const uint4 c1 = __ldcs(reinterpret_cast<const uint4 *>(m.codes + rb * rs + kk / 2));
    f.w0 = make_uint2(c0.x, c0.y);
    f.w0b = make_uint2(c0.z, c0.w);
    f.w1 = make_uint2(c1.x, c1.y);
    f.w1b = make_uint2(c1.z, c1.w);
  } else {
    f.w0 = __ldcs(reinterpret_cast<const uint2 *>(m.codes + ra * rs + kk / 4));
    f.w1 = __ldcs(reinterpret_cast<const uint2 *>(m.codes + rb * rs + kk / 4));
  }
  f.d0 = __ldcs(m.scales + ra * ss + kk / 32);
  f.d1 = __ldcs(m.scales + rb * ss + kk / 32);
  if (QT == 3) {
    f.h0 = __ldcs(reinterpret_cast<const uint32_t *>(m.hibits + ra * hs + kk / 8));
    f.h1 = __ldcs(reinterpret_cast<const uint32_t *>(m.hibits + rb * hs + kk / 8));
  }
}

// acc += W[r0..r0+15, steps s0..s0+NS-1] * X^T; all of the batch's loads are issued first
template <int QT, int NS>
__device__ __forceinline__ void rows16_batch(const MatView &m, int r0, int s0, int nsteps, const __half *xcol,
                                             bool colok, float acc[4]) {
  const int t = threadIdx.x & 3;
  StepFrag f[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) load_step<QT>(f[s], m, r0, s0 + s, s0 + s < nsteps);
  float acc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int kbase = (s0 + s) * kStepK + 64 * t;
    mma_step<QT>(acc, acc2, f[s], xcol, kbase, colok && (s0 + s < nsteps) && kbase < m.K);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] += acc2[e];
}

// full K of 16 rows: batches of 8 steps, then a tail batch of 4, 2 or 1
template <int QT>
__device__ __forceinline__ void rows16(const MatView &m, int r0, const __half *xcol, bool colok, float acc[4]) {
  const int nsteps = (m.K + kStepK - 1) / kStepK;
  int s = 0;
  for (; s + 8 <= nsteps; s += 8) rows16_batch<QT, 8>(m, r0, s, nsteps, xcol, colok, acc);
  const int rem = nsteps - s;
  if (rem > 4) rows16_batch<QT, 8>(m, r0, s, nsteps, xcol, colok, acc);
  else if (rem > 2) rows16_batch<QT, 4>(m, r0, s, nsteps, xcol, colok, acc);
  else if (rem == 2) rows16_batch<QT, 2>(m, r0, s, nsteps, xcol, colok, acc);
  else if (rem == 1) rows16_batch<QT, 1>(m, r0, s, nsteps, xcol, colok, acc);
}

// stage columns of the activation source into shared memory (fp16, padded layout). 16-byte
// loads, several issued before the first store, so the staging costs one memory round trip.
// returns true when a bf16 source value was beyond the fp16 range (it is staged as +-inf)
template <bool SRC_BF16>
__device__ __forceinline__ bool stage_x(const void *src, int row0, int mask, int H, __half *xs, int xstride) {
  bool bad = false;
  const int H8 = H / 8;
  const uint16_t *base = static_cast<const uint16_t *>(src);
  for (int c = 0; c < 8; ++c) {
    if (!((mask >> c) & 1)) continue;
    const uint4 *sp = reinterpret_cast<const uint4 *>(base + (size_t)(row0 + c) * H);
    for (int i0 = threadIdx.x; i0 < H8; i0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        v[j] = (i < H8) ? __ldg(sp + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        if (i >= H8) break;
        uint4 o = v[j];
        if (SRC_BF16) {
          const uint32_t in[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
          uint32_t out[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            __half2 h = __floats2half2_rn(__uint_as_float(in[q] << 16), __uint_as_float(in[q] & 0xffff0000u));
            out[q] = *reinterpret_cast<uint32_t *>(&h);
            bad |= f16x2_inf(out[q]);
          }
          o = make_uint4(out[0], out[1], out[2], out[3]);
        }
        // rows are 8-byte aligned (stride H+4 halves): two 8-byte stores
        uint2 *d = reinterpret_cast<uint2 *>(xs + (size_t)c * xstride + xs_pos(8 * i));
        d[0] = make_uint2(o.x, o.y);
        d[1] = make_uint2(o.z, o.w);
      }
    }
  }
  return bad;
}

// stage_x for an arbitrary token per column: column c < ncol is row tok[c] of the bf16 source
__device__ __forceinline__ bool stage_x_tokens(const uint16_t *src, const int *tok, int ncol, int H, __half *xs,
                                               int xstride) {
  bool bad = false;
  const int H8 = H / 8, n = ncol * H8;
  for (int i0 = threadIdx.x; i0 < n; i0 += 4 * blockDim.x) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = i0 + j * blockDim.x;
      v[j] = (i < n) ? __ldg(reinterpret_cast<const uint4 *>(src + (size_t)tok[i / H8] * H) + i % H8)
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = i0 + j * blockDim.x;
      if (i >= n) break;
      const uint32_t in[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      uint32_t out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __half2 h = __floats2half2_rn(__uint_as_float(in[q] << 16), __uint_as_float(in[q] & 0xffff0000u));
        out[q] = *reinterpret_cast<uint32_t *>(&h);
        bad |= f16x2_inf(out[q]);
      }
      uint2 *d = reinterpret_cast<uint2 *>(xs + (size_t)(i / H8) * xstride + xs_pos(8 * (i % H8)));
      d[0] = make_uint2(out[0], out[1]);
      d[1] = make_uint2(out[2], out[3]);
    }
  }
  return bad;
}

}  // namespace moe
