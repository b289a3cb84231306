// Mid-batch expert path: about 6 to 128 tokens per layer (MTP verify with prompt-lookup drafts,
// small batches). Strata DETAILS.md, "How it works": a verify pass carries the token and up to
// five prompt-lookup drafts (or up to three MTP drafts); "Two-Day Port, 8x Faster Prefill",
// "Where Strata Is Fast": batching amortises each expert's weight read over the tokens that chose
// it.
//
// At these sizes an expert is chosen by one to a few tokens (or, under a skewed router, by most of
// them), so the grouped GEMM's 16-row tiles are mostly padding and the permutation kernels cost
// more than the arithmetic; the fused decode kernel stages every h column of the step in one CTA,
// which stops fitting after about five tokens. This path works expert-major with no exchange
// between CTAs:
//   plan     one CTA: per selected expert a bit mask of the tokens that chose it; units of up to
//            NT of those tokens (ascending; NT = 8, 16 or 32 by the total work, below), then the
//            shared expert's units. Pair (t, j) writes partial row row_of[t*k+j] (the expert-major order of the
//            stable permutation), the shared expert's row of token t is n_pairs + t, and
//            row_tok[r] names the token of partial row r.
//   expert   persistent grid, items (unit, 128-feature slice): the unit's tokens are staged in
//            shared memory (fp16); warp w runs features 8w..8w+7 of the slice over all of H (gate
//            row as MMA row g, up row as MMA row g+8, so SwiGLU needs no exchange) for every
//            8-token column tile of the unit, each weight fragment dequantized once for all the
//            tiles; h goes to shared memory; then the slice's columns of the down rows (one
//            128-wide half step per 16-row block) give the item's fp32 partial output rows.
//   combine  y[t] = residual[t] + sum_j w[t,j] * sum_s part_s[row_of[t,j]] + sum_s part_s[shared row],
//            in that fixed order (deterministic).
// Work is bound by the dequantization (three instructions per weight pair) where units are small,
// so the tile loop reuses each fragment, and the activations sit in a padded layout whose B
// fragment addresses are a per-lane base plus compile-time offsets.
#include "common.cuh"
#include "dequant.cuh"
#include "gemv.cuh"

namespace moe {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kMxWarps = kMidFS / 8;  // one 8-feature block per warp in the gate/up phase
constexpr int kMxThreads = kMxWarps * 32;
constexpr int kMaxTiles = 4;          // 8-token column tiles per unit

// Padded activation layout: element k of a column at mid_pos(k) = k + 16 (k / 64), columns
// mid_stride(K) halves apart (4 mod 64). A 64-element chunk stays contiguous, consecutive chunks
// start 8 banks apart and consecutive columns 2 banks apart, so the B-fragment loads of a half
// warp (columns g = 0..3, chunks t = 0..3) fall on 16 distinct bank pairs.
__host__ __device__ inline int mid_stride(int K) { return ((K / 64) * 80 + 63) / 64 * 64 + 4; }
__device__ __forceinline__ int mid_pos(int k) { return k + 16 * (k >> 6); }

// exclusive prefix over the block of one int per thread; returns the block total in *total
__device__ int block_exclusive_scan(int v, int *warp_sums, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int ws = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, ws, o);
      if (lane >= o) ws += n;
    }
    if (lane < nw) warp_sums[lane] = ws;  // inclusive over warps
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + inc - v;
  *total = warp_sums[nw - 1];
  __syncthreads();  // warp_sums is reused by the next scan
  return before;
}

__global__ void __launch_bounds__(kPlanThreads) mid_plan_kernel(const int32_t *__restrict__ idx, int T, int k, int E,
                                                               int has_shared, int nt_max, int slices, int grid,
                                                               MidUnit *__restrict__ units,
                                                               int32_t *__restrict__ row_of,
                                                               int32_t *__restrict__ row_tok, Ctrl *__restrict__ ctrl) {
  extern __shared__ uint32_t sm[];
  uint32_t *mask = sm;                                      // [E][4] tokens that chose expert e
  int *coff = reinterpret_cast<int *>(sm + 4 * (size_t)E);  // [E] first partial row of expert e
  int *gbase = coff + E;                                    // [E] first unit of expert e
  __shared__ int s_ws[32];
  __shared__ int s_dup;
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, P = T * k;
  if (tid == 0) s_dup = 0;
  for (int i = tid; i < 4 * E; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = idx[p], t = p / k;
    if (e < 0 || e >= E) {
      set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, e);
      continue;
    }
    const uint32_t bit = 1u << (t & 31);
    if (atomicOr(&mask[4 * e + (t >> 5)], bit) & bit) s_dup = 1;  // an expert twice in one selection
  }
  __syncthreads();
  // per expert: tokens (partial rows) and units; exclusive prefixes in expert index order, each
  // thread taking up to four consecutive experts
  const int per = (E + blockDim.x - 1) / blockDim.x;  // <= 4 (E <= 4096)
  const int e0 = tid * per;
  int cnt[4], sc = 0, st = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + i;
    cnt[i] = (i < per && e < E)
                 ? __popc(mask[4 * e]) + __popc(mask[4 * e + 1]) + __popc(mask[4 * e + 2]) + __popc(mask[4 * e + 3])
                 : 0;
    sc += cnt[i];
    st += (cnt[i] + 7) >> 3;
  }
  // Unit size. An item costs about its number of 8-token column tiles (the tensor work of the
  // MMAs grows with the tiles, the dequantization does not), and the grid runs the items in about
  // max(total / grid, largest item). So units stay at 8 tokens while the one-tile items fill about
  // one round of the grid, and grow to 16 or 32 tokens (sharing each dequantized fragment) only as
  // the total work per CTA grows past that.
  int tiles8 = 0;
  (void)block_exclusive_scan(st, s_ws, &tiles8);
  tiles8 += has_shared ? (T + 7) / 8 : 0;
  const int share = (tiles8 * slices + grid - 1) / grid;
  const int NT = min(nt_max, 8 * max(1, min(4, share)));
  // partial rows in expert index order; units (the work list) with the experts whose first unit
  // has the most column tiles first (then by index), so that the persistent grid's round-robin
  // deals the costliest items first
  int n_pairs = 0, n_runits = 0;
  int rc = block_exclusive_scan(sc, s_ws, &n_pairs);
  int ub[5];  // units before this thread's experts, per tile bucket (4 tiles .. 1 tile)
  int bucket_base = 0;
#pragma unroll
  for (int b = 4; b >= 1; --b) {
    int su = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tiles = (min(cnt[i], NT) + 7) >> 3;
      if (cnt[i] > 0 && tiles == b) su += (cnt[i] + NT - 1) / NT;
    }
    int tot = 0;
    ub[b] = bucket_base + block_exclusive_scan(su, s_ws, &tot);
    bucket_base += tot;
  }
  n_runits = bucket_base;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + i;
    if (i < per && e < E) {
      coff[e] = rc;
      rc += cnt[i];
      if (cnt[i] > 0) {
        const int b = (min(cnt[i], NT) + 7) >> 3;
        gbase[e] = ub[b];
        ub[b] += (cnt[i] + NT - 1) / NT;
      } else {
        gbase[e] = 0;
      }
    }
  }
  __syncthreads();
  // every pair: its rank among the expert's tokens gives its unit and partial row
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = idx[p], t = p / k;
    if (e < 0 || e >= E) {
      row_of[p] = -1;
      continue;
    }
    const uint32_t *m = mask + 4 * e;
    int r = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int wd = 0; wd < (t >> 5); ++wd) r += __popc(m[wd]);
    row_of[p] = coff[e] + r;
    row_tok[coff[e] + r] = t;
    if (r % NT == 0) {
      const int n = __popc(m[0]) + __popc(m[1]) + __popc(m[2]) + __popc(m[3]);
      MidUnit &mu = units[gbase[e] + r / NT];
      mu.expert = e;
      mu.set = 0;
      mu.ncol = min(NT, n - r);
      mu.row0 = coff[e] + r;
    }
  }
  const int nsh = has_shared ? (T + NT - 1) / NT : 0;
  for (int i = tid; i < nsh; i += blockDim.x) {
    MidUnit &mu = units[n_runits + i];
    mu.expert = 0;
    mu.set = 1;
    mu.ncol = min(NT, T - NT * i);
    mu.row0 = n_pairs + NT * i;
  }
  if (has_shared)
    for (int t = tid; t < T; t += blockDim.x) row_tok[n_pairs + t] = t;
  if (tid == 0) {
    ctrl->n_units = n_runits + nsh;
    ctrl->mid_pairs = n_pairs;
    if (s_dup) set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, -2);
  }
}

// One 256-wide K step of 16 weight rows for every column tile: the same fragment decode and MMA-K
// order as mma_step, each dequantized fragment used for all `nt` tiles. xb: the lane's column g of
// tile 0 at the step's chunk (tile j is 8 * j columns further, tstride halves apart).
template <int QT>
__device__ __forceinline__ void gu_step_tiles(float acc[kMaxTiles][4], const StepFrag &f, const __half *xb,
                                              int tstride, int nt) {
  // each MMA's four A registers are dequantized right before it
  auto tiles = [&](const uint32_t a[4], int off) {
#pragma unroll
    for (int j = 0; j < kMaxTiles; ++j)
      if (j < nt) {
        const uint2 bv = *reinterpret_cast<const uint2 *>(xb + j * tstride + off);
        mma16816(acc[j], a, bv.x, bv.y);
      }
  };
  if constexpr (QT == 4) {
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
        tiles(a, 8 * wq + 4 * mm);
      }
    }
  } else {
#pragma unroll
    for (int wq = 0; wq < 4; ++wq) {
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
        tiles(a, 16 * wq + 4 * mm);
      }
    }
  }
}

// One 128-wide half step (the lane's 32-weight block) of 16 down rows for every column tile, as
// mma_half_step; hb: the lane's column g of tile 0 at its block
template <int QT>
__device__ __forceinline__ void dn_half_tiles(float acc[kMaxTiles][4], const HalfFrag &f, const __half *hb,
                                              int tstride, int nt) {
  const __half2 dd0 = __half2half2(__ushort_as_half(f.d0));
  const __half2 dd1 = __half2half2(__ushort_as_half(f.d1));
  auto tiles = [&](const uint32_t a[4], int off) {
#pragma unroll
    for (int j = 0; j < kMaxTiles; ++j)
      if (j < nt) {
        const uint2 bv = *reinterpret_cast<const uint2 *>(hb + j * tstride + off);
        mma16816(acc[j], a, bv.x, bv.y);
      }
  };
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
        tiles(a, 8 * wq + 4 * mm);
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
        tiles(a, 16 * wq + 4 * mm);
      }
    }
  }
}

// gate/up steps whose loads go out together (register budget: Q2 fragments are the smallest)
template <int QT>
constexpr int gu_batch() { return QT == 2 ? 4 : 2; }
// down row blocks whose loads go out together
template <int QT>
constexpr int dn_batch() { return QT == 4 ? 2 : 4; }

template <int QT>
__global__ void __launch_bounds__(kMxThreads, 1)
mid_expert_kernel(const uint16_t *__restrict__ x, int H, int I, int NT, moe_expert_set routed, moe_expert_set shared,
                  const MidUnit *__restrict__ units, const int32_t *__restrict__ row_tok, int n_rows,
                  float *__restrict__ part, Ctrl *__restrict__ ctrl) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int XS = mid_stride(H), HS = mid_stride(kMidFS);
  __half *xs = reinterpret_cast<__half *>(smem_raw);  // [NT][XS] the unit's tokens
  __half *hsm = xs + (size_t)NT * XS;                  // [NT][HS] the item's h
  __shared__ MidUnit s_un;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  pdl_wait();
  pdl_launch_dependents();
  const int S = I / kMidFS;
  const int n_items = ctrl->n_units * S;
  const int nsteps = (H + kStepK - 1) / kStepK;
  constexpr int NS = gu_batch<QT>(), ND = dn_batch<QT>();
  bool bad = false;
  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int u = it / S, sl = it % S;
    __syncthreads();  // the previous item's reads of xs, hsm and s_un are done
    if (threadIdx.x == 0) s_un = units[u];
    __syncthreads();
    const int expert = s_un.expert, set = s_un.set, ncol = s_un.ncol, row0 = s_un.row0;
    const int nexp = set ? shared.gate.n_experts : routed.gate.n_experts;
    if (expert < 0 || expert >= nexp || ncol < 1 || ncol > NT || row0 < 0 || row0 + ncol > n_rows) {
      if (threadIdx.x == 0 && sl == 0) set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, expert);
      continue;
    }
    const int nt = (ncol + 7) >> 3;
    const MatView mg = mat_sel(routed, shared, set, 0, expert);
    const MatView mu = mat_sel(routed, shared, set, 1, expert);
    const int fr = sl * kMidFS + 8 * warp + g;  // this lane's feature (gate row and up row)
    float acc[kMaxTiles][4];
#pragma unroll
    for (int j = 0; j < kMaxTiles; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
    const __half *xlane = xs + (size_t)g * XS + 80 * t;  // column g, the lane's chunk of step 0
    for (int s0 = 0; s0 < nsteps; s0 += NS) {
      StepFrag f[NS];
#pragma unroll
      for (int j = 0; j < NS; ++j) load_step_pair<QT>(f[j], mg, fr, mu, fr, s0 + j, s0 + j < nsteps);
      if (s0 == 0) {
        // the tokens are staged while the first batch of weights is in flight: 16-byte loads, all
        // of a thread's issued before its stores; columns beyond ncol up to the tile are zero
        const int H8 = H / 8, n = nt * 8 * H8;
        for (int i0 = threadIdx.x; i0 < n; i0 += 4 * kMxThreads) {
          uint4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kMxThreads, c = i / H8;
            v[j] = (i < n && c < ncol)
                       ? __ldg(reinterpret_cast<const uint4 *>(x + (size_t)row_tok[row0 + c] * H) + i % H8)
                       : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kMxThreads;
            if (i >= n) break;
            const uint32_t in[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              __half2 h2 = __floats2half2_rn(__uint_as_float(in[q] << 16), __uint_as_float(in[q] & 0xffff0000u));
              o[q] = *reinterpret_cast<uint32_t *>(&h2);
              bad |= f16x2_inf(o[q]);
            }
            uint2 *d = reinterpret_cast<uint2 *>(xs + (size_t)(i / H8) * XS + mid_pos(8 * (i % H8)));
            d[0] = make_uint2(o[0], o[1]);
            d[1] = make_uint2(o[2], o[3]);
          }
        }
        __syncthreads();
      }
#pragma unroll
      for (int j = 0; j < NS; ++j)
        if (s0 + j < nsteps && (s0 + j) * kStepK + 64 * t < H)
          gu_step_tiles<QT>(acc, f[j], xlane + 320 * (s0 + j), 8 * XS, nt);
    }
    // lane (g, t), tile j: gate of feature fr at columns 8j + 2t, 8j + 2t + 1 in acc[j][0..1], its up
    // in acc[j][2..3]
    {
      const int fp = mid_pos(8 * warp + g);
#pragma unroll
      for (int j = 0; j < kMaxTiles; ++j)
        if (j < nt) {
          const float g0 = acc[j][0], g1 = acc[j][1], u0 = acc[j][2], u1 = acc[j][3];
          const __half h0 = __float2half_rn(g0 / (1.0f + expf(-g0)) * u0);
          const __half h1 = __float2half_rn(g1 / (1.0f + expf(-g1)) * u1);
          bad |= f16_inf(__half_as_ushort(h0)) || f16_inf(__half_as_ushort(h1));
          hsm[(size_t)(8 * j + 2 * t) * HS + fp] = h0;
          hsm[(size_t)(8 * j + 2 * t + 1) * HS + fp] = h1;
        }
    }
    // down: row blocks warp, warp + kMxWarps, ...; K = this slice's 128 columns of the down rows
    const MatView md = mat_sel(routed, shared, set, 2, expert);
    const int nrb = H / 16;
    const int kk = sl * kMidFS + 32 * t;
    const __half *hlane = hsm + (size_t)g * HS + 32 * t + 16 * (t >> 1);  // = mid_pos(32 t)
    float *pbase = part + ((size_t)sl * n_rows + row0) * H;
    HalfFrag fd[ND];
    auto load_batch = [&](int b0) {
#pragma unroll
      for (int j = 0; j < ND; ++j) {
        const int rb = b0 + j * kMxWarps;
        if (rb < nrb) load_half<QT>(fd[j], md, rb * 16, kk);
      }
    };
    load_batch(warp);  // the first batch's loads go out before the wait for h
    __syncthreads();   // h complete
    for (int b0 = warp; b0 < nrb; b0 += ND * kMxWarps) {
      if (b0 != warp) load_batch(b0);
#pragma unroll
      for (int jb = 0; jb < ND; ++jb) {
        const int rb = b0 + jb * kMxWarps;
        if (rb >= nrb) break;
        float d[kMaxTiles][4];
#pragma unroll
        for (int j = 0; j < kMaxTiles; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[j][e] = 0.f;
        dn_half_tiles<QT>(d, fd[jb], hlane, 8 * HS, nt);
        const int row = rb * 16 + g;
#pragma unroll
        for (int j = 0; j < kMaxTiles; ++j) {
          const int c0 = 8 * j + 2 * t;
          if (c0 < ncol) {
            float *pr = pbase + (size_t)c0 * H;
            pr[row] = d[j][0];
            pr[row + 8] = d[j][2];
          }
          if (c0 + 1 < ncol) {
            float *pr = pbase + (size_t)(c0 + 1) * H;
            pr[row] = d[j][1];
            pr[row + 8] = d[j][3];
          }
        }
      }
    }
  }
  if (bad) set_device_error(ctrl, MOE_ERR_RANGE, 60);
}

// one thread per 4 consecutive outputs of a token
__global__ void __launch_bounds__(256)
mid_combine_kernel(const float *__restrict__ part, int S, int n_rows, const int32_t *__restrict__ row_of,
                   int has_shared, const float *__restrict__ w, int T, int k, int H,
                   const float *__restrict__ residual, float *__restrict__ y, Ctrl *__restrict__ ctrl) {
  pdl_wait();
  pdl_launch_dependents();
  // the token's partial-row indices and weights, staged once per CTA (one round trip), so each
  // slot below costs only its partial rows' loads
  __shared__ int s_r[kMaxK + 1];
  __shared__ float s_w[kMaxK];
  const int t = blockIdx.x, h4 = blockIdx.y * blockDim.x + threadIdx.x;
  if (threadIdx.x < k && t < T) {
    s_r[threadIdx.x] = row_of[t * k + threadIdx.x];
    s_w[threadIdx.x] = w[t * k + threadIdx.x];
  }
  if (threadIdx.x == 0 && t < T) s_r[k] = has_shared ? ctrl->mid_pairs + t : -1;
  __syncthreads();
  if (t >= T || 4 * h4 >= H) return;
  const size_t slice = (size_t)n_rows * H;
  auto row_sum = [&](int r) {
    const float *p = part + (size_t)r * H + 4 * h4;
    float4 a = __ldcg(reinterpret_cast<const float4 *>(p));
    for (int s = 1; s < S; ++s) {
      const float4 b = __ldcg(reinterpret_cast<const float4 *>(p + s * slice));
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    return a;
  };
  float4 acc = residual ? __ldg(reinterpret_cast<const float4 *>(residual + (size_t)t * H) + h4)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int j = 0; j < k; ++j) {
    const int r = s_r[j];
    if (r < 0) continue;
    const float wj = s_w[j];
    const float4 v = row_sum(r);
    acc.x = fmaf(wj, v.x, acc.x);
    acc.y = fmaf(wj, v.y, acc.y);
    acc.z = fmaf(wj, v.z, acc.z);
    acc.w = fmaf(wj, v.w, acc.w);
  }
  if (has_shared) {
    const float4 v = row_sum(s_r[k]);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  if (!isfinite(acc.x) || !isfinite(acc.y) || !isfinite(acc.z) || !isfinite(acc.w))
    set_device_error(ctrl, MOE_ERR_RANGE, 61);
  reinterpret_cast<float4 *>(y + (size_t)t * H)[h4] = acc;
}

size_t mid_expert_smem(int H) {
  const int NT = mid_unit_tokens(H);
  return (size_t)NT * (mid_stride(H) + mid_stride(kMidFS)) * 2;
}

template <int QT>
cudaError_t launch_mx(int H, int I, const uint16_t *x, const moe_expert_set &routed, const moe_expert_set &sh,
                      const MidUnit *units, const int32_t *row_tok, int n_rows, float *part, Ctrl *ctrl,
                      cudaStream_t s) {
  const size_t smem = mid_expert_smem(H);
  cudaError_t e = smem_limit_once(mid_expert_kernel<QT>, smem);
  if (e != cudaSuccess) return e;
  KTimer kt_(KID_MID_EXPERT, s);
  return launch_pdl(mid_expert_kernel<QT>, dim3(num_sms()), dim3(kMxThreads), smem, s, x, H, I, mid_unit_tokens(H),
                    routed, sh, units, row_tok, n_rows, part, ctrl);
}

}  // namespace

bool mid_shape_supported(int T, int H, int E, int I) {
  return T >= 1 && T <= kMidMaxT && H % 64 == 0 && H <= kMidMaxH && I % kMidFS == 0 && E <= kMaxE;
}

cudaError_t launch_mid_ffn(const uint16_t *x, int T, int H, int E, int k, int I, const int32_t *idx, const float *w,
                           const moe_expert_set &routed, const moe_expert_set *shared, const float *residual, float *y,
                           MidUnit *units, int32_t *row_of, int32_t *row_tok, float *part, Ctrl *ctrl,
                           cudaStream_t s) {
  if (!mid_shape_supported(T, H, E, I)) return cudaErrorNotSupported;
  const int hs = shared ? 1 : 0;
  const int n_rows = T * k + hs * T;
  {
    const size_t smem = (size_t)E * 6 * 4;
    cudaError_t e = smem_limit_once(mid_plan_kernel, smem);
    if (e != cudaSuccess) return e;
    KTimer kt_(KID_MID_PLAN, s);
    e = launch_pdl(mid_plan_kernel, dim3(1), dim3(kPlanThreads), smem, s, idx, T, k, E, hs, mid_unit_tokens(H),
                   I / kMidFS, num_sms(), units, row_of, row_tok, ctrl);
    if (e != cudaSuccess) return e;
  }
  const moe_expert_set sh = shared ? *shared : routed;
  const int qt = routed.gate.qtype;
  cudaError_t e = qt == MOE_Q3   ? launch_mx<3>(H, I, x, routed, sh, units, row_tok, n_rows, part, ctrl, s)
                  : qt == MOE_Q4 ? launch_mx<4>(H, I, x, routed, sh, units, row_tok, n_rows, part, ctrl, s)
                                 : launch_mx<2>(H, I, x, routed, sh, units, row_tok, n_rows, part, ctrl, s);
  if (e != cudaSuccess) return e;
  KTimer kt_(KID_MID_COMBINE, s);
  return launch_pdl(mid_combine_kernel, dim3(T, (H / 4 + 255) / 256), dim3(256), 0, s, part, I / kMidFS, n_rows,
                    row_of, hs, w, T, k, H, residual, y, ctrl);
}

}  // namespace moe
