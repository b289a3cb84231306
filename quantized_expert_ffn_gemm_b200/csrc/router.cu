// Router + top-k.
//
// Each token is scored against every routed expert and sent to the k best ("Strata vs Llama.cpp
// vs vLLM", chapter "How Strata is designed to work": 10 of 512 experts per layer). Logits are
// fp32 (x is exact in fp32), the top-k is taken on the fp32 logits with the lower expert index
// winning ties, slots are stored in descending logit order, and the weights are the softmax
// restricted to the selected set (the full softmax renormalised over the set).
//
// Decode (T <= 8): one kernel. Every warp produces whole logits (one expert, all T tokens,
// Wr read once with 128-bit loads); the last CTA to finish (atomic ticket) runs the top-k and,
// for the decode expert path, groups the selected (token, slot) pairs by distinct expert.
// 9..128 tokens: fp32 dot products with each expert's row held in registers, then one warp per
// token for the top-k. Prefill: tensor-core logits with an exact refine of the candidates near
// the k-th (or a tiled fp32 GEMM where that path does not apply), then the top-k.
#include "common.cuh"
#include "topk.cuh"

namespace moe {

// ---------------------------------------------------------------- decode router kernel
constexpr int kRouterDecWarps = 4;

__global__ void __launch_bounds__(kRouterDecWarps * 32)
router_decode_kernel(const uint16_t *__restrict__ x, int T, int H, const float *__restrict__ Wr,
                     const float *__restrict__ bias, int E, int k, int32_t *__restrict__ idx, float *__restrict__ w,
                     float *__restrict__ logits, int build, int has_shared, DecUnit *__restrict__ units,
                     Ctrl *__restrict__ ctrl) {
  extern __shared__ float4 smem4[];
  float *xs = reinterpret_cast<float *>(smem4);  // [T][H] fp32, later reused for [T][E] logits
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  {  // 16-byte loads of x, all of a thread's loads issued before its stores
    const int n8 = T * H / 8;
    for (int i0 = tid; i0 < n8; i0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        v[j] = (i < n8) ? __ldg(reinterpret_cast<const uint4 *>(x) + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        if (i < n8) {
          float4 *d = reinterpret_cast<float4 *>(xs + 8 * i);
          d[0] = make_float4(__uint_as_float(v[j].x << 16), __uint_as_float(v[j].x & 0xffff0000u),
                             __uint_as_float(v[j].y << 16), __uint_as_float(v[j].y & 0xffff0000u));
          d[1] = make_float4(__uint_as_float(v[j].z << 16), __uint_as_float(v[j].z & 0xffff0000u),
                             __uint_as_float(v[j].w << 16), __uint_as_float(v[j].w & 0xffff0000u));
        }
      }
    }
  }
  __syncthreads();

  const int H4 = H >> 2;
  for (int e = blockIdx.x * kRouterDecWarps + warp; e < E; e += gridDim.x * kRouterDecWarps) {
    const float4 *wr = reinterpret_cast<const float4 *>(Wr + (size_t)e * H);
    float acc[kDecodeMaxT];
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) acc[t] = 0.0f;
    for (int h0 = 0; h0 < H4; h0 += 32 * 16) {  // H = 2048: the whole row in one round of loads
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        int h4 = h0 + lane + 32 * u;
        v[u] = (h4 < H4) ? __ldcs(wr + h4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        int h4 = h0 + lane + 32 * u;
        if (h4 < H4) {
#pragma unroll
          for (int t = 0; t < kDecodeMaxT; ++t) {
            if (t < T) {
              float4 xv = reinterpret_cast<const float4 *>(xs + (size_t)t * H)[h4];
              acc[t] = fmaf(v[u].x, xv.x, acc[t]);
              acc[t] = fmaf(v[u].y, xv.y, acc[t]);
              acc[t] = fmaf(v[u].z, xv.z, acc[t]);
              acc[t] = fmaf(v[u].w, xv.w, acc[t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) {
      if (t < T) {
        float s = warp_sum(acc[t]);
        if (lane == 0) logits[(size_t)t * E + e] = s;
      }
    }
  }

  // last CTA to arrive does the top-k
  __shared__ unsigned s_last;
  __threadfence();
  __syncthreads();
  // atomicInc wraps the ticket back to 0 when the last CTA takes it
  if (tid == 0) s_last = (atomicInc(&ctrl->router_ticket, gridDim.x - 1) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float *ls = xs;  // [T][E]
  if ((E & 3) == 0) {
    for (int i = tid; i < T * E / 4; i += blockDim.x)
      reinterpret_cast<float4 *>(ls)[i] = __ldcg(reinterpret_cast<const float4 *>(logits) + i);
  } else {
    for (int i = tid; i < T * E; i += blockDim.x) ls[i] = __ldcg(logits + i);
  }
  __shared__ int32_t s_idx[kDecodeMaxT * kMaxK];
  __shared__ float s_w[kDecodeMaxT * kMaxK];
  __shared__ uint32_t s_taken[kRouterDecWarps][kMaxE / 32];
  __syncthreads();
  for (int t = warp; t < T; t += kRouterDecWarps) {
    if (E <= 512) {
      warp_topk<16>(ls + (size_t)t * E, bias, E, k, s_idx + t * k, s_w + t * k);
    } else {
      for (int i = lane; i < kMaxE / 32; i += 32) s_taken[warp][i] = 0;
      __syncwarp();
      warp_topk_generic(ls + (size_t)t * E, bias, E, k, s_idx + t * k, s_w + t * k, s_taken[warp]);
    }
  }
  __syncthreads();
  for (int i = tid; i < T * k; i += blockDim.x) {
    idx[i] = s_idx[i];
    w[i] = s_w[i];
  }
  if (bias) {  // logits output includes the bias
    for (int i = tid; i < T * E; i += blockDim.x) logits[i] = ls[i] + bias[i % E];
  }
  if (build) {  // every thread of this (last) CTA takes part
    __shared__ UnitScratch s_us;
    build_units(s_idx, s_w, T, k, E, has_shared, units, &ctrl->n_units, s_us);
  }
}

cudaError_t launch_router_decode(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k,
                                 int32_t *idx, float *w, float *logits, int build_units_flag, int has_shared,
                                 DecUnit *units, Ctrl *ctrl, cudaStream_t s) {
  size_t smem = (size_t)T * (H > E ? H : E) * sizeof(float);
  int grid = (E + kRouterDecWarps - 1) / kRouterDecWarps;
  cudaError_t e = smem_limit_once(router_decode_kernel, smem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_ROUTER_DECODE, s);
    router_decode_kernel<<<grid, kRouterDecWarps * 32, smem, s>>>(x, T, H, Wr, bias, E, k, idx, w, logits,
                                                                 build_units_flag, has_shared, units, ctrl);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- prefill: fp32 logits GEMM
// C[T][E] = X[T][H] Wr[E][H]^T, 128x128 tile per CTA, 256 threads, 8x8 outputs per thread,
// K-steps of 16 staged k-major in shared memory (double buffered).
constexpr int RBM = 128, RBN = 128, RBK = 16;

__global__ void __launch_bounds__(256)
router_gemm_kernel(const uint16_t *__restrict__ x, int T, int H, const float *__restrict__ Wr, int E,
                   float *__restrict__ C) {
  __shared__ __align__(16) float As[2][RBK][RBM + 4];
  __shared__ __align__(16) float Bs[2][RBK][RBN + 4];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * RBM, n0 = blockIdx.x * RBN;
  const int ty = tid / 16, tx = tid % 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  // loaders: A: 128 rows x 16 bf16 = 256 threads x 8 values (16 bytes); B: 128 rows x 16 fp32 = 256 x 8
  const int lrow = tid >> 1, lk = (tid & 1) * 8;
  auto load_regs = [&](int k0, uint4 &ra, float4 &rb0, float4 &rb1) {
    int gm = m0 + lrow, gn = n0 + lrow;
    ra = (gm < T) ? *reinterpret_cast<const uint4 *>(x + (size_t)gm * H + k0 + lk) : make_uint4(0, 0, 0, 0);
    if (gn < E) {
      const float4 *p = reinterpret_cast<const float4 *>(Wr + (size_t)gn * H + k0 + lk);
      rb0 = __ldg(p);
      rb1 = __ldg(p + 1);
    } else {
      rb0 = rb1 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store_smem = [&](int buf, const uint4 &ra, const float4 &rb0, const float4 &rb1) {
    const uint32_t av[4] = {ra.x, ra.y, ra.z, ra.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      As[buf][lk + 2 * i][lrow] = __uint_as_float(av[i] << 16);
      As[buf][lk + 2 * i + 1][lrow] = __uint_as_float(av[i] & 0xffff0000u);
    }
    Bs[buf][lk + 0][lrow] = rb0.x; Bs[buf][lk + 1][lrow] = rb0.y;
    Bs[buf][lk + 2][lrow] = rb0.z; Bs[buf][lk + 3][lrow] = rb0.w;
    Bs[buf][lk + 4][lrow] = rb1.x; Bs[buf][lk + 5][lrow] = rb1.y;
    Bs[buf][lk + 6][lrow] = rb1.z; Bs[buf][lk + 7][lrow] = rb1.w;
  };
  uint4 ra;
  float4 rb0, rb1;
  load_regs(0, ra, rb0, rb1);
  store_smem(0, ra, rb0, rb1);
  __syncthreads();
  const int nk = H / RBK;
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load_regs((kt + 1) * RBK, ra, rb0, rb1);
#pragma unroll
    for (int kk = 0; kk < RBK; ++kk) {
      float a[8], b[8];
      float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4]);
      float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][64 + ty * 4]);
      float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4]);
      float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w; a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w; b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nk) store_smem(buf ^ 1, ra, rb0, rb1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (gm >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (gn < E) C[(size_t)gm * E + gn] = acc[i][j];
    }
  }
}

// one warp per token; adds the bias into the stored logits
constexpr int kTopkWarps = 8;
__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(float *__restrict__ logits, const float *__restrict__ bias, int T, int E, int k, int32_t *__restrict__ idx,
            float *__restrict__ w) {
  __shared__ uint32_t s_taken[kTopkWarps][kMaxE / 32];
  // launched behind the router (programmatic stream serialization): its logits are read after the wait
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= T) return;
  float *l = logits + (size_t)t * E;
  if (E <= 512) {  // the biased logits go back as they are formed (each lane rewrites only its own)
    warp_topk<16>(l, bias, E, k, idx + (size_t)t * k, w + (size_t)t * k, bias ? l : nullptr);
  } else {
    for (int i = lane; i < kMaxE / 32; i += 32) s_taken[warp][i] = 0;
    __syncwarp();
    warp_topk_generic(l, bias, E, k, idx + (size_t)t * k, w + (size_t)t * k, s_taken[warp]);
    __syncwarp();
    if (bias)
      for (int e = lane; e < E; e += 32) l[e] += bias[e];
  }
}

// ---------------------------------------------------------------- screen + exact refine
// After the tensor-core logits (accurate to ~1e-5 only: the tensor core's fp32 accumulation over
// 3H terms is not an fp32 FMA chain), every expert whose approximate logit is within kMargin of
// the approximate k-th logit is a candidate; the exact top-k is always among them because the
// margin is far above twice the approximation error. Candidates get their logit recomputed with
// an fp32 dot product (x is exact in fp32) plus bias, the top-k (lower index wins ties) and the
// weights are taken from those exact values, and the exact values are written back.
constexpr float kRefineMargin = 2e-3f;
constexpr int kRefineWarps = 8;

__global__ void __launch_bounds__(kRefineWarps * 32)
topk_refine_kernel(float *__restrict__ logits, const uint16_t *__restrict__ x, const float *__restrict__ Wr,
                   const float *__restrict__ bias, int T, int H, int E, int k, int32_t *__restrict__ idx,
                   float *__restrict__ w) {
  __shared__ float s_ex[kRefineWarps][512];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRefineWarps + warp;
  if (t >= T) return;
  float *l = logits + (size_t)t * E;
  // approximate logits (bias included) and the approximate k-th value
  float val[16];
  uint32_t key[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int e = lane + 32 * i;
    val[i] = (e < E) ? l[e] : -INFINITY;
    key[i] = (e < E) ? logit_key(val[i]) : 0u;
  }
  uint32_t taken = 0;
  float vk = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;
    int bi = 0x7fffffff;
    float bv = -INFINITY;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = lane + 32 * i;
      const bool ok = (e < E) && !((taken >> i) & 1u);
      if (ok && (key[i] > bk || bi == 0x7fffffff)) { bk = key[i]; bi = e; bv = val[i]; }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bi == 0x7fffffff ? 0u : bk);
    const uint32_t cand = (bi != 0x7fffffff && bk == m) ? (uint32_t)bi : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if ((uint32_t)bi == win) taken |= 1u << ((bi - lane) / 32);
    vk = __shfl_sync(0xffffffffu, bv, (int)(win & 31u));
  }
  const float thr = vk - kRefineMargin;
  // x row in registers (fp32, exact), lane holds h = 4 * (lane + 32 j)
  float4 xr[16];
  const int H4 = H / 4;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int h4 = lane + 32 * j;
    if (h4 < H4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(x + (size_t)t * H) + h4);
      xr[j] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                          __uint_as_float(v.y & 0xffff0000u));
    } else {
      xr[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  float *ex = s_ex[warp];
  for (int e = lane; e < E; e += 32) ex[e] = -INFINITY;
  __syncwarp();
  // candidate c's exact value is also kept by lane c (the first 32), so the final top-k is one
  // 32-wide sort of the candidates instead of k rounds over all E entries
  int nc = 0, ce = 0;
  float cv = -INFINITY;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    unsigned bal = __ballot_sync(0xffffffffu, (lane + 32 * i < E) && val[i] >= thr);
    while (bal) {
      const int e = (__ffs(bal) - 1) + 32 * i;
      bal &= bal - 1;
      const float4 *wr = reinterpret_cast<const float4 *>(Wr + (size_t)e * H);
      float acc = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int h4 = lane + 32 * j;
        if (h4 < H4) {
          const float4 wv = __ldg(wr + h4);
          acc = fmaf(wv.x, xr[j].x, acc);
          acc = fmaf(wv.y, xr[j].y, acc);
          acc = fmaf(wv.z, xr[j].z, acc);
          acc = fmaf(wv.w, xr[j].w, acc);
        }
      }
      acc = warp_sum(acc);
      const float v = acc + (bias ? bias[e] : 0.0f);
      if (lane == 0) ex[e] = v;
      if (lane == nc) {  // nc is warp-uniform
        ce = e;
        cv = v;
      }
      ++nc;
    }
  }
  if (nc <= 32) {  // the top-k is among the candidates (every approximate top-k value is >= thr)
    unsigned long long code = (lane < nc) ? topk_code(cv, ce) : 0ull;
    code = warp_sort32_desc(code);
    const float my_val = key_to_logit((uint32_t)(code >> 32));
    const int my_idx = (int)(0xFFFFFFFFu - (uint32_t)code);
    topk_finish(my_val, my_idx, k, idx + (size_t)t * k, w + (size_t)t * k);
    if (lane < nc) l[ce] = cv;  // exact values where computed
    return;
  }
  __syncwarp();  // more than 32 candidates (a crowd of near-equal logits): over all E entries
  warp_topk<16>(ex, nullptr, E, k, idx + (size_t)t * k, w + (size_t)t * k);
  __syncwarp();
  for (int e = lane; e < E; e += 32)  // exact values where computed
    if (ex[e] != -INFINITY) l[e] = ex[e];
}

bool router_refine_supported(int H, int E) { return H <= 2048 && E <= 512; }

// ---------------------------------------------------------------- small batches (9..128 tokens)
// Plain fp32 dot products on the CUDA cores: at these sizes the tensor-core router's fixed costs
// (splitting Wr into planes, a K loop over 3H, the exact refine) dominate. A CTA takes 4 experts;
// warp (e, half) keeps its expert's fp32 row in registers (Wr read once). The tokens pass
// through shared memory in chunks of 8, the next chunk's async copies in flight while the current
// one is used, so each CTA reads x from L2 once (not once per expert) and every chunk costs one
// round trip at most; warp half h takes tokens 4h..4h+3 of a chunk. The logits are exact fp32 dot
// products (no refine needed); the bias is added by the top-k kernel.
constexpr int kRouterMidMaxT = 128;
constexpr int kRouterMidWarps = 8;
constexpr int kRmChunk = 8;  // tokens per staged chunk

__device__ __forceinline__ void rm_cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kRouterMidWarps * 32)
router_mid_kernel(const uint16_t *__restrict__ x, int T, int H, const float *__restrict__ Wr, int E,
                  float *__restrict__ logits) {
  extern __shared__ __align__(16) uint16_t s_xc[];  // [2][kRmChunk][H] bf16
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e = blockIdx.x * 4 + (warp & 3), half = warp >> 2;
  const bool has_e = e < E;  // every thread takes part in the staging and the barriers
  const int H4 = H >> 2;     // H <= 2048: at most 16 float4 per lane
  const float4 *wr = reinterpret_cast<const float4 *>(Wr + (size_t)(has_e ? e : 0) * H);
  float4 wv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int h4 = lane + 32 * j;
    wv[j] = (has_e && h4 < H4) ? __ldg(wr + h4) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // the router rows are weights, which no kernel of this library writes: they are requested before
  // the wait for the previous kernel, whose output (the tokens) is read after it
  pdl_launch_dependents();
  pdl_wait();
  const int nchunk = (T + kRmChunk - 1) / kRmChunk;
  auto stage = [&](int c) {  // chunk c's rows into buffer c % 2, 16-byte async copies
    const int t0 = c * kRmChunk, n16 = min(kRmChunk, T - t0) * H / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t0 * H);
    const uint32_t dst = (uint32_t)__cvta_generic_to_shared(s_xc + (size_t)(c & 1) * kRmChunk * H);
    for (int i = tid; i < n16; i += kRouterMidWarps * 32) rm_cp_async16(dst + 16u * i, src + i);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  stage(0);
  for (int c = 0; c < nchunk; ++c) {
    if (c + 1 < nchunk) {
      stage(c + 1);  // into the buffer chunk c - 1 used, freed by the barrier ending its iteration
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint16_t *xb = s_xc + (size_t)(c & 1) * kRmChunk * H;
    const int t0 = c * kRmChunk, nt = min(kRmChunk, T - t0);
    if (has_e) {
#pragma unroll 1
      for (int tt = 4 * half; tt < 4 * half + 4 && tt < nt; ++tt) {
        const uint2 *xr = reinterpret_cast<const uint2 *>(xb + (size_t)tt * H);
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int h4 = lane + 32 * j;
          const uint2 xv = (h4 < H4) ? xr[h4] : make_uint2(0u, 0u);
          acc = fmaf(wv[j].x, __uint_as_float(xv.x << 16), acc);
          acc = fmaf(wv[j].y, __uint_as_float(xv.x & 0xffff0000u), acc);
          acc = fmaf(wv[j].z, __uint_as_float(xv.y << 16), acc);
          acc = fmaf(wv[j].w, __uint_as_float(xv.y & 0xffff0000u), acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) logits[(size_t)(t0 + tt) * E + e] = acc;
      }
    }
    __syncthreads();  // this buffer is refilled two chunks on
  }
}

cudaError_t launch_router_prefill(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k,
                                  int32_t *idx, float *w, float *logits, uint16_t *wsplit, Ctrl *ctrl, cudaStream_t s) {
  cudaError_t e;
  if (T <= kRouterMidMaxT && H <= 2048) {
    {
      KTimer kt_(KID_ROUTER_GEMM, s);
      const size_t smem = (size_t)2 * kRmChunk * H * 2;
      if ((e = smem_limit_once(router_mid_kernel, smem)) != cudaSuccess) return e;
      e = launch_pdl(router_mid_kernel, dim3((E + 3) / 4), dim3(kRouterMidWarps * 32), smem, s, x, T, H, Wr, E,
                     logits);
      if (e != cudaSuccess) return e;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
      KTimer kt_(KID_TOPK, s);
      e = launch_pdl(topk_kernel, dim3((T + kTopkWarps - 1) / kTopkWarps), dim3(kTopkWarps * 32), 0, s, logits, bias,
                     T, E, k, idx, w);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  if (router_tc_supported(H, E) && router_refine_supported(H, E)) {
    e = launch_router_tc(x, T, H, Wr, bias, E, wsplit, logits, ctrl, s);  // logits include the bias
    if (e != cudaSuccess) return e;
    {
      KTimer kt_(KID_TOPK, s);
      topk_refine_kernel<<<(T + kRefineWarps - 1) / kRefineWarps, kRefineWarps * 32, 0, s>>>(logits, x, Wr, bias, T,
                                                                                         H, E, k, idx, w);
    }
    return cudaGetLastError();
  }
  const float *topk_bias = bias;
  {
    dim3 grid((E + RBN - 1) / RBN, (T + RBM - 1) / RBM);
    {
      KTimer kt_(KID_ROUTER_GEMM, s);
      router_gemm_kernel<<<grid, 256, 0, s>>>(x, T, H, Wr, E, logits);
    }
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_TOPK, s);
    topk_kernel<<<(T + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, s>>>(logits, topk_bias, T, E, k, idx, w);
  }
  return cudaGetLastError();
}

}  // namespace moe
