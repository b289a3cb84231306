// Fused decode / MTP-verify layer (1-8 tokens): one cooperative kernel per MoE layer.
//
// A decode step is bound by reading weights ("Strata vs Llama.cpp vs vLLM", chapter "Why LLM
// inference is a systems problem"), and at 1-4 tokens a layer moves only ~15 MB, so separate
// router / gate-up / down kernels spend most of their time in launch gaps and dependent memory
// round trips. Here one grid of one CTA per SM runs the three phases with two grid barriers:
//   P1  router logits: four warps per expert split H (128-bit loads of the fp32 router rows);
//       meanwhile the always-on shared expert's gate/up rows are prefetched into L2.
//   --  grid barrier
//   P1b every CTA computes the same top-k (partial top-k of 32-expert slices in all warps, then
//       one merge warp per token) and distinct-expert unit list from the logits (deterministic),
//       so no second exchange is needed; each CTA prefetches into L2 the down-projection rows it
//       will need in P3.
//   P2  gate/up + SwiGLU: one (unit, 16-row block) group per CTA at a time, 16 warps = gate/up x
//       8 K steps on the tensor cores (mma.sync, fp16 operands, fp32 accumulate), the next
//       group's weights requested before the current one is computed; h goes to the workspace.
//   --  grid barrier
//   P3  down projection fused with the weighted combine: each CTA owns 16 output features, its
//       warps split the (unit, K step) items, partials are reduced in fixed order (no atomics).
// The grid barrier is one 64-bit arrival counter in the workspace (every launch adds 2 x grid;
// a CTA waits for the launch's base + j x grid); its wait is bounded in time and reports
// MOE_ERR_TIMEOUT instead of hanging. Cross-CTA data is read with L1-bypassing loads.
#include "common.cuh"
#include "dequant.cuh"
#include "gemv.cuh"
#include "tc.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kFWarps = 16;
constexpr int kFThreads = kFWarps * 32;
constexpr int kFMaxUnits = kDecodeMaxT * kMaxK + 1;
constexpr int kFSlots = 64;  // h columns (token, expert) of a step staged for the down phase

struct FusedArgs {
  const uint16_t *x;
  int T, H, E, k, I, has_shared;
  const float *Wr;
  const float *bias;
  moe_expert_set routed, shared;
  const float *residual;
  float *y;
  float *logits;
  int32_t *idx;
  float *w;
  uint16_t *hdec;
  Ctrl *ctrl;
};

struct FusedLayout {
  size_t xraw, x16, hs, part, red, units, scratch, sidx, sw, misc, slot, src, plist, total;
};

__host__ __device__ inline size_t fl_align(size_t v) { return (v + 15) & ~(size_t)15; }

__host__ __device__ inline FusedLayout fused_layout(int T, int H, int I) {
  FusedLayout L{};
  size_t o = 0;
  auto take = [&](size_t b) { size_t r = o; o = fl_align(o + b); return r; };
  L.xraw = take((size_t)T * H * 2);
  L.x16 = take((size_t)8 * (H + 4) * 2);
  L.hs = take((size_t)kFSlots * (I + 4) * 2);
  L.part = take((size_t)kFWarps * 16 * 8 * 4);
  L.red = take((size_t)kFWarps * 16 * 8 * 4);
  L.units = take((size_t)kFMaxUnits * sizeof(DecUnit));
  L.scratch = take(sizeof(UnitScratch));
  L.sidx = take((size_t)kDecodeMaxT * kMaxK * 4);
  L.sw = take((size_t)kDecodeMaxT * kMaxK * 4);
  L.misc = take(16 * 4);
  L.slot = take((size_t)(kFMaxUnits + 1) * 4);
  L.src = take((size_t)kFSlots * 4);
  L.plist = take((size_t)2 * kDecodeMaxT * 16 * 16 * 8);  // top-16 code lists (tokens x 32-expert chunks), x2
  L.total = o;
  return L;
}

// all CTAs are co-resident (cooperative launch). Barrier j of a launch completes when the arrival
// counter reaches base + j * nblocks; false when the wait gave up.
__device__ bool grid_barrier(Ctrl *c, unsigned long long target, int where) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(&c->bar_arrivals) : "memory");
    int ok = 1;
    const uint64_t t0 = global_ns();
    while (true) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(&c->bar_arrivals) : "memory");
      if ((long long)(v - target) >= 0) break;
      __nanosleep(32);
      if (global_ns() - t0 > kWaitLimitNs) {
        ok = 0;
        set_device_error(c, MOE_ERR_TIMEOUT, where);
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// prefetch [p, p + bytes) into L2, lines spread over `nthr` threads starting at thread `first`
__device__ __forceinline__ void prefetch_range(const void *p, size_t bytes, int first, int nthr) {
  const char *c = static_cast<const char *>(p);
  for (size_t off = (size_t)first * 128; off < bytes; off += (size_t)nthr * 128) prefetch_l2(c + off);
}

}  // namespace

template <bool Q3>
__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(const FusedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int T = a.T, H = a.H, E = a.E, k = a.k, I = a.I;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const FusedLayout L = fused_layout(T, H, I);
  uint16_t *xraw = reinterpret_cast<uint16_t *>(smem + L.xraw);
  __half *x16 = reinterpret_cast<__half *>(smem + L.x16);
  __half *hs = reinterpret_cast<__half *>(smem + L.hs);
  float *part = reinterpret_cast<float *>(smem + L.part);
  float *red = reinterpret_cast<float *>(smem + L.red);
  DecUnit *su = reinterpret_cast<DecUnit *>(smem + L.units);
  UnitScratch &us = *reinterpret_cast<UnitScratch *>(smem + L.scratch);
  int32_t *s_idx = reinterpret_cast<int32_t *>(smem + L.sidx);
  float *s_w = reinterpret_cast<float *>(smem + L.sw);
  int *misc = reinterpret_cast<int *>(smem + L.misc);
  int *s_slot = reinterpret_cast<int *>(smem + L.slot);
  int *s_src = reinterpret_cast<int *>(smem + L.src);
  unsigned long long *plist = reinterpret_cast<unsigned long long *>(smem + L.plist);
  Ctrl *ctrl = a.ctrl;
  const int xs16 = H + 4;
  const unsigned nblk = gridDim.x;
  __shared__ unsigned long long s_base;
  if (tid == 0) {  // arrivals of earlier launches: a whole number of 2 x grid (before this CTA arrives)
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(&ctrl->bar_arrivals) : "memory");
    s_base = v - v % nblk;
  }

  // ---------------- P0: tokens into shared memory (raw bf16 for the router, fp16 rotated for the MMAs)
  {
    const int H8 = H / 8, n = T * H8;
    for (int i = tid; i < n; i += kFThreads) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.x) + i);
      reinterpret_cast<uint4 *>(xraw)[i] = v;
      const int t = i / H8, c = i % H8;
      const uint32_t in[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __half2 h = __floats2half2_rn(__uint_as_float(in[q] << 16), __uint_as_float(in[q] & 0xffff0000u));
        o[q] = *reinterpret_cast<uint32_t *>(&h);
      }
      uint2 *d = reinterpret_cast<uint2 *>(x16 + (size_t)t * xs16 + xs_pos(8 * c));
      d[0] = make_uint2(o[0], o[1]);
      d[1] = make_uint2(o[2], o[3]);
    }
  }
  {  // into L2 while the router runs: the shared expert's gate/up rows and the router bias
    const int nthr = gridDim.x * kFThreads, first = blockIdx.x * kFThreads + tid;
    if (a.has_shared) {
      const size_t cb = (size_t)I * H / 4, sb = (size_t)I * H / 32 * 2;
      prefetch_range(a.shared.gate.codes, cb, first, nthr);
      prefetch_range(a.shared.up.codes, cb, first, nthr);
      prefetch_range(a.shared.gate.scales, sb, first, nthr);
      prefetch_range(a.shared.up.scales, sb, first, nthr);
      if (Q3) {
        prefetch_range(a.shared.gate.hibits, cb / 2, first, nthr);
        prefetch_range(a.shared.up.hibits, cb / 2, first, nthr);
      }
    }
    if (a.bias) prefetch_range(a.bias, (size_t)E * 4, tid, kFThreads);
  }
  __syncthreads();

  // ---------------- P1: router logits, four warps per expert (each a quarter of H), fp32
  {
    const int H4 = H / 4, HQ = H4 / 4;  // float4 per quarter
    const int es = warp >> 2, qh = warp & 3;
    float *rp = red;  // [4 experts][4 quarters][T]
    for (int e0 = blockIdx.x; e0 < E; e0 += 4 * gridDim.x) {
      const int e = e0 + es * gridDim.x;
      float acc[kDecodeMaxT];
#pragma unroll
      for (int t = 0; t < kDecodeMaxT; ++t) acc[t] = 0.0f;
      if (e < E) {
        const float4 *wr = reinterpret_cast<const float4 *>(a.Wr + (size_t)e * H) + qh * HQ;
        for (int h0 = 0; h0 < HQ; h0 += 32 * 4) {
          float4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int h4 = h0 + lane + 32 * u;
            v[u] = (h4 < HQ) ? __ldcs(wr + h4) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int h4 = h0 + lane + 32 * u;
            if (h4 >= HQ) continue;
#pragma unroll
            for (int t = 0; t < kDecodeMaxT; ++t) {
              if (t < T) {
                const uint2 xb = reinterpret_cast<const uint2 *>(xraw + (size_t)t * H)[qh * HQ + h4];
                acc[t] = fmaf(v[u].x, __uint_as_float(xb.x << 16), acc[t]);
                acc[t] = fmaf(v[u].y, __uint_as_float(xb.x & 0xffff0000u), acc[t]);
                acc[t] = fmaf(v[u].z, __uint_as_float(xb.y << 16), acc[t]);
                acc[t] = fmaf(v[u].w, __uint_as_float(xb.y & 0xffff0000u), acc[t]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kDecodeMaxT; ++t) {
        if (t < T) {
          const float sum = warp_sum(acc[t]);
          if (lane == 0) rp[(es * 4 + qh) * kDecodeMaxT + t] = sum;
        }
      }
      __syncthreads();
      if (tid < 4 * T) {  // fixed-order sum of the four quarters
        const int ee = tid / T, t = tid % T, eg = e0 + ee * gridDim.x;
        if (eg < E) {
          const float* q4 = rp + ee * 4 * kDecodeMaxT;
          a.logits[(size_t)t * E + eg] = (q4[t] + q4[kDecodeMaxT + t]) + (q4[2 * kDecodeMaxT + t] + q4[3 * kDecodeMaxT + t]);
        }
      }
      __syncthreads();
    }
  }
  __threadfence();
  if (!grid_barrier(ctrl, s_base + nblk, 31)) return;

  // ---------------- P1b: top-k and unit list, computed identically by every CTA
  {
    float *ls = reinterpret_cast<float *>(hs);  // T * E floats, before h is staged there
    for (int i = tid; i < T * E; i += kFThreads) ls[i] = __ldcg(a.logits + i) + (a.bias ? __ldg(a.bias + i % E) : 0.f);
    __syncthreads();
    // top-k per token: every 32-expert chunk is sorted by one warp (top 16 kept), then the
    // chunks' lists are merged pairwise (bitonic merge of a list and its partner reversed)
    const int nch = (E + 31) / 32;
    int npow = 1;
    while (npow < nch) npow <<= 1;
    for (int task = warp; task < T * npow; task += kFWarps) {
      const int t = task / npow, c = task % npow, e = c * 32 + lane;
      unsigned long long v = (c < nch && e < E) ? topk_code(ls[(size_t)t * E + e], e) : 0ull;
      v = warp_sort32_desc(v);
      if (lane < 16) plist[(size_t)task * 16 + lane] = v;
    }
    __syncthreads();
    unsigned long long *cur = plist, *nxt = plist + (size_t)kDecodeMaxT * 16 * 16;  // ping-pong halves
    for (int len = npow; len > 1; len >>= 1) {  // lists of each token: len -> len / 2
      for (int task = warp; task < T * (len / 2); task += kFWarps) {
        const int t = task / (len / 2), c = task % (len / 2);
        const unsigned long long *la = cur + ((size_t)t * npow + 2 * c) * 16;
        const unsigned long long *lb = cur + ((size_t)t * npow + 2 * c + 1) * 16;
        unsigned long long v = (lane < 16) ? la[lane] : lb[31 - lane];
        v = warp_merge32_desc(v);
        if (lane < 16) nxt[((size_t)t * npow + c) * 16 + lane] = v;
      }
      __syncthreads();
      unsigned long long *tmp = cur;
      cur = nxt;
      nxt = tmp;
    }
    if (warp < T) {  // list 0 of token `warp` holds its top 16 in descending order
      const unsigned long long v = (lane < k) ? cur[(size_t)warp * npow * 16 + lane] : 0ull;
      const float val = (lane < k) ? key_to_logit((uint32_t)(v >> 32)) : -INFINITY;
      const int ix = (lane < k) ? (int)(0xFFFFFFFFu - (uint32_t)v) : 0;
      topk_finish(val, ix, k, s_idx + warp * k, s_w + warp * k);
    }
    __syncthreads();
    build_units(s_idx, s_w, T, k, E, a.has_shared, su, &misc[0], us);
    if (blockIdx.x == 0)
      for (int i = tid; i < T * k; i += kFThreads) {
        a.idx[i] = s_idx[i];
        a.w[i] = s_w[i];
      }
    if (warp == 0) {  // slot table of the down phase: present (unit, token) columns in unit order
      int used = 0;
      for (int base = 0; base < misc[0]; base += 32) {
        const int u = base + lane;
        const int c = (u < misc[0]) ? __popc(su[u].mask & 0xff) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        if (u < misc[0]) s_slot[u] = used + incl - c;
        used += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_slot[misc[0]] = used;
    }
    __syncthreads();
    for (int u = tid; u < misc[0]; u += kFThreads) {
      int sl = s_slot[u];
      const int m = su[u].mask & 0xff;
      for (int c = 0; c < 8; ++c)
        if ((m >> c) & 1) s_src[sl++] = u * 8 + c;
    }
    __syncthreads();
  }
  const int nu = misc[0];
  // down-projection rows of this CTA's P3 output block(s) into L2 (16 rows x I, for every unit)
  for (int rb = blockIdx.x; rb < H / 16; rb += gridDim.x) {
    const size_t rowb = (size_t)I / 4, srowb = (size_t)I / 32 * 2;
    for (int u = warp; u < nu; u += kFWarps) {
      const DecUnit &un = su[u];
      const MatView mv = mat_sel(a.routed, a.shared, un.set, 2, un.expert);
      prefetch_range(mv.codes + (size_t)rb * 16 * rowb, 16 * rowb, lane, 32);
      prefetch_range(mv.scales + (size_t)rb * 16 * (I / 32), 16 * srowb, lane, 32);
      if (Q3) prefetch_range(mv.hibits + (size_t)rb * 16 * (I / 8), 16 * rowb / 2, lane, 32);
    }
  }

  // ---------------- P2: gate/up + SwiGLU, one (unit, 16-row block) group per CTA at a time
  {
    const int rbs = I / 16, G2 = nu * rbs;
    const int mat = warp >> 3, slice = warp & 7;  // warps 0-7 gate, 8-15 up; slice = K step (mod 8)
    const int nsteps = (H + kStepK - 1) / kStepK;  // <= 8 (H <= 2048)
    const __half *xs_base = x16;
    StepFrag f;
    int gi = blockIdx.x;
    if (gi < G2) {
      const DecUnit &un = su[gi / rbs];
      load_step<Q3>(f, mat_sel(a.routed, a.shared, un.set, mat, un.expert), (gi % rbs) * 16, slice, slice < nsteps);
    }
    for (; gi < G2; gi += gridDim.x) {
      const int u = gi / rbs, r0 = (gi % rbs) * 16;
      const DecUnit &un = su[u];
      // next group's weights go out before this group is computed
      StepFrag fn;
      const int gn = gi + gridDim.x;
      if (gn < G2) {
        const DecUnit &un2 = su[gn / rbs];
        load_step<Q3>(fn, mat_sel(a.routed, a.shared, un2.set, mat, un2.expert), (gn % rbs) * 16, slice,
                      slice < nsteps);
      }
      const bool colok = (un.mask >> g) & 1;
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
      if (slice < nsteps)
        mma_step<Q3>(acc, acc2, f, xs_base + (size_t)g * xs16, slice * kStepK + 64 * t4,
                     colok && slice * kStepK + 64 * t4 < H);
      float *pw = part + warp * 16 * 8;
      pw[g * 8 + 2 * t4] = acc[0] + acc2[0];
      pw[g * 8 + 2 * t4 + 1] = acc[1] + acc2[1];
      pw[(g + 8) * 8 + 2 * t4] = acc[2] + acc2[2];
      pw[(g + 8) * 8 + 2 * t4 + 1] = acc[3] + acc2[3];
      __syncthreads();
      if (tid < 128) {  // one (row, column) per thread; fixed-order sums of the 8 K slices
        const int row = tid & 15, col = tid >> 4;
        if ((un.mask >> col) & 1) {
          float gv = 0.f, uv = 0.f;
#pragma unroll
          for (int sl = 0; sl < 8; ++sl) {
            gv += part[(sl * 16 + row) * 8 + col];
            uv += part[((8 + sl) * 16 + row) * 8 + col];
          }
          const float hv = gv / (1.0f + expf(-gv)) * uv;
          a.hdec[((size_t)u * 8 + col) * I + r0 + row] = __half_as_ushort(__float2half_rn(hv));
        }
      }
      __syncthreads();
      f = fn;
    }
  }
  __threadfence();
  if (!grid_barrier(ctrl, s_base + 2 * (unsigned long long)nblk, 32)) return;

  // ---------------- P3: down projection + weighted combine (+ residual) for 16 output features per CTA
  {
    const int nslots = s_slot[nu];
    const int nsteps = (I + kStepK - 1) / kStepK;
    const int xstride = I + 4;
    const int n_items = nu * nsteps;
    for (int rb = blockIdx.x; rb < H / 16; rb += gridDim.x) {
      const int r0 = rb * 16;
      // this warp's first two items' weights are requested before h is staged
      StepFrag f0, f1;
      if (warp < n_items) {
        const DecUnit &un = su[warp / nsteps];
        load_step<Q3>(f0, mat_sel(a.routed, a.shared, un.set, 2, un.expert), r0, warp % nsteps, true);
      }
      if (warp + kFWarps < n_items) {
        const DecUnit &un = su[(warp + kFWarps) / nsteps];
        load_step<Q3>(f1, mat_sel(a.routed, a.shared, un.set, 2, un.expert), r0, (warp + kFWarps) % nsteps, true);
      }
      {  // stage every present h column (16-byte loads, issued before the stores)
        const int I8 = I / 8, total = nslots * I8;
        for (int v0 = tid; v0 < total; v0 += 4 * kFThreads) {
          uint4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int vi = v0 + j * kFThreads;
            v[j] = (vi < total) ? __ldcg(reinterpret_cast<const uint4 *>(a.hdec + (size_t)s_src[vi / I8] * I) + vi % I8)
                                : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int vi = v0 + j * kFThreads;
            if (vi < total) {
              uint2 *d = reinterpret_cast<uint2 *>(hs + (size_t)(vi / I8) * xstride + xs_pos(8 * (vi % I8)));
              d[0] = make_uint2(v[j].x, v[j].y);
              d[1] = make_uint2(v[j].z, v[j].w);
            }
          }
        }
      }
      __syncthreads();
      float tot[4] = {0.f, 0.f, 0.f, 0.f};
      int j = 0;
      for (int it = warp; it < n_items; it += kFWarps, ++j) {
        const int u = it / nsteps, st = it % nsteps;
        const DecUnit &un = su[u];
        const bool colok = (un.mask >> g) & 1;
        const int slot = s_slot[u] + __popc(un.mask & ((1u << g) - 1u));
        const __half *xcol = hs + (size_t)(colok ? slot : 0) * xstride;
        StepFrag f;
        if (j == 0) f = f0;
        else if (j == 1) f = f1;
        else load_step<Q3>(f, mat_sel(a.routed, a.shared, un.set, 2, un.expert), r0, st, true);
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
        mma_step<Q3>(acc, acc2, f, xcol, st * kStepK + 64 * t4, colok && st * kStepK + 64 * t4 < I);
        const float wa = un.w[2 * t4], wb = un.w[2 * t4 + 1];
        tot[0] = fmaf(wa, acc[0] + acc2[0], tot[0]);
        tot[1] = fmaf(wb, acc[1] + acc2[1], tot[1]);
        tot[2] = fmaf(wa, acc[2] + acc2[2], tot[2]);
        tot[3] = fmaf(wb, acc[3] + acc2[3], tot[3]);
      }
      float *rw = red + warp * 16 * 8;
      rw[g * 8 + 2 * t4] = tot[0];
      rw[g * 8 + 2 * t4 + 1] = tot[1];
      rw[(g + 8) * 8 + 2 * t4] = tot[2];
      rw[(g + 8) * 8 + 2 * t4 + 1] = tot[3];
      __syncthreads();
      for (int i = tid; i < 16 * T; i += kFThreads) {
        const int row = i % 16, col = i / 16;
        float sum = a.residual ? a.residual[(size_t)col * H + r0 + row] : 0.0f;
#pragma unroll
        for (int wi = 0; wi < kFWarps; ++wi) sum += red[(wi * 16 + row) * 8 + col];
        a.y[(size_t)col * H + r0 + row] = sum;
      }
      __syncthreads();
    }
  }
}

cudaError_t launch_decode_fused(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k,
                                int I, const moe_expert_set &routed, const moe_expert_set *shared,
                                const float *residual, float *y, float *logits, int32_t *idx, float *w,
                                uint16_t *hdec, Ctrl *ctrl, cudaStream_t s) {
  const int hs_cols = T * k + (shared ? T : 0);
  if (T < 1 || T > kDecodeMaxT || E > 512 || H > 2048 || I > 1024 || hs_cols > kFSlots ||
      k > 16 ||
      (size_t)T * E * 4 > (size_t)kFSlots * (I + 4) * 2)
    return cudaErrorNotSupported;
  const FusedLayout L = fused_layout(T, H, I);
  const bool q3 = routed.gate.qtype == MOE_Q3;
  const void *fn = q3 ? reinterpret_cast<const void *>(decode_fused_kernel<true>)
                      : reinterpret_cast<const void *>(decode_fused_kernel<false>);
  cudaError_t e = smem_limit_once_impl(fn, L.total);
  if (e != cudaSuccess) return e;
  int dev = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorNotSupported;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kFThreads, L.total) != cudaSuccess || per_sm < 1)
    return cudaErrorNotSupported;
  FusedArgs a;
  a.x = x;
  a.T = T;
  a.H = H;
  a.E = E;
  a.k = k;
  a.I = I;
  a.has_shared = shared ? 1 : 0;
  a.Wr = Wr;
  a.bias = bias;
  a.routed = routed;
  a.shared = shared ? *shared : routed;
  a.residual = residual;
  a.y = y;
  a.logits = logits;
  a.idx = idx;
  a.w = w;
  a.hdec = hdec;
  a.ctrl = ctrl;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    KTimer kt_(KID_DECODE_FUSED, s);
    e = q3 ? cudaLaunchKernelEx(&cfg, decode_fused_kernel<true>, a) : cudaLaunchKernelEx(&cfg, decode_fused_kernel<false>, a);
  }
  return e;
}

}  // namespace moe
