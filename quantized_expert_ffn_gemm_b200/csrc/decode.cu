// Decode / MTP-verify expert path (1-8 activation rows per expert): memory-bound dequant-GEMV.
//
// Decode reads weights rather than computing ("Strata vs Llama.cpp vs vLLM", chapter "Why LLM
// inference is a systems problem"; "Two-Day Port ...", "Why Prefill Matters More Than Decode"),
// and verify passes carry up to 4 tokens (Strata DETAILS.md, "How it works": up to 3 drafts).
// So the weights of each distinct selected expert are streamed exactly once with 128-bit loads,
// all of a warp's loads issued before its first multiply, and every token that chose the
// expert is served from that one read.
//
// Inner product: a warp owns 16 weight rows; lane (g, t) holds rows g and g+8 and a 64-weight
// slice of K (one 16-byte load per row per 256-wide K step). Each 16-weight word is dequantized
// to fp16 pairs (exact for Q2) and fed to mma.sync m16n8k16 with the activations as the 8 MMA
// columns, accumulating in fp32. The MMA sums over K inside the warp, so the split-K reduction is
// done by the tensor core instead of a shuffle tree. Activations are staged in shared memory as
// fp16 in the padded layout of gemv.cuh (16 halves after every 64), so the fragment loads of the
// four K slices hit distinct banks.
#include "common.cuh"
#include "dequant.cuh"
#include "gemv.cuh"

namespace moe {

// ---------------------------------------------------------------- gate/up + SwiGLU
// grid (units, I/64); block = 8 warps: warps 0-3 gate, 4-7 up, for the same 16 rows of each of the
// CTA's four 16-feature blocks; warp slice q takes K steps q, q+4, ... so every warp has a short
// MMA chain and the SM has many warps in flight. Partials are summed in shared memory in fixed
// order.
constexpr int kGuWarps = 8;
constexpr int kGuBlocks = 4;  // 16-feature blocks per CTA (I % 64 == 0)

template <bool SRC_BF16, int QT>
__global__ void __launch_bounds__(kGuWarps * 32)
dec_gate_up_kernel(const void *__restrict__ x, int H, int I, moe_expert_set routed, moe_expert_set shared,
                   const DecUnit *__restrict__ units, Ctrl *__restrict__ ctrl, uint16_t *__restrict__ hdec) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int n_units = ctrl->n_units;
  const int xstride = xs_stride(H);
  __half *xs = reinterpret_cast<__half *>(smem_raw);
  __shared__ float part[kGuWarps][16][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int mat = warp >> 2, slice = warp & 3;
  const int nsteps = (H + kStepK - 1) / kStepK;
  const __half *xcol = xs + (size_t)g * xstride;
  // A CTA takes kGuBlocks consecutive 16-feature blocks of one unit, so the unit's activation
  // columns are staged once for all of them; the next block's weights are requested before the
  // current block's MMAs. Units are taken grid-stride (the grid is sized by the device, not by the
  // largest possible unit count, so an empty or short unit list costs no flood of idle CTAs).
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const DecUnit un = units[u];
    if (un.expert < 0 || un.expert >= (un.set ? shared.gate.n_experts : routed.gate.n_experts)) {
      if (threadIdx.x == 0 && blockIdx.y == 0) set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, un.expert);
      continue;
    }
    __syncthreads();  // the previous unit's reads of xs and part are done
    const MatView mv = mat_sel(routed, shared, un.set, mat, un.expert);
    const bool colok = (un.mask >> g) & 1;
    const int rb0 = blockIdx.y * kGuBlocks;
    StepFrag f[2];
    if (nsteps <= 8) {  // at most two steps per slice: the first block's are requested before staging
      load_step<QT>(f[0], mv, rb0 * 16, slice, slice < nsteps);
      load_step<QT>(f[1], mv, rb0 * 16, slice + 4, slice + 4 < nsteps);
    }
    bool bad = stage_x<SRC_BF16>(x, un.xrow0, un.mask, H, xs, xstride);
    __syncthreads();
    for (int b = 0; b < kGuBlocks; ++b) {
      const int r0 = (rb0 + b) * 16;
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
      if (nsteps <= 8) {
        StepFrag fn[2];
        const bool more = b + 1 < kGuBlocks;
        if (more) {
          load_step<QT>(fn[0], mv, r0 + 16, slice, slice < nsteps);
          load_step<QT>(fn[1], mv, r0 + 16, slice + 4, slice + 4 < nsteps);
        }
        if (slice < nsteps) mma_step<QT>(acc, acc2, f[0], xcol, slice * kStepK + 64 * t,
                                         colok && slice * kStepK + 64 * t < H);
        if (slice + 4 < nsteps) mma_step<QT>(acc, acc2, f[1], xcol, (slice + 4) * kStepK + 64 * t,
                                             colok && (slice + 4) * kStepK + 64 * t < H);
        if (more) {
          f[0] = fn[0];
          f[1] = fn[1];
        }
      } else {
        for (int st = slice; st < nsteps; st += 4) {
          StepFrag fs;
          load_step<QT>(fs, mv, r0, st, true);
          mma_step<QT>(acc, acc2, fs, xcol, st * kStepK + 64 * t, colok && st * kStepK + 64 * t < H);
        }
      }
      part[warp][g][2 * t] = acc[0] + acc2[0];
      part[warp][g][2 * t + 1] = acc[1] + acc2[1];
      part[warp][g + 8][2 * t] = acc[2] + acc2[2];
      part[warp][g + 8][2 * t + 1] = acc[3] + acc2[3];
      __syncthreads();
      if (threadIdx.x < 128) {  // one (row, column) per thread
        const int row = threadIdx.x & 15, col = threadIdx.x >> 4;
        if ((un.mask >> col) & 1) {
          const float gv = (part[0][row][col] + part[1][row][col]) + (part[2][row][col] + part[3][row][col]);
          const float uv = (part[4][row][col] + part[5][row][col]) + (part[6][row][col] + part[7][row][col]);
          const float hv = gv / (1.0f + expf(-gv)) * uv;
          const uint16_t hb = __half_as_ushort(__float2half_rn(hv));
          bad |= f16_inf(hb);
          hdec[((size_t)u * 8 + col) * I + r0 + row] = hb;
        }
      }
      __syncthreads();  // part is rewritten by the next block
    }
    if (bad) set_device_error(ctrl, MOE_ERR_RANGE, 2);
  }
}

template <bool B, int Q>
static cudaError_t launch_gu(dim3 grid, size_t smem, cudaStream_t s, const void *x, int H, int I,
                             const moe_expert_set &routed, const moe_expert_set &sh, const DecUnit *units, Ctrl *ctrl,
                             uint16_t *hdec) {
  cudaError_t e = smem_limit_once(dec_gate_up_kernel<B, Q>, smem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_DEC_GATE_UP, s);
    dec_gate_up_kernel<B, Q><<<grid, kGuWarps * 32, smem, s>>>(x, H, I, routed, sh, units, ctrl, hdec);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_gate_up(const void *x, int x_is_bf16, int H, int I, const moe_expert_set &routed,
                                  const moe_expert_set *shared, const DecUnit *units, int max_units, Ctrl *ctrl,
                                  uint16_t *hdec, cudaStream_t s) {
  const moe_expert_set sh = shared ? *shared : routed;
  // about eight CTAs per SM in all; each walks units grid-stride
  const int ny = I / (16 * kGuBlocks);
  const int cap = (8 * num_sms() + ny - 1) / ny;
  const dim3 grid(max_units < cap ? (max_units > 0 ? max_units : 1) : cap, ny);
  const size_t smem = (size_t)8 * xs_stride(H) * 2;
  const int qt = routed.gate.qtype;
#define MOE_GU(B, Q) launch_gu<B, Q>(grid, smem, s, x, H, I, routed, sh, units, ctrl, hdec)
  if (x_is_bf16)
    return qt == MOE_Q3 ? MOE_GU(true, 3) : qt == MOE_Q4 ? MOE_GU(true, 4) : MOE_GU(true, 2);
  return qt == MOE_Q3 ? MOE_GU(false, 3) : qt == MOE_Q4 ? MOE_GU(false, 4) : MOE_GU(false, 2);
#undef MOE_GU
}

// ---------------------------------------------------------------- down (+ weighted combine)
// grid H/16 (one 16-row output group per CTA); kDownWarps warps split the units (a whole unit per
// warp). Units are taken in chunks whose present h columns fit the shared budget; each warp
// issues its unit's weight loads, then the chunk's h columns are staged, then the MMAs run.
// Combine mode (y != NULL): acc_total += w_u[col] * (W_down[u] h_u) over units, reduced across
// warps in fixed order, then y = acc (+ residual). Rows mode: each unit's 16 x 8 result goes to
// its output rows.
constexpr int kDownWarps = 16;
constexpr int kDownSlots = 64;     // h columns staged at once
constexpr int kDownMaxUnits = 128; // unit records cached in shared memory at a time

template <int QT>
__global__ void __launch_bounds__(kDownWarps * 32)
dec_down_kernel(int H, int I, moe_expert_set routed, moe_expert_set shared, const DecUnit *__restrict__ units,
                Ctrl *__restrict__ ctrl, const uint16_t *__restrict__ hdec, float *__restrict__ y,
                const float *residual, int T, uint16_t *__restrict__ out_rows) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int nu = ctrl->n_units;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int r0 = blockIdx.x * 16;
  const int xstride = xs_stride(I);
  __half *hs = reinterpret_cast<__half *>(smem_raw);  // kDownSlots columns x xs_stride(I)
  __shared__ float red[kDownWarps][16][8];
  __shared__ __align__(16) DecUnit s_units[kDownMaxUnits];
  __shared__ int s_slot[kDownMaxUnits + 1];           // first staged slot of each unit of the chunk
  __shared__ int s_src[kDownSlots];                   // h row (unit*8 + column) of each staged slot
  __shared__ int s_u1;
  float tot[4] = {0.f, 0.f, 0.f, 0.f};
  const int nsteps = (I + kStepK - 1) / kStepK;
  for (int ub = 0; ub < nu; ub += kDownMaxUnits) {
    const int ue = min(nu, ub + kDownMaxUnits);
    // cache this batch of unit records (one coalesced read)
    {
      const int nwords = (ue - ub) * (int)(sizeof(DecUnit) / 16);
      const uint4 *src = reinterpret_cast<const uint4 *>(units + ub);
      uint4 *dst = reinterpret_cast<uint4 *>(s_units);
      for (int i = threadIdx.x; i < nwords; i += blockDim.x) dst[i] = __ldg(src + i);
    }
    __syncthreads();
    int u0 = ub;
    while (u0 < ue) {
      if (threadIdx.x == 0) {  // chunk [u0, u1): whole units whose columns fit kDownSlots slots
        int u1 = u0, used = 0;
        while (u1 < ue) {
          const int m = s_units[u1 - ub].mask & 0xff;
          const int c = __popc(m);
          if (used + c > kDownSlots) break;
          s_slot[u1 - u0] = used;
          for (int cc = 0; cc < 8; ++cc)
            if ((m >> cc) & 1) s_src[used++] = u1 * 8 + cc;
          ++u1;
        }
        s_slot[u1 - u0] = used;
        s_u1 = u1;
      }
      __syncthreads();
      const int u1 = s_u1, nslots = s_slot[u1 - u0];
      // work items: combine mode (unit, K step) pairs, rows mode whole units; item i goes to warp
      // i % kDownWarps. A warp's first two items' weights are requested before h is staged.
      const int per_unit = out_rows ? 1 : nsteps;
      const int n_items = (u1 - u0) * per_unit;
      StepFrag f[2];
      bool okv[2] = {false, false};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int it = warp + j * kDownWarps;
        if (it < n_items && (per_unit > 1 || nsteps == 1)) {
          const DecUnit &un = s_units[u0 + it / per_unit - ub];
          if (un.expert >= 0 && un.expert < (un.set ? shared.down.n_experts : routed.down.n_experts)) {
            load_step<QT>(f[j], mat_sel(routed, shared, un.set, 2, un.expert), r0, per_unit > 1 ? it % per_unit : 0,
                          true);
            okv[j] = true;
          }
        }
      }
      {  // stage the chunk's h columns: 16-byte loads, all of a thread's loads before its stores
        const int I8 = I / 8, total = nslots * I8;
        for (int v0 = threadIdx.x; v0 < total; v0 += 4 * blockDim.x) {
          uint4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int vi = v0 + j * blockDim.x;
            v[j] = (vi < total) ? __ldcg(reinterpret_cast<const uint4 *>(hdec + (size_t)s_src[vi / I8] * I) + vi % I8)
                                : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int vi = v0 + j * blockDim.x;
            if (vi < total) {  // rows are 8-byte aligned (stride I+4 halves): two 8-byte stores
              uint2 *d = reinterpret_cast<uint2 *>(hs + (size_t)(vi / I8) * xstride + xs_pos(8 * (vi % I8)));
              d[0] = make_uint2(v[j].x, v[j].y);
              d[1] = make_uint2(v[j].z, v[j].w);
            }
          }
        }
      }
      __syncthreads();
      for (int it = warp, j = 0; it < n_items; it += kDownWarps, ++j) {
        const int uu = u0 + it / per_unit;
        const DecUnit &un = s_units[uu - ub];
        if (un.expert < 0 || un.expert >= (un.set ? shared.down.n_experts : routed.down.n_experts)) {
          if (lane == 0 && blockIdx.x == 0) set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, un.expert);
          continue;
        }
        // this lane's column slot (absent columns feed zeros)
        const bool colok = (un.mask >> g) & 1;
        const int slot = s_slot[uu - u0] + __popc(un.mask & ((1u << g) - 1u));
        const __half *xcol = hs + (size_t)(colok ? slot : 0) * xstride;
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
        if (per_unit > 1 || nsteps == 1) {  // one K step
          const int st = per_unit > 1 ? it % per_unit : 0;
          StepFrag fl;
          if (j == 0 && okv[0]) fl = f[0];
          else if (j == 1 && okv[1]) fl = f[1];
          else load_step<QT>(fl, mat_sel(routed, shared, un.set, 2, un.expert), r0, st, true);
          mma_step<QT>(acc, acc2, fl, xcol, st * kStepK + 64 * t, colok && st * kStepK + 64 * t < I);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[e] += acc2[e];
        } else {  // rows mode with several K steps: two steps' loads in flight, then their MMAs
          const MatView mv = mat_sel(routed, shared, un.set, 2, un.expert);
          for (int st = 0; st < nsteps; st += 2) {
            StepFrag fl[2];
            load_step<QT>(fl[0], mv, r0, st, true);
            load_step<QT>(fl[1], mv, r0, st + 1, st + 1 < nsteps);
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              const int kb = (st + b) * kStepK + 64 * t;
              if (st + b < nsteps) mma_step<QT>(acc, acc2, fl[b], xcol, kb, colok && kb < I);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[e] += acc2[e];
        }
        if (out_rows) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = g + (e >> 1) * 8, col = 2 * t + (e & 1);
            if ((un.mask >> col) & 1)
            {
              const uint16_t ob = __half_as_ushort(__float2half_rn(acc[e]));
              if (f16_inf(ob)) set_device_error(ctrl, MOE_ERR_RANGE, 3);
              out_rows[(size_t)(un.xrow0 + col) * H + r0 + row] = ob;
            }
          }
        } else {
          const float wa = un.w[2 * t], wb = un.w[2 * t + 1];
          tot[0] = fmaf(wa, acc[0], tot[0]);
          tot[1] = fmaf(wb, acc[1], tot[1]);
          tot[2] = fmaf(wa, acc[2], tot[2]);
          tot[3] = fmaf(wb, acc[3], tot[3]);
        }
      }
      __syncthreads();  // before the next chunk overwrites the staged columns and slot tables
      u0 = u1;
    }
  }
  if (out_rows) return;
  red[warp][g][2 * t] = tot[0];
  red[warp][g][2 * t + 1] = tot[1];
  red[warp][g + 8][2 * t] = tot[2];
  red[warp][g + 8][2 * t + 1] = tot[3];
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * T; i += blockDim.x) {
    const int row = i % 16, col = i / 16;  // consecutive threads -> consecutive output features
    float sum = residual ? residual[(size_t)col * H + r0 + row] : 0.0f;
#pragma unroll
    for (int wi = 0; wi < kDownWarps; ++wi) sum += red[wi][row][col];
    y[(size_t)col * H + r0 + row] = sum;
  }
}

cudaError_t launch_decode_down(int H, int I, const moe_expert_set &routed, const moe_expert_set *shared,
                               const DecUnit *units, int max_units, Ctrl *ctrl, const uint16_t *hdec, float *y,
                               const float *residual, int T, uint16_t *out_rows, cudaStream_t s) {
  (void)max_units;
  const moe_expert_set sh = shared ? *shared : routed;
  const size_t smem = (size_t)kDownSlots * xs_stride(I) * 2;
  const int qt = routed.gate.qtype;
  auto fn = qt == MOE_Q3 ? dec_down_kernel<3> : qt == MOE_Q4 ? dec_down_kernel<4> : dec_down_kernel<2>;
  cudaError_t e = smem_limit_once(fn, smem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_DEC_DOWN, s);
    fn<<<H / 16, kDownWarps * 32, smem, s>>>(H, I, routed, sh, units, ctrl, hdec, y, residual, T, out_rows);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- units for grouped rows
// rows mode for moe_expert_ffn: group g's rows [off[g], off[g+1]) in chunks of 8 columns. One
// CTA: each thread takes a group, a block-wide exclusive scan of the groups' chunk counts gives
// each group's first unit, and the groups are walked in blocks of kUnitsThreads. Units come out
// in group order, then row order, as a serial walk would produce them.
constexpr int kUnitsThreads = 1024;

__global__ void __launch_bounds__(kUnitsThreads)
units_from_offsets_kernel(const int32_t *__restrict__ off, int n_groups, int shared_group, int n_rows,
                          DecUnit *__restrict__ units, Ctrl *__restrict__ ctrl) {
  __shared__ int s_warp[kUnitsThreads / 32];
  __shared__ int s_base, s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    s_base = 0;
    s_bad = 0x7fffffff;
  }
  __syncthreads();
  for (int gi = tid; gi < n_groups; gi += kUnitsThreads) {  // malformed offsets: flag, run nothing
    const int a = off[gi], b = off[gi + 1];
    if (a < 0 || b < a || b > n_rows) atomicMin(&s_bad, gi);
  }
  __syncthreads();
  if (s_bad != 0x7fffffff) {
    if (tid == 0) {
      set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, s_bad);
      ctrl->n_units = 0;
    }
    return;
  }
  for (int c0 = 0; c0 < n_groups; c0 += kUnitsThreads) {
    const int gi = c0 + tid;
    int a = 0, cnt = 0, nrow = 0;
    if (gi < n_groups) {
      a = off[gi];
      nrow = off[gi + 1] - a;
      cnt = (nrow + 7) / 8;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int v = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      s_warp[lane] = v;  // inclusive sums of the warps' totals
    }
    __syncthreads();
    const int first = s_base + (warp ? s_warp[warp - 1] : 0) + incl - cnt;
    for (int j = 0; j < cnt; ++j) {
      DecUnit un;
      un.expert = (gi == shared_group) ? 0 : gi;
      un.set = (gi == shared_group) ? 1 : 0;
      const int n = min(8, nrow - 8 * j);
      un.mask = (1 << n) - 1;
      un.xrow0 = a + 8 * j;
#pragma unroll
      for (int c = 0; c < 8; ++c) un.w[c] = 1.0f;
      units[first + j] = un;
    }
    __syncthreads();  // every thread has read s_base and s_warp
    if (tid == kUnitsThreads - 1) s_base = first + cnt;
    __syncthreads();
  }
  if (tid == 0) ctrl->n_units = s_base;
}

cudaError_t launch_decode_units_from_offsets(const int32_t *offsets, int n_groups, int has_shared_group, int n_rows,
                                             DecUnit *units, Ctrl *ctrl, cudaStream_t s) {
  {
    KTimer kt_(KID_DEC_UNITS, s);
    units_from_offsets_kernel<<<1, kUnitsThreads, 0, s>>>(offsets, n_groups, has_shared_group ? n_groups - 1 : -1,
                                                          n_rows, units, ctrl);
  }
  return cudaGetLastError();
}

}  // namespace moe
