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
// fp16 with a per-64-chunk rotation so the fragment loads of the four K slices hit distinct banks.
#include "common.cuh"
#include "dequant.cuh"

namespace moe {

constexpr int kStepK = 256;       // K covered by one warp step (4 lanes x 64 weights)
constexpr int kMaxSteps = 8;      // steps whose loads are issued together (K <= 2048 in one batch)

__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// shared-memory position of activation element k of a column (row stride added by the caller):
// 64-element chunk ch keeps its elements rotated by 16*(ch%4)
__device__ __forceinline__ int xs_pos(int k) {
  const int ch = k >> 6, q = k & 63;
  return (ch << 6) + ((q + 16 * (ch & 3)) & 63);
}

struct MatView {
  const uint8_t *codes;
  const uint8_t *hibits;
  const uint16_t *scales;
  int K;
  int q3;
};

__device__ __forceinline__ MatView mat_of(const moe_qmat &m, int expert) {
  MatView v;
  const size_t row0 = (size_t)expert * m.rows;
  v.codes = m.codes + row0 * (m.K / 4);
  v.hibits = m.hibits ? m.hibits + row0 * (m.K / 8) : nullptr;
  v.scales = m.scales + row0 * (m.K / 32);
  v.K = m.K;
  v.q3 = (m.qtype == MOE_Q3);
  return v;
}

// acc[4] += W[rows r0..r0+15] * X^T over the full K, X in shared memory (column c present iff
// bit c of `mask`, row stride `xstride` halves, rotated layout). Absent columns read as zero (their
// shared memory was never staged and may hold anything).
__device__ __forceinline__ void warp_rows16(const MatView &m, int r0, const __half *xs, int xstride, int mask,
                                            float acc[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int K = m.K;
  const size_t rs = (size_t)K / 4, ss = (size_t)K / 32, hs = (size_t)K / 8;
  const uint8_t *c0 = m.codes + (size_t)(r0 + g) * rs, *c1 = m.codes + (size_t)(r0 + g + 8) * rs;
  const uint16_t *s0 = m.scales + (size_t)(r0 + g) * ss, *s1 = m.scales + (size_t)(r0 + g + 8) * ss;
  const uint8_t *h0 = m.q3 ? m.hibits + (size_t)(r0 + g) * hs : nullptr;
  const uint8_t *h1 = m.q3 ? m.hibits + (size_t)(r0 + g + 8) * hs : nullptr;
  const bool colok = (mask >> g) & 1;
  const __half *xcol = xs + (size_t)g * xstride;
  const int nsteps = (K + kStepK - 1) / kStepK;
  for (int sb = 0; sb < nsteps; sb += kMaxSteps) {
    uint4 w0[kMaxSteps], w1[kMaxSteps];
    uint32_t d0[kMaxSteps], d1[kMaxSteps];
    uint2 hb0[kMaxSteps], hb1[kMaxSteps];
#pragma unroll
    for (int s = 0; s < kMaxSteps; ++s) {
      const int k0 = (sb + s) * kStepK + 64 * t;
      const bool ok = (sb + s < nsteps) && (k0 < K);
      w0[s] = ok ? __ldcs(reinterpret_cast<const uint4 *>(c0 + k0 / 4)) : make_uint4(0, 0, 0, 0);
      w1[s] = ok ? __ldcs(reinterpret_cast<const uint4 *>(c1 + k0 / 4)) : make_uint4(0, 0, 0, 0);
      d0[s] = ok ? __ldcs(reinterpret_cast<const uint32_t *>(s0 + k0 / 32)) : 0u;
      d1[s] = ok ? __ldcs(reinterpret_cast<const uint32_t *>(s1 + k0 / 32)) : 0u;
      if (m.q3) {
        hb0[s] = ok ? __ldcs(reinterpret_cast<const uint2 *>(h0 + k0 / 8)) : make_uint2(0, 0);
        hb1[s] = ok ? __ldcs(reinterpret_cast<const uint2 *>(h1 + k0 / 8)) : make_uint2(0, 0);
      } else {
        hb0[s] = hb1[s] = make_uint2(0, 0);
      }
    }
#pragma unroll
    for (int s = 0; s < kMaxSteps; ++s) {
      if (sb + s >= nsteps) break;
      const int kbase = (sb + s) * kStepK + 64 * t;
      // lanes past the K tail hold zero codes and zero scales (A = 0) and read no activations;
      // every lane still issues the warp-wide MMA
      const bool kin = kbase < K;
      const uint32_t wr0[4] = {w0[s].x, w0[s].y, w0[s].z, w0[s].w};
      const uint32_t wr1[4] = {w1[s].x, w1[s].y, w1[s].z, w1[s].w};
      const uint32_t hr0[2] = {hb0[s].x, hb0[s].y}, hr1[2] = {hb1[s].x, hb1[s].y};
#pragma unroll
      for (int wq = 0; wq < 4; ++wq) {  // word wq: block wq/2, half q = wq%2
        const int blk = wq >> 1, q = wq & 1;
        const __half2 dd0 = __half2half2(__ushort_as_half((uint16_t)(d0[s] >> (16 * blk))));
        const __half2 dd1 = __half2half2(__ushort_as_half((uint16_t)(d1[s] >> (16 * blk))));
        uint32_t p0[8], p1[8];
        if (m.q3) {
          dq3_word(wr0[wq], hr0[blk], q, dd0, p0);
          dq3_word(wr1[wq], hr1[blk], q, dd1, p1);
        } else {
          dq2_word(wr0[wq], dd0, p0);
          dq2_word(wr1[wq], dd1, p1);
        }
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {  // MMA m = 4*wq + mm uses pairs 2mm, 2mm+1 of this word
          const uint32_t a[4] = {p0[2 * mm], p1[2 * mm], p0[2 * mm + 1], p1[2 * mm + 1]};
          uint32_t b0 = 0, b1 = 0;
          if (colok && kin) {
            const int kk = kbase + 16 * wq + 4 * mm;
            const uint2 bv = *reinterpret_cast<const uint2 *>(xcol + xs_pos(kk));
            b0 = bv.x;
            b1 = bv.y;
          }
          mma16816(acc, a, b0, b1);
        }
      }
    }
  }
}

// stage columns of the activation source into shared memory (fp16, rotated layout)
template <bool SRC_BF16>
__device__ __forceinline__ void stage_x(const void *src, int row0, int mask, int H, __half *xs, int xstride) {
  const int H2 = H / 2;
  for (int c = 0; c < 8; ++c) {
    if (!((mask >> c) & 1)) continue;
    const uint32_t *s = reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(src) + (size_t)(row0 + c) * H);
    for (int i = threadIdx.x; i < H2; i += blockDim.x) {
      uint32_t v = s[i];
      __half2 h;
      if (SRC_BF16) h = __floats2half2_rn(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
      else h = *reinterpret_cast<__half2 *>(&v);
      *reinterpret_cast<__half2 *>(xs + (size_t)c * xstride + xs_pos(2 * i)) = h;
    }
  }
}

// ---------------------------------------------------------------- gate/up + SwiGLU
// grid (max_units, I/16); block = 2 warps: warp 0 gate rows, warp 1 up rows (same 16 rows)
template <bool SRC_BF16>
__global__ void __launch_bounds__(64)
dec_gate_up_kernel(const void *__restrict__ x, int H, int I, moe_expert_set routed, moe_expert_set shared,
                   const DecUnit *__restrict__ units, Ctrl *__restrict__ ctrl, uint16_t *__restrict__ hdec) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int u = blockIdx.x;
  if (u >= ctrl->n_units) return;
  const DecUnit un = units[u];
  if (un.expert < 0 || un.expert >= (un.set ? shared.gate.n_experts : routed.gate.n_experts)) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, un.expert);
    return;
  }
  const int xstride = H + 4;
  __half *xs = reinterpret_cast<__half *>(smem_raw);
  __shared__ float exch[16][8];
  stage_x<SRC_BF16>(x, un.xrow0, un.mask, H, xs, xstride);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const moe_expert_set &es = un.set ? shared : routed;
  const MatView mv = mat_of(warp == 0 ? es.gate : es.up, un.expert);
  const int r0 = blockIdx.y * 16;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  warp_rows16(mv, r0, xs, xstride, un.mask, acc);
  if (warp == 1) {
    exch[g][2 * t] = acc[0];
    exch[g][2 * t + 1] = acc[1];
    exch[g + 8][2 * t] = acc[2];
    exch[g + 8][2 * t + 1] = acc[3];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int row = g + (e >> 1) * 8, col = 2 * t + (e & 1);
      if (!((un.mask >> col) & 1)) continue;
      const float gv = acc[e], uv = exch[row][col];
      const float hv = gv / (1.0f + expf(-gv)) * uv;
      hdec[((size_t)u * 8 + col) * I + r0 + row] = __half_as_ushort(__float2half_rn(hv));
    }
  }
}

cudaError_t launch_decode_gate_up(const void *x, int x_is_bf16, int H, int I, const moe_expert_set &routed,
                                  const moe_expert_set *shared, const DecUnit *units, int max_units, Ctrl *ctrl,
                                  uint16_t *hdec, cudaStream_t s) {
  moe_expert_set sh = shared ? *shared : routed;
  dim3 grid(max_units, I / 16);
  size_t smem = (size_t)8 * (H + 4) * 2;
  if (x_is_bf16) {
    cudaError_t e = smem_limit_once(dec_gate_up_kernel<true>, smem);
    if (e != cudaSuccess) return e;
    {
      KTimer kt_(KID_DEC_GATE_UP, s);
      dec_gate_up_kernel<true><<<grid, 64, smem, s>>>(x, H, I, routed, sh, units, ctrl, hdec);
    }
  } else {
    cudaError_t e = smem_limit_once(dec_gate_up_kernel<false>, smem);
    if (e != cudaSuccess) return e;
    {
      KTimer kt_(KID_DEC_GATE_UP, s);
      dec_gate_up_kernel<false><<<grid, 64, smem, s>>>(x, H, I, routed, sh, units, ctrl, hdec);
    }
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- down (+ weighted combine)
// grid H/16 (one 16-row output group per CTA); kDownWarps warps split the units. Combine mode:
// acc_total += w_u[col] * (W_down[u] h_u) over units, reduced across warps in fixed order, then
// y = acc (+ residual). Rows mode: each unit's 16 x ncols result is written to its output rows.
constexpr int kDownWarps = 8;

__global__ void __launch_bounds__(kDownWarps * 32)
dec_down_kernel(int H, int I, moe_expert_set routed, moe_expert_set shared, const DecUnit *__restrict__ units,
                Ctrl *__restrict__ ctrl, const uint16_t *__restrict__ hdec, float *__restrict__ y,
                const float *residual, int T, uint16_t *__restrict__ out_rows) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int nu = ctrl->n_units;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int r0 = blockIdx.x * 16;
  const int xstride = I + 4;
  __half *hs = reinterpret_cast<__half *>(smem_raw);  // per warp: 8 columns x (I+4)
  __half *myh = hs + (size_t)warp * 8 * xstride;
  __shared__ float red[kDownWarps][16][8];
  float tot[4] = {0.f, 0.f, 0.f, 0.f};
  for (int u = warp; u < nu; u += kDownWarps) {
    const DecUnit un = units[u];
    if (un.expert < 0 || un.expert >= (un.set ? shared.down.n_experts : routed.down.n_experts)) {
      if (lane == 0 && blockIdx.x == 0) set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, un.expert);
      continue;
    }
    // stage this unit's h columns (warp-local)
    for (int c = 0; c < 8; ++c) {
      if (!((un.mask >> c) & 1)) continue;
      const uint32_t *src = reinterpret_cast<const uint32_t *>(hdec + ((size_t)u * 8 + c) * I);
      for (int i = lane; i < I / 2; i += 32)
        *reinterpret_cast<uint32_t *>(myh + (size_t)c * xstride + xs_pos(2 * i)) = __ldcg(src + i);
    }
    __syncwarp();
    const moe_expert_set &es = un.set ? shared : routed;
    const MatView mv = mat_of(es.down, un.expert);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    warp_rows16(mv, r0, myh, xstride, un.mask, acc);
    __syncwarp();
    if (out_rows) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = g + (e >> 1) * 8, col = 2 * t + (e & 1);
        if ((un.mask >> col) & 1)
          out_rows[(size_t)(un.xrow0 + col) * H + r0 + row] = __half_as_ushort(__float2half_rn(acc[e]));
      }
    } else {
      const float wa = un.w[2 * t], wb = un.w[2 * t + 1];
      tot[0] = fmaf(wa, acc[0], tot[0]);
      tot[1] = fmaf(wb, acc[1], tot[1]);
      tot[2] = fmaf(wa, acc[2], tot[2]);
      tot[3] = fmaf(wb, acc[3], tot[3]);
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
    float s = residual ? residual[(size_t)col * H + r0 + row] : 0.0f;
#pragma unroll
    for (int wi = 0; wi < kDownWarps; ++wi) s += red[wi][row][col];
    y[(size_t)col * H + r0 + row] = s;
  }
}

cudaError_t launch_decode_down(int H, int I, const moe_expert_set &routed, const moe_expert_set *shared,
                               const DecUnit *units, int max_units, Ctrl *ctrl, const uint16_t *hdec, float *y,
                               const float *residual, int T, uint16_t *out_rows, cudaStream_t s) {
  (void)max_units;
  moe_expert_set sh = shared ? *shared : routed;
  size_t smem = (size_t)kDownWarps * 8 * (I + 4) * 2;
  cudaError_t e = smem_limit_once(dec_down_kernel, smem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_DEC_DOWN, s);
    dec_down_kernel<<<H / 16, kDownWarps * 32, smem, s>>>(H, I, routed, sh, units, ctrl, hdec, y, residual, T, out_rows);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- units for grouped rows
// rows mode for moe_expert_ffn: group g's rows [off[g], off[g+1]) in chunks of 8 columns
__global__ void units_from_offsets_kernel(const int32_t *__restrict__ off, int n_groups, int shared_group,
                                          int n_rows, DecUnit *__restrict__ units, Ctrl *__restrict__ ctrl) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int nu = 0;
  for (int gi = 0; gi < n_groups; ++gi) {
    const int a = off[gi], b = off[gi + 1];
    if (a < 0 || b < a || b > n_rows) {  // malformed offsets: flag and run nothing
      set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, gi);
      nu = 0;
      break;
    }
    for (int r = a; r < b; r += 8) {
      DecUnit un;
      un.expert = (gi == shared_group) ? 0 : gi;
      un.set = (gi == shared_group) ? 1 : 0;
      const int n = min(8, b - r);
      un.mask = (1 << n) - 1;
      un.xrow0 = r;
#pragma unroll
      for (int c = 0; c < 8; ++c) un.w[c] = 1.0f;
      units[nu++] = un;
    }
  }
  ctrl->n_units = nu;
}

cudaError_t launch_decode_units_from_offsets(const int32_t *offsets, int n_groups, int has_shared_group, int n_rows,
                                             DecUnit *units, Ctrl *ctrl, cudaStream_t s) {
  {
    KTimer kt_(KID_DEC_UNITS, s);
    units_from_offsets_kernel<<<1, 32, 0, s>>>(offsets, n_groups, has_shared_group ? n_groups - 1 : -1, n_rows, units,
                                               ctrl);
  }
  return cudaGetLastError();
}

}  // namespace moe
