// Prefill expert gate/up with int8 activations on the 5th-generation tensor cores (MMQ-style).
//
// The pages' prefill speed-up came from "fused int8 tensor core kernels" ("Strata vs Llama.cpp vs
// vLLM", the v0.1.36 prompt-processing note) after a port of llama.cpp's quantized matmul, MMQ
// ("Two-Day Port, 8x Faster Prefill: Strata Engine Benchmarked", "Where Strata Is Fast: Not
// Magic, but Logistics"): activations quantized to int8, block weights kept as small integers,
// integer dot products per weight block, the block scales applied afterwards.
//
// Here, per expert-contiguous row r of x_perm and 32-value block b: d_x[r, b] = max|x| / 127 over
// the block, xq = rint(x / d_x) (int8). Q2 weights are the integers c - 2 in [-2, 1] (exact in
// int8) with one fp16 scale d_w per row and 32-weight block. One tcgen05.mma kind::i8 (M = 128
// weight rows, N <= 64 token rows, K = 32) computes a block's exact int32 dot products S_b into its
// own tensor-memory accumulator, and both block scales are applied on the read-back:
//   acc[row, n] += d_w[row, b] * d_x[n, b] * float(S_b[row, n]);   h = silu(gate) * up (fp16).
// The per-block rescale is the cost of the format: every block's 128 x N integer accumulator is
// read back and converted, about two instructions per element against the tensor core's one
// K = 32 MMA, so this path is bound by the read-back, not by the int8 MMA rate.
//
// Structure (a plain, non-pipelined prototype; one tile at a time per CTA, persistent grid):
//   tile     one expert group slice of <= 64 token rows x 64 features (A rows interleave the
//            features' gate and up rows, as the fp16 kernel does, so SwiGLU pairs adjacent lanes)
//   stage    K = 128: TMA brings the int8 token rows (128-byte swizzle) and the 128 weight rows'
//            2-bit codes; every thread decodes its weight row's 128 codes into int8 and stores
//            them to tensor memory (A operand); thread 0 issues the stage's four MMAs, one per
//            32-weight block, each into its own accumulator; every thread reads the four
//            accumulators of its row back, scales and adds them
// Every mbarrier wait is bounded in time and reports MOE_ERR_TIMEOUT through the control area.
#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {

namespace {

constexpr int kQThreads = 128;    // 4 warps: one tensor-memory lane quadrant each
constexpr int kQBM = 128;         // A rows: 64 features x (gate, up)
constexpr int kQBN = 64;          // token rows per tile (MMA N <= 64)
constexpr int kQBK = 128;         // K per stage (one 128-byte swizzle row of int8)
constexpr int kQBlocks = kQBK / 32;
// tensor memory (512 columns): A at columns 0..31 (128 int8 per lane, four per 32-bit column,
// the lowest K in the low byte), the four block accumulators at 64 + 64 b (N <= 64 columns each)
constexpr uint32_t kQACol = 0, kQDCol = 64;
constexpr int kQSmemB = kQBN * kQBK;            // 8 KB of int8 token rows (1024-byte aligned atoms)
constexpr int kQSmemCodes = kQBM * (kQBK / 4);  // 4 KB of 2-bit codes
constexpr int kQSmemDx = kQBlocks * kQBN * 4;  // the stage's activation block scales
constexpr int kQSmem = kQSmemB + kQSmemCodes + 64 + kQSmemDx + 1024;
// more dynamic shared memory than two CTAs can hold, so a CTA never waits on another CTA's
// tensor-memory allocation
constexpr int kQSmemRequest = 120 * 1024;

// instruction descriptor, kind::i8: signed int8 A and B, int32 accumulator, both K-major,
// M = 128, N (multiple of 16)
__device__ __forceinline__ uint32_t idesc_i8(int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16_i(uint32_t taddr, uint32_t r[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// one 32-bit word of the 2-bit plane (16 weights: weight 2i+h at bits 16h+2i) -> the int8 values
// c - 2 of weights 0..15 of the word, four per output word in K order (lowest K in the low byte)
__device__ __forceinline__ void q2_word_to_i8(uint32_t w, uint32_t out[4]) {
#pragma unroll
  for (int o = 0; o < 4; ++o) {  // output word o: weights 4o .. 4o+3 = pairs i = 2o, 2o+1
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int wi = 4 * o + j, i = wi >> 1, h = wi & 1;
      const int c = (int)((w >> (16 * h + 2 * i)) & 3u);
      v |= (uint32_t)(uint8_t)(int8_t)(c - 2) << (8 * j);
    }
    out[o] = v;
  }
}

struct MmqArgs {
  const int32_t *offsets;
  const int2 *tiles;
  Ctrl *ctrl;
  const float *dx;             // [row][H/32]: the int8 scales of x_perm's 32-value blocks
  uint16_t *h_perm;            // fp16 [rows][I]
  int H, I;
  int shared_group;            // group index served by the shared expert, -1 if none
  const uint16_t *scales[2][2];  // [set][gate/up]
};

__global__ void __launch_bounds__(kQThreads, 1)
mmq_gate_up_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_g_r,
                   const __grid_constant__ CUtensorMap tm_u_r, const __grid_constant__ CUtensorMap tm_g_s,
                   const __grid_constant__ CUtensorMap tm_u_s, const MmqArgs args) {
  extern __shared__ uint8_t smem_raw[];
  Ctrl *ctrl = args.ctrl;
  const int n_mtiles = args.I / 64;
  const int total = ctrl->n_tiles * n_mtiles;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - smem_u32(smem_raw));
  const uint32_t sB = base, sC = base + kQSmemB;
  const uint32_t bar_full = base + kQSmemB + kQSmemCodes, bar_mma = bar_full + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kQSmemB + kQSmemCodes + 16);
  float *s_dx = reinterpret_cast<float *>(gbase + kQSmemB + kQSmemCodes + 64);  // [block][token]
  const int warp = threadIdx.x >> 5, r = threadIdx.x;  // A row = TMEM lane = thread
  const int K = args.H, nk = K / kQBK;
  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  // A row r: gate row f0 + r/2 (even r) or up row f0 + r/2 (odd r); its codes sit in smem row
  // r/2 (gate, rows 0-63) or 64 + r/2 (up)
  const int mat = r & 1, crow = mat ? 64 + (r >> 1) : (r >> 1);
  uint32_t phase = 0;
  bool ok = true;
  for (int ti = blockIdx.x; ti < total && ok; ti += gridDim.x) {
    const int entry = ti / n_mtiles, mt = ti - entry * n_mtiles;
    const int2 e = args.tiles[entry];
    const int set = (e.x == args.shared_group) ? 1 : 0, expert = set ? 0 : e.x;
    const int row_base = args.offsets[e.x] + e.y;
    const int n_valid = min(kQBN, args.offsets[e.x + 1] - row_base);
    const int N = (n_valid + 15) & ~15;
    const uint32_t idesc = idesc_i8(N);
    const int wrow = expert * args.I + mt * 64;  // first gate / up row of the tile
    const uint16_t *sc = args.scales[set][mat] + ((size_t)expert * args.I + mt * 64 + (r >> 1)) * (K / 32);
    float acc[kQBN];
#pragma unroll
    for (int n = 0; n < kQBN; ++n) acc[n] = 0.0f;
    for (int ks = 0; ks < nk && ok; ++ks) {
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar_full, (uint32_t)(kQSmemB + kQSmemCodes));
        tma_load_2d(sB, &tm_x, ks * kQBK, row_base, bar_full);
        tma_load_2d(sC, set ? &tm_g_s : &tm_g_r, ks * (kQBK / 4), wrow, bar_full);
        tma_load_2d(sC + 64 * (kQBK / 4), set ? &tm_u_s : &tm_u_r, ks * (kQBK / 4), wrow, bar_full);
      }
      const uint2 dws = __ldg(reinterpret_cast<const uint2 *>(sc + ks * kQBlocks));  // the stage's 4 block scales
      for (int i = threadIdx.x; i < kQBlocks * kQBN; i += kQThreads) {  // and the tokens' 4 block scales
        const int b = i / kQBN, n = i % kQBN;
        s_dx[i] = (n < n_valid) ? __ldg(args.dx + (size_t)(row_base + n) * (K / 32) + ks * kQBlocks + b) : 0.0f;
      }
      const bool landed = mbar_wait(bar_full, phase);
      if (!landed) set_device_error(ctrl, MOE_ERR_TIMEOUT, 50);
      // this row's 128 codes -> 128 int8 (c - 2), 32 words -> tensor memory
      const uint4 *cw = reinterpret_cast<const uint4 *>(gbase + kQSmemB + crow * (kQBK / 4));
      const uint4 c0 = cw[0], c1 = cw[1];
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint32_t a[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) q2_word_to_i8(words[q], a + 4 * q);
      tmem_st16(tmem + lane_base + kQACol, a);
      tmem_st16(tmem + lane_base + kQACol + 16u, a + 16);
      tmem_st_wait();
      tc_fence_before();
      // every thread's wait decides together: a CTA-uniform stop (a wait that gave up)
      ok = __syncthreads_and(landed) != 0;
      if (!ok) break;
      if (threadIdx.x == 0) {
        tc_fence_after();
        const uint64_t db = sw128_desc(sB);
#pragma unroll
        for (int b = 0; b < kQBlocks; ++b)  // block b: A columns 8b.., B bytes 32b.. of each row
          tc_mma_i8_ts(tmem + kQDCol + 64u * b, tmem + kQACol + 8u * b, db + (uint64_t)((32 * b) >> 4), idesc, 0u);
        tc_commit(bar_mma);
      }
      const bool done = mbar_wait(bar_mma, phase);
      if (!done) set_device_error(ctrl, MOE_ERR_TIMEOUT, 51);
      phase ^= 1u;
      tc_fence_after();
      // read back each block's exact int32 sums and apply its scale
#pragma unroll
      for (int b = 0; b < kQBlocks; ++b) {
        const float dw = __half2float(__ushort_as_half((uint16_t)(((b < 2) ? dws.x : dws.y) >> (16 * (b & 1)))));
#pragma unroll
        for (int c0 = 0; c0 < kQBN; c0 += 16) {
          if (c0 < N) {
            uint32_t v[16];
            tmem_ld16_i(tmem + lane_base + kQDCol + 64u * b + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              acc[c0 + j] = fmaf(dw * s_dx[b * kQBN + c0 + j], (float)(int32_t)v[j], acc[c0 + j]);
          }
        }
      }
      tc_fence_before();
      // shared memory and tensor memory are rewritten by the next stage
      ok = __syncthreads_and(done) != 0;
    }
    if (!ok) break;
    // lanes 2i (gate) and 2i+1 (up) hold one feature's sums
    const int f = mt * 64 + (r >> 1);
    const bool up_lane = r & 1;
#pragma unroll
    for (int n = 0; n < kQBN; ++n) {
      const float v = acc[n];
      const float other = __shfl_xor_sync(0xffffffffu, v, 1);
      if (!up_lane && n < n_valid) {
        const float hv = v / (1.0f + expf(-v)) * other;
        const uint16_t hb = __half_as_ushort(__float2half_rn(hv));
        if (f16_inf(hb)) set_device_error(ctrl, MOE_ERR_RANGE, 52);
        args.h_perm[(size_t)(row_base + n) * args.I + f] = hb;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// x_perm fp16 rows -> int8 rows and one fp32 scale per 32-value block (max |x| / 127 over the
// block; an all-zero block gets scale 0 and zero codes). One warp per row, a lane 8 values, four
// lanes a block.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t *__restrict__ x, int rows, int H,
                                                           int8_t *__restrict__ xq, float *__restrict__ dx) {
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += gridDim.x * 8) {
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)r * H);
    for (int c = lane; c < H / 8; c += 32) {  // H % 256 == 0: every lane of the warp takes part
      const uint4 v = __ldg(xr + c);
      const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
      float f[8];
      float amax = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 t = __half22float2(*reinterpret_cast<const __half2 *>(&vv[q]));
        f[2 * q] = t.x;
        f[2 * q + 1] = t.y;
        amax = fmaxf(amax, fmaxf(fabsf(t.x), fabsf(t.y)));
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
      if ((lane & 3) == 0) dx[(size_t)r * (H / 32) + c / 4] = amax / 127.0f;
      uint32_t o2[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int a = max(-127, min(127, __float2int_rn(f[j] * inv)));
        o2[j >> 2] |= (uint32_t)(uint8_t)(int8_t)a << (8 * (j & 3));
      }
      reinterpret_cast<uint2 *>(xq + (size_t)r * H)[c] = make_uint2(o2[0], o2[1]);
    }
  }
}

}  // namespace

int mmq_shape_supported(int H, int I, int qtype) { return (qtype == MOE_Q2 && H % 256 == 0 && I % 64 == 0) ? 1 : 0; }

cudaError_t launch_mmq_gate_up(const uint16_t *x_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                               const moe_expert_set &routed, const moe_expert_set *shared, int8_t *x_q, float *dx,
                               uint16_t *h_perm, int2 *tiles, Ctrl *ctrl, cudaStream_t s) {
  const int G = E + (shared ? 1 : 0);
  const moe_expert_set &sh = shared ? *shared : routed;
  {
    KTimer kt_(KID_MMQ_QUANT, s);
    const int want = (n_rows + 7) / 8, cap = num_sms() * 16;
    quantize_rows_kernel<<<want < cap ? (want > 0 ? want : 1) : cap, 256, 0, s>>>(x_perm, n_rows, H, x_q, dx);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_tile_list(offsets, G, n_rows, kQBN, tiles, ctrl, s);
  if (e != cudaSuccess) return e;
  CUtensorMap tx, tg, tu, sg, su;
  auto code_map = [](CUtensorMap *m, const moe_qmat &q) {
    return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.codes, (uint64_t)q.K / 4,
                                (uint64_t)q.n_experts * q.rows, kQBK / 4, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
  };
  const bool mapped = encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, x_q, (uint64_t)H, (uint64_t)n_rows,
                                           kQBK, kQBN, CU_TENSOR_MAP_SWIZZLE_128B) &&
                      code_map(&tg, routed.gate) && code_map(&tu, routed.up) && code_map(&sg, sh.gate) &&
                      code_map(&su, sh.up);
  if (!mapped) return cudaErrorInvalidValue;
  MmqArgs a{};
  a.offsets = offsets;
  a.tiles = tiles;
  a.ctrl = ctrl;
  a.dx = dx;
  a.h_perm = h_perm;
  a.H = H;
  a.I = I;
  a.shared_group = shared ? E : -1;
  a.scales[0][0] = routed.gate.scales;
  a.scales[0][1] = routed.up.scales;
  a.scales[1][0] = sh.gate.scales;
  a.scales[1][1] = sh.up.scales;
  static_assert(kQSmem <= kQSmemRequest, "the stage fits the request");
  e = smem_limit_once(mmq_gate_up_kernel, kQSmemRequest);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_MMQ_GATE_UP, s);
    mmq_gate_up_kernel<<<num_sms(), kQThreads, kQSmemRequest, s>>>(tx, tg, tu, sg, su, a);
  }
  return cudaGetLastError();
}

}  // namespace moe
