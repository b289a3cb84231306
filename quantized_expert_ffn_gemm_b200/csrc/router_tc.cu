// Prefill router logits on the tensor cores.
//
// A prefill chunk scores every token against every expert: an [T x H] x [H x E] product
// ("Strata vs Llama.cpp vs vLLM", "How Strata is designed to work": tokens are routed to 10 of
// 512 experts; 8,192-token chunks). The router weights are fp32 and the top-k needs logits
// accurate to well under 1e-5, so fp32 weights are split exactly into three bf16 planes:
//   w = hi + mid + lo,  hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each subtraction is exact in fp32, and the leftover after three planes is below 2^-24 |w|).
// x is bf16 already, so x.w = x.hi + x.mid + x.lo with every product exact, accumulated in fp32
// by tcgen05.mma kind::f16 (bf16 x bf16 -> fp32) over K' = 3H: the A operand is the planes laid
// side by side along K, the B operand is x re-read once per plane (TMA coordinate k' mod H).
// Tile: 128 experts (M) x up to 256 tokens (N, chosen per launch so the tiles fill the SMs in one
// wave: 224 at 8,192 tokens and 512 experts, 148 CTAs). The epilogue adds the router bias and
// writes fp32 logits[t][e]; the top-k kernel then selects.
#include "common.cuh"
#include "tc.cuh"

namespace moe {

namespace {
constexpr int kRtStages = 4;
constexpr int kRtBK = 64;
constexpr int kRtThreads = 192;   // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 epilogue
constexpr int kRtA = 128 * kRtBK * 2;
constexpr int kRtB = 256 * kRtBK * 2;
constexpr int kRtStage = kRtA + kRtB;
constexpr int kRtSmem = kRtStages * kRtStage + (2 * kRtStages + 1) * 8 + 16 + 1024;
}  // namespace

// Wsp[e][p*H + h] = plane p of Wr[e][h]
__global__ void __launch_bounds__(256) router_split_kernel(const float *__restrict__ Wr, int E, int H,
                                                           __nv_bfloat16 *__restrict__ Wsp) {
  const size_t n = (size_t)E * H;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t e = i / H, h = i % H;
    const float w = Wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    __nv_bfloat16 *row = Wsp + e * (size_t)(3 * H);
    row[h] = hi;
    row[H + h] = mid;
    row[2 * H + h] = lo;
  }
}

__global__ void __launch_bounds__(kRtThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, int T, int H,
                 int E, const float *__restrict__ bias, float *__restrict__ logits, int ntile, Ctrl *ctrl) {
  extern __shared__ uint8_t smem_raw[];
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * ntile;
  const int n_valid = min(ntile, T - n0);
  if (n_valid <= 0) return;
  const int N = (n_valid + 15) & ~15;
  const int nbox = (N + 31) / 32;
  const int nk = 3 * H / kRtBK;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - smem_u32(smem_raw));
  auto sA = [&](int s) { return base + s * kRtStage; };
  auto sB = [&](int s) { return base + s * kRtStage + kRtA; };
  const uint32_t bar0 = base + kRtStages * kRtStage;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kRtStages + s); };
  const uint32_t accum = bar0 + 8u * (2 * kRtStages);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kRtStages * kRtStage + (2 * kRtStages + 1) * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t tx = kRtA + (uint32_t)nbox * 32 * kRtBK * 2;
      for (int ks = 0; ks < nk; ++ks) {
        const int s = ks % kRtStages;
        const uint32_t ph = (uint32_t)(ks / kRtStages) & 1u;
        if (!mbar_wait(empty(s), ph ^ 1u)) { set_device_error(ctrl, MOE_ERR_TIMEOUT, 11); break; }
        mbar_arrive_expect_tx(full(s), tx);
        tma_load_2d(sA(s), &tm_w, ks * kRtBK, m0, full(s));
        const int xk = (ks * kRtBK) % H;  // the same x columns for every weight plane
        for (int b = 0; b < nbox; ++b) tma_load_2d(sB(s) + b * 32 * kRtBK * 2, &tm_x, xk, n0 + 32 * b, full(s));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(N, true);
      bool ok = true;
      for (int ks = 0; ks < nk; ++ks) {
        const int s = ks % kRtStages;
        const uint32_t ph = (uint32_t)(ks / kRtStages) & 1u;
        if (!mbar_wait(full(s), ph)) { set_device_error(ctrl, MOE_ERR_TIMEOUT, 12); ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk)
          tc_mma(tmem, sw128_desc(sA(s) + kk * 32), sw128_desc(sB(s) + kk * 32), idesc, (ks | kk) != 0 ? 1u : 0u);
        tc_commit(empty(s));
      }
      if (ok) tc_commit(accum);
    }
  } else {
    // epilogue warps 2..5 cover TMEM lane quadrants 2, 3, 0, 1
    bool go = __all_sync(0xffffffffu, mbar_wait(accum, 0));
    if (go) {
      tc_fence_after();
      const int q = warp & 3;
      const int e = m0 + 32 * q + lane;
      const float b = bias ? bias[e] : 0.0f;
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
      for (int c0 = 0; c0 < N; c0 += 8) {
        uint32_t v[8];
        tmem_ld8(lane_addr + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = c0 + j;
          if (n < n_valid) logits[(size_t)(n0 + n) * E + e] = __uint_as_float(v[j]) + b;
        }
      }
    } else if (lane == 0) {
      set_device_error(ctrl, MOE_ERR_TIMEOUT, 13);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
  }
}

bool router_tc_supported(int H, int E) { return E % 128 == 0 && H % 64 == 0; }

cudaError_t launch_router_tc(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E,
                             uint16_t *wsplit, float *logits, Ctrl *ctrl, cudaStream_t s) {
  {
    KTimer kt_(KID_ROUTER_SPLIT, s);
    const size_t n = (size_t)E * H;
    const int grid = (int)((n + 255) / 256 < (size_t)num_sms() * 8 ? (n + 255) / 256 : (size_t)num_sms() * 8);
    router_split_kernel<<<grid, 256, 0, s>>>(Wr, E, H, reinterpret_cast<__nv_bfloat16 *>(wsplit));
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tw, tx;
  if (!encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wsplit, (uint64_t)3 * H, E, kRtBK, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, H, T, kRtBK, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  e = smem_limit_once(router_tc_kernel, kRtSmem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(KID_ROUTER_TC, s);
    // token tile: a multiple of 32 (the activation boxes), at most 256, and as small as one wave
    // of 128-expert x ntile tiles over the SMs allows
    const int rows_tiles = E / 128;
    int ntile = (int)(((size_t)T * rows_tiles + num_sms() - 1) / num_sms());
    ntile = ntile < 32 ? 32 : ntile > 256 ? 256 : (ntile + 31) & ~31;
    router_tc_kernel<<<dim3(rows_tiles, (T + ntile - 1) / ntile), kRtThreads, kRtSmem, s>>>(tw, tx, T, H, E, bias,
                                                                                        logits, ntile, ctrl);
  }
  return cudaGetLastError();
}

}  // namespace moe
