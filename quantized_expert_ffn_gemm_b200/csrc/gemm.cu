// Prefill expert path: grouped GEMM over expert-contiguous rows on the 5th-generation tensor cores.
//
// In a prefill chunk each active expert collects many tokens, so its weights are reused across
// all of them ("Two-Day Port, 8x Faster Prefill: Strata Engine Benchmarked", "Where Strata Is
// Fast: Not Magic, but Logistics": the larger the prefill batch, the more tokens per expert),
// and the expert matmul dequantizes block weights inside the multiply (same section, MMQ
// paragraph). On sm_100a this becomes, per tile (group g, 128 weight rows, <= 256 token rows):
//
//   TMA      activation rows (fp16, 128B-swizzled K-major) and the packed 2-bit code plane of
//            the 128 weight rows -> shared memory, one mbarrier per pipeline stage
//   dequant  8 warps turn codes (+ per-block fp16 scales, + the Q3 hi-bit plane) into fp16
//            weights written straight into the UMMA canonical 128B-swizzled K-major layout
//   MMA      one thread issues tcgen05.mma kind::f16 (fp16 x fp16 -> fp32) with the weights as
//            A (M = 128) and the tokens as B (N = token rows of the tile, multiple of 16), so a
//            group of ~160 rows is one N = 160 tile (swap-AB); accumulators live in TMEM
//   epilogue tcgen05.ld -> registers; gate/up: h = silu(g) * u (both accumulators in TMEM),
//            down: the expert output row; stored as fp16
//
// Kernel 1 (NMAT = 2) computes gate and up for the same 128 intermediate features and fuses
// SwiGLU; kernel 2 (NMAT = 1) is the down projection. Every mbarrier wait is bounded in time;
// a wait that gives up records MOE_ERR_TIMEOUT in the workspace and the CTA winds down, frees
// its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "dequant.cuh"
#include "tc.cuh"

namespace moe {

constexpr int kBK = 64;            // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int kBM = 128;           // weight rows per tile (MMA M)
constexpr int kBNMax = 256;        // token rows per tile (MMA N upper bound)
constexpr int kBoxRows = 32;       // rows per TMA box of the activation tile
constexpr int kThreads = 320;      // warp 0 TMA, warp 1 MMA/TMEM, warps 2..9 dequant + epilogue
constexpr int kDqThreads = 256;

struct GemmArgs {
  const int32_t *offsets;
  const int2 *tiles;
  Ctrl *ctrl;
  uint16_t *out;                   // h_perm (kernel 1) or out_perm (kernel 2)
  int ldo;                         // row stride of `out` in elements
  int K;                           // reduction dim (H for gate/up, I for down)
  int M;                           // weight rows per expert (I for gate/up, H for down)
  int shared_group;                // group index served by the shared expert, -1 if none
  int q3;
  const uint16_t *scales[2][2];    // [set][mat]
  const uint8_t *hibits[2][2];     // [set][mat]
};

__device__ __forceinline__ void record_timeout(Ctrl *c, int where) { set_device_error(c, MOE_ERR_TIMEOUT, where); }

// ---------------------------------------------------------------- the grouped GEMM kernel
template <int NMAT, int STAGES>
struct Smem {
  static constexpr int kB = kBNMax * kBK * 2;   // 32 KB activation tile
  static constexpr int kA = kBM * kBK * 2;      // 16 KB dequantized weight tile
  static constexpr int kRaw = kBM * kBK / 4;    // 2 KB packed codes
  static constexpr int kStage = kB + NMAT * kA + NMAT * kRaw;
  static constexpr int kBar = STAGES * kStage;  // barriers after the stages
  static constexpr int kBytes = kBar + (3 * STAGES + 1) * 8 + 16;
};

template <int NMAT, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
grouped_ffn_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c0r,
                   const __grid_constant__ CUtensorMap tm_c1r, const __grid_constant__ CUtensorMap tm_c0s,
                   const __grid_constant__ CUtensorMap tm_c1s, const GemmArgs args) {
  using SL = Smem<NMAT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  Ctrl *ctrl = args.ctrl;
  if ((int)blockIdx.x >= ctrl->n_tiles) return;
  const int2 tl = args.tiles[blockIdx.x];
  const int grp = tl.x, n0 = tl.y;
  const int set = (grp == args.shared_group) ? 1 : 0;
  const int expert = set ? 0 : grp;
  const int row_base = args.offsets[grp] + n0;
  const int n_valid = min(kBNMax, args.offsets[grp + 1] - row_base);
  if (n_valid <= 0) return;
  const int N = (n_valid + 15) & ~15;
  const int nbox = (N + kBoxRows - 1) / kBoxRows;
  const int m0 = blockIdx.y * kBM;
  const int K = args.K, nk = K / kBK;

  // 1024-byte aligned base (the 128B swizzle pattern is taken from address bits 4..9)
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - smem_u32(smem_raw));
  auto sB = [&](int s) { return base + s * SL::kStage; };
  auto sA = [&](int s, int m) { return base + s * SL::kStage + SL::kB + m * SL::kA; };
  auto sR = [&](int s, int m) { return base + s * SL::kStage + SL::kB + NMAT * SL::kA + m * SL::kRaw; };
  const uint32_t bar0 = base + SL::kBar;
  auto full_b = [&](int s) { return bar0 + 8u * s; };
  auto full_a = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  const uint32_t accum_full = bar0 + 8u * (3 * STAGES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + SL::kBar + (3 * STAGES + 1) * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_b(s), 1);
      mbar_init(full_a(s), kDqThreads);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum_full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap *mc0 = set ? &tm_c0s : &tm_c0r;
      const CUtensorMap *mc1 = set ? &tm_c1s : &tm_c1r;
      const uint32_t tx = (uint32_t)nbox * kBoxRows * kBK * 2 + NMAT * SL::kRaw;
      const int wrow = expert * args.M + m0;
      for (int ks = 0; ks < nk; ++ks) {
        const int s = ks % STAGES;
        const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
        if (!mbar_wait(empty(s), ph ^ 1u)) { record_timeout(ctrl, 1); break; }
        mbar_arrive_expect_tx(full_b(s), tx);
        for (int b = 0; b < nbox; ++b)
          tma_load_2d(sB(s) + b * kBoxRows * kBK * 2, &tm_b, ks * kBK, row_base + b * kBoxRows, full_b(s));
        tma_load_2d(sR(s, 0), mc0, ks * (kBK / 4), wrow, full_b(s));
        if (NMAT == 2) tma_load_2d(sR(s, 1), mc1, ks * (kBK / 4), wrow, full_b(s));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(N);
      bool ok = true;
      for (int ks = 0; ks < nk && ok; ++ks) {
        const int s = ks % STAGES;
        const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
        if (!mbar_wait(full_b(s), ph) || !mbar_wait(full_a(s), ph)) { record_timeout(ctrl, 2); ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t bd = sw128_desc(sB(s) + kk * 32);
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
            tc_mma(tmem + m * 256, sw128_desc(sA(s, m) + kk * 32), bd, idesc, (ks | kk) != 0 ? 1u : 0u);
        }
        tc_commit(empty(s));
      }
      if (ok) tc_commit(accum_full);
    }
  } else {
    // ------------------------------------------------ dequant warps
    const int td = threadIdx.x - 64;          // 0..255
    const int r = td >> 1, blk = td & 1;      // weight row within the tile, 32-weight block of the stage
    const size_t grow = (size_t)expert * args.M + m0 + r;
    const uint16_t *scp[NMAT];
    const uint8_t *hbp[NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {  // scalar selects keep the parameter block out of local memory
      const uint16_t *sc = set ? args.scales[1][m] : args.scales[0][m];
      const uint8_t *hb = set ? args.hibits[1][m] : args.hibits[0][m];
      scp[m] = sc + grow * (K / 32);
      hbp[m] = args.q3 ? hb + grow * (K / 8) : nullptr;
    }
    // scales (and Q3 hi words) for groups of 4 stages, prefetched one group ahead
    uint32_t sc_cur[NMAT][4], sc_nxt[NMAT][4], hb_cur[NMAT][4], hb_nxt[NMAT][4];
    auto load_group = [&](int gi, uint32_t (&sc)[NMAT][4], uint32_t (&hb)[NMAT][4]) {
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ks = 4 * gi + j;
          sc[m][j] = (ks < nk) ? (uint32_t)__ldg(scp[m] + 2 * ks + blk) : 0u;
          hb[m][j] = (args.q3 && ks < nk) ? __ldg(reinterpret_cast<const uint32_t *>(hbp[m]) + 2 * ks + blk) : 0u;
        }
    };
    load_group(0, sc_cur, hb_cur);
    bool ok = true;
    for (int gi = 0; gi * 4 < nk && ok; ++gi) {
      if ((gi + 1) * 4 < nk) load_group(gi + 1, sc_nxt, hb_nxt);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ks = 4 * gi + j;
        if (ks >= nk) break;
        const int s = ks % STAGES;
        const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
        if (!mbar_wait(full_b(s), ph)) { record_timeout(ctrl, 3); ok = false; break; }
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          const uint2 cw = *reinterpret_cast<const uint2 *>(gbase + (sR(s, m) - base) + r * 16 + blk * 8);
          const __half2 d2 = __half2half2(__ushort_as_half((uint16_t)sc_cur[m][j]));
          uint32_t p[16];
          if (args.q3) {
            dq3_word(cw.x, hb_cur[m][j], 0, d2, p);
            dq3_word(cw.y, hb_cur[m][j], 1, d2, p + 8);
          } else {
            dq2_word(cw.x, d2, p);
            dq2_word(cw.y, d2, p + 8);
          }
          uint8_t *arow = gbase + (sA(s, m) - base) + r * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int chunk = 4 * blk + c;
            *reinterpret_cast<uint4 *>(arow + ((chunk ^ (r & 7)) << 4)) =
                make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
          }
        }
        fence_async_smem();
        mbar_arrive(full_a(s));
      }
      if ((gi + 1) * 4 < nk) {
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            sc_cur[m][j] = sc_nxt[m][j];
            hb_cur[m][j] = hb_nxt[m][j];
          }
      }
    }
    // ------------------------------------------------ epilogue (same 8 warps)
    // the decision is made warp-uniform: tcgen05.ld is a warp-wide instruction
    bool go = __all_sync(0xffffffffu, ok);
    if (go) go = __all_sync(0xffffffffu, mbar_wait(accum_full, 0));
    if (go) {
      tc_fence_after();
      const int q = warp & 3, half = (warp - 2) >> 2;
      const int row = 32 * q + lane;
      const int f = m0 + row;
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
      const int c_begin = half * (N / 2), c_end = c_begin + N / 2;
      for (int c0 = c_begin; c0 < c_end; c0 += 8) {
        uint32_t a[8], b[8];
        tmem_ld8(lane_addr + c0, a);
        if (NMAT == 2) tmem_ld8(lane_addr + 256 + c0, b);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = c0 + j;
          if (n >= n_valid) break;
          float v = __uint_as_float(a[j]);
          if (NMAT == 2) {
            const float u = __uint_as_float(b[j]);
            v = v / (1.0f + expf(-v)) * u;
          }
          args.out[(size_t)(row_base + n) * args.ldo + f] = __half_as_ushort(__float2half_rn(v));
        }
      }
    } else if (ok && lane == 0) {
      record_timeout(ctrl, 4);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------- tile list
// entries (group, first row within the group) for every 256-row slice of every non-empty group
// (offsets that are not monotone or run past n_rows flag the error word and yield no tiles)
__global__ void __launch_bounds__(1024) tile_list_kernel(const int32_t *__restrict__ off, int G, int n_rows,
                                                         int2 *__restrict__ tiles, Ctrl *__restrict__ ctrl) {
  __shared__ int s_warp[32];
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int g = tid; g < G; g += blockDim.x)
    if (off[g] < 0 || off[g + 1] < off[g] || off[g + 1] > n_rows) s_bad = 1;
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      ctrl->n_tiles = 0;
      set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, -1);
    }
    return;
  }
  const int per = (G + 1023) / 1024;  // <= 5
  int cnt[5];
  int mine = 0;
  for (int i = 0; i < per; ++i) {
    const int g = tid * per + i;
    int c = 0;
    if (g < G) c = (off[g + 1] - off[g] + kBNMax - 1) / kBNMax;
    cnt[i] = c;
    mine += c;
  }
  int v = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int wv = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += n;
    }
    s_warp[lane] = wv;
  }
  __syncthreads();
  int pos = v - mine + (warp > 0 ? s_warp[warp - 1] : 0);
  for (int i = 0; i < per; ++i) {
    const int g = tid * per + i;
    for (int j = 0; j < cnt[i]; ++j) tiles[pos++] = make_int2(g, j * kBNMax);
  }
  if (tid == 1023) ctrl->n_tiles = pos;
}

// ---------------------------------------------------------------- host side
namespace {
}  // namespace

namespace {

bool make_code_map(CUtensorMap *map, const moe_qmat &m) {
  return encode_tensor_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, m.codes, (uint64_t)m.K / 4, (uint64_t)m.n_experts * m.rows,
                  kBK / 4, kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int NMAT, int STAGES>
cudaError_t launch_one(const CUtensorMap &tb, const CUtensorMap &c0r, const CUtensorMap &c1r, const CUtensorMap &c0s,
                       const CUtensorMap &c1s, const GemmArgs &a, int grid_x, int grid_y, cudaStream_t s) {
  const int smem = Smem<NMAT, STAGES>::kBytes + 1024;
  cudaError_t e = smem_limit_once(grouped_ffn_kernel<NMAT, STAGES>, smem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(NMAT == 2 ? KID_GEMM_GATE_UP : KID_GEMM_DOWN, s);
    grouped_ffn_kernel<NMAT, STAGES><<<dim3(grid_x, grid_y), kThreads, smem, s>>>(tb, c0r, c1r, c0s, c1s, a);
  }
  return cudaGetLastError();
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *ptr, uint64_t inner,
                          uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * (uint64_t)esize};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int gemm_shape_supported(int H, int I) { return (H % 128 == 0 && I % 128 == 0 && H >= 128 && I >= 128) ? 1 : 0; }

cudaError_t launch_grouped_ffn(const uint16_t *x_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                               const moe_expert_set &routed, const moe_expert_set *shared, uint16_t *h_perm,
                               uint16_t *out_perm, int2 *tiles, Ctrl *ctrl, cudaStream_t s) {
  const int G = E + (shared ? 1 : 0);
  const moe_expert_set &sh = shared ? *shared : routed;
  {
    KTimer kt_(KID_TILE_LIST, s);
    tile_list_kernel<<<1, 1024, 0, s>>>(offsets, G, n_rows, tiles, ctrl);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int max_tiles = n_rows / kBNMax + G + 1;

  CUtensorMap tx, th, cg, cu, cd, sg, su, sd;
  bool ok = encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x_perm, H, n_rows, kBK, kBoxRows,
                                 CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tensor_map_2d(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h_perm, I, n_rows, kBK, kBoxRows,
                                 CU_TENSOR_MAP_SWIZZLE_128B) &&
            make_code_map(&cg, routed.gate) && make_code_map(&cu, routed.up) && make_code_map(&cd, routed.down) &&
            make_code_map(&sg, sh.gate) && make_code_map(&su, sh.up) && make_code_map(&sd, sh.down);
  if (!ok) return cudaErrorInvalidValue;

  GemmArgs a{};
  a.offsets = offsets;
  a.tiles = tiles;
  a.ctrl = ctrl;
  a.shared_group = shared ? E : -1;
  a.q3 = routed.gate.qtype == MOE_Q3 ? 1 : 0;
  // kernel 1: gate/up + SwiGLU -> h_perm
  a.out = h_perm;
  a.ldo = I;
  a.K = H;
  a.M = I;
  a.scales[0][0] = routed.gate.scales;
  a.scales[0][1] = routed.up.scales;
  a.scales[1][0] = sh.gate.scales;
  a.scales[1][1] = sh.up.scales;
  a.hibits[0][0] = routed.gate.hibits;
  a.hibits[0][1] = routed.up.hibits;
  a.hibits[1][0] = sh.gate.hibits;
  a.hibits[1][1] = sh.up.hibits;
  e = launch_one<2, 3>(tx, cg, cu, sg, su, a, max_tiles, I / kBM, s);
  if (e != cudaSuccess) return e;
  // kernel 2: down -> out_perm
  a.out = out_perm;
  a.ldo = H;
  a.K = I;
  a.M = H;
  a.scales[0][0] = routed.down.scales;
  a.scales[0][1] = nullptr;
  a.scales[1][0] = sh.down.scales;
  a.scales[1][1] = nullptr;
  a.hibits[0][0] = routed.down.hibits;
  a.hibits[0][1] = nullptr;
  a.hibits[1][0] = sh.down.hibits;
  a.hibits[1][1] = nullptr;
  return launch_one<1, 4>(th, cd, cd, sd, sd, a, max_tiles, H / kBM, s);
}

}  // namespace moe
