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
//            weights and store them straight into tensor memory (tcgen05.st), one weight row per
//            TMEM lane: the A operand never touches shared memory, which leaves the shared-memory
//            bandwidth to the activation tiles (TMA writes and MMA reads)
//   MMA      one thread issues tcgen05.mma kind::f16 (fp16 x fp16 -> fp32) with the weights as
//            A (M = 128, from TMEM) and the tokens as B (N = token rows of the tile, multiple of
//            16, <= 192), so a group of ~160 rows is one N = 160 tile (swap-AB); accumulators
//            live in TMEM too
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

constexpr int kBK = 128;           // K per pipeline stage: two 64-wide 128-byte swizzle sub-tiles
constexpr int kSubK = 64;          // K of one swizzle sub-tile (128 bytes of fp16 per row)
constexpr int kBM = 128;           // weight rows per tile (MMA M)
constexpr int kBNMax = 192;        // token rows per tile (MMA N upper bound; TMEM: 2 x 192 + A ring)
constexpr int kBoxRows = 64;       // rows per TMA box of the activation tile (fewer, larger requests)

struct GemmArgs {
  const int32_t *offsets;
  const int2 *tiles;
  Ctrl *ctrl;
  uint16_t *out;                   // h_perm (kernel 1) or out_perm (kernel 2)
  int ldo;                         // row stride of `out` in elements
  int K;                           // reduction dim (H for gate/up, I for down)
  int M;                           // weight rows per expert (I for gate/up, H for down)
  int shared_group;                // group index served by the shared expert, -1 if none
  const uint16_t *scales[2][2];    // [set][mat]
  const uint8_t *hibits[2][2];     // [set][mat]
};

__device__ __forceinline__ void record_timeout(Ctrl *c, int where) { set_device_error(c, MOE_ERR_TIMEOUT, where); }

// ---------------------------------------------------------------- the grouped GEMM kernel
// Persistent: gridDim.x CTAs walk the tile list round-robin (tile ti = blockIdx.x + i * gridDim.x,
// entry = ti / n_mtiles, m-tile = ti % n_mtiles), so consecutive CTAs share a token block and the
// roles never drain between tiles.
//   warp 0      TMA producer: activation rows (swizzled) + the 128 weight rows' code plane
//   warp 1      TMEM owner and single-thread MMA issuer
//   warps 2-9   dequant: code plane + per-block scales (+ Q3 hi bits) -> fp16 A tile
//   warps 10-13 epilogue: TMEM -> registers -> global, one lane quadrant each
// A stage covers K = 128 (eight MMAs, one commit: every tcgen05.mma costs ~100 cycles of issue
// at these shapes, so the per-stage waits and commits are spread over eight of them). Two
// rings. Shared memory: kStagesB stages of activation tile (two 64-wide swizzled sub-tiles) +
// code plane (full_b: TMA landed, empty_b: the stage's MMAs are done). TMEM: kStagesA stages of
// the dequantized A tile, 128 lanes x 64 columns (full_a: written by the dequant warps; a stage
// is reused once empty_b of the stage kStagesA back has completed). TMEM (512 columns):
// accumulators at columns 0 and 256 (up to 192 columns each; acc_full: tile's MMAs done,
// acc_empty: drained), A stages at 192 and 448.
// MODE_GU: A row 2i is gate row f0+i and row 2i+1 the up row of the same feature (64 features,
// one accumulator holds both), so the epilogue pairs adjacent lanes with one shuffle per value
// and writes h = silu(gate) * up. The TMA still brings the 64 gate rows' codes (smem rows 0-63)
// and the 64 up rows' codes (rows 64-127); the dequant warps read them interleaved.
// MODE_DN: A rows are 128 rows of W_down.
enum { MODE_GU = 0, MODE_DN = 1 };

constexpr int kStagesB = 4;
constexpr int kStagesA = 2;
constexpr int kThreadsV2 = 448;
constexpr int kEpiWarp0 = 10;

// bytes of the code plane per weight row for K weights: 2-bit plane K/4, 4-bit plane (Q4) K/2
__host__ __device__ constexpr int gemm_code_bytes(int qt, int K) { return qt == 4 ? K / 2 : K / 4; }

template <int QT>
struct SmemV2 {
  static constexpr int kSub = kBNMax * kSubK * 2;  // 24 KB: one 64-wide sub-tile of the activation rows
  static constexpr int kB = 2 * kSub;              // 48 KB activation tile (K = 128)
  static constexpr int kRowCodes = gemm_code_bytes(QT, kBK);  // code bytes of one weight row per stage
  static constexpr int kRaw = kBM * kRowCodes;     // 4 KB packed codes (8 KB for the 4-bit plane)
  static constexpr int kStage = kB + kRaw;         // multiple of 1024 (128B-swizzle atoms)
  static constexpr int kBar = kStagesB * kStage;
  static constexpr int kNumBars = 2 * kStagesB + kStagesA + 4;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
};

static_assert(SmemV2<2>::kStage % 1024 == 0 && SmemV2<4>::kStage % 1024 == 0 && SmemV2<2>::kSub % 1024 == 0,
              "stages keep the 1024-byte swizzle alignment");
static_assert(SmemV2<4>::kBytes + 1024 <= 232448, "the 4-bit plane's stages fit the shared-memory limit");
static_assert(kStagesA == 2, "TMEM holds two A stages");

// TMEM column of A stage s (64 columns: 128 K of fp16 pairs)
__device__ __forceinline__ uint32_t a_col(int s) { return 192u + 256u * (uint32_t)s; }

struct TileInfo {
  int expert, set, row_base, n_valid, N, mt;
};

// A CTA's tiles, looked up once in the prologue: the lookup is a dependent pair of global loads
// (tile entry, then its group's offsets), and a role that did it at each tile switch stalled on
// both round trips there (measured: ~2,300 cycles per switch in the TMA producer and the MMA thread).
constexpr int kTileCache = 128;
struct TileC {
  int expert_set_mt;  // expert << 9 | set << 8 | m-tile
  int row_base, n_valid;
};
static_assert(SmemV2<4>::kBytes + 1024 + kTileCache * sizeof(TileC) <= 232448,
              "the stages and the tile cache fit the shared-memory limit");
__device__ __forceinline__ TileC tile_pack(const TileInfo &t) {
  return TileC{(t.expert << 9) | (t.set << 8) | t.mt, t.row_base, t.n_valid};
}
__device__ __forceinline__ TileInfo tile_unpack(const TileC &c) {
  TileInfo t;
  t.expert = c.expert_set_mt >> 9;
  t.set = (c.expert_set_mt >> 8) & 1;
  t.mt = c.expert_set_mt & 255;
  t.row_base = c.row_base;
  t.n_valid = c.n_valid;
  t.N = (c.n_valid + 15) & ~15;
  return t;
}

__device__ __forceinline__ TileInfo get_tile(const GemmArgs &a, int ti, int n_mtiles) {
  TileInfo t;
  const int entry = ti / n_mtiles;
  t.mt = ti - entry * n_mtiles;
  const int2 e = a.tiles[entry];
  t.set = (e.x == a.shared_group) ? 1 : 0;
  t.expert = t.set ? 0 : e.x;
  t.row_base = a.offsets[e.x] + e.y;
  t.n_valid = min(kBNMax, a.offsets[e.x + 1] - t.row_base);
  t.N = (t.n_valid + 15) & ~15;
  return t;
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

template <int MODE, int QT>
__global__ void __launch_bounds__(kThreadsV2, 1)
grouped_v2_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c0r,
                  const __grid_constant__ CUtensorMap tm_c1r, const __grid_constant__ CUtensorMap tm_c0s,
                  const __grid_constant__ CUtensorMap tm_c1s, const GemmArgs args) {
  using SL = SmemV2<QT>;
  extern __shared__ uint8_t smem_raw[];
  Ctrl *ctrl = args.ctrl;
  const int n_mtiles = (MODE == MODE_GU) ? args.M / 64 : args.M / kBM;
  const int total = ctrl->n_tiles * n_mtiles;
  const int G = gridDim.x;
  const int n_my = (total > (int)blockIdx.x) ? (total - (int)blockIdx.x + G - 1) / G : 0;
  if (n_my == 0) return;
  const int K = args.K, nk = K / kBK;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - smem_u32(smem_raw));
  auto sB = [&](int s) { return base + s * SL::kStage; };
  auto sR = [&](int s) { return base + s * SL::kStage + SL::kB; };
  const uint32_t bar0 = base + SL::kBar;
  auto full_b = [&](int s) { return bar0 + 8u * s; };
  auto empty_b = [&](int s) { return bar0 + 8u * (kStagesB + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * kStagesB + s); };
  constexpr int kB0 = 2 * kStagesB + kStagesA;
  auto acc_full = [&](int b) { return bar0 + 8u * (kB0 + b); };
  auto acc_empty = [&](int b) { return bar0 + 8u * (kB0 + 2 + b); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + SL::kBar + SL::kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ TileC s_tiles[kTileCache];
  for (int t = threadIdx.x; t < n_my && t < kTileCache; t += blockDim.x)
    s_tiles[t] = tile_pack(get_tile(args, blockIdx.x + t * G, n_mtiles));
  // tile tl of this CTA (from the prologue's copy; beyond it, looked up directly)
  auto tile_at = [&](int tl) -> TileInfo {
    return tl < kTileCache ? tile_unpack(s_tiles[tl]) : get_tile(args, blockIdx.x + tl * G, n_mtiles);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesB; ++s) {
      mbar_init(full_b(s), 1);
      mbar_init(empty_b(s), 1);
    }
    for (int s = 0; s < kStagesA; ++s) mbar_init(full_a(s), 256);  // all eight dequant warps
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 4);
    }
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
      TileInfo cur = tile_at(0);
      bool ok = true;
      for (int tl = 0; tl < n_my && ok; ++tl) {
        const TileInfo nxt = (tl + 1 < n_my) ? tile_at(tl + 1) : cur;
        const int nbox = (cur.N + kBoxRows - 1) / kBoxRows;
        const uint32_t tx = (uint32_t)nbox * kBoxRows * kBK * 2 + SL::kRaw;  // both sub-tiles + codes
        const CUtensorMap *mc0 = cur.set ? &tm_c0s : &tm_c0r;
        const CUtensorMap *mc1 = cur.set ? &tm_c1s : &tm_c1r;
        const int wrow = (MODE == MODE_GU) ? cur.expert * args.M + cur.mt * 64 : cur.expert * args.M + cur.mt * kBM;
        for (int ks = 0; ks < nk; ++ks) {
          const int g = tl * nk + ks;
          const int s = g % kStagesB;
          const uint32_t ph = (uint32_t)(g / kStagesB) & 1u;
          if (!mbar_wait(empty_b(s), ph ^ 1u)) { record_timeout(ctrl, 21); ok = false; break; }
          mbar_arrive_expect_tx(full_b(s), tx);
          for (int h = 0; h < 2; ++h)
            for (int b = 0; b < nbox; ++b)
              tma_load_2d(sB(s) + h * SL::kSub + b * kBoxRows * kSubK * 2, &tm_b, ks * kBK + h * kSubK,
                          cur.row_base + b * kBoxRows, full_b(s));
          if (MODE == MODE_GU) {  // gate rows -> A rows 0..63, up rows -> A rows 64..127
            tma_load_2d(sR(s), mc0, ks * SL::kRowCodes, wrow, full_b(s));
            tma_load_2d(sR(s) + 64 * SL::kRowCodes, mc1, ks * SL::kRowCodes, wrow, full_b(s));
          } else {
            tma_load_2d(sR(s), mc0, ks * SL::kRowCodes, wrow, full_b(s));
          }
        }
        cur = nxt;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      TileInfo cur = tile_at(0);
      bool ok = true;
      for (int tl = 0; tl < n_my && ok; ++tl) {
        const TileInfo nxt = (tl + 1 < n_my) ? tile_at(tl + 1) : cur;
        const int b = tl & 1;
        if (!mbar_wait(acc_empty(b), (((uint32_t)tl >> 1) & 1u) ^ 1u)) { record_timeout(ctrl, 22); ok = false; break; }
        tc_fence_after();
        const uint32_t idesc = idesc_f16(cur.N);
        const uint32_t d = tmem + (uint32_t)(b * 256);
        // the next stage's barriers are tested while this stage's MMAs queue up, so a stage whose
        // operands are already in place costs no wait between the MMA groups
        // full_a alone gates a stage: the dequant warps arrive on it only after they have seen
        // the stage's TMA complete (full_b), so the activation tile is in place too
        {
          const int g = tl * nk;
          if (!mbar_wait(full_a(g % kStagesA), (uint32_t)(g / kStagesA) & 1u)) {
            record_timeout(ctrl, 23);
            ok = false;
          }
        }
        for (int ks = 0; ks < nk && ok; ++ks) {
          const int g = tl * nk + ks;
          const int s = g % kStagesB, sa = g % kStagesA;
          // operand addresses of the stage's eight MMAs, computed before the first is issued (the
          // descriptor's start-address field is addr >> 4 in 14 bits; offsets inside the stage
          // never carry out of it: shared memory is below 256 KB)
          const uint64_t db = sw128_desc(sB(s));
          const uint32_t ta = tmem + a_col(sa);
          tc_fence_after();
          tc_mma_ts(d, ta, db, idesc, ks != 0 ? 1u : 0u);
          const bool more = ks + 1 < nk;
          const int sa1 = (g + 1) % kStagesA;
          const uint32_t pha1 = (uint32_t)((g + 1) / kStagesA) & 1u;
          bool ra = false;
#pragma unroll
          for (int kk = 1; kk < kBK / 16; ++kk) {  // sub-tile kk / 4, 32 bytes per 16 K inside it
            tc_mma_ts(d, ta + 8u * kk, db + (uint64_t)((((kk >> 2) * SL::kSub) + (kk & 3) * 32) >> 4), idesc, 1u);
            if (more && kk == 5) ra = mbar_test(full_a(sa1), pha1);  // next stage, tested while MMAs queue
          }
          tc_commit(empty_b(s));  // frees the smem stage, and (kStagesA stages on) the TMEM A stage
          if (more && !ra && !mbar_wait(full_a(sa1), pha1)) {
            record_timeout(ctrl, 23);
            ok = false;
          }
        }
        if (ok) tc_commit(acc_full(b));
        cur = nxt;
      }
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------ dequant warps
    // warp w writes TMEM lanes 32*(w%4)..+31 (the lanes a warp may access): A row r = that lane.
    // Warps 2-5 take K 0..63 of every stage and warps 6-9 K 64..127, a thread one 64-weight row
    // slice (two 32-weight blocks) per stage.
    const int qd = warp & 3;
    const int r = 32 * qd + lane, hh = (warp - 2) >> 2;
    const uint32_t a_lane = (uint32_t)(32 * qd) << 16;
    const int mat = (MODE == MODE_GU) ? (r & 1) : 0;
    const int crow = (MODE == MODE_GU) ? ((r & 1) ? 64 + (r >> 1) : (r >> 1)) : r;  // code row in the stage
    const int total_g = n_my * nk;
    // per-tile pointers to this row's scales (two per 64-weight slice: one u32) and Q3 hi words
    // (two per slice: one uint2); slice 2 ks + hh of the row is this thread's share of stage ks
    auto row_ptrs = [&](int tl, const uint32_t *&sp, const uint2 *&hp) {
      const TileInfo ti = tile_at(tl);
      const int mt = ti.mt, set = ti.set, expert = ti.expert;
      const int wrow = (MODE == MODE_GU) ? mt * 64 + (r >> 1) : mt * kBM + r;
      const size_t grow = (size_t)expert * args.M + wrow;
      const uint16_t *sc = set ? (mat ? args.scales[1][1] : args.scales[1][0])
                               : (mat ? args.scales[0][1] : args.scales[0][0]);
      const uint8_t *hb = set ? (mat ? args.hibits[1][1] : args.hibits[1][0])
                              : (mat ? args.hibits[0][1] : args.hibits[0][0]);
      sp = reinterpret_cast<const uint32_t *>(sc + grow * (K / 32)) + hh;
      hp = QT == 3 ? reinterpret_cast<const uint2 *>(hb + grow * (K / 8)) + hh : nullptr;
    };
    // scales (and Q3 hi words) are fetched four stages ahead into a 4-entry register ring
    int pf_tl = 0;
    const uint32_t *pf_sp;
    const uint2 *pf_hp;
    row_ptrs(0, pf_sp, pf_hp);
    auto fetch = [&](int g, uint32_t &scv, uint2 &hv) {
      const int tl = g / nk;
      if (tl != pf_tl) { pf_tl = tl; row_ptrs(tl, pf_sp, pf_hp); }
      scv = __ldg(pf_sp + 2 * (g % nk));
      if (QT == 3) hv = __ldg(pf_hp + 2 * (g % nk));
    };
    uint32_t sc[4];
    uint2 hw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sc[j] = 0u;
      hw[j] = make_uint2(0u, 0u);
      if (j < total_g) fetch(j, sc[j], hw[j]);
    }
    bool ok = true;
    for (int g0 = 0; g0 < total_g && ok; g0 += 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = g0 + j;
        if (g >= total_g) break;
        const int s = g % kStagesB, sa = g % kStagesA;
        const uint32_t ph = (uint32_t)(g / kStagesB) & 1u;
        // codes landed; and the MMAs that last read this A stage (stage g - kStagesA) are complete
        // (both waits come before the arithmetic: the out-of-line slow path of a wait would
        // otherwise have to save the 32 dequantized registers around its call)
        if (!mbar_wait(full_b(s), ph)) { record_timeout(ctrl, 24); ok = false; break; }
        if (g >= kStagesA &&
            !mbar_wait(empty_b((g - kStagesA) % kStagesB), (uint32_t)((g - kStagesA) / kStagesB) & 1u)) {
          record_timeout(ctrl, 24);
          ok = false;
          break;
        }
        tc_fence_after();
        // this thread's 64 weights of the stage: 16 code bytes (32 for the 4-bit plane)
        const uint8_t *cp = gbase + (sR(s) - base) + crow * SL::kRowCodes + hh * (SL::kRowCodes / 2);
        const uint4 cw = *reinterpret_cast<const uint4 *>(cp);
        const __half2 d0 = __half2half2(__ushort_as_half((uint16_t)(sc[j] & 0xffffu)));
        const __half2 d1 = __half2half2(__ushort_as_half((uint16_t)(sc[j] >> 16)));
        uint32_t p[32];
        if (QT == 4) {  // eight 8-weight words, words 0-3 in block 0 and 4-7 in block 1
          const uint4 cw2 = *reinterpret_cast<const uint4 *>(cp + 16);
          dq4_word(cw.x, d0, p);
          dq4_word(cw.y, d0, p + 4);
          dq4_word(cw.z, d0, p + 8);
          dq4_word(cw.w, d0, p + 12);
          dq4_word(cw2.x, d1, p + 16);
          dq4_word(cw2.y, d1, p + 20);
          dq4_word(cw2.z, d1, p + 24);
          dq4_word(cw2.w, d1, p + 28);
        } else if (QT == 3) {
          dq3_word(cw.x, hw[j].x, 0, d0, p);
          dq3_word(cw.y, hw[j].x, 1, d0, p + 8);
          dq3_word(cw.z, hw[j].y, 0, d1, p + 16);
          dq3_word(cw.w, hw[j].y, 1, d1, p + 24);
        } else {
          dq2_word(cw.x, d0, p);
          dq2_word(cw.y, d0, p + 8);
          dq2_word(cw.z, d1, p + 16);
          dq2_word(cw.w, d1, p + 24);
        }
        const uint32_t ta = tmem + a_lane + a_col(sa) + 32u * hh;
        tmem_st16(ta, p);
        tmem_st16(ta + 16u, p + 16);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(full_a(sa));
        const int gp = g + 4;  // refill this ring slot
        if (gp < total_g) fetch(gp, sc[j], hw[j]);
      }
    }
  } else {
    // ------------------------------------------------ epilogue warps 10..13 (lane quadrants 2, 3, 0, 1)
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    bool ok = true;
    TileInfo cur = tile_at(0);
    for (int tl = 0; tl < n_my && ok; ++tl) {
      const TileInfo nxt = (tl + 1 < n_my) ? tile_at(tl + 1) : cur;
      const int b = tl & 1;
      const bool go = __all_sync(0xffffffffu, mbar_wait(acc_full(b), ((uint32_t)tl >> 1) & 1u));
      if (!go) {
        if (lane == 0) record_timeout(ctrl, 25);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + lane_base + (uint32_t)(b * 256);
      if (MODE == MODE_DN) {
        const int f = cur.mt * kBM + 32 * q + lane;
        uint16_t *op = args.out + (size_t)cur.row_base * args.ldo + f;
        for (int c0 = 0; c0 < cur.N; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + c0, v);
          tmem_ld_wait16(v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < cur.n_valid) op[(size_t)n * args.ldo] = __half_as_ushort(__float2half_rn(__uint_as_float(v[j])));
          }
        }
      } else {
        // A rows alternate gate / up of the same feature, so lanes 2i and 2i+1 hold the gate and
        // up accumulators of feature f: per 16 columns each lane sends its partner the 8 values
        // the partner needs (one shuffle each); the gate lane finishes columns 0-7, the up lane 8-15
        const int f = cur.mt * 64 + 16 * q + (lane >> 1);
        const bool up_lane = lane & 1;
        uint16_t *op = args.out + (size_t)cur.row_base * args.ldo + f;
        for (int c0 = 0; c0 < cur.N; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + c0, v);
          tmem_ld_wait16(v);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float mine_lo = __uint_as_float(v[j]), mine_hi = __uint_as_float(v[j + 8]);
            const float other = __shfl_xor_sync(0xffffffffu, up_lane ? mine_lo : mine_hi, 1);
            const float gv = up_lane ? other : mine_lo;  // gate value of column c0 + j (+8 on the up lane)
            const float uv = up_lane ? mine_hi : other;
            const int n = c0 + j + (up_lane ? 8 : 0);
            const float hv = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
            if (n < cur.n_valid) op[(size_t)n * args.ldo] = __half_as_ushort(__float2half_rn(hv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(b));
      cur = nxt;
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
// Entries (group, first row within the group) for every `slice`-row slice (192 for this kernel) of every
// non-empty group, ordered longest first: by the slice's row count rounded up to the MMA's N
// granule of 16, descending (full 192-row slices first, the smallest remainders last). The
// persistent GEMM deals entries round-robin, so every CTA starts on the heavy tiles and the light
// ones fill the end of the schedule: with a skewed router a few experts take >1000 rows and many
// take a handful, and the long tiles no longer land at the tail. Within a size class the order
// is whatever the shared-memory cursors give; it does not change any result (every tile writes
// its own output rows). Offsets that are not monotone or run past n_rows flag the error word and
// yield no tiles.
constexpr int kTileClasses = kBNMax / 16;  // N granules 1..12

__global__ void __launch_bounds__(1024) tile_list_kernel(const int32_t *__restrict__ off, int G, int n_rows,
                                                         int slice, int2 *__restrict__ tiles,
                                                         Ctrl *__restrict__ ctrl) {
  const int nclass = slice / 16;  // <= kTileClasses
  __shared__ int s_cnt[kTileClasses + 1], s_cur[kTileClasses + 1];
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = 0;
  if (tid <= nclass) s_cnt[tid] = 0;
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
  // size class of a slice with n rows (1..slice): ceil(n / 16), 1..nclass
  for (int g = tid; g < G; g += blockDim.x) {
    const int n = off[g + 1] - off[g];
    if (n >= slice) atomicAdd(&s_cnt[nclass], n / slice);
    if (n % slice) atomicAdd(&s_cnt[(n % slice + 15) / 16], 1);
  }
  __syncthreads();
  if (tid == 0) {  // classes in descending order: each class's first position
    int pos = 0;
    for (int c = nclass; c >= 1; --c) {
      s_cur[c] = pos;
      pos += s_cnt[c];
    }
    ctrl->n_tiles = pos;
  }
  __syncthreads();
  for (int g = tid; g < G; g += blockDim.x) {
    const int n = off[g + 1] - off[g];
    const int full = n / slice;
    if (full) {
      const int p = atomicAdd(&s_cur[nclass], full);
      for (int j = 0; j < full; ++j) tiles[p + j] = make_int2(g, j * slice);
    }
    if (n % slice) tiles[atomicAdd(&s_cur[(n % slice + 15) / 16], 1)] = make_int2(g, full * slice);
  }
}

// ---------------------------------------------------------------- host side
namespace {
}  // namespace

namespace {

bool make_code_map(CUtensorMap *map, const moe_qmat &m, int box_rows) {
  return encode_tensor_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, m.codes, (uint64_t)gemm_code_bytes(m.qtype, m.K),
                              (uint64_t)m.n_experts * m.rows, gemm_code_bytes(m.qtype, kBK), box_rows,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int MODE, int QT>
cudaError_t launch_v2q(const CUtensorMap &tb, const CUtensorMap &c0r, const CUtensorMap &c1r, const CUtensorMap &c0s,
                       const CUtensorMap &c1s, const GemmArgs &a, cudaStream_t s) {
  const int smem = SmemV2<QT>::kBytes + 1024;
  cudaError_t e = smem_limit_once(grouped_v2_kernel<MODE, QT>, smem);
  if (e != cudaSuccess) return e;
  {
    KTimer kt_(MODE == MODE_GU ? KID_GEMM_GATE_UP : KID_GEMM_DOWN, s);
    grouped_v2_kernel<MODE, QT><<<num_sms(), kThreadsV2, smem, s>>>(tb, c0r, c1r, c0s, c1s, a);
  }
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_v2(const CUtensorMap &tb, const CUtensorMap &c0r, const CUtensorMap &c1r, const CUtensorMap &c0s,
                      const CUtensorMap &c1s, const GemmArgs &a, int qt, cudaStream_t s) {
  if (qt == MOE_Q3) return launch_v2q<MODE, 3>(tb, c0r, c1r, c0s, c1s, a, s);
  if (qt == MOE_Q4) return launch_v2q<MODE, 4>(tb, c0r, c1r, c0s, c1s, a, s);
  return launch_v2q<MODE, 2>(tb, c0r, c1r, c0s, c1s, a, s);
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

cudaError_t launch_tile_list(const int32_t *offsets, int n_groups, int n_rows, int slice, int2 *tiles, Ctrl *ctrl,
                             cudaStream_t s) {
  if (slice < 16 || slice > kBNMax || slice % 16) return cudaErrorInvalidValue;
  {
    KTimer kt_(KID_TILE_LIST, s);
    tile_list_kernel<<<1, 1024, 0, s>>>(offsets, n_groups, n_rows, slice, tiles, ctrl);
  }
  return cudaGetLastError();
}

int gemm_shape_supported(int H, int I) { return (H % 128 == 0 && I % 128 == 0 && H >= 128 && I >= 128) ? 1 : 0; }

cudaError_t launch_grouped_ffn(const uint16_t *x_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                               const moe_expert_set &routed, const moe_expert_set *shared, uint16_t *h_perm,
                               uint16_t *out_perm, int2 *tiles, Ctrl *ctrl, cudaStream_t s) {
  const int G = E + (shared ? 1 : 0);
  const moe_expert_set &sh = shared ? *shared : routed;
  cudaError_t e = launch_tile_list(offsets, G, n_rows, kBNMax, tiles, ctrl, s);
  if (e != cudaSuccess) return e;

  CUtensorMap tx, th, cg, cu, cd, sg, su, sd;
  bool ok = encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x_perm, H, n_rows, kSubK, kBoxRows,
                                 CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tensor_map_2d(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h_perm, I, n_rows, kSubK, kBoxRows,
                                 CU_TENSOR_MAP_SWIZZLE_128B) &&
            make_code_map(&cg, routed.gate, 64) && make_code_map(&cu, routed.up, 64) &&
            make_code_map(&cd, routed.down, kBM) && make_code_map(&sg, sh.gate, 64) && make_code_map(&su, sh.up, 64) &&
            make_code_map(&sd, sh.down, kBM);
  if (!ok) return cudaErrorInvalidValue;

  GemmArgs a{};
  a.offsets = offsets;
  a.tiles = tiles;
  a.ctrl = ctrl;
  a.shared_group = shared ? E : -1;
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
  e = launch_v2<MODE_GU>(tx, cg, cu, sg, su, a, routed.gate.qtype, s);
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
  return launch_v2<MODE_DN>(th, cd, cd, sd, sd, a, routed.gate.qtype, s);
}

cudaError_t launch_grouped_down(const uint16_t *h_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                                const moe_expert_set &routed, const moe_expert_set *shared, uint16_t *out_perm,
                                int2 *tiles, Ctrl *ctrl, cudaStream_t s) {
  const int G = E + (shared ? 1 : 0);
  const moe_expert_set &sh = shared ? *shared : routed;
  cudaError_t e = launch_tile_list(offsets, G, n_rows, kBNMax, tiles, ctrl, s);
  if (e != cudaSuccess) return e;
  CUtensorMap th, cd, sd;
  if (!(encode_tensor_map_2d(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h_perm, I, n_rows, kSubK, kBoxRows,
                             CU_TENSOR_MAP_SWIZZLE_128B) &&
        make_code_map(&cd, routed.down, kBM) && make_code_map(&sd, sh.down, kBM)))
    return cudaErrorInvalidValue;
  GemmArgs a{};
  a.offsets = offsets;
  a.tiles = tiles;
  a.ctrl = ctrl;
  a.shared_group = shared ? E : -1;
  a.out = out_perm;
  a.ldo = H;
  a.K = I;
  a.M = H;
  a.scales[0][0] = routed.down.scales;
  a.scales[1][0] = sh.down.scales;
  a.hibits[0][0] = routed.down.hibits;
  a.hibits[1][0] = sh.down.hibits;
  return launch_v2<MODE_DN>(th, cd, cd, sd, sd, a, routed.gate.qtype, s);
}

}  // namespace moe
