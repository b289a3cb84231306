// Fused decode / MTP-verify layer (1-8 tokens): one cooperative kernel per MoE layer.
//
// A decode step is bound by reading weights ("Strata vs Llama.cpp vs vLLM", chapter "Why LLM
// inference is a systems problem"), and at 1-4 tokens a layer moves only ~15 MB: spread over 148
// SMs that is ~100 KB per SM, less than one SM's shared memory. So the kernel asks for all of it
// at once: as soon as the routing is known, the warps of every CTA issue bulk async copies
// (cp.async.bulk, a few contiguous runs of rows per fill, the bytes counted on one mbarrier per
// slot) of the CTA's whole share of gate/up rows and down rows into a ring of shared-memory slots,
// and then work from shared memory as the slots fill; a slot that is read out is refilled at once
// by the warp that freed it. HBM
// then sees the layer's expert bytes requested within a few hundred nanoseconds instead of as a
// chain of dependent round trips.
//
// One grid of one CTA per SM (16 warps) runs three phases with no grid barrier:
//   P1  router logits: four warps per expert split H (the fp32 router rows are requested before
//       the tokens are staged); each logit is published as one 64-bit word (an atomic exchange),
//       this launch's tag in the high half and the fp32 value in the low half.
//   P1b every CTA polls the E logit words of its tokens until each carries this launch's tag (tag
//       and value arrive in one write, so a word that shows the tag holds its value; the shared
//       expert's rows are prefetched into L2 meanwhile), then computes the same top-k (a threshold from each 32-expert chunk's largest logits,
//       then one warp sorts the few logits above it) and the distinct-expert unit list
//       (deterministic), so no second exchange is needed. The warps then issue this CTA's
//       copies: gate/up items (unit, 8 features: 8 gate + 8 up rows over all of H) dealt
//       round-robin over CTAs, then the down rows of the CTA's 16 output features for every unit.
//   P2  gate/up + SwiGLU: two groups of 8 warps take alternate items; in a group warp j runs
//       K step j (256 wide) on the tensor cores (mma.sync m16n8k16 with A rows 0-7 = gate and
//       8-15 = up rows of the same features, fp16 operands, fp32 accumulate); the partials are
//       summed in fixed order and h is published: at one or two tokens as tagged words (two fp16
//       values and this launch's tag per 64-bit word, by atomic exchange: no fence, no counter);
//       at more tokens, whose down phase reads several times more h, as plain fp16 followed by an
//       add on the unit's readiness counter (released two items at a time, behind one fence).
//   P3  down projection fused with the weighted combine: each CTA owns 16 output features, its
//       warps take whole units (16 down rows over all of I, the half steps' loads issued
//       together). A unit's warp waits only for that unit's h (its tagged words, or its counter;
//       no second grid barrier: early units' down work overlaps later units' gate/up), stages
//       it, and runs; partials are reduced in fixed order (no atomics).
// Each slot's fills are consumed in phase order: the ring has an even number of slots so the
// gate/up items sharing a slot fall to one group, a CTA barrier separates a CTA's P2 from its
// P3, and a down piece first waits until the piece one ring behind it is consumed. A parity wait
// can then never run two phases ahead of its slot's last completed fill, where it would take the
// older phase for its own.
// A launch's tag is its number + 1: every CTA keeps its own count of started launches in the
// exchange area and advances it once per launch, so all CTAs of a launch agree on it (launches
// do not overlap past griddepcontrol.wait), and a word written by an earlier launch never carries
// it. The readiness counters come in two sets used by alternate launches; a launch zeroes the set
// the next one will use. The logit and h polls, the readiness waits and every mbarrier wait are
// bounded in time and report MOE_ERR_TIMEOUT instead of hanging;
// before the CTA exits it waits for the last fill of every slot (bounded too), so no copy is still
// writing its shared memory.
#include "common.cuh"
#include "dequant.cuh"
#include "gemv.cuh"
#include "tc.cuh"
#include "topk.cuh"

#include <mutex>
#include <vector>

namespace moe {

namespace {

constexpr int kFWarps = 16;
constexpr int kFThreads = kFWarps * 32;
constexpr int kFSlots = kFusedMaxCols;      // h columns (token, expert) of a step staged for the down phase
constexpr int kFMaxUnits = kFSlots + 1;
constexpr int kPairsPerLane = kFSlots / 32; // (token, slot) pairs per lane of the unit-list warp
static_assert(kFMaxUnits <= kFusedMaxUnits, "readiness counters per unit");
constexpr int kFMaxRing = 16;               // shared-memory slots for weight copies
constexpr int kFMaxE = kFusedMaxE;          // experts the fused kernel takes
constexpr int kFSmemMax = 226 * 1024;       // dynamic shared memory (a little is left for static)
constexpr int kDnBatch = 4;                 // down half steps (K = 128 each) whose loads go out together

// named barriers (0 is __syncthreads): one per gate/up group
constexpr int kBarGroup0 = 1;

struct FusedArgs {
  const uint16_t *x;       // bf16 tokens, or NULL when r_norm is given
  const float *r_norm;     // fp32 residual stream: x = bf16(RMSNorm_eps(r)) is computed here
  float eps;
  int T, H, E, k, I, has_shared;
  const float *Wr;
  const float *bias;
  const float *next_Wr;  // the next layer's router rows (stack), prefetched into L2 during P3, or NULL
  moe_expert_set routed, shared;
  const float *residual;
  float *y;
  int32_t *idx;
  float *w;
  Ctrl *ctrl;       // control block; the exchange area (tagged logit and h words) follows it
  int ring;        // slots in the ring
  int slot_bytes;  // bytes per slot
  int gu_bytes;    // bytes of one gate/up item
  int dn_bytes;    // bytes of one unit's 16 down rows
  int dpu;         // units per down slot
};

// matrix pointers of one decode unit (gate, up, down), looked up once per unit
struct UnitMats {
  const uint8_t *codes[3];
  const uint16_t *scales[3];
  const uint8_t *hibits[3];
};

struct FusedLayout {
  size_t xraw, x16, hs, part, red, units, umats, sidx, sw, misc, slot, src, keys, ctop, cand, firstof, pcnt, bars, ring,
      total;
};

__host__ __device__ inline size_t fl_align(size_t v, size_t a = 16) { return (v + a - 1) & ~(a - 1); }

__host__ __device__ inline FusedLayout fused_layout(int T, int H, int E, int I, int hs_cols, int ring, int slot_bytes) {
  FusedLayout L{};
  size_t o = 0;
  auto take = [&](size_t b) { size_t r = o; o = fl_align(o + b); return r; };
  // Phase-local buffers share one region: the tokens, logit keys and top-k lists serve P0-P2
  // only, the staged h columns P3 only, and a CTA's P3 starts after its P2 is complete.
  L.xraw = take((size_t)T * H * 2);
  L.x16 = take((size_t)T * xs_stride(H) * 2);
  L.keys = take((size_t)T * E * 4);              // [token][expert] order-preserving logit keys
  L.ctop = take((size_t)T * 32 * 8);             // [token][32] chunk-top codes (threshold candidates)
  L.cand = take((size_t)T * 32 * 8 + 128);       // [token][32] codes above the threshold, [8] counts, [8] tau
  L.firstof = take((size_t)E * 4);                // expert -> first pair choosing it
  const size_t early_end = o;
  o = 0;
  L.hs = take((size_t)hs_cols * xs_stride(I) * 2);    // staged h columns (down phase)
  o = early_end > o ? early_end : o;
  L.part = take((size_t)2 * 2 * 8 * 16 * 8 * 4);  // [group][buffer][K step][16 rows][8 columns]
  L.red = take((size_t)kFWarps * 16 * 8 * 4);
  L.units = take((size_t)kFMaxUnits * sizeof(DecUnit));
  L.umats = take((size_t)kFMaxUnits * sizeof(UnitMats));
  L.sidx = take((size_t)kDecodeMaxT * kMaxK * 4);
  L.sw = take((size_t)kDecodeMaxT * kMaxK * 4);
  L.misc = take(16 * 4);
  L.slot = take((size_t)(kFMaxUnits + 1) * 4);
  L.src = take((size_t)kFSlots * 4);
  L.pcnt = take((size_t)(kFMaxUnits + 1) * 4);
  L.bars = take((size_t)kFMaxRing * 8);
  o = fl_align(o, 128);
  L.ring = o;
  o += (size_t)ring * slot_bytes;
  L.total = o;
  return L;
}

// Poll a logit word until it carries `tag` (the writer's single 64-bit exchange makes tag and value
// arrive together, so no fence is needed), giving up after limit_ns or when *abort is set. The
// first load goes out at once; only a miss starts the clock.
__device__ __forceinline__ bool poll_tagged(const unsigned long long *p, uint32_t tag, uint64_t limit_ns,
                                            const volatile int *abort, unsigned long long &v) {
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  if ((uint32_t)(v >> 32) == tag) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    __nanosleep(32);
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    if ((uint32_t)(v >> 32) == tag) return true;
    if ((abort && *abort) || global_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ FusedSync *fused_sync(Ctrl *c) {
  return reinterpret_cast<FusedSync *>(reinterpret_cast<char *>(c) + kCtrlStride);
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// prefetch [p, p + bytes) into L2, lines spread over `nthr` threads starting at thread `first`
__device__ __forceinline__ void prefetch_range(const void *p, size_t bytes, int first, int nthr) {
  const char *c = static_cast<const char *>(p);
  for (size_t off = (size_t)first * 128; off < bytes; off += (size_t)nthr * 128) prefetch_l2(c + off);
}

// an expert set's single (shared) expert into L2, lines spread over the grid's threads
template <int QT>
__device__ __forceinline__ void prefetch_shared(const moe_expert_set &sh, int I, int H, int first, int nthr) {
  const size_t cb = (size_t)I * code_row_bytes(QT, H), sb = (size_t)I * H / 32 * 2;
  prefetch_range(sh.gate.codes, cb, first, nthr);
  prefetch_range(sh.up.codes, cb, first, nthr);
  prefetch_range(sh.down.codes, cb, first, nthr);
  prefetch_range(sh.gate.scales, sb, first, nthr);
  prefetch_range(sh.up.scales, sb, first, nthr);
  prefetch_range(sh.down.scales, sb, first, nthr);
  if (QT == 3) {
    prefetch_range(sh.gate.hibits, cb / 2, first, nthr);
    prefetch_range(sh.up.hibits, cb / 2, first, nthr);
    prefetch_range(sh.down.hibits, cb / 2, first, nthr);
  }
}

// bulk copy global -> this CTA's shared memory, counted in bytes on `bar` (16-byte aligned
// addresses, a multiple of 16 bytes)
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One contiguous piece of a slot fill, as (source, offset in the slot, bytes). With CR the code
// bytes of one gate/up row (H/4; H/2 for the 4-bit plane) and CD those of one down row:
//   gate/up slot: [gate codes 8 x CR][up codes 8 x CR][gate scales 8 x H/32][up scales]
//                 [gate hi 8 x H/8][up hi]                     (Q2 5H bytes, Q3 7H, Q4 9H)
//   down slot:    dpu pieces of [codes 16 x CD][scales 16 x I/32][hi 16 x I/8]   (Q2 5I, Q3 7I, Q4 9I)
struct CopyDesc {
  const void *src;
  uint32_t off, bytes;
};

template <int QT>
__device__ __forceinline__ CopyDesc gu_copy(const FusedArgs &a, const UnitMats &um, int r0, int c) {
  const int H = a.H, CR = code_row_bytes(QT, H);
  const int which = c & 1;  // 0 gate, 1 up
  CopyDesc d;
  if (c < 2) {
    d.src = um.codes[which] + (size_t)r0 * CR;
    d.bytes = 8 * CR;
    d.off = which * 8 * CR;
  } else if (c < 4) {
    d.src = um.scales[which] + (size_t)r0 * (H / 32);
    d.bytes = H / 2;
    d.off = 16 * CR + which * (H / 2);
  } else {
    d.src = um.hibits[which] + (size_t)r0 * (H / 8);
    d.bytes = H;
    d.off = 16 * CR + H + which * H;
  }
  return d;
}

template <int QT>
__device__ __forceinline__ CopyDesc dn_copy(const FusedArgs &a, const UnitMats &um, int rb, int slot_unit, int c) {
  const int I = a.I, CD = code_row_bytes(QT, I);
  const size_t row = (size_t)rb * 16;
  const uint32_t base = (uint32_t)(slot_unit * a.dn_bytes);
  CopyDesc d;
  if (c == 0) {
    d.src = um.codes[2] + row * CD;
    d.bytes = 16 * CD;
    d.off = base;
  } else if (c == 1) {
    d.src = um.scales[2] + row * (I / 32);
    d.bytes = I;
    d.off = base + 16 * CD;
  } else {
    d.src = um.hibits[2] + row * (I / 8);
    d.bytes = 2 * I;
    d.off = base + 16 * CD + I;
  }
  return d;
}

// one lane's share of a 16-row x 256-wide K step read from a staged slot: the code rows of MMA
// rows g and g+8 start at ca / cb, their scales at sa / sb (halves), their hi bits at ha / hb
template <int QT>
__device__ __forceinline__ void frag_from_smem(StepFrag &f, const uint8_t *ca, const uint8_t *cb, const uint16_t *sa,
                                               const uint16_t *sb, const uint8_t *ha, const uint8_t *hb, int k0) {
  const int co = code_row_bytes(QT, k0);
  f.w0 = *reinterpret_cast<const uint4 *>(ca + co);
  f.w1 = *reinterpret_cast<const uint4 *>(cb + co);
  if (QT == 4) {
    f.w0b = *reinterpret_cast<const uint4 *>(ca + co + 16);
    f.w1b = *reinterpret_cast<const uint4 *>(cb + co + 16);
  }
  f.d0 = *reinterpret_cast<const uint32_t *>(sa + k0 / 32);
  f.d1 = *reinterpret_cast<const uint32_t *>(sb + k0 / 32);
  if (QT == 3) {
    f.h0 = *reinterpret_cast<const uint2 *>(ha + k0 / 8);
    f.h1 = *reinterpret_cast<const uint2 *>(hb + k0 / 8);
  }
}

}  // namespace

// TMAX: the largest token count the instance takes (1, 2, 4 or 8); the token loops of the router
// are unrolled to TMAX, so the common single-token instance carries no code for the others.
template <int QT, int TMAX>
__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(const FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int T = a.T, H = a.H, E = a.E, k = a.k, I = a.I;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int hs_cols = T * k + (a.has_shared ? T : 0);
  const FusedLayout L = fused_layout(T, H, E, I, hs_cols, a.ring, a.slot_bytes);
  uint16_t *xraw = reinterpret_cast<uint16_t *>(smem + L.xraw);
  __half *x16 = reinterpret_cast<__half *>(smem + L.x16);
  __half *hs = reinterpret_cast<__half *>(smem + L.hs);
  float *part = reinterpret_cast<float *>(smem + L.part);
  float *red = reinterpret_cast<float *>(smem + L.red);
  DecUnit *su = reinterpret_cast<DecUnit *>(smem + L.units);
  UnitMats *s_um = reinterpret_cast<UnitMats *>(smem + L.umats);
  int32_t *s_idx = reinterpret_cast<int32_t *>(smem + L.sidx);
  float *s_w = reinterpret_cast<float *>(smem + L.sw);
  int *misc = reinterpret_cast<int *>(smem + L.misc);
  int *s_slot = reinterpret_cast<int *>(smem + L.slot);
  int *s_src = reinterpret_cast<int *>(smem + L.src);
  uint32_t *s_key = reinterpret_cast<uint32_t *>(smem + L.keys);
  unsigned long long *s_ctop = reinterpret_cast<unsigned long long *>(smem + L.ctop);
  unsigned long long *s_cand = reinterpret_cast<unsigned long long *>(smem + L.cand);
  int *s_ccnt = reinterpret_cast<int *>(smem + L.cand + (size_t)T * 32 * 8);  // [token] candidates found
  unsigned long long *s_tau = reinterpret_cast<unsigned long long *>(s_ccnt + kDecodeMaxT);  // [token] threshold
  int *s_firstof = reinterpret_cast<int *>(smem + L.firstof);
  int *s_pcnt = reinterpret_cast<int *>(smem + L.pcnt);
  const uint32_t bar_full0 = smem_u32(smem + L.bars);
  const uint32_t ring0 = smem_u32(smem + L.ring);
  const uint8_t *ringp = smem + L.ring;
  const int R = a.ring, S = a.slot_bytes;
  auto full = [&](int s) { return bar_full0 + 8u * (uint32_t)s; };
  Ctrl *ctrl = a.ctrl;
  const int xs16 = xs_stride(H);
  const int G = gridDim.x;
  FusedSync *const fs = fused_sync(ctrl);
  __shared__ uint32_t s_tag;
  __shared__ volatile int s_abort;
  __shared__ int s_lastq[kFMaxRing];  // the last fill issued into each slot (-1: none)
  // ---------------- P0: this warp's router rows are requested first, then the tokens are staged
  const int H4 = H / 4, HQ = H4 / 4;  // float4 per quarter of a router row (<= 128: H <= 2048)
  const int es = warp >> 2, qh = warp & 3;
  float4 rv[4];
  auto load_router = [&](int e) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h4 = lane + 32 * u;
      rv[u] = (e < E && h4 < HQ) ? __ldcs(reinterpret_cast<const float4 *>(a.Wr + (size_t)e * H) + qh * HQ + h4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // The router rows are weights, which no kernel of this library writes; and a launch can start
  // before its predecessor has finished only behind a kernel that allowed it (this library's
  // kernels do, at their entry). So they are requested before the wait below, and their fetch
  // overlaps the previous layer's last CTAs.
  load_router((int)blockIdx.x + es * G);
  // The next launch on the stream (the next layer) may be scheduled now; its CTAs take SMs as this
  // grid's CTAs leave them. Nothing the previous launch writes (the control words, the workspace,
  // the tokens) is touched before it has completed.
  pdl_launch_dependents();
  pdl_wait();
  // This launch's tag: one more than the launches this CTA's slot has counted (each CTA reads and
  // advances only its own slot, and every launch advances every slot once, so all of a launch's
  // CTAs read the same count; launches do not overlap past the wait above). The tag marks this
  // launch's logit and h words. The load's result is first needed after the tokens are staged.
  uint32_t launch_no = 0;
  if (tid == 0) {
    launch_no = *reinterpret_cast<volatile const uint32_t *>(&fs->seq[blockIdx.x]);
    s_abort = 0;
    for (int s = 0; s < R; ++s) {
      mbar_init(full(s), 1);  // the filling lane's arrival, and the fill's bytes
      s_lastq[s] = -1;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // a bounded wait that gives up at once after an earlier wait of this CTA gave up
  auto wait_bar = [&](uint32_t bar, uint32_t parity, int where) -> bool {
    if (s_abort) return false;
    if (mbar_wait(bar, parity)) return true;
    s_abort = 1;
    set_device_error(ctrl, MOE_ERR_TIMEOUT, where);
    return false;
  };
  // parity of fill q's phase: one phase per fill q, q + R, ... of the slot
  auto fill_parity = [&](int q) { return (uint32_t)(q / R) & 1u; };
  bool ok = true;
  const float *const lbias = a.bias;
  const moe_expert_set &lRS = a.routed;
  const moe_expert_set &lSS = a.shared;
  const float *const lrn = a.r_norm;
  const float *const lres = a.residual;

  __shared__ float s_inv[kDecodeMaxT];
  // token staging in chunks of 8 values: at most 4 per thread (T <= 8, H <= 2048)
  constexpr int kChunks = 4;
  const int H8 = H / 8, nchunk = T * H8;
  float4 cf[2 * kChunks];
  if (lrn) {
    // the stream's rows are requested first, then the RMSNorm sums, whose loads overlap them
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
      const int i = tid + j * kFThreads;
      if (i < nchunk) {
        cf[2 * j] = __ldcg(reinterpret_cast<const float4 *>(lrn) + 2 * i);
        cf[2 * j + 1] = __ldcg(reinterpret_cast<const float4 *>(lrn) + 2 * i + 1);
      }
    }
    // RMSNorm of the residual stream (no gain): the same summation order and rounding as the
    // stand-alone RMSNorm kernel (256 threads: strided fmaf chains, warp butterflies, 8 warp
    // partials in order), so u is bit-identical to it
    __shared__ float s_part[kDecodeMaxT][8];
    if (tid < 256) {
      for (int t = 0; t < T; ++t) {
        const float *row = lrn + (size_t)t * H;
        float rr[8];  // the thread's H / 256 <= 8 values, all requested before the chain
#pragma unroll
        for (int j = 0; j < 8; ++j) rr[j] = (tid + 256 * j < H) ? __ldcg(row + tid + 256 * j) : 0.0f;
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (tid + 256 * j < H) ss = fmaf(rr[j], rr[j], ss);
        ss = warp_sum(ss);
        if (lane == 0) s_part[t][warp] = ss;
      }
    }
    __syncthreads();
    if (tid < T) {
      float tot = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) tot += s_part[tid][i];
      s_inv[tid] = 1.0f / sqrtf(tot / (float)H + a.eps);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    const int i = tid + j * kFThreads;
    if (i >= nchunk) break;
    uint4 v;
    if (lrn) {
      const int t = i / H8;
      const float4 f0 = cf[2 * j], f1 = cf[2 * j + 1];
      const float iv = s_inv[t];
      auto pk = [&](float lo, float hi) {
        const __nv_bfloat16 bl = __float2bfloat16_rn(lo * iv), bh = __float2bfloat16_rn(hi * iv);
        return (uint32_t)*reinterpret_cast<const uint16_t *>(&bl) |
               ((uint32_t)*reinterpret_cast<const uint16_t *>(&bh) << 16);
      };
      v = make_uint4(pk(f0.x, f0.y), pk(f0.z, f0.w), pk(f1.x, f1.y), pk(f1.z, f1.w));
    } else {
      v = __ldg(reinterpret_cast<const uint4 *>(a.x) + i);
    }
    reinterpret_cast<uint4 *>(xraw)[i] = v;
    const int t = i / H8, c = i % H8;
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __half2 h = __floats2half2_rn(__uint_as_float(in[q] << 16), __uint_as_float(in[q] & 0xffff0000u));
      o[q] = *reinterpret_cast<uint32_t *>(&h);
      if (f16x2_inf(o[q])) set_device_error(ctrl, MOE_ERR_RANGE, 4);
    }
    uint2 *d = reinterpret_cast<uint2 *>(x16 + (size_t)t * xs16 + xs_pos(8 * c));
    d[0] = make_uint2(o[0], o[1]);
    d[1] = make_uint2(o[2], o[3]);
  }
  if (lbias) prefetch_range(lbias, (size_t)E * 4, tid, kFThreads);
  if (tid == 0) {
    s_tag = launch_no + 1u;
    fs->seq[blockIdx.x] = launch_no + 1u;  // read by this CTA's slot in the next launch only
  }
  __syncthreads();
  const uint32_t tag = s_tag;
  // h exchange: tagged words at one or two tokens, plain rows + per-unit readiness counters above
  constexpr bool kTaggedH = TMAX <= 2;
  unsigned *const ready = fs->ready[tag & 1u];
  // the other set serves the next launch: the previous launch, its last user, has completed
  if (!kTaggedH && blockIdx.x == 0)
    for (int u = tid; u < kFusedMaxUnits; u += kFThreads) fs->ready[(tag & 1u) ^ 1u][u] = 0u;

  // ---------------- P1: router logits, four warps per expert (each a quarter of H), fp32
  {
    float *rp = red;  // [4 experts][4 quarters][T]
    for (int e0 = blockIdx.x, it = 0; e0 < E; e0 += 4 * G, ++it) {
      const int e = e0 + es * G;
      if (it > 0) load_router(e);
      float acc[TMAX];
#pragma unroll
      for (int t = 0; t < TMAX; ++t) acc[t] = 0.0f;
      if (e < E) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h4 = lane + 32 * u;
          if (h4 >= HQ) continue;
#pragma unroll
          for (int t = 0; t < TMAX; ++t) {
            if (t < T) {
              const uint2 xb = reinterpret_cast<const uint2 *>(xraw + (size_t)t * H)[qh * HQ + h4];
              acc[t] = fmaf(rv[u].x, __uint_as_float(xb.x << 16), acc[t]);
              acc[t] = fmaf(rv[u].y, __uint_as_float(xb.x & 0xffff0000u), acc[t]);
              acc[t] = fmaf(rv[u].z, __uint_as_float(xb.y << 16), acc[t]);
              acc[t] = fmaf(rv[u].w, __uint_as_float(xb.y & 0xffff0000u), acc[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t < T) {
          const float sum = warp_sum(acc[t]);
          if (lane == 0) rp[(es * 4 + qh) * kDecodeMaxT + t] = sum;
        }
      }
      __syncthreads();
      if (tid < 4 * T) {  // fixed-order sum of the four quarters
        const int ee = tid / T, t = tid % T, eg = e0 + ee * G;
        if (eg < E) {
          const float *q4 = rp + ee * 4 * kDecodeMaxT;
          const float lg = (q4[t] + q4[kDecodeMaxT + t]) + (q4[2 * kDecodeMaxT + t] + q4[3 * kDecodeMaxT + t]);
          // an atomic exchange rather than a relaxed store: it is performed at L2 at once, so the
          // word reaches the polling CTAs sooner (measured: all logits in ~0.9 us earlier)
          const unsigned long long word = ((unsigned long long)tag << 32) | __float_as_uint(lg);
          atomicExch(fs->logit + (size_t)t * E + eg, word);
        }
      }
      __syncthreads();
    }
  }

  // ---------------- P1b: top-k and unit list, computed identically by every CTA
  if (ok) {
    // Top-k by threshold. Codes are (order-preserving 32-bit key of logit + bias) << 32 | ~index,
    // so code order is the routing order (larger logit first, equal logits: lower index first)
    // and codes are unique. (1) For every token each 32-expert chunk gives its m = ceil(k / nch)
    // largest codes (warp max reductions); the k-th largest of these nch * m <= 31 chunk tops is a
    // threshold tau no larger than the token's k-th largest code, since k distinct codes reach it.
    // (2) The codes >= tau (at least k; with the router's logits ~15, never more than 32 in the
    // workloads' statistics) are gathered and one warp sorts them: its first k lanes are the
    // top-k. (3) If more than 32 codes reach tau (mass ties), the warp instead takes k rounds of
    // arg-max over all E codes of the token.
    const int nch = (E + 31) / 32;       // <= 16
    const int m = (k + nch - 1) / nch;   // chunk tops per chunk: nch * m <= nch + k - 1 <= 31
#pragma unroll 1
    for (int task = warp; task < T * nch; task += kFWarps) {
      const int t = task / nch, c = task % nch, e = c * 32 + lane;
      uint32_t key = 0u;
      if (e < E) {  // the logit word of this launch (bounded wait for its writer)
        unsigned long long v;
        if (!poll_tagged(fs->logit + (size_t)t * E + e, tag, kWaitLimitNs, &s_abort, v) && !s_abort) {
          s_abort = 1;
          set_device_error(ctrl, MOE_ERR_TIMEOUT, 31);
        }
        key = logit_key(__uint_as_float((uint32_t)v) + (lbias ? __ldg(lbias + e) : 0.f));
        s_key[t * E + e] = key;
      }
      const uint32_t nidx = (e < E) ? 0xFFFFFFFFu - (uint32_t)e : 0u;
      uint32_t live = key;
#pragma unroll 1
      for (int r = 0; r < m; ++r) {  // the chunk's r-th largest code
        const uint32_t mk = __reduce_max_sync(0xffffffffu, live);
        const uint32_t lo = __reduce_max_sync(0xffffffffu, (live == mk) ? nidx : 0u);
        if (lane == 0) s_ctop[t * 32 + c * m + r] = ((unsigned long long)mk << 32) | lo;
        if (live == mk && nidx == lo) live = 0u;
      }
    }
    {  // into L2 while the top-k runs: the shared expert's rows (always selected)
      const int nthr = gridDim.x * kFThreads, first = blockIdx.x * kFThreads + tid;
      if (a.has_shared) prefetch_shared<QT>(lSS, I, H, first, nthr);
    }
    if (T > 1)
      for (int e = tid; e < E; e += kFThreads) s_firstof[e] = 0x7fffffff;
    __syncthreads();
    ok = ok && !s_abort;  // a logit that never arrived: no routing, no expert work
    if (warp < T) {  // the threshold: the k-th largest chunk top (0 when fewer than k are nonzero)
      if (lane == 0) {
        s_tau[warp] = 0ull;
        s_ccnt[warp] = 0;
      }
      __syncwarp();
      const int cnt = nch * m;
      if (lane < cnt) {
        const unsigned long long v = s_ctop[warp * 32 + lane];
        if (v != 0ull && rank_desc32(s_ctop + warp * 32, cnt, v) == k - 1) s_tau[warp] = v;
      }
    }
    __syncthreads();
#pragma unroll 1
    for (int task = warp; task < T * nch; task += kFWarps) {  // gather the codes >= tau
      const int t = task / nch, e = (task % nch) * 32 + lane;
      const unsigned long long code =
          (e < E) ? ((unsigned long long)s_key[t * E + e] << 32) | (0xFFFFFFFFu - (uint32_t)e) : 0ull;
      const bool in = (e < E) && code >= s_tau[t];
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      int base = 0;
      if (lane == 0 && bal) base = atomicAdd(&s_ccnt[t], __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      const int pos = base + __popc(bal & ((1u << lane) - 1u));
      if (in && pos < 32) s_cand[t * 32 + pos] = code;
    }
    __syncthreads();
    if (warp < T) {
      const int t = warp, n = s_ccnt[t];
      unsigned long long *sel = s_ctop + t * 32;  // reused: the selected codes in slot order
      if (n <= 32) {  // rank the candidates: slot r of sel gets the r-th largest
        // lane r's code goes to slot rank(code): the candidates are distinct, nonzero codes
        if (lane < n) {
          const unsigned long long v = s_cand[t * 32 + lane];
          const int r = rank_desc32(s_cand + t * 32, n, v);
          if (r < k) sel[r] = v;
        }
      } else {  // mass ties: k rounds of arg-max over the token's E codes
        uint32_t taken = 0u;  // bit i: expert lane + 32 i already selected
#pragma unroll 1
        for (int j = 0; j < k; ++j) {
          unsigned long long best = 0ull;
          int bi = -1;
#pragma unroll 1
          for (int i = 0; i < nch; ++i) {
            const int e = lane + 32 * i;
            if (e >= E || ((taken >> i) & 1u)) continue;
            const unsigned long long code = ((unsigned long long)s_key[t * E + e] << 32) | (0xFFFFFFFFu - (uint32_t)e);
            if (code > best) {
              best = code;
              bi = i;
            }
          }
          const uint32_t mk = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
          const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == mk ? (uint32_t)best : 0u);
          if (bi >= 0 && (uint32_t)(best >> 32) == mk && (uint32_t)best == lo) taken |= 1u << bi;
          if (lane == 0) sel[j] = ((unsigned long long)mk << 32) | lo;
        }
      }
      __syncwarp();
      const unsigned long long v = lane < k ? sel[lane] : 0ull;
      topk_finish(key_to_logit((uint32_t)(v >> 32)), (int)(0xFFFFFFFFu - (uint32_t)v), k, s_idx + t * k,
                  s_w + t * k);
    }
    __syncthreads();
    const int P = T * k;
    if (TMAX == 1) {
      // one token: its k experts are k distinct units in slot order, then the shared expert;
      // column slot u holds unit u's only column. Records, plane pointers and the routing
      // copy in one parallel step.
      const int nuu = k + (a.has_shared ? 1 : 0);
      if (tid < 3 * nuu) {
        const int u = tid / 3, which = tid % 3;
        const bool shu = u == k;
        const MatView mv = mat_sel(lRS, lSS, shu ? 1 : 0, which, shu ? 0 : s_idx[u]);
        s_um[u].codes[which] = mv.codes;
        s_um[u].scales[which] = mv.scales;
        s_um[u].hibits[which] = mv.hibits;
        if (which == 0) {
          DecUnit &d = su[u];
          d.expert = shu ? 0 : s_idx[u];
          d.set = shu ? 1 : 0;
          d.mask = 1;
          d.xrow0 = 0;
          d.w[0] = shu ? 1.0f : s_w[u];
#pragma unroll
          for (int cc = 1; cc < 8; ++cc) d.w[cc] = 0.0f;
          s_slot[u] = u;
          s_src[u] = u * 8;
        }
      }
      if (tid == 0) {
        misc[0] = nuu;
        s_slot[nuu] = nuu;
      }
      if (blockIdx.x == 0 && tid < k) {
        a.idx[tid] = s_idx[tid];
        a.w[tid] = s_w[tid];
      }
      __syncthreads();
    } else {
    if (T > 1) {  // expert -> first pair choosing it
      for (int p = tid; p < P; p += kFThreads) atomicMin(&s_firstof[s_idx[p]], p);
      __syncthreads();
    }
    if (warp == 0) {
      // units: the distinct experts of the P = T*k (<= kFSlots) selections in order of first
      // appearance (token-major), then the shared expert. Pair p leads its unit when it is the
      // first pair to choose its expert (one token's k experts are distinct, so at T = 1 every
      // pair leads); a leader's unit number is the count of leaders before it.
      int fp[kPairsPerLane];
      bool lead[kPairsPerLane];
      unsigned bl[kPairsPerLane];
#pragma unroll
      for (int hh = 0; hh < kPairsPerLane; ++hh) {
        const int p = lane + 32 * hh;
        fp[hh] = (p < P) ? (T > 1 ? s_firstof[s_idx[p]] : p) : p;
        lead[hh] = (p < P) && fp[hh] == p;
        bl[hh] = __ballot_sync(0xffffffffu, lead[hh]);
      }
      int nr = 0;
#pragma unroll
      for (int hh = 0; hh < kPairsPerLane; ++hh) nr += __popc(bl[hh]);
      auto unit_of = [&](int q) {
        int n = 0;
#pragma unroll
        for (int hh = 0; hh < kPairsPerLane; ++hh) {
          const int lo = 32 * hh;
          if (q >= lo + 32) n += __popc(bl[hh]);
          else if (q > lo) n += __popc(bl[hh] & ((1u << (q - lo)) - 1u));
        }
        return n;
      };
#pragma unroll
      for (int hh = 0; hh < kPairsPerLane; ++hh) {
        const int p = lane + 32 * hh;
        if (lead[hh]) {
          DecUnit &d = su[unit_of(p)];
          d.expert = s_idx[p];
          d.set = 0;
          d.mask = 0;
          d.xrow0 = 0;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) d.w[cc] = 0.0f;
        }
      }
      if (a.has_shared && lane == 0) {
        DecUnit &d = su[nr];
        d.expert = 0;
        d.set = 1;
        d.mask = (1 << T) - 1;
        d.xrow0 = 0;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) d.w[cc] = cc < T ? 1.0f : 0.0f;
      }
      __syncwarp();
      // every (unit, token) is one pair: an expert appears at most once per token
#pragma unroll
      for (int hh = 0; hh < kPairsPerLane; ++hh) {
        const int p = lane + 32 * hh;
        if (p < P) {
          DecUnit &d = su[unit_of(fp[hh])];
          atomicOr(&d.mask, 1 << (p / k));
          d.w[p / k] = s_w[p];
        }
      }
      __syncwarp();
      const int nu = nr + (a.has_shared ? 1 : 0);
      if (lane == 0) misc[0] = nu;
      // slot table of the down phase: present (unit, token) columns in unit order
      int used = 0;
      for (int base = 0; base < nu; base += 32) {
        const int u = base + lane;
        const int cnt = (u < nu) ? __popc(su[u].mask & 0xff) : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        if (u < nu) {
          int sl = used + incl - cnt;
          s_slot[u] = sl;
          const int m = su[u].mask & 0xff;
          for (int cc = 0; cc < 8; ++cc)
            if ((m >> cc) & 1) s_src[sl++] = u * 8 + cc;
        }
        used += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_slot[nu] = used;
    }
    if (blockIdx.x == 0)
      for (int i = tid; i < P; i += kFThreads) {
        a.idx[i] = s_idx[i];
        a.w[i] = s_w[i];
      }
    __syncthreads();
    // each unit's gate / up / down plane pointers, looked up once (the fills read them from here)
    for (int i = tid; i < 3 * misc[0]; i += kFThreads) {
      const int u = i / 3, which = i % 3;
      const MatView mv = mat_sel(lRS, lSS, su[u].set, which, su[u].expert);
      s_um[u].codes[which] = mv.codes;
      s_um[u].scales[which] = mv.scales;
      s_um[u].hibits[which] = mv.hibits;
    }
    __syncthreads();
    }  // T > 1
  }
  const int nu = ok ? misc[0] : 0;
  const int rbs8 = I / 8;                     // gate/up items per unit
  const int n_gu = nu * rbs8;
  const int n_mine = (n_gu > (int)blockIdx.x) ? (n_gu - (int)blockIdx.x + G - 1) / G : 0;
  const int n_rb = (H / 16 > (int)blockIdx.x) ? (H / 16 - (int)blockIdx.x + G - 1) / G : 0;  // down row blocks
  const int npieces = (nu + a.dpu - 1) / a.dpu;  // down slots per row block
  const int n_total = n_mine + n_rb * npieces;
  const int nsteps_gu = (H + kStepK - 1) / kStepK;  // <= 8
  const int nhalf_dn = (I + kStepK / 2 - 1) / (kStepK / 2);  // down items are half steps (128 wide)

  // ---------------- fills: fill q of this CTA (gate/up items, then down pieces) goes to slot
  // q % R; lane 0 of the calling warp posts the fill's byte count on the slot's barrier and issues
  // it as a few bulk copies (each a contiguous run of rows: codes, scales, hi bits), after a proxy
  // fence that orders the slot's earlier reads by the warps before the copies' writes. After a wait
  // of this CTA gave up, no fill goes out (its slot's previous fill may not have been waited on).
  auto issue_fill = [&](int q) {
    if (lane != 0 || s_abort) return;
    const int s = q % R;
    const uint32_t dst0 = ring0 + (uint32_t)(s * S);
    fence_async_smem();
    s_lastq[s] = q;
    if (q < n_mine) {
      const int i = (int)blockIdx.x + q * G;
      const UnitMats &um = s_um[i / rbs8];
      const int r0 = (i % rbs8) * 8;
      const int nc = QT == 3 ? 6 : 4;
      uint32_t tot = 0;
      for (int c = 0; c < nc; ++c) tot += gu_copy<QT>(a, um, r0, c).bytes;
      mbar_arrive_expect_tx(full(s), tot);
#pragma unroll 1
      for (int c = 0; c < nc; ++c) {
        const CopyDesc d = gu_copy<QT>(a, um, r0, c);
        bulk_g2s(dst0 + d.off, d.src, d.bytes, full(s));
      }
    } else {
      const int j = q - n_mine, rbl = j / npieces, dp = j % npieces;
      const int rb = (int)blockIdx.x + rbl * G;
      const int nun = min(a.dpu, nu - dp * a.dpu);
      const int per = QT == 3 ? 3 : 2;
      uint32_t tot = 0;
      for (int m = 0; m < nun; ++m)
        for (int c = 0; c < per; ++c) tot += dn_copy<QT>(a, s_um[dp * a.dpu + m], rb, m, c).bytes;
      mbar_arrive_expect_tx(full(s), tot);
      for (int m = 0; m < nun; ++m) {
        const UnitMats &um = s_um[dp * a.dpu + m];
#pragma unroll 1
        for (int c = 0; c < per; ++c) {
          const CopyDesc d = dn_copy<QT>(a, um, rb, m, c);
          bulk_g2s(dst0 + d.off, d.src, d.bytes, full(s));
        }
      }
    }
  };
  if (ok)
    for (int q = warp; q < min(n_total, R); q += kFWarps) issue_fill(q);

  // ---------------- P2: gate/up + SwiGLU; group grp takes this CTA's items grp, grp + 2, ...
  // The ring has an even number of slots, so the items that share a slot (q, q + R, ...) all
  // fall to one group, which takes them in order: a parity wait then never runs two phases
  // ahead of the slot's last completed fill (where it would mistake the older phase for its own).
  if (ok) {
    const int grp = warp >> 3, j8 = warp & 7, gtid = tid & 255;
    int buf = 0;
    int held = -1;  // counter path: a unit whose item's count waits for the group's next release
    for (int q = grp; q < n_mine; q += 2, buf ^= 1) {
      const int i = (int)blockIdx.x + q * G;
      const int u = i / rbs8, r0 = (i % rbs8) * 8;
      const DecUnit &un = su[u];
      const int s = q % R;
      const bool have = wait_bar(full(s), fill_parity(q), 42);
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
      const int k0 = j8 * kStepK + 64 * t4;
      if (have && j8 < nsteps_gu && k0 < H) {
        const uint8_t *sl = ringp + (size_t)s * S;
        const int CR = code_row_bytes(QT, H);
        const uint8_t *ca = sl + (size_t)g * CR, *cb = sl + 8 * CR + (size_t)g * CR;
        const uint16_t *sa = reinterpret_cast<const uint16_t *>(sl + 16 * CR) + (size_t)g * (H / 32);
        const uint16_t *sb = reinterpret_cast<const uint16_t *>(sl + 16 * CR + H / 2) + (size_t)g * (H / 32);
        const uint8_t *ha = sl + 16 * CR + H + (size_t)g * (H / 8), *hb = sl + 16 * CR + 2 * H + (size_t)g * (H / 8);
        StepFrag f;
        frag_from_smem<QT>(f, ca, cb, sa, sb, ha, hb, k0);
        mma_step<QT>(acc, acc2, f, x16 + (size_t)g * xs16, k0, (un.mask >> g) & 1);
      }
      float *pw = part + (((size_t)(grp * 2 + buf) * 8 + j8) * 16) * 8;
      pw[g * 8 + 2 * t4] = acc[0] + acc2[0];
      pw[g * 8 + 2 * t4 + 1] = acc[1] + acc2[1];
      pw[(g + 8) * 8 + 2 * t4] = acc[2] + acc2[2];
      pw[(g + 8) * 8 + 2 * t4 + 1] = acc[3] + acc2[3];
      named_sync(kBarGroup0 + grp, 256);
      // every warp of the group is done with the slot: its next fill goes out now
      if (j8 == 7 && q + R < n_total) issue_fill(q + R);
      if (gtid < 64) {  // one (feature, token) per thread (two whole warps); fixed-order sums of the 8 K steps
        const int row = gtid & 7, col = gtid >> 3;
        const bool present = (un.mask >> col) & 1;
        uint32_t hb = 0u;
        if (present) {
          const float *pb = part + ((size_t)(grp * 2 + buf) * 8 * 16) * 8;
          float gv = 0.f, uv = 0.f;
#pragma unroll
          for (int sl = 0; sl < 8; ++sl) {
            gv += pb[(sl * 16 + row) * 8 + col];
            uv += pb[(sl * 16 + 8 + row) * 8 + col];
          }
          const float hv = gv / (1.0f + expf(-gv)) * uv;
          hb = __half_as_ushort(__float2half_rn(hv));
          if (f16_inf((uint16_t)hb)) set_device_error(ctrl, MOE_ERR_RANGE, 5);
        }
        const int slot = s_slot[u] + __popc(un.mask & ((1u << col) - 1u));
        if constexpr (kTaggedH) {
          // features row and row + 1 of a column go out as one tagged word: the word carries its
          // own readiness, so neither a fence nor a counter is needed (an atomic exchange is
          // performed at L2 at once)
          const uint32_t hb1 = __shfl_down_sync(0xffffffffu, hb, 1);
          if (present && (row & 1) == 0) {
            const unsigned long long word = ((unsigned long long)tag << 32) | (hb1 << 16) | hb;
            atomicExch(fs->hword + (size_t)slot * (I / 2) + (r0 + row) / 2, word);
          }
        } else if (present) {
          fs->hval[(size_t)slot * I + r0 + row] = (uint16_t)hb;
        }
      }
      if constexpr (!kTaggedH) {
        // the item's h is written: count it for its unit. Releases go out for two items at a time
        // (one group barrier and one release fence, which orders both items' stores, then two
        // relaxed adds); an item's count is held back at most one item of its group.
        if (held < 0 && q + 2 < n_mine) {
          held = u;
        } else {
          named_sync(kBarGroup0 + grp, 256);
          if (gtid == 0) {
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            if (held >= 0) asm volatile("red.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(ready + held) : "memory");
            asm volatile("red.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(ready + u) : "memory");
          }
          held = -1;
        }
      }
    }
  }
  // This CTA's gate/up items are all consumed (the ring rule of P3 below needs it); no grid
  // barrier: each down unit waits for its own unit's h instead.
  __syncthreads();
  // in a stack, the next layer's router rows go to L2 now: HBM is otherwise idle in the down phase
  if (a.next_Wr) prefetch_range(a.next_Wr, (size_t)E * H * 4, (int)blockIdx.x * kFThreads + tid, G * kFThreads);
  // ---------------- P3: down projection + weighted combine (+ residual) for 16 output features per CTA.
  // Piece d of a row block shares its slot with piece d - R. Before waiting on piece d's fill a
  // warp waits until piece d - R is consumed (its last consumer then issues piece d's fill), so
  // the parity wait is at most one phase ahead; for d < R the slot's previous phase belongs to a
  // P2 item or to an earlier row block, consumed before this row block starts. Units are taken in
  // increasing order, so the lowest waiting piece can always proceed.
  if (ok) {
    const int xstride = xs_stride(I);
    const int dn = a.dn_bytes;
    for (int rbl = 0; rbl < n_rb; ++rbl) {
      const int r0 = ((int)blockIdx.x + rbl * G) * 16;
      const int qb = n_mine + rbl * npieces;
      for (int i = tid; i < npieces; i += kFThreads) s_pcnt[i] = 0;
      __syncthreads();
      float tot[4] = {0.f, 0.f, 0.f, 0.f};
      // one unit per warp item: its 16 down rows over all of K (the half steps' shared-memory
      // loads go out together, then the MMAs)
      for (int u = warp; u < nu; u += kFWarps) {
        const int d = u / a.dpu, qd = qb + d, s = qd % R;
        if (d >= R) {  // piece d - R, in the same slot, fully consumed first (bounded wait)
          const int need_n = min(a.dpu, nu - (d - R) * a.dpu);
          const uint64_t t0 = global_ns();
          while (!s_abort && *reinterpret_cast<volatile int *>(&s_pcnt[d - R]) < need_n) {
            if (global_ns() - t0 > kWaitLimitNs) {
              s_abort = 1;
              set_device_error(ctrl, MOE_ERR_TIMEOUT, 44);
            }
          }
          __syncwarp();
        }
        const DecUnit &un = su[u];
        if (rbl == 0) {
          if constexpr (kTaggedH) {
            // the unit's h columns (contiguous column slots c0..): a lane's sixteen words are
            // requested together and re-requested together (bounded) until every one carries this
            // launch's tag, then their values go to the staged columns; they stay for later row blocks
            const int I4 = I / 4, c0 = s_slot[u], nv = (s_slot[u + 1] - c0) * I4;
            const unsigned long long *hw = fs->hword + (size_t)c0 * (I / 2);
            for (int v0 = lane; v0 < nv; v0 += 8 * 32) {
              unsigned long long hv[8][2];
              auto load_missing = [&](bool first) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const int vi = v0 + 32 * j;
                  if (vi < nv && (first || (uint32_t)(hv[j][0] >> 32) != tag || (uint32_t)(hv[j][1] >> 32) != tag))
                    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];"
                                 : "=l"(hv[j][0]), "=l"(hv[j][1])
                                 : "l"(hw + 2 * (size_t)vi)
                                 : "memory");
                }
              };
              auto all_tagged = [&]() {
                bool ok_all = true;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  if (v0 + 32 * j < nv)
                    ok_all = ok_all && (uint32_t)(hv[j][0] >> 32) == tag && (uint32_t)(hv[j][1] >> 32) == tag;
                return ok_all;
              };
              load_missing(true);
              if (!all_tagged()) {
                const uint64_t t0 = global_ns();
                for (;;) {
                  __nanosleep(32);
                  load_missing(false);
                  if (all_tagged() || s_abort) break;
                  if (global_ns() - t0 > kWaitLimitNs) {
                    s_abort = 1;
                    set_device_error(ctrl, MOE_ERR_TIMEOUT, 45);
                    break;
                  }
                }
              }
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int vi = v0 + 32 * j;
                if (vi < nv) {
                  uint2 *dd = reinterpret_cast<uint2 *>(hs + (size_t)(c0 + vi / I4) * xstride + xs_pos(4 * (vi % I4)));
                  *dd = make_uint2((uint32_t)hv[j][0], (uint32_t)hv[j][1]);
                }
              }
            }
            __syncwarp();
          } else {
            // the unit's h: wait until all its gate/up items are counted (bounded), then stage its
            // present columns (contiguous column slots c0.., 16-byte loads from L2)
            if (lane == 0) {
              const uint64_t t0 = global_ns();
              for (;;) {
                unsigned v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ready + u) : "memory");
                if (v >= (unsigned)rbs8 || s_abort) break;
                __nanosleep(32);
                if (global_ns() - t0 > kWaitLimitNs) {
                  s_abort = 1;
                  set_device_error(ctrl, MOE_ERR_TIMEOUT, 45);
                  break;
                }
              }
            }
            __syncwarp();
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ready + u) : "memory");
            (void)v;
            // all of a lane's loads (eight per round) go out before its stores: one L2 round trip
            const int I8 = I / 8, c0 = s_slot[u], nv = (s_slot[u + 1] - c0) * I8;
            const uint4 *hsrc = reinterpret_cast<const uint4 *>(fs->hval + (size_t)c0 * I);
            for (int v0 = lane; v0 < nv; v0 += 8 * 32) {
              uint4 hv[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int vi = v0 + 32 * j;
                hv[j] = vi < nv ? __ldcg(hsrc + vi) : make_uint4(0, 0, 0, 0);
              }
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int vi = v0 + 32 * j;
                if (vi < nv) {
                  uint2 *dd = reinterpret_cast<uint2 *>(hs + (size_t)(c0 + vi / I8) * xstride + xs_pos(8 * (vi % I8)));
                  dd[0] = make_uint2(hv[j].x, hv[j].y);
                  dd[1] = make_uint2(hv[j].z, hv[j].w);
                }
              }
            }
            __syncwarp();
          }
        }
        const bool have = wait_bar(full(s), fill_parity(qd), 43);
        const bool colok = (un.mask >> g) & 1;
        const int slot = s_slot[u] + __popc(un.mask & ((1u << g) - 1u));
        const __half *xcol = hs + (size_t)(colok ? slot : 0) * xstride;
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
        if (have) {
          const uint8_t *pc = ringp + (size_t)s * S + (size_t)(u % a.dpu) * dn;
          const int CD = code_row_bytes(QT, I);
          const uint8_t *ca = pc + (size_t)g * CD, *cb = pc + (size_t)(g + 8) * CD;
          const uint16_t *sa = reinterpret_cast<const uint16_t *>(pc + 16 * CD) + (size_t)g * (I / 32);
          const uint16_t *sb = reinterpret_cast<const uint16_t *>(pc + 16 * CD) + (size_t)(g + 8) * (I / 32);
          const uint8_t *ha = pc + 16 * CD + I + (size_t)g * (I / 8), *hb = pc + 16 * CD + I + (size_t)(g + 8) * (I / 8);
          for (int h0 = 0; h0 < nhalf_dn; h0 += kDnBatch) {
            HalfFrag f[kDnBatch];
#pragma unroll
            for (int b = 0; b < kDnBatch; ++b) {
              const int k0 = (h0 + b) * (kStepK / 2) + 32 * t4;
              if (k0 < I) {
                if (QT == 4) {  // one 16-byte block per row
                  const uint4 c0 = *reinterpret_cast<const uint4 *>(ca + k0 / 2);
                  const uint4 c1 = *reinterpret_cast<const uint4 *>(cb + k0 / 2);
                  f[b].w0 = make_uint2(c0.x, c0.y);
                  f[b].w0b = make_uint2(c0.z, c0.w);
                  f[b].w1 = make_uint2(c1.x, c1.y);
                  f[b].w1b = make_uint2(c1.z, c1.w);
                } else {
                  f[b].w0 = *reinterpret_cast<const uint2 *>(ca + k0 / 4);
                  f[b].w1 = *reinterpret_cast<const uint2 *>(cb + k0 / 4);
                }
                f[b].d0 = sa[k0 / 32];
                f[b].d1 = sb[k0 / 32];
                if (QT == 3) {
                  f[b].h0 = *reinterpret_cast<const uint32_t *>(ha + k0 / 8);
                  f[b].h1 = *reinterpret_cast<const uint32_t *>(hb + k0 / 8);
                }
              }
            }
#pragma unroll
            for (int b = 0; b < kDnBatch; ++b) {
              const int k0 = (h0 + b) * (kStepK / 2) + 32 * t4;
              if (k0 < I) mma_half_step<QT>(acc, acc2, f[b], xcol, k0, colok);
            }
          }
        }
        const float wa = un.w[2 * t4], wb = un.w[2 * t4 + 1];
        tot[0] = fmaf(wa, acc[0] + acc2[0], tot[0]);
        tot[1] = fmaf(wb, acc[1] + acc2[1], tot[1]);
        tot[2] = fmaf(wa, acc[2] + acc2[2], tot[2]);
        tot[3] = fmaf(wb, acc[3] + acc2[3], tot[3]);
        // the warp that finishes a piece's last unit refills its slot at once
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          const int nun = min(a.dpu, nu - d * a.dpu);
          __threadfence_block();
          last = (atomicAdd(&s_pcnt[d], 1) == nun - 1) ? 1 : 0;
          __threadfence_block();
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last && qd + R < n_total) issue_fill(qd + R);
      }
      float *rw = red + warp * 16 * 8;
      rw[g * 8 + 2 * t4] = tot[0];
      rw[g * 8 + 2 * t4 + 1] = tot[1];
      rw[(g + 8) * 8 + 2 * t4] = tot[2];
      rw[(g + 8) * 8 + 2 * t4 + 1] = tot[3];
      __syncthreads();
      for (int i = tid; i < 16 * T; i += kFThreads) {
        const int row = i % 16, col = i / 16;
        float sum = lres ? lres[(size_t)col * H + r0 + row] : 0.0f;
#pragma unroll
        for (int wi = 0; wi < kFWarps; ++wi) sum += red[(wi * 16 + row) * 8 + col];
        a.y[(size_t)col * H + r0 + row] = sum;
      }
      __syncthreads();
    }
  }


  // ---------------- no copy may still be writing this CTA's shared memory when it exits: the
  // last fill of each slot has landed (an earlier one was waited on before its slot was refilled)
  __syncthreads();
  if (tid < R && s_lastq[tid] >= 0 && !mbar_wait(full(tid), fill_parity(s_lastq[tid])))
    set_device_error(ctrl, MOE_ERR_TIMEOUT, 47);
}

// Test hook of the failure path: one warp waits, with the fused kernel's logit-exchange wait, for
// a tag that no launch writes (launch tags count up from 1 and would reach this one only after
// 2^32 - 1 launches). Each lane's wait gives up after limit_ns and MOE_ERR_TIMEOUT is recorded;
// nothing is written but the error word, nothing traps and the context stays usable.
__global__ void wait_starve_kernel(Ctrl *ctrl, uint64_t limit_ns) {
  unsigned long long v;
  if (!poll_tagged(fused_sync(ctrl)->logit + threadIdx.x, 0xFFFFFFFFu, limit_ns, nullptr, v))
    set_device_error(ctrl, MOE_ERR_TIMEOUT, 39);
}

cudaError_t launch_wait_starve(Ctrl *ctrl, uint64_t limit_ns, cudaStream_t s) {
  wait_starve_kernel<<<1, 32, 0, s>>>(ctrl, limit_ns);
  return cudaGetLastError();
}

// Shapes, ring and shared-memory plan of a fused launch; false when the shape or the device cannot
// take the kernel.
static bool fused_plan(int T, int H, int E, int k, int I, const moe_expert_set &routed, bool has_shared,
                       FusedArgs &a, const void *&fn, size_t &smem) {
  const int hs_cols = T * k + (has_shared ? T : 0);
  if (T < 1 || T > kDecodeMaxT || E > kFMaxE || H > 2048 || I > 1024 || hs_cols > kFSlots || k > 16 ||
      num_sms() > kFusedMaxGrid)
    return false;
  const int qt = routed.gate.qtype;
  const int per = qt == MOE_Q3 ? 7 : qt == MOE_Q4 ? 9 : 5;  // bytes per 16 weights: codes, scales (, hi bits)
  const int gu_bytes = per * H;  // 8 gate + 8 up rows
  const int dn_bytes = per * I;  // 16 down rows
  const int slot_bytes = (int)fl_align((size_t)(gu_bytes > dn_bytes ? gu_bytes : dn_bytes), 128);
  const int dpu = slot_bytes / dn_bytes;
  const FusedLayout L0 = fused_layout(T, H, E, I, hs_cols, 0, slot_bytes);
  if (L0.total >= (size_t)kFSmemMax) return false;
  int ring = (int)(((size_t)kFSmemMax - L0.total) / slot_bytes);
  if (ring > kFMaxRing) ring = kFMaxRing;
  {  // no more slots than one CTA can fill: its gate/up items plus its down pieces at the most units
    const int G = num_sms(), max_units = T * k + (has_shared ? 1 : 0);
    const int need = (max_units * (I / 8) + G - 1) / G + ((H / 16 + G - 1) / G) * ((max_units + dpu - 1) / dpu);
    if (ring > need) ring = need;
  }
  ring &= ~1;  // even: the slots' items fall to one gate/up group each (see the kernel's P2)
  if (ring < 2) return false;
  const FusedLayout L = fused_layout(T, H, E, I, hs_cols, ring, slot_bytes);
  const int tmax = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8;
#define MOE_FUSED_FN(K, Q, TM) reinterpret_cast<const void *>(K<Q, TM>)
#define MOE_FUSED_T(K, Q) (tmax == 1 ? MOE_FUSED_FN(K, Q, 1) : tmax == 2 ? MOE_FUSED_FN(K, Q, 2) \
                           : tmax == 4 ? MOE_FUSED_FN(K, Q, 4) : MOE_FUSED_FN(K, Q, 8))
  fn = qt == MOE_Q3 ? MOE_FUSED_T(decode_fused_kernel, 3)
       : qt == MOE_Q4 ? MOE_FUSED_T(decode_fused_kernel, 4) : MOE_FUSED_T(decode_fused_kernel, 2);
#undef MOE_FUSED_T
#undef MOE_FUSED_FN
  if (smem_limit_once_impl(fn, kFSmemMax) != cudaSuccess) return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kFThreads, L.total) != cudaSuccess || per_sm < 1)
    return false;
  a = FusedArgs{};
  a.T = T;
  a.H = H;
  a.E = E;
  a.k = k;
  a.I = I;
  a.has_shared = has_shared ? 1 : 0;
  a.ring = ring;
  a.slot_bytes = slot_bytes;
  a.gu_bytes = gu_bytes;
  a.dn_bytes = dn_bytes;
  a.dpu = dpu;
  smem = L.total;
  return true;
}

// fused_plan, kept per (device, shape): the plan queries the occupancy calculator and raises the
// kernel's shared-memory limit, host work a decode step should not repeat
static bool fused_plan_cached(int T, int H, int E, int k, int I, const moe_expert_set &routed, bool has_shared,
                              FusedArgs &a, const void *&fn, size_t &smem) {
  struct Plan {
    int dev, T, H, E, k, I, qt, sh;
    bool ok;
    FusedArgs a;
    const void *fn;
    size_t smem;
  };
  static std::mutex mu;
  static std::vector<Plan> plans;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const int qt = routed.gate.qtype, sh = has_shared ? 1 : 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const Plan &q : plans)
      if (q.dev == dev && q.T == T && q.H == H && q.E == E && q.k == k && q.I == I && q.qt == qt && q.sh == sh) {
        a = q.a;
        fn = q.fn;
        smem = q.smem;
        return q.ok;
      }
  }
  const bool ok = fused_plan(T, H, E, k, I, routed, has_shared, a, fn, smem);
  if (!ok) (void)cudaGetLastError();
  std::lock_guard<std::mutex> lk(mu);
  if (plans.size() < 4096) plans.push_back({dev, T, H, E, k, I, qt, sh, ok, a, fn, smem});
  return ok;
}

bool decode_fused_fits(int T, int H, int E, int k, int I, const moe_expert_set &routed, bool has_shared) {
  FusedArgs a;
  const void *fn = nullptr;
  size_t smem = 0;
  return fused_plan_cached(T, H, E, k, I, routed, has_shared, a, fn, smem);
}

static cudaError_t fused_launch(const void *fn, size_t smem, void **args, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  KTimer kt_(KID_DECODE_FUSED, s);
  if (pdl_enabled()) {  // may start while the previous kernel on the stream finishes
    cfg.numAttrs = 2;
    if (cudaLaunchKernelExC(&cfg, fn, args) == cudaSuccess) return cudaSuccess;
    (void)cudaGetLastError();  // the attribute pair was refused: launch without the overlap
  }
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t launch_decode_fused(const uint16_t *x, const float *r_norm, float eps, int T, int H, const float *Wr,
                                const float *bias, int E, int k, int I, const moe_expert_set &routed,
                                const moe_expert_set *shared, const float *residual, float *y, int32_t *idx,
                                float *w, Ctrl *ctrl, cudaStream_t s, const float *next_Wr) {
  FusedArgs a;
  const void *fn = nullptr;
  size_t smem = 0;
  if (!fused_plan_cached(T, H, E, k, I, routed, shared != nullptr, a, fn, smem)) return cudaErrorNotSupported;
  a.x = x;
  a.r_norm = r_norm;
  a.eps = eps;
  a.Wr = Wr;
  a.bias = bias;
  a.next_Wr = next_Wr;
  a.routed = routed;
  a.shared = shared ? *shared : routed;
  a.residual = residual;
  a.y = y;
  a.idx = idx;
  a.w = w;
  a.ctrl = ctrl;
  void *args[] = {&a};
  return fused_launch(fn, smem, args, s);
}

}  // namespace moe
