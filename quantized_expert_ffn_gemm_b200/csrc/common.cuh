// Internal declarations shared by the kernels and the C-ABI layer of libmoe_ffn.so.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_ffn.h"

namespace moe {

constexpr int kMaxK = 32;          // routing slots per token
constexpr int kMaxE = 4096;        // experts per layer
constexpr int kDecodeMaxT = 8;     // tokens the decode (GEMV) path takes at once (MMA N = 8)
constexpr int kPermChunk = 1024;   // (token, slot) pairs per permute chunk (one CTA / one warp)

// ---------------------------------------------------------------- control area (workspace head)
// Everything here is left at zero by the kernels that use it (tickets are reset by the last CTA).
struct Ctrl {
  int err;                  // MOE_OK / MOE_ERR_DEVICE_CHECK / MOE_ERR_TIMEOUT (first error wins)
  int err_info;             // diagnostic: the offending value
  unsigned router_ticket;   // last-CTA election in the decode router
  unsigned pad0;
  unsigned gemm_ticket[4];  // tile counters of the persistent grouped GEMM
  int n_units;              // decode: number of (expert, token-set) units built by the router
  int n_tiles;              // prefill: number of (group, row-tile) entries in the tile list
  unsigned long long pad_u64;
  int mid_pairs;            // mid-batch path: routed (token, slot) pairs with a valid expert
  int pad2;
  int pad1[18];
};
static_assert(sizeof(Ctrl) == 128, "control block is 128 bytes");

// The fused decode kernel's exchange area, the rest of the control area (zeroed once by
// moe_workspace_init and used by that kernel only). Router logits cross CTAs as 64-bit words
// (launch tag << 32 | fp32 bits) that readers poll until they carry their own launch's tag, so no
// fence or counter is needed. The gate/up output h of one- and two-token launches goes the same
// way (two fp16 values and the tag per word, one row of I / 2 words per (unit, token) column of
// the down phase); larger launches, whose down phase reads several times more h, store plain fp16
// rows and count each unit's items on a readiness counter (two sets used by alternate launches; a
// launch zeroes the set the next one uses). Each CTA also keeps its count of the launches it has
// started (every launch runs one CTA per SM, so the counts agree). Tags start at 1 on zeroed
// memory, so no word left from earlier use carries a live tag.
constexpr int kFusedMaxE = 512;     // experts the fused decode kernel takes
constexpr int kFusedMaxCols = 96;   // (unit, token) h columns of one launch
constexpr int kFusedMaxUnits = 128;
constexpr int kFusedMaxI = 1024;    // intermediate size the fused decode kernel takes
constexpr int kFusedMaxGrid = 256;  // CTAs of a fused launch (one per SM)
struct FusedSync {
  unsigned long long logit[kDecodeMaxT * kFusedMaxE];
  unsigned long long hword[kFusedMaxCols * (kFusedMaxI / 2)];  // tagged h (1-2 tokens)
  uint16_t hval[kFusedMaxCols * kFusedMaxI];                   // plain h (3-8 tokens)
  unsigned ready[2][kFusedMaxUnits];
  unsigned seq[kFusedMaxGrid];  // per CTA: launches it has started (all equal between launches)
};
constexpr size_t kCtrlStride = 256;  // the control block, then the exchange area
constexpr size_t kControlBytes = kCtrlStride + sizeof(FusedSync);

// A decode "unit": one expert applied to up to 8 activation rows (MMA columns).
//   rows xrow0 .. xrow0+7 of the activation source, column c present iff bit c of mask;
//   w[c]: routing weight of column c (combine mode); h is stored at h[(u*8 + c)*I ..].
struct DecUnit {
  int expert;
  int set;       // 0 routed, 1 shared
  int mask;
  int xrow0;
  float w[8];
};

// A mid-batch unit: one expert applied to up to kMidNT tokens (MMA column tiles of 8), partial rows
// row0 .. row0 + ncol - 1, whose tokens are listed in row_tok (so no permuted copy of the
// activations is needed).
struct MidUnit {
  int expert;
  int set;   // 0 routed, 1 shared
  int ncol;  // 1..kMidNT
  int row0;
  int pad[8];
};
static_assert(sizeof(MidUnit) == sizeof(DecUnit), "mid units share the decode units' workspace region");

constexpr int kMidFS = 128;   // features per mid-batch work item (one 128-wide half step of a down row)
constexpr int kMidMaxT = 128; // tokens the mid-batch path takes
constexpr int kMidMaxH = 4096;
// tokens per mid-batch unit: four MMA column tiles while they fit in shared memory
__host__ __device__ constexpr int mid_unit_tokens(int H) { return H <= 2048 ? 32 : 16; }

// ---------------------------------------------------------------- workspace layout
struct WsLayout {
  size_t ctrl, logits, idx, w, hist, units, hdec, counts, offsets, row_of, src, xperm, hperm, operm, u16, tiles, wsplit,
      dx, mid, xio, yio, total;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline WsLayout ws_layout(int H, int E, int k, int I, int has_shared, int T) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  size_t Tk = (size_t)T * k;
  size_t rows = Tk + (has_shared ? (size_t)T : 0);
  size_t nchunks = (Tk + kPermChunk - 1) / kPermChunk;
  // decode units (distinct experts of <= 8 tokens) or row-chunk units of the GEMV rows path
  size_t units = (size_t)kDecodeMaxT * k + 1;
  size_t row_units = (rows + 7) / 8 + (size_t)E + 2;
  if (row_units > units) units = row_units;
  L.ctrl = take(kControlBytes);  // control block + the fused decode kernel's exchange area
  L.logits = take((size_t)T * E * 4);
  L.idx = take(Tk * 4);
  L.w = take(Tk * 4);
  L.hist = take((nchunks + 1) * (size_t)E * 4);
  L.units = take(units * sizeof(DecUnit));
  L.hdec = take(units * 8 * (size_t)I * 2);
  L.counts = take((size_t)(E + 2) * 4);
  L.offsets = take((size_t)(E + 2) * 4);
  L.row_of = take(Tk * 4);
  L.src = take(rows * 4);
  L.xperm = take(rows * (size_t)H * 2);
  L.hperm = take(rows * (size_t)I * 2);
  L.operm = take(rows * (size_t)H * 2);
  L.u16 = take((size_t)T * H * 2);
  L.tiles = take((rows / 16 + (size_t)E + 4) * 8);
  L.wsplit = take((size_t)E * 3 * H * 2);
  L.dx = take(rows * (size_t)(H / 32) * 4);  // int8-activation path: one scale per 32-value block
  {  // mid-batch path: fp32 partial outputs [I / kMidFS slices][rows][H], for up to kMidMaxT tokens
    const size_t tm = (size_t)(T < kMidMaxT ? T : kMidMaxT);
    L.mid = take(I % kMidFS == 0 ? (size_t)(I / kMidFS) * tm * (size_t)(k + has_shared) * H * 4 : 0);
  }
  L.xio = take((size_t)T * H * 2);  // host-buffer entry points: the tokens, and y or the residual stream
  L.yio = take((size_t)T * H * 4);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ void set_device_error(Ctrl *c, int code, int info) {
  if (atomicCAS(&c->err, 0, code) == 0) c->err_info = info;
}

// A value outside the fp16 range of the expert operands became +-inf on conversion (RNE: above
// 65504 by half an ulp). Callers collect this per thread and record MOE_ERR_RANGE once.
__device__ __forceinline__ bool f16_inf(uint16_t b) { return (b & 0x7fffu) == 0x7c00u; }
__device__ __forceinline__ bool f16x2_inf(uint32_t b) { return f16_inf((uint16_t)b) || f16_inf((uint16_t)(b >> 16)); }

// Programmatic dependent launch. A kernel launched with the programmatic stream-serialization
// attribute may be scheduled before the previous kernel on its stream has finished, once that
// kernel's CTAs have all executed pdl_launch_dependents (or exited). pdl_wait returns when the
// previous kernel has completed and its memory operations are visible, at once when the launch
// had no such predecessor; a kernel launched that way reads or writes nothing a predecessor may
// touch before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

bool pdl_enabled();

// launch a kernel that calls pdl_wait() before touching anything an earlier kernel on the stream
// writes, with programmatic stream serialization when enabled
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- kernel launchers (one per .cu)
// All return cudaSuccess or the launch error; none synchronises.
cudaError_t launch_router_decode(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k,
                                 int32_t *idx, float *w, float *logits, int build_units, int has_shared,
                                 DecUnit *units, Ctrl *ctrl, cudaStream_t s);
cudaError_t launch_router_prefill(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k,
                                  int32_t *idx, float *w, float *logits, uint16_t *wsplit, Ctrl *ctrl, cudaStream_t s);
// tensor-core router logits (fp32 weights split into three bf16 planes); logits include the bias
bool router_tc_supported(int H, int E);
cudaError_t launch_router_tc(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E,
                             uint16_t *wsplit, float *logits, Ctrl *ctrl, cudaStream_t s);
// 2-D TMA descriptor over a row-major [rows][inner] tensor
bool encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *ptr, uint64_t inner,
                          uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);
cudaError_t launch_permute(const int32_t *idx, int T, int k, int E, const uint16_t *x, int H, int with_shared,
                           int32_t *counts, int32_t *offsets, int32_t *row_of, int32_t *src, uint16_t *x_perm,
                           int32_t *hist, Ctrl *ctrl, cudaStream_t s);
// ctrl != NULL: a non-finite expert output records MOE_ERR_RANGE there
cudaError_t launch_combine(const uint16_t *out_perm, const int32_t *row_of, const float *w, int T, int k, int H,
                           const uint16_t *shared_out, const float *residual, float *y, cudaStream_t s,
                           Ctrl *ctrl = nullptr);
cudaError_t launch_rmsnorm(const float *r, int T, int H, float eps, uint16_t *u, cudaStream_t s);
cudaError_t launch_dequant_rows(const moe_qmat &m, int expert, int row0, int nrows, float *out_f32, uint16_t *out_f16,
                                cudaStream_t s);

// decode path: units are read from `units` (count in ctrl->n_units, at most max_units)
cudaError_t launch_decode_units_from_offsets(const int32_t *offsets, int n_groups, int has_shared_group, int n_rows,
                                             DecUnit *units, Ctrl *ctrl, cudaStream_t s);
cudaError_t launch_decode_gate_up(const void *x, int x_is_bf16, int H, int I, const moe_expert_set &routed,
                                  const moe_expert_set *shared, const DecUnit *units, int max_units, Ctrl *ctrl,
                                  uint16_t *hdec, cudaStream_t s);
// combine mode (y != NULL): y[t] = sum_u w_u[t] * down_u h_u[t] (+ residual); rows mode: out rows fp16
cudaError_t launch_decode_down(int H, int I, const moe_expert_set &routed, const moe_expert_set *shared,
                               const DecUnit *units, int max_units, Ctrl *ctrl, const uint16_t *hdec, float *y,
                               const float *residual, int T, uint16_t *out_rows, cudaStream_t s);

// fused decode layer (one cooperative kernel: router, top-k, gate/up, down + combine);
// returns cudaErrorNotSupported when the shape or the device cannot take it (callers fall back).
// With r_norm != NULL the tokens are x = bf16(RMSNorm_eps(r_norm)) (x unused), bit-identical to
// launch_rmsnorm followed by the layer. ctrl: the workspace's control area (control block and the
// exchange area behind it). next_Wr (optional): the router rows of the layer that follows in a
// stack, prefetched into L2 during the down phase.
cudaError_t launch_decode_fused(const uint16_t *x, const float *r_norm, float eps, int T, int H, const float *Wr,
                                const float *bias, int E, int k, int I, const moe_expert_set &routed,
                                const moe_expert_set *shared, const float *residual, float *y, int32_t *idx,
                                float *w, Ctrl *ctrl, cudaStream_t s, const float *next_Wr = nullptr);

// mid-batch path (about 6..128 tokens; I % kMidFS == 0): units of <= 8 tokens per selected expert
// built from the routing (no permutation), items (unit, kMidFS-feature slice) that run gate/up,
// SwiGLU and their slice of the down projection into fp32 partial rows, then a fixed-order combine
bool mid_shape_supported(int T, int H, int E, int I);
cudaError_t launch_mid_ffn(const uint16_t *x, int T, int H, int E, int k, int I, const int32_t *idx, const float *w,
                           const moe_expert_set &routed, const moe_expert_set *shared, const float *residual, float *y,
                           MidUnit *units, int32_t *row_of, int32_t *row_tok, float *part, Ctrl *ctrl, cudaStream_t s);

// copy `bytes` (a multiple of 16, both ends 16-byte aligned and device-addressable) with a kernel;
// early: the source is read before the wait for the previous kernel on the stream
cudaError_t launch_io_copy(const void *src, void *dst, size_t bytes, bool early, cudaStream_t s);

// whether launch_decode_fused takes this shape on the current device
bool decode_fused_fits(int T, int H, int E, int k, int I, const moe_expert_set &routed, bool has_shared);

// test hook: the fused kernel's logit exchange wait, for a tag no launch writes; it gives up after
// limit_ns with MOE_ERR_TIMEOUT in the control block
cudaError_t launch_wait_starve(Ctrl *ctrl, uint64_t limit_ns, cudaStream_t s);

// prefill path (tcgen05 grouped GEMM)
int gemm_shape_supported(int H, int I);
// tile list (group, first row) of slice-row slices (a multiple of 16, <= 192) of every group,
// longest slices first; count in ctrl->n_tiles
cudaError_t launch_tile_list(const int32_t *offsets, int n_groups, int n_rows, int slice, int2 *tiles, Ctrl *ctrl,
                             cudaStream_t s);
// int8-activation (MMQ-style) gate/up + SwiGLU on tcgen05 kind::i8, Q2 weights: x_perm is
// quantized per 32-value block into x_q [n_rows][H] int8 and dx [n_rows][H/32] fp32 (scratch),
// h_perm as the fp16 path writes it
int mmq_shape_supported(int H, int I, int qtype);
cudaError_t launch_mmq_gate_up(const uint16_t *x_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                               const moe_expert_set &routed, const moe_expert_set *shared, int8_t *x_q, float *dx,
                               uint16_t *h_perm, int2 *tiles, Ctrl *ctrl, cudaStream_t s);
// the down projection alone (grouped GEMM, second kernel of launch_grouped_ffn) over h_perm
cudaError_t launch_grouped_down(const uint16_t *h_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                                const moe_expert_set &routed, const moe_expert_set *shared, uint16_t *out_perm,
                                int2 *tiles, Ctrl *ctrl, cudaStream_t s);
cudaError_t launch_grouped_ffn(const uint16_t *x_perm, const int32_t *offsets, int n_rows, int E, int H, int I,
                               const moe_expert_set &routed, const moe_expert_set *shared, uint16_t *h_perm,
                               uint16_t *out_perm, int2 *tiles, Ctrl *ctrl, cudaStream_t s);

int num_sms();
// (pdl_enabled: programmatic dependent launches are on unless the environment sets MOE_PDL=0)

// shape rules every entry point applies: H and I multiples of 64 up to 16384, 1 <= E <= kMaxE,
// 1 <= k <= min(E, kMaxK); a layer outside them that is still well formed (H, I multiples of 32)
// gives MOE_ERR_UNSUPPORTED, anything else MOE_ERR_INVALID_ARG
bool layer_shape_ok(int H, int E, int k, int I);
moe_status layer_shape_status(int H, int E, int k, int I);

// Raise a kernel's dynamic shared memory limit once per process (kept out of later launches so
// that launches can be captured into CUDA graphs).
cudaError_t smem_limit_once_impl(const void *func, size_t bytes);
template <class F>
cudaError_t smem_limit_once(F *func, size_t bytes) {
  return smem_limit_once_impl(reinterpret_cast<const void *>(func), bytes);
}

// ---------------------------------------------------------------- per-kernel timing (optional)
enum KernelId {
  KID_ROUTER_DECODE = 0, KID_ROUTER_GEMM, KID_TOPK, KID_PERM_HIST, KID_PERM_SCAN, KID_PERM_SCATTER, KID_PERM_GATHER,
  KID_COMBINE, KID_RMSNORM, KID_DEQUANT_ROWS, KID_DEC_UNITS, KID_DEC_GATE_UP, KID_DEC_DOWN, KID_TILE_LIST, KID_GEMM_GATE_UP, KID_GEMM_DOWN, KID_ROUTER_SPLIT, KID_ROUTER_TC, KID_DECODE_FUSED, KID_MMQ_QUANT,
  KID_MMQ_GATE_UP, KID_MID_PLAN, KID_MID_EXPERT, KID_MID_COMBINE, KID_COUNT
};
void timer_begin(int kid, cudaStream_t s);
void timer_end(int kid, cudaStream_t s);

// brackets one kernel launch with timing events when timing is enabled
struct KTimer {
  int kid;
  cudaStream_t s;
  KTimer(int k, cudaStream_t st) : kid(k), s(st) { timer_begin(kid, s); }
  ~KTimer() { timer_end(kid, s); }
};

}  // namespace moe
