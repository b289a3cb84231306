// C-ABI entry points of libmoe_ffn.so (declared in include/moe_ffn.h): argument validation on
// the host, workspace carving, path selection and kernel launches. No entry point allocates
// device memory, synchronises (except moe_read_device_error) or aborts.
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------- per-kernel timing records
namespace {
struct TimingRec {
  int kid;
  cudaEvent_t begin, end;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  cudaEvent_t e = nullptr;
  if (!g_pool.empty()) {
    e = g_pool.back();
    g_pool.pop_back();
  } else if (cudaEventCreate(&e) != cudaSuccess) {
    e = nullptr;
  }
  return e;
}
const char *const kKernelNames[KID_COUNT] = {
    "router_decode", "router_gemm", "topk", "perm_hist", "perm_scan", "perm_scatter", "perm_gather", "combine", "rmsnorm", "dequant_rows", "dec_units", "dec_gate_up", "dec_down",
    "tile_list", "gemm_gate_up", "gemm_down", "router_split", "router_tc", "decode_fused", "mmq_quant",
    "mmq_gate_up", "mid_plan", "mid_expert", "mid_combine"};
}  // namespace

void timer_begin(int kid, cudaStream_t s) {
  if (!g_timing) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  TimingRec r{kid, take_event(), take_event()};
  if (!r.begin || !r.end) return;
  cudaEventRecord(r.begin, s);
  g_recs.push_back(r);
}

void timer_end(int kid, cudaStream_t s) {
  if (!g_timing) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  if (!g_recs.empty() && g_recs.back().kid == kid) cudaEventRecord(g_recs.back().end, s);
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool pdl_enabled() {
  static const bool on = [] {
    const char *v = getenv("MOE_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

cudaError_t smem_limit_once_impl(const void *func, size_t bytes) {
  // record of the limits already set, keyed by (device, kernel host stub): the attribute belongs
  // to the current device's context, so every device a process uses gets its own raise
  struct Done {
    int dev;
    const void *func;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Done> done;
  if (bytes == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  for (auto &d : done)
    if (d.dev == dev && d.func == func && d.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done.push_back({dev, func, bytes});
  return e;
}

bool layer_shape_ok(int H, int E, int k, int I) {
  return H > 0 && H % 64 == 0 && H <= 16384 && E >= 1 && E <= kMaxE && k >= 1 && k <= kMaxK && k <= E && I > 0 &&
         I % 64 == 0 && I <= 16384;
}

// H or I a multiple of 32 but not of 64 (or beyond the sizes above) is a valid layer the library
// does not run
moe_status layer_shape_status(int H, int E, int k, int I) {
  if (layer_shape_ok(H, E, k, I)) return MOE_OK;
  if (H > 0 && H % 32 == 0 && I > 0 && I % 32 == 0 && E >= 1 && E <= kMaxE && k >= 1 && k <= kMaxK && k <= E)
    return MOE_ERR_UNSUPPORTED;
  return MOE_ERR_INVALID_ARG;
}

}  // namespace moe

using namespace moe;

namespace {

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

inline bool shape_ok(int H, int E, int k, int I) { return layer_shape_ok(H, E, k, I); }
inline moe_status shape_status(int H, int E, int k, int I) { return layer_shape_status(H, E, k, I); }

moe_status check_qmat(const moe_qmat &m, int n_experts, int rows, int K) {
  if (m.qtype != MOE_Q2 && m.qtype != MOE_Q3 && m.qtype != MOE_Q4) return MOE_ERR_INVALID_ARG;
  if (m.n_experts != n_experts || m.rows != rows || m.K != K) return MOE_ERR_INVALID_ARG;
  if (!m.codes || !m.scales) return MOE_ERR_INVALID_ARG;
  if ((m.qtype == MOE_Q3) != (m.hibits != nullptr)) return MOE_ERR_INVALID_ARG;  // hi bits exactly for Q3
  if (!aligned16(m.codes) || !aligned16(m.scales) || (m.hibits && !aligned16(m.hibits))) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

moe_status check_set(const moe_expert_set *s, int n, int H, int I) {
  if (!s) return MOE_ERR_INVALID_ARG;
  moe_status st;
  if ((st = check_qmat(s->gate, n, I, H)) != MOE_OK) return st;
  if ((st = check_qmat(s->up, n, I, H)) != MOE_OK) return st;
  if ((st = check_qmat(s->down, n, H, I)) != MOE_OK) return st;
  if (s->gate.qtype != s->up.qtype || s->gate.qtype != s->down.qtype) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

template <class T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

// Expert FFN over expert-contiguous rows by path: GEMM (every group on the grouped GEMM), GEMV
// (every group on the GEMV kernels), MMQ (int8 gate/up, fp16 down), AUTO: the grouped GEMM where
// it takes the shape. (Splitting AUTO by group size, small groups on the GEMV kernels, was
// measured: a GEMM tile costs about the same whatever its row count up to ~96 rows, but the GEMV
// kernels were slower still on the small groups of a skewed 2048-token layer, 0.53 against
// 0.39 ms, and at 12-128 tokens.)
cudaError_t expert_rows(const uint16_t *xperm, const int32_t *offsets, int rows, int E, int H, int I,
                        const moe_expert_set &routed, const moe_expert_set *sh, uint16_t *hperm, uint16_t *operm,
                        int2 *tiles, DecUnit *units, uint16_t *hdec, Ctrl *ctrl, cudaStream_t s, int path, bool gemm_ok,
                        int8_t *xq = nullptr, float *dx = nullptr) {
  const int n_groups = E + (sh ? 1 : 0);
  if (path == MOE_PATH_MMQ) {  // int8-activation gate/up, then the fp16 down GEMM
    cudaError_t e = launch_mmq_gate_up(xperm, offsets, rows, E, H, I, routed, sh, xq, dx, hperm, tiles, ctrl, s);
    if (e == cudaSuccess) e = launch_grouped_down(hperm, offsets, rows, E, H, I, routed, sh, operm, tiles, ctrl, s);
    return e;
  }
  if (path == MOE_PATH_AUTO && gemm_ok) path = MOE_PATH_GEMM;
  if (path == MOE_PATH_GEMM)
    return launch_grouped_ffn(xperm, offsets, rows, E, H, I, routed, sh, hperm, operm, tiles, ctrl, s);
  // a group of n rows makes ceil(n / 8) units: at most rows / 8 + (non-empty groups) in all
  const int max_units = (rows + 7) / 8 + (n_groups < rows ? n_groups : rows);
  cudaError_t e = launch_decode_units_from_offsets(offsets, n_groups, sh ? 1 : 0, rows, units, ctrl, s);
  if (e == cudaSuccess) e = launch_decode_gate_up(xperm, 0, H, I, routed, sh, units, max_units, ctrl, hdec, s);
  if (e == cudaSuccess)
    e = launch_decode_down(H, I, routed, sh, units, max_units, ctrl, hdec, nullptr, nullptr, 0, operm, s);
  return e;
}

// token counts for which AUTO takes the mid-batch path when the fused decode kernel does not take
// the shape (bench.py --crossover on the decode-shaped layer, calls replayed from a CUDA graph:
// 0.82x the grouped GEMM at 12 tokens, 0.93x at 16; the grouped GEMM is 4% faster from 24 tokens)
constexpr int kAutoMidLo = 8;
constexpr int kAutoMidHi = 20;

bool decode_router_fits(int T, int H, int E) {
  return T <= kDecodeMaxT && (size_t)T * (H > E ? H : E) * 4 <= 200 * 1024;
}

}  // namespace

extern "C" {

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_RANGE: return "MOE_ERR_RANGE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

size_t moe_workspace_bytes(const moe_layer_desc *d, int32_t T) {
  if (!d || T < 0 || !shape_ok(d->H, d->E, d->k, d->I)) return 0;
  return ws_layout(d->H, d->E, d->k, d->I, d->has_shared ? 1 : 0, T).total;
}

moe_status moe_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < sizeof(Ctrl)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  // the control block and the fused decode kernel's exchange area behind it (a smaller buffer
  // serves no layer call; its control block is still cleared)
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes < kControlBytes ? ws_bytes : kControlBytes,
                                     (cudaStream_t)stream));
}

moe_status moe_rmsnorm_bf16(const float *r, int32_t T, int32_t H, float eps, uint16_t *u, void *stream) {
  if (T < 0 || H <= 0 || H % 64 != 0 || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!r || !u) return MOE_ERR_INVALID_ARG;
  if (!aligned16(r) || !aligned16(u)) return MOE_ERR_ALIGNMENT;
  return cuda_status(launch_rmsnorm(r, T, H, eps, u, (cudaStream_t)stream));
}

moe_status moe_router_topk(const uint16_t *x, int32_t T, int32_t H, const float *Wr, const float *bias, int32_t E,
                           int32_t k, int32_t *idx, float *w, float *logits_opt, void *ws, size_t ws_bytes,
                           void *stream) {
  moe_status st = shape_status(H, E, k, 64);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !idx || !w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wr) || !aligned16(idx) || !aligned16(w) || (bias && !aligned16(bias)) ||
      (logits_opt && !aligned16(logits_opt)))
    return MOE_ERR_ALIGNMENT;
  if (!ws) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(H, E, k, 64, 0, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  Ctrl *ctrl = at<Ctrl>(ws, L.ctrl);
  float *logits = logits_opt ? logits_opt : at<float>(ws, L.logits);
  cudaStream_t s = (cudaStream_t)stream;
  if (decode_router_fits(T, H, E))
    return cuda_status(launch_router_decode(x, T, H, Wr, bias, E, k, idx, w, logits, 0, 0, at<DecUnit>(ws, L.units),
                                            ctrl, s));
  return cuda_status(
      launch_router_prefill(x, T, H, Wr, bias, E, k, idx, w, logits, at<uint16_t>(ws, L.wsplit), ctrl, s));
}

moe_status moe_permute(const int32_t *idx, int32_t T, int32_t k, int32_t E, const uint16_t *x, int32_t H,
                       int32_t with_shared, int32_t *counts, int32_t *offsets, int32_t *row_of, int32_t *src,
                       uint16_t *x_perm, void *ws, size_t ws_bytes, void *stream) {
  moe_status st = shape_status(H, E, k, 64);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!idx || !x || !counts || !offsets || !row_of || !src || !x_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(x) || !aligned16(x_perm) || !aligned16(counts) || !aligned16(offsets) ||
      !aligned16(row_of) || !aligned16(src))
    return MOE_ERR_ALIGNMENT;
  if (!ws) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(H, E, k, 64, with_shared ? 1 : 0, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  return cuda_status(launch_permute(idx, T, k, E, x, H, with_shared ? 1 : 0, counts, offsets, row_of, src, x_perm,
                                    at<int32_t>(ws, L.hist), at<Ctrl>(ws, L.ctrl), (cudaStream_t)stream));
}

moe_status moe_expert_ffn(const uint16_t *x_perm, const int32_t *offsets, int32_t n_rows, int32_t E, int32_t H,
                          int32_t I, const moe_expert_set *routed, const moe_expert_set *shared_opt,
                          uint16_t *out_perm, int32_t path, void *ws, size_t ws_bytes, void *stream) {
  moe_status st = shape_status(H, E, 1, I);
  if (st != MOE_OK) return st;
  if (n_rows < 0 || path < 0 || path > 4) return MOE_ERR_INVALID_ARG;
  if (path == MOE_PATH_MID) return MOE_ERR_UNSUPPORTED;  // the mid-batch path works from the routing
  if ((st = check_set(routed, E, H, I)) != MOE_OK) return st;
  if (shared_opt && (st = check_set(shared_opt, 1, H, I)) != MOE_OK) return st;
  if (shared_opt && shared_opt->gate.qtype != routed->gate.qtype) return MOE_ERR_INVALID_ARG;  // one format a layer
  if (n_rows == 0) return MOE_OK;
  if (!x_perm || !offsets || !out_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(out_perm) || !aligned16(offsets)) return MOE_ERR_ALIGNMENT;
  if (!ws) return MOE_ERR_WORKSPACE;
  // rows are accounted as T = n_rows tokens with one slot each
  const WsLayout L = ws_layout(H, E, 1, I, 0, n_rows);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  const bool gemm_ok = gemm_shape_supported(H, I) != 0;
  if (path == MOE_PATH_GEMM && !gemm_ok) return MOE_ERR_UNSUPPORTED;
  if (path == MOE_PATH_MMQ && !(gemm_ok && mmq_shape_supported(H, I, routed->gate.qtype))) return MOE_ERR_UNSUPPORTED;
  Ctrl *ctrl = at<Ctrl>(ws, L.ctrl);
  // AUTO: the grouped GEMM above 64 rows where its shape rule holds, the GEMV otherwise
  const int p = (path == MOE_PATH_AUTO && !(gemm_ok && n_rows > 64)) ? MOE_PATH_GEMV : path;
  // the int8 rows go to the workspace's (unused here) permuted-activation region
  return cuda_status(expert_rows(x_perm, offsets, n_rows, E, H, I, *routed, shared_opt, at<uint16_t>(ws, L.hperm),
                                 out_perm, at<int2>(ws, L.tiles), at<DecUnit>(ws, L.units),
                                 at<uint16_t>(ws, L.hdec), ctrl, (cudaStream_t)stream, p, gemm_ok,
                                 at<int8_t>(ws, L.xperm), at<float>(ws, L.dx)));
}

moe_status moe_combine(const uint16_t *out_perm, const int32_t *row_of, const float *w, int32_t T, int32_t k,
                       int32_t H, const uint16_t *shared_out_opt, const float *residual_opt, float *y, void *stream) {
  if (T < 0 || k < 1 || k > kMaxK || H <= 0 || H % 64 != 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!out_perm || !row_of || !w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out_perm) || !aligned16(y) || (shared_out_opt && !aligned16(shared_out_opt)) ||
      (residual_opt && !aligned16(residual_opt)))
    return MOE_ERR_ALIGNMENT;
  return cuda_status(
      launch_combine(out_perm, row_of, w, T, k, H, shared_out_opt, residual_opt, y, (cudaStream_t)stream));
}

// the layer's argument checks and, with run set, its launches (the host-buffer entry point checks
// first and enqueues its copies only for a call that will run)
static moe_status layer_forward_impl(const uint16_t *x, int32_t T, const float *Wr, const float *bias,
                                     const moe_layer_desc *desc, const moe_expert_set *routed,
                                     const moe_expert_set *shared_opt, const float *residual_opt, float *y,
                                     int32_t *idx_out_opt, float *w_out_opt, int32_t path, void *ws, size_t ws_bytes,
                                     void *stream, bool run) {
  if (!desc) return MOE_ERR_INVALID_ARG;
  const int H = desc->H, E = desc->E, k = desc->k, I = desc->I, hs = desc->has_shared ? 1 : 0;
  moe_status st = shape_status(H, E, k, I);
  if (st != MOE_OK) return st;
  if (T < 0 || path < 0 || path > 4) return MOE_ERR_INVALID_ARG;
  if ((st = check_set(routed, E, H, I)) != MOE_OK) return st;
  if (hs && (st = check_set(shared_opt, 1, H, I)) != MOE_OK) return st;
  if (hs && shared_opt->gate.qtype != routed->gate.qtype) return MOE_ERR_INVALID_ARG;  // one format a layer
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wr) || !aligned16(y) || (bias && !aligned16(bias)) ||
      (residual_opt && !aligned16(residual_opt)) || (idx_out_opt && !aligned16(idx_out_opt)) ||
      (w_out_opt && !aligned16(w_out_opt)))
    return MOE_ERR_ALIGNMENT;
  if (!ws) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(H, E, k, I, hs, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  const bool gemm_ok = gemm_shape_supported(H, I) != 0;
  if (path == MOE_PATH_GEMM && !gemm_ok) return MOE_ERR_UNSUPPORTED;
  if (path == MOE_PATH_MMQ && !(gemm_ok && mmq_shape_supported(H, I, routed->gate.qtype))) return MOE_ERR_UNSUPPORTED;
  const bool mid_ok = mid_shape_supported(T, H, E, I);
  if (path == MOE_PATH_MID && !mid_ok) return MOE_ERR_UNSUPPORTED;
  const bool fused_fits = path == MOE_PATH_AUTO && T <= kDecodeMaxT && decode_router_fits(T, H, E) &&
                          decode_fused_fits(T, H, E, k, I, *routed, hs != 0);
  const bool mid = path == MOE_PATH_MID ||
                   (path == MOE_PATH_AUTO && !fused_fits && mid_ok && T >= kAutoMidLo && T <= kAutoMidHi);
  if (!run) return MOE_OK;

  cudaStream_t s = (cudaStream_t)stream;
  Ctrl *ctrl = at<Ctrl>(ws, L.ctrl);
  int32_t *idx = at<int32_t>(ws, L.idx);
  float *w = at<float>(ws, L.w);
  float *logits = at<float>(ws, L.logits);
  const moe_expert_set *sh = hs ? shared_opt : nullptr;
  cudaError_t e = cudaSuccess;

  // decode path (distinct experts' weights read once, tokens as MMA columns) up to 8 tokens: at
  // T = 5..8 it takes about half the time of the grouped GEMM, whose 16-row tiles are bound by MMA
  // issue (measured by bench.py --crossover)
  const bool decode = (T <= kDecodeMaxT) && !mid && path != MOE_PATH_GEMM && path != MOE_PATH_MMQ &&
                      decode_router_fits(T, H, E);
  if (decode) {
    DecUnit *units = at<DecUnit>(ws, L.units);
    uint16_t *hdec = at<uint16_t>(ws, L.hdec);
    const int max_units = T * k + hs;
    // auto: one cooperative kernel when the shape fits it; path GEMV (or a shape the fused kernel
    // does not take): separate router / gate-up / down kernels
    e = cudaErrorNotSupported;
    if (path == MOE_PATH_AUTO) {
      e = launch_decode_fused(x, nullptr, 0.0f, T, H, Wr, bias, E, k, I, *routed, sh, residual_opt, y, idx, w, ctrl,
                              s);
      if (e == cudaErrorCooperativeLaunchTooLarge) {
        (void)cudaGetLastError();
        e = cudaErrorNotSupported;
      }
    }
    if (e == cudaErrorNotSupported) {
      e = launch_router_decode(x, T, H, Wr, bias, E, k, idx, w, logits, 1, hs, units, ctrl, s);
      if (e == cudaSuccess) e = launch_decode_gate_up(x, 1, H, I, *routed, sh, units, max_units, ctrl, hdec, s);
      if (e == cudaSuccess)
        e = launch_decode_down(H, I, *routed, sh, units, max_units, ctrl, hdec, y, residual_opt, T, nullptr, s);
    }
  } else {
    const int P = T * k, rows = P + (hs ? T : 0);
    int32_t *counts = at<int32_t>(ws, L.counts), *offsets = at<int32_t>(ws, L.offsets);
    int32_t *row_of = at<int32_t>(ws, L.row_of), *src = at<int32_t>(ws, L.src);
    uint16_t *xperm = at<uint16_t>(ws, L.xperm), *operm = at<uint16_t>(ws, L.operm);
    if (decode_router_fits(T, H, E))
      e = launch_router_decode(x, T, H, Wr, bias, E, k, idx, w, logits, 0, 0, at<DecUnit>(ws, L.units), ctrl, s);
    else
      e = launch_router_prefill(x, T, H, Wr, bias, E, k, idx, w, logits, at<uint16_t>(ws, L.wsplit), ctrl, s);
    if (mid) {
      if (e == cudaSuccess)
        e = launch_mid_ffn(x, T, H, E, k, I, idx, w, *routed, sh, residual_opt, y, at<MidUnit>(ws, L.units), row_of,
                           src, at<float>(ws, L.mid), ctrl, s);  // src: the partial rows' tokens
    } else {
    if (e == cudaSuccess)
      e = launch_permute(idx, T, k, E, x, H, hs, counts, offsets, row_of, src, xperm, at<int32_t>(ws, L.hist), ctrl,
                         s);
    if (e == cudaSuccess)
      e = expert_rows(xperm, offsets, rows, E, H, I, *routed, sh, at<uint16_t>(ws, L.hperm), operm,
                      at<int2>(ws, L.tiles), at<DecUnit>(ws, L.units), at<uint16_t>(ws, L.hdec), ctrl, s, path,
                      gemm_ok, at<int8_t>(ws, L.operm), at<float>(ws, L.dx));  // int8 rows: out_perm's region, free until the down GEMM
    if (e == cudaSuccess)
      e = launch_combine(operm, row_of, w, T, k, H, hs ? operm + (size_t)P * H : nullptr, residual_opt, y, s, ctrl);
    }
  }
  if (e == cudaSuccess && idx_out_opt)
    e = cudaMemcpyAsync(idx_out_opt, idx, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && w_out_opt)
    e = cudaMemcpyAsync(w_out_opt, w, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, s);
  return cuda_status(e);
}

moe_status moe_layer_forward(const uint16_t *x, int32_t T, const float *Wr, const float *bias,
                             const moe_layer_desc *desc, const moe_expert_set *routed,
                             const moe_expert_set *shared_opt, const float *residual_opt, float *y,
                             int32_t *idx_out_opt, float *w_out_opt, int32_t path, void *ws, size_t ws_bytes,
                             void *stream) {
  return layer_forward_impl(x, T, Wr, bias, desc, routed, shared_opt, residual_opt, y, idx_out_opt, w_out_opt, path,
                            ws, ws_bytes, stream, true);
}

// Host <-> workspace copies of the host-buffer entry points: up to kSmallIo bytes between a
// device-mapped page-locked host buffer and the workspace run as a copy kernel (a few
// microseconds less latency per transfer than a copy-engine transfer); anything else, pageable
// memory included, through cudaMemcpyAsync.
constexpr size_t kSmallIo = 256 * 1024;

static const void *mapped_host(const void *p, size_t bytes) {
  if (bytes > kSmallIo || bytes % 16 != 0 || !aligned16(p)) return nullptr;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return (at.type == cudaMemoryTypeHost && at.devicePointer && aligned16(at.devicePointer)) ? at.devicePointer
                                                                                            : nullptr;
}

static cudaError_t copy_in(void *dst_dev, const void *src_host, size_t bytes, cudaStream_t s) {
  if (const void *d = mapped_host(src_host, bytes)) return launch_io_copy(d, dst_dev, bytes, true, s);
  return cudaMemcpyAsync(dst_dev, src_host, bytes, cudaMemcpyHostToDevice, s);
}

static cudaError_t copy_out(void *dst_host, const void *src_dev, size_t bytes, cudaStream_t s) {
  if (const void *d = mapped_host(dst_host, bytes)) return launch_io_copy(src_dev, const_cast<void *>(d), bytes, false, s);
  return cudaMemcpyAsync(dst_host, src_dev, bytes, cudaMemcpyDeviceToHost, s);
}

moe_status moe_layer_forward_host(const uint16_t *x_host, int32_t T, const float *Wr, const float *bias,
                                  const moe_layer_desc *desc, const moe_expert_set *routed,
                                  const moe_expert_set *shared_opt, float *y_host, int32_t *idx_out_opt,
                                  float *w_out_opt, int32_t path, void *ws, size_t ws_bytes, void *stream) {
  if (!desc || T < 0) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x_host || !y_host)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && !ws) return MOE_ERR_WORKSPACE;
  const int H = desc->H;
  const WsLayout L = ws_layout(H, desc->E, desc->k, desc->I, desc->has_shared ? 1 : 0, T);
  uint16_t *xd = T > 0 ? at<uint16_t>(ws, L.xio) : nullptr;
  float *yd = T > 0 ? at<float>(ws, L.yio) : nullptr;
  moe_status st = layer_forward_impl(xd, T, Wr, bias, desc, routed, shared_opt, nullptr, yd, idx_out_opt, w_out_opt,
                                     path, ws, ws_bytes, stream, false);
  if (st != MOE_OK || T == 0) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (copy_in(xd, x_host, (size_t)T * H * 2, s) != cudaSuccess) return MOE_ERR_CUDA;
  st = layer_forward_impl(xd, T, Wr, bias, desc, routed, shared_opt, nullptr, yd, idx_out_opt, w_out_opt, path, ws,
                          ws_bytes, stream, true);
  if (st != MOE_OK) return st;
  return cuda_status(copy_out(y_host, yd, (size_t)T * H * 4, s));
}

// the stack's argument checks and, with run set, its work (as layer_forward_impl)
static moe_status stack_forward_impl(const float *r_in, int32_t T, int32_t L, const float *const *Wr,
                                     const float *const *bias, const moe_layer_desc *desc,
                                     const moe_expert_set *routed, const moe_expert_set *shared, float eps,
                                     float *r_out, int32_t path, void *ws, size_t ws_bytes, void *stream, bool run) {
  if (!desc || L < 0 || T < 0 || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  const int H = desc->H, E = desc->E, k = desc->k, I = desc->I, hs = desc->has_shared ? 1 : 0;
  moe_status st = shape_status(H, E, k, I);
  if (st != MOE_OK) return st;
  if (T == 0 || L == 0) {
    if (run && T > 0 && r_out != r_in && r_in && r_out)
      return cuda_status(cudaMemcpyAsync(r_out, r_in, (size_t)T * H * 4, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
    return MOE_OK;
  }
  if (!r_in || !r_out || !Wr || !routed || (hs && !shared)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(r_in) || !aligned16(r_out)) return MOE_ERR_ALIGNMENT;
  if (!ws) return MOE_ERR_WORKSPACE;
  const WsLayout LY = ws_layout(H, E, k, I, hs, T);
  if (ws_bytes < LY.total) return MOE_ERR_WORKSPACE;
  for (int l = 0; l < L; ++l) {
    if ((st = check_set(&routed[l], E, H, I)) != MOE_OK) return st;
    if (hs && (st = check_set(&shared[l], 1, H, I)) != MOE_OK) return st;
    if (hs && shared[l].gate.qtype != routed[l].gate.qtype) return MOE_ERR_INVALID_ARG;  // one format a layer
    if (!Wr[l]) return MOE_ERR_INVALID_ARG;
  }
  for (int l = 0; l < L; ++l)
    if (!aligned16(Wr[l]) || (bias && bias[l] && !aligned16(bias[l]))) return MOE_ERR_ALIGNMENT;
  uint16_t *u = at<uint16_t>(ws, LY.u16);
  // what the layer entry point checks besides (the path and whether it takes this shape)
  st = layer_forward_impl(u, T, Wr[0], bias ? bias[0] : nullptr, desc, &routed[0], hs ? &shared[0] : nullptr, r_out,
                          r_out, nullptr, nullptr, path, ws, ws_bytes, stream, false);
  if (st != MOE_OK || !run) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // decode-sized batches: one launch of the fused layer kernel per layer, RMSNorm inside it (a
  // single launch walking all the layers with a grid barrier between them measured slower:
  // 28.2 against 22.6 us per layer at one token)
  const bool fused = path == MOE_PATH_AUTO && T <= kDecodeMaxT && decode_router_fits(T, H, E);
  for (int l = 0; l < L; ++l) {
    const float *r = (l == 0) ? r_in : r_out;
    if (fused) {
      cudaError_t e = launch_decode_fused(nullptr, r, eps, T, H, Wr[l], bias ? bias[l] : nullptr, E, k, I, routed[l],
                                          hs ? &shared[l] : nullptr, r, r_out, at<int32_t>(ws, LY.idx),
                                          at<float>(ws, LY.w), at<Ctrl>(ws, LY.ctrl), s,
                                          l + 1 < L ? Wr[l + 1] : nullptr);
      if (e == cudaSuccess) continue;
      if (e != cudaErrorNotSupported && e != cudaErrorCooperativeLaunchTooLarge) return cuda_status(e);
      (void)cudaGetLastError();
    }
    if ((st = moe_rmsnorm_bf16(r, T, H, eps, u, stream)) != MOE_OK) return st;
    st = moe_layer_forward(u, T, Wr[l], bias ? bias[l] : nullptr, desc, &routed[l], hs ? &shared[l] : nullptr, r, r_out,
                           nullptr, nullptr, path, ws, ws_bytes, s);
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

moe_status moe_stack_forward(const float *r_in, int32_t T, int32_t L, const float *const *Wr,
                             const float *const *bias, const moe_layer_desc *desc, const moe_expert_set *routed,
                             const moe_expert_set *shared, float eps, float *r_out, int32_t path, void *ws,
                             size_t ws_bytes, void *stream) {
  return stack_forward_impl(r_in, T, L, Wr, bias, desc, routed, shared, eps, r_out, path, ws, ws_bytes, stream, true);
}

moe_status moe_stack_forward_host(const float *r_in_host, int32_t T, int32_t L, const float *const *Wr,
                                  const float *const *bias, const moe_layer_desc *desc, const moe_expert_set *routed,
                                  const moe_expert_set *shared, float eps, float *r_out_host, int32_t path, void *ws,
                                  size_t ws_bytes, void *stream) {
  if (!desc || T < 0 || L < 0) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!r_in_host || !r_out_host)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && !ws) return MOE_ERR_WORKSPACE;
  const int H = desc->H;
  float *rd = T > 0 ? at<float>(ws, ws_layout(H, desc->E, desc->k, desc->I, desc->has_shared ? 1 : 0, T).yio)
                    : nullptr;
  // the stack runs in place on the staged stream (each layer reads its input rows before
  // writing them)
  moe_status st = stack_forward_impl(rd, T, L, Wr, bias, desc, routed, shared, eps, rd, path, ws, ws_bytes, stream,
                                     false);
  if (st != MOE_OK || T == 0) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (copy_in(rd, r_in_host, (size_t)T * H * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  st = stack_forward_impl(rd, T, L, Wr, bias, desc, routed, shared, eps, rd, path, ws, ws_bytes, stream, true);
  if (st != MOE_OK) return st;
  return cuda_status(copy_out(r_out_host, rd, (size_t)T * H * 4, s));
}

moe_status moe_dequant_rows(const moe_qmat *m, int32_t expert, int32_t row0, int32_t nrows, float *out_f32,
                            uint16_t *out_f16, void *stream) {
  if (!m) return MOE_ERR_INVALID_ARG;
  if (m->K <= 0 || m->K % 32 != 0 || m->rows <= 0 || m->n_experts <= 0) return MOE_ERR_INVALID_ARG;
  moe_status st = check_qmat(*m, m->n_experts, m->rows, m->K);
  if (st != MOE_OK) return st;
  if (expert < 0 || expert >= m->n_experts || row0 < 0 || nrows < 0 || row0 + nrows > m->rows)
    return MOE_ERR_INVALID_ARG;
  if (nrows == 0) return MOE_OK;
  if (!out_f32 && !out_f16) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_dequant_rows(*m, expert, row0, nrows, out_f32, out_f16, (cudaStream_t)stream));
}

moe_status moe_timing_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_tmu);
  if (on) {
    for (auto &r : g_recs) {
      g_pool.push_back(r.begin);
      g_pool.push_back(r.end);
    }
    g_recs.clear();
  }
  g_timing = on != 0;
  return MOE_OK;
}

moe_status moe_timing_read(int32_t kernel, double *total_ms, int32_t *launches) {
  if (kernel < 0 || kernel >= KID_COUNT || !total_ms || !launches) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_tmu);
  double tot = 0.0;
  int n = 0;
  for (auto &r : g_recs) {
    if (r.kid != kernel) continue;
    float ms = 0.0f;
    if (cudaEventSynchronize(r.end) != cudaSuccess || cudaEventElapsedTime(&ms, r.begin, r.end) != cudaSuccess)
      return MOE_ERR_CUDA;
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return MOE_OK;
}

int32_t moe_kernel_count(void) { return KID_COUNT; }

const char *moe_kernel_name(int32_t kernel) {
  return (kernel >= 0 && kernel < KID_COUNT) ? kKernelNames[kernel] : nullptr;
}

moe_status moe_test_wait_timeout(void *ws, size_t ws_bytes, int32_t limit_ms, void *stream) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if (ws_bytes < kControlBytes) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  if (limit_ms < 1 || limit_ms > 2000) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_wait_starve(static_cast<Ctrl *>(ws), (uint64_t)limit_ms * 1000000ull, (cudaStream_t)stream));
}

moe_status moe_read_device_error(void *ws, int32_t *code, void *stream) {
  if (!ws || !code) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
  cudaStream_t s = (cudaStream_t)stream;
  int v[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(v, ws, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, 2 * sizeof(int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *code = v[0];
  return MOE_OK;
}

}  // extern "C"
