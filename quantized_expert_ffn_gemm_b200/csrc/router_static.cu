// Router + top-k for callers that cannot allocate device memory.
//
// moe_router_topk needs a caller-provided workspace for its scratch (the last-CTA ticket and the
// [T][E] logits the top-k reads back). Some callers have no way to obtain one: plugins hosted by
// an application that owns and budgets every device allocation and hands its plugins none, or
// runtimes that lay out all device memory ahead of time and have no allocator to call at run
// time. This variant keeps its scratch in a fixed-size array inside the library instead, so the
// caller passes only inputs and outputs.
//
// The array lives in every GPU that loads the library until the process exits. In host code the
// array's name is only a host-side stand-in, so its device address is looked up once per device
// (cudaGetSymbolAddress, with that device current) on the first call and kept in a per-device
// table. All calls share the one array: calls that overlap on
// the GPU (different streams, or different host threads) race on it and must be serialised by
// the caller.
//
// The array also holds a control area with an error word. The router kernel records no
// device-side error (it has no bounded waits and no index inputs), so this word is only cleared
// by each call, never set, and nothing is lost by having no reader for it.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kStaticMaxT = 8;       // tokens per call
constexpr int kStaticMaxE = 4096;    // routed experts
constexpr size_t kStaticCtrlBytes = 256;
constexpr size_t kStaticScratchBytes = kStaticCtrlBytes + (size_t)kStaticMaxT * kStaticMaxE * sizeof(float);

// control word (zeroed on every call) followed by the [T][E] fp32 logits
static __device__ __align__(256) unsigned char g_router_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[64] = {};

// device address of the scratch array on the current device (looked up once per device)
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_router_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_router_topk_static(const uint16_t *x, int32_t T, int32_t H, const float *Wr,
                                             const float *bias, int32_t E, int32_t k, int32_t *idx, float *w,
                                             float *logits_opt, void *stream) {
  // the shape rules of moe_router_topk first (the same arguments get the same status) ...
  const moe_status st = layer_shape_status(H, E, k, 64);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  // ... then the limits of the fixed scratch
  if (T > kStaticMaxT || E > kStaticMaxE || (size_t)T * (H > E ? H : E) * 4 > 200 * 1024)
    return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch (or the single-kernel router's shared memory)
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !idx || !w) return MOE_ERR_INVALID_ARG;
  auto a16 = [](const void *p) { return ((uintptr_t)p & 15u) == 0; };
  if (!a16(x) || !a16(Wr) || !a16(idx) || !a16(w) || (bias && !a16(bias)) || (logits_opt && !a16(logits_opt)))
    return MOE_ERR_ALIGNMENT;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(scratch);
  float *logits = logits_opt ? logits_opt
                             : reinterpret_cast<float *>(static_cast<unsigned char *>(scratch) + kStaticCtrlBytes);
  // the array keeps the previous call's contents: the ticket and error word must start at zero
  if (cudaMemsetAsync(ctrl, 0, sizeof(Ctrl), s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = launch_router_decode(x, T, H, Wr, bias, E, k, idx, w, logits, 0, 0, nullptr, ctrl, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
