/*
 * moe_ffn.h -- C ABI of the B200 (sm_100a) quantized Mixture-of-Experts layer library
 * (libmoe_ffn.so).
 *
 * The library computes the forward pass of one sparse MoE layer whose expert weights are
 * low-bit block-quantized, and a stack of such layers:
 *
 *   router   logits = x Wr^T (+ bias), fp32 softmax, top-k, renormalised weights
 *   permute  token -> expert-contiguous rows (histogram, exclusive scan, stable scatter)
 *   experts  per active expert e: h = silu(x W_gate[e]^T) * (x W_up[e]^T), o = h W_down[e]^T
 *   combine  y[t] = sum_j w[t,j] o[t,j] + shared(x[t]) (+ residual[t])
 *
 * Passages this follows:
 *   - 512 routed experts per layer, 10 active per token, 48 layers, shared experts kept on the
 *     GPU: "Strata vs Llama.cpp vs vLLM", chapter "How Strata is designed to work";
 *     Strata DETAILS.md, section "How it works" (memory-tiers list).
 *   - the expert matmul dequantizes low-bit block weights during the multiply:
 *     "Two-Day Port, 8x Faster Prefill: Strata Engine Benchmarked", section
 *     "Where Strata Is Fast: Not Magic, but Logistics" (MMQ paragraph).
 *   - prefill chunks of up to 8,192 tokens; decode / MTP-verify passes of 1-4 tokens:
 *     "Strata vs Llama.cpp vs vLLM", same chapter; Strata DETAILS.md, "How it works".
 *   The pages do not fix the quantization formats; this library implements the stand-in:
 *     Q2: blocks of 32 weights, 2-bit codes c, one fp16 scale d, w = d*(c-2)
 *     Q3: blocks of 32 weights, 3-bit codes c, one fp16 scale d, w = d*(c-4)
 *     Q4: blocks of 32 weights, 4-bit codes c, one fp16 scale d, w = d*(c-8) (a further format of
 *         the same family, for layers that keep more bits)
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library allocates no
 *     device memory on any path, keeps no pointer after a call returns (apart from the
 *     per-process cache of the CUDA driver entry point) and never frees caller memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every call
 *     only enqueues work on it and returns; nothing synchronises except
 *     moe_read_device_error.
 *   - The library's kernels are launched with programmatic stream serialization: a launch may
 *     begin while the previous kernel on the stream finishes, but only when that kernel allows
 *     it (this library's kernels do, at their entry; set MOE_PDL=0 in the environment to turn
 *     it off). Everything a predecessor may write is read only after it has completed, except
 *     the layers' router weights Wr, which the fused decode kernel starts reading early: a
 *     kernel that writes Wr and allows its dependents to start before it ends (CUDA's
 *     programmatic launch completion) must not directly precede a layer call.
 *   - bf16 / fp16 tensors are passed as uint16_t bit patterns. Layouts are row-major and
 *     contiguous: x, y, r: [T,H]; idx, w: [T,k]; Wr: [E,H].
 *   - Arguments are validated on the host before anything is enqueued; on error nothing runs
 *     and a status code is returned. No entry point aborts, exits or traps.
 *   - T = 0 is a no-op that returns MOE_OK.
 *   - Device tensors must be 16-byte aligned (MOE_ERR_ALIGNMENT otherwise).
 *   - Faults the device detects (an expert index >= E handed to moe_permute, a bounded wait
 *     that timed out, a value outside the fp16 operand range) are recorded in the workspace's
 *     error word; read and clear the word with moe_read_device_error.
 *
 * Packed weight planes (moe_qmat)
 *   One matrix kind (gate, up or down) of n_experts experts: `rows` output features, reduction
 *   dimension K (a multiple of 32), blocks of 32 weights along K.
 *     codes  uint8 [n_experts][rows][K/4]  2-bit plane: Q2 codes, or the low 2 bits of Q3 codes.
 *            Per block, two 32-bit little-endian words; word q (weights 16q..16q+15) holds
 *            weight 16q+2i+h (i = 0..7, h = 0..1) at bits 16h+2i .. 16h+2i+1.
 *            Q4: uint8 [n_experts][rows][K/2], the 4-bit plane: per block four 32-bit
 *            little-endian words; word q (weights 8q..8q+7) holds weight 8q+2i+h (i = 0..3,
 *            h = 0..1) at bits 16h+4i .. 16h+4i+3.
 *     hibits uint8 [n_experts][rows][K/8]  Q3 only (NULL for Q2 and Q4): per block one 32-bit
 *            little-endian word holding bit 2 of the code of weight 16q+2i+h at bit 16h+8q+i.
 *     scales fp16  [n_experts][rows][K/32] one scale per block.
 *   gate and up: rows = I, K = H.  down: rows = H, K = I.
 *   (The bit order puts weights 2i and 2i+1 of each half-block in the two 16-bit halves of a
 *   word, so a single mask extracts an adjacent pair; the pages fix no layout.)
 *
 * Numerics
 *   router logits, softmax and routing weights: fp32 (x is exact in fp32). Top-k is taken on
 *   the fp32 logits; equal logits: the lower expert index wins; slots are stored in descending
 *   logit order. Expert contractions: fp16 operands (Q2 weights are exact in fp16, bf16 x is
 *   exact in fp16 in its normal range), fp32 accumulation; intermediate h and per-expert
 *   outputs are stored as fp16; y, the residual stream and the combine are fp32. A value that
 *   does not fit fp16 (|x| > 65504, or an h or expert output that overflows) is not rescaled:
 *   it becomes +-inf and moe_layer_forward / moe_stack_forward / moe_permute record
 *   MOE_ERR_RANGE in the workspace error word.
 */
#ifndef MOE_FFN_H
#define MOE_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t moe_status;
enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, k out of range, H or I not a multiple of 32 */
  MOE_ERR_ALIGNMENT = 2,     /* a device pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than moe_workspace_bytes() */
  MOE_ERR_UNSUPPORTED = 4,   /* valid request the library cannot run (e.g. forced GEMM path, H % 128 != 0) */
  MOE_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed (launch error, no device) */
  MOE_ERR_DEVICE_CHECK = 6,  /* reported by moe_read_device_error: a device-side index check failed */
  MOE_ERR_TIMEOUT = 7,       /* reported by moe_read_device_error: a bounded device wait gave up */
  MOE_ERR_RANGE = 8          /* reported by moe_read_device_error: a value left the fp16 range of the
                                expert operands (an input x above 65504 in magnitude, or an
                                intermediate h or expert output that overflowed); it became +-inf */
};

enum { MOE_Q2 = 2, MOE_Q3 = 3, MOE_Q4 = 4 };

/* expert-FFN path selection. MOE_PATH_MMQ: int8 activations (one scale per 32-value block) and
 * the Q2 weights' integer codes on tcgen05 kind::i8 for gate/up (exact integer block sums, both
 * block scales applied on the read-back), then the fp16 down GEMM; Q2 weights, H % 256 == 0,
 * I % 128 == 0 (MOE_ERR_UNSUPPORTED otherwise). The int8 activations change the numerics (the
 * oracle's fp64 definition is met within the usual 1e-2 only because the rounding is per block). */
/* MOE_PATH_MID (moe_layer_forward and moe_stack_forward only): the mid-batch path for 1..128 tokens
 * (small verify passes and batches; Strata DETAILS.md, "How it works"). Each selected expert's
 * tokens are grouped into units of up to 8 straight from the routing (no permuted copy); every
 * (unit, 128-feature slice) item runs gate/up + SwiGLU and that slice of the down projection into
 * fp32 partial rows, summed per token in a fixed order. Needs I % 128 == 0 and H <= 4096
 * (MOE_ERR_UNSUPPORTED otherwise; moe_expert_ffn returns it for this path). */
enum { MOE_PATH_AUTO = 0, MOE_PATH_GEMV = 1, MOE_PATH_GEMM = 2, MOE_PATH_MMQ = 3, MOE_PATH_MID = 4 };

typedef struct moe_qmat {
  int32_t qtype;            /* MOE_Q2, MOE_Q3 or MOE_Q4 (all matrices of a layer, shared expert included, share one; MOE_ERR_INVALID_ARG otherwise) */
  int32_t n_experts;
  int32_t rows;
  int32_t K;
  const uint8_t *codes;     /* [n_experts][rows][K/4]; Q4: [n_experts][rows][K/2] */
  const uint8_t *hibits;    /* [n_experts][rows][K/8] for Q3, NULL for Q2 and Q4 */
  const uint16_t *scales;   /* [n_experts][rows][K/32] fp16 bits */
} moe_qmat;

typedef struct moe_expert_set {
  moe_qmat gate;            /* rows = I, K = H */
  moe_qmat up;              /* rows = I, K = H */
  moe_qmat down;            /* rows = H, K = I */
} moe_expert_set;

typedef struct moe_layer_desc {
  int32_t H;                /* hidden size, multiple of 32 */
  int32_t E;                /* routed experts */
  int32_t k;                /* active experts per token, 1 <= k <= min(E, 32) */
  int32_t I;                /* expert intermediate size, multiple of 32 */
  int32_t has_shared;       /* 1: one always-on shared expert (unweighted) */
} moe_layer_desc;

/* Human-readable name of a status code (static string). */
const char *moe_status_string(moe_status s);

/* Bytes of device workspace that moe_layer_forward / moe_stack_forward need for T tokens of a
 * layer shaped like `desc`; the other entry points need no more than this. Returns 0 for an
 * invalid descriptor. */
size_t moe_workspace_bytes(const moe_layer_desc *desc, int32_t T);

/* Zero the workspace's control area (error word and the counters that the kernels leave at
 * zero on exit). Call once on a freshly allocated workspace before its first use. */
moe_status moe_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* RMSNorm with no learned gain, the stack's pre-router normalisation (the 48-layer stack of
 * "Strata vs Llama.cpp vs vLLM", "How Strata is designed to work"; the pages give no norm
 * details, so this is the plain reading: eps inside the square root, no gain, bf16 output):
 *   u[t,h] = bf16_rne( r[t,h] / sqrt(mean_h r[t,h]^2 + eps) ), fp32 arithmetic.
 * r fp32 [T,H] -> u bf16 [T,H]. */
moe_status moe_rmsnorm_bf16(const float *r, int32_t T, int32_t H, float eps, uint16_t *u, void *stream);

/* Router and top-k ("Strata vs Llama.cpp vs vLLM", "How Strata is designed to work": each
 * token is routed to 10 of 512 experts).
 *   logits[t,e] = sum_h x[t,h] Wr[e,h] + bias[e]            (fp32, bias optional: NULL = 0)
 *   idx[t,:]    = the k experts of largest logit, descending; ties -> lower index first
 *   w[t,j]      = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0)  (softmax restricted to the set,
 *                 equal to the full softmax renormalised over the set)
 * x bf16 [T,H]; Wr fp32 [E,H]; bias fp32 [E] or NULL; idx int32 [T,k]; w fp32 [T,k];
 * logits_opt fp32 [T,E] or NULL. Requires 1 <= k <= min(E,32), E <= 4096, H % 32 == 0.
 * ws: workspace of at least moe_workspace_bytes({H,E,k,32,0}, T) bytes, initialised. */
moe_status moe_router_topk(const uint16_t *x, int32_t T, int32_t H, const float *Wr, const float *bias,
                           int32_t E, int32_t k, int32_t *idx, float *w, float *logits_opt,
                           void *ws, size_t ws_bytes, void *stream);

/* Token permutation into expert-contiguous rows (stable counting sort by expert), so each active
 * expert's tokens form one block its weights are applied to at once ("Two-Day Port, 8x Faster
 * Prefill: Strata Engine Benchmarked", "Where Strata Is Fast: Not Magic, but Logistics": the
 * larger the batch, the more tokens share each expert's weights).
 *   counts[e]        number of (t,j) with idx[t,j] == e
 *   offsets[0..E]    exclusive scan of counts; with_shared: offsets[E+1] = T*k + T
 *   row_of[t*k+j]    row of pair (t,j); rows of one expert are in token order
 *   src[row]         token of the pair stored at `row` (row < T*k); with_shared, rows
 *                    T*k .. T*k+T-1 hold tokens 0..T-1 (src[T*k+t] = t) for the shared expert
 *   x_perm[row,:]    fp16(x[src[row],:])
 * idx int32 [T,k] with values in [0,E) (others are skipped and flagged in the error word);
 * x bf16 [T,H]; x_perm fp16 [T*k (+T), H]. */
moe_status moe_permute(const int32_t *idx, int32_t T, int32_t k, int32_t E, const uint16_t *x, int32_t H,
                       int32_t with_shared, int32_t *counts, int32_t *offsets, int32_t *row_of, int32_t *src,
                       uint16_t *x_perm, void *ws, size_t ws_bytes, void *stream);

/* Grouped expert FFN over expert-contiguous rows, dequantizing the block weights inside the
 * multiply ("Two-Day Port, 8x Faster Prefill: Strata Engine Benchmarked", "Where Strata Is Fast:
 * Not Magic, but Logistics", MMQ paragraph): for every row r < n_rows of group g
 * (offsets[g] <= r < offsets[g+1]):
 *   out_perm[r,:] = fp16( W_down[g] ( silu(W_gate[g] x_perm[r]) * (W_up[g] x_perm[r]) ) )
 * Groups 0..E-1 use `routed`; with shared_opt != NULL, group E (rows offsets[E]..offsets[E+1])
 * uses the shared expert. offsets (device) has E+1 (+1) monotone entries with
 * offsets[last] <= n_rows. path: MOE_PATH_GEMM = tcgen05 grouped GEMM (needs H % 128 == 0 and
 * I % 128 == 0), MOE_PATH_GEMV = dequant-GEMV, MOE_PATH_AUTO picks the GEMM when n_rows > 64
 * and the GEMM shape rule holds, the GEMV otherwise.
 * x_perm fp16 [n_rows,H]; out_perm fp16 [n_rows,H]. */
moe_status moe_expert_ffn(const uint16_t *x_perm, const int32_t *offsets, int32_t n_rows, int32_t E, int32_t H,
                          int32_t I, const moe_expert_set *routed, const moe_expert_set *shared_opt,
                          uint16_t *out_perm, int32_t path, void *ws, size_t ws_bytes, void *stream);

/* Un-permute and weighted combine (each token's output is its k experts' outputs weighted by
 * the routing weights, plus the always-on shared expert: "Strata vs Llama.cpp vs vLLM", "How
 * Strata is designed to work"; Strata DETAILS.md, "How it works"):
 *   y[t,:] = sum_{j<k} w[t,j] out_perm[row_of[t,j],:] + shared_out[t,:] + residual[t,:]
 * summed in fixed j order in fp32. out_perm fp16; shared_out_opt fp16 [T,H] or NULL;
 * residual_opt fp32 [T,H] or NULL (may alias y); y fp32 [T,H]. */
moe_status moe_combine(const uint16_t *out_perm, const int32_t *row_of, const float *w, int32_t T, int32_t k,
                       int32_t H, const uint16_t *shared_out_opt, const float *residual_opt, float *y,
                       void *stream);

/* One full MoE layer (512 routed experts, 10 active per token, a shared expert; 8,192-token
 * prefill chunks and 1-4-token decode / MTP-verify passes: "Strata vs Llama.cpp vs vLLM", "How
 * Strata is designed to work"; Strata DETAILS.md, "How it works"). T <= 8 with path AUTO or
 * GEMV: the decode path (router + top-k, then a
 * dequant-GEMV over the distinct selected experts with the tokens as MMA columns, down
 * projection fused with the weighted combine; under AUTO one cooperative kernel does the whole
 * layer where its shared-memory plan fits, T*k + T <= 96). AUTO with 8..20 tokens where that
 * kernel does not fit, or path MID: the mid-batch path (MOE_PATH_MID above). Otherwise: router +
 * top-k (fp32 dot products on the CUDA cores up to 128 tokens, tensor-core logits with an exact
 * refine of the candidates above), permute, the expert FFN (AUTO / GEMM: tcgen05 grouped GEMM
 * gate/up with fused SwiGLU, then down; GEMV: the decode GEMV kernels over 8-row chunks of each
 * expert's rows; MMQ: int8 activations for gate/up), combine. Every path computes the same
 * function within the parity tolerance.
 *   y = sum_j w_j FFN_{idx_j}(x) + FFN_shared(x) (+ residual)      fp32 [T,H]
 * x bf16 [T,H]; Wr fp32 [E,H]; bias fp32 [E] or NULL; routed: gate/up [E][I][H], down [E][H][I];
 * shared_opt: one expert (n_experts = 1) when desc->has_shared; residual_opt fp32 [T,H] or NULL
 * (may alias y); idx_out_opt int32 [T,k] / w_out_opt fp32 [T,k]: optional copies of the routing.
 * ws: at least moe_workspace_bytes(desc, T) bytes, initialised once with moe_workspace_init. */
moe_status moe_layer_forward(const uint16_t *x, int32_t T, const float *Wr, const float *bias,
                             const moe_layer_desc *desc, const moe_expert_set *routed,
                             const moe_expert_set *shared_opt, const float *residual_opt, float *y,
                             int32_t *idx_out_opt, float *w_out_opt, int32_t path,
                             void *ws, size_t ws_bytes, void *stream);

/* moe_layer_forward with the tokens and the output in HOST memory: x_host bf16 [T,H] is copied to
 * the workspace, the layer runs on it (no residual), and y lands in y_host fp32 [T,H]; one call
 * enqueues the host-to-device copy, the layer and the device-to-host copy on `stream` and returns
 * (the copies are asynchronous for page-locked host buffers, and those of up to 256 KB run as a
 * copy kernel reading or writing the mapped host buffer; y_host is complete once the stream has
 * reached this point). The weights, the workspace and the optional routing outputs stay in
 * device memory; other arguments and errors as moe_layer_forward (MOE_ERR_INVALID_ARG for a
 * NULL x_host or y_host). */
moe_status moe_layer_forward_host(const uint16_t *x_host, int32_t T, const float *Wr, const float *bias,
                                  const moe_layer_desc *desc, const moe_expert_set *routed,
                                  const moe_expert_set *shared_opt, float *y_host, int32_t *idx_out_opt,
                                  float *w_out_opt, int32_t path, void *ws, size_t ws_bytes, void *stream);

/* A stack of L layers with pre-router RMSNorm and a residual stream, attention omitted (the
 * 48 MoE layers of "Strata vs Llama.cpp vs vLLM", "How Strata is designed to work"):
 *   r_0 = r_in;  r_{l+1} = r_l + layer_l( bf16(RMSNorm_eps(r_l)) );  r_out = r_L
 * r_in, r_out fp32 [T,H] (r_out may equal r_in). Wr[l], bias[l] (bias may be NULL, or
 * bias[l] NULL), routed[l], shared[l] (NULL when desc->has_shared == 0): per-layer arrays
 * of HOST-side pointers/structs, each element as in moe_layer_forward. */
moe_status moe_stack_forward(const float *r_in, int32_t T, int32_t L, const float *const *Wr,
                             const float *const *bias, const moe_layer_desc *desc,
                             const moe_expert_set *routed, const moe_expert_set *shared, float eps,
                             float *r_out, int32_t path, void *ws, size_t ws_bytes, void *stream);

/* moe_stack_forward with the residual stream in HOST memory: r_in_host fp32 [T,H] is copied to the
 * workspace, the stack runs there in place, and the result lands in r_out_host fp32 [T,H] (may be
 * the same buffer); one call enqueues the two copies and the stack on `stream` and returns.
 * Weights and workspace in device memory; other arguments and errors as moe_stack_forward. */
moe_status moe_stack_forward_host(const float *r_in_host, int32_t T, int32_t L, const float *const *Wr,
                                  const float *const *bias, const moe_layer_desc *desc, const moe_expert_set *routed,
                                  const moe_expert_set *shared, float eps, float *r_out_host, int32_t path, void *ws,
                                  size_t ws_bytes, void *stream);

/* Test hook: dequantize rows row0..row0+nrows-1 of one expert with the decoder the expert
 * kernels use (the block formats are the stand-in stated at the top of this file).
 *   out_f32[r,k] = d*(c-q0) in fp32 (exact); out_f16[r,k] = fp16_rne(d*(c-q0)), the value the
 *   expert kernels feed to the tensor cores. Either output may be NULL. [nrows, K] each. */
moe_status moe_dequant_rows(const moe_qmat *m, int32_t expert, int32_t row0, int32_t nrows, float *out_f32,
                            uint16_t *out_f16, void *stream);

/* Router and top-k without a workspace, for callers that cannot allocate device memory: plugins
 * hosted by an application that owns and budgets all device memory and gives its plugins no
 * allocator, or runtimes that lay out all device memory ahead of time and have no allocator at
 * run time. The pages have no counterpart: this is a variant of moe_router_topk (same
 * arguments, same results, the same shape rules and status codes) whose scratch -- a control
 * word and the [T][E] fp32 logits -- is a fixed array inside the library (about 128 KB, held on
 * every GPU that loads the library until the process exits). Limits: T <= 8, E <= 4096 (and
 * T * max(H, E) * 4 <= 200 KB); larger requests return MOE_ERR_UNSUPPORTED. The first call on
 * each device looks up the array's device address (a host-side runtime query, kept per device).
 * All calls share the array, which keeps the last call's contents (each call clears what must
 * start at zero): calls that overlap on the GPU race and must be serialised by the caller. The
 * router kernel records no device-side error, so the array's error word needs no reader. It
 * allocates no memory. */
moe_status moe_router_topk_static(const uint16_t *x, int32_t T, int32_t H, const float *Wr, const float *bias,
                                  int32_t E, int32_t k, int32_t *idx, float *w, float *logits_opt, void *stream);

/* Per-kernel device timing, off by default. While enabled, the library records a pair of CUDA
 * events on the launching stream around every kernel it launches (from the calling host thread;
 * not for use during CUDA-graph capture) and keeps them in a process-wide list. Enabling (on = 1)
 * clears the list; on = 0 stops recording and keeps what was recorded.
 * moe_timing_read synchronises the recorded events and returns, for kernel id `kernel`
 * (0 <= kernel < moe_kernel_count()), the summed device time in milliseconds and the number of
 * launches. moe_kernel_name gives a static name for an id (NULL when out of range). */
moe_status moe_timing_enable(int32_t on);
moe_status moe_timing_read(int32_t kernel, double *total_ms, int32_t *launches);
int32_t moe_kernel_count(void);
const char *moe_kernel_name(int32_t kernel);

/* Synchronise `stream`, read the workspace's device error word into *code (MOE_OK,
 * MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT or MOE_ERR_RANGE; the first error recorded wins) and
 * clear it. */
moe_status moe_read_device_error(void *ws, int32_t *code, void *stream);

/* Test hook for the failure path of the device-side waits. Launches one warp that waits, with the
 * bounded wait the fused decode kernel uses for its exchanged router logits, for a logit word
 * whose launch tag no launch writes; every lane gives up after limit_ms (1..2000) and
 * MOE_ERR_TIMEOUT is recorded in the workspace error word (read and clear it with
 * moe_read_device_error). Nothing traps, the context stays usable and nothing but the error word
 * is written, so the workspace serves the next call unchanged. ws: an initialised workspace of at
 * least moe_workspace_bytes(desc, 1) bytes for some layer (its control area), 16-byte aligned;
 * errors: MOE_ERR_WORKSPACE / MOE_ERR_ALIGNMENT / MOE_ERR_INVALID_ARG on the host. */
moe_status moe_test_wait_timeout(void *ws, size_t ws_bytes, int32_t limit_ms, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FFN_H */
