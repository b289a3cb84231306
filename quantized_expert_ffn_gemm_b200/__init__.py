"""Thin Python binding of libmoe_ffn.so (quantized Mixture-of-Experts layer for B200, sm_100a).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels. PyTorch
supplies device memory and the current CUDA stream. If the shared library is missing or cannot
be loaded, importing works but every call raises (there is no fallback path).

Entry points mirror include/moe_ffn.h: rmsnorm_bf16, router_topk, permute, expert_ffn, combine,
layer_forward, stack_forward, dequant_rows, read_device_error, plus a Workspace helper.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_ffn.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_ALIGNMENT, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT, MOE_ERR_RANGE = 4, 5, 6, 7, 8
PATH_AUTO, PATH_GEMV, PATH_GEMM, PATH_MMQ, PATH_MID = 0, 1, 2, 3, 4
Q2, Q3, Q4 = 2, 3, 4

EXPORTED = ["moe_status_string", "moe_workspace_bytes", "moe_workspace_init", "moe_rmsnorm_bf16",
            "moe_router_topk", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
            "moe_stack_forward", "moe_dequant_rows", "moe_read_device_error", "moe_timing_enable",
            "moe_timing_read", "moe_kernel_count", "moe_kernel_name", "moe_router_topk_static",
            "moe_test_wait_timeout", "moe_layer_forward_host", "moe_stack_forward_host"]


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


class QMat(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("rows", ctypes.c_int32),
                ("K", ctypes.c_int32), ("codes", ctypes.c_void_p), ("hibits", ctypes.c_void_p),
                ("scales", ctypes.c_void_p)]


class ExpertSet(ctypes.Structure):
    _fields_ = [("gate", QMat), ("up", QMat), ("down", QMat)]


class LayerDesc(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("I", ctypes.c_int32),
                ("has_shared", ctypes.c_int32)]


_lib = None
_load_error: Optional[str] = None


def lib():
    """The loaded library; raises if it is missing (build it with build.py / __graft_entry__.build())."""
    global _lib, _load_error
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not found: build it with `python -m quantized_expert_ffn_gemm_b200.build`")
        _lib = ctypes.CDLL(LIB_PATH)
        _lib.moe_status_string.restype = ctypes.c_char_p
        _lib.moe_status_string.argtypes = [ctypes.c_int32]
        _lib.moe_workspace_bytes.restype = ctypes.c_size_t
        _lib.moe_workspace_bytes.argtypes = [ctypes.POINTER(LayerDesc), ctypes.c_int32]
        for name in EXPORTED[2:]:
            getattr(_lib, name).restype = ctypes.c_int32
        _lib.moe_kernel_name.restype = ctypes.c_char_p
        _lib.moe_kernel_name.argtypes = [ctypes.c_int32]
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def _check(fn: str, code: int):
    if code != MOE_OK:
        raise MoeError(fn, code)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


# the raw handle of a device's current stream, without building a Stream object (~3 us per call
# in the decode loop otherwise); torch's own accessor when the fast one is absent
_raw_stream_fn = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _raw_stream(dev: int) -> int:
    if _raw_stream_fn is not None:
        return _raw_stream_fn(dev)
    return torch.cuda.current_stream(dev).cuda_stream


def qmat(m) -> QMat:
    """QMat struct from an object with qtype, n, rows, K and codes / hibits / scales device tensors."""
    return QMat(int(m.qtype), int(m.n), int(m.rows), int(m.K), m.codes.data_ptr(),
                None if m.hibits is None else m.hibits.data_ptr(), m.scales.data_ptr())


def expert_set(es) -> ExpertSet:
    return ExpertSet(qmat(es.gate), qmat(es.up), qmat(es.down))


def layer_desc(H: int, E: int, k: int, I: int, has_shared: bool) -> LayerDesc:
    return LayerDesc(H, E, k, I, 1 if has_shared else 0)


def workspace_bytes(H: int, E: int, k: int, I: int, has_shared: bool, T: int) -> int:
    d = layer_desc(H, E, k, I, has_shared)
    return int(lib().moe_workspace_bytes(ctypes.byref(d), int(T)))


class Workspace:
    """Device workspace (caller-owned memory for the library), zero-initialised control area."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = int(max(nbytes, 256))
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        _check("moe_workspace_init", lib().moe_workspace_init(_p(self.buf), ctypes.c_size_t(self.nbytes), _stream()))

    @classmethod
    def for_layer(cls, H, E, k, I, has_shared, T, device="cuda"):
        n = workspace_bytes(H, E, k, I, has_shared, T)
        if n == 0:
            raise MoeError("moe_workspace_bytes", MOE_ERR_INVALID_ARG)
        return cls(n, device)

    @property
    def ptr(self):
        return _p(self.buf)

    @property
    def size(self):
        return ctypes.c_size_t(self.nbytes)


def _u16(t: torch.Tensor) -> torch.Tensor:
    return t  # bf16 / fp16 tensors are passed by pointer; bit patterns are what the ABI reads


# ----------------------------------------------------------------------------- entry points
def rmsnorm_bf16(r: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    T, H = r.shape
    u = torch.empty(T, H, dtype=torch.bfloat16, device=r.device)
    _check("moe_rmsnorm_bf16", lib().moe_rmsnorm_bf16(_p(r), T, H, ctypes.c_float(eps), _p(u), _stream()))
    return u


def router_topk(x: torch.Tensor, Wr: torch.Tensor, bias: Optional[torch.Tensor], k: int, ws: Workspace,
                want_logits: bool = False):
    T, H = x.shape
    E = Wr.shape[0]
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    logits = torch.empty(T, E, dtype=torch.float32, device=x.device) if want_logits else None
    _check("moe_router_topk", lib().moe_router_topk(_p(x), T, H, _p(Wr), _p(bias), E, k, _p(idx), _p(w), _p(logits),
                                                    ws.ptr, ws.size, _stream()))
    return (idx, w, logits) if want_logits else (idx, w)


def router_topk_static(x: torch.Tensor, Wr: torch.Tensor, bias: Optional[torch.Tensor], k: int,
                       want_logits: bool = False):
    """moe_router_topk_static: the same routing without a workspace (fixed scratch inside the library)."""
    T, H = x.shape
    E = Wr.shape[0]
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    logits = torch.empty(T, E, dtype=torch.float32, device=x.device) if want_logits else None
    _check("moe_router_topk_static", lib().moe_router_topk_static(_p(x), T, H, _p(Wr), _p(bias), E, k, _p(idx),
                                                                  _p(w), _p(logits), _stream()))
    return (idx, w, logits) if want_logits else (idx, w)


def permute(idx: torch.Tensor, E: int, x: torch.Tensor, with_shared: bool, ws: Workspace):
    T, k = idx.shape
    H = x.shape[1]
    rows = T * k + (T if with_shared else 0)
    dev = x.device
    counts = torch.empty(E + 1, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 2, dtype=torch.int32, device=dev)
    row_of = torch.empty(T, k, dtype=torch.int32, device=dev)
    src = torch.empty(max(rows, 1), dtype=torch.int32, device=dev)
    x_perm = torch.empty(max(rows, 1), H, dtype=torch.float16, device=dev)
    _check("moe_permute", lib().moe_permute(_p(idx), T, k, E, _p(x), H, 1 if with_shared else 0, _p(counts),
                                            _p(offsets), _p(row_of), _p(src), _p(x_perm), ws.ptr, ws.size, _stream()))
    return dict(counts=counts, offsets=offsets, row_of=row_of, src=src[:rows], x_perm=x_perm[:rows])


def expert_ffn(x_perm: torch.Tensor, offsets: torch.Tensor, E: int, routed, shared, ws: Workspace,
               path: int = PATH_AUTO) -> torch.Tensor:
    n_rows, H = x_perm.shape
    I = routed.gate.rows
    out = torch.empty(max(n_rows, 1), H, dtype=torch.float16, device=x_perm.device)
    rs = expert_set(routed)
    ss = expert_set(shared) if shared is not None else None
    _check("moe_expert_ffn", lib().moe_expert_ffn(_p(x_perm), _p(offsets), n_rows, E, H, I, ctypes.byref(rs),
                                                  ctypes.byref(ss) if ss is not None else None, _p(out), path,
                                                  ws.ptr, ws.size, _stream()))
    return out[:n_rows]


def combine(out_perm: torch.Tensor, row_of: torch.Tensor, w: torch.Tensor, shared_out: Optional[torch.Tensor] = None,
            residual: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, k = row_of.shape
    H = out_perm.shape[1]
    y = torch.empty(T, H, dtype=torch.float32, device=out_perm.device)
    _check("moe_combine", lib().moe_combine(_p(out_perm), _p(row_of), _p(w), T, k, H, _p(shared_out), _p(residual),
                                            _p(y), _stream()))
    return y


def layer_forward(x: torch.Tensor, Wr: torch.Tensor, bias: Optional[torch.Tensor], routed, shared, k: int,
                  ws: Workspace, residual: Optional[torch.Tensor] = None, path: int = PATH_AUTO,
                  y: Optional[torch.Tensor] = None, want_routing: bool = False):
    T, H = x.shape
    E = Wr.shape[0]
    I = routed.gate.rows
    d = layer_desc(H, E, k, I, shared is not None)
    if y is None:
        y = torch.empty(T, H, dtype=torch.float32, device=x.device)
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device) if want_routing else None
    w = torch.empty(T, k, dtype=torch.float32, device=x.device) if want_routing else None
    rs = expert_set(routed)
    ss = expert_set(shared) if shared is not None else None
    _check("moe_layer_forward", lib().moe_layer_forward(
        _p(x), T, _p(Wr), _p(bias), ctypes.byref(d), ctypes.byref(rs), ctypes.byref(ss) if ss is not None else None,
        _p(residual), _p(y), _p(idx), _p(w), path, ws.ptr, ws.size, _stream()))
    return (y, idx, w) if want_routing else y


class Stack:
    """Per-layer pointer arrays for moe_stack_forward (kept alive with the tensors they point to)."""

    def __init__(self, Wrs: Sequence[torch.Tensor], biases, routed: Sequence, shared: Optional[Sequence], k: int):
        self.L = len(Wrs)
        self.Wrs, self.biases, self.routed_py, self.shared_py = list(Wrs), biases, list(routed), shared
        self.H = Wrs[0].shape[1]
        self.E = Wrs[0].shape[0]
        self.I = routed[0].gate.rows
        self.k = k
        self.desc = layer_desc(self.H, self.E, k, self.I, shared is not None)
        self.wr_arr = (ctypes.c_void_p * self.L)(*[w.data_ptr() for w in Wrs])
        self.b_arr = None
        if biases is not None:
            self.b_arr = (ctypes.c_void_p * self.L)(*[None if b is None else b.data_ptr() for b in biases])
        self.r_arr = (ExpertSet * self.L)(*[expert_set(r) for r in routed])
        self.s_arr = (ExpertSet * self.L)(*[expert_set(s) for s in shared]) if shared is not None else None


def stack_forward(r_in: torch.Tensor, stack: Stack, ws: Workspace, eps: float = 1e-6, path: int = PATH_AUTO,
                  r_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, H = r_in.shape
    if r_out is None:
        r_out = torch.empty_like(r_in)
    _check("moe_stack_forward", lib().moe_stack_forward(
        _p(r_in), T, stack.L, stack.wr_arr, stack.b_arr, ctypes.byref(stack.desc), stack.r_arr, stack.s_arr,
        ctypes.c_float(eps), _p(r_out), path, ws.ptr, ws.size, _stream()))
    return r_out


def stack_forward_host(r_in_host: torch.Tensor, stack: Stack, ws: Workspace, eps: float = 1e-6,
                       path: int = PATH_AUTO, r_out_host: Optional[torch.Tensor] = None) -> torch.Tensor:
    """moe_stack_forward_host: the residual stream in host memory (page-locked for asynchronous
    copies); r_out_host may be r_in_host."""
    T, H = r_in_host.shape
    if r_out_host is None:
        r_out_host = torch.empty_like(r_in_host)
    _check("moe_stack_forward_host", lib().moe_stack_forward_host(
        _p(r_in_host), T, stack.L, stack.wr_arr, stack.b_arr, ctypes.byref(stack.desc), stack.r_arr, stack.s_arr,
        ctypes.c_float(eps), _p(r_out_host), path, ws.ptr, ws.size, _stream()))
    return r_out_host


def dequant_rows(m, expert: int, row0: int, nrows: int):
    """(fp32 [nrows,K], fp16 [nrows,K]) dequantized rows of one expert, computed on the GPU."""
    q = qmat(m)
    dev = m.codes.device
    f32 = torch.empty(nrows, m.K, dtype=torch.float32, device=dev)
    f16 = torch.empty(nrows, m.K, dtype=torch.float16, device=dev)
    _check("moe_dequant_rows", lib().moe_dequant_rows(ctypes.byref(q), expert, row0, nrows, _p(f32), _p(f16),
                                                      _stream()))
    return f32, f16


def test_wait_timeout(ws: Workspace, limit_ms: int = 50):
    """moe_test_wait_timeout: make the fused kernel's logit-exchange wait poll for a tag that no
    launch writes; the wait gives up after limit_ms and MOE_ERR_TIMEOUT lands in the workspace error
    word."""
    _check("moe_test_wait_timeout", lib().moe_test_wait_timeout(ws.ptr, ws.size, int(limit_ms), _stream()))


def read_device_error(ws: Workspace) -> int:
    code = ctypes.c_int32(0)
    _check("moe_read_device_error", lib().moe_read_device_error(ws.ptr, ctypes.byref(code), _stream()))
    return int(code.value)


# ----------------------------------------------------------------------------- per-kernel timing
def timing_enable(on: bool = True):
    _check("moe_timing_enable", lib().moe_timing_enable(1 if on else 0))


def kernel_names():
    return [lib().moe_kernel_name(i).decode() for i in range(lib().moe_kernel_count())]


def timing_read() -> dict:
    """{kernel name: (total device ms, launches)} for kernels launched while timing was enabled."""
    out = {}
    for i, n in enumerate(kernel_names()):
        ms = ctypes.c_double(0.0)
        cnt = ctypes.c_int32(0)
        _check("moe_timing_read", lib().moe_timing_read(i, ctypes.byref(ms), ctypes.byref(cnt)))
        if cnt.value:
            out[n] = (ms.value, cnt.value)
    return out


# ----------------------------------------------------------------------------- low-overhead layer handle
class LayerHandle:
    """A layer's weights bound once: descriptor and weight-plane structs are built at construction, so
    each forward() is a single C call with plain integer arguments (suitable for CUDA-graph capture
    and for tight decode loops)."""

    _fast = None
    _fast_host = None

    def __init__(self, Wr: torch.Tensor, bias: Optional[torch.Tensor], routed, shared, k: int, ws: Workspace):
        L = lib()
        if LayerHandle._fast is None:
            vp, i32 = ctypes.c_void_p, ctypes.c_int32
            proto = ctypes.CFUNCTYPE(i32, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, ctypes.c_size_t, vp)
            LayerHandle._fast = proto(("moe_layer_forward", L))
            proto_h = ctypes.CFUNCTYPE(i32, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, ctypes.c_size_t, vp)
            LayerHandle._fast_host = proto_h(("moe_layer_forward_host", L))
        self.refs = (Wr, bias, routed, shared, ws)  # keep the tensors alive
        self.H, self.E, self.k, self.I = Wr.shape[1], Wr.shape[0], k, routed.gate.rows
        self.desc = layer_desc(self.H, self.E, k, self.I, shared is not None)
        self.rs = expert_set(routed)
        self.ss = expert_set(shared) if shared is not None else None
        self._a = (Wr.data_ptr(), None if bias is None else bias.data_ptr(), ctypes.addressof(self.desc),
                   ctypes.addressof(self.rs), None if self.ss is None else ctypes.addressof(self.ss))
        self._ws = (ws.buf.data_ptr(), ws.nbytes)
        self._dev = Wr.device.index if Wr.device.index is not None else torch.cuda.current_device()
        self._fn = LayerHandle._fast

    def forward(self, x: torch.Tensor, y: torch.Tensor, residual: Optional[torch.Tensor] = None,
                idx_out: Optional[torch.Tensor] = None, w_out: Optional[torch.Tensor] = None, path: int = PATH_AUTO):
        wr, b, d, rs, ss = self._a
        code = self._fn(x.data_ptr(), x.shape[0], wr, b, d, rs, ss,
                        None if residual is None else residual.data_ptr(), y.data_ptr(),
                        None if idx_out is None else idx_out.data_ptr(), None if w_out is None else w_out.data_ptr(),
                        path, self._ws[0], self._ws[1], _raw_stream(self._dev))
        if code != MOE_OK:
            raise MoeError("moe_layer_forward", code)
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, idx_out: Optional[torch.Tensor] = None,
                     w_out: Optional[torch.Tensor] = None, path: int = PATH_AUTO):
        """moe_layer_forward_host: x and y in host memory (page-locked for asynchronous copies); the
        copies and the layer are enqueued on the current stream by one C call."""
        wr, b, d, rs, ss = self._a
        code = LayerHandle._fast_host(x_host.data_ptr(), x_host.shape[0], wr, b, d, rs, ss, y_host.data_ptr(),
                                      None if idx_out is None else idx_out.data_ptr(),
                                      None if w_out is None else w_out.data_ptr(), path, self._ws[0], self._ws[1],
                                      _raw_stream(self._dev))
        if code != MOE_OK:
            raise MoeError("moe_layer_forward_host", code)
        return y_host
