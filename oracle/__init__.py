"""CPU oracle for the quantized MoE layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline / reference legs may import
this package. The product (the CUDA library and its Python binding) never imports, loads or
calls it, and it never imports the product.

The arithmetic lives in plain C (`moe_oracle.c`, fp64, one OpenMP thread per token); this
module only marshals numpy arrays through ctypes. Each function names the passage it follows:
  - routing 10 of 512 experts, shared experts: "Strata vs Llama.cpp vs vLLM", chapter
    "How Strata is designed to work"; Strata DETAILS.md, "How it works";
  - quantized expert matmul that dequantizes on the fly: "Two-Day Port, 8x Faster Prefill:
    Strata Engine Benchmarked", section "Where Strata Is Fast: Not Magic, but Logistics";
  - MTP verify passes give the same output as one-token passes: Strata DETAILS.md,
    "How it works" (speculation bullet);
  - Q2/Q3 block formats: the stated stand-in (32 weights, fp16 scale d, w = d(c-2) / d(c-4));
    Q4 (4-bit codes, w = d(c-8)) is a further stand-in of the same family.

Parity status: every function here is pinned by `tests/test_oracle_pins.py` against closed
forms, brute force and textbook/library routines (the pages print no worked example).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, OpenMP over tokens, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _QMat(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("rows", ctypes.c_int32),
                ("K", ctypes.c_int32), ("codes", ctypes.c_void_p), ("hibits", ctypes.c_void_p),
                ("scales", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_half_to_double.restype = ctypes.c_double
        _lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        _lib.oracle_bf16_to_double.restype = ctypes.c_double
        _lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        _lib.oracle_double_to_half.restype = ctypes.c_uint16
        _lib.oracle_double_to_half.argtypes = [ctypes.c_double]
        _lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        _lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        _lib.oracle_weight.restype = ctypes.c_double
        _lib.oracle_code.restype = ctypes.c_int
        _lib.oracle_max_threads.restype = ctypes.c_int
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# ----------------------------------------------------------------------------- marshalling
def _np(t, dtype=None):
    """torch tensor or array -> contiguous numpy array (bf16/fp16 tensors become uint16 bits)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype in (torch.bfloat16, torch.float16):
                t = t.view(torch.int16).numpy().view(np.uint16)
            else:
                t = t.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(t)
    if dtype is not None:
        assert a.dtype == np.dtype(dtype), (a.dtype, dtype)
    return a


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class QMatView:
    """Keeps the numpy arrays alive and exposes the C struct."""

    def __init__(self, qm):
        assert qm.qtype in (2, 3, 4), f"unknown block format {qm.qtype}"
        self.codes = _np(qm.codes, np.uint8)
        self.hibits = None if qm.hibits is None else _np(qm.hibits, np.uint8)
        self.scales = _np(qm.scales, np.uint16)
        # plane shapes: codes K/4 bytes per row (K/2 for the 4-bit plane), hi bits K/8 for Q3 only,
        # one scale per 32-weight block; a wrong shape would make the C decoder read past the array
        n, rows, K = int(qm.n), int(qm.rows), int(qm.K)
        assert K % 32 == 0 and self.codes.shape[-1] == (K // 2 if qm.qtype == 4 else K // 4)
        assert self.codes.size == n * rows * self.codes.shape[-1]
        assert (self.hibits is not None) == (qm.qtype == 3)
        if self.hibits is not None:
            assert self.hibits.shape[-1] == K // 8 and self.hibits.size == n * rows * K // 8
        assert self.scales.size == n * rows * K // 32
        self.s = _QMat(qm.qtype, qm.n, qm.rows, qm.K, _ptr(self.codes), _ptr(self.hibits), _ptr(self.scales))

    @property
    def ref(self):
        return ctypes.byref(self.s)


# ----------------------------------------------------------------------------- number formats
def half_to_double(bits: int) -> float:
    return lib().oracle_half_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def double_to_half(v: float) -> int:
    return int(lib().oracle_double_to_half(float(v)))


def double_to_bf16(v: float) -> int:
    return int(lib().oracle_double_to_bf16(float(v)))


# ----------------------------------------------------------------------------- dequant
def code(qm, e: int, r: int, k: int) -> int:
    v = QMatView(qm)
    return int(lib().oracle_code(v.ref, e, r, k))


def dequant_rows(qm, e: int, row0: int, nrows: int):
    """Rows of expert e: (exact fp64 values [nrows,K], fp16 bit patterns of the same values)."""
    v = QMatView(qm)
    out = np.zeros((nrows, qm.K), np.float64)
    o16 = np.zeros((nrows, qm.K), np.uint16)
    lib().oracle_dequant_rows(v.ref, ctypes.c_int(e), ctypes.c_int(row0), ctypes.c_int(nrows), _ptr(out), _ptr(o16))
    return out, o16


# ----------------------------------------------------------------------------- RMSNorm
def rmsnorm_bf16(r, eps: float = 1e-6) -> np.ndarray:
    """u = bf16(r / sqrt(mean(r^2) + eps)) -> uint16 bits [T,H]."""
    r = _np(r, np.float32)
    T, H = r.shape
    u = np.zeros((T, H), np.uint16)
    lib().oracle_rmsnorm_bf16(_ptr(r), T, H, ctypes.c_double(eps), _ptr(u))
    return u


# ----------------------------------------------------------------------------- router
def router_topk(x, Wr, bias, k: int, nthreads: int = 0):
    """fp64 logits = x Wr^T + bias, top-k (descending, lower index wins ties), softmax over the set.
    Returns idx int32 [T,k], w fp64 [T,k], logits fp64 [T,E], gap fp64 [T]."""
    x = _np(x, np.uint16)
    Wr = _np(Wr, np.float32)
    b = None if bias is None else _np(bias, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    logits = np.zeros((T, E), np.float64)
    gap = np.zeros(T, np.float64)
    lib().oracle_router_topk(_ptr(x), T, H, _ptr(Wr), _ptr(b), E, k, _ptr(idx), _ptr(w), _ptr(logits), _ptr(gap),
                             ctypes.c_int(nthreads))
    return idx, w, logits, gap


# ----------------------------------------------------------------------------- permute
def permute(idx, E: int):
    """Stable counting sort of (token, slot) pairs by expert -> counts, offsets, row_of, src."""
    idx = _np(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    row_of = np.zeros((T, k), np.int32)
    src = np.zeros(T * k, np.int32)
    lib().oracle_permute(_ptr(idx), T, k, E, _ptr(counts), _ptr(offsets), _ptr(row_of), _ptr(src))
    return counts, offsets, row_of, src


# ----------------------------------------------------------------------------- int8 activations
def quantize_blocks_i8(x):
    """int8 quantization of fp16 activation rows in 32-value blocks, the MMQ-style input format
    ("Two-Day Port, 8x Faster Prefill: Strata Engine Benchmarked", "Where Strata Is Fast": MMQ;
    "Strata vs Llama.cpp vs vLLM": int8 tensor-core kernels). Per row and block:
      amax = max |x|,  d = amax / 127,  q = clamp(rint(x * (127 / amax)), -127, 127)  (q = 0, d = 0 for
      an all-zero block),
    every step in fp32 (the precision the GPU decides the integers in), ties to even.
    x: fp16 bits or values [R, H] (H % 32 == 0). Returns (q int8 [R, H], d fp32 [R, H/32])."""
    xf = np.asarray(x)
    if xf.dtype == np.uint16:
        xf = xf.view(np.float16)
    xf = xf.astype(np.float32)
    R, H = xf.shape
    blocks = xf.reshape(R, H // 32, 32)
    amax = np.abs(blocks).max(axis=-1).astype(np.float32)
    d = (amax / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(127.0) / amax, np.float32(0.0)).astype(np.float32)
    prod = (blocks * inv[..., None]).astype(np.float32)
    q = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    return q.reshape(R, H), d


def dequantize_blocks_i8(q, d) -> np.ndarray:
    """The fp64 values q * d the int8 blocks stand for."""
    q = np.asarray(q, np.int64)
    R, H = q.shape
    return (q.reshape(R, H // 32, 32) * np.asarray(d, np.float64)[..., None]).reshape(R, H)


# ----------------------------------------------------------------------------- FFN / layer
def expert_ffn_rows(es, e: int, x: np.ndarray, mirrored: bool = False) -> np.ndarray:
    """One expert (gate/up/down of set `es`) applied to fp64 rows x[n,H]."""
    x = np.ascontiguousarray(x, np.float64)
    n, H = x.shape
    I = es.gate.rows
    g, u, d = QMatView(es.gate), QMatView(es.up), QMatView(es.down)
    out = np.zeros((n, H), np.float64)
    lib().oracle_expert_ffn_rows(g.ref, u.ref, d.ref, e, _ptr(x), n, H, I, _ptr(out), int(mirrored))
    return out


def layer_forward(x, Wr, bias, k: int, routed, shared=None, residual=None, forced_idx=None,
                  mirrored: bool = False, nthreads: int = 0):
    """y = sum_j w_j FFN_{e_j}(x) + FFN_shared(x) (+ residual), per token, fp64.
    Returns (y fp64 [T,H], idx int32 [T,k], w fp64 [T,k], gap fp64 [T])."""
    x = _np(x, np.uint16)
    Wr = _np(Wr, np.float32)
    b = None if bias is None else _np(bias, np.float32)
    res = None if residual is None else _np(residual, np.float32)
    fi = None if forced_idx is None else _np(forced_idx, np.int32)
    T, H = x.shape
    E = Wr.shape[0]
    I = routed.gate.rows
    rg, ru, rd = QMatView(routed.gate), QMatView(routed.up), QMatView(routed.down)
    if shared is not None:
        sg, su, sd = QMatView(shared.gate), QMatView(shared.up), QMatView(shared.down)
        sgr, sur, sdr = sg.ref, su.ref, sd.ref
    else:
        sgr = sur = sdr = None
    y = np.zeros((T, H), np.float64)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    gap = np.zeros(T, np.float64)
    lib().oracle_layer_forward(_ptr(x), T, H, _ptr(Wr), _ptr(b), E, k, I, rg.ref, ru.ref, rd.ref, sgr, sur, sdr,
                               _ptr(res), _ptr(fi), _ptr(y), _ptr(idx), _ptr(w), _ptr(gap), int(mirrored),
                               ctypes.c_int(nthreads))
    return y, idx, w, gap


def stack_forward(r0, layers, k: int, eps: float = 1e-6, nthreads: int = 0):
    """48-layer-style stack: r_{l+1} = r_l + layer_l(bf16(RMSNorm(r_l))), r kept in fp32 between layers.
    `layers` is a list of (Wr, bias, routed, shared). Returns the final r (fp32) and per-layer idx."""
    r = _np(r0, np.float32).copy()
    idxs = []
    for (Wr, bias, routed, shared) in layers:
        u = rmsnorm_bf16(r, eps)
        y, idx, _, _ = layer_forward(u, Wr, bias, k, routed, shared, residual=r, nthreads=nthreads)
        r = y.astype(np.float32)
        idxs.append(idx)
    return r, idxs
