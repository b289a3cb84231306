"""Seeded synthetic inputs for the quantized MoE layer (shared by the oracle and the CUDA path).

This module holds no arithmetic of the method. It only draws inputs: activations, router
weights, per-expert router biases and packed Q2/Q3/Q4 expert weights, each from one
counter-based generator, so any slice (one expert, one token) can be regenerated alone and
the bits do not depend on the device or on the number of threads.

Generator (counter-based, splitmix64 finaliser):
    mix(z)   = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
    key      = mix(mix(seed + GAMMA) ^ tid)          (GAMMA = 0x9E3779B97F4A7C15, all mod 2^64)
    word[i]  = mix(key + (i + 1) * GAMMA)
Derived draws:
    uniform  u = (word >> 40) * 2^-24                  (24 bits, exact in fp32)
    normal   z = sqrt(-2 ln u1) cos(2 pi u2) in fp64, u1 = ((w[2i] >> 11) + 1) 2^-53, u2 = (w[2i+1] >> 11) 2^-53
    codes    the bytes of consecutive words, little-endian (uniform codes in every bit field)
    scale    d = fp16_rne(fp32(fp32(u * 0.015f) + 0.005f))   i.e. U(0.005, 0.02) rounded to fp16

Integer and single-rounding fp32 steps give identical bits on CPU and CUDA, so packed codes and
scales may be drawn on the GPU; normals (transcendentals) are always drawn on the CPU.

The workload recipes (shapes and distributions) follow the workload the pages describe:
512 routed experts with 10 active per token over 48 layers ("Strata vs Llama.cpp vs vLLM",
chapter "How Strata is designed to work"), 8,192-token prefill chunks (same chapter;
"Local AI Is Now 6x Faster on Your PC", "Prompt length and reading pipeline improvements"),
1-4 token decode / MTP-verify passes (Strata DETAILS.md, "How it works").
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

# tensor-id kinds
K_X = 1
K_ROUTER_W = 2
K_ROUTER_PERM = 3
K_CODES = 4
K_HIBITS = 5
K_SCALES = 6
K_RESID = 7

MAT_GATE, MAT_UP, MAT_DOWN = 0, 1, 2
SET_ROUTED, SET_SHARED = 0, 1

Q2, Q3, Q4 = 2, 3, 4


def tid(kind: int, layer: int = 0, mat: int = 0, index: int = 0) -> int:
    """Tensor id: one independent counter stream per (kind, layer, matrix, index)."""
    return (kind << 48) | (layer << 32) | (mat << 24) | index


# ----------------------------------------------------------------------------- scalar reference
def mix_int(z: int) -> int:
    """splitmix64 finaliser on Python ints (mod 2^64)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, t: int) -> int:
    return mix_int(mix_int((seed + GAMMA) & _MASK64) ^ (t & _MASK64))


def word_int(seed: int, t: int, i: int) -> int:
    return mix_int((stream_key(seed, t) + (i + 1) * GAMMA) & _MASK64)


# ----------------------------------------------------------------------------- vectorised (torch int64)
def _s64(c: int) -> int:
    c &= _MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    # logical shift right of int64 viewed as uint64
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(_M1)
    z = (z ^ _srl(z, 27)) * _s64(_M2)
    return z ^ _srl(z, 31)


def words(seed: int, tids, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """int64 words [len(tids), n] (or [n] for a scalar tid): word[j, i] = mix(key_j + (start+i+1)*GAMMA)."""
    scalar = isinstance(tids, int)
    tl = [tids] if scalar else list(tids)
    keys = torch.tensor([_s64(stream_key(seed, t)) for t in tl], dtype=torch.int64, device=device)
    ctr = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device) * _s64(GAMMA)
    out = _mix(keys[:, None] + ctr[None, :])
    return out[0] if scalar else out


def uniform24(w: torch.Tensor) -> torch.Tensor:
    """fp32 uniform on [0,1) with 24 random bits (exact)."""
    return _srl(w, 40).to(torch.float32) * (2.0 ** -24)


def normal_f64(seed: int, t: int, n: int) -> torch.Tensor:
    """n standard normals in fp64, Box-Muller, drawn on the CPU."""
    w = words(seed, t, 2 * n, "cpu")
    u1 = (_srl(w[0::2], 11).to(torch.float64) + 1.0) * (2.0 ** -53)
    u2 = _srl(w[1::2], 11).to(torch.float64) * (2.0 ** -53)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def random_bytes(seed: int, tids, nbytes: int, device="cpu") -> torch.Tensor:
    """uint8 [len(tids), nbytes]: little-endian bytes of consecutive words."""
    nw = (nbytes + 7) // 8
    w = words(seed, tids, nw, device)
    b = w.contiguous().view(torch.uint8)
    return b[..., :nbytes]


def scales_f16(seed: int, tids, n: int, device="cpu", lo: float = 0.005, hi: float = 0.02) -> torch.Tensor:
    """fp16 [len(tids), n]: U(lo, hi) drawn in fp32 then rounded to fp16 (RNE)."""
    u = uniform24(words(seed, tids, n, device))
    d = (u * (hi - lo)) + lo  # two separately rounded fp32 ops
    return d.to(torch.float16)


# ----------------------------------------------------------------------------- packed weights
@dataclass
class QMat:
    """One matrix kind (gate, up or down) for n experts: rows output features, K reduction dim.

    codes  uint8 [n, rows, K/4]   2-bit plane (Q2 codes, or the low 2 bits of Q3 codes);
                                  Q4: [n, rows, K/2], the 4-bit codes
    hibits uint8 [n, rows, K/8]   Q3 only: bit 2 of each code; None for Q2
    scales fp16  [n, rows, K/32]  one scale per block of 32 weights along K
    """
    qtype: int
    n: int
    rows: int
    K: int
    codes: torch.Tensor
    hibits: Optional[torch.Tensor]
    scales: torch.Tensor

    def to(self, device) -> "QMat":
        return QMat(self.qtype, self.n, self.rows, self.K, self.codes.to(device),
                    None if self.hibits is None else self.hibits.to(device), self.scales.to(device))

    def expert(self, e: int) -> "QMat":
        return QMat(self.qtype, 1, self.rows, self.K, self.codes[e:e + 1],
                    None if self.hibits is None else self.hibits[e:e + 1], self.scales[e:e + 1])

    @property
    def nbytes(self) -> int:
        b = self.codes.numel() + 2 * self.scales.numel()
        return b + (0 if self.hibits is None else self.hibits.numel())


@dataclass
class ExpertSet:
    gate: QMat
    up: QMat
    down: QMat

    def to(self, device) -> "ExpertSet":
        return ExpertSet(self.gate.to(device), self.up.to(device), self.down.to(device))

    def expert(self, e: int) -> "ExpertSet":
        return ExpertSet(self.gate.expert(e), self.up.expert(e), self.down.expert(e))

    @property
    def nbytes(self) -> int:
        return self.gate.nbytes + self.up.nbytes + self.down.nbytes


def make_qmat(seed: int, layer: int, set_id: int, mat: int, qtype: int, n: int, rows: int, K: int,
              device="cpu", experts=None) -> QMat:
    """Packed weights of experts `experts` (default 0..n-1); codes uniform, d ~ U(0.005, 0.02)."""
    assert K % 32 == 0 and qtype in (Q2, Q3, Q4)
    ex = list(range(n)) if experts is None else list(experts)
    m = set_id * 3 + mat
    cb = K // 2 if qtype == Q4 else K // 4  # bytes of the code plane per row (4-bit or 2-bit codes)
    codes = random_bytes(seed, [tid(K_CODES, layer, m, e) for e in ex], rows * cb, device)
    codes = codes.reshape(len(ex), rows, cb)
    hib = None
    if qtype == Q3:
        hib = random_bytes(seed, [tid(K_HIBITS, layer, m, e) for e in ex], rows * K // 8, device)
        hib = hib.reshape(len(ex), rows, K // 8)
    sc = scales_f16(seed, [tid(K_SCALES, layer, m, e) for e in ex], rows * K // 32, device)
    sc = sc.reshape(len(ex), rows, K // 32)
    return QMat(qtype, len(ex), rows, K, codes.contiguous(),
                None if hib is None else hib.contiguous(), sc.contiguous())


def make_expert_set(seed: int, layer: int, set_id: int, qtype: int, n: int, H: int, I: int,
                    device="cpu", experts=None) -> ExpertSet:
    return ExpertSet(make_qmat(seed, layer, set_id, MAT_GATE, qtype, n, I, H, device, experts),
                     make_qmat(seed, layer, set_id, MAT_UP, qtype, n, I, H, device, experts),
                     make_qmat(seed, layer, set_id, MAT_DOWN, qtype, n, H, I, device, experts))


def make_x(seed: int, T: int, H: int, stream: int = 0) -> torch.Tensor:
    """Activations x[T,H] ~ N(0,1) rounded to bf16 (via fp32). `stream` selects an independent batch."""
    z = normal_f64(seed, tid(K_X, 0, 0, stream), T * H)
    return z.to(torch.float32).to(torch.bfloat16).reshape(T, H)


def make_residual(seed: int, T: int, H: int, stream: int = 0) -> torch.Tensor:
    """fp32 residual stream r[T,H] ~ N(0,1) (input of a stack of layers)."""
    z = normal_f64(seed, tid(K_RESID, 0, 0, stream), T * H)
    return z.to(torch.float32).reshape(T, H)


def make_router(seed: int, layer: int, E: int, H: int, sigma: float = 0.02) -> torch.Tensor:
    """Router weights Wr[E,H] ~ N(0, sigma) in fp32."""
    z = normal_f64(seed, tid(K_ROUTER_W, layer), E * H) * sigma
    return z.to(torch.float32).reshape(E, H)


def zipf_bias(seed: int, layer: int, E: int, s: float) -> torch.Tensor:
    """Per-expert router bias b_e = -s ln(rank_e), rank = 1 + a seeded permutation of 0..E-1 (fp32)."""
    w = words(seed, tid(K_ROUTER_PERM, layer), E, "cpu")
    # order by the unsigned value of the word; rank of expert e = its position + 1
    key = w ^ _s64(1 << 63)  # flip the sign bit so signed order == unsigned order
    order = torch.argsort(key, stable=True)
    rank = torch.empty(E, dtype=torch.float64)
    rank[order] = torch.arange(1, E + 1, dtype=torch.float64)
    return (-s * torch.log(rank)).to(torch.float32)


# ----------------------------------------------------------------------------- workloads
@dataclass
class LayerShape:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    qtype: int
    shared: bool
    zipf_s: Optional[float]
    seed: int = 0


WORKLOADS = {
    # T=64, H=256, 16 experts, top-2, I=128, Q2, no shared expert, uniform router
    "tiny": LayerShape("tiny", 64, 256, 16, 2, 128, Q2, False, None),
    # decode step / MTP verify: T=1 or 4, Zipf(1.1) router bias, shared expert
    "decode1": LayerShape("decode1", 1, 2048, 512, 10, 512, Q2, True, 1.1),
    "decode4": LayerShape("decode4", 4, 2048, 512, 10, 512, Q2, True, 1.1),
    # verify pass over one token and five prompt-lookup drafts (T=6), same layer shape
    "verify6": LayerShape("verify6", 6, 2048, 512, 10, 512, Q2, True, 1.1),
    # pruned variant: 256 of the 512 experts kept per layer, otherwise the decode layer
    "decode1_pruned256": LayerShape("decode1_pruned256", 1, 2048, 256, 10, 512, Q2, True, 1.1),
    # prefill chunk: 8192 tokens, uniform router, shared expert
    "prefill8k": LayerShape("prefill8k", 8192, 2048, 512, 10, 512, Q2, True, None),
    # prefill with 3-bit weights and Zipf(1.2) skew, no shared expert
    "prefill2k_q3": LayerShape("prefill2k_q3", 2048, 2048, 512, 10, 512, Q3, False, 1.2),
    # the decode layer with 4-bit weights (the Q4 stand-in), otherwise decode1
    "decode1_q4": LayerShape("decode1_q4", 1, 2048, 512, 10, 512, Q4, True, 1.1),
    # a small batch of 32 tokens through the decode layer (between decode and prefill)
    "batch32": LayerShape("batch32", 32, 2048, 512, 10, 512, Q2, True, 1.1),
}

# 48-layer stack: RMSNorm (eps 1e-6) before each router, residual add, config-3 shaped layers
STACK = dict(L=48, H=2048, E=512, k=10, I=512, qtype=Q2, shared=True, eps=1e-6,
             prefill_T=8192, decode_steps=256)


@dataclass
class LayerInputs:
    shape: LayerShape
    x: torch.Tensor              # bf16 [T,H]
    Wr: torch.Tensor             # fp32 [E,H]
    bias: Optional[torch.Tensor]  # fp32 [E] or None
    routed: ExpertSet
    shared: Optional[ExpertSet]


def make_layer(shape: LayerShape, device="cpu", layer: int = 0, x_stream: int = 0) -> LayerInputs:
    s = shape
    x = make_x(s.seed, s.T, s.H, x_stream)
    Wr = make_router(s.seed, layer, s.E, s.H)
    bias = zipf_bias(s.seed, layer, s.E, s.zipf_s) if s.zipf_s else None
    routed = make_expert_set(s.seed, layer, SET_ROUTED, s.qtype, s.E, s.H, s.I, device)
    shared = make_expert_set(s.seed, layer, SET_SHARED, s.qtype, 1, s.H, s.I, device) if s.shared else None
    return LayerInputs(s, x.to(device), Wr.to(device), None if bias is None else bias.to(device), routed, shared)


def as_np_u16(t: torch.Tensor):
    """bf16/fp16 tensor -> numpy uint16 bit pattern (CPU)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
