"""Test-side packer for the Q2/Q3 block planes, written from the layout definition in
include/moe_ffn.h, and for the Q4 plane from its stated layout (4-bit codes; per 32-weight block
four 32-bit words, word q holding weight 8q+2i+h at bits 16h+4i), independently of the oracle's
and the CUDA library's decoders.

Used to build weights whose integer codes the test knows, so a decoder can be checked against
values that never went through it.
"""
import numpy as np


def pack_lo_plane(codes: np.ndarray) -> np.ndarray:
    """codes int [..., K] (values 0..3 after masking) -> uint8 [..., K/4] 2-bit plane.
    word q of a block holds weight 16q+2i+h at bits 16h+2i."""
    c = np.asarray(codes, np.int64) & 3
    *lead, K = c.shape
    assert K % 32 == 0
    c = c.reshape(*lead, K // 16, 8, 2)          # [..., word, i, h]
    shifts = (16 * np.arange(2)[None, :] + 2 * np.arange(8)[:, None])  # [i, h]
    words = (c << shifts).sum(axis=(-2, -1)).astype(np.uint32)  # [..., K/16]
    return words.view(np.uint8).reshape(*lead, K // 4)


def pack_hi_plane(codes: np.ndarray) -> np.ndarray:
    """codes int [..., K] (values 0..7) -> uint8 [..., K/8]; one word per block,
    bit 2 of weight 16q+2i+h at bit 16h+8q+i."""
    c = (np.asarray(codes, np.int64) >> 2) & 1
    *lead, K = c.shape
    c = c.reshape(*lead, K // 32, 2, 8, 2)       # [..., block, q, i, h]
    q = np.arange(2)[:, None, None]
    i = np.arange(8)[None, :, None]
    h = np.arange(2)[None, None, :]
    shifts = 16 * h + 8 * q + i
    words = (c << shifts).sum(axis=(-3, -2, -1)).astype(np.uint32)  # [..., K/32]
    return words.view(np.uint8).reshape(*lead, K // 8)


def pack_q4_plane(codes: np.ndarray) -> np.ndarray:
    """codes int [..., K] (values 0..15) -> uint8 [..., K/2] 4-bit plane; per block four words,
    word q holds weight 8q+2i+h at bits 16h+4i."""
    c = np.asarray(codes, np.int64) & 15
    *lead, K = c.shape
    assert K % 32 == 0
    c = c.reshape(*lead, K // 8, 4, 2)           # [..., word, i, h]
    shifts = (16 * np.arange(2)[None, :] + 4 * np.arange(4)[:, None])  # [i, h]
    words = (c << shifts).sum(axis=(-2, -1)).astype(np.uint32)  # [..., K/8]
    return words.view(np.uint8).reshape(*lead, K // 2)


class KnownQMat:
    """A QMat-like object built from known integer codes and fp16 scales."""

    def __init__(self, qtype, codes, scales_f16):
        codes = np.asarray(codes, np.int64)
        self.qtype = qtype
        self.n, self.rows, self.K = codes.shape
        self.int_codes = codes
        self.codes = pack_q4_plane(codes) if qtype == 4 else pack_lo_plane(codes)
        self.hibits = pack_hi_plane(codes) if qtype == 3 else None
        self.scales = np.asarray(scales_f16, np.float16).view(np.uint16)
        assert self.scales.shape == (self.n, self.rows, self.K // 32)

    def dense(self) -> np.ndarray:
        """fp64 weights [n, rows, K] = d * (c - q0), from the known codes (no decoding)."""
        q0 = {2: 2, 3: 4, 4: 8}[self.qtype]
        d = self.scales.view(np.float16).astype(np.float64)
        return np.repeat(d, 32, axis=-1) * (self.int_codes - q0)


class KnownSet:
    def __init__(self, gate, up, down):
        self.gate, self.up, self.down = gate, up, down


def random_known_set(rng, qtype, n, H, I, scale_range=(0.005, 0.02)):
    cmax = {2: 4, 3: 8, 4: 16}[qtype]

    def mat(rows, K):
        codes = rng.integers(0, cmax, size=(n, rows, K))
        sc = rng.uniform(*scale_range, size=(n, rows, K // 32)).astype(np.float16)
        return KnownQMat(qtype, codes, sc)

    return KnownSet(mat(I, H), mat(I, H), mat(H, I))


def silu(z):
    return z / (1.0 + np.exp(-z))


def dense_ffn(ks: KnownSet, e: int, x: np.ndarray) -> np.ndarray:
    """Textbook SwiGLU FFN with the known dense weights of expert e: x [n,H] -> [n,H] (fp64)."""
    Wg = ks.gate.dense()[e]
    Wu = ks.up.dense()[e]
    Wd = ks.down.dense()[e]
    h = silu(x @ Wg.T) * (x @ Wu.T)
    return h @ Wd.T
