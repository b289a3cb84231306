"""Exact logit ties on every GPU top-k path: the lower expert index must win, bit for bit.

The routing rule is "top-k by logit, ties broken by lower index". With random router weights
exact ties do not occur, and at an exact tie the oracle's k-th minus (k+1)-th gap is 0, which
the near-tie allowance of the other parity tests would accept whatever the GPU picked. So the
inputs here are built to tie exactly, and the GPU's indices must equal the oracle's with no
allowance at all:

  * groups of three experts share one router row and one bias value, so their logits are equal
    whatever the token (each path computes a logit by the same arithmetic for every expert);
  * the tied experts' indices are scattered (not adjacent, not in ascending position within a
    group, across 32-expert chunks and across the CTAs that compute logits), and a +10 bias
    lifts four groups (twelve experts) above all others, so with k = 10 the top three groups
    fill nine slots and the tenth slot must go to the lowest index of the fourth group;
  * a second construction makes rows that differ only in columns where every token's x is
    zero, which also gives equal logits without equal rows.

Paths: the fused one-kernel decode layer (1 and 4 tokens), the single-kernel decode router
(router_topk at 1..8 tokens, and the layer's GEMV path), the small-batch router (9..128 tokens)
with its top-k kernel, and the tensor-core router with its exact refine (more than 128 tokens).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_ffn_gemm_b200 as moe
import synth
from tests.gpu_util import W_TOL, check_layer, to_dev

pytestmark = pytest.mark.gpu

H, E, K, I = 2048, 512, 10, 128
GROUPS = [(417, 33, 250), (5, 300, 129), (480, 64, 199), (96, 351, 2)]   # first member: the shared row


def _tied_router(masked: bool):
    """(Wr fp32 [E,H], bias fp32 [E], zero_cols) with four tied groups lifted by the bias."""
    Wr = synth.make_router(11, 0, E, H).numpy().copy()
    bias = np.zeros(E, np.float32)
    zero_cols = np.arange(7, H, 97) if masked else np.zeros(0, np.int64)
    rng = np.random.default_rng(12)
    for g in GROUPS:
        for e in g[1:]:
            Wr[e] = Wr[g[0]]
            if masked:  # differ only where every token's x is zero
                Wr[e, zero_cols] = rng.normal(0, 0.05, zero_cols.size).astype(np.float32)
        for e in g:
            bias[e] = 10.0
    return torch.from_numpy(Wr), torch.from_numpy(bias), zero_cols


def _tokens(T, zero_cols, stream):
    x = synth.make_x(11, T, H, stream=stream).clone()
    if zero_cols.size:
        x[:, torch.from_numpy(zero_cols)] = 0
    return x


def _oracle_routing(x, Wr, bias):
    idx, w, logits, gap = oracle.router_topk(x, Wr, bias, K)
    # the construction really ties at the k-th slot: the tenth and eleventh logits are equal,
    # and the tenth slot holds the lowest index of its group
    assert (gap == 0.0).all()
    for t in range(idx.shape[0]):
        grp = next(g for g in GROUPS if idx[t, 9] in g)
        assert idx[t, 9] == min(grp)
    return idx, w


def _check(idx, w, idx_ref, w_ref):
    idx = idx.cpu().numpy()
    assert np.array_equal(idx, idx_ref), np.argwhere(idx != idx_ref)[:8]
    assert np.abs(w.cpu().numpy().astype(np.float64) - w_ref).max() <= W_TOL


_dev = {}


def _setup(masked):
    if masked not in _dev:
        Wr, bias, zc = _tied_router(masked)
        routed = synth.make_expert_set(11, 0, synth.SET_ROUTED, synth.Q2, E, H, I, device="cuda")
        shared = synth.make_expert_set(11, 0, synth.SET_SHARED, synth.Q2, 1, H, I, device="cuda")
        _dev[masked] = (Wr, bias, zc, Wr.cuda(), bias.cuda(), routed, shared)
    return _dev[masked]


@pytest.mark.parametrize("masked", [False, True])
@pytest.mark.parametrize("T", [1, 3, 8, 12, 100, 300, 2048])
def test_router_exact_ties_lower_index_wins(T, masked):
    Wr, bias, zc, Wr_d, b_d, _, _ = _setup(masked)
    x = _tokens(T, zc, stream=T)
    idx_ref, w_ref = _oracle_routing(x, Wr, bias)
    ws = moe.Workspace.for_layer(H, E, K, I, True, T)
    idx, w = moe.router_topk(x.cuda(), Wr_d, b_d, K, ws)
    assert moe.read_device_error(ws) == 0
    _check(idx, w, idx_ref, w_ref)


@pytest.mark.parametrize("masked", [False, True])
@pytest.mark.parametrize("T,path", [(1, moe.PATH_AUTO), (4, moe.PATH_AUTO), (4, moe.PATH_GEMV),
                                    (16, moe.PATH_AUTO)])
def test_layer_routing_exact_ties_lower_index_wins(T, path, masked):
    # AUTO at 1 and 4 tokens: the fused decode kernel's own top-k; GEMV: the decode router that
    # also builds the expert units; 16 tokens: the small-batch router before the grouped GEMM
    Wr, bias, zc, Wr_d, b_d, routed, shared = _setup(masked)
    x = _tokens(T, zc, stream=100 + T)
    idx_ref, w_ref = _oracle_routing(x, Wr, bias)
    ws = moe.Workspace.for_layer(H, E, K, I, True, T)
    _, idx, w = moe.layer_forward(x.cuda(), Wr_d, b_d, routed, shared, K, ws, path=path, want_routing=True)
    assert moe.read_device_error(ws) == 0
    _check(idx, w, idx_ref, w_ref)


@pytest.mark.parametrize("T", [1, 4, 12, 300])
def test_all_logits_equal_take_the_lowest_indices(T):
    # a zero router makes every logit 0: each token must take experts 0..k-1 in that order with
    # equal weights 1/k (more tied candidates than one warp holds: the paths' fallbacks run)
    _, _, _, _, _, routed, shared = _setup(False)
    Wr0 = torch.zeros(E, H, dtype=torch.float32, device="cuda")
    x = _tokens(T, np.zeros(0, np.int64), stream=200 + T)
    idx_ref, w_ref, _, gap = oracle.router_topk(x, Wr0.cpu(), None, K)
    assert (gap == 0).all() and (idx_ref == np.arange(K)).all()
    ws = moe.Workspace.for_layer(H, E, K, I, True, T)
    idx, w = moe.router_topk(x.cuda(), Wr0, None, K, ws)
    _check(idx, w, idx_ref, w_ref)
    if T <= 4:  # the fused decode kernel's own top-k
        _, idx, w = moe.layer_forward(x.cuda(), Wr0, None, routed, shared, K, ws, want_routing=True)
        _check(idx, w, idx_ref, w_ref)
    assert moe.read_device_error(ws) == 0


@pytest.mark.parametrize("E", [33, 40, 97])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_fused_topk_with_a_partial_last_chunk(E, T):
    # E not a multiple of 32: the last 32-expert chunk is partial, so some chunks hold fewer valid
    # experts than the chunk tops they contribute (at E = 33, k = 10: five tops from a 1-expert
    # chunk) and the threshold must fall to 0 with more candidates than one warp holds; the fused
    # decode kernel's routing and y still match the oracle
    s = synth.LayerShape(f"partial{E}", T, 256, E, 10, 128, synth.Q2, True, 1.1, seed=21)
    L = synth.make_layer(s)
    x, Wr, b, routed, shared = to_dev(L)
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, True, T)
    y, idx, w = moe.layer_forward(x, Wr, b, routed, shared, s.k, ws, want_routing=True)
    assert moe.read_device_error(ws) == 0
    check_layer(y.cpu().numpy(), idx.cpu().numpy(), L, range(T), w_gpu=w.cpu().numpy())
