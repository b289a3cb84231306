"""Helpers shared by the GPU parity tests: tolerance metric, routing comparison with the
near-tie rule, and moving synthetic layers to the device."""
import numpy as np
import torch

import oracle

Y_TOL = 1e-2        # max |y - y_ref| / rms(y_ref)
W_TOL = 1e-5        # routing weights, absolute
TIE_GAP = 1e-5      # oracle k-th minus (k+1)-th logit below which an index mismatch is allowed


def rel_err(y, y_ref) -> float:
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    return float(np.abs(y - y_ref).max() / np.sqrt((y_ref ** 2).mean()))


def to_dev(layer, device="cuda"):
    """(x, Wr, bias, routed, shared) of a synth.LayerInputs on the device."""
    return (layer.x.to(device), layer.Wr.to(device), None if layer.bias is None else layer.bias.to(device),
            layer.routed.to(device), None if layer.shared is None else layer.shared.to(device))


def _forced_weights(logits_ref_t, sel):
    """Softmax of the oracle's fp64 logits over a given selection, in the selection's slot order."""
    l = np.asarray(logits_ref_t, np.float64)[np.asarray(sel)]
    p = np.exp(l - l.max())
    return p / p.sum()


def compare_routing(idx, w, idx_ref, w_ref, gap_ref, logits_ref, log=None):
    """GPU routing against the oracle's, token by token.

    Indices must equal the oracle's bit for bit, slot order included. The only exception is an
    oracle near-tie: a token whose selected SET differs needs the oracle's k-th minus (k+1)-th
    logit gap below TIE_GAP, and every slot whose expert differs from the oracle's slot needs
    the two experts' oracle logits within TIE_GAP of each other (so a reordering inside the set
    is allowed only between near-equal logits). Such tokens are returned (and logged through
    `log` when given) for forced-routing checks of y.
    Weights (when `w` is given) must be within W_TOL of the oracle's for every token: of its own
    selection where the indices match, else of the softmax of the oracle's logits over the GPU's
    selection."""
    idx = np.asarray(idx)
    w = None if w is None else np.asarray(w, np.float64)
    flips = []
    for t in range(idx.shape[0]):
        if np.array_equal(idx[t], idx_ref[t]):
            if w is not None:
                assert np.abs(w[t] - w_ref[t]).max() <= W_TOL, (t, w[t], w_ref[t])
            continue
        lg = np.asarray(logits_ref[t], np.float64)
        if set(idx[t].tolist()) != set(idx_ref[t].tolist()):
            assert gap_ref[t] < TIE_GAP, ("selection differs without a near-tie", t, gap_ref[t])
        for j in range(idx.shape[1]):
            if idx[t, j] != idx_ref[t, j]:
                assert abs(lg[idx[t, j]] - lg[idx_ref[t, j]]) < TIE_GAP, ("slot differs without a near-tie", t, j)
        if w is not None:
            wf = _forced_weights(lg, idx[t])
            assert np.abs(w[t] - wf).max() <= W_TOL, (t, w[t], wf)
        if log is not None:
            log(f"near-tie token {t}: gpu {idx[t].tolist()} oracle {idx_ref[t].tolist()} gap {gap_ref[t]:.3e}")
        flips.append(t)
    return flips


def check_layer(y_gpu, idx_gpu, layer, tokens, residual=None, tol=Y_TOL, nthreads=0, w_gpu=None):
    """Oracle y for `tokens` against the GPU rows, and the GPU routing of those tokens against the
    oracle's (compare_routing: indices bit-exact except at logged near-ties, weights within
    W_TOL when `w_gpu` is given). Near-tie tokens are recomputed by the oracle with the GPU's
    selection (forced routing) before y is compared."""
    tokens = list(tokens)
    x = layer.x[tokens]
    res = None if residual is None else residual[tokens]
    k = idx_gpu.shape[1]
    y_ref, idx_ref, w_ref, gap = oracle.layer_forward(x, layer.Wr, layer.bias, k, layer.routed,
                                                      layer.shared, residual=res, nthreads=nthreads)
    _, _, lg_ref, _ = oracle.router_topk(x, layer.Wr, layer.bias, k, nthreads=nthreads)
    g_idx = np.asarray(idx_gpu)[tokens]
    g_w = None if w_gpu is None else np.asarray(w_gpu)[tokens]
    flips = compare_routing(g_idx, g_w, idx_ref, w_ref, gap, lg_ref, log=print)
    if flips:
        yf, _, _, _ = oracle.layer_forward(x[flips], layer.Wr, layer.bias, k, layer.routed,
                                           layer.shared, residual=None if res is None else res[flips],
                                           forced_idx=g_idx[flips], nthreads=nthreads)
        y_ref[flips] = yf
    err = rel_err(np.asarray(y_gpu)[tokens], y_ref)
    assert err <= tol, err
    return err, flips
