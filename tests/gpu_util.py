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


def compare_routing(idx, w, idx_ref, w_ref, gap_ref, logits_ref):
    """Indices must match exactly except where the oracle's logits are within TIE_GAP (a different
    set needs gap_ref < TIE_GAP; a different order inside the set needs the swapped logits within
    TIE_GAP). Weights must match within W_TOL wherever the selection matches.
    Returns the list of tokens whose selection differs (near-ties), for forced-routing checks."""
    idx = np.asarray(idx)
    w = np.asarray(w, np.float64)
    flips = []
    for t in range(idx.shape[0]):
        if np.array_equal(idx[t], idx_ref[t]):
            assert np.abs(w[t] - w_ref[t]).max() <= W_TOL, (t, w[t], w_ref[t])
            continue
        if set(idx[t].tolist()) == set(idx_ref[t].tolist()):
            # same set, order differs: every out-of-order slot pair must be an oracle near-tie
            lg = logits_ref[t]
            for j in range(idx.shape[1]):
                if idx[t, j] != idx_ref[t, j]:
                    assert abs(lg[idx[t, j]] - lg[idx_ref[t, j]]) < TIE_GAP, (t, j)
        else:
            assert gap_ref[t] < TIE_GAP, ("selection differs without a near-tie", t, gap_ref[t])
        flips.append(t)
    return flips


def check_layer(y_gpu, idx_gpu, layer, tokens, residual=None, tol=Y_TOL, nthreads=0):
    """Oracle y for `tokens` (with forced routing for near-tie tokens) against the GPU rows."""
    tokens = list(tokens)
    x = layer.x[tokens]
    res = None if residual is None else residual[tokens]
    y_ref, idx_ref, w_ref, gap = oracle.layer_forward(x, layer.Wr, layer.bias, idx_gpu.shape[1], layer.routed,
                                                      layer.shared, residual=res, nthreads=nthreads)
    g_idx = np.asarray(idx_gpu)[tokens]
    flips = [i for i in range(len(tokens)) if not np.array_equal(g_idx[i], idx_ref[i])]
    if flips:
        for i in flips:
            assert gap[i] < TIE_GAP or set(g_idx[i]) == set(idx_ref[i]), (tokens[i], gap[i])
        yf, _, _, _ = oracle.layer_forward(x[flips], layer.Wr, layer.bias, idx_gpu.shape[1], layer.routed,
                                           layer.shared, residual=None if res is None else res[flips],
                                           forced_idx=g_idx[flips], nthreads=nthreads)
        y_ref[flips] = yf
    err = rel_err(np.asarray(y_gpu)[tokens], y_ref)
    assert err <= tol, err
    return err, flips
