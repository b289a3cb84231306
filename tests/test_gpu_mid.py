"""GPU parity of the mid-batch expert path (MOE_PATH_MID) against the oracle.

The path groups each selected expert's tokens into units of up to 8 straight from the routing and
splits every unit into 128-feature items whose partial down outputs are summed per token. The
cases cover: the full-size decode-shaped layer (H=2048, E=512, top-10, I=512, shared expert, Q2,
Zipf(1.1) router bias) at 1..128 tokens; a small layer whose popular experts take many more than 8
tokens (several units per expert, the last one ragged); Q3 without a shared expert and Q4; the
residual added in place; bit-identical repeat calls; the stack; and the shapes the path refuses.
Routing is checked as in every layer test (indices bit-exact, slot order included, except at
logged oracle near-ties; weights within 1e-5).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_ffn_gemm_b200 as moe
import synth
from tests.gpu_util import Y_TOL, check_layer, rel_err, to_dev

pytestmark = pytest.mark.gpu

DEC = synth.LayerShape("mid_decode", 128, 2048, 512, 10, 512, synth.Q2, True, 1.1, seed=6)
# E = 32, k = 4: ~16 tokens per expert at 128 tokens, Zipf(1.1) makes the popular ones much larger
SMALL = synth.LayerShape("mid_small", 128, 512, 32, 4, 256, synth.Q2, True, 1.1, seed=7)
SMALL_Q3 = synth.LayerShape("mid_small_q3", 100, 512, 32, 4, 256, synth.Q3, False, 1.2, seed=8)
SMALL_Q4 = synth.LayerShape("mid_small_q4", 64, 512, 32, 4, 384, synth.Q4, True, 1.1, seed=9)

_cache = {}


def layer_of(shape):
    if shape.name not in _cache:
        L = synth.make_layer(shape)
        _cache[shape.name] = (L, to_dev(L))
    return _cache[shape.name]


def run(shape, T, residual=None, y=None, path=moe.PATH_MID):
    L, (x, Wr, b, routed, shared) = layer_of(shape)
    ws = moe.Workspace.for_layer(shape.H, shape.E, shape.k, shape.I, shape.shared, T)
    y, idx, w = moe.layer_forward(x[:T].contiguous(), Wr, b, routed, shared, shape.k, ws, residual=residual, y=y,
                                  path=path, want_routing=True)
    assert moe.read_device_error(ws) == 0
    return L, y, idx, w


@pytest.mark.parametrize("T", [1, 6, 9, 12, 32, 100, 128])
def test_mid_decode_layer(T):
    L, y, idx, w = run(DEC, T)
    idx_np = idx.cpu().numpy()
    if T <= 32:
        tokens = np.arange(T)
    else:  # sampled, plus tokens of the most popular expert (its rows fill several units)
        top = np.bincount(idx_np.reshape(-1), minlength=DEC.E).argmax()
        heavy = np.nonzero((idx_np == top).any(axis=1))[0]
        tokens = np.union1d(np.random.default_rng(T).choice(T, 24, replace=False),
                            heavy[np.linspace(0, len(heavy) - 1, 6).astype(int)])
    err, flips = check_layer(y.cpu().numpy(), idx_np, L, tokens, w_gpu=w.cpu().numpy())
    print(f"mid decode T={T}: max|dy|/rms = {err:.3e}, near-tie flips {len(flips)}")


@pytest.mark.parametrize("shape,T", [(SMALL, 128), (SMALL, 37), (SMALL_Q3, 100), (SMALL_Q4, 64), (SMALL_Q4, 3)])
def test_mid_many_tokens_per_expert(shape, T):
    L, y, idx, w = run(shape, T)
    idx_np = idx.cpu().numpy()
    counts = np.bincount(idx_np.reshape(-1), minlength=shape.E)
    if T >= 64:
        assert counts.max() > 16  # some expert spans three or more units
    err, flips = check_layer(y.cpu().numpy(), idx_np, L, np.arange(T), w_gpu=w.cpu().numpy())
    print(f"{shape.name} T={T}: max tokens per expert {counts.max()}, max|dy|/rms = {err:.3e}")


def test_mid_residual_in_place_and_repeatable():
    T = 48
    L, (x, Wr, b, routed, shared) = layer_of(SMALL)
    r = synth.make_residual(11, T, SMALL.H).cuda()
    _, y1, idx, w = run(SMALL, T, residual=r.clone())
    _, y2, _, _ = run(SMALL, T, residual=r.clone())
    assert torch.equal(y1, y2)  # fixed-order sums: bit-identical repeats
    y3 = r.clone()
    run(SMALL, T, residual=y3, y=y3)  # residual and y aliased
    assert torch.equal(y1, y3)
    check_layer(y1.cpu().numpy(), idx.cpu().numpy(), L, range(T), residual=r.cpu().numpy(), w_gpu=w.cpu().numpy())


@pytest.mark.parametrize("T", [12, 100])
def test_mid_agrees_with_grouped_gemm(T):
    _, y_mid, idx_mid, _ = run(DEC, T)
    _, y_gemm, idx_gemm, _ = run(DEC, T, path=moe.PATH_GEMM)
    same = (idx_mid.cpu().numpy() == idx_gemm.cpu().numpy()).all(axis=1)
    a, b = y_mid.cpu().double().numpy()[same], y_gemm.cpu().double().numpy()[same]
    assert same.sum() >= T - 2 and rel_err(a, b) <= Y_TOL


def test_mid_stack_small_full_compare():
    H, E, k, I, Lyr, T = 256, 16, 2, 128, 4, 12
    Wrs = [synth.make_router(0, l, E, H) for l in range(Lyr)]
    rs = [synth.make_expert_set(0, l, 0, 2, E, H, I) for l in range(Lyr)]
    ss = [synth.make_expert_set(0, l, 1, 2, 1, H, I) for l in range(Lyr)]
    r0 = synth.make_residual(0, T, H)
    st = moe.Stack([w.cuda() for w in Wrs], None, [r.to("cuda") for r in rs], [s.to("cuda") for s in ss], k)
    ws = moe.Workspace.for_layer(H, E, k, I, True, T)
    r_out = moe.stack_forward(r0.cuda(), st, ws, path=moe.PATH_MID).cpu().numpy()
    assert moe.read_device_error(ws) == 0
    ref, _ = oracle.stack_forward(r0, list(zip(Wrs, [None] * Lyr, rs, ss)), k)
    assert rel_err(r_out, ref) <= Y_TOL


def test_mid_refuses_what_it_does_not_take():
    L, (x, Wr, b, routed, shared) = layer_of(SMALL)
    # more tokens than the path takes
    x129 = synth.make_x(3, 129, SMALL.H).cuda()
    ws = moe.Workspace.for_layer(SMALL.H, SMALL.E, SMALL.k, SMALL.I, True, 129)
    with pytest.raises(moe.MoeError) as ei:
        moe.layer_forward(x129, Wr, b, routed, shared, SMALL.k, ws, path=moe.PATH_MID)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED
    # I not a multiple of 128
    s2 = synth.LayerShape("mid_i64", 16, 256, 8, 2, 64, synth.Q2, False, None, seed=2)
    L2, (x2, Wr2, b2, r2, _) = layer_of(s2)
    ws2 = moe.Workspace.for_layer(s2.H, s2.E, s2.k, s2.I, False, 16)
    with pytest.raises(moe.MoeError) as ei:
        moe.layer_forward(x2, Wr2, b2, r2, None, s2.k, ws2, path=moe.PATH_MID)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED
    # the rows entry point has no routing to work from
    rows = torch.zeros(8, SMALL.H, dtype=torch.float16, device="cuda")
    offs = torch.tensor([0] + [8] * SMALL.E + [8], dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.expert_ffn(rows, offs, SMALL.E, routed, shared, ws, path=moe.PATH_MID)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("T,expect", [(8, "decode_fused"), (9, "mid_expert"), (20, "mid_expert"), (21, "gemm_gate_up"),
                                      (64, "gemm_gate_up")])
def test_auto_path_by_token_count(T, expect):
    # AUTO: the fused decode kernel while its plan fits (8 tokens at top-10 with a shared expert),
    # the mid-batch path up to 20 tokens, the grouped GEMM above (bench.py --crossover); the
    # per-kernel timing hook shows which kernels a call launched
    L, (x, Wr, b, routed, shared) = layer_of(DEC)
    ws = moe.Workspace.for_layer(DEC.H, DEC.E, DEC.k, DEC.I, DEC.shared, T)
    moe.layer_forward(x[:T].contiguous(), Wr, b, routed, shared, DEC.k, ws)  # plans and limits set up
    torch.cuda.synchronize()
    moe.timing_enable(True)
    try:
        moe.layer_forward(x[:T].contiguous(), Wr, b, routed, shared, DEC.k, ws)
        torch.cuda.synchronize()
        ran = {n for n, (ms, cnt) in moe.timing_read().items() if cnt > 0}
    finally:
        moe.timing_enable(False)
    assert moe.read_device_error(ws) == 0
    assert expect in ran, (T, sorted(ran))
    others = {"decode_fused", "mid_expert", "gemm_gate_up"} - {expect}
    assert not (others & ran), (T, sorted(ran))
