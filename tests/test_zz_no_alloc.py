"""The workspace-free router entry point, moe_router_topk_static.

Some callers cannot allocate device memory: plugins whose host application owns and budgets
every device allocation and gives them no allocator, or runtimes that lay out all device memory
ahead of time and have no allocator at run time. For them the library offers a router/top-k
whose scratch is a fixed array inside the library, so nothing has to be allocated or passed in.

This file runs last (pytest collects files by name) so that, if it fails, a run stopping at the
first failure has already run everything else. Each test compares the workspace-free call with
the regular moe_router_topk on the same inputs, on two calls in a row (the shared scratch keeps
the previous call's contents, so the second call checks that nothing stale leaks through).
"""
import numpy as np
import pytest
import torch

import quantized_expert_ffn_gemm_b200 as moe
import synth

pytestmark = pytest.mark.gpu

W_TOL = 1e-5  # routing weights, absolute (the tolerance of the other router tests)


def _inputs(name, T=None):
    s = synth.WORKLOADS[name]
    T = T or s.T
    x = synth.make_x(s.seed, T, s.H).cuda()
    Wr = synth.make_router(s.seed, 0, s.E, s.H).cuda()
    b = synth.zipf_bias(s.seed, 0, s.E, s.zipf_s).cuda() if s.zipf_s else None
    return s, x, Wr, b


@pytest.mark.parametrize("name,T", [("decode1", 1), ("decode4", 4), ("tiny", 8)])
def test_static_router_matches_workspace_router_twice(name, T):
    s, x, Wr, b = _inputs(name, T)
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    idx_ref, w_ref, lg_ref = moe.router_topk(x, Wr, b, s.k, ws, want_logits=True)
    for _ in range(2):
        idx, w, lg = moe.router_topk_static(x, Wr, b, s.k, want_logits=True)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        assert float((w - w_ref).abs().max()) <= W_TOL
        assert torch.equal(lg, lg_ref)


def test_static_router_alternating_shapes():
    # a larger call followed by a smaller one: the second must not see the first one's logits
    s4, x4, Wr, b = _inputs("decode4", 4)
    ws = moe.Workspace.for_layer(s4.H, s4.E, s4.k, s4.I, True, 4)
    for xx in (x4, x4[:1], x4[2:4]):
        idx_ref, w_ref = moe.router_topk(xx, Wr, b, s4.k, ws)
        idx, w = moe.router_topk_static(xx, Wr, b, s4.k)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        assert float((w - w_ref).abs().max()) <= W_TOL


def test_static_router_rejects_sizes_beyond_its_scratch():
    s, x, Wr, b = _inputs("tiny", 9)
    with pytest.raises(moe.MoeError) as ei:
        moe.router_topk_static(x, Wr, b, s.k)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED


def test_static_router_applies_the_same_shape_rules():
    # the same arguments give the same status as moe_router_topk: H beyond 16384 is a valid but
    # unsupported shape, H not a multiple of 32 an invalid one, k > E invalid
    x = torch.zeros(1, 16448, dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros(16, 16448, dtype=torch.float32, device="cuda")
    ws = moe.Workspace.for_layer(256, 16, 2, 64, False, 1)
    for xx, WW, k, code in ((x, Wr, 2, moe.MOE_ERR_UNSUPPORTED), (x[:, :80], Wr[:, :80], 2, moe.MOE_ERR_INVALID_ARG),
                            (x[:, :256], Wr[:4, :256], 5, moe.MOE_ERR_INVALID_ARG)):
        with pytest.raises(moe.MoeError) as e_static:
            moe.router_topk_static(xx.contiguous(), WW.contiguous(), None, k)
        with pytest.raises(moe.MoeError) as e_ws:
            moe.router_topk(xx.contiguous(), WW.contiguous(), None, k, ws)
        assert e_static.value.code == e_ws.value.code == code
