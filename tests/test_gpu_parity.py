"""GPU parity: every C-ABI entry point against the CPU oracle on the same seeded inputs.

Integers (top-k indices, counts, offsets, permutation, dequantized values) must match bit for bit
(an index may differ only at an oracle near-tie, gap < 1e-5, and the oracle then recomputes y
with the GPU's selection); floating outputs must satisfy max|y - y_ref| / rms(y_ref) <= 1e-2 and
routing weights <= 1e-5 absolute. Full-size configs are checked on sampled tokens (tokens are
independent, so each sampled row is exact, not an approximation).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_ffn_gemm_b200 as moe
import synth
from tests.gpu_util import W_TOL, Y_TOL, check_layer, compare_routing, rel_err, to_dev

pytestmark = pytest.mark.gpu

MID = synth.LayerShape("mid", 300, 512, 32, 4, 256, synth.Q2, True, 1.1, seed=3)
MID_Q3 = synth.LayerShape("mid_q3", 200, 512, 32, 4, 256, synth.Q3, False, 1.2, seed=4)
MID_Q4 = synth.LayerShape("mid_q4", 300, 512, 32, 4, 256, synth.Q4, True, 1.1, seed=5)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    moe.lib()
    torch.cuda.init()


_cache = {}


def layer_of(name):
    if name not in _cache:
        shape = {"mid": MID, "mid_q3": MID_Q3, "mid_q4": MID_Q4}.get(name) or synth.WORKLOADS[name]
        L = synth.make_layer(shape)
        _cache[name] = (L, to_dev(L))
    return _cache[name]


def ws_for(L, T=None):
    s = L.shape
    return moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T or s.T)


# ----------------------------------------------------------------------------- generator on device
def test_generator_device_bits_match_cpu():
    a = synth.make_qmat(0, 1, 0, 2, synth.Q3, 3, 64, 256, device="cpu")
    b = synth.make_qmat(0, 1, 0, 2, synth.Q3, 3, 64, 256, device="cuda")
    assert torch.equal(a.codes, b.codes.cpu()) and torch.equal(a.hibits, b.hibits.cpu())
    assert torch.equal(a.scales.view(torch.int16), b.scales.cpu().view(torch.int16))


# ----------------------------------------------------------------------------- dequant
@pytest.mark.parametrize("qtype", [synth.Q2, synth.Q3, synth.Q4])
def test_dequant_rows_bit_exact(qtype):
    qm = synth.make_qmat(7, 0, 0, 0, qtype, 4, 96, 512)
    dm = qm.to("cuda")
    for e, r0, n in ((0, 0, 96), (3, 17, 5)):
        f32, f16 = moe.dequant_rows(dm, e, r0, n)
        ref, ref16 = oracle.dequant_rows(qm, e, r0, n)
        assert np.array_equal(f32.cpu().double().numpy(), ref)
        assert np.array_equal(f16.cpu().view(torch.int16).numpy().view(np.uint16), ref16)


# ----------------------------------------------------------------------------- router
@pytest.mark.parametrize("name", ["tiny", "decode1", "decode4", "mid", "prefill2k_q3"])
def test_router_topk(name):
    L, (x, Wr, b, _, _) = layer_of(name)
    ws = ws_for(L)
    idx, w, logits = moe.router_topk(x, Wr, b, L.shape.k, ws, want_logits=True)
    idx_ref, w_ref, lg_ref, gap = oracle.router_topk(L.x, L.Wr, L.bias, L.shape.k)
    lg = logits.cpu().double().numpy()
    assert np.abs(lg - lg_ref).max() < 1e-5 * max(1.0, np.abs(lg_ref).max())
    compare_routing(idx.cpu().numpy(), w.cpu().numpy(), idx_ref, w_ref, gap, lg_ref)
    assert moe.read_device_error(ws) == 0


@pytest.mark.parametrize("T", [12, 100])
def test_router_topk_mid_batch(T):
    # 9..128 tokens take the CUDA-core fp32 router (exact fp32 logits, no refine step)
    L0, (_, Wr, b, _, _) = layer_of("decode4")
    s = L0.shape
    x = synth.make_x(s.seed, T, s.H, stream=60 + T)
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    idx, w, logits = moe.router_topk(x.cuda(), Wr, b, s.k, ws, want_logits=True)
    idx_ref, w_ref, lg_ref, gap = oracle.router_topk(x, L0.Wr, L0.bias, s.k)
    lg = logits.cpu().double().numpy()
    assert np.abs(lg - lg_ref).max() < 1e-5 * max(1.0, np.abs(lg_ref).max())
    compare_routing(idx.cpu().numpy(), w.cpu().numpy(), idx_ref, w_ref, gap, lg_ref)
    assert moe.read_device_error(ws) == 0


def test_router_prefill_8k_all_tokens():
    L, (x, Wr, b, _, _) = layer_of("prefill8k")
    ws = ws_for(L)
    idx, w = moe.router_topk(x, Wr, b, 10, ws)
    idx_ref, w_ref, lg_ref, gap = oracle.router_topk(L.x, L.Wr, L.bias, 10)
    flips = compare_routing(idx.cpu().numpy(), w.cpu().numpy(), idx_ref, w_ref, gap, lg_ref)
    assert len(flips) < 64
    # uniform router: every expert gets a share near T*k/E = 160 rows
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=512)
    assert counts.min() > 60 and counts.max() < 320


# ----------------------------------------------------------------------------- permute / combine
@pytest.mark.parametrize("T,k,E,shared", [(8192, 10, 512, True), (37, 3, 16, False), (1, 10, 512, True),
                                          (5, 1, 4, False), (3000, 7, 301, True), (12000, 10, 512, False)])
def test_permute_bit_exact(T, k, E, shared):
    # the scan runs one of three ways: a single 1024-pair chunk (read in one round of loads), a
    # histogram staged in shared memory (8192 x 10 over 512 experts; 3000 x 7 over 301 experts,
    # an odd size), or, when the histogram is too large to stage (12000 x 10: 118 chunks), warp
    # passes over global memory
    rng = np.random.default_rng(T + k)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    x = synth.make_x(1, T, 256)
    ws = moe.Workspace.for_layer(256, E, k, 64, shared, T)
    out = moe.permute(torch.from_numpy(idx).cuda(), E, x.cuda(), shared, ws)
    counts, offsets, row_of, src = oracle.permute(idx, E)
    assert np.array_equal(out["counts"][:E].cpu().numpy(), counts)
    assert np.array_equal(out["offsets"][:E + 1].cpu().numpy(), offsets)
    assert np.array_equal(out["row_of"].cpu().numpy(), row_of)
    P = T * k
    assert np.array_equal(out["src"][:P].cpu().numpy(), src)
    xp = out["x_perm"].cpu()
    ref = x.float().half()
    assert torch.equal(xp[:P].view(torch.int16), ref[torch.from_numpy(src).long()].view(torch.int16))
    if shared:
        assert out["offsets"][E + 1].item() == P + T
        assert np.array_equal(out["src"][P:].cpu().numpy(), np.arange(T))
        assert torch.equal(xp[P:].view(torch.int16), ref.view(torch.int16))
    assert moe.read_device_error(ws) == 0


def test_permute_flags_bad_expert_index():
    idx = torch.tensor([[0, 1], [2, 7], [3, 0]], dtype=torch.int32, device="cuda")  # 7 >= E = 4
    ws = moe.Workspace.for_layer(256, 4, 2, 64, False, 3)
    out = moe.permute(idx, 4, synth.make_x(0, 3, 256).cuda(), False, ws)
    assert moe.read_device_error(ws) == moe.MOE_ERR_DEVICE_CHECK
    assert out["row_of"][1, 1].item() == -1
    assert moe.read_device_error(ws) == 0   # reading clears the word


def test_combine_matches_definition():
    rng = np.random.default_rng(0)
    T, k, H = 33, 4, 512
    rows = T * k + T
    outp = torch.from_numpy(rng.normal(size=(rows, H)).astype(np.float16))
    perm = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    w = torch.from_numpy(rng.uniform(size=(T, k)).astype(np.float32))
    res = torch.from_numpy(rng.normal(size=(T, H)).astype(np.float32))
    y = moe.combine(outp.cuda(), torch.from_numpy(perm).cuda(), w.cuda(), outp[T * k:].cuda(), res.cuda()).cpu()
    o = outp.double().numpy()
    ref = res.double().numpy() + o[T * k:] + np.einsum("tk,tkh->th", w.double().numpy(), o[perm])
    assert np.abs(y.double().numpy() - ref).max() < 1e-4


# ----------------------------------------------------------------------------- expert FFN (both paths)
@pytest.mark.parametrize("name", ["tiny", "mid", "mid_q3", "mid_q4"])
@pytest.mark.parametrize("path", [moe.PATH_GEMV, moe.PATH_GEMM, moe.PATH_AUTO])
def test_expert_ffn_rows(name, path):
    L, (x, Wr, b, routed, shared) = layer_of(name)
    s = L.shape
    idx_ref, _, _, _ = oracle.router_topk(L.x, L.Wr, L.bias, s.k)
    ws = ws_for(L)
    pm = moe.permute(torch.from_numpy(idx_ref).cuda(), s.E, x, s.shared, ws)
    n_rows = s.T * s.k + (s.T if s.shared else 0)
    ws2 = moe.Workspace.for_layer(s.H, s.E, 1, s.I, False, n_rows)
    out = moe.expert_ffn(pm["x_perm"], pm["offsets"], s.E, routed, shared, ws2, path=path)
    assert moe.read_device_error(ws2) == 0
    # oracle: each sampled row through its group's expert
    offs = pm["offsets"].cpu().numpy()
    xp = pm["x_perm"].cpu().double().numpy()
    rng = np.random.default_rng(1)
    sample = np.sort(rng.choice(n_rows, size=min(n_rows, 96), replace=False))
    ref = np.zeros((len(sample), s.H))
    for i, r in enumerate(sample):
        g = int(np.searchsorted(offs[:s.E + (1 if s.shared else 0) + 1], r, side="right") - 1)
        es, e = (L.shared, 0) if g == s.E else (L.routed, g)
        ref[i] = oracle.expert_ffn_rows(es, e, xp[r:r + 1])[0]
    got = out.cpu().double().numpy()[sample]
    assert rel_err(got, ref) <= Y_TOL


# ----------------------------------------------------------------------------- layer forward
@pytest.mark.parametrize("name,ntok", [("tiny", 64), ("decode1", 1), ("decode4", 4), ("verify6", 6),
                                       ("decode1_pruned256", 1), ("decode1_q4", 1), ("mid", 300),
                                       ("mid_q3", 200), ("mid_q4", 300), ("prefill8k", 24), ("prefill2k_q3", 64)])
def test_layer_forward(name, ntok):
    L, (x, Wr, b, routed, shared) = layer_of(name)
    s = L.shape
    ws = ws_for(L)
    y, idx, w = moe.layer_forward(x, Wr, b, routed, shared, s.k, ws, want_routing=True)
    assert moe.read_device_error(ws) == 0
    tokens = np.arange(s.T) if ntok >= s.T else np.sort(np.random.default_rng(5).choice(s.T, ntok, replace=False))
    if ntok < s.T:  # and tokens routed to the most popular expert (its rows fill several full tiles)
        flat = idx.cpu().numpy()
        top = np.bincount(flat.reshape(-1), minlength=s.E).argmax()
        heavy = np.nonzero((flat == top).any(axis=1))[0]
        tokens = np.union1d(tokens, heavy[np.linspace(0, len(heavy) - 1, 8).astype(int)])
    err, flips = check_layer(y.cpu().numpy(), idx.cpu().numpy(), L, tokens, w_gpu=w.cpu().numpy())
    print(f"{name}: max|dy|/rms = {err:.3e}, near-tie flips {len(flips)}")


def test_layer_forward_with_residual_in_place():
    L, (x, Wr, b, routed, shared) = layer_of("mid")
    s = L.shape
    r = synth.make_residual(9, s.T, s.H).cuda()
    ws = ws_for(L)
    y, idx, w = moe.layer_forward(x, Wr, b, routed, shared, s.k, ws, residual=r.clone(), want_routing=True)
    y2 = r.clone()
    moe.layer_forward(x, Wr, b, routed, shared, s.k, ws, residual=y2, y=y2)  # aliasing residual and y
    assert torch.equal(y, y2)
    check_layer(y.cpu().numpy(), idx.cpu().numpy(), L, range(0, s.T, 7), residual=r.cpu().numpy(),
                w_gpu=w.cpu().numpy())


@pytest.mark.parametrize("name,T", [("mid", 64), ("mid", 4), ("mid_q3", 4), ("tiny", 4), ("mid_q4", 64)])
def test_cross_path_gemv_vs_gemm(name, T):
    L, (x, Wr, b, routed, shared) = layer_of(name)
    s = L.shape
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    ya = moe.layer_forward(x[:T], Wr, b, routed, shared, s.k, ws, path=moe.PATH_GEMV)
    yb = moe.layer_forward(x[:T], Wr, b, routed, shared, s.k, ws, path=moe.PATH_GEMM)
    assert rel_err(ya.cpu().numpy(), yb.cpu().numpy()) <= Y_TOL


@pytest.mark.parametrize("name,T", [("mid", 5), ("mid", 8), ("decode4", 5), ("decode4", 6), ("decode4", 8),
                                    ("prefill8k", 4), ("prefill8k", 5), ("decode4", 12), ("prefill2k_q3", 100),
                                    ("decode1_q4", 4), ("decode1_q4", 8), ("mid_q4", 5)])
def test_layer_forward_decode_batches(name, T):
    # 5-8 tokens take the decode path under AUTO: the fused kernel where its shared-memory plan
    # fits (top-4 layer; top-10 at T=5), the separate decode kernels beyond (top-10 at T=6, 8).
    # With the uniform router of the prefill layer, 5 tokens choose ~50 distinct experts: more
    # down pieces than shared-memory slots, so two pieces of one row block share a slot.
    # 12 and 100 tokens: the small-batch router, then the grouped GEMM.
    # Fresh tokens on the cached layer's weights, every token against the oracle.
    L0, (_, Wr, b, routed, shared) = layer_of(name)
    s = L0.shape
    L = synth.LayerInputs(s, synth.make_x(s.seed, T, s.H, stream=40 + T), L0.Wr, L0.bias, L0.routed, L0.shared)
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    y, idx, w = moe.layer_forward(L.x.cuda(), Wr, b, routed, shared, s.k, ws, want_routing=True)
    assert moe.read_device_error(ws) == 0
    check_layer(y.cpu().numpy(), idx.cpu().numpy(), L, range(T), w_gpu=w.cpu().numpy())


def test_mtp_verify_T4_equals_four_T1():
    L, (x, Wr, b, routed, shared) = layer_of("decode4")
    ws = ws_for(L)
    y4 = moe.layer_forward(x, Wr, b, routed, shared, 10, ws).cpu().numpy()
    for t in range(4):
        y1 = moe.layer_forward(x[t:t + 1], Wr, b, routed, shared, 10, ws).cpu().numpy()
        assert rel_err(y1, y4[t:t + 1]) < 1e-5  # same arithmetic up to fp32 summation order


def test_zero_tokens_is_noop():
    L, (x, Wr, b, routed, shared) = layer_of("tiny")
    ws = ws_for(L)
    y = moe.layer_forward(x[:0], Wr, b, routed, shared, 2, ws)
    assert y.shape == (0, 256)


# ----------------------------------------------------------------------------- failure path
def test_starved_wait_times_out_and_context_survives():
    # The fused kernel's logit-exchange wait, polling for a tag that never arrives, gives up after
    # its limit, reports MOE_ERR_TIMEOUT through the workspace error word, and leaves the context
    # and the workspace fit for the next call (which must still match the oracle).
    L, (x, Wr, b, routed, shared) = layer_of("decode1")
    s = L.shape
    ws = ws_for(L)
    y0 = moe.layer_forward(x, Wr, b, routed, shared, s.k, ws)
    assert moe.read_device_error(ws) == 0
    import time
    t0 = time.perf_counter()
    moe.test_wait_timeout(ws, limit_ms=20)
    assert moe.read_device_error(ws) == moe.MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 1.5           # the limit, not a hang
    assert moe.read_device_error(ws) == 0            # reading cleared the word
    y1, idx, w = moe.layer_forward(x, Wr, b, routed, shared, s.k, ws, want_routing=True)
    assert moe.read_device_error(ws) == 0
    assert torch.equal(y0, y1)
    check_layer(y1.cpu().numpy(), idx.cpu().numpy(), L, range(s.T), w_gpu=w.cpu().numpy())


# ----------------------------------------------------------------------------- RMSNorm and stacks
def test_rmsnorm_matches_oracle():
    r = synth.make_residual(2, 64, 2048) * 3.0
    u = moe.rmsnorm_bf16(r.cuda()).cpu().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.rmsnorm_bf16(r)
    diff = np.abs(u.astype(np.int32) - ref.astype(np.int32))
    assert diff.max() <= 1                  # at most one bf16 ulp (fp32 vs fp64 rounding boundary)
    assert (diff > 0).mean() < 0.01


def test_stack_small_full_compare():
    H, E, k, I, Lyr, T = 256, 16, 2, 128, 4, 12
    Wrs = [synth.make_router(0, l, E, H) for l in range(Lyr)]
    rs = [synth.make_expert_set(0, l, 0, 2, E, H, I) for l in range(Lyr)]
    ss = [synth.make_expert_set(0, l, 1, 2, 1, H, I) for l in range(Lyr)]
    r0 = synth.make_residual(0, T, H)
    st = moe.Stack([w.cuda() for w in Wrs], None, [r.to("cuda") for r in rs], [s.to("cuda") for s in ss], k)
    ws = moe.Workspace.for_layer(H, E, k, I, True, T)
    r_out = moe.stack_forward(r0.cuda(), st, ws).cpu().numpy()
    ref, _ = oracle.stack_forward(r0, list(zip(Wrs, [None] * Lyr, rs, ss)), k)
    assert rel_err(r_out, ref) <= Y_TOL


# ----------------------------------------------------------------------------- fp16 operand range
@pytest.mark.parametrize("name,T", [("decode1", 1), ("decode4", 4), ("mid", 300)])
def test_fp16_range_is_flagged_not_silent(name, T):
    # The expert contractions take fp16 operands (x, h, expert outputs). Scaled by 300, x stays
    # inside fp16 but h = silu(x Wg) * (x Wu) grows ~9e4 times and overflows: the call must record
    # MOE_ERR_RANGE rather than return inf silently. Scaled by 20 (h ~400 times larger) nothing
    # overflows and the layer matches the oracle.
    L0, (_, Wr, b, routed, shared) = layer_of(name)
    s = L0.shape
    base = synth.make_x(s.seed, T, s.H, stream=500 + T).float()
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    for scale, overflow in ((300.0, True), (20.0, False)):
        x = (base * scale).to(torch.bfloat16)
        y, idx, w = moe.layer_forward(x.cuda(), Wr, b, routed, shared, s.k, ws, want_routing=True)
        code = moe.read_device_error(ws)
        if overflow:
            assert code == moe.MOE_ERR_RANGE
            assert not torch.isfinite(y).all()
        else:
            assert code == 0
            L = synth.LayerInputs(s, x, L0.Wr, L0.bias, L0.routed, L0.shared)
            check_layer(y.cpu().numpy(), idx.cpu().numpy(), L, range(min(T, 24)), w_gpu=w.cpu().numpy())


# ----------------------------------------------------------------------------- int8-activation (MMQ) path
def test_mmq_expert_ffn_rows_match_the_int8_definition():
    # MOE_PATH_MMQ quantizes each permuted activation row in 32-value blocks to int8 (the oracle's
    # quantize_blocks_i8 states the rule) and computes gate/up from exact integer block sums; the
    # oracle applies the same quantization and evaluates the FFN in fp64 on q * d. The deviation
    # from the unquantized FFN is the format's own error, printed beside it.
    L, (x, Wr, b, routed, shared) = layer_of("mid")
    s = L.shape
    idx_ref, _, _, _ = oracle.router_topk(L.x, L.Wr, L.bias, s.k)
    ws = ws_for(L)
    pm = moe.permute(torch.from_numpy(idx_ref).cuda(), s.E, x, s.shared, ws)
    n_rows = s.T * s.k + s.T
    ws2 = moe.Workspace.for_layer(s.H, s.E, 1, s.I, False, n_rows)
    out = moe.expert_ffn(pm["x_perm"], pm["offsets"], s.E, routed, shared, ws2, path=moe.PATH_MMQ)
    assert moe.read_device_error(ws2) == 0
    offs = pm["offsets"].cpu().numpy()
    xp16 = pm["x_perm"].cpu().view(torch.int16).numpy().view(np.uint16)
    q, d = oracle.quantize_blocks_i8(xp16)
    xq = oracle.dequantize_blocks_i8(q, d)
    xe = pm["x_perm"].cpu().double().numpy()
    rng = np.random.default_rng(2)
    sample = np.sort(rng.choice(n_rows, size=96, replace=False))
    ref = np.zeros((len(sample), s.H))
    exact = np.zeros((len(sample), s.H))
    for i, r in enumerate(sample):
        g = int(np.searchsorted(offs[:s.E + 2], r, side="right") - 1)
        es, e = (L.shared, 0) if g == s.E else (L.routed, g)
        ref[i] = oracle.expert_ffn_rows(es, e, xq[r:r + 1])[0]
        exact[i] = oracle.expert_ffn_rows(es, e, xe[r:r + 1])[0]
    got = out.cpu().double().numpy()[sample]
    err = rel_err(got, ref)
    print(f"MMQ vs its int8 definition {err:.2e}; int8 activations vs exact {rel_err(got, exact):.2e}")
    assert err <= Y_TOL


def test_mmq_rejects_formats_it_does_not_take():
    L, (x, Wr, b, routed, shared) = layer_of("mid_q3")
    s = L.shape
    ws = ws_for(L)
    with pytest.raises(moe.MoeError) as ei:
        moe.layer_forward(x, Wr, b, routed, shared, s.k, ws, path=moe.PATH_MMQ)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED


# ----------------------------------------------------------------------------- host-buffer entry points
@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("name,T,path", [("decode1", 1, moe.PATH_AUTO), ("decode4", 4, moe.PATH_AUTO),
                                         ("mid", 32, moe.PATH_MID), ("mid", 300, moe.PATH_AUTO)])
def test_layer_forward_host_buffers_match_the_device_call(name, T, path, pinned):
    # the tokens and y in host memory, one C call enqueuing copy, layer, copy: the same y, bit for
    # bit, as the device-pointer call (page-locked buffers move by a copy kernel when small,
    # pageable ones by cudaMemcpyAsync)
    L, (x, Wr, b, routed, shared) = layer_of(name)
    s = L.shape
    x = x[:T].contiguous()
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    h = moe.LayerHandle(Wr, b, routed, shared, s.k, ws)
    y_dev = torch.empty(T, s.H, dtype=torch.float32, device="cuda")
    h.forward(x, y_dev, path=path)
    x_host = x.cpu()
    y_host = torch.full((T, s.H), float("nan"), dtype=torch.float32)
    if pinned:
        x_host, y_host = x_host.pin_memory(), y_host.pin_memory()
    h.forward_host(x_host, y_host, path=path)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    assert torch.equal(y_host, y_dev.cpu())


@pytest.mark.parametrize("name,T", [("decode1", 1), ("decode4", 4)])
def test_layer_forward_host_buffers_reused_with_new_contents(name, T):
    # the same page-locked buffers for several calls, the host rewriting x between them (the copy
    # kernels read and write the mapped buffers): every call sees this call's x
    L, (x, Wr, b, routed, shared) = layer_of(name)
    s = L.shape
    ws = moe.Workspace.for_layer(s.H, s.E, s.k, s.I, s.shared, T)
    h = moe.LayerHandle(Wr, b, routed, shared, s.k, ws)
    x_host = torch.empty(T, s.H, dtype=torch.bfloat16).pin_memory()
    y_host = torch.empty(T, s.H, dtype=torch.float32).pin_memory()
    y_dev = torch.empty(T, s.H, dtype=torch.float32, device="cuda")
    for stream in range(3):
        xs = synth.make_x(s.seed, T, s.H, stream=stream + 1)
        x_host.copy_(xs)
        y_host.fill_(float("nan"))
        h.forward_host(x_host, y_host)
        torch.cuda.synchronize()
        h.forward(xs.cuda(), y_dev)
        torch.cuda.synchronize()
        assert moe.read_device_error(ws) == 0
        assert torch.equal(y_host, y_dev.cpu()), stream


def test_stack_forward_host_buffers_match_the_device_call():
    H, E, k, I, Lyr, T = 256, 16, 2, 128, 3, 5
    Wrs = [synth.make_router(0, l, E, H).cuda() for l in range(Lyr)]
    rs = [synth.make_expert_set(0, l, 0, 2, E, H, I, "cuda") for l in range(Lyr)]
    ss = [synth.make_expert_set(0, l, 1, 2, 1, H, I, "cuda") for l in range(Lyr)]
    st = moe.Stack(Wrs, None, rs, ss, k)
    ws = moe.Workspace.for_layer(H, E, k, I, True, T)
    r0 = synth.make_residual(4, T, H)
    dev = moe.stack_forward(r0.cuda(), st, ws).cpu()
    r_host = r0.clone().pin_memory()
    moe.stack_forward_host(r_host, st, ws, r_out_host=r_host)  # in place on the host buffer
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    assert torch.equal(r_host, dev)
