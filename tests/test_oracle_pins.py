"""Pins of the CPU oracle to things other than itself: hand-built fixtures, closed forms,
brute force on tiny inputs, textbook formulations and library routines.

The pages print no worked example for the layer (their numbers are whole-model tokens/s), so
every pin here comes from the definition of the stand-in formats and from mathematics. Each
test is chosen so that a plausible slip in the oracle (a dropped term, a wrong sign, a wrong
bit position, a transposed operand, a wrong tie rule) fails it.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.packing import KnownQMat, KnownSet, dense_ffn, pack_hi_plane, pack_lo_plane, random_known_set

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- number formats
def test_half_decode_matches_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(b) for b in bits[::7]])
    r = ref[::7]
    fin = np.isfinite(r)
    assert np.array_equal(got[fin], r[fin])
    assert np.array_equal(np.isnan(got), np.isnan(r))


def test_half_round_matches_numpy_rne():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.normal(0, 1, 2000), rng.normal(0, 1e-5, 500), rng.normal(0, 3e4, 500),
        # exact halfway points between neighbouring fp16 values (ties to even)
        (np.arange(1000, 1100, dtype=np.float64) + 0.5) / 1024.0,
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26]),
    ])
    for v in vals:
        with np.errstate(over="ignore"):
            ref = int(np.float16(v).view(np.uint16))
        assert oracle.double_to_half(v) == ref, v


def test_bf16_round_matches_torch_rne():
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.normal(0, 1, 3000).astype(np.float32),
                           (np.arange(256, 300, dtype=np.float32) + 0.5) / 256.0])  # ties
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, r in zip(vals, ref):
        assert oracle.double_to_bf16(float(v)) == int(r)
        assert oracle.bf16_to_double(int(r)) == float(torch.tensor([int(r)], dtype=torch.int32)
                                                        .to(torch.int16).view(torch.bfloat16).float())


# ----------------------------------------------------------------------------- dequant
def _read_blocks():
    cases = []
    with open(os.path.join(GOLDEN, "quant_blocks.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, qt, lo, hi, codes = [p.strip() for p in line.split("|")]
            lo_b = np.array([int(b, 16) for b in lo.split()], np.uint8)
            hi_b = None if hi == "-" else np.array([int(b, 16) for b in hi.split()], np.uint8)
            cases.append((name, int(qt), lo_b, hi_b, [int(c) for c in codes.split()]))
    return cases


class _Raw:
    def __init__(self, qtype, codes, hibits, scales, rows, K):
        self.qtype, self.n, self.rows, self.K = qtype, 1, rows, K
        self.codes, self.hibits, self.scales = codes, hibits, scales


@pytest.mark.parametrize("case", _read_blocks(), ids=lambda c: c[0])
def test_dequant_hand_built_blocks(case):
    name, qt, lo, hi, codes = case
    d16 = np.float16(0.0137)
    m = _Raw(qt, lo.reshape(1, 1, lo.size), None if hi is None else hi.reshape(1, 1, 4),
             np.array([[[d16.view(np.uint16)]]], np.uint16), 1, 32)
    assert lo.size == (16 if qt == 4 else 8)
    for k in range(32):
        assert oracle.code(m, 0, 0, k) == codes[k], (name, k)
    vals, v16 = oracle.dequant_rows(m, 0, 0, 1)
    q0 = {2: 2, 3: 4, 4: 8}[qt]
    expect = float(d16) * (np.array(codes) - q0)
    assert np.array_equal(vals[0], expect)                      # exact closed form d*(c-q0)
    assert np.array_equal(v16[0], expect.astype(np.float16).view(np.uint16))  # RNE to fp16


@pytest.mark.parametrize("qtype", [2, 3, 4])
def test_pack_decode_roundtrip_every_code_every_position(qtype):
    # every code value at every one of the 32 positions, several scale magnitudes and signs
    cmax = {2: 4, 3: 8, 4: 16}[qtype]
    rows = cmax * 32
    codes = np.zeros((1, rows, 64), np.int64)
    for c in range(cmax):
        for j in range(32):
            codes[0, c * 32 + j, j] = c          # first block: one marked position per row
            codes[0, c * 32 + j, 32 + (31 - j)] = (c + 1) % cmax  # second block, mirrored position
    sc = np.array([0.005, 0.0125, 0.02, 1.0, -0.5, 6.1e-5, 65504.0, 2.0 ** -24])
    scales = np.resize(sc, (1, rows, 2)).astype(np.float16)
    km = KnownQMat(qtype, codes, scales)
    for r in range(0, rows, 7):
        for k in range(64):
            assert oracle.code(km, 0, r, k) == codes[0, r, k]
    vals, _ = oracle.dequant_rows(km, 0, 0, rows)
    assert np.array_equal(vals, km.dense()[0])


@pytest.mark.parametrize("qtype,ncodes,bound", [(3, 8, 30.0), (4, 16, 45.0)])
def test_synth_planes_have_uniform_codes(qtype, ncodes, bound):
    qm = synth.make_qmat(0, 0, 0, 0, qtype, 2, 64, 256)
    cnt = np.zeros(ncodes)
    for r in range(64):
        for k in range(256):
            cnt[oracle.code(qm, 1, r, k)] += 1
    expect = cnt.sum() / ncodes
    chi2 = ((cnt - expect) ** 2 / expect).sum()
    assert chi2 < bound  # 7 / 15 dof; p ~ 1e-4


# ----------------------------------------------------------------------------- router / top-k
def _router_inputs(logits, bias=None):
    """x = e_0 and Wr[:,0] = logits, so the fp64 logits equal the given fp32 values exactly."""
    logits = np.asarray(logits, np.float32)
    T = 1 if logits.ndim == 1 else logits.shape[0]
    logits = logits.reshape(T, -1)
    E = logits.shape[1]
    H = 32
    x = np.zeros((T, H), np.uint16)
    Wr = np.zeros((E, H), np.float32)
    # token t uses column t of Wr: x[t, t] = 1 (bf16 0x3f80)
    for t in range(T):
        x[t, t] = 0x3F80
        Wr[:, t] = logits[t]
    return x, Wr, bias


def _brute_force_topk(l, k):
    """The unique k-subset S such that every selected e beats every unselected e':
    l_e > l_e' or (l_e == l_e' and e < e')."""
    E = len(l)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if all((l[e] > l[f]) or (l[e] == l[f] and e < f) for e in S for f in rest):
            found.append(S)
    assert len(found) == 1
    return set(found[0])


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    for E in range(2, 9):
        l = rng.integers(-3, 3, size=E).astype(np.float32)  # many exact ties
        for k in range(1, E + 1):
            x, Wr, _ = _router_inputs(l)
            idx, w, logits, gap = oracle.router_topk(x, Wr, None, k)
            assert set(idx[0].tolist()) == _brute_force_topk(l, k)
            # slots in descending logit order, ties by lower index
            keys = [(-l[e], e) for e in idx[0]]
            assert keys == sorted(keys)
            assert abs(w[0].sum() - 1.0) < 1e-12
            assert np.array_equal(logits[0], l.astype(np.float64))
            if k < E:
                srt = sorted(l.tolist(), reverse=True)
                assert gap[0] == srt[k - 1] - srt[k]


def test_topk_lower_index_wins_exact_tie():
    x, Wr, _ = _router_inputs([1.0, 3.0, 3.0, 2.0, 3.0])
    idx, w, _, _ = oracle.router_topk(x, Wr, None, 2)
    assert idx[0].tolist() == [1, 2]
    assert np.allclose(w[0], [0.5, 0.5], rtol=0, atol=1e-15)


def test_k2_weights_closed_form_sigmoid():
    rng = np.random.default_rng(3)
    for _ in range(50):
        l = rng.normal(0, 2, 6).astype(np.float32)
        x, Wr, _ = _router_inputs(l)
        idx, w, _, _ = oracle.router_topk(x, Wr, None, 2)
        l1, l2 = float(l[idx[0, 0]]), float(l[idx[0, 1]])
        assert abs(w[0, 0] - 1.0 / (1.0 + math.exp(l2 - l1))) < 1e-14
        assert abs(w[0, 1] - 1.0 / (1.0 + math.exp(l1 - l2))) < 1e-14


def test_weights_equal_full_softmax_renormalised():
    # restricted softmax == full softmax over all E, then renormalised over the selected set
    rng = np.random.default_rng(4)
    l = rng.normal(0, 1, 16).astype(np.float32)
    x, Wr, _ = _router_inputs(l)
    idx, w, _, _ = oracle.router_topk(x, Wr, None, 5)
    p = np.exp(l.astype(np.float64) - l.max())
    p /= p.sum()
    sel = p[idx[0]]
    assert np.allclose(w[0], sel / sel.sum(), rtol=1e-13, atol=0)


def test_router_bias_is_added_to_logits():
    l = np.array([0.5, 0.25, -1.0, 2.0], np.float32)
    b = np.array([0.0, 10.0, 0.0, -10.0], np.float32)
    x, Wr, _ = _router_inputs(l)
    idx, w, logits, _ = oracle.router_topk(x, Wr, b, 2)
    assert np.array_equal(logits[0], (l + b).astype(np.float64))
    assert idx[0].tolist() == [1, 0]


def test_router_logits_are_a_matrix_product():
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.normal(0, 1, (3, 64)).astype(np.float32)).to(torch.bfloat16)
    Wr = rng.normal(0, 0.02, (8, 64)).astype(np.float32)
    _, _, logits, _ = oracle.router_topk(x, Wr, None, 2)
    ref = x.double().numpy() @ Wr.astype(np.float64).T
    assert np.allclose(logits, ref, rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------- permute
@pytest.mark.parametrize("seed", range(4))
def test_permute_is_stable_sort(seed):
    rng = np.random.default_rng(seed)
    T, k, E = 37, 3, 11
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, row_of, src = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")          # library stable sort by expert key
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(src, order // k)
    assert np.array_equal(row_of.reshape(-1)[order], np.arange(T * k))
    # permute then unpermute is the identity on token rows
    x = rng.normal(size=(T, 5))
    x_perm = x[src]
    for t in range(T):
        for j in range(k):
            assert np.array_equal(x_perm[row_of[t, j]], x[t])


def test_permute_empty_and_single_expert():
    counts, offsets, row_of, src = oracle.permute(np.zeros((0, 2), np.int32), 4)
    assert counts.tolist() == [0, 0, 0, 0] and offsets.tolist() == [0, 0, 0, 0, 0]
    idx = np.full((5, 1), 2, np.int32)
    counts, offsets, row_of, src = oracle.permute(idx, 4)
    assert counts.tolist() == [0, 0, 5, 0] and src.tolist() == [0, 1, 2, 3, 4]


# ----------------------------------------------------------------------------- FFN and layer
def _bf16_rows(rng, T, H):
    x = torch.from_numpy(rng.normal(0, 1, (T, H)).astype(np.float32)).to(torch.bfloat16)
    return x, x.double().numpy()


@pytest.mark.parametrize("qtype", [2, 3, 4])
def test_one_hot_router_reduces_to_dense_swiglu(qtype):
    rng = np.random.default_rng(10 + qtype)
    T, H, E, I = 5, 64, 4, 32
    ks = random_known_set(rng, qtype, E, H, I)
    x, xd = _bf16_rows(rng, T, H)
    Wr = rng.normal(0, 0.02, (E, H)).astype(np.float32)
    bias = np.zeros(E, np.float32)
    bias[2] = 100.0
    y, idx, w, _ = oracle.layer_forward(x, Wr, bias, 1, ks)
    assert (idx == 2).all() and np.array_equal(w, np.ones((T, 1)))
    ref = dense_ffn(ks, 2, xd)  # textbook formulation with the known weights
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_expert_rows_hook_matches_dense():
    rng = np.random.default_rng(7)
    ks = random_known_set(rng, 2, 3, 64, 32)
    _, xd = _bf16_rows(rng, 4, 64)
    out = oracle.expert_ffn_rows(ks, 1, xd)
    assert np.allclose(out, dense_ffn(ks, 1, xd), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("qtype", [2, 3, 4])
def test_sparse_layer_equals_dense_mask_definition(qtype):
    # y_t = sum_{e<E} [e in S(t)] w_{t,e} FFN_e(x_t) + FFN_shared(x_t), all E experts evaluated densely
    rng = np.random.default_rng(20 + qtype)
    T, H, E, I, k = 6, 64, 6, 32, 3
    ks = random_known_set(rng, qtype, E, H, I)
    sh = random_known_set(rng, qtype, 1, H, I)
    x, xd = _bf16_rows(rng, T, H)
    Wr = rng.normal(0, 0.3, (E, H)).astype(np.float32)
    y, idx, w, _ = oracle.layer_forward(x, Wr, None, k, ks, sh)
    logits = xd @ Wr.astype(np.float64).T
    dense = np.stack([dense_ffn(ks, e, xd) for e in range(E)])  # [E,T,H]
    ref = dense_ffn(sh, 0, xd)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        p = np.exp(logits[t] - logits[t].max())
        mask = np.zeros(E)
        mask[order] = p[order] / p[order].sum()
        ref[t] += (mask[:, None] * dense[:, t, :]).sum(0)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-13)


def test_zero_scales_leave_shared_only_and_zero_codes_give_zero():
    rng = np.random.default_rng(30)
    T, H, E, I = 3, 64, 4, 32
    ks = random_known_set(rng, 2, E, H, I, scale_range=(0.0, 0.0))
    sh = random_known_set(rng, 2, 1, H, I)
    x, xd = _bf16_rows(rng, T, H)
    Wr = rng.normal(0, 0.02, (E, H)).astype(np.float32)
    y, _, _, _ = oracle.layer_forward(x, Wr, None, 2, ks, sh)
    assert np.allclose(y, dense_ffn(sh, 0, xd), rtol=1e-12, atol=1e-14)
    # every code equal to the offset q0 -> all weights are exactly zero -> y = residual
    for qtype, q0 in ((2, 2), (3, 4), (4, 8)):
        def m(rows, K):
            return KnownQMat(qtype, np.full((E, rows, K), q0), np.full((E, rows, K // 32), 0.01, np.float16))
        zs = KnownSet(m(I, H), m(I, H), m(H, I))
        res = rng.normal(size=(T, H)).astype(np.float32)
        y, _, _, _ = oracle.layer_forward(x, Wr, None, 2, zs, residual=res)
        assert np.array_equal(y, res.astype(np.float64))


def test_mtp_verify_T4_equals_four_T1():
    # a T=4 verify pass gives the per-token results of four one-token passes
    # (Strata DETAILS.md, "How it works": the drafts are checked, the output is the same)
    L = synth.make_layer(synth.LayerShape("t", 4, 256, 16, 2, 128, 2, True, 1.1))
    y4, i4, w4, _ = oracle.layer_forward(L.x, L.Wr, L.bias, 2, L.routed, L.shared)
    for t in range(4):
        y1, i1, w1, _ = oracle.layer_forward(L.x[t:t + 1], L.Wr, L.bias, 2, L.routed, L.shared)
        assert np.array_equal(y1[0], y4[t]) and np.array_equal(i1[0], i4[t]) and np.array_equal(w1[0], w4[t])


def test_forced_routing_reproduces_own_selection():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    y, idx, w, _ = oracle.layer_forward(L.x[:8], L.Wr, L.bias, 2, L.routed, L.shared)
    yf, idxf, wf, _ = oracle.layer_forward(L.x[:8], L.Wr, L.bias, 2, L.routed, L.shared, forced_idx=idx)
    assert np.array_equal(idx, idxf)
    assert np.allclose(w, wf, rtol=1e-15, atol=0)
    assert np.allclose(y, yf, rtol=1e-14, atol=0)


def test_mirrored_mode_is_close_to_exact_for_q2():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    y, _, _, _ = oracle.layer_forward(L.x[:16], L.Wr, L.bias, 2, L.routed)
    ym, _, _, _ = oracle.layer_forward(L.x[:16], L.Wr, L.bias, 2, L.routed, mirrored=True)
    assert np.abs(ym - y).max() / np.sqrt((y ** 2).mean()) < 5e-3
    assert not np.array_equal(ym, y)


# ----------------------------------------------------------------------------- RMSNorm
def test_rmsnorm_closed_forms():
    r = np.array([[3.0, 4.0], [1.0, -1.0], [0.0, 0.0]], np.float32)
    u = oracle.rmsnorm_bf16(r, 1e-6)
    inv = 1.0 / math.sqrt(12.5 + 1e-6)
    exp0 = torch.tensor([3 * inv, 4 * inv], dtype=torch.float64).to(torch.bfloat16)
    assert u[0].tolist() == exp0.view(torch.int16).numpy().view(np.uint16).tolist()
    assert u[1].tolist() == [0x3F80, 0xBF80]   # +-1/sqrt(1+1e-6) rounds to +-1.0 in bf16
    assert u[2].tolist() == [0, 0]


def test_rmsnorm_output_has_unit_rms():
    rng = np.random.default_rng(8)
    r = (rng.normal(0, 7, (4, 2048))).astype(np.float32)
    u = oracle.rmsnorm_bf16(r)
    uf = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.allclose(np.sqrt((uf ** 2).mean(1)), 1.0, atol=5e-3)
    assert (np.sign(uf) == np.sign(r)).all()


def test_stack_is_token_independent():
    s = synth.LayerShape("s", 6, 256, 16, 2, 128, 2, True, None)
    layers = []
    for l in range(3):
        layers.append((synth.make_router(0, l, 16, 256), None,
                       synth.make_expert_set(0, l, 0, 2, 16, 256, 128),
                       synth.make_expert_set(0, l, 1, 2, 1, 256, 128)))
    r0 = synth.make_residual(0, s.T, s.H)
    rT, _ = oracle.stack_forward(r0, layers, 2)
    for t in (0, 3, 5):
        r1, _ = oracle.stack_forward(r0[t:t + 1], layers, 2)
        assert np.array_equal(r1[0], rT[t])


def _bf16_rne(v: np.ndarray) -> np.ndarray:
    """Round fp64 values (normal range) to the nearest bfloat16, ties to even, exactly: an 8-bit
    significand m in [128, 256) scaled by a power of two (np.rint rounds half to even)."""
    m, e = np.frexp(v)                      # v = m 2^e, |m| in [0.5, 1)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def test_bf16_rne_helper_against_torch():
    # the test-side rounding used below agrees with torch on fp32 inputs (no double rounding there)
    rng = np.random.default_rng(41)
    v = rng.normal(0, 3, 5000).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    assert np.array_equal(_bf16_rne(v.astype(np.float64)), ref)


def test_stack_of_zero_weight_layers_is_the_identity():
    # every code equal to q0 makes every weight exactly 0: each layer adds 0 to the residual
    # stream, so the stack returns its input bit for bit (a dropped residual would return 0)
    rng = np.random.default_rng(42)
    T, H, E, I = 5, 64, 4, 32

    def zero_set(n, qtype):
        q0 = {2: 2, 3: 4}[qtype]
        m = lambda rows, K: KnownQMat(qtype, np.full((n, rows, K), q0), np.full((n, rows, K // 32), 0.01, np.float16))
        return KnownSet(m(I, H), m(I, H), m(H, I))

    layers = [(rng.normal(0, 0.02, (E, H)).astype(np.float32), None, zero_set(E, q), zero_set(1, q))
              for q in (2, 3, 2)]
    r0 = (rng.normal(0, 2, (T, H))).astype(np.float32)
    rL, _ = oracle.stack_forward(r0, layers, 2)
    assert np.array_equal(rL, r0)


def test_stack_of_one_hot_layers_matches_hand_composition():
    # r_{l+1} = r_l + FFN_{e_l}(u_l) + FFN_shared_l(u_l), u_l = bf16(r_l / sqrt(mean(r_l^2) + eps)),
    # the residual stream kept in fp32 between layers. A one-hot router (k = 1, a +100 bias on
    # expert e_l) makes the routed part the dense SwiGLU FFN of e_l with weight exactly 1.
    # Composed here from the known dense weights, numpy and an exact bf16 rounding; a large eps
    # (0.5) tells eps inside the square root from eps added to it, distinct experts per layer
    # make the layer order matter.
    rng = np.random.default_rng(43)
    T, H, E, I, eps = 4, 64, 4, 32, 0.5
    chosen = [2, 0, 3]
    layers = []
    for l, e in enumerate(chosen):
        Wr = rng.normal(0, 0.02, (E, H)).astype(np.float32)
        bias = np.zeros(E, np.float32)
        bias[e] = 100.0
        layers.append((Wr, bias, random_known_set(rng, 2 + (l % 2), E, H, I), random_known_set(rng, 2 + (l % 2), 1, H, I)))
    r0 = (rng.normal(0, 1.5, (T, H))).astype(np.float32)
    got, idxs = oracle.stack_forward(r0, layers, 1, eps=eps)
    r = r0.astype(np.float64)
    for (Wr, bias, ks, sh), e, idx in zip(layers, chosen, idxs):
        assert (idx == e).all()
        u = _bf16_rne(r / np.sqrt((r ** 2).mean(axis=1, keepdims=True) + eps))
        r = (r + dense_ffn(ks, e, u) + dense_ffn(sh, 0, u)).astype(np.float32).astype(np.float64)
    assert np.allclose(got, r, rtol=1e-9, atol=1e-12)
    assert not np.allclose(got, r0, rtol=1e-3)     # the layers did change the stream


# ----------------------------------------------------------------------------- int8 activation blocks
def test_int8_blocks_hand_worked():
    # a block whose largest magnitude is 2: d = 2/127, and 127/2 = 63.5 times each value rounds to
    # the nearest integer, ties to even (0.5 * 63.5 = 31.75 -> 32; 1/127 * 63.5 = 0.5 -> 0)
    x = np.zeros((1, 64), np.float16)
    x[0, :6] = [2.0, -2.0, 0.5, -1.0, 1.0 / 127.0, 0.25]
    q, d = oracle.quantize_blocks_i8(x)
    assert d[0, 0] == np.float32(2.0) / np.float32(127.0) and d[0, 1] == 0.0   # second block all zero
    v = np.float32(x[0, 4]) * (np.float32(127.0) / np.float32(2.0))
    assert q[0, :6].tolist() == [127, -127, 32, -64, int(np.rint(v)), 16]
    assert (q[0, 32:] == 0).all()


def test_int8_blocks_error_bound_and_extremes():
    rng = np.random.default_rng(44)
    x = (rng.normal(0, 3, (16, 256))).astype(np.float16)
    q, d = oracle.quantize_blocks_i8(x)
    xr = oracle.dequantize_blocks_i8(q, d)
    err = np.abs(xr - x.astype(np.float64)).reshape(16, 8, 32)
    assert (err <= d[..., None] * 0.5 * (1 + 1e-5)).all()    # half a step at most (fp32 scale rounding aside)
    amax_pos = np.abs(x.astype(np.float32)).reshape(16, 8, 32).argmax(-1)
    qb = np.abs(q.astype(np.int64)).reshape(16, 8, 32)
    assert (np.take_along_axis(qb, amax_pos[..., None], -1) == 127).all()  # the block maximum maps to +-127
    assert (qb <= 127).all()
