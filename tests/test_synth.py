"""The seeded input generator: its words equal a scalar big-int restatement of splitmix64, and the
derived draws have the stated ranges and distributions."""
import numpy as np
import torch

import synth


def test_words_match_bigint_reference():
    for seed, t in ((0, 1), (7, synth.tid(synth.K_CODES, 3, 2, 511)), (2 ** 40 + 3, 0)):
        w = synth.words(seed, t, 9, start=5)
        ref = [synth.word_int(seed, t, 5 + i) for i in range(9)]
        assert [int(v) & ((1 << 64) - 1) for v in w] == ref


def test_splitmix64_known_value():
    # splitmix64 with state 0: first output of the standard sequence (x += GAMMA; mix(x))
    assert synth.mix_int(synth.GAMMA) == 0xE220A8397B1DCDAF


def test_scales_range_and_determinism():
    s = synth.scales_f16(0, [1, 2], 5000)
    assert s.dtype == torch.float16 and s.shape == (2, 5000)
    assert float(s.min()) >= 0.005 - 1e-6 and float(s.max()) <= 0.02 + 1e-5
    assert torch.equal(s, synth.scales_f16(0, [1, 2], 5000))
    assert not torch.equal(s[0], s[1])


def test_expert_subset_regenerates_identically():
    full = synth.make_qmat(0, 2, 0, 1, 3, 6, 32, 64)
    part = synth.make_qmat(0, 2, 0, 1, 3, 6, 32, 64, experts=[4])
    assert torch.equal(full.codes[4], part.codes[0])
    assert torch.equal(full.hibits[4], part.hibits[0])
    assert torch.equal(full.scales[4], part.scales[0])


def test_normals_moments():
    z = synth.normal_f64(0, 99, 200000)
    assert abs(float(z.mean())) < 0.01 and abs(float(z.std()) - 1.0) < 0.01


def test_zipf_bias_is_minus_s_log_rank():
    b = synth.zipf_bias(0, 0, 512, 1.1).double()
    ranks = torch.exp(-b / 1.1)
    assert torch.allclose(torch.sort(ranks).values, torch.arange(1, 513, dtype=torch.float64), atol=1e-3)


def test_workload_shapes():
    L = synth.make_layer(synth.WORKLOADS["tiny"])
    assert L.x.shape == (64, 256) and L.x.dtype == torch.bfloat16
    assert L.Wr.shape == (16, 256) and L.Wr.dtype == torch.float32
    assert L.routed.gate.codes.shape == (16, 128, 64)
    assert L.routed.down.codes.shape == (16, 256, 32)
    assert L.shared is None and L.bias is None


def test_workload_table_matches_the_stated_configs():
    # the shapes the tests and the benchmark use: the decode, verify, pruned, prefill, skewed Q3 and
    # stack workloads (H=2048, E=512, top-10, I=512 unless stated otherwise)
    W = synth.WORKLOADS
    for name in ("decode1", "decode4", "verify6", "decode1_pruned256"):
        s = W[name]
        assert (s.H, s.k, s.I, s.qtype, s.shared, s.zipf_s) == (2048, 10, 512, synth.Q2, True, 1.1)
    assert [W[n].T for n in ("decode1", "decode4", "verify6", "decode1_pruned256")] == [1, 4, 6, 1]
    assert W["decode1"].E == W["decode4"].E == W["verify6"].E == 512 and W["decode1_pruned256"].E == 256
    p = W["prefill8k"]
    assert (p.T, p.H, p.E, p.k, p.I, p.qtype, p.shared, p.zipf_s) == (8192, 2048, 512, 10, 512, synth.Q2, True, None)
    q = W["prefill2k_q3"]
    assert (q.T, q.E, q.k, q.qtype, q.shared, q.zipf_s) == (2048, 512, 10, synth.Q3, False, 1.2)
    q4 = W["decode1_q4"]
    assert (q4.T, q4.H, q4.E, q4.k, q4.I, q4.qtype, q4.shared, q4.zipf_s) == (1, 2048, 512, 10, 512, synth.Q4, True, 1.1)
    assert synth.STACK["L"] == 48 and synth.STACK["eps"] == 1e-6
