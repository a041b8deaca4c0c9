"""The seeded generator: determinism, shapes, NaN padding and needle logits."""
import math

import numpy as np
import torch

import oracle
from long_context_token_b200 import workloads


def test_generator_is_deterministic_and_pads_with_nan():
    a = workloads.make_inputs(2, 500, n_q=1, h_q=16, kv="fp8", seed=4, lens=[500, 321], n_sparse=2)
    b = workloads.make_inputs(2, 500, n_q=1, h_q=16, kv="fp8", seed=4, lens=[500, 321], n_sparse=2)
    assert torch.equal(a.k, b.k) and torch.equal(a.v_scale[0], b.v_scale[0]) and torch.equal(a.q, b.q)
    assert torch.all(a.k[1, 321:] == 0x7F) and torch.isnan(a.k_scale[1, 321:]).all()
    assert not torch.isnan(a.k_scale[1, :321]).any()
    c = workloads.make_inputs(1, 300, n_q=1, h_q=16, seed=4, lens=[200])
    assert torch.isnan(c.k[0, 200:].float()).all() and not torch.isnan(c.k[0, :200].float()).any()


def test_needles_carry_the_planted_logit():
    w = workloads.WORKLOADS[1]
    inp = workloads.generate(w)
    bits = workloads.numpy_bits(inp)
    q = oracle.bf16_to_f64(bits["q"][0, 0])
    for pos, h in inp.needles[0]:
        k = oracle.bf16_to_f64(bits["k"][0, pos])
        s = bits["sm_scale"] * q[h] @ k
        assert abs(s - w.needle_delta) < 0.05


def test_ragged_lengths_are_in_range():
    w = workloads.WORKLOADS[3]
    g = torch.Generator().manual_seed(w.seed * 1000 + 500)
    lens = torch.randint(w.len_lo, w.max_len + 1, (w.batch,), generator=g)
    assert torch.all(lens >= 204800) and torch.all(lens <= 262144)


def test_sm_scale_is_float32_exact():
    s = workloads.default_sm_scale()
    assert np.float32(s) == s and abs(s - 1 / math.sqrt(128)) < 1e-8
